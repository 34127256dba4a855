"""Failure detection on the GPU without faulting it: every wait in the
kernels is bounded; the self-test kernel waits on a barrier phase that
nothing completes, with a short limit, through the same bounded wait. The
host then reads VDN_ERR_DEVICE_TIMEOUT from the device error word, the word
is cleared by the read, and the context keeps working (a layer call right
after still matches the oracle)."""
import numpy as np
import pytest

import oracle as O
import vdn_synth as S
from vdn_cases import OUT_MAX_ABS, OUT_REL_L2, max_abs, rel_l2, run_layer

pytestmark = pytest.mark.gpu

VDN_OK = 0
VDN_ERR_DEVICE_TIMEOUT = -6


@pytest.mark.parametrize("tmem_cols", [0, 512])
def test_bounded_wait_times_out_and_reports(tmem_cols):
    import video_diffusion_hybrid_block_b200 as V
    assert V.vdn_get_device_error() == VDN_OK  # nothing pending
    V.vdn_selftest_wait_timeout(2_000_000, tmem_cols)  # 2 ms
    assert V.vdn_get_device_error() == VDN_ERR_DEVICE_TIMEOUT
    assert V.vdn_get_device_error() == VDN_OK  # cleared by the read


def test_context_usable_after_timeout():
    import video_diffusion_hybrid_block_b200 as V
    V.vdn_selftest_wait_timeout(1_000_000, 512)
    assert V.vdn_get_device_error() == VDN_ERR_DEVICE_TIMEOUT
    # the TMEM the self-test held was freed: a full layer (which allocates all
    # 512 columns per CTA) runs and matches the oracle
    inp = S.make_inputs("tiny-scan")
    out = run_layer(inp).float().cpu().numpy()
    for h in range(inp["H"]):
        ref = O.layer_head(inp, h)["out"]
        assert rel_l2(out[:, h], ref) <= OUT_REL_L2
        assert max_abs(out[:, h], ref) <= OUT_MAX_ABS
    assert V.vdn_get_device_error() == VDN_OK
