"""The workspace-free linear-branch entry point (vdn_vda_scan_noalloc) gives
the same states as vdn_vda_scan with a caller-provided workspace.

It exists for callers that cannot allocate device memory at call time
(serving loops that cannot absorb the device-wide synchronisation of
cudaMalloc / cudaFree, plug-ins that do not own their process's allocator);
it uses a fixed device array inside the library instead. The array is shared
and keeps the previous call's contents, so two calls in a row are checked, on
two layouts of different size, and a read-states-only call (which writes
only part of the array) right after a larger call of another shape is
checked against the workspace path and the oracle. Collected last (file
name) so a failure here cannot hide any other test."""
import numpy as np
import pytest
import torch

import oracle as O
import vdn_synth as S
from vdn_cases import STATE_REL_FRO, device_inputs, make_shape, mid_case, rel_l2, run_scan

pytestmark = pytest.mark.gpu


def _noalloc(inp, dev, per_frame=True):
    import video_diffusion_hybrid_block_b200 as V
    shape = make_shape(inp)
    F, H, d = inp["F"], inp["H"], inp["d"]
    nb = -(-F // inp["block_frames"])
    R = torch.full((nb, H, d, d), float("nan"), device="cuda")
    St = torch.full((H, d, d), float("nan"), device="cuda") if per_frame else None
    Sf = torch.zeros((F, H, d, d), device="cuda") if per_frame else None
    Sb = torch.zeros((F, H, d, d), device="cuda") if per_frame else None
    V.vdn_vda_scan_noalloc(shape, dev["k"], dev["v"], dev["kt"], dev["vt"], R, St, Sf, Sb)
    torch.cuda.synchronize()
    assert V.vdn_get_device_error() == 0
    return R, St, Sf, Sb


@pytest.mark.parametrize("make", [lambda: mid_case(seed=21), lambda: S.make_inputs("tiny-scan")])
def test_noalloc_scan_matches_workspace_scan_twice(make):
    inp = make()
    dev = device_inputs(inp)
    ref = [x.cpu().numpy() for x in run_scan(inp, dev)]
    for _ in range(2):
        got = [x.cpu().numpy() for x in _noalloc(inp, dev)]
        R, St, Sf, Sb = got
        rR, rSt, rSf, rSb = ref
        for b in range(R.shape[0]):
            for h in range(R.shape[1]):
                assert rel_l2(R[b, h], rR[b, h]) <= STATE_REL_FRO
        for h in range(St.shape[0]):
            assert rel_l2(St[h], rSt[h]) <= STATE_REL_FRO
        F = inp["F"]
        for i in range(F - 1):
            assert rel_l2(Sf[i], rSf[i]) <= STATE_REL_FRO
        for j in range(1, F):
            assert rel_l2(Sb[j], rSb[j]) <= STATE_REL_FRO


def test_noalloc_read_states_only_after_a_larger_call():
    # The default path (read states only) trims the frames no read state
    # depends on and writes only part of the scratch. Run it right after a
    # larger per-frame call of another shape, whose leftovers fill the rest,
    # and hold it to the workspace path and to the oracle.
    big = S.make_inputs_from(24, [90] * 24, 20, 3, 128, "bf16", seed=22)
    _noalloc(big, device_inputs(big), per_frame=True)
    inp = S.make_inputs_from(21, [70, 3, 0, 55, 81, 9, 64, 2, 77, 40, 1, 66, 0, 35, 90, 12, 48,
                                  7, 60, 5, 33], 9, 2, 128, "bf16", seed=23)
    dev = device_inputs(inp)
    ref = run_scan(inp, dev, per_frame=False)[0].cpu().numpy()
    for _ in range(2):
        R = _noalloc(inp, dev, per_frame=False)[0].cpu().numpy()
        for h in range(inp["H"]):
            st = O.vda_states_head(inp["k"], inp["v"], inp["kt"], inp["vt"], inp["off"], h,
                                   inp["lam"], inp["block_frames"])
            for b in range(R.shape[0]):
                assert np.isfinite(R[b, h]).all()
                assert rel_l2(R[b, h], ref[b, h]) <= STATE_REL_FRO, (b, h)
                assert rel_l2(R[b, h], st["R"][b]) <= STATE_REL_FRO, (b, h)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import video_diffusion_hybrid_block_b200 as V
    from video_diffusion_hybrid_block_b200 import binding as B
    # 32 heads x (59 frames + 12 blocks) x 128 KiB > 64 MiB
    inp = S.make_inputs_from(60, [8] * 60, 4, 32, 128, "bf16", seed=0)
    dev = device_inputs(inp)
    shape = make_shape(inp)
    R = torch.empty((12, 32, 128, 128), device="cuda")
    with pytest.raises(B.VdnError) as e:
        V.vdn_vda_scan_noalloc(shape, dev["k"], dev["v"], dev["kt"], dev["vt"], R, None, None,
                               None)
    assert e.value.code == B.VDN_ERR_WORKSPACE_TOO_SMALL
