"""The layer at the boundary's index limit: N * H * 128 just below 2^31
(every [N, H, 128] tensor holds 2^31 - 2^19 elements, 4.3 GB in bf16).
Inputs are drawn on the device (vdn_synth.make_inputs_device); three heads
(first, middle, last) are checked against the fp64 oracle on sampled rows
and all their read states, which exercises every 64-bit offset the kernels
form from (row, head) near the top of the index range."""
import numpy as np
import pytest
import torch

import oracle as O
import vdn_synth as S
from vdn_cases import OUT_MAX_ABS, OUT_REL_L2, STATE_REL_FRO, max_abs, rel_l2

pytestmark = pytest.mark.gpu


def _head_inputs(dev, inp, h):
    """One head of the device inputs as the oracle's numpy arrays (H = 1)."""
    one = {k: dev[k][:, h:h + 1].float().cpu().numpy() for k in ("q", "k", "v", "kt", "vt")}
    one.update({k: dev[k][:, h:h + 1].float().cpu().numpy() for k in ("g_s", "g_l")})
    one["rms_w"] = dev["rms_w"][h:h + 1].cpu().numpy()
    one.update(off=inp["off"], F=inp["F"], T=inp["T"], H=1, d=inp["d"], N=inp["N"],
               dtype="bf16", block_frames=inp["block_frames"], lam=inp["lam"], eps=inp["eps"])
    return one


def test_layer_at_the_index_limit():
    import video_diffusion_hybrid_block_b200 as V
    F, n, T, H, d = 16, 256, 64, 4095, 128          # N * H * 128 = 2^31 - 2^19
    assert F * n * H * d < 2 ** 31 <= F * n * (H + 1) * d
    dev = S.make_inputs_device(F, [n] * F, T, H, d, seed=17)
    inp = {k: dev[k] for k in ("off", "F", "T", "H", "d", "N", "block_frames", "lam", "eps")}
    shape = V.Shape(inp["off"], T, H, d, inp["block_frames"], inp["lam"], inp["eps"], V.VDN_BF16)
    ws = V.alloc_workspace(shape)
    out = torch.empty_like(dev["q"])
    V.vdn_hybrid_attn_fwd(shape, dev["q"], dev["k"], dev["v"], dev["kt"], dev["vt"], dev["g_s"],
                          dev["g_l"], dev["rms_w"], out, ws)
    nb = O.num_blocks(F, inp["block_frames"])
    R = torch.empty((nb, H, d, d), dtype=torch.float32, device="cuda")
    V.vdn_vda_scan(shape, dev["k"], dev["v"], dev["kt"], dev["vt"], R, None, None, None, ws)
    torch.cuda.synchronize()
    assert V.vdn_get_device_error() == 0
    rows = np.unique(np.concatenate([np.random.default_rng(0).choice(inp["N"], 40, replace=False),
                                     [0, 127, 128, inp["N"] - 1]]))
    for h in (0, H // 2, H - 1):
        one = _head_inputs(dev, inp, h)
        res = O.layer_head(one, 0, rows=rows)
        got = out[torch.from_numpy(rows).cuda(), h].float().cpu().numpy()
        assert rel_l2(got, res["out"]) <= OUT_REL_L2, h
        assert max_abs(got, res["out"]) <= OUT_MAX_ABS, h
        Rh = R[:, h].cpu().numpy()
        for b in range(nb):
            assert rel_l2(Rh[b], res["states"]["R"][b]) <= STATE_REL_FRO, (h, b)
