"""Full-size parity on every head: the layer output on a fixed set of query
rows, the read states R_b and the text state of all H heads, and (all
workloads, long-clip included) every per-frame forward / backward state,
against the fp64 oracle. The rows include every block's first and last row,
the 128-row tile edges q0+127 / q0+128 and the 256-row CTA edges q0+255 /
q0+256, plus random rows. Worst margins are printed in the session summary.

Tolerances: layer output rel-L2 <= 2e-2 and max-abs <= 5e-2 per head; each
VDA state rel-Frobenius <= 1e-2."""
import numpy as np
import pytest
import torch

import oracle as O
import vdn_synth as S
from conftest import MARGINS
from vdn_cases import (OUT_MAX_ABS, OUT_REL_L2, STATE_REL_FRO, device_inputs, max_abs, rel_l2,
                       run_layer, run_scan)

pytestmark = pytest.mark.gpu

FULL = ["pages-scale", "long-clip", "hi-res", "vda-stress"]


def edge_rows(inp: dict, n_random: int = 12, seed: int = 1) -> np.ndarray:
    N, off, bf, F = inp["N"], inp["off"], inp["block_frames"], inp["F"]
    rows = set(np.random.default_rng(seed).choice(N, size=min(n_random, N), replace=False).tolist())
    for b in range(O.num_blocks(F, bf)):
        q0, q1 = int(off[bf * b]), int(off[min(bf * b + bf, F)])
        for r in (q0, q1 - 1, q0 + 127, q0 + 128, q0 + 255, q0 + 256):
            if q0 <= r < q1:
                rows.add(r)
    return np.array(sorted(rows))


@pytest.mark.parametrize("name", FULL)
def test_layer_every_head_full_size(name):
    inp = S.make_inputs(name)
    dev = device_inputs(inp)
    out = run_layer(inp, dev)
    R, St, Sf, Sb = run_scan(inp, dev, per_frame=True)
    rows = edge_rows(inp)
    got = out[torch.from_numpy(rows).cuda()].float().cpu().numpy()     # [rows, H, d]
    R, St, Sf, Sb = (x.cpu().numpy() for x in (R, St, Sf, Sb))
    F = inp["F"]
    worst = dict(out=(0.0, 0.0, -1), R=(0.0, 0.0, -1), text=(0.0, 0.0, -1), frames=(0.0, 0.0, -1))

    def note(key, a, b, h):
        r, m = rel_l2(a, b), max_abs(a, b)
        if r > worst[key][0]:
            worst[key] = (r, max(m, worst[key][1]), h)
        else:
            worst[key] = (worst[key][0], max(m, worst[key][1]), worst[key][2])
        return r, m

    for h in range(inp["H"]):
        res = O.layer_head(inp, h, rows=rows)
        r, m = note("out", got[:, h], res["out"], h)
        assert r <= OUT_REL_L2 and m <= OUT_MAX_ABS, (name, h, r, m)
        st = res["states"]
        r, _ = note("text", St[h], st["S_text"], h)
        assert r <= STATE_REL_FRO, (name, "S_text", h, r)
        for b in range(R.shape[0]):
            r, _ = note("R", R[b, h], st["R"][b], h)
            assert r <= STATE_REL_FRO, (name, "R", b, h, r)
        for i in range(F - 1):
            r, _ = note("frames", Sf[i, h], st["fwd"][i], h)
            assert r <= STATE_REL_FRO, (name, "fwd", i, h, r)
        for j in range(1, F):
            r, _ = note("frames", Sb[j, h], st["bwd"][j], h)
            assert r <= STATE_REL_FRO, (name, "bwd", j, h, r)
    MARGINS.append((f"{name} ({len(rows)} rows)", "out", *worst["out"], "2e-2 / 5e-2"))
    for key, what in (("R", "read states R_b"), ("text", "S_text"),
                      ("frames", "per-frame fwd/bwd")):
        MARGINS.append((name, what, *worst[key], "1e-2"))
