"""The FLOP convention bench.py reports TFLOP/s with, checked against a
brute-force count of the (query, key) pairs the method attends on small
layouts, and the published pages-scale figures."""
import os
import sys

import numpy as np
import pytest

import oracle as O
import vdn_synth as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def brute_softmax_pairs(off, bf, T):
    """Count (video query, key) pairs token by token with the dense mask rule."""
    off = np.asarray(off, np.int64)
    F = len(off) - 1
    frame = np.repeat(np.arange(F), np.diff(off))
    n = 0
    for i in range(len(frame)):
        allowed = set(O.softmax_key_frames(O.block_of(int(frame[i]), bf), F, bf))
        n += int(np.isin(frame, list(allowed)).sum()) + T
    return n


@pytest.mark.parametrize("sizes,bf,T", [([7, 3, 0, 5, 9, 2, 4, 6, 1, 8, 3, 5], 5, 4),
                                        ([4] * 17, 3, 0), ([6, 2], 5, 3)])
def test_softmax_flop_count_matches_brute_force(sizes, bf, T):
    off = S.frame_offsets(sizes)
    soft, _ = O.pair_counts(off, bf, T)
    inp = dict(N=int(off[-1]), T=T, H=3, d=32, F=len(sizes))
    fl = bench.layer_flops(inp, soft)
    assert fl["softmax"] == 4.0 * 32 * 3 * brute_softmax_pairs(off, bf, T)
    assert fl["total"] == fl["softmax"] + fl["vda"]


def test_pages_scale_softmax_flop():
    # 3.143 TFLOP of softmax work at pages-scale (82.2 % of the video pairs)
    inp = S.make_inputs("pages-scale")
    soft, _ = O.pair_counts(inp["off"], 5, inp["T"])
    fl = bench.layer_flops(inp, soft)
    assert abs(fl["softmax"] / 1e12 - 3.1431) < 5e-4
    video = soft[:, :-1].sum() / inp["N"] ** 2
    assert abs(video - 0.8222) < 5e-4


def test_workload_descriptions_and_l2_notes():
    for name in S.CONFIGS:
        assert name.split("-")[0] in bench.workload_desc(name)
    assert "> 126 MB L2" in bench.l2_note(400 * 2 ** 20)
    assert "fit in the 126 MB L2" in bench.l2_note(2 ** 20)


def test_vda_merge_roofline_bytes():
    # 625.7 MB at pages-scale: k, v, q, o_soft, out 124 MB each, kt, vt, gates
    inp = S.make_inputs("pages-scale")
    r = bench.vda_merge_roofline(inp, 2.766, 2.640, 6543.0)
    assert r["algorithmic_bytes"] == 5 * 15120 * 32 * 128 * 2 + 2 * 256 * 32 * 128 * 2 + 2 * 15120 * 32 * 2
    assert abs(r["roofline_ms"] - r["algorithmic_bytes"] / 6543e9 * 1e3) < 1e-4
    assert abs(r["marginal_ms"] - 0.126) < 1e-9 and abs(r["frac"] - r["roofline_ms"] / 0.126) < 1e-3
