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
    inp = dict(N=int(off[-1]), T=T, H=3, d=32, F=len(sizes), off=off, block_frames=bf)
    fl = bench.layer_flops(inp, soft)
    assert fl["softmax"] == 4.0 * 32 * 3 * brute_softmax_pairs(off, bf, T)
    assert fl["total"] == fl["softmax"] + fl["readout"] + fl["vda"]


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


@pytest.mark.parametrize("F,bf", [(2, 5), (10, 5), (11, 5), (15, 5), (20, 5), (30, 5), (60, 5),
                                  (9, 1), (30, 7), (14, 3)])
def test_needed_frames_are_the_linear_frames_of_some_block(F, bf):
    # the frames whose Grams/inverses the library computes are exactly the
    # frames some block folds into its read state (oracle's linear key frames)
    nf = bench.needed_frames(F, bf)
    want = sorted(set().union(*[O.linear_key_frames(b, F, bf) for b in range(O.num_blocks(F, bf))]))
    assert nf["frames"] == want
    i_f = [O.read_indices(b, F, bf)[0] for b in range(O.num_blocks(F, bf))]
    i_b = [O.read_indices(b, F, bf)[1] for b in range(O.num_blocks(F, bf))]
    assert nf["steps_fwd"] == 1 + max(i_f)
    assert nf["steps_bwd"] == 1 + (F - 1 - min(i_b))


def test_pages_scale_vda_counts_and_kernel_bytes():
    # pages-scale: 8 of 13 scanned frames are needed (1..4 and 10..13), 5 scan
    # steps per direction; the Gram kernel reads 136.3 MB of k, v and writes
    # 37.7 MB of C and W
    inp = S.make_inputs("pages-scale")
    soft, _ = O.pair_counts(inp["off"], 5, inp["T"])
    fl = bench.layer_flops(inp, soft)
    assert fl["n_mat"] == 9 and fl["scan_steps"] == 10
    assert fl["gram_rows"] == 256 + 8 * 1008
    assert fl["grams"] == 4.0 * (256 + 8 * 1008) * 128 ** 2 * 32
    kb = bench.kernel_bytes(inp, fl)
    assert kb["gram_inv"] == 2 * 8320 * 32 * 128 * 2 + 2 * 9 * 32 * 65536
    assert kb["gate_merge"] == 3 * 15120 * 32 * 128 * 2 + 2 * 15120 * 32 * 2 + 3 * 32 * 65536
    assert fl["total"] == fl["softmax"] + fl["readout"] + fl["vda"]


def test_reference_step_flops_brute_force():
    # one head's VDA work + 4 d |J(i)| per sampled row + 2 d^2 per row
    sizes = [7, 3, 0, 5, 9, 2, 4, 6, 1, 8, 3, 5]
    off = S.frame_offsets(sizes)
    T, d, H = 4, 32, 3
    soft, _ = O.pair_counts(off, 5, T)
    inp = dict(N=int(off[-1]), T=T, H=H, d=d, F=len(sizes), off=off, block_frames=5)
    fl = bench.layer_flops(inp, soft)
    rows = np.array([0, 6, 7, 20, 30, 52])
    frame = np.repeat(np.arange(len(sizes)), sizes)
    keys = 0
    for i in rows:
        allowed = set(O.softmax_key_frames(O.block_of(int(frame[i])), len(sizes)))
        keys += int(np.isin(frame, list(allowed)).sum()) + T
    want = fl["vda"] / H + 4.0 * d * keys + 2.0 * d * d * len(rows)
    assert bench.reference_step_flops(inp, soft, fl, rows) == pytest.approx(want, rel=1e-12)


def test_config_is_shared_by_both_arms():
    inp = S.make_inputs("tiny")
    soft, _ = O.pair_counts(inp["off"], 5, inp["T"])
    fl = bench.layer_flops(inp, soft)
    a = bench.config_of("tiny", inp, fl, 1)
    assert set(a) >= {"workload", "F", "N", "T", "H", "d", "parallelism", "l2"}
    assert "fit in the 126 MB L2" in a["l2"]


def test_clock_summary_drops_idle_samples_and_maps_reasons():
    """Idle samples stay out of the median; every slowdown bit seen in a busy
    sample is named (hardware power brake counts as hw_slowdown)."""
    C = bench.ClockSampler
    s = [(345.0, 1965.0, C.IDLE), (1965.0, 1965.0, 0x4), (1950.0, 1965.0, 0x4),
         (1800.0, 1965.0, 0x80), (300.0, 1965.0, C.IDLE | 0x20)]
    r = bench.summarize_clock_samples(s, C.IDLE, C.REASONS, "test")
    assert r["sm_mhz"] == 1950.0 and r["sm_max_mhz"] == 1965.0
    assert r["sm_mhz_min"] == 1800.0 and r["sm_mhz_mean"] == 1905.0
    assert r["samples"] == 3 and r["idle_samples"] == 2
    assert r["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert bench.summarize_clock_samples([], C.IDLE, C.REASONS, "test")["reasons"] == ["no samples"]
    # all samples idle: the median falls back to all of them
    r = bench.summarize_clock_samples(s[:1], C.IDLE, C.REASONS, "test")
    assert r["sm_mhz"] == 345.0
