"""The softmax kernel's numerical method, emulated in float32 on the CPU and
checked against the fp64 oracle: online softmax in the exp2 domain over
128-key tiles in the kernel's visiting order (text, then the merged frame
ranges), a running max raised only when a tile's max exceeds it by more than
8 (O and the row sum rescaled then), exp2 from the polynomial for one column
pair in four and from exp2 otherwise, P rounded to bf16 before the PV
product, fp32 row sums of the unrounded P, out = O / l. Run on the case whose
row maxima jump by far more than 8 between tiles and on a case with a wide
score range, it must stay inside the layer tolerance (rel-L2 2e-2, max-abs
5e-2), which pins the choice of threshold and rounding, not the kernel code.
The same holds for the split form a single-tile CTA of the softmax-only
kernel uses (two partial passes over alternate key tiles, joined with
weights 2^(m_i - m)); adding the partial results unweighted does not."""
import numpy as np
import pytest

import oracle as O
import vdn_synth as S
from test_exp2_poly import exp2_poly_f32


def bf16(x):
    return S.bf16_round(np.asarray(x, np.float32))


def key_segments(off, b, F, bf, T):
    """Key row ranges of block b in the kernel's order: the text, then the
    frame ranges {0}, window, {F-1}, merged where they touch; every segment
    starts a new 128-key tile."""
    w0, w1 = O.window(b, F, bf)
    ranges = [(0, 0), (w0, w1), (F - 1, F - 1)]
    merged = [list(ranges[0])]
    for a, e in ranges[1:]:
        if a <= merged[-1][1] + 1:
            merged[-1][1] = max(merged[-1][1], e)
        else:
            merged.append([a, e])
    segs = [("t", 0, T)] + [("v", int(off[a]), int(off[e + 1])) for a, e in merged]
    return [sg for sg in segs if sg[2] > sg[1]]


def online_pass(Q, K, Vv, tiles, scale, threshold):
    """One warpgroup's pass over its key tiles: running max in use, row sums
    of the unrounded P, O from bf16 P (all float32); m is None if no tile."""
    d = Vv.shape[1]
    m_use = None
    l = np.zeros(Q.shape[0], np.float32)
    Oacc = np.zeros((Q.shape[0], d), np.float32)
    for a, e in tiles:
        s = (Q @ K[a:e].T).astype(np.float32)
        m_tile = (s.max(axis=1) * scale).astype(np.float32)
        if m_use is None:
            m_use = m_tile
        else:
            need = m_tile > m_use + np.float32(threshold)
            factor = np.where(need, np.exp2(np.minimum(m_use - m_tile, 0)), np.float32(1)).astype(np.float32)
            m_use = np.where(need, m_tile, m_use)
            l *= factor
            Oacc *= factor[:, None]
        x = (s * scale - m_use[:, None]).astype(np.float32)
        p = np.exp2(x).astype(np.float32)
        cols = np.arange(e - a)
        poly = ((cols // 2) % 4) == 3          # one column pair in four
        p[:, poly] = exp2_poly_f32(x[:, poly])
        l += p.sum(axis=1, dtype=np.float32)
        Oacc += (bf16(p) @ Vv[a:e]).astype(np.float32)
    return m_use, l, Oacc


def combine_split(part0, part1, rescale=True):
    """Two partial softmaxes of the same rows (warpgroup 0: key tiles 0, 2,
    ...; warpgroup 1: 1, 3, ...) joined as the kernel's split CTA does:
    m = max(m_0, m_1), weights 2^(m_i - m), warpgroup 1 ignored when it had no
    tile (l_1 = 0)."""
    m0, l0, O0 = part0
    m1, l1, O1 = part1
    if m1 is None:
        return O0 / l0[:, None]
    if rescale:
        m = np.maximum(m0, m1)
        a0 = np.exp2(m0 - m).astype(np.float32)
        a1 = np.where(l1 > 0, np.exp2(m1 - m), 0).astype(np.float32)
    else:  # negative control: partial sums added as they are
        a0 = a1 = np.ones_like(l0)
    return (O0 * a0[:, None] + O1 * a1[:, None]) / (l0 * a0 + l1 * a1)[:, None]


def emulate_head(inp, h, threshold=8.0, split=False, rescale=True):
    """The kernel's softmax for head h; with `split`, every row as a
    single-tile CTA computes it (alternate key tiles, then combined)."""
    off, F, bf, T = inp["off"], inp["F"], inp["block_frames"], inp["T"]
    d = inp["d"]
    scale = np.float32(np.log2(np.e) / np.sqrt(d))
    out = np.zeros((inp["N"], d), np.float64)
    for b in range(O.num_blocks(F, bf)):
        q0, q1 = int(off[bf * b]), int(off[min(bf * b + bf, F)])
        if q1 == q0:
            continue
        Ks, Vs, tiles, base = [], [], [], 0
        for src, a, e in key_segments(off, b, F, bf, T):
            Ks.append((inp["kt"] if src == "t" else inp["k"])[a:e, h])
            Vs.append((inp["vt"] if src == "t" else inp["v"])[a:e, h])
            tiles += [(base + i, base + min(i + 128, e - a)) for i in range(0, e - a, 128)]
            base += e - a
        K = np.concatenate(Ks).astype(np.float32)
        Vv = np.concatenate(Vs).astype(np.float32)
        Q = inp["q"][q0:q1, h].astype(np.float32)
        if split:
            out[q0:q1] = combine_split(online_pass(Q, K, Vv, tiles[0::2], scale, threshold),
                                       online_pass(Q, K, Vv, tiles[1::2], scale, threshold),
                                       rescale)
        else:
            _, l, Oacc = online_pass(Q, K, Vv, tiles, scale, threshold)
            out[q0:q1] = Oacc / l[:, None]
    return out


def _max_jump():
    inp = S.make_inputs_from(12, [150] * 12, 40, 2, 128, "bf16", seed=8)
    k = inp["k"].copy()
    for f in range(12):
        k[inp["off"][f]:inp["off"][f + 1]] *= 2.0 ** (f // 2)
    inp["k"] = k
    return inp


def _wide_scores():
    # scores spread over hundreds of log2 units: exp2 without a rescale of
    # the running max overflows fp32
    inp = S.make_inputs_from(10, [90] * 10, 16, 1, 64, "bf16", seed=21)
    inp["q"] = S.bf16_round(inp["q"] * 400.0)
    return inp


@pytest.mark.parametrize("make", [_max_jump, _wide_scores], ids=["max-jump", "wide-scores"])
def test_kernel_softmax_method_within_tolerance(make):
    inp = make()
    for h in range(inp["H"]):
        got = emulate_head(inp, h)
        ref = O.softmax_branch_head(inp["q"], inp["k"], inp["v"], inp["kt"], inp["vt"],
                                    inp["off"], h, inp["block_frames"])
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert rel <= 2e-2 and np.abs(got - ref).max() <= 5e-2, (h, rel)


def test_without_the_rescale_the_method_breaks():
    # negative control: never raising the running max overflows on wide scores
    inp = _wide_scores()
    with np.errstate(over="ignore", invalid="ignore"):
        got = emulate_head(inp, 0, threshold=1e30)
    assert not np.all(np.isfinite(got))


@pytest.mark.parametrize("make", [_max_jump, _wide_scores], ids=["max-jump", "wide-scores"])
def test_split_key_tiles_within_tolerance(make):
    # a CTA with a single query tile: its two warpgroups take alternate key
    # tiles of the same rows, each with its own running max, and the partial
    # results are joined with weights 2^(m_i - m)
    inp = make()
    for h in range(inp["H"]):
        got = emulate_head(inp, h, split=True)
        ref = O.softmax_branch_head(inp["q"], inp["k"], inp["v"], inp["kt"], inp["vt"],
                                    inp["off"], h, inp["block_frames"])
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert rel <= 2e-2 and np.abs(got - ref).max() <= 5e-2, (h, rel)


def test_split_with_one_key_tile_uses_warpgroup_0_alone():
    # one key tile per block: the second warpgroup has nothing, its l is 0
    inp = S.make_inputs_from(2, [40, 30], 0, 1, 32, "bf16", seed=5)
    ref = O.softmax_branch_head(inp["q"], inp["k"], inp["v"], inp["kt"], inp["vt"],
                                inp["off"], 0, inp["block_frames"])
    got = emulate_head(inp, 0, split=True)
    assert np.all(np.isfinite(got))
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 2e-2


def test_split_without_the_max_weights_breaks():
    # negative control: adding the partial results without 2^(m_i - m) is
    # wrong as soon as the two running maxima differ
    inp = _max_jump()
    ref = O.softmax_branch_head(inp["q"], inp["k"], inp["v"], inp["kt"], inp["vt"],
                                inp["off"], 0, inp["block_frames"])
    got = emulate_head(inp, 0, split=True, rescale=False)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) > 0.1
