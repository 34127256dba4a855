"""Pins of the CPU oracle against facts that do not come from the oracle itself:
a second formulation (dense masked attention), closed forms (Sherman-Morrison,
ridge least squares, orthonormal-key delta steps, fixed points, RMSNorm),
invariants (non-expansiveness, pair-set coverage), library routines
(torch scaled_dot_product_attention in float64) and hand-derived integer
counts (tests/golden/pair_split.json)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle as O
import vdn_synth as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small_inputs(F, n=6, T=4, H=2, d=8, seed=0, sizes=None, rms_w=None):
    sizes = sizes if sizes is not None else [n] * F
    return S.make_inputs_from(F, sizes, T, H, d, dtype="f32", seed=seed,
                              rms_w=rms_w)


# ----------------------------------------------------------------- softmax --

@pytest.mark.parametrize("name", ["tiny", "tiny-scan"])
def test_block_sparse_equals_dense_mask(name):
    inp = S.make_inputs(name)
    for h in range(inp["H"]):
        a = O.softmax_branch_head(inp["q"], inp["k"], inp["v"], inp["kt"],
                                  inp["vt"], inp["off"], h)
        b = O.softmax_branch_dense_mask(inp["q"], inp["k"], inp["v"], inp["kt"],
                                        inp["vt"], inp["off"], h)
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_block_sparse_equals_dense_mask_ragged():
    # F not a multiple of 5, frames of different sizes (including 1 token)
    sizes = [3, 1, 7, 2, 5, 4, 6, 1, 2, 9, 3]
    inp = small_inputs(len(sizes), sizes=sizes, seed=3)
    for h in range(inp["H"]):
        a = O.softmax_branch_head(inp["q"], inp["k"], inp["v"], inp["kt"],
                                  inp["vt"], inp["off"], h)
        b = O.softmax_branch_dense_mask(inp["q"], inp["k"], inp["v"], inp["kt"],
                                        inp["vt"], inp["off"], h)
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_all_frames_visible_is_plain_attention():
    # F <= 10: every frame sits in every window, so the branch is ordinary
    # dense attention over all video and text keys (library routine).
    inp = S.make_inputs("tiny")
    for h in range(inp["H"]):
        a = O.softmax_branch_head(inp["q"], inp["k"], inp["v"], inp["kt"],
                                  inp["vt"], inp["off"], h)
        q = torch.from_numpy(inp["q"][:, h].astype(np.float64))[None]
        K = torch.from_numpy(np.concatenate([inp["k"][:, h], inp["kt"][:, h]])
                             .astype(np.float64))[None]
        V = torch.from_numpy(np.concatenate([inp["v"][:, h], inp["vt"][:, h]])
                             .astype(np.float64))[None]
        ref = torch.nn.functional.scaled_dot_product_attention(q, K, V)[0]
        np.testing.assert_allclose(a, ref.numpy(), rtol=0, atol=1e-12)


def test_softmax_rows_subset_matches_full():
    inp = S.make_inputs("tiny-scan")
    rows = np.array([0, 5, 23, 24, 100, 239, 240, 479])
    full = O.softmax_branch_head(inp["q"], inp["k"], inp["v"], inp["kt"],
                                 inp["vt"], inp["off"], 1)
    sub = O.softmax_branch_head(inp["q"], inp["k"], inp["v"], inp["kt"],
                                inp["vt"], inp["off"], 1, rows=rows)
    np.testing.assert_allclose(sub, full[rows], rtol=0, atol=1e-13)


# ------------------------------------------------------------ frame update --

def _rand_state(rng, d):
    return rng.standard_normal((d, d))


@pytest.mark.parametrize("lam", [1.0, 0.3, 4.0])
def test_single_token_frame_is_delta_rule(lam):
    # n = 1: (lam I + k k^T)^-1 (lam S + k v^T) = S + k (v - S^T k)^T / (lam + k^T k)
    rng = np.random.default_rng(1)
    d = 16
    for _ in range(5):
        S0 = _rand_state(rng, d)
        k = rng.standard_normal(d)
        k = k / np.linalg.norm(k) * rng.uniform(0.5, 2.0)
        v = rng.standard_normal(d)
        got = O.frame_update(S0, k[None, :], v[None, :], lam)
        ref = S0 + np.outer(k, v - S0.T @ k) / (lam + k @ k)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n", [0, 1, 5, 16, 40])
def test_frame_update_is_ridge_least_squares(n):
    # argmin_S ||K S - V||^2 + lam ||S - S_prev||^2  ==  lstsq([K; sqrt(lam) I], [V; sqrt(lam) S_prev])
    rng = np.random.default_rng(2 + n)
    d, lam = 12, 0.7
    K = O.l2_normalise(rng.standard_normal((n, d)))
    V = rng.standard_normal((n, d))
    S0 = _rand_state(rng, d)
    A = np.concatenate([K, np.sqrt(lam) * np.eye(d)])
    B = np.concatenate([V, np.sqrt(lam) * S0])
    ref = np.linalg.lstsq(A, B, rcond=None)[0]
    np.testing.assert_allclose(O.frame_update(S0, K, V, lam), ref, rtol=0,
                               atol=1e-11)


def test_text_state_is_ridge_from_zero():
    rng = np.random.default_rng(7)
    d, T, lam = 10, 13, 1.0
    Kt = O.l2_normalise(rng.standard_normal((T, d)))
    Vt = rng.standard_normal((T, d))
    A = np.concatenate([Kt, np.sqrt(lam) * np.eye(d)])
    B = np.concatenate([Vt, np.zeros((d, d))])
    ref = np.linalg.lstsq(A, B, rcond=None)[0]
    np.testing.assert_allclose(O.text_state(Kt, Vt, lam), ref, rtol=0, atol=1e-12)
    assert np.all(O.text_state(np.zeros((0, d)), np.zeros((0, d)), lam) == 0)


def test_orthonormal_keys_equal_sequential_delta_steps():
    # Orthonormal keys: the joint update equals n token-wise delta steps
    # S <- S + k (v - S^T k)^T / (lam + 1), in any order.
    rng = np.random.default_rng(4)
    d, n, lam = 16, 6, 1.0
    Qm, _ = np.linalg.qr(rng.standard_normal((d, n)))
    K = Qm.T
    V = rng.standard_normal((n, d))
    S0 = _rand_state(rng, d)
    got = O.frame_update(S0, K, V, lam)
    for order in (range(n), reversed(range(n)), rng.permutation(n)):
        S = S0.copy()
        for i in order:
            S = S + np.outer(K[i], V[i] - S.T @ K[i]) / (lam + 1.0)
        np.testing.assert_allclose(got, S, rtol=0, atol=1e-12)


def test_fixed_point():
    rng = np.random.default_rng(5)
    d, n = 12, 20
    Sstar = _rand_state(rng, d)
    K = O.l2_normalise(rng.standard_normal((n, d)))
    np.testing.assert_allclose(O.frame_update(Sstar, K, K @ Sstar, 1.0), Sstar,
                               rtol=0, atol=1e-12)


def test_large_lambda_keeps_state():
    rng = np.random.default_rng(6)
    d, n = 8, 30
    S0 = _rand_state(rng, d)
    K = O.l2_normalise(rng.standard_normal((n, d)))
    V = rng.standard_normal((n, d))
    got = O.frame_update(S0, K, V, 1e9)
    np.testing.assert_allclose(got, S0, rtol=0, atol=1e-6)


@pytest.mark.parametrize("n", [1, 7, 64, 300])
def test_zero_value_frame_is_non_expansive(n):
    rng = np.random.default_rng(10 + n)
    d = 32
    for _ in range(10):
        S0 = _rand_state(rng, d) * rng.uniform(0.1, 10)
        K = O.l2_normalise(rng.standard_normal((n, d)))
        S1 = O.frame_update(S0, K, np.zeros((n, d)), 1.0)
        assert np.linalg.norm(S1) <= np.linalg.norm(S0) * (1 + 1e-12)


def test_vda_stress_zero_frames_non_expansive():
    # every frame f % 11 == 10 of the vda-stress layout has v = 0; check the
    # scan never grows the state there (reduced head dim to keep this fast)
    cfg = S.CONFIGS["vda-stress"]
    sizes = S.frame_sizes(cfg) // 4
    inp = S.make_inputs_from(cfg["F"], sizes, 16, 1, 16, dtype="f32", seed=0,
                             zero_v_every=11)
    st = O.vda_states_head(inp["k"], inp["v"], inp["kt"], inp["vt"], inp["off"], 0)
    F = cfg["F"]
    hits = 0
    for f in range(1, F - 1):
        if f % 11 == 10:
            hits += 1
            assert np.linalg.norm(st["fwd"][f]) <= np.linalg.norm(st["fwd"][f - 1]) * (1 + 1e-12)
            assert np.linalg.norm(st["bwd"][f]) <= np.linalg.norm(st["bwd"][f + 1]) * (1 + 1e-12)
    assert hits == 5


# ------------------------------------------------------- scan / read states --

def test_short_clip_reads_text_twice():
    # F <= 10: the window covers everything, so each block reads S_text twice
    inp = S.make_inputs("tiny")
    st = O.vda_states_head(inp["k"], inp["v"], inp["kt"], inp["vt"], inp["off"], 0)
    for b in range(st["R"].shape[0]):
        np.testing.assert_allclose(st["R"][b], 2 * st["S_text"], rtol=0, atol=0)


@pytest.mark.parametrize("F", [11, 16, 20, 23])
def test_read_state_sees_exactly_the_linear_frames(F):
    # Put value mass in one frame g at a time (no text): the block read state
    # is nonzero iff g is a linear-branch frame of that block, where the
    # linear frames are the complement of the dense softmax mask rule.
    d = 4
    inp = small_inputs(F, n=3, T=0, H=1, d=d, seed=F)
    bf = 5
    nb = O.num_blocks(F, bf)
    blk = np.arange(F) // bf
    for g in range(F):
        v = np.zeros_like(inp["v"])
        v[inp["off"][g]:inp["off"][g + 1]] = inp["v"][inp["off"][g]:inp["off"][g + 1]]
        st = O.vda_states_head(inp["k"], v, inp["kt"], inp["vt"], inp["off"], 0)
        for b in range(nb):
            in_softmax = abs(blk[g] - b) <= 1 or g in (0, F - 1)
            nonzero = np.linalg.norm(st["R"][b]) > 1e-12
            assert nonzero == (not in_softmax), (F, g, b)


# ----------------------------------------------------------------- merge ----

def test_rmsnorm_closed_form():
    rng = np.random.default_rng(8)
    d, eps = 32, 1e-6
    o = rng.standard_normal((50, d)) * rng.uniform(1e-4, 10, size=(50, 1))
    y = O.rmsnorm(o, np.ones(d), eps)
    ms = np.mean(o * o, axis=1)
    np.testing.assert_allclose(np.sum(y * y, axis=1), d * ms / (ms + eps),
                               rtol=1e-12)
    w = rng.standard_normal(d)
    np.testing.assert_allclose(O.rmsnorm(o, w, eps), y * w, rtol=1e-12)


def test_gate_limits():
    rng = np.random.default_rng(9)
    n, d = 20, 16
    os_, ol = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    big = np.full(n, 50.0)
    np.testing.assert_allclose(O.gate_merge(os_, ol, big, -big, np.ones(d), 1e-6),
                               os_, atol=1e-20)
    np.testing.assert_allclose(O.gate_merge(os_, ol, -big, big, np.ones(d), 1e-6),
                               O.rmsnorm(ol, np.ones(d), 1e-6), atol=1e-20)
    z = np.zeros(n)
    np.testing.assert_allclose(O.gate_merge(os_, ol, z, z, np.ones(d), 1e-6),
                               0.5 * os_ + 0.5 * O.rmsnorm(ol, np.ones(d), 1e-6),
                               rtol=1e-14)


def test_layer_head_rows_subset():
    inp = S.make_inputs("tiny-scan")
    full = O.layer_head(inp, 1)
    rows = np.array([0, 1, 119, 120, 121, 300, 479])
    sub = O.layer_head(inp, 1, rows=rows)
    np.testing.assert_allclose(sub["out"], full["out"][rows], rtol=0, atol=1e-12)


# ------------------------------------------------------------- pair sets ----

def _brute_classes(F, bf):
    # independent token-free restatement: softmax iff |blk(f)-blk(g)| <= 1 or
    # g is an anchor; everything else belongs to the linear branch
    blk = np.arange(F) // bf
    soft = (np.abs(blk[:, None] - blk[None, :]) <= 1)
    soft[:, 0] = True
    soft[:, F - 1] = True
    return soft


@pytest.mark.parametrize("bf", [1, 2, 3, 5, 7])
def test_pair_sets_disjoint_and_covering(bf):
    for F in range(2, 71):
        C = O.pair_class_matrix(F, bf)
        assert np.all((C == 1) | (C == 2)), (F, bf)   # never both, never neither
        np.testing.assert_array_equal(C == 1, _brute_classes(F, bf))


def test_pair_split_golden():
    with open(os.path.join(GOLDEN, "pair_split.json")) as fh:
        gold = json.load(fh)["uniform"]
    for name, g in gold.items():
        cfg = S.CONFIGS[name]
        off = S.frame_offsets(S.frame_sizes(cfg))
        soft, lin = O.pair_counts(off, 5, cfg["T"])
        n = np.diff(off.astype(np.int64))
        assert soft[:, :-1].sum() + lin.sum() == n.sum() ** 2
        num, den = g["softmax_share"]
        assert soft[:, :-1].sum() * den == num * n.sum() ** 2, name
        F = cfg["F"]
        per_block = [len(O.softmax_key_frames(b, F)) for b in range(O.num_blocks(F))]
        assert per_block == g["visible_frames_per_block"]


def test_pair_split_vda_stress_token_level():
    # non-uniform frames: count token pairs with an explicit per-token rule
    cfg = S.CONFIGS["vda-stress"]
    off = S.frame_offsets(S.frame_sizes(cfg))
    F = cfg["F"]
    soft, lin = O.pair_counts(off, 5, cfg["T"])
    fid = np.repeat(np.arange(F), np.diff(off))
    blk = fid // 5
    cnt = 0
    for f in range(F):
        rows = fid == f
        b = f // 5
        cols = (np.abs(blk - b) <= 1) | (fid == 0) | (fid == F - 1)
        cnt += rows.sum() * cols.sum()
    assert soft[:, :-1].sum() == cnt
    N = int(off[-1])
    assert lin.sum() == N * N - cnt
    assert np.all(soft[:, -1] == np.diff(off) * cfg["T"])


def test_backward_scan_is_forward_scan_of_reversed_clip():
    # Reversing the frame order swaps the two scans: bwd[f] of the clip equals
    # fwd[F-1-f] of the reversed clip, for every frame 1..F-2.
    F = 13
    sizes = [3, 5, 2, 4, 6, 1, 3, 2, 5, 4, 3, 2, 6]
    inp = small_inputs(F, sizes=sizes, T=3, H=1, d=6, seed=11)
    off = inp["off"]
    order = np.concatenate([np.arange(off[f], off[f + 1]) for f in reversed(range(F))])
    roff = S.frame_offsets(list(reversed(sizes)))
    a = O.vda_states_head(inp["k"], inp["v"], inp["kt"], inp["vt"], off, 0)
    r = O.vda_states_head(inp["k"][order], inp["v"][order], inp["kt"], inp["vt"], roff, 0)
    assert sorted(a["bwd"]) == list(range(1, F))
    assert sorted(a["fwd"]) == list(range(0, F - 1))
    for f in range(1, F):
        np.testing.assert_allclose(a["bwd"][f], r["fwd"][F - 1 - f], rtol=0, atol=1e-12)


def test_linear_branch_normalises_keys():
    # keys are L2-normalised inside the linear branch: rescaling any key row
    # by a positive factor leaves every state unchanged
    inp = small_inputs(12, n=5, T=4, H=1, d=6, seed=12)
    rng = np.random.default_rng(0)
    k2 = inp["k"] * rng.uniform(0.1, 10.0, size=inp["k"].shape[:2] + (1,))
    kt2 = inp["kt"] * rng.uniform(0.1, 10.0, size=inp["kt"].shape[:2] + (1,))
    a = O.vda_states_head(inp["k"], inp["v"], inp["kt"], inp["vt"], inp["off"], 0)
    b = O.vda_states_head(k2, inp["v"], kt2, inp["vt"], inp["off"], 0)
    np.testing.assert_allclose(a["R"], b["R"], rtol=0, atol=1e-12)
    for f in a["fwd"]:
        np.testing.assert_allclose(a["fwd"][f], b["fwd"][f], rtol=0, atol=1e-12)


# ------------------------------------------- readout orientation, text start --

def test_readout_is_q_transpose_state_one_token_closed_form():
    # One video token (unit key k, value v) in frame 5 and no text: the
    # forward state after it is (I + k k^T)^-1 k v^T = k v^T / 2 (lambda = 1,
    # Sherman-Morrison), and frames 1..9 are the whole forward range block 3
    # of a 20-frame clip reads (its window is frames 10..19; its backward
    # read is the text state, here zero). A query q = k in block 3 must read
    # o_lin = q^T R = (k.k) v / 2 = v / 2, i.e. a vector along v. The
    # transposed readout R q = k (v.k) / 2 would point along k instead.
    F, d = 20, 8
    sizes = [2] + [0] * 4 + [1] + [0] * 4 + [3] * 10
    inp = small_inputs(F, sizes=sizes, T=0, H=1, d=d, seed=31)
    off = inp["off"]
    k = inp["k"][off[5], 0].astype(np.float64)
    v = inp["v"][off[5], 0].astype(np.float64)
    row = int(off[17])                       # a token of frame 17 (block 3)
    q = inp["q"].copy()
    q[row, 0] = k
    inp["q"] = q
    res = O.layer_head(inp, 0, rows=np.array([row]))
    # k is a float32 unit vector, so q . k_hat = ||k|| = 1 up to float32 rounding
    np.testing.assert_allclose(res["o_lin"][0], np.linalg.norm(k) * v / 2, rtol=0, atol=1e-12)
    cos_k = abs(res["o_lin"][0] @ k) / np.linalg.norm(res["o_lin"][0])
    assert cos_k < 0.9  # not along k (k and v are independent draws)


@pytest.mark.parametrize("F,seed", [(16, 41), (20, 42), (23, 43), (31, 44)])
def test_both_scans_start_from_text_state_closed_form(F, seed):
    # Every video key is the unit vector e1 and every video value is 0; frame
    # f holds n_f in {0, 1, 2, 3} tokens. A frame update is then
    # S -> (I + n e1 e1^T)^-1 S: row 0 of S is scaled by 1 / (1 + n) and the
    # other rows are unchanged. Both scans start from S_text, so block b reads
    #   R_b = 2 S_text with row 0 scaled by (a_f + a_b) / 2,
    #   a_f = prod_{f=1..i_f} 1/(1+n_f),  a_b = prod_{f=i_b..F-2} 1/(1+n_f),
    # with [w0, w1] = b's window, i_f = max(w0-1, 0), i_b = min(w1+1, F-1).
    # A scan started from zero gives R_b = 0; a missing direction drops a term.
    d = 6
    rng = np.random.default_rng(seed)
    sizes = rng.integers(0, 4, size=F)
    inp = small_inputs(F, sizes=sizes, T=5, H=1, d=d, seed=seed)
    k = np.zeros_like(inp["k"])
    k[:, 0, 0] = 1.0
    st = O.vda_states_head(k, np.zeros_like(inp["v"]), inp["kt"], inp["vt"],
                           inp["off"], 0)
    S_text = O.text_state(O.l2_normalise(inp["kt"][:, 0]), inp["vt"][:, 0], 1.0)
    assert np.linalg.norm(S_text) > 0.1
    for b in range(O.num_blocks(F)):
        w0 = 5 * max(b - 1, 0)
        w1 = min(5 * (b + 2), F) - 1
        i_f, i_b = max(w0 - 1, 0), min(w1 + 1, F - 1)
        a_f = np.prod([1.0 / (1 + sizes[f]) for f in range(1, i_f + 1)])
        a_b = np.prod([1.0 / (1 + sizes[f]) for f in range(i_b, F - 1)])
        ref = 2 * S_text
        ref[0] = (a_f + a_b) * S_text[0]
        np.testing.assert_allclose(st["R"][b], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("F", [16, 20, 30])
def test_text_values_reach_every_read_state(F):
    # With F >= 16 at least one block reads scan states that have passed
    # video frames; perturbing only the text values must still change every
    # block's read state (the text initialises both scans).
    inp = small_inputs(F, n=3, T=4, H=1, d=5, seed=F + 50)
    a = O.vda_states_head(inp["k"], inp["v"], inp["kt"], inp["vt"], inp["off"], 0)
    vt2 = inp["vt"] + 0.5 * np.random.default_rng(F).standard_normal(inp["vt"].shape)
    b = O.vda_states_head(inp["k"], inp["v"], inp["kt"], vt2, inp["off"], 0)
    assert any(i > 0 for i in (O.read_indices(bb, F)[0] for bb in range(O.num_blocks(F))))
    for bb in range(O.num_blocks(F)):
        assert np.linalg.norm(a["R"][bb] - b["R"][bb]) > 1e-6 * np.linalg.norm(a["R"][bb])
