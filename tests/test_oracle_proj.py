"""Pins of the oracle's per-branch output projections, and the CPU emulation
that derives the FP8 (e4m3) tolerance of the projected output.

The projection reading: each branch has its own sigmoid gate and output
projection before the merge (nav.superapi.store page, Technical Principles,
Gated Fusion Mechanism); with per-token, per-head gates the gate is applied
per head before the projection, y = W_s a_s + W_l a_l."""
import numpy as np
import pytest
import torch

import oracle as O
import vdn_synth as S


def _tiny(seed=0, F=12, H=2, d=4):
    return S.make_inputs_from(F, [3] * F, 2, H, d, dtype="f32", seed=seed)


def test_identity_weights_give_the_merged_layer():
    inp = S.make_inputs("tiny-scan")
    H, d = inp["H"], inp["d"]
    eye = np.eye(H * d)
    w_o = np.concatenate([eye, eye], axis=1)           # [I | I]
    rows = np.array([0, 7, 100, 250, 479])
    y = O.layer_proj(inp, w_o, rows=rows)
    out = np.stack([O.layer_head(inp, h, rows=rows)["out"] for h in range(H)], axis=1)
    np.testing.assert_allclose(y, out.reshape(len(rows), H * d), rtol=0, atol=1e-13)


def test_projection_equals_brute_force_loops():
    inp = _tiny(seed=3)
    H, d, D = inp["H"], inp["d"], 3
    w_o = np.random.default_rng(5).standard_normal((D, 2 * H * d))
    rows = np.array([0, 5, 17, 35])
    br = O.gated_branches(inp, rows)
    y = O.output_projection(br, w_o)
    for a, i in enumerate(rows):
        for o in range(D):
            acc = 0.0
            for branch in range(2):
                for h in range(H):
                    for j in range(d):
                        acc += w_o[o, branch * H * d + h * d + j] * br[a, branch, h, j]
            assert abs(y[a, o] - acc) < 1e-12


def test_gate_limits_select_one_projected_branch():
    # g_l -> -inf leaves W_s (sigmoid(g_s) o_soft); g_s -> -inf leaves
    # W_l (sigmoid(g_l) RMSNorm(o_lin)), built here from the pinned branch
    # functions
    inp = _tiny(seed=4)
    H, d, D = inp["H"], inp["d"], 5
    w_o = np.random.default_rng(6).standard_normal((D, 2 * H * d))
    N = inp["N"]
    rows = np.arange(N)
    a = dict(inp, g_l=np.full_like(inp["g_l"], -80.0))
    o_soft = np.stack([O.softmax_branch_head(inp["q"], inp["k"], inp["v"], inp["kt"], inp["vt"],
                                             inp["off"], h) for h in range(H)], axis=1)
    want = (O.sigmoid(inp["g_s"])[:, :, None] * o_soft).reshape(N, H * d) @ w_o[:, :H * d].T
    np.testing.assert_allclose(O.layer_proj(a, w_o, rows), want, rtol=0, atol=1e-12)
    b = dict(inp, g_s=np.full_like(inp["g_s"], -80.0))
    o_lin = np.stack([O.layer_head(inp, h)["o_lin"] for h in range(H)], axis=1)
    a_l = O.sigmoid(inp["g_l"])[:, :, None] * np.stack(
        [O.rmsnorm(o_lin[:, h], inp["rms_w"][h], inp["eps"]) for h in range(H)], axis=1)
    want = a_l.reshape(N, H * d) @ w_o[:, H * d:].T
    np.testing.assert_allclose(O.layer_proj(b, w_o, rows), want, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- FP8 ------
#
# FP8 reading (the CUDA path implements the same): each row r of a matrix X
# (a token's gated branches, or an output channel's weights) gets the scale
# s_r = amax_r / 448 (float32; 1 for an all-zero row) and the codes
# e4m3(X[r, k] * (448 / amax_r)) rounded to nearest even in float32;
# y = s_a s_w sum_k A8 W8. e4m3 keeps 3 mantissa bits: a normal code is off by
# at most 2^-4 of its value, so each product carries two such relative errors.
# With independent errors uniform in +-2^-4 (RMS 2^-4 / sqrt 3) the relative
# L2 error of a sum of many such products is about sqrt(2) * 0.036 = 0.051;
# rounding to nearest has a smaller RMS than that. The tolerance used for the
# FP8 projected output is rel-L2 <= 0.08 over the whole output and <= 0.15
# for any single row.
FP8_REL_L2 = 0.08
FP8_ROW_REL_L2 = 0.15


def e4m3_rows(x: np.ndarray):
    """Per-row e4m3 codes (as float64 values) and scales, float32 arithmetic."""
    x = np.asarray(x, np.float32)
    amax = np.max(np.abs(x), axis=1)
    inv = np.where(amax > 0, np.float32(448.0) / np.where(amax > 0, amax, 1), np.float32(1))
    inv = inv.astype(np.float32)
    scale = np.where(amax > 0, amax / np.float32(448.0), np.float32(1)).astype(np.float32)
    codes = torch.from_numpy((x * inv[:, None]).astype(np.float32)).to(torch.float8_e4m3fn)
    return codes.to(torch.float64).numpy(), scale


def test_e4m3_cast_properties():
    # the emulation's rounding: exact on representable values, relative error
    # <= 2^-4 on normal values, 448 is the largest finite code
    vals = np.array([0.0, 1.0, 1.125, 448.0, -448.0, 2.0 ** -6, 2.0 ** -9], np.float32)
    got = torch.from_numpy(vals).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(got, vals.astype(np.float64))
    x = np.random.default_rng(0).uniform(2.0 ** -6, 448, 100000).astype(np.float32)
    q = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.max(np.abs(q - x) / x) <= 2.0 ** -4 + 1e-12
    assert np.max(np.abs(q - x) / x) > 0.05       # the bound is nearly reached


@pytest.mark.parametrize("name", ["tiny-scan", "mid"])
def test_fp8_projection_error_within_derived_tolerance(name):
    if name == "mid":
        inp = S.make_inputs_from(12, [60] * 12, 16, 4, 128, "bf16", seed=7)
    else:
        inp = S.make_inputs(name)
    H, d = inp["H"], inp["d"]
    w_o = S.make_proj_weight(H, d, seed=1)
    br = O.gated_branches(inp).reshape(inp["N"], -1)
    exact = br @ w_o.astype(np.float64).T
    # the GPU stores the gated branches as bf16 before quantising them
    a_codes, sa = e4m3_rows(S.bf16_round(br.astype(np.float32)))
    w_codes, sw = e4m3_rows(w_o)
    y8 = (a_codes @ w_codes.T) * sa[:, None].astype(np.float64) * sw[None, :].astype(np.float64)
    rel = np.linalg.norm(y8 - exact) / np.linalg.norm(exact)
    row_rel = np.linalg.norm(y8 - exact, axis=1) / np.linalg.norm(exact, axis=1)
    assert 0.01 < rel <= FP8_REL_L2 * 0.75, rel        # derived bound holds with margin
    assert row_rel.max() <= FP8_ROW_REL_L2, row_rel.max()
