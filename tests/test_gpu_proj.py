"""Per-branch output projections on the GPU (through the C ABI) against the
fp64 oracle: the gated branches, the bf16 and e4m3 GEMMs, the per-row e4m3
quantiser (codes bit-exact against a float32 CPU emulation), and the whole
projected layer.

Tolerances: bf16 path as the layer (rel-L2 <= 2e-2, max-abs <= 5e-2);
e4m3 path rel-L2 <= 0.08 overall and <= 0.15 per row (derived from e4m3's
2^-4 relative rounding in tests/test_oracle_proj.py); the GEMMs against an
fp64 product of the same operands rel-L2 <= 1e-2 (fp32 accumulation, bf16
output)."""
import numpy as np
import pytest
import torch

import oracle as O
import vdn_synth as S
from test_oracle_proj import FP8_REL_L2, FP8_ROW_REL_L2, e4m3_rows
from vdn_cases import (OUT_MAX_ABS, OUT_REL_L2, device_inputs, make_shape, max_abs, mid_case,
                       rel_l2, run_layer)

pytestmark = pytest.mark.gpu

GEMM_REL_L2 = 1e-2


def _V():
    import video_diffusion_hybrid_block_b200 as V
    return V


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(S.bf16_round(np.asarray(x, np.float32)))).to(
        "cuda", torch.bfloat16)


def run_branches(inp, dev=None):
    V = _V()
    dev = dev or device_inputs(inp)
    shape = make_shape(inp)
    ws = V.alloc_workspace(shape)
    br = torch.empty((inp["N"], 2 * inp["H"], inp["d"]), dtype=torch.bfloat16, device="cuda")
    V.vdn_hybrid_attn_branches(shape, dev["q"], dev["k"], dev["v"], dev["kt"], dev["vt"],
                               dev["g_s"], dev["g_l"], dev["rms_w"], br, ws)
    torch.cuda.synchronize()
    assert V.vdn_get_device_error() == 0
    return br


def run_proj(inp, w_o, precision, dev=None):
    V = _V()
    dev = dev or device_inputs(inp)
    shape = make_shape(inp)
    D = w_o.shape[0]
    K = w_o.shape[1]
    ws = V.alloc_proj_workspace(shape, D, precision)
    y = torch.empty((inp["N"], D), dtype=torch.bfloat16, device="cuda")
    if precision == V.VDN_PROJ_FP8:
        w = _bf16(w_o)
        codes = torch.empty((D, K), dtype=torch.uint8, device="cuda")
        scale = torch.empty(D, dtype=torch.float32, device="cuda")
        V.vdn_quantize_rows_e4m3(w, D, K, codes, scale)
        V.vdn_hybrid_attn_proj_fwd(shape, dev["q"], dev["k"], dev["v"], dev["kt"], dev["vt"],
                                   dev["g_s"], dev["g_l"], dev["rms_w"], codes, scale, D,
                                   precision, y, ws)
    else:
        V.vdn_hybrid_attn_proj_fwd(shape, dev["q"], dev["k"], dev["v"], dev["kt"], dev["vt"],
                                   dev["g_s"], dev["g_l"], dev["rms_w"], _bf16(w_o), None, D,
                                   precision, y, ws)
    torch.cuda.synchronize()
    assert V.vdn_get_device_error() == 0
    return y.float().cpu().numpy()


@pytest.mark.parametrize("seed", [0, 1])
def test_gated_branches_match_oracle(seed):
    inp = mid_case(seed=seed + 20)
    br = run_branches(inp).float().cpu().numpy().reshape(inp["N"], 2, inp["H"], inp["d"])
    ref = O.gated_branches(inp)
    for b in range(2):
        for h in range(inp["H"]):
            assert rel_l2(br[:, b, h], ref[:, b, h]) <= OUT_REL_L2, (b, h)
            assert max_abs(br[:, b, h], ref[:, b, h]) <= OUT_MAX_ABS, (b, h)


def test_branch_sum_is_the_merged_layer():
    inp = mid_case(seed=22)
    dev = device_inputs(inp)
    br = run_branches(inp, dev).float()
    H = inp["H"]
    out = run_layer(inp, dev).float()
    assert rel_l2((br[:, :H] + br[:, H:]).cpu().numpy(), out.cpu().numpy()) <= 1e-2


@pytest.mark.parametrize("M,K,D", [(300, 272, 264), (1000, 1024, 520), (128, 64, 256),
                                   (5, 16, 8), (2500, 768, 1024)])
def test_linear_bf16_matches_fp64(M, K, D):
    V = _V()
    rng = np.random.default_rng(M + K + D)
    a = S.bf16_round(rng.standard_normal((M, K), dtype=np.float32))
    w = S.bf16_round(rng.standard_normal((D, K), dtype=np.float32) / np.float32(np.sqrt(K)))
    y = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
    V.vdn_linear(_bf16(a), None, _bf16(w), None, M, K, D, V.VDN_PROJ_BF16, y)
    torch.cuda.synchronize()
    assert V.vdn_get_device_error() == 0
    ref = a.astype(np.float64) @ w.astype(np.float64).T
    got = y.float().cpu().numpy()
    assert rel_l2(got, ref) <= GEMM_REL_L2
    assert max_abs(got, ref) <= 1e-2 * np.abs(ref).max() + 1e-3


@pytest.mark.parametrize("rows,K", [(37, 48), (1000, 6144), (5, 6160), (4, 16)])
def test_quantize_rows_bit_exact(rows, K):
    V = _V()
    rng = np.random.default_rng(rows)
    x = S.bf16_round(rng.standard_normal((rows, K), dtype=np.float32)
                     * rng.uniform(1e-3, 30, size=(rows, 1)).astype(np.float32))
    x[0] = 0.0  # an all-zero row gets scale 1 and zero codes
    codes = torch.empty((rows, K), dtype=torch.uint8, device="cuda")
    scale = torch.empty(rows, dtype=torch.float32, device="cuda")
    V.vdn_quantize_rows_e4m3(_bf16(x), rows, K, codes, scale)
    torch.cuda.synchronize()
    ref_codes, ref_scale = e4m3_rows(x)
    got = codes.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(got, ref_codes)
    np.testing.assert_array_equal(scale.cpu().numpy(), ref_scale)


@pytest.mark.parametrize("M,K,D", [(300, 272, 264), (1000, 1024, 520), (2500, 768, 1024)])
def test_linear_fp8_matches_dequantised_fp64(M, K, D):
    V = _V()
    rng = np.random.default_rng(M * 3 + K + D)
    a = S.bf16_round(rng.standard_normal((M, K), dtype=np.float32))
    w = S.bf16_round(rng.standard_normal((D, K), dtype=np.float32) / np.float32(np.sqrt(K)))
    ac = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sa = torch.empty(M, dtype=torch.float32, device="cuda")
    wc = torch.empty((D, K), dtype=torch.uint8, device="cuda")
    sw = torch.empty(D, dtype=torch.float32, device="cuda")
    V.vdn_quantize_rows_e4m3(_bf16(a), M, K, ac, sa)
    V.vdn_quantize_rows_e4m3(_bf16(w), D, K, wc, sw)
    y = torch.empty((M, D), dtype=torch.bfloat16, device="cuda")
    V.vdn_linear(ac, sa, wc, sw, M, K, D, V.VDN_PROJ_FP8, y)
    torch.cuda.synchronize()
    assert V.vdn_get_device_error() == 0
    a8, ra = e4m3_rows(a)
    w8, rw = e4m3_rows(w)
    ref = (a8 @ w8.T) * ra[:, None].astype(np.float64) * rw[None, :].astype(np.float64)
    got = y.float().cpu().numpy()
    assert rel_l2(got, ref) <= GEMM_REL_L2
    exact = a.astype(np.float64) @ w.astype(np.float64).T
    assert rel_l2(got, exact) <= FP8_REL_L2


def test_identity_weights_reproduce_the_layer():
    V = _V()
    inp = mid_case(seed=23)
    H, d = inp["H"], inp["d"]
    eye = np.eye(H * d, dtype=np.float32)
    y = run_proj(inp, np.concatenate([eye, eye], axis=1), V.VDN_PROJ_BF16)
    out = run_layer(inp).float().cpu().numpy().reshape(inp["N"], H * d)
    assert rel_l2(y, out) <= 1e-2


@pytest.mark.parametrize("precision", [0, 1])
def test_projected_layer_matches_oracle(precision):
    inp = mid_case(seed=24)
    w_o = S.make_proj_weight(inp["H"], inp["d"], seed=2)
    y = run_proj(inp, w_o, precision)
    ref = O.layer_proj(inp, w_o)
    if precision == 0:
        assert rel_l2(y, ref) <= OUT_REL_L2
        assert max_abs(y, ref) <= OUT_MAX_ABS
    else:
        assert rel_l2(y, ref) <= FP8_REL_L2
        row = np.linalg.norm(y - ref, axis=1) / np.linalg.norm(ref, axis=1)
        assert row.max() <= FP8_ROW_REL_L2


@pytest.mark.parametrize("name,precision", [("pages-scale", 0), ("pages-scale", 1),
                                            ("hi-res", 1)])
def test_projected_layer_full_size_sampled(name, precision):
    inp = S.make_inputs(name)
    w_o = S.make_proj_weight(inp["H"], inp["d"], seed=3)
    y = run_proj(inp, w_o, precision)
    rows = np.unique(np.concatenate([np.random.default_rng(4).choice(inp["N"], 24, replace=False),
                                     [0, inp["N"] - 1, 127, 128, 255, 256]]))
    ref = O.layer_proj(inp, w_o, rows=rows)
    got = y[rows]
    if precision == 0:
        assert rel_l2(got, ref) <= OUT_REL_L2
        assert max_abs(got, ref) <= OUT_MAX_ABS
    else:
        assert rel_l2(got, ref) <= FP8_REL_L2
        row = np.linalg.norm(got - ref, axis=1) / np.linalg.norm(ref, axis=1)
        assert row.max() <= FP8_ROW_REL_L2


@pytest.mark.parametrize("D,precision", [(200, 0), (200, 1), (776, 1)])
def test_projected_layer_other_widths(D, precision):
    # output widths other than H d, including ragged 256-column tiles
    inp = mid_case(seed=25)
    w_o = S.make_proj_weight(inp["H"], inp["d"], D=D, seed=4)
    y = run_proj(inp, w_o, precision)
    ref = O.layer_proj(inp, w_o)
    assert y.shape == (inp["N"], D)
    if precision == 0:
        assert rel_l2(y, ref) <= OUT_REL_L2
        assert max_abs(y, ref) <= OUT_MAX_ABS
    else:
        assert rel_l2(y, ref) <= FP8_REL_L2
