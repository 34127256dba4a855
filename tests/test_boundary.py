"""Host-side checks of the C-ABI boundary: the library loads, exports every
function include/vdn.h declares, sizes its workspace, and rejects bad
arguments with the documented error codes before touching the GPU.

Every call here fails host validation, so these tests never launch a kernel
and never dereference the fake (but aligned) device addresses they pass."""
import ctypes
import os
import re

import numpy as np
import pytest

import vdn_synth as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vdn.h")

V = pytest.importorskip("video_diffusion_hybrid_block_b200")
from video_diffusion_hybrid_block_b200 import binding as B  # noqa: E402

FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced
FAKE_MIS = FAKE + 8


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(B.LIB_PATH):
        from video_diffusion_hybrid_block_b200 import build
        build.build()
    return B.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vdn_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("vdn_hybrid_attn_fwd", "vdn_vda_scan", "vdn_gate_merge", "vdn_bsa_fwd",
              "vdn_pair_audit", "vdn_workspace_bytes", "vdn_get_device_error",
              "vdn_error_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(B.EXPORTED) == set(declared_functions())


def shape(off=None, T=8, H=2, d=128, bf=5, lam=1.0, eps=1e-6, dtype=0):
    if off is None:
        off = S.frame_offsets([24] * 10)
    return V.Shape(off, T, H, d, bf, lam, eps, dtype, device="cpu")


def test_workspace_bytes(lib):
    for name in ("tiny", "pages-scale", "vda-stress"):
        cfg = S.CONFIGS[name]
        off = S.frame_offsets(S.frame_sizes(cfg))
        n = V.vdn_workspace_bytes(shape(off, cfg["T"], cfg["H"], cfg["d"],
                                        dtype=0 if cfg["dtype"] == "bf16" else 1))
        N, F, H, T = int(off[-1]), len(off) - 1, cfg["H"], cfg["T"]
        a256 = lambda x: -(-x // 256) * 256  # noqa: E731
        staged = cfg["dtype"] != "bf16" or cfg["d"] != 128
        nb = -(-F // 5)
        want = (3 * a256(N * H * 256) + 2 * a256(T * H * 256) if staged else 0) \
            + 2 * a256((F - 1) * H * 65536) + a256(2 * nb * H * 65536) + a256(nb * H * 32768)
        # staged bf16 q,k,v,kt,vt (fp32 or d < 128 only), C and W per matrix,
        # the two read-state halves, the packed read-state tiles
        assert n == want, (name, n, want)
    assert V.vdn_workspace_bytes(shape(d=48)) == 0
    assert V.vdn_workspace_bytes(shape(off=[0, 5])) == 0   # F = 1


@pytest.mark.parametrize("kw,code", [
    (dict(off=[0, 5]), B.VDN_ERR_INVALID_ARG),                  # F < 2
    (dict(off=[1, 5, 9]), B.VDN_ERR_INVALID_ARG),               # off[0] != 0
    (dict(off=[0, 5, 3, 9]), B.VDN_ERR_INVALID_ARG),            # not monotone
    (dict(d=48), B.VDN_ERR_UNSUPPORTED),
    (dict(d=256), B.VDN_ERR_UNSUPPORTED),
    (dict(H=0), B.VDN_ERR_INVALID_ARG),
    (dict(T=-1), B.VDN_ERR_INVALID_ARG),
    (dict(bf=0), B.VDN_ERR_INVALID_ARG),
    (dict(lam=0.0), B.VDN_ERR_INVALID_ARG),
    (dict(lam=float("nan")), B.VDN_ERR_INVALID_ARG),
    (dict(eps=-1.0), B.VDN_ERR_INVALID_ARG),
    (dict(dtype=7), B.VDN_ERR_UNSUPPORTED),
])
def test_bad_shapes(lib, kw, code):
    s = shape(**kw)
    rc = lib.vdn_hybrid_attn_fwd(s.ref, *([FAKE] * 9), FAKE, 1 << 40, 0)
    assert rc == code
    rc = lib.vdn_bsa_fwd(s.ref, *([FAKE] * 7), FAKE, 1 << 40, 0)
    assert rc == code
    rc = lib.vdn_vda_scan(s.ref, *([FAKE] * 8), FAKE, 1 << 40, 0)
    assert rc == code


def test_null_shape(lib):
    assert lib.vdn_hybrid_attn_fwd(None, *([FAKE] * 9), FAKE, 1 << 40, 0) == B.VDN_ERR_INVALID_ARG
    assert lib.vdn_workspace_bytes(None) == 0


def test_null_and_misaligned_pointers(lib):
    s = shape()
    ptrs = [FAKE] * 9
    for i in range(9):
        p = list(ptrs)
        p[i] = 0
        assert lib.vdn_hybrid_attn_fwd(s.ref, *p, FAKE, 1 << 40, 0) == B.VDN_ERR_INVALID_ARG, i
        p[i] = FAKE_MIS
        assert lib.vdn_hybrid_attn_fwd(s.ref, *p, FAKE, 1 << 40, 0) == B.VDN_ERR_MISALIGNED, i
    # text pointers may be NULL when T == 0, but then the workspace check fails
    s0 = shape(T=0)
    p = [FAKE] * 9
    p[3] = p[4] = 0
    assert lib.vdn_hybrid_attn_fwd(s0.ref, *p, FAKE, 16, 0) == B.VDN_ERR_WORKSPACE_TOO_SMALL
    assert lib.vdn_pair_audit(s.ref, None, FAKE, 0) == B.VDN_ERR_INVALID_ARG


def test_workspace_too_small_and_misaligned(lib):
    s = shape()
    need = V.vdn_workspace_bytes(s)
    assert lib.vdn_hybrid_attn_fwd(s.ref, *([FAKE] * 9), FAKE, need - 1, 0) == \
        B.VDN_ERR_WORKSPACE_TOO_SMALL
    assert lib.vdn_hybrid_attn_fwd(s.ref, *([FAKE] * 9), None, need, 0) == \
        B.VDN_ERR_WORKSPACE_TOO_SMALL
    assert lib.vdn_hybrid_attn_fwd(s.ref, *([FAKE] * 9), FAKE_MIS, need, 0) == \
        B.VDN_ERR_MISALIGNED
    assert lib.vdn_vda_scan(s.ref, *([FAKE] * 8), FAKE, need - 1, 0) == \
        B.VDN_ERR_WORKSPACE_TOO_SMALL
    assert lib.vdn_gate_merge(s.ref, *([FAKE] * 7), FAKE, need - 1, 0) == \
        B.VDN_ERR_WORKSPACE_TOO_SMALL


def test_error_strings(lib):
    for code in range(-7, 1):
        assert len(B.vdn_error_string(code)) > 0
    assert B.vdn_error_string(-99) == "unknown error"


def test_binding_raises_on_error(lib):
    s = shape(d=48)
    with pytest.raises(B.VdnError) as e:
        V.vdn_hybrid_attn_fwd(s, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                              stream=0, ws_bytes=1 << 40)
    assert e.value.code == B.VDN_ERR_UNSUPPORTED


@pytest.mark.parametrize("limit_ns,cols", [(0, 0), (-5, 0), (1_000_000_001, 0), (1000, 48),
                                           (1000, 16), (1000, 1024), (1000, -32)])
def test_selftest_wait_timeout_rejects_bad_arguments(lib, limit_ns, cols):
    # out-of-range limits or TMEM column counts fail before any launch
    assert lib.vdn_selftest_wait_timeout(limit_ns, cols, None) == -1


def test_binding_rejects_tensors_the_kernels_would_overrun():
    # The binding checks sizes, element sizes and device before calling the
    # library: each case passes one host tensor (every other argument is a
    # never-dereferenced address), so it raises before reaching the library.
    import torch
    off = S.frame_offsets([24] * 10)
    sh = shape(off, T=8, H=2, d=128)            # bf16
    N = int(off[-1])
    act = N * 2 * 128
    t = lambda n, dt=torch.bfloat16: torch.zeros(n, dtype=dt)  # noqa: E731
    names = ("q", "k", "v", "kt", "vt", "g_s", "g_l", "rms_w", "out")

    def call(**kw):
        a = {n: FAKE for n in names}
        a.update(kw)
        V.vdn_hybrid_attn_fwd(sh, *(a[n] for n in names), FAKE, ws_bytes=1 << 40)
    with pytest.raises(ValueError, match="q: .* elements"):
        call(q=t(act - 1))
    with pytest.raises(ValueError, match="k: elements of 4 bytes, expected 2"):
        call(k=t(act, torch.float32))
    with pytest.raises(ValueError, match="rms_w: .* elements"):
        call(rms_w=t(2 * 128 - 8, torch.float32))
    with pytest.raises(ValueError, match="out: must be a CUDA tensor"):
        call(out=t(act))
    with pytest.raises(ValueError, match="read_states"):
        V.vdn_vda_scan(sh, FAKE, FAKE, FAKE, FAKE, t(1, torch.float32), None, None, None, FAKE,
                       ws_bytes=1 << 40)
    with pytest.raises(ValueError, match="soft_pairs"):
        V.vdn_pair_audit(sh, t(10 * 10, torch.int64), FAKE)


# ------------------------------------------------ per-branch projections ---

def test_proj_workspace_bytes(lib):
    s = shape(H=3)
    N = int(s.N)
    base = V.vdn_workspace_bytes(s)
    K = 2 * 3 * 128
    al = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert V.vdn_proj_workspace_bytes(s, 384, B.VDN_PROJ_BF16) == base + al(N * K * 2)
    assert V.vdn_proj_workspace_bytes(s, 384, B.VDN_PROJ_FP8) == \
        base + al(N * K * 2) + al(N * K) + al(N * 4)
    # bf16 with d = 128 only; D a positive multiple of 8; known precision
    assert V.vdn_proj_workspace_bytes(shape(d=64), 384, 0) == 0
    assert V.vdn_proj_workspace_bytes(shape(dtype=1), 384, 0) == 0
    assert V.vdn_proj_workspace_bytes(s, 12, 0) == 0
    assert V.vdn_proj_workspace_bytes(s, 384, 2) == 0


@pytest.mark.parametrize("M,K,D,prec,code", [
    (-1, 64, 64, 0, B.VDN_ERR_INVALID_ARG), (10, 8, 64, 0, B.VDN_ERR_INVALID_ARG),
    (10, 72, 64, 0, B.VDN_ERR_INVALID_ARG), (10, 64, 4, 0, B.VDN_ERR_INVALID_ARG),
    (10, 64, 68, 0, B.VDN_ERR_INVALID_ARG), (10, 64, 64, 3, B.VDN_ERR_UNSUPPORTED)])
def test_linear_rejects_bad_sizes(lib, M, K, D, prec, code):
    assert lib.vdn_linear(FAKE, FAKE, FAKE, FAKE, M, K, D, prec, FAKE, 0) == code


def test_linear_and_quant_pointer_checks(lib):
    assert lib.vdn_linear(None, None, FAKE, None, 10, 64, 64, 0, FAKE, 0) == B.VDN_ERR_INVALID_ARG
    assert lib.vdn_linear(FAKE_MIS, None, FAKE, None, 10, 64, 64, 0, FAKE, 0) == B.VDN_ERR_MISALIGNED
    # e4m3 needs both scale vectors
    assert lib.vdn_linear(FAKE, None, FAKE, FAKE, 10, 64, 64, 1, FAKE, 0) == B.VDN_ERR_INVALID_ARG
    assert lib.vdn_linear(FAKE, FAKE, FAKE, FAKE_MIS, 10, 64, 64, 1, FAKE, 0) == B.VDN_ERR_MISALIGNED
    assert lib.vdn_quantize_rows_e4m3(FAKE, 10, 24, FAKE, FAKE, 0) == B.VDN_ERR_INVALID_ARG
    assert lib.vdn_quantize_rows_e4m3(None, 10, 32, FAKE, FAKE, 0) == B.VDN_ERR_INVALID_ARG
    assert lib.vdn_quantize_rows_e4m3(FAKE, 10, 32, FAKE_MIS, FAKE, 0) == B.VDN_ERR_MISALIGNED
    assert lib.vdn_quantize_rows_e4m3(FAKE, 0, 32, None, None, 0) == B.VDN_OK


def test_proj_layer_checks(lib):
    s = shape()
    need = V.vdn_proj_workspace_bytes(s, 256, 1)
    args = [FAKE] * 8
    assert lib.vdn_hybrid_attn_proj_fwd(s.ref, *args, FAKE, None, 256, 1, FAKE, FAKE, need, 0) == \
        B.VDN_ERR_INVALID_ARG
    assert lib.vdn_hybrid_attn_proj_fwd(s.ref, *args, FAKE, FAKE, 256, 1, FAKE, FAKE, need - 1,
                                        0) == B.VDN_ERR_WORKSPACE_TOO_SMALL
    assert lib.vdn_hybrid_attn_proj_fwd(shape(d=64).ref, *args, FAKE, FAKE, 256, 1, FAKE, FAKE,
                                        need, 0) == B.VDN_ERR_UNSUPPORTED
    assert lib.vdn_hybrid_attn_branches(shape(dtype=1).ref, *([FAKE] * 9), FAKE, need, 0) == \
        B.VDN_ERR_UNSUPPORTED


def test_split_layer_checks(lib):
    s = shape()
    need = V.vdn_workspace_bytes(s)
    assert V.vdn_read_images_bytes(s) == 2 * 2 * 32768          # nb = 2 blocks, H = 2
    assert lib.vdn_vda_read_images(s.ref, FAKE, FAKE, FAKE, FAKE, None, FAKE, need, 0) == \
        B.VDN_ERR_INVALID_ARG
    assert lib.vdn_vda_read_images(s.ref, FAKE, FAKE, FAKE, FAKE, FAKE_MIS, FAKE, need, 0) == \
        B.VDN_ERR_MISALIGNED
    assert lib.vdn_vda_read_images(s.ref, *([FAKE] * 5), FAKE, need - 1, 0) == \
        B.VDN_ERR_WORKSPACE_TOO_SMALL
    args = [FAKE] * 8
    assert lib.vdn_bsa_merge_fwd(s.ref, *args, None, FAKE, FAKE, need, 0) == B.VDN_ERR_INVALID_ARG
    assert lib.vdn_bsa_merge_fwd(s.ref, *args, FAKE, FAKE, FAKE, need - 1, 0) == \
        B.VDN_ERR_WORKSPACE_TOO_SMALL


def test_index_limit(lib):
    # N * H * 128 must stay below 2^31; one head more than the largest
    # accepted count is rejected before any launch
    off = S.frame_offsets([256] * 16)
    ok, bad = shape(off=off, H=4095), shape(off=off, H=4096)
    assert V.vdn_workspace_bytes(ok) > 0
    assert V.vdn_workspace_bytes(bad) == 0
    assert lib.vdn_hybrid_attn_fwd(bad.ref, *([FAKE] * 9), FAKE, 1 << 40, 0) == \
        B.VDN_ERR_UNSUPPORTED


def test_fp8_entry_checks(lib):
    # e4m3 softmax branch and layer: bf16 with d = 128 only; a workspace
    # sized for the bf16 layer is too small for the e4m3 codes
    s = shape()
    need = V.vdn_workspace_bytes(s)
    need8 = lib.vdn_fp8_workspace_bytes(s.ref)
    assert need8 > need
    for bad in (shape(dtype=1), shape(d=64)):
        assert lib.vdn_fp8_workspace_bytes(bad.ref) == 0
        assert lib.vdn_bsa_fwd_fp8(bad.ref, *([FAKE] * 7), FAKE, 1 << 40, 0) == \
            B.VDN_ERR_UNSUPPORTED
        assert lib.vdn_hybrid_attn_fwd_fp8(bad.ref, *([FAKE] * 9), FAKE, 1 << 40, 0) == \
            B.VDN_ERR_UNSUPPORTED
    bsa = [FAKE] * 7  # q, k, v, kt, vt, o_soft, lse
    for i in (0, 1, 2, 5):
        p = list(bsa)
        p[i] = 0
        assert lib.vdn_bsa_fwd_fp8(s.ref, *p, FAKE, need8, 0) == B.VDN_ERR_INVALID_ARG, i
        p[i] = FAKE_MIS
        assert lib.vdn_bsa_fwd_fp8(s.ref, *p, FAKE, need8, 0) == B.VDN_ERR_MISALIGNED, i
    p = list(bsa)
    p[6] = FAKE_MIS
    assert lib.vdn_bsa_fwd_fp8(s.ref, *p, FAKE, need8, 0) == B.VDN_ERR_MISALIGNED
    for ws, n in ((FAKE, need8 - 1), (FAKE, need), (None, need8)):
        assert lib.vdn_bsa_fwd_fp8(s.ref, *bsa, ws, n, 0) == B.VDN_ERR_WORKSPACE_TOO_SMALL
        assert lib.vdn_hybrid_attn_fwd_fp8(s.ref, *([FAKE] * 9), ws, n, 0) == \
            B.VDN_ERR_WORKSPACE_TOO_SMALL
    assert lib.vdn_bsa_fwd_fp8(s.ref, *bsa, FAKE_MIS, need8, 0) == B.VDN_ERR_MISALIGNED
    for i in range(9):
        p = [FAKE] * 9
        p[i] = 0
        assert lib.vdn_hybrid_attn_fwd_fp8(s.ref, *p, FAKE, need8, 0) == \
            B.VDN_ERR_INVALID_ARG, i


def test_profile_entry_checks(lib):
    # iteration count 1..256 and a result array are required
    s = shape()
    need = V.vdn_workspace_bytes(s)
    ms = (ctypes.c_float * 5)()
    for iters in (0, -1, 257):
        assert lib.vdn_hybrid_attn_fwd_profile(s.ref, *([FAKE] * 9), FAKE, need, 0, iters,
                                               ms) == B.VDN_ERR_INVALID_ARG, iters
    assert lib.vdn_hybrid_attn_fwd_profile(s.ref, *([FAKE] * 9), FAKE, need, 0, 4, None) == \
        B.VDN_ERR_INVALID_ARG
    assert lib.vdn_hybrid_attn_fwd_profile(s.ref, *([FAKE] * 9), FAKE, need - 1, 0, 4, ms) == \
        B.VDN_ERR_WORKSPACE_TOO_SMALL
    p = [FAKE] * 9
    p[0] = 0
    assert lib.vdn_hybrid_attn_fwd_profile(s.ref, *p, FAKE, need, 0, 4, ms) == \
        B.VDN_ERR_INVALID_ARG
