"""ctypes binding of the C ABI declared in include/vdn.h.

Argument marshalling only: every step of the layer runs in the CUDA kernels
of libvdn.so. Tensors are torch CUDA tensors (PyTorch supplies device memory
and streams); the functions pass their data pointers and the current stream.
There is no fallback: if libvdn.so is missing this module raises on import
of the library.
"""
from __future__ import annotations

import ctypes
import os

import torch

VDN_OK = 0
VDN_ERR_INVALID_ARG = -1
VDN_ERR_UNSUPPORTED = -2
VDN_ERR_WORKSPACE_TOO_SMALL = -3
VDN_ERR_MISALIGNED = -4
VDN_ERR_CUDA = -5
VDN_ERR_DEVICE_TIMEOUT = -6
VDN_ERR_DEVICE = -7

VDN_BF16 = 0
VDN_F32 = 1

VDN_PROJ_BF16 = 0
VDN_PROJ_FP8 = 1

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvdn.so")


class VdnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {vdn_error_string(code)} ({code})")


class vdn_shape_t(ctypes.Structure):
    _fields_ = [
        ("F", ctypes.c_int32),
        ("T", ctypes.c_int32),
        ("H", ctypes.c_int32),
        ("d", ctypes.c_int32),
        ("block_frames", ctypes.c_int32),
        ("lambda_", ctypes.c_float),
        ("rms_eps", ctypes.c_float),
        ("dtype", ctypes.c_int32),
        ("off_host", ctypes.POINTER(ctypes.c_int32)),
        ("off_dev", ctypes.POINTER(ctypes.c_int32)),
    ]


_lib = None
_P = ctypes.c_void_p
_SZ = ctypes.c_size_t
_SIGS = {
    "vdn_workspace_bytes": (_SZ, [ctypes.POINTER(vdn_shape_t)]),
    "vdn_hybrid_attn_fwd": (ctypes.c_int, [ctypes.POINTER(vdn_shape_t)] + [_P] * 9 + [_P, _SZ, _P]),
    "vdn_hybrid_attn_fwd_profile": (ctypes.c_int, [ctypes.POINTER(vdn_shape_t)] + [_P] * 9
                                    + [_P, _SZ, _P, ctypes.c_int, ctypes.POINTER(ctypes.c_float)]),
    "vdn_proj_workspace_bytes": (_SZ, [ctypes.POINTER(vdn_shape_t), ctypes.c_int, ctypes.c_int]),
    "vdn_hybrid_attn_branches": (ctypes.c_int, [ctypes.POINTER(vdn_shape_t)] + [_P] * 9
                                 + [_P, _SZ, _P]),
    "vdn_linear": (ctypes.c_int, [_P, _P, _P, _P, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_int, _P, _P]),
    "vdn_quantize_rows_e4m3": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.c_int, _P, _P, _P]),
    "vdn_hybrid_attn_proj_fwd": (ctypes.c_int, [ctypes.POINTER(vdn_shape_t)] + [_P] * 8
                                 + [_P, _P, ctypes.c_int, ctypes.c_int, _P, _P, _SZ, _P]),
    "vdn_fp8_workspace_bytes": (_SZ, [ctypes.POINTER(vdn_shape_t)]),
    "vdn_bsa_fwd_fp8": (ctypes.c_int, [ctypes.POINTER(vdn_shape_t)] + [_P] * 7 + [_P, _SZ, _P]),
    "vdn_hybrid_attn_fwd_fp8": (ctypes.c_int, [ctypes.POINTER(vdn_shape_t)] + [_P] * 9
                                + [_P, _SZ, _P]),
    "vdn_read_images_bytes": (_SZ, [ctypes.POINTER(vdn_shape_t)]),
    "vdn_vda_read_images": (ctypes.c_int, [ctypes.POINTER(vdn_shape_t)] + [_P] * 5 + [_P, _SZ, _P]),
    "vdn_bsa_merge_fwd": (ctypes.c_int, [ctypes.POINTER(vdn_shape_t)] + [_P] * 10 + [_P, _SZ, _P]),
    "vdn_vda_scan": (ctypes.c_int, [ctypes.POINTER(vdn_shape_t)] + [_P] * 8 + [_P, _SZ, _P]),
    "vdn_gate_merge": (ctypes.c_int, [ctypes.POINTER(vdn_shape_t)] + [_P] * 7 + [_P, _SZ, _P]),
    "vdn_bsa_fwd": (ctypes.c_int, [ctypes.POINTER(vdn_shape_t)] + [_P] * 7 + [_P, _SZ, _P]),
    "vdn_pair_audit": (ctypes.c_int, [ctypes.POINTER(vdn_shape_t), _P, _P, _P]),
    "vdn_vda_scan_noalloc": (ctypes.c_int, [ctypes.POINTER(vdn_shape_t)] + [_P] * 8 + [_P]),
    "vdn_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int, _P]),
    "vdn_get_device_error": (ctypes.c_int, []),
    "vdn_error_string": (ctypes.c_char_p, [ctypes.c_int]),
}
EXPORTED = tuple(_SIGS)


def load_library(path: str = LIB_PATH):
    """Load libvdn.so (raises OSError if it is missing: no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise OSError(f"{path} is not built; run `python -m video_diffusion_hybrid_block_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def vdn_error_string(code: int) -> str:
    try:
        return load_library().vdn_error_string(int(code)).decode()
    except OSError:
        return f"error {code}"


def _ptr(t) -> int:
    if t is None:
        return 0
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors passed to the C ABI must be contiguous")
    return t.data_ptr()


def _need(t, count: int, esize: int, name: str):
    """Reject a tensor the kernels would read or write beyond its end: fewer
    elements than the shape needs, a different element size, or host memory.
    Larger tensors are accepted; ints (raw addresses) and None pass through."""
    if t is None or isinstance(t, int):
        return
    if t.numel() < count:
        raise ValueError(f"{name}: {t.numel()} elements, the shape needs {count}")
    if t.element_size() != esize:
        raise ValueError(f"{name}: elements of {t.element_size()} bytes, expected {esize}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")


def _check_acts(shape, q=None, k=None, v=None, kt=None, vt=None, g_s=None, g_l=None, out=None):
    e = 2 if shape.dtype == VDN_BF16 else 4
    act, txt, gate = shape.N * shape.H * shape.d, shape.T * shape.H * shape.d, shape.N * shape.H
    for t, n, name in ((q, act, "q"), (k, act, "k"), (v, act, "v"), (out, act, "out"),
                       (g_s, gate, "g_s"), (g_l, gate, "g_l")):
        _need(t, n, e, name)
    if shape.T > 0:
        _need(kt, txt, e, "kt")
        _need(vt, txt, e, "vt")


def _check_states(shape, read_states=None, text_state=None, fwd_states=None, bwd_states=None):
    dd = shape.H * shape.d * shape.d
    _need(read_states, shape.nb * dd, 4, "read_states")
    _need(text_state, dd, 4, "text_state")
    _need(fwd_states, shape.F * dd, 4, "fwd_states")
    _need(bwd_states, shape.F * dd, 4, "bwd_states")


def _nbytes(workspace, ws_bytes) -> int:
    if ws_bytes is not None:
        return int(ws_bytes)
    if workspace is None or isinstance(workspace, int):
        return 0
    return workspace.numel() * workspace.element_size()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class Shape:
    """Owns a vdn_shape_t plus the host/device frame-offset arrays it points to."""

    def __init__(self, off, T: int, H: int, d: int, block_frames: int = 5,
                 lam: float = 1.0, rms_eps: float = 1e-6, dtype: int = VDN_BF16,
                 device=None):
        self.off_host = torch.as_tensor(off, dtype=torch.int32).contiguous().cpu()
        # device copy read by the kernels; "cpu" only for host-side argument checks
        self.off_dev = self.off_host.clone() if str(device) == "cpu" else self.off_host.to(device or "cuda")
        self.F = len(self.off_host) - 1
        self.N = int(self.off_host[-1])
        self.T, self.H, self.d = int(T), int(H), int(d)
        self.dtype = int(dtype)
        self.block_frames = int(block_frames)
        self.nb = -(-self.F // self.block_frames) if self.block_frames > 0 else 0
        self.c = vdn_shape_t(
            self.F, self.T, self.H, self.d, self.block_frames, float(lam),
            float(rms_eps), int(dtype),
            ctypes.cast(self.off_host.data_ptr(), ctypes.POINTER(ctypes.c_int32)),
            ctypes.cast(self.off_dev.data_ptr(), ctypes.POINTER(ctypes.c_int32)))

    @property
    def ref(self):
        return ctypes.byref(self.c)


def _check(rc: int, where: str):
    if rc != VDN_OK:
        raise VdnError(rc, where)


def vdn_workspace_bytes(shape: Shape) -> int:
    return int(load_library().vdn_workspace_bytes(shape.ref))


def vdn_hybrid_attn_fwd(shape: Shape, q, k, v, kt, vt, g_s, g_l, rms_w, out, workspace,
                        stream=None, ws_bytes=None):
    _check_acts(shape, q, k, v, kt, vt, g_s, g_l, out)
    _need(rms_w, shape.H * shape.d, 4, "rms_w")
    rc = load_library().vdn_hybrid_attn_fwd(
        shape.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(kt), _ptr(vt), _ptr(g_s), _ptr(g_l),
        _ptr(rms_w), _ptr(out), _ptr(workspace), _nbytes(workspace, ws_bytes),
        _stream(stream))
    _check(rc, "vdn_hybrid_attn_fwd")
    return out


PROFILE_GROUPS = ("stage", "gram_inv", "scan", "pack", "softmax_merge")


def vdn_hybrid_attn_fwd_profile(shape: Shape, q, k, v, kt, vt, g_s, g_l, rms_w, out, workspace,
                                iters: int = 10, stream=None, ws_bytes=None) -> dict:
    """Runs the layer `iters` times with CUDA events between its kernels and
    returns the mean ms per layer of each launch group (PROFILE_GROUPS).
    Synchronises the stream (measurement helper)."""
    _check_acts(shape, q, k, v, kt, vt, g_s, g_l, out)
    _need(rms_w, shape.H * shape.d, 4, "rms_w")
    ms = (ctypes.c_float * len(PROFILE_GROUPS))()
    rc = load_library().vdn_hybrid_attn_fwd_profile(
        shape.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(kt), _ptr(vt), _ptr(g_s), _ptr(g_l),
        _ptr(rms_w), _ptr(out), _ptr(workspace), _nbytes(workspace, ws_bytes),
        _stream(stream), int(iters), ms)
    _check(rc, "vdn_hybrid_attn_fwd_profile")
    return dict(zip(PROFILE_GROUPS, (float(x) for x in ms)))


def vdn_vda_scan(shape: Shape, k, v, kt, vt, read_states, text_state, fwd_states, bwd_states,
                 workspace, stream=None, ws_bytes=None):
    _check_acts(shape, k=k, v=v, kt=kt, vt=vt)
    _check_states(shape, read_states, text_state, fwd_states, bwd_states)
    rc = load_library().vdn_vda_scan(
        shape.ref, _ptr(k), _ptr(v), _ptr(kt), _ptr(vt), _ptr(read_states), _ptr(text_state),
        _ptr(fwd_states), _ptr(bwd_states), _ptr(workspace),
        _nbytes(workspace, ws_bytes), _stream(stream))
    _check(rc, "vdn_vda_scan")
    return read_states


def vdn_vda_scan_noalloc(shape: Shape, k, v, kt, vt, read_states, text_state, fwd_states,
                         bwd_states, stream=None):
    """vdn_vda_scan without a workspace argument: the library's built-in
    64 MiB device scratch is used instead (see include/vdn.h for the limit)."""
    _check_acts(shape, k=k, v=v, kt=kt, vt=vt)
    _check_states(shape, read_states, text_state, fwd_states, bwd_states)
    rc = load_library().vdn_vda_scan_noalloc(
        shape.ref, _ptr(k), _ptr(v), _ptr(kt), _ptr(vt), _ptr(read_states), _ptr(text_state),
        _ptr(fwd_states), _ptr(bwd_states), _stream(stream))
    _check(rc, "vdn_vda_scan_noalloc")
    return read_states


def vdn_gate_merge(shape: Shape, q, read_states, o_soft, g_s, g_l, rms_w, out, workspace,
                   stream=None, ws_bytes=None):
    _check_acts(shape, q=q, g_s=g_s, g_l=g_l, out=out)
    _check_states(shape, read_states)
    _need(o_soft, shape.N * shape.H * shape.d, 2, "o_soft")
    _need(rms_w, shape.H * shape.d, 4, "rms_w")
    rc = load_library().vdn_gate_merge(
        shape.ref, _ptr(q), _ptr(read_states), _ptr(o_soft), _ptr(g_s), _ptr(g_l), _ptr(rms_w),
        _ptr(out), _ptr(workspace), _nbytes(workspace, ws_bytes),
        _stream(stream))
    _check(rc, "vdn_gate_merge")
    return out


def vdn_bsa_fwd(shape: Shape, q, k, v, kt, vt, o_soft, lse, workspace, stream=None,
                ws_bytes=None):
    _check_acts(shape, q, k, v, kt, vt)
    _need(o_soft, shape.N * shape.H * shape.d, 2, "o_soft")
    _need(lse, shape.H * shape.N, 4, "lse")
    rc = load_library().vdn_bsa_fwd(
        shape.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(kt), _ptr(vt), _ptr(o_soft), _ptr(lse),
        _ptr(workspace), _nbytes(workspace, ws_bytes), _stream(stream))
    _check(rc, "vdn_bsa_fwd")
    return o_soft


def vdn_pair_audit(shape: Shape, soft_pairs, lin_pairs, stream=None):
    _need(soft_pairs, shape.F * (shape.F + 1), 8, "soft_pairs")
    _need(lin_pairs, shape.F * shape.F, 8, "lin_pairs")
    rc = load_library().vdn_pair_audit(shape.ref, _ptr(soft_pairs), _ptr(lin_pairs),
                                       _stream(stream))
    _check(rc, "vdn_pair_audit")
    return soft_pairs, lin_pairs


def vdn_selftest_wait_timeout(limit_ns: int, tmem_cols: int = 0, stream=None):
    """Launches the bounded-wait failure check (see include/vdn.h); the
    timeout is then reported by vdn_get_device_error()."""
    rc = load_library().vdn_selftest_wait_timeout(int(limit_ns), int(tmem_cols), _stream(stream))
    _check(rc, "vdn_selftest_wait_timeout")


def vdn_get_device_error() -> int:
    return int(load_library().vdn_get_device_error())


# ------------------------------------------ layer split at the read states ---

def vdn_read_images_bytes(shape: Shape) -> int:
    return int(load_library().vdn_read_images_bytes(shape.ref))


def vdn_vda_read_images(shape: Shape, k, v, kt, vt, rimg, workspace, stream=None, ws_bytes=None):
    """Linear branch up to the packed read-state tiles (nb * H tiles of 32 KB)."""
    _check_acts(shape, k=k, v=v, kt=kt, vt=vt)
    _need(rimg, vdn_read_images_bytes(shape), 1, "rimg")
    rc = load_library().vdn_vda_read_images(
        shape.ref, _ptr(k), _ptr(v), _ptr(kt), _ptr(vt), _ptr(rimg), _ptr(workspace),
        _nbytes(workspace, ws_bytes), _stream(stream))
    _check(rc, "vdn_vda_read_images")
    return rimg


def vdn_bsa_merge_fwd(shape: Shape, q, k, v, kt, vt, g_s, g_l, rms_w, rimg, out, workspace,
                      stream=None, ws_bytes=None):
    """Softmax branch + fused readout / RMSNorm / gated merge on given read-state tiles."""
    _check_acts(shape, q, k, v, kt, vt, g_s, g_l, out)
    _need(rms_w, shape.H * shape.d, 4, "rms_w")
    _need(rimg, vdn_read_images_bytes(shape), 1, "rimg")
    rc = load_library().vdn_bsa_merge_fwd(
        shape.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(kt), _ptr(vt), _ptr(g_s), _ptr(g_l),
        _ptr(rms_w), _ptr(rimg), _ptr(out), _ptr(workspace), _nbytes(workspace, ws_bytes),
        _stream(stream))
    _check(rc, "vdn_bsa_merge_fwd")
    return out


# --------------------------------------------------- e4m3 softmax branch ---

def vdn_fp8_workspace_bytes(shape: Shape) -> int:
    return int(load_library().vdn_fp8_workspace_bytes(shape.ref))


def alloc_fp8_workspace(shape: Shape, device=None) -> torch.Tensor:
    n = vdn_fp8_workspace_bytes(shape)
    if n == 0:
        raise VdnError(VDN_ERR_UNSUPPORTED, "vdn_fp8_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def vdn_bsa_fwd_fp8(shape: Shape, q, k, v, kt, vt, o_soft, lse, workspace, stream=None,
                    ws_bytes=None):
    _check_acts(shape, q, k, v, kt, vt)
    _need(o_soft, shape.N * shape.H * shape.d, 2, "o_soft")
    _need(lse, shape.H * shape.N, 4, "lse")
    rc = load_library().vdn_bsa_fwd_fp8(
        shape.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(kt), _ptr(vt), _ptr(o_soft), _ptr(lse),
        _ptr(workspace), _nbytes(workspace, ws_bytes), _stream(stream))
    _check(rc, "vdn_bsa_fwd_fp8")
    return o_soft


def vdn_hybrid_attn_fwd_fp8(shape: Shape, q, k, v, kt, vt, g_s, g_l, rms_w, out, workspace,
                            stream=None, ws_bytes=None):
    _check_acts(shape, q, k, v, kt, vt, g_s, g_l, out)
    _need(rms_w, shape.H * shape.d, 4, "rms_w")
    rc = load_library().vdn_hybrid_attn_fwd_fp8(
        shape.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(kt), _ptr(vt), _ptr(g_s), _ptr(g_l),
        _ptr(rms_w), _ptr(out), _ptr(workspace), _nbytes(workspace, ws_bytes), _stream(stream))
    _check(rc, "vdn_hybrid_attn_fwd_fp8")
    return out


# ------------------------------------------------ per-branch projections ---

def _proj_K(shape: Shape) -> int:
    return 2 * shape.H * shape.d


def vdn_proj_workspace_bytes(shape: Shape, D: int, precision: int) -> int:
    return int(load_library().vdn_proj_workspace_bytes(shape.ref, int(D), int(precision)))


def alloc_proj_workspace(shape: Shape, D: int, precision: int, device=None) -> torch.Tensor:
    n = vdn_proj_workspace_bytes(shape, D, precision)
    if n == 0:
        raise VdnError(VDN_ERR_INVALID_ARG, "vdn_proj_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def vdn_hybrid_attn_branches(shape: Shape, q, k, v, kt, vt, g_s, g_l, rms_w, branches, workspace,
                             stream=None, ws_bytes=None):
    _check_acts(shape, q, k, v, kt, vt, g_s, g_l)
    _need(rms_w, shape.H * shape.d, 4, "rms_w")
    _need(branches, shape.N * _proj_K(shape), 2, "branches")
    rc = load_library().vdn_hybrid_attn_branches(
        shape.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(kt), _ptr(vt), _ptr(g_s), _ptr(g_l),
        _ptr(rms_w), _ptr(branches), _ptr(workspace), _nbytes(workspace, ws_bytes),
        _stream(stream))
    _check(rc, "vdn_hybrid_attn_branches")
    return branches


def vdn_linear(a, a_scale, w, w_scale, M: int, K: int, D: int, precision: int, y, stream=None):
    """y [M, D] bf16 = a [M, K] w [D, K]^T (e4m3 codes with row scales for
    VDN_PROJ_FP8)."""
    es = 1 if precision == VDN_PROJ_FP8 else 2
    _need(a, M * K, es, "a")
    _need(w, D * K, es, "w")
    _need(y, M * D, 2, "y")
    if precision == VDN_PROJ_FP8:
        _need(a_scale, M, 4, "a_scale")
        _need(w_scale, D, 4, "w_scale")
    rc = load_library().vdn_linear(_ptr(a), _ptr(a_scale), _ptr(w), _ptr(w_scale), int(M), int(K),
                                   int(D), int(precision), _ptr(y), _stream(stream))
    _check(rc, "vdn_linear")
    return y


def vdn_quantize_rows_e4m3(x, rows: int, K: int, codes, scales, stream=None):
    _need(x, rows * K, 2, "x")
    _need(codes, rows * K, 1, "codes")
    _need(scales, rows, 4, "scales")
    rc = load_library().vdn_quantize_rows_e4m3(_ptr(x), int(rows), int(K), _ptr(codes),
                                               _ptr(scales), _stream(stream))
    _check(rc, "vdn_quantize_rows_e4m3")
    return codes, scales


def vdn_hybrid_attn_proj_fwd(shape: Shape, q, k, v, kt, vt, g_s, g_l, rms_w, w_o, w_scale, D: int,
                             precision: int, y, workspace, stream=None, ws_bytes=None):
    _check_acts(shape, q, k, v, kt, vt, g_s, g_l)
    _need(rms_w, shape.H * shape.d, 4, "rms_w")
    _need(w_o, D * _proj_K(shape), 1 if precision == VDN_PROJ_FP8 else 2, "w_o")
    if precision == VDN_PROJ_FP8:
        _need(w_scale, D, 4, "w_scale")
    _need(y, shape.N * D, 2, "y")
    rc = load_library().vdn_hybrid_attn_proj_fwd(
        shape.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(kt), _ptr(vt), _ptr(g_s), _ptr(g_l),
        _ptr(rms_w), _ptr(w_o), _ptr(w_scale), int(D), int(precision), _ptr(y), _ptr(workspace),
        _nbytes(workspace, ws_bytes), _stream(stream))
    _check(rc, "vdn_hybrid_attn_proj_fwd")
    return y


def alloc_workspace(shape: Shape, device=None) -> torch.Tensor:
    n = vdn_workspace_bytes(shape)
    if n == 0:
        raise VdnError(VDN_ERR_INVALID_ARG, "vdn_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")
