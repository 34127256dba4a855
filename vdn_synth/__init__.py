"""Seeded synthetic inputs for the VideoDeltaNet hybrid attention layer.

This module only draws random tensors with the shapes and value distributions
of the workloads; it holds none of the layer's arithmetic. Both the CPU
oracle (``oracle/``) and the CUDA path (``video_diffusion_hybrid_block_b200``)
consume what it returns, and neither imports the other.

Workloads (frame grid, token counts, head counts) are synthetic stand-ins for
the clips the pages describe (somewhat more than ten latent frames, each with
more than a thousand latent tokens, plus text tokens) at 768p (VDN-MiniMax-H3 on openi.cn, section
"技术原理：局部精确、远程压缩"); the pages name no dataset or benchmark suite.

Recipe (numpy PCG64 ``default_rng(seed)``, all draws float32, in this order):
q, k, v, kt, vt, g_s, g_l.
* q, k, v ~ N(0, 1) with shape [N, H, d]; kt, vt ~ N(0, 1) with shape [T, H, d].
* k and kt are L2-normalised along d (in float32) before any rounding.
* "hi-res": k is drawn per frame and head as A @ B + 0.1 E with
  A ~ N(0,1) [n, 16], B ~ N(0,1)/4 [16, d], E ~ N(0,1) [n, d], then normalised.
* "vda-stress": frames f with f % 7 == 6 hold 64 tokens instead of 252, and
  frames f with f % 11 == 10 have v = 0.
* gate logits g_s, g_l ~ N(0, 1) with shape [N, H]; RMSNorm weight = 1 [H, d].
* bf16 workloads round every float input to bf16 (round to nearest even);
  the returned float32 arrays then hold exactly the bf16 values.
* make_inputs_device: the same distributions drawn on the device with
  torch's Philox generator (for shapes too large for the host).
* output-projection weights (make_proj_weight): w_o [D, 2 H d] ~
  N(0, 1) / sqrt(2 H d), default_rng(seed + 1000), bf16.
"""
from __future__ import annotations

import numpy as np

BLOCK_FRAMES = 5
LAMBDA = 1.0
RMS_EPS = 1e-6

# name -> workload description. "tokens" is tokens per frame (frame grid h x w).
CONFIGS = {
    "tiny": dict(F=10, grid=(4, 6), T=8, H=2, d=32, dtype="f32"),
    "tiny-scan": dict(F=20, grid=(4, 6), T=8, H=2, d=32, dtype="f32"),
    "pages-scale": dict(F=15, grid=(24, 42), T=256, H=32, d=128, dtype="bf16"),
    "long-clip": dict(F=30, grid=(24, 42), T=256, H=32, d=128, dtype="bf16"),
    "hi-res": dict(F=20, grid=(32, 56), T=512, H=24, d=128, dtype="bf16",
                   k_lowrank=16),
    "vda-stress": dict(F=60, grid=(12, 21), T=128, H=32, d=128, dtype="bf16",
                       short_every=7, short_n=64, zero_v_every=11),
}

# The five workloads in the order they are usually listed.
CONFIG_ORDER = ["tiny", "pages-scale", "long-clip", "hi-res", "vda-stress"]


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); float32 out."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The bf16 bit patterns (uint16) of float32 values that are already bf16."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def frame_sizes(cfg: dict) -> np.ndarray:
    F = cfg["F"]
    n = cfg["grid"][0] * cfg["grid"][1]
    sizes = np.full(F, n, dtype=np.int64)
    if "short_every" in cfg:
        e = cfg["short_every"]
        sizes[np.arange(F) % e == e - 1] = cfg["short_n"]
    return sizes


def frame_offsets(sizes) -> np.ndarray:
    sizes = np.asarray(sizes, dtype=np.int64)
    off = np.zeros(len(sizes) + 1, dtype=np.int64)
    off[1:] = np.cumsum(sizes)
    return off.astype(np.int32)


def _l2n(x: np.ndarray) -> np.ndarray:
    nrm = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / np.maximum(nrm, 1e-12)).astype(np.float32)


def make_inputs_from(F, sizes, T, H, d, dtype="bf16", seed=0, k_lowrank=None,
                     zero_v_every=None, rms_w=None):
    """Draw one layer's inputs for an explicit frame-size list."""
    rng = np.random.default_rng(seed)
    sizes = np.asarray(sizes, dtype=np.int64)
    assert len(sizes) == F
    off = frame_offsets(sizes)
    N = int(off[-1])
    q = rng.standard_normal((N, H, d), dtype=np.float32)
    if k_lowrank:
        k = np.empty((N, H, d), dtype=np.float32)
        for f in range(F):
            n = int(sizes[f])
            A = rng.standard_normal((H, n, k_lowrank), dtype=np.float32)
            B = rng.standard_normal((H, k_lowrank, d), dtype=np.float32) / 4
            E = rng.standard_normal((H, n, d), dtype=np.float32)
            kf = np.matmul(A, B) + np.float32(0.1) * E          # [H, n, d]
            k[off[f]:off[f + 1]] = kf.transpose(1, 0, 2)
    else:
        k = rng.standard_normal((N, H, d), dtype=np.float32)
    v = rng.standard_normal((N, H, d), dtype=np.float32)
    kt = rng.standard_normal((T, H, d), dtype=np.float32)
    vt = rng.standard_normal((T, H, d), dtype=np.float32)
    g_s = rng.standard_normal((N, H), dtype=np.float32)
    g_l = rng.standard_normal((N, H), dtype=np.float32)
    k = _l2n(k)
    kt = _l2n(kt)
    if zero_v_every:
        e = zero_v_every
        for f in range(F):
            if f % e == e - 1:
                v[off[f]:off[f + 1]] = 0.0
    if rms_w is None:
        rms_w = np.ones((H, d), dtype=np.float32)
    out = dict(q=q, k=k, v=v, kt=kt, vt=vt, g_s=g_s, g_l=g_l)
    if dtype == "bf16":
        out = {key: bf16_round(val) for key, val in out.items()}
    out.update(rms_w=np.asarray(rms_w, dtype=np.float32), off=off, F=F, T=T,
               H=H, d=d, N=N, dtype=dtype, block_frames=BLOCK_FRAMES,
               lam=LAMBDA, eps=RMS_EPS)
    return out


def make_proj_weight(H: int, d: int, D: int | None = None, seed: int = 0) -> np.ndarray:
    """Synthetic output-projection weight w_o [D, 2 H d] (D = H d by default):
    N(0, 1) / sqrt(2 H d) float32 from default_rng(seed + 1000), rounded to
    bf16. There are no trained weights; this only sets shapes and scale."""
    D = H * d if D is None else D
    rng = np.random.default_rng(seed + 1000)
    w = rng.standard_normal((D, 2 * H * d), dtype=np.float32) / np.float32(np.sqrt(2 * H * d))
    return bf16_round(w)


def make_inputs_device(F, sizes, T, H, d, seed=0, device="cuda"):
    """Inputs too large to draw on the host, drawn on the device: torch's
    Philox generator seeded with `seed`, float32 draws in the order q, k, v,
    kt, vt, g_s, g_l (N(0, 1); k and kt L2-normalised), rounded to bf16.
    Returns torch tensors plus the frame offsets and the layer constants."""
    import torch
    sizes = np.asarray(sizes, dtype=np.int64)
    off = frame_offsets(sizes)
    N = int(off[-1])
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = {}
    for key, shape in (("q", (N, H, d)), ("k", (N, H, d)), ("v", (N, H, d)), ("kt", (T, H, d)),
                       ("vt", (T, H, d)), ("g_s", (N, H)), ("g_l", (N, H))):
        x = torch.empty(shape, dtype=torch.bfloat16, device=device)
        # draw in row chunks so no full-size float32 copy is ever held
        rows = max(1, (1 << 26) // max(1, int(np.prod(shape[1:]))))
        for r0 in range(0, shape[0], rows):
            r1 = min(shape[0], r0 + rows)
            y = torch.randn((r1 - r0,) + shape[1:], generator=g, device=device,
                            dtype=torch.float32)
            if key in ("k", "kt"):
                y = y / torch.clamp(y.norm(dim=-1, keepdim=True), min=1e-12)
            x[r0:r1] = y.to(torch.bfloat16)
        out[key] = x
    out["rms_w"] = torch.ones((H, d), dtype=torch.float32, device=device)
    out.update(off=off, F=F, T=T, H=H, d=d, N=N, dtype="bf16", block_frames=BLOCK_FRAMES,
               lam=LAMBDA, eps=RMS_EPS)
    return out


def make_inputs(name: str, seed: int = 0) -> dict:
    """Inputs of one named workload (see CONFIGS)."""
    cfg = CONFIGS[name]
    return make_inputs_from(cfg["F"], frame_sizes(cfg), cfg["T"], cfg["H"],
                            cfg["d"], dtype=cfg["dtype"], seed=seed,
                            k_lowrank=cfg.get("k_lowrank"),
                            zero_v_every=cfg.get("zero_v_every"))
