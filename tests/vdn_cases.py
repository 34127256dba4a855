"""Shared helpers for the GPU tests: run the CUDA library through its C ABI on
seeded inputs and compare with the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import vdn_synth as S

# Tolerances of the layer (bf16 inputs, fp32 accumulation):
OUT_REL_L2 = 2e-2
OUT_MAX_ABS = 5e-2
STATE_REL_FRO = 1e-2


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def max_abs(a, b) -> float:
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)))) if np.size(a) else 0.0


def device_inputs(inp: dict, device="cuda") -> dict:
    """torch tensors of the generator's arrays in the workload's dtype."""
    dt = torch.bfloat16 if inp["dtype"] == "bf16" else torch.float32
    out = {}
    for key in ("q", "k", "v", "kt", "vt", "g_s", "g_l"):
        out[key] = torch.from_numpy(np.ascontiguousarray(inp[key])).to(device=device, dtype=dt)
    out["rms_w"] = torch.from_numpy(np.ascontiguousarray(inp["rms_w"])).to(device)
    return out


def make_shape(inp: dict, device="cuda"):
    import video_diffusion_hybrid_block_b200 as V
    return V.Shape(inp["off"], inp["T"], inp["H"], inp["d"], inp["block_frames"], inp["lam"],
                   inp["eps"], V.VDN_BF16 if inp["dtype"] == "bf16" else V.VDN_F32,
                   device=device)


def run_layer(inp: dict, dev: dict | None = None):
    import video_diffusion_hybrid_block_b200 as V
    dev = dev or device_inputs(inp)
    shape = make_shape(inp)
    ws = V.alloc_workspace(shape)
    out = torch.empty_like(dev["q"])
    V.vdn_hybrid_attn_fwd(shape, dev["q"], dev["k"], dev["v"], dev["kt"], dev["vt"], dev["g_s"],
                          dev["g_l"], dev["rms_w"], out, ws)
    torch.cuda.synchronize()
    assert V.vdn_get_device_error() == 0
    return out


def run_bsa(inp: dict, dev: dict | None = None, want_lse=False):
    import video_diffusion_hybrid_block_b200 as V
    dev = dev or device_inputs(inp)
    shape = make_shape(inp)
    ws = V.alloc_workspace(shape)
    o = torch.empty(dev["q"].shape, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((inp["H"], inp["N"]), dtype=torch.float32, device="cuda") if want_lse else None
    V.vdn_bsa_fwd(shape, dev["q"], dev["k"], dev["v"], dev["kt"], dev["vt"], o, lse, ws)
    torch.cuda.synchronize()
    assert V.vdn_get_device_error() == 0
    return o, lse


def run_scan(inp: dict, dev: dict | None = None, per_frame=True):
    import video_diffusion_hybrid_block_b200 as V
    dev = dev or device_inputs(inp)
    shape = make_shape(inp)
    ws = V.alloc_workspace(shape)
    F, H, d = inp["F"], inp["H"], inp["d"]
    nb = O.num_blocks(F, inp["block_frames"])
    R = torch.empty((nb, H, d, d), dtype=torch.float32, device="cuda")
    St = torch.empty((H, d, d), dtype=torch.float32, device="cuda")
    Sf = torch.zeros((F, H, d, d), dtype=torch.float32, device="cuda") if per_frame else None
    Sb = torch.zeros((F, H, d, d), dtype=torch.float32, device="cuda") if per_frame else None
    V.vdn_vda_scan(shape, dev["k"], dev["v"], dev["kt"], dev["vt"], R, St, Sf, Sb, ws)
    torch.cuda.synchronize()
    assert V.vdn_get_device_error() == 0
    return R, St, Sf, Sb


def run_audit(inp: dict):
    import video_diffusion_hybrid_block_b200 as V
    shape = make_shape(inp)
    F = inp["F"]
    soft = torch.empty((F, F + 1), dtype=torch.int64, device="cuda")
    lin = torch.empty((F, F), dtype=torch.int64, device="cuda")
    V.vdn_pair_audit(shape, soft, lin)
    torch.cuda.synchronize()
    return soft.cpu().numpy(), lin.cpu().numpy()


def sample_rows(inp: dict, n: int, seed: int = 0) -> np.ndarray:
    """Sorted random query rows, always including the first and last row of
    every block and of the clip."""
    N = inp["N"]
    off = inp["off"]
    bf = inp["block_frames"]
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(N, size=min(n, N), replace=False).tolist())
    for b in range(O.num_blocks(inp["F"], bf)):
        q0, q1 = int(off[bf * b]), int(off[min(bf * b + bf, inp["F"])])
        if q1 > q0:
            rows.update({q0, q1 - 1, min(q0 + 127, q1 - 1), min(q0 + 128, q1 - 1)})
    return np.array(sorted(rows))


def mid_case(seed=0, d=128, dtype="bf16", T=40, F=12, n=150, H=2, bf=5):
    """A case the oracle finishes in seconds that spans several 128-row tiles
    per block with a ragged tail, and partial key tiles."""
    return S.make_inputs_from(F, [n] * F, T, H, d, dtype=dtype, seed=seed)
