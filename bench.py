"""Benchmark of the hybrid attention layer forward on B200.

One step = one layer forward (softmax branch, VDA Grams/inverses, both
scans, read-state packing, softmax kernel with the fused readout + RMSNorm +
gated merge). The timed steps run through vdn_hybrid_attn_fwd_profile, the
same launches as vdn_hybrid_attn_fwd with CUDA events between the layer's
kernels, so the roofline's kernel time comes from the timed region itself. The headline line runs the hi-res workload, the
largest that fits one GPU: F=20 latent frames of 32x56=1792 tokens (35840
video tokens), T=512 text tokens, H=24 heads, d=128, bf16, low-rank keys,
seed 0. Inputs are synthetic (vdn_synth).

Prints one JSON line (rank 0). `value` is layer TFLOP/s (algorithmic FLOP of
the work the method needs: softmax over unmasked (query, key) pairs, VDA
Grams / inverses / scan products of the frames some read state depends on,
readout) summed over ranks; `ms_per_step` is the max over ranks. The line
also carries `workloads`: ms/layer, TFLOP/s, per-kernel times and roofline
fractions on every workload (the softmax kernel against the bf16 tensor peak,
the VDA kernels and the standalone merge against HBM bandwidth).
`--impl reference` times the fp64 CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "hybrid-attn layer fwd ms and TFLOP/s (frac. of bf16 peak), 1×B200"
HEADLINE = "hi-res"
WORKLOADS = ["tiny", "pages-scale", "long-clip", "hi-res", "vda-stress"]
L2_BYTES = 126 * 2 ** 20
REF_ROWS = 2048          # query rows per reference-arm step (one head)
CPU_BASELINE_HEADS = 24  # reference-arm steps in the GPU line's cpu_baseline
REST_S = 1.0             # idle time before each measurement (power back to idle)


# --------------------------------------------------------------- work model --

def needed_frames(F: int, bf: int):
    """Frames the read states depend on (the library skips the others when
    no per-frame states are requested): the forward scan runs frames
    1..fwd_last, the backward scan frames bwd_first..F-2; every needed frame
    gets one Gram + inverse, each scan step one d x d x d product."""
    fwd_last, bwd_first = 0, F - 1
    for b in range(-(-F // bf)):
        w0 = bf * max(b - 1, 0)
        w1 = min(bf * (b + 2), F) - 1
        fwd_last = max(fwd_last, max(w0 - 1, 0))
        bwd_first = min(bwd_first, min(w1 + 1, F - 1))
    frames = list(range(1, fwd_last + 1)) + list(range(max(bwd_first, fwd_last + 1), F - 1))
    return dict(frames=frames, steps_fwd=1 + fwd_last, steps_bwd=1 + (F - 1 - bwd_first))


def layer_flops(inp: dict, soft_pairs: np.ndarray) -> dict:
    """Algorithmic FLOP of one layer forward.

    softmax: 4 d H (video pairs + N T) over unmasked pairs (QK^T and PV);
    readout: 2 N d^2 H; VDA, over the text and the frames some read state
    depends on: Grams 4 rows d^2 H (K^T K and K^T V), one d x d inverse per
    matrix and head (2 d^3), one 2 d^3 product per scan step and head."""
    N, T, H, d, F = inp["N"], inp["T"], inp["H"], inp["d"], inp["F"]
    off = np.asarray(inp["off"], np.int64)
    nf = needed_frames(F, inp.get("block_frames", 5))
    rows = T + sum(int(off[f + 1] - off[f]) for f in nf["frames"])
    n_mat = 1 + len(nf["frames"])
    video_pairs = int(soft_pairs[:, :F].sum())
    softmax = 4.0 * d * H * (video_pairs + N * T)
    readout = 2.0 * N * d * d * H
    grams = 4.0 * rows * d * d * H
    inverses = 2.0 * d ** 3 * n_mat * H
    scans = 2.0 * d ** 3 * (nf["steps_fwd"] + nf["steps_bwd"]) * H
    vda = grams + inverses + scans
    return dict(softmax=softmax, readout=readout, grams=grams, inverses=inverses, scans=scans,
                vda=vda, total=softmax + readout + vda, gram_rows=rows, n_mat=n_mat,
                scan_steps=nf["steps_fwd"] + nf["steps_bwd"])


def kernel_bytes(inp: dict, fl: dict) -> dict:
    """Algorithmic HBM bytes per launch of the HBM-bound kernels (d = 128 bf16):
    Gram + inverse reads k, v of its rows once and writes C and W once; a scan
    step reads W_f and C_f once and the scans write the two read-state halves;
    packing reads both halves and writes one bf16 tile per (block, head); the
    standalone readout + merge reads q, o_soft, gates and R_b and writes out."""
    N, T, H, d, F = inp["N"], inp["T"], inp["H"], inp["d"], inp["F"]
    nb = -(-F // inp["block_frames"])
    mat = 128 * 128 * 4
    return dict(
        gram_inv=2 * fl["gram_rows"] * H * d * 2 + 2 * fl["n_mat"] * H * mat,
        scan=fl["scan_steps"] * H * 2 * mat + 2 * nb * H * mat,
        pack=2 * nb * H * mat + nb * H * 128 * 128 * 2,
        gate_merge=3 * N * H * d * 2 + 2 * N * H * 2 + nb * H * d * d * 4,
    )


def workload_desc(name: str) -> str:
    import vdn_synth as S
    c = S.CONFIGS[name]
    extra = ""
    if c.get("k_lowrank"):
        extra = f", keys rank {c['k_lowrank']} + 0.1 noise per frame"
    if c.get("short_every"):
        extra = (f", frames f%{c['short_every']}=={c['short_every'] - 1} hold {c['short_n']} "
                 f"tokens, frames f%{c['zero_v_every']}=={c['zero_v_every'] - 1} have v=0")
    return (f"{name}: F={c['F']} latent frames, {c['grid'][0]}x{c['grid'][1]} tokens/frame, "
            f"T={c['T']}, H={c['H']}, d={c['d']}, {c['dtype']}{extra}")


def input_bytes(inp: dict) -> int:
    e = 2 if inp["dtype"] == "bf16" else 4
    return (3 * inp["N"] + 2 * inp["T"]) * inp["H"] * inp["d"] * e + 2 * inp["N"] * inp["H"] * e


def l2_note(nbytes: int) -> str:
    if nbytes > L2_BYTES:
        return f"inputs {nbytes / 2 ** 20:.0f} MiB > 126 MB L2; no flush between steps"
    return "inputs fit in the 126 MB L2: L2 flushed (256 MiB write) before every timed step"


def config_of(name: str, inp: dict, fl: dict, world: int) -> dict:
    """The `config` object, identical for the CUDA and the reference arm."""
    return {"workload": workload_desc(name), "F": inp["F"],
            "tokens_per_frame": int(inp["N"] // inp["F"]), "N": inp["N"], "T": inp["T"],
            "H": inp["H"], "d": inp["d"], "layer_tflop": round(fl["total"] / 1e12, 4),
            "softmax_tflop": round(fl["softmax"] / 1e12, 4),
            "parallelism": f"replicas x{world}", "l2": l2_note(input_bytes(inp))}


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return dict(bf16_tflops=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    hbm_gbs=float(p["hbm_gbs"]), source="measured")
    return dict(bf16_tflops=1590.0, bf16_sustained=1400.0, hbm_gbs=6650.0, source="fallback")


def bsa_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("k_bsa_fwd.cuh", "layer_plan.cuh", "sm100_ptx.cuh"):
        with open(os.path.join(ROOT, "video_diffusion_hybrid_block_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the merged softmax kernel from the committed
    ncu summary, if it was taken on the current kernel source and workload."""
    path = os.path.join(ROOT, "profiles", "bsa_fwd_merge_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        rec = json.load(fh)
    if rec.get("source_hash") != bsa_source_hash() or rec.get("workload") != workload:
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and clock-event reasons of the GPU this process runs on, read
    (never set) while a timed region runs. NVML is polled every 5 ms from a
    thread; without NVML, nvidia-smi samples at its 200 ms floor. The device
    is found by its UUID, so the samples come from this process's GPU
    whatever CUDA_VISIBLE_DEVICES maps. Samples flagged GPU-idle are left
    out of the median (a region can hold idle pauses)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # clock-event reason bits of NVML's public header
    IDLE = 0x1
    REASONS = (("hw_slowdown", 0x8 | 0x80), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))
    PERIOD_S = 0.005

    def __init__(self, device: int):
        self.device = device
        self.samples = []  # (sm_mhz, sm_max_mhz, reason bits)
        self.proc = None
        self.path = None
        self.thread = None
        self.stop = None
        self.source = None

    def _uuid(self):
        try:
            import torch
            return "GPU-" + str(torch.cuda.get_device_properties(self.device).uuid)
        except Exception:
            return None

    def _nvml_poll(self, nv, h, ready):
        clk_sm = nv.NVML_CLOCK_SM
        reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        smax = nv.nvmlDeviceGetMaxClockInfo(h, clk_sm)
        while True:
            self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, clk_sm)), float(smax),
                                 int(reasons(h))))
            ready.set()
            if self.stop.wait(self.PERIOD_S):
                return

    def __enter__(self):
        import threading
        uuid = self._uuid()
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByUUID(uuid) if uuid else \
                nv.nvmlDeviceGetHandleByIndex(self.device)
            self.stop, ready = threading.Event(), threading.Event()
            self.thread = threading.Thread(target=self._nvml_poll, args=(nv, h, ready),
                                           daemon=True)
            self.thread.start()
            ready.wait(1.0)
            self.source = f"nvml every {self.PERIOD_S * 1e3:.0f} ms"
            return self
        except Exception:
            self.thread = None
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={uuid or self.device}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi every 200 ms"
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def _read_smi(self):
        if not (self.path and os.path.exists(self.path)):
            return
        names = dict(self.REASONS)
        with open(self.path) as fh:
            for line in fh:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 9 or not p[1].replace(".", "").isdigit():
                    continue
                bits = 0
                for i, n in enumerate(("hw_slowdown", "hw_thermal_slowdown",
                                       "sw_thermal_slowdown", "sw_power_cap")):
                    if p[5 + i] == "Active":
                        bits |= names[n]
                smax = float(p[2]) if p[2].replace(".", "").isdigit() else 0.0
                self.samples.append((float(p[1]), smax, bits))
        os.unlink(self.path)
        self.path = None

    def summary(self) -> dict:
        self._read_smi()
        return summarize_clock_samples(self.samples, self.IDLE, self.REASONS, self.source)


def summarize_clock_samples(samples, idle_bit: int, reasons, source) -> dict:
    """Median, mean and lowest SM clock over the busy samples, the max clock
    and every slowdown reason seen in any busy sample."""
    if not samples:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
    busy = [s for s in samples if not s[2] & idle_bit] or samples
    seen = sorted({n for _, _, b in busy for n, m in reasons if b & m})
    clk = [s[0] for s in busy]
    return {"sm_mhz": statistics.median(clk), "sm_mhz_mean": round(statistics.fmean(clk), 1),
            "sm_mhz_min": min(clk), "sm_max_mhz": max(s[1] for s in samples), "reasons": seen,
            "samples": len(busy), "idle_samples": len(samples) - len(busy), "source": source}


def max_over_ranks(dist, x: float, device) -> float:
    """The largest of the ranks' values (timing is the max over ranks); dist
    is torch.distributed or None for a single process. Every rank calls it at
    the same point."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world: int, flop_per_replica: float, ms: float) -> float:
    """TFLOP/s of N independent replicas finishing in the max-over-ranks time."""
    return world * flop_per_replica / (ms * 1e-3) / 1e12


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def cores_used() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


# ------------------------------------------------------------- CUDA arm -----

class Workload:
    """One workload's inputs on the device plus the buffers the entry points need."""

    def __init__(self, name: str, V, torch):
        import vdn_synth as S
        self.name = name
        self.inp = inp = S.make_inputs(name, seed=0)
        self.dt = torch.bfloat16 if inp["dtype"] == "bf16" else torch.float32
        self.host = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to(self.dt)
                     for k in ("q", "k", "v", "kt", "vt", "g_s", "g_l")}
        self.dev = {k: t.to("cuda") for k, t in self.host.items()}
        self.rms_w = torch.from_numpy(inp["rms_w"]).cuda()
        self.shape = V.Shape(inp["off"], inp["T"], inp["H"], inp["d"], inp["block_frames"],
                             inp["lam"], inp["eps"],
                             V.VDN_BF16 if inp["dtype"] == "bf16" else V.VDN_F32)
        self.ws = V.alloc_workspace(self.shape)
        self.out = torch.empty_like(self.dev["q"])
        soft = torch.empty((inp["F"], inp["F"] + 1), dtype=torch.int64, device="cuda")
        lin = torch.empty((inp["F"], inp["F"]), dtype=torch.int64, device="cuda")
        V.vdn_pair_audit(self.shape, soft, lin)
        self.fl = layer_flops(inp, soft.cpu().numpy())
        self.bytes = kernel_bytes(inp, self.fl)
        self.flush = input_bytes(inp) <= L2_BYTES

    def layer(self, V, stream, dev=None, out=None):
        d = dev or self.dev
        V.vdn_hybrid_attn_fwd(self.shape, d["q"], d["k"], d["v"], d["kt"], d["vt"], d["g_s"],
                              d["g_l"], self.rms_w, out if out is not None else self.out, self.ws,
                              stream)


def timed_layers(V, w: Workload, stream, steps: int) -> dict:
    """`steps` back-to-back layers through vdn_hybrid_attn_fwd_profile (at
    most 256 per call): mean ms per layer of each kernel group, measured with
    CUDA events between the layer's kernels on its stream; their sum is the
    layer's device time."""
    tot, done = {}, 0
    while done < steps:
        n = min(256, steps - done)
        k = V.vdn_hybrid_attn_fwd_profile(w.shape, w.dev["q"], w.dev["k"], w.dev["v"],
                                          w.dev["kt"], w.dev["vt"], w.dev["g_s"], w.dev["g_l"],
                                          w.rms_w, w.out, w.ws, iters=n, stream=stream)
        for g, t in k.items():
            tot[g] = tot.get(g, 0.0) + t * n
        done += n
    return {g: t / steps for g, t in tot.items()}


def time_launches(torch, stream, fn, n: int, flush=None) -> float:
    """Mean ms of `fn` over n launches, CUDA events on `stream`. With `flush`
    (a >L2 buffer), each launch is timed alone after overwriting L2."""
    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n
    tot = 0.0
    for _ in range(n):
        flush.add_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        tot += e0.elapsed_time(e1)
    return tot / n


def workload_report(V, torch, w: Workload, stream, steps: int, warmup: int, peaks: dict,
                    flush_buf, gpu_index: int, layer_ms=None, kern=None) -> dict:
    """ms/layer, TFLOP/s and per-kernel roofline fractions of one workload.
    Each measurement starts after REST_S of idle so that none of them runs on
    clocks lowered by the previous one's power draw; the SM clock sampled
    over the whole report is recorded beside it. The headline passes its
    timed region's layer time and per-kernel times."""
    for _ in range(warmup):
        w.layer(V, stream)
    torch.cuda.synchronize()
    rc = V.vdn_get_device_error()
    if rc != 0:
        raise RuntimeError(f"{w.name}: {V.vdn_error_string(rc)}")
    fb = flush_buf if w.flush else None
    with ClockSampler(gpu_index) as clk:
        if layer_ms is None:
            time.sleep(REST_S)
            layer_ms = time_launches(torch, stream, lambda: w.layer(V, stream), steps, fb)
        if kern is None:
            time.sleep(REST_S)
            kern = V.vdn_hybrid_attn_fwd_profile(w.shape, w.dev["q"], w.dev["k"], w.dev["v"],
                                                 w.dev["kt"], w.dev["vt"], w.dev["g_s"],
                                                 w.dev["g_l"], w.rms_w, w.out, w.ws,
                                                 iters=min(steps, 10), stream=stream)
        extra = {}
        if w.inp["d"] == 128 and w.inp["dtype"] == "bf16":
            extra = standalone_kernels(V, torch, w, stream, steps)
    ms = layer_ms
    fl = w.fl
    merged_flop = fl["softmax"] + fl["readout"]
    t_sm = kern["softmax_merge"]
    rep = {
        "ms_per_layer": round(ms, 4),
        "tflops": round(fl["total"] / (ms * 1e-3) / 1e12, 1),
        "layer_tflop": round(fl["total"] / 1e12, 4),
        "kernels_ms": {k: round(v, 4) for k, v in kern.items()},
        "softmax_merge": {
            "kernel": "k_bsa_fwd<merge>", "flop": merged_flop,
            "achieved_tflops": round(merged_flop / (t_sm * 1e-3) / 1e12, 1),
            "frac_burst": round(merged_flop / (t_sm * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
            "frac_sustained": round(merged_flop / (t_sm * 1e-3) / 1e12 / peaks["bf16_sustained"], 4),
        },
    }
    if extra:
        t_bsa = extra["bsa_ms"]
        rep["softmax_only"] = {"kernel": "k_bsa_fwd", "ms": round(t_bsa, 4),
                               "frac_burst": round(fl["softmax"] / (t_bsa * 1e-3) / 1e12
                                                   / peaks["bf16_tflops"], 4)}
        hbm = {}
        for key, t in (("gram_inv", kern["gram_inv"]), ("scan", kern["scan"]),
                       ("pack", kern["pack"]), ("gate_merge", extra["merge_ms"])):
            b = w.bytes[key]
            gbs = b / (t * 1e-3) / 1e9 if t > 0 else None
            hbm[key] = {"bytes": int(b), "ms": round(t, 4),
                        "gbs": round(gbs, 1) if gbs else None,
                        "frac": round(gbs / peaks["hbm_gbs"], 4) if gbs else None}
        hbm["gate_merge"]["kernel"] = "k_readout_merge_tma (vdn_gate_merge)"
        rep["hbm"] = hbm
    c = clk.summary()
    rep["sm_mhz"] = c["sm_mhz"]
    rep["sm_mhz_mean"] = c.get("sm_mhz_mean")
    rep["clock_reasons"] = c["reasons"]
    torch.cuda.synchronize()
    rc = V.vdn_get_device_error()
    if rc != 0:
        raise RuntimeError(f"{w.name}: {V.vdn_error_string(rc)}")
    return rep


def standalone_kernels(V, torch, w: Workload, stream, steps: int) -> dict:
    """The softmax branch alone (no merge epilogue) and the standalone
    readout + merge kernel, each timed by itself after a rest."""
    o_soft = torch.empty(w.dev["q"].shape, dtype=torch.bfloat16, device="cuda")
    R = torch.empty((w.shape.nb, w.inp["H"], 128, 128), device="cuda")
    d = w.dev
    V.vdn_vda_scan(w.shape, d["k"], d["v"], d["kt"], d["vt"], R, None, None, None, w.ws, stream)

    def bsa():
        V.vdn_bsa_fwd(w.shape, d["q"], d["k"], d["v"], d["kt"], d["vt"], o_soft, None, w.ws,
                      stream)

    def merge():
        V.vdn_gate_merge(w.shape, d["q"], R, o_soft, d["g_s"], d["g_l"], w.rms_w, w.out, w.ws,
                         stream)

    bsa()
    time.sleep(REST_S)
    t_bsa = time_launches(torch, stream, bsa, max(3, steps // 2))
    merge()
    time.sleep(REST_S)
    t_merge = time_launches(torch, stream, merge, max(5, steps))
    return dict(bsa_ms=t_bsa, merge_ms=t_merge)


def projection_report(V, torch, w: Workload, stream, steps: int, peaks: dict) -> dict:
    """The layer with per-branch output projections (w_o [H d, 2 H d],
    synthetic weights): whole-layer ms in bf16 and e4m3, and the projection
    GEMM and the activation quantiser timed alone."""
    import vdn_synth as S
    inp = w.inp
    H, d, N = inp["H"], inp["d"], inp["N"]
    D, K = H * d, 2 * H * d
    w_bf = torch.from_numpy(S.make_proj_weight(H, d, seed=0)).to("cuda", torch.bfloat16)
    w_codes = torch.empty((D, K), dtype=torch.uint8, device="cuda")
    w_scale = torch.empty(D, dtype=torch.float32, device="cuda")
    V.vdn_quantize_rows_e4m3(w_bf, D, K, w_codes, w_scale, stream)
    y = torch.empty((N, D), dtype=torch.bfloat16, device="cuda")
    dv = w.dev
    rep = {"D": D, "K": K, "weights": "synthetic N(0,1)/sqrt(2Hd), bf16; e4m3 per output channel",
           "gemm_tflop": round(2.0 * N * K * D / 1e12, 4)}
    for prec, name in ((V.VDN_PROJ_BF16, "bf16"), (V.VDN_PROJ_FP8, "fp8")):
        ws = V.alloc_proj_workspace(w.shape, D, prec)
        wo, sc = (w_bf, None) if prec == V.VDN_PROJ_BF16 else (w_codes, w_scale)

        def layer():
            V.vdn_hybrid_attn_proj_fwd(w.shape, dv["q"], dv["k"], dv["v"], dv["kt"], dv["vt"],
                                       dv["g_s"], dv["g_l"], w.rms_w, wo, sc, D, prec, y, ws,
                                       stream)

        layer()
        time.sleep(REST_S)
        t_layer = time_launches(torch, stream, layer, steps)
        rep[f"layer_{name}_ms"] = round(t_layer, 4)
        rep[f"layer_{name}_tflops"] = round((w.fl["total"] + 2.0 * N * K * D) / (t_layer * 1e-3)
                                            / 1e12, 1)
        del ws
    # the GEMMs alone on the layer's own gated branches
    br = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    ws = V.alloc_workspace(w.shape)
    V.vdn_hybrid_attn_branches(w.shape, dv["q"], dv["k"], dv["v"], dv["kt"], dv["vt"], dv["g_s"],
                               dv["g_l"], w.rms_w, br, ws, stream)
    a_codes = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    a_scale = torch.empty(N, dtype=torch.float32, device="cuda")
    V.vdn_quantize_rows_e4m3(br, N, K, a_codes, a_scale, stream)
    flop = 2.0 * N * K * D
    time.sleep(REST_S)
    t_bf = time_launches(torch, stream, lambda: V.vdn_linear(br, None, w_bf, None, N, K, D,
                                                             V.VDN_PROJ_BF16, y, stream), steps)
    time.sleep(REST_S)
    t_f8 = time_launches(torch, stream, lambda: V.vdn_linear(a_codes, a_scale, w_codes, w_scale, N,
                                                             K, D, V.VDN_PROJ_FP8, y, stream), steps)
    time.sleep(REST_S)
    t_q = time_launches(torch, stream, lambda: V.vdn_quantize_rows_e4m3(br, N, K, a_codes, a_scale,
                                                                        stream), steps)
    qbytes = N * K * 2 + N * K + N * 4
    rep["gemm_bf16"] = {"kernel": "k_linear<bf16>", "ms": round(t_bf, 4),
                        "tflops": round(flop / (t_bf * 1e-3) / 1e12, 1),
                        "frac": round(flop / (t_bf * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
                        "peak": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']}"}
    fp8_peak = 2 * peaks["bf16_tflops"]
    rep["gemm_fp8"] = {"kernel": "k_linear<e4m3>", "ms": round(t_f8, 4),
                       "tflops": round(flop / (t_f8 * 1e-3) / 1e12, 1),
                       "frac": round(flop / (t_f8 * 1e-3) / 1e12 / fp8_peak, 4),
                       "peak": f"2 x {peaks['source']} bf16 burst (nominal fp8/bf16 ratio) = "
                               f"{fp8_peak}"}
    rep["quant_e4m3"] = {"kernel": "k_quant_rows_e4m3", "ms": round(t_q, 4), "bytes": qbytes,
                         "frac": round(qbytes / (t_q * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
    del br, a_codes, ws
    torch.cuda.synchronize()
    rc = V.vdn_get_device_error()
    if rc != 0:
        raise RuntimeError(f"projections: {V.vdn_error_string(rc)}")
    return rep


def fp8_report(V, torch, w: Workload, stream, steps: int, peaks: dict) -> dict:
    """The e4m3 softmax branch and the layer with it: entry-point times (the
    quantisation pre-pass included) beside the bf16 softmax-only kernel."""
    d = w.dev
    ws8 = V.alloc_fp8_workspace(w.shape)
    o = torch.empty(d["q"].shape, dtype=torch.bfloat16, device="cuda")

    def bsa8():
        V.vdn_bsa_fwd_fp8(w.shape, d["q"], d["k"], d["v"], d["kt"], d["vt"], o, None, ws8, stream)

    def layer8():
        V.vdn_hybrid_attn_fwd_fp8(w.shape, d["q"], d["k"], d["v"], d["kt"], d["vt"], d["g_s"],
                                  d["g_l"], w.rms_w, w.out, ws8, stream)

    bsa8()
    time.sleep(REST_S)
    t_b = time_launches(torch, stream, bsa8, steps)
    layer8()
    time.sleep(REST_S)
    t_l = time_launches(torch, stream, layer8, steps)
    fl = w.fl
    fp8_peak = 2 * peaks["bf16_tflops"]
    del ws8, o
    torch.cuda.synchronize()
    rc = V.vdn_get_device_error()
    if rc != 0:
        raise RuntimeError(f"fp8: {V.vdn_error_string(rc)}")
    return {
        "softmax_fp8": {"entry": "vdn_bsa_fwd_fp8 (e4m3 pre-pass + k_bsa_fwd<e4m3>)",
                        "ms": round(t_b, 4),
                        "tflops": round(fl["softmax"] / (t_b * 1e-3) / 1e12, 1),
                        "frac": round(fl["softmax"] / (t_b * 1e-3) / 1e12 / fp8_peak, 4),
                        "peak": f"2 x {peaks['source']} bf16 burst (nominal fp8/bf16 ratio) = "
                                f"{fp8_peak}"},
        "layer_fp8": {"entry": "vdn_hybrid_attn_fwd_fp8", "ms": round(t_l, 4),
                      "tflops": round(fl["total"] / (t_l * 1e-3) / 1e12, 1)},
        "tolerance": "o_soft rel-L2 <= 0.06 vs the fp64 oracle (e4m3 operands)",
    }


def run_cuda(args) -> None:
    import torch

    import video_diffusion_hybrid_block_b200 as V

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    stream = torch.cuda.current_stream()
    peaks = load_peaks()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    # ---- headline workload: device-resident timing of the whole layer
    w = Workload(args.workload, V, torch)
    for _ in range(args.warmup):
        w.layer(V, stream)
    torch.cuda.synchronize()
    rc = V.vdn_get_device_error()
    if rc != 0:
        raise RuntimeError(V.vdn_error_string(rc))
    flush_buf = torch.empty(64 * 2 ** 20, dtype=torch.float32, device="cuda")  # 256 MiB
    time.sleep(REST_S)
    head_kern = None
    with ClockSampler(local) as clk:
        if w.flush:
            barrier()
            ms = time_launches(torch, stream, lambda: w.layer(V, stream), args.steps, flush_buf)
            barrier()
        else:
            # the timed layers run through the profiling entry point: the same
            # launches with CUDA events between the layer's kernels, so the
            # per-kernel times (and the roofline) come from the timed region
            barrier()
            head_kern = timed_layers(V, w, stream, args.steps)
            barrier()
            ms = sum(head_kern.values())
    ms = max_over_ranks(dist, ms, "cuda")
    if head_kern is not None:
        head_kern = {k: max_over_ranks(dist, t, "cuda") for k, t in head_kern.items()}
    clocks = clk.summary()
    launches_per_step = 4 + (0 if (w.inp["d"] == 128 and w.inp["dtype"] == "bf16") else 5)

    # ---- end to end through the C ABI with host buffers (H2D + layer + D2H).
    # Every step copies its inputs from pinned host memory and its output back.
    # Two device buffer sets let step i+1's upload (copy stream) run while step
    # i computes and step i-1's result downloads (second copy stream), as a
    # serving loop would; each step still moves all of its bytes.
    host = {k: t.pin_memory() for k, t in w.host.items()}
    out_host = torch.empty(w.out.shape, dtype=w.dt).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = w.out.numel() * w.out.element_size()
    sets = [w.dev, {k: torch.empty_like(t) for k, t in w.dev.items()}]
    outs = [w.out, torch.empty_like(w.out)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {n: [torch.cuda.Event(), torch.cuda.Event()] for n in ("up", "done", "down")}
    for b in range(2):  # all buffers free at the start
        for n in ("done", "down"):
            ev[n][b].record(stream)

    def e2e_step(i):
        b = i & 1
        d, o = sets[b], outs[b]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev["done"][b])   # the layer that last read set b finished
            for k, t in host.items():
                d[k].copy_(t, non_blocking=True)
            ev["up"][b].record(s_in)
        stream.wait_event(ev["up"][b])
        stream.wait_event(ev["down"][b])     # out b was downloaded
        w.layer(V, stream, dev=d, out=o)
        ev["done"][b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["done"][b])
            out_host.copy_(o, non_blocking=True)
            ev["down"][b].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(s_in)
    for i in range(args.steps):
        e2e_step(i)
    g1.record(s_out)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(dist, g0.elapsed_time(g1) / args.steps, "cuda")
    del sets[1], outs[1]

    # ---- every workload; the headline's report reuses its layer time
    reports = {}
    # the extra reports run at N = 1; at N > 1 (replicas) only the headline
    # workload is reported, which keeps the multi-GPU run short
    full_report = args.workloads == "all" or (args.workloads == "auto" and world == 1)
    names = WORKLOADS if full_report else [args.workload]
    for name in names:
        ww = w if name == args.workload else Workload(name, V, torch)
        reports[name] = workload_report(V, torch, ww, stream, args.steps, args.warmup, peaks,
                                        flush_buf, local,
                                        layer_ms=ms if name == args.workload else None,
                                        kern=head_kern if name == args.workload else None)
        if ww is not w:
            del ww
            torch.cuda.empty_cache()
    proj = fp8 = None
    if full_report and not args.no_projections and w.inp["d"] == 128 and w.inp["dtype"] == "bf16":
        proj = projection_report(V, torch, w, stream, args.steps, peaks)
        fp8 = fp8_report(V, torch, w, stream, args.steps, peaks)
    head = reports[args.workload]
    sm = head["softmax_merge"]

    value = whole_job_value(world, w.fl["total"], ms)
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": config_of(args.workload, w.inp, w.fl, world),
        "roofline": {"kernel": "k_bsa_fwd<merge> (softmax branch + fused readout, RMSNorm, "
                               "gated merge), timed inside the layers of the timed region",
                     "bound": "tensor", "achieved": sm["achieved_tflops"],
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": sm["frac_burst"],
                     "frac_sustained": sm["frac_sustained"],
                     "peak_source": f"{peaks['source']} bf16 burst "
                                    f"(sustained {peaks['bf16_sustained']})",
                     "launch_ms": head["kernels_ms"]["softmax_merge"],
                     "traffic": recorded_traffic(args.workload)},
        "e2e": {"value": round(whole_job_value(world, w.fl["total"], e2e_ms), 2),
                "unit": "TFLOP/s", "ms_per_step": round(e2e_ms, 4),
                "pipelining": "uploads, layer and downloads of consecutive steps overlap "
                              "(two device buffer sets, two copy streams)",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "workloads": reports,
    }
    if clocks.get("sm_mhz_mean") and clocks.get("sm_max_mhz"):
        # the burst peak was taken at the maximum SM clock; the timed region
        # runs under the power cap at a lower mean clock
        scale = clocks["sm_mhz_mean"] / clocks["sm_max_mhz"]
        line["roofline"]["frac_at_mean_clock"] = round(sm["achieved_tflops"]
                                                       / (peaks["bf16_tflops"] * scale), 4)
    if proj is not None:
        line["projections"] = proj
    if fp8 is not None:
        line["fp8"] = fp8
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w.inp, w.fl, args.workload, CPU_BASELINE_HEADS)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# --------------------------------------------------------- oracle (CPU) -----

def reference_rows(inp: dict, n: int = REF_ROWS) -> np.ndarray:
    """Query rows one reference step computes: n rows evenly spread over the clip."""
    return np.unique(np.linspace(0, inp["N"] - 1, min(n, inp["N"])).astype(np.int64))


def reference_step_flops(inp: dict, soft_pairs: np.ndarray, fl: dict, rows) -> float:
    """Algorithmic FLOP of one reference step: one head's VDA work plus the
    softmax and readout work of the given query rows of that head."""
    off = np.asarray(inp["off"], np.int64)
    F, d, H, T = inp["F"], inp["d"], inp["H"], inp["T"]
    n = np.diff(off)
    keys = np.where(n > 0, soft_pairs[:, :F].sum(axis=1) / np.maximum(n, 1), 0) + T
    frame = np.searchsorted(off, rows, side="right") - 1
    return fl["vda"] / H + 4.0 * d * float(keys[frame].sum()) + 2.0 * d * d * len(rows)


def oracle_steps(inp: dict, fl: dict, soft: np.ndarray, nsteps: int, warmup: int):
    """Runs the fp64 oracle as it stands: step s = head s % H, all of its VDA
    states and the whole layer for REF_ROWS query rows. Returns (seconds per
    step, FLOP per step)."""
    import oracle as O
    rows = reference_rows(inp)
    for s in range(warmup):
        O.layer_head(inp, s % inp["H"], rows=rows)
    t0 = time.perf_counter()
    for s in range(nsteps):
        O.layer_head(inp, s % inp["H"], rows=rows)
    dt = (time.perf_counter() - t0) / max(nsteps, 1)
    return dt, reference_step_flops(inp, soft, fl, rows)


def cpu_baseline(inp: dict, fl: dict, name: str, heads: int) -> dict:
    """The fp64 CPU oracle, as it stands, on a bounded sample of the workload."""
    import oracle as O
    soft, _ = O.pair_counts(inp["off"], inp["block_frames"], inp["T"])
    dt, flop = oracle_steps(inp, fl, soft, heads, 0)
    return {"value": round(flop / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores_used(),
            "kind": "oracle", "seconds": round(dt * heads, 2),
            "sample": f"fp64 numpy oracle, {heads} heads of {inp['H']}: each head's VDA states "
                      f"and the whole layer for {len(reference_rows(inp))} of {inp['N']} query "
                      f"rows, {name} workload"}


def run_reference(args) -> None:
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle as O
    import vdn_synth as S
    inp = S.make_inputs(args.workload, seed=0)
    soft, _ = O.pair_counts(inp["off"], inp["block_frames"], inp["T"])
    fl = layer_flops(inp, soft)
    dt, flop = oracle_steps(inp, fl, soft, args.steps, args.warmup)
    value = flop / dt / 1e12
    rows = reference_rows(inp)
    sample = (f"fp64 numpy oracle; one step = one head's VDA states and the whole layer for "
              f"{len(rows)} of {inp['N']} query rows, {args.workload} workload")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(args.workload, inp, fl, world),
        "step_tflop": round(flop / 1e12, 6),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores_used(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ ncu helper ----

def run_profile(args) -> None:
    """Runs `--steps` launches of one entry point (after `--warmup`) on a
    workload with optionally fewer heads, for bounded ncu captures."""
    import torch

    import video_diffusion_hybrid_block_b200 as V
    import vdn_synth as S

    cfg = dict(S.CONFIGS[args.workload])
    if args.heads:
        cfg["H"] = args.heads
    inp = S.make_inputs_from(cfg["F"], S.frame_sizes(cfg), cfg["T"], cfg["H"], cfg["d"],
                             dtype=cfg["dtype"], seed=0, k_lowrank=cfg.get("k_lowrank"),
                             zero_v_every=cfg.get("zero_v_every"))
    dt = torch.bfloat16 if cfg["dtype"] == "bf16" else torch.float32
    dev = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to("cuda", dt)
           for k in ("q", "k", "v", "kt", "vt", "g_s", "g_l")}
    rms_w = torch.from_numpy(inp["rms_w"]).cuda()
    shape = V.Shape(inp["off"], inp["T"], inp["H"], inp["d"], inp["block_frames"], inp["lam"],
                    inp["eps"], V.VDN_BF16 if cfg["dtype"] == "bf16" else V.VDN_F32)
    ws = V.alloc_workspace(shape)
    out = torch.empty_like(dev["q"])
    nb = -(-inp["F"] // inp["block_frames"])
    R = torch.empty((nb, inp["H"], inp["d"], inp["d"]), device="cuda")
    o_soft = torch.empty(dev["q"].shape, dtype=torch.bfloat16, device="cuda")

    D, K = inp["H"] * inp["d"], 2 * inp["H"] * inp["d"]
    if args.profile in ("proj", "proj8"):
        w_bf = torch.from_numpy(S.make_proj_weight(inp["H"], inp["d"], seed=0)).to("cuda",
                                                                                 torch.bfloat16)
        w_codes = torch.empty((D, K), dtype=torch.uint8, device="cuda")
        w_scale = torch.empty(D, dtype=torch.float32, device="cuda")
        V.vdn_quantize_rows_e4m3(w_bf, D, K, w_codes, w_scale)
        prec = V.VDN_PROJ_FP8 if args.profile == "proj8" else V.VDN_PROJ_BF16
        wsp = V.alloc_proj_workspace(shape, D, prec)
        y = torch.empty((inp["N"], D), dtype=torch.bfloat16, device="cuda")
    if args.profile == "bsa8":
        ws8 = V.alloc_fp8_workspace(shape)

    def once():
        if args.profile in ("proj", "proj8"):
            wo, sc = (w_codes, w_scale) if args.profile == "proj8" else (w_bf, None)
            V.vdn_hybrid_attn_proj_fwd(shape, dev["q"], dev["k"], dev["v"], dev["kt"], dev["vt"],
                                       dev["g_s"], dev["g_l"], rms_w, wo, sc, D, prec, y, wsp)
        elif args.profile == "bsa8":
            V.vdn_bsa_fwd_fp8(shape, dev["q"], dev["k"], dev["v"], dev["kt"], dev["vt"], o_soft,
                              None, ws8)
        elif args.profile == "layer":
            V.vdn_hybrid_attn_fwd(shape, dev["q"], dev["k"], dev["v"], dev["kt"], dev["vt"],
                                  dev["g_s"], dev["g_l"], rms_w, out, ws)
        elif args.profile == "bsa":
            V.vdn_bsa_fwd(shape, dev["q"], dev["k"], dev["v"], dev["kt"], dev["vt"], o_soft, None,
                          ws)
        elif args.profile == "merge":
            V.vdn_gate_merge(shape, dev["q"], R, o_soft, dev["g_s"], dev["g_l"], rms_w, out, ws)
        else:
            V.vdn_vda_scan(shape, dev["k"], dev["v"], dev["kt"], dev["vt"], R, None, None, None,
                           ws)

    if args.profile == "merge":
        # the merge reads real read states and o_soft
        V.vdn_vda_scan(shape, dev["k"], dev["v"], dev["kt"], dev["vt"], R, None, None, None, ws)
        V.vdn_bsa_fwd(shape, dev["q"], dev["k"], dev["v"], dev["kt"], dev["vt"], o_soft, None, ws)
    for _ in range(args.warmup + args.steps):
        once()
    torch.cuda.synchronize()
    rc = V.vdn_get_device_error()
    print(json.dumps({"profile": args.profile, "workload": args.workload, "H": inp["H"],
                      "launches": args.warmup + args.steps, "device_error": rc}))
    if rc != 0:
        sys.exit(1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-projections", action="store_true",
                    help="skip the per-branch output projection measurements")
    ap.add_argument("--workloads", default="auto", choices=["auto", "all", "none"],
                    help="also report every workload, the projections and the e4m3 figures "
                         "(auto: on one GPU only), or only the headline workload")
    ap.add_argument("--profile", choices=["layer", "bsa", "vda", "merge", "proj", "proj8", "bsa8"],
                    help="only run launches of one entry point (for ncu captures)")
    ap.add_argument("--workload", default=HEADLINE,
                    help="workload name (vdn_synth.CONFIGS); the default is the headline one")
    ap.add_argument("--heads", type=int, default=0, help="override head count for --profile")
    args = ap.parse_args()
    if args.profile:
        run_profile(args)
        return
    if args.warmup < 3 and args.impl == "cuda":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
