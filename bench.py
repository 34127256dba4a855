"""Benchmark of the hybrid attention layer forward on B200.

One step = one vdn_hybrid_attn_fwd call (softmax branch, VDA Grams/inverses,
both scans, readout + RMSNorm + gated merge) on the pages-scale workload:
F=15 latent frames of 24x42=1008 tokens (15120 video tokens), T=256 text
tokens, H=32 heads, d=128, bf16, seed 0. Inputs are synthetic (vdn_synth).

Prints one JSON line (rank 0). `value` is layer TFLOP/s (algorithmic FLOP:
softmax over unmasked (query, key) pairs + VDA Grams, inverses, scan products
and readout) summed over ranks; `ms_per_step` is the max over ranks.
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
WORKLOAD = "pages-scale"
WORKLOAD_DESC = ("pages-scale single layer: F=15 latent frames (3 blocks of 5), 24x42=1008 "
                 "tokens/frame (15120 video tokens), T=256 text tokens, H=32, d=128, bf16")
L2_BYTES = 126 * 2 ** 20


def layer_flops(inp: dict, soft_pairs: np.ndarray) -> dict:
    """Algorithmic FLOP of one layer forward.

    softmax: 4 d H (video pairs + N T) over unmasked pairs (QK^T and PV);
    VDA: Grams 4 (N+T) d^2 H, readout 2 N d^2 H, and per scanned matrix
    (F-2 frames + text) and head one d x d inverse (2 d^3) plus one d^3 x 2
    product per scan direction (4 d^3)."""
    N, T, H, d, F = inp["N"], inp["T"], inp["H"], inp["d"], inp["F"]
    video_pairs = int(soft_pairs[:, :F].sum())
    softmax = 4.0 * d * H * (video_pairs + N * T)
    grams = 4.0 * (N + T) * d * d * H
    readout = 2.0 * N * d * d * H
    solves = (F - 1) * H * (2.0 * d ** 3 + 4.0 * d ** 3)
    return dict(softmax=softmax, vda=grams + readout + solves,
                total=softmax + grams + readout + solves)


def vda_merge_roofline(inp: dict, layer_ms: float, softmax_ms: float, hbm_gbs: float) -> dict:
    """VDA + merge path against its HBM roofline. Algorithmic bytes: k, v, kt,
    vt read once, q, o_soft, g_s, g_l read and out written once (bf16). The
    merge runs fused in the softmax kernel's epilogue, so the path's cost is
    the layer time minus the softmax-only kernel."""
    N, T, H, d = inp["N"], inp["T"], inp["H"], inp["d"]
    act = N * H * d * 2
    nbytes = 2 * act + 2 * T * H * d * 2 + 2 * act + 2 * N * H * 2 + act
    roof_ms = nbytes / (hbm_gbs * 1e9) * 1e3
    marginal = layer_ms - softmax_ms
    return {"algorithmic_bytes": int(nbytes), "roofline_ms": round(roof_ms, 4),
            "marginal_ms": round(marginal, 4),
            "frac": round(roof_ms / marginal, 4) if marginal > 0 else None,
            "method": "layer time minus the softmax-only kernel (merge fused in its epilogue)"}


def workload_desc(name: str) -> str:
    if name == WORKLOAD:
        return WORKLOAD_DESC
    import vdn_synth as S
    c = S.CONFIGS[name]
    return (f"{name}: F={c['F']} latent frames, {c['grid'][0]}x{c['grid'][1]} tokens/frame, "
            f"T={c['T']}, H={c['H']}, d={c['d']}, {c['dtype']}")


def l2_note(input_bytes: int) -> str:
    if input_bytes > L2_BYTES:
        return f"inputs {input_bytes / 2 ** 20:.0f} MiB > 126 MB L2; no flush between steps"
    return "inputs fit in the 126 MB L2: warm-cache figure, no flush between steps"


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return dict(bf16_tflops=float(p["bf16_tflops"]), hbm_gbs=float(p["hbm_gbs"]),
                    source="measured")
    return dict(bf16_tflops=1590.0, hbm_gbs=6650.0, source="fallback")


def bsa_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("k_bsa_fwd.cuh", "layer_plan.cuh", "sm100_ptx.cuh"):
        with open(os.path.join(ROOT, "video_diffusion_hybrid_block_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per k_bsa_fwd launch from the committed ncu summary, if it
    was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "bsa_fwd_pages_scale_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        rec = json.load(fh)
    if rec.get("source_hash") != bsa_source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        if self.path and os.path.exists(self.path):
            with open(self.path) as fh:
                for line in fh:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


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


def run_cuda(args) -> None:
    import torch

    import video_diffusion_hybrid_block_b200 as V
    import vdn_synth as S

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    inp = S.make_inputs(args.workload, seed=0)
    dt = torch.bfloat16 if inp["dtype"] == "bf16" else torch.float32
    host = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to(dt).pin_memory()
            for k in ("q", "k", "v", "kt", "vt", "g_s", "g_l")}
    dev = {k: t.to("cuda", non_blocking=False) for k, t in host.items()}
    rms_w = torch.from_numpy(inp["rms_w"]).cuda()
    shape = V.Shape(inp["off"], inp["T"], inp["H"], inp["d"], inp["block_frames"], inp["lam"],
                    inp["eps"], V.VDN_BF16 if inp["dtype"] == "bf16" else V.VDN_F32)
    ws = V.alloc_workspace(shape)
    out = torch.empty_like(dev["q"])
    out_host = torch.empty(out.shape, dtype=dt).pin_memory()
    stream = torch.cuda.current_stream()

    soft = torch.empty((inp["F"], inp["F"] + 1), dtype=torch.int64, device="cuda")
    lin = torch.empty((inp["F"], inp["F"]), dtype=torch.int64, device="cuda")
    V.vdn_pair_audit(shape, soft, lin)
    fl = layer_flops(inp, soft.cpu().numpy())

    def step():
        V.vdn_hybrid_attn_fwd(shape, dev["q"], dev["k"], dev["v"], dev["kt"], dev["vt"],
                              dev["g_s"], dev["g_l"], rms_w, out, ws, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    rc = V.vdn_get_device_error()
    if rc != 0:
        raise RuntimeError(V.vdn_error_string(rc))

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    # ---- device-resident timing of the whole layer
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        barrier()
    ms = max_over_ranks(dist, e0.elapsed_time(e1) / args.steps, "cuda")
    clocks = clk.summary()
    launches_per_step = 4 + (0 if shape.d == 128 else 5)

    # ---- dominant kernel alone (softmax branch), CUDA events on its stream
    o_soft = torch.empty(dev["q"].shape, dtype=torch.bfloat16, device="cuda")

    def bsa():
        V.vdn_bsa_fwd(shape, dev["q"], dev["k"], dev["v"], dev["kt"], dev["vt"], o_soft, None,
                      ws, stream)

    for _ in range(3):
        bsa()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    b0.record(stream)
    nb_launch = max(args.steps, 5)
    for _ in range(nb_launch):
        bsa()
    b1.record(stream)
    barrier()
    bsa_ms = max_over_ranks(dist, b0.elapsed_time(b1) / nb_launch, "cuda")

    # ---- end to end through the C ABI with host buffers (H2D + layer + D2H).
    # Every step copies its inputs from pinned host memory and its output back.
    # Two device buffer sets let step i+1's upload (copy stream) run while step
    # i computes and step i-1's result downloads (second copy stream), as a
    # serving loop would; each step still moves all of its bytes.
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out.numel() * out.element_size()
    sets = [dev, {k: torch.empty_like(t) for k, t in dev.items()}]
    outs = [out, torch.empty_like(out)]
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
        V.vdn_hybrid_attn_fwd(shape, d["q"], d["k"], d["v"], d["kt"], d["vt"], d["g_s"], d["g_l"],
                              rms_w, o, ws, stream)
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

    peaks = load_peaks()
    achieved = fl["softmax"] / (bsa_ms * 1e-3) / 1e12
    value = whole_job_value(world, fl["total"], ms)
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
        "config": {"workload": workload_desc(args.workload), "F": inp["F"],
                   "tokens_per_frame": int(inp["N"] // inp["F"]),
                   "N": inp["N"], "T": inp["T"], "H": inp["H"], "d": inp["d"],
                   "layer_tflop": round(fl["total"] / 1e12, 4),
                   "softmax_tflop": round(fl["softmax"] / 1e12, 4),
                   "parallelism": f"replicas x{world}", "l2": l2_note(h2d)},
        "roofline": {"kernel": "k_bsa_fwd", "bound": "tensor", "achieved": round(achieved, 1),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(achieved / peaks["bf16_tflops"], 4),
                     "peak_source": f"{peaks['source']} bf16 burst",
                     "launch_ms": round(bsa_ms, 4),
                     "traffic": recorded_traffic() if args.workload == WORKLOAD else None},
        "e2e": {"value": round(whole_job_value(world, fl["total"], e2e_ms), 2),
                "unit": "TFLOP/s", "ms_per_step": round(e2e_ms, 4),
                "pipelining": "uploads, layer and downloads of consecutive steps overlap "
                              "(two device buffer sets, two copy streams)",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "vda_merge": vda_merge_roofline(inp, ms, bsa_ms, peaks["hbm_gbs"]),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload == WORKLOAD:
        line["cpu_baseline"] = cpu_baseline(inp, fl, args.cpu_heads)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def cpu_baseline(inp: dict, fl: dict, heads: int) -> dict:
    """The fp64 CPU oracle, as it stands, on `heads` of the workload's heads
    (every query row of those heads); scaled to the layer's FLOP per head."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        cores = os.cpu_count()
    t0 = time.perf_counter()
    for h in range(heads):
        O.layer_head(inp, h)
    dt = time.perf_counter() - t0
    flop = fl["total"] * heads / inp["H"]
    return {"value": round(flop / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"fp64 numpy oracle, whole layer for {heads} of {inp['H']} heads "
                      f"(all {inp['N']} query rows), pages-scale workload"}


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

    def once():
        if args.profile == "layer":
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


def run_reference(args) -> None:
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import vdn_synth as S
    import oracle as O
    inp = S.make_inputs(WORKLOAD, seed=0)
    soft, _ = O.pair_counts(inp["off"], inp["block_frames"], inp["T"])
    fl = layer_flops(inp, soft)
    for _ in range(args.warmup):
        O.layer_head(inp, 0)
    times = []
    for s in range(args.steps):
        t0 = time.perf_counter()
        O.layer_head(inp, s % inp["H"])
        times.append(time.perf_counter() - t0)
    per_head = sum(times) / len(times)
    flop = fl["total"] / inp["H"]
    value = flop / per_head / 1e12
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        cores = os.cpu_count()
    sample = (f"fp64 numpy oracle, one head (all {inp['N']} query rows) per step, "
              "pages-scale workload")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(per_head * 1e3 * inp["H"], 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC, "F": inp["F"], "N": inp["N"], "T": inp["T"],
                   "H": inp["H"], "d": inp["d"], "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--cpu-heads", type=int, default=6)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=["layer", "bsa", "vda", "merge"],
                    help="only run launches of one entry point (for ncu captures)")
    ap.add_argument("--workload", default=WORKLOAD,
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
