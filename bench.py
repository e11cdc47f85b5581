"""Benchmark of the FG^2-GDN chunkwise forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one gdn_chunk_fwd (or gdn_deltaproduct_fwd) call over one batch of
seeded synthetic input of the named workload (default: the 32K-token FG^2-GDN
prefill, B=1, H=16, T=32768, d=128, chunk 64, bf16).  Prints one JSON line.

  value     tokens/s (B*T per second, all heads, all ranks) with inputs resident
            in HBM, timed with CUDA events on the launching stream.
  e2e       the same metric through the C ABI with pinned host buffers: each step
            copies the inputs host->device, runs the call and reads out and
            S_final back, inside the timed region.
  roofline  algorithmic bytes per call / call time against the measured HBM copy
            bandwidth (the path is HBM-bound).
  cpu_baseline  the fp64 oracle on the host cores over a bounded sample.
With torchrun (N > 1) every rank runs its own replica of the workload on its GPU
(weak scaling; the heads are independent, there is no data-path collective).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_delta_rule_fg_b200.inputs import CONFIGS, make_inputs  # noqa: E402

METRIC = "tokens/s FG²-GDN chunked fwd (T=32K, d=128) and % of roofline, 1 B200"
L2_BYTES = 126 * 2 ** 20


def algorithmic_bytes(cfg) -> int:
    """Bytes the method must move per call: q, k, v, alpha, beta read, o written
    (+ S0 read, S_final written)."""
    e = 2 if cfg.dtype == "bf16" else 4
    th = cfg.B * cfg.T * cfg.H
    if cfg.deltaproduct_nh:
        nh = cfg.deltaproduct_nh
        per = cfg.dk * e + nh * (cfg.dk + cfg.dv) * e + 4 + nh * 4 + cfg.dv * e
    else:
        a = 4 if cfg.alpha_scalar else 4 * cfg.dk
        b = 4 if cfg.beta_scalar else 4 * cfg.dk
        per = cfg.dk * e * 2 + cfg.dv * e + a + b + cfg.dv * e
    state = cfg.B * cfg.H * cfg.dk * cfg.dv * 4
    return th * per + state * (2 if cfg.s0_std > 0 else 1)


def algorithmic_flops(cfg) -> float:
    """C (5 dk + 3 dv) + 6 dk dv per token-head (per sub-step for DeltaProduct)."""
    steps = cfg.B * cfg.T * cfg.H * max(1, cfg.deltaproduct_nh)
    return float(steps) * (cfg.chunk * (5 * cfg.dk + 3 * cfg.dv) + 6 * cfg.dk * cfg.dv)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def load_traffic(kernel: str, workload: str, source_hash: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kernel}:{workload}")
    if not e or e.get("source_hash") != source_hash:
        return None
    return float(e["dram_bytes_per_launch"])


TC_SOURCES = ("gdn_tc.cu", "gdn_sm100.cuh")     # the timed kernels' own code


def source_hash() -> str:
    """Hash of the sources of the kernels bench.py times; traffic counters taken on other
    sources are not reported."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_fg_b200", "csrc")
    for n in TC_SOURCES:
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(n.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background (every 200 ms)."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join(ROOT, "gpurun_out", f"clocks_gpu{gpu_index}.csv")

    def start(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for n, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "samples": len(sm), "reasons": sorted(reasons)}


def cpu_baseline(cfg, budget_s: float = 12.0):
    """Time the fp64 oracle (as it stands) on a bounded sample: whole heads of the
    workload, as many as fit the budget, one head per thread."""
    import oracle
    threads = oracle.max_threads()
    x = make_inputs(cfg, T=min(cfg.T, 2048), H=1, B=1)
    t0 = time.perf_counter()
    if cfg.deltaproduct_nh:
        oracle.deltaproduct_seq(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["S0"], nthreads=1)
    else:
        oracle.gdn_seq(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"],
                       alpha_scalar=cfg.alpha_scalar, beta_scalar=cfg.beta_scalar, nthreads=1)
    per_tok_head = (time.perf_counter() - t0) / x["q"].shape[1]
    # heads run in parallel, one per thread; pick a sample of whole heads that fits the budget
    nheads = max(1, min(cfg.B * cfg.H, threads))
    T_s = int(max(256, min(cfg.T, budget_s / max(per_tok_head, 1e-9))))
    H_s = min(cfg.H, nheads)
    x = make_inputs(cfg, T=T_s, H=H_s, B=1)
    t0 = time.perf_counter()
    if cfg.deltaproduct_nh:
        oracle.deltaproduct_seq(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["S0"], nthreads=threads)
    else:
        oracle.gdn_seq(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"],
                       alpha_scalar=cfg.alpha_scalar, beta_scalar=cfg.beta_scalar, nthreads=threads)
    dt = time.perf_counter() - t0
    token_heads = T_s * H_s
    tokens_per_s = token_heads / dt / cfg.H     # tokens/s counts B*T with all H heads
    return {"value": tokens_per_s, "unit": "tokens/s", "cores": min(threads, H_s), "kind": "oracle",
            "sample": f"{H_s} head(s) x {T_s} tokens of {cfg.name} (fp64 C oracle, one head per thread)",
            "seconds": dt}


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    vals, last = [], None
    # each step is a bounded sample, sized so that warm-up + timed steps end within minutes
    budget = max(0.5, min(args.ref_budget, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(max(0, args.warmup)):
        cpu_baseline(cfg, budget_s=budget)
    for _ in range(args.steps):
        last = cpu_baseline(cfg, budget_s=budget)
        vals.append(last["value"])
    v = float(np.median(vals))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * last["seconds"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "T": cfg.T, "dk": cfg.dk,
                       "dv": cfg.dv, "chunk": cfg.chunk},
            "cpu_baseline": dict(last, value=v),
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="fg2_prefill_32k", choices=sorted(CONFIGS))
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--ref-budget", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="only warm-up + timed steps (no clock soak, e2e or CPU baseline), for ncu")
    ap.add_argument("--B", type=int, default=None, help="override the workload's batch (small ncu captures)")
    ap.add_argument("--H", type=int, default=None, help="override the workload's heads")
    ap.add_argument("--T", type=int, default=None, help="override the workload's tokens per sequence")
    args = ap.parse_args()
    cfg = CONFIGS[args.workload]
    over = {k: getattr(args, k) for k in ("B", "H", "T") if getattr(args, k) is not None}
    if over:
        import dataclasses
        tag = ",".join(f"{k}={v}" for k, v in over.items())
        cfg = dataclasses.replace(cfg, name=f"{cfg.name}[{tag}]", **over)
    if args.impl == "reference":
        return run_reference(args, cfg)

    import torch
    import torch.distributed as dist
    from gated_delta_rule_fg_b200 import ops

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    # ---- inputs (resident in HBM), one replica per rank with its own seed
    x = make_inputs(cfg, seed=cfg.seed + 1000 * rank)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    host = {k: (torch.from_numpy(v).pin_memory() if v is not None else None) for k, v in x.items()}
    for kname in ("q", "k", "v"):
        host[kname] = host[kname].to(dt).pin_memory()
    d = {k: (v.to(dev, non_blocking=False) if v is not None else None) for k, v in host.items()}
    dp = cfg.deltaproduct_nh > 0
    code = ops.GDN_BF16 if cfg.dtype == "bf16" else ops.GDN_F32
    B, T, H = cfg.B, cfg.T, cfg.H
    out = torch.empty((B, T, H, cfg.dv), dtype=dt, device=dev)
    Sf = torch.empty((B, H, cfg.dk, cfg.dv), dtype=torch.float32, device=dev)
    if dp:
        nws = ops.deltaproduct_fwd_workspace_size(B, H, T, cfg.deltaproduct_nh, cfg.dk, cfg.dv, cfg.chunk, code)
        launches = ops.deltaproduct_fwd_launches(B, H, T, cfg.deltaproduct_nh, cfg.dk, cfg.dv, cfg.chunk, code)
    else:
        flags = (ops.GDN_ALPHA_SCALAR if cfg.alpha_scalar else 0) | (ops.GDN_BETA_SCALAR if cfg.beta_scalar else 0)
        nws = ops.chunk_fwd_workspace_size(B, H, T, cfg.dk, cfg.dv, cfg.chunk, code, flags)
        launches = ops.chunk_fwd_launches(B, H, T, cfg.dk, cfg.dv, cfg.chunk, code, flags)
    ws = ops.alloc_workspace(nws, dev)

    def step(src):
        if dp:
            ops.deltaproduct_fwd(src["q"], src["k"], src["v"], src["gamma"], src["beta"], src["S0"],
                                 chunk=cfg.chunk, out=out, S_final=Sf, workspace=ws, stream=stream)
        else:
            ops.chunk_fwd(src["q"], src["k"], src["v"], src["alpha"], src["beta"], src["S0"],
                          chunk=cfg.chunk, alpha_scalar=cfg.alpha_scalar, beta_scalar=cfg.beta_scalar,
                          out=out, S_final=Sf, workspace=ws, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        step(d)
    assert ops.workspace_status(ws) == ops.GDN_OK

    # ---- device-resident timed region (inputs >> L2, so every step streams from HBM)
    clocks = ClockSampler(local)
    if not args.profile:
        clocks.start()
        time.sleep(0.3)
        barrier()
        t_soak = time.perf_counter()
        while time.perf_counter() - t_soak < 1.0:          # keep the GPU busy for the clock sampler
            step(d)
            torch.cuda.synchronize()
    barrier()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step(d)
        ev[i][1].record(stream)
    e1.record(stream)
    barrier()
    clk = clocks.stop() if not args.profile else None
    total_ms = e0.elapsed_time(e1)
    per_call_ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    status = ops.workspace_status(ws)
    if status != ops.GDN_OK:
        raise SystemExit(f"device status after the timed region: {ops.status_string(status)}")
    t_max = torch.tensor([total_ms], device=dev)
    if world > 1:
        dist.all_reduce(t_max, op=dist.ReduceOp.MAX)
    total_ms = float(t_max.item())
    ms_per_step = total_ms / args.steps
    tokens = B * T * world
    value = tokens / (ms_per_step / 1000.0)

    # ---- end to end through the C ABI with pinned host buffers
    names = ["q", "k", "v", "gamma" if dp else "alpha", "beta", "S0"]
    h2d = sum(host[n].numel() * host[n].element_size() for n in names if host[n] is not None)
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    sf_h = torch.empty(Sf.shape, dtype=Sf.dtype).pin_memory()
    d2h = out_h.numel() * out_h.element_size() + sf_h.numel() * sf_h.element_size()
    dev_in = {n: (torch.empty_like(d[n]) if d[n] is not None else None) for n in names}
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(0 if args.profile else args.e2e_steps):
        for n in names:
            if host[n] is not None:
                dev_in[n].copy_(host[n], non_blocking=True)
        step(dev_in)
        out_h.copy_(out, non_blocking=True)
        sf_h.copy_(Sf, non_blocking=True)
    f1.record(stream)
    barrier()
    e2e_ms = f0.elapsed_time(f1) / max(1, args.e2e_steps)
    t_e = torch.tensor([e2e_ms], device=dev)
    if world > 1:
        dist.all_reduce(t_e, op=dist.ReduceOp.MAX)
    e2e_value = tokens / (float(t_e.item()) / 1000.0)

    hbm_gbs, bf16_tf, peak_kind = load_peaks()
    abytes = algorithmic_bytes(cfg)
    achieved = abytes / (per_call_ms / 1000.0) / 1e9
    kname = "gdn_chunk_fwd" if launches == 1 else f"gdn_chunk_fwd ({launches} kernels, whole call)"
    roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
            "frac": achieved / hbm_gbs, "traffic": load_traffic("gdn_chunk_fwd", cfg.name, source_hash()),
            "peak_kind": f"of {peak_kind} copy bandwidth", "kernel": kname,
            "algorithmic_bytes_per_launch": abytes, "algorithmic_flops_per_launch": algorithmic_flops(cfg),
            "flop_frac_of_bf16_peak": algorithmic_flops(cfg) / (per_call_ms / 1000.0) / (bf16_tf * 1e12),
            "launch_ms": per_call_ms}

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": cfg.dtype, "data": "synthetic (seeded numpy draws with the workload's distributions)",
            "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "T": cfg.T, "dk": cfg.dk,
                       "dv": cfg.dv, "chunk": cfg.chunk, "per_rank": "one replica per GPU",
                       "l2": f"inputs larger than L2 ({abytes / 1e9:.2f} GB per step vs {L2_BYTES / 2**20:.0f} MiB)"},
            "roofline": roof,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h)},
            "gpu_launches": int(launches * args.steps),
            "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.profile:
        cb = cpu_baseline(cfg)
        cb.pop("seconds", None)
        line["cpu_baseline"] = cb
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
