"""Benchmark of the FG^2-GDN chunkwise forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one gdn_chunk_fwd (or gdn_deltaproduct_fwd) call over one batch of
seeded synthetic input of the named workload (default: the 32K-token FG^2-GDN
prefill, B=1, H=16, T=32768, d=128, chunk 64, bf16).  Prints one JSON line.

  value     tokens/s (B*T per second, all heads, all ranks) with inputs resident
            in HBM, timed with CUDA events on the launching stream.
  e2e       the same metric through the C ABI with pinned host buffers: each step
            copies its inputs host->device, runs the call and reads out and
            S_final back, inside the timed region.  Consecutive steps are
            pipelined over two buffer sets (inputs in on one stream, the call on
            the launching stream, results out on a third), as a streaming caller
            would do; the first copy-in and the last copy-out are not hidden.
  roofline  algorithmic bytes per call / call time against the measured HBM copy
            bandwidth (the path is HBM-bound: about 80 flop per byte against a
            ridge near 250).
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
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, kind)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        burst = float(d["bf16_tflops"])
        return float(d["hbm_gbs"]), burst, float(d.get("bf16_tflops_sustained", burst)), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


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


TC_SOURCES = ("gdn_tc.cu", "gdn_tc2.cu", "gdn_scan2.cu", "gdn_tc_common.cuh",
              "gdn_sm100.cuh", "gdn_common.cuh")     # the timed kernels' own code


def code_only(text: str) -> str:
    """C/CUDA source without its comments and trailing blanks: what the compiler sees as
    code, so that an edit of a comment does not count as a change of the kernel."""
    out, i, n, in_str = [], 0, len(text), None
    while i < n:
        c = text[i]
        if in_str:
            out.append(c)
            if c == "\\" and i + 1 < n:
                out.append(text[i + 1])
                i += 1
            elif c == in_str:
                in_str = None
        elif c in "\"'":
            in_str = c
            out.append(c)
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
            continue
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            continue
        else:
            out.append(c)
        i += 1
    lines = (l.rstrip() for l in "".join(out).splitlines())
    return "\n".join(l for l in lines if l)


def source_hash() -> str:
    """Hash of the code (comments dropped) of the kernels bench.py times; traffic counters
    taken on other code are not reported."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_fg_b200", "csrc")
    for n in TC_SOURCES:
        with open(os.path.join(csrc, n), encoding="utf-8") as f:
            h.update(n.encode())
            h.update(code_only(f.read()).encode())
    return h.hexdigest()[:16]


class ClockSampler:
    """nvidia-smi clock / throttle sampling in the background (every 200 ms)."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        import tempfile
        self.path = os.path.join(tempfile.gettempdir(), f"gdn_bench_clocks_gpu{gpu_index}_{os.getpid()}.csv")

    def start(self):
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


def cpu_baseline(cfg, target_s: float = 12.0):
    """Time the fp64 oracle (as it stands) on a bounded sample: whole heads of the
    workload, as many as fit in about target_s seconds, one head per thread."""
    import oracle
    threads = oracle.max_threads()
    x1_T = min(cfg.T, 2048)
    x = make_inputs(cfg, T=x1_T, H=1, B=1)
    t0 = time.perf_counter()
    if cfg.deltaproduct_nh:
        oracle.deltaproduct_seq(x["q"], x["k"], x["v"], x["gamma"], x["beta"], x["S0"], nthreads=1)
    else:
        oracle.gdn_seq(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"],
                       alpha_scalar=cfg.alpha_scalar, beta_scalar=cfg.beta_scalar, nthreads=1)
    per_tok_head = (time.perf_counter() - t0) / x["q"].shape[1]
    one_core = 1.0 / (per_tok_head * cfg.H)        # tokens/s (all H heads) on one core
    # heads run in parallel, one per thread; pick a sample of whole heads that fits target_s
    nheads = max(1, min(cfg.B * cfg.H, threads))
    T_s = int(max(256, min(cfg.T, target_s / max(per_tok_head, 1e-9))))
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
            "one_core_value": one_core,
            "one_core_sample": f"1 head x {x1_T} tokens of {cfg.name} on one thread",
            "nproc": os.cpu_count(), "cpu_model": oracle.host_cpu(),
            "build": "gcc -O3 -march=native -fopenmp",
            "seconds": dt}


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    vals, last = [], None
    # each step is a bounded sample, sized so that warm-up + timed steps end within minutes
    per_step_s = max(0.5, min(args.ref_seconds, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(max(0, args.warmup)):
        cpu_baseline(cfg, target_s=per_step_s)
    for _ in range(args.steps):
        last = cpu_baseline(cfg, target_s=per_step_s)
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


def max_over_ranks(x: float, device, world: int) -> float:
    """The largest of every rank's x (each rank passes its own): all-reduce MAX."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(units_per_rank: int, world: int, ms_per_step: float) -> float:
    """Units all ranks processed per second, timed by the slowest rank (weak scaling)."""
    return units_per_rank * world / (ms_per_step / 1000.0)


class Op:
    """What one bench step runs: device inputs, the step, and the numbers that describe it."""

    def __init__(self, **kw):
        self.__dict__.update(kw)


def _fwd_bytes(cfg, plus=False):
    return algorithmic_bytes(cfg) + (cfg.B * cfg.T * cfg.H * (4 if cfg.beta_scalar else 4 * cfg.dv)
                                      if plus else 0)


def build_op(args, cfg, ops, torch, dev, stream, rank):
    """Inputs (resident in HBM, one replica per rank with its own seed) and the step for --op."""
    import dataclasses
    from gated_delta_rule_fg_b200.inputs import GdnConfig, round_bf16
    op = args.op
    if op == "plus":
        cfg = dataclasses.replace(cfg, plus=True, name=cfg.name + "+plus")
    if op == "decode":
        B = args.B if args.B is not None else 256
        H = args.H if args.H is not None else cfg.H
        cfg = GdnConfig(f"decode_b{B}_h{H}_d{cfg.dk}", B=B, H=H, T=1, dk=cfg.dk, dv=cfg.dv, chunk=cfg.chunk,
                        dtype=cfg.dtype, s0_std=0.01, seed=6)
    x = make_inputs(cfg, seed=cfg.seed + 1000 * rank)
    if op == "decode":      # one token: drop the T axis
        x = {k: (np.ascontiguousarray(v[:, 0]) if (v is not None and k != "S0") else v) for k, v in x.items()}
    if op == "bwd":
        r = np.random.default_rng(cfg.seed + 7)
        dO = r.standard_normal((cfg.B, cfg.T, cfg.H, cfg.dv), dtype=np.float32)
        x["dO"] = round_bf16(dO) if cfg.dtype == "bf16" else dO
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    host = {k: (torch.from_numpy(v).pin_memory() if v is not None else None) for k, v in x.items()}
    for kname in ("q", "k", "v", "dO"):
        if kname in host:
            host[kname] = host[kname].to(dt).pin_memory()
    d = {k: (v.to(dev, non_blocking=False) if v is not None else None) for k, v in host.items()}
    dp = cfg.deltaproduct_nh > 0
    code = ops.GDN_BF16 if cfg.dtype == "bf16" else ops.GDN_F32
    B, T, H = cfg.B, cfg.T, cfg.H
    flags = (ops.GDN_ALPHA_SCALAR if cfg.alpha_scalar else 0) | (ops.GDN_BETA_SCALAR if cfg.beta_scalar else 0)
    e = 2 if cfg.dtype == "bf16" else 4
    th = B * T * H

    if op == "decode":
        S = d["S0"]
        o = torch.empty((B, H, cfg.dv), dtype=dt, device=dev)

        def step(src, outs=None):
            ops.recurrent_step(src["q"], src["k"], src["v"], src["alpha"], src["beta"], S, in_place=True,
                               out=o if outs is None else outs[0], stream=stream)
        per_head = 2 * cfg.dk * cfg.dv * 4 + (2 * cfg.dk + 2 * cfg.dv) * e + 2 * cfg.dk * 4
        return Op(cfg=cfg, d=d, host=host, step=step, launches=1, ws=None,
                  abytes=B * H * per_head, flops=float(B * H * 6 * cfg.dk * cfg.dv), tokens=B,
                  metric=f"tokens/s FG²-GDN decode step (B={B} sequences, H={H}, d={cfg.dk}), 1 B200",
                  e2e_in=["q", "k", "v", "alpha", "beta"], e2e_out=[o], kernel="gdn_recurrent_step")
    if op == "gdn2":
        from gated_delta_rule_fg_b200.inputs import make_gdn2_inputs
        chunk = cfg.chunk
        g = make_gdn2_inputs(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, dtype=cfg.dtype, seed=cfg.seed + 1000 * rank)
        dg = {k: (torch.from_numpy(v).to(dev) if v is not None else None) for k, v in g.items()}
        for kname in ("q", "k", "v"):
            dg[kname] = dg[kname].to(dt)
        out = torch.empty((B, T, H, cfg.dv), dtype=dt, device=dev)
        Sf = torch.empty((B, H, cfg.dk, cfg.dv), dtype=torch.float32, device=dev)
        nws = ops.gdn2_chunk_fwd_workspace_size(B, H, T, cfg.dk, cfg.dv, chunk, code, 0)
        ws = ops.alloc_workspace(nws, dev)

        def step(src):
            ops.gdn2_chunk_fwd(src["q"], src["k"], src["v"], src["alpha"], src["eta"], src["b"], src["S0"],
                               mode=ops.GDN2_CLIP_DECAY, chunk=chunk, out=out, S_final=Sf, workspace=ws,
                               stream=stream)
        per = (2 * cfg.dk + 2 * cfg.dv) * e + 2 * cfg.dk * 4 + 4
        return Op(cfg=cfg, d=dg, host=None, step=step, ws=ws,
                  launches=int(ops.lib().gdn2_chunk_fwd_launches(B, H, T, cfg.dk, cfg.dv, chunk, code, 0)),
                  abytes=th * per + B * H * cfg.dk * cfg.dv * 4 * 2, flops=algorithmic_flops(cfg), tokens=B * T,
                  metric=f"tokens/s GDN2 chunked fwd with the decay clip (T={T}, d={cfg.dk}, chunk {chunk}), "
                         f"1 B200",
                  e2e_in=None, e2e_out=None, kernel="gdn2_chunk_fwd")
    if op == "bwd":
        chunk = args.chunk if args.chunk is not None else 16
        nws = ops.chunk_bwd_workspace_size(B, H, T, cfg.dk, cfg.dv, chunk, code, flags)
        ws = ops.alloc_workspace(nws, dev)
        res = {}

        def step(src):
            res["g"] = ops.chunk_bwd(src["q"], src["k"], src["v"], src["alpha"], src["beta"], src["S0"], src["dO"],
                                     None, chunk=chunk, alpha_scalar=cfg.alpha_scalar,
                                     beta_scalar=cfg.beta_scalar, workspace=ws, stream=stream)
        per = (2 * cfg.dk + cfg.dv) * e + cfg.dv * e + 2 * cfg.dk * 4 + (3 * cfg.dk + cfg.dv) * 4 + 4 * cfg.dk
        return Op(cfg=cfg, d=d, host=host, step=step, ws=ws,
                  launches=ops.chunk_bwd_launches(B, H, T, cfg.dk, cfg.dv, chunk, code, flags),
                  abytes=th * per + B * H * cfg.dk * cfg.dv * 4 * (2 if cfg.s0_std > 0 else 1),
                  flops=3.0 * algorithmic_flops(cfg), tokens=B * T,
                  metric=f"tokens/s FG²-GDN chunked bwd (T={T}, d={cfg.dk}, chunk {chunk}), 1 B200",
                  e2e_in=None, e2e_out=None, kernel="gdn_chunk_bwd", chunk=chunk)

    out = torch.empty((B, T, H, cfg.dv), dtype=dt, device=dev)
    Sf = torch.empty((B, H, cfg.dk, cfg.dv), dtype=torch.float32, device=dev)
    if dp:
        nws = ops.deltaproduct_fwd_workspace_size(B, H, T, cfg.deltaproduct_nh, cfg.dk, cfg.dv, cfg.chunk, code)
        launches = ops.deltaproduct_fwd_launches(B, H, T, cfg.deltaproduct_nh, cfg.dk, cfg.dv, cfg.chunk, code)
    elif op == "plus":
        nws = ops.plus_chunk_fwd_workspace_size(B, H, T, cfg.dk, cfg.dv, cfg.chunk, code, flags)
        launches = ops.plus_chunk_fwd_launches(B, H, T, cfg.dk, cfg.dv, cfg.chunk, code, flags)
    else:
        nws = ops.chunk_fwd_workspace_size(B, H, T, cfg.dk, cfg.dv, cfg.chunk, code, flags)
        launches = ops.chunk_fwd_launches(B, H, T, cfg.dk, cfg.dv, cfg.chunk, code, flags)
    ws = ops.alloc_workspace(nws, dev)

    def step(src, outs=None):
        o_, s_ = (out, Sf) if outs is None else outs
        if dp:
            ops.deltaproduct_fwd(src["q"], src["k"], src["v"], src["gamma"], src["beta"], src["S0"],
                                 chunk=cfg.chunk, out=o_, S_final=s_, workspace=ws, stream=stream)
        elif op == "plus":
            ops.plus_chunk_fwd(src["q"], src["k"], src["v"], src["alpha"], src["beta"], src["beta_v"], src["S0"],
                               chunk=cfg.chunk, alpha_scalar=cfg.alpha_scalar, beta_scalar=cfg.beta_scalar,
                               out=o_, S_final=s_, workspace=ws, stream=stream)
        else:
            ops.chunk_fwd(src["q"], src["k"], src["v"], src["alpha"], src["beta"], src["S0"],
                          chunk=cfg.chunk, alpha_scalar=cfg.alpha_scalar, beta_scalar=cfg.beta_scalar,
                          out=o_, S_final=s_, workspace=ws, stream=stream)
    names = ["q", "k", "v", "gamma" if dp else "alpha", "beta"] + (["beta_v"] if op == "plus" else []) + ["S0"]
    metric = METRIC if op == "fwd" else "tokens/s FG²-GDN+ chunked fwd (T=32K, d=128) and % of roofline, 1 B200"
    return Op(cfg=cfg, d=d, host=host, step=step, ws=ws, launches=launches,
              abytes=_fwd_bytes(cfg, op == "plus"), flops=algorithmic_flops(cfg), tokens=B * T,
              metric=metric, e2e_in=names, e2e_out=[out, Sf], kernel="gdn_chunk_fwd")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="fg2_prefill_32k", choices=sorted(CONFIGS))
    ap.add_argument("--op", default="fwd", choices=["fwd", "plus", "decode", "bwd", "gdn2"],
                    help="fwd: the chunked forward (the headline); plus: FG²-GDN+ forward; decode: one "
                         "recurrent step per sequence (B=256 by default); bwd: the chunked backward; "
                         "gdn2: GDN2 with the decay clip")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--ref-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="only warm-up + timed steps (no clock soak, e2e or CPU baseline), for ncu")
    ap.add_argument("--B", type=int, default=None, help="override the workload's batch (small ncu captures)")
    ap.add_argument("--H", type=int, default=None, help="override the workload's heads")
    ap.add_argument("--T", type=int, default=None, help="override the workload's tokens per sequence")
    ap.add_argument("--chunk", type=int, default=None,
                    help="override the chunk length (the backward's default is 16)")
    args = ap.parse_args()
    cfg = CONFIGS[args.workload]
    over = {k: getattr(args, k) for k in ("B", "H", "T") if getattr(args, k) is not None}
    if args.chunk is not None and args.op != "bwd":
        over["chunk"] = args.chunk
    if over and args.op != "decode":
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

    op = build_op(args, cfg, ops, torch, dev, stream, rank)
    cfg, d, host, step, ws = op.cfg, op.d, op.host, op.step, op.ws

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        step(d)
    if ws is not None:
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
    call_ms = [a.elapsed_time(b) for a, b in ev]
    per_call_ms = float(np.mean(call_ms))
    per_call_ms_median = float(np.median(call_ms))
    if ws is not None:
        status = ops.workspace_status(ws)
        if status != ops.GDN_OK:
            raise SystemExit(f"device status after the timed region: {ops.status_string(status)}")
    total_ms = max_over_ranks(total_ms, dev, world)
    ms_per_step = total_ms / args.steps
    tokens = op.tokens * world
    value = whole_job_value(op.tokens, world, ms_per_step)

    # ---- end to end through the C ABI with pinned host buffers
    e2e = None
    if op.e2e_in is not None and not args.profile:
        names = op.e2e_in
        h2d = sum(host[n].numel() * host[n].element_size() for n in names if host[n] is not None)
        # Two buffer sets and three streams: step k+1's inputs go host->device on `cs` and
        # step k-1's results device->host on `ds` while step k computes on `stream`; events
        # keep each buffer from being overwritten before its reader is done.
        outs_h = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in op.e2e_out] for _ in range(2)]
        d2h = sum(t.numel() * t.element_size() for t in outs_h[0])
        dev_in, dev_out = [], []
        for _ in range(2):
            di = dict(d)
            for n in names:
                di[n] = torch.empty_like(d[n]) if d[n] is not None else None
            dev_in.append(di)
            dev_out.append([torch.empty_like(t) for t in op.e2e_out])
        cs, ds = torch.cuda.Stream(), torch.cuda.Stream()
        ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "comp", "out")}
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        cs.wait_event(f0)
        for i in range(args.e2e_steps):
            sl = i % 2
            with torch.cuda.stream(cs):
                if i >= 2:
                    cs.wait_event(ev["comp"][sl])          # step i-2 has finished reading dev_in[sl]
                for n in names:
                    if host[n] is not None:
                        dev_in[sl][n].copy_(host[n], non_blocking=True)
                ev["in"][sl].record(cs)
            stream.wait_event(ev["in"][sl])
            if i >= 2:
                stream.wait_event(ev["out"][sl])           # step i-2's results have left dev_out[sl]
            step(dev_in[sl], dev_out[sl])
            ev["comp"][sl].record(stream)
            with torch.cuda.stream(ds):
                ds.wait_event(ev["comp"][sl])
                for th_, td_ in zip(outs_h[sl], dev_out[sl]):
                    th_.copy_(td_, non_blocking=True)
                ev["out"][sl].record(ds)
        stream.wait_stream(cs)
        stream.wait_stream(ds)
        f1.record(stream)
        barrier()
        e2e_ms = max_over_ranks(f0.elapsed_time(f1) / max(1, args.e2e_steps), dev, world)
        e2e = {"value": whole_job_value(op.tokens, world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h)}

    hbm_gbs, bf16_tf, bf16_tf_sus, peak_kind = load_peaks()
    abytes = op.abytes
    achieved = abytes / (per_call_ms / 1000.0) / 1e9
    kname = op.kernel if op.launches == 1 else f"{op.kernel} ({op.launches} kernels, whole call)"
    traffic = load_traffic(op.kernel, cfg.name, source_hash()) if args.op == "fwd" else None
    roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
            "frac": achieved / hbm_gbs, "traffic": traffic,
            "peak_kind": f"of {peak_kind} copy bandwidth", "kernel": kname,
            "algorithmic_bytes_per_launch": abytes, "algorithmic_flops_per_launch": op.flops,
            "flop_frac_of_bf16_peak": op.flops / (per_call_ms / 1000.0) / (bf16_tf * 1e12),
            "flop_frac_of_bf16_sustained": op.flops / (per_call_ms / 1000.0) / (bf16_tf_sus * 1e12),
            "launch_ms": per_call_ms, "launch_ms_median": per_call_ms_median}

    line = {"metric": op.metric, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": cfg.dtype, "data": "synthetic (seeded numpy draws with the workload's distributions)",
            "config": {"workload": cfg.name, "op": args.op, "B": cfg.B, "H": cfg.H, "T": cfg.T, "dk": cfg.dk,
                       "dv": cfg.dv, "chunk": getattr(op, "chunk", cfg.chunk), "per_rank": "one replica per GPU",
                       "l2": f"inputs larger than L2 ({abytes / 1e9:.2f} GB per step vs {L2_BYTES / 2**20:.0f} MiB)"},
            "roofline": roof,
            "e2e": e2e if e2e is not None else {"value": None, "unit": "tokens/s",
                                                "note": "not measured under --profile" if args.profile
                                                else "measured for the forward ops only"},
            "gpu_launches": int(op.launches * args.steps),
            "clocks": clk}
    if rank == 0 and world == 1 and args.op == "fwd" and not args.no_cpu_baseline and not args.profile:
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
