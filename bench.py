"""Benchmark of the Lightning Attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {cuda,reference}]

One step = one bf16 prefill (la_prefill) of the 32k-token workload: T = 32768
tokens, H = 64 heads, d = 128, B = 256, Q, K, V iid N(0,1) * d^-1/2 in bf16
(inputs 1.6 GB > L2, so nothing is flushed between steps). Rank 0 prints one
JSON line with tokens/s (whole job), TFLOP/s counted as 4*B*d + 4*d^2 per
token per head, the roofline of the main kernel (timed live with CUDA events
on its stream via la_set_kernel_timer), the decode step of the batched decode
workload (256 sequences x 64 heads, 128x128 fp32 states) as a sub-measurement,
an end-to-end number through host buffers, SM clocks sampled during the timed
region and the fp64 CPU oracle timed on a bounded sample on the host cores.

With N > 1 (torchrun, one process per GPU) every rank runs its own
independent prefill of the same size (weak scaling, no collective on the data
path); the timed region is bracketed by a barrier and a device synchronise on
every rank, and the time reported is the maximum over ranks.

--impl reference times the fp64 CPU oracle (the method written out plainly,
no tiling) on rank 0 over a bounded sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as wl  # noqa: E402

METRIC = "prefill tokens/s & TFLOP/s (% bf16 TC peak); decode state GB/s (% HBM)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def flops_per_token_head(B, d):
    return 4 * B * d + 4 * d * d


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": sorted(reasons)}
        loaded = [x for x in sm if smax and x > 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------------------- distributed
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus and world > 1:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
        pg = dist
    return rank, local, world, pg


def barrier(pg, local):
    if pg is not None:
        pg.barrier(device_ids=[local])


def max_over_ranks(pg, x: float) -> float:
    if pg is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------- cpu baseline
def cpu_oracle_sample(w, budget_s=15.0, seed_offset=0):
    """Times the fp64 oracle (recurrent form, OpenMP over heads) on a bounded
    sample of whole heads of the workload; returns tokens/s for the full
    workload's head count and a description of the sample."""
    import numpy as np
    import oracle
    T, H, d = w.total_tokens, w.heads, w.d
    threads = oracle.num_threads()
    # calibrate on one head of 2048 tokens
    q, k, v = (x.float().numpy().astype(np.float64) for x in wl.qkv(2048, 1, d, torch.bfloat16, w.seed + 17))
    t0 = time.perf_counter()
    oracle.recurrent(q, k, v)
    per_tok_head = (time.perf_counter() - t0) / 2048
    n_heads = max(1, min(H, int(budget_s * threads / (per_tok_head * T))))
    q, k, v = (x.float().numpy().astype(np.float64)
               for x in wl.qkv(T, n_heads, d, torch.bfloat16, w.seed + seed_offset))
    t0 = time.perf_counter()
    oracle.recurrent(q, k, v)
    dt = time.perf_counter() - t0
    tok_heads = T * n_heads
    return {"value": tok_heads / dt / H, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"fp64 recurrent oracle on {n_heads} of {H} heads x {T} tokens (d={d}), "
                      f"{dt:.1f} s; tokens/s = token-heads/s / {H}",
            "seconds": dt}


# ---------------------------------------------------------------------------- cuda arm
def run_cuda(args):
    import ctypes
    import causal_linear_attention_02_b200 as la

    rank, local, world, pg = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    la.load_library()
    pk, pk_kind = peaks()
    w = wl.BF16_32K
    T, H, d, B = w.total_tokens, w.heads, w.d, w.B
    q, k, v = wl.qkv(T, H, d, torch.bfloat16, w.seed + 7919 * rank, device=dev)
    o = torch.empty_like(q)
    ws_bytes = la.la_prefill_workspace_size(T, 1, H, d, B, la.LA_BF16)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = ctypes.c_void_p(stream.cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())

    def step(timer=None):
        if timer is not None:
            la.la_set_kernel_timer(ctypes.c_void_p(timer[0].cuda_event), ctypes.c_void_p(timer[1].cuda_event))
        s = la.la_prefill(P(q), P(k), P(v), P(o), None, 1, T, H, d, B, la.LA_BF16, None, P(ws), ws_bytes, sh)
        if s != 0:
            raise RuntimeError(f"la_prefill failed: {la.STATUS.get(s, s)}")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if la.device_status() != 0:
        raise RuntimeError("device status after warm-up")

    timers = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in timers:          # materialise the CUDA events
        a.record(); b.record()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        barrier(pg, local)
        torch.cuda.synchronize(dev)
        start.record(stream)
        for i in range(args.steps):
            step(timers[i])
        stop.record(stream)
        torch.cuda.synchronize(dev)
        barrier(pg, local)
    elapsed_ms = max_over_ranks(pg, start.elapsed_time(stop))
    kernel_ms = max_over_ranks(pg, statistics.mean(a.elapsed_time(b) for a, b in timers))
    if la.device_status() != 0:
        raise RuntimeError("device status after timed region")
    clk = clocks.summary()
    ms_per_step = elapsed_ms / args.steps
    tokens = T * args.steps * world
    value = tokens / (elapsed_ms / 1e3)
    flops_step = flops_per_token_head(B, d) * T * H
    tflops = flops_step * world / (ms_per_step / 1e3) / 1e12
    alg_bytes = 8 * d * T * H                      # read Q, K, V + write O, bf16
    achieved_gbs = alg_bytes / (kernel_ms / 1e3) / 1e9

    # ---- decode sub-measurement (batched decode workload, fp32 states)
    dec = None
    if not args.no_decode:
        dec = run_decode(la, dev, stream, args, pk, pg, local)

    # ---- end to end through host buffers: H2D q,k,v (pinned) + la_prefill + D2H o, per step
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    e2e_steps = max(1, min(args.steps, 5))
    for _ in range(1):
        q.copy_(hq, non_blocking=True); k.copy_(hk, non_blocking=True); v.copy_(hv, non_blocking=True)
        step(); ho.copy_(o, non_blocking=True)
    torch.cuda.synchronize(dev)
    barrier(pg, local)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        q.copy_(hq, non_blocking=True); k.copy_(hk, non_blocking=True); v.copy_(hv, non_blocking=True)
        step()
        ho.copy_(o, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(pg, local)
    e2e_ms = max_over_ranks(pg, e0.elapsed_time(e1))
    e2e = {"value": T * e2e_steps * world / (e2e_ms / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
           "d2h_bytes_per_step": o.numel() * o.element_size(), "steps": e2e_steps}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(w)
        cpu.pop("seconds", None)

    if rank == 0:
        launches_per_step = 5 if la.uses_tensor_cores(torch.bfloat16, d, B) else 5
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "tokens": T, "heads": H, "d": d, "B": B, "seed": w.seed,
                       "l2": "no flush: Q, K, V (1.6 GB) and O (0.5 GB) exceed the 126 MB L2",
                       "parallelism": f"independent problem per GPU x{world}"},
            "tflops": tflops,
            "tc_peak_frac": tflops / world / pk["bf16_tflops"],
            "tc_peak_kind": f"{pk_kind} bf16 {pk['bf16_tflops']} TFLOP/s (burst)",
            "roofline": {"bound": "hbm", "kernel": "prefill main kernel", "achieved": achieved_gbs,
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": achieved_gbs / pk["hbm_gbs"],
                         "peak_kind": pk_kind, "traffic": None, "kernel_ms": kernel_ms,
                         "algorithmic_bytes": alg_bytes},
            "decode": dec,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def run_decode(la, dev, stream, args, pk, pg, local):
    """Batched decode: 256 sequences x 64 heads, d = 128, fp32 states initialised
    from a 4096-token prefill per sequence; steps of fresh bf16 q, k, v."""
    import ctypes
    w = wl.DECODE
    Bt, H, d = w.decode_batch, w.heads, w.d
    n_steps = min(w.decode_steps, max(args.steps * 10, 50))
    T0 = Bt * w.prefill_len
    k0 = wl.normal_scaled((T0, H, d), d, torch.bfloat16, w.seed * 1000 + 1, device=dev)
    v0 = wl.normal_scaled((T0, H, d), d, torch.bfloat16, w.seed * 1000 + 2, device=dev)
    cu = wl.cu_seqlens([w.prefill_len] * Bt, device=dev)
    state = la.state_from_prefill(k0, v0, cu)
    del k0, v0
    torch.cuda.empty_cache()
    qs, ks, vs = wl.decode_inputs(Bt, H, d, n_steps, torch.bfloat16, w.seed, device=dev)
    o = torch.empty((Bt, H, d), dtype=torch.bfloat16, device=dev)
    sh = ctypes.c_void_p(stream.cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())

    def step(i, timer=None):
        if timer is not None:
            la.la_set_kernel_timer(ctypes.c_void_p(timer[0].cuda_event), ctypes.c_void_p(timer[1].cuda_event))
        s = la.la_decode_step(P(qs[i]), P(ks[i]), P(vs[i]), P(state), P(o), Bt, H, d, la.LA_BF16, sh)
        if s != 0:
            raise RuntimeError(f"la_decode_step failed: {la.STATUS.get(s, s)}")

    for i in range(max(3, args.warmup)):
        step(i % n_steps)
    timers = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_steps)]
    for a, b in timers:
        a.record(); b.record()
    torch.cuda.synchronize(dev)
    barrier(pg, local)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for i in range(n_steps):
        step(i, timers[i])
    a1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(pg, local)
    ms = max_over_ranks(pg, a0.elapsed_time(a1)) / n_steps
    kms = max_over_ranks(pg, statistics.mean(a.elapsed_time(b) for a, b in timers))
    state_bytes = 2 * 4 * d * d * Bt * H
    io_bytes = 4 * 2 * d * Bt * H
    gbs = (state_bytes + io_bytes) / (kms / 1e3) / 1e9
    if la.device_status() != 0:
        raise RuntimeError("device status after decode")
    return {"workload": w.name, "steps": n_steps, "ms_per_step": ms, "kernel_ms": kms,
            "value": gbs, "unit": "GB/s", "hbm_frac": gbs / pk["hbm_gbs"],
            "tokens_per_s": Bt / (ms / 1e3),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": None,
                         "algorithmic_bytes": state_bytes + io_bytes}}


# ---------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import numpy as np
    import oracle
    w = wl.BF16_32K
    T, H, d, B = w.total_tokens, w.heads, w.d, w.B
    threads = oracle.num_threads()
    # one step = the oracle over a bounded sample of heads (full sequence length)
    q1, k1, v1 = (x.float().numpy().astype(np.float64) for x in wl.qkv(1024, 1, d, torch.bfloat16, w.seed + 5))
    t0 = time.perf_counter()
    oracle.recurrent(q1, k1, v1)
    per = (time.perf_counter() - t0) / 1024
    budget = 60.0 / max(1, args.steps + args.warmup)
    n_heads = max(1, min(H, int(budget * threads / (per * T))))
    q, k, v = (x.float().numpy().astype(np.float64) for x in wl.qkv(T, n_heads, d, torch.bfloat16, w.seed))
    for _ in range(args.warmup):
        oracle.recurrent(q, k, v)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.recurrent(q, k, v)
    dt = (time.perf_counter() - t0) / args.steps
    value = T * n_heads / dt / H
    sample = (f"fp64 recurrent oracle on {n_heads} of {H} heads x {T} tokens (d={d}) per step; "
              f"tokens/s = token-heads/s / {H}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 * H / n_heads,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "tokens": T, "heads": H, "d": d, "B": B, "seed": w.seed},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
