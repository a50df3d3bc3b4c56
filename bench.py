"""Benchmark of the Lightning Attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {cuda,reference}]

One step = one bf16 prefill (la_prefill) of the 32k-token workload: T = 32768
tokens, H = 64 heads, d = 128, B = 256, Q, K, V iid N(0,1) * d^-1/2 in bf16
(inputs 1.6 GB > L2, so nothing is flushed between steps). Rank 0 prints one
JSON line with tokens/s (whole job), TFLOP/s counted as 4*B*d + 4*d^2 per
token per head, the roofline of the main kernel (timed live with CUDA events
on its stream via la_set_kernel_timer), an end-to-end number through host
buffers, SM clocks sampled during the timed region and the fp64 CPU oracle
timed on a bounded sample on the host cores. Sub-measurements of the same line,
each timed with CUDA events on its own stream after warm-up calls:

  decode    the batched decode workload (256 sequences x 64 heads, 128x128
            fp32 states, 1000 steps), GB/s against HBM; decode.decay the same
            with a decay rate per head
  decay     the prefill with a decay rate per head on the 32k inputs
  long      the million-token prefill (T = 1,048,576, H = 64), roofline and
            DRAM traffic of its launch
  varlen    the packed prefill of 16 sequences of U[1024, 65536] tokens
  backward  la_prefill_backward on the 32k inputs (dq, dk, dv, dS0)
  mixed     one la_prefill_with_state launch over 4 prompts and 2000
            one-token continuations, beside the split form (prompts through
            la_prefill_with_state, the continuations through la_decode_step)

--no-decode, --no-decay, --no-big (long, varlen), --no-backward, --no-mixed and
--no-cpu-baseline leave a sub-measurement out.

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
import sys
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


# DRAM bytes per launch of the main kernels (dram__bytes_read.sum +
# dram__bytes_write.sum from one ncu capture), stored in profiles/ with the
# SHA-256 of the kernel's source files at capture time. A figure is reported
# only while those sources are unchanged; otherwise traffic is null.
KERNEL_SOURCES = {
    "prefill_chain_kernel": ("chain.cuh", "pipe.cuh", "sm100.cuh", "common.cuh"),
    "prefill_chain_kernel_decay": ("chain.cuh", "pipe.cuh", "sm100.cuh", "common.cuh", "decay.cuh"),
    "prefill_fused_kernel": ("fused.cuh", "pipe.cuh", "sm100.cuh", "common.cuh"),
    "decode_step_kernel": ("decode.cuh", "common.cuh"),
    # the same kernel on the million-token and varlen workloads (traffic per launch differs)
    "prefill_chain_kernel_1m": ("chain.cuh", "pipe.cuh", "sm100.cuh", "common.cuh"),
    "prefill_chain_kernel_varlen": ("chain.cuh", "pipe.cuh", "sm100.cuh", "common.cuh"),
}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.txt")


def kernel_sources_sha(kernel):
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "causal_linear_attention_02_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def captured_traffic(kernel):
    """Bytes per launch for `kernel` if profiles/ holds a capture of its current sources."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    sha = kernel_sources_sha(kernel)
    for line in open(TRAFFIC_FILE):
        parts = line.split()
        if len(parts) >= 3 and not line.startswith("#") and parts[0] == kernel and parts[1] == sha:
            return float(parts[2])
    return None


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock, power and throttle reasons sampled every few milliseconds (NVML)
    while the timed region runs; read-only queries."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, device, period_s=0.002):
        self.device = device
        self.period = period_s
        self.samples = []
        self.smax = None
        self.err = None
        self._stop = threading.Event()
        self._thread = None

    def _handle(self, nv):
        props = torch.cuda.get_device_properties(self.device)
        bus = getattr(props, "pci_bus_id", None)
        if bus is not None:
            dom = getattr(props, "pci_domain_id", 0)
            devno = getattr(props, "pci_device_id", 0)
            try:
                return nv.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{devno:02x}.0".encode())
            except Exception:
                pass
        return nv.nvmlDeviceGetHandleByIndex(self.device.index or 0)

    def _run(self, nv, h):
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), int(get_reasons(h)),
                                     nv.nvmlDeviceGetPowerUsage(h) / 1000.0))
            except Exception as e:  # noqa: BLE001
                self.err = str(e)
                return
            time.sleep(self.period)

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, args=(nv, h), daemon=True)
            self._thread.start()
        except Exception as e:  # noqa: BLE001
            self.err = f"NVML unavailable: {e}"
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.smax, "reasons": [self.err or "no samples"]}
        sm = [x[0] for x in self.samples]
        reasons = sorted(n for n, bit in self.REASONS.items() if any(x[1] & bit for x in self.samples))
        loaded = [x for x in sm if self.smax and x > 0.5 * self.smax] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": self.smax, "reasons": reasons,
                "samples": len(sm), "sm_mhz_min": min(sm), "power_w_max": max(x[2] for x in self.samples),
                "source": f"NVML, every {self.period * 1e3:g} ms during the timed region"}


# ---------------------------------------------------------------------------- distributed
def dist_setup(n_gpus, backend="nccl"):
    """One process per GPU under torchrun (RANK, LOCAL_RANK, WORLD_SIZE, MASTER_* from the
    environment). The benchmark uses NCCL; gloo serves the host-side tests."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus and world > 1:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
        pg = dist
    return rank, local, world, pg


def _on_gpus(pg) -> bool:
    return pg.get_backend() == "nccl"


def barrier(pg, local):
    if pg is not None:
        if _on_gpus(pg):
            pg.barrier(device_ids=[local])
        else:
            pg.barrier()


def max_over_ranks(pg, x: float) -> float:
    """The largest of the ranks' values (every rank gets it): times are reported as the slowest rank's."""
    if pg is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if _on_gpus(pg) else "cpu")
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
    with ClockSampler(dev) as clocks:
        barrier(pg, local)
        torch.cuda.synchronize(dev)
        launches0 = la.la_launch_count()
        start.record(stream)
        for i in range(args.steps):
            step(timers[i])
        stop.record(stream)
        launches = la.la_launch_count() - launches0
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

    # ---- decay variant on the same inputs (the decay instance of the tensor-core kernel), per-head
    # rates of the decay recipe
    dcy = None
    if not args.no_decay:
        dcy = run_decay(la, dev, stream, args, pk, pg, local, q, k, v, o, w)

    # ---- backward pass on the 32k workload
    bwd = None
    if not args.no_backward:
        bwd = run_backward(la, dev, stream, args, pk, pg, local, q, k, v, w)

    # ---- a serving batch: prompts and one-token continuations in one launch
    mix = None
    if not args.no_mixed:
        mix = run_mixed(la, dev, stream, args, pk, pg, local)
        torch.cuda.empty_cache()

    # ---- the million-token and the varlen workloads (prefill, same kernel)
    big = {}
    if not args.no_big:
        for key, wk in (("long", wl.BF16_1M), ("varlen", wl.BF16_VARLEN)):
            big[key] = run_prefill_workload(la, dev, stream, args, pk, pg, local, wk, key)
            torch.cuda.empty_cache()

    # ---- end to end through host buffers, every step: H2D of q, k, v from pinned host memory,
    # la_prefill, D2H of o. Two device buffer sets and three streams, so that step i+1's upload
    # overlaps step i's compute and download (PCIe is full duplex); every copy is inside the
    # timed region, which runs from an event before the first upload to one after the last download.
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    sets = [(q, k, v, o)] + [tuple(torch.empty_like(t) for t in (q, k, v, o))]
    s_up, s_dn = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    e2e_steps = max(2, min(args.steps, 6))
    up_done = [torch.cuda.Event() for _ in sets]
    comp_done = [torch.cuda.Event() for _ in sets]
    dn_done = [torch.cuda.Event() for _ in sets]

    def e2e_step(i):
        sq, sk, sv, so = sets[i % 2]
        with torch.cuda.stream(s_up):
            if i >= 2:
                s_up.wait_event(comp_done[i % 2])           # the set's inputs were read
            sq.copy_(hq, non_blocking=True); sk.copy_(hk, non_blocking=True); sv.copy_(hv, non_blocking=True)
            up_done[i % 2].record(s_up)
        stream.wait_event(up_done[i % 2])
        if i >= 2:
            stream.wait_event(dn_done[i % 2])               # the set's output was downloaded
        st_ = la.la_prefill(P(sq), P(sk), P(sv), P(so), None, 1, T, H, d, B, la.LA_BF16, None, P(ws), ws_bytes, sh)
        if st_ != 0:
            raise RuntimeError(f"la_prefill failed: {la.STATUS.get(st_, st_)}")
        comp_done[i % 2].record(stream)
        with torch.cuda.stream(s_dn):
            s_dn.wait_event(comp_done[i % 2])
            ho.copy_(so, non_blocking=True)
            dn_done[i % 2].record(s_dn)

    for i in range(2):                                      # warm-up of the copy path
        e2e_step(i)
    torch.cuda.synchronize(dev)
    barrier(pg, local)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    stream.wait_event(e0)
    s_dn.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record(s_dn)                                         # after the last download, which follows all work
    torch.cuda.synchronize(dev)
    barrier(pg, local)
    e2e_ms = max_over_ranks(pg, e0.elapsed_time(e1))
    if la.device_status() != 0:
        raise RuntimeError("device status after the end-to-end steps")
    e2e = {"value": T * e2e_steps * world / (e2e_ms / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
           "d2h_bytes_per_step": o.numel() * o.element_size(), "steps": e2e_steps,
           "pipelining": "two device buffer sets; upload, compute and download on separate streams"}
    del sets

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(w)
        cpu.pop("seconds", None)

    if rank == 0:
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
            "roofline": {"bound": "hbm", "kernel": "prefill_chain_kernel", "achieved": achieved_gbs,
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": achieved_gbs / pk["hbm_gbs"],
                         "peak_kind": pk_kind, "traffic": captured_traffic("prefill_chain_kernel"),
                         "kernel_ms": kernel_ms,
                         "algorithmic_bytes": alg_bytes},
            "decode": dec,
            "decay": dcy,
            "backward": bwd,
            "mixed": mix,
            "long": big.get("long"),
            "varlen": big.get("varlen"),
            "e2e": e2e,
            "gpu_launches": launches,
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
    n_steps = w.decode_steps                     # the workload's 1000 steps, every run
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
    with ClockSampler(dev, period_s=0.002) as clocks:
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
    # the same steps with the decay recipe's per-head rates (la_decode_step_decay)
    decay = wl.decay_rates(H, device=dev)
    dtimers = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_steps)]
    for a, b in dtimers:
        a.record(); b.record()
    for i in range(3):
        la.la_decode_step_decay(P(qs[i]), P(ks[i]), P(vs[i]), P(state), P(o), Bt, H, d, la.LA_BF16, P(decay), sh)
    torch.cuda.synchronize(dev)
    for i in range(n_steps):
        la.la_set_kernel_timer(ctypes.c_void_p(dtimers[i][0].cuda_event), ctypes.c_void_p(dtimers[i][1].cuda_event))
        s = la.la_decode_step_decay(P(qs[i]), P(ks[i]), P(vs[i]), P(state), P(o), Bt, H, d, la.LA_BF16, P(decay), sh)
        if s != 0:
            raise RuntimeError(f"la_decode_step_decay failed: {la.STATUS.get(s, s)}")
    torch.cuda.synchronize(dev)
    if la.device_status() != 0:
        raise RuntimeError("device status after decode with decay")
    dkms = max_over_ranks(pg, statistics.mean(a.elapsed_time(b) for a, b in dtimers))
    dgbs = (state_bytes + io_bytes) / (dkms / 1e3) / 1e9
    return {"workload": w.name, "steps": n_steps, "ms_per_step": ms, "kernel_ms": kms,
            "value": gbs, "unit": "GB/s", "hbm_frac": gbs / pk["hbm_gbs"],
            "tokens_per_s": Bt / (ms / 1e3), "clocks": clocks.summary(),
            "decay": {"kernel_ms": dkms, "value": dgbs, "unit": "GB/s", "hbm_frac": dgbs / pk["hbm_gbs"]},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": captured_traffic("decode_step_kernel"),
                         "algorithmic_bytes": state_bytes + io_bytes}}


def run_decay(la, dev, stream, args, pk, pg, local, q, k, v, o, w):
    """la_prefill_decay on the 32k workload's inputs with the decay recipe's per-head rates
    (lambda_h = exp(-2^(-8 (h+1) / H))): the decay instance of the on-chip-state tensor-core
    kernel. Same algorithmic bytes and counted FLOPs as the prefill without decay."""
    import ctypes
    T, H, d, B = w.total_tokens, w.heads, w.d, w.B
    decay = wl.decay_rates(H, device=dev)
    ws_bytes = la.la_prefill_decay_workspace_size(T, 1, H, d, B, la.LA_BF16)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    sh = ctypes.c_void_p(stream.cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    n = max(10, min(args.steps, 100))

    def step(timer=None):
        if timer is not None:
            la.la_set_kernel_timer(ctypes.c_void_p(timer[0].cuda_event), ctypes.c_void_p(timer[1].cuda_event))
        s = la.la_prefill_decay(P(q), P(k), P(v), P(o), None, 1, T, H, d, B, la.LA_BF16, None, P(decay), None,
                                P(ws), ws_bytes, sh)
        if s != 0:
            raise RuntimeError(f"la_prefill_decay failed: {la.STATUS.get(s, s)}")

    for _ in range(max(3, args.warmup)):
        step()
    timers = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for a, b in timers:
        a.record(); b.record()
    torch.cuda.synchronize(dev)
    barrier(pg, local)
    launches0 = la.la_launch_count()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev, period_s=0.002) as clocks:
        a0.record(stream)
        for i in range(n):
            step(timers[i])
        a1.record(stream)
        launches = la.la_launch_count() - launches0
        torch.cuda.synchronize(dev)
    barrier(pg, local)
    ms = max_over_ranks(pg, a0.elapsed_time(a1)) / n
    kms = max_over_ranks(pg, statistics.mean(a.elapsed_time(b) for a, b in timers))
    if la.device_status() != 0:
        raise RuntimeError("device status after decay prefill")
    del ws
    alg_bytes = 8 * d * T * H
    gbs = alg_bytes / (kms / 1e3) / 1e9
    tflops = flops_per_token_head(B, d) * T * H / (ms / 1e3) / 1e12
    return {"workload": f"bf16 prefill with per-head decay T={T} H={H} d={d} B={B}",
            "rates": "lambda_h = exp(-2^(-8 (h+1) / H)), 0.40 .. 0.996",
            "steps": n, "ms_per_step": ms, "kernel_ms": kms, "tokens_per_s": T / (ms / 1e3),
            "tflops": tflops, "tc_peak_frac": tflops / pk["bf16_tflops"], "launches_per_step": launches / n,
            "clocks": clocks.summary(),
            "roofline": {"bound": "hbm", "kernel": "prefill_chain_kernel (decay instance)", "achieved": gbs,
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                         "traffic": captured_traffic("prefill_chain_kernel_decay"),
                         "algorithmic_bytes": alg_bytes}}


def _timed_calls(la, dev, stream, pg, local, call, n, warmup):
    """n timed calls after `warmup` untimed ones: (ms per call from events around all
    calls, mean main-kernel ms from la_set_kernel_timer, launches per call, SM clocks
    sampled during the timed calls)."""
    import ctypes
    for _ in range(warmup):
        call()
    timers = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for a, b in timers:
        a.record(); b.record()
    torch.cuda.synchronize(dev)
    barrier(pg, local)
    launches0 = la.la_launch_count()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev, period_s=0.002) as clocks:
        a0.record(stream)
        for i in range(n):
            la.la_set_kernel_timer(ctypes.c_void_p(timers[i][0].cuda_event), ctypes.c_void_p(timers[i][1].cuda_event))
            call()
        a1.record(stream)
        launches = la.la_launch_count() - launches0
        torch.cuda.synchronize(dev)
    barrier(pg, local)
    ms = max_over_ranks(pg, a0.elapsed_time(a1)) / n
    kms = max_over_ranks(pg, statistics.mean(a.elapsed_time(b) for a, b in timers))
    if la.device_status() != 0:
        raise RuntimeError("device status after a timed sub-measurement")
    return ms, kms, launches / n, clocks.summary()


def run_prefill_workload(la, dev, stream, args, pk, pg, local, w, key):
    """la_prefill on another workload of the same shape family: the million-token sequence
    (Q, K, V, O of 16 GiB each) or the 16-sequence varlen pack (int32 cu_seqlens, state reset
    at every sequence start). Same kernel, roofline and FLOP count as the main line."""
    import ctypes
    T, H, d, B = w.total_tokens, w.heads, w.d, w.B
    nseq = len(w.seq_lens)
    q, k, v = wl.qkv(T, H, d, torch.bfloat16, w.seed, device=dev)
    o = torch.empty_like(q)
    cu = wl.cu_seqlens(w.seq_lens, device=dev) if nseq > 1 else None
    ws_bytes = la.la_prefill_workspace_size(T, nseq, H, d, B, la.LA_BF16)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    sh = ctypes.c_void_p(stream.cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None

    def call():
        s = la.la_prefill(P(q), P(k), P(v), P(o), P(cu), nseq, T, H, d, B, la.LA_BF16, None, P(ws), ws_bytes, sh)
        if s != 0:
            raise RuntimeError(f"la_prefill ({key}) failed: {la.STATUS.get(s, s)}")

    n = 5 if T > 300000 else 10
    ms, kms, launches, clk = _timed_calls(la, dev, stream, pg, local, call, n, max(3, args.warmup))
    del q, k, v, o, ws
    alg_bytes = 8 * d * T * H
    gbs = alg_bytes / (kms / 1e3) / 1e9
    tflops = flops_per_token_head(B, d) * T * H / (ms / 1e3) / 1e12
    return {"workload": w.name, "tokens": T, "sequences": nseq, "seed": w.seed, "steps": n,
            "ms_per_step": ms, "kernel_ms": kms, "tokens_per_s": T / (ms / 1e3), "tflops": tflops,
            "tc_peak_frac": tflops / pk["bf16_tflops"], "launches_per_step": launches,
            "l2": "no flush: inputs far larger than the 126 MB L2", "clocks": clk,
            "roofline": {"bound": "hbm", "kernel": "prefill_chain_kernel", "achieved": gbs, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                         "traffic": captured_traffic("prefill_chain_kernel_" + ("1m" if key == "long" else key)),
                         "algorithmic_bytes": alg_bytes}}


def run_backward(la, dev, stream, args, pk, pg, local, q, k, v, w):
    """la_prefill_backward on the 32k workload (dO iid like the inputs): dq, dk, dv.
    Its launches run back to back, so the roofline uses the whole call's time:
    algorithmic bytes = read Q, K, V, dO + write dQ, dK, dV (bf16) = 14 d bytes per
    token-head; counted FLOPs = three forward products (dq, dk, dv), 3 (4 B d + 4 d^2)."""
    import ctypes
    T, H, d, B = w.total_tokens, w.heads, w.d, w.B
    do = wl.normal_scaled((T, H, d), d, torch.bfloat16, w.seed * 1000 + 3, device=dev)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws_bytes = la.la_prefill_backward_workspace_size(T, 1, H, d, B, la.LA_BF16)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    sh = ctypes.c_void_p(stream.cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())

    def call():
        s = la.la_prefill_backward(P(q), P(k), P(v), P(do), None, 1, T, H, d, B, la.LA_BF16, None, P(dq), P(dk), P(dv),
                                   None, P(ws), ws_bytes, sh)
        if s != 0:
            raise RuntimeError(f"la_prefill_backward failed: {la.STATUS.get(s, s)}")

    n = 10
    ms, _, launches, clk = _timed_calls(la, dev, stream, pg, local, call, n, max(3, args.warmup))
    del do, dq, dk, dv, ws
    alg_bytes = 14 * d * T * H
    gbs = alg_bytes / (ms / 1e3) / 1e9
    tflops = 3 * flops_per_token_head(B, d) * T * H / (ms / 1e3) / 1e12
    return {"workload": f"backward of the {w.name} prefill (dq, dk, dv)", "steps": n, "ms_per_step": ms,
            "tokens_per_s": T / (ms / 1e3), "tflops": tflops, "tc_peak_frac": tflops / pk["bf16_tflops"],
            "launches_per_step": launches, "clocks": clk,
            "roofline": {"bound": "hbm", "kernel": f"la_prefill_backward (whole call, {launches:g} launches)",
                         "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                         "traffic": None, "algorithmic_bytes": alg_bytes}}


def run_mixed(la, dev, stream, args, pk, pg, local):
    """A serving batch in one launch (la_prefill_with_state): 4 prompts (lengths iid
    U[1024, 5120], seed 6) and 2000 one-token continuations, each sequence with its own
    carried-in fp32 state, H = 64, d = 128, B = 256. Beside it the same work in two calls:
    la_prefill_with_state of the prompts, then la_decode_step of the continuations (whose
    states are one contiguous batch). Algorithmic bytes: 8 d per token-head of Q, K, V, O,
    plus the fp32 states, read (S0) and written (final state), 8 d^2 per (sequence, head)."""
    import ctypes
    H, d, B = 64, 128, 256
    prompts = wl.varlen_lengths(4, 1024, 5120, seed=6)
    n_cont = 2000
    lengths = prompts + [1] * n_cont
    T, nseq, Tp = sum(lengths), len(lengths), sum(prompts)
    q, k, v = wl.qkv(T, H, d, torch.bfloat16, 6, device=dev)
    o = torch.empty_like(q)
    init = wl.state_init(nseq, H, d, seed=6, device=dev, scale=0.2)
    st = torch.empty_like(init)
    cu = wl.cu_seqlens(lengths, device=dev)
    cu_p = wl.cu_seqlens(prompts, device=dev)
    ws_bytes = max(la.la_prefill_with_state_workspace_size(T, nseq, H, d, B, la.LA_BF16),
                   la.la_prefill_with_state_workspace_size(Tp, len(prompts), H, d, B, la.LA_BF16))
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    state_c = init[len(prompts):].clone()                    # the continuations' states, updated in place
    sh = ctypes.c_void_p(stream.cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())

    def mixed():
        s = la.la_prefill_with_state(P(q), P(k), P(v), P(o), P(cu), nseq, T, H, d, B, la.LA_BF16, P(init), P(st),
                                     P(ws), ws_bytes, sh)
        if s != 0:
            raise RuntimeError(f"la_prefill_with_state (mixed batch) failed: {la.STATUS.get(s, s)}")

    def split():
        s = la.la_prefill_with_state(P(q), P(k), P(v), P(o), P(cu_p), len(prompts), Tp, H, d, B, la.LA_BF16,
                                     P(init), P(st), P(ws), ws_bytes, sh)
        if s != 0:
            raise RuntimeError(f"la_prefill_with_state (prompts) failed: {la.STATUS.get(s, s)}")
        s = la.la_decode_step(P(q[Tp:]), P(k[Tp:]), P(v[Tp:]), P(state_c), P(o[Tp:]), n_cont, H, d, la.LA_BF16, sh)
        if s != 0:
            raise RuntimeError(f"la_decode_step (continuations) failed: {la.STATUS.get(s, s)}")

    n = 10
    ms, kms, launches, clk = _timed_calls(la, dev, stream, pg, local, mixed, n, max(3, args.warmup))
    ms_split, _, launches_split, clk_split = _timed_calls(la, dev, stream, pg, local, split, n,
                                                          max(3, args.warmup))
    del q, k, v, o, init, st, ws, state_c
    alg_bytes = 8 * d * T * H + 8 * d * d * nseq * H
    gbs = alg_bytes / (ms / 1e3) / 1e9
    return {"workload": f"serving batch: prompts {prompts} + {n_cont} one-token continuations, H={H} d={d} B={B}, "
                        "each sequence with its own fp32 state", "steps": n,
            "ms_per_step": ms, "kernel_ms": kms, "launches_per_step": launches,
            "split_ms_per_step": ms_split, "split_launches_per_step": launches_split,
            "one_launch_over_split": ms / ms_split, "tokens_per_s": T / (ms / 1e3),
            "clocks": clk, "split_clocks": clk_split,
            "roofline": {"bound": "hbm", "kernel": "prefill_chain_kernel (state-output instance)", "achieved": gbs,
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"], "traffic": None,
                         "algorithmic_bytes": alg_bytes}}


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
    # whole heads, at least one per host thread (the oracle runs heads in parallel)
    n_heads = max(min(H, threads), min(H, int(budget * threads / (per * T))))
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
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": min(threads, n_heads), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-decay", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-mixed", action="store_true")
    ap.add_argument("--no-big", action="store_true", help="skip the million-token and varlen sub-measurements")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
