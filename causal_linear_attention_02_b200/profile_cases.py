"""Fixed-size invocations of the library's kernels, for profilers.

    python -m causal_linear_attention_02_b200.profile_cases prefill [--tokens T] [--calls N]
    python -m causal_linear_attention_02_b200.profile_cases decode [--batch B] [--calls N]
    python -m causal_linear_attention_02_b200.profile_cases prefill_decay [--tokens T] [--calls N]
    python -m causal_linear_attention_02_b200.profile_cases prefill_varlen [--calls N]

Each case builds seeded synthetic inputs on cuda:0 (the generators of the
`workloads` module), then makes N calls of one entry point through the C ABI
and checks the device status afterwards, so that a profiler can select the
k-th launch of a kernel (`-k`, `-s`, `-c`) without the rest of a benchmark.

prefill: bf16, 64 heads, d = 128, B = 256, one sequence of T tokens
         (default 32768: Q, K, V, O of 0.5 GB each, larger than the L2).
decode:  bf16 inputs, 64 heads, d = 128, fp32 states of `batch` sequences
         (default 256: 1 GiB of state), states drawn iid instead of from a prefill.
prefill_decay: as prefill, through la_prefill_decay with the per-head rates
         lambda_h = exp(-2^(-8 (h+1) / H)) of `workloads.decay_rates`.
prefill_varlen: the packed 16-sequence workload (lengths iid U[1024, 65536],
         seed 4; 657,303 tokens), 64 heads, d = 128, B = 256, int32 cu_seqlens.

--path 1 or 2 forces the on-chip-state or the block-parallel look-back kernel for the
bf16 prefills (la_debug_set_path); 0 keeps the automatic choice.
"""
from __future__ import annotations

import argparse
import ctypes
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import causal_linear_attention_02_b200 as la  # noqa: E402
import workloads as wl  # noqa: E402


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def prefill_case(tokens: int, calls: int, decay: bool = False, lengths=None, seed: int = 2) -> None:
    dev = torch.device("cuda", 0)
    H, d, B = 64, 128, 256
    if lengths is not None:
        tokens = int(sum(lengths))
    nseq = 1 if lengths is None else len(lengths)
    q, k, v = wl.qkv(tokens, H, d, torch.bfloat16, seed, device=dev)
    o = torch.empty_like(q)
    cu = None if lengths is None else wl.cu_seqlens(lengths, device=dev)
    cu_p = None if cu is None else _ptr(cu)
    rates = wl.decay_rates(H, device=dev) if decay else None
    size = la.la_prefill_decay_workspace_size if decay else la.la_prefill_workspace_size
    ws_bytes = size(tokens, nseq, H, d, B, la.LA_BF16)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    sh = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    for _ in range(calls):
        if decay:
            s = la.la_prefill_decay(_ptr(q), _ptr(k), _ptr(v), _ptr(o), cu_p, nseq, tokens, H, d, B, la.LA_BF16,
                                    None, _ptr(rates), None, _ptr(ws), ws_bytes, sh)
        else:
            s = la.la_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(o), cu_p, nseq, tokens, H, d, B, la.LA_BF16, None,
                              _ptr(ws), ws_bytes, sh)
        if s != 0:
            raise la.LightningError(f"prefill: {la.STATUS.get(s, s)}", s)
    torch.cuda.synchronize(dev)
    if la.device_status() != 0:
        raise la.LightningError("device status after prefill")
    print(f"prefill{' with decay' if decay else ''} T={tokens} sequences={nseq} H={H} d={d} B={B}: "
          f"{calls} calls ok")


def decode_case(batch: int, calls: int) -> None:
    dev = torch.device("cuda", 0)
    H, d = 64, 128
    state = wl.state_init(batch, H, d, seed=5, device=dev)
    qs, ks, vs = wl.decode_inputs(batch, H, d, calls, torch.bfloat16, 5, device=dev)
    o = torch.empty((batch, H, d), dtype=torch.bfloat16, device=dev)
    sh = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    for i in range(calls):
        s = la.la_decode_step(_ptr(qs[i]), _ptr(ks[i]), _ptr(vs[i]), _ptr(state), _ptr(o), batch, H, d,
                              la.LA_BF16, sh)
        if s != 0:
            raise la.LightningError(f"la_decode_step: {la.STATUS.get(s, s)}", s)
    torch.cuda.synchronize(dev)
    if la.device_status() != 0:
        raise la.LightningError("device status after decode")
    print(f"decode batch={batch} H={H} d={d}: {calls} calls ok")


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["prefill", "decode", "prefill_decay", "prefill_varlen"])
    ap.add_argument("--tokens", type=int, default=32768)
    ap.add_argument("--batch", type=int, default=256)
    ap.add_argument("--calls", type=int, default=2)
    ap.add_argument("--path", type=int, default=0,
                    help="bf16 prefill kernel: 0 automatic, 1 on-chip-state, 2 block-parallel look-back")
    a = ap.parse_args()
    la.load_library()
    if a.path and la.la_debug_set_path(a.path) != 0:
        raise la.LightningError(f"la_debug_set_path({a.path}) refused")
    if a.case in ("prefill", "prefill_decay"):
        prefill_case(a.tokens, a.calls, decay=a.case == "prefill_decay")
    elif a.case == "prefill_varlen":
        w = wl.BF16_VARLEN
        prefill_case(0, a.calls, lengths=list(w.seq_lens), seed=w.seed)
    else:
        decode_case(a.batch, a.calls)


if __name__ == "__main__":
    main()
