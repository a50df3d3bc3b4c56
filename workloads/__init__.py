"""Seeded synthetic inputs for causal linear attention.

This module is shared by the oracle side and the CUDA side of the tests and by
the benchmark. It draws inputs only; it holds none of the attention arithmetic.

The workloads mirror the shapes and distributions used to exercise Lightning
Attention prefill and decode (page "MiniMax-01 Lightning Attention": 64 heads of
head dim 128, sections "模型架构" and "Lightning Attention 设计"; block size 256
from page "首个线性注意力架构的大模型来了…", section "4.1 创新的线性注意力"):

    Q, K, V iid N(0, 1) * d^-1/2, rounded to the compute dtype; layout [T, H, d].

Random draws come from torch's seeded generators (Philox on CUDA, mt19937 on
CPU). Large tensors are drawn chunk by chunk so that no fp32 temporary bigger
than ``_CHUNK_ELEMS`` elements is ever allocated.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np
import torch

_CHUNK_ELEMS = 1 << 28  # 1 GiB of fp32 scratch at most


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic configuration (sizes, dtype, seed)."""
    name: str
    dtype: str            # "bf16" or "fp32"
    heads: int
    d: int
    B: int
    seq_lens: tuple       # lengths of the packed sequences
    seed: int
    decode_batch: int = 0  # >0 only for the decode workload
    decode_steps: int = 0
    prefill_len: int = 0   # tokens per sequence used to initialise decode states

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seq_lens))


def varlen_lengths(nseq: int, lo: int, hi: int, seed: int) -> List[int]:
    """`nseq` lengths drawn iid uniform on the integers [lo, hi] (inclusive)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return [int(x) for x in rng.integers(lo, hi + 1, size=nseq)]


def cu_seqlens(lengths: Sequence[int], device="cpu") -> torch.Tensor:
    """int32 offsets [0, l0, l0+l1, ...] of packed sequences."""
    offs = [0]
    for n in lengths:
        if n < 0:
            raise ValueError("sequence lengths must be >= 0")
        offs.append(offs[-1] + int(n))
    if offs[-1] >= 2 ** 31:
        raise ValueError("total tokens must fit in int32 offsets")
    return torch.tensor(offs, dtype=torch.int32, device=device)


# The five workloads: a small fp32 case, the 32k-token bf16 prefill, the
# million-token prefill, a 16-sequence varlen pack and the batched decode.
FP32_SMALL = Workload("fp32 T=1024 H=2 d=64 B=64", "fp32", 2, 64, 64, (1024,), seed=1)
BF16_32K = Workload("bf16 prefill T=32768 H=64 d=128 B=256", "bf16", 64, 128, 256, (32768,), seed=2)
BF16_1M = Workload("bf16 prefill T=1048576 H=64 d=128 B=256", "bf16", 64, 128, 256, (1 << 20,), seed=3)
BF16_VARLEN = Workload("bf16 varlen 16 seqs U[1024,65536] H=64 d=128 B=256", "bf16", 64, 128, 256,
                       tuple(varlen_lengths(16, 1024, 65536, seed=4)), seed=4)
DECODE = Workload("decode batch=256 H=64 d=128 fp32 state, 1000 steps", "bf16", 64, 128, 256,
                  tuple([4096] * 256), seed=5, decode_batch=256, decode_steps=1000, prefill_len=4096)

WORKLOADS = {w.name: w for w in (FP32_SMALL, BF16_32K, BF16_1M, BF16_VARLEN, DECODE)}


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def _generator(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_scaled(shape, d: int, dtype: torch.dtype, seed: int, device="cpu",
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """iid N(0,1) * d^-1/2 drawn in fp32, then rounded (RNE) to `dtype`.

    Drawn in contiguous chunks of the flattened tensor with one generator, so
    the values depend only on (shape, seed, device type).
    """
    device = torch.device(device)
    if out is None:
        out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    g = _generator(device, seed)
    scale = 1.0 / math.sqrt(d)
    n = flat.numel()
    for s in range(0, n, _CHUNK_ELEMS):
        e = min(n, s + _CHUNK_ELEMS)
        tmp = torch.randn(e - s, generator=g, dtype=torch.float32, device=device)
        tmp.mul_(scale)
        flat[s:e].copy_(tmp)
        del tmp
    return out


def qkv(T: int, H: int, d: int, dtype: torch.dtype, seed: int, device="cpu"):
    """Q, K, V of shape [T, H, d]; independent streams per tensor (seed, seed+1, seed+2)."""
    return tuple(normal_scaled((T, H, d), d, dtype, seed * 1000 + i, device) for i in range(3))


def integer_qkv(T: int, H: int, d: int, dtype: torch.dtype, seed: int, device="cpu",
                values=(-1, 0, 1)):
    """Q, K, V with entries drawn uniformly from the small integer set `values`.

    With |values| <= 1, d <= 128 and short sequences every product and partial
    sum in the attention is a small integer, exactly representable in bf16 /
    fp32, so a correct kernel reproduces the fp64 result bit for bit.
    """
    g = _generator("cpu", seed)
    vals = torch.tensor(values, dtype=torch.float32)
    out = []
    for _ in range(3):
        idx = torch.randint(0, len(values), (T, H, d), generator=g)
        out.append(vals[idx].to(dtype).to(device))
    return tuple(out)


def decode_inputs(batch: int, H: int, d: int, steps: int, dtype: torch.dtype, seed: int,
                  device="cpu"):
    """Per-step q, k, v of shape [steps, batch, H, d] (drawn once, up front)."""
    return tuple(normal_scaled((steps, batch, H, d), d, dtype, seed * 1000 + 10 + i, device)
                 for i in range(3))


def state_init(nseq: int, H: int, d: int, seed: int, device="cpu", scale: float = 1.0):
    """A random fp32 carried-in state [nseq, H, d, d] (iid N(0,1) * scale / d)."""
    g = _generator(torch.device(device), seed)
    s = torch.randn((nseq, H, d, d), generator=g, dtype=torch.float32, device=device)
    return s.mul_(scale / d)


def decay_rates(H: int, device="cpu") -> torch.Tensor:
    """Per-head decay rates for the decay variant (fp32 [H], deterministic):
    lambda_h = exp(-2^(-8 (h + 1) / H)), the geometric slopes ALiBi gives its heads,
    turned into rates in (0, 1): from about 0.40 (h = 0 at H = 64) to 0.996."""
    h = torch.arange(H, dtype=torch.float64)
    lam = torch.exp(-torch.pow(2.0, -8.0 * (h + 1) / H))
    return lam.to(torch.float32).to(device)
