"""Sequence parallelism for the prefill (LASP+), one process per GPU.

Each rank holds a contiguous segment of the same sequences (rank r holds the
r-th segment of every sequence, ranks in sequence order). The prefill of a
segment needs only the state of everything before it, so the ranks

  1. compute their segments' states from a zero state (la_state_from_prefill),
  2. exchange them with one all-gather (torch.distributed; NCCL on GPUs),
  3. take a local exclusive prefix sum (la_state_exclusive_prefix), and
  4. run their own prefill from that state (la_prefill with init_state).

This is the all-gather + local prefix sum that replaces the serial
send/receive chain of linear-attention sequence parallelism (page "MiniMax-01
Lightning Attention", section "计算优化", item 3; page "首个线性注意力架构的大
模型来了…", section "4.2 计算优化"). Steps 1, 3 and 4 run in the library's
kernels; this module only moves tensors between them and the collective.

With a decay rate per head on the state (`decay=`, S_t = lambda S_{t-1} +
k_t^T v_t; not on the pages) the segment states are decayed to their segment's
end (la_state_decay), the ranks also all-gather their segment lengths, the
prefix discounts each earlier segment by lambda to the number of tokens after
it (la_state_exclusive_prefix_decay), and the prefill is la_prefill_decay.
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

from . import (prefill, prefill_decay, state_decay, state_exclusive_prefix, state_exclusive_prefix_decay,
               state_from_prefill)

__all__ = ["LibraryOps", "lasp_prefill"]


def _all_gather(out: torch.Tensor, x: torch.Tensor, group) -> None:
    """out[r] = rank r's x. NCCL (and any backend on host tensors) gathers in place;
    a gloo group with device tensors gathers host copies (gloo moves host memory only),
    which is how ranks that share one GPU, or a CPU-only cluster, run this driver."""
    if x.is_cuda and dist.get_backend(group) == "gloo":
        host = torch.empty(out.shape, dtype=out.dtype)
        dist.all_gather(list(host.unbind(0)), x.cpu(), group=group)
        out.copy_(host)
    else:
        dist.all_gather(list(out.unbind(0)), x, group=group)


class LibraryOps:
    """The three compute steps, on the library's CUDA kernels (decay: the rates, or None)."""

    @staticmethod
    def segment_state(k, v, cu_seqlens, decay=None):
        if decay is not None:
            return state_decay(k, v, decay, cu_seqlens)
        return state_from_prefill(k, v, cu_seqlens)

    @staticmethod
    def exclusive_prefix(gathered, rank, init_state, seg_lens=None, decay=None):
        if decay is not None:
            return state_exclusive_prefix_decay(gathered, seg_lens, rank, decay, init_state)
        return state_exclusive_prefix(gathered, rank, init_state)

    @staticmethod
    def prefill(q, k, v, cu_seqlens, B, init_state, out, decay=None):
        if decay is not None:
            return prefill_decay(q, k, v, decay, cu_seqlens, B=B, init_state=init_state, out=out)
        return prefill(q, k, v, cu_seqlens, B=B, init_state=init_state, out=out)


def lasp_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: Optional[torch.Tensor] = None, *,
                 B: int = 256, init_state: Optional[torch.Tensor] = None, group=None, out=None,
                 return_state: bool = False, decay: Optional[torch.Tensor] = None, ops=LibraryOps):
    """O of this rank's segment [T_r, H, d] of the sequences (see the module docstring).

    cu_seqlens (int32, [num_seqs + 1]) delimits this rank's segments of the
    num_seqs sequences, in sequence order; None means one sequence. init_state
    (fp32 [num_seqs, H, d, d]) is the state before the first segment, the same
    tensor on every rank. Every rank of `group` must call this with the same
    num_seqs, H and d. With return_state, also returns the state after the last
    segment (the state a decode continues from), identical on every rank.
    decay (fp32 [H], the same on every rank) selects the variant with a decay
    rate per head on the state.
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if decay is None:
        local = ops.segment_state(k, v, cu_seqlens)                    # [num_seqs, H, d, d], zero start
    else:
        local = ops.segment_state(k, v, cu_seqlens, decay)
    gathered = torch.empty((world,) + tuple(local.shape), dtype=local.dtype, device=local.device)
    _all_gather(gathered, local.contiguous(), group)
    if decay is None:
        start = ops.exclusive_prefix(gathered, rank, init_state)
        o = ops.prefill(q, k, v, cu_seqlens, B, start, out)
        return (o, ops.exclusive_prefix(gathered, world, init_state)) if return_state else o
    # decay: every rank's segment lengths too, [world, num_seqs] int32
    if cu_seqlens is None:
        lens = torch.tensor([q.shape[0]], dtype=torch.int32, device=q.device)
    else:
        lens = (cu_seqlens[1:] - cu_seqlens[:-1]).to(torch.int32).contiguous()
    seg_lens = torch.empty((world, lens.numel()), dtype=torch.int32, device=lens.device)
    _all_gather(seg_lens, lens, group)
    start = ops.exclusive_prefix(gathered, rank, init_state, seg_lens, decay)
    o = ops.prefill(q, k, v, cu_seqlens, B, start, out, decay)
    return (o, ops.exclusive_prefix(gathered, world, init_state, seg_lens, decay)) if return_state else o
