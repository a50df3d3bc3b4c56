"""torch.autograd glue for the prefill: forward with ``prefill``, backward with
``prefill_backward`` (both run in the library's kernels; this module only
connects them to autograd)."""
from __future__ import annotations

from typing import Optional

import torch

from . import prefill, prefill_backward

__all__ = ["LightningAttention", "lightning_attention"]


class LightningAttention(torch.autograd.Function):
    """O = causal linear attention of packed [T, H, d] q, k, v (optional fp32 S0)."""

    @staticmethod
    def forward(ctx, q, k, v, cu_seqlens, B, init_state):
        o = prefill(q, k, v, cu_seqlens, B=B, init_state=init_state)
        ctx.save_for_backward(q, k, v, cu_seqlens, init_state)
        ctx.B = B
        return o

    @staticmethod
    def backward(ctx, dout):
        q, k, v, cu_seqlens, init_state = ctx.saved_tensors
        need_init = init_state is not None and ctx.needs_input_grad[5]
        dq, dk, dv, dinit = prefill_backward(q, k, v, dout.contiguous(), cu_seqlens, B=ctx.B, init_state=init_state,
                                             need_init_grad=need_init)
        return dq, dk, dv, None, None, dinit


def lightning_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: Optional[torch.Tensor] = None,
                        B: int = 256, init_state: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Differentiable prefill: gradients flow to q, k, v and init_state."""
    return LightningAttention.apply(q, k, v, cu_seqlens, B, init_state)
