"""B200 (sm_100a) Lightning Attention: block-tiled causal linear attention.

Thin Python binding over the C ABI of ``liblightning_attention.so`` (declared
in ``include/lightning_attention.h``). Every step of the computation runs in
the library's CUDA kernels; this module only marshals torch tensors into
pointers and sizes. There is no fallback: if the library has not been built
(``python -m causal_linear_attention_02_b200.build``), every call raises.

The ``la_*`` functions mirror the C entry points one to one and return the
integer status. ``prefill``, ``state_from_prefill`` and ``decode_step`` are
conveniences that size and allocate outputs/workspace with torch, call the
``la_*`` function and raise ``LightningError`` on a non-zero status.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

__all__ = [
    "LightningError", "LA_BF16", "LA_FP32", "STATUS", "library_path", "load_library",
    "la_prefill_workspace_size", "la_prefill", "la_prefill_noalloc", "LA_NOALLOC_SCRATCH_BYTES",
    "la_state_workspace_size", "la_state_from_prefill", "la_state_exclusive_prefix",
    "la_prefill_backward_workspace_size", "la_prefill_backward",
    "la_prefill_with_state_workspace_size", "la_prefill_with_state",
    "la_decode_step", "la_prefill_decay_workspace_size", "la_prefill_decay", "la_state_decay_workspace_size",
    "la_state_decay", "la_decode_step_decay", "la_feature_map", "la_state_exclusive_prefix_decay",
    "la_prefill_backward_decay_workspace_size", "la_prefill_backward_decay",
    "la_get_device_status", "la_set_kernel_timer", "la_debug_set_fault", "la_debug_set_trace", "la_debug_set_path", "la_status_string", "la_version",
    "la_launch_count",
    "prefill", "prefill_with_state", "prefill_backward", "state_from_prefill", "state_exclusive_prefix", "decode_step", "device_status",
    "prefill_decay", "state_decay", "decode_step_decay", "feature_map", "state_exclusive_prefix_decay",
    "prefill_backward_decay",
    "uses_tensor_cores",
]

LA_BF16 = 0
LA_FP32 = 1
STATUS = {
    0: "LA_OK", 1: "LA_ERR_INVALID_ARGUMENT", 2: "LA_ERR_UNSUPPORTED", 3: "LA_ERR_MISALIGNED",
    4: "LA_ERR_WORKSPACE_TOO_SMALL", 5: "LA_ERR_CUDA", 6: "LA_ERR_TIMEOUT", 7: "LA_ERR_BAD_SEQLENS",
    8: "LA_ERR_BAD_DECAY",
}

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liblightning_attention.so")
_lock = threading.Lock()
_lib = None


class LightningError(RuntimeError):
    """A library call returned a non-zero status, or the library is missing."""

    def __init__(self, msg, status=None):
        super().__init__(msg)
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load the CUDA library (raises LightningError if it was never built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise LightningError(
                f"{_LIB_PATH} is missing: build it with `python -m causal_linear_attention_02_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        vp, sz, i32, i64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_int64
        lib.la_prefill_workspace_size.argtypes = [i64, i32, i32, i32, i32, i32]
        lib.la_prefill_workspace_size.restype = sz
        lib.la_prefill.argtypes = [vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, vp, vp, sz, vp]
        lib.la_prefill.restype = i32
        lib.la_prefill_noalloc.argtypes = [vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, vp, vp]
        lib.la_prefill_noalloc.restype = i32
        lib.la_state_workspace_size.argtypes = [i64, i32, i32, i32, i32]
        lib.la_state_workspace_size.restype = sz
        lib.la_state_from_prefill.argtypes = [vp, vp, vp, i32, i64, i32, i32, i32, vp, vp, vp, sz, vp]
        lib.la_state_from_prefill.restype = i32
        lib.la_prefill_with_state_workspace_size.argtypes = [i64, i32, i32, i32, i32, i32]
        lib.la_prefill_with_state_workspace_size.restype = sz
        lib.la_prefill_with_state.argtypes = [vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, vp, vp, vp, sz, vp]
        lib.la_prefill_with_state.restype = i32
        lib.la_prefill_backward_workspace_size.argtypes = [i64, i32, i32, i32, i32, i32]
        lib.la_prefill_backward_workspace_size.restype = sz
        lib.la_prefill_backward.argtypes = [vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp,
                                            sz, vp]
        lib.la_prefill_backward.restype = i32
        lib.la_state_exclusive_prefix.argtypes = [vp, i32, i32, i64, i32, vp, vp, vp]
        lib.la_state_exclusive_prefix.restype = i32
        lib.la_decode_step.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp]
        lib.la_decode_step.restype = i32
        lib.la_prefill_decay_workspace_size.argtypes = [i64, i32, i32, i32, i32, i32]
        lib.la_prefill_decay_workspace_size.restype = sz
        lib.la_prefill_decay.argtypes = [vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, vp, vp, vp, vp, sz, vp]
        lib.la_prefill_decay.restype = i32
        lib.la_state_decay_workspace_size.argtypes = [i64, i32, i32, i32, i32]
        lib.la_state_decay_workspace_size.restype = sz
        lib.la_state_decay.argtypes = [vp, vp, vp, i32, i64, i32, i32, i32, vp, vp, vp, vp, sz, vp]
        lib.la_state_decay.restype = i32
        lib.la_decode_step_decay.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, vp]
        lib.la_decode_step_decay.restype = i32
        lib.la_state_exclusive_prefix_decay.argtypes = [vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp]
        lib.la_state_exclusive_prefix_decay.restype = i32
        lib.la_prefill_backward_decay_workspace_size.argtypes = [i64, i32, i32, i32, i32, i32]
        lib.la_prefill_backward_decay_workspace_size.restype = sz
        lib.la_prefill_backward_decay.argtypes = [vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, vp, vp, vp, vp,
                                                  vp, vp, vp, sz, vp]
        lib.la_prefill_backward_decay.restype = i32
        lib.la_feature_map.argtypes = [vp, vp, i64, i32, ctypes.c_float, vp]
        lib.la_feature_map.restype = i32
        lib.la_get_device_status.argtypes = [vp]
        lib.la_get_device_status.restype = i32
        lib.la_status_string.argtypes = [i32]
        lib.la_status_string.restype = ctypes.c_char_p
        lib.la_debug_set_trace.argtypes = [vp, sz]
        lib.la_debug_set_trace.restype = i32
        lib.la_debug_set_fault.argtypes = [ctypes.c_longlong, ctypes.c_uint64]
        lib.la_debug_set_fault.restype = i32
        lib.la_set_kernel_timer.argtypes = [vp, vp]
        lib.la_set_kernel_timer.restype = i32
        lib.la_version.argtypes = []
        lib.la_version.restype = i32
        lib.la_debug_set_path.argtypes = [i32]
        lib.la_debug_set_path.restype = i32
        lib.la_launch_count.argtypes = []
        lib.la_launch_count.restype = ctypes.c_uint64
        _lib = lib
        return lib


# ---------------------------------------------------------------- C ABI mirrors
def la_prefill_workspace_size(total_tokens, num_seqs, heads, d, B, dtype) -> int:
    return int(load_library().la_prefill_workspace_size(total_tokens, num_seqs, heads, d, B, dtype))


def la_prefill(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype, init_state,
               workspace, workspace_bytes, stream) -> int:
    return int(load_library().la_prefill(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype,
                                         init_state, workspace, workspace_bytes, stream))


# Size of the static scratch of la_prefill_noalloc (LA_NOALLOC_SCRATCH_BYTES).
LA_NOALLOC_SCRATCH_BYTES = 64 << 20


def la_prefill_noalloc(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype, init_state,
                       stream) -> int:
    return int(load_library().la_prefill_noalloc(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B,
                                                 dtype, init_state, stream))


def la_state_workspace_size(total_tokens, num_seqs, heads, d, dtype) -> int:
    return int(load_library().la_state_workspace_size(total_tokens, num_seqs, heads, d, dtype))


def la_state_from_prefill(k, v, cu_seqlens, num_seqs, total_tokens, heads, d, dtype, init_state, state_out,
                          workspace, workspace_bytes, stream) -> int:
    return int(load_library().la_state_from_prefill(k, v, cu_seqlens, num_seqs, total_tokens, heads, d, dtype,
                                                    init_state, state_out, workspace, workspace_bytes, stream))


def la_prefill_with_state_workspace_size(total_tokens, num_seqs, heads, d, B, dtype) -> int:
    return int(load_library().la_prefill_with_state_workspace_size(total_tokens, num_seqs, heads, d, B, dtype))


def la_prefill_with_state(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype, init_state, state_out,
                          workspace, workspace_bytes, stream) -> int:
    return int(load_library().la_prefill_with_state(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B,
                                                    dtype, init_state, state_out, workspace, workspace_bytes, stream))


def la_prefill_backward_workspace_size(total_tokens, num_seqs, heads, d, B, dtype) -> int:
    return int(load_library().la_prefill_backward_workspace_size(total_tokens, num_seqs, heads, d, B, dtype))


def la_prefill_backward(q, k, v, dout, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype, init_state, dq, dk,
                        dv, dinit_state, workspace, workspace_bytes, stream) -> int:
    return int(load_library().la_prefill_backward(q, k, v, dout, cu_seqlens, num_seqs, total_tokens, heads, d, B,
                                                  dtype, init_state, dq, dk, dv, dinit_state, workspace,
                                                  workspace_bytes, stream))


def la_state_exclusive_prefix(gathered, world, rank, n, d, init, out, stream) -> int:
    return int(load_library().la_state_exclusive_prefix(gathered, world, rank, n, d, init, out, stream))


def la_decode_step(q, k, v, state, o, batch, heads, d, dtype, stream) -> int:
    return int(load_library().la_decode_step(q, k, v, state, o, batch, heads, d, dtype, stream))


def la_prefill_decay_workspace_size(total_tokens, num_seqs, heads, d, B, dtype) -> int:
    return int(load_library().la_prefill_decay_workspace_size(total_tokens, num_seqs, heads, d, B, dtype))


def la_prefill_decay(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype, init_state, decay,
                     state_out, workspace, workspace_bytes, stream) -> int:
    return int(load_library().la_prefill_decay(q, k, v, o, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype,
                                               init_state, decay, state_out, workspace, workspace_bytes, stream))


def la_state_decay_workspace_size(total_tokens, num_seqs, heads, d, dtype) -> int:
    return int(load_library().la_state_decay_workspace_size(total_tokens, num_seqs, heads, d, dtype))


def la_state_decay(k, v, cu_seqlens, num_seqs, total_tokens, heads, d, dtype, init_state, decay, state_out,
                   workspace, workspace_bytes, stream) -> int:
    return int(load_library().la_state_decay(k, v, cu_seqlens, num_seqs, total_tokens, heads, d, dtype, init_state,
                                             decay, state_out, workspace, workspace_bytes, stream))


def la_decode_step_decay(q, k, v, state, o, batch, heads, d, dtype, decay, stream) -> int:
    return int(load_library().la_decode_step_decay(q, k, v, state, o, batch, heads, d, dtype, decay, stream))


def la_state_exclusive_prefix_decay(gathered, seg_lens, world, rank, num_seqs, heads, d, decay, init, out,
                                    stream) -> int:
    return int(load_library().la_state_exclusive_prefix_decay(gathered, seg_lens, world, rank, num_seqs, heads, d,
                                                               decay, init, out, stream))


def la_prefill_backward_decay_workspace_size(total_tokens, num_seqs, heads, d, B, dtype) -> int:
    return int(load_library().la_prefill_backward_decay_workspace_size(total_tokens, num_seqs, heads, d, B, dtype))


def la_prefill_backward_decay(q, k, v, dout, cu_seqlens, num_seqs, total_tokens, heads, d, B, dtype, init_state,
                              decay, dq, dk, dv, dinit_state, workspace, workspace_bytes, stream) -> int:
    return int(load_library().la_prefill_backward_decay(q, k, v, dout, cu_seqlens, num_seqs, total_tokens, heads, d,
                                                        B, dtype, init_state, decay, dq, dk, dv, dinit_state,
                                                        workspace, workspace_bytes, stream))


def la_feature_map(x, y, n, dtype, alpha, stream) -> int:
    return int(load_library().la_feature_map(x, y, n, dtype, alpha, stream))


def la_get_device_status(stream) -> int:
    return int(load_library().la_get_device_status(stream))


def la_status_string(status: int) -> str:
    return load_library().la_status_string(int(status)).decode()


def la_debug_set_fault(suppress_tile: int, wait_ns: int) -> int:
    return int(load_library().la_debug_set_fault(suppress_tile, wait_ns))


def la_debug_set_path(path: int) -> int:
    return int(load_library().la_debug_set_path(path))


def la_debug_set_trace(device_buffer, nbytes: int) -> int:
    return int(load_library().la_debug_set_trace(device_buffer, nbytes))


def la_set_kernel_timer(start_event, stop_event) -> int:
    return int(load_library().la_set_kernel_timer(start_event, stop_event))


def la_version() -> int:
    return int(load_library().la_version())


def la_launch_count() -> int:
    return int(load_library().la_launch_count())


# ---------------------------------------------------------------- marshalling helpers
def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return LA_BF16
    if t == torch.float32:
        return LA_FP32
    raise LightningError(f"unsupported dtype {t} (bf16 or fp32)", 2)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream, device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, device=None):
    if not t.is_cuda:
        raise LightningError(f"{name} must be a CUDA tensor", 1)
    if not t.is_contiguous():
        raise LightningError(f"{name} must be contiguous", 1)
    if device is not None and t.device != device:
        raise LightningError(f"{name} is on {t.device}, expected {device}", 1)


def _raise(status: int, what: str):
    if status != 0:
        raise LightningError(f"{what}: {STATUS.get(status, status)} ({la_status_string(status)})", status)


def uses_tensor_cores(dtype: torch.dtype, d: int, B: int) -> bool:
    """True when la_prefill runs this shape on the tcgen05 path (bf16, d=128, B in {128, 256})."""
    return dtype == torch.bfloat16 and d == 128 and B in (128, 256)


# ---------------------------------------------------------------- conveniences
def prefill(q, k, v, cu_seqlens=None, B: int = 256, init_state=None, out=None, workspace=None, stream=None):
    """O = causal linear attention of packed [T, H, d] q, k, v (see la_prefill)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, q.device)
    if q.dim() != 3 or k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise LightningError("q, k, v must share one [T, H, d] shape and dtype", 1)
    T, H, d = q.shape
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", q.device)
        if cu_seqlens.dtype != torch.int32:
            raise LightningError("cu_seqlens must be int32", 1)
        nseq = cu_seqlens.numel() - 1
    else:
        nseq = 1
    if init_state is not None:
        _need(init_state, "init_state", q.device)
        if init_state.dtype != torch.float32 or tuple(init_state.shape) != (nseq, H, d, d):
            raise LightningError("init_state must be fp32 [num_seqs, H, d, d]", 1)
    code = _dtype_code(q.dtype)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", q.device)
    ws_bytes = la_prefill_workspace_size(T, nseq, H, d, B, code)
    if ws_bytes == 0:
        raise LightningError(f"unsupported prefill shape T={T} H={H} d={d} B={B}", 2)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    status = la_prefill(_p(q), _p(k), _p(v), _p(out), _p(cu_seqlens), nseq, T, H, d, B, code, _p(init_state),
                        _p(workspace), workspace.numel() * workspace.element_size(),
                        _stream_handle(stream, q.device))
    _raise(status, "la_prefill")
    return out


def prefill_with_state(q, k, v, cu_seqlens=None, B: int = 256, init_state=None, out=None, state_out=None,
                       workspace=None, stream=None):
    """(O, final state) of packed [T, H, d] q, k, v (see la_prefill_with_state); state_out may be
    init_state itself to update it in place."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, q.device)
    if q.dim() != 3 or k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise LightningError("q, k, v must share one [T, H, d] shape and dtype", 1)
    T, H, d = q.shape
    nseq = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", q.device)
    if init_state is not None:
        _need(init_state, "init_state", q.device)
    code = _dtype_code(q.dtype)
    if out is None:
        out = torch.empty_like(q)
    if state_out is None:
        state_out = torch.empty((nseq, H, d, d), dtype=torch.float32, device=q.device)
    _need(state_out, "state_out", q.device)
    ws_bytes = la_prefill_with_state_workspace_size(T, nseq, H, d, B, code)
    if ws_bytes == 0:
        raise LightningError(f"unsupported prefill shape T={T} H={H} d={d} B={B}", 2)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    status = la_prefill_with_state(_p(q), _p(k), _p(v), _p(out), _p(cu_seqlens), nseq, T, H, d, B, code,
                                   _p(init_state), _p(state_out), _p(workspace),
                                   workspace.numel() * workspace.element_size(), _stream_handle(stream, q.device))
    _raise(status, "la_prefill_with_state")
    return out, state_out


def prefill_backward(q, k, v, dout, cu_seqlens=None, B: int = 256, init_state=None, need_init_grad=False,
                     workspace=None, stream=None):
    """(dq, dk, dv, dinit) of L = sum_t dout_t . O_t for O = prefill(q, k, v, ...) (see
    la_prefill_backward); dinit is None unless need_init_grad."""
    for n, t in (("q", q), ("k", k), ("v", v), ("dout", dout)):
        _need(t, n, q.device)
    if q.dim() != 3 or any(t.shape != q.shape or t.dtype != q.dtype for t in (k, v, dout)):
        raise LightningError("q, k, v, dout must share one [T, H, d] shape and dtype", 1)
    T, H, d = q.shape
    nseq = 1
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", q.device)
        if cu_seqlens.dtype != torch.int32:
            raise LightningError("cu_seqlens must be int32", 1)
        nseq = cu_seqlens.numel() - 1
    if init_state is not None:
        _need(init_state, "init_state", q.device)
        if init_state.dtype != torch.float32 or tuple(init_state.shape) != (nseq, H, d, d):
            raise LightningError("init_state must be fp32 [num_seqs, H, d, d]", 1)
    code = _dtype_code(q.dtype)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    dinit = torch.empty((nseq, H, d, d), dtype=torch.float32, device=q.device) if need_init_grad else None
    ws_bytes = la_prefill_backward_workspace_size(T, nseq, H, d, B, code)
    if ws_bytes == 0:
        raise LightningError(f"unsupported prefill shape T={T} H={H} d={d} B={B}", 2)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    status = la_prefill_backward(_p(q), _p(k), _p(v), _p(dout), _p(cu_seqlens), nseq, T, H, d, B, code,
                                 _p(init_state), _p(dq), _p(dk), _p(dv), _p(dinit), _p(workspace),
                                 workspace.numel() * workspace.element_size(), _stream_handle(stream, q.device))
    _raise(status, "la_prefill_backward")
    return dq, dk, dv, dinit


def state_from_prefill(k, v, cu_seqlens=None, init_state=None, out=None, workspace=None, stream=None):
    """fp32 [num_seqs, H, d, d] state S0 + sum_t k_t^T v_t per sequence (see la_state_from_prefill)."""
    _need(k, "k"); _need(v, "v", k.device)
    if k.dim() != 3 or v.shape != k.shape or v.dtype != k.dtype:
        raise LightningError("k, v must share one [T, H, d] shape and dtype", 1)
    T, H, d = k.shape
    nseq = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", k.device)
    if out is None:
        out = torch.empty((nseq, H, d, d), dtype=torch.float32, device=k.device)
    _need(out, "out", k.device)
    if init_state is not None:
        _need(init_state, "init_state", k.device)
    code = _dtype_code(k.dtype)
    ws_bytes = la_state_workspace_size(T, nseq, H, d, code)
    if ws_bytes == 0:
        raise LightningError(f"unsupported state shape T={T} H={H} d={d}", 2)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=k.device)
    status = la_state_from_prefill(_p(k), _p(v), _p(cu_seqlens), nseq, T, H, d, code, _p(init_state), _p(out),
                                   _p(workspace), workspace.numel() * workspace.element_size(),
                                   _stream_handle(stream, k.device))
    _raise(status, "la_state_from_prefill")
    return out


def state_exclusive_prefix(gathered, rank, init=None, out=None, stream=None):
    """init + sum of gathered[:rank] for fp32 gathered [world, *S], S = [num_seqs, H, d, d]
    (see la_state_exclusive_prefix; rank = world gives the state after the last segment)."""
    _need(gathered, "gathered")
    if gathered.dtype != torch.float32 or gathered.dim() != 5 or gathered.shape[-1] != gathered.shape[-2]:
        raise LightningError("gathered must be fp32 [world, num_seqs, H, d, d]", 1)
    world, nseq, H, d = gathered.shape[0], gathered.shape[1], gathered.shape[2], gathered.shape[3]
    if out is None:
        out = torch.empty(gathered.shape[1:], dtype=torch.float32, device=gathered.device)
    _need(out, "out", gathered.device)
    if init is not None:
        _need(init, "init", gathered.device)
        if init.dtype != torch.float32 or init.shape != out.shape:
            raise LightningError("init must be fp32 [num_seqs, H, d, d]", 1)
    status = la_state_exclusive_prefix(_p(gathered), world, rank, nseq * H, d, _p(init), _p(out),
                                       _stream_handle(stream, gathered.device))
    _raise(status, "la_state_exclusive_prefix")
    return out


def decode_step(q, k, v, state, out=None, stream=None):
    """One step S <- S + k^T v, o = q S on [batch, H, d] inputs; state updated in place."""
    for n, t in (("q", q), ("k", k), ("v", v), ("state", state)):
        _need(t, n, q.device)
    if q.dim() != 3 or k.shape != q.shape or v.shape != q.shape:
        raise LightningError("q, k, v must share one [batch, H, d] shape", 1)
    batch, H, d = q.shape
    if state.dtype != torch.float32 or tuple(state.shape) != (batch, H, d, d):
        raise LightningError("state must be fp32 [batch, H, d, d]", 1)
    code = _dtype_code(q.dtype)
    if out is None:
        out = torch.empty_like(q)
    status = la_decode_step(_p(q), _p(k), _p(v), _p(state), _p(out), batch, H, d, code,
                            _stream_handle(stream, q.device))
    _raise(status, "la_decode_step")
    return out


def _decay_rates(decay, H, device):
    _need(decay, "decay", device)
    if decay.dtype != torch.float32 or tuple(decay.shape) != (H,):
        raise LightningError("decay must be fp32 [H]", 1)


def prefill_decay(q, k, v, decay, cu_seqlens=None, B: int = 256, init_state=None, return_state=False, out=None,
                  state_out=None, workspace=None, stream=None):
    """O (and optionally the final states) of causal linear attention with a per-head decay rate on the state,
    S_t = decay[h] S_{t-1} + k_t^T v_t, o_t = q_t S_t (see la_prefill_decay)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, q.device)
    if q.dim() != 3 or k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise LightningError("q, k, v must share one [T, H, d] shape and dtype", 1)
    T, H, d = q.shape
    _decay_rates(decay, H, q.device)
    nseq = 1
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", q.device)
        if cu_seqlens.dtype != torch.int32:
            raise LightningError("cu_seqlens must be int32", 1)
        nseq = cu_seqlens.numel() - 1
    if init_state is not None:
        _need(init_state, "init_state", q.device)
        if init_state.dtype != torch.float32 or tuple(init_state.shape) != (nseq, H, d, d):
            raise LightningError("init_state must be fp32 [num_seqs, H, d, d]", 1)
    code = _dtype_code(q.dtype)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", q.device)
    if return_state and state_out is None:
        state_out = torch.empty((nseq, H, d, d), dtype=torch.float32, device=q.device)
    if state_out is not None:
        _need(state_out, "state_out", q.device)
    ws_bytes = la_prefill_decay_workspace_size(T, nseq, H, d, B, code)
    if ws_bytes == 0:
        raise LightningError(f"unsupported prefill shape T={T} H={H} d={d} B={B}", 2)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    status = la_prefill_decay(_p(q), _p(k), _p(v), _p(out), _p(cu_seqlens), nseq, T, H, d, B, code, _p(init_state),
                              _p(decay), _p(state_out), _p(workspace), workspace.numel() * workspace.element_size(),
                              _stream_handle(stream, q.device))
    _raise(status, "la_prefill_decay")
    return (out, state_out) if (return_state or state_out is not None) else out


def state_decay(k, v, decay, cu_seqlens=None, init_state=None, out=None, workspace=None, stream=None):
    """fp32 [num_seqs, H, d, d] final states with decay (see la_state_decay)."""
    _need(k, "k"); _need(v, "v", k.device)
    if k.dim() != 3 or v.shape != k.shape or v.dtype != k.dtype:
        raise LightningError("k, v must share one [T, H, d] shape and dtype", 1)
    T, H, d = k.shape
    _decay_rates(decay, H, k.device)
    nseq = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", k.device)
    if out is None:
        out = torch.empty((nseq, H, d, d), dtype=torch.float32, device=k.device)
    _need(out, "out", k.device)
    if init_state is not None:
        _need(init_state, "init_state", k.device)
    code = _dtype_code(k.dtype)
    ws_bytes = la_state_decay_workspace_size(T, nseq, H, d, code)
    if ws_bytes == 0:
        raise LightningError(f"unsupported state shape T={T} H={H} d={d}", 2)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=k.device)
    status = la_state_decay(_p(k), _p(v), _p(cu_seqlens), nseq, T, H, d, code, _p(init_state), _p(decay), _p(out),
                            _p(workspace), workspace.numel() * workspace.element_size(),
                            _stream_handle(stream, k.device))
    _raise(status, "la_state_decay")
    return out


def decode_step_decay(q, k, v, state, decay, out=None, stream=None):
    """One step S <- decay[h] S + k^T v, o = q S on [batch, H, d] inputs; state updated in place."""
    for n, t in (("q", q), ("k", k), ("v", v), ("state", state)):
        _need(t, n, q.device)
    if q.dim() != 3 or k.shape != q.shape or v.shape != q.shape:
        raise LightningError("q, k, v must share one [batch, H, d] shape", 1)
    batch, H, d = q.shape
    _decay_rates(decay, H, q.device)
    if state.dtype != torch.float32 or tuple(state.shape) != (batch, H, d, d):
        raise LightningError("state must be fp32 [batch, H, d, d]", 1)
    code = _dtype_code(q.dtype)
    if out is None:
        out = torch.empty_like(q)
    status = la_decode_step_decay(_p(q), _p(k), _p(v), _p(state), _p(out), batch, H, d, code, _p(decay),
                                  _stream_handle(stream, q.device))
    _raise(status, "la_decode_step_decay")
    return out


def state_exclusive_prefix_decay(gathered, seg_lens, rank, decay, init=None, out=None, stream=None):
    """Rank `rank`'s starting state with per-head decay for fp32 gathered [world, num_seqs, H, d, d] segment
    states and int32 seg_lens [world, num_seqs] (see la_state_exclusive_prefix_decay)."""
    _need(gathered, "gathered")
    if gathered.dtype != torch.float32 or gathered.dim() != 5 or gathered.shape[-1] != gathered.shape[-2]:
        raise LightningError("gathered must be fp32 [world, num_seqs, H, d, d]", 1)
    world, nseq, H, d = gathered.shape[0], gathered.shape[1], gathered.shape[2], gathered.shape[3]
    _need(seg_lens, "seg_lens", gathered.device)
    if seg_lens.dtype != torch.int32 or tuple(seg_lens.shape) != (world, nseq):
        raise LightningError("seg_lens must be int32 [world, num_seqs]", 1)
    _decay_rates(decay, H, gathered.device)
    if out is None:
        out = torch.empty(gathered.shape[1:], dtype=torch.float32, device=gathered.device)
    _need(out, "out", gathered.device)
    if init is not None:
        _need(init, "init", gathered.device)
        if init.dtype != torch.float32 or init.shape != out.shape:
            raise LightningError("init must be fp32 [num_seqs, H, d, d]", 1)
    status = la_state_exclusive_prefix_decay(_p(gathered), _p(seg_lens), world, rank, nseq, H, d, _p(decay), _p(init),
                                             _p(out), _stream_handle(stream, gathered.device))
    _raise(status, "la_state_exclusive_prefix_decay")
    return out


def prefill_backward_decay(q, k, v, dout, decay, cu_seqlens=None, B: int = 256, init_state=None,
                           need_init_grad=False, workspace=None, stream=None):
    """(dq, dk, dv, dinit) of L = sum_t dout_t . O_t for O = prefill_decay(q, k, v, decay, ...) (see
    la_prefill_backward_decay); dinit is None unless need_init_grad."""
    for n, t in (("q", q), ("k", k), ("v", v), ("dout", dout)):
        _need(t, n, q.device)
    if q.dim() != 3 or any(t.shape != q.shape or t.dtype != q.dtype for t in (k, v, dout)):
        raise LightningError("q, k, v, dout must share one [T, H, d] shape and dtype", 1)
    T, H, d = q.shape
    _decay_rates(decay, H, q.device)
    nseq = 1
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", q.device)
        nseq = cu_seqlens.numel() - 1
    if init_state is not None:
        _need(init_state, "init_state", q.device)
    code = _dtype_code(q.dtype)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    dinit = torch.empty((nseq, H, d, d), dtype=torch.float32, device=q.device) if need_init_grad else None
    ws_bytes = la_prefill_backward_decay_workspace_size(T, nseq, H, d, B, code)
    if ws_bytes == 0:
        raise LightningError(f"unsupported prefill shape T={T} H={H} d={d} B={B}", 2)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    status = la_prefill_backward_decay(_p(q), _p(k), _p(v), _p(dout), _p(cu_seqlens), nseq, T, H, d, B, code,
                                       _p(init_state), _p(decay), _p(dq), _p(dk), _p(dv), _p(dinit), _p(workspace),
                                       workspace.numel() * workspace.element_size(), _stream_handle(stream, q.device))
    _raise(status, "la_prefill_backward_decay")
    return dq, dk, dv, dinit


def feature_map(x, alpha: float = 0.3, out=None, stream=None):
    """phi(x) = ELU(x) + alpha x elementwise (see la_feature_map); out may be x for in place."""
    _need(x, "x")
    code = _dtype_code(x.dtype)
    if out is None:
        out = torch.empty_like(x)
    _need(out, "out", x.device)
    if out.dtype != x.dtype or out.numel() != x.numel():
        raise LightningError("out must match x in dtype and size", 1)
    status = la_feature_map(_p(x), _p(out), x.numel(), code, float(alpha), _stream_handle(stream, x.device))
    _raise(status, "la_feature_map")
    return out


def device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    dev = torch.device("cuda", torch.cuda.current_device())
    return la_get_device_status(_stream_handle(stream, dev))
