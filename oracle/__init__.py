"""fp64 CPU oracle for causal linear attention (Lightning Attention).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference arm are the only callers. The product
library never imports this package, and this package never imports the
product library: the two share no code.

The arithmetic lives in ``lightning_oracle.c`` (plain loops, ``double``
throughout). This module compiles it with gcc on first use and exposes numpy
wrappers. Every wrapper takes float64 arrays in the layout

    q, k, v, o : [T, H, d]          (tokens of all sequences packed)
    cu_seqlens : int32 [nseq + 1]   (cu_seqlens[0] = 0, last = T)
    state      : [nseq, H, d, d]    (state[i, j] = sum_t k_t[i] * v_t[j])

and computes O_t = q_t . S0 + sum_{s <= t, same sequence} (q_t . k_s) v_s
(page "MiniMax-01 Lightning Attention", section "Lightning Attention 设计").

Parity status: every function here is pinned by the CPU tests in
``tests/test_oracle_pins.py`` (closed forms, exact rational brute force, a
hand-computed golden example, agreement of three independent associations,
linearity, causality and varlen invariants). ``backward`` (the gradients of
L = sum_t dO_t . O_t, the training pass; the pages give the forward only) is
pinned by central differences through the pinned forward, which are exact
because O is linear in each input taken alone, by a one-token closed form and
by the independence of packed sequences.

``decay_*`` (a per-head decay rate on the state, S_t = lambda S_{t-1} + k_t^T v_t;
not on the pages, the Lightning Attention-2 form taken in its plainest reading)
are pinned by reduction to the pinned no-decay functions through an exact
change of variables (q_t -> lambda^(t+1) q_t, k_s -> lambda^-(s+1) k_s), by
lambda = 1 and lambda = 0 closed forms, by a discounted cumulative sum computed
with scipy's IIR filter, and by the splitting of a sequence at any token.
``decay_backward`` (the gradients of the decay variant) is pinned by central
differences through the pinned ``decay_quadratic`` and by reduction to
``backward`` at lambda = 1.
``feature_map`` (phi(x) = ELU(x) + alpha x, page "MiniMax-M2.5语言模型：Linear
Attention架构解析与实践", section 2.2) is pinned by torch's ELU and by values
worked by hand.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lightning_oracle.c")
_LIB = os.path.join(_HERE, "liblightning_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (OpenMP, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int32)
            i = ctypes.c_int
            lib.oracle_quadratic.argtypes = [dp, dp, dp, dp, ip, i, i, i, dp]
            lib.oracle_recurrent.argtypes = [dp, dp, dp, dp, ip, i, i, i, dp, dp]
            lib.oracle_blocked.argtypes = [dp, dp, dp, dp, ip, i, i, i, i, dp, dp]
            lib.oracle_state.argtypes = [dp, dp, ip, i, i, i, dp, dp]
            lib.oracle_decode_step.argtypes = [dp, dp, dp, dp, dp, i, i, i]
            lib.oracle_backward.argtypes = [dp, dp, dp, dp, ip, i, i, i, dp, dp, dp, dp, dp]
            lib.oracle_decay_quadratic.argtypes = [dp, dp, dp, dp, ip, i, i, i, dp, dp]
            lib.oracle_decay_recurrent.argtypes = [dp, dp, dp, dp, ip, i, i, i, dp, dp, dp]
            lib.oracle_decay_blocked.argtypes = [dp, dp, dp, dp, ip, i, i, i, i, dp, dp, dp]
            lib.oracle_decay_state.argtypes = [dp, dp, ip, i, i, i, dp, dp, dp]
            lib.oracle_decay_decode_step.argtypes = [dp, dp, dp, dp, dp, i, i, i, dp]
            lib.oracle_decay_backward.argtypes = [dp, dp, dp, dp, ip, i, i, i, dp, dp, dp, dp, dp, dp]
            lib.oracle_feature_map.argtypes = [dp, dp, ctypes.c_int64, ctypes.c_double]
            lib.oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(a):
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    return a


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _cu(cu_seqlens, T):
    if cu_seqlens is None:
        cu_seqlens = [0, T]
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    if cu.ndim != 1 or cu.size < 1 or cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must start at 0, end at T and be non-decreasing")
    return cu, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def _check_qkv(q, k, v):
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim != 3 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one shape [T, H, d]")
    return q, k, v


def _init(init, nseq, H, d):
    if init is None:
        return None
    init = _f64(init)
    if init.shape != (nseq, H, d, d):
        raise ValueError("init state must be [nseq, H, d, d]")
    return init


def quadratic(q, k, v, cu_seqlens=None, init=None):
    """Masked left product over each whole sequence: O = tril(Q K^T) V + Q S0."""
    q, k, v = _check_qkv(q, k, v)
    T, H, d = q.shape
    cu, cup = _cu(cu_seqlens, T)
    init = _init(init, cu.size - 1, H, d)
    o = np.zeros_like(q)
    _load().oracle_quadratic(_ptr(q), _ptr(k), _ptr(v), _ptr(o), cup, cu.size - 1, H, d, _ptr(init))
    return o


def recurrent(q, k, v, cu_seqlens=None, init=None, return_state=False):
    """Token-by-token form: S += k^T v; o = q S. Optionally returns the final state."""
    q, k, v = _check_qkv(q, k, v)
    T, H, d = q.shape
    cu, cup = _cu(cu_seqlens, T)
    nseq = cu.size - 1
    init = _init(init, nseq, H, d)
    o = np.zeros_like(q)
    st = np.zeros((nseq, H, d, d)) if return_state else None
    _load().oracle_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(o), cup, nseq, H, d, _ptr(init), _ptr(st))
    return (o, st) if return_state else o


def blocked(q, k, v, B, cu_seqlens=None, init=None, return_state=False):
    """The pages' decomposition with block size B (intra left product, inter right product)."""
    q, k, v = _check_qkv(q, k, v)
    T, H, d = q.shape
    if int(B) < 1:
        raise ValueError("B must be >= 1")
    cu, cup = _cu(cu_seqlens, T)
    nseq = cu.size - 1
    init = _init(init, nseq, H, d)
    o = np.zeros_like(q)
    st = np.zeros((nseq, H, d, d)) if return_state else None
    _load().oracle_blocked(_ptr(q), _ptr(k), _ptr(v), _ptr(o), cup, nseq, H, d, int(B),
                           _ptr(init), _ptr(st))
    return (o, st) if return_state else o


def state(k, v, cu_seqlens=None, init=None):
    """Final state per (sequence, head): S0 + sum_t k_t^T v_t."""
    k, v = _f64(k), _f64(v)
    if k.ndim != 3 or k.shape != v.shape:
        raise ValueError("k, v must share one shape [T, H, d]")
    T, H, d = k.shape
    cu, cup = _cu(cu_seqlens, T)
    nseq = cu.size - 1
    init = _init(init, nseq, H, d)
    st = np.zeros((nseq, H, d, d))
    _load().oracle_state(_ptr(k), _ptr(v), cup, nseq, H, d, _ptr(init), _ptr(st))
    return st


def decode_step(q, k, v, state_in):
    """One recurrent step on [batch, H, d] inputs; returns (o, new_state); input untouched."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim != 3 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one shape [batch, H, d]")
    batch, H, d = q.shape
    st = np.array(state_in, dtype=np.float64, copy=True, order="C")
    if st.shape != (batch, H, d, d):
        raise ValueError("state must be [batch, H, d, d]")
    o = np.zeros_like(q)
    _load().oracle_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(st), _ptr(o), batch, H, d)
    return o, st


def backward(q, k, v, dout, cu_seqlens=None, init=None):
    """Gradients (dq, dk, dv, dinit) of L = sum_t dout_t . O_t, O the forward output."""
    q, k, v = _check_qkv(q, k, v)
    dout = _f64(dout)
    if dout.shape != q.shape:
        raise ValueError("dout must have the shape of q")
    T, H, d = q.shape
    cu, cup = _cu(cu_seqlens, T)
    nseq = cu.size - 1
    init = _init(init, nseq, H, d)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    dinit = np.zeros((nseq, H, d, d))
    _load().oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), cup, nseq, H, d, _ptr(init),
                            _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dinit))
    return dq, dk, dv, dinit


# ---------------------------------------------------------------- decay variant
# S_t = lambda_h S_{t-1} + k_t^T v_t, o_t = q_t S_t (lambda = 1: the functions above).

def _lam(decay, H):
    lam = _f64(decay)
    if lam.shape != (H,):
        raise ValueError("decay must be [H]")
    if np.any(~np.isfinite(lam)) or np.any(lam < 0) or np.any(lam > 1):
        raise ValueError("decay rates must lie in [0, 1]")
    return lam


def decay_quadratic(q, k, v, decay, cu_seqlens=None, init=None):
    """O_t = lambda^(t-start+1) q_t S0 + sum_{s<=t} lambda^(t-s) (q_t . k_s) v_s, term by term."""
    q, k, v = _check_qkv(q, k, v)
    T, H, d = q.shape
    cu, cup = _cu(cu_seqlens, T)
    init = _init(init, cu.size - 1, H, d)
    lam = _lam(decay, H)
    o = np.zeros_like(q)
    _load().oracle_decay_quadratic(_ptr(q), _ptr(k), _ptr(v), _ptr(o), cup, cu.size - 1, H, d,
                                   _ptr(init), _ptr(lam))
    return o


def decay_recurrent(q, k, v, decay, cu_seqlens=None, init=None, return_state=False):
    """S = lambda S + k^T v; o = q S, token by token. Optionally returns the final state."""
    q, k, v = _check_qkv(q, k, v)
    T, H, d = q.shape
    cu, cup = _cu(cu_seqlens, T)
    nseq = cu.size - 1
    init = _init(init, nseq, H, d)
    lam = _lam(decay, H)
    o = np.zeros_like(q)
    st = np.zeros((nseq, H, d, d)) if return_state else None
    _load().oracle_decay_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(o), cup, nseq, H, d,
                                   _ptr(init), _ptr(lam), _ptr(st))
    return (o, st) if return_state else o


def decay_blocked(q, k, v, decay, B, cu_seqlens=None, init=None, return_state=False):
    """Block decomposition with decay mask, lambda^(r+1)-scaled inter term and decayed prefix."""
    q, k, v = _check_qkv(q, k, v)
    T, H, d = q.shape
    if int(B) < 1:
        raise ValueError("B must be >= 1")
    cu, cup = _cu(cu_seqlens, T)
    nseq = cu.size - 1
    init = _init(init, nseq, H, d)
    lam = _lam(decay, H)
    o = np.zeros_like(q)
    st = np.zeros((nseq, H, d, d)) if return_state else None
    _load().oracle_decay_blocked(_ptr(q), _ptr(k), _ptr(v), _ptr(o), cup, nseq, H, d, int(B),
                                 _ptr(init), _ptr(lam), _ptr(st))
    return (o, st) if return_state else o


def decay_state(k, v, decay, cu_seqlens=None, init=None):
    """Final state per (sequence, head): lambda^n S0 + sum_t lambda^(end-1-t) k_t^T v_t."""
    k, v = _f64(k), _f64(v)
    if k.ndim != 3 or k.shape != v.shape:
        raise ValueError("k, v must share one shape [T, H, d]")
    T, H, d = k.shape
    cu, cup = _cu(cu_seqlens, T)
    nseq = cu.size - 1
    init = _init(init, nseq, H, d)
    lam = _lam(decay, H)
    st = np.zeros((nseq, H, d, d))
    _load().oracle_decay_state(_ptr(k), _ptr(v), cup, nseq, H, d, _ptr(init), _ptr(lam), _ptr(st))
    return st


def decay_decode_step(q, k, v, state_in, decay):
    """One step S = lambda S + k^T v; o = q S on [batch, H, d]; returns (o, new_state)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim != 3 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one shape [batch, H, d]")
    batch, H, d = q.shape
    st = np.array(state_in, dtype=np.float64, copy=True, order="C")
    if st.shape != (batch, H, d, d):
        raise ValueError("state must be [batch, H, d, d]")
    lam = _lam(decay, H)
    o = np.zeros_like(q)
    _load().oracle_decay_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(st), _ptr(o), batch, H, d, _ptr(lam))
    return o, st


def decay_backward(q, k, v, dout, decay, cu_seqlens=None, init=None):
    """Gradients (dq, dk, dv, dinit) of L = sum_t dout_t . O_t for the decay variant's O."""
    q, k, v = _check_qkv(q, k, v)
    dout = _f64(dout)
    if dout.shape != q.shape:
        raise ValueError("dout must have the shape of q")
    T, H, d = q.shape
    cu, cup = _cu(cu_seqlens, T)
    nseq = cu.size - 1
    init = _init(init, nseq, H, d)
    lam = _lam(decay, H)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    dinit = np.zeros((nseq, H, d, d))
    _load().oracle_decay_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), cup, nseq, H, d, _ptr(init), _ptr(lam),
                                  _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dinit))
    return dq, dk, dv, dinit


def feature_map(x, alpha=0.3):
    """phi(x) = ELU(x) + alpha x elementwise, same shape as x."""
    x = _f64(x)
    y = np.zeros_like(x)
    _load().oracle_feature_map(_ptr(x.reshape(-1)), _ptr(y.reshape(-1)), x.size, float(alpha))
    return y


def num_threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS or all host cores)."""
    return int(_load().oracle_num_threads())
