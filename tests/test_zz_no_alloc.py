"""la_prefill_noalloc: the prefill entry point for callers that cannot allocate.

Such callers (allocator-free runtimes, fixed memory budgets, hooks running
inside another library's memory manager) get the same prefill with the
scratch taken from a static device array built into the library. These checks
call it through the C ABI and compare it with the fp64 oracle and with the
workspace entry point, la_prefill, on two calls in a row (the second call
reuses the scratch the first one left behind), within the tolerances of the
parity tests.
This file sorts last so that a failure here cannot hide another test's.
"""
import ctypes

import numpy as np
import pytest
import torch

import causal_linear_attention_02_b200 as la
import oracle
import workloads as wl

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


@pytest.fixture(scope="module", autouse=True)
def _library():
    from causal_linear_attention_02_b200 import build
    build.build()
    la.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(DEV)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _rel(a, b):
    a = a.float().cpu().double().numpy()
    b = b.float().cpu().double().numpy()
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))


@pytest.mark.parametrize("dtype,d,B", [(torch.bfloat16, 128, 256), (torch.float32, 64, 64)],
                         ids=["bf16-tensor-cores", "fp32-cuda-cores"])
def test_noalloc_matches_workspace_prefill_twice(dtype, d, B):
    stream = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
    code = la.LA_BF16 if dtype == torch.bfloat16 else la.LA_FP32
    tol = 1e-2 if dtype == torch.bfloat16 else 1e-4
    for seed, lengths in ((21, [700, 1, 300]), (22, [1500])):      # two calls in a row
        T, H = sum(lengths), 4
        q, k, v = wl.qkv(T, H, d, dtype, seed, device=DEV)
        cu = wl.cu_seqlens(lengths, device=DEV)
        ref = la.prefill(q, k, v, cu, B=B)
        o = torch.full_like(q, float("nan"))
        status = la.la_prefill_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(cu), len(lengths), T, H, d, B,
                                       code, None, stream)
        assert status == 0, la.STATUS.get(status, status)
        assert la.device_status() == 0
        assert torch.isfinite(o.float()).all()
        r = _rel(o, ref)
        assert r <= tol, f"no-alloc vs workspace prefill: {r:.3e} > {tol:.0e}"
        f = lambda t: t.float().cpu().double().numpy()
        exact = oracle.recurrent(f(q), f(k), f(v), cu_seqlens=cu.cpu().numpy())
        e = float(np.abs(f(o) - exact).max() / np.abs(exact).max())
        assert e <= tol, f"no-alloc vs oracle: {e:.3e} > {tol:.0e}"


def test_noalloc_rejects_problems_beyond_its_scratch():
    # fp32 at B = 64 keeps two d x d states per (block, head): 8192 tokens x 8 heads need
    # about 132 MB of scratch, twice the static array
    T, H, d, B = 8192, 8, 128, 64
    assert la.la_prefill_workspace_size(T, 1, H, d, B, la.LA_FP32) > la.LA_NOALLOC_SCRATCH_BYTES
    q, k, v = wl.qkv(T, H, d, torch.float32, 23, device=DEV)
    o = torch.full_like(q, float("nan"))
    stream = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
    status = la.la_prefill_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), None, 1, T, H, d, B, la.LA_FP32, None, stream)
    assert status == 4                           # LA_ERR_WORKSPACE_TOO_SMALL, before anything is enqueued
    torch.cuda.synchronize(DEV)
    assert torch.isnan(o).all()                  # nothing was written
