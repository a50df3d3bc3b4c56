"""GPU parity: every entry point through the C ABI against the fp64 oracle.

Tolerances (bound on the whole output, relative to its largest magnitude):
  bf16 inputs, fp32 accumulation:  max|O - O_ref| <= 1e-2 * max|O_ref|
  fp32 inputs:                     max|O - O_ref| <= 1e-4 * max|O_ref|
Integer-valued inputs are exact in every intermediate, so there the bf16
output must equal the oracle result rounded to bf16, bit for bit.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import causal_linear_attention_02_b200 as la
import oracle
import workloads as wl

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
TOL = {torch.bfloat16: 1e-2, torch.float32: 1e-4}


@pytest.fixture(scope="module", autouse=True)
def _library():
    from causal_linear_attention_02_b200 import build
    build.build()
    la.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(DEV)


def f64(t):
    return t.detach().float().cpu().double().numpy() if t.dtype == torch.bfloat16 else \
        t.detach().cpu().double().numpy()


def rel_err(out, ref):
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(out - ref).max(initial=0.0) / max(np.abs(ref).max(initial=0.0), 1e-30))


def assert_close(out, ref, tol, what=""):
    r = rel_err(out, ref)
    assert r <= tol, f"{what}: max|O-O_ref|/max|O_ref| = {r:.3e} > {tol:.0e}"
    return r


def inputs(T, H, d, dtype, seed):
    return wl.qkv(T, H, d, dtype, seed, device=DEV)


def status_ok():
    s = la.device_status()
    assert s == 0, f"device status {la.STATUS.get(s, s)}"


def cu_of(lengths):
    return wl.cu_seqlens(lengths, device=DEV)


# The two tensor-core prefill kernels (la_debug_set_path): 1 = on-chip state,
# one CTA per (sequence, head, value-column half); 2 = block-parallel with a
# decoupled look-back scan. Tests taking `tc_path` run under both.
@pytest.fixture(params=[1, 2], ids=["onchip", "lookback"])
def tc_path(request):
    assert la.la_debug_set_path(request.param) == 0
    yield request.param
    la.la_debug_set_path(0)


def force_path(path):
    assert la.la_debug_set_path(path) == 0


# ------------------------------------------------------------------ decode
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("d", [16, 48, 64, 128])
def test_decode_steps(dtype, d):
    batch, H, steps = 5, 3, 3
    st = wl.state_init(batch, H, d, seed=d, device=DEV)
    ref_state = st.cpu().double().numpy()
    q, k, v = wl.decode_inputs(batch, H, d, steps, dtype, seed=7 + d, device=DEV)
    for t in range(steps):
        o = la.decode_step(q[t], k[t], v[t], st)
        ref_o, ref_state = oracle.decode_step(f64(q[t]), f64(k[t]), f64(v[t]), ref_state)
        assert_close(f64(o), ref_o, TOL[dtype], f"decode o step {t}")
    assert_close(st.cpu().double().numpy(), ref_state, 1e-5, "decode state")
    status_ok()


# ------------------------------------------------------------------ prefill, fp32 small workload
def test_prefill_fp32_small_workload():
    w = wl.FP32_SMALL
    q, k, v = inputs(w.total_tokens, w.heads, w.d, torch.float32, w.seed)
    o = la.prefill(q, k, v, B=w.B)
    status_ok()
    ref = oracle.quadratic(f64(q), f64(k), f64(v))
    assert_close(f64(o), ref, 1e-4, "fp32 T=1024 H=2 d=64 B=64")


# ------------------------------------------------------------------ prefill, tensor-core path
@pytest.mark.parametrize("B", [128, 256])
@pytest.mark.parametrize("T", [1, 37, 128, 255, 256, 257, 1000, 1500])
def test_prefill_tc_random(B, T, tc_path):
    H, d = 3, 128
    q, k, v = inputs(T, H, d, torch.bfloat16, seed=T * 7 + B)
    o = la.prefill(q, k, v, B=B)
    status_ok()
    ref = oracle.recurrent(f64(q), f64(k), f64(v))
    assert_close(f64(o), ref, 1e-2, f"tc T={T} B={B}")


@pytest.mark.parametrize("B,T", [(256, 512), (128, 384), (256, 300), (128, 200)])
def test_prefill_tc_integer_exact(B, T, tc_path):
    """{-1,0,1} inputs: scores, P, every prefix entry and O are exact integers in
    bf16/fp32, so the result must equal the oracle's rounded to bf16 bit for bit."""
    H, d = 2, 128
    q, k, v = wl.integer_qkv(T, H, d, torch.bfloat16, seed=B + T, device=DEV)
    for n in range(B, T, B):   # every prefix state the inter-block product uses
        assert np.abs(oracle.state(f64(k)[:n], f64(v)[:n])).max() <= 256, "precondition: bf16-exact prefix"
    o = la.prefill(q, k, v, B=B)
    status_ok()
    ref = torch.from_numpy(oracle.recurrent(f64(q), f64(k), f64(v))).to(torch.bfloat16)
    got = o.cpu()
    mism = (got.view(torch.int16) != ref.view(torch.int16)).sum().item()
    assert mism == 0, f"{mism} of {ref.numel()} outputs differ from the exact result"


def test_prefill_fp32_integer_exact():
    """The small fp32 workload's shape (T = 1024, H = 2, d = 64, B = 64: the CUDA-core
    three-kernel path) with {-1,0,1} inputs: every score, block state, prefix entry and
    output is an integer far below 2^24, exact in fp32, so the output must equal the
    oracle's bit for bit."""
    w = wl.FP32_SMALL
    T, H, d, B = w.total_tokens, w.heads, w.d, w.B
    q, k, v = wl.integer_qkv(T, H, d, torch.float32, seed=91, device=DEV)
    o = la.prefill(q, k, v, B=B)
    status_ok()
    ref = oracle.recurrent(f64(q), f64(k), f64(v))
    assert np.abs(ref).max() < 2 ** 24 and np.abs(oracle.state(f64(k), f64(v))).max() < 2 ** 24
    got = o.cpu().double().numpy()
    mism = int((got != ref).sum())
    assert mism == 0, f"{mism} of {ref.size} fp32 outputs differ from the exact result"


def test_lookback_finishes_beside_another_kernel():
    """The block-parallel kernel (forced) while another stream's matmul loop holds SMs for about
    a second, with the device wait limit cut to 300 ms: its CTAs take tiles by ticket, so a tile's
    predecessors always belong to CTAs that are already running, and the call ends with LA_OK and
    the oracle's result (it never waits on a CTA that is not resident)."""
    T, H, d, B = 12000, 2, 128, 256               # 47 blocks x 2 heads = 94 tiles
    q, k, v = inputs(T, H, d, torch.bfloat16, seed=77)
    ref = oracle.recurrent(f64(q), f64(k), f64(v))
    a = torch.randn(8192, 8192, device=DEV, dtype=torch.bfloat16)
    side = torch.cuda.Stream(DEV)
    torch.cuda.synchronize(DEV)
    assert la.la_debug_set_fault(-1, 300_000_000) == 0
    force_path(2)
    try:
        with torch.cuda.stream(side):
            for _ in range(1200):                 # about a second of 8192^3 bf16 products
                c = a @ a
        o = la.prefill(q, k, v, B=B)              # the current stream, beside them
        torch.cuda.synchronize(DEV)
    finally:
        la.la_debug_set_fault(-1, 0)
        force_path(0)
    del c
    status_ok()
    assert_close(f64(o), ref, 1e-2, "block-parallel prefill beside another kernel")


@pytest.mark.parametrize("B", [128, 256])
def test_prefill_tc_varlen(B, tc_path):
    lengths = [1, 255, 256, 0, 257, 700, 64, 513, 128]
    H, d = 2, 128
    T = sum(lengths)
    q, k, v = inputs(T, H, d, torch.bfloat16, seed=99 + B)
    cu = cu_of(lengths)
    o = la.prefill(q, k, v, cu, B=B)
    status_ok()
    ref = oracle.recurrent(f64(q), f64(k), f64(v), cu.cpu().numpy())
    assert_close(f64(o), ref, 1e-2, f"tc varlen B={B}")


@pytest.mark.parametrize("dtype,d,B", [(torch.bfloat16, 128, 256), (torch.bfloat16, 128, 128),
                                       (torch.float32, 64, 64), (torch.bfloat16, 64, 128)])
def test_prefill_init_state(dtype, d, B, tc_path):
    lengths = [300, 1, 520]
    H = 2
    T = sum(lengths)
    q, k, v = inputs(T, H, d, dtype, seed=5 + d)
    cu = cu_of(lengths)
    init = wl.state_init(len(lengths), H, d, seed=3, device=DEV, scale=4.0)
    o = la.prefill(q, k, v, cu, B=B, init_state=init)
    status_ok()
    ref = oracle.recurrent(f64(q), f64(k), f64(v), cu.cpu().numpy(), init=init.cpu().double().numpy())
    assert_close(f64(o), ref, TOL[dtype], "prefill with carried-in state")


# ------------------------------------------------------------------ prefill, CUDA-core path
@pytest.mark.parametrize("dtype,d,B", [
    (torch.float32, 64, 64), (torch.float32, 128, 256), (torch.float32, 48, 128), (torch.float32, 16, 64),
    (torch.bfloat16, 64, 128), (torch.bfloat16, 16, 64), (torch.bfloat16, 128, 64), (torch.bfloat16, 112, 256),
])
def test_prefill_simt_shapes(dtype, d, B):
    lengths = [70, 1, 0, 333, 64]
    H = 3
    T = sum(lengths)
    q, k, v = inputs(T, H, d, dtype, seed=d + B)
    cu = cu_of(lengths)
    o = la.prefill(q, k, v, cu, B=B)
    status_ok()
    ref = oracle.recurrent(f64(q), f64(k), f64(v), cu.cpu().numpy())
    assert_close(f64(o), ref, TOL[dtype], f"simt {dtype} d={d} B={B}")


def test_prefill_b_independence():
    """The result does not depend on B (up to rounding): B = 128 and 256 agree."""
    q, k, v = inputs(1200, 2, 128, torch.bfloat16, seed=4242)
    o1 = la.prefill(q, k, v, B=128)
    o2 = la.prefill(q, k, v, B=256)
    o3 = la.prefill(q, k, v, B=64)
    status_ok()
    ref = oracle.recurrent(f64(q), f64(k), f64(v))
    for o in (o1, o2, o3):
        assert_close(f64(o), ref, 1e-2, "B independence")


# ------------------------------------------------------------------ state and continuity
@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64), (torch.bfloat16, 32)])
def test_state_from_prefill(dtype, d):
    lengths = [5000, 0, 1, 2049, 300]
    H = 2
    T = sum(lengths)
    _, k, v = inputs(T, H, d, dtype, seed=31 + d)
    cu = cu_of(lengths)
    init = wl.state_init(len(lengths), H, d, seed=4, device=DEV)
    ref = oracle.state(f64(k), f64(v), cu.cpu().numpy(), init=init.cpu().double().numpy())
    st = la.state_from_prefill(k, v, cu, init_state=init)
    assert_close(st.cpu().double().numpy(), ref, 1e-5, "state")
    st2 = init.clone()
    la.state_from_prefill(k, v, cu, init_state=st2, out=st2)      # in-place accumulate
    status_ok()
    assert_close(st2.cpu().double().numpy(), ref, 1e-5, "state in place")


@pytest.mark.parametrize("B", [128, 256])
def test_prefill_state_decode_continuity(B):
    """Prefill of m tokens -> state -> decode steps reproduces the rows of one
    prefill over m + n tokens (ties the three entry points together)."""
    H, d, m, n = 4, 128, 700, 6
    q, k, v = inputs(m + n, H, d, torch.bfloat16, seed=77)
    full = la.prefill(q, k, v, B=B)
    st = la.state_from_prefill(k[:m].contiguous(), v[:m].contiguous())
    st = st.view(1, H, d, d).clone()
    outs = []
    for t in range(m, m + n):
        outs.append(la.decode_step(q[t:t + 1].contiguous(), k[t:t + 1].contiguous(), v[t:t + 1].contiguous(), st))
    status_ok()
    dec = torch.cat(outs)
    ref = oracle.recurrent(f64(q), f64(k), f64(v))
    assert_close(f64(dec), ref[m:], 1e-2, "decode rows vs oracle")
    assert_close(f64(full)[m:], ref[m:], 1e-2, "prefill rows vs oracle")


# ------------------------------------------------------------------ edge cases
def test_empty_input():
    q = torch.empty((0, 2, 128), dtype=torch.bfloat16, device=DEV)
    o = la.prefill(q, q, q.clone(), B=256)
    assert o.shape == (0, 2, 128)
    status_ok()


def test_bad_seqlens_reported_on_device():
    T, H, d = 20, 2, 64
    q, k, v = inputs(T, H, d, torch.float32, seed=1)
    cu = torch.tensor([0, 10, 5, 20], dtype=torch.int32, device=DEV)   # decreasing
    o = torch.full_like(q, 7.0)
    la.prefill(q, k, v, cu, B=64, out=o)
    assert la.device_status() == 7
    assert la.device_status() == 0                                    # cleared by the read
    assert torch.all(o == 7.0), "no output rows are written when cu_seqlens is rejected"
    cu2 = torch.tensor([0, 10, 19], dtype=torch.int32, device=DEV)    # does not end at T
    la.prefill(q, k, v, cu2, B=64, out=o)
    assert la.device_status() == 7


# ------------------------------------------------------------------ single-pass scheduling corners
@pytest.mark.parametrize("T,H,B", [
    (8192, 2, 256),      # 32 blocks per chain, few tiles: look-backs run deep and wait for inclusives
    (65536, 1, 256),     # one chain longer than the grid: predecessors on every other CTA
    (4096, 148, 128),    # one tile per SM per block: a tile's predecessor runs on its own CTA
    (20001, 7, 128),     # ragged tail, odd head count
    (3000, 64, 256),     # the 64-head shape, short
])
def test_prefill_single_pass_chains(T, H, B):
    q, k, v = inputs(T, H, 128, torch.bfloat16, seed=T + H + B)
    force_path(2)
    try:
        o = la.prefill(q, k, v, B=B)
    finally:
        force_path(0)
    status_ok()
    ref = oracle.recurrent(f64(q), f64(k), f64(v))
    assert_close(f64(o), ref, 1e-2, f"single pass T={T} H={H} B={B}")


def test_prefill_many_sequences_share_slots(tc_path):
    """Many packed sequences (some shorter than one block, some spanning many
    slot-ring generations) in one launch."""
    lengths = wl.varlen_lengths(40, 1, 3000, seed=8)
    H = 3
    T = sum(lengths)
    q, k, v = inputs(T, H, 128, torch.bfloat16, seed=88)
    cu = cu_of(lengths)
    init = wl.state_init(len(lengths), H, 128, seed=9, device=DEV)
    o = la.prefill(q, k, v, cu, B=256, init_state=init)
    status_ok()
    ref = oracle.recurrent(f64(q), f64(k), f64(v), cu.cpu().numpy(), init=init.cpu().double().numpy())
    assert_close(f64(o), ref, 1e-2, "40 packed sequences")


def test_lost_publication_ends_in_timeout_not_hang():
    """A tile that never publishes its state makes its successors' bounded
    waits expire: the launch ends by itself, the status word says TIMEOUT and
    the context stays usable for a correct run right after."""
    T, H, B = 4096, 4, 256
    q, k, v = inputs(T, H, 128, torch.bfloat16, seed=5150)
    suppress = 5 * H + 1                      # block 5 of head 1
    assert la.la_debug_set_fault(suppress, 200_000_000) == 0
    force_path(2)
    try:
        t0 = time.time()
        la.prefill(q, k, v, B=B)
        st = la.device_status()
        elapsed = time.time() - t0
    finally:
        la.la_debug_set_fault(-1, 0)
        force_path(0)
    assert st == 6, f"expected LA_ERR_TIMEOUT, got {la.STATUS.get(st, st)}"
    assert elapsed < 30, f"timed-out launch took {elapsed:.1f}s"
    o = la.prefill(q, k, v, B=B)
    status_ok()
    assert_close(f64(o), oracle.recurrent(f64(q), f64(k), f64(v)), 1e-2, "run after a timeout")


# ------------------------------------------------------------------ on-chip-state scheduling corners
@pytest.mark.parametrize("lengths,H,B", [
    ([8192], 2, 256),                       # 4 work items, 32 blocks each
    ([3000] * 3, 64, 256),                  # 384 work items: every CTA takes two or three
    ([4096], 148, 128),                     # 296 work items of equal length
    ([20001], 7, 128),                      # ragged tail, odd head count
    ([1, 2, 255, 256, 257, 4000, 0, 129, 1024, 3], 9, 256),   # mixed lengths, longest first
])
def test_prefill_onchip_scheduling(lengths, H, B):
    T = sum(lengths)
    q, k, v = inputs(T, H, 128, torch.bfloat16, seed=T + H + B + 1)
    cu = cu_of(lengths)
    force_path(1)
    try:
        o = la.prefill(q, k, v, cu, B=B)
    finally:
        force_path(0)
    status_ok()
    ref = oracle.recurrent(f64(q), f64(k), f64(v), cu.cpu().numpy())
    assert_close(f64(o), ref, 1e-2, f"on-chip state lengths={lengths[:4]} H={H} B={B}")


def test_withheld_prefix_ends_in_timeout_not_hang():
    """On the on-chip-state kernel, a work item whose state group never hands
    over a block prefix makes the tensor-core issuer's bounded wait expire:
    the launch ends by itself with LA_ERR_TIMEOUT and the next call is right."""
    T, H, B = 4096, 4, 256
    q, k, v = inputs(T, H, 128, torch.bfloat16, seed=5151)
    assert la.la_debug_set_fault(3, 200_000_000) == 0
    force_path(1)
    try:
        t0 = time.time()
        la.prefill(q, k, v, B=B)
        st = la.device_status()
        elapsed = time.time() - t0
    finally:
        la.la_debug_set_fault(-1, 0)
    try:
        assert st == 6, f"expected LA_ERR_TIMEOUT, got {la.STATUS.get(st, st)}"
        assert elapsed < 30, f"timed-out launch took {elapsed:.1f}s"
        o = la.prefill(q, k, v, B=B)
        status_ok()
    finally:
        force_path(0)
    assert_close(f64(o), oracle.recurrent(f64(q), f64(k), f64(v)), 1e-2, "run after a timeout")


# ---------------------------------------------------------------- sequence parallelism (LASP+)
@pytest.mark.gpu
def test_state_exclusive_prefix():
    W, nseq, H, d = 4, 3, 2, 128
    g = torch.randn(W, nseq, H, d, d, device=DEV, generator=torch.Generator(DEV).manual_seed(5))
    init = torch.randn(nseq, H, d, d, device=DEV, generator=torch.Generator(DEV).manual_seed(6))
    g64, i64 = g.double().cpu().numpy(), init.double().cpu().numpy()
    for rank in range(W + 1):
        for ini in (None, init):
            out = la.state_exclusive_prefix(g, rank, ini)
            ref = g64[:rank].sum(0) + (0.0 if ini is None else i64)
            assert_close(out.cpu().double().numpy(), ref, 1e-6, f"rank {rank}")
    inplace = init.clone()
    la.state_exclusive_prefix(g, 2, inplace, out=inplace)
    assert_close(inplace.cpu().double().numpy(), g64[:2].sum(0) + i64, 1e-6, "in place")
    status_ok()
    sh = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    n = nseq * H
    assert la.la_state_exclusive_prefix(P(g), W, W + 1, n, d, None, P(init), sh) == 1      # rank > world
    assert la.la_state_exclusive_prefix(P(g), W, 1, n, 100, None, P(init), sh) == 2        # d
    assert la.la_state_exclusive_prefix(P(g), W, 1, n, d, None, P(g[1]), sh) == 1          # out inside gathered
    assert la.la_state_exclusive_prefix(ctypes.c_void_p(g.data_ptr() + 4), W, 1, n, d, None, P(init), sh) == 3
    assert la.la_state_exclusive_prefix(P(g), W, 1, 0, d, None, P(init), sh) == 0          # nothing to do


@pytest.mark.gpu
@pytest.mark.parametrize("W,B", [(2, 256), (4, 256), (3, 128)])
def test_lasp_segments_on_one_gpu(W, B):
    """LASP+ composed from the library calls, the ranks emulated one after another
    on one GPU (the all-gather is a stack): every segment's output and the final
    state equal those of the whole sequences."""
    lengths, H, d = [1500, 777], 2, 128
    T = sum(lengths)
    q, k, v = inputs(T, H, d, torch.bfloat16, seed=70 + W)
    init = wl.state_init(len(lengths), H, d, seed=9, device=DEV)
    rng = np.random.default_rng(W)
    cuts = [[0, *np.sort(rng.choice(np.arange(1, L), size=W - 1, replace=False)).tolist(), L] for L in lengths]
    starts = np.cumsum([0] + lengths[:-1])
    rows = [np.concatenate([np.arange(s0 + c[r], s0 + c[r + 1]) for s0, c in zip(starts, cuts)]) for r in range(W)]
    segs = []
    for r in range(W):
        idx = torch.from_numpy(rows[r]).to(DEV)
        cu = cu_of([c[r + 1] - c[r] for c in cuts])
        segs.append((q[idx].contiguous(), k[idx].contiguous(), v[idx].contiguous(), cu))
    gathered = torch.stack([la.state_from_prefill(kr, vr, cu) for _, kr, vr, cu in segs])
    o = torch.empty_like(q)
    for r, (qr, kr, vr, cu) in enumerate(segs):
        start = la.state_exclusive_prefix(gathered, r, init)
        o[torch.from_numpy(rows[r]).to(DEV)] = la.prefill(qr, kr, vr, cu, B=B, init_state=start)
    final = la.state_exclusive_prefix(gathered, W, init)
    status_ok()
    cu_all = cu_of(lengths).cpu().numpy()
    ref = oracle.recurrent(f64(q), f64(k), f64(v), cu_all, init=init.cpu().double().numpy())
    assert_close(f64(o), ref, TOL[torch.bfloat16], "LASP+ output")
    ref_state = oracle.state(f64(k), f64(v), cu_all, init=init.cpu().double().numpy())
    assert_close(final.cpu().double().numpy(), ref_state, 1e-5, "LASP+ final state")


# ---------------------------------------------------------------- backward (training pass)
@pytest.mark.parametrize("dtype,d,B", [(torch.bfloat16, 128, 256), (torch.bfloat16, 128, 128),
                                       (torch.float32, 64, 64)], ids=["bf16-256", "bf16-128", "fp32-64"])
@pytest.mark.parametrize("with_init", [False, True], ids=["zero-S0", "S0"])
def test_prefill_backward(dtype, d, B, with_init, tc_path):
    """dq, dk, dv, dS0 of L = sum dO . O against the oracle's gradients."""
    if dtype == torch.float32 and tc_path == 2:
        pytest.skip("fp32 has one path")
    lengths, H = [700, 0, 1, 1300, 255], 2
    T = sum(lengths)
    q, k, v = inputs(T, H, d, dtype, seed=80 + d)
    dout = wl.normal_scaled((T, H, d), d, dtype, 81 + d, device=DEV)
    cu = cu_of(lengths)
    init = wl.state_init(len(lengths), H, d, seed=8, device=DEV) if with_init else None
    dq, dk, dv, dinit = la.prefill_backward(q, k, v, dout, cu, B=B, init_state=init, need_init_grad=True)
    status_ok()
    ref = oracle.backward(f64(q), f64(k), f64(v), f64(dout), cu.cpu().numpy(),
                          init=None if init is None else init.cpu().double().numpy())
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref[:3]):
        assert_close(f64(got), want, TOL[dtype], name)
    assert_close(dinit.cpu().double().numpy(), ref[3], 1e-5, "dS0")


def test_prefill_backward_default_path_many_heads():
    """32 heads: the automatic path is the on-chip-state kernel, so dk and dv come from its
    anti-causal instance (blocks walked from each sequence's end, ragged last blocks with 188,
    16 and 0 extra rows, a one-token sequence) with no sequence reversal; against the oracle."""
    lengths, H, d, B = [700, 1, 1296, 256, 40], 32, 128, 256
    T = sum(lengths)
    q, k, v = inputs(T, H, d, torch.bfloat16, seed=83)
    dout = wl.normal_scaled((T, H, d), d, torch.bfloat16, 84, device=DEV)
    cu = cu_of(lengths)
    init = wl.state_init(len(lengths), H, d, seed=9, device=DEV)
    dq, dk, dv, dinit = la.prefill_backward(q, k, v, dout, cu, B=B, init_state=init, need_init_grad=True)
    status_ok()
    heads = [0, 17, 31]
    sel = lambda t: f64(t[:, heads])
    ref = oracle.backward(sel(q), sel(k), sel(v), sel(dout), cu.cpu().numpy(),
                          init=init[:, heads].cpu().double().numpy())
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref[:3]):
        assert_close(sel(got), want, TOL[torch.bfloat16], name)
    assert_close(dinit[:, heads].cpu().double().numpy(), ref[3], 1e-5, "dS0")


@pytest.mark.gpu
def test_prefill_backward_arguments():
    T, H, d, B = 300, 2, 128, 256
    q, k, v = inputs(T, H, d, torch.bfloat16, seed=90)
    dout = wl.normal_scaled((T, H, d), d, torch.bfloat16, 91, device=DEV)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    sh = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
    wsb = la.la_prefill_backward_workspace_size(T, 1, H, d, B, la.LA_BF16)
    ws = torch.empty(wsb, dtype=torch.uint8, device=DEV)
    call = lambda dq_, ws_bytes=wsb: la.la_prefill_backward(P(q), P(k), P(v), P(dout), None, 1, T, H, d, B,
                                                             la.LA_BF16, None, P(dq_), P(dk), P(dv), None, P(ws),
                                                             ws_bytes, sh)
    assert call(q) == 1                       # dq aliases q
    assert call(dk) == 1                      # dq aliases dk
    assert call(dq, wsb - 256) == 4           # workspace too small
    assert call(dq) == 0
    status_ok()
    # no tokens: dS0 = 0
    z = torch.empty(0, H, d, dtype=torch.bfloat16, device=DEV)
    _, _, _, dinit = la.prefill_backward(z, z, z, z, need_init_grad=True)
    status_ok()
    assert torch.count_nonzero(dinit) == 0


@pytest.mark.gpu
def test_autograd_function_matches_backward():
    from causal_linear_attention_02_b200.autograd import lightning_attention
    lengths, H, d = [513, 300], 2, 128
    T = sum(lengths)
    q, k, v = (x.requires_grad_(True) for x in inputs(T, H, d, torch.bfloat16, seed=95))
    init = wl.state_init(len(lengths), H, d, seed=3, device=DEV).requires_grad_(True)
    cu = cu_of(lengths)
    dout = wl.normal_scaled((T, H, d), d, torch.bfloat16, 96, device=DEV)
    o = lightning_attention(q, k, v, cu, 256, init)
    o.backward(dout)
    status_ok()
    ref = oracle.backward(f64(q), f64(k), f64(v), f64(dout), cu.cpu().numpy(), init=init.detach().cpu().double().numpy())
    for name, got, want in zip(("dq", "dk", "dv"), (q.grad, k.grad, v.grad), ref[:3]):
        assert_close(f64(got), want, TOL[torch.bfloat16], name)
    assert_close(init.grad.cpu().double().numpy(), ref[3], 1e-5, "dS0")
    assert_close(f64(o.detach()), oracle.recurrent(f64(q), f64(k), f64(v), cu.cpu().numpy(),
                                                   init=init.detach().cpu().double().numpy()), TOL[torch.bfloat16], "O")


# ---------------------------------------------------------------- prefill with the final state
@pytest.mark.parametrize("lengths,H,B,dtype", [
    ([5000, 1, 15, 16, 17, 300, 0, 2049], 8, 256, torch.bfloat16),   # on-chip-state path, ragged tails
    ([1, 7, 130, 255, 256, 257], 16, 128, torch.bfloat16),
    ([700, 33], 2, 256, torch.bfloat16),                              # block-parallel path (few work items)
    ([300, 45], 2, 64, torch.float32),                                # SIMT path
], ids=["onchip-256", "onchip-128", "lookback", "fp32"])
@pytest.mark.parametrize("with_init", [False, True], ids=["zero-S0", "S0"])
def test_prefill_with_state(lengths, H, B, dtype, with_init):
    d = 128 if dtype == torch.bfloat16 else 64
    T = sum(lengths)
    q, k, v = inputs(T, H, d, dtype, seed=110 + len(lengths))
    cu = cu_of(lengths)
    init = wl.state_init(len(lengths), H, d, seed=11, device=DEV) if with_init else None
    o, st = la.prefill_with_state(q, k, v, cu, B=B, init_state=init)
    status_ok()
    init64 = None if init is None else init.cpu().double().numpy()
    ref_o, ref_s = oracle.recurrent(f64(q), f64(k), f64(v), cu.cpu().numpy(), init=init64, return_state=True)
    assert_close(f64(o), ref_o, TOL[dtype], "O")
    assert_close(st.cpu().double().numpy(), ref_s, 1e-5, "final state")
    if with_init:
        # in place: the state is updated from itself
        st2 = init.clone()
        o2, _ = la.prefill_with_state(q, k, v, cu, B=B, init_state=st2, state_out=st2)
        status_ok()
        assert_close(st2.cpu().double().numpy(), ref_s, 1e-5, "final state, in place")
        if dtype == torch.bfloat16 and 2 * len(lengths) * H < 64:
            # the block-parallel kernel's decoupled look-back adds the predecessors' aggregates and
            # inclusive prefixes in the order their flags arrive, so two calls agree up to fp32
            # rounding of the prefix, not bit for bit
            assert_close(f64(o2), ref_o, TOL[dtype], "O, in place")
        else:
            assert torch.equal(o2, o)


def _mixed_batch(seed, n_cont=500):
    """A serving batch: four prompts of 257 to 3001 tokens, n_cont one-token continuations and two
    empty sequences, shuffled together (the lengths in a seeded random order)."""
    rng = np.random.default_rng(seed)
    lengths = [3001, 1000, 1500, 257] + [1] * n_cont + [0, 0]
    return [int(x) for x in rng.permutation(lengths)]


@pytest.mark.parametrize("decay", [False, True], ids=["plain", "decay"])
@pytest.mark.parametrize("in_place", [False, True], ids=["out", "in-place"])
def test_prefill_with_state_mixed_batch(decay, in_place):
    """One launch for a mixed batch on the on-chip-state kernel's state-output instance: the
    prompts as chain work items, the one-token continuations as decode steps from their own
    carried-in states (taken by the CTAs once their chain items are done). O of every token
    and the final states of heads 0 and 31 against the oracle."""
    lengths, H, d, B = _mixed_batch(5 + decay + 2 * in_place), 32, 128, 256
    T = sum(lengths)
    q, k, v = inputs(T, H, d, torch.bfloat16, seed=140 + decay)
    cu = cu_of(lengths)
    init = wl.state_init(len(lengths), H, d, seed=12, device=DEV, scale=0.2)
    init64 = init[:, [0, H - 1]].cpu().double().numpy()
    singles = [s for s, n in enumerate(lengths) if n == 1]
    s0 = init[torch.tensor(singles, device=DEV)].cpu().double().numpy()   # before an in-place update
    rates = wl.decay_rates(H, device=DEV) if decay else None
    st = init if in_place else None
    if decay:
        o, st = la.prefill_decay(q, k, v, rates, cu, B=B, init_state=init, return_state=True,
                                 state_out=st)
    else:
        o, st = la.prefill_with_state(q, k, v, cu, B=B, init_state=init, state_out=st)
    status_ok()
    cu_h = cu.cpu().numpy()
    heads = [0, H - 1]
    sel = lambda t: f64(t[:, heads])
    if decay:
        ref_o, ref_s = oracle.decay_recurrent(sel(q), sel(k), sel(v), rates.cpu().double().numpy()[heads], cu_h,
                                              init=init64, return_state=True)
    else:
        ref_o, ref_s = oracle.recurrent(sel(q), sel(k), sel(v), cu_h, init=init64, return_state=True)
    assert_close(sel(o), ref_o, 1e-2, "O of the sampled heads")
    assert_close(st[:, heads].cpu().double().numpy(), ref_s, 5e-3 if decay else 1e-5, "final states")
    # every head: the one-token rows against the decode step from their own state
    rows = cu_h[singles]
    q1, k1, v1 = (f64(x[rows]) for x in (q, k, v))
    if decay:
        ref1, _ = oracle.decay_decode_step(q1, k1, v1, s0, rates.cpu().double().numpy())
    else:
        ref1, _ = oracle.decode_step(q1, k1, v1, s0)
    assert_close(f64(o[rows]), ref1, 1e-2, "O of the one-token sequences, every head")


@pytest.mark.parametrize("B", [128, 256])
def test_prefill_with_state_repeated(B):
    """The state-output instance of the on-chip-state kernel over many blocks, repeated: every call
    matches the oracle (the last block's state MMAs wait for the prefix to have been read)."""
    lengths, H = [129, 255, 2048], 12
    T = sum(lengths)
    q, k, v = inputs(T, H, 128, torch.bfloat16, seed=T + H)
    cu = cu_of(lengths)
    init = wl.state_init(len(lengths), H, 128, seed=11, device=DEV)
    ref_o, ref_s = oracle.recurrent(f64(q), f64(k), f64(v), cu.cpu().numpy(), init=init.cpu().double().numpy(),
                                    return_state=True)
    for rep in range(12):
        o, st = la.prefill_with_state(q, k, v, cu, B=B, init_state=init)
        status_ok()
        assert_close(f64(o), ref_o, 1e-2, f"O, call {rep}")
        assert_close(st.cpu().double().numpy(), ref_s, 1e-5, f"final state, call {rep}")
