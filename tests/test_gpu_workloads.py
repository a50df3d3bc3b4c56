"""GPU parity at the full sizes of the four GPU workloads, on sampled outputs.

Each test builds the workload exactly as the benchmark does (same generators,
seeds, shapes, block size and C-ABI call with a caller-owned workspace on the
current stream), runs the whole problem on the GPU, and checks sampled
(sequence, head) pairs in full length against the fp64 oracle's recurrent form
(the oracle can afford a few whole heads even at a million tokens):

  bf16 prefill T = 32768, H = 64, d = 128, B = 256          heads 0, 21, 42, 63
  bf16 prefill T = 1048576, H = 64, d = 128, B = 256        heads 0, 63
  bf16 varlen, 16 sequences U[1024, 65536], H = 64, B = 256  heads 5, 58, every sequence
  the same varlen workload with a decay rate per head          heads 0, 63, every sequence, final states
  decode, 256 sequences x 64 heads, states from a 4096-token prefill, 1000 steps,
                                                             8 (sequence, head) pairs, every step

Bound: max|O - O_ref| <= 1e-2 * max|O_ref| over the sampled outputs (bf16
inputs, fp32 accumulation), and the same bound per decode step; the decode
states, kept in fp32, within 1e-4 of their largest magnitude.

Per block: |O_t| grows like sqrt(t)/d, so the global bound is larger than the
whole first block's outputs at these lengths and would not see a wrong prefix
there. The prefill checks therefore also hold each of the first FIRST_BLOCKS
blocks (of B tokens) of every sampled (sequence, head) to BLOCK_TOL relative
to that block's own max|O_ref|, and report the worst block of the whole
sequence. BLOCK_TOL comes from the arithmetic: P, the bf16 copy of the prefix
and the stored O are each rounded to bf16 (relative 2^-9 of the values they
touch), so with the block's largest output as the scale the error stays near
3 * 2^-9 = 6e-3; a missed, doubled or shifted block contributes an error of
the order of the block's outputs themselves.
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
TOL = 1e-2
FIRST_BLOCKS = 4
BLOCK_TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _library():
    from causal_linear_attention_02_b200 import build
    build.build()
    la.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(DEV)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _heads_f64(x, heads):
    """[T, H, d] device tensor -> fp64 numpy [T, len(heads), d] of the chosen heads."""
    return x[:, heads, :].float().cpu().double().numpy()


def _rel(out, ref):
    return float(np.abs(out - ref).max() / max(np.abs(ref).max(), 1e-30))


def _prefill_like_bench(w, cu=None):
    T, H, d, B = w.total_tokens, w.heads, w.d, w.B
    q, k, v = wl.qkv(T, H, d, torch.bfloat16, w.seed, device=DEV)
    o = torch.full_like(q, float("nan"))
    nseq = len(w.seq_lens)
    ws_bytes = la.la_prefill_workspace_size(T, nseq, H, d, B, la.LA_BF16)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
    s = la.la_prefill(_p(q), _p(k), _p(v), _p(o), _p(cu), nseq, T, H, d, B, la.LA_BF16, None, _p(ws), ws_bytes,
                      stream)
    assert s == 0, la.STATUS.get(s, s)
    torch.cuda.synchronize(DEV)
    assert la.device_status() == 0
    del ws
    return q, k, v, o


def _check_blocks(out, ref, cu_host, B, what=""):
    """Per-block error relative to the block's own max|O_ref|, for every sequence and sampled
    head: the first FIRST_BLOCKS blocks gated at BLOCK_TOL; returns the worst of all blocks."""
    T = out.shape[0]
    cu = [0, T] if cu_host is None else [int(x) for x in cu_host]
    worst = 0.0
    for s in range(len(cu) - 1):
        a, e = cu[s], cu[s + 1]
        for b in range((e - a + B - 1) // B):
            rows = slice(a + b * B, min(a + (b + 1) * B, e))
            err = np.abs(out[rows] - ref[rows]).max(axis=(0, 2))       # per sampled head
            scale = np.maximum(np.abs(ref[rows]).max(axis=(0, 2)), 1e-30)
            r = float((err / scale).max())
            worst = max(worst, r)
            if b < FIRST_BLOCKS:
                assert r <= BLOCK_TOL, f"{what}: sequence {s} block {b}: {r:.3e} of the block's max > {BLOCK_TOL:.0e}"
    return worst


def _check_heads(q, k, v, o, heads, cu_host=None, what="", B=256):
    qs, ks, vs = (_heads_f64(x, heads) for x in (q, k, v))
    ref = oracle.recurrent(qs, ks, vs, cu_seqlens=cu_host)
    out = _heads_f64(o, heads)
    assert np.isfinite(out).all(), f"{what}: non-finite outputs"
    r = _rel(out, ref)
    assert r <= TOL, f"{what}: max|O-O_ref|/max|O_ref| = {r:.3e} > {TOL:.0e}"
    worst = _check_blocks(out, ref, cu_host, B, what)
    print(f"{what}: global {r:.2e}, worst block {worst:.2e}")
    return r


def test_bf16_32k_sampled_heads():
    w = wl.BF16_32K
    q, k, v, o = _prefill_like_bench(w)
    _check_heads(q, k, v, o, [0, 21, 42, 63], what=w.name)


def test_bf16_1m_sampled_heads():
    w = wl.BF16_1M
    q, k, v, o = _prefill_like_bench(w)
    _check_heads(q, k, v, o, [0, 63], what=w.name)
    del q, k, v, o
    torch.cuda.empty_cache()


def test_bf16_varlen_sampled_heads():
    w = wl.BF16_VARLEN
    cu = wl.cu_seqlens(w.seq_lens, device=DEV)
    q, k, v, o = _prefill_like_bench(w, cu)
    _check_heads(q, k, v, o, [5, 58], cu_host=np.asarray(cu.cpu().numpy(), dtype=np.int32), what=w.name)


def test_bf16_varlen_decay_sampled_heads():
    """The varlen workload through la_prefill_decay with the decay recipe's per-head rates, and the
    final state of every sequence: heads 0 and 63 (fastest and slowest decay) against the oracle's
    decay recurrence. O within 1e-2, states within the tensor-core path's 5e-3 (the state MMAs read
    bf16-rounded weighted V)."""
    w = wl.BF16_VARLEN
    T, H, d, B = w.total_tokens, w.heads, w.d, w.B
    nseq = len(w.seq_lens)
    cu = wl.cu_seqlens(w.seq_lens, device=DEV)
    q, k, v = wl.qkv(T, H, d, torch.bfloat16, w.seed, device=DEV)
    decay = wl.decay_rates(H, device=DEV)
    o = torch.full_like(q, float("nan"))
    st = torch.full((nseq, H, d, d), float("nan"), dtype=torch.float32, device=DEV)
    ws_bytes = la.la_prefill_decay_workspace_size(T, nseq, H, d, B, la.LA_BF16)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
    s = la.la_prefill_decay(_p(q), _p(k), _p(v), _p(o), _p(cu), nseq, T, H, d, B, la.LA_BF16, None, _p(decay),
                            _p(st), _p(ws), ws_bytes, stream)
    assert s == 0, la.STATUS.get(s, s)
    torch.cuda.synchronize(DEV)
    assert la.device_status() == 0
    del ws
    heads = [0, 63]
    cu_host = np.asarray(cu.cpu().numpy(), dtype=np.int32)
    ref_o, ref_st = oracle.decay_recurrent(*(_heads_f64(x, heads) for x in (q, k, v)),
                                           decay.cpu().double().numpy()[heads], cu_seqlens=cu_host,
                                           return_state=True)
    out = _heads_f64(o, heads)
    assert np.isfinite(out).all()
    r = _rel(out, ref_o)
    assert r <= TOL, f"decay varlen O: {r:.3e}"
    worst = _check_blocks(out, ref_o, cu_host, B, "decay varlen O")
    print(f"decay varlen: global {r:.2e}, worst block {worst:.2e}")
    got_st = st[:, heads].cpu().double().numpy()
    r = _rel(got_st, ref_st)
    assert r <= 5e-3, f"decay varlen final states: {r:.3e}"


def test_decode_workload_sampled_pairs():
    w = wl.DECODE
    Bt, H, d, steps, L = w.decode_batch, w.heads, w.d, w.decode_steps, w.prefill_len
    k0 = wl.normal_scaled((Bt * L, H, d), d, torch.bfloat16, w.seed * 1000 + 1, device=DEV)
    v0 = wl.normal_scaled((Bt * L, H, d), d, torch.bfloat16, w.seed * 1000 + 2, device=DEV)
    cu = wl.cu_seqlens([L] * Bt, device=DEV)
    state = la.state_from_prefill(k0, v0, cu)
    torch.cuda.synchronize(DEV)
    assert la.device_status() == 0
    pairs = [(0, 0), (1, 63), (77, 5), (128, 31), (200, 40), (254, 1), (255, 62), (31, 17)]
    seqs = [p[0] for p in pairs]
    hs = [p[1] for p in pairs]
    # oracle initial states of the sampled pairs from their own 4096-token prefixes
    idx_s, idx_h = torch.tensor(seqs, device=DEV), torch.tensor(hs, device=DEV)
    s_ref = np.empty((len(pairs), 1, d, d))
    for n, (sq, h) in enumerate(pairs):
        kk = k0[sq * L:(sq + 1) * L, h:h + 1, :].float().cpu().double().numpy()
        vv = v0[sq * L:(sq + 1) * L, h:h + 1, :].float().cpu().double().numpy()
        s_ref[n] = oracle.state(kk, vv)[0]
    del k0, v0
    torch.cuda.empty_cache()
    s0 = state[idx_s, idx_h].double().cpu().numpy()[:, None]
    r = _rel(s0, s_ref)
    assert r <= 1e-4, f"initial states: {r:.3e}"
    qs, ks, vs = wl.decode_inputs(Bt, H, d, steps, torch.bfloat16, w.seed, device=DEV)
    o = torch.empty((Bt, H, d), dtype=torch.bfloat16, device=DEV)
    o_hist = torch.empty((steps, len(pairs), d), dtype=torch.bfloat16, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
    for i in range(steps):
        s = la.la_decode_step(_p(qs[i]), _p(ks[i]), _p(vs[i]), _p(state), _p(o), Bt, H, d, la.LA_BF16, stream)
        assert s == 0, la.STATUS.get(s, s)
        o_hist[i] = o[idx_s, idx_h]
    torch.cuda.synchronize(DEV)
    assert la.device_status() == 0
    sel = lambda x: x[:, idx_s, idx_h].float().cpu().double().numpy()[:, :, None]   # [steps, n, 1, d]
    qn, kn, vn = sel(qs), sel(ks), sel(vs)
    out = o_hist.float().cpu().double().numpy()
    worst = 0.0
    for i in range(steps):
        o_ref, s_ref = oracle.decode_step(qn[i], kn[i], vn[i], s_ref)
        r = _rel(out[i], o_ref[:, 0])
        worst = max(worst, r)
        assert r <= TOL, f"decode step {i}: {r:.3e} > {TOL:.0e}"
    r = _rel(state[idx_s, idx_h].double().cpu().numpy()[:, None], s_ref)
    assert r <= 1e-4, f"states after {steps} steps: {r:.3e}"
