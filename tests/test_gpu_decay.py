"""GPU parity of the decay variant and of the feature map, through the C ABI,
against the fp64 oracle.

Decay (not on the pages; the Lightning Attention-2 form of the method):
S_t = lambda_h S_{t-1} + k_t^T v_t, o_t = q_t S_t. Tolerances as for the
method without decay: max|O - O_ref| <= 1e-2 max|O_ref| for bf16 inputs and
1e-4 for fp32; states 1e-4 max|S_ref| on the CUDA-core path (fp32 arithmetic
on both input types). On the tensor-core path (bf16, d = 128, B in {128, 256},
the on-chip-state kernel) the state MMAs read lambda^(n-1-c) v_c rounded to
bf16, one rounding of relative size <= 2^-9 per term, so its states are held
to 5e-3 max|S_ref|.
Feature map phi(x) = ELU(x) + alpha x: elementwise, within 2^-8 of |phi| for
bf16 outputs (one rounding to bf16) and 1e-6 for fp32.
"""
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
    return t.detach().float().cpu().double().numpy()


def assert_close(out, ref, tol, what=""):
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    r = float(np.abs(out - ref).max(initial=0.0) / max(np.abs(ref).max(initial=0.0), 1e-30))
    assert r <= tol, f"{what}: max|x - x_ref| / max|x_ref| = {r:.3e} > {tol:.0e}"


def status_ok():
    s = la.device_status()
    assert s == 0, f"device status {la.STATUS.get(s, s)}"


STATE_TOL = {"auto": 1e-4, "onchip": 5e-3}


@pytest.fixture(params=["auto", "onchip"])
def path(request):
    """auto: the path la_prefill_decay picks (CUDA cores below 64 work items); onchip: the
    on-chip-state tensor-core kernel forced (la_debug_set_path(1), bf16 d = 128 only)."""
    assert la.la_debug_set_path(1 if request.param == "onchip" else 0) == 0
    yield request.param
    la.la_debug_set_path(0)


RATES = {  # per-head rates: the edges 0 and 1, and rates in between
    2: [0.9, 0.999],
    4: [0.0, 0.5, 0.95, 1.0],
}


@pytest.mark.parametrize("dtype,d,B,lengths,H", [
    (torch.float32, 64, 64, [1024], 2),               # the small fp32 workload's shape
    (torch.bfloat16, 128, 256, [1000, 1, 0, 513], 4),
    (torch.bfloat16, 128, 128, [300, 129], 4),
    (torch.bfloat16, 32, 64, [77, 200], 2),
    (torch.float32, 16, 256, [600, 3], 4),
    (torch.float32, 128, 128, [257], 2),
], ids=lambda x: str(x).replace(" ", ""))
@pytest.mark.parametrize("with_init", [False, True], ids=["zero-S0", "S0"])
def test_prefill_decay(dtype, d, B, lengths, H, with_init, path):
    if path == "onchip" and not la.uses_tensor_cores(dtype, d, B):
        pytest.skip("no tensor-core path for this shape")
    T = sum(lengths)
    q, k, v = wl.qkv(T, H, d, dtype, seed=T + d, device=DEV)
    cu = wl.cu_seqlens(lengths, device=DEV)
    decay = torch.tensor(RATES[H], dtype=torch.float32, device=DEV)
    init = wl.state_init(len(lengths), H, d, seed=5, device=DEV) if with_init else None
    o, st = la.prefill_decay(q, k, v, decay, cu, B=B, init_state=init, return_state=True)
    status_ok()
    ref_o, ref_st = oracle.decay_recurrent(f64(q), f64(k), f64(v), decay.cpu().double().numpy(), cu.cpu().numpy(),
                                           init=None if init is None else init.cpu().double().numpy(),
                                           return_state=True)
    assert_close(f64(o), ref_o, TOL[dtype], "decay prefill O")
    assert_close(st.cpu().double().numpy(), ref_st, STATE_TOL[path], "decay prefill final state")
    # the state output is optional and changes nothing else, except that on the on-chip-state
    # kernel a one-token sequence with a state output is a decode step (fp32 on CUDA cores)
    # rather than a block of the tensor-core pipeline: equal up to rounding there
    o2 = la.prefill_decay(q, k, v, decay, cu, B=B, init_state=init)
    cu_h = cu.cpu().numpy()
    one = np.zeros(T, dtype=bool)
    for s_, n in enumerate(lengths):
        if n == 1:
            one[cu_h[s_]] = True
    multi = torch.from_numpy(~one).to(DEV)
    assert torch.equal(o2[multi], o[multi])
    if one.any():
        assert_close(f64(o2[~multi]), ref_o[one], TOL[dtype], "one-token rows without the state output")


@pytest.mark.parametrize("lengths,H,B", [
    ([1000, 1, 15, 16, 17, 0, 300], 8, 256),    # ragged tails of 1, 15, 16, 17 tokens, an empty sequence
    ([129, 255, 2048], 12, 128),
    ([4096], 64, 256),
])
def test_prefill_decay_onchip(lengths, H, B):
    """The tensor-core path with enough work items to be the automatic choice, the decay recipe's
    rates, S0 and the final state."""
    T = sum(lengths)
    q, k, v = wl.qkv(T, H, 128, torch.bfloat16, seed=T + H, device=DEV)
    cu = wl.cu_seqlens(lengths, device=DEV)
    decay = wl.decay_rates(H, device=DEV)
    init = wl.state_init(len(lengths), H, 128, seed=11, device=DEV)
    assert 2 * len(lengths) * H >= 64
    o, st = la.prefill_decay(q, k, v, decay, cu, B=B, init_state=init, return_state=True)
    status_ok()
    lam = decay.cpu().double().numpy()
    ref_o, ref_st = oracle.decay_recurrent(f64(q), f64(k), f64(v), lam, cu.cpu().numpy(),
                                           init=init.cpu().double().numpy(), return_state=True)
    assert_close(f64(o), ref_o, 1e-2, "O")
    assert_close(st.cpu().double().numpy(), ref_st, 5e-3, "final state")
    # without the state output (the other instance) the same O
    o2 = la.prefill_decay(q, k, v, decay, cu, B=B, init_state=init)
    status_ok()
    assert_close(f64(o2), ref_o, 1e-2, "O without the state output")


def test_prefill_decay_onchip_edge_rates():
    """Rates 0 and 1 on the tensor-core path: lambda = 1 is the method, lambda = 0 keeps the
    current token only."""
    T, H = 700, 32
    q, k, v = wl.qkv(T, H, 128, torch.bfloat16, seed=78, device=DEV)
    decay = torch.tensor([0.0, 1.0] * (H // 2), dtype=torch.float32, device=DEV)
    init = wl.state_init(1, H, 128, seed=12, device=DEV)
    o, st = la.prefill_decay(q, k, v, decay, B=256, init_state=init, return_state=True)
    status_ok()
    ref_o, ref_st = oracle.decay_recurrent(f64(q), f64(k), f64(v), decay.cpu().double().numpy(),
                                           init=init.cpu().double().numpy(), return_state=True)
    assert_close(f64(o), ref_o, 1e-2, "O")
    assert_close(st.cpu().double().numpy(), ref_st, 5e-3, "final state")
    ref_plain = la.prefill(q[:, 1::2].contiguous(), k[:, 1::2].contiguous(), v[:, 1::2].contiguous(), B=256,
                           init_state=init[:, 1::2].contiguous())
    assert_close(f64(o[:, 1::2]), f64(ref_plain), 1e-2, "lambda = 1 against la_prefill")


def test_prefill_decay_rate_one_is_the_method():
    T, H, d = 700, 2, 128
    q, k, v = wl.qkv(T, H, d, torch.bfloat16, seed=71, device=DEV)
    decay = torch.ones(H, dtype=torch.float32, device=DEV)
    o = la.prefill_decay(q, k, v, decay, B=256)
    status_ok()
    assert_close(f64(o), oracle.recurrent(f64(q), f64(k), f64(v)), 1e-2, "lambda = 1")


def test_prefill_decay_block_size_independence():
    T, H, d = 900, 4, 64
    q, k, v = wl.qkv(T, H, d, torch.float32, seed=72, device=DEV)
    decay = torch.tensor(RATES[4], dtype=torch.float32, device=DEV)
    outs = [la.prefill_decay(q, k, v, decay, B=B) for B in (64, 128, 256)]
    status_ok()
    for o in outs[1:]:
        assert_close(f64(o), f64(outs[0]), 1e-5, "B independence")


def test_prefill_decay_state_in_place():
    lengths, H, d = [400, 0, 90], 4, 128
    T = sum(lengths)
    q, k, v = wl.qkv(T, H, d, torch.bfloat16, seed=73, device=DEV)
    cu = wl.cu_seqlens(lengths, device=DEV)
    decay = torch.tensor(RATES[4], dtype=torch.float32, device=DEV)
    init = wl.state_init(3, H, d, seed=6, device=DEV)
    ref_st = oracle.decay_state(f64(k), f64(v), decay.cpu().double().numpy(), cu.cpu().numpy(),
                                init=init.cpu().double().numpy())
    ref_o = oracle.decay_recurrent(f64(q), f64(k), f64(v), decay.cpu().double().numpy(), cu.cpu().numpy(),
                                   init=init.cpu().double().numpy())
    o, st = la.prefill_decay(q, k, v, decay, cu, B=256, init_state=init, state_out=init)
    status_ok()
    assert st.data_ptr() == init.data_ptr()
    assert_close(f64(o), ref_o, 1e-2, "O with the state updated in place")
    assert_close(init.cpu().double().numpy(), ref_st, 1e-4, "state updated in place")


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
@pytest.mark.parametrize("with_init", [False, True], ids=["zero-S0", "S0"])
def test_state_decay(dtype, d, with_init):
    lengths, H = [5000, 0, 1, 2049], 4            # several 2048-token state blocks, empty and 1-token sequences
    T = sum(lengths)
    _, k, v = wl.qkv(T, H, d, dtype, seed=74, device=DEV)
    cu = wl.cu_seqlens(lengths, device=DEV)
    decay = torch.tensor(RATES[4], dtype=torch.float32, device=DEV)
    init = wl.state_init(4, H, d, seed=7, device=DEV) if with_init else None
    st = la.state_decay(k, v, decay, cu, init_state=init)
    status_ok()
    ref = oracle.decay_state(f64(k), f64(v), decay.cpu().double().numpy(), cu.cpu().numpy(),
                             init=None if init is None else init.cpu().double().numpy())
    assert_close(st.cpu().double().numpy(), ref, 1e-4, "decay state")


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 48)])
def test_decode_step_decay(dtype, d):
    batch, H, steps = 5, 4, 3
    st = wl.state_init(batch, H, d, seed=d, device=DEV)
    ref_state = st.cpu().double().numpy()
    decay = torch.tensor(RATES[4], dtype=torch.float32, device=DEV)
    q, k, v = wl.decode_inputs(batch, H, d, steps, dtype, seed=9 + d, device=DEV)
    for t in range(steps):
        o = la.decode_step_decay(q[t], k[t], v[t], st, decay)
        ref_o, ref_state = oracle.decay_decode_step(f64(q[t]), f64(k[t]), f64(v[t]), ref_state,
                                                    decay.cpu().double().numpy())
        assert_close(f64(o), ref_o, TOL[dtype], f"decay decode o step {t}")
    status_ok()
    assert_close(st.cpu().double().numpy(), ref_state, 1e-5, "decay decode state")


def test_decay_prefill_then_decode_continuity():
    """State of the first m tokens from the prefill, then decode steps: the rows of one prefill."""
    T, m, H, d = 600, 520, 4, 128
    q, k, v = wl.qkv(T, H, d, torch.bfloat16, seed=75, device=DEV)
    decay = wl.decay_rates(H, device=DEV)
    full = la.prefill_decay(q, k, v, decay, B=256)
    _, st = la.prefill_decay(q[:m], k[:m], v[:m], decay, B=256, return_state=True)
    rows = []
    for t in range(m, T):
        rows.append(la.decode_step_decay(q[t:t + 1], k[t:t + 1], v[t:t + 1], st, decay))
    status_ok()
    dec = torch.cat(rows)
    ref = oracle.decay_recurrent(f64(q), f64(k), f64(v), decay.cpu().double().numpy())[m:]
    assert_close(f64(dec), ref, 1e-2, "decode rows after a prefill")
    assert_close(f64(full[m:]), ref, 1e-2, "prefill rows")


@pytest.mark.parametrize("bad", [1.5, -0.25, float("nan")])
@pytest.mark.parametrize("dtype,d,H,B", [(torch.float32, 64, 4, 64), (torch.bfloat16, 128, 64, 256)],
                         ids=["cuda-cores", "tensor-cores"])
def test_bad_decay_rate_reported_on_device(bad, dtype, d, H, B):
    T = 300
    q, k, v = wl.qkv(T, H, d, dtype, seed=76, device=DEV)
    decay = torch.full((H,), 0.9, dtype=torch.float32, device=DEV)
    decay[1] = bad
    o = torch.full_like(q, 7.0)
    st_out = torch.full((1, H, d, d), 7.0, dtype=torch.float32, device=DEV)
    la.prefill_decay(q, k, v, decay, B=B, out=o, state_out=st_out)
    assert la.device_status() == 8                      # LA_ERR_BAD_DECAY
    assert torch.all(o == 7.0) and torch.all(st_out == 7.0), "a call with a bad rate writes nothing"
    la.prefill_decay(q, k, v, torch.full((H,), 0.9, dtype=torch.float32, device=DEV), B=B, out=o)
    status_ok()                                         # the next call with good rates runs
    assert not torch.any(o == 7.0)
    q, k, v = q[:, :4].contiguous(), k[:, :4].contiguous(), v[:, :4].contiguous()
    decay = decay[:4].contiguous()
    H = 4
    st = wl.state_init(2, H, d, seed=8, device=DEV)
    before = st.clone()
    la.decode_step_decay(q[:2], k[:2], v[:2], st, decay)
    assert la.device_status() == 8
    assert torch.equal(st[:, 1], before[:, 1]), "the state of a head with a bad rate is left as it was"
    assert la.device_status() == 0                      # the status word was cleared


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("n", [1, 7, 8, 9, 1000, 4099, 1 << 20])
@pytest.mark.parametrize("in_place", [False, True], ids=["out", "in-place"])
def test_feature_map(dtype, n, in_place):
    g = torch.Generator(device=DEV).manual_seed(n)
    x = (torch.randn(n, generator=g, device=DEV) * 4).to(dtype)
    if n >= 8:
        x[:6] = torch.tensor([0.0, -0.0, -100.0, 100.0, -1e-30, 1e-30]).to(dtype)
    ref = oracle.feature_map(f64(x), 0.3)
    y = la.feature_map(x.clone() if in_place else x, 0.3, out=None)
    if in_place:
        xi = x.clone()
        la.feature_map(xi, 0.3, out=xi)
        assert torch.equal(xi, y)
    status_ok()
    tol = 2.0 ** -8 if dtype == torch.bfloat16 else 1e-6
    err = np.abs(f64(y) - ref)
    assert np.all(err <= tol * np.abs(ref) + 1e-38), f"phi: worst relative error {np.max(err / (np.abs(ref) + 1e-38)):.3e}"


def test_feature_map_then_prefill_decay():
    """The pre-pass composes with a prefill: phi on q and k, then the decay prefill."""
    T, H, d = 333, 2, 64
    q, k, v = wl.qkv(T, H, d, torch.float32, seed=77, device=DEV)
    decay = torch.tensor(RATES[2], dtype=torch.float32, device=DEV)
    o = la.prefill_decay(la.feature_map(q), la.feature_map(k), v, decay, B=64)
    status_ok()
    ref = oracle.decay_recurrent(oracle.feature_map(f64(q)), oracle.feature_map(f64(k)), f64(v),
                                 decay.cpu().double().numpy())
    assert_close(f64(o), ref, 1e-4, "phi then decay prefill")


def test_decay_full_size_sampled_heads():
    """The bf16 32k workload (T = 32768, H = 64, d = 128, B = 256) with the decay recipe: the
    heads with the fastest and the slowest decay, in full length, against the oracle."""
    T, H, d = 32768, 64, 128
    q, k, v = wl.qkv(T, H, d, torch.bfloat16, seed=2, device=DEV)
    decay = wl.decay_rates(H, device=DEV)
    o, st = la.prefill_decay(q, k, v, decay, B=256, return_state=True)
    status_ok()
    lam = decay.cpu().double().numpy()
    for h in (0, H - 1):
        ref_o, ref_st = oracle.decay_recurrent(f64(q[:, h:h + 1]), f64(k[:, h:h + 1]), f64(v[:, h:h + 1]),
                                               lam[h:h + 1], return_state=True)
        assert_close(f64(o[:, h:h + 1]), ref_o, 1e-2, f"head {h} (lambda {lam[h]:.4f})")
        # tensor-core path (64 heads x 2 halves >= 64 work items): the state bound of that path
        assert_close(st[:, h:h + 1].cpu().double().numpy(), ref_st, 5e-3, f"final state of head {h}")


def test_decay_withheld_prefix_ends_in_timeout_not_hang():
    """The decay instance of the on-chip-state kernel under the same fault hook as the plain one
    (work item 3 never hands over its second block's prefix): every bounded wait of the instance,
    the weighted-V ring's included, gives up, the launch ends with LA_ERR_TIMEOUT and the next
    call is right."""
    import time
    T, H, B = 4096, 4, 256
    q, k, v = wl.qkv(T, H, 128, torch.bfloat16, seed=5152, device=DEV)
    decay = torch.tensor(RATES[4], dtype=torch.float32, device=DEV)
    assert la.la_debug_set_fault(3, 200_000_000) == 0
    assert la.la_debug_set_path(1) == 0
    try:
        t0 = time.time()
        la.prefill_decay(q, k, v, decay, B=B)
        st = la.device_status()
        elapsed = time.time() - t0
    finally:
        la.la_debug_set_fault(-1, 0)
    try:
        assert st == 6, f"expected LA_ERR_TIMEOUT, got {la.STATUS.get(st, st)}"
        assert elapsed < 30, f"timed-out launch took {elapsed:.1f}s"
        o = la.prefill_decay(q, k, v, decay, B=B)
        status_ok()
    finally:
        la.la_debug_set_path(0)
    ref = oracle.decay_recurrent(f64(q), f64(k), f64(v), decay.cpu().double().numpy())
    assert_close(f64(o), ref, 1e-2, "run after a timeout")


@pytest.mark.parametrize("B", [128, 256])
def test_prefill_decay_onchip_state_repeated(B):
    """Many blocks per work item, the final state on: repeated calls must all match the oracle.
    Guards the hand-off between the copy-out group's read (and decay rescale) of the last block's
    prefix and that block's state MMAs, which once raced in about one call in fifteen."""
    lengths, H = [129, 255, 2048], 12
    T = sum(lengths)
    q, k, v = wl.qkv(T, H, 128, torch.bfloat16, seed=T + H, device=DEV)
    cu = wl.cu_seqlens(lengths, device=DEV)
    decay = wl.decay_rates(H, device=DEV)
    init = wl.state_init(len(lengths), H, 128, seed=11, device=DEV)
    ref_o, ref_st = oracle.decay_recurrent(f64(q), f64(k), f64(v), decay.cpu().double().numpy(), cu.cpu().numpy(),
                                           init=init.cpu().double().numpy(), return_state=True)
    for rep in range(12):
        o, st = la.prefill_decay(q, k, v, decay, cu, B=B, init_state=init, return_state=True)
        status_ok()
        assert_close(f64(o), ref_o, 1e-2, f"O, call {rep}")
        assert_close(st.cpu().double().numpy(), ref_st, 5e-3, f"final state, call {rep}")


@pytest.mark.parametrize("W,B,H", [(2, 256, 32), (3, 128, 4), (4, 256, 4)])
def test_lasp_decay_segments_on_one_gpu(W, B, H):
    """LASP+ with decay composed from the library calls, the ranks emulated one after another on
    one GPU (the all-gathers are stacks): segment states (la_state_decay), the decayed exclusive
    prefix (la_state_exclusive_prefix_decay) and each segment's decay prefill from it equal the
    whole sequences' output and final state. H = 32 puts the segment prefills on the tensor-core
    path, H = 4 on CUDA cores."""
    lengths, d = [1500, 777], 128
    T = sum(lengths)
    q, k, v = wl.qkv(T, H, d, torch.bfloat16, seed=80 + W, device=DEV)
    init = wl.state_init(len(lengths), H, d, seed=9, device=DEV)
    decay = wl.decay_rates(H, device=DEV)
    rng = np.random.default_rng(W)
    cuts = [[0, *np.sort(rng.choice(np.arange(1, L), size=W - 1, replace=False)).tolist(), L] for L in lengths]
    starts = np.cumsum([0] + lengths[:-1])
    rows = [np.concatenate([np.arange(s0 + c[r], s0 + c[r + 1]) for s0, c in zip(starts, cuts)]) for r in range(W)]
    segs = []
    for r in range(W):
        idx = torch.from_numpy(rows[r]).to(DEV)
        cu = wl.cu_seqlens([c[r + 1] - c[r] for c in cuts], device=DEV)
        segs.append((q[idx].contiguous(), k[idx].contiguous(), v[idx].contiguous(), cu))
    gathered = torch.stack([la.state_decay(kr, vr, decay, cu) for _, kr, vr, cu in segs])
    seg_lens = torch.tensor([[c[r + 1] - c[r] for c in cuts] for r in range(W)], dtype=torch.int32, device=DEV)
    o = torch.empty_like(q)
    for r, (qr, kr, vr, cu) in enumerate(segs):
        start = la.state_exclusive_prefix_decay(gathered, seg_lens, r, decay, init)
        o[torch.from_numpy(rows[r]).to(DEV)] = la.prefill_decay(qr, kr, vr, decay, cu, B=B, init_state=start)
    final = la.state_exclusive_prefix_decay(gathered, seg_lens, W, decay, init)
    status_ok()
    cu_all = wl.cu_seqlens(lengths).numpy()
    ref, ref_state = oracle.decay_recurrent(f64(q), f64(k), f64(v), decay.cpu().double().numpy(), cu_all,
                                            init=init.cpu().double().numpy(), return_state=True)
    assert_close(f64(o), ref, 1e-2, "LASP+ output with decay")
    assert_close(final.cpu().double().numpy(), ref_state, 1e-4, "LASP+ final state with decay")


def test_state_exclusive_prefix_decay_arguments():
    """Bad rates and negative lengths are reported on the device and leave the state unwritten."""
    W, nseq, H, d = 2, 1, 2, 16
    gathered = torch.randn((W, nseq, H, d, d), device=DEV)
    seg_lens = torch.tensor([[3], [-1]], dtype=torch.int32, device=DEV)
    decay = torch.tensor([0.5, 0.9], device=DEV)
    out = torch.full((nseq, H, d, d), 7.0, device=DEV)
    la.state_exclusive_prefix_decay(gathered, seg_lens, 2, decay, out=out)
    assert la.device_status() == 7                      # LA_ERR_BAD_SEQLENS
    assert torch.all(out == 7.0)
    la.state_exclusive_prefix_decay(gathered, seg_lens, 1, torch.tensor([0.5, 2.0], device=DEV), out=out)
    assert la.device_status() == 8                      # LA_ERR_BAD_DECAY: head 1 unwritten
    assert torch.all(out[:, 1] == 7.0)
    assert torch.allclose(out[:, 0], gathered[0, :, 0])


@pytest.mark.parametrize("dtype,d,B,H,lengths", [
    (torch.bfloat16, 128, 256, 32, [700, 0, 300]),      # tensor-core decay prefills
    (torch.bfloat16, 128, 128, 4, [500, 1]),             # CUDA-core decay prefills (few work items)
    (torch.float32, 64, 64, 2, [333, 129]),
], ids=["bf16-onchip", "bf16-cudacores", "fp32"])
@pytest.mark.parametrize("with_init", [False, True], ids=["zero-S0", "S0"])
def test_prefill_backward_decay(dtype, d, B, H, lengths, with_init):
    """Gradients of the decay variant against the oracle's (dq, dk, dv within the O bound of the
    dtype, dS0 from a CUDA-core state pass within 1e-4)."""
    T = sum(lengths)
    q, k, v = wl.qkv(T, H, d, dtype, seed=90 + d, device=DEV)
    do = wl.normal_scaled((T, H, d), d, dtype, 91, device=DEV)
    cu = wl.cu_seqlens(lengths, device=DEV)
    decay = wl.decay_rates(H, device=DEV)
    init = wl.state_init(len(lengths), H, d, seed=12, device=DEV) if with_init else None
    dq, dk, dv, dinit = la.prefill_backward_decay(q, k, v, do, decay, cu, B=B, init_state=init, need_init_grad=True)
    status_ok()
    ref = oracle.decay_backward(f64(q), f64(k), f64(v), f64(do), decay.cpu().double().numpy(), cu.cpu().numpy(),
                                init=None if init is None else init.cpu().double().numpy())
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref[:3]):
        assert_close(f64(got), want, TOL[dtype], name)
    assert_close(dinit.cpu().double().numpy(), ref[3], 1e-4, "dS0")


def _bits_equal_bf16(o, ref):
    ref_b = torch.from_numpy(np.ascontiguousarray(ref)).to(torch.bfloat16)
    return int((o.cpu().view(torch.int16) != ref_b.view(torch.int16)).sum().item())


@pytest.mark.parametrize("B,T", [(256, 600), (128, 300)])
def test_prefill_decay_tc_integer_exact_rate_one(B, T):
    """Rate 1 on every head through the decay instance of the on-chip-state tensor-core kernel
    (forced), {-1,0,1} inputs over several blocks: every power of the rate is exactly 1, so
    the decay masks, weighted V and scaled Q rows change nothing, and the output must equal
    the method without decay bit for bit (scores, P, prefixes and O are integers that bf16
    and fp32 hold exactly)."""
    H, d = 2, 128
    q, k, v = wl.integer_qkv(T, H, d, torch.bfloat16, seed=B + T + 1, device=DEV)
    for n in range(B, T, B):
        assert np.abs(oracle.state(f64(k)[:n], f64(v)[:n])).max() <= 256, "precondition: bf16-exact prefix"
    force = la.la_debug_set_path(1)
    assert force == 0
    try:
        o = la.prefill_decay(q, k, v, torch.ones(H, dtype=torch.float32, device=DEV), B=B)
    finally:
        la.la_debug_set_path(0)
    status_ok()
    mism = _bits_equal_bf16(o, oracle.recurrent(f64(q), f64(k), f64(v)))
    assert mism == 0, f"{mism} outputs differ from the exact result"


@pytest.mark.parametrize("T", [8, 5])
def test_prefill_decay_tc_integer_exact_dyadic(T):
    """Dyadic rates 1/2 and 1/4 on the decay instance of the tensor-core kernel (forced), one
    short block with {-1,0,1} inputs and an integer carried-in state: every power of the rate
    is a power of two, every product (decay mask times score, rate times query row, weighted
    value) is exact in bf16, and every sum spans fewer than 24 bits, so the output must equal
    the exact result rounded to bf16 bit for bit. (Over longer sequences the powers 2^-n span
    more bits than fp32 holds, so exactness stops there; those lengths are held to the
    tolerance by the tests above.)"""
    H, d, B = 2, 128, 256
    rates = torch.tensor([0.5, 0.25], dtype=torch.float32, device=DEV)
    q, k, v = wl.integer_qkv(T, H, d, torch.bfloat16, seed=700 + T, device=DEV)
    g = torch.Generator().manual_seed(800 + T)
    s0 = (torch.randint(0, 3, (1, H, d, d), generator=g) - 1).float().to(DEV)
    assert la.la_debug_set_path(1) == 0
    try:
        o = la.prefill_decay(q, k, v, rates, B=B, init_state=s0)
    finally:
        la.la_debug_set_path(0)
    status_ok()
    ref = oracle.decay_recurrent(f64(q), f64(k), f64(v), rates.cpu().double().numpy(),
                                 init=s0.cpu().double().numpy())
    mism = _bits_equal_bf16(o, ref)
    assert mism == 0, f"{mism} of {ref.size} outputs differ from the exact result"
