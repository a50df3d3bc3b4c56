"""Pins for the fp64 oracle: facts fixed by the method and by mathematics.

Each ``pin_*`` takes an implementation object exposing the oracle's interface
(``quadratic``, ``recurrent``, ``blocked``, ``state``, ``decode_step``) and
raises AssertionError when that implementation disagrees with a fact that
does not come from the implementation itself:

* a hand-worked example (``tests/golden/hand_example.json``);
* closed forms on special inputs (one token; one-hot queries and keys, whose
  result is a count-and-select; all-ones scores, whose result is a cumulative
  sum);
* exact rational brute force on tiny integer inputs;
* invariants: three associations of the sum agree for every block size B,
  linearity in Q, K and V, causality, per-sequence independence of packed
  sequences, additivity of the state, prefill/decode continuity and resume
  from a carried-in state.

The method is causal linear attention as described on the page "MiniMax-01
Lightning Attention", section "Lightning Attention 设计": left product inside a
block, right product across blocks through a d x d KV state, and an O(d^2)
recurrent update at inference.
"""
from __future__ import annotations

import json
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_example.json")


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    scale = max(np.abs(b).max(initial=0.0), 1e-300)
    return float(np.abs(a - b).max(initial=0.0) / scale)


def _close(a, b, tol, what):
    r = _rel(a, b)
    assert r <= tol, f"{what}: relative max error {r:.3e} > {tol:.1e}"


def _rng(seed):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------- golden
def pin_golden(impl):
    g = json.load(open(GOLDEN))
    q, k, v = (np.array(g[x], dtype=np.float64) for x in ("q", "k", "v"))
    o = np.array(g["o"], dtype=np.float64)
    assert np.array_equal(impl.quadratic(q, k, v), o), "quadratic != hand example"
    assert np.array_equal(impl.recurrent(q, k, v), o), "recurrent != hand example"
    for B in (1, 2, 3):
        assert np.array_equal(impl.blocked(q, k, v, B), o), f"blocked(B={B}) != hand example"
    st = np.array(g["state"], dtype=np.float64)
    assert np.array_equal(impl.state(k, v), st), "state != hand example"
    dq, dk, dv = (np.array(g["decode"][x], dtype=np.float64) for x in ("q", "k", "v"))
    do, ds = impl.decode_step(dq, dk, dv, st)
    assert np.array_equal(do, np.array(g["decode"]["o"], dtype=np.float64)), "decode o != hand example"
    assert np.array_equal(ds, np.array(g["decode"]["state"], dtype=np.float64)), "decode state != hand example"


# --------------------------------------------------------------------------- closed forms
def pin_single_token(impl):
    """n = 1: O_1 = (q_1 . k_1) v_1; with a carried-in state add q_1 S0."""
    r = _rng(11)
    H, d = 3, 5
    q, k, v = (r.integers(-4, 5, size=(1, H, d)).astype(np.float64) for _ in range(3))
    want = np.zeros((1, H, d))
    for h in range(H):
        score = sum(q[0, h, i] * k[0, h, i] for i in range(d))
        want[0, h] = score * v[0, h]
    for f in (impl.quadratic, impl.recurrent):
        assert np.array_equal(f(q, k, v), want), "single token closed form"
    assert np.array_equal(impl.blocked(q, k, v, 4), want), "single token closed form (blocked)"
    S0 = r.integers(-3, 4, size=(1, H, d, d)).astype(np.float64)
    want0 = want.copy()
    for h in range(H):
        for j in range(d):
            want0[0, h, j] += sum(q[0, h, i] * S0[0, h, i, j] for i in range(d))
    for f in (impl.quadratic, impl.recurrent):
        assert np.array_equal(f(q, k, v, init=S0), want0), "single token with init state"
    assert np.array_equal(impl.blocked(q, k, v, 2, init=S0), want0), "single token with init (blocked)"
    # the state of one token is the outer product k^T v (row index from k)
    st = impl.state(k, v)
    for h in range(H):
        for i in range(d):
            for j in range(d):
                assert st[0, h, i, j] == k[0, h, i] * v[0, h, j], "state orientation k_i v_j"


def pin_onehot(impl):
    """q_t = e_{a_t}, k_s = e_{c_s}: O_t = sum of v_s over s <= t with c_s == a_t."""
    r = _rng(12)
    T, H, d = 41, 2, 6
    a = r.integers(0, d, size=(T, H))
    c = r.integers(0, d, size=(T, H))
    q = np.zeros((T, H, d)); k = np.zeros((T, H, d))
    for t in range(T):
        for h in range(H):
            q[t, h, a[t, h]] = 1.0
            k[t, h, c[t, h]] = 1.0
    v = r.integers(-9, 10, size=(T, H, d)).astype(np.float64)
    cu = [0, 17, 17, 41]
    want = np.zeros((T, H, d))
    for si in range(len(cu) - 1):
        for h in range(H):
            for t in range(cu[si], cu[si + 1]):
                for s in range(cu[si], t + 1):
                    if c[s, h] == a[t, h]:
                        want[t, h] += v[s, h]
    assert np.array_equal(impl.quadratic(q, k, v, cu), want), "one-hot count (quadratic)"
    assert np.array_equal(impl.recurrent(q, k, v, cu), want), "one-hot count (recurrent)"
    for B in (1, 3, 16, 64):
        assert np.array_equal(impl.blocked(q, k, v, B, cu), want), f"one-hot count (blocked B={B})"


def pin_cumsum(impl):
    """All scores equal to one (q = k = e_0): O is the per-sequence cumulative sum of V."""
    r = _rng(13)
    T, H, d = 30, 2, 4
    q = np.zeros((T, H, d)); q[:, :, 0] = 1.0
    k = q.copy()
    v = r.integers(-5, 6, size=(T, H, d)).astype(np.float64)
    cu = [0, 7, 30]
    want = np.concatenate([np.cumsum(v[cu[i]:cu[i + 1]], axis=0) for i in range(2)])
    for f in (impl.quadratic, impl.recurrent):
        assert np.array_equal(f(q, k, v, cu), want), "cumsum closed form"
    assert np.array_equal(impl.blocked(q, k, v, 4, cu), want), "cumsum closed form (blocked)"


def pin_bruteforce_exact(impl):
    """Exact rational arithmetic over every (t, s) pair on tiny integer inputs."""
    r = _rng(14)
    T, H, d = 7, 2, 3
    q, k, v = (r.integers(-3, 4, size=(T, H, d)) for _ in range(3))
    cu = [0, 3, 7]
    want = np.zeros((T, H, d))
    for si in range(2):
        for h in range(H):
            for t in range(cu[si], cu[si + 1]):
                acc = [Fraction(0)] * d
                for s in range(cu[si], t + 1):
                    score = Fraction(0)
                    for i in range(d):
                        score += Fraction(int(q[t, h, i])) * Fraction(int(k[s, h, i]))
                    for j in range(d):
                        acc[j] += score * Fraction(int(v[s, h, j]))
                want[t, h] = [float(x) for x in acc]
    qf, kf, vf = (x.astype(np.float64) for x in (q, k, v))
    assert np.array_equal(impl.quadratic(qf, kf, vf, cu), want), "brute force (quadratic)"
    assert np.array_equal(impl.recurrent(qf, kf, vf, cu), want), "brute force (recurrent)"
    for B in (1, 2, 3, 5, 8):
        assert np.array_equal(impl.blocked(qf, kf, vf, B, cu), want), f"brute force (blocked B={B})"


# --------------------------------------------------------------------------- invariants
def pin_forms_agree(impl):
    """quadratic == recurrent == blocked(B) for every B in 1..n (fp64, 1e-10 relative)."""
    r = _rng(15)
    T, H, d = 67, 2, 5
    q, k, v = (r.standard_normal((T, H, d)) for _ in range(3))
    ref = impl.quadratic(q, k, v)
    _close(impl.recurrent(q, k, v), ref, 1e-10, "recurrent vs quadratic")
    for B in range(1, T + 1):
        _close(impl.blocked(q, k, v, B), ref, 1e-10, f"blocked(B={B}) vs quadratic")
    # long sequence: recurrent vs quadratic
    T2 = 1500
    q, k, v = (r.standard_normal((T2, 1, 8)) / np.sqrt(8) for _ in range(3))
    _close(impl.recurrent(q, k, v), impl.quadratic(q, k, v), 1e-10, "recurrent vs quadratic (n=1500)")
    _close(impl.blocked(q, k, v, 256), impl.quadratic(q, k, v), 1e-10, "blocked(256) vs quadratic (n=1500)")


def pin_linearity(impl):
    """O is linear in each of Q, K and V separately."""
    r = _rng(16)
    T, H, d = 23, 2, 4
    q, k, v, x = (r.standard_normal((T, H, d)) for _ in range(4))
    alpha = 1.75
    o = impl.recurrent(q, k, v)
    _close(impl.recurrent(q, k, alpha * v + x), alpha * o + impl.recurrent(q, k, x), 1e-10, "linear in V")
    _close(impl.recurrent(alpha * q + x, k, v), alpha * o + impl.recurrent(x, k, v), 1e-10, "linear in Q")
    _close(impl.blocked(q, alpha * k + x, v, 5), alpha * o + impl.blocked(q, x, v, 5), 1e-10, "linear in K")


def pin_causality(impl):
    """Changing tokens after t0 leaves O_t (t <= t0) untouched; changing token t0 moves O_t0."""
    r = _rng(17)
    T, H, d, t0 = 20, 2, 4, 9
    q, k, v = (r.standard_normal((T, H, d)) for _ in range(3))
    base = {n: f(q, k, v) for n, f in (("q", impl.quadratic), ("r", impl.recurrent))}
    base["b"] = impl.blocked(q, k, v, 4)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[t0 + 1:] += 3.0; k2[t0 + 1:] -= 2.0; v2[t0 + 1:] *= -5.0
    for n, f in (("q", impl.quadratic), ("r", impl.recurrent)):
        assert np.array_equal(f(q2, k2, v2)[: t0 + 1], base[n][: t0 + 1]), "future tokens leak into the past"
    assert np.array_equal(impl.blocked(q2, k2, v2, 4)[: t0 + 1], base["b"][: t0 + 1]), "future leak (blocked)"
    # the diagonal is part of the sum: token t0's own key/value moves O_t0
    k3, v3 = k.copy(), v.copy()
    k3[t0] += 1.0; v3[t0] += 1.0
    for f in (impl.quadratic, impl.recurrent):
        assert not np.allclose(f(q, k3, v3)[t0], base["r"][t0]), "diagonal term missing"
    # and an earlier token moves every later output of its sequence
    v4 = v.copy(); v4[0] += 1.0
    assert not np.allclose(impl.recurrent(q, k, v4)[T - 1], base["r"][T - 1]), "earliest token ignored"


def pin_varlen(impl):
    """Packed sequences are independent: packing equals running each sequence alone."""
    r = _rng(18)
    lens = [5, 0, 13, 1, 9]
    H, d = 2, 3
    seqs = [tuple(r.standard_normal((n, H, d)) for _ in range(3)) for n in lens]
    q = np.concatenate([s[0] for s in seqs]); k = np.concatenate([s[1] for s in seqs])
    v = np.concatenate([s[2] for s in seqs])
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    packed = {"q": impl.quadratic(q, k, v, cu), "r": impl.recurrent(q, k, v, cu),
              "b": impl.blocked(q, k, v, 4, cu)}
    st = impl.state(k, v, cu)
    for i, n in enumerate(lens):
        sl = slice(int(cu[i]), int(cu[i + 1]))
        if n == 0:
            assert np.array_equal(st[i], np.zeros((H, d, d))), "empty sequence state"
            continue
        sq, sk, sv = seqs[i]
        _close(packed["q"][sl], impl.quadratic(sq, sk, sv), 1e-12, "varlen (quadratic)")
        _close(packed["r"][sl], impl.recurrent(sq, sk, sv), 1e-12, "varlen (recurrent)")
        _close(packed["b"][sl], impl.blocked(sq, sk, sv, 4), 1e-12, "varlen (blocked)")
        _close(st[i], impl.state(sk, sv)[0], 1e-12, "varlen state")


def pin_state(impl):
    """state(a || b) = state(a) + state(b); it equals the recurrent and blocked final states."""
    r = _rng(19)
    H, d = 2, 4
    ka, va = (r.standard_normal((11, H, d)) for _ in range(2))
    kb, vb = (r.standard_normal((6, H, d)) for _ in range(2))
    k = np.concatenate([ka, kb]); v = np.concatenate([va, vb])
    sab = impl.state(k, v)
    _close(sab, impl.state(ka, va) + impl.state(kb, vb), 1e-12, "state additivity")
    q = r.standard_normal(k.shape)
    _, s_rec = impl.recurrent(q, k, v, return_state=True)
    _, s_blk = impl.blocked(q, k, v, 4, return_state=True)
    _close(s_rec, sab, 1e-12, "recurrent final state")
    _close(s_blk, sab, 1e-12, "blocked final state")
    S0 = r.standard_normal((1, H, d, d))
    _close(impl.state(k, v, init=S0), sab + S0, 1e-12, "state with init")


def pin_decode_continuity(impl):
    """Prefill of the first m tokens, then decode steps, reproduces the full prefill rows."""
    r = _rng(20)
    T, m, H, d = 19, 12, 2, 4
    q, k, v = (r.standard_normal((T, H, d)) for _ in range(3))
    full = impl.quadratic(q, k, v)
    st = impl.state(k[:m], v[:m])
    for t in range(m, T):
        o, st = impl.decode_step(q[t:t + 1], k[t:t + 1], v[t:t + 1], st)
        _close(o[0], full[t], 1e-10, f"decode step at t={t}")
    _close(st, impl.state(k, v), 1e-12, "decode final state")
    # one step from a zero state is (q . k) v
    o1, _ = impl.decode_step(q[:1], k[:1], v[:1], np.zeros((1, H, d, d)))
    _close(o1, impl.quadratic(q[:1], k[:1], v[:1]), 1e-14, "decode from zero state")


def pin_resume(impl):
    """Prefill of b with init = state(a) equals the b rows of prefill over a || b."""
    r = _rng(21)
    H, d = 2, 4
    q, k, v = (r.standard_normal((25, H, d)) for _ in range(3))
    full = impl.recurrent(q, k, v)
    S0 = impl.state(k[:10], v[:10])
    for name, o in (("quadratic", impl.quadratic(q[10:], k[10:], v[10:], init=S0)),
                    ("recurrent", impl.recurrent(q[10:], k[10:], v[10:], init=S0)),
                    ("blocked", impl.blocked(q[10:], k[10:], v[10:], 4, init=S0))):
        _close(o, full[10:], 1e-10, f"resume from carried state ({name})")


ALL_PINS = [pin_golden, pin_single_token, pin_onehot, pin_cumsum, pin_bruteforce_exact,
            pin_forms_agree, pin_linearity, pin_causality, pin_varlen, pin_state,
            pin_decode_continuity, pin_resume]


# --------------------------------------------------------------------------- backward
# Pins for ``backward`` (the gradients of L = sum_t dO_t . O_t). The pages
# give the forward only; these tie the gradients to the forward definition.
def pin_backward_finite_differences(impl):
    """Every gradient equals the central difference of L through the forward
    (``quadratic``). O is linear in each of q, k, v and S0 taken alone, so with a
    step of 1 the central difference is the derivative exactly, up to rounding."""
    r = _rng(30)
    cu = [0, 5, 9]
    T, H, d = 9, 2, 3
    q, k, v, do = (r.standard_normal((T, H, d)) for _ in range(4))
    init = r.standard_normal((2, H, d, d))
    dq, dk, dv, dinit = impl.backward(q, k, v, do, cu, init)
    args = {"q": q, "k": k, "v": v, "init": init}

    def loss(a):
        return float((do * impl.quadratic(a["q"], a["k"], a["v"], cu, init=a["init"])).sum())

    for name, grad in (("q", dq), ("k", dk), ("v", dv), ("init", dinit)):
        x = args[name]
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            plus, minus = dict(args), dict(args)
            xp, xm = x.copy(), x.copy()
            xp[idx] += 1.0
            xm[idx] -= 1.0
            plus[name], minus[name] = xp, xm
            fd[idx] = 0.5 * (loss(plus) - loss(minus))
        _close(grad, fd, 1e-10, f"dL/d{name}")


def pin_backward_single_token(impl):
    """n = 1, O = (q . k) v + q S0: dq = (dO . v) k + S0 dO, dk = (dO . v) q,
    dv = (q . k) dO, dS0 = q^T dO."""
    r = _rng(31)
    H, d = 2, 4
    q, k, v, do = (r.standard_normal((1, H, d)) for _ in range(4))
    S0 = r.standard_normal((1, H, d, d))
    dq, dk, dv, dinit = impl.backward(q, k, v, do, None, S0)
    for h in range(H):
        a, b, c, g = q[0, h], k[0, h], v[0, h], do[0, h]
        _close(dq[0, h], (g @ c) * b + S0[0, h] @ g, 1e-14, "dq, one token")
        _close(dk[0, h], (g @ c) * a, 1e-14, "dk, one token")
        _close(dv[0, h], (a @ b) * g, 1e-14, "dv, one token")
        _close(dinit[0, h], np.outer(a, g), 1e-14, "dS0, one token")


def pin_backward_varlen(impl):
    """Packed sequences: the gradients of each sequence are those of the sequence alone."""
    r = _rng(32)
    lengths = [6, 1, 9]
    T, H, d = sum(lengths), 2, 3
    q, k, v, do = (r.standard_normal((T, H, d)) for _ in range(4))
    cu = np.cumsum([0] + lengths)
    packed = impl.backward(q, k, v, do, cu, None)
    for s in range(len(lengths)):
        a, b = cu[s], cu[s + 1]
        alone = impl.backward(q[a:b], k[a:b], v[a:b], do[a:b], None, None)
        for name, x, y in zip(("dq", "dk", "dv"), packed[:3], alone[:3]):
            _close(x[a:b], y, 1e-12, f"{name} of sequence {s}")
        _close(packed[3][s], alone[3][0], 1e-12, f"dS0 of sequence {s}")


BACKWARD_PINS = [pin_backward_finite_differences, pin_backward_single_token, pin_backward_varlen]


# --------------------------------------------------------------------------- decay variant
# Pins for ``decay_*``: a per-head decay rate lambda_h on the state,
#   S_t = lambda_h S_{t-1} + k_t^T v_t,  S_{start-1} = S0,  o_t = q_t S_t.
# The pages give no decay; this is the Lightning Attention-2 form of the same
# method in its plainest reading. The pins tie it to the pinned no-decay
# functions (``quadratic``, ``state``, ``decode_step``) of the same object, to
# closed forms and to a library IIR filter.
def _decay_case(seed, lengths=(13, 1, 0, 22), H=3, d=4):
    r = _rng(seed)
    T = sum(lengths)
    q, k, v = (r.standard_normal((T, H, d)) for _ in range(3))
    init = r.standard_normal((len(lengths), H, d, d))
    cu = np.cumsum([0, *lengths])
    return q, k, v, init, cu


def _reweight(q, k, cu, lam):
    """q_t -> lambda^(r+1) q_t and k_s -> lambda^-(r+1) k_s, r the position in the sequence.
    Then (q'_t . k'_s) = lambda^(t-s) (q_t . k_s) and q'_t S0 = lambda^(t-start+1) q_t S0:
    the no-decay method on (q', k', v) is the decay method on (q, k, v)."""
    qw, kw = q.copy(), k.copy()
    for s in range(len(cu) - 1):
        for t in range(cu[s], cu[s + 1]):
            e = t - cu[s] + 1
            qw[t] *= (lam ** e)[:, None]
            kw[t] *= (lam ** (-e))[:, None]
    return qw, kw


def pin_decay_change_of_variables(impl):
    """Every decay form equals the pinned no-decay quadratic form on reweighted q, k."""
    lam = np.array([0.5, 0.8, 0.97])
    q, k, v, init, cu = _decay_case(40)
    qw, kw = _reweight(q, k, cu, lam)
    want = impl.quadratic(qw, kw, v, cu, init=init)
    _close(impl.decay_quadratic(q, k, v, lam, cu, init=init), want, 1e-11, "decay quadratic")
    _close(impl.decay_recurrent(q, k, v, lam, cu, init=init), want, 1e-11, "decay recurrent")
    for B in (1, 2, 5, 8, 64):
        _close(impl.decay_blocked(q, k, v, lam, B, cu, init=init), want, 1e-11, f"decay blocked B={B}")
    # final state: lambda^n (S0 + sum_s lambda^-(r_s+1) k_s^T v_s) = lambda^n state(k', v, S0)
    n = np.diff(cu)
    st_want = impl.state(kw, v, cu, init=init) * (lam[None, :] ** n[:, None])[:, :, None, None]
    _close(impl.decay_state(k, v, lam, cu, init=init), st_want, 1e-11, "decay state")
    _, st_r = impl.decay_recurrent(q, k, v, lam, cu, init=init, return_state=True)
    _, st_b = impl.decay_blocked(q, k, v, lam, 4, cu, init=init, return_state=True)
    _close(st_r, st_want, 1e-11, "decay recurrent final state")
    _close(st_b, st_want, 1e-11, "decay blocked final state")
    # decode: lambda S + k^T v = lambda (S + (k / lambda)^T v), o = (lambda q)(S + (k / lambda)^T v)
    r = _rng(41)
    dq, dk, dv = (r.standard_normal((2, 3, 4)) for _ in range(3))
    S = r.standard_normal((2, 3, 4, 4))
    o_w, s_w = impl.decode_step(dq * lam[None, :, None], dk / lam[None, :, None], dv, S)
    o, s_new = impl.decay_decode_step(dq, dk, dv, S, lam)
    _close(o, o_w, 1e-13, "decay decode o")
    _close(s_new, s_w * lam[None, :, None, None], 1e-13, "decay decode state")


def pin_decay_one(impl):
    """lambda = 1 is the method without decay."""
    lam = np.ones(3)
    q, k, v, init, cu = _decay_case(42)
    want = impl.quadratic(q, k, v, cu, init=init)
    _close(impl.decay_quadratic(q, k, v, lam, cu, init=init), want, 1e-12, "lambda=1 quadratic")
    _close(impl.decay_recurrent(q, k, v, lam, cu, init=init), want, 1e-12, "lambda=1 recurrent")
    _close(impl.decay_blocked(q, k, v, lam, 4, cu, init=init), want, 1e-12, "lambda=1 blocked")
    _close(impl.decay_state(k, v, lam, cu, init=init), impl.state(k, v, cu, init=init), 1e-12, "lambda=1 state")


def pin_decay_zero(impl):
    """lambda = 0 keeps only the current token: O_t = (q_t . k_t) v_t, S0 unseen even at t = start;
    the final state is k_last^T v_last (S0 for an empty sequence)."""
    lam = np.zeros(3)
    q, k, v, init, cu = _decay_case(43)
    want = np.einsum("thi,thi->th", q, k)[:, :, None] * v
    for name, o in (("quadratic", impl.decay_quadratic(q, k, v, lam, cu, init=init)),
                    ("recurrent", impl.decay_recurrent(q, k, v, lam, cu, init=init)),
                    ("blocked", impl.decay_blocked(q, k, v, lam, 4, cu, init=init))):
        _close(o, want, 1e-14, f"lambda=0 {name}")
    st = impl.decay_state(k, v, lam, cu, init=init)
    for s in range(len(cu) - 1):
        for h in range(3):
            last = cu[s + 1] - 1
            exp = init[s, h] if cu[s + 1] == cu[s] else np.outer(k[last, h], v[last, h])
            _close(st[s, h], exp, 1e-14, f"lambda=0 state of sequence {s}")
    o, sn = impl.decay_decode_step(q[:2], k[:2], v[:2], init[:2], lam)
    _close(o, want[:2], 1e-14, "lambda=0 decode o")
    _close(sn, np.einsum("bhi,bhj->bhij", k[:2], v[:2]), 1e-14, "lambda=0 decode state")


def pin_decay_discounted_cumsum(impl):
    """All scores one (q = k = e_0): O_t = sum_{s<=t} lambda^(t-s) v_s + lambda^(t-start+1) S0[0, :],
    the first-order IIR filter y_t = v_t + lambda y_{t-1}, y_{start-1} = S0[0, :] (scipy's lfilter)."""
    from scipy.signal import lfilter
    lam = np.array([0.3, 0.9])
    lengths = (9, 14)
    T, H, d = sum(lengths), 2, 3
    r = _rng(44)
    q = np.zeros((T, H, d)); q[:, :, 0] = 1.0
    k = q.copy()
    v = r.standard_normal((T, H, d))
    init = r.standard_normal((2, H, d, d))
    cu = np.cumsum([0, *lengths])
    want = np.zeros_like(v)
    for s in range(2):
        for h in range(H):
            a, b = cu[s], cu[s + 1]
            want[a:b, h], _ = lfilter([1.0], [1.0, -lam[h]], v[a:b, h], axis=0, zi=lam[h] * init[s, h, 0][None, :])
    for name, o in (("quadratic", impl.decay_quadratic(q, k, v, lam, cu, init=init)),
                    ("recurrent", impl.decay_recurrent(q, k, v, lam, cu, init=init)),
                    ("blocked B=4", impl.decay_blocked(q, k, v, lam, 4, cu, init=init)),
                    ("blocked B=16", impl.decay_blocked(q, k, v, lam, 16, cu, init=init))):
        _close(o, want, 1e-12, f"discounted cumsum ({name})")


def pin_decay_split(impl):
    """Splitting a sequence anywhere: the tail run from the head's final state reproduces the
    tail rows, and decode steps from the state of a prefix reproduce the following rows."""
    lam = np.array([0.6, 0.95])
    r = _rng(45)
    T, H, d = 21, 2, 4
    q, k, v = (r.standard_normal((T, H, d)) for _ in range(3))
    S0 = r.standard_normal((1, H, d, d))
    full = impl.decay_quadratic(q, k, v, lam, init=S0)
    for m in (1, 8, 20):
        st = impl.decay_state(k[:m], v[:m], lam, init=S0)
        _close(impl.decay_recurrent(q[m:], k[m:], v[m:], lam, init=st), full[m:], 1e-11, f"resume at {m}")
        _close(impl.decay_blocked(q[m:], k[m:], v[m:], lam, 3, init=st), full[m:], 1e-11, f"resume blocked at {m}")
    st = impl.decay_state(k[:12], v[:12], lam, init=S0)
    for t in range(12, T):
        o, st = impl.decay_decode_step(q[t:t + 1], k[t:t + 1], v[t:t + 1], st, lam)
        _close(o[0], full[t], 1e-11, f"decay decode at t={t}")
    _close(st, impl.decay_state(k, v, lam, init=S0), 1e-11, "decay decode final state")


def pin_decay_bruteforce_exact(impl):
    """Exact rational arithmetic of the recurrence S_t = lambda S_{t-1} + k_t^T v_t, o_t = q_t S_t on
    tiny integer inputs with rates 1/2 and 3/4 and an integer S0: every value is a dyadic rational
    that fp64 holds exactly, so each form must match bit for bit."""
    r = _rng(46)
    T, H, d = 7, 2, 3
    q, k, v = (r.integers(-3, 4, size=(T, H, d)) for _ in range(3))
    S0 = r.integers(-2, 3, size=(2, H, d, d))
    lam = [Fraction(1, 2), Fraction(3, 4)]
    cu = [0, 3, 7]
    want = np.zeros((T, H, d))
    want_st = np.zeros((2, H, d, d))
    for si in range(2):
        for h in range(H):
            S = [[Fraction(int(S0[si, h, i, j])) for j in range(d)] for i in range(d)]
            for t in range(cu[si], cu[si + 1]):
                S = [[lam[h] * S[i][j] + int(k[t, h, i]) * int(v[t, h, j]) for j in range(d)] for i in range(d)]
                want[t, h] = [float(sum(int(q[t, h, i]) * S[i][j] for i in range(d))) for j in range(d)]
            want_st[si, h] = [[float(x) for x in row] for row in S]
    qf, kf, vf, s0 = (x.astype(np.float64) for x in (q, k, v, S0))
    lf = np.array([0.5, 0.75])
    assert np.array_equal(impl.decay_quadratic(qf, kf, vf, lf, cu, init=s0), want), "decay brute force (quadratic)"
    assert np.array_equal(impl.decay_recurrent(qf, kf, vf, lf, cu, init=s0), want), "decay brute force (recurrent)"
    for B in (1, 2, 3, 5, 8):
        assert np.array_equal(impl.decay_blocked(qf, kf, vf, lf, B, cu, init=s0), want), \
            f"decay brute force (blocked B={B})"
    assert np.array_equal(impl.decay_state(kf, vf, lf, cu, init=s0), want_st), "decay brute force (state)"


DECAY_PINS = [pin_decay_change_of_variables, pin_decay_one, pin_decay_zero, pin_decay_discounted_cumsum,
              pin_decay_split, pin_decay_bruteforce_exact]


# --------------------------------------------------------------------------- feature map
def pin_feature_map(impl):
    """phi(x) = ELU(x) + 0.3 x (page "MiniMax-M2.5语言模型：Linear Attention架构解析与实践",
    section 2.2): torch's ELU plus 0.3 x, and values worked by hand."""
    import math
    import torch
    x = np.concatenate([np.linspace(-30, 30, 601), [-1e-12, 0.0, 1e-12, -700.0, 5e3]])
    want = torch.nn.functional.elu(torch.from_numpy(x)).numpy() + 0.3 * x
    _close(impl.feature_map(x), want, 1e-15, "phi against torch ELU")
    got = impl.feature_map(np.array([0.0, 1.0, 2.0, -1.0, -2.0]))
    hand = [0.0, 1.3, 2.6, math.exp(-1.0) - 1.0 - 0.3, math.exp(-2.0) - 1.0 - 0.6]
    np.testing.assert_allclose(got, hand, rtol=1e-15, atol=1e-16, err_msg="phi by hand")
    tiny = impl.feature_map(np.array([-1e-20]))[0]          # e^x - 1 without cancellation
    assert abs(tiny + 1.3e-20) <= 1e-15 * 1.3e-20, "phi near zero keeps relative precision"
    y = impl.feature_map(np.ones((2, 3)) * -0.5, alpha=0.0)
    _close(y, np.full((2, 3), math.expm1(-0.5)), 1e-15, "alpha = 0 is ELU")


FEATURE_PINS = [pin_feature_map]


# --------------------------------------------------------------------------- decay backward
def pin_decay_backward_finite_differences(impl):
    """Every gradient of the decay variant equals the central difference of L through the pinned
    ``decay_quadratic``; O is linear in each of q, k, v and S0 taken alone, so a step of 1 gives
    the derivative exactly, up to rounding."""
    r = _rng(47)
    cu = [0, 5, 9]
    T, H, d = 9, 2, 3
    q, k, v, do = (r.standard_normal((T, H, d)) for _ in range(4))
    init = r.standard_normal((2, H, d, d))
    lam = np.array([0.6, 0.9])
    dq, dk, dv, dinit = impl.decay_backward(q, k, v, do, lam, cu, init)
    args = {"q": q, "k": k, "v": v, "init": init}

    def loss(a):
        return float((do * impl.decay_quadratic(a["q"], a["k"], a["v"], lam, cu, init=a["init"])).sum())

    for name, grad in (("q", dq), ("k", dk), ("v", dv), ("init", dinit)):
        x = args[name]
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            plus, minus = dict(args), dict(args)
            xp, xm = x.copy(), x.copy()
            xp[idx] += 1.0
            xm[idx] -= 1.0
            plus[name], minus[name] = xp, xm
            fd[idx] = 0.5 * (loss(plus) - loss(minus))
        _close(grad, fd, 1e-10, f"decay dL/d{name}")


def pin_decay_backward_one_and_zero(impl):
    """lambda = 1 is the backward without decay; lambda = 0 leaves O_t = (q_t . k_t) v_t, whose
    gradients are dq_t = (dO_t . v_t) k_t, dk_t = (dO_t . v_t) q_t, dv_t = (q_t . k_t) dO_t, dS0 = 0."""
    r = _rng(48)
    cu = [0, 4, 11]
    T, H, d = 11, 2, 3
    q, k, v, do = (r.standard_normal((T, H, d)) for _ in range(4))
    init = r.standard_normal((2, H, d, d))
    got = impl.decay_backward(q, k, v, do, np.ones(H), cu, init)
    want = impl.backward(q, k, v, do, cu, init)
    for name, a, b in zip(("dq", "dk", "dv", "dS0"), got, want):
        _close(a, b, 1e-12, f"lambda = 1: {name}")
    dq, dk, dv, dinit = impl.decay_backward(q, k, v, do, np.zeros(H), cu, init)
    gv = np.einsum("thj,thj->th", do, v)[:, :, None]
    qk = np.einsum("thi,thi->th", q, k)[:, :, None]
    _close(dq, gv * k, 1e-14, "lambda = 0: dq")
    _close(dk, gv * q, 1e-14, "lambda = 0: dk")
    _close(dv, qk * do, 1e-14, "lambda = 0: dv")
    assert np.array_equal(dinit, np.zeros_like(dinit)), "lambda = 0: dS0"


DECAY_BACKWARD_PINS = [pin_decay_backward_finite_differences, pin_decay_backward_one_and_zero]
