"""The pins are sharp: each plausible mistake, planted in a small numpy twin of
the oracle on the CPU, fails at least one pin, while the twin without a
mistake passes them all."""
import numpy as np
import pytest

import pins


class Twin:
    """numpy restatement of the oracle's five functions with an optional planted bug."""

    def __init__(self, bug=None):
        self.bug = bug

    # helpers ---------------------------------------------------------------
    @staticmethod
    def _cu(T, cu):
        return [0, T] if cu is None else [int(x) for x in cu]

    def _outer(self, kv, vv):
        return np.outer(vv, kv) if self.bug == "transpose_state" else np.outer(kv, vv)

    def _mask(self, n):
        if self.bug == "exclusive_mask":
            return np.tril(np.ones((n, n)), -1)
        if self.bug == "anticausal":
            return np.triu(np.ones((n, n)))
        return np.tril(np.ones((n, n)))

    def _scores(self, Q, K):
        return K @ Q.T if self.bug == "swap_qk" else Q @ K.T

    def _post(self, o, d):
        return o / np.sqrt(d) if self.bug == "scaled" else o

    def _init(self, init, s, h, d):
        if init is None or self.bug == "drop_init":
            return np.zeros((d, d))
        return np.array(init[s, h], dtype=np.float64)

    # interface ---------------------------------------------------------------
    def quadratic(self, q, k, v, cu_seqlens=None, init=None):
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        T, H, d = q.shape
        cu = self._cu(T, cu_seqlens)
        o = np.zeros_like(q)
        for s in range(len(cu) - 1):
            a, b = cu[s], cu[s + 1]
            for h in range(H):
                Q, K, V = q[a:b, h], k[a:b, h], v[a:b, h]
                o[a:b, h] = (self._scores(Q, K) * self._mask(b - a)) @ V + Q @ self._init(init, s, h, d)
        return self._post(o, d)

    def recurrent(self, q, k, v, cu_seqlens=None, init=None, return_state=False):
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        T, H, d = q.shape
        cu = self._cu(T, cu_seqlens)
        o = np.zeros_like(q)
        st = np.zeros((len(cu) - 1, H, d, d))
        carry = [np.zeros((d, d)) for _ in range(H)]
        for s in range(len(cu) - 1):
            for h in range(H):
                S = carry[h] if self.bug == "no_reset" else self._init(init, s, h, d)
                for t in range(cu[s], cu[s + 1]):
                    if self.bug == "output_before_update":
                        o[t, h] = q[t, h] @ S
                        S = S + self._outer(k[t, h], v[t, h])
                    else:
                        S = S + self._outer(k[t, h], v[t, h])
                        o[t, h] = q[t, h] @ S
                st[s, h] = S
                carry[h] = S
        o = self._post(o, d)
        return (o, st) if return_state else o

    def blocked(self, q, k, v, B, cu_seqlens=None, init=None, return_state=False):
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        T, H, d = q.shape
        cu = self._cu(T, cu_seqlens)
        o = np.zeros_like(q)
        st = np.zeros((len(cu) - 1, H, d, d))
        for s in range(len(cu) - 1):
            a, e = cu[s], cu[s + 1]
            for h in range(H):
                KV = self._init(init, s, h, d)
                starts = list(range(a, e, B))
                for i, b0 in enumerate(starts):
                    b1 = starts[i + 1] if i + 1 < len(starts) else e
                    Q, K, V = q[b0:b1, h], k[b0:b1, h], v[b0:b1, h]
                    upd = sum((self._outer(K[u], V[u]) for u in range(b1 - b0)), np.zeros((d, d)))
                    if self.bug == "prefix_inclusive":
                        KV = KV + upd
                    mask = np.ones((b1 - b0, b1 - b0)) if self.bug == "block_nomask" else self._mask(b1 - b0)
                    o[b0:b1, h] = (self._scores(Q, K) * mask) @ V
                    if self.bug != "no_inter":
                        o[b0:b1, h] += Q @ KV
                    if self.bug != "prefix_inclusive":
                        KV = KV + upd
                st[s, h] = KV
        o = self._post(o, d)
        return (o, st) if return_state else o

    def state(self, k, v, cu_seqlens=None, init=None):
        k, v = (np.asarray(x, dtype=np.float64) for x in (k, v))
        T, H, d = k.shape
        cu = self._cu(T, cu_seqlens)
        st = np.zeros((len(cu) - 1, H, d, d))
        for s in range(len(cu) - 1):
            for h in range(H):
                S = self._init(init, s, h, d)
                for t in range(cu[s], cu[s + 1]):
                    S = S + self._outer(k[t, h], v[t, h])
                st[s, h] = S
        return st

    def decode_step(self, q, k, v, state_in):
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        Bt, H, d = q.shape
        st = np.array(state_in, dtype=np.float64, copy=True)
        o = np.zeros_like(q)
        for b in range(Bt):
            for h in range(H):
                if self.bug == "output_before_update":
                    o[b, h] = q[b, h] @ st[b, h]
                    st[b, h] += self._outer(k[b, h], v[b, h])
                else:
                    st[b, h] += self._outer(k[b, h], v[b, h])
                    o[b, h] = q[b, h] @ st[b, h]
        return self._post(o, d), st


    def backward(self, q, k, v, dout, cu_seqlens=None, init=None):
        """Gradients of L = sum dO . O (restated: forward pass for dq, reverse for the rest)."""
        q, k, v, g = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dout))
        T, H, d = q.shape
        cu = self._cu(T, cu_seqlens)
        dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
        dinit = np.zeros((len(cu) - 1, H, d, d))
        for s in range(len(cu) - 1):
            a, b = cu[s], cu[s + 1]
            for h in range(H):
                S = np.zeros((d, d)) if self.bug == "bwd_dq_no_init" else self._init(init, s, h, d)
                for t in range(a, b):
                    S = S + np.outer(k[t, h], v[t, h])
                    dq[t, h] = g[t, h] @ S if self.bug == "bwd_dq_untransposed" else S @ g[t, h]
                R = np.zeros((d, d))
                for t in range(b - 1, a - 1, -1):
                    if self.bug == "bwd_exclusive_reverse":
                        dk[t, h], dv[t, h] = R @ v[t, h], R.T @ k[t, h]
                        R = R + np.outer(q[t, h], g[t, h])
                        continue
                    R = R + np.outer(q[t, h], g[t, h])
                    dk[t, h] = R @ v[t, h]
                    dv[t, h] = R @ k[t, h] if self.bug == "bwd_dv_untransposed" else R.T @ k[t, h]
                dinit[s, h] = R.T if self.bug == "bwd_dinit_transposed" else R
        return dq, dk, dv, dinit


BUGS = ["exclusive_mask", "anticausal", "transpose_state", "drop_init", "output_before_update",
        "no_inter", "prefix_inclusive", "no_reset", "swap_qk", "scaled", "block_nomask"]


def _failing_pins(impl):
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(impl)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


def test_clean_twin_passes_every_pin():
    assert _failing_pins(Twin()) == []


@pytest.mark.parametrize("bug", BUGS)
def test_planted_bug_is_caught(bug):
    failed = _failing_pins(Twin(bug))
    assert failed, f"no pin catches the planted bug {bug!r}"


BACKWARD_BUGS = ["bwd_dq_no_init", "bwd_dq_untransposed", "bwd_exclusive_reverse", "bwd_dv_untransposed",
                 "bwd_dinit_transposed"]


def _failing_backward_pins(impl):
    failed = []
    for pin in pins.BACKWARD_PINS:
        try:
            pin(impl)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


def test_clean_twin_passes_every_backward_pin():
    assert _failing_backward_pins(Twin()) == []


@pytest.mark.parametrize("bug", BACKWARD_BUGS)
def test_planted_backward_bug_is_caught(bug):
    failed = _failing_backward_pins(Twin(bug))
    assert failed, f"no backward pin catches the planted bug {bug!r}"


class DecayTwin(Twin):
    """numpy restatement of the decay functions, with an optional planted bug; the
    no-decay functions it inherits are the clean twin's."""

    def __init__(self, bug=None):
        super().__init__(None)
        self.dbug = bug

    def _lam(self, lam, h):
        return lam[0] if self.dbug == "decay_head0" else lam[h]

    def _inter_pow(self, r):
        return r if self.dbug == "decay_inter_pow_r" else r + 1

    def _intra_pow(self, t, u):
        return t - u + 1 if self.dbug == "decay_intra_pow_plus1" else t - u

    def decay_quadratic(self, q, k, v, decay, cu_seqlens=None, init=None):
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        T, H, d = q.shape
        cu = self._cu(T, cu_seqlens)
        o = np.zeros_like(q)
        for s in range(len(cu) - 1):
            a, b = cu[s], cu[s + 1]
            for h in range(H):
                lam = self._lam(decay, h)
                S0 = self._init(init, s, h, d)
                for t in range(a, b):
                    acc = lam ** self._inter_pow(t - a) * (q[t, h] @ S0)
                    for u in range(a, t + 1):
                        acc = acc + lam ** self._intra_pow(t, u) * (q[t, h] @ k[u, h]) * v[u, h]
                    o[t, h] = acc
        return o

    def decay_recurrent(self, q, k, v, decay, cu_seqlens=None, init=None, return_state=False):
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        T, H, d = q.shape
        cu = self._cu(T, cu_seqlens)
        o = np.zeros_like(q)
        st = np.zeros((len(cu) - 1, H, d, d))
        for s in range(len(cu) - 1):
            for h in range(H):
                lam = self._lam(decay, h)
                S = self._init(init, s, h, d)
                for t in range(cu[s], cu[s + 1]):
                    if self.dbug == "decay_after_add":
                        S = lam * (S + np.outer(k[t, h], v[t, h]))
                    else:
                        S = lam * S + np.outer(k[t, h], v[t, h])
                    o[t, h] = q[t, h] @ S
                st[s, h] = S
        return (o, st) if return_state else o

    def decay_blocked(self, q, k, v, decay, B, cu_seqlens=None, init=None, return_state=False):
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        T, H, d = q.shape
        cu = self._cu(T, cu_seqlens)
        o = np.zeros_like(q)
        st = np.zeros((len(cu) - 1, H, d, d))
        for s in range(len(cu) - 1):
            a, e = cu[s], cu[s + 1]
            for h in range(H):
                lam = self._lam(decay, h)
                KV = self._init(init, s, h, d)
                for b0 in range(a, e, B):
                    b1 = min(b0 + B, e)
                    n = b1 - b0
                    r = np.arange(n)
                    M = np.tril(lam ** np.maximum(self._intra_pow(r[:, None], r[None, :]), 0))
                    Q, K, V = q[b0:b1, h], k[b0:b1, h], v[b0:b1, h]
                    o[b0:b1, h] = ((Q @ K.T) * M) @ V + (lam ** self._inter_pow(r))[:, None] * (Q @ KV)
                    kpow = n - r if self.dbug == "decay_key_pow" else n - 1 - r
                    blk = (K * (lam ** kpow)[:, None]).T @ V
                    KV = blk + (KV if self.dbug == "decay_prefix_undecayed" else lam ** n * KV)
                st[s, h] = KV
        return (o, st) if return_state else o

    def decay_state(self, k, v, decay, cu_seqlens=None, init=None):
        k, v = (np.asarray(x, dtype=np.float64) for x in (k, v))
        T, H, d = k.shape
        cu = self._cu(T, cu_seqlens)
        st = np.zeros((len(cu) - 1, H, d, d))
        for s in range(len(cu) - 1):
            a, b = cu[s], cu[s + 1]
            for h in range(H):
                lam = self._lam(decay, h)
                n = b - a
                S = (lam ** (n if self.dbug != "decay_state_init_undecayed" else 0)) * self._init(init, s, h, d)
                for t in range(a, b):
                    S = S + lam ** (b - 1 - t) * np.outer(k[t, h], v[t, h])
                st[s, h] = S
        return st

    def decay_decode_step(self, q, k, v, state_in, decay):
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        Bt, H, d = q.shape
        st = np.array(state_in, dtype=np.float64, copy=True)
        o = np.zeros_like(q)
        for b in range(Bt):
            for h in range(H):
                lam = self._lam(decay, h)
                if self.dbug == "decay_decode_output_first":
                    o[b, h] = q[b, h] @ st[b, h]
                    st[b, h] = lam * st[b, h] + np.outer(k[b, h], v[b, h])
                else:
                    st[b, h] = lam * st[b, h] + np.outer(k[b, h], v[b, h])
                    o[b, h] = q[b, h] @ st[b, h]
        return o, st


DECAY_BUGS = ["decay_head0", "decay_inter_pow_r", "decay_intra_pow_plus1", "decay_after_add", "decay_key_pow",
              "decay_prefix_undecayed", "decay_state_init_undecayed", "decay_decode_output_first"]


def _failing_decay_pins(impl):
    failed = []
    for pin in pins.DECAY_PINS:
        try:
            pin(impl)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


def test_clean_decay_twin_passes_every_decay_pin():
    assert _failing_decay_pins(DecayTwin()) == []


@pytest.mark.parametrize("bug", DECAY_BUGS)
def test_planted_decay_bug_is_caught(bug):
    failed = _failing_decay_pins(DecayTwin(bug))
    assert failed, f"no decay pin catches the planted bug {bug!r}"


class FeatureTwin:
    def __init__(self, bug=None):
        self.bug = bug

    def feature_map(self, x, alpha=0.3):
        x = np.asarray(x, dtype=np.float64)
        with np.errstate(over="ignore"):
            return self._phi(x, alpha)

    def _phi(self, x, alpha):
        if self.bug == "elu_exp_not_expm1":
            e = np.where(x > 0, x, np.exp(x) - 1.0)
        elif self.bug == "elu_plus_one":
            e = np.where(x > 0, x, np.expm1(x)) + 1.0
        elif self.bug == "alpha_on_negative_only":
            return np.where(x > 0, x, np.expm1(x) + alpha * x)
        else:
            e = np.where(x > 0, x, np.expm1(np.minimum(x, 0.0)))
        return e + alpha * x


@pytest.mark.parametrize("bug", [None, "elu_exp_not_expm1", "elu_plus_one", "alpha_on_negative_only"])
def test_feature_map_pin_is_sharp(bug):
    try:
        pins.pin_feature_map(FeatureTwin(bug))
        caught = False
    except AssertionError:
        caught = True
    assert caught == (bug is not None)


class DecayBackwardTwin(DecayTwin):
    """numpy restatement of the decay variant's gradients with an optional planted bug (its
    forward and plain backward are the clean twin's)."""

    def __init__(self, bug=None):
        super().__init__(None)
        self.gbug = bug

    def decay_backward(self, q, k, v, dout, decay, cu_seqlens=None, init=None):
        q, k, v, g = (np.asarray(x, dtype=np.float64) for x in (q, k, v, dout))
        T, H, d = q.shape
        cu = self._cu(T, cu_seqlens)
        dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
        dinit = np.zeros((len(cu) - 1, H, d, d))
        for s in range(len(cu) - 1):
            a, b = cu[s], cu[s + 1]
            for h in range(H):
                lam = decay[h]
                S = self._init(init, s, h, d)
                for t in range(a, b):
                    S = (S if self.gbug == "gbwd_forward_undecayed" else lam * S) + np.outer(k[t, h], v[t, h])
                    dq[t, h] = S @ g[t, h]
                R = np.zeros((d, d))
                for t in range(b - 1, a - 1, -1):
                    R = (R if self.gbug == "gbwd_reverse_undecayed" else lam * R) + np.outer(q[t, h], g[t, h])
                    dk[t, h] = R @ v[t, h]
                    dv[t, h] = R.T @ k[t, h]
                dinit[s, h] = R if self.gbug == "gbwd_dinit_undecayed" else lam * R
        return dq, dk, dv, dinit


DECAY_BACKWARD_BUGS = ["gbwd_forward_undecayed", "gbwd_reverse_undecayed", "gbwd_dinit_undecayed"]


def _failing_decay_backward_pins(impl):
    failed = []
    for pin in pins.DECAY_BACKWARD_PINS:
        try:
            pin(impl)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


def test_clean_decay_backward_twin_passes():
    assert _failing_decay_backward_pins(DecayBackwardTwin()) == []


@pytest.mark.parametrize("bug", DECAY_BACKWARD_BUGS)
def test_planted_decay_backward_bug_is_caught(bug):
    assert _failing_decay_backward_pins(DecayBackwardTwin(bug)), f"no pin catches {bug!r}"
