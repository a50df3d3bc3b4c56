"""The C-ABI library loads, exports every function the header declares, and
rejects bad arguments on the host before anything is enqueued (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

import causal_linear_attention_02_b200 as la

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        for m in re.finditer(r"\b(la_[a-z0-9_]+)\s*\(", text):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    from causal_linear_attention_02_b200 import build
    build.build()
    return la.load_library()


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("la_prefill", "la_state_from_prefill", "la_decode_step", "la_prefill_workspace_size",
              "la_state_workspace_size", "la_get_device_status", "la_status_string", "la_version"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", la.library_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = sorted(n for n in declared_functions() if n not in exported)
    assert not missing, f"declared but not exported: {missing}"
    for n in declared_functions():
        assert hasattr(lib, n)


def test_status_strings(lib):
    for code in la.STATUS:
        assert la.la_status_string(code)
    assert la.la_version() >= 100


P = 1 << 20          # fake, 256-aligned "device" addresses: never dereferenced, the host checks fail first
BIG = 1 << 40

# The checks with fabricated addresses run only where no CUDA device is visible: on a
# machine with a GPU a regression in a host check must not hand a kernel an unmapped
# pointer. (The GPU suites call every entry point with real buffers.)
fake_pointers = pytest.mark.skipif(__import__("torch").cuda.is_available(),
                                   reason="fabricated device addresses are only used where no GPU exists")


def prefill(**kw):
    a = dict(q=P, k=2 * P, v=3 * P, o=4 * P, cu=None, nseq=1, T=64, H=2, d=128, B=256, dt=la.LA_BF16,
             init=None, ws=5 * P, wsb=BIG, stream=None)
    a.update(kw)
    return la.la_prefill(a["q"], a["k"], a["v"], a["o"], a["cu"], a["nseq"], a["T"], a["H"], a["d"], a["B"],
                         a["dt"], a["init"], a["ws"], a["wsb"], a["stream"])


@fake_pointers
def test_prefill_argument_errors(lib):
    assert prefill(T=-1) == 1
    assert prefill(H=0) == 1
    assert prefill(nseq=0) == 1
    assert prefill(nseq=2, cu=None) == 1                # several sequences need cu_seqlens
    assert prefill(d=100) == 2
    assert prefill(d=256) == 2
    assert prefill(B=96) == 2
    assert prefill(dt=7) == 2
    assert prefill(q=P + 8) == 3                        # not 16-byte aligned
    assert prefill(o=4 * P + 4) == 3
    assert prefill(init=P + 4) == 3
    assert prefill(ws=5 * P + 16) == 3                  # workspace must be 256-byte aligned
    assert prefill(o=P) == 1                            # output aliases q
    assert prefill(o=P + 64 * 2 * 128 * 2 - 256) == 1  # partial overlap with q
    assert prefill(wsb=16) == 4
    assert prefill(ws=None) == 1
    assert prefill(q=None) == 1
    assert prefill(T=0) == 0                            # empty input: nothing to do, nothing enqueued


@fake_pointers
def test_decode_argument_errors(lib):
    def dec(**kw):
        a = dict(q=P, k=2 * P, v=3 * P, s=8 * P, o=4 * P, b=4, H=2, d=128, dt=la.LA_BF16)
        a.update(kw)
        return la.la_decode_step(a["q"], a["k"], a["v"], a["s"], a["o"], a["b"], a["H"], a["d"], a["dt"], None)
    assert dec(b=-1) == 1
    assert dec(H=0) == 1
    assert dec(d=8) == 2
    assert dec(dt=5) == 2
    assert dec(s=None) == 1
    assert dec(q=P + 2) == 3
    assert dec(o=P) == 1                                # output aliases q
    assert dec(s=2 * P) == 1                            # state overlaps k
    assert dec(b=0) == 0


@fake_pointers
def test_state_argument_errors(lib):
    def st(**kw):
        a = dict(k=P, v=2 * P, cu=None, nseq=1, T=64, H=2, d=64, dt=la.LA_FP32, init=None, out=4 * P,
                 ws=5 * P, wsb=BIG)
        a.update(kw)
        return la.la_state_from_prefill(a["k"], a["v"], a["cu"], a["nseq"], a["T"], a["H"], a["d"], a["dt"],
                                        a["init"], a["out"], a["ws"], a["wsb"], None)
    assert st(out=None) == 1
    assert st(T=-5) == 1
    assert st(d=50) == 2
    assert st(k=P + 4) == 3
    assert st(wsb=8) == 4
    assert st(init=4 * P + 1024) == 1                   # partial overlap of init and out


@fake_pointers
def test_decay_argument_errors(lib):
    """Host checks of the decay entry points (each case fails before any launch)."""
    def pre(**kw):
        a = dict(q=P, k=2 * P, v=3 * P, o=4 * P, cu=None, nseq=1, T=64, H=2, d=128, B=256, dt=la.LA_BF16,
                 init=None, decay=6 * P, out=None, ws=5 * P, wsb=BIG)
        a.update(kw)
        return la.la_prefill_decay(a["q"], a["k"], a["v"], a["o"], a["cu"], a["nseq"], a["T"], a["H"], a["d"],
                                   a["B"], a["dt"], a["init"], a["decay"], a["out"], a["ws"], a["wsb"], None)
    assert pre(decay=None) == 1
    assert pre(decay=6 * P + 2) == 3                    # rates are 4-byte aligned fp32
    assert pre(decay=4 * P) == 1                        # rates inside the output
    assert pre(d=100) == 2
    assert pre(B=32) == 2
    assert pre(out=8 * P + 4) == 3
    assert pre(out=4 * P) == 1                          # state_out overlaps o
    assert pre(init=8 * P, out=8 * P + 4096) == 1       # state_out partially overlaps init
    assert pre(wsb=16) == 4
    assert pre(ws=None) == 1
    assert pre(T=0) == 0                                # nothing to compute, no state asked for

    def st(**kw):
        a = dict(k=P, v=2 * P, cu=None, nseq=1, T=64, H=2, d=64, dt=la.LA_FP32, init=None, decay=6 * P,
                 out=4 * P, ws=5 * P, wsb=BIG)
        a.update(kw)
        return la.la_state_decay(a["k"], a["v"], a["cu"], a["nseq"], a["T"], a["H"], a["d"], a["dt"], a["init"],
                                 a["decay"], a["out"], a["ws"], a["wsb"], None)
    assert st(decay=None) == 1
    assert st(out=None) == 1
    assert st(decay=4 * P) == 1                         # rates inside the state
    assert st(wsb=8) == 4

    def dec(**kw):
        a = dict(q=P, k=2 * P, v=3 * P, s=8 * P, o=4 * P, b=4, H=2, d=128, dt=la.LA_BF16, decay=6 * P)
        a.update(kw)
        return la.la_decode_step_decay(a["q"], a["k"], a["v"], a["s"], a["o"], a["b"], a["H"], a["d"], a["dt"],
                                       a["decay"], None)
    assert dec(decay=None) == 1
    assert dec(decay=8 * P) == 1                        # rates inside the state
    assert dec(decay=6 * P + 1) == 3
    assert dec(s=2 * P) == 1
    assert dec(b=0) == 0

    def pre_decay(**kw):
        a = dict(g=P, lens=2 * P, world=2, rank=1, nseq=3, H=2, d=64, decay=3 * P, init=None, out=4 * P)
        a.update(kw)
        return la.la_state_exclusive_prefix_decay(a["g"], a["lens"], a["world"], a["rank"], a["nseq"], a["H"], a["d"],
                                                  a["decay"], a["init"], a["out"], None)
    assert pre_decay(rank=3) == 1                       # rank above world
    assert pre_decay(H=0) == 1
    assert pre_decay(d=20) == 2
    assert pre_decay(decay=None) == 1
    assert pre_decay(lens=None) == 1                    # rank > 0 needs the segment lengths
    assert pre_decay(lens=2 * P + 2) == 3
    assert pre_decay(out=P) == 1                        # out inside the gathered states
    assert pre_decay(nseq=0) == 0

    def bwd(**kw):
        a = dict(q=P, k=2 * P, v=3 * P, do=4 * P, cu=None, nseq=1, T=64, H=2, d=64, B=64, dt=la.LA_FP32, init=None,
                 decay=9 * P, dq=5 * P, dk=6 * P, dv=7 * P, dinit=None, ws=8 * P, wsb=BIG)
        a.update(kw)
        return la.la_prefill_backward_decay(a["q"], a["k"], a["v"], a["do"], a["cu"], a["nseq"], a["T"], a["H"],
                                            a["d"], a["B"], a["dt"], a["init"], a["decay"], a["dq"], a["dk"], a["dv"],
                                            a["dinit"], a["ws"], a["wsb"], None)
    assert bwd(decay=None) == 1
    assert bwd(decay=9 * P + 2) == 3
    assert bwd(decay=5 * P) == 1                        # rates inside dq
    assert bwd(dq=P) == 1                               # dq aliases q
    assert bwd(decay=8 * P + 4096) == 1                 # rates inside the workspace
    assert bwd(dinit=10 * P, decay=10 * P + 64) == 1    # rates inside dinit_state
    assert bwd(B=96) == 2
    assert bwd(wsb=16) == 4
    assert la.la_prefill_backward_decay_workspace_size(4096, 2, 4, 64, 64, la.LA_FP32) > 0
    assert la.la_prefill_backward_decay_workspace_size(4096, 2, 4, 64, 48, la.LA_FP32) == 0

    def fm(**kw):
        a = dict(x=P, y=2 * P, n=100, dt=la.LA_BF16, alpha=0.3)
        a.update(kw)
        return la.la_feature_map(a["x"], a["y"], a["n"], a["dt"], a["alpha"], None)
    assert fm(n=-1) == 1
    assert fm(dt=3) == 2
    assert fm(x=None) == 1
    assert fm(x=P + 8) == 3
    assert fm(y=P + 64) == 1                            # partial overlap (in place is y == x)
    assert fm(alpha=float("nan")) == 1
    assert fm(alpha=float("inf")) == 1
    assert fm(n=0) == 0


def test_workspace_sizes(lib):
    assert la.la_prefill_workspace_size(32768, 1, 64, 128, 256, la.LA_BF16) > 0
    assert la.la_prefill_workspace_size(32768, 1, 64, 100, 256, la.LA_BF16) == 0
    assert la.la_prefill_workspace_size(-1, 1, 64, 128, 256, la.LA_BF16) == 0
    a = la.la_prefill_workspace_size(1000, 1, 4, 128, 256, la.LA_BF16)
    b = la.la_prefill_workspace_size(2000, 1, 4, 128, 256, la.LA_BF16)
    assert b > a
    assert la.la_state_workspace_size(4096, 2, 4, 64, la.LA_FP32) > 0
    assert la.la_prefill_workspace_size(100, 1, 1, 64, 64, la.LA_FP32) % 256 == 0
    assert la.la_prefill_decay_workspace_size(32768, 1, 64, 128, 256, la.LA_BF16) > 0
    assert la.la_prefill_decay_workspace_size(32768, 1, 64, 128, 48, la.LA_BF16) == 0
    assert la.la_state_decay_workspace_size(4096, 2, 4, 64, la.LA_FP32) > 0


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    import importlib
    monkeypatch.setattr(la, "_LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(la, "_lib", None)
    with pytest.raises(la.LightningError):
        la.load_library()


def test_decay_conveniences_reject_host_tensors():
    """The decay and feature-map conveniences take device tensors only; host tensors raise
    (the library has no CPU path)."""
    import torch
    x = torch.zeros(8, 2, 16)
    rates = torch.ones(2)
    for call in (lambda: la.prefill_decay(x, x, x, rates),
                 lambda: la.state_decay(x, x, rates),
                 lambda: la.decode_step_decay(x, x, x, torch.zeros(8, 2, 16, 16), rates),
                 lambda: la.feature_map(x),
                 lambda: la.state_exclusive_prefix_decay(torch.zeros(2, 1, 2, 16, 16),
                                                         torch.zeros(2, 1, dtype=torch.int32), 1, rates)):
        with pytest.raises(la.LightningError):
            call()
