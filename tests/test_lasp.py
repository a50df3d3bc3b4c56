"""Sequence parallelism (LASP+) over several ranks: the driver's collective
plumbing on CPU (gloo, one process per rank), checked against the oracle on
the whole sequences, with and without a decay rate per head.

The three compute steps of ``lasp_prefill`` (segment state, exclusive prefix,
prefill from a state) are passed in as oracle-backed ops here, so the test
runs without a GPU; the library's kernels for the same steps are checked on
the GPU in test_gpu_parity.py.
"""
import os
import socket
import tempfile
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import workloads as wl


class OracleOps:
    """fp64 CPU stand-ins for the library's three LASP+ steps (decay: the per-head rates, or None)."""

    @staticmethod
    def segment_state(k, v, cu, decay=None):
        if decay is not None:
            return torch.from_numpy(oracle.decay_state(k.numpy(), v.numpy(), decay.numpy(), cu.numpy()))
        return torch.from_numpy(oracle.state(k.numpy(), v.numpy(), cu.numpy()))

    @staticmethod
    def exclusive_prefix(gathered, rank, init, seg_lens=None, decay=None):
        if decay is None:
            s = gathered[:rank].sum(0)
            return s if init is None else s + init
        # the state before rank `rank`'s segment: run the earlier segments' states forward, each
        # discounted by lambda to the power of its segment's length before the next is added
        lam = decay.double().numpy()[None, :, None, None]              # [1, H, 1, 1]
        acc = np.zeros(gathered.shape[1:]) if init is None else init.double().numpy().copy()
        for r in range(rank):
            n = seg_lens[r].numpy().astype(np.float64)[:, None, None, None]   # [nseq, 1, 1, 1]
            acc = lam ** n * acc + gathered[r].double().numpy()
        return torch.from_numpy(acc)

    @staticmethod
    def prefill(q, k, v, cu, B, init, out, decay=None):
        if decay is not None:
            return torch.from_numpy(oracle.decay_blocked(q.numpy(), k.numpy(), v.numpy(), decay.numpy(), B,
                                                         cu.numpy(), init=init.numpy()))
        return torch.from_numpy(oracle.blocked(q.numpy(), k.numpy(), v.numpy(), B, cu.numpy(), init=init.numpy()))


def _case(world, seed):
    """Two sequences, each cut into `world` uneven contiguous segments."""
    rng = np.random.default_rng(seed)
    lengths = [301, 190]
    H, d, B = 2, 8, 16
    T = sum(lengths)
    q, k, v = (rng.standard_normal((T, H, d)) / np.sqrt(d) for _ in range(3))
    init = rng.standard_normal((len(lengths), H, d, d)) * 0.1
    cuts = []                           # cuts[s] = segment boundaries of sequence s
    for L in lengths:
        inner = np.sort(rng.choice(np.arange(1, L), size=world - 1, replace=False))
        cuts.append([0, *inner.tolist(), L])
    return lengths, H, d, B, q, k, v, init, cuts


def _segment(arr, lengths, cuts, r):
    """Rank r's packed rows: the r-th segment of every sequence, in sequence order."""
    starts = np.cumsum([0] + lengths[:-1])
    parts = [arr[s0 + c[r]: s0 + c[r + 1]] for s0, c in zip(starts, cuts)]
    return np.concatenate(parts, axis=0)


def _worker(rank, world, port, seed, outdir, with_decay=False):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from causal_linear_attention_02_b200.lasp import lasp_prefill
        lengths, H, d, B, q, k, v, init, cuts = _case(world, seed)
        seg_len = [c[rank + 1] - c[rank] for c in cuts]
        cu = torch.tensor(np.cumsum([0] + seg_len), dtype=torch.int32)
        qr, kr, vr = (torch.from_numpy(_segment(a, lengths, cuts, rank)) for a in (q, k, v))
        decay = torch.from_numpy(np.array([0.7, 0.97])) if with_decay else None
        o, st = lasp_prefill(qr, kr, vr, cu, B=B, init_state=torch.from_numpy(init), return_state=True,
                             decay=decay, ops=OracleOps)
        np.save(os.path.join(outdir, f"o{rank}.npy"), o.numpy())
        np.save(os.path.join(outdir, f"s{rank}.npy"), st.numpy())
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("with_decay", [False, True], ids=["plain", "decay"])
@pytest.mark.parametrize("world", [2, 3])
def test_lasp_prefill_matches_whole_sequences(world, with_decay):
    seed = 40 + world
    with tempfile.TemporaryDirectory() as outdir:
        mp.spawn(_worker, args=(world, _free_port(), seed, outdir, with_decay), nprocs=world, join=True)
        lengths, H, d, B, q, k, v, init, cuts = _case(world, seed)
        cu = wl.cu_seqlens(lengths).numpy()
        if with_decay:
            lam = np.array([0.7, 0.97])
            ref, ref_state = oracle.decay_recurrent(q, k, v, lam, cu, init=init, return_state=True)
        else:
            ref = oracle.recurrent(q, k, v, cu, init=init)
            ref_state = oracle.state(k, v, cu, init=init)
        for r in range(world):
            o = np.load(os.path.join(outdir, f"o{r}.npy"))
            want = _segment(ref, lengths, cuts, r)
            np.testing.assert_allclose(o, want, rtol=0, atol=1e-10 * np.abs(ref).max())
            st = np.load(os.path.join(outdir, f"s{r}.npy"))
            np.testing.assert_allclose(st, ref_state, rtol=0, atol=1e-10 * np.abs(ref_state).max())


def test_segments_cover_sequences():
    """The test's own split: every row of every sequence lands on exactly one rank."""
    lengths, H, d, B, q, k, v, init, cuts = _case(3, 7)
    rows = np.arange(sum(lengths))[:, None, None] * np.ones((1, H, d))
    got = np.concatenate([_segment(rows, lengths, cuts, r)[:, 0, 0] for r in range(3)])
    assert sorted(got.tolist()) == list(range(sum(lengths)))
