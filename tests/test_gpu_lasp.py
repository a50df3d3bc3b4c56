"""LASP+ sequence parallelism run end to end on the GPU: lasp_prefill with the
library's own kernels (LibraryOps: la_state_from_prefill / la_state_decay, the
exclusive prefix kernels, la_prefill / la_prefill_decay) in 2 processes.

The two ranks share cuda:0 and exchange their segment states through a gloo
group (the driver gathers host copies under gloo). Their kernels never wait on
each other: the only exchange is the collective on the host. Every rank's rows
and the returned final state are compared with the fp64 oracle run on the
whole sequences.

Shapes: bf16, d = 128, B = 256, 32 heads and two sequences (1000 and 777
tokens) cut unevenly into two segments, so every segment state comes from the
tensor-core state pass and every segment prefill from the on-chip-state
tensor-core kernel (2 x 2 x 32 = 128 work items). Tolerances as in the parity
tests: O within 1e-2 of max|O_ref|; final states within 1e-4 of max|S_ref|
without decay, 5e-3 with decay (the tensor-core decay path rounds its weighted
values to bf16).
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

pytestmark = pytest.mark.gpu

LENGTHS = [1000, 777]
CUTS = [[0, 613, 1000], [0, 300, 777]]       # segment boundaries of each sequence (2 ranks)
H, D, B = 32, 128, 256
RATES_SEED = 97


def _inputs():
    T = sum(LENGTHS)
    q, k, v = wl.qkv(T, H, D, torch.bfloat16, seed=31)
    g = torch.Generator().manual_seed(32)
    init = torch.randn((len(LENGTHS), H, D, D), generator=g) * 0.05
    decay = wl.decay_rates(H)
    return q, k, v, init, decay


def _segment(x, r):
    starts = np.cumsum([0] + LENGTHS[:-1])
    return torch.cat([x[s0 + c[r]: s0 + c[r + 1]] for s0, c in zip(starts, CUTS)], dim=0)


def _worker(rank, world, port, outdir, with_decay):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    try:
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        import causal_linear_attention_02_b200 as la
        from causal_linear_attention_02_b200.lasp import lasp_prefill
        la.load_library()
        q, k, v, init, decay = _inputs()
        seg = [c[rank + 1] - c[rank] for c in CUTS]
        cu = torch.tensor(np.cumsum([0] + seg), dtype=torch.int32, device=dev)
        qr, kr, vr = (_segment(x, rank).to(dev) for x in (q, k, v))
        o, st = lasp_prefill(qr, kr, vr, cu, B=B, init_state=init.to(dev), return_state=True,
                             decay=decay.to(dev) if with_decay else None)
        torch.cuda.synchronize(dev)
        status = la.device_status()
        np.save(os.path.join(outdir, f"o{rank}.npy"), o.float().cpu().numpy())
        np.save(os.path.join(outdir, f"s{rank}.npy"), st.cpu().numpy())
        np.save(os.path.join(outdir, f"status{rank}.npy"), np.array([status]))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("with_decay", [False, True], ids=["plain", "decay"])
def test_lasp_prefill_library_ops_on_gpu(with_decay):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from causal_linear_attention_02_b200 import build
    build.build()
    world = 2
    with tempfile.TemporaryDirectory() as outdir:
        mp.spawn(_worker, args=(world, _free_port(), outdir, with_decay), nprocs=world, join=True)
        q, k, v, init, decay = _inputs()
        f = lambda t: t.float().double().numpy()
        cu = wl.cu_seqlens(LENGTHS).numpy()
        if with_decay:
            ref, ref_state = oracle.decay_recurrent(f(q), f(k), f(v), decay.double().numpy(), cu,
                                                    init=init.double().numpy(), return_state=True)
            state_tol = 5e-3
        else:
            ref, ref_state = oracle.recurrent(f(q), f(k), f(v), cu, init=init.double().numpy(), return_state=True)
            state_tol = 1e-4
        for r in range(world):
            assert int(np.load(os.path.join(outdir, f"status{r}.npy"))[0]) == 0, f"rank {r} device status"
            o = np.load(os.path.join(outdir, f"o{r}.npy"))
            want = _segment(torch.from_numpy(ref), r).numpy()
            err = np.abs(o - want).max() / np.abs(want).max()
            assert err <= 1e-2, f"rank {r} rows: {err:.3e}"
            st = np.load(os.path.join(outdir, f"s{r}.npy"))
            err = np.abs(st - ref_state).max() / np.abs(ref_state).max()
            assert err <= state_tol, f"rank {r} final state: {err:.3e}"
