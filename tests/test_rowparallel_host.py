"""Row-parallel (d-split) tensor parallelism: the host logic on CPU ranks
(gloo, world size 2 and 3).

Each rank takes its slice of the input width from ``rowparallel_slices``,
computes its share, and ``row_parallel_norm_proj`` sums the shares with one
all-reduce and post-scales.  On CPU ranks the two library calls are replaced
(patched in each worker) by the oracle's statement of them, so what is
checked here is the plumbing:
slicing, the buffer layout ([M, ncols] products then [M] sums of squares),
the collective, and that every rank ends with the single-device result.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(M, d, N, swiglu):
    rng = np.random.default_rng(77)
    x = rng.standard_normal((M, d)) * np.exp(rng.uniform(-2, 2, (M, 1)))
    Wg = rng.standard_normal((d, N)) / np.sqrt(d)
    Wu = rng.standard_normal((d, N)) / np.sqrt(d)
    return x, Wg, Wu


def _worker(rank, world, port, swiglu, q, exchange="allreduce", M=4):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    sys.path.insert(0, ROOT)
    import oracle as O
    from rmsnorm_linear_projection_flashnorm_b200 import torch_api as T
    from rmsnorm_linear_projection_flashnorm_b200 import tp
    d, N = 384, 256
    x, Wg, Wu = _inputs(M, d, N, swiglu)
    W = O.interleave128(Wg, Wu) if swiglu else Wg
    k0, k1 = tp.rowparallel_slices(d, world, align=64)[rank]

    def partial_cpu(xl, Wl, ncols, scales=None, ws=None):
        acc, ssq = O.rowparallel_partial(xl.numpy(), Wl.numpy())
        assert acc.shape == (M, ncols)
        return torch.from_numpy(np.concatenate([acc.reshape(-1), ssq]))

    def post_cpu(part, M_, N_, d_total, eps, swiglu=False):
        p = part.numpy()
        ncols = 2 * N_ if swiglu else N_
        return torch.from_numpy(O.rowparallel_finish(p[:M_ * ncols].reshape(M_, ncols), p[M_ * ncols:], d_total, eps,
                                                     swiglu))

    T.norm_proj_partial, T.post_scale = partial_cpu, post_cpu   # this worker process only
    y = tp.row_parallel_norm_proj(torch.from_numpy(x[:, k0:k1].copy()), torch.from_numpy(W[k0:k1].copy()), N, 1e-6,
                                  d, swiglu=swiglu, exchange=exchange)
    q.put((rank, (k0, k1), y.numpy()))
    dist.destroy_process_group()


@pytest.mark.parametrize("world,swiglu,exchange,M", [
    (2, False, "allreduce", 4), (2, True, "allreduce", 4), (3, True, "allreduce", 4),
    (2, False, "reduce_scatter", 6), (3, True, "reduce_scatter", 6),
    (3, False, "reduce_scatter", 4),    # M not divisible by the world size: the all-reduce path
])
def test_row_parallel_exchange_gives_every_rank_the_full_result(world, swiglu, exchange, M):
    sys.path.insert(0, ROOT)
    import oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, swiglu, q, exchange, M)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted([q.get(timeout=120) for _ in range(world)], key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    d, N = 384, 256
    x, Wg, Wu = _inputs(M, d, N, swiglu)
    want = O.norm_proj_swiglu(x, np.ones(d), Wg, Wu, 1e-6) if swiglu else O.norm_proj(x, np.ones(d), Wg, 1e-6)
    spans = [s for _, s, _ in out]
    assert spans[0][0] == 0 and spans[-1][1] == d
    assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
    for _, _, y in out:
        assert np.max(np.abs(y - want) / (1 + np.abs(want))) < 1e-12


def test_rowparallel_slices():
    from rmsnorm_linear_projection_flashnorm_b200 import tp
    assert tp.rowparallel_slices(4096, 8) == [(512 * r, 512 * (r + 1)) for r in range(8)]
    s = tp.rowparallel_slices(5120, 3, align=128)
    assert s[0][0] == 0 and s[-1][1] == 5120 and all(a % 128 == 0 and b % 128 == 0 for a, b in s)
    assert max(b - a for a, b in s) - min(b - a for a, b in s) <= 128
    with pytest.raises(ValueError):
        tp.rowparallel_slices(128, 3, align=64)
    with pytest.raises(ValueError):
        tp.rowparallel_slices(100, 2, align=64)
