"""Host side of the context-parallel decode, on CPU: the position ranges the
ranks hold partition every sequence, the partials are gathered in rank order
over a 2-rank gloo group, and the log-sum-exp merge of per-range softmaxes
equals the softmax over the whole sequence ("Gated MLA 计算公式" §二)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cp():
    # the module only marshals; importing it needs the library file, not a GPU
    from gated_mla_b200 import context_parallel
    return context_parallel


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_ranges_partition_each_sequence_on_tile_boundaries(world):
    cp = _cp()
    for n in (0, 1, 127, 128, 129, 1000, 131072, 5 * 128 + 3):
        ranges = [cp.shard_ranges(n, world, r) for r in range(world)]
        assert ranges[0][0] == 0 and ranges[-1][1] == n
        for (s0, e0), (s1, e1) in zip(ranges, ranges[1:]):
            assert e0 == s1
        for s, e in ranges:
            assert s <= e and s % 128 == 0


def _lse_partial(z, C, s, e):
    """One rank's share: normalised weighted sum over [s, e) and its log-sum-exp."""
    if e <= s:
        return np.zeros(C.shape[1]), -np.inf
    zz = z[s:e]
    m = zz.max()
    w = np.exp(zz - m)
    return (w @ C[s:e]) / w.sum(), m + np.log(w.sum())


def _rank(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from gated_mla_b200 import context_parallel as cp
        rng = np.random.default_rng(0)                      # the same problem on every rank
        L, dc = 1000, 8
        z = rng.standard_normal(L) * 3.0
        C = rng.standard_normal((L, dc))
        s, e = cp.shard_ranges(L, world, rank)
        o, lse = _lse_partial(z, C, s, e)
        part = torch.tensor(np.concatenate([o, [lse, 0, 0, 0]]), dtype=torch.float64)
        allp = cp.gather_partials(part).numpy()             # [world, dc + 4], rank order
        lses = allp[:, dc]
        M = lses.max()
        w = np.exp(lses - M)
        merged = (w[:, None] * allp[:, :dc]).sum(0) / w.sum()
        a = np.exp(z - z.max())
        full = (a / a.sum()) @ C
        q.put((rank, float(np.max(np.abs(merged - full))), allp[:, dc].tolist()))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_gathered_lse_merge_equals_the_whole_softmax_on_two_ranks():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, err, lses in got:
        assert err < 1e-12
    assert got[0][2] == got[1][2]                            # both ranks see the same gathered partials
