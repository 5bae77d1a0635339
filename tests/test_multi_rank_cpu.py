"""World-size-2 tests of the multi-rank host logic on CPU (gloo).

Each rank takes its shard of a packed batch (sequence ranges) or of the heads,
computes it independently (the float64 oracle stands in for the per-rank GPU
call, since these run without a GPU), and the gathered shards must equal the
unsharded result exactly: the path shards with no data-path collective.  The
max-over-ranks timing reduction bench.py uses is checked the same way.
"""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_delta_rule_159_b200 import shard


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _problem(seed=0):
    rng = np.random.default_rng(seed)
    lens = [7, 0, 33, 12, 5, 21]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    T, H, d = int(cu[-1]), 3, 4
    f = lambda *s: rng.standard_normal(s)  # noqa: E731
    q, k, v = f(T, H, d), f(T, H, d), f(T, H, d)
    la = -rng.uniform(0, 0.3, (T, H, d))
    b, w = rng.uniform(0, 1, (T, H, d)), rng.uniform(0, 1, (T, H, d))
    S0 = 0.1 * f(len(lens), H, d, d)
    return cu, (q, k, v, la, b, w), S0


def _worker(rank, world, port, mode, out_q):
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cu, xs, S0 = _problem()
        if mode == "sequences":
            lo, hi, t0, t1, lcu = shard.local_problem(cu, rank, world)
            o, S = oracle.gdn2_fwd(*(x[t0:t1] for x in xs), S0=S0[lo:hi], cu_seqlens=lcu) if hi > lo else \
                (np.zeros((0,) + xs[2].shape[1:]), np.zeros((0,) + S0.shape[1:]))
            piece = (lo, hi, t0, t1, o, S)
        else:
            h0, h1 = shard.head_range(xs[0].shape[1], rank, world)
            o, S = oracle.gdn2_fwd(*(x[:, h0:h1] for x in xs), S0=S0[:, h0:h1], cu_seqlens=cu)
            piece = (h0, h1, o, S)
        gathered = [None] * world
        dist.all_gather_object(gathered, piece)
        # bench.py's max-over-ranks timing reduction
        import torch
        t = torch.tensor([1.5 + rank], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            out_q.put((gathered, float(t.item())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode", ["sequences", "heads"])
def test_two_rank_shards_equal_unsharded(mode):
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, mode, q)) for r in range(2)]
    for p in procs:
        p.start()
    gathered, tmax = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cu, xs, S0 = _problem()
    o_ref, S_ref = oracle.gdn2_fwd(*xs, S0=S0, cu_seqlens=cu)
    o = np.zeros_like(o_ref)
    S = np.zeros_like(S_ref)
    if mode == "sequences":
        covered = []
        for lo, hi, t0, t1, og, Sg in gathered:
            o[t0:t1], S[lo:hi] = og, Sg
            covered += list(range(lo, hi))
        assert covered == list(range(len(cu) - 1))
    else:
        for h0, h1, og, Sg in gathered:
            o[:, h0:h1], S[:, h0:h1] = og, Sg
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(S, S_ref)
    assert tmax == 2.5


def test_sequence_ranges_balance_tokens():
    cu = [0, 10, 20, 30, 1000, 1010]
    r = shard.sequence_ranges(cu, 2)
    assert r[0][0] == 0 and r[-1][1] == 5 and r[0][1] == r[1][0]
    assert shard.sequence_ranges([0, 5], 3) == [(0, 0), (0, 1), (1, 1)]
    assert [shard.head_range(16, r, 3) for r in range(3)] == [(0, 6), (6, 11), (11, 16)]
