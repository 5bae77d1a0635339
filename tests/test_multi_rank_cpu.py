"""World-size-2 tests of the multi-rank host logic on CPU (gloo).

Each rank takes its shard of a packed batch (sequence ranges) or of the heads,
computes it independently (the float64 oracle stands in for the per-rank GPU
call, since these run without a GPU), and the gathered shards must equal the
unsharded result exactly: the path shards with no data-path collective.  The
max-over-ranks timing reduction bench.py uses is checked the same way.
"""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_delta_rule_159_b200 import shard


def _free_port():
    """A rendezvous for the ranks: a fresh file (no TCP port, so parallel test workers cannot
    collide)."""
    import tempfile
    fd, path = tempfile.mkstemp(prefix="gdn2_rdzv_")
    os.close(fd)
    os.unlink(path)
    return path


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
    dist.init_process_group("gloo", init_method=f"file://{port}", rank=rank, world_size=world)
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


# ----------------------------------------------------------------- sequence parallelism across ranks
class _OracleSegmentOps:
    """The three per-rank calls of gdn2.chunk_fwd_seq_ranks computed by the float64 oracle
    (these tests run without a GPU; the library's own calls are checked on the GPU)."""

    @staticmethod
    def _run(q, k, v, log_a, b, w, S0):
        import oracle
        N, L, H, d = q.shape
        flat = lambda t: None if t is None else t.reshape((N * L,) + tuple(t.shape[2:])).double().numpy()  # noqa: E731
        cu = np.arange(N + 1, dtype=np.int64) * L
        o, S = oracle.gdn2_fwd(flat(q), flat(k), flat(v), flat(log_a), flat(b), flat(w),
                               S0=None if S0 is None else S0.double().numpy(), cu_seqlens=cu)
        return torch.from_numpy(o.reshape(N, L, H, -1)), torch.from_numpy(S)

    @staticmethod
    def segment_maps(q, k, v, log_a, b, w, S0, **flags):
        N, L, H, d = q.shape
        o, G = _OracleSegmentOps._run(q, k, v, log_a, b, w, S0)
        ident = torch.eye(d, dtype=torch.float64).expand(N, H, d, d).contiguous()
        _, F = _OracleSegmentOps._run(q, k, torch.zeros_like(v), log_a, b, w, ident)
        return o, F, G

    @staticmethod
    def affine_prefix(F_all, G_all, seg):
        S, start = torch.zeros_like(F_all[0]), None
        for j in range(F_all.shape[0]):
            if j == seg:
                start = S.clone()
            S = F_all[j] @ S + G_all[j]
        return start, S

    @staticmethod
    def segment_correct(q, k, log_a, b, w, start, o, **flags):
        N, L, H, _ = q.shape
        dv = o.shape[-1]
        o2, _ = _OracleSegmentOps._run(q, k, torch.zeros(N, L, H, dv, dtype=q.dtype), log_a, b, w, start)
        o += o2
        return o


def _seq_problem(N=2, T=48, H=2, d=4, seed=3):
    g = torch.Generator().manual_seed(seed)
    f = lambda *s: torch.randn(*s, generator=g, dtype=torch.float64)  # noqa: E731
    q, k, v = f(N, T, H, d), f(N, T, H, d), f(N, T, H, d)
    log_a = -0.3 * torch.rand(N, T, H, d, generator=g, dtype=torch.float64)
    b, w = torch.rand(N, T, H, d, generator=g, dtype=torch.float64), torch.rand(N, T, H, d, generator=g,
                                                                                 dtype=torch.float64)
    S0 = 0.1 * f(N, H, d, d)
    return (q, k, v, log_a, b, w), S0


def _seq_worker(rank, world, port, out_q):
    from gated_delta_rule_159_b200 import gdn2
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    dist.init_process_group("gloo", init_method=f"file://{port}", rank=rank, world_size=world)
    try:
        xs, S0 = _seq_problem()
        T = xs[0].shape[1]
        lo, hi = rank * T // world, (rank + 1) * T // world
        local = [x[:, lo:hi].contiguous() for x in xs]
        o, S_T = gdn2.chunk_fwd_seq_ranks(*local, S0, ops=_OracleSegmentOps)
        gathered = [None] * world
        dist.all_gather_object(gathered, (lo, hi, o, S_T))
        if rank == 0:
            # numpy arrays travel by value; a tensor's storage would be shared through a file
            # descriptor that the receiver can only fetch while this process still lives
            out_q.put([(a, z, oo.numpy(), ss.numpy()) for a, z, oo, ss in gathered])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_ranks_equal_unsplit(world):
    """Each rank holds a slice of every sequence; the gathered outputs and every rank's S_T
    equal the unsplit recurrence (only the (F, G) maps cross ranks)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_seq_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    gathered = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    xs, S0 = _seq_problem()
    o_ref, S_ref = _OracleSegmentOps._run(*xs, S0)
    o = torch.zeros_like(o_ref)
    for lo, hi, o_r, S_r in gathered:
        o_r, S_r = torch.from_numpy(o_r), torch.from_numpy(S_r)
        o[:, lo:hi] = o_r
        assert torch.allclose(S_r, S_ref, rtol=1e-10, atol=1e-12)
    assert torch.allclose(o, o_ref, rtol=1e-10, atol=1e-12)
