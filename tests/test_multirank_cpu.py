"""The multi-rank host logic of bench.py on CPU: two gloo ranks, max-over-ranks timing and the
whole-job (weak-scaling) rate. The data path has no collective; only these reductions cross ranks."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    import bench

    local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
    m = bench.max_over_ranks(local_ms, dist, "cpu")
    rate = bench.whole_job_rate(1000, 4, world, m)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, m, rate))


def test_two_ranks_max_time_and_weak_scaling_rate():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, m, rate in res:
        assert m == 15.0
        assert rate == pytest.approx(1000 * 4 * 2 / 0.015)


def test_single_rank_needs_no_process_group():
    import bench

    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5


# ------------------------------------------------------------------------------------------------
# the two partitions of parameter_space_moe_swimba_b200.parallel, with the oracle standing in for
# the kernels (gloo, world size 2)
# ------------------------------------------------------------------------------------------------

def test_batch_shards_and_sequence_pieces_cover_everything_once():
    from parameter_space_moe_swimba_b200.parallel import batch_shard, sequence_piece

    for B in [1, 3, 8, 9]:
        for world in [1, 2, 3, 8]:
            got = [batch_shard(B, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == B
            assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
            sizes = [b - a for a, b in got]
            assert max(sizes) - min(sizes) <= 1
    for L in [1, 15, 16, 45, 4096, 65536, 65537]:
        for world in [1, 2, 3, 8]:
            got = [sequence_piece(L, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == L
            assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
            assert all(b % 16 == 0 for _, b in got[:-1])  # cuts on whole 16-token chunks


def _problem(L=45, Bsz=2, D=6, N=4, E=5, k=2, seed=3):
    import numpy as np

    rng = np.random.default_rng(seed)
    x = rng.standard_normal((Bsz, L, D))
    z = rng.standard_normal((Bsz, L, D))
    dt = rng.normal(-2, 1, (Bsz, L, D))
    Bm = rng.standard_normal((Bsz, L, N))
    Cm = rng.standard_normal((Bsz, L, N))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(Bsz * L)]).reshape(Bsz, L, k).astype(np.int32)
    g = rng.random((Bsz, L, k))
    g /= g.sum(-1, keepdims=True)
    A = -np.exp(rng.uniform(-1, 3, (E, D, N)))
    Dsk = rng.standard_normal(D)
    h0 = rng.standard_normal((Bsz, D, N))
    return x, z, dt, Bm, Cm, idx, g, A, Dsk, h0


class _OracleOps:
    """The sequence split's steps on the fp64 oracle (CPU tensors)."""

    def __init__(self, A, Dsk):
        self.A, self.Dsk = A, Dsk

    def summary(self, piece):
        from oracle import swimba_oracle as O

        x, z, dt, Bm, Cm, idx, g = piece
        hz, ld = O.scan_summary(x, dt, Bm, idx, g, self.A)
        return torch.from_numpy(hz), torch.from_numpy(ld)

    def chain(self, hz_all, ld_all, h0):
        from oracle import swimba_oracle as O

        return torch.from_numpy(O.chain_summaries(hz_all.numpy(), ld_all.numpy(), h0=h0))

    def scan(self, piece, h_start):
        from oracle import swimba_oracle as O

        x, z, dt, Bm, Cm, idx, g = piece
        return O.selective_scan(x, z, dt, Bm, Cm, idx, g, self.A, self.Dsk, h0=h_start.numpy())


def _split_worker(rank, world, port, q, mode):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    from oracle import swimba_oracle as O
    from parameter_space_moe_swimba_b200 import parallel as PAR

    x, z, dt, Bm, Cm, idx, g, A, Dsk, h0 = _problem()
    if mode == "sequence":
        a, b = PAR.sequence_piece(x.shape[1], world, rank)
        piece = tuple(v[:, a:b] for v in (x, z, dt, Bm, Cm, idx, g))
        (y, out, hT, _), h_end = PAR.sequence_parallel_scan(_OracleOps(A, Dsk), piece, dist, h0=h0)
        q.put((rank, y, out, hT, h_end.numpy()))
    else:
        a, b = PAR.batch_shard(x.shape[0], world, rank)
        y, out, hT, _ = O.selective_scan(x[a:b], z[a:b], dt[a:b], Bm[a:b], Cm[a:b], idx[a:b], g[a:b], A, Dsk,
                                         h0=h0[a:b])
        q.put((rank, y, out, hT, None))
    dist.barrier()
    dist.destroy_process_group()


def _run_split(mode, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, q, mode)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    return res


def test_sequence_split_two_ranks_matches_the_whole_sequence():
    """Each rank summarises its piece, one all_gather exchanges the summaries, the chain gives each
    piece's start state, and the pieces scanned from there equal the single-rank scan of the whole
    sequence (fp64, 1e-12)."""
    import numpy as np

    from oracle import swimba_oracle as O

    res = _run_split("sequence")
    x, z, dt, Bm, Cm, idx, g, A, Dsk, h0 = _problem()
    y, out, hT, _ = O.selective_scan(x, z, dt, Bm, Cm, idx, g, A, Dsk, h0=h0)
    np.testing.assert_allclose(np.concatenate([r[1] for r in res], 1), y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(np.concatenate([r[2] for r in res], 1), out, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(res[-1][3], hT, rtol=1e-12, atol=1e-12)  # the last piece ends the sequence
    for r in res:  # every rank knows the final state
        np.testing.assert_allclose(r[4], hT, rtol=1e-12, atol=1e-12)


def test_batch_split_two_ranks_matches_the_whole_batch():
    import numpy as np

    from oracle import swimba_oracle as O

    res = _run_split("batch")
    x, z, dt, Bm, Cm, idx, g, A, Dsk, h0 = _problem()
    y, out, hT, _ = O.selective_scan(x, z, dt, Bm, Cm, idx, g, A, Dsk, h0=h0)
    np.testing.assert_array_equal(np.concatenate([r[1] for r in res], 0), y)
    np.testing.assert_array_equal(np.concatenate([r[3] for r in res], 0), hT)
