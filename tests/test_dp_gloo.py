"""Data-parallel e-means on CPU ranks (gloo), at the level of the oracle.

The pages' DistributedEmeans loop ([README] "Several GPUs"): every rank holds its
own rows and walks them in its own fresh order each pass; the recipe is that of
all ranks' rows; at each step every rank takes an even share of the batch
(positions [pos // W, (pos + B) // W) of its order), computes the per-cluster
counts and sums of its share, the ranks add them (with the batch error) in one
all-reduce, and every rank applies the same EMA update and the same revival check
(its draws are keyed by seed, step and cluster, so no further exchange is
needed). These tests check:
* a run on 2 and 3 gloo ranks against one process that replays every rank's share
  of every batch with no collective (and planted broken exchanges fail that);
* the library's host plan of each rank's batches (em_dp_schedule) against the
  oracle's protocol, step by step;
* the bench's aggregation of timings and row counts over ranks, the communicator
  id exchange and the FP8 converter over ranks.
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import emeans_oracle as O


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _data(n=1200, d=12, comps=10, seed=3):
    rng = np.random.default_rng(seed)
    mu = rng.normal(0, 4.0, size=(comps, d))
    x = mu[rng.integers(comps, size=n)] + rng.normal(size=(n, d))
    return O.search_copy_of_data(x.astype(np.float32))


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))


def _rank_rows(rank, n_local=600, d=12, comps=10):
    """Rank `rank`'s own rows: every rank holds a different share of one mixture."""
    return _data(n=n_local, d=d, comps=comps, seed=3 + 100 * rank)


def _dp_worker(rank, world, port, out_dir, k, epochs, batch, plant=None):
    """One rank of the pages' data-parallel loop ([README] "Several GPUs"), as the
    oracle runs it: own rows, own per-pass order, an even share of each batch, one
    all-reduce of (n_j, s_j, batch error) per step, rank 0's starting rows.
    `plant` breaks the protocol on purpose (the checks must then fail):
    "no_reduce" skips the all-reduce, "sums_not_reduced" adds the counts but keeps
    each rank's own sums, "rank_blind_order" gives every rank rank 0's order key."""
    _init(rank, world, port)
    try:
        xq = _rank_rows(rank)

        def all_reduce(v):
            buf = torch.from_numpy(np.array(v, dtype=np.float64))
            if plant == "sums_not_reduced":
                head = buf[:k].contiguous()
                dist.all_reduce(head)
                buf[:k] = head
            elif plant != "no_reduce":
                dist.all_reduce(buf)
            return buf.numpy().copy()

        orc = O.EmeansOracle(xq.shape[1], k, seed=5, batch_size=batch, world=world, rank=rank,
                             all_reduce=all_reduce)
        if plant == "rank_blind_order":
            orc.order_key = lambda p: p
        c0 = torch.from_numpy(xq[O.starting_rows(len(xq), k, 5)].copy())
        dist.broadcast(c0, src=0)  # rank 0's starting rows
        orc.begin(xq, epochs, start_centroids=c0.numpy())
        while not orc.done:
            orc.step()
        c = orc.finalize()
        np.save(os.path.join(out_dir, f"c{rank}.npy"), c)
        np.save(os.path.join(out_dir, f"N{rank}.npy"), orc.N)
        np.save(os.path.join(out_dir, f"obj{rank}.npy"), np.array(orc.obj))
        np.save(os.path.join(out_dir, f"splits{rank}.npy"), np.array([orc.n_splits]))
    finally:
        dist.destroy_process_group()


def _replay_all_ranks(world, k, epochs, batch):
    """One process replays every rank's share of every batch: rank r's rows are
    positions [pos // W, (pos + B) // W) of the order keyed by pass + r x 2^32 of
    its own rows; the batch's labels, counts and sums are computed over the union
    of the ranks' shares, with no collective at all."""
    xs = [_rank_rows(r) for r in range(world)]
    err = {}

    orc = O.EmeansOracle(xs[0].shape[1], k, seed=5, batch_size=batch, world=world, rank=0,
                         all_reduce=lambda v: np.concatenate([v[:-1], [err["total"]]]))

    def union_stats(_rows, _labels, kk):
        lo, hi = orc.batch_positions()
        parts = [x[O.pass_order(len(x), 5, orc.pass_index + (r << 32))[lo:hi]] for r, x in enumerate(xs)]
        rows = np.concatenate(parts)
        labels, best, _ = O.assign(rows, O.search_copy_of_centroids(orc.c))
        err["total"] = float(best.sum())
        return O.batch_stats(rows, labels, kk)

    orc.begin(xs[0], epochs)
    while not orc.done:
        orc.step(stats=union_stats)
    return orc.finalize(), orc


def _check_against_single_process(tmp_path, world, k, epochs, batch):
    c = [np.load(tmp_path / f"c{r}.npy") for r in range(world)]
    N = [np.load(tmp_path / f"N{r}.npy") for r in range(world)]
    # the ranks hold the same model, bit for bit
    assert all(np.array_equal(c[0], x) for x in c) and all(np.array_equal(N[0], x) for x in N)
    # and it is the one-process replay of every rank's rows, up to the order of the fp64 sums
    c_ref, ref = _replay_all_ranks(world, k, epochs, batch)
    np.testing.assert_allclose(c[0], c_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(N[0], ref.N, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(np.load(tmp_path / "obj0.npy"), ref.obj, rtol=1e-12)
    assert int(np.load(tmp_path / "splits0.npy")[0]) == ref.n_splits


@pytest.mark.parametrize("world,k,epochs,batch", [(2, 24, 2.0, 128), (2, 40, 1.5, 96), (3, 16, 2.5, 96)])
def test_data_parallel_run_matches_one_process_replay(tmp_path, world, k, epochs, batch):
    mp.spawn(_dp_worker, args=(world, _free_port(), str(tmp_path), k, epochs, batch), nprocs=world, join=True)
    _check_against_single_process(tmp_path, world, k, epochs, batch)


@pytest.mark.parametrize("plant", ["no_reduce", "sums_not_reduced", "rank_blind_order"])
def test_checks_catch_a_broken_exchange(tmp_path, plant):
    world, k, epochs, batch = 2, 24, 2.0, 128
    mp.spawn(_dp_worker, args=(world, _free_port(), str(tmp_path), k, epochs, batch, plant), nprocs=world,
             join=True)
    with pytest.raises(AssertionError):
        _check_against_single_process(tmp_path, world, k, epochs, batch)


@pytest.mark.parametrize("n_local,world,k,epochs,batch", [
    (600, 2, 24, 2.0, 128), (600, 2, 40, 1.5, 96), (600, 3, 16, 2.5, 96), (4096, 4, 64, 3.0, 0),
    (1000, 8, 10, 1.25, 64)])
def test_library_rank_schedule_is_the_oracles(em_lib, n_local, world, k, epochs, batch):
    """The library's host plan of a rank's batches (em_dp_schedule: the code em_step
    and the gather use) against the oracle's protocol, step by step: the pass, the
    positions of the rank's own order and that order's key."""
    em = em_lib
    for rank in range(world):
        orc = O.EmeansOracle(1, k, seed=5, batch_size=batch or None, law="throughput", world=world, rank=rank,
                             all_reduce=lambda v: v)
        xq = O.search_copy_of_data(np.random.default_rng(rank).standard_normal((n_local, 1)).astype(np.float32))
        orc.begin(xq, epochs, start_centroids=np.zeros((k, 1)))
        want = []
        while not orc.done:
            lo, hi = orc.batch_positions()
            want.append((orc.pass_index, lo, hi - lo, orc.order_key(orc.pass_index)))
            orc.step(auto_revive=False)
        got = em.dp_schedule(n_local, k, epochs, world, rank, len(want), law=0, batch_size=batch)
        assert [tuple(int(a[t]) for a in got) for t in range(len(want))] == want
        # each pass, the rank's positions cover its own rows exactly once (a fractional
        # last pass: its first rows)
        for p in set(w[0] for w in want):
            spans = sorted((w[1], w[1] + w[2]) for w in want if w[0] == p)
            assert spans[0][0] == 0 and all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            assert spans[-1][1] == (n_local if p < orc.r["epoch_rows"].__len__() - 1 else
                                    orc.r["epoch_rows"][-1] // world)


def test_library_rejects_a_batch_that_does_not_divide(em_lib):
    em = em_lib
    with pytest.raises(em.EmeansError) as e:
        em.dp_schedule(600, 24, 2.0, 3, 0, 1, batch_size=128)
    assert e.value.code == em.EM_E_INVAL
    with pytest.raises(em.EmeansError):
        em.dp_schedule(600, 24, 2.0, 2, 2, 1, batch_size=128)  # rank outside [0, world)


def _agg_worker(rank, world, port, out_dir):
    _init(rank, world, port)
    try:
        import bench

        ms, rows = (12.5, 1000) if rank == 0 else (17.25, 1500)
        ms_max, rows_all = bench.reduce_over_ranks(ms, rows, torch.device("cpu"), world)
        np.save(os.path.join(out_dir, f"agg{rank}.npy"), np.array([ms_max, rows_all]))
    finally:
        dist.destroy_process_group()


def test_bench_aggregates_max_time_and_total_rows(tmp_path):
    world = 2
    mp.spawn(_agg_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    for r in range(world):
        ms_max, rows_all = np.load(tmp_path / f"agg{r}.npy")
        assert ms_max == 17.25 and rows_all == 2500


def _id_worker(rank, world, port, out_dir):
    _init(rank, world, port)
    try:
        import mini_ema_means_b200 as em

        w, r, uid = em.exchange_dp_id()
        assert (w, r) == (world, rank) and len(uid) == em.EM_NCCL_ID_BYTES
        with open(os.path.join(out_dir, f"id{rank}.bin"), "wb") as f:
            f.write(uid)
    finally:
        dist.destroy_process_group()


def test_communicator_id_reaches_every_rank(tmp_path, em_lib):
    """Model.dp_init's first half on two gloo ranks: rank 0 makes the NCCL id (host
    code of the library) and every rank receives the same bytes."""
    world = 2
    mp.spawn(_id_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    ids = [open(tmp_path / f"id{r}.bin", "rb").read() for r in range(world)]
    assert ids[0] == ids[1] and len(ids[0]) == 128 and any(ids[0])


@pytest.fixture(scope="module")
def em_lib():
    import importlib.util

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("_b", os.path.join(root, "mini_ema_means_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()
    import mini_ema_means_b200

    return mini_ema_means_b200


def test_rank_orders_are_the_oracles_bijections(em_lib):
    """A data-parallel rank r walks its own rows in the library's order keyed by
    pass + r * 2^32 (rank 0: the single-GPU order); the host code of that order is
    the oracle's bijection for those keys too."""
    em = em_lib
    n = 7001
    idx = np.arange(n, dtype=np.int64)
    for rank, p in ((0, 0), (1, 0), (3, 2)):
        which = p + (rank << 32)
        lib = em.permutation(n, 1234, 2, which, idx)
        assert np.array_equal(lib, O.pass_order(n, 1234, which))
        assert np.array_equal(np.sort(lib), idx)
    assert not np.array_equal(em.permutation(n, 1234, 2, 1 << 32, idx), em.permutation(n, 1234, 2, 0, idx))


def _fp8_worker(rank, world, port, out_dir):
    """One rank of the FP8 converter fit: the minimum and maximum of each dimension
    over this rank's first rows, combined over the ranks, then the converter of
    that range."""
    _init(rank, world, port)
    try:
        xq = _data(n=700 + 300 * rank, d=9, seed=20 + rank) * (1.0 + rank)
        first = np.asarray(xq[:O.FP8_CALIBRATION_ROWS], dtype=np.float32)
        lo, hi = torch.from_numpy(first.min(axis=0)), torch.from_numpy(first.max(axis=0))
        dist.all_reduce(lo, op=dist.ReduceOp.MIN)
        dist.all_reduce(hi, op=dist.ReduceOp.MAX)
        shift, scale = O.fp8_calibrate(np.vstack([lo.numpy(), hi.numpy()]))
        np.save(os.path.join(out_dir, f"fp8_{rank}.npy"), np.concatenate([shift.astype(np.float64), [scale]]))
    finally:
        dist.destroy_process_group()


def test_fp8_converter_over_ranks_is_the_fit_on_all_ranks_first_rows(tmp_path):
    """The FP8 converter reading for several ranks: fitted on each rank's first
    rows together (the ranks' minima and maxima combined)."""
    world = 2
    mp.spawn(_fp8_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r0, r1 = np.load(tmp_path / "fp8_0.npy"), np.load(tmp_path / "fp8_1.npy")
    assert np.array_equal(r0, r1)
    rows = [_data(n=700 + 300 * r, d=9, seed=20 + r) * (1.0 + r) for r in range(world)]
    shift, scale = O.fp8_calibrate(np.vstack([x[:O.FP8_CALIBRATION_ROWS] for x in rows]))
    assert np.array_equal(r0[:-1], shift.astype(np.float64)) and r0[-1] == scale
