"""Data-parallel e-means on two CPU ranks (gloo), at the level of the oracle.

The method shards by batch rows: every rank assigns its share of each mini-batch,
computes the per-cluster counts and sums of its rows, the ranks add them with one
all-reduce of k (d + 1) values, and every rank applies the same EMA update and the
same revival check (the revival draws are keyed by seed, step and cluster, so no
further exchange is needed). These tests check that protocol against the
single-process oracle run, that the ranks stay bit-identical, and the bench's
aggregation of timings and row counts over ranks.
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


def _dp_worker(rank, world, port, out_dir, k, epochs, batch, plant=None):
    """One rank of the protocol. `plant` breaks the exchange on purpose (the checks
    must then fail): "no_reduce" skips the all-reduce, "sums_not_reduced" adds the
    counts but keeps each rank's own sums."""
    _init(rank, world, port)
    try:
        xq = _data()
        orc = O.EmeansOracle(xq.shape[1], k, seed=5, batch_size=batch)
        orc.begin(xq, epochs)

        def shard_stats(rows, labels, kk):
            # this rank's share of the batch, then one all-reduce of (n_j, s_j)
            part = np.array_split(np.arange(len(rows)), world)[rank]
            n_j, s_j = O.batch_stats(rows[part], labels[part], kk)
            buf = torch.from_numpy(np.concatenate([n_j[:, None], s_j], axis=1))
            if plant == "sums_not_reduced":
                counts = buf[:, :1].contiguous()
                dist.all_reduce(counts)
                buf[:, :1] = counts
            elif plant != "no_reduce":
                dist.all_reduce(buf)
            return buf[:, 0].numpy().copy(), buf[:, 1:].numpy().copy()

        while not orc.done:
            orc.step(stats=shard_stats)
        c = orc.finalize()
        np.save(os.path.join(out_dir, f"c{rank}.npy"), c)
        np.save(os.path.join(out_dir, f"N{rank}.npy"), orc.N)
        np.save(os.path.join(out_dir, f"splits{rank}.npy"), np.array([orc.n_splits]))
    finally:
        dist.destroy_process_group()


def _check_against_single_process(tmp_path, k, epochs, batch):
    c0, c1 = np.load(tmp_path / "c0.npy"), np.load(tmp_path / "c1.npy")
    N0, N1 = np.load(tmp_path / "N0.npy"), np.load(tmp_path / "N1.npy")
    # the ranks hold the same model, bit for bit
    assert np.array_equal(c0, c1) and np.array_equal(N0, N1)
    # and it is the single-process run up to the order of the fp64 sums
    xq = _data()
    ref = O.EmeansOracle(xq.shape[1], k, seed=5, batch_size=batch)
    c_ref, _ = ref.train(xq, epochs)
    np.testing.assert_allclose(c0, c_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(N0, ref.N, rtol=1e-12, atol=1e-12)
    assert int(np.load(tmp_path / "splits0.npy")[0]) == ref.n_splits


@pytest.mark.parametrize("k,epochs,batch", [(24, 2.0, 128), (40, 1.5, 96)])
def test_data_parallel_step_matches_single_process(tmp_path, k, epochs, batch):
    world = 2
    mp.spawn(_dp_worker, args=(world, _free_port(), str(tmp_path), k, epochs, batch), nprocs=world, join=True)
    _check_against_single_process(tmp_path, k, epochs, batch)


@pytest.mark.parametrize("plant", ["no_reduce", "sums_not_reduced"])
def test_checks_catch_a_broken_exchange(tmp_path, plant):
    world, k, epochs, batch = 2, 24, 2.0, 128
    mp.spawn(_dp_worker, args=(world, _free_port(), str(tmp_path), k, epochs, batch, plant), nprocs=world,
             join=True)
    with pytest.raises(AssertionError):
        _check_against_single_process(tmp_path, k, epochs, batch)


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
