"""Data-parallel e-means (README "Several GPUs", DistributedEmeans) on one GPU.

The library's data-parallel step leaves each rank's per-cluster statistics, adds
them across ranks with an NCCL all-reduce and applies the EMA from the sums. With
one rank that exchange is the identity, and fp64 sums of bf16 rows are exact, so
a one-rank run must equal the single-GPU run bit for bit: batch order, labels,
per-pass errors, revivals, closing mean. (Several ranks need several GPUs; the
protocol itself is checked on gloo ranks in tests/test_dp_gloo.py.)
"""

import numpy as np
import pytest
import torch

from datagen import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def em():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mini_ema_means_b200

    return mini_ema_means_b200


def _one_rank(em, model):
    model.dp_init_id(1, 0, em.dp_unique_id())
    assert model.dp_world() == (1, 0)


def _train(em, x, d, k, dp, epochs, **opts):
    m = em.Model(d, k, seed=11, **opts)
    if dp:
        _one_rank(em, m)
    m.train(x.cuda(), epochs=epochs)
    c = torch.empty(k, d)
    m.centroids(c)
    lab = torch.empty(x.shape[0], dtype=torch.int64)
    m.labels(lab)
    out = (c, lab, m.obj(), m.stats()["n_splits"], m.stats()["rows_assigned"])
    m.close()
    return out


@pytest.mark.parametrize("d,k,epochs,opts", [
    (64, 50, 2.5, dict(graphs=1)),
    (96, 300, 1.5, dict(graphs=0, revival="resample")),
    (768, 64, 1.0, dict(graphs=1, spherical=1)),
    (40, 100, 2.0, dict(graphs=1, prefetch=0, batch_size=512)),
])
def test_one_rank_run_equals_single_gpu(em, d, k, epochs, opts):
    x = synth.hand_shape(4000, d, max(2, k // 2), seed=d + k, normalized=bool(opts.get("spherical")))
    ref = _train(em, x, d, k, False, epochs, **opts)
    got = _train(em, x, d, k, True, epochs, **opts)
    assert torch.equal(got[0], ref[0]), "centroids differ"
    assert torch.equal(got[1], ref[1]), "last-pass labels differ"
    assert np.array_equal(got[2], ref[2]), "per-pass errors differ"
    assert got[3:] == ref[3:]


def test_one_rank_lloyd_equals_single_gpu(em):
    x = synth.hand_shape(5000, 48, 20, seed=3)
    cs = []
    for dp in (False, True):
        m = em.Model(48, 40, seed=2)
        if dp:
            _one_rank(em, m)
        m.lloyd(x.cuda(), 8)
        c = torch.empty(40, 48)
        m.centroids(c)
        cs.append((c, m.mse(x.cuda())))
        m.close()
    assert torch.equal(cs[0][0], cs[1][0]) and cs[0][1] == cs[1][1]


def test_data_parallel_argument_errors(em):
    m = em.Model(32, 10, seed=1)
    uid = em.dp_unique_id()
    with pytest.raises(em.EmeansError):
        m.dp_init_id(2, 2, uid)  # rank out of range: refused before any communication
    _one_rank(em, m)
    x = synth.hand_shape(1000, 32, 8, seed=1)
    m.begin(x.cuda(), epochs=1.0)
    with pytest.raises(em.EmeansError):
        m.dp_init_id(1, 0, uid)  # not during a run
    m.finalize()
    m.close()


@pytest.mark.parametrize("d,k,epochs,batch", [(64, 50, 2.0, 512), (264, 120, 1.5, None)])
def test_one_rank_statistics_path_against_the_oracle(em, d, k, epochs, batch):
    """The data-parallel statistics path (this rank's sums and counts into the
    exchange buffer, the all-reduce, the update from the buffer) checked against
    the fp64 oracle itself, step by step under teacher forcing, not only against the
    single-GPU run: batch order, labels, N, S and c after every step, revivals."""
    from oracle import emeans_oracle as O
    from tests.helpers import teacher_forced_run

    x = synth.hand_shape(3000, d, max(2, k // 2), seed=d + k + 1)
    xq = O.search_copy_of_data(x.numpy())
    opts = dict(auto_revive=0, revival="split")
    if batch:
        opts["batch_size"] = batch
    m = em.Model(d, k, seed=13, **opts)
    _one_rank(em, m)
    orc = O.EmeansOracle(d, k, seed=13, revival="split", batch_size=batch)
    res = teacher_forced_run(m, orc, x.cuda(), xq, epochs, "split")
    assert res["rows"] == int(round(epochs * 3000))
    m.close()
