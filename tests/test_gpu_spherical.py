"""GPU parity of spherical e-means (faiss e-means README, "Spherical e-means"): unit
centroids, highest dot product, closing mean rescaled to norm 1, error 2 - 2 x
similarity. The CUDA path through the C ABI against EmeansOracle(spherical=True).
Tolerances: tests/helpers.py.
"""

import numpy as np
import pytest
import torch

from datagen import synth
from oracle import emeans_oracle as O
from tests.helpers import (CENTROID_REL, MSE_REL, LabelBook, assert_centroids_close, centroid_rel_err, gpu_state,
                           teacher_forced_run)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def em():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mini_ema_means_b200

    return mini_ema_means_b200


def _unit_data(n, d, ncomp, seed):
    return synth.hand_shape(n, d, ncomp, seed=seed, normalized=True)


@pytest.mark.parametrize("n,d,k,epochs,batch,revival", [
    (3000, 32, 40, 2.0, None, "split"),
    (4000, 64, 100, 1.5, 512, "resample"),
    (2600, 96, 257, 1.5, 256, "split"),
    (1500, 768, 64, 1.0, 256, "split"),     # d >= 256: near ties settled in fp64
    (2500, 264, 300, 1.25, None, "split"),  # ragged K chunk, three column tiles
    (2000, 8, 30, 2.0, None, "none"),
])
def test_spherical_teacher_forced(em, n, d, k, epochs, batch, revival):
    x = _unit_data(n, d, max(2, k // 2), seed=n + d)
    xq = O.search_copy_of_data(x.numpy())
    opts = dict(auto_revive=0, revival=revival, spherical=1)
    if batch:
        opts["batch_size"] = batch
    m = em.Model(d, k, seed=7, **opts)
    orc = O.EmeansOracle(d, k, seed=7, revival=revival, batch_size=batch, spherical=True)
    res = teacher_forced_run(m, orc, x.cuda(), xq, epochs, revival)
    m.finalize()
    orc.finalize()
    _, _, c, _ = gpu_state(m, k, d)
    assert_centroids_close(c, orc.c, "spherical closing mean")
    nrm = np.linalg.norm(c, axis=1)
    assert np.all(np.abs(nrm[nrm > 0] - 1.0) <= 1e-6)
    lab = torch.empty(n, dtype=torch.int64)
    m.labels(lab)
    assert np.array_equal(lab.numpy(), orc.labels_last)
    # the pass errors are means of 2 - 2 x similarity
    obj = m.obj()
    assert len(obj) == len(orc.obj)
    assert all(0.0 <= v <= 4.0 for v in obj)
    if revival != "none":
        assert res["worst"]["revive_c"] <= CENTROID_REL


@pytest.mark.parametrize("n,d,k", [(1, 32, 1), (129, 96, 257), (5000, 768, 4096), (3000, 128, 600),
                                   (4100, 256, 2048)])
def test_spherical_assign_returns_similarity(em, n, d, k):
    g = torch.Generator().manual_seed(n * 31 + k)
    x = _unit_data(n, d, 16, seed=n + k)
    c = (x[torch.randint(0, n, (k,), generator=g)] + 0.2 * torch.randn(k, d, generator=g)).float()
    m = em.Model(d, k, seed=1, spherical=1)
    m.set_state(c=c)  # rescaled to norm 1 on the way in
    c_gpu = torch.empty(k, d)
    m.centroids(c_gpu)
    c_unit = O.unit_rows(c.numpy().astype(np.float64))
    np.testing.assert_allclose(c_gpu.numpy(), c_unit, rtol=1e-6, atol=1e-7)
    labels = torch.empty(n, dtype=torch.int64, device="cuda")
    sims = torch.empty(n, dtype=torch.float32, device="cuda")
    m.assign(x.cuda(), labels=labels, dists=sims)
    xq = O.search_copy_of_data(x.numpy())
    cq = O.search_copy_of_centroids(c_gpu.numpy().astype(np.float64))
    book = LabelBook(spherical=True)
    _, best_err = book.compare(labels.cpu().numpy(), xq, cq)
    book.finish()
    sim_ref = 1.0 - 0.5 * best_err
    np.testing.assert_allclose(sims.cpu().numpy(), sim_ref, rtol=0, atol=2e-5)
    err = m.mse(x.cuda())
    assert abs(err - best_err.mean()) <= MSE_REL * best_err.mean() + 1e-6
    assert abs(err - O.spherical_error(xq, c_gpu.numpy().astype(np.float64))) <= MSE_REL * err + 1e-6


def test_spherical_zero_centroid_stays_zero(em):
    d, k = 64, 8
    x = _unit_data(500, d, 4, seed=3)
    c = x[:k].clone()
    c[3] = 0.0
    m = em.Model(d, k, seed=1, spherical=1)
    m.set_state(c=c)
    out = torch.empty(k, d)
    m.centroids(out)
    assert torch.all(out[3] == 0)
    np.testing.assert_allclose(out.norm(dim=1)[[0, 1, 2, 4, 5, 6, 7]].numpy(), 1.0, atol=1e-6)


def test_spherical_lloyd_matches_oracle(em):
    n, d, k = 4000, 48, 32
    x = _unit_data(n, d, 24, seed=9)
    xq = O.search_copy_of_data(x.numpy())
    m = em.Model(d, k, seed=1234, spherical=1)
    m.lloyd(x.cuda(), 10)
    _, _, c, _ = gpu_state(m, k, d)
    c0 = xq[O.starting_rows(n, k, 1234)]
    c_ref, hist = O.lloyd(xq, c0, 10, spherical=True)
    rel = centroid_rel_err(c, c_ref)
    assert np.mean(rel <= CENTROID_REL) >= 0.95
    err = m.mse(x.cuda())
    assert abs(err - O.spherical_error(xq, c_ref)) <= MSE_REL * err


def test_spherical_independent_run_final_error(em):
    n, d, k = 6000, 64, 48
    x = _unit_data(n, d, 40, seed=21)
    xq = O.search_copy_of_data(x.numpy())
    m = em.Model(d, k, seed=1234, spherical=1)
    m.train(x.cuda(), epochs=3.0)
    orc = O.EmeansOracle(d, k, seed=1234, spherical=True)
    c_ref, _ = orc.train(xq, 3.0)
    err_gpu, err_ref = m.mse(x.cuda()), O.spherical_error(xq, c_ref)
    assert abs(err_gpu - err_ref) <= 5 * MSE_REL * err_ref
    np.testing.assert_allclose(m.obj(), orc.obj, rtol=5e-3)
    st = m.stats()
    assert st["n_splits"] == orc.n_splits


def test_spherical_graphs_match_direct_launches(em):
    x = _unit_data(3000, 96, 30, seed=5)
    out = []
    for graphs in (1, 0):
        m = em.Model(96, 50, seed=3, spherical=1, graphs=graphs)
        m.train(x.cuda(), epochs=2.0)
        c = torch.empty(50, 96)
        m.centroids(c)
        out.append(c)
    assert torch.equal(out[0], out[1])


def test_spherical_is_fixed_during_a_run(em):
    x = _unit_data(1000, 32, 8, seed=1)
    m = em.Model(32, 10, seed=3, spherical=1)
    m.begin(x.cuda(), epochs=1.0)
    with pytest.raises(em.EmeansError):
        m.set_option("spherical", 0)
    m.finalize()
    m.set_option("spherical", 0)
    assert m.get_option("spherical") == 0
