"""Whole runs at full size: the CUDA path and the fp64 oracle each train e-means
from the same seed on the same data, independently, and their final test MSE
must agree within 0.1 %.

Independent runs are not expected to keep identical centroids: a near-tie row
(best and second distances within the fp32 accumulation error of the tensor
cores) may take the other label, and the trajectories part from there. The test
MSE, an average over every test row and every cluster, is what the method fixes.
The per-centroid differences are printed as a distribution (with -s). The
oracle's search is run in row blocks on a thread pool (tests/helpers.py
`threaded_assign`, row for row the same result) so that a whole run takes a few
minutes of host time.
"""

import numpy as np
import pytest
import torch

import datagen
from oracle import emeans_oracle as O
from tests.helpers import MSE_REL, centroid_rel_err, threaded_assign

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def em():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mini_ema_means_b200

    return mini_ema_means_b200


@pytest.mark.parametrize("name", ["emb768", "deep96"])
def test_whole_run_final_test_mse_matches_oracle_run(em, name, monkeypatch):
    w, xt, xs = datagen.make(name, device="cuda", seed=0)
    k, d = w.k, w.d
    m = em.Model(d, k, seed=1234)
    m.train(xt, epochs=w.epochs)
    c = torch.empty(k, d, device="cuda")
    m.centroids(c)
    mse_gpu = m.mse(xs)
    obj_gpu = np.asarray(m.obj())
    splits_gpu = m.stats()["n_splits"]
    m.close()
    c_gpu = c.double().cpu().numpy()
    xq = O.search_copy_of_data(xt.float().cpu().numpy())
    xsq = O.search_copy_of_data(xs.float().cpu().numpy())
    del xt, xs, c
    torch.cuda.empty_cache()

    monkeypatch.setattr(O, "assign", threaded_assign(O.assign))
    orc = O.EmeansOracle(d, k, seed=1234)
    c_ref, _ = orc.train(xq, w.epochs)
    mse_ref = O.mse(xsq, c_ref)
    # the library's test MSE is the MSE of its own centroids
    mse_own = O.mse(xsq, c_gpu)
    assert abs(mse_gpu - mse_own) <= 1e-5 * mse_own, (mse_gpu, mse_own)
    # and the two whole runs end within 0.1 % of each other
    rel = centroid_rel_err(c_gpu, c_ref)
    q = np.quantile(rel, [0.5, 0.9, 0.99, 1.0])
    print(f"\n{name}: test MSE GPU {mse_gpu:.6f} oracle {mse_ref:.6f} (rel {abs(mse_gpu / mse_ref - 1):.2e}); "
          f"centroid rel L2 error median {q[0]:.2e} p90 {q[1]:.2e} p99 {q[2]:.2e} max {q[3]:.2e}; "
          f"{int(np.sum(rel <= 1e-3))} of {k} within 1e-3; splits GPU {splits_gpu} oracle {orc.n_splits}; "
          f"pass errors GPU {np.round(obj_gpu, 6).tolist()} oracle {np.round(orc.obj, 6).tolist()}")
    assert abs(mse_gpu - mse_ref) <= MSE_REL * mse_ref, (mse_gpu, mse_ref)
    # the first pass's training error, before trajectories can part much
    assert abs(obj_gpu[0] - orc.obj[0]) <= MSE_REL * orc.obj[0], (obj_gpu[0], orc.obj[0])
