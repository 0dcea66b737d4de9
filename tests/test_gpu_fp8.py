"""GPU parity of the FP8 (E4M3) search (faiss e-means README, "Data precision"):
a converter with a shift per dimension and one power-of-two scale, fitted on the
first rows of the data; rows and centroids searched as E4M3 codes on the tensor
cores' FP8 path; counts, sums and centroids in fp32; distances in the data's units.
The CUDA path through the C ABI against EmeansOracle(search="fp8"). Tolerances:
tests/helpers.py (labels compared on the codes; another label is accepted where its code
distance is within the FP8 accumulation bound of the best).
"""

import numpy as np
import pytest
import torch

from datagen import synth
from oracle import emeans_oracle as O
from tests.helpers import (CENTROID_REL, FP8_GAP_REL, MSE_REL, LabelBook, assert_centroids_close, centroid_rel_err,
                           gpu_state, teacher_forced_run)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def em():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mini_ema_means_b200

    return mini_ema_means_b200


@pytest.mark.parametrize("n,d", [(3000, 32), (70000, 96), (1000, 8), (2000, 264)])
def test_converter_is_the_oracles(em, n, d):
    """Shift and scale fitted on the first 65,536 rows equal the oracle's, bit for bit."""
    x = synth.hand_shape(n, d, 12, seed=n + d)
    xq = O.search_copy_of_data(x.numpy())
    m = em.Model(d, 10, seed=1, search_format="fp8")
    m.begin(x.cuda(), epochs=1.0)
    shift, scale = m.fp8_converter()
    ref_shift, ref_scale = O.fp8_calibrate(xq)
    assert scale == ref_scale and np.array_equal(shift, ref_shift)
    m.finalize()
    m.close()


@pytest.mark.parametrize("n,d,k,epochs,batch,revival", [
    (3000, 32, 40, 2.0, None, "split"),
    (2600, 96, 257, 1.5, 256, "split"),
    (1500, 768, 64, 1.0, 256, "split"),   # six 128-code chunks per row
    (2500, 264, 300, 1.25, None, "resample"),  # a ragged last chunk
    (2000, 8, 30, 2.0, None, "none"),     # one chunk, mostly zero columns
    (4000, 200, 520, 1.0, 512, "split"),  # three column tiles, A stationary (d <= 256)
])
def test_fp8_teacher_forced(em, n, d, k, epochs, batch, revival):
    x = synth.hand_shape(n, d, max(2, k // 2), seed=n + d)
    xq = O.search_copy_of_data(x.numpy())
    opts = dict(auto_revive=0, revival=revival, search_format="fp8")
    if batch:
        opts["batch_size"] = batch
    m = em.Model(d, k, seed=7, **opts)
    orc = O.EmeansOracle(d, k, seed=7, revival=revival, batch_size=batch, search="fp8")
    teacher_forced_run(m, orc, x.cuda(), xq, epochs, revival)
    m.finalize()
    orc.finalize()
    _, _, c, _ = gpu_state(m, k, d)
    assert_centroids_close(c, orc.c, "FP8 closing mean")
    lab = torch.empty(n, dtype=torch.int64)
    m.labels(lab)
    assert np.array_equal(lab.numpy(), orc.labels_last)


@pytest.mark.parametrize("n,d,k", [(1, 32, 1), (129, 96, 257), (5000, 768, 4096), (3000, 128, 600)])
def test_fp8_assign_and_mse(em, n, d, k):
    """A model with a converter from its run assigns new rows with it; labels on the
    codes, squared distances in the data's units."""
    g = torch.Generator().manual_seed(n * 31 + k)
    x = synth.hand_shape(max(n, 2 * k), d, 16, seed=n + k)
    m = em.Model(d, k, seed=1, search_format="fp8")
    m.train(x.cuda(), epochs=1.0)
    shift, scale = m.fp8_converter()
    q = (x[:n] + 0.05 * torch.randn(n, d, generator=g)).float()
    c = torch.empty(k, d)
    m.centroids(c)
    labels = torch.empty(n, dtype=torch.int64, device="cuda")
    dists = torch.empty(n, dtype=torch.float32, device="cuda")
    m.assign(q.cuda(), labels=labels, dists=dists)
    xq = O.search_copy_of_data(q.numpy())
    xr = O.fp8_codes(xq, shift, scale)
    cr = O.fp8_search_copy_of_centroids(c.numpy().astype(np.float64), shift, scale)
    book = LabelBook(fp8=True)
    lab = labels.cpu().numpy()
    _, best = book.compare(lab, xr, cr, dscale=1.0 / scale ** 2)
    book.finish()
    # the GPU's distance of its own label, within twice the accumulation bound
    own = ((xr - cr[lab]) ** 2).sum(axis=1) / scale ** 2
    mag = np.einsum("ij,ij->i", np.abs(xr), np.abs(cr[lab])) / scale ** 2
    assert np.all(np.abs(dists.cpu().numpy() - own) <= 4.0 * FP8_GAP_REL * mag + 1e-5 * own + 1e-6)
    mse = m.mse(q.cuda())
    assert abs(mse - own.mean()) <= MSE_REL * own.mean() + 4.0 * FP8_GAP_REL * mag.mean()
    m.close()


def test_fp8_lloyd_matches_oracle(em):
    x = synth.hand_shape(4000, 48, 20, seed=9)
    xq = O.search_copy_of_data(x.numpy())
    m = em.Model(48, 32, seed=1234, search_format="fp8")
    m.lloyd(x.cuda(), 10)
    _, _, c, _ = gpu_state(m, 32, 48)
    conv = O.fp8_calibrate(xq)
    c0 = xq[O.starting_rows(4000, 32, 1234)]
    c_ref, _ = O.lloyd(xq, c0, 10, fp8=conv)
    rel = centroid_rel_err(c, c_ref)
    assert np.mean(rel <= CENTROID_REL) >= 0.95
    assert abs(m.mse(x.cuda()) - O.mse_fp8(xq, c_ref, *conv)) <= MSE_REL * O.mse_fp8(xq, c_ref, *conv)


def test_fp8_graphs_prefetch_and_one_rank_dp_agree(em):
    """Graph replay, inline gathers and a one-rank data-parallel run give the same
    FP8 run, bit for bit."""
    x = synth.hand_shape(5000, 96, 30, seed=5)
    outs = []
    for graphs, prefetch, dp in ((1, 1, False), (0, 0, False), (1, 1, True)):
        m = em.Model(96, 60, seed=3, search_format="fp8", graphs=graphs, prefetch=prefetch)
        if dp:
            m.dp_init_id(1, 0, em.dp_unique_id())
        m.train(x.cuda(), epochs=2.0)
        c = torch.empty(60, 96)
        m.centroids(c)
        outs.append((c, m.obj()))
        m.close()
    for c, obj in outs[1:]:
        assert torch.equal(c, outs[0][0]) and np.array_equal(obj, outs[0][1])


def test_fp8_independent_run_close_to_oracle(em):
    x = synth.hand_shape(6000, 64, 40, seed=21)
    xq = O.search_copy_of_data(x.numpy())
    m = em.Model(64, 48, seed=1234, search_format="fp8")
    m.train(x.cuda(), epochs=3.0)
    orc = O.EmeansOracle(64, 48, seed=1234, search="fp8")
    c_ref, _ = orc.train(xq, 3.0)
    err_gpu, err_ref = m.mse(x.cuda()), O.mse_fp8(xq, c_ref, *orc.fp8)
    assert abs(err_gpu - err_ref) <= 5 * MSE_REL * err_ref
    np.testing.assert_allclose(m.obj(), orc.obj, rtol=5e-3)
    m.close()


def test_fp8_refuses_spherical(em):
    x = synth.hand_shape(500, 16, 4, seed=1, normalized=True)
    m = em.Model(16, 8, seed=1, search_format="fp8", spherical=1)
    with pytest.raises(em.EmeansError):
        m.train(x.cuda(), epochs=1.0)
    m.close()
