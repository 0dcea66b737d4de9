"""Full-size parity on sampled outputs, in the launch configuration bench.py times.

At the workloads' real sizes the oracle cannot redo whole steps quickly, so each
checked step compares what it can compute one by one:
* batch row ids at sampled positions (bit-exact, the per-pass order);
* the labels and distances of 2048 sampled batch rows (near-tie rule);
* N, S and c after the EMA for 96 sampled clusters, recomputed in fp64 from every
  batch row the GPU assigned to them (teacher forcing: the oracle starts from the
  GPU's state before the step);
* after a revival check: every running count (bit-exact halvings) and the
  centroids of the clusters it touched;
* after the run: the test MSE of 8192 sampled test rows (2048 when k > 16384)
  under the GPU's centroids.

The four workloads are the 1M x 768 embedding-like set, the 1M x 96 subspace set,
the 10M x 128 integer-valued set and the 100M x 128 streamed set (25.6 GB of bf16
resident, batches of 4M rows gathered from HBM).
"""

import numpy as np
import pytest
import torch

import datagen
from oracle import emeans_oracle as O
from tests.helpers import LabelBook, assert_centroids_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def em():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mini_ema_means_b200

    return mini_ema_means_b200


def _rows(x, idx):
    """Search copy (fp64) of the given rows of a device matrix."""
    t = torch.as_tensor(np.asarray(idx, dtype=np.int64), device=x.device)
    return O.search_copy_of_data(x.index_select(0, t).float().cpu().numpy())


def _state(m, k, d):
    N = torch.empty(k, device="cuda")
    S = torch.empty(k, d, device="cuda")
    c = torch.empty(k, d, device="cuda")
    m.get_state(N=N, S=S, c=c)
    return N.double(), S.double(), c.double()


@pytest.mark.parametrize("name", ["emb768", "deep96", "sift128", "stream128"])
def test_full_size_sampled_steps(em, name):
    w, xt, xs = datagen.make(name, device="cuda", seed=0)
    k, d = w.k, w.d
    m = em.Model(d, k, seed=1234, auto_revive=0)
    rec = m.begin(xt, epochs=w.epochs)
    ref = O.recipe(w.n_train, k, w.epochs)
    assert rec["batch_size"] == ref["batch_size"] and rec["total_steps"] == ref["total_steps"]
    total, B, full = rec["total_steps"], rec["batch_size"], rec["steps_full_pass"]
    rng = np.random.default_rng(0)
    checks = {0, 1, 4, total // 2, total - 1}
    book = LabelBook()
    order = {}
    for t in range(total):
        p = t // full
        if p not in order:
            order[p] = None  # computed lazily at sampled positions below
        if t not in checks:
            m.step(1)
            if (t + 1) % 5 == 0:
                m.revive()
            continue
        N0, S0, c0 = _state(m, k, d)
        m.step(1)
        rows = m.last_batch()
        ids = torch.empty(rows, dtype=torch.int64)
        labels = torch.empty(rows, dtype=torch.int64)
        dists = torch.empty(rows, dtype=torch.float32)
        m.last_batch(ids=ids, labels=labels, dists=dists)
        ids, labels, dists = ids.numpy(), labels.numpy(), dists.numpy().astype(np.float64)
        # batch order at sampled positions
        pos = rng.choice(rows, size=min(rows, 4096), replace=False)
        start = (t - p * full) * B
        ref_ids = O.permute((start + pos).astype(np.uint64), w.n_train, 1234, O.STREAM_PASS, p)
        assert np.array_equal(ids[pos], ref_ids)
        # labels and distances of sampled rows
        samp = rng.choice(rows, size=min(rows, 2048), replace=False)
        cq = O.search_copy_of_centroids(c0.cpu().numpy())
        xq = _rows(xt, ids[samp])
        _, best = book.compare(labels[samp], xq, cq)
        np.testing.assert_allclose(dists[samp], best, rtol=1e-4, atol=1e-5)
        # EMA of sampled clusters from all of their batch rows (GPU labels)
        N1, S1, c1 = _state(m, k, d)
        alpha = O.alpha_at(t, total, rec["alpha0"])
        present = np.unique(labels)
        js = np.unique(np.concatenate([rng.choice(present, size=min(64, len(present)), replace=False),
                                       rng.choice(k, size=32, replace=False)]))
        for j in js:
            members = ids[labels == j]
            s_j = _rows(xt, members).sum(axis=0) if len(members) else np.zeros(d)
            n_j = float(len(members))
            N_ref = (1 - alpha) * N0[j].item() + alpha * n_j
            S_ref = (1 - alpha) * S0[j].cpu().numpy() + alpha * s_j
            c_ref = S_ref / N_ref if N_ref > 0 else c0[j].cpu().numpy()
            assert abs(N1[j].item() - N_ref) <= 2e-6 * max(N_ref, 1e-30)
            assert_centroids_close(c1[j].cpu().numpy()[None], c_ref[None], f"{name} step {t} cluster {j}")
        if (t + 1) % 5 == 0:
            m.revive()
            N2, S2, c2 = _state(m, k, d)
            Nr, Sr, cr, dead, donors = O.revive(N1.cpu().numpy(), S1.cpu().numpy(), c1.cpu().numpy(), t, 1234)
            np.testing.assert_array_equal(N2.cpu().numpy(), Nr)
            touched = np.unique(np.concatenate([dead, donors[donors >= 0]])).astype(np.int64)
            if len(touched):
                assert_centroids_close(c2.cpu().numpy()[touched], cr[touched], f"{name} step {t} revival")
    book.finish()
    m.finalize()
    # test MSE of sampled test rows under the GPU's final centroids
    c = torch.empty(k, d, device="cuda")
    m.centroids(c)
    samp = rng.choice(w.n_test, size=8192 if k <= 16384 else 2048, replace=False)
    dg = torch.empty(w.n_test, dtype=torch.float32, device="cuda")
    m.assign(xs, dists=dg)
    _, best, _ = O.assign(_rows(xs, samp), O.search_copy_of_centroids(c.double().cpu().numpy()))
    gpu = dg.cpu().numpy().astype(np.float64)[samp]
    assert abs(gpu.mean() - best.mean()) <= 1e-3 * best.mean()
    m.close()


def test_revival_ablation_ordering_full_size(em):
    """The pages' ablation on the 1M x 96 stand-in data (one seed): splitting leaves
    far fewer unused clusters (fewer rows than a tenth of the mean in a full pass)
    than no revival, and a lower test MSE."""
    w, xt, xs = datagen.make("deep96", device="cuda", seed=0)
    labels = torch.empty(w.n_train, dtype=torch.int64, device="cuda")
    res = {}
    for mode in ("split", "none"):
        m = em.Model(w.d, w.k, seed=0, revival=mode)
        m.train(xt, epochs=w.epochs)
        m.assign(xt, labels=labels)
        cnt = torch.bincount(labels, minlength=w.k).double()
        res[mode] = (int((cnt < 0.1 * cnt.mean()).sum().item()), m.mse(xs))
        m.close()
    assert res["split"][0] * 4 < res["none"][0], res
    assert res["split"][1] < res["none"][1], res
