"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Teacher-forced runs give the oracle the GPU's state before every step and compare
the batch order (bit-exact), labels (near-tie rule), distances, running counts,
sums, centroids, revivals and the closing mean. Tolerances: tests/helpers.py.
"""

import numpy as np
import pytest
import torch

from datagen import synth
import datagen
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


def _finish_and_compare(m, orc, n, xq):
    m.finalize()
    orc.finalize()
    _, _, c, _ = gpu_state(m, orc.k, orc.d)
    assert_centroids_close(c, orc.c, "closing mean")
    if m.get_option("capture_labels"):
        lab = torch.empty(n, dtype=torch.int64)
        m.labels(lab)
        assert np.array_equal(lab.numpy(), orc.labels_last)
    return c


def test_smoke_entry_point():
    import __graft_entry__

    __graft_entry__.smoke()


@pytest.mark.parametrize("revival", ["split", "resample", "none"])
def test_tiny_teacher_forced_every_step(em, revival):
    w, xt, _ = datagen.make("tiny")
    xq = O.search_copy_of_data(xt.numpy())
    m = em.Model(w.d, w.k, seed=1234, auto_revive=0, revival=revival)
    orc = O.EmeansOracle(w.d, w.k, seed=1234, revival=revival)
    res = teacher_forced_run(m, orc, xt.cuda(), xq, w.epochs, revival)
    assert res["rows"] == 5 * w.n_train
    if revival != "none":
        assert res["revived"] > 0
    _finish_and_compare(m, orc, w.n_train, xq)
    obj = m.obj()
    assert len(obj) == 5


@pytest.mark.parametrize("n,d,k,epochs,batch,revival", [
    (3000, 16, 40, 2.0, None, "split"),
    (5000, 96, 300, 1.5, 512, "split"),
    (2000, 128, 513, 2.0, 256, "split"),
    (1500, 768, 64, 1.0, 256, "split"),
    (4097, 40, 100, 1.25, 300, "resample"),
    (1000, 8, 1, 1.0, 100, "split"),
    (2600, 264, 257, 1.5, None, "split"),
    (3333, 100, 77, 1.0, 1000, "none"),
    (3000, 2, 20, 2.0, None, "split"),    # d <= 2: the default threshold turns revival off
    (4000, 12, 50, 2.0, None, "split"),   # d <= 16: the default batch law is the quality law
    # the streamed sums' row geometries: 32 lanes of one vector (d = 200), four
    # vectors per lane (d = 1000), two column slices (d = 1100), and many more rows
    # than one range per warp holds (8,192-row batches cut into 64-row ranges)
    (1200, 200, 90, 1.5, 256, "split"),
    (1100, 1000, 40, 1.0, 256, "split"),
    (1000, 1100, 33, 1.0, 200, "none"),
    (60000, 24, 700, 1.0, 8192, "split"),
])
def test_hand_shapes_teacher_forced(em, n, d, k, epochs, batch, revival):
    x = synth.hand_shape(n, d, max(2, k // 2), seed=n + d)
    xq = O.search_copy_of_data(x.numpy())
    opts = dict(auto_revive=0, revival=revival)
    if batch:
        opts["batch_size"] = batch
    m = em.Model(d, k, seed=7, **opts)
    orc = O.EmeansOracle(d, k, seed=7, revival=revival, batch_size=batch)
    teacher_forced_run(m, orc, x.cuda(), xq, epochs, revival)
    _finish_and_compare(m, orc, n, xq)


def test_bf16_input_in_place_and_padded(em):
    for d in (64, 36):  # 16-byte rows are used in place; others are copied with padding
        x = synth.hand_shape(2500, d, 20, seed=d, storage="bf16")
        xq = x.to(torch.float64).numpy()
        m = em.Model(d, 30, seed=3, auto_revive=0)
        orc = O.EmeansOracle(d, 30, seed=3)
        teacher_forced_run(m, orc, x.cuda(), xq, 1.0, "split")
        _finish_and_compare(m, orc, 2500, xq)


def test_host_input_goes_through_the_same_path(em):
    x = synth.hand_shape(3000, 32, 16, seed=11)
    m1 = em.Model(32, 24, seed=5)
    m1.train(x.cuda(), epochs=2.0)
    m2 = em.Model(32, 24, seed=5)
    m2.train(x.contiguous(), epochs=2.0)  # host tensor: copied to the device inside the call
    c1, c2 = torch.empty(24, 32), torch.empty(24, 32)
    m1.centroids(c1)
    m2.centroids(c2)
    assert torch.equal(c1, c2)


@pytest.mark.parametrize("n,d,k", [(1, 32, 1), (127, 64, 5), (129, 96, 257), (5000, 768, 4096),
                                   (3000, 128, 600), (777, 100, 300), (20000, 32, 64), (4100, 256, 2048),
                                   # more row tiles than SMs: whole row tiles first, the last
                                   # wave's split into centroid-tile groups (on 148 SMs: 296
                                   # whole and 17 split 8 ways; 148 whole and 9 split 2 ways)
                                   (40000, 32, 2000), (20000, 40, 300), (20000, 256, 512),
                                   # the folded search (|c~|^2 as one more K = 16 MMA step) at
                                   # d <= 96 with many tiles: K chunks of 32 (one, two, three)
                                   # and of 64, the last centroid tile partly empty
                                   (30000, 96, 1100), (25000, 40, 2100), (30000, 64, 1500)])
def test_assign_and_mse_match_oracle(em, n, d, k):
    g = torch.Generator().manual_seed(n * 31 + k)
    x = synth.hand_shape(n, d, 16, seed=n + k)
    c = (x[torch.randint(0, n, (k,), generator=g)] + 0.3 * torch.randn(k, d, generator=g)).float()
    m = em.Model(d, k, seed=1)
    m.set_state(c=c)
    labels = torch.empty(n, dtype=torch.int64, device="cuda")
    dists = torch.empty(n, dtype=torch.float32, device="cuda")
    m.assign(x.cuda(), labels=labels, dists=dists)
    xq = O.search_copy_of_data(x.numpy())
    cq = O.search_copy_of_centroids(c.numpy().astype(np.float64))
    book = LabelBook()
    _, best = book.compare(labels.cpu().numpy(), xq, cq)
    book.finish()
    xn = np.einsum("ij,ij->i", xq, xq)
    np.testing.assert_allclose(dists.cpu().numpy(), best, rtol=1e-4, atol=1e-5 * (xn.mean() + 1))
    mse = m.mse(x.cuda())
    assert abs(mse - best.mean()) <= MSE_REL * best.mean() + 1e-12
    # host outputs take the same path
    lab_h = torch.empty(n, dtype=torch.int64)
    m.assign(x, labels=lab_h)
    assert torch.equal(lab_h, labels.cpu())


def test_simt_and_tensor_core_search_agree(em):
    x = synth.hand_shape(3000, 96, 30, seed=2)
    k = 700
    c = x[:k].clone() + 0.01
    out = []
    for kernel in (0, 1):
        m = em.Model(96, k, seed=1, assign_kernel=kernel)
        m.set_state(c=c)
        lab = torch.empty(3000, dtype=torch.int64, device="cuda")
        m.assign(x.cuda(), labels=lab)
        out.append(lab.cpu().numpy())
    assert np.mean(out[0] != out[1]) <= 1e-3


def _one_flip_fixes(j, c_gpu_j, xq, labels, tie_rows, runner_up, prev, k):
    """Whether moving one near-tie row to its runner-up cluster makes cluster j's
    Lloyd mean (alpha = 1 from prev) match the GPU's centroid j."""
    for r in tie_rows:
        if j not in (labels[r], runner_up[r]):
            continue
        alt = labels.copy()
        alt[r] = runner_up[r]
        n_j, s_j = O.batch_stats(xq, alt, k)
        _, _, c_alt = O.ema_update(np.zeros(k), np.zeros_like(prev), prev, n_j, s_j, 1.0)
        if centroid_rel_err(c_gpu_j[None], c_alt[j][None])[0] <= CENTROID_REL:
            return True
    return False


def test_lloyd_mode_matches_oracle(em):
    """Lloyd mode (B = n, alpha = 1, natural order, 25 iterations), checked
    iteration by iteration under teacher forcing: the oracle takes one Lloyd step
    from the GPU's centroids after t iterations, and EVERY centroid of the GPU's
    next iterate must match it within the centroid tolerance. The labels of each
    iteration (the search at the GPU's c_t) follow the near-tie rule and budget.
    A cluster may differ from the oracle's step only if one near-tie row, moved
    between its two near-tied clusters, makes it match."""
    w, xt, xs = datagen.make("tiny")
    xq, xsq = O.search_copy_of_data(xt.numpy()), O.search_copy_of_data(xs.numpy())
    n, k, d = w.n_train, w.k, w.d
    xg = xt.cuda()
    m = em.Model(d, k, seed=1234)
    probe = em.Model(d, k, seed=1234)  # the search at c_t, through em_assign
    m.lloyd(xg, 0)
    _, _, prev, _ = gpu_state(m, k, d)
    assert np.array_equal(prev, xq[O.starting_rows(n, k, 1234)]), "Lloyd's starting rows differ"
    lab_dev = torch.empty(n, dtype=torch.int64, device="cuda")
    book = LabelBook()
    worst, exempt = 0.0, 0
    for t in range(25):
        m.lloyd(xg, t + 1)
        _, _, c_next, _ = gpu_state(m, k, d)
        probe.set_state(c=torch.as_tensor(prev, dtype=torch.float32))
        probe.assign(xg, labels=lab_dev)
        cq = O.search_copy_of_centroids(prev)
        accepted, best = book.compare(lab_dev.cpu().numpy(), xq, cq)
        n_j, s_j = O.batch_stats(xq, accepted, k)
        _, _, c_ref = O.ema_update(np.zeros(k), np.zeros((k, d)), prev, n_j, s_j, 1.0)
        rel = centroid_rel_err(c_next, c_ref)
        bad = np.flatnonzero(rel > CENTROID_REL)
        if len(bad):
            d2 = O.squared_distances(xq, cq)
            order = np.argsort(d2, axis=1, kind="stable")[:, :2]
            two = np.take_along_axis(d2, order, axis=1)
            tie_rows = np.flatnonzero((two[:, 1] - two[:, 0]) < 1e-3 * np.maximum(two[:, 0], 1e-30))
            runner_up = np.where(order[:, 0] == accepted, order[:, 1], order[:, 0])
            for j in bad:
                assert _one_flip_fixes(j, c_next[j], xq, accepted, tie_rows, runner_up, prev, k), (
                    f"iteration {t}: centroid {j} off by {rel[j]:.3e} with no near tie to explain it")
            assert len(bad) <= 2 * max(1, int(1e-4 * n)), f"iteration {t}: {len(bad)} clusters off"
            exempt += len(bad)
        worst = max(worst, float(np.max(np.delete(rel, bad), initial=0.0)))
        prev = c_next
    book.finish()
    print(f"Lloyd teacher-forced: worst centroid rel err {worst:.2e}, {book.mismatch} near-tie flips, "
          f"{exempt} clusters explained by a near tie")
    # the MSE the library reports, against the oracle's under the GPU's centroids
    mse_gpu = m.mse(xs.cuda())
    assert abs(mse_gpu - O.mse(xsq, prev)) <= MSE_REL * mse_gpu
    # and an independent oracle Lloyd run from the same starting rows
    c_ref, _ = O.lloyd(xq, xq[O.starting_rows(n, k, 1234)], 25)
    assert abs(mse_gpu - O.mse(xsq, c_ref)) <= MSE_REL * mse_gpu
    probe.close()
    m.close()


def test_tiny_independent_run_final_mse(em):
    w, xt, xs = datagen.make("tiny")
    xq, xsq = O.search_copy_of_data(xt.numpy()), O.search_copy_of_data(xs.numpy())
    m = em.Model(w.d, w.k, seed=1234)
    m.train(xt.cuda(), epochs=w.epochs)
    orc = O.EmeansOracle(w.d, w.k, seed=1234)
    c_ref, lab_ref = orc.train(xq, w.epochs)
    mse_gpu, mse_ref = m.mse(xs.cuda()), O.mse(xsq, c_ref)
    assert abs(mse_gpu - mse_ref) <= MSE_REL * mse_ref
    obj = m.obj()
    np.testing.assert_allclose(obj, orc.obj, rtol=1e-3)
    st = m.stats()
    assert st["steps_done"] == 50 and st["rows_assigned"] == 5 * w.n_train
    assert st["n_splits"] == orc.n_splits


def test_fractional_epochs_and_labels(em):
    x = synth.hand_shape(2000, 32, 10, seed=4)
    m = em.Model(32, 20, seed=9, batch_size=256)
    m.train(x.cuda(), epochs=1.5)
    lab = torch.empty(2000, dtype=torch.int64)
    m.labels(lab)
    assert int((lab >= 0).sum()) == 1000 and int((lab == -1).sum()) == 1000
    r = m.recipe()
    assert r["passes"] == 2 and r["rows_last_pass"] == 1000 and r["total_steps"] == 8 + 4


def test_state_roundtrip_and_errors(em):
    m = em.Model(16, 8, seed=1)
    with pytest.raises(em.EmeansError) as e:
        m.step(1)
    assert e.value.code == em.EM_E_STATE
    x = synth.hand_shape(100, 16, 4, seed=1)
    with pytest.raises(em.EmeansError) as e:
        m.train(x[:5].cuda(), epochs=1.0)  # fewer rows than clusters
    assert e.value.code == em.EM_E_INVAL
    N = torch.rand(8)
    S = torch.randn(8, 16)
    c = torch.randn(8, 16)
    m.set_state(N=N, S=S, c=c)
    N2, S2, c2 = torch.empty(8), torch.empty(8, 16), torch.empty(8, 16)
    m.get_state(N=N2, S=S2, c=c2)
    assert torch.equal(N, N2) and torch.equal(S, S2) and torch.equal(c, c2)
    bad = x.clone()
    bad[3, 2] = float("nan")
    m.set_option("check_finite", 1)
    with pytest.raises(em.EmeansError) as e:
        m.train(bad.cuda(), epochs=1.0)
    assert e.value.code == em.EM_E_NONFINITE


def test_step_graphs_match_direct_launches(em):
    """A run replayed from captured step graphs equals the same run launched kernel by
    kernel, bit for bit, and a second run (graph cache hit) equals the first."""
    x = synth.hand_shape(6000, 64, 30, seed=12)
    outs = []
    for graphs in (0, 1, 1):
        m = em.Model(64, 50, seed=21, graphs=graphs)
        m.train(x.cuda(), epochs=3.0)
        c = torch.empty(50, 64)
        m.centroids(c)
        lab = torch.empty(6000, dtype=torch.int64)
        m.labels(lab)
        outs.append((c, lab, m.obj(), m.stats()["n_splits"]))
        if graphs:
            m.train(x.cuda(), epochs=3.0)  # same run again: replayed from the cache
            c2 = torch.empty(50, 64)
            m.centroids(c2)
            assert torch.equal(c, c2)
    for c, lab, obj, splits in outs[1:]:
        assert torch.equal(c, outs[0][0]) and torch.equal(lab, outs[0][1])
        assert np.array_equal(obj, outs[0][2]) and splits == outs[0][3]


@pytest.mark.parametrize("graphs", [0, 1])
def test_dependent_launches_match_plain_launches(em, graphs):
    """Letting each kernel of a step launch while its predecessor finishes
    (programmatic dependent launch, every kernel waiting on the device) gives the
    same run, bit for bit, as plain stream-ordered launches: with revivals, the
    FP8 search and spherical e-means too."""
    x = synth.hand_shape(5000, 96, 30, seed=17)
    xs = synth.hand_shape(5000, 96, 30, seed=17, normalized=True)
    for opts, data in ((dict(), x), (dict(search_format="fp8"), x), (dict(spherical=1), xs)):
        outs = []
        for pdl in (0, 1):
            m = em.Model(96, 70, seed=5, graphs=graphs, pdl=pdl, **opts)
            m.train(data.cuda(), epochs=2.5)
            c = torch.empty(70, 96)
            m.centroids(c)
            lab = torch.empty(5000, dtype=torch.int64)
            m.labels(lab)
            outs.append((c, lab, m.obj(), m.stats()["n_splits"]))
            m.close()
        assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1]), opts
        assert np.array_equal(outs[0][2], outs[1][2]) and outs[0][3] == outs[1][3], opts


@pytest.mark.parametrize("graphs", [0, 1])
def test_prefetched_batches_match_inline_gathers(em, graphs):
    """Gathering the next step's rows on the side stream while a step updates gives
    the same run, bit for bit, as gathering every step's rows in turn: stepped one at
    a time, in uneven ranges (graphs), across pass ends and a fractional last pass,
    with a state reset in the middle and the revival's resampling reading the rows."""
    x = synth.hand_shape(5000, 96, 30, seed=14)
    outs = []
    for prefetch in (0, 1):
        m = em.Model(96, 70, seed=5, graphs=graphs, prefetch=prefetch, revival="resample")
        m.begin(x.cuda(), epochs=2.5)
        total = m.recipe()["total_steps"]
        done = 0
        for chunk in (1, 3, 2, 7, 1):
            done += m.step(chunk)
        N, S, c, step = gpu_state(m, 70, 96)
        m.set_state(N=torch.from_numpy(N.astype(np.float32)), S=torch.from_numpy(S.astype(np.float32)),
                    c=torch.from_numpy(c.astype(np.float32)), step=step)
        while done < total:
            done += m.step(4)
        ids = torch.empty(m.recipe()["batch_size"], dtype=torch.int64)
        r = m.last_batch(ids=ids)
        m.finalize()
        cc = torch.empty(70, 96)
        m.centroids(cc)
        lab = torch.empty(5000, dtype=torch.int64)
        m.labels(lab)
        outs.append((cc, lab, m.obj(), ids[:r].clone()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    assert np.array_equal(outs[0][2], outs[1][2]) and torch.equal(outs[0][3], outs[1][3])


@pytest.mark.parametrize("d", [64, 96, 768])
def test_exact_ties_reproduce_the_fp64_argmin(em, d):
    """Centroids come in pairs one bf16 step apart, so most rows are near ties of
    their pair; with exact tie settling the labels equal the fp64 oracle's, and
    exact duplicates go to the lower index."""
    n, pairs = 4000, 40
    g = torch.Generator().manual_seed(d)
    x = synth.hand_shape(n, d, 10, seed=d)
    base = x[torch.randint(0, n, (pairs,), generator=g)] + 0.5 * torch.randn(pairs, d, generator=g)
    base = base.to(torch.bfloat16).float()
    twin = base.clone()
    idx = torch.randint(0, d, (pairs,), generator=g)
    for i in range(pairs):  # move one coordinate of the twin by one bf16 step
        v = twin[i, idx[i]].to(torch.bfloat16)
        twin[i, idx[i]] = (v.view(torch.int16) + 1).view(torch.bfloat16).float()
    c = torch.stack([base, twin], 1).reshape(2 * pairs, d)
    c[-1] = c[0]  # an exact duplicate: ties go to the lower index
    m = em.Model(d, 2 * pairs, seed=1, exact_ties=1)
    m.set_state(c=c)
    labels = torch.empty(n, dtype=torch.int64, device="cuda")
    m.assign(x.cuda(), labels=labels)
    xq = O.search_copy_of_data(x.numpy())
    ref, _, _ = O.assign(xq, O.search_copy_of_centroids(c.numpy().astype(np.float64)))
    assert np.array_equal(labels.cpu().numpy(), ref)


def test_failure_path_reports_timeout_and_bounds_and_recovers(em):
    """Failure detection without a fault: a bounded device-side wait on a barrier
    nothing arrives on gives up after its limit and the host reads EM_E_TIMEOUT; a
    failed index check reaches the host as EM_E_BOUNDS; afterwards the same model
    trains as a fresh one does."""
    import time

    x = synth.hand_shape(2000, 32, 10, seed=2)
    m = em.Model(32, 20, seed=4)
    t0 = time.time()
    assert m.selftest(0, wait_ms=300.0) == em.EM_E_TIMEOUT
    assert 0.25 <= time.time() - t0 < 5.0
    assert m.selftest(1) == em.EM_E_BOUNDS
    m.train(x.cuda(), epochs=1.0)
    c = torch.empty(20, 32)
    m.centroids(c)
    ref = em.Model(32, 20, seed=4)
    ref.train(x.cuda(), epochs=1.0)
    c2 = torch.empty(20, 32)
    ref.centroids(c2)
    assert torch.equal(c, c2)
    assert m.selftest(2) == em.EM_E_INVAL


@pytest.mark.parametrize("k", [70, 3000, 6000, 12000, 20000])
def test_overlapped_selection_matches_serial_revival(em, k):
    """The revival check's donor selection runs beside the segmented sums, deriving
    the new running counts from N_prev and the segment sizes; with profiling on it
    runs in line after the update. Both give the same run, bit for bit (dead sets,
    donors, counts, centroids), on the two-level trees of every group size
    (k <= 16,384) and the radix-128 one."""
    x = synth.hand_shape(max(4 * k, 6000), 24, max(8, k // 3), seed=k)
    outs = []
    for profile in (0, 1):
        m = em.Model(24, k, seed=9, profile=profile)
        m.train(x.cuda(), epochs=2.0)
        c = torch.empty(k, 24)
        m.centroids(c)
        N = torch.empty(k)
        m.get_state(N=N)
        outs.append((c, N, m.obj(), m.stats()["n_splits"]))
        m.close()
    assert outs[0][3] > 0
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    assert np.array_equal(outs[0][2], outs[1][2]) and outs[0][3] == outs[1][3]
