"""Pins that tie the fp64 oracle to the pages and to mathematics, not to itself.

Each test checks the oracle against something independent of its own code: an
independent library implementation (numpy's Philox, torch's bf16 cast), a
brute-force definition, a closed form, an invariant the pages state, or a
number the pages print (fixtures under tests/golden/ carry their citations).
"""

import math

import numpy as np
import pytest
import torch

from oracle import emeans_oracle as O
from tests.conftest import golden
import datagen
from datagen import synth


# ---------------------------------------------------------------- generator

@pytest.mark.parametrize("ctr,key", [
    ((0, 0, 0, 0), (0, 0)),
    ((5, 0, 0, 0), (1234, 2)),
    ((0xFFFFFFFFFFFFFFFE, 7, 9, 11), (0xDEADBEEF, 3)),
    ((123456789, 2 ** 63 + 5, 1, 2 ** 40), (2 ** 64 - 1, 2 ** 62)),
])
def test_philox_matches_numpy_bit_generator(ctr, key):
    # numpy's Philox (4x64, 10 rounds) increments its counter before each block,
    # so the block at counter c is numpy's first output when started at c - 1.
    value = sum(int(w) << (64 * i) for i, w in enumerate(ctr))
    value = (value - 1) % 2 ** 256  # 256-bit counter, borrow across words
    start = np.array([(value >> (64 * i)) & (2 ** 64 - 1) for i in range(4)], dtype=np.uint64)
    ref = np.random.Philox(counter=start, key=np.array(key, dtype=np.uint64)).random_raw(4)
    mine = O.philox4x64_10(*[np.uint64(c) for c in ctr], np.uint64(key[0]), np.uint64(key[1]))
    assert [int(v) for v in ref] == [int(m) for m in mine]


def test_philox_vectorised_equals_scalar_calls():
    c0 = np.arange(100, dtype=np.uint64) * np.uint64(0x9E37)
    vec = O.philox4x64_10(c0, np.uint64(3), np.uint64(4), np.uint64(5), np.uint64(99), np.uint64(1))
    for i in (0, 17, 99):
        one = O.philox4x64_10(c0[i], np.uint64(3), np.uint64(4), np.uint64(5), np.uint64(99), np.uint64(1))
        assert [int(v[i]) for v in vec] == [int(v) for v in one]


def test_uniform_draws_are_in_unit_interval_and_spread():
    u = O.draw_uniform(1234, O.STREAM_REVIVE, 7, np.arange(20000))
    assert u.min() >= 0.0 and u.max() < 1.0
    assert abs(u.mean() - 0.5) < 0.01
    hist = np.bincount(np.floor(u * 10).astype(int), minlength=10)
    assert hist.min() > 1800


# ---------------------------------------------------------------- number formats

def test_bf16_rounding_matches_torch_cast():
    g = np.random.default_rng(0)
    x = np.concatenate([
        g.standard_normal(20000).astype(np.float32),
        (g.standard_normal(2000) * 1e30).astype(np.float32),
        (g.standard_normal(2000) * 1e-38).astype(np.float32),  # subnormals
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, -3.4e38, np.inf, -np.inf], np.float32),
    ])
    # exact ties between two bf16 neighbours, both parities of the kept bit
    ties = (np.arange(1, 500, dtype=np.uint32) << np.uint32(16)) | np.uint32(0x8000)
    x = np.concatenate([x, (ties + np.uint32(0x3F800000)).view(np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(O.f32_to_bf16(x).view(np.uint32), ref.view(np.uint32))


def test_centroid_search_copy_rounds_through_fp32():
    c = np.array([1.0 + 2 ** -9 + 2 ** -30, -(1.0 + 2 ** -9 - 2 ** -40)])
    # fp64 -> fp32 keeps the value just above the tie, fp32 -> bf16 rounds it up
    # (nearest-even for an exact fp32 tie would round down for the second value)
    out = O.search_copy_of_centroids(c)
    ref = torch.tensor(c).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(out, ref)


# ---------------------------------------------------------------- per-pass order

@pytest.mark.parametrize("n", [1, 2, 3, 7, 120, 1000, 10000, 65537])
def test_pass_order_is_a_bijection(n):
    p = O.pass_order(n, 1234, 0)
    assert p.dtype == np.int64 and len(p) == n
    assert np.array_equal(np.sort(p), np.arange(n))


def test_pass_orders_differ_between_passes_and_seeds():
    a, b, c = O.pass_order(5000, 1234, 0), O.pass_order(5000, 1234, 1), O.pass_order(5000, 99, 0)
    assert not np.array_equal(a, b) and not np.array_equal(a, c)
    # a fresh random order: roughly half the positions of a uniform shuffle move by > n/4
    assert np.mean(np.abs(a - np.arange(5000)) > 1250) > 0.4


def test_starting_rows_are_distinct_training_rows():
    rows = O.starting_rows(10000, 64, 1234)
    assert len(set(rows.tolist())) == 64 and rows.min() >= 0 and rows.max() < 10000
    # a random choice over the whole training set, not a block of it: 64 uniform
    # draws from [0, 10000) span more than half the range and have a mean near the
    # middle (both fail with probability far below 1e-6)
    assert rows.max() - rows.min() > 5000 and abs(rows.mean() - 5000) < 2000
    assert not np.array_equal(rows, O.starting_rows(10000, 64, 99))


def test_every_row_once_per_pass_and_fractional_last_pass():
    x = np.random.default_rng(1).standard_normal((1000, 4))
    em = O.EmeansOracle(4, 8, seed=3, batch_size=64, revival="none")
    em.begin(x, 2.5)
    seen = [[] for _ in range(3)]
    while not em.done:
        p = em.pass_index
        seen[p].extend(em.step()["ids"].tolist())
    assert sorted(seen[0]) == list(range(1000)) and sorted(seen[1]) == list(range(1000))
    assert len(seen[2]) == 500 and len(set(seen[2])) == 500
    # labels of the last pass cover exactly its rows; the others are -1
    assert np.count_nonzero(em.labels_last >= 0) == 500


# ---------------------------------------------------------------- recipe

def test_blog_toy_update_count():
    g = golden("blog_toy.json")
    r = O.recipe(g["points"], g["k"], g["epochs"], batch_size=g["batch_size"], alpha0=g["alpha0"])
    assert r["total_steps"] == g["emeans_updates"]
    assert r["alpha0"] == g["alpha0"]


@pytest.mark.parametrize("n,k,T", [(10_000, 64, 5), (1_000_000, 4096, 5), (1_000_000, 16384, 5),
                                   (10_000_000, 65536, 5), (100_000_000, 262144, 3)])
def test_recipe_agrees_with_independently_quoted_rounded_law(n, k, T):
    g = golden("scaling_law_rounded.json")
    b, a = g["batch"], g["alpha0"]
    b_rounded_law = b["const"] * k ** b["k_exp"] * n ** b["n_exp"] * T ** b["T_exp"]
    r = O.recipe(n, k, T)
    # the unrounded batch agrees within the rounding of the quoted constants
    assert abs(math.log(r["batch_raw"] / b_rounded_law)) < 0.08
    # and rounds to the same power of two (capped at n/2)
    assert O.round_batch(b_rounded_law, n) == r["batch_size"]
    a_rounded_law = min(a["cap"], a["const"] * k ** a["k_exp"] * r["batch_size"] ** a["B_exp"]
                        * n ** a["n_exp"] * T ** a["T_exp"])
    assert abs(r["alpha0"] / a_rounded_law - 1) < 0.05


def test_recipe_invariants():
    for n, k, T in [(10, 2, 1), (1000, 10, 0.5), (12345, 100, 2.5), (10 ** 6, 4096, 5), (3 * 10 ** 8, 10 ** 6, 2)]:
        r = O.recipe(n, k, T)
        b = r["batch_size"]
        assert b & (b - 1) == 0 and b <= max(1, n // 2)
        assert 1e-4 <= r["alpha0"] <= 1.0
        assert r["steps_per_pass"] == [-(-rows // b) for rows in r["epoch_rows"]]
        assert sum(r["epoch_rows"]) == pytest.approx(n * T, abs=1)
    # the quality law gives a batch about 8x smaller ([README] "Core configuration")
    rt, rq = O.recipe(10 ** 7, 65536, 5), O.recipe(10 ** 7, 65536, 5, law="quality")
    assert rt["batch_size"] / rq["batch_size"] == 8
    # a manual batch size re-derives alpha0 from equation (3) ([README] "Manual overrides")
    r = O.recipe(10 ** 6, 4096, 5, batch_size=8192)
    assert r["batch_size"] == 8192 and r["alpha0"] == O.alpha0_law(10 ** 6, 4096, 8192, 5)
    assert r["alpha0"] < O.recipe(10 ** 6, 4096, 5)["alpha0"]


def test_batch_rounding_is_nearest_power_in_log2_and_capped():
    assert O.round_batch(730, 10 ** 6) == 1024  # log2(730) = 9.51
    assert O.round_batch(720, 10 ** 6) == 512   # log2(720) = 9.49
    assert O.round_batch(5e6, 10 ** 6) == 2 ** 18  # cap: largest power of two <= n/2
    assert O.round_batch(0.3, 10) == 1


# ---------------------------------------------------------------- schedule

def test_cosine_schedule_endpoints_and_shape():
    a0, S = 0.6485, 80
    a = np.array([O.alpha_at(t, S, a0) for t in range(S)])
    assert a[0] == pytest.approx(a0, rel=1e-15)
    assert a[-1] == pytest.approx(0.1 * a0, rel=1e-12)   # "down to a tenth of its starting value"
    assert np.all(np.diff(a) < 0)
    # cosine: symmetric around the midpoint value (a0 + a0/10) / 2
    assert np.allclose(a + a[::-1], 1.1 * a0, rtol=0, atol=1e-12)
    assert O.alpha_at(0, 1, 0.3) == pytest.approx(0.3, rel=1e-15)
    # interior points where the cosine has a closed form: with 13 steps, t = 3, 4, 6, 8
    # are a quarter, a third, a half and two thirds of the way; cos(pi/4) = sqrt(2)/2,
    # cos(pi/3) = 1/2, cos(pi/2) = 0, cos(2 pi/3) = -1/2.  A linear, power-law or other
    # symmetric decay with the same endpoints misses at least one of them.
    a_min = 0.1 * a0
    span = a0 - a_min
    for t, half_one_plus_cos in ((3, (1.0 + np.sqrt(2.0) / 2.0) / 2.0), (4, 0.75), (6, 0.5), (8, 0.25)):
        assert O.alpha_at(t, 13, a0) == pytest.approx(a_min + span * half_one_plus_cos, rel=1e-14), t


# ---------------------------------------------------------------- assignment

def test_assign_matches_brute_force_definition():
    g = np.random.default_rng(2)
    x = O.search_copy_of_data(g.standard_normal((300, 5)).astype(np.float32))
    c = O.search_copy_of_centroids(g.standard_normal((17, 5)))
    labels, best, second = O.assign(x, c, chunk=64)
    for i in range(300):
        d = [sum((x[i, t] - c[j, t]) ** 2 for t in range(5)) for j in range(17)]
        j = min(range(17), key=lambda q: (d[q], q))
        assert labels[i] == j
        assert best[i] == pytest.approx(d[j], rel=1e-12, abs=1e-12)
        assert second[i] == pytest.approx(sorted(d)[1], rel=1e-12, abs=1e-12)


def test_assign_ties_go_to_lowest_index():
    c = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 0.0]])
    x = np.array([[0.5, 0.5], [1.0, 0.0], [2.0, 0.0]])
    labels, best, _ = O.assign(x, c)
    assert labels.tolist() == [0, 0, 0]
    assert best[1] == 0.0


# ---------------------------------------------------------------- update rule

def _brute_lloyd_step(x, c):
    k = c.shape[0]
    out = c.copy()
    members = [[] for _ in range(k)]
    for i in range(x.shape[0]):
        d = [float(np.sum((x[i] - c[j]) ** 2)) for j in range(k)]
        members[int(np.argmin(d))].append(i)
    for j in range(k):
        if members[j]:
            out[j] = np.mean(x[members[j]], axis=0)
    return out


def test_full_batch_unit_step_is_one_lloyd_iteration():
    """[README] "How the centroid updates work": whole dataset as one batch and a
    step of 1 is exactly one Lloyd iteration ([Blog] "Lloyd is a special case")."""
    g = np.random.default_rng(3)
    x = g.standard_normal((400, 3)) + np.repeat(g.standard_normal((4, 3)) * 4, 100, axis=0)
    c = x[[0, 100, 200, 7, 399]].copy()
    em = O.EmeansOracle(3, 5, seed=1, batch_size=400, alpha0=1.0, revival="none", closing_mean=False)
    em.begin(x, 1.0, start_rows=[0, 100, 200, 7, 399])
    em.order = np.arange(400)  # natural order; the batch is the whole set either way
    # one update with alpha = 1 (the schedule of a single step is alpha0)
    labels, _, _ = O.assign(x, c)
    n_j, s_j = O.batch_stats(x, labels, 5)
    _, _, c1 = O.ema_update(np.zeros(5), np.zeros((5, 3)), c, n_j, s_j, 1.0)
    assert np.allclose(c1, _brute_lloyd_step(x, c), rtol=1e-12, atol=1e-12)
    # and through the loop: the only step of a 1-epoch, B = n run
    em.c = c.copy()
    em.xq = x
    em.step()
    # the loop searches with bf16 copies; on this data the labels are unchanged
    assert np.allclose(em.c, _brute_lloyd_step(x, c), rtol=1e-12, atol=1e-12)


def test_constant_step_single_cluster_is_exponentially_weighted_mean():
    g = np.random.default_rng(4)
    batches = [g.standard_normal((int(m), 6)) for m in g.integers(5, 40, size=12)]
    alpha = 0.3
    N, S, c = np.zeros(1), np.zeros((1, 6)), np.zeros((1, 6))
    for b in batches:
        n_j, s_j = O.batch_stats(b, np.zeros(len(b), dtype=np.int64), 1)
        N, S, c = O.ema_update(N, S, c, n_j, s_j, alpha)
    T = len(batches)
    w = [alpha * (1 - alpha) ** (T - 1 - t) for t in range(T)]
    S_closed = sum(wt * b.sum(axis=0) for wt, b in zip(w, batches))
    N_closed = sum(wt * len(b) for wt, b in zip(w, batches))
    assert np.allclose(S[0], S_closed, rtol=1e-13) and N[0] == pytest.approx(N_closed, rel=1e-13)
    assert np.allclose(c[0], S_closed / N_closed, rtol=1e-13)


def test_centroids_stay_in_convex_hull_of_points_ever_assigned():
    """[Blog] "A design note": the EMA keeps each centroid inside the convex hull
    of the points ever assigned to its cluster. Tracked with explicit weights."""
    x = O.search_copy_of_data(synth.hand_shape(600, 4, 6, seed=5).numpy())
    k = 8
    em = O.EmeansOracle(4, k, seed=11, revival="none", closing_mean=False, batch_size=64)
    em.begin(x, 3.0)
    W = np.zeros((k, x.shape[0]))  # weight of each row in each cluster's running sum
    start = em.c.copy()
    ever = [set() for _ in range(k)]
    while not em.done:
        info = em.step()
        a = info["alpha"]
        W *= (1 - a)
        for r, lab in zip(info["ids"], info["labels"]):
            W[lab, r] += a
            ever[lab].add(int(r))
    for j in range(k):
        if em.N[j] > 0:
            assert np.all(W[j] >= 0)
            assert W[j].sum() == pytest.approx(em.N[j], rel=1e-12)
            assert np.allclose(W[j] @ x / W[j].sum(), em.c[j], rtol=1e-10, atol=1e-12)
            pts = x[sorted(ever[j])]
            assert np.all(em.c[j] >= pts.min(0) - 1e-12) and np.all(em.c[j] <= pts.max(0) + 1e-12)
        else:
            assert np.array_equal(em.c[j], start[j])


def test_lloyd_loss_does_not_increase():
    """[Blog] "Lloyd's loss only decreases"; with fp64 search this holds exactly."""
    x = O.search_copy_of_data(synth.hand_shape(2000, 8, 20, seed=6).numpy())
    c = x[O.starting_rows(2000, 16, 1234)].copy()
    hist = []
    for _ in range(15):
        labels, best, _ = O.assign(x, c)
        hist.append(best.mean())
        n_j, s_j = O.batch_stats(x, labels, 16)
        _, _, c = O.ema_update(np.zeros(16), np.zeros_like(c), c, n_j, s_j, 1.0)
    assert np.all(np.diff(hist) <= 1e-12 * hist[0])
    # with the bf16 search copy the decrease holds up to the search rounding
    _, h16 = O.lloyd(x, x[O.starting_rows(2000, 16, 1234)].copy(), 15)
    assert np.all(np.diff(h16) <= 1e-3 * h16[0])


def test_lloyd_iterations_match_a_hand_written_lloyd():
    """[Blog] "Still Lloyd's 1957 algorithm": assign every row to its nearest
    centroid, then move each centroid to the mean of its rows (a centroid with no
    rows stays). Written out with loops; the search uses the bf16 copy of the
    centroids (fp64 -> fp32 -> bf16, by torch's cast), the means are fp64."""
    g = np.random.default_rng(11)
    x = O.search_copy_of_data(g.standard_normal((120, 3)).astype(np.float32))
    c0 = np.vstack([x[:5], [[40.0, 40.0, 40.0]]])  # the last centroid never wins a row
    c = c0.copy()
    hist = []
    for _ in range(3):
        cb = torch.tensor(c, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
        labels = []
        for i in range(len(x)):
            d = [sum((x[i, t] - cb[j, t]) ** 2 for t in range(3)) for j in range(len(c))]
            labels.append(min(range(len(c)), key=lambda q: (d[q], q)))
        hist.append(np.mean([sum((x[i, t] - cb[labels[i], t]) ** 2 for t in range(3)) for i in range(len(x))]))
        new = c.copy()
        for j in range(len(c)):
            rows = [x[i] for i in range(len(x)) if labels[i] == j]
            if rows:
                new[j] = np.sum(rows, axis=0) / len(rows)
        c = new
    c_or, h_or = O.lloyd(x, c0, 3)
    assert np.allclose(c_or, c, rtol=1e-13, atol=1e-13)
    assert np.array_equal(c_or[5], c0[5])
    assert np.allclose(h_or, hist, rtol=1e-12, atol=1e-12)


def test_batch_stats_against_loops():
    g = np.random.default_rng(7)
    rows = g.standard_normal((200, 3))
    lab = g.integers(0, 9, 200)
    n_j, s_j = O.batch_stats(rows, lab, 10)
    for j in range(10):
        assert n_j[j] == sum(1 for v in lab if v == j)
        assert np.allclose(s_j[j], sum((rows[i] for i in range(200) if lab[i] == j), np.zeros(3)), atol=1e-12)


# ---------------------------------------------------------------- revival

def test_dead_set_uses_strict_threshold_on_mean_count():
    N = np.array([10.0, 0.0, 0.99, 1.0, 20.0, 8.01])  # mean 6.666..., threshold 0.6666
    S = N[:, None] * np.ones((6, 2))
    c = np.ones((6, 2))
    _, _, _, dead, donors = O.revive(N, S, c, t=4, seed=1, mode="split", tau=0.1)
    assert dead.tolist() == [1]
    N2 = np.array([10.0, 1.0, 1.0, 1.0, 1.0, 1.0])  # mean 2.5, threshold 0.25 -> none dead
    assert len(O.revive(N2, N2[:, None] * c, c, 4, 1)[3]) == 0
    # a count exactly at the threshold is not below it: mean 1.25, and 0.1 x 1.25
    # rounds to 0.125 exactly in fp64
    N3 = np.array([0.125, 1.875, 1.5, 1.5])
    assert 0.1 * (N3.sum() / 4) == 0.125
    assert len(O.revive(N3, N3[:, None] * c[:4], c[:4], 4, 1, tau=0.1)[3]) == 0
    assert O.revive(N3 * [0.999, 1, 1, 1], N3[:, None] * c[:4], c[:4], 4, 1, tau=0.1)[3].tolist() == [0]


def test_split_halves_count_and_keeps_sums_consistent():
    N = np.array([0.0, 30.0, 50.0, 0.01])
    c = np.array([[9.0, 9.0, 9.0], [1.0, 2.0, 3.0], [-1.0, -2.0, 4.0], [5.0, 5.0, 5.0]])
    S = N[:, None] * c
    N2, S2, c2, dead, donors = O.revive(N, S, c, t=9, seed=5)
    assert dead.tolist() == [0, 3]
    for j, d in zip(dead, donors):
        assert d in (1, 2)
    assert np.allclose(S2, N2[:, None] * c2)
    # counts: every donor halved once per time chosen; the dead take the halves
    assert N2.sum() == pytest.approx(N[1] + N[2])
    eps = O.SPLIT_EPS
    sgn = np.array([1.0, -1.0, 1.0])
    d0 = donors[0]
    assert np.allclose(c2[0], c[d0] * (1 - eps * sgn))


def test_split_is_sequential_a_halved_donor_is_lighter():
    # one heavy donor (index 2) and a light one; after the first dead cluster takes
    # half of the heavy donor, the second draw sees the halved weight
    k = 6
    N = np.array([0.0, 0.0, 1000.0, 0.0, 40.0, 960.0])  # threshold 0.1 * 2000 / 6 = 33.3
    c = np.arange(k * 2, dtype=float).reshape(k, 2)
    S = N[:, None] * c
    counts = {2: 0, 5: 0, 4: 0}
    for t in range(4, 4000, 5):
        N2, _, _, dead, donors = O.revive(N, S, c, t=t, seed=2)
        assert dead.tolist() == [0, 1, 3]
        for d in donors:
            counts[int(d)] += 1
        # replay the draws by hand with the sequentially updated weights
        w = N.copy()
        w[[0, 1, 3]] = 0.0
        u = O.draw_uniform(2, O.STREAM_REVIVE, t, dead)
        for i in range(3):
            cdf = np.cumsum(w)
            pick = int(np.searchsorted(cdf, u[i] * cdf[-1], side="right"))
            assert pick == donors[i]
            w[pick] /= 2.0
    # donors are drawn in proportion to size: the tiny cluster is almost never picked
    assert counts[4] < 0.05 * (counts[2] + counts[5])
    assert 0.8 < counts[2] / counts[5] < 1.25


def test_donor_frequency_proportional_to_size():
    k = 5
    N = np.array([0.0, 10.0, 20.0, 30.0, 40.0])
    c = np.ones((k, 2))
    hits = np.zeros(k)
    trials = 6000
    for t in range(trials):
        _, _, _, dead, donors = O.revive(N, N[:, None] * c, c, t=5 * t + 4, seed=3)
        hits[donors[0]] += 1
    expect = np.array([0, 0.1, 0.2, 0.3, 0.4]) * trials
    chi2 = sum((hits[i] - expect[i]) ** 2 / expect[i] for i in range(1, k))
    assert hits[0] == 0 and chi2 < 16.3  # 3 dof, p = 0.001


def test_resample_and_none_modes():
    N = np.array([0.0, 5.0, 5.0])
    c = np.zeros((3, 2))
    S = N[:, None] * c
    batch = np.array([[7.0, 7.0], [8.0, 8.0], [9.0, 9.0]])
    N2, S2, c2, dead, picks = O.revive(N, S, c, t=4, seed=1, mode="resample", batch_rows=batch)
    assert dead.tolist() == [0] and N2[0] == 0 and np.all(S2[0] == 0)
    assert any(np.array_equal(c2[0], b) for b in batch)
    N3, S3, c3, dead3, _ = O.revive(N, S, c, t=4, seed=1, mode="none")
    assert len(dead3) == 0 and np.array_equal(N3, N) and np.array_equal(c3, c)


def test_revival_happens_every_fifth_step_only():
    x = O.search_copy_of_data(synth.hand_shape(2000, 8, 10, seed=8).numpy())
    em = O.EmeansOracle(8, 64, seed=1, batch_size=128)
    em.begin(x, 1.0)
    checks = []
    while not em.done:
        info = em.step()
        checks.append(info["revived"] is not None)
    assert checks == [(t + 1) % 5 == 0 for t in range(len(checks))]


def _unused_fraction(xq, c, tau=0.1):
    labels, _, _ = O.assign(xq, O.search_copy_of_centroids(c))
    cnt = np.bincount(labels, minlength=c.shape[0])
    return np.mean(cnt < tau * cnt.mean())


def test_revival_ablation_ordering_on_stand_in_data():
    """Ordering of the pages' ablation (fixture): split leaves far fewer unused
    clusters than no revival, resample sits in between, and the test loss follows."""
    g = golden("revival_ablation.json")["arms"]
    assert g["split"]["dead"] < g["resample"]["dead"] < g["none"]["dead"]
    xt, xs = synth.subspace_mixture(31250, 5000, 96, 25000, 1.5, 0, "cpu")
    xq, xtq = O.search_copy_of_data(xt.numpy()), O.search_copy_of_data(xs.numpy())
    res = {}
    for mode in ("split", "resample", "none"):
        em = O.EmeansOracle(96, 512, seed=0, revival=mode)
        c, _ = em.train(xq, 5.0)
        res[mode] = (_unused_fraction(xq, c), O.mse(xtq, c))
    assert res["split"][0] < 0.02 and res["none"][0] > 0.15
    assert res["split"][0] <= res["resample"][0] <= res["none"][0]
    assert res["split"][1] < res["none"][1]


def test_low_dimension_defaults():
    """[README] `batch_law` / `unused_threshold` and "Note on low dimension": the
    default ("auto") batch law is the quality law for d <= 16 and the throughput law
    above; for d <= 2 the default threshold is 0, so no cluster is ever revived."""
    n, k, T = 200_000, 256, 5.0
    for d, law in ((2, "quality"), (16, "quality"), (17, "throughput"), (768, "throughput")):
        em = O.EmeansOracle(d, k)
        assert em.law == law
        assert O.recipe(n, k, T, law)["batch_size"] == O.recipe(n, k, T, em.law)["batch_size"]
    assert O.EmeansOracle(2, k).tau == 0.0 and O.EmeansOracle(3, k).tau == O.DEFAULT_TAU
    # the quality batch differs from the throughput batch at these sizes (so the rule shows)
    assert O.recipe(n, k, T, "quality")["batch_size"] < O.recipe(n, k, T, "throughput")["batch_size"]
    # d = 2: a revival check with every cluster but one dead revives nothing
    em = O.EmeansOracle(2, 4, seed=1)
    em.N = np.array([100.0, 0.0, 0.0, 0.0])
    em.S = np.zeros((4, 2))
    em.c = np.arange(8.0).reshape(4, 2)
    dead, donors = em.maybe_revive(np.zeros((10, 2)), t=4)
    assert len(dead) == 0 and len(donors) == 0 and np.array_equal(em.N, [100.0, 0.0, 0.0, 0.0])


# ---------------------------------------------------------------- whole runs

def test_blog_toy_lloyd_stuck_and_emeans_can_escape():
    """[Blog] Figure 2 simulation, on our own blob data: Lloyd from the bad start
    stays with two centroids in one blob; e-means (25 updates) escapes for some
    seeds. The pages' values (5.39, 1.28) are for unpublished data: unpinned."""
    g = golden("blog_toy.json")
    x, start = datagen.blobs3()
    x, start = x.numpy(), start.numpy()
    c = start.copy()
    for _ in range(g["lloyd_passes_reported"]):
        labels, best, _ = O.assign(x, c)
        n_j, s_j = O.batch_stats(x, labels, 3)
        _, _, c = O.ema_update(np.zeros(3), np.zeros_like(c), c, n_j, s_j, 1.0)
    lloyd_mse = O.assign(x, c)[1].mean()
    escaped = 0
    for seed in range(1, 9):
        em = O.EmeansOracle(2, 3, seed=seed, batch_size=g["batch_size"], alpha0=g["alpha0"], closing_mean=False)
        em.begin(x, g["epochs"])
        em.c = start.copy()
        n_up = 0
        while not em.done:
            em.step()
            n_up += 1
        assert n_up == g["emeans_updates"]
        escaped += O.assign(x, em.c)[1].mean() < 0.5 * lloyd_mse
    assert lloyd_mse > 10.0 and escaped >= 1


def test_tiny_run_beats_lloyd25_and_respects_noise_floor():
    w, xt, xs = datagen.make("tiny")
    xq, xtq = O.search_copy_of_data(xt.numpy()), O.search_copy_of_data(xs.numpy())
    em = O.EmeansOracle(w.d, w.k, seed=1234)
    c, labels = em.train(xq, w.epochs)
    assert em.r["total_steps"] == 50 and em.r["batch_size"] == 1024
    assert np.all(labels >= 0)
    c0 = xq[O.starting_rows(len(xq), w.k, 1234)]
    cl, _ = O.lloyd(xq, c0, 25)
    e_mse, l_mse = O.mse(xtq, c), O.mse(xtq, cl)
    floor = synth.expected_tiny_noise_floor(w.d)
    assert e_mse < l_mse
    assert e_mse > 0.9 * floor
    # the per-pass error decreases over the run
    assert em.obj[-1] < em.obj[0]


def test_closing_mean_is_exact_mean_of_last_pass_assignments():
    x = O.search_copy_of_data(synth.hand_shape(3000, 6, 12, seed=9).numpy())
    em = O.EmeansOracle(6, 16, seed=4)
    c, labels = em.train(x, 2.0)
    for j in range(16):
        m = labels == j
        if m.any():
            assert np.allclose(c[j], x[m].mean(axis=0), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- spherical e-means

def _unit(x):
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def test_unit_rows_rescales_and_keeps_zero_rows():
    c = np.array([[3.0, 4.0], [0.0, 0.0], [-1e-3, 0.0]])
    u = O.unit_rows(c)
    assert np.allclose(u[0], [0.6, 0.8]) and np.array_equal(u[1], [0.0, 0.0]) and np.allclose(u[2], [-1.0, 0.0])


def test_assign_dot_matches_brute_force_with_lowest_index_ties():
    g = np.random.default_rng(5)
    x = O.search_copy_of_data(_unit(g.standard_normal((60, 5))))
    c = O.search_copy_of_centroids(_unit(g.standard_normal((9, 5))))
    c[7] = c[2]  # an exact tie: the lower index must win
    labels, best, second = O.assign_dot(x, c)
    for i in range(60):
        dots = [float(np.dot(x[i], c[j])) for j in range(9)]
        top = max(dots)
        assert labels[i] == dots.index(top) and best[i] == top
        assert second[i] == sorted(dots)[-2]


def test_similarity_and_distance_agree_on_the_unit_sphere():
    """[README] "Spherical e-means": on vectors of norm 1 the squared distance is
    2 - 2 x cosine, so the highest dot product is the nearest centroid."""
    g = np.random.default_rng(6)
    x, c = _unit(g.standard_normal((500, 12))), _unit(g.standard_normal((40, 12)))
    d2 = O.squared_distances(x, c)
    assert np.allclose(d2, 2.0 - 2.0 * (x @ c.T), atol=1e-12)
    assert np.array_equal(np.argmin(d2, axis=1), np.argmax(x @ c.T, axis=1))


def test_spherical_lloyd_step_is_the_normalised_mean():
    """B = n and alpha = 1: one spherical update is each cluster's mean rescaled to
    norm 1 (brute force over the assignment)."""
    g = np.random.default_rng(7)
    xq = O.search_copy_of_data(_unit(g.standard_normal((400, 6))))
    c0 = _unit(g.standard_normal((5, 6)))
    c1, hist = O.lloyd(xq, c0, 1, spherical=True)
    cq = O.search_copy_of_centroids(O.unit_rows(c0))
    for j in range(5):
        members = [i for i in range(400) if int(np.argmax(xq[i] @ cq.T)) == j]
        if members:
            m = xq[members].mean(axis=0)
            assert np.allclose(c1[j], m / np.linalg.norm(m), atol=1e-12)
    assert hist[0] == pytest.approx(float(np.mean(2.0 - 2.0 * (xq @ cq.T).max(axis=1))))


def test_spherical_run_keeps_unit_centroids_and_error_definition():
    g = np.random.default_rng(8)
    xq = O.search_copy_of_data(_unit(g.standard_normal((3000, 8)) + np.repeat(g.standard_normal((6, 8)) * 3, 500, 0)))
    em = O.EmeansOracle(8, 12, seed=2, spherical=True, law="throughput")
    c, _ = em.train(xq, 2.0)
    nrm = np.linalg.norm(c, axis=1)
    assert np.allclose(nrm[nrm > 0], 1.0, atol=1e-12)
    err = O.spherical_error(xq, c)
    _, sim, _ = O.assign_dot(xq, O.search_copy_of_centroids(c))
    assert err == pytest.approx(float(np.mean(2.0 - 2.0 * sim))) and 0.0 <= err < 2.0
    # it clusters: far below the error of one random unit centroid per row (about 2)
    assert err < 1.0


# ---------------------------------------------------------------- FP8 search

def test_e4m3_table_fixed_points():
    """E4M3 (OCP 8-bit float, 4 exponent bits, bias 7, no infinities): 1.0 is
    0x38, the largest value 448 is 0x7E, the smallest subnormal 2^-9 is 0x01 and
    the smallest normal 2^-6 is 0x08; values grow with the code."""
    t = O.e4m3_table()
    assert len(t) == 127 and np.all(np.diff(t) > 0)
    assert t[0x38] == 1.0 and t[0x7E] == 448.0 and t[0x01] == 2.0 ** -9 and t[0x08] == 2.0 ** -6
    assert t[0x07] == 7.0 / 8.0 * 2.0 ** -6 and t[0x7D] == 416.0


def test_e4m3_rounding_matches_torch_and_breaks_ties_to_even():
    """Nearest rounding against torch's float8_e4m3fn cast (an independent library
    routine) on in-range values, every exact midpoint between neighbouring codes
    going to the even code, and saturation of finite values beyond 448."""
    g = np.random.default_rng(12)
    x = np.concatenate([g.standard_normal(20000) * 60.0, g.standard_normal(5000) * 1e-2,
                        g.uniform(-448, 448, 5000)])
    ref = torch.tensor(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(O.e4m3_round(x), ref)
    t = O.e4m3_table()
    mids = (t[:-1] + t[1:]) / 2.0
    got = O.e4m3_round(mids)
    codes = np.searchsorted(t, got)
    assert np.all(codes % 2 == 0) and np.all(t[codes] == got)
    assert np.array_equal(O.e4m3_round(-mids), -got)
    assert np.array_equal(O.e4m3_round([449.0, 463.9, 1e6, -5000.0]), [448.0, 448.0, 448.0, -448.0])


def test_fp8_calibration_is_midrange_shift_and_largest_power_of_two():
    g = np.random.default_rng(13)
    x = O.search_copy_of_data(g.standard_normal((3000, 9)) * np.arange(1, 10) + np.arange(9) * 5.0)
    shift, scale = O.fp8_calibrate(x)
    lo, hi = x.min(axis=0), x.max(axis=0)
    assert np.array_equal(shift, ((lo.astype(np.float32) + hi.astype(np.float32)) * np.float32(0.5)))
    m = np.maximum(hi - shift, shift - lo).max()
    assert math.log2(scale) == int(math.log2(scale))
    assert m * scale <= 448.0 < m * scale * 2.0
    # only the first rows calibrate; a constant sample keeps scale 1
    big = np.vstack([x, np.full((1, 9), 1e9)])
    assert O.fp8_calibrate(big[: len(x)])[1] == scale
    assert O.fp8_calibrate(np.ones((10, 3)))[1] == 1.0


def test_fp8_search_is_the_argmin_over_codes():
    """Brute force on tiny inputs: the FP8 search picks the centroid whose codes are
    nearest to the row's codes (ties to the lowest index), and reports that
    squared distance divided by scale^2."""
    g = np.random.default_rng(14)
    x = O.search_copy_of_data(g.standard_normal((40, 5)) * 3.0)
    c = g.standard_normal((7, 5)) * 3.0
    shift, scale = O.fp8_calibrate(x)
    lab, best, _ = O.assign_fp8(x, c, shift, scale)
    xc, cc = O.fp8_codes(x, shift, scale), O.fp8_codes(O.to_f32(c), shift, scale)
    for i in range(40):
        d = [float(((xc[i] - cc[j]) ** 2).sum()) for j in range(7)]
        assert lab[i] == d.index(min(d)) and best[i] == min(d) / scale ** 2


def test_fp8_distances_within_the_quantisation_bound():
    """Each code is within half an E4M3 step (relative 2^-4, or 2^-10 among the
    subnormals) of a = (x - shift) * scale. By the triangle inequality the FP8
    distance |x' - c'| of a row to a centroid is then within |x' - a| + |c' - b| of
    |a - b|; on separated clusters the FP8 and bf16 searches pick the same labels."""
    g = np.random.default_rng(15)
    mu = g.standard_normal((6, 16)) * 20.0
    x = O.search_copy_of_data(mu[g.integers(6, size=2000)] + g.standard_normal((2000, 16)))
    shift, scale = O.fp8_calibrate(x)
    xc = O.fp8_codes(x, shift, scale)
    a = (x.astype(np.float32) - shift).astype(np.float64) * scale
    assert np.all(np.abs(xc - a) <= np.maximum(np.abs(a) * 2.0 ** -4, 2.0 ** -10) + 1e-12)
    lab8, best8, _ = O.assign_fp8(x, mu, shift, scale)
    lab, _, _ = O.assign(x, O.search_copy_of_centroids(mu))
    assert np.mean(lab8 == lab) == 1.0
    cc = O.fp8_codes(O.to_f32(mu), shift, scale)
    b = (O.to_f32(mu) - shift).astype(np.float64) * scale
    ex, ec = np.linalg.norm(xc - a, axis=1), np.linalg.norm(cc - b, axis=1)
    d_exact = np.linalg.norm(a - b[lab8], axis=1)
    assert np.all(np.abs(np.sqrt(best8) * scale - d_exact) <= ex + ec[lab8] + 1e-9)


def test_fp8_training_run_clusters_like_bf16():
    """An FP8-search run of the oracle on separated clusters ends near the bf16
    run (same rows, same seed): the search precision is the only change."""
    g = np.random.default_rng(16)
    mu = g.standard_normal((12, 8)) * 10.0
    x = O.search_copy_of_data(mu[g.integers(12, size=6000)] + g.standard_normal((6000, 8)))
    e8 = O.EmeansOracle(8, 16, seed=3, search="fp8")
    e16 = O.EmeansOracle(8, 16, seed=3)
    c8, _ = e8.train(x, 2.0)
    c16, _ = e16.train(x, 2.0)
    assert e8.fp8 is not None and e16.fp8 is None
    assert abs(O.mse(x, c8) - O.mse(x, c16)) <= 0.05 * O.mse(x, c16)
    with pytest.raises(ValueError):
        O.EmeansOracle(8, 16, spherical=True, search="fp8")
