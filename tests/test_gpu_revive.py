"""Revival check on the GPU against the fp64 oracle, from crafted running counts.

The donor search keeps a tree of prefix sums whose shape depends on k (up to
16,384 clusters a root of group totals in registers over groups of 32, 64 or 128
clusters in shared memory, the root holding up to 32, 64 or 128 entries; up to
1,048,576 a root over a shared-memory level over groups of 128 in global memory,
prefetched ahead of the draws; above that radix-128 levels), so k runs over the
boundaries of those shapes. Each case sets
N, S and c, runs one revival check through the C ABI and compares with the
oracle's revival (split arm: sequential size-proportional donor draws):

* the running counts bit for bit, after rounding the oracle's fp64 halvings to
  the fp32 the state is stored in;
* the centroids of every cluster the check touched (per-centroid relative L2);
* the number of dead clusters and of splits.

Patterns: random counts with a dead fraction (300 dead clusters at the largest
k, where the oracle recomputes a million-entry cumulative sum per draw); one live
cluster serving every dead one (its weight halves at each draw until it runs out,
so the later dead clusters stay unrevived); a few heavy clusters among many light
ones.
"""

import numpy as np
import pytest
import torch

from oracle import emeans_oracle as O
from tests.helpers import assert_centroids_close

pytestmark = pytest.mark.gpu

SEED = 99


@pytest.fixture(scope="module")
def em():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mini_ema_means_b200

    return mini_ema_means_b200


def _counts(pattern, k, rng):
    if pattern == "random":
        N = rng.uniform(0.5, 200.0, size=k)
        dead = rng.random(k) < min(0.2, 3000.0 / k)
        N[dead] = rng.uniform(0.0, 1.0, size=int(dead.sum()))
    elif pattern == "one_live":
        N = np.zeros(k)
        N[rng.integers(k)] = 1000.0
    elif pattern == "few_dead":  # (300 dead clusters: keeps the oracle's sequential draws short at large k)
        N = rng.uniform(20.0, 200.0, size=k)
        dead = rng.choice(k, size=min(k, 300), replace=False)
        N[dead] = rng.uniform(0.0, 1.0, size=len(dead))
    elif pattern == "heavy_few":
        N = rng.uniform(0.0, 0.5, size=k)
        heavy = rng.choice(k, size=max(1, k // 50), replace=False)
        N[heavy] = rng.uniform(100.0, 5000.0, size=len(heavy))
    else:
        raise KeyError(pattern)
    return N.astype(np.float32)


def _model_at_step_one(em, k, d):
    """A running model of k clusters on n >= k rows, after one step."""
    n = max(k, 256)
    x = torch.from_numpy(np.random.default_rng(k).standard_normal((n, d)).astype(np.float32)).cuda()
    m = em.Model(d, k, seed=SEED, auto_revive=0, revival="split", batch_size=min(n, 4096))
    m.begin(x, epochs=1.0)
    assert m.step(1) == 1
    return m


CASES = [(k, "random") for k in (1, 2, 31, 33, 127, 128, 129, 1024, 1025, 2048, 2049, 4096, 4097, 8192,
                                 8193, 16383, 16384, 16385, 20000, 65536, 131073, 300000)]
CASES += [(600000, "few_dead"), (1100000, "few_dead")]
CASES += [(4096, "one_live"), (300, "one_live"), (8000, "one_live"), (16000, "one_live"), (70000, "one_live")]
CASES += [(16384, "heavy_few"), (8193, "heavy_few"), (2000, "heavy_few"), (65536, "heavy_few")]


@pytest.mark.parametrize("k,pattern", CASES)
def test_revival_matches_oracle(em, k, pattern):
    d = 8
    rng = np.random.default_rng(k * 7 + len(pattern))
    N = _counts(pattern, k, rng)
    c = rng.standard_normal((k, d)).astype(np.float32)
    S = (N[:, None] * c).astype(np.float32)
    m = _model_at_step_one(em, k, d)
    m.set_state(N=torch.from_numpy(N).cuda(), S=torch.from_numpy(S).cuda(), c=torch.from_numpy(c).cuda(), step=1)
    m.revive()
    N2 = torch.empty(k)
    c2 = torch.empty(k, d)
    m.get_state(N=N2, c=c2)
    # the check after global step t = 0 (the revival draws are keyed by it)
    Nr, _, cr, dead, donors = O.revive(N.astype(np.float64), S.astype(np.float64), c.astype(np.float64), 0, SEED)
    st = m.stats()
    assert st["last_dead"] == len(dead)
    np.testing.assert_array_equal(N2.numpy(), Nr.astype(np.float32))
    touched = np.unique(np.concatenate([dead, donors[donors >= 0]])).astype(np.int64)
    if len(touched):
        assert_centroids_close(c2.numpy().astype(np.float64)[touched], cr[touched], f"k={k} {pattern}")
    untouched = np.setdiff1d(np.arange(k), touched)
    assert np.array_equal(c2.numpy()[untouched], c[untouched])
    if pattern == "one_live" and k > 1100:
        # the single donor's weight underflows to zero before every dead cluster is served
        assert (donors < 0).any()
    m.close()
