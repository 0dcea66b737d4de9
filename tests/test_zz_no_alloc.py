"""em_assign_noalloc, the assignment entry point that allocates nothing.

Some callers cannot call cudaMalloc: their device memory belongs to another
allocator or is fixed when the process starts (a serving process that forbids
allocation after start-up, a library running inside a framework's memory pool).
For them the library offers one assignment call whose scratch lives in a
file-scope device array. This test calls it through the C ABI, several times in a
row (each call reuses the shared scratch array the one before filled), and checks
its labels and distances against the fp64 oracle and against the ones em_assign
(the allocating entry point) returns, with the tolerances of the other parity
tests, at the documented limits too: the largest row count, the largest k and
k x d, and a row count where the fixed key region lowers the search's split.

The file name makes pytest collect it last, so a run that stops at the first
failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _noalloc(em, x, c, n, d, k):
    labels = torch.empty(n, dtype=torch.int64, device="cuda")
    dists = torch.empty(n, dtype=torch.float32, device="cuda")
    rc = em.lib.em_assign_noalloc(x.data_ptr(), n, d, c.data_ptr(), k, labels.data_ptr(), dists.data_ptr(),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == em.EM_OK, em.em_last_error()
    return labels.cpu().numpy(), dists.cpu().numpy()


def _allocating(em, x, c, n, d, k):
    m = em.Model(d, k, seed=1)
    m.set_state(c=c)
    labels = torch.empty(n, dtype=torch.int64, device="cuda")
    dists = torch.empty(n, dtype=torch.float32, device="cuda")
    m.assign(x, labels=labels, dists=dists)
    m.close()
    return labels.cpu().numpy(), dists.cpu().numpy()


def _against_oracle(x, c, got):
    """Labels and distances of em_assign_noalloc against the fp64 oracle's search on
    the same bf16 rows and bf16 copies of the centroids (near-tie rule, tests/helpers.py)."""
    from oracle import emeans_oracle as O
    from tests.helpers import LabelBook, threaded_assign

    lab, dist = got
    xq = O.search_copy_of_data(x.float().cpu().numpy())
    cq = O.search_copy_of_centroids(c.cpu().numpy().astype(np.float64))
    book = LabelBook()
    orig = O.assign
    O.assign = threaded_assign(orig)
    try:
        _, best = book.compare(lab, xq, cq)
    finally:
        O.assign = orig
    book.finish()
    xn = np.einsum("ij,ij->i", xq, xq)
    np.testing.assert_allclose(dist, best, rtol=1e-4, atol=1e-5 * (xn.mean() + 1))


def _against_em_assign(x, c, got, ref):
    from oracle import emeans_oracle as O
    from tests.helpers import LABEL_GAP_REL, LABEL_MISMATCH_FRACTION

    (lab, dist), (lab_ref, dist_ref) = got, ref
    diff = np.flatnonzero(lab != lab_ref)
    if len(diff):
        xq = x.float().cpu().numpy().astype(np.float64)[diff]
        cq = O.search_copy_of_centroids(c.cpu().numpy().astype(np.float64))
        d_got = ((xq - cq[lab[diff]]) ** 2).sum(axis=1)
        d_ref = ((xq - cq[lab_ref[diff]]) ** 2).sum(axis=1)
        assert np.all(np.abs(d_got - d_ref) <= LABEL_GAP_REL * np.minimum(d_got, d_ref)), "labels differ"
    assert len(diff) <= max(1, int(LABEL_MISMATCH_FRACTION * len(lab)))
    np.testing.assert_allclose(dist, dist_ref, rtol=1e-4, atol=1e-6)


def _case(n, d, k, seed):
    from datagen import synth

    x32 = synth.hand_shape(n, d, 24, seed=seed)
    g = torch.Generator().manual_seed(seed)
    c = (x32[torch.randint(0, n, (k,), generator=g)] + 0.2 * torch.randn(k, d, generator=g)).float()
    return x32.to(torch.bfloat16).cuda().contiguous(), c


def test_noalloc_assignment_matches_oracle_and_em_assign_on_calls_in_a_row():
    """Calls in a row, each against the oracle and against em_assign:
    * 20,000 x 128 rows, k = 1,000;
    * 777 x 768 rows, k = 300 (smaller than the call before: stale scratch must not leak);
    * 524,288 x 64 rows, k = 512: the largest row count, the whole key region in use;
    * 3,000 x 64 rows, k = 65,536: the largest k and k x d = 4,194,304, the whole
      operand region in use;
    * 90,000 x 128 rows, k = 4,096: em_assign splits each row tile of the last wave
      8 ways, which the key region cannot hold at this row count, so this call
      splits at most 4 ways (split x rows <= the row limit)."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mini_ema_means_b200 as em

    torch.cuda.set_device(0)
    assert em.EM_NOALLOC_MAX_ROWS == 524288 and em.EM_NOALLOC_MAX_K * 64 == em.EM_NOALLOC_MAX_KD
    split, _ = em.search_schedule(90000, 4096, torch.cuda.get_device_properties(0).multi_processor_count)
    assert split * 90000 > em.EM_NOALLOC_MAX_ROWS  # the capped schedule really differs here
    cases = [(20000, 128, 1000, 5), (777, 768, 300, 6), (em.EM_NOALLOC_MAX_ROWS, 64, 512, 7),
             (3000, 64, em.EM_NOALLOC_MAX_K, 8), (90000, 128, 4096, 9)]
    for n, d, k, seed in cases:
        x, c = _case(n, d, k, seed)
        cd = c.cuda().contiguous()
        got = _noalloc(em, x, cd, n, d, k)
        _against_oracle(x, c, got)
        _against_em_assign(x, c, got, _allocating(em, x, cd, n, d, k))


def test_noalloc_rejects_sizes_beyond_its_limit():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mini_ema_means_b200 as em

    x = torch.zeros(16, 8, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(4, 8, device="cuda")
    out = torch.empty(16, dtype=torch.int64, device="cuda")
    rc = em.lib.em_assign_noalloc(x.data_ptr(), em.EM_NOALLOC_MAX_ROWS + 1, 8, c.data_ptr(), 4, out.data_ptr(),
                                  None, None)
    assert rc == em.EM_E_INVAL and b"rows" in em.em_last_error()
    rc = em.lib.em_assign_noalloc(x.data_ptr(), 16, 12, c.data_ptr(), 4, out.data_ptr(), None, None)
    assert rc == em.EM_E_INVAL
