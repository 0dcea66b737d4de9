"""em_assign_noalloc, the assignment entry point that allocates nothing.

Some callers cannot call cudaMalloc: their device memory belongs to another
allocator or is fixed when the process starts (a serving process that forbids
allocation after start-up, a library running inside a framework's memory pool).
For them the library offers one assignment call whose scratch lives in a
file-scope device array. This test calls it through the C ABI and checks its
labels and distances against the ones em_assign (the allocating entry point)
returns, with the tolerances of the other parity tests, on two calls in a row:
the second call reuses the shared scratch array the first one filled.

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


def _compare(x, c, got, ref):
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


def test_noalloc_assignment_matches_em_assign_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import mini_ema_means_b200 as em
    from datagen import synth

    torch.cuda.set_device(0)
    cases = [(20000, 128, 1000, 5), (777, 768, 300, 6)]  # the second call is smaller: stale scratch must not leak
    for n, d, k, seed in cases:
        x32 = synth.hand_shape(n, d, 24, seed=seed)
        g = torch.Generator().manual_seed(seed)
        c = (x32[torch.randint(0, n, (k,), generator=g)] + 0.2 * torch.randn(k, d, generator=g)).float()
        x = x32.to(torch.bfloat16).cuda().contiguous()
        cd = c.cuda().contiguous()
        got = _noalloc(em, x, cd, n, d, k)
        ref = _allocating(em, x, cd, n, d, k)
        _compare(x, c, got, ref)


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
