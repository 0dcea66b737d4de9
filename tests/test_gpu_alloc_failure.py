"""Out-of-memory paths, exercised by failing one device allocation at a time.

em_fail_allocation makes the library's nth device allocation fail as a failed
cudaMalloc does, without running out of memory (no GPU fault is involved: the
allocation is never made). The test counts the allocations of a whole sequence
(create, train, assign, Lloyd, FP8 and spherical runs), then fails each one in
turn and checks that:
* the failing call returns EM_E_NOMEM (em_create: NULL with that code);
* the model it leaves can be destroyed;
* or used again: with injection off, the same calls then give the same centroids,
  bit for bit, as a model that never failed;
* no device memory is left behind.
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


def _calls(em, m, x, xs):
    """The sequence of calls under test on model m; returns its final centroids."""
    m.train(x, epochs=2.5)
    lab = torch.empty(xs.shape[0], dtype=torch.int64, device="cuda")
    m.assign(xs, labels=lab)
    m.mse(xs)
    m.lloyd(x, 3)
    m.train(x[:1500], epochs=1.0)  # a smaller run after a larger one
    c = torch.empty(m.k, m.d, device="cuda")
    m.centroids(c)
    return c.cpu()


@pytest.mark.parametrize("options", [{}, {"search_format": 1}, {"spherical": 1}])
def test_every_allocation_failure_is_reported_and_recoverable(em, options):
    d, k = 40, 24
    x = synth.hand_shape(3000, d, 12, seed=11).cuda()
    xs = synth.hand_shape(700, d, 12, seed=12).cuda()
    em.fail_allocation(0)
    m = em.Model(d, k, seed=77, **options)
    ref = _calls(em, m, x, xs)
    m.close()
    total = em.fail_allocation(0)
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    assert total >= 20, total
    for nth in range(1, total + 1):
        em.fail_allocation(nth)
        try:
            m = em.Model(d, k, seed=77, **options)
        except em.EmeansError as e:
            assert e.code == em.EM_E_NOMEM, (nth, str(e))
            em.fail_allocation(0)
            continue
        try:
            _calls(em, m, x, xs)
            failed = False
        except em.EmeansError as e:
            assert e.code == em.EM_E_NOMEM, (nth, str(e))
            assert b"injected" in em.em_last_error()
            failed = True
        assert failed, f"allocation {nth} of {total} was not reported"
        em.fail_allocation(0)
        if nth % 2:  # reuse the model that failed: the same calls give the same centroids
            again = _calls(em, m, x, xs)
            assert torch.equal(again, ref), f"allocation {nth}: the reused model differs"
        m.close()  # or just destroy it
    em.fail_allocation(0)
    torch.cuda.synchronize()
    # nothing leaked: every model above was destroyed, failed or not
    assert torch.cuda.mem_get_info()[0] >= free_before - (8 << 20)
