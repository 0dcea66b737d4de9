"""bench.py counts, for every timed step, the rows the step processes: a full batch,
or what is left of its pass. Checked against the oracle's recipe (rows of each pass
and steps per pass) on the host recipe of the library, without a GPU."""

import pytest

from oracle import emeans_oracle as O


@pytest.mark.parametrize("n,k,epochs", [(10_000, 64, 5.0), (12_345, 100, 2.5), (1_000_000, 4096, 5.0),
                                        (1000, 10, 0.5), (65_537, 300, 1.25), (100_000, 16_384, 3.0)])
def test_step_rows_follow_the_passes(n, k, epochs):
    import bench
    import mini_ema_means_b200 as em

    rec = em.compute_recipe(n, k, epochs)
    ref = O.recipe(n, k, epochs)
    assert rec["batch_size"] == ref["batch_size"] and rec["total_steps"] == ref["total_steps"]
    got = [bench.step_rows(rec, n, s) for s in range(rec["total_steps"])]
    B = ref["batch_size"]
    want = []
    for rows, steps in zip(ref["epoch_rows"], ref["steps_per_pass"]):
        want += [B] * (steps - 1) + [rows - (steps - 1) * B]
    assert got == want
    assert sum(got) == sum(ref["epoch_rows"]) and min(got) > 0
