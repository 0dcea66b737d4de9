"""The oracle's pins catch plausible mistakes. Each case plants one mistake in one
oracle function on the CPU (a dropped term, a wrong sign, index or constant, a
rounding mode, a threshold's strictness), runs the pins that tie that function to
the pages or to mathematics, and expects at least one of them to fail. Nothing
here touches the CUDA path."""

import functools

import numpy as np
import pytest

from oracle import emeans_oracle as O
from tests import test_oracle_pins as P

_orig = {name: getattr(O, name) for name in (
    "ema_update", "alpha_at", "squared_distances", "assign", "batch_stats", "f32_to_bf16", "revive",
    "split_sign", "philox4x64_10", "pass_order", "batch_size_law", "alpha0_law", "unit_rows", "e4m3_round",
    "fp8_calibrate", "assign_dot", "round_batch", "EmeansOracle", "draw_uniform", "lloyd", "assign_fp8")}


# ---------------------------------------------------------------- the mistakes

def ema_without_decay(N, S, c, n_j, s_j, alpha):
    """N and S keep their old values in full: the (1 - alpha) factor is dropped."""
    N = N + alpha * n_j
    S = S + alpha * s_j
    c = c.copy()
    live = N > 0
    c[live] = S[live] / N[live][:, None]
    return N, S, c


def ema_weights_swapped(N, S, c, n_j, s_j, alpha):
    """alpha on the old statistics and (1 - alpha) on the batch's."""
    return _orig["ema_update"](n_j, s_j, c, N, S, alpha)


def alpha_to_zero(t, total_steps, alpha0):
    """The cosine reaches 0 instead of a tenth of alpha0."""
    import math
    frac = 0.0 if total_steps <= 1 else t / (total_steps - 1)
    return alpha0 * 0.5 * (1.0 + math.cos(math.pi * frac))


def alpha_linear(t, total_steps, alpha0):
    """A linear decay between the right endpoints instead of the cosine."""
    frac = 0.0 if total_steps <= 1 else t / (total_steps - 1)
    return alpha0 - 0.9 * alpha0 * frac


def alpha_power(t, total_steps, alpha0):
    """A power-law decay between the right endpoints (not symmetric about the middle)."""
    frac = 0.0 if total_steps <= 1 else t / (total_steps - 1)
    return alpha0 - 0.9 * alpha0 * frac ** 1.5


def alpha_smoothstep(t, total_steps, alpha0):
    """A smoothstep decay 1 - (3f^2 - 2f^3): right endpoints, decreasing and symmetric
    about the middle like the cosine, but a different curve."""
    frac = 0.0 if total_steps <= 1 else t / (total_steps - 1)
    return 0.1 * alpha0 + 0.9 * alpha0 * (1.0 - (3.0 * frac ** 2 - 2.0 * frac ** 3))


def distances_without_centroid_norm(xq, cq):
    """|x|^2 - 2 x.c: the |c|^2 term is dropped."""
    xn = np.einsum("ij,ij->i", xq, xq)
    return xn[:, None] - 2.0 * (xq @ cq.T)


def distances_with_plus_cross_term(xq, cq):
    """|x|^2 + |c|^2 + 2 x.c: the cross term's sign is wrong."""
    xn = np.einsum("ij,ij->i", xq, xq)
    cn = np.einsum("ij,ij->i", cq, cq)
    return xn[:, None] + cn[None, :] + 2.0 * (xq @ cq.T)


def assign_ties_to_highest(xq, cq, chunk=4096):
    """Ties go to the highest centroid index."""
    k = cq.shape[0]
    labels, best, second = _orig["assign"](xq, cq[::-1], chunk)
    return (k - 1 - labels), best, second


def stats_labels_shifted(rows, labels, k):
    """Each row's statistics land on the next cluster (an index off by one)."""
    return _orig["batch_stats"](rows, (labels + 1) % k, k)


def bf16_truncates(x32):
    """bf16 by truncation instead of round-to-nearest-even."""
    x32 = np.ascontiguousarray(x32, dtype=np.float32)
    u = x32.view(np.uint32)
    return (u & np.uint32(0xFFFF0000)).view(np.float32)


def revive_threshold_not_strict(N, S, c, t, seed, mode="split", tau=O.DEFAULT_TAU, batch_rows=None):
    """A cluster exactly at tau x the mean count counts as dead (<= instead of <)."""
    return _orig["revive"](N, S, c, t, seed, mode=mode, tau=tau * (1.0 + 1e-12), batch_rows=batch_rows)


def split_sign_flipped(d):
    """The perturbation's signs are the other way round."""
    return -_orig["split_sign"](d)


def philox_keys_swapped(c0, c1, c2, c3, k0, k1):
    """The two key words are swapped."""
    return _orig["philox4x64_10"](c0, c1, c2, c3, k1, k0)


def pass_order_not_a_bijection(n, seed, pass_index):
    """An off-by-one in the cycle walk: the last position repeats another row."""
    p = _orig["pass_order"](n, seed, pass_index).copy()
    if n > 1:
        p[-1] = p[0]
    return p


def batch_law_wrong_n_exponent(n, k, epochs, law="throughput"):
    """n^0.8 in equation (1) instead of the fitted exponent."""
    return O.LAW_CONST[law] * k ** 0.134749 * n ** 0.8 * epochs ** 0.813344


def alpha0_law_wrong_batch_sign(n, k, b, epochs):
    """The batch exponent of equation (3) with the wrong sign."""
    a = 0.8244 * k ** -0.4617 * b ** -0.9003 * n ** -0.4498 * epochs ** -0.1057
    return float(min(1.0, max(1e-4, a)))


def unit_rows_identity(c):
    """The rescaling to norm 1 is skipped."""
    return np.array(c, dtype=np.float64, copy=True)


def e4m3_ties_away_from_zero(v):
    """Halfway values round away from zero instead of to the even code."""
    v = np.asarray(v, dtype=np.float64)
    tab = O.e4m3_table()
    a = np.minimum(np.abs(v), O.E4M3_MAX)
    hi = np.clip(np.searchsorted(tab, a, side="left"), 0, len(tab) - 1)
    lo = np.maximum(hi - 1, 0)
    pick_hi = (tab[hi] - a) <= (a - tab[lo])
    return np.copysign(np.where(pick_hi, tab[hi], tab[lo]), v)


def fp8_shift_is_the_mean(xq):
    """The shift is each dimension's mean instead of its midrange."""
    shift, scale = _orig["fp8_calibrate"](xq)
    sample = np.asarray(xq[:O.FP8_CALIBRATION_ROWS], dtype=np.float32)
    return sample.mean(axis=0).astype(np.float32), scale


def assign_dot_lowest_similarity(xq, cq, chunk=4096):
    """The lowest dot product wins."""
    labels, best, second = _orig["assign_dot"](-xq, cq, chunk)
    return labels, -best, -second


def round_batch_floor(b_raw, n):
    """The batch rounds down to a power of two instead of to the nearest (in log2)."""
    import math
    b = 2 ** int(math.floor(math.log2(max(b_raw, 1.0))))
    cap = 2 ** int(math.floor(math.log2(max(n / 2.0, 1.0))))
    return int(max(1, min(b, cap)))


def revive_donor_uniform(N, S, c, t, seed, mode="split", tau=O.DEFAULT_TAU, batch_rows=None):
    """Donors drawn uniformly among the live clusters instead of in proportion to
    their counts (the same dead set: every live count replaced by 1)."""
    k = len(N)
    live = ~(N < tau * (N.sum() / k))
    return _orig["revive"](np.where(live, 1.0, 0.0), S, c, t, seed, mode=mode, tau=tau, batch_rows=batch_rows)


class ClosingMeanForgotten(O.EmeansOracle):
    """finalize keeps the running centroids: the closing mean of the last pass is
    never taken."""

    def finalize(self):
        self.closing = False
        return super().finalize()


def alpha_off_by_one(t, total_steps, alpha0):
    """Step t takes the step size of step t + 1."""
    return _orig["alpha_at"](t + 1, total_steps, alpha0)


def ema_centroid_before_update(N, S, c, n_j, s_j, alpha):
    """c = S / N taken from the statistics before the update."""
    N2, S2, _ = _orig["ema_update"](N, S, c, n_j, s_j, alpha)
    c = c.copy()
    live = N > 0
    c[live] = S[live] / N[live][:, None]
    return N2, S2, c


def bf16_round_half_up(x32):
    """bf16 rounding with halfway cases rounded up (in magnitude) instead of to even."""
    x32 = np.ascontiguousarray(x32, dtype=np.float32)
    u = x32.view(np.uint32).astype(np.uint64)
    r = ((u + np.uint64(0x8000)) >> np.uint64(16)) << np.uint64(16)
    return (r & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def e4m3_no_saturation(v):
    """Values beyond 448 are not clamped to the largest finite code."""
    v = np.asarray(v, dtype=np.float64)
    r = _orig["e4m3_round"](v)
    return np.where(np.abs(v) > O.E4M3_MAX, np.nan, r)


def fp8_scale_not_a_power_of_two(xq):
    """The scale maps the largest |x - shift| exactly onto 448."""
    shift, _ = _orig["fp8_calibrate"](xq)
    sample = np.asarray(xq[:O.FP8_CALIBRATION_ROWS], dtype=np.float32)
    half = np.maximum(sample.max(axis=0) - shift, shift - sample.min(axis=0)).astype(np.float64)
    m = float(half.max()) if half.size else 0.0
    return shift, (O.E4M3_MAX / m if m > 0 else 1.0)


def rows_per_pass_floor(n, epochs):
    """A fractional last pass is dropped (the epochs rounded down)."""
    import math
    return [n] * int(math.floor(epochs)) or [n]


def draw_uniform_ignores_step(seed, stream, t, j):
    """The step is left out of the counter: every revival check draws the same."""
    return _orig["draw_uniform"](seed, stream, 0, j)


def spherical_error_one_minus(xq, c64):
    """1 - similarity instead of 2 - 2 x similarity."""
    return float((1.0 - O.assign_dot(xq, O.search_copy_of_centroids(c64))[1]).mean())


def fp8_codes_scale_before_shift(v, shift, scale):
    """v x scale - shift: the shift is applied after the scaling."""
    d32 = (np.asarray(v, dtype=np.float64) * scale).astype(np.float32) - np.asarray(shift, dtype=np.float32)
    return O.e4m3_round(d32.astype(np.float64))


def lloyd_half_step(xq, c0, iters, spherical=False, fp8=None):
    """Lloyd's update with alpha = 0.5 instead of 1: each centroid only half-way to
    its rows' mean after the first iteration."""
    k = c0.shape[0]
    N, S, c = np.zeros(k), np.zeros_like(c0), c0.copy()
    history = []
    for _ in range(iters):
        labels, best, _ = O.assign(xq, O.search_copy_of_centroids(c))
        history.append(float(best.mean()))
        n_j, s_j = O.batch_stats(xq, labels, k)
        N, S, c = O.ema_update(N, S, c, n_j, s_j, 0.5)
    return c, history


def spherical_lloyd_not_rescaled(xq, c0, iters, spherical=False, fp8=None):
    """Spherical Lloyd whose centroids are left at the rows' mean, not rescaled to
    norm 1 after the update."""
    if not spherical:
        return _orig["lloyd"](xq, c0, iters, spherical, fp8)
    k = c0.shape[0]
    N, S, c = np.zeros(k), np.zeros_like(c0), O.unit_rows(c0)
    history = []
    for _ in range(iters):
        labels, sim, _ = O.assign_dot(xq, O.search_copy_of_centroids(c))
        history.append(float((2.0 - 2.0 * sim).mean()))
        n_j, s_j = O.batch_stats(xq, labels, k)
        N, S, c = O.ema_update(N, S, c, n_j, s_j, 1.0)
    return c, history


def assign_fp8_in_code_units(xq, c64, shift, scale):
    """FP8 distances reported in code units (not divided by scale^2)."""
    labels, best, second = _orig["assign_fp8"](xq, c64, shift, scale)
    return labels, best * scale ** 2, second * scale ** 2


def starting_rows_first_k(n, k, seed):
    """The first k training rows instead of a keyed random choice."""
    return np.arange(k, dtype=np.int64)


MUTATIONS = [
    ("ema_update", ema_without_decay, [P.test_constant_step_single_cluster_is_exponentially_weighted_mean]),
    ("ema_update", ema_weights_swapped, [P.test_full_batch_unit_step_is_one_lloyd_iteration,
                                         P.test_constant_step_single_cluster_is_exponentially_weighted_mean]),
    ("alpha_at", alpha_to_zero, [P.test_cosine_schedule_endpoints_and_shape]),
    ("alpha_at", alpha_linear, [P.test_cosine_schedule_endpoints_and_shape]),
    ("alpha_at", alpha_power, [P.test_cosine_schedule_endpoints_and_shape]),
    ("alpha_at", alpha_smoothstep, [P.test_cosine_schedule_endpoints_and_shape]),
    ("squared_distances", distances_without_centroid_norm, [P.test_assign_matches_brute_force_definition]),
    ("squared_distances", distances_with_plus_cross_term, [P.test_assign_matches_brute_force_definition]),
    ("assign", assign_ties_to_highest, [P.test_assign_ties_go_to_lowest_index]),
    ("batch_stats", stats_labels_shifted, [P.test_batch_stats_against_loops]),
    ("f32_to_bf16", bf16_truncates, [P.test_bf16_rounding_matches_torch_cast]),
    ("revive", revive_threshold_not_strict, [P.test_dead_set_uses_strict_threshold_on_mean_count]),
    ("split_sign", split_sign_flipped, [P.test_split_halves_count_and_keeps_sums_consistent]),
    ("philox4x64_10", philox_keys_swapped,
     [functools.partial(P.test_philox_matches_numpy_bit_generator, (5, 0, 0, 0), (1234, 2))]),
    ("pass_order", pass_order_not_a_bijection, [functools.partial(P.test_pass_order_is_a_bijection, 1000)]),
    ("batch_size_law", batch_law_wrong_n_exponent,
     [functools.partial(P.test_recipe_agrees_with_independently_quoted_rounded_law, 1_000_000, 4096, 5)]),
    ("alpha0_law", alpha0_law_wrong_batch_sign,
     [functools.partial(P.test_recipe_agrees_with_independently_quoted_rounded_law, 1_000_000, 4096, 5),
      P.test_recipe_invariants]),
    ("round_batch", round_batch_floor, [P.test_batch_rounding_is_nearest_power_in_log2_and_capped]),
    ("unit_rows", unit_rows_identity, [P.test_unit_rows_rescales_and_keeps_zero_rows]),
    ("e4m3_round", e4m3_ties_away_from_zero, [P.test_e4m3_rounding_matches_torch_and_breaks_ties_to_even]),
    ("fp8_calibrate", fp8_shift_is_the_mean, [P.test_fp8_calibration_is_midrange_shift_and_largest_power_of_two]),
    ("assign_dot", assign_dot_lowest_similarity, [P.test_assign_dot_matches_brute_force_with_lowest_index_ties]),
    ("revive", revive_donor_uniform, [P.test_donor_frequency_proportional_to_size]),
    ("EmeansOracle", ClosingMeanForgotten, [P.test_closing_mean_is_exact_mean_of_last_pass_assignments]),
    ("alpha_at", alpha_off_by_one, [P.test_cosine_schedule_endpoints_and_shape]),
    ("ema_update", ema_centroid_before_update, [P.test_full_batch_unit_step_is_one_lloyd_iteration,
                                                P.test_constant_step_single_cluster_is_exponentially_weighted_mean]),
    ("f32_to_bf16", bf16_round_half_up, [P.test_bf16_rounding_matches_torch_cast]),
    ("e4m3_round", e4m3_no_saturation, [P.test_e4m3_rounding_matches_torch_and_breaks_ties_to_even]),
    ("fp8_calibrate", fp8_scale_not_a_power_of_two,
     [P.test_fp8_calibration_is_midrange_shift_and_largest_power_of_two]),
    ("REVIVE_EVERY", 4, [P.test_revival_happens_every_fifth_step_only]),
    ("rows_per_pass", rows_per_pass_floor, [P.test_every_row_once_per_pass_and_fractional_last_pass,
                                            P.test_recipe_invariants]),
    ("draw_uniform", draw_uniform_ignores_step, [P.test_donor_frequency_proportional_to_size]),
    ("spherical_error", spherical_error_one_minus, [P.test_spherical_run_keeps_unit_centroids_and_error_definition]),
    ("fp8_codes", fp8_codes_scale_before_shift, [P.test_fp8_search_is_the_argmin_over_codes,
                                                 P.test_fp8_distances_within_the_quantisation_bound]),
    ("lloyd", lloyd_half_step, [P.test_lloyd_iterations_match_a_hand_written_lloyd]),
    ("lloyd", spherical_lloyd_not_rescaled, [P.test_spherical_lloyd_step_is_the_normalised_mean]),
    ("assign_fp8", assign_fp8_in_code_units, [P.test_fp8_distances_within_the_quantisation_bound]),
    ("starting_rows", starting_rows_first_k, [P.test_starting_rows_are_distinct_training_rows]),
]


@pytest.mark.parametrize("name,mutant,pins", MUTATIONS,
                         ids=[getattr(m[1], "__name__", f"{m[0]}={m[1]}") for m in MUTATIONS])
def test_planted_mistake_fails_a_pin(monkeypatch, name, mutant, pins):
    # the pins hold for the oracle as it stands
    for pin in pins:
        pin()
    monkeypatch.setattr(O, name, mutant)
    failed = []
    for pin in pins:
        try:
            pin()
        except Exception as e:  # an assertion, or an error the mistake causes
            failed.append(f"{getattr(pin, '__name__', getattr(pin, 'func', pin).__name__)}: {type(e).__name__}")
    assert failed, f"no pin caught the planted mistake in {name} ({mutant.__name__})"
