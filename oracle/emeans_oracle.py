"""Plain fp64 CPU oracle for e-means (mini-batch EMA k-means).

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import, call or
execute this file: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it. It shares
no code, tables or constants generator with the CUDA library; it is written
from the pages that describe the method:

* [README]  faiss ``contrib/e_means/README.md`` ("e-means: outperforming k-means
  in one-tenth the epochs"), sections named below.
* [Blog]    "k-means Reads Your Data 25 Times. Two Would Do." (jecision.com, the
  zh-TW and English versions of the same essay), sections named below.
* [News]    "e-means speeds up k-means by 45x in faiss" (ic.work analysis).

Everything is fp64 except where the method itself fixes a narrower format: the
nearest-centroid search runs on bf16 copies of the data and of the centroids
([README] "Data precision": only the search uses the smaller format), so the
oracle rounds both operands exactly as the method does and then computes
distances in fp64.

Readings taken where the pages are silent:

R1  batch size rounds to the nearest power of two in log2, capped at the
    largest power of two <= n/2 ([README] "Scaling laws");
R2  alpha0 is computed from the rounded batch size;
R3  cosine schedule alpha_t = a_min + (a0 - a_min)(1 + cos(pi t/(S-1)))/2 with
    a_min = a0/10 and t counted over all passes;
R4  the last, partial batch of a pass gets the scheduled alpha unchanged;
R5  N = S = 0 at the start; c_j keeps its value while N_j = 0;
R6  every cluster decays every step, hit or not;
R7  a revival check follows global step t when (t+1) % 5 == 0; dead clusters
    are those with N_j < tau * mean(N), fixed before any split;
R8  split: dead clusters in increasing index; each draws a donor outside the
    dead set with probability proportional to its current N (sequential, so a
    donor halved earlier in the same check is lighter); N_j = N_d/2,
    N_d <- N_d/2, c_j = c_d (1 - eps s), c_d <- c_d (1 + eps s), s_i = +1 for
    even i and -1 for odd i, eps = 2^-10, S = N c for both;
R9  resample: c_j <- a uniformly drawn row of the current batch, N_j = S_j = 0;
R10 Lloyd mode: B = n, alpha = 1, natural row order, no revival;
R11 reported distances and MSE use the bf16 search operands, clamped at 0;
R12 closing mean: clusters without points in the last pass keep their EMA
    centroid;
R13 FP8 search: the converter's shift is each dimension's midrange and its scale
    the largest power of two keeping the sample within 448, fitted on the first
    65,536 rows of the bf16 search copy; rows and centroids are encoded from their
    bf16 / fp32 values; the running sums stay those of the bf16 rows.
R14 data parallelism ([README] "Several GPUs", the DistributedEmeans loop): each
    of W ranks holds its own n_local rows; the recipe is that of n_local x W rows;
    at the step covering positions [pos, pos + rows) of a pass, a rank takes the
    positions [pos // W, (pos + rows) // W) of its own per-pass order of its own
    rows, the order keyed by pass + rank x 2^32 (rank 0: the one-rank order); the
    per-cluster counts and sums (and the batch error) are added over the ranks,
    and every rank applies the same update; rank 0's starting rows are used.

Random draws (starting rows, per-pass order, donor draws, resample rows) come
from the counter-based generator Philox4x64-10 (Salmon, Moraes, Dror, Shaw,
"Parallel random numbers: as easy as 1, 2, 3", SC'11), written here from that
paper's definition; the per-pass order is a keyed 4-round Feistel bijection
with cycle walking (Black & Rogaway, "Ciphers with arbitrary finite domains",
CT-RSA 2002).
"""

from __future__ import annotations

import math

import numpy as np

U64 = np.uint64
MASK32 = U64(0xFFFFFFFF)

# Philox4x64 constants (Salmon et al. 2011, Philox4x64: multipliers and the
# Weyl increments of the key schedule).
PHILOX_M0 = U64(0xD2E7470EE14C6C93)
PHILOX_M1 = U64(0xCA5A826395121157)
PHILOX_W0 = U64(0x9E3779B97F4A7C15)
PHILOX_W1 = U64(0xBB67AE8584CAA73B)

# Purposes of the random draws: the second key word of every Philox call.
STREAM_INIT = 1
STREAM_PASS = 2
STREAM_REVIVE = 3
STREAM_RESAMPLE = 4

SPLIT_EPS = 2.0 ** -10
REVIVE_EVERY = 5
DEFAULT_TAU = 0.1


# --------------------------------------------------------------------------
# Number formats ([README] "Data precision")
# --------------------------------------------------------------------------

def to_f32(x) -> np.ndarray:
    """Round to fp32, nearest-even (numpy's conversion)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def f32_to_bf16(x32) -> np.ndarray:
    """Round fp32 values to bf16, nearest-even; the result is held in fp32.

    bf16 keeps the upper 16 bits of the fp32 encoding; round-to-nearest-even
    adds 0x7FFF plus the lowest kept bit before truncating.
    """
    x32 = np.ascontiguousarray(x32, dtype=np.float32)
    u = x32.view(np.uint32).astype(np.uint64)
    lsb = (u >> U64(16)) & U64(1)
    r = ((u + U64(0x7FFF) + lsb) >> U64(16)) << U64(16)
    nan = np.isnan(x32)
    r = np.where(nan, (u | U64(0x00400000)) & U64(0xFFFF0000), r)
    return (r & MASK32).astype(np.uint32).view(np.float32)


def search_copy_of_data(x) -> np.ndarray:
    """fp32 data -> bf16 search copy, as fp64 values ([README] "Data precision")."""
    return f32_to_bf16(to_f32(x)).astype(np.float64)


def search_copy_of_centroids(c64) -> np.ndarray:
    """fp64 centroids -> fp32 (the stored format) -> bf16 (the search format)."""
    return f32_to_bf16(to_f32(c64)).astype(np.float64)


# --------------------------------------------------------------------------
# FP8 search ([README] "Data precision": an FP8 (E4M3) converter calibrated on a
# sample, with a shift per dimension and one power-of-two scale; values beyond
# the range clamp to the edge, 448 for FP8; only the search uses the format)
# --------------------------------------------------------------------------

E4M3_MAX = 448.0
FP8_CALIBRATION_ROWS = 65536


def e4m3_table() -> np.ndarray:
    """Values of the 127 non-negative finite E4M3 codes 0x00..0x7E, in code order.

    E4M3 (the OCP 8-bit float with 4 exponent bits, bias 7, 3 mantissa bits, no
    infinities): exponent field 0 holds the subnormals m/8 * 2^-6; fields 1..15
    hold (1 + m/8) * 2^(e - 7), except that field 15 with mantissa 7 is NaN, so
    the largest value is 1.75 * 2^8 = 448.
    """
    vals = []
    for code in range(127):
        e, m = code >> 3, code & 7
        vals.append(m / 8.0 * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(vals)


def e4m3_round(v) -> np.ndarray:
    """Each value rounded to E4M3, nearest with ties to the even code, saturating at
    +-448 (a finite value beyond it clamps); returned as fp64 values."""
    v = np.asarray(v, dtype=np.float64)
    tab = e4m3_table()
    a = np.minimum(np.abs(v), E4M3_MAX)
    hi = np.clip(np.searchsorted(tab, a, side="left"), 0, len(tab) - 1)  # first value >= a
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - tab[lo], tab[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    r = np.where(a == tab[hi], tab[hi], np.where(pick_hi, tab[hi], tab[lo]))
    return np.copysign(r, v)


def fp8_calibrate(xq: np.ndarray):
    """(shift, scale) of the FP8 converter, fitted on the first FP8_CALIBRATION_ROWS
    rows of the search copy: the shift is each dimension's midrange, computed in
    fp32 ((min + max) / 2), and the scale the largest power of two that keeps
    the largest |x - shift| of the sample within 448 (1 when the sample is constant)."""
    sample = np.asarray(xq[:FP8_CALIBRATION_ROWS], dtype=np.float32)
    lo, hi = sample.min(axis=0), sample.max(axis=0)
    shift = ((lo + hi) * np.float32(0.5)).astype(np.float32)
    half = np.maximum(hi - shift, shift - lo).astype(np.float64)
    m = float(half.max()) if half.size else 0.0
    if not m > 0.0:
        return shift, 1.0
    e = math.floor(math.log2(E4M3_MAX / m))
    while m * 2.0 ** e > E4M3_MAX:  # guard the floating-point log
        e -= 1
    while m * 2.0 ** (e + 1) <= E4M3_MAX:
        e += 1
    return shift, 2.0 ** e


def fp8_codes(v, shift, scale) -> np.ndarray:
    """E4M3 codes of (v - shift) * scale, as fp64 values: the subtraction in fp32
    (the stored format of the shift), the power-of-two scaling exact, then one
    rounding to E4M3."""
    d32 = np.asarray(v, dtype=np.float32) - np.asarray(shift, dtype=np.float32)
    return e4m3_round(d32.astype(np.float64) * scale)


def fp8_search_copy_of_centroids(c64, shift, scale) -> np.ndarray:
    """fp64 centroids -> fp32 (the stored format) -> FP8 codes."""
    return fp8_codes(to_f32(c64), shift, scale)


def mse_fp8(xq: np.ndarray, c64: np.ndarray, shift, scale) -> float:
    """Mean squared distance to the nearest centroid with the FP8 search (data units)."""
    return float(assign_fp8(xq, c64, shift, scale)[1].mean())


def assign_fp8(xq: np.ndarray, c64: np.ndarray, shift, scale):
    """Nearest centroid of each row with the FP8 search: the argmin of |x' - c'|^2
    over the codes (fp64, ties to the lowest index), reported as squared distances
    in the data's units, |x' - c'|^2 / scale^2. Returns (labels, best, second)."""
    xc = fp8_codes(xq, shift, scale)
    cc = fp8_search_copy_of_centroids(c64, shift, scale)
    labels, best, second = assign(xc, cc)
    return labels, best / scale ** 2, second / scale ** 2


# --------------------------------------------------------------------------
# Counter-based generator: Philox4x64-10
# --------------------------------------------------------------------------

def _mulhilo64(a: np.ndarray, m: np.uint64):
    """64x64 -> 128-bit product of uint64 array a and constant m, as (hi, lo)."""
    a = np.asarray(a, dtype=np.uint64)
    a_lo, a_hi = a & MASK32, a >> U64(32)
    m_lo, m_hi = m & MASK32, m >> U64(32)
    ll = a_lo * m_lo
    lh = a_lo * m_hi
    hl = a_hi * m_lo
    hh = a_hi * m_hi
    mid = (ll >> U64(32)) + (lh & MASK32) + (hl & MASK32)
    hi = hh + (lh >> U64(32)) + (hl >> U64(32)) + (mid >> U64(32))
    with np.errstate(over="ignore"):
        lo = a * m
    return hi, lo


def philox4x64_10(c0, c1, c2, c3, k0, k1):
    """Philox4x64 with 10 rounds on arrays of counters; returns 4 uint64 arrays.

    One round: (x0, x1, x2, x3) -> (hi(M1 x2) ^ x1 ^ k0, lo(M1 x2),
    hi(M0 x0) ^ x3 ^ k1, lo(M0 x0)); the key advances by the Weyl increments.
    """
    shape = np.broadcast(c0, c1, c2, c3, k0, k1).shape
    x = [np.broadcast_to(np.asarray(v, dtype=np.uint64), shape).copy() for v in (c0, c1, c2, c3)]
    k0 = np.broadcast_to(np.asarray(k0, dtype=np.uint64), shape).copy()
    k1 = np.broadcast_to(np.asarray(k1, dtype=np.uint64), shape).copy()
    with np.errstate(over="ignore"):
        for _ in range(10):
            hi0, lo0 = _mulhilo64(x[0], PHILOX_M0)
            hi1, lo1 = _mulhilo64(x[2], PHILOX_M1)
            x = [hi1 ^ x[1] ^ k0, lo1, hi0 ^ x[3] ^ k1, lo0]
            k0 = k0 + PHILOX_W0
            k1 = k1 + PHILOX_W1
    return x


def uniform01(bits64) -> np.ndarray:
    """Top 53 bits of a 64-bit draw as a double in [0, 1)."""
    return (np.asarray(bits64, dtype=np.uint64) >> U64(11)).astype(np.float64) * (2.0 ** -53)


def draw_uniform(seed: int, stream: int, t: int, j) -> np.ndarray:
    """u(seed, stream, t, j) in [0, 1): counter (t, j, 0, 0), key (seed, stream)."""
    out = philox4x64_10(U64(t), np.asarray(j, dtype=np.uint64), U64(0), U64(0), U64(seed), U64(stream))
    return uniform01(out[0])


# --------------------------------------------------------------------------
# Per-pass random order: a bijection on [0, n) ([README] "Data too big for
# memory": a fresh random order every pass, every vector exactly once)
# --------------------------------------------------------------------------

def feistel_half_bits(n: int) -> int:
    bits = max(1, math.ceil(math.log2(n))) if n > 1 else 1
    return max(1, (bits + 1) // 2)


def _feistel_encrypt(v: np.ndarray, h: int, seed: int, stream: int, which: int) -> np.ndarray:
    mask = U64((1 << h) - 1)
    left, right = v >> U64(h), v & mask
    for r in range(4):
        f = philox4x64_10(right, U64(r), U64(which), U64(0), U64(seed), U64(stream))[0] & mask
        left, right = right, left ^ f
    return (left << U64(h)) | right


def permute(idx, n: int, seed: int, stream: int, which: int) -> np.ndarray:
    """pi(idx) for the keyed bijection on [0, n) selected by (seed, stream, which).

    A 4-round balanced Feistel network over 2h bits (2^(2h) >= n) whose round
    function is the low h bits of Philox4x64-10 at counter (R, round, which, 0)
    and key (seed, stream); values that land outside [0, n) are re-encrypted
    until they fall inside (cycle walking), which keeps the map a bijection.
    """
    h = feistel_half_bits(n)
    v = _feistel_encrypt(np.asarray(idx, dtype=np.uint64), h, seed, stream, which)
    out = v.copy()
    bad = out >= U64(n)
    while np.any(bad):
        out[bad] = _feistel_encrypt(out[bad], h, seed, stream, which)
        bad = out >= U64(n)
    return out.astype(np.int64)


def pass_order(n: int, seed: int, pass_index: int) -> np.ndarray:
    return permute(np.arange(n, dtype=np.uint64), n, seed, STREAM_PASS, pass_index)


def dp_share(pos: int, rows: int, world: int):
    """The positions [lo, hi) of a rank's own per-pass order that it takes when the
    whole job's batch covers positions [pos, pos + rows) of the pass ([README]
    "Several GPUs": with the batch summed over all GPUs, every rank takes an even
    share; the pages' loop slices [start // world, (start + B) // world))."""
    return pos // world, (pos + rows) // world


def starting_rows(n: int, k: int, seed: int) -> np.ndarray:
    """k distinct training rows: the first k images of the start permutation."""
    return permute(np.arange(k, dtype=np.uint64), n, seed, STREAM_INIT, 0)


# --------------------------------------------------------------------------
# Recipe ([README] "Scaling laws", "Manual overrides", "Core configuration")
# --------------------------------------------------------------------------

LAW_CONST = {"throughput": 0.035134, "quality": 0.00439175}


def batch_size_law(n: int, k: int, epochs: float, law: str = "throughput") -> float:
    """Equation (1) ("throughput") or (2) ("quality") before rounding."""
    return LAW_CONST[law] * k ** 0.134749 * n ** 0.876473 * epochs ** 0.813344


def round_batch(b_raw: float, n: int) -> int:
    """Nearest power of two (in log2), capped at the largest power of two <= n/2."""
    b = 2 ** int(round(math.log2(max(b_raw, 1.0))))
    cap = 2 ** int(math.floor(math.log2(max(n / 2.0, 1.0))))
    return int(max(1, min(b, cap)))


def alpha0_law(n: int, k: int, b: int, epochs: float) -> float:
    """Equation (3), clamped to [1e-4, 1]."""
    a = 0.8244 * k ** -0.4617 * b ** 0.9003 * n ** -0.4498 * epochs ** -0.1057
    return float(min(1.0, max(1e-4, a)))


def rows_per_pass(n: int, epochs: float) -> list[int]:
    """Rows of each pass: n for every whole pass, round(frac * n) for a fractional last one."""
    whole = int(math.floor(epochs))
    rows = [n] * whole
    frac = epochs - whole
    if frac > 0:
        rows.append(max(1, int(math.floor(frac * n + 0.5))))
    return rows


def recipe(n: int, k: int, epochs: float, law: str = "throughput", batch_size=None, alpha0=None) -> dict:
    if batch_size is None:
        b_raw = batch_size_law(n, k, epochs, law)
        b = round_batch(b_raw, n)
    else:
        b_raw, b = float(batch_size), int(batch_size)
    a0 = alpha0_law(n, k, b, epochs) if alpha0 is None else float(alpha0)
    epoch_rows = rows_per_pass(n, epochs)
    steps = [-(-r // b) for r in epoch_rows]
    return dict(batch_raw=b_raw, batch_size=b, alpha0=a0, epoch_rows=epoch_rows,
                steps_per_pass=steps, total_steps=int(sum(steps)))


def alpha_at(t: int, total_steps: int, alpha0: float) -> float:
    """Cosine step size from alpha0 down to alpha0/10 ([README] "How the centroid
    updates work"; [Blog] "Two: alpha is not constant")."""
    a_min = 0.1 * alpha0
    frac = 0.0 if total_steps <= 1 else t / (total_steps - 1)
    return a_min + (alpha0 - a_min) * 0.5 * (1.0 + math.cos(math.pi * frac))


# --------------------------------------------------------------------------
# Assignment ([Blog] "Still Lloyd's 1957 algorithm": a(i) = argmin_j |x_i - c_j|^2)
# --------------------------------------------------------------------------

def squared_distances(xq: np.ndarray, cq: np.ndarray) -> np.ndarray:
    """|x - c|^2 for every (row, centroid) pair, fp64, via |x|^2 + |c|^2 - 2 x.c."""
    xn = np.einsum("ij,ij->i", xq, xq)
    cn = np.einsum("ij,ij->i", cq, cq)
    return xn[:, None] + cn[None, :] - 2.0 * (xq @ cq.T)


def assign(xq: np.ndarray, cq: np.ndarray, chunk: int = 4096):
    """Nearest search copy of each row. Returns (labels, best, second) where best
    and second are the two smallest squared distances (clamped at 0); ties go to
    the lowest centroid index."""
    n = xq.shape[0]
    labels = np.empty(n, dtype=np.int64)
    best = np.empty(n)
    second = np.full(n, np.inf)
    for s in range(0, n, chunk):
        dist = squared_distances(xq[s:s + chunk], cq)
        lab = np.argmin(dist, axis=1)
        labels[s:s + chunk] = lab
        rows = np.arange(dist.shape[0])
        best[s:s + chunk] = dist[rows, lab]
        if cq.shape[0] > 1:
            dist[rows, lab] = np.inf
            second[s:s + chunk] = dist.min(axis=1)
    return labels, np.maximum(best, 0.0), np.maximum(second, 0.0)


def mse(xq: np.ndarray, c64: np.ndarray) -> float:
    """Mean over rows of the squared distance to the nearest centroid, searched
    and measured with the bf16 search copies ([Blog] the MSE objective)."""
    _, best, _ = assign(xq, search_copy_of_centroids(c64))
    return float(best.mean())


# --------------------------------------------------------------------------
# Spherical e-means ([README] "Spherical e-means"): centroids rescaled to norm 1
# before every use, the highest dot product wins, error 2 - 2 x similarity
# --------------------------------------------------------------------------

def unit_rows(c: np.ndarray) -> np.ndarray:
    """Each row rescaled to norm 1; a zero row stays zero."""
    nrm = np.sqrt(np.einsum("ij,ij->i", c, c))
    out = np.array(c, dtype=np.float64, copy=True)
    nz = nrm > 0
    out[nz] = out[nz] / nrm[nz][:, None]
    return out


def assign_dot(xq: np.ndarray, cq: np.ndarray, chunk: int = 4096):
    """Centroid with the highest dot product with each row (search copies). Returns
    (labels, best, second): the two highest dot products; ties go to the lowest
    centroid index."""
    n = xq.shape[0]
    labels = np.empty(n, dtype=np.int64)
    best = np.empty(n)
    second = np.full(n, -np.inf)
    for s in range(0, n, chunk):
        neg = -(xq[s:s + chunk] @ cq.T)
        lab = np.argmin(neg, axis=1)
        labels[s:s + chunk] = lab
        rows = np.arange(neg.shape[0])
        best[s:s + chunk] = -neg[rows, lab]
        if cq.shape[0] > 1:
            neg[rows, lab] = np.inf
            second[s:s + chunk] = -neg.min(axis=1)
    return labels, best, second


def spherical_error(xq: np.ndarray, c64: np.ndarray) -> float:
    """Mean of 2 - 2 x (highest similarity) over the rows, with the bf16 search
    copies of the centroids ([README] "Spherical e-means": the reported error)."""
    _, best, _ = assign_dot(xq, search_copy_of_centroids(c64))
    return float((2.0 - 2.0 * best).mean())


# --------------------------------------------------------------------------
# Per-batch statistics and the EMA update ([README] "How the centroid updates work")
# --------------------------------------------------------------------------

def batch_stats(rows: np.ndarray, labels: np.ndarray, k: int):
    """n_j = number of batch rows assigned to j, s_j = their sum (fp64)."""
    n_j = np.bincount(labels, minlength=k).astype(np.float64)
    s_j = np.zeros((k, rows.shape[1]))
    order = np.argsort(labels, kind="stable")
    lab_sorted = labels[order]
    starts = np.flatnonzero(np.r_[True, lab_sorted[1:] != lab_sorted[:-1]])
    if len(order):
        s_j[lab_sorted[starts]] = np.add.reduceat(rows[order], starts, axis=0)
    return n_j, s_j


def ema_update(N, S, c, n_j, s_j, alpha):
    """N <- (1-a) N + a n; S <- (1-a) S + a s; c = S / N where N > 0, else unchanged."""
    N = (1.0 - alpha) * N + alpha * n_j
    S = (1.0 - alpha) * S + alpha * s_j
    c = c.copy()
    live = N > 0
    c[live] = S[live] / N[live][:, None]
    return N, S, c


# --------------------------------------------------------------------------
# Dead-cluster revival ([README] `unused_threshold`; [Blog] "Three: dead
# clusters must be revived"; [News] revival by size-proportional split)
# --------------------------------------------------------------------------

def split_sign(d: int) -> np.ndarray:
    return np.where(np.arange(d) % 2 == 0, 1.0, -1.0)


def revive(N, S, c, t, seed, mode="split", tau=DEFAULT_TAU, batch_rows=None):
    """One revival check after global step t. Returns (N, S, c, dead_indices, donors)."""
    N, S, c = N.copy(), S.copy(), c.copy()
    k = N.shape[0]
    if mode == "none" or tau <= 0:
        return N, S, c, np.empty(0, np.int64), np.empty(0, np.int64)
    mean = N.sum() / k
    dead = np.flatnonzero(N < tau * mean)
    donors = np.full(len(dead), -1, dtype=np.int64)
    if len(dead) == 0:
        return N, S, c, dead, donors
    if mode == "resample":
        if batch_rows is None or len(batch_rows) == 0:
            return N, S, c, dead, donors
        u = draw_uniform(seed, STREAM_RESAMPLE, t, dead)
        pick = np.minimum(np.floor(u * len(batch_rows)).astype(np.int64), len(batch_rows) - 1)
        c[dead] = batch_rows[pick]
        N[dead] = 0.0
        S[dead] = 0.0
        return N, S, c, dead, pick
    assert mode == "split", mode
    eligible = np.ones(k, dtype=bool)
    eligible[dead] = False
    sgn = split_sign(c.shape[1])
    u_all = draw_uniform(seed, STREAM_REVIVE, t, dead)
    for i, j in enumerate(dead):
        w = np.where(eligible, N, 0.0)
        cdf = np.cumsum(w)
        total = cdf[-1]
        if not total > 0:
            break
        donor = int(np.searchsorted(cdf, u_all[i] * total, side="right"))
        donor = min(donor, k - 1)
        while not eligible[donor] or w[donor] <= 0:  # guard against a zero-width bin at the edge
            donor -= 1
        donors[i] = donor
        half = N[donor] / 2.0
        N[j] = half
        N[donor] = half
        cd = c[donor].copy()
        c[j] = cd * (1.0 - SPLIT_EPS * sgn)
        c[donor] = cd * (1.0 + SPLIT_EPS * sgn)
        S[j] = N[j] * c[j]
        S[donor] = N[donor] * c[donor]
    return N, S, c, dead, donors


# --------------------------------------------------------------------------
# The training loop ([README] "Data too big for memory": begin, accumulate,
# update, end_epoch, finalize; "train runs exactly this loop internally")
# --------------------------------------------------------------------------

class EmeansOracle:
    """e-means in fp64 on the bf16 search copy of the data."""

    def __init__(self, d, k, seed=1234, revival="split", tau=None, closing_mean=True,
                 law="auto", batch_size=None, alpha0=None, spherical=False, search="bf16",
                 world=1, rank=0, all_reduce=None):
        self.d, self.k, self.seed = int(d), int(k), int(seed)
        # data parallelism (R14): `all_reduce` adds a float64 vector over the ranks
        self.world, self.rank, self.all_reduce = int(world), int(rank), all_reduce
        if not 0 <= self.rank < self.world:
            raise ValueError("rank outside [0, world)")
        self.spherical = bool(spherical)
        if search not in ("bf16", "fp8"):
            raise ValueError(search)
        if search == "fp8" and self.spherical:  # [README] "Spherical e-means": 32- and 16-bit floats only
            raise ValueError("spherical e-means does not take the FP8 search")
        self.search = search
        self.fp8 = None  # (shift, scale) of the FP8 converter, fitted at begin
        # defaults that depend on the dimension ([README] `batch_law`, `unused_threshold`
        # and "Note on low dimension"): the quality batch law for d <= 16, no revival
        # (threshold 0) for d <= 2
        if tau is None:
            tau = 0.0 if self.d <= 2 else DEFAULT_TAU
        if law == "auto":
            law = "quality" if self.d <= 16 else "throughput"
        self.revival, self.tau, self.closing = revival, float(tau), bool(closing_mean)
        self.law, self.batch_override, self.alpha_override = law, batch_size, alpha0
        self.n_splits = 0

    # begin: recipe, starting centroids, zero statistics
    def begin(self, xq: np.ndarray, epochs: float, start_rows=None, start_centroids=None):
        """Recipe, starting centroids, zero statistics. With several ranks (R14), xq is
        this rank's rows and start_centroids rank 0's starting rows (ranks other
        than 0 must pass them)."""
        n = xq.shape[0]
        if n < self.k:
            raise ValueError("need at least k rows")
        self.xq = xq
        self.n = n
        W = self.world
        self.r = recipe(n * W, self.k, epochs, self.law, self.batch_override, self.alpha_override)
        if W > 1:
            if self.r["batch_size"] % W or self.r["epoch_rows"][-1] % W:
                raise ValueError("the batch and the rows of every pass must divide by the number of ranks")
            if self.revival == "resample" or self.search == "fp8":
                raise ValueError("several ranks: resampling and the FP8 search are not modelled")
        if self.search == "fp8":
            self.fp8 = fp8_calibrate(xq)
        if start_centroids is not None:
            self.c = np.array(start_centroids, dtype=np.float64)
        else:
            if self.rank != 0:
                raise ValueError("ranks other than 0 start from rank 0's rows")
            rows = starting_rows(n, self.k, self.seed) if start_rows is None else np.asarray(start_rows)
            self.c = xq[rows].copy()
        if self.spherical:
            self.c = unit_rows(self.c)
        self.N = np.zeros(self.k)
        self.S = np.zeros((self.k, self.d))
        self.t = 0
        self.pass_index, self.pos = 0, 0
        self.order = pass_order(n, self.seed, self.order_key(0))
        self.labels_last = np.full(n, -1, dtype=np.int64)
        self.close_sum = np.zeros((self.k, self.d))
        self.close_cnt = np.zeros(self.k)
        self.obj = []
        self._pass_err = 0.0
        return self.r

    @property
    def done(self):
        return self.pass_index >= len(self.r["epoch_rows"])

    def order_key(self, pass_index):
        """Key of this rank's order in a pass (R14): the pass plus rank x 2^32."""
        return pass_index + (self.rank << 32)

    def batch_rows(self):
        """Rows of the whole job's current batch: positions [pos, pos + rows) of the pass."""
        return min(self.r["batch_size"], self.r["epoch_rows"][self.pass_index] - self.pos)

    def batch_positions(self):
        """This rank's positions of its own order in the current batch (R14; one rank:
        the batch's own positions)."""
        return dp_share(self.pos, self.batch_rows(), self.world)

    def next_batch_ids(self):
        lo, hi = self.batch_positions()
        return self.order[lo:hi]

    def step(self, forced_labels=None, auto_revive=True, stats=None):
        """One mini-batch: assign, per-cluster statistics, EMA, then revival if due.

        `stats`, if given, replaces the per-cluster statistics of the batch:
        stats(rows, labels, k) -> (n_j, s_j). The data-parallel protocol uses it to
        add the statistics of every rank's share of the batch."""
        ids = self.next_batch_ids()
        xb = self.xq[ids]
        if self.spherical:  # highest similarity; the error of a row is 2 - 2 x similarity
            labels, sim, sim2 = assign_dot(xb, search_copy_of_centroids(self.c))
            best, second = 2.0 - 2.0 * sim, 2.0 - 2.0 * sim2
        elif self.search == "fp8":
            labels, best, second = assign_fp8(xb, self.c, *self.fp8)
        else:
            labels, best, second = assign(xb, search_copy_of_centroids(self.c))
        used = labels if forced_labels is None else np.asarray(forced_labels, dtype=np.int64)
        n_j, s_j = (batch_stats if stats is None else stats)(xb, used, self.k)
        err = float(best.sum())
        if self.world > 1:  # R14: the counts, sums and batch error added over the ranks
            buf = self.all_reduce(np.concatenate([n_j, s_j.ravel(), [err]]))
            n_j, s_j, err = buf[:self.k], buf[self.k:-1].reshape(self.k, self.d), float(buf[-1])
        alpha = alpha_at(self.t, self.r["total_steps"], self.r["alpha0"])
        self.N, self.S, self.c = ema_update(self.N, self.S, self.c, n_j, s_j, alpha)
        if self.spherical:
            self.c = unit_rows(self.c)
        last_pass = self.pass_index == len(self.r["epoch_rows"]) - 1
        if last_pass:
            self.labels_last[ids] = used
            self.close_sum += s_j
            self.close_cnt += n_j
        self._pass_err += err
        info = dict(t=self.t, ids=ids, labels=labels, best=best, second=second, alpha=alpha,
                    n_j=n_j, s_j=s_j, revived=None)
        if auto_revive:
            info["revived"] = self.maybe_revive(xb)
        self.t += 1
        self.pos += self.batch_rows()
        if self.pos >= self.r["epoch_rows"][self.pass_index]:
            self.obj.append(self._pass_err / self.r["epoch_rows"][self.pass_index])
            self._pass_err = 0.0
            self.pass_index += 1
            self.pos = 0
            if not self.done:
                self.order = pass_order(self.n, self.seed, self.order_key(self.pass_index))
        return info

    def maybe_revive(self, batch_rows, t=None):
        t = self.t if t is None else t
        if (t + 1) % REVIVE_EVERY != 0 or self.revival == "none":
            return None
        self.N, self.S, self.c, dead, donors = revive(
            self.N, self.S, self.c, t, self.seed, self.revival, self.tau, batch_rows)
        if self.spherical:
            self.c = unit_rows(self.c)
        self.n_splits += int(np.count_nonzero(donors >= 0))
        return dead, donors

    def finalize(self):
        """Closing mean: each centroid becomes the exact mean of the rows the last
        pass assigned to it ([README] "How the centroid updates work")."""
        if self.closing:
            hit = self.close_cnt > 0
            self.c[hit] = self.close_sum[hit] / self.close_cnt[hit][:, None]
        if self.spherical:
            self.c = unit_rows(self.c)
        return self.c

    def train(self, xq: np.ndarray, epochs: float):
        self.begin(xq, epochs)
        while not self.done:
            self.step()
        return self.finalize(), self.labels_last


def lloyd(xq: np.ndarray, c0: np.ndarray, iters: int, spherical: bool = False, fp8=None):
    """Lloyd's k-means as the B = n, alpha = 1 case of the same update ([README]
    "How the centroid updates work"; [Blog] "Lloyd is a special case"); spherical:
    highest similarity, centroids rescaled to norm 1 ([README] "Spherical e-means")."""
    k = c0.shape[0]
    N, S, c = np.zeros(k), np.zeros_like(c0), (unit_rows(c0) if spherical else c0.copy())
    history = []
    for _ in range(iters):
        if spherical:
            labels, sim, _ = assign_dot(xq, search_copy_of_centroids(c))
            history.append(float((2.0 - 2.0 * sim).mean()))
        elif fp8 is not None:  # the FP8 search with the converter (shift, scale)
            labels, best, _ = assign_fp8(xq, c, *fp8)
            history.append(float(best.mean()))
        else:
            labels, best, _ = assign(xq, search_copy_of_centroids(c))
            history.append(float(best.mean()))
        n_j, s_j = batch_stats(xq, labels, k)
        N, S, c = ema_update(N, S, c, n_j, s_j, 1.0)
        if spherical:
            c = unit_rows(c)
    return c, history
