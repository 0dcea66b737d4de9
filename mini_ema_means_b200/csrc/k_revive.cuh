// k_revive.cuh -- dead-cluster revival, run after every 5th step.
//
// faiss e-means README (`unused_threshold`, "How the centroid updates work") and
// the jecision.com essay ("Three: dead clusters must be revived"): a cluster
// whose running count N_j falls below tau times the mean count is revived by
// splitting a busy cluster in two, the busy cluster being drawn with probability
// proportional to its size. Readings fixed here:
//   * the dead set D is fixed before any split; dead clusters are served in
//     increasing index; each draws its donor among the clusters outside D with
//     probability proportional to their CURRENT N (a donor halved earlier in the
//     same check is lighter), with u = Philox(seed, stream 3, t, j);
//   * split: N_j = N_d / 2, N_d <- N_d / 2, c_j = c_d (1 - eps s),
//     c_d <- c_d (1 + eps s) with s_i = +1 (even i), -1 (odd i), eps = 2^-10,
//     and S = N c for both;
//   * resample (the EnCodec-style arm of the ablation): c_j <- a row of the
//     current batch drawn with Philox(seed, stream 4, t, j), N_j = S_j = 0.
//
// The draws are inherently sequential, so one warp makes them on an fp64 tree of
// prefix sums, the uniform draws having been made in parallel beforehand. Up to
// 16,384 clusters the tree has 32 children per node, one per lane, and lives in
// shared memory with its top level in registers: a draw costs one load, one
// compare, one ballot and one shuffle per level. Larger k use 128 children per
// node (four per lane), with the lower levels in global memory when shared memory
// runs out. The donor's
// current weight is read back as the difference of two prefix values, and the
// number of earlier splits from the same donor is counted per batch of 32 draws
// with one warp match. The vector work is then done in parallel from the closed
// form: the o-th split taken from donor d (0-based) sees c_d (1 + eps s)^o and
// N_d / 2^o.
#pragma once

#include "k_reduce.cuh"

namespace em {

struct ReviveScratch {
    int32_t* dead;    // k: dead clusters in increasing order
    int32_t* donor;   // k: donor of each dead cluster (-1 if none)
    int32_t* order;   // k: how many earlier splits took this donor in this check
    int32_t* times;   // k: splits taken from each donor in this check
    double* target;   // k: u of each dead cluster (precomputed in parallel)
    double* tree;     // leaf weights and prefix levels that do not fit in shared memory
    int32_t* ndead;   // 1: |D| of the most recent check
    int64_t* n_splits;  // 1: cumulative number of revived clusters
};

// Donor tree, 128 children per node (four per lane of a warp). Level 0 holds, for
// every group of 128 consecutive clusters, the inclusive prefix sums of their
// current weights within the group (N_j, or 0 for a dead cluster); level l + 1
// holds the same over the group totals of level l; the top level (at most 128
// entries, one group) is kept in the drawing warp's registers. Padding positions
// of a group repeat its total. Every sum is exact in fp64 (the weights are fp32
// counts and their halvings), so `offset + within-group prefix` is exactly the
// cumulative weight up to that cluster and each comparison below is the one a
// search over the cumulative sums of all k weights would make.
constexpr int kRadix = 128;
constexpr int kTreeLevels = 5;  // 128^5 > 2^30 clusters

// Shared memory the selection kernel may use (bytes).
constexpr int kReviveSmemBytes = 200 * 1024;

struct TreeLayout {
    int levels;                   // including the top
    int size[kTreeLevels];        // entries per level
    int64_t offset[kTreeLevels];  // doubles; every level padded to a multiple of kRadix
    int64_t total;                // doubles over all levels
    int smem_from;                // levels in [smem_from, levels - 1) live in shared memory
    int64_t smem_base;            // offset[smem_from]: where the shared levels start
    int64_t smem_end;             // offset[levels - 1]: where they end
    int times_smem;               // split counters in shared memory too
    int64_t smem_bytes;           // top staging area + shared levels (+ counters)
};

EM_HD TreeLayout tree_layout(int k) {
    TreeLayout L{};
    int s = k;
    int64_t off = 0;
    bool done = false;
#pragma unroll
    for (int l = 0; l < kTreeLevels; ++l) {
        if (!done) {
            L.size[l] = s;
            L.offset[l] = off;
            off += ((int64_t)(s + kRadix - 1) / kRadix) * kRadix;
            L.levels = l + 1;
            L.smem_end = L.offset[l];  // the top level's offset, once the loop stops
            done = s <= kRadix;
            s = (s + kRadix - 1) / kRadix;
        }
    }
    L.total = off;
    // shared memory: the top level's staging group, then the levels below the top
    // from the top down while they fit, then the per-donor counters if they fit
    int64_t bytes = kRadix * 8;
    L.smem_from = L.levels - 1;
    L.smem_base = L.smem_end;
    bool stop = false;
#pragma unroll
    for (int l = kTreeLevels - 2; l >= 0; --l) {
        if (l <= L.levels - 2 && !stop) {
            const int64_t lb = ((int64_t)(L.size[l] + kRadix - 1) / kRadix) * kRadix * 8;
            if (bytes + lb <= kReviveSmemBytes) {
                bytes += lb;
                L.smem_from = l;
                L.smem_base = L.offset[l];
            } else {
                stop = true;
            }
        }
    }
    L.times_smem = (L.smem_from == 0 && bytes + (int64_t)k * 4 <= kReviveSmemBytes) ? 1 : 0;
    if (L.times_smem) bytes += (int64_t)k * 4;
    L.smem_bytes = bytes;
    return L;
}

EM_HD int64_t tree_smem_bytes(const TreeLayout& L, int) { return L.smem_bytes; }

__device__ __forceinline__ double warp_incl_scan(double v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double t = __shfl_up_sync(0xFFFFFFFFu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

// Inclusive prefix over one group of 128 values, four consecutive values per lane.
__device__ __forceinline__ void group_scan(double v[4], int lane) {
    v[1] += v[0];
    v[2] += v[1];
    v[3] += v[2];
    const double inc = warp_incl_scan(v[3], lane);
    double ex = __shfl_up_sync(0xFFFFFFFFu, inc, 1);
    if (lane == 0) ex = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] += ex;
}

// Unbiased binary exponent of a positive finite double (subnormals included),
// from the IEEE 754 encoding.
__device__ __forceinline__ int exponent_of(double x) {
    const unsigned long long b = (unsigned long long)__double_as_longlong(x);
    const int e = (int)((b >> 52) & 0x7FF);
    if (e) return e - 1023;
    const unsigned long long mant = b & 0xFFFFFFFFFFFFFull;
    return -1023 - (__clzll(mant) - 12);
}

// One step of the descent inside a group whose four prefix values this lane holds.
// Returns the child position (0..127) and, in *before / *w, the within-group
// prefix before it and its weight (*w only when want_w). `last`: the target fell
// on the total, take the last child with positive weight (the first position that
// reaches the group total). Written without branches: the fallback mask is formed
// alongside the normal one and the ballot picks, and lane L (the lane holding the
// chosen child) selects its values from differences computed before the ballot.
template <bool want_w>
__device__ __forceinline__ int group_select(const double P[4], double base, double t, bool last, int lane,
                                            double* before, double* w) {
    const double prev3 = __shfl_up_sync(0xFFFFFFFFu, P[3], 1);
    const double tot = __shfl_sync(0xFFFFFFFFu, P[3], 31);
    const double Pprev = lane ? prev3 : 0.0;
    unsigned mt = 0, mf = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        mt |= (base + P[i] > t) ? (1u << i) : 0u;
        mf |= (P[i] >= tot) ? (1u << i) : 0u;
    }
    const unsigned bt = __ballot_sync(0xFFFFFFFFu, mt != 0);
    const unsigned bf = __ballot_sync(0xFFFFFFFFu, mf != 0);
    // never empty in exact arithmetic unless the target is on the total
    const bool use_t = !last && bt != 0;
    const unsigned bal = use_t ? bt : bf;
    const unsigned m4 = use_t ? mt : mf;
    const int L = __ffs(bal) - 1;
    const int sub = m4 ? __ffs(m4) - 1 : 0;
    // prefix before each of the lane's positions, then the one at `sub`
    const double b = sub == 0 ? Pprev : (sub == 1 ? P[0] : (sub == 2 ? P[1] : P[2]));
    const int s = __shfl_sync(0xFFFFFFFFu, sub, L);
    *before = __shfl_sync(0xFFFFFFFFu, b, L);
    if (want_w) {
        const double wl = (sub == 0 ? P[0] : (sub == 1 ? P[1] : (sub == 2 ? P[2] : P[3]))) - b;
        *w = __shfl_sync(0xFFFFFFFFu, wl, L);
    }
    return 4 * L + s;
}

// Subtracts delta from the group positions at or after pos (this lane's four).
__device__ __forceinline__ bool group_sub(double P[4], int pos, double delta, int lane) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (4 * lane + i >= pos) P[i] -= delta;
    return 4 * lane + 3 >= pos;
}

// ---- radix-32 tree for k <= kFastK: one value per lane at every level
//
// Level 0 holds, for each group of 32 consecutive clusters, the inclusive prefix
// sums of their current weights within the group; level 1 the same over the group
// totals of level 0; level 2 over those of level 1. The top level (at most 32
// entries) sits in the drawing warp's registers, one entry per lane, and the levels
// below it in shared memory. A draw then costs, per level, one load, one compare,
// one ballot and one shuffle, about a third of the instructions of the radix-128
// descent; a single warp issuing alone is bound by that count.
constexpr int kFastK = 16384;

struct Tree32 {
    int levels;   // 1 (k <= 32), 2 (k <= 1024) or 3
    int n1;       // entries of level 1 = groups of level 0
    int n2;       // entries of level 2 = groups of level 1
    int off1;     // doubles: level 1 (levels == 3), after the top staging group
    int off0;     // doubles: level 0 (levels >= 2)
    int times;    // doubles: per-donor split counters (ints), -1 when they do not fit
    int bytes;    // shared memory
};

EM_HD Tree32 tree32(int k) {
    Tree32 T{};
    T.n1 = (k + 31) / 32;
    T.n2 = (T.n1 + 31) / 32;
    T.levels = k <= 32 ? 1 : (k <= 1024 ? 2 : 3);
    int off = 32;  // top staging group
    T.off1 = off;
    if (T.levels == 3) off += T.n2 * 32;  // level 1, padded to whole groups
    T.off0 = off;
    if (T.levels >= 2) off += T.n1 * 32;  // level 0, padded to whole groups
    const int base = off * 8;
    const int tb = ((k * 4 + 15) / 16) * 16;
    T.times = base + tb <= kReviveSmemBytes ? off : -1;
    T.bytes = base + (T.times >= 0 ? tb : 0);
    return T;
}

// Inclusive prefix of one value per lane.
__device__ __forceinline__ double lane_scan(double v, int lane) { return warp_incl_scan(v, lane); }

// First lane whose value passes (ballot, then the lowest set lane); -1 if none.
__device__ __forceinline__ int first_lane(bool pred) {
    const unsigned b = __ballot_sync(0xFFFFFFFFu, pred);
    return b ? __ffs(b) - 1 : -1;
}

// Sequential donor draws of dead clusters [0, nd) on the radix-32 tree, by one warp.
// T / Tprev: this lane's inclusive / exclusive prefix of the top level; W: the total.
// Writes donor, order (earlier splits of the same donor in this check) and the
// per-donor counters; returns the number of splits.
template <int LEVELS>
__device__ __forceinline__ int64_t draw_radix32(double* smem_d, const Tree32& TL, int nd, const ReviveScratch& sc,
                                                int32_t* times, int lane) {
    double T = smem_d[lane];
    double Tprev = lane ? smem_d[lane - 1] : 0.0;
    double W = __shfl_sync(0xFFFFFFFFu, T, 31);
    double* L1 = smem_d + TL.off1;
    double* L0 = smem_d + TL.off0;
    int64_t splits = 0;
    int i_end = nd;
    for (int i0 = 0; i0 < nd; i0 += 32) {
        const int cnt = min(32, nd - i0);
        const double my_u = lane < cnt ? sc.target[i0 + lane] : 0.0;
        int my_dn = -1;
        for (int q = 0; q < cnt; ++q) {
            if (!(W > 0.0)) {
                i_end = i0 + q;
                break;
            }
            const double tg = __shfl_sync(0xFFFFFFFFu, my_u, q) * W;
            // a target on (or, rounded, past) the total takes the last cluster with
            // weight: at every level, the first position whose prefix reaches its total
            const bool on_total = !(tg < W);
            int g2 = first_lane(on_total ? T >= W : T > tg);
            if (g2 < 0) g2 = first_lane(T >= W);
            double before = __shfl_sync(0xFFFFFFFFu, Tprev, g2);
            int d, l1 = 0, l0 = 0, base1 = 0, base0 = 0;
            double v1 = 0.0, v0 = 0.0, w;
            if (LEVELS == 1) {
                d = g2;
                w = __shfl_sync(0xFFFFFFFFu, T - Tprev, g2);
            } else {
                int g1 = g2;
                if (LEVELS == 3) {
                    base1 = g2 * 32;
                    v1 = L1[base1 + lane];
                    const double v1p = lane ? L1[base1 + lane - 1] : 0.0;
                    const double tot1 = __shfl_sync(0xFFFFFFFFu, v1, 31);
                    l1 = first_lane(on_total ? v1 >= tot1 : before + v1 > tg);
                    if (l1 < 0) l1 = first_lane(v1 >= tot1);  // (exact sums: never)
                    before += __shfl_sync(0xFFFFFFFFu, v1p, l1);
                    g1 = base1 + l1;
                }
                base0 = g1 * 32;
                v0 = L0[base0 + lane];
                const double v0p = lane ? L0[base0 + lane - 1] : 0.0;
                const double tot0 = __shfl_sync(0xFFFFFFFFu, v0, 31);
                l0 = first_lane(on_total ? v0 >= tot0 : before + v0 > tg);
                if (l0 < 0) l0 = first_lane(v0 >= tot0);  // (exact sums: never)
                d = base0 + l0;
                w = __shfl_sync(0xFFFFFFFFu, v0 - v0p, l0);
            }
            // the donor keeps the rounded half of its weight; explicit roundings, since
            // a fused multiply-add would round the half differently in the subnormal range
            const double keep = __dmul_rn(0.5, w);
            const double delta = __dsub_rn(w, keep);
            if (LEVELS >= 2 && lane >= l0) L0[base0 + lane] = v0 - delta;
            if (LEVELS == 3 && lane >= l1) L1[base1 + lane] = v1 - delta;
            if (lane >= g2) T -= delta;
            if (lane > g2) Tprev -= delta;
            W -= delta;
            if (lane == q) my_dn = d;
            __syncwarp();  // the group stored above may be the next draw's
        }
        const bool has = lane < cnt && my_dn >= 0;
        const unsigned peers = __match_any_sync(0xFFFFFFFFu, has ? my_dn : -1);
        const int leader = __ffs(peers) - 1;
        int old = 0;
        if (has && lane == leader) old = times[my_dn];
        old = __shfl_sync(0xFFFFFFFFu, old, leader);
        if (has) {
            const int rk = __popc(peers & ((1u << lane) - 1u));
            sc.donor[i0 + lane] = my_dn;
            sc.order[i0 + lane] = old + rk;
            if (lane == leader) times[my_dn] = old + __popc(peers);
        } else if (lane < cnt) {
            sc.donor[i0 + lane] = -1;
        }
        splits += __popc(__ballot_sync(0xFFFFFFFFu, has));
        __syncwarp();  // the counters written above are read by other lanes next batch
        if (i_end < nd) break;
    }
    for (int i = (i_end / 32 + 1) * 32 + lane; i < nd; i += 32) sc.donor[i] = -1;
    return splits;
}

// One CTA of kSelectThreads threads: dead set, donor tree, sequential donor draws
// by warp 0 (which keeps one group per tree level in registers).
constexpr int kSelectThreads = 512;
constexpr int kSelectWarps = kSelectThreads / 32;

// Where the selection reads the running counts: N itself, or (off set) the counts
// this step's update is writing, derived from N_prev and the segment sizes with the
// update's own arithmetic (ema_count), so that the selection can run beside it.
struct CountSource {
    const float* N;
    const float* N_prev;
    const int32_t* off;
    double alpha;
    __device__ __forceinline__ float operator()(int j) const {
        return off ? ema_count(N_prev[j], (double)(off[j + 1] - off[j]), alpha) : N[j];
    }
};

__global__ void __launch_bounds__(kSelectThreads) k_revive_select(CountSource N, int k, double tau, uint64_t seed,
                                                        int64_t t, int mode, ReviveScratch sc, int* err) {
    pdl_wait();
    __shared__ double red[32];
    __shared__ int32_t wcount[32];
    __shared__ int32_t base_s;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;

    // total count in a fixed order
    double part = 0.0;
    for (int j = tid; j < k; j += kSelectThreads) part += (double)N(j);
    part = warp_sum(part);
    if (lane == 0) red[w] = part;
    __syncthreads();
    if (w == 0) {
        double v = warp_sum(lane < kSelectWarps ? red[lane] : 0.0);
        if (lane == 0) red[0] = v;
    }
    __syncthreads();
    const double total = red[0];
    const double mean = total / (double)k;
    const double thr = tau * mean;

    // dead set, compacted in increasing index
    if (tid == 0) base_s = 0;
    __syncthreads();
    for (int b = 0; b < k; b += kSelectThreads) {
        const int j = b + tid;
        const bool dead = j < k && (double)N(j) < thr;
        const unsigned m = __ballot_sync(0xFFFFFFFFu, dead);
        if (lane == 0) wcount[w] = __popc(m);
        __syncthreads();
        if (w == 0) {
            const int c = lane < kSelectWarps ? wcount[lane] : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int tt = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += tt;
            }
            wcount[lane] = incl - c;
        }
        __syncthreads();
        if (dead) sc.dead[base_s + wcount[w] + __popc(m & ((1u << lane) - 1u))] = j;
        __syncthreads();
        if (tid == kSelectThreads - 1) base_s += wcount[kSelectWarps - 1] + __popc(m);
        __syncthreads();
    }
    const int nd = base_s;
    if (tid == 0) *sc.ndead = nd;
    if (mode != EM_REVIVE_SPLIT || nd == 0 || !(total > 0.0)) {
        for (int i = tid; i < nd; i += kSelectThreads) sc.donor[i] = -1;
        for (int j = tid; j < k; j += kSelectThreads) sc.times[j] = 0;
        return;
    }

    // draws of every dead cluster, in parallel (they do not depend on each other)
    for (int i = tid; i < nd; i += kSelectThreads) sc.target[i] = draw_uniform(seed, kStreamRevive, t, sc.dead[i]);

    extern __shared__ __align__(16) double smem_d[];
    if (k <= kFastK) {  // radix-32 tree in shared memory
        const Tree32 TL = tree32(k);
        int32_t* times = TL.times >= 0 ? reinterpret_cast<int32_t*>(smem_d + TL.times) : sc.times;
        for (int j = tid; j < k; j += kSelectThreads) times[j] = 0;
        // level 0 (the staging group when it is the top)
        double* L0 = TL.levels == 1 ? smem_d : smem_d + TL.off0;
        for (int g = w; g < TL.n1; g += kSelectWarps) {
            const int j = g * 32 + lane;
            const float nj = j < k ? N(j) : 0.0f;
            const double v = (j < k && !((double)nj < thr)) ? (double)nj : 0.0;
            L0[g * 32 + lane] = lane_scan(v, lane);
        }
        __syncthreads();
        if (TL.levels >= 2) {  // level 1 (staged when it is the top)
            double* L1 = TL.levels == 2 ? smem_d : smem_d + TL.off1;
            for (int g = w; g < TL.n2; g += kSelectWarps) {
                const int i = g * 32 + lane;
                const double v = i < TL.n1 ? L0[i * 32 + 31] : 0.0;
                L1[g * 32 + lane] = lane_scan(v, lane);
            }
            __syncthreads();
        }
        if (TL.levels == 3) {  // level 2, the top
            if (w == 0) {
                const double v = lane < TL.n2 ? smem_d[TL.off1 + lane * 32 + 31] : 0.0;
                smem_d[lane] = lane_scan(v, lane);
            }
            __syncthreads();
        }
        if (w == 0) {
            const int64_t splits = TL.levels == 1   ? draw_radix32<1>(smem_d, TL, nd, sc, times, lane)
                                   : TL.levels == 2 ? draw_radix32<2>(smem_d, TL, nd, sc, times, lane)
                                                    : draw_radix32<3>(smem_d, TL, nd, sc, times, lane);
            if (lane == 0) *sc.n_splits += splits;
        }
        __syncthreads();
        if (TL.times >= 0)
            for (int j = tid; j < k; j += kSelectThreads) sc.times[j] = times[j];
        return;
    }

    // donor tree for larger k (loops over levels have a fixed trip count so that
    // the layout stays in registers)
    const TreeLayout L = tree_layout(k);
    const int top = L.levels - 1;
    double* level_ptr[kTreeLevels];
#pragma unroll
    for (int l = 0; l < kTreeLevels; ++l) {
        if (l == top)
            level_ptr[l] = smem_d;  // staging group of the top level
        else if (l >= L.smem_from)
            level_ptr[l] = smem_d + kRadix + (L.offset[l] - L.smem_base);
        else
            level_ptr[l] = sc.tree + L.offset[l];
    }
    int32_t* times = L.times_smem
                         ? reinterpret_cast<int32_t*>(smem_d + kRadix + (L.smem_end - L.smem_base))
                         : sc.times;
    for (int j = tid; j < k; j += kSelectThreads) times[j] = 0;
#pragma unroll
    for (int l = 0; l < kTreeLevels; ++l) {
        if (l <= top) {
            const int sz = L.size[l];
            const int ngroups = (sz + kRadix - 1) / kRadix;
            double* dst = level_ptr[l];
            const double* below = level_ptr[l > 0 ? l - 1 : 0];
            for (int g = w; g < ngroups; g += kSelectWarps) {
                double v[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int j = g * kRadix + 4 * lane + i;
                    v[i] = 0.0;
                    if (j < sz) {
                        if (l == 0) {
                            const float nj = N(j);
                            v[i] = ((double)nj < thr) ? 0.0 : (double)nj;
                        } else {
                            v[i] = below[(int64_t)j * kRadix + kRadix - 1];  // total of child group j
                        }
                    }
                }
                group_scan(v, lane);
                double2* o = reinterpret_cast<double2*>(dst + (int64_t)g * kRadix + 4 * lane);
                o[0] = make_double2(v[0], v[1]);
                o[1] = make_double2(v[2], v[3]);
            }
        }
        __syncthreads();
    }

    // sequential draws by warp 0: the top group in registers, one group load and
    // store per lower level per draw
    if (w == 0) {
        double T[4];
        {
            const double2* s = reinterpret_cast<const double2*>(smem_d + 4 * lane);
            const double2 a = s[0], b = s[1];
            T[0] = a.x; T[1] = a.y; T[2] = b.x; T[3] = b.y;
        }
        double W = __shfl_sync(0xFFFFFFFFu, T[3], 31);
        int64_t splits = 0;
        int i_end = nd;  // draws from i_end on get no donor (no weight left)
        // deeper trees or global levels: one group per level, any depth
        for (int i0 = 0; i0 < nd; i0 += 32) {
            const int cnt = min(32, nd - i0);
            const double my_u = lane < cnt ? sc.target[i0 + lane] : 0.0;
            int my_dn = -1;
            for (int q = 0; q < cnt; ++q) {
                if (!(W > 0.0)) {
                    i_end = i0 + q;
                    break;
                }
                const double tg = __shfl_sync(0xFFFFFFFFu, my_u, q) * W;
                const bool last = !(tg < W);
                double before, wsel = 0.0;
                // (the weight is needed from the top group only when it is the leaf level)
                int node = top == 0 ? group_select<true>(T, 0.0, tg, last, lane, &before, &wsel)
                                    : group_select<false>(T, 0.0, tg, last, lane, &before, &wsel);
                double base = before;
                const int node_top = node;
                int nodes[kTreeLevels - 1];
                double P[kTreeLevels - 1][4];
#pragma unroll
                for (int l = kTreeLevels - 2; l >= 0; --l) {
                    if (l < top) {
                        const int64_t g0 = (int64_t)node * kRadix + 4 * lane;
                        double2 a, b;
                        if (l >= L.smem_from) {
                            const double2* s = reinterpret_cast<const double2*>(
                                smem_d + kRadix + (L.offset[l] - L.smem_base) + g0);
                            a = s[0];
                            b = s[1];
                        } else {
                            const double2* s = reinterpret_cast<const double2*>(sc.tree + L.offset[l] + g0);
                            a = s[0];
                            b = s[1];
                        }
                        P[l][0] = a.x; P[l][1] = a.y; P[l][2] = b.x; P[l][3] = b.y;
                        const int c = l == 0 ? group_select<true>(P[l], base, tg, last, lane, &before, &wsel)
                                             : group_select<false>(P[l], base, tg, last, lane, &before, &wsel);
                        base += before;
                        node = node * kRadix + c;
                        nodes[l] = node;
                    }
                }
                // the donor keeps the rounded half of its weight (what halving N_d gives);
                // explicit roundings: a fused multiply-add here would round the half
                // differently in the subnormal range
                const double keep = __dmul_rn(0.5, wsel);
                const double delta = __dsub_rn(wsel, keep);
#pragma unroll
                for (int l = 0; l < kTreeLevels - 1; ++l) {
                    if (l < top) {
                        const int g = nodes[l] / kRadix;
                        const int pos = nodes[l] - g * kRadix;
                        const bool st = group_sub(P[l], pos, delta, lane);
                        if (st) {
                            const int64_t g0 = (int64_t)g * kRadix + 4 * lane;
                            double2* s = l >= L.smem_from
                                             ? reinterpret_cast<double2*>(smem_d + kRadix +
                                                                          (L.offset[l] - L.smem_base) + g0)
                                             : reinterpret_cast<double2*>(sc.tree + L.offset[l] + g0);
                            s[0] = make_double2(P[l][0], P[l][1]);
                            s[1] = make_double2(P[l][2], P[l][3]);
                        }
                    }
                }
                group_sub(T, node_top, delta, lane);
                W -= delta;
                if (lane == q) my_dn = node;
            }
            // record the batch: donor, and how many earlier splits took the same donor
            const bool has = lane < cnt && my_dn >= 0;
            const unsigned peers = __match_any_sync(0xFFFFFFFFu, has ? my_dn : -1);
            const int leader = __ffs(peers) - 1;
            int old = 0;
            if (has && lane == leader) old = times[my_dn];
            old = __shfl_sync(0xFFFFFFFFu, old, leader);
            if (has) {
                const int rk = __popc(peers & ((1u << lane) - 1u));
                sc.donor[i0 + lane] = my_dn;
                sc.order[i0 + lane] = old + rk;
                if (lane == leader) times[my_dn] = old + __popc(peers);
            } else if (lane < cnt) {
                sc.donor[i0 + lane] = -1;
            }
            splits += __popc(__ballot_sync(0xFFFFFFFFu, has));
            __syncwarp();  // the counters written above are read by other lanes next batch
            if (i_end < nd) break;
        }
        for (int i = (i_end / 32 + 1) * 32 + lane; i < nd; i += 32) sc.donor[i] = -1;
        if (lane == 0) *sc.n_splits += splits;
    }
    __syncthreads();
    if (L.times_smem)
        for (int j = tid; j < k; j += kSelectThreads) sc.times[j] = times[j];
}

// Dead clusters take their half of the donor (reads the donors' state before
// k_revive_donors changes it).
__global__ void k_revive_dead(ClusterState st, int nv, ReviveScratch sc) {
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int nd = *sc.ndead;
    for (int i = warp; i < nd; i += nwarps) {
        const int dn = sc.donor[i];
        if (dn < 0) continue;
        const int j = sc.dead[i];
        const int o = sc.order[i];
        const float Nj = ldexpf(st.N[dn], -(o + 1));
        float cn_part = 0.0f;
        for (int v = lane; v < nv; v += 32) {
            const float4* cr = reinterpret_cast<const float4*>(st.c + (int64_t)dn * st.ld) + 2 * v;
            const float4 a = cr[0], b = cr[1];
            float cv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            float sv[8];
#pragma unroll
            for (int tt = 0; tt < 8; ++tt) {
                const float sg = ((8 * v + tt) & 1) ? -1.0f : 1.0f;
                float x = cv[tt];
                for (int r = 0; r < o; ++r) x *= (1.0f + kSplitEps * sg);
                x *= (1.0f - kSplitEps * sg);
                cv[tt] = x;
                sv[tt] = Nj * x;
            }
            store_centroid_vec(st.c + (int64_t)j * st.ld, st.cq + (int64_t)j * st.ld, v, cv, cn_part);
            float4* sr = reinterpret_cast<float4*>(st.S + (int64_t)j * st.ld) + 2 * v;
            sr[0] = make_float4(sv[0], sv[1], sv[2], sv[3]);
            sr[1] = make_float4(sv[4], sv[5], sv[6], sv[7]);
        }
        cn_part = warp_sum(cn_part);
        if (lane == 0) {
            st.N[j] = Nj;
            st.cn[j] = cn_part;
        }
    }
}

// Each donor, once, after all its splits: c_d (1 + eps s)^m, N_d / 2^m, S = N c.
__global__ void k_revive_donors(ClusterState st, int nv, ReviveScratch sc) {
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int nd = *sc.ndead;
    for (int i = warp; i < nd; i += nwarps) {
        const int dn = sc.donor[i];
        if (dn < 0) continue;
        const int m = sc.times[dn];
        if (sc.order[i] != m - 1) continue;  // only the last split of this donor acts
        const float Nd = ldexpf(st.N[dn], -m);
        float cn_part = 0.0f;
        for (int v = lane; v < nv; v += 32) {
            float4* cr = reinterpret_cast<float4*>(st.c + (int64_t)dn * st.ld) + 2 * v;
            const float4 a = cr[0], b = cr[1];
            float cv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            float sv[8];
#pragma unroll
            for (int tt = 0; tt < 8; ++tt) {
                const float sg = ((8 * v + tt) & 1) ? -1.0f : 1.0f;
                float x = cv[tt];
                for (int r = 0; r < m; ++r) x *= (1.0f + kSplitEps * sg);
                cv[tt] = x;
                sv[tt] = Nd * x;
            }
            store_centroid_vec(st.c + (int64_t)dn * st.ld, st.cq + (int64_t)dn * st.ld, v, cv, cn_part);
            float4* sr = reinterpret_cast<float4*>(st.S + (int64_t)dn * st.ld) + 2 * v;
            sr[0] = make_float4(sv[0], sv[1], sv[2], sv[3]);
            sr[1] = make_float4(sv[4], sv[5], sv[6], sv[7]);
        }
        cn_part = warp_sum(cn_part);
        if (lane == 0) {
            st.N[dn] = Nd;
            st.cn[dn] = cn_part;
        }
    }
}

// Resample arm: each dead cluster restarts from a row of the current batch.
__global__ void k_revive_resample(ClusterState st, int nv, ReviveScratch sc, const __nv_bfloat16* __restrict__ Xb,
                                  int rows, uint64_t seed, int64_t t) {
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int nd = *sc.ndead;
    for (int i = warp; i < nd; i += nwarps) {
        const int j = sc.dead[i];
        const double u = draw_uniform(seed, kStreamResample, t, j);
        int r = (int)floor(u * (double)rows);
        if (r > rows - 1) r = rows - 1;
        float cn_part = 0.0f;
        for (int v = lane; v < nv; v += 32) {
            float x[8];
            unpack8_bf16(reinterpret_cast<const uint4*>(Xb + (int64_t)r * st.ld)[v], x);
            store_centroid_vec(st.c + (int64_t)j * st.ld, st.cq + (int64_t)j * st.ld, v, x, cn_part);
            float4* sr = reinterpret_cast<float4*>(st.S + (int64_t)j * st.ld) + 2 * v;
            sr[0] = make_float4(0, 0, 0, 0);
            sr[1] = make_float4(0, 0, 0, 0);
        }
        cn_part = warp_sum(cn_part);
        if (lane == 0) {
            st.N[j] = 0.0f;
            st.cn[j] = cn_part;
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) *sc.n_splits += nd;
}

}  // namespace em
