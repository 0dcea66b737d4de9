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
// 16,384 clusters the tree has two levels: groups of 32, 64 or 128 clusters in
// shared memory and a root of at most 128 group totals in the drawing warp's
// registers, each lane holding every 32nd position; a level costs a few compares,
// ballots and population counts. Larger k use 128 children per node (four per
// lane) on as many levels as needed, the lower ones in global memory when shared
// memory runs out. The number of earlier splits from the same donor is counted
// per batch of 32 draws with one warp match. The vector work is then done in
// parallel from the closed form: the o-th split taken from donor d (0-based) sees
// c_d (1 + eps s)^o and N_d / 2^o.
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

// The selection's common start: the total count (in a fixed order), the dead set in
// increasing index, its count, and the uniform draw of every dead cluster. Returns
// false (with the donors and counters written) when no donor is drawn.
__device__ __forceinline__ bool select_prologue(const CountSource& N, int k, double tau, uint64_t seed, int64_t t,
                                                int mode, const ReviveScratch& sc, int& nd_out, double& thr_out) {
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
    thr_out = thr;

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
    nd_out = nd;
    if (tid == 0) *sc.ndead = nd;
    if (mode != EM_REVIVE_SPLIT || nd == 0 || !(total > 0.0)) {
        for (int i = tid; i < nd; i += kSelectThreads) sc.donor[i] = -1;
        for (int j = tid; j < k; j += kSelectThreads) sc.times[j] = 0;
        return false;
    }

    // draws of every dead cluster, in parallel (they do not depend on each other)
    for (int i = tid; i < nd; i += kSelectThreads) sc.target[i] = draw_uniform(seed, kStreamRevive, t, sc.dead[i]);
    return true;
}

__global__ void __launch_bounds__(kSelectThreads) k_revive_select(CountSource N, int k, double tau, uint64_t seed,
                                                        int64_t t, int mode, ReviveScratch sc, int* err) {
    pdl_wait();
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    int nd = 0;
    double thr = 0.0;
    if (!select_prologue(N, k, tau, seed, t, mode, sc, nd, thr)) return;

    extern __shared__ __align__(16) double smem_d[];
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

// ---- two-level tree for k <= kFastK, drawn without a shared-memory round trip
//
// Level 0 holds, for every group of G0 = 32 S0 consecutive clusters, the inclusive
// prefix sums of their current weights within the group (dead clusters and the
// padding past k weigh 0, so padding repeats the group total). The root holds the
// inclusive prefix of the group totals, at most 32 SR entries, in the drawing
// warp's registers. Lane l holds position 32 s + l of a group (or of the root) in
// its slot s, so each lane only ever reads and writes its own positions and the
// descent needs no warp barrier.
//
// A draw counts the positions whose cumulative weight is at most the target: the
// first position past the target is the donor, as in a search of the cumulative
// sums of all k weights. Each level costs S (slots) compares, S ballots and S
// population counts, with no find-first-set and no select over fp64 values. The
// compares are made on the IEEE 754 encodings: for non-negative doubles the order
// of the bit patterns as signed 64-bit integers is the order of the values. A
// target on (or rounded past) the total becomes the largest double below the
// total, so that the first position reaching the total (the last cluster with
// weight) is taken, without a branch.
constexpr int kFastK = 16384;

template <int S0>
EM_HD int flat_groups(int k) { return (k + 32 * S0 - 1) / (32 * S0); }

template <int S0>
EM_HD int flat_smem_bytes(int k) {
    return flat_groups<S0>(k) * 32 * S0 * 8 + ((k * 4 + 15) / 16) * 16;
}

__device__ __forceinline__ long long dbits(double x) { return __double_as_longlong(x); }

// Slot `s` of a lane's N values (N = 1, 2, 4 or 8; any slot when s is out of
// range), by selects on the bits of s: an index into a register array would move
// the array to local memory.
template <int N>
__device__ __forceinline__ double pick(const double (&x)[N], int s) {
    static_assert(N == 1 || N == 2 || N == 4 || N == 8, "1, 2, 4 or 8 slots");
    if (N == 1) return x[0];
    const double a = (s & 1) ? x[1 % N] : x[0];
    if (N == 2) return a;
    const double b = (s & 1) ? x[3 % N] : x[2 % N];
    const double lo = (s & 2) ? b : a;
    if (N == 4) return lo;
    const double c = (s & 1) ? x[5 % N] : x[4 % N];
    const double e = (s & 1) ? x[7 % N] : x[6 % N];
    const double hi = (s & 2) ? e : c;
    return (s & 4) ? hi : lo;
}

template <int S0, int SR>
__global__ void __launch_bounds__(kSelectThreads) k_revive_select_flat(CountSource N, int k, double tau, uint64_t seed,
                                                             int64_t t, int mode, ReviveScratch sc) {
    pdl_wait();
    constexpr int G0 = 32 * S0;
    constexpr int RMAX = kFastK / kSelectThreads;  // rows of kSelectThreads clusters
    __shared__ double red[kSelectWarps];
    __shared__ double ctot[RMAX * kSelectWarps];    // per (row, warp) chunk totals
    __shared__ int32_t rcnt[RMAX * kSelectWarps];   // per (row, warp) dead counts, then offsets
    __shared__ int32_t wsum[kSelectWarps];
    __shared__ double gtot[32 * SR];                // group totals (the root's entries)
    extern __shared__ __align__(16) double smem_d[];
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int R = (k + kSelectThreads - 1) / kSelectThreads;
    const int ngroups = flat_groups<S0>(k);
    double* L0 = smem_d;
    int32_t* times = reinterpret_cast<int32_t*>(smem_d + (int64_t)ngroups * G0);

    // running counts of cluster tid + kSelectThreads r, loaded once; total in the
    // order of the other selection kernel (r, then lanes, then warps)
    float nv[RMAX];
    double part = 0.0;
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        const int j = tid + kSelectThreads * r;
        nv[r] = (r < R && j < k) ? N(j) : 0.0f;
        if (r < R && j < k) part += (double)nv[r];
    }
    part = warp_sum(part);
    if (lane == 0) red[w] = part;
    for (int j = tid; j < k; j += kSelectThreads) times[j] = 0;
    __syncthreads();
    const double total = warp_sum(lane < kSelectWarps ? red[lane] : 0.0);
    const double thr = tau * (total / (double)k);

    // dead set in increasing index: counts per (row, warp), their exclusive scan in
    // row-major order, then each dead cluster's place
    unsigned dmask = 0;
    int my_rc = 0;
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        if (r < R) {
            const int j = tid + kSelectThreads * r;
            const bool dead = j < k && (double)nv[r] < thr;
            dmask |= dead ? (1u << r) : 0u;
            const int c = __popc(__ballot_sync(0xFFFFFFFFu, dead));
            if (lane == r) my_rc = c;
        }
    }
    if (lane < R) rcnt[lane * kSelectWarps + w] = my_rc;
    __syncthreads();
    const int c_in = tid < R * kSelectWarps ? rcnt[tid] : 0;
    int incl = c_in;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[w] = incl;
    __syncthreads();
    const int wv = lane < kSelectWarps ? wsum[lane] : 0;
    int before_w = lane < w ? wv : 0;
    int nd = wv;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        before_w += __shfl_xor_sync(0xFFFFFFFFu, before_w, o);
        nd += __shfl_xor_sync(0xFFFFFFFFu, nd, o);
    }
    if (tid < R * kSelectWarps) rcnt[tid] = before_w + incl - c_in;
    __syncthreads();
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        if (r < R) {
            const bool dead = (dmask >> r) & 1u;
            const unsigned b = __ballot_sync(0xFFFFFFFFu, dead);
            if (dead) sc.dead[rcnt[r * kSelectWarps + w] + __popc(b & ((1u << lane) - 1u))] = tid + kSelectThreads * r;
        }
    }
    if (tid == 0) *sc.ndead = nd;
    if (mode != EM_REVIVE_SPLIT || nd == 0 || !(total > 0.0)) {
        for (int i = tid; i < nd; i += kSelectThreads) sc.donor[i] = -1;
        for (int j = tid; j < k; j += kSelectThreads) sc.times[j] = 0;
        return;
    }

    // level 0 from the loaded counts: warp w's row r is 32 consecutive positions of
    // group (kSelectThreads r + 32 w) / G0, scanned here; the S0 chunks of a group
    // are then joined in order (every sum is exact, see above)
#pragma unroll
    for (int r = 0; r < RMAX; ++r) {
        if (r < R) {
            const int j = tid + kSelectThreads * r;
            const double v = ((dmask >> r) & 1u) || j >= k ? 0.0 : (double)nv[r];
            const double x = warp_incl_scan(v, lane);
            if (j < ngroups * G0) L0[j] = x;
            if (S0 == 1 && lane == 31 && j < ngroups * G0) gtot[j / G0] = x;
            if (S0 > 1 && lane == 31) ctot[r * kSelectWarps + w] = x;
        }
    }
    __syncthreads();  // (also publishes the dead list written above)
    if (S0 > 1) {
#pragma unroll
        for (int r = 0; r < RMAX; ++r) {
            const int j = tid + kSelectThreads * r;
            if (r < R && j < ngroups * G0) {
                const int first = w - (w % S0);
                if (w != first) {
                    double off = 0.0;
                    for (int q = first; q < w; ++q) off += ctot[r * kSelectWarps + q];
                    const double x = L0[j] + off;
                    L0[j] = x;
                    if (lane == 31 && w - first == S0 - 1) gtot[j / G0] = x;
                }
            }
        }
    }
    // draws of every dead cluster, in parallel (they do not depend on each other)
    for (int i = tid; i < nd; i += kSelectThreads) sc.target[i] = draw_uniform(seed, kStreamRevive, t, sc.dead[i]);
    __syncthreads();

    if (w == 0) {
        double T[SR];
        double carry = 0.0;
#pragma unroll
        for (int s = 0; s < SR; ++s) {
            const int pos = 32 * s + lane;
            const double x = warp_incl_scan(pos < ngroups ? gtot[pos] : 0.0, lane) + carry;
            carry = __shfl_sync(0xFFFFFFFFu, x, 31);
            T[s] = pos < ngroups ? x : __longlong_as_double(0x7FF0000000000000ll);  // +inf past the root
        }
        double W = carry;
        int64_t splits = 0;
        double u_cur = lane < nd ? sc.target[lane] : 0.0;
        for (int i0 = 0; i0 < nd; i0 += 32) {
            const int cnt = min(32, nd - i0);
            const double u_next = i0 + 32 + lane < nd ? sc.target[i0 + 32 + lane] : 0.0;
            int my_dn = -1;
            double u = __shfl_sync(0xFFFFFFFFu, u_cur, 0);  // this draw's uniform, taken one draw ahead
            for (int q = 0; q < cnt; ++q) {
                const bool live = W > 0.0;
                const double tg = __dmul_rn(u, W);
                u = __shfl_sync(0xFFFFFFFFu, u_cur, (q + 1) & 31);
                const long long tb = min(dbits(tg), dbits(W) - 1);
                int g = 0;
#pragma unroll
                for (int s = 0; s < SR; ++s) g += __popc(__ballot_sync(0xFFFFFFFFu, dbits(T[s]) <= tb));
                g = min(g, ngroups - 1);
                // cumulative weight of the groups before g: root position g - 1
                const int gp = g - 1;
                const double ts = pick<SR>(T, gp >> 5);
                double before = __shfl_sync(0xFFFFFFFFu, ts, gp & 31);
                if (g == 0) before = 0.0;
                double* grp = L0 + (int64_t)g * G0;
                double v[S0];
#pragma unroll
                for (int s = 0; s < S0; ++s) v[s] = grp[32 * s + lane];
                int p = 0;
#pragma unroll
                for (int s = 0; s < S0; ++s)
                    p += __popc(__ballot_sync(0xFFFFFFFFu, dbits(__dadd_rn(before, v[s])) <= tb));
                p = min(p, G0 - 1);
                // the donor's weight: within-group prefix at p minus the one before it
                const double va = pick<S0>(v, p >> 5);
                const double vb = pick<S0>(v, (p - 1) >> 5);
                const double a = __shfl_sync(0xFFFFFFFFu, va, p & 31);
                double b = __shfl_sync(0xFFFFFFFFu, vb, (p - 1) & 31);
                if (p == 0) b = 0.0;
                const double wt = __dsub_rn(a, b);
                // the donor keeps the rounded half of its weight (what halving N_d gives);
                // explicit roundings: a fused multiply-add would round the half
                // differently in the subnormal range
                const double keep = __dmul_rn(0.5, wt);
                const double delta = live ? __dsub_rn(wt, keep) : 0.0;
#pragma unroll
                for (int s = 0; s < S0; ++s)
                    if (32 * s + lane >= p) grp[32 * s + lane] = __dsub_rn(v[s], delta);
#pragma unroll
                for (int s = 0; s < SR; ++s)
                    if (32 * s + lane >= g) T[s] = __dsub_rn(T[s], delta);
                W = __dsub_rn(W, delta);
                // (a position past k or a drained total can only come from inexact
                // sums, which the weights' range rules out: no donor then)
                const int d = g * G0 + p;
                if (lane == q) my_dn = live && d < k ? d : -1;
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
            u_cur = u_next;
        }
        if (lane == 0) *sc.n_splits += splits;
    }
    __syncthreads();
    for (int j = tid; j < k; j += kSelectThreads) sc.times[j] = times[j];
}

// ---- wide tree for kFastK < k <= kWideK: level 0 in global memory, prefetched ahead
//
// Level 0 (global memory) holds the inclusive prefix of the weights within groups
// of 128 clusters, lane l holding positions 32 s + l (s = 0..3); level 1 (shared
// memory) the inclusive prefix of the level-0 group totals within groups of 32;
// the root (the drawing warp's registers, SR slots) that of the level-1 group
// totals. A draw descends as on the two-level tree. The level-0 group it needs
// is a global load, so each draw also makes the descent of the draw kWideAhead
// places later on the current tree and starts loading the group that one points
// at. When that draw comes, its exact descent decides: if it ends in the same
// group (it nearly always does: the target has moved by a few clusters' weight),
// the copy is used after the updates made since it was loaded, in their order
// (each subtracts the same delta from the same positions as the stored values
// received); else the group is loaded again.
constexpr int kWideG0 = 128;
constexpr int kWideAhead = 4;
constexpr int kWideK = 32 * 8 * 32 * kWideG0;  // with a root of 8 slots per lane

EM_HD int wide_groups0(int k) { return (k + kWideG0 - 1) / kWideG0; }
EM_HD int wide_groups1(int k) { return (wide_groups0(k) + 31) / 32; }
EM_HD int wide_smem_bytes(int k) { return wide_groups1(k) * 32 * 8; }
// root slots per lane for k (1, 2, 4 or 8)
EM_HD int wide_root_slots(int k) {
    const int r = (wide_groups1(k) + 31) / 32;
    return r <= 1 ? 1 : (r <= 2 ? 2 : (r <= 4 ? 4 : 8));
}

template <int SR>
__global__ void __launch_bounds__(kSelectThreads) k_revive_select_wide(CountSource N, int k, double tau,
                                                                      uint64_t seed, int64_t t, int mode,
                                                                      ReviveScratch sc) {
    pdl_wait();
    constexpr int D = kWideAhead;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    int nd = 0;
    double thr = 0.0;
    if (!select_prologue(N, k, tau, seed, t, mode, sc, nd, thr)) return;
    extern __shared__ __align__(16) double smem_d[];
    double* L1 = smem_d;
    double* L0 = sc.tree;
    int32_t* times = sc.times;
    const int n0 = wide_groups0(k), n1 = wide_groups1(k);
    // level 0, one group per warp at a time (the four slots' counts loaded first)
    for (int g0 = w; g0 < n0; g0 += kSelectWarps) {
        double wv[4];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int j = g0 * kWideG0 + 32 * s + lane;
            const float nj = j < k ? N(j) : 0.0f;
            wv[s] = (j < k && !((double)nj < thr)) ? (double)nj : 0.0;
        }
        double carry = 0.0;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const double x = warp_incl_scan(wv[s], lane) + carry;
            carry = __shfl_sync(0xFFFFFFFFu, x, 31);
            L0[(int64_t)g0 * kWideG0 + 32 * s + lane] = x;
        }
        if (lane == 0) L1[g0] = carry;  // the group's total, scanned below
    }
    for (int i = n0 + tid; i < n1 * 32; i += kSelectThreads) L1[i] = 0.0;
    for (int j = tid; j < k; j += kSelectThreads) times[j] = 0;
    __syncthreads();
    for (int g1 = w; g1 < n1; g1 += kSelectWarps) L1[g1 * 32 + lane] = warp_incl_scan(L1[g1 * 32 + lane], lane);
    __syncthreads();  // (also publishes level 0 and the counters to warp 0)
    if (w != 0) return;

    double T[SR];
    double carry = 0.0;
#pragma unroll
    for (int s = 0; s < SR; ++s) {
        const int pos = 32 * s + lane;
        const double x = warp_incl_scan(pos < n1 ? L1[pos * 32 + 31] : 0.0, lane) + carry;
        carry = __shfl_sync(0xFFFFFFFFu, x, 31);
        T[s] = pos < n1 ? x : __longlong_as_double(0x7FF0000000000000ll);
    }
    double W = carry;
    // the descent above level 0 for target bits tb, on the current root and level 1
    auto upper = [&](long long tb, int& g1, double& v1, int& c1, int& g0, double& before0) {
        int gg = 0;
#pragma unroll
        for (int s = 0; s < SR; ++s) gg += __popc(__ballot_sync(0xFFFFFFFFu, dbits(T[s]) <= tb));
        g1 = min(gg, n1 - 1);
        const int gp = g1 - 1;
        double b1 = __shfl_sync(0xFFFFFFFFu, pick<SR>(T, gp >> 5), gp & 31);
        if (g1 == 0) b1 = 0.0;
        v1 = L1[g1 * 32 + lane];
        c1 = min(__popc(__ballot_sync(0xFFFFFFFFu, dbits(__dadd_rn(b1, v1)) <= tb)), 31);
        const double vp = __shfl_sync(0xFFFFFFFFu, v1, (c1 - 1) & 31);
        before0 = c1 ? __dadd_rn(b1, vp) : b1;
        g0 = min(g1 * 32 + c1, n0 - 1);
    };
    // prefetched groups: slot i is for the draw i + 1 places on, loaded before the
    // updates of the draws in between; ug/up/ud: those updates (group, position,
    // delta), oldest first
    double sv[D][4];
    int sg[D], ug[D], up[D];
    double ud[D];
#pragma unroll
    for (int i = 0; i < D; ++i) {
        sg[i] = -1;
        ug[i] = -1;
        up[i] = 0;
        ud[i] = 0.0;
#pragma unroll
        for (int s = 0; s < 4; ++s) sv[i][s] = 0.0;
    }
    int64_t splits = 0;
    double u_cur = lane < nd ? sc.target[lane] : 0.0;
    for (int i0 = 0; i0 < nd; i0 += 32) {
        const int cnt = min(32, nd - i0);
        const double u_next = i0 + 32 + lane < nd ? sc.target[i0 + 32 + lane] : 0.0;
        int my_dn = -1;
        double u = __shfl_sync(0xFFFFFFFFu, u_cur, 0);
        for (int q = 0; q < cnt; ++q) {
            const bool live = W > 0.0;
            const double tg = __dmul_rn(u, W);
            const long long tb = min(dbits(tg), dbits(W) - 1);
            u = __shfl_sync(0xFFFFFFFFu, u_cur, (q + 1) & 31);
            // the uniform of the draw D places on (this batch or the next)
            const int qa = q + D;
            const double ua = qa < 32 ? __shfl_sync(0xFFFFFFFFu, u_cur, qa & 31)
                                      : __shfl_sync(0xFFFFFFFFu, u_next, (qa - 32) & 31);
            const bool ahead = i0 + qa < nd;
            int g1, c1, g0;
            double v1, before0;
            upper(tb, g1, v1, c1, g0, before0);
            // this draw's level-0 group: the copy loaded D draws ago, brought up to date
            double v0[4];
            if (sg[0] == g0) {
#pragma unroll
                for (int s = 0; s < 4; ++s) v0[s] = sv[0][s];
#pragma unroll
                for (int i = 0; i < D; ++i)
                    if (ug[i] == g0)
#pragma unroll
                        for (int s = 0; s < 4; ++s)
                            if (32 * s + lane >= up[i]) v0[s] = __dsub_rn(v0[s], ud[i]);
            } else {
#pragma unroll
                for (int s = 0; s < 4; ++s) v0[s] = L0[(int64_t)g0 * kWideG0 + 32 * s + lane];
            }
            // the descent of the draw D places on, on the tree as it is now, and its load
            int ag0 = -1;
            double av[4] = {0.0, 0.0, 0.0, 0.0};
            if (ahead) {
                const double tga = __dmul_rn(ua, W);
                const long long tba = min(dbits(tga), dbits(W) - 1);
                int a1, ac1;
                double av1, ab0;
                upper(tba, a1, av1, ac1, ag0, ab0);
#pragma unroll
                for (int s = 0; s < 4; ++s) av[s] = L0[(int64_t)ag0 * kWideG0 + 32 * s + lane];
            }
            // level 0 of this draw
            int p = 0;
#pragma unroll
            for (int s = 0; s < 4; ++s)
                p += __popc(__ballot_sync(0xFFFFFFFFu, dbits(__dadd_rn(before0, v0[s])) <= tb));
            p = min(p, kWideG0 - 1);
            const double va = pick<4>(v0, p >> 5);
            const double vb = pick<4>(v0, (p - 1) >> 5);
            const double a = __shfl_sync(0xFFFFFFFFu, va, p & 31);
            double b = __shfl_sync(0xFFFFFFFFu, vb, (p - 1) & 31);
            if (p == 0) b = 0.0;
            const double wt = __dsub_rn(a, b);
            // the donor keeps the rounded half of its weight (explicit roundings, as above)
            const double keep = __dmul_rn(0.5, wt);
            const double delta = live ? __dsub_rn(wt, keep) : 0.0;
#pragma unroll
            for (int s = 0; s < 4; ++s)
                if (32 * s + lane >= p) L0[(int64_t)g0 * kWideG0 + 32 * s + lane] = __dsub_rn(v0[s], delta);
            if (lane >= c1) L1[g1 * 32 + lane] = __dsub_rn(v1, delta);
#pragma unroll
            for (int s = 0; s < SR; ++s)
                if (32 * s + lane >= g1) T[s] = __dsub_rn(T[s], delta);
            W = __dsub_rn(W, delta);
            // the rings move on by one draw
#pragma unroll
            for (int i = 0; i + 1 < D; ++i) {
                sg[i] = sg[i + 1];
                ug[i] = ug[i + 1];
                up[i] = up[i + 1];
                ud[i] = ud[i + 1];
#pragma unroll
                for (int s = 0; s < 4; ++s) sv[i][s] = sv[i + 1][s];
            }
            sg[D - 1] = ag0;
            ug[D - 1] = g0;
            up[D - 1] = p;
            ud[D - 1] = delta;
#pragma unroll
            for (int s = 0; s < 4; ++s) sv[D - 1][s] = av[s];
            const int d = g0 * kWideG0 + p;
            if (lane == q) my_dn = live && d < k ? d : -1;
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
        u_cur = u_next;
    }
    if (lane == 0) *sc.n_splits += splits;
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
