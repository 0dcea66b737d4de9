// k_reduce.cuh -- per-cluster count and sum of a batch, fused with the EMA update.
//
// faiss e-means README, "How the centroid updates work": with n_j and s_j the
// count and sum of the batch rows assigned to cluster j,
//     N_j <- (1 - a) N_j + a n_j,   S_j <- (1 - a) S_j + a s_j,   c_j = S_j / N_j.
//
// The batch is grouped by label instead of adding rows into S with global atomics:
//   k_labels   decodes each row's search key, counts labels per cluster with
//              warp-aggregated atomics (__match_any_sync: one atomic per distinct
//              label per warp) and records each row's rank inside its cluster;
//   k_offsets  exclusive scans of the counts (segment starts) and of the chunk
//              counts (work items), batch error sum;
//   k_scatter  writes row ids into label order (perm) and one work item per chunk;
//   k_segsum   one warp per (chunk of at most R rows of one cluster, 256-dim
//              slice), so a cluster with many rows is spread over many warps and
//              small clusters never wait on each other: a cluster of one chunk is
//              summed (fp64) and updated at once; the chunks of a larger cluster
//              leave partial sums;
//   k_clusters one warp per cluster: adds the chunk partials of large clusters in
//              chunk order and updates them, decays clusters that received no row,
//              and assembles |bf16(c)|^2.
// Sums are accumulated in fp64 from bf16 values, which makes them independent of
// the order rows arrive in (the fp64 sum of bf16 values is exact for the data
// ranges used here), so the update is deterministic.
#pragma once

#include "k_data.cuh"

namespace em {

struct StepParams {
    double alpha;        // step size of this step
    int last_pass;       // accumulate the closing-mean statistics
    int capture_labels;  // record the last-pass label of each row
    // Data-parallel steps: instead of updating the clusters, the sums leave this
    // rank's batch statistics in stats (k x ld fp64 sums s_j, then k counts n_j,
    // then the error sum), to be added across ranks before k_apply_stats. nullptr:
    // the update is applied here.
    double* stats;
};

// ---------------------------------------------------------------- labels + histogram

// Relative size of a near tie, measured against |x|^2 + |s1| + |s2|: a gap between the
// two best scores above this can not be reversed by the fp32 accumulation of the
// search, a smaller one is settled exactly.
constexpr float kTieRel = 3e-5f;

// Best and second best keys of row r over the splits of the search.
__device__ __forceinline__ void merge_keys(const unsigned long long* __restrict__ keys, int64_t rows, int nsplit,
                                           int64_t r, unsigned long long& k1, unsigned long long& k2) {
    k1 = kEmptyKey;
    k2 = kEmptyKey;
    // the first eight splits: all loads issued before the first compare
    unsigned long long c[8][2];
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        c[g][0] = c[g][1] = kEmptyKey;
        if (g < nsplit) {
            const ulonglong2 kk = reinterpret_cast<const ulonglong2*>(keys)[(int64_t)g * rows + r];
            c[g][0] = kk.x;
            c[g][1] = kk.y;
        }
    }
    for (int g = 8; g < nsplit; ++g) {  // more splits (small inputs of a full pass)
        const ulonglong2 kk = reinterpret_cast<const ulonglong2*>(keys)[(int64_t)g * rows + r];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const unsigned long long x = e ? kk.y : kk.x;
            if (x < k1) {
                k2 = k1;
                k1 = x;
            } else if (x < k2) {
                k2 = x;
            }
        }
    }
#pragma unroll
    for (int g = 0; g < 8; ++g)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const unsigned long long x = c[g][e];
            if (x < k1) {
                k2 = k1;
                k1 = x;
            } else if (x < k2) {
                k2 = x;
            }
        }
}

// What the per-row value written by the label kernels means. The search score of a
// row is s = |bf16(c)|^2 - 2 x.bf16(c) for k-means and s = -2 x.bf16(c) for spherical
// e-means (faiss e-means README, "Spherical e-means": unit centroids, highest dot
// product, error 2 - 2 x similarity).
enum RowValue : int {
    kSquaredDistance = 0,  // max(0, |x|^2 + s): the squared distance
    kSphericalError = 1,   // 2 + s = 2 - 2 x.c: the spherical error of the row
    kSimilarity = 2,       // -s / 2 = x.c: the similarity (spherical assign)
};

// How a squared distance follows from a score: (x2 + mul * score) * dscale. The bf16
// search has mul = dscale = 1; the FP8 search scores half the squared distance in
// code units (mul = 2) and reports it in the data's units (dscale = 1 / scale^2).
// tie_rel: the near-tie window settled in fp64 (kTieRel), or < 0 for none (the
// FP8 search, whose exact comparison would be on codes the settling does not read).
struct ScoreScale {
    float mul, dscale, tie_rel;
};

__device__ __forceinline__ float row_value(int kind, float x2, float s, ScoreScale sc = {1.0f, 1.0f, kTieRel}) {
    if (kind == kSquaredDistance) return fmaxf(0.0f, x2 + sc.mul * s) * sc.dscale;
    if (kind == kSphericalError) return 2.0f + s;
    return -0.5f * s;
}

// The row's contribution to the error sum: the squared distance, or 2 - 2 x similarity.
__device__ __forceinline__ float row_error(int kind, float x2, float s, ScoreScale sc = {1.0f, 1.0f, kTieRel}) {
    return kind == kSquaredDistance ? fmaxf(0.0f, x2 + sc.mul * s) * sc.dscale : 2.0f + s;
}

// fp64 comparison value of candidate q for a near tie, from the bf16 row x and the
// bf16 operand q (= -2 bf16(c), so c = -q / 2 exactly): |x - c|^2 for k-means, the
// score x.q = -2 x.c for spherical e-means. Lanes add disjoint 8-element vectors.
__device__ __forceinline__ void tie_terms(bool spherical, const uint4& xv, const uint4& qa_v, const uint4& qb_v,
                                          double& da, double& db) {
    float x[8], qa[8], qb[8];
    unpack8_bf16(xv, x);
    unpack8_bf16(qa_v, qa);
    unpack8_bf16(qb_v, qb);
    if (spherical) {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            da += (double)x[t] * (double)qa[t];
            db += (double)x[t] * (double)qb[t];
        }
    } else {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const double ea = (double)x[t] + 0.5 * (double)qa[t];
            const double eb = (double)x[t] + 0.5 * (double)qb[t];
            da += ea * ea;
            db += eb * eb;
        }
    }
}

// For every lane of the warp whose row is a near tie (flag), the warp recomputes
// the comparison value of both candidates in fp64 (tie_terms) and keeps the smaller
// (the lower index on an exact tie).
__device__ __forceinline__ void settle_ties(bool flag, int64_t row, uint32_t& l1, float& s1, uint32_t l2, float s2,
                                            const __nv_bfloat16* __restrict__ A, int ld,
                                            const __nv_bfloat16* __restrict__ cq, bool spherical, int lane) {
    unsigned fm = __ballot_sync(0xFFFFFFFFu, flag);
    const int nv = ld / 8;
    while (fm) {
        const int q = __ffs(fm) - 1;
        fm &= fm - 1;
        const int64_t rq = __shfl_sync(0xFFFFFFFFu, row, q);
        const uint32_t la = __shfl_sync(0xFFFFFFFFu, l1, q), lb = __shfl_sync(0xFFFFFFFFu, l2, q);
        double da = 0.0, db = 0.0;
        for (int v = lane; v < nv; v += 32)
            tie_terms(spherical, reinterpret_cast<const uint4*>(A + rq * ld)[v],
                      reinterpret_cast<const uint4*>(cq + (int64_t)la * ld)[v],
                      reinterpret_cast<const uint4*>(cq + (int64_t)lb * ld)[v], da, db);
        da = warp_sum(da);
        db = warp_sum(db);
        if (lane == q && (db < da || (db == da && lb < la))) {
            l1 = lb;
            s1 = s2;
        }
    }
}

// Near-tie rows are settled after the label kernels, one warp per row and all rows
// in parallel (k_settle): the label kernels write the provisional best candidate
// and append the row here.
struct TieList {
    int4* e;       // (row, first label, second label, bits of the second score)
    int* n;        // entries
    double* corr;  // sum of the distance changes of the rows k_settle relabels
};

// Appends this warp's flagged rows to the tie list (one atomic per warp).
__device__ __forceinline__ void push_ties(bool flag, int64_t r, uint32_t l1, uint32_t l2, float s2, const TieList& tl,
                                          int lane) {
    const unsigned m = __ballot_sync(0xFFFFFFFFu, flag);
    if (!m) return;
    int base = 0;
    if (lane == 0) base = atomicAdd(tl.n, __popc(m));
    base = __shfl_sync(0xFFFFFFFFu, base, 0);
    if (flag) tl.e[base + __popc(m & ((1u << lane) - 1u))] = make_int4((int)r, (int)l1, (int)l2, __float_as_int(s2));
}

__global__ void k_labels(const unsigned long long* __restrict__ keys, int nsplit, const float* __restrict__ xn,
                         int rows, int k, const __nv_bfloat16* __restrict__ A, int ld,
                         const __nv_bfloat16* __restrict__ cq, const int32_t* __restrict__ ids,
                         int32_t* __restrict__ labels, float* __restrict__ dists, int32_t* __restrict__ cnt,
                         int32_t* __restrict__ rank, double* __restrict__ block_err, int64_t* __restrict__ labels_last,
                         int capture, int kind, ScoreScale sc, TieList tl, const float* __restrict__ N,
                         float* __restrict__ N_prev, int* err) {
    pdl_wait();
    pdl_release();
    __shared__ double warp_err[32];
    const int lane = threadIdx.x & 31;
    double e = 0.0;
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    const bool active = r < rows;
    // the running counts of before this step (N_prev), which the update and the
    // revival selection derive the new counts from: one per thread across the grid
    for (int j = r; j < k; j += gridDim.x * blockDim.x) N_prev[j] = N[j];
    uint32_t l1 = 0, l2 = 0;
    float s1 = 0.0f, s2 = 0.0f, x2 = 0.0f;
    bool tie = false;
    if (active) {
        unsigned long long k1, k2;
        merge_keys(keys, rows, nsplit, r, k1, k2);
        l1 = key_label(k1);
        s1 = key_score(k1);
        x2 = xn[r];
        if (l1 >= (uint32_t)k) {  // a row that was never searched, or a corrupted key
            raise_error(err, EM_E_BOUNDS);
            l1 = 0;
        }
        if (k2 != kEmptyKey) {
            l2 = key_label(k2);
            s2 = key_score(k2);
            tie = sc.tie_rel >= 0.0f && l2 < (uint32_t)k && s2 - s1 <= sc.tie_rel * (x2 + fabsf(s1) + fabsf(s2));
        }
    }
    // a near tie is left to k_settle: provisional label and distance now, counted there
    const bool defer = tie && tl.e != nullptr;
    if (tl.e)
        push_ties(defer, r, l1, l2, s2, tl, lane);
    else
        settle_ties(tie, r, l1, s1, l2, s2, A, ld, cq, kind != kSquaredDistance, lane);
    int lab = -1;
    if (active) {
        lab = (int)l1;
        labels[r] = lab;
        dists[r] = row_value(kind, x2, s1, sc);
        e = (double)row_error(kind, x2, s1, sc);
        if (capture && !defer) labels_last[ids[r]] = lab;
    }
    const bool counted = active && !defer;
    const unsigned amask = __ballot_sync(0xFFFFFFFFu, counted);
    if (counted) {
        const unsigned peers = __match_any_sync(amask, lab);
        const int leader = __ffs(peers) - 1;
        const int before = __popc(peers & ((1u << lane) - 1u));
        int base = 0;
        if (lane == leader) base = atomicAdd(&cnt[lab], __popc(peers));
        base = __shfl_sync(peers, base, leader);
        rank[r] = base + before;
    }
    e = warp_sum(e);
    if (lane == 0) warp_err[threadIdx.x >> 5] = e;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += warp_err[w];
        block_err[blockIdx.x] = t;
    }
}

// Exclusive scans of the counts (segment starts off[0..k]) and of the chunk counts
// ceil(n_j / R) (first work item of each cluster, poff[0..k]); one CTA of 1024
// threads, 16 consecutive clusters per thread (one pass up to 16,384 clusters).
// Also adds the per-block error sums in a fixed order (each thread its strided
// share, then a fixed butterfly and the warps in order), issued ahead of the scan.
constexpr int kOffsetsPer = 16;

__global__ void __launch_bounds__(1024) k_offsets(const int32_t* __restrict__ cnt, int k, int rows, int R,
                                                  int32_t* __restrict__ off, int32_t* __restrict__ poff,
                                                  const double* __restrict__ block_err, int nblocks,
                                                  double* __restrict__ err_sum_out, TieList tl, int* err) {
    pdl_wait();
    pdl_release();
    __shared__ int2 warp_tot[32];
    __shared__ int2 carry_s;
    __shared__ double warp_err[32];
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    double e = 0.0;
    for (int b = tid; b < nblocks; b += 1024) e += block_err[b];
    if (tid == 0) carry_s = make_int2(0, 0);
    e = warp_sum(e);
    if (lane == 0) warp_err[w] = e;
    __syncthreads();
    const bool vec = (k % 4) == 0;  // 16-byte loads and stores of the counts and offsets
    for (int base = 0; base < k; base += 1024 * kOffsetsPer) {
        int v[kOffsetsPer], c[kOffsetsPer];
        const int i0 = base + tid * kOffsetsPer;
        if (vec && i0 + kOffsetsPer <= k) {
#pragma unroll
            for (int q = 0; q < kOffsetsPer / 4; ++q) {
                const int4 x = reinterpret_cast<const int4*>(cnt + i0)[q];
                v[4 * q] = x.x; v[4 * q + 1] = x.y; v[4 * q + 2] = x.z; v[4 * q + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < kOffsetsPer; ++i) v[i] = (i0 + i < k) ? cnt[i0 + i] : 0;
        }
        int local_v = 0, local_c = 0;
#pragma unroll
        for (int i = 0; i < kOffsetsPer; ++i) {
            c[i] = (v[i] + R - 1) / R;
            local_v += v[i];
            local_c += c[i];
        }
        int iv = local_v, ic = local_c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int tv = __shfl_up_sync(0xFFFFFFFFu, iv, o);
            const int tc = __shfl_up_sync(0xFFFFFFFFu, ic, o);
            if (lane >= o) {
                iv += tv;
                ic += tc;
            }
        }
        if (lane == 31) warp_tot[w] = make_int2(iv, ic);
        __syncthreads();
        if (w == 0) {
            const int2 x = warp_tot[lane];
            int xv = x.x, xc = x.y;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int tv = __shfl_up_sync(0xFFFFFFFFu, xv, o);
                const int tc = __shfl_up_sync(0xFFFFFFFFu, xc, o);
                if (lane >= o) {
                    xv += tv;
                    xc += tc;
                }
            }
            warp_tot[lane] = make_int2(xv - x.x, xc - x.y);  // exclusive prefixes of the warp totals
        }
        __syncthreads();
        const int2 carry = carry_s;
        int rv = carry.x + warp_tot[w].x + iv - local_v;
        int rc = carry.y + warp_tot[w].y + ic - local_c;
        int ov[kOffsetsPer], oc[kOffsetsPer];
#pragma unroll
        for (int i = 0; i < kOffsetsPer; ++i) {
            ov[i] = rv;
            oc[i] = rc;
            rv += v[i];
            rc += c[i];
        }
        if (vec && i0 + kOffsetsPer <= k) {
#pragma unroll
            for (int q = 0; q < kOffsetsPer / 4; ++q) {
                reinterpret_cast<int4*>(off + i0)[q] = make_int4(ov[4 * q], ov[4 * q + 1], ov[4 * q + 2], ov[4 * q + 3]);
                reinterpret_cast<int4*>(poff + i0)[q] = make_int4(oc[4 * q], oc[4 * q + 1], oc[4 * q + 2], oc[4 * q + 3]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < kOffsetsPer; ++i)
                if (i0 + i < k) {
                    off[i0 + i] = ov[i];
                    poff[i0 + i] = oc[i];
                }
        }
        __syncthreads();
        if (tid == 1023) carry_s = make_int2(rv, rc);
        __syncthreads();
    }
    if (w == 0) {  // batch error: the warps' sums in warp order
        double t = warp_err[lane];
        t = warp_sum(t);
        if (lane == 0) {
            off[k] = carry_s.x;
            poff[k] = carry_s.y;
            if (carry_s.x != rows) raise_error(err, EM_E_BOUNDS);
            if (tl.n) {  // the relabelled near ties (k_settle ran before), then an empty list
                t += *tl.corr;
                *tl.n = 0;
                *tl.corr = 0.0;
            }
            *err_sum_out = t;
        }
    }
}

// perm[pos] is the row the segmented sums read. The first row of every chunk of R
// rows of a cluster also writes that chunk's work item (cluster, first sorted position).
__global__ void k_scatter(const int32_t* __restrict__ labels, const int32_t* __restrict__ rank,
                          const int32_t* __restrict__ off, const int32_t* __restrict__ poff, int rows, int R,
                          int32_t* __restrict__ perm, int4* __restrict__ items, int* err) {
    pdl_wait();
    pdl_release();
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    const int lab = labels[r];
    const int rk = rank[r];
    const int pos = off[lab] + rk;
    if (pos < 0 || pos >= rows) {
        raise_error(err, EM_E_BOUNDS);
        return;
    }
    perm[pos] = r;
    if (rk % R == 0) {  // work item: (cluster, first row, end row, cluster fits in one chunk)
        const int s0 = off[lab], s1 = off[lab + 1];
        items[poff[lab] + rk / R] = make_int4(lab, pos, min(pos + R, s1), s1 - s0 <= R ? 1 : 0);
    }
}

// ---------------------------------------------------------------- segmented sums + EMA

// State the update kernels read and write. N_prev is the running count before this
// step (copied by k_offsets), so that every slice of a cluster derives the same new
// count; cnp[s * k + j] is slice s's part of |bf16(c_j)|^2, added in slice order by
// k_clusters.
struct ClusterState {
    float* N;
    float* N_prev;
    float* S;
    float* c;
    __nv_bfloat16* cq;
    float* cn;
    float* cnp;
    double* close_sum;
    double* close_cnt;
    int ld;
    int k;
};

// A slice is 32 16-byte vectors (256 dims) of a row. A warp covers a slice of
// `rpi` rows at once: lane l handles vector (l % lpr) of row (l / lpr), lpr being
// the lanes per row (32, or fewer when the row has fewer than 32 vectors).
struct SliceGeom {
    int vbase;  // first vector of the slice
    int nvs;    // vectors in this slice
    int lpr;    // lanes per row (power of two >= nvs, <= 32)
    int rpi;    // rows per warp iteration = 32 / lpr
};

__device__ __forceinline__ SliceGeom slice_geom(int slice, int nv) {
    SliceGeom g;
    g.vbase = slice * 32;
    g.nvs = min(32, nv - g.vbase);
    int l = 1;
    while (l < g.nvs) l <<= 1;
    g.lpr = l;
    g.rpi = 32 / l;
    return g;
}

// Rows per work item of the grouped update (one chunk of a cluster).
// Launch-shape constants of the grouped update (set at build time for sweeps).
#ifndef EM_CHUNK_ROWS
#define EM_CHUNK_ROWS 64
#endif
constexpr int kChunkRows = EM_CHUNK_ROWS;

// Row groups of a work item in flight per warp in k_segsum (a group is the `rpi`
// rows a warp covers at once), staged through a ring in shared memory.
constexpr int kSegsumDepth = 12;
static_assert(kChunkRows <= 64, "an item's row ids are preloaded two per lane");

__device__ __forceinline__ void seg_cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void seg_cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void seg_cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// sum_rows with the rows staged through shared memory: the item's row ids are
// loaded at once (two per lane, coalesced) and handed out by shuffles, and every
// lane copies its own 16-byte vector of each row with cp.async, kSegsumDepth row
// groups ahead of the adds. Each lane reads back only the vectors it copied
// itself, so the lanes need no barrier. The sums are the same fp64 sums as
// sum_rows (exact, so the order of the rows does not matter).
__device__ __forceinline__ void sum_rows_staged(double acc[8], const __nv_bfloat16* __restrict__ src, int ld,
                                                const int32_t* __restrict__ perm, int s0, int s1,
                                                const SliceGeom& g, int lane, uint4* ring) {
    constexpr int D = kSegsumDepth;
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[t] = 0.0;
    const int n = s1 - s0;
    const int sub = lane / g.lpr, vi = lane % g.lpr;
    const bool vec_ok = vi < g.nvs;
    const int v = g.vbase + vi;
    const int id0 = lane < n ? perm[s0 + lane] : 0;
    const int id1 = 32 + lane < n ? perm[s0 + 32 + lane] : 0;
    const int ngroups = (n + g.rpi - 1) / g.rpi;
    const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
    auto issue = [&](int grp) {
        const int p = grp * g.rpi + sub;  // row of the item (only p < 64 is ever used)
        const int a = __shfl_sync(0xFFFFFFFFu, id0, p & 31);
        const int b = __shfl_sync(0xFFFFFFFFu, id1, p & 31);
        if (grp < ngroups && vec_ok && p < n)
            seg_cp_async16(ring_s + (uint32_t)(((grp % D) * 32 + lane) * 16),
                           src + (int64_t)(p < 32 ? a : b) * ld + 8 * v);
        seg_cp_async_commit();  // (an empty group past the end keeps the count)
    };
#pragma unroll 1
    for (int grp = 0; grp < D; ++grp) issue(grp);
#pragma unroll 1
    for (int grp = 0; grp < ngroups; ++grp) {
        seg_cp_async_wait<D - 1>();  // this lane's copy of group grp has landed
        const int p = grp * g.rpi + sub;
        if (vec_ok && p < n) {
            float x[8];
            unpack8_bf16(ring[(grp % D) * 32 + lane], x);
#pragma unroll
            for (int t = 0; t < 8; ++t) acc[t] += (double)x[t];
        }
        issue(grp + D);
    }
    seg_cp_async_wait<0>();
    for (int o = g.lpr; o < 32; o <<= 1)
#pragma unroll
        for (int t = 0; t < 8; ++t) acc[t] += __shfl_xor_sync(0xFFFFFFFFu, acc[t], o);
}

// S row slice of cluster j for lanes l < nvs (vector vbase + l), loaded ahead of use.
__device__ __forceinline__ void load_s(const ClusterState& st, int j, const SliceGeom& g, int lane, float so[8]) {
    if (lane < g.nvs) {
        const float4* sp = reinterpret_cast<const float4*>(st.S + (int64_t)j * st.ld) + 2 * (g.vbase + lane);
        const float4 s0 = sp[0], s1 = sp[1];
        so[0] = s0.x; so[1] = s0.y; so[2] = s0.z; so[3] = s0.w;
        so[4] = s1.x; so[5] = s1.y; so[6] = s1.z; so[7] = s1.w;
    }
}

// The running count after the step: (1 - a) N_prev + a n_j, with explicit roundings
// so that every kernel that recomputes it (the revival selection overlaps the
// segmented sums and derives the counts itself) gets the same fp32 value.
__device__ __forceinline__ float ema_count(float nprev, double nj, double alpha) {
    const double a1 = __dsub_rn(1.0, alpha);
    if (nj == 0.0) return (float)__dmul_rn(a1, (double)nprev);
    return (float)__dadd_rn(__dmul_rn(a1, (double)nprev), __dmul_rn(alpha, nj));
}

// The centroid is S / N rounded to fp32, computed as the IEEE fp32 quotient of the
// fp32 S and N: dividing in fp64 and rounding to fp32 gives the same value, since
// a 53-bit quotient rounded again to 24 bits is the correctly rounded 24-bit
// quotient (53 >= 2 x 24 + 2; Figueroa, "When is double rounding innocuous?",
// 1995), and fp32 operands can neither overflow nor underflow in fp64.
// EMA of one slice of cluster j from its batch sums (lanes l < nvs hold vector
// vbase + l) and its previous sums so[]: writes S, c, the bf16 operand and the
// closing-mean sums; slice 0 also writes N and the closing-mean count. Returns
// the slice's part of |bf16(c_j)|^2 (the same value in every lane).
__device__ __forceinline__ float ema_slice(const ClusterState& st, int j, double nj, float nprev, int slice,
                                           const SliceGeom& g, const double acc[8], const float so[8], int lane,
                                           double alpha, int last_pass) {
    const double a1 = 1.0 - alpha;
    const float Nnew = ema_count(nprev, nj, alpha);
    float cn_part = 0.0f;
    if (lane < g.nvs) {
        const int v = g.vbase + lane;
        float sn[8], cv[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            sn[t] = (float)(a1 * (double)so[t] + alpha * acc[t]);
            cv[t] = __fdiv_rn(sn[t], Nnew);  // = (float)((double)sn / (double)N): see above
        }
        float4* sp = reinterpret_cast<float4*>(st.S + (int64_t)j * st.ld) + 2 * v;
        sp[0] = make_float4(sn[0], sn[1], sn[2], sn[3]);
        sp[1] = make_float4(sn[4], sn[5], sn[6], sn[7]);
        store_centroid_vec(st.c + (int64_t)j * st.ld, st.cq + (int64_t)j * st.ld, v, cv, cn_part);
        if (last_pass) {
            double* cs = st.close_sum + (int64_t)j * st.ld + 8 * v;
#pragma unroll
            for (int t = 0; t < 8; ++t) cs[t] += acc[t];
        }
    }
    cn_part = warp_sum(cn_part);
    if (lane == 0 && slice == 0) {
        st.N[j] = Nnew;
        if (last_pass) st.close_cnt[j] += nj;
    }
    return cn_part;
}

// One warp per (work item, slice). A work item is a chunk of at most R label-sorted
// rows of one cluster, and carries (cluster, first row, end row, whether the
// cluster fits in one chunk), so that the row ids, the S slice and the previous
// count are all fetched right after the item; the rows stream through the warp's
// ring in shared memory (sum_rows_staged). A
// cluster that fits in one chunk is updated here; the chunks of a larger cluster
// leave their slice sums in part[item] for k_clusters.
#ifndef EM_SEGSUM_MIN_BLOCKS
#define EM_SEGSUM_MIN_BLOCKS 3
#endif
__global__ void __launch_bounds__(256, EM_SEGSUM_MIN_BLOCKS) k_segsum(const __nv_bfloat16* __restrict__ src,
                                                   const int32_t* __restrict__ perm, const int4* __restrict__ items,
                                                   const int32_t* __restrict__ poff, int nslices, int nv,
                                                   ClusterState st, StepParams sp, double* __restrict__ part) {
    pdl_wait();
    pdl_release();
    extern __shared__ __align__(16) uint4 seg_ring[];  // kSegsumDepth x 32 vectors per warp
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int item = warp / nslices, slice = warp - item * nslices;
    if (item >= poff[st.k]) return;
    const int4 it = items[item];
    const int j = it.x, n = it.z - it.y;
    const SliceGeom g = slice_geom(slice, nv);
    float so[8];
    float nprev = 0.0f;
    if (it.w) {
        load_s(st, j, g, lane, so);
        nprev = st.N_prev[j];
    }
    double acc[8];
    sum_rows_staged(acc, src, st.ld, perm, it.y, it.z, g, lane,
                    seg_ring + (size_t)(threadIdx.x >> 5) * kSegsumDepth * 32);
    if (it.w && sp.stats) {  // this rank's sums of the cluster, for the exchange
        if (lane < g.nvs) {
            double* dst = sp.stats + (int64_t)j * st.ld + 8 * (g.vbase + lane);
#pragma unroll
            for (int t = 0; t < 8; ++t) dst[t] = acc[t];
        }
        if (lane == 0 && slice == 0) sp.stats[(int64_t)st.k * st.ld + j] = (double)n;
    } else if (it.w) {
        const float cn_part = ema_slice(st, j, (double)n, nprev, slice, g, acc, so, lane, sp.alpha, sp.last_pass);
        if (lane == 0) st.cnp[(int64_t)slice * st.k + j] = cn_part;
    } else if (lane < g.nvs) {
        double* dst = part + (int64_t)item * st.ld + 8 * (g.vbase + lane);
#pragma unroll
        for (int t = 0; t < 8; ++t) dst[t] = acc[t];
    }
}

// One warp per cluster, after k_segsum: a cluster without rows decays (S and N by
// 1 - alpha; its centroid S/N is unchanged); a cluster of one chunk gets
// |bf16(c)|^2 as the sum of its slice parts in slice order; a cluster of several
// chunks adds their partial sums in chunk order (four in flight) and is updated
// here. Clears the counts for the next step.
__global__ void k_clusters(const int32_t* __restrict__ off, const int32_t* __restrict__ poff,
                           int32_t* __restrict__ cnt, int R, int nslices, int nv, ClusterState st, StepParams sp,
                           const double* __restrict__ part) {
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const double a1 = 1.0 - sp.alpha;
    for (int j = warp; j < st.k; j += nwarps) {
        const int nj = off[j + 1] - off[j];
        if (lane == 0) cnt[j] = 0;
        if (sp.stats) {  // this rank's statistics of cluster j, for the exchange
            double* row = sp.stats + (int64_t)j * st.ld;
            if (nj == 0) {
                for (int v = lane; v < st.ld / 4; v += 32)
                    reinterpret_cast<double4*>(row)[v] = make_double4(0.0, 0.0, 0.0, 0.0);
                if (lane == 0) sp.stats[(int64_t)st.k * st.ld + j] = 0.0;
            } else if (nj > R) {
                const int p0 = poff[j], p1 = poff[j + 1];
                for (int slice = 0; slice < nslices; ++slice) {
                    const SliceGeom g = slice_geom(slice, nv);
                    if (lane < g.nvs) {
                        double acc[8];
#pragma unroll
                        for (int t = 0; t < 8; ++t) acc[t] = 0.0;
                        const double* base = part + 8 * (g.vbase + lane);
                        for (int p = p0; p < p1; ++p)
#pragma unroll
                            for (int t = 0; t < 8; ++t) acc[t] += base[(int64_t)p * st.ld + t];
                        double* dst = row + 8 * (g.vbase + lane);
#pragma unroll
                        for (int t = 0; t < 8; ++t) dst[t] = acc[t];
                    }
                }
                if (lane == 0) sp.stats[(int64_t)st.k * st.ld + j] = (double)nj;
            }
            continue;
        }
        if (nj == 0) {
            float4* row = reinterpret_cast<float4*>(st.S + (int64_t)j * st.ld);
            for (int v = lane; v < st.ld / 4; v += 32) {
                const float4 x = row[v];
                row[v] = make_float4((float)(a1 * (double)x.x), (float)(a1 * (double)x.y), (float)(a1 * (double)x.z),
                                     (float)(a1 * (double)x.w));
            }
            if (lane == 0) st.N[j] = ema_count(st.N_prev[j], 0.0, sp.alpha);
        } else if (nj <= R) {
            if (lane == 0) {
                float c = 0.0f;
                for (int s = 0; s < nslices; ++s) c += st.cnp[(int64_t)s * st.k + j];
                st.cn[j] = c;
            }
        } else {
            const int p0 = poff[j], p1 = poff[j + 1];
            const float nprev = st.N_prev[j];
            float cn_total = 0.0f;
            for (int slice = 0; slice < nslices; ++slice) {
                const SliceGeom g = slice_geom(slice, nv);
                float so[8];
                load_s(st, j, g, lane, so);
                double acc[8];
#pragma unroll
                for (int t = 0; t < 8; ++t) acc[t] = 0.0;
                if (lane < g.nvs) {
                    const double* base = part + 8 * (g.vbase + lane);
                    int p = p0;
                    for (; p + 3 < p1; p += 4) {
                        double x[4][8];
#pragma unroll
                        for (int q = 0; q < 4; ++q)
#pragma unroll
                            for (int t = 0; t < 8; ++t) x[q][t] = base[(int64_t)(p + q) * st.ld + t];
#pragma unroll
                        for (int q = 0; q < 4; ++q)
#pragma unroll
                            for (int t = 0; t < 8; ++t) acc[t] += x[q][t];
                    }
                    for (; p < p1; ++p)
#pragma unroll
                        for (int t = 0; t < 8; ++t) acc[t] += base[(int64_t)p * st.ld + t];
                }
                cn_total += ema_slice(st, j, (double)nj, nprev, slice, g, acc, so, lane, sp.alpha, sp.last_pass);
            }
            if (lane == 0) st.cn[j] = cn_total;
        }
    }
}

// Data-parallel steps, after the ranks have added their statistics: one warp per
// cluster applies the EMA from the summed (n_j, s_j), with the same arithmetic as
// the single-GPU update (a cluster without rows decays; the others go through
// ema_slice slice by slice), and thread 0 stores the summed error of the step.
__global__ void k_apply_stats(int nslices, int nv, ClusterState st, StepParams sp, double* __restrict__ err_out) {
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const double a1 = 1.0 - sp.alpha;
    const double* nsum = sp.stats + (int64_t)st.k * st.ld;
    if (blockIdx.x == 0 && threadIdx.x == 0) *err_out = nsum[st.k];
    for (int j = warp; j < st.k; j += nwarps) {
        const double nj = nsum[j];
        if (nj == 0.0) {
            float4* row = reinterpret_cast<float4*>(st.S + (int64_t)j * st.ld);
            for (int v = lane; v < st.ld / 4; v += 32) {
                const float4 x = row[v];
                row[v] = make_float4((float)(a1 * (double)x.x), (float)(a1 * (double)x.y), (float)(a1 * (double)x.z),
                                     (float)(a1 * (double)x.w));
            }
            if (lane == 0) st.N[j] = ema_count(st.N_prev[j], 0.0, sp.alpha);
            continue;
        }
        const float nprev = st.N_prev[j];
        float cn_total = 0.0f;
        for (int slice = 0; slice < nslices; ++slice) {
            const SliceGeom g = slice_geom(slice, nv);
            float so[8];
            load_s(st, j, g, lane, so);
            double acc[8];
            if (lane < g.nvs) {
                const double* src = sp.stats + (int64_t)j * st.ld + 8 * (g.vbase + lane);
#pragma unroll
                for (int t = 0; t < 8; ++t) acc[t] = src[t];
            }
            cn_total += ema_slice(st, j, nj, nprev, slice, g, acc, so, lane, sp.alpha, sp.last_pass);
        }
        if (lane == 0) st.cn[j] = cn_total;
    }
}

// ---------------------------------------------------------------- full assignment pass

// Labels and row values of a full pass (em_assign / em_mse): int64 labels, fp32
// values of the given kind (squared distances, or similarities), per-block fp64
// error sums; near ties are settled exactly as in k_labels.
__global__ void k_assign_out(const unsigned long long* __restrict__ keys, int nsplit, const float* __restrict__ xn,
                             int64_t rows, int k, const __nv_bfloat16* __restrict__ A, int ld,
                             const __nv_bfloat16* __restrict__ cq, int64_t* __restrict__ labels,
                             float* __restrict__ dists, int32_t* __restrict__ labels32, double* __restrict__ block_err,
                             int kind, ScoreScale sc, TieList tl, int* err) {
    pdl_wait();
    __shared__ double warp_err[32];
    const int lane = threadIdx.x & 31;
    double e = 0.0;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < rows; base += stride) {
        const int64_t r = base + lane;
        const bool active = r < rows;
        uint32_t l1 = 0, l2 = 0;
        float s1 = 0.0f, s2 = 0.0f, x2 = 0.0f;
        bool tie = false;
        if (active) {
            unsigned long long k1, k2;
            merge_keys(keys, rows, nsplit, r, k1, k2);
            l1 = key_label(k1);
            s1 = key_score(k1);
            x2 = xn[r];
            if (l1 >= (uint32_t)k) {
                raise_error(err, EM_E_BOUNDS);
                l1 = 0;
            }
            if (k2 != kEmptyKey) {
                l2 = key_label(k2);
                s2 = key_score(k2);
                tie = sc.tie_rel >= 0.0f && l2 < (uint32_t)k && s2 - s1 <= sc.tie_rel * (x2 + fabsf(s1) + fabsf(s2));
            }
        }
        if (tl.e)
            push_ties(tie, r, l1, l2, s2, tl, lane);
        else
            settle_ties(tie, r, l1, s1, l2, s2, A, ld, cq, kind != kSquaredDistance, lane);
        if (active) {
            if (labels) labels[r] = (int64_t)l1;
            if (labels32) labels32[r] = (int32_t)l1;
            if (dists) dists[r] = row_value(kind, x2, s1, sc);
            e += (double)row_error(kind, x2, s1, sc);
        }
    }
    e = warp_sum(e);
    if ((threadIdx.x & 31) == 0) warp_err[threadIdx.x >> 5] = e;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += warp_err[w];
        block_err[blockIdx.x] = t;
    }
}

__global__ void k_sum_blocks(const double* __restrict__ block_err, int nblocks, double* __restrict__ out,
                             TieList tl) {
    pdl_wait();
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        double t = 0.0;
        for (int b = 0; b < nblocks; ++b) t += block_err[b];
        if (tl.n) {
            t += *tl.corr;
            *tl.n = 0;
            *tl.corr = 0.0;
        }
        *out = t;
    }
}

// One warp per near-tie row: recomputes the comparison value of both candidates in
// fp64 from the bf16 row and the bf16 operands (tie_terms), keeps the smaller (the
// lower index on an exact tie), writes the label (int32 and/or int64), and for a
// relabelled row its value (of the given kind) and the change of the error sum. With
// cnt, also the row's rank in its cluster (an atomic on the count), and the last-pass
// label. The error changes are fp32 differences added in fp64; with few, small terms
// their sum does not depend on the order the atomics land in.
__global__ void k_settle(TieList tl, const float* __restrict__ xn, const __nv_bfloat16* __restrict__ A, int ld,
                         const __nv_bfloat16* __restrict__ cq, int32_t* __restrict__ labels32,
                         int64_t* __restrict__ labels64, float* __restrict__ dists, int32_t* __restrict__ cnt,
                         int32_t* __restrict__ rank, const int32_t* __restrict__ ids,
                         int64_t* __restrict__ labels_last, int capture, int kind) {
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int n = *tl.n;
    const int nv = ld / 8;
    for (int i = warp; i < n; i += nwarps) {
        const int4 t = tl.e[i];
        const int64_t r = t.x;
        const uint32_t la = (uint32_t)t.y, lb = (uint32_t)t.z;
        double da = 0.0, db = 0.0;
        const bool spherical = kind != kSquaredDistance;
        for (int v = lane; v < nv; v += 32)
            tie_terms(spherical, reinterpret_cast<const uint4*>(A + r * ld)[v],
                      reinterpret_cast<const uint4*>(cq + (int64_t)la * ld)[v],
                      reinterpret_cast<const uint4*>(cq + (int64_t)lb * ld)[v], da, db);
        da = warp_sum(da);
        db = warp_sum(db);
        if (lane == 0) {
            const bool swap = db < da || (db == da && lb < la);
            const int lab = (int)(swap ? lb : la);
            if (swap) {
                const float old = dists[r];
                const float nval = row_value(kind, xn[r], __int_as_float(t.w));
                dists[r] = nval;
                // a similarity v stands for the error 2 - 2 v
                const double scale = kind == kSimilarity ? -2.0 : 1.0;
                atomicAdd(tl.corr, scale * ((double)nval - (double)old));
            }
            if (labels32) labels32[r] = lab;
            if (labels64) labels64[r] = (int64_t)lab;
            if (cnt) rank[r] = atomicAdd(&cnt[lab], 1);
            if (capture) labels_last[ids[r]] = lab;
        }
    }
}

// Closing mean: c_j = exact mean of the rows the last pass assigned to j, for the
// clusters that received rows (faiss e-means README, "How the centroid updates work").
__global__ void k_closing_mean(ClusterState st, int k, int nv) {
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int j = warp; j < k; j += nwarps) {
        const double cntj = st.close_cnt[j];
        if (!(cntj > 0.0)) continue;
        float cn_part = 0.0f;
        for (int v = lane; v < nv; v += 32) {
            const double* cs = st.close_sum + (int64_t)j * st.ld + 8 * v;
            float cv[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) cv[t] = (float)(cs[t] / cntj);
            store_centroid_vec(st.c + (int64_t)j * st.ld, st.cq + (int64_t)j * st.ld, v, cv, cn_part);
        }
        cn_part = warp_sum(cn_part);
        if (lane == 0) st.cn[j] = cn_part;
    }
}

// Refreshes the search operand and |bf16(c)|^2 from c (after em_set_state).
__global__ void k_refresh_operand(ClusterState st, int k, int nv) {
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int j = warp; j < k; j += nwarps) {
        float cn_part = 0.0f;
        for (int v = lane; v < nv; v += 32) {
            const float4* cr = reinterpret_cast<const float4*>(st.c + (int64_t)j * st.ld) + 2 * v;
            const float4 a = cr[0], b = cr[1];
            const float cv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            store_centroid_vec(st.c + (int64_t)j * st.ld, st.cq + (int64_t)j * st.ld, v, cv, cn_part);
        }
        cn_part = warp_sum(cn_part);
        if (lane == 0) st.cn[j] = cn_part;
    }
}

// Spherical e-means (faiss e-means README, "Spherical e-means"): before it is used,
// every centroid is rescaled to norm 1; a zero centroid stays zero. One warp per
// cluster: the norm of the fp32 centroid in fp64, c <- c / |c| rounded to fp32, the
// search operand -2 bf16(c), and |c|^2 := 0 since the spherical score has no norm term.
__global__ void k_normalize(ClusterState st, int k, int nv) {
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int j = warp; j < k; j += nwarps) {
        const float4* cr = reinterpret_cast<const float4*>(st.c + (int64_t)j * st.ld);
        double ss = 0.0;
        for (int v = lane; v < nv; v += 32) {
            const float4 a = cr[2 * v], b = cr[2 * v + 1];
            ss += (double)a.x * a.x + (double)a.y * a.y + (double)a.z * a.z + (double)a.w * a.w;
            ss += (double)b.x * b.x + (double)b.y * b.y + (double)b.z * b.z + (double)b.w * b.w;
        }
        ss = warp_sum(ss);
        const double nrm = ss > 0.0 ? sqrt(ss) : 1.0;
        float cn_unused = 0.0f;
        for (int v = lane; v < nv; v += 32) {
            const float4 a = cr[2 * v], b = cr[2 * v + 1];
            const float cv[8] = {(float)(a.x / nrm), (float)(a.y / nrm), (float)(a.z / nrm), (float)(a.w / nrm),
                                 (float)(b.x / nrm), (float)(b.y / nrm), (float)(b.z / nrm), (float)(b.w / nrm)};
            store_centroid_vec(st.c + (int64_t)j * st.ld, st.cq + (int64_t)j * st.ld, v, cv, cn_unused);
        }
        if (lane == 0) st.cn[j] = 0.0f;
    }
}

}  // namespace em
