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
// prefix sums in shared memory (32 children per node: one load and one ballot per
// level; a halving updates one suffix of each level with one lane-parallel
// subtraction); the uniform draws are made in parallel beforehand. The donor's
// current weight is read back as the difference of two prefix values. The vector
// work is then done in parallel from the closed form:
// the o-th split taken from donor d (0-based) sees c_d (1 + eps s)^o and N_d / 2^o.
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

// Donor tree, 32 children per node, every level stored as inclusive prefix sums
// within its groups of 32: level 0 over the current weights of the clusters (N_j,
// or 0 for a dead one), level l >= 1 over the totals of the groups of level l-1.
// A search costs one shared-memory load and one ballot per level.
struct TreeLayout {
    int levels;
    int size[6];
    int64_t offset[6];
    int64_t total;   // doubles
};

// Shared memory the selection kernel may use (bytes).
constexpr int kReviveSmemBytes = 200 * 1024;

constexpr int kMaxLevels = 6;  // 32^6 > 2^30 clusters

EM_HD TreeLayout tree_layout(int k) {
    TreeLayout L{};
    int s = k;
    int64_t off = 0;
    L.levels = 0;
    bool done = false;
#pragma unroll
    for (int l = 0; l < kMaxLevels; ++l) {
        if (!done) {
            L.size[l] = s;
            L.offset[l] = off;
            off += ((s + 31) / 32) * 32;
            L.levels = l + 1;
            done = s <= 32;
            s = (s + 31) / 32;
        }
    }
    L.total = off;
    return L;
}

// 0: every level and the split counts in shared memory; 1: level 0 and the split
// counts in global memory, upper levels shared; 2: everything in global memory.
EM_HD int tree_placement(const TreeLayout& L, int k) {
    const int64_t upper = (L.levels > 1 ? L.total - L.offset[1] : 0) * 8;
    if (L.total * 8 + (int64_t)k * 4 <= kReviveSmemBytes) return 0;
    if (L.levels > 1 && upper <= kReviveSmemBytes) return 1;
    return 2;
}

EM_HD int64_t tree_smem_bytes(const TreeLayout& L, int k) {
    const int p = tree_placement(L, k);
    if (p == 0) return L.total * 8 + (int64_t)k * 4;
    if (p == 1) return (L.total - L.offset[1]) * 8;
    return 0;
}

__device__ __forceinline__ double warp_incl_scan(double v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double t = __shfl_up_sync(0xFFFFFFFFu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

// One CTA of 1024 threads: dead set, donor tree, sequential donor draws.
__global__ void __launch_bounds__(1024) k_revive_select(const float* __restrict__ N, int k, double tau, uint64_t seed,
                                                        int64_t t, int mode, ReviveScratch sc, int* err) {
    __shared__ double red[32];
    __shared__ int32_t wcount[32];
    __shared__ int32_t base_s;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;

    // total count in a fixed order
    double part = 0.0;
    for (int j = tid; j < k; j += 1024) part += (double)N[j];
    part = warp_sum(part);
    if (lane == 0) red[w] = part;
    __syncthreads();
    if (w == 0) {
        double v = warp_sum(red[lane]);
        if (lane == 0) red[0] = v;
    }
    __syncthreads();
    const double total = red[0];
    const double mean = total / (double)k;
    const double thr = tau * mean;

    // dead set, compacted in increasing index
    if (tid == 0) base_s = 0;
    __syncthreads();
    for (int b = 0; b < k; b += 1024) {
        const int j = b + tid;
        const bool dead = j < k && (double)N[j] < thr;
        const unsigned m = __ballot_sync(0xFFFFFFFFu, dead);
        if (lane == 0) wcount[w] = __popc(m);
        __syncthreads();
        if (w == 0) {
            const int c = wcount[lane];
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
        if (tid == 1023) base_s += wcount[31] + __popc(m);
        __syncthreads();
    }
    const int nd = base_s;
    if (tid == 0) *sc.ndead = nd;
    if (mode != EM_REVIVE_SPLIT || nd == 0 || !(total > 0.0)) {
        for (int i = tid; i < nd; i += 1024) sc.donor[i] = -1;
        for (int j = tid; j < k; j += 1024) sc.times[j] = 0;
        return;
    }

    // draws of every dead cluster, in parallel (they do not depend on each other)
    for (int i = tid; i < nd; i += 1024) sc.target[i] = draw_uniform(seed, kStreamRevive, t, sc.dead[i]);

    // donor tree
    extern __shared__ double smem_d[];
    const TreeLayout L = tree_layout(k);
    const int placement = tree_placement(L, k);
    // (all loops over levels below have a fixed trip count so that levp[] and
    // L.size[] are indexed by constants and stay in registers)
    double* levp[kMaxLevels];
#pragma unroll
    for (int l = 0; l < kMaxLevels; ++l) {
        if (placement == 0)
            levp[l] = smem_d + L.offset[l];
        else if (placement == 1 && l > 0)
            levp[l] = smem_d + (L.offset[l] - L.offset[1]);
        else
            levp[l] = sc.tree + L.offset[l];
    }
    int32_t* times = placement == 0 ? reinterpret_cast<int32_t*>(smem_d + L.total) : sc.times;
    for (int j = tid; j < k; j += 1024) times[j] = 0;
#pragma unroll
    for (int l = 0; l < kMaxLevels; ++l) {
        if (l < L.levels) {
            const int sz = L.size[l];
            const int ngroups = (sz + 31) / 32;
            for (int gidx = w; gidx < ngroups; gidx += 32) {
                const int i = gidx * 32 + lane;
                double v = 0.0;
                if (i < sz) {
                    if (l == 0) {
                        const float nj = N[i];
                        v = ((double)nj < thr) ? 0.0 : (double)nj;
                    } else {
                        v = levp[l > 0 ? l - 1 : 0][i * 32 + 31];  // prefix at the end of child group i
                    }
                }
                levp[l][gidx * 32 + lane] = warp_incl_scan(v, lane);
            }
        }
        __syncthreads();
    }

    // sequential draws by warp 0
    if (w == 0) {
        const int top = L.levels - 1;
        double W = 0.0;
#pragma unroll
        for (int l = 0; l < kMaxLevels; ++l)
            if (l == top) W = levp[l][31];
        bool exhausted = false;
        for (int i0 = 0; i0 < nd; i0 += 32) {
            const int cnt = min(32, nd - i0);
            const double my_u = lane < cnt ? sc.target[i0 + lane] : 0.0;
            for (int q = 0; q < cnt; ++q) {
                const int i = i0 + q;
                if (exhausted || !(W > 0.0)) {
                    exhausted = true;
                    if (lane == 0) sc.donor[i] = -1;
                    continue;
                }
                double target = __shfl_sync(0xFFFFFFFFu, my_u, q) * W;
                int node = 0;
                double wsel = 0.0;  // current weight of the chosen child at the last level
#pragma unroll
                for (int l = kMaxLevels - 1; l >= 0; --l) {
                    if (l <= top) {
                        const int base = node * 32;
                        const double* lev = levp[l];
                        const bool valid = base + lane < L.size[l];
                        const double P = valid ? lev[base + lane] : 0.0;
                        const unsigned above = __ballot_sync(0xFFFFFFFFu, valid && P > target);
                        int c;
                        if (above) {
                            c = __ffs(above) - 1;
                        } else {  // target rounded onto the total: the last child with weight
                            const double Pp = __shfl_up_sync(0xFFFFFFFFu, P, 1);
                            const unsigned pos = __ballot_sync(0xFFFFFFFFu, valid && P > (lane ? Pp : 0.0));
                            c = pos ? 31 - __clz(pos) : 0;
                        }
                        const double before = c > 0 ? lev[base + c - 1] : 0.0;  // broadcast load
                        if (l == 0) wsel = lev[base + c] - before;
                        target -= before;
                        node = base + c;
                    }
                }
                const int dn = node;
                const double delta = 0.5 * wsel;  // half of the donor's current weight
                if (lane == 0) {
                    const int old = times[dn];
                    times[dn] = old + 1;
                    sc.donor[i] = dn;
                    sc.order[i] = old;
                }
                int idx = dn;
#pragma unroll
                for (int l = 0; l < kMaxLevels; ++l) {
                    if (l < L.levels) {
                        const int gb = (idx >> 5) << 5;
                        if (gb + lane >= idx && gb + lane < L.size[l]) levp[l][gb + lane] -= delta;
                        idx >>= 5;
                    }
                }
                W -= delta;
                __syncwarp();
            }
        }
        if (lane == 0) {
            int done = 0;
            for (int i = 0; i < nd; ++i) done += sc.donor[i] >= 0;
            *sc.n_splits += done;
        }
    }
    __syncthreads();
    if (placement == 0)
        for (int j = tid; j < k; j += 1024) sc.times[j] = times[j];
}

// Dead clusters take their half of the donor (reads the donors' state before
// k_revive_donors changes it).
__global__ void k_revive_dead(ClusterState st, int nv, ReviveScratch sc) {
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
