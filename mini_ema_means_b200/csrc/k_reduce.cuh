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
//   k_offsets  exclusive scan of the counts (segment starts), batch error sum;
//   k_scatter  writes row ids into label order (perm) with their labels (slab);
//   k_segsum   walks perm in fixed-size tiles (one warp per tile, so a cluster
//              with many rows is spread over many warps): a run of equal labels
//              that lies inside one tile is summed (fp64) and updated at once;
//              a run cut by a tile edge leaves its partial sum in a per-tile slot;
//   k_fixup    adds the partial sums of every cut cluster in tile order and
//              updates it, and decays clusters that received no row.
// Sums are accumulated in fp64 from bf16 values, which makes them independent of
// the order rows arrive in (the fp64 sum of bf16 values is exact for the data
// ranges used here), so the update is deterministic.
#pragma once

#include "k_data.cuh"

namespace em {

constexpr int kMaxVpl = 8;  // 16-byte vectors per lane in one slice: 32 lanes x 8 x 8 = 2048 dims

struct StepParams {
    double alpha;        // step size of this step
    int last_pass;       // accumulate the closing-mean statistics
    int capture_labels;  // record the last-pass label of each row
};

// ---------------------------------------------------------------- labels + histogram

__global__ void k_labels(const unsigned long long* __restrict__ keys, const float* __restrict__ xn, int rows, int k,
                         const int32_t* __restrict__ ids, int32_t* __restrict__ labels, float* __restrict__ dists,
                         int32_t* __restrict__ cnt, int32_t* __restrict__ rank, double* __restrict__ block_err,
                         int64_t* __restrict__ labels_last, int capture, int* err) {
    __shared__ double warp_err[32];
    const int lane = threadIdx.x & 31;
    double e = 0.0;
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    const bool active = r < rows;
    int lab = -1;
    if (active) {
        const unsigned long long key = keys[r];
        uint32_t l = key_label(key);
        if (l >= (uint32_t)k) {  // a row that was never searched, or a corrupted key
            raise_error(err, EM_E_BOUNDS);
            l = 0;
        }
        lab = (int)l;
        const float dist = fmaxf(0.0f, xn[r] + key_score(key));
        labels[r] = lab;
        dists[r] = dist;
        e = (double)dist;
        if (capture) labels_last[ids[r]] = lab;
    }
    const unsigned amask = __ballot_sync(0xFFFFFFFFu, active);
    if (active) {
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

// Exclusive scan of cnt[0..k) into off[0..k]; one CTA of 1024 threads in tiles of
// 4096 counts. Also adds the per-block error sums in block order.
__global__ void __launch_bounds__(1024) k_offsets(const int32_t* __restrict__ cnt, int k, int rows,
                                                  int32_t* __restrict__ off, const double* __restrict__ block_err,
                                                  int nblocks, double* __restrict__ err_sum_out, int* err) {
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t carry_s;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    if (tid == 0) carry_s = 0;
    __syncthreads();
    for (int base = 0; base < k; base += 4096) {
        int v[4];
        const int i0 = base + tid * 4;
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = (i0 + i < k) ? cnt[i0 + i] : 0;
        const int local = v[0] + v[1] + v[2] + v[3];
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += t;
        }
        if (lane == 31) warp_tot[w] = incl;
        __syncthreads();
        if (w == 0) {
            int x = warp_tot[lane];
            int xi = x;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xFFFFFFFFu, xi, o);
                if (lane >= o) xi += t;
            }
            warp_tot[lane] = xi - x;  // exclusive prefix of warp totals
        }
        __syncthreads();
        const int carry = carry_s;
        int run = carry + warp_tot[w] + incl - local;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (i0 + i < k) off[i0 + i] = run;
            run += v[i];
        }
        __syncthreads();
        if (tid == 1023) carry_s = run;
        __syncthreads();
    }
    if (tid == 0) {
        off[k] = carry_s;
        if (carry_s != rows) raise_error(err, EM_E_BOUNDS);
        double t = 0.0;
        for (int b = 0; b < nblocks; ++b) t += block_err[b];
        *err_sum_out = t;
    }
}

__global__ void k_scatter(const int32_t* __restrict__ labels, const int32_t* __restrict__ rank,
                          const int32_t* __restrict__ off, int rows, int32_t* __restrict__ perm,
                          int32_t* __restrict__ slab, int* err) {
    const int r = blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    const int lab = labels[r];
    const int pos = off[lab] + rank[r];
    if (pos < 0 || pos >= rows) {
        raise_error(err, EM_E_BOUNDS);
        return;
    }
    perm[pos] = r;
    slab[pos] = lab;
}

// ---------------------------------------------------------------- EMA of one cluster

// Sums of one slice of dimensions, held by one warp: lane owns vectors
// v = slice_base + i * 32 + lane (i < VPL) of 8 dims each.
template <int VPL>
struct SliceAcc {
    double a[VPL][8];
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < VPL; ++i)
#pragma unroll
            for (int t = 0; t < 8; ++t) a[i][t] = 0.0;
    }
};

template <int VPL>
__device__ __forceinline__ void acc_rows(SliceAcc<VPL>& acc, const __nv_bfloat16* __restrict__ src, int ld,
                                         const int32_t* __restrict__ perm, int s0, int s1, int vbase, int nv,
                                         int lane) {
    int s = s0;
    for (; s + 1 < s1; s += 2) {  // two rows in flight
        const int64_t r0 = perm[s], r1 = perm[s + 1];
        const uint4* p0 = reinterpret_cast<const uint4*>(src + r0 * ld);
        const uint4* p1 = reinterpret_cast<const uint4*>(src + r1 * ld);
        uint4 u0[VPL], u1[VPL];
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int v = vbase + i * 32 + lane;
            if (v < nv) {
                u0[i] = p0[v];
                u1[i] = p1[v];
            }
        }
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int v = vbase + i * 32 + lane;
            if (v < nv) {
                float x0[8], x1[8];
                unpack8_bf16(u0[i], x0);
                unpack8_bf16(u1[i], x1);
#pragma unroll
                for (int t = 0; t < 8; ++t) acc.a[i][t] += (double)x0[t] + (double)x1[t];
            }
        }
    }
    if (s < s1) {
        const int64_t r0 = perm[s];
        const uint4* p0 = reinterpret_cast<const uint4*>(src + r0 * ld);
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            const int v = vbase + i * 32 + lane;
            if (v < nv) {
                float x0[8];
                unpack8_bf16(p0[v], x0);
#pragma unroll
                for (int t = 0; t < 8; ++t) acc.a[i][t] += (double)x0[t];
            }
        }
    }
}

struct ClusterState {
    float* N;
    float* S;
    float* c;
    __nv_bfloat16* cq;
    float* cn;
    double* close_sum;
    double* close_cnt;
    int ld;
};

// EMA update of one slice of cluster j with batch count nj and slice sums acc.
// Returns this lane's part of |bf16(c_j)|^2 over the slice.
template <int VPL>
__device__ __forceinline__ float ema_slice(const ClusterState& st, int j, double nj, double Nnew_d, float Nnew,
                                           const SliceAcc<VPL>& acc, int vbase, int nv, int lane, double alpha,
                                           int last_pass) {
    const double a1 = 1.0 - alpha;
    float cn_part = 0.0f;
    float* Srow = st.S + (int64_t)j * st.ld;
    float* crow = st.c + (int64_t)j * st.ld;
    __nv_bfloat16* qrow = st.cq + (int64_t)j * st.ld;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int v = vbase + i * 32 + lane;
        if (v < nv) {
            float4* sp = reinterpret_cast<float4*>(Srow) + 2 * v;
            const float4 s0 = sp[0], s1 = sp[1];
            const float so[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
            float sn[8], cv[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                sn[t] = (float)(a1 * (double)so[t] + alpha * acc.a[i][t]);
                cv[t] = Nnew > 0.0f ? (float)((double)sn[t] / (double)Nnew) : 0.0f;
            }
            sp[0] = make_float4(sn[0], sn[1], sn[2], sn[3]);
            sp[1] = make_float4(sn[4], sn[5], sn[6], sn[7]);
            if (Nnew > 0.0f) store_centroid_vec(crow, qrow, v, cv, cn_part);
            if (last_pass) {
                double* cs = st.close_sum + (int64_t)j * st.ld + 8 * v;
#pragma unroll
                for (int t = 0; t < 8; ++t) cs[t] += acc.a[i][t];
            }
        }
    }
    (void)nj;
    (void)Nnew_d;
    return cn_part;
}

// Full EMA of cluster j (all slices) from sums that are already complete in acc
// (single-slice case) -- used by k_segsum for runs inside one tile.
template <int VPL>
__device__ __forceinline__ void ema_cluster_begin(const ClusterState& st, int j, double nj, double alpha,
                                                  float& Nnew, double& Nnew_d) {
    const float Nold = st.N[j];
    Nnew_d = (1.0 - alpha) * (double)Nold + alpha * nj;
    Nnew = (float)Nnew_d;
}

template <int VPL>
__device__ __forceinline__ void ema_cluster_end(const ClusterState& st, int j, double nj, float Nnew, float cn_part,
                                                int lane, int last_pass) {
    cn_part = warp_sum(cn_part);
    if (lane == 0) {
        st.N[j] = Nnew;
        if (Nnew > 0.0f) st.cn[j] = cn_part;
        if (last_pass) st.close_cnt[j] += nj;
    }
}

// ---------------------------------------------------------------- segmented sum

template <int VPL>
__global__ void k_segsum(const __nv_bfloat16* __restrict__ src, const int32_t* __restrict__ perm,
                         const int32_t* __restrict__ slab, const int32_t* __restrict__ off, int rows, int R,
                         int nv, ClusterState st, StepParams sp, double* __restrict__ pfirst,
                         double* __restrict__ plast) {
    const int lane = threadIdx.x & 31;
    const int tile = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int t0 = tile * R;
    if (t0 >= rows) return;
    const int t1 = min(t0 + R, rows);
    const int slice_v = 32 * VPL;
    int slot = t0;
    while (slot < t1) {
        const int j = slab[slot];
        const int js = off[j], je = off[j + 1];
        const int e = min(je, t1);
        const bool complete = js >= t0 && je <= t1;
        const double nj = (double)(je - js);
        float Nnew = 0.0f;
        double Nnew_d = 0.0;
        if (complete) ema_cluster_begin<VPL>(st, j, nj, sp.alpha, Nnew, Nnew_d);
        float cn_part = 0.0f;
        for (int vb = 0; vb < nv; vb += slice_v) {
            SliceAcc<VPL> acc;
            acc.zero();
            acc_rows<VPL>(acc, src, st.ld, perm, slot, e, vb, nv, lane);
            if (complete) {
                cn_part += ema_slice<VPL>(st, j, nj, Nnew_d, Nnew, acc, vb, nv, lane, sp.alpha, sp.last_pass);
            } else {
                double* dst = (js < t0 ? pfirst : plast) + (int64_t)tile * (nv * 8);
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    const int v = vb + i * 32 + lane;
                    if (v < nv) {
#pragma unroll
                        for (int t = 0; t < 8; ++t) dst[8 * v + t] = acc.a[i][t];
                    }
                }
            }
        }
        if (complete) ema_cluster_end<VPL>(st, j, nj, Nnew, cn_part, lane, sp.last_pass);
        slot = e;
    }
}

// Clusters cut by tile edges (owned by the tile where their run starts) and
// clusters that received no row. Also clears the counts for the next step.
template <int VPL>
__global__ void k_fixup(const int32_t* __restrict__ slab, const int32_t* __restrict__ off, int32_t* __restrict__ cnt,
                        int rows, int R, int ntiles, int k, int nv, ClusterState st, StepParams sp,
                        const double* __restrict__ pfirst, const double* __restrict__ plast) {
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int slice_v = 32 * VPL;
    for (int tile = warp; tile < ntiles; tile += nwarps) {
        const int t0 = tile * R, t1 = min(t0 + R, rows);
        if (t1 <= t0) continue;
        const int j = slab[t1 - 1];
        const int js = off[j], je = off[j + 1];
        if (!(js >= t0 && je > t1)) continue;
        const int last_tile = (je - 1) / R;
        const double nj = (double)(je - js);
        float Nnew;
        double Nnew_d;
        ema_cluster_begin<VPL>(st, j, nj, sp.alpha, Nnew, Nnew_d);
        float cn_part = 0.0f;
        for (int vb = 0; vb < nv; vb += slice_v) {
            SliceAcc<VPL> acc;
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int v = vb + i * 32 + lane;
#pragma unroll
                for (int t = 0; t < 8; ++t) acc.a[i][t] = v < nv ? plast[(int64_t)tile * (nv * 8) + 8 * v + t] : 0.0;
            }
            for (int u = tile + 1; u <= last_tile; ++u) {
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    const int v = vb + i * 32 + lane;
                    if (v < nv) {
#pragma unroll
                        for (int t = 0; t < 8; ++t) acc.a[i][t] += pfirst[(int64_t)u * (nv * 8) + 8 * v + t];
                    }
                }
            }
            cn_part += ema_slice<VPL>(st, j, nj, Nnew_d, Nnew, acc, vb, nv, lane, sp.alpha, sp.last_pass);
        }
        ema_cluster_end<VPL>(st, j, nj, Nnew, cn_part, lane, sp.last_pass);
    }
    // clusters without rows: N and S decay, the centroid S/N is unchanged
    const float a1 = (float)(1.0 - sp.alpha);
    for (int j = warp; j < k; j += nwarps) {
        const bool empty = off[j + 1] == off[j];
        if (lane == 0) cnt[j] = 0;
        if (!empty) continue;
        float* Srow = st.S + (int64_t)j * st.ld;
        for (int e = lane; e < nv * 8; e += 32) Srow[e] = (float)((double)a1 * 0.0 + (1.0 - sp.alpha) * (double)Srow[e]);
        if (lane == 0) st.N[j] = (float)((1.0 - sp.alpha) * (double)st.N[j]);
    }
}

// ---------------------------------------------------------------- full assignment pass

// Labels and distances of a full pass (em_assign / em_mse / Lloyd): int64 labels,
// fp32 squared distances max(0, |x|^2 + score), per-block fp64 sums.
__global__ void k_assign_out(const unsigned long long* __restrict__ keys, const float* __restrict__ xn, int64_t rows,
                             int k, int64_t* __restrict__ labels, float* __restrict__ dists,
                             int32_t* __restrict__ labels32, double* __restrict__ block_err, int* err) {
    __shared__ double warp_err[32];
    double e = 0.0;
    for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < rows; r += (int64_t)gridDim.x * blockDim.x) {
        const unsigned long long key = keys[r];
        uint32_t l = key_label(key);
        if (l >= (uint32_t)k) {
            raise_error(err, EM_E_BOUNDS);
            l = 0;
        }
        const float dist = fmaxf(0.0f, xn[r] + key_score(key));
        if (labels) labels[r] = (int64_t)l;
        if (labels32) labels32[r] = (int32_t)l;
        if (dists) dists[r] = dist;
        e += (double)dist;
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

__global__ void k_sum_blocks(const double* __restrict__ block_err, int nblocks, double* __restrict__ out) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        double t = 0.0;
        for (int b = 0; b < nblocks; ++b) t += block_err[b];
        *out = t;
    }
}

// Closing mean: c_j = exact mean of the rows the last pass assigned to j, for the
// clusters that received rows (faiss e-means README, "How the centroid updates work").
__global__ void k_closing_mean(ClusterState st, int k, int nv) {
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

}  // namespace em
