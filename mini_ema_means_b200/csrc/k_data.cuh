// k_data.cuh -- input preparation, starting centroids and the per-step batch gather.
//
// Layout: every bf16 matrix the kernels read (data, batch, centroid operand) has
// rows padded to ld = round_up(d, 8) elements (16-byte rows for TMA and for the
// 16-byte vector loads); padding columns are zero.
#pragma once

#include <cstring>

#include "common.cuh"
#include "k_fp8_codec.cuh"

namespace em {

__device__ __forceinline__ uint4 pack8_bf16(const float v[8]) {
    uint4 o;
    __nv_bfloat162 p0 = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 p1 = __floats2bfloat162_rn(v[2], v[3]);
    __nv_bfloat162 p2 = __floats2bfloat162_rn(v[4], v[5]);
    __nv_bfloat162 p3 = __floats2bfloat162_rn(v[6], v[7]);
    memcpy(&o.x, &p0, 4);
    memcpy(&o.y, &p1, 4);
    memcpy(&o.z, &p2, 4);
    memcpy(&o.w, &p3, 4);
    return o;
}

__device__ __forceinline__ void unpack8_bf16(uint4 u, float v[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// fp32 n x d (row stride d) -> bf16 n x ld, round-to-nearest-even (the search
// copy of fp32 data; faiss e-means README, "Data precision").
__global__ void k_cast_f32_bf16(const float* __restrict__ src, int64_t n, int d, int ld,
                                __nv_bfloat16* __restrict__ dst, int vec_ok) {
    pdl_wait();
    const int nv = ld / 8;
    const int64_t total = n * nv;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = e / nv;
        const int col = (int)(e - row * nv) * 8;
        const float* s = src + row * d + col;
        float v[8];
        if (vec_ok && col + 8 <= d) {
            float4 a = __ldcs(reinterpret_cast<const float4*>(s));
            float4 b = __ldcs(reinterpret_cast<const float4*>(s + 4));
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = (col + i < d) ? s[i] : 0.0f;
        }
        reinterpret_cast<uint4*>(dst + row * ld)[col / 8] = pack8_bf16(v);
    }
}

// bf16 n x d (row stride d) -> bf16 n x ld (padding copy for unaligned rows).
__global__ void k_pad_bf16(const __nv_bfloat16* __restrict__ src, int64_t n, int d, int ld,
                           __nv_bfloat16* __restrict__ dst) {
    pdl_wait();
    const int64_t total = n * ld;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = e / ld;
        const int col = (int)(e - row * ld);
        dst[e] = col < d ? src[row * d + col] : __float2bfloat16_rn(0.0f);
    }
}

// Sets *flag if any of the first `count` values is NaN or infinite.
__global__ void k_check_finite(const void* __restrict__ src, int64_t count, int is_bf16, int* flag) {
    pdl_wait();
    int bad = 0;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < count;
         e += (int64_t)gridDim.x * blockDim.x) {
        float v = is_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(src)[e])
                          : reinterpret_cast<const float*>(src)[e];
        bad |= !isfinite(v);
    }
    if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) atomicOr(flag, 1);
}

// Writes centroid j's fp32 row from fp32 values v (8 per lane-vector), refreshes its
// search operand (-2 * bf16(c), exact) and accumulates |bf16(c)|^2 into cn_part.
__device__ __forceinline__ void store_centroid_vec(float* __restrict__ c_row, __nv_bfloat16* __restrict__ cq_row,
                                                   int vec, const float v[8], float& cn_part) {
    float4* cr = reinterpret_cast<float4*>(c_row) + 2 * vec;
    cr[0] = make_float4(v[0], v[1], v[2], v[3]);
    cr[1] = make_float4(v[4], v[5], v[6], v[7]);
    float q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float b = __bfloat162float(__float2bfloat16_rn(v[i]));
        cn_part = fmaf(b, b, cn_part);
        q[i] = -2.0f * b;
    }
    reinterpret_cast<uint4*>(cq_row)[vec] = pack8_bf16(q);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// Starting centroids: k distinct training rows, the first k images of the start
// permutation (random data points, no k-means++: ic.work analysis and the faiss
// README's manual loop). N = S = 0.
__global__ void k_init_centroids(const __nv_bfloat16* __restrict__ X, int64_t n, int ld, int k, uint64_t seed,
                                 float* __restrict__ c, float* __restrict__ S, float* __restrict__ N,
                                 __nv_bfloat16* __restrict__ cq, float* __restrict__ cn, int* err) {
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const Feistel perm(n, seed, kStreamInit, 0);
    const int nv = ld / 8;
    for (int j = warp; j < k; j += nwarps) {
        int64_t row = 0;
        if (lane == 0) {
            bool ok;
            row = perm((uint64_t)j, &ok);
            if (!ok || row < 0 || row >= n) {
                raise_error(err, EM_E_BOUNDS);
                row = 0;
            }
        }
        row = __shfl_sync(0xFFFFFFFFu, row, 0);
        float cn_part = 0.0f;
        for (int v = lane; v < nv; v += 32) {
            float x[8];
            unpack8_bf16(reinterpret_cast<const uint4*>(X + row * ld)[v], x);
            store_centroid_vec(c + (int64_t)j * ld, cq + (int64_t)j * ld, v, x, cn_part);
            float4* sr = reinterpret_cast<float4*>(S + (int64_t)j * ld) + 2 * v;
            sr[0] = make_float4(0, 0, 0, 0);
            sr[1] = make_float4(0, 0, 0, 0);
        }
        cn_part = warp_sum(cn_part);
        if (lane == 0) {
            cn[j] = cn_part;
            N[j] = 0.0f;
        }
    }
}

// Batch gather: row r of the batch is data row pi_pass(base + r); copies it into the
// contiguous batch buffer, records its id and its squared norm |x|^2 (fp32, from the
// bf16 values). Each lane computes one row id; the warp then moves the 32 rows four
// at a time, with every vector of the four rows (up to 1,024 dims per round) loaded
// before the first store, so that a warp keeps up to 8 KB of reads in flight.
// With an FP8 search (Fp8Out.X8 set), the rows' E4M3 codes and |x'|^2 are written
// too (k_fp8.cuh: e4m3((x - shift) * scale), code 0 past the d real columns).
struct Fp8Out {
    uint8_t* X8;         // batch codes, pitch ld8 bytes (nullptr: bf16 search)
    float* xn8;          // |x'|^2 per batch row
    const float* shift;  // ld values
    float scale;
    int ld8, d;
};

template <bool F8>
__global__ void k_gather(const __nv_bfloat16* __restrict__ X, int64_t n, int ld, uint64_t seed, int64_t pass,
                         int64_t base, int rows, int natural_order, __nv_bfloat16* __restrict__ Xb,
                         float* __restrict__ xn, int32_t* __restrict__ ids, int* err, Fp8Out f8) {
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const Feistel perm(n, seed, kStreamPass, pass);
    const int nv = ld / 8;
    for (int r0 = warp * 32; r0 < rows; r0 += nwarps * 32) {
        const int r = r0 + lane;
        int64_t id = 0;
        if (r < rows) {
            const uint64_t pos = (uint64_t)(base + r);
            bool ok = true;
            id = natural_order ? (int64_t)pos : perm(pos, &ok);
            if (!ok || id < 0 || id >= n) {
                raise_error(err, EM_E_BOUNDS);
                id = 0;
            }
            ids[r] = (int32_t)id;
        }
        const int cnt = min(32, rows - r0);
        for (int q = 0; q < cnt; q += 4) {
            int64_t src[4];
            float acc[4], acc8[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                src[u] = __shfl_sync(0xFFFFFFFFu, id, min(q + u, cnt - 1));
                acc[u] = 0.0f;
                acc8[u] = 0.0f;
            }
            // up to 4 x 32 vectors (1,024 dims) of the four rows in flight per round
            for (int vb = 0; vb < nv; vb += 128) {
                uint4 val[4][4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int it = 0; it < 4; ++it) {
                        const int v = vb + 32 * it + lane;
                        if (v < nv) val[u][it] = reinterpret_cast<const uint4*>(X + src[u] * ld)[v];
                    }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    if (q + u < cnt) {
#pragma unroll
                        for (int it = 0; it < 4; ++it) {
                            const int v = vb + 32 * it + lane;
                            if (v < nv) {
                                reinterpret_cast<uint4*>(Xb + (int64_t)(r0 + q + u) * ld)[v] = val[u][it];
                                float x[8];
                                unpack8_bf16(val[u][it], x);
#pragma unroll
                                for (int i = 0; i < 8; ++i) acc[u] = fmaf(x[i], x[i], acc[u]);
                                if (F8) {
                                    float sh[8];
                                    const float4 s0 = reinterpret_cast<const float4*>(f8.shift)[2 * v];
                                    const float4 s1 = reinterpret_cast<const float4*>(f8.shift)[2 * v + 1];
                                    sh[0] = s0.x; sh[1] = s0.y; sh[2] = s0.z; sh[3] = s0.w;
                                    sh[4] = s1.x; sh[5] = s1.y; sh[6] = s1.z; sh[7] = s1.w;
                                    reinterpret_cast<uint2*>(f8.X8 + (int64_t)(r0 + q + u) * f8.ld8)[v] =
                                        encode8_e4m3(x, sh, f8.scale, f8.d - 8 * v, acc8[u]);
                                }
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[u] = warp_sum(acc[u]);
            if (F8) {
#pragma unroll
                for (int u = 0; u < 4; ++u) acc8[u] = warp_sum(acc8[u]);
            }
            if (lane == 0) {
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (q + u < cnt) {
                        xn[r0 + q + u] = acc[u];
                        if (F8) f8.xn8[r0 + q + u] = acc8[u];
                    }
            }
        }
    }
}

// |x|^2 of every row of X in place (no copy): the prologue of a full assignment
// pass (em_assign, em_mse, Lloyd iterations).
__global__ void k_rownorm(const __nv_bfloat16* __restrict__ X, int64_t rows, int ld, float* __restrict__ xn) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int nv = ld / 8;
    for (int64_t r = warp; r < rows; r += nwarps) {
        const uint4* s = reinterpret_cast<const uint4*>(X + r * ld);
        float acc = 0.0f;
        for (int v = lane; v < nv; v += 32) {
            float x[8];
            unpack8_bf16(s[v], x);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc = fmaf(x[i], x[i], acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) xn[r] = acc;
    }
}

}  // namespace em
