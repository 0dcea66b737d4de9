// k_fp8.cuh -- the FP8 (E4M3) search format.
//
// faiss e-means README, "Data precision": the nearest-centroid search may run in
// FP8 (E4M3). A converter calibrated on a sample holds a shift per dimension and
// one power-of-two scale; a value v is searched as e4m3((v - shift) * scale), and
// values beyond the sample's range clamp to the edge, 448. Only the search uses
// the format: the running counts, sums and centroids stay fp32 (the sums are those
// of the bf16 rows, as in the bf16 search), and distances come back in the data's
// units. Readings fixed here:
//   * calibration sample: the first 65,536 rows of the bf16 copy; shift = the
//     midrange (min + max) / 2 of each dimension in fp32; scale = the largest
//     power of two with max |v - shift| * scale <= 448 (1 for a constant sample);
//   * v - shift is computed in fp32, the scaling is exact, then one round-to-
//     nearest-even to E4M3 with saturation (CUDA's conversion with __NV_SATFINITE);
//   * the search operand of a centroid is the NEGATED code -c' with |c'|^2 / 2
//     beside it, so that the tensor cores produce |c'|^2 / 2 - x'.c', half the
//     squared distance in code units less |x'|^2 / 2 (-2 c' could leave the
//     format's range); the distance is (|x'|^2 + 2 score) / scale^2.
#pragma once

#include "k_data.cuh"

namespace em {

// Calibration, pass 1: per-dimension min and max of rows [0, rows) of X, one
// partial per (row block, dimension): part_lo / part_hi[blockIdx.y * d + j].
__global__ void k_fp8_minmax(const __nv_bfloat16* __restrict__ X, int64_t rows, int d, int ld,
                             float* __restrict__ part_lo, float* __restrict__ part_hi) {
    pdl_wait();
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= d) return;
    float lo = INFINITY, hi = -INFINITY;
    for (int64_t r = blockIdx.y; r < rows; r += gridDim.y) {
        const float v = __bfloat162float(X[r * ld + j]);
        lo = fminf(lo, v);
        hi = fmaxf(hi, v);
    }
    part_lo[(int64_t)blockIdx.y * d + j] = lo;
    part_hi[(int64_t)blockIdx.y * d + j] = hi;
}

// Calibration, pass 2: the minimum and maximum over the row blocks.
__global__ void k_fp8_minmax_reduce(const float* __restrict__ part_lo, const float* __restrict__ part_hi, int nparts,
                                    int d, float* __restrict__ lo, float* __restrict__ hi) {
    pdl_wait();
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= d) return;
    float a = INFINITY, b = -INFINITY;
    for (int p = 0; p < nparts; ++p) {
        a = fminf(a, part_lo[(int64_t)p * d + j]);
        b = fmaxf(b, part_hi[(int64_t)p * d + j]);
    }
    lo[j] = a;
    hi[j] = b;
}

// FP8 codes of whole rows (a full assignment pass): row r of X (bf16, pitch ld)
// -> X8 row r (pitch ld8 bytes) and xn8[r] = |x'|^2. One warp per row.
__global__ void k_fp8_rows(const __nv_bfloat16* __restrict__ X, int64_t rows, int d, int ld,
                           const float* __restrict__ shift, float scale, uint8_t* __restrict__ X8, int ld8,
                           float* __restrict__ xn8) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int nv = ld / 8;
    for (int64_t r = warp; r < rows; r += nwarps) {
        float sq = 0.0f;
        for (int v = lane; v < nv; v += 32) {
            float x[8], sh[8];
            unpack8_bf16(reinterpret_cast<const uint4*>(X + r * ld)[v], x);
            load8_f32(shift + 8 * v, sh);
            reinterpret_cast<uint2*>(X8 + r * ld8)[v] = encode8_e4m3(x, sh, scale, d - 8 * v, sq);
        }
        sq = warp_sum(sq);
        if (lane == 0) xn8[r] = sq;
    }
}

// The FP8 search operand of every centroid: -e4m3((c - shift) * scale) and
// |c'|^2 / 2. One warp per cluster.
__global__ void k_fp8_operand(const float* __restrict__ c, int k, int d, int ld, const float* __restrict__ shift,
                              float scale, uint8_t* __restrict__ cq8, int ld8, float* __restrict__ cn8) {
    pdl_wait();
    pdl_release();
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int nv = ld / 8;
    for (int j = warp; j < k; j += nwarps) {
        float sq = 0.0f;
        for (int v = lane; v < nv; v += 32) {
            float x[8], sh[8];
            load8_f32(c + (int64_t)j * ld + 8 * v, x);
            load8_f32(shift + 8 * v, sh);
            uint2 code = encode8_e4m3(x, sh, scale, d - 8 * v, sq);
            code.x ^= 0x80808080u;  // negation flips the sign bits
            code.y ^= 0x80808080u;
            reinterpret_cast<uint2*>(cq8 + (int64_t)j * ld8)[v] = code;
        }
        sq = warp_sum(sq);
        if (lane == 0) cn8[j] = 0.5f * sq;
    }
}

}  // namespace em
