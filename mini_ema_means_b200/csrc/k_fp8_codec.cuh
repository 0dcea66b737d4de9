// k_fp8_codec.cuh -- E4M3 encoding of the FP8 search format (k_fp8.cuh says what
// the format is and which readings it takes).
#pragma once

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace em {

constexpr int kFp8CalibRows = 65536;
constexpr float kE4M3Max = 448.0f;

// E4M3 codes of (v[i] - sh[i]) * scale for 8 values; lanes past the real width
// (valid < 8) get code 0. *sq accumulates the squares of the decoded codes.
__device__ __forceinline__ uint2 encode8_e4m3(const float v[8], const float sh[8], float scale, int valid, float& sq) {
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float a = i < valid ? (v[i] - sh[i]) * scale : 0.0f;
        const __nv_fp8_storage_t code = __nv_cvt_float_to_fp8(a, __NV_SATFINITE, __NV_E4M3);
        const __half_raw hr = __nv_cvt_fp8_to_halfraw(code, __NV_E4M3);
        __half h;
        memcpy(&h, &hr, 2);
        const float dq = __half2float(h);
        sq = fmaf(dq, dq, sq);
        w[i >> 2] |= (uint32_t)code << (8 * (i & 3));  // byte i of the 8-byte group
    }
    return make_uint2(w[0], w[1]);
}

__device__ __forceinline__ void load8_f32(const float* __restrict__ p, float v[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

}  // namespace em
