// common.cuh -- helpers shared by the e-means kernels and the host orchestration.
//
// Random draws of the method (starting rows, the per-pass order, revival donors
// and resampled rows) use the counter-based generator Philox4x64-10 (Salmon,
// Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC'11).
// The per-pass order is a keyed 4-round Feistel bijection with cycle walking
// (Black & Rogaway, "Ciphers with arbitrary finite domains", CT-RSA 2002), so a
// batch's row ids are computed where they are needed instead of being stored.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/emeans.h"

#define EM_HD __host__ __device__ __forceinline__

namespace em {

// Programmatic dependent launch: every kernel of the library starts by waiting for
// the grids it depends on (a no-op unless it was launched with programmatic stream
// serialization), so that the host may let a kernel launch while its predecessor on
// the stream is still finishing; pdl_release lets the next kernel launch early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// ---------------------------------------------------------------- generator

constexpr uint64_t kPhiloxM0 = 0xD2E7470EE14C6C93ull;
constexpr uint64_t kPhiloxM1 = 0xCA5A826395121157ull;
constexpr uint64_t kPhiloxW0 = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kPhiloxW1 = 0xBB67AE8584CAA73Bull;

// Purposes of the draws (second key word).
constexpr int kStreamInit = 1;
constexpr int kStreamPass = 2;
constexpr int kStreamRevive = 3;
constexpr int kStreamResample = 4;

EM_HD void mulhilo64(uint64_t a, uint64_t b, uint64_t& hi, uint64_t& lo) {
#ifdef __CUDA_ARCH__
    lo = a * b;
    hi = __umul64hi(a, b);
#else
    unsigned __int128 p = (unsigned __int128)a * b;
    lo = (uint64_t)p;
    hi = (uint64_t)(p >> 64);
#endif
}

// Philox4x64 with 10 rounds; c is the 256-bit counter, (k0, k1) the key.
EM_HD void philox4x64_10(uint64_t c[4], uint64_t k0, uint64_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        uint64_t hi0, lo0, hi1, lo1;
        mulhilo64(kPhiloxM0, c[0], hi0, lo0);
        mulhilo64(kPhiloxM1, c[2], hi1, lo1);
        uint64_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
        c[0] = n0;
        c[1] = lo1;
        c[2] = n2;
        c[3] = lo0;
        k0 += kPhiloxW0;
        k1 += kPhiloxW1;
    }
}

// First output word at counter (a, b, 0, 0) under key (seed, stream).
EM_HD uint64_t philox_word(uint64_t seed, uint64_t stream, uint64_t a, uint64_t b, uint64_t c2 = 0) {
    uint64_t c[4] = {a, b, c2, 0};
    philox4x64_10(c, seed, stream);
    return c[0];
}

// Top 53 bits as a double in [0, 1).
EM_HD double to_unit(uint64_t bits) { return (double)(bits >> 11) * (1.0 / 9007199254740992.0); }

// u(seed, stream, t, j): the draw a revival at step t makes for cluster j.
EM_HD double draw_uniform(uint64_t seed, int stream, int64_t t, int64_t j) {
    return to_unit(philox_word(seed, (uint64_t)stream, (uint64_t)t, (uint64_t)j));
}

// ---------------------------------------------------------------- per-pass order

EM_HD int feistel_half_bits(int64_t n) {
    int bits = 1;
    if (n > 1) {
        uint64_t v = (uint64_t)(n - 1);
        bits = 0;
        while (v) {
            ++bits;
            v >>= 1;
        }
    }
    int h = (bits + 1) / 2;
    return h < 1 ? 1 : h;
}

struct Feistel {
    uint64_t n, mask, seed, stream, which;
    int h;
    EM_HD Feistel(int64_t n_, uint64_t seed_, int stream_, int64_t which_)
        : n((uint64_t)n_), seed(seed_), stream((uint64_t)stream_), which((uint64_t)which_) {
        h = feistel_half_bits(n_);
        mask = (1ull << h) - 1ull;
    }
    EM_HD uint64_t encrypt(uint64_t v) const {
        uint64_t left = v >> h, right = v & mask;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            uint64_t f = philox_word(seed, stream, right, (uint64_t)r, which) & mask;
            uint64_t nl = right;
            right = left ^ f;
            left = nl;
        }
        return (left << h) | right;
    }
    // pi(i) for i in [0, n). Cycle walking ends because encrypt is a bijection on
    // [0, 2^(2h)) and i's own cycle returns to [0, n); the bound only guards the
    // loop (the expected walk is below 4 steps since 2^(2h) < 4n).
    EM_HD int64_t operator()(uint64_t i, bool* ok = nullptr) const {
        uint64_t v = encrypt(i);
        uint32_t guard = 0;
        while (v >= n && guard < (1u << 24)) {
            v = encrypt(v);
            ++guard;
        }
        if (ok) *ok = v < n;
        return (int64_t)v;
    }
};

// ---------------------------------------------------------------- search keys

// Order-preserving map fp32 -> uint32 (for non-NaN values): a smaller float gives
// a smaller unsigned integer, so (score, index) packs into one 64-bit key whose
// unsigned minimum is the smallest score with the lowest index.
EM_HD uint32_t f32_order(float f) {
#ifdef __CUDA_ARCH__
    uint32_t u = __float_as_uint(f);
#else
    uint32_t u;
    memcpy(&u, &f, 4);
#endif
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

EM_HD float f32_unorder(uint32_t o) {
    uint32_t u = (o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o;
#ifdef __CUDA_ARCH__
    return __uint_as_float(u);
#else
    float f;
    memcpy(&f, &u, 4);
    return f;
#endif
}

EM_HD uint64_t pack_key(float score, uint32_t j) { return ((uint64_t)f32_order(score) << 32) | j; }
EM_HD uint32_t key_label(uint64_t key) { return (uint32_t)(key & 0xFFFFFFFFull); }
EM_HD float key_score(uint64_t key) { return f32_unorder((uint32_t)(key >> 32)); }

constexpr uint64_t kEmptyKey = ~0ull;

// ---------------------------------------------------------------- device errors

// First error wins; the host reads and clears the word at synchronisation points.
__device__ __forceinline__ void raise_error(int* err, int code) { atomicCAS(err, 0, code); }

__device__ __forceinline__ bool error_raised(const int* err) {
    return *(volatile const int*)err != 0;
}

// Split constants of the revival (size-proportional split of a donor cluster).
constexpr float kSplitEps = 1.0f / 1024.0f;
constexpr int kReviveEvery = 5;

}  // namespace em
