// k_assign.cuh -- fused nearest-centroid search on the sm_100a tensor cores.
//
// For each row x of A (bf16) and each centroid operand q_j = -2 bf16(c_j):
//     score_ij = |bf16(c_j)|^2 + x_i . q_j   (= |x - c_j|^2 - |x|^2)
// and the row keeps the smallest score with the lowest j (faiss e-means README,
// "Kernels": the distance computation is fused with the selection of the nearest
// centroid, so no n x k distance matrix is ever written).
//
// Structure of one CTA (320 threads, one CTA per SM, persistent over work units):
//   warp 0      TMA producer: 128 x KC tiles of A and 256 x KC tiles of the
//               centroid operand into a STAGES-deep shared-memory ring (with the
//               batch tile stationary, a stage holds a whole 256-row centroid tile,
//               so that a tile costs one barrier round trip, not one per K chunk)
//   warp 1      allocates 512 TMEM columns; one thread issues tcgen05.mma
//               (M=128, N=256, K=16, bf16 x bf16 -> fp32) into one of two
//               TMEM accumulators and commits to mbarriers
//   warps 2..9  epilogue: thread = accumulator row; warps w and w + 4 share the
//               TMEM lane quadrant w % 4 and take the left and right 128 columns
//               of the tile: tcgen05.ld of 32 columns at a time (the next load in
//               flight while a chunk is scanned), free the accumulator after the
//               last, add |c|^2, running argmin. The eight warps never wait for each
//               other: each stages its own |c|^2 values and writes its own keys
//               (one key set per column half), and the label kernel merges the key
//               sets
// A work unit is (128-row tile, group of 256-wide centroid tiles). Every group
// writes its own per-row results ((order-preserving score, index) keys), two key
// sets per group, and the label kernel merges them. The host either splits every
// row tile into the same number of groups or, when the row tiles fill whole waves
// of CTAs before a partial one, keeps those whole (one group each, emptying the
// other groups' key sets) and splits only the last wave's row tiles. With
// TOP2 the epilogue also keeps the second best candidate, so that near ties can be
// settled exactly afterwards.
#pragma once

#include "common.cuh"

namespace em {
namespace tc {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kThreads = 64 + kEpiThreads;

// Epilogue groups. With the batch tile stationary and a plain argmin (rows of at
// most 128 dims) a tile holds little tensor work (six K = 16 MMAs at d = 96), and
// one group of eight warps scanning every tile would keep the tensor pipe waiting.
// There two groups take the two accumulators in turn, so that each has the time of
// two tiles for the epilogue of one; at the end of a unit the second group hands
// its rows' best to the first through shared memory, and the first writes the keys.
template <bool TOP2, bool AST>
__host__ __device__ constexpr int epi_groups() { return (AST && !TOP2) ? 2 : 1; }
template <int G>
__host__ __device__ constexpr int threads_for() { return 64 + kEpiThreads * G; }
constexpr int kKeySets = kEpiWarps / 4;  // key sets per centroid-tile group (the two column halves)
constexpr int kEpiCols = BN / kKeySets;  // columns of a tile per epilogue warp
static_assert(kEpiCols % 64 == 0, "the epilogue scans pairs of 32-column chunks");

// AST ("A stationary", rows of at most 128 dims): the CTA keeps its 128-row tile of
// the batch in shared memory for the whole work unit (two buffers, so that the
// next unit's tile loads while this one is used) and streams only centroid tiles
// through the ring: a third less traffic from L2 per tile.
constexpr int kAstBufBytes = 32 * 1024;  // one A-stationary buffer: nkc * BM * KC * 2 bytes at most

// FOLD (with the batch tile stationary and a plain argmin): |c~|^2 enters the MMAs
// as one more K = 16 step, ones(128 x 16) x norms(256 x 16), where each centroid's
// row of the norms operand is (h, m, l, 0, ...) with h + m + l = |c~|^2 exactly (the
// fp32 value split into three bf16 parts) and each batch row's is (1, 1, 1, 0, ...).
// The accumulator then holds the score itself, and the epilogue adds nothing. Both
// extension tiles are 16 wide (32-byte rows, the 32-byte swizzle).
constexpr int kExtK = 16;
constexpr int kExtABytes = BM * kExtK * 2;  // the ones tile, loaded once per CTA
constexpr int kExtBBytes = BN * kExtK * 2;  // a centroid tile's norms, with its chunks
constexpr uint64_t kExtLayout = 6ull;       // UMMA 32B swizzle
constexpr uint32_t kExtSBO = 8u * kExtK * 2u;

template <int KC, bool AST = false, int G = 1, bool FOLD = false>
struct Cfg {
    static constexpr int kABytes = BM * KC * 2;
    static constexpr int kBBytes = BN * KC * 2;
    static constexpr int kStageBytes = AST ? kBBytes : kABytes + kBBytes;
    // (A stationary: 9 stages of 16 KB or 4 of 32 KB fit beside the two A buffers)
    static constexpr int kStages = AST ? (KC == 32 ? 9 : 4) : (KC == 64 ? 4 : 8);
    static constexpr int kAreaBytes = AST ? 2 * kAstBufBytes + (FOLD ? kExtABytes : 0) : 0;  // A buffers
    static constexpr uint64_t kLayout = KC == 64 ? 2ull : 4ull;  // UMMA 128B / 64B swizzle
    static constexpr uint32_t kSBO = 8u * KC * 2u;                // bytes between 8-row groups
    static constexpr int kBarBytes = 256;
    // two groups: per warp pair and unit parity 32 (best, index) pairs, and a full
    // and an empty barrier
    static constexpr int kMergeBytes = G == 2 ? 8 * 2 * 32 * 8 + 8 * 2 * 2 * 8 : 0;
    // + the epilogue warps' |c|^2 values: two tiles of 128 columns per warp (one
    // group) or one (two groups), then the merge area
    static constexpr int kSmemBytes =
        1024 + kStages * kStageBytes + kAreaBytes + kBarBytes + kEpiWarps * 2 * kEpiCols * 4 + kMergeBytes;
};

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulate (bits 4-5 = 1),
// A and B bf16 (bits 7-9 = 1, 10-12 = 1), both K-major (bits 15, 16 = 0),
// N >> 3 in bits 17-22, M >> 4 in bits 24-28.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

// The same for tcgen05.mma kind::f8f6f4 with A and B both E4M3 (format 0 in bits
// 7-9 and 10-12). A row chunk of 128 E4M3 values is 128 bytes, like a chunk of 64
// bf16 values, and one MMA consumes K = 32 of them, 32 bytes, like K = 16 bf16: the
// shared-memory tiles, descriptors and the K loop are byte for byte the bf16 ones.
constexpr uint32_t kIdescE4M3 = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase of `bar` with the given parity to complete. Gives up after
// `limit` clock cycles (raising EM_E_TIMEOUT and the CTA-wide abort flag) or as
// soon as another thread or CTA has raised an error.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, long long limit, int* err,
                                          volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0) {
            if (*abort_flag || error_raised(err)) {
                *abort_flag = 1;
                return false;
            }
            if (clock64() - t0 > limit) {
                raise_error(err, EM_E_TIMEOUT);
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// Time-bounded wait used on the error path to let in-flight copies and MMAs land
// before the CTA releases its shared memory and tensor memory.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity, long long limit) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit) return;
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* tm, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"((uint64_t)tm), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor (K-major, swizzled): start address >> 4 in bits
// 0-13, leading byte offset (unused for swizzled K-major, 16 B) in 16-29, stride
// byte offset between 8-row groups >> 4 in 32-45, descriptor version 1 in bit 46,
// layout (swizzle mode) in bits 61-63.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint64_t layout, uint32_t sbo) {
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | (1ull << 16) | ((uint64_t)(sbo >> 4) << 32) | (1ull << 46) |
           (layout << 61);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(kIdescE4M3), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// Waits for this thread's TMEM loads, with the 32 registers of the last one as
// operands: every use of the loaded values is ordered after the wait.
__device__ __forceinline__ void tmem_wait_ld32(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                   "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                   "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

// One 32-column chunk of a row's scores: adds |c|^2 (c4: the chunk's 32 values) to
// the raw accumulators v (in place, two lanes per packed add) and updates the
// running best (TOP2: best two) with the lowest column on ties. Without TOP2 the
// chunk's minimum is taken as a tree of three-input minima and only a row it
// improves looks for the lowest column that reaches it: first the triple of the
// tree's lowest level, then the column within it (a 32-column equality scan here
// made the search of d = 96 rows 8 % slower).
// Two fp32 additions in one packed instruction (add.rn.f32x2): each lane rounds as a
// scalar add does, so the scores are the same bits.
__device__ __forceinline__ void add2_f32(uint32_t& a0, uint32_t& a1, float b0, float b1) {
    asm("{\n\t.reg .b64 x, y, z;\n\t"
        "mov.b64 x, {%0, %1};\n\t"
        "mov.b64 y, {%2, %3};\n\t"
        "add.rn.f32x2 z, x, y;\n\t"
        "mov.b64 {%0, %1}, z;\n\t}"
        : "+r"(a0), "+r"(a1)
        : "r"(__float_as_uint(b0)), "r"(__float_as_uint(b1)));
}

// The minimum of three fp32 values in one instruction (exact).
__device__ __forceinline__ float min3_f32(float a, float b, float c) {
    float d;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

template <bool TOP2, bool ADD = true>
__device__ __forceinline__ void scan_chunk(uint32_t (&v)[32], const float4* c4, int jb, float& best, int& bidx,
                                           float& best2, int& bidx2) {
    if (ADD) {  // (without: the norms are already in the accumulator)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 cc = c4[i];
            add2_f32(v[4 * i + 0], v[4 * i + 1], cc.x, cc.y);
            add2_f32(v[4 * i + 2], v[4 * i + 3], cc.z, cc.w);
        }
    }
    if (TOP2) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {  // branch-free: a divergent skip test measured slower
            const float x = __uint_as_float(v[e]);
            const bool p1 = x < best, p2 = x < best2;
            best2 = p1 ? best : (p2 ? x : best2);
            bidx2 = p1 ? bidx : (p2 ? jb + e : bidx2);
            best = p1 ? x : best;
            bidx = p1 ? jb + e : bidx;
        }
    } else {
        // the chunk's minimum as a tree of three-input minima (32 -> 11 -> 4 -> 1)
        float t11[11];
#pragma unroll
        for (int e = 0; e < 10; ++e)
            t11[e] = min3_f32(__uint_as_float(v[3 * e]), __uint_as_float(v[3 * e + 1]), __uint_as_float(v[3 * e + 2]));
        t11[10] = fminf(__uint_as_float(v[30]), __uint_as_float(v[31]));
        const float u0 = min3_f32(t11[0], t11[1], t11[2]), u1 = min3_f32(t11[3], t11[4], t11[5]);
        const float u2 = min3_f32(t11[6], t11[7], t11[8]), u3 = fminf(t11[9], t11[10]);
        const float mn = min3_f32(u0, u1, fminf(u2, u3));
        if (mn < best) {
            // the first triple whose minimum is mn holds the first column that is
            // (every column of an earlier triple is above mn); then the first of its
            // two or three columns
            unsigned tm = 0;
#pragma unroll
            for (int e = 0; e < 11; ++e) tm |= (t11[e] == mn) ? (1u << e) : 0u;
            const int h = __ffs(tm) - 1;
            float a = __uint_as_float(v[0]), b = __uint_as_float(v[1]);
#pragma unroll
            for (int e = 1; e < 11; ++e) {
                a = h == e ? __uint_as_float(v[3 * e]) : a;
                b = h == e ? __uint_as_float(v[3 * e + 1]) : b;
            }
            best = mn;
            bidx = jb + 3 * h + (a == mn ? 0 : (b == mn ? 1 : 2));
        }
    }
}

// Output: for every row, column half h of the split g of the centroid tiles it
// covers writes two keys at keys[((2 g + h) * rows + row) * 2 + {0, 1}]: the best
// (score, index) and, with TOP2, the second best (without it the second key is
// empty).
// Self-test of the failure path: one thread waits on an mbarrier that nothing
// arrives on, with the search kernel's bounded wait, so the wait gives up after
// `wait_limit` cycles and raises EM_E_TIMEOUT in the error word; or (which = 1) the
// kernel raises EM_E_BOUNDS as a failed index check would. Nothing faults or hangs.
__global__ void k_selftest(int which, long long wait_limit, int* err) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    if (which == 1) {
        raise_error(err, EM_E_BOUNDS);
        return;
    }
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_wait(smem_u32(&bar), 0u, wait_limit, err, &abort_flag);  // phase 0 never completes
}

// A work unit: row tile m, centroid-tile group g, centroid tiles [nt0, nt1). The
// first m_full row tiles are one unit each, over all n_tiles centroid tiles (group
// 0); every later row tile is n_split units of tpg tiles.
struct Unit {
    int m, g, nt0, nt1;
};
__device__ __forceinline__ Unit unit_of(int u, int m_full, int n_split, int tpg, int n_tiles) {
    if (u < m_full) return Unit{u, 0, 0, n_tiles};
    const int v = u - m_full;
    const int q = v / n_split;
    const int g = v - q * n_split;
    return Unit{m_full + q, g, g * tpg, min(g * tpg + tpg, n_tiles)};
}

// F8: the batch rows and the centroid operand are E4M3 codes (KC = 64 only: row
// chunks of 128 bytes = 128 codes).
template <int KC, bool TOP2, bool AST, bool F8 = false, bool FOLD = false>
__global__ void __launch_bounds__(threads_for<epi_groups<TOP2, AST>()>(), 1)
    k_assign_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmN, const __grid_constant__ CUtensorMap tmO,
                const float* __restrict__ cn, int k, int rows, int nkc, int n_tiles, int n_split, int m_full,
                unsigned long long* __restrict__ keys, long long wait_limit, int* err) {
    constexpr int G = epi_groups<TOP2, AST>();
    static_assert(!FOLD || (AST && !TOP2 && !F8), "the folded norms need the stationary batch tile and bf16");
    using C = Cfg<KC, AST, G, FOLD>;
    constexpr int S = C::kStages;
    static_assert(!F8 || KC == 64, "E4M3 rows use 128-byte chunks");
    constexpr int KX = F8 ? 2 * KC : KC;  // elements per row chunk (the TMA x step)
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // ring: (A, B) per stage, or B only with the A buffers after the ring (AST)
    uint8_t* sA = smem;
    uint8_t* sB = AST ? smem : smem + S * C::kABytes;
    uint8_t* sArea = smem + S * C::kStageBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::kStageBytes + C::kAreaBytes);
    uint64_t* full = bars;
    uint64_t* empty = bars + S;
    uint64_t* tfull = bars + 2 * S;
    uint64_t* tempty = bars + 2 * S + 2;
    uint64_t* drain = bars + 2 * S + 4;
    uint64_t* afull = bars + 2 * S + 5;   // AST: A buffer loaded
    uint64_t* aempty = bars + 2 * S + 7;  // AST: A buffer no longer read by the MMAs
    uint64_t* xbar = bars + 2 * S + 9;    // FOLD: the ones tile loaded
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 10);
    uint8_t* sOnes = sArea + 2 * kAstBufBytes;  // FOLD: the ones tile (1024-aligned, after the A buffers)
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* cn_s = reinterpret_cast<float*>(smem + S * C::kStageBytes + C::kAreaBytes + C::kBarBytes);
    // (two groups) merge slots [warp pair][unit parity][lane], then their barriers
    float2* mslot = reinterpret_cast<float2*>(cn_s + kEpiWarps * 2 * kEpiCols);
    uint64_t* mfull = reinterpret_cast<uint64_t*>(mslot + 8 * 2 * 32);
    uint64_t* mempty = mfull + 16;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // the error-path drains get at least ~2 s whatever limit the caller chose
    const long long drain_limit = wait_limit > 4000000000ll ? wait_limit : 4000000000ll;
    const int m_tiles = (rows + BM - 1) / BM;
    const int tpg = (n_tiles + n_split - 1) / n_split;
    const int units = m_full + (m_tiles - m_full) * n_split;
    // ring stages in use: chunk stages, or (A stationary) whole centroid tiles of nkc
    // chunks each, so that a tile costs one barrier round trip instead of nkc
    // a tile's bytes in the ring (A stationary: its nkc chunks, and with FOLD its norms)
    const int tile_bytes = nkc * C::kBBytes + (FOLD ? kExtBBytes : 0);
    const int st_n = AST ? (S * C::kBBytes) / tile_bytes : S;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), kEpiThreads);
        }
        mbar_init(smem_u32(drain), 1);
        mbar_init(smem_u32(xbar), 1);
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&afull[a]), 1);
            mbar_init(smem_u32(&aempty[a]), 1);
        }
        if (G == 2)
            for (int i = 0; i < 16; ++i) {
                mbar_init(smem_u32(&mfull[i]), 32);
                mbar_init(smem_u32(&mempty[i]), 32);
            }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(512u)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmA) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmB) : "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // the set-up above overlaps the previous kernel; the operands are read after it
    pdl_wait();

    if (warp == 0) {
        // ---------------- TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            uint32_t armed = 0, armed_parity = 0;  // per-stage bit masks
            uint32_t aarmed = 0, aarmed_parity = 0;  // the two A buffers (AST)
            int ua = 0;                              // units started (AST)
            if (FOLD && (int)blockIdx.x < units) {  // the ones tile, once
                mbar_expect_tx(smem_u32(xbar), (uint32_t)kExtABytes);
                tma_load_2d(smem_u32(sOnes), &tmO, 0, 0, smem_u32(xbar));
            }
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                const Unit w = unit_of(u, m_full, n_split, tpg, n_tiles);
                const int m = w.m, nt0 = w.nt0, nt1 = w.nt1;
                if (AST) {  // the unit's rows, once, into A buffer ua % 2
                    const int ab = ua & 1;
                    const uint32_t par = (uint32_t)(ua >> 1) & 1u;
                    if (!mbar_wait(smem_u32(&aempty[ab]), par ^ 1u, wait_limit, err, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&afull[ab]);
                    aarmed |= 1u << ab;
                    aarmed_parity = (aarmed_parity & ~(1u << ab)) | (par << ab);
                    mbar_expect_tx(fb, (uint32_t)(nkc * C::kABytes));
                    for (int kc = 0; kc < nkc; ++kc)
                        tma_load_2d(smem_u32(sArea + ab * kAstBufBytes + kc * C::kABytes), &tmA, kc * KX, m * BM, fb);
                    ++ua;
                }
                for (int nt = nt0; nt < nt1 && ok; ++nt) {
                    if (AST) {  // the whole centroid tile into one stage of nkc chunks, one barrier
                        if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, wait_limit, err, abort_flag)) {
                            ok = false;
                            break;
                        }
                        const uint32_t fb = smem_u32(&full[stage]);
                        armed |= 1u << stage;
                        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                        mbar_expect_tx(fb, (uint32_t)tile_bytes);
                        uint8_t* tb = sB + stage * tile_bytes;
                        for (int kc = 0; kc < nkc; ++kc)
                            tma_load_2d(smem_u32(tb + kc * C::kBBytes), &tmB, kc * KX, nt * BN, fb);
                        if (FOLD) tma_load_2d(smem_u32(tb + nkc * C::kBBytes), &tmN, 0, nt * BN, fb);
                        if (++stage == st_n) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    } else {
                        for (int kc = 0; kc < nkc; ++kc) {
                            if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, wait_limit, err, abort_flag)) {
                                ok = false;
                                break;
                            }
                            const uint32_t fb = smem_u32(&full[stage]);
                            armed |= 1u << stage;
                            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                            mbar_expect_tx(fb, C::kStageBytes);
                            tma_load_2d(smem_u32(sA + stage * C::kABytes), &tmA, kc * KX, m * BM, fb);
                            tma_load_2d(smem_u32(sB + stage * C::kBBytes), &tmB, kc * KX, nt * BN, fb);
                            if (++stage == S) {
                                stage = 0;
                                phase ^= 1u;
                            }
                        }
                    }
                }
            }
            if (!ok) {  // let every copy this thread started land before shared memory is released
                for (int s2 = 0; s2 < S; ++s2)
                    if (armed & (1u << s2)) mbar_drain(smem_u32(&full[s2]), (armed_parity >> s2) & 1u, drain_limit);
                for (int a2 = 0; a2 < 2; ++a2)
                    if (aarmed & (1u << a2)) mbar_drain(smem_u32(&afull[a2]), (aarmed_parity >> a2) & 1u, drain_limit);
                if (FOLD && (int)blockIdx.x < units) mbar_drain(smem_u32(xbar), 0u, drain_limit);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (one thread)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            int ua = 0;
            if (FOLD && (int)blockIdx.x < units) {
                ok = mbar_wait(smem_u32(xbar), 0u, wait_limit, err, abort_flag);
                tc_fence_after();
            }
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                const Unit w = unit_of(u, m_full, n_split, tpg, n_tiles);
                const int nt0 = w.nt0, nt1 = w.nt1;
                const int ab = ua & 1;
                if (AST) {
                    if (!mbar_wait(smem_u32(&afull[ab]), (uint32_t)(ua >> 1) & 1u, wait_limit, err, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                for (int nt = nt0; nt < nt1 && ok; ++nt) {
                    if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, wait_limit, err, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                    if (AST) {  // one stage holds the tile's nkc chunks
                        if (!mbar_wait(smem_u32(&full[stage]), phase, wait_limit, err, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        uint8_t* tb = sB + stage * tile_bytes;
                        for (int kc = 0; kc < nkc; ++kc) {
                            const uint32_t a0 = smem_u32(sArea + ab * kAstBufBytes + kc * C::kABytes);
                            const uint32_t b0 = smem_u32(tb + kc * C::kBBytes);
#pragma unroll
                            for (int kk = 0; kk < KC / 16; ++kk) {
                                const uint64_t ad = smem_desc(a0 + kk * 32, C::kLayout, C::kSBO);
                                const uint64_t bd = smem_desc(b0 + kk * 32, C::kLayout, C::kSBO);
                                if (F8)
                                    umma_e4m3(d_tmem, ad, bd, (kc | kk) != 0);
                                else
                                    umma_bf16(d_tmem, ad, bd, (kc | kk) != 0);
                            }
                        }
                        if (FOLD)  // + (1, 1, 1) . (h, m, l) = |c~|^2 on every row
                            umma_bf16(d_tmem, smem_desc(smem_u32(sOnes), kExtLayout, kExtSBO),
                                      smem_desc(smem_u32(tb + nkc * C::kBBytes), kExtLayout, kExtSBO), 1u);
                        umma_commit(smem_u32(&empty[stage]));
                        if (++stage == st_n) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    } else {
                        for (int kc = 0; kc < nkc; ++kc) {
                            if (!mbar_wait(smem_u32(&full[stage]), phase, wait_limit, err, abort_flag)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            const uint32_t a0 = smem_u32(sA + stage * C::kABytes);
                            const uint32_t b0 = smem_u32(sB + stage * C::kBBytes);
#pragma unroll
                            for (int kk = 0; kk < KC / 16; ++kk) {
                                const uint64_t ad = smem_desc(a0 + kk * 32, C::kLayout, C::kSBO);
                                const uint64_t bd = smem_desc(b0 + kk * 32, C::kLayout, C::kSBO);
                                if (F8)
                                    umma_e4m3(d_tmem, ad, bd, (kc | kk) != 0);
                                else
                                    umma_bf16(d_tmem, ad, bd, (kc | kk) != 0);
                            }
                            umma_commit(smem_u32(&empty[stage]));
                            if (++stage == S) {
                                stage = 0;
                                phase ^= 1u;
                            }
                        }
                        if (!ok) break;
                    }
                    umma_commit(smem_u32(&tfull[acc]));
                    acc ^= 1;
                    if (acc == 0) acc_phase ^= 1u;
                }
                if (AST && ok) {  // the unit's MMAs are issued: its A buffer frees once they complete
                    umma_commit(smem_u32(&aempty[ab]));
                    ++ua;
                }
            }
            if (!ok) {  // wait for every MMA this thread issued before TMEM is freed
                umma_commit(smem_u32(drain));
                mbar_drain(smem_u32(drain), 0u, drain_limit);
            }
        }
    } else {
        // ---------------- epilogue: 8 G warps, thread = accumulator row, warp = column half
        const int ew = warp - 2;
        const int grp = G == 2 ? ew >> 3 : 0;  // the accumulator this warp's group takes (G = 2)
        const int wi = ew & 7;                 // the warp's place in its group
        const int q = warp & 3;
        const int half = wi >> 2;          // column part of the tile
        const int rl = 32 * q + lane;      // row within the tile
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        float* cn_w = cn_s + ew * (2 / G) * kEpiCols;  // this warp's |c|^2 buffers (two, or one)
        int acc = 0;
        uint32_t acc_phase = 0;
        int cnbuf = 0;
        int uc = 0;  // units done (the merge slots alternate)
        bool ok = true;
        // this lane's |c|^2 values of the next tile the warp handles, one tile ahead
        constexpr int kPer = kEpiCols / 32;
        float cn_next[kPer];
        auto cn_of = [&](int j) {
            if (kPer == 4 && j + 4 <= k) {  // (j is a multiple of 4: one 16-byte load)
                const float4 v = *reinterpret_cast<const float4*>(cn + j);
                cn_next[0] = v.x;
                cn_next[1 % kPer] = v.y;
                cn_next[2 % kPer] = v.z;
                cn_next[3 % kPer] = v.w;
                return;
            }
#pragma unroll
            for (int i = 0; i < kPer; ++i) cn_next[i] = j + i < k ? cn[j + i] : __int_as_float(0x7f800000);
        };
        // the tile after (u2, nt2) in this CTA's sequence (u2 >= units: none)
        auto step_tile = [&](int& u2, int& nt2) {
            if (nt2 + 1 < unit_of(u2, m_full, n_split, tpg, n_tiles).nt1) {
                ++nt2;
                return;
            }
            u2 += gridDim.x;
            if (u2 < units) nt2 = unit_of(u2, m_full, n_split, tpg, n_tiles).nt0;
        };
#pragma unroll
        for (int i = 0; i < kPer; ++i) cn_next[i] = 0.0f;
        if (!FOLD) {  // the first tile of this warp: the first of the sequence, or of its accumulator
            int u2 = blockIdx.x, nt2 = 0;
            if (u2 < units) nt2 = unit_of(u2, m_full, n_split, tpg, n_tiles).nt0;
            for (int i = 0; i < grp && u2 < units; ++i) step_tile(u2, nt2);
            if (u2 < units) cn_of(nt2 * BN + half * kEpiCols + kPer * lane);
        }
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            const Unit w = unit_of(u, m_full, n_split, tpg, n_tiles);
            const int m = w.m, g = w.g, nt0 = w.nt0, nt1 = w.nt1;
            float best = __int_as_float(0x7f800000);  // +inf
            float best2 = best;
            int bidx = 0, bidx2 = 0;
            for (int nt = nt0; nt < nt1; ++nt) {
                if (G == 1 || acc == grp) {
                    float* cnb = cn_w + cnbuf * kEpiCols;
                    const int j0 = nt * BN;
                    if (!FOLD) {
                        if (G == 2) __syncwarp();  // (one buffer) every lane is done with the last tile's
#pragma unroll
                        for (int i = 0; i < kPer; ++i) cnb[kPer * lane + i] = cn_next[i];
                    }
                    if (!FOLD) {  // the warp's next tile, G tiles on
                        int u2 = u, nt2 = nt;
                        if (nt + G < nt1) {
                            nt2 = nt + G;
                        } else {
                            for (int i = 0; i < G && u2 < units; ++i) step_tile(u2, nt2);
                        }
                        if (u2 < units) cn_of(nt2 * BN + half * kEpiCols + kPer * lane);
                    }
                    // the whole warp takes one decision (a lane that gave up takes the warp with it)
                    const bool got = __all_sync(
                        0xFFFFFFFFu, mbar_wait(smem_u32(&tfull[acc]), acc_phase, wait_limit, err, abort_flag));
                    if (!got) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    __syncwarp();  // also publishes this warp's |c|^2 values
                    const uint32_t tbase = tmem_base + lane_base + (uint32_t)(acc * BN + half * kEpiCols);
                    const float4* c4 = reinterpret_cast<const float4*>(cnb);
                    const int jh = j0 + half * kEpiCols;
                    // chunks of 32 columns, the load of the next in flight while one is
                    // scanned; the accumulator goes back once the last chunk is in registers
                    {
                        constexpr int kChunks = kEpiCols / 32;
                        uint32_t va[32], vb[32];
                        tmem_ld32(tbase, va);
                        tmem_wait_ld32(va);
#pragma unroll
                        for (int c = 0; c < kChunks; c += 2) {
                            tmem_ld32(tbase + 32 * (c + 1), vb);
                            scan_chunk<TOP2, !FOLD>(va, c4 + 8 * c, jh + 32 * c, best, bidx, best2, bidx2);
                            tmem_wait_ld32(vb);
                            if (c + 2 < kChunks) {
                                tmem_ld32(tbase + 32 * (c + 2), va);
                            } else {
                                tc_fence_before();
                                mbar_arrive(smem_u32(&tempty[acc]));
                            }
                            scan_chunk<TOP2, !FOLD>(vb, c4 + 8 * (c + 1), jh + 32 * (c + 1), best, bidx, best2, bidx2);
                            if (c + 2 < kChunks) tmem_wait_ld32(va);
                        }
                    }
                    if (G == 1) cnbuf ^= 1;
                }
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (!ok) break;
            if (G == 2) {
                // the second group hands its rows' best of this unit to the first
                const int slot = wi * 2 + (uc & 1);
                const uint32_t par = (uint32_t)(uc >> 1) & 1u;
                ++uc;
                if (grp == 1) {
                    const bool free_slot = __all_sync(
                        0xFFFFFFFFu, mbar_wait(smem_u32(&mempty[slot]), par ^ 1u, wait_limit, err, abort_flag));
                    if (!free_slot) {
                        ok = false;
                        break;
                    }
                    mslot[slot * 32 + lane] = make_float2(best, __int_as_float(bidx));
                    mbar_arrive(smem_u32(&mfull[slot]));
                    continue;
                }
                const bool arrived = __all_sync(
                    0xFFFFFFFFu, mbar_wait(smem_u32(&mfull[slot]), par, wait_limit, err, abort_flag));
                if (!arrived) {
                    ok = false;
                    break;
                }
                const float2 o = mslot[slot * 32 + lane];
                mbar_arrive(smem_u32(&mempty[slot]));
                const int oi = __float_as_int(o.y);
                if (o.x < best || (o.x == best && oi < bidx)) {  // lower score, then lower column
                    best = o.x;
                    bidx = oi;
                }
            }
            // this column half's key set: (score, index) keys order as the argmin does
            // (lower score, then lower index)
            const int row = m * BM + rl;
            if (row < rows) {
                unsigned long long* out = keys + ((int64_t)(kKeySets * g + half) * rows + row) * 2;
                out[0] = best < __int_as_float(0x7f800000) ? pack_key(best, (uint32_t)bidx) : kEmptyKey;
                out[1] = TOP2 && best2 < __int_as_float(0x7f800000) ? pack_key(best2, (uint32_t)bidx2) : kEmptyKey;
                // a whole row tile also empties the other groups' key sets, which the
                // label kernel reads for every row
                if (u < m_full)
                    for (int g2 = 1; g2 < n_split; ++g2)
                        reinterpret_cast<ulonglong2*>(keys)[(int64_t)(kKeySets * g2 + half) * rows + row] =
                            make_ulonglong2(kEmptyKey, kEmptyKey);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512u) : "memory");
    }
}

// The folded search's norms operand: row j is (h, m, l, 0, ...) in bf16 with
// h + m + l = |c~_j|^2: h the fp32 value rounded to bf16, m the remainder rounded,
// l the rest, each remainder exact in fp32 (its operands are within a factor of two
// of each other), so the three parts carry all 24 bits. A non-finite value goes
// into h alone. The rows from k to k_pad (the rest of the last centroid tile) hold
// +inf, so that the tile's missing centroids (zero operand rows) never win.
__global__ void k_fold_norms(const float* __restrict__ cn, int k, int k_pad, __nv_bfloat16* __restrict__ cn3) {
    pdl_wait();
    pdl_release();
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < k_pad; j += gridDim.x * blockDim.x) {
        const float c = j < k ? cn[j] : __int_as_float(0x7f800000);
        const __nv_bfloat16 h = __float2bfloat16_rn(c);
        __nv_bfloat16 mid = __float2bfloat16_rn(0.0f), lo = mid;
        if (isfinite(c)) {
            const float r1 = c - __bfloat162float(h);
            mid = __float2bfloat16_rn(r1);
            lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
        }
        uint4 v0;
        v0.x = (uint32_t)__bfloat16_as_ushort(h) | ((uint32_t)__bfloat16_as_ushort(mid) << 16);
        v0.y = (uint32_t)__bfloat16_as_ushort(lo);
        v0.z = 0u;
        v0.w = 0u;
        uint4* row = reinterpret_cast<uint4*>(cn3 + (int64_t)j * kExtK);
        row[0] = v0;
        row[1] = make_uint4(0u, 0u, 0u, 0u);
    }
}

}  // namespace tc

// Plain SIMT search (one thread per row, fp32 FMA over bf16 operands). Not used
// by training unless selected explicitly; it exists to tell a tensor-core fault
// apart from a fault elsewhere in the step when a parity test fails.
__global__ void k_assign_simt(const __nv_bfloat16* __restrict__ A, int ld, int rows, const __nv_bfloat16* __restrict__ cq,
                              const float* __restrict__ cn, int k, int d, unsigned long long* __restrict__ keys) {
    pdl_wait();
    const int row = blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= rows) return;
    const __nv_bfloat16* x = A + (int64_t)row * ld;
    float best = __int_as_float(0x7f800000);
    int bidx = 0;
    for (int j = 0; j < k; ++j) {
        const __nv_bfloat16* q = cq + (int64_t)j * ld;
        float acc = 0.0f;
        for (int e = 0; e < d; ++e) acc = fmaf(__bfloat162float(x[e]), __bfloat162float(q[e]), acc);
        const float s = cn[j] + acc;
        if (s < best) {
            best = s;
            bidx = j;
        }
    }
    keys[(int64_t)row * 2] = pack_key(best, (uint32_t)bidx);
    keys[(int64_t)row * 2 + 1] = kEmptyKey;
}

}  // namespace em
