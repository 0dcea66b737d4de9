// emeans.cu -- host orchestration and the C ABI of the B200 e-means library.
//
// One training step (faiss e-means README, "Data too big for memory": accumulate
// then update, run by `train` internally) is this kernel sequence on the model's
// stream:
//   k_gather        batch rows pi_pass(pos..pos+B) -> contiguous bf16 batch, |x|^2
//                   (and E4M3 codes with the FP8 search); prefetched: the next
//                   step's rows are gathered on a second stream beside the search
//   k_fold_norms    (d < 128 with many tiles) the norms operand the search folds in
//   k_assign_tc     nearest centroid of every batch row (tcgen05 + TMA)
//   k_labels        labels, distances, per-cluster counts and ranks
//   k_settle        near ties re-decided in fp64
//   k_offsets       segment starts and work-item starts, batch error sum
//   k_scatter       rows in label order, one work item per chunk of a cluster
//   k_segsum        per-chunk sums (fp64) fused with the EMA update of small clusters
//   k_clusters      large clusters (chunk sums in order), clusters without rows
//   k_normalize / k_fp8_operand   spherical rescaling / the E4M3 operand, if on
//   k_revive_*      every 5th step: dead-cluster revival (the donor selection runs
//                   on the second stream beside k_scatter .. k_clusters)
// The kernels launch with programmatic stream serialization, each waiting on the
// device for its predecessor. No host synchronisation happens inside a run; the
// step size of step t is computed on the host (cosine schedule) and passed by
// value; ranges of steps are captured and replayed as CUDA graphs.
//
// Data-parallel runs (README "Several GPUs": DistributedEmeans, one process per
// GPU, each with its own share of the rows): every rank searches its share of each
// batch and k_segsum / k_clusters leave its per-cluster statistics (n_j, s_j, in
// fp64) instead of updating; one NCCL all-reduce adds them across ranks on the
// model's stream, and k_apply_stats applies the same EMA on every rank. NCCL is
// loaded at run time, only when a communicator is created.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <dlfcn.h>
#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include <nccl.h>  // types and prototypes only: the library is loaded with dlopen

#include "common.cuh"
#include "k_assign.cuh"
#include "k_data.cuh"
#include "k_reduce.cuh"
#include "k_revive.cuh"
#include "k_fp8.cuh"

using namespace em;

// ------------------------------------------------------------------ errors

static thread_local char g_err[1024] = "";
static thread_local int g_err_code = 0;

static int fail(int code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    g_err_code = code;
    return code;
}

#define CK(call)                                                                                 \
    do {                                                                                         \
        cudaError_t e_ = (call);                                                                 \
        if (e_ != cudaSuccess) return fail(EM_E_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
    } while (0)

#define CKR(expr)              \
    do {                       \
        int r_ = (expr);       \
        if (r_ != EM_OK) return r_; \
    } while (0)

// ------------------------------------------------------------------ recipe (host)

static const double kLawConst[2] = {0.035134, 0.00439175};

static int compute_recipe(int64_t n, int64_t k, int64_t d, double epochs, int law, int64_t batch_override,
                          double alpha_override, em_recipe_t* r) {
    if (n < 1 || k < 1 || !(epochs > 0.0) || law < 0 || law > 1) return fail(EM_E_INVAL, "bad recipe arguments");
    memset(r, 0, sizeof(*r));
    r->n = n;
    r->k = k;
    r->d = d;
    r->epochs = epochs;
    // equations (1)/(2), nearest power of two in log2, capped at the largest power of two <= n/2
    int64_t b;
    if (batch_override > 0) {
        b = batch_override;
        r->batch_raw = (double)b;
    } else {
        r->batch_raw = kLawConst[law] * pow((double)k, 0.134749) * pow((double)n, 0.876473) * pow(epochs, 0.813344);
        const double lb = log2(std::max(r->batch_raw, 1.0));
        const long e = lround(lb);  // halves round away from zero, as Python's round never sees them here
        b = (int64_t)1 << std::min<long>(e, 62);
        const double half = std::max((double)n / 2.0, 1.0);
        const int64_t cap = (int64_t)1 << (int)floor(log2(half));
        b = std::max<int64_t>(1, std::min(b, cap));
    }
    r->batch_size = b;
    // equation (3), clamped to [1e-4, 1]
    if (alpha_override > 0.0) {
        r->alpha0 = alpha_override;
    } else {
        double a = 0.8244 * pow((double)k, -0.4617) * pow((double)b, 0.9003) * pow((double)n, -0.4498) *
                   pow(epochs, -0.1057);
        r->alpha0 = std::min(1.0, std::max(1e-4, a));
    }
    const double whole = floor(epochs);
    const double frac = epochs - whole;
    r->passes = (int64_t)whole + (frac > 0 ? 1 : 0);
    r->rows_last_pass = frac > 0 ? std::max<int64_t>(1, (int64_t)floor(frac * (double)n + 0.5)) : n;
    r->steps_full_pass = (n + b - 1) / b;
    r->steps_last_pass = (r->rows_last_pass + b - 1) / b;
    r->total_steps = (r->passes - 1) * r->steps_full_pass + r->steps_last_pass;
    return EM_OK;
}

// Launch shapes of the near-tie settling and the cluster pass (set at build time
// for sweeps): k_settle blocks per SM, k_clusters threads per block.
#ifndef EM_SETTLE_BLOCKS_PER_SM
#define EM_SETTLE_BLOCKS_PER_SM 8
#endif
#ifndef EM_CLUSTERS_BLOCK
#define EM_CLUSTERS_BLOCK 256
#endif

// cosine step size from alpha0 down to alpha0 / 10 over all steps
static double alpha_at(int64_t t, int64_t total, double alpha0) {
    const double amin = 0.1 * alpha0;
    const double frac = total <= 1 ? 0.0 : (double)t / (double)(total - 1);
    return amin + (alpha0 - amin) * 0.5 * (1.0 + cos(M_PI * frac));
}

static uint32_t __float_as_uint_host(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    return u;
}

// Launches `kern` on `stream`, with programmatic stream serialization when `pdl`
// is set: the kernel may then launch while its predecessor on the stream is still
// finishing, and waits for it with griddepcontrol.wait (every kernel of the
// library starts with that wait).
template <typename... KArgs, typename... Args>
static cudaError_t launch_k(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                           Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ------------------------------------------------------------------ NCCL (loaded on demand)

struct NcclApi {
    bool ok = false;
    decltype(&ncclGetUniqueId) get_id = nullptr;
    decltype(&ncclCommInitRank) init_rank = nullptr;
    decltype(&ncclAllReduce) all_reduce = nullptr;
    decltype(&ncclBroadcast) broadcast = nullptr;
    decltype(&ncclCommDestroy) destroy = nullptr;
    decltype(&ncclGetErrorString) error_string = nullptr;
};

// The process's libnccl.so.2 (the one already loaded, if any, else the first on the
// library path).
static const NcclApi& nccl() {
    static NcclApi api;
    static std::once_flag once;
    std::call_once(once, [] {
        void* h = dlopen("libnccl.so.2", RTLD_NOW | RTLD_GLOBAL);
        if (!h) h = dlopen("libnccl.so", RTLD_NOW | RTLD_GLOBAL);
        if (!h) return;
        api.get_id = reinterpret_cast<decltype(api.get_id)>(dlsym(h, "ncclGetUniqueId"));
        api.init_rank = reinterpret_cast<decltype(api.init_rank)>(dlsym(h, "ncclCommInitRank"));
        api.all_reduce = reinterpret_cast<decltype(api.all_reduce)>(dlsym(h, "ncclAllReduce"));
        api.broadcast = reinterpret_cast<decltype(api.broadcast)>(dlsym(h, "ncclBroadcast"));
        api.destroy = reinterpret_cast<decltype(api.destroy)>(dlsym(h, "ncclCommDestroy"));
        api.error_string = reinterpret_cast<decltype(api.error_string)>(dlsym(h, "ncclGetErrorString"));
        api.ok = api.get_id && api.init_rank && api.all_reduce && api.broadcast && api.destroy && api.error_string;
    });
    return api;
}

#define NCK(call)                                                                                  \
    do {                                                                                           \
        const ncclResult_t r_ = (call);                                                            \
        if (r_ != ncclSuccess) return fail(EM_E_COMM, "%s: %s", #call, nccl().error_string(r_));   \
    } while (0)

// ------------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// 2-D bf16 tensor map over `rows` rows of d values (row pitch ld elements), boxes
// of kc x box_rows with the swizzle the UMMA descriptors expect.
static int make_tmap(CUtensorMap* tm, const void* base, int64_t rows, int d, int ld, int box_rows, int kc) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(EM_E_CUDA, "cuTensorMapEncodeTiled is not available");
    if ((reinterpret_cast<uintptr_t>(base) & 15) != 0) return fail(EM_E_INVAL, "tensor base not 16-byte aligned");
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)std::max<int64_t>(rows, 1)};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    cuuint32_t box[2] = {(cuuint32_t)kc, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, kc == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(EM_E_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return EM_OK;
}

// 2-D tensor map over `rows` rows of 16 bf16 values (32-byte rows, the 32-byte
// swizzle), boxes of box_rows rows: the folded search's norms and ones operands.
static int make_tmap_ext(CUtensorMap* tm, const void* base, int64_t rows, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(EM_E_CUDA, "cuTensorMapEncodeTiled is not available");
    if ((reinterpret_cast<uintptr_t>(base) & 15) != 0) return fail(EM_E_INVAL, "tensor base not 16-byte aligned");
    cuuint64_t dims[2] = {(cuuint64_t)tc::kExtK, (cuuint64_t)std::max<int64_t>(rows, 1)};
    cuuint64_t strides[1] = {(cuuint64_t)tc::kExtK * 2};
    cuuint32_t box[2] = {(cuuint32_t)tc::kExtK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(EM_E_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return EM_OK;
}

// 2-D tensor map over `rows` rows of d E4M3 codes (row pitch ld8 bytes), boxes of
// 128 codes (128 bytes, the 128-byte swizzle) x box_rows; columns past d read as 0.
static int make_tmap8(CUtensorMap* tm, const void* base, int64_t rows, int d, int ld8, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(EM_E_CUDA, "cuTensorMapEncodeTiled is not available");
    if ((reinterpret_cast<uintptr_t>(base) & 15) != 0 || (ld8 & 15) != 0)
        return fail(EM_E_INVAL, "E4M3 rows must be 16-byte aligned");
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)std::max<int64_t>(rows, 1)};
    cuuint64_t strides[1] = {(cuuint64_t)ld8};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(EM_E_CUDA, "cuTensorMapEncodeTiled (E4M3) failed (%d)", (int)r);
    return EM_OK;
}

// ------------------------------------------------------------------ model

// Allocation-failure injection (em_fail_allocation): the countdown to the device
// allocation that fails, and the number of allocations attempted.
static std::atomic<int64_t> g_alloc_fail_at{0};
static std::atomic<int64_t> g_alloc_attempts{0};

// Whether this allocation attempt is the one em_fail_allocation asked to fail.
static bool injected_alloc_failure() {
    g_alloc_attempts.fetch_add(1, std::memory_order_relaxed);
    int64_t left = g_alloc_fail_at.load(std::memory_order_relaxed);
    while (left > 0) {
        if (g_alloc_fail_at.compare_exchange_weak(left, left - 1, std::memory_order_relaxed)) return left == 1;
    }
    return false;
}

template <class T>
struct DBuf {
    T* p = nullptr;
    size_t cap = 0;  // elements
    int ensure(size_t count) {
        if (count <= cap && p) return EM_OK;
        if (p) cudaFree(p);
        p = nullptr;
        cap = 0;
        if (injected_alloc_failure())
            return fail(EM_E_NOMEM, "cudaMalloc of %zu bytes failed (injected by em_fail_allocation)",
                        count * sizeof(T));
        if (cudaMalloc(&p, std::max<size_t>(count, 1) * sizeof(T)) != cudaSuccess) {
            cudaGetLastError();
            p = nullptr;
            return fail(EM_E_NOMEM, "cudaMalloc of %zu bytes failed", count * sizeof(T));
        }
        cap = count;
        return EM_OK;
    }
    void release() {
        if (p) cudaFree(p);
        p = nullptr;
        cap = 0;
    }
};

struct em_model {
    int dev = 0, sms = 148;
    long long wait_cycles = 0;
    cudaStream_t stream = nullptr;
    bool own_stream = false;
    int64_t d = 0, k = 0;
    int ld = 0, nv = 0, kc = 64;
    uint64_t seed = 1234;
    // options
    int64_t opt_batch = 0;
    double opt_alpha0 = 0.0, tau = -1.0, wait_ms = 2000.0;  // tau < 0: the default for d
    int revival = EM_REVIVE_SPLIT, finalize = 1, law = 2, in_dtype = 0, check_finite = 0;
    int auto_revive = 1, capture = 1, graphs = 1, assign_kernel = 0, exact_ties = -1;
    int spherical = 0;  // spherical e-means: unit centroids, highest dot product
    int pdl = 1;        // EM_OPT_PDL: programmatic dependent launch of the step's kernels
    // FP8 search (EM_OPT_SEARCH_FORMAT = 1): the converter fitted at em_begin /
    // em_lloyd (shift per dimension, power-of-two scale) and the E4M3 operand
    int fp8 = 0;
    int ld8 = 0;           // bytes per E4M3 row: d rounded up to 16
    bool fp8_ready = false;
    float fp8_scale = 1.0f;
    DBuf<float> fp8_shift;  // ld values (zero past d)
    DBuf<float> fp8_lohi, fp8_part;
    DBuf<uint8_t> cq8, X8full;
    DBuf<float> cn8, xn8full;
    CUtensorMap tm_cq8;
    // data parallelism (em_dp_init): this rank's share of each batch, statistics
    // added across ranks with NCCL
    int dp_world = 1, dp_rank = 0;
    ncclComm_t comm = nullptr;
    DBuf<double> stats;  // k x ld sums, k counts, the error sum
    int last_split = 1;  // centroid-tile groups of the most recent search (keys per row)
    // state
    DBuf<float> N, N_prev, S, c, cn, cnp;
    DBuf<__nv_bfloat16> cq;
    DBuf<__nv_bfloat16> cn3, ones3;  // the folded search's norms (k x 16) and ones (128 x 16) operands
    DBuf<double> close_sum, close_cnt;
    DBuf<int> err, flag;
    // data of the current run
    const __nv_bfloat16* X = nullptr;
    int64_t n = 0;        // rows of a pass over all ranks (the recipe's n)
    int64_t n_local = 0;  // rows in X (this rank's share in a data-parallel run)
    DBuf<__nv_bfloat16> Xown;
    DBuf<uint8_t> stage;  // host-input staging
    // batch buffers
    int64_t bcap = 0;
    int R = 32;
    // The rows of step t live in slot t & 1. While step t runs its update and
    // revival on the model's stream, the rows of step t + 1 are gathered into the
    // other slot on the side stream (EM_OPT_PREFETCH).
    struct BatchSlot {
        DBuf<__nv_bfloat16> X;  // the batch rows, bf16
        DBuf<float> xn;         // their |x|^2
        DBuf<int32_t> ids;      // their data row ids
        CUtensorMap tm;         // search operand map over X
        DBuf<uint8_t> X8;       // FP8 search: the rows' E4M3 codes (pitch ld8 bytes)
        DBuf<float> xn8;        // and their |x'|^2
        CUtensorMap tm8;
    };
    BatchSlot slot[2];
    int prefetch = 1;
    int64_t ready = -1;        // step whose rows are in slot[ready & 1] (gathered or in flight); -1: none
    bool ready_synced = true;  // the model's stream is already ordered after that gather
    bool capturing = false;    // a step range is being captured into a graph
    cudaStream_t side = nullptr, side_cap = nullptr;
    cudaEvent_t ev_fork = nullptr, ev_sel = nullptr, ev_gathered[2] = {nullptr, nullptr};
    DBuf<float> xn, dists;  // xn: |x|^2 of a full pass (assign, MSE, Lloyd)
    DBuf<int32_t> labels, cnt, rank, off, poff, perm;
    DBuf<int4> items;
    DBuf<unsigned long long> keys;
    DBuf<double> block_err, part, step_err, scalar;
    DBuf<int64_t> labels_last, labels64;
    // revival scratch
    DBuf<int32_t> rv_dead, rv_donor, rv_order, rv_times, rv_ndead;
    DBuf<double> rv_tree, rv_target;
    DBuf<int4> ties;          // near-tie rows waiting for k_settle
    DBuf<int> tie_n;          // their number
    DBuf<double> tie_corr;    // error-sum change of the rows k_settle relabels
    DBuf<int64_t> rv_splits;
    // run progress
    em_recipe_t rec{};
    bool running = false, have_run = false;
    int64_t t = 0, pass = 0, pos = 0, rows_assigned = 0;
    int64_t last_rows = 0;
    double last_alpha = 0.0;
    int last_was_lloyd = 0;
    CUtensorMap tm_cq;
    CUtensorMap tm_cn3, tm_ones3;
    // profiling (EM_OPT_PROFILE) and launch counting
    int profile = 0;
    int64_t launches = 0;
    struct Span {
        int phase;
        cudaEvent_t a, b;
        double flops, bytes;
    };
    std::vector<Span> pending;
    std::vector<cudaEvent_t> pool;
    em_profile_t totals{};
    // CUDA graphs of step ranges (EM_OPT_GRAPHS), keyed by everything they bake in
    struct GraphEntry {
        std::vector<uint64_t> sig;
        int64_t t0, count, launches;
        cudaGraphExec_t exec;
    };
    std::vector<GraphEntry> graph_cache;
    cudaStream_t cap_stream = nullptr;
};

// Opens an event span of `phase` on the model's stream (-1 when profiling is off).
static int span_begin(em_model* m, int phase) {
    if (!m->profile) return -1;
    cudaEvent_t ev[2];
    for (int i = 0; i < 2; ++i) {
        if (!m->pool.empty()) {
            ev[i] = m->pool.back();
            m->pool.pop_back();
        } else if (cudaEventCreate(&ev[i]) != cudaSuccess) {
            cudaGetLastError();
            return -1;
        }
    }
    cudaEventRecord(ev[0], m->stream);
    m->pending.push_back({phase, ev[0], ev[1], 0.0, 0.0});
    return (int)m->pending.size() - 1;
}

static void span_end(em_model* m, int idx, double flops = 0.0, double bytes = 0.0) {
    if (idx < 0) return;
    em_model::Span& sp = m->pending[idx];
    sp.flops = flops;
    sp.bytes = bytes;
    cudaEventRecord(sp.b, m->stream);
}

#define EM_LAUNCHED(m, count) ((m)->launches += (count))

static int set_device(const em_model* m) {
    CK(cudaSetDevice(m->dev));
    return EM_OK;
}

static int check_device_errors(em_model* m) {
    if (m->side) CK(cudaStreamSynchronize(m->side));  // a prefetch gather also reports here
    int h = 0;
    CK(cudaMemcpyAsync(&h, m->err.p, sizeof(int), cudaMemcpyDeviceToHost, m->stream));
    CK(cudaStreamSynchronize(m->stream));
    if (h != 0) {
        CK(cudaMemsetAsync(m->err.p, 0, sizeof(int), m->stream));
        CK(cudaStreamSynchronize(m->stream));
        return fail(h, h == EM_E_TIMEOUT ? "a device-side wait exceeded its limit"
                                         : "a kernel's index check failed (device error %d)",
                    h);
    }
    return EM_OK;
}

static bool is_device_ptr(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

static int grid_for(int64_t work, int block, int sms, int per_sm = 8) {
    int64_t g = (work + block - 1) / block;
    g = std::min<int64_t>(g, (int64_t)sms * per_sm);
    return (int)std::max<int64_t>(g, 1);
}

// Makes a bf16 n x ld device copy of X (or uses X in place). *out receives the
// row source the kernels read.
static int prepare_input(em_model* m, const void* X, int64_t n, DBuf<__nv_bfloat16>& own,
                         const __nv_bfloat16** out) {
    if (!X || n < 1) return fail(EM_E_INVAL, "X is NULL or n < 1");
    const bool dev = is_device_ptr(X);
    const size_t esz = m->in_dtype == 1 ? 2 : 4;
    const size_t raw_bytes = (size_t)n * (size_t)m->d * esz;
    const void* src = X;
    if (!dev) {  // host input: copy to the device first
        CKR(m->stage.ensure(raw_bytes));
        CK(cudaMemcpyAsync(m->stage.p, X, raw_bytes, cudaMemcpyHostToDevice, m->stream));
        src = m->stage.p;
    }
    if (m->check_finite) {
        CK(cudaMemsetAsync(m->flag.p, 0, sizeof(int), m->stream));
        k_check_finite<<<grid_for(n * m->d, 256, m->sms), 256, 0, m->stream>>>(src, n * m->d, m->in_dtype == 1,
                                                                                m->flag.p);
        CK(cudaGetLastError());
        int h = 0;
        CK(cudaMemcpyAsync(&h, m->flag.p, sizeof(int), cudaMemcpyDeviceToHost, m->stream));
        CK(cudaStreamSynchronize(m->stream));
        if (h) return fail(EM_E_NONFINITE, "input holds NaN or infinite values");
    }
    if (m->in_dtype == 1 && m->ld == m->d && (reinterpret_cast<uintptr_t>(src) & 15) == 0) {
        *out = reinterpret_cast<const __nv_bfloat16*>(src);
        return EM_OK;
    }
    CKR(own.ensure((size_t)n * m->ld));
    if (m->in_dtype == 1) {
        k_pad_bf16<<<grid_for(n * m->ld, 256, m->sms), 256, 0, m->stream>>>(
            reinterpret_cast<const __nv_bfloat16*>(src), n, (int)m->d, m->ld, own.p);
    } else {
        const int vec_ok = (m->d % 4 == 0) && ((reinterpret_cast<uintptr_t>(src) & 15) == 0);
        k_cast_f32_bf16<<<grid_for(n * m->nv, 256, m->sms), 256, 0, m->stream>>>(
            reinterpret_cast<const float*>(src), n, (int)m->d, m->ld, own.p, vec_ok);
    }
    CK(cudaGetLastError());
    EM_LAUNCHED(m, 1);
    *out = own.p;
    return EM_OK;
}

static ClusterState cluster_state(em_model* m) {
    ClusterState st;
    st.N = m->N.p;
    st.N_prev = m->N_prev.p;
    st.cnp = m->cnp.p;
    st.k = (int)m->k;
    st.S = m->S.p;
    st.c = m->c.p;
    st.cq = m->cq.p;
    st.cn = m->cn.p;
    st.close_sum = m->close_sum.p;
    st.close_cnt = m->close_cnt.p;
    st.ld = m->ld;
    return st;
}

static int ensure_batch_buffers(em_model* m, int64_t cap) {
    m->R = kChunkRows;
    const int64_t max_items = m->k + (cap + m->R - 1) / m->R;
    CKR(m->xn.ensure(cap));
    CKR(m->dists.ensure(cap));
    CKR(m->labels.ensure(cap));
    CKR(m->rank.ensure(cap));
    CKR(m->perm.ensure(cap));
    CKR(m->keys.ensure(cap));
    CKR(m->ties.ensure(cap));
    CKR(m->cnt.ensure(m->k));
    CKR(m->off.ensure(m->k + 1));
    CKR(m->poff.ensure(m->k + 1));
    CKR(m->items.ensure(max_items));
    CKR(m->block_err.ensure((cap + 255) / 256 + 1));
    CKR(m->part.ensure((size_t)max_items * m->ld));
    m->bcap = cap;
    return EM_OK;
}

// Work units of the search over m_tiles row tiles and n_tiles centroid tiles on
// `sms` persistent CTAs. A row tile split into s groups is s units, each keeping
// its own running minimum per row, and the epilogue's cost grows with the new
// minima it meets; so splitting is used only where it shortens the longest CTA,
// either for every row tile or, once the row tiles have filled whole waves, only
// for those of the last wave (the first m_full row tiles stay whole). Candidates
// are taken in order of split units; a later one wins only if its longest CTA
// (in centroid tiles) is at least 1.5 % shorter.
struct Schedule {
    int split;
    int m_full;
};

static Schedule choose_schedule(int64_t m_tiles, int64_t n_tiles, int sms, int max_split = 8) {
    struct Cand {
        double cost;
        int64_t split_units;
        Schedule s;
    };
    Cand c[8];
    int nc = 0;
    const int64_t waves = m_tiles / sms, m_full = waves * sms, rest = m_tiles - m_full;
    for (int s = 1; s <= 8; s <<= 1) {
        if (s > n_tiles || s > max_split) break;
        const int64_t tpg = (n_tiles + s - 1) / s;
        c[nc++] = Cand{(double)(((m_tiles * s + sms - 1) / sms) * tpg), s > 1 ? m_tiles * s : 0, Schedule{s, 0}};
        if (s > 1 && m_full > 0 && rest > 0)
            c[nc++] = Cand{(double)(waves * n_tiles + ((rest * s + sms - 1) / sms) * tpg), rest * s,
                           Schedule{s, (int)m_full}};
    }
    std::stable_sort(c, c + nc, [](const Cand& a, const Cand& b) { return a.split_units < b.split_units; });
    Cand best = c[0];
    for (int i = 1; i < nc; ++i)
        if (c[i].cost < best.cost * 0.985) best = c[i];
    return best.s;
}

// Whether the search keeps the best two (score, index) keys per key set, so that
// near ties can be settled exactly afterwards.
static bool use_top2(const em_model* m) {
    if (m->fp8) return false;  // the FP8 search keeps the plain argmin (no exact settling of ties)
    return m->exact_ties == 1 || (m->exact_ties < 0 && m->d >= 256);
}

static Schedule schedule_for(const em_model* m, int64_t rows) {
    const int64_t m_tiles = (rows + tc::BM - 1) / tc::BM;
    const int64_t n_tiles = (m->k + tc::BN - 1) / tc::BN;
    return choose_schedule(m_tiles, n_tiles, m->sms);
}

// Keys the search writes for `rows` rows: two per row per key set, two key sets
// (column halves) per centroid-tile group.
static size_t keys_needed(const em_model* m, int64_t rows) {
    return rows > 0 ? (size_t)schedule_for(m, rows).split * tc::kKeySets * (size_t)rows * 2 : 0;
}

static TieList tie_list(em_model* m) { return TieList{m->ties.p, m->tie_n.p, m->tie_corr.p}; }

// Value of a training row (labels kernel): its squared distance, or its spherical error.
static int training_kind(const em_model* m) { return m->spherical ? kSphericalError : kSquaredDistance; }

// After every change of the centroids: spherical e-means rescales each to norm 1
// (README "Spherical e-means"), and the FP8 search rebuilds its E4M3 operand.
static int after_centroid_change(em_model* m);

// How the labels kernels turn a search score into a squared distance.
static ScoreScale score_scale(const em_model* m) {
    return m->fp8 ? ScoreScale{2.0f, 1.0f / (m->fp8_scale * m->fp8_scale), -1.0f} : ScoreScale{1.0f, 1.0f, kTieRel};
}

// Settles the near ties the label kernel of `rows` rows queued (a no-op launch when
// there are none): one warp per row over a fixed grid.
static int launch_settle(em_model* m, const __nv_bfloat16* A, const float* xn, int32_t* labels32, int64_t* labels64,
                         float* dists, bool count, const int32_t* ids, int64_t* labels_last, int capture) {
    const int kind = (count || !m->spherical) ? training_kind(m) : kSimilarity;
    launch_k(m->pdl, k_settle, m->sms * EM_SETTLE_BLOCKS_PER_SM, 256, 0, m->stream, tie_list(m), xn, A, m->ld, m->cq.p, labels32,
                                                                    labels64, dists,
                                                count ? m->cnt.p : nullptr, m->rank.p, ids, labels_last, capture,
                                                kind);
    CK(cudaGetLastError());
    EM_LAUNCHED(m, 1);
    return EM_OK;
}

// Every variant of the search kernel: KC (64 or 32 columns per K chunk), TOP2 (keep
// the two best), AST (the batch tile stays in shared memory for a whole work unit;
// rows of at most 128 dims).
static bool ast_fits(int64_t d, int kc) {
    const int64_t nkc = (d + kc - 1) / kc;
    return nkc * tc::BM * kc * 2 <= tc::kAstBufBytes;
}

// Whether the folded-norm search fits: with its norms tile beside the nkc chunks, a
// centroid tile must still leave two stages in the ring.
static bool fold_fits(int kc, int nkc) {
    const int ring = kc == 64 ? tc::Cfg<64, true, 2, true>::kStages * tc::Cfg<64, true, 2, true>::kBBytes
                              : tc::Cfg<32, true, 2, true>::kStages * tc::Cfg<32, true, 2, true>::kBBytes;
    const int tile = nkc * tc::BN * kc * 2 + tc::kExtBBytes;
    return ring / tile >= 2;
}

// tmN / tmO: the norms and ones operands of the folded search (fold), else unused.
static void launch_search(int kc, bool top2, bool ast, int grid, cudaStream_t stream, const CUtensorMap& tmA,
                          const CUtensorMap& tmB, const float* cn, int k, int rows, int nkc, int n_tiles, Schedule sc,
                          unsigned long long* keys, long long wait, int* err, bool f8 = false, bool pdl = false,
                          bool fold = false, const CUtensorMap* tmN = nullptr, const CUtensorMap* tmO = nullptr) {
    const int split = sc.split, m_full = sc.m_full;
    const CUtensorMap& tn = tmN ? *tmN : tmB;
    const CUtensorMap& to = tmO ? *tmO : tmB;
#define EM_GO(KC, T2, AST, FD)                                                                              \
    launch_k(pdl, tc::k_assign_tc<KC, T2, AST, false, FD>, grid, tc::threads_for<tc::epi_groups<T2, AST>()>(), \
             tc::Cfg<KC, AST, tc::epi_groups<T2, AST>(), FD>::kSmemBytes, stream, tmA, tmB, tn, to, cn, k, rows, \
             nkc, n_tiles, split, m_full, keys, wait, err)
    if (f8) {  // E4M3 rows and operand, 128-code chunks, plain argmin
        if (ast)
            launch_k(pdl, tc::k_assign_tc<64, false, true, true>, grid, tc::threads_for<tc::epi_groups<false, true>()>(),
                     tc::Cfg<64, true, tc::epi_groups<false, true>()>::kSmemBytes, stream, tmA, tmB, tn, to, cn, k, rows,
                     nkc, n_tiles, split, m_full, keys, wait, err);
        else
            launch_k(pdl, tc::k_assign_tc<64, false, false, true>, grid, tc::kThreads, tc::Cfg<64, false>::kSmemBytes,
                     stream, tmA, tmB, tn, to, cn, k, rows, nkc, n_tiles, split, m_full, keys, wait, err);
        return;
    }
    if (kc == 64) {
        if (top2) {
            if (ast) EM_GO(64, true, true, false); else EM_GO(64, true, false, false);
        } else {
            if (ast && fold) EM_GO(64, false, true, true);
            else if (ast) EM_GO(64, false, true, false);
            else EM_GO(64, false, false, false);
        }
    } else {
        if (top2) {
            if (ast) EM_GO(32, true, true, false); else EM_GO(32, true, false, false);
        } else {
            if (ast && fold) EM_GO(32, false, true, true);
            else if (ast) EM_GO(32, false, true, false);
            else EM_GO(32, false, false, false);
        }
    }
#undef EM_GO
}

static bool search_smem_attributes() {
#define EM_ATTR(KC, T2, AST, FD)                                                                            \
    (cudaFuncSetAttribute(tc::k_assign_tc<KC, T2, AST, false, FD>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                          tc::Cfg<KC, AST, tc::epi_groups<T2, AST>(), FD>::kSmemBytes) == cudaSuccess)
    return EM_ATTR(64, false, false, false) && EM_ATTR(64, true, false, false) && EM_ATTR(32, false, false, false) &&
           EM_ATTR(32, true, false, false) && EM_ATTR(64, false, true, false) && EM_ATTR(64, true, true, false) &&
           EM_ATTR(32, false, true, false) && EM_ATTR(32, true, true, false) && EM_ATTR(64, false, true, true) &&
           EM_ATTR(32, false, true, true) &&
           cudaFuncSetAttribute(tc::k_assign_tc<64, false, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                tc::Cfg<64, false>::kSmemBytes) == cudaSuccess &&
           cudaFuncSetAttribute(tc::k_assign_tc<64, false, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                tc::Cfg<64, true, tc::epi_groups<false, true>()>::kSmemBytes) == cudaSuccess;
#undef EM_ATTR
}

// Nearest-centroid search of `rows` rows described by tmA (row source A for the
// SIMT path) into m->keys. Every key set the label kernel reads is written.
static int launch_assign(em_model* m, const CUtensorMap& tmA, const __nv_bfloat16* A, int64_t rows) {
    if (rows <= 0) return EM_OK;
    if (m->keys.cap < keys_needed(m, rows)) return fail(EM_E_STATE, "search key buffer too small");
    if (m->assign_kernel == 1) {
        k_assign_simt<<<(int)((rows + 127) / 128), 128, 0, m->stream>>>(A, m->ld, (int)rows, m->cq.p, m->cn.p,
                                                                         (int)m->k, (int)m->d, m->keys.p);
        CK(cudaGetLastError());
        EM_LAUNCHED(m, 1);
        m->last_split = 1;
        return EM_OK;
    }
    const int64_t m_tiles = (rows + tc::BM - 1) / tc::BM;
    const int64_t n_tiles = (m->k + tc::BN - 1) / tc::BN;
    const Schedule sc = schedule_for(m, rows);
    const int64_t units = sc.m_full + (m_tiles - sc.m_full) * sc.split;
    const int grid = (int)std::min<int64_t>(units, m->sms);
    if (m->fp8) {  // tmA maps E4M3 rows; chunks of 128 codes
        const int nkc8 = (int)((m->d + 127) / 128);
        const bool ast8 = (int64_t)nkc8 * tc::BM * 128 <= tc::kAstBufBytes;
        launch_search(64, false, ast8, grid, m->stream, tmA, m->tm_cq8, m->cn8.p, (int)m->k, (int)rows, nkc8,
                      (int)n_tiles, sc, m->keys.p, m->wait_cycles, m->err.p, true, m->pdl != 0);
    } else {
        const int nkc = (int)((m->d + m->kc - 1) / m->kc);
        const bool top2 = use_top2(m), ast = ast_fits(m->d, m->kc);
        // the folded search takes |c~|^2 from the MMAs: its norms operand is refreshed first
        // (one more launch, so only where the tiles are many enough for the epilogue to
        // matter)
        const bool fold = ast && !top2 && fold_fits(m->kc, nkc) && n_tiles >= 4 && m_tiles * n_tiles >= 4 * m->sms;
        if (fold) {
            launch_k(m->pdl, tc::k_fold_norms, grid_for(n_tiles * tc::BN, 256, m->sms), 256, 0, m->stream, m->cn.p,
                     (int)m->k, (int)(n_tiles * tc::BN), m->cn3.p);
            EM_LAUNCHED(m, 1);
        }
        launch_search(m->kc, top2, ast, grid, m->stream, tmA, m->tm_cq, m->cn.p, (int)m->k, (int)rows, nkc,
                      (int)n_tiles, sc, m->keys.p, m->wait_cycles, m->err.p, false, m->pdl != 0, fold, &m->tm_cn3,
                      &m->tm_ones3);
    }
    CK(cudaGetLastError());
    EM_LAUNCHED(m, 1);
    m->last_split = sc.split * tc::kKeySets;
    return EM_OK;
}

static int launch_select(em_model* m, int64_t t, cudaStream_t stream, bool pdl, CountSource src);

// Group rows by label and apply the EMA update (k_offsets .. k_clusters); labels,
// ranks and counts are already in place. `src` holds the rows (batch or data).
static int launch_reduce(em_model* m, const __nv_bfloat16* src, int64_t rows, int nblocks_labels, double alpha,
                         int last_pass, double* err_sum_out, int64_t select_t = -1) {
    const bool dp = m->comm != nullptr;
    double* const stats_err = m->stats.p + (int64_t)m->k * m->ld + m->k;
    const StepParams sp{alpha, last_pass, 0, dp ? m->stats.p : nullptr};
    double* const step_err = err_sum_out;
    if (dp) err_sum_out = stats_err;  // the error sum travels with the statistics
    launch_k(m->pdl, k_offsets, 1, 1024, 0, m->stream, m->cnt.p, (int)m->k, (int)rows, m->R, m->off.p, m->poff.p, m->block_err.p,
                                         nblocks_labels, err_sum_out, tie_list(m), m->err.p);
    CK(cudaGetLastError());
    if (select_t >= 0) {
        // The revival check after this step: its donor selection needs only the new
        // running counts, which follow from N_prev and the segment sizes k_offsets
        // has just written, so it runs on the side stream beside the segmented
        // sums; the model's stream waits for it before the splits (launch_revive).
        cudaStream_t side = m->capturing ? m->side_cap : m->side;
        CK(cudaEventRecord(m->ev_fork, m->stream));
        CK(cudaStreamWaitEvent(side, m->ev_fork, 0));
        CKR(launch_select(m, select_t, side, false, CountSource{nullptr, m->N_prev.p, m->off.p, alpha}));
        CK(cudaEventRecord(m->ev_sel, side));
    }
    launch_k(m->pdl, k_scatter, (int)((rows + 255) / 256), 256, 0, m->stream, m->labels.p, m->rank.p, m->off.p, m->poff.p,
                                                                 (int)rows, m->R, m->perm.p, m->items.p, m->err.p);
    CK(cudaGetLastError());
    const ClusterState st = cluster_state(m);
    const int64_t max_items = m->k + (rows + m->R - 1) / m->R;
    const int nslices = (m->nv + 31) / 32;
    const int seg_blocks = (int)((max_items * nslices * 32 + 255) / 256);
    launch_k(m->pdl, k_segsum, seg_blocks, 256, 8 * kSegsumDepth * 32 * 16, m->stream, src, m->perm.p, m->items.p, m->poff.p, nslices, m->nv, st, sp,
                                                m->part.p);
    launch_k(m->pdl, k_clusters, grid_for(m->k * 32, EM_CLUSTERS_BLOCK, m->sms, 16), EM_CLUSTERS_BLOCK, 0, m->stream, 
        m->off.p, m->poff.p, m->cnt.p, m->R, nslices,
                                                                         m->nv, st, sp, m->part.p);
    CK(cudaGetLastError());
    EM_LAUNCHED(m, 4);
    if (dp) {  // add the ranks' statistics, then the same update on every rank
        NCK(nccl().all_reduce(m->stats.p, m->stats.p, (size_t)m->k * m->ld + m->k + 1, ncclFloat64, ncclSum, m->comm,
                              m->stream));
        launch_k(m->pdl, k_apply_stats, grid_for(m->k * 32, 256, m->sms), 256, 0, m->stream, nslices, m->nv, st, sp, step_err);
        CK(cudaGetLastError());
        EM_LAUNCHED(m, 1);
    }
    return after_centroid_change(m);
}

static ReviveScratch revive_scratch(em_model* m) {
    ReviveScratch sc;
    sc.dead = m->rv_dead.p;
    sc.donor = m->rv_donor.p;
    sc.order = m->rv_order.p;
    sc.times = m->rv_times.p;
    sc.tree = m->rv_tree.p;
    sc.target = m->rv_target.p;
    sc.ndead = m->rv_ndead.p;
    sc.n_splits = m->rv_splits.p;
    return sc;
}

// The defaults that depend on the dimension (README `batch_law`, `unused_threshold`
// and "Note on low dimension"): the quality batch law for d <= 16, no revival for
// d <= 2.
static int effective_law(const em_model* m) { return m->law == 2 ? (m->d <= 16 ? 1 : 0) : m->law; }
static double effective_tau(const em_model* m) { return m->tau < 0.0 ? (m->d <= 2 ? 0.0 : 0.1) : m->tau; }

static bool revival_on(const em_model* m) { return m->revival != EM_REVIVE_NONE && effective_tau(m) > 0.0; }

// Shared memory the donor selection kernels may take (the tree and the split counters).
static bool select_smem_attributes() {
    const int b = kReviveSmemBytes;
    const cudaFuncAttribute a = cudaFuncAttributeMaxDynamicSharedMemorySize;
    return cudaFuncSetAttribute(k_revive_select, a, b) == cudaSuccess &&
           cudaFuncSetAttribute(k_revive_select_flat<1, 1>, a, b) == cudaSuccess &&
           cudaFuncSetAttribute(k_revive_select_flat<1, 2>, a, b) == cudaSuccess &&
           cudaFuncSetAttribute(k_revive_select_flat<1, 4>, a, b) == cudaSuccess &&
           cudaFuncSetAttribute(k_revive_select_flat<2, 4>, a, b) == cudaSuccess &&
           cudaFuncSetAttribute(k_revive_select_flat<4, 4>, a, b) == cudaSuccess &&
           cudaFuncSetAttribute(k_revive_select_wide<1>, a, b) == cudaSuccess &&
           cudaFuncSetAttribute(k_revive_select_wide<2>, a, b) == cudaSuccess &&
           cudaFuncSetAttribute(k_revive_select_wide<4>, a, b) == cudaSuccess &&
           cudaFuncSetAttribute(k_revive_select_wide<8>, a, b) == cudaSuccess;
}

// The donor selection of the revival check after step t, on `stream`, reading the
// running counts from `src`.
static int launch_select(em_model* m, int64_t t, cudaStream_t stream, bool pdl, CountSource src) {
    const ReviveScratch sc = revive_scratch(m);
    const int k = (int)m->k;
    const double tau = effective_tau(m);
    // two-level trees (group size 32 S0, root of at most 32 SR entries) up to kFastK
    if (k <= 1024)
        launch_k(pdl, k_revive_select_flat<1, 1>, 1, kSelectThreads, flat_smem_bytes<1>(k), stream, src, k, tau,
                 m->seed, t, m->revival, sc);
    else if (k <= 2048)
        launch_k(pdl, k_revive_select_flat<1, 2>, 1, kSelectThreads, flat_smem_bytes<1>(k), stream, src, k, tau,
                 m->seed, t, m->revival, sc);
    else if (k <= 4096)
        launch_k(pdl, k_revive_select_flat<1, 4>, 1, kSelectThreads, flat_smem_bytes<1>(k), stream, src, k, tau,
                 m->seed, t, m->revival, sc);
    else if (k <= 8192)
        launch_k(pdl, k_revive_select_flat<2, 4>, 1, kSelectThreads, flat_smem_bytes<2>(k), stream, src, k, tau,
                 m->seed, t, m->revival, sc);
    else if (k <= kFastK)
        launch_k(pdl, k_revive_select_flat<4, 4>, 1, kSelectThreads, flat_smem_bytes<4>(k), stream, src, k, tau,
                 m->seed, t, m->revival, sc);
    // level 0 in global memory, prefetched ahead of the draws, up to kWideK
    else if (k <= kWideK && wide_root_slots(k) == 1)
        launch_k(pdl, k_revive_select_wide<1>, 1, kSelectThreads, wide_smem_bytes(k), stream, src, k, tau, m->seed,
                 t, m->revival, sc);
    else if (k <= kWideK && wide_root_slots(k) == 2)
        launch_k(pdl, k_revive_select_wide<2>, 1, kSelectThreads, wide_smem_bytes(k), stream, src, k, tau, m->seed,
                 t, m->revival, sc);
    else if (k <= kWideK && wide_root_slots(k) == 4)
        launch_k(pdl, k_revive_select_wide<4>, 1, kSelectThreads, wide_smem_bytes(k), stream, src, k, tau, m->seed,
                 t, m->revival, sc);
    else if (k <= kWideK)
        launch_k(pdl, k_revive_select_wide<8>, 1, kSelectThreads, wide_smem_bytes(k), stream, src, k, tau, m->seed,
                 t, m->revival, sc);
    else
        launch_k(pdl, k_revive_select, 1, kSelectThreads, (int)tree_smem_bytes(tree_layout(k), k), stream, src, k,
                 tau, m->seed, t, m->revival, sc, m->err.p);
    CK(cudaGetLastError());
    EM_LAUNCHED(m, 1);
    return EM_OK;
}

// The revival check after step t. `selected`: its donor selection already ran
// (beside the step's update; launch_reduce), and the model's stream waits for it.
static int launch_revive(em_model* m, int64_t t, int64_t rows, const __nv_bfloat16* Xb, bool selected = false) {
    if (!revival_on(m)) return EM_OK;
    const ReviveScratch sc = revive_scratch(m);
    if (selected)
        CK(cudaStreamWaitEvent(m->stream, m->ev_sel, 0));
    else
        CKR(launch_select(m, t, m->stream, m->pdl != 0, CountSource{m->N.p, nullptr, nullptr, 0.0}));
    const ClusterState st = cluster_state(m);
    const int blocks = grid_for(m->k * 32, 256, m->sms);
    if (m->revival == EM_REVIVE_SPLIT) {
        launch_k(m->pdl, k_revive_dead, blocks, 256, 0, m->stream, st, m->nv, sc);
        launch_k(m->pdl, k_revive_donors, blocks, 256, 0, m->stream, st, m->nv, sc);
        EM_LAUNCHED(m, 2);
    } else {
        launch_k(m->pdl, k_revive_resample, blocks, 256, 0, m->stream, st, m->nv, sc, Xb, (int)rows, m->seed, t);
        EM_LAUNCHED(m, 1);
    }
    CK(cudaGetLastError());
    return after_centroid_change(m);
}

// One training step of the current run: what it does (host-side plan), the
// kernels it launches, and the host bookkeeping after it.
struct StepPlan {
    int64_t t, pass, pos, rows;
    int last_pass, revive;
    double alpha;
};

// Step t of a run whose recipe is `rec` over n rows (all ranks' rows in a data-
// parallel run), at row `pos` of pass `pass`. Host code only: em_dp_schedule runs
// it without a model.
static StepPlan plan_rows(const em_recipe_t& rec, int64_t n, bool auto_revive, int64_t t, int64_t pass,
                          int64_t pos) {
    StepPlan p;
    const int64_t rows_pass = (pass == rec.passes - 1) ? rec.rows_last_pass : n;
    p.t = t;
    p.pass = pass;
    p.pos = pos;
    p.rows = std::min<int64_t>(rec.batch_size, rows_pass - pos);
    p.last_pass = (pass == rec.passes - 1) ? 1 : 0;
    p.alpha = alpha_at(t, rec.total_steps, rec.alpha0);
    p.revive = (auto_revive && (t + 1) % kReviveEvery == 0) ? 1 : 0;
    return p;
}

// The step after p: the next batch of the pass, or the first of the next pass.
static StepPlan plan_next(const em_recipe_t& rec, int64_t n, bool auto_revive, const StepPlan& p) {
    const int64_t rows_pass = (p.pass == rec.passes - 1) ? rec.rows_last_pass : n;
    int64_t pass = p.pass, pos = p.pos + p.rows;
    if (pos >= rows_pass) {
        pass += 1;
        pos = 0;
    }
    return plan_rows(rec, n, auto_revive, p.t + 1, pass, pos);
}

static StepPlan plan_at(const em_model* m, int64_t t, int64_t pass, int64_t pos) {
    return plan_rows(m->rec, m->n, m->auto_revive != 0, t, pass, pos);
}

static StepPlan plan_step(const em_model* m) { return plan_at(m, m->t, m->pass, m->pos); }

// The step after p (same rules as advance_step).
static StepPlan plan_after(const em_model* m, const StepPlan& p) {
    return plan_next(m->rec, m->n, m->auto_revive != 0, p);
}

// A rank's share of step p's batch (README "Several GPUs": every rank walks its own
// rows in its own per-pass order and takes an even share of each batch): positions
// [pos / world, (pos + rows) / world) of its order, whose key is the pass plus
// rank * 2^32 (rank 0: the single-GPU order).
struct RankShare {
    int64_t first, rows, key;
};

static RankShare rank_share(const StepPlan& p, int64_t world, int64_t rank) {
    return RankShare{p.pos / world, p.rows / world, p.pass + (rank << 32)};
}

// README "Several GPUs": the batch and the rows of every pass divide by the ranks.
static int check_dp_recipe(const em_recipe_t& rec, int64_t world) {
    if (world > 1 && (rec.batch_size % world || rec.rows_last_pass % world))
        return fail(EM_E_INVAL, "the batch (%lld rows) and the rows of every pass (last: %lld) must divide by "
                                "the number of ranks (%lld)",
                    (long long)rec.batch_size, (long long)rec.rows_last_pass, (long long)world);
    return EM_OK;
}

// Whether step t gathers the rows of step t + 1 on the side stream.
static bool prefetches(const em_model* m, int64_t t) {
    return m->prefetch && !m->profile && t + 1 < m->rec.total_steps;
}

// Gathers this rank's rows of step p into slot p.t & 1 on `stream`. A rank takes
// the positions [pos / world, (pos + rows) / world) of its own order of its own
// rows; rank r's order is keyed by the pass plus r * 2^32 (rank 0: the single-GPU
// order).
static int launch_gather(em_model* m, const StepPlan& p, cudaStream_t stream) {
    em_model::BatchSlot& b = m->slot[p.t & 1];
    const RankShare sh = rank_share(p, m->dp_world, m->dp_rank);
    const int64_t rows = sh.rows;
    const int64_t key = sh.key;
    if (m->fp8) {
        const Fp8Out f8{b.X8.p, b.xn8.p, m->fp8_shift.p, m->fp8_scale, m->ld8, (int)m->d};
        launch_k(m->pdl, k_gather<true>, grid_for(rows, 128, m->sms), 128, 0, stream, 
            m->X, m->n_local, m->ld, m->seed, key, sh.first, (int)rows, 0, b.X.p, b.xn.p, b.ids.p, m->err.p, f8);
    } else {
        launch_k(m->pdl, k_gather<false>, grid_for(rows, 128, m->sms), 128, 0, stream, 
            m->X, m->n_local, m->ld, m->seed, key, sh.first, (int)rows, 0, b.X.p, b.xn.p, b.ids.p, m->err.p,
            Fp8Out{});
    }
    CK(cudaGetLastError());
    EM_LAUNCHED(m, 1);
    return EM_OK;
}

// Makes the rows of step p available to the model's stream: gathers them there, or
// orders the stream after the side-stream gather that a previous step started.
static int prime_batch(em_model* m, const StepPlan& p) {
    if (m->ready != p.t) {
        CKR(launch_gather(m, p, m->stream));
        m->ready = p.t;
    } else if (!m->ready_synced) {
        CK(cudaStreamWaitEvent(m->stream, m->ev_gathered[p.t & 1], 0));
    }
    m->ready_synced = true;
    return EM_OK;
}

// Orders the model's stream after any side-stream gather still in flight and
// forgets the prefetched rows (before buffers change or a run is repositioned).
static int drop_prefetch(em_model* m) {
    if (m->ready >= 0 && !m->ready_synced) CK(cudaStreamWaitEvent(m->stream, m->ev_gathered[m->ready & 1], 0));
    m->ready = -1;
    m->ready_synced = true;
    return EM_OK;
}

static void advance_step(em_model* m, const StepPlan& p) {
    const int64_t rows_pass = (m->pass == m->rec.passes - 1) ? m->rec.rows_last_pass : m->n;
    m->last_rows = rank_share(p, m->dp_world, m->dp_rank).rows;
    m->last_alpha = p.alpha;
    m->rows_assigned += p.rows;
    m->t += 1;
    m->pos += p.rows;
    if (m->pos >= rows_pass) {
        m->pass += 1;
        m->pos = 0;
    }
}

static int launch_step(em_model* m, const StepPlan& p) {
    const int64_t rows = rank_share(p, m->dp_world, m->dp_rank).rows;  // this rank's share
    const double rd = (double)rows, dd = (double)m->d, kd = (double)m->k;
    em_model::BatchSlot& b = m->slot[p.t & 1];
    int sp = span_begin(m, EM_PHASE_GATHER);
    const bool inline_gather = m->ready != p.t;
    CKR(prime_batch(m, p));
    span_end(m, sp, 0.0, inline_gather ? 4.0 * rd * dd : 0.0);
    // The next step's rows are gathered on the side stream while this step searches
    // and updates: the search holds one CTA per SM with registers and threads to
    // spare, so the memory-bound gather runs beside the tensor-bound search. Slot
    // (t + 1) & 1 was last read by step t - 1, whose work is all ordered before the
    // fork. The gather is submitted after the search (and, in graphs, at a lower
    // priority) so that the search's CTAs are placed first.
    const bool pf = prefetches(m, p.t);
    if (pf) CK(cudaEventRecord(m->ev_fork, m->stream));
    sp = span_begin(m, EM_PHASE_ASSIGN);
    CKR(launch_assign(m, m->fp8 ? b.tm8 : b.tm, b.X.p, rows));
    span_end(m, sp, 2.0 * rd * kd * dd, 0.0);
    if (pf) {
        cudaStream_t side = m->capturing ? m->side_cap : m->side;
        const StepPlan q = plan_after(m, p);
        CK(cudaStreamWaitEvent(side, m->ev_fork, 0));
        CKR(launch_gather(m, q, side));
        CK(cudaEventRecord(m->ev_gathered[q.t & 1], side));
    }
    sp = span_begin(m, EM_PHASE_UPDATE);
    const int nbl = (int)((rows + 255) / 256);
    const int capture = (m->capture && p.last_pass) ? 1 : 0;
    launch_k(m->pdl, k_labels, nbl, 256, 0, m->stream, m->keys.p, m->last_split, m->fp8 ? b.xn8.p : b.xn.p, (int)rows,
                                         (int)m->k, b.X.p, m->ld, m->cq.p, b.ids.p, m->labels.p, m->dists.p,
                                         m->cnt.p, m->rank.p, m->block_err.p, m->labels_last.p, capture,
                                         training_kind(m), score_scale(m), tie_list(m), m->N.p, m->N_prev.p,
                                         m->err.p);
    CK(cudaGetLastError());
    EM_LAUNCHED(m, 1);
    CKR(launch_settle(m, b.X.p, b.xn.p, m->labels.p, nullptr, m->dists.p, true, b.ids.p, m->labels_last.p,
                      capture));
    // the revival check's donor selection beside the segmented sums (not while
    // profiling, so that each phase is timed alone; not in data-parallel runs, whose
    // counts come from the exchange)
    const bool overlap = p.revive && revival_on(m) && !m->profile && m->comm == nullptr;
    CKR(launch_reduce(m, b.X.p, rows, nbl, p.alpha, m->finalize ? p.last_pass : 0, m->step_err.p + p.t,
                      overlap ? p.t : -1));
    span_end(m, sp, 0.0, 2.0 * rd * dd + 16.0 * rd + 14.0 * kd * dd);
    if (p.revive) {
        sp = span_begin(m, EM_PHASE_REVIVE);
        CKR(launch_revive(m, p.t, rows, b.X.p, overlap));
        span_end(m, sp);
    }
    if (pf) {
        m->ready = p.t + 1;
        m->ready_synced = false;
    }
    return EM_OK;
}

static int run_step(em_model* m) {
    const StepPlan p = plan_step(m);
    CKR(launch_step(m, p));
    advance_step(m, p);
    return EM_OK;
}

// Everything a captured step range bakes in: buffer addresses, sizes, options.
static std::vector<uint64_t> graph_signature(const em_model* m) {
    const void* ptrs[] = {m->X, m->slot[0].X.p, m->slot[0].xn.p, m->slot[0].ids.p, m->slot[1].X.p,
                          m->slot[1].xn.p, m->slot[1].ids.p, m->dists.p, m->labels.p, m->cnt.p, m->rank.p,
                          m->N_prev.p, m->cnp.p,
                          m->off.p, m->perm.p, m->poff.p, m->items.p, m->keys.p, m->block_err.p, m->part.p,
                          m->step_err.p, m->labels_last.p, m->N.p, m->S.p, m->c.p, m->cn.p, m->cq.p,
                          m->close_sum.p, m->close_cnt.p, m->err.p, m->rv_dead.p, m->rv_donor.p, m->rv_order.p,
                          m->rv_times.p, m->rv_ndead.p, m->rv_tree.p, m->rv_target.p, m->rv_splits.p,
                          m->ties.p, m->tie_n.p, m->tie_corr.p};
    std::vector<uint64_t> sig;
    for (const void* q : ptrs) sig.push_back((uint64_t)(uintptr_t)q);
    const int64_t ints[] = {m->n, m->d, m->k, m->ld, m->kc, m->R, m->sms, m->rec.batch_size, m->rec.total_steps,
                            m->rec.passes, m->rec.rows_last_pass, (int64_t)m->seed, m->revival, m->finalize,
                            m->capture, m->auto_revive, m->assign_kernel, m->wait_cycles, m->exact_ties,
                            m->spherical, m->prefetch, m->n_local, m->dp_world, m->dp_rank,
                            (int64_t)(uintptr_t)m->comm, (int64_t)(uintptr_t)m->stats.p, m->fp8,
                            (int64_t)(uintptr_t)m->slot[0].X8.p, (int64_t)(uintptr_t)m->slot[1].X8.p,
                            (int64_t)(uintptr_t)m->cq8.p, (int64_t)(uintptr_t)m->fp8_shift.p,
                            (int64_t)__float_as_uint_host(m->fp8_scale), m->pdl};
    for (int64_t v : ints) sig.push_back((uint64_t)v);
    double dbl[] = {m->rec.alpha0, m->tau};
    for (double v : dbl) {
        uint64_t u;
        memcpy(&u, &v, 8);
        sig.push_back(u);
    }
    return sig;
}

// Runs `count` steps from the current position as one CUDA graph (captured on a
// private stream the first time this exact range is asked for, then replayed).
static int run_steps_graph(em_model* m, int64_t count) {
    const std::vector<uint64_t> sig = graph_signature(m);
    const int64_t t0 = m->t;
    // a graph starts from the first step's rows in place and ordered before it
    CKR(prime_batch(m, plan_step(m)));
    for (auto& g : m->graph_cache) {
        if (g.t0 == t0 && g.count == count && g.sig == sig) {
            CK(cudaGraphLaunch(g.exec, m->stream));
            for (int64_t i = 0; i < count; ++i) advance_step(m, plan_step(m));
            // the graph ends with the prefetch of the next range's first step joined
            m->ready = prefetches(m, m->t - 1) ? m->t : -1;
            m->ready_synced = true;
            EM_LAUNCHED(m, g.launches);
            return EM_OK;
        }
    }
    if (!m->cap_stream || !m->side_cap) {  // the step kernels above the side-stream gathers
        int least = 0, greatest = 0;
        CK(cudaDeviceGetStreamPriorityRange(&least, &greatest));
        if (!m->cap_stream) CK(cudaStreamCreateWithPriority(&m->cap_stream, cudaStreamNonBlocking, greatest));
        if (!m->side_cap) CK(cudaStreamCreateWithPriority(&m->side_cap, cudaStreamNonBlocking, least));
    }
    const int64_t save_t = m->t, save_pass = m->pass, save_pos = m->pos, save_rows = m->rows_assigned;
    const int64_t save_last = m->last_rows, save_launches = m->launches;
    const double save_alpha = m->last_alpha;
    cudaStream_t user = m->stream;
    m->stream = m->cap_stream;
    m->capturing = true;
    CK(cudaStreamBeginCapture(m->cap_stream, cudaStreamCaptureModeThreadLocal));
    int rc = EM_OK;
    for (int64_t i = 0; i < count && rc == EM_OK; ++i) rc = run_step(m);
    // join the last step's prefetch so that the graph ends with it
    if (rc == EM_OK && m->ready >= 0 && !m->ready_synced &&
        cudaStreamWaitEvent(m->cap_stream, m->ev_gathered[m->ready & 1], 0) != cudaSuccess)
        rc = EM_E_CUDA;
    cudaGraph_t graph = nullptr;
    const cudaError_t ce = cudaStreamEndCapture(m->cap_stream, &graph);
    m->stream = user;
    m->capturing = false;
    m->ready_synced = true;
    cudaGraphExec_t exec = nullptr;
    if (rc == EM_OK && ce == cudaSuccess && graph &&
        cudaGraphInstantiateWithFlags(&exec, graph, cudaGraphInstantiateFlagUseNodePriority) == cudaSuccess) {
        cudaGraphDestroy(graph);
        const int64_t launches = m->launches - save_launches;
        if (m->graph_cache.size() >= 64) {
            cudaGraphExecDestroy(m->graph_cache.front().exec);
            m->graph_cache.erase(m->graph_cache.begin());
        }
        m->graph_cache.push_back({sig, t0, count, launches, exec});
        CK(cudaGraphLaunch(exec, m->stream));
        return EM_OK;
    }
    // capture did not work: undo the bookkeeping and launch the steps directly
    if (graph) cudaGraphDestroy(graph);
    cudaGetLastError();
    m->t = save_t;
    m->pass = save_pass;
    m->pos = save_pos;
    m->rows_assigned = save_rows;
    m->last_rows = save_last;
    m->last_alpha = save_alpha;
    m->launches = save_launches;
    m->ready = t0;  // primed before the capture
    m->ready_synced = true;
    for (int64_t i = 0; i < count; ++i) CKR(run_step(m));
    return EM_OK;
}

// The E4M3 operand -e4m3((c - shift) * scale) and |c'|^2 / 2 of every centroid.
static int fp8_operand(em_model* m) {
    // (without a converter yet, the first search calibrates one and builds the operand)
    if (!m->fp8 || !m->fp8_ready) return EM_OK;
    launch_k(m->pdl, k_fp8_operand, grid_for(m->k * 32, 256, m->sms), 256, 0, m->stream, 
        m->c.p, (int)m->k, (int)m->d, m->ld, m->fp8_shift.p, m->fp8_scale, m->cq8.p, m->ld8, m->cn8.p);
    CK(cudaGetLastError());
    EM_LAUNCHED(m, 1);
    return EM_OK;
}

static int after_centroid_change(em_model* m) {
    if (m->spherical) {
        launch_k(m->pdl, k_normalize, grid_for(m->k * 32, 256, m->sms), 256, 0, m->stream, cluster_state(m), (int)m->k, m->nv);
        CK(cudaGetLastError());
        EM_LAUNCHED(m, 1);
    }
    return fp8_operand(m);
}

// Fits the FP8 converter on the first rows of X (bf16, n rows; README "Data
// precision": a shift per dimension and one power-of-two scale, calibrated on a
// sample): shift = each dimension's midrange in fp32, scale = the largest power of
// two keeping max |x - shift| within 448. In a data-parallel run the ranks' minima
// and maxima are combined first, so that every rank holds the same converter.
static int fp8_calibrate(em_model* m, const __nv_bfloat16* X, int64_t n) {
    const int64_t rows = std::min<int64_t>(n, kFp8CalibRows);
    const int d = (int)m->d;
    const int parts = (int)std::max<int64_t>(1, std::min<int64_t>(rows, 256));
    CKR(m->fp8_part.ensure((size_t)2 * parts * d));
    CKR(m->fp8_lohi.ensure((size_t)2 * d));
    float* lo = m->fp8_lohi.p;
    float* hi = m->fp8_lohi.p + d;
    k_fp8_minmax<<<dim3((d + 255) / 256, parts), 256, 0, m->stream>>>(X, rows, d, m->ld, m->fp8_part.p,
                                                                       m->fp8_part.p + (size_t)parts * d);
    k_fp8_minmax_reduce<<<(d + 255) / 256, 256, 0, m->stream>>>(m->fp8_part.p, m->fp8_part.p + (size_t)parts * d,
                                                                 parts, d, lo, hi);
    CK(cudaGetLastError());
    EM_LAUNCHED(m, 2);
    if (m->comm && m->dp_world > 1) {
        NCK(nccl().all_reduce(lo, lo, (size_t)d, ncclFloat32, ncclMin, m->comm, m->stream));
        NCK(nccl().all_reduce(hi, hi, (size_t)d, ncclFloat32, ncclMax, m->comm, m->stream));
    }
    std::vector<float> h(2 * (size_t)d);
    CK(cudaMemcpyAsync(h.data(), lo, 2 * (size_t)d * sizeof(float), cudaMemcpyDeviceToHost, m->stream));
    CK(cudaStreamSynchronize(m->stream));
    std::vector<float> shift(m->ld, 0.0f);
    double mx = 0.0;
    for (int j = 0; j < d; ++j) {
        const float l = h[j], u = h[d + j];
        const float sh = (l + u) * 0.5f;
        shift[j] = sh;
        mx = std::max(mx, (double)std::max(u - sh, sh - l));
    }
    double scale = 1.0;
    if (mx > 0.0) {
        int e = (int)std::floor(std::log2((double)kE4M3Max / mx));
        while (mx * std::ldexp(1.0, e) > (double)kE4M3Max) --e;
        while (mx * std::ldexp(1.0, e + 1) <= (double)kE4M3Max) ++e;
        scale = std::ldexp(1.0, e);
    }
    if (!(scale >= 0x1p-126 && scale <= 0x1p+126)) return fail(EM_E_INVAL, "the data's range is outside FP8 reach");
    CKR(m->fp8_shift.ensure(m->ld));
    CK(cudaMemcpyAsync(m->fp8_shift.p, shift.data(), m->ld * sizeof(float), cudaMemcpyHostToDevice, m->stream));
    CK(cudaStreamSynchronize(m->stream));
    m->fp8_scale = (float)scale;
    m->fp8_ready = true;
    return EM_OK;
}

// A run (or Lloyd) on X with the FP8 search: the operand buffers and the converter.
static int prepare_fp8(em_model* m, const __nv_bfloat16* X, int64_t n) {
    if (!m->fp8) return EM_OK;
    if (m->spherical) return fail(EM_E_INVAL, "spherical e-means takes the bf16 search only");
    if (m->assign_kernel != 0) return fail(EM_E_INVAL, "the FP8 search runs on the tensor-core kernel only");
    m->fp8_ready = false;  // until the operand buffers and the new converter are in place
    CKR(m->cq8.ensure((size_t)m->k * m->ld8));
    CKR(m->cn8.ensure(m->k));
    CKR(make_tmap8(&m->tm_cq8, m->cq8.p, m->k, (int)m->d, m->ld8, tc::BN));
    return fp8_calibrate(m, X, n);
}

// E4M3 codes and |x'|^2 of all n rows of A (a full pass) into X8full / xn8full, and
// the search map over them.
static int fp8_rows(em_model* m, const __nv_bfloat16* A, int64_t n, CUtensorMap* tm) {
    CKR(m->X8full.ensure((size_t)n * m->ld8));
    CKR(m->xn8full.ensure(n));
    k_fp8_rows<<<grid_for(n * 32, 256, m->sms), 256, 0, m->stream>>>(A, n, (int)m->d, m->ld, m->fp8_shift.p,
                                                                     m->fp8_scale, m->X8full.p, m->ld8,
                                                                     m->xn8full.p);
    CK(cudaGetLastError());
    EM_LAUNCHED(m, 1);
    return make_tmap8(tm, m->X8full.p, n, (int)m->d, m->ld8, tc::BM);
}

static int start_centroids(em_model* m) {
    k_init_centroids<<<grid_for(m->k * 32, 256, m->sms), 256, 0, m->stream>>>(
        m->X, m->n_local, m->ld, (int)m->k, m->seed, m->c.p, m->S.p, m->N.p, m->cq.p, m->cn.p, m->err.p);
    CK(cudaGetLastError());
    EM_LAUNCHED(m, 1);
    return after_centroid_change(m);
}

// ------------------------------------------------------------------ ABI

extern "C" {

const char* em_last_error(void) { return g_err; }

int em_last_error_code(void) { return g_err_code; }

int64_t em_fail_allocation(int64_t nth) {
    const int64_t attempts = g_alloc_attempts.exchange(0);
    g_alloc_fail_at.store(nth > 0 ? nth : 0);
    return attempts;
}

int em_device_count(void) {
    int n = 0;
    if (cudaGetDeviceCount(&n) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

int em_compute_recipe(int64_t n, int64_t k, double epochs, int law, int64_t batch_override, double alpha_override,
                      em_recipe_t* out) {
    if (!out) return fail(EM_E_INVAL, "out is NULL");
    return compute_recipe(n, k, 0, epochs, law, batch_override, alpha_override, out);
}

int em_permutation(int64_t n, uint64_t seed, int stream, int64_t which, const int64_t* idx, int64_t count,
                   int64_t* out) {
    if (n < 1 || count < 0 || (count > 0 && (!idx || !out))) return fail(EM_E_INVAL, "bad permutation arguments");
    const Feistel f(n, seed, stream, which);
    for (int64_t i = 0; i < count; ++i) {
        if (idx[i] < 0 || idx[i] >= n) return fail(EM_E_INVAL, "index out of range");
        bool ok = true;
        out[i] = f((uint64_t)idx[i], &ok);
        if (!ok) return fail(EM_E_BOUNDS, "cycle walk did not end");
    }
    return EM_OK;
}

int em_dp_schedule(int64_t n_local, int64_t k, double epochs, int law, int64_t batch_override,
                   double alpha_override, int64_t world, int64_t rank, int64_t count, int64_t* pass, int64_t* first,
                   int64_t* rows, int64_t* key) {
    if (n_local < 1 || world < 1 || rank < 0 || rank >= world || count < 0)
        return fail(EM_E_INVAL, "bad data-parallel schedule arguments");
    if (count > 0 && (!pass || !first || !rows || !key)) return fail(EM_E_INVAL, "an output is NULL");
    em_recipe_t rec;
    CKR(compute_recipe(n_local * world, k, 0, epochs, law, batch_override, alpha_override, &rec));
    if (rec.batch_size > rec.n) return fail(EM_E_INVAL, "batch size larger than n");
    CKR(check_dp_recipe(rec, world));
    if (count > rec.total_steps) return fail(EM_E_INVAL, "count is beyond the run's %lld steps",
                                             (long long)rec.total_steps);
    StepPlan p = plan_rows(rec, rec.n, false, 0, 0, 0);
    for (int64_t t = 0; t < count; ++t) {
        if (t) p = plan_next(rec, rec.n, false, p);
        const RankShare sh = rank_share(p, world, rank);
        pass[t] = p.pass;
        first[t] = sh.first;
        rows[t] = sh.rows;
        key[t] = sh.key;
    }
    return EM_OK;
}

int em_search_schedule(int64_t rows, int64_t k, int sms, int* split, int* m_full) {
    if (rows < 1 || k < 1 || sms < 1 || !split || !m_full) return fail(EM_E_INVAL, "bad search schedule arguments");
    const Schedule sc = choose_schedule((rows + tc::BM - 1) / tc::BM, (k + tc::BN - 1) / tc::BN, sms);
    *split = sc.split;
    *m_full = sc.m_full;
    return EM_OK;
}

em_model* em_create(int64_t d, int64_t k, uint64_t seed) {
    if (d < 1 || d > 8192 || k < 1 || k > (1ll << 30)) {
        fail(EM_E_INVAL, "need 1 <= d <= 8192 and 1 <= k <= 2^30");
        return nullptr;
    }
    if (em_device_count() < 1) {
        fail(EM_E_NODEVICE, "no CUDA device");
        return nullptr;
    }
    em_model* m = new em_model();
    m->d = d;
    m->k = k;
    m->seed = seed;
    m->ld = (int)((d + 7) / 8 * 8);
    m->ld8 = (int)((d + 15) / 16 * 16);
    m->nv = m->ld / 8;
    m->kc = (d % 64 == 0) ? 64 : 32;
    auto bail = [&](int code, const char* what) -> em_model* {
        fail(code, "%s", what);
        em_destroy(m);
        return nullptr;
    };
    if (cudaGetDevice(&m->dev) != cudaSuccess) return bail(EM_E_CUDA, "cudaGetDevice failed");
    int clock_khz = 1965000;
    cudaDeviceGetAttribute(&m->sms, cudaDevAttrMultiProcessorCount, m->dev);
    cudaDeviceGetAttribute(&clock_khz, cudaDevAttrClockRate, m->dev);
    m->wait_cycles = (long long)(m->wait_ms * (double)clock_khz);
    int cc_major = 0, cc_minor = 0;
    cudaDeviceGetAttribute(&cc_major, cudaDevAttrComputeCapabilityMajor, m->dev);
    cudaDeviceGetAttribute(&cc_minor, cudaDevAttrComputeCapabilityMinor, m->dev);
    if (cc_major != 10 || cc_minor != 0) return bail(EM_E_NODEVICE, "this library is built for sm_100a (B200)");
    if (cudaStreamCreateWithFlags(&m->stream, cudaStreamNonBlocking) != cudaSuccess)
        return bail(EM_E_CUDA, "cudaStreamCreate failed");
    m->own_stream = true;
    if (cudaStreamCreateWithFlags(&m->side, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&m->ev_fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&m->ev_sel, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&m->ev_gathered[0], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&m->ev_gathered[1], cudaEventDisableTiming) != cudaSuccess)
        return bail(EM_E_CUDA, "stream or event creation failed");
    const size_t kd = (size_t)k * m->ld;
    if (m->N.ensure(k) || m->N_prev.ensure(k) || m->cnp.ensure((size_t)k * ((m->nv + 31) / 32)) ||
        m->S.ensure(kd) || m->c.ensure(kd) || m->cn.ensure(k) || m->cq.ensure(kd) ||
        m->close_sum.ensure(kd) || m->close_cnt.ensure(k) || m->err.ensure(1) || m->flag.ensure(1) ||
        m->scalar.ensure(4) || m->rv_dead.ensure(k) || m->rv_donor.ensure(k) || m->rv_order.ensure(k) ||
        m->rv_times.ensure(k) || m->rv_ndead.ensure(1) || m->rv_splits.ensure(1) || m->rv_target.ensure(k) ||
        m->rv_tree.ensure((size_t)tree_layout((int)k).total) || m->tie_n.ensure(1) || m->tie_corr.ensure(1))
        return bail(EM_E_NOMEM, "device allocation failed");
    cudaMemset(m->err.p, 0, sizeof(int));
    cudaMemset(m->tie_n.p, 0, sizeof(int));
    cudaMemset(m->tie_corr.p, 0, sizeof(double));
    cudaMemset(m->rv_splits.p, 0, sizeof(int64_t));
    cudaMemset(m->rv_ndead.p, 0, sizeof(int32_t));
    cudaMemset(m->N.p, 0, k * sizeof(float));
    cudaMemset(m->S.p, 0, kd * sizeof(float));
    cudaMemset(m->c.p, 0, kd * sizeof(float));
    cudaMemset(m->cq.p, 0, kd * sizeof(__nv_bfloat16));
    cudaMemset(m->cn.p, 0, k * sizeof(float));
    if (!search_smem_attributes() || !select_smem_attributes())
        return bail(EM_E_CUDA, "cudaFuncSetAttribute failed");
    if (make_tmap(&m->tm_cq, m->cq.p, k, (int)d, m->ld, tc::BN, m->kc) != EM_OK) {
        em_destroy(m);
        return nullptr;
    }
    {  // the folded search's operands: each batch row's (1, 1, 1, 0, ...), and the norms tiles
        std::vector<__nv_bfloat16> ones((size_t)tc::BM * tc::kExtK, __float2bfloat16(0.0f));
        for (int r = 0; r < tc::BM; ++r)
            for (int e = 0; e < 3; ++e) ones[(size_t)r * tc::kExtK + e] = __float2bfloat16(1.0f);
        // (the norms operand covers whole centroid tiles: rows past k hold +inf)
        const int64_t k_pad = (k + tc::BN - 1) / tc::BN * tc::BN;
        if (m->cn3.ensure((size_t)k_pad * tc::kExtK) || m->ones3.ensure((size_t)tc::BM * tc::kExtK))
            return bail(EM_E_NOMEM, "device allocation failed");
        cudaMemset(m->cn3.p, 0, (size_t)k_pad * tc::kExtK * sizeof(__nv_bfloat16));
        if (cudaMemcpy(m->ones3.p, ones.data(), ones.size() * sizeof(__nv_bfloat16), cudaMemcpyHostToDevice) !=
                cudaSuccess ||
            make_tmap_ext(&m->tm_cn3, m->cn3.p, k_pad, tc::BN) != EM_OK ||
            make_tmap_ext(&m->tm_ones3, m->ones3.p, tc::BM, tc::BM) != EM_OK) {
            em_destroy(m);
            return nullptr;
        }
    }
    if (cudaDeviceSynchronize() != cudaSuccess) return bail(EM_E_CUDA, "device initialisation failed");
    return m;
}

void em_destroy(em_model* m) {
    if (!m) return;
    cudaSetDevice(m->dev);
    if (m->stream) cudaStreamSynchronize(m->stream);
    m->N.release(); m->N_prev.release(); m->cnp.release(); m->S.release(); m->c.release(); m->cn.release();
    m->cq.release();
    m->cn3.release();
    m->ones3.release();
    m->close_sum.release(); m->close_cnt.release(); m->err.release(); m->flag.release();
    if (m->side) cudaStreamSynchronize(m->side);
    for (auto& b : m->slot) {
        b.X.release();
        b.xn.release();
        b.ids.release();
        b.X8.release();
        b.xn8.release();
    }
    m->Xown.release(); m->stage.release(); m->xn.release(); m->dists.release();
    m->labels.release(); m->cnt.release(); m->rank.release(); m->off.release();
    m->perm.release(); m->poff.release(); m->items.release(); m->keys.release(); m->block_err.release();
    m->part.release(); m->step_err.release(); m->scalar.release(); m->labels_last.release();
    m->labels64.release(); m->rv_dead.release(); m->rv_donor.release(); m->rv_order.release();
    m->rv_times.release(); m->rv_ndead.release(); m->rv_tree.release(); m->rv_splits.release();
    m->ties.release(); m->tie_n.release(); m->tie_corr.release(); m->stats.release();
    m->fp8_shift.release(); m->fp8_lohi.release(); m->fp8_part.release(); m->cq8.release(); m->X8full.release();
    m->cn8.release(); m->xn8full.release();
    m->rv_target.release();
    for (auto& sp : m->pending) {
        cudaEventDestroy(sp.a);
        cudaEventDestroy(sp.b);
    }
    for (auto ev : m->pool) cudaEventDestroy(ev);
    for (auto& g : m->graph_cache) cudaGraphExecDestroy(g.exec);  // graphs may hold NCCL calls
    if (m->comm) nccl().destroy(m->comm);
    if (m->cap_stream) cudaStreamDestroy(m->cap_stream);
    if (m->side_cap) cudaStreamDestroy(m->side_cap);
    if (m->side) cudaStreamDestroy(m->side);
    if (m->ev_fork) cudaEventDestroy(m->ev_fork);
    if (m->ev_sel) cudaEventDestroy(m->ev_sel);
    for (auto ev : m->ev_gathered)
        if (ev) cudaEventDestroy(ev);
    if (m->own_stream && m->stream) cudaStreamDestroy(m->stream);
    delete m;
}

int em_set_option(em_model* m, int opt, double v) {
    if (!m) return fail(EM_E_INVAL, "model is NULL");
    switch (opt) {
        case EM_OPT_BATCH_SIZE:
            if (v < 0 || v != floor(v)) return fail(EM_E_INVAL, "batch size must be a non-negative integer");
            m->opt_batch = (int64_t)v;
            break;
        case EM_OPT_ALPHA0:
            if (v < 0 || v > 1) return fail(EM_E_INVAL, "alpha0 must be in [0, 1]");
            m->opt_alpha0 = v;
            break;
        case EM_OPT_UNUSED_THRESHOLD:
            if (v != -1 && (!(v >= 0) || v > 1)) return fail(EM_E_INVAL, "threshold must be in [0, 1], or -1");
            m->tau = v;
            break;
        case EM_OPT_REVIVAL:
            if (v != 0 && v != 1 && v != 2) return fail(EM_E_INVAL, "revival mode is 0, 1 or 2");
            m->revival = (int)v;
            break;
        case EM_OPT_FINALIZE: m->finalize = v != 0; break;
        case EM_OPT_LAW:
            if (v != 0 && v != 1 && v != 2) return fail(EM_E_INVAL, "law is 0, 1 or 2");
            m->law = (int)v;
            break;
        case EM_OPT_INPUT_DTYPE:
            if (v != 0 && v != 1) return fail(EM_E_INVAL, "input dtype is 0 (fp32) or 1 (bf16)");
            m->in_dtype = (int)v;
            break;
        case EM_OPT_CHECK_FINITE: m->check_finite = v != 0; break;
        case EM_OPT_WAIT_LIMIT_MS: {
            if (!(v > 0)) return fail(EM_E_INVAL, "wait limit must be positive");
            int clock_khz = 1965000;
            cudaDeviceGetAttribute(&clock_khz, cudaDevAttrClockRate, m->dev);
            m->wait_ms = v;
            m->wait_cycles = (long long)(v * (double)clock_khz);
            break;
        }
        case EM_OPT_AUTO_REVIVE: m->auto_revive = v != 0; break;
        case EM_OPT_CAPTURE_LABELS: m->capture = v != 0; break;
        case EM_OPT_GRAPHS: m->graphs = v != 0; break;
        case EM_OPT_ASSIGN_KERNEL:
            if (v != 0 && v != 1) return fail(EM_E_INVAL, "assign kernel is 0 or 1");
            m->assign_kernel = (int)v;
            break;
        case EM_OPT_PROFILE: m->profile = v != 0; break;
        case EM_OPT_EXACT_TIES:
            if (v != -1 && v != 0 && v != 1) return fail(EM_E_INVAL, "exact ties is -1, 0 or 1");
            m->exact_ties = (int)v;
            break;
        case EM_OPT_PDL:
            if (v != 0 && v != 1) return fail(EM_E_INVAL, "pdl is 0 or 1");
            m->pdl = (int)v;
            break;
        case EM_OPT_SEARCH_FORMAT:
            if (v != 0 && v != 1) return fail(EM_E_INVAL, "search format is 0 (bf16) or 1 (fp8 e4m3)");
            if (m->running) return fail(EM_E_STATE, "the search format can not change during a run");
            if ((int)v != m->fp8) {
                m->fp8 = (int)v;
                m->fp8_ready = false;  // a new converter at the next run
            }
            break;
        case EM_OPT_PREFETCH:
            if (v != 0 && v != 1) return fail(EM_E_INVAL, "prefetch is 0 or 1");
            m->prefetch = (int)v;
            break;
        case EM_OPT_SPHERICAL:
            if (v != 0 && v != 1) return fail(EM_E_INVAL, "spherical is 0 or 1");
            if (m->running) return fail(EM_E_STATE, "spherical can not change during a run");
            m->spherical = (int)v;
            break;
        default: return fail(EM_E_INVAL, "unknown option %d", opt);
    }
    return EM_OK;
}

int em_get_option(const em_model* m, int opt, double* v) {
    if (!m || !v) return fail(EM_E_INVAL, "NULL argument");
    switch (opt) {
        case EM_OPT_BATCH_SIZE: *v = (double)m->opt_batch; break;
        case EM_OPT_ALPHA0: *v = m->opt_alpha0; break;
        case EM_OPT_UNUSED_THRESHOLD: *v = m->tau; break;
        case EM_OPT_REVIVAL: *v = m->revival; break;
        case EM_OPT_FINALIZE: *v = m->finalize; break;
        case EM_OPT_LAW: *v = m->law; break;
        case EM_OPT_INPUT_DTYPE: *v = m->in_dtype; break;
        case EM_OPT_CHECK_FINITE: *v = m->check_finite; break;
        case EM_OPT_WAIT_LIMIT_MS: *v = m->wait_ms; break;
        case EM_OPT_AUTO_REVIVE: *v = m->auto_revive; break;
        case EM_OPT_CAPTURE_LABELS: *v = m->capture; break;
        case EM_OPT_GRAPHS: *v = m->graphs; break;
        case EM_OPT_ASSIGN_KERNEL: *v = m->assign_kernel; break;
        case EM_OPT_PROFILE: *v = m->profile; break;
        case EM_OPT_EXACT_TIES: *v = m->exact_ties; break;
        case EM_OPT_SPHERICAL: *v = m->spherical; break;
        case EM_OPT_PREFETCH: *v = m->prefetch; break;
        case EM_OPT_SEARCH_FORMAT: *v = m->fp8; break;
        case EM_OPT_PDL: *v = m->pdl; break;
        default: return fail(EM_E_INVAL, "unknown option %d", opt);
    }
    return EM_OK;
}

int em_set_stream(em_model* m, void* stream) {
    if (!m) return fail(EM_E_INVAL, "model is NULL");
    CKR(set_device(m));
    CK(cudaStreamSynchronize(m->stream));
    if (m->own_stream) cudaStreamDestroy(m->stream);
    m->stream = reinterpret_cast<cudaStream_t>(stream);
    m->own_stream = false;
    return EM_OK;
}

int em_begin(em_model* m, const void* X, int64_t n, double epochs) {
    if (!m) return fail(EM_E_INVAL, "model is NULL");
    if (n < m->k) return fail(EM_E_INVAL, "need at least k rows (n = %lld, k = %lld)", (long long)n, (long long)m->k);
    if (n >= (1ll << 31)) return fail(EM_E_INVAL, "n must be below 2^31");
    if (!(epochs > 0.0)) return fail(EM_E_INVAL, "epochs must be positive");
    CKR(set_device(m));
    // a data-parallel run: n is this rank's share, the recipe is the whole job's
    const int64_t W = m->dp_world, n_total = n * W;
    if (n_total >= (1ll << 31)) return fail(EM_E_INVAL, "the rows of all ranks must be below 2^31");
    CKR(compute_recipe(n_total, m->k, m->d, epochs, effective_law(m), m->opt_batch, m->opt_alpha0, &m->rec));
    if (m->rec.batch_size > n_total) return fail(EM_E_INVAL, "batch size larger than n");
    if (W > 1) {
        CKR(check_dp_recipe(m->rec, W));
        if (m->revival == EM_REVIVE_RESAMPLE)
            return fail(EM_E_INVAL, "resampling draws rows of the whole batch; use it with one rank");
    }
    m->running = false;
    m->n = n_total;
    m->n_local = n;
    const int sp = span_begin(m, EM_PHASE_PREPARE);
    CKR(prepare_input(m, X, n, m->Xown, &m->X));
    CKR(prepare_fp8(m, m->X, n));
    const int64_t b = m->rec.batch_size / W;  // this rank's rows of a full batch
    CKR(drop_prefetch(m));
    CK(cudaStreamSynchronize(m->stream));  // no gather of a previous run still writes the slots
    for (auto& bs : m->slot) {
        CKR(bs.X.ensure((size_t)b * m->ld));
        CKR(bs.xn.ensure(b));
        CKR(bs.ids.ensure(b));
        CKR(make_tmap(&bs.tm, bs.X.p, b, (int)m->d, m->ld, tc::BM, m->kc));
        if (m->fp8) {
            CKR(bs.X8.ensure((size_t)b * m->ld8));
            CKR(bs.xn8.ensure(b));
            CKR(make_tmap8(&bs.tm8, bs.X8.p, b, (int)m->d, m->ld8, tc::BM));
        }
    }
    CKR(ensure_batch_buffers(m, b));
    {  // every batch size the run will see: full batches and the last, partial ones
        const int64_t B = m->rec.batch_size;
        const int64_t sizes[3] = {b, (n_total % B) / W, (m->rec.rows_last_pass % B) / W};
        size_t need = 0;
        for (int64_t r : sizes) need = std::max(need, keys_needed(m, r));
        CKR(m->keys.ensure(need));
    }
    CKR(m->step_err.ensure(m->rec.total_steps));
    CK(cudaMemsetAsync(m->step_err.p, 0, m->rec.total_steps * sizeof(double), m->stream));
    CK(cudaMemsetAsync(m->cnt.p, 0, m->k * sizeof(int32_t), m->stream));
    CK(cudaMemsetAsync(m->close_sum.p, 0, (size_t)m->k * m->ld * sizeof(double), m->stream));
    CK(cudaMemsetAsync(m->close_cnt.p, 0, m->k * sizeof(double), m->stream));
    CK(cudaMemsetAsync(m->rv_splits.p, 0, sizeof(int64_t), m->stream));
    CK(cudaMemsetAsync(m->rv_ndead.p, 0, sizeof(int32_t), m->stream));
    if (m->capture) {
        CKR(m->labels_last.ensure(n));
        CK(cudaMemsetAsync(m->labels_last.p, 0xFF, n * sizeof(int64_t), m->stream));
    }
    if (m->comm) CKR(m->stats.ensure((size_t)m->k * m->ld + m->k + 1));
    CKR(start_centroids(m));
    if (m->comm && W > 1) {  // README "Several GPUs": rank 0's starting centroids are used
        const size_t kd = (size_t)m->k * m->ld;
        NCK(nccl().broadcast(m->c.p, m->c.p, kd, ncclFloat32, 0, m->comm, m->stream));
        NCK(nccl().broadcast(m->cq.p, m->cq.p, kd * sizeof(__nv_bfloat16), ncclUint8, 0, m->comm, m->stream));
        NCK(nccl().broadcast(m->cn.p, m->cn.p, (size_t)m->k, ncclFloat32, 0, m->comm, m->stream));
        CKR(fp8_operand(m));
    }
    span_end(m, sp);
    m->t = m->pass = m->pos = m->rows_assigned = 0;
    m->last_rows = 0;
    m->last_alpha = 0.0;
    m->running = true;
    m->have_run = true;
    m->last_was_lloyd = 0;
    return EM_OK;
}

int em_step(em_model* m, int64_t nsteps, int64_t* done) {
    if (done) *done = 0;
    if (!m) return fail(EM_E_INVAL, "model is NULL");
    if (!m->running) return fail(EM_E_STATE, "no run in progress (call em_begin)");
    CKR(set_device(m));
    const int64_t count = std::max<int64_t>(0, std::min(nsteps, m->rec.total_steps - m->t));
    if (m->graphs && !m->profile && count >= 2) {
        CKR(run_steps_graph(m, count));
    } else {
        for (int64_t i = 0; i < count; ++i) CKR(run_step(m));
    }
    if (done) *done = count;
    return EM_OK;
}

int em_revive(em_model* m) {
    if (!m) return fail(EM_E_INVAL, "model is NULL");
    if (!m->running || m->t == 0) return fail(EM_E_STATE, "no step has run");
    CKR(set_device(m));
    return launch_revive(m, m->t - 1, m->last_rows, m->slot[(m->t - 1) & 1].X.p);
}

int em_finalize(em_model* m) {
    if (!m) return fail(EM_E_INVAL, "model is NULL");
    if (!m->running) return fail(EM_E_STATE, "no run in progress");
    CKR(set_device(m));
    CKR(drop_prefetch(m));
    if (m->finalize && m->t >= m->rec.total_steps) {
        const int sp = span_begin(m, EM_PHASE_FINALIZE);
        k_closing_mean<<<grid_for(m->k * 32, 256, m->sms), 256, 0, m->stream>>>(cluster_state(m), (int)m->k,
                                                                                  m->nv);
        CK(cudaGetLastError());
        EM_LAUNCHED(m, 1);
        CKR(after_centroid_change(m));
        span_end(m, sp);
    }
    m->running = false;
    return check_device_errors(m);
}

int em_train(em_model* m, const void* X, int64_t n, double epochs) {
    CKR(em_begin(m, X, n, epochs));
    CKR(em_step(m, m->rec.total_steps, nullptr));
    return em_finalize(m);
}

int em_lloyd(em_model* m, const void* X, int64_t n, int64_t iters) {
    if (!m) return fail(EM_E_INVAL, "model is NULL");
    if (n < m->k || n >= (1ll << 31) || iters < 0) return fail(EM_E_INVAL, "bad Lloyd arguments");
    CKR(set_device(m));
    CKR(drop_prefetch(m));
    m->running = false;
    m->n_local = n;
    m->n = n * m->dp_world;  // data-parallel: every rank's rows, one summed update per iteration
    CKR(prepare_input(m, X, n, m->Xown, &m->X));
    CKR(prepare_fp8(m, m->X, n));
    CKR(ensure_batch_buffers(m, n));
    if (m->comm) CKR(m->stats.ensure((size_t)m->k * m->ld + m->k + 1));
    CKR(m->keys.ensure(keys_needed(m, n)));
    CK(cudaMemsetAsync(m->cnt.p, 0, m->k * sizeof(int32_t), m->stream));
    CKR(start_centroids(m));
    if (m->comm && m->dp_world > 1) {  // rank 0's starting rows
        const size_t kd = (size_t)m->k * m->ld;
        NCK(nccl().broadcast(m->c.p, m->c.p, kd, ncclFloat32, 0, m->comm, m->stream));
        NCK(nccl().broadcast(m->cq.p, m->cq.p, kd * sizeof(__nv_bfloat16), ncclUint8, 0, m->comm, m->stream));
        NCK(nccl().broadcast(m->cn.p, m->cn.p, (size_t)m->k, ncclFloat32, 0, m->comm, m->stream));
        CKR(fp8_operand(m));
    }
    CUtensorMap tmx;
    CKR(make_tmap(&tmx, m->X, n, (int)m->d, m->ld, tc::BM, m->kc));
    if (m->fp8) CKR(fp8_rows(m, m->X, n, &tmx));  // the rows' codes do not change between iterations
    const float* x2 = m->fp8 ? m->xn8full.p : m->xn.p;
    const int nbl = (int)((n + 255) / 256);
    for (int64_t it = 0; it < iters; ++it) {
        if (!m->fp8) {
            k_rownorm<<<grid_for(n * 32, 256, m->sms), 256, 0, m->stream>>>(m->X, n, m->ld, m->xn.p);
            CK(cudaGetLastError());
            EM_LAUNCHED(m, 1);
        }
        CKR(launch_assign(m, tmx, m->X, n));
        launch_k(m->pdl, k_labels, nbl, 256, 0, m->stream, m->keys.p, m->last_split, x2, (int)n, (int)m->k, m->X, m->ld,
                                             m->cq.p, nullptr, m->labels.p, m->dists.p, m->cnt.p, m->rank.p,
                                             m->block_err.p, nullptr, 0, training_kind(m), score_scale(m),
                                             tie_list(m), m->N.p, m->N_prev.p, m->err.p);
        CK(cudaGetLastError());
        EM_LAUNCHED(m, 1);
        CKR(launch_settle(m, m->X, m->xn.p, m->labels.p, nullptr, m->dists.p, true, nullptr, nullptr, 0));
        CKR(launch_reduce(m, m->X, n, nbl, 1.0, 0, m->scalar.p));
    }
    m->have_run = false;
    m->last_was_lloyd = 1;
    return check_device_errors(m);
}

static int assign_pass(em_model* m, const void* X, int64_t n, int64_t* labels_dev, float* dists_dev,
                       double* sum_dev, DBuf<__nv_bfloat16>& tmp) {
    const __nv_bfloat16* A = nullptr;
    CKR(prepare_input(m, X, n, tmp, &A));
    CKR(m->xn.ensure(n));
    CKR(m->keys.ensure(keys_needed(m, n)));
    CKR(m->ties.ensure(n));
    CKR(m->block_err.ensure((n + 255) / 256 + 1));
    if (!dists_dev) {  // k_settle needs the provisional distances of relabelled rows
        CKR(m->dists.ensure(n));
        dists_dev = m->dists.p;
    }
    CUtensorMap tmx;
    if (m->fp8) {  // the model's converter (fitted on this data if the model has none yet)
        if (!m->fp8_ready) {
            CKR(prepare_fp8(m, A, n));
            CKR(fp8_operand(m));
        }
        CKR(fp8_rows(m, A, n, &tmx));
    } else {
        k_rownorm<<<grid_for(n * 32, 256, m->sms), 256, 0, m->stream>>>(A, n, m->ld, m->xn.p);
        CK(cudaGetLastError());
        EM_LAUNCHED(m, 1);
        CKR(make_tmap(&tmx, A, n, (int)m->d, m->ld, tc::BM, m->kc));
    }
    CKR(launch_assign(m, tmx, A, n));
    const int blocks = grid_for(n, 256, m->sms);
    k_assign_out<<<blocks, 256, 0, m->stream>>>(m->keys.p, m->last_split, m->fp8 ? m->xn8full.p : m->xn.p, n,
                                                (int)m->k, A, m->ld, m->cq.p, labels_dev, dists_dev, nullptr,
                                                m->block_err.p, m->spherical ? kSimilarity : kSquaredDistance,
                                                score_scale(m), tie_list(m), m->err.p);
    CK(cudaGetLastError());
    EM_LAUNCHED(m, 1);
    CKR(launch_settle(m, A, m->xn.p, nullptr, labels_dev, dists_dev, false, nullptr, nullptr, 0));
    k_sum_blocks<<<1, 32, 0, m->stream>>>(m->block_err.p, blocks, sum_dev, tie_list(m));
    CK(cudaGetLastError());
    EM_LAUNCHED(m, 1);
    return EM_OK;
}

int em_assign(em_model* m, const void* X, int64_t n, int64_t* labels, float* dists) {
    if (!m) return fail(EM_E_INVAL, "model is NULL");
    if (n < 1 || n >= (1ll << 31)) return fail(EM_E_INVAL, "need 1 <= n < 2^31");
    CKR(set_device(m));
    const bool lab_dev = labels && is_device_ptr(labels);
    const bool dist_dev = dists && is_device_ptr(dists);
    int64_t* lab_p = nullptr;
    float* dist_p = nullptr;
    DBuf<float> dtmp;
    if (labels) {
        if (lab_dev) {
            lab_p = labels;
        } else {
            CKR(m->labels64.ensure(n));
            lab_p = m->labels64.p;
        }
    }
    if (dists) {
        if (dist_dev) {
            dist_p = dists;
        } else {
            CKR(dtmp.ensure(n));
            dist_p = dtmp.p;
        }
    }
    DBuf<__nv_bfloat16> tmp;
    int rc = assign_pass(m, X, n, lab_p, dist_p, m->scalar.p, tmp);
    if (rc == EM_OK && labels && !lab_dev)
        rc = cudaMemcpyAsync(labels, lab_p, n * sizeof(int64_t), cudaMemcpyDeviceToHost, m->stream) == cudaSuccess
                 ? EM_OK
                 : fail(EM_E_CUDA, "copy of labels failed");
    if (rc == EM_OK && dists && !dist_dev)
        rc = cudaMemcpyAsync(dists, dist_p, n * sizeof(float), cudaMemcpyDeviceToHost, m->stream) == cudaSuccess
                 ? EM_OK
                 : fail(EM_E_CUDA, "copy of distances failed");
    if (rc == EM_OK) rc = check_device_errors(m);
    cudaStreamSynchronize(m->stream);
    tmp.release();
    dtmp.release();
    return rc;
}

int em_mse(em_model* m, const void* X, int64_t n, double* out) {
    if (!m || !out) return fail(EM_E_INVAL, "NULL argument");
    if (n < 1 || n >= (1ll << 31)) return fail(EM_E_INVAL, "need 1 <= n < 2^31");
    CKR(set_device(m));
    DBuf<__nv_bfloat16> tmp;
    int rc = assign_pass(m, X, n, nullptr, nullptr, m->scalar.p, tmp);
    double s = 0.0;
    if (rc == EM_OK)
        rc = cudaMemcpyAsync(&s, m->scalar.p, sizeof(double), cudaMemcpyDeviceToHost, m->stream) == cudaSuccess
                 ? EM_OK
                 : fail(EM_E_CUDA, "copy failed");
    if (rc == EM_OK) rc = check_device_errors(m);
    cudaStreamSynchronize(m->stream);
    tmp.release();
    if (rc == EM_OK) *out = s / (double)n;
    return rc;
}

int em_centroids(const em_model* m, float* out) {
    if (!m || !out) return fail(EM_E_INVAL, "NULL argument");
    CKR(set_device(m));
    CK(cudaMemcpy2DAsync(out, m->d * sizeof(float), m->c.p, m->ld * sizeof(float), m->d * sizeof(float), m->k,
                         cudaMemcpyDefault, m->stream));
    CK(cudaStreamSynchronize(m->stream));
    return EM_OK;
}

int em_labels(const em_model* m, int64_t* out) {
    if (!m || !out) return fail(EM_E_INVAL, "NULL argument");
    if (!m->capture || !m->labels_last.p || m->last_was_lloyd) return fail(EM_E_STATE, "no captured labels");
    CKR(set_device(m));
    CK(cudaMemcpyAsync(out, m->labels_last.p, m->n_local * sizeof(int64_t), cudaMemcpyDefault, m->stream));
    CK(cudaStreamSynchronize(m->stream));
    return EM_OK;
}

int em_recipe(const em_model* m, em_recipe_t* out) {
    if (!m || !out) return fail(EM_E_INVAL, "NULL argument");
    if (!m->have_run) return fail(EM_E_STATE, "no run started");
    *out = m->rec;
    return EM_OK;
}

int em_stats(const em_model* m, em_stats_t* out) {
    if (!m || !out) return fail(EM_E_INVAL, "NULL argument");
    CKR(set_device(m));
    memset(out, 0, sizeof(*out));
    out->steps_done = m->t;
    out->passes_done = m->pass;
    out->rows_assigned = m->rows_assigned;
    out->last_alpha = m->last_alpha;
    int64_t splits = 0;
    int32_t nd = 0;
    std::vector<float> N(m->k);
    CK(cudaMemcpyAsync(&splits, m->rv_splits.p, sizeof(int64_t), cudaMemcpyDeviceToHost, m->stream));
    CK(cudaMemcpyAsync(&nd, m->rv_ndead.p, sizeof(int32_t), cudaMemcpyDeviceToHost, m->stream));
    CK(cudaMemcpyAsync(N.data(), m->N.p, m->k * sizeof(float), cudaMemcpyDeviceToHost, m->stream));
    CK(cudaStreamSynchronize(m->stream));
    out->n_splits = splits;
    out->last_dead = nd;
    double sum = 0.0, mx = 0.0;
    for (float v : N) {
        sum += v;
        mx = std::max(mx, (double)v);
    }
    out->imbalance = sum > 0 ? mx / (sum / (double)m->k) : 0.0;
    return EM_OK;
}

int em_obj(const em_model* m, double* out, int64_t cap, int64_t* count) {
    if (!m || (cap > 0 && !out)) return fail(EM_E_INVAL, "NULL argument");
    if (!m->have_run) return fail(EM_E_STATE, "no run started");
    CKR(set_device(m));
    std::vector<double> se(std::max<int64_t>(m->t, 1));
    if (m->t > 0) {
        CK(cudaMemcpyAsync(se.data(), m->step_err.p, m->t * sizeof(double), cudaMemcpyDeviceToHost, m->stream));
        CK(cudaStreamSynchronize(m->stream));
    }
    int64_t avail = 0, s = 0;
    for (int64_t p = 0; p < m->pass; ++p) {
        const int64_t steps = (p == m->rec.passes - 1) ? m->rec.steps_last_pass : m->rec.steps_full_pass;
        const int64_t rows = (p == m->rec.passes - 1) ? m->rec.rows_last_pass : m->n;
        double tot = 0.0;
        for (int64_t q = 0; q < steps; ++q) tot += se[s + q];
        s += steps;
        if (avail < cap) out[avail] = tot / (double)rows;
        ++avail;
    }
    if (count) *count = avail;
    return EM_OK;
}

int em_get_state(const em_model* m, float* N, float* S, float* c, int64_t* step) {
    if (!m) return fail(EM_E_INVAL, "model is NULL");
    CKR(set_device(m));
    if (N) CK(cudaMemcpyAsync(N, m->N.p, m->k * sizeof(float), cudaMemcpyDefault, m->stream));
    if (S)
        CK(cudaMemcpy2DAsync(S, m->d * sizeof(float), m->S.p, m->ld * sizeof(float), m->d * sizeof(float), m->k,
                             cudaMemcpyDefault, m->stream));
    if (c)
        CK(cudaMemcpy2DAsync(c, m->d * sizeof(float), m->c.p, m->ld * sizeof(float), m->d * sizeof(float), m->k,
                             cudaMemcpyDefault, m->stream));
    if (step) *step = m->t;
    CK(cudaStreamSynchronize(m->stream));
    return EM_OK;
}

int em_set_state(em_model* m, const float* N, const float* S, const float* c, int64_t step) {
    if (!m) return fail(EM_E_INVAL, "model is NULL");
    if (m->running && (step < 0 || step > m->rec.total_steps)) return fail(EM_E_INVAL, "step out of range");
    CKR(set_device(m));
    CKR(drop_prefetch(m));
    if (N) CK(cudaMemcpyAsync(m->N.p, N, m->k * sizeof(float), cudaMemcpyDefault, m->stream));
    if (S)
        CK(cudaMemcpy2DAsync(m->S.p, m->ld * sizeof(float), S, m->d * sizeof(float), m->d * sizeof(float), m->k,
                             cudaMemcpyDefault, m->stream));
    if (c)
        CK(cudaMemcpy2DAsync(m->c.p, m->ld * sizeof(float), c, m->d * sizeof(float), m->d * sizeof(float), m->k,
                             cudaMemcpyDefault, m->stream));
    k_refresh_operand<<<grid_for(m->k * 32, 256, m->sms), 256, 0, m->stream>>>(cluster_state(m), (int)m->k, m->nv);
    CK(cudaGetLastError());
    CKR(after_centroid_change(m));
    if (m->running) {
        // move the run's position to `step` (passes are n rows except a fractional last one)
        m->t = step;
        m->pass = std::min<int64_t>(step / m->rec.steps_full_pass, m->rec.passes - 1);
        const int64_t in_pass = step - m->pass * m->rec.steps_full_pass;
        m->pos = in_pass * m->rec.batch_size;
    }
    CK(cudaStreamSynchronize(m->stream));
    return EM_OK;
}

int em_last_batch(const em_model* m, int64_t* ids, int64_t* labels, float* dists, int64_t* rows) {
    if (!m) return fail(EM_E_INVAL, "model is NULL");
    CKR(set_device(m));
    const int64_t r = m->last_rows;
    if (rows) *rows = r;
    if (r == 0) return EM_OK;
    std::vector<int32_t> tmp(r);
    std::vector<int64_t> wide(r);
    if (ids) {
        CK(cudaMemcpyAsync(tmp.data(), m->slot[(m->t - 1) & 1].ids.p, r * sizeof(int32_t), cudaMemcpyDeviceToHost,
                           m->stream));
        CK(cudaStreamSynchronize(m->stream));
        for (int64_t i = 0; i < r; ++i) wide[i] = tmp[i];
        CK(cudaMemcpy(ids, wide.data(), r * sizeof(int64_t), cudaMemcpyDefault));
    }
    if (labels) {
        CK(cudaMemcpyAsync(tmp.data(), m->labels.p, r * sizeof(int32_t), cudaMemcpyDeviceToHost, m->stream));
        CK(cudaStreamSynchronize(m->stream));
        for (int64_t i = 0; i < r; ++i) wide[i] = tmp[i];
        CK(cudaMemcpy(labels, wide.data(), r * sizeof(int64_t), cudaMemcpyDefault));
    }
    if (dists) {
        CK(cudaMemcpyAsync(dists, m->dists.p, r * sizeof(float), cudaMemcpyDefault, m->stream));
        CK(cudaStreamSynchronize(m->stream));
    }
    return EM_OK;
}

int em_profile(em_model* m, em_profile_t* out, int reset) {
    if (!m) return fail(EM_E_INVAL, "model is NULL");
    CKR(set_device(m));
    CK(cudaStreamSynchronize(m->stream));
    for (auto& sp : m->pending) {
        float ms = 0.0f;
        if (cudaEventElapsedTime(&ms, sp.a, sp.b) == cudaSuccess) {
            m->totals.ms[sp.phase] += ms;
            m->totals.spans[sp.phase] += 1;
            if (sp.phase == EM_PHASE_ASSIGN) m->totals.assign_flops += sp.flops;
            if (sp.phase == EM_PHASE_UPDATE) m->totals.update_bytes += sp.bytes;
            if (sp.phase == EM_PHASE_GATHER) m->totals.gather_bytes += sp.bytes;
        } else {
            cudaGetLastError();
        }
        m->pool.push_back(sp.a);
        m->pool.push_back(sp.b);
    }
    m->pending.clear();
    m->totals.launches = m->launches;
    if (out) *out = m->totals;
    if (reset) {
        m->totals = em_profile_t{};
        m->launches = 0;
    }
    return EM_OK;
}

int em_fp8_converter(const em_model* m, float* shift, float* scale) {
    if (!m) return fail(EM_E_INVAL, "model is NULL");
    if (!m->fp8 || !m->fp8_ready) return fail(EM_E_STATE, "no FP8 converter has been fitted");
    CKR(set_device(m));
    if (shift) {
        CK(cudaMemcpyAsync(shift, m->fp8_shift.p, m->d * sizeof(float), cudaMemcpyDefault, m->stream));
        CK(cudaStreamSynchronize(m->stream));
    }
    if (scale) *scale = m->fp8_scale;
    return EM_OK;
}

int em_dp_unique_id(void* id_out) {
    if (!id_out) return fail(EM_E_INVAL, "NULL argument");
    if (!nccl().ok) return fail(EM_E_COMM, "libnccl.so.2 could not be loaded");
    NCK(nccl().get_id(reinterpret_cast<ncclUniqueId*>(id_out)));
    return EM_OK;
}

int em_dp_init(em_model* m, int world, int rank, const void* id) {
    if (!m || !id) return fail(EM_E_INVAL, "NULL argument");
    if (world < 1 || rank < 0 || rank >= world) return fail(EM_E_INVAL, "need 0 <= rank < world");
    if (m->running) return fail(EM_E_STATE, "a run is in progress");
    if (!nccl().ok) return fail(EM_E_COMM, "libnccl.so.2 could not be loaded");
    CKR(set_device(m));
    CKR(drop_prefetch(m));
    CK(cudaStreamSynchronize(m->stream));
    for (auto& g : m->graph_cache) cudaGraphExecDestroy(g.exec);
    m->graph_cache.clear();
    if (m->comm) {
        nccl().destroy(m->comm);
        m->comm = nullptr;
    }
    ncclUniqueId uid;
    memcpy(&uid, id, sizeof(uid));
    NCK(nccl().init_rank(&m->comm, world, uid, rank));
    m->dp_world = world;
    m->dp_rank = rank;
    m->have_run = false;
    return EM_OK;
}

int em_dp_world(const em_model* m, int* world, int* rank) {
    if (!m) return fail(EM_E_INVAL, "model is NULL");
    if (world) *world = m->dp_world;
    if (rank) *rank = m->dp_rank;
    return EM_OK;
}

int em_sync(em_model* m) {
    if (!m) return fail(EM_E_INVAL, "model is NULL");
    CKR(set_device(m));
    CK(cudaStreamSynchronize(m->stream));
    return check_device_errors(m);
}

int em_selftest(em_model* m, int which, double wait_ms) {
    if (!m) return fail(EM_E_INVAL, "model is NULL");
    if (which != 0 && which != 1) return fail(EM_E_INVAL, "which is 0 (bounded wait) or 1 (index check)");
    if (!(wait_ms > 0.0 && wait_ms <= 10000.0)) return fail(EM_E_INVAL, "wait_ms must be in (0, 10000]");
    CKR(set_device(m));
    CKR(drop_prefetch(m));
    int clock_khz = 1965000;
    cudaDeviceGetAttribute(&clock_khz, cudaDevAttrClockRate, m->dev);
    tc::k_selftest<<<1, 32, 0, m->stream>>>(which, (long long)(wait_ms * (double)clock_khz), m->err.p);
    CK(cudaGetLastError());
    EM_LAUNCHED(m, 1);
    return em_sync(m);
}

}  // extern "C"

// ------------------------------------------------------------------ assignment without allocation
//
// em_assign_noalloc keeps all of its scratch in this file-scope array. In host
// code `g_noalloc_scratch` names a host-side stand-in, not device memory: the
// device address is looked up once per device with cudaGetSymbolAddress.

static __device__ __align__(256) unsigned char g_noalloc_scratch[EM_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr size_t kNaErr = 0;                                                   // int error word
constexpr size_t kNaCn = 256;                                                  // fp32 [MAX_K]
constexpr size_t kNaOperand = kNaCn + (size_t)EM_NOALLOC_MAX_K * 4;            // bf16 [MAX_KD]
constexpr size_t kNaXn = kNaOperand + (size_t)EM_NOALLOC_MAX_KD * 2;           // fp32 [MAX_ROWS]
constexpr size_t kNaKeys = kNaXn + (size_t)EM_NOALLOC_MAX_ROWS * 4;            // u64 [2 * kKeySets * MAX_ROWS]
constexpr size_t kNaBlocks = kNaKeys + (size_t)EM_NOALLOC_MAX_ROWS * 16 * tc::kKeySets;  // fp64 [kNaMaxBlocks]
constexpr int kNaMaxBlocks = 4096;
constexpr size_t kNaEnd = kNaBlocks + (size_t)kNaMaxBlocks * 8;
static_assert(kNaEnd <= EM_NOALLOC_SCRATCH_BYTES, "scratch layout exceeds the array");
static_assert(kNaOperand % 256 == 0 && kNaXn % 256 == 0 && kNaKeys % 256 == 0 && kNaBlocks % 256 == 0,
              "scratch regions must stay 256-byte aligned");

constexpr int kNaMaxDevices = 64;
std::mutex g_na_mu;
unsigned char* g_na_base[kNaMaxDevices] = {};

// Search operand -2 bf16(c) and |bf16(c)|^2 from caller centroids (k x d, d % 8 == 0).
__global__ void k_operand_from_centroids(const float* __restrict__ c, int k, int d, __nv_bfloat16* __restrict__ cq,
                                         float* __restrict__ cn) {
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int nv = d / 8;
    for (int j = warp; j < k; j += nwarps) {
        float part = 0.0f;
        for (int v = lane; v < nv; v += 32) {
            const float4* cr = reinterpret_cast<const float4*>(c + (int64_t)j * d) + 2 * v;
            const float4 a = cr[0], b = cr[1];
            const float cv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            float q[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const float bv = __bfloat162float(__float2bfloat16_rn(cv[t]));
                part = fmaf(bv, bv, part);
                q[t] = -2.0f * bv;
            }
            reinterpret_cast<uint4*>(cq + (int64_t)j * d)[v] = pack8_bf16(q);
        }
        part = warp_sum(part);
        if (lane == 0) cn[j] = part;
    }
}

// Device address of the scratch array on the current device (looked up once).
int noalloc_scratch(int dev, unsigned char** out) {
    if (dev < 0 || dev >= kNaMaxDevices) return fail(EM_E_INVAL, "device index out of range");
    std::lock_guard<std::mutex> lock(g_na_mu);
    if (!g_na_base[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return fail(EM_E_CUDA, "cudaGetSymbolAddress of the scratch array failed: %s", cudaGetErrorString(e));
        }
        if (!search_smem_attributes()) return fail(EM_E_CUDA, "cudaFuncSetAttribute failed");
        g_na_base[dev] = static_cast<unsigned char*>(p);
    }
    *out = g_na_base[dev];
    return EM_OK;
}

}  // namespace

extern "C" int em_assign_noalloc(const void* X, int64_t n, int64_t d, const float* centroids, int64_t k,
                                 int64_t* labels, float* dists, void* stream_) {
    if (!X || !centroids) return fail(EM_E_INVAL, "X and centroids are required");
    if (n < 1 || n > EM_NOALLOC_MAX_ROWS)
        return fail(EM_E_INVAL, "n = %lld is outside [1, %d] rows", (long long)n, EM_NOALLOC_MAX_ROWS);
    if (k < 1 || k > EM_NOALLOC_MAX_K) return fail(EM_E_INVAL, "k = %lld is outside [1, %d]", (long long)k, EM_NOALLOC_MAX_K);
    if (d < 8 || d > 8192 || d % 8 != 0) return fail(EM_E_INVAL, "d must be a multiple of 8 in [8, 8192]");
    if (k * d > EM_NOALLOC_MAX_KD) return fail(EM_E_INVAL, "k * d = %lld exceeds %d", (long long)(k * d), EM_NOALLOC_MAX_KD);
    if ((reinterpret_cast<uintptr_t>(X) & 15) || (reinterpret_cast<uintptr_t>(centroids) & 15))
        return fail(EM_E_INVAL, "X and centroids must be 16-byte aligned");
    if (!is_device_ptr(X) || !is_device_ptr(centroids) || (labels && !is_device_ptr(labels)) ||
        (dists && !is_device_ptr(dists)))
        return fail(EM_E_INVAL, "em_assign_noalloc takes device pointers only");
    int dev = 0;
    CK(cudaGetDevice(&dev));
    unsigned char* base = nullptr;
    CKR(noalloc_scratch(dev, &base));
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int sms = 148, clock_khz = 1965000;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&clock_khz, cudaDevAttrClockRate, dev);
    int* err = reinterpret_cast<int*>(base + kNaErr);
    float* cn = reinterpret_cast<float*>(base + kNaCn);
    __nv_bfloat16* cq = reinterpret_cast<__nv_bfloat16*>(base + kNaOperand);
    float* xn = reinterpret_cast<float*>(base + kNaXn);
    unsigned long long* keys = reinterpret_cast<unsigned long long*>(base + kNaKeys);
    double* blocks = reinterpret_cast<double*>(base + kNaBlocks);
    const int kc = (d % 64 == 0) ? 64 : 32;
    CUtensorMap tmA, tmB;
    CKR(make_tmap(&tmA, X, n, (int)d, (int)d, tc::BM, kc));
    CKR(make_tmap(&tmB, cq, k, (int)d, (int)d, tc::BN, kc));
    const auto X16 = reinterpret_cast<const __nv_bfloat16*>(X);
    CK(cudaMemsetAsync(err, 0, sizeof(int), stream));  // the previous call's error word is stale
    k_operand_from_centroids<<<grid_for(k * 32, 256, sms), 256, 0, stream>>>(centroids, (int)k, (int)d, cq, cn);
    k_rownorm<<<grid_for(n * 32, 256, sms), 256, 0, stream>>>(X16, n, (int)d, xn);
    const int64_t m_tiles = (n + tc::BM - 1) / tc::BM;
    const int64_t n_tiles = (k + tc::BN - 1) / tc::BN;
    const int nkc = (int)((d + kc - 1) / kc);
    // the key region holds 2 keys per key set for each of EM_NOALLOC_MAX_ROWS rows, and
    // the search writes 2 keys per key set for each of its n rows in each of its split
    // centroid-tile groups: split * n <= EM_NOALLOC_MAX_ROWS
    const Schedule sc = choose_schedule(m_tiles, n_tiles, sms,
                                        (int)std::max<int64_t>(1, EM_NOALLOC_MAX_ROWS / n));
    const bool top2 = d >= 256;
    const int grid = (int)std::min<int64_t>(sc.m_full + (m_tiles - sc.m_full) * sc.split, sms);
    const long long wait_cycles = (long long)(2000.0 * (double)clock_khz);
    launch_search(kc, top2, ast_fits(d, kc), grid, static_cast<cudaStream_t>(stream), tmA, tmB, cn, (int)k, (int)n,
                  nkc, (int)n_tiles, sc, keys, wait_cycles, err);
    const int oblocks = std::min(grid_for(n, 256, sms), kNaMaxBlocks);
    k_assign_out<<<oblocks, 256, 0, stream>>>(keys, sc.split * tc::kKeySets, xn, n, (int)k, X16, (int)d, cq, labels,
                                             dists, nullptr, blocks, kSquaredDistance, ScoreScale{1.0f, 1.0f, kTieRel},
                                             TieList{nullptr, nullptr, nullptr}, err);
    CK(cudaGetLastError());
    int h = 0;
    CK(cudaMemcpyAsync(&h, err, sizeof(int), cudaMemcpyDeviceToHost, stream));
    CK(cudaStreamSynchronize(stream));
    if (h != 0) return fail(h, "device-side error %d in the assignment", h);
    return EM_OK;
}
