/*
 * emeans.h -- C ABI of the B200 e-means library (mini-batch EMA k-means).
 *
 * The method and its interface are those of the faiss e-means README
 * ("e-means: outperforming k-means in one-tenth the epochs"): the model is
 * built from (d, k, seed) as in its section "Settings and results"
 * (`Emeans(d, k, nepochs=5, seed=1234)`), trained with `train(x)` and queried
 * with `assign(x)`; the manual loop of its section "Data too big for memory"
 * (begin / accumulate+update / end_epoch / finalize) is exposed as
 * em_begin / em_step / em_finalize.
 *
 * Conventions shared by every entry point
 *  - Return value: EM_OK (0) on success, a negative EM_E_* code on failure.
 *    em_last_error() then returns a message for the calling thread.
 *  - Matrices are row-major, rows contiguous: X is n x d, centroids k x d.
 *  - Pointers may be host or device memory (CUDA unified addressing is used
 *    to tell them apart). Host input is copied to the device inside the call;
 *    host output is written after the device work of the call has finished.
 *    Device pointers must belong to the model's device. Pointers are never
 *    retained after a call returns, except the X given to em_begin (see there).
 *  - All device work is ordered on the model's stream (em_set_stream; by
 *    default a stream the model creates). Calls that return data to a host
 *    pointer synchronise that stream; the others do not.
 *  - Nothing is checked for NaN or infinity unless EM_OPT_CHECK_FINITE is set
 *    (the README, section "Data and centroids fit on 1 GPU", documents the GPU
 *    path as unchecked).
 *  - There is no CPU fallback: without a CUDA device every compute entry point
 *    fails with EM_E_NODEVICE.
 */
#ifndef EMEANS_H
#define EMEANS_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---- */
#define EM_OK 0
#define EM_E_INVAL (-1)     /* bad argument (sizes, pointers, option values)          */
#define EM_E_NOMEM (-2)     /* device or pinned-host allocation failed                */
#define EM_E_CUDA (-3)      /* a CUDA runtime call failed                             */
#define EM_E_BOUNDS (-4)    /* a kernel's own index check caught an out-of-range index */
#define EM_E_TIMEOUT (-5)   /* a bounded device-side wait gave up                     */
#define EM_E_NONFINITE (-6) /* EM_OPT_CHECK_FINITE found NaN or infinity in the input */
#define EM_E_STATE (-7)     /* call out of order (e.g. em_step before em_begin)       */
#define EM_E_NODEVICE (-8)  /* no CUDA device is present                              */
#define EM_E_COMM (-9)      /* the collective library (NCCL) is missing or a call failed */

/* ---- options (em_set_option / em_get_option; values are doubles) ---- */
enum em_option {
    EM_OPT_BATCH_SIZE = 1,       /* 0 (default): from the scaling law; else the batch size,
                                    and alpha0 follows equation (3) (README "Manual overrides") */
    EM_OPT_ALPHA0 = 2,           /* 0 (default): from equation (3); else the starting step    */
    EM_OPT_UNUSED_THRESHOLD = 3, /* tau: revive clusters whose running count is below tau x the
                                    mean count (README `unused_threshold`). 0 = off; -1
                                    (default): 0.1, or 0 for d <= 2 (README "Note on low
                                    dimension")                                              */
    EM_OPT_REVIVAL = 4,          /* 0 none, 1 split a size-proportional donor (default),
                                    2 resample from the current batch                          */
    EM_OPT_FINALIZE = 5,         /* 1 (default): closing mean at the end of the last pass; 0 off */
    EM_OPT_LAW = 6,              /* 0 "throughput" law (1); 1 "quality" law (2); 2 "auto"
                                    (default): quality for d <= 16, else throughput (README
                                    `batch_law`, "Note on low dimension")                      */
    EM_OPT_INPUT_DTYPE = 7,      /* dtype of X: 0 fp32 (default), 1 bf16                       */
    EM_OPT_CHECK_FINITE = 8,     /* 1: scan X for NaN/Inf in em_begin/em_train (EM_E_NONFINITE) */
    EM_OPT_WAIT_LIMIT_MS = 9,    /* limit of every device-side spin wait, ms (default 2000)    */
    EM_OPT_AUTO_REVIVE = 10,     /* 1 (default): em_step runs the revival check after every 5th
                                    step; 0: only em_revive does (step-by-step inspection)      */
    EM_OPT_CAPTURE_LABELS = 11,  /* 1 (default): keep each row's last-pass label (em_labels)   */
    EM_OPT_GRAPHS = 12,          /* 1 (default): em_step replays CUDA graphs of whole steps     */
    EM_OPT_ASSIGN_KERNEL = 13,   /* 0 (default): tcgen05 tensor-core assignment; 1: a plain
                                    SIMT kernel kept only to localise faults in tests           */
    EM_OPT_PROFILE = 14,         /* 1: bracket every phase of every step with CUDA events on the
                                    model's stream (read with em_profile); 0 (default): off     */
    EM_OPT_EXACT_TIES = 15,      /* 1: the search also keeps each row's second best centroid and
                                    rows whose two best fp32 scores are within the accumulation
                                    error are settled with exact fp64 distances; 0: plain fp32
                                    argmin; -1 (default): on when d >= 256                       */
    EM_OPT_SPHERICAL = 16,       /* 1: spherical e-means (README "Spherical e-means"): every
                                    centroid is rescaled to norm 1 before each use (a zero
                                    centroid stays zero), each row goes to the centroid with the
                                    highest dot product, the closing mean is rescaled to norm 1,
                                    and the error of a row is 2 - 2 x its similarity. The rows
                                    are used as given: normalise them first for cosine
                                    similarity. 0 (default): k-means. Not changeable during a run */
    EM_OPT_PREFETCH = 17,        /* 1 (default): while a step updates the centroids, the rows of
                                    the next step are gathered into a second batch buffer on a
                                    second stream the model owns; 0: each step gathers its own
                                    rows first. Off while EM_OPT_PROFILE is on                  */
    EM_OPT_SEARCH_FORMAT = 18,   /* 0 (default): the search runs on bf16 copies; 1: on FP8 (E4M3)
                                    codes (README "Data precision"): a converter fitted on the
                                    first 65,536 rows of each run's data holds a shift per
                                    dimension (the midrange) and one power-of-two scale (the
                                    largest keeping the sample within 448); rows and centroids
                                    are searched as e4m3((v - shift) * scale), saturating at
                                    448, on the tensor cores' FP8 path. Counts, sums and
                                    centroids stay fp32 (sums of the bf16 rows); distances are
                                    reported in the data's units. Not with spherical e-means or
                                    the SIMT search; near ties are not settled exactly. Not
                                    changeable during a run; em_assign on a model without a
                                    converter fits one on its own rows                          */
    EM_OPT_PDL = 19              /* 1 (default): the kernels of a step launch with programmatic
                                    stream serialization, each starting while its predecessor
                                    finishes and waiting for it on the device; 0: plain launches */
};

/* Phases timed by EM_OPT_PROFILE (em_profile_t.ms / spans index). */
#define EM_PHASE_PREPARE 0   /* input copy / cast, starting centroids                        */
#define EM_PHASE_GATHER 1    /* batch gather in the per-pass order                            */
#define EM_PHASE_ASSIGN 2    /* fused nearest-centroid search                                 */
#define EM_PHASE_UPDATE 3    /* labels, grouping by label, segmented sums + EMA update        */
#define EM_PHASE_REVIVE 4    /* dead-cluster revival                                           */
#define EM_PHASE_FINALIZE 5  /* closing mean                                                   */
#define EM_NPHASES 6

/* revival modes for EM_OPT_REVIVAL */
#define EM_REVIVE_NONE 0
#define EM_REVIVE_SPLIT 1
#define EM_REVIVE_RESAMPLE 2

/* Training recipe (README "Scaling laws" and "Settings and results": batch_size,
 * alpha0, steps_per_pass, epoch_rows). Every pass but a fractional last one has n rows. */
typedef struct em_recipe_t {
    int64_t n, k, d;
    double epochs;
    double batch_raw;        /* equation (1)/(2) before rounding (or the manual size)        */
    int64_t batch_size;      /* nearest power of two in log2, capped at the largest <= n/2  */
    double alpha0;           /* equation (3), clamped to [1e-4, 1] (or the manual value)    */
    int64_t passes;          /* ceil(epochs)                                                  */
    int64_t rows_last_pass;  /* n, or round(frac(epochs) * n) for a fractional last pass      */
    int64_t steps_full_pass; /* ceil(n / batch_size)                                          */
    int64_t steps_last_pass; /* ceil(rows_last_pass / batch_size)                             */
    int64_t total_steps;     /* sum over passes                                               */
} em_recipe_t;

/* Counters kept on the model (README "Settings and results": iteration_stats, n_splits). */
typedef struct em_stats_t {
    int64_t steps_done;      /* mini-batch steps run since em_begin                          */
    int64_t passes_done;     /* completed passes                                              */
    int64_t rows_assigned;   /* rows assigned by training steps since em_begin                */
    int64_t n_splits;        /* dead clusters revived since em_begin                         */
    int64_t last_dead;       /* clusters found dead at the most recent revival check          */
    double imbalance;        /* max(N) / mean(N) after the most recent step                   */
    double last_alpha;       /* step size of the most recent step                             */
} em_stats_t;

/* Device time per phase and launch counts (EM_OPT_PROFILE). */
typedef struct em_profile_t {
    double ms[EM_NPHASES];      /* summed span durations, CUDA events on the model's stream      */
    int64_t spans[EM_NPHASES];  /* number of spans timed per phase                               */
    int64_t launches;           /* kernels launched by the library (counted with or without
                                   EM_OPT_PROFILE)                                               */
    double assign_flops;        /* 2 * rows * k * d summed over the timed assignment spans      */
    double update_bytes;        /* algorithmic bytes of the timed update spans:
                                   2*rows*d (batch rows) + 16*rows (keys, labels, order)
                                   + 14*k*d (S read + write, c fp32 and bf16 writes)            */
    double gather_bytes;        /* 4*rows*d: batch rows read and written (bf16)                  */
} em_profile_t;

/* ---- library ---- */

/* Message of the last failing call on this thread ("" if none). Never NULL. */
const char* em_last_error(void);

/* EM_E_* code of the last failing call on this thread (0 if none): what a call
 * that returns a pointer (em_create: NULL) failed with. */
int em_last_error_code(void);

/* Allocation-failure injection, for testing the out-of-memory paths without
 * running out of memory (host code, no device work).
 * After em_fail_allocation(nth), nth >= 1, the nth device allocation the library
 * attempts (in any thread, counting from 1) fails as a failed cudaMalloc does,
 * without calling it: the call that made it returns EM_E_NOMEM (em_create:
 * NULL). The allocations after it run normally. nth <= 0 switches injection off.
 * Returns the number of device allocations the library attempted since the
 * previous em_fail_allocation call, so a test can count a sequence of calls'
 * allocations and then fail each in turn. A model whose call failed this way can
 * be destroyed, or used again (em_begin / em_train re-acquire what they need). */
int64_t em_fail_allocation(int64_t nth);

/* Number of CUDA devices visible to the library (0 without a GPU). Host-only. */
int em_device_count(void);

/* Host-only helpers that run the library's own host code, for checking it
 * without a GPU. em_compute_recipe evaluates equations (1)-(3) and the rounding
 * rules (README "Scaling laws", "Manual overrides"); law 0 = throughput,
 * 1 = quality; batch_override <= 0 and alpha_override <= 0 mean "from the law". */
int em_compute_recipe(int64_t n, int64_t k, double epochs, int law, int64_t batch_override,
                      double alpha_override, em_recipe_t* out);

/* The library's per-pass order: out[i] = pi(idx[i]) for the keyed bijection on
 * [0, n) selected by (seed, stream, which): stream 1 = starting rows (which = 0),
 * stream 2 = pass order (which = pass index). Same code as the device kernels. */
int em_permutation(int64_t n, uint64_t seed, int stream, int64_t which, const int64_t* idx,
                   int64_t count, int64_t* out);

/* The rows that rank `rank` of `world` takes at each of the first `count` steps of a
 * data-parallel run over n_local rows per rank (README "Several GPUs": the recipe
 * is that of all ranks' rows, n_local x world, and each batch is split evenly; the
 * pages' loop has every rank take positions [start / world, (start + B) / world)
 * of its own fresh random order of its own rows each pass). Host code only: the
 * same functions that plan em_step's batches and gathers. For step t: pass[t] is
 * the pass, first[t] and rows[t] the positions [first, first + rows) of the
 * rank's order that it takes, key[t] the key of that order (em_permutation with
 * stream 2 and which = key[t]: the pass plus rank x 2^32). law, batch_override and
 * alpha_override as in em_compute_recipe. EM_E_INVAL for bad sizes, a rank
 * outside [0, world), count beyond the run's steps, NULL outputs, or a batch or
 * last pass that does not divide by world (em_begin's check). */
int em_dp_schedule(int64_t n_local, int64_t k, double epochs, int law, int64_t batch_override,
                   double alpha_override, int64_t world, int64_t rank, int64_t count, int64_t* pass,
                   int64_t* first, int64_t* rows, int64_t* key);

/* The work split of the nearest-centroid search that em_train, em_step, em_lloyd,
 * em_assign and em_mse use for `rows` rows and k centroids on a device with `sms`
 * SMs (host code, no device work; em_assign_noalloc may split less, to fit its
 * fixed key region). The search's units are 128-row tiles times groups of 256-wide
 * centroid tiles: the first *m_full row tiles are one unit each, over all of k,
 * and every later row tile is *split units (1, 2, 4 or 8). EM_E_INVAL for rows, k
 * or sms below 1 or a NULL output. */
int em_search_schedule(int64_t rows, int64_t k, int sms, int* split, int* m_full);

/* ---- model ---- */

/* New model for k clusters of d-dimensional vectors on the current CUDA device
 * (README "Settings and results": only d and k are required; seed seeds the
 * starting centroids, the per-pass order and the revivals; the README default is
 * 1234). Returns NULL on failure (em_last_error). d in [1, 8192], k >= 1. */
struct em_model;
typedef struct em_model em_model;
em_model* em_create(int64_t d, int64_t k, uint64_t seed);

/* Frees every device and host buffer of the model. NULL is ignored. */
void em_destroy(em_model* m);

int em_set_option(em_model* m, int opt, double value);
int em_get_option(const em_model* m, int opt, double* value);

/* Orders all later work of the model on `stream` (a cudaStream_t; NULL = the
 * legacy default stream). The model does not take ownership. */
int em_set_stream(em_model* m, void* stream);

/* ---- training (README "Quick start", "Data and centroids fit on 1 GPU") ---- */

/* Trains on X (n x d rows, dtype per EM_OPT_INPUT_DTYPE) for `epochs` passes
 * (fractional allowed): em_begin + em_step until done + em_finalize. Needs
 * n >= k. Afterwards em_centroids / em_labels / em_stats / em_obj hold the
 * results. Synchronises the stream and reports device-side errors. */
int em_train(em_model* m, const void* X, int64_t n, double epochs);

/* Starts a run: computes the recipe, makes the bf16 search copy of X (fp32 input
 * is rounded to nearest-even; README "Data precision"), picks k distinct rows as
 * starting centroids (README: random data points, no k-means++) and zeroes the
 * running counts and sums. A device bf16 X whose rows are 16-byte aligned
 * (d % 8 == 0) is used in place and must stay valid and unchanged until the
 * run ends (em_finalize or the next em_begin); any other X is copied. */
int em_begin(em_model* m, const void* X, int64_t n, double epochs);

/* Runs up to `nsteps` further mini-batch steps of the run (assignment of the
 * batch, per-cluster count and sum, EMA update with the cosine step size and,
 * every 5th step, the revival check; README "How the centroid updates work").
 * *done (may be NULL) receives the number of steps run. Does not synchronise. */
int em_step(em_model* m, int64_t nsteps, int64_t* done);

/* Ends the run: applies the closing mean if EM_OPT_FINALIZE is on (each
 * centroid becomes the exact mean of the rows the last pass assigned to it;
 * clusters without such rows keep their EMA centroid). Synchronises. */
int em_finalize(em_model* m);

/* Runs the revival check for the most recent step now (for EM_OPT_AUTO_REVIVE
 * = 0). The batch of that step is the one resampling draws from. */
int em_revive(em_model* m);

/* Lloyd's k-means (README "How the centroid updates work": the whole dataset as
 * one batch with a step of 1) for `iters` iterations, from the same starting
 * rows em_begin would pick for this seed. Natural row order, no revival. The
 * centroids are left on the model. */
int em_lloyd(em_model* m, const void* X, int64_t n, int64_t iters);

/* ---- queries ---- */

/* Nearest centroid of every row of X (README "Settings and results":
 * `assign` returns each vector's nearest centroid and its squared distance).
 * labels: n int64 (may be NULL); dists: n fp32 squared distances computed with
 * the bf16 search copies and clamped at 0 (may be NULL). Ties go to the lowest
 * centroid index. With EM_OPT_SPHERICAL, the centroid of highest dot product and
 * dists = that dot product x . bf16(c) (README "Spherical e-means": higher is
 * closer). */
int em_assign(em_model* m, const void* X, int64_t n, int64_t* labels, float* dists);

/* Mean over the rows of X of the squared distance to the nearest centroid
 * (fp64 accumulation), as em_assign measures it; with EM_OPT_SPHERICAL, the mean
 * of 2 - 2 x the highest similarity. Synchronises. */
int em_mse(em_model* m, const void* X, int64_t n, double* out);

/* Copies the k x d fp32 centroids into out. */
int em_centroids(const em_model* m, float* out);

/* Copies each training row's label from the last pass (int64; -1 for rows a
 * fractional last pass did not visit) into out (n entries of the last run). */
int em_labels(const em_model* m, int64_t* out);

int em_recipe(const em_model* m, em_recipe_t* out);
int em_stats(const em_model* m, em_stats_t* out);

/* Error of each completed pass, measured while the centroids move (README
 * `obj`): mean squared distance of the pass's rows at the time they were
 * assigned (spherical: mean of 2 - 2 x similarity). Writes up to cap values;
 * *count receives the number available. */
int em_obj(const em_model* m, double* out, int64_t cap, int64_t* count);

/* Model state: running counts N (k fp32), running sums S (k x d fp32),
 * centroids c (k x d fp32) and the global step counter. Any pointer may be
 * NULL. em_set_state replaces the state of the current run (checkpoint resume,
 * step-by-step comparison); the bf16 search copy is refreshed from c (with
 * EM_OPT_SPHERICAL, c is first rescaled to norm 1). */
int em_get_state(const em_model* m, float* N, float* S, float* c, int64_t* step);
int em_set_state(em_model* m, const float* N, const float* S, const float* c, int64_t step);

/* The most recent training batch: its row ids (int64), labels (int64), squared
 * distances (fp32; spherical: 2 - 2 x similarity) and row count. Any pointer may
 * be NULL. */
int em_last_batch(const em_model* m, int64_t* ids, int64_t* labels, float* dists, int64_t* rows);

/* Synchronises the model's stream, adds the pending event spans to the totals and
 * copies the totals to *out; reset != 0 clears them (and the launch count). */
int em_profile(em_model* m, em_profile_t* out, int reset);

/* ---- assignment without any allocation ----
 *
 * (k-means only: squared distances to centroids taken as given.)
 * The paper has no counterpart to this entry point. It serves callers that cannot
 * call cudaMalloc: code whose device memory is owned by another allocator or fixed
 * up front (a serving process that forbids allocation after start-up, a library
 * running inside a framework's memory pool), or that runs where an allocation would
 * be an error. It computes the same labels and squared distances as em_assign, with
 * the same kernels, but needs no model and allocates nothing: its scratch (search
 * operand, norms, per-row keys, error word) is one file-scope __device__ array of
 * EM_NOALLOC_SCRATCH_BYTES that every GPU which loads the library holds until exit.
 *
 * X: device bf16, n x d row-major, 16-byte aligned, d a multiple of 8 (read in
 * place). centroids: device fp32, k x d, 16-byte aligned. labels (int64, n) and
 * dists (fp32, n) are device outputs; either may be NULL. stream: a cudaStream_t
 * (NULL = legacy default stream). Sizes beyond the limits below return EM_E_INVAL;
 * host pointers return EM_E_INVAL.
 *
 * The first call on a device looks up the array's device address (and sets the
 * kernels' shared-memory limits); make that first call before any stream capture.
 * Every call shares the one array, which keeps the previous call's contents: calls
 * that overlap on the GPU (other threads, other streams) race and must be ordered
 * by the caller. The call waits for `stream` before it returns, to report
 * device-side errors. */
#define EM_NOALLOC_MAX_ROWS 524288
#define EM_NOALLOC_MAX_K 65536
#define EM_NOALLOC_MAX_KD 4194304 /* k * d */
#define EM_NOALLOC_SCRATCH_BYTES 28311552 /* 27 MiB */
int em_assign_noalloc(const void* X, int64_t n, int64_t d, const float* centroids, int64_t k, int64_t* labels,
                      float* dists, void* stream);

/* Waits for the model's stream and reports device-side errors (EM_E_BOUNDS,
 * EM_E_TIMEOUT) raised since the last check. */
int em_sync(em_model* m);

/* Exercises the failure path without a fault: which = 0 runs the search kernel's
 * bounded mbarrier wait on a barrier nothing arrives on, which gives up after
 * wait_ms and returns EM_E_TIMEOUT; which = 1 raises the index-check error and
 * returns EM_E_BOUNDS. The error word is cleared when reported, so the model stays
 * usable. wait_ms in (0, 10000]. */
int em_selftest(em_model* m, int which, double wait_ms);

/* The FP8 converter of the model (EM_OPT_SEARCH_FORMAT = 1) fitted by the last
 * em_begin / em_lloyd (or first em_assign): the shift of each dimension (d fp32
 * values, host or device pointer, may be NULL) and the power-of-two scale.
 * EM_E_STATE before any fit. */
int em_fp8_converter(const em_model* m, float* shift, float* scale);

/* ---- data parallelism (README "Several GPUs": DistributedEmeans) ----
 *
 * One process per GPU, each holding its own share of the rows. After em_dp_init,
 * em_begin / em_train / em_lloyd take this rank's rows (X, n): the recipe is
 * computed for the rows of all ranks (n x world), every batch is split evenly
 * across the ranks (each takes its share of a batch from its own per-pass order
 * of its own rows; rank r's order is keyed by the pass and r), the ranks' per-
 * cluster statistics (n_j, s_j, fp64, with the batch error) are added with one
 * NCCL all-reduce per step on the model's stream, and every rank applies the same
 * EMA update and revival, so all ranks hold the same model. Rank 0's starting
 * centroids are used (one broadcast at em_begin). Sums of bf16 rows in fp64 are
 * exact, so the result does not depend on the order the ranks' sums are added
 * in; with world = 1 a run equals the single-GPU run bit for bit.
 *
 * Requirements (README "Several GPUs"): every rank makes the same calls with the
 * same options and the same n; the batch size and the rows of every pass divide by
 * world (em_begin returns EM_E_INVAL otherwise); resampling revival needs world = 1.
 * em_assign / em_mse / em_labels stay local to the rank's rows.
 *
 * NCCL is loaded at run time (libnccl.so.2 already in the process, else the first
 * on the library path); without it these calls return EM_E_COMM. */
#define EM_NCCL_ID_BYTES 128

/* Writes a fresh communicator id (EM_NCCL_ID_BYTES bytes) to id_out. Rank 0 calls
 * it and hands the bytes to the other ranks by any means (a torch.distributed
 * broadcast, a file). Host-only. */
int em_dp_unique_id(void* id_out);

/* Joins the model to the communicator `id` as `rank` of `world` ranks, on the
 * model's device (collective: every rank calls it). Replaces an earlier
 * communicator; not allowed during a run. */
int em_dp_init(em_model* m, int world, int rank, const void* id);

/* The model's world size and rank (1 and 0 without em_dp_init). */
int em_dp_world(const em_model* m, int* world, int* rank);

#ifdef __cplusplus
}
#endif
#endif /* EMEANS_H */
