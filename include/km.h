/*
 * km.h -- C ABI of libkm.so: one batched exact Lloyd k-means iteration on an
 * NVIDIA B200 (sm_100a), in hand-written CUDA.
 *
 * The method is Flash-KMeans as described on the papernotes.org page
 * "Flash-KMeans: Fast and Memory-Efficient Exact K-Means" (method section
 * 方法详解): an iteration is an assignment step (FlashAssign, 关键设计 1) and
 * an update step (Sort-Inverse Update, 关键设计 2), repeated (整体框架 and its
 * flowchart).  The result is exactly Lloyd's k-means; only the data movement
 * differs (7minutos.es article, opening section).
 *
 * Conventions shared by every entry point
 *   - All arrays are dense and row-major.  X is [B, N, d] in `dtype`;
 *     centroids C, C_init, C_out and sums are [B, K, d] fp32; labels, mindist
 *     and sorted_idx are [B, N]; counts is [B, K]; offsets is [B, K + 1].
 *     Labels and sorted indices are 0-based and index within their batch.
 *   - The B problems are independent; each has its own K centroids.
 *   - Pointers are device pointers unless stated otherwise; the caller owns
 *     (allocates and frees) every array it passes.  Scratch memory is taken
 *     stream-ordered from the library's memory pool on `stream` and released
 *     to it before return on the same stream (see km_release_cached).  No
 *     other state survives a call except a per-device cache of the capability
 *     check.
 *   - `stream` is a cudaStream_t (NULL means the legacy default stream).
 *     Every call is asynchronous on it: results are ready once the stream is
 *     synchronised.  Argument errors return before any work is enqueued.
 *   - Supported: B >= 1, N >= 1, K >= 1, B*N < 2^31, K < 2^24, 1 <= d <= 16384,
 *     d * sizeof(dtype) a multiple of 16 bytes, X and the [B, K, d] arrays
 *     (C, C_init, C_out, sums) 16-byte aligned, every other array 4-byte
 *     aligned, a device of compute capability 10.0.
 *     Anything else returns KM_E_UNSUPPORTED (KM_E_INVALID for null pointers
 *     and non-positive sizes).  There is no CPU fallback.
 *   - Inputs must be finite; non-finite values are outside the contract.
 */
#ifndef KM_H
#define KM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KM_API __attribute__((visibility("default")))
#else
#define KM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { KM_F32 = 0, KM_F16 = 1 } km_dtype;

typedef enum {
    KM_OK = 0,
    KM_E_INVALID = 1,     /* null pointer, non-positive size, unknown dtype */
    KM_E_UNSUPPORTED = 2, /* shape, alignment or device outside the supported range */
    KM_E_NOMEM = 3,       /* scratch allocation failed */
    KM_E_CUDA = 4,        /* a CUDA call or kernel launch failed */
    KM_E_TIMEOUT = 5      /* a bounded wait expired (see km_device_fault) */
} km_status;

/*
 * Assignment step (FlashAssign; papernotes.org page, 关键设计 1).
 * For every point x_i of every batch:
 *     labels[b][i]  = argmin_k ||x_i - c_k||^2, the lowest k among equal distances,
 *     mindist[b][i] = that minimum squared distance (clamped at 0).
 * The distance is expanded as ||x||^2 + ||c||^2 - 2 x.c; the N x K distance
 * matrix is never written to memory.  The centroids are first rounded
 * (round-to-nearest-even) to `dtype`, and x.c is accumulated in fp32:
 *   - fp16, 64 <= d <= 128: on the tensor cores;
 *   - fp16, d in {192, 256, ..., 512}: on the tensor cores, the centroids
 *     streamed in 64-dimension chunks;
 *   - fp16, d a multiple of 64 above 512 (the split-D path of the 7minutos.es
 *     article, "Usándolo"): on the tensor cores, points and centroids both
 *     streamed in 64-dimension chunks, each point chunk meeting 512 centroids;
 *   - fp32, d in {32, 64, 96, 128}: on the tensor cores from tf32 head/tail
 *     splits of both operands (three products);
 *   - other shapes: direct differences sum_j (x_j - c_j)^2 on the CUDA cores.
 * On the tensor-core paths each point's label is certified against the
 * rounding-error bound of its scores, from its best two scores; a point that
 * is not certified (near ties, near-duplicate centroids, data far from the
 * origin, fp16 centroid norms beyond the folded norm term's range of ~3.4e10)
 * is re-scanned exactly on the CUDA cores (see km_assign_rescans).  So every fp32 label is the exact argmin up
 * to fp32 rounding, and every fp16 label is the exact argmin unless the two
 * smallest exact distances d1 <= d2 of the point satisfy d2 - d1 < 1e-3 d2,
 * in which case its distance is within 1e-3 d2 of d1.
 *   X       [B, N, d] dtype, device.     C [B, K, d] fp32, device.
 *   labels  [B, N] int32, device, written.
 *   mindist [B, N] fp32, device, written; may be NULL.
 */
KM_API km_status km_assign(const void* X, const float* C, int64_t B, int64_t N, int64_t K, int64_t d, int dtype,
                    int32_t* labels, float* mindist, void* stream);

/*
 * Label argsort (papernotes.org page, 关键设计 2: the labels alone are sorted;
 * X is never permuted).  A stable device sort of each batch's labels (one
 * launch, a thread-block cluster per batch, for N <= 65536 and K <= 1024;
 * otherwise an LSD radix sort):
 *   sorted_idx[b][p] = index of the point at sorted position p (ascending
 *                      label, ties by ascending point index; unique),
 *   counts[b][k]     = number of points with label k,
 *   offsets[b][k]    = first sorted position of label k (offsets[b][K] = N).
 * Labels must lie in [0, K); others give undefined (but in-bounds) output.
 *   labels [B, N] int32, device.  sorted_idx [B, N] int32, device, written.
 *   counts [B, K] int32, device, written.  offsets [B, K+1] int32, device,
 *   written; may be NULL.
 */
KM_API km_status km_sort_labels(const int32_t* labels, int64_t B, int64_t N, int64_t K, int32_t* sorted_idx,
                         int32_t* counts, int32_t* offsets, void* stream);

/*
 * Update step (Sort-Inverse Update; papernotes.org page, 关键设计 2).
 * Sorts the labels, then each CTA walks a fixed run of sorted positions,
 * gathers the rows of X through the sorted indices, reduces each cluster's
 * rows on chip, and adds to global memory atomically only for the clusters
 * that cross its run boundaries:
 *   sums[b][k]   = sum of the rows labelled k (fp32 accumulation),
 *   counts[b][k] = their number,
 *   C_out[b][k]  = sums / counts if counts > 0, else unchanged.
 * C_out is in/out: on entry it holds the previous centroids (an empty cluster
 * keeps its centroid, bit for bit); it must not alias X, sums or labels.
 *   X [B, N, d] dtype, device.  labels [B, N] int32 in [0, K), device.
 *   sums [B, K, d] fp32, device, written.  counts [B, K] int32, device, written.
 *   C_out [B, K, d] fp32, device, read and written.
 */
KM_API km_status km_update(const void* X, const int32_t* labels, int64_t B, int64_t N, int64_t K, int64_t d, int dtype,
                    float* sums, int32_t* counts, float* C_out, void* stream);

/*
 * `iters` Lloyd iterations (assign, sort, update), all enqueued on `stream`
 * with no host synchronisation inside the loop (papernotes.org page, 整体框架:
 * the loop returns to the assignment until the iteration budget is spent).
 *   X        [B, N, d] dtype, device memory; or pinned host memory
 *            (cudaHostAlloc / cudaHostRegister), in which case it is streamed
 *            to the device in chunks of rows with copies overlapped with the
 *            computation (papernotes.org page, 关键设计 3).
 *   C_init   [B, K, d] fp32, device.  C_out [B, K, d] fp32, device, written
 *            (may equal C_init).
 *   labels   [B, N] int32: the assignment of the LAST iteration, made against
 *            the centroids before its update; device memory, or pinned host
 *            memory when X is host memory.
 *   objective [iters, B] fp32, device, may be NULL: per iteration and batch,
 *            the sum of the assignment's minimum distances.
 * iters = 0 copies C_init to C_out.
 */
KM_API km_status km_lloyd(const void* X, const float* C_init, int64_t B, int64_t N, int64_t K, int64_t d, int dtype,
                   int iters, int32_t* labels, float* C_out, float* objective, void* stream);

/*
 * km_lloyd until convergence (papernotes.org page, 整体框架 flowchart:
 * iterate "until converged or the maximum number of iterations").  After each
 * iteration the device sums, per batch, the squared shift of the centroids,
 * shift_b = sum_k ||c_new - c_old||^2 (empty clusters do not move), and the
 * loop stops once every batch has shift_b <= tol -- the decision is taken on
 * the device: all max_iters iterations are enqueued at once and those after
 * the stop return immediately (no host synchronisation per iteration).  All
 * batches run the same number of iterations.  tol = 0 asks for an exact fixed
 * point (no centroid moved); the update combines the partial sums of a
 * cluster that spans several CTA runs with fp32 atomics, whose order can
 * change the last bit from one iteration to the next, so a tol slightly above
 * 0 is the robust way to ask for a settled state.
 *   X        [B, N, d] dtype, device memory only (else KM_E_UNSUPPORTED).
 *   iters_run int32, device, written: the number of iterations performed
 *            (1..max_iters); labels, C_out and objective rows [0, iters_run)
 *            are those of km_lloyd with iters = iters_run; later objective
 *            rows are not written.
 * Other arguments as km_lloyd.  max_iters >= 1 and tol >= 0 (else
 * KM_E_INVALID).
 */
KM_API km_status km_lloyd_tol(const void* X, const float* C_init, int64_t B, int64_t N, int64_t K, int64_t d,
                              int dtype, int max_iters, double tol, int32_t* labels, float* C_out, float* objective,
                              int32_t* iters_run, void* stream);

/*
 * km_assign without any device-memory allocation.  The pages have no
 * counterpart: this entry point exists for callers that cannot allocate --
 * e.g. a framework that has reserved the device's memory for its own pool,
 * or a latency-critical loop that must not enter the allocator, which can
 * synchronise and take locks.  Same arguments, results and kernels as
 * km_assign; the scratch (the prepared centroids, their norm bound, and the
 * list of points left to the exact re-scan) lives in one fixed array of
 * km_assign_noalloc_limit() bytes (16 MiB) compiled into the library, which
 * every GPU that loads the library holds until exit.
 *   - The prepared centroids need 2*B*K*d (fp16) or 8*B*K*d (fp32) bytes plus
 *     32*B*ceil(K/256)*256 and 8*B on the tensor-core paths (fp16 with
 *     64 <= d <= 128 or d a multiple of 64 above 128; fp32 with d in
 *     {32, 64, 96, 128}; nothing otherwise); larger problems return
 *     KM_E_UNSUPPORTED with the sizes in km_last_error().  The rest of the
 *     array holds the re-scan lists; a batch with more listed points than fit
 *     is re-scanned whole (same labels; its mindist then all from the CUDA
 *     cores).
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls share the array and it keeps the last call's contents; each
 *     call rewrites what it reads.  Calls whose work overlaps on the GPU
 *     (e.g. on two streams without ordering) race on it: order them.
 */
KM_API km_status km_assign_noalloc(const void* X, const float* C, int64_t B, int64_t N, int64_t K, int64_t d,
                                   int dtype, int32_t* labels, float* mindist, void* stream);
KM_API size_t km_assign_noalloc_limit(void);

/*
 * The update split in its two halves, for callers that combine the sums of
 * several shards of the points before dividing (e.g. one shard per GPU with
 * an all-reduce in between; see flashassign_b200.sharded).
 * km_update_sums: sort the labels and gather-reduce as km_update does,
 *   sums[b][k] = sum of the rows labelled k, counts[b][k] = their number;
 *   no centroid is written.  Arguments as km_update.
 * km_finalize: C_out[b][k] = sums[b][k] / counts[b][k] where counts > 0, else
 *   unchanged (C_out is in/out, [B, K, d] fp32, 16-byte aligned).
 */
KM_API km_status km_update_sums(const void* X, const int32_t* labels, int64_t B, int64_t N, int64_t K, int64_t d,
                                int dtype, float* sums, int32_t* counts, void* stream);

/*
 * km_assign that also returns, per batch, the objective of the assignment it
 * made: objective[b] = sum_i mindist[b][i] (fp64, device, [B], 8-byte
 * aligned, written), accumulated by the assignment kernels themselves (the
 * sharded loop adds it over the shards).  Other arguments as km_assign.
 */
KM_API km_status km_assign_objective(const void* X, const float* C, int64_t B, int64_t N, int64_t K, int64_t d,
                                     int dtype, int32_t* labels, float* mindist, double* objective, void* stream);
KM_API km_status km_finalize(const float* sums, const int32_t* counts, int64_t B, int64_t K, int64_t d, float* C_out,
                             void* stream);

/*
 * Baselines the method replaces, for measurement (papernotes.org page,
 * 方法详解 and 关键设计 1-2: the standard implementations whose memory
 * traffic and atomic contention Flash-KMeans removes).  Same results as
 * km_assign and km_update, never used by km_lloyd.
 *
 * km_assign_dense: the distance matrix materialised.  The tensor-core
 * assignment writes every score s = x.c - ||c||^2/2 to a [B, K', N] fp32
 * scratch matrix in HBM (K' = K rounded up to 256; 4*B*N*K' bytes, taken with
 * cudaMallocAsync: KM_E_NOMEM when it does not fit), then a second kernel
 * reads it back and takes each point's argmax (lowest index among equal
 * scores), certified and re-scanned as in km_assign.  fp16 points with
 * 64 <= d <= 128 only (else KM_E_UNSUPPORTED).
 * Arguments as km_assign.
 */
KM_API km_status km_assign_dense(const void* X, const float* C, int64_t B, int64_t N, int64_t K, int64_t d, int dtype,
                                 int32_t* labels, float* mindist, void* stream);

/*
 * km_update_scatter: the update with one atomic addition per point
 * coordinate into its cluster's fp32 sum and one per point into its count
 * (B*N*d + B*N atomics, contended on large clusters), then the same
 * finalisation as km_update.  Arguments as km_update; labels must lie in
 * [0, K) (others are skipped).
 */
KM_API km_status km_update_scatter(const void* X, const int32_t* labels, int64_t B, int64_t N, int64_t K, int64_t d,
                                   int dtype, float* sums, int32_t* counts, float* C_out, void* stream);

/*
 * Scratch memory comes from a stream-ordered memory pool of the library's own
 * (one per device, created on first use) that keeps what its calls free, so
 * repeated calls do not map and unmap device memory each time.  This returns
 * the pools' unused memory to the devices (memory still in use by enqueued
 * work is kept).  The pools hold at most the largest scratch of any one call
 * per stream in flight.
 */
KM_API km_status km_release_cached(void);

/* Rows per chunk used by km_lloyd for host-resident X (0 restores the default:
 * 2^23 rows, fewer when that would exceed 4 GiB, i.e. min(2^23, 2^32 / (d * sizeof(dtype)))). */
KM_API void km_set_chunk_rows(int64_t rows);

/*
 * Tracing.  While enabled (process-wide), every call records a CUDA event pair
 * on its stream around each kernel phase it enqueues and counts the kernels it
 * launches.  km_trace_read waits for the recorded events, returns for each
 * phase the summed GPU time in milliseconds and the number of kernel
 * launches, and clears the record.  Phases: see km_phase.  Arrays have
 * `nphases` entries (at most KM_NUM_PHASES are filled); either may be NULL.
 */
typedef enum {
    KM_PHASE_PREP = 0,     /* centroid rounding and half norms */
    KM_PHASE_ASSIGN = 1,   /* FlashAssign */
    KM_PHASE_SORT = 2,     /* label argsort, segment offsets, counts */
    KM_PHASE_UPDATE = 3,   /* segmented gather-reduce of the sums */
    KM_PHASE_FINALIZE = 4, /* centroid division (and next preparation) */
    KM_PHASE_OTHER = 5,    /* zeroing of sums, objective, copies */
    KM_NUM_PHASES = 6
} km_phase;
KM_API void km_trace_enable(int on);
KM_API km_status km_trace_read(double* ms, int64_t* launches, int nphases);

/* Static description of a status code. */
KM_API const char* km_status_string(km_status s);

/* Detail of the last error on the calling host thread ("" if none). */
KM_API const char* km_last_error(void);

/*
 * Reads and clears the device fault word of the current device: a kernel
 * whose bounded wait expired records a non-zero code there instead of hanging
 * (1: a TMA or MMA pipeline wait timed out).  Synchronises `stream`.
 * Returns KM_OK with *code = 0 when no fault was recorded.
 */
KM_API km_status km_device_fault(int32_t* code, void* stream);

/*
 * Reads and clears the number of points, on the current device, that the
 * tensor-core assignments could not certify within their error bound and
 * handed to the exact CUDA-core re-scan since the last call (near ties,
 * duplicate centroids, data far from the origin, fp16 norms beyond the
 * folded term's range).  Not a result of the method -- an observability
 * counter for its numerics; 0 on the CUDA-core paths.  Synchronises `stream`.
 */
KM_API km_status km_assign_rescans(int64_t* count, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KM_H */
