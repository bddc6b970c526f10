// Internal declarations shared by the libkm translation units: launchers,
// the per-thread error detail, and the device fault word.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/km.h"

namespace km {

// Per-thread error detail (km_last_error).
void set_error(const char* fmt, ...);
km_status cuda_error(cudaError_t e, const char* what);

// Device fault word: kernels write a non-zero code when a bounded wait expires.
enum : int32_t { FAULT_NONE = 0, FAULT_PIPELINE_TIMEOUT = 1 };
int32_t* fault_word();  // device address of the word on the current device
// Running count of points the tensor-core assignments left to the exact
// re-scan (device address on the current device).
unsigned long long* rescan_word();

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Tile width of the tensor-core assignment along K; the centroids' norm-slice
// array [B, padded_k(K), 16] is padded to a multiple of it with rows whose
// score is -inf, so that padded columns never win.
constexpr int kAssignTileK = 256;
inline int64_t padded_k(int64_t K) { return ceil_div(K, kAssignTileK) * kAssignTileK; }

// ---- the folded norm term of the fp16 tensor-core assignment ----
// -||c||^2/2 enters the MMA as one more K = 16 step: the points' side of that
// step is a constant slice of power-of-two weights w_j, the centroid's side 16
// fp16 pieces p_j with sum_j w_j p_j = -||c||^2/2.  The weights repeat after
// eight (both 16-byte halves of the 32-byte slice are equal, so the slice
// reads the same whatever the 32-byte swizzle does to them): five of 2^15,
// two of 1, one of 2^-13.  The 2^15 pieces take the bulk of a large norm
// (up to ~1.7e10, i.e. ||c||^2 ~ 3.4e10), the others refine what is left to
// within ~2^-27 absolute.  A centroid beyond that range makes its batch's
// norm bound +inf, so that every point of the batch is re-scanned exactly.
constexpr int kNormPieces = 16;
__host__ __device__ constexpr float norm_piece_weight(int j) {
    return (j & 7) < 5 ? 32768.f : (j & 7) < 7 ? 1.f : 0x1p-13f;
}
// The points' slice as four 32-bit words of fp16 pairs (one 16-byte half).
constexpr uint32_t kNormWeightW01 = 0x78007800u, kNormWeightW23 = 0x78007800u, kNormWeightW45 = 0x3C007800u,
                   kNormWeightW67 = 0x08003C00u;

// Error bound of a folded fp16 tensor-core score s_k = x.c_k - ||c_k||^2/2:
// every accumulating MMA step (ceil(d/16) steps of x.c and the norm step;
// products of fp16 values are exact) is taken to err by at most kMmaStepErr
// times the largest partial sum, itself at most ||x|| ||c_k|| + ||c_k||^2/2.
// Per point, with cmax^2 >= max_k ||c_k||^2,
//     e = fp16_score_err(d) * (||x|| cmax + cmax^2 / 2)
// bounds |computed - exact| for every score of the point.  The step bound is
// 4x what was measured on B200: a K = 16 fp16 MMA with fp32 accumulation
// sums its 16 exact products and rounds the result toward zero once (a sum of
// 1 and fifteen 2^-24 comes out as 1 + 14 * 2^-24), i.e. less than 2^-23 of
// the result, and over 320,000 points of d = 64 .. 1024, near the origin and
// offset from it, the largest error of a computed distance was 2^-22.8 of
// (||x|| cmax + cmax^2 / 2) per step.
constexpr double kMmaStepErr = 0x1p-21;
inline float fp16_score_err(int64_t d) { return (float)((double)(ceil_div(d, 16) + 1) * kMmaStepErr); }
// The fp16 label tolerance of the method's exactness contract: a label must be
// the exact argmin unless the two smallest exact distances differ by less than
// this fraction of the second one (then any centroid within that fraction of
// the smallest distance will do).
constexpr float kLabelTolF16 = 1e-3f;

// ---- programmatic dependent launch ----
// Kernels on the iteration's path are launched with programmatic stream
// serialisation: a kernel may start (prologue, resource allocation) while
// its predecessor in the stream is still draining, and waits for it with
// pdl_wait() before reading anything the predecessor wrote.  Every kernel
// calls pdl_wait() in every thread before its first dependent access and
// before it exits, so a grid never completes ahead of its predecessor and
// the chain stays ordered transitively.  Without the launch attribute both
// instructions are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Whether launches carry the attribute: off while per-phase event tracing is
// on, so that traced kernel times are not overlapped with their neighbours.
bool pdl_enabled();

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                          Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

struct DeviceInfo {
    int device = -1;
    int sms = 0;
    int cc_major = 0, cc_minor = 0;
};
km_status device_info(DeviceInfo* out);

// ---- launchers (all asynchronous on `st`) ----
// Where an assignment lists the points it could not certify: per batch a
// counter (zero on entry) and up to `cap` row indices rows[b * cap + i]; a
// counter above cap tells the re-scan to take the whole batch.  The bound of
// a point's scores is err * (||x|| cmax + cmax^2 / 2) <= err (||x||^2/2 +
// cmax^2) (fp16_score_err), that of its computed ||x||^2 is xerr * ||x||^2,
// and tau the label tolerance; c_x, c_c fold them into the certificate's
// threshold on a computed distance, c_x ||x||^2 + c_c cmax^2 (certify.cuh).
struct RescanList {
    const float* cmax = nullptr;          // [B] bound of max_k ||c_k||^2 (+inf: certify nothing)
    int32_t* count = nullptr;             // [B]
    int32_t* rows = nullptr;              // [B, cap]
    int64_t cap = 0;
    unsigned long long* total = nullptr;  // running count of listed points (nullable)
    float err = 0.f, xerr = 0.f, tau = 0.f;
    float c_x = 0.f, c_c = 0.f;
    // the fp16 certificate's constants for width d (fp16_score_err, kLabelTolF16)
    void set_fp16(int64_t d) {
        err = fp16_score_err(d);
        xerr = (float)((double)(d + 2) * 0x1p-24);
        tau = kLabelTolF16;
        const double k = (4.0 / (double)tau + 2.0) * (double)err;
        c_x = (float)(0.5 * k + (double)xerr);
        c_c = (float)k;
    }
};

// Centroids prepared for a tensor-core assignment (buffers owned by the caller):
//  fp16 X: chat = [B, K, d] fp16, C rounded RNE; cext = [B, Kp, 16] fp16 pieces
//          whose weighted sum (norm_piece_weight) is -||chat_k||^2 / 2; cmax =
//          [B] running upper bound of max_k ||chat_k||^2, +inf once a centroid's
//          norm is beyond the pieces' range (atomic max; zero it first);
//  fp32 X: chat = [B, K, 2d] fp32, each row the tf32 heads of c (low 13 mantissa
//          bits cleared) then the tails c - head; cext = [B, Kp, 8] tf32-exact
//          fp32 pieces summing to -||c_k||^2 / 2; cmax = [B] running upper bound
//          of max_k ||c_k||^2 (atomic max; zero it before the first preparation).
// Rows K <= k < Kp = padded_k(K) of cext give the score -inf.
struct PreparedC {
    void* chat = nullptr;
    void* cext = nullptr;
    float* cmax = nullptr;
};
cudaError_t launch_prep_centroids(const float* C, int64_t B, int64_t K, int64_t d, int dtype, PreparedC p,
                                  cudaStream_t st);

// C_out[b][k] = sums / n_k where n_k > 0 (else unchanged), n_k taken from the
// segment offsets [B, K+1] (and written to counts when non-null); when `next`
// holds buffers, also prepares the next assignment's centroids from C_out;
// with zero_sums the sums are reset to 0 once consumed.
// When obj_out is non-null, obj_out[b] = obj_acc[b] (as fp32) and obj_acc[b] = 0.
// n_k is taken from counts_in when it is non-null, else from the offsets.
// When shift is non-null, shift[b] += sum_k ||C_new[b][k] - C_old[b][k]||^2 (the
// centroid shift of the iteration, for convergence tests).
// Every launcher's `stop` (nullable): when *stop is set at run time, the
// launch does nothing (a converged iteration loop, see launch_converge_check).
cudaError_t launch_finalize(float* sums, const int32_t* offsets, int64_t B, int64_t K, int64_t d, float* C_out,
                            int dtype, PreparedC next, int32_t* counts, bool zero_sums, double* obj_acc,
                            float* obj_out, cudaStream_t st, const int32_t* counts_in = nullptr,
                            const int32_t* stop = nullptr, double* shift = nullptr);

// Tensor-core assignment (fp16, 64 <= d <= 128).  Returns cudaErrorNotSupported
// for shapes it does not take.
bool assign_tc_supported(int64_t d, int dtype);
// obj_acc (nullable, [B] double) accumulates the sum of minimum distances.
// Points that the scores' error bound (list.err, list.cmax) does not certify
// (certify.cuh) are not resolved: they are appended to `list`
// (its counters zero on entry) for launch_rescan and left out of obj_acc.
// xnorm_out (nullable, [B, N]) receives ||x||^2 of every point; xnorm_in
// (nullable) gives them, as an earlier launch on the same X wrote them, so
// that the kernel reads instead of computing them and releases each X tile
// as soon as its MMAs are done.
cudaError_t launch_assign_tc(const __half* X, const __half* chat, const __half* cext, int64_t B, int64_t N, int64_t K,
                             int64_t d, int32_t* labels, float* mindist, double* obj_acc, const RescanList& list,
                             int sms, cudaStream_t st, const int32_t* stop = nullptr,
                             const float* xnorm_in = nullptr, float* xnorm_out = nullptr);

// Tensor-core assignment of wide fp16 points (128 < d <= 512, d % 64 == 0):
// the centroid tiles stream in 64-dimension chunks, the points stay resident.
// Same prepared centroids and results as launch_assign_tc.
bool assign_wide_supported(int64_t d, int dtype);
cudaError_t launch_assign_wide(const __half* X, const __half* chat, const __half* cext, int64_t B, int64_t N,
                               int64_t K, int64_t d, int32_t* labels, float* mindist, double* obj_acc,
                               const RescanList& list, int sms, cudaStream_t st, const int32_t* stop = nullptr);

// Tensor-core assignment of fp16 points with d > 512 (d % 64 == 0): points and
// centroids both stream in 64-dimension chunks, each point chunk meeting two
// centroid tiles.  Same prepared centroids and results as launch_assign_tc.
bool assign_split_supported(int64_t d, int dtype);
cudaError_t launch_assign_split(const __half* X, const __half* chat, const __half* cext, int64_t B, int64_t N,
                                int64_t K, int64_t d, int32_t* labels, float* mindist, double* obj_acc,
                                const RescanList& list, int sms, cudaStream_t st, const int32_t* stop = nullptr);

// Tensor-core assignment of fp32 points (tf32 head/tail split, 32 <= d <= 128,
// d % 32 == 0).  Points whose best two scores lie within the split's error
// bound are not resolved: they are appended to `list` (list.cmax is the
// prepared bound; list.err, xerr and tau are not used) for launch_rescan,
// and left out of obj_acc.
bool assign_tf32_supported(int64_t d);
cudaError_t launch_assign_tf32(const float* X, const float* csplit, const float* cext, int64_t B, int64_t N,
                               int64_t K, int64_t d, int32_t* labels, float* mindist, double* obj_acc,
                               const RescanList& list, int sms, cudaStream_t st, const int32_t* stop = nullptr);

// CUDA-core assignment for every supported shape: direct-difference
// distances, every point of every batch.
cudaError_t launch_assign_simt(const void* X, int dtype, const float* C, int64_t B, int64_t N, int64_t K, int64_t d,
                               int32_t* labels, float* mindist, double* obj_acc, cudaStream_t st,
                               const int32_t* stop = nullptr);

// The exact re-scan of the points a tensor-core assignment listed: for each of
// the list.count[b] points list.rows[b * list.cap + r] of each batch (every
// point of the batch when the count exceeds the capacity), the nearest
// centroid by direct differences in fp32 (C rounded to X's dtype), lowest
// index on ties; writes its label, mindist and objective share.  `reset`
// (nullable, [B]) is zeroed on the way, ready for the next assignment's list.
cudaError_t launch_rescan(const void* X, int dtype, const float* C, int64_t B, int64_t N, int64_t K, int64_t d,
                          int32_t* labels, float* mindist, double* obj_acc, const RescanList& list, int sms,
                          cudaStream_t st, const int32_t* stop = nullptr, int32_t* reset = nullptr);

// Stable LSD radix argsort of labels in [0, K).  Scratch: sort_scratch_bytes().
size_t sort_scratch_bytes(int64_t B, int64_t N, int64_t K);
int sort_kernel_launches(int64_t N, int64_t K, bool with_counts, bool bounds = true);
// With bounds = false the segment offsets (and counts) are left to the caller
// (the update kernel writes them while it walks the sorted labels).
cudaError_t launch_sort(const int32_t* labels, int64_t B, int64_t N, int64_t K, int32_t* a_sorted,
                        int32_t* sorted_idx, int32_t* counts, int32_t* offsets, void* scratch, cudaStream_t st,
                        bool bounds = true, const int32_t* stop = nullptr);

// Segmented gather-reduce over the sorted order (sums must be zeroed first);
// when offsets [B, K+1] is non-null it also writes the segment offsets.
// With accumulate, the sums are added to (points streamed in chunks).
cudaError_t launch_update_sums(const void* X, int dtype, const int32_t* a_sorted, const int32_t* sorted_idx,
                               int64_t B, int64_t N, int64_t K, int64_t d, float* sums, int32_t* offsets,
                               cudaStream_t st, bool accumulate = false, const int32_t* stop = nullptr);

// ---- baselines the method replaces (measurement only, never on its path) ----
// The dense-distance assignment: the tensor-core kernel's MMA pipeline writing
// every score s = x.c - ||c||^2/2 to dense [B, padded_k(K), N] fp32 and ||x||^2
// to xnorm [B, N]; then a separate pass takes each row's argmax.
cudaError_t launch_assign_tc_dense(const __half* X, const __half* chat, const __half* cext, int64_t B, int64_t N,
                                   int64_t K, int64_t d, float* dense, float* xnorm, int sms, cudaStream_t st);
// The argmax of each row's scores with the fused kernel's certification: points
// it cannot certify go to `list` for the exact re-scan.
cudaError_t launch_dense_argmin(const float* D, const float* xnorm, int64_t B, int64_t N, int64_t K, int32_t* labels,
                                float* mindist, const RescanList& list, cudaStream_t st);
// The scatter-atomic update: sums and counts (zeroed by the caller) receive one
// atomic addition per coordinate and one per point.
cudaError_t launch_scatter_update(const void* X, int dtype, const int32_t* labels, int64_t B, int64_t N, int64_t K,
                                  int64_t d, float* sums, int32_t* counts, cudaStream_t st);

// counts[b][k] += offsets[b][k+1] - offsets[b][k] (chunked accumulation of cluster sizes).
// Convergence test after an iteration's finalisation: unless *stop is already
// set, ++*iters_run, and *stop = 1 when every batch's shift[b] <= tol; shift is
// reset to 0.
cudaError_t launch_converge_check(double* shift, int64_t B, double tol, int32_t* stop, int32_t* iters_run,
                                  cudaStream_t st);
cudaError_t launch_add_counts(const int32_t* offsets, int64_t B, int64_t K, int32_t* counts, cudaStream_t st);


}  // namespace km
