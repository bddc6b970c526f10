// The two standard implementations whose costs Flash-KMeans removes, kept as
// measurable baselines (papernotes.org "Flash-KMeans" page, 方法详解: the
// assignment that materialises the N x K distance matrix and reads it back,
// 关键设计 1; the update that scatters every point into its cluster with
// atomic additions, 关键设计 2).  They compute the same results as the
// method's kernels and are never on its path.
//   * dense_argmin_kernel: the second half of the dense assignment -- reads
//     the score matrix that the tensor-core kernel wrote in its dense mode
//     (s = x.c - ||c||^2/2, [B, padded K, N] fp32) and takes each point's
//     argmax (lowest index among equal scores), mindist = ||x||^2 - 2 s, with
//     the fused kernel's certification and exact re-scan of the rest.
//   * scatter_update_kernel: one thread per (point, coordinate), an fp32
//     atomic addition into the cluster's sum per coordinate and an integer
//     one per point into its count: B*N*d + B*N atomics.
#include "certify.cuh"

namespace km {
namespace {

constexpr int kArgminThreads = 256;

// One thread per point: column k of the scores is D[b][k][0..N), so the warp's
// loads of one column are consecutive.  The best score (strict > over
// ascending k keeps the lowest index among equal scores) and the second best
// certify the label as in the fused kernel; the rest go to the re-scan list.
__global__ void __launch_bounds__(kArgminThreads) dense_argmin_kernel(const float* __restrict__ D,
                                                                      const float* __restrict__ xnorm, int64_t N,
                                                                      int64_t K, int64_t Kp,
                                                                      int32_t* __restrict__ labels,
                                                                      float* __restrict__ mindist, RescanList list) {
    pdl_trigger();
    pdl_wait();
    const int64_t b = blockIdx.y;
    const int64_t n = (int64_t)blockIdx.x * kArgminThreads + threadIdx.x;
    const bool valid = n < N;  // every lane stays for the warp-wide listing
    float best = -INFINITY, second = -INFINITY;
    int idx = -1;
    if (valid) {
        const float* d = D + b * Kp * N + n;
#pragma unroll 8
        for (int64_t k = 0; k < K; ++k) {
            const float v = d[k * N];
            second = fmaxf(second, fminf(best, v));
            if (v > best) {
                best = v;
                idx = (int)k;
            }
        }
    }
    certify_top2(list, list.cmax[b], b, N, n, valid, best, second, idx, valid ? xnorm[b * N + n] : 0.f, labels,
                 mindist, threadIdx.x & 31);
}

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__half>(__half v) { return __half2float(v); }

template <typename T>
__global__ void __launch_bounds__(256) scatter_update_kernel(const T* __restrict__ X, const int32_t* __restrict__ labels,
                                                             int64_t N, int64_t K, int64_t d,
                                                             float* __restrict__ sums, int32_t* __restrict__ counts) {
    pdl_trigger();
    pdl_wait();
    const int64_t b = blockIdx.y;
    const int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x;  // element of batch b's [N, d]
    if (e >= N * d) return;
    const int64_t i = e / d, j = e - i * d;
    const int32_t lab = labels[b * N + i];
    if (lab < 0 || lab >= K) return;
    atomicAdd(sums + (b * K + lab) * d + j, to_f<T>(X[b * N * d + e]));
    if (j == 0) atomicAdd(counts + b * K + lab, 1);
}

}  // namespace

cudaError_t launch_dense_argmin(const float* D, const float* xnorm, int64_t B, int64_t N, int64_t K, int32_t* labels,
                                float* mindist, const RescanList& list, cudaStream_t st) {
    if (!list.cmax || !list.count || !list.rows) return cudaErrorInvalidValue;
    return launch_kernel(dense_argmin_kernel, dim3((unsigned)ceil_div(N, kArgminThreads), (unsigned)B),
                         dim3(kArgminThreads), 0, st, D, xnorm, N, K, padded_k(K), labels, mindist, list);
}

cudaError_t launch_scatter_update(const void* X, int dtype, const int32_t* labels, int64_t B, int64_t N, int64_t K,
                                  int64_t d, float* sums, int32_t* counts, cudaStream_t st) {
    const dim3 grid((unsigned)ceil_div(N * d, 256), (unsigned)B);
    if (dtype == KM_F16)
        return launch_kernel(scatter_update_kernel<__half>, grid, dim3(256), 0, st, (const __half*)X, labels, N, K, d,
                             sums, counts);
    return launch_kernel(scatter_update_kernel<float>, grid, dim3(256), 0, st, (const float*)X, labels, N, K, d, sums,
                         counts);
}

}  // namespace km
