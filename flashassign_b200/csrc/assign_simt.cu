// CUDA-core assignment kernel: the FlashAssign recurrence of the
// papernotes.org "Flash-KMeans" page (关键设计 1) -- a running (m_i, a_i)
// starting at (+inf, -1), updated tile by tile over the centroids, the N x K
// distances never leaving registers -- computed with direct differences
// sum_j (x_j - c_j)^2 in fp32.
//
// It serves the shapes the tensor-core kernels do not take (fp16 with d < 64
// or d not a multiple of 64 above 128, fp32 with d not a multiple of 32 or
// d > 128).  Each thread owns one point;
// centroids and a 32-wide slice of the block's points are staged in shared
// memory, so the loop is a register-blocked [128 points x 32 centroids] tile.
#include "km_internal.cuh"

namespace km {
namespace {

constexpr int kThreads = 128;  // points per block
constexpr int kTileK = 32;     // centroids per tile
constexpr int kTileD = 32;     // dims per slice

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__half>(__half v) { return __half2float(v); }

// Points of batch b: rows [0, N); blocks stride over them.
template <typename T>
__global__ void __launch_bounds__(kThreads) assign_simt_kernel(const T* __restrict__ X, const float* __restrict__ C,
                                                               int64_t N, int64_t K, int64_t d,
                                                               int32_t* __restrict__ labels,
                                                               float* __restrict__ mindist,
                                                               double* __restrict__ obj_acc,
                                                               const int32_t* __restrict__ stop) {
    pdl_trigger();
    pdl_wait();
    if (stop && *stop) return;
    __shared__ float xs[kThreads][kTileD + 1];
    __shared__ float cs[kTileK][kTileD + 1];
    __shared__ int64_t rows[kThreads];
    const int64_t b = blockIdx.y;
    const T* Xb = X + b * N * d;
    const float* Cb = C + b * K * d;
    const int64_t count = N;

    for (int64_t i0 = (int64_t)blockIdx.x * kThreads; i0 < count; i0 += (int64_t)gridDim.x * kThreads) {
        __syncthreads();  // the previous round's readers of rows[] are done
        const bool mine = i0 + threadIdx.x < count;
        rows[threadIdx.x] = mine ? i0 + threadIdx.x : -1;
        float best = INFINITY;
        int32_t arg = -1;
        for (int64_t k0 = 0; k0 < K; k0 += kTileK) {
            float acc[kTileK];
#pragma unroll
            for (int c = 0; c < kTileK; ++c) acc[c] = 0.f;
            for (int64_t j0 = 0; j0 < d; j0 += kTileD) {
                __syncthreads();
                // stage a [128 points x 32 dims] slice (zeros past the ends)
                for (int t = threadIdx.x; t < kThreads * kTileD; t += kThreads) {
                    const int r = t / kTileD, j = t % kTileD;
                    const int64_t gi = rows[r], gj = j0 + j;
                    xs[r][j] = (gi >= 0 && gj < d) ? to_f<T>(Xb[gi * d + gj]) : 0.f;
                }
                // and a [32 centroids x 32 dims] slice, rounded to X's dtype
                for (int t = threadIdx.x; t < kTileK * kTileD; t += kThreads) {
                    const int r = t / kTileD, j = t % kTileD;
                    const int64_t gk = k0 + r, gj = j0 + j;
                    float v = (gk < K && gj < d) ? Cb[gk * d + gj] : 0.f;
                    if (sizeof(T) == 2) v = __half2float(__float2half_rn(v));
                    cs[r][j] = v;
                }
                __syncthreads();
#pragma unroll 4
                for (int j = 0; j < kTileD; ++j) {
                    const float xv = xs[threadIdx.x][j];
#pragma unroll
                    for (int c = 0; c < kTileK; ++c) {
                        const float diff = xv - cs[c][j];
                        acc[c] = fmaf(diff, diff, acc[c]);
                    }
                }
            }
#pragma unroll
            for (int c = 0; c < kTileK; ++c) {
                if (k0 + c < K && acc[c] < best) {  // strict: the lowest index keeps ties
                    best = acc[c];
                    arg = (int32_t)(k0 + c);
                }
            }
        }
        const int64_t i = rows[threadIdx.x];
        if (mine) {
            labels[b * N + i] = arg;
            if (mindist) mindist[b * N + i] = best;
        }
        if (obj_acc) {  // the objective: one atomic per warp
            float part = mine ? best : 0.f;  // fp32 within the warp, fp64 across
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            if ((threadIdx.x & 31) == 0) atomicAdd(obj_acc + b, (double)part);
        }
    }
}

}  // namespace

cudaError_t launch_assign_simt(const void* X, int dtype, const float* C, int64_t B, int64_t N, int64_t K, int64_t d,
                               int32_t* labels, float* mindist, double* obj_acc, cudaStream_t st, const int32_t* stop) {
    const dim3 grid((unsigned)ceil_div(N, kThreads), (unsigned)B);
    if (dtype == KM_F16)
        return launch_kernel(assign_simt_kernel<__half>, grid, dim3(kThreads), 0, st, (const __half*)X, C, N, K, d,
                             labels, mindist, obj_acc, stop);
    return launch_kernel(assign_simt_kernel<float>, grid, dim3(kThreads), 0, st, (const float*)X, C, N, K, d, labels,
                         mindist, obj_acc, stop);
}

}  // namespace km
