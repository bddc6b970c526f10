// Centroid-side kernels of the Lloyd iteration:
//  * preparation for the assignment: round the fp32 centroids to the dtype of
//    X (fp16), or split them into tf32 heads and tails (fp32), and write
//    -||c||^2/2 as a slice of pieces that the tensor cores add to x.c (the
//    ||c||^2 term of the expansion ||x - c||^2 = ||x||^2 + ||c||^2 - 2 x.c,
//    papernotes.org "Flash-KMeans" page, 关键设计 1);
//  * finalisation of the update: c_k = s_k / n_k, an empty cluster keeping its
//    previous centroid (the flowchart's C_new on the same page, 整体框架);
//  * the per-batch objective: the assignment accumulates the sum of minimum
//    distances, the finalisation hands it out and resets the accumulator.
// All three are tiny next to the assignment and the gather; the preparation
// takes one warp per centroid row, the finalisation eight lanes per row.
#include "km_internal.cuh"

#include <cmath>

namespace km {
namespace {

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// The centroid's norm slice for the fp16 tensor-core assignment: 16 fp16
// pieces p_j with sum_j w_j p_j = -v, w_j = norm_piece_weight(j), stored as
// two 16-byte vectors.  Greedy from the largest weight down: each piece is the
// fp16 nearest to what is left divided by its weight (clamped to the fp16
// range; a piece that would be subnormal is left at 0, so nothing depends on
// how the tensor cores treat subnormal inputs).  Returns false when the
// remainder is not within 2^-30 of v (plus 2^-27): v beyond the pieces' range.
__device__ __forceinline__ bool write_norm_slice(__half* out, double v) {
    double r = -v;
    unsigned short bits[kNormPieces];
    // positions in decreasing weight: 2^15 at 0-4 and 8-12, 1 at 5, 6, 13, 14, 2^-13 at 7 and 15
    constexpr int kOrder[kNormPieces] = {0, 1, 2, 3, 4, 8, 9, 10, 11, 12, 5, 6, 13, 14, 7, 15};
#pragma unroll
    for (int i = 0; i < kNormPieces; ++i) {
        const int j = kOrder[i];
        const double w = (double)norm_piece_weight(j);
        // r / w as r times the exact reciprocal of the power-of-two weight: the same value, no division
        const double q = fmin(fmax(r * (double)(1.f / norm_piece_weight(j)), -65504.0), 65504.0);
        __half p = __float2half_rn((float)q);
        if (fabsf(__half2float(p)) < 0x1p-14f) p = __float2half(0.f);
        bits[j] = __half_as_ushort(p);
        r -= w * (double)__half2float(p);
    }
    uint32_t wd[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) wd[i] = (uint32_t)bits[2 * i] | ((uint32_t)bits[2 * i + 1] << 16);
    reinterpret_cast<uint4*>(out)[0] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
    reinterpret_cast<uint4*>(out)[1] = make_uint4(wd[4], wd[5], wd[6], wd[7]);
    return fabs(r) <= 0x1p-30 * fabs(v) + 0x1p-27;
}

// tf32 head of an fp32 value: its low 13 mantissa bits cleared (exact in tf32).
__device__ __forceinline__ float tf32_head(float v) { return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u); }

// The same for the fp32 (tf32) assignment: 8 tf32-exact fp32 pieces whose sum
// is -v (each piece takes ~10 more bits of what is left).
__device__ __forceinline__ void write_norm_pieces_tf32(float* out, double v) {
    double r = -v;
    float p[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        p[i] = tf32_head((float)r);
        r -= (double)p[i];
    }
    reinterpret_cast<float4*>(out)[0] = make_float4(p[0], p[1], p[2], p[3]);
    reinterpret_cast<float4*>(out)[1] = make_float4(p[4], p[5], p[6], p[7]);
}

// Everything the assignment needs of one centroid row, from the warp's sum of
// squares `acc` (lane 0 writes): the norm slice, and the running bound of
// max_k ||c_k||^2 (non-negative floats order like their bit patterns; +inf
// when an fp16 norm slice cannot hold the norm).
__device__ __forceinline__ void write_row_norm(const PreparedC& p, int dtype, int64_t b, int64_t slice_row,
                                               double acc) {
    bool ok = true;
    if (dtype == KM_F16)
        ok = write_norm_slice(static_cast<__half*>(p.cext) + slice_row * kNormPieces, 0.5 * acc);
    else
        write_norm_pieces_tf32(static_cast<float*>(p.cext) + slice_row * 8, 0.5 * acc);
    if (p.cmax)
        atomicMax(reinterpret_cast<int*>(p.cmax + b), ok ? __float_as_int((float)(acc * (1.0 + 1e-6))) : 0x7F800000);
}

// One warp per centroid row of [B, Kp]: fp16 rounds C (chat) and writes the
// fp16 norm slice; fp32 writes each row's tf32 heads and tails (chat = [B, K, 2d])
// and the tf32 norm pieces.  Padding rows K <= k < Kp get a -inf score.
__global__ void prep_kernel(const float* __restrict__ C, int64_t B, int64_t K, int64_t Kp, int64_t d, int dtype,
                            PreparedC p) {
    pdl_trigger();
    pdl_wait();
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    if (row >= B * Kp) return;
    const int64_t b = row / Kp, k = row % Kp;
    if (k >= K) {  // padding centroid: score -inf, never the maximum
        if (dtype == KM_F16) {
            if (lane < 16)
                static_cast<__half*>(p.cext)[row * 16 + lane] =
                    lane == 0 ? __ushort_as_half((unsigned short)0xFC00) : __float2half(0.f);
        } else if (lane < 8) {
            static_cast<float*>(p.cext)[row * 8 + lane] = lane == 0 ? -INFINITY : 0.f;
        }
        return;
    }
    const int64_t base = (b * K + k) * d;
    double acc = 0.0;
    for (int64_t j = lane; j < d; j += 32) {
        float v = C[base + j];
        if (dtype == KM_F16) {
            const __half h = __float2half_rn(v);
            if (p.chat) static_cast<__half*>(p.chat)[base + j] = h;
            v = __half2float(h);
        } else {
            float* row2 = static_cast<float*>(p.chat) + 2 * base;
            const float hv = tf32_head(v);
            row2[j] = hv;
            row2[d + j] = v - hv;
        }
        acc += (double)v * (double)v;
    }
    acc = warp_sum(acc);
    if (lane == 0) write_row_norm(p, dtype, b, row, acc);
}

// Lanes per centroid row in the finalisation (L = 8 below d = 512, where a
// warp finalises four rows at once; L = 32, a warp per row, from d = 512 on):
// each lane takes every L-th 4-wide chunk of the row.
constexpr int kFinThreads = 256;

// n_k comes from the sort's segment offsets (offsets[k+1] - offsets[k]); it is
// also written to counts when that is non-null.  With zero_sums the consumed
// sums are reset to 0, ready for the next iteration's boundary atomics.  When
// `next` holds buffers, the new centroids are prepared for the next
// assignment as prep_kernel does.  Grid: (rows of a batch * L / 256, B).
template <int kFinLanes>
__global__ void __launch_bounds__(kFinThreads) finalize_kernel(
    float* __restrict__ sums, const int32_t* __restrict__ offsets, int64_t K, int64_t Kp, int64_t d,
    float* __restrict__ C_out, int dtype, PreparedC next, int32_t* __restrict__ counts, int zero_sums,
    double* __restrict__ obj_acc, float* __restrict__ obj_out, const int32_t* __restrict__ counts_in,
    const int32_t* __restrict__ stop, double* __restrict__ shift) {
    pdl_trigger();
    pdl_wait();
    if (stop && *stop) return;
    const int64_t b = blockIdx.y;
    const int sub = threadIdx.x % kFinLanes;
    const int64_t k = ((int64_t)blockIdx.x * kFinThreads + threadIdx.x) / kFinLanes;
    if (obj_out && blockIdx.x == 0 && threadIdx.x == 0) {  // this iteration's objective, and a fresh accumulator
        obj_out[b] = (float)obj_acc[b];
        obj_acc[b] = 0.0;
    }
    const bool valid = k < K;  // the warp's shuffles below need every lane, valid or not
    const int64_t row = b * K + k;
    int32_t n = 0;
    if (valid) n = counts_in ? counts_in[row] : offsets[b * (K + 1) + k + 1] - offsets[b * (K + 1) + k];
    if (valid && counts && sub == 0) counts[row] = n;
    const float inv = n > 0 ? 1.0f / (float)n : 0.f;  // the mean as s * (1/n): within 1 ulp of s / n
    const int64_t base = row * d;
    double acc = 0.0, moved = 0.0;
    constexpr int kAhead = 4;  // float4 steps of a row loaded before any is stored
    if (valid) {
        for (int64_t j0 = 4 * sub; j0 < d; j0 += kAhead * 4 * kFinLanes) {
            // The loads of a group are issued together: the stores below go through
            // pointers the compiler cannot separate from these, so a load after a
            // store would wait for it.  An empty cluster keeps its centroid.
            float4 sv[kAhead];
#pragma unroll
            for (int u = 0; u < kAhead; ++u) {
                const int64_t j = j0 + (int64_t)u * 4 * kFinLanes;
                if (j < d) sv[u] = *reinterpret_cast<const float4*>((n > 0 ? sums : C_out) + base + j);
            }
#pragma unroll
            for (int u = 0; u < kAhead; ++u) {
                const int64_t j = j0 + (int64_t)u * 4 * kFinLanes;
                if (j >= d) break;
                float4 v = sv[u];
                if (n > 0) {
                    v = make_float4(v.x * inv, v.y * inv, v.z * inv, v.w * inv);
                    if (shift) {  // this centroid's squared shift
                        const float4 o = *reinterpret_cast<const float4*>(C_out + base + j);
                        const double dx = (double)v.x - o.x, dy = (double)v.y - o.y, dz = (double)v.z - o.z,
                                     dw = (double)v.w - o.w;
                        moved += dx * dx + dy * dy + dz * dz + dw * dw;
                    }
                    *reinterpret_cast<float4*>(C_out + base + j) = v;
                    if (zero_sums) *reinterpret_cast<float4*>(sums + base + j) = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                if (!next.cext) continue;
                if (dtype == KM_F16) {
                    const __half2 h01 = __floats2half2_rn(v.x, v.y), h23 = __floats2half2_rn(v.z, v.w);
                    __half* chat = static_cast<__half*>(next.chat);
                    *reinterpret_cast<__half2*>(chat + base + j) = h01;
                    *reinterpret_cast<__half2*>(chat + base + j + 2) = h23;
                    const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
                    v = make_float4(f01.x, f01.y, f23.x, f23.y);
                } else {
                    float* row2 = static_cast<float*>(next.chat) + 2 * base;
                    const float4 hv = make_float4(tf32_head(v.x), tf32_head(v.y), tf32_head(v.z), tf32_head(v.w));
                    *reinterpret_cast<float4*>(row2 + j) = hv;
                    *reinterpret_cast<float4*>(row2 + d + j) =
                        make_float4(v.x - hv.x, v.y - hv.y, v.z - hv.z, v.w - hv.w);
                }
                acc += (double)v.x * v.x + (double)v.y * v.y + (double)v.z * v.z + (double)v.w * v.w;
            }
        }
    }
    if (next.cext) {
#pragma unroll
        for (int o = kFinLanes / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (valid && sub == 0) write_row_norm(next, dtype, b, b * Kp + k, acc);
    }
    if (shift) {  // the warp's rows, one atomic
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) moved += __shfl_xor_sync(0xffffffffu, moved, o);
        if ((threadIdx.x & 31) == 0 && moved != 0.0) atomicAdd(shift + b, moved);
    }
}

// After an iteration: unless the loop has stopped, count the iteration and
// stop it when every batch's centroid shift is within tol; reset the shifts.
__global__ void converge_check_kernel(double* __restrict__ shift, int64_t B, double tol, int32_t* __restrict__ stop,
                                      int32_t* __restrict__ iters_run) {
    pdl_trigger();
    pdl_wait();
    __shared__ int all_in;
    if (threadIdx.x == 0) all_in = 1;
    __syncthreads();
    const bool running = *stop == 0;
    for (int64_t b = threadIdx.x; b < B; b += blockDim.x) {
        if (!(shift[b] <= tol)) all_in = 0;  // benign race: every writer stores 0
        shift[b] = 0.0;
    }
    __syncthreads();
    if (threadIdx.x == 0 && running) {
        *iters_run += 1;
        if (all_in) *stop = 1;
    }
}

__global__ void add_counts_kernel(const int32_t* __restrict__ offsets, int64_t B, int64_t K,
                                  int32_t* __restrict__ counts) {
    pdl_trigger();
    pdl_wait();
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= B * K) return;
    const int64_t b = t / K, k = t % K;
    counts[t] += offsets[b * (K + 1) + k + 1] - offsets[b * (K + 1) + k];
}

}  // namespace

cudaError_t launch_add_counts(const int32_t* offsets, int64_t B, int64_t K, int32_t* counts, cudaStream_t st) {
    return launch_kernel(add_counts_kernel, dim3((unsigned)ceil_div(B * K, 256)), dim3(256), 0, st, offsets, B, K,
                         counts);
}

cudaError_t launch_prep_centroids(const float* C, int64_t B, int64_t K, int64_t d, int dtype, PreparedC p,
                                  cudaStream_t st) {
    const int64_t Kp = padded_k(K);
    const int64_t rows = B * Kp;
    const int warps = 8;
    return launch_kernel(prep_kernel, dim3((unsigned)ceil_div(rows, warps)), dim3(warps * 32), 0, st, C, B, K, Kp, d,
                         dtype, p);
}

cudaError_t launch_finalize(float* sums, const int32_t* offsets, int64_t B, int64_t K, int64_t d, float* C_out,
                            int dtype, PreparedC next, int32_t* counts, bool zero_sums, double* obj_acc,
                            float* obj_out, cudaStream_t st, const int32_t* counts_in, const int32_t* stop,
                            double* shift) {
    if (d >= 512) {
        const dim3 grid((unsigned)ceil_div(K * 32, kFinThreads), (unsigned)B);
        return launch_kernel(finalize_kernel<32>, grid, dim3(kFinThreads), 0, st, sums, offsets, K, padded_k(K), d,
                             C_out, dtype, next, counts, zero_sums ? 1 : 0, obj_acc, obj_out, counts_in, stop, shift);
    }
    const dim3 grid((unsigned)ceil_div(K * 8, kFinThreads), (unsigned)B);
    return launch_kernel(finalize_kernel<8>, grid, dim3(kFinThreads), 0, st, sums, offsets, K, padded_k(K), d, C_out,
                         dtype, next, counts, zero_sums ? 1 : 0, obj_acc, obj_out, counts_in, stop, shift);
}

cudaError_t launch_converge_check(double* shift, int64_t B, double tol, int32_t* stop, int32_t* iters_run,
                                  cudaStream_t st) {
    return launch_kernel(converge_check_kernel, dim3(1), dim3(256), 0, st, shift, B, tol, stop, iters_run);
}

}  // namespace km
