// The exact re-scan of the points that a tensor-core assignment could not
// certify (near ties, duplicate centroids, data far from the origin, fp16
// norms beyond the folded term's range): for each listed point the nearest
// centroid under direct differences sum_j (x_j - c_j)^2 in fp32, lowest index
// on ties -- the FlashAssign recurrence of the papernotes.org "Flash-KMeans"
// page (关键设计 1) without the norm expansion, so no cancellation.
//
// A thread-block cluster takes 32 listed points of one batch at a time and
// splits the batch's centroids among its CTAs.  In a CTA, each warp holds 4 of
// the points and each lane 4 centroids of a 128-centroid block, so that every
// staged value feeds 16 differences (register tiles of 4 points x 4
// centroids); the lanes' nearest centroids are joined by shuffles and the
// CTAs' through distributed shared memory by CTA 0, which writes the label,
// mindist and the objective share.  The distance of each (point, centroid) is
// summed over ascending dimensions, as the CUDA-core assignment kernel sums
// it.  The launch does not know how long the lists are (they are filled on the
// device): it is sized to fill the GPU when they are long, and a CTA whose
// batch has nothing listed returns at once.
#include "km_internal.cuh"

#include <algorithm>
#include <atomic>

namespace km {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kPts = 4;                     // points per warp (every lane holds all 4)
constexpr int kPoints = kWarps * kPts;      // points per chunk (32)
constexpr int kPerLane = 4;                 // centroids per lane per block
constexpr int kBlockK = 32 * kPerLane;      // centroids per CTA per block (128)
constexpr int kSlice = 32;                  // dimensions per staged slice
constexpr int kXStride = kPoints + 4;       // staged rows, padded (and 16-byte aligned for float4 reads)
constexpr int kCStride = kBlockK + 4;
constexpr int kClusterMax = 16;             // non-portable on sm_100, checked placeable

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__half>(__half v) { return __half2float(v); }

__device__ __forceinline__ uint32_t cl_rank() {
    uint32_t r;
    asm("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cl_size() {
    uint32_t r;
    asm("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cl_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// (distance, index) of point `lane` in CTA `rank`'s result slots
__device__ __forceinline__ void ld_peer(const float* d_local, const int* k_local, uint32_t rank, float& dv, int& kv) {
    uint32_t da = (uint32_t)__cvta_generic_to_shared(d_local), ka = (uint32_t)__cvta_generic_to_shared(k_local);
    asm volatile("mapa.shared::cluster.u32 %0, %0, %1;" : "+r"(da) : "r"(rank));
    asm volatile("mapa.shared::cluster.u32 %0, %0, %1;" : "+r"(ka) : "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(dv) : "r"(da) : "memory");
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(kv) : "r"(ka) : "memory");
}
// Whether (d, k) is nearer than (bd, bk): a smaller distance, or an equal one at a lower index.
__device__ __forceinline__ bool nearer(float d, int k, float bd, int bk) {
    return k >= 0 && (bk < 0 || d < bd || (d == bd && k < bk));
}

// grid = (cluster size * clusters per batch, B); each cluster takes the
// chunks c, c + clusters, ... of its batch's list (the whole batch when its
// count exceeds the capacity: the list overflowed).
template <typename T>
__global__ void __launch_bounds__(kThreads) rescan_kernel(const T* __restrict__ X, const float* __restrict__ C,
                                                          int64_t N, int64_t K, int64_t d,
                                                          const int32_t* __restrict__ list,
                                                          const int32_t* __restrict__ list_count, int64_t cap,
                                                          int32_t* __restrict__ reset, int32_t* __restrict__ labels,
                                                          float* __restrict__ mindist, double* __restrict__ obj_acc,
                                                          const int32_t* __restrict__ stop) {
    pdl_trigger();
    pdl_wait();
    if (stop && *stop) return;  // read by every CTA of the cluster alike
    __shared__ __align__(16) float xs[kSlice][kXStride];  // the chunk's points, a slice of dimensions, transposed
    __shared__ __align__(16) float cs[kSlice][kCStride];  // a block's centroids, the same slice, transposed
    __shared__ float res_d[kPoints];
    __shared__ int res_k[kPoints];
    __shared__ int64_t rows[kPoints];

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t b = blockIdx.y;
    const uint32_t rank = cl_rank(), csize = cl_size();
    const int64_t cluster = blockIdx.x / csize, clusters = gridDim.x / csize;
    if (reset && cluster == 0 && rank == 0 && threadIdx.x == 0) reset[b] = 0;
    const int64_t listed = list_count[b];
    const bool whole = listed > cap;
    const int64_t npts = whole ? N : listed;
    const int64_t chunks = (npts + kPoints - 1) / kPoints;
    const int64_t per_cta = (K + csize - 1) / csize;
    const int64_t k_lo = (int64_t)rank * per_cta, k_hi = k_lo + per_cta < K ? k_lo + per_cta : K;
    const T* Xb = X + b * N * d;
    const float* Cb = C + b * K * d;

    for (int64_t ch = cluster; ch < chunks; ch += clusters) {
        if (threadIdx.x < kPoints) {
            const int64_t p = ch * kPoints + threadIdx.x;
            rows[threadIdx.x] = p >= npts ? -1 : whole ? p : (int64_t)list[b * cap + p];
        }
        __syncthreads();
        float best[kPts];
        int bk[kPts];
#pragma unroll
        for (int i = 0; i < kPts; ++i) {
            best[i] = INFINITY;
            bk[i] = -1;
        }
        for (int64_t kb = k_lo; kb < k_hi; kb += kBlockK) {
            float acc[kPts][kPerLane];
#pragma unroll
            for (int i = 0; i < kPts; ++i)
#pragma unroll
                for (int c = 0; c < kPerLane; ++c) acc[i][c] = 0.f;
            for (int64_t j0 = 0; j0 < d; j0 += kSlice) {
                for (int t = threadIdx.x; t < kPoints * kSlice; t += kThreads) {
                    const int r = t / kSlice, j = t % kSlice;
                    const int64_t gi = rows[r], gj = j0 + j;
                    xs[j][r] = (gi >= 0 && gj < d) ? to_f<T>(Xb[gi * d + gj]) : 0.f;
                }
                for (int t = threadIdx.x; t < kBlockK * kSlice; t += kThreads) {
                    const int r = t / kSlice, j = t % kSlice;
                    const int64_t gk = kb + r, gj = j0 + j;
                    float v = (gk < k_hi && gj < d) ? Cb[gk * d + gj] : 0.f;
                    if (sizeof(T) == 2) v = __half2float(__float2half_rn(v));  // the centroids as the assignment sees them
                    cs[j][r] = v;
                }
                __syncthreads();
#pragma unroll 8
                for (int j = 0; j < kSlice; ++j) {
                    const float4 xv = *reinterpret_cast<const float4*>(&xs[j][warp * kPts]);
                    const float4 cv = *reinterpret_cast<const float4*>(&cs[j][lane * kPerLane]);
                    const float xa[kPts] = {xv.x, xv.y, xv.z, xv.w}, ca[kPerLane] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
                    for (int i = 0; i < kPts; ++i)
#pragma unroll
                        for (int c = 0; c < kPerLane; ++c) {
                            const float diff = xa[i] - ca[c];
                            acc[i][c] = fmaf(diff, diff, acc[i][c]);
                        }
                }
                __syncthreads();
            }
            // each point's nearest centroid of the block: the lane's four (ascending k: strict keeps
            // the lowest), then across the lanes
#pragma unroll
            for (int i = 0; i < kPts; ++i) {
                float bd = INFINITY;
                int kk = -1;
#pragma unroll
                for (int c = 0; c < kPerLane; ++c) {
                    const int64_t k = kb + lane * kPerLane + c;
                    if (k < k_hi && acc[i][c] < bd) {
                        bd = acc[i][c];
                        kk = (int)k;
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float od = __shfl_xor_sync(0xffffffffu, bd, o);
                    const int ok = __shfl_xor_sync(0xffffffffu, kk, o);
                    if (nearer(od, ok, bd, kk)) {
                        bd = od;
                        kk = ok;
                    }
                }
                if (nearer(bd, kk, best[i], bk[i])) {
                    best[i] = bd;
                    bk[i] = kk;
                }
            }
        }
        // this CTA's nearest centroid of each point (every lane of a warp holds its four)
        if (lane < kPts) {
            float rd = best[0];
            int rk = bk[0];
#pragma unroll
            for (int i = 1; i < kPts; ++i)
                if (lane == i) {
                    rd = best[i];
                    rk = bk[i];
                }
            res_d[warp * kPts + lane] = rd;
            res_k[warp * kPts + lane] = rk;
        }
        cl_sync();  // every CTA's result is visible to the cluster
        if (rank == 0 && warp == 0) {
            float bd = res_d[lane];
            int kk = res_k[lane];
            for (uint32_t q = 1; q < csize; ++q) {
                float dv;
                int kv;
                ld_peer(&res_d[lane], &res_k[lane], q, dv, kv);
                if (nearer(dv, kv, bd, kk)) {
                    bd = dv;
                    kk = kv;
                }
            }
            const int64_t i = rows[lane];
            if (i >= 0) {
                labels[b * N + i] = kk;
                if (mindist) mindist[b * N + i] = bd;
            }
            if (obj_acc) {  // the listed points' share of the objective: one atomic per chunk
                float part = i >= 0 ? bd : 0.f;  // fp32 within the warp, fp64 across
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
                if (lane == 0 && part != 0.f) atomicAdd(obj_acc + b, (double)part);
            }
        }
        cl_sync();  // no CTA refills its result slots while CTA 0 may still read them
    }
}

// How many clusters of 16 CTAs this device holds at once (checked once per
// device; 0 when such clusters cannot be placed at all).
int max_clusters16() {
    static std::atomic<int> state[64];  // per device: 0 unknown, else 1 + the count
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return 0;
    }
    int s = state[dev].load(std::memory_order_acquire);
    if (s == 0) {
        bool ok = cudaFuncSetAttribute(rescan_kernel<__half>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                      cudaSuccess &&
                  cudaFuncSetAttribute(rescan_kernel<float>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                      cudaSuccess;
        int most = 1 << 30;
        for (int which = 0; ok && which < 2; ++which) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(kClusterMax, 1, 1);
            cfg.blockDim = dim3(kThreads, 1, 1);
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = kClusterMax;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int n = 0;
            ok = (which == 0 ? cudaOccupancyMaxActiveClusters(&n, rescan_kernel<__half>, &cfg)
                             : cudaOccupancyMaxActiveClusters(&n, rescan_kernel<float>, &cfg)) == cudaSuccess &&
                 n >= 1;
            most = std::min(most, n);
        }
        if (!ok) cudaGetLastError();
        s = 1 + (ok ? most : 0);
        state[dev].store(s, std::memory_order_release);
    }
    return s - 1;
}

}  // namespace

cudaError_t launch_rescan(const void* X, int dtype, const float* C, int64_t B, int64_t N, int64_t K, int64_t d,
                          int32_t* labels, float* mindist, double* obj_acc, const RescanList& list, int sms,
                          cudaStream_t st, const int32_t* stop, int32_t* reset) {
    if (!list.count || !list.rows) return cudaErrorInvalidValue;
    // enough clusters per batch to fill the GPU about four times when the lists are long; clusters of 16
    // CTAs (the centroids split 16 ways) only while all of them fit on the device at once: a second
    // wave of clusters costs even a launch whose lists are empty (~6 us for 32 batches)
    auto per_batch_for = [&](int c) {
        return std::max<int64_t>(1, std::min<int64_t>(ceil_div(N, kPoints), 4 * sms / (c * B)));
    };
    const int most16 = max_clusters16();
    const int cs = most16 > 0 && B * per_batch_for(kClusterMax) <= most16 ? kClusterMax : 8;
    const int64_t per_batch = per_batch_for(cs);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(cs * per_batch), (unsigned)B, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 2 : 1;
    if (dtype == KM_F16)
        return cudaLaunchKernelEx(&cfg, rescan_kernel<__half>, (const __half*)X, C, N, K, d, (const int32_t*)list.rows,
                                  (const int32_t*)list.count, list.cap, reset, labels, mindist, obj_acc, stop);
    return cudaLaunchKernelEx(&cfg, rescan_kernel<float>, (const float*)X, C, N, K, d, (const int32_t*)list.rows,
                              (const int32_t*)list.count, list.cap, reset, labels, mindist, obj_acc, stop);
}

}  // namespace km
