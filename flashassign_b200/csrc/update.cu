// Sort-Inverse Update, the gather-reduce half (papernotes.org "Flash-KMeans"
// page, 关键设计 2).  After the labels are argsorted, each CTA takes a fixed run
// of B_N consecutive sorted positions, splits it where the sorted label
// changes (the intervals [u, v) of the page), gathers the rows of X through
// sorted_idx, reduces each interval on chip, and touches global memory
// atomically only for intervals that may continue into a neighbouring CTA.
// The page's count of O((K + ceil(N / B_N)) d) atomic additions is met
// exactly: at most two intervals per CTA are added atomically; every other
// interval is a whole cluster owned by this CTA and is written with a plain
// store.  Cluster counts come from the segment offsets of the sorted labels
// (exact integers), which this kernel also writes while it walks them, so no
// counter atomics and no separate pass are needed.
//
// Layout of a CTA (16-byte chunks of a row per thread):
//   rows longer than 1 KB are split into 1 KB slices of W dimensions, one
//   slice per grid z (the same positions in every slice), so a CTA covers W = d
//   or W = 1024 / sizeof(T) dimensions of each row;
//   tpr = W * sizeof(T) / 16 threads cover one row; G = 256 / tpr row-lanes;
//   row-lane g walks 32 consecutive sorted positions (B_N = 32 G); each
//   thread streams its 16-byte chunk of the walk's rows through a ring of
//   four asynchronous copies in shared memory (so the bytes in flight cost
//   no registers) and keeps a running fp32 partial sum in registers.  A label
//   change inside the walk ends a piece:
//   pieces strictly inside the walk are whole clusters and are stored at once;
//   the first and last piece of each walk go to shared memory, where one pass
//   in position order joins equal labels across row-lanes and decides, from
//   the labels just outside the CTA's run, whether each joined interval is the
//   whole cluster (plain store) or a part of it (fp32 vector atomic add).
// In accumulate mode (points streamed in chunks, sums carried across
// launches) the plain stores become read-add-writes: within one launch each
// such cluster still has exactly one writer.
#include "km_internal.cuh"

namespace km {
namespace {

constexpr int kRowsPerLane = 32;
constexpr int kRing = 4;  // row chunks in flight per thread (a shared-memory ring, not registers)

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a)
                 : "memory");
    return v;
}
__device__ __forceinline__ uint32_t smem_u32addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
// 0, computed from v: an instruction that must wait for v, placed before a
// copy that reuses v's ring slot
__device__ __forceinline__ int zero_after(const uint4& v) {
    int z;
    asm volatile("and.b32 %0, %1, 0;" : "=r"(z) : "r"(v.x));
    return z;
}

template <typename T>
struct Chunk;
template <>
struct Chunk<__half> {
    static constexpr int kElems = 8;
    static __device__ __forceinline__ void add(float* acc, const uint4& v) {
        const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(h[e]);
            acc[2 * e] += f.x;
            acc[2 * e + 1] += f.y;
        }
    }
};
template <>
struct Chunk<float> {
    static constexpr int kElems = 4;
    static __device__ __forceinline__ void add(float* acc, const uint4& v) {
        acc[0] += __uint_as_float(v.x);
        acc[1] += __uint_as_float(v.y);
        acc[2] += __uint_as_float(v.z);
        acc[3] += __uint_as_float(v.w);
    }
};

// kSliced: rows are cut into slices of W dimensions along grid z; otherwise a
// CTA covers whole rows (W = d) and every slice term folds away at compile time.
// The gathers are latency-bound: resident warps and bytes in flight set the
// bandwidth.  At d = 128 (fp16) the whole-row form takes 40 registers and
// 36 KB of shared memory, six CTAs per SM; rings of 2 or 8 slots, or walks of
// 16 or 64 rows, measured slower.  Folding the slice terms in at run time
// (register-held gathers then) cost four registers, one CTA per SM and 17%.
template <typename T, bool kSliced>
__global__ void __launch_bounds__(256) update_kernel(const T* __restrict__ X, const int32_t* __restrict__ a_sorted,
                                                     const int32_t* __restrict__ sorted_idx, int64_t N, int64_t K,
                                                     int64_t d, int64_t W, int tpr, int G, float* __restrict__ sums,
                                                     int32_t* __restrict__ offsets, int accumulate,
                                                     const int32_t* __restrict__ stop) {
    pdl_trigger();
    pdl_wait();
    if (stop && *stop) return;
    constexpr int E = Chunk<T>::kElems;
    extern __shared__ __align__(16) unsigned char smem[];
    const int BN = G * kRowsPerLane;
    const int64_t Wd = kSliced ? W : d;                  // dimensions per CTA
    float* head_vec = reinterpret_cast<float*>(smem);    // [G][Wd]
    float* tail_vec = head_vec + (size_t)G * Wd;         // [G][Wd]
    int* s_lab = reinterpret_cast<int*>(tail_vec + (size_t)G * Wd);  // [BN]
    int* s_idx = s_lab + BN;                             // [BN]
    int* head_lab = s_idx + BN;                          // [G]
    int* tail_lab = head_lab + G;                        // [G]
    // [kRing][threads] 16-byte slots: slot i of thread t at ring0 + (i * threads + t) * 16
    const uint32_t ring0 = (smem_u32addr(tail_lab + G) + 15u) & ~15u;

    const int64_t b = blockIdx.y;
    const int64_t z0 = kSliced ? (int64_t)blockIdx.z * W : 0;  // first dimension of this slice
    const int Wz = kSliced ? (int)min(W, d - z0) : (int)d;      // its width
    const int64_t p0 = (int64_t)blockIdx.x * BN;
    const int64_t pend = min(p0 + BN, N);
    const int n = (int)(pend - p0);
    const int32_t* ab = a_sorted + b * N;
    for (int t = threadIdx.x; t < n; t += blockDim.x) {
        s_lab[t] = ab[p0 + t];
        s_idx[t] = sorted_idx[b * N + p0 + t];
    }
    __syncthreads();
    if (offsets && (!kSliced || blockIdx.z == 0)) {
        // Segment offsets of the sorted labels: position p starts every label k
        // with a[p-1] < k <= a[p] (labels clamped so nothing is written out of
        // bounds); the last run also closes labels above a[N-1] at N.
        int32_t* ob = offsets + b * (K + 1);
        for (int t = threadIdx.x; t <= n; t += blockDim.x) {
            const int64_t p = p0 + t;
            if (t == n && p != N) break;
            int64_t prev = t > 0 ? s_lab[t - 1] : (p0 > 0 ? ab[p0 - 1] : -1);
            int64_t cur = p == N ? K : s_lab[t];
            prev = min(max(prev, (int64_t)-1), K);
            cur = min(max(cur, (int64_t)-1), K);
            for (int64_t k = prev + 1; k <= cur; ++k) ob[k] = (int32_t)p;
        }
    }

    const int g = threadIdx.x / tpr, c = threadIdx.x % tpr;
    const int r0 = g * kRowsPerLane, r1 = min(r0 + kRowsPerLane, n);
    float* sums_b = sums + b * K * d + z0 + (int64_t)c * E;
    if (r0 >= r1) {
        if (c == 0) head_lab[g] = tail_lab[g] = -1;
    } else if (!kSliced || c * E < Wz) {  // (chunks past a narrower last slice idle; c = 0 never does)
        const T* xb = X + b * N * d + z0 + (int64_t)c * E;
        float acc[E];
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = 0.f;
        int cur = s_lab[r0];
        int piece = 0;
        // The walk's rows stream through a ring of kRing 16-byte slots per
        // thread (asynchronous copies, one commit group per row, empty past
        // the walk's end): the chunks in flight cost shared memory, not registers.
        const uint32_t slot_stride = blockDim.x * 16u;
        const uint32_t ring = ring0 + threadIdx.x * 16u;
#pragma unroll
        for (int i = 0; i < kRing; ++i) {
            if (r0 + i < r1) cp_async16(ring + i * slot_stride, xb + (int64_t)s_idx[r0 + i] * d);
            cp_async_commit();
        }
        for (int r = r0; r < r1; ++r) {
            cp_async_wait<kRing - 1>();  // row r's group has landed
            const uint32_t slot = ring + (uint32_t)((r - r0) & (kRing - 1)) * slot_stride;
            const uint4 vr = lds128(slot);
            if (r + kRing < r1) cp_async16(slot, xb + ((int64_t)s_idx[r + kRing] + zero_after(vr)) * d);
            cp_async_commit();
            {
                const int lab = s_lab[r];
                if (lab != cur) {
                    if (piece == 0) {
                        if (c == 0) head_lab[g] = cur;
#pragma unroll
                        for (int e = 0; e < E; ++e) head_vec[(size_t)g * Wd + c * E + e] = acc[e];
                    } else if (cur >= 0 && cur < K) {  // a whole cluster inside this walk
#pragma unroll
                        for (int e = 0; e < E; e += 4) {
                            float4* dst = reinterpret_cast<float4*>(sums_b + (int64_t)cur * d + e);
                            float4 o = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
                            if (accumulate) {  // this CTA is the only writer of the cluster in this launch
                                const float4 prev = *dst;
                                o.x += prev.x; o.y += prev.y; o.z += prev.z; o.w += prev.w;
                            }
                            *dst = o;
                        }
                    }
                    ++piece;
#pragma unroll
                    for (int e = 0; e < E; ++e) acc[e] = 0.f;
                    cur = lab;
                }
                Chunk<T>::add(acc, vr);
            }
        }
        cp_async_wait<0>();
        if (piece == 0) {  // the whole walk is one label: a head piece with no tail
            if (c == 0) {
                head_lab[g] = cur;
                tail_lab[g] = -1;
            }
#pragma unroll
            for (int e = 0; e < E; ++e) head_vec[(size_t)g * Wd + c * E + e] = acc[e];
        } else {
            if (c == 0) tail_lab[g] = cur;
#pragma unroll
            for (int e = 0; e < E; ++e) tail_vec[(size_t)g * Wd + c * E + e] = acc[e];
        }
    }
    __syncthreads();

    // Join the boundary pieces in position order; one thread per 4 dims.
    const int j4 = threadIdx.x * 4;
    if (j4 >= Wz) return;
    const int before = p0 > 0 ? ab[p0 - 1] : -1;   // label just before the run
    const int after = pend < N ? ab[pend] : -1;    // label just after it
    int run_lab = -1;
    bool run_first = false;
    float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
    bool seen = false;
    auto emit = [&](int lab, float4 v, bool first, bool last) {
        if (lab < 0 || lab >= K) return;
        const bool shared_left = first && before == lab;
        const bool shared_right = last && after == lab;
        float* dst = sums + (b * K + lab) * d + z0 + j4;
        if (shared_left || shared_right) {
            atomicAdd(reinterpret_cast<float4*>(dst), v);
        } else if (accumulate) {
            const float4 prev = *reinterpret_cast<const float4*>(dst);
            *reinterpret_cast<float4*>(dst) = make_float4(prev.x + v.x, prev.y + v.y, prev.z + v.z, prev.w + v.w);
        } else {
            *reinterpret_cast<float4*>(dst) = v;
        }
    };
    for (int gg = 0; gg < G; ++gg) {
#pragma unroll
        for (int which = 0; which < 2; ++which) {
            const int lab = which == 0 ? head_lab[gg] : tail_lab[gg];
            if (lab < 0) continue;
            const float4 v = *reinterpret_cast<const float4*>((which == 0 ? head_vec : tail_vec) + (size_t)gg * Wd + j4);
            if (seen && lab == run_lab) {
                run.x += v.x; run.y += v.y; run.z += v.z; run.w += v.w;
            } else {
                if (seen) emit(run_lab, run, run_first, false);
                run_first = !seen;
                seen = true;
                run_lab = lab;
                run = v;
            }
        }
    }
    if (seen) emit(run_lab, run, run_first, true);
}

template <typename T>
cudaError_t launch_t(const void* X, const int32_t* a_sorted, const int32_t* sorted_idx, int64_t B, int64_t N,
                     int64_t K, int64_t d, float* sums, int32_t* offsets, bool accumulate, cudaStream_t st,
                     const int32_t* stop) {
    const int64_t W = d * (int64_t)sizeof(T) <= 1024 ? d : 1024 / (int64_t)sizeof(T);  // dims per slice
    const int tpr = (int)(W * (int64_t)sizeof(T) / 16);                                 // <= 64
    const int G = 256 / tpr;                                                              // >= 4
    const int BN = G * kRowsPerLane;
    const size_t smem = sizeof(float) * 2 * (size_t)G * W + sizeof(int) * (2 * (size_t)BN + 2 * (size_t)G) + 16 +
                        (size_t)kRing * (size_t)(G * tpr) * 16;
    const bool sliced = W != d;
    void (*kernel)(const T*, const int32_t*, const int32_t*, int64_t, int64_t, int64_t, int64_t, int, int, float*,
                   int32_t*, int, const int32_t*) = sliced ? update_kernel<T, true> : update_kernel<T, false>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const dim3 grid((unsigned)ceil_div(N, BN), (unsigned)B, (unsigned)ceil_div(d, W));
    return launch_kernel(kernel, grid, dim3(G * tpr), smem, st, (const T*)X, a_sorted, sorted_idx, N, K, d, W, tpr, G,
                         sums, offsets, accumulate ? 1 : 0, stop);
}

}  // namespace

cudaError_t launch_update_sums(const void* X, int dtype, const int32_t* a_sorted, const int32_t* sorted_idx,
                               int64_t B, int64_t N, int64_t K, int64_t d, float* sums, int32_t* offsets,
                               cudaStream_t st, bool accumulate, const int32_t* stop) {
    if (dtype == KM_F16)
        return launch_t<__half>(X, a_sorted, sorted_idx, B, N, K, d, sums, offsets, accumulate, st, stop);
    return launch_t<float>(X, a_sorted, sorted_idx, B, N, K, d, sums, offsets, accumulate, st, stop);
}

}  // namespace km
