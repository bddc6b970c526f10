// FlashAssign for fp32 points on the fifth-generation tensor cores (sm_100a).
//
// What it computes (papernotes.org "Flash-KMeans" page, 关键设计 1): for every
// point the nearest centroid under ||x - c||^2 = ||x||^2 + ||c||^2 - 2 x.c,
// lowest index on ties, the N x K distances reduced on chip as they are
// produced so that only O(N d + K d) bytes cross HBM.
//
// fp32 on tf32 tensor cores.  An MMA of kind::tf32 reads 10 mantissa bits of
// each operand, so every fp32 value v is split into a head h (v with its low
// 13 mantissa bits cleared: exact in tf32) and a tail t = v - h (exact in
// fp32, read by the MMA to within one tf32 unit), and
//     x.c  ~=  x_h.c_h + x_h.c_t + x_t.c_h,
// three MMA products accumulated in fp32 (the dropped x_t.c_t and the tails'
// tf32 reading are below 3 * 2^-20 of sum_j |x_j c_j|).  The score
// s_k = x.c_k - ||c_k||^2 / 2 (the norm term added by one more K=8 step of
// tf32-exact pieces against a ones slice) is then within
//     e_k <= 2^-16.6 * (||x|| ||c_k|| + ||c_k||^2 / 2)
// of the exact value, fp32 accumulation over the 3 d/8 + 1 steps included.
// The epilogue keeps the best score s1 (its index) and the second best s2 of
// every point; when s1 - s2 >= delta = 2^-14 * (2 ||x|| cmax + cmax^2), with
// cmax^2 an upper bound of max_k ||c_k||^2, the two errors cannot reorder
// any pair and the tensor-core argmax is the exact argmin.  Every other
// point (near ties, duplicate centroids, non-finite scores) is appended to a
// per-batch list and re-scanned exactly, with direct differences on the CUDA
// cores (assign_simt.cu), which also writes its mindist and objective share.
//
// Layout per CTA pair (cluster of 2, tcgen05.mma.cta_group::2, kind::tf32,
// M=256, N=256, K=8):
//   * each CTA keeps its 128 point rows of the current unit resident, head
//     and tail (2 x 64 KB at d = 128): its own X producer thread loads the
//     tile by TMA, the epilogue warps split it in place (tail to the second
//     buffer), summing ||x||^2 on the way, and release it to the MMA issuer;
//   * centroid tiles of 256 (128 per CTA) stream as d/32 chunks -- head and
//     tail boxes of [128 x 32 fp32], 32 KB per CTA -- through a 2-stage ring,
//     the norm slice riding with the last chunk of each tile;
//   * one MMA issuer thread in the leader CTA (12 MMAs per chunk), two
//     256-column TMEM accumulator sets, 8 epilogue warps (TMEM lane quarter x
//     128-column half) joined per unit through a double-buffered shared slot.
// Every mbarrier wait is bounded (2 s of %globaltimer); on expiry the kernel
// records a fault code in the device fault word, stops issuing work, frees
// its TMEM and returns.
#include "tc_ptx.cuh"

namespace km {
using namespace ptx;
namespace {

constexpr int kRows = 128;                      // point rows per CTA per unit (TMEM lanes)
constexpr int kUnitRows = 2 * kRows;            // points per unit (per CTA pair)
constexpr int kTileK = kAssignTileK;            // centroids per K tile (MMA N) = 256
constexpr int kHalfTile = kTileK / 2;           // centroids staged per CTA per tile (128)
constexpr int kBoxF = 32;                       // fp32 elements per 128-byte swizzle row
constexpr int kMaxBoxes = 4;                    // d <= 128
constexpr int kCStages = 2;
constexpr int kAccSets = 2;                     // 2 x 256 TMEM columns
constexpr int kBoxBytes = kRows * 128;          // X: [128 rows x 32 fp32], 128-byte swizzled
constexpr int kCBoxBytes = kHalfTile * 128;     // C: [128 centroids x 32 fp32], 128-byte swizzled
constexpr int kExtBytes = 128 * 32;             // [128 rows x 8 fp32], 32-byte swizzled: ones / norm pieces
constexpr int kThreads = 320;                   // 10 warps: producers, MMA issuer, 8 epilogue
constexpr int kEpiWarp0 = 2;
constexpr int kEpiWarps = 8;
constexpr int kPartCols = kTileK / 2;           // 128 columns of each tile per epilogue warp
constexpr uint32_t kTmemCols = 512;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int kXHiOff = 0;
constexpr int kXLoOff = kXHiOff + kMaxBoxes * kBoxBytes;            // 64 KB of heads
constexpr int kCOff = kXLoOff + kMaxBoxes * kBoxBytes;              // 64 KB of tails
constexpr int kCStageBytes = 2 * kCBoxBytes + kExtBytes;            // 36 KB: head box, tail box, norm slice
constexpr int kOnesOff = kCOff + kCStages * kCStageBytes;
constexpr int kMergeOff = kOnesOff + kExtBytes;                     // 2 slots x 128 rows x (s1, s2, idx, xnorm)
constexpr int kMergeBytes = 2 * kRows * 16;
constexpr int kBarOff = kMergeOff + kMergeBytes;
// x_full, x_split, x_empty, c_full[2], c_empty[2], acc_full[2], acc_empty[2], m_full[2], m_empty[2]
constexpr int kNumBars = 3 + 2 * kCStages + 2 * kAccSets + 4;
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;      // + tmem slot, flag, alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget of one CTA exceeded");
static_assert(kCStageBytes % 1024 == 0 && kOnesOff % 256 == 0, "swizzle atoms must stay aligned");

// Instruction descriptor, kind::tf32: D fp32, A and B tf32 (format 2), both K-major, N=256, M=256.
constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(kTileK >> 3) << 17) |
                            ((uint32_t)(kUnitRows >> 4) << 24);

// Relative error budget of one score difference (see the header): twice the
// per-score bound 2^-16.6 rounded up to 2^-14, a 6x margin.
constexpr float kTieRel = 1.0f / 16384.0f;

__device__ __forceinline__ void umma_pair_tf32(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}
// TMA tile load into this CTA's shared memory completing on its own barrier.
__device__ __forceinline__ void tma_load_own(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
            "r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}
// Arrive on a barrier of either CTA of the pair, publishing this thread's
// earlier shared-memory writes at cluster scope.
__device__ __forceinline__ void mbar_arrive_release_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Bounded wait that also acquires, at cluster scope, what the arriving
// threads of either CTA released (their shared-memory writes).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                  int32_t* fault) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait_cluster(bar, parity)) {
        if (*abort_flag) return false;
        if (globaltimer() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicExch(fault, FAULT_PIPELINE_TIMEOUT);
            return false;
        }
    }
    return true;
}
__device__ __forceinline__ float tf32_head(float v) { return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u); }

struct Params {
    int64_t B, N, K, d;
    int64_t units_per_batch, units, pairs;
    int ktiles, boxes;
    const float* cmax;    // [B] upper bound of max_k ||c_k||^2
    int32_t* labels;
    float* mindist;
    double* obj_acc;      // [B] running sum of minimum distances of the resolved points, nullable
    int32_t* flag_count;  // [B] points listed for the exact re-scan (zero on entry)
    int32_t* flag_rows;   // [B, list_cap] their indices within the batch
    int64_t list_cap;     // a count above it makes the re-scan take the whole batch
    unsigned long long* rescans;  // running total of listed points (observability, nullable)
    const int32_t* stop;  // nullable: when *stop, the launch does nothing
    int32_t* fault;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    assign_tf32_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_c,
                       const __grid_constant__ CUtensorMap tmap_e, const Params P) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t xhi_base = sbase + kXHiOff, xlo_base = sbase + kXLoOff;
    const uint32_t c_base = sbase + kCOff;
    const uint32_t ones_base = sbase + kOnesOff;
    const uint32_t bars = sbase + kBarOff;
    const uint32_t bar_x_full = bars, bar_x_split = bars + 8, bar_x_empty = bars + 16;
    const uint32_t bar_c_full = bars + 24, bar_c_empty = bar_c_full + 8 * kCStages;
    const uint32_t bar_acc_full = bar_c_empty + 8 * kCStages, bar_acc_empty = bar_acc_full + 8 * kAccSets;
    const uint32_t bar_m_full = bar_acc_empty + 8 * kAccSets, bar_m_empty = bar_m_full + 16;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + kNumBars * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kBarOff + kNumBars * 8 + 4);
    float4* merge = reinterpret_cast<float4*>(smem + kMergeOff);  // [2][128] (s1, s2, idx bits, xnorm part)

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cta_rank();  // 0: leader CTA of the pair (issues the MMAs)
    const int64_t pair = blockIdx.x / 2;

    if (threadIdx.x == 0) {
        mbar_init(bar_x_full, 1);               // this CTA's producer: its expect_tx
        mbar_init(bar_x_split, 2 * kEpiWarps);  // leader: epilogue warps of both CTAs, tile split
        mbar_init(bar_x_empty, 1);              // the issuer's end-of-unit commit
        for (int i = 0; i < kCStages; ++i) {
            mbar_init(bar_c_full + 8 * i, 1);   // leader: its expect_tx; bytes from both CTAs
            mbar_init(bar_c_empty + 8 * i, 1);
        }
        for (int i = 0; i < kAccSets; ++i) {
            mbar_init(bar_acc_full + 8 * i, 1);
            mbar_init(bar_acc_empty + 8 * i, 2 * kEpiWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_m_full + 8 * i, 4);   // the warps of column half 1
            mbar_init(bar_m_empty + 8 * i, 4);  // the warps of column half 0
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // the points' extra K=8 step: all ones (any layout of it reads as ones)
    for (int i = threadIdx.x; i < kExtBytes / 16; i += kThreads) {
        const uint32_t one = 0x3F800000u;
        reinterpret_cast<uint4*>(smem + kOnesOff)[i] = make_uint4(one, one, one, one);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic-proxy writes visible to the MMA
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // everything above overlaps the previous kernel's tail; the centroid
    // tiles, their norm bound and the flag counters are written by it
    pdl_trigger();
    pdl_wait();
    // a converged iteration loop has set the stop flag: no units (straight to the teardown)
    const int64_t n_units = (P.stop && *P.stop) ? 0 : P.units;

    const int boxes = P.boxes;
    const int dcols = (int)P.d;
    const uint32_t x_bytes = (uint32_t)(boxes * kBoxBytes);

    if (warp == 0) {
        // ------------------------------ TMA producers (both CTAs) ------------------------------
        if (lane == 16) {
            // this CTA's X tiles, one unit at a time (the buffer is free once the unit's MMAs are done)
            uint32_t it_x = 0;
            for (int64_t u = pair; u < n_units; u += P.pairs, ++it_x) {
                const int b = (int)(u / P.units_per_batch);
                const int n0 = (int)((u % P.units_per_batch) * kUnitRows) + (int)rank * kRows;
                if (!mbar_wait(bar_x_empty, (it_x & 1) ^ 1, abort_flag, P.fault)) break;
                mbar_expect_tx(bar_x_full, x_bytes);
                for (int kb = 0; kb < boxes; ++kb)
                    tma_load_own(xhi_base + kb * kBoxBytes, &tmap_x, kb * kBoxF, n0, b, bar_x_full);
            }
        } else if (lane == 0) {
            // centroid chunks: head and tail boxes of 32 dimensions, the norm slice with the last
            uint32_t it_c = 0;
            bool ok = true;
            for (int64_t u = pair; u < n_units && ok; u += P.pairs) {
                const int b = (int)(u / P.units_per_batch);
                for (int kt = 0; kt < P.ktiles && ok; ++kt) {
                    const int k0 = kt * kTileK + (int)rank * kHalfTile;
                    for (int j = 0; j < boxes; ++j, ++it_c) {
                        const uint32_t cs = it_c % kCStages;
                        if (!(ok = mbar_wait(bar_c_empty + 8 * cs, ((it_c / kCStages) & 1) ^ 1, abort_flag, P.fault)))
                            break;
                        const bool last = j == boxes - 1;
                        if (rank == 0)
                            mbar_expect_tx(bar_c_full + 8 * cs, (uint32_t)(2 * (2 * kCBoxBytes + (last ? kExtBytes : 0))));
                        const uint32_t cfull_leader = map_to_rank(bar_c_full + 8 * cs, 0);
                        const uint32_t stage = c_base + cs * kCStageBytes;
                        tma_load_pair(stage, &tmap_c, j * kBoxF, k0, b, cfull_leader);
                        tma_load_pair(stage + kCBoxBytes, &tmap_c, dcols + j * kBoxF, k0, b, cfull_leader);
                        if (last) tma_load_pair(stage + 2 * kCBoxBytes, &tmap_e, 0, k0, b, cfull_leader);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer (leader CTA) ------------------------------
        if (rank == 0 && lane == 0) {
            uint32_t it_x = 0, it_c = 0, it_a = 0;
            bool ok = true;
            for (int64_t u = pair; u < n_units && ok; u += P.pairs, ++it_x) {
                if (!(ok = mbar_wait_cluster(bar_x_split, it_x & 1, abort_flag, P.fault))) break;
                tc_fence_after();
                for (int kt = 0; kt < P.ktiles && ok; ++kt, ++it_a) {
                    const uint32_t s = it_a % kAccSets;
                    if (!(ok = mbar_wait(bar_acc_empty + 8 * s, ((it_a / kAccSets) & 1) ^ 1, abort_flag, P.fault)))
                        break;
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + s * kTileK;
                    for (int j = 0; j < boxes; ++j, ++it_c) {
                        const uint32_t cs = it_c % kCStages;
                        if (!(ok = mbar_wait(bar_c_full + 8 * cs, (it_c / kCStages) & 1, abort_flag, P.fault))) break;
                        tc_fence_after();
                        const uint32_t stage = c_base + cs * kCStageBytes;
                        const uint64_t ah = umma_desc_sw128(xhi_base + j * kBoxBytes);
                        const uint64_t al = umma_desc_sw128(xlo_base + j * kBoxBytes);
                        const uint64_t bh = umma_desc_sw128(stage);
                        const uint64_t bl = umma_desc_sw128(stage + kCBoxBytes);
#pragma unroll
                        for (int ks = 0; ks < kBoxF / 8; ++ks) {
                            const uint64_t off = (uint64_t)((ks * 32) >> 4);  // 32 bytes per K=8 step
                            umma_pair_tf32(d_tmem, ah + off, bh + off, (j > 0 || ks > 0) ? 1u : 0u);
                            umma_pair_tf32(d_tmem, ah + off, bl + off, 1u);
                            umma_pair_tf32(d_tmem, al + off, bh + off, 1u);
                        }
                        if (j == boxes - 1)  // the norm term: ones (points) x (-||c||^2/2 pieces)
                            umma_pair_tf32(d_tmem, umma_desc_sw32(ones_base), umma_desc_sw32(stage + 2 * kCBoxBytes),
                                           1u);
                        umma_commit_pair(bar_c_empty + 8 * cs);
                    }
                    if (ok) umma_commit_pair(bar_acc_full + 8 * s);
                }
                if (ok) umma_commit_pair(bar_x_empty);
            }
        }
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kEpiWarps) {
        // ------------------------------ epilogue (both CTAs) ------------------------------
        const int e = warp - kEpiWarp0;
        const int q = warp % 4;   // TMEM lane quarter this warp may access
        const int h = e / 4;      // which 128-column half of each 256-column tile
        const int row = q * 32 + lane;
        const uint32_t acc_empty_leader0 = map_to_rank(bar_acc_empty, 0);
        const uint32_t x_split_leader = map_to_rank(bar_x_split, 0);
        uint32_t it_x = 0, it_a = 0;
        bool ok = true;
        const int units = (int)n_units, pairs = (int)P.pairs;  // < 2^23: 32-bit counters
        for (int u = (int)pair; u < units && ok; u += pairs, ++it_x) {
            // split this CTA's tile: head in place, tail to the second buffer; ||x||^2 on the way
            if (!(ok = mbar_wait(bar_x_full, it_x & 1, abort_flag, P.fault))) break;
            float xnorm = 0.f;
            for (int kb = h; kb < boxes; kb += 2) {
                float4* hi = reinterpret_cast<float4*>(smem + kXHiOff + kb * kBoxBytes + row * 128);
                float4* lo = reinterpret_cast<float4*>(smem + kXLoOff + kb * kBoxBytes + row * 128);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int cc = (c + lane) & 7;  // lanes start on different banks
                    const float4 v = hi[cc];
                    const float4 vh = make_float4(tf32_head(v.x), tf32_head(v.y), tf32_head(v.z), tf32_head(v.w));
                    hi[cc] = vh;
                    lo[cc] = make_float4(v.x - vh.x, v.y - vh.y, v.z - vh.z, v.w - vh.w);
                    xnorm = fmaf(v.x, v.x, xnorm);
                    xnorm = fmaf(v.y, v.y, xnorm);
                    xnorm = fmaf(v.z, v.z, xnorm);
                    xnorm = fmaf(v.w, v.w, xnorm);
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive_release_cluster(x_split_leader);

            float m1 = -INFINITY, m2 = -INFINITY;  // best and second-best score of this row's half
            int idx = -1;
            for (int kt = 0; kt < P.ktiles; ++kt, ++it_a) {
                const uint32_t s = it_a % kAccSets;
                if (!(ok = mbar_wait(bar_acc_full + 8 * s, (it_a / kAccSets) & 1, abort_flag, P.fault))) break;
                __syncwarp();  // tcgen05.ld below is warp-collective
                tc_fence_after();
                const uint32_t tcol = tmem_base + ((uint32_t)(q * 32) << 16) + s * kTileK + h * kPartCols;
#pragma unroll 1
                for (int sub = 0; sub < kPartCols / 64; ++sub) {
                    float v[64];
                    tmem_ld64(tcol + sub * 64, v);
                    if (sub == kPartCols / 64 - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(acc_empty_leader0 + 8 * s);
                    }
                    const int col0 = kt * kTileK + h * kPartCols + sub * 64;
#pragma unroll
                    for (int j = 0; j < 64; ++j) {
                        m2 = fmaxf(m2, fminf(m1, v[j]));
                        const bool better = v[j] > m1;  // strict: the lower column keeps ties
                        m1 = better ? v[j] : m1;
                        idx = better ? col0 + j : idx;
                    }
                }
            }
            if (!ok) break;
            // join the two halves of each row through a double-buffered slot
            const uint32_t ms = it_x & 1, mph = (it_x >> 1) & 1;
            if (h == 1) {
                if (!(ok = mbar_wait(bar_m_empty + 8 * ms, mph ^ 1, abort_flag, P.fault))) break;
                merge[ms * kRows + row] = make_float4(m1, m2, __int_as_float(idx), xnorm);
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_m_full + 8 * ms);
            } else {
                if (!(ok = mbar_wait(bar_m_full + 8 * ms, mph, abort_flag, P.fault))) break;
                const float4 o = merge[ms * kRows + row];
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_m_empty + 8 * ms);
                const int oidx = __float_as_int(o.z);
                // half 0 holds the lower columns: it keeps equal scores
                if (o.x > m1) {
                    m2 = fmaxf(o.y, m1);
                    m1 = o.x;
                    idx = oidx;
                } else {
                    m2 = fmaxf(m2, o.x);
                }
                xnorm += o.w;
                const int upb = (int)P.units_per_batch;
                const int b = u / upb;
                const int n = (u - b * upb) * kUnitRows + (int)rank * kRows + row;
                const bool valid = n < P.N;
                const float cm = P.cmax[b];
                const float delta = kTieRel * (2.f * sqrtf(xnorm) * sqrtf(cm) + cm);
                const bool listed = valid && !(m1 - m2 >= delta);  // NaN or -inf scores are listed too
                const float md = fmaxf(fmaf(-2.f, m1, xnorm), 0.f);
                if (valid) {
                    const int64_t o64 = (int64_t)b * P.N + n;
                    P.labels[o64] = idx;
                    if (P.mindist) P.mindist[o64] = md;
                }
                if (P.obj_acc) {  // the resolved points' share of the objective: one atomic per warp
                    float part = (valid && !listed) ? md : 0.f;  // fp32 within the warp, fp64 across
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
                    if (lane == 0) atomicAdd(P.obj_acc + b, (double)part);
                }
                const unsigned mask = __ballot_sync(0xffffffffu, listed);
                if (mask) {
                    int base = 0;
                    if (lane == 0) {
                        base = atomicAdd(P.flag_count + b, __popc(mask));
                        if (P.rescans) atomicAdd(P.rescans, (unsigned long long)__popc(mask));
                    }
                    base = __shfl_sync(0xffffffffu, base, 0);
                    const int pos = base + __popc(mask & ((1u << lane) - 1u));
                    if (listed && pos < P.list_cap) P.flag_rows[(int64_t)b * P.list_cap + pos] = n;
                }
            }
        }
    }

    // teardown: every role of both CTAs is done (or aborted); free the pair's TMEM
    tc_fence_before();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) __nanosleep(1000000);  // let in-flight async copies land
    cluster_sync();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace

bool assign_tf32_supported(int64_t d) { return d >= 32 && d <= 128 && d % 32 == 0; }

cudaError_t launch_assign_tf32(const float* X, const float* csplit, const float* cext, int64_t B, int64_t N,
                               int64_t K, int64_t d, int32_t* labels, float* mindist, double* obj_acc,
                               const RescanList& list, int sms, cudaStream_t st, const int32_t* stop) {
    if (!assign_tf32_supported(d)) return cudaErrorNotSupported;
    if (!list.cmax || !list.count || !list.rows) return cudaErrorInvalidValue;
    CUtensorMap mx, mc, me;
    if (!make_map(&mx, X, 4, B, N, d, kBoxF, kRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mc, csplit, 4, B, K, 2 * d, kBoxF, kHalfTile, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&me, cext, 4, B, padded_k(K), 8, 8, kHalfTile, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(assign_tf32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    Params P;
    P.B = B; P.N = N; P.K = K; P.d = d;
    P.units_per_batch = ceil_div(N, kUnitRows);
    P.units = B * P.units_per_batch;
    P.ktiles = (int)ceil_div(K, kTileK);
    P.boxes = (int)(d / kBoxF);
    P.cmax = list.cmax;
    P.labels = labels;
    P.mindist = mindist;
    P.obj_acc = obj_acc;
    P.flag_count = list.count;
    P.flag_rows = list.rows;
    P.list_cap = list.cap;
    P.rescans = list.total;
    P.stop = stop;
    P.fault = fault_word();
    static std::atomic<int> pair_cache[kMaxDevices];
    const int max_pairs = co_resident_pairs((const void*)assign_tf32_kernel, kThreads, kSmemBytes, sms, pair_cache);
    P.pairs = P.units < max_pairs ? P.units : max_pairs;
    return launch_kernel(assign_tf32_kernel, dim3((unsigned)(2 * P.pairs)), dim3(kThreads), kSmemBytes, st, mx, mc, me,
                         P);
}

}  // namespace km
