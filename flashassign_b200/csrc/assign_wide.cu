// FlashAssign for wide fp16 points (128 < d <= 512) on the fifth-generation
// tensor cores (sm_100a).
//
// What it computes (papernotes.org "Flash-KMeans" page, 关键设计 1): for every
// point the nearest centroid under ||x - c||^2 = ||x||^2 + ||c||^2 - 2 x.c,
// lowest index on ties, the N x K distances reduced on chip as they are
// produced.  The page's benchmarks go to d = 512 (its N = 1M, K = 65536,
// d = 512 row), and the 7minutos.es article ("Usándolo") describes one
// kernel path for d <= 512 and one split along d for larger d.  The d <= 128
// kernel (assign_tc.cu) stages a whole centroid tile per pipeline stage,
// which at d = 512 would be 128 KB a stage; here the reduction dimension is
// split: the unit's 128 point rows per CTA stay resident (128 KB at d = 512),
// the centroid tiles stream in 64-dimension chunks, and each chunk's four
// K=16 MMAs accumulate into the same TMEM accumulator.
//
// Layout per CTA pair (cluster of 2, tcgen05.mma.cta_group::2, kind::f16,
// M=256, N=256, K=16), the same score arithmetic as assign_tc.cu (the
// -||c||^2/2 term folded in as one more K=16 step of fp16 pieces against a
// slice of power-of-two weights, so s = x.c - ||c||^2/2 and the epilogue
// tracks the best two scores of each point, whose gap certifies its label,
// certify.cuh):
//   * X: one buffer of 128 rows x d fp16 per CTA (d/64 boxes of [128 x 64],
//     128-byte swizzled), loaded by TMA once its previous unit's MMAs are done
//     and the epilogue has summed ||x||^2 from it;
//   * C: [128 centroids x 64 fp16] chunks (16 KB per CTA) through a 4-stage
//     ring, the norm slice riding with the last chunk of each tile;
//   * one MMA issuer thread in the leader CTA (4 MMAs per chunk), two
//     256-column TMEM accumulator sets, 8 epilogue warps (TMEM lane quarter x
//     128-column half) joined per unit through a double-buffered shared slot.
// Every mbarrier wait is bounded (2 s of %globaltimer); on expiry the kernel
// records a fault code in the device fault word, stops issuing work, frees
// its TMEM and returns.
#include "certify.cuh"
#include "tc_ptx.cuh"

namespace km {
using namespace ptx;
namespace {

constexpr int kRows = 128;                      // point rows per CTA per unit (TMEM lanes)
constexpr int kUnitRows = 2 * kRows;            // points per unit (per CTA pair)
constexpr int kTileK = kAssignTileK;            // centroids per K tile (MMA N) = 256
constexpr int kHalfTile = kTileK / 2;           // centroids staged per CTA per tile (128)
constexpr int kBoxK = 64;                       // fp16 elements per 128-byte swizzle row
constexpr int kMaxBoxes = 8;                    // d <= 512
constexpr int kCStages = 4;
constexpr int kAccSets = 2;                     // 2 x 256 TMEM columns
constexpr int kBoxBytes = kRows * 128;          // X: [128 rows x 64 fp16], 128-byte swizzled
constexpr int kCBoxBytes = kHalfTile * 128;     // C: [128 centroids x 64 fp16], 128-byte swizzled
constexpr int kExtBytes = 128 * 32;             // [128 rows x 16 fp16], 32-byte swizzled: ones / norm pieces
constexpr int kThreads = 320;                   // 10 warps: producers, MMA issuer, 8 epilogue
constexpr int kEpiWarp0 = 2;
constexpr int kEpiWarps = 8;
constexpr int kColParts = 2;                    // column halves per TMEM lane quarter
constexpr int kPartCols = kTileK / kColParts;   // 128 columns of each tile per epilogue warp
static_assert(kPartCols == 128, "the epilogue reduces 128-column slices (grid_rows, grid_top2)");
constexpr uint32_t kTmemCols = 512;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int kXOff = 0;                                            // 128 KB of point rows
constexpr int kCOff = kXOff + kMaxBoxes * kBoxBytes;
constexpr int kCStageBytes = kCBoxBytes + kExtBytes;                // 20 KB: a chunk and the norm slice
constexpr int kOnesOff = kCOff + kCStages * kCStageBytes;
constexpr int kMergeOff = kOnesOff + kExtBytes;                     // 2 slots x 128 rows x (best, second, label)
constexpr int kMergeBytes = 2 * kRows * 12;
constexpr int kBarOff = kMergeOff + kMergeBytes;
// x_full[2], x_empty[2], c_full[4], c_empty[4], acc_full[2], acc_empty[2], m_full[2], m_empty[2]
constexpr int kNumBars = 4 + 2 * kCStages + 2 * kAccSets + 4;
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;      // + tmem slot, flag, alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget of one CTA exceeded");
static_assert(kCStageBytes % 1024 == 0 && kOnesOff % 256 == 0, "swizzle atoms must stay aligned");

// Instruction descriptor, kind::f16: D fp32, A and B fp16, both K-major, N=256, M=256.
constexpr uint32_t kIdesc = (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(kTileK >> 3) << 17) |
                            ((uint32_t)(kUnitRows >> 4) << 24);

__device__ __forceinline__ void umma_pair_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

struct Params {
    int64_t B, N, K, d;
    int64_t units_per_batch, units, pairs;
    int ktiles, boxes;
    int32_t* labels;
    float* mindist;
    double* obj_acc;      // [B] running sum of minimum distances, nullable
    const int32_t* stop;  // nullable: when *stop, the launch does nothing
    int32_t* fault;
    RescanList list;      // the points left to the exact re-scan
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    assign_wide_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_c,
                       const __grid_constant__ CUtensorMap tmap_e, const Params P) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t x_base = sbase + kXOff;
    const uint32_t c_base = sbase + kCOff;
    const uint32_t ones_base = sbase + kOnesOff;
    const uint32_t bars = sbase + kBarOff;
    // the X region holds two buffers of half its size when the rows fit (d <= 256), else one
    const int boxes = P.boxes;
    const int xbufs = boxes <= kMaxBoxes / 2 ? 2 : 1;
    const int xbuf_boxes = kMaxBoxes / xbufs;
    const uint32_t bar_x_full = bars, bar_x_empty = bars + 16;
    const uint32_t bar_c_full = bars + 32, bar_c_empty = bar_c_full + 8 * kCStages;
    const uint32_t bar_acc_full = bar_c_empty + 8 * kCStages, bar_acc_empty = bar_acc_full + 8 * kAccSets;
    const uint32_t bar_m_full = bar_acc_empty + 8 * kAccSets, bar_m_empty = bar_m_full + 16;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + kNumBars * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kBarOff + kNumBars * 8 + 4);
    float* merge_score = reinterpret_cast<float*>(smem + kMergeOff);                // [2][128]
    float* merge_second = reinterpret_cast<float*>(smem + kMergeOff + 8 * kRows);  // [2][128]
    int* merge_label = reinterpret_cast<int*>(smem + kMergeOff + 16 * kRows);      // [2][128]

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cta_rank();  // 0: leader CTA of the pair (issues the MMAs)
    const int64_t pair = blockIdx.x / 2;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_x_full + 8 * i, 1);               // leader: its expect_tx; bytes from both CTAs
            mbar_init(bar_x_empty + 8 * i, 1 + kEpiWarps);  // the issuer's end-of-unit commit + epilogue warps
        }
        for (int i = 0; i < kCStages; ++i) {
            mbar_init(bar_c_full + 8 * i, 1);
            mbar_init(bar_c_empty + 8 * i, 1);
        }
        for (int i = 0; i < kAccSets; ++i) {
            mbar_init(bar_acc_full + 8 * i, 1);
            mbar_init(bar_acc_empty + 8 * i, 2 * kEpiWarps);  // leader: epilogue warps of both CTAs
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_m_full + 8 * i, kEpiWarps / kColParts);  // the warps of column half 1
            mbar_init(bar_m_empty + 8 * i, kEpiWarps / kColParts); // the warps of column half 0
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // the points' extra K slice: the norm pieces' weights, the same in both
    // 16-byte halves of every row (so the 32-byte swizzle leaves it as it is)
    for (int i = threadIdx.x; i < kExtBytes / 16; i += kThreads)
        reinterpret_cast<uint4*>(smem + kOnesOff)[i] =
            make_uint4(kNormWeightW01, kNormWeightW23, kNormWeightW45, kNormWeightW67);
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
    // everything above overlaps the previous kernel's tail; the centroid tiles
    // and the objective accumulator are written by it
    pdl_trigger();
    pdl_wait();
    // a converged iteration loop has set the stop flag: no units (straight to the teardown)
    const int64_t n_units = (P.stop && *P.stop) ? 0 : P.units;
    const uint32_t x_bytes_pair = (uint32_t)(2 * boxes * kBoxBytes);

    if (warp == 0) {
        // ------------------------------ TMA producers (both CTAs) ------------------------------
        if (lane == 16) {
            uint32_t it_x = 0;
            for (int64_t u = pair; u < n_units; u += P.pairs, ++it_x) {
                const int b = (int)(u / P.units_per_batch);
                const int n0 = (int)((u % P.units_per_batch) * kUnitRows) + (int)rank * kRows;
                const uint32_t xb = it_x % xbufs;
                if (!mbar_wait(bar_x_empty + 8 * xb, ((it_x / xbufs) & 1) ^ 1, abort_flag, P.fault)) break;
                if (rank == 0) mbar_expect_tx(bar_x_full + 8 * xb, x_bytes_pair);
                const uint32_t xfull_leader = map_to_rank(bar_x_full + 8 * xb, 0);
                for (int kb = 0; kb < boxes; ++kb)
                    tma_load_pair(x_base + (xb * xbuf_boxes + kb) * kBoxBytes, &tmap_x, kb * kBoxK, n0, b,
                                  xfull_leader);
            }
        } else if (lane == 0) {
            // centroid chunks of 64 dimensions, the norm slice with the last of each tile
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
                            mbar_expect_tx(bar_c_full + 8 * cs, (uint32_t)(2 * (kCBoxBytes + (last ? kExtBytes : 0))));
                        const uint32_t cfull_leader = map_to_rank(bar_c_full + 8 * cs, 0);
                        const uint32_t stage = c_base + cs * kCStageBytes;
                        tma_load_pair(stage, &tmap_c, j * kBoxK, k0, b, cfull_leader);
                        if (last) tma_load_pair(stage + kCBoxBytes, &tmap_e, 0, k0, b, cfull_leader);
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
                const uint32_t xb = it_x % xbufs;
                if (!(ok = mbar_wait(bar_x_full + 8 * xb, (it_x / xbufs) & 1, abort_flag, P.fault))) break;
                tc_fence_after();
                const uint32_t xbuf = x_base + xb * xbuf_boxes * kBoxBytes;
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
                        const uint64_t a_desc = umma_desc_sw128(xbuf + j * kBoxBytes);
                        const uint64_t b_desc = umma_desc_sw128(stage);
#pragma unroll
                        for (int ks = 0; ks < kBoxK / 16; ++ks) {
                            const uint64_t off = (uint64_t)((ks * 32) >> 4);  // 32 bytes per K=16 step
                            umma_pair_f16(d_tmem, a_desc + off, b_desc + off, (j > 0 || ks > 0) ? 1u : 0u);
                        }
                        if (j == boxes - 1)  // the norm term: ones (points) x (-||c||^2/2 pieces)
                            umma_pair_f16(d_tmem, umma_desc_sw32(ones_base), umma_desc_sw32(stage + kCBoxBytes), 1u);
                        umma_commit_pair(bar_c_empty + 8 * cs);
                    }
                    if (ok) umma_commit_pair(bar_acc_full + 8 * s);
                }
                if (ok) umma_commit_pair(bar_x_empty + 8 * xb);
            }
        }
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kEpiWarps) {
        // ------------------------------ epilogue (both CTAs) ------------------------------
        const int e = warp - kEpiWarp0;
        const int q = warp % 4;   // TMEM lane quarter this warp may access
        const int h = e / 4;      // which 128-column half of each 256-column tile
        const int row = q * 32 + lane;
        const uint32_t acc_empty_leader0 = map_to_rank(bar_acc_empty, 0);
        uint32_t it_x = 0, it_a = 0;
        bool ok = true;
        const int units = (int)n_units, pairs = (int)P.pairs;  // < 2^23: 32-bit counters
        for (int u = (int)pair; u < units && ok; u += pairs, ++it_x) {
            const uint32_t xb = it_x % xbufs;
            float xnorm = 0.f;
            float best = -INFINITY, second = -INFINITY;
            int label = -1;  // column of the running best
            for (int kt = 0; kt < P.ktiles; ++kt, ++it_a) {
                const uint32_t s = it_a % kAccSets;
                if (!(ok = mbar_wait(bar_acc_full + 8 * s, (it_a / kAccSets) & 1, abort_flag, P.fault))) break;
                __syncwarp();  // tcgen05.ld below is warp-collective
                tc_fence_after();
                const uint32_t tcol = tmem_base + ((uint32_t)(q * 32) << 16) + s * kTileK + h * kPartCols;
                float v[kPartCols];
                tmem_ld128(tcol, v);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(acc_empty_leader0 + 8 * s);
                top2_slice128(v, kt * kTileK + h * kPartCols, best, second, label);
                if (kt == 0) {
                    // The MMA has consumed this unit's X tile, so it is in place.
                    // ||x||^2 from it (half 0 of each row; the swizzle permutes
                    // 16-byte chunks within a 128-byte row, so each row's bytes
                    // are all in that row); then the buffer may be refilled.
                    if (h == 0) {
                        for (int kb = 0; kb < boxes; ++kb)
                            xnorm = add_sq_row_sw128_f16(smem + kXOff + (xb * xbuf_boxes + kb) * kBoxBytes + row * 128,
                                                         lane, xnorm);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_x_empty + 8 * xb);
                }
            }
            if (!ok) break;
            // join the column halves of each row (the best two scores, the lower
            // index on equal ones) through a double-buffered shared slot with
            // bounded handoffs, then certify and write
            const uint32_t ms = it_x & 1, mph = (it_x >> 1) & 1;
            if (h == 1) {
                if (!(ok = mbar_wait(bar_m_empty + 8 * ms, mph ^ 1, abort_flag, P.fault))) break;
                merge_score[ms * kRows + row] = best;
                merge_second[ms * kRows + row] = second;
                merge_label[ms * kRows + row] = label;
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_m_full + 8 * ms);
            } else {
                if (!(ok = mbar_wait(bar_m_full + 8 * ms, mph, abort_flag, P.fault))) break;
                const float ob = merge_score[ms * kRows + row];
                const float os = merge_second[ms * kRows + row];
                const int ol = merge_label[ms * kRows + row];
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_m_empty + 8 * ms);
                top2_join(best, second, label, ob, os, ol);  // this half holds the lower columns
                const int upb = (int)P.units_per_batch;
                const int b = u / upb;
                const int n = (u - b * upb) * kUnitRows + (int)rank * kRows + row;
                float part = certify_top2(P.list, P.list.cmax[b], b, P.N, n, n < P.N, best, second, label, xnorm,
                                                P.labels, P.mindist, lane);
                if (P.obj_acc) {  // the objective: this warp's certified rows, one atomic per warp
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
                    if (lane == 0) atomicAdd(P.obj_acc + b, (double)part);
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

bool assign_wide_supported(int64_t d, int dtype) { return dtype == KM_F16 && d > 128 && d <= 512 && d % 64 == 0; }

cudaError_t launch_assign_wide(const __half* X, const __half* chat, const __half* cext, int64_t B, int64_t N,
                               int64_t K, int64_t d, int32_t* labels, float* mindist, double* obj_acc,
                               const RescanList& list, int sms, cudaStream_t st, const int32_t* stop) {
    if (!assign_wide_supported(d, KM_F16)) return cudaErrorNotSupported;
    if (!list.cmax || !list.count || !list.rows) return cudaErrorInvalidValue;
    CUtensorMap mx, mc, me;
    if (!make_map(&mx, X, 2, B, N, d, kBoxK, kRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mc, chat, 2, B, K, d, kBoxK, kHalfTile, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&me, cext, 2, B, padded_k(K), 16, 16, kHalfTile, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(assign_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    Params P;
    P.B = B; P.N = N; P.K = K; P.d = d;
    P.units_per_batch = ceil_div(N, kUnitRows);
    P.units = B * P.units_per_batch;
    P.ktiles = (int)ceil_div(K, kTileK);
    P.boxes = (int)(d / kBoxK);
    P.labels = labels;
    P.mindist = mindist;
    P.obj_acc = obj_acc;
    P.stop = stop;
    P.fault = fault_word();
    P.list = list;
    static std::atomic<int> pair_cache[kMaxDevices];
    const int max_pairs = co_resident_pairs((const void*)assign_wide_kernel, kThreads, kSmemBytes, sms, pair_cache);
    P.pairs = P.units < max_pairs ? P.units : max_pairs;
    return launch_kernel(assign_wide_kernel, dim3((unsigned)(2 * P.pairs)), dim3(kThreads), kSmemBytes, st, mx, mc, me,
                         P);
}

}  // namespace km
