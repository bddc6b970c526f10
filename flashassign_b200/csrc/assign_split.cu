// FlashAssign split along the feature dimension, for fp16 points with
// d > 512, on the fifth-generation tensor cores (sm_100a).
//
// What it computes (papernotes.org "Flash-KMeans" page, 关键设计 1): for every
// point the nearest centroid under ||x - c||^2 = ||x||^2 + ||c||^2 - 2 x.c,
// lowest index on ties, the distances reduced on chip as they are produced
// and never written out.  The 7minutos.es article ("Usándolo") describes a
// second kernel path that splits the feature dimension for d beyond 512, and
// the papernotes.org page (局限与展望) names large d (4096 and up) as the
// limit of keeping point and centroid tiles on chip.  Past d = 512 the point
// rows of a unit no longer fit in shared memory beside a centroid pipeline
// (128 rows x d fp16 is 256 KB at d = 1024), so here both operands stream:
// every pipeline stage holds one 64-dimension chunk of the unit's points and
// the same chunk of two 256-centroid tiles, and the chunk's K=16 MMAs
// accumulate into two TMEM accumulators at once (one per tile).  Each point
// chunk therefore serves 512 centroids per pass, which halves the point
// re-reads (from L2) against one tile per pass.  The accumulators are freed
// one at a time, so the first tile's MMAs of the next pass wait only for the
// first accumulator's read-out.
//
// Layout per CTA pair (cluster of 2, tcgen05.mma.cta_group::2, kind::f16,
// M=256, N=256, K=16), the score arithmetic of the other fp16 kernels (the
// -||c||^2/2 term folded in as one more K=16 step of fp16 pieces against a
// slice of power-of-two weights, so s = x.c - ||c||^2/2 and the epilogue
// tracks the best two scores of each point, whose gap certifies its label,
// certify.cuh):
//   * stages: [128 points x 64 fp16] + 2 x [128 centroids x 64 fp16], all
//     128-byte swizzled, 48 KB per CTA, 4 stages;
//   * norm slices of both tiles ride with a pass's last chunk into one of two
//     slots (a slot is reused two passes later, after the MMAs that read it);
//   * ||x||^2 of the unit's rows is summed from global memory by the epilogue
//     warps while the unit's first pass is in the tensor pipe;
//   * one MMA issuer thread in the leader CTA, 8 epilogue warps (TMEM lane
//     quarter x 128-column half) joined per unit through a shared slot.
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
constexpr int kStages = 4;
constexpr int kAccSets = 2;                     // 2 x 256 TMEM columns: the two tiles of a pass
constexpr int kBoxBytes = kRows * 128;          // [128 rows x 64 fp16], 128-byte swizzled
constexpr int kExtBytes = 128 * 32;             // [128 rows x 16 fp16], 32-byte swizzled: ones / norm pieces
constexpr int kThreads = 320;                   // 10 warps: producer, MMA issuer, 8 epilogue
constexpr int kEpiWarp0 = 2;
constexpr int kEpiWarps = 8;
constexpr int kColParts = 2;                    // column halves per TMEM lane quarter
constexpr int kPartCols = kTileK / kColParts;   // 128 columns of each tile per epilogue warp
static_assert(kPartCols == 128, "the epilogue reduces 128-column slices (grid_rows, grid_top2)");
constexpr uint32_t kTmemCols = 512;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int kStageBytes = 3 * kBoxBytes;                          // points, tile 0, tile 1
constexpr int kStageOff = 0;
constexpr int kExtOff = kStageOff + kStages * kStageBytes;          // 2 slots x 2 tiles of norm pieces
constexpr int kOnesOff = kExtOff + 2 * kAccSets * kExtBytes;
constexpr int kMergeOff = kOnesOff + kExtBytes;                     // 2 slots x 128 rows x (best, second, label)
constexpr int kMergeBytes = 2 * kRows * 12;
constexpr int kBarOff = kMergeOff + kMergeBytes;
// c_full[4], c_empty[4], acc_full[2], acc_empty[2], m_full[2], m_empty[2]
constexpr int kNumBars = 2 * kStages + 2 * kAccSets + 4;
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;      // + tmem slot, flag, alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget of one CTA exceeded");
static_assert(kStageBytes % 1024 == 0 && kExtOff % 1024 == 0 && kOnesOff % 256 == 0,
              "swizzle atoms must stay aligned");

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
    int ktiles, passes, boxes;
    const __half* X;      // [B, N, d], for ||x||^2
    int32_t* labels;
    float* mindist;
    double* obj_acc;      // [B] running sum of minimum distances, nullable
    const int32_t* stop;  // nullable: when *stop, the launch does nothing
    int32_t* fault;
    RescanList list;      // the points left to the exact re-scan
};

// Sum of squares of rows n0 + 0..31 of batch b (rows past N give 0): the warp
// reads one row at a time, 16 bytes per lane, and lane r keeps row r's total.
__device__ __forceinline__ float row_norms(const __half* __restrict__ X, int64_t b, int64_t N, int64_t d, int64_t n0,
                                           int lane) {
    float mine = 0.f;
    const int64_t chunks = d / 8;
    for (int r = 0; r < 32; ++r) {
        float part = 0.f;
        if (n0 + r < N) {
            const uint4* row = reinterpret_cast<const uint4*>(X + (b * N + n0 + r) * d);
            for (int64_t c = lane; c < chunks; c += 32) {
                const uint4 xv = __ldg(row + c);
                const __half2* hh = reinterpret_cast<const __half2*>(&xv);
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const float2 f = __half22float2(hh[t]);
                    part = fmaf(f.x, f.x, part);
                    part = fmaf(f.y, f.y, part);
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (lane == r) mine = part;
    }
    return mine;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    assign_split_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_c,
                        const __grid_constant__ CUtensorMap tmap_e, const Params P) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t stage_base = sbase + kStageOff;
    const uint32_t ext_base = sbase + kExtOff;
    const uint32_t ones_base = sbase + kOnesOff;
    const uint32_t bars = sbase + kBarOff;
    const uint32_t bar_c_full = bars, bar_c_empty = bar_c_full + 8 * kStages;
    const uint32_t bar_acc_full = bar_c_empty + 8 * kStages, bar_acc_empty = bar_acc_full + 8 * kAccSets;
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
        for (int i = 0; i < kStages; ++i) {
            mbar_init(bar_c_full + 8 * i, 1);   // leader: its expect_tx; bytes from both CTAs
            mbar_init(bar_c_empty + 8 * i, 1);  // the issuer's commit
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
    const int boxes = P.boxes;

    if (warp == 0) {
        // ------------------------------ TMA producer (both CTAs) ------------------------------
        if (lane == 0) {
            uint32_t it_c = 0, it_p = 0;
            bool ok = true;
            for (int64_t u = pair; u < n_units && ok; u += P.pairs) {
                const int b = (int)(u / P.units_per_batch);
                const int n0 = (int)((u % P.units_per_batch) * kUnitRows) + (int)rank * kRows;
                for (int p = 0; p < P.passes && ok; ++p, ++it_p) {
                    const bool two = 2 * p + 1 < P.ktiles;
                    const int k0 = 2 * p * kTileK + (int)rank * kHalfTile;  // this CTA's rows of the first tile
                    const uint32_t slot = ext_base + (it_p & 1) * (kAccSets * kExtBytes);
                    for (int j = 0; j < boxes; ++j, ++it_c) {
                        const uint32_t cs = it_c % kStages;
                        if (!(ok = mbar_wait(bar_c_empty + 8 * cs, ((it_c / kStages) & 1) ^ 1, abort_flag, P.fault)))
                            break;
                        const bool last = j == boxes - 1;
                        const uint32_t tiles = two ? 2u : 1u;
                        if (rank == 0)
                            mbar_expect_tx(bar_c_full + 8 * cs,
                                           2u * (kBoxBytes + tiles * (kBoxBytes + (last ? kExtBytes : 0))));
                        const uint32_t cfull_leader = map_to_rank(bar_c_full + 8 * cs, 0);
                        const uint32_t stage = stage_base + cs * kStageBytes;
                        tma_load_pair(stage, &tmap_x, j * kBoxK, n0, b, cfull_leader);
                        tma_load_pair(stage + kBoxBytes, &tmap_c, j * kBoxK, k0, b, cfull_leader);
                        if (two) tma_load_pair(stage + 2 * kBoxBytes, &tmap_c, j * kBoxK, k0 + kTileK, b, cfull_leader);
                        if (last) {
                            tma_load_pair(slot, &tmap_e, 0, k0, b, cfull_leader);
                            if (two) tma_load_pair(slot + kExtBytes, &tmap_e, 0, k0 + kTileK, b, cfull_leader);
                        }
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer (leader CTA) ------------------------------
        if (rank == 0 && lane == 0) {
            uint32_t it_c = 0, it_p = 0, use0 = 0, use1 = 0;
            bool ok = true;
            for (int64_t u = pair; u < n_units && ok; u += P.pairs) {
                for (int p = 0; p < P.passes && ok; ++p, ++it_p) {
                    const bool two = 2 * p + 1 < P.ktiles;
                    const uint32_t slot = ext_base + (it_p & 1) * (kAccSets * kExtBytes);
                    if (!(ok = mbar_wait(bar_acc_empty, (use0 & 1) ^ 1, abort_flag, P.fault))) break;
                    tc_fence_after();
                    for (int j = 0; j < boxes; ++j, ++it_c) {
                        const uint32_t cs = it_c % kStages;
                        if (!(ok = mbar_wait(bar_c_full + 8 * cs, (it_c / kStages) & 1, abort_flag, P.fault))) break;
                        tc_fence_after();
                        const uint32_t stage = stage_base + cs * kStageBytes;
                        const uint64_t a_desc = umma_desc_sw128(stage);
                        const uint64_t b0_desc = umma_desc_sw128(stage + kBoxBytes);
                        const uint64_t b1_desc = umma_desc_sw128(stage + 2 * kBoxBytes);
#pragma unroll
                        for (int ks = 0; ks < kBoxK / 16; ++ks) {
                            const uint64_t off = (uint64_t)((ks * 32) >> 4);  // 32 bytes per K=16 step
                            umma_pair_f16(tmem_base, a_desc + off, b0_desc + off, (j > 0 || ks > 0) ? 1u : 0u);
                        }
                        if (two) {
                            if (j == 0) {  // the second accumulator is needed only now
                                if (!(ok = mbar_wait(bar_acc_empty + 8, (use1 & 1) ^ 1, abort_flag, P.fault))) break;
                                tc_fence_after();
                            }
#pragma unroll
                            for (int ks = 0; ks < kBoxK / 16; ++ks) {
                                const uint64_t off = (uint64_t)((ks * 32) >> 4);
                                umma_pair_f16(tmem_base + kTileK, a_desc + off, b1_desc + off,
                                              (j > 0 || ks > 0) ? 1u : 0u);
                            }
                        }
                        if (j == boxes - 1) {  // the norm terms: ones (points) x (-||c||^2/2 pieces)
                            umma_pair_f16(tmem_base, umma_desc_sw32(ones_base), umma_desc_sw32(slot), 1u);
                            if (two)
                                umma_pair_f16(tmem_base + kTileK, umma_desc_sw32(ones_base),
                                              umma_desc_sw32(slot + kExtBytes), 1u);
                        }
                        umma_commit_pair(bar_c_empty + 8 * cs);
                    }
                    if (!ok) break;
                    umma_commit_pair(bar_acc_full);
                    ++use0;
                    if (two) {
                        umma_commit_pair(bar_acc_full + 8);
                        ++use1;
                    }
                }
            }
        }
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kEpiWarps) {
        // ------------------------------ epilogue (both CTAs) ------------------------------
        const int e = warp - kEpiWarp0;
        const int q = warp % 4;   // TMEM lane quarter this warp may access
        const int h = e / 4;      // which 128-column half of each 256-column tile
        const int row = q * 32 + lane;
        const uint32_t acc_empty_leader0 = map_to_rank(bar_acc_empty, 0);
        uint32_t it_x = 0, use[kAccSets] = {0u, 0u};
        bool ok = true;
        const int units = (int)n_units, pairs = (int)P.pairs;  // < 2^23: 32-bit counters
        const int upb = (int)P.units_per_batch;
        for (int u = (int)pair; u < units && ok; u += pairs, ++it_x) {
            const int b = u / upb;
            const int nq = (u - b * upb) * kUnitRows + (int)rank * kRows + q * 32;  // this warp's first row
            // ||x||^2 of the warp's 32 rows (half 0), while the first pass is in the tensor pipe
            const float xnorm = h == 0 ? row_norms(P.X, b, P.N, P.d, nq, lane) : 0.f;
            float best = -INFINITY, second = -INFINITY;
            int label = -1;  // column of the running best
            for (int p = 0; p < P.passes && ok; ++p) {
                const int tiles = 2 * p + 1 < P.ktiles ? 2 : 1;
                for (int s = 0; s < tiles; ++s) {
                    if (!(ok = mbar_wait(bar_acc_full + 8 * s, use[s] & 1, abort_flag, P.fault))) break;
                    ++use[s];
                    __syncwarp();  // tcgen05.ld below is warp-collective
                    tc_fence_after();
                    const uint32_t tcol = tmem_base + ((uint32_t)(q * 32) << 16) + s * kTileK + h * kPartCols;
                    float v[kPartCols];
                    tmem_ld128(tcol, v);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(acc_empty_leader0 + 8 * s);
                    const int kt = 2 * p + s;
                    top2_slice128(v, kt * kTileK + h * kPartCols, best, second, label);
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
                const int n = nq + lane;
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

bool assign_split_supported(int64_t d, int dtype) { return dtype == KM_F16 && d > 512 && d % 64 == 0; }

cudaError_t launch_assign_split(const __half* X, const __half* chat, const __half* cext, int64_t B, int64_t N,
                                int64_t K, int64_t d, int32_t* labels, float* mindist, double* obj_acc,
                                const RescanList& list, int sms, cudaStream_t st, const int32_t* stop) {
    if (!assign_split_supported(d, KM_F16)) return cudaErrorNotSupported;
    if (!list.cmax || !list.count || !list.rows) return cudaErrorInvalidValue;
    CUtensorMap mx, mc, me;
    if (!make_map(&mx, X, 2, B, N, d, kBoxK, kRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mc, chat, 2, B, K, d, kBoxK, kHalfTile, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&me, cext, 2, B, padded_k(K), 16, 16, kHalfTile, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(assign_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    Params P;
    P.B = B; P.N = N; P.K = K; P.d = d;
    P.units_per_batch = ceil_div(N, kUnitRows);
    P.units = B * P.units_per_batch;
    P.ktiles = (int)ceil_div(K, kTileK);
    P.passes = (P.ktiles + 1) / 2;
    P.boxes = (int)(d / kBoxK);
    P.X = X;
    P.labels = labels;
    P.mindist = mindist;
    P.obj_acc = obj_acc;
    P.stop = stop;
    P.fault = fault_word();
    P.list = list;
    static std::atomic<int> pair_cache[kMaxDevices];
    const int max_pairs = co_resident_pairs((const void*)assign_split_kernel, kThreads, kSmemBytes, sms, pair_cache);
    P.pairs = P.units < max_pairs ? P.units : max_pairs;
    return launch_kernel(assign_split_kernel, dim3((unsigned)(2 * P.pairs)), dim3(kThreads), kSmemBytes, st, mx, mc,
                         me, P);
}

}  // namespace km
