// FlashAssign on the fifth-generation tensor cores (sm_100a).
//
// What it computes (papernotes.org "Flash-KMeans" page, 关键设计 1): for every
// point, the nearest centroid under ||x - c||^2 = ||x||^2 + ||c||^2 - 2 x.c,
// with the N x K distances reduced on chip as they are produced (running
// minimum m_i from +inf and index a_i from -1, a strict "<" so the lowest
// index keeps ties) -- the distance matrix never reaches HBM, so the kernel
// reads O(N d + K d) bytes instead of writing and re-reading O(N K).
//
// How, on a B200 (the page's design is Triton on an H200 with cp.async double
// buffering; this is a re-design for tcgen05/TMEM/TMA):
//   * persistent grid, one CTA per SM; a work unit is 256 consecutive points of
//     one batch (two 128-row MMA tiles), units strided over the grid so that
//     concurrently running CTAs share their batch's centroids in L2;
//   * warp 0 issues TMA loads: the unit's X tile (kept for all K) into one of
//     two X buffers, and 128-centroid tiles of C (fp16, pre-rounded) into a
//     3-stage ring, all 128-byte swizzled;
//   * warp 1 (one thread) issues tcgen05.mma kind::f16, M=128 N=128 K=16, fp32
//     accumulation in TMEM: for each C tile, both row tiles of the unit into
//     one of two 256-column accumulator sets, so the epilogue of tile t
//     overlaps the MMAs of tile t+1;
//   * warps 4..11 (one thread per point row, TMEM lane = row) read their row
//     32 columns at a time with tcgen05.ld, form s = ||c||^2/2 - x.c, and keep
//     the running minimum with a per-32-column group test: the group minimum is
//     compared with the running best, and only when it improves is the group's
//     32 scores kept in registers; the winning column is resolved once per
//     unit from the kept group (first column equal to the minimum).
//     mindist = ||x||^2 + 2 * min s, with ||x||^2 summed from the staged X tile.
// Every mbarrier wait is bounded (2 s of %globaltimer); on expiry the kernel
// records a fault code in the device fault word, stops issuing work, frees
// its TMEM and returns.
#include "km_internal.cuh"

#include <cuda.h>

namespace km {
namespace {

constexpr int kRowsPerTile = 128;               // MMA M and TMEM lanes
constexpr int kRowTiles = 2;                    // row tiles per unit
constexpr int kUnitRows = kRowsPerTile * kRowTiles;
constexpr int kTileK = kAssignTileK;            // centroids per C tile (MMA N)
constexpr int kBoxK = 64;                       // fp16 elements per 128-byte swizzle row
constexpr int kMaxBoxes = 2;                    // d <= 128
constexpr int kCStages = 3;
constexpr int kXBufs = 2;
constexpr int kAccSets = 2;
constexpr int kBoxBytes = kRowsPerTile * 128;   // one [128 rows x 64 fp16] swizzled box: 16 KB
constexpr int kThreads = 384;                   // 12 warps
constexpr int kEpiWarp0 = 4;
constexpr int kEpiWarps = 8;
constexpr uint32_t kTmemCols = 512;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

constexpr int kNStages = 3;                      // half-norm tiles in flight
constexpr int kNBytesPerStage = kTileK * 4;      // 128 fp32 half norms

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int kXBytes = kXBufs * kRowTiles * kMaxBoxes * kBoxBytes;  // 128 KB
constexpr int kCBytes = kCStages * kMaxBoxes * kBoxBytes;            // 96 KB
constexpr int kNOff = kXBytes + kCBytes;
constexpr int kBarOff = kNOff + kNStages * kNBytesPerStage;
constexpr int kNumBars = 2 * kXBufs + 2 * kCStages + 2 * kAccSets + 2 * kNStages;
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;  // + tmem slot, flags, alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget of one CTA exceeded");

// ---- PTX wrappers -------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: false when the CTA is aborting or the limit expired (which
// starts the abort and records the fault).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int32_t* fault) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            atomicExch(fault, FAULT_PIPELINE_TIMEOUT);
            return false;
        }
    }
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}
// UMMA shared-memory descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row core groups 1024 bytes apart (SBO), LBO unused (1),
// descriptor version 1 (sm_100).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor, kind::f16: D fp32, A and B fp16, both K-major, N, M.
constexpr uint32_t kIdesc = (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(kTileK >> 3) << 17) |
                            ((uint32_t)(kRowsPerTile >> 4) << 24);

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// 64 consecutive fp32 columns of this thread's TMEM lane, waited on.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* v) {
    uint32_t r[64];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
          "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
          "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int j = 0; j < 64; ++j) v[j] = __uint_as_float(r[j]);
}

struct Params {
    int64_t B, N, K, d;
    int64_t units_per_batch, units;
    int ktiles, ksteps, boxes;
    const float* cnh;  // [B, padded K] half squared norms, +inf padding
    int32_t* labels;
    float* mindist;
    int32_t* fault;
};

__global__ void __launch_bounds__(kThreads, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_c,
                     const Params P) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t x_base = sbase;
    const uint32_t c_base = sbase + kXBytes;
    const uint32_t bars = sbase + kBarOff;
    // barrier indices
    const uint32_t bar_x_full = bars, bar_x_empty = bars + 8 * kXBufs;
    const uint32_t bar_c_full = bars + 16 * kXBufs, bar_c_empty = bar_c_full + 8 * kCStages;
    const uint32_t bar_acc_full = bar_c_empty + 8 * kCStages, bar_acc_empty = bar_acc_full + 8 * kAccSets;
    const uint32_t bar_n_full = bar_acc_empty + 8 * kAccSets, bar_n_empty = bar_n_full + 8 * kNStages;
    const uint32_t n_base = sbase + kNOff;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + kNumBars * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kBarOff + kNumBars * 8 + 4);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kXBufs; ++i) {
            mbar_init(bar_x_full + 8 * i, 1);
            mbar_init(bar_x_empty + 8 * i, 1 + kEpiWarps);  // last MMA commit + every epilogue warp
        }
        for (int i = 0; i < kCStages; ++i) {
            mbar_init(bar_c_full + 8 * i, 1);
            mbar_init(bar_c_empty + 8 * i, 1);
        }
        for (int i = 0; i < kAccSets; ++i) {
            mbar_init(bar_acc_full + 8 * i, 1);
            mbar_init(bar_acc_empty + 8 * i, kEpiWarps);
        }
        for (int i = 0; i < kNStages; ++i) {
            mbar_init(bar_n_full + 8 * i, 1);
            mbar_init(bar_n_empty + 8 * i, kEpiWarps);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int boxes = P.boxes;
    const uint32_t x_tile_bytes = (uint32_t)(kRowTiles * boxes * kBoxBytes);
    const uint32_t c_tile_bytes = (uint32_t)(boxes * kBoxBytes);

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            uint32_t it_x = 0, it_c = 0;
            bool ok = true;
            for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x, ++it_x) {
                const int b = (int)(u / P.units_per_batch);
                const int n0 = (int)((u % P.units_per_batch) * kUnitRows);
                const uint32_t xb = it_x % kXBufs;
                if (!(ok = mbar_wait(bar_x_empty + 8 * xb, ((it_x / kXBufs) & 1) ^ 1, abort_flag, P.fault))) break;
                mbar_expect_tx(bar_x_full + 8 * xb, x_tile_bytes);
                for (int rt = 0; rt < kRowTiles; ++rt)
                    for (int kb = 0; kb < boxes; ++kb)
                        tma_load_3d(x_base + ((xb * kRowTiles + rt) * kMaxBoxes + kb) * kBoxBytes, &tmap_x,
                                    kb * kBoxK, n0 + rt * kRowsPerTile, b, bar_x_full + 8 * xb);
                for (int kt = 0; kt < P.ktiles; ++kt, ++it_c) {
                    const uint32_t cs = it_c % kCStages;
                    if (!(ok = mbar_wait(bar_c_empty + 8 * cs, ((it_c / kCStages) & 1) ^ 1, abort_flag, P.fault)))
                        break;
                    mbar_expect_tx(bar_c_full + 8 * cs, c_tile_bytes);
                    for (int kb = 0; kb < boxes; ++kb)
                        tma_load_3d(c_base + (cs * kMaxBoxes + kb) * kBoxBytes, &tmap_c, kb * kBoxK, kt * kTileK, b,
                                    bar_c_full + 8 * cs);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            uint32_t it_x = 0, it_c = 0, it_a = 0;
            bool ok = true;
            for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x, ++it_x) {
                const uint32_t xb = it_x % kXBufs;
                if (!(ok = mbar_wait(bar_x_full + 8 * xb, (it_x / kXBufs) & 1, abort_flag, P.fault))) break;
                for (int kt = 0; kt < P.ktiles; ++kt, ++it_c, ++it_a) {
                    const uint32_t cs = it_c % kCStages;
                    const uint32_t s = it_a % kAccSets;
                    if (!(ok = mbar_wait(bar_c_full + 8 * cs, (it_c / kCStages) & 1, abort_flag, P.fault))) break;
                    if (!(ok = mbar_wait(bar_acc_empty + 8 * s, ((it_a / kAccSets) & 1) ^ 1, abort_flag, P.fault)))
                        break;
                    tc_fence_after();
                    for (int rt = 0; rt < kRowTiles; ++rt) {
                        const uint32_t d_tmem = tmem_base + s * (kRowTiles * kTileK) + rt * kTileK;
                        for (int ks = 0; ks < P.ksteps; ++ks) {
                            const int kb = ks / 4;
                            const uint32_t koff = (uint32_t)(ks % 4) * 32;
                            const uint32_t a_addr = x_base + ((xb * kRowTiles + rt) * kMaxBoxes + kb) * kBoxBytes + koff;
                            const uint32_t b_addr = c_base + (cs * kMaxBoxes + kb) * kBoxBytes + koff;
                            umma_f16(d_tmem, umma_desc_sw128(a_addr), umma_desc_sw128(b_addr), ks > 0 ? 1u : 0u);
                        }
                    }
                    umma_commit(bar_c_empty + 8 * cs);
                    umma_commit(bar_acc_full + 8 * s);
                }
                if (ok) umma_commit(bar_x_empty + 8 * xb);
            }
        }
    } else if (warp == 2) {
        // ------------------------------ half-norm producer ------------------------------
        if (lane == 0) {
            uint32_t it_n = 0;
            bool ok = true;
            for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x) {
                const float* cnh_b = P.cnh + (u / P.units_per_batch) * (int64_t)P.ktiles * kTileK;
                for (int kt = 0; kt < P.ktiles; ++kt, ++it_n) {
                    const uint32_t ns = it_n % kNStages;
                    if (!(ok = mbar_wait(bar_n_empty + 8 * ns, ((it_n / kNStages) & 1) ^ 1, abort_flag, P.fault)))
                        break;
                    mbar_expect_tx(bar_n_full + 8 * ns, kNBytesPerStage);
                    bulk_load(n_base + ns * kNBytesPerStage, cnh_b + kt * kTileK, kNBytesPerStage, bar_n_full + 8 * ns);
                }
            }
        }
    } else if (warp >= kEpiWarp0) {
        // ------------------------------ epilogue ------------------------------
        const int e = warp - kEpiWarp0;
        const int q = warp % 4;            // TMEM lane quarter this warp may access
        const int rt = e / 4;              // row tile of the unit
        const int row_in_unit = rt * kRowsPerTile + q * 32 + lane;
        const int row_in_tile = q * 32 + lane;
        uint32_t it_x = 0, it_a = 0;
        bool ok = true;
        for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x, ++it_x) {
            const int64_t b = u / P.units_per_batch;
            const int64_t n = (u % P.units_per_batch) * kUnitRows + row_in_unit;
            const uint32_t xb = it_x % kXBufs;
            if (!(ok = mbar_wait(bar_x_full + 8 * xb, (it_x / kXBufs) & 1, abort_flag, P.fault))) break;
            // ||x||^2 from the staged tile: the swizzle permutes 16-byte chunks
            // within a 128-byte row, so the row's bytes are all in place.
            float xnorm = 0.f;
            for (int kb = 0; kb < boxes; ++kb) {
                const uint4* rowp = reinterpret_cast<const uint4*>(
                    smem + ((xb * kRowTiles + rt) * kMaxBoxes + kb) * kBoxBytes + row_in_tile * 128);
#pragma unroll
                for (int cch = 0; cch < 8; ++cch) {
                    const uint4 v = rowp[(cch + lane) & 7];  // lanes start on different banks
                    const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const float2 f = __half22float2(h[t]);
                        xnorm = fmaf(f.x, f.x, xnorm);
                        xnorm = fmaf(f.y, f.y, xnorm);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_x_empty + 8 * xb);

            float best = INFINITY;
            int gbest = -1;
            float kept[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) kept[j] = INFINITY;
            for (int kt = 0; kt < P.ktiles; ++kt, ++it_a) {
                const uint32_t s = it_a % kAccSets;
                const uint32_t ns = it_a % kNStages;
                if (!(ok = mbar_wait(bar_n_full + 8 * ns, (it_a / kNStages) & 1, abort_flag, P.fault))) break;
                if (!(ok = mbar_wait(bar_acc_full + 8 * s, (it_a / kAccSets) & 1, abort_flag, P.fault))) break;
                __syncwarp();  // tcgen05.ld below is warp-collective
                tc_fence_after();
                const uint32_t tcol = tmem_base + ((uint32_t)(q * 32) << 16) + s * (kRowTiles * kTileK) + rt * kTileK;
                const float4* cn = reinterpret_cast<const float4*>(smem + kNOff + ns * kNBytesPerStage);
#pragma unroll 1
                for (int half = 0; half < kTileK / 64; ++half) {
                    float v[64];
                    tmem_ld64(tcol + half * 64, v);
                    if (half == kTileK / 64 - 1) {
                        // every column of this tile is in registers: hand the accumulator back
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_acc_empty + 8 * s);
                    }
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        float* w = v + 32 * g;
                        float gmin = INFINITY;
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4) {
                            const float4 c = cn[half * 16 + g * 8 + j4];
                            w[4 * j4 + 0] = c.x - w[4 * j4 + 0];
                            w[4 * j4 + 1] = c.y - w[4 * j4 + 1];
                            w[4 * j4 + 2] = c.z - w[4 * j4 + 2];
                            w[4 * j4 + 3] = c.w - w[4 * j4 + 3];
                            gmin = fminf(gmin, fminf(fminf(w[4 * j4], w[4 * j4 + 1]), fminf(w[4 * j4 + 2], w[4 * j4 + 3])));
                        }
                        const bool better = gmin < best;  // strict: an earlier group keeps ties
                        if (__any_sync(0xffffffffu, better)) {
#pragma unroll
                            for (int j = 0; j < 32; ++j) kept[j] = better ? w[j] : kept[j];
                        }
                        if (better) {
                            best = gmin;
                            gbest = kt * (kTileK / 32) + half * 2 + g;
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_n_empty + 8 * ns);
            }
            if (!ok) break;
            // resolve the column: first position in the kept group equal to the minimum
            int jbest = 31;
#pragma unroll
            for (int j = 31; j >= 0; --j) jbest = (kept[j] == best) ? j : jbest;
            if (n < P.N) {
                P.labels[b * P.N + n] = gbest < 0 ? -1 : gbest * 32 + jbest;
                if (P.mindist) P.mindist[b * P.N + n] = fmaxf(fmaf(2.f, best, xnorm), 0.f);
            }
        }
    }

    // teardown: every role is done (or aborted); free TMEM
    tc_fence_before();
    __syncthreads();
    if (*abort_flag && threadIdx.x == 0) __nanosleep(1000000);  // let in-flight async copies land
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

// ---- host side ------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [B, rows, d] fp16, boxes of [1, 128 rows, 64 cols], 128-byte swizzle, zero fill.
bool make_map(CUtensorMap* m, const void* base, int64_t B, int64_t rows, int64_t d) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)B};
    cuuint64_t strides[2] = {(cuuint64_t)(d * 2), (cuuint64_t)(rows * d * 2)};
    cuuint32_t box[3] = {(cuuint32_t)kBoxK, (cuuint32_t)kRowsPerTile, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool assign_tc_supported(int64_t d, int dtype) { return dtype == KM_F16 && d >= 64 && d <= 128 && d % 8 == 0; }

cudaError_t launch_assign_tc(const __half* X, const __half* chat, const float* cnh, int64_t B, int64_t N, int64_t K,
                             int64_t d, int32_t* labels, float* mindist, int sms, cudaStream_t st) {
    if (!assign_tc_supported(d, KM_F16)) return cudaErrorNotSupported;
    CUtensorMap mx, mc;
    if (!make_map(&mx, X, B, N, d) || !make_map(&mc, chat, B, K, d)) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(assign_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    Params P;
    P.B = B; P.N = N; P.K = K; P.d = d;
    P.units_per_batch = ceil_div(N, kUnitRows);
    P.units = B * P.units_per_batch;
    P.ktiles = (int)ceil_div(K, kTileK);
    P.ksteps = (int)ceil_div(d, 16);
    P.boxes = (int)ceil_div(d, kBoxK);
    P.cnh = cnh;
    P.labels = labels;
    P.mindist = mindist;
    P.fault = fault_word();
    const int64_t grid = P.units < sms ? P.units : sms;
    assign_tc_kernel<<<(unsigned)grid, kThreads, kSmemBytes, st>>>(mx, mc, P);
    return cudaGetLastError();
}

}  // namespace km
