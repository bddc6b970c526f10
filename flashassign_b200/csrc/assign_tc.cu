// FlashAssign on the fifth-generation tensor cores (sm_100a), two SMs per MMA.
//
// What it computes (papernotes.org "Flash-KMeans" page, 关键设计 1): for every
// point the nearest centroid under ||x - c||^2 = ||x||^2 + ||c||^2 - 2 x.c, the
// N x K distances reduced on chip as they are produced -- a running extremum
// per point from its initial value and index -1, replaced only on strict
// improvement, so the lowest index keeps ties -- so that the distance matrix
// never reaches HBM and the kernel reads O(N d + K d) bytes, not O(N K).
//
// How, on a B200 (the page's kernel is Triton on an H200 with cp.async double
// buffering; this is a re-design for tcgen05 / TMEM / TMA / CTA pairs):
//   * The score of centroid k for point x is s = x.c_k - ||c_k||^2 / 2, and
//     argmin_k ||x - c_k||^2 = argmax_k s.  The whole score comes out of the
//     tensor cores: each point row gets one extra 16-wide K slice of ones and
//     each centroid row the matching slice holding -||c||^2/2 split into fp16
//     pieces against power-of-two weights on the points' side
//     (norm_piece_weight), so one more K=16 MMA step adds the norm term in
//     fp32 and the epilogue only tracks maxima.
//   * CTA pairs (a cluster of 2) run tcgen05.mma.cta_group::2 with M=256,
//     N=256, K=16: each CTA stages its own 128 point rows and its own half
//     (128) of each 256-centroid tile, so every instruction runs at the full
//     N=256 rate (128 cycles) while each SM reads only half of the B operand:
//     about 64 B/cycle of operand reads plus ~31 B/cycle of TMA writes, within
//     the shared-memory bandwidth (an N=128 tile would need ~125 B/cycle).
//     Two 256-column accumulator sets fill the 512 TMEM columns.
//   * Persistent grid of pairs; a work unit is 256 consecutive points of one
//     batch; units are strided over the pairs so that pairs running at the
//     same time share their batch's centroids in L2.  When a batch's tiles
//     fit the ring one per stage (an even count, at most four: K in
//     (256, 512] or (768, 1024]) they stay resident over a pair's run of units
//     in one batch instead of being reloaded for every unit (4% at K = 1024).
//   * Warp roles per CTA (12 warps): warp 0 issues TMA loads (one thread:
//     X tiles of the units into two buffers; another: centroid tiles plus
//     their norm slices into a 4-stage ring, so that with two tiles in the
//     tensor pipe two more are in flight from L2), completing on the leader
//     CTA's barriers; warp 1 allocates TMEM for the pair; in the leader CTA, warps
//     1 and 10 issue the MMAs (alternate tiles) and commit them to both CTAs'
//     barriers; warps 2..9 are the epilogue: TMEM lane = point row, two warps
//     per row split each tile's 256 columns in 128-column slices, read in one
//     128-column TMEM load, the accumulator released as soon as they are in
//     registers; warp 11 finishes each unit (below), so that nothing but tile
//     work sits between two accumulator releases of the epilogue warps.
//   * Epilogue: each warp's 128-column slice of a tile is reduced to every
//     point's best and second-best score as an 8 x 16 grid (row and column
//     maxima, about 1.5 ALU instructions per score; certify.cuh) and folded
//     into the running (best, second, label); at the end of a unit each
//     epilogue warp posts them to a double-buffered shared slot.
//   * Unit finish (warp 11): ||x||^2 of each row is either read (the later
//     assignments of a Lloyd loop, from an array the first one wrote), or
//     summed from the staged X tile as soon as the unit's first tile of MMAs
//     has completed (a commit on a per-buffer barrier), the X buffer being
//     released right after; at the unit's end the two column slices are
//     joined (larger score, then lower index), and each point whose label
//     the scores' error bound certifies (certify.cuh) gets its label and
//     mindist = ||x||^2 - 2 * best and adds to the objective (summed in fp32,
//     one fp64 atomic per unit); the others are listed for the exact
//     re-scan.  Three X buffers with the release at the unit's end left room
//     for only three centroid stages: 5% slower at K = 1024.
//   * The issuers carry their unit and batch counters in 32 bits (a 64-bit
//     division between two units' MMAs cost 7% at K = 1024) and issue each
//     tile's K steps unrolled, with immediate descriptor offsets.
//   * Two accumulator sets bound the rate at K = 1024: tile t+2 starts only
//     after tile t's MMAs have completed, its TMEM has been read and the
//     release has reached the issuer (~2900 cycles for two tiles against 2300
//     of MMA work).  Narrower tiles would give more sets but read the points'
//     operand twice as often from shared memory (above).
//   * Measured on B200: in a long loop the 1 kW power cap lowers the SM
//     clock (~1.6-1.7 GHz at K = 1024 under the profiler, ~1.4 GHz at
//     K = 4096), so part of any saving in cycles per tile is paid back as a
//     lower clock.
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
constexpr int kMaxBoxes = 2;                    // d <= 128
constexpr int kCStages = 4;
constexpr int kXBufs = 2;
constexpr int kAccSets = 2;                     // 2 x 256 TMEM columns
constexpr int kBoxBytes = 128 * 128;            // X: [128 rows x 64 fp16], 128-byte swizzled
constexpr int kCBoxBytes = kHalfTile * 128;     // C: [128 centroids x 64 fp16], 128-byte swizzled
constexpr int kExtBytes = 128 * 32;             // ones: [128 rows x 16 fp16], 32-byte swizzled
constexpr int kCExtBytes = kHalfTile * 32;      // norm slice: [128 centroids x 16 fp16], 32-byte swizzled
constexpr int kThreads = 384;                   // 12 warps: producers, MMA issuer A, 8 epilogue, issuer B, merge
constexpr int kEpiWarp0 = 2;
constexpr int kMmaWarpB = 10;                   // second issuer, on another SMSP than warp 1
constexpr int kMergeWarp = 11;                  // joins the halves, ||x||^2, outputs (warps go in fours: no extra registers)
constexpr int kEpiWarps = 8;                    // at most 3 warps per SMSP: up to 168 registers each
constexpr int kColParts = kEpiWarps / 4;        // warps per TMEM lane quarter, each with a column slice
constexpr int kMaxKSteps = kMaxBoxes * kBoxK / 16;  // K=16 MMA steps of the widest points (d = 128)
constexpr int kPartCols = kTileK / kColParts;   // 128 columns of each tile per epilogue warp
static_assert(kPartCols == 128, "the epilogue reduces 128-column slices (grid_rows, grid_top2)");
constexpr uint32_t kTmemCols = 512;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int kXOff = 0;
constexpr int kXBytes = kXBufs * kMaxBoxes * kBoxBytes;             // 64 KB
constexpr int kCOff = kXOff + kXBytes;
constexpr int kCStageBytes = kMaxBoxes * kCBoxBytes + kCExtBytes;  // 36 KB: centroid boxes + norm slice
constexpr int kCBytes = kCStages * kCStageBytes;                    // 144 KB
constexpr int kAOnesOff = kCOff + kCBytes;                          // 4 KB of ones (the points' extra slice)
constexpr int kMergeOff = kAOnesOff + kExtBytes;  // 2 slots x 2 halves x 128 rows x (best, second, label)
constexpr int kMergeSlots = 2 * kColParts * kRows;
constexpr int kMergeBytes = kMergeSlots * 12;
constexpr int kBarOff = kMergeOff + kMergeBytes;
// x_full/x_empty, c_full/c_empty, acc_full/acc_empty, merge handoff (2 slots x full/empty), x_used
constexpr int kNumBars = 2 * kXBufs + 2 * kCStages + 2 * kAccSets + 4 + kXBufs;
constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16 + 1024;      // + tmem slot, flag, alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget of one CTA exceeded");
static_assert(kCStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");

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
    int ktiles, ksteps, boxes;
    int resident;  // the batch's centroid tiles stay in the ring across the units of a batch (see the producer)
    int32_t* labels;
    float* mindist;
    double* obj_acc;  // [B] running sum of minimum distances, nullable
    float* dense;     // dense mode: [B, padded K, N] scores, written instead of reduced
    float* xnorm;     // [B, N] ||x||^2, written when non-null (always in dense mode)
    const float* xnorm_in;  // [B, N] ||x||^2 of these points from an earlier launch (nullable): read, not computed
    const int32_t* stop;  // nullable: when *stop, the launch does nothing
    int32_t* fault;
    RescanList list;      // the points left to the exact re-scan
};

// kDense (the dense-distance ablation): the same MMA pipeline, but every
// tile's scores are written to P.dense and ||x||^2 to P.xnorm instead of
// being reduced on chip -- the N x K matrix round trip that FlashAssign avoids.
template <bool kDense>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_c,
                     const __grid_constant__ CUtensorMap tmap_e, const Params P) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t x_base = sbase + kXOff;
    const uint32_t c_base = sbase + kCOff;
    const uint32_t ones_base = sbase + kAOnesOff;
    const uint32_t bars = sbase + kBarOff;
    const uint32_t bar_x_full = bars, bar_x_empty = bars + 8 * kXBufs;
    const uint32_t bar_c_full = bars + 16 * kXBufs, bar_c_empty = bar_c_full + 8 * kCStages;
    const uint32_t bar_acc_full = bar_c_empty + 8 * kCStages, bar_acc_empty = bar_acc_full + 8 * kAccSets;
    const uint32_t bar_m_full = bar_acc_empty + 8 * kAccSets, bar_m_empty = bar_m_full + 16;
    const uint32_t bar_x_used = bar_m_empty + 16;  // a unit's first tile of MMAs has completed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + kNumBars * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kBarOff + kNumBars * 8 + 4);
    float* merge_score = reinterpret_cast<float*>(smem + kMergeOff);                      // [2][parts][128]
    float* merge_second = reinterpret_cast<float*>(smem + kMergeOff + 4 * kMergeSlots);  // [2][parts][128]
    int* merge_label = reinterpret_cast<int*>(smem + kMergeOff + 8 * kMergeSlots);       // [2][parts][128]

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cta_rank();         // 0: leader CTA of the pair (issues the MMAs)
    const int64_t pair = blockIdx.x / 2;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kXBufs; ++i) {
            mbar_init(bar_x_full + 8 * i, 1);               // leader: its expect_tx; bytes from both CTAs
            // both issuers' end-of-unit commits, and the merge warp once it has
            // read ||x||^2 from the buffer (not when the norms are given)
            mbar_init(bar_x_empty + 8 * i, P.xnorm_in ? 2 : 3);
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
            mbar_init(bar_m_full + 8 * i, kEpiWarps);      // every epilogue warp has posted its half
            mbar_init(bar_m_empty + 8 * i, 1);             // the merge warp has read the slot
        }
        for (int i = 0; i < kXBufs; ++i) mbar_init(bar_x_used + 8 * i, 1);  // the issuer of a unit's first tile
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // the points' extra K slice: the norm pieces' weights, the same in both
    // 16-byte halves of every row (so the 32-byte swizzle leaves it as it is)
    for (int i = threadIdx.x; i < kExtBytes / 16; i += kThreads)
        reinterpret_cast<uint4*>(smem + kAOnesOff)[i] =
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
    const uint32_t x_bytes_pair = (uint32_t)(2 * boxes * kBoxBytes);
    const uint32_t c_bytes_pair = (uint32_t)(2 * (boxes * kCBoxBytes + kCExtBytes));

    if (warp == 0) {
        // ------------------------------ TMA producers (both CTAs) ------------------------------
        // lane 16 streams the units' X tiles (a unit ahead, so HBM latency is
        // hidden behind a whole unit of MMAs); lane 0 streams the centroid
        // tiles and their norm slices through the 4-stage ring.
        const int units = (int)n_units, pairs = (int)P.pairs, upb = (int)P.units_per_batch;  // < 2^23
        if (lane == 16) {
            uint32_t it_x = 0;
            int b = (int)pair / upb, r = (int)pair % upb;  // unit u's batch and index in it, carried along
            for (int u = (int)pair; u < units; u += pairs, ++it_x) {
                const int n0 = r * kUnitRows + (int)rank * kRows;
                const uint32_t xb = it_x % kXBufs;
                if (!mbar_wait(bar_x_empty + 8 * xb, ((it_x / kXBufs) & 1) ^ 1, abort_flag, P.fault)) break;
                if (rank == 0) mbar_expect_tx(bar_x_full + 8 * xb, x_bytes_pair);
                const uint32_t xfull_leader = map_to_rank(bar_x_full + 8 * xb, 0);
                for (int kb = 0; kb < boxes; ++kb)
                    tma_load_pair(x_base + (xb * kMaxBoxes + kb) * kBoxBytes, &tmap_x, kb * kBoxK, n0, b, xfull_leader);
                r += pairs;
                if (r >= upb) {
                    b += r / upb;
                    r %= upb;
                }
            }
        } else if (lane == 0) {
            // Resident mode (an even number of tiles, at most one per stage): tile
            // kt of the batch lives in stage kt and is loaded once per run of the
            // pair's units in one batch (an epoch), not once per unit; a stage is
            // refilled after the epoch's last MMA on it, so a batch change still
            // streams tile by tile.
            uint32_t it_c = 0, ep = 0;
            int prev_b = -1;
            bool ok = true;
            for (int u = (int)pair; u < units && ok; u += pairs) {
                const int b = u / upb;
                if (P.resident) {
                    if (b == prev_b) continue;  // this batch's tiles are in place
                    if (prev_b >= 0) ++ep;
                    prev_b = b;
                }
                for (int kt = 0; kt < P.ktiles; ++kt, ++it_c) {
                    const uint32_t cs = P.resident ? (uint32_t)kt : it_c % kCStages;
                    const uint32_t epar = P.resident ? (ep & 1) ^ 1 : ((it_c / kCStages) & 1) ^ 1;
                    if (!(ok = mbar_wait(bar_c_empty + 8 * cs, epar, abort_flag, P.fault)))
                        break;
                    if (rank == 0) mbar_expect_tx(bar_c_full + 8 * cs, c_bytes_pair);
                    const uint32_t cfull_leader = map_to_rank(bar_c_full + 8 * cs, 0);
                    const int k0 = kt * kTileK + (int)rank * kHalfTile;
                    const uint32_t stage = c_base + cs * kCStageBytes;
                    for (int kb = 0; kb < boxes; ++kb)
                        tma_load_pair(stage + kb * kCBoxBytes, &tmap_c, kb * kBoxK, k0, b, cfull_leader);
                    tma_load_pair(stage + kMaxBoxes * kCBoxBytes, &tmap_e, 0, k0, b, cfull_leader);
                }
            }
        }
    } else if (warp == 1 || warp == kMmaWarpB) {
        // ------------------------------ MMA issuers (leader CTA) ------------------------------
        // One thread issues at most about one tcgen05.mma per ~100 cycles, so
        // two threads on different SMSPs share the work: issuer A takes the
        // even tiles (accumulator set 0), issuer B the odd ones (set 1).  Each
        // C stage is only ever used by one of them (4 stages, 2 issuers).
        const uint32_t mine = warp == 1 ? 0u : 1u;
        if (rank == 0 && lane == 0) {
            uint32_t it_x = 0, it_c = 0, it_a = 0, ep = 0;
            bool ok = true;
            // 32-bit unit counters (< 2^23), and unit u's batch b and index r in it
            // carried along as u advances: no division between two units' MMAs
            const int units = (int)n_units, pairs = (int)P.pairs, upb = (int)P.units_per_batch;
            int b = (int)pair / upb, r = (int)pair % upb;
            for (int u = (int)pair; u < units && ok; u += pairs, ++it_x) {
                int nb = b, nr = r + pairs;  // the next unit's batch and index
                if (nr >= upb) {
                    nb += nr / upb;
                    nr %= upb;
                }
                const uint32_t xb = it_x % kXBufs;
                // resident mode: the stages are released only after the epoch's last unit
                // (with an even tile count each stage has one issuer, whose commit covers
                // all of its earlier MMAs on that stage)
                const bool release_c = !P.resident || u + pairs >= units || nb != b;
                if (!(ok = mbar_wait(bar_x_full + 8 * xb, (it_x / kXBufs) & 1, abort_flag, P.fault))) break;
                const uint64_t a_desc0 = umma_desc_sw128(x_base + xb * kMaxBoxes * kBoxBytes);
                for (int kt = 0; kt < P.ktiles; ++kt, ++it_c, ++it_a) {
                    if ((it_a & 1u) != mine) continue;
                    const uint32_t cs = P.resident ? (uint32_t)kt : it_c % kCStages;
                    const uint32_t s = it_a % kAccSets;
                    const uint32_t fpar = P.resident ? (ep & 1) : (it_c / kCStages) & 1;
                    if (!(ok = mbar_wait(bar_c_full + 8 * cs, fpar, abort_flag, P.fault))) break;
                    if (!(ok = mbar_wait(bar_acc_empty + 8 * s, ((it_a / kAccSets) & 1) ^ 1, abort_flag, P.fault)))
                        break;
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + s * kTileK;
                    const uint32_t stage = c_base + cs * kCStageBytes;
                    const uint64_t b_desc0 = umma_desc_sw128(stage);
                    // unrolled, so that each step's descriptor offsets are immediates: one
                    // thread issues a tcgen05.mma only about every 100 cycles at best
#pragma unroll
                    for (int ks = 0; ks < kMaxKSteps; ++ks) {
                        if (ks < P.ksteps) {
                            // start-address field advance (16-byte units): box, then 32 bytes per K=16 step
                            const uint64_t a_off = (uint64_t)(((ks >> 2) * kBoxBytes + (ks & 3) * 32) >> 4);
                            const uint64_t b_off = (uint64_t)(((ks >> 2) * kCBoxBytes + (ks & 3) * 32) >> 4);
                            umma_pair_f16(d_tmem, a_desc0 + a_off, b_desc0 + b_off, ks > 0 ? 1u : 0u);
                        }
                    }
                    // the norm slice: ones (points) x (-||c||^2/2 pieces) (centroids)
                    umma_pair_f16(d_tmem, umma_desc_sw32(ones_base), umma_desc_sw32(stage + kMaxBoxes * kCBoxBytes),
                                  1u);
                    if (release_c) umma_commit_pair(bar_c_empty + 8 * cs);
                    umma_commit_pair(bar_acc_full + 8 * s);
                    if (kt == 0 && !P.xnorm_in) umma_commit_pair(bar_x_used + 8 * xb);  // the unit's X tile is in place
                }
                if (ok) umma_commit_pair(bar_x_empty + 8 * xb);
                if (P.resident && nb != b) ++ep;  // the next unit starts a new epoch
                b = nb;
                r = nr;
            }
        }
    } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kEpiWarps) {
        // ------------------------------ epilogue (both CTAs) ------------------------------
        // Per tile: read this warp's 128 columns, hand the accumulator back,
        // reduce.  Per unit only the (score, label) of this half is posted to
        // the merge warp, so nothing but tile work sits between two releases.
        const int e = warp - kEpiWarp0;
        const int q = warp % 4;   // TMEM lane quarter this warp may access
        const int h = e / 4;      // which 128-column slice of each 256-column tile
        const int row = q * 32 + lane;
        const uint32_t acc_empty_leader0 = map_to_rank(bar_acc_empty, 0);
        uint32_t it_x = 0, it_a = 0;
        bool ok = true;
        const int units = (int)n_units, pairs = (int)P.pairs;  // < 2^23: 32-bit counters
        for (int u = (int)pair; u < units && ok; u += pairs, ++it_x) {
            float best = -INFINITY, second = -INFINITY;
            int label = -1;    // column of the running best
            for (int kt = 0; kt < P.ktiles; ++kt, ++it_a) {
                const uint32_t s = it_a % kAccSets;
                if (!(ok = mbar_wait(bar_acc_full + 8 * s, (it_a / kAccSets) & 1, abort_flag, P.fault))) break;
                __syncwarp();  // tcgen05.ld below is warp-collective
                tc_fence_after();
                const uint32_t tcol = tmem_base + ((uint32_t)(q * 32) << 16) + s * kTileK + h * kPartCols;
                if constexpr (kDense) {
                    // this warp's 128 columns in one load, the accumulator handed back at once
                    float v[kPartCols];
                    tmem_ld128(tcol, v);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(acc_empty_leader0 + 8 * s);
                    const int upb = (int)P.units_per_batch;
                    const int b = u / upb;
                    const int n = (u - b * upb) * kUnitRows + (int)rank * kRows + row;
                    if (n < P.N) {
                        // [B, K', N]: a warp's 32 consecutive points of one column are one 128-byte line
                        float* out = P.dense + ((int64_t)b * P.ktiles * kTileK + kt * kTileK + h * kPartCols) * P.N + n;
#pragma unroll
                        for (int j = 0; j < kPartCols; ++j) out[(int64_t)j * P.N] = v[j];
                    }
                } else {
                    // this warp's 128 columns in one load; the accumulator is handed
                    // back as soon as they are in registers, and reduced after
                    float v[kPartCols];
                    tmem_ld128(tcol, v);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(acc_empty_leader0 + 8 * s);
                    top2_slice128(v, kt * kTileK + h * kPartCols, best, second, label);
                }
            }
            if (!ok) break;
            // post this half's result (the dense mode posts only the arrival)
            const uint32_t ms = it_x & 1, mph = (it_x >> 1) & 1;
            if (!(ok = mbar_wait(bar_m_empty + 8 * ms, mph ^ 1, abort_flag, P.fault))) break;
            if constexpr (!kDense) {
                const int slot = ((int)ms * kColParts + h) * kRows + row;
                merge_score[slot] = best;
                merge_second[slot] = second;
                merge_label[slot] = label;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_m_full + 8 * ms);
        }
    } else if (warp == kMergeWarp) {
        // ------------------------------ merge warp (both CTAs) ------------------------------
        // ||x||^2 of each row from the staged tile (the swizzle permutes
        // 16-byte chunks within a 128-byte row, so each row's bytes are all in
        // that row), then, once every epilogue warp has posted unit u, the
        // column slices joined (larger score, then the lower index; slice 0
        // holds the lower columns), the labels, mindist and the objective.
        uint32_t it_x = 0;
        bool ok = true;
        const int units = (int)n_units, pairs = (int)P.pairs;
        const int upb = (int)P.units_per_batch;
        for (int u = (int)pair; u < units && ok; u += pairs, ++it_x) {
            const uint32_t xb = it_x % kXBufs;
            const uint32_t ms = it_x & 1, mph = (it_x >> 1) & 1;
            const int b = u / upb;
            const int n0 = (u - b * upb) * kUnitRows + (int)rank * kRows;
            float cmax2 = 0.f;  // the batch's norm bound, loaded while the unit runs
            if constexpr (!kDense) cmax2 = P.list.cmax[b];
            float xn[kRows / 32];
            if (P.xnorm_in) {
                // given: loaded now, used at the unit's end (the X buffer is the issuers' alone)
#pragma unroll
                for (int rq = 0; rq < kRows / 32; ++rq) {
                    const int n = n0 + rq * 32 + lane;
                    xn[rq] = n < P.N ? P.xnorm_in[(int64_t)b * P.N + n] : 0.f;
                }
            } else {
                // ||x||^2 as soon as the unit's first tile of MMAs has completed
                // (its X tile is then in place in both CTAs); the X buffer is
                // released right after, while the unit's other tiles run
                if (!(ok = mbar_wait(bar_x_used + 8 * xb, (it_x / kXBufs) & 1, abort_flag, P.fault))) break;
#pragma unroll
                for (int rq = 0; rq < kRows / 32; ++rq) {
                    const int r = rq * 32 + lane;
                    float xnorm = 0.f;
                    for (int kb = 0; kb < boxes; ++kb)
                        xnorm = add_sq_row_sw128_f16(smem + kXOff + (xb * kMaxBoxes + kb) * kBoxBytes + r * 128, lane,
                                                     xnorm);
                    xn[rq] = xnorm;
                    if (P.xnorm && n0 + r < P.N) P.xnorm[(int64_t)b * P.N + n0 + r] = xnorm;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_x_empty + 8 * xb);
            }
            // the unit's results, once every epilogue warp has posted its column slice
            if (!(ok = mbar_wait(bar_m_full + 8 * ms, mph, abort_flag, P.fault))) break;
            float obj = 0.f;  // the unit's certified rows' share of the objective
            if constexpr (!kDense) {
                float fb[kRows / 32], fs[kRows / 32];
                int fl[kRows / 32];
#pragma unroll
                for (int rq = 0; rq < kRows / 32; ++rq) {
                    const int r = rq * 32 + lane;
                    const int s0 = ((int)ms * kColParts) * kRows + r;
                    fb[rq] = merge_score[s0];
                    fs[rq] = merge_second[s0];
                    fl[rq] = merge_label[s0];
#pragma unroll
                    for (int part = 1; part < kColParts; ++part) {  // slice 0 holds the lower columns
                        const int slot = ((int)ms * kColParts + part) * kRows + r;
                        top2_join(fb[rq], fs[rq], fl[rq], merge_score[slot], merge_second[slot], merge_label[slot]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_m_empty + 8 * ms);  // the slot is read: the epilogue may refill it
#pragma unroll
                for (int rq = 0; rq < kRows / 32; ++rq) {
                    const int n = n0 + rq * 32 + lane;
                    obj += certify_top2(P.list, cmax2, b, P.N, n, n < P.N, fb[rq], fs[rq], fl[rq], xn[rq], P.labels,
                                        P.mindist, lane);
                }
            } else {
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_m_empty + 8 * ms);
            }
            if (!kDense && P.obj_acc) {  // the objective of the unit's certified rows, one atomic
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) obj += __shfl_xor_sync(0xffffffffu, obj, o);
                if (lane == 0) atomicAdd(P.obj_acc + b, (double)obj);
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

// ---- host side ------------------------------------------------------------------
}  // namespace

bool assign_tc_supported(int64_t d, int dtype) { return dtype == KM_F16 && d >= 64 && d <= 128 && d % 8 == 0; }

template <bool kDense>
cudaError_t launch_tc(const __half* X, const __half* chat, const __half* cext, int64_t B, int64_t N, int64_t K,
                      int64_t d, int32_t* labels, float* mindist, double* obj_acc, const RescanList& list, float* dense,
                      float* xnorm, const float* xnorm_in, int sms, cudaStream_t st, const int32_t* stop) {
    if (!assign_tc_supported(d, KM_F16)) return cudaErrorNotSupported;
    CUtensorMap mx, mc, me;
    if (!make_map(&mx, X, 2, B, N, d, kBoxK, kRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mc, chat, 2, B, K, d, kBoxK, kHalfTile, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&me, cext, 2, B, padded_k(K), 16, 16, kHalfTile, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    cudaError_t e =
        cudaFuncSetAttribute(assign_tc_kernel<kDense>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    Params P;
    P.B = B; P.N = N; P.K = K; P.d = d;
    P.units_per_batch = ceil_div(N, kUnitRows);
    P.units = B * P.units_per_batch;
    if (P.units >= (int64_t(1) << 30)) return cudaErrorInvalidValue;  // the kernel counts units in 32 bits
    P.ktiles = (int)ceil_div(K, kTileK);
    P.ksteps = (int)ceil_div(d, 16);
    P.boxes = (int)ceil_div(d, kBoxK);
    P.resident = (P.ktiles % 2 == 0 && P.ktiles <= kCStages) ? 1 : 0;
    P.labels = labels;
    P.mindist = mindist;
    P.obj_acc = obj_acc;
    P.dense = dense;
    P.xnorm = xnorm;
    P.xnorm_in = xnorm_in;
    P.stop = stop;
    P.fault = fault_word();
    P.list = list;
    static std::atomic<int> pair_cache[kMaxDevices];  // per instantiation
    const int max_pairs = co_resident_pairs((const void*)assign_tc_kernel<kDense>, kThreads, kSmemBytes, sms, pair_cache);
    P.pairs = P.units < max_pairs ? P.units : max_pairs;
    return launch_kernel(assign_tc_kernel<kDense>, dim3((unsigned)(2 * P.pairs)), dim3(kThreads), kSmemBytes, st, mx,
                         mc, me, P);
}

cudaError_t launch_assign_tc(const __half* X, const __half* chat, const __half* cext, int64_t B, int64_t N, int64_t K,
                             int64_t d, int32_t* labels, float* mindist, double* obj_acc, const RescanList& list,
                             int sms, cudaStream_t st, const int32_t* stop, const float* xnorm_in, float* xnorm_out) {
    if (!list.cmax || !list.count || !list.rows) return cudaErrorInvalidValue;
    return launch_tc<false>(X, chat, cext, B, N, K, d, labels, mindist, obj_acc, list, nullptr, xnorm_out, xnorm_in,
                            sms, st, stop);
}

cudaError_t launch_assign_tc_dense(const __half* X, const __half* chat, const __half* cext, int64_t B, int64_t N,
                                   int64_t K, int64_t d, float* dense, float* xnorm, int sms, cudaStream_t st) {
    return launch_tc<true>(X, chat, cext, B, N, K, d, nullptr, nullptr, nullptr, RescanList(), dense, xnorm, nullptr,
                           sms, st, nullptr);
}

}  // namespace km
