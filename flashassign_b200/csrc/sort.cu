// Device argsort of the 1-D label vector, the first half of Sort-Inverse
// Update (papernotes.org "Flash-KMeans" page, 关键设计 2: only the labels are
// sorted -- a radix sort giving sorted_idx and the sorted labels -- and the
// point matrix X is never moved).
//
// Batches of at most 65,536 labels below 1024 are sorted by a single-launch
// counting sort (one thread-block cluster per batch, below).  Otherwise:
// a stable least-significant-digit radix sort, batched over B (grid.y), with
// digits of at most 8 bits: ceil(log2 K) bits in ceil(bits/8) passes (K=1024:
// two 5-bit passes; K=65536: two 8-bit passes).  Each pass is
//   1. a per-tile digit histogram (2048 keys per CTA),
//   2. an exclusive scan over (digit, tile) per batch (done by each scatter
//      CTA itself when the histogram is small),
//   3. a scatter in which each warp ranks its keys by ballots over the digit
//      bits (which lanes hold an equal digit), the warps of a tile are
//      combined by a per-digit scan (equal digits keep their input order:
//      stability), the tile is laid out digit by digit in shared memory, and
//      each digit's run is written to consecutive global positions.
// The segment offsets and counts then follow from the sorted labels without
// any atomics: position p starts label k exactly when a[p-1] < k <= a[p].
#include "km_internal.cuh"

#include <atomic>

namespace km {
namespace {

constexpr int kThreads = 256;
constexpr int kItems = 8;
constexpr int kTile = kThreads * kItems;  // 2048 keys per CTA
constexpr int kWarps = kThreads / 32;

struct Plan {
    int passes = 0;
    int shift[4] = {0, 0, 0, 0};
    int bits[4] = {0, 0, 0, 0};
    int64_t tiles = 0;
};

Plan make_plan(int64_t N, int64_t K) {
    int total = 1;
    while (total < 31 && (int64_t(1) << total) < K) ++total;
    Plan p;
    p.passes = (total + 7) / 8;
    const int per = (total + p.passes - 1) / p.passes;
    int shift = 0;
    for (int i = 0; i < p.passes; ++i) {
        p.shift[i] = shift;
        p.bits[i] = (total - shift < per) ? total - shift : per;
        shift += p.bits[i];
    }
    p.tiles = ceil_div(N, kTile);
    return p;
}

// A histogram of at most this many (digit, tile) entries per batch is summed
// by each scatter CTA itself instead of a separate scan pass.
bool small_hist(int bins, int64_t tiles) { return (int64_t)bins * tiles <= 8192; }

__global__ void __launch_bounds__(kThreads) radix_hist_kernel(const int32_t* __restrict__ keys, int64_t N, int shift,
                                                              int bits, int64_t T, int32_t* __restrict__ hist,
                                                              const int32_t* __restrict__ stop) {
    pdl_trigger();
    pdl_wait();
    if (stop && *stop) return;
    __shared__ int s[256];
    const int64_t b = blockIdx.y, tile = blockIdx.x;
    const int bins = 1 << bits, mask = bins - 1;
    for (int t = threadIdx.x; t < bins; t += kThreads) s[t] = 0;
    __syncthreads();
    const int32_t* kb = keys + b * N;
#pragma unroll
    for (int k = 0; k < kItems; ++k) {
        const int64_t i = tile * kTile + k * kThreads + threadIdx.x;
        if (i < N) atomicAdd(&s[(kb[i] >> shift) & mask], 1);
    }
    __syncthreads();
    for (int t = threadIdx.x; t < bins; t += kThreads) hist[(b * bins + t) * T + tile] = s[t];
}

// In-place exclusive scan of `len` ints per batch (one 1024-thread block per batch).
__global__ void __launch_bounds__(1024) exclusive_scan_kernel(int32_t* __restrict__ data, int64_t len,
                                                              const int32_t* __restrict__ stop) {
    pdl_trigger();
    pdl_wait();
    if (stop && *stop) return;
    __shared__ int warp_tot[32];
    __shared__ int carry_s;
    int32_t* p = data + (int64_t)blockIdx.x * len;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    if (threadIdx.x == 0) carry_s = 0;
    __syncthreads();
    for (int64_t base = 0; base < len; base += 1024) {
        const int64_t idx = base + threadIdx.x;
        const int v = idx < len ? p[idx] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) warp_tot[w] = incl;
        __syncthreads();
        if (w == 0) {
            int t = warp_tot[lane];
            int ti = t;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, ti, o);
                if (lane >= o) ti += y;
            }
            warp_tot[lane] = ti - t;  // exclusive prefix of the warp totals
        }
        __syncthreads();
        const int carry = carry_s;
        if (idx < len) p[idx] = carry + warp_tot[w] + incl - v;
        __syncthreads();
        if (threadIdx.x == 1023) carry_s = carry + warp_tot[w] + incl;
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kThreads) radix_scatter_kernel(const int32_t* __restrict__ keys_in,
                                                                 const int32_t* __restrict__ vals_in,
                                                                 int32_t* __restrict__ keys_out,
                                                                 int32_t* __restrict__ vals_out, int64_t N, int shift,
                                                                 int bits, int64_t T,
                                                                 const int32_t* __restrict__ offs,
                                                                 const int32_t* __restrict__ hist,
                                                                 const int32_t* __restrict__ stop) {
    pdl_trigger();
    pdl_wait();
    if (stop && *stop) return;
    __shared__ int wh[kWarps][256];      // per-warp digit counts, then per-warp exclusive offsets
    __shared__ int gstart[256];          // global first position of each digit of this tile (hist path)
    __shared__ int tstart[256];          // first tile-local position of each digit
    __shared__ int s_key[kTile];         // the tile's keys in tile-sorted (stable) order
    __shared__ int s_val[kTile];
    const int64_t b = blockIdx.y, tile = blockIdx.x;
    const int bins = 1 << bits, mask = bins - 1;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int t = threadIdx.x; t < kWarps * 256; t += kThreads) (&wh[0][0])[t] = 0;
    __syncthreads();

    // 1. rank each key among the equal digits before it (warp by warp, in input order)
    const uint32_t lt = (1u << lane) - 1u;
    const int64_t base = tile * kTile + (int64_t)w * (kItems * 32);
    int key[kItems], val[kItems], rank[kItems];
#pragma unroll
    for (int s = 0; s < kItems; ++s) {
        const int64_t i = base + s * 32 + lane;
        const bool valid = i < N;
        key[s] = valid ? keys_in[b * N + i] : 0;
        val[s] = valid ? (vals_in ? vals_in[b * N + i] : (int)i) : 0;
    }
#pragma unroll
    for (int s = 0; s < kItems; ++s) {
        const int64_t i = base + s * 32 + lane;
        const bool valid = i < N;
        const int dig = (key[s] >> shift) & mask;
        // the lanes holding the same digit: one ballot per digit bit
        uint32_t peers = __ballot_sync(0xffffffffu, valid);
#pragma unroll
        for (int bit = 0; bit < 8; ++bit) {
            if (bit < bits) {
                const bool on = (dig >> bit) & 1;
                const uint32_t bal = __ballot_sync(0xffffffffu, on);
                peers &= on ? bal : ~bal;
            }
        }
        const int cnt = valid ? wh[w][dig] : 0;
        rank[s] = cnt + __popc(peers & lt);
        __syncwarp();
        if (valid && lane == __ffs(peers) - 1) wh[w][dig] = cnt + __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    // 2. per digit: exclusive offsets across warps, and the digit's total in this tile
    int total = 0;
    if (threadIdx.x < bins) {
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) {
            const int t = wh[ww][threadIdx.x];
            wh[ww][threadIdx.x] = total;
            total += t;
        }
    }
    // 3. exclusive scan of the digit totals (bins <= 256 = kThreads): where each digit starts in the tile
    {
        __shared__ int warp_sum[kWarps];
        int incl = total;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) warp_sum[w] = incl;
        __syncthreads();
        int before = 0;
        for (int ww = 0; ww < w; ++ww) before += warp_sum[ww];
        if (threadIdx.x < bins) tstart[threadIdx.x] = before + incl - total;
    }
    __syncthreads();
    // 4. place the keys in tile-sorted order in shared memory
#pragma unroll
    for (int s = 0; s < kItems; ++s) {
        const int64_t i = base + s * 32 + lane;
        if (i < N) {
            const int dig = (key[s] >> shift) & mask;
            const int lp = tstart[dig] + wh[w][dig] + rank[s];
            s_key[lp] = key[s];
            s_val[lp] = val[s];
        }
    }
    __syncthreads();
    // 5. global start of each digit of this tile.  With a small histogram the
    //    CTA sums it itself (all earlier digits of the batch plus this digit's
    //    earlier tiles); otherwise the scanned offsets are read.
    if (hist) {
        // each warp sums digits w, w + 8, ...: its lanes load a digit's tiles
        // side by side (all loads of a warp independent), a warp reduction
        // gives the digit's total and its count in the tiles before this one
        __shared__ int wsum[kWarps];
        __shared__ int d_tot[256], d_mine[256];
        for (int d0 = w; d0 < bins; d0 += kWarps) {
            const int32_t* hd = hist + (b * bins + d0) * T;
            int tot_l = 0, mine_l = 0;
            for (int64_t t2 = lane; t2 < T; t2 += 32) {
                const int c = hd[t2];
                tot_l += c;
                mine_l += t2 < tile ? c : 0;
            }
            tot_l = __reduce_add_sync(0xffffffffu, tot_l);
            mine_l = __reduce_add_sync(0xffffffffu, mine_l);
            if (lane == 0) {
                d_tot[d0] = tot_l;
                d_mine[d0] = mine_l;
            }
        }
        __syncthreads();
        const int tot = threadIdx.x < bins ? d_tot[threadIdx.x] : 0;
        const int mine = threadIdx.x < bins ? d_mine[threadIdx.x] : 0;
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[w] = incl;
        __syncthreads();
        int before = 0;
        for (int ww = 0; ww < w; ++ww) before += wsum[ww];
        if (threadIdx.x < bins) gstart[threadIdx.x] = before + incl - tot + mine;
    } else if (threadIdx.x < bins) {
        gstart[threadIdx.x] = offs[(b * bins + threadIdx.x) * T + tile];
    }
    __syncthreads();
    // 6. write out: consecutive tile positions of one digit go to consecutive global positions
    const int n_here = (int)min((int64_t)kTile, N - tile * kTile);
    for (int lp = threadIdx.x; lp < n_here; lp += kThreads) {
        const int k = s_key[lp];
        const int dig = (k >> shift) & mask;
        const int64_t pos = (int64_t)gstart[dig] + (lp - tstart[dig]);
        keys_out[b * N + pos] = k;
        vals_out[b * N + pos] = s_val[lp];
    }
}

// offsets[b][k] = first sorted position holding a label >= k (offsets[b][K] = N).
__global__ void seg_bounds_kernel(const int32_t* __restrict__ a, int64_t N, int64_t K, int32_t* __restrict__ offsets) {
    pdl_trigger();
    pdl_wait();
    const int64_t b = blockIdx.y;
    const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (p > N) return;
    // clamped so that out-of-range labels cannot write outside offsets
    const int64_t prev = p == 0 ? -1 : min(max((int64_t)a[b * N + p - 1], (int64_t)-1), K);
    const int64_t cur = p == N ? K : min(max((int64_t)a[b * N + p], (int64_t)-1), K);
    for (int64_t k = prev + 1; k <= cur; ++k) offsets[b * (K + 1) + k] = (int32_t)p;
}

__global__ void counts_kernel(const int32_t* __restrict__ offsets, int64_t B, int64_t K, int32_t* __restrict__ counts) {
    pdl_trigger();
    pdl_wait();
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= B * K) return;
    const int64_t b = t / K, k = t % K;
    counts[t] = offsets[b * (K + 1) + k + 1] - offsets[b * (K + 1) + k];
}


// ---- single-launch counting sort of short batches ----------------------------
// For N <= kCsMaxN points per batch and labels of at most kCsMaxBits bits, one
// thread-block cluster of C = ceil(N / kCsTile) CTAs sorts one batch in a
// single launch, with the full label as the digit:
//   1. CTA r of the cluster takes keys [kCsTile r, kCsTile (r + 1)); each warp
//      ranks its keys among the equal labels before it (ballots over the label
//      bits, per-warp bin counters), a per-bin scan across the warps gives the
//      CTA's histogram and each warp's offset within a bin (stable order);
//   2. after a cluster barrier every CTA reads the C histograms through
//      distributed shared memory: a key of label k at CTA-local rank q goes to
//        (keys of the batch with labels < k) + (keys of label k in CTAs < r) + q;
//   3. the keys are laid out label by label in shared memory first, so the run
//      of each label that a CTA holds is written to consecutive positions.
// CTA 0 of each cluster also writes the segment offsets and the counts when
// they are asked for.  At 32 batches of 65,536 labels below 1024 this one
// launch replaces the radix sort's four (a histogram and a scatter per 5-bit
// pass, each mostly latency on 2^21 keys) and takes about half their time; it
// is bound by the issue of the ranking's ballots, not by memory.
constexpr int kCsThreads = 256;
constexpr int kCsWarps = kCsThreads / 32;
constexpr int kCsItems = 16;
constexpr int kCsTile = kCsThreads * kCsItems;  // 4096 keys per CTA
constexpr int kCsMaxCluster = 16;               // a non-portable cluster size on sm_100
constexpr int64_t kCsMaxN = (int64_t)kCsTile * kCsMaxCluster;
constexpr int kCsMaxBits = 10;
constexpr int kCsBins = 1 << kCsMaxBits;
static_assert(kCsBins == 4 * kCsThreads, "each thread owns four consecutive bins");
static_assert(kCsMaxN <= 65536, "point indices are staged as 16-bit values");
static_assert(kCsItems * 32 < 65536, "per-warp bin counters are 16-bit");

struct CsSmem {
    uint16_t wcnt[kCsWarps][kCsBins];  // per-warp bin counts, then each warp's offset within a bin
    int hist[kCsBins];                 // this CTA's bin counts (read by the whole cluster)
    int lstart[kCsBins];               // first CTA-local sorted position of a bin; then global minus local
    uint16_t din[kCsTile];             // the CTA's digits in input order, kOutOfRange if flagged
    uint16_t key[kCsTile];             // the same in CTA-sorted (stable) order
    uint16_t val[kCsTile];             // their point indices within the batch
    int wsum[2][kCsWarps];
};
// A label outside [0, 2^bits) is sorted by its low bits like any other and
// comes out as -1, which the update skips, as it skips every label outside [0, K).
constexpr uint32_t kOutOfRange = 0x8000u;

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
// Relaxed arrive: callers order their own memory accesses first (a fence, or
// having consumed the values they loaded).
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
// Four ints at the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ int4 ld_cluster_int4(const void* local, uint32_t rank) {
    const uint32_t a = (uint32_t)__cvta_generic_to_shared(local);
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    int4 v;
    asm volatile("ld.shared::cluster.v4.s32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(ra)
                 : "memory");
    return v;
}

// Exclusive scan over the CTA of the four consecutive values each thread holds
// (thread t: bins 4t .. 4t+3).  Contains a __syncthreads().
__device__ __forceinline__ int4 cs_exscan4(int4 x, int* wsum) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int s = x.x + x.y + x.z + x.w;
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[w] = incl;
    __syncthreads();
    int before = 0;
#pragma unroll
    for (int ww = 0; ww < kCsWarps; ++ww) before += ww < w ? wsum[ww] : 0;
    int4 e;
    e.x = before + incl - s;
    e.y = e.x + x.x;
    e.z = e.y + x.y;
    e.w = e.z + x.z;
    return e;
}

__global__ void __launch_bounds__(kCsThreads, 4)
    cluster_sort_kernel(const int32_t* __restrict__ keys_in, int64_t N, int64_t K, int bits,
                        int32_t* __restrict__ keys_out, int32_t* __restrict__ vals_out, int32_t* __restrict__ counts,
                        int32_t* __restrict__ offsets, const int32_t* __restrict__ stop) {
    pdl_trigger();
    extern __shared__ __align__(16) unsigned char cs_raw[];
    CsSmem& sm = *reinterpret_cast<CsSmem*>(cs_raw);
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const uint32_t mask = (1u << bits) - 1u;
    // the counters do not depend on the previous kernel: zero them before the wait
    for (int i = t; i < kCsWarps * kCsBins / 2; i += kCsThreads) reinterpret_cast<uint32_t*>(&sm.wcnt[0][0])[i] = 0u;
    __syncthreads();
    pdl_wait();
    // every CTA of the cluster reads the same flag, written before this grid started
    if (stop && *stop) return;
    const uint32_t r = cluster_rank(), C = cluster_size();
    const int64_t b = blockIdx.y;
    // N <= kCsMaxN: positions within a batch fit in 32 bits
    const int n = (int)N;
    const int base = (int)r * kCsTile + w * (kCsItems * 32);
    const int nw = max(0, min(kCsItems * 32, n - base));  // this warp's keys
    const int32_t* kb = keys_in + b * N;

    // 1a. the digits to shared memory in input order (din: digit | kOutOfRange);
    //     then per round of 32 keys, which lanes hold the same digit (one ballot
    //     per digit bit), with no shared-memory writes, so the rounds overlap.
    //     Per key, 16 bits of info: rank among the equal digits of its round
    //     (5 bits) | round leader (1 bit) | their number (6 bits).
    const uint32_t lt = (1u << lane) - 1u;
    uint16_t* din = sm.din + w * (kCsItems * 32) + lane;  // this lane's keys, a round apart
    uint32_t info[kCsItems / 2];
#pragma unroll
    for (int s = 0; s < kCsItems; ++s) {
        const int key = s * 32 + lane < nw ? kb[base + s * 32 + lane] : 0;
        din[s * 32] = (uint16_t)(((uint32_t)key & mask) | ((uint32_t)key > mask ? kOutOfRange : 0u));
    }
#pragma unroll
    for (int s = 0; s < kCsItems; ++s) {
        const bool valid = s * 32 + lane < nw;
        const uint32_t dig = din[s * 32] & mask;
        uint32_t peers = __ballot_sync(0xffffffffu, valid);
#pragma unroll
        for (int bit = 0; bit < kCsMaxBits; ++bit) {
            if (bit < bits) {
                const uint32_t on = (dig >> bit) & 1u;
                const uint32_t bal = __ballot_sync(0xffffffffu, on);
                peers &= ~(bal ^ (0u - on));  // keep the lanes whose bit equals mine
            }
        }
        const uint32_t i16 = (uint32_t)__popc(peers & lt) | ((uint32_t)(lane == __ffs(peers) - 1) << 5) |
                             ((uint32_t)__popc(peers) << 6);
        if (s % 2 == 0) info[s / 2] = i16;
        else info[s / 2] |= i16 << 16;
    }
    // 1b. in round order: add the counts of the earlier rounds (per-warp bin
    //     counters); info becomes the key's rank among the warp's equal digits.
#pragma unroll
    for (int s = 0; s < kCsItems; ++s) {
        const bool valid = s * 32 + lane < nw;
        const uint32_t sh = 16 * (s % 2);
        const uint32_t dig = din[s * 32] & mask;
        const uint32_t u = (info[s / 2] >> sh) & 0xffffu;
        const uint32_t cnt = valid ? sm.wcnt[w][dig] : 0u;
        __syncwarp();
        if (valid && (u & 32u)) sm.wcnt[w][dig] = (uint16_t)(cnt + (u >> 6));
        __syncwarp();
        info[s / 2] = (info[s / 2] & ~(0xffffu << sh)) | ((cnt + (u & 31u)) << sh);
    }
    __syncthreads();

    // 2. per bin: each warp's offset within the bin, and the CTA's histogram
    int4 h4;
    {
        int tot[4] = {0, 0, 0, 0};
#pragma unroll
        for (int ww = 0; ww < kCsWarps; ++ww) {
            uint2 packed = *reinterpret_cast<const uint2*>(&sm.wcnt[ww][4 * t]);
            const uint32_t c[4] = {packed.x & 0xffffu, packed.x >> 16, packed.y & 0xffffu, packed.y >> 16};
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                o[j] = (uint32_t)tot[j];
                tot[j] += (int)c[j];
            }
            packed.x = o[0] | (o[1] << 16);
            packed.y = o[2] | (o[3] << 16);
            *reinterpret_cast<uint2*>(&sm.wcnt[ww][4 * t]) = packed;
        }
        h4 = make_int4(tot[0], tot[1], tot[2], tot[3]);
        *reinterpret_cast<int4*>(&sm.hist[4 * t]) = h4;
    }
    // publish the histogram to the cluster: the block barrier orders every
    // thread's writes before one thread's cluster-scope fence, after which the
    // arrives need no release of their own
    __syncthreads();
    if (t == 0) asm volatile("fence.acq_rel.cluster;" ::: "memory");
    cluster_arrive_relaxed();
    const int4 l4 = cs_exscan4(h4, sm.wsum[0]);
    *reinterpret_cast<int4*>(&sm.lstart[4 * t]) = l4;
    __syncthreads();

    // 3. the keys in CTA-sorted order in shared memory
#pragma unroll
    for (int s = 0; s < kCsItems; ++s) {
        if (s * 32 + lane < nw) {
            const uint32_t sh = 16 * (s % 2);
            const uint32_t d16 = din[s * 32];
            const uint32_t dig = d16 & mask;
            const int lp = sm.lstart[dig] + sm.wcnt[w][dig] + (int)((info[s / 2] >> sh) & 0xffffu);
            sm.key[lp] = (uint16_t)d16;
            sm.val[lp] = (uint16_t)(base + s * 32 + lane);
        }
    }

    // 4. the cluster's histograms: keys of each bin in the whole batch and in the CTAs before this one
    cluster_wait();
    int4 tot4 = make_int4(0, 0, 0, 0), bef4 = make_int4(0, 0, 0, 0);
#pragma unroll
    for (uint32_t q = 0; q < kCsMaxCluster; ++q) {  // all remote loads in flight together
        if (q >= C) break;
        const int4 c = ld_cluster_int4(&sm.hist[4 * t], q);
        tot4.x += c.x;
        tot4.y += c.y;
        tot4.z += c.z;
        tot4.w += c.w;
        if (q < r) {
            bef4.x += c.x;
            bef4.y += c.y;
            bef4.z += c.z;
            bef4.w += c.w;
        }
    }
    const int4 g4 = cs_exscan4(tot4, sm.wsum[1]);  // first position of each label in the batch
    // the remote values are consumed (the scan used them): this CTA is done
    // with the other CTAs' shared memory
    cluster_arrive_relaxed();
    if (r == 0 && (counts || offsets)) {
        const int gs[4] = {g4.x, g4.y, g4.z, g4.w}, gt[4] = {tot4.x, tot4.y, tot4.z, tot4.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t k = 4 * t + j;
            if (k < K) {
                if (offsets) offsets[b * (K + 1) + k] = gs[j];
                if (counts) counts[b * K + k] = gt[j];
            }
        }
        if (offsets && t == 0) offsets[b * (K + 1) + K] = (int32_t)N;
    }
    // global position = CTA-local sorted position + (global start of this CTA's run - its local start)
    *reinterpret_cast<int4*>(&sm.lstart[4 * t]) =
        make_int4(g4.x + bef4.x - l4.x, g4.y + bef4.y - l4.y, g4.z + bef4.z - l4.z, g4.w + bef4.w - l4.w);
    __syncthreads();

    // 5. write out: each label's run of this CTA to consecutive global positions
    const int n_here = min(kCsTile, n - (int)r * kCsTile);
    int32_t* ko = keys_out + b * N;
    int32_t* vo = vals_out + b * N;
#pragma unroll 4
    for (int lp = t; lp < n_here; lp += kCsThreads) {
        const uint32_t d16 = sm.key[lp];
        const int pos = sm.lstart[d16 & mask] + lp;
        ko[pos] = (d16 & kOutOfRange) ? -1 : (int32_t)(d16 & mask);
        vo[pos] = (int32_t)sm.val[lp];
    }
    cluster_wait();  // no CTA leaves while another may still read its histogram
}

}  // namespace

// Whether the single-launch cluster sort takes this shape on the current
// device: short batches, labels of at most kCsMaxBits bits, and a cluster of
// kCsMaxCluster CTAs placeable at once (checked once per device).
bool use_cluster_sort(int64_t N, int64_t K) {
    if (N > kCsMaxN) return false;
    int total = 1;
    while (total < 31 && (int64_t(1) << total) < K) ++total;
    if (total > kCsMaxBits) return false;
    static std::atomic<int> state[64];  // per device: 0 not yet known, 1 usable, 2 not usable
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return false;
    }
    int st = state[dev].load(std::memory_order_acquire);
    if (st == 0) {
        bool ok = cudaFuncSetAttribute(cluster_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sizeof(CsSmem)) == cudaSuccess &&
                  cudaFuncSetAttribute(cluster_sort_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                      cudaSuccess;
        if (ok) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(kCsMaxCluster, 1, 1);
            cfg.blockDim = dim3(kCsThreads, 1, 1);
            cfg.dynamicSmemBytes = sizeof(CsSmem);
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = kCsMaxCluster;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int n = 0;
            ok = cudaOccupancyMaxActiveClusters(&n, cluster_sort_kernel, &cfg) == cudaSuccess && n >= 1;
        }
        if (!ok) cudaGetLastError();
        st = ok ? 1 : 2;
        state[dev].store(st, std::memory_order_release);
    }
    return st == 1;
}

int sort_kernel_launches(int64_t N, int64_t K, bool with_counts, bool bounds) {
    if (use_cluster_sort(N, K)) return 1;
    const Plan p = make_plan(N, K);
    int n = 0;
    for (int i = 0; i < p.passes; ++i) n += small_hist(1 << p.bits[i], p.tiles) ? 2 : 3;
    return n + (bounds ? 1 + (with_counts ? 1 : 0) : 0);
}

size_t sort_scratch_bytes(int64_t B, int64_t N, int64_t K) {
    const Plan p = make_plan(N, K);
    size_t bytes = 0;
    bytes += 2 * sizeof(int32_t) * (size_t)(B * N);     // ping-pong keys and values
    bytes += sizeof(int32_t) * (size_t)(B * 256 * p.tiles);  // tile histograms
    bytes += sizeof(int32_t) * (size_t)(B * (K + 1));   // offsets when the caller passes none
    return bytes;
}

cudaError_t launch_sort(const int32_t* labels, int64_t B, int64_t N, int64_t K, int32_t* a_sorted,
                        int32_t* sorted_idx, int32_t* counts, int32_t* offsets, void* scratch, cudaStream_t st,
                        bool bounds, const int32_t* stop) {
    if (use_cluster_sort(N, K)) {
        int total = 1;
        while (total < 31 && (int64_t(1) << total) < K) ++total;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)ceil_div(N, kCsTile), (unsigned)B, 1);
        cfg.blockDim = dim3(kCsThreads, 1, 1);
        cfg.dynamicSmemBytes = sizeof(CsSmem);
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = cfg.gridDim.x;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = pdl_enabled() ? 2 : 1;
        // offsets and counts only where the caller wants the bounds
        return cudaLaunchKernelEx(&cfg, cluster_sort_kernel, labels, N, K, total, a_sorted, sorted_idx,
                                  bounds ? counts : (int32_t*)nullptr, bounds ? offsets : (int32_t*)nullptr, stop);
    }
    const Plan p = make_plan(N, K);
    int32_t* tmp_k = (int32_t*)scratch;
    int32_t* tmp_v = tmp_k + B * N;
    int32_t* hist = tmp_v + B * N;
    int32_t* offs_scratch = hist + B * 256 * p.tiles;
    if (!offsets) offsets = offs_scratch;

    const int32_t* in_k = labels;
    const int32_t* in_v = nullptr;
    const dim3 grid((unsigned)p.tiles, (unsigned)B);
    for (int i = 0; i < p.passes; ++i) {
        const bool to_final = ((p.passes - 1 - i) % 2) == 0;
        int32_t* out_k = to_final ? a_sorted : tmp_k;
        int32_t* out_v = to_final ? sorted_idx : tmp_v;
        const int bins = 1 << p.bits[i];
        cudaError_t e = launch_kernel(radix_hist_kernel, grid, dim3(kThreads), 0, st, in_k, N, p.shift[i], p.bits[i],
                                      p.tiles, hist, stop);
        if (e != cudaSuccess) return e;
        if (small_hist(bins, p.tiles)) {
            e = launch_kernel(radix_scatter_kernel, grid, dim3(kThreads), 0, st, in_k, in_v, out_k, out_v, N,
                              p.shift[i], p.bits[i], p.tiles, (const int32_t*)nullptr, (const int32_t*)hist, stop);
        } else {
            e = launch_kernel(exclusive_scan_kernel, dim3((unsigned)B), dim3(1024), 0, st, hist,
                              (int64_t)bins * p.tiles, stop);
            if (e != cudaSuccess) return e;
            e = launch_kernel(radix_scatter_kernel, grid, dim3(kThreads), 0, st, in_k, in_v, out_k, out_v, N,
                              p.shift[i], p.bits[i], p.tiles, (const int32_t*)hist, (const int32_t*)nullptr, stop);
        }
        if (e != cudaSuccess) return e;
        in_k = out_k;
        in_v = out_v;
    }
    if (bounds) {
        cudaError_t e = launch_kernel(seg_bounds_kernel, dim3((unsigned)ceil_div(N + 1, 256), (unsigned)B), dim3(256),
                                      0, st, (const int32_t*)a_sorted, N, K, offsets);
        if (e != cudaSuccess || !counts) return e;
        return launch_kernel(counts_kernel, dim3((unsigned)ceil_div(B * K, 256)), dim3(256), 0, st,
                             (const int32_t*)offsets, B, K, counts);
    }
    return cudaSuccess;
}

}  // namespace km
