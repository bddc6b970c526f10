// Device argsort of the 1-D label vector, the first half of Sort-Inverse
// Update (papernotes.org "Flash-KMeans" page, 关键设计 2: only the labels are
// sorted -- a radix sort giving sorted_idx and the sorted labels -- and the
// point matrix X is never moved).
//
// Stable least-significant-digit radix sort, batched over B (grid.y), with
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

}  // namespace

int sort_kernel_launches(int64_t N, int64_t K, bool with_counts, bool bounds) {
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
