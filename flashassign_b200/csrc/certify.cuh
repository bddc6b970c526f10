// Certification of the labels of the fp16 tensor-core assignment kernels.
//
// The kernels keep, per point, the best score s = x.c - ||c||^2/2 (the
// nearest centroid of papernotes.org "Flash-KMeans" 关键设计 1; lowest index
// on equal scores, the page's strict-improvement recurrence).  Every score
// carries a rounding error of at most e (fp16_score_err), so a label is only
// as good as the gap between the best score and the others -- which, near the
// origin, is large against e, but far from it (||x||^2 and ||c||^2 dwarfing
// the distances) may not be.  The kernels also keep the second-best score,
// and a label is certified when
//   * best - second > 2e: no two scores can be in the wrong order, so the
//     label is the exact argmin; or
//   * the computed distance of the second best, d2 = ||x||^2 - 2 second, is
//     above (4 / tau + 2) e + (the error of ||x||^2): a label other than the
//     exact argmin o is at most 4e farther from the point than o, the exact
//     second-smallest distance then exceeds 4e / tau, the exact relative
//     top-2 gap of such a point is below tau, and the label is within tau d2
//     of the smallest distance -- exact up to the label tolerance.
// The second test alone, made from the best score (d1 in place of d2), would
// spare the second-best score but not cover a point lying on the centroid of
// a one-member cluster (d1 = 0), which Lloyd iterations keep producing.  The
// points neither test covers
// (near ties, data far from the origin, norms beyond the folded term's range,
// where the bound is +inf) are listed for the exact re-scan on the CUDA cores
// (rescan.cu).
#pragma once

#include "km_internal.cuh"

namespace km {

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// The best, the second-best (with multiplicity) and the index of the best of
// one group of 32 scores w[0..31] of this lane's row, without branches.
//
// The group is read as a 4 x 8 grid (row r = w[8r .. 8r+7], column c =
// w[c], w[8+c], w[16+c], w[24+c]).  Any element other than the maximum lies
// in another grid row or another grid column than the maximum, so the
// group's second-best value (with multiplicity: equal to the best when the
// best occurs twice) is the larger of the second-largest row maximum and the
// second-largest column maximum -- 12 maxima of 32 values instead of a scan.
// The index is the lowest grid row and lowest grid column that reach the
// maximum: the maximum's column when it occurs once (a repeated maximum has
// g2 == g1, and the caller resolves it to its first column).
__device__ __forceinline__ void group_top2(const float* w, float& g1, float& g2, int& gi) {
    float R[4], M[8];
#pragma unroll
    for (int r = 0; r < 4; ++r)
        R[r] = fmax3(fmax3(w[8 * r], w[8 * r + 1], w[8 * r + 2]), fmax3(w[8 * r + 3], w[8 * r + 4], w[8 * r + 5]),
                     fmaxf(w[8 * r + 6], w[8 * r + 7]));
#pragma unroll
    for (int c = 0; c < 8; ++c) M[c] = fmax3(w[c], w[8 + c], fmaxf(w[16 + c], w[24 + c]));
    const float ra = fmaxf(R[0], R[1]), rb = fmaxf(R[2], R[3]);
    g1 = fmaxf(ra, rb);
    const float r2 = fmax3(fminf(ra, rb), fminf(R[0], R[1]), fminf(R[2], R[3]));
    const float ca = fmaxf(M[0], M[1]), cb = fmaxf(M[2], M[3]), cc = fmaxf(M[4], M[5]), cd = fmaxf(M[6], M[7]);
    const float sab = fmax3(fminf(ca, cb), fminf(M[0], M[1]), fminf(M[2], M[3]));
    const float scd = fmax3(fminf(cc, cd), fminf(M[4], M[5]), fminf(M[6], M[7]));
    g2 = fmaxf(r2, fmax3(fminf(fmaxf(ca, cb), fmaxf(cc, cd)), sab, scd));
    int rs = 3, cs = 7;
    rs = R[2] == g1 ? 2 : rs;
    rs = R[1] == g1 ? 1 : rs;
    rs = R[0] == g1 ? 0 : rs;
#pragma unroll
    for (int c = 6; c >= 0; --c) cs = M[c] == g1 ? c : cs;
    gi = 8 * rs + cs;
}

// A tile slice of kGroups * 32 scores v[] (columns col0 ...) folded into the
// running (best, second, label): every group's (best, second, index) first,
// with no branch between them, then the groups in ascending order (strict
// improvement: an earlier group keeps an equal score).
template <int kGroups>
__device__ __forceinline__ void top2_tile(const float* v, int col0, float& best, float& second, int& label) {
    float g1[kGroups], g2[kGroups];
    int gi[kGroups];
#pragma unroll
    for (int g = 0; g < kGroups; ++g) group_top2(v + 32 * g, g1[g], g2[g], gi[g]);
    // a maximum held by two columns of a group (duplicate centroids, exact ties): its first column
    bool tie = false;
#pragma unroll
    for (int g = 0; g < kGroups; ++g) tie = tie || (g2[g] == g1[g] && g1[g] > -INFINITY);
    if (__any_sync(0xffffffffu, tie)) {
#pragma unroll
        for (int g = 0; g < kGroups; ++g) {
            if (g2[g] == g1[g]) {
                const float* w = v + 32 * g;
                int j0 = 31;
#pragma unroll
                for (int j = 31; j >= 0; --j) j0 = (w[j] == g1[g]) ? j : j0;
                gi[g] = j0;
            }
        }
    }
#pragma unroll
    for (int g = 0; g < kGroups; ++g) {
        const bool better = g1[g] > best;
        label = better ? col0 + 32 * g + gi[g] : label;
        second = fmax3(fminf(best, g1[g]), second, g2[g]);
        best = fmaxf(best, g1[g]);
    }
}

// Joins two partial results of one row; (best, second, label) holds the lower
// columns and keeps an equal best score.
__device__ __forceinline__ void top2_join(float& best, float& second, int& label, float ob, float os, int ol) {
    second = fmax3(fminf(best, ob), second, os);
    if (ob > best) label = ol;
    best = fmaxf(best, ob);
}

// The outputs of one point (lane = row of the warp) once its best and
// second-best scores, label and ||x||^2 are final: a certified point gets its
// label and mindist = ||x||^2 - 2 best, and its mindist is returned as its
// share of the objective; the others are listed (one atomic per warp, every
// lane of the warp calling) and left to the re-scan, which writes all three;
// 0 is returned for them.  NaN or -inf scores are never certified.  cmax2:
// the batch's bound of max_k ||c_k||^2 (+inf: certify nothing); the error
// bound e is taken as err (||x||^2/2 + cmax^2) >= err (||x|| cmax + cmax^2/2),
// which needs no square root.
__device__ __forceinline__ double certify_top2(const RescanList& L, float cmax2, int64_t b, int64_t N, int64_t n,
                                               bool valid, float best, float second, int label, float xnorm,
                                               int32_t* __restrict__ labels, float* __restrict__ mindist, int lane) {
    const float e = L.err * fmaf(0.5f, xnorm, cmax2);  // >= err (||x|| cmax + cmax^2/2)
    const float d2 = fmaf(-2.f, second, xnorm);
    const bool certified = best - second > 2.f * e || d2 > fmaf(L.c_x, xnorm, L.c_c * cmax2);
    const bool listed = valid && !certified;
    const float md = fmaxf(fmaf(-2.f, best, xnorm), 0.f);
    if (valid && certified) {
        const int64_t o = b * N + n;
        labels[o] = label;
        if (mindist) mindist[o] = md;
    }
    const unsigned mask = __ballot_sync(0xffffffffu, listed);
    if (mask) {
        int base = 0;
        if (lane == 0) {
            base = atomicAdd(L.count + b, __popc(mask));
            if (L.total) atomicAdd(L.total, (unsigned long long)__popc(mask));
        }
        base = __shfl_sync(0xffffffffu, base, 0) + __popc(mask & ((1u << lane) - 1u));
        if (listed && base < L.cap) L.rows[b * L.cap + base] = (int32_t)n;
    }
    return (valid && certified) ? (double)md : 0.0;
}

}  // namespace km
