// Certification of the labels of the fp16 tensor-core assignment kernels.
//
// The kernels keep, per point, the best score s = x.c - ||c||^2/2 (the
// nearest centroid of papernotes.org "Flash-KMeans" 关键设计 1; lowest index
// on equal scores, the page's strict-improvement recurrence).  Every score
// carries a rounding error of at most e (fp16_score_err), so a label is only
// as good as the gap between the best score and the others -- which, near the
// origin, is large against e, but far from it (||x||^2 and ||c||^2 dwarfing
// the distances) may not be.  Two certificates:
//   * from the best score alone (the d <= 128 kernel, whose epilogue is the
//     kernel's limit): with d1 = ||x||^2 - 2 best (the computed smallest
//     distance), a label other than the exact argmin o is at most 4e farther
//     from the point than o, so if d1 > (4 / tau + 2) e + (the error of
//     ||x||^2), the exact second-smallest distance d2 >= d1 exceeds 4e / tau,
//     the exact relative top-2 gap (d2 - d1) / d2 of such a point is below
//     tau, and the label is within tau d2 of the smallest distance: exact up
//     to the label tolerance;
//   * from the best two scores (the wide and split-D kernels, whose epilogue
//     has time to spare behind their d/16 MMA steps per tile, and whose bound
//     e grows with d beyond what the first certificate can use): the label is
//     exact when best - second > 2e, and exact up to the tolerance when the
//     computed distance of the second best, ||x||^2 - 2 second, is above
//     (4 / tau + 2) e + (the error of ||x||^2) (the argument above with d2
//     bounded below directly).
// The points neither covers (near-duplicates of a centroid, data far from the
// origin, norms beyond the folded term's range, where the bound is +inf) are
// listed for the exact re-scan on the CUDA cores (rescan.cu).
#pragma once

#include "km_internal.cuh"

namespace km {

// certify_best: the outputs of one point (lane = row of the warp) once its best score,
// label and ||x||^2 are final, certified from the best score alone (the bound
// of the scores' error taken as err (||x||^2/2 + cmax^2) >= err (||x|| cmax +
// cmax^2/2), so that no square root is needed): a certified point gets its label and mindist =
// ||x||^2 - 2 best, and its mindist is returned as its share of the objective;
// the others are listed (one atomic per warp, every lane of the warp calling)
// and left to the re-scan, which writes all three; 0 is returned for them.
// NaN or -inf scores are never certified.  cmax2: the batch's bound of
// max_k ||c_k||^2 (+inf: certify nothing).
__device__ __forceinline__ double certify_best(const RescanList& L, float cmax2, int64_t b, int64_t N, int64_t n,
                                                    bool valid, float best, int label, float xnorm,
                                                    int32_t* __restrict__ labels, float* __restrict__ mindist,
                                                    int lane) {
    // e <= err (||x|| cmax + cmax^2/2) <= err (||x||^2/2 + cmax^2): no square roots
    const float d1 = fmaf(-2.f, best, xnorm);
    const bool certified = d1 > fmaf(L.c_x, xnorm, L.c_c * cmax2);
    const bool listed = valid && !certified;
    const float md = fmaxf(d1, 0.f);
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

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// One group of 32 consecutive scores w[0..31] of this lane's row (columns
// col0 .. col0+31) folded into the running (best, second, label).
//
// The group is read as a 4 x 8 grid (row r = w[8r .. 8r+7], column c =
// w[c], w[8+c], w[16+c], w[24+c]).  Any element other than the maximum lies
// in another grid row or another grid column than the maximum, so the
// group's second-best value (with multiplicity: equal to the best when the
// best occurs twice) is the larger of the second-largest row maximum and the
// second-largest column maximum -- 12 maxima of 32 values instead of a scan.
// The maximum's index (wanted only when it improves the running best in some
// lane of the warp) is the lowest grid row and lowest grid column that reach
// it; when the maximum is repeated (second == best) that pair need not be one
// of its columns, and the group is scanned for the first column holding it,
// so equal scores resolve to the lowest index as the strict recurrence does.
__device__ __forceinline__ void top2_group(const float* w, int col0, float& best, float& second, int& label) {
    float R[4], M[8];
#pragma unroll
    for (int r = 0; r < 4; ++r)
        R[r] = fmax3(fmax3(w[8 * r], w[8 * r + 1], w[8 * r + 2]), fmax3(w[8 * r + 3], w[8 * r + 4], w[8 * r + 5]),
                     fmaxf(w[8 * r + 6], w[8 * r + 7]));
#pragma unroll
    for (int c = 0; c < 8; ++c) M[c] = fmax3(w[c], w[8 + c], fmaxf(w[16 + c], w[24 + c]));
    // the largest and second-largest of the row maxima
    const float ra = fmaxf(R[0], R[1]), rb = fmaxf(R[2], R[3]);
    const float g1 = fmaxf(ra, rb);
    const float r2 = fmax3(fminf(ra, rb), fminf(R[0], R[1]), fminf(R[2], R[3]));
    // the second-largest of the column maxima
    const float ca = fmaxf(M[0], M[1]), cb = fmaxf(M[2], M[3]), cc = fmaxf(M[4], M[5]), cd = fmaxf(M[6], M[7]);
    const float sab = fmax3(fminf(ca, cb), fminf(M[0], M[1]), fminf(M[2], M[3]));
    const float scd = fmax3(fminf(cc, cd), fminf(M[4], M[5]), fminf(M[6], M[7]));
    const float c2 = fmax3(fminf(fmaxf(ca, cb), fmaxf(cc, cd)), sab, scd);
    const float g2 = fmaxf(r2, c2);
    const bool better = g1 > best;  // strict: an earlier group keeps an equal score
    if (__any_sync(0xffffffffu, better)) {
        int rs = 3, cs = 7;
        rs = R[2] == g1 ? 2 : rs;
        rs = R[1] == g1 ? 1 : rs;
        rs = R[0] == g1 ? 0 : rs;
#pragma unroll
        for (int c = 6; c >= 0; --c) cs = M[c] == g1 ? c : cs;
        if (better) label = col0 + 8 * rs + cs;
        // a maximum held by two columns (duplicate centroids, exact ties): its first column
        const bool tied = better && g2 == g1;
        if (__any_sync(0xffffffffu, tied)) {
            int j0 = 31;
#pragma unroll
            for (int j = 31; j >= 0; --j) j0 = (w[j] == g1) ? j : j0;
            if (tied) label = col0 + j0;
        }
    }
    second = fmax3(fminf(best, g1), second, g2);
    best = fmaxf(best, g1);
}

// Joins two partial results of one row; (best, second, label) holds the lower
// columns and keeps an equal best score.
__device__ __forceinline__ void top2_join(float& best, float& second, int& label, float ob, float os, int ol) {
    second = fmax3(fminf(best, ob), second, os);
    if (ob > best) label = ol;
    best = fmaxf(best, ob);
}

// certify_top2: as certify_best, from the best and second-best scores.
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
