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
//     of the smallest distance -- exact up to the label tolerance; a point
//     whose best two scores are equal is never certified this way (its
//     label would be a matter of index order, which the reductions leave to
//     the re-scan).
// The second test alone, made from the best score (d1 in place of d2), would
// spare the second-best score but not cover a point lying on the centroid of
// a one-member cluster (d1 = 0), which Lloyd iterations keep producing.  The
// points neither test covers
// (near and exact ties, data far from the origin, norms beyond the folded term's range,
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

__device__ __forceinline__ float fmax4(float a, float b, float c, float d) { return fmax3(a, b, fmaxf(c, d)); }

// The largest of w[0..15] in eight instructions.
__device__ __forceinline__ float max16(const float* w) {
    const float a = fmax3(w[0], w[1], w[2]), b = fmax3(w[3], w[4], w[5]), c = fmax3(w[6], w[7], w[8]);
    const float d = fmax3(w[9], w[10], w[11]), e = fmax3(w[12], w[13], w[14]);
    return fmaxf(fmax3(a, b, c), fmax3(d, e, w[15]));
}

// The second-largest of four values, with multiplicity (equal to the largest
// when it occurs twice): the smaller of the two pair maxima or the larger of
// the two pair minima.
__device__ __forceinline__ float second4(float a, float b, float c, float d) {
    return fmax3(fminf(fmaxf(a, b), fmaxf(c, d)), fminf(a, b), fminf(c, d));
}

// 1.0f where a == b, else 0.0f: the comparison's outcome as a number, so that
// the index below is summed on the FMA pipe rather than selected on the ALU
// pipe, which the reduction already fills.
__device__ __forceinline__ float eqf(float a, float b) {
    float r;
    asm("set.eq.f32.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// Top-2 of a 128-column slice of one row (scores v[0..127] of this lane's
// point), read as an 8 x 16 grid: grid row r = v[16r .. 16r+15], grid column
// c = v[c], v[16+c], ..., v[112+c].  Any score other than the maximum lies
// in another grid row or another grid column than the maximum, so the
// second-best score (with multiplicity) is the larger of the second-largest
// row maximum and the second-largest column maximum; the rows and columns
// cost about one instruction per score, and the two second-largest values
// are taken the same way on the 8 row maxima (a 2 x 4 grid) and the 16
// column maxima (a 4 x 4 grid).  When the maximum is unique, exactly one row
// maximum and one column maximum (and one of each at the next level) equal
// it, and their positions sum to its column; a repeated maximum leaves
// second == best, which the certificate never accepts, so such a point goes
// to the exact re-scan, which resolves the tie to the lowest index.
//
// grid_rows covers half of the grid, 64 scores (the first half: rows 0-3;
// the second: rows 4-7), so that a kernel can reduce one half while the other
// is still being loaded; grid_top2 then folds the slice (columns col0 ...)
// into the running (best, second, label) of the point, an earlier slice
// keeping an equal score.
template <bool kSecondHalf>
__device__ __forceinline__ void grid_rows(const float* v, float (&R)[8], float (&M)[16]) {
#pragma unroll
    for (int r = 0; r < 4; ++r) R[(kSecondHalf ? 4 : 0) + r] = max16(v + 16 * r);
#pragma unroll
    for (int c = 0; c < 16; ++c)
        M[c] = kSecondHalf ? fmax3(fmax3(M[c], v[c], v[16 + c]), v[32 + c], v[48 + c])
                           : fmax4(v[c], v[16 + c], v[32 + c], v[48 + c]);
}

__device__ __forceinline__ void grid_top2(const float (&R)[8], const float (&M)[16], int col0, float& best,
                                          float& second, int& label) {
    const float ra = fmax4(R[0], R[1], R[2], R[3]), rb = fmax4(R[4], R[5], R[6], R[7]);
    const float g1 = fmaxf(ra, rb);
    float Q[4], Nr[4], Nc[4];  // column maxima of the row maxima; row and column maxima of the column maxima
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        Q[i] = fmaxf(R[i], R[4 + i]);
        Nr[i] = fmax4(M[4 * i], M[4 * i + 1], M[4 * i + 2], M[4 * i + 3]);
        Nc[i] = fmax4(M[i], M[4 + i], M[8 + i], M[12 + i]);
    }
    const float g2 = fmax3(fminf(ra, rb), fmaxf(second4(Q[0], Q[1], Q[2], Q[3]), second4(Nr[0], Nr[1], Nr[2], Nr[3])),
                           second4(Nc[0], Nc[1], Nc[2], Nc[3]));
    // column of the maximum = 16 (4 [rb] + i[Q]) + 4 i[Nr] + i[Nc], summed from 2^23 so that its bits
    // are 0x4B000000 + the column
    float acc = fmaf(eqf(rb, g1), 64.f, 0x1p23f);
#pragma unroll
    for (int i = 1; i < 4; ++i) {
        acc = fmaf(eqf(Q[i], g1), 16.f * i, acc);
        acc = fmaf(eqf(Nr[i], g1), 4.f * i, acc);
        acc = fmaf(eqf(Nc[i], g1), (float)i, acc);
    }
    label = g1 > best ? __float_as_int(acc) + (col0 - 0x4B000000) : label;
    second = fmax3(fminf(best, g1), second, g2);
    best = fmaxf(best, g1);
}

// grid_rows and grid_top2 over a slice that is all in registers.
__device__ __forceinline__ void top2_slice128(const float* v, int col0, float& best, float& second, int& label) {
    float R[8], M[16];
    grid_rows<false>(v, R, M);
    grid_rows<true>(v + 64, R, M);
    grid_top2(R, M, col0, best, second, label);
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
// 0 is returned for them (the caller sums the shares in fp32 and adds the
// sum to the fp64 accumulator: fp64 arithmetic in the per-unit path measured
// ~13% of the iteration).  NaN or -inf scores are never certified.  cmax2:
// the batch's bound of max_k ||c_k||^2 (+inf: certify nothing); the error
// bound e is taken as err (||x||^2/2 + cmax^2) >= err (||x|| cmax + cmax^2/2),
// which needs no square root.
__device__ __forceinline__ float certify_top2(const RescanList& L, float cmax2, int64_t b, int64_t N, int64_t n,
                                               bool valid, float best, float second, int label, float xnorm,
                                               int32_t* __restrict__ labels, float* __restrict__ mindist, int lane) {
    const float e = L.err * fmaf(0.5f, xnorm, cmax2);  // >= err (||x|| cmax + cmax^2/2)
    const float d2 = fmaf(-2.f, second, xnorm);
    const bool certified = best - second > 2.f * e || (best > second && d2 > fmaf(L.c_x, xnorm, L.c_c * cmax2));
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
    return (valid && certified) ? md : 0.f;
}

}  // namespace km
