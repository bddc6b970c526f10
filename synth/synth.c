/*
 * Seeded synthetic inputs for the batched Lloyd iteration: Gaussian-mixture
 * points and random draws.  This file holds random-number generation only;
 * it computes nothing of the k-means method itself (no distances, no argmin,
 * no averaging), so that both the CPU oracle and the CUDA path can be fed the
 * same bytes without sharing any of the method's arithmetic.
 *
 * Generator: Philox4x32-10, the counter-based generator of Salmon, Moraes,
 * Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3" (SC'11).
 * Every value is a pure function of (key, counter), so any row range of any
 * batch can be regenerated on its own (needed for inputs streamed from host
 * memory in chunks).  Normal deviates use the Box-Muller transform.
 *
 * Counter layout: c0 = row (low 32 bits), c1 = row (high 32 bits),
 * c2 = (dim block | stream << 24), c3 = batch.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

enum { ST_CENTER = 1, ST_COMP = 2, ST_NOISE = 3, ST_UNIFORM = 4 };

void synth_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        uint64_t p0 = (uint64_t)PHILOX_M0 * c0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
        k0 += PHILOX_W0; k1 += PHILOX_W1;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

static inline void draw(uint64_t seed, int stream, int64_t batch, int64_t row, int64_t blk, uint32_t out[4]) {
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t ctr[4] = {(uint32_t)row, (uint32_t)((uint64_t)row >> 32),
                       (uint32_t)blk | ((uint32_t)stream << 24), (uint32_t)batch};
    synth_philox4x32_10(ctr, key, out);
}

/* uniform in (0, 1]: never 0, so log() below is finite */
static inline double u01_open0(uint32_t x) { return ((double)x + 1.0) * (1.0 / 4294967296.0); }
/* 53-bit uniform in [0, 1) from two words */
static inline double u53(uint32_t a, uint32_t b) {
    return ((double)(a >> 5) * 67108864.0 + (double)(b >> 6)) * (1.0 / 9007199254740992.0);
}

/* four standard normals from one Philox block (two Box-Muller pairs) */
static inline void normals4(const uint32_t r[4], double z[4]) {
    const double two_pi = 6.283185307179586476925286766559;
    for (int p = 0; p < 2; ++p) {
        double u1 = u01_open0(r[2 * p]);
        double u2 = (double)r[2 * p + 1] * (1.0 / 4294967296.0);
        double rad = sqrt(-2.0 * log(u1));
        z[2 * p] = rad * cos(two_pi * u2);
        z[2 * p + 1] = rad * sin(two_pi * u2);
    }
}

/* Standard normals for (batch, row, dims [0, d)) in a given stream. */
static void normal_row(uint64_t seed, int stream, int64_t b, int64_t row, int64_t d, double* z) {
    uint32_t r[4];
    double q[4];
    for (int64_t j = 0; j < d; j += 4) {
        draw(seed, stream, b, row, j / 4, r);
        normals4(r, q);
        for (int t = 0; t < 4 && j + t < d; ++t) z[j + t] = q[t];
    }
}

/* ---- public: raw uniforms, for init index selection on the Python side ---- */
void synth_uniform53(uint64_t seed, int64_t batch, int64_t n, double* out) {
    uint32_t r[4];
    for (int64_t i = 0; i < n; ++i) {
        draw(seed, ST_UNIFORM, batch, i, 0, r);
        out[i] = u53(r[0], r[1]);
    }
}

void synth_normal(uint64_t seed, int stream, int64_t batch, int64_t row0, int64_t nrows, int64_t d,
                  double* out) {
    for (int64_t i = 0; i < nrows; ++i) normal_row(seed, stream, batch, row0 + i, d, out + i * d);
}

/* ---- mixture generation ---- */
typedef struct {
    uint64_t seed;
    int64_t B, N, d, ncomp;
    int center_kind; /* 0: N(0,1) per coordinate; 1: uniform in [c_lo, c_hi) */
    double c_lo, c_hi, sigma;
    const double* cdf;     /* [ncomp] cumulative weights, last = 1 */
    const double* centers; /* [B, ncomp, d] */
    int64_t row0, nrows;
    int out_f16;
    void* out;          /* [B, nrows, d] */
    int32_t* comp_out;  /* [B, nrows] or NULL */
    int64_t t_begin, t_end; /* flattened (b, row) work range */
} mix_job;

static int64_t pick_comp(const double* cdf, int64_t ncomp, double u) {
    int64_t lo = 0, hi = ncomp - 1;
    while (lo < hi) {
        int64_t mid = (lo + hi) / 2;
        if (u < cdf[mid]) hi = mid; else lo = mid + 1;
    }
    return lo;
}

static void* mix_worker(void* arg) {
    mix_job* J = (mix_job*)arg;
    double* z = (double*)malloc(sizeof(double) * (size_t)(J->d + 4));
    uint32_t r[4];
    for (int64_t t = J->t_begin; t < J->t_end; ++t) {
        int64_t b = t / J->nrows, i = t % J->nrows, row = J->row0 + i;
        draw(J->seed, ST_COMP, b, row, 0, r);
        int64_t c = pick_comp(J->cdf, J->ncomp, u53(r[0], r[1]));
        normal_row(J->seed, ST_NOISE, b, row, J->d, z);
        const double* ctr = J->centers + ((size_t)b * J->ncomp + c) * J->d;
        if (J->comp_out) J->comp_out[t] = (int32_t)c;
        if (J->out_f16) {
            _Float16* o = (_Float16*)J->out + (size_t)t * J->d;
            for (int64_t j = 0; j < J->d; ++j) o[j] = (_Float16)(ctr[j] + J->sigma * z[j]);
        } else {
            float* o = (float*)J->out + (size_t)t * J->d;
            for (int64_t j = 0; j < J->d; ++j) o[j] = (float)(ctr[j] + J->sigma * z[j]);
        }
    }
    free(z);
    return NULL;
}

/*
 * Points of a Gaussian mixture, rows [row0, row0 + nrows) of every batch.
 * Component weights: equal when zipf_s == 0, else w_r proportional to r^-zipf_s
 * for r = 1..ncomp.  Component centres are drawn per batch (stream ST_CENTER,
 * row = component id), so they do not depend on which rows are generated.
 * Returns 0 on success, -1 on allocation failure.
 */
int synth_mixture(uint64_t seed, int64_t B, int64_t N, int64_t d, int64_t ncomp, int center_kind,
                  double c_lo, double c_hi, double sigma, double zipf_s, int64_t row0, int64_t nrows,
                  int out_f16, void* out, int32_t* comp_out, int nthreads) {
    (void)N;
    double* cdf = (double*)malloc(sizeof(double) * (size_t)ncomp);
    double* centers = (double*)malloc(sizeof(double) * (size_t)(B * ncomp * d + 4));
    if (!cdf || !centers) { free(cdf); free(centers); return -1; }
    double tot = 0.0;
    for (int64_t r = 0; r < ncomp; ++r) {
        tot += (zipf_s == 0.0) ? 1.0 : pow((double)(r + 1), -zipf_s);
        cdf[r] = tot;
    }
    for (int64_t r = 0; r < ncomp; ++r) cdf[r] /= tot;
    cdf[ncomp - 1] = 1.0;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t c = 0; c < ncomp; ++c) {
            double* ctr = centers + ((size_t)b * ncomp + c) * d;
            if (center_kind == 0) {
                normal_row(seed, ST_CENTER, b, c, d, ctr);
            } else {
                uint32_t r[4];
                for (int64_t j = 0; j < d; ++j) {
                    draw(seed, ST_CENTER, b, c, j, r);
                    ctr[j] = c_lo + (c_hi - c_lo) * u53(r[0], r[1]);
                }
            }
        }
    }
    if (nthreads < 1) nthreads = 1;
    int64_t total = B * nrows;
    if (nthreads > total) nthreads = (int)(total > 0 ? total : 1);
    mix_job* jobs = (mix_job*)calloc((size_t)nthreads, sizeof(mix_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int k = 0; k < nthreads; ++k) {
        mix_job* J = &jobs[k];
        J->seed = seed; J->B = B; J->N = N; J->d = d; J->ncomp = ncomp;
        J->center_kind = center_kind; J->c_lo = c_lo; J->c_hi = c_hi; J->sigma = sigma;
        J->cdf = cdf; J->centers = centers; J->row0 = row0; J->nrows = nrows;
        J->out_f16 = out_f16; J->out = out; J->comp_out = comp_out;
        J->t_begin = total * k / nthreads; J->t_end = total * (k + 1) / nthreads;
        pthread_create(&th[k], NULL, mix_worker, J);
    }
    for (int k = 0; k < nthreads; ++k) pthread_join(th[k], NULL);
    free(jobs); free(th); free(cdf); free(centers);
    return 0;
}
