// CPU oracle for one batched exact Lloyd k-means iteration.
//
// TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
// baseline leg of the benchmark may load this library.  The product path (the
// CUDA library under flashassign_b200/) never calls it and shares no code,
// header or table with it.
//
// What it computes, and where the pages define it (Flash-KMeans pages):
//   * papernotes.org "Flash-KMeans: Fast and Memory-Efficient Exact K-Means",
//     section 方法详解 / 整体框架 and its flowchart: each iteration assigns every
//     point to its nearest centroid, then recomputes each centroid from its
//     members, and loops back to assignment.
//   * 7minutos.es (Spanish Marktechpost article), opening paragraphs: the
//     method is exactly Lloyd's k-means, with no approximation; the update
//     averages the points of each cluster.
//   * papernotes.org, 关键设计 1 (FlashAssign): running state per point starts
//     at (m = +inf, a = -1) and keeps the smaller distance; taken here as a
//     strict "<" over ascending centroid index, so ties go to the lowest index.
//   * papernotes.org, 关键设计 2 (Sort-Inverse Update): the labels are argsorted
//     and each cluster is a contiguous run [u, v) of the sorted order; the
//     cluster sum is the sum of the rows in that run.
// Readings where the pages are silent:
//   * an empty cluster keeps its previous centroid, bit for bit;
//   * the assignment sees the centroids rounded (round-to-nearest-even) to the
//     dtype of X, since the points are FP16 data and the distance is taken
//     between two FP16 vectors;
//   * the argsort is stable (ascending label, ties by ascending point index);
//   * labels are 0-based; centroids are stored as fp32 between iterations.
//
// Arithmetic is the plain definition in double precision: the squared
// distance is summed from direct differences (no norm expansion), sums are
// accumulated in sorted order, and the mean is s_k / n_k rounded to fp32.
// The binary16 codec is written from the IEEE-754 binary16 format definition.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

// ---- IEEE-754 binary16 -------------------------------------------------------
// Layout: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
double f16_decode(uint16_t h) {
    const int sign = h >> 15;
    const int e = (h >> 10) & 0x1F;
    const int m = h & 0x3FF;
    double v;
    if (e == 0) {
        v = std::ldexp(static_cast<double>(m), -24);  // subnormal: m * 2^-24
    } else if (e == 31) {
        v = m ? std::numeric_limits<double>::quiet_NaN() : std::numeric_limits<double>::infinity();
    } else {
        v = std::ldexp(static_cast<double>(1024 + m), e - 25);  // (1 + m/1024) * 2^(e-15)
    }
    return sign ? -v : v;
}

// Round a non-negative double holding a value below 2^53 to the nearest integer,
// ties to even.
double round_half_even(double q) {
    double fl = std::floor(q);
    double r = q - fl;  // exact
    if (r > 0.5) return fl + 1.0;
    if (r < 0.5) return fl;
    return (std::fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

uint16_t f16_encode(double x) {
    if (std::isnan(x)) return 0x7E00;
    const uint16_t sign = std::signbit(x) ? 0x8000 : 0;
    double ax = std::fabs(x);
    // Largest finite value 65504 = (2 - 2^-10) * 2^15; halfway to the next
    // step (2^16) is 65520, which rounds to even, i.e. overflows to infinity.
    if (ax >= 65520.0) return sign | 0x7C00;
    if (ax < std::ldexp(1.0, -14)) {
        // subnormal range: value = q * 2^-24 with integer q in [0, 1024]
        double q = round_half_even(ax * std::ldexp(1.0, 24));
        return sign | static_cast<uint16_t>(q);  // q == 1024 encodes the smallest normal
    }
    int ex;
    std::frexp(ax, &ex);  // ax = f * 2^ex, f in [0.5, 1)
    int E = ex - 1;       // ax in [2^E, 2^(E+1))
    double q = round_half_even(std::ldexp(ax, 10 - E));  // in [1024, 2048]
    if (q == 2048.0) { q = 1024.0; E += 1; }
    if (E + 15 >= 31) return sign | 0x7C00;
    return sign | static_cast<uint16_t>(((E + 15) << 10) | (static_cast<int>(q) - 1024));
}

// ---- helpers -----------------------------------------------------------------
void load_row(const void* X, int dtype, int64_t row, int64_t d, double* out) {
    if (dtype == 1) {
        const uint16_t* p = static_cast<const uint16_t*>(X) + row * d;
        for (int64_t j = 0; j < d; ++j) out[j] = f16_decode(p[j]);
    } else {
        const float* p = static_cast<const float*>(X) + row * d;
        for (int64_t j = 0; j < d; ++j) out[j] = static_cast<double>(p[j]);
    }
}

template <class F>
void parallel_for(int64_t n, int nthreads, F f) {
    if (nthreads < 1) nthreads = 1;
    if (n < nthreads) nthreads = static_cast<int>(n > 0 ? n : 1);
    if (nthreads == 1) { f(0, n); return; }
    std::vector<std::thread> th;
    for (int t = 0; t < nthreads; ++t) {
        int64_t lo = n * t / nthreads, hi = n * (t + 1) / nthreads;
        th.emplace_back([=]() { f(lo, hi); });
    }
    for (auto& x : th) x.join();
}

}  // namespace

extern "C" {

int oracle_hw_threads() { return static_cast<int>(std::thread::hardware_concurrency()); }

void oracle_f16_decode(const uint16_t* in, double* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = f16_decode(in[i]);
}

void oracle_f16_encode(const double* in, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = f16_encode(in[i]);
}

// The centroids as the assignment sees them: fp32 C rounded to the dtype of X
// (dtype 1 = fp16, RNE; dtype 0 = fp32, unchanged), returned exactly in double.
void oracle_round_centroids(const float* C, int dtype, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i)
        out[i] = (dtype == 1) ? f16_decode(f16_encode(static_cast<double>(C[i]))) : static_cast<double>(C[i]);
}

// Assignment step for a set of rows.  For row r of batch b (flattened index
// rows[t] = b * N + r, or every row when rows == nullptr):
//   labels[t] = argmin_k ||x - chat_k||^2 with the lowest k on ties,
//   d1[t] = that minimum, d2[t] = the second smallest (+inf when K == 1).
int oracle_assign(const void* X, int dtype, const double* Chat, int64_t B, int64_t N, int64_t K, int64_t d,
                  const int64_t* rows, int64_t nrows, int32_t* labels, double* d1, double* d2, int nthreads) {
    if (!X || !Chat || B < 1 || N < 1 || K < 1 || d < 1) return 1;
    const int64_t total = rows ? nrows : B * N;
    parallel_for(total, nthreads, [&](int64_t lo, int64_t hi) {
        std::vector<double> x(d);
        for (int64_t t = lo; t < hi; ++t) {
            const int64_t g = rows ? rows[t] : t;
            const int64_t b = g / N;
            load_row(X, dtype, g, d, x.data());
            double best = std::numeric_limits<double>::infinity();
            double second = std::numeric_limits<double>::infinity();
            int32_t a = -1;
            const double* cb = Chat + b * K * d;
            for (int64_t k = 0; k < K; ++k) {
                const double* c = cb + k * d;
                double dist = 0.0;
                for (int64_t j = 0; j < d; ++j) {
                    const double diff = x[j] - c[j];
                    dist += diff * diff;
                }
                if (dist < best) {
                    second = best;
                    best = dist;
                    a = static_cast<int32_t>(k);
                } else if (dist < second) {
                    second = dist;
                }
            }
            labels[t] = a;
            if (d1) d1[t] = best;
            if (d2) d2[t] = second;
        }
    });
    return 0;
}

// Stable argsort of the labels of each batch by counting: counts[b][k] = n_k,
// offsets[b][k] = sum_{j<k} n_j (K+1 entries), sorted_idx[b][p] = the point
// index at sorted position p (ascending label, then ascending point index).
int oracle_sort(const int32_t* labels, int64_t B, int64_t N, int64_t K, int32_t* sorted_idx, int32_t* counts,
                int32_t* offsets) {
    if (!labels || B < 1 || N < 1 || K < 1) return 1;
    std::vector<int64_t> cnt(K), next(K);
    for (int64_t b = 0; b < B; ++b) {
        const int32_t* a = labels + b * N;
        std::fill(cnt.begin(), cnt.end(), 0);
        for (int64_t i = 0; i < N; ++i) {
            if (a[i] < 0 || a[i] >= K) return 2;
            ++cnt[a[i]];
        }
        int64_t run = 0;
        for (int64_t k = 0; k < K; ++k) {
            if (counts) counts[b * K + k] = static_cast<int32_t>(cnt[k]);
            if (offsets) offsets[b * (K + 1) + k] = static_cast<int32_t>(run);
            next[k] = run;
            run += cnt[k];
        }
        if (offsets) offsets[b * (K + 1) + K] = static_cast<int32_t>(run);
        if (sorted_idx)
            for (int64_t i = 0; i < N; ++i) sorted_idx[b * N + next[a[i]]++] = static_cast<int32_t>(i);
    }
    return 0;
}

// Update step: for each cluster k with members (in stable sorted order),
// s_k = sum of member rows (double), C_out[k] = fp32(s_k / n_k); an empty
// cluster copies C_prev[k] bit for bit.  sums (double, nullable) receives s_k.
int oracle_update(const void* X, int dtype, const int32_t* labels, int64_t B, int64_t N, int64_t K, int64_t d,
                  const float* C_prev, float* C_out, double* sums, int32_t* counts_out, int nthreads) {
    if (!X || !labels || !C_prev || !C_out || B < 1 || N < 1 || K < 1 || d < 1) return 1;
    std::vector<int32_t> sidx(B * N), cnt(B * K), off(B * (K + 1));
    int rc = oracle_sort(labels, B, N, K, sidx.data(), cnt.data(), off.data());
    if (rc) return rc;
    parallel_for(B * K, nthreads, [&](int64_t lo, int64_t hi) {
        std::vector<double> s(d), x(d);
        for (int64_t t = lo; t < hi; ++t) {
            const int64_t b = t / K, k = t % K;
            const int64_t u = off[b * (K + 1) + k], v = off[b * (K + 1) + k + 1];
            std::fill(s.begin(), s.end(), 0.0);
            for (int64_t p = u; p < v; ++p) {
                load_row(X, dtype, b * N + sidx[b * N + p], d, x.data());
                for (int64_t j = 0; j < d; ++j) s[j] += x[j];
            }
            const int64_t n = v - u;
            if (sums)
                for (int64_t j = 0; j < d; ++j) sums[t * d + j] = s[j];
            if (n > 0) {
                for (int64_t j = 0; j < d; ++j) C_out[t * d + j] = static_cast<float>(s[j] / static_cast<double>(n));
            } else {
                std::memcpy(C_out + t * d, C_prev + t * d, sizeof(float) * d);
            }
        }
    });
    if (counts_out) std::memcpy(counts_out, cnt.data(), sizeof(int32_t) * B * K);
    return 0;
}

// Objective of a labelling against given centroids (double): per batch,
// J_b = sum_i ||x_i - C[a_i]||^2.
int oracle_cost(const void* X, int dtype, const double* C, const int32_t* labels, int64_t B, int64_t N, int64_t K,
                int64_t d, double* J) {
    if (!X || !C || !labels || !J) return 1;
    std::vector<double> x(d);
    for (int64_t b = 0; b < B; ++b) {
        double acc = 0.0;
        for (int64_t i = 0; i < N; ++i) {
            const int32_t a = labels[b * N + i];
            if (a < 0 || a >= K) return 2;
            load_row(X, dtype, b * N + i, d, x.data());
            const double* c = C + (b * K + a) * d;
            for (int64_t j = 0; j < d; ++j) {
                const double diff = x[j] - c[j];
                acc += diff * diff;
            }
        }
        J[b] = acc;
    }
    return 0;
}

// `iters` full Lloyd iterations from C_init.  labels: the last iteration's
// assignment (made against the centroids before the final update).
// objective[t * B + b] = sum of the assignment's minimum distances at iteration t.
int oracle_lloyd(const void* X, int dtype, const float* C_init, int64_t B, int64_t N, int64_t K, int64_t d,
                 int iters, int32_t* labels, float* C_out, double* objective, int nthreads) {
    if (!X || !C_init || !labels || !C_out || iters < 0) return 1;
    std::vector<float> C(C_init, C_init + B * K * d), Cn(B * K * d);
    std::vector<double> chat(B * K * d), d1(B * N);
    for (int t = 0; t < iters; ++t) {
        oracle_round_centroids(C.data(), dtype, B * K * d, chat.data());
        int rc = oracle_assign(X, dtype, chat.data(), B, N, K, d, nullptr, 0, labels, d1.data(), nullptr, nthreads);
        if (rc) return rc;
        if (objective)
            for (int64_t b = 0; b < B; ++b) {
                double j = 0.0;
                for (int64_t i = 0; i < N; ++i) j += d1[b * N + i];
                objective[t * B + b] = j;
            }
        rc = oracle_update(X, dtype, labels, B, N, K, d, C.data(), Cn.data(), nullptr, nullptr, nthreads);
        if (rc) return rc;
        C.swap(Cn);
    }
    std::memcpy(C_out, C.data(), sizeof(float) * B * K * d);
    return 0;
}

// Lloyd iterations until convergence (papernotes.org page, 整体框架 flowchart:
// after each update, "converged?" either ends the loop or returns to the
// assignment).  The pages give no test; the reading taken: after iteration t,
// every batch's squared centroid shift shift_b = sum_k ||C_{t+1,k} - C_{t,k}||^2
// (fp32 centroids, summed in double; an empty cluster keeps its centroid and
// so does not move) is compared with tol, and the loop ends after the first
// iteration at which shift_b <= tol holds for every batch, or after max_iters.
// *iters_run = the number of iterations performed; labels, C_out and the
// objective rows [0, *iters_run) are those of oracle_lloyd with that count;
// shift[t * B + b] (nullable, [max_iters, B]) = shift_b of iteration t.
int oracle_lloyd_tol(const void* X, int dtype, const float* C_init, int64_t B, int64_t N, int64_t K, int64_t d,
                     int max_iters, double tol, int32_t* labels, float* C_out, double* objective, int32_t* iters_run,
                     double* shift, int nthreads) {
    if (!X || !C_init || !labels || !C_out || !iters_run || max_iters < 1) return 1;
    std::vector<float> C(C_init, C_init + B * K * d), Cn(B * K * d);
    std::vector<double> chat(B * K * d), d1(B * N);
    int t = 0;
    bool settled = false;
    while (t < max_iters && !settled) {
        oracle_round_centroids(C.data(), dtype, B * K * d, chat.data());
        int rc = oracle_assign(X, dtype, chat.data(), B, N, K, d, nullptr, 0, labels, d1.data(), nullptr, nthreads);
        if (rc) return rc;
        if (objective)
            for (int64_t b = 0; b < B; ++b) {
                double j = 0.0;
                for (int64_t i = 0; i < N; ++i) j += d1[b * N + i];
                objective[t * B + b] = j;
            }
        rc = oracle_update(X, dtype, labels, B, N, K, d, C.data(), Cn.data(), nullptr, nullptr, nthreads);
        if (rc) return rc;
        settled = true;
        for (int64_t b = 0; b < B; ++b) {
            double sb = 0.0;
            for (int64_t e = b * K * d; e < (b + 1) * K * d; ++e) {
                const double diff = static_cast<double>(Cn[e]) - static_cast<double>(C[e]);
                sb += diff * diff;
            }
            if (shift) shift[t * B + b] = sb;
            if (!(sb <= tol)) settled = false;
        }
        C.swap(Cn);
        ++t;
    }
    *iters_run = t;
    std::memcpy(C_out, C.data(), sizeof(float) * B * K * d);
    return 0;
}

}  // extern "C"
