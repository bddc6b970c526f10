// The extern "C" entry points of libkm.so (declared in include/km.h):
// argument validation, stream-ordered scratch, and the composition of the
// kernels into the assignment, sort, update and full Lloyd iterations
// (papernotes.org "Flash-KMeans" page, 方法详解: 整体框架 and 关键设计 1-3).
#include "km_internal.cuh"

#include <algorithm>
#include <atomic>
#include <chrono>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <thread>
#include <vector>

namespace km {

namespace {
thread_local char g_err[512] = "";
__device__ int32_t g_fault;  // device fault word (see km_device_fault)
__device__ unsigned long long g_rescans;  // points handed to the exact re-scan (see km_assign_rescans)

bool inject(const char* what) {
    const char* f = std::getenv("KM_FAULT");
    return f && std::strcmp(f, what) == 0;
}

// The library's stream-ordered memory pool on the current device, created on
// first use.  Unlike the device's default pool it keeps the memory freed into
// it (release threshold: unlimited), so a call does not map and unmap its
// scratch every time; km_release_cached() returns it to the device.
std::mutex g_pool_mu;
cudaMemPool_t g_pool[64] = {nullptr};

cudaError_t scratch_pool(cudaMemPool_t* out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_pool_mu);
    if (!g_pool[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.handleTypes = cudaMemHandleTypeNone;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        if ((e = cudaMemPoolCreate(&pool, &props)) != cudaSuccess) return e;
        uint64_t keep = ~uint64_t(0);
        if ((e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep)) != cudaSuccess) {
            cudaMemPoolDestroy(pool);
            return e;
        }
        g_pool[dev] = pool;
    }
    *out = g_pool[dev];
    return cudaSuccess;
}

// Scratch taken stream-ordered from the library's pool on one stream, released
// (to the pool) on scope exit.
class Scratch {
  public:
    explicit Scratch(cudaStream_t st) : st_(st) {}
    ~Scratch() {
        for (void* p : ptrs_) cudaFreeAsync(p, st_);
    }
    template <typename T>
    km_status get(T** out, size_t count, const char* what) {
        *out = nullptr;
        if (count == 0) return KM_OK;
        void* p = nullptr;
        cudaMemPool_t pool = nullptr;
        cudaError_t e = inject("alloc") ? cudaErrorMemoryAllocation : scratch_pool(&pool);
        if (e == cudaSuccess) e = cudaMallocFromPoolAsync(&p, count * sizeof(T), pool, st_);
        if (e != cudaSuccess) {
            cudaGetLastError();
            set_error("scratch allocation of %zu bytes for %s failed: %s", count * sizeof(T), what,
                      cudaGetErrorString(e));
            return KM_E_NOMEM;
        }
        ptrs_.push_back(p);
        *out = static_cast<T*>(p);
        return KM_OK;
    }

  private:
    cudaStream_t st_;
    std::vector<void*> ptrs_;
};

// ---- tracing: CUDA event pairs around each kernel phase ----
std::atomic<bool> g_trace_on{false};
std::mutex g_trace_mu;
struct TraceRec {
    int phase;
    cudaEvent_t a, b;
    int launches;
};
std::vector<TraceRec> g_trace;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
    std::lock_guard<std::mutex> lk(g_trace_mu);
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return e;
}

class PhaseScope {
  public:
    PhaseScope(cudaStream_t st, int phase, int launches) : st_(st), phase_(phase), launches_(launches) {
        if (g_trace_on.load(std::memory_order_relaxed)) {
            a_ = take_event();
            if (a_) cudaEventRecord(a_, st_);
        }
    }
    ~PhaseScope() {
        if (!a_) return;
        cudaEvent_t b = take_event();
        if (!b) return;
        cudaEventRecord(b, st_);
        std::lock_guard<std::mutex> lk(g_trace_mu);
        g_trace.push_back({phase_, a_, b, launches_});
    }

  private:
    cudaStream_t st_;
    int phase_, launches_;
    cudaEvent_t a_ = nullptr;
};

constexpr int kMaxDim = 16384;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

km_status check_shape(int64_t B, int64_t N, int64_t K, int64_t d, int dtype) {
    if (B < 1 || N < 1 || K < 1 || d < 1) {
        set_error("sizes must be positive (B=%lld N=%lld K=%lld d=%lld)", (long long)B, (long long)N, (long long)K,
                  (long long)d);
        return KM_E_INVALID;
    }
    if (dtype != KM_F32 && dtype != KM_F16) {
        set_error("unknown dtype %d", dtype);
        return KM_E_INVALID;
    }
    if (B > 65535 || B * N >= (int64_t(1) << 31) || K >= (int64_t(1) << 24) || d > kMaxDim) {
        set_error("outside the supported range: B <= 65535, B*N < 2^31, K < 2^24, d <= %d", kMaxDim);
        return KM_E_UNSUPPORTED;
    }
    const int64_t s = dtype == KM_F16 ? 2 : 4;
    if ((d * s) % 16 != 0) {
        set_error("d * sizeof(dtype) = %lld bytes is not a multiple of 16", (long long)(d * s));
        return KM_E_UNSUPPORTED;
    }
    return KM_OK;
}

km_status check_device(DeviceInfo* info) {
    km_status st = device_info(info);
    if (st != KM_OK) return st;
    if (info->cc_major != 10 || info->cc_minor != 0) {
        set_error("device %d has compute capability %d.%d; this library is built for sm_100a (10.0)", info->device,
                  info->cc_major, info->cc_minor);
        return KM_E_UNSUPPORTED;
    }
    return KM_OK;
}

km_status launched(cudaError_t e, const char* what) {
    if (inject("launch")) e = cudaErrorLaunchFailure;
    if (e != cudaSuccess) return cuda_error(e, what);
    return KM_OK;
}

#define KM_TRY(expr)                       \
    do {                                   \
        km_status _s = (expr);             \
        if (_s != KM_OK) return _s;        \
    } while (0)

bool uses_tc(int dtype, int64_t d) {
    return dtype == KM_F16 ? (assign_tc_supported(d, dtype) || assign_wide_supported(d, dtype) ||
                              assign_split_supported(d, dtype))
                           : assign_tf32_supported(d);
}

// Scratch of a tensor-core assignment: the prepared centroids and the lists of
// points left to the exact re-scan.  The list counters come in two sets of
// `lists` entries used in turn: an assignment appends to one set while its
// re-scan zeroes the other, ready for the next assignment, so that no memset
// sits between the kernels of an iteration.
struct TcScratch {
    PreparedC prep;
    int32_t* flag_count = nullptr;  // [2, lists]
    int32_t* flag_rows = nullptr;   // [lists, cap]
    int64_t lists = 0, cap = 0;
    int parity = 0;                 // the counter set the next assignment appends to
    // ||x||^2 of every point ([B, N], nullable): the first assignment of a
    // loop over the same X writes it, the later ones read it
    float* xnorm = nullptr;
    bool xnorm_valid = false;
    // batch b alone: its prepared centroids; the chunk pipeline (one batch at a
    // time, lists == 1) keeps the single list, which serves every chunk in turn
    TcScratch batch(int64_t b, int64_t K, int64_t d, int dtype) const {
        TcScratch t = *this;
        const int64_t Kp = padded_k(K);
        if (dtype == KM_F16) {
            t.prep.chat = static_cast<__half*>(prep.chat) + b * K * d;
            t.prep.cext = static_cast<__half*>(prep.cext) + b * Kp * kNormPieces;
        } else {
            t.prep.chat = static_cast<float*>(prep.chat) + b * K * 2 * d;
            t.prep.cext = static_cast<float*>(prep.cext) + b * Kp * 8;
        }
        t.prep.cmax = prep.cmax + b;
        t.xnorm = nullptr;  // the norms are kept for whole loops over all batches only
        t.xnorm_valid = false;
        return t;
    }
};

// Takes the tensor-core scratch for B batches of K centroids from `s`, with
// `lists` re-scan lists of `cap` rows, and zeroes the norm bound and the list
// counters.
km_status alloc_tc(Scratch& s, int dtype, int64_t B, int64_t K, int64_t d, int64_t lists, int64_t cap,
                   cudaStream_t st, TcScratch* out) {
    const int64_t Kp = padded_k(K);
    if (dtype == KM_F16) {
        __half *chat = nullptr, *cext = nullptr;
        KM_TRY(s.get(&chat, (size_t)(B * K * d), "rounded centroids"));
        KM_TRY(s.get(&cext, (size_t)(B * Kp * kNormPieces), "centroid norm slices"));
        out->prep.chat = chat;
        out->prep.cext = cext;
    } else {
        float *chat = nullptr, *cext = nullptr;
        KM_TRY(s.get(&chat, (size_t)(B * K * 2 * d), "centroid heads and tails"));
        KM_TRY(s.get(&cext, (size_t)(B * Kp * 8), "centroid norm pieces"));
        out->prep.chat = chat;
        out->prep.cext = cext;
    }
    KM_TRY(s.get(&out->prep.cmax, (size_t)B, "centroid norm bound"));
    KM_TRY(s.get(&out->flag_count, (size_t)(2 * lists), "re-scan counters"));
    KM_TRY(s.get(&out->flag_rows, (size_t)(lists * cap), "re-scan lists"));
    out->lists = lists;
    out->cap = cap;
    out->parity = 0;
    KM_TRY(launched(cudaMemsetAsync(out->prep.cmax, 0, sizeof(float) * (size_t)B, st), "zero norm bound"));
    return launched(cudaMemsetAsync(out->flag_count, 0, sizeof(int32_t) * (size_t)(2 * lists), st),
                    "zero re-scan counters");
}

// The re-scan list of the next assignment with `tc` (counter set tc->parity).
RescanList rescan_list(const TcScratch& tc, int dtype, int64_t d) {
    RescanList L;
    L.cmax = tc.prep.cmax;
    L.count = tc.flag_count + tc.parity * tc.lists;
    L.rows = tc.flag_rows;
    L.cap = tc.cap;
    L.total = rescan_word();
    if (dtype == KM_F16) L.set_fp16(d);
    return L;
}

// The assignment for one iteration, given prepared centroids (tc == nullptr:
// the CUDA-core kernel).  On tensor cores it is two launches: the tensor-core
// kernel, which certifies each point's label from its best two scores and
// lists the rest, then the exact re-scan of the listed points (which also
// zeroes the other counter set; tc->parity flips).
km_status run_assign(const void* X, int dtype, const float* C, TcScratch* tc, int64_t B, int64_t N, int64_t K,
                     int64_t d, int32_t* labels, float* mindist, double* obj_acc, const DeviceInfo& dev,
                     cudaStream_t st, const int32_t* stop = nullptr) {
    if (!tc) {
        PhaseScope ph(st, KM_PHASE_ASSIGN, 1);
        return launched(launch_assign_simt(X, dtype, C, B, N, K, d, labels, mindist, obj_acc, st, stop),
                        "assign (CUDA cores)");
    }
    if (tc->cap < N && obj_acc) {
        set_error("internal: a re-scan list shorter than a batch cannot carry the objective");
        return KM_E_INVALID;
    }
    PhaseScope ph(st, KM_PHASE_ASSIGN, 2);
    const RescanList L = rescan_list(*tc, dtype, d);
    int32_t* next = tc->flag_count + (1 - tc->parity) * tc->lists;
    tc->parity ^= 1;
    cudaError_t e;
    const char* what;
    if (dtype == KM_F16) {
        const __half* Xh = static_cast<const __half*>(X);
        const __half* chat = static_cast<const __half*>(tc->prep.chat);
        const __half* cext = static_cast<const __half*>(tc->prep.cext);
        if (assign_split_supported(d, dtype)) {
            e = launch_assign_split(Xh, chat, cext, B, N, K, d, labels, mindist, obj_acc, L, dev.sms, st, stop);
            what = "assign (tensor cores, points and centroids streamed along d)";
        } else if (assign_wide_supported(d, dtype)) {
            e = launch_assign_wide(Xh, chat, cext, B, N, K, d, labels, mindist, obj_acc, L, dev.sms, st, stop);
            what = "assign (tensor cores, d split in chunks)";
        } else {
            const bool have = tc->xnorm && tc->xnorm_valid;
            e = launch_assign_tc(Xh, chat, cext, B, N, K, d, labels, mindist, obj_acc, L, dev.sms, st, stop,
                                 have ? tc->xnorm : nullptr, have ? nullptr : tc->xnorm);
            tc->xnorm_valid = tc->xnorm != nullptr;
            what = "assign (tensor cores)";
        }
    } else {
        e = launch_assign_tf32(static_cast<const float*>(X), static_cast<const float*>(tc->prep.chat),
                               static_cast<const float*>(tc->prep.cext), B, N, K, d, labels, mindist, obj_acc, L,
                               dev.sms, st, stop);
        what = "assign (tf32 tensor cores)";
    }
    KM_TRY(launched(e, what));
    return launched(launch_rescan(X, dtype, C, B, N, K, d, labels, mindist, obj_acc, L, dev.sms, st, stop, next),
                    "assign (exact re-scan of listed points)");
}

std::atomic<int64_t> g_chunk_rows{0};
constexpr int64_t kDefaultChunkRows = int64_t(1) << 23;
constexpr int64_t kDefaultChunkBytes = int64_t(1) << 32;  // the default chunk also stays within 4 GiB
constexpr int kSlots = 2;

// Host-side wait for a stream, polled against a deadline (KM_HOST_TIMEOUT_S,
// default 3600 s) so that a caller never blocks forever.
km_status wait_stream(cudaStream_t st, const char* what) {
    double limit_s = 3600.0;
    if (const char* e = std::getenv("KM_HOST_TIMEOUT_S")) limit_s = std::atof(e) > 0 ? std::atof(e) : limit_s;
    const auto t0 = std::chrono::steady_clock::now();
    while (true) {
        cudaError_t e = cudaStreamQuery(st);
        if (e == cudaSuccess) return KM_OK;
        if (e != cudaErrorNotReady) return cuda_error(e, what);
        if (std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count() > limit_s) {
            set_error("%s: still running after %.0f s", what, limit_s);
            return KM_E_TIMEOUT;
        }
        std::this_thread::sleep_for(std::chrono::microseconds(200));
    }
}

// Makes `st` wait for everything enqueued on `side` (on every exit path), so
// that stream-ordered frees on `st` never overtake a copy still in flight.
struct JoinGuard {
    cudaStream_t st, side;
    ~JoinGuard() {
        cudaEvent_t ev = nullptr;
        if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) == cudaSuccess) {
            cudaEventRecord(ev, side);
            cudaStreamWaitEvent(st, ev, 0);
            cudaEventDestroy(ev);
        } else {
            cudaGetLastError();
            cudaStreamSynchronize(side);
        }
    }
};

// RAII holder for the pipeline's side stream and events.
struct PipelineRes {
    cudaStream_t copy = nullptr;
    cudaEvent_t ready[kSlots] = {nullptr, nullptr}, freed[kSlots] = {nullptr, nullptr};
    ~PipelineRes() {
        for (int i = 0; i < kSlots; ++i) {
            if (ready[i]) cudaEventDestroy(ready[i]);
            if (freed[i]) cudaEventDestroy(freed[i]);
        }
        if (copy) cudaStreamDestroy(copy);
    }
};

// km_lloyd with X in pinned host memory: every iteration streams X through
// kSlots device slots of R rows (papernotes.org "Flash-KMeans" page, 关键设计 3:
// chunked, multi-stream H2D overlapped with the assignment and update).  A
// side stream copies chunk r+1 while the caller's stream assigns, sorts and
// accumulates chunk r; slots are recycled through events.  Sums and counts
// accumulate over the chunks of an iteration; the centroids are finalised
// once per iteration.  The call waits for the work (bounded) before returning.
km_status lloyd_host(const void* X, int64_t B, int64_t N, int64_t K, int64_t d, int dtype, int iters,
                     int32_t* labels, bool labels_on_host, float* C_out, float* objective, const DeviceInfo& dev,
                     cudaStream_t st) {
    const int64_t s = dtype == KM_F16 ? 2 : 4;
    int64_t R = g_chunk_rows.load();
    if (R <= 0) R = std::max<int64_t>(1, std::min(kDefaultChunkRows, kDefaultChunkBytes / (d * s)));
    if (R > N) R = N;
    const bool tc = uses_tc(dtype, d);
    const int64_t Kp = padded_k(K);
    PipelineRes res;
    cudaError_t e = cudaStreamCreateWithFlags(&res.copy, cudaStreamNonBlocking);
    if (e != cudaSuccess) return cuda_error(e, "cudaStreamCreateWithFlags");
    for (int i = 0; i < kSlots; ++i) {
        if ((e = cudaEventCreateWithFlags(&res.ready[i], cudaEventDisableTiming)) != cudaSuccess ||
            (e = cudaEventCreateWithFlags(&res.freed[i], cudaEventDisableTiming)) != cudaSuccess)
            return cuda_error(e, "cudaEventCreate");
    }
    km_status status = KM_OK;
    {
        Scratch scratch(st);
        JoinGuard join{st, res.copy};  // destroyed before `scratch`: frees wait for the copies
        unsigned char* slot[kSlots] = {nullptr, nullptr};
        TcScratch tcs;
        float* sums = nullptr;
        double* obj_acc = nullptr;
        int32_t *lab = nullptr, *a_sorted = nullptr, *sidx = nullptr, *offs = nullptr, *counts = nullptr;
        unsigned char* work = nullptr;
        for (int i = 0; i < kSlots && status == KM_OK; ++i) status = scratch.get(&slot[i], (size_t)(R * d * s), "X slot");
        if (status == KM_OK && tc) status = alloc_tc(scratch, dtype, B, K, d, 1, R, st, &tcs);
        if (status == KM_OK) status = scratch.get(&sums, (size_t)(B * K * d), "cluster sums");
        if (status == KM_OK) status = scratch.get(&counts, (size_t)(B * K), "cluster counts");
        if (status == KM_OK && objective) status = scratch.get(&obj_acc, (size_t)B, "objective accumulator");
        if (status == KM_OK) status = scratch.get(&lab, (size_t)R, "chunk labels");
        if (status == KM_OK) status = scratch.get(&a_sorted, (size_t)R, "sorted labels");
        if (status == KM_OK) status = scratch.get(&sidx, (size_t)R, "sorted indices");
        if (status == KM_OK) status = scratch.get(&offs, (size_t)(K + 1), "segment offsets");
        if (status == KM_OK) status = scratch.get(&work, sort_scratch_bytes(1, R, K), "radix sort buffers");
        if (status != KM_OK) return status;

        if (tc) {
            PhaseScope ph(st, KM_PHASE_PREP, 1);
            KM_TRY(launched(launch_prep_centroids(C_out, B, K, d, dtype, tcs.prep, st), "centroid preparation"));
        }
        {
            PhaseScope ph(st, KM_PHASE_OTHER, 0);
            KM_TRY(launched(cudaMemsetAsync(sums, 0, sizeof(float) * (size_t)(B * K * d), st), "zero sums"));
            if (obj_acc) KM_TRY(launched(cudaMemsetAsync(obj_acc, 0, sizeof(double) * B, st), "zero objective"));
        }
        const int sort_launches = sort_kernel_launches(R, K, false, false);
        int64_t g = 0;  // global chunk counter: slot = g % kSlots
        for (int t = 0; t < iters; ++t) {
            KM_TRY(launched(cudaMemsetAsync(counts, 0, sizeof(int32_t) * (size_t)(B * K), st), "zero counts"));
            for (int64_t b = 0; b < B; ++b) {
                for (int64_t r0 = 0; r0 < N; r0 += R, ++g) {
                    const int64_t rows = (N - r0) < R ? (N - r0) : R;
                    const int si = (int)(g % kSlots);
                    // copy stream: reuse the slot only once the compute stream released it
                    if (g >= kSlots) KM_TRY(launched(cudaStreamWaitEvent(res.copy, res.freed[si], 0), "wait slot"));
                    KM_TRY(launched(cudaMemcpyAsync(slot[si], static_cast<const unsigned char*>(X) + (b * N + r0) * d * s,
                                                    (size_t)(rows * d * s), cudaMemcpyHostToDevice, res.copy),
                                    "copy X chunk"));
                    KM_TRY(launched(cudaEventRecord(res.ready[si], res.copy), "record chunk ready"));
                    // compute stream
                    KM_TRY(launched(cudaStreamWaitEvent(st, res.ready[si], 0), "wait chunk"));
                    TcScratch tcb = tc ? tcs.batch(b, K, d, dtype) : TcScratch();
                    KM_TRY(run_assign(slot[si], dtype, C_out + b * K * d, tc ? &tcb : nullptr, 1, rows, K, d, lab,
                                      nullptr, obj_acc ? obj_acc + b : nullptr, dev, st));
                    tcs.parity = tcb.parity;
                    {
                        PhaseScope ph(st, KM_PHASE_SORT, sort_launches);
                        KM_TRY(launched(launch_sort(lab, 1, rows, K, a_sorted, sidx, nullptr, nullptr, work, st, false),
                                        "label sort"));
                    }
                    {
                        PhaseScope ph(st, KM_PHASE_UPDATE, 2);
                        KM_TRY(launched(launch_update_sums(slot[si], dtype, a_sorted, sidx, 1, rows, K, d,
                                                           sums + b * K * d, offs, st, true),
                                        "segmented update"));
                        KM_TRY(launched(launch_add_counts(offs, 1, K, counts + b * K, st), "chunk counts"));
                    }
                    if (t == iters - 1) {
                        PhaseScope ph(st, KM_PHASE_OTHER, 0);
                        KM_TRY(launched(cudaMemcpyAsync(labels + b * N + r0, lab, sizeof(int32_t) * (size_t)rows,
                                                        labels_on_host ? cudaMemcpyDeviceToHost
                                                                       : cudaMemcpyDeviceToDevice,
                                                        st),
                                        "copy labels"));
                    }
                    KM_TRY(launched(cudaEventRecord(res.freed[si], st), "record slot free"));
                }
            }
            const bool prep_next = tc && t + 1 < iters;
            PhaseScope ph(st, KM_PHASE_FINALIZE, 1);
            KM_TRY(launched(launch_finalize(sums, nullptr, B, K, d, C_out, dtype, prep_next ? tcs.prep : PreparedC(),
                                            nullptr, true, obj_acc,
                                            objective ? objective + (size_t)t * B : nullptr, st, counts),
                            "centroid finalize"));
        }
    }  // scratch released on the stream
    return wait_stream(st, "km_lloyd (host-resident X)");
}

// Convergence control of the device-path iteration loop: after each
// iteration the finalisation sums every batch's squared centroid shift on the
// device, a one-block kernel counts the iteration into *iters_run and sets a
// stop flag once every batch has shift <= tol, and every kernel of the later
// iterations, already enqueued, reads the flag and returns at once -- no host
// synchronisation per iteration.
struct Converge {
    double tol;
    int32_t* iters_run;
};

// The device-path iteration loop of km_lloyd (cv == nullptr) and km_lloyd_tol.
km_status lloyd_device(const void* X, int64_t B, int64_t N, int64_t K, int64_t d, int dtype, int iters,
                       int32_t* labels, float* C_out, float* objective, const DeviceInfo& dev, cudaStream_t st,
                       const Converge* cv) {
    const size_t ckd = (size_t)(B * K * d);
    Scratch scratch(st);
    const bool tc = uses_tc(dtype, d);
    TcScratch tcs;
    float* sums = nullptr;
    double* obj_acc = nullptr;
    int32_t *a_sorted = nullptr, *sidx = nullptr, *offs = nullptr;
    unsigned char* work = nullptr;
    int32_t* stop = nullptr;
    double* shift = nullptr;
    if (tc) KM_TRY(alloc_tc(scratch, dtype, B, K, d, B, N, st, &tcs));
    if (tc && dtype == KM_F16 && assign_tc_supported(d, dtype))  // X is the same in every iteration
        KM_TRY(scratch.get(&tcs.xnorm, (size_t)(B * N), "point norms"));
    if (cv) {
        KM_TRY(scratch.get(&stop, 1, "stop flag"));
        KM_TRY(scratch.get(&shift, (size_t)B, "centroid shifts"));
    }
    if (objective) KM_TRY(scratch.get(&obj_acc, (size_t)B, "objective accumulator"));
    KM_TRY(scratch.get(&sums, ckd, "cluster sums"));
    KM_TRY(scratch.get(&offs, (size_t)(B * (K + 1)), "segment offsets"));
    KM_TRY(scratch.get(&a_sorted, (size_t)(B * N), "sorted labels"));
    KM_TRY(scratch.get(&sidx, (size_t)(B * N), "sorted indices"));
    KM_TRY(scratch.get(&work, sort_scratch_bytes(B, N, K), "radix sort buffers"));

    if (tc) {
        PhaseScope ph(st, KM_PHASE_PREP, 1);
        KM_TRY(launched(launch_prep_centroids(C_out, B, K, d, dtype, tcs.prep, st), "centroid preparation"));
    }
    {
        PhaseScope ph(st, KM_PHASE_OTHER, 0);
        KM_TRY(launched(cudaMemsetAsync(sums, 0, sizeof(float) * ckd, st), "zero sums"));
        if (obj_acc) KM_TRY(launched(cudaMemsetAsync(obj_acc, 0, sizeof(double) * B, st), "zero objective"));
        if (cv) {
            KM_TRY(launched(cudaMemsetAsync(stop, 0, sizeof(int32_t), st), "zero stop flag"));
            KM_TRY(launched(cudaMemsetAsync(shift, 0, sizeof(double) * B, st), "zero shifts"));
            KM_TRY(launched(cudaMemsetAsync(cv->iters_run, 0, sizeof(int32_t), st), "zero iteration count"));
        }
    }
    const int sort_launches = sort_kernel_launches(N, K, false, false);
    for (int t = 0; t < iters; ++t) {
        KM_TRY(run_assign(X, dtype, C_out, tc ? &tcs : nullptr, B, N, K, d, labels, nullptr, obj_acc, dev, st, stop));
        {
            PhaseScope ph(st, KM_PHASE_SORT, sort_launches);
            KM_TRY(launched(launch_sort(labels, B, N, K, a_sorted, sidx, nullptr, nullptr, work, st, false, stop),
                            "label sort"));
        }
        {
            PhaseScope ph(st, KM_PHASE_UPDATE, 1);
            KM_TRY(launched(launch_update_sums(X, dtype, a_sorted, sidx, B, N, K, d, sums, offs, st, false, stop),
                            "segmented update"));
        }
        const bool prep_next = tc && t + 1 < iters;
        PhaseScope ph(st, KM_PHASE_FINALIZE, cv ? 2 : 1);
        // the finalize zeroes the consumed sums, so the next update starts from 0
        KM_TRY(launched(launch_finalize(sums, offs, B, K, d, C_out, dtype, prep_next ? tcs.prep : PreparedC(),
                                        nullptr, true, obj_acc,
                                        objective ? objective + (size_t)t * B : nullptr, st, nullptr, stop, shift),
                        "centroid finalize"));
        if (cv) KM_TRY(launched(launch_converge_check(shift, B, cv->tol, stop, cv->iters_run, st), "convergence test"));
    }
    return KM_OK;
}

}  // namespace

void set_error(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
}

km_status cuda_error(cudaError_t e, const char* what) {
    set_error("%s: %s", what, cudaGetErrorString(e));
    return e == cudaErrorMemoryAllocation ? KM_E_NOMEM : KM_E_CUDA;
}

bool pdl_enabled() { return !g_trace_on.load(std::memory_order_relaxed); }

int32_t* fault_word() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fault) != cudaSuccess) return nullptr;
    return static_cast<int32_t*>(p);
}

unsigned long long* rescan_word() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_rescans) != cudaSuccess) return nullptr;
    return static_cast<unsigned long long*>(p);
}

km_status device_info(DeviceInfo* out) {
    // per-device attributes, filled on first use; the lock keeps a reader from
    // seeing an entry that another thread is still writing
    static DeviceInfo cache[64];
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) {
        set_error("device ordinal %d out of range", dev);
        return KM_E_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lk(mu);
    DeviceInfo& c = cache[dev];
    if (c.device != dev) {
        DeviceInfo n;
        n.device = dev;
        if ((e = cudaDeviceGetAttribute(&n.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&n.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&n.cc_minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
            return cuda_error(e, "cudaDeviceGetAttribute");
        c = n;
    }
    *out = c;
    return KM_OK;
}

}  // namespace km

using namespace km;

extern "C" {

const char* km_status_string(km_status s) {
    switch (s) {
        case KM_OK: return "ok";
        case KM_E_INVALID: return "invalid argument";
        case KM_E_UNSUPPORTED: return "unsupported shape, alignment or device";
        case KM_E_NOMEM: return "out of device memory";
        case KM_E_CUDA: return "CUDA error";
        case KM_E_TIMEOUT: return "bounded wait expired";
    }
    return "unknown status";
}

const char* km_last_error(void) { return g_err; }

km_status km_assign(const void* X, const float* C, int64_t B, int64_t N, int64_t K, int64_t d, int dtype,
                    int32_t* labels, float* mindist, void* stream) {
    g_err[0] = 0;
    if (!X || !C || !labels) {
        set_error("km_assign: X, C and labels must be non-null");
        return KM_E_INVALID;
    }
    KM_TRY(check_shape(B, N, K, d, dtype));
    if (!aligned(X, 16) || !aligned(C, 16) || !aligned(labels, 4) || (mindist && !aligned(mindist, 4))) {
        set_error("km_assign: X and C must be 16-byte aligned, labels and mindist 4-byte aligned");
        return KM_E_UNSUPPORTED;
    }
    DeviceInfo dev;
    KM_TRY(check_device(&dev));
    cudaStream_t st = (cudaStream_t)stream;
    Scratch scratch(st);
    const bool tc = uses_tc(dtype, d);
    TcScratch tcs;
    if (tc) {
        KM_TRY(alloc_tc(scratch, dtype, B, K, d, B, N, st, &tcs));
        PhaseScope ph(st, KM_PHASE_PREP, 1);
        KM_TRY(launched(launch_prep_centroids(C, B, K, d, dtype, tcs.prep, st), "centroid preparation"));
    }
    return run_assign(X, dtype, C, tc ? &tcs : nullptr, B, N, K, d, labels, mindist, nullptr, dev, st);
}

km_status km_assign_objective(const void* X, const float* C, int64_t B, int64_t N, int64_t K, int64_t d, int dtype,
                              int32_t* labels, float* mindist, double* objective, void* stream) {
    g_err[0] = 0;
    if (!X || !C || !labels || !objective) {
        set_error("km_assign_objective: X, C, labels and objective must be non-null");
        return KM_E_INVALID;
    }
    KM_TRY(check_shape(B, N, K, d, dtype));
    if (!aligned(X, 16) || !aligned(C, 16) || !aligned(labels, 4) || (mindist && !aligned(mindist, 4)) ||
        !aligned(objective, 8)) {
        set_error("km_assign_objective: X and C must be 16-byte aligned, labels and mindist 4-byte aligned, "
                  "objective 8-byte aligned");
        return KM_E_UNSUPPORTED;
    }
    DeviceInfo dev;
    KM_TRY(check_device(&dev));
    cudaStream_t st = (cudaStream_t)stream;
    Scratch scratch(st);
    const bool tc = uses_tc(dtype, d);
    TcScratch tcs;
    {
        PhaseScope ph(st, KM_PHASE_OTHER, 0);
        KM_TRY(launched(cudaMemsetAsync(objective, 0, sizeof(double) * (size_t)B, st), "zero objective"));
    }
    if (tc) {
        KM_TRY(alloc_tc(scratch, dtype, B, K, d, B, N, st, &tcs));
        PhaseScope ph(st, KM_PHASE_PREP, 1);
        KM_TRY(launched(launch_prep_centroids(C, B, K, d, dtype, tcs.prep, st), "centroid preparation"));
    }
    return run_assign(X, dtype, C, tc ? &tcs : nullptr, B, N, K, d, labels, mindist, objective, dev, st);
}

km_status km_sort_labels(const int32_t* labels, int64_t B, int64_t N, int64_t K, int32_t* sorted_idx,
                         int32_t* counts, int32_t* offsets, void* stream) {
    g_err[0] = 0;
    if (!labels || !sorted_idx || !counts) {
        set_error("km_sort_labels: labels, sorted_idx and counts must be non-null");
        return KM_E_INVALID;
    }
    KM_TRY(check_shape(B, N, K, 16, KM_F16));
    if (!aligned(labels, 4) || !aligned(sorted_idx, 4) || !aligned(counts, 4) || (offsets && !aligned(offsets, 4))) {
        set_error("km_sort_labels: arrays must be 4-byte aligned");
        return KM_E_UNSUPPORTED;
    }
    DeviceInfo dev;
    KM_TRY(check_device(&dev));
    cudaStream_t st = (cudaStream_t)stream;
    Scratch scratch(st);
    int32_t* a_sorted = nullptr;
    unsigned char* work = nullptr;
    KM_TRY(scratch.get(&a_sorted, (size_t)(B * N), "sorted labels"));
    KM_TRY(scratch.get(&work, sort_scratch_bytes(B, N, K), "radix sort buffers"));
    PhaseScope ph(st, KM_PHASE_SORT, sort_kernel_launches(N, K, true));
    return launched(launch_sort(labels, B, N, K, a_sorted, sorted_idx, counts, offsets, work, st), "label sort");
}

km_status km_update(const void* X, const int32_t* labels, int64_t B, int64_t N, int64_t K, int64_t d, int dtype,
                    float* sums, int32_t* counts, float* C_out, void* stream) {
    g_err[0] = 0;
    if (!X || !labels || !sums || !counts || !C_out) {
        set_error("km_update: X, labels, sums, counts and C_out must be non-null");
        return KM_E_INVALID;
    }
    KM_TRY(check_shape(B, N, K, d, dtype));
    if (!aligned(X, 16) || !aligned(sums, 16) || !aligned(C_out, 16) || !aligned(labels, 4) || !aligned(counts, 4)) {
        set_error("km_update: X, sums and C_out must be 16-byte aligned, labels and counts 4-byte aligned");
        return KM_E_UNSUPPORTED;
    }
    DeviceInfo dev;
    KM_TRY(check_device(&dev));
    cudaStream_t st = (cudaStream_t)stream;
    Scratch scratch(st);
    int32_t *a_sorted = nullptr, *sidx = nullptr, *offs = nullptr;
    unsigned char* work = nullptr;
    KM_TRY(scratch.get(&a_sorted, (size_t)(B * N), "sorted labels"));
    KM_TRY(scratch.get(&sidx, (size_t)(B * N), "sorted indices"));
    KM_TRY(scratch.get(&offs, (size_t)(B * (K + 1)), "segment offsets"));
    KM_TRY(scratch.get(&work, sort_scratch_bytes(B, N, K), "radix sort buffers"));
    {
        PhaseScope ph(st, KM_PHASE_OTHER, 0);
        KM_TRY(launched(cudaMemsetAsync(sums, 0, sizeof(float) * (size_t)(B * K * d), st), "zero sums"));
    }
    {
        PhaseScope ph(st, KM_PHASE_SORT, sort_kernel_launches(N, K, false, false));
        KM_TRY(launched(launch_sort(labels, B, N, K, a_sorted, sidx, nullptr, nullptr, work, st, false),
                        "label sort"));
    }
    {
        PhaseScope ph(st, KM_PHASE_UPDATE, 1);
        KM_TRY(launched(launch_update_sums(X, dtype, a_sorted, sidx, B, N, K, d, sums, offs, st),
                        "segmented update"));
    }
    PhaseScope ph(st, KM_PHASE_FINALIZE, 1);
    return launched(
        launch_finalize(sums, offs, B, K, d, C_out, dtype, PreparedC(), counts, false, nullptr, nullptr, st),
        "centroid finalize");
}

km_status km_update_sums(const void* X, const int32_t* labels, int64_t B, int64_t N, int64_t K, int64_t d, int dtype,
                         float* sums, int32_t* counts, void* stream) {
    g_err[0] = 0;
    if (!X || !labels || !sums || !counts) {
        set_error("km_update_sums: X, labels, sums and counts must be non-null");
        return KM_E_INVALID;
    }
    KM_TRY(check_shape(B, N, K, d, dtype));
    if (!aligned(X, 16) || !aligned(sums, 16) || !aligned(labels, 4) || !aligned(counts, 4)) {
        set_error("km_update_sums: X and sums must be 16-byte aligned, labels and counts 4-byte aligned");
        return KM_E_UNSUPPORTED;
    }
    DeviceInfo dev;
    KM_TRY(check_device(&dev));
    cudaStream_t st = (cudaStream_t)stream;
    Scratch scratch(st);
    int32_t *a_sorted = nullptr, *sidx = nullptr, *offs = nullptr;
    unsigned char* work = nullptr;
    KM_TRY(scratch.get(&a_sorted, (size_t)(B * N), "sorted labels"));
    KM_TRY(scratch.get(&sidx, (size_t)(B * N), "sorted indices"));
    KM_TRY(scratch.get(&offs, (size_t)(B * (K + 1)), "segment offsets"));
    KM_TRY(scratch.get(&work, sort_scratch_bytes(B, N, K), "radix sort buffers"));
    {
        PhaseScope ph(st, KM_PHASE_OTHER, 0);
        KM_TRY(launched(cudaMemsetAsync(sums, 0, sizeof(float) * (size_t)(B * K * d), st), "zero sums"));
        KM_TRY(launched(cudaMemsetAsync(counts, 0, sizeof(int32_t) * (size_t)(B * K), st), "zero counts"));
    }
    {
        PhaseScope ph(st, KM_PHASE_SORT, sort_kernel_launches(N, K, false, false));
        KM_TRY(launched(launch_sort(labels, B, N, K, a_sorted, sidx, nullptr, nullptr, work, st, false),
                        "label sort"));
    }
    PhaseScope ph(st, KM_PHASE_UPDATE, 2);
    KM_TRY(launched(launch_update_sums(X, dtype, a_sorted, sidx, B, N, K, d, sums, offs, st), "segmented update"));
    return launched(launch_add_counts(offs, B, K, counts, st), "cluster counts");
}

km_status km_finalize(const float* sums, const int32_t* counts, int64_t B, int64_t K, int64_t d, float* C_out,
                      void* stream) {
    g_err[0] = 0;
    if (!sums || !counts || !C_out) {
        set_error("km_finalize: sums, counts and C_out must be non-null");
        return KM_E_INVALID;
    }
    KM_TRY(check_shape(B, 1, K, d, KM_F32));
    if (!aligned(sums, 16) || !aligned(C_out, 16) || !aligned(counts, 4)) {
        set_error("km_finalize: sums and C_out must be 16-byte aligned, counts 4-byte aligned");
        return KM_E_UNSUPPORTED;
    }
    DeviceInfo dev;
    KM_TRY(check_device(&dev));
    cudaStream_t st = (cudaStream_t)stream;
    PhaseScope ph(st, KM_PHASE_FINALIZE, 1);
    return launched(launch_finalize(const_cast<float*>(sums), nullptr, B, K, d, C_out, KM_F32, PreparedC(), nullptr,
                                    false, nullptr, nullptr, st, counts),
                    "centroid finalize");
}

km_status km_assign_dense(const void* X, const float* C, int64_t B, int64_t N, int64_t K, int64_t d, int dtype,
                          int32_t* labels, float* mindist, void* stream) {
    g_err[0] = 0;
    if (!X || !C || !labels) {
        set_error("km_assign_dense: X, C and labels must be non-null");
        return KM_E_INVALID;
    }
    KM_TRY(check_shape(B, N, K, d, dtype));
    if (dtype != KM_F16 || !assign_tc_supported(d, dtype)) {
        set_error("km_assign_dense: fp16 points with 64 <= d <= 128 only (the tensor-core kernel's range)");
        return KM_E_UNSUPPORTED;
    }
    if (!aligned(X, 16) || !aligned(C, 16) || !aligned(labels, 4) || (mindist && !aligned(mindist, 4))) {
        set_error("km_assign_dense: X and C must be 16-byte aligned, labels and mindist 4-byte aligned");
        return KM_E_UNSUPPORTED;
    }
    DeviceInfo dev;
    KM_TRY(check_device(&dev));
    cudaStream_t st = (cudaStream_t)stream;
    Scratch scratch(st);
    TcScratch tcs;
    float *dense = nullptr, *xnorm = nullptr;
    KM_TRY(alloc_tc(scratch, dtype, B, K, d, B, N, st, &tcs));
    KM_TRY(scratch.get(&dense, (size_t)(B * N * padded_k(K)), "dense score matrix"));
    KM_TRY(scratch.get(&xnorm, (size_t)(B * N), "point norms"));
    {
        PhaseScope ph(st, KM_PHASE_PREP, 1);
        KM_TRY(launched(launch_prep_centroids(C, B, K, d, dtype, tcs.prep, st), "centroid preparation"));
    }
    PhaseScope ph(st, KM_PHASE_ASSIGN, 3);
    KM_TRY(launched(launch_assign_tc_dense((const __half*)X, static_cast<const __half*>(tcs.prep.chat),
                                           static_cast<const __half*>(tcs.prep.cext), B, N, K, d, dense, xnorm,
                                           dev.sms, st),
                    "dense scores (tensor cores)"));
    const RescanList L = rescan_list(tcs, dtype, d);
    KM_TRY(launched(launch_dense_argmin(dense, xnorm, B, N, K, labels, mindist, L, st),
                    "argmin over the dense scores"));
    return launched(launch_rescan(X, dtype, C, B, N, K, d, labels, mindist, nullptr, L, dev.sms, st),
                    "assign (exact re-scan of listed points)");
}

km_status km_update_scatter(const void* X, const int32_t* labels, int64_t B, int64_t N, int64_t K, int64_t d,
                            int dtype, float* sums, int32_t* counts, float* C_out, void* stream) {
    g_err[0] = 0;
    if (!X || !labels || !sums || !counts || !C_out) {
        set_error("km_update_scatter: X, labels, sums, counts and C_out must be non-null");
        return KM_E_INVALID;
    }
    KM_TRY(check_shape(B, N, K, d, dtype));
    if (!aligned(X, 16) || !aligned(sums, 16) || !aligned(C_out, 16) || !aligned(labels, 4) || !aligned(counts, 4)) {
        set_error("km_update_scatter: X, sums and C_out must be 16-byte aligned, labels and counts 4-byte aligned");
        return KM_E_UNSUPPORTED;
    }
    DeviceInfo dev;
    KM_TRY(check_device(&dev));
    cudaStream_t st = (cudaStream_t)stream;
    {
        PhaseScope ph(st, KM_PHASE_OTHER, 0);
        KM_TRY(launched(cudaMemsetAsync(sums, 0, sizeof(float) * (size_t)(B * K * d), st), "zero sums"));
        KM_TRY(launched(cudaMemsetAsync(counts, 0, sizeof(int32_t) * (size_t)(B * K), st), "zero counts"));
    }
    {
        PhaseScope ph(st, KM_PHASE_UPDATE, 1);
        KM_TRY(launched(launch_scatter_update(X, dtype, labels, B, N, K, d, sums, counts, st), "scatter update"));
    }
    PhaseScope ph(st, KM_PHASE_FINALIZE, 1);
    return launched(launch_finalize(sums, nullptr, B, K, d, C_out, dtype, PreparedC(), nullptr, false, nullptr,
                                    nullptr, st, counts),
                    "centroid finalize");
}

km_status km_lloyd(const void* X, const float* C_init, int64_t B, int64_t N, int64_t K, int64_t d, int dtype,
                   int iters, int32_t* labels, float* C_out, float* objective, void* stream) {
    g_err[0] = 0;
    if (!X || !C_init || !labels || !C_out) {
        set_error("km_lloyd: X, C_init, labels and C_out must be non-null");
        return KM_E_INVALID;
    }
    if (iters < 0) {
        set_error("km_lloyd: iters must be >= 0");
        return KM_E_INVALID;
    }
    KM_TRY(check_shape(B, N, K, d, dtype));
    if (!aligned(X, 16) || !aligned(C_init, 16) || !aligned(C_out, 16) || !aligned(labels, 4) ||
        (objective && !aligned(objective, 4))) {
        set_error("km_lloyd: X, C_init and C_out must be 16-byte aligned, labels and objective 4-byte aligned");
        return KM_E_UNSUPPORTED;
    }
    DeviceInfo dev;
    KM_TRY(check_device(&dev));
    cudaPointerAttributes pa;
    cudaError_t e = cudaPointerGetAttributes(&pa, X);
    if (e != cudaSuccess) return cuda_error(e, "cudaPointerGetAttributes(X)");
    const bool host_x = pa.type == cudaMemoryTypeHost;
    if (!host_x && pa.type != cudaMemoryTypeDevice && pa.type != cudaMemoryTypeManaged) {
        set_error("km_lloyd: X must be device memory or pinned host memory (cudaHostAlloc / cudaHostRegister)");
        return KM_E_UNSUPPORTED;
    }
    bool labels_on_host = false;
    if (host_x) {
        cudaPointerAttributes pl;
        if ((e = cudaPointerGetAttributes(&pl, labels)) != cudaSuccess) return cuda_error(e, "cudaPointerGetAttributes");
        labels_on_host = pl.type == cudaMemoryTypeHost;
        if (!labels_on_host && pl.type != cudaMemoryTypeDevice && pl.type != cudaMemoryTypeManaged) {
            set_error("km_lloyd: with host-resident X, labels must be pinned host or device memory");
            return KM_E_UNSUPPORTED;
        }
    }
    cudaStream_t st = (cudaStream_t)stream;
    const size_t ckd = (size_t)(B * K * d);
    if (C_out != C_init)
        KM_TRY(launched(cudaMemcpyAsync(C_out, C_init, sizeof(float) * ckd, cudaMemcpyDeviceToDevice, st),
                        "copy C_init"));
    if (iters == 0) return KM_OK;
    if (host_x) return lloyd_host(X, B, N, K, d, dtype, iters, labels, labels_on_host, C_out, objective, dev, st);

    return lloyd_device(X, B, N, K, d, dtype, iters, labels, C_out, objective, dev, st, nullptr);
}

km_status km_lloyd_tol(const void* X, const float* C_init, int64_t B, int64_t N, int64_t K, int64_t d, int dtype,
                       int max_iters, double tol, int32_t* labels, float* C_out, float* objective, int32_t* iters_run,
                       void* stream) {
    g_err[0] = 0;
    if (!X || !C_init || !labels || !C_out || !iters_run) {
        set_error("km_lloyd_tol: X, C_init, labels, C_out and iters_run must be non-null");
        return KM_E_INVALID;
    }
    if (max_iters < 1 || !(tol >= 0.0)) {
        set_error("km_lloyd_tol: max_iters must be >= 1 and tol a number >= 0");
        return KM_E_INVALID;
    }
    KM_TRY(check_shape(B, N, K, d, dtype));
    if (!aligned(X, 16) || !aligned(C_init, 16) || !aligned(C_out, 16) || !aligned(labels, 4) ||
        !aligned(iters_run, 4) || (objective && !aligned(objective, 4))) {
        set_error("km_lloyd_tol: X, C_init and C_out must be 16-byte aligned, labels, iters_run and objective "
                  "4-byte aligned");
        return KM_E_UNSUPPORTED;
    }
    DeviceInfo dev;
    KM_TRY(check_device(&dev));
    cudaPointerAttributes pa;
    cudaError_t e = cudaPointerGetAttributes(&pa, X);
    if (e != cudaSuccess) return cuda_error(e, "cudaPointerGetAttributes(X)");
    if (pa.type != cudaMemoryTypeDevice && pa.type != cudaMemoryTypeManaged) {
        set_error("km_lloyd_tol: X must be device memory (host-resident X: use km_lloyd)");
        return KM_E_UNSUPPORTED;
    }
    cudaStream_t st = (cudaStream_t)stream;
    if (C_out != C_init)
        KM_TRY(launched(cudaMemcpyAsync(C_out, C_init, sizeof(float) * (size_t)(B * K * d), cudaMemcpyDeviceToDevice,
                                        st),
                        "copy C_init"));
    const Converge cv{tol, iters_run};
    return lloyd_device(X, B, N, K, d, dtype, max_iters, labels, C_out, objective, dev, st, &cv);
}

km_status km_release_cached(void) {
    g_err[0] = 0;
    std::lock_guard<std::mutex> lk(g_pool_mu);
    for (int dev = 0; dev < 64; ++dev) {
        if (!g_pool[dev]) continue;
        cudaError_t e = cudaMemPoolTrimTo(g_pool[dev], 0);
        if (e != cudaSuccess) return cuda_error(e, "cudaMemPoolTrimTo");
    }
    return KM_OK;
}

void km_set_chunk_rows(int64_t rows) { g_chunk_rows.store(rows > 0 ? rows : 0); }

void km_trace_enable(int on) { g_trace_on.store(on != 0); }

km_status km_trace_read(double* ms, int64_t* launches, int nphases) {
    g_err[0] = 0;
    std::vector<TraceRec> recs;
    {
        std::lock_guard<std::mutex> lk(g_trace_mu);
        recs.swap(g_trace);
    }
    for (int p = 0; p < nphases; ++p) {
        if (ms) ms[p] = 0.0;
        if (launches) launches[p] = 0;
    }
    km_status st = KM_OK;
    for (const TraceRec& r : recs) {
        float t = 0.f;
        cudaError_t e = cudaEventSynchronize(r.b);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.a, r.b);
        if (e != cudaSuccess && st == KM_OK) st = cuda_error(e, "trace event");
        if (r.phase < nphases) {
            if (ms) ms[r.phase] += t;
            if (launches) launches[r.phase] += r.launches;
        }
    }
    std::lock_guard<std::mutex> lk(g_trace_mu);
    for (const TraceRec& r : recs) {
        g_event_pool.push_back(r.a);
        g_event_pool.push_back(r.b);
    }
    return st;
}

km_status km_device_fault(int32_t* code, void* stream) {
    g_err[0] = 0;
    if (!code) {
        set_error("km_device_fault: code must be non-null");
        return KM_E_INVALID;
    }
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_error(e, "cudaStreamSynchronize");
    int32_t v = 0, zero = 0;
    if ((e = cudaMemcpyFromSymbol(&v, g_fault, sizeof(v))) != cudaSuccess) return cuda_error(e, "read fault word");
    if ((e = cudaMemcpyToSymbol(g_fault, &zero, sizeof(zero))) != cudaSuccess) return cuda_error(e, "clear fault word");
    *code = v;
    return KM_OK;
}

km_status km_assign_rescans(int64_t* count, void* stream) {
    g_err[0] = 0;
    if (!count) {
        set_error("km_assign_rescans: count must be non-null");
        return KM_E_INVALID;
    }
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_error(e, "cudaStreamSynchronize");
    unsigned long long v = 0, zero = 0;
    if ((e = cudaMemcpyFromSymbol(&v, g_rescans, sizeof(v))) != cudaSuccess) return cuda_error(e, "read re-scan count");
    if ((e = cudaMemcpyToSymbol(g_rescans, &zero, sizeof(zero))) != cudaSuccess)
        return cuda_error(e, "clear re-scan count");
    *count = (int64_t)v;
    return KM_OK;
}

}  // extern "C"
