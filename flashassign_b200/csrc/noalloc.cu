// km_assign_noalloc: the assignment step without any device-memory allocation.
//
// km_assign takes its scratch (the centroids rounded to the dtype of X and
// their norm slices) from the stream-ordered allocator.  Some callers cannot
// allocate: a framework that reserved the whole device for its own pool, or
// a latency-critical loop that must not enter the allocator (which can
// synchronise and take locks).  This variant runs the same kernels with that
// scratch in one fixed array compiled into the library instead: the
// centroid preparation, the tensor-core assignment (fp16, or fp32 on tf32)
// and the exact re-scan of the points it could not certify.
//
// The array is a file-scope __device__ object, so every GPU that loads the
// library holds kNoAllocScratchBytes of it until the process exits.  Host
// code cannot use the array's name as a device address (on the host it is
// only a stand-in symbol); the device address is looked up once per device
// with cudaGetSymbolAddress, with that device current, the first time the
// entry point runs on it.
#include "km_internal.cuh"

#include <algorithm>
#include <mutex>

namespace km {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {nullptr};

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Device address of the scratch array on the current device (looked up once).
km_status scratch_address(int dev, void** out) {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_error(e, "cudaGetSymbolAddress(no-allocation scratch)");
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return KM_OK;
}

}  // namespace
}  // namespace km

using namespace km;

extern "C" size_t km_assign_noalloc_limit(void) { return kNoAllocScratchBytes; }

extern "C" km_status km_assign_noalloc(const void* X, const float* C, int64_t B, int64_t N, int64_t K, int64_t d,
                                       int dtype, int32_t* labels, float* mindist, void* stream) {
    set_error("%s", "");
    if (!X || !C || !labels) {
        set_error("km_assign_noalloc: X, C and labels must be non-null");
        return KM_E_INVALID;
    }
    if (B < 1 || N < 1 || K < 1 || d < 1) {
        set_error("km_assign_noalloc: sizes must be positive");
        return KM_E_INVALID;
    }
    if (dtype != KM_F32 && dtype != KM_F16) {
        set_error("km_assign_noalloc: unknown dtype %d", dtype);
        return KM_E_INVALID;
    }
    const int64_t s = dtype == KM_F16 ? 2 : 4;
    if (B > 65535 || B * N >= (int64_t(1) << 31) || K >= (int64_t(1) << 24) || d > 16384 || (d * s) % 16 != 0) {
        set_error("km_assign_noalloc: outside the supported range (B <= 65535, B*N < 2^31, K < 2^24, d <= 16384, "
                  "d * sizeof(dtype) a multiple of 16 bytes)");
        return KM_E_UNSUPPORTED;
    }
    if ((reinterpret_cast<uintptr_t>(X) % 16) || (reinterpret_cast<uintptr_t>(C) % 16) ||
        (reinterpret_cast<uintptr_t>(labels) % 4) || (mindist && reinterpret_cast<uintptr_t>(mindist) % 4)) {
        set_error("km_assign_noalloc: X and C must be 16-byte aligned, labels and mindist 4-byte aligned");
        return KM_E_UNSUPPORTED;
    }
    DeviceInfo dev;
    km_status st = device_info(&dev);
    if (st != KM_OK) return st;
    if (dev.cc_major != 10 || dev.cc_minor != 0) {
        set_error("km_assign_noalloc: device %d has compute capability %d.%d; built for sm_100a", dev.device,
                  dev.cc_major, dev.cc_minor);
        return KM_E_UNSUPPORTED;
    }
    cudaStream_t stm = (cudaStream_t)stream;
    const bool tc = dtype == KM_F16 ? (assign_tc_supported(d, dtype) || assign_wide_supported(d, dtype) ||
                                       assign_split_supported(d, dtype))
                                    : assign_tf32_supported(d);
    if (!tc) {  // the CUDA-core kernel reads C directly and needs no scratch
        cudaError_t e = launch_assign_simt(X, dtype, C, B, N, K, d, labels, mindist, nullptr, stm);
        return e == cudaSuccess ? KM_OK : cuda_error(e, "km_assign_noalloc: assign (CUDA cores)");
    }
    // the array holds, in order: the prepared centroids (fp16: rounded rows and
    // norm slices; fp32: tf32 heads and tails and norm pieces), the per-batch
    // norm bound, the re-scan counters, and as many re-scan rows per batch as
    // fit (up to N; a batch whose list overflows is re-scanned whole)
    const int64_t Kp = padded_k(K);
    const size_t chat_bytes =
        round_up((dtype == KM_F16 ? sizeof(__half) : 2 * sizeof(float)) * (size_t)(B * K * d), 256);
    const size_t cext_bytes =
        round_up(dtype == KM_F16 ? sizeof(__half) * (size_t)(B * Kp * kNormPieces) : sizeof(float) * (size_t)(B * Kp * 8),
                 256);
    const size_t fixed = chat_bytes + cext_bytes + round_up(sizeof(float) * (size_t)B, 256) +
                         round_up(sizeof(int32_t) * (size_t)B, 256);
    if (fixed > kNoAllocScratchBytes) {
        set_error("km_assign_noalloc: needs %zu bytes of scratch for the prepared centroids (fp16: 2*B*K*d + "
                  "32*B*ceil(K/256)*256; fp32: 8*B*K*d + 32*B*ceil(K/256)*256; plus 8*B), above the fixed %zu-byte "
                  "array; use km_assign",
                  fixed, kNoAllocScratchBytes);
        return KM_E_UNSUPPORTED;
    }
    void* base = nullptr;
    if ((st = scratch_address(dev.device, &base)) != KM_OK) return st;
    unsigned char* p = static_cast<unsigned char*>(base);
    PreparedC prep;
    prep.chat = p;
    prep.cext = p + chat_bytes;
    prep.cmax = reinterpret_cast<float*>(p + chat_bytes + cext_bytes);
    RescanList L;
    L.cmax = prep.cmax;
    L.count = reinterpret_cast<int32_t*>(p + chat_bytes + cext_bytes + round_up(sizeof(float) * (size_t)B, 256));
    L.rows = reinterpret_cast<int32_t*>(p + fixed);
    L.cap = std::min<int64_t>(N, (int64_t)((kNoAllocScratchBytes - fixed) / (sizeof(int32_t) * (size_t)B)));
    L.total = rescan_word();
    if (dtype == KM_F16) L.set_fp16(d);
    // the bound and the counters must start at zero; every other element that
    // the kernels read is written first by the preparation or the assignment
    cudaError_t e = cudaMemsetAsync(prep.cmax, 0, sizeof(float) * (size_t)B, stm);
    if (e == cudaSuccess) e = cudaMemsetAsync(L.count, 0, sizeof(int32_t) * (size_t)B, stm);
    if (e != cudaSuccess) return cuda_error(e, "km_assign_noalloc: clear the scratch's counters");
    e = launch_prep_centroids(C, B, K, d, dtype, prep, stm);
    if (e != cudaSuccess) return cuda_error(e, "km_assign_noalloc: centroid preparation");
    if (dtype == KM_F16) {
        const __half* Xh = static_cast<const __half*>(X);
        const __half* chat = static_cast<const __half*>(prep.chat);
        const __half* cext = static_cast<const __half*>(prep.cext);
        if (assign_split_supported(d, dtype))
            e = launch_assign_split(Xh, chat, cext, B, N, K, d, labels, mindist, nullptr, L, dev.sms, stm);
        else if (assign_wide_supported(d, dtype))
            e = launch_assign_wide(Xh, chat, cext, B, N, K, d, labels, mindist, nullptr, L, dev.sms, stm);
        else
            e = launch_assign_tc(Xh, chat, cext, B, N, K, d, labels, mindist, nullptr, L, dev.sms, stm);
    } else {
        e = launch_assign_tf32(static_cast<const float*>(X), static_cast<const float*>(prep.chat),
                               static_cast<const float*>(prep.cext), B, N, K, d, labels, mindist, nullptr, L, dev.sms,
                               stm);
    }
    if (e != cudaSuccess) return cuda_error(e, "km_assign_noalloc: assign (tensor cores)");
    e = launch_rescan(X, dtype, C, B, N, K, d, labels, mindist, nullptr, L, dev.sms, stm);
    return e == cudaSuccess ? KM_OK : cuda_error(e, "km_assign_noalloc: exact re-scan of listed points");
}
