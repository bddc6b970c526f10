// km_assign_noalloc: the assignment step without any device-memory allocation.
//
// km_assign takes its scratch (the centroids rounded to the dtype of X and
// their norm slices) from the stream-ordered allocator.  Some callers cannot
// allocate: a framework that reserved the whole device for its own pool, or
// a latency-critical loop that must not enter the allocator (which can
// synchronise and take locks).  This variant runs the same kernels with that
// scratch in one fixed array compiled into the library instead.
//
// The array is a file-scope __device__ object, so every GPU that loads the
// library holds kNoAllocScratchBytes of it until the process exits.  Host
// code cannot use the array's name as a device address (on the host it is
// only a stand-in symbol); the device address is looked up once per device
// with cudaGetSymbolAddress, with that device current, the first time the
// entry point runs on it.
#include "km_internal.cuh"

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
    const bool tc = dtype == KM_F16 && (assign_tc_supported(d, dtype) || assign_wide_supported(d, dtype) ||
                                        assign_split_supported(d, dtype));
    if (!tc) {  // the CUDA-core kernel reads C directly and needs no scratch
        cudaError_t e = launch_assign_simt(X, dtype, C, B, N, K, d, labels, mindist, nullptr, stm);
        return e == cudaSuccess ? KM_OK : cuda_error(e, "km_assign_noalloc: assign (CUDA cores)");
    }
    const size_t chat_bytes = round_up(sizeof(__half) * (size_t)(B * K * d), 256);
    const size_t cext_bytes = sizeof(__half) * (size_t)(B * padded_k(K) * 16);
    if (chat_bytes + cext_bytes > kNoAllocScratchBytes) {
        set_error("km_assign_noalloc: needs %zu bytes of scratch (2*B*K*d + 32*B*ceil(K/256)*256), above the "
                  "fixed %zu-byte array; use km_assign",
                  chat_bytes + cext_bytes, kNoAllocScratchBytes);
        return KM_E_UNSUPPORTED;
    }
    void* base = nullptr;
    if ((st = scratch_address(dev.device, &base)) != KM_OK) return st;
    __half* chat = static_cast<__half*>(base);
    __half* cext = reinterpret_cast<__half*>(static_cast<unsigned char*>(base) + chat_bytes);
    // every element of both scratch regions that the assignment reads is written here first
    PreparedC prep;
    prep.chat = chat;
    prep.cext = cext;
    cudaError_t e = launch_prep_centroids(C, B, K, d, dtype, prep, stm);
    if (e != cudaSuccess) return cuda_error(e, "km_assign_noalloc: centroid preparation");
    const __half* Xh = static_cast<const __half*>(X);
    if (assign_split_supported(d, dtype))
        e = launch_assign_split(Xh, chat, cext, B, N, K, d, labels, mindist, nullptr, dev.sms, stm);
    else if (assign_wide_supported(d, dtype))
        e = launch_assign_wide(Xh, chat, cext, B, N, K, d, labels, mindist, nullptr, dev.sms, stm);
    else
        e = launch_assign_tc(Xh, chat, cext, B, N, K, d, labels, mindist, nullptr, dev.sms, stm);
    return e == cudaSuccess ? KM_OK : cuda_error(e, "km_assign_noalloc: assign (tensor cores)");
}
