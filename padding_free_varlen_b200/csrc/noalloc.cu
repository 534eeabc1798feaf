// Packing of a padded batch without any device allocation.
//
// Some callers cannot allocate device memory at the point where they need to
// pack a batch: an inference runtime's per-request enqueue hook that forbids
// allocation after start-up, a process whose device memory is owned by a pool
// manager that must not be bypassed, or code that has no place to keep a
// caller-owned workspace.  energon_rce_remove_padding_noalloc serves them: it
// computes the per-sequence offsets into a fixed scratch array that is part of
// the library image (a file-scope __device__ array, present on every GPU that
// loads the library until the process exits) and gathers the valid rows from
// there, so the caller only passes inputs and outputs.
//
// The array holds batch + 1 offsets for batch <= ENERGON_NOALLOC_MAX_BATCH.
// Every call on a device shares it and it keeps the last call's contents; the
// offsets kernel rewrites every entry a call reads before the gather reads
// it, so nothing has to be cleared between calls.  Calls that can overlap on
// the GPU (different streams without ordering) race on the array.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace energon {
void record_error(int code, const char* msg);
}

// The offsets scratch: batch + 1 int32 entries, 64 KiB + 4 bytes at the maximum batch.
static __device__ __align__(256) int32_t g_noalloc_offsets[ENERGON_NOALLOC_MAX_BATCH + 1];

namespace {

constexpr int kMaxDevices = 128;
std::mutex g_addr_mu;
int32_t* g_addr[kMaxDevices] = {};
CUcontext g_addr_ctx[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// The driver's cuCtxGetCurrent, found through the runtime (the library does not link
// the driver library directly); null if it cannot be found.
CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and reused.  The lookup is keyed by the
// device's current context as well: cudaDeviceReset destroys the context and the
// library's device image with it, and the first call after it (in the new
// context) looks the address up again instead of using the old one.
cudaError_t scratch_address(int32_t** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    CtxGetCurrentFn get = ctx_get_current();
    if (get == nullptr) return cudaErrorInitializationError;
    CUcontext ctx = nullptr;
    if (get(&ctx) != CUDA_SUCCESS) ctx = nullptr;  // null until the runtime has set up this device
    std::lock_guard<std::mutex> lock(g_addr_mu);
    if (g_addr[dev] == nullptr || ctx == nullptr || g_addr_ctx[dev] != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_offsets);  // sets up the primary context if needed
        if (e != cudaSuccess) return e;
        if (get(&ctx) != CUDA_SUCCESS) ctx = nullptr;
        g_addr[dev] = static_cast<int32_t*>(p);
        g_addr_ctx[dev] = ctx;
    }
    *out = g_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" int energon_rce_remove_padding_noalloc(const void* padded, const int32_t* lengths, int batch, int pad_len,
                                                  int hidden, int elem_bytes, void* packed, int32_t* d_status,
                                                  void* stream) {
    using namespace energon;
    record_error(ENERGON_OK, "");
    if (!padded || !packed || !d_status || (batch > 0 && !lengths)) {
        record_error(ENERGON_ERR_INVALID_ARGUMENT, "remove_noalloc: NULL pointer");
        return ENERGON_ERR_INVALID_ARGUMENT;
    }
    if (batch < 0 || pad_len < 0 || hidden < 0) {
        record_error(ENERGON_ERR_INVALID_ARGUMENT, "remove_noalloc: negative size");
        return ENERGON_ERR_INVALID_ARGUMENT;
    }
    if (batch > ENERGON_NOALLOC_MAX_BATCH) {
        record_error(ENERGON_ERR_INVALID_ARGUMENT,
                     "remove_noalloc: batch exceeds ENERGON_NOALLOC_MAX_BATCH (16384); use "
                     "energon_rce_offsets + energon_rce_remove_padding with caller-owned offsets");
        return ENERGON_ERR_INVALID_ARGUMENT;
    }
    if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8) {
        record_error(ENERGON_ERR_INVALID_ARGUMENT, "remove_noalloc: elem_bytes must be 1, 2, 4 or 8");
        return ENERGON_ERR_INVALID_ARGUMENT;
    }
    if ((int64_t)batch * pad_len > (int64_t)0x7fffff00) {
        record_error(ENERGON_ERR_INVALID_ARGUMENT, "remove_noalloc: batch * pad_len exceeds the int32 token index");
        return ENERGON_ERR_INVALID_ARGUMENT;
    }
    int32_t* offsets = nullptr;
    cudaError_t e = scratch_address(&offsets);
    if (e != cudaSuccess) {
        record_error(ENERGON_ERR_CUDA, "remove_noalloc: cudaGetSymbolAddress of the offsets scratch failed");
        return ENERGON_ERR_CUDA;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    e = launch_offsets(lengths, batch, pad_len, offsets, d_status, st);
    if (e == cudaSuccess)
        e = launch_remove(padded, offsets, batch, pad_len, (int64_t)hidden * elem_bytes, packed,
                          (int64_t)batch * pad_len, d_status, st);
    if (e != cudaSuccess) {
        record_error(ENERGON_ERR_CUDA, cudaGetErrorString(e));
        return ENERGON_ERR_CUDA;
    }
    return ENERGON_OK;
}
