// Offsets, transpose_padding_remove and transpose_padding_rebuild.
//
// QbitAI article "最新大模型推理系统Energon-AI开源", section "Runtime": the
// two operators pack the valid tokens of a variable-length batch so that the
// layers skip the padding, and scatter the result back afterwards.  The
// packing is driven by the exclusive prefix sum of the per-sequence lengths.
//
// All three are HBM-bound (or launch-bound) byte movement: no tensor cores.
// remove/rebuild move 16-byte vectors when the row size and both base
// pointers allow it, one warp per row, grid-stride over rows; the grid is a
// multiple of the SM count so every SM keeps several rows in flight.
#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "internal.h"

namespace energon {

int device_cached(const void* key, int what, const std::function<int()>& compute) {
    static std::mutex mu;
    static std::map<std::tuple<int, const void*, int>, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        dev = -1;
    }
    const auto k = std::make_tuple(dev, key, what);
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find(k);
        if (it != cache.end()) return it->second;
    }
    // Computed without the lock (compute may itself ask the cache, e.g. for the SM count);
    // two threads may both compute it once, the first stored value wins.
    const int v = compute();
    std::lock_guard<std::mutex> lock(mu);
    return cache.emplace(k, v).first->second;
}

cudaError_t prepare_smem(const void* kernel, int bytes) {
    return (cudaError_t)device_cached(kernel, 0, [&] {
        return (int)cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    });
}

int device_sm_count() {
    static const int tag = 0;
    return device_cached(&tag, 0, [] {
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
            (void)cudaGetLastError();
            sms = 148;
        }
        return sms;
    });
}

// ------------------------------------------------------------------ offsets

__global__ void __launch_bounds__(1024) offsets_kernel(const int32_t* __restrict__ lengths, int batch, int pad_len,
                                                      int32_t* __restrict__ cu, int32_t* __restrict__ status) {
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t carry;
    __shared__ int32_t bad;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    if (tid == 0) {
        carry = 0;
        bad = 0;
        cu[0] = 0;
    }
    __syncthreads();
    for (int base = 0; base < batch; base += blockDim.x) {
        const int b = base + tid;
        const int32_t v = b < batch ? lengths[b] : 0;
        if (b < batch && (v < 0 || v > pad_len)) bad = 1;
        // inclusive scan inside the warp
        int32_t x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_tot[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int32_t w = lane < nwarps ? warp_tot[lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int32_t y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            warp_tot[lane] = w;  // inclusive totals of warps 0..lane
        }
        __syncthreads();
        const int32_t incl = carry + (warp > 0 ? warp_tot[warp - 1] : 0) + x;
        if (b < batch) cu[b + 1] = incl;
        __syncthreads();
        if (tid == blockDim.x - 1) carry = incl;
        __syncthreads();
    }
    if (bad) {
        for (int b = tid; b <= batch; b += blockDim.x) cu[b] = 0;
    }
    if (tid == 0) *status = bad ? ENERGON_DEVICE_BAD_LENGTH : ENERGON_DEVICE_OK;
}

cudaError_t kernel_binary_version(int* version) {
    cudaFuncAttributes a;
    cudaError_t e = cudaFuncGetAttributes(&a, offsets_kernel);
    if (e == cudaSuccess) *version = a.binaryVersion;
    return e;
}

cudaError_t launch_offsets(const int32_t* lengths, int batch, int pad_len, int32_t* cu, int32_t* status,
                           cudaStream_t st) {
    int threads = batch >= 1024 ? 1024 : ((batch + 31) / 32) * 32;
    if (threads < 32) threads = 32;
    offsets_kernel<<<1, threads, 0, st>>>(lengths, batch, pad_len, cu, status);
    return cudaGetLastError();
}

__global__ void padded_starts_kernel(int batch, int pad_len, int32_t* cu_pad) {
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b <= batch; b += gridDim.x * blockDim.x)
        cu_pad[b] = b * pad_len;
}

cudaError_t launch_padded_starts(int batch, int pad_len, int32_t* cu_pad, const int32_t*, cudaStream_t st) {
    int blocks = (batch + 1 + 255) / 256;
    padded_starts_kernel<<<blocks, 256, 0, st>>>(batch, pad_len, cu_pad);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ remove / rebuild

template <typename V, int UNROLL>
__device__ __forceinline__ void warp_copy_row(const V* __restrict__ src, V* __restrict__ dst, int64_t nvec, int lane) {
    for (int64_t base = lane; base < nvec; base += 32 * UNROLL) {
        V tmp[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            int64_t i = base + (int64_t)u * 32;
            if (i < nvec) tmp[u] = __ldcs(src + i);
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            int64_t i = base + (int64_t)u * 32;
            if (i < nvec) dst[i] = tmp[u];
        }
    }
}

template <typename V>
__device__ __forceinline__ void warp_zero_row(V* __restrict__ dst, int64_t nvec, int lane) {
    V z;
    memset(&z, 0, sizeof(V));
    for (int64_t i = lane; i < nvec; i += 32) __stcs(dst + i, z);
}

template <typename V, int UNROLL>
__global__ void __launch_bounds__(256) remove_kernel(const V* __restrict__ padded, const int32_t* __restrict__ cu,
                                                     int batch, int pad_len, int64_t row_vecs, V* __restrict__ packed,
                                                     int64_t packed_rows_cap, const int32_t* status) {
    if (status_bad(status) || batch <= 0) return;
    int64_t T = __ldg(cu + batch);
    const int64_t cap = (int64_t)batch * pad_len;
    if (T > cap) T = cap;
    if (T > packed_rows_cap) T = packed_rows_cap;
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < T; r += warps) {
        const int b = owner_of(cu, batch, r);
        const int64_t s = r - __ldg(cu + b);
        if (s < 0 || s >= pad_len) continue;  // offsets inconsistent with pad_len: skip the row
        warp_copy_row<V, UNROLL>(padded + ((int64_t)b * pad_len + s) * row_vecs, packed + r * row_vecs, row_vecs,
                                 lane);
    }
}

template <typename V, int UNROLL>
__global__ void __launch_bounds__(256) rebuild_kernel(const V* __restrict__ packed, const int32_t* __restrict__ starts,
                                                      const int32_t* __restrict__ lens_cu, int batch, int pad_len,
                                                      int64_t row_vecs, int64_t packed_rows_cap, V* __restrict__ padded) {
    const int lane = threadIdx.x & 31;
    const int64_t rows = (int64_t)batch * pad_len;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const int b = (int)(r / pad_len);
        const int s = (int)(r - (int64_t)b * pad_len);
        const int len = __ldg(lens_cu + b + 1) - __ldg(lens_cu + b);
        const int64_t src = (int64_t)__ldg(starts + b) + s;
        V* dst = padded + r * row_vecs;
        if (s < len && src >= 0 && src < packed_rows_cap)
            warp_copy_row<V, UNROLL>(packed + src * row_vecs, dst, row_vecs, lane);
        else
            warp_zero_row<V>(dst, row_vecs, lane);
    }
}

static int row_grid(int64_t rows) {
    const int64_t per_sm = 8;  // 8 blocks of 8 warps = 64 warps per SM
    int64_t want = (rows + 7) / 8;
    int64_t cap = per_sm * device_sm_count();
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    return (int)want;
}

cudaError_t launch_remove(const void* padded, const int32_t* cu, int batch, int pad_len, int64_t row_bytes,
                          void* packed, int64_t packed_rows_cap, const int32_t* status, cudaStream_t st) {
    if (batch <= 0 || row_bytes == 0) return cudaSuccess;
    const int grid = row_grid((int64_t)batch * pad_len);
    const uintptr_t align = reinterpret_cast<uintptr_t>(padded) | reinterpret_cast<uintptr_t>(packed);
    if (row_bytes % 16 == 0 && align % 16 == 0) {
        remove_kernel<uint4, 4><<<grid, 256, 0, st>>>((const uint4*)padded, cu, batch, pad_len, row_bytes / 16,
                                                      (uint4*)packed, packed_rows_cap, status);
    } else if (row_bytes % 4 == 0 && align % 4 == 0) {
        remove_kernel<uint32_t, 8><<<grid, 256, 0, st>>>((const uint32_t*)padded, cu, batch, pad_len, row_bytes / 4,
                                                         (uint32_t*)packed, packed_rows_cap, status);
    } else {
        remove_kernel<uint8_t, 8><<<grid, 256, 0, st>>>((const uint8_t*)padded, cu, batch, pad_len, row_bytes,
                                                        (uint8_t*)packed, packed_rows_cap, status);
    }
    return cudaGetLastError();
}

cudaError_t launch_rebuild(const void* packed, const int32_t* starts, const int32_t* lens_cu, int batch, int pad_len,
                           int64_t row_bytes, int64_t packed_rows_cap, void* padded, cudaStream_t st) {
    if (batch <= 0 || pad_len <= 0 || row_bytes == 0) return cudaSuccess;
    const int grid = row_grid((int64_t)batch * pad_len);
    const uintptr_t align = reinterpret_cast<uintptr_t>(padded) | reinterpret_cast<uintptr_t>(packed);
    if (row_bytes % 16 == 0 && align % 16 == 0) {
        rebuild_kernel<uint4, 4><<<grid, 256, 0, st>>>((const uint4*)packed, starts, lens_cu, batch, pad_len,
                                                       row_bytes / 16, packed_rows_cap, (uint4*)padded);
    } else if (row_bytes % 4 == 0 && align % 4 == 0) {
        rebuild_kernel<uint32_t, 8><<<grid, 256, 0, st>>>((const uint32_t*)packed, starts, lens_cu, batch, pad_len,
                                                          row_bytes / 4, packed_rows_cap, (uint32_t*)padded);
    } else {
        rebuild_kernel<uint8_t, 8><<<grid, 256, 0, st>>>((const uint8_t*)packed, starts, lens_cu, batch, pad_len,
                                                         row_bytes, packed_rows_cap, (uint8_t*)padded);
    }
    return cudaGetLastError();
}

// Zero the pad rows (s >= len_b) of a padded [batch, pad_len] tensor; valid rows untouched.
// The pad rows of one sequence are one contiguous byte range, so blocks (blockIdx.y: the
// sequence, grid-strided) sweep that range with consecutive 16-byte stores.
// Each thread keeps four independent 16-byte stores in flight per step.
template <typename V>
__global__ void __launch_bounds__(256) zero_pads_kernel(const int32_t* __restrict__ cu, int batch, int pad_len,
                                                        int64_t row_vecs, V* __restrict__ padded) {
    V z;
    memset(&z, 0, sizeof(V));
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int b = blockIdx.y; b < batch; b += gridDim.y) {
        int len = __ldg(cu + b + 1) - __ldg(cu + b);
        len = len < 0 ? 0 : (len > pad_len ? pad_len : len);
        V* dst = padded + ((int64_t)b * pad_len + len) * row_vecs;
        const int64_t n = (int64_t)(pad_len - len) * row_vecs;
        int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
        for (; i + 3 * stride < n; i += 4 * stride) {
            __stcs(dst + i, z);
            __stcs(dst + i + stride, z);
            __stcs(dst + i + 2 * stride, z);
            __stcs(dst + i + 3 * stride, z);
        }
        for (; i < n; i += stride) __stcs(dst + i, z);
    }
}

cudaError_t launch_zero_pads(const int32_t* cu, int batch, int pad_len, int64_t row_bytes, void* padded,
                             cudaStream_t st) {
    if (batch <= 0 || pad_len <= 0 || row_bytes == 0) return cudaSuccess;
    const int gy = batch < 65535 ? batch : 65535;
    int gx = (8 * device_sm_count() + gy - 1) / gy;  // about eight blocks per SM in all
    if (gx < 1) gx = 1;
    const dim3 grid(gx, gy);
    if (row_bytes % 16 == 0 && reinterpret_cast<uintptr_t>(padded) % 16 == 0)
        zero_pads_kernel<uint4><<<grid, 256, 0, st>>>(cu, batch, pad_len, row_bytes / 16, (uint4*)padded);
    else if (row_bytes % 4 == 0 && reinterpret_cast<uintptr_t>(padded) % 4 == 0)
        zero_pads_kernel<uint32_t><<<grid, 256, 0, st>>>(cu, batch, pad_len, row_bytes / 4, (uint32_t*)padded);
    else
        zero_pads_kernel<uint8_t><<<grid, 256, 0, st>>>(cu, batch, pad_len, row_bytes, (uint8_t*)padded);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ head-transposing forms
//
// A packed token row holds `parts` blocks of n_heads heads of head_vecs vectors;
// the head-major padded tensor is [parts][batch][n_heads][pad_len][head_vecs].
// One warp per row (a padded position for rebuild, a packed token for remove):
// consecutive lanes walk the packed row, so its reads (rebuild) or writes
// (remove) are contiguous, and each head's run of head_vecs vectors lands in one
// contiguous segment of the head-major tensor.

struct HeadMap {
    int n_heads, head_vecs, row_vecs;  // row_vecs = parts * n_heads * head_vecs
    int batch, pad_len;
    int step_blk, step_j;              // 32 vectors = step_blk whole heads + step_j vectors
};

// Walks the vectors lane, lane + 32, lane + 64, ... of one packed row and keeps
// their head coordinates (block c, head h, vector j) up to date by addition, so
// the per-vector cost is a few integer adds instead of two divisions.
struct HeadCursor {
    int c, h, j;
    __device__ __forceinline__ HeadCursor(const HeadMap& m, int lane) {
        const int blk = lane / m.head_vecs;
        j = lane - blk * m.head_vecs;
        c = blk / m.n_heads;
        h = blk - c * m.n_heads;
    }
    __device__ __forceinline__ void advance(const HeadMap& m) {
        j += m.step_j;
        int dh = m.step_blk;
        if (j >= m.head_vecs) j -= m.head_vecs, ++dh;
        h += dh;
        while (h >= m.n_heads) h -= m.n_heads, ++c;  // at most step_blk / n_heads + 1 turns
    }
    // head-major offset (in vectors) of this vector at position (b, s)
    __device__ __forceinline__ int64_t offset(const HeadMap& m, int b, int s) const {
        return ((((int64_t)c * m.batch + b) * m.n_heads + h) * m.pad_len + s) * m.head_vecs + j;
    }
};

template <typename V, int UNROLL>
__global__ void __launch_bounds__(256) transpose_rebuild_kernel(const V* __restrict__ packed,
                                                                const int32_t* __restrict__ cu, HeadMap m,
                                                                int64_t packed_rows_cap, V* __restrict__ heads) {
    const int lane = threadIdx.x & 31;
    const int64_t rows = (int64_t)m.batch * m.pad_len;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    V z;
    memset(&z, 0, sizeof(V));
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const int b = (int)(r / m.pad_len);
        const int s = (int)(r - (int64_t)b * m.pad_len);
        const int len = __ldg(cu + b + 1) - __ldg(cu + b);
        const int64_t src = (int64_t)__ldg(cu + b) + s;
        const bool valid = s < len && src >= 0 && src < packed_rows_cap;
        const V* row = packed + (valid ? src : 0) * m.row_vecs;
        HeadCursor cur(m, lane);
        for (int base = lane; base < m.row_vecs; base += 32 * UNROLL) {
            V tmp[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int v = base + u * 32;
                tmp[u] = (valid && v < m.row_vecs) ? __ldcs(row + v) : z;
            }
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                if (base + u * 32 < m.row_vecs) __stcs(heads + cur.offset(m, b, s), tmp[u]);
                cur.advance(m);
            }
        }
    }
}

template <typename V, int UNROLL>
__global__ void __launch_bounds__(256) transpose_remove_kernel(const V* __restrict__ heads,
                                                               const int32_t* __restrict__ cu, HeadMap m,
                                                               int64_t packed_rows_cap, V* __restrict__ packed) {
    if (m.batch <= 0) return;
    int64_t T = __ldg(cu + m.batch);
    const int64_t cap = (int64_t)m.batch * m.pad_len;
    if (T > cap) T = cap;
    if (T > packed_rows_cap) T = packed_rows_cap;
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < T; r += warps) {
        const int b = owner_of(cu, m.batch, r);
        const int64_t s = r - __ldg(cu + b);
        if (s < 0 || s >= m.pad_len) continue;  // offsets inconsistent with pad_len: skip the row
        V* row = packed + r * m.row_vecs;
        HeadCursor cur(m, lane);
        for (int base = lane; base < m.row_vecs; base += 32 * UNROLL) {
            V tmp[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                if (base + u * 32 < m.row_vecs) tmp[u] = __ldcs(heads + cur.offset(m, b, (int)s));
                cur.advance(m);
            }
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int v = base + u * 32;
                if (v < m.row_vecs) row[v] = tmp[u];
            }
        }
    }
}

template <typename V>
static HeadMap head_map(int batch, int pad_len, int parts, int n_heads, int64_t head_bytes) {
    HeadMap m;
    m.n_heads = n_heads;
    m.head_vecs = (int)(head_bytes / (int64_t)sizeof(V));
    m.row_vecs = parts * n_heads * m.head_vecs;
    m.batch = batch;
    m.pad_len = pad_len;
    m.step_blk = 32 / m.head_vecs;
    m.step_j = 32 - m.step_blk * m.head_vecs;
    return m;
}

cudaError_t launch_transpose_rebuild(const void* packed, const int32_t* cu, int batch, int pad_len, int parts,
                                     int n_heads, int64_t head_bytes, int64_t packed_rows_cap, void* heads,
                                     cudaStream_t st) {
    if (batch <= 0 || pad_len <= 0 || head_bytes == 0) return cudaSuccess;
    const int grid = row_grid((int64_t)batch * pad_len);
    const uintptr_t align = reinterpret_cast<uintptr_t>(packed) | reinterpret_cast<uintptr_t>(heads);
    if (head_bytes % 16 == 0 && align % 16 == 0) {
        transpose_rebuild_kernel<uint4, 4><<<grid, 256, 0, st>>>(
            (const uint4*)packed, cu, head_map<uint4>(batch, pad_len, parts, n_heads, head_bytes), packed_rows_cap,
            (uint4*)heads);
    } else if (head_bytes % 4 == 0 && align % 4 == 0) {
        transpose_rebuild_kernel<uint32_t, 8><<<grid, 256, 0, st>>>(
            (const uint32_t*)packed, cu, head_map<uint32_t>(batch, pad_len, parts, n_heads, head_bytes),
            packed_rows_cap, (uint32_t*)heads);
    } else {
        transpose_rebuild_kernel<uint8_t, 8><<<grid, 256, 0, st>>>(
            (const uint8_t*)packed, cu, head_map<uint8_t>(batch, pad_len, parts, n_heads, head_bytes),
            packed_rows_cap, (uint8_t*)heads);
    }
    return cudaGetLastError();
}

cudaError_t launch_transpose_remove(const void* heads, const int32_t* cu, int batch, int pad_len, int parts,
                                    int n_heads, int64_t head_bytes, int64_t packed_rows_cap, void* packed,
                                    cudaStream_t st) {
    if (batch <= 0 || head_bytes == 0) return cudaSuccess;
    const int grid = row_grid((int64_t)batch * pad_len);
    const uintptr_t align = reinterpret_cast<uintptr_t>(packed) | reinterpret_cast<uintptr_t>(heads);
    if (head_bytes % 16 == 0 && align % 16 == 0) {
        transpose_remove_kernel<uint4, 4><<<grid, 256, 0, st>>>(
            (const uint4*)heads, cu, head_map<uint4>(batch, pad_len, parts, n_heads, head_bytes), packed_rows_cap,
            (uint4*)packed);
    } else if (head_bytes % 4 == 0 && align % 4 == 0) {
        transpose_remove_kernel<uint32_t, 8><<<grid, 256, 0, st>>>(
            (const uint32_t*)heads, cu, head_map<uint32_t>(batch, pad_len, parts, n_heads, head_bytes),
            packed_rows_cap, (uint32_t*)packed);
    } else {
        transpose_remove_kernel<uint8_t, 8><<<grid, 256, 0, st>>>(
            (const uint8_t*)heads, cu, head_map<uint8_t>(batch, pad_len, parts, n_heads, head_bytes),
            packed_rows_cap, (uint8_t*)packed);
    }
    return cudaGetLastError();
}

// ------------------------------------------------------------------ bounded-wait self-test

__global__ void wait_selftest_kernel(int32_t* status, uint64_t timeout_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // Nobody arrives on `bar`: the wait must give up by itself.
        if (!mbar_wait_bounded(&bar, 0, nullptr, timeout_ns)) status_or(status, ENERGON_DEVICE_TIMEOUT);
    }
    __syncthreads();
}

cudaError_t launch_wait_selftest(int32_t* status, uint64_t timeout_ns, cudaStream_t st) {
    wait_selftest_kernel<<<1, 32, 0, st>>>(status, timeout_ns);
    return cudaGetLastError();
}

}  // namespace energon
