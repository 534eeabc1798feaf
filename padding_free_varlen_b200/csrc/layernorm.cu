// LayerNorm of the pre-LN GPT layer: y = (x - mean) / sqrt(var + eps) * g + b,
// biased variance, statistics in fp32, output rounded to the storage type.
// (The normalisation of the bias + residual + LayerNorm step in the QbitAI
// article's FasterTransformer excerpt, section "易用性", placed before each
// sub-layer as in GPT-2/3.)
//
// One thread block per row (grid-stride over the device-side row count).  For
// 16-bit rows of up to 16384 elements each thread keeps its slice in registers
// as 16-byte vectors, so the row is read from HBM once and written once.
//
// Gather form (transpose_padding_remove fused into the first LayerNorm): packed
// row r reads padded row (b, r - cu[b]) of a [batch, pad_len, H] tensor and also
// writes that raw row to `copy` (the packed residual stream), so the padded input
// is read once for both.
#include "common.cuh"
#include "internal.h"

namespace energon {

// Sum over the block; every thread gets the result.  `red` holds 32 floats.
__device__ __forceinline__ float block_sum(float v, float* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();  // red may still be read from a previous call
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = lane < nw ? red[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    return t;
}

// Source row of packed row r: itself, or (gather) padded row (b, r - cu[b]); -1 if
// the offsets put it outside the padded tensor.
__device__ __forceinline__ int64_t ln_src_row(const LnGather& gth, int r) {
    if (gth.cu == nullptr) return r;
    const int b = owner_of(gth.cu, gth.batch, r);
    const int64_t s = (int64_t)r - __ldg(gth.cu + b);
    return (s >= 0 && s < gth.pad_len) ? (int64_t)b * gth.pad_len + s : -1;
}

template <typename T>
__global__ void __launch_bounds__(256) ln_generic_kernel(const T* __restrict__ x, const T* __restrict__ g,
                                                         const T* __restrict__ bb, T* __restrict__ y,
                                                         const int32_t* d_rows, int rows_cap, int H, float eps,
                                                         const int32_t* status, LnGather gth) {
    __shared__ float red[32];
    if (status_bad(status)) return;
    const int rows = min(*d_rows, rows_cap);
    for (int r = blockIdx.x; r < rows; r += gridDim.x) {
        const int64_t src = ln_src_row(gth, r);
        if (src < 0) continue;
        const T* xr = x + src * H;
        if (gth.copy != nullptr) {
            T* cr = static_cast<T*>(gth.copy) + (int64_t)r * H;
            for (int k = threadIdx.x; k < H; k += blockDim.x) cr[k] = xr[k];
        }
        float s = 0.0f;
        for (int k = threadIdx.x; k < H; k += blockDim.x) s += to_f(xr[k]);
        const float mean = block_sum(s, red) / H;
        float q = 0.0f;
        for (int k = threadIdx.x; k < H; k += blockDim.x) {
            float d = to_f(xr[k]) - mean;
            q += d * d;
        }
        const float var = block_sum(q, red) / H;
        const float inv = 1.0f / sqrtf(var + eps);
        T* yr = y + (int64_t)r * H;
        for (int k = threadIdx.x; k < H; k += blockDim.x)
            yr[k] = from_f<T>((to_f(xr[k]) - mean) * inv * to_f(g[k]) + to_f(bb[k]));
    }
}

// 16-bit types, H % 8 == 0, H / 8 <= 256 * VPT, 16-byte aligned pointers.
template <typename T, int VPT>
__global__ void __launch_bounds__(256) ln_vec_kernel(const T* __restrict__ x, const T* __restrict__ g,
                                                     const T* __restrict__ bb, T* __restrict__ y,
                                                     const int32_t* d_rows, int rows_cap, int H, float eps,
                                                     const int32_t* status, LnGather gth) {
    __shared__ float red[32];
    if (status_bad(status)) return;
    const int rows = min(*d_rows, rows_cap);
    const int nvec = H / 8;
    uint4* copy = static_cast<uint4*>(gth.copy);
    for (int r = blockIdx.x; r < rows; r += gridDim.x) {
        const int64_t src = ln_src_row(gth, r);
        if (src < 0) continue;
        const uint4* xr = reinterpret_cast<const uint4*>(x + src * H);
        uint4 v[VPT];
        float s = 0.0f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int idx = i * blockDim.x + threadIdx.x;
            if (idx < nvec) {
                v[i] = xr[idx];
                if (copy != nullptr) copy[(int64_t)r * nvec + idx] = v[i];
                const uint32_t* w = reinterpret_cast<const uint32_t*>(&v[i]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float2 f = unpack2<T>(w[j]);
                    s += f.x + f.y;
                }
            }
        }
        const float mean = block_sum(s, red) / H;
        float q = 0.0f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int idx = i * blockDim.x + threadIdx.x;
            if (idx < nvec) {
                const uint32_t* w = reinterpret_cast<const uint32_t*>(&v[i]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float2 f = unpack2<T>(w[j]);
                    q += (f.x - mean) * (f.x - mean) + (f.y - mean) * (f.y - mean);
                }
            }
        }
        const float var = block_sum(q, red) / H;
        const float inv = 1.0f / sqrtf(var + eps);
        uint4* yr = reinterpret_cast<uint4*>(y + (int64_t)r * H);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int idx = i * blockDim.x + threadIdx.x;
            if (idx < nvec) {
                const uint4 gv = __ldg(reinterpret_cast<const uint4*>(g) + idx);
                const uint4 bv = __ldg(reinterpret_cast<const uint4*>(bb) + idx);
                const uint32_t* w = reinterpret_cast<const uint32_t*>(&v[i]);
                const uint32_t* gw = reinterpret_cast<const uint32_t*>(&gv);
                const uint32_t* bw = reinterpret_cast<const uint32_t*>(&bv);
                uint4 o;
                uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float2 f = unpack2<T>(w[j]), gf = unpack2<T>(gw[j]), bf = unpack2<T>(bw[j]);
                    ow[j] = pack2<T>((f.x - mean) * inv * gf.x + bf.x, (f.y - mean) * inv * gf.y + bf.y);
                }
                yr[idx] = o;
            }
        }
    }
}

// Blocks of `kernel` (256 threads) that fit on the GPU at once: the row loop then runs
// in a single wave of blocks instead of leaving a second wave to start late.
template <typename K>
static int resident_blocks(K kernel) {
    return device_cached((const void*)kernel, 1, [&] {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, 256, 0) != cudaSuccess || per_sm < 1) {
            (void)cudaGetLastError();
            per_sm = 1;
        }
        return per_sm * device_sm_count();
    });
}

static int ln_grid(int rows_cap, int resident) {
    return rows_cap < resident ? (rows_cap > 0 ? rows_cap : 1) : resident;
}

template <typename T>
static cudaError_t ln_dispatch(const void* x, const void* g, const void* b, void* y, const int32_t* d_rows,
                               int rows_cap, int H, float eps, const int32_t* status, const LnGather& gth,
                               cudaStream_t st) {
    const T *xp = (const T*)x, *gp = (const T*)g, *bp = (const T*)b;
    T* yp = (T*)y;
    const uintptr_t al = (uintptr_t)x | (uintptr_t)g | (uintptr_t)b | (uintptr_t)y | (uintptr_t)gth.copy;
    const int nvec = H / 8;
    const int vpt = (nvec + 255) / 256;
    if (sizeof(T) == 2 && H % 8 == 0 && al % 16 == 0 && vpt >= 1 && vpt <= 8) {
        switch (vpt) {
#define LN_CASE(V)                                                                                      \
    case V: {                                                                                           \
        const int resident = resident_blocks(ln_vec_kernel<T, V>);                                      \
        ln_vec_kernel<T, V><<<ln_grid(rows_cap, resident), 256, 0, st>>>(xp, gp, bp, yp, d_rows, rows_cap, H, \
                                                                         eps, status, gth);             \
        break;                                                                                          \
    }
            LN_CASE(1) LN_CASE(2) LN_CASE(3) LN_CASE(4) LN_CASE(5) LN_CASE(6) LN_CASE(7) LN_CASE(8)
#undef LN_CASE
        }
    } else {
        const int resident = resident_blocks(ln_generic_kernel<T>);
        ln_generic_kernel<T><<<ln_grid(rows_cap, resident), 256, 0, st>>>(xp, gp, bp, yp, d_rows, rows_cap, H, eps,
                                                                         status, gth);
    }
    return cudaGetLastError();
}

// The vector kernel only exists for 16-bit types; fp32 always takes the generic one.
template <>
cudaError_t ln_dispatch<float>(const void* x, const void* g, const void* b, void* y, const int32_t* d_rows,
                               int rows_cap, int H, float eps, const int32_t* status, const LnGather& gth,
                               cudaStream_t st) {
    const int resident = resident_blocks(ln_generic_kernel<float>);
    ln_generic_kernel<float><<<ln_grid(rows_cap, resident), 256, 0, st>>>(
        (const float*)x, (const float*)g, (const float*)b, (float*)y, d_rows, rows_cap, H, eps, status, gth);
    return cudaGetLastError();
}

cudaError_t launch_layernorm(int dtype, const void* x, const void* g, const void* b, void* y, const int32_t* d_rows,
                             int rows_cap, int H, float eps, const int32_t* status, cudaStream_t st,
                             const LnGather& gth) {
    switch (dtype) {
    case ENERGON_F32: return ln_dispatch<float>(x, g, b, y, d_rows, rows_cap, H, eps, status, gth, st);
    case ENERGON_F16: return ln_dispatch<__half>(x, g, b, y, d_rows, rows_cap, H, eps, status, gth, st);
    case ENERGON_BF16: return ln_dispatch<__nv_bfloat16>(x, g, b, y, d_rows, rows_cap, H, eps, status, gth, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace energon
