// LayerNorm of the pre-LN GPT layer: y = (x - mean) / sqrt(var + eps) * g + b,
// biased variance, statistics in fp32.  (The normalisation of the bias +
// residual + LayerNorm step in the QbitAI article's FasterTransformer excerpt,
// section "易用性", placed before each sub-layer as in GPT-2/3.)
//
// Two forms:
//  - ln_rows_kernel: the LayerNorm before the MLP.  Its input is the fp32
//    residual after attention, its output (the FFN1 operand) the storage type.
//    One thread block per row; each thread keeps its slice of the row in
//    registers, so the row is read from HBM once and written once.
//  - ln_fold_kernel: the LayerNorm before the QKV projection, folded into that
//    GEMM (one warp per row; the row is streamed, not kept; buffers of at most
//    512 rows take ln_fold_rows_kernel, a block per row with the row in
//    registers).  It writes u = x * g (rounded to the storage type: exact when
//    g is 1) and the row statistics (rstd, mean * rstd); the GEMM's epilogue finishes
//    LN(x) W^T + b = rstd (u W^T) - mean rstd c + d with c = W g, d = b + W beta
//    (ln_fold_weights_kernel).  The tensor cores then see the layer input
//    itself instead of a rounded normalisation of it, which the attention
//    scores that follow are sensitive to.
//    Gather form (transpose_padding_remove fused into the first LayerNorm):
//    packed row r reads padded row (b, r - cu[b]) of a [batch, pad_len, H]
//    tensor and also writes that raw row to `copy` (the packed residual stream),
//    so the padded input is read once for both.
//
// Row statistics use sums shifted by the row's first element, s1 = sum (x - x0)
// and s2 = sum (x - x0)^2 (one block reduction of the pair): mean = x0 + s1 / H,
// var = s2 / H - (s1 / H)^2.  The shift keeps the subtraction benign when the
// mean is large against the spread.
#include "common.cuh"
#include "internal.h"

namespace energon {

// N elements of T in one aligned vector (16 bytes for the vector paths).
template <typename T, int N>
struct alignas(N * sizeof(T)) Pack {
    T v[N];
};

template <typename T, int N>
__device__ __forceinline__ void load_f(const T* p, float* f) {
    const Pack<T, N> pk = *reinterpret_cast<const Pack<T, N>*>(p);
#pragma unroll
    for (int i = 0; i < N; ++i) f[i] = to_f(pk.v[i]);
}
template <typename T, int N>
__device__ __forceinline__ void load_f_ldg(const T* p, float* f) {
    Pack<T, N> pk;
    if constexpr (sizeof(Pack<T, N>) == 16) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(p));
        pk = *reinterpret_cast<const Pack<T, N>*>(&w);
    } else {
        pk = *reinterpret_cast<const Pack<T, N>*>(p);
    }
#pragma unroll
    for (int i = 0; i < N; ++i) f[i] = to_f(pk.v[i]);
}
template <typename T, int N>
__device__ __forceinline__ void store_f(T* p, const float* f) {
    Pack<T, N> pk;
#pragma unroll
    for (int i = 0; i < N; ++i) pk.v[i] = from_f<T>(f[i]);
    *reinterpret_cast<Pack<T, N>*>(p) = pk;
}

// Sum of a float pair over the block; every thread gets the result.  `red` holds 32 pairs.
__device__ __forceinline__ float2 block_sum2(float2 v, float2* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        v.x += __shfl_xor_sync(0xffffffffu, v.x, o);
        v.y += __shfl_xor_sync(0xffffffffu, v.y, o);
    }
    __syncthreads();  // red may still be read from the previous row
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float2 t = lane < nw ? red[lane] : make_float2(0.0f, 0.0f);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        t.x += __shfl_xor_sync(0xffffffffu, t.x, o);
        t.y += __shfl_xor_sync(0xffffffffu, t.y, o);
    }
    return t;
}

// (mean, 1 / sqrt(var + eps)) from the shifted sums of a row of H elements.
__device__ __forceinline__ float2 row_stats(float x0, float2 s, int H, float eps) {
    const float m1 = s.x / H;
    const float var = fmaxf(s.y / H - m1 * m1, 0.0f);
    return make_float2(x0 + m1, rsqrtf(var + eps));
}

// Source row of packed row r: itself, or (gather) padded row (b, r - cu[b]); -1 if
// the offsets put it outside the padded tensor.
__device__ __forceinline__ int64_t ln_src_row(const LnGather& gth, int r) {
    if (gth.cu == nullptr) return r;
    const int b = owner_of(gth.cu, gth.batch, r);
    const int64_t s = (int64_t)r - __ldg(gth.cu + b);
    return (s >= 0 && s < gth.pad_len) ? (int64_t)b * gth.pad_len + s : -1;
}

// ------------------------------------------------------------------ LayerNorm (row in registers)

// Tin: input element type (the storage type, or float for the fp32 residual), Tout: the
// storage type.  N = elements per 16-byte input vector; VPT vectors per thread (the row
// has H / N vectors, H % N == 0, at most 256 * VPT of them).
template <typename Tin, typename Tout, int VPT>
__global__ void __launch_bounds__(256) ln_rows_kernel(const Tin* __restrict__ x, const Tout* __restrict__ g,
                                                      const Tout* __restrict__ bb, Tout* __restrict__ y,
                                                      const int32_t* d_rows, int rows_cap, int H, float eps,
                                                      const int32_t* status) {
    constexpr int N = 16 / sizeof(Tin);
    __shared__ float2 red[32];
    if (status_bad(status)) return;
    const int rows = min(*d_rows, rows_cap);
    const int nvec = H / N;
    for (int r = blockIdx.x; r < rows; r += gridDim.x) {
        const Tin* xr = x + (int64_t)r * H;
        const float x0 = to_f(xr[0]);
        float f[VPT][N];
        float2 s = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int idx = i * blockDim.x + threadIdx.x;
            if (idx < nvec) {
                load_f<Tin, N>(xr + (int64_t)idx * N, f[i]);
#pragma unroll
                for (int j = 0; j < N; ++j) {
                    const float d = f[i][j] - x0;
                    s.x += d;
                    s.y = fmaf(d, d, s.y);
                }
            }
        }
        const float2 mi = row_stats(x0, block_sum2(s, red), H, eps);
        Tout* yr = y + (int64_t)r * H;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int idx = i * blockDim.x + threadIdx.x;
            if (idx < nvec) {
                float gv[N], bv[N], o[N];
                load_f_ldg<Tout, N>(g + (int64_t)idx * N, gv);
                load_f_ldg<Tout, N>(bb + (int64_t)idx * N, bv);
#pragma unroll
                for (int j = 0; j < N; ++j) o[j] = (f[i][j] - mi.x) * mi.y * gv[j] + bv[j];
                store_f<Tout, N>(yr + (int64_t)idx * N, o);
            }
        }
    }
}

// Any H, any alignment: three passes over the row (L1/L2 serve the repeats).
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) ln_rows_generic_kernel(const Tin* __restrict__ x, const Tout* __restrict__ g,
                                                              const Tout* __restrict__ bb, Tout* __restrict__ y,
                                                              const int32_t* d_rows, int rows_cap, int H, float eps,
                                                              const int32_t* status) {
    __shared__ float2 red[32];
    if (status_bad(status)) return;
    const int rows = min(*d_rows, rows_cap);
    for (int r = blockIdx.x; r < rows; r += gridDim.x) {
        const Tin* xr = x + (int64_t)r * H;
        const float x0 = to_f(xr[0]);
        float2 s = make_float2(0.0f, 0.0f);
        for (int k = threadIdx.x; k < H; k += blockDim.x) {
            const float d = to_f(xr[k]) - x0;
            s.x += d;
            s.y = fmaf(d, d, s.y);
        }
        const float2 mi = row_stats(x0, block_sum2(s, red), H, eps);
        Tout* yr = y + (int64_t)r * H;
        for (int k = threadIdx.x; k < H; k += blockDim.x)
            yr[k] = from_f<Tout>((to_f(xr[k]) - mi.x) * mi.y * to_f(g[k]) + to_f(bb[k]));
    }
}

// ------------------------------------------------------------------ LayerNorm folded into the GEMM

// u = x * g, stats = (rstd, mean * rstd); N elements per step (16-byte vectors when VEC).
// One warp per row (the row is streamed, nothing of it is kept), eight rows per block:
// every row of the batch is in flight at once, each lane with eight vectors outstanding,
// and the row statistics need only shuffles.
template <typename T, bool VEC>
__global__ void __launch_bounds__(256) ln_fold_kernel(const T* __restrict__ x, const T* __restrict__ g,
                                                      T* __restrict__ u, float2* __restrict__ stats,
                                                      const int32_t* d_rows, int rows_cap, int H, float eps,
                                                      const int32_t* status, LnGather gth) {
    constexpr int N = VEC ? 16 / sizeof(T) : 1;
    constexpr int U = 8;
    if (status_bad(status)) return;
    const int rows = min(*d_rows, rows_cap);
    const int nvec = H / N;
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    T* copy = static_cast<T*>(gth.copy);
    for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
        const int64_t src = ln_src_row(gth, r);
        if (src < 0) continue;
        const T* xr = x + src * H;
        T* ur = u + (int64_t)r * H;
        T* cr = copy ? copy + (int64_t)r * H : nullptr;
        const float x0 = to_f(xr[0]);
        float2 s = make_float2(0.0f, 0.0f);
        for (int base = lane; base < nvec; base += 32 * U) {
            Pack<T, N> xv[U];
#pragma unroll
            for (int k = 0; k < U; ++k) {
                const int idx = base + 32 * k;
                if (idx < nvec) xv[k] = *reinterpret_cast<const Pack<T, N>*>(xr + (int64_t)idx * N);
            }
#pragma unroll
            for (int k = 0; k < U; ++k) {
                const int idx = base + 32 * k;
                if (idx >= nvec) continue;
                const int64_t e = (int64_t)idx * N;
                if (cr) *reinterpret_cast<Pack<T, N>*>(cr + e) = xv[k];
                float gv[N], o[N];
                load_f_ldg<T, N>(g + e, gv);
#pragma unroll
                for (int j = 0; j < N; ++j) {
                    const float v = to_f(xv[k].v[j]);
                    const float d = v - x0;
                    s.x += d;
                    s.y = fmaf(d, d, s.y);
                    o[j] = v * gv[j];
                }
                store_f<T, N>(ur + e, o);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            s.x += __shfl_xor_sync(0xffffffffu, s.x, o);
            s.y += __shfl_xor_sync(0xffffffffu, s.y, o);
        }
        if (lane == 0) {
            const float2 mi = row_stats(x0, s, H, eps);
            stats[r] = make_float2(mi.y, mi.x * mi.y);
        }
    }
}

// The same outputs with one block of 256 threads per row and the row in registers, for
// batches of few rows: a warp streaming a 12288-element row alone waits on a chain of
// dependent loads (tens of microseconds at 32 rows), where a block has its whole row in
// flight at once.  VPT 16-byte vectors per thread (the row has H / N of them, at most
// 256 * VPT).
template <typename T, int VPT>
__global__ void __launch_bounds__(256) ln_fold_rows_kernel(const T* __restrict__ x, const T* __restrict__ g,
                                                           T* __restrict__ u, float2* __restrict__ stats,
                                                           const int32_t* d_rows, int rows_cap, int H, float eps,
                                                           const int32_t* status, LnGather gth) {
    constexpr int N = 16 / sizeof(T);
    __shared__ float2 red[32];
    if (status_bad(status)) return;
    const int rows = min(*d_rows, rows_cap);
    const int nvec = H / N;
    T* copy = static_cast<T*>(gth.copy);
    for (int r = blockIdx.x; r < rows; r += gridDim.x) {
        const int64_t src = ln_src_row(gth, r);
        if (src < 0) continue;  // the same for every thread of the block
        const T* xr = x + src * H;
        T* ur = u + (int64_t)r * H;
        T* cr = copy ? copy + (int64_t)r * H : nullptr;
        const float x0 = to_f(xr[0]);
        Pack<T, N> xv[VPT];
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int idx = i * blockDim.x + threadIdx.x;
            if (idx < nvec) xv[i] = *reinterpret_cast<const Pack<T, N>*>(xr + (int64_t)idx * N);
        }
        float2 s = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int idx = i * blockDim.x + threadIdx.x;
            if (idx >= nvec) continue;
            const int64_t e = (int64_t)idx * N;
            if (cr) *reinterpret_cast<Pack<T, N>*>(cr + e) = xv[i];
            float gv[N], o[N];
            load_f_ldg<T, N>(g + e, gv);
#pragma unroll
            for (int j = 0; j < N; ++j) {
                const float v = to_f(xv[i].v[j]);
                const float d = v - x0;
                s.x += d;
                s.y = fmaf(d, d, s.y);
                o[j] = v * gv[j];
            }
            store_f<T, N>(ur + e, o);
        }
        const float2 mi = row_stats(x0, block_sum2(s, red), H, eps);
        if (threadIdx.x == 0) stats[r] = make_float2(mi.y, mi.x * mi.y);
    }
}

// c[n] = sum_k g[k] W[n][k], d[n] = bias[n] + sum_k beta[k] W[n][k].  A block of 256
// threads owns RPB consecutive rows of W; thread t takes the 16-byte vectors t, t + 256,
// ... of every row, two vector steps at a time, so each thread has 2 * (RPB + 2) loads in
// flight (the weights stream from HBM once).  Per-thread partial sums, then a fixed
// shuffle tree and a fixed order across the warps (deterministic).
template <typename T, bool VEC, int RPB>
__global__ void __launch_bounds__(256) ln_fold_weights_kernel(const T* __restrict__ W, const T* __restrict__ g,
                                                              const T* __restrict__ beta, const T* __restrict__ bias,
                                                              int Nrows, int K, float* __restrict__ c,
                                                              float* __restrict__ d, const int32_t* status) {
    constexpr int N = VEC ? 16 / sizeof(T) : 1;
    __shared__ float red[8][2 * RPB];
    if (status_bad(status)) return;
    const int n0 = blockIdx.x * RPB;
    const int nvec = K / N;
    float ac[RPB], ad[RPB];
#pragma unroll
    for (int i = 0; i < RPB; ++i) ac[i] = ad[i] = 0.0f;
    for (int v0 = threadIdx.x; v0 < nvec; v0 += 2 * blockDim.x) {
        // raw vectors first (all loads in flight), converted while accumulating
        Pack<T, N> gp[2], bp[2], wp[2][RPB];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int v = v0 + u * blockDim.x;
            const int64_t e = (int64_t)(v < nvec ? v : 0) * N;
            gp[u] = *reinterpret_cast<const Pack<T, N>*>(g + e);
            bp[u] = *reinterpret_cast<const Pack<T, N>*>(beta + e);
#pragma unroll
            for (int i = 0; i < RPB; ++i)
                wp[u][i] = *reinterpret_cast<const Pack<T, N>*>(W + (int64_t)(n0 + i < Nrows ? n0 + i : n0) * K + e);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (v0 + u * (int)blockDim.x >= nvec) continue;
#pragma unroll
            for (int j = 0; j < N; ++j) {
                const float gj = to_f(gp[u].v[j]), bj = to_f(bp[u].v[j]);
#pragma unroll
                for (int i = 0; i < RPB; ++i) {
                    const float w = to_f(wp[u][i].v[j]);
                    ac[i] = fmaf(gj, w, ac[i]);
                    ad[i] = fmaf(bj, w, ad[i]);
                }
            }
        }
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int i = 0; i < RPB; ++i) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ac[i] += __shfl_xor_sync(0xffffffffu, ac[i], o);
            ad[i] += __shfl_xor_sync(0xffffffffu, ad[i], o);
        }
    }
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < RPB; ++i) red[warp][i] = ac[i], red[warp][RPB + i] = ad[i];
    }
    __syncthreads();
    if (threadIdx.x < 2 * RPB) {
        float s = 0.0f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w][threadIdx.x];
        const int i = threadIdx.x % RPB;
        if (n0 + i < Nrows) {
            if (threadIdx.x < RPB) c[n0 + i] = s;
            else d[n0 + i] = s + (bias ? to_f(bias[n0 + i]) : 0.0f);
        }
    }
}

// ------------------------------------------------------------------ host side

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

// Buffers of at most this many rows take the block-per-row form of the folded LayerNorm.
constexpr int LN_FOLD_BLOCK_ROWS = 512;

static int row_grid(int rows_cap, int resident) {
    return rows_cap < resident ? (rows_cap > 0 ? rows_cap : 1) : resident;
}

template <typename Tin, typename Tout, int VPT>
static void ln_rows_launch(const void* x, const void* g, const void* b, void* y, const int32_t* d_rows, int rows_cap,
                           int H, float eps, const int32_t* status, cudaStream_t st) {
    auto k = ln_rows_kernel<Tin, Tout, VPT>;
    k<<<row_grid(rows_cap, resident_blocks(k)), 256, 0, st>>>((const Tin*)x, (const Tout*)g, (const Tout*)b,
                                                              (Tout*)y, d_rows, rows_cap, H, eps, status);
}

template <typename Tin, typename Tout>
static cudaError_t ln_rows_dispatch(const void* x, const void* g, const void* b, void* y, const int32_t* d_rows,
                                    int rows_cap, int H, float eps, const int32_t* status, cudaStream_t st) {
    constexpr int N = 16 / sizeof(Tin);
    constexpr int NO = N;  // output elements per vector step (N * sizeof(Tout) bytes)
    const uintptr_t al = (uintptr_t)x | (uintptr_t)g | (uintptr_t)b | (uintptr_t)y;
    const int nvec = H / N;
    const int vpt = (nvec + 255) / 256;
    const bool vec = H % N == 0 && al % 16 == 0 && (NO * sizeof(Tout)) % 4 == 0 && vpt >= 1 && vpt <= 16;
    if (vec) {
        if (vpt <= 1) ln_rows_launch<Tin, Tout, 1>(x, g, b, y, d_rows, rows_cap, H, eps, status, st);
        else if (vpt <= 2) ln_rows_launch<Tin, Tout, 2>(x, g, b, y, d_rows, rows_cap, H, eps, status, st);
        else if (vpt <= 4) ln_rows_launch<Tin, Tout, 4>(x, g, b, y, d_rows, rows_cap, H, eps, status, st);
        else if (vpt <= 6) ln_rows_launch<Tin, Tout, 6>(x, g, b, y, d_rows, rows_cap, H, eps, status, st);
        else if (vpt <= 8) ln_rows_launch<Tin, Tout, 8>(x, g, b, y, d_rows, rows_cap, H, eps, status, st);
        else if (vpt <= 12) ln_rows_launch<Tin, Tout, 12>(x, g, b, y, d_rows, rows_cap, H, eps, status, st);
        else ln_rows_launch<Tin, Tout, 16>(x, g, b, y, d_rows, rows_cap, H, eps, status, st);
    } else {
        auto k = ln_rows_generic_kernel<Tin, Tout>;
        k<<<row_grid(rows_cap, resident_blocks(k)), 256, 0, st>>>((const Tin*)x, (const Tout*)g, (const Tout*)b,
                                                                  (Tout*)y, d_rows, rows_cap, H, eps, status);
    }
    return cudaGetLastError();
}

cudaError_t launch_layernorm(int dtype, const void* x, const void* g, const void* b, void* y, const int32_t* d_rows,
                             int rows_cap, int H, float eps, const int32_t* status, cudaStream_t st,
                             const LnGather& gth, bool x_f32) {
    if (gth.cu != nullptr) return cudaErrorInvalidValue;  // the gather form is the folded LayerNorm's
    switch (dtype) {
    case ENERGON_F32: return ln_rows_dispatch<float, float>(x, g, b, y, d_rows, rows_cap, H, eps, status, st);
    case ENERGON_F16:
        return x_f32 ? ln_rows_dispatch<float, __half>(x, g, b, y, d_rows, rows_cap, H, eps, status, st)
                     : ln_rows_dispatch<__half, __half>(x, g, b, y, d_rows, rows_cap, H, eps, status, st);
    case ENERGON_BF16:
        return x_f32 ? ln_rows_dispatch<float, __nv_bfloat16>(x, g, b, y, d_rows, rows_cap, H, eps, status, st)
                     : ln_rows_dispatch<__nv_bfloat16, __nv_bfloat16>(x, g, b, y, d_rows, rows_cap, H, eps, status,
                                                                       st);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
static cudaError_t ln_fold_dispatch(const void* x, const void* g, void* u, float2* stats, const int32_t* d_rows,
                                    int rows_cap, int H, float eps, const int32_t* status, const LnGather& gth,
                                    cudaStream_t st) {
    constexpr int N = 16 / sizeof(T);
    const uintptr_t al = (uintptr_t)x | (uintptr_t)g | (uintptr_t)u | (uintptr_t)gth.copy;
    const int vpt = (H / N + 255) / 256;
    if (H % N == 0 && al % 16 == 0 && rows_cap <= LN_FOLD_BLOCK_ROWS && vpt <= 8) {
        // few rows: a block per row
        auto launch = [&](auto k) {
            k<<<row_grid(rows_cap, resident_blocks(k)), 256, 0, st>>>((const T*)x, (const T*)g, (T*)u, stats, d_rows,
                                                                      rows_cap, H, eps, status, gth);
        };
        if (vpt <= 2) launch(ln_fold_rows_kernel<T, 2>);
        else if (vpt <= 4) launch(ln_fold_rows_kernel<T, 4>);
        else if (vpt <= 6) launch(ln_fold_rows_kernel<T, 6>);
        else launch(ln_fold_rows_kernel<T, 8>);
        return cudaGetLastError();
    }
    // eight rows (warps) per block, as many blocks as the rows need or the GPU holds
    const int row_blocks = (rows_cap + 7) / 8;
    if (H % N == 0 && al % 16 == 0) {
        auto k = ln_fold_kernel<T, true>;
        k<<<row_grid(row_blocks, resident_blocks(k)), 256, 0, st>>>((const T*)x, (const T*)g, (T*)u, stats, d_rows,
                                                                    rows_cap, H, eps, status, gth);
    } else {
        auto k = ln_fold_kernel<T, false>;
        k<<<row_grid(row_blocks, resident_blocks(k)), 256, 0, st>>>((const T*)x, (const T*)g, (T*)u, stats, d_rows,
                                                                    rows_cap, H, eps, status, gth);
    }
    return cudaGetLastError();
}

cudaError_t launch_ln_fold(int dtype, const void* x, const void* g, void* u, float2* stats, const int32_t* d_rows,
                           int rows_cap, int H, float eps, const int32_t* status, cudaStream_t st,
                           const LnGather& gth) {
    switch (dtype) {
    case ENERGON_F32: return ln_fold_dispatch<float>(x, g, u, stats, d_rows, rows_cap, H, eps, status, gth, st);
    case ENERGON_F16: return ln_fold_dispatch<__half>(x, g, u, stats, d_rows, rows_cap, H, eps, status, gth, st);
    case ENERGON_BF16:
        return ln_fold_dispatch<__nv_bfloat16>(x, g, u, stats, d_rows, rows_cap, H, eps, status, gth, st);
    }
    return cudaErrorInvalidValue;
}

template <typename T>
static cudaError_t fold_weights_dispatch(const void* W, const void* g, const void* beta, const void* bias, int Nr,
                                         int K, float* c, float* d, const int32_t* status, cudaStream_t st) {
    constexpr int N = 16 / sizeof(T), RPB = 8;
    const int blocks = (Nr + RPB - 1) / RPB;
    const uintptr_t al = (uintptr_t)W | (uintptr_t)g | (uintptr_t)beta;
    if (K % N == 0 && al % 16 == 0)
        ln_fold_weights_kernel<T, true, RPB><<<blocks, 256, 0, st>>>((const T*)W, (const T*)g, (const T*)beta,
                                                                    (const T*)bias, Nr, K, c, d, status);
    else
        ln_fold_weights_kernel<T, false, RPB><<<blocks, 256, 0, st>>>((const T*)W, (const T*)g, (const T*)beta,
                                                                     (const T*)bias, Nr, K, c, d, status);
    return cudaGetLastError();
}

cudaError_t launch_ln_fold_weights(int dtype, const void* W, const void* g, const void* beta, const void* bias,
                                   int N, int K, float* c, float* d, const int32_t* status, cudaStream_t st) {
    if (N <= 0 || K <= 0) return cudaSuccess;
    switch (dtype) {
    case ENERGON_F32: return fold_weights_dispatch<float>(W, g, beta, bias, N, K, c, d, status, st);
    case ENERGON_F16: return fold_weights_dispatch<__half>(W, g, beta, bias, N, K, c, d, status, st);
    case ENERGON_BF16: return fold_weights_dispatch<__nv_bfloat16>(W, g, beta, bias, N, K, c, d, status, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace energon
