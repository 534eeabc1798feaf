// Causal self-attention on packed tokens, driven by cu_seqlens.
//
// For sequence b (packed rows cu[b] .. cu[b+1]-1), head j and position s:
//     o_j(s) = sum_{t <= s} softmax_t(q_j(s) . k_j(t) / sqrt(d)) v_j(t)
// with q, k, v read from the fused projection qkv [rows, 3H] (columns Q | K | V,
// head-major inside each); when the low halves qk_lo [rows, 2H] are given, q and
// k are hi + lo.  Keys never cross a sequence boundary, so padding
// and other sequences never enter: this is what lets the layer run on the
// packed tokens only (EnergonAI README, "Scaling Ability": redundant
// computation elimination in the GPT-3 layers).
//
// CUDA-core kernel (fp32, head_dim 64; the 16-bit head_dim-128 case runs on the
// tensor cores, attention_tc.cu): one block per (64-query tile, head, sequence), 8 warps,
// each warp owning 8 queries; keys and values are staged through shared
// memory 64 at a time and combined with an online (running-max) softmax in
// fp32.  Key chunks beyond a query are fully masked and leave its state
// bit-for-bit unchanged, so a query's result does not depend on how many
// chunks its block visits (packed and padded runs agree exactly).
#include <float.h>

#include "common.cuh"
#include "internal.h"

namespace energon {

namespace {
constexpr int AQB = 64;  // queries per block
constexpr int AKB = 64;  // keys per shared-memory chunk
constexpr int ANW = 8;   // warps per block
}

template <int HD>
constexpr int attn_smem_bytes() {
    return (AQB * HD + AKB * (HD + 1) + AKB * HD) * (int)sizeof(float);
}

template <typename T, int HD>
__global__ void __launch_bounds__(256) attn_simt_kernel(const T* __restrict__ qkv, const T* __restrict__ qk_lo,
                                                        T* __restrict__ out, const int32_t* __restrict__ cu, int H,
                                                        float scale, const int32_t* status) {
    constexpr int QPW = AQB / ANW;  // queries per warp
    constexpr int DPL = HD / 32;    // output dims per lane
    extern __shared__ float smem[];
    float* Qs = smem;                    // [AQB][HD]
    float* Ks = Qs + AQB * HD;           // [AKB][HD + 1]
    float* Vs = Ks + AKB * (HD + 1);     // [AKB][HD]
    if (status_bad(status)) return;

    const int b = blockIdx.z, j = blockIdx.y;
    const int start = cu[b], len = cu[b + 1] - start;
    const int q0 = blockIdx.x * AQB;
    if (q0 >= len) return;
    const int q_end = min(q0 + AQB, len);
    const int64_t ld = 3 * (int64_t)H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    const int64_t ldl = 2 * (int64_t)H;  // qk_lo: the low halves of Q | K (q = hi + lo)
    for (int e = tid; e < AQB * HD; e += blockDim.x) {
        const int r = e / HD, d = e % HD;
        float qv = 0.0f;
        if (q0 + r < q_end) {
            const int64_t row = start + q0 + r;
            qv = to_f(qkv[row * ld + (int64_t)j * HD + d]);
            if (qk_lo) qv += to_f(qk_lo[row * ldl + (int64_t)j * HD + d]);
        }
        Qs[e] = qv;
    }

    float m[QPW], l[QPW], acc[QPW][DPL];
#pragma unroll
    for (int qi = 0; qi < QPW; ++qi) {
        m[qi] = -INFINITY;
        l[qi] = 0.0f;
#pragma unroll
        for (int d = 0; d < DPL; ++d) acc[qi][d] = 0.0f;
    }

    for (int kc0 = 0; kc0 < q_end; kc0 += AKB) {
        const int kn = min(AKB, q_end - kc0);
        __syncthreads();
        for (int e = tid; e < AKB * HD; e += blockDim.x) {
            const int t = e / HD, d = e % HD;
            float kv = 0.0f, vv = 0.0f;
            if (t < kn) {
                const int64_t tok = start + kc0 + t;
                const int64_t row = tok * ld + (int64_t)j * HD + d;
                kv = to_f(qkv[row + H]);
                if (qk_lo) kv += to_f(qk_lo[tok * ldl + H + (int64_t)j * HD + d]);
                vv = to_f(qkv[row + 2 * (int64_t)H]);
            }
            Ks[t * (HD + 1) + d] = kv;
            Vs[t * HD + d] = vv;
        }
        __syncthreads();
#pragma unroll
        for (int qi = 0; qi < QPW; ++qi) {
            const int r = qi * ANW + warp;  // query row inside the block
            const int s = q0 + r;           // position inside the sequence
            if (s >= q_end) continue;
            float sc[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int t = lane + 32 * h;
                if (t < kn && kc0 + t <= s) {
                    float dot = 0.0f;
                    const float* qr = Qs + r * HD;
                    const float* kr = Ks + t * (HD + 1);
#pragma unroll 16
                    for (int d = 0; d < HD; ++d) dot = fmaf(qr[d], kr[d], dot);
                    sc[h] = dot * scale;
                } else {
                    sc[h] = -INFINITY;
                }
            }
            float mx = fmaxf(sc[0], sc[1]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float m_new = fmaxf(m[qi], mx);
            const float p0 = expf(sc[0] - m_new), p1 = expf(sc[1] - m_new);
            const float corr = expf(m[qi] - m_new);
            float ps = p0 + p1;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
            l[qi] = l[qi] * corr + ps;
#pragma unroll
            for (int d = 0; d < DPL; ++d) acc[qi][d] *= corr;
            const int tmax = min(kn, s - kc0 + 1);
            for (int t = 0; t < tmax; ++t) {
                const float pt = __shfl_sync(0xffffffffu, t < 32 ? p0 : p1, t & 31);
                const float* vr = Vs + t * HD + lane * DPL;
#pragma unroll
                for (int d = 0; d < DPL; ++d) acc[qi][d] = fmaf(pt, vr[d], acc[qi][d]);
            }
            m[qi] = m_new;
        }
    }
#pragma unroll
    for (int qi = 0; qi < QPW; ++qi) {
        const int s = q0 + qi * ANW + warp;
        if (s >= q_end) continue;
        const float inv = 1.0f / l[qi];
        T* orow = out + (int64_t)(start + s) * H + (int64_t)j * HD + lane * DPL;
#pragma unroll
        for (int d = 0; d < DPL; ++d) orow[d] = from_f<T>(acc[qi][d] * inv);
    }
}

template <typename T, int HD>
static cudaError_t attn_launch(const void* qkv, const void* qk_lo, void* o, const int32_t* cu, int batch,
                               int max_len, int H, int n_heads, const int32_t* status, cudaStream_t st) {
    constexpr int smem = attn_smem_bytes<HD>();
    cudaError_t e = prepare_smem((const void*)attn_simt_kernel<T, HD>, smem);
    if (e != cudaSuccess) return e;
    dim3 grid((max_len + AQB - 1) / AQB, n_heads, batch);
    const float scale = (float)(1.0 / sqrt((double)HD));
    attn_simt_kernel<T, HD><<<grid, 256, smem, st>>>((const T*)qkv, (const T*)qk_lo, (T*)o, cu, H, scale, status);
    return cudaGetLastError();
}

cudaError_t launch_attention(int dtype, const void* qkv, const void* qk_lo, void* o, const int32_t* cu, int batch,
                             int max_len, int H, int n_heads, int qkv_rows, int32_t* status, uint64_t timeout_ns,
                             cudaStream_t st) {
    if (batch <= 0 || max_len <= 0) return cudaSuccess;
    if (attention_tc_supported(dtype, H, n_heads, qkv, qk_lo, o, qkv_rows))
        return launch_attention_tc(dtype, qkv, qk_lo, o, cu, batch, max_len, H, n_heads, qkv_rows, status, timeout_ns,
                                   st);
    const int hd = H / n_heads;
    if (hd != 64 && hd != 128) return cudaErrorInvalidValue;
#define ATTN_CASE(T)                                                                                     \
    return hd == 64 ? attn_launch<T, 64>(qkv, qk_lo, o, cu, batch, max_len, H, n_heads, status, st)     \
                    : attn_launch<T, 128>(qkv, qk_lo, o, cu, batch, max_len, H, n_heads, status, st);
    switch (dtype) {
    case ENERGON_F32: ATTN_CASE(float)
    case ENERGON_F16: ATTN_CASE(__half)
    case ENERGON_BF16: ATTN_CASE(__nv_bfloat16)
    }
#undef ATTN_CASE
    return cudaErrorInvalidValue;
}

}  // namespace energon
