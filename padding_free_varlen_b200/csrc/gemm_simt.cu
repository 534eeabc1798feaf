// CUDA-core GEMM y = A W^T + epilogue for the fp32 layer and for shapes the
// tcgen05 kernel does not take.  64 x 64 output tile per 256-thread block,
// 4 x 4 outputs per thread, K staged through shared memory in steps of 16.
// Same epilogue semantics as the tensor-core kernel (the Epilogue enum): fp32
// accumulate, then the folded LayerNorm or bias, optional GELU, optional
// residual, one rounding to the output type.  The valid row count is read on
// the device.
#include "common.cuh"
#include "internal.h"

namespace energon {

namespace {
constexpr int SBM = 64, SBN = 64, SBK = 16;
}

template <typename T, int EPI>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const T* __restrict__ A, const T* __restrict__ W,
                                                        const GemmArgs a) {
    __shared__ float As[SBK][SBM + 4];
    __shared__ float Ws[SBK][SBN + 4];
    if (status_bad(a.status)) return;
    const int M = min(*a.d_rows, a.M_cap);
    const int N = a.N, K = a.K;
    const int m0 = blockIdx.y * SBM, n0 = blockIdx.x * SBN;
    if (m0 >= M) return;
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += SBK) {
        // 64 x 16 tiles of A and W: 1024 elements each, 4 per thread.
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = tid + i * 256;
            const int r = e / SBK, k = e % SBK;
            const int gk = k0 + k;
            const int gm = m0 + r, gn = n0 + r;
            As[k][r] = (gm < M && gk < K) ? to_f(A[(int64_t)gm * K + gk]) : 0.0f;
            Ws[k][r] = (gn < N && gk < K) ? to_f(W[(int64_t)gn * K + gk]) : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < SBK; ++k) {
            float av[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                av[i] = As[k][ty * 4 + i];
                bv[i] = Ws[k][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
    const T* bias = static_cast<const T*>(a.bias);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int gm = m0 + ty * 4 + i;
        if (gm >= M) continue;
        const float2 fs = EPI == EPI_LN_FOLD ? a.fold_stats[gm] : make_float2(0.0f, 0.0f);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int gn = n0 + tx * 4 + j;
            if (gn >= N) continue;
            const int64_t o = (int64_t)gm * N + gn;
            float v = acc[i][j];
            if (EPI == EPI_LN_FOLD) v = fmaf(v, fs.x, fmaf(-fs.y, a.fold_c[gn], a.fold_d[gn]));
            else if (bias) v += to_f(bias[gn]);
            if (EPI == EPI_BIAS_GELU) v = gelu_f(v, a.gelu_tanh != 0);
            if (EPI == EPI_BIAS_RESIDUAL || EPI == EPI_RES_OUT32) v += to_f(static_cast<const T*>(a.residual)[o]);
            if (EPI == EPI_RES32) v += static_cast<const float*>(a.residual)[o];
            if (EPI == EPI_RES_OUT32) {
                static_cast<float*>(a.out)[o] = v;
            } else {
                const T h = from_f<T>(v);
                static_cast<T*>(a.out)[o] = h;
                if (EPI == EPI_LN_FOLD && a.lo != nullptr && gn < a.lo_cols)
                    static_cast<T*>(a.lo)[(int64_t)gm * a.lo_cols + gn] = from_f<T>(v - to_f(h));
            }
        }
    }
}

template <typename T>
static void simt_dispatch(const GemmArgs& a, cudaStream_t st) {
    dim3 grid((a.N + SBN - 1) / SBN, (a.M_cap + SBM - 1) / SBM);
    const T *A = (const T*)a.A, *W = (const T*)a.W;
    switch (a.epilogue) {
    case EPI_BIAS: gemm_simt_kernel<T, EPI_BIAS><<<grid, 256, 0, st>>>(A, W, a); break;
    case EPI_BIAS_GELU: gemm_simt_kernel<T, EPI_BIAS_GELU><<<grid, 256, 0, st>>>(A, W, a); break;
    case EPI_BIAS_RESIDUAL: gemm_simt_kernel<T, EPI_BIAS_RESIDUAL><<<grid, 256, 0, st>>>(A, W, a); break;
    case EPI_LN_FOLD: gemm_simt_kernel<T, EPI_LN_FOLD><<<grid, 256, 0, st>>>(A, W, a); break;
    case EPI_RES_OUT32: gemm_simt_kernel<T, EPI_RES_OUT32><<<grid, 256, 0, st>>>(A, W, a); break;
    default: gemm_simt_kernel<T, EPI_RES32><<<grid, 256, 0, st>>>(A, W, a); break;
    }
}

cudaError_t launch_gemm_simt(const GemmArgs& a, cudaStream_t st) {
    if (a.M_cap <= 0 || a.N <= 0) return cudaSuccess;
    switch (a.dtype) {
    case ENERGON_F32: simt_dispatch<float>(a, st); break;
    case ENERGON_F16: simt_dispatch<__half>(a, st); break;
    case ENERGON_BF16: simt_dispatch<__nv_bfloat16>(a, st); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace energon
