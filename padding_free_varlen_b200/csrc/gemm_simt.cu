// CUDA-core GEMM y = A W^T + bias (+ GELU) (+ residual) for the fp32 layer and
// for shapes the tcgen05 kernel does not take.  64 x 64 output tile per
// 256-thread block, 4 x 4 outputs per thread, K staged through shared memory
// in steps of 16.  Same epilogue semantics as the tensor-core kernel: fp32
// accumulate, bias, optional GELU, optional residual, one rounding to the
// storage type.  The valid row count is read on the device.
#include "common.cuh"
#include "internal.h"

namespace energon {

namespace {
constexpr int SBM = 64, SBN = 64, SBK = 16;
}

template <typename T, int EPI>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const T* __restrict__ A, const T* __restrict__ W,
                                                        const T* __restrict__ bias, const T* residual, T* out,
                                                        const int32_t* d_rows, int M_cap, int N, int K, int gelu_tanh,
                                                        const int32_t* status) {
    __shared__ float As[SBK][SBM + 4];
    __shared__ float Ws[SBK][SBN + 4];
    if (status_bad(status)) return;
    const int M = min(*d_rows, M_cap);
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
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = As[k][ty * 4 + i];
                b[i] = Ws[k][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int gm = m0 + ty * 4 + i;
        if (gm >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int gn = n0 + tx * 4 + j;
            if (gn >= N) continue;
            float v = acc[i][j];
            if (bias) v += to_f(bias[gn]);
            if (EPI == EPI_BIAS_GELU) v = gelu_f(v, gelu_tanh != 0);
            if (EPI == EPI_BIAS_RESIDUAL) v += to_f(residual[(int64_t)gm * N + gn]);
            out[(int64_t)gm * N + gn] = from_f<T>(v);
        }
    }
}

template <typename T>
static void simt_dispatch(const GemmArgs& a, cudaStream_t st) {
    dim3 grid((a.N + SBN - 1) / SBN, (a.M_cap + SBM - 1) / SBM);
    const T *A = (const T*)a.A, *W = (const T*)a.W, *b = (const T*)a.bias, *r = (const T*)a.residual;
    T* o = (T*)a.out;
    switch (a.epilogue) {
    case EPI_BIAS:
        gemm_simt_kernel<T, EPI_BIAS><<<grid, 256, 0, st>>>(A, W, b, r, o, a.d_rows, a.M_cap, a.N, a.K, a.gelu_tanh,
                                                            a.status);
        break;
    case EPI_BIAS_GELU:
        gemm_simt_kernel<T, EPI_BIAS_GELU><<<grid, 256, 0, st>>>(A, W, b, r, o, a.d_rows, a.M_cap, a.N, a.K,
                                                                 a.gelu_tanh, a.status);
        break;
    default:
        gemm_simt_kernel<T, EPI_BIAS_RESIDUAL><<<grid, 256, 0, st>>>(A, W, b, r, o, a.d_rows, a.M_cap, a.N, a.K,
                                                                     a.gelu_tanh, a.status);
        break;
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
