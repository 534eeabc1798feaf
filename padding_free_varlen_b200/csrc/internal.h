// Internal launchers shared by the C-ABI layer (capi.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <functional>

namespace energon {

// Host-side launch facts (a kernel's shared-memory opt-in, its occupancy, the SM count) hold
// per device: device_cached returns compute() for (current device, key, what), computing it
// once per triple; thread-safe.
int device_cached(const void* key, int what, const std::function<int()>& compute);
// Sets a kernel's dynamic shared-memory limit on the current device once; returns the
// cudaError_t of that one call on every later call too.
cudaError_t prepare_smem(const void* kernel, int bytes);

// Offsets: cu[b+1] = cu[b] + lengths[b]; validates lengths into *status (SET).
cudaError_t launch_offsets(const int32_t* lengths, int batch, int pad_len, int32_t* cu, int32_t* status,
                           cudaStream_t st);
// cu_pad[b] = b * pad_len for b in [0, batch] (the padded path's row starts).
cudaError_t launch_padded_starts(int batch, int pad_len, int32_t* cu_pad, const int32_t* status, cudaStream_t st);

// transpose_padding_remove: packed[cu[b] + s] = padded[b, s] for s < cu[b+1] - cu[b].
cudaError_t launch_remove(const void* padded, const int32_t* cu, int batch, int pad_len, int64_t row_bytes,
                          void* packed, int64_t packed_rows_cap, const int32_t* status, cudaStream_t st);
// transpose_padding_rebuild: padded[b, s] = s < len_b ? packed[starts[b] + s] : 0,
// len_b = lens_cu[b+1] - lens_cu[b].  Writes every padded row.
cudaError_t launch_rebuild(const void* packed, const int32_t* starts, const int32_t* lens_cu, int batch,
                           int pad_len, int64_t row_bytes, int64_t packed_rows_cap, void* padded, cudaStream_t st);
// Head-transposing forms: packed rows of `parts` blocks of n_heads heads of
// head_bytes bytes <-> head-major [parts][batch][n_heads][pad_len][head_bytes].
cudaError_t launch_transpose_rebuild(const void* packed, const int32_t* cu, int batch, int pad_len, int parts,
                                     int n_heads, int64_t head_bytes, int64_t packed_rows_cap, void* heads,
                                     cudaStream_t st);
cudaError_t launch_transpose_remove(const void* heads, const int32_t* cu, int batch, int pad_len, int parts,
                                    int n_heads, int64_t head_bytes, int64_t packed_rows_cap, void* packed,
                                    cudaStream_t st);

// Zero the pad rows (s >= cu[b+1] - cu[b]) of padded [batch, pad_len] rows of row_bytes.
cudaError_t launch_zero_pads(const int32_t* cu, int batch, int pad_len, int64_t row_bytes, void* padded,
                             cudaStream_t st);

// LayerNorm gather (transpose_padding_remove fused into a LayerNorm): with cu set, row
// r of the output reads padded row (b, r - cu[b]) of x [batch, pad_len, H] and, with
// copy set, also writes that raw row to copy[r].
struct LnGather {
    const int32_t* cu = nullptr;
    int batch = 0, pad_len = 0;
    void* copy = nullptr;
};
// LayerNorm over rows [0, min(*d_rows, rows_cap)) of x [rows_cap, H] -> y.  x_f32: the
// input rows are fp32 (the residual after attention), y is of the storage type.
cudaError_t launch_layernorm(int dtype, const void* x, const void* g, const void* b, void* y, const int32_t* d_rows,
                             int rows_cap, int H, float eps, const int32_t* status, cudaStream_t st,
                             const LnGather& gth = LnGather(), bool x_f32 = false);

// LayerNorm folded into the GEMM that follows it.  For each row r of x (storage type):
//   u[r][k] = x[r][k] * g[k] rounded to the storage type (exact when g is 1),
//   stats[r] = (rstd_r, mean_r * rstd_r) in fp32,
// so that LN(x) W^T + b = rstd_r (u W^T) - mean_r rstd_r c + d with the vectors of
// launch_ln_fold_weights.  Gather form as in launch_layernorm.
cudaError_t launch_ln_fold(int dtype, const void* x, const void* g, void* u, float2* stats, const int32_t* d_rows,
                           int rows_cap, int H, float eps, const int32_t* status, cudaStream_t st,
                           const LnGather& gth = LnGather());
// c[n] = sum_k g[k] W[n][k], d[n] = bias[n] + sum_k beta[k] W[n][k] (fp32) for W [N, K].
cudaError_t launch_ln_fold_weights(int dtype, const void* W, const void* g, const void* beta, const void* bias,
                                   int N, int K, float* c, float* d, const int32_t* status, cudaStream_t st);

// Epilogue variants of the GEMM y = A W^T + bias (+ GELU) (+ residual).
//   EPI_LN_FOLD: y = rstd_r acc - (mean rstd)_r c[n] + d[n] (the folded LayerNorm,
//     see launch_ln_fold); columns below lo_cols also store y - round(y), rounded,
//     to `lo` (the low half of a two-term 16-bit value).
//   EPI_RES_OUT32: y = acc + bias + residual (storage type), stored as fp32.
//   EPI_RES32: y = acc + bias + residual (fp32), stored in the storage type.
enum Epilogue { EPI_BIAS = 0, EPI_BIAS_GELU = 1, EPI_BIAS_RESIDUAL = 2, EPI_LN_FOLD = 3, EPI_RES_OUT32 = 4,
                EPI_RES32 = 5 };

struct GemmArgs {
    int dtype;                 // energon_dtype
    const void* A;             // [M_cap, K]
    const void* W;             // [N, K]
    const void* bias;          // [N] or null
    const void* residual;      // [M_cap, N] or null (EPI_BIAS_RESIDUAL)
    void* out;                 // [M_cap, N]
    const int32_t* d_rows;     // device: valid rows M (<= M_cap)
    int M_cap, N, K;
    int A_rows;                // rows allocated in A (>= M_cap; a multiple of 256 for the tensor-core path)
    float* partials;           // optional fp32 scratch for split-K of buffers of <= 128 rows
    size_t partials_bytes;
    int epilogue;
    int gelu_tanh;
    int32_t* status;
    uint64_t timeout_ns;
    // Optional transpose_padding_rebuild in the epilogue: output row r is stored at padded
    // row b * scatter_pad_len + r - scatter_cu[b] of out [scatter_batch, scatter_pad_len, N].
    const int32_t* scatter_cu = nullptr;
    int scatter_batch = 0, scatter_pad_len = 0;
    // EPI_LN_FOLD: per-row (rstd, mean * rstd), per-column c and d, and the low halves
    const float2* fold_stats = nullptr;
    const float* fold_c = nullptr;
    const float* fold_d = nullptr;
    void* lo = nullptr;        // [M_cap, lo_cols] or null
    int lo_cols = 0;
};

// True when the tcgen05 path can run this GEMM (16-bit types, alignment, tile multiples).
bool gemm_tc_supported(const GemmArgs& a);
// True when it runs on the CTA-pair kernel, the one whose epilogue can scatter.
bool gemm_tc_scatter_ok(const GemmArgs& a);
cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t st, char* err, size_t errlen);
cudaError_t launch_gemm_simt(const GemmArgs& a, cudaStream_t st);

// Causal attention within each sequence: qkv [rows, 3H] -> o [rows, H].  The
// tensor-core kernel runs for 16-bit types with head_dim 128 (qkv_rows: rows
// allocated in qkv, the extent of its tensor map); otherwise the CUDA-core one.
// qk_lo [rows, 2H] (optional): the low halves of Q | K, so that q = hi + lo to about twice
// the storage type's precision; the scores then use both halves.
cudaError_t launch_attention(int dtype, const void* qkv, const void* qk_lo, void* o, const int32_t* cu, int batch,
                             int max_len, int H, int n_heads, int qkv_rows, int32_t* status, uint64_t timeout_ns,
                             cudaStream_t st);
bool attention_tc_supported(int dtype, int H, int n_heads, const void* qkv, const void* qk_lo, const void* o,
                            int qkv_rows);
cudaError_t launch_attention_tc(int dtype, const void* qkv, const void* qk_lo, void* o, const int32_t* cu, int batch,
                                int max_len, int H, int n_heads, int qkv_rows, int32_t* status, uint64_t timeout_ns,
                                cudaStream_t st);

// The binary version (major * 10 + minor) the runtime reports for the library's kernels.
cudaError_t kernel_binary_version(int* version);

// Self-test kernel of the bounded wait.
cudaError_t launch_wait_selftest(int32_t* status, uint64_t timeout_ns, cudaStream_t st);

int device_sm_count();

}  // namespace energon
