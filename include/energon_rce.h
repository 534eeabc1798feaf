/*
 * energon_rce.h - C ABI of the padding-free variable-length ("redundant
 * computation elimination") GPT-3 decoder-layer stack for NVIDIA B200 (sm_100a).
 *
 * What the calls compute follows the Energon-AI pages:
 *  - "最新大模型推理系统Energon-AI开源，来自Colossal-AI团队" (QbitAI article),
 *    section "Runtime": the transpose_padding_remove / transpose_padding_rebuild
 *    operators that let encoder and decoder models skip the redundant work of
 *    padding in variable-length NLP batches; section "易用性": the
 *    bias + GELU and bias + residual steps around the MLP GEMMs.
 *  - EnergonAI README, section "Scaling Ability": GPT-3 layers in FP16 with the
 *    redundant computation elimination method, sequence length half the
 *    padding length; section "Batching": lengths up to 256 padded to the batch
 *    maximum.
 *
 * Conventions for every call:
 *  - Every pointer argument is a DEVICE pointer owned by the caller, except the
 *    config / weight-table structs, which are host structs read during the call.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Calls are asynchronous on that stream; nothing is read back to the host.
 *  - Row-major layouts, innermost dimension contiguous.  Weights use the
 *    nn.Linear layout W[out_features, in_features].
 *  - The library allocates no device memory per call: scratch space comes from
 *    the caller's workspace (see energon_workspace_bytes).
 *  - Return value: ENERGON_OK or an energon_status code.  No exception crosses
 *    the ABI; energon_last_error() gives a message for the calling thread.
 *  - Device status word (int32_t, caller-owned, device memory): invalid lengths
 *    and bounded-wait timeouts are detected on the device and recorded there
 *    (ENERGON_DEVICE_* bits).  Kernels of a call that find a nonzero word do no
 *    work.  Read it after synchronising the stream.
 */
#ifndef ENERGON_RCE_H
#define ENERGON_RCE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ENERGON_API __attribute__((visibility("default")))
#else
#define ENERGON_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Host-side return codes. */
typedef enum {
    ENERGON_OK = 0,
    ENERGON_ERR_INVALID_ARGUMENT = 1, /* null pointer, negative size, bad enum */
    ENERGON_ERR_UNSUPPORTED = 2,      /* dtype / shape the library does not run */
    ENERGON_ERR_MISALIGNED = 3,       /* a pointer breaks an alignment the path needs */
    ENERGON_ERR_CUDA = 4,             /* a CUDA runtime / launch error */
    ENERGON_ERR_WORKSPACE_TOO_SMALL = 5,
    ENERGON_ERR_DEVICE_TIMEOUT = 6    /* reserved for synchronous helpers */
} energon_status;

/* Bits of the device status word. */
#define ENERGON_DEVICE_OK 0
#define ENERGON_DEVICE_BAD_LENGTH 1 /* a length outside [0, pad_len] */
#define ENERGON_DEVICE_TIMEOUT 2    /* a bounded wait inside a kernel ran out */

/* Element types. */
typedef enum { ENERGON_F32 = 0, ENERGON_F16 = 1, ENERGON_BF16 = 2 } energon_dtype;

/*
 * Offsets of the packed layout: the exclusive prefix sum of the per-sequence
 * lengths (QbitAI article, "Runtime": the packing behind
 * transpose_padding_remove).
 *   lengths     [batch] int32, each in [0, pad_len]
 *   cu_seqlens  [batch + 1] int32 out: cu[0] = 0, cu[b+1] = cu[b] + lengths[b];
 *               cu[batch] = T, the number of valid tokens, stays on the device.
 *   d_status    int32 out: SET to ENERGON_DEVICE_OK, or to
 *               ENERGON_DEVICE_BAD_LENGTH when some length lies outside
 *               [0, pad_len]; in that case every cu entry is written as 0.
 * batch >= 0, pad_len >= 0.  One launch of one thread block.
 */
ENERGON_API int energon_rce_offsets(const int32_t* lengths, int batch, int pad_len, int32_t* cu_seqlens,
                        int32_t* d_status, void* stream);

/*
 * transpose_padding_remove (QbitAI article, "Runtime"): gathers the valid rows
 * of a padded tensor into a packed one.
 *   padded      [batch, pad_len, hidden] elements of elem_bytes bytes
 *   cu_seqlens  [batch + 1] from energon_rce_offsets (device)
 *   packed      out, at least batch * pad_len rows of hidden elements; row
 *               cu[b] + s receives padded row (b, s) for s < len[b].  Rows at or
 *               beyond T are not written.
 * A byte copy (bit-exact).  elem_bytes in {1, 2, 4, 8}; any hidden >= 0; any
 * pointer alignment (16-byte vector path when rows and pointers allow it).
 * Rows whose offsets would fall outside either buffer are skipped.
 */
ENERGON_API int energon_rce_remove_padding(const void* padded, const int32_t* cu_seqlens, int batch,
                               int pad_len, int hidden, int elem_bytes, void* packed,
                               void* stream);

/*
 * transpose_padding_rebuild (QbitAI article, "Runtime"): scatters packed rows
 * back to the padded layout.
 *   packed      [>= T, hidden]
 *   padded      out [batch, pad_len, hidden]: EVERY row is written; row (b, s) is
 *               packed row cu[b] + s when s < len[b], all-zero bytes otherwise.
 * Same element and alignment rules as energon_rce_remove_padding.
 */
ENERGON_API int energon_rce_rebuild_padding(const void* packed, const int32_t* cu_seqlens, int batch,
                                int pad_len, int hidden, int elem_bytes, void* padded,
                                void* stream);

/*
 * Head-transposing forms of the two operations above (QbitAI article, "Runtime",
 * which names transpose_padding_rebuild / transpose_padding_remove and nothing
 * more; the "transpose" is read as the [token, head] <-> [head, token] exchange
 * that an attention stage on the padded, head-major layout needs).
 *   packed      [>= T, parts * n_heads * head_dim]: a token row holds `parts`
 *               blocks (1 for an attention output, 3 for Q | K | V), each of
 *               n_heads heads of head_dim elements of elem_bytes bytes
 *   heads       [parts, batch, n_heads, pad_len, head_dim]
 *   cu_seqlens  [batch + 1] from energon_rce_offsets (device)
 * transpose_padding_rebuild writes EVERY element of `heads`: (c, b, h, s, :) is
 * block c, head h of packed row cu[b] + s when s < len[b], all-zero bytes
 * otherwise.  transpose_padding_remove writes packed rows 0 .. T-1 only: row
 * cu[b] + s, block c, head h receives heads (c, b, h, s, :); pad positions of
 * `heads` are never read.  Byte copies (bit-exact).  elem_bytes in {1, 2, 4, 8};
 * parts >= 1, n_heads >= 1, head_dim >= 0, parts * n_heads * head_dim *
 * elem_bytes < 2^31; any pointer alignment (16-byte vector path when head_dim *
 * elem_bytes and both pointers allow it).  The buffers are the caller's;
 * nothing is allocated.  Errors: NULL pointer, negative size or a bad
 * elem_bytes -> ENERGON_ERR_INVALID_ARGUMENT before any launch.
 */
ENERGON_API int energon_rce_transpose_padding_rebuild(const void* packed, const int32_t* cu_seqlens, int batch,
                                          int pad_len, int parts, int n_heads, int head_dim, int elem_bytes,
                                          void* heads, void* stream);
ENERGON_API int energon_rce_transpose_padding_remove(const void* heads, const int32_t* cu_seqlens, int batch,
                                         int pad_len, int parts, int n_heads, int head_dim, int elem_bytes,
                                         void* packed, void* stream);

/* Weights of one pre-LN GPT decoder layer, all of the config's dtype, device:
 *   ln1_g, ln1_b [H]; w_qkv [3H, H], b_qkv [3H] (output columns Q | K | V, each
 *   head-major); w_o [H, H], b_o [H]; ln2_g, ln2_b [H]; w_1 [F, H], b_1 [F];
 *   w_2 [H, F], b_2 [H].
 *   ln1_fold: optional, fp32 [6H], 16-byte aligned: the first LayerNorm's fold
 *   vectors c = W_qkv ln1_g [3H] followed by d = b_qkv + W_qkv ln1_b [3H], as
 *   energon_layer_fold_weights writes them.  They depend on the weights only;
 *   NULL makes every layer call compute them into its workspace (one pass over
 *   W_qkv per call). */
typedef struct {
    const void *ln1_g, *ln1_b, *w_qkv, *b_qkv, *w_o, *b_o, *ln2_g, *ln2_b, *w_1, *b_1, *w_2, *b_2;
    const float* ln1_fold;
} energon_layer_weights;


/* hidden H, n_heads (head_dim = H / n_heads), ffn F, dtype (energon_dtype),
 * LayerNorm epsilon, gelu_tanh (1: tanh approximation as in GPT-2/3, 0: erf). */
typedef struct {
    int hidden, n_heads, ffn, dtype;
    float ln_eps;
    int gelu_tanh;
} energon_layer_config;

/*
 * The first LayerNorm of a layer is folded into its QKV projection:
 *   LN(x) W_qkv^T + b_qkv = rstd (x * ln1_g) W_qkv^T - mean rstd c + d
 * with c = W_qkv ln1_g and d = b_qkv + W_qkv ln1_b, so that the tensor cores read
 * the layer input itself (times ln1_g) rather than a rounded normalisation of it.
 * This call computes c and d once for a set of weights (a weight-load step, like
 * any layout preparation of the weights): fold [6H] fp32 device memory owned by
 * the caller, 16-byte aligned; c, then d.  Reads w_qkv, b_qkv, ln1_g, ln1_b only.
 * Asynchronous on `stream`; fp32 sums in a fixed order (the same values a layer
 * call computes for itself when ln1_fold is NULL, bit for bit).
 * Errors: invalid config, NULL pointer or misaligned fold -> ENERGON_ERR_* before
 * any launch.
 */
ENERGON_API int energon_layer_fold_weights(const energon_layer_config* cfg, const energon_layer_weights* w,
                                           float* fold, void* stream);

/*
 * Workspace bytes that energon_layer_forward and energon_stack_forward need for
 * this config at capacity batch * pad_len tokens (the larger of the two).
 * Returns 0 for an invalid config.  Host-only; launches nothing.
 *
 * Layout (part of the ABI; each region starts on a 1024-byte boundary, e =
 * element bytes, R = batch * pad_len rounded up to a multiple of 256):
 *   a [R, H]      GEMM operand of the LayerNorms: u = x * ln1_g for the folded
 *                 first LayerNorm, then the second LayerNorm's output
 *   qkv [R, 3H]   Q | K | V (for 16-bit types, Q and K are the high halves)
 *   qk_lo [R, 2H] low halves of Q | K (16-bit types; 0 bytes for fp32)
 *   o [R, H]      attention output
 *   x1 [R, H]     fp32: the residual after attention
 *   f [R, F]      GELU output
 *   p32           fp32 split-K partial sums, 4 * 128 * max(3H, F) floats when
 *                 batch * pad_len <= 128, else 0 bytes
 *   stats [R]     float2 per row: (rstd, mean * rstd) of the first LayerNorm
 *   fold [6H]     fp32: c = W_qkv ln1_g [3H], then d = b_qkv + W_qkv ln1_b [3H]
 *   x [R, H], cu [batch + 1] int32, cu_pad [batch + 1] int32 - stack only
 * After a call completes, the regions hold that call's (last layer's)
 * intermediates for the first T rows, which makes every step inspectable
 * (the stack with remove_padding = 2 reuses qkv and o for the packed fp32
 * input and the packed output of the last MLP).
 */
ENERGON_API size_t energon_workspace_bytes(const energon_layer_config* cfg, int batch, int pad_len);

/*
 * One pre-LN GPT decoder layer on packed tokens (EnergonAI README, "Scaling
 * Ability": the GPT-3 layer run with redundant computation elimination):
 *     a = LN(x; ln1),  qkv = a W_qkv^T + b_qkv,  o = causal attention within
 *     each sequence (cu_seqlens), x1 = x + o W_o^T + b_o,
 *     y = x1 + GELU(LN(x1; ln2) W_1^T + b_1) W_2^T + b_2
 *   x_packed, y_packed [batch * max_len, H] capacity; only the first
 *   T = cu_seqlens[batch] rows are read / written.  y_packed == x_packed allowed.
 *   max_len: the largest sequence length (pad_len); sizes the launch grids.
 *   d_status: optional device status word (NULL allowed); kernels skip work when
 *   it is nonzero and OR ENERGON_DEVICE_TIMEOUT into it if a bounded wait expires.
 * LayerNorm statistics, accumulation and softmax are fp32.  The first LayerNorm
 * is folded into the QKV GEMM (its operand is the layer input times ln1_g, one
 * rounding, exact when ln1_g is 1; the epilogue applies the row statistics), Q
 * and K are kept as two 16-bit terms for the attention scores, and the residual
 * after attention stays in fp32; the other kernel boundaries (V, the attention
 * output, the second LayerNorm, the GELU output, y) round to the storage dtype.
 * fp16 / bf16 use the tcgen05 tensor-core GEMM when H % 256 == 0 and
 * F % 256 == 0 (other shapes run the CUDA-core GEMM, traced as "gemm_simt");
 * fp32 uses CUDA-core kernels.  head_dim must be 64 or 128.
 */
ENERGON_API int energon_layer_forward(const energon_layer_config* cfg, const energon_layer_weights* w,
                          const void* x_packed, const int32_t* cu_seqlens, int batch, int max_len,
                          void* y_packed, int32_t* d_status, void* workspace, size_t ws_bytes,
                          void* stream);

/*
 * The whole hot path: offsets -> transpose_padding_remove -> n_layers decoder
 * layers on packed tokens -> transpose_padding_rebuild.  With remove_padding = 1
 * the remove is fused into the first LayerNorm (it gathers the valid rows) and
 * the rebuild into the last FFN2 GEMM's epilogue (it stores each row at its
 * padded position; the pad rows are zeroed by a separate launch) whenever that
 * GEMM runs on the CTA-pair kernel, i.e. more than 128 rows of capacity.
 *   layers        host array of n_layers weight tables
 *   padded_in     [batch, pad_len, H] device; pad positions may hold anything
 *   lengths       [batch] int32, device
 *   remove_padding 1: run the layers on the T valid tokens (the service
 *                  config's rm_padding = True in the QbitAI article's usability
 *                  example); 0: run them on all batch * pad_len rows (the padded
 *                  baseline the pages compare against); 2: eliminate the padding
 *                  in the MLP only, as the article's "Runtime" section states
 *                  it - each layer's attention sub-layer on all rows, then
 *                  remove, the MLP on the valid tokens, rebuild.  Valid rows are
 *                  the same in all three modes.
 *   padded_out    [batch, pad_len, H]: valid rows hold the stack's output, pad
 *                 rows are zero.  With invalid lengths: all zero, d_status = 1.
 *   d_status      required; SET by the offsets step, then OR-ed by later kernels.
 * No final LayerNorm.  padded_out must not alias padded_in.
 */
ENERGON_API int energon_stack_forward(const energon_layer_config* cfg, const energon_layer_weights* layers,
                          int n_layers, const void* padded_in, const int32_t* lengths, int batch,
                          int pad_len, int remove_padding, void* padded_out, int32_t* d_status,
                          void* workspace, size_t ws_bytes, void* stream);

/*
 * Self-test of the bounded wait used by every kernel that waits on an
 * mbarrier: launches one block that waits on a barrier nobody arrives at.  The
 * wait gives up after timeout_us microseconds, ORs ENERGON_DEVICE_TIMEOUT into
 * *d_status and the kernel returns normally, leaving the context usable.
 */
ENERGON_API int energon_selftest_bounded_wait(int32_t* d_status, uint32_t timeout_us, void* stream);

/*
 * Build check (diagnostic; no counterpart in the pages): the binary version that
 * the CUDA runtime reports for the library's kernels on the current device
 * (cudaFuncGetAttributes, major * 10 + minor: 100 for the sm_100a build).
 * Needs a device; launches nothing.  Errors: NULL -> ENERGON_ERR_INVALID_ARGUMENT;
 * no device or no kernel image for it -> ENERGON_ERR_CUDA.
 */
ENERGON_API int energon_kernel_binary_version(int* version);

/* Upper limit, in microseconds, of every bounded wait inside the kernels
 * (default 2,000,000).  Process-wide. */
ENERGON_API void energon_set_wait_timeout_us(uint32_t timeout_us);

/*
 * Launch tracing (profiling aid).  Between energon_trace_start and
 * energon_trace_stop, every kernel that energon_layer_forward and
 * energon_stack_forward launch is bracketed by two CUDA events on the call's
 * stream.  energon_trace_stop synchronises those events and writes, per kernel
 * name ("gemm_qkv", "attention", "layernorm", "layernorm_remove", "zero_pads",
 * "gemm_ffn2_rebuild", "remove_padding", ...), the number
 * of launches and their summed device time in milliseconds.  Recording adds a
 * pair of event records per launch and nothing else.  Process-wide; not
 * thread-safe.  *n_entries receives the number of names (at most capacity are
 * written).
 */
typedef struct {
    char name[48];
    int launches;
    double total_ms;
} energon_trace_entry;

ENERGON_API int energon_trace_start(void);
ENERGON_API int energon_trace_stop(energon_trace_entry* entries, int capacity, int* n_entries);

/*
 * transpose_padding_remove for callers that cannot allocate device memory.
 * The Energon-AI pages have no counterpart to this entry point: it exists for
 * callers with no cudaMalloc and no workspace at hand, such as an inference
 * runtime's per-request hook that forbids allocation after start-up, or a
 * process whose device memory belongs to a pool manager.
 *   padded, packed, hidden, elem_bytes: as in energon_rce_remove_padding
 *   lengths   [batch] int32 (device), each in [0, pad_len]
 *   d_status  int32 out (device): SET as by energon_rce_offsets; with an invalid
 *             length nothing is gathered
 * The per-sequence offsets go to a fixed scratch array inside the library image
 * (present on every GPU that loads the library until the process exits), so
 * batch may not exceed ENERGON_NOALLOC_MAX_BATCH: larger batches are refused
 * with ENERGON_ERR_INVALID_ARGUMENT before anything is launched.  The call
 * allocates nothing.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress), so make that first call before any stream
 * capture.  The address is kept per device and per context: cudaDeviceReset
 * unloads the library's device image, and the first call after it looks the
 * address up again in the new context (make that call before any capture too).
 * All calls on a device share the array: calls that may overlap on the GPU
 * (unordered streams) race; calls ordered on one stream do not.
 */
#define ENERGON_NOALLOC_MAX_BATCH 16384
ENERGON_API int energon_rce_remove_padding_noalloc(const void* padded, const int32_t* lengths, int batch,
                                                   int pad_len, int hidden, int elem_bytes, void* packed,
                                                   int32_t* d_status, void* stream);

/*
 * Dynamic batching of a request queue (host runtime; no device memory, no GPU
 * needed).  The QbitAI article's "Serving" section and the EnergonAI README's
 * "Batching" section: queued requests are packed into batches as the machine's
 * performance suits best, and the batch of highest priority - from the waiting
 * time, the batch size and the batch's length after padding - runs first,
 * avoiding starvation; the method follows TurboTransformer's dynamic-programming
 * batch scheduler and is compared against FIFO packing.  The pages give no
 * formula; the reading implemented here:
 *   packing   requests sorted by (length, arrival, index) are cut into
 *             consecutive groups of at most max_batch minimising the summed cost
 *             cost(b, s) = cost_table[(b - 1) * table_max_len + (s - 1)] of b
 *             sequences padded to s tokens (measured on the machine; any positive
 *             unit); the scan over group starts keeps the first minimum;
 *   priority  (tokens of the group) / cost(size, longest length)
 *             * (1 + (now_s - earliest arrival in the group) / age_scale_s).
 *   reqs       [n] requests (length in [1, table_max_len], finite arrival_s)
 *   cost_table [max_batch * table_max_len] doubles, finite and > 0 (only rows
 *              b <= min(max_batch, n) are read)
 *   group_of   out [n]: group of each request; groups are numbered in ascending
 *              length order
 *   n_groups   out: number of groups
 *   order      out [n] (first *n_groups used): group indices by descending
 *              priority, ties by ascending index
 * All buffers are host memory owned by the caller.  Errors (before any output
 * is written): NULL pointer, n < 0, max_batch or table_max_len < 1, a length out
 * of range, a non-finite time, age_scale_s <= 0, a bad cost entry ->
 * ENERGON_ERR_INVALID_ARGUMENT.
 */
typedef struct {
    int32_t length;   /* valid tokens of the request */
    double arrival_s; /* arrival time, seconds on any common clock */
} energon_request;

ENERGON_API int energon_sched_plan(const energon_request* reqs, int n, double now_s, int max_batch,
                       const double* cost_table, int table_max_len, double age_scale_s,
                       int32_t* group_of, int32_t* n_groups, int32_t* order);

/*
 * FIFO packing, the pages' comparison: requests in arrival order (ties by
 * index) cut into consecutive groups of max_batch.  group_of [n] and n_groups
 * out (host memory).  Errors: NULL pointer, n < 0, max_batch < 1, a non-finite
 * time -> ENERGON_ERR_INVALID_ARGUMENT.
 */
ENERGON_API int energon_sched_fifo(const energon_request* reqs, int n, int max_batch, int32_t* group_of,
                       int32_t* n_groups);

/* Message describing the last failed call on this thread ("" if none). */
ENERGON_API const char* energon_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ENERGON_RCE_H */
