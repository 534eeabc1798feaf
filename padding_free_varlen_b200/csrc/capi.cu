// C ABI of the library: argument checks, workspace layout and the launch
// sequence of one layer and of the whole stack.  Device-side facts (the token
// count T, invalid lengths, bounded-wait timeouts) never come back to the host
// during a call: T is read by the kernels from cu_seqlens[batch], and problems
// are recorded in the caller's device status word.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <string>
#include <vector>

#include "../../include/energon_rce.h"
#include "internal.h"

using namespace energon;

namespace {

thread_local std::string g_last_error;
uint64_t g_timeout_ns = 2000000000ull;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char* where) {
    return fail(ENERGON_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

#define CK(expr, where)                          \
    do {                                         \
        cudaError_t e_ = (expr);                 \
        if (e_ != cudaSuccess) return cuda_fail(e_, where); \
    } while (0)

// ------------------------------------------------------------------ launch tracing

struct TraceRec {
    const char* name;
    cudaEvent_t start, stop;
};
bool g_trace_on = false;
std::vector<TraceRec> g_trace;
std::vector<cudaEvent_t> g_event_pool;
size_t g_event_used = 0;

cudaEvent_t trace_event() {
    if (g_event_used == g_event_pool.size()) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
        g_event_pool.push_back(e);
    }
    return g_event_pool[g_event_used++];
}

// Runs `launch`, bracketed by events on `st` while tracing is on.
template <typename F>
cudaError_t traced(const char* name, cudaStream_t st, F&& launch) {
    if (!g_trace_on) return launch();
    cudaEvent_t a = trace_event(), b = trace_event();
    if (a) cudaEventRecord(a, st);
    cudaError_t e = launch();
    if (b) cudaEventRecord(b, st);
    if (a && b) g_trace.push_back({name, a, b});
    return e;
}

size_t dtype_bytes(int dtype) {
    switch (dtype) {
    case ENERGON_F32: return 4;
    case ENERGON_F16:
    case ENERGON_BF16: return 2;
    }
    return 0;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Rows allocated for every activation buffer: batch * pad_len rounded up to the
// 256-row GEMM tile of a CTA pair, so tensor-map boxes never reach past an allocation.
int64_t rows_alloc(int batch, int pad_len) { return (int64_t)align_up((size_t)batch * (size_t)pad_len, 256); }

struct LayerWs {
    void *a, *qkv, *qk_lo, *o, *f;
    float* x1;      // residual after attention, fp32
    float* p32;     // split-K partial sums (buffers of <= 128 rows only)
    size_t p32_bytes;
    float2* stats;  // folded LayerNorm: (rstd, mean * rstd) per row
    float *fold_c, *fold_d;
    size_t bytes;
};

// Split-K scratch for weight-streaming GEMMs: up to 4 splits of 128 rows of the widest output.
size_t splitk_bytes(const energon_layer_config& c, int batch, int pad_len) {
    if ((int64_t)batch * pad_len > 128) return 0;
    const size_t widest = (size_t)(3 * c.hidden > c.ffn ? 3 * c.hidden : c.ffn);
    return 4 * 128 * widest * sizeof(float);
}

LayerWs layer_ws_layout(const energon_layer_config& c, int batch, int pad_len, void* base) {
    const size_t e = dtype_bytes(c.dtype);
    const size_t R = (size_t)rows_alloc(batch, pad_len);
    const size_t H = (size_t)c.hidden, F = (size_t)c.ffn;
    uint8_t* p = static_cast<uint8_t*>(base);
    size_t off = 0;
    LayerWs w;
    auto take = [&](size_t bytes) {
        void* r = (p && bytes) ? p + off : nullptr;
        off = align_up(off + bytes, 1024);
        return r;
    };
    w.a = take(R * H * e);
    w.qkv = take(R * 3 * H * e);
    // low halves of Q | K: 16-bit types only (fp32 values need no second term)
    w.qk_lo = take(c.dtype == ENERGON_F32 ? 0 : R * 2 * H * e);
    w.o = take(R * H * e);
    w.x1 = static_cast<float*>(take(R * H * sizeof(float)));
    w.f = take(R * F * e);
    w.p32_bytes = splitk_bytes(c, batch, pad_len);
    w.p32 = static_cast<float*>(take(w.p32_bytes));
    w.stats = static_cast<float2*>(take(R * sizeof(float2)));
    w.fold_c = static_cast<float*>(take(2 * 3 * H * sizeof(float)));
    w.fold_d = w.fold_c ? w.fold_c + 3 * H : nullptr;
    w.bytes = off;
    return w;
}

struct StackWs {
    LayerWs layer;
    void* x;
    int32_t *cu, *cu_pad;
    size_t bytes;
};

StackWs stack_ws_layout(const energon_layer_config& c, int batch, int pad_len, void* base) {
    StackWs s;
    s.layer = layer_ws_layout(c, batch, pad_len, base);
    const size_t e = dtype_bytes(c.dtype);
    const size_t R = (size_t)rows_alloc(batch, pad_len);
    uint8_t* p = static_cast<uint8_t*>(base);
    size_t off = s.layer.bytes;
    auto take = [&](size_t bytes) {
        void* r = p ? p + off : nullptr;
        off = align_up(off + bytes, 1024);
        return r;
    };
    s.x = take(R * (size_t)c.hidden * e);
    s.cu = static_cast<int32_t*>(take(((size_t)batch + 1) * 4));
    s.cu_pad = static_cast<int32_t*>(take(((size_t)batch + 1) * 4));
    s.bytes = off;
    return s;
}

int check_config(const energon_layer_config* c) {
    if (!c) return fail(ENERGON_ERR_INVALID_ARGUMENT, "config is NULL");
    if (dtype_bytes(c->dtype) == 0) return fail(ENERGON_ERR_INVALID_ARGUMENT, "unknown dtype %d", c->dtype);
    if (c->hidden <= 0 || c->n_heads <= 0 || c->ffn <= 0)
        return fail(ENERGON_ERR_INVALID_ARGUMENT, "hidden, n_heads and ffn must be positive");
    if (c->hidden % c->n_heads != 0)
        return fail(ENERGON_ERR_INVALID_ARGUMENT, "hidden %d is not a multiple of n_heads %d", c->hidden, c->n_heads);
    const int hd = c->hidden / c->n_heads;
    if (hd != 64 && hd != 128) return fail(ENERGON_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128)", hd);
    if (!(c->ln_eps >= 0.0f)) return fail(ENERGON_ERR_INVALID_ARGUMENT, "ln_eps must be >= 0");
    return ENERGON_OK;
}

int check_sizes(int batch, int pad_len) {
    if (batch < 1 || pad_len < 1) return fail(ENERGON_ERR_INVALID_ARGUMENT, "batch and pad_len must be >= 1");
    if ((int64_t)batch * pad_len > (int64_t)0x7fffff00)
        return fail(ENERGON_ERR_INVALID_ARGUMENT, "batch * pad_len exceeds the int32 token index");
    return ENERGON_OK;
}

int check_weights(const energon_layer_weights* w) {
    if (!w) return fail(ENERGON_ERR_INVALID_ARGUMENT, "weights are NULL");
    const void* ps[] = {w->ln1_g, w->ln1_b, w->w_qkv, w->b_qkv, w->w_o, w->b_o,
                        w->ln2_g, w->ln2_b, w->w_1,   w->b_1,   w->w_2, w->b_2};
    for (const void* p : ps)
        if (!p) return fail(ENERGON_ERR_INVALID_ARGUMENT, "a weight pointer is NULL");
    if ((uintptr_t)w->ln1_fold % 16 != 0)
        return fail(ENERGON_ERR_MISALIGNED, "ln1_fold must be 16-byte aligned");
    return ENERGON_OK;
}

int run_gemm(GemmArgs& g, cudaStream_t st, const char* what) {
    char err[256] = {0};
    if (gemm_tc_supported(g)) {
        cudaError_t e = traced(what, st, [&] { return launch_gemm_tc(g, st, err, sizeof(err)); });
        if (e != cudaSuccess) {
            if (err[0]) return fail(ENERGON_ERR_CUDA, "%s: %s", what, err);
            return cuda_fail(e, what);
        }
        return ENERGON_OK;
    }
    // Shapes the tensor-core kernel does not take (fp32, or 16-bit N / K off its tile
    // multiples) run on the CUDA-core kernel; the trace names it apart.
    CK(traced("gemm_simt", st, [&] { return launch_gemm_simt(g, st); }), what);
    return ENERGON_OK;
}

GemmArgs gemm_base(const energon_layer_config& c, const int32_t* cu, int batch, int max_len, int32_t* status,
                   const LayerWs& ws) {
    GemmArgs g{};
    g.dtype = c.dtype;
    g.d_rows = cu + batch;
    g.M_cap = batch * max_len;
    g.A_rows = (int)rows_alloc(batch, max_len);
    g.gelu_tanh = c.gelu_tanh;
    g.status = status;
    g.timeout_ns = g_timeout_ns;
    g.partials = ws.p32_bytes ? ws.p32 : nullptr;
    g.partials_bytes = ws.p32_bytes;
    return g;
}

// Attention sub-layer on the rows described by cu (row starts; rows valid = cu[batch]):
//   x1 = x + attention(LN1(x) W_qkv^T + b_qkv) W_o^T + b_o      (x1 in fp32)
// LN1 is folded into the QKV GEMM: the GEMM reads u = x * ln1_g and its epilogue applies
// the row statistics and c = W_qkv ln1_g, d = b_qkv + W_qkv ln1_b; Q and K are kept as
// two 16-bit terms (qkv holds the high, qk_lo the low halves) for the attention scores.
// With `padded` set, x is gathered from that [batch, max_len, H] tensor by the folded
// LayerNorm (transpose_padding_remove fused into it), which also writes the packed rows
// to x (then the residual stream's buffer).
int attention_sublayer(const energon_layer_config& c, const energon_layer_weights& w, const void* x,
                       const int32_t* cu, int batch, int max_len, float* x1, int32_t* status, const LayerWs& ws,
                       cudaStream_t st, const void* padded = nullptr) {
    const int H = c.hidden;
    const int M_cap = batch * max_len;
    const int A_rows = (int)rows_alloc(batch, max_len);
    const int32_t* d_rows = cu + batch;
    LnGather gth;
    if (padded != nullptr) gth.cu = cu, gth.batch = batch, gth.pad_len = max_len, gth.copy = const_cast<void*>(x);
    CK(traced(padded ? "layernorm_remove" : "ln_fold", st,
              [&] {
                  return launch_ln_fold(c.dtype, padded ? padded : x, w.ln1_g, ws.a, ws.stats, d_rows, M_cap, H,
                                        c.ln_eps, status, st, gth);
              }),
       padded ? "ln1 fold + remove" : "ln1 fold");
    // c and d: prepared with the weights (energon_layer_fold_weights), else computed here
    const float* fold_c = w.ln1_fold;
    const float* fold_d = w.ln1_fold ? w.ln1_fold + 3 * (size_t)H : nullptr;
    if (fold_c == nullptr) {
        CK(traced("ln_fold_weights", st,
                  [&] {
                      return launch_ln_fold_weights(c.dtype, w.w_qkv, w.ln1_g, w.ln1_b, w.b_qkv, 3 * H, H, ws.fold_c,
                                                    ws.fold_d, status, st);
                  }),
           "ln1 fold weights");
        fold_c = ws.fold_c, fold_d = ws.fold_d;
    }
    GemmArgs g = gemm_base(c, cu, batch, max_len, status, ws);
    g.A = ws.a, g.W = w.w_qkv, g.bias = nullptr, g.residual = nullptr, g.out = ws.qkv;
    g.N = 3 * H, g.K = H, g.epilogue = EPI_LN_FOLD;
    g.fold_stats = ws.stats, g.fold_c = fold_c, g.fold_d = fold_d;
    g.lo = ws.qk_lo, g.lo_cols = ws.qk_lo ? 2 * H : 0;
    if (int r = run_gemm(g, st, "gemm_qkv")) return r;
    CK(traced("attention", st,
              [&] {
                  return launch_attention(c.dtype, ws.qkv, ws.qk_lo, ws.o, cu, batch, max_len, H, c.n_heads, A_rows,
                                          status, g_timeout_ns, st);
              }),
       "attention");
    g = gemm_base(c, cu, batch, max_len, status, ws);
    g.A = ws.o, g.W = w.w_o, g.bias = w.b_o, g.residual = x, g.out = x1;
    g.N = H, g.K = H, g.epilogue = EPI_RES_OUT32;
    return run_gemm(g, st, "gemm_out_proj");
}

// MLP sub-layer: y = x1 + GELU(LN2(x1) W_1^T + b_1) W_2^T + b_2, x1 in fp32, y in the
// storage type (y may alias nothing but itself).  With `padded_out` set and the FFN2 GEMM
// on the CTA-pair kernel, its epilogue stores each row at its padded position in
// padded_out (transpose_padding_rebuild fused into it; pad rows are left alone) and
// *scattered is set; otherwise the rows go to y.
int mlp_sublayer(const energon_layer_config& c, const energon_layer_weights& w, const float* x1, const int32_t* cu,
                 int batch, int max_len, void* y, int32_t* status, const LayerWs& ws, cudaStream_t st,
                 void* padded_out = nullptr, bool* scattered = nullptr) {
    const int H = c.hidden, F = c.ffn;
    const int M_cap = batch * max_len;
    const int32_t* d_rows = cu + batch;
    CK(traced("layernorm", st,
              [&] {
                  return launch_layernorm(c.dtype, x1, w.ln2_g, w.ln2_b, ws.a, d_rows, M_cap, H, c.ln_eps, status, st,
                                          LnGather(), true);
              }),
       "ln2");
    GemmArgs g = gemm_base(c, cu, batch, max_len, status, ws);
    g.A = ws.a, g.W = w.w_1, g.bias = w.b_1, g.residual = nullptr, g.out = ws.f;
    g.N = F, g.K = H, g.epilogue = EPI_BIAS_GELU;
    if (int r = run_gemm(g, st, "gemm_ffn1")) return r;
    g.A = ws.f, g.W = w.w_2, g.bias = w.b_2, g.residual = x1, g.out = y;
    g.N = H, g.K = F, g.epilogue = EPI_RES32;
    if (scattered) *scattered = false;
    if (padded_out != nullptr) {
        GemmArgs gs = g;
        gs.out = padded_out;
        gs.scatter_cu = cu, gs.scatter_batch = batch, gs.scatter_pad_len = max_len;
        if (gemm_tc_scatter_ok(gs)) {
            if (scattered) *scattered = true;
            return run_gemm(gs, st, "gemm_ffn2_rebuild");
        }
    }
    return run_gemm(g, st, "gemm_ffn2");
}

// One layer; cu = row starts of the sequences (device), rows valid = cu[batch].
int layer_impl(const energon_layer_config& c, const energon_layer_weights& w, const void* x, const int32_t* cu,
               int batch, int max_len, void* y, int32_t* status, const LayerWs& ws, cudaStream_t st) {
    if (int r = attention_sublayer(c, w, x, cu, batch, max_len, ws.x1, status, ws, st)) return r;
    return mlp_sublayer(c, w, ws.x1, cu, batch, max_len, y, status, ws, st);
}

}  // namespace

namespace energon {
// Lets the other translation units of the library report through energon_last_error().
void record_error(int code, const char* msg) {
    if (code == ENERGON_OK) g_last_error.clear();
    else g_last_error = msg;
}
}  // namespace energon

extern "C" {

const char* energon_last_error(void) { return g_last_error.c_str(); }

void energon_set_wait_timeout_us(uint32_t timeout_us) {
    g_timeout_ns = (uint64_t)(timeout_us == 0 ? 1 : timeout_us) * 1000ull;
}

int energon_rce_offsets(const int32_t* lengths, int batch, int pad_len, int32_t* cu_seqlens, int32_t* d_status,
                        void* stream) {
    g_last_error.clear();
    if (!cu_seqlens || !d_status || (batch > 0 && !lengths))
        return fail(ENERGON_ERR_INVALID_ARGUMENT, "offsets: NULL pointer");
    if (batch < 0 || pad_len < 0) return fail(ENERGON_ERR_INVALID_ARGUMENT, "offsets: negative size");
    CK(launch_offsets(lengths, batch, pad_len, cu_seqlens, d_status, (cudaStream_t)stream), "offsets");
    return ENERGON_OK;
}

int energon_rce_remove_padding(const void* padded, const int32_t* cu_seqlens, int batch, int pad_len, int hidden,
                               int elem_bytes, void* packed, void* stream) {
    g_last_error.clear();
    if (!padded || !cu_seqlens || !packed) return fail(ENERGON_ERR_INVALID_ARGUMENT, "remove: NULL pointer");
    if (batch < 0 || pad_len < 0 || hidden < 0) return fail(ENERGON_ERR_INVALID_ARGUMENT, "remove: negative size");
    if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8)
        return fail(ENERGON_ERR_INVALID_ARGUMENT, "remove: elem_bytes must be 1, 2, 4 or 8");
    CK(launch_remove(padded, cu_seqlens, batch, pad_len, (int64_t)hidden * elem_bytes, packed,
                     (int64_t)batch * pad_len, nullptr, (cudaStream_t)stream),
       "remove");
    return ENERGON_OK;
}

int energon_rce_rebuild_padding(const void* packed, const int32_t* cu_seqlens, int batch, int pad_len, int hidden,
                                int elem_bytes, void* padded, void* stream) {
    g_last_error.clear();
    if (!padded || !cu_seqlens || !packed) return fail(ENERGON_ERR_INVALID_ARGUMENT, "rebuild: NULL pointer");
    if (batch < 0 || pad_len < 0 || hidden < 0) return fail(ENERGON_ERR_INVALID_ARGUMENT, "rebuild: negative size");
    if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8)
        return fail(ENERGON_ERR_INVALID_ARGUMENT, "rebuild: elem_bytes must be 1, 2, 4 or 8");
    CK(launch_rebuild(packed, cu_seqlens, cu_seqlens, batch, pad_len, (int64_t)hidden * elem_bytes,
                      (int64_t)batch * pad_len, padded, (cudaStream_t)stream),
       "rebuild");
    return ENERGON_OK;
}

static int check_head_form(const char* what, const void* a, const void* b, const int32_t* cu, int batch,
                           int pad_len, int parts, int n_heads, int head_dim, int elem_bytes) {
    if (!a || !b || !cu) return fail(ENERGON_ERR_INVALID_ARGUMENT, "%s: NULL pointer", what);
    if (batch < 0 || pad_len < 0 || head_dim < 0 || parts < 1 || n_heads < 1)
        return fail(ENERGON_ERR_INVALID_ARGUMENT, "%s: negative size, or parts / n_heads below 1", what);
    if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4 && elem_bytes != 8)
        return fail(ENERGON_ERR_INVALID_ARGUMENT, "%s: elem_bytes must be 1, 2, 4 or 8", what);
    if ((int64_t)parts * n_heads * head_dim * elem_bytes > (int64_t)0x7fffffff)
        return fail(ENERGON_ERR_INVALID_ARGUMENT, "%s: packed row of 2^31 bytes or more", what);
    if ((int64_t)batch * pad_len > (int64_t)0x7fffff00)
        return fail(ENERGON_ERR_INVALID_ARGUMENT, "%s: batch * pad_len exceeds the int32 token index", what);
    return ENERGON_OK;
}

int energon_rce_transpose_padding_rebuild(const void* packed, const int32_t* cu_seqlens, int batch, int pad_len,
                                          int parts, int n_heads, int head_dim, int elem_bytes, void* heads,
                                          void* stream) {
    g_last_error.clear();
    if (int r = check_head_form("transpose rebuild", packed, heads, cu_seqlens, batch, pad_len, parts, n_heads,
                                head_dim, elem_bytes))
        return r;
    CK(launch_transpose_rebuild(packed, cu_seqlens, batch, pad_len, parts, n_heads, (int64_t)head_dim * elem_bytes,
                                (int64_t)batch * pad_len, heads, (cudaStream_t)stream),
       "transpose rebuild");
    return ENERGON_OK;
}

int energon_rce_transpose_padding_remove(const void* heads, const int32_t* cu_seqlens, int batch, int pad_len,
                                         int parts, int n_heads, int head_dim, int elem_bytes, void* packed,
                                         void* stream) {
    g_last_error.clear();
    if (int r = check_head_form("transpose remove", heads, packed, cu_seqlens, batch, pad_len, parts, n_heads,
                                head_dim, elem_bytes))
        return r;
    CK(launch_transpose_remove(heads, cu_seqlens, batch, pad_len, parts, n_heads, (int64_t)head_dim * elem_bytes,
                               (int64_t)batch * pad_len, packed, (cudaStream_t)stream),
       "transpose remove");
    return ENERGON_OK;
}

size_t energon_workspace_bytes(const energon_layer_config* cfg, int batch, int pad_len) {
    if (check_config(cfg) != ENERGON_OK || check_sizes(batch, pad_len) != ENERGON_OK) return 0;
    return stack_ws_layout(*cfg, batch, pad_len, nullptr).bytes;
}

int energon_layer_forward(const energon_layer_config* cfg, const energon_layer_weights* w, const void* x_packed,
                          const int32_t* cu_seqlens, int batch, int max_len, void* y_packed, int32_t* d_status,
                          void* workspace, size_t ws_bytes, void* stream) {
    g_last_error.clear();
    if (int r = check_config(cfg)) return r;
    if (int r = check_weights(w)) return r;
    if (int r = check_sizes(batch, max_len)) return r;
    if (!x_packed || !cu_seqlens || !y_packed || !workspace)
        return fail(ENERGON_ERR_INVALID_ARGUMENT, "layer: NULL pointer");
    const LayerWs ws = layer_ws_layout(*cfg, batch, max_len, workspace);
    if (ws_bytes < ws.bytes)
        return fail(ENERGON_ERR_WORKSPACE_TOO_SMALL, "layer: workspace %zu < %zu bytes", ws_bytes, ws.bytes);
    return layer_impl(*cfg, *w, x_packed, cu_seqlens, batch, max_len, y_packed, d_status, ws, (cudaStream_t)stream);
}

int energon_stack_forward(const energon_layer_config* cfg, const energon_layer_weights* layers, int n_layers,
                          const void* padded_in, const int32_t* lengths, int batch, int pad_len, int remove_padding,
                          void* padded_out, int32_t* d_status, void* workspace, size_t ws_bytes, void* stream) {
    g_last_error.clear();
    if (int r = check_config(cfg)) return r;
    if (int r = check_sizes(batch, pad_len)) return r;
    if (n_layers < 0 || (n_layers > 0 && !layers)) return fail(ENERGON_ERR_INVALID_ARGUMENT, "stack: bad layers");
    for (int l = 0; l < n_layers; ++l)
        if (int r = check_weights(&layers[l])) return r;
    if (!padded_in || !lengths || !padded_out || !d_status || !workspace)
        return fail(ENERGON_ERR_INVALID_ARGUMENT, "stack: NULL pointer");
    if (padded_in == padded_out) return fail(ENERGON_ERR_INVALID_ARGUMENT, "stack: padded_out aliases padded_in");
    if (remove_padding < 0 || remove_padding > 2)
        return fail(ENERGON_ERR_INVALID_ARGUMENT, "stack: remove_padding must be 0, 1 or 2");
    const StackWs ws = stack_ws_layout(*cfg, batch, pad_len, workspace);
    if (ws_bytes < ws.bytes)
        return fail(ENERGON_ERR_WORKSPACE_TOO_SMALL, "stack: workspace %zu < %zu bytes", ws_bytes, ws.bytes);
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t row_bytes = (int64_t)cfg->hidden * (int64_t)dtype_bytes(cfg->dtype);
    const int64_t R = rows_alloc(batch, pad_len);

    CK(traced("offsets", st, [&] { return launch_offsets(lengths, batch, pad_len, ws.cu, d_status, st); }),
       "offsets");
    if (remove_padding == 1 && n_layers == 0) {
        CK(traced("remove_padding", st,
                  [&] { return launch_remove(padded_in, ws.cu, batch, pad_len, row_bytes, ws.x, R, d_status, st); }),
           "remove");
        CK(traced("rebuild_padding", st,
                  [&] { return launch_rebuild(ws.x, ws.cu, ws.cu, batch, pad_len, row_bytes, R, padded_out, st); }),
           "rebuild");
    } else if (remove_padding == 1) {
        // The packing is fused into the first LayerNorm (it gathers the valid rows of
        // padded_in and writes them to the residual stream ws.x) and the scatter back into
        // the last FFN2 GEMM's epilogue (each row stored at its padded position); the pad
        // rows of padded_out are zeroed up front.
        CK(traced("zero_pads", st, [&] { return launch_zero_pads(ws.cu, batch, pad_len, row_bytes, padded_out, st); }),
           "zero pads");
        bool scattered = false;
        for (int l = 0; l < n_layers; ++l) {
            const energon_layer_weights& w = layers[l];
            if (int r = attention_sublayer(*cfg, w, ws.x, ws.cu, batch, pad_len, ws.layer.x1, d_status, ws.layer, st,
                                           l == 0 ? padded_in : nullptr))
                return r;
            if (int r = mlp_sublayer(*cfg, w, ws.layer.x1, ws.cu, batch, pad_len, ws.x, d_status, ws.layer, st,
                                     l + 1 == n_layers ? padded_out : nullptr, &scattered))
                return r;
        }
        if (!scattered)
            CK(traced("rebuild_padding", st,
                      [&] {
                          return launch_rebuild(ws.x, ws.cu, ws.cu, batch, pad_len, row_bytes, R, padded_out, st);
                      }),
               "rebuild");
    } else if (remove_padding == 2) {
        // Elimination for the MLP only, as the QbitAI article's "Runtime" section states it:
        // each layer's attention sub-layer runs on all batch * pad_len rows; its output is
        // packed (remove), the MLP sub-layer runs on the valid tokens, and the result is
        // scattered back (rebuild, zero pads) for the next layer.
        CK(traced("padded_starts", st, [&] { return launch_padded_starts(batch, pad_len, ws.cu_pad, d_status, st); }),
           "padded starts");
        const void* src = padded_in;
        float* x1_pk = static_cast<float*>(ws.layer.qkv);   // free once attention has consumed it
        void* y_pk = ws.layer.o;                            // free once the out-projection has consumed it
        const int64_t x1_row_bytes = (int64_t)cfg->hidden * (int64_t)sizeof(float);
        for (int l = 0; l < n_layers; ++l) {
            if (int r = attention_sublayer(*cfg, layers[l], src, ws.cu_pad, batch, pad_len, ws.layer.x1, d_status,
                                           ws.layer, st))
                return r;
            CK(traced("remove_padding", st,
                      [&] {
                          return launch_remove(ws.layer.x1, ws.cu, batch, pad_len, x1_row_bytes, x1_pk, R, d_status,
                                               st);
                      }),
               "remove");
            if (int r = mlp_sublayer(*cfg, layers[l], x1_pk, ws.cu, batch, pad_len, y_pk, d_status, ws.layer, st))
                return r;
            void* dst = (l + 1 == n_layers) ? padded_out : ws.x;
            CK(traced("rebuild_padding", st,
                      [&] { return launch_rebuild(y_pk, ws.cu, ws.cu, batch, pad_len, row_bytes, R, dst, st); }),
               "rebuild");
            src = ws.x;
        }
        if (n_layers == 0)
            CK(traced("rebuild_padding", st,
                      [&] {
                          return launch_rebuild(padded_in, ws.cu_pad, ws.cu, batch, pad_len, row_bytes, R, padded_out,
                                                st);
                      }),
               "rebuild");
    } else {
        // Padded baseline: every one of the batch * pad_len rows goes through the layers.
        CK(traced("padded_starts", st, [&] { return launch_padded_starts(batch, pad_len, ws.cu_pad, d_status, st); }),
           "padded starts");
        const void* src = padded_in;
        for (int l = 0; l < n_layers; ++l) {
            if (int r = layer_impl(*cfg, layers[l], src, ws.cu_pad, batch, pad_len, ws.x, d_status, ws.layer, st))
                return r;
            src = ws.x;
        }
        CK(traced("rebuild_padding", st,
                  [&] { return launch_rebuild(src, ws.cu_pad, ws.cu, batch, pad_len, row_bytes, R, padded_out, st); }),
           "rebuild");
    }
    return ENERGON_OK;
}

int energon_trace_start(void) {
    g_last_error.clear();
    g_trace.clear();
    g_event_used = 0;
    g_trace_on = true;
    return ENERGON_OK;
}

int energon_trace_stop(energon_trace_entry* entries, int capacity, int* n_entries) {
    g_last_error.clear();
    g_trace_on = false;
    std::vector<energon_trace_entry> agg;
    for (const TraceRec& r : g_trace) {
        cudaError_t e = cudaEventSynchronize(r.stop);
        if (e != cudaSuccess) return cuda_fail(e, "trace: event synchronise");
        float ms = 0.0f;
        e = cudaEventElapsedTime(&ms, r.start, r.stop);
        if (e != cudaSuccess) return cuda_fail(e, "trace: elapsed time");
        size_t i = 0;
        while (i < agg.size() && strcmp(agg[i].name, r.name) != 0) ++i;
        if (i == agg.size()) {
            energon_trace_entry t{};
            snprintf(t.name, sizeof(t.name), "%s", r.name);
            agg.push_back(t);
        }
        agg[i].launches += 1;
        agg[i].total_ms += ms;
    }
    g_trace.clear();
    g_event_used = 0;
    if (n_entries) *n_entries = (int)agg.size();
    for (int i = 0; entries && i < capacity && i < (int)agg.size(); ++i) entries[i] = agg[i];
    return ENERGON_OK;
}

int energon_layer_fold_weights(const energon_layer_config* cfg, const energon_layer_weights* w, float* fold,
                               void* stream) {
    g_last_error.clear();
    if (int r = check_config(cfg)) return r;
    if (!w || !w->w_qkv || !w->b_qkv || !w->ln1_g || !w->ln1_b || !fold)
        return fail(ENERGON_ERR_INVALID_ARGUMENT, "fold weights: NULL pointer");
    if ((uintptr_t)fold % 16 != 0) return fail(ENERGON_ERR_MISALIGNED, "fold weights: fold must be 16-byte aligned");
    const int H = cfg->hidden;
    CK(launch_ln_fold_weights(cfg->dtype, w->w_qkv, w->ln1_g, w->ln1_b, w->b_qkv, 3 * H, H, fold,
                              fold + 3 * (size_t)H, nullptr, (cudaStream_t)stream),
       "fold weights");
    return ENERGON_OK;
}

int energon_kernel_binary_version(int* version) {
    g_last_error.clear();
    if (!version) return fail(ENERGON_ERR_INVALID_ARGUMENT, "kernel_binary_version: NULL pointer");
    CK(kernel_binary_version(version), "kernel_binary_version");
    return ENERGON_OK;
}

int energon_selftest_bounded_wait(int32_t* d_status, uint32_t timeout_us, void* stream) {
    g_last_error.clear();
    if (!d_status) return fail(ENERGON_ERR_INVALID_ARGUMENT, "selftest: NULL status");
    CK(launch_wait_selftest(d_status, (uint64_t)timeout_us * 1000ull, (cudaStream_t)stream), "selftest");
    return ENERGON_OK;
}

}  // extern "C"
