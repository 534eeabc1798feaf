// Causal self-attention on packed tokens with the 5th-generation tensor cores.
//
// The attention of the GPT-3 layer run on the valid tokens only (EnergonAI
// README, "Scaling Ability": redundant computation elimination), driven by
// cu_seqlens: sequence b owns packed rows cu[b] .. cu[b+1]-1 of the fused
// projection qkv [rows, 3H] (columns Q | K | V, head-major inside each).  For
// head j and position s:  o_j(s) = sum_{t <= s} softmax_t(q_j(s) . k_j(t) / sqrt(d)) v_j(t).
//
// One CTA = 128 queries of one (sequence, head), head_dim 128, 128 threads;
// thread i owns query row i, which is TMEM lane i.  Per block of KB keys:
//   TMA   Q (once) and the key block's K and V tiles straight from the packed
//         qkv rows (128-byte swizzle), plus the low halves of Q and K (qk_lo)
//   MMA   S = Q K^T (tcgen05.mma kind::f16, M = 128, N = KB, K = 128) into TMEM
//         columns 0..KB-1, from the two-term Q and K: Qh Kh^T + Qh Kl^T + Ql Kh^T
//   ALU   each thread reads its S row from TMEM, applies the causal mask, keeps
//         a running max / sum (online softmax, fp32, exp2 with the scale folded
//         in) and writes P, rounded to the storage type, into shared memory
//   MMA   O += P V  (V used as an MN-major operand, no transpose) into TMEM 128..255
// With the low halves, KB = 64 keeps a CTA at 112 KiB of shared memory and 256
// TMEM columns, so that two CTAs share an SM and one's copies and MMAs overlap
// the other's softmax.  Keys past the sequence are masked; their V rows are
// zeroed in shared memory first, so stale workspace contents can never reach a
// valid row (0 * NaN).  A query tile visits the key blocks 0 .. its diagonal that
// hold keys of the sequence, whether the sequence is packed or padded.
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace energon {

namespace {
constexpr int ATQ = 128;                 // queries per CTA
constexpr int AHD = 128;                 // head dim
constexpr int QTILE = 128 * 64 * 2;      // 128 rows x 64 columns of 16-bit = 16 KiB, one swizzle block column
constexpr uint32_t AT_TMEM_COLS = 256;   // S: 0..KB-1, O: 128..255
constexpr int KB_LO = 64;                // key block with the low halves (two CTAs per SM)

// Shared memory of one CTA: Q (2 tiles), the key block's K and V (2 boxes each of KB rows
// x 64 columns), with LO the low halves of Q (2 tiles) and K (2 boxes); 128 bytes of
// barriers; slack to align the tiles to 1024 bytes.
template <int KB, bool LO>
struct AttnCfg {
    static constexpr int KTILE = KB * 64 * 2;
    static constexpr int TILES = (LO ? 4 : 2) * QTILE + (LO ? 6 : 4) * KTILE;
    static constexpr int SMEM = TILES + 1024;  // barriers go in the alignment slack or after the tiles
};
}  // namespace

struct AttnTcParams {
    const int32_t* cu;
    void* out;
    int32_t* status;
    int H;
    float scale_log2e;  // log2(e) / sqrt(head_dim)
    uint64_t timeout_ns;
};

// Thread 0 waits (bounded); every thread learns the outcome at the same barrier.
__device__ __forceinline__ bool block_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
    int ok = 1;
    if (threadIdx.x == 0) ok = mbar_wait_bounded(bar, parity, nullptr, timeout_ns) ? 1 : 0;
    return __syncthreads_and(ok) != 0;
}

// tmq / tmql: Q and its low halves in boxes of 128 rows; tmk / tmkl: K, V and K's low
// halves in boxes of KB rows.
template <typename T, int KB, bool LO>
__global__ void __launch_bounds__(128) attn_tc_kernel(const __grid_constant__ CUtensorMap tmq,
                                                      const __grid_constant__ CUtensorMap tmk,
                                                      const __grid_constant__ CUtensorMap tmql,
                                                      const __grid_constant__ CUtensorMap tmkl, const AttnTcParams p) {
    using C = AttnCfg<KB, LO>;
    constexpr int KT = C::KTILE;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = base;                    // Q: head dims 0..63 | 64..127
    uint8_t* sQl = sQ + 2 * QTILE;         // low half of Q (LO)
    uint8_t* sK = sQ + (LO ? 4 : 2) * QTILE;  // K: head dims 0..63 | 64..127; then P (128 x KB)
    uint8_t* sKl = sK + 2 * KT;            // low half of K (LO)
    uint8_t* sV = sK + (LO ? 4 : 2) * KT;  // V: head dims 0..63 | 64..127, one row per key
    // barriers: in the alignment slack when it holds them, else after the tiles
    uint64_t* bars = (base - smem_raw >= 128) ? reinterpret_cast<uint64_t*>(smem_raw)
                                              : reinterpret_cast<uint64_t*>(base + C::TILES);
    uint64_t* bar_q = bars;
    uint64_t* bar_kv = bars + 1;
    uint64_t* bar_mma = bars + 2;
    uint64_t* drain = bars + 3;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);

    const int tid = threadIdx.x, warp = tid >> 5;
    if (status_bad(p.status)) return;
    const int b = blockIdx.z, j = blockIdx.y, q0 = blockIdx.x * ATQ;
    const int start = p.cu[b], len = p.cu[b + 1] - start;
    if (q0 >= len) return;
    // causal: key blocks 0 .. the one holding query q0 + 127, and only blocks with keys < len
    const int n_kb = min((q0 + ATQ - 1) / KB + 1, (len + KB - 1) / KB);
    const int q = q0 + tid;
    const bool row_ok = q < len;

    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, AT_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t S_t = tmem + lane_base, O_t = tmem + lane_base + 128;

    // Q | K | V at columns j*d, H + j*d, 2H + j*d of qkv; the low halves at j*d, H + j*d of qk_lo
    const int colQ = j * AHD, colK = p.H + j * AHD, colV = 2 * p.H + j * AHD;
    bool q_pending = false, kv_pending = false;
    uint32_t kv_parity = 0;
    auto issue_kv = [&](int kb) {
        const int y = start + kb * KB;
        mbar_arrive_expect_tx(bar_kv, (LO ? 6 : 4) * KT);
        tma_load_2d(sK, &tmk, bar_kv, colK, y);
        tma_load_2d(sK + KT, &tmk, bar_kv, colK + 64, y);
        tma_load_2d(sV, &tmk, bar_kv, colV, y);
        tma_load_2d(sV + KT, &tmk, bar_kv, colV + 64, y);
        if (LO) {
            tma_load_2d(sKl, &tmkl, bar_kv, colK, y);
            tma_load_2d(sKl + KT, &tmkl, bar_kv, colK + 64, y);
        }
        kv_pending = true;
    };
    if (tid == 0) {
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmk);
        if (LO) {
            tma_prefetch_desc(&tmql);
            tma_prefetch_desc(&tmkl);
        }
        mbar_arrive_expect_tx(bar_q, (LO ? 4 : 2) * QTILE);
        tma_load_2d(sQ, &tmq, bar_q, colQ, start + q0);
        tma_load_2d(sQ + QTILE, &tmq, bar_q, colQ + 64, start + q0);
        if (LO) {
            tma_load_2d(sQl, &tmql, bar_q, colQ, start + q0);
            tma_load_2d(sQl + QTILE, &tmql, bar_q, colQ + 64, start + q0);
        }
        q_pending = true;
        issue_kv(0);
    }
    constexpr uint32_t fmt = std::is_same<T, __half>::value ? 0u : 1u;
    constexpr uint32_t idesc_s = idesc_f16(fmt, ATQ, KB, 0);
    constexpr uint32_t idesc_o = idesc_f16(fmt, ATQ, AHD, 1);

    float m_i = -INFINITY, l_i = 0.0f;
    uint32_t mma_phase = 0;
    bool ok = block_wait(bar_q, 0, p.timeout_ns);
    if (ok) q_pending = false;
    uint32_t r[32];
    for (int kb = 0; ok && kb < n_kb; ++kb) {
        ok = block_wait(bar_kv, kv_parity, p.timeout_ns);
        if (!ok) break;
        kv_pending = false;
        kv_parity ^= 1u;
        const int kbase = kb * KB;
        if (tid < KB && kbase + tid >= len) {  // key row past the sequence: zero its V row
            const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                reinterpret_cast<uint4*>(sV + tid * 128)[c] = z;
                reinterpret_cast<uint4*>(sV + KT + tid * 128)[c] = z;
            }
            fence_proxy_async_smem();
        }
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < AHD / 16; ++k) {
                const uint64_t a = smem_desc_k128(smem_u32(sQ + (k >> 2) * QTILE)) + 2 * (k & 3);
                const uint64_t bk = smem_desc_k128(smem_u32(sK + (k >> 2) * KT)) + 2 * (k & 3);
                umma_f16(tmem, a, bk, idesc_s, k > 0 ? 1u : 0u);
                if (LO) {
                    const uint64_t al = smem_desc_k128(smem_u32(sQl + (k >> 2) * QTILE)) + 2 * (k & 3);
                    const uint64_t bl = smem_desc_k128(smem_u32(sKl + (k >> 2) * KT)) + 2 * (k & 3);
                    umma_f16(tmem, a, bl, idesc_s, 1u);
                    umma_f16(tmem, al, bk, idesc_s, 1u);
                }
            }
            umma_commit(bar_mma);
        }
        ok = block_wait(bar_mma, mma_phase, p.timeout_ns);
        mma_phase ^= 1u;
        if (!ok) break;
        tc_fence_after();

        // ---- online softmax of this thread's row
        const int nvalid = row_ok ? min(KB, q - kbase + 1) : 0;  // keys kbase .. kbase+nvalid-1 are visible
        float mx = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < KB / 32; ++c) {
            tmem_ld_x32(S_t + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e)
                if (c * 32 + e < nvalid) mx = fmaxf(mx, __uint_as_float(r[e]));
        }
        const float m_new = row_ok ? fmaxf(m_i, mx) : 0.0f;
        const float alpha = row_ok ? exp2f((m_i - m_new) * p.scale_log2e) : 1.0f;
        float rs = 0.0f;
        uint8_t* sP = sK;  // P: 128 rows x KB keys, 128-byte rows, one swizzle block column per 64 keys
#pragma unroll 1
        for (int c = 0; c < KB / 32; ++c) {
            tmem_ld_x32(S_t + c * 32, r);
            tmem_wait_ld();
            float pv[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                pv[e] = (c * 32 + e < nvalid) ? exp2f((__uint_as_float(r[e]) - m_new) * p.scale_log2e) : 0.0f;
                rs += pv[e];
            }
            // keys c*32 .. c*32+31: swizzle block c/2, 16-byte chunks (c%2)*4 .. +3 of row tid
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                uint4 w;
                w.x = pack2<T>(pv[8 * g + 0], pv[8 * g + 1]);
                w.y = pack2<T>(pv[8 * g + 2], pv[8 * g + 3]);
                w.z = pack2<T>(pv[8 * g + 4], pv[8 * g + 5]);
                w.w = pack2<T>(pv[8 * g + 6], pv[8 * g + 7]);
                const int ch = (c & 1) * 4 + g;
                *reinterpret_cast<uint4*>(sP + (c >> 1) * QTILE + tid * 128 + ((ch ^ (tid & 7)) << 4)) = w;
            }
        }
        l_i = l_i * alpha + rs;
        if (row_ok) m_i = m_new;
        if (kb > 0) {  // earlier blocks were summed against a smaller max: rescale O
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                tmem_ld_x32(O_t + c * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                tmem_st_x32(O_t + c * 32, r);
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < KB / 16; ++k) {
                const uint64_t a = smem_desc_k128(smem_u32(sP + (k >> 2) * QTILE)) + 2 * (k & 3);
                const uint64_t bv = smem_desc_mn128(smem_u32(sV + k * 2048), KT, 1024);
                umma_f16(tmem + 128, a, bv, idesc_o, (kb > 0 || k > 0) ? 1u : 0u);
            }
            umma_commit(bar_mma);
        }
        ok = block_wait(bar_mma, mma_phase, p.timeout_ns);
        mma_phase ^= 1u;
        if (!ok) break;
        tc_fence_after();
        if (kb + 1 < n_kb && tid == 0) issue_kv(kb + 1);
    }
    if (ok) {
        const float inv = row_ok ? 1.0f / l_i : 0.0f;
        T* orow = static_cast<T*>(p.out) + (int64_t)(start + q) * p.H + j * AHD;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            tmem_ld_x32(O_t + c * 32, r);
            tmem_wait_ld();
            if (row_ok) {
                uint4* op = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint4 w;
                    w.x = pack2<T>(__uint_as_float(r[8 * g + 0]) * inv, __uint_as_float(r[8 * g + 1]) * inv);
                    w.y = pack2<T>(__uint_as_float(r[8 * g + 2]) * inv, __uint_as_float(r[8 * g + 3]) * inv);
                    w.z = pack2<T>(__uint_as_float(r[8 * g + 4]) * inv, __uint_as_float(r[8 * g + 5]) * inv);
                    w.w = pack2<T>(__uint_as_float(r[8 * g + 6]) * inv, __uint_as_float(r[8 * g + 7]) * inv);
                    op[g] = w;
                }
            }
        }
    } else if (tid == 0) {
        // A bounded wait ran out: record it, let every MMA and copy in flight finish, leave.
        status_or(p.status, ENERGON_DEVICE_TIMEOUT);
        umma_commit(drain);
        mbar_wait_bounded(drain, 0, nullptr, p.timeout_ns);
        if (q_pending) mbar_wait_bounded(bar_q, 0, nullptr, p.timeout_ns);
        if (kv_pending) mbar_wait_bounded(bar_kv, kv_parity, nullptr, p.timeout_ns);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, AT_TMEM_COLS);
}

// ------------------------------------------------------------------ host side

static PFN_cuTensorMapEncodeTiled_v12000 attn_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

bool attention_tc_supported(int dtype, int H, int n_heads, const void* qkv, const void* qk_lo, const void* o,
                            int qkv_rows) {
    if (dtype != ENERGON_F16 && dtype != ENERGON_BF16) return false;
    if (n_heads <= 0 || H % n_heads != 0 || H / n_heads != AHD) return false;
    if (((uintptr_t)qkv | (uintptr_t)qk_lo | (uintptr_t)o) % 16 != 0 || qkv_rows < 1) return false;
    return attn_encode_fn() != nullptr;
}

// [rows, cols] 16-bit tensor, box 64 x box_rows, 128-byte swizzle.
static CUresult attn_tmap(CUtensorMap* m, int dtype, const void* ptr, int64_t cols, int64_t rows, uint32_t box_rows) {
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt =
        dtype == ENERGON_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    return attn_encode_fn()(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

template <typename T, int KB, bool LO>
static cudaError_t attn_tc_launch(const void* qkv, const void* qk_lo, int dtype, int H, int qkv_rows,
                                  const AttnTcParams& p, dim3 grid, cudaStream_t st) {
    CUtensorMap tmq, tmk, tmql, tmkl;
    if (attn_tmap(&tmq, dtype, qkv, 3 * (int64_t)H, qkv_rows, ATQ) != CUDA_SUCCESS ||
        attn_tmap(&tmk, dtype, qkv, 3 * (int64_t)H, qkv_rows, KB) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    if (LO) {
        if (attn_tmap(&tmql, dtype, qk_lo, 2 * (int64_t)H, qkv_rows, ATQ) != CUDA_SUCCESS ||
            attn_tmap(&tmkl, dtype, qk_lo, 2 * (int64_t)H, qkv_rows, KB) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    } else {
        tmql = tmq, tmkl = tmk;
    }
    using C = AttnCfg<KB, LO>;
    cudaError_t e = prepare_smem((const void*)attn_tc_kernel<T, KB, LO>, C::SMEM);
    if (e != cudaSuccess) return e;
    attn_tc_kernel<T, KB, LO><<<grid, 128, C::SMEM, st>>>(tmq, tmk, tmql, tmkl, p);
    return cudaGetLastError();
}

cudaError_t launch_attention_tc(int dtype, const void* qkv, const void* qk_lo, void* o, const int32_t* cu, int batch,
                                int max_len, int H, int n_heads, int qkv_rows, int32_t* status, uint64_t timeout_ns,
                                cudaStream_t st) {
    if (batch <= 0 || max_len <= 0) return cudaSuccess;
    AttnTcParams p;
    p.cu = cu;
    p.out = o;
    p.status = status;
    p.H = H;
    p.scale_log2e = (float)(1.4426950408889634 / sqrt((double)AHD));
    p.timeout_ns = timeout_ns;
    dim3 grid((max_len + ATQ - 1) / ATQ, n_heads, batch);
    // With the low halves, 64-key blocks fit two CTAs per SM; without them 128-key blocks do.
    if (dtype == ENERGON_BF16)
        return qk_lo ? attn_tc_launch<__nv_bfloat16, KB_LO, true>(qkv, qk_lo, dtype, H, qkv_rows, p, grid, st)
                     : attn_tc_launch<__nv_bfloat16, 128, false>(qkv, qk_lo, dtype, H, qkv_rows, p, grid, st);
    return qk_lo ? attn_tc_launch<__half, KB_LO, true>(qkv, qk_lo, dtype, H, qkv_rows, p, grid, st)
                 : attn_tc_launch<__half, 128, false>(qkv, qk_lo, dtype, H, qkv_rows, p, grid, st);
}

}  // namespace energon
