// Causal self-attention on packed tokens with the 5th-generation tensor cores.
//
// The attention of the GPT-3 layer run on the valid tokens only (EnergonAI
// README, "Scaling Ability": redundant computation elimination), driven by
// cu_seqlens: sequence b owns packed rows cu[b] .. cu[b+1]-1 of the fused
// projection qkv [rows, 3H] (columns Q | K | V, head-major inside each).  For
// head j and position s:  o_j(s) = sum_{t <= s} softmax_t(q_j(s) . k_j(t) / sqrt(d)) v_j(t).
//
// One CTA = 128 queries of one (sequence, head), head_dim 128, 128 threads;
// thread i owns query row i, which is TMEM lane i.  Per block of 64 keys:
//   TMA   Q (once) and the key block's K and V tiles straight from the packed
//         qkv rows (128-byte swizzle), plus the low halves of Q and K (qk_lo)
//   MMA   S = Q K^T (tcgen05.mma kind::f16, M = 128, N = 64, K = 128) into TMEM
//         columns 0..63, from the two-term Q and K: Qh Kh^T + Qh Kl^T + Ql Kh^T
//   ALU   each thread reads its S row from TMEM, applies the causal mask, keeps
//         a running max / sum (online softmax, fp32, exp2 with the scale folded
//         in) and writes P, rounded to the storage type, back into TMEM
//         (columns 64..95, two keys per column)
//   MMA   O += P V with P read from TMEM and V from shared memory as an MN-major
//         operand (no transpose), into TMEM columns 128..255
//   out   O / l staged in the Q buffer and stored by TMA (a full tile) or row by row with
//         whole 256-byte rows per half warp (a partial tile)
// P never touches shared memory, so the K buffer is free as soon as the S MMAs
// are done: the next block's K is fetched while this block's softmax runs, and
// the next block's V while the next S and softmax run.  A CTA holds 112 KiB of
// shared memory and 256 TMEM columns, so that two CTAs share an SM and one's
// copies and MMAs overlap the other's softmax.  Keys past the sequence are
// masked; their V rows are zeroed in shared memory first, so stale workspace
// contents can never reach a valid row (0 * NaN).  A query tile visits the key
// blocks 0 .. its diagonal that hold keys of the sequence, whether the sequence
// is packed or padded.
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace energon {

namespace {
constexpr int ATQ = 128;                 // queries per CTA
constexpr int AHD = 128;                 // head dim
constexpr int KB = 64;                   // keys per block
constexpr int QTILE = 128 * 64 * 2;      // 128 rows x 64 columns of 16-bit = 16 KiB, one swizzle block column
constexpr int KTILE = KB * 64 * 2;       // KB rows x 64 columns of 16-bit
constexpr uint32_t AT_TMEM_COLS = 256;   // S: 0..63, P: 64..95, O: 128..255
constexpr uint32_t P_COL = 64, O_COL = 128;

// Shared memory of one CTA: Q (2 tiles), the key block's K and V (2 boxes each of 64 rows
// x 64 columns), with LO the low halves of Q (2 tiles) and K (2 boxes); barriers in the
// alignment slack or after the tiles.
template <bool LO>
struct AttnCfg {
    static constexpr int TILES = (LO ? 4 : 2) * QTILE + (LO ? 6 : 4) * KTILE;
    static constexpr int SMEM = TILES + 1024;
};

// O (or S) += A B with A (M = 128 rows, 16-bit, two per 32-bit column) read from TMEM.
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                                uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 lanes x 32 bits, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
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
// halves in boxes of 64 rows.
template <typename T, bool LO>
__global__ void __launch_bounds__(128) attn_tc_kernel(const __grid_constant__ CUtensorMap tmq,
                                                      const __grid_constant__ CUtensorMap tmk,
                                                      const __grid_constant__ CUtensorMap tmql,
                                                      const __grid_constant__ CUtensorMap tmkl,
                                                      const __grid_constant__ CUtensorMap tmo, const AttnTcParams p) {
    using C = AttnCfg<LO>;
    constexpr int KT = KTILE;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = base;                       // Q: head dims 0..63 | 64..127
    uint8_t* sQl = sQ + 2 * QTILE;            // low half of Q (LO)
    uint8_t* sK = sQ + (LO ? 4 : 2) * QTILE;  // K: head dims 0..63 | 64..127
    uint8_t* sKl = sK + 2 * KT;               // low half of K (LO)
    uint8_t* sV = sK + (LO ? 4 : 2) * KT;     // V: head dims 0..63 | 64..127, one row per key
    // barriers: in the alignment slack when it holds them, else after the tiles
    uint64_t* bars = (base - smem_raw >= 128) ? reinterpret_cast<uint64_t*>(smem_raw)
                                              : reinterpret_cast<uint64_t*>(base + C::TILES);
    uint64_t* bar_q = bars;      // Q landed
    uint64_t* bar_k = bars + 1;  // the block's K landed
    uint64_t* bar_v = bars + 2;  // the block's V landed
    uint64_t* bar_s = bars + 3;  // the S MMAs (and every MMA before them) done
    uint64_t* bar_o = bars + 4;  // the PV MMAs done
    uint64_t* drain = bars + 5;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 6);

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
        for (int i = 0; i < 6; ++i) mbar_init(&bars[i], 1);
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
    const uint32_t S_t = tmem + lane_base, P_t = tmem + lane_base + P_COL, O_t = tmem + lane_base + O_COL;

    // Q | K | V at columns j*d, H + j*d, 2H + j*d of qkv; the low halves at j*d, H + j*d of qk_lo
    const int colQ = j * AHD, colK = p.H + j * AHD, colV = 2 * p.H + j * AHD;
    bool q_pending = false, k_pending = false, v_pending = false;  // thread 0's copies in flight
    uint32_t k_par = 0, v_par = 0;
    auto issue_k = [&](int kb) {
        const int y = start + kb * KB;
        mbar_arrive_expect_tx(bar_k, (LO ? 4 : 2) * KT);
        tma_load_2d(sK, &tmk, bar_k, colK, y);
        tma_load_2d(sK + KT, &tmk, bar_k, colK + 64, y);
        if (LO) {
            tma_load_2d(sKl, &tmkl, bar_k, colK, y);
            tma_load_2d(sKl + KT, &tmkl, bar_k, colK + 64, y);
        }
        k_pending = true;
    };
    auto issue_v = [&](int kb) {
        const int y = start + kb * KB;
        mbar_arrive_expect_tx(bar_v, 2 * KT);
        tma_load_2d(sV, &tmk, bar_v, colV, y);
        tma_load_2d(sV + KT, &tmk, bar_v, colV + 64, y);
        v_pending = true;
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
        issue_k(0);
        issue_v(0);
    }
    constexpr uint32_t fmt = std::is_same<T, __half>::value ? 0u : 1u;
    constexpr uint32_t idesc_s = idesc_f16(fmt, ATQ, KB, 0);
    constexpr uint32_t idesc_o = idesc_f16(fmt, ATQ, AHD, 1);

    float m_i = -INFINITY, l_i = 0.0f;
    uint32_t s_phase = 0, o_phase = 0;
    bool ok = block_wait(bar_q, 0, p.timeout_ns);
    if (ok) q_pending = false;
    uint32_t r[32];
    for (int kb = 0; ok && kb < n_kb; ++kb) {
        ok = block_wait(bar_k, k_par, p.timeout_ns);
        if (!ok) break;
        k_pending = false;
        k_par ^= 1u;
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
            umma_commit(bar_s);
        }
        ok = block_wait(bar_s, s_phase, p.timeout_ns);
        s_phase ^= 1u;
        if (!ok) break;
        tc_fence_after();
        // The S MMAs are done, and every MMA before them (the previous block's PV): the K
        // buffer is free for the next block, O holds the sum over the earlier blocks.
        if (tid == 0 && kb + 1 < n_kb) issue_k(kb + 1);

        // ---- online softmax of this thread's row
        const int kbase = kb * KB;
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
#pragma unroll 1
        for (int c = 0; c < KB / 32; ++c) {
            tmem_ld_x32(S_t + c * 32, r);
            tmem_wait_ld();
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float p0 = (c * 32 + 2 * e < nvalid)
                                     ? exp2f((__uint_as_float(r[2 * e]) - m_new) * p.scale_log2e) : 0.0f;
                const float p1 = (c * 32 + 2 * e + 1 < nvalid)
                                     ? exp2f((__uint_as_float(r[2 * e + 1]) - m_new) * p.scale_log2e) : 0.0f;
                rs += p0;
                rs += p1;
                pk[e] = pack2<T>(p0, p1);  // keys 2e, 2e + 1 of this chunk in one column
            }
            tmem_st_x16(P_t + c * 16, pk);
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
        }
        tmem_wait_st();
        tc_fence_before();
        ok = block_wait(bar_v, v_par, p.timeout_ns);  // the block's V has landed
        if (!ok) break;
        v_pending = false;
        v_par ^= 1u;
        if (tid < KB && kbase + tid >= len) {  // key row past the sequence: zero its V row
            const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                reinterpret_cast<uint4*>(sV + tid * 128)[c] = z;
                reinterpret_cast<uint4*>(sV + KT + tid * 128)[c] = z;
            }
            fence_proxy_async_smem();
        }
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < KB / 16; ++k) {
                const uint64_t bv = smem_desc_mn128(smem_u32(sV + k * 2048), KT, 1024);
                umma_f16_tmem_a(tmem + O_COL, tmem + P_COL + (uint32_t)(k * 8), bv, idesc_o,
                                (kb > 0 || k > 0) ? 1u : 0u);
            }
            umma_commit(bar_o);
        }
        ok = block_wait(bar_o, o_phase, p.timeout_ns);
        o_phase ^= 1u;
        if (!ok) break;
        tc_fence_after();
        if (tid == 0 && kb + 1 < n_kb) issue_v(kb + 1);  // the PV MMAs no longer read V
    }
    if (ok) {
        // O, normalised and rounded, staged in the Q buffer (no MMA reads it any more) in the
        // 128-byte swizzle; a tile whose 128 rows are all valid leaves with two TMA stores, a
        // partial one row by row, 16 lanes x 16 bytes per row (whole 256-byte rows per
        // instruction instead of one row per lane)
        const float inv = row_ok ? 1.0f / l_i : 0.0f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            tmem_ld_x32(O_t + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                uint4 w;
                w.x = pack2<T>(__uint_as_float(r[8 * g + 0]) * inv, __uint_as_float(r[8 * g + 1]) * inv);
                w.y = pack2<T>(__uint_as_float(r[8 * g + 2]) * inv, __uint_as_float(r[8 * g + 3]) * inv);
                w.z = pack2<T>(__uint_as_float(r[8 * g + 4]) * inv, __uint_as_float(r[8 * g + 5]) * inv);
                w.w = pack2<T>(__uint_as_float(r[8 * g + 6]) * inv, __uint_as_float(r[8 * g + 7]) * inv);
                const int ch = (c & 1) * 4 + g;
                *reinterpret_cast<uint4*>(sQ + (c >> 1) * QTILE + tid * 128 + ((ch ^ (tid & 7)) << 4)) = w;
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        const int rows = min(ATQ, len - q0);
        if (rows == ATQ) {
            if (tid == 0) {
                tma_store_2d(&tmo, sQ, j * AHD, start + q0);
                tma_store_2d(&tmo, sQ + QTILE, j * AHD + 64, start + q0);
                bulk_commit();
                bulk_wait_read<0>();  // the buffer stays until the stores have read it
            }
        } else {
            const int lane = tid & 31, k = lane & 15;
            for (int rr = warp * 2 + (lane >> 4); rr < rows; rr += 8) {
                const uint4 w =
                    *reinterpret_cast<const uint4*>(sQ + (k >> 3) * QTILE + rr * 128 + (((k & 7) ^ (rr & 7)) << 4));
                reinterpret_cast<uint4*>(static_cast<T*>(p.out) + (int64_t)(start + q0 + rr) * p.H + j * AHD)[k] = w;
            }
        }
    } else if (tid == 0) {
        // A bounded wait ran out: record it, let every MMA and copy in flight finish, leave.
        status_or(p.status, ENERGON_DEVICE_TIMEOUT);
        umma_commit(drain);
        mbar_wait_bounded(drain, 0, nullptr, p.timeout_ns);
        if (q_pending) mbar_wait_bounded(bar_q, 0, nullptr, p.timeout_ns);
        if (k_pending) mbar_wait_bounded(bar_k, k_par, nullptr, p.timeout_ns);
        if (v_pending) mbar_wait_bounded(bar_v, v_par, nullptr, p.timeout_ns);
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

template <typename T, bool LO>
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
    CUtensorMap tmo;  // the output [rows, H], 128-row boxes
    if (attn_tmap(&tmo, dtype, p.out, H, qkv_rows, ATQ) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    using C = AttnCfg<LO>;
    cudaError_t e = prepare_smem((const void*)attn_tc_kernel<T, LO>, C::SMEM);
    if (e != cudaSuccess) return e;
    attn_tc_kernel<T, LO><<<grid, 128, C::SMEM, st>>>(tmq, tmk, tmql, tmkl, tmo, p);
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
    if (dtype == ENERGON_BF16)
        return qk_lo ? attn_tc_launch<__nv_bfloat16, true>(qkv, qk_lo, dtype, H, qkv_rows, p, grid, st)
                     : attn_tc_launch<__nv_bfloat16, false>(qkv, qk_lo, dtype, H, qkv_rows, p, grid, st);
    return qk_lo ? attn_tc_launch<__half, true>(qkv, qk_lo, dtype, H, qkv_rows, p, grid, st)
                 : attn_tc_launch<__half, false>(qkv, qk_lo, dtype, H, qkv_rows, p, grid, st);
}

}  // namespace energon
