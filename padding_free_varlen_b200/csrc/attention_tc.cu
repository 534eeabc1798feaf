// Causal self-attention on packed tokens with the 5th-generation tensor cores.
//
// The attention of the GPT-3 layer run on the valid tokens only (EnergonAI
// README, "Scaling Ability": redundant computation elimination), driven by
// cu_seqlens: sequence b owns packed rows cu[b] .. cu[b+1]-1 of the fused
// projection qkv [rows, 3H] (columns Q | K | V, head-major inside each).  For
// head j and position s:  o_j(s) = sum_{t <= s} softmax_t(q_j(s) . k_j(t) / sqrt(d)) v_j(t).
//
// Work item = 128 queries of one (sequence, head), head_dim 128; persistent CTAs of
// 128 threads walk the items, thread i owning query row i (TMEM lane i).  Per 128-key block:
//   TMA   Q (once per item, prefetched during the item before), K and V tiles straight
//         from the packed qkv rows (128-byte swizzle), plus the low halves of Q and K
//   MMA   S = Q K^T  (tcgen05.mma kind::f16, M = N = K = 128) into TMEM columns 0..127,
//         from the two-term Q and K: Qh Kh^T + Qh Kl^T + Ql Kh^T
//   ALU   each thread reads its S row from TMEM, applies the causal mask, keeps
//         a running max / sum (online softmax, fp32, exp2 with the scale folded
//         in) and writes P, rounded to the storage type, into shared memory
//   MMA   O += P V  (V used as an MN-major operand, no transpose) into TMEM 128..255
// Keys past the sequence are masked; their V rows are zeroed in shared memory
// first, so stale workspace contents can never reach a valid row (0 * NaN).
// Causality bounds the key blocks of query tile qb to 0..qb, so a query visits
// the same blocks whether its sequence is packed or padded.
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace energon {

namespace {
constexpr int ATQ = 128;                // queries per CTA
constexpr int ATK = 128;                // keys per block
constexpr int AHD = 128;                // head dim
constexpr int ATILE = 128 * 64 * 2;     // 128 rows x 64 columns of 16-bit = 16 KiB, one swizzle block column
// Q, K, V (and with the low halves of Q and K, two more) tiles of 128 x 128.
// Two Q slots of 2 tiles (4 with the low halves), K and V of 2 tiles each, the K low half.
template <bool LO>
constexpr int at_smem() { return (LO ? 14 : 8) * ATILE + 1024 + 128; }
constexpr uint32_t AT_TMEM_COLS = 256;  // S: 0..127, O: 128..255
}  // namespace

struct AttnTcParams {
    const int32_t* cu;
    void* out;
    int32_t* status;
    int H;
    int n_heads, n_qt, total;  // work items: n_qt query tiles x n_heads x batch
    float scale_log2e;         // log2(e) / sqrt(head_dim)
    uint64_t timeout_ns;
};

// Thread 0 waits (bounded); every thread learns the outcome at the same barrier.
__device__ __forceinline__ bool block_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
    int ok = 1;
    if (threadIdx.x == 0) ok = mbar_wait_bounded(bar, parity, nullptr, timeout_ns) ? 1 : 0;
    return __syncthreads_and(ok) != 0;
}

// Work item i = (query tile, head, sequence), query tiles fastest.  Empty items (a query
// tile past its sequence's length) are skipped by every thread alike.
struct AttnItem {
    int b, j, q0, start, len, n_kb;
};

__device__ __forceinline__ bool attn_item(const AttnTcParams& p, int i, AttnItem& it) {
    const int qt = i % p.n_qt;
    const int rest = i / p.n_qt;
    it.j = rest % p.n_heads;
    it.b = rest / p.n_heads;
    it.q0 = qt * ATQ;
    it.start = __ldg(p.cu + it.b);
    it.len = __ldg(p.cu + it.b + 1) - it.start;
    it.n_kb = it.q0 / ATK + 1;  // causal: key blocks 0 .. the diagonal one
    return it.q0 < it.len;
}

// The first non-empty item at or after i on this CTA's stride (i >= total: none).
__device__ __forceinline__ int attn_next(const AttnTcParams& p, int i, AttnItem& it) {
    for (; i < p.total; i += gridDim.x)
        if (attn_item(p, i, it)) return i;
    return p.total;
}

// Persistent CTAs (one per SM), 128 threads; thread i owns query row i of the current
// item (TMEM lane i); thread 0 also issues every copy and MMA.  Shared memory holds two
// Q slots (the next item's Q arrives while the current item runs), the current key
// block's K (its rows are reused for P once S is computed) and V, and with LO the low
// halves of Q and K.  Copies are issued as soon as their buffer is free: the next key
// block's K low half right after S, its K and V right after P V, the Q two items ahead
// right after the current item's last S.
//
// LO: the low halves of Q and K (tensor map tml over qk_lo [rows, 2H]) enter the scores,
// S = Qh Kh^T + Qh Kl^T + Ql Kh^T (the Ql Kl^T term is below fp32 resolution).
template <typename T, bool LO>
__global__ void __launch_bounds__(128) attn_tc_kernel(const __grid_constant__ CUtensorMap tm,
                                                      const __grid_constant__ CUtensorMap tml, const AttnTcParams p) {
    constexpr int QT = LO ? 4 : 2;  // tiles per Q slot
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQs = base;                         // [2][Qh 0..63 | 64..127 (| Ql 0..63 | 64..127)]
    uint8_t* sK = base + 2 * QT * ATILE;         // K: head dims 0..63 | 64..127; then P: keys 0..63 | 64..127
    uint8_t* sV = sK + 2 * ATILE;                // V: head dims 0..63 | 64..127, one row per key
    uint8_t* sKl = sV + 2 * ATILE;               // low half of K (LO)
    uint64_t* bars = reinterpret_cast<uint64_t*>(sKl + (LO ? 2 : 0) * ATILE);
    uint64_t* bar_q = bars;        // [2]
    uint64_t* bar_kl = bars + 2;
    uint64_t* bar_kv = bars + 3;
    uint64_t* bar_mma = bars + 4;
    uint64_t* drain = bars + 5;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 6);

    const int tid = threadIdx.x, warp = tid >> 5;
    if (status_bad(p.status)) return;
    AttnItem cur;
    int icur = attn_next(p, blockIdx.x, cur);
    if (icur >= p.total) return;

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
    const uint32_t S_t = tmem + lane_base, O_t = tmem + lane_base + 128;
    constexpr uint32_t fmt = std::is_same<T, __half>::value ? 0u : 1u;
    constexpr uint32_t idesc_s = idesc_f16(fmt, ATQ, ATK, 0);
    constexpr uint32_t idesc_o = idesc_f16(fmt, ATQ, AHD, 1);

    // copies (thread 0); pend: bit 0/1 Q slots, bit 2 K low half, bit 3 K + V in flight
    uint32_t pend = 0, qpar = 0, klpar = 0, kvpar = 0, mma_phase = 0;
    auto issue_q = [&](int slot, const AttnItem& it) {
        uint8_t* q = sQs + slot * QT * ATILE;
        const int y = it.start + it.q0;
        mbar_arrive_expect_tx(&bar_q[slot], QT * ATILE);
        tma_load_2d(q, &tm, &bar_q[slot], it.j * AHD, y);
        tma_load_2d(q + ATILE, &tm, &bar_q[slot], it.j * AHD + 64, y);
        if (LO) {
            tma_load_2d(q + 2 * ATILE, &tml, &bar_q[slot], it.j * AHD, y);
            tma_load_2d(q + 3 * ATILE, &tml, &bar_q[slot], it.j * AHD + 64, y);
        }
        pend |= 1u << slot;
    };
    auto issue_kl = [&](const AttnItem& it, int kb) {
        if (!LO) return;
        const int y = it.start + kb * ATK;
        mbar_arrive_expect_tx(bar_kl, 2 * ATILE);
        tma_load_2d(sKl, &tml, bar_kl, p.H + it.j * AHD, y);
        tma_load_2d(sKl + ATILE, &tml, bar_kl, p.H + it.j * AHD + 64, y);
        pend |= 4u;
    };
    auto issue_kv = [&](const AttnItem& it, int kb) {
        const int y = it.start + kb * ATK;
        mbar_arrive_expect_tx(bar_kv, 4 * ATILE);
        tma_load_2d(sK, &tm, bar_kv, p.H + it.j * AHD, y);
        tma_load_2d(sK + ATILE, &tm, bar_kv, p.H + it.j * AHD + 64, y);
        tma_load_2d(sV, &tm, bar_kv, 2 * p.H + it.j * AHD, y);
        tma_load_2d(sV + ATILE, &tm, bar_kv, 2 * p.H + it.j * AHD + 64, y);
        pend |= 8u;
    };

    AttnItem nxt, nn;
    int inxt = attn_next(p, icur + gridDim.x, nxt);
    if (tid == 0) {
        tma_prefetch_desc(&tm);
        if (LO) tma_prefetch_desc(&tml);
        issue_q(0, cur);
        issue_kl(cur, 0);
        issue_kv(cur, 0);
        if (inxt < p.total) issue_q(1, nxt);
    }
    uint32_t r[32];
    bool ok = true;
    for (int local = 0; ok && icur < p.total; ++local) {
        const int slot = local & 1;
        const uint8_t* sQ = sQs + slot * QT * ATILE;
        const uint8_t* sQl = sQ + 2 * ATILE;
        ok = block_wait(&bar_q[slot], (qpar >> slot) & 1u, p.timeout_ns);
        if (!ok) break;
        qpar ^= 1u << slot;
        if (tid == 0) pend &= ~(1u << slot);
        const int q = cur.q0 + tid;
        const bool row_ok = q < cur.len;
        int inn = p.total;
        float m_i = -INFINITY, l_i = 0.0f;
        for (int kb = 0; kb < cur.n_kb; ++kb) {
            if (LO) {
                ok = block_wait(bar_kl, klpar, p.timeout_ns);
                if (!ok) break;
                klpar ^= 1u;
                if (tid == 0) pend &= ~4u;
            }
            ok = block_wait(bar_kv, kvpar, p.timeout_ns);
            if (!ok) break;
            kvpar ^= 1u;
            if (tid == 0) pend &= ~12u;
            const int kbase = kb * ATK;
            if (kbase + tid >= cur.len) {  // key row past the sequence: zero its V row
                const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    reinterpret_cast<uint4*>(sV + tid * 128)[c] = z;
                    reinterpret_cast<uint4*>(sV + ATILE + tid * 128)[c] = z;
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < AHD / 16; ++k) {
                    const uint64_t a = smem_desc_k128(smem_u32(sQ + (k >> 2) * ATILE)) + 2 * (k & 3);
                    const uint64_t bk = smem_desc_k128(smem_u32(sK + (k >> 2) * ATILE)) + 2 * (k & 3);
                    umma_f16(tmem, a, bk, idesc_s, k > 0 ? 1u : 0u);
                    if (LO) {
                        const uint64_t al = smem_desc_k128(smem_u32(sQl + (k >> 2) * ATILE)) + 2 * (k & 3);
                        const uint64_t bl = smem_desc_k128(smem_u32(sKl + (k >> 2) * ATILE)) + 2 * (k & 3);
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
            // S is in TMEM: the K low half is free, and after the item's last block its Q slot
            const bool last = kb + 1 == cur.n_kb;
            if (last) inn = attn_next(p, inxt + gridDim.x, nn);
            if (tid == 0) {
                if (!last) issue_kl(cur, kb + 1);
                else if (inxt < p.total) issue_kl(nxt, 0);
                if (last && inn < p.total) issue_q(slot, nn);
            }

            // ---- online softmax of this thread's row
            const int nvalid = row_ok ? min(ATK, q - kbase + 1) : 0;  // keys kbase .. kbase+nvalid-1 are visible
            float mx = -INFINITY;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                tmem_ld_x32(S_t + c * 32, r);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    if (c * 32 + e < nvalid) mx = fmaxf(mx, __uint_as_float(r[e]));
            }
            const float m_new = row_ok ? fmaxf(m_i, mx) : 0.0f;
            const float alpha = row_ok ? exp2f((m_i - m_new) * p.scale_log2e) : 1.0f;
            float rs = 0.0f;
            uint8_t* sP = sK;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
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
                    *reinterpret_cast<uint4*>(sP + (c >> 1) * ATILE + tid * 128 + ((ch ^ (tid & 7)) << 4)) = w;
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
                for (int k = 0; k < ATK / 16; ++k) {
                    const uint64_t a = smem_desc_k128(smem_u32(sP + (k >> 2) * ATILE)) + 2 * (k & 3);
                    const uint64_t bv = smem_desc_mn128(smem_u32(sV + k * 2048), ATILE, 1024);
                    umma_f16(tmem + 128, a, bv, idesc_o, (kb > 0 || k > 0) ? 1u : 0u);
                }
                umma_commit(bar_mma);
            }
            ok = block_wait(bar_mma, mma_phase, p.timeout_ns);
            mma_phase ^= 1u;
            if (!ok) break;
            tc_fence_after();
            // P V done: K (now P) and V are free for the next block, of this item or the next
            if (tid == 0) {
                if (!last) issue_kv(cur, kb + 1);
                else if (inxt < p.total) issue_kv(nxt, 0);
            }
        }
        if (!ok) break;
        // ---- output: O / l, one rounding, this thread's row
        const float inv = row_ok ? 1.0f / l_i : 0.0f;
        T* orow = static_cast<T*>(p.out) + (int64_t)(cur.start + q) * p.H + cur.j * AHD;
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
        // every thread has read O before the next item's first P V overwrites it
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        icur = inxt, cur = nxt;
        inxt = inn, nxt = nn;
    }
    if (!ok && tid == 0) {
        // A bounded wait ran out: record it, let every MMA and copy in flight finish, leave.
        status_or(p.status, ENERGON_DEVICE_TIMEOUT);
        umma_commit(drain);
        mbar_wait_bounded(drain, 0, nullptr, p.timeout_ns);
        for (int s = 0; s < 2; ++s)
            if (pend & (1u << s)) mbar_wait_bounded(&bar_q[s], (qpar >> s) & 1u, nullptr, p.timeout_ns);
        if (pend & 4u) mbar_wait_bounded(bar_kl, klpar, nullptr, p.timeout_ns);
        if (pend & 8u) mbar_wait_bounded(bar_kv, kvpar, nullptr, p.timeout_ns);
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

// [rows, cols] 16-bit tensor, box 64 x 128, 128-byte swizzle (the Q / K / V tiles).
static CUresult attn_tmap(CUtensorMap* m, int dtype, const void* ptr, int64_t cols, int64_t rows) {
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt =
        dtype == ENERGON_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    return attn_encode_fn()(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

template <typename T, bool LO>
static cudaError_t attn_tc_launch(const CUtensorMap& tm, const CUtensorMap& tml, const AttnTcParams& p,
                                  cudaStream_t st) {
    const void* k = (const void*)attn_tc_kernel<T, LO>;
    cudaError_t e = prepare_smem(k, at_smem<LO>());
    if (e != cudaSuccess) return e;
    // persistent: as many CTAs as fit on the device at once, at most one per work item
    const int resident = device_cached(k, 1, [&] {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attn_tc_kernel<T, LO>, 128, at_smem<LO>()) !=
                cudaSuccess ||
            per_sm < 1) {
            (void)cudaGetLastError();
            per_sm = 1;
        }
        return per_sm * device_sm_count();
    });
    const int grid = p.total < resident ? p.total : resident;
    attn_tc_kernel<T, LO><<<grid, 128, at_smem<LO>(), st>>>(tm, tml, p);
    return cudaGetLastError();
}

cudaError_t launch_attention_tc(int dtype, const void* qkv, const void* qk_lo, void* o, const int32_t* cu, int batch,
                                int max_len, int H, int n_heads, int qkv_rows, int32_t* status, uint64_t timeout_ns,
                                cudaStream_t st) {
    if (batch <= 0 || max_len <= 0) return cudaSuccess;
    CUtensorMap tm, tml;
    if (attn_tmap(&tm, dtype, qkv, 3 * (int64_t)H, qkv_rows) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    if (qk_lo != nullptr) {
        if (attn_tmap(&tml, dtype, qk_lo, 2 * (int64_t)H, qkv_rows) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    } else {
        tml = tm;
    }
    AttnTcParams p;
    p.cu = cu;
    p.out = o;
    p.status = status;
    p.H = H;
    p.scale_log2e = (float)(1.4426950408889634 / sqrt((double)AHD));
    p.timeout_ns = timeout_ns;
    p.n_heads = n_heads;
    p.n_qt = (max_len + ATQ - 1) / ATQ;
    const int64_t total = (int64_t)p.n_qt * n_heads * batch;
    if (total > 0x7fffffff) return cudaErrorInvalidValue;
    p.total = (int)total;
    if (dtype == ENERGON_BF16)
        return qk_lo ? attn_tc_launch<__nv_bfloat16, true>(tm, tml, p, st)
                     : attn_tc_launch<__nv_bfloat16, false>(tm, tml, p, st);
    return qk_lo ? attn_tc_launch<__half, true>(tm, tml, p, st) : attn_tc_launch<__half, false>(tm, tml, p, st);
}

}  // namespace energon
