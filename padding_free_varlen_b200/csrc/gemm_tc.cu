// Tensor-core GEMM for sm_100a: y = A W^T + bias (+ GELU) (+ residual).
//
// The QKV, output-projection and FFN contractions of the GPT-3 layer, run on
// the packed tokens only (QbitAI article "最新大模型推理系统Energon-AI开源",
// section "Runtime": GEMM time dominates as models grow; section "易用性": the
// bias + GELU and bias + residual steps that follow the MLP GEMMs, fused here
// into the epilogue instead of separate passes over HBM).
//
// Two persistent kernels.  gemm_tc2_kernel, for buffers of more than 128 rows,
// runs on CTA pairs (cta_group::2) with 512 x 256 pair tiles; it is described
// before its definition below.  gemm_tc_kernel, for buffers of at most 128 rows
// (the weight-streaming case, with split K), is the single-CTA form:
//   - 128 x 256 output tiles, K consumed 64 elements (128 bytes) at a time.
//   - warp 0: TMA producer.  A [rows, K] and W [N, K] tiles land in a 4-stage
//     shared-memory ring (128-byte swizzle), completion counted on mbarriers.
//   - warp 1: MMA issuer.  One thread issues tcgen05.mma (kind::f16, fp32
//     accumulate) into TMEM; tcgen05.commit frees each ring slot and, at the
//     end of a tile, hands the accumulator to the epilogue.
//   - warp 2: allocates / frees 512 TMEM columns = two 128 x 256 fp32
//     accumulators, so the epilogue of tile i overlaps the MMAs of tile i+1.
//   - warps 4-7: epilogue.  tcgen05.ld (each warp owns 32 TMEM lanes = 32 rows),
//     bias / GELU / residual in fp32, one rounding to the 16-bit type, stores.
//   - The number of valid rows M is read on the device (cu_seqlens[batch]);
//     tiles past M are never scheduled, rows past M are never stored.
//   - Tiles are rasterised in groups of `group_m` row tiles so that the A
//     panels of a group stay in L2 while the weight panels stream past once.
//   - Every mbarrier wait is bounded: on expiry the kernel records
//     ENERGON_DEVICE_TIMEOUT, lets the other roles stop, waits (bounded) for
//     its copies and MMAs in flight, frees TMEM and returns.
#include <cudaTypedefs.h>

#include <stdio.h>

#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace energon {

namespace {
constexpr int TBM = 128, TBN = 256, TBK = 64, TSTAGES = 4;
constexpr int A_STAGE = TBM * TBK * 2;  // 16 KiB
constexpr int B_STAGE = TBN * TBK * 2;  // 32 KiB
constexpr uint32_t TMEM_COLS = 2 * TBN;
constexpr int TC_SMEM = TSTAGES * (A_STAGE + B_STAGE) + 1024 + 256;

// CTA-pair (cta_group::2) kernel: 256 x 256 tiles, each CTA stages 128 rows of A
// and 128 rows of W (its half of the tile's N) per 64-wide K step.
constexpr int PBM = 256, PBN = 256, PBK = 64;
constexpr int PA_STAGE = 128 * PBK * 2;  // 16 KiB
constexpr int PB_STAGE = 128 * PBK * 2;  // 16 KiB
}  // namespace

struct TcParams {
    const void* bias;
    const void* residual;
    void* out;
    const int32_t* d_rows;
    int32_t* status;
    int M_cap, N, K, group_m, gelu_tanh;
    int raster;     // tile order, see tile_coords
    int k_splits;   // single-CTA kernel: K ranges per output tile (1: no split)
    float* partials;  // k_splits > 1: fp32 [k_splits][M_cap][N] partial sums
    uint64_t timeout_ns;
    // transpose_padding_rebuild fused into the epilogue (pair kernel only): output row r
    // goes to padded row b * scatter_pad_len + r - scatter_cu[b] of a [batch, pad_len, N] tensor
    const int32_t* scatter_cu;
    int scatter_batch, scatter_pad_len;
    // EPI_LN_FOLD: per-row (rstd, mean * rstd), per-column c and d, low halves [M_cap, lo_cols]
    const float2* fold_stats;
    const float* fold_c;
    const float* fold_d;
    void* lo;
    int lo_cols;
    // the fp32 residual rows the main drain reads row per lane (EPI_RES32) start on 32-byte
    // boundaries: it uses 32-byte loads
    int wide32;
};

// Destination row of packed row `row` (its padded position when the epilogue scatters).
__device__ __forceinline__ int64_t out_row_of(const TcParams& p, int row) {
    if (p.scatter_cu == nullptr) return row;
    const int b = owner_of(p.scatter_cu, p.scatter_batch, row);
    return (int64_t)b * p.scatter_pad_len + (row - __ldg(p.scatter_cu + b));
}

__device__ __forceinline__ void tile_mn(int t, int num_m, int num_n, int group_m, int& m, int& n) {
    const int per_group = group_m * num_n;
    const int g = t / per_group;
    const int r = t - g * per_group;
    const int first_m = g * group_m;
    const int gm = min(group_m, num_m - first_m);
    n = r / gm;
    m = first_m + (r - n * gm);
}

// Tile t -> (m, n).  raster 0: groups of `group` row tiles, columns outermost
// inside a group (n varies slowest); raster 1: groups of `group` column tiles,
// rows fastest (every row tile of a column before the next column).
__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int group, int raster, int& m, int& n) {
    if (raster == 0) {
        tile_mn(t, num_m, num_n, group, m, n);
        return;
    }
    const int per_group = group * num_m;
    const int g = t / per_group;
    const int r = t - g * per_group;
    const int first_n = g * group;
    const int gn = min(group, num_n - first_n);
    m = r / gn;
    n = first_n + (r - m * gn);
}

// Lane 0 waits, the warp learns the outcome.  SPIN: poll without suspending (the
// producer and MMA roles, whose wake-up latency stalls the ring); otherwise the
// suspending wait (the epilogue, which must not steal issue slots from them).
template <bool SPIN = false>
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const volatile int* abort_flag,
                                          uint64_t timeout_ns) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0)
        ok = SPIN ? mbar_spin_bounded(bar, parity, abort_flag, timeout_ns)
                  : mbar_wait_bounded(bar, parity, abort_flag, timeout_ns);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// ------------------------------------------------------------------ epilogue
//
// Per 32-column chunk of one output row (the accumulator columns a thread holds):
//   EPI_LN_FOLD    v = rstd acc - (mean rstd) c + d; columns below lo_cols also store
//                  the low half round(v - round(v)) to `lo`
//   EPI_BIAS_GELU  v = GELU(acc + bias)
//   EPI_RES_OUT32  v = acc + bias + residual (storage type), stored as fp32
//   EPI_RES32      v = acc + bias + residual (fp32), stored in the storage type
// One rounding to the output type at the end.

template <int EPI>
struct Epi {
    static constexpr bool FOLD = EPI == EPI_LN_FOLD;
    static constexpr bool GELU = EPI == EPI_BIAS_GELU;
    static constexpr bool RES_T = EPI == EPI_RES_OUT32;   // residual in the storage type
    static constexpr bool RES_F32 = EPI == EPI_RES32;     // residual in fp32
    static constexpr bool OUT_F32 = EPI == EPI_RES_OUT32;
    static constexpr int RES_VECS = RES_F32 ? 8 : (RES_T ? 4 : 0);  // 16-byte vectors per 32 columns
};

// 32-byte global loads: a lane that owns a row reads whole 32-byte sectors, so a warp
// instruction touches 32 sectors instead of 32 half sectors (half the requests of 16-byte
// loads for the row-per-lane fp32 residual).
__device__ __forceinline__ void ld_global32B(const void* a, uint4& lo, uint4& hi) {
    unsigned long long a0, a1, a2, a3;  // as four 64-bit words
    asm volatile("ld.global.v4.b64 {%0, %1, %2, %3}, [%4];" : "=l"(a0), "=l"(a1), "=l"(a2), "=l"(a3) : "l"(a));
    lo = make_uint4((unsigned)a0, (unsigned)(a0 >> 32), (unsigned)a1, (unsigned)(a1 >> 32));
    hi = make_uint4((unsigned)a2, (unsigned)(a2 >> 32), (unsigned)a3, (unsigned)(a3 >> 32));
}

// Residual of one row's 32 columns [col0, col0 + 32), read straight from global memory.
// WIDE: in 32-byte accesses (the main drain, when the residual rows are 32-byte aligned).
template <typename T, int EPI, bool WIDE = false>
__device__ __forceinline__ void load_residual32(const TcParams& p, int row, int col0, bool live, uint4* res) {
    constexpr int NV = Epi<EPI>::RES_VECS;
    if (NV > 0 && live) {
        const size_t eb = Epi<EPI>::RES_F32 ? 4 : sizeof(T);
        const uint4* rp = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.residual) +
                                                         ((size_t)row * p.N + col0) * eb);
        if constexpr (WIDE && NV % 2 == 0) {
#pragma unroll
            for (int q = 0; q < NV; q += 2) ld_global32B(rp + q, res[q], res[q + 1]);
        } else {
#pragma unroll
            for (int q = 0; q < NV; ++q) res[q] = rp[q];
        }
    }
}

// Accumulator chunk -> final fp32 values (before the one rounding).
template <typename T, int EPI>
__device__ __forceinline__ void epi_math(float* v, const uint32_t* acc, const TcParams& p, int col0, float2 fs,
                                         const uint4* res) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(acc[j]);
    if (Epi<EPI>::FOLD) {
        const float4* cp = reinterpret_cast<const float4*>(p.fold_c + col0);
        const float4* dp = reinterpret_cast<const float4*>(p.fold_d + col0);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 c = __ldg(cp + q), d = __ldg(dp + q);
            v[4 * q + 0] = fmaf(v[4 * q + 0], fs.x, fmaf(-fs.y, c.x, d.x));
            v[4 * q + 1] = fmaf(v[4 * q + 1], fs.x, fmaf(-fs.y, c.y, d.y));
            v[4 * q + 2] = fmaf(v[4 * q + 2], fs.x, fmaf(-fs.y, c.z, d.z));
            v[4 * q + 3] = fmaf(v[4 * q + 3], fs.x, fmaf(-fs.y, c.w, d.w));
        }
    } else if (p.bias != nullptr) {
        const uint4* bp = reinterpret_cast<const uint4*>(static_cast<const T*>(p.bias) + col0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 w = __ldg(bp + q);
            const uint32_t* ww = reinterpret_cast<const uint32_t*>(&w);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float2 f = unpack2<T>(ww[h]);
                v[q * 8 + 2 * h] += f.x;
                v[q * 8 + 2 * h + 1] += f.y;
            }
        }
    }
    if (Epi<EPI>::GELU) {
        if (p.gelu_tanh) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = gelu_tanh_fast(v[j]);
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = gelu_f(v[j], false);
        }
    }
    if (Epi<EPI>::RES_T) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t* ww = reinterpret_cast<const uint32_t*>(&res[q]);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float2 f = unpack2<T>(ww[h]);
                v[q * 8 + 2 * h] += f.x;
                v[q * 8 + 2 * h + 1] += f.y;
            }
        }
    }
    if (Epi<EPI>::RES_F32) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            v[4 * q + 0] += __uint_as_float(res[q].x);
            v[4 * q + 1] += __uint_as_float(res[q].y);
            v[4 * q + 2] += __uint_as_float(res[q].z);
            v[4 * q + 3] += __uint_as_float(res[q].w);
        }
    }
}

// 32 values -> 4 words of two storage-type elements each (hi), and the low halves.
template <typename T>
__device__ __forceinline__ uint4 pack8(const float* v) {
    uint4 o;
    o.x = pack2<T>(v[0], v[1]);
    o.y = pack2<T>(v[2], v[3]);
    o.z = pack2<T>(v[4], v[5]);
    o.w = pack2<T>(v[6], v[7]);
    return o;
}
// The low half of a two-term value: round(v - round(v)); v - round(v) is exact in fp32.
template <typename T>
__device__ __forceinline__ uint32_t pack2_lo(float a, float b, uint32_t hi) {
    const float2 h = unpack2<T>(hi);
    return pack2<T>(a - h.x, b - h.y);
}
template <typename T>
__device__ __forceinline__ uint4 pack8_lo(const float* v, uint4 hi) {
    uint4 o;
    o.x = pack2_lo<T>(v[0], v[1], hi.x);
    o.y = pack2_lo<T>(v[2], v[3], hi.y);
    o.z = pack2_lo<T>(v[4], v[5], hi.z);
    o.w = pack2_lo<T>(v[6], v[7], hi.w);
    return o;
}

// Row-per-thread store of one chunk (the path for rows past a full 32-row box).
template <typename T, int EPI>
__device__ __forceinline__ void epilogue_store32(uint32_t* acc, const uint4* res, const TcParams& p, int row,
                                                 int64_t out_row, int col0, float2 fs) {
    float* v = reinterpret_cast<float*>(acc);  // the values replace the accumulator bits
    epi_math<T, EPI>(v, acc, p, col0, fs, res);
    if (Epi<EPI>::OUT_F32) {
        float4* op = reinterpret_cast<float4*>(static_cast<float*>(p.out) + out_row * p.N + col0);
#pragma unroll
        for (int q = 0; q < 8; ++q) op[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        return;
    }
    uint4* op = reinterpret_cast<uint4*>(static_cast<T*>(p.out) + out_row * p.N + col0);
    const bool lo = Epi<EPI>::FOLD && p.lo != nullptr && col0 < p.lo_cols;
    uint4* lp = lo ? reinterpret_cast<uint4*>(static_cast<T*>(p.lo) + (int64_t)row * p.lo_cols + col0) : nullptr;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 h = pack8<T>(v + 8 * q);
        op[q] = h;
        if (lo) lp[q] = pack8_lo<T>(v + 8 * q, h);
    }
}

// One warp drains CH x 32 accumulator columns of its 32 TMEM lanes (= 32 output rows),
// 32 columns at a time, row per thread; the TMEM load of the next chunk is issued before
// the current chunk is processed.
template <typename T, int EPI, int CH = 8>
__device__ __forceinline__ void drain_256(uint32_t tbase, const TcParams& p, int row, int col_base, int M) {
    // The path for the one box per tile that holds row M - 1 (and boxes that straddle two
    // sequences when scattering): the residual is loaded chunk by chunk, not ahead.
    constexpr int NV = Epi<EPI>::RES_VECS > 0 ? Epi<EPI>::RES_VECS : 1;
    uint32_t r[2][32];
    uint4 res[NV];
    const bool row_ok = row < M;
    const int64_t out_row = row_ok ? out_row_of(p, row) : 0;
    const float2 fs = (Epi<EPI>::FOLD && row_ok) ? p.fold_stats[row] : make_float2(0.0f, 0.0f);
    tmem_ld_x16(tbase, r[0]);
    tmem_ld_x16(tbase + 16, r[0] + 16);
#pragma unroll
    for (int c = 0; c < CH; ++c) {
        const int cur = c & 1;
        const int col0 = col_base + c * 32;
        const bool live = row_ok && col0 < p.N;
        load_residual32<T, EPI>(p, row, col0, live, res);
        tmem_wait_ld_regs(r[cur]);
        if (c + 1 < CH) {
            tmem_ld_x16(tbase + (c + 1) * 32, r[cur ^ 1]);
            tmem_ld_x16(tbase + (c + 1) * 32 + 16, r[cur ^ 1] + 16);
        }
        if (live) epilogue_store32<T, EPI>(r[cur], res, p, row, out_row, col0, fs);
    }
}

// Staging buffer of one epilogue warp: 32 rows x 64 bytes (32 columns of 16-bit values,
// or 16 of fp32), in the TMA 64-byte swizzle (the 16-byte chunk index is XORed with bits
// 1-2 of the row), so that 32 threads each touching their own row hit every bank once
// per 128 bytes.
__device__ __forceinline__ uint32_t stage_off(int row, int chunk) {
    return (uint32_t)(row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4));
}

// One warp drains 256 accumulator columns of its 32 rows through shared memory: per
// 32-column chunk, TMEM -> registers -> epilogue math -> one rounding -> a staging
// buffer -> one TMA store of the 32 x 32 box (and, for the low halves, a second box
// from the other buffer).  Residuals in the storage type are fetched by TMA into the
// other buffer one chunk ahead; fp32 residuals are loaded into registers one chunk
// ahead; fp32 outputs go out through the buffer the chunk's residual has just left, 16
// columns (one 32 x 16 fp32 box, 64-byte rows) per TMA store.  The accumulator is handed back (arrival on
// `tempty_cluster`) as soon as its last columns are in registers.  Every row of the
// warp must be valid (rows < M); the warp holding the last valid row takes drain_256
// instead.  Returns false if a residual copy timed out.
template <typename T, int EPI, int CH = 8>
__device__ __forceinline__ bool drain_256_staged(uint32_t tbase, const TcParams& p, const CUtensorMap* tmO,
                                                 const CUtensorMap* tmR, const CUtensorMap* tmL, uint8_t* sbuf,
                                                 uint64_t* rbar, uint32_t& rpar, int row_base, int out_row_base,
                                                 int col_base, uint32_t tempty_cluster,
                                                 const volatile int* abort_flag) {
    using E = Epi<EPI>;
    constexpr bool TMA_RES = E::RES_T;                 // residual boxes through shared memory
    constexpr int NV = E::RES_F32 ? 8 : 1;
    // With fp32 residuals in registers (two chunks' worth), the accumulator chunk is not
    // double-buffered: each chunk's TMEM load is issued and awaited in its own iteration.
    constexpr int RB = E::RES_F32 ? 1 : 2;
    const int lane = threadIdx.x & 31;
    const int row = row_base + lane;
    const bool lo = E::FOLD && p.lo != nullptr && col_base < p.lo_cols;   // uniform over the tile
    uint32_t r[RB][32];
    uint4 res[2][NV];
    bool ok = true;
    uint32_t pend = 0;  // buffers with a residual copy in flight
    const float2 fs = E::FOLD ? p.fold_stats[row] : make_float2(0.0f, 0.0f);
    if (lane == 0) {
        bulk_wait_read<0>();  // the previous tile's stores no longer read either buffer
        if (TMA_RES) {
            mbar_arrive_expect_tx(&rbar[0], 32 * 64);
            tma_load_2d(sbuf, tmR, &rbar[0], col_base, row_base);
        }
    }
    if (TMA_RES) pend = 1u;
    __syncwarp();
    if (E::RES_F32) {
        if (p.wide32) load_residual32<T, EPI, true>(p, row, col_base, true, res[0]);
        else load_residual32<T, EPI>(p, row, col_base, true, res[0]);
    }
    if (RB == 2) {
        tmem_ld_x16(tbase, r[0]);
        tmem_ld_x16(tbase + 16, r[0] + 16);
    }
#pragma unroll
    for (int c = 0; c < CH; ++c) {
        const int cur = c & 1;
        const int rc = RB == 2 ? cur : 0;
        uint8_t* buf = sbuf + cur * 2048;
        if (RB == 1) {
            tmem_ld_x16(tbase + c * 32, r[0]);
            tmem_ld_x16(tbase + c * 32 + 16, r[0] + 16);
            if (c + 1 < CH) {
                if (p.wide32) load_residual32<T, EPI, true>(p, row, col_base + (c + 1) * 32, true, res[cur ^ 1]);
                else load_residual32<T, EPI>(p, row, col_base + (c + 1) * 32, true, res[cur ^ 1]);
            }
        }
        tmem_wait_ld_regs(r[rc]);
        if (c + 1 < CH) {
            if (RB == 2) {
                tmem_ld_x16(tbase + (c + 1) * 32, r[rc ^ 1]);
                tmem_ld_x16(tbase + (c + 1) * 32 + 16, r[rc ^ 1] + 16);
            }
        } else {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_cluster);
        }
        const int col0 = col_base + c * 32;
        if (TMA_RES && c + 1 < CH) {
            if (lane == 0) {
                if (E::OUT_F32) bulk_wait_read<0>();  // the previous chunk's output stores used that buffer
                mbar_arrive_expect_tx(&rbar[cur ^ 1], 32 * 64);
                tma_load_2d(sbuf + (cur ^ 1) * 2048, tmR, &rbar[cur ^ 1], col0 + 32, row_base);
            }
            pend |= 1u << (cur ^ 1);
        }
        uint4 rt[4];
        if (TMA_RES) {
            const bool got = mbar_wait_bounded(&rbar[cur], (rpar >> cur) & 1u, abort_flag, p.timeout_ns);
            if (!__all_sync(0xffffffffu, got)) {
                // copies still in flight get one more bounded wait before the warp gives up
                if (lane == 0)
                    for (int b = 0; b < 2; ++b)
                        if (pend & (1u << b)) mbar_wait_bounded(&rbar[b], (rpar >> b) & 1u, nullptr, p.timeout_ns);
                ok = false;
                break;
            }
            rpar ^= 1u << cur;
            pend &= ~(1u << cur);
#pragma unroll
            for (int q = 0; q < 4; ++q) rt[q] = *reinterpret_cast<const uint4*>(buf + stage_off(lane, q));
            // every lane has read this buffer before lane 0 refills it (two chunks on)
            fence_proxy_async_smem();
            __syncwarp();
        }
        float* v = reinterpret_cast<float*>(r[rc]);  // the chunk's values replace its accumulator bits
        epi_math<T, EPI>(v, r[rc], p, col0, fs, TMA_RES ? rt : res[cur]);
        if (E::OUT_F32) {
            // this chunk's residual has been read out of buf: it takes the fp32 output, 16
            // columns (64-byte rows) at a time, each half one TMA store
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                if (hh == 1) {
                    if (lane == 0) bulk_wait_read<0>();
                    __syncwarp();
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<float4*>(buf + stage_off(lane, q)) =
                        make_float4(v[16 * hh + 4 * q], v[16 * hh + 4 * q + 1], v[16 * hh + 4 * q + 2],
                                    v[16 * hh + 4 * q + 3]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(tmO, buf, col0 + 16 * hh, out_row_base);
                    bulk_commit();
                }
            }
            continue;
        }
        if (lo) {
            // both buffers take this chunk (high and low halves): the previous chunk's two
            // stores must have read them
            if (lane == 0) bulk_wait_read<0>();
            __syncwarp();
            uint8_t* b0 = sbuf;
            uint8_t* b1 = sbuf + 2048;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 h = pack8<T>(v + 8 * q);
                *reinterpret_cast<uint4*>(b0 + stage_off(lane, q)) = h;
                *reinterpret_cast<uint4*>(b1 + stage_off(lane, q)) = pack8_lo<T>(v + 8 * q, h);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_2d(tmO, b0, col0, out_row_base);
                tma_store_2d(tmL, b1, col0, row_base);
                bulk_commit();
            }
            continue;
        }
        if (c >= 2) {
            if (lane == 0) bulk_wait_read<1>();  // chunk c-2's store has read this buffer
            __syncwarp();
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4*>(buf + stage_off(lane, q)) = pack8<T>(v + 8 * q);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(tmO, buf, col0, out_row_base);
            bulk_commit();
        }
    }
    return ok;
}

// Out-of-line forms of the two drains for the rare cases (the box holding row M - 1,
// boxes that straddle two sequences, and the wave-tail units of half a tile's columns),
// so that their registers do not add to the main path's.
template <typename T, int EPI, int CH>
__device__ __noinline__ void drain_rows_rare(uint32_t tbase, const TcParams& p, int row, int col_base, int M) {
    drain_256<T, EPI, CH>(tbase, p, row, col_base, M);
}
template <typename T, int EPI, int CH>
__device__ __noinline__ bool drain_staged_rare(uint32_t tbase, const TcParams& p, const CUtensorMap* tmO,
                                               const CUtensorMap* tmR, const CUtensorMap* tmL, uint8_t* sbuf,
                                               uint64_t* rbar, uint32_t& rpar, int row_base, int out_row_base,
                                               int col_base, uint32_t tempty_cluster, const volatile int* abort_flag) {
    return drain_256_staged<T, EPI, CH>(tbase, p, tmO, tmR, tmL, sbuf, rbar, rpar, row_base, out_row_base, col_base,
                                        tempty_cluster, abort_flag);
}

// One warp writes its 32 rows x 256 accumulator columns as fp32 partial sums.
__device__ __forceinline__ void drain_256_partial(uint32_t tbase, float* part, int N, int row, int col_base, int M) {
#pragma unroll 1
    for (int c = 0; c < 256; c += 32) {
        uint32_t r[32];
        tmem_ld_x16(tbase + c, r);
        tmem_ld_x16(tbase + c + 16, r + 16);
        tmem_wait_ld_regs(r);
        const int col0 = col_base + c;
        if (row < M && col0 < N) {
            uint4* dst = reinterpret_cast<uint4*>(part + (int64_t)row * N + col0);
#pragma unroll
            for (int q = 0; q < 8; ++q) dst[q] = make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
        }
    }
}

// Split-K finish: out[row][cols] = epilogue(sum over s = 0 .. S-1 of partials[s][row][cols]),
// the splits summed in index order (deterministic), 32 columns per thread, through the
// same epilogue code as the tile kernels.
template <typename T, int EPI>
__global__ void __launch_bounds__(256) splitk_finish_kernel(const float* __restrict__ partials, int S, TcParams p) {
    if (status_bad(p.status)) return;
    const int M = min(*p.d_rows, p.M_cap);
    const int chunks = p.N / 32;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < (int64_t)M * chunks;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int row = (int)(i / chunks), col0 = (int)(i % chunks) * 32;
        uint32_t acc[32];
        const float4* p0 = reinterpret_cast<const float4*>(partials + (int64_t)row * p.N + col0);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 a = p0[q];
            acc[4 * q] = __float_as_uint(a.x), acc[4 * q + 1] = __float_as_uint(a.y);
            acc[4 * q + 2] = __float_as_uint(a.z), acc[4 * q + 3] = __float_as_uint(a.w);
        }
        for (int s = 1; s < S; ++s) {
            const float4* ps = reinterpret_cast<const float4*>(partials + ((int64_t)s * p.M_cap + row) * p.N + col0);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 a = ps[q];
                acc[4 * q] = __float_as_uint(__uint_as_float(acc[4 * q]) + a.x);
                acc[4 * q + 1] = __float_as_uint(__uint_as_float(acc[4 * q + 1]) + a.y);
                acc[4 * q + 2] = __float_as_uint(__uint_as_float(acc[4 * q + 2]) + a.z);
                acc[4 * q + 3] = __float_as_uint(__uint_as_float(acc[4 * q + 3]) + a.w);
            }
        }
        constexpr int NV = Epi<EPI>::RES_VECS > 0 ? Epi<EPI>::RES_VECS : 1;
        uint4 res[NV];
        load_residual32<T, EPI>(p, row, col0, true, res);
        const float2 fs = Epi<EPI>::FOLD ? p.fold_stats[row] : make_float2(0.0f, 0.0f);
        epilogue_store32<T, EPI>(acc, res, p, row, row, col0, fs);
    }
}

template <typename T, int EPI>
__global__ void __launch_bounds__(256, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                                                         const __grid_constant__ CUtensorMap tmB, const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = base;
    uint8_t* sB = base + TSTAGES * A_STAGE;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + TSTAGES * B_STAGE);
    uint64_t* empty = full + TSTAGES;
    uint64_t* tfull = empty + TSTAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (status_bad(p.status)) return;
    const int M = min(*p.d_rows, p.M_cap);
    if (M <= 0) return;
    const int num_m = (M + TBM - 1) / TBM, num_n = (p.N + TBN - 1) / TBN;
    // Work unit t = output tile t / S over the K range t % S (S = k_splits, dividing the
    // K blocks evenly); with S > 1 the epilogue writes fp32 partial sums instead.
    const int S = p.k_splits;
    const int total = num_m * num_n * S;
    if ((int)blockIdx.x >= total) return;
    const int num_kb = (p.K + TBK - 1) / TBK / S;

    if (threadIdx.x == 0) {
        for (int s = 0; s < TSTAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 2) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        int stage = 0;
        uint32_t phase = 0, pend_mask = 0, pend_par = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            int m, n;
            tile_coords(t / S, num_m, num_n, p.group_m, p.raster, m, n);
            const int kb0 = (t % S) * num_kb;
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!warp_wait<true>(&empty[stage], phase ^ 1u, abort_flag, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[stage], A_STAGE + B_STAGE);
                    tma_load_2d(sA + stage * A_STAGE, &tmA, &full[stage], (kb0 + kb) * TBK, m * TBM);
                    tma_load_2d(sB + stage * B_STAGE, &tmB, &full[stage], (kb0 + kb) * TBK, n * TBN);
                }
                pend_mask |= 1u << stage;
                pend_par = (pend_par & ~(1u << stage)) | (phase << stage);
                if (++stage == TSTAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            status_or(p.status, ENERGON_DEVICE_TIMEOUT);
            // Let every copy already issued land before the block releases its shared memory.
            for (int s = 0; s < TSTAGES; ++s)
                if (pend_mask & (1u << s)) mbar_wait_bounded(&full[s], (pend_par >> s) & 1u, nullptr, p.timeout_ns);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        constexpr uint32_t fmt = sizeof(T) == 2 && !std::is_same<T, __half>::value ? 1u : 0u;
        constexpr uint32_t idesc = idesc_f16(fmt, TBM, TBN);
        int stage = 0, local = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++local) {
            const int acc = local & 1;
            if (!warp_wait<true>(&tempty[acc], ((local >> 1) & 1) ^ 1, abort_flag, p.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem + (uint32_t)(acc * TBN);
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!warp_wait<true>(&full[stage], phase, abort_flag, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint64_t a0 = smem_desc_k128(smem_u32(sA + stage * A_STAGE));
                    const uint64_t b0 = smem_desc_k128(smem_u32(sB + stage * B_STAGE));
#pragma unroll
                    for (int k = 0; k < TBK / 16; ++k)  // 16 elements = 32 bytes = 2 descriptor units
                        umma_f16(d_tmem, a0 + 2 * k, b0 + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
                    umma_commit(&empty[stage]);
                }
                __syncwarp();
                if (++stage == TSTAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (lane == 0) umma_commit(&tfull[acc]);
            __syncwarp();
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            status_or(p.status, ENERGON_DEVICE_TIMEOUT);
            umma_commit(drain);  // completes once every MMA issued so far has finished
            mbar_wait_bounded(drain, 0, nullptr, p.timeout_ns);
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        int local = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++local) {
            const int acc = local & 1;
            if (!warp_wait(&tfull[acc], (local >> 1) & 1, abort_flag, p.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            int m, n;
            tile_coords(t / S, num_m, num_n, p.group_m, p.raster, m, n);
            const int row = m * TBM + q * 32 + lane;
            const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * TBN);
            if (S == 1)
                drain_256<T, EPI>(tbase, p, row, n * TBN, M);
            else
                drain_256_partial(tbase, p.partials + ((int64_t)(t % S) * p.M_cap) * p.N, p.N, row, n * TBN, M);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            status_or(p.status, ENERGON_DEVICE_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 2) tmem_dealloc(tmem, TMEM_COLS);
}

// Spin for about `ns` nanoseconds (used only on the abort path to let copies land).
__device__ __forceinline__ void spin_ns(uint64_t ns) {
    const uint64_t t0 = global_ns();
    for (uint32_t it = 0; it < (1u << 26) && global_ns() - t0 < ns; ++it) {
    }
}

// The CTA-pair variant.  Both CTAs of a 2-CTA cluster load their halves of A
// (by rows) and W (by the tile's columns) into their own shared memory; the
// completion of every copy is counted on the leader CTA's `full` barrier.  The
// leader's MMA thread issues tcgen05.mma.cta_group::2 over both CTAs' shared
// memory; each CTA receives its 128 accumulator rows in its own TMEM.  Commits
// multicast to both CTAs (ring slots and accumulator hand-off); the peer's
// epilogue hands accumulators back by arriving on the leader's barrier.
//
// MT = row tiles per pair tile, BN = the tile's columns.  MT = 1: 256 x BN tiles,
// 6-stage ring, two TMEM accumulators so the epilogue of one tile overlaps the MMAs of
// the next.  MT = 2: 512 x BN tiles, the staged W panel feeds both row tiles (a quarter
// less L2 -> SMEM traffic and shared-memory bandwidth per flop than MT = 1 at BN = 256),
// 4-stage ring; the accumulators of two tiles fit in TMEM only for BN <= 128, otherwise
// one accumulator is drained by eight epilogue warps between tiles.  BN in {128, 192, 256}:
// narrower tiles leave less of the last round of tiles idle when N / BN tiles do not fill
// the CTA pairs evenly.
template <int MT, int BN = 256>
struct PairCfg {
    static_assert(BN % 64 == 0 && BN >= 128 && BN <= 256, "tile columns");
    static constexpr int STAGES = MT == 1 ? 6 : 4;
    static constexpr int A_STAGE = MT * PA_STAGE;        // MT boxes of 128 rows x 64
    static constexpr int B_STAGE = (BN / 2) * PBK * 2;   // this CTA's BN / 2 rows of W x 64
    static constexpr int STAGE = A_STAGE + B_STAGE;
    static constexpr int SLOT_COLS = MT * BN;
    static constexpr int SLOTS = 2 * SLOT_COLS <= 512 ? 2 : 1;  // TMEM accumulator slots
    static constexpr int CH = BN / 32;                   // 32-column epilogue chunks per row tile
    static constexpr int EPI_WARPS = 4 * MT;
    static constexpr int THREADS = 128 + 32 * EPI_WARPS;
    static constexpr int EPI_STAGE = 4096;  // per epilogue warp: two 32 x 32 staging buffers
    static constexpr int SMEM = STAGES * STAGE + EPI_WARPS * EPI_STAGE + 1024 + 384;
    static_assert(SMEM <= 232448, "shared memory per CTA");
};

template <typename T, int EPI, int MT, int BN>
__global__ void __launch_bounds__(PairCfg<MT, BN>::THREADS, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmBq, const __grid_constant__ CUtensorMap tmO,
                    const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmL,
                    const TcParams p) {
    using C = PairCfg<MT, BN>;
    constexpr int NST = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = base;                    // [stage][MT][128 rows x 128 B]
    uint8_t* sB = base + NST * C::A_STAGE;  // [stage][BN / 2 rows x 128 B]
    uint8_t* sE = sB + NST * C::B_STAGE;    // [epilogue warp][2][32 rows x 64 B]
    uint64_t* full = reinterpret_cast<uint64_t*>(sE + C::EPI_WARPS * C::EPI_STAGE);
    uint64_t* empty = full + NST;
    uint64_t* tfull = empty + NST;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint64_t* rbar = drain + 1;             // [epilogue warp][2] residual copies
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rbar + 2 * C::EPI_WARPS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    // Every early exit below is taken by both CTAs of the pair or by neither.
    if (status_bad(p.status)) return;
    const int M = min(*p.d_rows, p.M_cap);
    if (M <= 0) return;
    const int num_m = (M + PBM - 1) / PBM;               // 256-row tiles
    const int num_mt = (num_m + MT - 1) / MT;            // pair tiles along M
    const int num_n = (p.N + BN - 1) / BN;
    const int total = num_mt * num_n;
    // Wave tail: the tiles of the last, partly filled round are cut into s units (s = 1,
    // 2 or 4, the one that finishes the round soonest): 2 = one row tile each, 4 = one row
    // tile and half the columns each (MMA N = BN / 2).  A row's arithmetic is the same in
    // every cut (the same MMA per row and column, the same K order), so results do not
    // depend on how the tiles were cut.
    int full_units = total, split_tiles = 0, split = 1;
    if (MT == 2) {
        const int rem = total % npairs;
        const int full_rounds = total / npairs;
        if (rem != 0) {
            // round time of the tail in units of a full tile: ceil(rem s / npairs) / s
            int best = 1;
            float best_t = (float)((rem + npairs - 1) / npairs);
            for (int s = 2; s <= 4; s *= 2) {
                const float t_s = (float)((rem * s + npairs - 1) / npairs) / (float)s;
                if (t_s < best_t - 1e-6f) best_t = t_s, best = s;
            }
            if (best > 1) full_units = full_rounds * npairs, split_tiles = rem, split = best;
        }
    }
    const int units = full_units + split * split_tiles;
    if (pair >= units) return;
    const int num_kb = (p.K + PBK - 1) / PBK;
    // Tile order: groups of 8 pair tiles (4096 rows); inside a group every row tile of a
    // column runs before the next column, so the pairs that share a weight panel mostly
    // run in the same round and fetch it once.  The K direction alternates from one
    // round's worth of panels to the next: a round then starts on the K slices of A that
    // the previous round fetched last, while they are still in L2.  Against groups of 4
    // pair tiles walked forwards this read 8-18 % fewer DRAM bytes on the four GPT-3
    // shapes at T = 4096 and ran about 1 % faster; L2 eviction-priority hints made the
    // kernel 10 % slower.
    const int group = 8;
    // unit u -> pair tile t, its row tiles [i0, i1) and column half h (-1: all columns).  A
    // full tile of the last pair row keeps only the row tiles that hold rows below M (an odd
    // number of 256-row tiles leaves the last pair row half empty: its MMAs are skipped).
    auto unit_of = [&](int u, int& t, int& i0, int& i1, int& h) {
        h = -1;
        if (u < full_units) {
            t = u, i0 = 0, i1 = MT;
            if (MT > 1 && num_m % MT != 0) {
                int mt_, n_;
                tile_coords(t, num_mt, num_n, group, 0, mt_, n_);
                if (mt_ == num_mt - 1) i1 = num_m - mt_ * MT;
            }
        } else {
            const int v = u - full_units;
            if (split == 2) {
                t = full_units + (v >> 1), i0 = v & 1;
            } else {
                t = full_units + (v >> 2), i0 = (v >> 1) & 1, h = v & 1;
            }
            i1 = i0 + 1;
        }
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 2 * C::EPI_WARPS);  // every epilogue warp of both CTAs
        }
        mbar_init(drain, 1);
        for (int w = 0; w < 2 * C::EPI_WARPS; ++w) mbar_init(&rbar[w], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (!Epi<EPI>::OUT_F32) tma_prefetch_desc(&tmO);
        if (Epi<EPI>::RES_T) tma_prefetch_desc(&tmR);
        if (Epi<EPI>::FOLD && p.lo != nullptr) tma_prefetch_desc(&tmL);
    }
    if (warp == 2) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised, TMEM of both allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer (both CTAs)
        int stage = 0;
        uint32_t phase = 0, pend_mask = 0, pend_par = 0;
        bool ok = true;
        for (int u = pair; u < units && ok; u += npairs) {
            int t, i0, i1, h, mt, n;
            unit_of(u, t, i0, i1, h);
            tile_coords(t, num_mt, num_n, group, 0, mt, n);
            // K direction of column panel n: it flips every npairs / group panels, about once a
            // round, and depends on the panel alone, so a row's result is the same whichever
            // round and row tile it lands in (packed, padded and per-MLP runs agree bit for bit)
            const bool rev = (((n * group) / npairs) & 1) != 0;
            const uint32_t tx = 2u * (uint32_t)((i1 - i0) * PA_STAGE + (h < 0 ? C::B_STAGE : C::B_STAGE / 2));
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!warp_wait<true>(&empty[stage], phase ^ 1u, abort_flag, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    const int kc = (rev ? num_kb - 1 - kb : kb) * PBK;
                    const uint32_t bar0 = mapa_shared(smem_u32(&full[stage]), 0);
                    if (leader) mbar_arrive_expect_tx(&full[stage], tx);
#pragma unroll
                    for (int i = 0; i < MT; ++i)
                        if (i >= i0 && i < i1)
                            tma_load_2d_pair(sA + stage * C::A_STAGE + i * PA_STAGE, &tmA, bar0, kc,
                                             (mt * MT + i) * PBM + (int)rank * 128);
                    if (h < 0)
                        tma_load_2d_pair(sB + stage * C::B_STAGE, &tmB, bar0, kc, n * BN + (int)rank * (BN / 2));
                    else  // this CTA's BN / 4 rows of the column half
                        tma_load_2d_pair(sB + stage * C::B_STAGE, &tmBq, bar0, kc,
                                         n * BN + h * (BN / 2) + (int)rank * (BN / 4));
                }
                pend_mask |= 1u << stage;
                pend_par = (pend_par & ~(1u << stage)) | (phase << stage);
                if (++stage == NST) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            status_or(p.status, ENERGON_DEVICE_TIMEOUT);
            if (leader) {
                for (int s = 0; s < NST; ++s)
                    if (pend_mask & (1u << s))
                        mbar_wait_bounded(&full[s], (pend_par >> s) & 1u, nullptr, p.timeout_ns);
            } else {
                // The peer's copies report to the leader's barriers; give them time to land.
                spin_ns(p.timeout_ns < 1000000ull ? p.timeout_ns : 1000000ull);
            }
        }
    } else if (warp == 1 && leader) {
        // ---------------------------------------------------------------- MMA issuer (leader CTA)
        constexpr uint32_t fmt = sizeof(T) == 2 && !std::is_same<T, __half>::value ? 1u : 0u;
        constexpr uint32_t idesc = idesc_f16(fmt, PBM, BN);
        constexpr uint32_t idesc_h = idesc_f16(fmt, PBM, BN / 2);
        int stage = 0, local = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int u = pair; u < units && ok; u += npairs, ++local) {
            int t, i0, i1, h;
            unit_of(u, t, i0, i1, h);
            const int slot = local % C::SLOTS;
            const uint32_t use = (uint32_t)(local / C::SLOTS) & 1u;
            if (!warp_wait<true>(&tempty[slot], use ^ 1u, abort_flag, p.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem + (uint32_t)(slot * C::SLOT_COLS);
            for (int kb = 0; kb < num_kb; ++kb) {
                if (!warp_wait<true>(&full[stage], phase, abort_flag, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (lane == 0) {
                    const uint64_t b0 = smem_desc_k128(smem_u32(sB + stage * C::B_STAGE));
                    // One thread issues an MMA every ~128 tensor cycles here, so the issue
                    // loops stay fully unrolled (a runtime-bounded loop measured 11 % slower).
                    if (i1 - i0 == MT) {
#pragma unroll
                        for (int k = 0; k < PBK / 16; ++k) {
#pragma unroll
                            for (int i = 0; i < MT; ++i) {
                                const uint64_t a0 =
                                    smem_desc_k128(smem_u32(sA + stage * C::A_STAGE + i * PA_STAGE));
                                umma_f16_pair(d_tmem + (uint32_t)(i * BN), a0 + 2 * k, b0 + 2 * k, idesc,
                                              (kb | k) != 0 ? 1u : 0u);
                            }
                        }
                    } else if (h < 0) {
                        const uint64_t a0 = smem_desc_k128(smem_u32(sA + stage * C::A_STAGE + i0 * PA_STAGE));
                        const uint32_t dt = d_tmem + (uint32_t)(i0 * BN);
#pragma unroll
                        for (int k = 0; k < PBK / 16; ++k)
                            umma_f16_pair(dt, a0 + 2 * k, b0 + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
                    } else {
                        const uint64_t a0 = smem_desc_k128(smem_u32(sA + stage * C::A_STAGE + i0 * PA_STAGE));
                        const uint32_t dt = d_tmem + (uint32_t)(i0 * BN + h * (BN / 2));
#pragma unroll
                        for (int k = 0; k < PBK / 16; ++k)
                            umma_f16_pair(dt, a0 + 2 * k, b0 + 2 * k, idesc_h, (kb | k) != 0 ? 1u : 0u);
                    }
                    umma_commit_pair(&empty[stage], 0x3);
                }
                __syncwarp();
                if (++stage == NST) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (lane == 0) umma_commit_pair(&tfull[slot], 0x3);
            __syncwarp();
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            status_or(p.status, ENERGON_DEVICE_TIMEOUT);
            umma_commit_pair(drain, 0x1);
            mbar_wait_bounded(drain, 0, nullptr, p.timeout_ns);
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- epilogue (both CTAs)
        const int q = warp & 3;             // TMEM lane quarter this warp may access
        const int i = (warp - 4) >> 2;      // row tile of the pair tile this warp drains
        uint8_t* sbuf = sE + (warp - 4) * C::EPI_STAGE;
        uint64_t* rb = rbar + 2 * (warp - 4);
        uint32_t rpar = 0;
        int local = 0;
        bool ok = true;
        for (int u = pair; u < units; u += npairs, ++local) {
            int t, i0, i1, h;
            unit_of(u, t, i0, i1, h);
            const int slot = local % C::SLOTS;
            const uint32_t use = (uint32_t)(local / C::SLOTS) & 1u;
            if (!warp_wait(&tfull[slot], use, abort_flag, p.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tempty_cluster = mapa_shared(smem_u32(&tempty[slot]), 0);
            bool handed_back = false;
            if (i >= i0 && i < i1) {  // a half unit leaves the other row tile's warps idle
                int mt, n;
                tile_coords(t, num_mt, num_n, group, 0, mt, n);
                const int row_base = (mt * MT + i) * PBM + (int)rank * 128 + q * 32;
                const int cofs = h < 0 ? 0 : h * (BN / 2);  // first column of this unit in the tile
                const uint32_t tbase =
                    tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(slot * C::SLOT_COLS + i * BN + cofs);
                // a 32-row box is one TMA store when its rows are valid and (scattering)
                // lie in one sequence, so that their padded rows are consecutive too
                bool box = row_base + 32 <= M;
                int out_base = row_base;
                if (box && p.scatter_cu != nullptr) {
                    const int b = owner_of(p.scatter_cu, p.scatter_batch, row_base);
                    const int start = __ldg(p.scatter_cu + b);
                    box = row_base + 32 <= __ldg(p.scatter_cu + b + 1);
                    out_base = b * p.scatter_pad_len + (row_base - start);
                }
                if (box && h < 0) {
                    ok = drain_256_staged<T, EPI, C::CH>(tbase, p, &tmO, &tmR, &tmL, sbuf, rb, rpar, row_base,
                                                         out_base, n * BN, tempty_cluster, abort_flag);
                    handed_back = ok;
                } else if (box) {
                    ok = drain_staged_rare<T, EPI, C::CH / 2>(tbase, p, &tmO, &tmR, &tmL, sbuf, rb, rpar, row_base,
                                                              out_base, n * BN + cofs, tempty_cluster, abort_flag);
                    handed_back = ok;
                } else if (h < 0) {
                    drain_rows_rare<T, EPI, C::CH>(tbase, p, row_base + lane, n * BN, M);
                } else {
                    drain_rows_rare<T, EPI, C::CH / 2>(tbase, p, row_base + lane, n * BN + cofs, M);
                }
            }
            if (!ok) break;
            if (!handed_back) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(tempty_cluster);
            }
        }
        if (lane == 0) {
            if (!ok) {
                *abort_flag = 1;
                status_or(p.status, ENERGON_DEVICE_TIMEOUT);
            }
            bulk_wait<0>();  // every output store has landed before the CTA retires
        }
        __syncwarp();
    }
    tc_fence_before();
    cluster_sync();  // neither CTA leaves while its pair may still read or signal its shared memory
    tc_fence_after();
    if (warp == 2) tmem_dealloc_pair(tmem, TMEM_COLS);
}

// ------------------------------------------------------------------ host side

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D K-major tensor [rows, K] of 16-bit elements, box 64 x box_rows, 128-byte swizzle.
static CUresult make_tmap(CUtensorMap* m, int dtype, const void* ptr, int64_t K, int64_t rows, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return CUDA_ERROR_NOT_FOUND;
    const CUtensorMapDataType dt =
        dtype == ENERGON_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {(cuuint32_t)TBK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// 2-D row-major tensor [rows, N] of 16-bit elements, box 32 x 32, 64-byte swizzle.
static CUresult make_tmap_io(CUtensorMap* m, int dtype, const void* ptr, int64_t N, int64_t rows) {
    auto fn = encode_fn();
    if (!fn) return CUDA_ERROR_NOT_FOUND;
    const CUtensorMapDataType dt =
        dtype == ENERGON_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)N * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// fp32 [rows, N] in 16 x 32 boxes, 64-byte swizzle (the staging buffers' layout).
static CUresult make_tmap_f32(CUtensorMap* m, const void* ptr, int64_t N, int64_t rows) {
    auto fn = encode_fn();
    if (!fn) return CUDA_ERROR_NOT_FOUND;
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)N * 4};
    cuuint32_t box[2] = {16, 32};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// Single-CTA tiles for a GEMM whose rows fit in one 128-row tile (the skinny,
// weight-streaming case): more CTAs stream weights than with 256-row pair tiles.
static bool use_single_cta(const GemmArgs& a) { return a.M_cap <= TBM; }

bool gemm_tc_scatter_ok(const GemmArgs& a) { return gemm_tc_supported(a) && !use_single_cta(a); }

// The epilogues the layer uses: the folded LayerNorm (QKV), bias + GELU (FFN1), bias +
// residual into fp32 (out-projection), bias + fp32 residual (FFN2).
static bool tc_epilogue(int epi) {
    return epi == EPI_LN_FOLD || epi == EPI_BIAS_GELU || epi == EPI_RES_OUT32 || epi == EPI_RES32;
}

bool gemm_tc_supported(const GemmArgs& a) {
    if (a.dtype != ENERGON_F16 && a.dtype != ENERGON_BF16) return false;
    if (!tc_epilogue(a.epilogue)) return false;
    if (a.K < TBK || a.K % TBK != 0 || a.N < TBN || a.N % TBN != 0) return false;
    if (a.M_cap <= 0 || a.A_rows < PBM || a.A_rows % PBM != 0 || a.A_rows < a.M_cap) return false;
    const bool res = a.epilogue == EPI_RES_OUT32 || a.epilogue == EPI_RES32;
    if (res && a.residual == nullptr) return false;
    if (a.epilogue == EPI_LN_FOLD) {
        if (!a.fold_stats || !a.fold_c || !a.fold_d) return false;
        if (a.lo != nullptr && (a.lo_cols <= 0 || a.lo_cols % TBN != 0 || a.lo_cols > a.N)) return false;
    }
    const uintptr_t al = (uintptr_t)a.A | (uintptr_t)a.W | (uintptr_t)a.out | (uintptr_t)a.bias |
                         (uintptr_t)(res ? a.residual : nullptr) | (uintptr_t)a.lo | (uintptr_t)a.fold_c |
                         (uintptr_t)a.fold_d | (uintptr_t)a.fold_stats;
    if (al % 16 != 0) return false;
    return encode_fn() != nullptr;
}

template <typename T, int EPI>
static cudaError_t tc_launch(const CUtensorMap& ta, const CUtensorMap& tb, const TcParams& p, int grid,
                             cudaStream_t st) {
    cudaError_t e = prepare_smem((const void*)gemm_tc_kernel<T, EPI>, TC_SMEM);
    if (e != cudaSuccess) return e;
    gemm_tc_kernel<T, EPI><<<grid, 256, TC_SMEM, st>>>(ta, tb, p);
    return cudaGetLastError();
}

template <typename T, int EPI, int MT, int BN = 256>
static cudaError_t tc2_launch(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tbq,
                              const CUtensorMap& to, const CUtensorMap& tr, const CUtensorMap& tl, const TcParams& p,
                              int pairs, cudaStream_t st) {
    using C = PairCfg<MT, BN>;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    const void* kernel = (const void*)gemm_tc2_kernel<T, EPI, MT, BN>;
    cudaError_t e = prepare_smem(kernel, C::SMEM);
    if (e != cudaSuccess) return e;
    // CTA pairs that fit on this device at once (the persistent grid)
    const int max_pairs = device_cached(kernel, 1, [&] {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (device_sm_count() / 2));
        cfg.blockDim = dim3(C::THREADS);
        cfg.dynamicSmemBytes = C::SMEM;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, gemm_tc2_kernel<T, EPI, MT, BN>, &cfg) != cudaSuccess ||
            clusters < 1)
            clusters = device_sm_count() / 2;
        (void)cudaGetLastError();
        return clusters;
    });
    if (pairs > max_pairs) pairs = max_pairs;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemm_tc2_kernel<T, EPI, MT, BN>, ta, tb, tbq, to, tr, tl, p);
}

template <typename T, int MT>
static cudaError_t tc2_dispatch(int epi, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tbq,
                                const CUtensorMap& to, const CUtensorMap& tr, const CUtensorMap& tl, const TcParams& p,
                                int pairs, cudaStream_t st) {
    switch (epi) {
    case EPI_LN_FOLD: return tc2_launch<T, EPI_LN_FOLD, MT>(ta, tb, tbq, to, tr, tl, p, pairs, st);
    case EPI_BIAS_GELU: return tc2_launch<T, EPI_BIAS_GELU, MT>(ta, tb, tbq, to, tr, tl, p, pairs, st);
    case EPI_RES_OUT32: return tc2_launch<T, EPI_RES_OUT32, MT>(ta, tb, tbq, to, tr, tl, p, pairs, st);
    default: return tc2_launch<T, EPI_RES32, MT>(ta, tb, tbq, to, tr, tl, p, pairs, st);
    }
}

template <typename T>
static cudaError_t single_dispatch(int epi, const CUtensorMap& ta, const CUtensorMap& tb, const TcParams& p,
                                   int grid, int fgrid, cudaStream_t st) {
    cudaError_t e;
    switch (epi) {
    case EPI_LN_FOLD: e = tc_launch<T, EPI_LN_FOLD>(ta, tb, p, grid, st); break;
    case EPI_BIAS_GELU: e = tc_launch<T, EPI_BIAS_GELU>(ta, tb, p, grid, st); break;
    case EPI_RES_OUT32: e = tc_launch<T, EPI_RES_OUT32>(ta, tb, p, grid, st); break;
    default: e = tc_launch<T, EPI_RES32>(ta, tb, p, grid, st); break;
    }
    if (e != cudaSuccess || p.k_splits == 1) return e;
    switch (epi) {
    case EPI_LN_FOLD: splitk_finish_kernel<T, EPI_LN_FOLD><<<fgrid, 256, 0, st>>>(p.partials, p.k_splits, p); break;
    case EPI_BIAS_GELU:
        splitk_finish_kernel<T, EPI_BIAS_GELU><<<fgrid, 256, 0, st>>>(p.partials, p.k_splits, p);
        break;
    case EPI_RES_OUT32:
        splitk_finish_kernel<T, EPI_RES_OUT32><<<fgrid, 256, 0, st>>>(p.partials, p.k_splits, p);
        break;
    default: splitk_finish_kernel<T, EPI_RES32><<<fgrid, 256, 0, st>>>(p.partials, p.k_splits, p); break;
    }
    return cudaGetLastError();
}

cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t st, char* err, size_t errlen) {
    const bool single = use_single_cta(a);
    CUtensorMap ta, tb;
    CUresult r1 = make_tmap(&ta, a.dtype, a.A, a.K, a.A_rows, single ? TBM : 128);
    CUresult r2 = make_tmap(&tb, a.dtype, a.W, a.K, a.N, single ? TBN : 128);
    if (r1 != CUDA_SUCCESS || r2 != CUDA_SUCCESS) {
        if (err) snprintf(err, errlen, "cuTensorMapEncodeTiled failed (A: %d, W: %d)", (int)r1, (int)r2);
        return cudaErrorInvalidValue;
    }
    TcParams p{};
    p.bias = a.bias;
    p.residual = a.residual;
    p.out = a.out;
    p.d_rows = a.d_rows;
    p.status = a.status;
    p.M_cap = a.M_cap;
    p.N = a.N;
    p.K = a.K;
    p.gelu_tanh = a.gelu_tanh;
    p.timeout_ns = a.timeout_ns;
    p.k_splits = 1;
    p.partials = nullptr;
    p.scatter_cu = a.scatter_cu;
    p.scatter_batch = a.scatter_batch;
    p.scatter_pad_len = a.scatter_pad_len;
    p.fold_stats = a.fold_stats;
    p.fold_c = a.fold_c;
    p.fold_d = a.fold_d;
    p.lo = a.epilogue == EPI_LN_FOLD ? a.lo : nullptr;
    p.lo_cols = p.lo ? a.lo_cols : 0;
    {
        const void* rows32 = a.epilogue == EPI_RES32 ? a.residual : nullptr;
        p.wide32 = rows32 != nullptr && (uintptr_t)rows32 % 32 == 0 && ((size_t)a.N * 4) % 32 == 0 ? 1 : 0;
    }
    const bool bf = a.dtype == ENERGON_BF16;
    if (a.scatter_cu != nullptr && (single || a.epilogue == EPI_RES_OUT32 || a.epilogue == EPI_LN_FOLD)) {
        if (err) snprintf(err, errlen, "a scattering epilogue needs the CTA-pair path (more than %d rows) and a "
                                       "16-bit output without low halves", TBM);
        return cudaErrorInvalidValue;
    }
    if (!single) {
        // Pair tiles of two row tiles (512 x 256) once the buffer can hold two: every
        // staged weight panel then feeds 512 rows.
        const int mt = a.M_cap > PBM ? 2 : 1;
        const int num_m_cap = (a.M_cap + PBM * mt - 1) / (PBM * mt), num_n = a.N / PBN;
        p.raster = 0;
        p.group_m = 1;
        const int64_t tiles_cap = (int64_t)num_m_cap * num_n;
        const int pairs = (int)(tiles_cap < device_sm_count() / 2 ? tiles_cap : device_sm_count() / 2);
        // Output, residual and low halves as 32 x 32 boxes, 64-byte swizzle: the epilogue's
        // staged stores and residual loads.  Only boxes of rows below the live row count are
        // ever copied, so the maps may span the whole buffer capacity.  A map the epilogue
        // does not use is a copy of one that exists.
        CUtensorMap to, tr, tl;
        const int64_t out_rows = a.scatter_cu ? (int64_t)a.scatter_batch * a.scatter_pad_len : a.M_cap;
        CUresult r3 = CUDA_SUCCESS, r4 = CUDA_SUCCESS, r5 = CUDA_SUCCESS;
        if (a.epilogue == EPI_RES_OUT32) {
            r4 = make_tmap_io(&tr, a.dtype, a.residual, a.N, a.M_cap);
            r3 = make_tmap_f32(&to, a.out, a.N, a.M_cap);
        } else {
            r3 = make_tmap_io(&to, a.dtype, a.out, a.N, out_rows);
            tr = to;
        }
        if (p.lo != nullptr) r5 = make_tmap_io(&tl, a.dtype, p.lo, p.lo_cols, a.M_cap);
        else tl = to;
        // W boxes of half the height, for the wave-tail units that take half of a tile's columns
        CUtensorMap tbq;
        CUresult r6 = make_tmap(&tbq, a.dtype, a.W, a.K, a.N, 64);
        if (r6 != CUDA_SUCCESS) {
            if (err) snprintf(err, errlen, "cuTensorMapEncodeTiled failed (W half boxes: %d)", (int)r6);
            return cudaErrorInvalidValue;
        }
        if (r3 != CUDA_SUCCESS || r4 != CUDA_SUCCESS || r5 != CUDA_SUCCESS) {
            if (err)
                snprintf(err, errlen, "cuTensorMapEncodeTiled failed (out: %d, residual: %d, low halves: %d)", (int)r3,
                         (int)r4, (int)r5);
            return cudaErrorInvalidValue;
        }
        if (mt == 2)
            return bf ? tc2_dispatch<__nv_bfloat16, 2>(a.epilogue, ta, tb, tbq, to, tr, tl, p, pairs, st)
                      : tc2_dispatch<__half, 2>(a.epilogue, ta, tb, tbq, to, tr, tl, p, pairs, st);
        return bf ? tc2_dispatch<__nv_bfloat16, 1>(a.epilogue, ta, tb, tbq, to, tr, tl, p, pairs, st)
                  : tc2_dispatch<__half, 1>(a.epilogue, ta, tb, tbq, to, tr, tl, p, pairs, st);
    }
    const int num_m_cap = (a.M_cap + TBM - 1) / TBM, num_n = a.N / TBN;
    // Rows of A kept hot per raster group: about 48 MiB of the 126 MB L2.
    int gm = (int)((48ll << 20) / ((int64_t)TBM * a.K * 2));
    p.group_m = gm < 1 ? 1 : (gm > num_m_cap ? num_m_cap : gm);
    p.raster = 0;
    // Weight-streaming GEMMs with few output tiles split K so that every SM streams:
    // S minimises (rounds of units over the SMs) / S, e.g. 48 tiles -> 3 splits.
    const int sms = device_sm_count();
    const int64_t tiles = (int64_t)num_m_cap * num_n;
    const int num_kb = a.K / TBK;
    int S = 1;
    double best = (double)((tiles + sms - 1) / sms);
    for (int cand = 2; cand <= 4; ++cand) {
        if (num_kb % cand != 0) continue;
        if (a.partials == nullptr || (size_t)cand * a.M_cap * a.N * sizeof(float) > a.partials_bytes) continue;
        const double cost = (double)((tiles * cand + sms - 1) / sms) / cand;
        if (cost < best - 1e-9) {
            best = cost;
            S = cand;
        }
    }
    p.k_splits = S;
    p.partials = a.partials;
    const int64_t units = tiles * S;
    const int grid = (int)(units < sms ? units : sms);
    const int64_t work = (int64_t)a.M_cap * (a.N / 32);
    const int fgrid = (int)((work + 255) / 256 < 4 * sms ? (work + 255) / 256 : 4 * sms);
    return bf ? single_dispatch<__nv_bfloat16>(a.epilogue, ta, tb, p, grid, fgrid, st)
              : single_dispatch<__half>(a.epilogue, ta, tb, p, grid, fgrid, st);
}

}  // namespace energon
