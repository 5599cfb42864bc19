// attn_tc.cu -- block-sparse attention forward on the 5th-generation tensor
// cores (tcgen05, TMEM accumulators, TMA tile loads).
//
// [Prism guide, Method section 3, last sentence]: each query block attends,
// under one online softmax, to the tokens of the key blocks in S_i.
//
// Work unit: one 128-row query tile of one head (a 256-token block gives two
// tiles, a 128-token block one, a 64-token block one tile whose upper 64 rows
// are computed and discarded).  The selected key blocks are streamed as
// 64-row segments; two segments form a 128-key chunk.
//
// Warp roles (192 threads):
//   warp 0       TMA producer: Q tile once, then K and V chunks into a
//                two-stage ring (each stage 128 keys x D, 128-byte swizzle).
//   warp 1       MMA issuer (one thread): S_c = Q K_c^T into one of two TMEM
//                S buffers, then O += P_c V_c with P_c read from TMEM.
//   warps 2..5   softmax, one query row per thread (= TMEM lane): row max,
//                exp2, running sum; P_c written back over S_c as bf16; O is
//                rescaled in TMEM only when the running max grows by more
//                than 2^8.  Epilogue: O / l to the user layout, log-sum-exp.
// TMEM columns: S buffer 0 [0,128), S buffer 1 [128,256), O [256, 256+D).
#include <cuda.h>

#include "tc_common.cuh"

namespace prism {

using namespace tc;

namespace fwdtc {

constexpr int kThreads = 192;
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct Layout {
    static constexpr int kHalves = D / 64;               // 64-column (128 B) swizzle atoms along D
    static constexpr uint32_t kTileBytes = 128 * 128;    // 128 rows x 128 B
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK0 = kQ + kHalves * kTileBytes;
    static constexpr uint32_t kStageBytes = 2 * kHalves * kTileBytes;  // K and V
    static constexpr uint32_t kBars = kK0 + kStages * kStageBytes;
    // barriers: q, k[S], v[S], kv_empty[S], s[2], p[2], o  (8 B each) + tmem slot + abort
    static constexpr uint32_t kNumBars = 1 + 3 * kStages + 2 + 2 + 1;
    static constexpr uint32_t kBytes = kBars + kNumBars * 8 + 16;
    static constexpr uint32_t kAlloc = kBytes + 1024;  // slack to align the base to 1024
};

// Site codes recorded with a timeout.
enum { kSiteQ = 1, kSiteK, kSiteV, kSiteEmpty, kSiteS, kSiteP, kSiteO };

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_fwd_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, Geo g, const int *__restrict__ nqt,
                  const int *__restrict__ qt_row, const int *__restrict__ qt_blk, const int *__restrict__ blk_off,
                  const int *__restrict__ row_ptr, const int *__restrict__ col, const int *__restrict__ perm,
                  __nv_bfloat16 *__restrict__ O, float *__restrict__ lse_user, float *__restrict__ lse_p,
                  float scale_log2, int *__restrict__ status) {
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);

    const int tile = blockIdx.x, bh = blockIdx.y, b = bh / g.heads, h = bh % g.heads;
    if (tile >= nqt[b]) return;
    if (*reinterpret_cast<volatile int *>(status) != 0) return;  // an earlier CTA timed out: fail fast
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int *bo = blk_off + (size_t)b * (g.nbmax + 1);
    const int q0 = qt_row[(size_t)b * g.nbmax + tile];
    const int iblk = qt_blk[(size_t)b * g.nbmax + tile];
    const int qvalid = min(128, bo[iblk + 1] - q0);
    const size_t crow = (size_t)bh * g.nbmax + iblk;
    const int c_begin = row_ptr[crow], c_end = row_ptr[crow + 1];

    // number of 64-row key segments of the selection (every warp computes it)
    int nseg = 0;
    for (int u = c_begin + lane; u < c_end; u += 32) {
        const int j = col[u];
        nseg += (bo[j + 1] - bo[j]) >> 6;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nseg += __shfl_xor_sync(0xffffffffu, nseg, o);
    const int nchunk = (nseg + 1) >> 1;

    const uint32_t bar_q = sbase + L::kBars;
    const uint32_t bar_k = bar_q + 8;                  // [kStages]
    const uint32_t bar_v = bar_k + 8 * kStages;        // [kStages]
    const uint32_t bar_e = bar_v + 8 * kStages;        // [kStages] kv stage empty
    const uint32_t bar_s = bar_e + 8 * kStages;        // [2]
    const uint32_t bar_p = bar_s + 16;                 // [2]
    const uint32_t bar_o = bar_p + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kBars + L::kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kBars + L::kNumBars * 8 + 8);

    if (warp == 0) {
        if (lane == 0) {
            mbar_init(bar_q, 1);
            for (int s = 0; s < kStages; ++s) {
                mbar_init(bar_k + 8 * s, 1);
                mbar_init(bar_v + 8 * s, 1);
                mbar_init(bar_e + 8 * s, 1);
            }
            for (int s = 0; s < 2; ++s) {
                mbar_init(bar_s + 8 * s, 1);
                mbar_init(bar_p + 8 * s, 128);
            }
            mbar_init(bar_o, 1);
            *abort_flag = 0;
            mbar_fence_init();
            prefetch_map(&tmQ);
            prefetch_map(&tmK);
            prefetch_map(&tmV);
        }
        __syncwarp();
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS0 = tmem, tO = tmem + 256;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const int rowbase = bh * g.N;
            mbar_expect_tx(bar_q, 128 * D * 2);
            for (int hf = 0; hf < L::kHalves; ++hf)
                for (int rh = 0; rh < 2; ++rh)
                    tma_load_2d(sbase + L::kQ + hf * L::kTileBytes + rh * 8192, &tmQ, bar_q, hf * 64,
                                rowbase + q0 + rh * 64);
            int u = c_begin, r = 0, r_end = 0;
            if (u < c_end) {
                r = bo[col[u]];
                r_end = bo[col[u] + 1];
            }
            int issued = 0;
            for (int c = 0; c < nchunk; ++c) {
                const int st = c % kStages;
                if (c >= kStages && !mbar_wait(bar_e + 8 * st, ((c / kStages) + 1) & 1, status, kSiteEmpty,
                                               abort_flag))
                    break;
                const int nsg = min(2, nseg - 2 * c);
                const uint32_t bytes = nsg * 64 * D * 2;
                const uint32_t sK = sbase + L::kK0 + st * L::kStageBytes;
                const uint32_t sV = sK + L::kHalves * L::kTileBytes;
                int rows[2];
                for (int gsg = 0; gsg < nsg; ++gsg) {
                    rows[gsg] = r;
                    r += 64;
                    if (r >= r_end && ++u < c_end) {
                        r = bo[col[u]];
                        r_end = bo[col[u] + 1];
                    }
                }
                mbar_expect_tx(bar_k + 8 * st, bytes);
                for (int gsg = 0; gsg < nsg; ++gsg)
                    for (int hf = 0; hf < L::kHalves; ++hf)
                        tma_load_2d(sK + hf * L::kTileBytes + gsg * 8192, &tmK, bar_k + 8 * st, hf * 64,
                                    rowbase + rows[gsg]);
                mbar_expect_tx(bar_v + 8 * st, bytes);
                for (int gsg = 0; gsg < nsg; ++gsg)
                    for (int hf = 0; hf < L::kHalves; ++hf)
                        tma_load_2d(sV + hf * L::kTileBytes + gsg * 8192, &tmV, bar_v + 8 * st, hf * 64,
                                    rowbase + rows[gsg]);
                issued = c + 1;
            }
            // drain: every issued load must land before the CTA may exit
            for (int c = max(0, issued - kStages); c < issued; ++c) {
                const int st = c % kStages;
                mbar_wait(bar_k + 8 * st, (c / kStages) & 1, status, kSiteK, abort_flag);
                mbar_wait(bar_v + 8 * st, (c / kStages) & 1, status, kSiteV, abort_flag);
            }
            mbar_wait(bar_q, 0, status, kSiteQ, abort_flag);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        {  // the whole warp runs the issue loop; elect.sync picks one lane
            constexpr uint32_t idS128 = idesc_bf16(128, 128, false), idS64 = idesc_bf16(128, 64, false);
            constexpr uint32_t idPV = idesc_bf16(128, D, true);
            bool ok = __all_sync(0xffffffffu, mbar_wait(bar_q, 0, status, kSiteQ, abort_flag));
            auto issue_s = [&](int c) -> bool {
                const int st = c % kStages;
                if (!__all_sync(0xffffffffu, mbar_wait(bar_k + 8 * st, (c / kStages) & 1, status, kSiteK, abort_flag))) return false;
                tc_fence_after();
                const uint32_t sK = sbase + L::kK0 + st * L::kStageBytes;
                const bool full = (2 * c + 1) < nseg;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * L::kTileBytes + (kk & 3) * 32;
                    mma_ss(tS0 + (c & 1) * 128, sdesc(sbase + L::kQ + off, 16, 1024), sdesc(sK + off, 16, 1024),
                           full ? idS128 : idS64, kk > 0);
                }
                mma_commit(bar_s + 8 * (c & 1));
                return true;
            };
            if (ok && nchunk > 0) ok = issue_s(0);
            for (int c = 0; ok && c < nchunk; ++c) {
                if (c + 1 < nchunk && !issue_s(c + 1)) break;
                const int st = c % kStages;
                if (!__all_sync(0xffffffffu, mbar_wait(bar_p + 8 * (c & 1), (c >> 1) & 1, status, kSiteP, abort_flag))) break;
                if (!__all_sync(0xffffffffu, mbar_wait(bar_v + 8 * st, (c / kStages) & 1, status, kSiteV, abort_flag))) break;
                tc_fence_after();
                const uint32_t sV = sbase + L::kK0 + st * L::kStageBytes + L::kHalves * L::kTileBytes;
                const int nk = ((2 * c + 1) < nseg) ? 128 : 64;
                for (int kk = 0; kk < nk / 16; ++kk)
                    mma_ts(tO, tS0 + (c & 1) * 128 + kk * 8, sdesc(sV + kk * 2048, L::kTileBytes, 1024), idPV,
                           (c > 0 || kk > 0) ? 1u : 0u);
                mma_commit(bar_e + 8 * st);
                mma_commit(bar_o);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int quad = warp & 3;
        const int rowid = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int c = 0; c < nchunk; ++c) {
            const int sb = c & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(bar_s + 8 * sb, (c >> 1) & 1, status, kSiteS, abort_flag));
            if (!ok) break;
            tc_fence_after();
            const bool full = (2 * c + 1) < nseg;
            const uint32_t tS = tS0 + sb * 128 + lane_off;
            uint32_t sr[4][32];
            tmem_ld32(tS, sr[0]);
            tmem_ld32(tS + 32, sr[1]);
            if (full) {
                tmem_ld32(tS + 64, sr[2]);
                tmem_ld32(tS + 96, sr[3]);
            }
            tmem_wait_ld();
            float mx = -INFINITY;
#pragma unroll
            for (int q = 0; q < 2; ++q)
#pragma unroll
                for (int e = 0; e < 32; ++e) mx = fmaxf(mx, __uint_as_float(sr[q][e]));
            if (full) {
#pragma unroll
                for (int q = 2; q < 4; ++q)
#pragma unroll
                    for (int e = 0; e < 32; ++e) mx = fmaxf(mx, __uint_as_float(sr[q][e]));
            }
            const float mx2 = mx * scale_log2;
            const bool need = (c > 0) && (mx2 > m + kRescaleThreshold);
            if (c == 0) m = mx2;
            // TMEM loads / stores are warp-collective: the whole warp rescales
            // when any of its rows needs it (a row whose max did not grow gets 1)
            if (__any_sync(0xffffffffu, need)) {
                // O must hold every earlier chunk before it is rescaled
                ok = __all_sync(0xffffffffu, mbar_wait(bar_o, (c - 1) & 1, status, kSiteO, abort_flag));
                if (!ok) break;
                tc_fence_after();
                const float mnew = fmaxf(m, mx2);
                const float corr = ex2(m - mnew);
#pragma unroll 1
                for (int q = 0; q < D / 32; ++q) {
                    uint32_t orr[32];
                    tmem_ld32(tO + lane_off + q * 32, orr);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * corr);
                    tmem_st32(tO + lane_off + q * 32, orr);
                }
                tmem_wait_st();
                l *= corr;
                m = mnew;
            }
            float sum = 0.f;
            uint32_t pk[2][32];
#pragma unroll
            for (int q = 0; q < 2; ++q)
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float p0 = ex2(fmaf(__uint_as_float(sr[q][2 * e]), scale_log2, -m));
                    const float p1 = ex2(fmaf(__uint_as_float(sr[q][2 * e + 1]), scale_log2, -m));
                    sum += p0 + p1;
                    pk[q >> 1][(q & 1) * 16 + e] = pack_bf16x2(p0, p1);
                }
            if (full) {
#pragma unroll
                for (int q = 2; q < 4; ++q)
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float p0 = ex2(fmaf(__uint_as_float(sr[q][2 * e]), scale_log2, -m));
                        const float p1 = ex2(fmaf(__uint_as_float(sr[q][2 * e + 1]), scale_log2, -m));
                        sum += p0 + p1;
                        pk[q >> 1][(q & 1) * 16 + e] = pack_bf16x2(p0, p1);
                    }
            }
            l += sum;
            tmem_st32(tS, pk[0]);
            if (full) tmem_st32(tS + 32, pk[1]);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_p + 8 * sb);
        }
        // epilogue: wait for the last two PV products, in phase order
        if (ok && nchunk > 0) {
            for (int ph = max(0, nchunk - 2); ph < nchunk && ok; ++ph)
                ok = __all_sync(0xffffffffu, mbar_wait(bar_o, ph & 1, status, kSiteO, abort_flag));
        }
        if (ok && nchunk > 0) {
            tc_fence_after();
            const float inv = 1.f / l;
            const int n = q0 + rowid;
            const bool write = rowid < qvalid;
            const int tok = write ? perm[(size_t)b * g.N + n] : 0;
            __nv_bfloat16 *dst = O + (((size_t)b * g.N + tok) * g.heads + h) * D;
#pragma unroll 1
            for (int q = 0; q < D / 32; ++q) {
                uint32_t orr[32];
                tmem_ld32(tO + lane_off + q * 32, orr);
                tmem_wait_ld();
                uint4 pkt[4];
                uint32_t *pw = reinterpret_cast<uint32_t *>(pkt);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pw[e] = pack_bf16x2(__uint_as_float(orr[2 * e]) * inv, __uint_as_float(orr[2 * e + 1]) * inv);
                if (write) {
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst + q * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e) d4[e] = pkt[e];
                }
            }
            if (write) {
                const float lse2 = m + __log2f(l);  // log2 units, as the backward consumes it
                lse_p[(size_t)bh * g.N + n] = lse2;
                if (lse_user) lse_user[(size_t)bh * g.N + tok] = lse2 * 0.69314718055994531f;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace fwdtc

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2D map over a [rows][cols] bf16 matrix, boxes of 64 rows x 64 columns
// (128 bytes, the 128-byte swizzle span).
static prism_status make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(PRISM_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PRISM_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return PRISM_OK;
}

// 2D map over a [rows][D] fp32 matrix, boxes of 64 rows x D columns, no
// swizzle (reduce-add target of the backward's dQ tiles).
static prism_status make_map_f32_rows(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(PRISM_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 4};
    cuuint32_t box[2] = {(cuuint32_t)cols, 64};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PRISM_ERR_CUDA, "cuTensorMapEncodeTiled (fp32) failed (%d)", (int)r);
    return PRISM_OK;
}

prism_status make_tensor_maps(Plan &pl) {
    const uint64_t rows = (uint64_t)pl.g.batch * pl.g.heads * pl.g.N;
    prism_status s = make_map(&pl.tmQ, pl.Qp, rows, pl.g.D);
    if (s == PRISM_OK) s = make_map(&pl.tmK, pl.Kp, rows, pl.g.D);
    if (s == PRISM_OK) s = make_map(&pl.tmV, pl.Vp, rows, pl.g.D);
    if (s == PRISM_OK) s = make_map(&pl.tmdO, pl.dOp, rows, pl.g.D);
    if (s == PRISM_OK) s = make_map_f32_rows(&pl.tmdQ, pl.dQacc, rows, pl.g.D);
    return s;
}

template <int D>
static prism_status fwd_tc_impl(Plan &pl, void *O, float *lse, cudaStream_t st) {
    const Geo &g = pl.g;
    const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    TimerScope ts(pl, kTAttnFwd, st);
    fwdtc::k_attn_fwd_tc<D><<<dim3(g.nbmax, g.batch * g.heads), fwdtc::kThreads, fwdtc::Layout<D>::kAlloc, st>>>(
        pl.tmQ, pl.tmK, pl.tmV, g, pl.nqt, pl.qt_row, pl.qt_blk, pl.blk_off, pl.row_ptr, pl.col, pl.perm,
        static_cast<__nv_bfloat16 *>(O), lse, pl.lse_p, scale_log2, pl.status);
    PRISM_CUDA_OK(cudaGetLastError());
    return PRISM_OK;
}

prism_status configure_attn_tc_kernels() {
    PRISM_CUDA_OK(cudaFuncSetAttribute(fwdtc::k_attn_fwd_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)fwdtc::Layout<64>::kAlloc));
    PRISM_CUDA_OK(cudaFuncSetAttribute(fwdtc::k_attn_fwd_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)fwdtc::Layout<128>::kAlloc));
    return PRISM_OK;
}

prism_status launch_attn_fwd_tc(Plan &pl, void *O, float *lse, cudaStream_t st) {
    return pl.g.D == 64 ? fwd_tc_impl<64>(pl, O, lse, st) : fwd_tc_impl<128>(pl, O, lse, st);
}

}  // namespace prism
