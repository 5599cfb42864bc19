// attn_bwd_tc.cu -- block-sparse attention backward on the tcgen05 tensor
// cores, key-stationary.
//
// Gradient of sum(O * dO) through softmax attention restricted to the
// selected block pairs [Prism guide, Method section 3; the backward is the
// standard softmax-attention gradient]:
//   P = exp(S*scale - LSE), dP = dO V^T, dS = P (dP - Delta),
//   dV = P^T dO, dK = scale dS^T Q, dQ = scale dS K.
//
// Work unit: one 128-key tile of one head (a 256-token key block gives two,
// a 128-token block one, and two consecutive 64-token blocks j, j+1 share
// one).  The CTA walks the query blocks of the key block's CSC column as
// 64-row chunks; a shared tile walks the union of its two columns, and the
// key rows of a block whose column lacks the chunk's query block (a whole
// warp's rows) take P = dS = 0 for that chunk.
//
// Per chunk c (b = c & 1):
//   S^T  = K Q_c^T         M=128 keys, N=64 queries   -> TMEM ST[b]
//   dP^T = V dO_c^T        M=128 keys, N=64 queries   -> TMEM DP[b]
//   softmax warps: P^T, dS^T (bf16, packed over their own ST[b] columns),
//                  dS^T also to shared memory DS[b]
//   dQ^T = K^T dS^T        both operands MN-major     -> TMEM DP[b] (dP^T is
//                                                        consumed by then)
//   dV  += P^T dO_c        A = P^T from TMEM          -> TMEM dV
//   dK  += dS^T Q_c        A = dS^T from TMEM         -> TMEM dK
//   drain warps: dQ^T rows (lane = head-dim index) -> a [64 x D] fp32 tile in
//                shared memory -> one TMA reduce-add into the dQ accumulator
// Two ST and two DP buffers: S^T and dP^T of chunk c+2 are issued behind
// chunk c's products, so the softmax of chunk c+1 (whose S^T and dP^T were
// issued a chunk earlier) runs while the tensor cores work on chunk c.  dQ^T
// is issued first among a chunk's products, so the drain reads it while dV,
// dK and S^T of c+2 run; dP^T of c+2 then reuses the buffer.
// TMEM columns: dK [0,128), dV [128,256), ST[2] [256,384), DP[2] [384,512).
// In an ST buffer, after the softmax, columns [16g, 16g+8) hold P^T and
// [16g+8, 16g+16) hold dS^T of queries [16g, 16g+16) (g = 0..3), packed as
// bf16 pairs.
//
// The softmax runs in two groups of 8 warps that take alternate chunks (even
// chunks, odd chunks), so one group's TMEM loads and stores overlap the other
// group's exponentials.  In a group each warp owns one TMEM lane quadrant (32
// key rows) and 32 query columns, taken as two 16-column halves, and does its
// arithmetic in packed fp32 pairs.  The group issues its own products: a
// named barrier closes the group's softmax of a chunk, and the group's first
// warp issues dQ^T, dV, dK of that chunk and S^T, dP^T of the chunk two ahead
// (no hand-off to a separate MMA warp).  The two groups' dV and dK products
// accumulate into the same TMEM columns: a token passed between the groups
// keeps them in chunk order (deterministic sums), and dK and dV start from zero
// (written by the drain warps before the first chunk), so no product needs to
// know whether it is the first.
// Warp roles (704 threads): warp 0 TMA producer (K, V once; Q, dO, LSE,
// Delta per chunk into a three-stage ring; LSE is kept negated, in log2
// units), warp 1 idle, warps 2..17 softmax and MMA issue, warps 18..21 dQ
// drain (one head-dim row each).
#include <cuda.h>

#include "tc_common.cuh"

namespace prism {

using namespace tc;

namespace bwdtc {

constexpr int kSoftmaxWarps = 16;
constexpr int kThreads = 32 * (2 + kSoftmaxWarps + 4);
constexpr int kStages = 3;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDK = 0, kColDV = 128, kColST = 256, kColDP = 384;  // ST[2], DP[2]: 64 columns each

template <int D>
struct Layout {
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static constexpr int kHalves = D / 64;          // 64-column (128 B) swizzle atoms along D
    static constexpr uint32_t kKVHalf = 128 * 128;  // 128 rows x 128 B
    static constexpr uint32_t kQHalf = 64 * 128;    // 64 rows x 128 B
    static constexpr uint32_t kK = 0;
    static constexpr uint32_t kV = kK + kHalves * kKVHalf;
    static constexpr uint32_t kQ0 = kV + kHalves * kKVHalf;  // stage s: Q at kQ0 + s*kStage, dO at + kHalves*kQHalf
    static constexpr uint32_t kStage = 2 * kHalves * kQHalf;
    static constexpr uint32_t kDS = kQ0 + kStages * kStage;  // [2] x 128 key rows x 128 B (64 queries bf16)
    static constexpr uint32_t kVec = kDS + 2 * 16384;        // stage s: -LSE [64] f32 then Delta [64] f32
    static constexpr uint32_t kDQ = kVec + kStages * 512;    // dQ staging tile [64 queries][D] f32 (128-B aligned)
    static constexpr uint32_t kBars = kDQ + 64 * D * 4;
    // kv, q_full[kStages], q_empty[kStages], s_full[2], dq_full[2], dq_empty[2], done, token
    static constexpr uint32_t kNumBars = 9 + 2 * kStages;
    // then per stage the column mask of its query chunk in a shared tile
    static constexpr uint32_t kMaskS = kBars + kNumBars * 8 + 16;
    static constexpr uint32_t kBytes = kMaskS + 16;
    static constexpr uint32_t kAlloc = kBytes + 1024;
    static_assert(kAlloc <= 232448, "shared memory per block");
    static_assert(kDQ % 128 == 0, "TMA source alignment");
};

// S^T / dP^T: contraction over the head dimension, A (K or V rows) and B (Q or
// dO rows) K-major, their 64-column halves kKVHalf and kQHalf bytes apart.
template <int D>
__device__ __forceinline__ void mma_over_d(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc) {
    if constexpr (D == 128)
        mma_ss8<2, 4, 6, 1024, 1026, 1028, 1030, 2, 4, 6, 512, 514, 516, 518>(d_tmem, adesc, bdesc, idesc, 0u);
    else
        mma_ss4<2, 4, 6, 2, 4, 6>(d_tmem, adesc, bdesc, idesc, 0u);
}

enum { kSiteKV = 11, kSiteQFull, kSiteQEmpty, kSiteS, kSiteDQFull = 16, kSiteDQEmpty, kSiteDone, kSiteToken };

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_bwd_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmdQ, Geo g,
                  const int *__restrict__ nqt, const int *__restrict__ qt_row, const int *__restrict__ qt_blk,
                  const int *__restrict__ blk_off, const int *__restrict__ colT_ptr, const int *__restrict__ rowT,
                  const int *__restrict__ perm, const float *__restrict__ nlse_p, const float *__restrict__ delta,
                  float *__restrict__ dQacc, __nv_bfloat16 *__restrict__ dK, __nv_bfloat16 *__restrict__ dV,
                  float scale, float scale_log2, int *__restrict__ status) {
    using L = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t sbase = smem_u32(smem);

    const int tile = blockIdx.x, bh = blockIdx.y, b = bh / g.heads, h = bh % g.heads;
    if (tile >= nqt[b]) return;
    if (*reinterpret_cast<volatile int *>(status) != 0) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int *bo = blk_off + (size_t)b * (g.nbmax + 1);
    const int k0 = qt_row[(size_t)b * g.nbmax + tile];
    int jblk, jblk2;
    tile_blocks(qt_blk[(size_t)b * g.nbmax + tile], jblk, jblk2);
    const bool shared_tile = jblk2 >= 0;
    const int kvalid = min(128, bo[(shared_tile ? jblk2 : jblk) + 1] - k0);
    const size_t colid = (size_t)bh * g.nbmax + jblk;
    const int u_begin = colT_ptr[colid], u_end = colT_ptr[colid + 1];
    // the second key block's column (empty unless the tile is shared)
    const int u2_begin = shared_tile ? colT_ptr[colid + 1] : 0, u2_end = shared_tile ? colT_ptr[colid + 2] : 0;

    // 64-row query chunks of the column(s)
    const int nchunk = union_segments(rowT + u_begin, u_end - u_begin, rowT + u2_begin, u2_end - u2_begin, bo, lane);

    const uint32_t bar_kv = sbase + L::kBars;
    const uint32_t bar_qf = bar_kv + 8, bar_qe = bar_qf + 8 * kStages, bar_sf = bar_qe + 8 * kStages;
    const uint32_t bar_df = bar_sf + 16, bar_de = bar_df + 16;
    const uint32_t bar_done = bar_de + 16;
    const uint32_t bar_tok = bar_done + 8;  // dV, dK of a chunk have been issued
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kBars + L::kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kBars + L::kNumBars * 8 + 8);
    volatile int *drain_fail = abort_flag + 1;  // a drain warp's wait failed
    volatile uint32_t *mask_s = reinterpret_cast<volatile uint32_t *>(smem + L::kMaskS);

    if (warp == 0) {
        if (lane == 0) {
            mbar_init(bar_kv, 1);
            for (int s = 0; s < kStages; ++s) {
                mbar_init(bar_qf + 8 * s, 1);
                mbar_init(bar_qe + 8 * s, 1);
            }
            for (int s = 0; s < 2; ++s) {
                mbar_init(bar_sf + 8 * s, 1);
                mbar_init(bar_df + 8 * s, 1);
                mbar_init(bar_de + 8 * s, 128);
            }
            mbar_init(bar_done, 2);
            mbar_init(bar_tok, 1);
            *abort_flag = 0;
            *drain_fail = 0;
            mbar_fence_init();
            prefetch_map(&tmQ);
            prefetch_map(&tmK);
            prefetch_map(&tmV);
            prefetch_map(&tmdO);
            prefetch_map(&tmdQ);
        }
        __syncwarp();
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int rowbase = bh * g.N;
    if (warp >= 2 + kSoftmaxWarps) {  // dK, dV start from zero: both groups' products accumulate
        const uint32_t lo = (uint32_t)((warp & 3) * 32) << 16;
        uint32_t z[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) z[e] = 0u;
#pragma unroll 1
        for (int q = 0; q < 16; ++q) tmem_st16(tmem + kColDK + q * 16 + lo, z);
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_expect_tx(bar_kv, 2 * 128 * D * 2);
            for (int hf = 0; hf < L::kHalves; ++hf)
                for (int rh = 0; rh < 2; ++rh) {
                    tma_load_2d(sbase + L::kK + hf * L::kKVHalf + rh * 8192, &tmK, bar_kv, hf * 64,
                                rowbase + k0 + rh * 64);
                    tma_load_2d(sbase + L::kV + hf * L::kKVHalf + rh * 8192, &tmV, bar_kv, hf * 64,
                                rowbase + k0 + rh * 64);
                }
            SegWalk wk;
            wk.init(u_begin, u_end, u2_begin, u2_end, rowT, bo);
            int issued = 0;
            for (int c = 0; c < nchunk; ++c) {
                const int st = c % kStages;
                if (c >= kStages &&
                    !mbar_wait(bar_qe + 8 * st, ((c / kStages) + 1) & 1, status, kSiteQEmpty, abort_flag))
                    break;
                const uint32_t sQ = sbase + L::kQ0 + st * L::kStage, sO = sQ + L::kHalves * L::kQHalf;
                const uint32_t sVec = sbase + L::kVec + st * 512;
                const uint32_t bar = bar_qf + 8 * st;
                const int r = wk.r;
                mask_s[st] = (uint32_t)wk.mask;  // published by the arrive below
                mbar_expect_tx(bar, 2 * 64 * D * 2 + 512);
                for (int hf = 0; hf < L::kHalves; ++hf) {
                    tma_load_2d(sQ + hf * L::kQHalf, &tmQ, bar, hf * 64, rowbase + r);
                    tma_load_2d(sO + hf * L::kQHalf, &tmdO, bar, hf * 64, rowbase + r);
                }
                bulk_load(sVec, nlse_p + (size_t)rowbase + r, 256, bar);
                bulk_load(sVec + 256, delta + (size_t)rowbase + r, 256, bar);
                issued = c + 1;
                wk.advance(rowT, bo);
            }
            for (int c = max(0, issued - kStages); c < issued; ++c)
                mbar_wait(bar_qf + 8 * (c % kStages), (c / kStages) & 1, status, kSiteQFull, abort_flag);
            mbar_wait(bar_kv, 0, status, kSiteKV, abort_flag);
        }
    } else if (warp == 1) {
        // no role: the softmax groups issue their own products
    } else if (warp < 2 + kSoftmaxWarps) {
        // ------------------------------------------------------------ softmax (key rows)
        const int quad = warp & 3;               // TMEM lane quadrant this warp may access
        const int grp = (warp - 2) >> 3;         // the chunks of this parity
        const int cg2 = ((warp - 2) >> 2) & 1;   // its 32 query columns [32 cg2, 32 cg2 + 32)
        const int cg = (warp - 2) >> 2;          // epilogue column group
        const int rowid = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const bool live = rowid < kvalid;
        const int half = shared_tile ? (quad >> 1) : 0;  // which key block's rows (warp-uniform)
        bool ok = true;
        const bool issuer = ((warp - 2) & 7) == 0;  // the group's first warp issues its products
        constexpr uint32_t idST = idesc_bf16(128, 64, false);
        constexpr uint32_t idAcc = idesc_bf16(128, D, true);
        constexpr uint32_t idDQ = idesc_bf16(128, 64, true, true);
        // S^T and dP^T of chunk c into ST[c & 1] and DP[c & 1]; dP^T waits for the
        // drain of chunk c - 2 to have read its dQ^T out of DP[c & 1]
        auto issue_sdp = [&](int c) -> bool {
            const int st = c % kStages;
            if (!__all_sync(0xffffffffu, mbar_wait(bar_qf + 8 * st, (c / kStages) & 1, status, kSiteQFull, abort_flag))) return false;
            tc_fence_after();
            const uint32_t sQ = sbase + L::kQ0 + st * L::kStage, sO = sQ + L::kHalves * L::kQHalf;
            mma_over_d<D>(tmem + kColST + (c & 1) * 64, sdesc(sbase + L::kK, 16, 1024), sdesc(sQ, 16, 1024), idST);
            if (c >= 2 && !__all_sync(0xffffffffu, mbar_wait(bar_de + 8 * (c & 1), ((c - 2) >> 1) & 1, status,
                                                             kSiteDQEmpty, abort_flag)))
                return false;
            tc_fence_after();
            mma_over_d<D>(tmem + kColDP + (c & 1) * 64, sdesc(sbase + L::kV, 16, 1024), sdesc(sO, 16, 1024), idST);
            mma_commit(bar_sf + 8 * (c & 1));
            return true;
        };
        if (issuer && grp < nchunk) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar_kv, 0, status, kSiteKV, abort_flag));
            if (ok) ok = issue_sdp(grp);
        }
        // every warp of the group passes exactly one named barrier per chunk, on
        // every path, so a failed wait cannot leave the others blocked
        for (int c = grp; c < nchunk; c += 2) {
            const int st = c % kStages;
            if (ok)
                ok = __all_sync(0xffffffffu, mbar_wait(bar_sf + 8 * (c & 1), (c >> 1) & 1, status, kSiteS, abort_flag) &&
                                                 mbar_wait(bar_qf + 8 * st, (c / kStages) & 1, status, kSiteQFull,
                                                           abort_flag));
            if (ok) {
                tc_fence_after();
                const bool act = live && ((mask_s[st] >> half) & 1u);
                const uint32_t dsrow = sbase + L::kDS + (c & 1) * 16384 + rowid * 128;
#pragma unroll 1
                for (int sub = 0; sub < 2; ++sub) {
                    const int cq = 2 * cg2 + sub;  // 16 query columns [16 cq, 16 cq + 16)
                    const uint32_t tST = tmem + kColST + (c & 1) * 64 + 16 * cq + lane_off;
                    uint32_t sv[16], dv[16];
                    tmem_ld16(tST, sv);
                    tmem_ld16(tmem + kColDP + (c & 1) * 64 + 16 * cq + lane_off, dv);
                    const uint32_t vec = sbase + L::kVec + st * 512 + cq * 64;
                    float4 N4[4], D4[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        N4[j] = lds_f4(vec + 16 * j);
                        D4[j] = lds_f4(vec + 256 + 16 * j);
                    }
                    tmem_wait_ld();
                    uint32_t pd[16];
                    if (act) {
                        const uint64_t s2 = splat2(scale_log2);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int q = 4 * j;
                            float x0, x1, x2, x3, d0, d1, d2, d3;
                            fma2(__uint_as_float(sv[q]), __uint_as_float(sv[q + 1]), s2, pair2(N4[j].x, N4[j].y), x0, x1);
                            fma2(__uint_as_float(sv[q + 2]), __uint_as_float(sv[q + 3]), s2, pair2(N4[j].z, N4[j].w), x2, x3);
                            const float p0 = ex2(x0), p1 = ex2(x1), p2 = ex2(x2), p3 = ex2(x3);
                            mul_sub2(p0, p1, __uint_as_float(dv[q]), __uint_as_float(dv[q + 1]), D4[j].x, D4[j].y, d0, d1);
                            mul_sub2(p2, p3, __uint_as_float(dv[q + 2]), __uint_as_float(dv[q + 3]), D4[j].z, D4[j].w, d2, d3);
                            pd[2 * j] = pack_bf16x2(p0, p1);
                            pd[2 * j + 1] = pack_bf16x2(p2, p3);
                            pd[8 + 2 * j] = pack_bf16x2(d0, d1);
                            pd[8 + 2 * j + 1] = pack_bf16x2(d2, d3);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) pd[e] = 0u;
                    }
                    tmem_st16(tST, pd);
                    sts_u4(dsrow + (((2 * cq) ^ (rowid & 7)) << 4), pd[8], pd[9], pd[10], pd[11]);
                    sts_u4(dsrow + (((2 * cq + 1) ^ (rowid & 7)) << 4), pd[12], pd[13], pd[14], pd[15]);
                }
                tmem_wait_st();
                fence_async_smem();
            }
            tc_fence_before();
            named_bar_sync(2 + grp, 32 * kSoftmaxWarps / 2);
            if (issuer && ok && !*abort_flag) {
                tc_fence_after();
                const uint32_t sQ = sbase + L::kQ0 + st * L::kStage, sO = sQ + L::kHalves * L::kQHalf;
                const uint32_t tSTc = tmem + kColST + (c & 1) * 64;
                const uint32_t sDS = sbase + L::kDS + (c & 1) * 16384;
                mma_ss8<128, 256, 384, 512, 640, 768, 896, 128, 256, 384, 512, 640, 768, 896>(
                    tmem + kColDP + (c & 1) * 64, sdesc(sbase + L::kK, L::kKVHalf, 1024), sdesc(sDS, 8192, 1024), idDQ,
                    0u);
                mma_commit(bar_df + 8 * (c & 1));
                // dV, dK in chunk order (the other group has issued those of chunk c - 1),
                // so that their fp32 sums do not depend on the two groups' timing
                if (c >= 1)
                    ok = __all_sync(0xffffffffu, mbar_wait(bar_tok, (c - 1) & 1, status, kSiteToken, abort_flag));
                if (ok) {
                    tc_fence_after();
                    mma_ts4x2<16, 32, 48, 128, 256, 384>(tmem + kColDV, tSTc, sdesc(sO, L::kQHalf, 1024),
                                                          tmem + kColDK, tSTc + 8, sdesc(sQ, L::kQHalf, 1024), idAcc, 1u);
                    tc_fence_before();
                    if (lane == 0) mbar_arrive(bar_tok);
                    __syncwarp();
                    mma_commit(bar_qe + 8 * st);
                    if (c + 2 < nchunk) ok = issue_sdp(c + 2);
                }
            }
        }
        if (issuer) mma_commit(bar_done);  // both groups' products: done counts two commits
        // epilogue: column groups 0, 1 write halves of dK (scaled), 2, 3 halves of dV
        if (ok && nchunk > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_done, 0, status, kSiteDone, abort_flag));
        if (ok) {
            tc_fence_after();
            const int tok = live ? perm[(size_t)b * g.N + k0 + rowid] : 0;
            const int c0 = (cg & 1) * (D / 2);
            __nv_bfloat16 *dst = (cg < 2 ? dK : dV) + (((size_t)b * g.N + tok) * g.heads + h) * D + c0;
            const uint32_t src = tmem + (cg < 2 ? kColDK : kColDV) + c0 + lane_off;
            const float f = (cg < 2) ? scale : 1.0f;
#pragma unroll 1
            for (int q = 0; q < D / 64; ++q) {
                uint32_t a[32];
                if (nchunk > 0) {
                    tmem_ld32(src + q * 32, a);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) a[e] = 0u;
                }
                uint4 pa[4];
                uint32_t *wa = reinterpret_cast<uint32_t *>(pa);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    wa[e] = pack_bf16x2(__uint_as_float(a[2 * e]) * f, __uint_as_float(a[2 * e + 1]) * f);
                if (live) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) reinterpret_cast<uint4 *>(dst + q * 32)[e] = pa[e];
                }
            }
        }
    } else {
        // ------------------------------------------------------------ dQ drain (head-dim rows)
        const int quad = warp & 3;
        const int d = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const bool leader = (warp == 2 + kSoftmaxWarps && lane == 0);
        SegWalk wk;
        wk.init(u_begin, u_end, u2_begin, u2_end, rowT, bo);
        for (int c = 0; c < nchunk; ++c) {
            if (!__all_sync(0xffffffffu,
                            mbar_wait(bar_df + 8 * (c & 1), (c >> 1) & 1, status, kSiteDQFull, abort_flag))) {
                // meet the other drain warps at this chunk's first barrier and leave with them
                if (lane == 0) *drain_fail = 1;
                named_bar_sync(1, 128);
                break;
            }
            tc_fence_after();
            uint32_t v[32], w[32];
            tmem_ld32(tmem + kColDP + (c & 1) * 64 + lane_off, v);
            tmem_ld32(tmem + kColDP + (c & 1) * 64 + lane_off + 32, w);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(bar_de + 8 * (c & 1));
            // the staging tile is free once the previous reduce has read it
            if (leader) bulk_wait_read_all();
            named_bar_sync(1, 128);
            // the same answer in every drain warp: they write the flag only before this barrier
            if (*drain_fail) break;
            const uint32_t stage = sbase + L::kDQ + d * 4;
            if (d < D) {  // head_dim 64: dQ^T rows 64..127 are padding
#pragma unroll
                for (int q = 0; q < 32; ++q) sts_f32(stage + q * D * 4, __uint_as_float(v[q]) * scale);
#pragma unroll
                for (int q = 0; q < 32; ++q) sts_f32(stage + (q + 32) * D * 4, __uint_as_float(w[q]) * scale);
            }
            fence_async_smem();
            named_bar_sync(1, 128);
            if (leader) {
                tma_reduce_add_2d(&tmdQ, sbase + L::kDQ, 0, rowbase + wk.r);
                bulk_commit();
            }
            wk.advance(rowT, bo);
        }
        if (leader) bulk_wait_all();  // every reduce has landed before the CTA exits
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace bwdtc

prism_status configure_attn_bwd_tc_kernels() {
    PRISM_CUDA_OK(cudaFuncSetAttribute(bwdtc::k_attn_bwd_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bwdtc::Layout<64>::kAlloc));
    PRISM_CUDA_OK(cudaFuncSetAttribute(bwdtc::k_attn_bwd_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bwdtc::Layout<128>::kAlloc));
    return PRISM_OK;
}

// Runs the tensor-core key-stationary backward; the caller has zeroed dQacc
// and written dOp and delta.
template <int D>
static prism_status bwd_tc_main(Plan &pl, void *dK, void *dV, cudaStream_t st) {
    const Geo &g = pl.g;
    const double scale = 1.0 / sqrt((double)D);
    TimerScope ts(pl, kTAttnBwd, st);
    bwdtc::k_attn_bwd_tc<D><<<dim3(g.nbmax, g.batch * g.heads), bwdtc::kThreads, bwdtc::Layout<D>::kAlloc, st>>>(
        pl.tmQ, pl.tmK, pl.tmV, pl.tmdO, pl.tmdQ, g, pl.nqt, pl.qt_row, pl.qt_blk, pl.blk_off, pl.colT_ptr, pl.rowT,
        pl.perm, pl.nlse_p, pl.delta, pl.dQacc, static_cast<__nv_bfloat16 *>(dK), static_cast<__nv_bfloat16 *>(dV),
        (float)scale, (float)(scale * 1.4426950408889634), pl.status);
    PRISM_CUDA_OK(cudaGetLastError());
    return PRISM_OK;
}

prism_status launch_attn_bwd_tc_main(Plan &pl, void *dK, void *dV, cudaStream_t st) {
    return pl.g.D == 64 ? bwd_tc_main<64>(pl, dK, dV, st) : bwd_tc_main<128>(pl, dK, dV, st);
}

}  // namespace prism
