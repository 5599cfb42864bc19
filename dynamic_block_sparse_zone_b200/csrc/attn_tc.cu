// attn_tc.cu -- block-sparse attention forward on the 5th-generation tensor
// cores (tcgen05, TMEM accumulators, TMA tile loads).
//
// [Prism guide, Method section 3, last sentence]: each query block attends,
// under one online softmax, to the tokens of the key blocks in S_i.
//
// Work unit: one 128-row query tile of one head (a 256-token block gives two
// tiles, a 128-token block one, and two consecutive 64-token blocks i, i+1
// share one).  The selected key blocks are streamed as 64-row segments; two
// segments form a 128-key chunk.  A shared tile streams S_i U S_{i+1}: the
// producer writes, per chunk, which of the two sets each segment belongs to,
// and each row half (whole softmax warps) gives the segments outside its own
// set P = 0.
//
// Two CTAs share an SM (96 KB of shared memory and 256 TMEM columns each), so
// while one CTA's softmax works the tensor cores run the other CTA's MMAs;
// inside a CTA the chunk pipeline is strictly ordered:
//   S_c = Q K_c^T (TMEM S) -> softmax (P_c over S, bf16) -> O += P_c V_c -> S_{c+1}
// Warp roles (192 threads):
//   warp 0       TMA producer: Q once; K_c into the K buffer once S_{c-1} has
//                read it, V_c into the V buffer once P_{c-1} V_{c-1} has.
//   warp 1       MMA issuer (whole warp, one elected lane issues).
//   warps 2..5   softmax, one query row per thread (= TMEM lane): the S row
//                comes into registers in one TMEM round trip; pass 1 row
//                max, pass 2 exp2 / running sum / bf16 P written back over S;
//                P of the first 64 keys is published as soon as it is stored,
//                so the first half of P V overlaps the rest of the softmax.
//                O is rescaled in TMEM only when the running max grows by more
//                than 2^8 (it is current then: S_c was issued after PV_{c-1}).
//                Epilogue: O / l to the user layout, log-sum-exp.
// TMEM columns: S / P [0,128), O [128, 128+D).
//
// Taylor variant (kTaylor) [In-Context Sparse Attention article, grouped
// computation: the flat path scores block-mean keys and keeps the zeroth-order
// term of the exponential]: after the selected blocks, the same pipeline
// streams the head's pooled keys kbar_j and mean values vbar_j (bf16, 128 per
// chunk).  Block j then adds |B_j| exp2(x) with x its scaled pooled score: its
// softmax column gets the bias log2 |B_j|, or -inf when j is in S_i (those
// blocks are already exact) or past the last block.  The CTA first tabulates
// log2 |B_j| of every key block in shared memory (one byte each, -1 for the
// blocks of S_i); each softmax warp then turns a chunk's 128 entries into
// float biases in its own buffer.  One online softmax covers both parts.
#include <cuda.h>

#include "tc_common.cuh"

namespace prism {

using namespace tc;

namespace fwdtc {

constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct Layout {
    static constexpr int kHalves = D / 64;               // 64-column (128 B) swizzle atoms along D
    static constexpr uint32_t kTileBytes = 128 * 128;    // 128 rows x 128 B
    static constexpr uint32_t kQ = 0;
    static constexpr uint32_t kK = kQ + kHalves * kTileBytes;
    static constexpr uint32_t kV = kK + kHalves * kTileBytes;
    static constexpr uint32_t kBars = kV + kHalves * kTileBytes;
    // barriers: q, k_full, k_empty, v_full, v_empty, s, p, o, p2, mask[2]  (8 B each)
    // + tmem slot + abort, then the two segment-mask words of a shared tile
    static constexpr uint32_t kNumBars = 11;
    static constexpr uint32_t kMaskW = kBars + kNumBars * 8 + 16;
    static constexpr uint32_t kBytes = kMaskW + 8;
    static constexpr uint32_t kAlloc = kBytes + 1024;  // slack to align the base to 1024
    // Taylor variant: per-softmax-warp bias of a chunk, then two log2 |B_j|
    // tables (int8, -1 for the blocks of S_i; the second for the second block
    // of a shared tile)
    static constexpr uint32_t kBias = (kBytes + 15) & ~15u;
    static constexpr uint32_t kLg = kBias + 4 * 128 * 4;
    __host__ __device__ static uint32_t lg_stride(int nbmax) { return (nbmax + 15) & ~15u; }
    static uint32_t taylor_alloc(int nbmax) { return kLg + 2 * lg_stride(nbmax) + 1024; }
};

// Site codes recorded with a timeout.
enum { kSiteQ = 1, kSiteK, kSiteV, kSiteKEmpty, kSiteVEmpty, kSiteS, kSiteP, kSiteO, kSiteMask };

template <int D, bool kTaylor>
__global__ void __launch_bounds__(kThreads, 2)
    k_attn_fwd_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
                  const __grid_constant__ CUtensorMap tmVb, const int *__restrict__ nbv, Geo g,
                  const int *__restrict__ nqt,
                  const int *__restrict__ qt_row, const int *__restrict__ qt_blk, const int *__restrict__ blk_off,
                  const int *__restrict__ row_ptr, const int *__restrict__ col, const int *__restrict__ perm,
                  __nv_bfloat16 *__restrict__ O, float *__restrict__ lse_user, float *__restrict__ nlse_p,
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
    int iblk, iblk2;
    tile_blocks(qt_blk[(size_t)b * g.nbmax + tile], iblk, iblk2);
    const bool shared_tile = iblk2 >= 0;
    const int qvalid = min(128, bo[(shared_tile ? iblk2 : iblk) + 1] - q0);
    const size_t crow = (size_t)bh * g.nbmax + iblk;
    const int c_begin = row_ptr[crow], c_end = row_ptr[crow + 1];
    // the second query block's selection (empty unless the tile is shared)
    const int c2_begin = shared_tile ? row_ptr[crow + 1] : 0, c2_end = shared_tile ? row_ptr[crow + 2] : 0;

    // number of 64-row key segments of the selection (every warp computes it)
    const int nseg = union_segments(col + c_begin, c_end - c_begin, col + c2_begin, c2_end - c2_begin, bo, lane);
    const int nchunk = (nseg + 1) >> 1;
    // Taylor variant: pooled chunks follow the selected ones
    const int nbb = kTaylor ? nbv[b] : 0;
    const int nseg_t = (nbb + 63) >> 6;
    const int nchunk_all = nchunk + ((nseg_t + 1) >> 1);
    auto chunk_full = [&](int c) { return c < nchunk ? (2 * c + 1) < nseg : (2 * (c - nchunk) + 1) < nseg_t; };
    int8_t *lg = reinterpret_cast<int8_t *>(smem + L::kLg);
    const uint32_t lgs = L::lg_stride(g.nbmax);
    if constexpr (kTaylor)  // block volumes are powers of two: log2 |B_j| is exact
        for (int j = threadIdx.x; j < nbb; j += kThreads) {
            const int8_t v = (int8_t)(31 - __clz(bo[j + 1] - bo[j]));
            lg[j] = v;
            lg[lgs + j] = v;
        }

    const uint32_t bar_q = sbase + L::kBars;
    const uint32_t bar_kf = bar_q + 8, bar_ke = bar_q + 16, bar_vf = bar_q + 24, bar_ve = bar_q + 32;
    const uint32_t bar_s = bar_q + 40, bar_p = bar_q + 48, bar_o = bar_q + 56;
    const uint32_t bar_p2 = bar_q + 64;  // P of keys 64..127 (bar_p: keys 0..63)
    const uint32_t bar_mk = bar_q + 72;  // [2]: the mask word of chunk c is in slot c & 1
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kBars + L::kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kBars + L::kNumBars * 8 + 8);
    volatile uint32_t *mask_w = reinterpret_cast<volatile uint32_t *>(smem + L::kMaskW);

    if (warp == 0) {
        if (lane == 0) {
            mbar_init(bar_q, 1);
            mbar_init(bar_kf, 1);
            mbar_init(bar_ke, 1);
            mbar_init(bar_vf, 1);
            mbar_init(bar_ve, 1);
            mbar_init(bar_s, 1);
            mbar_init(bar_p, 128);
            mbar_init(bar_p2, 128);
            mbar_init(bar_o, 1);
            mbar_init(bar_mk, 1);
            mbar_init(bar_mk + 8, 1);
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
    if constexpr (kTaylor) {  // the blocks of S_i are exact: no pooled term
        for (int u = c_begin + threadIdx.x; u < c_end; u += kThreads) lg[col[u]] = -1;
        for (int u = c2_begin + threadIdx.x; u < c2_end; u += kThreads) lg[lgs + col[u]] = -1;
        __syncthreads();
    }
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tO = tmem + 128;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const int rowbase = bh * g.N;
            mbar_expect_tx(bar_q, 128 * D * 2);
            for (int hf = 0; hf < L::kHalves; ++hf)
                for (int rh = 0; rh < 2; ++rh)
                    tma_load_2d(sbase + L::kQ + hf * L::kTileBytes + rh * 8192, &tmQ, bar_q, hf * 64,
                                rowbase + q0 + rh * 64);
            SegWalk wk;
            wk.init(c_begin, c_end, c2_begin, c2_end, col, bo);
            int kissued = 0, vissued = 0;
            for (int c = 0; c < nchunk_all; ++c) {
                const bool pooled = kTaylor && c >= nchunk;
                const int nsg = pooled ? min(2, nseg_t - 2 * (c - nchunk)) : min(2, nseg - 2 * c);
                const uint32_t bytes = nsg * 64 * D * 2;
                const CUtensorMap *mK = pooled ? &tmKb : &tmK, *mV = pooled ? &tmVb : &tmV;
                int rows[2];
                uint32_t segmask = 0;  // bits 2s, 2s+1: segment s in S_i, in S_{i+1}
                if (pooled) {  // rows of the pooled [batch*heads][nbmax][D] copies
                    for (int gsg = 0; gsg < nsg; ++gsg) rows[gsg] = bh * g.nbmax + 128 * (c - nchunk) + 64 * gsg;
                } else {
                    for (int gsg = 0; gsg < nsg; ++gsg) {
                        rows[gsg] = rowbase + wk.r;
                        segmask |= (uint32_t)wk.mask << (2 * gsg);
                        wk.advance(col, bo);
                    }
                }
                // K_c once S_{c-1} has consumed the K buffer
                if (c > 0 && !mbar_wait(bar_ke, (c - 1) & 1, status, kSiteKEmpty, abort_flag)) break;
                if (shared_tile && !pooled) {  // the softmax has read this slot for chunk c - 2
                    mask_w[c & 1] = segmask;
                    mbar_arrive(bar_mk + 8 * (c & 1));
                }
                mbar_expect_tx(bar_kf, bytes);
                for (int gsg = 0; gsg < nsg; ++gsg)
                    for (int hf = 0; hf < L::kHalves; ++hf)
                        tma_load_2d(sbase + L::kK + hf * L::kTileBytes + gsg * 8192, mK, bar_kf, hf * 64,
                                    rows[gsg]);
                kissued = c + 1;
                // V_c once P_{c-1} V_{c-1} has consumed the V buffer
                if (c > 0 && !mbar_wait(bar_ve, (c - 1) & 1, status, kSiteVEmpty, abort_flag)) break;
                mbar_expect_tx(bar_vf, bytes);
                for (int gsg = 0; gsg < nsg; ++gsg)
                    for (int hf = 0; hf < L::kHalves; ++hf)
                        tma_load_2d(sbase + L::kV + hf * L::kTileBytes + gsg * 8192, mV, bar_vf, hf * 64,
                                    rows[gsg]);
                vissued = c + 1;
            }
            // drain: every issued load must land before the CTA may exit
            if (kissued > 0) mbar_wait(bar_kf, (kissued - 1) & 1, status, kSiteK, abort_flag);
            if (vissued > 0) mbar_wait(bar_vf, (vissued - 1) & 1, status, kSiteV, abort_flag);
            mbar_wait(bar_q, 0, status, kSiteQ, abort_flag);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        {  // the whole warp runs the issue loop; elect.sync picks one lane
            constexpr uint32_t idS128 = idesc_bf16(128, 128, false), idS64 = idesc_bf16(128, 64, false);
            constexpr uint32_t idPV = idesc_bf16(128, D, true);
            bool ok = __all_sync(0xffffffffu, mbar_wait(bar_q, 0, status, kSiteQ, abort_flag));
            for (int c = 0; ok && c < nchunk_all; ++c) {
                const bool full = chunk_full(c);
                if (!__all_sync(0xffffffffu, mbar_wait(bar_kf, c & 1, status, kSiteK, abort_flag))) break;
                tc_fence_after();
                // k-step kk: 32 B along a 128-B row, the second 64 columns a tile further
                const uint64_t aQ = sdesc(sbase + L::kQ, 16, 1024), bK = sdesc(sbase + L::kK, 16, 1024);
                if constexpr (D == 128)
                    mma_ss8<2, 4, 6, 1024, 1026, 1028, 1030, 2, 4, 6, 1024, 1026, 1028, 1030>(
                        tS, aQ, bK, full ? idS128 : idS64, 0u);
                else
                    mma_ss4<2, 4, 6, 2, 4, 6>(tS, aQ, bK, full ? idS128 : idS64, 0u);
                mma_commit(bar_s);
                mma_commit(bar_ke);
                // P V in two halves: keys 0..63 as soon as the softmax has stored their P
                // (it goes on with keys 64..127 meanwhile), then keys 64..127
                if (!__all_sync(0xffffffffu, mbar_wait(bar_p, c & 1, status, kSiteP, abort_flag))) break;
                if (!__all_sync(0xffffffffu, mbar_wait(bar_vf, c & 1, status, kSiteV, abort_flag))) break;
                tc_fence_after();
                // k-step kk (16 keys): P columns 8 kk, V rows 2048 B (128 descriptor units) further
                const uint64_t bV = sdesc(sbase + L::kV, L::kTileBytes, 1024);
                mma_ts4<8, 16, 24, 128, 256, 384>(tO, tS, bV, idPV, c > 0);
                if (!__all_sync(0xffffffffu, mbar_wait(bar_p2, c & 1, status, kSiteP, abort_flag))) break;
                tc_fence_after();
                if (full) mma_ts4<8, 16, 24, 128, 256, 384>(tO, tS + 32, bV + 512, idPV, 1u);
                mma_commit(bar_ve);
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
        const uint32_t bias_s = sbase + L::kBias + quad * 512;  // this warp's 128 column biases
        const int half = shared_tile ? (quad >> 1) : 0;        // which query block's rows (warp-uniform)
        const int8_t *lgh = lg + half * lgs;
        for (int c = 0; c < nchunk_all; ++c) {
            const bool pooled = kTaylor && c >= nchunk;
            // segments of this chunk outside this half's selection get P = 0
            bool live0 = true, live1 = true;
            if (shared_tile && !pooled) {
                ok = __all_sync(0xffffffffu, mbar_wait(bar_mk + 8 * (c & 1), (c >> 1) & 1, status, kSiteMask, abort_flag));
                if (!ok) break;
                const uint32_t mw = mask_w[c & 1];
                live0 = (mw >> half) & 1u;
                live1 = (mw >> (2 + half)) & 1u;
            }
            if (pooled) {  // biases of this chunk's pooled keys, before S lands
                float *bias = reinterpret_cast<float *>(smem + L::kBias + quad * 512);
                __syncwarp();  // the warp has read the previous chunk's biases
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = 128 * (c - nchunk) + 32 * e + lane;
                    const int v = j < nbb ? lgh[j] : -1;
                    bias[32 * e + lane] = v < 0 ? -INFINITY : (float)v;
                }
                __syncwarp();
            }
            ok = __all_sync(0xffffffffu, mbar_wait(bar_s, c & 1, status, kSiteS, abort_flag));
            if (!ok) break;
            tc_fence_after();
            const int nq = chunk_full(c) ? 4 : 2;  // 32-column groups of S in this chunk
            const uint32_t tSr = tS + lane_off;
            // the whole S row into registers: one TMEM round trip for both passes
            uint32_t sr[128];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (q < nq) tmem_ld32(tSr + q * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * q]));
            tmem_wait_ld();
            // pass 1: row max (three-input max, four independent chains).  Pooled
            // chunks first turn S into x = S*scale*log2e + bias in place.
            float mxa = -INFINITY, mxb = -INFINITY, mxc = -INFINITY, mxd = -INFINITY;
            if (pooled) {
                const uint64_t s2 = splat2(scale_log2);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (q < nq) {
#pragma unroll
                        for (int e = 0; e < 32; e += 4) {
                            const float4 bb = lds_f4(bias_s + (32 * q + e) * 4);
                            float x0, x1, x2, x3;
                            fma2(__uint_as_float(sr[32 * q + e]), __uint_as_float(sr[32 * q + e + 1]), s2,
                                 pair2(bb.x, bb.y), x0, x1);
                            fma2(__uint_as_float(sr[32 * q + e + 2]), __uint_as_float(sr[32 * q + e + 3]), s2,
                                 pair2(bb.z, bb.w), x2, x3);
                            sr[32 * q + e] = __float_as_uint(x0);
                            sr[32 * q + e + 1] = __float_as_uint(x1);
                            sr[32 * q + e + 2] = __float_as_uint(x2);
                            sr[32 * q + e + 3] = __float_as_uint(x3);
                            if (e & 4) {
                                mxc = fmax3(mxc, x0, x1);
                                mxd = fmax3(mxd, x2, x3);
                            } else {
                                mxa = fmax3(mxa, x0, x1);
                                mxb = fmax3(mxb, x2, x3);
                            }
                        }
                    }
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (q < nq && (q < 2 ? live0 : live1)) {
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            const float *v = reinterpret_cast<const float *>(&sr[32 * q + e]);
                            mxa = fmax3(mxa, v[0], v[1]);
                            mxb = fmax3(mxb, v[2], v[3]);
                            mxc = fmax3(mxc, v[4], v[5]);
                            mxd = fmax3(mxd, v[6], v[7]);
                        }
                    }
            }
            const float mx = fmaxf(fmaxf(mxa, mxb), fmaxf(mxc, mxd));
            const float mx2 = pooled ? mx : mx * scale_log2;
            const bool need = (c > 0) && (mx2 > m + kRescaleThreshold);
            if (c == 0) m = mx2;
            // TMEM loads / stores are warp-collective: the whole warp rescales when
            // any of its rows needs it (a row whose max did not grow gets 1).  O
            // holds every earlier chunk: S_c was issued after P_{c-1} V_{c-1}.
            if (__any_sync(0xffffffffu, need)) {
                const float mnew = fmaxf(m, mx2);
                const float corr = ex2(m - mnew);
#pragma unroll 1
                for (int q = 0; q < D / 16; ++q) {
                    uint32_t orr[16];
                    tmem_ld16(tO + lane_off + q * 16, orr);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * corr);
                    tmem_st16(tO + lane_off + q * 16, orr);
                }
                l *= corr;
                m = mnew;
            }
            // pass 2: P = exp2(S*scale*log2e - m), bf16 pairs written over S
            // (group q packs into columns [16q, 16q+16); all of S is in registers).
            // (scale, -m) and the running sum as packed fp32 pairs; a pooled
            // chunk's registers already hold the scaled, biased x.
            const uint64_t s2 = splat2(pooled ? 1.0f : scale_log2), c2 = splat2(-m);
            uint64_t acc2 = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (q < nq) {
                    uint32_t pk[16];
                    if (q < 2 ? live0 : live1) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            float x0, x1;
                            fma2(__uint_as_float(sr[32 * q + 2 * e]), __uint_as_float(sr[32 * q + 2 * e + 1]), s2, c2,
                                 x0, x1);
                            const float p0 = ex2(x0), p1 = ex2(x1);
                            add2(acc2, p0, p1);
                            pk[e] = pack_bf16x2(p0, p1);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) pk[e] = 0u;
                    }
                    tmem_st16(tSr + q * 16, pk);
                    if (q == 1) {  // P of keys 0..63 is in TMEM: the first half of P V may start
                        tmem_wait_st();
                        tc_fence_before();
                        mbar_arrive(bar_p);
                    }
                }
            const float sum = sum2(acc2);
            l += sum;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_p2);
        }
        // epilogue: the last product P V must have landed
        if (ok && nchunk_all > 0)
            ok = __all_sync(0xffffffffu, mbar_wait(bar_o, (nchunk_all - 1) & 1, status, kSiteO, abort_flag));
        if (ok && nchunk_all > 0) {
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
                const float lse2 = m + __log2f(l);
                if (!kTaylor) nlse_p[(size_t)bh * g.N + n] = -lse2;  // negated, log2 units: the backward's exp2 addend
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

// Exercises the bounded-wait failure path: one thread waits on an mbarrier
// that nothing arrives on, with the same helper the attention kernels use,
// and records the timeout in the plan's status word.
__global__ void k_selftest_bounded_wait(int *status) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(smem_u32(&bar), 1);
        mbar_fence_init();
        mbar_wait(smem_u32(&bar), 0, status, 99, &abort_flag);
    }
}

prism_status launch_selftest_bounded_wait(Plan &pl, cudaStream_t st) {
    k_selftest_bounded_wait<<<1, 32, 0, st>>>(pl.status);
    PRISM_CUDA_OK(cudaGetLastError());
    return PRISM_OK;
}

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
    const uint64_t prow = (uint64_t)pl.g.batch * pl.g.heads * pl.g.nbmax;
    prism_status s = make_map(&pl.tmQ, pl.Qp, rows, pl.g.D);
    if (s == PRISM_OK) s = make_map(&pl.tmKb, pl.Kb, prow, pl.g.D);
    if (s == PRISM_OK) s = make_map(&pl.tmVb, pl.Vb, prow, pl.g.D);
    if (s == PRISM_OK) s = make_map(&pl.tmK, pl.Kp, rows, pl.g.D);
    if (s == PRISM_OK) s = make_map(&pl.tmV, pl.Vp, rows, pl.g.D);
    if (s == PRISM_OK) s = make_map(&pl.tmdO, pl.dOp, rows, pl.g.D);
    if (s == PRISM_OK) s = make_map_f32_rows(&pl.tmdQ, pl.dQacc, rows, pl.g.D);
    return s;
}

template <int D, bool kTaylor>
static prism_status fwd_tc_impl(Plan &pl, void *O, float *lse, cudaStream_t st) {
    const Geo &g = pl.g;
    const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    const uint32_t smem = kTaylor ? fwdtc::Layout<D>::taylor_alloc(g.nbmax) : fwdtc::Layout<D>::kAlloc;
    TimerScope ts(pl, kTaylor ? kTAttnFwdTaylor : kTAttnFwd, st);
    fwdtc::k_attn_fwd_tc<D, kTaylor><<<dim3(g.nbmax, g.batch * g.heads), fwdtc::kThreads, smem, st>>>(
        pl.tmQ, pl.tmK, pl.tmV, pl.tmKb, pl.tmVb, pl.nb, g, pl.nqt, pl.qt_row, pl.qt_blk, pl.blk_off, pl.row_ptr,
        pl.col, pl.perm, static_cast<__nv_bfloat16 *>(O), lse, pl.nlse_p, scale_log2, pl.status);
    PRISM_CUDA_OK(cudaGetLastError());
    return PRISM_OK;
}

// Largest dynamic shared memory of a CTA on sm_100 (227 KB).
constexpr int kMaxDynSmem = 232448;

prism_status configure_attn_tc_kernels() {
    PRISM_CUDA_OK(cudaFuncSetAttribute(fwdtc::k_attn_fwd_tc<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)fwdtc::Layout<64>::kAlloc));
    PRISM_CUDA_OK(cudaFuncSetAttribute(fwdtc::k_attn_fwd_tc<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)fwdtc::Layout<128>::kAlloc));
    PRISM_CUDA_OK(cudaFuncSetAttribute(fwdtc::k_attn_fwd_tc<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kMaxDynSmem));
    PRISM_CUDA_OK(cudaFuncSetAttribute(fwdtc::k_attn_fwd_tc<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kMaxDynSmem));
    return PRISM_OK;
}

prism_status launch_attn_fwd_tc(Plan &pl, void *O, float *lse, cudaStream_t st) {
    return pl.g.D == 64 ? fwd_tc_impl<64, false>(pl, O, lse, st) : fwd_tc_impl<128, false>(pl, O, lse, st);
}

bool taylor_fits(const Geo &g) {
    const uint32_t need = g.D == 64 ? fwdtc::Layout<64>::taylor_alloc(g.nbmax) : fwdtc::Layout<128>::taylor_alloc(g.nbmax);
    return need <= (uint32_t)kMaxDynSmem;
}

// Pooled bf16 copies for the Taylor term, one CTA per (block j, sample*head):
// Kb_j = bf16(kbar_j) from the plan's fp64 pooled keys; Vb_j = bf16(mean of
// the block's rows of the permuted V), summed in fp32.
__global__ void __launch_bounds__(256) k_taylor_pool(Geo g, const int *__restrict__ nbv,
                                                     const int *__restrict__ blk_off,
                                                     const double *__restrict__ Kbar,
                                                     const __nv_bfloat16 *__restrict__ Vp,
                                                     __nv_bfloat16 *__restrict__ Kb, __nv_bfloat16 *__restrict__ Vb) {
    __shared__ float part[256 * 8];
    const int j = blockIdx.x, bh = blockIdx.y, b = bh / g.heads;
    if (j >= nbv[b]) return;
    const int *bo = blk_off + (size_t)b * (g.nbmax + 1);
    const int r0 = bo[j], r1 = bo[j + 1];
    const size_t prow = (size_t)bh * g.nbmax + j;
    for (int d = threadIdx.x; d < g.D; d += blockDim.x) Kb[prow * g.D + d] = __double2bfloat16(Kbar[prow * g.D + d]);
    const int lpr = g.D / 8, groups = 256 / lpr;  // 16-byte lanes per row, rows in flight
    const int ln = threadIdx.x % lpr, grp = threadIdx.x / lpr;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const __nv_bfloat16 *src = Vp + ((size_t)bh * g.N) * g.D + ln * 8;
    for (int r = r0 + grp; r < r1; r += groups) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(src + (size_t)r * g.D));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            acc[2 * k] += __uint_as_float(w[k] << 16);
            acc[2 * k + 1] += __uint_as_float(w[k] & 0xFFFF0000u);
        }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) part[threadIdx.x * 8 + k] = acc[k];
    __syncthreads();
    const float inv = 1.0f / (float)(r1 - r0);  // a power of two: exact
    for (int d = threadIdx.x; d < g.D; d += blockDim.x) {
        const int l = d / 8, k = d % 8;
        float sum = 0.f;
        for (int q = 0; q < groups; ++q) sum += part[(q * lpr + l) * 8 + k];
        Vb[prow * g.D + d] = __float2bfloat16_rn(sum * inv);
    }
}

prism_status launch_attn_fwd_taylor(Plan &pl, void *O, float *lse, cudaStream_t st) {
    const Geo &g = pl.g;
    {
        TimerScope ts(pl, kTTaylorPool, st);
        k_taylor_pool<<<dim3(g.nbmax, g.batch * g.heads), 256, 0, st>>>(g, pl.nb, pl.blk_off, pl.Kbar, pl.Vp,
                                                                        pl.Kb, pl.Vb);
        PRISM_CUDA_OK(cudaGetLastError());
    }
    return g.D == 64 ? fwd_tc_impl<64, true>(pl, O, lse, st) : fwd_tc_impl<128, true>(pl, O, lse, st);
}

}  // namespace prism
