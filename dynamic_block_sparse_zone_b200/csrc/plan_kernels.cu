// plan_kernels.cu -- the Prism planner on sm_100a.
//
// Steps [Prism guide = paper guide "Prism: Dynamic Sparse Attention cho Huan
// luyen Mo hinh Tao Video-Am thanh Dong thoi Do phan giai Goc 2K", xyznot.com
// 2610.05416]:
//   k_zone_stats_v / k_zone_stats_a  Method section 1: directional variances of
//                                    slice means of V (all heads x head_dim
//                                    channels) and of the audio norms a
//   k_zone_decide                    Method sections 1-2: r, vhat, abar, g_d,
//                                    density rho, volume B(m) from tau_128 /
//                                    tau_256, l*_d, nearest candidate shape;
//                                    block table of the block-contiguous order
//                                    (or the table alone, for decisions the
//                                    caller gives)
//   k_permute_pool                   block-contiguous head-major copies of Q,K,V
//                                    and the mean-pooled blocks (Method section 3)
//   k_select                         Method section 3: pooled block scores, block
//                                    probabilities, S_i = Top-k U Top-p (+ cap)
//   k_scan_* / k_csr_* / k_csc_*     compaction into a block CSR and its transpose
//
// Decision arithmetic (everything that turns a number into a choice) is fp64
// with explicitly rounded operations (no contraction), so that a choice can
// differ from an fp64 reference only where two candidates are within rounding
// of each other.
#include <float.h>
#include <math.h>

#include "prism_internal.cuh"

namespace prism {

// Candidate table: edge exponents (eT,eH,eW) in {1,2,3}^3, volumes 64, 128, 256
// in that order, lexicographic inside a volume [Prism guide, core ideas bullet 3].
// Filled once per device by upload_shape_table().
__constant__ int c_shape_exp[kNumShapes][3];

int host_shape_table(int (*e)[3]) {
    int n = 0;
    for (int vol_log = 6; vol_log <= 8; ++vol_log)
        for (int a = 1; a <= 3; ++a)
            for (int b = 1; b <= 3; ++b) {
                int c = vol_log - a - b;
                if (c >= 1 && c <= 3) {
                    e[n][0] = a; e[n][1] = b; e[n][2] = c;
                    ++n;
                }
            }
    return n;
}

prism_status upload_shape_table() {
    int e[kNumShapes][3];
    host_shape_table(e);
    PRISM_CUDA_OK(cudaMemcpyToSymbol(c_shape_exp, e, sizeof e));
    return PRISM_OK;
}

// ---------------------------------------------------------------------------
// small device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 ld_stream(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void bf16x8_to_float(const uint4 &r, float *x) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        x[2 * k] = __uint_as_float(w[k] << 16);
        x[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// ---------------------------------------------------------------------------
// K1: per (zone, 128-channel chunk): sum over channels of the three
// directional variances of slice means of V.
// CTA = 128 threads: half-warp s (0..7) walks t-slice s of the zone; each of
// its 16 lanes owns 8 consecutive channels (one 16-byte load per token).
// Phase 1 keeps fp32 partial sums over 8 tokens; phase 2 (thread = channel)
// combines them in fp64.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) k_zone_stats_v(const __nv_bfloat16 *__restrict__ V, Geo g,
                                                      double *__restrict__ zone_part) {
    extern __shared__ float4 smem_f4[];
    float *hpart = reinterpret_cast<float *>(smem_f4);  // [t][h][128]
    float *wpart = hpart + 8 * 8 * kStatChunk;          // [t][w][128]
    __shared__ double red[4][3];
    const int chunk = blockIdx.x, m = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, ts = tid >> 4, l = tid & 15;
    const int zt = m / (g.MH * g.MW), zh = (m / g.MW) % g.MH, zw = m % g.MW;
    const int c0 = chunk * kStatChunk + l * 8;
    const bool valid = c0 < g.C;
    float wacc[8][8];
#pragma unroll
    for (int w = 0; w < 8; ++w)
#pragma unroll
        for (int k = 0; k < 8; ++k) wacc[w][k] = 0.f;
    const __nv_bfloat16 *base = V + (size_t)b * g.N * g.C + c0;
#pragma unroll 1
    for (int h = 0; h < 8; ++h) {
        const size_t tok0 = ((size_t)(zt * 8 + ts) * g.H + (zh * 8 + h)) * g.W + zw * 8;
        uint4 raw[8];
#pragma unroll
        for (int w = 0; w < 8; ++w)
            raw[w] = valid ? ld_stream(base + (tok0 + w) * g.C) : make_uint4(0, 0, 0, 0);
        float hacc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) hacc[k] = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            float x[8];
            bf16x8_to_float(raw[w], x);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                hacc[k] += x[k];
                wacc[w][k] += x[k];
            }
        }
        float4 *dst = reinterpret_cast<float4 *>(hpart + (ts * 8 + h) * kStatChunk + l * 8);
        dst[0] = make_float4(hacc[0], hacc[1], hacc[2], hacc[3]);
        dst[1] = make_float4(hacc[4], hacc[5], hacc[6], hacc[7]);
    }
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        float4 *dst = reinterpret_cast<float4 *>(wpart + (ts * 8 + w) * kStatChunk + l * 8);
        dst[0] = make_float4(wacc[w][0], wacc[w][1], wacc[w][2], wacc[w][3]);
        dst[1] = make_float4(wacc[w][4], wacc[w][5], wacc[w][6], wacc[w][7]);
    }
    __syncthreads();

    double v3[3] = {0.0, 0.0, 0.0};
    const int ch = tid;
    if (chunk * kStatChunk + ch < g.C) {
        double ST[8], SH[8], SW[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) ST[i] = SH[i] = SW[i] = 0.0;
#pragma unroll
        for (int t = 0; t < 8; ++t)
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                double x = (double)hpart[(t * 8 + h) * kStatChunk + ch];
                ST[t] = __dadd_rn(ST[t], x);
                SH[h] = __dadd_rn(SH[h], x);
            }
#pragma unroll
        for (int t = 0; t < 8; ++t)
#pragma unroll
            for (int w = 0; w < 8; ++w) SW[w] = __dadd_rn(SW[w], (double)wpart[(t * 8 + w) * kStatChunk + ch]);
        double tot = 0.0;
#pragma unroll
        for (int t = 0; t < 8; ++t) tot = __dadd_rn(tot, ST[t]);
        const double mu = tot / 512.0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            double dT = __dadd_rn(ST[i] / 64.0, -mu), dH = __dadd_rn(SH[i] / 64.0, -mu),
                   dW = __dadd_rn(SW[i] / 64.0, -mu);
            v3[0] = __dadd_rn(v3[0], __dmul_rn(dT, dT));
            v3[1] = __dadd_rn(v3[1], __dmul_rn(dH, dH));
            v3[2] = __dadd_rn(v3[2], __dmul_rn(dW, dW));
        }
#pragma unroll
        for (int d = 0; d < 3; ++d) v3[d] = v3[d] / 8.0;
    }
#pragma unroll
    for (int d = 0; d < 3; ++d) v3[d] = warp_sum_d(v3[d]);
    if ((tid & 31) == 0)
        for (int d = 0; d < 3; ++d) red[tid >> 5][d] = v3[d];
    __syncthreads();
    if (tid < 3) {
        double s = 0.0;
        for (int wq = 0; wq < 4; ++wq) s = __dadd_rn(s, red[wq][tid]);
        // chunk-major: a rank's heads are one contiguous slice of the layer's partials
        zone_part[(((size_t)(g.chunk0 + chunk) * g.batch + b) * g.M + m) * 3 + tid] = s;
    }
}

// ---------------------------------------------------------------------------
// K1a: per zone: directional variances of slice means of a, its zone mean and
// zone maximum.  512 threads, one per token of the zone.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(512) k_zone_stats_a(const float *__restrict__ a, Geo g,
                                                      double *__restrict__ zone_a) {
    __shared__ float cube[512];
    __shared__ double slice[3][8];
    __shared__ double tot_s, max_s;
    const int m = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const int zt = m / (g.MH * g.MW), zh = (m / g.MW) % g.MH, zw = m % g.MW;
    const int t = tid >> 6, h = (tid >> 3) & 7, w = tid & 7;
    cube[tid] = a[(size_t)b * g.N + ((size_t)(zt * 8 + t) * g.H + (zh * 8 + h)) * g.W + zw * 8 + w];
    __syncthreads();
    if (tid < 24) {
        const int d = tid >> 3, i = tid & 7;
        double s = 0.0;
        for (int u = 0; u < 8; ++u)
            for (int v = 0; v < 8; ++v) {
                int tt, hh, ww;
                if (d == 0) { tt = i; hh = u; ww = v; }
                else if (d == 1) { tt = u; hh = i; ww = v; }
                else { tt = u; hh = v; ww = i; }
                s = __dadd_rn(s, (double)cube[(tt * 8 + hh) * 8 + ww]);
            }
        slice[d][i] = s;
    } else if (tid == 32) {
        double s = 0.0, mx = -DBL_MAX;
        for (int u = 0; u < 512; ++u) {
            s = __dadd_rn(s, (double)cube[u]);
            mx = fmax(mx, (double)cube[u]);
        }
        tot_s = s;
        max_s = mx;
    }
    __syncthreads();
    if (tid == 0) {
        const double mu = tot_s / 512.0;
        double *o = zone_a + ((size_t)b * g.M + m) * 5;
        for (int d = 0; d < 3; ++d) {
            double acc = 0.0;
            for (int i = 0; i < 8; ++i) {
                double dd = __dadd_rn(slice[d][i] / 64.0, -mu);
                acc = __dadd_rn(acc, __dmul_rn(dd, dd));
            }
            o[d] = acc / 8.0;
        }
        o[3] = mu;
        o[4] = max_s;
    }
}

// ---------------------------------------------------------------------------
// K2: per sample, one CTA: indicator, density, volume, shape, block table.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int block_scan_excl_1024(int v, int *buf, int *total) {
    // Exclusive scan over blockDim.x (<= 1024) ints; deterministic.
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) buf[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int nw = (blockDim.x + 31) >> 5;
        int s = lane < nw ? buf[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        buf[32 + lane] = s;  // inclusive warp totals
    }
    __syncthreads();
    int excl = x - v + (wid > 0 ? buf[32 + wid - 1] : 0);
    *total = buf[32 + ((blockDim.x + 31) >> 5) - 1];
    __syncthreads();
    return excl;
}

// sigma^2_{v,d}(m): the chunk partials of zone zm (= b * M + m) summed in chunk
// order over the whole layer's channels, divided by their count
__device__ __forceinline__ double zone_sig(const double *zone_part, const Geo &g, size_t zm, int d) {
    const size_t bm = (size_t)g.batch * g.M;
    double s = 0.0;
    for (int c = 0; c < g.nchunk_tot; ++c) s = __dadd_rn(s, zone_part[(c * bm + zm) * 3 + d]);
    return s / (double)g.Ctot;
}

// given: zone_B / zone_shape already hold the decisions (checked on the
// host); only the block table is built.
__global__ void __launch_bounds__(1024) k_zone_decide(Geo g, const double *__restrict__ zone_part,
                                                      const double *__restrict__ zone_a, double eps,
                                                      int fixed_idx, bool given, int *__restrict__ zone_B,
                                                      int *__restrict__ zone_shape, int *__restrict__ zone_blk0,
                                                      int *__restrict__ nb_out, int *__restrict__ blk_off,
                                                      int *__restrict__ tile_blk, int *__restrict__ zone_qt0,
                                                      int *__restrict__ nqt, int *__restrict__ qt_row,
                                                      int *__restrict__ qt_blk) {
    __shared__ double red_s[32], red_a[32];
    __shared__ int sbuf[64];
    __shared__ double s_max_sh, a_max_sh;
    const int b = blockIdx.x, tid = threadIdx.x;
    const int M = g.M;
    // pass 1: maxima of s(m) and of a over the grid
    double smax = 0.0, amax = -DBL_MAX;
    for (int m = given ? M : tid; m < M; m += blockDim.x) {
        size_t zm = (size_t)b * M + m;
        double s = __dadd_rn(__dadd_rn(zone_sig(zone_part, g, zm, 0), zone_sig(zone_part, g, zm, 1)),
                             zone_sig(zone_part, g, zm, 2));
        smax = fmax(smax, s);
        amax = fmax(amax, zone_a[zm * 5 + 4]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        smax = fmax(smax, __shfl_xor_sync(0xffffffffu, smax, o));
        amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    }
    if ((tid & 31) == 0) {
        red_s[tid >> 5] = smax;
        red_a[tid >> 5] = amax;
    }
    __syncthreads();
    if (tid == 0) {
        double s = 0.0, a = -DBL_MAX;
        for (int w = 0; w < (int)((blockDim.x + 31) >> 5); ++w) {
            s = fmax(s, red_s[w]);
            a = fmax(a, red_a[w]);
        }
        s_max_sh = s;
        a_max_sh = a;
    }
    __syncthreads();
    const double s_max = s_max_sh, a_max = a_max_sh;

    // pass 2: decisions, then a running exclusive scan of blocks per zone
    int carry = 0, carry_t = 0;
    for (int base = 0; base < M; base += blockDim.x) {
        const int m = base + tid;
        int nblk = 0, ntile = 0;
        if (m < M && given) {
            nblk = kZoneVol / zone_B[(size_t)b * M + m];
            ntile = kZoneVol / 128;
        } else if (m < M) {
            size_t zm = (size_t)b * M + m;
            double sg[3], sa[3];
            for (int d = 0; d < 3; ++d) {
                sg[d] = zone_sig(zone_part, g, zm, d);
                sa[d] = zone_a[zm * 5 + d];
            }
            const double sv = __dadd_rn(__dadd_rn(sg[0], sg[1]), sg[2]);
            const double sat = __dadd_rn(__dadd_rn(sa[0], sa[1]), sa[2]);
            const double abar = (a_max > 0.0) ? zone_a[zm * 5 + 3] / a_max : 0.0;
            double gd[3];
            for (int d = 0; d < 3; ++d) {
                double r = (sv < 1e-30) ? (1.0 / 3.0) : sg[d] / sv;
                double vh = (sat < 1e-30) ? (1.0 / 3.0) : sa[d] / sat;
                gd[d] = __dadd_rn(__dadd_rn(r, __dmul_rn(abar, vh)), eps);
            }
            double rv = (s_max > 0.0) ? sv / s_max : 0.0;
            double rho = rv > abar ? rv : abar;
            if (rho > 1.0) rho = 1.0;
            int idx, B;
            if (fixed_idx >= 0) {
                idx = fixed_idx;
                B = 1 << (c_shape_exp[idx][0] + c_shape_exp[idx][1] + c_shape_exp[idx][2]);
            } else {
                B = (rho >= 0.5) ? 64 : ((rho >= 0.25) ? 128 : 256);
                const int S = (B == 64) ? 6 : ((B == 128) ? 7 : 8);
                // l*_d = -1/2 log2 g_d + 1/3 (S + 1/2 sum_d' log2 g_d')  [Method section 2]
                const double hl = __dadd_rn(__dadd_rn(__dmul_rn(0.5, log2(gd[0])), __dmul_rn(0.5, log2(gd[1]))),
                                            __dmul_rn(0.5, log2(gd[2])));
                double l[3];
                for (int d = 0; d < 3; ++d)
                    l[d] = __dadd_rn(__dmul_rn(-0.5, log2(gd[d])), __dmul_rn(1.0 / 3.0, __dadd_rn((double)S, hl)));
                double best = DBL_MAX;
                idx = -1;
                for (int c = 0; c < kNumShapes; ++c) {
                    if (c_shape_exp[c][0] + c_shape_exp[c][1] + c_shape_exp[c][2] != S) continue;
                    double dist = 0.0;
                    for (int d = 0; d < 3; ++d) {
                        double df = __dadd_rn(l[d], -(double)c_shape_exp[c][d]);
                        dist = __dadd_rn(dist, __dmul_rn(df, df));
                    }
                    if (dist < best) {
                        best = dist;
                        idx = c;
                    }
                }
            }
            zone_B[zm] = B;
            zone_shape[zm] = idx;
            nblk = kZoneVol / B;
            ntile = kZoneVol / 128;  // 128-row tiles of the zone (two 64-token blocks share one)
        }
        int total, total_t;
        const int excl = block_scan_excl_1024(nblk, sbuf, &total);
        const int excl_t = block_scan_excl_1024(ntile, sbuf, &total_t);
        if (m < M) {
            zone_blk0[(size_t)b * (M + 1) + m] = carry + excl;
            zone_qt0[(size_t)b * (M + 1) + m] = carry_t + excl_t;
        }
        carry += total;
        carry_t += total_t;
    }
    if (tid == 0) {
        zone_blk0[(size_t)b * (M + 1) + M] = carry;
        zone_qt0[(size_t)b * (M + 1) + M] = carry_t;
        nb_out[b] = carry;
        nqt[b] = carry_t;
        blk_off[(size_t)b * (g.nbmax + 1) + carry] = g.N;
    }
    __syncthreads();
    // pass 3: block table (block-contiguous token offsets) and 64-row tile map
    for (int m = tid; m < M; m += blockDim.x) {
        size_t zm = (size_t)b * M + m;
        const int B = zone_B[zm];
        const int j0 = zone_blk0[(size_t)b * (M + 1) + m];
        int t = zone_qt0[(size_t)b * (M + 1) + m];
        for (int l = 0; l < kZoneVol / B; ++l) {
            const int off = m * kZoneVol + l * B;
            blk_off[(size_t)b * (g.nbmax + 1) + j0 + l] = off;
            for (int u = 0; u < B / kTile; ++u) tile_blk[(size_t)b * g.nbmax + off / kTile + u] = j0 + l;
            if (B == 64) {  // blocks l, l+1 share a tile, marked by the complement of the first
                if ((l & 1) == 0) {
                    qt_row[(size_t)b * g.nbmax + t] = off;
                    qt_blk[(size_t)b * g.nbmax + t] = ~(j0 + l);
                    ++t;
                }
                continue;
            }
            for (int r = 0; r < B; r += 128, ++t) {
                qt_row[(size_t)b * g.nbmax + t] = off + r;
                qt_blk[(size_t)b * g.nbmax + t] = j0 + l;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// K3: block-contiguous, head-major copies of Q, K, V and the fp64 block means
// of Q and K.  One CTA per (block, slice of kPPThreads x 8 channels); a thread
// owns 8 channels of one head and walks the block's tokens.
// ---------------------------------------------------------------------------
constexpr int kPPThreads = 128;
struct BlockGeom {
    int off, B, t0, h0, w0, bT, bH, bW, eH, eW;  // edges bT x bH x bW; bH = 2^eH, bW = 2^eW
};

__device__ __forceinline__ BlockGeom block_geom(const Geo &g, const int *blk_off_b, const int *zone_shape_b, int j) {
    BlockGeom r;
    r.off = blk_off_b[j];
    r.B = blk_off_b[j + 1] - r.off;
    const int m = r.off / kZoneVol;
    const int s = zone_shape_b[m];
    r.eH = c_shape_exp[s][1];
    r.eW = c_shape_exp[s][2];
    r.bT = 1 << c_shape_exp[s][0];
    r.bH = 1 << r.eH;
    r.bW = 1 << r.eW;
    const int lidx = (r.off - m * kZoneVol) / r.B;
    const int nW = 8 / r.bW, nH = 8 / r.bH;
    const int iw = lidx % nW, ih = (lidx / nW) % nH, it = lidx / (nW * nH);
    const int zt = m / (g.MH * g.MW), zh = (m / g.MW) % g.MH, zw = m % g.MW;
    r.t0 = zt * 8 + it * r.bT;
    r.h0 = zh * 8 + ih * r.bH;
    r.w0 = zw * 8 + iw * r.bW;
    return r;
}

__device__ __forceinline__ int block_token(const Geo &g, const BlockGeom &bg, int r) {
    const int tt = r >> (bg.eH + bg.eW), hh = (r >> bg.eW) & (bg.bH - 1), ww = r & (bg.bW - 1);
    return ((bg.t0 + tt) * g.H + (bg.h0 + hh)) * g.W + (bg.w0 + ww);
}

// kPerm: the blocks are runs of an existing permutation (Hilbert-order plans),
// which is read instead of derived from the zone shapes and written.
template <bool kPerm>
__global__ void __launch_bounds__(kPPThreads, 5) k_permute_pool(const __nv_bfloat16 *__restrict__ Q,
                                                      const __nv_bfloat16 *__restrict__ K,
                                                      const __nv_bfloat16 *__restrict__ V, Geo g,
                                                      const int *__restrict__ nb, const int *__restrict__ blk_off,
                                                      const int *__restrict__ zone_shape, int *__restrict__ perm,
                                                      __nv_bfloat16 *__restrict__ Qp, __nv_bfloat16 *__restrict__ Kp,
                                                      __nv_bfloat16 *__restrict__ Vp, double *__restrict__ Qbar,
                                                      double *__restrict__ Kbar) {
    const int nslice = (g.C / 8 + kPPThreads - 1) / kPPThreads;
    const int j = blockIdx.x / nslice, slice = blockIdx.x % nslice, b = blockIdx.y;
    if (j >= nb[b]) return;
    BlockGeom bg;
    if constexpr (kPerm) {
        const int *bo = blk_off + (size_t)b * (g.nbmax + 1);
        bg.off = bo[j];
        bg.B = bo[j + 1] - bo[j];
    } else {
        bg = block_geom(g, blk_off + (size_t)b * (g.nbmax + 1), zone_shape + (size_t)b * g.M, j);
        if (slice == 0)
            for (int r = threadIdx.x; r < bg.B; r += blockDim.x)
                perm[(size_t)b * g.N + bg.off + r] = block_token(g, bg, r);
    }
    const int *pb = perm + (size_t)b * g.N + bg.off;
    const int G = g.C / 8;
    const double inv = 1.0 / (double)bg.B;  // B is a power of two: exact
    const int grp = slice * kPPThreads + threadIdx.x;
    if (grp < G) {
        const int hd = (grp * 8) / g.D, d0 = (grp * 8) % g.D;
        const size_t bh = (size_t)b * g.heads + hd;
        double sq[8], sk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) sq[k] = sk[k] = 0.0;
        const __nv_bfloat16 *srcQ = Q + (size_t)b * g.N * g.C + grp * 8;
        const __nv_bfloat16 *srcK = K + (size_t)b * g.N * g.C + grp * 8;
        const __nv_bfloat16 *srcV = V + (size_t)b * g.N * g.C + grp * 8;
        const size_t dst0 = (bh * g.N + bg.off) * g.D + d0;
#pragma unroll 4
        for (int r = 0; r < bg.B; ++r) {
            const size_t tok = kPerm ? (size_t)pb[r] : (size_t)block_token(g, bg, r);
            const uint4 q = ld_stream(srcQ + tok * g.C);
            const uint4 k = ld_stream(srcK + tok * g.C);
            const uint4 v = ld_stream(srcV + tok * g.C);
            *reinterpret_cast<uint4 *>(Qp + dst0 + (size_t)r * g.D) = q;
            *reinterpret_cast<uint4 *>(Kp + dst0 + (size_t)r * g.D) = k;
            *reinterpret_cast<uint4 *>(Vp + dst0 + (size_t)r * g.D) = v;
            float xq[8], xk[8];
            bf16x8_to_float(q, xq);
            bf16x8_to_float(k, xk);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                sq[e] = __dadd_rn(sq[e], (double)xq[e]);
                sk[e] = __dadd_rn(sk[e], (double)xk[e]);
            }
        }
        double *oq = Qbar + (bh * g.nbmax + j) * g.D + d0;
        double *ok = Kbar + (bh * g.nbmax + j) * g.D + d0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            oq[e] = sq[e] * inv;
            ok[e] = sk[e] * inv;
        }
    }
}

// ---------------------------------------------------------------------------
// K4: selection.  One CTA (256 threads) per (sample*head, query block i).
// Keys: z_ij = Qbar_i . Kbar_j / sqrt(D) in fp64 (sequential over channels, no
// contraction), mapped to order-preserving u64.  The order is (z desc, j asc).
// At most `cap` blocks can be kept, so the top-`cap` candidates are isolated
// with an MSB-first radix select on the keys (counts only, exact), sorted
// with a bitonic network, and scanned for the Top-p cut.
// ---------------------------------------------------------------------------
constexpr int kSelThreads = 256;

__device__ __forceinline__ uint64_t order_key(double z) {
    if (z == 0.0) z = 0.0;  // one zero
    const uint64_t u = (uint64_t)__double_as_longlong(z);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}
__device__ __forceinline__ double key_value(uint64_t k) {
    const uint64_t u = (k >> 63) ? (k & 0x7fffffffffffffffull) : ~k;
    return __longlong_as_double((long long)u);
}
// a precedes c in the selection order
__device__ __forceinline__ bool precedes(uint64_t ka, int ja, uint64_t kc, int jc) {
    return ka > kc || (ka == kc && ja < jc);
}

__device__ __forceinline__ double block_sum_d(double v, double *red) {
    v = warp_sum_d(v);
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (lane == 0) red[wid] = v;
    __syncthreads();
    double s = 0.0;
    for (int w = 0; w < kSelThreads / 32; ++w) s = __dadd_rn(s, red[w]);
    __syncthreads();
    return s;
}

__device__ __forceinline__ unsigned long long block_max_u64(unsigned long long v, unsigned long long *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        unsigned long long y = __shfl_xor_sync(0xffffffffu, v, o);
        v = y > v ? y : v;
    }
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    if (lane == 0) red[wid] = v;
    __syncthreads();
    unsigned long long s = 0;
    for (int w = 0; w < kSelThreads / 32; ++w) s = red[w] > s ? red[w] : s;
    __syncthreads();
    return s;
}

// exclusive scan over the CTA (256 threads) of ints, returns the total in *tot
__device__ __forceinline__ int block_scan_256(int v, int *buf, int *tot) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) buf[wid] = x;
    __syncthreads();
    int before = 0, all = 0;
    for (int w = 0; w < kSelThreads / 32; ++w) {
        if (w < wid) before += buf[w];
        all += buf[w];
    }
    __syncthreads();
    *tot = all;
    return before + x - v;
}

struct SelSmem {
    // layout inside the dynamic buffer (offsets in bytes)
    size_t keys, sk, sj, pr, bits;
    size_t bytes;
};

__host__ __device__ inline int pow2_at_least(int x) {
    int p = 1;
    while (p < x) p <<= 1;
    return p;
}

__host__ __device__ inline SelSmem sel_smem_layout(int D, int nbmax, int cap_stride) {
    SelSmem L;
    const int SP = pow2_at_least(cap_stride);
    size_t o = 0;
    L.keys = o; o += (size_t)nbmax * 8;
    L.sk = o;   o += (size_t)SP * 8;
    L.pr = o;   o += (size_t)SP * 8;
    L.sj = o;   o += (size_t)SP * 4;
    L.bits = o; o += (size_t)((nbmax + 31) / 32) * 4;
    L.bytes = (o + 15) & ~(size_t)15;
    return L;
}

// Pooled block scores of a group of heads: z_ij = Qbar_i . Kbar_j / sqrt(D),
// stored as order-preserving u64 keys in keys[head of group][i][j].  A CTA
// computes a 64 x 64 block; each thread keeps 16 scores in flight, each one
// summed over the channels in ascending order with explicitly rounded fp64
// operations (the oracle's order).
constexpr int kScoreTile = 64;
constexpr int kScoreSlice = 32;

__global__ void __launch_bounds__(256) k_scores(Geo g, const int *__restrict__ nb_arr,
                                                const double *__restrict__ Qbar, const double *__restrict__ Kbar,
                                                int bh0, unsigned long long *__restrict__ keys) {
    __shared__ double sq[kScoreTile][kScoreSlice + 1], sk[kScoreTile][kScoreSlice + 1];
    const int jt = blockIdx.x, it = blockIdx.y, bh = bh0 + blockIdx.z;
    if (bh >= g.batch * g.heads) return;
    const int nb = nb_arr[bh / g.heads];
    const int i0 = it * kScoreTile, j0 = jt * kScoreTile;
    if (i0 >= nb || j0 >= nb) return;
    const int tid = threadIdx.x, ti = tid >> 4, tj = tid & 15;
    const double *qb = Qbar + (size_t)bh * g.nbmax * g.D;
    const double *kb = Kbar + (size_t)bh * g.nbmax * g.D;
    double acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c] = 0.0;
    for (int c0 = 0; c0 < g.D; c0 += kScoreSlice) {
        for (int idx = tid; idx < kScoreTile * kScoreSlice; idx += 256) {
            const int r = idx / kScoreSlice, c = idx % kScoreSlice;
            sq[r][c] = (i0 + r < nb) ? qb[(size_t)(i0 + r) * g.D + c0 + c] : 0.0;
            sk[r][c] = (j0 + r < nb) ? kb[(size_t)(j0 + r) * g.D + c0 + c] : 0.0;
        }
        __syncthreads();
#pragma unroll 4
        for (int c = 0; c < kScoreSlice; ++c) {
            double qa[4], kc[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) qa[a] = sq[ti + 16 * a][c];
#pragma unroll
            for (int e = 0; e < 4; ++e) kc[e] = sk[tj + 16 * e][c];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[a][e] = __dadd_rn(acc[a][e], __dmul_rn(qa[a], kc[e]));
        }
        __syncthreads();
    }
    const double sqrtD = __dsqrt_rn((double)g.D);
    unsigned long long *out = keys + (size_t)blockIdx.z * g.nbmax * g.nbmax;
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int i = i0 + ti + 16 * a, j = j0 + tj + 16 * e;
            if (i < nb && j < nb) out[(size_t)i * g.nbmax + j] = order_key(__ddiv_rn(acc[a][e], sqrtD));
        }
}

__global__ void __launch_bounds__(kSelThreads) k_select(Geo g, const int *__restrict__ nb_arr,
                                                        const unsigned long long *__restrict__ keys_in, int bh0,
                                                        int top_k, double top_p, float max_frac, int cap_stride,
                                                        int *__restrict__ cnt, int *__restrict__ cols_pad) {
    extern __shared__ __align__(16) unsigned char sel_raw[];
    __shared__ int hist[256];
    __shared__ int ibuf[64];
    __shared__ double dred[32];
    __shared__ unsigned long long ured[32];
    __shared__ int s_digit, s_rem, s_done, s_fill, s_np;
    const int i = blockIdx.x, bh = bh0 + blockIdx.y, b = bh / g.heads;
    if (bh >= g.batch * g.heads) return;
    const int tid = threadIdx.x;
    const size_t row = (size_t)bh * g.nbmax + i;
    const int nb = nb_arr[b];
    if (i >= nb) {
        if (tid == 0) cnt[row] = 0;
        return;
    }
    const SelSmem L = sel_smem_layout(g.D, g.nbmax, cap_stride);
    uint64_t *keys = reinterpret_cast<uint64_t *>(sel_raw + L.keys);
    uint64_t *sk = reinterpret_cast<uint64_t *>(sel_raw + L.sk);
    double *pr = reinterpret_cast<double *>(sel_raw + L.pr);
    int *sj = reinterpret_cast<int *>(sel_raw + L.sj);
    uint32_t *bits = reinterpret_cast<uint32_t *>(sel_raw + L.bits);

    // scores of this row (written by k_scores)
    const unsigned long long *krow = keys_in + ((size_t)blockIdx.y * g.nbmax + i) * g.nbmax;
    unsigned long long kmax = 0;
    for (int j = tid; j < nb; j += kSelThreads) {
        const unsigned long long key = krow[j];
        keys[j] = key;
        kmax = key > kmax ? key : kmax;
    }
    kmax = block_max_u64(kmax, ured);
    const double zmax = key_value(kmax);
    double part = 0.0;
    for (int j = tid; j < nb; j += kSelThreads) part = __dadd_rn(part, exp(__dadd_rn(key_value(keys[j]), -zmax)));
    const double denom = block_sum_d(part, dred);

    const int cap = cap_for(nb, top_k, max_frac);
    const int msel = cap;  // no row keeps more than cap blocks
    // ---- isolate the top-msel (key desc, j asc) ----
    if (tid == 0) s_fill = 0;
    if (msel >= nb) {
        __syncthreads();
        for (int j = tid; j < nb; j += kSelThreads) {
            sk[j] = keys[j];
            sj[j] = j;
        }
    } else {
        uint64_t prefix = 0, mask = 0;
        int remaining = msel;
        bool done = false;
        for (int shift = 56; shift >= 0 && !done; shift -= 8) {
            hist[tid] = 0;
            __syncthreads();
            for (int j = tid; j < nb; j += kSelThreads) {
                const uint64_t k = keys[j];
                if ((k & mask) == prefix) atomicAdd(&hist[(int)((k >> shift) & 255u)], 1);
            }
            __syncthreads();
            if (tid < 32) {
                // lane L covers buckets 255-8L down to 248-8L
                int loc = 0;
                for (int q = 0; q < 8; ++q) loc += hist[255 - 8 * tid - q];
                int incl = loc;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    int y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (tid >= o) incl += y;
                }
                const int excl = incl - loc;
                const unsigned ball = __ballot_sync(0xffffffffu, incl >= remaining);
                const int first = __ffs(ball) - 1;
                if (tid == first) {
                    int acc = excl;
                    for (int q = 0; q < 8; ++q) {
                        const int d = 255 - 8 * tid - q;
                        if (acc + hist[d] >= remaining) {
                            s_digit = d;
                            s_rem = remaining - acc;
                            s_done = (hist[d] == remaining - acc);
                            break;
                        }
                        acc += hist[d];
                    }
                }
            }
            __syncthreads();
            prefix |= (uint64_t)s_digit << shift;
            mask |= (uint64_t)0xff << shift;
            remaining = s_rem;
            done = s_done != 0;
            __syncthreads();
        }
        // strictly above the boundary prefix: kept
        for (int j = tid; j < nb; j += kSelThreads) {
            const uint64_t k = keys[j];
            if ((k & mask) > prefix || (done && (k & mask) == prefix)) {
                const int pos = atomicAdd(&s_fill, 1);
                if (pos < msel) {
                    sk[pos] = k;
                    sj[pos] = j;
                }
            }
        }
        if (!done) {
            // exact key ties at the boundary: the `remaining` lowest j
            int base = 0;
            for (int j0 = 0; j0 < nb; j0 += kSelThreads) {
                const int j = j0 + tid;
                const int f = (j < nb && keys[j] == prefix) ? 1 : 0;
                int tot;
                const int rk = block_scan_256(f, ibuf, &tot) + base;
                if (f && rk < remaining) {
                    const int pos = atomicAdd(&s_fill, 1);
                    if (pos < msel) {
                        sk[pos] = prefix;
                        sj[pos] = j;
                    }
                }
                base += tot;
            }
        }
    }
    __syncthreads();
    const int SP = pow2_at_least(msel);
    for (int u = msel + tid; u < SP; u += kSelThreads) {
        sk[u] = 0;
        sj[u] = 0x7fffffff;
    }
    __syncthreads();
    // ---- bitonic sort into selection order ----
    for (int kk = 2; kk <= SP; kk <<= 1) {
        for (int jj = kk >> 1; jj > 0; jj >>= 1) {
            for (int u = tid; u < SP; u += kSelThreads) {
                const int v = u ^ jj;
                if (v > u) {
                    const uint64_t ka = sk[u], kc = sk[v];
                    const int ja = sj[u], jc = sj[v];
                    const bool swap = ((u & kk) == 0) ? precedes(kc, jc, ka, ja) : precedes(ka, ja, kc, jc);
                    if (swap) {
                        sk[u] = kc; sk[v] = ka;
                        sj[u] = jc; sj[v] = ja;
                    }
                }
            }
            __syncthreads();
        }
    }
    // ---- Top-p cut: shortest prefix with cumulative probability >= p ----
    for (int u = tid; u < msel; u += kSelThreads) pr[u] = exp(__dadd_rn(key_value(sk[u]), -zmax)) / denom;
    __syncthreads();
    if (tid == 0) {
        double cum = 0.0;
        int np_ = nb;
        for (int u = 0; u < msel; ++u) {
            cum = __dadd_rn(cum, pr[u]);
            if (cum >= top_p) {
                np_ = u + 1;
                break;
            }
        }
        s_np = np_;
    }
    __syncthreads();
    const int nk = top_k < nb ? top_k : nb;
    const int want = nk > s_np ? nk : s_np;
    const int n = want < cap ? want : cap;
    // ---- emit ascending block ids ----
    const int nwords = (nb + 31) >> 5;
    for (int wq = tid; wq < nwords; wq += kSelThreads) bits[wq] = 0u;
    __syncthreads();
    for (int u = tid; u < n; u += kSelThreads)
        if (sj[u] < nb) atomicOr(&bits[sj[u] >> 5], 1u << (sj[u] & 31));
    __syncthreads();
    int base = 0;
    int *out = cols_pad + row * cap_stride;
    for (int w0 = 0; w0 < nwords; w0 += kSelThreads) {
        const int wq = w0 + tid;
        const uint32_t word = wq < nwords ? bits[wq] : 0u;
        int tot;
        int pos = block_scan_256(__popc(word), ibuf, &tot) + base;
        uint32_t x = word;
        while (x) {
            const int bit = __ffs(x) - 1;
            x &= x - 1;
            if (pos < cap_stride) out[pos] = wq * 32 + bit;
            ++pos;
        }
        base += tot;
    }
    if (tid == 0) cnt[row] = n;
}

// ---------------------------------------------------------------------------
// Scans (exclusive, int) over long arrays: per-1024 chunk scan, scan of chunk
// totals, add-back.  out has n+1 entries (out[n] = total).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) k_scan_chunks(const int *__restrict__ in, int n, int *__restrict__ out,
                                                      int *__restrict__ totals) {
    __shared__ int buf[64];
    const int i = blockIdx.x * 1024 + threadIdx.x;
    const int v = i < n ? in[i] : 0;
    int tot;
    const int ex = block_scan_excl_1024(v, buf, &tot);
    if (i < n) out[i] = ex;
    if (threadIdx.x == 0) totals[blockIdx.x] = tot;
}

__global__ void __launch_bounds__(1024) k_scan_totals(int *__restrict__ totals, int nchunks, int *__restrict__ out,
                                                      int n) {
    __shared__ int buf[64];
    int carry = 0;
    for (int base = 0; base < nchunks; base += 1024) {
        const int i = base + threadIdx.x;
        const int v = i < nchunks ? totals[i] : 0;
        int tot;
        const int ex = block_scan_excl_1024(v, buf, &tot);
        if (i < nchunks) totals[i] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0) out[n] = carry;
}

__global__ void __launch_bounds__(1024) k_scan_add(int *__restrict__ out, int n, const int *__restrict__ totals) {
    const int i = blockIdx.x * 1024 + threadIdx.x;
    if (i < n) out[i] += totals[blockIdx.x];
}

// Compact the padded selection into the CSR and count entries per column.
__global__ void k_csr_compact(Geo g, int cap_stride, const int *__restrict__ cnt, const int *__restrict__ cols_pad,
                              const int *__restrict__ row_ptr, int *__restrict__ col, int *__restrict__ col_count) {
    const size_t rows = (size_t)g.batch * g.heads * g.nbmax;
    const int lane = threadIdx.x & 31;
    for (size_t r = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
         r += (size_t)gridDim.x * (blockDim.x >> 5)) {
        const int n = cnt[r], p0 = row_ptr[r];
        const size_t colbase = (r / g.nbmax) * g.nbmax;
        for (int u = lane; u < n; u += 32) {
            const int j = cols_pad[r * cap_stride + u];
            col[p0 + u] = j;
            atomicAdd(&col_count[colbase + j], 1);
        }
    }
}

// Scatter rows into columns (order inside a column fixed afterwards).
__global__ void k_csc_fill(Geo g, const int *__restrict__ row_ptr, const int *__restrict__ col,
                           const int *__restrict__ colT_ptr, int *__restrict__ cursor, int *__restrict__ rowT) {
    const size_t rows = (size_t)g.batch * g.heads * g.nbmax;
    const int lane = threadIdx.x & 31;
    for (size_t r = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
         r += (size_t)gridDim.x * (blockDim.x >> 5)) {
        const int p0 = row_ptr[r], p1 = row_ptr[r + 1];
        const size_t colbase = (r / g.nbmax) * g.nbmax;
        const int i = (int)(r % g.nbmax);
        for (int u = p0 + lane; u < p1; u += 32) {
            const size_t c = colbase + col[u];
            rowT[colT_ptr[c] + atomicAdd(&cursor[c], 1)] = i;
        }
    }
}

// Sort every column's row list ascending (deterministic CSC).
__global__ void __launch_bounds__(256) k_csc_sort(size_t ncols, const int *__restrict__ colT_ptr,
                                                  int *__restrict__ rowT, int sp_max) {
    extern __shared__ int sbuf[];
    for (size_t c = blockIdx.x; c < ncols; c += gridDim.x) {
        const int p0 = colT_ptr[c], len = colT_ptr[c + 1] - p0;
        if (len <= 1) continue;
        const int SP = pow2_at_least(len);
        if (SP > sp_max) continue;  // cannot happen: len <= nbmax
        for (int u = threadIdx.x; u < SP; u += blockDim.x) sbuf[u] = u < len ? rowT[p0 + u] : 0x7fffffff;
        __syncthreads();
        for (int kk = 2; kk <= SP; kk <<= 1)
            for (int jj = kk >> 1; jj > 0; jj >>= 1) {
                for (int u = threadIdx.x; u < SP; u += blockDim.x) {
                    const int v = u ^ jj;
                    if (v > u) {
                        const int a = sbuf[u], cc = sbuf[v];
                        const bool swap = ((u & kk) == 0) ? (a > cc) : (a < cc);
                        if (swap) {
                            sbuf[u] = cc;
                            sbuf[v] = a;
                        }
                    }
                }
                __syncthreads();
            }
        for (int u = threadIdx.x; u < len; u += blockDim.x) rowT[p0 + u] = sbuf[u];
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// host: launch the whole planner
// ---------------------------------------------------------------------------
prism_status scan_ints(const int *in, size_t n, int *out, int *tmp, cudaStream_t st) {
    const int nchunks = (int)((n + 1023) / 1024);
    k_scan_chunks<<<nchunks, 1024, 0, st>>>(in, (int)n, out, tmp);
    k_scan_totals<<<1, 1024, 0, st>>>(tmp, nchunks, out, (int)n);
    k_scan_add<<<nchunks, 1024, 0, st>>>(out, (int)n, tmp);
    PRISM_CUDA_OK(cudaGetLastError());
    return PRISM_OK;
}

size_t select_smem_bytes(const Plan &pl) { return sel_smem_layout(pl.g.D, pl.g.nbmax, pl.cap_stride).bytes; }

// Zone statistics of this plan's heads (their chunks of the layer's partials)
// and of the audio guidance.
prism_status launch_plan_stats(Plan &pl, const void *Vv, const float *a, cudaStream_t st) {
    const Geo &g = pl.g;
    const auto *V = static_cast<const __nv_bfloat16 *>(Vv);
    const int nchunk = (g.C + kStatChunk - 1) / kStatChunk;
    const size_t smem_v = 2 * 8 * 8 * kStatChunk * sizeof(float);
    { TimerScope ts(pl, kTZoneV, st);
    k_zone_stats_v<<<dim3(nchunk, g.M, g.batch), 128, smem_v, st>>>(V, g, pl.zone_part); }
    { TimerScope ts(pl, kTZoneA, st);
    k_zone_stats_a<<<dim3(g.M, g.batch), 512, 0, st>>>(a, g, pl.zone_a); }
    PRISM_CUDA_OK(cudaGetLastError());
    return PRISM_OK;
}

static prism_status launch_gather_select(Plan &pl, const __nv_bfloat16 *Q, const __nv_bfloat16 *K,
                                        const __nv_bfloat16 *V, cudaStream_t st);

prism_status launch_plan(Plan &pl, const void *Qv, const void *Kv, const void *Vv, const float *a,
                         cudaStream_t st) {
    if (pl.p.hilbert_block)  // fixed order and blocks: gather, pool, select
        return launch_gather_select(pl, static_cast<const __nv_bfloat16 *>(Qv),
                                    static_cast<const __nv_bfloat16 *>(Kv), static_cast<const __nv_bfloat16 *>(Vv), st);
    prism_status s = launch_plan_stats(pl, Vv, a, st);
    return s == PRISM_OK ? launch_plan_finish(pl, Qv, Kv, Vv, st) : s;
}

// Everything after the zone statistics (which hold every chunk of the layer
// by now): decisions, block table, permutation and pooling, selection, CSR/CSC.
prism_status launch_plan_finish(Plan &pl, const void *Qv, const void *Kv, const void *Vv, cudaStream_t st) {
    const Geo &g = pl.g;
    const auto *Q = static_cast<const __nv_bfloat16 *>(Qv);
    const auto *K = static_cast<const __nv_bfloat16 *>(Kv);
    const auto *V = static_cast<const __nv_bfloat16 *>(Vv);
    { TimerScope ts(pl, kTDecide, st);
    k_zone_decide<<<g.batch, 1024, 0, st>>>(g, pl.zone_part, pl.zone_a, pl.p.eps, pl.fixed_idx, false,
                                            pl.zone_B, pl.zone_shape, pl.zone_blk0, pl.nb, pl.blk_off,
                                            pl.tile_blk, pl.zone_qt0, pl.nqt, pl.qt_row, pl.qt_blk); }
    return launch_gather_select(pl, Q, K, V, st);
}

// The plan from decisions already in zone_B / zone_shape: block table, then
// as launch_plan_finish.
prism_status launch_plan_given(Plan &pl, const void *Qv, const void *Kv, const void *Vv, cudaStream_t st) {
    const Geo &g = pl.g;
    { TimerScope ts(pl, kTDecide, st);
    k_zone_decide<<<g.batch, 1024, 0, st>>>(g, pl.zone_part, pl.zone_a, pl.p.eps, pl.fixed_idx, true,
                                            pl.zone_B, pl.zone_shape, pl.zone_blk0, pl.nb, pl.blk_off,
                                            pl.tile_blk, pl.zone_qt0, pl.nqt, pl.qt_row, pl.qt_blk); }
    PRISM_CUDA_OK(cudaGetLastError());
    return launch_gather_select(pl, static_cast<const __nv_bfloat16 *>(Qv), static_cast<const __nv_bfloat16 *>(Kv),
                                static_cast<const __nv_bfloat16 *>(Vv), st);
}

static void launch_permute_pool(Plan &pl, const __nv_bfloat16 *Q, const __nv_bfloat16 *K, const __nv_bfloat16 *V,
                                cudaStream_t st) {
    const Geo &g = pl.g;
    TimerScope ts(pl, kTPermutePool, st);
    if (pl.p.hilbert_block)
        k_permute_pool<true><<<dim3((g.C / 8 + kPPThreads - 1) / kPPThreads * g.nbmax, g.batch), kPPThreads, 0, st>>>(
            Q, K, V, g, pl.nb, pl.blk_off, pl.zone_shape, pl.perm, pl.Qp, pl.Kp, pl.Vp, pl.Qbar, pl.Kbar);
    else
        k_permute_pool<false><<<dim3((g.C / 8 + kPPThreads - 1) / kPPThreads * g.nbmax, g.batch), kPPThreads, 0, st>>>(
            Q, K, V, g, pl.nb, pl.blk_off, pl.zone_shape, pl.perm, pl.Qp, pl.Kp, pl.Vp, pl.Qbar, pl.Kbar);
}

// The block-contiguous copies and pooled means, then scores, selection and
// the CSR / CSC (the block table is in place).
static prism_status launch_gather_select(Plan &pl, const __nv_bfloat16 *Q, const __nv_bfloat16 *K,
                                        const __nv_bfloat16 *V, cudaStream_t st) {
    const Geo &g = pl.g;
    launch_permute_pool(pl, Q, K, V, st);
    PRISM_CUDA_OK(cudaGetLastError());
    const size_t rows = (size_t)g.batch * g.heads * g.nbmax;
    {
        // scores and selection, a group of heads at a time (the score scratch
        // holds score_group heads of N_b x N_b keys); one timer record per launch
        const int BH = g.batch * g.heads;
        const int nt = (g.nbmax + kScoreTile - 1) / kScoreTile;
        for (int bh0 = 0; bh0 < BH; bh0 += pl.score_group) {
            const int G = BH - bh0 < pl.score_group ? BH - bh0 : pl.score_group;
            {
                TimerScope ts(pl, kTSelect, st);
                k_scores<<<dim3(nt, nt, G), 256, 0, st>>>(g, pl.nb, pl.Qbar, pl.Kbar, bh0, pl.score_keys);
            }
            {
                TimerScope ts(pl, kTSelect, st);
                k_select<<<dim3(g.nbmax, G), kSelThreads, select_smem_bytes(pl), st>>>(
                    g, pl.nb, pl.score_keys, bh0, pl.p.top_k, (double)pl.p.top_p, pl.p.max_frac, pl.cap_stride,
                    pl.cnt, pl.cols_pad);
            }
        }
    }
    PRISM_CUDA_OK(cudaGetLastError());
    TimerScope ts_csr(pl, kTCsr, st);
    prism_status s = scan_ints(pl.cnt, rows, pl.row_ptr, pl.scan_tmp, st);
    if (s != PRISM_OK) return s;
    PRISM_CUDA_OK(cudaMemsetAsync(pl.colT_cursor, 0, rows * sizeof(int), st));
    k_csr_compact<<<1184, 256, 0, st>>>(g, pl.cap_stride, pl.cnt, pl.cols_pad, pl.row_ptr, pl.col, pl.colT_cursor);
    PRISM_CUDA_OK(cudaGetLastError());
    s = scan_ints(pl.colT_cursor, rows, pl.colT_ptr, pl.scan_tmp, st);
    if (s != PRISM_OK) return s;
    PRISM_CUDA_OK(cudaMemsetAsync(pl.colT_cursor, 0, rows * sizeof(int), st));
    k_csc_fill<<<1184, 256, 0, st>>>(g, pl.row_ptr, pl.col, pl.colT_ptr, pl.colT_cursor, pl.rowT);
    const int sp_max = pow2_at_least(g.nbmax);
    k_csc_sort<<<4 * 1184, 256, sp_max * sizeof(int), st>>>(rows, pl.colT_ptr, pl.rowT, sp_max);
    PRISM_CUDA_OK(cudaGetLastError());
    return PRISM_OK;
}

prism_status configure_plan_kernels(const Plan &pl) {
    PRISM_CUDA_OK(cudaFuncSetAttribute(k_zone_stats_v, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       2 * 8 * 8 * kStatChunk * (int)sizeof(float)));
    PRISM_CUDA_OK(cudaFuncSetAttribute(k_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)select_smem_bytes(pl)));
    const int sp_max = pow2_at_least(pl.g.nbmax);
    PRISM_CUDA_OK(cudaFuncSetAttribute(k_csc_sort, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       sp_max * (int)sizeof(int)));
    return upload_shape_table();
}

// Re-gathers new Q, K, V into the plan's block-contiguous copies with the
// plan's existing block table (the selection is kept; the refreshed pooled
// keys feed only the Taylor forward).
prism_status launch_regather(Plan &pl, const void *Qv, const void *Kv, const void *Vv, cudaStream_t st) {
    launch_permute_pool(pl, static_cast<const __nv_bfloat16 *>(Qv), static_cast<const __nv_bfloat16 *>(Kv),
                        static_cast<const __nv_bfloat16 *>(Vv), st);
    PRISM_CUDA_OK(cudaGetLastError());
    return PRISM_OK;
}

// Zone statistics and volume / shape decisions alone, on caller-provided
// buffers (used by the allocation-free entry point).  Scratch arrays are laid
// out by the caller; the kernels are the planner's own.
prism_status launch_zone_decisions(const Geo &g, double eps, int fixed_idx, const __nv_bfloat16 *V, const float *a,
                                   double *zone_part, double *zone_a, int *zone_B, int *zone_shape, int *zone_blk0,
                                   int *nb, int *blk_off, int *tile_blk, int *zone_qt0, int *nqt, int *qt_row,
                                   int *qt_blk, cudaStream_t st) {
    const int nchunk = (g.C + kStatChunk - 1) / kStatChunk;
    const size_t smem_v = 2 * 8 * 8 * kStatChunk * sizeof(float);
    k_zone_stats_v<<<dim3(nchunk, g.M, g.batch), 128, smem_v, st>>>(V, g, zone_part);
    k_zone_stats_a<<<dim3(g.M, g.batch), 512, 0, st>>>(a, g, zone_a);
    k_zone_decide<<<g.batch, 1024, 0, st>>>(g, zone_part, zone_a, eps, fixed_idx, false, zone_B, zone_shape,
                                            zone_blk0, nb, blk_off, tile_blk, zone_qt0, nqt, qt_row, qt_blk);
    PRISM_CUDA_OK(cudaGetLastError());
    return PRISM_OK;
}

// Kernel attributes and the candidate table for launch_zone_decisions.
prism_status configure_zone_kernels() {
    PRISM_CUDA_OK(cudaFuncSetAttribute(k_zone_stats_v, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       2 * 8 * 8 * kStatChunk * (int)sizeof(float)));
    return upload_shape_table();
}

}  // namespace prism
