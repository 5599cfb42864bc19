// prism_internal.cuh -- shared declarations of the CUDA library (not part of
// the C ABI).  Layout of every internal buffer is documented in the plan
// struct below.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/prism.h"

namespace prism {

constexpr int kZone = 8;           // macro-zone edge [Prism guide, core ideas, bullet 1]
constexpr int kZoneVol = 512;
constexpr int kTile = 64;          // every block is a multiple of 64 tokens
constexpr int kStatChunk = 128;    // channels per zone-statistics CTA
constexpr int kNumShapes = 16;

enum TimerId {
    kTZoneV = 0, kTZoneA, kTDecide, kTPermutePool, kTSelect, kTCsr, kTAttnFwd, kTBwdPre, kTAttnBwd, kTDqFinal,
    kTTaylorPool, kTAttnFwdTaylor, kTCount
};
static_assert(kTCount == PRISM_NUM_TIMERS, "timer count");

struct TimerState;  // event pools, defined in prism_api.cu
struct HostPipe;    // host-buffer step pipeline, defined in host_pipeline.cu

// Per-launch problem geometry, passed by value to kernels.
struct Geo {
    int batch, T, H, W, heads, D;
    int N, M, MT, MH, MW, nbmax, C;  // C = heads * D: the channels this plan holds
    // Zone statistics are kept per 128-channel chunk of the whole layer
    // (heads_total * D channels, Ctot); this plan's heads are chunks
    // [chunk0, chunk0 + C / 128) of nchunk_tot.  Unsharded: Ctot = C, chunk0 = 0.
    int Ctot, chunk0, nchunk_tot;
};

// Everything a plan owns (device pointers unless noted).
struct Plan {
    prism_params p;
    Geo g;
    int fixed_idx;          // table index of the fixed shape, -1 = dynamic
    int cap_stride;         // worst-case selected blocks per row
    int device;
    bool have_fwd;
    bool built;
    bool have_stats;        // zone statistics computed since the last finished build
    // zone statistics and decisions
    double *zone_part;      // [nchunk_tot][batch][M][3] per 128-channel chunk: sum_c of directional variances
    double *zone_a;         // [batch][M][5]  sigma2_a T,H,W, mean a, max a
    int *zone_B;            // [batch][M]
    int *zone_shape;        // [batch][M]
    int *zone_blk0;         // [batch][M+1]  first block of each zone
    int *nb;                // [batch]
    int *blk_off;           // [batch][nbmax+1]
    int *tile_blk;          // [batch][nbmax]  64-row tile -> block
    int *zone_qt0;          // [batch][M+1]  first 128-row query tile of each zone
    int *nqt;               // [batch]       number of 128-row tiles (query tiles of the
                            //               forward, key tiles of the backward)
    int *qt_row;            // [batch][nbmax] first block-contiguous row of each tile
    int *qt_blk;            // [batch][nbmax] block of each tile; ~j for a tile holding the
                            //               two 64-token blocks j and j+1
    int *perm;              // [batch][N]  block-contiguous position -> raster token
    // permuted head-major inputs and pooled blocks
    __nv_bfloat16 *Qp, *Kp, *Vp;   // [batch*heads][N][D]
    double *Qbar, *Kbar;           // [batch*heads][nbmax][D]
    __nv_bfloat16 *Kb, *Vb;        // [batch*heads][nbmax][D] bf16 pooled keys / mean values (Taylor term),
                                   // zeroed at creation so rows past a build's last block stay finite
    // selection
    unsigned long long *score_keys;  // [score_group][nbmax][nbmax] order-preserving score keys
    int score_group;        // heads scored per pass
    int *cnt;               // [batch*heads*nbmax]
    int *cols_pad;          // [batch*heads*nbmax][cap_stride]
    int *row_ptr;           // [rows+1]
    int *col;               // [rows*cap_stride]
    int *colT_ptr;          // [rows+1]   CSC over (b*heads+h)*nbmax + j
    int *rowT;              // [rows*cap_stride]
    int *colT_cursor;       // [rows]
    int *scan_tmp;          // block partial sums for scans
    // attention statistics / backward scratch
    float *nlse_p;          // [batch*heads][N] minus the log2-unit LSE of the scaled scores, permuted order
    __nv_bfloat16 *dOp;     // [batch*heads][N][D]
    float *delta;           // [batch*heads][N]
    float *dQacc;           // [batch*heads][N][D]
    int *status;            // device error word (0 = ok)
    int *host_nb;           // pinned host copy of nb
    TimerState *timers;     // NULL unless timing is on
    HostPipe *pipe;         // NULL until the first host-buffer step
    // TMA descriptors of the permuted copies, viewed as [batch*heads*N][D] bf16
    CUtensorMap tmQ, tmK, tmV, tmdO;
    CUtensorMap tmKb, tmVb;  // the pooled bf16 copies, viewed as [batch*heads*nbmax][D]
    CUtensorMap tmdQ;       // fp32 [batch*heads*N][D], 64-row boxes, reduce-add target
};

// Records CUDA events around the launches in its scope when timing is on.
struct TimerScope {
    Plan &pl;
    int id;
    cudaStream_t st;
    TimerScope(Plan &p, int i, cudaStream_t s);
    ~TimerScope();
};

#define PRISM_CUDA_OK(call)                                                       \
    do {                                                                          \
        cudaError_t e_ = (call);                                                  \
        if (e_ != cudaSuccess) return prism::fail_cuda(e_, #call, __FILE__, __LINE__); \
    } while (0)

prism_status fail(prism_status s, const char *fmt, ...);
prism_status fail_cuda(cudaError_t e, const char *what, const char *file, int line);

// Launchers (each returns PRISM_OK or an error after checking the launch).
prism_status launch_plan(Plan &pl, const void *Q, const void *K, const void *V, const float *a,
                         cudaStream_t st);
prism_status launch_plan_stats(Plan &pl, const void *V, const float *a, cudaStream_t st);
prism_status launch_plan_finish(Plan &pl, const void *Q, const void *K, const void *V, cudaStream_t st);
prism_status launch_plan_given(Plan &pl, const void *Q, const void *K, const void *V, cudaStream_t st);
prism_status launch_attn_fwd_tc(Plan &pl, void *O, float *lse, cudaStream_t st);
prism_status launch_attn_fwd_taylor(Plan &pl, void *O, float *lse, cudaStream_t st);
bool taylor_fits(const Geo &g);  // the Taylor forward's shared memory fits one CTA
prism_status launch_regather(Plan &pl, const void *Q, const void *K, const void *V, cudaStream_t st);
prism_status make_tensor_maps(Plan &pl);
prism_status launch_attn_bwd_tc_main(Plan &pl, void *dK, void *dV, cudaStream_t st);
prism_status launch_attn_bwd(Plan &pl, const void *O, const void *dO, void *dQ, void *dK, void *dV,
                             cudaStream_t st);

prism_status launch_audio_norms(const void *h, float *a, long long rows, int C, cudaStream_t st);

// Exclusive scan of n ints into out[0..n] (out[n] = total); tmp holds
// (n + 1023) / 1024 + 1 ints.
prism_status scan_ints(const int *in, size_t n, int *out, int *tmp, cudaStream_t st);

// Hilbert-order fixed-block plans (hilbert_plan.cu): the curve's level k
// (2^k >= T, H, W) and the one-time order and block tables of a new plan.
int hilbert_level(const Geo &g);
prism_status setup_hilbert_plan(Plan &pl);

// Host-buffer steps (host_pipeline.cu).
prism_status host_step(Plan &pl, const prism_host_io &io, cudaStream_t user, unsigned long long *ticket);
prism_status host_step_join(Plan &pl, unsigned long long ticket, cudaStream_t st);
prism_status host_step_wait(Plan &pl, unsigned long long ticket);
void release_host_pipe(Plan &pl);

__host__ __device__ inline int cap_for(int nb, int k, float max_frac) {
    if (!(max_frac > 0.0f)) return nb;
    int c = (int)floor((double)max_frac * (double)nb);
    if (c < k) c = k;
    if (c > nb) c = nb;
    return c;
}

}  // namespace prism
