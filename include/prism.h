/*
 * prism.h -- C ABI of the B200 (sm_100a) implementation of Prism's dynamic
 * sparse video self-attention hot path.
 *
 * Source of the method: paper guide "Prism: Dynamic Sparse Attention cho Huan
 * luyen Mo hinh Tao Video-Am thanh Dong thoi Do phan giai Goc 2K" (xyznot.com,
 * paper 2610.05416), cited as [Prism guide, <section>].
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Plain C types only.  "device" pointers are CUDA global-memory addresses of
 *   the device that was current when the plan was created; "host" pointers are
 *   ordinary CPU memory.  `stream` is a cudaStream_t passed as void* (NULL =
 *   the legacy default stream).
 * - Tensor layouts (row-major, no padding):
 *     Q, K, V, O, dO, dQ, dK, dV : bf16 [batch][N][heads][head_dim]
 *     a_norm                     : fp32 [batch][T][H][W]
 *     lse                        : fp32 [batch][heads][N]
 *   with N = T*H*W and tokens in raster order n = (t*H + h)*W + w.
 * - Ownership: the caller owns every tensor argument and the stream.  The plan
 *   owns its internal device buffers (permuted copies, pooled tensors, block
 *   CSR and CSC, softmax statistics) and frees them in prism_plan_destroy.
 * - Errors: every call returns a prism_status; no exception crosses the ABI.
 *   Argument errors are detected on the host before any launch.  Launch
 *   failures return PRISM_ERR_CUDA.  prism_last_error() gives a message for
 *   the calling thread's last failure.
 * - Synchronisation: prism_plan_build, prism_attn_fwd and prism_attn_bwd only
 *   enqueue work on `stream`; they never wait for the device.  Calls on one
 *   plan must be ordered on one stream (or by the caller's events).
 *   prism_plan_view and prism_plan_check synchronise the stream they are given.
 */
#ifndef PRISM_H
#define PRISM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PRISM_API __attribute__((visibility("default")))
#else
#define PRISM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum prism_status {
    PRISM_OK = 0,
    PRISM_ERR_INVALID_ARG = 1,  /* a NULL pointer, a size out of range        */
    PRISM_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. odd grid)   */
    PRISM_ERR_CUDA = 3,         /* a CUDA call or kernel launch failed         */
    PRISM_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up          */
    PRISM_ERR_NOMEM = 5,        /* device allocation failed                    */
    PRISM_ERR_STATE = 6         /* call out of order (e.g. bwd before fwd)     */
} prism_status;

/* Problem description.
 * T, H, W: latent grid, each a positive multiple of 8 (the 8x8x8 macro-zone,
 *   [Prism guide, core ideas, bullet 1]).
 * heads, head_dim: head_dim is 64 or 128.
 * top_k >= 1, 0 < top_p <= 1: hybrid selection S_i = Top-k U Top-p
 *   [Prism guide, Method section 3].
 * max_frac: 0 means no per-row cap; otherwise a query block keeps at most
 *   max(top_k, floor(max_frac * N_b)) key blocks (N_b = number of blocks).
 * fixed_shape: {0,0,0} selects the dynamic shape of every zone
 *   [Prism guide, Method sections 1-2]; otherwise every zone uses this edge
 *   triple, which must be one of the 16 candidates (edges in {2,4,8}).
 * eps: the epsilon of the indicator g_d (1e-6 when <= 0 is given).
 * heads_total, head_offset: head sharding.  0, 0 (or heads_total == heads)
 *   = the plan holds every head of the layer.  Otherwise the plan holds
 *   heads [head_offset, head_offset + heads) of heads_total, Q/K/V carry only
 *   those heads, and the plan is built in two halves around one exchange of
 *   zone statistics between the ranks (prism_plan_build_stats,
 *   prism_plan_stats_slice, prism_plan_build_finish); heads * head_dim and
 *   head_offset * head_dim must be multiples of 128.  (A Hilbert-order plan
 *   needs no exchange: it is built with prism_plan_build on any shard.)
 * hilbert_block: 0 = Prism's zone plan.  64, 128 or 256 = the comparison
 *   baseline of the DFSAttn page's first component: tokens ordered along
 *   the 3D Hilbert curve of the smallest 2^k cube holding the grid (Skilling's
 *   index, t before h before w; the grid's tokens in the cube's curve order),
 *   blocks of hilbert_block consecutive tokens of that order, then Prism's
 *   pooled scoring, selection and attention.  No zone statistics: a_norm and
 *   fixed_shape are unused (fixed_shape must be {0,0,0}); the grid's longest
 *   side must be at most 512.  The order is computed once by
 *   prism_plan_create (which then synchronises the device).                */
typedef struct prism_params {
    int batch, T, H, W, heads, head_dim;
    int top_k;
    float top_p;
    float max_frac;
    int fixed_shape[3];
    double eps;
    int heads_total, head_offset;
    int hilbert_block;
} prism_params;

typedef struct prism_plan prism_plan;

/* Read-only device views of a built plan (all arrays are device memory of
 * the plan; valid until the next prism_plan_build or prism_plan_destroy).
 * NBMAX = N/64 is the most blocks a sample can have; every per-block array is
 * sized for it, entries past a sample's n_blocks are unspecified.
 *   zone_B      int [batch][N/512]      block volume B(m) in {64,128,256}
 *                                       (0 in a Hilbert-order plan)
 *   zone_shape  int [batch][N/512]      (-1 in a Hilbert-order plan)
 *                                       index into the 16-entry candidate
 *                                       table (volume 64: 0-6, 128: 7-12,
 *                                       256: 13-15; lexicographic (bT,bH,bW))
 *   perm        int [batch][N]          perm[n_new] = raster index of the
 *                                       token stored at block-contiguous
 *                                       position n_new
 *   blk_off     int [batch][NBMAX+1]    first block-contiguous position of
 *                                       each block; blk_off[n_blocks] = N
 *   row_ptr     int [batch*heads*NBMAX+1]  block CSR over rows
 *                                       r = (b*heads + h)*NBMAX + i
 *   col_idx     int [nnz]               selected key blocks, ascending per row
 *   n_blocks    host copy, one per sample (first `batch` entries)          */
typedef struct prism_plan_view {
    const int *zone_B, *zone_shape, *perm, *blk_off, *row_ptr, *col_idx;
    int nbmax;
    long long nnz;
    int n_blocks[64];
} prism_plan_view;

/* Allocates a plan and all of its device buffers for the worst case
 * (N/64 blocks per sample).  Validates params.  *out receives the plan.    */
PRISM_API prism_status prism_plan_create(const prism_params *params, prism_plan **out);

/* Device bytes a plan with these params holds (0 on invalid params).      */
PRISM_API size_t prism_plan_bytes(const prism_params *params);

/* Builds the plan from one batch of inputs [Prism guide, Method sections
 * 1-3]: per-zone statistics and the indicator g_d from V and a_norm, block
 * volume and shape, the block-contiguous permutation (Q, K, V are gathered
 * into the plan's head-major permuted copies), mean-pooled Q and K per block,
 * pooled block scores and the hybrid Top-k U Top-p key-block CSR and its
 * transpose.  Q, K, V, a_norm: device, layouts above; read only.            */
PRISM_API prism_status prism_plan_build(prism_plan *plan, const void *Q, const void *K, const void *V,
                              const float *a_norm, void *stream);

/* The plan build in two halves, for head-sharded plans (one rank per GPU,
 * each holding some heads of the layer).  The zone decisions need the
 * statistics of every channel of the layer; after the decisions the heads are
 * independent [Prism guide, Method sections 1-3].
 *   prism_plan_build_stats: zone statistics of this plan's heads (V, device,
 *     [batch][N][heads][head_dim]) and of a_norm.
 *   prism_plan_stats_slice: the plan's device buffer of per-chunk zone
 *     statistics of the whole layer (*buf, *total_bytes) and this plan's
 *     slice of it (*slice_offset bytes in, *slice_bytes long).  Slices are
 *     contiguous and ordered by head, so with ranks holding equal consecutive
 *     head ranges one all-gather (each rank sending its slice, receiving the
 *     whole buffer in rank order) gives every rank the layer's statistics.
 *     The buffer belongs to the plan.
 *   prism_plan_build_finish: decisions, permutation and pooling, selection,
 *     CSR / CSC from the (complete) statistics, Q, K, V of this plan's heads.
 * Every rank computes the same zone shapes and permutation, bit for bit the
 * ones an unsharded plan of the whole layer computes.  prism_plan_build is
 * build_stats followed by build_finish and is refused (PRISM_ERR_STATE) for a
 * sharded plan, as is prism_step_host.                                     */
PRISM_API prism_status prism_plan_build_stats(prism_plan *plan, const void *V, const float *a_norm, void *stream);
PRISM_API prism_status prism_plan_stats_slice(prism_plan *plan, void **buf, size_t *slice_offset, size_t *slice_bytes,
                                              size_t *total_bytes);
PRISM_API prism_status prism_plan_build_finish(prism_plan *plan, const void *Q, const void *K, const void *V,
                                               void *stream);

/* Builds the plan from zone decisions the caller gives instead of the zone
 * statistics [Prism guide, Method section 2: each zone's block volume B(m)
 * and block shape; this call takes them as inputs and performs the rest of
 * the plan]: the block table, the permutation and pooling, the selection and
 * the CSR / CSC, exactly as prism_plan_build does after its own decisions.
 *   zone_B      host int [batch][N/512]: 64, 128 or 256
 *   zone_shape  host int [batch][N/512]: index into the 16-entry candidate
 *               table (see prism_plan_view) whose volume is zone_B
 *   Q, K, V     device, as prism_plan_build (16-byte aligned)
 * Both host arrays are read before the call returns (the caller keeps them;
 * being pageable host memory, their copy may wait for work already queued on
 * the stream).
 * fixed_shape is not applied; a head-sharded plan needs no statistics
 * exchange on this path.  Errors: PRISM_ERR_INVALID_ARG for a NULL or
 * misaligned pointer or an entry outside the table (message names the zone),
 * PRISM_ERR_STATE for a Hilbert-order plan (it has no zones).  Use: stage-wise
 * checks of the downstream steps, and decisions computed once for several
 * layers.                                                                    */
PRISM_API prism_status prism_plan_build_with_zones(prism_plan *plan, const void *Q, const void *K, const void *V,
                                                   const int *zone_B, const int *zone_shape, void *stream);

/* Plan reuse: gathers new Q, K, V (device, layouts above) into the plan's
 * block-contiguous copies using the plan's existing zone shapes, permutation
 * and selection, which are not recomputed.  Subsequent prism_attn_fwd /
 * prism_attn_bwd attend with the new inputs under the cached plan -- the
 * reuse of a sparsity plan across diffusion steps or layers that the DFSAttn
 * page describes as adaptive mask caching (its third component).  Returns
 * PRISM_ERR_STATE before the first prism_plan_build.                       */
PRISM_API prism_status prism_plan_update_qkv(prism_plan *plan, const void *Q, const void *K, const void *V,
                                             void *stream);

/* Sparse attention forward over the selected blocks of the last build
 * [Prism guide, Method section 3, last sentence]: each query token of block
 * i attends under one online softmax to every token of the key blocks in
 * S_i.  Reads the permuted Q, K, V of the last build or update.  Writes O (device,
 * bf16, user layout) and, if lse != NULL, the natural-log log-sum-exp of the
 * scaled scores (device, fp32 [batch][heads][N], raster token order).  The
 * plan keeps its own copy of the statistics for prism_attn_bwd.           */
PRISM_API prism_status prism_attn_fwd(prism_plan *plan, void *O, float *lse, void *stream);

/* Forward with a zeroth-order Taylor term for the key blocks outside S_i
 * [In-Context Sparse Attention article, grouped computation: the flat path
 * scores block-mean keys and keeps the zeroth-order term of the
 * exponential].  The blocks of S_i enter exactly, as in prism_attn_fwd; each
 * other key block j enters once, through its mean key kbar_j and mean value
 * vbar_j (both rounded to bf16), as if all |B_j| of its tokens scored
 * q.kbar_j / sqrt(D):
 *   O_q = (sum_{t in S_i} e^{s_qt} v_t + sum_{j not in S_i} |B_j| e^{q.kbar_j/sqrt D} vbar_j)
 *         / (the same sums without v).
 * Same arguments, layouts and errors as prism_attn_fwd; lse (optional) is
 * the log of the whole denominator.  Reads the plan's pooled keys and its
 * permuted V of the last build or update; enqueues a pooling kernel and the
 * attention kernel.  It leaves the statistics that prism_attn_bwd uses
 * untouched: the backward differentiates the sparse forward only.
 * PRISM_ERR_UNSUPPORTED when the per-CTA table of key blocks (one byte
 * each) does not fit a CTA's shared memory (more than about 128 thousand
 * blocks, i.e. over 8 million tokens per sample).                          */
PRISM_API prism_status prism_attn_fwd_taylor(prism_plan *plan, void *O, float *lse, void *stream);

/* Gradient of sum(O * dO) with respect to Q, K, V through the same sparse
 * attention (the plan and the forward's statistics are reused).  The pages
 * define no such call: it is the standard softmax-attention gradient taken
 * over the selected blocks S_i only [Prism guide, Method section 3 restricts
 * the attention to S_i; the model is trained through it]:
 *   P = exp(S/sqrt(D) - LSE), dV = P^T dO, dP = dO V^T,
 *   dS = P (dP - rowsum(dO * O)), dQ = dS K / sqrt(D), dK = dS^T Q / sqrt(D).
 * O is the forward's output and dO the incoming gradient (device, bf16, user
 * layout); dQ, dK, dV are written (device, bf16, user layout).  dQ is summed
 * in fp32 before its bf16 rounding.  Repeated calls on the same plan and
 * inputs give bit-identical dK and dV (their fp32 sums are formed in one
 * order); dQ's partial sums from different key tiles are added in the order
 * they arrive, so dQ can differ in its last bit.  Returns PRISM_ERR_STATE if
 * no forward ran since the last build.                                     */
PRISM_API prism_status prism_attn_bwd(prism_plan *plan, const void *O, const void *dO, void *dQ, void *dK,
                            void *dV, void *stream);

/* Audio guidance for the plan: a[b][t][h][w] = || h^[b][n][:] ||_2, the L2
 * norm over `channels` of the audio-to-video cross-attention output of video
 * token n = (t*H + h)*W + w [Prism guide, Method section 1, the sentence
 * before the g_d equation]; a layer computes it after its cross-attention and
 * the next layer's prism_plan_build takes it as a_norm.  h: device, bf16
 * [batch][T*H*W][channels], read only; a: device, fp32 [batch][T][H][W],
 * written.  The caller owns both.  Sums of squares in fp32 (relative error
 * of a below 1e-5 for channels <= 65536).  Enqueues one kernel on `stream`
 * on the current device; no plan is needed.  PRISM_ERR_INVALID_ARG for NULL
 * pointers, dimensions < 1 or channels outside [1, 2^20].                  */
PRISM_API prism_status prism_audio_norms(const void *h, float *a, int batch, int T, int H, int W, int channels,
                                         void *stream);

/* One layer step from HOST buffers: copy the inputs to the device, build the
 * plan, run the forward and (when dO is given) the backward, and copy the
 * outputs back -- the same computation as prism_plan_build + prism_attn_fwd
 * + prism_attn_bwd on device tensors.  The pages define no such call; it is
 * the runtime that feeds the hot path from host memory.
 *
 * Every field is a HOST pointer in the layouts above; the caller owns all of
 * them.  Q, K, V, a_norm, O are required; lse may be NULL; dO == NULL means
 * forward only, otherwise dQ, dK, dV are required.  Page-locked buffers
 * (cudaHostAlloc / cudaHostRegister) let the copies run asynchronously;
 * pageable ones work but their copies are not overlapped.
 *
 * prism_step_host only enqueues work and returns *ticket (1, 2, ...).  The
 * plan runs steps on three streams of its own -- host->device copies into
 * one of two device staging sets, the plan + attention kernels, and
 * device->host copies -- so the copies of one step overlap the kernels of
 * the next and the previous one.  The step's first copy waits for the work
 * enqueued on `stream` before the call.  The caller must leave the input
 * buffers unchanged, and must not read the output buffers, until the step has
 * completed: prism_step_wait blocks the host until then; prism_step_join makes
 * `stream` wait for it on the device.  At most 8 steps are in flight: the
 * ninth call first waits on the host for the first one.  Staging buffers are
 * allocated on the first step that needs them: two sets of the inputs and
 * outputs used (2 x 9 bf16 tensors of batch*N*heads*head_dim at most) and
 * freed with the plan.  Do not interleave host steps with the device-pointer
 * calls on one plan without prism_step_wait in between: both use the plan's
 * internal buffers.  PRISM_ERR_INVALID_ARG for a NULL required field, for
 * taylor with dO, or a ticket that was never issued.                        */
typedef struct prism_host_io {
    const void *Q, *K, *V;  /* bf16, host                                     */
    const float *a_norm;    /* fp32, host                                     */
    const void *dO;         /* bf16, host; NULL = forward only                */
    void *O;                /* bf16, host, written                            */
    float *lse;             /* fp32, host, written; may be NULL               */
    void *dQ, *dK, *dV;     /* bf16, host, written when dO != NULL            */
    int taylor;             /* nonzero: the forward of prism_attn_fwd_taylor  */
                            /* (forward-only steps: dO must be NULL)          */
} prism_host_io;
PRISM_API prism_status prism_step_host(prism_plan *plan, const prism_host_io *io, void *stream,
                                       unsigned long long *ticket);
PRISM_API prism_status prism_step_join(prism_plan *plan, unsigned long long ticket, void *stream);
PRISM_API prism_status prism_step_wait(prism_plan *plan, unsigned long long ticket);

/* Synchronises `stream`, then fills *view (device pointers + host n_blocks).*/
PRISM_API prism_status prism_plan_view_get(prism_plan *plan, prism_plan_view *view, void *stream);

/* Synchronises `stream` and reports a device-side error recorded by a
 * kernel of this plan (PRISM_ERR_TIMEOUT for a bounded wait that gave up),
 * then clears it.                                                          */
PRISM_API prism_status prism_plan_check(prism_plan *plan, void *stream);

/* Diagnostic of the failure path: enqueues one thread that waits on a
 * device barrier nothing arrives on, through the same bounded wait the
 * attention kernels use.  It gives up after its poll limit (about a second)
 * and records a timeout in the plan's status word,
 * so the next prism_plan_check returns PRISM_ERR_TIMEOUT; while the word is
 * set, the plan's attention kernels return at once.  No fault, no hang.   */
PRISM_API prism_status prism_plan_selftest_timeout(prism_plan *plan, void *stream);

/* Optional per-kernel timing with CUDA events recorded on the launch stream
 * around every kernel of the plan (off by default; adds two event records
 * per launch).  prism_plan_read_timing waits for the recorded events, writes
 * for each timer id the summed milliseconds and the number of launches since
 * the previous read (arrays of PRISM_NUM_TIMERS host entries), and resets.
 * Timer ids and names: prism_timer_name(id).                               */
#define PRISM_NUM_TIMERS 12
PRISM_API prism_status prism_plan_set_timing(prism_plan *plan, int enable);
PRISM_API prism_status prism_plan_read_timing(prism_plan *plan, float *total_ms, int *launches);
PRISM_API const char *prism_timer_name(int id);

/* Allocation-free variant of the planner's first stage (per-zone statistics,
 * density, block volume B(m) and shape), for callers that cannot call
 * cudaMalloc: an application whose caching allocator owns all device memory,
 * or a loop that cannot afford cudaMalloc's implicit device synchronisation.
 * The paper has no counterpart of this entry point; it writes the same
 * zone_B / zone_shape that prism_plan_build computes (see prism_plan_view).
 * Reads params' batch, grid, heads, head_dim, fixed_shape and eps; V (device,
 * bf16 [batch][N][heads][head_dim]) and a_norm (device, fp32 [batch][T][H][W]).
 * Writes zone_B and zone_shape (device, int [batch][N/512], caller-owned).
 * Scratch comes from one fixed device array of PRISM_NOALLOC_SCRATCH_BYTES
 * compiled into the library, which every GPU that loads the library holds
 * until the process exits; a problem needing more (about
 * 24 * batch * N/512 * ceil(heads*head_dim/128) bytes plus 20 bytes per 64
 * tokens) returns PRISM_ERR_UNSUPPORTED before anything is launched.  The
 * first call in a CUDA context (per device; again after cudaDeviceReset has
 * replaced the device's primary context) looks up the array's device address,
 * sets kernel attributes and uploads a small constant table; make that first
 * call before any stream capture.  params' heads_total must be 0 or heads and
 * head_offset 0 (the whole layer; no head shards).  All calls
 * share the array (nothing in it has to start at zero), so calls whose work
 * overlaps on the GPU (other streams or host threads) race: order them.
 * Only enqueues work on `stream`.                                          */
#define PRISM_NOALLOC_SCRATCH_BYTES (4u << 20)
PRISM_API prism_status prism_zone_shapes_noalloc(const prism_params *params, const void *V, const float *a_norm,
                                                 int *zone_B, int *zone_shape, void *stream);

/* Frees the plan and its device buffers (NULL is ignored).                 */
PRISM_API void prism_plan_destroy(prism_plan *plan);

/* Message of the calling thread's last failed call ("" if none).          */
PRISM_API const char *prism_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* PRISM_H */
