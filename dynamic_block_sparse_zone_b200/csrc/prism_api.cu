// prism_api.cu -- the C ABI declared in include/prism.h: parameter checks,
// plan allocation and the three hot-path calls.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <new>
#include <string>
#include <utility>
#include <vector>

#include "prism_internal.cuh"

namespace prism {

static thread_local std::string g_last_error;

prism_status fail(prism_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

prism_status fail_cuda(cudaError_t e, const char *what, const char *file, int line) {
    const prism_status s = (e == cudaErrorMemoryAllocation) ? PRISM_ERR_NOMEM : PRISM_ERR_CUDA;
    return fail(s, "%s failed: %s (%s:%d)", what, cudaGetErrorString(e), file, line);
}

int host_shape_table(int (*e)[3]);
prism_status configure_plan_kernels(const Plan &pl);
prism_status configure_attn_tc_kernels();
prism_status configure_attn_bwd_tc_kernels();
prism_status launch_selftest_bounded_wait(Plan &pl, cudaStream_t st);
size_t select_smem_bytes(const Plan &pl);

static int log2_exact(int x) {
    for (int k = 0; k < 31; ++k)
        if ((1 << k) == x) return k;
    return -1;
}

// Validates params and fills geometry; returns PRISM_OK or an error with a message.
static prism_status check_params(const prism_params *p, Geo *g, int *fixed_idx, int *cap_stride) {
    if (!p) return fail(PRISM_ERR_INVALID_ARG, "params is NULL");
    if (p->batch < 1 || p->batch > 64) return fail(PRISM_ERR_INVALID_ARG, "batch must be in [1, 64]");
    if (p->T <= 0 || p->H <= 0 || p->W <= 0) return fail(PRISM_ERR_INVALID_ARG, "grid sizes must be positive");
    if (p->T % 8 || p->H % 8 || p->W % 8)
        return fail(PRISM_ERR_UNSUPPORTED, "grid T x H x W = %d x %d x %d is not a multiple of the 8x8x8 macro-zone",
                    p->T, p->H, p->W);
    if (p->heads < 1) return fail(PRISM_ERR_INVALID_ARG, "heads must be >= 1");
    if (p->head_dim != 64 && p->head_dim != 128)
        return fail(PRISM_ERR_UNSUPPORTED, "head_dim %d unsupported (64 or 128)", p->head_dim);
    if (p->top_k < 1) return fail(PRISM_ERR_INVALID_ARG, "top_k must be >= 1");
    if (!(p->top_p > 0.0f && p->top_p <= 1.0f)) return fail(PRISM_ERR_INVALID_ARG, "top_p must be in (0, 1]");
    if (!(p->max_frac >= 0.0f && p->max_frac <= 1.0f)) return fail(PRISM_ERR_INVALID_ARG, "max_frac must be in [0, 1]");
    const long long N = (long long)p->T * p->H * p->W;
    if (N > (1ll << 26)) return fail(PRISM_ERR_UNSUPPORTED, "grid too large (N = %lld tokens)", N);
    *fixed_idx = -1;
    const int *fs = p->fixed_shape;
    if (fs[0] || fs[1] || fs[2]) {
        const int e0 = log2_exact(fs[0]), e1 = log2_exact(fs[1]), e2 = log2_exact(fs[2]);
        int table[kNumShapes][3];
        host_shape_table(table);
        for (int c = 0; c < kNumShapes; ++c)
            if (table[c][0] == e0 && table[c][1] == e1 && table[c][2] == e2) *fixed_idx = c;
        if (*fixed_idx < 0)
            return fail(PRISM_ERR_INVALID_ARG, "fixed_shape %dx%dx%d is not one of the 16 candidates", fs[0], fs[1],
                        fs[2]);
    }
    g->batch = p->batch;
    g->T = p->T;
    g->H = p->H;
    g->W = p->W;
    g->heads = p->heads;
    g->D = p->head_dim;
    g->N = (int)N;
    g->MT = p->T / 8;
    g->MH = p->H / 8;
    g->MW = p->W / 8;
    g->M = g->MT * g->MH * g->MW;
    g->nbmax = g->N / 64;
    g->C = p->heads * p->head_dim;
    // head sharding: this plan holds heads [head_offset, head_offset + heads) of heads_total
    const int htot = p->heads_total ? p->heads_total : p->heads;
    if (p->head_offset < 0 || p->head_offset + p->heads > htot)
        return fail(PRISM_ERR_INVALID_ARG, "heads [%d, %d) do not lie within heads_total %d", p->head_offset,
                    p->head_offset + p->heads, htot);
    if (htot != p->heads && ((p->heads * p->head_dim) % kStatChunk || (p->head_offset * p->head_dim) % kStatChunk))
        return fail(PRISM_ERR_UNSUPPORTED, "a head shard must cover whole %d-channel chunks", kStatChunk);
    g->Ctot = htot * p->head_dim;
    g->chunk0 = p->head_offset * p->head_dim / kStatChunk;
    g->nchunk_tot = (g->Ctot + kStatChunk - 1) / kStatChunk;
    *cap_stride = cap_for(g->nbmax, p->top_k, p->max_frac);
    const long long rows = (long long)g->batch * g->heads * g->nbmax;
    if (rows * (long long)*cap_stride >= (1ll << 31))
        return fail(PRISM_ERR_UNSUPPORTED, "selection too large for 32-bit CSR offsets (%lld x %d)", rows, *cap_stride);
    if ((long long)g->batch * g->heads * g->N * g->D >= (1ll << 40))
        return fail(PRISM_ERR_UNSUPPORTED, "tensors too large");
    if (p->hilbert_block) {
        if (p->hilbert_block != 64 && p->hilbert_block != 128 && p->hilbert_block != 256)
            return fail(PRISM_ERR_INVALID_ARG, "hilbert_block must be 0, 64, 128 or 256");
        if (fs[0] || fs[1] || fs[2]) return fail(PRISM_ERR_INVALID_ARG, "hilbert_block and fixed_shape exclude each other");
        if (hilbert_level(*g) > 9)
            return fail(PRISM_ERR_UNSUPPORTED, "Hilbert order: grid side above 512 (the cube's flags would exceed 2^27)");
    }
    const double head_scores = (double)g->nbmax * g->nbmax * 8.0;  // bytes of one head's block scores
    if (head_scores > 2.0 * (1ull << 30))
        return fail(PRISM_ERR_UNSUPPORTED, "too many blocks for the score scratch (%d blocks per sample)", g->nbmax);
    return PRISM_OK;
}

// Heads whose block scores are held at once: as many as fit in 1 GiB.
static int score_group_for(const Geo &g) {
    const double head_scores = (double)g.nbmax * g.nbmax * 8.0;
    int G = (int)((double)(1ull << 30) / head_scores);
    if (G < 1) G = 1;
    if (G > g.batch * g.heads) G = g.batch * g.heads;
    return G;
}

struct Alloc {
    void **ptr;
    size_t bytes;
};

static size_t plan_allocs(Plan &pl, Alloc *out) {
    const Geo &g = pl.g;
    const size_t BH = (size_t)g.batch * g.heads, rows = BH * g.nbmax;
    const int nchunk = g.nchunk_tot;  // partials of the whole layer's channels
    const size_t nnz = rows * (size_t)pl.cap_stride;
    size_t n = 0;
    auto add = [&](void **p, size_t b) { out[n++] = Alloc{p, b}; };
    add((void **)&pl.zone_part, (size_t)g.batch * g.M * nchunk * 3 * sizeof(double));
    add((void **)&pl.zone_a, (size_t)g.batch * g.M * 5 * sizeof(double));
    add((void **)&pl.zone_B, (size_t)g.batch * g.M * sizeof(int));
    add((void **)&pl.zone_shape, (size_t)g.batch * g.M * sizeof(int));
    add((void **)&pl.zone_blk0, (size_t)g.batch * (g.M + 1) * sizeof(int));
    add((void **)&pl.nb, (size_t)g.batch * sizeof(int));
    add((void **)&pl.blk_off, (size_t)g.batch * (g.nbmax + 1) * sizeof(int));
    add((void **)&pl.tile_blk, (size_t)g.batch * g.nbmax * sizeof(int));
    add((void **)&pl.zone_qt0, (size_t)g.batch * (g.M + 1) * sizeof(int));
    add((void **)&pl.nqt, (size_t)g.batch * sizeof(int));
    add((void **)&pl.qt_row, (size_t)g.batch * g.nbmax * sizeof(int));
    add((void **)&pl.qt_blk, (size_t)g.batch * g.nbmax * sizeof(int));
    add((void **)&pl.perm, (size_t)g.batch * g.N * sizeof(int));
    add((void **)&pl.Qp, BH * g.N * g.D * 2);
    add((void **)&pl.Kp, BH * g.N * g.D * 2);
    add((void **)&pl.Vp, BH * g.N * g.D * 2);
    add((void **)&pl.Qbar, rows * g.D * sizeof(double));
    add((void **)&pl.Kbar, rows * g.D * sizeof(double));
    add((void **)&pl.Kb, rows * g.D * 2);
    add((void **)&pl.Vb, rows * g.D * 2);
    add((void **)&pl.score_keys, (size_t)pl.score_group * g.nbmax * g.nbmax * sizeof(unsigned long long));
    add((void **)&pl.cnt, rows * sizeof(int));
    add((void **)&pl.cols_pad, nnz * sizeof(int));
    add((void **)&pl.row_ptr, (rows + 1) * sizeof(int));
    add((void **)&pl.col, nnz * sizeof(int));
    add((void **)&pl.colT_ptr, (rows + 1) * sizeof(int));
    add((void **)&pl.rowT, nnz * sizeof(int));
    add((void **)&pl.colT_cursor, rows * sizeof(int));
    add((void **)&pl.scan_tmp, ((rows + 1023) / 1024 + 1) * sizeof(int));
    add((void **)&pl.nlse_p, BH * g.N * sizeof(float));
    add((void **)&pl.dOp, BH * g.N * g.D * 2);
    add((void **)&pl.delta, BH * g.N * sizeof(float));
    add((void **)&pl.dQacc, BH * g.N * g.D * sizeof(float));
    add((void **)&pl.status, 16 * sizeof(int));
    return n;
}

// ---------------------------------------------------------------------------
// per-kernel event timing
// ---------------------------------------------------------------------------
struct TimerState {
    std::vector<cudaEvent_t> pool;                              // free events
    std::vector<std::pair<cudaEvent_t, cudaEvent_t>> rec[kTCount];
    cudaEvent_t take() {
        if (pool.empty()) {
            cudaEvent_t e;
            if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
            return e;
        }
        cudaEvent_t e = pool.back();
        pool.pop_back();
        return e;
    }
    ~TimerState() {
        for (auto e : pool) cudaEventDestroy(e);
        for (auto &v : rec)
            for (auto &pr : v) {
                cudaEventDestroy(pr.first);
                cudaEventDestroy(pr.second);
            }
    }
};

TimerScope::TimerScope(Plan &p, int i, cudaStream_t s) : pl(p), id(i), st(s) {
    if (!pl.timers) return;
    cudaEvent_t a = pl.timers->take(), b = pl.timers->take();
    if (!a || !b) return;
    cudaEventRecord(a, st);
    pl.timers->rec[id].push_back({a, b});
}

TimerScope::~TimerScope() {
    if (!pl.timers || pl.timers->rec[id].empty()) return;
    cudaEventRecord(pl.timers->rec[id].back().second, st);
}

static void release_buffers(Plan &pl) {
    release_host_pipe(pl);  // first: its streams may still use the plan's buffers
    Alloc a[64];
    const size_t n = plan_allocs(pl, a);
    for (size_t k = 0; k < n; ++k)
        if (*a[k].ptr) {
            cudaFree(*a[k].ptr);
            *a[k].ptr = nullptr;
        }
    if (pl.host_nb) {
        cudaFreeHost(pl.host_nb);
        pl.host_nb = nullptr;
    }
    delete pl.timers;
    pl.timers = nullptr;
}

}  // namespace prism

using namespace prism;

struct prism_plan {
    Plan pl;
};

extern "C" {

const char *prism_last_error(void) { return g_last_error.c_str(); }

size_t prism_plan_bytes(const prism_params *params) {
    Plan pl;
    memset(&pl, 0, sizeof pl);
    if (check_params(params, &pl.g, &pl.fixed_idx, &pl.cap_stride) != PRISM_OK) return 0;
    pl.score_group = score_group_for(pl.g);
    Alloc a[64];
    const size_t n = plan_allocs(pl, a);
    size_t tot = 0;
    for (size_t k = 0; k < n; ++k) tot += (a[k].bytes + 255) & ~(size_t)255;
    return tot;
}

prism_status prism_plan_create(const prism_params *params, prism_plan **out) {
    g_last_error.clear();
    if (!out) return fail(PRISM_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    prism_plan *h = new (std::nothrow) prism_plan;
    if (!h) return fail(PRISM_ERR_NOMEM, "host allocation failed");
    memset(&h->pl, 0, sizeof h->pl);
    Plan &pl = h->pl;
    prism_status s = check_params(params, &pl.g, &pl.fixed_idx, &pl.cap_stride);
    if (s != PRISM_OK) {
        delete h;
        return s;
    }
    pl.p = *params;
    if (!(pl.p.eps > 0.0)) pl.p.eps = 1e-6;
    pl.score_group = score_group_for(pl.g);
    if (select_smem_bytes(pl) > 220 * 1024) {
        delete h;
        return fail(PRISM_ERR_UNSUPPORTED, "selection working set (%zu bytes of shared memory) too large",
                    select_smem_bytes(pl));
    }
    cudaError_t e = cudaGetDevice(&pl.device);
    if (e != cudaSuccess) {
        delete h;
        return fail_cuda(e, "cudaGetDevice", __FILE__, __LINE__);
    }
    Alloc a[64];
    const size_t n = plan_allocs(pl, a);
    for (size_t k = 0; k < n; ++k) *a[k].ptr = nullptr;
    for (size_t k = 0; k < n; ++k) {
        e = cudaMalloc(a[k].ptr, a[k].bytes);
        if (e != cudaSuccess) {
            *a[k].ptr = nullptr;
            release_buffers(pl);
            delete h;
            return fail_cuda(e, "cudaMalloc", __FILE__, __LINE__);
        }
    }
    e = cudaMallocHost((void **)&pl.host_nb, 64 * sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(pl.status, 0, 16 * sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(pl.Kb, 0, (size_t)pl.g.batch * pl.g.heads * pl.g.nbmax * pl.g.D * 2);
    if (e == cudaSuccess) e = cudaMemset(pl.Vb, 0, (size_t)pl.g.batch * pl.g.heads * pl.g.nbmax * pl.g.D * 2);
    if (e != cudaSuccess) {
        release_buffers(pl);
        delete h;
        return fail_cuda(e, "plan setup", __FILE__, __LINE__);
    }
    s = configure_plan_kernels(pl);
    if (s == PRISM_OK) s = configure_attn_tc_kernels();
    if (s == PRISM_OK) s = configure_attn_bwd_tc_kernels();
    if (s == PRISM_OK) s = make_tensor_maps(pl);
    if (s == PRISM_OK && pl.p.hilbert_block) s = setup_hilbert_plan(pl);

    if (s != PRISM_OK) {
        release_buffers(pl);
        delete h;
        return s;
    }
    *out = h;
    return PRISM_OK;
}

void prism_plan_destroy(prism_plan *plan) {
    if (!plan) return;
    release_buffers(plan->pl);
    delete plan;
}

static prism_status device_guard(const Plan &pl) {
    int cur = -1;
    PRISM_CUDA_OK(cudaGetDevice(&cur));
    if (cur != pl.device)
        return fail(PRISM_ERR_INVALID_ARG, "current device %d is not the plan's device %d", cur, pl.device);
    return PRISM_OK;
}

prism_status prism_plan_build(prism_plan *plan, const void *Q, const void *K, const void *V, const float *a_norm,
                              void *stream) {
    g_last_error.clear();
    if (!plan || !Q || !K || !V || (!a_norm && !plan->pl.p.hilbert_block))
        return fail(PRISM_ERR_INVALID_ARG, "NULL argument to prism_plan_build");
    prism_status s = device_guard(plan->pl);
    if (s != PRISM_OK) return s;
    const uintptr_t al = (uintptr_t)Q | (uintptr_t)K | (uintptr_t)V;
    if (al & 15) return fail(PRISM_ERR_INVALID_ARG, "Q, K, V must be 16-byte aligned");
    if (plan->pl.g.Ctot != plan->pl.g.C && !plan->pl.p.hilbert_block)
        return fail(PRISM_ERR_STATE, "a head-sharded plan is built with build_stats, an exchange and build_finish");
    plan->pl.have_fwd = false;
    s = launch_plan(plan->pl, Q, K, V, a_norm, static_cast<cudaStream_t>(stream));
    if (s == PRISM_OK) plan->pl.built = true;
    return s;
}

prism_status prism_plan_build_stats(prism_plan *plan, const void *V, const float *a_norm, void *stream) {
    g_last_error.clear();
    if (!plan || !V || !a_norm) return fail(PRISM_ERR_INVALID_ARG, "NULL argument to prism_plan_build_stats");
    prism_status s = device_guard(plan->pl);
    if (s != PRISM_OK) return s;
    if ((uintptr_t)V & 15) return fail(PRISM_ERR_INVALID_ARG, "V must be 16-byte aligned");
    if (plan->pl.p.hilbert_block)
        return fail(PRISM_ERR_STATE, "a Hilbert-order plan has no zone statistics: build it with prism_plan_build");
    plan->pl.have_fwd = false;
    plan->pl.built = false;
    s = launch_plan_stats(plan->pl, V, a_norm, static_cast<cudaStream_t>(stream));
    plan->pl.have_stats = s == PRISM_OK;
    return s;
}

prism_status prism_plan_stats_slice(prism_plan *plan, void **buf, size_t *slice_offset, size_t *slice_bytes,
                                    size_t *total_bytes) {
    g_last_error.clear();
    if (!plan || !buf || !slice_offset || !slice_bytes || !total_bytes)
        return fail(PRISM_ERR_INVALID_ARG, "NULL argument to prism_plan_stats_slice");
    const Geo &g = plan->pl.g;
    const size_t per_chunk = (size_t)g.batch * g.M * 3 * sizeof(double);
    *buf = plan->pl.zone_part;
    *slice_offset = (size_t)g.chunk0 * per_chunk;
    *slice_bytes = (size_t)((g.C + kStatChunk - 1) / kStatChunk) * per_chunk;
    *total_bytes = (size_t)g.nchunk_tot * per_chunk;
    return PRISM_OK;
}

prism_status prism_plan_build_finish(prism_plan *plan, const void *Q, const void *K, const void *V, void *stream) {
    g_last_error.clear();
    if (!plan || !Q || !K || !V) return fail(PRISM_ERR_INVALID_ARG, "NULL argument to prism_plan_build_finish");
    prism_status s = device_guard(plan->pl);
    if (s != PRISM_OK) return s;
    const uintptr_t al = (uintptr_t)Q | (uintptr_t)K | (uintptr_t)V;
    if (al & 15) return fail(PRISM_ERR_INVALID_ARG, "Q, K, V must be 16-byte aligned");
    if (!plan->pl.have_stats) return fail(PRISM_ERR_STATE, "prism_plan_build_finish needs prism_plan_build_stats first");
    plan->pl.have_fwd = false;
    plan->pl.have_stats = false;
    s = launch_plan_finish(plan->pl, Q, K, V, static_cast<cudaStream_t>(stream));
    if (s == PRISM_OK) plan->pl.built = true;
    return s;
}

prism_status prism_plan_build_with_zones(prism_plan *plan, const void *Q, const void *K, const void *V,
                                        const int *zone_B, const int *zone_shape, void *stream) {
    g_last_error.clear();
    if (!plan || !Q || !K || !V || !zone_B || !zone_shape)
        return fail(PRISM_ERR_INVALID_ARG, "NULL argument to prism_plan_build_with_zones");
    prism_status s = device_guard(plan->pl);
    if (s != PRISM_OK) return s;
    Plan &pl = plan->pl;
    if (pl.p.hilbert_block) return fail(PRISM_ERR_STATE, "a Hilbert-order plan has no zones");
    const uintptr_t al = (uintptr_t)Q | (uintptr_t)K | (uintptr_t)V;
    if (al & 15) return fail(PRISM_ERR_INVALID_ARG, "Q, K, V must be 16-byte aligned");
    int table[kNumShapes][3];
    host_shape_table(table);
    const size_t nz = (size_t)pl.g.batch * pl.g.M;
    for (size_t z = 0; z < nz; ++z) {
        const int B = zone_B[z], c = zone_shape[z];
        if (B != 64 && B != 128 && B != 256)
            return fail(PRISM_ERR_INVALID_ARG, "zone %zu (sample %zu): volume %d is not 64, 128 or 256", z % pl.g.M,
                        z / pl.g.M, B);
        if (c < 0 || c >= kNumShapes || (1 << (table[c][0] + table[c][1] + table[c][2])) != B)
            return fail(PRISM_ERR_INVALID_ARG, "zone %zu (sample %zu): shape %d is not a candidate of volume %d",
                        z % pl.g.M, z / pl.g.M, c, B);
    }
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    pl.have_fwd = false;
    pl.built = false;
    pl.have_stats = false;
    PRISM_CUDA_OK(cudaMemcpyAsync(pl.zone_B, zone_B, nz * sizeof(int), cudaMemcpyHostToDevice, st));
    PRISM_CUDA_OK(cudaMemcpyAsync(pl.zone_shape, zone_shape, nz * sizeof(int), cudaMemcpyHostToDevice, st));
    s = launch_plan_given(pl, Q, K, V, st);
    if (s == PRISM_OK) pl.built = true;
    return s;
}

prism_status prism_plan_update_qkv(prism_plan *plan, const void *Q, const void *K, const void *V, void *stream) {
    g_last_error.clear();
    if (!plan || !Q || !K || !V) return fail(PRISM_ERR_INVALID_ARG, "NULL argument to prism_plan_update_qkv");
    prism_status s = device_guard(plan->pl);
    if (s != PRISM_OK) return s;
    if (!plan->pl.built) return fail(PRISM_ERR_STATE, "prism_plan_update_qkv needs a built plan");
    const uintptr_t al = (uintptr_t)Q | (uintptr_t)K | (uintptr_t)V;
    if (al & 15) return fail(PRISM_ERR_INVALID_ARG, "Q, K, V must be 16-byte aligned");
    plan->pl.have_fwd = false;
    return launch_regather(plan->pl, Q, K, V, static_cast<cudaStream_t>(stream));
}

prism_status prism_attn_fwd(prism_plan *plan, void *O, float *lse, void *stream) {
    g_last_error.clear();
    if (!plan || !O) return fail(PRISM_ERR_INVALID_ARG, "NULL argument to prism_attn_fwd");
    prism_status s = device_guard(plan->pl);
    if (s != PRISM_OK) return s;
    if (!plan->pl.built) return fail(PRISM_ERR_STATE, "prism_attn_fwd needs a built plan");
    if ((uintptr_t)O & 15) return fail(PRISM_ERR_INVALID_ARG, "O must be 16-byte aligned");
    s = launch_attn_fwd_tc(plan->pl, O, lse, static_cast<cudaStream_t>(stream));
    if (s == PRISM_OK) plan->pl.have_fwd = true;
    return s;
}

prism_status prism_attn_fwd_taylor(prism_plan *plan, void *O, float *lse, void *stream) {
    g_last_error.clear();
    if (!plan || !O) return fail(PRISM_ERR_INVALID_ARG, "NULL argument to prism_attn_fwd_taylor");
    prism_status s = device_guard(plan->pl);
    if (s != PRISM_OK) return s;
    if (!plan->pl.built) return fail(PRISM_ERR_STATE, "prism_attn_fwd_taylor needs a built plan");
    if ((uintptr_t)O & 15) return fail(PRISM_ERR_INVALID_ARG, "O must be 16-byte aligned");
    if (!taylor_fits(plan->pl.g))
        return fail(PRISM_ERR_UNSUPPORTED, "too many key blocks for the Taylor forward's shared-memory table");
    return launch_attn_fwd_taylor(plan->pl, O, lse, static_cast<cudaStream_t>(stream));
}

prism_status prism_attn_bwd(prism_plan *plan, const void *O, const void *dO, void *dQ, void *dK, void *dV,
                            void *stream) {
    g_last_error.clear();
    if (!plan || !O || !dO || !dQ || !dK || !dV) return fail(PRISM_ERR_INVALID_ARG, "NULL argument to prism_attn_bwd");
    prism_status s = device_guard(plan->pl);
    if (s != PRISM_OK) return s;
    if (!plan->pl.have_fwd)
        return fail(PRISM_ERR_STATE, "prism_attn_bwd needs a prism_attn_fwd after the last build or update");
    const uintptr_t al = (uintptr_t)O | (uintptr_t)dO | (uintptr_t)dQ | (uintptr_t)dK | (uintptr_t)dV;
    if (al & 15) return fail(PRISM_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
    return launch_attn_bwd(plan->pl, O, dO, dQ, dK, dV, static_cast<cudaStream_t>(stream));
}

prism_status prism_audio_norms(const void *h, float *a, int batch, int T, int H, int W, int channels, void *stream) {
    g_last_error.clear();
    if (!h || !a) return fail(PRISM_ERR_INVALID_ARG, "NULL argument to prism_audio_norms");
    if (batch < 1 || T < 1 || H < 1 || W < 1) return fail(PRISM_ERR_INVALID_ARG, "batch, T, H, W must be >= 1");
    if (channels < 1 || channels > (1 << 20)) return fail(PRISM_ERR_INVALID_ARG, "channels must be in [1, 2^20]");
    return launch_audio_norms(h, a, (long long)batch * T * H * W, channels, static_cast<cudaStream_t>(stream));
}

prism_status prism_step_host(prism_plan *plan, const prism_host_io *io, void *stream, unsigned long long *ticket) {
    g_last_error.clear();
    if (!plan || !io || !ticket) return fail(PRISM_ERR_INVALID_ARG, "NULL argument to prism_step_host");
    if (!io->Q || !io->K || !io->V || (!io->a_norm && !plan->pl.p.hilbert_block) || !io->O)
        return fail(PRISM_ERR_INVALID_ARG, "prism_step_host needs Q, K, V, a_norm and O");
    if (io->dO && (!io->dQ || !io->dK || !io->dV))
        return fail(PRISM_ERR_INVALID_ARG, "prism_step_host with dO needs dQ, dK and dV");
    if (io->taylor && io->dO)
        return fail(PRISM_ERR_INVALID_ARG, "a Taylor forward has no backward: taylor steps are forward-only");
    if (io->taylor && !taylor_fits(plan->pl.g))
        return fail(PRISM_ERR_UNSUPPORTED, "too many key blocks for the Taylor forward's shared-memory table");
    if (plan->pl.g.Ctot != plan->pl.g.C && !plan->pl.p.hilbert_block)
        return fail(PRISM_ERR_STATE, "prism_step_host runs unsharded zone plans only");
    prism_status s = device_guard(plan->pl);
    if (s != PRISM_OK) return s;
    return host_step(plan->pl, *io, static_cast<cudaStream_t>(stream), ticket);
}

prism_status prism_step_join(prism_plan *plan, unsigned long long ticket, void *stream) {
    g_last_error.clear();
    if (!plan) return fail(PRISM_ERR_INVALID_ARG, "plan is NULL");
    prism_status s = device_guard(plan->pl);
    if (s != PRISM_OK) return s;
    return host_step_join(plan->pl, ticket, static_cast<cudaStream_t>(stream));
}

prism_status prism_step_wait(prism_plan *plan, unsigned long long ticket) {
    g_last_error.clear();
    if (!plan) return fail(PRISM_ERR_INVALID_ARG, "plan is NULL");
    prism_status s = device_guard(plan->pl);
    if (s != PRISM_OK) return s;
    return host_step_wait(plan->pl, ticket);
}

prism_status prism_plan_view_get(prism_plan *plan, prism_plan_view *view, void *stream) {
    g_last_error.clear();
    if (!plan || !view) return fail(PRISM_ERR_INVALID_ARG, "NULL argument to prism_plan_view_get");
    Plan &pl = plan->pl;
    prism_status s = device_guard(pl);
    if (s != PRISM_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t rows = (size_t)pl.g.batch * pl.g.heads * pl.g.nbmax;
    int nnz = 0;
    PRISM_CUDA_OK(cudaMemcpyAsync(pl.host_nb, pl.nb, pl.g.batch * sizeof(int), cudaMemcpyDeviceToHost, st));
    PRISM_CUDA_OK(cudaMemcpyAsync(&nnz, pl.row_ptr + rows, sizeof(int), cudaMemcpyDeviceToHost, st));
    PRISM_CUDA_OK(cudaStreamSynchronize(st));
    memset(view, 0, sizeof *view);
    view->zone_B = pl.zone_B;
    view->zone_shape = pl.zone_shape;
    view->perm = pl.perm;
    view->blk_off = pl.blk_off;
    view->row_ptr = pl.row_ptr;
    view->col_idx = pl.col;
    view->nbmax = pl.g.nbmax;
    view->nnz = nnz;
    for (int b = 0; b < pl.g.batch; ++b) view->n_blocks[b] = pl.host_nb[b];
    return PRISM_OK;
}

static const char *const kTimerNames[kTCount] = {"zone_stats_v", "zone_stats_a", "zone_decide", "permute_pool",
                                                  "select", "csr_csc", "attn_fwd", "attn_bwd_pre", "attn_bwd",
                                                  "dq_finalize", "taylor_pool", "attn_fwd_taylor"};

const char *prism_timer_name(int id) { return (id >= 0 && id < kTCount) ? kTimerNames[id] : ""; }

prism_status prism_plan_set_timing(prism_plan *plan, int enable) {
    g_last_error.clear();
    if (!plan) return fail(PRISM_ERR_INVALID_ARG, "plan is NULL");
    if (enable && !plan->pl.timers) {
        plan->pl.timers = new (std::nothrow) TimerState;
        if (!plan->pl.timers) return fail(PRISM_ERR_NOMEM, "timer allocation failed");
    } else if (!enable && plan->pl.timers) {
        cudaDeviceSynchronize();
        delete plan->pl.timers;
        plan->pl.timers = nullptr;
    }
    return PRISM_OK;
}

prism_status prism_plan_read_timing(prism_plan *plan, float *total_ms, int *launches) {
    g_last_error.clear();
    if (!plan || !total_ms || !launches) return fail(PRISM_ERR_INVALID_ARG, "NULL argument to prism_plan_read_timing");
    TimerState *ts = plan->pl.timers;
    for (int k = 0; k < kTCount; ++k) {
        total_ms[k] = 0.f;
        launches[k] = 0;
        if (!ts) continue;
        for (auto &pr : ts->rec[k]) {
            PRISM_CUDA_OK(cudaEventSynchronize(pr.second));
            float ms = 0.f;
            PRISM_CUDA_OK(cudaEventElapsedTime(&ms, pr.first, pr.second));
            total_ms[k] += ms;
            launches[k] += 1;
            ts->pool.push_back(pr.first);
            ts->pool.push_back(pr.second);
        }
        ts->rec[k].clear();
    }
    return PRISM_OK;
}

prism_status prism_plan_selftest_timeout(prism_plan *plan, void *stream) {
    g_last_error.clear();
    if (!plan) return fail(PRISM_ERR_INVALID_ARG, "plan is NULL");
    prism_status s = device_guard(plan->pl);
    if (s != PRISM_OK) return s;
    return launch_selftest_bounded_wait(plan->pl, static_cast<cudaStream_t>(stream));
}

prism_status prism_plan_check(prism_plan *plan, void *stream) {
    g_last_error.clear();
    if (!plan) return fail(PRISM_ERR_INVALID_ARG, "plan is NULL");
    Plan &pl = plan->pl;
    prism_status s = device_guard(pl);
    if (s != PRISM_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int word[2] = {0, 0};
    PRISM_CUDA_OK(cudaMemcpyAsync(word, pl.status, sizeof word, cudaMemcpyDeviceToHost, st));
    PRISM_CUDA_OK(cudaStreamSynchronize(st));
    PRISM_CUDA_OK(cudaGetLastError());
    if (word[0] != 0) {
        PRISM_CUDA_OK(cudaMemsetAsync(pl.status, 0, 16 * sizeof(int), st));
        PRISM_CUDA_OK(cudaStreamSynchronize(st));
        return fail(PRISM_ERR_TIMEOUT, "device-side wait gave up (code %d, site %d)", word[0], word[1]);
    }
    return PRISM_OK;
}

}  // extern "C"
