// host_pipeline.cu -- layer steps fed from host memory, pipelined across
// calls on three streams of the plan's own:
//   h2d   copies step t's inputs into device staging set t % 2,
//   comp  builds the plan and runs the attention kernels on that set,
//   d2h   copies step t's outputs back to the caller's host buffers.
// Cross-stream order, per staging set s and step t (s = t % 2):
//   h2d(t)  waits for comp(t-2)  (comp(t-2) has read the inputs of set s)
//   comp(t) waits for Q, K, V, a of h2d(t) before the plan, and for dO of
//           h2d(t) only before the backward
//   comp(t) waits for d2h(t-2)   (outputs of set s copied out)
//   d2h(t)  copies O (and lse) once the forward of t is done, the gradients
//           once its backward is
// The kernels of consecutive steps stay in order on `comp`, so the plan's
// internal buffers (permuted copies, CSR, statistics) are never shared by two
// steps at once.
#include <string.h>

#include <new>

#include "prism_internal.cuh"

namespace prism {

namespace {
constexpr int kSets = 2;    // device staging sets
constexpr int kRing = 8;    // completion events kept: steps in flight at most
enum { kQ = 0, kK, kV, kA, kdO, kNumIn };
enum { kO = 0, kLse, kdQ, kdK, kdV, kNumOut };
}  // namespace

struct HostPipe {
    cudaStream_t h2d = nullptr, comp = nullptr, d2h = nullptr;
    cudaEvent_t user = nullptr;                       // the caller's stream at each call
    cudaEvent_t in_ready[kSets] = {}, dO_ready[kSets] = {}, fwd_done[kSets] = {}, comp_done[kSets] = {};
    cudaEvent_t out_done[kRing] = {};                 // step t -> out_done[(t-1) % kRing]
    void *in[kSets][kNumIn] = {};
    void *out[kSets][kNumOut] = {};
    unsigned long long issued = 0;
};

static prism_status ensure(void **p, size_t bytes) {
    if (*p) return PRISM_OK;
    cudaError_t e = cudaMalloc(p, bytes);
    if (e != cudaSuccess) {
        *p = nullptr;
        return e == cudaErrorMemoryAllocation ? fail(PRISM_ERR_NOMEM, "staging allocation of %zu bytes failed", bytes)
                                              : fail_cuda(e, "cudaMalloc", __FILE__, __LINE__);
    }
    return PRISM_OK;
}

static prism_status create_pipe(Plan &pl) {
    HostPipe *hp = new (std::nothrow) HostPipe;
    if (!hp) return fail(PRISM_ERR_NOMEM, "host allocation failed");
    pl.pipe = hp;  // released by release_host_pipe, also on a failure below
    PRISM_CUDA_OK(cudaStreamCreateWithFlags(&hp->h2d, cudaStreamNonBlocking));
    PRISM_CUDA_OK(cudaStreamCreateWithFlags(&hp->comp, cudaStreamNonBlocking));
    PRISM_CUDA_OK(cudaStreamCreateWithFlags(&hp->d2h, cudaStreamNonBlocking));
    PRISM_CUDA_OK(cudaEventCreateWithFlags(&hp->user, cudaEventDisableTiming));
    for (int s = 0; s < kSets; ++s) {
        PRISM_CUDA_OK(cudaEventCreateWithFlags(&hp->in_ready[s], cudaEventDisableTiming));
        PRISM_CUDA_OK(cudaEventCreateWithFlags(&hp->dO_ready[s], cudaEventDisableTiming));
        PRISM_CUDA_OK(cudaEventCreateWithFlags(&hp->fwd_done[s], cudaEventDisableTiming));
        PRISM_CUDA_OK(cudaEventCreateWithFlags(&hp->comp_done[s], cudaEventDisableTiming));
    }
    for (int r = 0; r < kRing; ++r) PRISM_CUDA_OK(cudaEventCreateWithFlags(&hp->out_done[r], cudaEventDisableTiming));
    return PRISM_OK;
}

void release_host_pipe(Plan &pl) {
    HostPipe *hp = pl.pipe;
    if (!hp) return;
    for (cudaStream_t st : {hp->h2d, hp->comp, hp->d2h})
        if (st) cudaStreamSynchronize(st);
    for (int s = 0; s < kSets; ++s) {
        for (void *p : hp->in[s])
            if (p) cudaFree(p);
        for (void *p : hp->out[s])
            if (p) cudaFree(p);
        if (hp->in_ready[s]) cudaEventDestroy(hp->in_ready[s]);
        if (hp->dO_ready[s]) cudaEventDestroy(hp->dO_ready[s]);
        if (hp->fwd_done[s]) cudaEventDestroy(hp->fwd_done[s]);
        if (hp->comp_done[s]) cudaEventDestroy(hp->comp_done[s]);
    }
    for (cudaEvent_t e : hp->out_done)
        if (e) cudaEventDestroy(e);
    if (hp->user) cudaEventDestroy(hp->user);
    for (cudaStream_t st : {hp->h2d, hp->comp, hp->d2h})
        if (st) cudaStreamDestroy(st);
    delete hp;
    pl.pipe = nullptr;
}

prism_status host_step(Plan &pl, const prism_host_io &io, cudaStream_t user, unsigned long long *ticket) {
    if (!pl.pipe) {
        prism_status s = create_pipe(pl);
        if (s != PRISM_OK) {
            release_host_pipe(pl);
            return s;
        }
    }
    HostPipe &hp = *pl.pipe;
    const Geo &g = pl.g;
    const bool bwd = io.dO != nullptr;
    const size_t qkv = (size_t)g.batch * g.N * g.heads * g.D * sizeof(__nv_bfloat16);
    const size_t abytes = (size_t)g.batch * g.N * sizeof(float);
    const size_t lbytes = (size_t)g.batch * g.heads * g.N * sizeof(float);

    const unsigned long long t = hp.issued + 1;
    const int s = (int)((t - 1) % kSets);
    const int r = (int)((t - 1) % kRing);
    // staging set s (allocated on first use; a failed allocation leaves nothing enqueued)
    prism_status st = PRISM_OK;
    for (int k : {kQ, kK, kV}) st = st == PRISM_OK ? ensure(&hp.in[s][k], qkv) : st;
    if (st == PRISM_OK) st = ensure(&hp.in[s][kA], abytes);
    if (st == PRISM_OK) st = ensure(&hp.out[s][kO], qkv);
    if (st == PRISM_OK && io.lse) st = ensure(&hp.out[s][kLse], lbytes);
    if (bwd)
        for (int k : {kdQ, kdK, kdV}) st = st == PRISM_OK ? ensure(&hp.out[s][k], qkv) : st;
    if (st == PRISM_OK && bwd) st = ensure(&hp.in[s][kdO], qkv);
    if (st != PRISM_OK) return st;

    // the ring slot is reused: its previous step (t - kRing) must be complete
    if (t > (unsigned long long)kRing) PRISM_CUDA_OK(cudaEventSynchronize(hp.out_done[r]));

    // h2d: after the caller's prior work and after comp(t-2) has read set s
    PRISM_CUDA_OK(cudaEventRecord(hp.user, user));
    PRISM_CUDA_OK(cudaStreamWaitEvent(hp.h2d, hp.user, 0));
    if (t > (unsigned long long)kSets) PRISM_CUDA_OK(cudaStreamWaitEvent(hp.h2d, hp.comp_done[s], 0));
    PRISM_CUDA_OK(cudaMemcpyAsync(hp.in[s][kQ], io.Q, qkv, cudaMemcpyHostToDevice, hp.h2d));
    PRISM_CUDA_OK(cudaMemcpyAsync(hp.in[s][kK], io.K, qkv, cudaMemcpyHostToDevice, hp.h2d));
    PRISM_CUDA_OK(cudaMemcpyAsync(hp.in[s][kV], io.V, qkv, cudaMemcpyHostToDevice, hp.h2d));
    if (io.a_norm)  // a Hilbert-order plan has no use for it
        PRISM_CUDA_OK(cudaMemcpyAsync(hp.in[s][kA], io.a_norm, abytes, cudaMemcpyHostToDevice, hp.h2d));
    PRISM_CUDA_OK(cudaEventRecord(hp.in_ready[s], hp.h2d));
    if (bwd) {
        PRISM_CUDA_OK(cudaMemcpyAsync(hp.in[s][kdO], io.dO, qkv, cudaMemcpyHostToDevice, hp.h2d));
        PRISM_CUDA_OK(cudaEventRecord(hp.dO_ready[s], hp.h2d));
    }

    // comp: after the inputs landed and after d2h(t-2) has read set s's outputs
    PRISM_CUDA_OK(cudaStreamWaitEvent(hp.comp, hp.in_ready[s], 0));
    if (t > (unsigned long long)kSets)
        PRISM_CUDA_OK(cudaStreamWaitEvent(hp.comp, hp.out_done[(t - 1 - kSets) % kRing], 0));
    pl.have_fwd = false;
    st = launch_plan(pl, hp.in[s][kQ], hp.in[s][kK], hp.in[s][kV], static_cast<const float *>(hp.in[s][kA]), hp.comp);
    if (st != PRISM_OK) return st;
    pl.built = true;
    float *lse_dev = io.lse ? static_cast<float *>(hp.out[s][kLse]) : nullptr;
    st = io.taylor ? launch_attn_fwd_taylor(pl, hp.out[s][kO], lse_dev, hp.comp)
                   : launch_attn_fwd_tc(pl, hp.out[s][kO], lse_dev, hp.comp);
    if (st != PRISM_OK) return st;
    pl.have_fwd = true;
    PRISM_CUDA_OK(cudaEventRecord(hp.fwd_done[s], hp.comp));
    if (bwd) {
        PRISM_CUDA_OK(cudaStreamWaitEvent(hp.comp, hp.dO_ready[s], 0));
        st = launch_attn_bwd(pl, hp.out[s][kO], hp.in[s][kdO], hp.out[s][kdQ], hp.out[s][kdK], hp.out[s][kdV],
                             hp.comp);
        if (st != PRISM_OK) return st;
    }
    PRISM_CUDA_OK(cudaEventRecord(hp.comp_done[s], hp.comp));

    // d2h: O and lse as soon as the forward is done, the gradients after the backward
    PRISM_CUDA_OK(cudaStreamWaitEvent(hp.d2h, hp.fwd_done[s], 0));
    PRISM_CUDA_OK(cudaMemcpyAsync(io.O, hp.out[s][kO], qkv, cudaMemcpyDeviceToHost, hp.d2h));
    if (io.lse) PRISM_CUDA_OK(cudaMemcpyAsync(io.lse, hp.out[s][kLse], lbytes, cudaMemcpyDeviceToHost, hp.d2h));
    PRISM_CUDA_OK(cudaStreamWaitEvent(hp.d2h, hp.comp_done[s], 0));
    if (bwd) {
        PRISM_CUDA_OK(cudaMemcpyAsync(io.dQ, hp.out[s][kdQ], qkv, cudaMemcpyDeviceToHost, hp.d2h));
        PRISM_CUDA_OK(cudaMemcpyAsync(io.dK, hp.out[s][kdK], qkv, cudaMemcpyDeviceToHost, hp.d2h));
        PRISM_CUDA_OK(cudaMemcpyAsync(io.dV, hp.out[s][kdV], qkv, cudaMemcpyDeviceToHost, hp.d2h));
    }
    PRISM_CUDA_OK(cudaEventRecord(hp.out_done[r], hp.d2h));
    hp.issued = t;
    *ticket = t;
    return PRISM_OK;
}

// A ticket at least kRing steps old completed before a later step reused its
// event (host_step waits for it), so only the last kRing tickets need a wait.
static prism_status ticket_event(Plan &pl, unsigned long long ticket, cudaEvent_t *ev) {
    *ev = nullptr;
    if (ticket == 0 || !pl.pipe || ticket > pl.pipe->issued)
        return fail(PRISM_ERR_INVALID_ARG, "step ticket %llu was not issued by this plan", ticket);
    if (ticket + kRing > pl.pipe->issued) *ev = pl.pipe->out_done[(ticket - 1) % kRing];
    return PRISM_OK;
}

prism_status host_step_join(Plan &pl, unsigned long long ticket, cudaStream_t st) {
    cudaEvent_t ev;
    prism_status s = ticket_event(pl, ticket, &ev);
    if (s != PRISM_OK || !ev) return s;
    PRISM_CUDA_OK(cudaStreamWaitEvent(st, ev, 0));
    return PRISM_OK;
}

prism_status host_step_wait(Plan &pl, unsigned long long ticket) {
    cudaEvent_t ev;
    prism_status s = ticket_event(pl, ticket, &ev);
    if (s != PRISM_OK || !ev) return s;
    PRISM_CUDA_OK(cudaEventSynchronize(ev));
    return PRISM_OK;
}

}  // namespace prism
