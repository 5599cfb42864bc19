// noalloc.cu -- zone statistics and block volume / shape decisions without
// any device allocation.
//
// Some callers cannot call cudaMalloc: an application whose caching allocator
// owns all device memory and forbids allocations outside it, or a loop where
// cudaMalloc's implicit device synchronisation and latency are not
// acceptable.  prism_zone_shapes_noalloc gives them the planner's first stage
// (per-zone statistics, density, block volume B(m) and shape) with all scratch
// taken from one fixed array compiled into the library, of size
// PRISM_NOALLOC_SCRATCH_BYTES, which every GPU that loads the library keeps
// until the process exits.
#include <mutex>

#include "prism_internal.cuh"

namespace prism {

int host_shape_table(int (*e)[3]);
prism_status launch_zone_decisions(const Geo &g, double eps, int fixed_idx, const __nv_bfloat16 *V, const float *a,
                                   double *zone_part, double *zone_a, int *zone_B, int *zone_shape, int *zone_blk0,
                                   int *nb, int *blk_off, int *tile_blk, int *zone_qt0, int *nqt, int *qt_row,
                                   int *qt_blk, cudaStream_t st);
prism_status configure_zone_kernels();

// The scratch.  In host code this name is only a stand-in for the device
// array: kernels must receive the address cudaGetSymbolAddress returns.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PRISM_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
// Per device: the scratch address and the id of the CUDA context it was
// looked up in.  A device address belongs to one context; after
// cudaDeviceReset the device's next primary context has a new id, so the
// address, the kernel attributes and the constant table are set up again.
unsigned char *g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// The id of the calling thread's current context (unique for the life of the
// process; ids are never reused, unlike CUcontext handles).
prism_status current_context_id(unsigned long long *id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    if (!get_current || !get_id) {
        void *p1 = nullptr, *p2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p1, cudaEnableDefault, &q1) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess ||
            cudaGetDriverEntryPoint("cuCtxGetId", &p2, cudaEnableDefault, &q2) != cudaSuccess ||
            q2 != cudaDriverEntryPointSuccess)
            return fail(PRISM_ERR_CUDA, "cuCtxGetCurrent / cuCtxGetId unavailable");
        get_current = reinterpret_cast<CtxGetCurrentFn>(p1);
        get_id = reinterpret_cast<CtxGetIdFn>(p2);
    }
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS) return fail(PRISM_ERR_CUDA, "cuCtxGetCurrent failed");
    if (!ctx) {  // the runtime has not made its primary context current on this thread yet
        int dev = 0;
        PRISM_CUDA_OK(cudaGetDevice(&dev));
        PRISM_CUDA_OK(cudaSetDevice(dev));
        if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return fail(PRISM_ERR_CUDA, "no current CUDA context");
    }
    if (get_id(ctx, id) != CUDA_SUCCESS) return fail(PRISM_ERR_CUDA, "cuCtxGetId failed");
    return PRISM_OK;
}
}  // namespace

// Once per CUDA context of a device, with that device current: the device
// address of the scratch array, kernel attributes and the candidate-shape
// table.
static prism_status noalloc_setup(int dev, unsigned char **out) {
    std::lock_guard<std::mutex> lock(g_setup_mu);
    unsigned long long ctx = 0;
    prism_status s = current_context_id(&ctx);
    if (s != PRISM_OK) return s;
    if (!g_scratch_ptr[dev] || g_scratch_ctx[dev] != ctx) {
        unsigned char *p = nullptr;
        PRISM_CUDA_OK(cudaGetSymbolAddress(reinterpret_cast<void **>(&p), g_noalloc_scratch));
        s = configure_zone_kernels();
        if (s != PRISM_OK) return s;
        g_scratch_ptr[dev] = p;
        g_scratch_ctx[dev] = ctx;
    }
    *out = g_scratch_ptr[dev];
    return PRISM_OK;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace prism

using namespace prism;

extern "C" PRISM_API prism_status prism_zone_shapes_noalloc(const prism_params *p, const void *V, const float *a_norm,
                                                            int *zone_B, int *zone_shape, void *stream) {
    if (!p || !V || !a_norm || !zone_B || !zone_shape)
        return fail(PRISM_ERR_INVALID_ARG, "NULL argument to prism_zone_shapes_noalloc");
    if (p->batch < 1 || p->T <= 0 || p->H <= 0 || p->W <= 0 || p->heads < 1 || p->T % 8 || p->H % 8 || p->W % 8)
        return fail(PRISM_ERR_INVALID_ARG, "grid must be positive multiples of 8 and batch, heads >= 1");
    if (p->head_dim != 64 && p->head_dim != 128)
        return fail(PRISM_ERR_UNSUPPORTED, "head_dim %d unsupported (64 or 128)", p->head_dim);
    if ((uintptr_t)V & 15) return fail(PRISM_ERR_INVALID_ARG, "V must be 16-byte aligned");
    if (p->hilbert_block) return fail(PRISM_ERR_UNSUPPORTED, "a Hilbert-order plan has no zone shapes");
    Geo g;
    g.batch = p->batch;
    g.T = p->T;
    g.H = p->H;
    g.W = p->W;
    g.heads = p->heads;
    g.D = p->head_dim;
    const long long N = (long long)p->T * p->H * p->W;
    if (N > (1ll << 26)) return fail(PRISM_ERR_UNSUPPORTED, "grid too large (N = %lld tokens)", N);
    g.N = (int)N;
    g.MT = p->T / 8;
    g.MH = p->H / 8;
    g.MW = p->W / 8;
    g.M = g.MT * g.MH * g.MW;
    g.nbmax = g.N / 64;
    g.C = p->heads * p->head_dim;
    if ((p->heads_total != 0 && p->heads_total != p->heads) || p->head_offset != 0)
        return fail(PRISM_ERR_UNSUPPORTED,
                    "prism_zone_shapes_noalloc takes every head of the layer (heads_total 0 or heads, head_offset 0)");
    g.Ctot = g.C;
    g.chunk0 = 0;
    g.nchunk_tot = (g.C + kStatChunk - 1) / kStatChunk;
    int fixed_idx = -1;
    if (p->fixed_shape[0] || p->fixed_shape[1] || p->fixed_shape[2]) {
        int table[kNumShapes][3];
        host_shape_table(table);
        for (int c = 0; c < kNumShapes; ++c)
            if ((1 << table[c][0]) == p->fixed_shape[0] && (1 << table[c][1]) == p->fixed_shape[1] &&
                (1 << table[c][2]) == p->fixed_shape[2])
                fixed_idx = c;
        if (fixed_idx < 0) return fail(PRISM_ERR_INVALID_ARG, "fixed_shape is not one of the 16 candidates");
    }
    // scratch layout
    const size_t B = (size_t)g.batch, M = (size_t)g.M, nbmax = (size_t)g.nbmax;
    const size_t nchunk = (size_t)(g.C + kStatChunk - 1) / kStatChunk;
    size_t off[11], o = 0;
    const size_t bytes[11] = {B * M * nchunk * 3 * sizeof(double), B * M * 5 * sizeof(double),
                              B * (M + 1) * sizeof(int),           B * sizeof(int),
                              B * (nbmax + 1) * sizeof(int),       B * nbmax * sizeof(int),
                              B * (M + 1) * sizeof(int),           B * sizeof(int),
                              B * nbmax * sizeof(int),             B * nbmax * sizeof(int),
                              0};
    for (int k = 0; k < 10; ++k) {
        off[k] = o;
        o += align256(bytes[k]);
    }
    if (o > PRISM_NOALLOC_SCRATCH_BYTES)
        return fail(PRISM_ERR_UNSUPPORTED, "problem needs %zu bytes of scratch; the fixed scratch holds %zu", o,
                    (size_t)PRISM_NOALLOC_SCRATCH_BYTES);
    int dev = -1;
    PRISM_CUDA_OK(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(PRISM_ERR_UNSUPPORTED, "device index %d out of range", dev);
    unsigned char *scr = nullptr;
    prism_status s = noalloc_setup(dev, &scr);
    if (s != PRISM_OK) return s;
    double eps = p->eps > 0.0 ? p->eps : 1e-6;
    return launch_zone_decisions(
        g, eps, fixed_idx, static_cast<const __nv_bfloat16 *>(V), a_norm, reinterpret_cast<double *>(scr + off[0]),
        reinterpret_cast<double *>(scr + off[1]), zone_B, zone_shape, reinterpret_cast<int *>(scr + off[2]),
        reinterpret_cast<int *>(scr + off[3]), reinterpret_cast<int *>(scr + off[4]),
        reinterpret_cast<int *>(scr + off[5]), reinterpret_cast<int *>(scr + off[6]),
        reinterpret_cast<int *>(scr + off[7]), reinterpret_cast<int *>(scr + off[8]),
        reinterpret_cast<int *>(scr + off[9]), static_cast<cudaStream_t>(stream));
}
