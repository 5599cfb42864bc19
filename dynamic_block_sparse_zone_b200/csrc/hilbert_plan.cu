// hilbert_plan.cu -- Hilbert-order fixed-block plans, the comparison baseline
// from the DFSAttn page (its first component: tokens reordered along a 3D
// Hilbert curve, so that neighbours in the order are neighbours in space and
// time, then grouped into blocks).
//
// The order depends on the grid alone, so it is built once when the plan is
// created; a build then only gathers Q, K, V through it, pools the blocks and
// selects (the selection and attention kernels are Prism's own).
//
// Curve: the one of the smallest 2^k cube holding the grid, restricted to the
// grid's tokens.  Index of a cube point (t, h, w): Skilling's method
// ("Programming the Hilbert curve", AIP Conf. Proc. 707, 2004) -- a pass over
// the bit levels from the top that inverts or exchanges the lower bits of the
// first coordinate, a Gray encoding across the coordinates, then the bits read
// level by level from the top, t's before h's before w's.
//
// Rank of a token along the curve without a sort: one flag per cube point
// (1 where a grid token sits), an exclusive scan of the flags, and the scan's
// value at the token's index.  The cube has at most 2^27 points (k <= 9).
#include "prism_internal.cuh"

namespace prism {

namespace {

__device__ __forceinline__ uint32_t hilbert3(uint32_t t, uint32_t h, uint32_t w, int k) {
    uint32_t c[3] = {t, h, w};
    const uint32_t top = 1u << (k - 1);
    for (uint32_t q = top; q > 1; q >>= 1) {
        const uint32_t low = q - 1;
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            if (c[i] & q) {
                c[0] ^= low;
            } else {
                const uint32_t x = (c[0] ^ c[i]) & low;
                c[0] ^= x;
                c[i] ^= x;
            }
        }
    }
    c[1] ^= c[0];
    c[2] ^= c[1];
    uint32_t flip = 0;
    for (uint32_t q = top; q > 1; q >>= 1)
        if (c[2] & q) flip ^= q - 1;
    uint32_t idx = 0;
    for (int b = k - 1; b >= 0; --b)
#pragma unroll
        for (int i = 0; i < 3; ++i) idx = (idx << 1) | (((c[i] ^ flip) >> b) & 1u);
    return idx;
}

__global__ void k_hilbert_flags(Geo g, int k, int *__restrict__ flags) {
    for (int n = blockIdx.x * blockDim.x + threadIdx.x; n < g.N; n += gridDim.x * blockDim.x) {
        const int t = n / (g.H * g.W), h = (n / g.W) % g.H, w = n % g.W;
        flags[hilbert3(t, h, w, k)] = 1;
    }
}

// perm[b][rank] = token for every sample (the order is the same for all).
__global__ void k_hilbert_perm(Geo g, int k, const int *__restrict__ rank, int *__restrict__ perm) {
    for (int n = blockIdx.x * blockDim.x + threadIdx.x; n < g.N; n += gridDim.x * blockDim.x) {
        const int t = n / (g.H * g.W), h = (n / g.W) % g.H, w = n % g.W;
        const int r = rank[hilbert3(t, h, w, k)];
        for (int b = 0; b < g.batch; ++b) perm[(size_t)b * g.N + r] = n;
    }
}

// Fixed blocks of B tokens: block table, 64-row tile map and 128-row tiles
// (two 64-token blocks share a tile, marked by the complement of the first).
__global__ void k_hilbert_tables(Geo g, int B, int *__restrict__ nb, int *__restrict__ blk_off,
                                 int *__restrict__ tile_blk, int *__restrict__ nqt, int *__restrict__ qt_row,
                                 int *__restrict__ qt_blk) {
    const int nbk = g.N / B, tpb = B >= 128 ? B / 128 : 1;
    const int b = blockIdx.y;
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j <= nbk; j += gridDim.x * blockDim.x) {
        blk_off[(size_t)b * (g.nbmax + 1) + j] = j * B;
        if (j == nbk) {
            nb[b] = nbk;
            nqt[b] = B == 64 ? nbk / 2 : nbk * tpb;
            continue;
        }
        for (int u = 0; u < B / kTile; ++u) tile_blk[(size_t)b * g.nbmax + j * (B / kTile) + u] = j;
        if (B == 64) {
            if ((j & 1) == 0) {
                qt_row[(size_t)b * g.nbmax + j / 2] = j * B;
                qt_blk[(size_t)b * g.nbmax + j / 2] = ~j;
            }
            continue;
        }
        for (int r = 0; r < tpb; ++r) {
            qt_row[(size_t)b * g.nbmax + j * tpb + r] = j * B + r * 128;
            qt_blk[(size_t)b * g.nbmax + j * tpb + r] = j;
        }
    }
}

}  // namespace

int hilbert_level(const Geo &g) {
    int k = 1;
    while ((1 << k) < g.T || (1 << k) < g.H || (1 << k) < g.W) ++k;
    return k;
}

prism_status setup_hilbert_plan(Plan &pl) {
    const Geo &g = pl.g;
    const int k = hilbert_level(g);
    const size_t cube = (size_t)1 << (3 * k);
    int *flags = nullptr, *rank = nullptr, *tmp = nullptr;
    cudaError_t e = cudaMalloc(&flags, cube * sizeof(int));
    if (e == cudaSuccess) e = cudaMalloc(&rank, (cube + 1) * sizeof(int));
    if (e == cudaSuccess) e = cudaMalloc(&tmp, ((cube + 1023) / 1024 + 1) * sizeof(int));
    prism_status s = PRISM_OK;
    if (e == cudaSuccess) e = cudaMemset(flags, 0, cube * sizeof(int));
    if (e == cudaSuccess) {
        k_hilbert_flags<<<1184, 256>>>(g, k, flags);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) s = scan_ints(flags, cube, rank, tmp, 0);
    if (e == cudaSuccess && s == PRISM_OK) {
        k_hilbert_perm<<<1184, 256>>>(g, k, rank, pl.perm);
        const int B = pl.p.hilbert_block;
        k_hilbert_tables<<<dim3((g.N / B + 256) / 256, g.batch), 256>>>(g, B, pl.nb, pl.blk_off, pl.tile_blk, pl.nqt,
                                                                     pl.qt_row, pl.qt_blk);
        e = cudaGetLastError();
    }
    // zones are not used: volume 0 and shape -1 in the plan's view
    if (e == cudaSuccess) e = cudaMemset(pl.zone_B, 0, (size_t)g.batch * g.M * sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(pl.zone_shape, 0xFF, (size_t)g.batch * g.M * sizeof(int));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    cudaFree(flags);
    cudaFree(rank);
    cudaFree(tmp);
    if (e != cudaSuccess) return fail_cuda(e, "Hilbert order setup", __FILE__, __LINE__);
    return s;
}

}  // namespace prism
