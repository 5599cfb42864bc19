// attn_bwd_aux.cu -- the memory-bound steps around the tensor-core backward:
//   k_attn_bwd_pre   Delta_q = rowsum(dO_q * O_q) from the forward's bf16 O and
//                    the block-contiguous, head-major copy of dO
//   k_dq_finalize    fp32 dQ accumulator (block-contiguous) -> bf16 dQ in the
//                    caller's raster layout
// and the launcher of the whole backward [Prism guide, Method section 3; the
// standard softmax-attention gradient through the selected block pairs].
#include "prism_internal.cuh"

namespace prism {

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// ---------------------------------------------------------------------------
// backward, part 1: Delta = rowsum(dO * O) and the permuted copy of dO
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) k_attn_bwd_pre(Geo g, const __nv_bfloat16 *__restrict__ O,
                                                      const __nv_bfloat16 *__restrict__ dO,
                                                      const int *__restrict__ perm, __nv_bfloat16 *__restrict__ dOp,
                                                      float *__restrict__ delta) {
    constexpr int L = D / 8;  // lanes per (token, head)
    const int b = blockIdx.y;
    const int G = g.C / 8;
    const size_t items = (size_t)kTile * G;
    for (size_t it = threadIdx.x; it < items; it += blockDim.x) {
        const int nl = (int)(it / G), grp = (int)(it % G);
        const int n = blockIdx.x * kTile + nl;
        const int tok = perm[(size_t)b * g.N + n];
        const size_t src = ((size_t)b * g.N + tok) * g.C + grp * 8;
        const uint4 ov = *reinterpret_cast<const uint4 *>(O + src);
        const uint4 dv = *reinterpret_cast<const uint4 *>(dO + src);
        const int hd = grp * 8 / D, d0 = grp * 8 % D;
        const size_t bh = (size_t)b * g.heads + hd;
        *reinterpret_cast<uint4 *>(dOp + (bh * g.N + n) * D + d0) = dv;
        const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w}, dw[4] = {dv.x, dv.y, dv.z, dv.w};
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            acc += __uint_as_float(ow[k] << 16) * __uint_as_float(dw[k] << 16);
            acc += __uint_as_float(ow[k] & 0xffff0000u) * __uint_as_float(dw[k] & 0xffff0000u);
        }
#pragma unroll
        for (int o2 = L / 2; o2 > 0; o2 >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o2, L);
        if ((threadIdx.x & (L - 1)) == 0) delta[bh * g.N + n] = acc;
    }
}

// dQ (fp32, permuted, head-major) -> bf16 user layout
template <int D>
__global__ void __launch_bounds__(256) k_dq_finalize(Geo g, const float *__restrict__ dQacc,
                                                     const int *__restrict__ perm, __nv_bfloat16 *__restrict__ dQ) {
    const int b = blockIdx.y;
    const int G = g.C / 8;
    const size_t items = (size_t)kTile * G;
    for (size_t it = threadIdx.x; it < items; it += blockDim.x) {
        const int nl = (int)(it / G), grp = (int)(it % G);
        const int n = blockIdx.x * kTile + nl;
        const int hd = grp * 8 / D, d0 = grp * 8 % D;
        const size_t bh = (size_t)b * g.heads + hd;
        const float4 *src = reinterpret_cast<const float4 *>(dQacc + (bh * g.N + n) * D + d0);
        const float4 x = src[0], y = src[1];
        uint4 v;
        v.x = pack_bf16(x.x, x.y);
        v.y = pack_bf16(x.z, x.w);
        v.z = pack_bf16(y.x, y.y);
        v.w = pack_bf16(y.z, y.w);
        const int tok = perm[(size_t)b * g.N + n];
        *reinterpret_cast<uint4 *>(dQ + ((size_t)b * g.N + tok) * g.C + grp * 8) = v;
    }
}

// ---------------------------------------------------------------------------
// launcher
// ---------------------------------------------------------------------------
template <int D>
static prism_status bwd_impl(Plan &pl, const void *O, const void *dO, void *dQ, void *dK, void *dV,
                             cudaStream_t st) {
    const Geo &g = pl.g;
    PRISM_CUDA_OK(cudaMemsetAsync(pl.dQacc, 0, (size_t)g.batch * g.heads * g.N * D * sizeof(float), st));
    {
        TimerScope ts(pl, kTBwdPre, st);
        k_attn_bwd_pre<D><<<dim3(g.nbmax, g.batch), 256, 0, st>>>(g, static_cast<const __nv_bfloat16 *>(O),
                                                                 static_cast<const __nv_bfloat16 *>(dO), pl.perm,
                                                                 pl.dOp, pl.delta);
        PRISM_CUDA_OK(cudaGetLastError());
    }
    prism_status s = launch_attn_bwd_tc_main(pl, dK, dV, st);
    if (s != PRISM_OK) return s;
    TimerScope ts(pl, kTDqFinal, st);
    k_dq_finalize<D><<<dim3(g.nbmax, g.batch), 256, 0, st>>>(g, pl.dQacc, pl.perm,
                                                            static_cast<__nv_bfloat16 *>(dQ));
    PRISM_CUDA_OK(cudaGetLastError());
    return PRISM_OK;
}

prism_status launch_attn_bwd(Plan &pl, const void *O, const void *dO, void *dQ, void *dK, void *dV,
                             cudaStream_t st) {
    return pl.g.D == 64 ? bwd_impl<64>(pl, O, dO, dQ, dK, dV, st) : bwd_impl<128>(pl, O, dO, dQ, dK, dV, st);
}

}  // namespace prism
