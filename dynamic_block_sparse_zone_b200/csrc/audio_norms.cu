// audio_norms.cu -- the audio guidance of the plan, a_{t,h,w} = ||h^_{t,h,w}||_2
// [Prism guide, Method section 1, the sentence before the g_d equation]: the
// L2 norm over the channels of the audio-to-video cross-attention output of
// every video token, which a layer caches for the next layer's plan.
//
// HBM-bound: one read of h (rows x C bf16), one fp32 write per row.  One warp
// per row; with C a multiple of 8 and h 16-byte aligned each lane reads 16
// bytes (8 channels) per step, otherwise one channel per lane and step.
// Squares of bf16 values are exact in fp32; they are summed in eight partial
// sums per lane and then across the warp (relative error of the sum below
// (C/256 + 8) * 2^-24).
#include "prism_internal.cuh"

namespace prism {

namespace {
constexpr int kWarps = 8;  // rows per CTA

__global__ void __launch_bounds__(kWarps * 32) k_audio_norms(const __nv_bfloat16 *__restrict__ h,
                                                             float *__restrict__ a, long long rows, int C,
                                                             bool vec) {
    const int lane = threadIdx.x & 31;
    const long long stride = (long long)gridDim.x * kWarps;
    for (long long r = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5); r < rows; r += stride) {
        const __nv_bfloat16 *row = h + r * (long long)C;
        float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (vec) {
            const uint4 *v = reinterpret_cast<const uint4 *>(row);
            for (int i = lane; i < C / 8; i += 32) {
                const uint4 u = __ldg(v + i);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float lo = __uint_as_float(w[k] << 16), hi = __uint_as_float(w[k] & 0xFFFF0000u);
                    s[2 * k] = fmaf(lo, lo, s[2 * k]);
                    s[2 * k + 1] = fmaf(hi, hi, s[2 * k + 1]);
                }
            }
        } else {
            for (int c = lane, k = 0; c < C; c += 32, k = (k + 1) & 7) {
                const float x = __bfloat162float(row[c]);
                s[k] = fmaf(x, x, s[k]);
            }
        }
        float t = ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if (lane == 0) a[r] = sqrtf(t);
    }
}
}  // namespace

prism_status launch_audio_norms(const void *h, float *a, long long rows, int C, cudaStream_t st) {
    if (rows == 0) return PRISM_OK;
    const long long blocks = (rows + kWarps - 1) / kWarps;
    const int grid = (int)(blocks < 148 * 32 ? blocks : 148 * 32);
    const bool vec = (C % 8) == 0 && (reinterpret_cast<uintptr_t>(h) & 15) == 0;
    k_audio_norms<<<grid, kWarps * 32, 0, st>>>(static_cast<const __nv_bfloat16 *>(h), a, rows, C, vec);
    PRISM_CUDA_OK(cudaGetLastError());
    return PRISM_OK;
}

}  // namespace prism
