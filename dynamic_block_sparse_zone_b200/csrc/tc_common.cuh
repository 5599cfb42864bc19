// tc_common.cuh -- sm_100a building blocks used by the tensor-core attention
// kernels: mbarriers with bounded waits, 2D TMA loads (no multicast), TMEM
// allocation, tcgen05.mma (kind::f16, bf16 in / fp32 accumulate), commits and
// TMEM loads / stores, and the shared-memory matrix descriptors.
//
// Every wait on an mbarrier is bounded: after kSpinLimit polls it records an
// error code and the wait site in the plan's status word and raises the CTA's
// abort flag; the kernel then winds down without touching further work.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "prism_internal.cuh"

namespace prism {
namespace tc {

constexpr long long kSpinLimit = 1ll << 18;  // ~1 s: each unsatisfied try_wait suspends a few microseconds
constexpr int kErrTimeout = 1;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarriers ----
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Waits for the phase of `parity` to complete; false on timeout or abort.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int *status, int site,
                                          volatile int *abort_flag) {
    for (long long it = 0; it < kSpinLimit; ++it) {
        if (mbar_try(bar, parity)) return true;
        if ((it & 255) == 255 && *abort_flag) return false;
    }
    if (atomicCAS(status, 0, kErrTimeout) == 0) status[1] = site;
    *abort_flag = 1;
    return false;
}

// ---- the block lists a 128-row tile streams ----
// A tile holds one block (qt_blk = j) or the two 64-token blocks j, j+1
// (qt_blk = ~j); j2 = -1 when there is no second block.
__device__ __forceinline__ void tile_blocks(int code, int &j1, int &j2) {
    j1 = code < 0 ? ~code : code;
    j2 = code < 0 ? j1 + 1 : -1;
}
// Is j in the ascending list L[0..n)?
__device__ __forceinline__ bool sorted_has(const int *L, int n, int j) {
    int lo = 0, hi = n - 1;
    while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        const int v = L[mid];
        if (v == j) return true;
        if (v < j) lo = mid + 1;
        else hi = mid - 1;
    }
    return false;
}
// 64-row segments of the union of two ascending block lists (every lane of
// the warp gets the total).
__device__ __forceinline__ int union_segments(const int *A, int na, const int *B, int nb, const int *bo, int lane) {
    int n = 0;
    for (int u = lane; u < na; u += 32) n += (bo[A[u] + 1] - bo[A[u]]) >> 6;
    for (int u = lane; u < nb; u += 32)
        if (!sorted_has(A, na, B[u])) n += (bo[B[u] + 1] - bo[B[u]]) >> 6;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
    return n;
}
// Walk over those segments in ascending block order, the two lists being the
// index ranges [ua, a_end) and [ub, b_end) of one array L: r is the
// segment's first block-contiguous row, mask bit 0 / bit 1 say whether its
// block is in the first / second list.  L and the block offsets bo are passed
// to each step rather than kept (the kernels are short of registers).
struct SegWalk {
    int ua, a_end, ub, b_end;
    int r, r_end, mask;
    __device__ __forceinline__ void pick(const int *L, const int *bo) {
        const int ja = ua < a_end ? L[ua] : 0x7fffffff, jb = ub < b_end ? L[ub] : 0x7fffffff;
        const int j = min(ja, jb);
        mask = (ja == j ? 1 : 0) | (jb == j ? 2 : 0);
        ua += ja == j;
        ub += jb == j;
        if (j != 0x7fffffff) {
            r = bo[j];
            r_end = bo[j + 1];
        } else {
            r = r_end = 0;
            mask = 0;
        }
    }
    __device__ __forceinline__ void init(int a0, int a1, int b0, int b1, const int *L, const int *bo) {
        ua = a0;
        a_end = a1;
        ub = b0;
        b_end = b1;
        pick(L, bo);
    }
    __device__ __forceinline__ void advance(const int *L, const int *bo) {
        r += 64;
        if (r >= r_end) pick(L, bo);
    }
};

// ---- TMA (2D tiled, this GPU's own memory, no multicast) ----
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];\n" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}
// 1D bulk copy global -> shared (16-byte aligned, size a multiple of 16)
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}
// 2D tiled reduce-add of a shared-memory tile into global memory (fp32 add),
// tracked by the bulk-group of the issuing thread.
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap *map, uint32_t src, int x, int y) {
    asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%2, %3}], [%1];\n" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;\n" ::: "memory"); }
// the sources of every committed bulk group have been read (smem reusable)
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory"); }
// every committed bulk group has completed (writes visible in global memory)
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory"); }
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(nthreads) : "memory");
}
// shared-memory accesses by 32-bit shared-window address
__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];\n" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ void sts_u4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ void sts_f32(uint32_t addr, float v) {
    asm volatile("st.shared.f32 [%0], %1;\n" ::"r"(addr), "f"(v) : "memory");
}
// generic-proxy shared-memory writes -> visible to the async proxy (tensor cores)
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }
__device__ __forceinline__ void prefetch_map(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- TMEM ----
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n"
                 :
                 : "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
                 : "memory");
}

// ---- MMA ----
// The issuing helpers are executed by a whole, converged warp: operands are
// warp-uniform and elect.sync picks the single lane that issues.  The same
// lane is elected every time (lowest lane of a full mask), so a commit tracks
// the MMAs issued before it.  kind::f16: D[tmem] (+)= A * B^T, one CTA.
// Batched issue.  A run of MMAs issued from ONE inline-asm block, with the
// descriptor steps computed inside it, issues at the tensor-core rate on
// sm_100a; the same MMAs issued one asm block each measured 1.5-2x slower per
// instruction (an issue-rate probe: 8 x M128 N128 K16 smem-operand MMAs took
// 64 cycles each batched and about 105 one by one).  Offsets are template
// immediates: descriptor offsets in 16-byte units (the start-address field),
// TMEM offsets in columns.  The first MMA of a run takes `accumulate`; the
// rest accumulate.
#define PRISM_MMA_HEAD                   \
    "{\n\t.reg .pred p, e, t;\n\t"       \
    ".reg .b64 x, y;\n\t.reg .b32 z;\n\t" \
    "setp.ne.b32 p, %4, 0;\n\t"          \
    "setp.ne.b32 t, %3, 0;\n\t"          \
    "elect.sync _|e, 0xffffffff;\n\t"
#define PRISM_MMA_SS_FIRST "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
#define PRISM_MMA_SS_NEXT(ia, ib) \
    "add.s64 x, %1, %" #ia ";\n\tadd.s64 y, %2, %" #ib ";\n\t@e tcgen05.mma.cta_group::1.kind::f16 [%0], x, y, %3, t;\n\t"

// Eight smem-operand MMAs into one accumulator: A = a + A_i, B = b + B_i.
template <uint32_t A1, uint32_t A2, uint32_t A3, uint32_t A4, uint32_t A5, uint32_t A6, uint32_t A7, uint32_t B1,
          uint32_t B2, uint32_t B3, uint32_t B4, uint32_t B5, uint32_t B6, uint32_t B7>
__device__ __forceinline__ void mma_ss8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(PRISM_MMA_HEAD PRISM_MMA_SS_FIRST PRISM_MMA_SS_NEXT(5, 12) PRISM_MMA_SS_NEXT(6, 13)
                     PRISM_MMA_SS_NEXT(7, 14) PRISM_MMA_SS_NEXT(8, 15) PRISM_MMA_SS_NEXT(9, 16)
                         PRISM_MMA_SS_NEXT(10, 17) PRISM_MMA_SS_NEXT(11, 18) "}\n" ::"r"(d_tmem),
                 "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "n"(A1), "n"(A2), "n"(A3), "n"(A4), "n"(A5),
                 "n"(A6), "n"(A7), "n"(B1), "n"(B2), "n"(B3), "n"(B4), "n"(B5), "n"(B6), "n"(B7)
                 : "memory");
}
// Four smem-operand MMAs into one accumulator.
template <uint32_t A1, uint32_t A2, uint32_t A3, uint32_t B1, uint32_t B2, uint32_t B3>
__device__ __forceinline__ void mma_ss4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(PRISM_MMA_HEAD PRISM_MMA_SS_FIRST PRISM_MMA_SS_NEXT(5, 8) PRISM_MMA_SS_NEXT(6, 9)
                     PRISM_MMA_SS_NEXT(7, 10) "}\n" ::"r"(d_tmem),
                 "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "n"(A1), "n"(A2), "n"(A3), "n"(B1), "n"(B2),
                 "n"(B3)
                 : "memory");
}
#define PRISM_MMA_TS_FIRST(dd) "@e tcgen05.mma.cta_group::1.kind::f16 [%" #dd "], [%1], %2, %3, p;\n\t"
#define PRISM_MMA_TS_NEXT(dd, ia, ib, pr)                                                 \
    "add.u32 z, %1, %" #ia ";\n\tadd.s64 y, %2, %" #ib ";\n\t@e tcgen05.mma.cta_group::1.kind::f16 [%" #dd \
    "], [z], y, %3, " #pr ";\n\t"
#define PRISM_MMA_TS2_FIRST "@e tcgen05.mma.cta_group::1.kind::f16 [%5], [%6], %7, %3, p;\n\t"
#define PRISM_MMA_TS2_NEXT(ia, ib)                                                                   \
    "add.u32 z, %6, %" #ia ";\n\tadd.s64 y, %7, %" #ib ";\n\t@e tcgen05.mma.cta_group::1.kind::f16 [%5], [z], y, %3, " \
    "t;\n\t"
// Two runs of four MMAs with A from TMEM and B from shared memory, the same
// steps in both: d0 (+)= [a0 + A_i] * (b0 + B_i), then d1 (+)= [a1 + A_i] *
// (b1 + B_i).  Each run's first MMA takes `accumulate`.
template <uint32_t A1, uint32_t A2, uint32_t A3, uint32_t B1, uint32_t B2, uint32_t B3>
__device__ __forceinline__ void mma_ts4x2(uint32_t d0, uint32_t a0, uint64_t b0, uint32_t d1, uint32_t a1,
                                          uint64_t b1, uint32_t idesc, uint32_t accumulate) {
    asm volatile(PRISM_MMA_HEAD PRISM_MMA_TS_FIRST(0) PRISM_MMA_TS_NEXT(0, 8, 11, t) PRISM_MMA_TS_NEXT(0, 9, 12, t)
                     PRISM_MMA_TS_NEXT(0, 10, 13, t) PRISM_MMA_TS2_FIRST PRISM_MMA_TS2_NEXT(8, 11)
                         PRISM_MMA_TS2_NEXT(9, 12) PRISM_MMA_TS2_NEXT(10, 13) "}\n" ::"r"(d0),
                 "r"(a0), "l"(b0), "r"(idesc), "r"(accumulate), "r"(d1), "r"(a1), "l"(b1), "n"(A1), "n"(A2), "n"(A3),
                 "n"(B1), "n"(B2), "n"(B3)
                 : "memory");
}
// Four MMAs with A from TMEM into one accumulator.
template <uint32_t A1, uint32_t A2, uint32_t A3, uint32_t B1, uint32_t B2, uint32_t B3>
__device__ __forceinline__ void mma_ts4(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(PRISM_MMA_HEAD PRISM_MMA_TS_FIRST(0) PRISM_MMA_TS_NEXT(0, 5, 8, t) PRISM_MMA_TS_NEXT(0, 6, 9, t)
                     PRISM_MMA_TS_NEXT(0, 7, 10, t) "}\n" ::"r"(d_tmem),
                 "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate), "n"(A1), "n"(A2), "n"(A3), "n"(B1), "n"(B2),
                 "n"(B3)
                 : "memory");
}

// Arrive on `bar` once every MMA issued so far by the elected lane completes.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}\n" ::"r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format: start
// address, leading / stride byte offsets in 16-byte units, version 1,
// layout type 2 = SWIZZLE_128B).  K-major operands: rows of 128 B, 8-row
// groups `sbo` apart (lbo unused).  MN-major operands: 64-element runs along
// M/N `lbo` apart, 8-row groups along K `sbo` apart.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B,
// each operand K-major or MN-major (A from TMEM must be K-major), shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major, bool a_mn_major = false) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %2, %1;\n" : "=r"(r) : "f"(lo), "f"(hi));
    return r;
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic): one instruction for two lanes,
// where the softmax loops are instruction-issue bound.  (y0, y1) = (x0, x1) * s2 + c2.
__device__ __forceinline__ void fma2(float x0, float x1, uint64_t s2, uint64_t c2, float &y0, float &y1) {
    asm("{\n\t.reg .b64 x, y;\n\tmov.b64 x, {%2, %3};\n\tfma.rn.f32x2 y, x, %4, %5;\n\tmov.b64 {%0, %1}, y;\n\t}\n"
        : "=f"(y0), "=f"(y1)
        : "f"(x0), "f"(x1), "l"(s2), "l"(c2));
}
// (d0, d1) = (p0, p1) * ((a0, a1) - (b0, b1)), each step rounded as in scalar code
__device__ __forceinline__ void mul_sub2(float p0, float p1, float a0, float a1, float b0, float b1, float &d0,
                                         float &d1) {
    asm("{\n\t.reg .b64 p, a, b, t;\n\tmov.b64 p, {%2, %3};\n\tmov.b64 a, {%4, %5};\n\tmov.b64 b, {%6, %7};\n\t"
        "sub.rn.f32x2 t, a, b;\n\tmul.rn.f32x2 t, p, t;\n\tmov.b64 {%0, %1}, t;\n\t}\n"
        : "=f"(d0), "=f"(d1)
        : "f"(p0), "f"(p1), "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ uint64_t pair2(float lo, float hi) {
    return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}
// acc2 += (p0, p1)
__device__ __forceinline__ void add2(uint64_t &acc2, float p0, float p1) {
    asm("{\n\t.reg .b64 p;\n\tmov.b64 p, {%1, %2};\n\tadd.rn.f32x2 %0, %0, p;\n\t}\n" : "+l"(acc2) : "f"(p0), "f"(p1));
}
__device__ __forceinline__ uint64_t splat2(float v) {
    return (uint64_t)__float_as_uint(v) | ((uint64_t)__float_as_uint(v) << 32);
}
__device__ __forceinline__ float sum2(uint64_t acc2) {
    return __uint_as_float((uint32_t)acc2) + __uint_as_float((uint32_t)(acc2 >> 32));
}
// max of three
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;\n" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace tc
}  // namespace prism
