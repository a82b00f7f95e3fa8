// Thin inline-PTX wrappers for sm_100a: mbarriers, TMA (tiled and bulk), tcgen05
// (TMEM allocation, MMA, scale-factor copy, loads), and the bounded waits every
// kernel in this library uses.  No waiting loop here can spin forever: each gives up
// after FT_WAIT_NS nanoseconds of the global timer and reports it to the caller.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ft {

// Device status word values (mirrors ft_status in include/fourtune.h).
constexpr int kStatusOk = 0;
constexpr int kStatusTimeout = 7;

// A bounded wait gives up after this long (2 s): far above any legitimate wait in
// these kernels (microseconds), far below anything that looks like a hang.
#ifndef FT_WAIT_NS
#define FT_WAIT_NS 2000000000ull
#endif

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Programmatic dependent launch: let the next kernel on the stream be scheduled now /
// wait until every kernel this one depends on has completed and its writes are visible.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete.  Returns false (and waits no
// longer) if `abort_flag` becomes non-zero or FT_WAIT_NS elapses; in the timeout case
// it also raises the CTA's abort flag and the global status word.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int* status, uint64_t limit_ns = FT_WAIT_NS) {
#pragma unroll 1
    for (int i = 0; i < 256; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
#pragma unroll 1
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit_ns) {
            *abort_flag = 1;
            if (status) atomicExch(status, kStatusTimeout);
            return false;
        }
    }
}

// ---------------------------------------------------------------------------
// TMA
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled load of the box at (x = inner coordinate in elements, y = row) into smem.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                           int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

// 2-D tiled store of an smem box to global (x inner coordinate, y row).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int32_t x,
                                            int32_t y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_group_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// The bulk groups this thread committed, except the most recent one, have finished
// reading their shared-memory source (double-buffered staging).
__device__ __forceinline__ void bulk_wait_group_read1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(p)));
}

__device__ __forceinline__ void bulk_wait_group0() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Contiguous bulk copy global -> smem (both 16-byte aligned, bytes % 16 == 0).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05 (5th-generation tensor cores, accumulators in tensor memory)
// ---------------------------------------------------------------------------
// Tensor memory address: bits 31..16 lane, bits 15..0 column (32-bit columns).
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, 16-bit inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= (A * SFA) * (B * SFB)^T with packed E2M1 operands and one UE4M3 scale per
// 16 elements along K (scales read from tensor memory).
__device__ __forceinline__ void mma_fp4_block16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                uint32_t idesc, uint32_t sfa_tmem,
                                                uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], "
        "p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Arrive on an mbarrier once every tcgen05 operation this thread issued so far is done.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

// Each thread of the warp reads 32 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// Each thread of the warp writes 16 consecutive 32-bit columns of its own TMEM lane
// (lane = the warp's quarter base + lane id).
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------
// CTA pairs (clusters of two CTAs sharing one tcgen05.mma.cta_group::2)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(addr), "r"(rank));
    return out;
}

// Arrive on an mbarrier given by its shared::cluster address (this CTA's or the peer's).
// Default (cta-scope) release: a cluster-scope release costs ~8x as much (~450 cycles on
// B200); what the waiter reads next is tensor memory and TMA-written shared memory, ordered
// by the tcgen05 fences and the barrier itself.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// 256-row block-scaled MMA over the pair: A rows 0..127 from this CTA's shared memory and
// 128..255 from the peer's (same offsets), B's N rows split the same way; each CTA's
// tensor memory holds its 128 accumulator rows and its own scale factors.
__device__ __forceinline__ void mma_fp4_block16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                     uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                                     uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], "
        "p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on the barrier at shared::cluster address `bar` (either CTA of the pair)
// when every tcgen05 operation this thread issued so far is complete.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// The same commit arriving once on the mbarrier at this shared-memory offset in both CTAs
// of the pair (CTA mask 0b11): one tensor-pipe commit instead of two.  An arrival, not a
// data movement: no memory is read through the multicast.
__device__ __forceinline__ void tc_commit_pair_both(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
        "h"(static_cast<uint16_t>(3))
        : "memory");
}

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: rows of 128 bytes, groups
// of 8 rows 1024 bytes apart.  Stepping along K inside the 128-byte row is done by
// advancing the start address (16-byte units).
__device__ __forceinline__ uint64_t sdesc_kmajor_sw128(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFF);  // start address
    d |= static_cast<uint64_t>(1) << 16;                    // leading byte offset (unused)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;            // stride byte offset: 8-row group
    d |= static_cast<uint64_t>(1) << 46;                    // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2) << 61;                    // 128-byte swizzle
    return d;
}

// Shared-memory descriptor, MN-major, 128-byte swizzle: 128-byte rows run along M (or
// N), 8 consecutive K rows form a 1024-byte swizzle atom.  `lbo` is the byte distance
// between 64-element MN chunks, `sbo` between 8-row K groups.
__device__ __forceinline__ uint64_t sdesc_mnmajor_sw128(uint32_t smem_addr, uint32_t lbo,
                                                        uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFF);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// Instruction descriptor, kind::f16 with bf16 inputs and fp32 accumulation, both
// operands K-major unless a_mn / b_mn.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn = false,
                                                  bool b_mn = false) {
    return (1u << 4)                      // D format fp32
           | (1u << 7)                    // A bf16
           | (1u << 10)                   // B bf16
           | ((a_mn ? 1u : 0u) << 15)     // A major
           | ((b_mn ? 1u : 0u) << 16)     // B major
           | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor, kind::mxf4nvf4 with E2M1 A and B, UE4M3 scales per 16
// elements, dense K = 64, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_fp4_block16(int M, int N) {
    return (1u << 7)      // A E2M1
           | (1u << 10)   // B E2M1
           | (static_cast<uint32_t>(N >> 3) << 17)
           | (0u << 23)   // scale format UE4M3
           | (static_cast<uint32_t>(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// Conversions
// ---------------------------------------------------------------------------
// Two fp32 -> one byte of E2M1 codes, round-to-nearest-even, saturating; `lo` goes to
// the low nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .b8 b;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\t"
        "cvt.u32.u8 %0, b;\n\t}"
        : "=r"(out)
        : "f"(hi), "f"(lo));
    return out;
}

// Eight fp32 -> eight E2M1 codes in one 32-bit word (element i in nibble i), each
// round-to-nearest-even and saturating.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&v)[8]) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return out;
}

// The IEEE fp32 quotient a / 6 for a = any finite bf16 value, without a division: the
// product with RN(1/6) plus one Markstein correction step (the residual a - 6 q0 is
// exact in an FMA).  Identical to a / 6 for all 2^15 non-negative bf16 inputs (checked
// exhaustively against the IEEE division).
__device__ __forceinline__ float div6_bf16(float a) {
    const float r6 = 0.16666667163372040f;  // RN(1/6)
    const float q0 = __fmul_rn(a, r6);
    const float res = __fmaf_rn(-6.0f, q0, a);
    return __fmaf_rn(res, r6, q0);
}

// fp32 (non-negative) -> UE4M3 code, round-to-nearest-even, saturating at 448.
__device__ __forceinline__ uint32_t cvt_ue4m3(float v) {
    uint16_t out;
    asm volatile("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(v));
    return out & 0xFFu;
}

// Exact fp32 value of a UE4M3 code.
__device__ __forceinline__ float ue4m3_to_f32(uint32_t code) {
    uint32_t h2;
    const uint16_t c = static_cast<uint16_t>(code & 0xFF);
    asm volatile("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFF)));
}

// GELU, tanh form: 0.5 p (1 + tanh(u)), u = sqrt(2/pi) (p + 0.044715 p^3), evaluated as
// p * sigmoid(2u), the same function (0.5 (1 + tanh u) = 1 / (1 + exp(-2u))), which keeps
// full relative accuracy for large negative p where 1 + tanh(u) cancels.  The exponential
// and the divisions are CUDA's fast intrinsics (__expf, __fdividef: a few ulp, ~1e-6
// relative for the arguments that reach a bf16 result), so the GEMM epilogue that applies
// it stays cheap next to the tile's MMAs; the polynomial steps are explicitly rounded.
// The stand-alone kernels use these same functions, so they and the epilogue agree bit
// for bit.  For |2u| beyond the fp32 exp range the sigmoid goes to 0 or 1 as it should
// (__fdividef(x, inf) = 0).  The derivative: dP = dH * gelu'(P) with s = sigmoid(2u),
// gelu' = s + 2 p s (1 - s) u'; with e = exp(-2u), s = 1 / (1 + e) and 1 - s = e s (one
// exponential and one reciprocal: the special-function pipe bounds that epilogue), the
// exponent capped at 80 so e stays finite (then s ~ 1e-35 and e s = 1 to within rounding).
// The arithmetic runs on packed fp32 pairs (the GELU epilogues are issue-bound: two
// elements per instruction), each lane rounded to nearest as __fmul_rn / __fadd_rn do;
// only the exponential and the divisions are per element.
struct F2 {
    float a, b;
};
__device__ __forceinline__ F2 f2_mul(F2 x, F2 y) {
    F2 r;
    asm("{\n\t.reg .b64 p, q, z;\n\tmov.b64 p, {%2, %3};\n\tmov.b64 q, {%4, %5};\n\t"
        "mul.rn.f32x2 z, p, q;\n\tmov.b64 {%0, %1}, z;\n\t}"
        : "=f"(r.a), "=f"(r.b)
        : "f"(x.a), "f"(x.b), "f"(y.a), "f"(y.b));
    return r;
}
__device__ __forceinline__ F2 f2_add(F2 x, F2 y) {
    F2 r;
    asm("{\n\t.reg .b64 p, q, z;\n\tmov.b64 p, {%2, %3};\n\tmov.b64 q, {%4, %5};\n\t"
        "add.rn.f32x2 z, p, q;\n\tmov.b64 {%0, %1}, z;\n\t}"
        : "=f"(r.a), "=f"(r.b)
        : "f"(x.a), "f"(x.b), "f"(y.a), "f"(y.b));
    return r;
}
__device__ __forceinline__ F2 f2(float v) { return F2{v, v}; }

// u = sqrt(2/pi) (p + 0.044715 p^3) of both lanes, each step rounded; p2 = p * p is
// returned for reuse
__device__ __forceinline__ F2 gelu_tanh_u2(F2 p, F2& p2) {
    p2 = f2_mul(p, p);
    return f2_mul(f2(0.7978845608028654f), f2_add(p, f2_mul(f2(0.044715f), f2_mul(p2, p))));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t out;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(out) : "f"(hi), "f"(lo));
    return out;
}

// Two fp32 products rounded to nearest in one packed instruction: (a * s, b * s).
__device__ __forceinline__ void mul2_rn(float a, float b, float s, float& ra, float& rb) {
    asm("{\n\t.reg .b64 x, y, z;\n\tmov.b64 x, {%2, %3};\n\tmov.b64 y, {%4, %4};\n\t"
        "mul.rn.f32x2 z, x, y;\n\tmov.b64 {%0, %1}, z;\n\t}"
        : "=f"(ra), "=f"(rb)
        : "f"(a), "f"(b), "f"(s));
}

// Per 16-bit half: a bf16 whose magnitude is max(|a|, |b|) (sign bit meaningless; NaN
// inputs are outside the domain: the other operand wins).
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two packed bf16 gradients dh -> bf16(dh * gelu_tanh'(p)) each (p: two packed bf16).
__device__ __forceinline__ uint32_t gelu_bwd_bf16x2(uint32_t dh, uint32_t p) {
    const F2 P{bf16lo_to_f32(p), bf16hi_to_f32(p)};
    F2 pp;
    const F2 u = gelu_tanh_u2(P, pp);
    const F2 m2u = f2_mul(f2(-2.0f), u);
    const F2 e{__expf(fminf(m2u.a, 80.0f)), __expf(fminf(m2u.b, 80.0f))};
    const F2 den = f2_add(f2(1.0f), e);
    const F2 sg{__fdividef(1.0f, den.a), __fdividef(1.0f, den.b)};
    const F2 one_minus = f2_mul(e, sg);
    const F2 du = f2_mul(f2(0.7978845608028654f), f2_add(f2(1.0f), f2_mul(f2(3.0f * 0.044715f), pp)));
    const F2 g = f2_add(sg, f2_mul(f2_mul(f2_mul(f2_mul(f2(2.0f), P), sg), one_minus), du));
    const F2 r = f2_mul(F2{bf16lo_to_f32(dh), bf16hi_to_f32(dh)}, g);
    return pack_bf16x2(r.a, r.b);
}

// Two packed bf16 -> bf16(gelu_tanh(.)) each, packed the same way; hmax takes the larger
// of itself and the two results' magnitudes (fmaxf: a NaN never wins).
__device__ __forceinline__ uint32_t gelu_bf16x2(uint32_t w, float& hmax) {
    const F2 P{bf16lo_to_f32(w), bf16hi_to_f32(w)};
    F2 pp;
    const F2 m2u = f2_mul(f2(-2.0f), gelu_tanh_u2(P, pp));
    const F2 den = f2_add(f2(1.0f), F2{__expf(m2u.a), __expf(m2u.b)});
    const uint32_t r = pack_bf16x2(__fdividef(P.a, den.a), __fdividef(P.b, den.b));
    hmax = fmaxf(hmax, fmaxf(fabsf(bf16lo_to_f32(r)), fabsf(bf16hi_to_f32(r))));
    return r;
}

}  // namespace ft
