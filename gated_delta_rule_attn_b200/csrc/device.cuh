// device.cuh — sm_100a building blocks written as inline PTX: shared-memory
// addresses, mbarriers with bounded waits, TMA tile loads, tcgen05 tensor
// memory allocation, MMA issue/commit and TMEM loads, and the 128-byte swizzle
// used by every bf16 operand tile.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace la {

// Device-wide error word (read and cleared by la_check_device).  The library is
// one translation unit, so the definition lives here.
enum : uint32_t { kErrTimeout = 1u, kErrRange = 2u, kErrSeqlen = 4u };
__device__ uint32_t g_error_word = 0;

__device__ __forceinline__ void raise_error(uint32_t bit) { atomicOr(&g_error_word, bit); }

// Where sequence b's tokens sit on the token axis: rows row0 .. row0+len-1 of a
// [*, T, H, d] tensor viewed as rows of [H, d], and the (t, b) coordinates of its
// first token for a 4-D tensor map.  Dense layout ([B, T, H, d], cu == nullptr):
// row0 = b*T, len = T, map coordinates (0, b).  Packed layout (one token axis
// of `total` tokens): row0 = cu[b], len = cu[b+1] - cu[b], map coordinates
// (cu[b], 0).  Offsets are clamped into [0, total] and lengths to max_len, so a
// bad offset array cannot move an access out of the tensors; `report` raises
// kErrSeqlen when clamping changed anything.
struct SeqSpan {
    int64_t row0, len;
    int t0, b0;
};
__device__ __forceinline__ SeqSpan seq_span(const int64_t *cu, int64_t b, int64_t T, int64_t max_len,
                                            bool report) {
    if (!cu) return SeqSpan{b * T, T, 0, (int)b};
    const int64_t s_raw = cu[b], e_raw = cu[b + 1];
    const int64_t s = s_raw < 0 ? 0 : (s_raw > T ? T : s_raw);
    const int64_t e = e_raw < s ? s : (e_raw > T ? T : e_raw);
    const int64_t len = e - s > max_len ? max_len : e - s;
    if (report && (s != s_raw || e != e_raw || len != e - s)) raise_error(kErrSeqlen);
    return SeqSpan{s, len, (int)s, 0};
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// One potentially blocking test: the hardware suspends the calling thread until
// the phase completes or about `kSuspendNs` nanoseconds pass, so waiting warps
// do not spin on the issue slots and shared-memory pipe that working warps use.
constexpr uint32_t kSuspendNs = 1000000;
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
        : "memory");
    return ok != 0;
}

// Spin limit for every wait in this library: about one second at boost clock.
constexpr long long kWaitLimitCycles = 2000000000LL;

// Non-blocking test of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// The limit ordinary waits use, in constant memory (a cached read per wait).  It
// is kWaitLimitCycles unless the library's testing hook (la_testing_set_wait_limit)
// shortened it so that a test makes waits run out and exercises the abort paths.
// A suspended try_wait may sleep until its phase completes, so a shortened limit
// is enforced by non-blocking polls instead.  Drain waits, which guard the
// release of TMEM and the exit of a CTA with copies in flight, always keep
// kWaitLimitCycles.
__constant__ long long g_wait_limit = kWaitLimitCycles;

__device__ __forceinline__ bool mbar_wait_for(uint64_t *bar, uint32_t parity, long long limit) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > limit) {
            raise_error(kErrTimeout);
            return false;
        }
    }
    return true;
}

// Bounded wait on an mbarrier phase.  Returns false (and raises kErrTimeout) if
// the phase did not complete within g_wait_limit cycles.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    if (mbar_test(bar, parity)) return true;   // the phase is done: no limit needed
    const long long limit = g_wait_limit;
    if (limit >= kWaitLimitCycles) return mbar_wait_for(bar, parity, limit);
    const long long t0 = clock64();
    while (!mbar_test(bar, parity)) {
        if (clock64() - t0 > limit) {
            raise_error(kErrTimeout);
            return false;
        }
    }
    return true;
}

// Wait for asynchronous work this CTA issued (copies, MMAs) before it frees the
// resources that work uses; bounded by kWaitLimitCycles whatever g_wait_limit is.
__device__ __forceinline__ bool mbar_drain(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    return mbar_wait_for(bar, parity, kWaitLimitCycles);
}

// ---------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor), no multicast.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 4-D tile load: coordinates innermost first (element units).
__device__ __forceinline__ void tma_load_4d(void *smem_dst, const CUtensorMap *map, uint64_t *bar,
                                            int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2),
        "r"(c3)
        : "memory");
}

// L2 prefetch of one 4-D tile (no shared-memory destination, no barrier).
__device__ __forceinline__ void tma_prefetch_l2_4d(const CUtensorMap *map, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}

// L2 prefetch of `bytes` (a multiple of 16) at a 16-byte aligned global address
// (no shared-memory destination, no barrier).
__device__ __forceinline__ void bulk_prefetch_l2(const void *gptr, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(gptr)),
                 "r"(bytes)
                 : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory, MMA, loads.
// ---------------------------------------------------------------------------
// Allocate `ncols` TMEM columns (power of two >= 32); executed by one full warp.
__device__ __forceinline__ void tmem_alloc(uint32_t *slot_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 accumulation.
//   bits 4-5 D format (1 = f32), 7-9 A format (1 = bf16), 10-12 B format,
//   15 A major (0 = K, 1 = MN), 16 B major, 17-22 N>>3, 24-28 M>>4.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
           ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor.
//   bits 0-13 start address >> 4, 16-29 leading-dimension byte offset >> 4,
//   32-45 stride-dimension byte offset >> 4, 46-47 version (1 on sm_100),
//   49-51 base offset (0: atoms are 1024-byte aligned), 61-63 swizzle mode
//   (0 none, 2 = 128-byte, 4 = 64-byte, 6 = 32-byte).
enum : uint32_t { kSwizzleNone = 0, kSwizzle128 = 2, kSwizzle64 = 4 };

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t swz) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)swz << 61);
}

// D[tmem] (+)= A * B, issued by a single thread.  Ordered after earlier
// fences and barriers by asm volatile; no memory clobber so that descriptor
// arithmetic can be scheduled around consecutive issues.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Arrive (once) on `bar` when all previously issued MMAs of this thread finish.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns: thread i of the warp gets
// columns [col, col+16) of TMEM lane (warp quadrant base + i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16]) {
    uint32_t *u = reinterpret_cast<uint32_t *>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
          "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]),
          "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
        : "r"(taddr)
        : "memory");
}

// Same with 32 columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&r)[32]) {
    uint32_t *u = reinterpret_cast<uint32_t *>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
          "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]),
          "=r"(u[13]), "=r"(u[14]), "=r"(u[15]), "=r"(u[16]), "=r"(u[17]), "=r"(u[18]),
          "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]), "=r"(u[24]),
          "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]),
          "=r"(u[31])
        : "r"(taddr)
        : "memory");
}

// 16 lanes x 32 bit in two halves (for M=64 accumulators, whose 16 rows per
// warp quadrant sit in TMEM lanes base..base+15): threads 0-15 read lanes
// base..base+15 at columns [col, col+N), threads 16-31 the same lanes at
// columns [col+OFF, col+OFF+N).
template <int OFF>
__device__ __forceinline__ void tmem_ld16x2_16(uint32_t taddr, float (&r)[16]) {
    uint32_t *u = reinterpret_cast<uint32_t *>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], %17;"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
          "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]),
          "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
        : "r"(taddr), "n"(OFF)
        : "memory");
}

template <int OFF>
__device__ __forceinline__ void tmem_ld16x2_32(uint32_t taddr, float (&r)[32]) {
    uint32_t *u = reinterpret_cast<uint32_t *>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], %33;"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
          "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]),
          "=r"(u[13]), "=r"(u[14]), "=r"(u[15]), "=r"(u[16]), "=r"(u[17]), "=r"(u[18]),
          "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]), "=r"(u[24]),
          "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]),
          "=r"(u[31])
        : "r"(taddr), "n"(OFF)
        : "memory");
}

// TMEM address of (lane, column).
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) {
    return base + (lane << 16) + col;
}

// ---------------------------------------------------------------------------
// 128-byte swizzle: a tile of rows of 64 bf16 (128 bytes); 16-byte chunk c of
// row r lives at chunk (c ^ (r & 7)).  Atoms of 8 rows are 1024 bytes and must
// be 1024-byte aligned.  Returns the byte offset of element (r, col) with
// 0 <= col < 64.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t sw128_off(uint32_t r, uint32_t col) {
    return r * 128u + ((((col >> 3) ^ r) & 7u) << 4) + ((col & 7u) << 1);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&u);
    return __bfloat1622float2(v);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// phi(x) = ELU(x) + 1 (ELU alpha = 1): x + 1 for x > 0, e^x otherwise.
__device__ __forceinline__ float elu_feature(float x) { return x > 0.f ? x + 1.f : __expf(x); }

// 1/x from the special-function unit's approximate reciprocal (relative error
// about 1 ulp), for normal x; one instruction.
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x on the special-function unit (approximate, flush-to-zero; relative
// error about 1e-6 on the range the feature map uses).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// phi(x) = ELU(x) + 1 for two lanes, written as max(x, 0) + exp(min(x, 0)):
// x + 1 for x > 0 and e^x otherwise, with no select.  Measured on B200 this
// form runs at about 15 elements per clock per SM (the special-function unit's
// rate) against about 10 for a range-reduced polynomial on the FMA pipe, and
// leaves the FMA and integer pipes to the surrounding work.
__device__ __forceinline__ float2 elu_feature2(float2 x) {
    const float2 t = __fmul2_rn(make_float2(fminf(x.x, 0.f), fminf(x.y, 0.f)),
                                make_float2(1.4426950408889634f, 1.4426950408889634f));
    return make_float2(fmaxf(x.x, 0.f) + ex2_approx(t.x), fmaxf(x.y, 0.f) + ex2_approx(t.y));
}


// SMs of the current device (148 on B200; also the plan without a device).
inline int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    return n;
}

}  // namespace la
