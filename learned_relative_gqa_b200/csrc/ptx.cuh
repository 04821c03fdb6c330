// ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers (with bounded
// waits), TMA tile loads, tcgen05 (TMEM alloc, MMA, commit, ld/st, fences),
// per-thread cp.async and a few scalar helpers. Written against the public PTX
// ISA; descriptor bit layouts follow the sm_100 "shared memory descriptor" and
// "instruction descriptor" tables.
#pragma once

#include <cstdint>
#include <cuda.h>

namespace ira {

// Limit of the teardown drain waits (nanoseconds), independent of the pipeline limit.
constexpr uint64_t kDrainTimeoutNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Same, but the thread may sleep (not issue) until the phase completes or about
// kSuspendHintNs pass, so waiting warps leave the issue slots to working warps.
constexpr uint32_t kSuspendHintNs = 20000;
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "n"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

// Shared control block of a CTA: `abort` is raised by the first wait that
// runs out so that every other role stops waiting too.
struct CtaControl {
    int abort;
    int pad[3];
};

// Bounded wait on an mbarrier phase. Returns false when the CTA is aborting or
// when the limit runs out; in the latter case the CTA abort flag is raised and
// `site` is recorded (first writer wins) in the device error word.
// Limits below the suspend hint poll without sleeping, so that the limit itself is
// what ends the wait (a sleeping try_wait resumes when the phase completes).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, CtaControl* ctl, int* gerr,
                                          int site, uint64_t timeout_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    const bool sleep = timeout_ns >= kSuspendHintNs;
    while (true) {
        if (sleep ? mbar_try_wait_sleep(bar, parity) : mbar_try_wait(bar, parity)) return true;
        if (*reinterpret_cast<volatile int*>(&ctl->abort)) return false;
        if (globaltimer_ns() - t0 > timeout_ns) {
            atomicExch(&ctl->abort, 1);
            if (gerr) atomicCAS(gerr, 0, site);
            return false;
        }
    }
}

// Warp-uniform bounded wait: every lane polls, and the warp proceeds only if
// all lanes saw the phase complete (so warp-collective tcgen05.ld/st that
// follow are executed by the whole warp or by none of it).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, CtaControl* ctl, int* gerr, int site,
                                          uint64_t timeout_ns) {
    const bool ok = mbar_wait(bar, parity, ctl, gerr, site, timeout_ns);
    return __all_sync(0xffffffffu, ok);
}

// Bounded wait used while draining at teardown: ignores the abort flag and always
// allows the default limit (whatever limit the pipeline waits were given), so that a
// CTA leaves no tensor copy or MMA of its own in flight when it exits. A phase that
// can no longer complete (a partner arrival skipped by an aborting CTA) costs that
// limit once.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_sleep(bar, parity)) {
        if (globaltimer_ns() - t0 > kDrainTimeoutNs) return false;
    }
    return true;
}

// ---------------------------------------------------------------------------
// TMA (tensor tile loads, no multicast)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_4d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, "
        "%6}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
            "r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}
// Tensor tile store from shared memory (bulk async group of the issuing thread).
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* smem_src, int c0, int c1, int c2,
                                             int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(smem_src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until every bulk async group of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Bring a tile of a tensor map into L2 (no shared-memory destination, nothing to
// wait for). Only in-range tiles are prefetched by the callers.
__device__ __forceinline__ void tma_prefetch_l2_4d(const CUtensorMap* map, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------
// per-thread cp.async (16 bytes, zero-fill beyond src_bytes)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async_16(uint32_t smem_addr, const void* gptr, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr), "l"(gptr), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// wait until at most N committed groups of this thread are still in flight
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// bring the line holding `ptr` into L2 (no register result, no completion to wait for)
__device__ __forceinline__ void prefetch_l2(const void* ptr) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
}

// ---------------------------------------------------------------------------
// tcgen05
// ---------------------------------------------------------------------------
// Whole warp: allocate `ncols` TMEM columns, base address written to *dst.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Orders this thread's generic-proxy shared-memory writes before later async-proxy
// accesses (tensor-core operand reads, tensor copies) of the same bytes.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on `bar` once every tcgen05 operation issued so far by this thread completes.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 consecutive 32-bit columns: thread t gets lane (base lane + t), columns [col, col+32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
// 32 lanes x 8 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}
// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
// 32 lanes x 32 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
        "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// Per-warpgroup register budget (every warp of the warpgroup executes it).
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------------------
// descriptors
// ---------------------------------------------------------------------------
// Instruction descriptor, kind::f16 with BF16 A/B and FP32 accumulator.
// a_mn / b_mn select MN-major operands (transpose bits 15 / 16).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn) {
    return (1u << 4)                      // D format: F32
           | (1u << 7)                    // A format: BF16
           | (1u << 10)                   // B format: BF16
           | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16)
           | (uint32_t(N >> 3) << 17)     // N / 8
           | (uint32_t(M >> 4) << 24);    // M / 16
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand (the layout
// TMA writes with CU_TENSOR_MAP_SWIZZLE_128B; tiles are 1024-byte aligned).
//   K-major:  rows of 64 bf16 (128 B), 8-row atoms; SBO = 1024 B between atoms
//             along M/N; LBO unused (encoded 1). Advance K by 16 -> +32 B.
//   MN-major: 64 MN-contiguous bf16 per 128-B row, one row per K index; SBO =
//             1024 B between 8-K-row atoms; LBO = bytes between 64-wide MN
//             blocks. Advance K by 16 -> +2048 B.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= uint64_t((saddr & 0x3FFFFu) >> 4);
    d |= uint64_t((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= uint64_t((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= uint64_t(1) << 46;  // descriptor version for sm_100
    d |= uint64_t(2) << 61;  // SWIZZLE_128B
    return d;
}

// ---------------------------------------------------------------------------
// shared-memory loads by 32-bit shared address
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ int lds_s32(uint32_t addr) {
    int v;
    asm volatile("ld.shared.s32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ float4 lds_f32x4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ int4 lds_s32x4(uint32_t addr) {
    int4 v;
    asm volatile("ld.shared.v4.s32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// ---------------------------------------------------------------------------
// scalar helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// 2^t for two values on the FMA and integer pipes, so that a share of the softmax
// exponentials leaves the MUFU (which also performs the BF16 conversions) free.
// Method: Cody-Waite style range reduction t = n + f with n = round(t) obtained by
// adding and subtracting 1.5 * 2^23 (round-to-nearest in FP32), f in [-1/2, 1/2];
// 2^f from a cubic fitted here to 2^f on that interval (weighted least squares towards
// minimax relative error; max relative error 7.6e-5 when evaluated in FP32 by Horner's
// rule); n is then added to the exponent field. Inputs are clamped to >= -125 so the
// exponent stays in range (results below 2^-125 come out as about 2^-125, not 0); the
// callers' arguments never exceed +9.
__device__ __forceinline__ float2 exp2_fma2(float2 t) {
    constexpr float kRound = 12582912.f;  // 1.5 * 2^23
    constexpr float c0 = 0.9999282360076904f, c1 = 0.6932609677314758f, c2 = 0.24260851740837097f,
                    c3 = 0.05517049878835678f;
    t = make_float2(fmaxf(t.x, -125.f), fmaxf(t.y, -125.f));
    const float2 r = __fadd2_rn(t, make_float2(kRound, kRound));         // n in the low mantissa bits
    const float2 nf = __fadd2_rn(r, make_float2(-kRound, -kRound));      // n as a float
    const float2 f = __ffma2_rn(nf, make_float2(-1.f, -1.f), t);          // t - n
    float2 q = __ffma2_rn(f, make_float2(c3, c3), make_float2(c2, c2));
    q = __ffma2_rn(q, f, make_float2(c1, c1));
    q = __ffma2_rn(q, f, make_float2(c0, c0));
    return make_float2(__int_as_float(__float_as_int(q.x) + (__float_as_int(r.x) << 23)),
                       __int_as_float(__float_as_int(q.y) + (__float_as_int(r.y) << 23)));
}

// max of three floats (single sm_100 instruction)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint32_t funnel_r(uint32_t lo, uint32_t hi, uint32_t shift) {
    return __funnelshift_r(lo, hi, shift);
}
__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Barrier over `nthreads` threads that also ANDs a predicate across them.
// Every participating thread must reach it (after bounded waits only), so a
// group can leave its loop together when any of its warps gave up a wait.
__device__ __forceinline__ bool named_bar_and(int id, int nthreads, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %2, 0;\n\tbar.red.and.pred p, %1, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"(id), "r"(uint32_t(v)), "r"(nthreads)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// optional pipeline timeline (compiled only with -DINKLING_TRACE)
// ---------------------------------------------------------------------------
// Slot (step * 64 + event) of buf receives the SM clock; only CTA `cta`
// records, steps >= 8192 are dropped. No atomics, so recording does not stall.
__device__ __forceinline__ void trace_event(unsigned long long* buf, int cta, int ev, int step) {
    if (buf != nullptr && int(blockIdx.x) == cta && step < 8192) buf[step * 64 + ev] = clock64();
}

// Whole-grid record: slot (0..7) of this CTA's 8-word row in kernel kid's table
// (8192 CTAs at most) after the step timeline receives the global timer
// (nanoseconds), or `v` for trace_grid_value.
__device__ __forceinline__ void trace_grid(unsigned long long* buf, int kid, int slot) {
    if (buf != nullptr && blockIdx.x < 8192) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        buf[8192 * 64 + kid * 65536 + blockIdx.x * 8 + slot] = t;
    }
}
__device__ __forceinline__ void trace_grid_value(unsigned long long* buf, int kid, int slot, unsigned long long v) {
    if (buf != nullptr && blockIdx.x < 8192) buf[8192 * 64 + kid * 65536 + blockIdx.x * 8 + slot] = v;
}
__device__ __forceinline__ unsigned smid() {
    unsigned r;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
    return r;
}

}  // namespace ira

#ifdef INKLING_TRACE
#define IRA_TRACE(p, ev, step) ::ira::trace_event((p).trace, (p).trace_cta, (ev), (step))
#define IRA_TRACE_GRID(p, kid, slot) ::ira::trace_grid((p).trace, (kid), (slot))
#define IRA_TRACE_GRID_INFO(p, kid, n) \
    ::ira::trace_grid_value((p).trace, (kid), 6, (unsigned long long)::ira::smid() | ((unsigned long long)(n) << 32))
#else
#define IRA_TRACE(p, ev, step) ((void)0)
#define IRA_TRACE_GRID(p, kid, slot) ((void)0)
#define IRA_TRACE_GRID_INFO(p, kid, n) ((void)0)
#endif
