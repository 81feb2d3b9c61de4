// common.cuh -- device helpers shared by the NVFP4 kernels (sm_100a only).
//
// Thin inline-PTX wrappers: number-format conversions, mbarriers, TMA, and the
// tcgen05 (5th-generation tensor core / tensor memory) instructions.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nvfp4.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a (B200) only"
#endif

namespace nvfp4 {

constexpr int kMaxPartials = 1024;            // CTAs of the amax pass
constexpr size_t kQuantWorkspace = kMaxPartials * sizeof(float);
constexpr float kFp4E4m3Range = 2688.0f;      // 448 (E4M3 max) * 6 (E2M1 max)
constexpr float kAmaxFloor = 1e-12f;

// ---------------------------------------------------------------------------
// number formats
// ---------------------------------------------------------------------------

// E4M3 byte of a non-negative fp32 value: round to nearest even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_from_f32(float v) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
    return r & 0xffu;
}

// Block-scale byte of a block whose scaled maximum is y = rn(gsf * bmax) >= 0:
// E4M3(rn(y / 6)), with the quotient rounded correctly without a divide instruction.
// With r = rn(1/6) (within half an ulp of 1/6) the first quotient q0 = rn(y * r) is
// faithful, the remainder y - 6 * q0 is then exact in one FMA, and q0 + rem * r rounded
// once is rn(y / 6): the correction step of Markstein's division theorem.  y above
// 6000 is clamped first (every y / 6 >= 448 saturates to the same byte, and the clamp
// keeps the remainder finite); NaN passes through to the NaN byte as before.
__device__ __forceinline__ uint32_t e4m3_scale_of_scaled_max(float y) {
    const float r = __uint_as_float(0x3e2aaaabu);   // rn(1/6)
    y = (y > 6000.0f) ? 6000.0f : y;
    const float q0 = __fmul_rn(y, r);
    const float rem = __fmaf_rn(-q0, 6.0f, y);
    return e4m3_from_f32(__fmaf_rn(rem, r, q0));
}

// fp32 value of an E4M3 byte (exact: E4M3 -> f16 -> f32 are both widening).
__device__ __forceinline__ float f32_from_e4m3(uint32_t b) {
    uint32_t h2;
    uint16_t in = (uint16_t)b;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xffffu)));
}

// fp32 value of an E2M1 code (bit 3 = sign; magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6).
__device__ __forceinline__ float e2m1_value(uint32_t code) {
    const uint32_t mag = code & 7u, e = mag >> 1, m = mag & 1u;
    const float v = e ? (1.0f + 0.5f * (float)m) * (float)(1u << (e - 1)) : 0.5f * (float)m;
    return (code & 8u) ? -v : v;
}

// Eight fp32 values -> eight E2M1 codes (RNE, saturating), element 0 in bits 0..3.
__device__ __forceinline__ uint32_t e2m1x8_from_f32(const float (&v)[8]) {
    uint32_t out;
    asm("{\n\t"
        ".reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t"
        "}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return out;
}

// Two fp32 values -> one byte of two E2M1 codes (a in bits 0..3, b in bits 4..7).
__device__ __forceinline__ uint32_t e2m1x2_from_f32(float a, float b) {
    uint16_t out;
    asm("{\n\t"
        ".reg .b8 b0;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "mov.b16 %0, {b0, b0};\n\t"
        "}"
        : "=h"(out)
        : "f"(a), "f"(b));
    return out & 0xffu;
}

// bf16 pair (packed in a 32-bit word, element 0 in the low half) -> fp32.
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two fp32 -> bf16 pair, each rounded to nearest even (a in the low half).
__device__ __forceinline__ uint32_t bf16x2_rn(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Lane-wise max(|a|, |b|) of two bf16 pairs.  The magnitudes are exact; the sign
// bits of the result are not meaningful (callers take magnitudes).
__device__ __forceinline__ uint32_t absmax2_bf16(uint32_t a, uint32_t b) {
    uint32_t m;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(a), "r"(b));
    return m;
}

// Both magnitudes of the largest-|.| pair of four bf16 pairs (one 8-value chunk).
__device__ __forceinline__ uint32_t absmax_word4(const uint4& w) {
    return absmax2_bf16(absmax2_bf16(w.x, w.y), absmax2_bf16(w.z, w.w));
}

// The larger magnitude of a bf16 pair as a float.
__device__ __forceinline__ float absmax_of_pair(uint32_t m) {
    return fmaxf(fabsf(__uint_as_float(m << 16)), fabsf(__uint_as_float(m & 0xffff0000u)));
}

__device__ __forceinline__ float absmax_words4(const uint4& w) {
    return absmax_of_pair(absmax_word4(w));
}

// Division of 32-bit unsigned integers by an invariant divisor d >= 1 with one
// multiply-high, an add and two shifts, exact for every n < 2^32 (Granlund and
// Montgomery, "Division by Invariant Integers using Multiplication", figure 4.1).
struct FastDiv {
    uint32_t mul, s1, s2;
};

inline FastDiv make_fastdiv(uint32_t d) {
    uint32_t l = 0;
    while ((uint64_t(1) << l) < d) ++l;                 // ceil(log2 d)
    FastDiv f;
    f.mul = (uint32_t)((((uint64_t(1) << l) - d) << 32) / d + 1);
    f.s1 = l < 1 ? l : 1;
    f.s2 = l > 1 ? l - 1 : 0;
    return f;
}

__device__ __forceinline__ uint32_t fast_div(uint32_t n, const FastDiv& f) {
    const uint32_t t = __umulhi(n, f.mul);
    return (t + ((n - t) >> f.s1)) >> f.s2;
}

// ---------------------------------------------------------------------------
// time and the per-device asynchronous status word
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void record_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// ---------------------------------------------------------------------------
// mbarrier (shared::cta)
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t"
        ".reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t"
        "}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for phase `parity` of `bar`.  Gives up when *abort is set by
// another thread or when `budget_ns` of wall time has passed; then records a
// timeout, raises *abort for the rest of the block and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort, int* status,
                                                  uint64_t budget_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > budget_ns) {
            record_status(status, NVFP4_ERR_TIMEOUT);
            *abort = 1;
            return false;
        }
    }
}

// ---------------------------------------------------------------------------
// TMA and bulk copies (no multicast anywhere)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// The same load with an L2 eviction-priority policy (from l2_policy_*).
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, uint64_t* bar,
                                                 int32_t x, int32_t y, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

// L2 policies: keep lines that will be read again soon, or let read-once lines go first.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int32_t x,
                                             int32_t y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::
                     "l"(reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N committed bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until every committed bulk group has fully completed.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async proxy.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Warp-issued tcgen05 operations: the whole warp executes the call, converged, and
// elect.sync lets one lane (the lowest, the same one every time, so its commits track all
// of its operations) issue the operation.  The issuing loops stay warp-uniform, which
// lets the compiler hold descriptors, addresses and counters in uniform registers; the
// same operations issued from a loop run by a single lane of the warp reached the tensor
// pipe at 0.65x the rate.
__device__ __forceinline__ void mma_i8_w(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t"
        ".reg .pred p, e;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t"
        "}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void tc_commit_w(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
            smem_u32(bar))
        : "memory");
}

// One K step of the block-scaled MMA, warp-issued with a single election: the step's
// three scale chunks into tensor memory with 32x128b.warpx4 copies -- A at sfa_t, B's
// two 128-row halves at sfb_t = sfa_t + 4 and sfa_t + 8, the second half's source
// descriptor HALF units (16 bytes each) after the first -- then the MMA that reads them.
template <int HALF>
__device__ __forceinline__ void mma_step_nvf4_w(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                uint32_t idesc, uint32_t sfa_t, uint64_t sfa_desc,
                                                uint64_t sfb_desc, uint32_t accumulate) {
    asm volatile(
        "{\n\t"
        ".reg .pred p, e;\n\t"
        ".reg .b32 t, u;\n\t"
        ".reg .b64 s;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "add.u32 t, %5, 4;\n\t"
        "add.u32 u, %5, 8;\n\t"
        "add.u64 s, %7, %8;\n\t"
        "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%5], %6;\n\t"
        "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [t], %7;\n\t"
        "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [u], s;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], "
        "[t], p;\n\t"
        "}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_t), "l"(sfa_desc),
        "l"(sfb_desc), "n"(HALF)
        : "memory");
}

// Warp-issued forms of a stage fill (the same election): the transaction count, a tiled
// TMA load and a plain bulk copy, all completing on the stage's barrier.
__device__ __forceinline__ void mbar_arrive_expect_tx_w(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
                 "@e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void tma_load_2d_w(void* dst, const CUtensorMap* map, uint64_t* bar,
                                              int32_t x, int32_t y) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4}], [%2];\n\t}" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void bulk_load_w(void* dst, const void* src, uint32_t bytes,
                                            uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, "
        "[%3];\n\t}" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Bounded wait taken by a whole warp: every lane polls, lane 0's outcome decides for all,
// so the warp stays converged.
__device__ __forceinline__ bool mbar_wait_bounded_warp(uint64_t* bar, uint32_t parity,
                                                       volatile int* abort, int* status,
                                                       uint64_t budget_ns) {
    const bool ok = mbar_wait_bounded(bar, parity, abort, status, budget_ns);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// --- programmatic dependent launch ------------------------------------------------------
// A kernel launched with programmatic stream serialization may start while the kernel
// before it on the stream is finishing.  It sets up its shared and tensor memory, then
// waits here until that kernel has completed and its memory is visible; nothing before
// this wait reads or writes global memory.  (A no-op for an ordinary launch.)
__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Lets the next kernel on the stream be scheduled as SMs free up (it still runs its own
// griddep_wait before touching memory).
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// --- thread-block clusters -----------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Every thread of every CTA of the cluster arrives and waits (per-thread form, no
// warp convergence required): the shared-memory writes before it are visible to the
// whole cluster after it.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile(
        "barrier.cluster.arrive.release;\n\t"
        "barrier.cluster.wait.acquire;" ::: "memory");
}

// The address of the same shared-memory offset in the CTA of cluster rank `rank`.
__device__ __forceinline__ uint32_t dsmem_addr(uint32_t local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}

__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// Shared-memory matrix descriptor (sm_100 version 1): K-major, 128-byte swizzle,
// 8-row core groups 1024 bytes apart (SBO), leading offset unused.
__device__ __forceinline__ uint64_t sdesc_kmajor_sw128(uint32_t smem_addr) {
    return (uint64_t)((smem_addr >> 4) & 0x3fffu) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Descriptor for tcgen05.cp of a 32-row x 16-byte block: no swizzle, 8-row core
// matrices 128 bytes apart.
__device__ __forceinline__ uint64_t sdesc_sf(uint32_t smem_addr) {
    return (uint64_t)((smem_addr >> 4) & 0x3fffu) | ((uint64_t)(128 >> 4) << 32) |
           ((uint64_t)1 << 46);
}

}  // namespace nvfp4
