// sm100.cuh: sm_100a device primitives written as inline PTX.
//
// mbarrier (with bounded waits), TMA tile loads, and the 5th-generation
// tensor-core interface: TMEM allocation, tcgen05.mma with operands in shared
// memory or TMEM, tcgen05.commit, and TMEM <-> register moves.
#pragma once

#include <cuda.h>
#include <cstdint>

namespace fa {

// Device error word: the first failure of any kernel stores its code here.
// kErrTimeoutBase + site: a bounded wait ran out; kErrSmemAlign: the dynamic
// shared memory window was not 1024-byte aligned (the kernel did nothing);
// kErrSeqlenBound: a varlen sequence was longer than the max_seqlen bound the
// caller gave (or had a negative length), so only its first max_seqlen rows or
// keys were processed.
enum : int { kErrTimeoutBase = 0x1000, kErrSmemAlign = 0x2000, kErrSeqlenBound = 0x3000 };

// ---------------------------------------------------------------------------
// generic helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// True if the dynamic shared memory window starts on a 1024-byte boundary;
// otherwise records kErrSmemAlign (uniform over the CTA, so all threads leave).
__device__ __forceinline__ bool smem_base_ok(const void* smem, int* err) {
    if ((static_cast<uint32_t>(__cvta_generic_to_shared(smem)) & 1023u) == 0) return true;
    if (threadIdx.x == 0) atomicCAS(err, 0, kErrSmemAlign);
    return false;
}

// Varlen: records kErrSeqlenBound if sequence b of cu_seqlens_q / cu_seqlens_k is
// longer than its bound or has a negative length (the kernels clip to the bound).
__device__ __forceinline__ void check_seqlens(const int* cu_q, const int* cu_k, int b, int max_q, int max_k,
                                              int* err) {
    const int lq = cu_q[b + 1] - cu_q[b], lk = cu_k[b + 1] - cu_k[b];
    if (lq < 0 || lq > max_q || lk < 0 || lk > max_k) atomicCAS(err, 0, kErrSeqlenBound);
}

__device__ __forceinline__ int warp_id() { return static_cast<int>(threadIdx.x >> 5); }
__device__ __forceinline__ int lane_id() { return static_cast<int>(threadIdx.x & 31); }

// ---------------------------------------------------------------------------
// mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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

// Shared state of the bounded waits of one CTA.
struct WaitCtx {
    volatile int* abort;  // shared flag: set once any wait of the CTA gave up
    int* err;             // global error word
};

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s without progress

// Wait for the phase with parity `parity` of `bar` to complete. Returns false
// (and marks the CTA aborted) after kWaitLimitNs, or at once if another wait of
// the CTA has already given up. `site` identifies the wait in the error word.
__device__ __forceinline__ bool wait_slow(uint32_t bar, uint32_t parity, WaitCtx ctx, int site) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 15u) {
            if (*ctx.abort) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                *ctx.abort = 1;
                atomicCAS(ctx.err, 0, kErrTimeoutBase + site);
                __threadfence();
                return false;
            }
        }
    }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, WaitCtx ctx, int site) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    return wait_slow(a, parity, ctx, site);
}


__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

// Time-bounded wait used only while draining at exit (ignores the abort flag).
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
    const uint32_t a = smem_u32(bar);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(a, parity)) {
        if (globaltimer_ns() - t0 > 200000000ull) break;
    }
}

// ---------------------------------------------------------------------------
// TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 4-D tiled load of one box into shared memory, completing on `bar` (tx bytes).
// c0 is the innermost coordinate (elements); it is always a multiple of 64 here.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* m, uint64_t* bar, int c0, int c1,
                                            int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// Prefetch one box of a 4-D tensor map into the L2 (no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch_l2_4d(const CUtensorMap* m, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}

// ---------------------------------------------------------------------------
// TMEM allocation (whole warp)
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
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
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive once on `bar` when every tcgen05 operation issued so far by this
// thread has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// ---------------------------------------------------------------------------
// Descriptors
//
// Shared-memory matrix descriptor (tcgen05 form): start address, leading and
// stride byte offsets (all >> 4), version 1 at bit 46, layout type at bit 61.
// Every operand here uses the 128-byte swizzle (layout type 2): rows of 128 B,
// the 16-byte chunk c of row r stored at chunk c ^ (r % 8), 8-row atoms of
// 1024 B that start on 1024-byte boundaries.
//   K-major operand:  SBO = 1024 (next 8 rows); LBO unused (1).
//   MN-major operand: SBO = 1024 (next 8 rows along K); LBO = byte distance to
//                     the next 64-element block along M/N.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// The same descriptor as two 32-bit words: lo = start address >> 4 (bits 0-13) and
// LBO >> 4 (bits 16-29), hi = SBO >> 4, the version and the layout type. An operand
// that starts k x 16 bytes further on has lo + k: shared memory addresses stay below
// 2^18, so the start-address field never carries into the LBO field. Stepping
// through an operand then costs one 32-bit add per instruction.
struct SDesc {
    uint32_t lo, hi;
};
__device__ __forceinline__ SDesc sdesc_sw128_split(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return {((saddr >> 4) & 0x3FFFu) | (((lbo >> 4) & 0x3FFFu) << 16),
            ((sbo >> 4) & 0x3FFFu) | (1u << 14) | (2u << 29)};
}

// Instruction descriptor of kind::f16 with fp32 accumulation: D format at
// bit 4, A and B formats at bits 7 and 10 (0 = f16, 1 = bf16), A/B major at
// bits 15/16 (0 = K-major, 1 = MN-major), N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool bf16, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((a_mn_major ? 1u : 0u) << 15) |
           ((b_mn_major ? 1u : 0u) << 16) | ((static_cast<uint32_t>(N) >> 3) << 17) |
           ((static_cast<uint32_t>(M) >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T  (one instruction, K = 16 for 16-bit types)
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// mma_ss with split descriptors: A = {a_lo + a_step, a.hi}, B = {b_lo + b_step, b.hi}.
__device__ __forceinline__ void mma_ss_split(uint32_t d_tmem, SDesc a, uint32_t a_step, SDesc b, uint32_t b_step,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "mov.b64 da, {%1, %2};\n\t"
        "mov.b64 db, {%3, %4};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, p;\n\t}" ::"r"(d_tmem),
        "r"(a.lo + a_step), "r"(a.hi), "r"(b.lo + b_step), "r"(b.hi), "r"(idesc), "r"(accumulate)
        : "memory");
}

// mma_ts with a split descriptor for B: B = {b_lo + b_step, b.hi}.
__device__ __forceinline__ void mma_ts_split(uint32_t d_tmem, uint32_t a_tmem, SDesc b, uint32_t b_step,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "mov.b64 db, {%2, %3};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "r"(b.lo + b_step), "r"(b.hi), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T; A holds M lanes x K 16-bit values, two per column.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Instruction descriptor of kind::f8f6f4 with E4M3 A and B (format 0 at bits 7
// and 10) and fp32 accumulation; the other fields as in idesc_f16. K = 32 per
// instruction.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
           ((static_cast<uint32_t>(N) >> 3) << 17) | ((static_cast<uint32_t>(M) >> 4) << 24);
}

// kind::f8f6f4 forms of mma_ss / mma_ts (K = 32 one-byte values per instruction;
// a TMEM A operand holds four per column, the lowest K index in the low byte).
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Four floats to four E4M3 bytes (round to nearest even, saturating to +-448),
// x0 in the low byte.
__device__ __forceinline__ uint32_t pack4_e4m3(float x0, float x1, float x2, float x3) {
    uint16_t lo, hi;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(x1), "f"(x0));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(x3), "f"(x2));
    return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// ---------------------------------------------------------------------------
// TMEM <-> registers. A warp reaches the 32 lanes 32 * (warp % 4) ... + 31;
// with the 32x32b shape thread t of the warp holds lane 32 * (warp % 4) + t and
// register i holds column (address column + i).
#define FA_R8(a, o) "=r"(a[o + 0]), "=r"(a[o + 1]), "=r"(a[o + 2]), "=r"(a[o + 3]), "=r"(a[o + 4]), \
                    "=r"(a[o + 5]), "=r"(a[o + 6]), "=r"(a[o + 7])
#define FA_W8(a, o) "r"(a[o + 0]), "r"(a[o + 1]), "r"(a[o + 2]), "r"(a[o + 3]), "r"(a[o + 4]), \
                    "r"(a[o + 5]), "r"(a[o + 6]), "r"(a[o + 7])
#define FA_RW8(a, o) "+r"(a[o + 0]), "+r"(a[o + 1]), "+r"(a[o + 2]), "+r"(a[o + 3]), "+r"(a[o + 4]), \
                     "+r"(a[o + 5]), "+r"(a[o + 6]), "+r"(a[o + 7])

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : FA_R8(r, 0), FA_R8(r, 8), FA_R8(r, 16), FA_R8(r, 24)
        : "r"(taddr)
        : "memory");
}

// Wait for this thread's outstanding TMEM loads. The registers are passed
// through the asm so no use of them can be scheduled before the wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;" : FA_RW8(r, 0), FA_RW8(r, 8), FA_RW8(r, 16), FA_RW8(r, 24)
                 :
                 : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        FA_W8(r, 0), FA_W8(r, 8), FA_W8(r, 16), FA_W8(r, 24)
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        FA_W8(r, 0), FA_W8(r, 8)
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------------------
// misc synchronisation
// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor-core operand reads) ordered after a following barrier.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Named barrier over `nthreads` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Vector fp32 reduction into global memory (16-byte aligned address).
__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// ---------------------------------------------------------------------------
// Register reallocation between warpgroups (all warps of a warpgroup execute it).
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------------------
// math helpers (hardware instructions)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Pack two floats into a 16-bit pair, round to nearest even; `lo` ends up in
// the low half (the element with the lower index).
template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    uint32_t r;
    if constexpr (BF16) {
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    } else {
        asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    }
    return r;
}

// Pairs of fp32 in one 64-bit register, for the packed f32x2 arithmetic of sm_100.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ float f2_sum(uint64_t v) {
    float a, b;
    f2_unpack(v, a, b);
    return a + b;
}
// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// The element of a packed 16-bit pair as fp32 (exact).
template <bool BF16>
__device__ __forceinline__ float unpack_lo(uint32_t u) {
    if constexpr (BF16) {
        return __uint_as_float(u << 16);
    } else {
        float f;
        asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.f32.f16 %0, lo;\n\t}" : "=f"(f) : "r"(u));
        return f;
    }
}
template <bool BF16>
__device__ __forceinline__ float unpack_hi(uint32_t u) {
    if constexpr (BF16) {
        return __uint_as_float(u & 0xFFFF0000u);
    } else {
        float f;
        asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.f32.f16 %0, hi;\n\t}" : "=f"(f) : "r"(u));
        return f;
    }
}

// Online softmax: rescale the partial output only once the row max has grown by
// more than 2^8 since the last rescale (log2 units; exact, since O and the
// normaliser share the reference max).
constexpr float kRescaleThreshold = 8.0f;
constexpr float kLn2 = 0.69314718055994530942f;

}  // namespace fa
