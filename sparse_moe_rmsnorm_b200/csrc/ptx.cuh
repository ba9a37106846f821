// Thin inline-PTX wrappers for sm_100a: mbarriers with bounded waits, TMA
// (tiled and untiled bulk loads), and tcgen05 (TMEM alloc, MMA, ld/st, fences).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>

namespace moe {

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------- programmatic dependent launch
// A kernel launched with programmatic stream serialization may start while the
// kernel before it in the stream is still running: pdl_wait() blocks until
// that kernel has completed and its memory writes are visible (it returns at
// once for a kernel launched without the attribute); pdl_trigger() lets the
// next kernel in the stream start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait with a suspend-time hint: a thread whose phase is not complete may
// sleep in the barrier unit, up to `hint_ns`, until the phase completes,
// instead of polling (polling warps take issue slots and shared-memory
// pipe cycles from the producer and MMA warps of the same SM).
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

constexpr uint32_t MBAR_SUSPEND_HINT_NS = 1000000;   // 1 ms per sleep; the wait limit is checked after each

// Shared state of the bounded waits of one CTA.  `abort` lives in shared
// memory: once any thread's wait runs out, every other wait in the CTA gives
// up at its next poll.
struct WaitCtl {
    volatile int *abort;        // shared flag
    unsigned int *err;          // device error word (bit per kernel)
    unsigned int err_bit;
    unsigned long long limit_ns;
};

// Wait for the phase of `bar` with the given parity.  Returns false when the
// CTA has aborted or this wait ran out (which aborts the CTA).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, const WaitCtl &w) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t start = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_hint(bar, parity, MBAR_SUSPEND_HINT_NS)) return true;
        if (*w.abort) return false;
        if (globaltimer_ns() - start > w.limit_ns) {
            *w.abort = 1;
            atomicOr(w.err, w.err_bit);
            return false;
        }
    }
}

// --------------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const void *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ----------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
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

// ------------------------------------------------------------ E4M3 / E8M0

// E8M0 exponent s of a block with maximum magnitude amax so that amax / 2^s
// fits the largest E4M3 value 448 = 1.75 * 2^8, clamped to [-126, 126].
__device__ __forceinline__ int e4m3_block_exp(float amax) {
    const uint32_t b = __float_as_uint(amax);
    int x = (int)((b >> 23) & 0xFFu) - 127;
    int s = x - 8 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    return min(max(s, -126), 126);
}

// 2^e as a float for e in [-126, 127].
__device__ __forceinline__ float pow2f(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

// Two floats to two E4M3 bytes, `lo` in the low byte (round to nearest even,
// saturating to +-448).
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// E4M3 byte back to a float (exact).
__device__ __forceinline__ float e4m3_to_f32(uint32_t v) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)(v & 0xFFu)));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// Two E4M3 bytes (low byte first) back to floats (exact).
__device__ __forceinline__ void e4m3x2_to_f32x2(uint32_t v, float &lo, float &hi) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)(v & 0xFFFFu)));
    lo = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
    hi = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
}

// ------------------------------------------------- converged-warp issue forms
// Every lane of a converged warp makes the call and one lane, chosen by
// elect.sync inside the instruction sequence, issues.  On B200 a tcgen05.mma
// issued this way frees the warp after about 20 cycles, while one issued by a
// lone lane of a divergent warp holds it for 50-120 cycles, so the MMA and
// TMA producer roles run as whole warps through these forms.

__device__ __forceinline__ void mma_commit_w(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t.reg .b32 r;\n\telect.sync r|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_w(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t.reg .b32 r;\n\t.reg .b64 st;\n\telect.sync r|e, 0xffffffff;\n\t"
        "@e mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx_w(uint64_t *bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t.reg .b32 r;\n\t.reg .b64 st;\n\telect.sync r|e, 0xffffffff;\n\t"
        "@e mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_addr(bar)),
        "r"(bytes)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d_w(void *dst, const void *map, uint64_t *bar, int c0, int c1, int c2) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t.reg .b32 r;\n\telect.sync r|e, 0xffffffff;\n\t"
        "@e cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
        "%5}], [%2];\n\t}" ::"r"(smem_addr(dst)),
        "l"(map), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void tma_load_5d_w(void *dst, const void *map, uint64_t *bar, int c0, int c1, int c2,
                                              int c3, int c4) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t.reg .b32 r;\n\telect.sync r|e, 0xffffffff;\n\t"
        "@e cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
        "%5, %6, %7}], [%2];\n\t}" ::"r"(smem_addr(dst)),
        "l"(map), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
        : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T with E8M0 block scales (one per 32 K
// elements) read from TMEM: kind::mxf8f6f4, one CTA.  The scale addresses must
// be 4-column aligned (a misaligned one faults); the byte within each 32-bit
// scale column is chosen by the descriptor's scale-factor ids.
__device__ __forceinline__ void mma_mx_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t.reg .b32 r;\n\telect.sync r|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

__device__ __forceinline__ void bulk_load_w(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t.reg .b32 r;\n\telect.sync r|e, 0xffffffff;\n\t"
        "@e cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n\t}" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t (&r)[4]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
                 "r"(r[2]), "r"(r[3])
                 : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}

// The same stores with the registers named one by one (no array copy).
__device__ __forceinline__ void tmem_st2v(uint32_t taddr, uint32_t a, uint32_t b) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};" ::"r"(taddr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ void tmem_st4v(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}
__device__ __forceinline__ void tmem_st8v(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t e,
                                          uint32_t f, uint32_t g, uint32_t h) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr), "r"(a),
                 "r"(b), "r"(c), "r"(d), "r"(e), "r"(f), "r"(g), "r"(h)
                 : "memory");
}

// Load with acquire semantics at GPU scope (a flag or counter another CTA releases).
__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Order this thread's generic-proxy global-memory accesses with its async-proxy ones
// (TMA copies of data other CTAs wrote, after acquiring their flag).
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to later
// async-proxy reads (TMA, tcgen05.mma operands).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Each thread of the warp reads 16 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// Shared-memory matrix descriptor of a K-major operand in the 128-byte
// swizzled canonical layout: rows of 128 bytes, 8-row groups 1024 bytes
// apart (SBO), the 16-byte chunks of row r permuted by XOR with (r mod 8).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);          // start address
    d |= (uint64_t)(16u >> 4) << 16;                  // leading byte offset (unused for this layout)
    d |= (uint64_t)(1024u >> 4) << 32;                // stride byte offset: next 8-row group
    d |= (uint64_t)1 << 46;                           // descriptor version for tcgen05
    d |= (uint64_t)2 << 61;                           // 128-byte swizzle
    return d;
}

// ------------------------------------------------------------- MXFP4 decode

// Eight E2M1 codes (one 32-bit word, element 2m in the low nibble of byte m)
// to four fp16 pairs, exactly; pair i holds elements 2i (low half) and 2i+1.
__device__ __forceinline__ void e2m1x8_to_half2x4(uint32_t codes, uint32_t (&o)[4]) {
    asm volatile(
        "{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
        : "r"(codes));
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// fp32 2^e for an integer e, exact over the whole fp32 range (0 below it).
__device__ __forceinline__ float exp2i(int e) {
    if (e >= -126) return __int_as_float((min(e, 127) + 127) << 23);
    if (e >= -149) return __int_as_float(1 << (e + 149));
    return 0.0f;
}

// Row shift c of one weight row: the row is decoded as value * 2^-c so that
// its largest block lands at exponent 13 (6 * 2^13 < 65504); every block whose
// E8M0 byte is within 36 of the row's largest is then exact in fp16.  Bytes
// of 255 (NaN) are left out of the maximum.
__device__ __forceinline__ int row_shift_from_max(int smax) { return smax < 0 ? 0 : smax - 140; }

// Multiplier of one block (E8M0 byte s) under row shift c, as an fp16 pair:
// 2^(s-127-c), rounded to fp16 (exact down to 2^-24), NaN for s = 255.
__device__ __forceinline__ uint32_t block_multiplier(int s, int c) {
    if (s == 255) return 0x7E007E00u;
    float m = exp2i(s - 127 - c);
    __half h = __float2half_rn(m);
    uint32_t u = (uint32_t)__half_as_ushort(h);
    return u | (u << 16);
}

}  // namespace moe
