// common.cuh -- device helpers shared by the NVFP4 kernels (sm_100a only).
//
// Number formats follow the published NVFP4 format (E2M1 codes, E4M3 block scales, FP32 tensor
// scale; round to nearest even, saturating).  The element and scale encoders use the Blackwell
// hardware conversions (cvt.rn.satfinite.e2m1x2.f32 / e4m3x2.f32); decoders use the matching
// cvt.rn.f16x2.{e2m1x2,e4m3x2}.  All FP32 arithmetic that decides a code is written with the
// explicitly rounded intrinsics (__fdiv_rn, __frcp_rn, __fmul_rn) so that no contraction or
// approximation can change a code.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/nvfp4.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ != 1000)
#error "this library is written for sm_100a only"
#endif

namespace nvfp4 {

constexpr float kE2M1Max = 6.0f;
constexpr float kE4M3Max = 448.0f;
constexpr float kGlobalDen = kE2M1Max * kE4M3Max;   // 2688: maps the tensor max to both grid tops

// ---- programmatic dependent launch --------------------------------------------------------------
//
// Every kernel of the library is launched with programmatic stream serialization (launch_pdl) and
// calls griddep_wait() before its first global memory access: that returns once the preceding
// kernel in the stream has completed and its writes are visible, so only the launch and the
// prologue overlap the predecessor's tail.  One exception, argued where it is made: the
// column-wise pass of a both-layouts quantization runs concurrently with the row-wise pass and
// waits at exit instead.  griddep_launch_dependents() (after the wait) lets the
// next kernel be scheduled early.  Both are no-ops in a launch without the attribute.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- status word ------------------------------------------------------------------------------

__device__ __forceinline__ void set_status(int32_t *st, int32_t code) {
    if (st) atomicCAS(st, 0, code);
}

// ---- checked build ------------------------------------------------------------------------------
//
// Compiled with NVFP4_DEBUG_CHECKS, NVFP4_CHECKED(off, len, extent, status) is true when the access
// [off, off + len) lies inside a buffer of `extent` units (elements or bytes, as the call site
// states) and otherwise writes NVFP4_ERR_OUT_OF_BOUNDS to the status word and returns false, so
// the caller skips the access.  The extents come from the host, computed from the tensor shapes
// the caller declared, independently of the kernels' index arithmetic.  In the release build the
// macro is the constant true and compiles away.
#ifdef NVFP4_DEBUG_CHECKS
__device__ __forceinline__ bool dbg_in_bounds(int64_t off, int64_t len, int64_t extent, int32_t *status) {
    if (off >= 0 && len >= 0 && off <= extent - len) return true;
    set_status(status, NVFP4_ERR_OUT_OF_BOUNDS);
    return false;
}
#define NVFP4_CHECKED(off, len, extent, status) \
    ::nvfp4::dbg_in_bounds((int64_t)(off), (int64_t)(len), (int64_t)(extent), (status))
#else
#define NVFP4_CHECKED(off, len, extent, status) true
#endif

// ---- conversions ------------------------------------------------------------------------------

// Eight FP32 -> 32 bits of packed E2M1 codes, element 0 in the lowest nibble.
__device__ __forceinline__ uint32_t e2m1x8(const float q[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
    return out;
}

// FP32 -> E4M3 byte (round to nearest even, saturating to +-448).
__device__ __forceinline__ uint32_t e4m3(float v) {
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(v));
    return out & 0xFFu;
}

// E4M3 byte -> FP32 (exact).
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
    uint32_t h2;
    uint16_t in = (uint16_t)(b & 0xFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// Four bytes of packed E2M1 codes -> four f16x2 words (exact); element 2i in the low half of
// out[i].
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t codes, uint32_t out[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3]) : "r"(codes));
}

// Two FP32 -> packed BF16x2 (round to nearest even); `lo` in the low half.
__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
    uint32_t out;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(out) : "f"(hi), "f"(lo));
    return out;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Per-tensor decode scale from amax (FP32 IEEE division).
__device__ __forceinline__ float global_scale(float amax) {
    return amax == 0.0f ? 1.0f : __fdiv_rn(amax, kGlobalDen);
}

// ---- the 16-block quantization step -----------------------------------------------------------
//
// A block's scale byte and r = 1/d (0 when d == 0, meaning every code of the block is +0).
struct BlockScale {
    uint32_t sf;
    float r;
    bool r_inf;   // d so small that 1/d overflows: x*r is then +-inf (or NaN for x == 0)
};


// Two BF16 (one packed word) times r: both products in FP32 (IEEE RN, one paired multiply).
__device__ __forceinline__ void mul_bf16x2(uint32_t w, float r, float &lo, float &hi) {
    unsigned long long p;
    asm("{\n\t.reg .b64 a, b;\n\t"
        "mov.b64 a, {%1, %2};\n\t"
        "mov.b64 b, {%3, %3};\n\t"
        "mul.rn.f32x2 %0, a, b;\n\t}"
        : "=l"(p) : "r"(w << 16), "r"(w & 0xFFFF0000u), "f"(r));
    lo = __uint_as_float((uint32_t)p);
    hi = __uint_as_float((uint32_t)(p >> 32));
}

// Eight BF16 (as 4 packed words) -> 8 E2M1 codes given the block's reciprocal scale.
// q = x*r in FP32 (IEEE RN); when r overflowed, zero inputs give +0 (their product would be
// NaN, which encodes as +0) and the rest saturate.
__device__ __forceinline__ uint32_t encode8(const uint32_t w[4], const BlockScale &s) {
    float q[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) mul_bf16x2(w[i], s.r, q[2 * i], q[2 * i + 1]);
    if (s.r_inf) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (bf16_lo(w[i]) == 0.0f) q[2 * i] = 0.0f;
            if (bf16_hi(w[i]) == 0.0f) q[2 * i + 1] = 0.0f;
        }
    }
    return e2m1x8(q);
}

// Max of |x| over 8 BF16 in 4 words, as BF16 magnitude bits (monotone in the magnitude).
__device__ __forceinline__ uint32_t absmax_bits8(const uint32_t w[4]) {
    uint32_t m = __vmaxu2(w[0] & 0x7FFF7FFFu, w[1] & 0x7FFF7FFFu);
    m = __vmaxu2(m, __vmaxu2(w[2] & 0x7FFF7FFFu, w[3] & 0x7FFF7FFFu));
    return max(m & 0xFFFFu, m >> 16);
}

// Max of |x| over 16 BF16 in 8 words, as BF16 magnitude bits: paired abs-max (sign bits are
// masked off at the end), NaN-propagating so that a NaN still compares above 0x7F80.
__device__ __forceinline__ uint32_t absmax_bits16(const uint32_t w[8]) {
    uint32_t a, b, c, d;
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(a) : "r"(w[0]), "r"(w[1]));
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(b) : "r"(w[2]), "r"(w[3]));
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(c) : "r"(w[4]), "r"(w[5]));
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(w[6]), "r"(w[7]));
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(a) : "r"(a), "r"(b));
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(c) : "r"(c), "r"(d));
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(a) : "r"(a), "r"(c));
    a &= 0x7FFF7FFFu;
    return max(a & 0xFFFFu, a >> 16);
}

// The per-tensor scale record (see ScaleRecord in launch.h) as a kernel keeps it in shared memory.
struct SmemRecord {
    float r_tab[128];
    float den, inv_den;
    uint32_t ok;
};

// The record's entries from g (one definition for the record kernel and for the quantize passes
// that build their record themselves from a given amax): r_tab[sf] = RN(1 / RN(e4m3(sf) * g)),
// 0 where that product is 0; den = RN(g * 6); inv_den = RN(1 / den), or 0 when den < 2^-125 (the
// scale quotient then divides).
__device__ __forceinline__ float record_r_entry(uint32_t sf, float g) {
    const float d = __fmul_rn(e4m3_to_f32(sf), g);
    return (d == 0.0f) ? 0.0f : __frcp_rn(d);
}
__device__ __forceinline__ float record_den(float g) { return __fmul_rn(g, kE2M1Max); }
__device__ __forceinline__ float record_inv_den(float den) { return den >= 0x1p-125f ? __frcp_rn(den) : 0.0f; }

// A quantize pass whose amax is given builds the record in shared memory itself (threads
// 0..128 of the CTA; a barrier must follow).  The CTA with `report` set also writes g to the
// nullable g_out pointers and, for a non-finite amax, NVFP4_ERR_NONFINITE to the status word
// (the record's ok flag is then 0 and the pass writes nothing), as the record kernel does.
__device__ __forceinline__ void build_record(float amax, SmemRecord &s, bool report, float *g_out0, float *g_out1,
                                             int32_t *status) {
    const bool finite = isfinite(amax);
    const float g = global_scale(amax);
    if (threadIdx.x < 128) s.r_tab[threadIdx.x] = record_r_entry(threadIdx.x, g);
    if (threadIdx.x == 128) {
        const float den = record_den(g);
        s.den = den;
        s.inv_den = record_inv_den(den);
        s.ok = finite ? 1u : 0u;
        if (report) {
            if (!finite) {
                set_status(status, NVFP4_ERR_NONFINITE);
            } else {
                if (g_out0) *g_out0 = g;
                if (g_out1) *g_out1 = g;
            }
        }
    }
}

// ---- the 16-block step --------------------------------------------------------------------------
//
// sf = e4m3(RN(b / den)).  The quotient comes from q0 = RN(b * y), y = RN(1/den), corrected once:
// q = RN(q0 + RN(b - q0 * den) * y) with both steps fused multiply-adds.  This is the last step of
// Markstein's division and returns RN(b/den) exactly as long as the residual b - q0*den does not
// underflow; b >= 2^-100 and den >= 2^-125 (where y is stored nonzero) keep it normal, and every
// other case takes the IEEE division.  (An exhaustive host-side check over all positive finite
// BF16 b and ~800 den values, quotients up to 448, found no difference.)  r = 1/d comes from the
// record's table; d == 0 gives r == 0, meaning every code of the block is +0.
__device__ __forceinline__ BlockScale block_scale(float b, const SmemRecord &rec) {
    BlockScale s;
    float q;
    if (b >= 0x1p-100f && rec.inv_den != 0.0f) {
        const float q0 = __fmul_rn(b, rec.inv_den);
        q = __fmaf_rn(__fmaf_rn(-q0, rec.den, b), rec.inv_den, q0);
    } else {
        q = __fdiv_rn(b, rec.den);
    }
    s.sf = (b == 0.0f) ? 0u : e4m3(q);
    s.r = rec.r_tab[s.sf];
    s.r_inf = isinf(s.r);
    return s;
}

__device__ __forceinline__ void quantize16(const uint32_t w[8], const SmemRecord &rec,
                                           uint32_t &c0, uint32_t &c1, uint32_t &sf) {
    const uint32_t bm = absmax_bits16(w);
    const BlockScale s = block_scale(__uint_as_float(bm << 16), rec);
    sf = s.sf;
    c0 = c1 = 0;
    if (s.r != 0.0f) {
        c0 = encode8(w, s);
        c1 = encode8(w + 4, s);
    }
}

// ---- tensor-core scale layout -----------------------------------------------------------------

// Byte offset of scale (row i, 16-block b) in the 128x4-atom tcgen05 block-scaling layout.
__host__ __device__ __forceinline__ int64_t sf_mma_offset(int64_t i, int64_t b, int64_t atoms_per_row) {
    return ((i >> 7) * atoms_per_row + (b >> 2)) * 512 + (i & 31) * 16 + ((i & 127) >> 5) * 4 + (b & 3);
}

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---- bounded waits ----------------------------------------------------------------------------

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(done) : "r"(bar), "r"(parity) : "memory");
    return done != 0;
}

// try_wait with a suspend-time hint: a thread whose phase is not complete sleeps in hardware
// until it completes or `ns` nanoseconds pass, instead of spinning on issue slots the working
// warps of the CTA need (measured: attention 9.09 -> 8.45 ms, GEMM ~2%).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t ns) {
    uint32_t done;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(done) : "r"(bar), "r"(parity), "r"(ns) : "memory");
    return done != 0;
}

// Wait for phase `parity` of an mbarrier, giving up after limit_ns or when *abort is raised.
// Returns false when it gave up.  Each retry sleeps up to 20 us in hardware (woken at once when
// the phase completes), so the abort flag and the time limit are checked at least that often.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  const volatile int *abort, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if (abort && *abort) return false;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

// Warp-wide form of mbar_wait_bounded, called by all 32 lanes of a converged warp.  Every lane
// tests the phase in the same instruction and the outcome is taken with a vote, so a wait on a
// phase that is already complete costs no more than any other instruction; only an open phase
// falls through to the sleeping, time-bounded loop, whose decisions are voted too (warp-uniform).
// (A lane-0 wait followed by a shuffle broadcast cost ~110-170 cycles per call on a complete
// phase, and an MMA-issuing warp pays that between every group of MMAs.)
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, const volatile int *abort,
                                               uint64_t limit_ns) {
    if (__any_sync(0xFFFFFFFFu, mbar_try_wait(bar, parity))) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (__any_sync(0xFFFFFFFFu, mbar_try_wait_sleep(bar, parity, 20000u))) return true;
        if (__any_sync(0xFFFFFFFFu, (abort && *abort) || globaltimer_ns() - t0 > limit_ns)) return false;
    }
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s: far beyond any legitimate wait

}  // namespace nvfp4
