// attention.cu -- softmax attention of BF16 queries over a window of NVFP4 KV-cache slots, with
// the restore fused into the kernel's K/V tile loads (the restored BF16 K and V never reach HBM).
//
// LongLive-2.0 keeps its KV cache in NVFP4 and restores it with a parallel dequantization kernel
// before attention (d9249.github.io review, section "핵심 아이디어 / 구조 / 동작 방식"; the arXiv
// abstract on fugumt.com: NVFP4 KV cache for memory savings).  This kernel computes the same
// attention without the restored copy:
//   O[i,h,:] = sum_j softmax_j(scale * q[i,h,:] . k[j,h,:]) v[j,h,:],
// k and v being exactly the values the restore produces, BF16(FP32(e2m1 * sf) * g).
//
// Structure (sm_100a, tcgen05): a CTA owns 256 queries of one head as two 128-row Q tiles and
// walks the window in 128-token K/V tiles.  640 threads, five warpgroups:
//   warps 0-3   softmax of Q tile 0: thread = query row = tensor-memory lane
//   warps 4-7   softmax of Q tile 1 (same lanes, its own tensor-memory columns)
//   warps 8-11  K producer: both Q tiles once, then per K/V tile the restore of one token row
//               of K into shared memory (two stages)
//   warps 12-15 V producer: the same for V (two stages)
//   warp 16     MMA issuer (tcgen05.mma kind::f16, BF16 in, FP32 accumulate in tensor memory):
//                 S_t = Q_t K_i^T  (A = Q_t, B = K_i: both K-major, 128-byte swizzle, in smem)
//                 O_t += P_t V_i   (A = P_t in TENSOR memory, B = V_i: MN-major in smem)
//   warps 17-19 idle (they complete the fifth warpgroup for the register split)
// Each warpgroup resizes its registers first (setmaxnreg): 176 per softmax thread, 40 per
// producer thread, 48 in the last warpgroup; per warp-scheduler slice that is 5 x 96, the 96 per
// thread the block launched with (the launcher checks the 96).  A softmax thread holds the
// tile's whole S row (128 FP32 values) and reads tensor memory once per tile.
// Tensor memory (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,384), O_1 [384,512); the
// softmax writes P_t (BF16 pairs) over the first 64 columns of S_t once it has read S_t.
// The two Q tiles alternate: while one softmax warpgroup works on tile i, the tensor core runs
// the other Q tile's S or P.V.  Per Q tile the order is S(i) -> softmax(i) -> P.V(i) ->
// S(i + 1); one thread issues all MMAs, whose execution is in issue order, so S(i + 1)
// overwrites P(i) only after P.V(i) has read it.  K and V stages are released separately: a K
// stage once both S of its tile have read it, a V stage after both P.V, so the restore of tile
// i + 2 runs while tile i + 1 is still in flight.  A CTA whose second Q tile holds no query row
// (the last, partial pair of rows of every head) skips that tile's MMAs and softmax; those CTAs
// come last in the grid, after every CTA with two live tiles.
//
// Barriers (all waits time-bounded; a wait that gives up raises the abort flag and writes
// NVFP4_ERR_TIMEOUT to the status word, and every role leaves its loop):
//   k_full[2]    count 128: the K producers restored K of the stage (before tile 0: also both Q
//                tiles)
//   k_empty[2]   count 1:   commit after the last S that reads the stage
//   v_full[2]    count 128: the V producers restored V of the stage
//   v_empty[2]   count 1:   commit after the last P.V that reads the stage
//   s_full[t]    count 1:   commit after S_t(i) (implies P.V_t(i - 1) done, so O_t is stable)
//   p_full[t]    count 128: softmax t wrote P_t(i) and rescaled O_t
//   o_done[t]    count 1:   commit after the last P.V_t
//   drain        count 1:   every MMA retired (before tensor memory is freed)
#include <atomic>
#include <cmath>

#include "common.cuh"
#include "attention.h"

namespace nvfp4 {

namespace {

constexpr int kD = 128, kBQ = 128, kBKV = 128;
constexpr int kQTiles = 2;                         // Q tiles per CTA
constexpr int kThreads = 640;
constexpr int kMmaWarp = 16;
// registers per thread at launch (the most __launch_bounds__(kThreads, 1) allows) and the
// warpgroups' shares after setmaxnreg: two softmax, two producer, one MMA warpgroup
constexpr int kLaunchRegs = (65536 / kThreads) & ~7;
constexpr int kRegsSoftmax = 176, kRegsProducer = 40, kRegsMma = 48;
static_assert(2 * kRegsSoftmax + 2 * kRegsProducer + kRegsMma == 5 * kLaunchRegs,
              "the register split must add up to the launch's registers");
constexpr int kRegion = 128 * 128;                 // bytes: 128 rows x 128 B (one 64-wide d half)
constexpr int OFF_Q = 0;                           // Q tile t at t * 2 regions
constexpr int OFF_KV = kQTiles * 2 * kRegion;      // stage s: K at OFF_KV + s * 4R, V at + 2R
constexpr int KV_STAGE = 4 * kRegion;
constexpr int OFF_BAR = OFF_KV + 2 * KV_STAGE;
constexpr int NUM_BARS = 2 + 2 + 2 + 2 + 2 + 2 + 2 + 1;
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int kSmemBytes = OFF_MISC + 16 + 1024;
constexpr uint32_t TMEM_COLS = 512, S_COL = 0, O_COL = 256;

static_assert(kSmemBytes <= 232448, "shared memory budget");

// kind::f16 instruction descriptors: F32 accumulate (bit 4), A and B BF16 (bits 7, 10), N >> 3
// at bit 17, M >> 4 at bit 24; b_major (bit 16) = 1 for the MN-major V operand.
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBKV >> 3) << 17) |
                             ((uint32_t)(kBQ >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(kD >> 3) << 17) |
                              ((uint32_t)(kBQ >> 4) << 24);

// K-major SW128 shared-memory descriptor (SBO = 1024: 8 rows of 128 B), version 1, layout 2.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// MN-major SW128 descriptor: LBO = distance of the two 64-wide d halves (one region), SBO = 1024
// (8 token rows of 128 B).
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(kRegion >> 4) << 16) | ((uint64_t)(1024 >> 4) << 32) |
           (1ull << 46) | (2ull << 61);
}

// Byte offset of 16-byte chunk c (0..15 along a 256-byte logical row) of row r in a pair of SW128
// regions (chunks 0-7 in the first region, 8-15 in the second).
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
    return (uint32_t)((c >> 3) * kRegion + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
                 "@p tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}"
                 :: "r"(bar) : "memory");
}

// D (tensor memory) = / += A (shared memory) . B (shared memory)
__device__ __forceinline__ void tc_mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accum) {
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accum) : "memory");
}

// D (tensor memory) = / += A (tensor memory) . B (shared memory)
__device__ __forceinline__ void tc_mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t accum) {
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
                 :: "r"(d), "r"(a), "l"(b), "r"(idesc), "r"(accum) : "memory");
}

__device__ __forceinline__ void tc_ld32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
                 "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
                   "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
                   "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
}

__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tc_st32(uint32_t taddr, const uint32_t *r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
                 "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
                 "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
                 :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
                    "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
                    "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
                    "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
                 : "memory");
}

// The block scale byte as an f16 pair (sf, sf) (E4M3 -> f16 is exact).
__device__ __forceinline__ uint32_t sf_f16x2(uint32_t byte) {
    uint32_t h2;
    const uint16_t in = (uint16_t)((byte & 0xFFu) * 0x101u);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return h2;
}

// Eight restored values y = BF16(FP32(e2m1 * sf) * g) from 8 codes packed in one word, the
// restore's rounding steps: e2m1 * sf is formed in f16 pairs, where it is exact (at most 6
// significant bits, 2^-10 <= |product| <= 2688), widened to FP32 exactly, multiplied by g in FP32
// (one rounding, paired) and rounded to BF16.
__device__ __forceinline__ uint4 restore8(uint32_t codes, uint32_t sfh2, float g) {
    uint32_t h[4];
    e2m1x8_to_f16x2(codes, h);
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t pr;
        asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(pr) : "r"(h[i]), "r"(sfh2));
        const float lo = __half2float(__ushort_as_half((unsigned short)(pr & 0xFFFFu)));
        const float hi = __half2float(__ushort_as_half((unsigned short)(pr >> 16)));
        unsigned long long d;
        asm("{\n\t.reg .b64 x, y;\n\t"
            "mov.b64 x, {%1, %2};\n\t"
            "mov.b64 y, {%3, %3};\n\t"
            "mul.rn.f32x2 %0, x, y;\n\t}"
            : "=l"(d) : "f"(lo), "f"(hi), "f"(g));
        o[i] = bf16x2(__uint_as_float((uint32_t)d), __uint_as_float((uint32_t)(d >> 32)));
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint2 ldg_nc_v2(const void *p) {
    uint2 v;
    asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

__device__ __forceinline__ void sts_v4(uint32_t saddr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" :: "r"(saddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// (a.x, a.y) * (b, b) + (c, c) and (a.x, a.y) + (b.x, b.y): paired FP32 operations, IEEE RN
__device__ __forceinline__ float2 fma2(float2 a, float b, float c) {
    unsigned long long d;
    asm("{\n\t.reg .b64 x, y, z;\n\t"
        "mov.b64 x, {%1, %2};\n\t"
        "mov.b64 y, {%3, %3};\n\t"
        "mov.b64 z, {%4, %4};\n\t"
        "fma.rn.f32x2 %0, x, y, z;\n\t}"
        : "=l"(d) : "f"(a.x), "f"(a.y), "f"(b), "f"(c));
    return make_float2(__uint_as_float((uint32_t)d), __uint_as_float((uint32_t)(d >> 32)));
}

__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    unsigned long long d;
    asm("{\n\t.reg .b64 x, y;\n\t"
        "mov.b64 x, {%1, %2};\n\t"
        "mov.b64 y, {%3, %4};\n\t"
        "add.rn.f32x2 %0, x, y;\n\t}"
        : "=l"(d) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return make_float2(__uint_as_float((uint32_t)d), __uint_as_float((uint32_t)(d >> 32)));
}

// max(a, b, c) in one instruction (sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__global__ void __launch_bounds__(kThreads, 1) kv_attention_kernel(const __grid_constant__ AttnJob j,
                                                                    int32_t *status) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sbase = smem_raw + (base - raw);
    const uint32_t bar_k_full = base + OFF_BAR, bar_k_empty = bar_k_full + 16;
    const uint32_t bar_v_full = bar_k_empty + 16, bar_v_empty = bar_v_full + 16;
    const uint32_t bar_s_full = bar_v_empty + 16, bar_p_full = bar_s_full + 16;
    const uint32_t bar_o_done = bar_p_full + 16, bar_drain = bar_o_done + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sbase + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sbase + OFF_MISC + 4);
    const int warp = __shfl_sync(0xFFFFFFFFu, (int)(threadIdx.x >> 5), 0);
    const int lane = threadIdx.x & 31;
    // CTAs with two live Q tiles first (head-major, so a head's CTAs run together and share its
    // K/V in L2), the cheaper CTAs of the partial last pair of every head at the end of the grid
    const int nfull = (int)(j.tq / (kQTiles * kBQ));
    const int bid = blockIdx.x;
    const int head = bid < j.heads * nfull ? bid / nfull : bid - j.heads * nfull;
    const int64_t q0 = (int64_t)(bid < j.heads * nfull ? bid % nfull : nfull) * (kQTiles * kBQ);
    const int ntiles = (int)((j.total_tokens + kBKV - 1) / kBKV);
    const bool q1_live = q0 + kBQ < j.tq;                // Q tile 1 holds at least one query row

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_k_full + 8 * i, 128);
            mbar_init(bar_k_empty + 8 * i, 1);
            mbar_init(bar_v_full + 8 * i, 128);
            mbar_init(bar_v_empty + 8 * i, 1);
            mbar_init(bar_s_full + 8 * i, 1);
            mbar_init(bar_p_full + 8 * i, 128);
            mbar_init(bar_o_done + 8 * i, 1);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_addr(tmem_slot)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = __shfl_sync(0xFFFFFFFFu, *tmem_slot, 0);
    griddep_wait();                                       // the cache and q written by earlier kernels
    griddep_launch_dependents();

    auto give_up = [&]() {
        *abort_flag = 1;
        set_status(status, NVFP4_ERR_TIMEOUT);
    };
    // every lane of a converged warp tests the phase (a vote decides), so no warp diverges on it
    auto warp_wait = [&](uint32_t bar, uint32_t parity) -> bool {
        const bool ok = mbar_wait_warp(bar, parity, abort_flag, kWaitLimitNs);
        if (!ok && lane == 0) give_up();
        return ok;
    };

    // Each warpgroup first resizes its registers, out of the 96 per thread the block launched with
    // (per warp-scheduler slice: 2 x 176 + 2 x 40 + 48 = 5 x 96), so that a softmax thread holds a
    // whole S row.
    if (warp >= 8 && warp < 16) {
        // ------------------------------------------------------------ producers (K: warps 8-11,
        // V: warps 12-15), one token row of the tile per thread
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(kRegsProducer) : "memory");
        const bool is_v = warp >= 12;
        const int t = threadIdx.x & 127;
        if (!is_v) {                                      // both Q tiles, before K(0)
#pragma unroll 1
            for (int qt = 0; qt < kQTiles; ++qt) {
                const int64_t r = q0 + qt * kBQ + t;
                const uint16_t *src = j.q + r * j.ldq + head * kD;
                const uint32_t qb = base + OFF_Q + qt * 2 * kRegion;
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const uint4 v = r < j.tq && NVFP4_CHECKED(r * j.ldq + head * kD + 8 * c, 8, j.q_elems, status)
                                        ? ldg_nc_v4(src + 8 * c) : make_uint4(0, 0, 0, 0);
                    sts_v4(qb + sw_off(t, c), v);
                }
            }
        }
        // the raw NVFP4 bytes of this thread's token row of a tile
        struct RawRow {
            uint4 c[4];
            uint2 sf;
            float g;
        };
        int si = 0;
        auto load_row = [&](int i, RawRow &rr) -> bool {
            const int64_t tok = (int64_t)i * kBKV + t;
            if (i >= ntiles || tok >= j.total_tokens) return false;
            while (si + 1 < j.nslots && tok >= j.slot[si + 1].tok_begin) ++si;
            const AttnSlot &s = j.slot[si];
            const int64_t tt = tok - s.tok_begin;
            const int64_t cb = tt * j.row_bytes + head * (kD / 2), sb = tt * j.row_sf + head * (kD / 16);
            // checked build: the token row's codes (64 B) and scales (8 B) inside the slot
            if (!(NVFP4_CHECKED(cb, kD / 2, s.ntok * j.row_bytes, status) &&
                  NVFP4_CHECKED(sb, kD / 16, s.ntok * j.row_sf, status)))
                return false;
            const uint8_t *codes = is_v ? s.codes_v : s.codes_k;
            rr.g = is_v ? *s.g_v : *s.g_k;
            rr.sf = ldg_nc_v2((is_v ? s.sf_v : s.sf_k) + sb);
#pragma unroll
            for (int q = 0; q < 4; ++q) rr.c[q] = ldg_nc_v4(codes + cb + 16 * q);
            return true;
        };
        const uint32_t full = is_v ? bar_v_full : bar_k_full, empty = is_v ? bar_v_empty : bar_k_empty;
        const uint32_t off = is_v ? 2 * kRegion : 0;
        RawRow cur;
        for (int i = 0; i < ntiles; ++i) {
            const int st = i & 1;
            const bool clive = load_row(i, cur);          // in flight while the stage is awaited
            const uint32_t sb = base + OFF_KV + st * KV_STAGE + off;
            // the stage once the MMAs of tile i - 2 that read it (both S, or both P.V) are done
            if (i >= 2 && !warp_wait(empty + 8 * st, ((i >> 1) - 1) & 1)) break;
            if (clive) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {             // 16 B of codes = 32 elements = chunks 4q..4q+3
                    const uint32_t w = q < 2 ? cur.sf.x : cur.sf.y;
                    const uint32_t s0 = sf_f16x2(w >> (16 * (q & 1))), s1 = sf_f16x2(w >> (16 * (q & 1) + 8));
                    sts_v4(sb + sw_off(t, 4 * q + 0), restore8(cur.c[q].x, s0, cur.g));
                    sts_v4(sb + sw_off(t, 4 * q + 1), restore8(cur.c[q].y, s0, cur.g));
                    sts_v4(sb + sw_off(t, 4 * q + 2), restore8(cur.c[q].z, s1, cur.g));
                    sts_v4(sb + sw_off(t, 4 * q + 3), restore8(cur.c[q].w, s1, cur.g));
                }
            } else {                                      // past the window: zero rows
#pragma unroll
                for (int c = 0; c < 16; ++c) sts_v4(sb + sw_off(t, c), make_uint4(0, 0, 0, 0));
            }
            fence_async_smem();                           // generic-proxy writes -> tensor core
            mbar_arrive(full + 8 * st);
        }
    } else if (warp >= 16) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(kRegsMma) : "memory");
        if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer (whole warp)
        bool ok = true, issued = false;
        // S_t(i) = Q_t K_i^T into S_t; the stage's K is read by both Q tiles
        auto issue_s = [&](int qt, int i) {
            const uint64_t qdesc = kmajor_desc(base + OFF_Q + qt * 2 * kRegion);
            const uint64_t kdesc = kmajor_desc(base + OFF_KV + (i & 1) * KV_STAGE);
#pragma unroll 1
            for (int kk = 0; kk < kD / 16; ++kk) {
                // K step kk: region kk / 4, 32 bytes per step inside the 128-byte row
                const uint64_t off = (uint64_t)((kk >> 2) * (kRegion >> 4) + 2 * (kk & 3));
                tc_mma_ss(tmem + S_COL + 128 * qt, qdesc + off, kdesc + off, kIdescS, kk != 0);
            }
            tc_commit(bar_s_full + 8 * qt);
            issued = true;
        };
        // O_t += P_t(i) V_i: A = P_t (BF16 pairs in the first 64 columns of S_t), B = V_i
        auto issue_pv = [&](int qt, int i) {
            const uint32_t vbase = base + OFF_KV + (i & 1) * KV_STAGE + 2 * kRegion;
#pragma unroll 1
            for (int kt = 0; kt < kBKV / 16; ++kt)
                tc_mma_ts(tmem + O_COL + 128 * qt, tmem + S_COL + 128 * qt + 8 * kt, mnmajor_desc(vbase + 2048 * kt),
                          kIdescPV, (i | kt) != 0);
        };
        auto wait_k = [&](int i) -> bool {
            if (!warp_wait(bar_k_full + 8 * (i & 1), (i >> 1) & 1)) return false;
            tc_fence_after();
            return true;
        };
        // S of both Q tiles, then K's stage goes back to the producer
        auto issue_s_pair = [&](int i) {
            issue_s(0, i);
            if (q1_live) issue_s(1, i);
            tc_commit(bar_k_empty + 8 * (i & 1));
        };
        if (ntiles > 0 && wait_k(0)) {
            issue_s_pair(0);
        } else {
            ok = false;
        }
        for (int i = 0; ok && i < ntiles; ++i) {
            const bool more = i + 1 < ntiles;
            // Q tile 0: P.V(i) once its P and V(i) are in place
            if (!warp_wait(bar_p_full, i & 1) || !warp_wait(bar_v_full + 8 * (i & 1), (i >> 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            issue_pv(0, i);
            if (!q1_live) tc_commit(bar_v_empty + 8 * (i & 1));
            if (!more) tc_commit(bar_o_done);
            // S_0(i + 1) as soon as K(i + 1) is restored; S_1(i + 1) after P.V_1(i) (P_1 lives in S_1)
            if (more) {
                if (!wait_k(i + 1)) { ok = false; break; }
                issue_s(0, i + 1);
            }
            if (q1_live) {
                if (!warp_wait(bar_p_full + 8, i & 1)) { ok = false; break; }
                tc_fence_after();
                issue_pv(1, i);
                tc_commit(bar_v_empty + 8 * (i & 1));
                if (!more) tc_commit(bar_o_done + 8);
                if (more) issue_s(1, i + 1);
            }
            if (more) tc_commit(bar_k_empty + 8 * ((i + 1) & 1));
        }
        if (issued) {
            tc_commit(bar_drain);
            if (lane == 0 && !mbar_wait_bounded(bar_drain, 0, nullptr, kWaitLimitNs)) give_up();
        }
        __syncwarp();
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" :: "n"(kRegsSoftmax) : "memory");
        if (warp < 4 || q1_live) {
        // ------------------------------------------------------------ softmax + epilogue
        const int qt = warp >> 2;                         // Q tile of this warpgroup
        const int r = threadIdx.x & 127;                  // query row = tensor-memory lane
        const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t scol = lane_base + S_COL + 128 * qt, ocol = lane_base + O_COL + 128 * qt;
        const uint32_t s_full = bar_s_full + 8 * qt, p_full = bar_p_full + 8 * qt;
        const float c2 = j.scale_log2;
        const bool pos = c2 >= 0.0f;
        float m = -INFINITY, l = 0.0f;
        bool ok = true;
        for (int i = 0; ok && i < ntiles; ++i) {
            if (!warp_wait(s_full, i & 1)) { ok = false; break; }
            tc_fence_after();
            const int64_t t0 = (int64_t)i * kBKV;
            const bool full = t0 + kBKV <= j.total_tokens;
            // the tile's 128 raw scores of this row, in one batch of tensor-memory loads
            uint32_t s[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tc_ld32_nowait(scol + 32 * c, s[c]);
            tc_wait_ld();
            // the row maximum of the raw scores (tokens past the window excluded); scaling it
            // afterwards gives the maximum of the scaled scores exactly (rounding is monotone), for a
            // positive scale; a negative scale takes the minimum instead
            float xm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            if (full && pos) {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; e += 2)
                        xm[(e >> 1) & 3] = fmax3(xm[(e >> 1) & 3], __uint_as_float(s[c][e]), __uint_as_float(s[c][e + 1]));
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (t0 + 32 * c + e < j.total_tokens)
                            xm[e & 3] = fmaxf(xm[e & 3], pos ? __uint_as_float(s[c][e]) : -__uint_as_float(s[c][e]));
            }
            const float xr = fmaxf(fmaxf(xm[0], xm[1]), fmaxf(xm[2], xm[3]));
            const float x = xr == -INFINITY ? -INFINITY : (pos ? xr * c2 : -xr * c2);
            const float mn = fmaxf(m, x);
            const float b = mn == -INFINITY ? 0.0f : mn;
            const float alpha = ex2(m - b);
            // P = 2^(s * c2 - b) (BF16 pairs) and its row sum, paired FP32 arithmetic; P's 64 words go
            // to S columns [0, 64), already read
            float2 sum2[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t p[32];
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int c = 2 * hh + cc;
                    if (full) {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const float2 tv = fma2(make_float2(__uint_as_float(s[c][e]), __uint_as_float(s[c][e + 1])), c2, -b);
                            const float2 pp = make_float2(ex2(tv.x), ex2(tv.y));
                            sum2[(e >> 1) & 1] = add2(sum2[(e >> 1) & 1], pp);
                            p[16 * cc + e / 2] = bf16x2(pp.x, pp.y);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const float2 tv = fma2(make_float2(__uint_as_float(s[c][e]), __uint_as_float(s[c][e + 1])), c2, -b);
                            const float p0 = t0 + 32 * c + e < j.total_tokens ? ex2(tv.x) : 0.0f;
                            const float p1 = t0 + 32 * c + e + 1 < j.total_tokens ? ex2(tv.y) : 0.0f;
                            sum2[(e >> 1) & 1] = add2(sum2[(e >> 1) & 1], make_float2(p0, p1));
                            p[16 * cc + e / 2] = bf16x2(p0, p1);
                        }
                    }
                }
                tc_st32(scol + 32 * hh, p);
            }
            // O_t is stable here (s_full(i) implies P.V(i - 1) done; P.V(i) waits for p_full): rescale
            // it when any row of the warp moved its maximum (tcgen05.ld/st are warp-wide)
            if (i > 0 && __any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
#pragma unroll 1
                for (int c = 0; c < 4; c += 2) {
                    uint32_t v0[32], v1[32];
                    tc_ld32_nowait(ocol + 32 * c, v0);
                    tc_ld32_nowait(ocol + 32 * c + 32, v1);
                    tc_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        v0[e] = __float_as_uint(__uint_as_float(v0[e]) * alpha);
                        v1[e] = __float_as_uint(__uint_as_float(v1[e]) * alpha);
                    }
                    tc_st32(ocol + 32 * c, v0);
                    tc_st32(ocol + 32 * c + 32, v1);
                }
            }
            const float sum = (sum2[0].x + sum2[0].y) + (sum2[1].x + sum2[1].y);
            l = l * alpha + sum;
            m = mn;
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(p_full);
        }
        if (ok && ntiles > 0 && warp_wait(bar_o_done + 8 * qt, 0)) {
            tc_fence_after();
            const float inv = 1.0f / l;
            const int64_t row = q0 + qt * kBQ + r;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t v[32];
                tc_ld32_nowait(ocol + 32 * c, v);
                tc_wait_ld();
                if (row < j.tq && NVFP4_CHECKED(row * j.ldo + head * kD + 32 * c, 32, j.o_elems, status)) {
                    uint16_t *dst = j.o + row * j.ldo + head * kD + 32 * c;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 w = make_uint4(
                            bf16x2(__uint_as_float(v[8 * q + 0]) * inv, __uint_as_float(v[8 * q + 1]) * inv),
                            bf16x2(__uint_as_float(v[8 * q + 2]) * inv, __uint_as_float(v[8 * q + 3]) * inv),
                            bf16x2(__uint_as_float(v[8 * q + 4]) * inv, __uint_as_float(v[8 * q + 5]) * inv),
                            bf16x2(__uint_as_float(v[8 * q + 6]) * inv, __uint_as_float(v[8 * q + 7]) * inv));
                        *reinterpret_cast<uint4 *>(dst + 8 * q) = w;
                    }
                }
            }
        }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

}  // namespace

cudaError_t launch_kv_attention(const AttnJob &j, int32_t *status, cudaStream_t s) {
    if (j.tq <= 0) return cudaSuccess;
    static std::atomic<bool> attr_set[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(kv_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        // setmaxnreg.inc draws on the registers the block launched with: launched with fewer
        // than the split assumes, the softmax warpgroups would wait for registers forever
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, kv_attention_kernel);
        if (e != cudaSuccess) return e;
        if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
        attr_set[dev].store(true, std::memory_order_release);
    }
    const dim3 grid((unsigned)(ceil_div(j.tq, kQTiles * kBQ) * j.heads));
    return launch_pdl(kv_attention_kernel, grid, dim3(kThreads), kSmemBytes, s, j, status);
}

}  // namespace nvfp4
