// gemm.cu -- NVFP4 W4A4 GEMM on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// Y[M,N] = alpha * A[M,K] . B[N,K]^T (+ bias | + residual), A and B NVFP4 (E2M1 codes with one
// E4M3 scale per 16 elements along K), FP32 accumulation in tensor memory, alpha = gA*gB.
// LongLive-2.0 runs its linear layers as W4A4 NVFP4 GEMMs on Blackwell and accelerates its
// training GEMMs with NVFP4 (abstract, fugumt.com mirror; yourai.pro: the speed-up depends on
// Blackwell's FP4 tensor cores).
//
// Design:
//   - Persistent CTAs (one per SM, 221 KB of shared memory each), tiles of 128 x 256 outputs,
//     tile t -> (m-block t % mt, n-block t / mt) so that concurrently running CTAs share B tiles
//     and all of A in L2.
//   - Warp 0: producer.  Per 256-wide K tile it TMA-loads the A and B code tiles (128-byte rows,
//     128B swizzle) and bulk-copies the matching scale atoms, which the quantizer already wrote
//     in the tensor-core scale layout (4 contiguous 512-byte atoms per 128 rows), into a 4-stage
//     mbarrier pipeline.
//   - Warp 1: MMA issuer.  Copies each stage's scale atoms shared -> tensor memory
//     (tcgen05.cp 32x128b.warpx4) and issues four tcgen05.mma kind::mxf4nvf4 block16
//     (M=128, N=256, K=64) per stage; tcgen05.commit frees the stage and, after the last K
//     tile, signals the epilogue.
//   - Warps 2-5: epilogue.  tcgen05.ld 32 columns at a time, t = alpha*acc (+bias | +R) in FP32,
//     BF16 RNE (or FP32) stores, then release the accumulator.
//   - Tensor memory: 512 columns; accumulator in columns [0,256), scales after it.
//   - Every mbarrier wait is bounded (2 s); a wait that gives up raises an abort flag shared by
//     all roles, writes NVFP4_ERR_TIMEOUT to the status word, drains the copies and MMAs this
//     CTA has in flight (bounded), frees tensor memory and returns.
#include <atomic>
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "launch.h"

namespace nvfp4 {

namespace {

constexpr int BM = 128, BN = 256, BK = 256;     // elements; a K tile is 128 bytes of codes per row
constexpr int KSTEP = 64;                        // K of one kind::mxf4nvf4 MMA
constexpr int KSTEPS_PER_TILE = BK / KSTEP;      // 4
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK / 2;             // 16384 bytes
constexpr int B_STAGE = BN * BK / 2;             // 32768 bytes
constexpr int SFA_STAGE = KSTEPS_PER_TILE * 512; // 2048: one 128x4 atom per K step
constexpr int SFB_STAGE = 2 * SFA_STAGE;         // 4096: two 128-row atoms per K step
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_STAGE;
constexpr int OFF_SFA = OFF_B + STAGES * B_STAGE;
constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_STAGE;
constexpr int OFF_BAR = OFF_SFB + STAGES * SFB_STAGE;
constexpr int NUM_BARS = 2 * STAGES + 3;         // full[], empty[], tmem_full, tmem_empty, drain
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024; // + slack for the 1024-byte alignment
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0, SFA_COL = 256, SFB_COL = 256 + 4 * KSTEPS_PER_TILE;

static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// Instruction descriptor of tcgen05.mma kind::mxf4nvf4: A and B E2M1 (format 1), K-major, UE4M3
// scales (scale format 0), dense K = 64, M = 128 (m_dim = M>>4 at bit 24), N = 256 (n_dim = N>>3
// at bit 17), scale-factor ids 0.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

// Shared-memory matrix descriptor, K-major, 128B swizzle: start>>4, SBO = 1024 bytes (8 rows of
// 128 bytes), descriptor version 1 (bit 46), layout type 2 (SWIZZLE_128B) at bit 61.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Descriptor of a 512-byte scale atom for tcgen05.cp: no swizzle, 8-row core matrices of 16-byte
// rows stored contiguously (SBO = 128 bytes).
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 32) | (1ull << 46);
}

// The issue helpers below are executed by all 32 lanes of a converged warp with warp-uniform
// operands; elect.sync picks the one lane that issues.  Issuing from a divergent lane-0 branch
// instead makes the compiler move every operand into uniform registers lane by lane, which costs
// ~100 cycles per instruction and starves the tensor core.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
                 "@p cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n\t}"
                 :: "r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar) : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
                 "@p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n\t}"
                 :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

__device__ __forceinline__ void arrive_expect_tx_elect(uint32_t bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
                 "@p mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t}"
                 :: "r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
                 "@p tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}"
                 :: "r"(bar) : "memory");
}

__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t desc) {
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
                 "@p tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;\n\t}"
                 :: "r"(taddr), "l"(desc) : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accum,
                                       uint32_t sfa, uint32_t sfb) {
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
                 :: "r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accum), "r"(sfa), "r"(sfb) : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns of tensor memory -> 32 registers per thread.
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
                 "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
                   "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
                   "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint4 ldg_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ void stg_v4(void *p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                  const __grid_constant__ GemmArgs args) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sbase = smem_raw + (base - raw);
    const uint32_t bar_full = base + OFF_BAR, bar_empty = bar_full + 8 * STAGES;
    const uint32_t bar_tmem_full = bar_empty + 8 * STAGES, bar_tmem_empty = bar_tmem_full + 8;
    const uint32_t bar_drain = bar_tmem_empty + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sbase + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sbase + OFF_MISC + 4);

    const int warp = __shfl_sync(0xFFFFFFFFu, (int)(threadIdx.x >> 5), 0);   // warp-uniform
    const int lane = threadIdx.x & 31;
    const int64_t M = args.M, N = args.N, K = args.K;
    const int mt = (int)ceil_div(M, BM), nt = (int)ceil_div(N, BN);
    const int num_tiles = mt * nt;
    const int ksteps = (int)ceil_div(K, KSTEP);          // also scale atoms per 128-row block
    const int nkt = (ksteps + KSTEPS_PER_TILE - 1) / KSTEPS_PER_TILE;
    const int b_row_atoms = (int)ceil_div(N, 128);

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(bar_full + 8 * i, 1);
            mbar_init(bar_empty + 8 * i, 1);
        }
        mbar_init(bar_tmem_full, 1);
        mbar_init(bar_tmem_empty, 128);
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
        asm volatile("prefetch.tensormap [%0];" :: "l"(&map_a) : "memory");
        asm volatile("prefetch.tensormap [%0];" :: "l"(&map_b) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_addr(tmem_slot)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = __shfl_sync(0xFFFFFFFFu, *tmem_slot, 0);
    griddep_wait();                                       // operands written by earlier kernels
    griddep_launch_dependents();
    __shared__ SmemRecord qrec;                           // NVFP4-emitting epilogue only
    if (args.q_rec) {
        load_record_plain(args.q_rec, qrec);
        __syncthreads();
    }

    auto give_up = [&]() {
        *abort_flag = 1;
        set_status(args.status, NVFP4_ERR_TIMEOUT);
    };
    // lane 0 of the warp waits; the outcome is broadcast so the warp never diverges on it
    auto warp_wait = [&](uint32_t bar, uint32_t parity) -> bool {
        const bool ok = mbar_wait_warp(bar, parity, abort_flag, kWaitLimitNs);
        if (!ok && lane == 0) give_up();
        return ok;
    };

    if (warp == 0) {
        // ---------------------------------------------------------------- producer (whole warp,
        // converged; one elected lane issues)
        uint32_t stage = 0, phase = 0;
        uint32_t used = 0, last_parity = 0;               // per-stage bit masks
        bool ok = true;
        for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
            const int mb = t % mt, nb = t / mt;
            const bool b_hi = (2 * nb + 1) < b_row_atoms;
            for (int kt = 0; kt < nkt; ++kt) {
                if (!warp_wait(bar_empty + 8 * stage, phase ^ 1)) {
                    ok = false;
                    break;
                }
                const int nsteps = min(KSTEPS_PER_TILE, ksteps - kt * KSTEPS_PER_TILE);
                const uint32_t sf_bytes = (uint32_t)nsteps * 512u;
                const uint32_t bytes = A_STAGE + B_STAGE + sf_bytes * (b_hi ? 3u : 2u);
                const uint32_t fb = bar_full + 8 * stage;
                arrive_expect_tx_elect(fb, bytes);
                tma_load_2d(base + OFF_A + stage * A_STAGE, &map_a, kt * (BK / 2), mb * BM, fb);
                tma_load_2d(base + OFF_B + stage * B_STAGE, &map_b, kt * (BK / 2), nb * BN, fb);
                const int64_t k_atom = (int64_t)kt * KSTEPS_PER_TILE;
                bulk_load(base + OFF_SFA + stage * SFA_STAGE,
                          args.a_sf + ((int64_t)mb * ksteps + k_atom) * 512, sf_bytes, fb);
                bulk_load(base + OFF_SFB + stage * SFB_STAGE,
                          args.b_sf + ((int64_t)(2 * nb) * ksteps + k_atom) * 512, sf_bytes, fb);
                if (b_hi)
                    bulk_load(base + OFF_SFB + stage * SFB_STAGE + SFA_STAGE,
                              args.b_sf + ((int64_t)(2 * nb + 1) * ksteps + k_atom) * 512, sf_bytes, fb);
                used |= 1u << stage;
                last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        }
        // every issued copy must land before this CTA's shared memory can be released
        if (lane == 0) {
            for (int i = 0; i < STAGES; ++i)
                if (((used >> i) & 1u) &&
                    !mbar_wait_bounded(bar_full + 8 * i, (last_parity >> i) & 1u, nullptr, kWaitLimitNs))
                    give_up();
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer (whole warp,
        // converged; one elected lane issues)
        uint32_t stage = 0, phase = 0, acc_phase = 0;
        bool ok = true, issued = false;
        for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
            if (!warp_wait(bar_tmem_empty, acc_phase ^ 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            for (int kt = 0; kt < nkt; ++kt) {
                if (!warp_wait(bar_full + 8 * stage, phase)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int nsteps = min(KSTEPS_PER_TILE, ksteps - kt * KSTEPS_PER_TILE);
                const uint32_t sfa_s = base + OFF_SFA + stage * SFA_STAGE;
                const uint32_t sfb_s = base + OFF_SFB + stage * SFB_STAGE;
                const uint64_t adesc = sw128_desc(base + OFF_A + stage * A_STAGE);
                const uint64_t bdesc = sw128_desc(base + OFF_B + stage * B_STAGE);
                for (int j = 0; j < nsteps; ++j) {
                    tc_cp_sf(tmem + SFA_COL + 4 * j, sf_desc(sfa_s + 512 * j));
                    tc_cp_sf(tmem + SFB_COL + 8 * j, sf_desc(sfb_s + 512 * j));
                    tc_cp_sf(tmem + SFB_COL + 8 * j + 4, sf_desc(sfb_s + SFA_STAGE + 512 * j));
                }
                for (int j = 0; j < nsteps; ++j) {
                    // a K step is 64 codes = 32 bytes along the swizzled 128-byte row
                    tc_mma(tmem + ACC_COL, adesc + 2 * j, bdesc + 2 * j, kIdesc, (kt | j) != 0,
                           tmem + SFA_COL + 4 * j, tmem + SFB_COL + 8 * j);
                }
                tc_commit(bar_empty + 8 * stage);
                issued = true;
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok) break;
            tc_commit(bar_tmem_full);
            acc_phase ^= 1;
        }
        // wait for every MMA / copy issued here before tensor memory is freed
        if (issued) {
            tc_commit(bar_drain);
            if (lane == 0 && !mbar_wait_bounded(bar_drain, 0, nullptr, kWaitLimitNs)) give_up();
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue (warps 2..5)
        const int sub = warp & 3;                         // tensor-memory lane quarter of this warp
        const float alpha = __fmul_rn(*args.ga, *args.gb);
        const bool quant = args.q_rec && qrec.ok;
        const int64_t q_rows = args.q_sf_layout ? 128 * ceil_div(M, 128) : M;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
            if (!warp_wait(bar_tmem_full, acc_phase)) break;
            tc_fence_after();
            const int mb = t % mt, nb = t / mt;
            const int64_t m = (int64_t)mb * BM + sub * 32 + lane;
            const bool row_ok = m < M;
            const uint32_t trow = tmem + ((uint32_t)(sub * 32) << 16) + ACC_COL;
            uint32_t cam0 = 0, cam1 = 0;                  // max |Y| of this warp's two 32 x 128 blocks
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tc_ld32(trow + c * 32, r);
                const int64_t n0 = (int64_t)nb * BN + c * 32;
                if (!row_ok || n0 >= N) {
                    if (quant && n0 < N && m < q_rows) store_sf_pair(args, m, n0 >> 4, 0u);   // scale padding rows
                    continue;
                }
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(alpha, __uint_as_float(r[i]));
                if (args.bias) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (n0 + 8 * q >= N || !NVFP4_CHECKED(n0 + 8 * q, 8, args.bias_elems, args.status)) break;
                        const uint4 b = ldg_v4(args.bias + n0 + 8 * q);
                        const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            v[8 * q + 2 * i] = __fadd_rn(v[8 * q + 2 * i], bf16_lo(bw[i]));
                            v[8 * q + 2 * i + 1] = __fadd_rn(v[8 * q + 2 * i + 1], bf16_hi(bw[i]));
                        }
                    }
                } else if (args.resid) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (n0 + 8 * q >= N ||
                            !NVFP4_CHECKED(m * args.ldy + n0 + 8 * q, 8, args.resid_elems, args.status))
                            break;
                        const uint4 b = ldg_v4(args.resid + m * args.ldy + n0 + 8 * q);
                        const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            v[8 * q + 2 * i] = __fadd_rn(v[8 * q + 2 * i], bf16_lo(bw[i]));
                            v[8 * q + 2 * i + 1] = __fadd_rn(v[8 * q + 2 * i + 1], bf16_hi(bw[i]));
                        }
                    }
                }
                if (!args.y_f32) {
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) w[i] = bf16x2(v[2 * i], v[2 * i + 1]);
                    if (args.y) {
                        uint16_t *yrow = reinterpret_cast<uint16_t *>(args.y) + m * args.ldy + n0;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            if (n0 + 8 * q >= N || !NVFP4_CHECKED(m * args.ldy + n0 + 8 * q, 8, args.y_elems, args.status))
                                break;
                            stg_v4(yrow + 8 * q, make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]));
                        }
                    }
                    if (quant) emit_nvfp4_chunk(args, qrec, m, n0, w);
                    if (args.cam_partial) {
                        const uint32_t b = max(absmax_bits16(w), absmax_bits16(w + 8));
                        if (c < 4) cam0 = max(cam0, b);
                        else cam1 = max(cam1, b);
                    }
                } else {
                    float *yrow = reinterpret_cast<float *>(args.y) + m * args.ldy + n0;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (n0 + 4 * q >= N || !NVFP4_CHECKED(m * args.ldy + n0 + 4 * q, 4, args.y_elems, args.status))
                            break;
                        stg_v4(yrow + 4 * q, make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                                                        __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3])));
                    }
                }
            }
            if (args.cam_partial) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    cam0 = max(cam0, __shfl_xor_sync(0xFFFFFFFFu, cam0, o));
                    cam1 = max(cam1, __shfl_xor_sync(0xFFFFFFFFu, cam1, o));
                }
                const int64_t r32 = ((int64_t)mb * BM + sub * 32) >> 5;
                const int64_t c128 = ((int64_t)nb * BN) >> 7;
                if (lane == 0 && r32 < ceil_div(M, 32)) {
                    if (c128 < args.cam_n128 &&
                        NVFP4_CHECKED(r32 * args.cam_n128 + c128, 1, args.cam_elems, args.status))
                        args.cam_partial[r32 * args.cam_n128 + c128] = cam0;
                    if (c128 + 1 < args.cam_n128 &&
                        NVFP4_CHECKED(r32 * args.cam_n128 + c128 + 1, 1, args.cam_elems, args.status))
                        args.cam_partial[r32 * args.cam_n128 + c128 + 1] = cam1;
                }
            }
            tc_fence_before();
            mbar_arrive(bar_tmem_empty);
            acc_phase ^= 1;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D uint8 map over a code matrix [rows][pitch] with a (128-byte x box_rows) box, 128B swizzle.
bool make_code_map(CUtensorMap *map, const void *ptr, int64_t rows, int64_t pitch, uint32_t box_rows) {
    auto fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)pitch, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)pitch};
    cuuint32_t box[2] = {128u, box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_gemm(const GemmArgs &args, cudaStream_t s) {
    if (args.M > BM) return launch_gemm_2sm(args, s);     // CTA pairs once M spans two row blocks
    static std::atomic<bool> attr_set[64];             // per device; a repeated set is harmless
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(nvfp4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true, std::memory_order_release);
    }
    CUtensorMap ma, mb;
    if (!make_code_map(&ma, args.a_codes, args.M, args.a_pitch, BM) ||
        !make_code_map(&mb, args.b_codes, args.N, args.b_pitch, BN))
        return cudaErrorInvalidValue;
    const int64_t tiles = ceil_div(args.M, BM) * ceil_div(args.N, BN);
    int grid = num_sms();
    if (tiles < grid) grid = (int)tiles;
    return launch_pdl(nvfp4_gemm_kernel, dim3(grid), dim3(NUM_THREADS), SMEM_BYTES, s, ma, mb, args);
}

}  // namespace nvfp4
