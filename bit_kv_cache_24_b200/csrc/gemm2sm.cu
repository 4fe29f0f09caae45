// gemm2sm.cu -- NVFP4 W4A4 GEMM on CTA pairs (tcgen05 cta_group::2, sm_100a).
//
// Same operation as gemm.cu (Y = gA*gB * A.B^T (+bias | +residual), E2M1 x E4M3/16-block operands,
// FP32 accumulation in tensor memory; LongLive-2.0's W4A4 NVFP4 linear layers and NVFP4 training
// GEMMs), for M > 128.
//
// Why pairs: a 128 x 256 tile per SM needs 54 KB of operands per 256-wide K step, more than the
// ~64 B/clk an SM's TMA path sustains at full tensor rate.  Two CTAs of a cluster compute one
// 256 x 256 tile with tcgen05.mma.cta_group::2 (M = 256): each CTA loads its own 128 rows of A and
// 128 of the 256 rows of B, and the pair's tensor cores share the B halves, so an SM loads 38 KB
// per K step for the same FLOPs.
//
// Roles (384 threads per CTA):
//   warp 0      producer (both CTAs): TMA loads of A, B, SFA, SFB codes/scales for its CTA; the
//               loads signal the leader CTA's full barrier (cp.async.bulk.tensor .cta_group::2);
//               the leader's producer posts the pair's transaction bytes.
//   warp 1      MMA issuer (leader): 4 x tcgen05.mma.cta_group::2 kind::mxf4nvf4 per K step of 256,
//               commits multicast to both CTAs' empty barriers and, per tile, tmem_full.
//   warp 2      scale copier (leader): tcgen05.cp.cta_group::2 of each stage's scale atoms into a
//               per-stage tensor-memory buffer (each CTA's shared memory -> its own tensor memory),
//               then commits to sf_full.  Separate from the MMA warp so the two issue streams run
//               in parallel.
//   warps 4-11  epilogue (both CTAs): two warps per tensor-memory lane quarter, 128 columns each;
//               a warp drains its columns to registers and releases tensor memory before the
//               scaling, bias/residual add, rounding and stores, which overlap the next tile.
//               BF16 output leaves through shared memory: per 32 x 32 chunk a warp writes its
//               rows into a 64-byte-swizzled staging buffer (two per warp) and one lane issues a
//               TMA tensor store, so every global write is a full line (per-lane 16-byte row
//               stores to 32 different rows ran the epilogue at ~1.3 TB/s and bounded the GEMM
//               on the short-K shapes).  FP32 output (accuracy checks) keeps direct stores.
// Tile order: M-fastest, or N-fastest when A is the larger operand (then a few A stripes are
// live at a time and all of B stays in L2, instead of every A stripe being re-read per N tile).
// Tensor memory per CTA: accumulator columns [0, 256), scale buffers per stage after it.
// Scale tiles are read through 2-D tensor maps over the 512-byte atoms (viewed as uint64), so
// atom rows past M or N are zero-filled by TMA like the code tiles.
// Every wait is time-bounded; a wait that gives up reports NVFP4_ERR_TIMEOUT and the CTA returns.
#include <atomic>
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "launch.h"

namespace nvfp4 {

namespace {

constexpr int BM = 256, BN = 256, BK = 256;         // pair tile; K tile = 128 bytes of codes per row
constexpr int BM_CTA = 128, BN_CTA = 128;           // rows of A and of B each CTA loads
constexpr int KSTEP = 64;
constexpr int KSTEPS_PER_TILE = BK / KSTEP;         // 4
constexpr int STAGES = 5;
constexpr int A_STAGE = BM_CTA * BK / 2;            // 16384
constexpr int B_STAGE = BN_CTA * BK / 2;            // 16384
constexpr int SFA_STAGE = KSTEPS_PER_TILE * 512;    // 2048: this CTA's 128 rows
constexpr int SFB_STAGE = 2 * SFA_STAGE;            // 4096: all 256 columns of the pair tile
constexpr uint32_t STAGE_TX_PAIR = 2u * (A_STAGE + B_STAGE + SFA_STAGE + SFB_STAGE);
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_STAGE;
constexpr int OFF_SFA = OFF_B + STAGES * B_STAGE;
constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_STAGE;
constexpr int OFF_EPI = OFF_SFB + STAGES * SFB_STAGE;   // output staging, 1024-aligned
constexpr int EPI_BUF = 2048;                           // one warp's 32 rows x 32 BF16 columns
constexpr int OFF_BAR = OFF_EPI + 8 * 2 * EPI_BUF;      // two buffers per epilogue warp
static_assert(OFF_EPI % 1024 == 0, "staging alignment (64-byte swizzle period)");
constexpr int NUM_BARS = 3 * STAGES + 3;            // full[], empty[], sf_full[], tmem_full, tmem_empty, drain
constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
constexpr int NUM_THREADS = 384;
constexpr int EPI_WARP0 = 4, EPI_WARPS = 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0, SF_COL0 = 256, SF_STAGE_COLS = 48;   // per stage: SFA 16 + SFB 32
static_assert(SF_COL0 + STAGES * SF_STAGE_COLS <= TMEM_COLS, "tensor memory budget");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// tcgen05.mma kind::mxf4nvf4 descriptor: E2M1 x E2M1, UE4M3 scales, K-major, M = 256 (pair), N = 256.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 32) | (1ull << 46);
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Shared::cluster address of the same shared-memory offset in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(saddr), "r"(rank));
    return out;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// 2-D TMA tile load into this CTA's shared memory whose completion is counted on `bar`, which may
// be the leader CTA's barrier (cta_group::2 form).  Converged warp, one elected lane issues.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
                 "@p cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n\t}"
                 :: "r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar) : "memory");
}

__device__ __forceinline__ void arrive_expect_tx_elect(uint32_t bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
                 "@p mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t}"
                 :: "r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Commit of this thread's earlier cta_group::2 tcgen05 operations to the barrier at the same
// offset in every CTA of `mask`.
__device__ __forceinline__ void tc_commit_mc(uint32_t bar, uint16_t mask) {
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
                 "@p tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n\t}"
                 :: "r"(bar), "h"(mask) : "memory");
}

__device__ __forceinline__ void tc_commit_local(uint32_t bar) {
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
                 "@p tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}"
                 :: "r"(bar) : "memory");
}

__device__ __forceinline__ void tc_cp_sf_pair(uint32_t taddr, uint64_t desc) {
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
                 "@p tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;\n\t}"
                 :: "r"(taddr), "l"(desc) : "memory");
}

__device__ __forceinline__ void tc_mma_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accum,
                                            uint32_t sfa, uint32_t sfb) {
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
                 :: "r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accum), "r"(sfa), "r"(sfb) : "memory");
}

// 32 lanes x 32 consecutive 32-bit tensor-memory columns -> 32 registers per thread, without the
// wait: several loads are issued back to back, then one tcgen05.wait::ld.
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

__device__ __forceinline__ uint4 ldg_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ void stg_v4(void *p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

struct Maps {
    CUtensorMap a, b, sfa, sfb, y;
    int y_tma;      // BF16 output through the y map (else direct stores)
    int n_fast;     // tile order: N index fastest
};

__device__ __forceinline__ void sts_v4(uint32_t saddr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" :: "r"(saddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
nvfp4_gemm_2sm_kernel(const __grid_constant__ Maps maps, const __grid_constant__ GemmArgs args) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sbase = smem_raw + (base - raw);
    const uint32_t bar_full = base + OFF_BAR, bar_empty = bar_full + 8 * STAGES, bar_sf = bar_empty + 8 * STAGES;
    const uint32_t bar_tmem_full = bar_sf + 8 * STAGES, bar_tmem_empty = bar_tmem_full + 8;
    const uint32_t bar_drain = bar_tmem_empty + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sbase + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sbase + OFF_MISC + 4);

    const int warp = __shfl_sync(0xFFFFFFFFu, (int)(threadIdx.x >> 5), 0);
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int64_t M = args.M, N = args.N, K = args.K;
    const int mt = (int)ceil_div(M, BM), nt = (int)ceil_div(N, BN);
    const int num_tiles = mt * nt;
    const int ksteps = (int)ceil_div(K, KSTEP);
    const int nkt = (ksteps + KSTEPS_PER_TILE - 1) / KSTEPS_PER_TILE;
    const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(bar_full + 8 * i, 1);
            mbar_init(bar_empty + 8 * i, 1);
            mbar_init(bar_sf + 8 * i, 1);
        }
        mbar_init(bar_tmem_full, 1);
        mbar_init(bar_tmem_empty, 2 * EPI_WARPS);          // one arrival per epilogue warp of the pair
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    if (warp == 0) {
        asm volatile("prefetch.tensormap [%0];" :: "l"(&maps.a) : "memory");
        asm volatile("prefetch.tensormap [%0];" :: "l"(&maps.b) : "memory");
        asm volatile("prefetch.tensormap [%0];" :: "l"(&maps.sfa) : "memory");
        asm volatile("prefetch.tensormap [%0];" :: "l"(&maps.sfb) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     :: "r"(smem_addr(tmem_slot)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();                                       // barriers and tensor memory of both CTAs ready
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
    auto warp_wait = [&](uint32_t bar, uint32_t parity) -> bool {
        const bool ok = mbar_wait_warp(bar, parity, abort_flag, kWaitLimitNs);
        if (!ok && lane == 0) give_up();
        return ok;
    };

    if (warp == 0) {
        // ------------------------------------------------------------------------ producer
        const uint32_t lead_full = map_to_rank(bar_full, 0);
        uint32_t stage = 0, phase = 0, used = 0, last_parity = 0;
        bool ok = true;
        for (int t = cluster; ok && t < num_tiles; t += nclusters) {
            const int mb = maps.n_fast ? t / nt : t % mt, nb = maps.n_fast ? t % nt : t / mt;
            for (int kt = 0; kt < nkt; ++kt) {
                if (!warp_wait(bar_empty + 8 * stage, phase ^ 1)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = lead_full + 8 * stage;
                if (leader) arrive_expect_tx_elect(bar_full + 8 * stage, STAGE_TX_PAIR);
                tma_load_2d_pair(base + OFF_A + stage * A_STAGE, &maps.a, kt * (BK / 2), mb * BM + (int)rank * BM_CTA, fb);
                tma_load_2d_pair(base + OFF_B + stage * B_STAGE, &maps.b, kt * (BK / 2), nb * BN + (int)rank * BN_CTA, fb);
                tma_load_2d_pair(base + OFF_SFA + stage * SFA_STAGE, &maps.sfa, kt * 256, 2 * mb + (int)rank, fb);
                tma_load_2d_pair(base + OFF_SFB + stage * SFB_STAGE, &maps.sfb, kt * 256, 2 * nb, fb);
                used |= 1u << stage;
                last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        }
        // the leader's full barriers count both CTAs' loads: make sure they all landed
        if (leader && lane == 0) {
            for (int i = 0; i < STAGES; ++i)
                if (((used >> i) & 1u) &&
                    !mbar_wait_bounded(bar_full + 8 * i, (last_parity >> i) & 1u, nullptr, kWaitLimitNs))
                    give_up();
        }
        __syncwarp();
    } else if (warp == 2 && leader) {
        // ------------------------------------------------------------------------ scale copier
        uint32_t stage = 0, phase = 0;
        bool ok = true;
        for (int t = cluster; ok && t < num_tiles; t += nclusters) {
            for (int kt = 0; kt < nkt; ++kt) {
                if (!warp_wait(bar_full + 8 * stage, phase)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int nsteps = min(KSTEPS_PER_TILE, ksteps - kt * KSTEPS_PER_TILE);
                const uint32_t sfa_s = base + OFF_SFA + stage * SFA_STAGE;
                const uint32_t sfb_s = base + OFF_SFB + stage * SFB_STAGE;
                const uint32_t col = tmem + SF_COL0 + stage * SF_STAGE_COLS;
                for (int j = 0; j < nsteps; ++j) {
                    tc_cp_sf_pair(col + 4 * j, sf_desc(sfa_s + 512 * j));
                    tc_cp_sf_pair(col + 16 + 8 * j, sf_desc(sfb_s + 512 * j));
                    tc_cp_sf_pair(col + 16 + 8 * j + 4, sf_desc(sfb_s + SFA_STAGE + 512 * j));
                }
                tc_commit_local(bar_sf + 8 * stage);
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
        }
    } else if (warp == 1 && leader) {
        // ------------------------------------------------------------------------ MMA issuer
        uint32_t stage = 0, phase = 0, acc_phase = 0;
        bool ok = true, issued = false;
        for (int t = cluster; ok && t < num_tiles; t += nclusters) {
            if (!warp_wait(bar_tmem_empty, acc_phase ^ 1)) break;
            tc_fence_after();
            for (int kt = 0; kt < nkt; ++kt) {
                if (!warp_wait(bar_full + 8 * stage, phase) || !warp_wait(bar_sf + 8 * stage, phase)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int nsteps = min(KSTEPS_PER_TILE, ksteps - kt * KSTEPS_PER_TILE);
                const uint64_t adesc = sw128_desc(base + OFF_A + stage * A_STAGE);
                const uint64_t bdesc = sw128_desc(base + OFF_B + stage * B_STAGE);
                const uint32_t col = tmem + SF_COL0 + stage * SF_STAGE_COLS;
                for (int j = 0; j < nsteps; ++j)
                    tc_mma_pair(tmem + ACC_COL, adesc + 2 * j, bdesc + 2 * j, kIdesc, (kt | j) != 0,
                                col + 4 * j, col + 16 + 8 * j);
                tc_commit_mc(bar_empty + 8 * stage, 0x3);
                issued = true;
                if (++stage == STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok) break;
            tc_commit_mc(bar_tmem_full, 0x3);
            acc_phase ^= 1;
        }
        if (issued) {
            tc_commit_local(bar_drain);
            if (lane == 0 && !mbar_wait_bounded(bar_drain, 0, nullptr, kWaitLimitNs)) give_up();
        }
        __syncwarp();
    } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + EPI_WARPS) {
        // ------------------------------------------------------------------------ epilogue
        const int q = warp & 3;                           // tensor-memory lane quarter
        const int half = (warp - EPI_WARP0) >> 2;         // which 128 of the 256 columns
        const uint32_t lead_tmem_empty = map_to_rank(bar_tmem_empty, 0);
        const float alpha = __fmul_rn(*args.ga, *args.gb);
        const bool quant = args.q_rec && qrec.ok;
        const int64_t q_rows = args.q_sf_layout ? 128 * ceil_div(M, 128) : M;
        uint32_t acc_phase = 0;
        const bool y_tma = maps.y_tma != 0;
        uint32_t nstores = 0;                             // TMA stores issued by lane 0 of this warp
        const uint32_t sbuf0 = base + OFF_EPI + (uint32_t)(warp - EPI_WARP0) * 2 * EPI_BUF;
        for (int t = cluster; t < num_tiles; t += nclusters) {
            if (!warp_wait(bar_tmem_full, acc_phase)) break;
            tc_fence_after();
            const int mb = maps.n_fast ? t / nt : t % mt, nb = maps.n_fast ? t % nt : t / mt;
            const int64_t m = (int64_t)mb * BM + (int64_t)rank * BM_CTA + q * 32 + lane;
            const bool row_ok = m < M;
            const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16) + ACC_COL + half * 128;
            // drain this warp's 128 accumulator columns, then hand tensor memory back at once so
            // the pair's next tile accumulates while this one is scaled, rounded and stored
            uint32_t r[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tc_ld32_nowait(trow + c * 32, r[c]);
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" :: "r"(lead_tmem_empty) : "memory");
            uint32_t cam = 0;                             // max |Y| of this warp's 32 x 128 block
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int64_t n0 = (int64_t)nb * BN + half * 128 + c * 32;
                if (y_tma) {
                    const int ym = mb * BM + (int)rank * BM_CTA + q * 32;   // the warp's first row
                    if (n0 >= N) continue;                                    // warp-uniform
                    if (ym >= M) {                                            // warp-uniform: no live row
                        if (quant && m < q_rows) store_sf_pair(args, m, n0 >> 4, 0u);   // scale padding rows
                        continue;
                    }
                    float v[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(alpha, __uint_as_float(r[c][i]));
                    const uint16_t *addsrc = args.bias ? args.bias + n0
                                                       : (args.resid && row_ok ? args.resid + m * args.ldy + n0 : nullptr);
                    const int64_t addoff = args.bias ? n0 : m * args.ldy + n0;      // checked build
                    const int64_t addext = args.bias ? args.bias_elems : args.resid_elems;
                    (void)addoff;
                    (void)addext;
                    if (addsrc) {
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            if (n0 + 8 * g >= N) break;
                            if (!NVFP4_CHECKED(addoff + 8 * g, 8, addext, args.status)) break;
                            const uint4 b = ldg_v4(addsrc + 8 * g);
                            const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                v[8 * g + 2 * i] = __fadd_rn(v[8 * g + 2 * i], bf16_lo(bw[i]));
                                v[8 * g + 2 * i + 1] = __fadd_rn(v[8 * g + 2 * i + 1], bf16_hi(bw[i]));
                            }
                        }
                    }
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) w[i] = bf16x2(v[2 * i], v[2 * i + 1]);
                    const uint32_t sbuf = sbuf0 + (nstores & 1) * EPI_BUF;
                    // the store issued from this buffer two chunks ago must have finished reading it
                    if (lane == 0 && nstores >= 2) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                    __syncwarp();
                    // lane = row: 64-byte rows, 16-byte chunk g at (g ^ (row / 2) % 4) (SWIZZLE_64B);
                    // rows past M are written here but clipped by the store
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        sts_v4(sbuf + lane * 64 + ((g ^ ((lane >> 1) & 3)) << 4),
                               make_uint4(w[4 * g], w[4 * g + 1], w[4 * g + 2], w[4 * g + 3]));
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) {
                        asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
                                     :: "l"(&maps.y), "r"((int)n0), "r"(ym), "r"(sbuf) : "memory");
                        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                    }
                    ++nstores;
                    if (row_ok) {
                        if (quant) emit_nvfp4_chunk(args, qrec, m, n0, w);
                        if (args.cam_partial) cam = max(cam, max(absmax_bits16(w), absmax_bits16(w + 8)));
                    } else if (quant && m < q_rows) {
                        store_sf_pair(args, m, n0 >> 4, 0u);
                    }
                    continue;
                }
                if (!row_ok || n0 >= N) {
                    if (quant && n0 < N && m < q_rows) store_sf_pair(args, m, n0 >> 4, 0u);   // scale padding rows
                    continue;
                }
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(alpha, __uint_as_float(r[c][i]));
                const uint16_t *addsrc = args.bias ? args.bias + n0 : (args.resid ? args.resid + m * args.ldy + n0 : nullptr);
                const int64_t addoff = args.bias ? n0 : m * args.ldy + n0;          // checked build
                const int64_t addext = args.bias ? args.bias_elems : args.resid_elems;
                (void)addoff;
                (void)addext;
                if (addsrc) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        if (n0 + 8 * g >= N) break;
                        if (!NVFP4_CHECKED(addoff + 8 * g, 8, addext, args.status)) break;
                        const uint4 b = ldg_v4(addsrc + 8 * g);
                        const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            v[8 * g + 2 * i] = __fadd_rn(v[8 * g + 2 * i], bf16_lo(bw[i]));
                            v[8 * g + 2 * i + 1] = __fadd_rn(v[8 * g + 2 * i + 1], bf16_hi(bw[i]));
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
                        for (int g = 0; g < 4; ++g) {
                            if (n0 + 8 * g >= N || !NVFP4_CHECKED(m * args.ldy + n0 + 8 * g, 8, args.y_elems, args.status))
                                break;
                            stg_v4(yrow + 8 * g, make_uint4(w[4 * g], w[4 * g + 1], w[4 * g + 2], w[4 * g + 3]));
                        }
                    }
                    if (quant) emit_nvfp4_chunk(args, qrec, m, n0, w);
                    if (args.cam_partial) cam = max(cam, max(absmax_bits16(w), absmax_bits16(w + 8)));
                } else {
                    float *yrow = reinterpret_cast<float *>(args.y) + m * args.ldy + n0;
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        if (n0 + 4 * g >= N || !NVFP4_CHECKED(m * args.ldy + n0 + 4 * g, 4, args.y_elems, args.status))
                            break;
                        stg_v4(yrow + 4 * g, make_uint4(__float_as_uint(v[4 * g]), __float_as_uint(v[4 * g + 1]),
                                                        __float_as_uint(v[4 * g + 2]), __float_as_uint(v[4 * g + 3])));
                    }
                }
            }
            if (args.cam_partial) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) cam = max(cam, __shfl_xor_sync(0xFFFFFFFFu, cam, o));
                const int64_t r32 = ((int64_t)mb * BM + (int64_t)rank * BM_CTA + q * 32) >> 5;
                const int64_t c128 = ((int64_t)nb * BN + half * 128) >> 7;
                if (lane == 0 && r32 < ceil_div(M, 32) && c128 < args.cam_n128)
                    if (NVFP4_CHECKED(r32 * args.cam_n128 + c128, 1, args.cam_elems, args.status))
                        args.cam_partial[r32 * args.cam_n128 + c128] = cam;
            }
            acc_phase ^= 1;
        }
        // the TMA stores must have read the staging buffers and written Y before the CTA exits
        if (lane == 0 && nstores > 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();                                       // neither CTA leaves while its pair still uses it
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

bool encode_2d(CUtensorMap *map, CUtensorMapDataType dt, uint32_t esize, const void *ptr, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1u, 1u};
    (void)esize;
    return fn(map, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_gemm_2sm(const GemmArgs &args, cudaStream_t s) {
    static std::atomic<bool> attr_set[64];             // per device; a repeated set is harmless
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(nvfp4_gemm_2sm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true, std::memory_order_release);
    }
    const int64_t ksteps = ceil_div(args.K, KSTEP);        // scale atoms per 128-row block
    Maps maps;
    const bool ok =
        encode_2d(&maps.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, args.a_codes, args.a_pitch, args.M, args.a_pitch, 128,
                  BM_CTA, CU_TENSOR_MAP_SWIZZLE_128B) &&
        encode_2d(&maps.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, args.b_codes, args.b_pitch, args.N, args.b_pitch, 128,
                  BN_CTA, CU_TENSOR_MAP_SWIZZLE_128B) &&
        encode_2d(&maps.sfa, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, args.a_sf, ksteps * 64, ceil_div(args.M, 128),
                  ksteps * 512, 256, 1, CU_TENSOR_MAP_SWIZZLE_NONE) &&
        encode_2d(&maps.sfb, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, args.b_sf, ksteps * 64, ceil_div(args.N, 128),
                  ksteps * 512, 256, 2, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return cudaErrorInvalidValue;
    maps.y_tma = 0;
    if (args.y && !args.y_f32) {      // BF16 Y: 32 x 32 boxes, 64-byte swizzle (row stride ldy % 8 == 0)
        if (!encode_2d(&maps.y, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, args.y, args.N, args.M, args.ldy * 2, 32, 32,
                       CU_TENSOR_MAP_SWIZZLE_64B))
            return cudaErrorInvalidValue;
        maps.y_tma = 1;
    }
    maps.n_fast = args.M * args.a_pitch > args.N * args.b_pitch ? 1 : 0;
    const int64_t tiles = ceil_div(args.M, BM) * ceil_div(args.N, BN);
    int clusters = num_sms() / 2;
    if (tiles < clusters) clusters = (int)tiles;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // see griddep_wait
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, nvfp4_gemm_2sm_kernel, maps, args);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace nvfp4
