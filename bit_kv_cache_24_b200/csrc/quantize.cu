// quantize.cu -- BF16 -> NVFP4 quantizer kernels (HBM-bound): per-tensor amax, the per-tensor
// scale record, row-wise quantization (16-blocks along the contiguous dim) and column-wise
// quantization (16-blocks along the token dim, i.e. the row-wise quantization of the transpose).
//
// Method: LongLive-2.0 quantizes activations and weights to NVFP4 for its W4A4 linear layers
// and its NVFP4 training GEMMs (abstract, fugumt.com mirror); the numeric steps are those of
// the published NVFP4 format (see include/nvfp4.h).
//
// Design (B200).  One quantization is three launches (four for both layouts) chained with
// programmatic dependent launch (each kernel waits for its predecessor before touching global
// memory, so the next kernel's launch and prologue overlap the previous one's tail; the column
// pass after a row pass runs concurrently with it, see quantize_cols_kernel):
//   1. amax pass: 32-byte loads, 128 bytes in flight per thread; one partial maximum per CTA as
//      BF16 magnitude bits (an integer max: deterministic, no atomics, no memset).
//   2. scale record (one CTA per tensor): reduces the partials and writes g, den = 6g, RN(1/den)
//      and the table r_tab[sf] = 1/(e4m3(sf) * g) of the 128 possible scale bytes.  Doing this
//      once instead of in every CTA of the quantize pass took ~3 us and ~17% of the
//      instructions off a 4680 x 3072 quantization.
//   3. quantize pass: the quantizers are issue-bound (~100 instructions per 16-block before this
//      design), so the block step is written for instruction count: a paired BF16 abs-max tree,
//      the scale quotient b/den by one correction step on b * RN(1/den) (exact, see
//      block_scale), 1/d from the record's table, paired FP32 multiplies and the hardware E2M1
//      conversion.
// Row-wise, a thread owns four consecutive 16-blocks of one row (four 32-byte loads), stores
// its 32 code bytes as two 16-byte stores and its four scales as one 32-bit word (adjacent in
// the tensor-core layout).  Measured alternatives that were slower on 4680 x 3072 .. 37440 x
// 3072: a persistent kernel with a per-thread cp.async ring, a warp-specialized kernel fed by
// bulk (TMA) copies (16 consumer warps per SM are too few to hide the block step's dependent
// chains), one 16-block per thread, 128-thread CTAs, and a single cooperative launch with a
// grid-wide amax.
#include "common.cuh"
#include "launch.h"

namespace nvfp4 {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kAmaxBytes = 128;    // bytes in flight per thread in the amax pass

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// 16 or 32 bytes (8 or 16 BF16) of one row.
template <int kWords>
struct Unit {
    uint32_t w[kWords];
};

template <int kWords>
__device__ __forceinline__ Unit<kWords> ldg_unit(const uint16_t *p) {
    Unit<kWords> u;
    if constexpr (kWords == 8) {
        asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=r"(u.w[0]), "=r"(u.w[1]), "=r"(u.w[2]), "=r"(u.w[3]),
                       "=r"(u.w[4]), "=r"(u.w[5]), "=r"(u.w[6]), "=r"(u.w[7]) : "l"(p));
    } else {
        const uint4 v = ldg_nc_v4(p);
        u.w[0] = v.x; u.w[1] = v.y; u.w[2] = v.z; u.w[3] = v.w;
    }
    return u;
}

__device__ __forceinline__ void stg_v4(void *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" :: "l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ uint32_t warp_max(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// Block-wide max of n <= kMaxPartials partials (BF16 magnitude bits).  Called by all kThreads
// threads; red: kWarps words of shared memory.
__device__ uint32_t reduce_partials(const uint32_t *partial, int n, uint32_t *red) {
    constexpr int kPer = kMaxPartials / kThreads;
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int k = threadIdx.x + i * kThreads;
        m = max(m, k < n ? partial[k] : 0u);
    }
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    m = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) m = max(m, red[w]);
    return m;
}
static_assert(kMaxPartials % kThreads == 0, "partials split evenly over the threads");

__device__ __forceinline__ uint32_t ldg_cg_u32(const void *p) {
    uint32_t v;
    asm volatile("ld.global.cg.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ldg_cg_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Copy the record to shared memory (after griddep_wait, or through L2 with kL2 set); a barrier
// must follow.
template <bool kL2 = false>
__device__ __forceinline__ void load_record(const ScaleRecord *rec, SmemRecord &s) {
    if (threadIdx.x < 128)
        s.r_tab[threadIdx.x] = kL2 ? __uint_as_float(ldg_cg_u32(rec->r_tab + threadIdx.x)) : rec->r_tab[threadIdx.x];
    if (threadIdx.x == 128) {
        s.den = kL2 ? __uint_as_float(ldg_cg_u32(&rec->den)) : rec->den;
        s.inv_den = kL2 ? __uint_as_float(ldg_cg_u32(&rec->inv_den)) : rec->inv_den;
        s.ok = kL2 ? ldg_cg_u32(&rec->ok) : rec->ok;
    }
}

// ---------------------------------------------------------------------------------------------
// Pass 1: per-CTA partial max of |x| as BF16 magnitude bits (inf/NaN compare above 0x7F80).
// A unit index maps to (row, unit in row) by one 32-bit division unless the rows are contiguous.
template <int kWords>
__global__ void __launch_bounds__(kThreads) amax_partial_kernel(const __grid_constant__ RowJobs jobs) {
    griddep_wait();
    griddep_launch_dependents();
    const RowJob &j = jobs.job[blockIdx.y];
    constexpr int kElems = 2 * kWords;
    constexpr int kUnroll = kAmaxBytes / (4 * kWords);
    const uint32_t upr = (uint32_t)(j.cols / kElems);    // units per row (cols % kElems == 0)
    const uint32_t total = (uint32_t)j.rows * upr;         // < 2^31 (checked by the host)
    const bool flat = j.ld == j.cols;
    const uint32_t stride = gridDim.x * kThreads;
    uint32_t m = 0;
    for (uint32_t u0 = blockIdx.x * kThreads + threadIdx.x; u0 < total; u0 += stride * kUnroll) {
        Unit<kWords> v[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const uint32_t u = u0 + (uint32_t)k * stride;
            if (u < total) {
                const uint32_t row = flat ? 0u : u / upr;
                const int64_t off = flat ? (int64_t)u * kElems : (int64_t)row * j.ld + (int64_t)(u - row * upr) * kElems;
                if (NVFP4_CHECKED(off, kElems, j.x_elems, j.status)) {
                    v[k] = ldg_unit<kWords>(j.x + off);
                } else {
#pragma unroll
                    for (int i = 0; i < kWords; ++i) v[k].w[i] = 0;
                }
            } else {
#pragma unroll
                for (int i = 0; i < kWords; ++i) v[k].w[i] = 0;
            }
        }
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
#pragma unroll
            for (int i = 0; i < kWords; i += 4) m = max(m, absmax_bits8(v[k].w + i));
        }
    }
    __shared__ uint32_t red[kWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    m = warp_max(m);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t r = 0;
        for (int w = 0; w < kWarps; ++w) r = max(r, red[w]);
        if (NVFP4_CHECKED(blockIdx.x, 1, kMaxPartials, j.status)) j.partial[blockIdx.x] = r;
    }
}

// nvfp4_amax's final step: partials -> amax float (one CTA).
__global__ void __launch_bounds__(kThreads) amax_finish_kernel(const uint32_t *partial, int n, float *amax_out, int32_t *status) {
    griddep_wait();
    griddep_launch_dependents();
    __shared__ uint32_t red[kWarps];
    const uint32_t bits = reduce_partials(partial, n, red);
    if (threadIdx.x == 0) {
        if (bits >= 0x7F80u) {
            set_status(status, NVFP4_ERR_NONFINITE);
            *amax_out = __uint_as_float(0x7FC00000u);
        } else {
            *amax_out = __uint_as_float(bits << 16);
        }
    }
}

// Column-group amax of a GEMM output from its per-block partials (nvfp4_gemm_colamax): CTA g
// reduces the blocks of columns [g * group_cols, (g + 1) * group_cols); inf/NaN reports
// NVFP4_ERR_NONFINITE and stores NaN.
__global__ void __launch_bounds__(kThreads) colamax_finish_kernel(const uint32_t *partial, int64_t rows32, int64_t n128,
                                                                  int64_t group_cols, float *amax_out, int32_t *status) {
    griddep_wait();
    griddep_launch_dependents();
    __shared__ uint32_t red[kWarps];
    // the group's rows32 x cpg partials as one flat range: each thread issues all of its loads
    // (16 in flight) before using any (the partials are few: latency, not bandwidth, sets this
    // kernel's time, and every lane of every warp takes part)
    constexpr int kInFlight = 16;
    const int64_t cpg = group_cols >> 7;
    const uint32_t total = (uint32_t)(rows32 * cpg);        // < 2^31 (checked by the host)
    const uint32_t ucpg = (uint32_t)cpg;
    uint32_t m = 0;
    for (uint32_t f0 = threadIdx.x; f0 < total; f0 += (uint32_t)kThreads * kInFlight) {
        uint32_t v[kInFlight];
#pragma unroll
        for (int u = 0; u < kInFlight; ++u) {
            const uint32_t f = f0 + (uint32_t)u * kThreads;
            const uint32_t r = f / ucpg, c = f - r * ucpg;
            const int64_t idx = (int64_t)r * n128 + (int64_t)blockIdx.x * cpg + c;
            v[u] = f < total && NVFP4_CHECKED(idx, 1, rows32 * n128, status) ? partial[idx] : 0u;
        }
#pragma unroll
        for (int u = 0; u < kInFlight; ++u) m = max(m, v[u]);
    }
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = 0;
        for (int w = 0; w < kWarps; ++w) b = max(b, red[w]);
        if (b >= 0x7F80u) {
            set_status(status, NVFP4_ERR_NONFINITE);
            amax_out[blockIdx.x] = __uint_as_float(0x7FC00000u);
        } else {
            amax_out[blockIdx.x] = __uint_as_float(b << 16);
        }
    }
}

// Pass 2: the scale record of each tensor (one CTA per job) from its partials or its amax_in.
__global__ void __launch_bounds__(kThreads) scale_record_kernel(const __grid_constant__ RecJobs jobs, int32_t *status) {
    griddep_wait();
    griddep_launch_dependents();
    const RecJob &j = jobs.job[blockIdx.x];
    __shared__ uint32_t red[kWarps];
    float amax;
    bool finite;
    if (j.amax_in) {
        amax = *j.amax_in;
        finite = isfinite(amax);
    } else {
        const uint32_t bits = reduce_partials(j.partial, jobs.npartial, red);
        finite = bits < 0x7F80u;
        amax = __uint_as_float(bits << 16);
    }
    ScaleRecord *rec = j.rec;
    if (!finite) {
        if (threadIdx.x == 0) {
            rec->ok = 0;
            set_status(status, NVFP4_ERR_NONFINITE);
        }
        return;
    }
    const float g = global_scale(amax);
    const float den = record_den(g);
    if (threadIdx.x < 128) rec->r_tab[threadIdx.x] = record_r_entry(threadIdx.x, g);
    if (threadIdx.x == 128) {
        rec->g = g;
        rec->den = den;
        rec->inv_den = record_inv_den(den);
        rec->ok = 1;
        if (j.g_out[0]) *j.g_out[0] = g;
        if (j.g_out[1]) *j.g_out[1] = g;
    }
}

// ---------------------------------------------------------------------------------------------
// Pass 3, row-wise (cols % 16 == 0).  A thread owns quad (row, q): 16-blocks 4q..4q+3 of a row,
// 64 elements.  Rows run to a multiple of 128 in the tensor-core scale layout, whose padding rows
// get zero scales (no loads, no codes); blocks past the row's end quantize to zero codes and
// scales, which writes the code padding (to a multiple of 32 elements) and the scale padding
// (to a multiple of 64) of the tensor-core layout.
template <bool kV8, bool kMma>
__global__ void __launch_bounds__(kThreads) quantize_rows_kernel(const __grid_constant__ RowJobs jobs) {
    const RowJob &j = jobs.job[blockIdx.y];
    const bool early = j.x_early != 0;                     // x complete before the amax pass read it
    if (!early) {
        griddep_wait();
        griddep_launch_dependents();
    }
    __shared__ SmemRecord rec;
    const uint32_t rows = (uint32_t)j.rows;
    const uint32_t nb = (uint32_t)(j.cols >> 4);            // 16-blocks per row
    const uint32_t nq = (nb + 3) >> 2;                      // quads per row
    const uint32_t rows_total = kMma ? 128u * ((rows + 127u) >> 7) : rows;
    const uint32_t idx = blockIdx.x * kThreads + threadIdx.x;
    const bool active = idx < rows_total * nq;              // < 2^31 (checked by the host)
    const uint32_t row = active ? idx / nq : 0u;
    const uint32_t q = idx - row * nq;
    const bool live = active && row < rows;                 // a row of x (not scale padding)

    uint32_t w[4][8];
    const uint16_t *xr = j.x + (int64_t)row * j.ld + 64 * q;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        if (live && 4 * q + b < nb &&
            NVFP4_CHECKED((int64_t)row * j.ld + 64 * q + 16 * b, 16, j.x_elems, j.status)) {
            if constexpr (kV8) {
                const Unit<8> u = ldg_unit<8>(xr + 16 * b);
#pragma unroll
                for (int i = 0; i < 8; ++i) w[b][i] = u.w[i];
            } else {
                const uint4 u0 = ldg_nc_v4(xr + 16 * b), u1 = ldg_nc_v4(xr + 16 * b + 8);
                w[b][0] = u0.x; w[b][1] = u0.y; w[b][2] = u0.z; w[b][3] = u0.w;
                w[b][4] = u1.x; w[b][5] = u1.y; w[b][6] = u1.z; w[b][7] = u1.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) w[b][i] = 0;
        }
    }
    if (early) {                                          // the record kernel's output from here on
        griddep_wait();
        griddep_launch_dependents();
    }
    if (j.amax_in)
        build_record(*j.amax_in, rec, j.report_record && blockIdx.x == 0, j.g_out[0], j.g_out[1], j.status);
    else
        load_record(j.rec, rec);
    __syncthreads();
    if (!active || !rec.ok) return;

    uint32_t c[8], sfw = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        uint32_t sf;
        quantize16(w[b], rec, c[2 * b], c[2 * b + 1], sf);
        sfw |= sf << (8 * b);
    }
    if (live) {
        const int64_t co = (int64_t)row * j.pitch + 32 * q;
        uint8_t *cr = j.codes + co;
        if (32 * q < j.pitch && NVFP4_CHECKED(co, 16, j.codes_bytes, j.status)) stg_v4(cr, c[0], c[1], c[2], c[3]);
        if (32 * q + 16 < j.pitch && NVFP4_CHECKED(co + 16, 16, j.codes_bytes, j.status))
            stg_v4(cr + 16, c[4], c[5], c[6], c[7]);
    }
    if constexpr (kMma) {
        const int64_t so = sf_mma_offset(row, 4 * q, nq);
        if (NVFP4_CHECKED(so, 4, j.sf_bytes, j.status)) *reinterpret_cast<uint32_t *>(j.sf + so) = sfw;
    } else if (live) {
        const int64_t so = (int64_t)row * nb + 4 * q;
        uint8_t *sr = j.sf + so;
        if (4 * q + 3 < nb && ((reinterpret_cast<uintptr_t>(sr) & 3) == 0)) {
            if (NVFP4_CHECKED(so, 4, j.sf_bytes, j.status)) *reinterpret_cast<uint32_t *>(sr) = sfw;
        } else {
#pragma unroll
            for (int b = 0; b < 4; ++b)
                if (4 * q + b < nb && NVFP4_CHECKED(so + b, 1, j.sf_bytes, j.status)) sr[b] = (uint8_t)(sfw >> (8 * b));
        }
    }
}

// ---------------------------------------------------------------------------------------------
// Pass 3, column-wise: 16-blocks along the rows (m) of x [M][K]; output row k holds x[:, k].
// Transpose in registers: a thread loads a 16 (m) x 8 (k) patch (sixteen 16-byte row pieces, all
// in flight at once) and emits the eight 16-blocks of its eight columns.  Lanes 0-7 of a warp
// take adjacent 8-column chunks (a full 128-byte line of each row) and lane groups 0-3 adjacent
// 16-row blocks, so a warp covers 64 x 64 and each 8-byte code store instruction writes eight
// output rows x 32 contiguous bytes.  Output rows run to a multiple of 128 and scale columns to
// a multiple of 4 in the tensor-core layout (zero scales); code columns run to a multiple of 32.
//
// kConcurrent: launched right after the row pass of the same call (both layouts), whose inputs
// it shares.  It then starts while the row pass runs: x and the scale record were complete
// before the row pass could start (the row pass triggers its dependents only after its own
// wait, which follows the record kernel), so the kernel reads them at once, through L2, and
// waits for its predecessor only at exit -- every thread, so that this grid cannot complete
// before the row pass and whatever waits on this grid also sees the row-wise outputs.
template <bool kConcurrent>
__device__ __forceinline__ void cols_body(const RowJob &j, SmemRecord &rec) {
    const bool mma = j.sf_layout != 0;
    const uint32_t M = (uint32_t)j.rows, K = (uint32_t)j.cols;   // x is [M][K]; output is [K][M]
    const uint32_t nb = (M + 15) >> 4;                      // scale columns of the output
    const uint32_t nb_pad = mma ? 4 * ((nb + 3) >> 2) : nb;
    const uint32_t atoms = (nb + 3) >> 2;
    const uint32_t code_cols = 32 * ((M + 31) >> 5);
    const uint32_t mb_total = (mma ? 16 * nb_pad : code_cols) >> 4;   // 16-row blocks to cover
    const uint32_t k_extent = mma ? 128 * ((K + 127) >> 7) : K;
    const uint32_t kc_total = k_extent >> 3;                // 8-column chunks (K % 8 == 0)
    const uint32_t tiles_k = (kc_total + 7) >> 3, tiles_m = (mb_total + 3) >> 2;
    const uint32_t lane = threadIdx.x & 31;
    const uint32_t wt = blockIdx.x * kWarps + (threadIdx.x >> 5);      // warp tile, k fastest
    const bool active = wt < tiles_k * tiles_m;
    const uint32_t tk = active ? wt % tiles_k : 0u, tm = active ? wt / tiles_k : 0u;
    const uint32_t kc = 8 * tk + (lane & 7), mb = 4 * tm + (lane >> 3);
    const uint32_t k0 = 8 * kc, m0 = 16 * mb;

    uint32_t w[16][4];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const uint32_t m = m0 + r;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (active && m < M && k0 < K && NVFP4_CHECKED((int64_t)m * j.ld + k0, 8, j.x_elems, j.status)) {
            const uint16_t *p = j.x + (int64_t)m * j.ld + k0;
            v = kConcurrent ? ldg_cg_v4(p) : ldg_nc_v4(p);
        }
        w[r][0] = v.x; w[r][1] = v.y; w[r][2] = v.z; w[r][3] = v.w;
    }
    if (j.amax_in)   // concurrent: complete before the row pass started, read through L2
        build_record(kConcurrent ? __uint_as_float(ldg_cg_u32(j.amax_in)) : *j.amax_in, rec,
                     j.report_record && blockIdx.x == 0, j.g_out[0], j.g_out[1], j.status);
    else
        load_record<kConcurrent>(j.rec, rec);
    __syncthreads();
    if (!active || !rec.ok || kc >= kc_total || mb >= mb_total) return;

#pragma unroll
    for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t k = k0 + 2 * c + h;
            uint32_t b[8];                                   // column k, rows m0..m0+15 as BF16 pairs
#pragma unroll
            for (int i = 0; i < 8; ++i) b[i] = __byte_perm(w[2 * i][c], w[2 * i + 1][c], h ? 0x7632 : 0x5410);
            uint32_t c0, c1, sf;
            quantize16(b, rec, c0, c1, sf);
            if (k < K) {
                const int64_t co = (int64_t)k * j.pitch + (m0 >> 1);
                if (m0 < code_cols && NVFP4_CHECKED(co, 8, j.codes_bytes, j.status))
                    *reinterpret_cast<uint2 *>(j.codes + co) = make_uint2(c0, c1);
                if (!mma && mb < nb && NVFP4_CHECKED((int64_t)k * nb + mb, 1, j.sf_bytes, j.status))
                    j.sf[(int64_t)k * nb + mb] = (uint8_t)sf;
            }
            if (mma && NVFP4_CHECKED(sf_mma_offset(k, mb, atoms), 1, j.sf_bytes, j.status))
                j.sf[sf_mma_offset(k, mb, atoms)] = (uint8_t)sf;
        }
    }
}

template <bool kConcurrent>
__global__ void __launch_bounds__(kThreads) quantize_cols_kernel(const __grid_constant__ RowJob j) {
    __shared__ SmemRecord rec;
    if constexpr (!kConcurrent) griddep_wait();
    griddep_launch_dependents();
    cols_body<kConcurrent>(j, rec);
    if constexpr (kConcurrent) griddep_wait();
}

// ---------------------------------------------------------------------------------------------
// Test support: the hardware encoders exactly as the quantizer applies them.
__global__ void encode_elements_kernel(const float *in, int64_t n, uint8_t *e2m1_out, uint8_t *e4m3_out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float v = in[i];
    if (e2m1_out) {
        float q[8] = {v, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        e2m1_out[i] = (uint8_t)(e2m1x8(q) & 0xFu);
    }
    if (e4m3_out) e4m3_out[i] = (uint8_t)e4m3(fabsf(v));
}

// Test support: a bounded wait on an mbarrier that nothing completes.
__global__ void wait_timeout_kernel(int32_t *status, int64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t a = smem_addr(&bar);
    if (threadIdx.x == 0) {
        mbar_init(a, 1);
        fence_mbarrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (!mbar_wait_bounded(a, 0, nullptr, (uint64_t)limit_ns)) set_status(status, NVFP4_ERR_TIMEOUT);
    }
}

// Test support: one guarded byte write (see nvfp4_selftest_bounds).
__global__ void bounds_selftest_kernel(uint8_t *buf, int64_t extent, int64_t index, int32_t *status) {
    (void)extent;
    (void)status;
    if (NVFP4_CHECKED(index, 1, extent, status)) buf[index] = 0xAB;
}

bool all_v8(const RowJobs &jobs) {
    for (int i = 0; i < jobs.njobs; ++i) {
        const RowJob &j = jobs.job[i];
        if ((reinterpret_cast<uintptr_t>(j.x) & 31) || (j.ld & 15) || (j.cols & 15)) return false;
    }
    return true;
}

}  // namespace

int amax_blocks(int64_t rows) {
    (void)rows;
    return 4 * num_sms() < kMaxPartials ? 4 * num_sms() : kMaxPartials;   // 4 x 256 threads per SM
}

cudaError_t launch_amax(const RowJobs &jobs, int32_t *status, float *amax_out, cudaStream_t s) {
    const dim3 grid(jobs.npartial, jobs.njobs);
    cudaError_t e = all_v8(jobs) ? launch_pdl(amax_partial_kernel<8>, grid, dim3(kThreads), 0, s, jobs)
                                 : launch_pdl(amax_partial_kernel<4>, grid, dim3(kThreads), 0, s, jobs);
    if (e == cudaSuccess && amax_out)
        e = launch_pdl(amax_finish_kernel, dim3(1), dim3(kThreads), 0, s,
                       (const uint32_t *)jobs.job[0].partial, (int)jobs.npartial, amax_out, status);
    return e;
}

cudaError_t launch_colamax_finish(const uint32_t *partial, int64_t rows32, int64_t n128, int64_t group_cols,
                                  int64_t groups, float *amax_out, int32_t *status, cudaStream_t s) {
    return launch_pdl(colamax_finish_kernel, dim3((unsigned)groups), dim3(kThreads), 0, s, partial, rows32, n128,
                      group_cols, amax_out, status);
}

cudaError_t launch_scale_record(const RecJobs &jobs, int32_t *status, cudaStream_t s) {
    return launch_pdl(scale_record_kernel, dim3(jobs.njobs), dim3(kThreads), 0, s, jobs, status);
}

cudaError_t launch_quantize_rows(const RowJobs &jobs, cudaStream_t s) {
    int64_t quads = 0;
    for (int i = 0; i < jobs.njobs; ++i) {
        const RowJob &j = jobs.job[i];
        const int64_t rows = j.sf_layout ? 128 * ceil_div(j.rows, 128) : j.rows;
        const int64_t n = rows * ceil_div(j.cols / 16, 4);
        if (n > quads) quads = n;
    }
    const dim3 grid((unsigned)ceil_div(quads, kThreads), jobs.njobs), block(kThreads);
    const bool v8 = all_v8(jobs), mma = jobs.job[0].sf_layout != 0;   // jobs of one launch share the layout
    if (v8 && mma) return launch_pdl(quantize_rows_kernel<true, true>, grid, block, 0, s, jobs);
    if (v8) return launch_pdl(quantize_rows_kernel<true, false>, grid, block, 0, s, jobs);
    if (mma) return launch_pdl(quantize_rows_kernel<false, true>, grid, block, 0, s, jobs);
    return launch_pdl(quantize_rows_kernel<false, false>, grid, block, 0, s, jobs);
}

cudaError_t launch_quantize_cols(const RowJob &j, bool after_rows, cudaStream_t s) {
    const int64_t nb = ceil_div(j.rows, 16);
    const int64_t m_extent = j.sf_layout ? 64 * ceil_div(nb, 4) : 32 * ceil_div(j.rows, 32);
    const int64_t k_extent = j.sf_layout ? 128 * ceil_div(j.cols, 128) : j.cols;
    const int64_t warp_tiles = ceil_div(k_extent / 8, 8) * ceil_div(m_extent / 16, 4);
    const dim3 grid((unsigned)ceil_div(warp_tiles, kWarps)), block(kThreads);
    return after_rows ? launch_pdl(quantize_cols_kernel<true>, grid, block, 0, s, j)
                      : launch_pdl(quantize_cols_kernel<false>, grid, block, 0, s, j);
}

cudaError_t launch_encode_elements(const float *in, int64_t n, uint8_t *e2m1_out, uint8_t *e4m3_out, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    encode_elements_kernel<<<(unsigned)ceil_div(n, 256), 256, 0, s>>>(in, n, e2m1_out, e4m3_out);
    return cudaGetLastError();
}

cudaError_t launch_bounds_selftest(uint8_t *buf, int64_t extent, int64_t index, int32_t *status, cudaStream_t s) {
    bounds_selftest_kernel<<<1, 1, 0, s>>>(buf, extent, index, status);
    return cudaGetLastError();
}

cudaError_t launch_wait_timeout(int32_t *status, int64_t limit_ns, cudaStream_t s) {
    wait_timeout_kernel<<<1, 32, 0, s>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace nvfp4
