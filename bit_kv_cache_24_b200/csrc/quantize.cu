// quantize.cu -- BF16 -> NVFP4 quantizer kernels (HBM-bound): per-tensor amax, row-wise
// quantization (16-blocks along the contiguous dim) and column-wise quantization (16-blocks
// along the token dim, i.e. the row-wise quantization of the transpose).
//
// Method: LongLive-2.0 quantizes activations and weights to NVFP4 for its W4A4 linear layers
// and its NVFP4 training GEMMs (abstract, fugumt.com mirror); the numeric steps are those of
// the published NVFP4 format (see include/nvfp4.h).
//
// Design (B200): 16-byte coalesced loads, one warp covers 256 contiguous elements of a row
// (8 per lane, a 16-block per lane pair, block max by one shuffle), packed 4-byte code stores
// (a warp writes 128 contiguous bytes).  The amax pass writes one partial maximum per CTA
// (BF16 magnitude bits, so the reduction is an integer max and deterministic); every CTA of the
// quantize pass reduces the partials itself, so no atomics, memsets or grid barriers are needed.
#include "common.cuh"
#include "launch.h"

namespace nvfp4 {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kAmaxUnroll = 8;     // 16-byte loads in flight per lane in the amax pass
constexpr int kRowGroup = 4;       // 256-element segments a warp quantizes per iteration

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t warp_max(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// Block-wide reduction of the amax partials of one job; returns BF16 magnitude bits, or
// 0xFFFFFFFF when the input held inf/NaN.  Called by all threads.
__device__ uint32_t reduce_partials(const uint32_t *partial, int n, uint32_t *smem_slot) {
    if (threadIdx.x < 32) {
        uint32_t m = 0;
        for (int i = threadIdx.x; i < n; i += 32) m = max(m, partial[i]);
        m = warp_max(m);
        if (threadIdx.x == 0) *smem_slot = m;
    }
    __syncthreads();
    uint32_t m = *smem_slot;
    return m >= 0x7F80u ? 0xFFFFFFFFu : m;
}

// amax of one job -> g (and the non-finite check).  Returns false (after reporting) on inf/NaN.
__device__ bool job_scale(const RowJob &j, int npartial, int32_t *status, uint32_t *smem_slot,
                          float &g, float &den) {
    float amax;
    if (j.amax_in) {
        amax = *j.amax_in;
        if (!isfinite(amax)) {
            if (threadIdx.x == 0) set_status(status, NVFP4_ERR_NONFINITE);
            return false;
        }
    } else {
        uint32_t bits = reduce_partials(j.partial, npartial, smem_slot);
        if (bits == 0xFFFFFFFFu) {
            if (threadIdx.x == 0) set_status(status, NVFP4_ERR_NONFINITE);
            return false;
        }
        amax = __uint_as_float(bits << 16);
    }
    g = global_scale(amax);
    den = __fmul_rn(g, kE2M1Max);
    return true;
}

// ---------------------------------------------------------------------------------------------
// Pass 1: per-CTA partial max of |x| as BF16 magnitude bits (inf/NaN compare above 0x7F80).
__global__ void __launch_bounds__(kThreads) amax_partial_kernel(const __grid_constant__ RowJobs jobs) {
    const RowJob &j = jobs.job[blockIdx.y];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t cpr = j.cols >> 3;                      // 8-element chunks per row
    uint32_t m = 0;
    for (int64_t row = (int64_t)blockIdx.x * kWarps + warp; row < j.rows; row += (int64_t)gridDim.x * kWarps) {
        const uint16_t *xr = j.x + row * j.ld;
        int64_t c = lane;
        for (; c + 32 * (kAmaxUnroll - 1) < cpr; c += 32 * kAmaxUnroll) {   // kAmaxUnroll loads in flight
            uint4 v[kAmaxUnroll];
#pragma unroll
            for (int u = 0; u < kAmaxUnroll; ++u) v[u] = ldg_nc_v4(xr + 8 * (c + 32 * u));
#pragma unroll
            for (int u = 0; u < kAmaxUnroll; ++u) {
                const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                m = max(m, absmax_bits8(w));
            }
        }
        for (; c < cpr; c += 32) {
            uint4 v = ldg_nc_v4(xr + 8 * c);
            uint32_t w[4] = {v.x, v.y, v.z, v.w};
            m = max(m, absmax_bits8(w));
        }
    }
    __shared__ uint32_t red[kWarps];
    m = warp_max(m);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t r = 0;
        for (int w = 0; w < kWarps; ++w) r = max(r, red[w]);
        j.partial[blockIdx.x] = r;
    }
}

// Final step of nvfp4_amax: partials -> amax float (one CTA).
__global__ void amax_finish_kernel(const uint32_t *partial, int n, float *amax_out, int32_t *status) {
    __shared__ uint32_t slot;
    uint32_t bits = reduce_partials(partial, n, &slot);
    if (threadIdx.x == 0) {
        if (bits == 0xFFFFFFFFu) {
            set_status(status, NVFP4_ERR_NONFINITE);
            *amax_out = __uint_as_float(0x7FC00000u);
        } else {
            *amax_out = __uint_as_float(bits << 16);
        }
    }
}

// ---------------------------------------------------------------------------------------------
// Pass 2, row-wise.  Work item = (row, 256-element segment); rows are extended to a multiple of
// 128 for the tensor-core scale layout so that its padding rows get zero scales.  Loads outside
// the matrix read as zero, which quantizes to zero codes and zero scales: that writes every
// padding byte of codes (to a multiple of 32 elements) and scales (to a multiple of 64).
__global__ void __launch_bounds__(kThreads) quantize_rows_kernel(const __grid_constant__ RowJobs jobs, int32_t *status) {
    const RowJob j = jobs.job[blockIdx.y];
    __shared__ uint32_t slot;
    float g, den;
    if (!job_scale(j, jobs.npartial, status, &slot, g, den)) return;
    if (blockIdx.x == 0 && threadIdx.x == 0) *j.g_out = g;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool mma = j.sf_layout != 0;
    const int64_t nb = ceil_div(j.cols, 16);
    const int64_t nb_pad = mma ? 4 * ceil_div(nb, 4) : nb;
    const int64_t atoms = ceil_div(nb, 4);
    const int64_t code_cols = 32 * ceil_div(j.cols, 32);
    const int64_t rows_total = mma ? 128 * ceil_div(j.rows, 128) : j.rows;
    const int64_t nseg = ceil_div(mma ? 16 * nb_pad : code_cols, 256);
    const int64_t ngrp = ceil_div(nseg, kRowGroup);
    const int64_t items = rows_total * ngrp;

    for (int64_t it = (int64_t)blockIdx.x * kWarps + warp; it < items; it += (int64_t)gridDim.x * kWarps) {
        const int64_t row = it / ngrp;
        const int64_t e0 = (it - row * ngrp) * (256 * kRowGroup) + lane * 8;
        uint4 v[kRowGroup];
#pragma unroll
        for (int u = 0; u < kRowGroup; ++u) {           // all loads of the group first
            const int64_t e = e0 + 256 * u;
            v[u] = make_uint4(0, 0, 0, 0);
            if (row < j.rows && e < j.cols) v[u] = ldg_nc_v4(j.x + row * j.ld + e);
        }
#pragma unroll
        for (int u = 0; u < kRowGroup; ++u) {
            const int64_t e = e0 + 256 * u;
            if (e >= nseg * 256) break;                 // past the last segment (warp-uniform)
            const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            uint32_t bm = absmax_bits8(w);
            bm = max(bm, __shfl_xor_sync(0xFFFFFFFFu, bm, 1));
            const BlockScale sc = block_scale(__uint_as_float(bm << 16), g, den);
            const uint32_t codes = (sc.r == 0.0f) ? 0u : encode8(w, sc);
            if (row < j.rows && e < code_cols)
                *reinterpret_cast<uint32_t *>(j.codes + row * j.pitch + (e >> 1)) = codes;
            if ((lane & 1) == 0) {
                const int64_t blk = e >> 4;
                if (!mma) {
                    if (row < j.rows && blk < nb) j.sf[row * nb + blk] = (uint8_t)sc.sf;
                } else if (blk < nb_pad) {
                    j.sf[sf_mma_offset(row, blk, atoms)] = (uint8_t)sc.sf;
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------------------------
// Pass 2, column-wise: 16-blocks along the rows (m) of x [M][K]; output row k holds x[:, k].
// A CTA stages a 256 (m) x 32 (k) BF16 tile in shared memory (16 KB), words XOR-swizzled by the
// 16-row group so that the 16 threads reading one k down 16 different m-blocks hit 16 banks.
// Thread (k, m-block) then quantizes 16 values; lanes 0-15 of a warp share k, so a warp writes
// 128 contiguous code bytes per output row.
constexpr int kColTileM = 256, kColTileK = 32;

__global__ void __launch_bounds__(kThreads) quantize_cols_kernel(RowJob j, int32_t npartial, int32_t *status) {
    __shared__ uint32_t tile[kColTileM * (kColTileK / 2)];
    __shared__ uint32_t slot;
    float g, den;
    if (!job_scale(j, npartial, status, &slot, g, den)) return;
    if (blockIdx.x == 0 && threadIdx.x == 0) *j.g_out = g;

    const bool mma = j.sf_layout != 0;
    const int64_t M = j.rows, K = j.cols;                 // x is [M][K]; output is [K][M]
    const int64_t nb = ceil_div(M, 16);                   // scale columns of the output
    const int64_t nb_pad = mma ? 4 * ceil_div(nb, 4) : nb;
    const int64_t atoms = ceil_div(nb, 4);
    const int64_t code_cols = 32 * ceil_div(M, 32);
    const int64_t m_extent = mma ? 16 * nb_pad : code_cols;
    const int64_t k_extent = mma ? 128 * ceil_div(K, 128) : K;
    const int64_t tiles_m = ceil_div(m_extent, kColTileM), tiles_k = ceil_div(k_extent, kColTileK);
    const int t = threadIdx.x;

    for (int64_t tile_id = blockIdx.x; tile_id < tiles_m * tiles_k; tile_id += gridDim.x) {
        const int64_t m0 = (tile_id % tiles_m) * kColTileM, k0 = (tile_id / tiles_m) * kColTileK;
        __syncthreads();                                  // previous tile fully consumed
        // load: thread t covers rows t/4 + 64*i, 8-element chunk t%4 of the 32 k
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = (t >> 2) + 64 * i, c = t & 3;
            const int64_t m = m0 + r, k = k0 + 8 * c;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (m < M && k < K) v = ldg_nc_v4(j.x + m * j.ld + k);
            const int swz = (r >> 4) & 15;
            uint32_t *row = tile + r * (kColTileK / 2);
            row[(4 * c + 0) ^ swz] = v.x;
            row[(4 * c + 1) ^ swz] = v.y;
            row[(4 * c + 2) ^ swz] = v.z;
            row[(4 * c + 3) ^ swz] = v.w;
        }
        __syncthreads();
#pragma unroll
        for (int p2 = 0; p2 < 2; ++p2) {
            const int p = t + kThreads * p2;
            const int kl = p >> 4, mb = p & 15;           // local k row, local 16-block
            const int shift = (kl & 1) * 16;
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r0 = mb * 16 + 2 * i, r1 = r0 + 1;
                const uint32_t a = tile[r0 * (kColTileK / 2) + ((kl >> 1) ^ mb)] >> shift;
                const uint32_t b = tile[r1 * (kColTileK / 2) + ((kl >> 1) ^ mb)] >> shift;
                w[i] = (a & 0xFFFFu) | (b << 16);
            }
            const uint32_t bm = max(absmax_bits8(w), absmax_bits8(w + 4));
            const BlockScale s = block_scale(__uint_as_float(bm << 16), g, den);
            uint2 codes = make_uint2(0, 0);
            if (s.r != 0.0f) {
                codes.x = encode8(w, s);
                codes.y = encode8(w + 4, s);
            }
            const int64_t k = k0 + kl, m = m0 + 16 * mb, blk = m >> 4;
            if (k < K && m < code_cols)
                *reinterpret_cast<uint2 *>(j.codes + k * j.pitch + (m >> 1)) = codes;
            if (!mma) {
                if (k < K && blk < nb) j.sf[k * nb + blk] = (uint8_t)s.sf;
            } else if (k < k_extent && blk < nb_pad) {
                j.sf[sf_mma_offset(k, blk, atoms)] = (uint8_t)s.sf;
            }
        }
    }
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

}  // namespace

int amax_blocks(int64_t rows) {
    int64_t b = ceil_div(rows, kWarps);
    const int64_t cap = 6 * (int64_t)num_sms();          // 6 x 256 threads per SM
    if (b > cap) b = cap;
    if (b > kMaxPartials) b = kMaxPartials;
    return (int)(b < 1 ? 1 : b);
}

cudaError_t launch_amax(const RowJobs &jobs, int32_t *status, float *amax_out, cudaStream_t s) {
    dim3 grid(jobs.npartial, jobs.njobs);
    amax_partial_kernel<<<grid, kThreads, 0, s>>>(jobs);
    if (amax_out) amax_finish_kernel<<<1, 32, 0, s>>>(jobs.job[0].partial, jobs.npartial, amax_out, status);
    return cudaGetLastError();
}

cudaError_t launch_quantize_rows(const RowJobs &jobs, int32_t *status, cudaStream_t s) {
    int64_t items = 0;
    for (int i = 0; i < jobs.njobs; ++i) {
        const RowJob &j = jobs.job[i];
        const int64_t rows = j.sf_layout ? 128 * ceil_div(j.rows, 128) : j.rows;
        const int64_t it = rows * ceil_div(ceil_div(64 * ceil_div(j.cols, 64), 256), kRowGroup);
        if (it > items) items = it;
    }
    int64_t blocks = ceil_div(items, kWarps);
    const int64_t cap = 8 * (int64_t)num_sms();            // 8 x 256 threads fill an SM
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    quantize_rows_kernel<<<dim3((unsigned)blocks, jobs.njobs), kThreads, 0, s>>>(jobs, status);
    return cudaGetLastError();
}

cudaError_t launch_quantize_cols(const RowJob &j, int32_t npartial, int32_t *status, cudaStream_t s) {
    const int64_t nb = ceil_div(j.rows, 16);
    const int64_t m_extent = j.sf_layout ? 64 * ceil_div(nb, 4) : 32 * ceil_div(j.rows, 32);
    const int64_t k_extent = j.sf_layout ? 128 * ceil_div(j.cols, 128) : j.cols;
    int64_t tiles = ceil_div(m_extent, kColTileM) * ceil_div(k_extent, kColTileK);
    const int64_t cap = 6 * (int64_t)num_sms();
    if (tiles > cap) tiles = cap;
    quantize_cols_kernel<<<(unsigned)tiles, kThreads, 0, s>>>(j, npartial, status);
    return cudaGetLastError();
}

cudaError_t launch_encode_elements(const float *in, int64_t n, uint8_t *e2m1_out, uint8_t *e4m3_out, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    encode_elements_kernel<<<(unsigned)ceil_div(n, 256), 256, 0, s>>>(in, n, e2m1_out, e4m3_out);
    return cudaGetLastError();
}

cudaError_t launch_wait_timeout(int32_t *status, int64_t limit_ns, cudaStream_t s) {
    wait_timeout_kernel<<<1, 32, 0, s>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace nvfp4
