// attention.cu -- softmax attention of BF16 queries over a window of NVFP4 KV-cache slots, with
// the restore fused into the K/V tile loads.
//
// LongLive-2.0 keeps its KV cache in NVFP4 and restores it with a parallel dequantization kernel
// before attention, FlashAttention being its attention backend (d9249.github.io review, section
// "핵심 아이디어 / 구조 / 동작 방식"; yourai.pro report).  Here the restore happens inside the
// attention kernel: a CTA reads the window's codes and scales (0.5625 B per element) and
// dequantizes every K/V tile into shared memory, so the BF16 K and V (2 B per element) are
// neither written to nor read from HBM.
//
// O[i,h,:] = sum_j softmax_j(scale * q[i,h,:] . k[j,h,:]) v[j,h,:] over the window's tokens, with
// k, v = BF16(FP32(e2m1 * sf) * g), the values the restore kernel produces.  No mask.
//
// Design (warp-level BF16 MMA, FlashAttention-2 structure):
//   - CTA = 128 query rows of one head, 8 warps x 16 rows; Q stays in registers as MMA A
//     fragments. Each CTA dequantizes its head's whole window once, so more rows per CTA means
//     less dequantization per FLOP.
//   - Per 64-token tile, each thread holds the raw bytes of half a token row of K or of V (32
//     code bytes, 4 scale bytes) fetched one tile ahead. It dequantizes them into a
//     double-buffered shared-memory tile. Rows are padded to 272 B, so neither the 16-byte
//     stores nor ldmatrix conflict on banks.
//   - S = Q K^T runs on mma.sync m16n8k16 with FP32 accumulation. Then an online softmax in
//     base 2, with the row max and sum combined across the quad by shuffles.
//   - P is rounded to BF16 for O += P V (V fragments by ldmatrix.trans).
//   - Tokens past the window's end score -inf. The only waits are __syncthreads.
#include <atomic>
#include <cmath>

#include "common.cuh"
#include "attention.h"

namespace nvfp4 {

namespace {

constexpr int kD = 128;                     // head_dim
constexpr int kBQ = 128;                    // query rows per CTA
constexpr int kBK = 64;                     // window tokens per tile
constexpr int kThreads = 256;
constexpr int kPitch = kD * 2 + 16;         // bytes per shared-memory tile row
constexpr int kTileBytes = kBK * kPitch;
constexpr int kSmemBytes = 4 * kTileBytes;  // K and V, two buffers each

static_assert(kThreads == 4 * kBK, "a thread loads half a token row of K or of V");
static_assert(kBQ == 16 * (kThreads / 32), "a warp owns 16 query rows");

// y = BF16(FP32(e2m1 * sf) * g) for the 8 codes of one word: the restore's rounding steps (the
// e2m1 * sf product is exact in FP32, one rounding by g, one to BF16).
__device__ __forceinline__ uint4 restore8(uint32_t codes, float sf, float g) {
    uint32_t h[4];
    e2m1x8_to_f16x2(codes, h);
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float lo = __fmul_rn(__half2float(__ushort_as_half((unsigned short)(h[i] & 0xFFFFu))), sf);
        const float hi = __fmul_rn(__half2float(__ushort_as_half((unsigned short)(h[i] >> 16))), sf);
        o[i] = bf16x2(__fmul_rn(lo, g), __fmul_rn(hi, g));
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ldg_nc_u32(const void *p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ void sts_v4(uint32_t saddr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" :: "r"(saddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t saddr, uint32_t r[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(saddr) : "memory");
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t saddr, uint32_t r[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(saddr) : "memory");
}

// c += a . b for one 16 x 8 x 16 BF16 tile, FP32 accumulation.
__device__ __forceinline__ void mma_bf16(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Raw NVFP4 bytes of half a token row (64 elements) of K or of V, and the slot's g.
struct Raw {
    uint4 c[2];
    uint32_t sf;
    float g;
};

// Fetch window token `tok` of K (v == 0) or V (v == 1), zeros past the end; `si` is the
// thread's running slot index (tokens only grow, so it only moves forward).
__device__ __forceinline__ void fetch(const AttnJob &j, int64_t tok, int &si, int head, int hf, int v, Raw &w) {
    w.c[0] = w.c[1] = make_uint4(0, 0, 0, 0);
    w.sf = 0;
    w.g = 0.0f;
    if (tok >= j.total_tokens) return;
    while (si + 1 < j.nslots && tok >= j.slot[si + 1].tok_begin) ++si;
    const AttnSlot &s = j.slot[si];
    const int64_t t = tok - s.tok_begin;
    const uint8_t *codes = v ? s.codes_v : s.codes_k;
    const int64_t cb = t * j.row_bytes + head * (kD / 2) + hf * 32;
    w.c[0] = ldg_nc_v4(codes + cb);
    w.c[1] = ldg_nc_v4(codes + cb + 16);
    w.sf = ldg_nc_u32((v ? s.sf_v : s.sf_k) + t * j.row_sf + head * (kD / 16) + hf * 4);
    w.g = *(v ? s.g_v : s.g_k);
}

// Dequantize one half row (8 words of codes, 4 block scales) into shared memory at `dst`.
__device__ __forceinline__ void put_half(uint32_t dst, const uint4 c[2], uint32_t sf, float g) {
    const uint32_t cw[8] = {c[0].x, c[0].y, c[0].z, c[0].w, c[1].x, c[1].y, c[1].z, c[1].w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float s = e4m3_to_f32((sf >> (8 * (i >> 1))) & 0xFFu);   // 16-block i/2
        sts_v4(dst + 16 * i, restore8(cw[i], s, g));
    }
}

__global__ void __launch_bounds__(kThreads, 1) kv_attention_kernel(const __grid_constant__ AttnJob j) {
    extern __shared__ __align__(128) uint8_t smem[];
    griddep_wait();                                       // the cache and q written by earlier kernels
    griddep_launch_dependents();
    const int head = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq4 = lane & 3;              // MMA fragment row group, column pair
    const int64_t r0 = (int64_t)blockIdx.x * kBQ + warp * 16 + g, r1 = r0 + 8;

    // Q A fragments of this warp's 16 rows (rows past tq are zero and not stored)
    uint32_t qa[kD / 16][4];
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) {
        const int c = head * kD + kk * 16 + tq4 * 2;
        qa[kk][0] = r0 < j.tq ? *reinterpret_cast<const uint32_t *>(j.q + r0 * j.ldq + c) : 0u;
        qa[kk][1] = r1 < j.tq ? *reinterpret_cast<const uint32_t *>(j.q + r1 * j.ldq + c) : 0u;
        qa[kk][2] = r0 < j.tq ? *reinterpret_cast<const uint32_t *>(j.q + r0 * j.ldq + c + 8) : 0u;
        qa[kk][3] = r1 < j.tq ? *reinterpret_cast<const uint32_t *>(j.q + r1 * j.ldq + c + 8) : 0u;
    }

    float o[kD / 8][4];
#pragma unroll
    for (int n = 0; n < kD / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.0f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;   // rows g and g + 8

    // loader: token row, half of it, K or V
    const int lr = threadIdx.x & (kBK - 1), hf = (threadIdx.x / kBK) & 1, lv = threadIdx.x / (2 * kBK);
    const int mi = lane >> 3, mr = lane & 7;              // ldmatrix: matrix, row within it
    int si = 0;
    Raw w;
    fetch(j, lr, si, head, hf, lv, w);
    const uint32_t sbase = smem_addr(smem);
    const int64_t ntiles = (j.total_tokens + kBK - 1) / kBK;
    for (int64_t it = 0; it < ntiles; ++it) {
        // Buffer it & 1: every warp finished tile it - 2 (which used it) before passing the
        // barrier of tile it - 1, so it can be overwritten now.
        const uint32_t kb = sbase + (uint32_t)(it & 1) * 2u * kTileBytes, vb = kb + kTileBytes;
        put_half((lv ? vb : kb) + lr * kPitch + hf * 128, w.c, w.sf, w.g);
        if (it + 1 < ntiles) fetch(j, (it + 1) * kBK + lr, si, head, hf, lv, w);
        __syncthreads();

        // S = Q K^T: 16 rows x 64 tokens per warp
        float s[kBK / 8][4];
#pragma unroll
        for (int n = 0; n < kBK / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.0f;
#pragma unroll
        for (int np = 0; np < kBK / 16; ++np) {
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
                uint32_t b[4];
                ldmatrix_x4(kb + (np * 16 + (mi >> 1) * 8 + mr) * kPitch + (kk * 16 + (mi & 1) * 8) * 2, b);
                mma_bf16(s[2 * np], qa[kk], b[0], b[1]);
                mma_bf16(s[2 * np + 1], qa[kk], b[2], b[3]);
            }
        }

        // online softmax (base 2): scale, mask the tokens past the window, new row maxima
        const int64_t t0 = it * kBK;
        float x0 = -INFINITY, x1 = -INFINITY;
#pragma unroll
        for (int n = 0; n < kBK / 8; ++n) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const bool ok = t0 + n * 8 + tq4 * 2 + e < j.total_tokens;
                s[n][e] = ok ? s[n][e] * j.scale_log2 : -INFINITY;
                s[n][2 + e] = ok ? s[n][2 + e] * j.scale_log2 : -INFINITY;
                x0 = fmaxf(x0, s[n][e]);
                x1 = fmaxf(x1, s[n][2 + e]);
            }
        }
        x0 = fmaxf(x0, __shfl_xor_sync(0xFFFFFFFFu, x0, 1));
        x0 = fmaxf(x0, __shfl_xor_sync(0xFFFFFFFFu, x0, 2));
        x1 = fmaxf(x1, __shfl_xor_sync(0xFFFFFFFFu, x1, 1));
        x1 = fmaxf(x1, __shfl_xor_sync(0xFFFFFFFFu, x1, 2));
        const float n0 = fmaxf(m0, x0), n1 = fmaxf(m1, x1);
        const float b0 = n0 == -INFINITY ? 0.0f : n0, b1 = n1 == -INFINITY ? 0.0f : n1;   // no inf - inf
        const float a0 = exp2f(m0 - b0), a1 = exp2f(m1 - b1);
        m0 = n0;
        m1 = n1;
        l0 *= a0;
        l1 *= a1;
#pragma unroll
        for (int n = 0; n < kD / 8; ++n) {
            o[n][0] *= a0;
            o[n][1] *= a0;
            o[n][2] *= a1;
            o[n][3] *= a1;
        }

        // P (BF16) as A fragments: tokens 16kk..16kk+15 come from S tiles 2kk and 2kk + 1
        uint32_t pa[kBK / 16][4];
#pragma unroll
        for (int n = 0; n < kBK / 8; ++n) {
            const float p00 = exp2f(s[n][0] - b0), p01 = exp2f(s[n][1] - b0);
            const float p10 = exp2f(s[n][2] - b1), p11 = exp2f(s[n][3] - b1);
            l0 += p00 + p01;
            l1 += p10 + p11;
            pa[n >> 1][(n & 1) * 2] = bf16x2(p00, p01);
            pa[n >> 1][(n & 1) * 2 + 1] = bf16x2(p10, p11);
        }

        // O += P V
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
#pragma unroll
            for (int dp = 0; dp < kD / 16; ++dp) {
                uint32_t b[4];
                ldmatrix_x4_trans(vb + (kk * 16 + (mi & 1) * 8 + mr) * kPitch + (dp * 16 + (mi >> 1) * 8) * 2, b);
                mma_bf16(o[2 * dp], pa[kk], b[0], b[1]);
                mma_bf16(o[2 * dp + 1], pa[kk], b[2], b[3]);
            }
        }
    }

    // normalise and store (each row's sum >= 1: its maximum contributes exp2(0))
    l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 1);
    l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 2);
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 1);
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 2);
    const float i0 = 1.0f / l0, i1 = 1.0f / l1;
#pragma unroll
    for (int n = 0; n < kD / 8; ++n) {
        const int c = head * kD + n * 8 + tq4 * 2;
        if (r0 < j.tq) *reinterpret_cast<uint32_t *>(j.o + r0 * j.ldo + c) = bf16x2(o[n][0] * i0, o[n][1] * i0);
        if (r1 < j.tq) *reinterpret_cast<uint32_t *>(j.o + r1 * j.ldo + c) = bf16x2(o[n][2] * i1, o[n][3] * i1);
    }
}

}  // namespace

cudaError_t launch_kv_attention(const AttnJob &j, int32_t *status, cudaStream_t s) {
    (void)status;                                         // this kernel never waits
    if (j.tq <= 0) return cudaSuccess;
    static std::atomic<bool> attr_set[64];               // per device; a repeated set is harmless
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(kv_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(true, std::memory_order_release);
    }
    const dim3 grid((unsigned)ceil_div(j.tq, kBQ), (unsigned)j.heads);
    return launch_pdl(kv_attention_kernel, grid, dim3(kThreads), kSmemBytes, s, j);
}

}  // namespace nvfp4
