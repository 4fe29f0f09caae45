// kv_cache.cu -- parallel NVFP4 -> BF16 restore of a KV-cache window.
//
// LongLive-2.0 stores the KV cache in NVFP4 and restores it with a parallel dequantization
// kernel before attention (d9249.github.io review, section "핵심 아이디어 / 구조 / 동작 방식";
// yourai.pro: "faster FP4 dequantization", in-place quantized cache updates).  The append side
// is the row-wise quantizer of quantize.cu run on the chunk's K and V in one launch.
//
// Design (B200, HBM-bound: 0.5625 B read + 2 B written per element): one warp restores one
// token row at a time; per step a lane decodes 8 codes (a 4-byte load; the warp reads 128
// contiguous bytes) with the hardware E2M1 -> f16x2 conversion, scales them in FP32 and writes
// 16 bytes (the warp writes 512 contiguous bytes).  K and V are the two halves of the grid.
// The slot table (which slot's storage feeds which output tokens) is a kernel parameter, so
// the host builds no device-side state.
#include "common.cuh"
#include "launch.h"

namespace nvfp4 {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint32_t ldg_nc_u32(const void *p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ void stg_v4(void *p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// y = BF16(FP32(e2m1 * sf) * g) for 8 codes packed in one word.
__device__ __forceinline__ uint4 dequant8(uint32_t codes, float sf, float g) {
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

__global__ void __launch_bounds__(kThreads) kv_dequant_kernel(const __grid_constant__ DequantJob jk,
                                                              const __grid_constant__ DequantJob jv) {
    const DequantJob &j = blockIdx.y == 0 ? jk : jv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t row_bytes = j.row_elems >> 1, row_sf = j.row_elems >> 4, chunks = j.row_elems >> 3;
    for (int64_t r = (int64_t)blockIdx.x * kWarps + warp; r < j.total_tokens; r += (int64_t)gridDim.x * kWarps) {
        // slot holding output token r: last slot with tok_begin <= r (warp-uniform search)
        int lo = 0, hi = j.nslots - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (j.slot[mid].tok_begin <= r) lo = mid; else hi = mid - 1;
        }
        const DequantSlot &s = j.slot[lo];
        const int64_t t = r - s.tok_begin;
        const uint8_t *codes = s.codes + t * row_bytes;
        const uint8_t *sf = s.sf + t * row_sf;
        const float g = *s.g;
        uint16_t *out = j.out + r * j.row_elems;
        int64_t c = lane;
        for (; c + 96 < chunks; c += 128) {
            uint32_t w[4];
            float f[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                w[u] = ldg_nc_u32(codes + 4 * (c + 32 * u));
                f[u] = e4m3_to_f32(sf[(c + 32 * u) >> 1]);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) stg_v4(out + 8 * (c + 32 * u), dequant8(w[u], f[u], g));
        }
        for (; c < chunks; c += 32) {
            const uint32_t w = ldg_nc_u32(codes + 4 * c);
            stg_v4(out + 8 * c, dequant8(w, e4m3_to_f32(sf[c >> 1]), g));
        }
    }
}

}  // namespace

cudaError_t launch_kv_dequant(const DequantJob *k, const DequantJob *v, int32_t *status, cudaStream_t s) {
    (void)status;
    const int64_t tokens = k->total_tokens;
    if (tokens <= 0) return cudaSuccess;
    int64_t blocks = ceil_div(tokens, kWarps);
    const int64_t cap = 8 * (int64_t)num_sms();
    if (blocks > cap) blocks = cap;
    kv_dequant_kernel<<<dim3((unsigned)blocks, 2), kThreads, 0, s>>>(*k, *v);
    return cudaGetLastError();
}

}  // namespace nvfp4
