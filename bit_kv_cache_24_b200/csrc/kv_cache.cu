// kv_cache.cu -- parallel NVFP4 -> BF16 restore of a KV-cache window.
//
// LongLive-2.0 stores the KV cache in NVFP4 and restores it with a parallel dequantization
// kernel before attention (d9249.github.io review, section "핵심 아이디어 / 구조 / 동작 방식";
// yourai.pro: "faster FP4 dequantization", in-place quantized cache updates).  The append side
// is the row-wise quantizer of quantize.cu run on the chunk's K and V in one launch.
//
// Design (B200, HBM-bound: 0.5625 B read + 2 B written per element): a lane restores 32
// consecutive elements from one 16-byte code load and one 2-byte scale load (the hardware
// E2M1 -> f16x2 conversion, FP32 scaling, BF16 packing); a warp keeps two 1024-element spans in
// flight, stages each span's 2 KB of output in shared memory and writes it with one bulk (TMA)
// store.  K and V are the two halves of the grid.
// The slot table (which slot's storage feeds which output tokens) is a kernel parameter, so
// the host builds no device-side state.
#include "common.cuh"
#include "launch.h"

namespace nvfp4 {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kSpan = 1024;                 // elements of a token row one warp restores per item
constexpr int kItems = 2;                   // items a warp keeps in flight

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

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ldg_nc_u16(const void *p) {
    unsigned short v;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ void sts_v4(uint32_t saddr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" :: "r"(saddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// Bulk (TMA) store of `bytes` from shared to global memory, issued by one elected lane of a
// converged warp, tracked in the issuing thread's bulk-async group.
__device__ __forceinline__ void bulk_store(void *gdst, uint32_t ssrc, uint32_t bytes) {
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
                 "@p cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;\n\t"
                 "@p cp.async.bulk.commit_group;\n\t}"
                 :: "l"(gdst), "r"(ssrc), "r"(bytes) : "memory");
}

// Wait until the bulk stores of this thread have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
                 "@p cp.async.bulk.wait_group.read 0;\n\t}" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
                 "@p cp.async.bulk.wait_group 0;\n\t}" ::: "memory");
}

// Work item = (token row, 1024-element span): lane l restores elements [32l, 32l+32) of the span
// from one 16-byte code load and one 2-byte scale load (two 16-blocks), a warp keeps kItems
// items in flight.  The span's 2 KB of BF16 output is staged in shared memory and written with
// one bulk (TMA) store, so global writes are whole contiguous lines.
__global__ void __launch_bounds__(kThreads) kv_dequant_kernel(const __grid_constant__ DequantJob jk,
                                                              const __grid_constant__ DequantJob jv) {
    __shared__ __align__(128) uint8_t stage[kWarps][kItems][kSpan * 2];
    griddep_wait();                                       // the cache written by earlier kernels
    griddep_launch_dependents();
    const DequantJob &j = blockIdx.y == 0 ? jk : jv;
    const int lane = threadIdx.x & 31;
    const int warp = __shfl_sync(0xFFFFFFFFu, (int)(threadIdx.x >> 5), 0);
    const int64_t row_bytes = j.row_elems >> 1, row_sf = j.row_elems >> 4;
    const int64_t spans = (j.row_elems + kSpan - 1) / kSpan;
    const int64_t items = j.total_tokens * spans;
    const int64_t stride = (int64_t)gridDim.x * kWarps * kItems;
    for (int64_t it0 = ((int64_t)blockIdx.x * kWarps + warp) * kItems; it0 < items; it0 += stride) {
        uint4 cw[kItems];
        uint32_t sfw[kItems];
        float gv[kItems];
        int64_t r[kItems], e[kItems];
#pragma unroll
        for (int u = 0; u < kItems; ++u) {
            const int64_t it = it0 + u;
            r[u] = it / spans;
            e[u] = (it - r[u] * spans) * kSpan;
            cw[u] = make_uint4(0, 0, 0, 0);
            sfw[u] = 0;
            gv[u] = 0.0f;
            if (it < items) {
                // slot holding output token r: last slot with tok_begin <= r (warp-uniform search)
                int lo = 0, hi = j.nslots - 1;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (j.slot[mid].tok_begin <= r[u]) lo = mid; else hi = mid - 1;
                }
                const DequantSlot &sl = j.slot[lo];
                const int64_t t = r[u] - sl.tok_begin;
                const int64_t el = e[u] + lane * 32;
                gv[u] = *sl.g;
                if (el < j.row_elems && NVFP4_CHECKED(t * row_bytes + (el >> 1), 16, sl.ntok * row_bytes, j.status) &&
                    NVFP4_CHECKED(t * row_sf + (el >> 4), 2, sl.ntok * row_sf, j.status)) {
                    cw[u] = ldg_nc_v4(sl.codes + t * row_bytes + (el >> 1));
                    sfw[u] = ldg_nc_u16(sl.sf + t * row_sf + (el >> 4));
                }
            }
        }
        bulk_wait_read();                                 // the previous iteration's stores left smem
        __syncwarp();
#pragma unroll
        for (int u = 0; u < kItems; ++u) {
            const uint32_t sb = smem_addr(&stage[warp][u][lane * 64]);
            const float s0 = e4m3_to_f32(sfw[u] & 0xFFu), s1 = e4m3_to_f32(sfw[u] >> 8);
            sts_v4(sb, dequant8(cw[u].x, s0, gv[u]));
            sts_v4(sb + 16, dequant8(cw[u].y, s0, gv[u]));
            sts_v4(sb + 32, dequant8(cw[u].z, s1, gv[u]));
            sts_v4(sb + 48, dequant8(cw[u].w, s1, gv[u]));
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // smem writes -> async proxy
        __syncwarp();
#pragma unroll
        for (int u = 0; u < kItems; ++u) {
            if (it0 + u >= items) break;
            const int64_t n = j.row_elems - e[u] < kSpan ? j.row_elems - e[u] : kSpan;
            if (NVFP4_CHECKED(r[u] * j.row_elems + e[u], n, j.total_tokens * j.row_elems, j.status))
                bulk_store(j.out + r[u] * j.row_elems + e[u], smem_addr(&stage[warp][u][0]), (uint32_t)(n * 2));
        }
    }
    bulk_wait_all();                                      // stores done before shared memory goes away
}

}  // namespace

cudaError_t launch_kv_dequant(const DequantJob *k, const DequantJob *v, int32_t *status, cudaStream_t s) {
    (void)status;
    const int64_t tokens = k->total_tokens;
    if (tokens <= 0) return cudaSuccess;
    const int64_t items = tokens * ((k->row_elems + kSpan - 1) / kSpan);
    // one pass: every CTA restores kWarps * kItems spans and exits (a grid capped at 8 CTAs per SM
    // looping over the items measured 146 us for the 56160-token window, one pass 136 us); the
    // grid-stride loop remains for grids past 2^31
    int64_t blocks = ceil_div(items, (int64_t)kWarps * kItems);
    if (blocks > 0x7FFFFFFF) blocks = 0x7FFFFFFF;
    return launch_pdl(kv_dequant_kernel, dim3((unsigned)blocks, 2), dim3(kThreads), 0, s, *k, *v);
}

}  // namespace nvfp4
