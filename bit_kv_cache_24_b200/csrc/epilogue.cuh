// epilogue.cuh -- the NVFP4-emitting part of the GEMM epilogue, shared by both GEMM kernels.
//
// LongLive-2.0 runs its linear layers in W4A4 NVFP4, so a layer's output is the NVFP4 operand of
// the next GEMM; emitting it from the epilogue, with a per-tensor scale fixed in advance (amax
// given, e.g. from the previous step), saves writing and re-reading the BF16 output.  The codes
// and scales are exactly those of nvfp4_quantize(Y, amax_in) on the BF16 values the epilogue
// rounds (the same 16-block step, see quantize16 in common.cuh).
#pragma once

#include "common.cuh"
#include "launch.h"

namespace nvfp4 {

// Copy the scale record to shared memory (after griddep_wait; threads 0..128 of the CTA); a
// barrier must follow.
__device__ __forceinline__ void load_record_plain(const ScaleRecord *rec, SmemRecord &s) {
    if (threadIdx.x < 128) s.r_tab[threadIdx.x] = rec->r_tab[threadIdx.x];
    if (threadIdx.x == 128) {
        s.den = rec->den;
        s.inv_den = rec->inv_den;
        s.ok = rec->ok;
    }
}

// The two scale bytes of 16-blocks blk and blk + 1 (blk even) of row m, adjacent in both layouts.
__device__ __forceinline__ void store_sf_pair(const GemmArgs &a, int64_t m, int64_t blk, uint32_t two) {
    const int64_t nb = a.N >> 4;
    const int64_t off = a.q_sf_layout ? sf_mma_offset(m, blk, (nb + 3) >> 2) : m * nb + blk;
    if (NVFP4_CHECKED(off, 2, a.q_sf_bytes, a.status)) *reinterpret_cast<uint16_t *>(a.q_sf + off) = (uint16_t)two;
}

// Row-wise NVFP4 of one 32-column chunk of output row m (columns n0 .. n0 + 31, n0 % 32 == 0,
// all inside N): w holds the chunk's BF16 values as 16 packed words (element 2i in the low half
// of w[i]).
__device__ __forceinline__ void emit_nvfp4_chunk(const GemmArgs &a, const SmemRecord &rec, int64_t m, int64_t n0,
                                                 const uint32_t w[16]) {
    uint32_t c0, c1, s0, c2, c3, s1;
    quantize16(w, rec, c0, c1, s0);
    quantize16(w + 8, rec, c2, c3, s1);
    if (NVFP4_CHECKED(m * a.q_pitch + (n0 >> 1), 16, a.q_codes_bytes, a.status))
        *reinterpret_cast<uint4 *>(a.q_codes + m * a.q_pitch + (n0 >> 1)) = make_uint4(c0, c1, c2, c3);
    store_sf_pair(a, m, n0 >> 4, s0 | (s1 << 8));
}

}  // namespace nvfp4
