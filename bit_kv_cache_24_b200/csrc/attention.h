// attention.h -- launcher interface of the attention that reads the NVFP4 KV cache directly.
#pragma once

#include "launch.h"

namespace nvfp4 {

// One slot of the window: its K/V codes and scales from its first token, its two g, and the
// window position of that first token.
struct AttnSlot {
    const uint8_t *codes_k, *codes_v;   // [ntok][row_bytes]
    const uint8_t *sf_k, *sf_v;         // [ntok][row_sf]
    const float *g_k, *g_v;
    int64_t tok_begin;
    int64_t ntok;                       // tokens the slot holds (extent of its arrays, checked build)
};

struct AttnJob {
    AttnSlot slot[kMaxDequantSlots];    // non-empty slots, window order
    int32_t nslots;
    int32_t heads;
    int64_t total_tokens;               // window tokens (>= 1)
    int64_t row_bytes, row_sf;          // heads * head_dim / 2, heads * head_dim / 16
    const uint16_t *q;                  // [tq][ldq] BF16, head h at columns [h * 128, h * 128 + 128)
    int64_t ldq, tq;
    uint16_t *o;                        // [tq][ldo] BF16, same column layout
    int64_t ldo;
    float scale_log2;                   // softmax scale * log2(e)
    int64_t q_elems, o_elems;           // extents of q and o from their starts (checked build)
};

// head_dim is 128 (checked by the caller).  status: the optional device status word (a bounded
// wait that gives up writes NVFP4_ERR_TIMEOUT there).
cudaError_t launch_kv_attention(const AttnJob &j, int32_t *status, cudaStream_t s);

}  // namespace nvfp4
