// launch.h -- internal host-side launch interface between the C ABI (capi.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace nvfp4 {

constexpr int kMaxPartials = 1024;        // per-CTA partial maxima of one amax pass
constexpr int kMaxJobs = 2;               // tensors quantized by one launch (K and V)

// One tensor to reduce / quantize row-wise.
struct RowJob {
    const uint16_t *x;      // BF16 [rows][ld]
    int64_t rows, cols, ld;
    uint8_t *codes;         // [rows][pitch]
    int64_t pitch;
    uint8_t *sf;
    int32_t sf_layout;      // 0 linear [rows][ceil(cols/16)], 1 tensor-core layout
    float *g_out;
    const float *amax_in;   // nullable device pointer
    uint32_t *partial;      // [kMaxPartials] partial maxima (BF16 magnitude bits)
};

struct RowJobs {
    RowJob job[kMaxJobs];
    int32_t njobs;
    int32_t npartial;
};

cudaError_t launch_amax(const RowJobs &jobs, int32_t *status, float *amax_out, cudaStream_t s);
cudaError_t launch_quantize_rows(const RowJobs &jobs, int32_t *status, cudaStream_t s);
// Column-wise: blocks along the rows of x; output [cols][pitch(rows)].
cudaError_t launch_quantize_cols(const RowJob &job, int32_t npartial, int32_t *status, cudaStream_t s);
int amax_blocks(int64_t rows);

struct DequantSlot {
    const uint8_t *codes;   // [ntok][row_bytes]
    const uint8_t *sf;      // [ntok][row_sf]
    const float *g;
    int64_t tok_begin;      // first output token of this slot
};

constexpr int kMaxDequantSlots = 128;

struct DequantJob {
    DequantSlot slot[kMaxDequantSlots];
    int32_t nslots;
    int64_t total_tokens;
    int64_t row_elems;      // heads * head_dim
    uint16_t *out;          // [total_tokens][row_elems]
};

cudaError_t launch_kv_dequant(const DequantJob *k, const DequantJob *v, int32_t *status, cudaStream_t s);

struct GemmArgs {
    const uint8_t *a_codes, *b_codes;
    const uint8_t *a_sf, *b_sf;          // tensor-core layout
    const float *ga, *gb;
    int64_t M, N, K;
    int64_t a_pitch, b_pitch;             // bytes per code row
    const uint16_t *bias, *resid;
    void *y;
    int64_t ldy;
    int32_t y_f32;
    int32_t *status;
};

cudaError_t launch_gemm(const GemmArgs &args, cudaStream_t s);
// CTA-pair (cta_group::2) variant for M > 128; launch_gemm dispatches to it.
cudaError_t launch_gemm_2sm(const GemmArgs &args, cudaStream_t s);

cudaError_t launch_encode_elements(const float *in, int64_t n, uint8_t *e2m1_out, uint8_t *e4m3_out, cudaStream_t s);
cudaError_t launch_wait_timeout(int32_t *status, int64_t limit_ns, cudaStream_t s);

int num_sms();

// Text returned by nvfp4_last_error() on this thread.
void record_error(const char *msg);

}  // namespace nvfp4
