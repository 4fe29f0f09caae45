// launch.h -- internal host-side launch interface between the C ABI (capi.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace nvfp4 {

constexpr int kMaxPartials = 1024;        // per-CTA partial maxima of one amax pass
constexpr int kMaxJobs = 2;               // tensors quantized by one launch (K and V)

// Per-tensor scale record: written once per quantization by the record kernel from the amax,
// read by every CTA of the quantize passes.
struct ScaleRecord {
    uint32_t ok;            // 0: the tensor (or amax_in) was non-finite; the quantize passes skip
    float g;                // decode scale amax / 2688 (1 when amax == 0)
    float den;              // g * 6
    float inv_den;          // RN(1 / den), or 0 when den < 2^-125 (the quotient then divides)
    float r_tab[128];       // r_tab[sf] = RN(1 / RN(e4m3(sf) * g)), 0 where that product is 0
};

// Device workspace of one quantized tensor: the amax partials, then its scale record.
constexpr size_t kRecordOffset = kMaxPartials * sizeof(uint32_t);
constexpr size_t kTensorScratchBytes = kRecordOffset + 1024;
static_assert(sizeof(ScaleRecord) <= 1024, "record fits its slot");

// One tensor to reduce / quantize.
struct RowJob {
    const uint16_t *x;      // BF16 [rows][ld]
    int64_t rows, cols, ld;
    uint8_t *codes;         // [rows][pitch] (column-wise: [cols][pitch])
    int64_t pitch;
    uint8_t *sf;
    int32_t sf_layout;      // 0 linear [rows][ceil(cols/16)], 1 tensor-core layout
    uint32_t *partial;      // [kMaxPartials] partial maxima (BF16 magnitude bits), amax pass
    const ScaleRecord *rec; // read by the quantize passes (unless amax_in is set)
    // Given amax (device float, nullable): the quantize pass builds its scale record itself
    // (no record kernel) and, when report_record is set, its first CTA writes g to g_out[]
    // (nullable) or, for a non-finite amax, NVFP4_ERR_NONFINITE to status.
    const float *amax_in;
    float *g_out[2];
    int32_t report_record;
    // Set only when x was complete before this job's own amax pass read it (amax pass, record
    // kernel, then this pass): the row pass then loads x before its dependency wait, overlapping
    // the loads with the record kernel, and waits only before reading the record.
    int32_t x_early;
    int32_t *status;
    // buffer extents for the checked build (see NVFP4_CHECKED): elements of x from its start,
    // bytes of codes and of sf
    int64_t x_elems, codes_bytes, sf_bytes;
};

struct RowJobs {
    RowJob job[kMaxJobs];
    int32_t njobs;
    int32_t npartial;
};

// One tensor's scale record: from the partials of its amax pass, or from amax_in when non-null.
struct RecJob {
    const uint32_t *partial;
    const float *amax_in;
    ScaleRecord *rec;
    float *g_out[2];        // nullable: receive g (row- and column-wise outputs)
};

struct RecJobs {
    RecJob job[kMaxJobs];
    int32_t njobs;
    int32_t npartial;
};

cudaError_t launch_amax(const RowJobs &jobs, int32_t *status, float *amax_out, cudaStream_t s);
cudaError_t launch_scale_record(const RecJobs &jobs, int32_t *status, cudaStream_t s);
cudaError_t launch_quantize_rows(const RowJobs &jobs, cudaStream_t s);
// Column-wise: blocks along the rows of x; output [cols][pitch(rows)].  after_rows: launched
// directly after launch_quantize_rows of the same x and record (runs concurrently with it).
cudaError_t launch_quantize_cols(const RowJob &job, bool after_rows, cudaStream_t s);
int amax_blocks(int64_t rows);

// Launch with programmatic stream serialization (see griddep_wait in common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

struct DequantSlot {
    const uint8_t *codes;   // [ntok][row_bytes]
    const uint8_t *sf;      // [ntok][row_sf]
    const float *g;
    int64_t tok_begin;      // first output token of this slot
    int64_t ntok;           // tokens the slot holds (extent of codes and sf, checked build)
};

constexpr int kMaxDequantSlots = 128;

struct DequantJob {
    DequantSlot slot[kMaxDequantSlots];
    int32_t nslots;
    int64_t total_tokens;
    int64_t row_elems;      // heads * head_dim
    uint16_t *out;          // [total_tokens][row_elems]
    int32_t *status;        // status word (checked build)
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
    // optional NVFP4-emitting epilogue: the row-wise quantization of the BF16 output with the
    // scale record q_rec (computed from a given amax); y may then be null
    const ScaleRecord *q_rec;
    uint8_t *q_codes;
    uint8_t *q_sf;
    int64_t q_pitch;
    int32_t q_sf_layout;
    // optional per-block amax of the BF16 output: max |Y| (BF16 magnitude bits) of each 32-row x
    // 128-column block, at cam_partial[(row / 32) * cam_n128 + col / 128] (N % 256 == 0)
    uint32_t *cam_partial;
    int64_t cam_n128;
    // buffer extents for the checked build (elements of y, bias and resid; bytes of q_codes and
    // q_sf; words of cam_partial)
    int64_t y_elems, bias_elems, resid_elems, q_codes_bytes, q_sf_bytes, cam_elems;
};

// Column-group amax from the GEMM's block partials: amax_out[g] = max over the blocks of columns
// [g * group_cols, (g + 1) * group_cols) (one CTA per group).
cudaError_t launch_colamax_finish(const uint32_t *partial, int64_t rows32, int64_t n128, int64_t group_cols,
                                  int64_t groups, float *amax_out, int32_t *status, cudaStream_t s);

cudaError_t launch_gemm(const GemmArgs &args, cudaStream_t s);
// CTA-pair (cta_group::2) variant for M > 128; launch_gemm dispatches to it.
cudaError_t launch_gemm_2sm(const GemmArgs &args, cudaStream_t s);

cudaError_t launch_encode_elements(const float *in, int64_t n, uint8_t *e2m1_out, uint8_t *e4m3_out, cudaStream_t s);
cudaError_t launch_wait_timeout(int32_t *status, int64_t limit_ns, cudaStream_t s);
cudaError_t launch_bounds_selftest(uint8_t *buf, int64_t extent, int64_t index, int32_t *status, cudaStream_t s);

int num_sms();

// Text returned by nvfp4_last_error() on this thread.
void record_error(const char *msg);

}  // namespace nvfp4
