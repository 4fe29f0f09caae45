// capi.cu -- the C ABI declared in include/nvfp4.h: argument validation, layout arithmetic,
// architecture checks and kernel dispatch.  No allocation, no synchronisation.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "attention.h"

namespace nvfp4 {

namespace {

thread_local char g_last_error[256] = "";

nvfp4_status cuda_fail(cudaError_t e, const char *where) {
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorString(e));
    return NVFP4_ERR_CUDA;
}

struct DevInfo {
    std::atomic<bool> probed{false};   // set (release) after the fields below
    bool sm100 = false;
    int sms = 148;
};
DevInfo g_dev[64];
std::mutex g_dev_mutex;

// The current device's properties, probed once per device (thread-safe).
const DevInfo *device_info() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    DevInfo &d = g_dev[dev];
    if (!d.probed.load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lock(g_dev_mutex);
        if (!d.probed.load(std::memory_order_relaxed)) {
            int major = 0, minor = 0, sms = 0;
            if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
                cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
                return nullptr;
            d.sm100 = (major == 10 && minor == 0);
            d.sms = sms;
            d.probed.store(true, std::memory_order_release);
        }
    }
    return &d;
}

// Common pre-flight: a usable sm_100 device is current.
nvfp4_status check_device() {
    const DevInfo *d = device_info();
    if (!d) return cuda_fail(cudaGetLastError(), "device query");
    if (!d->sm100) return NVFP4_ERR_UNSUPPORTED;
    return NVFP4_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t codes_pitch(int64_t cols) { return 16 * ceil_div(cols, 32); }

int64_t sf_bytes(int64_t rows, int64_t cols, int32_t layout) {
    if (rows < 0 || cols < 0) return -1;
    const int64_t nb = ceil_div(cols, 16);
    if (layout == NVFP4_SF_LINEAR) return rows * nb;
    if (layout == NVFP4_SF_MMA) return 128 * ceil_div(rows, 128) * 4 * ceil_div(nb, 4);
    return -1;
}

// The quantizers index the units of one tensor, padding included, with 32-bit integers.
bool too_large(int64_t rows, int64_t cols) {
    return (uint64_t)(rows + 128) * (uint64_t)(cols + 128) >= (1ull << 35);
}

// Shared argument checks and GemmArgs of nvfp4_gemm / nvfp4_gemm_quant_out (y may be null only
// when allow_no_y).
nvfp4_status gemm_args(const nvfp4_tensor *A, const nvfp4_tensor *B, const void *bias_bf16, const void *resid_bf16,
                       void *y, int64_t ldy, int32_t y_dtype, bool allow_no_y, int32_t *dev_status, GemmArgs &a) {
    if (!A || !B || (!y && !allow_no_y) || !A->codes || !B->codes || !A->sf || !B->sf || !A->g || !B->g)
        return NVFP4_ERR_INVALID_ARG;
    if (A->rows <= 0 || B->rows <= 0 || A->cols <= 0 || A->cols != B->cols) return NVFP4_ERR_INVALID_ARG;
    if (bias_bf16 && resid_bf16) return NVFP4_ERR_INVALID_ARG;
    if (y_dtype != NVFP4_OUT_BF16 && y_dtype != NVFP4_OUT_F32) return NVFP4_ERR_INVALID_ARG;
    if ((y || resid_bf16) && ldy < B->rows) return NVFP4_ERR_INVALID_ARG;
    if (A->sf_layout != NVFP4_SF_MMA || B->sf_layout != NVFP4_SF_MMA) return NVFP4_ERR_UNSUPPORTED;
    if ((B->rows & 7) || ((y || resid_bf16) && (ldy & 7))) return NVFP4_ERR_UNSUPPORTED;
    if (!aligned16(A->codes) || !aligned16(B->codes) || !aligned16(A->sf) || !aligned16(B->sf) || (y && !aligned16(y)))
        return NVFP4_ERR_UNSUPPORTED;
    if ((bias_bf16 && !aligned16(bias_bf16)) || (resid_bf16 && !aligned16(resid_bf16))) return NVFP4_ERR_UNSUPPORTED;
    if ((A->rows + 127) / 128 > 0x7FFFFFFF / 128) return NVFP4_ERR_UNSUPPORTED;
    a = GemmArgs{};
    a.a_codes = A->codes;
    a.b_codes = B->codes;
    a.a_sf = A->sf;
    a.b_sf = B->sf;
    a.ga = A->g;
    a.gb = B->g;
    a.M = A->rows;
    a.N = B->rows;
    a.K = A->cols;
    a.a_pitch = codes_pitch(A->cols);
    a.b_pitch = codes_pitch(B->cols);
    a.bias = static_cast<const uint16_t *>(bias_bf16);
    a.resid = static_cast<const uint16_t *>(resid_bf16);
    a.y = y;
    a.ldy = ldy;
    a.y_f32 = y_dtype == NVFP4_OUT_F32;
    a.status = dev_status;
    a.y_elems = (A->rows - 1) * ldy + B->rows;
    a.bias_elems = B->rows;
    a.resid_elems = (A->rows - 1) * ldy + B->rows;
    return NVFP4_OK;
}


bool tensor_ok(const nvfp4_tensor *t, int64_t rows, int64_t cols) {
    return t && t->codes && t->sf && t->g && t->rows == rows && t->cols == cols &&
           (t->sf_layout == NVFP4_SF_LINEAR || t->sf_layout == NVFP4_SF_MMA);
}

}  // namespace

int num_sms() {
    const DevInfo *d = device_info();
    return d ? d->sms : 148;
}

void record_error(const char *msg) { std::snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }

}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

int32_t nvfp4_version(void) { return 100; }

int32_t nvfp4_checked_build(void) {
#ifdef NVFP4_DEBUG_CHECKS
    return 1;
#else
    return 0;
#endif
}

const char *nvfp4_last_error(void) { return g_last_error; }

const char *nvfp4_status_string(int32_t status) {
    switch (status) {
        case NVFP4_OK: return "ok";
        case NVFP4_ERR_INVALID_ARG: return "invalid argument";
        case NVFP4_ERR_UNSUPPORTED: return "unsupported shape, alignment, layout or architecture";
        case NVFP4_ERR_NONFINITE: return "non-finite input";
        case NVFP4_ERR_TIMEOUT: return "bounded on-chip wait timed out";
        case NVFP4_ERR_CUDA: return "CUDA error";
        case NVFP4_ERR_OUT_OF_BOUNDS: return "checked build: an access outside its buffer was skipped";
        default: return "unknown status";
    }
}

int64_t nvfp4_codes_pitch(int64_t cols) { return cols < 0 ? -1 : codes_pitch(cols); }

int64_t nvfp4_sf_bytes(int64_t rows, int64_t cols, int32_t layout) { return sf_bytes(rows, cols, layout); }

nvfp4_status nvfp4_sf_to_linear(const uint8_t *sf_mma, int64_t rows, int64_t cols, uint8_t *sf_linear) {
    if (!sf_mma || !sf_linear || rows <= 0 || cols <= 0) return NVFP4_ERR_INVALID_ARG;
    const int64_t nb = ceil_div(cols, 16), apr = ceil_div(nb, 4);
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t b = 0; b < nb; ++b) sf_linear[i * nb + b] = sf_mma[sf_mma_offset(i, b, apr)];
    return NVFP4_OK;
}

nvfp4_status nvfp4_sf_to_mma(const uint8_t *sf_linear, int64_t rows, int64_t cols, uint8_t *sf_mma) {
    if (!sf_mma || !sf_linear || rows <= 0 || cols <= 0) return NVFP4_ERR_INVALID_ARG;
    const int64_t nb = ceil_div(cols, 16), apr = ceil_div(nb, 4);
    memset(sf_mma, 0, (size_t)sf_bytes(rows, cols, NVFP4_SF_MMA));
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t b = 0; b < nb; ++b) sf_mma[sf_mma_offset(i, b, apr)] = sf_linear[i * nb + b];
    return NVFP4_OK;
}

size_t nvfp4_quantize_workspace(int64_t rows, int64_t cols) {
    (void)rows;
    (void)cols;
    return kTensorScratchBytes;
}

size_t nvfp4_kv_append_workspace(int64_t ntok, int32_t heads, int32_t head_dim) {
    (void)ntok;
    (void)heads;
    (void)head_dim;
    return 2 * kTensorScratchBytes;
}

nvfp4_status nvfp4_amax(const void *x_bf16, int64_t M, int64_t K, int64_t ld, float *amax_out, void *ws,
                        size_t ws_bytes, int32_t *dev_status, nvfp4_stream stream) {
    if (!x_bf16 || !amax_out || !ws || M < 0 || K < 0 || ld < K) return NVFP4_ERR_INVALID_ARG;
    if (ws_bytes < nvfp4_quantize_workspace(M, K)) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || !aligned16(ws) || (ld & 7) || (K & 7) || too_large(M, K)) return NVFP4_ERR_UNSUPPORTED;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    RowJobs jobs{};
    jobs.njobs = 1;
    jobs.npartial = amax_blocks(M);
    jobs.job[0].x = static_cast<const uint16_t *>(x_bf16);
    jobs.job[0].rows = M;
    jobs.job[0].cols = K;
    jobs.job[0].ld = ld;
    jobs.job[0].partial = static_cast<uint32_t *>(ws);
    jobs.job[0].status = dev_status;
    jobs.job[0].x_elems = M > 0 ? (M - 1) * ld + K : 0;
    cudaError_t e = launch_amax(jobs, dev_status, amax_out, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "nvfp4_amax");
}

nvfp4_status nvfp4_quantize(const void *x_bf16, int64_t M, int64_t K, int64_t ld, int32_t dir,
                            const float *amax_in, const nvfp4_tensor *out, void *ws, size_t ws_bytes,
                            int32_t *dev_status, nvfp4_stream stream) {
    if (!x_bf16 || !out || M <= 0 || K <= 0 || ld < K) return NVFP4_ERR_INVALID_ARG;
    if (dir != NVFP4_ROWWISE && dir != NVFP4_COLWISE && dir != NVFP4_ROWCOL) return NVFP4_ERR_INVALID_ARG;
    const nvfp4_tensor *row_out = dir != NVFP4_COLWISE ? &out[0] : nullptr;
    const nvfp4_tensor *col_out = dir == NVFP4_COLWISE ? &out[0] : (dir == NVFP4_ROWCOL ? &out[1] : nullptr);
    if (row_out && !tensor_ok(row_out, M, K)) return NVFP4_ERR_INVALID_ARG;
    if (col_out && !tensor_ok(col_out, K, M)) return NVFP4_ERR_INVALID_ARG;
    if (!ws || ws_bytes < nvfp4_quantize_workspace(M, K)) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || (ld & 7) || (K & 7) || too_large(M, K)) return NVFP4_ERR_UNSUPPORTED;
    if (row_out && (K & 15)) return NVFP4_ERR_UNSUPPORTED;
    if ((row_out && !aligned16(row_out->codes)) || (col_out && !aligned16(col_out->codes)) || !aligned16(ws))
        return NVFP4_ERR_UNSUPPORTED;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *scratch = static_cast<uint8_t *>(ws);
    ScaleRecord *rec = reinterpret_cast<ScaleRecord *>(scratch + kRecordOffset);

    // amax pass (unless amax_in), the scale record, then one pass per requested layout
    RowJobs jobs{};
    jobs.njobs = 1;
    jobs.npartial = amax_blocks(M);
    RowJob &j = jobs.job[0];
    j.x = static_cast<const uint16_t *>(x_bf16);
    j.rows = M;
    j.cols = K;
    j.ld = ld;
    j.partial = reinterpret_cast<uint32_t *>(scratch);
    j.rec = rec;
    j.status = dev_status;
    j.x_elems = (M - 1) * ld + K;
    RecJobs rj{};
    rj.njobs = 1;
    rj.npartial = jobs.npartial;
    rj.job[0].partial = j.partial;
    rj.job[0].amax_in = amax_in;
    rj.job[0].rec = rec;
    rj.job[0].g_out[0] = row_out ? row_out->g : nullptr;
    rj.job[0].g_out[1] = col_out ? col_out->g : nullptr;
    cudaError_t e = cudaSuccess;
    if (amax_in) {
        // one launch per layout: the quantize passes build the scale record from amax_in
        // themselves; the first pass reports g (both outputs) and a non-finite amax
        j.amax_in = amax_in;
        j.report_record = 1;
        j.g_out[0] = row_out ? row_out->g : col_out->g;
        j.g_out[1] = row_out && col_out ? col_out->g : nullptr;
    } else {
        e = launch_amax(jobs, dev_status, nullptr, s);
        if (e == cudaSuccess) e = launch_scale_record(rj, dev_status, s);
        j.x_early = 1;                                    // the amax pass read x after its wait
    }
    if (e == cudaSuccess && row_out) {
        j.codes = row_out->codes;
        j.pitch = codes_pitch(K);
        j.sf = row_out->sf;
        j.sf_layout = row_out->sf_layout;
        j.codes_bytes = M * codes_pitch(K);
        j.sf_bytes = sf_bytes(M, K, row_out->sf_layout);
        e = launch_quantize_rows(jobs, s);
    }
    if (e == cudaSuccess && col_out) {
        RowJob jc = j;
        if (row_out) jc.report_record = 0;                // the row pass reported already
        jc.codes = col_out->codes;
        jc.pitch = codes_pitch(M);
        jc.sf = col_out->sf;
        jc.sf_layout = col_out->sf_layout;
        jc.codes_bytes = K * codes_pitch(M);
        jc.sf_bytes = sf_bytes(K, M, col_out->sf_layout);
        e = launch_quantize_cols(jc, row_out != nullptr, s);
    }
    return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "nvfp4_quantize");
}

nvfp4_status nvfp4_gemm(const nvfp4_tensor *A, const nvfp4_tensor *B, const void *bias_bf16,
                        const void *resid_bf16, void *y, int64_t ldy, int32_t y_dtype, int32_t *dev_status,
                        nvfp4_stream stream) {
    GemmArgs a;
    nvfp4_status st = gemm_args(A, B, bias_bf16, resid_bf16, y, ldy, y_dtype, false, dev_status, a);
    if (st != NVFP4_OK) return st;
    st = check_device();
    if (st != NVFP4_OK) return st;
    cudaError_t e = launch_gemm(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "nvfp4_gemm");
}

nvfp4_status nvfp4_gemm_quant_out(const nvfp4_tensor *A, const nvfp4_tensor *B, const void *bias_bf16,
                                  const void *resid_bf16, void *y_bf16, int64_t ldy, const float *amax_in,
                                  const nvfp4_tensor *q_out, void *ws, size_t ws_bytes, int32_t *dev_status,
                                  nvfp4_stream stream) {
    GemmArgs a;
    nvfp4_status st = gemm_args(A, B, bias_bf16, resid_bf16, y_bf16, ldy, NVFP4_OUT_BF16, true, dev_status, a);
    if (st != NVFP4_OK) return st;
    if (!amax_in || !ws || ws_bytes < kTensorScratchBytes) return NVFP4_ERR_INVALID_ARG;
    if (!tensor_ok(q_out, A->rows, B->rows)) return NVFP4_ERR_INVALID_ARG;
    if ((B->rows & 63) || !aligned16(q_out->codes) || !aligned16(q_out->sf) || !aligned16(ws))
        return NVFP4_ERR_UNSUPPORTED;
    st = check_device();
    if (st != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    ScaleRecord *rec = reinterpret_cast<ScaleRecord *>(static_cast<uint8_t *>(ws) + kRecordOffset);
    RecJobs rj{};
    rj.njobs = 1;
    rj.npartial = 0;
    rj.job[0].partial = nullptr;
    rj.job[0].amax_in = amax_in;
    rj.job[0].rec = rec;
    rj.job[0].g_out[0] = q_out->g;
    rj.job[0].g_out[1] = nullptr;
    a.q_rec = rec;
    a.q_codes = q_out->codes;
    a.q_sf = q_out->sf;
    a.q_pitch = codes_pitch(B->rows);
    a.q_sf_layout = q_out->sf_layout;
    a.q_codes_bytes = A->rows * a.q_pitch;
    a.q_sf_bytes = sf_bytes(A->rows, B->rows, q_out->sf_layout);
    cudaError_t e = launch_scale_record(rj, dev_status, s);
    if (e == cudaSuccess) e = launch_gemm(a, s);
    return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "nvfp4_gemm_quant_out");
}

size_t nvfp4_gemm_colamax_workspace(int64_t M, int64_t N) {
    if (M <= 0 || N <= 0) return 0;
    return (size_t)ceil_div(M, 32) * (size_t)ceil_div(N, 128) * sizeof(uint32_t);
}

nvfp4_status nvfp4_gemm_colamax(const nvfp4_tensor *A, const nvfp4_tensor *B, const void *bias_bf16,
                                const void *resid_bf16, void *y_bf16, int64_t ldy, int64_t group_cols,
                                float *amax_out, void *ws, size_t ws_bytes, int32_t *dev_status,
                                nvfp4_stream stream) {
    GemmArgs a;
    nvfp4_status st = gemm_args(A, B, bias_bf16, resid_bf16, y_bf16, ldy, NVFP4_OUT_BF16, false, dev_status, a);
    if (st != NVFP4_OK) return st;
    const int64_t M = A->rows, N = B->rows;
    if (!amax_out || !ws || group_cols <= 0 || ws_bytes < nvfp4_gemm_colamax_workspace(M, N))
        return NVFP4_ERR_INVALID_ARG;
    if ((group_cols & 255) || N % group_cols || !aligned16(ws)) return NVFP4_ERR_UNSUPPORTED;
    if (ceil_div(M, 32) * (group_cols / 128) >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED;   // finish indexing
    st = check_device();
    if (st != NVFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    a.cam_partial = static_cast<uint32_t *>(ws);
    a.cam_n128 = N / 128;
    a.cam_elems = ceil_div(M, 32) * (N / 128);
    cudaError_t e = launch_gemm(a, s);
    if (e == cudaSuccess)
        e = launch_colamax_finish(a.cam_partial, ceil_div(M, 32), N / 128, group_cols, N / group_cols, amax_out,
                                  dev_status, s);
    return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "nvfp4_gemm_colamax");
}

int64_t nvfp4_kv_cache_bytes(int32_t layers, int32_t heads, int32_t head_dim, int32_t slots, int32_t slot_tokens,
                             int32_t which) {
    if (layers <= 0 || heads <= 0 || head_dim <= 0 || slots <= 0 || slot_tokens <= 0) return -1;
    const int64_t row = (int64_t)heads * head_dim, n = (int64_t)layers * slots;
    switch (which) {
        case 0: return n * slot_tokens * (row / 2);
        case 1: return n * slot_tokens * (row / 16);
        case 2: return n * (int64_t)sizeof(float);
        default: return -1;
    }
}

static bool kv_ok(const nvfp4_kv_cache *c) {
    if (!c || c->layers <= 0 || c->heads <= 0 || c->head_dim <= 0 || c->slots <= 0 || c->slot_tokens <= 0) return false;
    if (!c->codes_k || !c->codes_v || !c->sf_k || !c->sf_v || !c->g_k || !c->g_v || !c->len) return false;
    return true;
}

nvfp4_status kv_quant_append(nvfp4_kv_cache *cache, int32_t layer, int32_t slot, const void *k_bf16,
                             const void *v_bf16, int64_t ntok, int64_t ld, void *ws, size_t ws_bytes,
                             int32_t *dev_status, nvfp4_stream stream) {
    return kv_quant_append_amax(cache, layer, slot, k_bf16, v_bf16, ntok, ld, nullptr, ws, ws_bytes, dev_status,
                                stream);
}

nvfp4_status kv_quant_append_amax(nvfp4_kv_cache *cache, int32_t layer, int32_t slot, const void *k_bf16,
                                  const void *v_bf16, int64_t ntok, int64_t ld, const float *amax_kv, void *ws,
                                  size_t ws_bytes, int32_t *dev_status, nvfp4_stream stream) {
    if (!kv_ok(cache) || !k_bf16 || !v_bf16 || !ws) return NVFP4_ERR_INVALID_ARG;
    if (layer < 0 || layer >= cache->layers || slot < 0 || slot >= cache->slots) return NVFP4_ERR_INVALID_ARG;
    const int64_t row = (int64_t)cache->heads * cache->head_dim;
    if (ntok <= 0 || ntok > cache->slot_tokens || ld < row) return NVFP4_ERR_INVALID_ARG;
    if (ws_bytes < nvfp4_kv_append_workspace(ntok, cache->heads, cache->head_dim)) return NVFP4_ERR_INVALID_ARG;
    if ((cache->head_dim & 15) || (row & 31) || (ld & 7) || too_large(ntok, row)) return NVFP4_ERR_UNSUPPORTED;
    if (!aligned16(k_bf16) || !aligned16(v_bf16) || !aligned16(ws) || !aligned16(cache->codes_k) ||
        !aligned16(cache->codes_v))
        return NVFP4_ERR_UNSUPPORTED;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    const int64_t slot_index = (int64_t)layer * cache->slots + slot;
    const int64_t tok0 = slot_index * cache->slot_tokens;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    RowJobs jobs{};
    jobs.njobs = 2;
    jobs.npartial = amax_blocks(ntok);
    RecJobs rj{};
    rj.njobs = 2;
    rj.npartial = jobs.npartial;
    for (int i = 0; i < 2; ++i) {
        uint8_t *scratch = static_cast<uint8_t *>(ws) + i * kTensorScratchBytes;
        RowJob &j = jobs.job[i];
        j.x = static_cast<const uint16_t *>(i == 0 ? k_bf16 : v_bf16);
        j.rows = ntok;
        j.cols = row;
        j.ld = ld;
        j.codes = (i == 0 ? cache->codes_k : cache->codes_v) + tok0 * (row / 2);
        j.pitch = row / 2;
        j.sf = (i == 0 ? cache->sf_k : cache->sf_v) + tok0 * (row / 16);
        j.sf_layout = NVFP4_SF_LINEAR;
        j.partial = reinterpret_cast<uint32_t *>(scratch);
        j.rec = reinterpret_cast<ScaleRecord *>(scratch + kRecordOffset);
        j.status = dev_status;
        j.x_elems = (ntok - 1) * ld + row;
        j.codes_bytes = ntok * (row / 2);
        j.sf_bytes = ntok * (row / 16);
        rj.job[i].partial = j.partial;
        rj.job[i].amax_in = amax_kv ? amax_kv + i : nullptr;
        rj.job[i].rec = reinterpret_cast<ScaleRecord *>(scratch + kRecordOffset);
        rj.job[i].g_out[0] = (i == 0 ? cache->g_k : cache->g_v) + slot_index;
        rj.job[i].g_out[1] = nullptr;
        if (amax_kv) {                                    // one launch: the row pass builds the record
            j.amax_in = amax_kv + i;
            j.g_out[0] = rj.job[i].g_out[0];
            j.report_record = 1;
        }
    }
    cudaError_t e = cudaSuccess;
    if (!amax_kv) {
        e = launch_amax(jobs, dev_status, nullptr, s);
        if (e == cudaSuccess) e = launch_scale_record(rj, dev_status, s);
        for (int i = 0; i < 2; ++i) jobs.job[i].x_early = 1;   // the amax pass read x after its wait
    }
    if (e == cudaSuccess) e = launch_quantize_rows(jobs, s);
    if (e != cudaSuccess) return cuda_fail(e, "kv_quant_append");
    cache->len[slot_index] = (int32_t)ntok;
    return NVFP4_OK;
}

nvfp4_status kv_dequant(const nvfp4_kv_cache *cache, int32_t layer, const int32_t *slots, int32_t nslots,
                        void *k_out_bf16, void *v_out_bf16, int32_t *dev_status, nvfp4_stream stream) {
    if (!kv_ok(cache) || !slots || !k_out_bf16 || !v_out_bf16) return NVFP4_ERR_INVALID_ARG;
    if (layer < 0 || layer >= cache->layers || nslots <= 0 || nslots > kMaxDequantSlots) return NVFP4_ERR_INVALID_ARG;
    const int64_t row = (int64_t)cache->heads * cache->head_dim;
    if ((cache->head_dim & 15) || (row & 31)) return NVFP4_ERR_UNSUPPORTED;
    if (!aligned16(k_out_bf16) || !aligned16(v_out_bf16) || !aligned16(cache->codes_k) ||
        !aligned16(cache->codes_v) || !aligned16(cache->sf_k) || !aligned16(cache->sf_v))
        return NVFP4_ERR_UNSUPPORTED;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    static thread_local DequantJob jk, jv;
    int64_t tok = 0;
    int32_t n = 0;
    for (int32_t i = 0; i < nslots; ++i) {
        const int32_t s = slots[i];
        if (s < 0 || s >= cache->slots) return NVFP4_ERR_INVALID_ARG;
        const int64_t slot_index = (int64_t)layer * cache->slots + s;
        const int32_t len = cache->len[slot_index];
        if (len < 0 || len > cache->slot_tokens) return NVFP4_ERR_INVALID_ARG;
        if (len == 0) continue;
        const int64_t tok0 = slot_index * cache->slot_tokens;
        jk.slot[n] = DequantSlot{cache->codes_k + tok0 * (row / 2), cache->sf_k + tok0 * (row / 16),
                                 cache->g_k + slot_index, tok, len};
        jv.slot[n] = DequantSlot{cache->codes_v + tok0 * (row / 2), cache->sf_v + tok0 * (row / 16),
                                 cache->g_v + slot_index, tok, len};
        tok += len;
        ++n;
    }
    if (n == 0) return NVFP4_OK;
    jk.nslots = jv.nslots = n;
    jk.total_tokens = jv.total_tokens = tok;
    jk.row_elems = jv.row_elems = row;
    jk.out = static_cast<uint16_t *>(k_out_bf16);
    jv.out = static_cast<uint16_t *>(v_out_bf16);
    jk.status = jv.status = dev_status;
    cudaError_t e = launch_kv_dequant(&jk, &jv, dev_status, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "kv_dequant");
}

nvfp4_status kv_attention(const nvfp4_kv_cache *cache, int32_t layer, const int32_t *slots, int32_t nslots,
                          const void *q_bf16, int64_t tq, int64_t ldq, float scale, void *o_bf16, int64_t ldo,
                          int32_t *dev_status, nvfp4_stream stream) {
    if (!kv_ok(cache) || !slots || tq < 0 || (tq > 0 && (!q_bf16 || !o_bf16)) || !std::isfinite(scale))
        return NVFP4_ERR_INVALID_ARG;
    if (layer < 0 || layer >= cache->layers || nslots <= 0 || nslots > kMaxDequantSlots) return NVFP4_ERR_INVALID_ARG;
    const int64_t row = (int64_t)cache->heads * cache->head_dim;
    if (ldq < row || ldo < row) return NVFP4_ERR_INVALID_ARG;
    if (cache->head_dim != 128 || cache->heads > 65535 || (ldq & 7) || (ldo & 7) || !aligned16(q_bf16) ||
        !aligned16(o_bf16) || !aligned16(cache->codes_k) || !aligned16(cache->codes_v) ||
        !aligned16(cache->sf_k) || !aligned16(cache->sf_v))
        return NVFP4_ERR_UNSUPPORTED;
    if (ceil_div(tq, 64) > 0x7FFFFFFF) return NVFP4_ERR_UNSUPPORTED;
    static thread_local AttnJob j;
    int64_t tok = 0;
    int32_t n = 0;
    for (int32_t i = 0; i < nslots; ++i) {
        const int32_t s = slots[i];
        if (s < 0 || s >= cache->slots) return NVFP4_ERR_INVALID_ARG;
        const int64_t slot_index = (int64_t)layer * cache->slots + s;
        const int32_t len = cache->len[slot_index];
        if (len < 0 || len > cache->slot_tokens) return NVFP4_ERR_INVALID_ARG;
        if (len == 0) continue;
        const int64_t tok0 = slot_index * cache->slot_tokens;
        j.slot[n] = AttnSlot{cache->codes_k + tok0 * (row / 2), cache->codes_v + tok0 * (row / 2),
                             cache->sf_k + tok0 * (row / 16), cache->sf_v + tok0 * (row / 16),
                             cache->g_k + slot_index, cache->g_v + slot_index, tok, len};
        tok += len;
        ++n;
    }
    if (tok == 0) return NVFP4_ERR_INVALID_ARG;           // attention over an empty window
    if (tq == 0) return NVFP4_OK;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    j.nslots = n;
    j.heads = cache->heads;
    j.total_tokens = tok;
    j.row_bytes = row / 2;
    j.row_sf = row / 16;
    j.q = static_cast<const uint16_t *>(q_bf16);
    j.ldq = ldq;
    j.tq = tq;
    j.o = static_cast<uint16_t *>(o_bf16);
    j.ldo = ldo;
    j.scale_log2 = (float)((double)scale * 1.4426950408889634);   // log2(e)
    j.q_elems = (tq - 1) * ldq + row;
    j.o_elems = (tq - 1) * ldo + row;
    cudaError_t e = launch_kv_attention(j, dev_status, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "kv_attention");
}

nvfp4_status nvfp4_encode_elements(const float *in, int64_t n, uint8_t *e2m1_out, uint8_t *e4m3_out,
                                   nvfp4_stream stream) {
    if (!in || n < 0) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    cudaError_t e = launch_encode_elements(in, n, e2m1_out, e4m3_out, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "nvfp4_encode_elements");
}

nvfp4_status nvfp4_selftest_wait_timeout(int32_t *dev_status, int64_t limit_ns, nvfp4_stream stream) {
    if (!dev_status || limit_ns <= 0 || limit_ns > 10000000000ll) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    cudaError_t e = launch_wait_timeout(dev_status, limit_ns, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "nvfp4_selftest_wait_timeout");
}

nvfp4_status nvfp4_selftest_bounds(uint8_t *buf, int64_t extent, int64_t index, int32_t *dev_status,
                                   nvfp4_stream stream) {
    if (!buf || extent < 0 || index < 0) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_device();
    if (st != NVFP4_OK) return st;
    cudaError_t e = launch_bounds_selftest(buf, extent, index, dev_status, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "nvfp4_selftest_bounds");
}

}  // extern "C"
