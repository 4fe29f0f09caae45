// noalloc.cu -- nvfp4_quantize_noalloc: the quantizer for callers that cannot allocate.
//
// nvfp4_quantize needs a small device workspace for the per-CTA partial maxima of its amax
// pass and the per-tensor scale record.  Some callers have no way to provide one: plugin or enqueue hooks of inference engines
// and embedded host programs that receive only their input and output buffers and have neither
// an allocator nor a workspace to hand over (and must not call cudaMalloc on their hot path).
// This entry point keeps that scratch in a file-scope device array instead, so the caller
// passes inputs and outputs only and nothing is allocated.
//
// Contract:
//   - The scratch is 5 KB of static device memory (1024 32-bit partial slots and one scale
//     record), held by every GPU that loads the library until the process exits.
//   - A call needs one slot per CTA of the amax pass, whose grid is capped at 1024 CTAs, so
//     every shape fits.  A failed CUDA call returns NVFP4_ERR_CUDA with a message in
//     nvfp4_last_error().
//   - All calls share the one array and it keeps the last call's contents.  Nothing in it needs
//     to start at zero: each call's amax pass writes every slot its record kernel reads, and the
//     record kernel writes the whole record its quantize pass reads.  Calls
//     whose kernels overlap on the GPU (different streams without ordering, several host
//     threads) race on the array and give wrong results; order them on one stream.
//   - The first call on each device looks up the array's device address (cudaGetSymbolAddress,
//     with that device current) and caches it; make that first call before any stream capture.
//     The cached address stays valid as long as the device's primary context lives: a caller
//     that resets the device (cudaDeviceReset) must not call this entry point afterwards.
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace nvfp4 {

namespace {

constexpr int kNoAllocPartials = 1024;
static_assert(kNoAllocPartials >= kMaxPartials, "scratch must hold a full amax pass");
static_assert(kNoAllocPartials * sizeof(uint32_t) == kRecordOffset, "partials, then the record");

static __device__ __align__(256) uint8_t g_noalloc_scratch[kTensorScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
uint8_t *g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up once per device).
cudaError_t scratch_for_current_device(uint8_t **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = static_cast<uint8_t *>(p);
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

nvfp4_status nvfp4_quantize_noalloc(const void *x_bf16, int64_t M, int64_t K, int64_t ld, int32_t dir,
                                    const nvfp4_tensor *out, int32_t *dev_status, nvfp4_stream stream) {
    if (!x_bf16 || !out || !out->codes || !out->sf || !out->g || M <= 0 || K <= 0 || ld < K)
        return NVFP4_ERR_INVALID_ARG;
    if (dir != NVFP4_ROWWISE && dir != NVFP4_COLWISE) return NVFP4_ERR_INVALID_ARG;
    if (out->sf_layout != NVFP4_SF_LINEAR && out->sf_layout != NVFP4_SF_MMA) return NVFP4_ERR_INVALID_ARG;
    const int64_t orows = dir == NVFP4_ROWWISE ? M : K, ocols = dir == NVFP4_ROWWISE ? K : M;
    if (out->rows != orows || out->cols != ocols) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(x_bf16) || (ld & 7) || (K & 7)) return NVFP4_ERR_UNSUPPORTED;
    if ((uint64_t)(M + 128) * (uint64_t)(K + 128) >= (1ull << 35)) return NVFP4_ERR_UNSUPPORTED;   // 32-bit unit indexing
    if (dir == NVFP4_ROWWISE && (K & 15)) return NVFP4_ERR_UNSUPPORTED;
    if (!aligned16(out->codes)) return NVFP4_ERR_UNSUPPORTED;
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (major != 10 || minor != 0) return NVFP4_ERR_UNSUPPORTED;

    const int npartial = amax_blocks(M);
    if (npartial > kNoAllocPartials) {   // static guard: amax_blocks() never exceeds kMaxPartials
        char msg[160];
        std::snprintf(msg, sizeof(msg),
                      "nvfp4_quantize_noalloc: the amax pass needs %d scratch slots, the static scratch holds %d",
                      npartial, kNoAllocPartials);
        record_error(msg);
        return NVFP4_ERR_UNSUPPORTED;
    }
    uint8_t *scratch = nullptr;
    cudaError_t e = scratch_for_current_device(&scratch);
    if (e != cudaSuccess) {
        char msg[160];
        std::snprintf(msg, sizeof(msg), "nvfp4_quantize_noalloc: scratch lookup: %s", cudaGetErrorString(e));
        record_error(msg);
        return NVFP4_ERR_CUDA;
    }

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    RowJobs jobs{};
    jobs.njobs = 1;
    jobs.npartial = npartial;
    RowJob &j = jobs.job[0];
    j.x = static_cast<const uint16_t *>(x_bf16);
    j.rows = M;
    j.cols = K;
    j.ld = ld;
    j.codes = out->codes;
    j.pitch = 16 * ceil_div(ocols, 32);
    j.sf = out->sf;
    j.sf_layout = out->sf_layout;
    j.partial = reinterpret_cast<uint32_t *>(scratch);
    j.rec = reinterpret_cast<ScaleRecord *>(scratch + kRecordOffset);
    j.status = dev_status;
    j.x_elems = (M - 1) * ld + K;
    j.codes_bytes = orows * j.pitch;
    j.sf_bytes = out->sf_layout == NVFP4_SF_MMA ? 128 * ceil_div(orows, 128) * 4 * ceil_div(ceil_div(ocols, 16), 4)
                                                : orows * ceil_div(ocols, 16);
    RecJobs rj{};
    rj.njobs = 1;
    rj.npartial = npartial;
    rj.job[0].partial = j.partial;
    rj.job[0].amax_in = nullptr;
    rj.job[0].rec = reinterpret_cast<ScaleRecord *>(scratch + kRecordOffset);
    rj.job[0].g_out[0] = out->g;
    rj.job[0].g_out[1] = nullptr;
    e = launch_amax(jobs, dev_status, nullptr, s);
    if (e == cudaSuccess) e = launch_scale_record(rj, dev_status, s);
    if (e == cudaSuccess) e = dir == NVFP4_ROWWISE ? launch_quantize_rows(jobs, s) : launch_quantize_cols(j, false, s);
    if (e != cudaSuccess) {
        char msg[160];
        std::snprintf(msg, sizeof(msg), "nvfp4_quantize_noalloc: %s", cudaGetErrorString(e));
        record_error(msg);
        return NVFP4_ERR_CUDA;
    }
    return NVFP4_OK;
}

}  // extern "C"
