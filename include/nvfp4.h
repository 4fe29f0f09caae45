/*
 * nvfp4.h -- C ABI of the NVFP4 W4A4 linear-layer and NVFP4 KV-cache library (sm_100a / B200).
 *
 * The method: LongLive-2.0 ("An NVFP4 Parallel Infrastructure for Long Video Generation",
 * arXiv 2605.18739).  Its abstract (fugumt.com mirror) says that on Blackwell GPUs inference
 * runs "W4A4 NVFP4" linear layers and keeps the KV cache in NVFP4 for memory savings, and that
 * training accelerates its GEMMs with NVFP4; the d9249.github.io review (section
 * "핵심 아이디어 / 구조 / 동작 방식") adds that the cache is restored by a parallel dequantization
 * kernel, and the yourai.pro page lists in-place updates of the quantized cache and faster FP4
 * dequantization.  The pages do not define NVFP4 numerically; this library implements the
 * published NVFP4 format:
 *   - E2M1 element codes (values 0, 0.5, 1, 1.5, 2, 3, 4, 6 and their negatives), two per byte,
 *     the low nibble holding the even element, sign in bit 3 of each nibble;
 *   - one E4M3 (FN, max 448) scale per 16 consecutive elements of a row;
 *   - one FP32 per-tensor decode scale g = amax/2688 (g = 1 for an all-zero tensor);
 *   - FP32 op order per 16-block: sf = E4M3_rne_sat(b / (g*6)) with b the block's max |x|
 *     (sf = 0 when b = 0), d = sf*g, r = 1/d, code = E2M1_rne_sat(x*r) (all codes 0 when d = 0);
 *   - dequantization y = BF16_rne(FP32(E2M1*sf) * g).
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library never allocates,
 *     frees or synchronises.  Calls are asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).
 *   - The synchronous return value reports argument, shape, alignment, architecture (sm_100
 *     only) and launch errors.  Data-dependent errors are written to the optional device word
 *     `dev_status` (int32, caller zeroes it; the first non-zero code wins): NVFP4_ERR_NONFINITE
 *     for inf/NaN input (outputs then unspecified), NVFP4_ERR_TIMEOUT if a bounded on-chip wait
 *     gave up (the kernel returns instead of hanging).
 *   - Pointers must be 16-byte aligned; BF16 row strides must be multiples of 8 elements.
 *
 * Layouts:
 *   codes: [rows][nvfp4_codes_pitch(cols)] bytes; each row padded with zero codes to a multiple
 *          of 32 elements (16 bytes).
 *   scales, NVFP4_SF_LINEAR: [rows][ceil(cols/16)] bytes.
 *   scales, NVFP4_SF_MMA: the tcgen05 block-scaling layout: rows padded to 128 and scale
 *          columns to 4 (padding zero), 512-byte atoms of 128 rows x 4 scales ordered
 *          scale-column fastest; scale (i, b) sits at
 *          ((i/128)*ceil(ceil(cols/16)/4) + b/4)*512 + (i%32)*16 + ((i%128)/32)*4 + b%4.
 *          GEMM operands must use this layout.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,  /* null pointer, negative size, inconsistent shapes */
    NVFP4_ERR_UNSUPPORTED = 2,  /* alignment, stride, layout or GPU architecture not supported */
    NVFP4_ERR_NONFINITE = 3,    /* device side: inf/NaN in the input */
    NVFP4_ERR_TIMEOUT = 4,      /* device side: a bounded wait gave up */
    NVFP4_ERR_CUDA = 5,         /* a CUDA runtime/driver call failed */
    NVFP4_ERR_OUT_OF_BOUNDS = 6 /* device side, checked build only: an access outside its buffer
                                   was skipped (see nvfp4_checked_build) */
} nvfp4_status;

typedef enum { NVFP4_ROWWISE = 0, NVFP4_COLWISE = 1, NVFP4_ROWCOL = 2 } nvfp4_dir;
typedef enum { NVFP4_SF_LINEAR = 0, NVFP4_SF_MMA = 1 } nvfp4_sf_layout;
typedef enum { NVFP4_OUT_BF16 = 0, NVFP4_OUT_F32 = 1 } nvfp4_out_dtype;

typedef void *nvfp4_stream; /* cudaStream_t */

/* A quantized matrix of `rows` x `cols` logical elements.  All pointers are device memory. */
typedef struct {
    uint8_t *codes;    /* [rows][nvfp4_codes_pitch(cols)] */
    uint8_t *sf;       /* nvfp4_sf_bytes(rows, cols, sf_layout) bytes */
    float *g;          /* one float: the per-tensor decode scale */
    int64_t rows, cols;
    int32_t sf_layout; /* nvfp4_sf_layout */
} nvfp4_tensor;

/* Chunk-slot NVFP4 KV cache.  Per layer there are `slots` chunk slots of `slot_tokens` tokens;
 * K and V are stored separately, each token row of heads*head_dim elements quantized row-wise
 * with 16-blocks along head_dim (8 scales per head for head_dim 128) and LINEAR scales, and one
 * per-tensor scale g per (layer, slot) for K and for V.  Storage is caller-owned:
 *   codes_k/v: [layers][slots][slot_tokens][heads*head_dim/2] bytes      (device)
 *   sf_k/v:    [layers][slots][slot_tokens][heads*head_dim/16] bytes     (device)
 *   g_k/v:     [layers][slots] floats                                    (device)
 *   len:       [layers][slots] int32 tokens held per slot                (HOST; written by
 *              kv_quant_append, read by kv_dequant and kv_attention)
 * Ordering: `len` is host bookkeeping, read and written when a call is ENQUEUED, not when its
 * kernels run.  kv_quant_append sets len[slot] before it returns, i.e. before the slot's bytes
 * exist on the device; a later kv_dequant / kv_attention sizes its launch from it at once.  So
 * a call that reads a slot must be enqueued after the append that wrote it, on the same stream
 * or on a stream that waits for an event recorded after the append.  An append that returns an
 * error leaves len unchanged. */
typedef struct {
    int32_t layers, heads, head_dim, slots, slot_tokens;
    uint8_t *codes_k, *codes_v;
    uint8_t *sf_k, *sf_v;
    float *g_k, *g_v;
    int32_t *len;
} nvfp4_kv_cache;

/* ---- sizes ---------------------------------------------------------------------------------- */

/* Bytes of one packed code row: 16 * ceil(cols / 32). */
NVFP4_API int64_t nvfp4_codes_pitch(int64_t cols);

/* Bytes of the scale array of a rows x cols matrix in `layout`; -1 on bad arguments. */
NVFP4_API int64_t nvfp4_sf_bytes(int64_t rows, int64_t cols, int32_t layout);

/* Scale layout conversion on HOST memory (no device work), e.g. to read the tensor-core scale
 * layout of a GEMM operand as a plain table.
 * nvfp4_sf_to_linear: sf_mma (nvfp4_sf_bytes(rows, cols, NVFP4_SF_MMA) bytes) -> sf_linear
 * ([rows][ceil(cols/16)] bytes); the layout's padding is dropped.
 * nvfp4_sf_to_mma: the inverse, with the padding rows and scale columns written as zero.
 * NVFP4_ERR_INVALID_ARG on a NULL pointer or rows, cols <= 0. */
NVFP4_API nvfp4_status nvfp4_sf_to_linear(const uint8_t *sf_mma, int64_t rows, int64_t cols, uint8_t *sf_linear);
NVFP4_API nvfp4_status nvfp4_sf_to_mma(const uint8_t *sf_linear, int64_t rows, int64_t cols, uint8_t *sf_mma);

/* Bytes of device workspace nvfp4_quantize / nvfp4_amax need (per-CTA partial maxima and the
 * per-tensor scale record; 5 KB). */
NVFP4_API size_t nvfp4_quantize_workspace(int64_t rows, int64_t cols);

/* Bytes of device workspace kv_quant_append needs (the same, for K and for V). */
NVFP4_API size_t nvfp4_kv_append_workspace(int64_t ntok, int32_t heads, int32_t head_dim);

/* ---- the four calls of the path ------------------------------------------------------------- */

/*
 * Per-tensor absolute maximum of a BF16 [M, K] matrix (row stride ld elements) written to the
 * device float *amax_out.  Deterministic (max is order independent).  Optional first pass of
 * nvfp4_quantize, exposed so callers can reuse one amax (amax_in) across several quantizations
 * of the same tensor (row- and column-wise).  Requires ws of nvfp4_quantize_workspace(M, K)
 * bytes.  Non-finite input sets NVFP4_ERR_NONFINITE in *dev_status.
 */
NVFP4_API nvfp4_status nvfp4_amax(const void *x_bf16, int64_t M, int64_t K, int64_t ld, float *amax_out,
                        void *ws, size_t ws_bytes, int32_t *dev_status, nvfp4_stream stream);

/*
 * nvfp4_quantize -- BF16 [M, K] (row stride ld elements, K % 8 == 0) to NVFP4.
 * Defining passage: the LongLive-2.0 arXiv abstract (fugumt.com page) -- the linear layers run
 * "W4A4 NVFP4" in inference and NVFP4 GEMMs in training, so every activation (and, once, every
 * weight) is quantized to NVFP4; the d9249.github.io review, section "핵심 아이디어 / 구조 / 동작
 * 방식", for NVFP4 training and W4A4 inference.  The numeric format is the published NVFP4 one
 * (top of this file); the pages do not define it.
 *   dir = NVFP4_ROWWISE: 16-blocks along K (the contiguous dim); out->rows = M, out->cols = K.
 *         Requires K % 16 == 0.
 *   dir = NVFP4_COLWISE: 16-blocks along M (the token dim), i.e. the row-wise quantization of
 *         x^T, as needed for the wgrad/dgrad operands of NVFP4 training GEMMs; out->rows = K,
 *         out->cols = M; a trailing partial block (M % 16 != 0) is zero-padded.
 *   dir = NVFP4_ROWCOL: both layouts with one amax in one call: `out` points to two tensors,
 *         out[0] row-wise ([M, K]) and out[1] column-wise ([K, M]).  Requires K % 16 == 0.
 * amax_in: nullable DEVICE pointer to a precomputed amax of x (from nvfp4_amax); when NULL a
 * first pass computes it.  out->g receives g; out->sf uses out->sf_layout.  All padding bytes of
 * codes and scales are written (zero).  ws: nvfp4_quantize_workspace(M, K) bytes of device
 * memory (16-byte aligned, no initialisation needed), required in every call: it holds the
 * amax partials and the per-tensor scale record.  (M + 128) * (K + 128) must be below 2^35,
 * else NVFP4_ERR_UNSUPPORTED.
 */
NVFP4_API nvfp4_status nvfp4_quantize(const void *x_bf16, int64_t M, int64_t K, int64_t ld, int32_t dir,
                            const float *amax_in, const nvfp4_tensor *out, void *ws,
                            size_t ws_bytes, int32_t *dev_status, nvfp4_stream stream);

/*
 * Defining passage: the LongLive-2.0 arXiv abstract (fugumt.com page) -- W4A4 NVFP4 linear layers
 * in inference and NVFP4-accelerated GEMMs in training, whose share of the DiT's work grows with
 * video length (d9249.github.io review, section "핵심 아이디어 / 구조 / 동작 방식", and its
 * Table 1 training times).
 * nvfp4_gemm -- Y[M, N] = alpha * A . B^T (+ bias[n] | + resid[m, n]), alpha = gA * gB, with
 * A = [M, K] and B = [N, K] NVFP4 (both K-major, scales in NVFP4_SF_MMA layout) and FP32
 * accumulation in tensor memory (tcgen05 block-scaled MMA, kind::mxf4nvf4).  Epilogue in FP32:
 * t = alpha*acc; t = t + bias[n] (or + resid[m*ldy + n]); then BF16 round-to-nearest-even
 * (y_dtype NVFP4_OUT_BF16) or stored as FP32 (NVFP4_OUT_F32, for accuracy checks).
 * bias_bf16: nullable [N]; resid_bf16: nullable [M, ldy], may alias y (in-place residual).
 * At most one of bias/resid.  Requires N % 8 == 0 and ldy % 8 == 0.
 */
NVFP4_API nvfp4_status nvfp4_gemm(const nvfp4_tensor *A, const nvfp4_tensor *B, const void *bias_bf16,
                        const void *resid_bf16, void *y, int64_t ldy, int32_t y_dtype,
                        int32_t *dev_status, nvfp4_stream stream);

/*
 * nvfp4_gemm_quant_out -- nvfp4_gemm whose epilogue also emits the row-wise NVFP4 quantization
 * of its BF16 output Y (the next linear layer's A operand in a W4A4 network), with the
 * per-tensor scale fixed in advance: g = amax_in / 2688 (amax_in: DEVICE float, e.g. the amax of
 * the previous step's output; values above it saturate).  q_out (rows = M, cols = N, either
 * scale layout) receives exactly nvfp4_quantize(Y, NVFP4_ROWWISE, amax_in) of the BF16 Y this
 * call computes, codes and scales including all padding; q_out->g receives g.  y_bf16 may be
 * NULL (then only q_out is written; ldy is used for resid_bf16 only).  Requires N % 64 == 0, the
 * nvfp4_gemm requirements otherwise, and ws of nvfp4_quantize_workspace bytes (the scale record).
 * A non-finite amax_in sets NVFP4_ERR_NONFINITE in *dev_status and leaves q_out unwritten.
 * It fuses the activation quantization of the W4A4 path (LongLive-2.0 abstract: NVFP4 linear
 * layers in training and inference) into the producing GEMM.
 */
NVFP4_API nvfp4_status nvfp4_gemm_quant_out(const nvfp4_tensor *A, const nvfp4_tensor *B, const void *bias_bf16,
                                  const void *resid_bf16, void *y_bf16, int64_t ldy, const float *amax_in,
                                  const nvfp4_tensor *q_out, void *ws, size_t ws_bytes, int32_t *dev_status,
                                  nvfp4_stream stream);

/*
 * nvfp4_gemm_colamax -- nvfp4_gemm (BF16 output) whose epilogue also reduces max |Y| of the BF16
 * output over column groups of group_cols columns: amax_out[g] (DEVICE float[N / group_cols]) =
 * max |Y[:, g*group_cols : (g+1)*group_cols]|, exact (a max of the stored BF16 values), e.g. the
 * amax of the K and V slices of a fused QKV projection.  Requires group_cols % 256 == 0,
 * N % group_cols == 0, and ws of nvfp4_gemm_colamax_workspace(M, N) bytes (per-block partial
 * maxima; no initialisation needed); NVFP4_ERR_UNSUPPORTED when a group holds 2^31 or more of
 * those partials (ceil(M / 32) * group_cols / 128).  inf/NaN in a group sets NVFP4_ERR_NONFINITE
 * and stores NaN.
 */
NVFP4_API size_t nvfp4_gemm_colamax_workspace(int64_t M, int64_t N);
NVFP4_API nvfp4_status nvfp4_gemm_colamax(const nvfp4_tensor *A, const nvfp4_tensor *B, const void *bias_bf16,
                                const void *resid_bf16, void *y_bf16, int64_t ldy, int64_t group_cols,
                                float *amax_out, void *ws, size_t ws_bytes, int32_t *dev_status,
                                nvfp4_stream stream);

/* Bytes of each cache array: which = 0 codes (one of K/V), 1 scales (one of K/V), 2 g (one of
 * K/V); -1 on bad arguments. */
NVFP4_API int64_t nvfp4_kv_cache_bytes(int32_t layers, int32_t heads, int32_t head_dim, int32_t slots,
                             int32_t slot_tokens, int32_t which);

/*
 * Defining passage: the LongLive-2.0 arXiv abstract (fugumt.com page) keeps the KV cache in NVFP4
 * to cut memory (Table 3 of the paper, as the d9249.github.io review reports it: 29.7 -> 19.4 GB);
 * the yourai.pro report lists in-place updates of the quantized cache data.
 * kv_quant_append -- quantize one chunk's K and V ([ntok, heads*head_dim] BF16, row stride ld
 * elements; e.g. slices of a fused QKV GEMM output) into slot `slot` of layer `layer`, in place:
 * nothing else in the cache is touched and older slots are never re-quantized.  Each of K and V
 * gets its own per-tensor scale (g_k/g_v[layer*slots + slot]).  Sets cache->len[layer*slots +
 * slot] = ntok (host).  Requires ntok <= slot_tokens, head_dim % 16 == 0, ws of
 * nvfp4_kv_append_workspace bytes, (ntok + 128) * (heads * head_dim + 128) below 2^35.
 */
NVFP4_API nvfp4_status kv_quant_append(nvfp4_kv_cache *cache, int32_t layer, int32_t slot,
                             const void *k_bf16, const void *v_bf16, int64_t ntok, int64_t ld,
                             void *ws, size_t ws_bytes, int32_t *dev_status,
                             nvfp4_stream stream);

/*
 * kv_quant_append_amax -- kv_quant_append with the amax of K and of V given (amax_kv: DEVICE
 * float[2], K then V; e.g. from nvfp4_gemm_colamax of the GEMM that produced them), so no amax
 * pass reads K and V.  With the exact amax of the chunk the cache bytes equal kv_quant_append's.
 * A non-finite amax sets NVFP4_ERR_NONFINITE in *dev_status and leaves the slot unwritten.
 */
NVFP4_API nvfp4_status kv_quant_append_amax(nvfp4_kv_cache *cache, int32_t layer, int32_t slot,
                                  const void *k_bf16, const void *v_bf16, int64_t ntok, int64_t ld,
                                  const float *amax_kv, void *ws, size_t ws_bytes, int32_t *dev_status,
                                  nvfp4_stream stream);

/*
 * Defining passage: the d9249.github.io review, section "핵심 아이디어 / 구조 / 동작 방식" -- the
 * NVFP4 KV cache is restored by a parallel dequantization kernel to lower the restore cost; the
 * yourai.pro report lists faster FP4 dequantization among the inference-path optimizations.
 * kv_dequant -- parallel restore of a window of slots of one layer to BF16: the listed slots
 * (host array `slots`, nslots <= 128, in the given order) are dequantized and concatenated
 * token-wise into k_out / v_out ([sum of len, heads, head_dim] BF16, contiguous).
 */
NVFP4_API nvfp4_status kv_dequant(const nvfp4_kv_cache *cache, int32_t layer, const int32_t *slots,
                        int32_t nslots, void *k_out_bf16, void *v_out_bf16, int32_t *dev_status,
                        nvfp4_stream stream);

/*
 * kv_attention -- softmax attention of BF16 queries over a window of NVFP4 cache slots, with the
 * restore fused into the kernel's K/V tile loads: the window's BF16 K and V never reach HBM.
 * LongLive-2.0 restores its NVFP4 KV cache for attention with a parallel dequantization kernel
 * (d9249.github.io review, section "핵심 아이디어 / 구조 / 동작 방식"); this call computes the
 * same attention without the restored copy.  For every head h and query row i:
 *   O[i, h, :] = sum_j softmax_j(scale * q[i, h, :] . k[j, h, :]) v[j, h, :]
 * over the tokens j of the listed slots (host array `slots`, nslots <= 128, layer `layer`). k and
 * v are the values kv_dequant restores, BF16(FP32(e2m1 * sf) * g). The slot order changes only
 * the summation order. No mask.
 *   q:  [tq, heads, head_dim] BF16 (DEVICE), token row stride ldq elements (e.g. the Q third of
 *       a fused QKV GEMM output, ldq = 3 * heads * head_dim);
 *   o:  [tq, heads, head_dim] BF16 (DEVICE), token row stride ldo elements; must not overlap q;
 *   scale: the softmax scale (commonly 1 / sqrt(head_dim)), finite.
 * Requires head_dim == 128, ldq and ldo >= heads * head_dim and multiples of 8, q and o 16-byte
 * aligned, a window of at least one token (else NVFP4_ERR_INVALID_ARG / NVFP4_ERR_UNSUPPORTED).
 * tq == 0 is a no-op. Scores must stay finite in FP32 (|scale * q.k| < 2^127) for a finite
 * result.  dev_status (nullable): the kernel's on-chip waits are time-bounded, and one that gives
 * up writes NVFP4_ERR_TIMEOUT there (the output is then unspecified).
 * Arithmetic (tcgen05 tensor cores): FP32 scores and output accumulation in tensor memory, the
 * probabilities 2^(scale * log2(e) * s - max) from the hardware exp2 approximation (results below
 * 2^-126 flush to 0) rounded to BF16 for the P.V product, the row sums in FP32, the output
 * rounded to BF16 (nearest even).
 */
NVFP4_API nvfp4_status kv_attention(const nvfp4_kv_cache *cache, int32_t layer, const int32_t *slots,
                                    int32_t nslots, const void *q_bf16, int64_t tq, int64_t ldq, float scale,
                                    void *o_bf16, int64_t ldo, int32_t *dev_status, nvfp4_stream stream);

/*
 * nvfp4_quantize_noalloc -- nvfp4_quantize without a workspace: for callers that cannot
 * allocate, such as plugin/enqueue hooks of inference engines and embedded host programs that
 * receive only their input and output buffers and have no allocator or workspace to hand over.
 * No counterpart in the paper: it is a deployment variant of the quantizer above.
 * Accepts dir = NVFP4_ROWWISE or NVFP4_COLWISE only (NVFP4_ROWCOL returns
 * NVFP4_ERR_INVALID_ARG) and a single output tensor `out`; otherwise the same arguments, layouts
 * and results as nvfp4_quantize with amax_in = NULL, bit for bit.  The amax partial maxima and
 * the scale record go to a 5 KB static device array held by every GPU that loads the library.
 * Nothing is allocated.  The amax pass never launches more than 1024 CTAs, so every shape fits
 * the array's 1024 partial slots.  All calls share the array: calls whose kernels overlap on the
 * GPU race and must be ordered on one stream.  The first call on each device looks up the
 * array's device address and caches it for the life of the process; make that first call before
 * any stream capture.  The cache assumes the device's primary context is never reset
 * (cudaDeviceReset) while the library is loaded.
 */
NVFP4_API nvfp4_status nvfp4_quantize_noalloc(const void *x_bf16, int64_t M, int64_t K, int64_t ld, int32_t dir,
                                              const nvfp4_tensor *out, int32_t *dev_status,
                                              nvfp4_stream stream);

/* ---- support --------------------------------------------------------------------------------- */

/* Static description of a status code. */
NVFP4_API const char *nvfp4_status_string(int32_t status);

/* Last CUDA error text recorded by a call that returned NVFP4_ERR_CUDA (per thread). */
NVFP4_API const char *nvfp4_last_error(void);

/* Library ABI version (major*100 + minor). */
NVFP4_API int32_t nvfp4_version(void);

/*
 * 1 for the bounds-checked debug build (libnvfp4_checked.so, compiled with NVFP4_DEBUG_CHECKS),
 * 0 for the release build.  In the checked build every kernel access whose address is computed
 * from indexes is compared with the extent of its buffer, derived on the host from the caller's
 * tensor shapes; an access outside it is skipped and NVFP4_ERR_OUT_OF_BOUNDS is written to the
 * status word instead (no trap, the CUDA context stays usable).  TMA tensor loads and stores are
 * bounded by their tensor maps and need no check.  Same ABI and results otherwise; slower.
 */
NVFP4_API int32_t nvfp4_checked_build(void);

/*
 * Test support: element-wise hardware encoders of the CUDA path on n FP32 inputs:
 * e2m1_out[i] = E2M1 code of in[i] as the quantizer computes it, e4m3_out[i] = E4M3 byte of
 * |in[i]| as the scale step computes it (either output may be NULL).  Device pointers.
 */
NVFP4_API nvfp4_status nvfp4_encode_elements(const float *in, int64_t n, uint8_t *e2m1_out,
                                   uint8_t *e4m3_out, nvfp4_stream stream);

/*
 * Test support: run one bounded on-chip wait on a barrier that nothing completes, with a limit
 * of `limit_ns` nanoseconds; the kernel must give up, write NVFP4_ERR_TIMEOUT to *dev_status
 * and return.  Exercises the timeout path without hanging the GPU.
 */
NVFP4_API nvfp4_status nvfp4_selftest_wait_timeout(int32_t *dev_status, int64_t limit_ns,
                                         nvfp4_stream stream);

/*
 * Test support for the checked build: one device thread writes 0xAB to buf[index] if index lies
 * inside [0, extent) -- in the checked build that comparison is the library's bounds check, which
 * skips the write and sets NVFP4_ERR_OUT_OF_BOUNDS in *dev_status otherwise; the release build
 * writes unconditionally.  The caller's buffer must hold index + 1 bytes either way (the test
 * declares a smaller extent than it allocates), so no call of it can write outside memory.
 */
NVFP4_API nvfp4_status nvfp4_selftest_bounds(uint8_t *buf, int64_t extent, int64_t index, int32_t *dev_status,
                                             nvfp4_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
