/*
 * mxq.h - C ABI of the microscaled (NVFP4 / MXFP8) linear layer for B200.
 *
 * The operation (B200 MXFP8/NVFP4 diffusion article, "Detailed by section"
 * and "Glossary"): a diffusion transformer's nn.Linear layers run as
 *   1. dynamic quantisation of the bf16 activation X [M,K] on every call, to
 *      NVFP4 (E2M1 codes, 16-element blocks, E4M3 block scale, fp32
 *      per-tensor scale from the tensor's amax) or MXFP8 (E4M3 codes,
 *      32-element blocks, E8M0 power-of-two scale);  weights W [N,K] are
 *      quantised once, the same way;
 *   2. a block-scaled GEMM Y = X W^T (+ bias) on the tensor cores, bf16 out;
 *   3. selective quantisation: a layer with min(M,K,N) < 1024, or flagged as
 *      accuracy-sensitive, stays a plain bf16 GEMM.
 *
 * Conventions for every call below.
 *   - Memory: every pointer named *_dev, and every data pointer, is CUDA
 *     device memory owned by the caller.  The library never allocates or
 *     frees and keeps no per-call state.  Scalars that the GPU produces
 *     (amax, per-tensor scales) stay on the device, so no call synchronises
 *     the host with the GPU except mxq_get_device_error.
 *   - Layout: bf16 matrices are row-major with a leading dimension `ld` in
 *     elements (ld >= k, ld a multiple of 8).  Codes are row-major, K-fastest:
 *     NVFP4 [rows][k/2] bytes with element 2j in the low nibble of byte j;
 *     MXFP8 [rows][k] bytes.  Scale factors use the tensor-core block-scaling
 *     layout (tiles of 128 rows x 4 scale columns = 512 bytes; inside a tile,
 *     byte (r%32)*16 + ((r/32)%4)*4 + (c%4); tiles ordered row-block-major,
 *     tile = (r/128)*ceil(C/4) + c/4; rows padded to 128 and columns to 4
 *     with zero bytes), C = k/16 (NVFP4) or k/32 (MXFP8).
 *   - Alignment: every data pointer 16-byte aligned.
 *   - Streams: work is enqueued on `stream` (NULL = the legacy default
 *     stream) and returns immediately.
 *   - Errors: arguments, shapes, alignment and the device architecture
 *     (sm_100 family) are checked on the host before anything is enqueued; on
 *     failure the call returns a non-zero status and enqueues nothing.  A
 *     failed launch returns MXQ_ERR_CUDA.  Every wait inside a kernel is
 *     bounded; a wait that runs out records MXQ_ERR_TIMEOUT in a device error
 *     word and the kernel returns early, which mxq_get_device_error reports.
 *   - Empty problems (rows, M or N equal to 0) are valid and enqueue nothing.
 */
#ifndef MXQ_H_
#define MXQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st* mxq_stream_t;

typedef enum mxq_status {
  MXQ_OK = 0,
  MXQ_ERR_INVALID_ARG = 1,       /* NULL pointer, negative size, bad enum    */
  MXQ_ERR_ALIGNMENT = 2,         /* pointer or leading dimension misaligned  */
  MXQ_ERR_UNSUPPORTED_SHAPE = 3, /* k not a multiple of the block rule       */
  MXQ_ERR_WORKSPACE = 4,         /* workspace / storage smaller than needed  */
  MXQ_ERR_ARCH = 5,              /* no CUDA device, or not an sm_100 device  */
  MXQ_ERR_CUDA = 6,              /* a CUDA runtime/driver call failed        */
  MXQ_ERR_TIMEOUT = 7            /* a bounded device-side wait ran out       */
} mxq_status;

typedef enum mxq_format {
  MXQ_NVFP4 = 1,
  MXQ_MXFP8 = 2,
  MXQ_BF16 = 3
} mxq_format;

/* Human-readable name of a status code (static string). */
const char* mxq_status_string(mxq_status s);

/* ABI version: (major << 16) | minor. */
int mxq_version(void);

/* Last CUDA error code seen by the calling thread's library calls (0 = none). */
int mxq_last_cuda_error(void);

/* ---------------------------------------------------------------- sizes -- */

/* Bytes of the swizzled scale-factor array of a [rows, k] tensor:
 * pad128(rows) * pad4(k / block), block = 16 (NVFP4) or 32 (MXFP8); 0 for
 * MXQ_BF16 or an invalid format. */
size_t mxq_sf_bytes(int64_t rows, int64_t k, mxq_format f);

/* Bytes of the element codes of a [rows, k] tensor: rows*k/2 (NVFP4),
 * rows*k (MXFP8), rows*k*2 (BF16). */
size_t mxq_codes_bytes(int64_t rows, int64_t k, mxq_format f);

/* ------------------------------------------------------ quantisation ---- */

/*
 * mxq_amax - global max |x| of a bf16 matrix X [rows, k] (leading dim ld).
 * Source: NVFP4's dynamic per-tensor scale is computed from the tensor's amax
 * on every call (the article's TorchAO listing, use_dynamic_per_tensor_scale).
 * Output: *amax_dev (fp32, device) = max |x| (exact).  The call overwrites it
 * (it zeroes it first on `stream`).  rows*k == 0 writes 0.
 * Errors: NULL x (with rows*k > 0) or amax_dev, negative sizes, ld < k or ld
 * not a multiple of 8 -> INVALID_ARG / ALIGNMENT.
 */
mxq_status mxq_amax(const void* x_bf16, int64_t rows, int64_t k, int64_t ld,
                    float* amax_dev, mxq_stream_t stream);

/*
 * mxq_quantize_nvfp4 - NVFP4 quantisation of X [rows, k] (article, Glossary
 * "NVFP4" and "Microscaling Formats"; per-tensor scale from amax).
 *   g = amax / 2688 (fp32; 1 when amax == 0) is written to *g_dev;
 *   per 16-element block: sf = E4M3(bamax / (6 g)), s = value(sf) * g,
 *   code = E2M1(x * (1/s)) (0 when s == 0); all fp32, round-to-nearest-even,
 *   saturating, sign kept.
 * Inputs: x_bf16 [rows][ld]; amax_dev: fp32 amax of the tensor (device),
 *   usually from mxq_amax (it may be any amax the caller chooses, e.g. a
 *   reduction over shards).  amax_dev == NULL selects NVFP4 without a
 *   per-tensor scale (the listing's use_dynamic_per_tensor_scale switched
 *   off): g = 1, so sf = E4M3(bamax / 6), saturating at 448.
 * Outputs: codes [rows][k/2] bytes (mxq_codes_bytes), sf_swz
 *   (mxq_sf_bytes bytes, padding written as 0), *g_dev.
 * Errors: k % 64 != 0 -> UNSUPPORTED_SHAPE (whole 4-column scale tiles);
 *   NULL x / codes / sf_swz / g_dev, misalignment as above.
 */
mxq_status mxq_quantize_nvfp4(const void* x_bf16, int64_t rows, int64_t k, int64_t ld,
                              const float* amax_dev, uint8_t* codes, uint8_t* sf_swz,
                              float* g_dev, mxq_stream_t stream);

/*
 * mxq_quantize_mxfp8 - MXFP8 quantisation of X [rows, k] (article, Glossary
 * "MXFP8": the OCP MX standard 8-bit format).  Per 32-element block:
 *   X = clamp(floor(log2 bamax) - 8, -127, 127) (a zero block gets -127),
 *   sf = X + 127 (E8M0), code = E4M3(x * 2^-X), saturating at 448.
 * Outputs: codes [rows][k] bytes, sf_swz (mxq_sf_bytes bytes, zero padded).
 * Errors: k % 128 != 0 -> UNSUPPORTED_SHAPE; NULL pointers, misalignment.
 */
mxq_status mxq_quantize_mxfp8(const void* x_bf16, int64_t rows, int64_t k, int64_t ld,
                              uint8_t* codes, uint8_t* sf_swz, mxq_stream_t stream);

/* MXFP8 scale rules: the OCP floor rule above, or the ceiling rule (TorchAO's
 * RCEIL; not in the pages): X = the smallest integer with bamax <= 448 * 2^X,
 * clamped to [-127, 127], so no element saturates. */
enum { MXQ_SCALE_FLOOR = 0, MXQ_SCALE_RCEIL = 1 };

/* mxq_quantize_mxfp8 with a scale rule (MXQ_SCALE_*; other values ->
 * INVALID_ARG).  Same arguments, outputs and errors otherwise. */
mxq_status mxq_quantize_mxfp8_rule(const void* x_bf16, int64_t rows, int64_t k, int64_t ld,
                                   int scale_rule, uint8_t* codes, uint8_t* sf_swz,
                                   mxq_stream_t stream);

/* ------------------------------------------------------------- GEMM ----- */

/*
 * mxq_gemm_blockscaled - Y [M,N] = alpha * (A . B^T) + bias, bf16 out, on the
 * 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
 * Source: the quantised linear of the article (its speed-up tables measure
 * it); alpha = g_A * g_B for NVFP4, 1 otherwise.
 *   f = MXQ_NVFP4: A codes [M][K/2], B codes [N][K/2] (NVFP4 layout above),
 *       a_sf / b_sf swizzled E4M3 scales, a_g_dev / b_g_dev fp32 per-tensor
 *       scales on the device.  K % 64 == 0.
 *   f = MXQ_MXFP8: A [M][K], B [N][K] E4M3 codes, E8M0 swizzled scales;
 *       the g pointers are ignored (may be NULL).  K % 128 == 0.
 *   f = MXQ_BF16:  A [M][K], B [N][K] bf16 (row stride K); scale pointers
 *       ignored.  K % 8 == 0.
 *   bias_bf16: [N] bf16 or NULL.  y_bf16: [M][ldy], ldy >= N, ldy % 8 == 0.
 * Y[m,n] = bf16_rne(alpha * sum_k deq(A)[m,k] deq(B)[n,k] + bias[n]) with
 * fp32 accumulation.  K == 0 is rejected (UNSUPPORTED_SHAPE).
 */
mxq_status mxq_gemm_blockscaled(mxq_format f, int64_t M, int64_t N, int64_t K,
                                const void* a_codes, const uint8_t* a_sf, const float* a_g_dev,
                                const void* b_codes, const uint8_t* b_sf, const float* b_g_dev,
                                const void* bias_bf16, void* y_bf16, int64_t ldy,
                                mxq_stream_t stream);

/* ----------------------------------------------------- weights / linear -- */

/* Flags of mxq_weight_prepare and mxq_weight.flags. */
enum {
  MXQ_WEIGHT_KEEP_BF16 = 1,       /* always run this layer as a bf16 GEMM          */
  MXQ_WEIGHT_NO_TENSOR_SCALE = 2, /* NVFP4 without a per-tensor scale: g = 1 for
                                     both W and every activation (no amax pass)    */
  MXQ_WEIGHT_MXFP8_RCEIL = 4      /* MXFP8 with the ceiling scale rule for W and
                                     every activation                              */
};

/*
 * A prepared linear layer.  Plain data: device pointers plus sizes.  Filled
 * by mxq_weight_prepare; the caller owns every buffer it points to and must
 * keep w_bf16, bias_bf16 and the storage alive while the handle is used.
 */
typedef struct mxq_weight {
  int32_t format;         /* mxq_format the weight is quantised to           */
  int32_t flags;          /* MXQ_WEIGHT_* bits                               */
  int64_t N, K;           /* W is [N, K]                                     */
  const void* w_bf16;     /* original bf16 weights [N][K] (row stride K)     */
  const void* bias_bf16;  /* [N] bf16 or NULL                                */
  const uint8_t* codes;   /* quantised codes inside the storage (or NULL)    */
  const uint8_t* sf;      /* swizzled scales inside the storage (or NULL)    */
  const float* g_dev;     /* NVFP4 per-tensor scale g_W (device) or NULL     */
  const float* amax_dev;  /* amax of W (device; 0 without a per-tensor scale)
                             or NULL                                         */
} mxq_weight;

/* Device bytes mxq_weight_prepare needs for format f (0 for MXQ_BF16). */
size_t mxq_weight_storage_bytes(int64_t N, int64_t K, mxq_format f);

/*
 * mxq_weight_prepare - quantise W [N,K] once, offline (the article quantises
 * weights ahead of time in the same format as the activations, "...NVFP4
 * Weight" in its TorchAO config name).  Runs mxq_amax + mxq_quantize_* on W
 * into `storage` (mxq_weight_storage_bytes bytes, 256-byte aligned) and fills
 * *out.  flags: MXQ_WEIGHT_* bits (0 = the defaults; other bits ->
 * INVALID_ARG).  With MXQ_WEIGHT_KEEP_BF16 or f == MXQ_BF16 nothing is
 * quantised (storage may be NULL) and the layer always runs in bf16.  With
 * MXQ_WEIGHT_NO_TENSOR_SCALE (NVFP4 only, else INVALID_ARG) W is quantised
 * with g_W = 1 and mxq_linear quantises activations with g = 1 (no amax).
 * With MXQ_WEIGHT_MXFP8_RCEIL (MXFP8 only, else INVALID_ARG) W and every
 * activation of the layer use the ceiling scale rule (MXQ_SCALE_RCEIL).
 */
mxq_status mxq_weight_prepare(mxq_format f, const void* w_bf16, int64_t N, int64_t K,
                              const void* bias_bf16, int flags, void* storage,
                              size_t storage_bytes, mxq_weight* out, mxq_stream_t stream);

/* Activation applied in the GEMM epilogue (mxq_linear_opts.activation). */
enum {
  MXQ_ACT_NONE = 0,
  MXQ_ACT_GELU = 1 /* x * Phi(x) with the error function (not the tanh form); erf evaluated in
                      fp32 by Abramowitz and Stegun 7.1.26, |error| <= 1.5e-7 */
};

/* Options of mxq_linear.  A NULL pointer means the defaults; a zeroed struct
 * is the defaults too. */
typedef struct mxq_linear_opts {
  int64_t min_dim;          /* bf16 when min(M,K,N) < min_dim; 0 -> 1024 (the article's rule) */
  void* gemm_event_start;   /* optional cudaEvent_t (NULL: none): mxq_linear records it on the
                               stream right before its GEMM launch and gemm_event_end right
                               after, so a caller can time the GEMM inside a step.  Both or
                               neither; the events stay the caller's. */
  void* gemm_event_end;
  /* Producer epilogue (kernel fusion of the activation and of the next layer's amax; the
   * devin.kr Blackwell FLUX page, section "연산 효율화와 가속 기술": activation functions fused
   * into the custom GEMM).  Available on the CTA-pair GEMM (M > 128); with M <= 128 either
   * option gives MXQ_ERR_UNSUPPORTED_SHAPE. */
  int32_t activation;       /* MXQ_ACT_*: applied to alpha*acc + bias before the bf16 rounding */
  int32_t reserved;         /* 0 */
  float* y_amax_dev;        /* optional device float (4-byte aligned): receives max |y| over the
                               bf16 output (zeroed on the stream first) */
  /* Consumer side: the input's amax already known (e.g. the producing layer's y_amax_dev).
   * The NVFP4 path (with a per-tensor scale) then skips its amax pass: one quantisation
   * kernel reads x once.  Ignored by the other paths.  Must not alias y_amax_dev. */
  const float* x_amax_dev;
} mxq_linear_opts;

/*
 * mxq_linear_path - the format mxq_linear would run for M rows: MXQ_BF16
 * when w->flags has MXQ_WEIGHT_KEEP_BF16, when w->format is MXQ_BF16, or when
 * min(M, K, N) <
 * min_dim (article, "Detailed by section": selective quantisation, layers
 * too small to gain, or accuracy-sensitive embeddings, stay in bf16);
 * w->format otherwise.  Pure host function.  Returns 0 for a NULL w.
 */
int mxq_linear_path(const mxq_weight* w, int64_t M, const mxq_linear_opts* opts);

/* Workspace bytes mxq_linear needs for M rows of K in format f
 * (the quantised activation, its scales and two fp32 scalars). */
size_t mxq_linear_workspace_bytes(int64_t M, int64_t K, mxq_format f);

/*
 * mxq_linear - y = x W^T + bias for x [M, K] bf16 (row stride K), y [M][N]
 * (row stride N).  Dispatch per mxq_linear_path: bf16 GEMM, or
 * amax -> NVFP4 quantise -> block-scaled GEMM, or MXFP8 quantise ->
 * block-scaled GEMM.  ws: device workspace of at least
 * mxq_linear_workspace_bytes(M, K, w->format) bytes, 256-byte aligned
 * (unused on the bf16 path; may be NULL there).  Its contents on entry do not
 * matter (nothing in it has to start at zero).
 * NVFP4 activations that fit in the shared memory of one CTA per SM are
 * quantised by one cooperative kernel (amax and quantisation in one pass
 * over HBM, the amax exchanged through a bounded grid barrier whose state
 * lives in the workspace); larger ones by two kernels (partial maxima, then
 * quantisation).  A weight prepared with MXQ_WEIGHT_NO_TENSOR_SCALE takes
 * no amax: one quantisation kernel with g = 1, then the GEMM (alpha = 1).
 * Calls sharing one workspace must be ordered on the GPU.
 */
mxq_status mxq_linear(const mxq_weight* w, const void* x_bf16, int64_t M, void* y_bf16,
                      void* ws, size_t ws_bytes, const mxq_linear_opts* opts,
                      mxq_stream_t stream);

/* Size of the device scratch array that mxq_linear_noalloc uses (64 MiB). */
#define MXQ_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/*
 * mxq_linear_noalloc - mxq_linear for callers that cannot allocate device
 * memory: for example a host whose device-memory budget is fixed at start-up
 * and that forbids allocations afterwards, or a latency-critical loop where
 * cudaMalloc (it may synchronise the device and its latency is unbounded) is
 * not acceptable.  The method has no such call: it is an addition of this
 * library.
 * Same arguments and result as mxq_linear, without ws / ws_bytes: the
 * workspace for the quantised activation lives in a file-scope device array of
 * MXQ_NOALLOC_SCRATCH_BYTES that every GPU loading this library holds until
 * the process exits.  Nothing is allocated by the call.
 *  - The first call on a device (with that device current) looks up the
 *    array's address and caches it; make that first call before any stream
 *    capture.
 *  - All calls share the array and it keeps the previous call's contents,
 *    which is all mxq_linear needs (no value in its workspace has to start at
 *    zero).  Calls that can overlap on the GPU (other streams, unordered host
 *    threads) race on the array: serialise them.
 *  - A quantised path whose workspace (mxq_linear_workspace_bytes) exceeds
 *    MXQ_NOALLOC_SCRATCH_BYTES returns MXQ_ERR_WORKSPACE and enqueues nothing;
 *    the bf16 path needs no workspace.
 */
mxq_status mxq_linear_noalloc(const mxq_weight* w, const void* x_bf16, int64_t M, void* y_bf16,
                              const mxq_linear_opts* opts, mxq_stream_t stream);

/* ------------------------------------------------------- attention ----- */

/*
 * 8-bit attention with per-token scales (the devin.kr page on Blackwell FLUX
 * image generation, "엔비디아 블랙웰 기반 플럭스 3 이미지 생성 4.45배 가속",
 * section "연산 효율화와 가속 기술": a dedicated 8-bit floating-point attention
 * path that corrects the quantisation error token by token).  Per head, with
 * T tokens and head dimension d = 128:
 *   Q, K -> MXFP8 (E4M3 codes, one power-of-two scale per token and per 32
 *   channels), V -> MXFP8 of V^T (per channel and per 32 tokens);
 *   S = deq(Q) deq(K)^T on the tensor cores (fp32); softmax along keys with
 *   scale tau through the weights E = 2^(t - m) in fp32, t = S tau log2 e,
 *   m an integer (any integer gives the same codes: a power-of-two factor
 *   moves only a block's shared exponent; the kernel takes a running
 *   maximum in one pass over the keys); E -> MXFP8 along keys (ceiling scale
 *   rule, no saturation); O = deq(E) deq(V^T)^T / rowsum(deq(E)) on the
 *   tensor cores (fp32; each query row divided by the sum of its quantised
 *   weights, the per-token correction of their rounding), bf16 out.
 * Accuracy: |O - O_exact| <= 0.14 * T + 2^-11 * max_j |V[j, c]| + 1e-6 per
 * element, with O_exact the float64 attention on the quantised Q, K, V and
 * T = sum_j P[i, j] |V[j, c]| -- the rounding of E to E4M3 (at most 2^-4 of
 * each weight, twice through the renormalisation) dominates.
 *
 * mxq_attention_workspace_bytes - device bytes mxq_attention_mxfp8 needs
 * (the quantised Q, K, V^T and their scales); 0 for unsupported arguments.
 */
size_t mxq_attention_workspace_bytes(int64_t heads, int64_t tokens, int64_t d);

/*
 * mxq_attention_mxfp8 - out = attention(q, k, v) per head.
 *   q, k, v, out: [heads][tokens][d] bf16, contiguous, device, 16-byte aligned.
 *   d must be 128 and tokens a multiple of 128 (else UNSUPPORTED_SHAPE).
 *   tau: softmax scale; 0 (or any non-positive or non-finite value) means
 *   1/sqrt(d).
 *   ws: device workspace of mxq_attention_workspace_bytes(heads, tokens, d)
 *   bytes, 256-byte aligned; any contents on entry.
 * Four launches on `stream` (Q and K quantisation, V^T quantisation, the
 * attention kernel), no host synchronisation, nothing allocated.  Argument
 * errors return before anything is enqueued; device-side timeouts show in
 * mxq_get_device_error.  Calls sharing a workspace must be ordered on the GPU.
 */
mxq_status mxq_attention_mxfp8(const void* q_bf16, const void* k_bf16, const void* v_bf16,
                               int64_t heads, int64_t tokens, int64_t d, float tau, void* out_bf16,
                               void* ws, size_t ws_bytes, mxq_stream_t stream);

/* ---------------------------------------------------- diagnostics ------- */

/*
 * mxq_linear_kernel_count - how many kernels one mxq_linear call with these
 * arguments launches on the current device: 1 (bf16 GEMM), 2 (MXFP8
 * quantise + GEMM, single-pass NVFP4 quantise + GEMM, or NVFP4 without a
 * per-tensor scale: quantise + GEMM) or 3 (NVFP4 partial
 * maxima + quantise + GEMM); 0 when M or N is 0 (nothing is launched) or w
 * is NULL; -1 when the current device cannot be queried.  Uses the same
 * decisions as mxq_linear.  No GPU work.
 */
int mxq_linear_kernel_count(const mxq_weight* w, int64_t M, const mxq_linear_opts* opts);

/*
 * mxq_get_device_error - synchronise `stream`, then read and clear the
 * current device's error word.  Returns MXQ_OK, MXQ_ERR_TIMEOUT (a bounded
 * wait inside a kernel ran out and that kernel returned early; its outputs
 * are undefined) or MXQ_ERR_CUDA (the synchronisation itself failed).
 */
mxq_status mxq_get_device_error(mxq_stream_t stream);

/*
 * mxq_convert_f32 - element-wise conversion with the exact device routines
 * the quantisers use, for exhaustive conversion checks.
 * code_fmt 1: E2M1 (out[i] = 4-bit code in the low nibble),
 * code_fmt 2: E4M3.  in: n fp32 values (device); out: n bytes (device).
 */
mxq_status mxq_convert_f32(const float* in, int64_t n, int code_fmt, uint8_t* out,
                           mxq_stream_t stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* MXQ_H_ */
