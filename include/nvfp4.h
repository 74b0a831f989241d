/*
 * nvfp4.h -- C ABI of libnvfp4.so: NVFP4 (e2m1 values, 16-element blocks, ue4m3 block
 * scales) quantization and block-scaled FP4 GEMMs for NVIDIA B200 (sm_100a).
 *
 * Sources, cited by page title and section:
 *   [TRT] TensorRT-LLM NVFP4LinearMethod.create_weights
 *   [FV]  FastVideo PR #1350 "Add NVFP4QAT linear layer", code-review thread (_global_sf)
 *   [FI3] flashinfer PR #1774 "Masked batch nvfp4 quantization"
 *   [FI5] flashinfer docs flashinfer.gemm.mm_nvfp4_svdquant (signature, Parameters)
 *   [NVF] NVIDIA/Fuser PR #5737 "Benchmark for nvfp4 scaled mm" (module tree, forward)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers are CUDA device pointers owned by the caller unless stated otherwise.
 *    Sizes are element counts.  bf16 tensors are passed as `const void*`.
 *  - Tensors are dense and row-major.  Packed FP4 tensors are uint8 [rows, k/2] with two
 *    e2m1 codes per byte: byte i of a row holds element 2i in its low nibble and element
 *    2i+1 in its high nibble.  e2m1 magnitudes are {0, .5, 1, 1.5, 2, 3, 4, 6}; bit 3
 *    is the sign.
 *  - A block-scale buffer holds one ue4m3 byte per 16-element block along k, in the
 *    128x4 swizzled layout [TRT, FI5 a_sf]: nvfp4_scale_bytes(rows, k) bytes, a
 *    sequence of 512-byte chunks, one per (128-row tile, 4-block group) with the group
 *    index fastest; the scale of row r, block c is at chunk byte
 *    (r % 32) * 16 + ((r % 128) / 32) * 4 + c % 4.  Padding entries (rows >= rows or
 *    blocks >= k/16) are written as 0 by the dense quantizer.
 *  - The global scale is gsf = 448*6 / amax with amax = max|x| (NaN counted as 0,
 *    +-Inf as FLT_MAX, clamped below at 1e-12) [FV, TRT input_scale].  The GEMM factor
 *    is alpha = amax_a * amax_b / (448*6)^2 [TRT alpha].  Both are fp32 DEVICE values,
 *    so no call reads a scalar back to the host: calls are ordered by their stream alone.
 *  - Every call launches on `stream` (a cudaStream_t; NULL is the legacy default
 *    stream) and allocates nothing per call.  The first call on a device sets up the
 *    library's per-device state: it allocates the status word and the 32 KB SiLU table
 *    with cudaMalloc and fills the table with one kernel on the legacy default stream,
 *    waiting for it (the only host synchronization outside nvfp4_device_status).  The
 *    first global-scale reduction on a stream allocates that stream's small workspace.
 *    Make both first calls before capturing a stream into a CUDA graph.
 *  - Arguments are validated before anything is launched: a call that returns an
 *    error has written nothing.
 *  - Return value: NVFP4_OK or one of the NVFP4_ERR_* codes below.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *nvfp4_stream_t;

enum nvfp4_status {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARGUMENT = 1, /* null/misaligned pointer, unsupported size or rank */
  NVFP4_ERR_UNSUPPORTED_DEVICE = 2, /* the current device is not compute capability 10.0 */
  NVFP4_ERR_CUDA = 3,             /* a CUDA runtime/driver call or a launch failed */
  NVFP4_ERR_DEVICE_TIMEOUT = 4,   /* a bounded device-side wait gave up (see nvfp4_device_status) */
  NVFP4_ERR_OUT_OF_MEMORY = 5,    /* the one-time workspace allocation failed */
  NVFP4_ERR_INDEX = 6             /* debug builds: a kernel computed an index outside its operand */
};

/* Human-readable name of a status code (static string, never NULL). */
NVFP4_API const char *nvfp4_status_string(int status);

/*
 * Bytes of a block-scale buffer for `rows` rows of `k` elements:
 * pad_up(rows, 128) * pad_up(k / 16, 4) = ceil(rows/128)*128 * ceil(k/64)*4
 * [TRT create_weights weight_scale padding; FI5 a_sf numel].  Returns -1 when
 * rows < 0 or k is negative or not a multiple of 16.  Host-only, never fails otherwise.
 */
NVFP4_API int64_t nvfp4_scale_bytes(int64_t rows, int64_t k);

/*
 * Global scale of a bf16 tensor [FV _global_sf; TRT input_scale and alpha].
 *   x_bf16     [numel] bf16, 16-byte aligned.  numel >= 0 (0 gives amax = 1e-12).
 *   amax_out   nullable; receives the clamped amax (fp32 [1]).
 *   gsf_out    required; receives 448*6/amax (fp32 [1]).
 *   other_amax nullable; the amax of the GEMM's other operand (fp32 [1]).  When given,
 *   alpha_out  (required then) receives amax * other_amax / (448*6)^2 (fp32 [1]).
 * One kernel launch; all outputs are written by its last block.
 */
NVFP4_API int nvfp4_global_scale(const void *x_bf16, int64_t numel, float *amax_out, float *gsf_out,
                       const float *other_amax, float *alpha_out, nvfp4_stream_t stream);

/*
 * Per-item global scale over the valid rows of a batch [FI3 per-item global_scale;
 * the domain of each item's amax is its rows r < mask[i]].
 *   x_bf16   [b, m, k] bf16, or [b, m, 2k] when silu_mul != 0 (gate | up halves), in
 *            which case amax is taken over h = bf16(silu(gate) * up).  16-byte aligned.
 *   mask     nullable int32 [b]: valid rows per item (values clamped to [0, m]); NULL
 *            means every row.
 *   amax_out nullable fp32 [b]; gsf_out required fp32 [b].
 * Requires k % 8 == 0 and b <= 4096.
 */
NVFP4_API int nvfp4_global_scale_batched(const void *x_bf16, int64_t b, int64_t m, int64_t k,
                               const int32_t *mask, int silu_mul, float *amax_out,
                               float *gsf_out, nvfp4_stream_t stream);

/*
 * Non-allocating variant of nvfp4_global_scale_batched (same arguments, same results).
 * The pages have no counterpart of this entry point.  It exists for callers that cannot
 * let the library call cudaMalloc: hosts whose device memory belongs to their own
 * allocator or is a fixed budget set at start-up (a pre-sized pool in an inference
 * server, an embedded deployment), and latency-critical paths that must not risk the
 * implicit device synchronization an allocation can cause.  Its reduction scratch is a
 * fixed device array inside the library (4100 bytes, held by every GPU that loads the
 * library until the process exits) instead of the per-stream workspace.
 *   b must be at most 1024; larger b returns NVFP4_ERR_INVALID_ARGUMENT before anything
 *   is launched.
 *   The first call on each device looks up the array's device address (no allocation);
 *   make that first call before any stream capture.
 *   Every call clears the words it uses and shares the same array: calls that overlap on
 *   the GPU (concurrent streams) race with each other and must be ordered by the caller.
 *   Calls on one stream are ordered and safe.
 * Calls no cudaMalloc, cudaFree or other allocating routine.
 */
NVFP4_API int nvfp4_global_scale_batched_noalloc(const void *x_bf16, int64_t b, int64_t m, int64_t k,
                                                 const int32_t *mask, int silu_mul, float *amax_out,
                                                 float *gsf_out, nvfp4_stream_t stream);

/*
 * Dense NVFP4 quantize [TRT create_weights; FI3 fp4_quantize(x, global_scale, 16, ...)].
 *   x_bf16 [m, k] bf16, 16-byte aligned; k % 16 == 0, m >= 0.
 *   gsf    fp32 [1] device: the global scale 448*6/amax.
 *   q_out  uint8 [m, k/2] packed e2m1 (4-byte aligned).
 *   sf_out uint8 [nvfp4_scale_bytes(m, k)] ue4m3 scales, swizzled; padding entries 0.
 * Per 16-element block: s = ue4m3_rn_satfinite((max|x| / 6) * gsf); each element is
 * encoded as e2m1_rn_satfinite(x * (s == 0 ? 0 : gsf / s)).
 */
NVFP4_API int nvfp4_quantize(const void *x_bf16, int64_t m, int64_t k, const float *gsf,
                   uint8_t *q_out, uint8_t *sf_out, nvfp4_stream_t stream);

/*
 * Global scale and dense quantize in one launch: the results of nvfp4_global_scale
 * followed by nvfp4_quantize with its gsf, bit for bit [FV _global_sf; TRT input_scale;
 * FI3 fp4_quantize].  The pages compute the two in sequence; fusing them is this
 * library's: one persistent grid reduces max|x| (keeping x in L2), meets at a grid-wide
 * barrier, and quantizes, reading most of x a second time from L2 instead of HBM.
 *   x_bf16     [m, k] bf16, 16-byte aligned; k % 16 == 0, k > 0, m >= 0 (m = 0 writes
 *              only the scalars: amax = 1e-12).
 *   amax_out   nullable fp32 [1]; gsf_out required fp32 [1]; other_amax / alpha_out as in
 *              nvfp4_global_scale (both or neither).
 *   q_out      uint8 [m, k/2] (8-byte aligned); sf_out uint8 [nvfp4_scale_bytes(m, k)] (both may
 *              be NULL when m = 0).
 * Uses the stream's reduction workspace (allocated on the stream's first use, like
 * nvfp4_global_scale).  The grid is a cooperative launch (all CTAs resident) of at most
 * three CTAs per SM; it is not chained to its predecessor by programmatic dependent
 * launch.  The barrier wait is bounded (1 s): if it runs out, nothing is written,
 * NVFP4_ERR_DEVICE_TIMEOUT is recorded in the device status word, and clearing that word
 * with nvfp4_device_status also re-zeroes the device's reduction workspaces.
 */
NVFP4_API int nvfp4_global_scale_quantize(const void *x_bf16, int64_t m, int64_t k, float *amax_out,
                                          float *gsf_out, const float *other_amax, float *alpha_out,
                                          uint8_t *q_out, uint8_t *sf_out, nvfp4_stream_t stream);

/*
 * Masked batched quantize [FI3 nvfp4_batched_quantize(..., mask)].
 *   x_bf16 [b, m, k] bf16; mask nullable int32 [b] (NULL: all rows); gsf fp32 [b].
 *   q_out  uint8 [b, m, k/2]; sf_out uint8 [b][nvfp4_scale_bytes(m, k)].
 * Item i is quantized as nvfp4_quantize on its rows r < mask[i] with gsf[i].  Rows at
 * or beyond mask[i] and their scale entries are NOT written (they keep whatever the
 * caller left there).  With mask == NULL, the padding rows' scale entries are zeroed.
 */
NVFP4_API int nvfp4_quantize_masked_batched(const void *x_bf16, int64_t b, int64_t m, int64_t k,
                                  const int32_t *mask, const float *gsf, uint8_t *q_out,
                                  uint8_t *sf_out, nvfp4_stream_t stream);

/*
 * SiLU-and-mul fused quantize [FI3 silu_and_mul_fp4_batched_quantize; the
 * "2*hidden -> hidden" mapping, k_by_2 % 2 == 0 check].
 *   x_bf16 [b, m, 2k] bf16: gate = x[..., :k], up = x[..., k:].
 *   k      the OUTPUT width; k % 16 == 0.
 *   mask, gsf, q_out [b, m, k/2], sf_out [b][nvfp4_scale_bytes(m, k)] as in
 *   nvfp4_quantize_masked_batched.
 * h = bf16(silu(gate) * up) with silu(g) = g / (1 + exp(-g)), where exp is the
 * library's specified fp32 exponential (Cody-Waite reduction, degree-7 Taylor
 * polynomial, exact 2^n scaling); h is then quantized as above.  silu(g) of a bf16 g is
 * read from a table the library computes once per device with exactly that arithmetic
 * (32 KB of device memory, allocated with the status word on the first call on the
 * device), so the kernel's h equals the definition for every bf16 input.
 */
NVFP4_API int nvfp4_silu_mul_quantize_batched(const void *x_bf16, int64_t b, int64_t m, int64_t k,
                                    const int32_t *mask, const float *gsf, uint8_t *q_out,
                                    uint8_t *sf_out, nvfp4_stream_t stream);

/*
 * Dense block-scaled FP4 GEMM  out = bf16(alpha * (a @ b^T) [+ bias])
 * [FI5 mm_nvfp4_svdquant without the low-rank term; NVF f16a_nvfp4weight_scaled_mm
 * output [M, N] bf16; TRT weight [out, in/2]].
 *   a     uint8 [m, k/2] packed e2m1 (row-major, K contiguous), 16-byte aligned.
 *   b     uint8 [n, k/2] packed e2m1 (the weight, [out_features, in_features/2]).
 *   a_sf  uint8 [nvfp4_scale_bytes(m, k)], b_sf uint8 [nvfp4_scale_bytes(n, k)],
 *         16-byte aligned.
 *   alpha fp32 [1] device scalar.
 *   bias  nullable bf16 [n] (added after the alpha scaling, not scaled).
 *   out   bf16 [m, n], 16-byte aligned; n % 8 == 0.
 *   k % 64 == 0 (one 64-element MMA step and a full 4-block scale group), k > 0.
 * Accumulation is fp32 in tensor memory (tcgen05 block-scaled MMA).
 */
NVFP4_API int nvfp4_gemm(const uint8_t *a, const uint8_t *b, const uint8_t *a_sf, const uint8_t *b_sf,
               const float *alpha, const void *bias_bf16, void *out_bf16, int64_t m, int64_t n,
               int64_t k, nvfp4_stream_t stream);

/*
 * bf16-activation NVFP4 linear [NVF f16a_nvfp4weight_scaled_mm: bf16 activation, NVFP4
 * weight, bf16 [M, N] out; its compiler path quantizes the activation and runs the scaled
 * FP4 matmul]:  out = nvfp4_gemm(quantize(a, gsf_a), b, alpha) with the activation's global
 * scale computed on the device (dynamic), alpha = amax_a * amax_b / (448*6)^2.
 *   a_bf16     [m, k] bf16, 16-byte aligned; k % 64 == 0, k > 0, m >= 0.
 *   b, b_sf    the NVFP4 weight [n, k/2] and its scales, as in nvfp4_gemm.
 *   b_amax     fp32 [1] device: the weight's amax (its global scale is 448*6 / b_amax; the
 *              pages pass weight_global_scale, this library keeps amaxes so that alpha is
 *              the [TRT] product formula).
 *   bias_bf16  nullable bf16 [n]; out_bf16 bf16 [m, n] as in nvfp4_gemm.
 *   a_q_ws     caller workspace uint8 [m, k/2] (16-byte aligned): the quantized activation.
 *   a_sf_ws    caller workspace uint8 [nvfp4_scale_bytes(m, k)] (16-byte aligned).
 *   scalars_ws caller workspace fp32 [3]: receives amax_a, gsf_a and alpha.
 * Two launches on `stream` (nvfp4_global_scale_quantize, then nvfp4_gemm); allocates
 * nothing beyond the stream's reduction workspace (allocated on its first use).  The
 * quantized activation is left in the workspace and equals nvfp4_quantize's bit for bit.
 */
NVFP4_API int nvfp4_gemm_bf16a(const void *a_bf16, const uint8_t *b, const uint8_t *b_sf, const float *b_amax,
                               const void *bias_bf16, void *out_bf16, uint8_t *a_q_ws, uint8_t *a_sf_ws,
                               float *scalars_ws, int64_t m, int64_t n, int64_t k, nvfp4_stream_t stream);

/*
 * bf16-activation NVFP4 linear with a static activation scale [NVF
 * f16a_nvfp4weight_scaled_mm: bf16 activation, NVFP4 weight, bf16 [M, N] out, which the
 * compiler path runs as the activation's block quantization and the scaled FP4 matmul; TRT
 * create_weights: a calibrated input_scale for the activation]:
 *   out = nvfp4_gemm(quantize(a, a_gsf), b, alpha)
 *   a_bf16     [m, k] bf16, 16-byte aligned; k % 64 == 0, n % 8 == 0.
 *   b, b_sf    the NVFP4 weight [n, k/2] and its scales, as in nvfp4_gemm.
 *   a_gsf      fp32 [1] device: the activation's static global scale (448*6 / calibrated amax).
 *   alpha      fp32 [1] device: calibrated amax_a * amax_b / (448*6)^2.
 *   bias_bf16  nullable bf16 [n]; out_bf16 bf16 [m, n] as in nvfp4_gemm.
 *   a_q_ws     caller workspace uint8 [m, k/2] (16-byte aligned): receives the quantized
 *              activation, equal to nvfp4_quantize(a_bf16, a_gsf) bit for bit.
 *   a_sf_ws    caller workspace uint8 [nvfp4_scale_bytes(m, k)] (16-byte aligned), likewise.
 *   one_launch 0: nvfp4_quantize then nvfp4_gemm on `stream` (the faster form on B200).
 *              1: one GEMM launch whose epilogue warps, before draining any accumulator,
 *              quantize a share of the activation (128-row slab x 256-column K chunk units,
 *              K chunks first) into the workspace and count each finished chunk; a CTA's TMA
 *              producer loads chunk c of A only after every slab's chunk c is counted.  Needs
 *              k <= 16384; uses the stream's reduction workspace (allocated on its first use)
 *              for the chunk counters and leaves it zeroed.  Every CTA of the grid (one 2-CTA
 *              cluster per pair of SMs) must be resident at once, as the persistent GEMM's
 *              grid is when nothing else holds the SMs; a counter wait that runs out (1 s)
 *              records NVFP4_ERR_DEVICE_TIMEOUT.
 * Both forms give the same bytes.  With n = 0 only the workspace is written (nvfp4_quantize);
 * every argument is checked before anything is launched, so an invalid call writes nothing.
 */
NVFP4_API int nvfp4_gemm_bf16a_static(const void *a_bf16, const uint8_t *b, const uint8_t *b_sf, const float *a_gsf,
                                      const float *alpha, const void *bias_bf16, void *out_bf16, uint8_t *a_q_ws,
                                      uint8_t *a_sf_ws, int64_t m, int64_t n, int64_t k, int one_launch,
                                      nvfp4_stream_t stream);

/*
 * Masked grouped GEMM for MoE experts [FI3: inputs for grouped_gemm_nt_masked; NVF
 * routed_experts GroupedLinear].  For every expert e and row i < mask[e]:
 *   out[e, i, :] = bf16(alpha[e] * a[e, i, :] @ b[e]^T)
 *   a     uint8 [E, mmax, k/2]; a_sf uint8 [E][nvfp4_scale_bytes(mmax, k)]
 *   b     uint8 [E, n, k/2];    b_sf uint8 [E][nvfp4_scale_bytes(n, k)]
 *   mask  int32 [E] device (values clamped to [0, mmax]); alpha fp32 [E] device.
 *   out   bf16 [E, mmax, n]; rows i >= mask[e] are not written.
 * Constraints as nvfp4_gemm.  Empty rows cost no tensor-core work: the device-side
 * scheduler walks only the row tiles below each expert's mask.
 */
NVFP4_API int nvfp4_grouped_gemm_masked(const uint8_t *a, const uint8_t *b, const uint8_t *a_sf,
                              const uint8_t *b_sf, const int32_t *mask, const float *alpha,
                              void *out_bf16, int64_t E, int64_t mmax, int64_t n, int64_t k,
                              nvfp4_stream_t stream);

/*
 * Low-rank-corrected GEMM (SVDQuant) [FI5 mm_nvfp4_svdquant]:
 *   out = bf16(alpha * (a @ b^T + d @ l1^T) [+ bias])
 * i.e. the FP4 K-loop and then a bf16 MMA of d @ l1^T into the same fp32 accumulator,
 * with the epilogue alpha * acc + bias; l1 is the LoRA-up weight, already divided by alpha
 * by the caller.
 *   d     bf16 [m, r] contiguous, 16-byte aligned (LoRA-down output).
 *   l1    bf16 [n, r] contiguous, 16-byte aligned.
 *   r     rank: a positive multiple of 32, at most 256.
 *   Other arguments and constraints as nvfp4_gemm.
 */
NVFP4_API int nvfp4_gemm_lowrank_bias(const uint8_t *a, const uint8_t *b, const uint8_t *a_sf,
                            const uint8_t *b_sf, const float *alpha, const void *d_bf16,
                            const void *l1_bf16, int64_t r, const void *bias_bf16,
                            void *out_bf16, int64_t m, int64_t n, int64_t k,
                            nvfp4_stream_t stream);

/*
 * Gate/up projection with SiLU * up and NVFP4 quantization in the GEMM epilogue (the
 * SwiGLU block's first half) [NVF module tree: NVFP4InferenceSwiGLU gate_proj / up_proj;
 * FI3 silu_and_mul_fp4_batched_quantize, the quantizer it replaces]:
 *   g = bf16(alpha_gate * (a @ b_gate^T)),  u = bf16(alpha_up * (a @ b_up^T)),
 *   h = bf16(silu(g) * u),  (q_out, sf_out) = NVFP4 quantization of h with gsf_h.
 * Each of g, u, h and the quantized output is rounded exactly as by nvfp4_gemm (no
 * bias) followed by nvfp4_silu_mul_quantize_batched on [g | u], so the result equals
 * that two-call sequence on the same accumulator values; the bf16 g and u never
 * reach memory.
 *   a          uint8 [m, k/2] packed e2m1; a_sf [nvfp4_scale_bytes(m, k)].
 *   b_gate     uint8 [n, k/2] (gate_proj weight); b_gate_sf [nvfp4_scale_bytes(n, k)].
 *   b_up       uint8 [n, k/2] (up_proj weight);   b_up_sf   [nvfp4_scale_bytes(n, k)].
 *              A concatenated [2n, k/2] gate/up weight quantized as one tensor is passed
 *              as b_gate = w, b_up = w + n*k/2, b_up_sf = w_sf + nvfp4_scale_bytes(n, k)
 *              and the same alpha twice.
 *   alpha_gate, alpha_up  fp32 [1] device scalars.
 *   gsf_h      fp32 [1] device scalar: the global scale of h (448*6 / amax(h), taken
 *              from calibration because amax(h) is not known before the GEMM).
 *   q_out      uint8 [m, n/2]; sf_out uint8 [nvfp4_scale_bytes(m, n)]; padding rows
 *              m <= r < pad_up(m, 128) of sf_out are written as 0.
 *   n % 128 == 0 (n is the width of h); k % 64 == 0; 16-byte aligned buffers.
 */
NVFP4_API int nvfp4_gemm_silu_mul_quantize(const uint8_t *a, const uint8_t *b_gate, const uint8_t *b_up,
                                 const uint8_t *a_sf, const uint8_t *b_gate_sf,
                                 const uint8_t *b_up_sf, const float *alpha_gate,
                                 const float *alpha_up, const float *gsf_h, uint8_t *q_out,
                                 uint8_t *sf_out, int64_t m, int64_t n, int64_t k,
                                 nvfp4_stream_t stream);

/*
 * Masked grouped form for the routed experts [NVF NVFP4InferenceGroupedSwiGLU; FI3
 * masked silu_and_mul quantize]: for every expert e and row i < mask[e], the computation
 * of nvfp4_gemm_silu_mul_quantize with a[e], b_gate[e], b_up[e], alpha_gate[e],
 * alpha_up[e] and gsf_h[e].
 *   a [E, mmax, k/2]; a_sf [E][nvfp4_scale_bytes(mmax, k)].
 *   b_gate, b_up [E, n, k/2]; b_gate_sf, b_up_sf [E][nvfp4_scale_bytes(n, k)].
 *   mask int32 [E]; alpha_gate, alpha_up, gsf_h fp32 [E] (device).
 *   q_out [E, mmax, n/2]; sf_out [E][nvfp4_scale_bytes(mmax, n)].  Rows i >= mask[e]
 *   (codes and scale entries) are not written, as in nvfp4_silu_mul_quantize_batched.
 */
NVFP4_API int nvfp4_grouped_gemm_silu_mul_quantize_masked(
    const uint8_t *a, const uint8_t *b_gate, const uint8_t *b_up, const uint8_t *a_sf,
    const uint8_t *b_gate_sf, const uint8_t *b_up_sf, const int32_t *mask, const float *alpha_gate,
    const float *alpha_up, const float *gsf_h, uint8_t *q_out, uint8_t *sf_out, int64_t E, int64_t mmax,
    int64_t n, int64_t k, nvfp4_stream_t stream);

/*
 * SiLU-and-mul without quantization [FI3 silu_and_mul, the unfused reference of the
 * fused quantizer]: h[r, c] = bf16(silu(x[r, c]) * x[r, k + c]) with silu(g) = g / (1 + exp(-g))
 * and the library's specified fp32 exponential -- the same arithmetic, bit for bit, as
 * nvfp4_silu_mul_quantize_batched and the SiLU * up GEMM epilogue.
 *   x_bf16 [rows, 2k] bf16 (gate | up), h_bf16 [rows, k] bf16; k % 8 == 0; 16-byte aligned.
 */
NVFP4_API int nvfp4_silu_and_mul(const void *x_bf16, int64_t rows, int64_t k, void *h_bf16, nvfp4_stream_t stream);

/*
 * Smooth quantize: the SVDQuant activation quantizer [FI5 mm_nvfp4_svdquant, Parameters a:
 * produced by nvfp4_quantize_smooth, which folds the pre-quantization scale in; TRT
 * pre_quant_scale].  x_hat[r, c] = bf16(x[r, c] * pre_quant_scale[c]) (one fp32
 * multiplication rounded to bf16), then quantized exactly as nvfp4_quantize.
 *   x_bf16 [m, k] bf16; pre_quant_scale_bf16 [k] bf16 (16-byte aligned); k % 16 == 0.
 *   gsf    fp32 [1] device: the global scale of x_hat (448*6 / amax(x_hat)).
 *   q_out, sf_out as nvfp4_quantize.
 */
NVFP4_API int nvfp4_quantize_smooth(const void *x_bf16, int64_t m, int64_t k, const void *pre_quant_scale_bf16,
                                    const float *gsf, uint8_t *q_out, uint8_t *sf_out, nvfp4_stream_t stream);

/*
 * LoRA-down product of an SVDQuant layer [FI5 mm_nvfp4_svdquant, Parameters d: the rank-r
 * operand is x times the pre-quantization-scaled down projection, in bf16]:
 *   d = bf16(x @ w^T), accumulated in fp32 on the tensor cores.
 *   x_bf16 [m, k] bf16 (the unsmoothed activation), k % 64 == 0.
 *   w_bf16 [r, k] bf16: row j is (pre_quant_scale * L2[j, :]), prepared once per layer.
 *   r      rank: a multiple of 32 in [32, 256].
 *   d_bf16 [m, r] bf16 output, 16-byte aligned.
 */
NVFP4_API int nvfp4_lora_down(const void *x_bf16, int64_t m, int64_t k, const void *w_bf16, int64_t r,
                              void *d_bf16, nvfp4_stream_t stream);

/*
 * Both of the above in one pass over x (the pages run them as two ops): the NVFP4 operand
 * of nvfp4_quantize_smooth and the d of nvfp4_lora_down, bit-identical to the separate
 * calls' q_out / sf_out and to nvfp4_lora_down's d.  Arguments as in the two calls;
 * k % 64 == 0.  Each 128-row tile of x is read once by a cluster of 4 CTAs that split its
 * K range; their partial d are summed through distributed shared memory.
 */
NVFP4_API int nvfp4_quantize_smooth_lora_down(const void *x_bf16, int64_t m, int64_t k,
                                              const void *pre_quant_scale_bf16, const float *gsf,
                                              const void *w_bf16, int64_t r, uint8_t *q_out,
                                              uint8_t *sf_out, void *d_bf16, nvfp4_stream_t stream);

/*
 * Programmatic dependent launch [FI5 mm_nvfp4_svdquant, Parameters: enable_pdl, which
 * defaults to the device default].  When enabled (the default: compute capability 10.0
 * supports it), every kernel of the library is launched with programmatic stream
 * serialization: it may start while the preceding kernel of its stream is finishing, runs
 * its set-up (barriers, tensor memory, descriptor prefetch), and waits for that kernel to
 * complete before its first global memory access; it lets the next kernel start in the
 * same way.  Results are identical either way; only launch latency overlaps.  The setting
 * is process-wide and applies to launches made after the call, including launches
 * captured into CUDA graphs.  nvfp4_set_pdl returns NVFP4_OK; nvfp4_get_pdl returns the
 * current setting (0 or 1).
 */
NVFP4_API int nvfp4_set_pdl(int enable);
NVFP4_API int nvfp4_get_pdl(void);

/*
 * Device-side status word of the current device.  GEMM kernels bound every wait; a
 * wait that runs out records NVFP4_ERR_DEVICE_TIMEOUT here and the kernel returns
 * without hanging the GPU.  Synchronizes the device, then stores the word in
 * *status_out and, when clear != 0, resets it to NVFP4_OK.
 */
NVFP4_API int nvfp4_device_status(int *status_out, int clear);

/*
 * Self-tests of the failure detection (the pages have no counterpart; they exist so that
 * the bounded waits can be exercised on a GPU without faulting or hanging it).
 *
 * nvfp4_selftest_bounded_wait launches one thread that waits, through the same bounded
 * wait the GEMM kernels use, for an mbarrier phase that nothing ever completes; after about
 * one second the wait gives up and NVFP4_ERR_DEVICE_TIMEOUT is recorded in the device
 * status word (read it with nvfp4_device_status).
 *
 * nvfp4_selftest_gemm_stall runs nvfp4_gemm on the given operands (same arguments and
 * constraints) with the loads of the first K stage of each pair's first tile withheld: the
 * MMA issuer's wait for that stage runs out, records NVFP4_ERR_DEVICE_TIMEOUT, and every
 * role of both CTAs of each pair unwinds (bounded drain, cluster barrier, tensor memory
 * freed) within a few seconds.  out_bf16 is left unspecified.  The device stays usable.
 *
 * nvfp4_selftest_grid_barrier runs nvfp4_global_scale_quantize (same constraints) with one
 * more barrier arrival expected than the grid has CTAs: every CTA's barrier wait runs out
 * after about one second, NVFP4_ERR_DEVICE_TIMEOUT is recorded, and nothing is written.
 * The stream's reduction workspace is left set until the status word is cleared with
 * nvfp4_device_status (which re-zeroes it); the next call then computes correctly.
 */
NVFP4_API int nvfp4_selftest_bounded_wait(nvfp4_stream_t stream);

/*
 * Debug builds (libnvfp4_debug.so, built with `python -m nvfp4_block_scaled_16_b200.build
 * --debug`) check every global-memory index a kernel computes for a plain load or store (TMA
 * transfers are bounded by their tensor maps) against the extent the call's arguments give the
 * operand; an index out of range is not accessed and NVFP4_ERR_INDEX is recorded in the device
 * status word (read it with nvfp4_device_status).  Release builds compile the checks away.
 * nvfp4_debug_index_checks returns 1 in a debug build, 0 otherwise.
 * nvfp4_selftest_index_check launches one thread that submits an index equal to its extent to
 * the check: a debug build records NVFP4_ERR_INDEX, a release build records nothing.  No
 * memory is accessed either way.  (The pages have no counterpart of these two calls.)
 */
NVFP4_API int nvfp4_debug_index_checks(void);
NVFP4_API int nvfp4_selftest_index_check(nvfp4_stream_t stream);
NVFP4_API int nvfp4_selftest_gemm_stall(const uint8_t *a, const uint8_t *b, const uint8_t *a_sf,
                                        const uint8_t *b_sf, const float *alpha, void *out_bf16, int64_t m,
                                        int64_t n, int64_t k, nvfp4_stream_t stream);
NVFP4_API int nvfp4_selftest_grid_barrier(const void *x_bf16, int64_t m, int64_t k, float *gsf_out,
                                          uint8_t *q_out, uint8_t *sf_out, nvfp4_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
