// bf16a.cu -- the bf16-activation NVFP4 linear: dynamic global scale and NVFP4 quantization
// of the activation, then the block-scaled FP4 GEMM against an NVFP4 weight.
//
// Source (page title, section): NVIDIA/Fuser PR #5737 "Benchmark for nvfp4 scaled mm",
// description and reviewer guide: f16a_nvfp4weight_scaled_mm(activation_bf16, fp4_weight,
// weight_scaling_factor, weight_global_scale) -> bf16 [M, N], which the compiler path runs
// as a block quantization of the activation followed by the scaled FP4 matmul.
//
// Two launches of this library on the caller's stream: nvfp4_global_scale_quantize (the
// activation's amax, gsf = 448*6/amax and alpha from the weight's amax, and the quantized
// activation, in one cooperative launch) and nvfp4_gemm, which programmatic dependent launch
// lets start its set-up while the first one finishes.  The quantized activation goes to
// caller-provided workspace, so the call allocates nothing.
//
// With a static (calibrated) activation scale [TensorRT-LLM create_weights: input_scale] the
// amax pass drops out.  Two forms: nvfp4_quantize then nvfp4_gemm (PDL-chained), or one GEMM
// launch whose epilogue warps quantize the activation before they drain any accumulator.  The
// first is the faster on B200 at every measured shape: the GEMM's four or eight epilogue warps
// per SM convert bf16 to e2m1 far slower than the standalone quantizer at full occupancy, and
// until every slab's first K chunks are done the mainloop waits.
#include "common.cuh"

namespace {

// the argument checks both bf16-activation forms share; an invalid call writes nothing
int check_bf16a(const void* a_bf16, const uint8_t* b, const uint8_t* b_sf, const void* bias_bf16, void* out_bf16,
                uint8_t* a_q_ws, uint8_t* a_sf_ws, int64_t m, int64_t n, int64_t k) {
  using nvfp4::aligned;
  if (m < 0 || n < 0 || k <= 0 || k % 64 != 0 || n % 8 != 0) return NVFP4_ERR_INVALID_ARGUMENT;
  if (m > (1 << 30) || n > (1 << 29) || k > (1 << 30)) return NVFP4_ERR_INVALID_ARGUMENT;
  if (m > 0 && (!a_bf16 || !a_q_ws || !a_sf_ws)) return NVFP4_ERR_INVALID_ARGUMENT;
  if (m > 0 && n > 0 && (!b || !b_sf || !out_bf16)) return NVFP4_ERR_INVALID_ARGUMENT;
  if ((a_bf16 && !aligned(a_bf16, 16)) || (a_q_ws && !aligned(a_q_ws, 16)) || (a_sf_ws && !aligned(a_sf_ws, 16)) ||
      (b && !aligned(b, 16)) || (b_sf && !aligned(b_sf, 16)) || (out_bf16 && !aligned(out_bf16, 16)) ||
      (bias_bf16 && !aligned(bias_bf16, 16)))
    return NVFP4_ERR_INVALID_ARGUMENT;
  return NVFP4_OK;
}

}  // namespace

extern "C" int nvfp4_gemm_bf16a(const void* a_bf16, const uint8_t* b, const uint8_t* b_sf, const float* b_amax,
                                const void* bias_bf16, void* out_bf16, uint8_t* a_q_ws, uint8_t* a_sf_ws,
                                float* scalars_ws, int64_t m, int64_t n, int64_t k, nvfp4_stream_t stream) {
  using namespace nvfp4;
  // every argument of both launches is checked first, so an invalid call writes nothing
  int st = check_bf16a(a_bf16, b, b_sf, bias_bf16, out_bf16, a_q_ws, a_sf_ws, m, n, k);
  if (st != NVFP4_OK) return st;
  if (!b_amax || !scalars_ws || !aligned(scalars_ws, 4) || !aligned(b_amax, 4)) return NVFP4_ERR_INVALID_ARGUMENT;
  // scalars_ws: [0] amax of the activation, [1] its global scale, [2] alpha
  st = nvfp4_global_scale_quantize(a_bf16, m, k, scalars_ws, scalars_ws + 1, b_amax, scalars_ws + 2, a_q_ws,
                                   a_sf_ws, stream);
  if (st != NVFP4_OK || m == 0 || n == 0) return st;
  return nvfp4_gemm(a_q_ws, b, a_sf_ws, b_sf, scalars_ws + 2, bias_bf16, out_bf16, m, n, k, stream);
}

extern "C" int nvfp4_gemm_bf16a_static(const void* a_bf16, const uint8_t* b, const uint8_t* b_sf, const float* a_gsf,
                                       const float* alpha, const void* bias_bf16, void* out_bf16, uint8_t* a_q_ws,
                                       uint8_t* a_sf_ws, int64_t m, int64_t n, int64_t k, int one_launch,
                                       nvfp4_stream_t stream) {
  using namespace nvfp4;
  int st = check_bf16a(a_bf16, b, b_sf, bias_bf16, out_bf16, a_q_ws, a_sf_ws, m, n, k);
  if (st != NVFP4_OK) return st;
  if (!a_gsf || !alpha || !aligned(a_gsf, 4) || !aligned(alpha, 4)) return NVFP4_ERR_INVALID_ARGUMENT;
  if (one_launch != 0 && one_launch != 1) return NVFP4_ERR_INVALID_ARGUMENT;
  if (one_launch && k > 16384) return NVFP4_ERR_INVALID_ARGUMENT;
  if (m == 0) return NVFP4_OK;
  if (n == 0 || !one_launch) {
    // no output (only the workspace is written), or the two-launch form
    st = nvfp4_quantize(a_bf16, m, k, a_gsf, a_q_ws, a_sf_ws, stream);
    if (st != NVFP4_OK || n == 0) return st;
    return nvfp4_gemm(a_q_ws, b, a_sf_ws, b_sf, alpha, bias_bf16, out_bf16, m, n, k, stream);
  }
  return gemm_quantize_a(a_bf16, b, b_sf, a_gsf, alpha, bias_bf16, out_bf16, a_q_ws, a_sf_ws, m, n, k, stream);
}
