/*
 * nvfp4_oracle.c -- plain, slow CPU oracle for NVFP4 (16-element block) quantization
 * and block-scaled FP4 GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load this
 * file.  Its only users are the tests, the smoke check and the CPU-baseline leg of the
 * benchmark.  It shares no code, header, table or constant generator with the CUDA
 * library; the two are written independently from the same pages.
 *
 * Style rules (so a reader can check it against the definitions by eye):
 *   - every value is produced by its definition, one element at a time, in the order
 *     the definition states; no blocking, no fusion, no vectorisation;
 *   - encoders are exhaustive nearest-value searches over the code table (ties go to
 *     the even code), decoders evaluate the bit-field definition;
 *   - fp32 steps are single IEEE operations (built with -ffp-contract=off, no fast
 *     math); GEMM references are accumulated in fp64;
 *   - OpenMP only splits independent rows across threads; it does not change any
 *     arithmetic.
 *
 * Sources (cited by page title and section):
 *   [TRT]  TensorRT-LLM NVFP4LinearMethod.create_weights: the
 *          [out, in/2] packed weight, the block-16 scale buffer padded to
 *          pad_up(rows,128) x pad_up(in/16,4), input_scale = 448*6/amax_input,
 *          alpha = amax_input*amax_weight/(448*6*448*6).
 *   [FV]   FastVideo PR #1350 "Add NVFP4QAT linear layer", code-review thread: the
 *          _global_sf helper (abs, nan_to_num, max, clamp(min=1e-12), 448*6/maxabs).
 *   [FI3]  flashinfer PR #1774 "Masked batch nvfp4 quantization": masked batched
 *          quantize, per-item global scale, silu_and_mul with 2*hidden -> hidden,
 *          uint8 outputs [b, m, k/2] and [b, m*k/16].
 *   [FI5]  flashinfer docs flashinfer.gemm.mm_nvfp4_svdquant, signature and
 *          Parameters: packed e2m1 operands (m, k/2) and (n, k/2), ue4m3 block scales
 *          in the 128x4 swizzled layout with numel ceil(m/128)*128*ceil(k/16/4)*4,
 *          alpha device scalar, d (m, r), l1 (n, r) pre-divided by alpha, bias (n,),
 *          epilogue out = alpha*acc + bias.
 * Readings where the pages are silent are named R1..R13 in the comments below.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define NVO_API __attribute__((visibility("default")))

static int g_threads = 1;

NVO_API void nvo_set_threads(int n) { g_threads = n > 0 ? n : 1; }
NVO_API int nvo_get_threads(void) { return g_threads; }

/* ------------------------------------------------------------------------------- */
/* bf16 <-> fp32                                                                    */
/* ------------------------------------------------------------------------------- */

static float bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round-to-nearest-even fp32 -> bf16 (finite inputs; NaN maps to a quiet NaN). */
static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

NVO_API uint16_t nvo_f32_to_bf16(float f) { return f32_to_bf16_rne(f); }
NVO_API float nvo_bf16_to_f32(uint16_t h) { return bf16_to_f32(h); }

/* ------------------------------------------------------------------------------- */
/* FP4 e2m1: the value grid {0, 0.5, 1, 1.5, 2, 3, 4, 6} with a sign bit (bit 3).    */
/* ------------------------------------------------------------------------------- */

static const double E2M1_MAGNITUDE[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

NVO_API double nvo_e2m1_value(uint8_t code) {
    double mag = E2M1_MAGNITUDE[code & 7u];
    return (code & 8u) ? -mag : mag;
}

/*
 * Nearest e2m1 code to v: the magnitude is the grid value nearest |v| (ties to the
 * even code, i.e. the code whose last bit is 0); values beyond 6 saturate to 6 (the
 * nearest grid value anyway).  The sign bit is signbit(v), so a negative value that
 * rounds to zero gives code 0x8 (reading R5).
 */
NVO_API uint8_t nvo_e2m1_encode(float v) {
    double a = fabs((double)v);
    if (a >= 6.0) return (uint8_t)(7 | (signbit(v) ? 8 : 0));   /* satfinite */
    int best = 0;
    double best_err = fabs(a - E2M1_MAGNITUDE[0]);
    for (int c = 1; c < 8; ++c) {
        double err = fabs(a - E2M1_MAGNITUDE[c]);
        if (err < best_err || (err == best_err && (c % 2) == 0 && (best % 2) != 0)) {
            best = c;
            best_err = err;
        }
    }
    return (uint8_t)(best | (signbit(v) ? 8 : 0));
}

/* ------------------------------------------------------------------------------- */
/* Scale format ue4m3: fp8 e4m3 without its sign, bias 7, codes 0x00..0x7E finite.   */
/* ------------------------------------------------------------------------------- */

NVO_API double nvo_e4m3_value(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 15;
    int m = code & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;            /* 0x7F / 0xFF are NaN */
    if (e == 0) mag = ldexp((double)m, -9);      /* subnormal: m/8 * 2^-6 */
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* The 127 finite non-negative e4m3 values, filled once from the definition above. */
static double UE4M3_VALUE[0x7F];

__attribute__((constructor)) static void fill_ue4m3_table(void) {
    for (int c = 0; c <= 0x7E; ++c) UE4M3_VALUE[c] = nvo_e4m3_value((uint8_t)c);
}

/*
 * Nearest non-negative finite e4m3 code to s >= 0 (reading R3: round to nearest,
 * ties to the even code, saturate at 448 = code 0x7E).
 */
NVO_API uint8_t nvo_ue4m3_encode(float s) {
    double a = (double)s;
    if (a >= 448.0) return 0x7E;                                  /* satfinite */
    int best = 0;
    double best_err = fabs(a - UE4M3_VALUE[0]);
    for (int c = 1; c <= 0x7E; ++c) {
        double err = fabs(a - UE4M3_VALUE[c]);
        if (err < best_err || (err == best_err && (c % 2) == 0 && (best % 2) != 0)) {
            best = c;
            best_err = err;
        }
    }
    return (uint8_t)best;
}

/* ------------------------------------------------------------------------------- */
/* Scale-buffer geometry [TRT] padding comment, [FI5] a_sf parameter.               */
/* ------------------------------------------------------------------------------- */

static int64_t pad_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

/* pad_up(rows, 128) * pad_up(k/16, 4) bytes. */
NVO_API int64_t nvo_scale_bytes(int64_t rows, int64_t k) {
    return pad_up(rows, 128) * pad_up(k / 16, 4);
}

/*
 * Byte offset of the scale of row r, scale column c (c = 16-element block index
 * along K) in the 128x4 swizzled layout (reading R6): the buffer is a sequence of
 * 512-byte chunks, one per (128-row tile, 4-column group), ordered with the column
 * group fastest; inside a chunk, byte (r%32)*16 + ((r%128)/32)*4 + c%4.
 */
NVO_API int64_t nvo_sf_offset(int64_t r, int64_t c, int64_t k) {
    int64_t groups = pad_up(k / 16, 4) / 4;
    int64_t chunk = (r / 128) * groups + c / 4;
    return chunk * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

/* ------------------------------------------------------------------------------- */
/* Global scale [FV] _global_sf, [TRT] input_scale and alpha.                       */
/* ------------------------------------------------------------------------------- */

/* |x| with NaN -> 0 and +-Inf -> FLT_MAX (torch.nan_to_num defaults). */
static float abs_nan_to_num(float x) {
    float a = fabsf(x);
    if (isnan(a)) return 0.0f;
    if (isinf(a)) return FLT_MAX;
    return a;
}

static void finish_global_scale(float amax, float *amax_out, float *gsf_out) {
    if (amax < 1e-12f) amax = 1e-12f;      /* clamp(min=1e-12) */
    if (amax_out) *amax_out = amax;
    *gsf_out = 2688.0f / amax;             /* (448 * 6) / maxabs, fp32 */
}

NVO_API void nvo_global_scale(const uint16_t *x, int64_t numel, float *amax_out, float *gsf_out) {
    float amax = 0.0f;
    for (int64_t i = 0; i < numel; ++i) {
        float a = abs_nan_to_num(bf16_to_f32(x[i]));
        if (a > amax) amax = a;
    }
    finish_global_scale(amax, amax_out, gsf_out);
}

/* alpha = amax_a * amax_b / (448*6 * 448*6) in fp32 ([TRT] alpha comment). */
NVO_API float nvo_alpha(float amax_a, float amax_b) {
    float prod = amax_a * amax_b;
    return prod / 7225344.0f;            /* 2688 * 2688 */
}

/* ------------------------------------------------------------------------------- */
/* Specified fp32 exp for SiLU (reading R8).                                        */
/*                                                                                  */
/* Cody-Waite range reduction x = n*ln2 + r with ln2 split in a 16-significant-bit  */
/* head and an fp32 tail, then the degree-7 Taylor polynomial of e^r by Horner with */
/* fused multiply-adds, then an exact scaling by 2^n.  Every step is one correctly  */
/* rounded fp32 operation, so any IEEE implementation reproduces it bit for bit.    */
/* ------------------------------------------------------------------------------- */

static float pow2i(int n) {          /* 2^n for -126 <= n <= 127, exact */
    uint32_t u = (uint32_t)(n + 127) << 23;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

NVO_API float nvo_exp_spec(float x) {
    if (isnan(x)) return x;
    if (x > 89.0f) return INFINITY;
    if (x < -104.0f) return 0.0f;
    const float log2e = 0x1.715476p+0f;
    const float ln2_hi = 0x1.62e4p-1f;
    const float ln2_lo = 0x1.7f7d1cp-20f;
    float n = rintf(x * log2e);
    float r = fmaf(n, -ln2_hi, x);
    r = fmaf(n, -ln2_lo, r);
    float p = 0x1.a01a02p-13f;           /* 1/7! */
    p = fmaf(p, r, 0x1.6c16c2p-10f);     /* 1/6! */
    p = fmaf(p, r, 0x1.111112p-7f);      /* 1/5! */
    p = fmaf(p, r, 0x1.555556p-5f);      /* 1/4! */
    p = fmaf(p, r, 0x1.555556p-3f);      /* 1/3! */
    p = fmaf(p, r, 0x1.0p-1f);           /* 1/2! */
    p = fmaf(p, r, 1.0f);                /* 1/1! */
    p = fmaf(p, r, 1.0f);                /* 1/0! */
    int ni = (int)n;
    if (ni > 127) return (p * pow2i(127)) * pow2i(ni - 127);
    if (ni < -126) return (p * pow2i(-126)) * pow2i(ni + 126);
    return p * pow2i(ni);
}

/* h = bf16( (g / (1 + exp(-g))) * u ), each step one fp32 op (reading R8). */
NVO_API uint16_t nvo_silu_mul_bf16(uint16_t g_bits, uint16_t u_bits) {
    float g = bf16_to_f32(g_bits);
    float u = bf16_to_f32(u_bits);
    float e = nvo_exp_spec(-g);
    float den = 1.0f + e;
    float s = g / den;
    float p = s * u;
    return f32_to_bf16_rne(p);
}

/* ------------------------------------------------------------------------------- */
/* Block quantization of one row of k bf16 values (k % 16 == 0).                    */
/*   per 16-element block j:                                                        */
/*     vmax = max |x|                                                               */
/*     s32  = (vmax / 6) * gsf                (reading R2)                          */
/*     s8   = ue4m3(s32)                      (reading R3)                          */
/*     inv  = s8 == 0 ? 0 : gsf / value(s8)   (reading R4)                          */
/*     code = e2m1(x * inv)                   (reading R5)                          */
/*   packing: byte 8j+i of the row holds code[16j+2i] (low nibble) and             */
/*   code[16j+2i+1] (high nibble)              (reading R7)                          */
/* ------------------------------------------------------------------------------- */

static void quantize_row(const float *xr, int64_t k, float gsf, uint8_t *qr, uint8_t *sf,
                         int64_t row, int64_t kfull) {
    int64_t nb = k / 16;
    for (int64_t j = 0; j < nb; ++j) {
        const float *blk = xr + 16 * j;
        float vmax = 0.0f;
        for (int e = 0; e < 16; ++e) {
            float a = fabsf(blk[e]);
            if (a > vmax) vmax = a;
        }
        float s32 = (vmax / 6.0f) * gsf;
        uint8_t s8 = nvo_ue4m3_encode(s32);
        float sd = (float)nvo_e4m3_value(s8);
        float inv = (sd == 0.0f) ? 0.0f : gsf / sd;
        uint8_t code[16];
        for (int e = 0; e < 16; ++e) code[e] = nvo_e2m1_encode(blk[e] * inv);
        for (int i = 0; i < 8; ++i)
            qr[8 * j + i] = (uint8_t)(code[2 * i] | (code[2 * i + 1] << 4));
        sf[nvo_sf_offset(row, j, kfull)] = s8;
    }
}

/* Scale entries of a valid row beyond its last block (padding columns) are 0 (R9). */
static void zero_row_padding_cols(uint8_t *sf, int64_t row, int64_t k) {
    int64_t nb = k / 16;
    for (int64_t c = nb; c < pad_up(nb, 4); ++c) sf[nvo_sf_offset(row, c, k)] = 0;
}

static void zero_padding_rows(uint8_t *sf, int64_t m, int64_t k) {
    int64_t cpad = pad_up(k / 16, 4);
    for (int64_t r = m; r < pad_up(m, 128); ++r)
        for (int64_t c = 0; c < cpad; ++c) sf[nvo_sf_offset(r, c, k)] = 0;
}

/* Dense quantize: x [m, k] -> q [m, k/2], sf [scale_bytes(m, k)]. */
NVO_API void nvo_quantize(const uint16_t *x, int64_t m, int64_t k, float gsf, uint8_t *q, uint8_t *sf) {
    #pragma omp parallel for schedule(static) num_threads(g_threads)
    for (int64_t r = 0; r < m; ++r) {
        float xr[k > 0 ? k : 1];
        for (int64_t i = 0; i < k; ++i) xr[i] = bf16_to_f32(x[r * k + i]);
        quantize_row(xr, k, gsf, q + r * (k / 2), sf, r, k);
        zero_row_padding_cols(sf, r, k);
    }
    zero_padding_rows(sf, m, k);
}

/*
 * Masked batched quantize [FI3]: item i of x [b, m, k] uses gsf[i]; only rows
 * r < mask[i] are written (mask == NULL means every row); other rows of q and their
 * scale entries are left untouched (reading R11).  Item i writes q + i*m*k/2 and
 * sf + i*scale_bytes(m, k).  With mask == NULL the padding rows are zeroed as in
 * the dense quantizer.
 */
NVO_API void nvo_quantize_masked_batched(const uint16_t *x, int64_t b, int64_t m, int64_t k,
                                         const int32_t *mask, const float *gsf,
                                         uint8_t *q, uint8_t *sf) {
    int64_t sb = nvo_scale_bytes(m, k);
    for (int64_t i = 0; i < b; ++i) {
        int64_t valid = mask ? (int64_t)mask[i] : m;
        if (valid > m) valid = m;
        if (valid < 0) valid = 0;
        const uint16_t *xi = x + i * m * k;
        uint8_t *qi = q + i * m * (k / 2);
        uint8_t *sfi = sf + i * sb;
        #pragma omp parallel for schedule(static) num_threads(g_threads)
        for (int64_t r = 0; r < valid; ++r) {
            float xr[k > 0 ? k : 1];
            for (int64_t c = 0; c < k; ++c) xr[c] = bf16_to_f32(xi[r * k + c]);
            quantize_row(xr, k, gsf[i], qi + r * (k / 2), sfi, r, k);
            zero_row_padding_cols(sfi, r, k);
        }
        if (!mask) zero_padding_rows(sfi, m, k);
    }
}

/*
 * SiLU-and-mul fused quantize [FI3]: x [b, m, 2k]; gate g = x[..., c], up u =
 * x[..., k + c] for c < k (reading R8: gate is the first half); h = bf16(silu(g)*u)
 * [b, m, k] is then quantized exactly as nvo_quantize_masked_batched.
 */
NVO_API void nvo_silu_mul_quantize_batched(const uint16_t *x, int64_t b, int64_t m, int64_t k,
                                           const int32_t *mask, const float *gsf,
                                           uint8_t *q, uint8_t *sf) {
    int64_t sb = nvo_scale_bytes(m, k);
    for (int64_t i = 0; i < b; ++i) {
        int64_t valid = mask ? (int64_t)mask[i] : m;
        if (valid > m) valid = m;
        if (valid < 0) valid = 0;
        const uint16_t *xi = x + i * m * 2 * k;
        uint8_t *qi = q + i * m * (k / 2);
        uint8_t *sfi = sf + i * sb;
        #pragma omp parallel for schedule(static) num_threads(g_threads)
        for (int64_t r = 0; r < valid; ++r) {
            float hr[k > 0 ? k : 1];
            for (int64_t c = 0; c < k; ++c)
                hr[c] = bf16_to_f32(nvo_silu_mul_bf16(xi[r * 2 * k + c], xi[r * 2 * k + k + c]));
            quantize_row(hr, k, gsf[i], qi + r * (k / 2), sfi, r, k);
            zero_row_padding_cols(sfi, r, k);
        }
        if (!mask) zero_padding_rows(sfi, m, k);
    }
}

/* h = bf16(silu(g) * u) for a whole [rows, 2k] tensor (test helper). */
NVO_API void nvo_silu_mul(const uint16_t *x, int64_t rows, int64_t k, uint16_t *h) {
    #pragma omp parallel for schedule(static) num_threads(g_threads)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < k; ++c)
            h[r * k + c] = nvo_silu_mul_bf16(x[r * 2 * k + c], x[r * 2 * k + k + c]);
}

/*
 * Per-item global scale over valid rows (reading R1): amax over rows r < mask[i]
 * (all rows when mask == NULL) of item i; with silu_mul != 0 the amax is taken over
 * h = bf16(silu(g)*u) of x [b, m, 2k], otherwise over x [b, m, k].
 */
NVO_API void nvo_global_scale_batched(const uint16_t *x, int64_t b, int64_t m, int64_t k,
                                      const int32_t *mask, int silu_mul,
                                      float *amax_out, float *gsf_out) {
    int64_t width = silu_mul ? 2 * k : k;
    for (int64_t i = 0; i < b; ++i) {
        int64_t valid = mask ? (int64_t)mask[i] : m;
        if (valid > m) valid = m;
        if (valid < 0) valid = 0;
        const uint16_t *xi = x + i * m * width;
        float amax = 0.0f;
        for (int64_t r = 0; r < valid; ++r) {
            for (int64_t c = 0; c < k; ++c) {
                uint16_t v = silu_mul ? nvo_silu_mul_bf16(xi[r * width + c], xi[r * width + k + c])
                                      : xi[r * width + c];
                float a = abs_nan_to_num(bf16_to_f32(v));
                if (a > amax) amax = a;
            }
        }
        finish_global_scale(amax, amax_out ? amax_out + i : NULL, gsf_out + i);
    }
}

/* ------------------------------------------------------------------------------- */
/* Logical decode: value(q) * value(s8) for every element (gsf not applied).        */
/* ------------------------------------------------------------------------------- */

static double logical_value(const uint8_t *q, const uint8_t *sf, int64_t row, int64_t col, int64_t k) {
    uint8_t byte = q[row * (k / 2) + col / 2];
    uint8_t code = (col % 2) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15u);
    uint8_t s8 = sf[nvo_sf_offset(row, col / 16, k)];
    return nvo_e2m1_value(code) * nvo_e4m3_value(s8);
}

NVO_API void nvo_dequantize_logical(const uint8_t *q, const uint8_t *sf, int64_t rows, int64_t k, double *out) {
    #pragma omp parallel for schedule(static) num_threads(g_threads)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < k; ++c) out[r * k + c] = logical_value(q, sf, r, c, k);
}

/* ------------------------------------------------------------------------------- */
/* GEMM reference in fp64 [FI5] description and Parameters, [TRT] alpha:            */
/*   ref[i,j] = alpha * ( sum_k A[i,k]*B[j,k] + sum_t d[i,t]*l1[j,t] ) + bias[j]     */
/* with A, B the logical values above; d, l1, bias optional (NULL).                 */
/* ------------------------------------------------------------------------------- */

static double ref_element(const uint8_t *a, const uint8_t *b, const uint8_t *a_sf, const uint8_t *b_sf,
                          double alpha, const uint16_t *d, const uint16_t *l1, int64_t r,
                          const uint16_t *bias, int64_t i, int64_t j, int64_t k) {
    double acc = 0.0;
    for (int64_t c = 0; c < k; ++c)
        acc += logical_value(a, a_sf, i, c, k) * logical_value(b, b_sf, j, c, k);
    if (d && l1)
        for (int64_t t = 0; t < r; ++t)
            acc += (double)bf16_to_f32(d[i * r + t]) * (double)bf16_to_f32(l1[j * r + t]);
    double out = alpha * acc;
    if (bias) out += (double)bf16_to_f32(bias[j]);
    return out;
}

NVO_API void nvo_gemm_ref(const uint8_t *a, const uint8_t *b, const uint8_t *a_sf, const uint8_t *b_sf,
                          float alpha, const uint16_t *d, const uint16_t *l1, int64_t r,
                          const uint16_t *bias, int64_t m, int64_t n, int64_t k, double *out) {
    #pragma omp parallel for schedule(dynamic, 1) num_threads(g_threads)
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < n; ++j)
            out[i * n + j] = ref_element(a, b, a_sf, b_sf, (double)alpha, d, l1, r, bias, i, j, k);
}

/* The same reference at listed (i, j) positions only. */
NVO_API void nvo_gemm_ref_sampled(const uint8_t *a, const uint8_t *b, const uint8_t *a_sf, const uint8_t *b_sf,
                                  float alpha, const uint16_t *d, const uint16_t *l1, int64_t r,
                                  const uint16_t *bias, int64_t k, const int64_t *ii, const int64_t *jj,
                                  int64_t count, double *out) {
    #pragma omp parallel for schedule(dynamic, 16) num_threads(g_threads)
    for (int64_t s = 0; s < count; ++s)
        out[s] = ref_element(a, b, a_sf, b_sf, (double)alpha, d, l1, r, bias, ii[s], jj[s], k);
}

/*
 * Masked grouped GEMM reference (reading R13): for expert e and row i < mask[e],
 * out[e, i, :] = alpha[e] * A_e[i, :] . B_e^T with A_e = a + e*mmax*k/2 and
 * a_sf + e*scale_bytes(mmax, k), B_e = b + e*n*k/2 and b_sf + e*scale_bytes(n, k).
 * Rows i >= mask[e] of out are not written.
 */
NVO_API void nvo_grouped_gemm_ref(const uint8_t *a, const uint8_t *b, const uint8_t *a_sf, const uint8_t *b_sf,
                                  const int32_t *mask, const float *alpha, int64_t E, int64_t mmax,
                                  int64_t n, int64_t k, double *out) {
    int64_t sba = nvo_scale_bytes(mmax, k), sbb = nvo_scale_bytes(n, k);
    for (int64_t e = 0; e < E; ++e) {
        int64_t valid = mask[e] < 0 ? 0 : (mask[e] > mmax ? mmax : mask[e]);
        const uint8_t *ae = a + e * mmax * (k / 2), *be = b + e * n * (k / 2);
        const uint8_t *ase = a_sf + e * sba, *bse = b_sf + e * sbb;
        #pragma omp parallel for schedule(dynamic, 1) num_threads(g_threads)
        for (int64_t i = 0; i < valid; ++i)
            for (int64_t j = 0; j < n; ++j)
                out[(e * mmax + i) * n + j] =
                    ref_element(ae, be, ase, bse, (double)alpha[e], NULL, NULL, 0, NULL, i, j, k);
    }
}

/* ------------------------------------------------------------------------------- */
/* SwiGLU first half: gate/up projections, then SiLU-and-mul quantization           */
/* [NVF] NVIDIA/Fuser PR #5737, module tree: NVFP4InferenceSwiGLU (gate_proj,       */
/* up_proj, down_proj) and its grouped form for the routed experts; [FI3] the        */
/* silu_and_mul quantizer that consumes [gate | up].                                 */
/*   g = bf16(alpha_gate * A.Bg^T),  u = bf16(alpha_up * A.Bu^T)                     */
/*   (q, sf) = nvo_silu_mul_quantize_batched([g | u], gsf_h)                         */
/* The projections are the fp64 GEMM reference rounded once to bf16.                 */
/* ------------------------------------------------------------------------------- */

/* bf16 nearest to the double v, ties to even: 8 significant bits, fp32's exponent
 * range (subnormal spacing 2^-133), overflow to infinity. */
static uint16_t f64_to_bf16_rne(double v) {
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);                           /* 2^(e-1) <= a < 2^e */
    int q = e - 8;                          /* spacing of 8 significant bits */
    if (q < -133) q = -133;
    double r = ldexp(nearbyint(ldexp(a, -q)), q);   /* default mode: ties to even */
    if (r > 0x1.FEp127) return sign | 0x7F80;
    float f = (float)r;                     /* exact */
    uint32_t bits;
    memcpy(&bits, &f, 4);
    return sign | (uint16_t)(bits >> 16);
}

NVO_API uint16_t nvo_f64_to_bf16(double v) { return f64_to_bf16_rne(v); }

/* [g | u] rows (bf16 bits, [rows, 2n]) for rows ii[0..count) of A. */
static void gate_up_rows(const uint8_t *a, const uint8_t *b_gate, const uint8_t *b_up, const uint8_t *a_sf,
                         const uint8_t *b_gate_sf, const uint8_t *b_up_sf, float alpha_gate, float alpha_up,
                         int64_t n, int64_t k, const int64_t *ii, int64_t count, uint16_t *x) {
    #pragma omp parallel for schedule(dynamic, 1) num_threads(g_threads)
    for (int64_t s = 0; s < count; ++s)
        for (int64_t j = 0; j < n; ++j) {
            double g = ref_element(a, b_gate, a_sf, b_gate_sf, (double)alpha_gate, NULL, NULL, 0, NULL, ii[s], j, k);
            double u = ref_element(a, b_up, a_sf, b_up_sf, (double)alpha_up, NULL, NULL, 0, NULL, ii[s], j, k);
            x[s * 2 * n + j] = f64_to_bf16_rne(g);
            x[s * 2 * n + n + j] = f64_to_bf16_rne(u);
        }
}

/* The bf16 [g | u] rows ii[0..count) -> x [count, 2n] (e.g. to calibrate gsf_h). */
NVO_API void nvo_gemm_gate_up_bf16(const uint8_t *a, const uint8_t *b_gate, const uint8_t *b_up,
                                   const uint8_t *a_sf, const uint8_t *b_gate_sf, const uint8_t *b_up_sf,
                                   float alpha_gate, float alpha_up, int64_t n, int64_t k, const int64_t *ii,
                                   int64_t count, uint16_t *x) {
    gate_up_rows(a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf, alpha_gate, alpha_up, n, k, ii, count, x);
}

/* Dense: a [m, k/2], b_gate / b_up [n, k/2] -> q [m, n/2], sf [scale_bytes(m, n)]. */
NVO_API void nvo_gemm_silu_mul_quantize(const uint8_t *a, const uint8_t *b_gate, const uint8_t *b_up,
                                        const uint8_t *a_sf, const uint8_t *b_gate_sf, const uint8_t *b_up_sf,
                                        float alpha_gate, float alpha_up, float gsf_h, int64_t m, int64_t n,
                                        int64_t k, uint8_t *q, uint8_t *sf) {
    uint16_t *x = (uint16_t *)malloc((size_t)(m > 0 ? m : 1) * 2 * n * sizeof(uint16_t));
    int64_t *ii = (int64_t *)malloc((size_t)(m > 0 ? m : 1) * sizeof(int64_t));
    for (int64_t i = 0; i < m; ++i) ii[i] = i;
    gate_up_rows(a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf, alpha_gate, alpha_up, n, k, ii, m, x);
    nvo_silu_mul_quantize_batched(x, 1, m, n, NULL, &gsf_h, q, sf);
    free(ii);
    free(x);
}

/* Masked grouped: per expert e, rows i < mask[e] only (other rows and their scale
 * entries untouched), with alpha_gate[e], alpha_up[e], gsf_h[e]. */
NVO_API void nvo_grouped_gemm_silu_mul_quantize(const uint8_t *a, const uint8_t *b_gate, const uint8_t *b_up,
                                                const uint8_t *a_sf, const uint8_t *b_gate_sf,
                                                const uint8_t *b_up_sf, const int32_t *mask,
                                                const float *alpha_gate, const float *alpha_up,
                                                const float *gsf_h, int64_t E, int64_t mmax, int64_t n,
                                                int64_t k, uint8_t *q, uint8_t *sf) {
    int64_t sba = nvo_scale_bytes(mmax, k), sbb = nvo_scale_bytes(n, k), sbh = nvo_scale_bytes(mmax, n);
    uint16_t *x = (uint16_t *)calloc((size_t)(mmax > 0 ? mmax : 1) * 2 * n, sizeof(uint16_t));
    int64_t *ii = (int64_t *)malloc((size_t)(mmax > 0 ? mmax : 1) * sizeof(int64_t));
    for (int64_t i = 0; i < mmax; ++i) ii[i] = i;
    for (int64_t e = 0; e < E; ++e) {
        int64_t valid = mask[e] < 0 ? 0 : (mask[e] > mmax ? mmax : mask[e]);
        gate_up_rows(a + e * mmax * (k / 2), b_gate + e * n * (k / 2), b_up + e * n * (k / 2), a_sf + e * sba,
                     b_gate_sf + e * sbb, b_up_sf + e * sbb, alpha_gate[e], alpha_up[e], n, k, ii, valid, x);
        nvo_silu_mul_quantize_batched(x, 1, mmax, n, mask + e, gsf_h + e, q + e * mmax * (n / 2), sf + e * sbh);
    }
    free(ii);
    free(x);
}

/* Rows ii[0..count) of the dense result, each quantized on its own: q_rows [count, n/2]
 * and the row's scale codes in logical order, s_rows [count, n/16]. */
NVO_API void nvo_gemm_silu_mul_quantize_rows(const uint8_t *a, const uint8_t *b_gate, const uint8_t *b_up,
                                             const uint8_t *a_sf, const uint8_t *b_gate_sf,
                                             const uint8_t *b_up_sf, float alpha_gate, float alpha_up,
                                             float gsf_h, int64_t n, int64_t k, const int64_t *ii,
                                             int64_t count, uint8_t *q_rows, uint8_t *s_rows) {
    uint16_t *x = (uint16_t *)malloc((size_t)(count > 0 ? count : 1) * 2 * n * sizeof(uint16_t));
    uint8_t *sf1 = (uint8_t *)malloc((size_t)nvo_scale_bytes(1, n));
    gate_up_rows(a, b_gate, b_up, a_sf, b_gate_sf, b_up_sf, alpha_gate, alpha_up, n, k, ii, count, x);
    for (int64_t s = 0; s < count; ++s) {
        nvo_silu_mul_quantize_batched(x + s * 2 * n, 1, 1, n, NULL, &gsf_h, q_rows + s * (n / 2), sf1);
        for (int64_t c = 0; c < n / 16; ++c) s_rows[s * (n / 16) + c] = sf1[nvo_sf_offset(0, c, n)];
    }
    free(sf1);
    free(x);
}

/* ------------------------------------------------------------------------------- */
/* SVDQuant input stage [FI5] Parameters a and d: the activation operand is x        */
/* quantized with the pre-quantization scale folded in, and d is the LoRA-down       */
/* product of x with the pre-quantization-scaled down projection.                    */
/* ------------------------------------------------------------------------------- */

/* Smooth quantize (reading R20): x_hat[r, c] = bf16(float(x[r, c]) * float(pqs[c])),
 * one fp32 multiplication rounded to bf16, then the dense quantizer with gsf. */
NVO_API void nvo_quantize_smooth(const uint16_t *x, int64_t m, int64_t k, const uint16_t *pqs, float gsf,
                                 uint8_t *q, uint8_t *sf) {
    #pragma omp parallel for schedule(static) num_threads(g_threads)
    for (int64_t r = 0; r < m; ++r) {
        float xr[k > 0 ? k : 1];
        for (int64_t i = 0; i < k; ++i) {
            float prod = bf16_to_f32(x[r * k + i]) * bf16_to_f32(pqs[i]);
            xr[i] = bf16_to_f32(f32_to_bf16_rne(prod));
        }
        quantize_row(xr, k, gsf, q + r * (k / 2), sf, r, k);
        zero_row_padding_cols(sf, r, k);
    }
    zero_padding_rows(sf, m, k);
}

/* LoRA-down: d[i, j] = sum_c x[i, c] * w[j, c] in fp64 (w = [r, k], the down projection
 * already scaled by the pre-quantization scale); out is [m, r]. */
NVO_API void nvo_lora_down(const uint16_t *x, int64_t m, int64_t k, const uint16_t *w, int64_t r, double *out) {
    #pragma omp parallel for schedule(static) num_threads(g_threads)
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t c = 0; c < k; ++c)
                acc += (double)bf16_to_f32(x[i * k + c]) * (double)bf16_to_f32(w[j * k + c]);
            out[i * r + j] = acc;
        }
}
