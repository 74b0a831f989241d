// nvfp4_math.cuh -- device arithmetic of NVFP4 quantization shared by the quantizers and
// the GEMM epilogue that quantizes SiLU(gate) * up: e4m3 / e2m1 conversions, the specified
// fp32 exponential, h = bf16(silu(g) * u), and one 16-element block (scale + codes).
//
// Sources (page title, section): TensorRT-LLM NVFP4LinearMethod.create_weights (block size
// 16, ue4m3 block scales, global scale 448*6/amax); flashinfer PR #1774 "Masked batch nvfp4
// quantization" (silu_and_mul fused variant); flashinfer docs mm_nvfp4_svdquant,
// Parameters a / a_sf (packed e2m1, 128x4-swizzled ue4m3 scales).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace nvfp4 {
namespace {

// ---- bf16 / fp8 / fp4 conversions ------------------------------------------------------

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// ue4m3 code of s >= 0: round to nearest even, saturate to 448.  Both halves of the
// packed pair convert the same value, so the pair order does not matter.
__device__ __forceinline__ uint32_t ue4m3_encode(float s) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(r) : "f"(s));
  return r & 0xffu;
}

// Exact value of an e4m3 code (through f16, which holds every e4m3 value).
__device__ __forceinline__ float e4m3_decode(uint32_t code) {
  const uint16_t pair = static_cast<uint16_t>(code | (code << 8));
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
  return __half2float(__ushort_as_half(static_cast<uint16_t>(h2 & 0xffffu)));
}

// Eight e2m1 codes, round to nearest even, saturate to +-6; element 2i goes to the low
// nibble of byte i (the cvt's second source is its low nibble).
__device__ __forceinline__ uint32_t e2m1x8(const float* t) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(t[0]), "f"(t[1]), "f"(t[2]), "f"(t[3]), "f"(t[4]), "f"(t[5]), "f"(t[6]), "f"(t[7]));
  return r;
}

// ---- the specified fp32 exponential used by SiLU -----------------------------------------
// x = n*ln2 + r (Cody-Waite, ln2 split into a 16-significant-bit head and an fp32 tail),
// e^r by the degree-7 Taylor polynomial in Horner form with fused multiply-adds, then an
// exact multiplication by 2^n (two steps when 2^n is not a normal fp32).  Every step is a
// single correctly rounded operation, so the result is reproducible bit for bit.

__device__ __forceinline__ float pow2_int(int n) { return __uint_as_float(static_cast<uint32_t>(n + 127) << 23); }

__device__ __forceinline__ float exp_specified(float x) {
  if (x != x) return x;
  if (x > 89.0f) return __uint_as_float(0x7f800000u);
  if (x < -104.0f) return 0.0f;
  const float n = rintf(__fmul_rn(x, 0x1.715476p+0f));
  float r = __fmaf_rn(n, -0x1.62e4p-1f, x);
  r = __fmaf_rn(n, -0x1.7f7d1cp-20f, r);
  float p = 0x1.a01a02p-13f;
  p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);
  p = __fmaf_rn(p, r, 0x1.111112p-7f);
  p = __fmaf_rn(p, r, 0x1.555556p-5f);
  p = __fmaf_rn(p, r, 0x1.555556p-3f);
  p = __fmaf_rn(p, r, 0x1.0p-1f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const int ni = static_cast<int>(n);
  if (ni > 127) return __fmul_rn(__fmul_rn(p, pow2_int(127)), pow2_int(ni - 127));
  if (ni < -126) return __fmul_rn(__fmul_rn(p, pow2_int(-126)), pow2_int(ni + 126));
  return __fmul_rn(p, pow2_int(ni));
}

// h = bf16(silu(g) * u), returned as the fp32 value of that bf16.
__device__ __forceinline__ float silu_mul_bf16(float g, float u) {
  const float e = exp_specified(-g);
  const float den = __fadd_rn(1.0f, e);
  const float s = __fdiv_rn(g, den);
  const float p = __fmul_rn(s, u);
  return __bfloat162float(__float2bfloat16_rn(p));
}

// ---- pairs of values in packed f32x2 registers ----------------------------------------------
// Each lane of mul.rn.f32x2 is one correctly rounded fp32 multiplication.

__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t splat2(float v) { return pack2(v, v); }

// ---- SiLU of a bf16 value: a per-device table and closed forms ----------------------------
// s(g) = g / (1 + exp_specified(-g)) (one correctly rounded addition and division) depends
// only on the 16 bits of a bf16 g, so the kernels read it from a table computed once per
// device with exactly that arithmetic, for both signs of every magnitude in [2^-25, 96):
// entry 2 * (mag - kSiluMagLo) + sign.  Outside that range s has closed forms that follow
// from the definition of exp_specified:
//   |g| < 2^-25: n = 0 and both Horner steps that add 1 round to 1, so e = 1, 1 + e = 2 and
//     s = g / 2, exact for every bf16 g (subnormal ones included);
//   g >= 96: e = exp_specified(-g) < 2^-138 is below half an ulp of 1, so 1 + e = 1, s = g;
//   g <= -96: the argument of exp_specified exceeds 89, e = +inf and s = g / inf = -0,
//     written g * 0 so that -inf and NaN give NaN as the division does.
constexpr uint32_t kSiluMagLo = 0x3300;                                 // 2^-25
constexpr uint32_t kSiluMagHi = 0x42c0;                                 // 96
constexpr uint32_t kSiluEntries = 2 * (kSiluMagHi - kSiluMagLo);        // 8064
constexpr uint32_t kSiluTableBytes = kSiluEntries * 4;                  // 32 256, a multiple of 16

// Table entry i, computed with the scalar definition.
__device__ __forceinline__ float silu_table_entry(uint32_t i) {
  const uint32_t mag = kSiluMagLo + (i >> 1);
  const float g = __uint_as_float((((i & 1u) << 15) | mag) << 16);
  return __fdiv_rn(g, __fadd_rn(1.0f, exp_specified(-g)));
}

// Table index of the bf16 pattern b (16 bits): 2 * magnitude + sign, less the start of the
// table; magnitudes outside [kSiluMagLo, kSiluMagHi) give kSiluEntries or more (unsigned).
__device__ __forceinline__ uint32_t silu_index(uint32_t b) {
  return (((b << 1) & 0xfffeu) | (b >> 15)) - 2 * kSiluMagLo;
}

// s(g) for a bf16-valued g outside the table's magnitude range.
__device__ __forceinline__ float silu_closed(float g) {
  const uint32_t b = __float_as_uint(g) >> 16;
  const float f = (b & 0x7fffu) < kSiluMagLo ? 0.5f : ((b & 0x8000u) ? 0.0f : 1.0f);
  return __fmul_rn(g, f);
}

// s of the two bf16 values packed in w (element 0 in the low half), from the table `tab`
// (shared memory); both loads are clamped into the table, and the rare element outside its
// range is replaced by its closed form.
__device__ __forceinline__ void silu_pair(const float* tab, uint32_t w, float& s0, float& s1) {
  const uint32_t i0 = silu_index(w & 0xffffu), i1 = silu_index(w >> 16);
  s0 = tab[min(i0, kSiluEntries - 1)];
  s1 = tab[min(i1, kSiluEntries - 1)];
  if (max(i0, i1) >= kSiluEntries) {
    if (i0 >= kSiluEntries) s0 = silu_closed(bf16_lo(w));
    if (i1 >= kSiluEntries) s1 = silu_closed(bf16_hi(w));
  }
}

// h = bf16(s(g) * u) for the pair of bf16 gate values packed in g2 and up values u0, u1, as
// fp32 values; equal to silu_mul_bf16.
__device__ __forceinline__ void silu_mul_bf16_tab2(const float* tab, uint32_t g2, float u0, float u1, float& h0,
                                                   float& h1) {
  float s0, s1;
  silu_pair(tab, g2, s0, s1);
  float p0, p1;
  unpack2(mul2(pack2(s0, s1), pack2(u0, u1)), p0, p1);
  uint32_t b2;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(b2) : "f"(p1), "f"(p0));   // p0 -> low half
  h0 = __uint_as_float(b2 << 16);
  h1 = __uint_as_float(b2 & 0xffff0000u);
}

// Copies the table from global memory into shared memory with `threads` threads starting at
// thread index `t`; the caller synchronizes before the first lookup.
__device__ __forceinline__ void silu_table_load(float* dst, const float* src, int t, int threads) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
  uint4* d = reinterpret_cast<uint4*>(dst);
  for (int i = t; i < static_cast<int>(kSiluTableBytes / 16); i += threads) d[i] = __ldg(s + i);
}

// ---- one 16-element block ------------------------------------------------------------------

struct QBlock {
  uint32_t lo, hi;  // 16 packed e2m1 codes
  uint32_t s8;      // ue4m3 scale code
};

// vmax / 6, correctly rounded, for a bf16-valued vmax >= 0: the product with fp32(1/6)
// followed by one Markstein correction step (the remainder vmax - 6q is exact as an fma,
// and q + rem/6 is rounded once).  It equals the IEEE division for every non-negative
// finite bf16 value (checked exhaustively); +inf passes through as the division would.
__device__ __forceinline__ float div6_bf16(float vmax) {
  const float q = __fmul_rn(vmax, 0x1.555556p-3f);
  const float rem = __fmaf_rn(-q, 6.0f, vmax);
  return vmax == __uint_as_float(0x7f800000u) ? vmax : __fmaf_rn(rem, 0x1.555556p-3f, q);
}

// The codes and scale of one 16-element block given its scale code s8 and the factor
// inv = gsf / e4m3(s8) (0 when the scale decodes to 0).
__device__ __forceinline__ QBlock quantize16_codes(const float* v, uint32_t s8, float inv) {
  const uint64_t inv2 = pack2(inv, inv);
  float t[16];
#pragma unroll
  for (int i = 0; i < 16; i += 2) unpack2(mul2(pack2(v[i], v[i + 1]), inv2), t[i], t[i + 1]);
  QBlock b;
  b.s8 = s8;
  b.lo = e2m1x8(t);
  b.hi = e2m1x8(t + 8);
  return b;
}

__device__ __forceinline__ uint32_t block_scale_code(const float* v, float gsf) {
  float vmax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) vmax = fmaxf(vmax, fabsf(v[i]));
  return ue4m3_encode(__fmul_rn(div6_bf16(vmax), gsf));
}

__device__ __forceinline__ float inv_scale(uint32_t s8, float gsf) {
  const float sd = e4m3_decode(s8);
  return sd == 0.0f ? 0.0f : __fdiv_rn(gsf, sd);
}

// One 16-element block of bf16-valued inputs.
__device__ __forceinline__ QBlock quantize16(const float* v, float gsf) {
  const uint32_t s8 = block_scale_code(v, gsf);
  return quantize16_codes(v, s8, inv_scale(s8, gsf));
}

// The same block with inv read from inv_tab[code] = inv_scale(code, gsf) for the 128 scale
// codes a block can get (one division per code instead of one per block).
__device__ __forceinline__ QBlock quantize16(const float* v, float gsf, const float* inv_tab) {
  const uint32_t s8 = block_scale_code(v, gsf);
  return quantize16_codes(v, s8, inv_tab[s8]);
}

// Byte offset of the scale of (row r, block c) in the 128x4 swizzled layout;
// groups = pad_up(k/16, 4) / 4.
__device__ __forceinline__ int64_t sf_offset(uint32_t r, uint32_t c, uint32_t groups) {
  const int64_t chunk = static_cast<int64_t>(r >> 7) * groups + (c >> 2);
  return chunk * 512 + (r & 31u) * 16 + ((r >> 5) & 3u) * 4 + (c & 3u);
}

}  // namespace
}  // namespace nvfp4
