// quantize.cu -- global scale (amax) reductions and the NVFP4 block quantizers.
//
// Sources (page title, section):
//   TensorRT-LLM NVFP4LinearMethod.create_weights (linear.py:871-915): block size 16,
//     [out, in/2] packed weight, scale buffer pad_up(rows,128) x pad_up(in/16,4),
//     input_scale = 448*6/amax_input, alpha = amax_in*amax_w/(448*6*448*6).
//   FastVideo PR #1350 "Add NVFP4QAT linear layer", review thread: _global_sf
//     (abs, nan_to_num, max, clamp(min=1e-12), 448*6/maxabs).
//   flashinfer PR #1774 "Masked batch nvfp4 quantization": masked batched quantize with
//     a per-item global scale, silu_and_mul fused variant (2*hidden -> hidden).
//   flashinfer docs mm_nvfp4_svdquant, Parameters a / a_sf: packed e2m1, ue4m3 scales
//     in the 128x4 swizzled layout.
//
// Design (memory-bound, HBM3e): one thread owns one 16-element block; it issues its
// 16-byte streaming loads for several blocks before computing any of them, so each SM
// keeps ~100+ KB of loads in flight.  A warp covers 32 consecutive blocks of a row
// (1 KB of contiguous bf16), stores 8 packed bytes per block (256 contiguous bytes per
// warp) and one scale byte at its swizzled position.  Conversions use the sm_100a
// round-to-nearest-even, saturate-to-finite cvt instructions.
#include <cfloat>
#include <mutex>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int kThreads = 256;

// ---- bf16 / fp8 / fp4 conversions ------------------------------------------------------

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float* f) {
  f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
  f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
  f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

__device__ __forceinline__ uint4 load_stream(const void* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}

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

// ---- the same arithmetic on pairs of values with packed f32x2 instructions -----------------
// Each lane of fma/mul/add.rn.f32x2 is one correctly rounded fp32 operation, so the pair
// functions return exactly what the scalar ones return.

__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t splat2(float v) { return pack2(v, v); }

// exp_specified of a pair.  The input is clamped to [-104, 89], which leaves every result
// unchanged (e^x overflows to +inf for x > 88.73 and rounds to 0 for x <= -104), and 2^n
// is applied as two exact power-of-two multiplications 2^(n/2) * 2^(n - n/2): both halves
// are normal numbers for n in [-150, 128], so only the last multiplication can round --
// the same single rounding as the three-way scaling of exp_specified.  NaN stays NaN.
__device__ __forceinline__ void exp_specified2(float x0, float x1, float& e0, float& e1) {
  const float c0 = fmaxf(fminf(x0, 89.0f), -104.0f);
  const float c1 = fmaxf(fminf(x1, 89.0f), -104.0f);
  const uint64_t x = pack2(c0, c1);
  float t0, t1;
  unpack2(mul2(x, splat2(0x1.715476p+0f)), t0, t1);
  const float n0 = rintf(t0), n1 = rintf(t1);
  const uint64_t n = pack2(n0, n1);
  uint64_t r = fma2(n, splat2(-0x1.62e4p-1f), x);
  r = fma2(n, splat2(-0x1.7f7d1cp-20f), r);
  uint64_t p = splat2(0x1.a01a02p-13f);
  p = fma2(p, r, splat2(0x1.6c16c2p-10f));
  p = fma2(p, r, splat2(0x1.111112p-7f));
  p = fma2(p, r, splat2(0x1.555556p-5f));
  p = fma2(p, r, splat2(0x1.555556p-3f));
  p = fma2(p, r, splat2(0x1.0p-1f));
  p = fma2(p, r, splat2(1.0f));
  p = fma2(p, r, splat2(1.0f));
  const int i0 = static_cast<int>(n0), i1 = static_cast<int>(n1);
  const int h0 = i0 / 2, h1 = i1 / 2;
  p = mul2(p, pack2(pow2_int(h0), pow2_int(h1)));
  p = mul2(p, pack2(pow2_int(i0 - h0), pow2_int(i1 - h1)));
  unpack2(p, e0, e1);
  if (x0 != x0) e0 = x0;
  if (x1 != x1) e1 = x1;
}

// silu_mul_bf16 of a pair: h = bf16((g / (1 + exp(-g))) * u), as fp32 values.
__device__ __forceinline__ void silu_mul_bf16_2(float g0, float g1, float u0, float u1, float& h0, float& h1) {
  float e0, e1;
  exp_specified2(-g0, -g1, e0, e1);
  const float s0 = __fdiv_rn(g0, __fadd_rn(1.0f, e0));
  const float s1 = __fdiv_rn(g1, __fadd_rn(1.0f, e1));
  float p0, p1;
  unpack2(mul2(pack2(s0, s1), pack2(u0, u1)), p0, p1);
  uint32_t b2;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(b2) : "f"(p1), "f"(p0));   // p0 -> low half
  h0 = __uint_as_float(b2 << 16);
  h1 = __uint_as_float(b2 & 0xffff0000u);
}

// ---- one 16-element block ------------------------------------------------------------------

struct QBlock {
  uint32_t lo, hi;  // 16 packed e2m1 codes
  uint32_t s8;      // ue4m3 scale code
};

__device__ __forceinline__ QBlock quantize16(const float* v, float gsf) {
  float vmax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) vmax = fmaxf(vmax, fabsf(v[i]));
  const float s32 = __fmul_rn(__fdiv_rn(vmax, 6.0f), gsf);
  QBlock b;
  b.s8 = ue4m3_encode(s32);
  const float sd = e4m3_decode(b.s8);
  const float inv = sd == 0.0f ? 0.0f : __fdiv_rn(gsf, sd);
  const uint64_t inv2 = pack2(inv, inv);
  float t[16];
#pragma unroll
  for (int i = 0; i < 16; i += 2) unpack2(mul2(pack2(v[i], v[i + 1]), inv2), t[i], t[i + 1]);
  b.lo = e2m1x8(t);
  b.hi = e2m1x8(t + 8);
  return b;
}

// Byte offset of the scale of (row r, block c) in the 128x4 swizzled layout;
// groups = pad_up(k/16, 4) / 4.
__device__ __forceinline__ int64_t sf_offset(uint32_t r, uint32_t c, uint32_t groups) {
  const int64_t chunk = static_cast<int64_t>(r >> 7) * groups + (c >> 2);
  return chunk * 512 + (r & 31u) * 16 + ((r >> 5) & 3u) * 4 + (c & 3u);
}

// ---- quantize kernel -------------------------------------------------------------------------

struct QuantParams {
  const uint16_t* x;       // item 0
  int64_t x_item_stride;   // elements between items
  int64_t x_row_stride;    // elements between rows (k, or 2k for SiLU)
  uint8_t* q;
  int64_t q_item_stride;   // bytes
  uint8_t* sf;
  int64_t sf_item_stride;  // bytes
  const int32_t* mask;     // nullable
  const float* gsf;        // [items]
  int32_t m;               // rows per item
  int32_t k;               // output width (elements)
  uint32_t nb;             // k / 16
  uint32_t cpad;           // pad_up(nb, 4)
  uint32_t rows_pad;       // pad_up(m, 128)
  uint32_t blocks;         // rows_pad * cpad (per item)
};

template <bool kSilu, int kUnroll>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const QuantParams p) {
  const int item = blockIdx.y;
  int valid = p.m;
  if (p.mask) valid = min(max(__ldg(p.mask + item), 0), p.m);
  // Rows at or beyond `limit` are never touched: with a mask, rows >= mask; without one,
  // only the padding rows beyond rows_pad (which do not exist).
  const uint32_t limit = p.mask ? static_cast<uint32_t>(valid) : p.rows_pad;
  const uint32_t base = blockIdx.x * (kThreads * kUnroll);
  if (base / p.cpad >= limit) return;

  const float gsf = __ldg(p.gsf + item);
  const uint16_t* x = p.x + item * p.x_item_stride;
  uint8_t* q = p.q + item * p.q_item_stride;
  uint8_t* sf = p.sf + item * p.sf_item_stride;
  const uint32_t groups = p.cpad >> 2;

  constexpr int kVec = kSilu ? 4 : 2;
  uint4 raw[kUnroll][kVec];
  uint32_t rr[kUnroll], cc[kUnroll];
  bool live[kUnroll];

#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    const uint32_t f = base + u * kThreads + threadIdx.x;
    const uint32_t r = f / p.cpad;
    const uint32_t c = f - r * p.cpad;
    rr[u] = r;
    cc[u] = c;
    live[u] = f < p.blocks && r < static_cast<uint32_t>(valid) && c < p.nb;
    if (live[u]) {
      const uint16_t* src = x + static_cast<int64_t>(r) * p.x_row_stride + c * 16;
      raw[u][0] = load_stream(src);
      raw[u][1] = load_stream(src + 8);
      if constexpr (kSilu) {
        raw[u][2] = load_stream(src + p.k);
        raw[u][3] = load_stream(src + p.k + 8);
      }
    }
  }

#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    const uint32_t r = rr[u], c = cc[u];
    if (live[u]) {
      float v[16];
      unpack_bf16x8(raw[u][0], v);
      unpack_bf16x8(raw[u][1], v + 8);
      if constexpr (kSilu) {
        float up[16];
        unpack_bf16x8(raw[u][2], up);
        unpack_bf16x8(raw[u][3], up + 8);
#pragma unroll
        for (int i = 0; i < 16; i += 2) silu_mul_bf16_2(v[i], v[i + 1], up[i], up[i + 1], v[i], v[i + 1]);
      }
      const QBlock b = quantize16(v, gsf);
      *reinterpret_cast<uint2*>(q + static_cast<int64_t>(r) * (p.k / 2) + c * 8) = make_uint2(b.lo, b.hi);
      sf[sf_offset(r, c, groups)] = static_cast<uint8_t>(b.s8);
    } else if (base + u * kThreads + threadIdx.x < p.blocks) {
      // Padding scale entries: a column beyond the last block of a valid row, or (no mask)
      // a padding row below m.
      const bool pad_col = r < static_cast<uint32_t>(valid) && c >= p.nb;
      const bool pad_row = p.mask == nullptr && r >= static_cast<uint32_t>(p.m);
      if (pad_col || pad_row) sf[sf_offset(r, c, groups)] = 0;
    }
  }
}

// ---- global scale reductions -------------------------------------------------------------

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float absmax8(const uint4& w, float m) {
  float f[8];
  unpack_bf16x8(w, f);
#pragma unroll
  for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));  // fmaxf drops NaN (counted as 0)
  return m;
}

// Block-reduces `local`, folds it into ws[1 + item] with an atomic max on the fp32 bits
// (monotonic for non-negative values), and lets the last block of the grid finalize every
// item: amax = clamp(min(amax, FLT_MAX), 1e-12), gsf = 2688 / amax, optional alpha.  The
// last block leaves the workspace zeroed for the next call on this stream.
__device__ void reduce_and_finalize(float local, uint32_t* ws, int item, int items, uint32_t total_blocks,
                                    float* amax_out, float* gsf_out, const float* other_amax,
                                    float* alpha_out) {
  __shared__ float red[kThreads / 32];
  __shared__ bool last;
  local = warp_max(local);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = local;
  __syncthreads();
  if (threadIdx.x == 0) {
    float v = red[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) v = fmaxf(v, red[w]);
    atomicMax(ws + 1 + item, __float_as_uint(v));
    __threadfence();
    const uint32_t ticket = atomicAdd(ws, 1u);
    last = ticket == total_blocks - 1;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int i = threadIdx.x; i < items; i += blockDim.x) {
    float a = __uint_as_float(atomicExch(ws + 1 + i, 0u));
    a = fmaxf(fminf(a, FLT_MAX), 1e-12f);
    if (amax_out) amax_out[i] = a;
    gsf_out[i] = __fdiv_rn(2688.0f, a);
    if (other_amax) alpha_out[i] = __fdiv_rn(__fmul_rn(a, other_amax[i]), 7225344.0f);
  }
  __syncthreads();
  if (threadIdx.x == 0) atomicExch(ws, 0u);
}

__global__ void __launch_bounds__(kThreads) amax_dense_kernel(const uint16_t* x, int64_t numel, uint32_t* ws,
                                                              float* amax_out, float* gsf_out,
                                                              const float* other_amax, float* alpha_out) {
  float m = 0.0f;
  const int64_t nvec = numel / 8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  for (; i + 3 * stride < nvec; i += 4 * stride) {
    const uint4 a = load_stream(x + 8 * i);
    const uint4 b = load_stream(x + 8 * (i + stride));
    const uint4 c = load_stream(x + 8 * (i + 2 * stride));
    const uint4 d = load_stream(x + 8 * (i + 3 * stride));
    m = absmax8(a, m); m = absmax8(b, m); m = absmax8(c, m); m = absmax8(d, m);
  }
  for (; i < nvec; i += stride) m = absmax8(load_stream(x + 8 * i), m);
  if (blockIdx.x == 0 && threadIdx.x < numel - 8 * nvec) {
    const float t = __uint_as_float(static_cast<uint32_t>(x[8 * nvec + threadIdx.x]) << 16);
    m = fmaxf(m, fabsf(t));
  }
  reduce_and_finalize(m, ws, 0, 1, gridDim.x, amax_out, gsf_out, other_amax, alpha_out);
}

// Per-item amax over rows r < mask[item]; x is [items, m, k] or, with kSilu, [items, m, 2k]
// and the amax is over h = bf16(silu(gate) * up).
template <bool kSilu>
__global__ void __launch_bounds__(kThreads) amax_batched_kernel(const uint16_t* x, int32_t m, int32_t k,
                                                                const int32_t* mask, uint32_t* ws,
                                                                float* amax_out, float* gsf_out) {
  const int item = blockIdx.y;
  const int valid = mask ? min(max(__ldg(mask + item), 0), m) : m;
  const int64_t width = kSilu ? 2 * static_cast<int64_t>(k) : k;
  const uint16_t* xi = x + item * static_cast<int64_t>(m) * width;
  const int64_t per_row = k / 8;
  const int64_t nvec = static_cast<int64_t>(valid) * per_row;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  float mx = 0.0f;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < nvec; i += stride) {
    if constexpr (kSilu) {
      const int64_t r = i / per_row;
      const int64_t c = (i - r * per_row) * 8;
      const uint4 g = load_stream(xi + r * width + c);
      const uint4 u = load_stream(xi + r * width + k + c);
      float gf[8], uf[8];
      unpack_bf16x8(g, gf);
      unpack_bf16x8(u, uf);
#pragma unroll
      for (int j = 0; j < 8; ++j) mx = fmaxf(mx, fabsf(silu_mul_bf16(gf[j], uf[j])));
    } else {
      mx = absmax8(load_stream(xi + 8 * i), mx);
    }
  }
  reduce_and_finalize(mx, ws, item, gridDim.y, gridDim.x * gridDim.y, amax_out, gsf_out, nullptr, nullptr);
}

// ---- host helpers -------------------------------------------------------------------------

int launch_quantize(const void* x, int64_t b, int64_t m, int64_t k, bool silu, const int32_t* mask,
                    const float* gsf, uint8_t* q, uint8_t* sf, cudaStream_t stream) {
  if (b < 0 || m < 0 || k < 0 || k % 16 != 0) return NVFP4_ERR_INVALID_ARGUMENT;
  if (b == 0 || m == 0 || k == 0) return NVFP4_OK;
  if (!x || !gsf || !q || !sf) return NVFP4_ERR_INVALID_ARGUMENT;
  if (!aligned(x, 16) || !aligned(q, 8) || !aligned(gsf, 4) || (mask && !aligned(mask, 4)))
    return NVFP4_ERR_INVALID_ARGUMENT;
  if (b > 65535 || m > (1 << 30) || k > (1 << 30)) return NVFP4_ERR_INVALID_ARGUMENT;
  const int64_t nb = k / 16, cpad = (nb + 3) / 4 * 4, rows_pad = (m + 127) / 128 * 128;
  if (rows_pad * cpad >= (int64_t(1) << 31)) return NVFP4_ERR_INVALID_ARGUMENT;
  DeviceInfo info;
  int st = current_device(&info);
  if (st != NVFP4_OK) return st;

  QuantParams p;
  p.x = static_cast<const uint16_t*>(x);
  p.x_row_stride = silu ? 2 * k : k;
  p.x_item_stride = m * p.x_row_stride;
  p.q = q;
  p.q_item_stride = m * (k / 2);
  p.sf = sf;
  p.sf_item_stride = rows_pad * cpad;
  p.mask = mask;
  p.gsf = gsf;
  p.m = static_cast<int32_t>(m);
  p.k = static_cast<int32_t>(k);
  p.nb = static_cast<uint32_t>(nb);
  p.cpad = static_cast<uint32_t>(cpad);
  p.rows_pad = static_cast<uint32_t>(rows_pad);
  p.blocks = static_cast<uint32_t>(rows_pad * cpad);
  if (silu) {
    constexpr int U = 2;
    dim3 grid(static_cast<unsigned>((p.blocks + kThreads * U - 1) / (kThreads * U)), static_cast<unsigned>(b));
    quantize_kernel<true, U><<<grid, kThreads, 0, stream>>>(p);
  } else {
    constexpr int U = 4;
    dim3 grid(static_cast<unsigned>((p.blocks + kThreads * U - 1) / (kThreads * U)), static_cast<unsigned>(b));
    quantize_kernel<false, U><<<grid, kThreads, 0, stream>>>(p);
  }
  return launch_status();
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

int nvfp4_global_scale(const void* x_bf16, int64_t numel, float* amax_out, float* gsf_out,
                       const float* other_amax, float* alpha_out, nvfp4_stream_t stream) {
  if (numel < 0 || !gsf_out || (numel > 0 && !x_bf16)) return NVFP4_ERR_INVALID_ARGUMENT;
  if ((other_amax == nullptr) != (alpha_out == nullptr)) return NVFP4_ERR_INVALID_ARGUMENT;
  if ((x_bf16 && !aligned(x_bf16, 16)) || !aligned(gsf_out, 4) || (amax_out && !aligned(amax_out, 4)) ||
      (other_amax && (!aligned(other_amax, 4) || !aligned(alpha_out, 4))))
    return NVFP4_ERR_INVALID_ARGUMENT;
  DeviceInfo info;
  int st = current_device(&info);
  if (st != NVFP4_OK) return st;
  uint32_t* ws = nullptr;
  st = stream_workspace(stream, &ws);
  if (st != NVFP4_OK) return st;
  const int64_t nvec = numel / 8;
  int64_t blocks = (nvec + kThreads * 4 - 1) / (kThreads * 4);
  blocks = blocks < 1 ? 1 : (blocks > info.sm_count * 8 ? info.sm_count * 8 : blocks);
  amax_dense_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
      static_cast<const uint16_t*>(x_bf16), numel, ws, amax_out, gsf_out, other_amax, alpha_out);
  return launch_status();
}

int nvfp4_global_scale_batched(const void* x_bf16, int64_t b, int64_t m, int64_t k, const int32_t* mask,
                               int silu_mul, float* amax_out, float* gsf_out, nvfp4_stream_t stream) {
  if (b < 0 || m < 0 || k < 0 || k % 8 != 0 || b > kMaxItems || m > (1 << 30) || k > (1 << 30))
    return NVFP4_ERR_INVALID_ARGUMENT;
  if (b == 0) return NVFP4_OK;
  if (!gsf_out || (m > 0 && k > 0 && !x_bf16)) return NVFP4_ERR_INVALID_ARGUMENT;
  if ((x_bf16 && !aligned(x_bf16, 16)) || !aligned(gsf_out, 4) || (amax_out && !aligned(amax_out, 4)) ||
      (mask && !aligned(mask, 4)))
    return NVFP4_ERR_INVALID_ARGUMENT;
  DeviceInfo info;
  int st = current_device(&info);
  if (st != NVFP4_OK) return st;
  uint32_t* ws = nullptr;
  st = stream_workspace(stream, &ws);
  if (st != NVFP4_OK) return st;
  const int64_t nvec = m * (k / 8);
  int64_t gx = (nvec + kThreads * 4 - 1) / (kThreads * 4);
  int64_t cap = (info.sm_count * 8 + b - 1) / b;
  gx = gx < 1 ? 1 : (gx > cap ? cap : gx);
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(b));
  const uint16_t* x = static_cast<const uint16_t*>(x_bf16);
  if (silu_mul)
    amax_batched_kernel<true><<<grid, kThreads, 0, stream>>>(x, static_cast<int32_t>(m), static_cast<int32_t>(k),
                                                             mask, ws, amax_out, gsf_out);
  else
    amax_batched_kernel<false><<<grid, kThreads, 0, stream>>>(x, static_cast<int32_t>(m), static_cast<int32_t>(k),
                                                              mask, ws, amax_out, gsf_out);
  return launch_status();
}

int nvfp4_quantize(const void* x_bf16, int64_t m, int64_t k, const float* gsf, uint8_t* q_out, uint8_t* sf_out,
                   nvfp4_stream_t stream) {
  return launch_quantize(x_bf16, 1, m, k, false, nullptr, gsf, q_out, sf_out, stream);
}

int nvfp4_quantize_masked_batched(const void* x_bf16, int64_t b, int64_t m, int64_t k, const int32_t* mask,
                                  const float* gsf, uint8_t* q_out, uint8_t* sf_out, nvfp4_stream_t stream) {
  return launch_quantize(x_bf16, b, m, k, false, mask, gsf, q_out, sf_out, stream);
}

int nvfp4_silu_mul_quantize_batched(const void* x_bf16, int64_t b, int64_t m, int64_t k, const int32_t* mask,
                                    const float* gsf, uint8_t* q_out, uint8_t* sf_out, nvfp4_stream_t stream) {
  return launch_quantize(x_bf16, b, m, k, true, mask, gsf, q_out, sf_out, stream);
}

}  // extern "C"

// ---- non-allocating variant of the batched global scale ------------------------------------
//
// Some callers cannot let the library call cudaMalloc: code that is being captured into a
// CUDA graph (allocation is not a capturable operation), hosts whose device memory is
// owned by their own allocator or fixed at start-up (inference servers with a pre-sized
// pool, embedded deployments), and latency-critical paths that must not risk the implicit
// device synchronization cudaMalloc can cause.  nvfp4_global_scale_batched_noalloc serves
// them: its reduction scratch is the file-scope device array below instead of the lazily
// allocated per-stream workspace, so the call allocates nothing, ever.
namespace nvfp4 {
namespace {

constexpr int kNoAllocMaxItems = 1024;
// word 0: ticket counter; words 1..kNoAllocMaxItems: per-item amax bits.  Every GPU that
// loads this library holds it until the process exits.
static __device__ __align__(256) uint32_t g_noalloc_scratch[1 + kNoAllocMaxItems];

std::mutex g_noalloc_mu;
uint32_t* g_noalloc_ptr[64] = {};   // device address of g_noalloc_scratch, per device
int g_noalloc_sms[64] = {};

// Once per device, with that device current: look up the array's device address (host
// code cannot use the symbol itself) and the SM count.  Allocates nothing.
int noalloc_setup(int* dev_out, uint32_t** ptr_out, int* sms_out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return NVFP4_ERR_UNSUPPORTED_DEVICE;
    uint32_t* ptr = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    g_noalloc_sms[dev] = sms;
    g_noalloc_ptr[dev] = ptr;
  }
  *dev_out = dev;
  *ptr_out = g_noalloc_ptr[dev];
  *sms_out = g_noalloc_sms[dev];
  return NVFP4_OK;
}

}  // namespace
}  // namespace nvfp4

extern "C" int nvfp4_global_scale_batched_noalloc(const void* x_bf16, int64_t b, int64_t m, int64_t k,
                                                  const int32_t* mask, int silu_mul, float* amax_out,
                                                  float* gsf_out, nvfp4_stream_t stream) {
  using namespace nvfp4;
  if (b < 0 || m < 0 || k < 0 || k % 8 != 0 || b > kNoAllocMaxItems || m > (1 << 30) || k > (1 << 30))
    return NVFP4_ERR_INVALID_ARGUMENT;
  if (b == 0) return NVFP4_OK;
  if (!gsf_out || (m > 0 && k > 0 && !x_bf16)) return NVFP4_ERR_INVALID_ARGUMENT;
  if ((x_bf16 && !aligned(x_bf16, 16)) || !aligned(gsf_out, 4) || (amax_out && !aligned(amax_out, 4)) ||
      (mask && !aligned(mask, 4)))
    return NVFP4_ERR_INVALID_ARGUMENT;
  int dev = -1, sms = 0;
  uint32_t* scratch = nullptr;
  int st = noalloc_setup(&dev, &scratch, &sms);
  if (st != NVFP4_OK) return st;
  // The array keeps whatever the previous call left: the counter and the used amax words
  // must start at zero.
  if (cudaMemsetAsync(scratch, 0, sizeof(uint32_t) * (1 + b), stream) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  const int64_t nvec = m * (k / 8);
  int64_t gx = (nvec + kThreads * 4 - 1) / (kThreads * 4);
  const int64_t cap = (sms * 8 + b - 1) / b;
  gx = gx < 1 ? 1 : (gx > cap ? cap : gx);
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(b));
  const uint16_t* x = static_cast<const uint16_t*>(x_bf16);
  if (silu_mul)
    amax_batched_kernel<true><<<grid, kThreads, 0, stream>>>(x, static_cast<int32_t>(m), static_cast<int32_t>(k), mask,
                                                             scratch, amax_out, gsf_out);
  else
    amax_batched_kernel<false><<<grid, kThreads, 0, stream>>>(x, static_cast<int32_t>(m), static_cast<int32_t>(k), mask,
                                                              scratch, amax_out, gsf_out);
  return launch_status();
}
