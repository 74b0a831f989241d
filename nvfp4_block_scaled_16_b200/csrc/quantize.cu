// quantize.cu -- global scale (amax) reductions and the NVFP4 block quantizers.
//
// Sources (page title, section):
//   TensorRT-LLM NVFP4LinearMethod.create_weights: block size 16,
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
#include "nvfp4_math.cuh"
#include "tc_common.cuh"

namespace nvfp4 {
namespace {

constexpr int kThreads = 256;

// ---- bf16 streaming helpers ----------------------------------------------------------

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float* f) {
  f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
  f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
  f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

__device__ __forceinline__ uint4 load_stream(const void* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
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
  const uint16_t* pqs;     // smoothing: bf16 [k] pre-quantization scale (x_hat = bf16(x * pqs))
  int32_t m;               // rows per item
  int32_t k;               // output width (elements)
  uint32_t nb;             // k / 16
  uint32_t cpad;           // pad_up(nb, 4)
  uint32_t rows_pad;       // pad_up(m, 128)
  uint32_t blocks;         // rows_pad * cpad (per item)
  uint32_t cpad_magic;     // f / cpad = umulhi(f, cpad_magic) >> cpad_shift for f < 2^31
  uint32_t cpad_shift;
  const float* silu_tab;   // SiLU table in global memory (SiLU variant)
  uint32_t chunks_per_item;
  uint32_t items;
#ifdef NVFP4_DEBUG_INDEX
  int* status;             // device status word (debug-build index checks; the member alone
                           // costs the persistent quantizer a register spill in release builds)
#endif
};
#ifdef NVFP4_DEBUG_INDEX
#define QSTATUS(p) ((p).status)
#else
#define QSTATUS(p) static_cast<int*>(nullptr)
#endif

// Division by cpad (a multiple of 4) with the Granlund-Montgomery multiplier of 31-bit
// dividends: with l = ceil(log2 cpad) and m = ceil(2^(31+l) / cpad), floor(f / cpad) =
// floor(f m / 2^(31+l)) for every f < 2^31.
__device__ __forceinline__ uint32_t div_cpad(const QuantParams& p, uint32_t f) {
  return __umulhi(f, p.cpad_magic) >> p.cpad_shift;
}

void set_cpad_divisor(QuantParams& p) {
  uint32_t l = 0;
  while ((uint64_t(1) << l) < p.cpad) ++l;
  p.cpad_magic = static_cast<uint32_t>(((uint64_t(1) << (31 + l)) + p.cpad - 1) / p.cpad);
  p.cpad_shift = l - 1;
}

// inv_tab[code] = inv_scale(code, gsf) for the 128 block-scale codes, by threads [0, 128).
__device__ __forceinline__ void inv_table_build(float* inv_tab, float gsf) {
  if (threadIdx.x < 128) inv_tab[threadIdx.x] = inv_scale(threadIdx.x, gsf);
}

// One chunk: kThreads * kUnroll consecutive 16-element blocks of one item, row-major over
// rows_pad x cpad; thread t owns blocks base + u * kThreads + t.  chunk_load issues the
// chunk's loads, chunk_store computes and writes it, so a caller can overlap the loads of the
// next chunk with the arithmetic of this one.
template <bool kSilu, int kUnroll>
struct Chunk {
  static constexpr int kVec = kSilu ? 4 : 2;   // 16-byte loads per block
  uint4 raw[kUnroll][kVec];
  uint32_t r[kUnroll], c[kUnroll];
  bool live[kUnroll];     // a block of a valid row and column: quantized
  bool active;            // false: the chunk lies beyond the item's row limit, nothing is touched
  int item, valid;
  uint32_t base;
  uint32_t end;           // blocks at or beyond end belong to someone else
};

// Blocks f = base + u * kThreads + threadIdx.x with f < end (and f < p.blocks) are this
// chunk's.
template <bool kSilu, int kUnroll>
__device__ __forceinline__ void chunk_load(const QuantParams& p, int item, uint32_t base, Chunk<kSilu, kUnroll>& ch,
                                           uint32_t end = 0xffffffffu) {
  int valid = p.m;
  if (p.mask) valid = min(max(__ldg(p.mask + item), 0), p.m);
  // Rows at or beyond `limit` are never touched: with a mask, rows >= mask; without one,
  // only the padding rows beyond rows_pad (which do not exist).
  const uint32_t limit = p.mask ? static_cast<uint32_t>(valid) : p.rows_pad;
  ch.item = item;
  ch.valid = valid;
  ch.base = base;
  ch.end = end;
  ch.active = div_cpad(p, base) < limit;
  if (!ch.active) return;
  const uint16_t* x = p.x + item * p.x_item_stride;
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    const uint32_t f = base + u * kThreads + threadIdx.x;
    const uint32_t r = div_cpad(p, f);
    const uint32_t c = f - r * p.cpad;
    ch.r[u] = r;
    ch.c[u] = c;
    ch.live[u] = f < p.blocks && f < end && r < static_cast<uint32_t>(valid) && c < p.nb;
    if (kDebugIndex && ch.live[u])    // the block's last element (of the up half with SiLU) lies in the item
      ch.live[u] = index_ok(static_cast<uint64_t>(r) * p.x_row_stride + c * 16 + (kSilu ? p.k : 0) + 15,
                            static_cast<uint64_t>(p.x_item_stride), QSTATUS(p));
    if (ch.live[u]) {
      const uint16_t* src = x + static_cast<int64_t>(r) * p.x_row_stride + c * 16;
      ch.raw[u][0] = load_stream(src);
      ch.raw[u][1] = load_stream(src + 8);
      if constexpr (kSilu) {
        ch.raw[u][2] = load_stream(src + p.k);
        ch.raw[u][3] = load_stream(src + p.k + 8);
      }
    }
  }
}

// With kSilu, `tab` is the SiLU table in shared memory.
// inv_tab: the inverse block scales of the chunk's item (inv_table_build with its gsf).
template <bool kSilu, bool kSmooth, int kUnroll>
__device__ __forceinline__ void chunk_store(const QuantParams& p, const Chunk<kSilu, kUnroll>& ch, const float* tab,
                                            float gsf, const float* inv_tab) {
  if (!ch.active) return;
  uint8_t* q = p.q + ch.item * p.q_item_stride;
  uint8_t* sf = p.sf + ch.item * p.sf_item_stride;
  const uint32_t groups = p.cpad >> 2;
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    const uint32_t r = ch.r[u], c = ch.c[u];
    if (ch.live[u]) {
      float v[16];
      if constexpr (kSilu) {
        float up[16];
        unpack_bf16x8(ch.raw[u][2], up);
        unpack_bf16x8(ch.raw[u][3], up + 8);
        const uint32_t gw[8] = {ch.raw[u][0].x, ch.raw[u][0].y, ch.raw[u][0].z, ch.raw[u][0].w,
                                ch.raw[u][1].x, ch.raw[u][1].y, ch.raw[u][1].z, ch.raw[u][1].w};
#pragma unroll
        for (int i = 0; i < 8; ++i) silu_mul_bf16_tab2(tab, gw[i], up[2 * i], up[2 * i + 1], v[2 * i], v[2 * i + 1]);
      } else {
        unpack_bf16x8(ch.raw[u][0], v);
        unpack_bf16x8(ch.raw[u][1], v + 8);
      }
      if constexpr (kSmooth) {
        // x_hat = bf16(x * pre_quant_scale) for the block's 16 columns (the scale vector is
        // the same for every row: these loads hit in L1 / L2)
        float sc[16] = {};
        if (index_ok(c * 16 + 15, static_cast<uint64_t>(p.k), QSTATUS(p))) {
          unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(p.pqs + c * 16)), sc);
          unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(p.pqs + c * 16 + 8)), sc + 8);
        }
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          float a, b;
          unpack2(mul2(pack2(v[i], v[i + 1]), pack2(sc[i], sc[i + 1])), a, b);
          uint32_t w;
          asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(b), "f"(a));   // a -> low half
          v[i] = bf16_lo(w);
          v[i + 1] = bf16_hi(w);
        }
      }
      const QBlock b = quantize16(v, gsf, inv_tab);
      const int64_t qo = static_cast<int64_t>(r) * (p.k / 2) + c * 8, so = sf_offset(r, c, groups);
      if (index_ok(qo + 7, static_cast<uint64_t>(p.q_item_stride), QSTATUS(p)))
        *reinterpret_cast<uint2*>(q + qo) = make_uint2(b.lo, b.hi);
      if (index_ok(so, static_cast<uint64_t>(p.sf_item_stride), QSTATUS(p))) sf[so] = static_cast<uint8_t>(b.s8);
    } else if (ch.base + u * kThreads + threadIdx.x < min(p.blocks, ch.end)) {
      // Padding scale entries: a column beyond the last block of a valid row, or (no mask)
      // a padding row below m.
      const bool pad_col = r < static_cast<uint32_t>(ch.valid) && c >= p.nb;
      const bool pad_row = p.mask == nullptr && r >= static_cast<uint32_t>(p.m);
      if ((pad_col || pad_row) && index_ok(sf_offset(r, c, groups), static_cast<uint64_t>(p.sf_item_stride), QSTATUS(p)))
        sf[sf_offset(r, c, groups)] = 0;
    }
  }
}

// One chunk per CTA: grid (chunks per item, items).
template <bool kSmooth, int kUnroll>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const QuantParams p) {
  __shared__ float inv_tab[128];
  pdl_launch_dependents();
  pdl_wait();
  Chunk<false, kUnroll> ch;
  chunk_load(p, blockIdx.y, blockIdx.x * (kThreads * kUnroll), ch);
  const float gsf = __ldg(p.gsf + blockIdx.y);
  inv_table_build(inv_tab, gsf);
  __syncthreads();
  chunk_store<false, kSmooth>(p, ch, nullptr, gsf, inv_tab);
}

// Persistent CTAs that walk the chunks of all items (item-major) with a grid stride, so the
// live chunks of every item are spread over all CTAs whatever the masks are, and chunks
// beyond an item's mask cost a few instructions instead of a CTA launch.  Used for SiLU * up
// (which loads the SiLU table into shared memory once per CTA) and for the masked
// quantizer.  (Issuing the next chunk's loads before the current chunk's arithmetic, with
// one or two blocks per thread and 2-6 CTAs per SM, measured 2-15% slower for SiLU * up than
// this plain loop with two blocks per thread and four CTAs per SM.)
template <bool kSilu>
constexpr int kPersistUnroll = kSilu ? 2 : 4;
constexpr int kPersistCtasPerSm = 4;
// The SiLU table fits the default 48 KB of dynamic shared memory (no opt-in attribute needed).
static_assert(kSiluTableBytes <= 48 * 1024, "SiLU table exceeds the default dynamic shared memory");
template <bool kSilu>
__global__ void __launch_bounds__(kThreads, kPersistCtasPerSm) persistent_quantize_kernel(const QuantParams p) {
  extern __shared__ float4 silu_smem[];
  __shared__ float inv_tab[128];
  float* tab = reinterpret_cast<float*>(silu_smem);
  pdl_launch_dependents();
  pdl_wait();
  if constexpr (kSilu) silu_table_load(tab, p.silu_tab, threadIdx.x, kThreads);
  constexpr int kUnroll = kPersistUnroll<kSilu>;
  const uint64_t total = static_cast<uint64_t>(p.chunks_per_item) * p.items;
  Chunk<kSilu, kUnroll> ch;
  uint32_t table_item = 0xffffffffu;           // the item whose inverse scales inv_tab holds
  float gsf = 0.0f;
  for (uint64_t chunk = blockIdx.x; chunk < total; chunk += gridDim.x) {
    const uint32_t item = static_cast<uint32_t>(chunk / p.chunks_per_item);
    const uint32_t local = static_cast<uint32_t>(chunk - static_cast<uint64_t>(item) * p.chunks_per_item);
    chunk_load(p, static_cast<int>(item), local * (kThreads * kUnroll), ch);
    if (item != table_item) {                   // uniform over the CTA
      __syncthreads();                          // the previous item's table is no longer read
      gsf = __ldg(p.gsf + item);
      inv_table_build(inv_tab, gsf);
      table_item = item;
      __syncthreads();                          // (also orders the SiLU table's first load)
    }
    chunk_store<kSilu, false>(p, ch, tab, gsf, inv_tab);
  }
}

// ---- SiLU-and-mul without quantization ---------------------------------------------------

// h[r, c] = bf16(silu(x[r, c]) * x[r, k + c]) for rows of width 2k; 8 outputs per thread.
__global__ void __launch_bounds__(kThreads) silu_and_mul_kernel(const uint16_t* x, int64_t rows, int32_t k,
                                                                uint16_t* h, const float* silu_tab, int* status) {
  extern __shared__ float4 silu_smem[];
  float* tab = reinterpret_cast<float*>(silu_smem);
  pdl_launch_dependents();
  pdl_wait();
  silu_table_load(tab, silu_tab, threadIdx.x, kThreads);
  __syncthreads();
  const int64_t per_row = k / 8;
  const int64_t total = rows * per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * kThreads) {
    const int64_t r = i / per_row;
    const int64_t c = (i - r * per_row) * 8;
    if (!index_ok(r * 2 * k + k + c + 7, static_cast<uint64_t>(rows) * 2 * k, status) ||
        !index_ok(r * k + c + 7, static_cast<uint64_t>(rows) * k, status))
      continue;
    float u[8], o[8];
    const uint4 g = load_stream(x + r * 2 * k + c);
    unpack_bf16x8(load_stream(x + r * 2 * k + k + c), u);
    const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) silu_mul_bf16_tab2(tab, gw[e], u[2 * e], u[2 * e + 1], o[2 * e], o[2 * e + 1]);
    uint4 w;
    w.x = (__float_as_uint(o[0]) >> 16) | (__float_as_uint(o[1]) & 0xffff0000u);
    w.y = (__float_as_uint(o[2]) >> 16) | (__float_as_uint(o[3]) & 0xffff0000u);
    w.z = (__float_as_uint(o[4]) >> 16) | (__float_as_uint(o[5]) & 0xffff0000u);
    w.w = (__float_as_uint(o[6]) >> 16) | (__float_as_uint(o[7]) & 0xffff0000u);
    *reinterpret_cast<uint4*>(h + r * k + c) = w;
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
                                                              const float* other_amax, float* alpha_out, int* status) {
  pdl_launch_dependents();
  pdl_wait();
  float m = 0.0f;
  const int64_t nvec = numel / 8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  for (; i + 3 * stride < nvec; i += 4 * stride) {
    if (!index_ok(8 * (i + 3 * stride) + 7, static_cast<uint64_t>(numel), status)) break;
    const uint4 a = load_stream(x + 8 * i);
    const uint4 b = load_stream(x + 8 * (i + stride));
    const uint4 c = load_stream(x + 8 * (i + 2 * stride));
    const uint4 d = load_stream(x + 8 * (i + 3 * stride));
    m = absmax8(a, m); m = absmax8(b, m); m = absmax8(c, m); m = absmax8(d, m);
  }
  for (; i < nvec; i += stride)
    if (index_ok(8 * i + 7, static_cast<uint64_t>(numel), status)) m = absmax8(load_stream(x + 8 * i), m);
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
                                                                float* amax_out, float* gsf_out, int* status) {
  pdl_launch_dependents();
  pdl_wait();
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
      if (!index_ok(r * width + k + c + 7, static_cast<uint64_t>(m) * width, status)) continue;
      const uint4 g = load_stream(xi + r * width + c);
      const uint4 u = load_stream(xi + r * width + k + c);
      float gf[8], uf[8];
      unpack_bf16x8(g, gf);
      unpack_bf16x8(u, uf);
#pragma unroll
      for (int j = 0; j < 8; ++j) mx = fmaxf(mx, fabsf(silu_mul_bf16(gf[j], uf[j])));
    } else if (index_ok(8 * i + 7, static_cast<uint64_t>(m) * width, status)) {
      mx = absmax8(load_stream(xi + 8 * i), mx);
    }
  }
  reduce_and_finalize(mx, ws, item, gridDim.y, gridDim.x * gridDim.y, amax_out, gsf_out, nullptr, nullptr);
}

// ---- global scale and quantize in one launch -----------------------------------------------
//
// The global scale needs the amax of the whole tensor before any block can be quantized.
// One persistent grid, one CTA per SM, every CTA resident at once (a cooperative launch),
// does both, for k % 64 == 0 (k / 16 blocks per row fill whole 4-block scale groups).  x is
// viewed as rows of 128 bytes, one 4-block scale group each (group g holds blocks 4g..4g+3,
// which are the 64 elements of x at 64 g, and its codes are the 32 bytes of q at 32 g), and
// CTA j takes the contiguous groups [j R / G, (j + 1) R / G).  A producer warp streams the
// CTA's groups through a ring of three 60 KB shared-memory slots with tiled TMA loads (480
// groups per slot, 128-byte swizzle, so a compute thread reads its 16-byte chunks without
// bank conflicts); 30 compute warps take half a group (two blocks) per thread and slot.
//   phase 1: the slots pass through the ring once (x read from HBM once); the compute warps
//     take max |x| of each (packed bf16 pairs, NaN dropped like fmaxf) and release it,
//     except the last three, which stay resident; the CTA folds its max into the workspace
//     with an atomic max and arrives on a grid barrier (bounded spin on an acquire load).
//     Slots that phase 2 reads again are loaded with the L2 evict-last policy.
//   phase 2: every CTA computes gsf from the same maximum, quantizes the resident slots,
//     while the producer reloads the earlier slots from L2 into the freed ones, last first.
//     Each pair of threads writes its group's 32 code bytes and its four scale bytes (one
//     word of the 128x4 layout, assembled by a shuffle), and the CTA zeroes its share of the
//     padding rows' scale words.
// Workspace words: 0 = barrier arrivals, 1 = CTAs done reading the maximum, 2 = amax bits,
// 3 = set by a CTA whose own bounded ring wait gave up (then no CTA writes anything); the
// last CTA to read the maximum resets all four for the next call on the stream.
constexpr int kGsqComputeWarps = 30;
constexpr int kGsqCompute = 32 * kGsqComputeWarps;              // compute threads: half a group each per slot
constexpr int kGsqThreads = kGsqCompute + 32;                   // and the producer warp (at most 1024)
constexpr uint32_t kGsqSlotGroups = kGsqCompute / 2;            // 480 groups = 60 KB of x per slot
constexpr uint32_t kGsqSlotBytes = kGsqSlotGroups * 128;
constexpr uint32_t kGsqSlots = 3;
constexpr uint32_t kGsqSmemBytes = kGsqSlots * kGsqSlotBytes + 1024;   // + alignment to 1024 bytes
constexpr uint32_t kGsqBox = kGsqSlotGroups / 2;                // groups per TMA box (two per slot)
static_assert(kGsqThreads <= 1024 && kGsqBox <= 256, "block size or TMA box too large");
static_assert((kGsqBox * 128) % 1024 == 0, "every TMA box lands 1024-byte aligned (128-byte swizzle)");

struct GsqParams {
  uint8_t* q;
  uint8_t* sf;
  uint32_t groups_total;   // m * nb / 4
  uint32_t nb4;            // groups per row of x: nb / 4
  uint32_t nb4_magic, nb4_shift;   // g / nb4 = (g * magic) >> shift for g < 2^31
  uint32_t m, rows_pad;
};

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint2 ld_relaxed_gpu_v2(const uint32_t* p) {
  uint2 v;
  asm volatile("ld.relaxed.gpu.global.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint64_t l2_policy(bool keep) {
  uint64_t pol;
  if (keep)
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  else
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Tiled TMA load of kGsqBox groups (rows of 128 bytes) starting at group `row` into this
// CTA's shared memory, completing on `bar`, with an L2 eviction policy.
__device__ __forceinline__ void gsq_tma_load(void* dst, const CUtensorMap* map, uint64_t* bar, int row, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%3, %4}], "
      "[%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(0), "r"(row), "l"(pol)
      : "memory");
}

__device__ __forceinline__ __nv_bfloat162 as_bf162(uint32_t w) {
  return *reinterpret_cast<const __nv_bfloat162*>(&w);
}

// Running max |x| over the 8 bf16 values of a 16-byte chunk, as packed pairs.
__device__ __forceinline__ __nv_bfloat162 absmax_chunk(const uint4& c, __nv_bfloat162 m) {
  m = __hmax2(m, __habs2(as_bf162(c.x)));
  m = __hmax2(m, __habs2(as_bf162(c.y)));
  m = __hmax2(m, __habs2(as_bf162(c.z)));
  m = __hmax2(m, __habs2(as_bf162(c.w)));
  return m;
}
__device__ __forceinline__ float bf162_max(__nv_bfloat162 m) {
  return fmaxf(__bfloat162float(m.x), __bfloat162float(m.y));
}

// One 16-element block (two chunks) with the block maximum taken on packed bf16 pairs: the
// same value as block_scale_code's fp32 maximum (every |x| is a bf16 value), so the result
// equals quantize16 bit for bit.
__device__ __forceinline__ QBlock gsq_block(const uint4& lo4, const uint4& hi4, float gsf, const float* inv_tab) {
  const __nv_bfloat162 zero = __floats2bfloat162_rn(0.0f, 0.0f);
  const float vmax = bf162_max(absmax_chunk(hi4, absmax_chunk(lo4, zero)));
  const uint32_t s8 = ue4m3_encode(__fmul_rn(div6_bf16(vmax), gsf));
  float v[16];
  unpack_bf16x8(lo4, v);
  unpack_bf16x8(hi4, v + 8);
  return quantize16_codes(v, s8, inv_tab[s8]);
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// Thread t's half of group t / 2 in a 128-byte-swizzled slot at shared address `slot`:
// chunks 4 h .. 4 h + 3 (h = t % 2), chunk j of row g being at 16-byte position j ^ (g % 8).
// The eight threads of a quarter warp read eight different 16-byte bank groups.
__device__ __forceinline__ void gsq_read_half(uint32_t slot, uint32_t t, uint4 (&c)[4]) {
  const uint32_t g = t >> 1, h = t & 1;
  const uint32_t row = slot + g * 128;
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i] = lds128(row + (((4 * h + i) ^ (g & 7)) << 4));
}

__global__ void __launch_bounds__(kGsqThreads, 1)
    global_scale_quantize_kernel(const __grid_constant__ CUtensorMap xmap, const GsqParams p, uint32_t* ws,
                                 float* amax_out, float* gsf_out, const float* other_amax, float* alpha_out,
                                 int* status, uint32_t withheld) {
  extern __shared__ uint8_t gsq_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gsq_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[kGsqSlots], empty[kGsqSlots];
  __shared__ int32_t abort_flag;
  __shared__ float red[kGsqComputeWarps];
  __shared__ float s_amax;
  __shared__ float inv_tab[128];
  pdl_wait();
  const int warp = threadIdx.x >> 5;
  const uint32_t t = threadIdx.x;
  const bool producer = warp == kGsqComputeWarps;
  const uint32_t grid = gridDim.x;
  const uint32_t expected = grid + withheld;   // self-test: arrivals that never come
  const uint32_t g_lo = static_cast<uint32_t>(static_cast<uint64_t>(p.groups_total) * blockIdx.x / grid);
  const uint32_t g_hi = static_cast<uint32_t>(static_cast<uint64_t>(p.groups_total) * (blockIdx.x + 1) / grid);
  const uint32_t slots_total = (g_hi - g_lo + kGsqSlotGroups - 1) / kGsqSlotGroups;   // pieces of the range
  const uint32_t resident = min(slots_total, kGsqSlots);     // pieces that stay in the ring after phase 1
  if (threadIdx.x == 0) {
    for (uint32_t i = 0; i < kGsqSlots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kGsqComputeWarps);
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  uint32_t fpar = 0, epar = 0;      // per-slot phase parity bits of full / empty waits

  // ---------------------------------------------------------------- phase 1
  float mx = 0.0f;
  if (producer) {
    if (elect_one()) {
      prefetch_map(&xmap);
      for (uint32_t piece = 0; piece < slots_total; ++piece) {
        const uint32_t s = piece % kGsqSlots;
        if (piece >= kGsqSlots) {
          if (!mbar_wait_fast(&empty[s], (epar >> s) & 1u, &abort_flag, status)) break;
          epar ^= 1u << s;
        }
        const uint64_t pol = l2_policy(piece + resident < slots_total);   // read again in phase 2
        uint8_t* dst = ring + s * kGsqSlotBytes;
        const int row = static_cast<int>(g_lo + piece * kGsqSlotGroups);
        mbar_arrive_expect_tx(&full[s], kGsqSlotBytes);
        gsq_tma_load(dst, &xmap, &full[s], row, pol);
        gsq_tma_load(dst + kGsqBox * 128, &xmap, &full[s], row + static_cast<int>(kGsqBox), pol);
      }
    }
    __syncwarp();
  } else {
    const __nv_bfloat162 zero = __floats2bfloat162_rn(0.0f, 0.0f);
    __nv_bfloat162 m2 = zero;
    for (uint32_t piece = 0; piece < slots_total; ++piece) {
      const uint32_t s = piece % kGsqSlots;
      // warp-uniform outcome, so that the warp's lanes leave the loop together
      if (!__all_sync(0xffffffffu, mbar_wait_fast(&full[s], (fpar >> s) & 1u, &abort_flag, status))) break;
      fpar ^= 1u << s;
      if (g_lo + piece * kGsqSlotGroups + (t >> 1) < g_hi) {
        uint4 c[4];
        gsq_read_half(smem_u32(ring) + s * kGsqSlotBytes, t, c);
#pragma unroll
        for (int j = 0; j < 4; ++j) m2 = absmax_chunk(c[j], m2);
      }
      __syncwarp();
      if (piece + resident < slots_total && (t & 31) == 0) mbar_arrive(&empty[s]);
    }
    mx = bf162_max(m2);
  }
  mx = warp_max(mx);
  if ((threadIdx.x & 31) == 0 && !producer) red[warp] = mx;
  __syncthreads();
  bool passed = false;                                 // thread 0: passed the barrier (takes a ticket)
  if (threadIdx.x == 0) {
    float v = red[0];
#pragma unroll
    for (int w = 1; w < kGsqComputeWarps; ++w) v = fmaxf(v, red[w]);
    if (abort_flag) atomicExch(ws + 3, 1u);            // a ring wait gave up: nobody writes
    atomicMax(ws + 2, __float_as_uint(v));
    // arrive, ordered after the atomic max (and ws[3]) by release semantics
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ws) : "memory");
    // grid barrier, bounded: every CTA is resident, so only a fault elsewhere can stall it
    const uint64_t t0 = global_ns();
    bool ok = true;
    for (uint32_t i = 1; ld_acquire_gpu(ws) < expected; ++i) {
      if ((i & 63u) == 0 && global_ns() - t0 > kWaitLimitNs) {
        ok = false;
        atomicExch(status, NVFP4_ERR_DEVICE_TIMEOUT);
        break;
      }
    }
    float a = -1.0f;                                   // -1: give up, write nothing
    if (ok) {
      // the maximum and the abort word in one load, ordered after the acquire load that saw
      // every arrival (each CTA wrote both before its release)
      const uint2 ma = ld_relaxed_gpu_v2(ws + 2);
      if (ma.y == 0u) a = fmaxf(fminf(__uint_as_float(ma.x), FLT_MAX), 1e-12f);
    }
    s_amax = a;
    passed = ok;
  }
  __syncthreads();
  if (passed && atomicAdd(ws + 1, 1u) == grid - 1) {   // every CTA has read the maximum
    atomicExch(ws + 2, 0u);
    atomicExch(ws + 3, 0u);
    atomicExch(ws + 1, 0u);
    atomicExch(ws, 0u);
  }
  const float amax = s_amax;
  if (amax < 0.0f) {
    if (abort_flag) {
      // a ring wait gave up: give outstanding TMA loads a bounded time to land before the
      // CTA's shared memory is released
      const uint64_t t0 = global_ns();
      while (global_ns() - t0 < 2000000ull) {
      }
    }
    return;
  }
  pdl_launch_dependents();            // every CTA of this grid is past the barrier
  const float gsf = __fdiv_rn(2688.0f, amax);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (amax_out) *amax_out = amax;
    *gsf_out = gsf;
    if (other_amax) *alpha_out = __fdiv_rn(__fmul_rn(amax, *other_amax), 7225344.0f);
  }
  if (threadIdx.x < 128) inv_tab[threadIdx.x] = inv_scale(threadIdx.x, gsf);
  __syncthreads();

  // ---------------------------------------------------------------- phase 2: last piece first
  if (producer) {
    if (elect_one()) {
      const uint64_t pol = l2_policy(false);
      for (uint32_t i = resident; i < slots_total; ++i) {
        const uint32_t piece = slots_total - 1 - i;
        const uint32_t s = piece % kGsqSlots;
        if (!mbar_wait_fast(&empty[s], (epar >> s) & 1u, &abort_flag, status)) break;
        epar ^= 1u << s;
        uint8_t* dst = ring + s * kGsqSlotBytes;
        const int row = static_cast<int>(g_lo + piece * kGsqSlotGroups);
        mbar_arrive_expect_tx(&full[s], kGsqSlotBytes);
        gsq_tma_load(dst, &xmap, &full[s], row, pol);
        gsq_tma_load(dst + kGsqBox * 128, &xmap, &full[s], row + static_cast<int>(kGsqBox), pol);
      }
    }
    __syncwarp();
  } else {
    const uint32_t groups4 = p.nb4;           // 4-block groups per row of the scale layout
    for (uint32_t i = 0; i < slots_total; ++i) {
      const uint32_t piece = slots_total - 1 - i;
      const uint32_t s = piece % kGsqSlots;
      if (i >= resident) {                     // reloaded from L2
        if (!__all_sync(0xffffffffu, mbar_wait_fast(&full[s], (fpar >> s) & 1u, &abort_flag, status))) break;
        fpar ^= 1u << s;
      }
      const uint32_t g = g_lo + piece * kGsqSlotGroups + (t >> 1);
      uint32_t scales = 0;                     // this thread's two scale bytes
      if (g < g_hi) {                          // the same for both threads of a group
        uint4 c[4];
        gsq_read_half(smem_u32(ring) + s * kGsqSlotBytes, t, c);
        const QBlock b0 = gsq_block(c[0], c[1], gsf, inv_tab);
        const QBlock b1 = gsq_block(c[2], c[3], gsf, inv_tab);
        if (index_ok(static_cast<uint64_t>(g) * 32 + (t & 1) * 16 + 15, static_cast<uint64_t>(p.groups_total) * 32,
                     status))
          *reinterpret_cast<uint4*>(p.q + static_cast<int64_t>(g) * 32 + (t & 1) * 16) =
              make_uint4(b0.lo, b0.hi, b1.lo, b1.hi);
        scales = b0.s8 | (b1.s8 << 8);
      }
      const uint32_t other = __shfl_xor_sync(0xffffffffu, scales, 1);
      if (g < g_hi && (t & 1) == 0) {
        const uint32_t r = static_cast<uint32_t>((static_cast<uint64_t>(g) * p.nb4_magic) >> p.nb4_shift);
        const uint32_t c0 = (g - r * groups4) * 4;
        if (index_ok(sf_offset(r, c0, groups4) + 3, static_cast<uint64_t>(p.rows_pad) * groups4 * 4, status))
          *reinterpret_cast<uint32_t*>(p.sf + sf_offset(r, c0, groups4)) = scales | (other << 16);
      }
      __syncwarp();
      if ((t & 31) == 0) mbar_arrive(&empty[s]);
    }
    // padding rows [m, rows_pad): their scale words are zero
    const uint32_t pad_words = (p.rows_pad - p.m) * groups4;
    for (uint32_t i = blockIdx.x * kGsqCompute + t; i < pad_words; i += grid * kGsqCompute) {
      const uint32_t r = p.m + i / groups4;
      if (index_ok(sf_offset(r, (i % groups4) * 4, groups4) + 3, static_cast<uint64_t>(p.rows_pad) * groups4 * 4, status))
        *reinterpret_cast<uint32_t*>(p.sf + sf_offset(r, (i % groups4) * 4, groups4)) = 0u;
    }
  }
}

// ---- host helpers -------------------------------------------------------------------------

// nvfp4_global_scale: one launch of amax_dense_kernel.
int launch_amax_dense(const void* x_bf16, int64_t numel, float* amax_out, float* gsf_out, const float* other_amax,
                      float* alpha_out, cudaStream_t stream) {
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
  return launch_kernel(amax_dense_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), 0, stream,
                       static_cast<const uint16_t*>(x_bf16), numel, ws, amax_out, gsf_out, other_amax, alpha_out,
                       info.status);
}

int launch_quantize(const void* x, int64_t b, int64_t m, int64_t k, bool silu, const int32_t* mask,
                    const float* gsf, uint8_t* q, uint8_t* sf, cudaStream_t stream, const void* pqs = nullptr) {
  if (b < 0 || m < 0 || k < 0 || k % 16 != 0) return NVFP4_ERR_INVALID_ARGUMENT;
  if (b == 0 || m == 0 || k == 0) return NVFP4_OK;
  if (!x || !gsf || !q || !sf) return NVFP4_ERR_INVALID_ARGUMENT;
  if (!aligned(x, 16) || !aligned(q, 8) || !aligned(gsf, 4) || (mask && !aligned(mask, 4)) ||
      (pqs && !aligned(pqs, 16)))
    return NVFP4_ERR_INVALID_ARGUMENT;
  if (b > 65535 || m > (1 << 30) || k > (1 << 30)) return NVFP4_ERR_INVALID_ARGUMENT;
  const int64_t nb = k / 16, cpad = (nb + 3) / 4 * 4, rows_pad = (m + 127) / 128 * 128;
  if (rows_pad * cpad >= (int64_t(1) << 31) - 4096) return NVFP4_ERR_INVALID_ARGUMENT;   // f < 2^31
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
  p.pqs = static_cast<const uint16_t*>(pqs);
  p.m = static_cast<int32_t>(m);
  p.k = static_cast<int32_t>(k);
  p.nb = static_cast<uint32_t>(nb);
  p.cpad = static_cast<uint32_t>(cpad);
  p.rows_pad = static_cast<uint32_t>(rows_pad);
  p.blocks = static_cast<uint32_t>(rows_pad * cpad);
  set_cpad_divisor(p);
  p.silu_tab = info.silu_table;
  p.items = static_cast<uint32_t>(b);
#ifdef NVFP4_DEBUG_INDEX
  p.status = info.status;
#endif
  if (silu || mask) {
    // persistent grid over the chunks of all items
    const int U = silu ? kPersistUnroll<true> : kPersistUnroll<false>;
    p.chunks_per_item = (p.blocks + kThreads * U - 1) / (kThreads * U);
    const int64_t chunks = static_cast<int64_t>(p.chunks_per_item) * b;
    const int64_t cap = static_cast<int64_t>(info.sm_count) * kPersistCtasPerSm;
    const dim3 grid(static_cast<unsigned>(chunks < cap ? chunks : cap));
    if (silu) return launch_kernel(persistent_quantize_kernel<true>, grid, dim3(kThreads), kSiluTableBytes, stream, p);
    if (!pqs) return launch_kernel(persistent_quantize_kernel<false>, grid, dim3(kThreads), 0, stream, p);
  }
  constexpr int U = 4;
  p.chunks_per_item = (p.blocks + kThreads * U - 1) / (kThreads * U);
  dim3 grid(p.chunks_per_item, static_cast<unsigned>(b));
  if (pqs) return launch_kernel(quantize_kernel<true, U>, grid, dim3(kThreads), 0, stream, p);
  return launch_kernel(quantize_kernel<false, U>, grid, dim3(kThreads), 0, stream, p);
}

// nvfp4_global_scale_quantize; `withheld` > 0 (self-test only) makes the grid barrier wait
// for arrivals that never come.  k % 64 == 0 and m > 0 take the one-launch kernel; other
// shapes take the amax kernel and then the dense quantizer (the same results).
int launch_global_scale_quantize(const void* x_bf16, int64_t m, int64_t k, float* amax_out, float* gsf_out,
                                 const float* other_amax, float* alpha_out, uint8_t* q_out, uint8_t* sf_out,
                                 cudaStream_t stream, uint32_t withheld) {
  if (m < 0 || k <= 0 || k % 16 != 0 || m > (1 << 30) || k > (1 << 30)) return NVFP4_ERR_INVALID_ARGUMENT;
  if ((other_amax == nullptr) != (alpha_out == nullptr)) return NVFP4_ERR_INVALID_ARGUMENT;
  if (!gsf_out || (m > 0 && (!x_bf16 || !q_out || !sf_out))) return NVFP4_ERR_INVALID_ARGUMENT;
  if ((x_bf16 && !aligned(x_bf16, 16)) || !aligned(q_out, 8) || !aligned(gsf_out, 4) ||
      (amax_out && !aligned(amax_out, 4)) || (other_amax && (!aligned(other_amax, 4) || !aligned(alpha_out, 4))))
    return NVFP4_ERR_INVALID_ARGUMENT;
  const int64_t nb = k / 16, cpad = (nb + 3) / 4 * 4, rows_pad = (m + 127) / 128 * 128;
  if (rows_pad * cpad >= (int64_t(1) << 31) - 4096) return NVFP4_ERR_INVALID_ARGUMENT;   // indices < 2^31
  if (k % 64 != 0 || m == 0) {
    if (withheld) return NVFP4_ERR_INVALID_ARGUMENT;   // the self-test needs the one-launch kernel
    int st = launch_amax_dense(x_bf16, m * k, amax_out, gsf_out, other_amax, alpha_out, stream);
    if (st != NVFP4_OK) return st;
    return launch_quantize(x_bf16, 1, m, k, false, nullptr, gsf_out, q_out, sf_out, stream);
  }
  if (!aligned(q_out, 16) || !aligned(sf_out, 4)) return NVFP4_ERR_INVALID_ARGUMENT;
  DeviceInfo info;
  int st = current_device(&info);
  if (st != NVFP4_OK) return st;
  uint32_t* ws = nullptr;
  st = stream_workspace(stream, &ws);
  if (st != NVFP4_OK) return st;
  const int smem = static_cast<int>(kGsqSmemBytes);
  int per_sm = 0;          // co-resident CTAs per SM (the grid must be resident at once), per device
  st = kernel_setup(reinterpret_cast<const void*>(global_scale_quantize_kernel), info.device, [&](int* out) {
    int n = 0;
    if (cudaFuncSetAttribute(global_scale_quantize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, global_scale_quantize_kernel, kGsqThreads, smem) !=
            cudaSuccess ||
        n <= 0) {
      cudaGetLastError();
      return static_cast<int>(NVFP4_ERR_CUDA);
    }
    *out = n;
    return static_cast<int>(NVFP4_OK);
  }, &per_sm);
  if (st != NVFP4_OK) return st;
  GsqParams p = {};
  p.q = q_out;
  p.sf = sf_out;
  p.m = static_cast<uint32_t>(m);
  p.rows_pad = static_cast<uint32_t>(rows_pad);
  p.nb4 = static_cast<uint32_t>(nb / 4);
  p.groups_total = static_cast<uint32_t>(m * (nb / 4));
  // Granlund-Montgomery: with l = ceil(log2 nb4) and magic = ceil(2^(31 + l) / nb4),
  // floor(g / nb4) = floor(g * magic / 2^(31 + l)) for every g < 2^31 (magic < 2^32).
  uint32_t l = 0;
  while ((uint64_t(1) << l) < p.nb4) ++l;
  p.nb4_magic = static_cast<uint32_t>(((uint64_t(1) << (31 + l)) + p.nb4 - 1) / p.nb4);
  p.nb4_shift = 31 + l;
  // x as rows of 128 bytes (one 4-block group each), boxes of 256 rows, 128-byte swizzle;
  // rows beyond the tensor read as zeros
  CUtensorMap xmap;
  EncodeTiledFn encode = encode_tiled_fn();
  if (!encode) return NVFP4_ERR_CUDA;
  const cuuint64_t dims[2] = {128, p.groups_total};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {128, kGsqBox};
  const cuuint32_t elem_strides[2] = {1, 1};
  if (encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(x_bf16), dims, strides, box, elem_strides,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return NVFP4_ERR_INVALID_ARGUMENT;
  const int64_t want = (static_cast<int64_t>(p.groups_total) + kGsqSlotGroups - 1) / kGsqSlotGroups;
  const int64_t cap = static_cast<int64_t>(info.sm_count) * per_sm;
  const unsigned grid = static_cast<unsigned>(want < 1 ? 1 : (want < cap ? want : cap));
  return launch_kernel_cooperative(global_scale_quantize_kernel, dim3(grid), dim3(kGsqThreads),
                                   static_cast<size_t>(smem), stream, xmap, p, ws, amax_out, gsf_out, other_amax,
                                   alpha_out, info.status, withheld);
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

int nvfp4_global_scale(const void* x_bf16, int64_t numel, float* amax_out, float* gsf_out,
                       const float* other_amax, float* alpha_out, nvfp4_stream_t stream) {
  return launch_amax_dense(x_bf16, numel, amax_out, gsf_out, other_amax, alpha_out, stream);
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
  return launch_kernel(silu_mul ? amax_batched_kernel<true> : amax_batched_kernel<false>, grid, dim3(kThreads), 0,
                       stream, x, static_cast<int32_t>(m), static_cast<int32_t>(k), mask, ws, amax_out, gsf_out,
                       info.status);
}

int nvfp4_quantize(const void* x_bf16, int64_t m, int64_t k, const float* gsf, uint8_t* q_out, uint8_t* sf_out,
                   nvfp4_stream_t stream) {
  return launch_quantize(x_bf16, 1, m, k, false, nullptr, gsf, q_out, sf_out, stream);
}

int nvfp4_silu_and_mul(const void* x_bf16, int64_t rows, int64_t k, void* h_bf16, nvfp4_stream_t stream) {
  if (rows < 0 || k < 0 || k % 8 != 0 || k > (1 << 30)) return NVFP4_ERR_INVALID_ARGUMENT;
  if (rows == 0 || k == 0) return NVFP4_OK;
  if (!x_bf16 || !h_bf16 || !aligned(x_bf16, 16) || !aligned(h_bf16, 16)) return NVFP4_ERR_INVALID_ARGUMENT;
  DeviceInfo info;
  int st = current_device(&info);
  if (st != NVFP4_OK) return st;
  const int64_t total = rows * (k / 8);
  int64_t blocks = (total + kThreads - 1) / kThreads;
  blocks = blocks > info.sm_count * 4 ? info.sm_count * 4 : blocks;
  return launch_kernel(silu_and_mul_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), kSiluTableBytes,
                       stream, static_cast<const uint16_t*>(x_bf16), rows, static_cast<int32_t>(k),
                       static_cast<uint16_t*>(h_bf16), info.silu_table, info.status);
}

int nvfp4_quantize_smooth(const void* x_bf16, int64_t m, int64_t k, const void* pre_quant_scale_bf16,
                          const float* gsf, uint8_t* q_out, uint8_t* sf_out, nvfp4_stream_t stream) {
  if (!pre_quant_scale_bf16 && m > 0 && k > 0) return NVFP4_ERR_INVALID_ARGUMENT;
  return launch_quantize(x_bf16, 1, m, k, false, nullptr, gsf, q_out, sf_out, stream, pre_quant_scale_bf16);
}

int nvfp4_global_scale_quantize(const void* x_bf16, int64_t m, int64_t k, float* amax_out, float* gsf_out,
                                const float* other_amax, float* alpha_out, uint8_t* q_out, uint8_t* sf_out,
                                nvfp4_stream_t stream) {
  return launch_global_scale_quantize(x_bf16, m, k, amax_out, gsf_out, other_amax, alpha_out, q_out, sf_out, stream, 0);
}

int nvfp4_selftest_grid_barrier(const void* x_bf16, int64_t m, int64_t k, float* gsf_out, uint8_t* q_out,
                                uint8_t* sf_out, nvfp4_stream_t stream) {
  return launch_global_scale_quantize(x_bf16, m, k, nullptr, gsf_out, nullptr, nullptr, q_out, sf_out, stream, 1);
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
// Some callers cannot let the library call cudaMalloc: hosts whose device memory is owned
// by their own allocator or fixed at start-up (inference servers with a pre-sized pool,
// embedded deployments), and latency-critical paths that must not risk the implicit device
// synchronization cudaMalloc can cause.  nvfp4_global_scale_batched_noalloc serves them:
// its reduction scratch is the file-scope device array below instead of the lazily
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
  return launch_kernel(silu_mul ? amax_batched_kernel<true> : amax_batched_kernel<false>, grid, dim3(kThreads), 0,
                       stream, x, static_cast<int32_t>(m), static_cast<int32_t>(k), mask, scratch, amax_out, gsf_out,
                       static_cast<int*>(nullptr));
}
