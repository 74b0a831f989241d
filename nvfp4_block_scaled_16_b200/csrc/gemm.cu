// gemm.cu -- block-scaled NVFP4 GEMMs on the 5th-generation tensor cores (tcgen05).
//
//   nvfp4_gemm                 out = bf16(alpha * a @ b^T [+ bias])
//   nvfp4_gemm_lowrank_bias    out = bf16(alpha * (a @ b^T + d @ l1^T) [+ bias])
//   nvfp4_grouped_gemm_masked  out[e, i] = bf16(alpha[e] * a[e, i] @ b[e]^T), i < mask[e]
//   nvfp4_gemm_silu_mul_quantize (and its masked grouped form)
//                              g = bf16(alpha_gate * a @ b_gate^T), u = bf16(alpha_up * a @ b_up^T),
//                              h = bf16(silu(g) * u) quantized to NVFP4 in the epilogue
//
// Sources (page title, section): flashinfer docs mm_nvfp4_svdquant (signature,
// Parameters: packed (m, k/2) and (n, k/2) operands, 128x4-swizzled ue4m3 scales,
// alpha device scalar; the rank-r bf16 correction is one more MMA that adds into the
// FP4 K-loop's TMEM accumulator once that loop ends; epilogue alpha*acc + bias); TensorRT-LLM
// NVFP4LinearMethod.create_weights (weight [out, in/2], alpha); flashinfer PR #1774
// "Masked batch nvfp4 quantization" (masked per-expert operands for the grouped GEMM, and
// the silu_and_mul quantizer whose input is the gate/up projection's output); the Llama4
// MoE description on the same pages (routed experts: gate/up projection, SiLU * up, down
// projection).
//
// Kernel structure.  CTA pairs (clusters of 2 on one TPC) are persistent over output
// tiles of 256 x 256.  Each CTA of a pair owns 128 rows of the A tile and 128 rows (one
// half of N) of the B tile; the leader CTA issues tcgen05.mma.cta_group::2 (M = 256,
// N = 256, K = 64, kind::mxf4nvf4 with ue4m3 scales per 16 values) for both, so each
// SM streams only its own operand halves through shared memory.  Each CTA's tensor
// memory holds the scales of its own 128 A rows and of all 256 B rows of the tile.
//   warp 0      TMA producer (both CTAs): tiled loads (cta_group::2 form, no multicast)
//               of the packed operands (128-byte swizzle, one 128-byte K row = 256 FP4
//               values per stage) and of the scale chunks (each 128-row x 4-block group
//               of the 128x4 layout is one contiguous 512-byte chunk); all loads of both
//               CTAs complete on the leader's stage barrier.  5-stage ring.
//   warp 1      TMEM allocator (both CTAs) and MMA issuer (leader, one thread): per
//               K-step one tcgen05.cp (32x128b, replicated to the 4 lane quarters) of the
//               SFA chunk and two of the SFB chunks, each CTA from its own shared memory
//               into its own tensor memory, then the MMA; the low-rank term follows as kind::f16 (bf16) MMAs into the same
//               accumulator.  Commits are multicast to both CTAs.
//   warps 2-9   epilogue (both CTAs): tcgen05.ld of the CTA's 128 x 256 fp32 accumulator,
//               two warps per 32-lane TMEM quarter (each warp can only read its own
//               quarter), each draining two of the four 64-column subtiles: alpha * acc +
//               bias, bf16 staged in shared memory and written by TMA stores (one 32 x 64
//               tile at a time).  The grouped bf16 kernel keeps one warp per quarter
//               (warps 2-5, all four subtiles).  The SiLU * up epilogue: two warps per
//               quarter, each with 64 of the tile's 128 h columns.
// Two accumulators of 256 columns share TMEM columns [192, 256): the epilogue drains that
// overlap first and releases the accumulator, so the next tile's MMAs overlap the rest of
// the epilogue.  Scale factors use columns [448, 496).
// SiLU * up epilogue: the B half of CTA 0 is 128 rows of the gate weight and the B half of
// CTA 1 the same 128 rows of the up weight, so accumulator columns [0, 128) hold g and
// [128, 256) hold u for 128 columns of h.  Each thread owns 64 columns of one row: it rounds
// g and u to bf16 exactly as the bf16 epilogue would, forms h with silu(g) from the SiLU table
// (copied into shared memory by the epilogue warps at the start), and quantizes each
// 16-value block with the caller's global scale (32 code bytes and 4 scale bytes per row,
// warp and tile).  Every
// epilogue warp loads all its accumulator columns before any arithmetic and releases the
// accumulator right after, so the next tile's MMAs overlap the whole SiLU and quantization.
// Every mbarrier wait is bounded (about one second of global time); a wait that runs out
// records NVFP4_ERR_DEVICE_TIMEOUT in the device status word and the CTA unwinds without
// hanging the GPU.
#include <cstddef>
#include <cuda_bf16.h>

#include "common.cuh"
#include "nvfp4_math.cuh"
#include "tc_common.cuh"

namespace nvfp4 {
namespace {

constexpr int kBM = 128;                 // A rows per CTA (MMA M = 256 per pair)
constexpr int kBN = 256;                 // MMA N per pair tile
constexpr int kBNHalf = 128;             // B rows per CTA
constexpr int kTileM = 2 * kBM;          // output tile rows per pair
constexpr int kStageK = 256;             // FP4 values of K per stage (128 bytes per row)
constexpr int kStageBytesRow = kStageK / 2;
constexpr int kStages = 5;
constexpr int kABytes = kBM * kStageBytesRow;        // 16 KB
constexpr int kBBytes = kBNHalf * kStageBytesRow;    // 16 KB
constexpr int kSfaBytes = 4 * 512;                   // 4 K-steps x one 512-byte chunk
constexpr int kSfbBytes = 2 * 4 * 512;               // both 128-row halves of the N tile
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;  // 38 KB
constexpr uint32_t kFp4TxBytes = 2u * kStageBytes;              // both CTAs
constexpr uint32_t kLrTxBytes = 2u * (kABytes + kBBytes);
constexpr int kMaxExperts = 1024;
// Warps: 0 TMA producer, 1 MMA issuer, then kQW epilogue warps per TMEM lane quarter.  Two
// per quarter (each draining half of the tile's columns) halve a tile's epilogue, which pays
// when the epilogue is on the critical path: short K loops, few tiles.  On long K loops the
// epilogue hides behind the next tile's mainloop anyway, and one warp per quarter (with two
// staging tiles) leaves more issue slots to the producer and MMA warps: measured 118.9 against
// 122.9 us on 8192 x 5120 x 8192 and 233.5 against 247.8 us on 8192 x 16384 x 5120, but 30.7
// against 28.7 us on 4096 x 3072 x 3072.  The SiLU * up epilogue always uses two.
template <int kQW>
constexpr int kEpiWarps = 4 * kQW;
template <int kQW>
constexpr int kThreads = 64 + 32 * kEpiWarps<kQW>;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccOverlapCol = 192;          // accumulator 1 starts here
constexpr uint32_t kSfaCol = 448;                 // SFA: 448 + 4j, SFB: 464 + 8j (+4 upper half)
constexpr uint32_t kSfbCol = 464;

// smem layout after the stage ring
struct __align__(8) Control {
  uint64_t full[kStages];     // leader: all loads of a stage (both CTAs) landed
  uint64_t empty[kStages];    // both: the stage's MMAs completed (multicast commit)
  uint64_t acc_full;          // both: the tile's accumulator is complete (multicast commit)
  uint64_t acc_empty;         // leader: the epilogues of both CTAs drained the overlap
  uint32_t tmem_base;
  int32_t abort;
  int32_t prefix[kMaxExperts + 1];   // grouped: prefix sums of pair tiles per expert
};
// bf16 epilogue: 32-row x 64-column bf16 staging tiles (4 KB, 128-byte swizzle) per epilogue
// warp, written to global memory by TMA stores: two per warp (one store in flight while the
// next tile is written) with one warp per quarter, one with two (or in the grouped kernel,
// whose expert prefix table takes the room).
constexpr int kStoreTileBytes = 32 * 128;
template <bool kGrouped, bool kSwiGLU, int kQW>
constexpr int kStagingBuffers = kSwiGLU ? 0 : ((kQW == 1 && !kGrouped) ? 2 : 1);
template <bool kGrouped, bool kSwiGLU, int kQW>
constexpr int kStagingBytes = kStagingBuffers<kGrouped, kSwiGLU, kQW> * kEpiWarps<kQW> * kStoreTileBytes;
// SiLU * up epilogue: the SiLU table (32 KB) after the ring.
template <bool kSwiGLU>
constexpr int kTableBytes = kSwiGLU ? static_cast<int>(kSiluTableBytes) : 0;
// The expert prefix table (the last member of Control) is only allocated for grouped kernels;
// the fused activation quantizer keeps its 128 inverse block scales in its first 512 bytes.
template <bool kGrouped, bool kQuantA = false>
constexpr int kControlBytes = kGrouped  ? static_cast<int>(sizeof(Control))
                              : kQuantA ? static_cast<int>(offsetof(Control, prefix)) + 512
                                        : static_cast<int>(offsetof(Control, prefix)) + 8;
template <bool kGrouped, bool kSwiGLU, int kQW, bool kQuantA = false>
constexpr int kSmemBytes = kStages * kStageBytes + kStagingBytes<kGrouped, kSwiGLU, kQW> + kTableBytes<kSwiGLU> +
                           kControlBytes<kGrouped, kQuantA> + 1024;
constexpr int kMaxDynamicSmem = 227 * 1024;      // sm_100 opt-in limit per block
static_assert(kSmemBytes<false, false, 1> <= kMaxDynamicSmem && kSmemBytes<false, false, 2> <= kMaxDynamicSmem &&
                  kSmemBytes<true, false, 1> <= kMaxDynamicSmem && kSmemBytes<false, true, 2> <= kMaxDynamicSmem &&
                  kSmemBytes<true, true, 2> <= kMaxDynamicSmem && kSmemBytes<false, false, 1, true> <= kMaxDynamicSmem &&
                  kSmemBytes<false, false, 2, true> <= kMaxDynamicSmem,
              "shared memory layout exceeds the per-block limit");
constexpr int kQuantAMaxChunks = 64;             // fused activation quantizer: k <= 64 * 256

// Instruction descriptors (tcgen05 "instruction descriptor" bit fields).
//   kind::mxf4nvf4: A/B format E2M1 (1) at bits 7..9 / 10..12, both K-major, N>>3 at
//   bits 17..22, ue4m3 scale format (0) at bit 23, M>>4 at bits 24..28, scale ids 0.
constexpr uint32_t kIdescFp4 = (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) | (uint32_t(kTileM >> 4) << 24);
//   kind::f16: fp32 accumulator (1) at bits 4..5, A/B bf16 (1), K-major, N, M as above.
constexpr uint32_t kIdescBf16 =
    (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) | (uint32_t(kTileM >> 4) << 24);

// ---- PTX wrappers ---------------------------------------------------------------------------

// Tiled TMA loads into this CTA's shared memory, completing on the barrier at the
// shared::cluster address `bar` (the leader's; the .cta_group::2 form allows either CTA
// of the pair).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint32_t bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint32_t bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// One 512-byte scale chunk as 32 rows x 16 bytes: 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t sf_desc(uint32_t addr) { return smem_desc(addr, 0, 128, 0); }

// Copies a 512-byte scale chunk at the same smem address of both CTAs into 4 TMEM columns
// (all 128 lanes) of both CTAs.
__device__ __forceinline__ void tc_copy_sf(uint32_t tmem_col_addr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(tmem_col_addr), "l"(desc) : "memory");
}

__device__ __forceinline__ void mma_fp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t sfa, uint32_t sfb,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(kIdescFp4), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(kIdescBf16), "r"(accumulate)
      : "memory");
}

// Arrives on the barrier at the same smem offset in both CTAs once every prior
// tcgen05 operation of this thread has completed.
__device__ __forceinline__ void mma_commit_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}

// bf16(alpha * a), bf16(alpha * b) packed (a in the low half): the rounding of the bf16
// epilogue, applied to two fp32 accumulator values given as bits.
__device__ __forceinline__ uint32_t scale_round_bf16x2(float alpha, uint32_t a, uint32_t b) {
  float pa, pb;
  unpack2(mul2(pack2(__uint_as_float(a), __uint_as_float(b)), splat2(alpha)), pa, pb);
  uint32_t w;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(pb), "f"(pa));   // pa -> low half
  return w;
}

// ---- problem description ----------------------------------------------------------------------

struct GemmParams {
  const float* alpha;         // [1] or [E]
  const __nv_bfloat16* bias;  // nullable [n]
  __nv_bfloat16* out;         // [E, mmax, n] (E = 1 for dense)
  const int32_t* mask;        // grouped only
  int* status;
  int32_t m;                  // rows per expert (mmax)
  int32_t n;
  int32_t k;
  int32_t experts;
  int32_t rank;               // low-rank r (0 = none)
  int32_t n_tiles;            // ceil(n / 256)
  int32_t m_tiles;            // dense: ceil(m / 256)
  int32_t k_stages;           // ceil(k / 256)
  int32_t k_steps;            // k / 64
  int32_t sf_groups;          // k / 64: 512-byte chunks per 128-row tile
  // SiLU * up epilogue (n is the width of h; b is the gate weight, b2 the up weight)
  const float* alpha_up;      // [1] or [E]: alpha of the up projection (alpha: gate)
  const float* gsf_h;         // [1] or [E]: global scale of h
  uint8_t* q;                 // [E, mmax, n/2] packed codes of h
  uint8_t* sf;                // [E][nvfp4_scale_bytes(mmax, n)] swizzled scales of h
  int64_t sf_item_stride;     // nvfp4_scale_bytes(mmax, n)
  int32_t rows_pad;           // pad_up(mmax, 128)
  int32_t stall_stage;        // self-test only: K stage of each pair's first tile whose loads
                              // are withheld, so a bounded wait runs out (-1: none)
  const float* silu_tab;      // SiLU * up epilogue: the SiLU table in global memory
  // fused activation quantizer (the bf16-activation linear with a static activation scale):
  // A is x quantized with qa_gsf into qa_q / qa_sf (which the A and SFA tensor maps read)
  const uint16_t* qa_x;       // [m, k] bf16
  const float* qa_gsf;        // [1] static global scale of x
  uint8_t* qa_q;              // [m, k/2]
  uint8_t* qa_sf;             // [nvfp4_scale_bytes(m, k)]
  uint32_t* qa_ws;            // stream workspace: [0] CTAs finished, [1 + c] 128-row slabs of K chunk c done
  int32_t qa_slabs;           // ceil(m / 128)
};

struct TileCoord {
  int expert, m_tile, n_tile, valid_rows;
};

template <bool kGrouped>
__device__ __forceinline__ bool tile_coord(const GemmParams& p, const Control& ctl, int tile, TileCoord& t) {
  if constexpr (!kGrouped) {
    if (tile >= p.m_tiles * p.n_tiles) return false;
    t.expert = 0;
    t.m_tile = tile % p.m_tiles;
    t.n_tile = tile / p.m_tiles;
    t.valid_rows = p.m;
    return true;
  } else {
    if (tile >= ctl.prefix[p.experts]) return false;
    int e = 0;
    while (ctl.prefix[e + 1] <= tile) ++e;
    const int local = tile - ctl.prefix[e];
    const int mt = (ctl.prefix[e + 1] - ctl.prefix[e]) / p.n_tiles;
    t.expert = e;
    t.m_tile = local % mt;
    t.n_tile = local / mt;
    t.valid_rows = min(max(p.mask[e], 0), p.m);
    return true;
  }
}

struct Maps {
  CUtensorMap a, b, sfa, sfb, d, l1;
  CUtensorMap b2, sfb2;       // SiLU * up: the up weight and its scales
  CUtensorMap out;            // bf16 output [E, mmax, n], boxes of 32 rows x 64 columns
};

// ---- fused activation quantizer ------------------------------------------------------------------
// The work is split into units of one 128-row slab x one 256-column K chunk of x (2048 blocks
// of 16 values), numbered chunk-major (u = c * slabs + s), so that every slab's early chunks are
// ready first; CTA j quantizes units j, j + grid, ... with its epilogue warps before they drain
// any accumulator, and counts each finished unit in qa_ws[1 + c] with release semantics.  A
// producer loads chunk c of a slab only after it has seen qa_ws[1 + c] == slabs (acquire), and
// remembers the chunks it has seen.

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// orders this thread's generic-proxy global accesses with its async-proxy (TMA) ones
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// Quantizes this CTA's units with the kEpi epilogue threads (t = thread index among them):
// item i = it * kEpi + t of a unit is row i / 16, block i % 16 of the chunk, so a warp reads
// two rows' 512 contiguous bytes and writes their 128 contiguous code bytes; the four blocks
// of a scale group sit in adjacent lanes and one of them writes the group's 4-byte word.
template <int kEpi>
__device__ void quantize_a_units(const GemmParams& p, int t, float* inv_tab) {
  constexpr int kItems = 2048 / kEpi;            // items per thread and unit
  constexpr int kBatch = kItems < 8 ? kItems : 8; // loads in flight per thread
  const float gsf = __ldg(p.qa_gsf);
  if (t < 128) inv_tab[t] = inv_scale(static_cast<uint32_t>(t), gsf);
  asm volatile("bar.sync 1, %0;" ::"n"(kEpi) : "memory");
  const int nb = p.k / 16;
  const uint32_t groups = static_cast<uint32_t>(p.sf_groups);
  const int units = p.qa_slabs * p.k_stages;
  const int lane = t & 31;
  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const int c = u / p.qa_slabs, slab = u - c * p.qa_slabs;
    const int nblk = min(16, nb - 16 * c);       // blocks of this chunk in a row (a multiple of 4)
    for (int it0 = 0; it0 < kItems; it0 += kBatch) {
      uint4 raw[kBatch][2];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int i = (it0 + b) * kEpi + t;
        const int row = slab * 128 + i / 16, blk = i % 16;
        if (row < p.m && blk < nblk &&
            index_ok(static_cast<uint64_t>(row) * p.k + (16 * c + blk) * 16 + 15, static_cast<uint64_t>(p.m) * p.k,
                     p.status)) {
          const uint16_t* src = p.qa_x + static_cast<int64_t>(row) * p.k + (16 * c + blk) * 16;
          raw[b][0] = __ldg(reinterpret_cast<const uint4*>(src));
          raw[b][1] = __ldg(reinterpret_cast<const uint4*>(src + 8));
        } else {
          raw[b][0] = raw[b][1] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        const int i = (it0 + b) * kEpi + t;
        const int row = slab * 128 + i / 16, blk = i % 16;
        float v[16];
        const uint32_t w[8] = {raw[b][0].x, raw[b][0].y, raw[b][0].z, raw[b][0].w,
                               raw[b][1].x, raw[b][1].y, raw[b][1].z, raw[b][1].w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          v[2 * e] = bf16_lo(w[e]);
          v[2 * e + 1] = bf16_hi(w[e]);
        }
        const QBlock qb = quantize16(v, gsf, inv_tab);
        // the scale group's four bytes, from the lanes of blocks 4g .. 4g + 3 (lane = i % 32)
        const uint32_t s1 = __shfl_down_sync(0xffffffffu, qb.s8, 1);
        const uint32_t s2 = __shfl_down_sync(0xffffffffu, qb.s8, 2);
        const uint32_t s3 = __shfl_down_sync(0xffffffffu, qb.s8, 3);
        if (blk < nblk && row < p.m) {
          const int64_t qo = static_cast<int64_t>(row) * (p.k / 2) + (16 * c + blk) * 8;
          if (index_ok(qo + 7, static_cast<uint64_t>(p.m) * (p.k / 2), p.status))
            *reinterpret_cast<uint2*>(p.qa_q + qo) = make_uint2(qb.lo, qb.hi);
        }
        if (blk < nblk && (lane & 3) == 0 && row < slab * 128 + 128) {
          // rows of the slab beyond m are padding: their scale words are zero
          const uint32_t word = row < p.m ? (qb.s8 | (s1 << 8) | (s2 << 16) | (s3 << 24)) : 0u;
          const int64_t so = sf_offset(static_cast<uint32_t>(row), static_cast<uint32_t>(16 * c + blk), groups);
          if (index_ok(so + 3, static_cast<uint64_t>(p.qa_slabs) * 128 * groups * 4, p.status))
            *reinterpret_cast<uint32_t*>(p.qa_sf + so) = word;
        }
      }
    }
    fence_proxy_async_global();                  // the producers read these bytes with TMA
    asm volatile("bar.sync 1, %0;" ::"n"(kEpi) : "memory");
    if (t == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(p.qa_ws + 1 + c) : "memory");
  }
}

// ---- the kernel ---------------------------------------------------------------------------------

template <bool kGrouped, bool kLowRank, bool kSwiGLU, int kQW, bool kQuantA = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads<kQW>, 1)
    nvfp4_gemm_kernel(const __grid_constant__ Maps maps, const GemmParams p) {
  static_assert(!kQuantA || (!kGrouped && !kLowRank && !kSwiGLU), "the fused activation quantizer is dense only");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + kStages * kStageBytes;     // 1024-byte aligned (the ring is 190 KB)
  float* silu_tab = reinterpret_cast<float*>(staging + kStagingBytes<kGrouped, kSwiGLU, kQW>);
  Control& ctl = *reinterpret_cast<Control*>(staging + kStagingBytes<kGrouped, kSwiGLU, kQW> + kTableBytes<kSwiGLU>);
  volatile int32_t* abort = &ctl.abort;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();           // 0 = leader of the pair
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.empty[s], 1);
    }
    mbar_init(&ctl.acc_full, 1);
    mbar_init(&ctl.acc_empty, 2 * kEpiWarps<kQW>);   // every epilogue warp of both CTAs
    ctl.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&ctl.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();      // the leader's barriers are initialized before the peer signals them
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  // Programmatic dependent launch: the set-up above touched only this CTA's own resources;
  // global memory is accessed only after the preceding kernel of the stream has finished.
  pdl_launch_dependents();
  pdl_wait();
  if constexpr (kGrouped) {
    if (threadIdx.x == 32) {
      int acc = 0;
      ctl.prefix[0] = 0;
      for (int e = 0; e < p.experts; ++e) {
        const int valid = min(max(p.mask[e], 0), p.m);
        acc += (valid + kTileM - 1) / kTileM * p.n_tiles;
        ctl.prefix[e + 1] = acc;
      }
    }
    __syncthreads();
  }

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    // The whole warp runs the loop; one elected lane issues each stage's loads.
    if (elect_one()) {
      prefetch_map(&maps.a);
      prefetch_map(&maps.b);
      prefetch_map(&maps.sfa);
      prefetch_map(&maps.sfb);
      if constexpr (kSwiGLU) {
        prefetch_map(&maps.b2);
        prefetch_map(&maps.sfb2);
      }
      if constexpr (kLowRank) {
        prefetch_map(&maps.d);
        prefetch_map(&maps.l1);
      }
    }
    __syncwarp();
    const int lr_stages = kLowRank ? (p.rank + 63) / 64 : 0;
    uint32_t s = 0, phase = 0;
    bool wrapped = false;      // the ring has been filled once: every later stage waits for its slot
    bool ok = true;
    uint64_t chunks_ready = 0;   // fused activation quantizer: K chunks seen complete for every slab
    TileCoord t;
    for (int tile = pair; ok && tile_coord<kGrouped>(p, ctl, tile, t); tile += pairs) {
      const int a_row = t.m_tile * kTileM + static_cast<int>(rank) * kBM;
      // 128-row tiles of B in the two halves of the pair tile: adjacent tiles of b, or for
      // the SiLU * up epilogue the same tile of the gate weight (b) and the up weight (b2)
      const int b_tile0 = kSwiGLU ? t.n_tile : 2 * t.n_tile;
      const int b_tile1 = kSwiGLU ? t.n_tile : 2 * t.n_tile + 1;
      const int b_row = (rank ? b_tile1 : b_tile0) * kBNHalf;
      const CUtensorMap* b_map = (kSwiGLU && rank) ? &maps.b2 : &maps.b;
      const CUtensorMap* sfb1_map = kSwiGLU ? &maps.sfb2 : &maps.sfb;
      // scale chunk rows (128 bytes each, 4 per chunk): this CTA's 128 A rows, both B halves
      const int sfa_row0 = ((2 * t.m_tile + static_cast<int>(rank)) * p.sf_groups) * 4;
      const int sfb_row0 = (b_tile0 * p.sf_groups) * 4;
      const int sfb_row1 = (b_tile1 * p.sf_groups) * 4;
      for (int ks = 0; ks < p.k_stages + lr_stages; ++ks) {
        if (wrapped && !(ok = mbar_wait_fast(&ctl.empty[s], phase, abort, p.status))) break;
        uint8_t* st = smem + s * kStageBytes;
        const uint32_t full_bar = map_to_rank(&ctl.full[s], 0);
        const bool withheld = ks == p.stall_stage && tile == pair;   // self-test: nothing completes it
        if constexpr (kQuantA) {
          if (ks < p.k_stages && !((chunks_ready >> ks) & 1ull)) {
            // wait (bounded) until every slab's chunk ks is quantized: each poll reads the
            // counters of all chunks not yet seen (lane l: chunks l and l + 32) in one round
            // trip, and the chunks found complete are remembered
            const uint64_t t0 = global_ns();
            for (uint32_t i = 0;; ++i) {
              uint32_t lo = 0, hi = 0;
              if (lane < p.k_stages && !((chunks_ready >> lane) & 1ull))
                lo = ld_acquire_u32(p.qa_ws + 1 + lane) >= static_cast<uint32_t>(p.qa_slabs);
              if (lane + 32 < p.k_stages && !((chunks_ready >> (lane + 32)) & 1ull))
                hi = ld_acquire_u32(p.qa_ws + 33 + lane) >= static_cast<uint32_t>(p.qa_slabs);
              chunks_ready |= static_cast<uint64_t>(__ballot_sync(0xffffffffu, lo)) |
                              (static_cast<uint64_t>(__ballot_sync(0xffffffffu, hi)) << 32);
              if ((chunks_ready >> ks) & 1ull) break;
              if ((i & 15u) == 15u) {
                bool give_up = *abort != 0;
                if (!give_up && global_ns() - t0 > kWaitLimitNs) {
                  give_up = true;
                  if (lane == 0) {
                    *abort = 1;
                    atomicExch(p.status, NVFP4_ERR_DEVICE_TIMEOUT);
                  }
                }
                if (__any_sync(0xffffffffu, give_up)) break;
              }
            }
            if (!(ok = ((chunks_ready >> ks) & 1ull) != 0)) break;
            fence_proxy_async_global();   // the TMA loads below read what other CTAs stored
          }
        }
        if (!withheld && elect_one()) {
          if (ks < p.k_stages) {
            if (leader) mbar_arrive_expect_tx(&ctl.full[s], kFp4TxBytes);
            if constexpr (kGrouped) {
              tma_load_3d(st, &maps.a, full_bar, ks * kStageBytesRow, a_row, t.expert);
              tma_load_3d(st + kABytes, b_map, full_bar, ks * kStageBytesRow, b_row, t.expert);
              tma_load_3d(st + kABytes + kBBytes, &maps.sfa, full_bar, 0, sfa_row0 + 16 * ks, t.expert);
              tma_load_3d(st + kABytes + kBBytes + kSfaBytes, &maps.sfb, full_bar, 0, sfb_row0 + 16 * ks, t.expert);
              tma_load_3d(st + kABytes + kBBytes + kSfaBytes + kSfaBytes, sfb1_map, full_bar, 0, sfb_row1 + 16 * ks,
                          t.expert);
            } else {
              tma_load_2d(st, &maps.a, full_bar, ks * kStageBytesRow, a_row);
              tma_load_2d(st + kABytes, b_map, full_bar, ks * kStageBytesRow, b_row);
              tma_load_2d(st + kABytes + kBBytes, &maps.sfa, full_bar, 0, sfa_row0 + 16 * ks);
              tma_load_2d(st + kABytes + kBBytes + kSfaBytes, &maps.sfb, full_bar, 0, sfb_row0 + 16 * ks);
              tma_load_2d(st + kABytes + kBBytes + kSfaBytes + kSfaBytes, sfb1_map, full_bar, 0, sfb_row1 + 16 * ks);
            }
          } else if constexpr (kLowRank) {
            const int c = ks - p.k_stages;
            if (leader) mbar_arrive_expect_tx(&ctl.full[s], kLrTxBytes);
            tma_load_2d(st, &maps.d, full_bar, c * 64, a_row);
            tma_load_2d(st + kABytes, &maps.l1, full_bar, c * 64, b_row);
          }
        }
        __syncwarp();
        if (++s == kStages) {
          s = 0;
          if (wrapped) phase ^= 1u;
          wrapped = true;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader)
    // The whole warp runs the loop; one elected lane issues each stage's tcgen05 ops.  The
    // loop is kept lean (stage slot and phase tracked incrementally, descriptors built
    // once per stage and advanced by 32 bytes per K-step): the tensor pipe finishes one
    // M256 N256 K64 MMA every ~128 cycles, so issue overhead shows directly in the rate.
    if (leader) {
      const int lr_stages = kLowRank ? (p.rank + 63) / 64 : 0;
      const uint32_t smem0 = smem_u32(smem);
      const uint64_t a_desc0 = operand_desc(smem0);
      const uint64_t b_desc0 = operand_desc(smem0 + kABytes);
      const uint64_t sfa_desc0 = sf_desc(smem0 + kABytes + kBBytes);
      const uint64_t sfb_desc0 = sf_desc(smem0 + kABytes + kBBytes + kSfaBytes);
      uint32_t s = 0, phase = 0, tcount = 0;
      bool ok = true;
      TileCoord t;
      for (int tile = pair; ok && tile_coord<kGrouped>(p, ctl, tile, t); tile += pairs, ++tcount) {
        const uint32_t acc = tmem + ((tcount & 1) ? kAccOverlapCol : 0u);
        if (tcount > 0) {
          if (!(ok = mbar_wait_fast(&ctl.acc_empty, (tcount - 1) & 1, abort, p.status))) break;
          tc_fence_after();
        }
        for (int ks = 0; ks < p.k_stages + lr_stages; ++ks) {
          if (!(ok = mbar_wait_fast(&ctl.full[s], phase, abort, p.status))) break;
          tc_fence_after();
          const uint64_t off = (s * kStageBytes) >> 4;     // descriptor address units (16 bytes)
          const uint64_t da = a_desc0 + off, db = b_desc0 + off;
          if (elect_one()) {
            if (ks < p.k_stages) {
              const uint64_t dsa = sfa_desc0 + off, dsb = sfb_desc0 + off;
              const uint32_t acc_first = ks > 0 ? 1u : 0u;
              const int nks = p.k_steps - 4 * ks;
              if (nks >= 4) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  tc_copy_sf(tmem + kSfaCol + 4 * j, dsa + 32 * j);
                  tc_copy_sf(tmem + kSfbCol + 8 * j, dsb + 32 * j);
                  tc_copy_sf(tmem + kSfbCol + 8 * j + 4, dsb + (kSfaBytes >> 4) + 32 * j);
                  mma_fp4(acc, da + 2 * j, db + 2 * j, tmem + kSfaCol + 4 * j, tmem + kSfbCol + 8 * j,
                          j > 0 ? 1u : acc_first);
                }
              } else {
                for (int j = 0; j < nks; ++j) {
                  tc_copy_sf(tmem + kSfaCol + 4 * j, dsa + 32 * j);
                  tc_copy_sf(tmem + kSfbCol + 8 * j, dsb + 32 * j);
                  tc_copy_sf(tmem + kSfbCol + 8 * j + 4, dsb + (kSfaBytes >> 4) + 32 * j);
                  mma_fp4(acc, da + 2 * j, db + 2 * j, tmem + kSfaCol + 4 * j, tmem + kSfbCol + 8 * j,
                          j > 0 ? 1u : acc_first);
                }
              }
            } else if constexpr (kLowRank) {
              const int c = ks - p.k_stages;
              const int steps = min(4, (p.rank - 64 * c) / 16);
              for (int j = 0; j < steps; ++j) mma_bf16(acc, da + 2 * j, db + 2 * j, 1u);
            }
            mma_commit_both(&ctl.empty[s]);
          }
          __syncwarp();
          if (++s == kStages) {
            s = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (elect_one()) mma_commit_both(&ctl.acc_full);
        __syncwarp();
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;              // TMEM lane quarter this warp may access
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t acc_empty_leader = map_to_rank(&ctl.acc_empty, 0);
    if constexpr (kSwiGLU) {
      // the epilogue warps load the SiLU table while the first tile's mainloop runs
      silu_table_load(silu_tab, p.silu_tab, threadIdx.x - 64, 32 * kEpiWarps<kQW>);
      asm volatile("bar.sync 1, %0;" ::"n"(32 * kEpiWarps<kQW>) : "memory");
    }
    if constexpr (kQuantA) quantize_a_units<32 * kEpiWarps<kQW>>(p, threadIdx.x - 64, reinterpret_cast<float*>(ctl.prefix));
    uint32_t tcount = 0;
    TileCoord t;
    uint32_t nstore = 0;                       // TMA stores issued by this warp (bf16 epilogue)
    for (int tile = pair; tile_coord<kGrouped>(p, ctl, tile, t); tile += pairs, ++tcount) {
      // per-tile scalars, loaded before the wait so their latency hides behind the mainloop
      const float alpha = __ldg(p.alpha + t.expert);
      float gsf = 0.0f, alpha_u = 0.0f;
      if constexpr (kSwiGLU) {
        gsf = __ldg(p.gsf_h + t.expert);
        alpha_u = __ldg(p.alpha_up + t.expert);
      }
      if (!mbar_wait(&ctl.acc_full, tcount & 1, abort, p.status)) break;
      tc_fence_after();
      const uint32_t buf = tcount & 1;
      const uint32_t col0 = buf ? kAccOverlapCol : 0u;
      const int row = t.m_tile * kTileM + static_cast<int>(rank) * kBM + row_in_tile;
      const bool row_ok = row < t.valid_rows;
      if constexpr (kSwiGLU) {
        // h columns [128 n_tile, 128 n_tile + 128): g in accumulator columns [0, 128), u in
        // [128, 256); this warp's half of them is loaded whole, then the accumulator released.
        const bool pad_row = !kGrouped && row >= p.m && row < p.rows_pad;   // zero scales
        uint8_t* q_row = p.q + (static_cast<int64_t>(t.expert) * p.m + row) * (p.n / 2) + t.n_tile * 64;
        uint8_t* sf_e = p.sf + static_cast<int64_t>(t.expert) * p.sf_item_stride;
        const uint32_t groups = static_cast<uint32_t>(p.n / 64);
        {
          constexpr int kQuarterWarps = kQW;                     // epilogue warps per lane quarter
          constexpr int kCols = 128 / kQuarterWarps;            // h columns of this warp
          constexpr int kBlocks = kCols / 16;                   // 16-value blocks per thread
          const int part = (warp - 2) >> 2;                     // which kCols-wide slice
          uint32_t g[kCols], u[kCols];
          if constexpr (kCols == 64) {
            tmem_load_64(tmem + col0 + part * kCols + lane_base, g);
            tmem_load_64(tmem + col0 + 128 + part * kCols + lane_base, u);
          } else {
            tmem_load_32(tmem + col0 + part * kCols + lane_base, g);
            tmem_load_32(tmem + col0 + 128 + part * kCols + lane_base, u);
          }
          tmem_wait_ld<kCols>(g);
          tmem_wait_ld<kCols>(u);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
          const uint32_t c0 = static_cast<uint32_t>(t.n_tile * 8 + part * kBlocks);   // first block column
          if (row_ok) {
            uint32_t codes[2 * kBlocks];
            uint32_t scales = 0;
#pragma unroll
            for (int blk = 0; blk < kBlocks; ++blk) {
              float h[16];
#pragma unroll
              for (int e = 0; e < 16; e += 2) {
                const uint32_t g2 = scale_round_bf16x2(alpha, g[16 * blk + e], g[16 * blk + e + 1]);
                const uint32_t u2 = scale_round_bf16x2(alpha_u, u[16 * blk + e], u[16 * blk + e + 1]);
                silu_mul_bf16_tab2(silu_tab, g2, bf16_lo(u2), bf16_hi(u2), h[e], h[e + 1]);
              }
              const QBlock qb = quantize16(h, gsf);
              codes[2 * blk] = qb.lo;
              codes[2 * blk + 1] = qb.hi;
              scales |= qb.s8 << (8 * blk);
            }
            uint4* dst = reinterpret_cast<uint4*>(q_row + part * (kCols / 2));
            uint8_t* sdst = sf_e + sf_offset(static_cast<uint32_t>(row), c0, groups);
            const bool in_range =
                index_ok(static_cast<uint64_t>(reinterpret_cast<uint8_t*>(dst) - p.q) + kCols / 2 - 1,
                         static_cast<uint64_t>(p.experts) * p.m * (p.n / 2), p.status) &&
                index_ok(static_cast<uint64_t>(sdst - p.sf) + kBlocks - 1,
                         static_cast<uint64_t>(p.experts) * p.sf_item_stride, p.status);
            if (!in_range) {
            } else if constexpr (kBlocks == 4) {
              dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
              dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
              *reinterpret_cast<uint32_t*>(sdst) = scales;
            } else {
              dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
              *reinterpret_cast<uint16_t*>(sdst) = static_cast<uint16_t>(scales);
            }
          } else if (pad_row) {
            uint8_t* sdst = sf_e + sf_offset(static_cast<uint32_t>(row), c0, groups);
            if (!index_ok(static_cast<uint64_t>(sdst - p.sf) + kBlocks - 1,
                          static_cast<uint64_t>(p.experts) * p.sf_item_stride, p.status)) {
            } else if constexpr (kBlocks == 4) {
              *reinterpret_cast<uint32_t*>(sdst) = 0u;
            } else {
              *reinterpret_cast<uint16_t*>(sdst) = 0;
            }
          }
        }
      } else {
        // This warp's 32-row slab of the tile goes out through its staging tile and a TMA
        // store (rows >= m and columns >= n are clipped by the tensor bounds).  A grouped
        // slab that crosses the expert's mask is stored row by row instead, so rows beyond
        // the mask stay untouched.
        const int slab_row = t.m_tile * kTileM + static_cast<int>(rank) * kBM + quarter * 32;
        const bool use_tma = kGrouped ? slab_row + 32 <= t.valid_rows : slab_row < p.m;
        constexpr int kBufs = kStagingBuffers<kGrouped, kSwiGLU, kQW>;
        uint8_t* stage_warp = staging + (warp - 2) * kBufs * kStoreTileBytes;
        __nv_bfloat16* out_row = p.out + (static_cast<int64_t>(t.expert) * p.m + row) * p.n;
        // The quarter's warps split the four 64-column subtiles in drain order: accumulator 0
        // drains its last 64 columns first, accumulator 1 its first 64 (the columns the next
        // tile's accumulator overlaps), and each warp releases the accumulator after its
        // first subtile.  A warp that never reads the overlap may release it at once; the
        // tile after next reuses this accumulator only after every warp has released the
        // next tile's, which it does after finishing this one.
        constexpr int kSubs = 4 / kQW;                          // subtiles per warp
        const int part = (warp - 2) >> 2;
        for (int j = 0; j < kSubs; ++j) {
          const int i = part * kSubs + j;
          const int sub = buf ? i : 3 - i;
          const int col_base = t.n_tile * kBN + sub * 64;
          uint4 bias8[8];                      // issued before the TMEM load to hide its latency
#pragma unroll
          for (int g = 0; g < 8; ++g)
            bias8[g] = (p.bias && col_base + 8 * g < p.n &&
                        index_ok(static_cast<uint64_t>(col_base + 8 * g + 7), static_cast<uint64_t>(p.n), p.status))
                           ? __ldg(reinterpret_cast<const uint4*>(p.bias + col_base + 8 * g))
                           : make_uint4(0u, 0u, 0u, 0u);
          uint32_t v[64];
          tmem_load_64(tmem + col0 + sub * 64 + lane_base, v);
          tmem_wait_ld<64>(v);
          if (j == 0) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
          }
          if (col_base >= p.n || !(use_tma || row_ok)) continue;
          uint4 o[8];
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const int col = col_base + 8 * g;
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * g + e]);
            if (p.bias && col < p.n) {
              const uint32_t bb[4] = {bias8[g].x, bias8[g].y, bias8[g].z, bias8[g].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                f[2 * e] = __fmaf_rn(alpha, f[2 * e], __uint_as_float(bb[e] << 16));
                f[2 * e + 1] = __fmaf_rn(alpha, f[2 * e + 1], __uint_as_float(bb[e] & 0xffff0000u));
              }
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e) f[e] = __fmul_rn(alpha, f[e]);
            }
            o[g].x = pack_bf16x2(f[0], f[1]);
            o[g].y = pack_bf16x2(f[2], f[3]);
            o[g].z = pack_bf16x2(f[4], f[5]);
            o[g].w = pack_bf16x2(f[6], f[7]);
          }
          if (use_tma) {
            uint8_t* stage_tile = stage_warp + (nstore % kBufs) * kStoreTileBytes;
            const uint32_t stage_row = smem_u32(stage_tile) + lane * 128;
            if (lane == 0) bulk_wait_read<kBufs - 1>();   // the store that last used this tile has read it
            __syncwarp();
            // 128-byte swizzle: 16-byte chunk g of row r sits at chunk position g ^ (r % 8)
#pragma unroll
            for (int g = 0; g < 8; ++g) st_shared_v4(stage_row + ((g ^ (lane & 7)) << 4), o[g]);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              if constexpr (kGrouped) {
                tma_store_3d(&maps.out, stage_tile, col_base, slab_row, t.expert);
              } else {
                tma_store_2d(&maps.out, stage_tile, col_base, slab_row);
              }
              bulk_commit();
            }
            ++nstore;
          } else {
#pragma unroll
            for (int g = 0; g < 8; ++g)
              if (col_base + 8 * g < p.n &&
                  index_ok(static_cast<uint64_t>(out_row + col_base + 8 * g - p.out) + 7,
                           static_cast<uint64_t>(p.experts) * p.m * p.n, p.status))
                *reinterpret_cast<uint4*>(out_row + col_base + 8 * g) = o[g];
          }
        }
      }
    }
    if constexpr (!kSwiGLU) {
      if (lane == 0) bulk_wait_all();         // this warp's TMA stores are complete
      __syncwarp();
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (*abort) {
    // Unwinding after a timed-out wait: give outstanding tensor-core and TMA operations a
    // bounded time to drain before the tensor memory and the CTA's smem are released.
    const uint64_t t0 = global_ns();
    while (global_ns() - t0 < 2000000ull) {
    }
  }
  cluster_sync();      // no CTA leaves while its peer may still signal its barriers
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
  if constexpr (kQuantA) {
    // the last CTA to finish (every producer has read its counters, every unit is counted)
    // re-zeroes the workspace words for the next call on the stream
    if (threadIdx.x == 0) {
      __threadfence();
      if (atomicAdd(p.qa_ws, 1u) == gridDim.x - 1) {
        for (int c = 0; c < p.k_stages; ++c) atomicExch(p.qa_ws + 1 + c, 0u);
        atomicExch(p.qa_ws, 0u);
      }
    }
  }
}

// ---- host side ------------------------------------------------------------------------------------

int make_map(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t rank, const void* base, const uint64_t* dims,
             const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn encode = encode_tiled_fn();
  if (!encode) return NVFP4_ERR_CUDA;
  uint32_t elem_strides[3] = {1, 1, 1};
  CUresult r = encode(map, dtype, rank, const_cast<void*>(base), dims, strides_bytes, box, elem_strides,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_INVALID_ARGUMENT;
}

// Packed FP4 operand [experts, rows, k/2] as a tiled uint8 tensor with boxes of 128 bytes
// (one stage of K) by 128 rows, 128-byte swizzle.
int make_operand_map(CUtensorMap* map, const uint8_t* base, int64_t experts, int64_t rows, int64_t k, bool grouped) {
  const uint64_t dims[3] = {static_cast<uint64_t>(k / 2), static_cast<uint64_t>(rows), static_cast<uint64_t>(experts)};
  const uint64_t strides[2] = {static_cast<uint64_t>(k / 2), static_cast<uint64_t>(rows * (k / 2))};
  const uint32_t box[3] = {kStageBytesRow, 128, 1};
  return make_map(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, grouped ? 3 : 2, base, dims, strides, box,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

// Scale buffer [experts][nvfp4_scale_bytes(rows, k)] viewed as rows of 128 bytes; a box
// of 16 rows is 4 consecutive 512-byte chunks (one stage of K for one 128-row tile).
int make_scale_map(CUtensorMap* map, const uint8_t* base, int64_t experts, int64_t rows, int64_t k, bool grouped) {
  const int64_t bytes = nvfp4_scale_bytes(rows, k);
  const uint64_t dims[3] = {128, static_cast<uint64_t>(bytes / 128), static_cast<uint64_t>(experts)};
  const uint64_t strides[2] = {128, static_cast<uint64_t>(bytes)};
  const uint32_t box[3] = {128, 16, 1};
  return make_map(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, grouped ? 3 : 2, base, dims, strides, box,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
}

// bf16 output [experts, rows, n] with boxes of 64 columns (128 bytes) by 32 rows, 128-byte
// swizzle (the epilogue's staging layout).
int make_output_map(CUtensorMap* map, const void* base, int64_t experts, int64_t rows, int64_t n, bool grouped) {
  const uint64_t dims[3] = {static_cast<uint64_t>(n), static_cast<uint64_t>(rows), static_cast<uint64_t>(experts)};
  const uint64_t strides[2] = {static_cast<uint64_t>(n * 2), static_cast<uint64_t>(rows * n * 2)};
  const uint32_t box[3] = {64, 32, 1};
  return make_map(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, grouped ? 3 : 2, base, dims, strides, box,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

// bf16 low-rank operand [rows, r] with boxes of 64 values (128 bytes) by 128 rows.
int make_lowrank_map(CUtensorMap* map, const void* base, int64_t rows, int64_t r) {
  const uint64_t dims[2] = {static_cast<uint64_t>(r), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(r * 2)};
  const uint32_t box[2] = {64, 128};
  return make_map(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Operands of one call; unused members are null / zero.
struct GemmArgs {
  const uint8_t *a = nullptr, *b = nullptr, *a_sf = nullptr, *b_sf = nullptr;
  const float* alpha = nullptr;
  const void *d = nullptr, *l1 = nullptr;  // low-rank
  int64_t r = 0;
  const void* bias = nullptr;
  const int32_t* mask = nullptr;           // grouped
  void* out = nullptr;                     // bf16 output
  const uint8_t *b2 = nullptr, *b2_sf = nullptr;  // SiLU * up: up weight (b: gate weight)
  const float *alpha2 = nullptr, *gsf_h = nullptr;
  uint8_t *q = nullptr, *sf = nullptr;
  const void* qa_x = nullptr;              // fused activation quantizer: bf16 x (a, a_sf: its workspace)
  const float* qa_gsf = nullptr;
  int64_t E = 1, m = 0, n = 0, k = 0;      // n: output width (the width of h for SiLU * up)
  int32_t stall_stage = -1;                // self-test only
};

// Launches the kernel instantiation with kQW epilogue warps per lane quarter: the one-time
// set-up per instantiation and device (dynamic shared memory opt-in, the number of 2-CTA
// clusters that fit on the device at once: the persistent grid size), then a grid of
// min(tiles, clusters) pairs.
template <bool kGrouped, bool kLowRank, bool kSwiGLU, int kQW, bool kQuantA = false>
int run_gemm(const Maps& maps, const GemmParams& p, int64_t tiles, const DeviceInfo& info, cudaStream_t stream) {
  auto kernel = nvfp4_gemm_kernel<kGrouped, kLowRank, kSwiGLU, kQW, kQuantA>;
  constexpr int kSmem = kSmemBytes<kGrouped, kSwiGLU, kQW, kQuantA>;
  int max_clusters = 0;
  const int st = kernel_setup(reinterpret_cast<const void*>(kernel), info.device, [&](int* clusters_out) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess) {
      cudaGetLastError();
      return static_cast<int>(NVFP4_ERR_CUDA);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(info.sm_count / 2 * 2);
    cfg.blockDim = dim3(kThreads<kQW>);
    cfg.dynamicSmemBytes = kSmem;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg) != cudaSuccess || clusters <= 0) {
      cudaGetLastError();
      clusters = info.sm_count / 2;
    }
    *clusters_out = clusters;
    return static_cast<int>(NVFP4_OK);
  }, &max_clusters);
  if (st != NVFP4_OK) return st;
  const int64_t max_pairs = max_clusters;
  const int pairs = static_cast<int>(tiles < max_pairs ? tiles : max_pairs);
  return launch_kernel(kernel, dim3(2 * pairs), dim3(kThreads<kQW>), kSmem, stream, maps, p);
}

template <bool kGrouped, bool kLowRank, bool kSwiGLU, bool kQuantA = false>
int launch_gemm(const GemmArgs& g, cudaStream_t stream) {
  const int64_t E = g.E, m = g.m, n = g.n, k = g.k;
  if (E < 0 || m < 0 || n < 0 || k <= 0 || k % 64 != 0 || n % 8 != 0) return NVFP4_ERR_INVALID_ARGUMENT;
  if (kSwiGLU && n % 128 != 0) return NVFP4_ERR_INVALID_ARGUMENT;
  if (m > (1 << 30) || n > (1 << 29) || k > (1 << 30) || E > kMaxExperts) return NVFP4_ERR_INVALID_ARGUMENT;
  if (kLowRank && (g.r <= 0 || g.r % 32 != 0 || g.r > 256)) return NVFP4_ERR_INVALID_ARGUMENT;
  if (E == 0 || m == 0 || n == 0) return NVFP4_OK;
  if (!g.a || !g.b || !g.a_sf || !g.b_sf || !g.alpha) return NVFP4_ERR_INVALID_ARGUMENT;
  if (!aligned(g.a, 16) || !aligned(g.b, 16) || !aligned(g.a_sf, 16) || !aligned(g.b_sf, 16) || !aligned(g.alpha, 4))
    return NVFP4_ERR_INVALID_ARGUMENT;
  if (kSwiGLU) {
    if (!g.b2 || !g.b2_sf || !g.alpha2 || !g.q || !g.sf || !g.gsf_h) return NVFP4_ERR_INVALID_ARGUMENT;
    if (!aligned(g.b2, 16) || !aligned(g.b2_sf, 16) || !aligned(g.alpha2, 4) || !aligned(g.q, 16) ||
        !aligned(g.sf, 16) || !aligned(g.gsf_h, 4))
      return NVFP4_ERR_INVALID_ARGUMENT;
  } else {
    if (!g.out || !aligned(g.out, 16) || (g.bias && !aligned(g.bias, 16))) return NVFP4_ERR_INVALID_ARGUMENT;
  }
  if (kGrouped && (!g.mask || !aligned(g.mask, 4))) return NVFP4_ERR_INVALID_ARGUMENT;
  if (kLowRank && (!g.d || !g.l1 || !aligned(g.d, 16) || !aligned(g.l1, 16))) return NVFP4_ERR_INVALID_ARGUMENT;
  if (kQuantA && (!g.qa_x || !g.qa_gsf || !aligned(g.qa_x, 16) || !aligned(g.qa_gsf, 4) ||
                  (k + kStageK - 1) / kStageK > kQuantAMaxChunks))
    return NVFP4_ERR_INVALID_ARGUMENT;

  DeviceInfo info;
  int st = current_device(&info);
  if (st != NVFP4_OK) return st;

  Maps maps;
  memset(&maps, 0, sizeof(maps));
  if ((st = make_operand_map(&maps.a, g.a, E, m, k, kGrouped)) != NVFP4_OK) return st;
  if ((st = make_operand_map(&maps.b, g.b, E, n, k, kGrouped)) != NVFP4_OK) return st;
  if ((st = make_scale_map(&maps.sfa, g.a_sf, E, m, k, kGrouped)) != NVFP4_OK) return st;
  if ((st = make_scale_map(&maps.sfb, g.b_sf, E, n, k, kGrouped)) != NVFP4_OK) return st;
  if (kSwiGLU) {
    if ((st = make_operand_map(&maps.b2, g.b2, E, n, k, kGrouped)) != NVFP4_OK) return st;
    if ((st = make_scale_map(&maps.sfb2, g.b2_sf, E, n, k, kGrouped)) != NVFP4_OK) return st;
  } else {
    if ((st = make_output_map(&maps.out, g.out, E, m, n, kGrouped)) != NVFP4_OK) return st;
  }
  if (kLowRank) {
    if ((st = make_lowrank_map(&maps.d, g.d, m, g.r)) != NVFP4_OK) return st;
    if ((st = make_lowrank_map(&maps.l1, g.l1, n, g.r)) != NVFP4_OK) return st;
  }

  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.alpha = g.alpha;
  p.bias = static_cast<const __nv_bfloat16*>(g.bias);
  p.out = static_cast<__nv_bfloat16*>(g.out);
  p.mask = g.mask;
  p.status = info.status;
  p.silu_tab = info.silu_table;
  p.m = static_cast<int32_t>(m);
  p.n = static_cast<int32_t>(n);
  p.k = static_cast<int32_t>(k);
  p.experts = static_cast<int32_t>(E);
  p.rank = static_cast<int32_t>(g.r);
  p.n_tiles = static_cast<int32_t>(kSwiGLU ? n / kBNHalf : (n + kBN - 1) / kBN);
  p.m_tiles = static_cast<int32_t>((m + kTileM - 1) / kTileM);
  p.k_stages = static_cast<int32_t>((k + kStageK - 1) / kStageK);
  p.k_steps = static_cast<int32_t>(k / 64);
  p.sf_groups = static_cast<int32_t>(k / 64);
  p.stall_stage = g.stall_stage;
  uint32_t* qa_ws = nullptr;
  if (kQuantA) {
    if ((st = stream_workspace(stream, &qa_ws)) != NVFP4_OK) return st;
    p.qa_x = static_cast<const uint16_t*>(g.qa_x);
    p.qa_gsf = g.qa_gsf;
    p.qa_q = const_cast<uint8_t*>(g.a);
    p.qa_sf = const_cast<uint8_t*>(g.a_sf);
    p.qa_ws = qa_ws;
    p.qa_slabs = static_cast<int32_t>((m + 127) / 128);
  }
  if (kSwiGLU) {
    p.alpha_up = g.alpha2;
    p.gsf_h = g.gsf_h;
    p.q = g.q;
    p.sf = g.sf;
    p.sf_item_stride = nvfp4_scale_bytes(m, n);
    p.rows_pad = static_cast<int32_t>((m + 127) / 128 * 128);
  }

  const int64_t tiles = kGrouped ? static_cast<int64_t>(E) * p.m_tiles * p.n_tiles
                                 : static_cast<int64_t>(p.m_tiles) * p.n_tiles;
  if (tiles >= (int64_t(1) << 31)) return NVFP4_ERR_INVALID_ARGUMENT;
  if constexpr (kQuantA) {
    if (k >= 4096 && tiles >= static_cast<int64_t>(info.sm_count))
      return run_gemm<false, false, false, 1, true>(maps, p, tiles, info, stream);
    return run_gemm<false, false, false, 2, true>(maps, p, tiles, info, stream);
  } else if constexpr (kSwiGLU) {
    return run_gemm<kGrouped, kLowRank, kSwiGLU, 2>(maps, p, tiles, info, stream);
  } else if constexpr (kGrouped) {
    return run_gemm<kGrouped, kLowRank, kSwiGLU, 1>(maps, p, tiles, info, stream);
  } else {
    // one epilogue warp per lane quarter when the K loop hides the epilogue and there are
    // at least two waves of tiles; two otherwise (see kEpiWarps)
    if (k >= 4096 && tiles >= static_cast<int64_t>(info.sm_count))
      return run_gemm<kGrouped, kLowRank, kSwiGLU, 1>(maps, p, tiles, info, stream);
    return run_gemm<kGrouped, kLowRank, kSwiGLU, 2>(maps, p, tiles, info, stream);
  }
}

// Self-test of the bounded wait: one thread waits for an mbarrier phase that nothing ever
// completes; the wait gives up after its limit and records NVFP4_ERR_DEVICE_TIMEOUT.
__global__ void bounded_wait_selftest_kernel(int* status) {
  __shared__ uint64_t bar;
  __shared__ int32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, status);
}

}  // namespace

int gemm_quantize_a(const void* a_bf16, const uint8_t* b, const uint8_t* b_sf, const float* a_gsf, const float* alpha,
                    const void* bias_bf16, void* out_bf16, uint8_t* a_q_ws, uint8_t* a_sf_ws, int64_t m, int64_t n,
                    int64_t k, cudaStream_t stream) {
  GemmArgs g;
  g.a = a_q_ws; g.b = b; g.a_sf = a_sf_ws; g.b_sf = b_sf; g.alpha = alpha; g.bias = bias_bf16; g.out = out_bf16;
  g.qa_x = a_bf16; g.qa_gsf = a_gsf;
  g.m = m; g.n = n; g.k = k;
  return launch_gemm<false, false, false, true>(g, stream);
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

int nvfp4_gemm(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, const uint8_t* b_sf, const float* alpha,
               const void* bias_bf16, void* out_bf16, int64_t m, int64_t n, int64_t k, nvfp4_stream_t stream) {
  GemmArgs g;
  g.a = a; g.b = b; g.a_sf = a_sf; g.b_sf = b_sf; g.alpha = alpha; g.bias = bias_bf16; g.out = out_bf16;
  g.m = m; g.n = n; g.k = k;
  return launch_gemm<false, false, false>(g, stream);
}

int nvfp4_grouped_gemm_masked(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, const uint8_t* b_sf,
                              const int32_t* mask, const float* alpha, void* out_bf16, int64_t E, int64_t mmax,
                              int64_t n, int64_t k, nvfp4_stream_t stream) {
  GemmArgs g;
  g.a = a; g.b = b; g.a_sf = a_sf; g.b_sf = b_sf; g.alpha = alpha; g.mask = mask; g.out = out_bf16;
  g.E = E; g.m = mmax; g.n = n; g.k = k;
  return launch_gemm<true, false, false>(g, stream);
}

int nvfp4_gemm_lowrank_bias(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, const uint8_t* b_sf,
                            const float* alpha, const void* d_bf16, const void* l1_bf16, int64_t r,
                            const void* bias_bf16, void* out_bf16, int64_t m, int64_t n, int64_t k,
                            nvfp4_stream_t stream) {
  GemmArgs g;
  g.a = a; g.b = b; g.a_sf = a_sf; g.b_sf = b_sf; g.alpha = alpha; g.d = d_bf16; g.l1 = l1_bf16; g.r = r;
  g.bias = bias_bf16; g.out = out_bf16;
  g.m = m; g.n = n; g.k = k;
  return launch_gemm<false, true, false>(g, stream);
}

int nvfp4_gemm_silu_mul_quantize(const uint8_t* a, const uint8_t* b_gate, const uint8_t* b_up, const uint8_t* a_sf,
                                 const uint8_t* b_gate_sf, const uint8_t* b_up_sf, const float* alpha_gate,
                                 const float* alpha_up, const float* gsf_h, uint8_t* q_out, uint8_t* sf_out,
                                 int64_t m, int64_t n, int64_t k, nvfp4_stream_t stream) {
  GemmArgs g;
  g.a = a; g.b = b_gate; g.b2 = b_up; g.a_sf = a_sf; g.b_sf = b_gate_sf; g.b2_sf = b_up_sf;
  g.alpha = alpha_gate; g.alpha2 = alpha_up; g.gsf_h = gsf_h; g.q = q_out; g.sf = sf_out;
  g.m = m; g.n = n; g.k = k;
  return launch_gemm<false, false, true>(g, stream);
}

int nvfp4_grouped_gemm_silu_mul_quantize_masked(const uint8_t* a, const uint8_t* b_gate, const uint8_t* b_up,
                                                const uint8_t* a_sf, const uint8_t* b_gate_sf,
                                                const uint8_t* b_up_sf, const int32_t* mask,
                                                const float* alpha_gate, const float* alpha_up,
                                                const float* gsf_h, uint8_t* q_out, uint8_t* sf_out, int64_t E,
                                                int64_t mmax, int64_t n, int64_t k, nvfp4_stream_t stream) {
  GemmArgs g;
  g.a = a; g.b = b_gate; g.b2 = b_up; g.a_sf = a_sf; g.b_sf = b_gate_sf; g.b2_sf = b_up_sf; g.mask = mask;
  g.alpha = alpha_gate; g.alpha2 = alpha_up; g.gsf_h = gsf_h; g.q = q_out; g.sf = sf_out;
  g.E = E; g.m = mmax; g.n = n; g.k = k;
  return launch_gemm<true, false, true>(g, stream);
}

int nvfp4_selftest_bounded_wait(nvfp4_stream_t stream) {
  DeviceInfo info;
  int st = current_device(&info);
  if (st != NVFP4_OK) return st;
  return launch_kernel(bounded_wait_selftest_kernel, dim3(1), dim3(32), 0, stream, info.status);
}

int nvfp4_selftest_gemm_stall(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, const uint8_t* b_sf,
                              const float* alpha, void* out_bf16, int64_t m, int64_t n, int64_t k,
                              nvfp4_stream_t stream) {
  GemmArgs g;
  g.a = a; g.b = b; g.a_sf = a_sf; g.b_sf = b_sf; g.alpha = alpha; g.out = out_bf16;
  g.m = m; g.n = n; g.k = k;
  g.stall_stage = 0;
  return launch_gemm<false, false, false>(g, stream);
}

}  // extern "C"
