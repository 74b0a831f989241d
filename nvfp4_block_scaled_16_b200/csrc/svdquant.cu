// svdquant.cu -- the input stage of an SVDQuant NVFP4 linear layer on tcgen05.
//
//   nvfp4_lora_down                   d = bf16(x @ w^T), fp32 accumulation
//   nvfp4_quantize_smooth_lora_down   the same d, and the NVFP4 quantization of
//                                     x_hat = bf16(x * pre_quant_scale), in one pass over x
//
// Sources (page title, section): flashinfer docs mm_nvfp4_svdquant, Parameters a and d:
// the GEMM's activation operand is x quantized with the SVDQuant pre-quantization scale
// folded in (nvfp4_quantize_smooth), and its rank-r operand d is the LoRA-down product of x
// with the pre-quantization-scaled down projection, w = (pre_quant_scale[:, None] * L2^T)^T
// ([r, k], prepared offline), computed in bf16.  TensorRT-LLM NVFP4LinearMethod.create_weights
// carries the same pre_quant_scale for o_proj / down_proj style layers.
//
// Kernel structure.  A cluster of kSvdSplit CTAs shares one 128-row tile of x and splits its
// K range; every CTA streams its 128 x (k/kSvdSplit) slice of x (and the matching columns of w)
// through a 4-stage ring of 64-column TMA tiles (128-byte swizzle).
//   warp 0      TMA producer (one elected lane).
//   warp 1      TMEM allocator and MMA issuer: per stage four tcgen05.mma.cta_group::1
//               kind::f16 (bf16 x bf16 -> fp32, M = 128, N = r, K = 16) into a 128 x r fp32
//               accumulator in tensor memory.
//   warps 2-9   quantizer (fused op only): a thread owns one row of the tile and half of the
//               stage's 4 blocks (two warps per 32 rows); per stage it reads its 32 values
//               from the swizzled tile, forms x_hat, and writes 2 blocks: 16 code bytes and
//               two scale bytes (a stage is exactly one 4-block group of the 128x4 scale
//               layout).  Afterwards warps 2-5 drain the accumulator into shared memory
//               (column-major fp32) and, after a cluster barrier, CTA c sums its share of
//               the tile's rows over the cluster's partials through distributed shared
//               memory and writes them as bf16.
// Every mbarrier wait is bounded; the two cluster barriers are executed on every path.
#include <cuda_bf16.h>

#include "common.cuh"
#include "nvfp4_math.cuh"
#include "tc_common.cuh"

namespace nvfp4 {
namespace {

constexpr int kSvdRows = 128;            // rows of x per cluster (MMA M)
constexpr int kSvdChunk = 64;            // bf16 values of K per stage (128-byte rows)
constexpr int kSvdMinStages = 4;
constexpr int kSvdMaxStages = 8;         // the ring takes as many stages as fit (r = 64: 8)
constexpr bool kSvdInterleave = true;    // CTA c of a cluster takes K chunks c, c + split, ...
constexpr int kSvdSplit = 4;             // CTAs per cluster, splitting K
static_assert(kSvdSplit == 4 || kSvdSplit == 8, "the reduction splits 128 threads over 128 / kSvdSplit rows");
constexpr int kSvdXBytes = kSvdRows * 128;   // 16 KB per stage
constexpr int kSvdMaxRank = 256;
// Quantizer warps: 16 / kSvdQuantWarps of a row's 4 blocks per stage per thread; the first
// four of them also drain and reduce the accumulator.
constexpr int kSvdQuantWarps = 8;
constexpr int kSvdBlocksPerThread = 16 / kSvdQuantWarps;
constexpr int kSvdThreads = 64 + 32 * kSvdQuantWarps;
static_assert(kSvdQuantWarps == 4 || kSvdQuantWarps == 8 || kSvdQuantWarps == 16, "1, 2 or 4 blocks per thread");

struct __align__(8) SvdControl {
  uint64_t full[kSvdMaxStages];
  uint64_t empty[kSvdMaxStages];
  uint64_t acc_full;
  uint32_t tmem_base;
  int32_t abort;
};

__host__ __device__ constexpr int svd_stage_bytes(int r) { return kSvdXBytes + r * 128; }
// The stage's 64 pre-quantization scales (128 bytes) travel with it in a small ring of their
// own after the main one (the main ring's tiles stay 1024-byte aligned).
constexpr int kSvdPqsBytes = kSvdChunk * 2;
// dynamic shared memory available to the ring (227 KB less the static inverse-scale table,
// the pre-quantization-scale ring, the control block and the alignment slack)
constexpr int kSvdRingBudget =
    227 * 1024 - 512 - kSvdMaxStages * kSvdPqsBytes - static_cast<int>(sizeof(SvdControl)) - 1024;
__host__ __device__ constexpr int svd_stages(int r) {
  return kSvdRingBudget / svd_stage_bytes(r) < kSvdMaxStages ? kSvdRingBudget / svd_stage_bytes(r) : kSvdMaxStages;
}
__host__ __device__ constexpr int svd_smem_bytes(int r) {
  return svd_stages(r) * svd_stage_bytes(r) + kSvdMaxStages * kSvdPqsBytes + static_cast<int>(sizeof(SvdControl)) +
         1024;
}
static_assert(svd_stages(kSvdMaxRank) >= kSvdMinStages, "the ring needs at least four stages");
static_assert(svd_smem_bytes(32) <= 227 * 1024 - 512 && svd_smem_bytes(kSvdMaxRank) <= 227 * 1024 - 512,
              "shared memory layout exceeds the per-block limit");
// the fp32 partial accumulator (128 x r) reuses the stage ring after the K loop
static_assert(kSvdRows * kSvdMaxRank * 4 <= svd_stages(kSvdMaxRank) * svd_stage_bytes(kSvdMaxRank), "partials do not fit");
static_assert(kSvdRows * 32 * 4 <= svd_stages(32) * svd_stage_bytes(32), "partials do not fit");

struct SvdParams {
  const uint16_t* pqs;      // [k] bf16 pre-quantization scale (fused op)
  const float* gsf;         // [1] global scale of x_hat (fused op)
  uint8_t* q;               // [m, k/2]
  uint8_t* sf;              // [nvfp4_scale_bytes(m, k)]
  __nv_bfloat16* d;         // [m, r]
  int* status;
  int32_t m, k, r;
  int32_t rows_pad;         // pad_up(m, 128)
  int32_t chunks;           // k / 64
};

struct SvdMaps {
  CUtensorMap x, w;
};

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) from global memory
// into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load_cta(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Tiled TMA load into this CTA's shared memory (plain, single-CTA form).
__device__ __forceinline__ void tma_load_2d_cta(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void mma_bf16_cta(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit_cta(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_local(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// 16 bytes of row `row` of a 128-byte-swizzled tile: chunk c sits at position c ^ (row % 8).
__device__ __forceinline__ uint4 ld_swizzled_chunk(uint32_t tile, int row, int c) {
  uint4 v;
  const uint32_t addr = tile + row * 128 + ((c ^ (row & 7)) << 4);
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

template <bool kQuant>
__global__ void __cluster_dims__(kSvdSplit, 1, 1) __launch_bounds__(kSvdThreads, 1)
    svdquant_input_kernel(const __grid_constant__ SvdMaps maps, const SvdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stage_bytes = svd_stage_bytes(p.r);
  const int stages = svd_stages(p.r);
  uint8_t* pqs_ring = smem + stages * stage_bytes;
  SvdControl& ctl = *reinterpret_cast<SvdControl*>(pqs_ring + kSvdMaxStages * kSvdPqsBytes);
  volatile int32_t* abort = &ctl.abort;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int row0 = blockIdx.y * kSvdRows;
  // this CTA's share of the K chunks
  // this CTA's K chunks: interleaved (c, c + split, ...), so that the cluster's CTAs read
  // adjacent 128-byte pieces of the same rows at the same time; or one contiguous range
  const int per = (p.chunks + kSvdSplit - 1) / kSvdSplit;
  const int c_begin = kSvdInterleave ? static_cast<int>(rank) : min(static_cast<int>(rank) * per, p.chunks);
  const int c_step = kSvdInterleave ? kSvdSplit : 1;
  const int nch = kSvdInterleave ? (p.chunks - static_cast<int>(rank) + kSvdSplit - 1) / kSvdSplit
                                 : min(c_begin + per, p.chunks) - c_begin;
  // the accumulator is drained 64 columns at a time, so at least 64 columns are allocated
  const uint32_t tmem_cols = p.r <= 64 ? 64u : (p.r <= 128 ? 128u : 256u);

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.empty[s], kQuant ? 1 + kSvdQuantWarps : 1);   // the MMA commit (+ the quantizer warps)
    }
    mbar_init(&ctl.acc_full, 1);
    ctl.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&ctl.tmem_base)),
                 "r"(tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;
  pdl_launch_dependents();
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (elect_one()) {
      prefetch_map(&maps.x);
      prefetch_map(&maps.w);
    }
    __syncwarp();
    const uint32_t tx = static_cast<uint32_t>(stage_bytes + (kQuant ? kSvdPqsBytes : 0));
    for (int i = 0; i < nch; ++i) {
      const int s = i % stages;
      if (i >= stages && !mbar_wait_fast(&ctl.empty[s], ((i / stages) - 1) & 1, abort, p.status)) break;
      uint8_t* st = smem + s * stage_bytes;
      if (elect_one()) {
        mbar_arrive_expect_tx(&ctl.full[s], tx);
        tma_load_2d_cta(st, &maps.x, &ctl.full[s], (c_begin + i * c_step) * kSvdChunk, row0);
        tma_load_2d_cta(st + kSvdXBytes, &maps.w, &ctl.full[s], (c_begin + i * c_step) * kSvdChunk, 0);
        if constexpr (kQuant)
          bulk_load_cta(pqs_ring + s * kSvdPqsBytes, p.pqs + (c_begin + i * c_step) * kSvdChunk, kSvdPqsBytes,
                        &ctl.full[s]);
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(p.r >> 3) << 17) |
                           (static_cast<uint32_t>(kSvdRows >> 4) << 24);
    const uint64_t a0 = operand_desc(smem_u32(smem));
    const uint64_t b0 = operand_desc(smem_u32(smem + kSvdXBytes));
    bool ok = true;
    for (int i = 0; i < nch; ++i) {
      const int s = i % stages;
      if (!(ok = mbar_wait_fast(&ctl.full[s], (i / stages) & 1, abort, p.status))) break;
      tc_fence_after();
      const uint64_t off = static_cast<uint64_t>(s * stage_bytes) >> 4;
      if (elect_one()) {
#pragma unroll
        for (int j = 0; j < 4; ++j) mma_bf16_cta(tmem, a0 + off + 2 * j, b0 + off + 2 * j, idesc, (i > 0 || j > 0) ? 1u : 0u);
        mma_commit_cta(&ctl.empty[s]);
      }
      __syncwarp();
    }
    if (ok && nch > 0 && elect_one()) mma_commit_cta(&ctl.acc_full);
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ quantizer + epilogue
    const int qw = warp - 2;
    const int row = (qw & 3) * 32 + lane;           // row of the tile; also its TMEM lane
    const int part = qw >> 2;                       // which blocks of the stage this thread takes
    const int grow = row0 + row;
    bool ok = true;
    if constexpr (kQuant) {
      const float gsf = __ldg(p.gsf);
      // inverse block scales of the 128 scale codes, one division each
      __shared__ float inv_tab[128];
      if (threadIdx.x - 64 < 128) inv_tab[threadIdx.x - 64] = inv_scale(threadIdx.x - 64, gsf);
      asm volatile("bar.sync 2, %0;" ::"n"(32 * kSvdQuantWarps) : "memory");
      const uint32_t groups = static_cast<uint32_t>(p.chunks);     // k / 64 scale groups per row
      for (int i = 0; i < nch; ++i) {
        const int s = i % stages;
        const int kc = (c_begin + i * c_step) * kSvdChunk;
        const int b0 = part * kSvdBlocksPerThread;   // first block (of 4) of this thread
        if (!(ok = mbar_wait_fast(&ctl.full[s], (i / stages) & 1, abort, p.status))) break;
        uint4 sc_raw[2 * kSvdBlocksPerThread];      // its pre-quantization scales (arrived with the stage)
#pragma unroll
        for (int c = 0; c < 2 * kSvdBlocksPerThread; ++c)
          sc_raw[c] = reinterpret_cast<const uint4*>(pqs_ring + s * kSvdPqsBytes)[2 * b0 + c];
        const uint32_t tile = smem_u32(smem + s * stage_bytes);
        const uint32_t sf_word = static_cast<uint32_t>(
            sf_offset(static_cast<uint32_t>(grow), static_cast<uint32_t>(kc / 16 + b0), groups));
        if (grow < p.m) {
          uint32_t codes[2 * kSvdBlocksPerThread];
          uint32_t scales = 0;
#pragma unroll
          for (int blk = 0; blk < kSvdBlocksPerThread; ++blk) {
            float v[16];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int c = 2 * (b0 + blk) + h;       // 16-byte chunk of the 128-byte row
              const uint4 xr = ld_swizzled_chunk(tile, row, c);
              const uint4 sr = sc_raw[2 * blk + h];
              const uint32_t xw[4] = {xr.x, xr.y, xr.z, xr.w};
              const uint32_t sw[4] = {sr.x, sr.y, sr.z, sr.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                float a, b;
                unpack2(mul2(pack2(bf16_lo(xw[e]), bf16_hi(xw[e])), pack2(bf16_lo(sw[e]), bf16_hi(sw[e]))), a, b);
                uint32_t w;
                asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(b), "f"(a));   // a -> low half
                v[8 * h + 2 * e] = bf16_lo(w);
                v[8 * h + 2 * e + 1] = bf16_hi(w);
              }
            }
            const QBlock qb = quantize16(v, gsf, inv_tab);
            codes[2 * blk] = qb.lo;
            codes[2 * blk + 1] = qb.hi;
            scales |= qb.s8 << (8 * blk);
          }
          uint8_t* qdst = p.q + static_cast<int64_t>(grow) * (p.k / 2) + kc / 2 + 8 * b0;
          const bool in_range =
              index_ok(static_cast<uint64_t>(qdst - p.q) + 8 * kSvdBlocksPerThread - 1,
                       static_cast<uint64_t>(p.m) * (p.k / 2), p.status) &&
              index_ok(sf_word + kSvdBlocksPerThread - 1, static_cast<uint64_t>(p.rows_pad) * (p.k / 16), p.status);
          if (!in_range) {
          } else if constexpr (kSvdBlocksPerThread == 4) {
            reinterpret_cast<uint4*>(qdst)[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
            reinterpret_cast<uint4*>(qdst)[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
            *reinterpret_cast<uint32_t*>(p.sf + sf_word) = scales;
          } else if constexpr (kSvdBlocksPerThread == 2) {
            *reinterpret_cast<uint4*>(qdst) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
            *reinterpret_cast<uint16_t*>(p.sf + sf_word) = static_cast<uint16_t>(scales);
          } else {
            *reinterpret_cast<uint2*>(qdst) = make_uint2(codes[0], codes[1]);
            p.sf[sf_word] = static_cast<uint8_t>(scales);
          }
        } else if (grow < p.rows_pad) {
          if (!index_ok(sf_word + kSvdBlocksPerThread - 1, static_cast<uint64_t>(p.rows_pad) * (p.k / 16), p.status)) {
          } else if constexpr (kSvdBlocksPerThread == 4) {
            *reinterpret_cast<uint32_t*>(p.sf + sf_word) = 0u;
          } else if constexpr (kSvdBlocksPerThread == 2) {
            *reinterpret_cast<uint16_t*>(p.sf + sf_word) = 0;
          } else {
            p.sf[sf_word] = 0;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_local(&ctl.empty[s]);
      }
    }
    // The partials overwrite the stage ring: every quantizer warp must be done reading it
    // (a warp whose rows all lie beyond m has no quantizing work and would get here first).
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kSvdQuantWarps) : "memory");
    // warps 2-5 drain this CTA's partial accumulator into shared memory, column-major:
    // part[col][row]
    if (qw < 4) {
      float* partial = reinterpret_cast<float*>(smem);
      const int tmem_row = (warp & 3) * 32 + lane;   // TMEM lane quarter of this warp
      if (ok && nch > 0 && mbar_wait(&ctl.acc_full, 0, abort, p.status)) {
        tc_fence_after();
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        for (int c0 = 0; c0 < p.r; c0 += 64) {
          uint32_t v[64];
          tmem_load_64(tmem + c0 + lane_base, v);
          tmem_wait_ld<64>(v);
#pragma unroll
          for (int j = 0; j < 64; ++j)
            if (c0 + j < p.r) partial[(c0 + j) * kSvdRows + tmem_row] = __uint_as_float(v[j]);
        }
      } else {
        for (int j = 0; j < p.r; ++j) partial[j * kSvdRows + tmem_row] = 0.0f;
      }
    }
  }

  // ---------------------------------------------------------------- cluster reduction of d
  tc_fence_before();
  __syncwarp();
  __syncthreads();
  cluster_sync();          // every CTA's partials are in its shared memory
  if (warp >= 2 && warp < 6 && !*abort) {
    // CTA c reduces rows [c * kRows, (c + 1) * kRows) of the tile; the 128 threads of warps
    // 2-5 take one row and one of kGroups column ranges each
    constexpr int kRows = kSvdRows / kSvdSplit;
    constexpr int kGroups = 128 / kRows;
    const int t = threadIdx.x - 64;
    const int row = static_cast<int>(rank) * kRows + t % kRows;
    const int grow = row0 + row;
    const int cols = p.r / kGroups;                       // a multiple of 4 (r is a multiple of 32)
    const int col0 = (t / kRows) * cols;
    const float* part = reinterpret_cast<const float*>(smem);
    uint32_t peer[kSvdSplit];
#pragma unroll
    for (int q = 0; q < kSvdSplit; ++q) peer[q] = map_to_rank(part, static_cast<uint32_t>(q));
    if (grow < p.m) {
      __nv_bfloat16* drow = p.d + static_cast<int64_t>(grow) * p.r + col0;
      for (int j = 0; j < cols; j += 4) {
        if (!index_ok(static_cast<uint64_t>(drow + j - p.d) + 3, static_cast<uint64_t>(p.m) * p.r, p.status)) continue;
        float acc[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t off = static_cast<uint32_t>(((col0 + j + e) * kSvdRows + row) * 4);
          float sum = 0.0f;
#pragma unroll
          for (int q = 0; q < kSvdSplit; ++q) sum = __fadd_rn(sum, ld_shared_cluster_f32(peer[q] + off));
          acc[e] = sum;
        }
        *reinterpret_cast<uint2*>(drow + j) = make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]));
      }
    }
  }
  if (*abort) {
    const uint64_t t0 = global_ns();
    while (global_ns() - t0 < 2000000ull) {
    }
  }
  __syncwarp();
  cluster_sync();          // no CTA leaves while a peer may still read its shared memory
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tmem_cols) : "memory");
  }
}

int make_bf16_map(CUtensorMap* map, const void* base, int64_t rows, int64_t k, uint32_t box_rows) {
  EncodeTiledFn encode = encode_tiled_fn();
  if (!encode) return NVFP4_ERR_CUDA;
  const uint64_t dims[2] = {static_cast<uint64_t>(k), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(k * 2)};
  const uint32_t box[2] = {static_cast<uint32_t>(kSvdChunk), box_rows};
  const uint32_t elem_strides[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                      elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_INVALID_ARGUMENT;
}

template <bool kQuant>
int launch_svdquant(const void* x, int64_t m, int64_t k, const void* pqs, const float* gsf, const void* w, int64_t r,
                    uint8_t* q, uint8_t* sf, void* d, cudaStream_t stream) {
  if (m < 0 || k <= 0 || k % kSvdChunk != 0 || k > (1 << 30) || r < 32 || r > kSvdMaxRank || r % 32 != 0)
    return NVFP4_ERR_INVALID_ARGUMENT;
  if (m > static_cast<int64_t>(65535) * kSvdRows) return NVFP4_ERR_INVALID_ARGUMENT;
  if (m == 0) return NVFP4_OK;
  if (!x || !w || !d || !aligned(x, 16) || !aligned(w, 16) || !aligned(d, 16)) return NVFP4_ERR_INVALID_ARGUMENT;
  if (kQuant && (!pqs || !gsf || !q || !sf || !aligned(pqs, 16) || !aligned(gsf, 4) || !aligned(q, 16) ||
                 !aligned(sf, 16)))
    return NVFP4_ERR_INVALID_ARGUMENT;
  DeviceInfo info;
  int st = current_device(&info);
  if (st != NVFP4_OK) return st;
  SvdMaps maps;
  memset(&maps, 0, sizeof(maps));
  if ((st = make_bf16_map(&maps.x, x, m, k, kSvdRows)) != NVFP4_OK) return st;
  if ((st = make_bf16_map(&maps.w, w, r, k, static_cast<uint32_t>(r))) != NVFP4_OK) return st;
  SvdParams p;
  p.pqs = static_cast<const uint16_t*>(pqs);
  p.gsf = gsf;
  p.q = q;
  p.sf = sf;
  p.d = static_cast<__nv_bfloat16*>(d);
  p.status = info.status;
  p.m = static_cast<int32_t>(m);
  p.k = static_cast<int32_t>(k);
  p.r = static_cast<int32_t>(r);
  p.rows_pad = static_cast<int32_t>((m + 127) / 128 * 128);
  p.chunks = static_cast<int32_t>(k / kSvdChunk);
  auto kernel = svdquant_input_kernel<kQuant>;
  const int smem = svd_smem_bytes(static_cast<int>(r));
  constexpr int kOptIn = 227 * 1024 - 512;   // every ring size fits below this (static table: 512 B)
  static_assert(svd_smem_bytes(96) <= kOptIn && svd_smem_bytes(128) <= kOptIn, "ring larger than the opt-in");
  int configured = 0;      // the shared-memory opt-in is a per-device setting
  const int st_cfg = kernel_setup(reinterpret_cast<const void*>(kernel), info.device, [&](int* out) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kOptIn) != cudaSuccess) {
      cudaGetLastError();
      return static_cast<int>(NVFP4_ERR_CUDA);
    }
    *out = 1;
    return static_cast<int>(NVFP4_OK);
  }, &configured);
  if (st_cfg != NVFP4_OK) return st_cfg;
  if (smem > kOptIn) return NVFP4_ERR_INVALID_ARGUMENT;
  dim3 grid(kSvdSplit, static_cast<unsigned>((m + kSvdRows - 1) / kSvdRows));
  return launch_kernel(kernel, grid, dim3(kSvdThreads), static_cast<size_t>(smem), stream, maps, p);
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

int nvfp4_lora_down(const void* x_bf16, int64_t m, int64_t k, const void* w_bf16, int64_t r, void* d_bf16,
                    nvfp4_stream_t stream) {
  return launch_svdquant<false>(x_bf16, m, k, nullptr, nullptr, w_bf16, r, nullptr, nullptr, d_bf16, stream);
}

int nvfp4_quantize_smooth_lora_down(const void* x_bf16, int64_t m, int64_t k, const void* pre_quant_scale_bf16,
                                    const float* gsf, const void* w_bf16, int64_t r, uint8_t* q_out,
                                    uint8_t* sf_out, void* d_bf16, nvfp4_stream_t stream) {
  return launch_svdquant<true>(x_bf16, m, k, pre_quant_scale_bf16, gsf, w_bf16, r, q_out, sf_out, d_bf16, stream);
}

}  // extern "C"
