// gemm.cu -- block-scaled NVFP4 GEMMs on the 5th-generation tensor cores (tcgen05).
//
//   nvfp4_gemm                 out = bf16(alpha * a @ b^T [+ bias])
//   nvfp4_gemm_lowrank_bias    out = bf16(alpha * (a @ b^T + d @ l1^T) [+ bias])
//   nvfp4_grouped_gemm_masked  out[e, i] = bf16(alpha[e] * a[e, i] @ b[e]^T), i < mask[e]
//
// Sources (page title, section): flashinfer docs mm_nvfp4_svdquant (signature,
// Parameters: packed (m, k/2) and (n, k/2) operands, 128x4-swizzled ue4m3 scales,
// alpha device scalar, rank-r bf16 correction issued as a second MMA into the same
// accumulator after the FP4 K-loop, epilogue alpha*acc + bias); TensorRT-LLM
// NVFP4LinearMethod.create_weights (weight [out, in/2], alpha); flashinfer PR #1774
// "Masked batch nvfp4 quantization" (masked per-expert operands for the grouped GEMM).
//
// Kernel structure (one CTA per SM, persistent over output tiles of 128 x 256):
//   warp 0      TMA producer: 2-D/3-D tiled loads of the packed operands (128-byte
//               swizzle, one 128-byte K row = 256 FP4 values per stage) and 1-D bulk
//               copies of the scale chunks, which are contiguous 512-byte blocks in the
//               128x4 layout, into a 4-stage shared-memory ring.
//   warp 1      TMEM allocator + MMA issuer (one thread): moves the stage's scale chunks
//               to tensor memory with tcgen05.cp (32x128b, replicated to the 4 lane
//               quarters) and issues tcgen05.mma kind::mxf4nvf4 (K = 64, ue4m3 scales per
//               16 values) into an fp32 accumulator in TMEM; the low-rank term follows
//               as kind::f16 (bf16) MMAs into the same accumulator.
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (each warp owns its 32-lane TMEM
//               quarter = 32 rows), alpha * acc + bias, bf16 stores.
// Two accumulators of 256 columns share TMEM columns [192, 256): the epilogue drains that
// overlap first and releases the accumulator, so the next tile's MMAs overlap the rest of
// the epilogue.  Scale factors use columns [448, 496).
// Every mbarrier wait is bounded (about one second of global time); a wait that runs out
// records NVFP4_ERR_DEVICE_TIMEOUT in the device status word and the whole CTA unwinds
// without hanging the GPU.
#include <cuda_bf16.h>

#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int kBM = 128;                 // output tile rows (MMA M)
constexpr int kBN = 256;                 // output tile columns (MMA N)
constexpr int kStageK = 256;             // FP4 values of K per stage (128 bytes per row)
constexpr int kStageBytesRow = kStageK / 2;
constexpr int kStages = 4;
constexpr int kABytes = kBM * kStageBytesRow;     // 16 KB
constexpr int kBBytes = kBN * kStageBytesRow;     // 32 KB
constexpr int kSfaBytes = 4 * 512;                // 4 K-steps x one 512-byte chunk
constexpr int kSfbBytes = 2 * 4 * 512;            // two 128-row halves x 4 K-steps
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;  // 55296 = 54 KB
constexpr int kMaxExperts = 1024;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccOverlapCol = 192;          // accumulator 1 starts here
constexpr uint32_t kSfCol = 448;                  // SFA: +0..15, SFB: +16..47
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

// smem layout after the stage ring
struct __align__(8) Control {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint32_t tmem_base;
  int32_t abort;
  int32_t prefix[kMaxExperts + 1];   // grouped: prefix sums of tiles per expert
};
constexpr int kSmemBytes = kStages * kStageBytes + sizeof(Control) + 1024;

// Instruction descriptors (tcgen05 "instruction descriptor" bit fields).
//   kind::mxf4nvf4: A/B format E2M1 (1) at bits 7..9 / 10..12, both K-major, N>>3 at
//   bits 17..22, ue4m3 scale format (0) at bit 23, M>>4 at bits 24..28, scale ids 0.
constexpr uint32_t kIdescFp4 = (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
//   kind::f16: fp32 accumulator (1) at bits 4..5, A/B bf16 (1), K-major, N, M as above.
constexpr uint32_t kIdescBf16 =
    (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) | (uint32_t(kBM >> 4) << 24);

// ---- PTX wrappers ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase of `bar` with the given parity to complete.  Returns false
// (and makes every other role of the CTA give up too) when the CTA is aborting or the
// wait exceeded the limit; the latter is recorded in the device status word.
__device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int32_t* abort, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15u) == 0) {
      if (*abort) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        *abort = 1;
        atomicExch(status, NVFP4_ERR_DEVICE_TIMEOUT);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: start address, leading / stride byte offsets (>>4),
// the sm_100 descriptor version (1 at bit 46) and the swizzle mode at bits 61..63.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t swizzle) {
  return static_cast<uint64_t>((addr >> 4) & 0x3fffu) | (static_cast<uint64_t>((lbo >> 4) & 0x3fffu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3fffu) << 32) | (1ull << 46) |
         (static_cast<uint64_t>(swizzle) << 61);
}
// K-major operand tile with 128-byte rows and the 128-byte swizzle: 8-row groups 1 KB apart.
__device__ __forceinline__ uint64_t operand_desc(uint32_t addr) { return smem_desc(addr, 16, 1024, 2); }
// One 512-byte scale chunk as 32 rows x 16 bytes: 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t sf_desc(uint32_t addr) { return smem_desc(addr, 0, 128, 0); }

__device__ __forceinline__ void tc_copy_sf(uint32_t tmem_col_addr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(tmem_col_addr), "l"(desc) : "memory");
}

__device__ __forceinline__ void mma_fp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t sfa, uint32_t sfb,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(kIdescFp4), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(kIdescBf16), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 32 lanes x 64 consecutive fp32 columns: thread i of the warp gets lane (quarter*32 + i).
__device__ __forceinline__ void tmem_load_64(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31]),
        "=r"(v[32]), "=r"(v[33]), "=r"(v[34]), "=r"(v[35]), "=r"(v[36]), "=r"(v[37]), "=r"(v[38]), "=r"(v[39]),
        "=r"(v[40]), "=r"(v[41]), "=r"(v[42]), "=r"(v[43]), "=r"(v[44]), "=r"(v[45]), "=r"(v[46]), "=r"(v[47]),
        "=r"(v[48]), "=r"(v[49]), "=r"(v[50]), "=r"(v[51]), "=r"(v[52]), "=r"(v[53]), "=r"(v[54]), "=r"(v[55]),
        "=r"(v[56]), "=r"(v[57]), "=r"(v[58]), "=r"(v[59]), "=r"(v[60]), "=r"(v[61]), "=r"(v[62]), "=r"(v[63])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
  const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return a | (b << 16);
}

// ---- problem description ----------------------------------------------------------------------

struct GemmParams {
  const uint8_t* a_sf;     // expert 0
  const uint8_t* b_sf;
  int64_t a_sf_stride;     // bytes between experts
  int64_t b_sf_stride;
  const float* alpha;      // [1] or [E]
  const __nv_bfloat16* bias;  // nullable [n]
  __nv_bfloat16* out;      // [E, mmax, n] (E = 1 for dense)
  const int32_t* mask;     // grouped only
  int* status;
  int32_t m;               // rows per expert (mmax)
  int32_t n;
  int32_t k;
  int32_t experts;
  int32_t rank;            // low-rank r (0 = none)
  int32_t n_tiles;
  int32_t m_tiles;         // dense: ceil(m / 128)
  int32_t k_stages;        // ceil(k / 256)
  int32_t k_steps;         // k / 64
  int32_t sf_groups;       // ceil(k / 64): 512-byte chunks per 128-row tile
  int32_t sf_row_tiles_b;  // ceil(n / 128)
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

// ---- the kernel ---------------------------------------------------------------------------------

template <bool kGrouped, bool kLowRank>
__global__ void __launch_bounds__(kThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                      const __grid_constant__ CUtensorMap map_d, const __grid_constant__ CUtensorMap map_l1,
                      const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Control& ctl = *reinterpret_cast<Control*>(smem + kStages * kStageBytes);
  volatile int32_t* abort = &ctl.abort;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.empty[s], 1);
    }
    mbar_init(&ctl.acc_full, 1);
    mbar_init(&ctl.acc_empty, 4);
    ctl.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if constexpr (kGrouped) {
    if (threadIdx.x == 32) {
      int acc = 0;
      ctl.prefix[0] = 0;
      for (int e = 0; e < p.experts; ++e) {
        const int valid = min(max(p.mask[e], 0), p.m);
        acc += (valid + kBM - 1) / kBM * p.n_tiles;
        ctl.prefix[e + 1] = acc;
      }
    }
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&ctl.tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_map(&map_a);
      prefetch_map(&map_b);
      if constexpr (kLowRank) {
        prefetch_map(&map_d);
        prefetch_map(&map_l1);
      }
      const int lr_stages = kLowRank ? (p.rank + 63) / 64 : 0;
      uint32_t it = 0;
      bool ok = true;
      TileCoord t;
      for (int tile = blockIdx.x; ok && tile_coord<kGrouped>(p, ctl, tile, t); tile += gridDim.x) {
        const uint8_t* a_sf = p.a_sf + t.expert * p.a_sf_stride;
        const uint8_t* b_sf = p.b_sf + t.expert * p.b_sf_stride;
        for (int ks = 0; ks < p.k_stages + lr_stages; ++ks, ++it) {
          const uint32_t s = it % kStages, round = it / kStages;
          if (round > 0 && !(ok = mbar_wait(&ctl.empty[s], (round - 1) & 1, abort, p.status))) break;
          uint8_t* st = smem + s * kStageBytes;
          if (ks < p.k_stages) {
            const int nks = min(4, p.k_steps - 4 * ks);
            const int halves = min(2, p.sf_row_tiles_b - 2 * t.n_tile);
            mbar_arrive_expect_tx(&ctl.full[s], kABytes + kBBytes + nks * 512 * (1 + halves));
            if constexpr (kGrouped) {
              tma_load_3d(st, &map_a, &ctl.full[s], ks * kStageBytesRow, t.m_tile * kBM, t.expert);
              tma_load_3d(st + kABytes, &map_b, &ctl.full[s], ks * kStageBytesRow, t.n_tile * kBN, t.expert);
            } else {
              tma_load_2d(st, &map_a, &ctl.full[s], ks * kStageBytesRow, t.m_tile * kBM);
              tma_load_2d(st + kABytes, &map_b, &ctl.full[s], ks * kStageBytesRow, t.n_tile * kBN);
            }
            const int64_t chunk_a = static_cast<int64_t>(t.m_tile) * p.sf_groups + 4 * ks;
            bulk_load(st + kABytes + kBBytes, a_sf + chunk_a * 512, nks * 512, &ctl.full[s]);
            for (int h = 0; h < halves; ++h) {
              const int64_t chunk_b = static_cast<int64_t>(2 * t.n_tile + h) * p.sf_groups + 4 * ks;
              bulk_load(st + kABytes + kBBytes + kSfaBytes + h * 4 * 512, b_sf + chunk_b * 512, nks * 512,
                        &ctl.full[s]);
            }
          } else if constexpr (kLowRank) {
            const int c = ks - p.k_stages;
            mbar_arrive_expect_tx(&ctl.full[s], kABytes + kBBytes);
            tma_load_2d(st, &map_d, &ctl.full[s], c * 64, t.m_tile * kBM);
            tma_load_2d(st + kABytes, &map_l1, &ctl.full[s], c * 64, t.n_tile * kBN);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const int lr_stages = kLowRank ? (p.rank + 63) / 64 : 0;
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      TileCoord t;
      for (int tile = blockIdx.x; ok && tile_coord<kGrouped>(p, ctl, tile, t); tile += gridDim.x, ++tcount) {
        const uint32_t acc = tmem + ((tcount & 1) ? kAccOverlapCol : 0u);
        if (tcount > 0) {
          if (!(ok = mbar_wait(&ctl.acc_empty, (tcount - 1) & 1, abort, p.status))) break;
          tc_fence_after();
        }
        for (int ks = 0; ks < p.k_stages + lr_stages; ++ks, ++it) {
          const uint32_t s = it % kStages;
          if (!(ok = mbar_wait(&ctl.full[s], (it / kStages) & 1, abort, p.status))) break;
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * kStageBytes);
          if (ks < p.k_stages) {
            const int nks = min(4, p.k_steps - 4 * ks);
            const uint32_t sfa_s = st + kABytes + kBBytes;
            const uint32_t sfb_s = sfa_s + kSfaBytes;
            for (int j = 0; j < nks; ++j) {
              tc_copy_sf(tmem + kSfCol + 4 * j, sf_desc(sfa_s + 512 * j));
              tc_copy_sf(tmem + kSfCol + 16 + 8 * j, sf_desc(sfb_s + 512 * j));
              tc_copy_sf(tmem + kSfCol + 16 + 8 * j + 4, sf_desc(sfb_s + 4 * 512 + 512 * j));
            }
            for (int j = 0; j < nks; ++j) {
              mma_fp4(acc, operand_desc(st + 32 * j), operand_desc(st + kABytes + 32 * j), tmem + kSfCol + 4 * j,
                      tmem + kSfCol + 16 + 8 * j, (ks > 0 || j > 0) ? 1u : 0u);
            }
          } else if constexpr (kLowRank) {
            const int c = ks - p.k_stages;
            const int steps = min(4, (p.rank - 64 * c) / 16);
            for (int j = 0; j < steps; ++j)
              mma_bf16(acc, operand_desc(st + 32 * j), operand_desc(st + kABytes + 32 * j), 1u);
          }
          mma_commit(&ctl.empty[s]);
        }
        if (!ok) break;
        mma_commit(&ctl.acc_full);
      }
      if (!ok) {
        // Unwinding: wait (bounded) for this thread's MMAs to finish before TMEM is freed.
        mma_commit(&ctl.acc_empty);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;              // TMEM lane quarter this warp may access
    const int row_in_tile = quarter * 32 + lane;
    uint32_t tcount = 0;
    TileCoord t;
    for (int tile = blockIdx.x; tile_coord<kGrouped>(p, ctl, tile, t); tile += gridDim.x, ++tcount) {
      if (!mbar_wait(&ctl.acc_full, tcount & 1, abort, p.status)) break;
      tc_fence_after();
      const uint32_t buf = tcount & 1;
      const uint32_t col0 = buf ? kAccOverlapCol : 0u;
      const float alpha = __ldg(p.alpha + t.expert);
      const int row = t.m_tile * kBM + row_in_tile;
      const bool row_ok = row < t.valid_rows;
      __nv_bfloat16* out_row = p.out + (static_cast<int64_t>(t.expert) * p.m + row) * p.n;
      for (int i = 0; i < 4; ++i) {
        // accumulator 0 drains its last 64 columns first, accumulator 1 its first 64
        const int sub = buf ? i : 3 - i;
        uint32_t v[64];
        tmem_load_64(tmem + col0 + sub * 64 + (static_cast<uint32_t>(quarter * 32) << 16), v);
        if (i == 0) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl.acc_empty);
        }
        const int col_base = t.n_tile * kBN + sub * 64;
        if (row_ok) {
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const int col = col_base + 8 * g;
            if (col < p.n) {
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * g + e]);
              if (p.bias) {
                const uint4 bw = __ldg(reinterpret_cast<const uint4*>(p.bias + col));
                const uint32_t bb[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  f[2 * e] = __fmaf_rn(alpha, f[2 * e], __uint_as_float(bb[e] << 16));
                  f[2 * e + 1] = __fmaf_rn(alpha, f[2 * e + 1], __uint_as_float(bb[e] & 0xffff0000u));
                }
              } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = __fmul_rn(alpha, f[e]);
              }
              uint4 o;
              o.x = pack_bf16x2(f[0], f[1]);
              o.y = pack_bf16x2(f[2], f[3]);
              o.z = pack_bf16x2(f[4], f[5]);
              o.w = pack_bf16x2(f[6], f[7]);
              *reinterpret_cast<uint4*>(out_row + col) = o;
            }
          }
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (*abort) {
      // The issuer committed a final arrival on acc_empty when it unwound; give the
      // outstanding MMAs a bounded time to finish before the columns are released.
      const uint64_t t0 = global_ns();
      while (global_ns() - t0 < 2000000ull) {
      }
    }
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ---- host side ------------------------------------------------------------------------------------

int make_map(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t rank, const void* base, const uint64_t* dims,
             const uint64_t* strides_bytes, const uint32_t* box) {
  EncodeTiledFn encode = encode_tiled_fn();
  if (!encode) return NVFP4_ERR_CUDA;
  uint32_t elem_strides[3] = {1, 1, 1};
  CUresult r = encode(map, dtype, rank, const_cast<void*>(base), dims, strides_bytes, box, elem_strides,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_INVALID_ARGUMENT;
}

// Packed FP4 operand [experts, rows, k/2] as a tiled uint8 tensor with boxes of 128 bytes
// (one stage of K) by box_rows rows.
int make_operand_map(CUtensorMap* map, const uint8_t* base, int64_t experts, int64_t rows, int64_t k,
                     uint32_t box_rows, bool grouped) {
  const uint64_t dims[3] = {static_cast<uint64_t>(k / 2), static_cast<uint64_t>(rows), static_cast<uint64_t>(experts)};
  const uint64_t strides[2] = {static_cast<uint64_t>(k / 2), static_cast<uint64_t>(rows * (k / 2))};
  const uint32_t box[3] = {kStageBytesRow, box_rows, 1};
  return make_map(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, grouped ? 3 : 2, base, dims, strides, box);
}

// bf16 low-rank operand [rows, r] with boxes of 64 values (128 bytes) by box_rows rows.
int make_lowrank_map(CUtensorMap* map, const void* base, int64_t rows, int64_t r, uint32_t box_rows) {
  const uint64_t dims[2] = {static_cast<uint64_t>(r), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(r * 2)};
  const uint32_t box[2] = {64, box_rows};
  return make_map(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box);
}

template <bool kGrouped, bool kLowRank>
int launch_gemm(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, const uint8_t* b_sf, const float* alpha,
                const void* d, const void* l1, int64_t r, const void* bias, const int32_t* mask, void* out,
                int64_t E, int64_t m, int64_t n, int64_t k, cudaStream_t stream) {
  if (E < 0 || m < 0 || n < 0 || k <= 0 || k % 64 != 0 || n % 8 != 0) return NVFP4_ERR_INVALID_ARGUMENT;
  if (m > (1 << 30) || n > (1 << 30) || k > (1 << 30) || E > kMaxExperts) return NVFP4_ERR_INVALID_ARGUMENT;
  if (kLowRank && (r <= 0 || r % 32 != 0 || r > 256)) return NVFP4_ERR_INVALID_ARGUMENT;
  if (E == 0 || m == 0 || n == 0) return NVFP4_OK;
  if (!a || !b || !a_sf || !b_sf || !alpha || !out) return NVFP4_ERR_INVALID_ARGUMENT;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(a_sf, 16) || !aligned(b_sf, 16) || !aligned(out, 16) ||
      !aligned(alpha, 4) || (bias && !aligned(bias, 16)))
    return NVFP4_ERR_INVALID_ARGUMENT;
  if (kGrouped && (!mask || !aligned(mask, 4))) return NVFP4_ERR_INVALID_ARGUMENT;
  if (kLowRank && (!d || !l1 || !aligned(d, 16) || !aligned(l1, 16))) return NVFP4_ERR_INVALID_ARGUMENT;

  DeviceInfo info;
  int st = current_device(&info);
  if (st != NVFP4_OK) return st;

  CUtensorMap map_a, map_b, map_d, map_l1;
  memset(&map_d, 0, sizeof(map_d));
  memset(&map_l1, 0, sizeof(map_l1));
  if ((st = make_operand_map(&map_a, a, E, m, k, kBM, kGrouped)) != NVFP4_OK) return st;
  if ((st = make_operand_map(&map_b, b, E, n, k, kBN, kGrouped)) != NVFP4_OK) return st;
  if (kLowRank) {
    if ((st = make_lowrank_map(&map_d, d, m, r, kBM)) != NVFP4_OK) return st;
    if ((st = make_lowrank_map(&map_l1, l1, n, r, kBN)) != NVFP4_OK) return st;
  }

  GemmParams p;
  p.a_sf = a_sf;
  p.b_sf = b_sf;
  p.a_sf_stride = nvfp4_scale_bytes(m, k);
  p.b_sf_stride = nvfp4_scale_bytes(n, k);
  p.alpha = alpha;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.mask = mask;
  p.status = info.status;
  p.m = static_cast<int32_t>(m);
  p.n = static_cast<int32_t>(n);
  p.k = static_cast<int32_t>(k);
  p.experts = static_cast<int32_t>(E);
  p.rank = static_cast<int32_t>(r);
  p.n_tiles = static_cast<int32_t>((n + kBN - 1) / kBN);
  p.m_tiles = static_cast<int32_t>((m + kBM - 1) / kBM);
  p.k_stages = static_cast<int32_t>((k + kStageK - 1) / kStageK);
  p.k_steps = static_cast<int32_t>(k / 64);
  p.sf_groups = static_cast<int32_t>(k / 64);
  p.sf_row_tiles_b = static_cast<int32_t>((n + 127) / 128);

  auto kernel = nvfp4_gemm_kernel<kGrouped, kLowRank>;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    attr_set = true;
  }
  int64_t tiles = kGrouped ? static_cast<int64_t>(E) * p.m_tiles * p.n_tiles : static_cast<int64_t>(p.m_tiles) * p.n_tiles;
  if (tiles >= (int64_t(1) << 31)) return NVFP4_ERR_INVALID_ARGUMENT;
  const int grid = static_cast<int>(tiles < info.sm_count ? tiles : info.sm_count);
  kernel<<<grid, kThreads, kSmemBytes, stream>>>(map_a, map_b, map_d, map_l1, p);
  return launch_status();
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

int nvfp4_gemm(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, const uint8_t* b_sf, const float* alpha,
               const void* bias_bf16, void* out_bf16, int64_t m, int64_t n, int64_t k, nvfp4_stream_t stream) {
  return launch_gemm<false, false>(a, b, a_sf, b_sf, alpha, nullptr, nullptr, 0, bias_bf16, nullptr, out_bf16, 1, m,
                                   n, k, stream);
}

int nvfp4_grouped_gemm_masked(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, const uint8_t* b_sf,
                              const int32_t* mask, const float* alpha, void* out_bf16, int64_t E, int64_t mmax,
                              int64_t n, int64_t k, nvfp4_stream_t stream) {
  return launch_gemm<true, false>(a, b, a_sf, b_sf, alpha, nullptr, nullptr, 0, nullptr, mask, out_bf16, E, mmax, n,
                                  k, stream);
}

int nvfp4_gemm_lowrank_bias(const uint8_t* a, const uint8_t* b, const uint8_t* a_sf, const uint8_t* b_sf,
                            const float* alpha, const void* d_bf16, const void* l1_bf16, int64_t r,
                            const void* bias_bf16, void* out_bf16, int64_t m, int64_t n, int64_t k,
                            nvfp4_stream_t stream) {
  return launch_gemm<false, true>(a, b, a_sf, b_sf, alpha, d_bf16, l1_bf16, r, bias_bf16, nullptr, out_bf16, 1, m, n,
                                  k, stream);
}

}  // extern "C"
