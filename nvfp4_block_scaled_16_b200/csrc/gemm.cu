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
//   warps 2-5   epilogue (both CTAs): tcgen05.ld of the CTA's 128 x 256 fp32 accumulator
//               (each warp owns its 32-lane TMEM quarter), alpha * acc + bias, bf16 stores.
// Two accumulators of 256 columns share TMEM columns [192, 256): the epilogue drains that
// overlap first and releases the accumulator, so the next tile's MMAs overlap the rest of
// the epilogue.  Scale factors use columns [448, 496).
// Every mbarrier wait is bounded (about one second of global time); a wait that runs out
// records NVFP4_ERR_DEVICE_TIMEOUT in the device status word and the CTA unwinds without
// hanging the GPU.
#include <cuda_bf16.h>

#include "common.cuh"

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
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccOverlapCol = 192;          // accumulator 1 starts here
constexpr uint32_t kSfaCol = 448;                 // SFA: 448 + 4j, SFB: 464 + 8j (+4 upper half)
constexpr uint32_t kSfbCol = 464;
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

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
constexpr int kSmemBytes = kStages * kStageBytes + sizeof(Control) + 1024;

// Instruction descriptors (tcgen05 "instruction descriptor" bit fields).
//   kind::mxf4nvf4: A/B format E2M1 (1) at bits 7..9 / 10..12, both K-major, N>>3 at
//   bits 17..22, ue4m3 scale format (0) at bit 23, M>>4 at bits 24..28, scale ids 0.
constexpr uint32_t kIdescFp4 = (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) | (uint32_t(kTileM >> 4) << 24);
//   kind::f16: fp32 accumulator (1) at bits 4..5, A/B bf16 (1), K-major, N, M as above.
constexpr uint32_t kIdescBf16 =
    (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) | (uint32_t(kTileM >> 4) << 24);

// ---- PTX wrappers ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// True in exactly one lane of a converged warp.  tcgen05 and TMA instructions are issued
// from a converged warp through this election: issuing them from a lone lane of a
// diverged warp serializes the tensor pipe.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred;
  asm volatile("{\n\t.reg .pred q;\n\telect.sync _|q, 0xffffffff;\n\tselp.u32 %0, 1, 0, q;\n\t}" : "=r"(pred));
  return pred != 0;
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Shared::cluster address of the same smem variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(const void* p, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_u32(p)), "r"(rank));
  return out;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

// Arrive on a barrier given by its shared::cluster address (possibly in the peer CTA).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
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
};

// ---- the kernel ---------------------------------------------------------------------------------

template <bool kGrouped, bool kLowRank>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ Maps maps, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Control& ctl = *reinterpret_cast<Control*>(smem + kStages * kStageBytes);
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
    mbar_init(&ctl.acc_empty, 8);     // 4 epilogue warps in each CTA of the pair
    ctl.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
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

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    // The whole warp runs the loop; one elected lane issues each stage's loads.
    if (elect_one()) {
      prefetch_map(&maps.a);
      prefetch_map(&maps.b);
      prefetch_map(&maps.sfa);
      prefetch_map(&maps.sfb);
      if constexpr (kLowRank) {
        prefetch_map(&maps.d);
        prefetch_map(&maps.l1);
      }
    }
    __syncwarp();
    const int lr_stages = kLowRank ? (p.rank + 63) / 64 : 0;
    uint32_t it = 0;
    bool ok = true;
    TileCoord t;
    for (int tile = pair; ok && tile_coord<kGrouped>(p, ctl, tile, t); tile += pairs) {
      const int a_row = t.m_tile * kTileM + static_cast<int>(rank) * kBM;
      const int b_row = t.n_tile * kBN + static_cast<int>(rank) * kBNHalf;
      // scale chunk rows (128 bytes each, 4 per chunk): this CTA's 128 A rows, both B halves
      const int sfa_row0 = ((2 * t.m_tile + static_cast<int>(rank)) * p.sf_groups) * 4;
      const int sfb_row0 = ((2 * t.n_tile) * p.sf_groups) * 4;
      const int sfb_row1 = sfb_row0 + p.sf_groups * 4;
      for (int ks = 0; ks < p.k_stages + lr_stages; ++ks, ++it) {
        const uint32_t s = it % kStages, round = it / kStages;
        if (round > 0 && !(ok = mbar_wait(&ctl.empty[s], (round - 1) & 1, abort, p.status))) break;
        uint8_t* st = smem + s * kStageBytes;
        const uint32_t full_bar = map_to_rank(&ctl.full[s], 0);
        if (elect_one()) {
          if (ks < p.k_stages) {
            if (leader) mbar_arrive_expect_tx(&ctl.full[s], kFp4TxBytes);
            if constexpr (kGrouped) {
              tma_load_3d(st, &maps.a, full_bar, ks * kStageBytesRow, a_row, t.expert);
              tma_load_3d(st + kABytes, &maps.b, full_bar, ks * kStageBytesRow, b_row, t.expert);
              tma_load_3d(st + kABytes + kBBytes, &maps.sfa, full_bar, 0, sfa_row0 + 16 * ks, t.expert);
              tma_load_3d(st + kABytes + kBBytes + kSfaBytes, &maps.sfb, full_bar, 0, sfb_row0 + 16 * ks, t.expert);
              tma_load_3d(st + kABytes + kBBytes + kSfaBytes + kSfaBytes, &maps.sfb, full_bar, 0, sfb_row1 + 16 * ks,
                          t.expert);
            } else {
              tma_load_2d(st, &maps.a, full_bar, ks * kStageBytesRow, a_row);
              tma_load_2d(st + kABytes, &maps.b, full_bar, ks * kStageBytesRow, b_row);
              tma_load_2d(st + kABytes + kBBytes, &maps.sfa, full_bar, 0, sfa_row0 + 16 * ks);
              tma_load_2d(st + kABytes + kBBytes + kSfaBytes, &maps.sfb, full_bar, 0, sfb_row0 + 16 * ks);
              tma_load_2d(st + kABytes + kBBytes + kSfaBytes + kSfaBytes, &maps.sfb, full_bar, 0, sfb_row1 + 16 * ks);
            }
          } else if constexpr (kLowRank) {
            const int c = ks - p.k_stages;
            if (leader) mbar_arrive_expect_tx(&ctl.full[s], kLrTxBytes);
            tma_load_2d(st, &maps.d, full_bar, c * 64, a_row);
            tma_load_2d(st + kABytes, &maps.l1, full_bar, c * 64, b_row);
          }
        }
        __syncwarp();
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader)
    // The whole warp runs the loop; one elected lane issues each batch of tcgen05 ops.
    if (leader) {
      const int lr_stages = kLowRank ? (p.rank + 63) / 64 : 0;
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      TileCoord t;
      for (int tile = pair; ok && tile_coord<kGrouped>(p, ctl, tile, t); tile += pairs, ++tcount) {
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
          if (elect_one()) {
            if (ks < p.k_stages) {
              const int nks = min(4, p.k_steps - 4 * ks);
              const uint32_t sfa_s = st + kABytes + kBBytes;
              const uint32_t sfb_s = sfa_s + kSfaBytes;
              for (int j = 0; j < nks; ++j) {
                tc_copy_sf(tmem + kSfaCol + 4 * j, sf_desc(sfa_s + 512 * j));
                tc_copy_sf(tmem + kSfbCol + 8 * j, sf_desc(sfb_s + 512 * j));
                tc_copy_sf(tmem + kSfbCol + 8 * j + 4, sf_desc(sfb_s + kSfaBytes + 512 * j));
                mma_fp4(acc, operand_desc(st + 32 * j), operand_desc(st + kABytes + 32 * j), tmem + kSfaCol + 4 * j,
                        tmem + kSfbCol + 8 * j, (ks > 0 || j > 0) ? 1u : 0u);
              }
            } else if constexpr (kLowRank) {
              const int c = ks - p.k_stages;
              const int steps = min(4, (p.rank - 64 * c) / 16);
              for (int j = 0; j < steps; ++j)
                mma_bf16(acc, operand_desc(st + 32 * j), operand_desc(st + kABytes + 32 * j), 1u);
            }
            mma_commit_both(&ctl.empty[s]);
          }
          __syncwarp();
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
    const uint32_t acc_empty_leader = map_to_rank(&ctl.acc_empty, 0);
    uint32_t tcount = 0;
    TileCoord t;
    for (int tile = pair; tile_coord<kGrouped>(p, ctl, tile, t); tile += pairs, ++tcount) {
      if (!mbar_wait(&ctl.acc_full, tcount & 1, abort, p.status)) break;
      tc_fence_after();
      const uint32_t buf = tcount & 1;
      const uint32_t col0 = buf ? kAccOverlapCol : 0u;
      const float alpha = __ldg(p.alpha + t.expert);
      const int row = t.m_tile * kTileM + static_cast<int>(rank) * kBM + row_in_tile;
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
          if (lane == 0) mbar_arrive_cluster(acc_empty_leader);
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

// bf16 low-rank operand [rows, r] with boxes of 64 values (128 bytes) by 128 rows.
int make_lowrank_map(CUtensorMap* map, const void* base, int64_t rows, int64_t r) {
  const uint64_t dims[2] = {static_cast<uint64_t>(r), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(r * 2)};
  const uint32_t box[2] = {64, 128};
  return make_map(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
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

  Maps maps;
  memset(&maps, 0, sizeof(maps));
  if ((st = make_operand_map(&maps.a, a, E, m, k, kGrouped)) != NVFP4_OK) return st;
  if ((st = make_operand_map(&maps.b, b, E, n, k, kGrouped)) != NVFP4_OK) return st;
  if ((st = make_scale_map(&maps.sfa, a_sf, E, m, k, kGrouped)) != NVFP4_OK) return st;
  if ((st = make_scale_map(&maps.sfb, b_sf, E, n, k, kGrouped)) != NVFP4_OK) return st;
  if (kLowRank) {
    if ((st = make_lowrank_map(&maps.d, d, m, r)) != NVFP4_OK) return st;
    if ((st = make_lowrank_map(&maps.l1, l1, n, r)) != NVFP4_OK) return st;
  }

  GemmParams p;
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
  p.m_tiles = static_cast<int32_t>((m + kTileM - 1) / kTileM);
  p.k_stages = static_cast<int32_t>((k + kStageK - 1) / kStageK);
  p.k_steps = static_cast<int32_t>(k / 64);
  p.sf_groups = static_cast<int32_t>(k / 64);

  auto kernel = nvfp4_gemm_kernel<kGrouped, kLowRank>;
  // One-time set-up per kernel instantiation: the dynamic shared memory opt-in and the
  // number of 2-CTA clusters that fit on the device at once (the persistent grid size).
  static int max_clusters = 0;
  if (max_clusters == 0) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(info.sm_count / 2 * 2);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg) != cudaSuccess || clusters <= 0) {
      cudaGetLastError();
      clusters = info.sm_count / 2;
    }
    max_clusters = clusters;
  }
  const int64_t tiles = kGrouped ? static_cast<int64_t>(E) * p.m_tiles * p.n_tiles
                                 : static_cast<int64_t>(p.m_tiles) * p.n_tiles;
  if (tiles >= (int64_t(1) << 31)) return NVFP4_ERR_INVALID_ARGUMENT;
  const int64_t max_pairs = max_clusters;
  const int pairs = static_cast<int>(tiles < max_pairs ? tiles : max_pairs);
  kernel<<<2 * pairs, kThreads, kSmemBytes, stream>>>(maps, p);
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
