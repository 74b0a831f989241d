// common.cuh -- internal declarations shared by the libnvfp4 translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <functional>
#include <utility>

#include "nvfp4.h"

namespace nvfp4 {

// ---- host side ------------------------------------------------------------------------

struct DeviceInfo {
  int device = -1;
  int sm_count = 0;
  int* status = nullptr;  // device-side status word (NVFP4_OK or NVFP4_ERR_DEVICE_TIMEOUT)
  const float* silu_table = nullptr;  // SiLU of every bf16 value the closed forms do not cover
};

// Checks that the current device is compute capability 10.0 and returns its info; the
// first call on a device allocates the status word and computes the SiLU table (one kernel
// on the legacy default stream, waited for before returning).
int current_device(DeviceInfo* out);

// Library-owned scratch of the global-scale reductions, one per (device, stream): word 0
// is the ticket counter, words 1..kMaxItems hold per-item amax bits.  Allocated and
// zeroed on the first call for a stream; the reduction kernels leave it zeroed.
constexpr int kMaxItems = 4096;
int stream_workspace(cudaStream_t stream, uint32_t** out);

// Maps the last CUDA error (launch configuration, ...) to a status code.
int launch_status();

// One-time launch set-up of `kernel` on `device` (the current device): the first call for
// the pair runs `setup`, which may opt the kernel into dynamic shared memory and query its
// occupancy (both are properties of the current device), and caches the value it stores;
// later calls for the pair return the cached value.  Runs under the library lock, so
// `setup` must not call current_device or stream_workspace.  Returns setup's status.
int kernel_setup(const void* kernel, int device, const std::function<int(int*)>& setup, int* value);

// Whether kernels are launched with programmatic dependent launch (nvfp4_set_pdl).
bool pdl_enabled();

// The dense GEMM whose epilogue warps first quantize the bf16 activation a_bf16 [m, k] with
// the static global scale a_gsf into a_q_ws / a_sf_ws, from which its producers load A chunk
// by chunk (gemm.cu).  Checks its own arguments; k <= 16384.
int gemm_quantize_a(const void* a_bf16, const uint8_t* b, const uint8_t* b_sf, const float* a_gsf, const float* alpha,
                    const void* bias_bf16, void* out_bf16, uint8_t* a_q_ws, uint8_t* a_sf_ws, int64_t m, int64_t n,
                    int64_t k, cudaStream_t stream);

// Launches `kernel` on `stream`, with the programmatic-stream-serialization attribute when
// PDL is enabled: the kernel may then start while its predecessor in the stream finishes,
// and every kernel of this library waits (griddepcontrol.wait) before its first global
// memory access, so the predecessor's results are complete when it reads or overwrites
// them.  Returns NVFP4_OK or NVFP4_ERR_CUDA.
template <typename... KernelArgs, typename... Args>
int launch_kernel(void (*kernel)(KernelArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                  Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  return NVFP4_OK;
}

// Launches `kernel` as a cooperative grid (every CTA resident at once; the launch fails
// if the grid cannot be) for kernels whose CTAs wait on one another.  It is not given the
// programmatic-serialization attribute, so it starts after its predecessor in the stream
// completes.
template <typename... KernelArgs, typename... Args>
int launch_kernel_cooperative(void (*kernel)(KernelArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  return NVFP4_OK;
}

// ---- device side --------------------------------------------------------------------

// Lets the next kernel of the stream (launched with PDL) start its launch and prologue.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Waits until the preceding kernel of the stream has completed and its memory operations
// are visible (returns at once when the kernel was not launched with PDL).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Index checks of plain global loads and stores: in debug builds (-DNVFP4_DEBUG_INDEX) an
// index at or beyond the operand's extent is reported as NVFP4_ERR_INDEX in the device status
// word and the caller skips the access; release builds compile the check to `true`.
#ifdef NVFP4_DEBUG_INDEX
constexpr bool kDebugIndex = true;
__device__ __forceinline__ bool index_ok(uint64_t index, uint64_t extent, int* status) {
  if (index < extent) return true;
  if (status) atomicExch(status, NVFP4_ERR_INDEX);   // (a kernel without a status word passes null)
  return false;
}
#else
constexpr bool kDebugIndex = false;
__device__ __forceinline__ bool index_ok(uint64_t, uint64_t, int*) { return true; }
#endif

// cuTensorMapEncodeTiled, fetched from the driver through the runtime (no -lcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

}  // namespace nvfp4
