// common.cuh -- internal declarations shared by the libnvfp4 translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "nvfp4.h"

namespace nvfp4 {

// ---- host side ------------------------------------------------------------------------

struct DeviceInfo {
  int device = -1;
  int sm_count = 0;
  int* status = nullptr;  // device-side status word (NVFP4_OK or NVFP4_ERR_DEVICE_TIMEOUT)
};

// Checks that the current device is compute capability 10.0 and returns its info; the
// first call on a device allocates the status word.
int current_device(DeviceInfo* out);

// Library-owned scratch of the global-scale reductions, one per (device, stream): word 0
// is the ticket counter, words 1..kMaxItems hold per-item amax bits.  Allocated and
// zeroed on the first call for a stream; the reduction kernels leave it zeroed.
constexpr int kMaxItems = 4096;
int stream_workspace(cudaStream_t stream, uint32_t** out);

// Maps the last CUDA error (launch configuration, ...) to a status code.
int launch_status();

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// cuTensorMapEncodeTiled, fetched from the driver through the runtime (no -lcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

}  // namespace nvfp4
