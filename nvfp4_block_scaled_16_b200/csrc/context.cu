// context.cu -- per-device state, per-stream reduction scratch, status codes.
#include <atomic>
#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "nvfp4_math.cuh"

namespace nvfp4 {
namespace {

// One index equal to its extent, submitted to the debug-build check (nothing is accessed).
__global__ void index_check_selftest_kernel(int* status) {
  if (threadIdx.x == 0) (void)index_ok(1, 1, status);
}

__global__ void silu_table_kernel(float* tab) {
  const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < kSiluEntries) tab[i] = silu_table_entry(i);
}

std::mutex g_mu;
std::atomic<int> g_pdl{1};      // programmatic dependent launch, on by default (sm_100 supports it)
DeviceInfo g_dev[64];
std::map<std::pair<int, cudaStream_t>, uint32_t*> g_ws;
std::map<std::pair<const void*, int>, int> g_kernel_cfg;   // (kernel, device) -> launch set-up value

}  // namespace

int current_device(DeviceInfo* out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.device < 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return NVFP4_ERR_UNSUPPORTED_DEVICE;
    int* status = nullptr;
    if (cudaMalloc(&status, sizeof(int)) != cudaSuccess) {
      cudaGetLastError();
      return NVFP4_ERR_OUT_OF_MEMORY;
    }
    if (cudaMemset(status, 0, sizeof(int)) != cudaSuccess) {
      cudaGetLastError();
      cudaFree(status);
      return NVFP4_ERR_CUDA;
    }
    float* tab = nullptr;
    if (cudaMalloc(&tab, kSiluTableBytes) != cudaSuccess) {
      cudaGetLastError();
      cudaFree(status);
      return NVFP4_ERR_OUT_OF_MEMORY;
    }
    silu_table_kernel<<<(kSiluEntries + 255) / 256, 256>>>(tab);
    if (cudaGetLastError() != cudaSuccess || cudaStreamSynchronize(0) != cudaSuccess) {
      cudaGetLastError();
      cudaFree(tab);
      cudaFree(status);
      return NVFP4_ERR_CUDA;
    }
    d.status = status;
    d.silu_table = tab;
    d.sm_count = sms;
    d.device = dev;
  }
  *out = d;
  return NVFP4_OK;
}

int stream_workspace(cudaStream_t stream, uint32_t** out) {
  DeviceInfo info;
  int st = current_device(&info);
  if (st != NVFP4_OK) return st;
  std::lock_guard<std::mutex> lock(g_mu);
  auto key = std::make_pair(info.device, stream);
  auto it = g_ws.find(key);
  if (it != g_ws.end()) {
    *out = it->second;
    return NVFP4_OK;
  }
  uint32_t* ws = nullptr;
  const size_t bytes = sizeof(uint32_t) * (1 + kMaxItems);
  if (cudaMalloc(&ws, bytes) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_OUT_OF_MEMORY;
  }
  if (cudaMemset(ws, 0, bytes) != cudaSuccess) {
    cudaGetLastError();
    cudaFree(ws);
    return NVFP4_ERR_CUDA;
  }
  g_ws[key] = ws;
  *out = ws;
  return NVFP4_OK;
}

int kernel_setup(const void* kernel, int device, const std::function<int(int*)>& setup, int* value) {
  std::lock_guard<std::mutex> lock(g_mu);
  const auto key = std::make_pair(kernel, device);
  auto it = g_kernel_cfg.find(key);
  if (it != g_kernel_cfg.end()) {
    *value = it->second;
    return NVFP4_OK;
  }
  int v = 0;
  const int st = setup(&v);
  if (st != NVFP4_OK) return st;
  g_kernel_cfg[key] = v;
  *value = v;
  return NVFP4_OK;
}

bool pdl_enabled() { return g_pdl.load(std::memory_order_relaxed) != 0; }

int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

}  // namespace nvfp4

extern "C" {

const char* nvfp4_status_string(int status) {
  switch (status) {
    case NVFP4_OK: return "NVFP4_OK";
    case NVFP4_ERR_INVALID_ARGUMENT: return "NVFP4_ERR_INVALID_ARGUMENT";
    case NVFP4_ERR_UNSUPPORTED_DEVICE: return "NVFP4_ERR_UNSUPPORTED_DEVICE";
    case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA";
    case NVFP4_ERR_DEVICE_TIMEOUT: return "NVFP4_ERR_DEVICE_TIMEOUT";
    case NVFP4_ERR_OUT_OF_MEMORY: return "NVFP4_ERR_OUT_OF_MEMORY";
    case NVFP4_ERR_INDEX: return "NVFP4_ERR_INDEX";
    default: return "NVFP4_ERR_UNKNOWN";
  }
}

int64_t nvfp4_scale_bytes(int64_t rows, int64_t k) {
  if (rows < 0 || k < 0 || k % 16 != 0) return -1;
  const int64_t rp = (rows + 127) / 128 * 128;
  const int64_t cp = (k / 16 + 3) / 4 * 4;
  return rp * cp;
}

int nvfp4_debug_index_checks(void) { return nvfp4::kDebugIndex ? 1 : 0; }

int nvfp4_selftest_index_check(nvfp4_stream_t stream) {
  nvfp4::DeviceInfo info;
  int st = nvfp4::current_device(&info);
  if (st != NVFP4_OK) return st;
  return nvfp4::launch_kernel(nvfp4::index_check_selftest_kernel, dim3(1), dim3(32), 0, stream, info.status);
}

int nvfp4_set_pdl(int enable) {
  nvfp4::g_pdl.store(enable ? 1 : 0, std::memory_order_relaxed);
  return NVFP4_OK;
}

int nvfp4_get_pdl(void) { return nvfp4::g_pdl.load(std::memory_order_relaxed); }

int nvfp4_device_status(int* status_out, int clear) {
  if (!status_out) return NVFP4_ERR_INVALID_ARGUMENT;
  nvfp4::DeviceInfo info;
  int st = nvfp4::current_device(&info);
  if (st != NVFP4_OK) return st;
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  int v = 0;
  if (cudaMemcpy(&v, info.status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  if (clear && cudaMemset(info.status, 0, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  if (clear && v != NVFP4_OK) {
    // a kernel that gave up a wait may have left its reduction words set: zero this
    // device's per-stream workspaces (the device is idle after the synchronize above)
    std::lock_guard<std::mutex> lock(nvfp4::g_mu);
    for (auto& kv : nvfp4::g_ws) {
      if (kv.first.first == info.device &&
          cudaMemset(kv.second, 0, sizeof(uint32_t) * (1 + nvfp4::kMaxItems)) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
      }
    }
  }
  *status_out = v;
  return NVFP4_OK;
}

}  // extern "C"
