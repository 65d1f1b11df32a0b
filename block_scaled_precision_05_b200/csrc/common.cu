// common.cu -- status strings, device checks, the device error word, and the
// tensor-map encoder lookup.
#include <mutex>

#include "bsp_internal.h"

// One error word per device; kernels OR codes into it when a bounded wait
// runs out (bsp_device.cuh: kErrTimeout).
__device__ uint32_t g_bsp_error_word;

namespace bsp {

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
DeviceInfo g_info[kMaxDevices];
}  // namespace

int current_device(DeviceInfo* out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return BSP_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_info[dev];
  if (d.id < 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return BSP_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return BSP_ERR_UNSUPPORTED_DEVICE;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bsp_error_word) != cudaSuccess) {
      cudaGetLastError();
      return BSP_ERR_CUDA;
    }
    d.sm_count = sms;
    d.err_word = static_cast<uint32_t*>(p);
    d.id = dev;
  }
  *out = d;
  return BSP_OK;
}

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      p = nullptr;
    }
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

}  // namespace bsp

extern "C" {

const char* bsp_status_string(int status) {
  switch (status) {
    case BSP_OK: return "BSP_OK";
    case BSP_ERR_INVALID_ARG: return "BSP_ERR_INVALID_ARG: an argument is out of range or NULL";
    case BSP_ERR_ALIGNMENT: return "BSP_ERR_ALIGNMENT: a pointer or leading dimension is misaligned";
    case BSP_ERR_UNSUPPORTED_DEVICE: return "BSP_ERR_UNSUPPORTED_DEVICE: the current device is not sm_100";
    case BSP_ERR_CUDA: return "BSP_ERR_CUDA: a CUDA runtime call or kernel launch failed";
    case BSP_ERR_TIMEOUT: return "BSP_ERR_TIMEOUT: a bounded wait inside a kernel ran out";
    default: return "BSP_ERR_UNKNOWN";
  }
}

int bsp_version(void) { return 100; }

size_t bsp_nvfp4_sf_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K < 0 || K % 16 != 0) return 0;
  return static_cast<size_t>(bsp::round_up(rows, 128) * bsp::round_up(K / 16, 4));
}

size_t bsp_nvfp4_sf_bytes_layout(int64_t rows, int64_t K, int sf_layout) {
  if (sf_layout == BSP_SF_LAYOUT_128X4) return bsp_nvfp4_sf_bytes(rows, K);
  if (sf_layout != BSP_SF_LAYOUT_8X4 || rows < 0 || K < 0 || K % 16 != 0) return 0;
  return static_cast<size_t>(bsp::round_up(rows, 8) * bsp::round_up(K / 16, 4));
}

size_t bsp_mxfp8_sf_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K < 0 || K % 32 != 0) return 0;
  return static_cast<size_t>(bsp::round_up(rows, 128) * bsp::round_up(K / 32, 4));
}

int bsp_device_status(bsp_stream_t stream) {
  bsp::DeviceInfo dev;
  int st = bsp::current_device(&dev);
  if (st != BSP_OK) return st;
  if (cudaStreamSynchronize(stream) != cudaSuccess) {
    cudaGetLastError();
    return BSP_ERR_CUDA;
  }
  uint32_t word = 0;
  if (cudaMemcpyFromSymbol(&word, g_bsp_error_word, sizeof(word)) != cudaSuccess) {
    cudaGetLastError();
    return BSP_ERR_CUDA;
  }
  if (word != 0) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(g_bsp_error_word, &zero, sizeof(zero)) != cudaSuccess) {
      cudaGetLastError();
      return BSP_ERR_CUDA;
    }
    return BSP_ERR_TIMEOUT;
  }
  return BSP_OK;
}

}  // extern "C"
