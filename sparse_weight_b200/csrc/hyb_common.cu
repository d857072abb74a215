// hyb_common.cu -- status handling, workspace initialisation and the
// per-device SM-count cache of libhyb.
#include <mutex>

#include "hyb_internal.cuh"

namespace hyb {

int device_sm_count(int *out) {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HYB_ERR_CUDA;
  if (dev < 0 || dev >= 64) return HYB_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
        cudaSuccess)
      return HYB_ERR_CUDA;
    cache[dev] = sms;
  }
  *out = cache[dev];
  return HYB_OK;
}

}  // namespace hyb

extern "C" {

const char *hyb_status_string(int status) {
  switch (status) {
    case HYB_OK: return "ok";
    case HYB_ERR_INVALID_ARG: return "invalid argument (shape, null pointer or enum)";
    case HYB_ERR_UNSUPPORTED: return "unsupported configuration";
    case HYB_ERR_ALIGNMENT: return "pointer or leading dimension not 16-byte aligned";
    case HYB_ERR_WORKSPACE: return "workspace missing or too small";
    case HYB_ERR_CUDA: return "CUDA runtime error";
    case HYB_ERR_DEVICE_CHECK: return "device-side data check failed (NaN weight or bad tile map)";
    case HYB_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out (outputs incomplete)";
    default: return "unknown status";
  }
}

int hyb_workspace_init(void *ws, size_t ws_bytes, hyb_stream_t stream) {
  if (ws == nullptr || ws_bytes < hyb::kHeaderBytes) return HYB_ERR_WORKSPACE;
  if (cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream) != cudaSuccess)
    return HYB_ERR_CUDA;
  return HYB_OK;
}

int hyb_check_status(void *ws, hyb_stream_t stream, uint32_t *flags) {
  if (ws == nullptr) return HYB_ERR_WORKSPACE;
  uint32_t host = 0;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&host, ws, sizeof host, cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return HYB_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return HYB_ERR_CUDA;
  if (host != 0) {
    if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return HYB_ERR_CUDA;
  }
  if (flags) *flags = host;
  if (host & hyb::kStatusTimeout) return HYB_ERR_TIMEOUT;
  return host ? HYB_ERR_DEVICE_CHECK : HYB_OK;
}

}  // extern "C"
