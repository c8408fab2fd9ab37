// Status codes, workspace initialisation and status-word readback.
#include <cuda_runtime.h>

#include "common.cuh"

extern "C" const char* moe_error_string(int code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_CUDA: return "CUDA runtime or launch error";
    case MOE_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_DEVICE_BOUNDS: return "device-side bounds check failed";
    default: return "unknown status";
  }
}

extern "C" int moe_workspace_init(void* ws, size_t bytes, void* stream) {
  if (!ws || bytes == 0) return MOE_ERR_INVALID_ARG;
  const cudaError_t e = cudaMemsetAsync(ws, 0, bytes, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_status(void* ws, void* stream, int32_t* status, int clear) {
  if (!ws || !status) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  if (clear && v != 0) {
    if (cudaMemsetAsync(ws, 0, sizeof(moe::WsHeader), st) != cudaSuccess) return MOE_ERR_CUDA;
  }
  *status = v;
  return MOE_OK;
}
