// api.cu -- status strings, version, workspace initialisation and status readback.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

extern "C" const char* moe_status_string(moe_status_t status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: size beyond the library's limits (E or E_local > 1024, k > 32)";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing or too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA launch or copy failed";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: a bounded device wait ran out";
    case MOE_ERR_BAD_EXPERT_ID: return "MOE_ERR_BAD_EXPERT_ID: expert id or map value out of range (slot dropped)";
    case MOE_ERR_BAD_ROW: return "MOE_ERR_BAD_ROW: inv_perm row out of range (slot skipped)";
    default: return "MOE_ERR_UNKNOWN";
  }
}

extern "C" int32_t moe_version(void) { return 100; /* 0.1.0 */ }

extern "C" moe_status_t moe_workspace_init(void* workspace, size_t bytes, void* stream) {
  if (workspace == nullptr && bytes > 0) return MOE_ERR_INVALID_ARG;
  if (bytes == 0) return MOE_OK;
  return cudaMemsetAsync(workspace, 0, bytes, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MOE_OK
                                                                                                : MOE_ERR_CUDA;
}

extern "C" moe_status_t moe_read_status(int32_t* device_status_word, void* stream, moe_status_t* device_status) {
  if (device_status_word == nullptr || device_status == nullptr) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t host = 0;
  if (cudaMemcpyAsync(&host, device_status_word, sizeof(host), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaMemsetAsync(device_status_word, 0, sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  *device_status = static_cast<moe_status_t>(host);
  return MOE_OK;
}
