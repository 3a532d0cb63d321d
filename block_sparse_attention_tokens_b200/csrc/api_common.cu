// Status strings, error bookkeeping and the workspace status reader of libbsa.
#include <cstdio>
#include <cstring>

#include "bsa_common.cuh"
#include "nvtx_range.cuh"

namespace bsa {

static thread_local char g_last_error[256] = "";

int record_cuda_error(cudaError_t err) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(err),
                cudaGetErrorString(err));
  return BSA_ERR_CUDA;
}

int record_error_message(const char* msg) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s", msg);
  return 0;
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static int cached[64] = {0};
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

}  // namespace bsa

extern "C" const char* bsa_status_string(int status) {
  switch (status) {
    case BSA_OK: return "BSA_OK";
    case BSA_ERR_INVALID_ARG: return "BSA_ERR_INVALID_ARG";
    case BSA_ERR_UNSUPPORTED: return "BSA_ERR_UNSUPPORTED";
    case BSA_ERR_WORKSPACE: return "BSA_ERR_WORKSPACE";
    case BSA_ERR_CUDA: return "BSA_ERR_CUDA";
    case BSA_ERR_TIMEOUT: return "BSA_ERR_TIMEOUT";
    default: return "BSA_ERR_UNKNOWN";
  }
}

extern "C" const char* bsa_last_error_message(void) { return bsa::g_last_error; }

extern "C" int bsa_version(void) { return 201; }

extern "C" int bsa_read_status(void* ws, int* status, void* stream) {
  BSA_NVTX_RANGE("bsa_read_status");
  if (!ws || !status) return BSA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int value = 0;
  cudaError_t e = cudaMemcpyAsync(&value, ws, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(int), s);
  if (e != cudaSuccess) return bsa::record_cuda_error(e);
  *status = value;
  return BSA_OK;
}
