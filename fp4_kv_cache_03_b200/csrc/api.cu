// Status-word helpers and device queries of the CSA2 C ABI.
#include "common.cuh"

extern "C" csa2_status_t csa2_status_reset(void* workspace, void* stream) {
  if (!workspace) return CSA2_ERR_INVALID_ARG;
  return cudaMemsetAsync(workspace, 0, sizeof(int), (cudaStream_t)stream) == cudaSuccess
             ? CSA2_OK
             : CSA2_ERR_CUDA;
}

extern "C" csa2_status_t csa2_status_fetch(const void* workspace, void* stream) {
  if (!workspace) return CSA2_ERR_INVALID_ARG;
  int v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, (cudaStream_t)stream) !=
      cudaSuccess)
    return CSA2_ERR_CUDA;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return CSA2_ERR_CUDA;
  return (v >= CSA2_OK && v <= CSA2_ERR_TIMEOUT) ? (csa2_status_t)v : CSA2_ERR_CUDA;
}

extern "C" const char* csa2_status_string(csa2_status_t s) {
  switch (s) {
    case CSA2_OK: return "ok";
    case CSA2_ERR_INVALID_ARG: return "invalid argument";
    case CSA2_ERR_UNSUPPORTED: return "unsupported shape";
    case CSA2_ERR_CAPACITY: return "capacity exceeded (workspace or cache rows)";
    case CSA2_ERR_CUDA: return "CUDA runtime error";
    case CSA2_ERR_TIMEOUT: return "bounded device wait timed out";
  }
  return "unknown status";
}

extern "C" int32_t csa2_device_sms(void) {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}
