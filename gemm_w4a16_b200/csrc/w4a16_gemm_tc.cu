// Tensor-core (tcgen05) path -- placeholder until the kernel lands.
#include "w4a16_internal.cuh"

namespace w4a16 {

__device__ int g_device_status = 0;

int gemv_max_n() { return 1 << 20; }

cudaError_t launch_gemm_tc(const uint8_t*, const uint16_t*, const uint8_t*, const uint16_t*,
                           uint16_t*, int, int, int, cudaStream_t) {
  return cudaErrorNotSupported;
}

cudaError_t read_and_clear_device_status(cudaStream_t stream, int* status) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
  if (e != cudaSuccess) return e;
  int zero = 0;
  e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
  if (e != cudaSuccess) return e;
  *status = v ? W4A16_ERR_TIMEOUT : W4A16_OK;
  return cudaSuccess;
}

}  // namespace w4a16
