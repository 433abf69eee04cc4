// Small device helpers used by the fused drivers.
#include "common.cuh"
#include "kernels.h"

namespace csa {

__global__ void fill_i32_kernel(int32_t* p, int count, int value) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < count) p[i] = value;
}

// p[s * n + t] = t: query positions of a prefill where every token is a query.
__global__ void iota_positions_kernel(int32_t* p, int b, int n) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < (size_t)b * n) p[i] = (int32_t)(i % n);
}

csa_status launch_fill_i32(int32_t* p, int count, int value, cudaStream_t st) {
  if (count <= 0) return CSA_OK;
  fill_i32_kernel<<<(count + 255) / 256, 256, 0, st>>>(p, count, value);
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

csa_status launch_iota_positions(int32_t* p, int b, int n, cudaStream_t st) {
  const size_t tot = (size_t)b * n;
  if (tot == 0) return CSA_OK;
  iota_positions_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, st>>>(p, b, n);
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

}  // namespace csa
