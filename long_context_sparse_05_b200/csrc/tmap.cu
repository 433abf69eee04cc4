// Host helpers for TMA tensor maps (driver entry point fetched at run time, so
// the library needs no link-time dependency on libcuda) and the device error
// word of the bounded waits.
#include <cudaTypedefs.h>

#include "tc_common.cuh"

namespace csa {

namespace {
__device__ int g_device_error = 0;
}

int* device_error_word() {
  static int* ptr[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    ptr[dev] = static_cast<int*>(p);
  }
  return ptr[dev];
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess || q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool encode(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
            uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bool make_tmap_2d_u8(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
                     uint32_t box_bytes, uint32_t box_rows) {
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, row_bytes, rows, row_bytes, box_bytes,
                box_rows);
}

bool make_tmap_2d_u8_swz(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
                         uint32_t box_bytes, uint32_t box_rows, int swizzle_bytes) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_bytes, box_rows};
  cuuint32_t es[2] = {1, 1};
  const CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                               : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                               : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                     : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                  es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_1d_f32(CUtensorMap* m, const void* base, uint64_t n, uint32_t box) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[1] = {n};
  cuuint64_t strides[1] = {4};   // unused for rank 1
  cuuint32_t bx[1] = {box};
  cuuint32_t es[1] = {1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 1, const_cast<void*>(base), dims, strides, bx,
                  es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_2d_b16(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                      uint32_t box_cols, uint32_t box_rows) {
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, cols, rows, cols * 2, box_cols,
                box_rows);
}

}  // namespace csa

extern "C" int csa_device_error(cudaStream_t stream) {
  int* p = csa::device_error_word();
  if (!p) return CSA_ERR_CUDA;
  int v = 0;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return CSA_ERR_CUDA;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return CSA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return CSA_ERR_CUDA;
  return v;
}

namespace csa {
namespace {
// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// ever arrives on; the wait gives up after limit_ns and records CSA_ERR_TIMEOUT.
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns, int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_barrier_init();
    tc::mbar_wait(&bar, 0, err, limit_ns);
  }
}
}  // namespace
}  // namespace csa

extern "C" csa_status csa_selftest_bounded_wait(int limit_us, cudaStream_t stream) {
  if (limit_us < 1 || limit_us > 100000) return CSA_ERR_INVALID_ARG;
  int* err = csa::device_error_word();
  if (!err) return CSA_ERR_CUDA;
  csa::bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>((uint64_t)limit_us * 1000u, err);
  return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}
