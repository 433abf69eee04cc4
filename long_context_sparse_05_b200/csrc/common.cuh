// Shared device helpers of the CSA library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_fp4.h>
#include <stdint.h>

#include <utility>

#include "csa.h"

namespace csa {

constexpr int kWarp = 32;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// E4M3 code -> float (exact).
__device__ __forceinline__ float e4m3_to_f32(uint8_t code) {
  __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3);
  return __half2float(__half(h));
}

// float -> E4M3 code, round to nearest even, saturating to +-448.
__device__ __forceinline__ uint8_t f32_to_e4m3(float x) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

// Two floats -> packed E2M1 pair (lo in bits 0-3, hi in bits 4-7), RNE, saturating to +-6.
__device__ __forceinline__ uint8_t f32x2_to_e2m1x2(float lo, float hi) {
  return static_cast<uint8_t>(
      __nv_cvt_float2_to_fp4x2(make_float2(lo, hi), __NV_E2M1, cudaRoundNearest));
}

// E2M1 code (low 4 bits) -> float (exact).
__device__ __forceinline__ float e2m1_to_f32(uint8_t code) {
  __half_raw h = __nv_cvt_fp4_to_halfraw(static_cast<__nv_fp4_storage_t>(code & 0xF), __NV_E2M1);
  return __half2float(__half(h));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide sum / max; every thread gets the result.  `red` needs blockDim/32 floats.
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float r = 0.f;
  for (int i = 0; i < nw; ++i) r += red[i];
  return r;
}
__device__ __forceinline__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float r = -INFINITY;
  for (int i = 0; i < nw; ++i) r = fmaxf(r, red[i]);
  return r;
}

// Programmatic dependent launch: wait until the preceding grid of the stream has
// completed and its writes are visible (a no-op when the grid was launched
// without the programmatic attribute), and allow the next grid to launch early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// NVFP4 key-scale layout.  A sequence's key scales are stored in tiles of 128
// entries, each tile in the order the block-scaled tensor-core MMA reads from
// tensor memory (tcgen05.cp 32x128b, 4x replicated): for every 64-element K
// block, 512 bytes laid out as [row % 32][row / 32][block % 4].  A sequence of
// E_cap entries occupies ceil(E_cap / 128) tiles of 128 * c / 16 bytes
// (c a multiple of 64).
__host__ __device__ __forceinline__ size_t nvfp4_key_scale_offset(long long e, int blk, int c) {
  const long long tile = e >> 7;
  const int r = (int)(e & 127);
  return (size_t)tile * (size_t)(8 * c) + (size_t)(blk >> 2) * 512 + (size_t)(r & 31) * 16 +
         (size_t)(r >> 5) * 4 + (size_t)(blk & 3);
}
__host__ __device__ __forceinline__ size_t nvfp4_key_scale_seq_bytes(long long E_cap, int c) {
  return (size_t)((E_cap + 127) >> 7) * (size_t)(8 * c);
}

// Rotation angle p * inv_freq reduced to [-pi, pi] in float64 (Cody-Waite reduction
// with 2*pi split into a head and a tail), then float32 sin / cos of the reduced angle.
__device__ __forceinline__ void rope_angle(double ang, float* sn, float* cs) {
  const double kTwoPiHi = 6.283185307179586;          // 2*pi rounded to float64
  const double kTwoPiLo = 2.4492935982947064e-16;     // 2*pi - kTwoPiHi
  const double k = rint(ang * (1.0 / 6.283185307179586));
  double r = fma(-k, kTwoPiHi, ang);
  r = fma(-k, kTwoPiLo, r);
  sincosf((float)r, sn, cs);
}

// Inverse RoPE of one output element: dim d of a head whose last d_rope dims are rotary
// (interleaved pairs), at query position t.  x is the element's value, y its pair
// partner's; the pair is rotated by -t * inv_freq[j].
__device__ __forceinline__ float inv_rope_elem(float x, float y, int d, int D, int d_rope,
                                               float sn, float cs) {
  const int u = d - (D - d_rope);
  if (u < 0) return x;
  return (u & 1) == 0 ? fmaf(x, cs, y * sn) : fmaf(x, cs, -y * sn);
}

// Visible entries of query position t: floor((t+1)/m), clamped to [0, E].
__device__ __forceinline__ int visible_entries(int t, int m, int E) {
  int e = t < 0 ? 0 : (t + 1) / m;
  return e < E ? e : E;
}

}  // namespace csa

// Launches `kern` on `st`; with pdl, as a programmatic dependent of the preceding grid.
template <typename... KArgs, typename... Args>
inline cudaError_t csa_launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? at : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

#define CSA_CHECK_LAUNCH()                                  \
  do {                                                      \
    cudaError_t e_ = cudaGetLastError();                    \
    if (e_ != cudaSuccess) return CSA_ERR_CUDA;             \
  } while (0)
