// Lightning indexer on CUDA cores, for any head count / key width and every
// operand type.  It serves the small fp32 configuration and any shape the
// tensor-core kernels do not cover.
//
// Method: "DeepSeek Technical Reports", section DSA (I[t,s] = sum_j w[t,j] *
// ReLU(q[t,j] . k[s])); "DeepSeek V4 结构速览", section "Lightning Indexer".
//
// One CTA per (query, 128-entry tile); the query's dequantised heads sit in
// shared memory, each thread scores one entry.
#include "common.cuh"
#include "kernels.h"

namespace csa {

// Element e of row `row`.  NVFP4 scale byte: `soff` = byte offset of the row's
// block-0 scale for row-major query scales (scale of block j at soff + j), or,
// with `tiled`, the key-scale layout (sequence base + entry index in `soff`).
__device__ __forceinline__ float load_code(const void* base, int dtype, size_t row, int d, int e,
                                           const void* scales, size_t srow, bool tiled = false,
                                           const uint8_t* seq_scales = nullptr, long long ent = 0) {
  if (dtype == CSA_F32) return reinterpret_cast<const float*>(base)[row * d + e];
  if (dtype == CSA_FP8_E4M3)
    return e4m3_to_f32(reinterpret_cast<const uint8_t*>(base)[row * d + e]) *
           reinterpret_cast<const float*>(scales)[srow];
  const uint8_t byte = reinterpret_cast<const uint8_t*>(base)[row * (d / 2) + e / 2];
  const float v = e2m1_to_f32((e & 1) ? (byte >> 4) : (byte & 0xF));
  const uint8_t sc = tiled ? seq_scales[nvfp4_key_scale_offset(ent, e / 16, d)]
                           : reinterpret_cast<const uint8_t*>(scales)[srow * (d / 16) + e / 16];
  return v * e4m3_to_f32(sc);
}

__global__ void __launch_bounds__(128) index_scores_simt_kernel(IndexArgs a) {
  extern __shared__ float s_q[];   // [H][d] dequantised query heads, then [H] weights
  const int tq = blockIdx.y;       // query within the sequence
  const int sb = blockIdx.z;       // sequence
  const size_t qrow = (size_t)sb * a.T + tq;
  const int H = a.H, d = a.d;
  float* s_w = s_q + H * d;
  for (int x = threadIdx.x; x < H * d; x += blockDim.x) {
    const int j = x / d, e = x % d;
    const size_t r = qrow * H + j;
    s_q[x] = load_code(a.q, a.qk_dtype, r, d, e, a.q_scales, r);
  }
  for (int j = threadIdx.x; j < H; j += blockDim.x) s_w[j] = a.w[qrow * H + j];
  __syncthreads();
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  if (s >= a.E) return;
  const int ev = visible_entries(a.q_pos[qrow], a.m, a.E);
  float score = -INFINITY;
  if (s < ev) {
    const size_t krow = (size_t)sb * a.E_cap + s;
    const bool tiled = a.qk_dtype == CSA_NVFP4;
    const uint8_t* seq_sc = tiled ? reinterpret_cast<const uint8_t*>(a.k_scales) +
                                        (size_t)sb * nvfp4_key_scale_seq_bytes(a.E_cap, d)
                                  : nullptr;
    score = 0.f;
    for (int j = 0; j < H; ++j) {
      float dot = 0.f;
      for (int e = 0; e < d; ++e)
        dot = fmaf(s_q[j * d + e],
                   load_code(a.k, a.qk_dtype, krow, d, e, a.k_scales, krow, tiled, seq_sc, s), dot);
      score = fmaf(s_w[j], fmaxf(dot, 0.f), score);
    }
  }
  const size_t o = qrow * a.E + s;
  if (a.score_dtype == CSA_F32) reinterpret_cast<float*>(a.scores)[o] = score;
  else reinterpret_cast<__nv_bfloat16*>(a.scores)[o] = __float2bfloat16_rn(score);
}

csa_status launch_index_scores_simt(const IndexArgs& a, int b, cudaStream_t st) {
  if (a.block_table) return CSA_ERR_UNSUPPORTED;   // paged keys: tensor-core shapes only
  if (a.T == 0 || a.E == 0 || b == 0) return CSA_OK;
  const size_t smem = ((size_t)a.H * a.d + a.H) * sizeof(float);
  if (smem > 200 * 1024) return CSA_ERR_UNSUPPORTED;
  cudaFuncSetAttribute(index_scores_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  dim3 grid((a.E + 127) / 128, a.T, b);
  index_scores_simt_kernel<<<grid, 128, smem, st>>>(a);
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

}  // namespace csa
