// Shared-latent MQA with window and sink on CUDA cores, for any head count /
// head dim (float32 or bf16).  It serves the small fp32 configuration and any
// shape the tensor-core kernel does not cover.
//
// Method: "DeepSeek Technical Reports", section DSA (attention over the top-k
// entries) and section CSA (sliding window of raw tokens); "DeepSeek V4
// 结构速览", sections "CSA（c4a 路线）" (window rows concatenated with the
// selected entries; K = V) and "HCA（c128a 路线）" (dense; attention sink).
//
// One CTA per query.  Heads run one after another: a thread per row forms
// the logits, a block reduction gives max and denominator (the sink joins
// both), and a thread per channel accumulates the weighted rows.
#include "common.cuh"
#include "kernels.h"

#include <climits>

namespace csa {

constexpr int kSkipRow = INT_MIN;

template <typename T>
__global__ void __launch_bounds__(256) attn_simt_kernel(AttnArgs a) {
  extern __shared__ float sm[];
  const int tq = blockIdx.x, sb = blockIdx.y;
  const size_t qrow = (size_t)sb * a.T + tq;
  // positions and indices come from device memory: anything out of range is skipped
  const int t = min(a.q_pos[qrow], a.n - 1);
  int nsel = a.idx ? a.count[qrow] : visible_entries(t, a.m, a.E_cap);
  nsel = max(0, min(nsel, a.idx ? a.k : a.E_cap));
  const int w0 = max(0, t - a.n_w + 1);
  const int nwin = t >= 0 ? t - w0 + 1 : 0;
  const int R = nsel + nwin;
  float* s_q = sm;                 // [d]
  float* s_l = s_q + a.d;          // [R]
  int* s_row = reinterpret_cast<int*>(s_l + R);   // [R] encoded row: >=0 cache entry, <0 window token
  float* s_red = reinterpret_cast<float*>(s_row + R);   // [32]
  // entry e / window token u of this sequence (paged entries, ring window as the args say)
  const T* kv = reinterpret_cast<const T*>(a.kv) + (a.block_table ? 0 : (size_t)sb * a.E_cap * a.d);
  const T* win = reinterpret_cast<const T*>(a.win) +
                 (size_t)sb * (a.win_ring ? a.win_ring : a.n) * a.d;
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    if (r < nsel) {
      int e = a.idx ? a.idx[qrow * a.k + r] : r;
      if (e >= 0 && e < a.E_cap && a.block_table) {
        const int pg = a.block_table[(size_t)sb * a.max_pages + e / kPageEntries];
        e = (unsigned)pg < (unsigned)a.num_pages ? pg * kPageEntries + e % kPageEntries : -1;
      }
      s_row[r] = (e >= 0 && (a.block_table || e < a.E_cap)) ? e : kSkipRow;
    } else {
      const int u = w0 + (r - nsel);
      s_row[r] = -1 - (a.win_ring ? u % a.win_ring : u);
    }
  }
  __syncthreads();
  for (int h = 0; h < a.H; ++h) {
    const T* qh = reinterpret_cast<const T*>(a.q) + (qrow * a.H + h) * a.d;
    for (int e = threadIdx.x; e < a.d; e += blockDim.x) s_q[e] = to_f32(qh[e]);
    __syncthreads();
    float lmax = -INFINITY;
    for (int r = threadIdx.x; r < R; r += blockDim.x) {
      const int code = s_row[r];
      float l = -INFINITY;
      if (code != kSkipRow) {
        const T* row = code >= 0 ? kv + (size_t)code * a.d : win + (size_t)(-1 - code) * a.d;
        float dot = 0.f;
        for (int e = 0; e < a.d; ++e) dot = fmaf(s_q[e], to_f32(row[e]), dot);
        l = a.scale * dot;
      }
      s_l[r] = l;
      lmax = fmaxf(lmax, l);
    }
    const float sink = a.sink[h];
    const float M = fmaxf(block_max(lmax, s_red), sink);
    float psum = 0.f;
    for (int r = threadIdx.x; r < R; r += blockDim.x) {
      const float p = expf(s_l[r] - M);
      s_l[r] = p;
      psum += p;
    }
    const float den = block_sum(psum, s_red) + expf(sink - M);
    __syncthreads();
    const float inv = 1.f / den;
    T* oh = reinterpret_cast<T*>(a.out) + (qrow * a.H + h) * a.d;
    // a thread per channel, or per rotary pair in the last d_rope_out channels (inverse
    // RoPE at the query position)
    const int base = a.d - a.d_rope_out;
    for (int e = threadIdx.x; e < base + a.d_rope_out / 2; e += blockDim.x) {
      const int c0 = e < base ? e : base + 2 * (e - base);
      const int nc = e < base ? 1 : 2;
      float acc[2] = {0.f, 0.f};
      for (int r = 0; r < R; ++r) {
        const int code = s_row[r];
        if (code == kSkipRow) continue;
        const T* row = code >= 0 ? kv + (size_t)code * a.d : win + (size_t)(-1 - code) * a.d;
        for (int u = 0; u < nc; ++u) acc[u] = fmaf(s_l[r], to_f32(row[c0 + u]), acc[u]);
      }
      if (nc == 1) {
        oh[c0] = from_f32<T>(acc[0] * inv);
      } else {
        float sn, cs;
        rope_angle((double)t * pow(a.theta, -2.0 * (double)(e - base) / (double)a.d_rope_out), &sn, &cs);
        const float x0 = acc[0] * inv, x1 = acc[1] * inv;
        oh[c0] = from_f32<T>(inv_rope_elem(x0, x1, c0, a.d, a.d_rope_out, sn, cs));
        oh[c0 + 1] = from_f32<T>(inv_rope_elem(x1, x0, c0 + 1, a.d, a.d_rope_out, sn, cs));
      }
    }
    if (a.lse && threadIdx.x == 0) a.lse[qrow * a.H + h] = M + logf(den);
    __syncthreads();
  }
}

csa_status launch_attn_simt(const AttnArgs& a, int b, int dtype, cudaStream_t st) {
  if (a.T == 0 || b == 0) return CSA_OK;
  const int Rmax = (a.idx ? a.k : a.E_cap) + a.n_w;
  const size_t smem = (size_t)(a.d + 2 * Rmax + 32) * sizeof(float);
  if (smem > 200 * 1024) return CSA_ERR_UNSUPPORTED;
  dim3 grid(a.T, b);
  if (dtype == CSA_F32) {
    cudaFuncSetAttribute(attn_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attn_simt_kernel<float><<<grid, 256, smem, st>>>(a);
  } else {
    cudaFuncSetAttribute(attn_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attn_simt_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(a);
  }
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

}  // namespace csa
