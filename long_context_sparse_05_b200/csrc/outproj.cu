// Grouped output projection on the tcgen05 tensor cores (sm_100a).
//
// Method: "DeepSeek-V4 技术解读", section 2.1 (分组输出投影: the attention output of
// the H heads is split into g groups, each group projected on its own, which cuts the
// projection's work g-fold): group i = heads [i H/g, (i+1) H/g), concatenated into
// K = H/g * d values, y[t, i d_g + n] = sum_k o[t, i, k] W[i][n][k].
//
// One CTA per tile of 128 tokens (MMA M) x 256 outputs (MMA N) of one group, optionally
// over a slice of K (split-K, for a few tokens, when tiles alone would leave SMs idle):
//   warp 0     TMA producer: per 64-element K block one 128-byte-swizzled box of the
//              token rows (16 KB) and one of the weight rows (32 KB) into a 4-stage ring;
//              token rows past T are zero-filled by the TMA;
//   warp 1     MMA issuer (one thread): four tcgen05.mma kind::f16 (K = 16) per block
//              into a 256-column fp32 TMEM accumulator;
//   warps 2-5  epilogue: tcgen05.ld of the accumulator, one token row per thread,
//              bf16 (or, with split-K, fp32 partials that a small kernel adds).
#include "kernels.h"
#include "tc_common.cuh"

namespace csa {

namespace {

constexpr int kBM = 128;                    // tokens per tile
constexpr int kBN = 256;                    // outputs per tile
constexpr int kBK = 64;                     // bf16 per K block (one 128-byte swizzle row)
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;      // 16 KB
constexpr int kBBytes = kBN * kBK * 2;      // 32 KB
constexpr int kThreadsP = 192;
constexpr size_t kSmemP = 1024 + (size_t)kStages * (kABytes + kBBytes) + (2 * kStages + 1) * 8 + 16;

struct ProjArgs {
  __nv_bfloat16* y; float* part;
  int* err;
  int T, K, d_g, ks, kbps, n_out;
};

__global__ void __launch_bounds__(kThreadsP, 1)
out_proj_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                ProjArgs p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = base;
  uint8_t* sB = sA + kStages * kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kStages * kBBytes);
  uint64_t* empty = full + kStages;
  uint64_t* accf = empty + kStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accf + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = blockIdx.x, nt = blockIdx.y;
  const int grp = blockIdx.z / p.ks, split = blockIdx.z % p.ks;
  const int nkb = p.K / kBK;
  const int kb0 = split * p.kbps, kb1 = min(nkb, kb0 + p.kbps);

  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) { tc::mbar_init(&full[i], 1); tc::mbar_init(&empty[i], 1); }
    tc::mbar_init(accf, 1);
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&tmA);
    tc::tma_prefetch_desc(&tmB);
  }
  if (warp == 0) tc::tmem_alloc(tmem_holder, kBN);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tacc = *tmem_holder;
  pdl_wait();   // the attention output comes from the preceding kernel

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      for (int kb = kb0, it = 0; kb < kb1 && ok; ++kb, ++it) {
        const int s = it % kStages;
        ok = tc::mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, p.err);
        if (!ok) break;
        tc::mbar_arrive_expect_tx(&full[s], kABytes + kBBytes);
        tc::tma_load_2d(sA + s * kABytes, &tmA, grp * p.K + kb * kBK, mt * kBM, &full[s]);
        tc::tma_load_2d(sB + s * kBBytes, &tmB, kb * kBK, grp * p.d_g + nt * kBN, &full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = tc::instr_desc(kBM, kBN, 1, 1, 0, 0);   // bf16 x bf16 -> f32
      bool ok = true;
      for (int kb = kb0, it = 0; kb < kb1 && ok; ++kb, ++it) {
        const int s = it % kStages;
        ok = tc::mbar_wait(&full[s], (it / kStages) & 1, p.err);
        if (!ok) break;
        tc::tc_fence_after();
        const uint64_t a = tc::smem_desc_sw128(tc::smem_u32(sA + s * kABytes), 16, 1024);
        const uint64_t b = tc::smem_desc_sw128(tc::smem_u32(sB + s * kBBytes), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)   // K = 16 bf16 = 32 bytes per MMA
          tc::mma_f16(tacc, a + 2 * kk, b + 2 * kk, idesc, kb > kb0 || kk > 0);
        tc::mma_commit(&empty[s]);
      }
      tc::mma_commit(accf);   // every MMA issued above is complete when this arrives
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32 (w % 4) .. +32, one token row per thread
    const int q = warp & 3;
    const int row = mt * kBM + q * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(q * 32) << 16;
    const bool ok = tc::mbar_wait(accf, 0, p.err) && kb1 > kb0;
    tc::tc_fence_after();
    const int col0 = (int)(blockIdx.z / p.ks) * p.d_g + nt * kBN;
#pragma unroll 1
    for (int c = 0; c < kBN / 32; ++c) {
      uint32_t v[32];
      tc::tmem_ld32(tacc + c * 32 + lane_addr, v);
      tc::tmem_ld_wait(v);
      if (row >= p.T) continue;
      if (p.ks == 1) {
        uint4* dst = reinterpret_cast<uint4*>(p.y + (size_t)row * p.n_out + col0 + c * 32);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = ok ? __uint_as_float(v[8 * u + 2 * e]) : __int_as_float(0x7fc00000);
            const float x1 = ok ? __uint_as_float(v[8 * u + 2 * e + 1]) : __int_as_float(0x7fc00000);
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(x0, x1);
            w4[e] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          dst[u] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      } else {
        float4* dst = reinterpret_cast<float4*>(p.part + ((size_t)split * p.T + row) * p.n_out +
                                                col0 + c * 32);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float4 f = make_float4(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1]),
                                 __uint_as_float(v[4 * u + 2]), __uint_as_float(v[4 * u + 3]));
          if (!ok) f = make_float4(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000),
                                   __int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
          dst[u] = f;
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tacc, kBN);
  }
}

// y[t][n] = sum over the K slices of the fp32 partials; four outputs per thread.
__global__ void out_proj_reduce_kernel(const float* __restrict__ part, int ks, size_t n,
                                       __nv_bfloat16* __restrict__ y) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i >= n) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < ks; ++s) {
    const float4 v = *reinterpret_cast<const float4*>(part + (size_t)s * n + i);
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
  const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
  uint2 u;
  u.x = *reinterpret_cast<const uint32_t*>(&lo);
  u.y = *reinterpret_cast<const uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(y + i) = u;
}

struct ProjPlan { int mt, nt, ks, kbps; };

ProjPlan proj_plan(int T, int g, int d_g, int K) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  ProjPlan P;
  P.mt = (T + kBM - 1) / kBM;
  P.nt = d_g / kBN;
  const int nkb = K / kBK;
  const long long tiles = (long long)P.mt * P.nt * g;
  int ks = 1;
  if (tiles < sms) ks = (int)std::min<long long>(nkb, (sms + tiles - 1) / tiles);
  P.kbps = (nkb + ks - 1) / ks;
  P.ks = (nkb + P.kbps - 1) / P.kbps;
  return P;
}

}  // namespace

bool out_proj_supported(int H, int d, int g, int d_g) {
  if (g < 1 || H % g || d_g % kBN) return false;
  const long long K = (long long)(H / g) * d;
  return K % kBK == 0 && K <= (1 << 24);
}

size_t out_proj_workspace_bytes(int T, int H, int d, int g, int d_g) {
  if (T <= 0 || !out_proj_supported(H, d, g, d_g)) return 0;
  const ProjPlan P = proj_plan(T, g, d_g, (H / g) * d);
  return P.ks > 1 ? (size_t)P.ks * T * g * d_g * 4 + 256 : 0;
}

int out_proj_launch_count(int T, int H, int d, int g, int d_g) {
  if (T <= 0 || !out_proj_supported(H, d, g, d_g)) return 0;
  return proj_plan(T, g, d_g, (H / g) * d).ks > 1 ? 2 : 1;
}

csa_status launch_out_proj(const void* o, const void* W, int T, int H, int d, int g, int d_g,
                           void* y, void* ws, size_t ws_bytes, cudaStream_t st, bool pdl) {
  if (!out_proj_supported(H, d, g, d_g)) return CSA_ERR_UNSUPPORTED;
  const int K = (H / g) * d;
  const ProjPlan P = proj_plan(T, g, d_g, K);
  const size_t need = out_proj_workspace_bytes(T, H, d, g, d_g);
  if (need && (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 15)))
    return CSA_ERR_INVALID_ARG;
  CUtensorMap tmA, tmB;
  if (!make_tmap_2d_b16(&tmA, o, (uint64_t)H * d, (uint64_t)T, kBK, kBM) ||
      !make_tmap_2d_b16(&tmB, W, (uint64_t)K, (uint64_t)g * d_g, kBK, kBN))
    return CSA_ERR_CUDA;
  ProjArgs p{};
  p.y = static_cast<__nv_bfloat16*>(y);
  p.part = static_cast<float*>(ws);
  p.err = device_error_word();
  if (!p.err) return CSA_ERR_CUDA;
  p.T = T; p.K = K; p.d_g = d_g; p.ks = P.ks; p.kbps = P.kbps; p.n_out = g * d_g;
  if (cudaFuncSetAttribute(out_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemP) != cudaSuccess)
    return CSA_ERR_CUDA;
  if (csa_launch(out_proj_kernel, dim3(P.mt, P.nt, g * P.ks), dim3(kThreadsP), kSmemP, st, pdl,
                 tmA, tmB, p) != cudaSuccess)
    return CSA_ERR_CUDA;
  if (P.ks > 1) {
    const size_t n = (size_t)T * g * d_g;
    const unsigned blocks = (unsigned)((n / 4 + 255) / 256);
    if (csa_launch(out_proj_reduce_kernel, dim3(blocks), dim3(256), 0, st, true,
                   (const float*)p.part, P.ks, n, p.y) != cudaSuccess)
      return CSA_ERR_CUDA;
  }
  return CSA_OK;
}

}  // namespace csa
