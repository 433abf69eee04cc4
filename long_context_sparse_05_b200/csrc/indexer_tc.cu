// Lightning indexer on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// Method: "DeepSeek Technical Reports", section DSA (I[t,s] = sum_j w[t,j] *
// ReLU(q[t,j] . k[s])); "DeepSeek V4 结构速览", section "Lightning Indexer"
// (low-precision QK path, ReLU, per-head weighted sum, BF16 scores, causal range).
//
// Shape covered: 64 index heads of 128 dims, FP8 E4M3 operands with one fp32
// scale per key row and per (query, head).  Everything else goes to the
// CUDA-core kernel.
//
// The score of one (query, entry) pair needs all 64 heads, so the tensor-core
// product is laid out with entries on M (TMEM lanes) and heads on N (TMEM
// columns): D[s, (q, j)] = K[s] . Q[q, j], M = 128 entries, N = 64 x QG
// queries, K = 128 (four MMAs of K = 32).  Each epilogue thread then owns one
// entry and forms sum_j w[q,j] qs[q,j] ReLU(D[s,(q,j)]) * ks[s] in registers,
// with no cross-thread reduction (ReLU commutes with the positive scales).
//
// Persistent, warp-specialised CTA (192 threads):
//   warp 0  TMA producer: key tiles [128 x 128 B] through an S-stage ring and
//           the query group [64 QG x 128 B] once per work unit (2 buffers);
//   warp 1  MMA issuer (one thread): 4 x tcgen05.mma kind::f8f6f4 per tile into
//           one of two TMEM accumulators, commits release the smem stage and
//           hand the accumulator to the epilogue;
//   warps 2-5 epilogue: tcgen05.ld of the accumulator, the weighted ReLU sum,
//           the causal mask, bf16 / fp32 store; tiles no query of the group can
//           see are written as -inf without any MMA.
// A work unit is (sequence, query group, chunk of entry tiles); units are dealt
// round-robin to the persistent CTAs, and every role walks the same sequence.
#include "kernels.h"
#include "tc_common.cuh"

namespace csa {

namespace {

constexpr int kTileE = 128;          // entries per tile (MMA M)
constexpr int kHeads = 64;           // index heads
constexpr int kDim = 128;            // index dim (bytes per FP8 row)
constexpr int kTileBytes = kTileE * kDim;

struct IdxTc {
  const float* w;
  const float* q_scales;
  const float* k_scales;
  const int32_t* q_pos;
  void* scores;
  int* err;
  int T, E_cap, E, m;
  int n_qg, tiles, chunk, n_chunks, units;
  int score_f32;
};

struct Unit {
  int sb, g, j0, j1, vis_tiles, nq;
};

template <int QG>
__device__ __forceinline__ Unit decode_unit(const IdxTc& p, int u) {
  Unit U;
  const int ch = u % p.n_chunks;
  const int tmp = u / p.n_chunks;
  U.g = tmp % p.n_qg;
  U.sb = tmp / p.n_qg;
  U.j0 = ch * p.chunk;
  U.j1 = min(p.tiles, U.j0 + p.chunk);
  U.nq = min(QG, p.T - U.g * QG);
  int ev = 0;
  for (int q = 0; q < U.nq; ++q)
    ev = max(ev, visible_entries(p.q_pos[(size_t)U.sb * p.T + U.g * QG + q], p.m, p.E));
  U.vis_tiles = (ev + kTileE - 1) / kTileE;
  return U;
}

template <int QG>
__device__ __forceinline__ int computed_tiles(const Unit& U) {
  return max(0, min(U.j1, U.vis_tiles) - U.j0);
}

template <int QG, int S>
__global__ void __launch_bounds__(192, 1)
index_scores_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                       IdxTc p) {
  constexpr int N = kHeads * QG;
  constexpr int kQBytes = N * kDim;
  constexpr uint32_t kTmemCols = (2 * N <= 32) ? 32 : (2 * N <= 64 ? 64 : (2 * N <= 128 ? 128 : (2 * N <= 256 ? 256 : 512)));
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = base;                                   // S x 16 KB
  uint8_t* sB = sA + S * kTileBytes;                    // 2 x kQBytes
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + 2 * kQBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* bfull = bars + 2 * S;
  uint64_t* bempty = bfull + 2;
  uint64_t* tfull = bempty + 2;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + 2);
  float* s_wq = reinterpret_cast<float*>(tmem_holder + 4);   // [QG][64]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { tc::mbar_init(&full[i], 1); tc::mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bfull[i], 1); tc::mbar_init(&bempty[i], 1);
      tc::mbar_init(&tfull[i], 1); tc::mbar_init(&tempty[i], 4);
    }
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&tmK);
    tc::tma_prefetch_desc(&tmQ);
  }
  if (warp == 0) tc::tmem_alloc(tmem_holder, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      uint32_t it = 0, ul = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        const Unit U = decode_unit<QG>(p, u);
        const int nc = computed_tiles<QG>(U);
        if (nc == 0) continue;
        const int bb = ul & 1;
        ok = tc::mbar_wait(&bempty[bb], ((ul >> 1) & 1) ^ 1, p.err);
        if (!ok) break;
        tc::mbar_arrive_expect_tx(&bfull[bb], kQBytes);
        tc::tma_load_2d(sB + bb * kQBytes, &tmQ, 0, (U.sb * p.T + U.g * QG) * kHeads, &bfull[bb]);
        for (int j = U.j0; j < U.j0 + nc; ++j, ++it) {
          const int s = it % S;
          ok = tc::mbar_wait(&empty[s], ((it / S) & 1) ^ 1, p.err);
          if (!ok) break;
          tc::mbar_arrive_expect_tx(&full[s], kTileBytes);
          tc::tma_load_2d(sA + s * kTileBytes, &tmK, 0, U.sb * p.E_cap + j * kTileE, &full[s]);
        }
        ++ul;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = tc::instr_desc(kTileE, N, 0, 0, 0, 0);   // e4m3 x e4m3 -> f32
      uint32_t it = 0, ul = 0, at = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        const Unit U = decode_unit<QG>(p, u);
        const int nc = computed_tiles<QG>(U);
        if (nc == 0) continue;
        const int bb = ul & 1;
        ok = tc::mbar_wait(&bfull[bb], (ul >> 1) & 1, p.err);
        if (!ok) break;
        const uint64_t bdesc = tc::smem_desc_sw128(tc::smem_u32(sB + bb * kQBytes), 16, 1024);
        for (int j = 0; j < nc; ++j, ++it, ++at) {
          const int s = it % S;
          const int acc = at & 1;
          ok = tc::mbar_wait(&full[s], (it / S) & 1, p.err);
          if (!ok) break;
          ok = tc::mbar_wait(&tempty[acc], ((at >> 1) & 1) ^ 1, p.err);
          if (!ok) break;
          tc::tc_fence_after();
          const uint64_t adesc = tc::smem_desc_sw128(tc::smem_u32(sA + s * kTileBytes), 16, 1024);
          const uint32_t d = tmem_base + acc * N;
#pragma unroll
          for (int kk = 0; kk < kDim / 32; ++kk)   // K = 32 bytes of E4M3 per MMA
            tc::mma_f8f6f4(d, adesc + 2 * kk, bdesc + 2 * kk, idesc, kk > 0);
          tc::mma_commit(&empty[s]);
          tc::mma_commit(&tfull[acc]);
        }
        if (!ok) break;
        tc::mma_commit(&bempty[bb]);
        ++ul;
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int ew = warp - 2;                 // 0..3
    const int lane_base = (warp & 3) * 32;   // TMEM lanes this warp may access
    const int etid = threadIdx.x - 64;       // 0..127
    uint32_t at = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
      const Unit U = decode_unit<QG>(p, u);
      tc::named_bar(1, 128);
      for (int x = etid; x < U.nq * kHeads; x += 128) {
        const size_t r = ((size_t)U.sb * p.T + U.g * QG) * kHeads + x;
        s_wq[x] = p.w[r] * p.q_scales[r];
      }
      tc::named_bar(1, 128);
      int tq[QG], evq[QG];
#pragma unroll
      for (int q = 0; q < QG; ++q) {
        tq[q] = q < U.nq ? U.g * QG + q : 0;
        evq[q] = q < U.nq ? visible_entries(p.q_pos[(size_t)U.sb * p.T + tq[q]], p.m, p.E) : 0;
      }
      for (int j = U.j0; j < U.j1; ++j) {
        const int e = j * kTileE + lane_base + lane;
        float sc[QG];
        if (j < U.vis_tiles && ok) {
          const int acc = at & 1;
          ok = tc::mbar_wait(&tfull[acc], (at >> 1) & 1, p.err);
          tc::tc_fence_after();
          const float ks = (e < p.E) ? p.k_scales[(size_t)U.sb * p.E_cap + e] : 0.f;
#pragma unroll
          for (int q = 0; q < QG; ++q) {
            uint32_t r0[32], r1[32];
            const uint32_t ta = tmem_base + ((uint32_t)lane_base << 16) + acc * N + q * kHeads;
            tc::tmem_ld32(ta, r0);
            tc::tmem_ld32(ta + 32, r1);
            tc::tmem_ld_wait(r0);
            tc::reg_fence(r1);
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int h = 0; h < 32; ++h) {
              a0 = fmaf(s_wq[q * kHeads + h], fmaxf(__uint_as_float(r0[h]), 0.f), a0);
              a1 = fmaf(s_wq[q * kHeads + 32 + h], fmaxf(__uint_as_float(r1[h]), 0.f), a1);
            }
            sc[q] = (a0 + a1) * ks;
          }
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&tempty[acc]);
          ++at;
        } else {
#pragma unroll
          for (int q = 0; q < QG; ++q) sc[q] = -INFINITY;
        }
        if (e < p.E) {
#pragma unroll
          for (int q = 0; q < QG; ++q) {
            if (q >= U.nq) break;
            const float v = (e < evq[q] && ok) ? sc[q] : (ok ? -INFINITY : __int_as_float(0x7fc00000));
            const size_t o = ((size_t)U.sb * p.T + tq[q]) * p.E + e;
            if (p.score_f32) reinterpret_cast<float*>(p.scores)[o] = v;
            else reinterpret_cast<__nv_bfloat16*>(p.scores)[o] = __float2bfloat16_rn(v);
          }
        }
      }
      (void)ew;
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int QG, int S>
csa_status launch_qg(const IndexArgs& a, int b, cudaStream_t st) {
  CUtensorMap tmK, tmQ;
  if (!make_tmap_2d_u8(&tmK, a.k, kDim, (uint64_t)b * a.E_cap, kDim, kTileE)) return CSA_ERR_CUDA;
  if (!make_tmap_2d_u8(&tmQ, a.q, kDim, (uint64_t)b * a.T * kHeads, kDim, kHeads * QG))
    return CSA_ERR_CUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  IdxTc p{};
  p.w = a.w; p.q_scales = reinterpret_cast<const float*>(a.q_scales);
  p.k_scales = reinterpret_cast<const float*>(a.k_scales); p.q_pos = a.q_pos; p.scores = a.scores;
  p.err = device_error_word();
  if (!p.err) return CSA_ERR_CUDA;
  p.T = a.T; p.E_cap = a.E_cap; p.E = a.E; p.m = a.m;
  p.n_qg = (a.T + QG - 1) / QG;
  p.tiles = (a.E + kTileE - 1) / kTileE;
  const long long groups = (long long)b * p.n_qg;
  // split each query group's tiles into chunks so that there are at least ~2 units per SM
  int nch = (int)((2LL * sms + groups - 1) / groups);
  nch = max(1, min(nch, p.tiles));
  p.chunk = (p.tiles + nch - 1) / nch;
  p.n_chunks = (p.tiles + p.chunk - 1) / p.chunk;
  const long long units = groups * p.n_chunks;
  if (units > 0x7fffffff) return CSA_ERR_UNSUPPORTED;
  p.units = (int)units;
  p.score_f32 = a.score_dtype == CSA_F32;
  const size_t smem = 1024 + (size_t)S * kTileBytes + 2 * (size_t)kHeads * QG * kDim +
                      (2 * S + 8) * 8 + 16 + QG * kHeads * 4;
  auto kern = index_scores_tc_kernel<QG, S>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return CSA_ERR_CUDA;
  const int grid = (int)(units < sms ? units : sms);
  kern<<<grid, 192, smem, st>>>(tmK, tmQ, p);
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

}  // namespace

csa_status launch_index_scores_tc(const IndexArgs& a, int b, cudaStream_t st) {
  if (a.qk_dtype != CSA_FP8_E4M3 || a.H != kHeads || a.d != kDim) return CSA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(a.k) & 15) || (reinterpret_cast<uintptr_t>(a.q) & 15))
    return CSA_ERR_UNSUPPORTED;
  if (a.T >= 4) return launch_qg<4, 4>(a, b, st);
  return launch_qg<1, 8>(a, b, st);
}

}  // namespace csa
