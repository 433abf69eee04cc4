// Lightning indexer with NVFP4 operands on tcgen05 block-scaled MMAs (sm_100a).
//
// Method: "DeepSeek Technical Reports", section DSA (I[t,s] = sum_j w[t,j] *
// ReLU(q[t,j] . k[s])); "DeepSeek V4 结构速览", section "Lightning Indexer"
// (the QK path of the indexer runs in FP4 end to end; ReLU; per-head weights;
// BF16 scores).
//
// Operands: keys [E][64 B] and queries [64 heads][64 B] of packed E2M1 codes,
// each 16-element block scaled by one UE4M3 byte.  The block scales are applied
// by the tensor core itself (tcgen05.mma kind::mxf4nvf4, 16-element scale
// vectors), so the accumulator already holds q[t,j] . k[s] and the epilogue only
// forms sum_j w[t,j] ReLU(acc) per entry.
//
// Layout of one MMA (M = 128 entries, N = 64 heads, K = 64 elements): A and B are
// K-major tiles with 64-byte swizzle (rows of 64 bytes = all 128 elements, two
// MMAs of 32 bytes each).  Scale factors live in TMEM: for each K block of 64,
// four columns hold the four UE4M3 scales of rows 0-31, 32-63, 64-95, 96-127
// (one byte per 16-element block), replicated in all four lane quarters; they are
// brought there from shared memory by tcgen05.cp 32x128b.warpx4 after the MMA warp
// has rearranged the raw per-row scales (8 bytes per row) into that order.
//
// CTA (192 threads), one query per work unit (decode):
//   warp 0  TMA producer: per tile the key block (8 KB) and its raw scales (1 KB);
//           per unit the query block (4 KB), its raw scales and head weights;
//   warp 1  scale rearrangement (all lanes) and MMA issue (lane 0);
//   warps 2-5 epilogue: tcgen05.ld, weighted ReLU head sum, causal mask, store.
#include "kernels.h"
#include "tc_common.cuh"

namespace csa {

namespace {

constexpr int kTileE = 128;
constexpr int kHeads = 64;
constexpr int kRowB = 64;                    // bytes per FP4 row (128 elements)
constexpr int kSfRowB = 8;                   // scale bytes per row
constexpr int kTileBytes = kTileE * kRowB;   // 8 KB
constexpr int kTileSf = kTileE * kSfRowB;    // 1 KB raw scales
constexpr int kQBytes = kHeads * kRowB;      // 4 KB
constexpr int kQSf = kHeads * kSfRowB;       // 512 B raw scales
constexpr int kPermBytes = 2 * 512;          // two K blocks in the tcgen05.cp layout
constexpr int NACC = 4;
constexpr int S = 12;                        // stages: also keeps one CTA per SM (TMEM)
constexpr int kMaxLocalUnits = 256;

struct IdxFp4 {
  void* scores;
  const int32_t* q_pos;
  int* err;
  int T, E_cap, E, m;
  int tiles, chunk, n_chunks, units;
  int score_f32;
  int all_visible;   // every query sees all E entries: q_pos is not read
  int dep_tile;      // tiles >= dep_tile hold entries the preceding kernel writes
};

// Stage layout (bytes): keys | raw scales | rearranged scales.
constexpr int kStage = kTileBytes + kTileSf + kPermBytes;   // 10 KB: keeps 1 KB alignment
static_assert(kStage % 1024 == 0, "stages must keep the swizzle alignment");
// Query buffer: codes | raw scales | rearranged scales | weights, padded to 1 KB so
// that the swizzled code block of either buffer starts on a 1 KB boundary.
constexpr int kQBuf = ((kQBytes + kQSf + kPermBytes + kHeads * 4) + 1023) / 1024 * 1024;

__device__ __forceinline__ uint64_t smem_desc_sw64(uint32_t saddr, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;                       // leading byte offset (unused when swizzled)
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)4 << 61;                       // SWIZZLE_64B
  return d;
}

// Source of tcgen05.cp 32x128b: 32 rows of 16 bytes, 8-row core matrices 128 B apart.
__device__ __forceinline__ uint64_t smem_desc_cp(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)((512 >> 4) & 0x3FFF) << 16;   // leading byte offset: one 16-byte column only
  d |= (uint64_t)((128 >> 4) & 0x3FFF) << 32;   // stride byte offset: next 8 rows
  d |= (uint64_t)1 << 46;                       // no swizzle
  return d;
}

// Block-scaled instruction descriptor: E2M1 x E2M1, UE4M3 scales, M = 128, N, K = 64.
__host__ __device__ constexpr uint32_t idesc_mxf4(int M, int N) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (0u << 23) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_mxf4nvf4(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                             uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb) : "memory");
}

__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// Lane m0 of the warp rearranges the raw scales of `rows` rows (8 bytes each) into the
// tcgen05.cp order for both K blocks: word (m0, m1) of block kb = raw word (m0 + 32 m1) * 2 + kb.
__device__ __forceinline__ void rearrange_scales(const uint8_t* raw, uint8_t* perm, int rows,
                                                 int lane) {
  const uint32_t* rw = reinterpret_cast<const uint32_t*>(raw);
#pragma unroll
  for (int kb = 0; kb < 2; ++kb) {
    uint32_t w[4];
#pragma unroll
    for (int m1 = 0; m1 < 4; ++m1) {
      const int r = lane + 32 * m1;
      w[m1] = r < rows ? rw[r * 2 + kb] : 0u;
    }
    *reinterpret_cast<uint4*>(perm + kb * 512 + lane * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

__global__ void __launch_bounds__(192, 1)
index_scores_fp4_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmKS,
                        const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQS,
                        const __grid_constant__ CUtensorMap tmW, IdxFp4 p) {
  constexpr int N = kHeads;
  constexpr uint32_t kTmemCols = 512;    // 4 x 64 accumulator + 4 x 8 key-scale + 2 x 8 query-scale
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sStage = base;                               // S x kStage
  uint8_t* sQ = sStage + S * kStage;                    // 2 x kQBuf
  uint64_t* bars = reinterpret_cast<uint64_t*>(sQ + 2 * kQBuf);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* bfull = bars + 2 * S;
  uint64_t* bempty = bfull + 2;
  uint64_t* tfull = bempty + 2;
  uint64_t* tempty = tfull + NACC;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + NACC);
  float* s_w = reinterpret_cast<float*>(tmem_holder + 4);     // [64] weights of the current unit
  int* s_vis = reinterpret_cast<int*>(s_w + N);               // [kMaxLocalUnits]
  int* s_ev = s_vis + kMaxLocalUnits;                         // [kMaxLocalUnits]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  pdl_launch_dependents();
  if (!p.all_visible) pdl_wait();   // the query positions come from the preceding kernel

  for (int i = threadIdx.x; i * (int)gridDim.x + (int)blockIdx.x < p.units && i < kMaxLocalUnits;
       i += blockDim.x) {
    const int u = blockIdx.x + i * gridDim.x;
    const int row = u / p.n_chunks;
    const int ev = p.all_visible ? p.E : visible_entries(p.q_pos[row], p.m, p.E);
    s_ev[i] = ev;
    s_vis[i] = (ev + kTileE - 1) / kTileE;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { tc::mbar_init(&full[i], 1); tc::mbar_init(&empty[i], 1 + 4); }
    for (int i = 0; i < 2; ++i) { tc::mbar_init(&bfull[i], 1); tc::mbar_init(&bempty[i], 1 + 4); }
    for (int i = 0; i < NACC; ++i) { tc::mbar_init(&tfull[i], 1); tc::mbar_init(&tempty[i], 4); }
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&tmK);
    tc::tma_prefetch_desc(&tmKS);
  }
  if (warp == 0) tc::tmem_alloc(tmem_holder, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t t_sfa = tmem_base + NACC * N;          // NACC x 8 columns
  const uint32_t t_sfb = t_sfa + NACC * 8;              // 2 x 8 columns

  auto unit = [&](int u, int i, int& row, int& j0, int& j1, int& nc) {
    row = u / p.n_chunks;
    const int ch = u % p.n_chunks;
    j0 = ch * p.chunk;
    j1 = min(p.tiles, j0 + p.chunk);
    nc = max(0, min(j1, s_vis[i]) - j0);
  };

  if (warp == 0) {
    if (lane == 0) {
      // key tiles the preceding kernel does not write are fetched before waiting on it
      uint32_t npre = 0;
      for (int u = blockIdx.x, i = 0; u < p.units && npre == 0; u += gridDim.x, ++i) {
        int row, j0, j1, nc;
        unit(u, i, row, j0, j1, nc);
        if (nc == 0) continue;
        const int sb = row / p.T;
        for (int j = j0; j < j0 + nc && (int)npre < S && j < p.dep_tile; ++j, ++npre) {
          const int row0 = sb * p.E_cap + j * kTileE;
          uint8_t* st = sStage + npre * kStage;
          tc::mbar_arrive_expect_tx(&full[npre], kTileBytes + kTileSf);
          tc::tma_load_2d(st, &tmK, 0, row0, &full[npre]);
          tc::tma_load_2d(st + kTileBytes, &tmKS, 0, row0 / 2, &full[npre]);
        }
        break;
      }
      pdl_wait();
      uint32_t it = 0, ul = 0;
      bool ok = true;
      for (int u = blockIdx.x, i = 0; u < p.units && ok; u += gridDim.x, ++i) {
        int row, j0, j1, nc;
        unit(u, i, row, j0, j1, nc);
        if (nc == 0) continue;
        const int bb = ul & 1;
        ok = tc::mbar_wait(&bempty[bb], ((ul >> 1) & 1) ^ 1, p.err);
        if (!ok) break;
        uint8_t* qb = sQ + bb * kQBuf;
        tc::mbar_arrive_expect_tx(&bfull[bb], kQBytes + kQSf + kHeads * 4);
        tc::tma_load_2d(qb, &tmQ, 0, row * kHeads, &bfull[bb]);
        tc::tma_load_2d(qb + kQBytes, &tmQS, 0, row * kHeads / 2, &bfull[bb]);
        tc::tma_load_1d(qb + kQBytes + kQSf + kPermBytes, &tmW, row * kHeads, &bfull[bb]);
        const int sb = row / p.T;
        for (int j = j0; j < j0 + nc; ++j, ++it) {
          if (it < npre) continue;                       // fetched before the wait
          const int s = it % S;
          ok = tc::mbar_wait(&empty[s], ((it / S) & 1) ^ 1, p.err);
          if (!ok) break;
          const int row0 = sb * p.E_cap + j * kTileE;
          uint8_t* st = sStage + s * kStage;
          tc::mbar_arrive_expect_tx(&full[s], kTileBytes + kTileSf);
          tc::tma_load_2d(st, &tmK, 0, row0, &full[s]);
          tc::tma_load_2d(st + kTileBytes, &tmKS, 0, row0 / 2, &full[s]);
        }
        ++ul;
      }
    }
  } else if (warp == 1) {
    constexpr uint32_t idesc = idesc_mxf4(kTileE, N);
    uint32_t it = 0, ul = 0, at = 0;
    bool ok = true;
    for (int u = blockIdx.x, i = 0; u < p.units && ok; u += gridDim.x, ++i) {
      int row, j0, j1, nc;
      unit(u, i, row, j0, j1, nc);
      if (nc == 0) continue;
      const int bb = ul & 1;
      uint8_t* qb = sQ + bb * kQBuf;
      ok = tc::mbar_wait(&bfull[bb], (ul >> 1) & 1, p.err);
      if (!ok) break;
      rearrange_scales(qb + kQBytes, qb + kQBytes + kQSf, kHeads, lane);
      tc::fence_proxy_async();
      __syncwarp();
      const uint32_t sfb = t_sfb + bb * 8;
      if (lane == 0) {
        tc::tc_fence_after();
        tmem_cp_32x128b_x4(sfb, smem_desc_cp(tc::smem_u32(qb + kQBytes + kQSf)));
        tmem_cp_32x128b_x4(sfb + 4, smem_desc_cp(tc::smem_u32(qb + kQBytes + kQSf + 512)));
      }
      const uint64_t bdesc = smem_desc_sw64(tc::smem_u32(qb), 512);
      for (int j = 0; j < nc; ++j, ++it, ++at) {
        const int s = it % S;
        const int acc = at % NACC;
        uint8_t* st = sStage + s * kStage;
        ok = tc::mbar_wait(&full[s], (it / S) & 1, p.err);
        if (!ok) break;
        rearrange_scales(st + kTileBytes, st + kTileBytes + kTileSf, kTileE, lane);
        tc::fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
          ok = tc::mbar_wait(&tempty[acc], ((at / NACC) & 1) ^ 1, p.err);
          if (ok) {
            tc::tc_fence_after();
            const uint32_t sfa = t_sfa + acc * 8;
            tmem_cp_32x128b_x4(sfa, smem_desc_cp(tc::smem_u32(st + kTileBytes + kTileSf)));
            tmem_cp_32x128b_x4(sfa + 4, smem_desc_cp(tc::smem_u32(st + kTileBytes + kTileSf + 512)));
            const uint64_t adesc = smem_desc_sw64(tc::smem_u32(st), 512);
            const uint32_t d = tmem_base + acc * N;
#pragma unroll
            for (int kb = 0; kb < 2; ++kb)   // K = 64 elements = 32 bytes per MMA
              mma_mxf4nvf4(d, adesc + 2 * kb, bdesc + 2 * kb, idesc, sfa + 4 * kb, sfb + 4 * kb,
                           kb > 0);
            tc::mma_commit(&empty[s]);
            tc::mma_commit(&tfull[acc]);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
      if (!ok) break;
      if (lane == 0) tc::mma_commit(&bempty[bb]);
      __syncwarp();
      ++ul;
    }
  } else {
    const int lane_base = (warp & 3) * 32;
    const int etid = threadIdx.x - 64;
    uint32_t it = 0, at = 0, ul = 0;
    bool ok = true;
    for (int u = blockIdx.x, i = 0; u < p.units; u += gridDim.x, ++i) {
      int row, j0, j1, nc;
      unit(u, i, row, j0, j1, nc);
      if (nc > 0) {
        const int bb = ul & 1;
        tc::named_bar(1, 128);
        ok = ok && tc::mbar_wait(&bfull[bb], (ul >> 1) & 1, p.err);
        const float* wsrc = reinterpret_cast<const float*>(sQ + bb * kQBuf + kQBytes + kQSf + kPermBytes);
        if (etid < N) s_w[etid] = wsrc[etid];
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bempty[bb]);
        tc::named_bar(1, 128);
        ++ul;
      }
      const int ev = s_ev[i];
      for (int j = j0; j < j1; ++j) {
        const int e = j * kTileE + lane_base + lane;
        float sc = -INFINITY;
        if (j < j0 + nc && ok) {
          const int s = it % S;
          const int acc = at % NACC;
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&empty[s]);   // epilogue reads nothing from the stage
          ok = tc::mbar_wait(&tfull[acc], (at / NACC) & 1, p.err);
          tc::tc_fence_after();
          uint32_t r0[32], r1[32];
          const uint32_t ta = tmem_base + ((uint32_t)lane_base << 16) + acc * N;
          tc::tmem_ld32(ta, r0);
          tc::tmem_ld32(ta + 32, r1);
          tc::tmem_ld_wait(r0);
          tc::reg_fence(r1);
          float a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int h = 0; h < 32; ++h) {
            a0 = fmaf(s_w[h], fmaxf(__uint_as_float(r0[h]), 0.f), a0);
            a1 = fmaf(s_w[32 + h], fmaxf(__uint_as_float(r1[h]), 0.f), a1);
          }
          sc = a0 + a1;
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&tempty[acc]);
          ++it;
          ++at;
        }
        if (e < p.E) {
          const float v = !ok ? __int_as_float(0x7fc00000) : (e < ev ? sc : -INFINITY);
          const size_t o = (size_t)row * p.E + e;
          if (p.score_f32) reinterpret_cast<float*>(p.scores)[o] = v;
          else reinterpret_cast<__nv_bfloat16*>(p.scores)[o] = __float2bfloat16_rn(v);
        }
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

csa_status launch_index_scores_fp4_tc(const IndexArgs& a, int b, cudaStream_t st) {
  if (a.qk_dtype != CSA_NVFP4 || a.H != kHeads || a.d != 128 || a.T != 1) return CSA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(a.k) & 15) || (reinterpret_cast<uintptr_t>(a.q) & 15) ||
      (reinterpret_cast<uintptr_t>(a.k_scales) & 15) || (reinterpret_cast<uintptr_t>(a.q_scales) & 15) ||
      (reinterpret_cast<uintptr_t>(a.w) & 15) || (a.E_cap % 4))
    return CSA_ERR_UNSUPPORTED;
  CUtensorMap tmK, tmKS, tmQ, tmQS, tmW;
  const uint64_t krows = (uint64_t)b * a.E_cap, qrows = (uint64_t)b * a.T * kHeads;
  if (!make_tmap_2d_u8_swz(&tmK, a.k, kRowB, krows, kRowB, kTileE, 64) ||
      !make_tmap_2d_u8_swz(&tmKS, a.k_scales, 16, krows / 2, 16, kTileE / 2, 0) ||
      !make_tmap_2d_u8_swz(&tmQ, a.q, kRowB, qrows, kRowB, kHeads, 64) ||
      !make_tmap_2d_u8_swz(&tmQS, a.q_scales, 16, qrows / 2, 16, kHeads / 2, 0) ||
      !make_tmap_1d_f32(&tmW, a.w, qrows, kHeads))
    return CSA_ERR_CUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  IdxFp4 p{};
  p.scores = a.scores; p.q_pos = a.q_pos;
  p.err = device_error_word();
  if (!p.err) return CSA_ERR_CUDA;
  p.T = a.T; p.E_cap = a.E_cap; p.E = a.E; p.m = a.m;
  p.tiles = (a.E + kTileE - 1) / kTileE;
  const long long rows = (long long)b * a.T;
  int nch = (int)((2LL * sms + rows - 1) / rows);
  nch = max(1, min(nch, p.tiles));
  p.chunk = (p.tiles + nch - 1) / nch;
  p.n_chunks = (p.tiles + p.chunk - 1) / p.chunk;
  const long long units = rows * p.n_chunks;
  if (units > 0x7fffffff) return CSA_ERR_UNSUPPORTED;
  p.units = (int)units;
  p.score_f32 = a.score_dtype == CSA_F32;
  p.all_visible = a.all_visible;
  p.dep_tile = a.dep_entry < 0 ? 0 : a.dep_entry / kTileE;
  long long grid = units < sms ? units : sms;
  const long long min_grid = (units + kMaxLocalUnits - 1) / kMaxLocalUnits;
  if (grid < min_grid) grid = min_grid;
  const size_t smem = 1024 + (size_t)S * kStage + 2 * (size_t)kQBuf + (2 * S + 4 + 2 * NACC) * 8 +
                      16 + kHeads * 4 + (size_t)kMaxLocalUnits * 2 * 4;
  if (cudaFuncSetAttribute(index_scores_fp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return CSA_ERR_CUDA;
  if (csa_launch(index_scores_fp4_kernel, dim3((unsigned)grid), dim3(192), smem, st, a.pdl != 0,
                 tmK, tmKS, tmQ, tmQS, tmW, p) != cudaSuccess)
    return CSA_ERR_CUDA;
  return CSA_OK;
}

}  // namespace csa
