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
// product puts entries on M (TMEM lanes) and heads on N (TMEM columns):
// D[s, (q, j)] = K[s] . Q[q, j], M = 128 entries, N = 64 x QG queries, K = 128
// (four MMAs of K = 32).  Each epilogue thread owns one entry and forms
// sum_j (w qs)[q,j] ReLU(D[s,(q,j)]) * ks[s] in registers (ReLU commutes with the
// positive scales): no cross-thread reduction.
//
// A pipeline stage holds TPS tiles of 128 entries (two for one query per unit,
// one for four): on sm_100a a thread's first shared-memory access after issuing
// tcgen05 operations costs a few hundred cycles, so the MMA warp's two waits per
// stage are amortised over 4 x TPS MMAs.
//
// Persistent, warp-specialised CTA (320 threads):
//   warp 0  TMA producer: per stage one 2-D box of 128 TPS key rows (128-byte
//           swizzle) and their fp32 key scales into an S-stage ring; per work unit
//           the query group (64 QG x 128 B), its head weights and query scales
//           into one of two buffers.  Decode with bf16 index queries: the
//           epilogue warps quantise each unit's 64 query rows (FP8, one scale per
//           row) into the buffer, a unit ahead, and the producer brings only the
//           head weights, so that only the key stage holding the entry the
//           preceding kernel writes waits for that kernel;
//   warp 1  MMA issuer (one thread): 4 TPS x tcgen05.mma kind::f8f6f4 per stage
//           into one of NACC TMEM accumulators;
//   warps 2-9 epilogue, two warpgroups taking alternate stages (warps w and w+4
//           share a TMEM lane quarter), so one group's TMEM loads overlap the
//           other's arithmetic: tcgen05.ld of the accumulator, the weighted ReLU
//           sum (weights in registers for one query, 128-bit shared loads for
//           four), the causal mask, bf16 / fp32 store; stages no query of the
//           group can see are written as -inf without any MMA.
// Every operand the epilogue needs arrives by TMA with its stage, so no thread
// waits on global memory inside the loop.  A stage is released when the MMAs
// have read the keys and the four epilogue warps of its group have read the key
// scales.  A work unit is (sequence, query group, chunk of stages); units are
// dealt round-robin to the CTAs and their causal extents are computed once.
#include "kernels.h"
#include "tc_common.cuh"

#include <climits>

namespace csa {

namespace {

constexpr int kTileE = 128;          // entries per tile (MMA M)
constexpr int kHeads = 64;           // index heads
constexpr int kDim = 128;            // index dim (bytes per FP8 row)
constexpr int kTileBytes = kTileE * kDim;
constexpr int kMaxLocalUnits = 256;  // units one CTA walks (grid is sized to respect it)
constexpr int kPagedSlots = 1024;    // page ids of the stages a CTA loads, kept in shared memory
constexpr int kEpiGroups = 2;        // epilogue warpgroups, alternating stages
constexpr int kThreads = 64 + 128 * kEpiGroups;

struct IdxTc {
  void* scores;
  const int32_t* q_pos;
  int* err;
  int T, E_cap, E, m;
  int n_qg, tiles, stages, chunk, n_chunks, units;
  int score_f32;
  int all_visible;   // every query sees all E entries: q_pos is not read
  int dep_stage;     // stages >= dep_stage hold entries the preceding kernel writes
  const int32_t* block_table;   // paged keys (one query per sequence: a stage is one page)
  int max_pages, num_pages;
  int pos_input;     // q_pos is an input: read before the wait; per-sequence dependent stage
  const __nv_bfloat16* q_raw;   // QG = 1: bf16 index queries quantised here (else q by TMA)
};

// Raw index queries (bf16 [row][128]) of one warp's 8 rows r0 .. r0 + 7, four lanes per
// row: lane l holds row r0 + l / 4, elements 32 (l % 4) .. 32 (l % 4) + 31.
struct QRows { uint4 v[4]; };
__device__ __forceinline__ void qrows_load(QRows& q, const __nv_bfloat16* row0, int lane) {
  const uint4* src = reinterpret_cast<const uint4*>(row0 + (size_t)(lane >> 2) * kDim) + (lane & 3) * 4;
#pragma unroll
  for (int j = 0; j < 4; ++j) q.v[j] = __ldg(src + j);
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// FP8 quantisation of those rows (scale = amax / 448 per row, code = e4m3(x / scale), the
// arithmetic of the stand-alone quantiser) into the 128-byte-swizzled B tile and the row
// scales.  The code loop is rolled (it runs a few times per CTA, so its code is fetched
// once); the register rows move to the front instead of being indexed.
__device__ __noinline__ void qrows_quantise(QRows q, uint8_t* tile, float* scales, int r0, int lane) {
  float am = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t w[4] = {q.v[j].x, q.v[j].y, q.v[j].z, q.v[j].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) am = fmaxf(am, fmaxf(fabsf(bf16_lo(w[e])), fabsf(bf16_hi(w[e]))));
  }
  am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
  am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
  const float sc = am / 448.f;
  const int row = r0 + (lane >> 2), qq = lane & 3;
#pragma unroll 1
  for (int j = 0; j < 4; ++j) {   // eight elements -> eight codes
    const uint32_t w[4] = {q.v[0].x, q.v[0].y, q.v[0].z, q.v[0].w};
    uint32_t c2[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t lo = sc > 0.f ? (uint32_t)f32_to_e4m3(bf16_lo(w[e]) / sc) : 0u;
      const uint32_t hi = sc > 0.f ? (uint32_t)f32_to_e4m3(bf16_hi(w[e]) / sc) : 0u;
      c2[e >> 1] |= (lo | (hi << 8)) << (16 * (e & 1));
    }
    const int chunk = 2 * qq + (j >> 1);   // 16-byte chunk of the row
    *reinterpret_cast<uint2*>(tile + row * 128 + ((chunk ^ (row & 7)) << 4) + (j & 1) * 8) =
        make_uint2(c2[0], c2[1]);
    q.v[0] = q.v[1]; q.v[1] = q.v[2]; q.v[2] = q.v[3];
  }
  if (qq == 0) scales[row] = sc;
}

template <int QG>
struct Layout {
  static constexpr int N = kHeads * QG;
  static constexpr int TPS = QG == 1 ? 2 : 1;          // tiles per stage
  static constexpr int kStageE = kTileE * TPS;
  static constexpr int NACC = QG == 1 ? 4 : 2;
  static constexpr int kAccCols = TPS * N;
  static constexpr int kStageKeyB = TPS * kTileBytes;
  static constexpr int kQBytes = N * kDim;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(NACC * kAccCols <= 512, "TMEM budget");
};

template <int QG, int S>
__global__ void __launch_bounds__(kThreads, 1)
index_scores_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmKS, const __grid_constant__ CUtensorMap tmW,
                       const __grid_constant__ CUtensorMap tmQS, IdxTc p) {
  using LY = Layout<QG>;
  constexpr int N = LY::N;
  constexpr int TPS = LY::TPS;
  constexpr int NACC = LY::NACC;
  constexpr int kQBytes = LY::kQBytes;
  constexpr int kStageE = LY::kStageE;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = base;                                           // S x TPS x 16 KB key tiles
  float* sKS = reinterpret_cast<float*>(sA + S * LY::kStageKeyB);   // S x kStageE key scales
  uint8_t* sB = reinterpret_cast<uint8_t*>(sKS + S * kStageE);  // 2 x kQBytes query groups
  float* sW = reinterpret_cast<float*>(sB + 2 * kQBytes);       // 2 x N head weights
  float* sQS = sW + 2 * N;                                      // 2 x N query scales
  uint64_t* bars = reinterpret_cast<uint64_t*>(sQS + 2 * N);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* bfull = bars + 2 * S;
  uint64_t* bempty = bfull + 2;
  uint64_t* tfull = bempty + 2;
  uint64_t* tempty = tfull + NACC;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + NACC);
  float* s_wq = reinterpret_cast<float*>(tmem_holder + 4);    // [kEpiGroups][N] w * qs of the unit
  int* s_vis = reinterpret_cast<int*>(s_wq + kEpiGroups * N); // [kMaxLocalUnits] visible stages
  int* s_ev = s_vis + kMaxLocalUnits;                         // [kMaxLocalUnits][QG] visible entries
  int* s_pg = s_ev + kMaxLocalUnits * QG;                     // [kPagedSlots] page of each stage

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  pdl_launch_dependents();
  // raw index queries: the epilogue warps fetch their rows of the CTA's first unit now, so
  // that the memory round trip overlaps the set-up (an input of the call)
  QRows qfirst;
  if (QG == 1 && p.q_raw && warp >= 2 && (int)blockIdx.x < p.units) {
    const int sb0 = ((int)blockIdx.x / p.n_chunks) / p.n_qg, g0 = ((int)blockIdx.x / p.n_chunks) % p.n_qg;
    qrows_load(qfirst, p.q_raw + ((size_t)(sb0 * p.T + g0 * QG) * kHeads + 8 * (warp - 2)) * kDim, lane);
  }
  if (p.block_table) {
    // page ids of every stage of every unit this CTA walks, [local unit][stage of the
    // chunk]: inputs of the call, fetched at once while the CTA sets up instead of one
    // dependent load before each stage's copy
    const int nloc = min(kMaxLocalUnits, (p.units - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x);
    for (int x = threadIdx.x; x < nloc * p.chunk && x < kPagedSlots; x += blockDim.x) {
      const int i = x / p.chunk, j = x % p.chunk;
      const int u = blockIdx.x + i * gridDim.x;
      const int sb = (u / p.n_chunks) / p.n_qg;
      const int js = (u % p.n_chunks) * p.chunk + j;
      s_pg[x] = js < p.max_pages ? p.block_table[(size_t)sb * p.max_pages + js] : -1;
    }
  }
  if (!p.all_visible && !p.pos_input) pdl_wait();   // the positions come from the preceding kernel

  // causal extent of every unit this CTA will walk
  for (int i = threadIdx.x; i * (int)gridDim.x + (int)blockIdx.x < p.units && i < kMaxLocalUnits;
       i += blockDim.x) {
    const int u = blockIdx.x + i * gridDim.x;
    const int tmp = u / p.n_chunks;
    const int g = tmp % p.n_qg, sb = tmp / p.n_qg;
    const int nq = min(QG, p.T - g * QG);
    int evmax = 0;
    for (int q = 0; q < QG; ++q) {
      const int ev = q >= nq ? 0 : p.all_visible ? p.E
                   : visible_entries(p.q_pos[(size_t)sb * p.T + g * QG + q], p.m, p.E);
      s_ev[i * QG + q] = ev;
      evmax = max(evmax, ev);
    }
    s_vis[i] = (evmax + kStageE - 1) / kStageE;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { tc::mbar_init(&full[i], 1); tc::mbar_init(&empty[i], 1 + 4); }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bfull[i], 1 + (p.q_raw ? 4 * kEpiGroups : 0));
      tc::mbar_init(&bempty[i], 1 + 4 * kEpiGroups);
    }
    for (int i = 0; i < NACC; ++i) { tc::mbar_init(&tfull[i], 1); tc::mbar_init(&tempty[i], 4); }
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&tmK);
    tc::tma_prefetch_desc(&tmQ);
    tc::tma_prefetch_desc(&tmKS);
  }
  if (warp == 0) tc::tmem_alloc(tmem_holder, LY::kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // per-unit geometry shared by all roles: stages [js0, js1), the first nc computed
  auto unit = [&](int u, int i, int& sb, int& g, int& js0, int& js1, int& nc, int& nq) {
    const int ch = u % p.n_chunks;
    const int tmp = u / p.n_chunks;
    g = tmp % p.n_qg;
    sb = tmp / p.n_qg;
    js0 = ch * p.chunk;
    js1 = min(p.stages, js0 + p.chunk);
    nq = min(QG, p.T - g * QG);
    nc = max(0, min(js1, s_vis[i]) - js0);
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    // (lane 0 issues the copies; with raw index queries the whole warp quantises them)
    auto load_stage = [&](int slot, int sb, int js, int li) {
      int row0 = sb * p.E_cap + js * kStageE;
      if (p.block_table) {
        const uint32_t fl = (uint32_t)(li * p.chunk + js % p.chunk);
        const int pg = fl < (uint32_t)kPagedSlots ? s_pg[fl]
                                                    : p.block_table[(size_t)sb * p.max_pages + js];
        row0 = ((unsigned)pg < (unsigned)p.num_pages ? pg : 0) * kStageE;
      }
      tc::mbar_arrive_expect_tx(&full[slot], LY::kStageKeyB + kStageE * 4);
      tc::tma_load_2d(sA + slot * LY::kStageKeyB, &tmK, 0, row0, &full[slot]);
      tc::tma_load_1d(sKS + slot * kStageE, &tmKS, row0, &full[slot]);
    };
    // first stage of sequence sb holding an entry the preceding kernel writes
    auto dep_of = [&](int sb) {
      if (!p.pos_input) return p.dep_stage;
      const int t = p.q_pos[sb];   // the stage holding the entry the new token completes
      return (t + 1) % p.m == 0 ? ((t + 1) / p.m - 1) / kStageE : INT_MAX;
    };
    // Key stages the preceding kernel does not write are fetched before waiting on it,
    // into the first free slots, so that HBM streaming overlaps that kernel.
    uint32_t npre = 0;
    if (lane == 0) {
      for (int u = blockIdx.x, i = 0; u < p.units && npre == 0; u += gridDim.x, ++i) {
        int sb, g, js0, js1, nc, nq;
        unit(u, i, sb, g, js0, js1, nc, nq);
        if (nc == 0) continue;
        const int dep = dep_of(sb);
        for (int js = js0; js < js0 + nc && (int)npre < S && js < dep; ++js, ++npre)
          load_stage(npre, sb, js, i);
        break;
      }
    }
    npre = __shfl_sync(0xffffffffu, npre, 0);
    // quantised queries from the preceding kernel: wait for it before the first unit
    bool waited = p.q_raw == nullptr;
    if (waited) pdl_wait();
    uint32_t it = 0, ul = 0;
    bool ok = true;
    for (int u = blockIdx.x, i = 0; u < p.units && ok; u += gridDim.x, ++i) {
      int sb, g, js0, js1, nc, nq;
      unit(u, i, sb, g, js0, js1, nc, nq);
      if (nc == 0) continue;
      const int bb = ul & 1;
      if (lane == 0) ok = tc::mbar_wait(&bempty[bb], ((ul >> 1) & 1) ^ 1, p.err);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      const int qrow0 = (sb * p.T + g * QG) * kHeads;
      if (p.q_raw) {                  // the codes and scales come from the epilogue warps
        if (lane == 0) {
          tc::mbar_arrive_expect_tx(&bfull[bb], N * 4);
          tc::tma_load_1d(sW + bb * N, &tmW, qrow0, &bfull[bb]);
        }
      } else if (lane == 0) {
        tc::mbar_arrive_expect_tx(&bfull[bb], kQBytes + 2 * N * 4);
        tc::tma_load_2d(sB + bb * kQBytes, &tmQ, 0, qrow0, &bfull[bb]);
        tc::tma_load_1d(sW + bb * N, &tmW, qrow0, &bfull[bb]);
        tc::tma_load_1d(sQS + bb * N, &tmQS, qrow0, &bfull[bb]);
      }
      const int dep = waited ? INT_MAX : dep_of(sb);
      for (int js = js0; js < js0 + nc; ++js, ++it) {
        if (it < npre) continue;                       // fetched before the wait
        if (js >= dep && !waited) {                    // this stage holds an entry the
          pdl_wait();                                  // preceding kernel writes
          waited = true;
        }
        const int s = it % S;
        if (lane == 0) {
          ok = tc::mbar_wait(&empty[s], ((it / S) & 1) ^ 1, p.err);
          if (ok) load_stage(s, sb, js, i);
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
      ++ul;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = tc::instr_desc(kTileE, N, 0, 0, 0, 0);   // e4m3 x e4m3 -> f32
      uint32_t it = 0, ul = 0;
      bool ok = true;
      for (int u = blockIdx.x, i = 0; u < p.units && ok; u += gridDim.x, ++i) {
        int sb, g, js0, js1, nc, nq;
        unit(u, i, sb, g, js0, js1, nc, nq);
        if (nc == 0) continue;
        const int bb = ul & 1;
        ok = tc::mbar_wait(&bfull[bb], (ul >> 1) & 1, p.err);
        if (!ok) break;
        const uint64_t bdesc = tc::smem_desc_sw128(tc::smem_u32(sB + bb * kQBytes), 16, 1024);
        for (int j = 0; j < nc; ++j, ++it) {
          const int s = it % S;
          const int acc = it % NACC;
          // both waits back to back: the first shared-memory access after the previous
          // stage's tcgen05 operations carries the cost, the second is cheap
          ok = tc::mbar_wait(&full[s], (it / S) & 1, p.err) &&
               tc::mbar_wait(&tempty[acc], ((it / NACC) & 1) ^ 1, p.err);
          if (!ok) break;
          tc::tc_fence_after();
#pragma unroll
          for (int t = 0; t < TPS; ++t) {
            const uint64_t adesc =
                tc::smem_desc_sw128(tc::smem_u32(sA + s * LY::kStageKeyB + t * kTileBytes), 16, 1024);
            const uint32_t d = tmem_base + acc * LY::kAccCols + t * N;
#pragma unroll
            for (int kk = 0; kk < kDim / 32; ++kk)   // K = 32 bytes of E4M3 per MMA
              tc::mma_f8f6f4(d, adesc + 2 * kk, bdesc + 2 * kk, idesc, kk > 0);
          }
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
    const int ew = warp - 2;                 // 0..7
    const int grp = ew >> 2;                 // warpgroup: takes stages with c % 2 == grp
    const int lane_base = (warp & 3) * 32;   // TMEM lanes this warp may access
    const int gtid = (ew & 3) * 32 + lane;   // 0..127 within the group
    float* my_wq = s_wq + grp * N;
    float wq1[QG == 1 ? kHeads : 1];         // one query: its 64 weights live in registers
    uint32_t c = 0, ul = 0;                  // computed stages seen, units with work seen
    bool ok = true;
    // raw index queries: this warp's 8 rows of the unit with work `nth` after (u, i), into
    // buffer bb once its previous use is over (QG = 1)
    auto quantise_unit = [&](int u, int i, int nth, uint32_t unit_no) {
      for (; u < p.units; u += gridDim.x, ++i) {
        int sb, g, js0, js1, nc, nq;
        unit(u, i, sb, g, js0, js1, nc, nq);
        if (nc == 0) continue;
        if (nth-- > 0) continue;
        const int bb = unit_no & 1;
        ok = ok && tc::mbar_wait(&bempty[bb], ((unit_no >> 1) & 1) ^ 1, p.err);
        const int r0 = 8 * ew;
        QRows q = qfirst;                              // fetched at kernel start
        if (u != (int)blockIdx.x)
          qrows_load(q, p.q_raw + ((size_t)(sb * p.T + g * QG) * kHeads + r0) * kDim, lane);
        qrows_quantise(q, sB + bb * kQBytes, sQS + bb * N, r0, lane);
        tc::fence_proxy_async();   // the MMA reads the codes through the async proxy
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bfull[bb]);
        return;
      }
    };
    if (QG == 1 && p.q_raw) {        // the first two units' queries, one per buffer
      quantise_unit(blockIdx.x, 0, 0, 0);
      quantise_unit(blockIdx.x, 0, 1, 1);
    }
    for (int u = blockIdx.x, i = 0; u < p.units; u += gridDim.x, ++i) {
      int sb, g, js0, js1, nc, nq;
      unit(u, i, sb, g, js0, js1, nc, nq);
      if (nc > 0) {
        const int bb = ul & 1;
        // the queries of the unit after this one, into the buffer the previous unit freed
        if (QG == 1 && p.q_raw && ul >= 1) quantise_unit(u, i, 1, ul + 1);
        tc::named_bar(1 + grp, 128);                   // previous unit's my_wq no longer read
        ok = ok && tc::mbar_wait(&bfull[bb], (ul >> 1) & 1, p.err);
        for (int x = gtid; x < N; x += 128) my_wq[x] = sW[bb * N + x] * sQS[bb * N + x];
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bempty[bb]);
        tc::named_bar(1 + grp, 128);
        if constexpr (QG == 1) {
#pragma unroll
          for (int h = 0; h < kHeads; h += 4) {
            const float4 w4 = *reinterpret_cast<const float4*>(my_wq + h);
            wq1[h] = w4.x; wq1[h + 1] = w4.y; wq1[h + 2] = w4.z; wq1[h + 3] = w4.w;
          }
        }
        ++ul;
      }
      for (int js = js0; js < js1; ++js) {
        float sc[TPS][QG];
#pragma unroll
        for (int t = 0; t < TPS; ++t)
#pragma unroll
          for (int q = 0; q < QG; ++q) sc[t][q] = -INFINITY;
        if (js < js0 + nc) {
          const uint32_t cc = c++;
          if ((int)(cc & 1) != grp) continue;           // the other warpgroup's stage
          if (ok) {
            const int s = cc % S;
            const int acc = cc % NACC;
            ok = tc::mbar_wait(&full[s], (cc / S) & 1, p.err);   // the stage's key scales landed
            float ks[TPS];
#pragma unroll
            for (int t = 0; t < TPS; ++t) ks[t] = sKS[s * kStageE + t * kTileE + lane_base + lane];
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&empty[s]);
            ok = ok && tc::mbar_wait(&tfull[acc], (cc / NACC) & 1, p.err);
            tc::tc_fence_after();
#pragma unroll
            for (int t = 0; t < TPS; ++t) {
#pragma unroll
              for (int q = 0; q < QG; ++q) {
                uint32_t r0[32], r1[32];
                const uint32_t ta = tmem_base + ((uint32_t)lane_base << 16) + acc * LY::kAccCols +
                                    t * N + q * kHeads;
                tc::tmem_ld32(ta, r0);
                tc::tmem_ld32(ta + 32, r1);
                tc::tmem_ld_wait(r0);
                tc::reg_fence(r1);
                float a[4] = {0.f, 0.f, 0.f, 0.f};
                if constexpr (QG == 1) {
#pragma unroll
                  for (int h = 0; h < 32; ++h) {
                    a[h & 3] = fmaf(wq1[h], fmaxf(__uint_as_float(r0[h]), 0.f), a[h & 3]);
                    a[h & 3] = fmaf(wq1[32 + h], fmaxf(__uint_as_float(r1[h]), 0.f), a[h & 3]);
                  }
                } else {
                  const float4* w4p = reinterpret_cast<const float4*>(my_wq + q * kHeads);
#pragma unroll
                  for (int h4 = 0; h4 < 8; ++h4) {
                    const float4 wa = w4p[h4], wb = w4p[8 + h4];
                    a[0] = fmaf(wa.x, fmaxf(__uint_as_float(r0[4 * h4]), 0.f), a[0]);
                    a[1] = fmaf(wa.y, fmaxf(__uint_as_float(r0[4 * h4 + 1]), 0.f), a[1]);
                    a[2] = fmaf(wa.z, fmaxf(__uint_as_float(r0[4 * h4 + 2]), 0.f), a[2]);
                    a[3] = fmaf(wa.w, fmaxf(__uint_as_float(r0[4 * h4 + 3]), 0.f), a[3]);
                    a[0] = fmaf(wb.x, fmaxf(__uint_as_float(r1[4 * h4]), 0.f), a[0]);
                    a[1] = fmaf(wb.y, fmaxf(__uint_as_float(r1[4 * h4 + 1]), 0.f), a[1]);
                    a[2] = fmaf(wb.z, fmaxf(__uint_as_float(r1[4 * h4 + 2]), 0.f), a[2]);
                    a[3] = fmaf(wb.w, fmaxf(__uint_as_float(r1[4 * h4 + 3]), 0.f), a[3]);
                  }
                }
                sc[t][q] = ((a[0] + a[1]) + (a[2] + a[3])) * ks[t];
              }
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&tempty[acc]);
          }
        } else if ((js & 1) != grp) {
          continue;                                     // fills alternate between the groups
        }
#pragma unroll
        for (int t = 0; t < TPS; ++t) {
          const int e = (js * TPS + t) * kTileE + lane_base + lane;
          if (e < p.E) {
#pragma unroll
            for (int q = 0; q < QG; ++q) {
              if (q >= nq) break;
              const int ev = s_ev[i * QG + q];
              const float v = !ok ? __int_as_float(0x7fc00000) : (e < ev ? sc[t][q] : -INFINITY);
              const size_t o = ((size_t)sb * p.T + g * QG + q) * p.E + e;
              if (p.score_f32) reinterpret_cast<float*>(p.scores)[o] = v;
              else reinterpret_cast<__nv_bfloat16*>(p.scores)[o] = __float2bfloat16_rn(v);
            }
          }
        }
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem_base, LY::kTmemCols);
  }
}

template <int QG, int S>
csa_status launch_qg(const IndexArgs& a, int b, cudaStream_t st) {
  using LY = Layout<QG>;
  CUtensorMap tmK, tmQ, tmKS, tmW, tmQS;
  const uint64_t qrows = (uint64_t)b * a.T * kHeads;
  const uint64_t krows = a.block_table ? (uint64_t)a.num_pages * kPageEntries : (uint64_t)b * a.E_cap;
  if (!make_tmap_2d_u8(&tmK, a.k, kDim, krows, kDim, LY::kStageE) ||
      !make_tmap_1d_f32(&tmKS, a.k_scales, krows, LY::kStageE) ||
      !make_tmap_1d_f32(&tmW, a.w, qrows, LY::N))
    return CSA_ERR_CUDA;
  if (a.q_raw) {           // quantised in the kernel: the query maps are not read
    tmQ = tmK;
    tmQS = tmKS;
  } else if (!make_tmap_2d_u8(&tmQ, a.q, kDim, qrows, kDim, LY::N) ||
             !make_tmap_1d_f32(&tmQS, a.q_scales, qrows, LY::N)) {
    return CSA_ERR_CUDA;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  IdxTc p{};
  p.scores = a.scores; p.q_pos = a.q_pos;
  p.err = device_error_word();
  if (!p.err) return CSA_ERR_CUDA;
  p.T = a.T; p.E_cap = a.E_cap; p.E = a.E; p.m = a.m;
  p.n_qg = (a.T + QG - 1) / QG;
  p.tiles = (a.E + kTileE - 1) / kTileE;
  p.stages = (p.tiles + LY::TPS - 1) / LY::TPS;
  const long long groups = (long long)b * p.n_qg;
  // split each query group's stages into chunks so that there are at least ~2 units per SM
  int nch = (int)((2LL * sms + groups - 1) / groups);
  nch = max(1, min(nch, p.stages));
  p.chunk = (p.stages + nch - 1) / nch;
  p.n_chunks = (p.stages + p.chunk - 1) / p.chunk;
  const long long units = groups * p.n_chunks;
  if (units > 0x7fffffff) return CSA_ERR_UNSUPPORTED;
  p.units = (int)units;
  p.score_f32 = a.score_dtype == CSA_F32;
  p.all_visible = a.all_visible;
  p.dep_stage = a.dep_entry < 0 ? 0 : a.dep_entry / LY::kStageE;
  p.block_table = a.block_table; p.max_pages = a.max_pages; p.num_pages = a.num_pages;
  p.pos_input = a.pos_input;
  p.q_raw = reinterpret_cast<const __nv_bfloat16*>(a.q_raw);
  long long grid = units < sms ? units : sms;
  const long long min_grid = (units + kMaxLocalUnits - 1) / kMaxLocalUnits;
  if (grid < min_grid) grid = min_grid;
  const size_t smem = 1024 + (size_t)S * (LY::kStageKeyB + LY::kStageE * 4) + 2 * (size_t)LY::kQBytes +
                      4 * (size_t)LY::N * 4 + (2 * S + 4 + 2 * LY::NACC) * 8 + 16 +
                      kEpiGroups * (size_t)LY::N * 4 + (size_t)kMaxLocalUnits * (1 + QG) * 4 +
                      (size_t)kPagedSlots * 4;
  auto kern = index_scores_tc_kernel<QG, S>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return CSA_ERR_CUDA;
  if (csa_launch(kern, dim3((unsigned)grid), dim3(kThreads), smem, st, a.pdl != 0, tmK, tmQ, tmKS,
                 tmW, tmQS, p) != cudaSuccess)
    return CSA_ERR_CUDA;
  return CSA_OK;
}

}  // namespace

csa_status launch_index_scores_tc(const IndexArgs& a, int b, cudaStream_t st) {
  if (a.qk_dtype != CSA_FP8_E4M3 || a.H != kHeads || a.d != kDim) return CSA_ERR_UNSUPPORTED;
  if (a.block_table && (a.T != 1 || Layout<1>::kStageE != kPageEntries)) return CSA_ERR_UNSUPPORTED;
  if (a.q_raw && a.T != 1) return CSA_ERR_UNSUPPORTED;
  const void* qp = a.q_raw ? a.q_raw : a.q;
  const void* qsp = a.q_raw ? a.k_scales : a.q_scales;
  if ((reinterpret_cast<uintptr_t>(a.k) & 15) || (reinterpret_cast<uintptr_t>(qp) & 15) ||
      (reinterpret_cast<uintptr_t>(a.k_scales) & 15) || (reinterpret_cast<uintptr_t>(a.w) & 15) ||
      (reinterpret_cast<uintptr_t>(qsp) & 15) || (a.E_cap % 4))
    return CSA_ERR_INVALID_ARG;   // the TMA copies need 16-byte aligned rows and scale runs
  if (a.T >= 4) return launch_qg<4, 4>(a, b, st);
  return launch_qg<1, 5>(a, b, st);
}

}  // namespace csa
