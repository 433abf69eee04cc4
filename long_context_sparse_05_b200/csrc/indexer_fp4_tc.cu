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
// four columns hold the four UE4M3 scales of rows 0-31, 32-63, 64-95, 96-127,
// replicated in all four lane quarters (the layout tcgen05.cp 32x128b.warpx4 makes).
// The key cache keeps its scales in exactly that order (tiles of 128 entries, see
// nvfp4_key_scale_offset), so a stage's scales go from HBM to shared memory in
// one bulk copy and on to TMEM without any rearrangement.  Query scales arrive
// row-major and are rearranged once per work unit (tcgen05.cp by the MMA warp).
// Key scales are written into TMEM by the epilogue warps (tcgen05.st, each warp its
// lane quarter) rather than by tcgen05.cp: on sm_100a the MMA thread's shared-memory
// accesses after tcgen05 operations wait for the tensor pipe, so every copy in
// the MMA thread's stream lengthens each stage, while the epilogue warps have room.
//
// Pipeline granularity: a stage is two tiles (256 entries, 16 KB of codes + 2 KB
// of scales), so the MMA warp pays one round of barrier waits per four MMAs.
//
// CTA (480 threads), one query per work unit (decode):
//   warp 0  producer: per stage one 2-D TMA box of 256 key rows and one bulk copy
//           of the stage's scales; per unit the query codes (TMA), its raw scales
//           and head weights;
//   warp 1  query-scale rearrangement (all lanes, once per unit) and MMA issue
//           (lane 0): 4 MMAs per stage into one of NACC accumulators of 2 x 64
//           columns, each with its own 16 key-scale columns.  Per stage it touches
//           no shared memory: on sm_100a a warp's shared-memory access after its own
//           tcgen05 operations waits for the tensor pipe, so the stage barriers are
//           polled by warp 14, which hands each ready stage over at a named barrier
//           (a barrier reduction also carries a failed wait);
//   warps 2-13 epilogue, three warpgroups, group g taking the stages s with
//           s % 3 == g, i.e. accumulator g (one consumer per accumulator barrier):
//           tcgen05.ld, weighted ReLU head sum with the weights read as broadcast
//           128-bit shared loads, causal mask, store; then the key scales of the
//           group's next stage (three ahead, same accumulator) into its scale
//           columns.  tempty[a] thus means "accumulator a is free and holds the
//           scales of its next stage"; its phase k belongs to stage a + 3k, and the
//           scales of stages 0-2 are written up front.
#include "kernels.h"
#include "tc_common.cuh"

#include <climits>

namespace csa {

namespace {

constexpr int kTileE = 128;
constexpr int kTPS = 2;                          // tiles per stage
constexpr int kStageE = kTileE * kTPS;           // 256 entries
constexpr int kHeads = 64;
constexpr int kDim = 128;                        // elements per row
constexpr int kRowB = 64;                        // bytes per FP4 row
constexpr int kSfTileB = 1024;                   // scale bytes of one tile (tiled layout)
constexpr int kKeyB = kStageE * kRowB;           // 16 KB
constexpr int kStage = kKeyB + kTPS * kSfTileB;  // 18 KB, a multiple of 1 KB
constexpr int kQBytes = kHeads * kRowB;          // 4 KB
constexpr int kQSf = kHeads * 8;                 // 512 B raw query scales
constexpr int kPermBytes = 2 * 512;              // query scales in the tcgen05.cp layout
constexpr int NACC = 3;                          // accumulators of kTPS x 64 columns
constexpr int S = 8;                             // stages
constexpr int kMaxLocalUnits = 256;
constexpr int kPagedSlots = 1024;    // page ids of the stages a CTA loads, kept in shared memory
constexpr int kEpiGroups = 3;                    // one epilogue warpgroup per accumulator
constexpr int kThreads = 96 + 128 * kEpiGroups;   // producer, MMA, 12 epilogue, waiter
constexpr int kWaitWarp = kThreads / 32 - 1;       // warp 14
static_assert(NACC == kEpiGroups, "each accumulator has its own epilogue warpgroup");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = kTPS * kHeads;     // 128
constexpr uint32_t kSfaCol = NACC * kAccCols;    // 384: NACC x (kTPS x 8) key-scale columns
constexpr uint32_t kSfbCol = kSfaCol + NACC * kTPS * 8;   // 432: 2 x 8 query-scale columns
static_assert(kSfbCol + 16 <= kTmemCols, "TMEM budget");
static_assert(kStage % 1024 == 0, "stages must keep the swizzle alignment");
static_assert(kStageE == kPageEntries, "a stage of the paged key cache is one page");

struct IdxFp4 {
  void* scores;
  const int32_t* q_pos;
  const uint8_t* k_scales;
  int* err;
  int T, E_cap, E, m;
  int tiles, sf_tiles_cap, stages, chunk, n_chunks, units;
  int score_f32;
  int all_visible;   // every query sees all E entries: q_pos is not read
  int dep_stage;     // stages >= dep_stage hold entries the preceding kernel writes
  const int32_t* block_table;   // paged keys (one query per sequence: a stage is one page)
  int max_pages, num_pages;
  int pos_input;     // q_pos is an input: read before the wait; per-sequence dependent stage
};

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

// 16 consecutive 32-bit TMEM columns of this warp's lane quarter from registers.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
        "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
        "r"(r[14]), "r"(r[15]) : "memory");
}

// Untiled bulk copy global -> shared; completion counted on `bar` as transaction bytes.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(tc::smem_u32(dst)), "l"(src), "r"(bytes), "r"(tc::smem_u32(bar)) : "memory");
}

// Lane m0 of the warp rearranges the row-major query scales (8 bytes per row, `rows`
// rows) into the tcgen05.cp order for both K blocks: word (m0, m1) of block kb =
// raw word (m0 + 32 m1) * 2 + kb.
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

__global__ void __launch_bounds__(kThreads, 1)
index_scores_fp4_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmQS, const __grid_constant__ CUtensorMap tmW,
                        IdxFp4 p) {
  constexpr int N = kHeads;
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
  int* s_vis = reinterpret_cast<int*>(tmem_holder + 4);      // [kMaxLocalUnits] visible stages
  int* s_ev = s_vis + kMaxLocalUnits;                         // [kMaxLocalUnits] visible entries
  int* s_pg = s_ev + kMaxLocalUnits;                          // [kPagedSlots] page of each stage

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  pdl_launch_dependents();
  if (p.block_table) {
    // page ids of every stage of every unit this CTA walks, [local unit][stage of the
    // chunk]: inputs of the call, fetched at once while the CTA sets up instead of one
    // dependent load before each stage's copy
    const int nloc = min(kMaxLocalUnits, (p.units - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x);
    for (int x = threadIdx.x; x < nloc * p.chunk && x < kPagedSlots; x += blockDim.x) {
      const int i = x / p.chunk, j = x % p.chunk;
      const int u = blockIdx.x + i * gridDim.x;
      const int sb = u / p.n_chunks;
      const int js = (u % p.n_chunks) * p.chunk + j;
      s_pg[x] = js < p.max_pages ? p.block_table[(size_t)sb * p.max_pages + js] : -1;
    }
  }
  if (!p.all_visible && !p.pos_input) pdl_wait();   // the positions come from the preceding kernel

  for (int i = threadIdx.x; i * (int)gridDim.x + (int)blockIdx.x < p.units && i < kMaxLocalUnits;
       i += blockDim.x) {
    const int u = blockIdx.x + i * gridDim.x;
    const int row = u / p.n_chunks;
    const int ev = p.all_visible ? p.E : visible_entries(p.q_pos[row], p.m, p.E);
    s_ev[i] = ev;
    s_vis[i] = (ev + kStageE - 1) / kStageE;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { tc::mbar_init(&full[i], 1); tc::mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bfull[i], 1);
      tc::mbar_init(&bempty[i], 1 + 4 * kEpiGroups);
    }
    for (int i = 0; i < NACC; ++i) { tc::mbar_init(&tfull[i], 1); tc::mbar_init(&tempty[i], 4); }
    tc::fence_barrier_init();
    tc::tma_prefetch_desc(&tmK);
  }
  if (warp == 0) tc::tmem_alloc(tmem_holder, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // stages [js0, js1) of row `row`; the first nc of them are visible and computed
  auto unit = [&](int u, int i, int& row, int& js0, int& js1, int& nc) {
    row = u / p.n_chunks;
    const int ch = u % p.n_chunks;
    js0 = ch * p.chunk;
    js1 = min(p.stages, js0 + p.chunk);
    nc = max(0, min(js1, s_vis[i]) - js0);
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      const int sf_seq = p.sf_tiles_cap;
      auto load_stage = [&](int slot, int row, int js, int li) {
        const int sb = row / p.T;
        const int j0 = js * kTPS;                                // first tile of the stage
        const int nsf = min(kTPS, sf_seq - j0);                  // scale tiles inside the sequence
        uint8_t* st = sStage + slot * kStage;
        if (p.block_table) {
          // a stage is one page: its keys and its whole scale tiles
          const uint32_t fl = (uint32_t)(li * p.chunk + js % p.chunk);
          const int pg0 = fl < (uint32_t)kPagedSlots ? s_pg[fl]
                                                       : p.block_table[(size_t)sb * p.max_pages + js];
          const int pg = (unsigned)pg0 < (unsigned)p.num_pages ? pg0 : 0;
          tc::mbar_arrive_expect_tx(&full[slot], kKeyB + kTPS * kSfTileB);
          tc::tma_load_2d(st, &tmK, 0, pg * kStageE, &full[slot]);
          bulk_load(st + kKeyB, p.k_scales + (size_t)pg * kTPS * kSfTileB, kTPS * kSfTileB,
                    &full[slot]);
          return;
        }
        tc::mbar_arrive_expect_tx(&full[slot], kKeyB + nsf * kSfTileB);
        tc::tma_load_2d(st, &tmK, 0, sb * p.E_cap + j0 * kTileE, &full[slot]);
        bulk_load(st + kKeyB, p.k_scales + ((size_t)sb * sf_seq + j0) * kSfTileB,
                  nsf * kSfTileB, &full[slot]);
      };
      // key stages the preceding kernel does not write are fetched before waiting on it
      uint32_t npre = 0;
      for (int u = blockIdx.x, i = 0; u < p.units && npre == 0; u += gridDim.x, ++i) {
        int row, js0, js1, nc;
        unit(u, i, row, js0, js1, nc);
        if (nc == 0) continue;
        int dep = p.dep_stage;
        if (p.pos_input) {   // the stage holding the entry the sequence's new token completes
          const int t = p.q_pos[row];
          dep = (t + 1) % p.m == 0 ? ((t + 1) / p.m - 1) / kStageE : INT_MAX;
        }
        for (int js = js0; js < js0 + nc && (int)npre < S && js < dep; ++js, ++npre)
          load_stage(npre, row, js, i);
        break;
      }
      pdl_wait();
      uint32_t it = 0, ul = 0;
      bool ok = true;
      for (int u = blockIdx.x, i = 0; u < p.units && ok; u += gridDim.x, ++i) {
        int row, js0, js1, nc;
        unit(u, i, row, js0, js1, nc);
        if (nc == 0) continue;
        const int bb = ul & 1;
        ok = tc::mbar_wait(&bempty[bb], ((ul >> 1) & 1) ^ 1, p.err);
        if (!ok) break;
        uint8_t* qb = sQ + bb * kQBuf;
        tc::mbar_arrive_expect_tx(&bfull[bb], kQBytes + kQSf + kHeads * 4);
        tc::tma_load_2d(qb, &tmQ, 0, row * kHeads, &bfull[bb]);
        tc::tma_load_2d(qb + kQBytes, &tmQS, 0, row * kHeads / 2, &bfull[bb]);
        tc::tma_load_1d(qb + kQBytes + kQSf + kPermBytes, &tmW, row * kHeads, &bfull[bb]);
        for (int js = js0; js < js0 + nc; ++js, ++it) {
          if (it < npre) continue;                       // fetched before the wait
          const int s = it % S;
          ok = tc::mbar_wait(&empty[s], ((it / S) & 1) ^ 1, p.err);
          if (!ok) break;
          load_stage(s, row, js, i);
        }
        ++ul;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_mxf4(kTileE, N);
    uint32_t it = 0, ul = 0;
    bool ok = true;
    // every stage of every unit goes through the rendezvous with the waiter warp, also
    // after a failure (then nothing is issued), so that neither warp is left waiting
    for (int u = blockIdx.x, i = 0; u < p.units; u += gridDim.x, ++i) {
      int row, js0, js1, nc;
      unit(u, i, row, js0, js1, nc);
      if (nc == 0) continue;
      const int bb = ul & 1;
      uint8_t* qb = sQ + bb * kQBuf;
      if (ok) ok = tc::mbar_wait(&bfull[bb], (ul >> 1) & 1, p.err);
      if (ok) {
        rearrange_scales(qb + kQBytes, qb + kQBytes + kQSf, kHeads, lane);
        tc::fence_proxy_async();
      }
      __syncwarp();
      const uint32_t sfb = tmem_base + kSfbCol + bb * 8;
      if (ok && lane == 0) {
        tc::tc_fence_after();
        tmem_cp_32x128b_x4(sfb, smem_desc_cp(tc::smem_u32(qb + kQBytes + kQSf)));
        tmem_cp_32x128b_x4(sfb + 4, smem_desc_cp(tc::smem_u32(qb + kQBytes + kQSf + 512)));
      }
      const uint64_t bdesc = smem_desc_sw64(tc::smem_u32(qb), 512);
      for (int j = 0; j < nc; ++j, ++it) {
        // the waiter has seen this stage's accumulator free (with its key scales) and
        // its key codes landed (bar.red is warp-aligned: the warp reconverges first)
        __syncwarp();
        const bool failed = tc::bar_red_or(1, 64, false);
        ok = ok && !failed;
        if (!ok || lane != 0) continue;
        tc::tc_fence_after();
        const int s = it % S;
        const int acc = it % NACC;
        uint8_t* st = sStage + s * kStage;
        const uint32_t sfa = tmem_base + kSfaCol + acc * (kTPS * 8);
#pragma unroll
        for (int t = 0; t < kTPS; ++t) {
          const uint64_t adesc = smem_desc_sw64(tc::smem_u32(st + t * kTileE * kRowB), 512);
          const uint32_t d = tmem_base + acc * kAccCols + t * N;
#pragma unroll
          for (int kb = 0; kb < 2; ++kb)   // K = 64 elements = 32 bytes per MMA
            mma_mxf4nvf4(d, adesc + 2 * kb, bdesc + 2 * kb, idesc, sfa + t * 8 + 4 * kb,
                         sfb + 4 * kb, kb > 0);
        }
        tc::mma_commit(&empty[s]);
        tc::mma_commit(&tfull[acc]);
      }
      if (ok && lane == 0) tc::mma_commit(&bempty[bb]);
      ++ul;
    }
  } else if (warp == kWaitWarp) {
    // ------------------------------------------------------------------ stage waiter
    uint32_t it = 0;
    bool ok = true;
    for (int u = blockIdx.x, i = 0; u < p.units; u += gridDim.x, ++i) {
      int row, js0, js1, nc;
      unit(u, i, row, js0, js1, nc);
      for (int j = 0; j < nc; ++j, ++it) {
        // accumulator free with this stage's key scales in place (phase it / NACC),
        // and the stage's key codes landed
        if (ok && lane == 0)
          ok = tc::mbar_wait(&tempty[it % NACC], (it / NACC) & 1, p.err) &&
               tc::mbar_wait(&full[it % S], (it / S) & 1, p.err);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        tc::bar_red_or(1, 64, !ok);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int grp = (warp - 2) >> 2;         // warpgroup: takes stages with c % 3 == grp
    const int lane_base = (warp & 3) * 32;   // TMEM lanes this warp may access
    uint32_t c = 0, ul = 0;                  // computed stages seen, units with work seen
    bool ok = true;
    uint32_t total_c = 0;                    // stages this CTA computes
    for (int u = blockIdx.x, i = 0; u < p.units; u += gridDim.x, ++i) {
      int row, js0, js1, nc;
      unit(u, i, row, js0, js1, nc);
      total_c += nc;
    }
    // key scales of stage x into the scale columns of accumulator x % NACC (this
    // warp's lane quarter; the four warps of the group write the same values, the
    // layout tcgen05.cp 32x128b.warpx4 would produce)
    auto write_sfa = [&](uint32_t x) -> bool {
      const int s = x % S;
      if (!tc::mbar_wait(&full[s], (x / S) & 1, p.err)) return false;
      const uint8_t* src = sStage + s * kStage + kKeyB + lane * 16;
      uint32_t v[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {            // q = tile * 2 + K block: 512-byte blocks
        const uint4 w = *reinterpret_cast<const uint4*>(src + q * 512);
        v[4 * q] = w.x; v[4 * q + 1] = w.y; v[4 * q + 2] = w.z; v[4 * q + 3] = w.w;
      }
      tmem_st16(tmem_base + ((uint32_t)lane_base << 16) + kSfaCol + (x % NACC) * (kTPS * 8), v);
      tc::tmem_st_wait();
      return true;
    };
    for (uint32_t x = grp; x < (uint32_t)NACC; x += kEpiGroups) {   // phase 0 of tempty[x]
      if (ok && x < total_c) ok = write_sfa(x);
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&tempty[x]);
    }
    for (int u = blockIdx.x, i = 0; u < p.units; u += gridDim.x, ++i) {
      int row, js0, js1, nc;
      unit(u, i, row, js0, js1, nc);
      // head weights of the unit, read (broadcast) from the query buffer, which is
      // released once this warp is done with the unit
      const float4* w4p = reinterpret_cast<const float4*>(sQ + (ul & 1) * kQBuf + kQBytes + kQSf +
                                                          kPermBytes);
      if (nc > 0) ok = ok && tc::mbar_wait(&bfull[ul & 1], (ul >> 1) & 1, p.err);
      const int ev = s_ev[i];
      for (int js = js0; js < js1; ++js) {
        float sc[kTPS];
#pragma unroll
        for (int t = 0; t < kTPS; ++t) sc[t] = -INFINITY;
        if (js < js0 + nc) {
          const uint32_t cc = c++;
          if ((int)(cc % kEpiGroups) != grp) continue;  // another warpgroup's stage
          if (ok) {
            const int acc = cc % NACC;
            ok = tc::mbar_wait(&tfull[acc], (cc / NACC) & 1, p.err);
            tc::tc_fence_after();
#pragma unroll
            for (int t = 0; t < kTPS; ++t) {
              uint32_t r0[32], r1[32];
              const uint32_t ta = tmem_base + ((uint32_t)lane_base << 16) + acc * kAccCols + t * N;
              tc::tmem_ld32(ta, r0);
              tc::tmem_ld32(ta + 32, r1);
              tc::tmem_ld_wait(r0);
              tc::reg_fence(r1);
              float a[4] = {0.f, 0.f, 0.f, 0.f};
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
              sc[t] = (a[0] + a[1]) + (a[2] + a[3]);
            }
            if (ok && cc + NACC < total_c) ok = write_sfa(cc + NACC);
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&tempty[acc]);
          }
        } else if (js % kEpiGroups != grp) {
          continue;                                     // fills rotate over the groups
        }
#pragma unroll
        for (int t = 0; t < kTPS; ++t) {
          const int e = (js * kTPS + t) * kTileE + lane_base + lane;
          if (e < p.E) {
            const float v = !ok ? __int_as_float(0x7fc00000) : (e < ev ? sc[t] : -INFINITY);
            const size_t o = (size_t)row * p.E + e;
            if (p.score_f32) reinterpret_cast<float*>(p.scores)[o] = v;
            else reinterpret_cast<__nv_bfloat16*>(p.scores)[o] = __float2bfloat16_rn(v);
          }
        }
      }
      if (nc > 0) {
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bempty[ul & 1]);
        ++ul;
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
  if (a.qk_dtype != CSA_NVFP4 || a.H != kHeads || a.d != kDim || a.T != 1) return CSA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(a.k) & 15) || (reinterpret_cast<uintptr_t>(a.q) & 15) ||
      (reinterpret_cast<uintptr_t>(a.k_scales) & 15) || (reinterpret_cast<uintptr_t>(a.q_scales) & 15) ||
      (reinterpret_cast<uintptr_t>(a.w) & 15))
    return CSA_ERR_INVALID_ARG;   // the TMA copies need 16-byte aligned rows and scale runs
  CUtensorMap tmK, tmQ, tmQS, tmW;
  const uint64_t krows = a.block_table ? (uint64_t)a.num_pages * kPageEntries : (uint64_t)b * a.E_cap;
  const uint64_t qrows = (uint64_t)b * a.T * kHeads;
  if (!make_tmap_2d_u8_swz(&tmK, a.k, kRowB, krows, kRowB, kStageE, 64) ||
      !make_tmap_2d_u8_swz(&tmQ, a.q, kRowB, qrows, kRowB, kHeads, 64) ||
      !make_tmap_2d_u8_swz(&tmQS, a.q_scales, 16, qrows / 2, 16, kHeads / 2, 0) ||
      !make_tmap_1d_f32(&tmW, a.w, qrows, kHeads))
    return CSA_ERR_CUDA;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  IdxFp4 p{};
  p.scores = a.scores; p.q_pos = a.q_pos;
  p.k_scales = reinterpret_cast<const uint8_t*>(a.k_scales);
  p.err = device_error_word();
  if (!p.err) return CSA_ERR_CUDA;
  p.T = a.T; p.E_cap = a.E_cap; p.E = a.E; p.m = a.m;
  p.tiles = (a.E + kTileE - 1) / kTileE;
  p.sf_tiles_cap = (a.E_cap + kTileE - 1) / kTileE;
  p.stages = (p.tiles + kTPS - 1) / kTPS;
  const long long rows = (long long)b * a.T;
  int nch = (int)((2LL * sms + rows - 1) / rows);
  nch = max(1, min(nch, p.stages));
  p.chunk = (p.stages + nch - 1) / nch;
  p.n_chunks = (p.stages + p.chunk - 1) / p.chunk;
  const long long units = rows * p.n_chunks;
  if (units > 0x7fffffff) return CSA_ERR_UNSUPPORTED;
  p.units = (int)units;
  p.score_f32 = a.score_dtype == CSA_F32;
  p.all_visible = a.all_visible;
  p.block_table = a.block_table; p.max_pages = a.max_pages; p.num_pages = a.num_pages;
  p.pos_input = a.pos_input;
  p.dep_stage = a.dep_entry < 0 ? 0 : a.dep_entry / kStageE;
  long long grid = units < sms ? units : sms;
  const long long min_grid = (units + kMaxLocalUnits - 1) / kMaxLocalUnits;
  if (grid < min_grid) grid = min_grid;
  const size_t smem = 1024 + (size_t)S * kStage + 2 * (size_t)kQBuf + (2 * S + 4 + 2 * NACC) * 8 +
                      16 + (size_t)kMaxLocalUnits * 2 * 4 + (size_t)kPagedSlots * 4;
  if (cudaFuncSetAttribute(index_scores_fp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return CSA_ERR_CUDA;
  if (csa_launch(index_scores_fp4_kernel, dim3((unsigned)grid), dim3(kThreads), smem, st,
                 a.pdl != 0, tmK, tmQ, tmQS, tmW, p) != cudaSuccess)
    return CSA_ERR_CUDA;
  return CSA_OK;
}

}  // namespace csa
