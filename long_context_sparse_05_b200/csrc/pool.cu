// Hierarchical sparse indexer (the Reindex mode of CSA2): score only a candidate pool.
//
// Method: "DeepSeek Technical Reports", section CSA2 (Hierarchical Sparse
// Indexer: a full indexer yields a larger candidate pool; a later Reindex layer
// scores again with its own query, searching only that pool, and keeps its k
// best).
//
// The pool of every query row is gathered into a key set of its own, so that the
// tensor-core indexer scores it unchanged (one "sequence" of P entries per query
// row, one query each) and the top-k selects positions in it:
//   pool_gather_kernel  CTA per (query row, 256 pool slots): compacts the pool entries
//                       visible to the row's position (counts and a block scan keep their
//                       order), copies their index-key rows and scales (FP8: one float per
//                       row; NVFP4: the tiled key-scale layout, re-tiled for the new
//                       positions), zeroes the rest of the last 256-entry stage, and writes
//                       the position m * count - 1 whose causal range is exactly the
//                       compacted pool;
//   pool_map_kernel     replaces each selected position by the entry it holds
//                       (ascending positions of an ascending pool are ascending entries).
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr int kGatherThreads = 256;

__device__ __forceinline__ int block_excl_scan_i(int v, int* s_warp, int& total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) s_warp[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int w = lane < nw ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) s_warp[lane] = w;
  }
  __syncthreads();
  total = s_warp[nw - 1];
  return (wid > 0 ? s_warp[wid - 1] : 0) + x - v;
}

struct PoolArgs {
  const int32_t* pool; const int32_t* pool_count; const int32_t* q_pos;
  const uint8_t* k; const void* k_scales;
  uint8_t* gk; void* gks; int32_t* gpool; int32_t* gpos;
  int T, P, P_cap, E_cap, E, m, row_bytes, d, fmt;   // fmt: CSA_F32, CSA_FP8_E4M3 or CSA_NVFP4
};

// Sums of a and b over the CTA (every thread gets both).
__device__ __forceinline__ void block_sum2_i(int& a, int& b, int* s_warp) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  a = __reduce_add_sync(0xffffffffu, a);
  b = __reduce_add_sync(0xffffffffu, b);
  __syncthreads();
  if (lane == 0) { s_warp[wid] = a; s_warp[16 + wid] = b; }
  __syncthreads();
  a = 0; b = 0;
  for (int w = 0; w < nw; ++w) { a += s_warp[w]; b += s_warp[16 + w]; }
  __syncthreads();
}

// CTA (query row r, chunk c of kGatherThreads pool slots), one slot per thread.  The
// entries the row sees keep their order: an entry's compacted position is the count of
// kept entries before its chunk (every CTA counts them itself, in one coalesced pass over
// the pool) plus its rank among its chunk's kept entries.  Each thread then copies its
// entry's key row and scales, and zeroes position j0 + tid if that lies between the
// compacted count and the end of its 256-entry stage; chunk 0 writes the position
// m * count - 1 whose causal range is exactly the compacted pool.
__global__ void __launch_bounds__(kGatherThreads) pool_gather_kernel(PoolArgs a) {
  __shared__ int s_warp[32];
  pdl_launch_dependents();
  pdl_wait();   // the pool, the positions and the newest key may come from preceding kernels
  const int r = blockIdx.x;
  const int j0 = blockIdx.y * kGatherThreads;
  const int sb = r / a.T;
  const int ev = visible_entries(a.q_pos[r], a.m, a.E);
  const int pc = min(a.pool_count[r], a.P);
  const int32_t* pl = a.pool + (size_t)r * a.P;
  int before = 0, cnt = 0;
  for (int j = threadIdx.x; j < pc; j += kGatherThreads) {
    const int e = pl[j];
    const int keep = (e >= 0 && e < ev) ? 1 : 0;
    cnt += keep;
    before += j < j0 ? keep : 0;
  }
  block_sum2_i(before, cnt, s_warp);
  const int j = j0 + threadIdx.x;
  const int e = j < pc ? pl[j] : -1;
  const int keep = (e >= 0 && e < ev) ? 1 : 0;
  int tot;
  const int pos = before + block_excl_scan_i(keep, s_warp, tot);
  if (blockIdx.y == 0 && threadIdx.x == 0) a.gpos[r] = a.m * cnt - 1;
  const int rb = a.row_bytes, cpr = rb / 16;
  const uint8_t* kseq = a.k + (size_t)sb * a.E_cap * rb;
  uint8_t* gkr = a.gk + (size_t)r * a.P_cap * rb;
  const int zend = min(a.P_cap, (cnt + 255) / 256 * 256);
  const bool zero = j >= cnt && j < zend;       // slot j of the compacted pool is padding
  if (keep) {
    a.gpool[(size_t)r * a.P + pos] = e;
    const uint4* src = reinterpret_cast<const uint4*>(kseq + (size_t)e * rb);
    uint4* dst = reinterpret_cast<uint4*>(gkr + (size_t)pos * rb);
    for (int x0 = 0; x0 < cpr; x0 += 8) {       // up to eight 16-byte loads in flight
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (x0 + u < cpr) v[u] = __ldg(src + x0 + u);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (x0 + u < cpr) dst[x0 + u] = v[u];
    }
  }
  if (zero) {
    uint4* dst = reinterpret_cast<uint4*>(gkr + (size_t)j * rb);
    for (int x = 0; x < cpr; ++x) dst[x] = make_uint4(0u, 0u, 0u, 0u);
  }
  if (a.fmt == CSA_FP8_E4M3) {
    const float* ks = static_cast<const float*>(a.k_scales) + (size_t)sb * a.E_cap;
    float* g = static_cast<float*>(a.gks) + (size_t)r * a.P_cap;
    if (keep) g[pos] = ks[e];
    if (zero) g[j] = 0.f;
  } else if (a.fmt == CSA_NVFP4) {
    const int nb = a.d / 16;
    const uint8_t* ks = static_cast<const uint8_t*>(a.k_scales) +
                        (size_t)sb * nvfp4_key_scale_seq_bytes(a.E_cap, a.d);
    uint8_t* g = static_cast<uint8_t*>(a.gks) + (size_t)r * nvfp4_key_scale_seq_bytes(a.P_cap, a.d);
    for (int blk = 0; blk < nb; ++blk) {
      if (keep) g[nvfp4_key_scale_offset(pos, blk, a.d)] = ks[nvfp4_key_scale_offset(e, blk, a.d)];
      if (zero) g[nvfp4_key_scale_offset(j, blk, a.d)] = 0;
    }
  }
}

// CTA (query row, chunk of kGatherThreads selection slots): each slot's position in the
// compacted pool is replaced by the entry it holds.
__global__ void __launch_bounds__(kGatherThreads) pool_map_kernel(const int32_t* gpool, int P,
                                                                  int k, int32_t* idx,
                                                                  const int32_t* count) {
  pdl_launch_dependents();
  pdl_wait();
  const int r = blockIdx.x;
  const int j = blockIdx.y * kGatherThreads + threadIdx.x;
  if (j >= k) return;
  const int c = count[r];
  int32_t* o = idx + (size_t)r * k;
  const int pos = o[j];
  o[j] = (j < c && pos >= 0 && pos < P) ? gpool[(size_t)r * P + pos] : -1;
}

}  // namespace

int pool_row_bytes(int fmt, int d) {
  return fmt == CSA_F32 ? 4 * d : fmt == CSA_FP8_E4M3 ? d : d / 2;
}

size_t pool_gather_bytes(int fmt, int rows, int P, int d, size_t* off_scales, size_t* off_pool,
                         size_t* off_pos) {
  const int P_cap = (P + 255) / 256 * 256;
  const size_t rb = (size_t)pool_row_bytes(fmt, d);
  auto a256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  size_t o = a256((size_t)rows * P_cap * rb);
  if (off_scales) *off_scales = o;
  o += a256(fmt == CSA_F32 ? 0
            : fmt == CSA_FP8_E4M3 ? (size_t)rows * P_cap * 4
                                  : (size_t)rows * nvfp4_key_scale_seq_bytes(P_cap, d));
  if (off_pool) *off_pool = o;
  o += a256((size_t)rows * P * 4);
  if (off_pos) *off_pos = o;
  o += a256((size_t)rows * 4);
  return o;
}

csa_status launch_pool_gather(int fmt, const int32_t* pool, const int32_t* pool_count,
                              const int32_t* q_pos, const void* k, const void* k_scales, int rows,
                              int T, int P, int E_cap, int E, int m, int d, void* ws,
                              cudaStream_t st, bool pdl) {
  if (rows <= 0) return CSA_OK;
  size_t o_sc, o_pl, o_ps;
  pool_gather_bytes(fmt, rows, P, d, &o_sc, &o_pl, &o_ps);
  PoolArgs a{};
  a.pool = pool; a.pool_count = pool_count; a.q_pos = q_pos;
  a.k = static_cast<const uint8_t*>(k); a.k_scales = k_scales;
  uint8_t* w = static_cast<uint8_t*>(ws);
  a.gk = w; a.gks = w + o_sc; a.gpool = reinterpret_cast<int32_t*>(w + o_pl);
  a.gpos = reinterpret_cast<int32_t*>(w + o_ps);
  a.T = T; a.P = P; a.P_cap = (P + 255) / 256 * 256; a.E_cap = E_cap; a.E = E; a.m = m;
  a.row_bytes = pool_row_bytes(fmt, d); a.d = d; a.fmt = fmt;
  if (csa_launch(pool_gather_kernel, dim3(rows, a.P_cap / kGatherThreads), dim3(kGatherThreads), 0,
                 st, pdl, a) != cudaSuccess)
    return CSA_ERR_CUDA;
  return CSA_OK;
}

csa_status launch_pool_map(const void* ws, int fmt, int rows, int P, int d, int k, int32_t* idx,
                           const int32_t* count, cudaStream_t st, bool pdl) {
  if (rows <= 0) return CSA_OK;
  size_t o_pl;
  pool_gather_bytes(fmt, rows, P, d, nullptr, &o_pl, nullptr);
  const int32_t* gpool = reinterpret_cast<const int32_t*>(static_cast<const uint8_t*>(ws) + o_pl);
  if (csa_launch(pool_map_kernel, dim3(rows, (k + kGatherThreads - 1) / kGatherThreads),
                 dim3(kGatherThreads), 0, st, pdl, gpool, P, k, idx, count) != cudaSuccess)
    return CSA_ERR_CUDA;
  return CSA_OK;
}

}  // namespace csa
