// Causal top-k, search-based (no atomics), one CTA or one 8-CTA cluster per query.
//
// Method: "DeepSeek Technical Reports", section DSA (Top-k over the index
// scores of a query); "DeepSeek V4 结构速览", sections "核心设计" item 2 and
// "Lightning Indexer" (k among the causally visible entries).
//
// Index scores are non-negative sums of ReLU terms, so their bf16 patterns
// crowd into a handful of exponents: a byte-wise radix histogram sends almost
// every element to the same few bins and serialises on shared-memory atomics.
// This kernel instead searches the key space.  Scores become order-preserving
// unsigned keys; the row is staged once through shared memory so each thread
// owns EPT consecutive entries in registers.  Each round splits the candidate
// key range [lo, hi] at three points and counts, over the whole row, the keys
// at or above each point (warp redux, a block reduction, and for clustered rows
// a sum over the 8 CTAs through distributed shared memory); the range shrinks to
// the quarter holding the k-th largest key.  After ceil(bits / 2) rounds lo is
// that key tau exactly.  A last count gives how many keys lie strictly above
// tau, so `need` = k - that many keys equal to tau are taken, lowest entries
// first.  One packed block scan (keys above tau in the low 16 bits, keys equal
// to tau in the high 16) orders the output ascending by entry.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace csa {

namespace {

template <typename S> struct Keys;
template <> struct Keys<__nv_bfloat16> {
  static constexpr uint32_t kMax = 0xffffu;
  __device__ static __forceinline__ uint32_t key(uint32_t u) {
    if ((u & 0x7fffu) == 0) u = 0;   // -0 ties with +0
    return (u & 0x8000u) ? (~u & 0xffffu) : (u | 0x8000u);
  }
  __device__ static __forceinline__ uint32_t load(const __nv_bfloat16* p, int s) {
    return key(reinterpret_cast<const uint16_t*>(p)[s]);
  }
};
template <> struct Keys<float> {
  static constexpr uint32_t kMax = 0xffffffffu;
  __device__ static __forceinline__ uint32_t key(uint32_t u) {
    if ((u & 0x7fffffffu) == 0) u = 0;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  }
  __device__ static __forceinline__ uint32_t load(const float* p, int s) {
    return key(__float_as_uint(p[s]));
  }
};

constexpr int kEPT = 32;   // entries per thread

// Sums NV per-thread values over the CTA (and over the cluster when CL > 1).
// `slot` is a per-round double buffer of NV counters in shared memory.
template <int CL, int NV>
__device__ __forceinline__ void row_sum(uint32_t (&v)[NV], uint32_t* s_warp, uint32_t* slot,
                                        cg::cluster_group& cluster) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const uint32_t w = __reduce_add_sync(0xffffffffu, v[i]);
    if (lane == 0) s_warp[wid * NV + i] = w;
  }
  __syncthreads();
  if (wid == 0) {
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const uint32_t x = lane < nw ? s_warp[lane * NV + i] : 0u;
      const uint32_t tot = __reduce_add_sync(0xffffffffu, x);
      if (lane == 0) slot[i] = tot;
    }
  }
  if constexpr (CL > 1) {
    cluster.sync();   // every CTA's slot is written
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      uint32_t tot = 0;
#pragma unroll
      for (int r = 0; r < CL; ++r) tot += cluster.map_shared_rank(slot, r)[i];
      v[i] = tot;
    }
  } else {
    __syncthreads();
#pragma unroll
    for (int i = 0; i < NV; ++i) v[i] = slot[i];
  }
}

template <typename S, int CL>
__global__ void __launch_bounds__(1024) topk_search_kernel(
    const S* __restrict__ scores, const int32_t* __restrict__ q_pos, int m, int E, int k,
    int32_t* __restrict__ idx, int32_t* __restrict__ count) {
  using K = Keys<S>;
  extern __shared__ uint32_t s_keys[];               // [NT * EPT] staged keys
  __shared__ uint32_t s_warp[32 * 3];
  __shared__ uint32_t s_slot[2][4];                  // per-round double buffer (DSMEM-visible)
  __shared__ uint32_t s_tot[4];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = CL > 1 ? (int)cluster.block_rank() : 0;
  const int row = blockIdx.x / CL;
  const int tid = threadIdx.x;
  const int NT = blockDim.x;
  const S* sc = scores + (size_t)row * E;
  int32_t* out = idx + (size_t)row * k;
  const int ev = visible_entries(q_pos[row], m, E);

  if (ev <= k) {                                      // every CTA of the cluster takes this branch
    if (rank == 0) {
      for (int j = tid; j < k; j += NT) out[j] = j < ev ? j : -1;
      if (tid == 0) count[row] = ev;
    }
    return;
  }

  const int cap = NT * kEPT;
  const int beg = rank * cap;
  const int nloc = max(0, min(ev - beg, cap));
#pragma unroll
  for (int i = 0; i < kEPT; ++i) {               // all loads of a thread in flight together
    const int j = i * NT + tid;
    s_keys[j] = j < nloc ? K::load(sc, beg + j) : 0u;
  }
  __syncthreads();
  // thread tid owns entries tid*EPT .. tid*EPT+EPT-1; it visits them rotated by tid, which
  // spreads the 32 lanes of a warp over the 32 shared-memory banks
  const uint32_t* my = s_keys + tid * kEPT;
#define KEY(e) my[((e) + tid) & (kEPT - 1)]

  uint32_t lo = 0, hi = K::kMax;
  int round = 0;
  while (lo < hi) {
    const uint64_t R = (uint64_t)hi - lo + 1;
    uint32_t sp[3];
#pragma unroll
    for (int i = 0; i < 3; ++i) sp[i] = lo + (uint32_t)((R * (uint64_t)(i + 1)) >> 2);
    uint32_t c[3] = {0u, 0u, 0u};
#pragma unroll
    for (int e = 0; e < kEPT; ++e) {
#pragma unroll
      for (int i = 0; i < 3; ++i) c[i] += KEY(e) >= sp[i] ? 1u : 0u;
    }
    row_sum<CL, 3>(c, s_warp, s_slot[round & 1], cluster);
    // largest split with at least k keys at or above it
    uint32_t nlo = lo, nhi = hi;
    if (c[2] >= (uint32_t)k) { nlo = sp[2]; }
    else if (c[1] >= (uint32_t)k) { nlo = sp[1]; nhi = sp[2] - 1; }
    else if (c[0] >= (uint32_t)k) { nlo = sp[0]; nhi = sp[1] - 1; }
    else { nhi = sp[0] - 1; }
    if (nlo < lo) nlo = lo;               // splits equal to lo carry no information
    lo = nlo; hi = nhi;
    ++round;
  }
  const uint32_t tau = lo;

  // keys strictly above tau and keys equal to tau: per thread, then over the row
  uint32_t n_gt = 0, n_eq = 0;
#pragma unroll
  for (int e = 0; e < kEPT; ++e) { n_gt += KEY(e) > tau; n_eq += KEY(e) == tau; }
  uint32_t tot[2] = {n_gt, n_eq};
  row_sum<CL, 2>(tot, s_warp, s_slot[round & 1], cluster);
  const int need = k - (int)tot[0];        // equal keys to take, lowest entries first

  // this CTA's base among the CTAs of the cluster
  uint32_t base_gt = 0, base_eq = 0;
  if constexpr (CL > 1) {
    // per-CTA totals: reuse the last round's buffer pattern with a fresh buffer
    uint32_t mine[2] = {n_gt, n_eq};
    const int lane = tid & 31, wid = tid >> 5, nw = NT >> 5;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint32_t w = __reduce_add_sync(0xffffffffu, mine[i]);
      if (lane == 0) s_warp[wid * 2 + i] = w;
    }
    __syncthreads();
    if (wid == 0) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint32_t x = lane < nw ? s_warp[lane * 2 + i] : 0u;
        const uint32_t t = __reduce_add_sync(0xffffffffu, x);
        if (lane == 0) s_tot[i] = t;
      }
    }
    cluster.sync();
    for (int r = 0; r < rank; ++r) {
      const uint32_t* o = cluster.map_shared_rank(s_tot, r);
      base_gt += o[0];
      base_eq += o[1];
    }
  }

  // block exclusive scan of (gt | eq << 16) per thread
  const uint32_t packed = n_gt | (n_eq << 16);
  uint32_t x = packed;
  const int lane = tid & 31, wid = tid >> 5, nw = NT >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) s_warp[wid] = x;
  __syncthreads();
  if (wid == 0) {
    uint32_t w = lane < nw ? s_warp[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) s_warp[lane] = w;
  }
  __syncthreads();
  const uint32_t excl = (wid > 0 ? s_warp[wid - 1] : 0u) + x - packed;
  const uint32_t gt_before = base_gt + (excl & 0xffffu);
  const uint32_t eq_before = base_eq + (excl >> 16);
  // masks of this thread's entries (bit e = entry tid * EPT + e), read bank-conflict free
  uint32_t gt_mask = 0, eq_mask = 0;
#pragma unroll
  for (int e = 0; e < kEPT; ++e) {
    const int b = (e + tid) & (kEPT - 1);
    gt_mask |= (KEY(e) > tau ? 1u : 0u) << b;
    eq_mask |= (KEY(e) == tau ? 1u : 0u) << b;
  }
  // equal keys: take this thread's lowest entries while the row still needs some
  int take_eq = min(max(need - (int)eq_before, 0), __popc(eq_mask));
  uint32_t eq_take = 0, rest = eq_mask;
  for (int i = 0; i < take_eq; ++i) {
    const uint32_t low = rest & (0u - rest);
    eq_take |= low;
    rest ^= low;
  }
  uint32_t sel = gt_mask | eq_take;
  int pos = (int)gt_before + min((int)eq_before, need);
  while (sel) {
    const int e = __ffs(sel) - 1;
    sel &= sel - 1;
    const int j = tid * kEPT + e;
    if (j < nloc && pos < k) out[pos] = beg + j;
    ++pos;
  }
#undef KEY
  if (rank == 0 && tid == 0) count[row] = k;
  if constexpr (CL > 1) cluster.sync();   // keep shared memory alive for remote readers
}

template <typename S, int CL>
csa_status launch_search(const void* scores, const int32_t* q_pos, int m, int rows, int E, int k,
                         int32_t* idx, int32_t* count, int nt, cudaStream_t st) {
  const size_t smem = (size_t)nt * kEPT * sizeof(uint32_t);
  auto kern = topk_search_kernel<S, CL>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return CSA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows * CL);
  cfg.blockDim = dim3(nt);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, reinterpret_cast<const S*>(scores), q_pos, m, E, k, idx,
                         count) != cudaSuccess)
    return CSA_ERR_CUDA;
  return CSA_OK;
}

}  // namespace

// Rows of up to 512 x 32 entries: one CTA; up to 8 x 1024 x 32: one 8-CTA cluster;
// longer rows go to the histogram kernel.  k must fit the 16-bit packed counters.
csa_status launch_topk_search(const void* scores, int score_dtype, const int32_t* q_pos, int m,
                              int rows, int E, int k, int32_t* idx, int32_t* count,
                              cudaStream_t st) {
  if (rows == 0) return CSA_OK;
  if (E <= 512 * kEPT) {
    const int nt = E <= 128 * kEPT ? 128 : (E <= 256 * kEPT ? 256 : 512);
    return score_dtype == CSA_BF16
               ? launch_search<__nv_bfloat16, 1>(scores, q_pos, m, rows, E, k, idx, count, nt, st)
               : launch_search<float, 1>(scores, q_pos, m, rows, E, k, idx, count, nt, st);
  }
  if (E <= 8 * 1024 * kEPT)
    return score_dtype == CSA_BF16
               ? launch_search<__nv_bfloat16, 8>(scores, q_pos, m, rows, E, k, idx, count, 1024, st)
               : launch_search<float, 8>(scores, q_pos, m, rows, E, k, idx, count, 1024, st);
  return CSA_ERR_UNSUPPORTED;
}

}  // namespace csa
