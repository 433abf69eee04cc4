// Context-parallel decode: each sequence's compressed entries sharded over ranks.
//
// Method: the selection and attention of "DeepSeek Technical Reports", section DSA (the
// top-k of a query's index scores, attention over the selected entries), computed over a
// cache split into contiguous shards of entries.  Each rank scores its shard and keeps
// its own top-k; the global top-k is contained in the union of the shards' top-k (an
// entry among the k best overall is among the k best of its shard under the same order:
// score descending, entry ascending), so the top-k of the gathered candidates is exactly
// the top-k of the whole cache.  The selected rows then travel to every rank.
//
//   cp_candidates_kernel  a rank's top-k as (score, global entry) pairs, -inf / -1 padded;
//   cp_permute_kernel     the ranks' candidates of a query side by side, rank-major (so
//                         candidate positions ascend with the entry), and the position
//                         that makes every candidate visible to the top-k;
//   cp_map_kernel         selected positions -> entries, dropping padding (the order is
//                         kept: ascending entries), and the row list 0 .. count - 1 of the
//                         gathered rows;
//   cp_pack_kernel        the selected rows this rank holds into their selection slots
//                         (zeros elsewhere), so that a sum over the ranks gathers them.
// Each is launched as a programmatic dependent of the kernel before it on the stream and
// waits for that kernel before it reads anything.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr int kCpThreads = 256;

__global__ void __launch_bounds__(kCpThreads) cp_candidates_kernel(
    const __nv_bfloat16* __restrict__ scores, int E_local, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ count, int k, int offset, __nv_bfloat16* __restrict__ cand_s,
    int32_t* __restrict__ cand_i) {
  pdl_launch_dependents();
  pdl_wait();
  const int q = blockIdx.x;
  const int n = count[q];
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    const int e = j < n ? idx[(size_t)q * k + j] : -1;
    const bool ok = e >= 0 && e < E_local;
    cand_s[(size_t)q * k + j] = ok ? scores[(size_t)q * E_local + e] : __float2bfloat16_rn(-INFINITY);
    cand_i[(size_t)q * k + j] = ok ? offset + e : -1;
  }
}

// [G][b][k] -> [b][G k], and the all-visible position G k - 1 (m = 1) per query.
__global__ void __launch_bounds__(kCpThreads) cp_permute_kernel(
    const __nv_bfloat16* __restrict__ cand_s, const int32_t* __restrict__ cand_i, int G, int b,
    int k, __nv_bfloat16* __restrict__ row_s, int32_t* __restrict__ row_i, int32_t* __restrict__ pos) {
  pdl_launch_dependents();
  pdl_wait();
  const int q = blockIdx.x;
  const int n = G * k;
  for (int x = threadIdx.x; x < n; x += blockDim.x) {
    const int g = x / k, j = x - g * k;
    const size_t src = ((size_t)g * b + q) * k + j;
    row_s[(size_t)q * n + x] = cand_s[src];
    row_i[(size_t)q * n + x] = cand_i[src];
  }
  if (threadIdx.x == 0) pos[q] = n - 1;
}

__device__ __forceinline__ int cp_excl_scan(int v, int* s_warp, int& total) {
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

// Selected candidate positions (ascending, sel_cnt of them) -> entries, without padding.
__global__ void __launch_bounds__(kCpThreads) cp_map_kernel(
    const int32_t* __restrict__ sel, const int32_t* __restrict__ sel_cnt,
    const int32_t* __restrict__ row_i, int n, int k, int32_t* __restrict__ idx,
    int32_t* __restrict__ count, int32_t* __restrict__ rows_idx) {
  __shared__ int s_warp[32];
  pdl_launch_dependents();
  pdl_wait();
  const int q = blockIdx.x;
  const int ns = sel_cnt[q];
  int base = 0;
  for (int j0 = 0; j0 < k; j0 += blockDim.x) {
    const int j = j0 + threadIdx.x;
    int e = -1;
    if (j < k && j < ns) {
      const int p = sel[(size_t)q * k + j];
      if (p >= 0 && p < n) e = row_i[(size_t)q * n + p];
    }
    int tot;
    const int o = cp_excl_scan(e >= 0 ? 1 : 0, s_warp, tot);
    if (e >= 0) idx[(size_t)q * k + base + o] = e;
    base += tot;
  }
  for (int j = base + threadIdx.x; j < k; j += blockDim.x) idx[(size_t)q * k + j] = -1;
  for (int j = threadIdx.x; j < k; j += blockDim.x) rows_idx[(size_t)q * k + j] = j < base ? j : -1;
  if (threadIdx.x == 0) count[q] = base;
}

// Slot j of query q: entry idx[q][j] if this rank holds it (offset <= e < offset + E_local),
// its row of `row_bytes` copied from kv; zeros otherwise.  A warp per slot, 16-byte pieces.
__global__ void __launch_bounds__(kCpThreads) cp_pack_kernel(
    const uint8_t* __restrict__ kv, int E_cap_local, int E_local, int offset, size_t row_bytes,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ count, int k,
    uint8_t* __restrict__ rows) {
  pdl_launch_dependents();
  pdl_wait();
  const int q = blockIdx.y;
  const int warps = blockDim.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * warps + (threadIdx.x >> 5);
  if (j >= k) return;
  const int e = j < count[q] ? idx[(size_t)q * k + j] : -1;
  const bool mine = e >= offset && e < offset + E_local;
  const uint4* src = mine ? reinterpret_cast<const uint4*>(kv + ((size_t)q * E_cap_local + (e - offset)) * row_bytes)
                          : nullptr;
  uint4* dst = reinterpret_cast<uint4*>(rows + ((size_t)q * k + j) * row_bytes);
  const size_t n16 = row_bytes / 16;
  for (size_t x = lane; x < n16; x += 32) dst[x] = mine ? __ldg(src + x) : make_uint4(0u, 0u, 0u, 0u);
}

}  // namespace

csa_status launch_cp_candidates(const void* scores, int E_local, const int32_t* idx,
                                const int32_t* count, int b, int k, int offset, void* cand_s,
                                int32_t* cand_i, cudaStream_t st) {
  if (csa_launch(cp_candidates_kernel, dim3(b), dim3(kCpThreads), 0, st, true,
                 reinterpret_cast<const __nv_bfloat16*>(scores), E_local, idx, count, k, offset,
                 static_cast<__nv_bfloat16*>(cand_s), cand_i) != cudaSuccess)
    return CSA_ERR_CUDA;
  return CSA_OK;
}

size_t cp_merge_bytes(int G, int b, int k, size_t topk_ws) {
  const size_t n = (size_t)G * k;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  return al((size_t)b * n * 2) + al((size_t)b * n * 4) + al((size_t)b * 4) + al((size_t)b * k * 4) +
         al((size_t)b * 4) + al(topk_ws);
}

csa_status launch_cp_merge(const void* cand_s, const int32_t* cand_i, int G, int b, int k,
                           int32_t* idx, int32_t* count, int32_t* rows_idx, void* ws,
                           size_t ws_bytes, cudaStream_t st) {
  const int n = G * k;
  const size_t topk_ws = topk_workspace_bytes(b, n, k, CSA_BF16);
  if (!ws || ws_bytes < cp_merge_bytes(G, b, k, topk_ws)) return CSA_ERR_INVALID_ARG;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  uint8_t* p = static_cast<uint8_t*>(ws);
  auto* row_s = reinterpret_cast<__nv_bfloat16*>(p);      p += al((size_t)b * n * 2);
  auto* row_i = reinterpret_cast<int32_t*>(p);            p += al((size_t)b * n * 4);
  auto* pos = reinterpret_cast<int32_t*>(p);              p += al((size_t)b * 4);
  auto* sel = reinterpret_cast<int32_t*>(p);              p += al((size_t)b * k * 4);
  auto* sel_cnt = reinterpret_cast<int32_t*>(p);          p += al((size_t)b * 4);
  void* tws = topk_ws ? p : nullptr;
  if (csa_launch(cp_permute_kernel, dim3(b), dim3(kCpThreads), 0, st, true,
                 reinterpret_cast<const __nv_bfloat16*>(cand_s), cand_i, G, b, k, row_s, row_i,
                 pos) != cudaSuccess)
    return CSA_ERR_CUDA;
  csa_status r = launch_topk_search(row_s, CSA_BF16, pos, 1, b, n, k, sel, sel_cnt, tws, topk_ws, st,
                                    true);
  if (r == CSA_ERR_UNSUPPORTED) r = launch_topk(row_s, CSA_BF16, pos, 1, b, n, k, sel, sel_cnt, st);
  if (r) return r;
  if (csa_launch(cp_map_kernel, dim3(b), dim3(kCpThreads), 0, st, true, sel, sel_cnt, row_i, n, k,
                 idx, count, rows_idx) != cudaSuccess)
    return CSA_ERR_CUDA;
  return CSA_OK;
}

csa_status launch_cp_pack(const void* kv, int E_cap_local, int E_local, int offset, size_t row_bytes,
                          const int32_t* idx, const int32_t* count, int b, int k, void* rows,
                          cudaStream_t st) {
  const int warps = kCpThreads / 32;
  dim3 grid((k + warps - 1) / warps, b);
  if (csa_launch(cp_pack_kernel, grid, dim3(kCpThreads), 0, st, true,
                 static_cast<const uint8_t*>(kv), E_cap_local, E_local, offset, row_bytes, idx, count,
                 k, static_cast<uint8_t*>(rows)) != cudaSuccess)
    return CSA_ERR_CUDA;
  return CSA_OK;
}

}  // namespace csa
