// Causal top-k, search-based (no atomics), one CTA per query (or per chunk of a
// long query row, followed by a top-k of the chunks' top-k).
//
// Method: "DeepSeek Technical Reports", section DSA (Top-k over the index
// scores of a query); "DeepSeek V4 结构速览", sections "核心设计" item 2 and
// "Lightning Indexer" (k among the causally visible entries).
//
// Index scores are non-negative sums of ReLU terms, so their bf16 patterns
// crowd into a handful of exponents: a byte-wise radix histogram sends almost
// every element to the same few bins and serialises on shared-memory atomics.
// This kernel searches the key space instead.  Scores become order-preserving
// unsigned keys held in registers, 32 consecutive entries per thread.  The
// candidate range starts at the row's [min, max] key; each round splits it at
// three points and counts, over the row, the keys at or above each point (warp
// redux, then one shared-memory pass), keeping the quarter that holds the k-th
// largest key.  When the range is a single key it is the k-th key tau exactly;
// `need` = k - (keys above tau) keys equal to tau are taken, lowest entries first.
// One packed block scan (keys above tau in the low 16 bits, keys equal to tau in
// the high 16) writes the selection in ascending entry order.
//
// Rows longer than one CTA holds (512 threads x 32) are cut into chunks: every
// chunk keeps its own top-k (the global top-k is contained in the union, and
// since chunks are contiguous index ranges the lowest-index rule for ties
// carries over), and a second pass selects the top-k of the candidates.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

constexpr int kEPT = 32;            // entries per thread
constexpr int kNT = 512;            // threads of the largest CTA
constexpr int kChunk = kNT * kEPT;  // entries one CTA holds

template <typename S> struct Keys;
template <> struct Keys<__nv_bfloat16> {
  using Bits = uint16_t;
  static constexpr uint32_t kMax = 0xffffu;
  static constexpr Bits kSentinel = 0xffffu;   // pattern whose key is 0: below every score
  __device__ static __forceinline__ uint32_t key(uint32_t u) {
    if ((u & 0x7fffu) == 0) u = 0;   // -0 ties with +0
    return (u & 0x8000u) ? (~u & 0xffffu) : (u | 0x8000u);
  }
};
template <> struct Keys<float> {
  using Bits = uint32_t;
  static constexpr uint32_t kMax = 0xffffffffu;
  static constexpr Bits kSentinel = 0xffffffffu;
  __device__ static __forceinline__ uint32_t key(uint32_t u) {
    if ((u & 0x7fffffffu) == 0) u = 0;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  }
};

// Block-wide sums of NV unsigned values (every thread gets them), with one barrier:
// each warp writes its partial sums into one of two buffers (alternating per call, so
// a fast warp's next call cannot overwrite a buffer still being read), and every
// thread adds up the warps' partials itself.  s_red holds 2 x 64 words (NV <= 2).
template <int NV>
__device__ __forceinline__ void block_sums(uint32_t (&v)[NV], uint32_t* s_red, uint32_t& parity) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  static_assert(NV <= 2, "two 64-word buffers");
  uint32_t* buf = s_red + parity * 64;
  parity ^= 1u;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const uint32_t w = __reduce_add_sync(0xffffffffu, v[i]);
    if (lane == 0) buf[wid * NV + i] = w;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < NV; ++i) v[i] = 0u;
  for (int w = 0; w < nw; ++w) {
#pragma unroll
    for (int i = 0; i < NV; ++i) v[i] += buf[w * NV + i];
  }
}

// Top-k of one row (or chunk) of `n` entries held by the CTA.
//   src       scores (type S); entry j of the chunk is src[j]
//   map       optional: output index of entry j is map[j] (candidate pass), else base + j
//   out/cnt   output row (k slots, -1 padded) and its count (cnt may be NULL)
//   out_keys  optional: the scores of the kept entries, in output order (chunk pass)
template <typename S>
__device__ __forceinline__ void cta_topk(const S* __restrict__ src, int n, int k,
                                         const int32_t* __restrict__ map, int base,
                                         int32_t* __restrict__ out, int32_t* cnt,
                                         S* __restrict__ out_keys, uint32_t* s_red) {
  using K = Keys<S>;
  using Bits = typename K::Bits;
  const int tid = threadIdx.x;
  const int NT = blockDim.x;
  uint32_t parity = 0;                           // block_sums buffer selector
  if (n <= k) {                                  // everything is kept
    for (int j = tid; j < k; j += NT) {
      const bool v = j < n;
      out[j] = v ? (map ? map[j] : base + j) : -1;
      if (out_keys) {
        const Bits b = v ? reinterpret_cast<const Bits*>(src)[j] : K::kSentinel;
        reinterpret_cast<Bits*>(out_keys)[j] = b;
      }
    }
    if (tid == 0 && cnt) *cnt = n;
    return;
  }

  // this thread's 32 consecutive entries as keys (entries past n are key 0)
  uint32_t key[kEPT];
  const int j0 = tid * kEPT;
  const Bits* bits = reinterpret_cast<const Bits*>(src);
  const bool vec = ((reinterpret_cast<uintptr_t>(bits + j0) & 15) == 0) && j0 + kEPT <= n;
  if (vec) {
    constexpr int kPer = 16 / sizeof(Bits);
#pragma unroll
    for (int v = 0; v < kEPT / kPer; ++v) {
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(bits + j0) + v);
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if constexpr (sizeof(Bits) == 2) {
          key[v * kPer + 2 * i] = K::key(w[i] & 0xffffu);
          key[v * kPer + 2 * i + 1] = K::key(w[i] >> 16);
        } else {
          key[v * kPer + i] = K::key(w[i]);
        }
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < kEPT; ++e) key[e] = j0 + e < n ? K::key(bits[j0 + e]) : 0u;
  }

  // initial range: [min, max] of the valid keys
  uint32_t kmin = 0xffffffffu, kmax = 0;
#pragma unroll
  for (int e = 0; e < kEPT; ++e) {
    const bool v = j0 + e < n;
    kmin = v ? min(kmin, key[e]) : kmin;
    kmax = v ? max(kmax, key[e]) : kmax;
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  {
    const int lane = tid & 31, wid = tid >> 5, nw = NT >> 5;
    if (lane == 0) { s_red[wid] = kmin; s_red[32 + wid] = kmax; }
    __syncthreads();
    if (wid == 0) {
      const uint32_t a = lane < nw ? s_red[lane] : 0xffffffffu;
      const uint32_t b = lane < nw ? s_red[32 + lane] : 0u;
      const uint32_t ra = __reduce_min_sync(0xffffffffu, a);
      const uint32_t rb = __reduce_max_sync(0xffffffffu, b);
      if (lane == 0) { s_red[64] = ra; s_red[65] = rb; }
    }
    __syncthreads();
    kmin = s_red[64];
    kmax = s_red[65];
    __syncthreads();
  }
  // invariant: at least k keys are >= lo, fewer than k keys are > hi
  uint32_t lo = kmin, hi = kmax;
  while (lo < hi) {
    const uint64_t R = (uint64_t)hi - lo + 1;
    uint32_t sp[3];
#pragma unroll
    for (int i = 0; i < 3; ++i) sp[i] = lo + (uint32_t)((R * (uint64_t)(i + 1)) >> 2);
    // counts packed two per word (a CTA holds at most 16384 entries)
    uint32_t c[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < kEPT; ++e) {
      c[0] += (key[e] >= sp[0] ? 1u : 0u) | (key[e] >= sp[1] ? 0x10000u : 0u);
      c[1] += key[e] >= sp[2] ? 1u : 0u;
    }
    block_sums<2>(c, s_red, parity);
    const uint32_t c0 = c[0] & 0xffffu, c1 = c[0] >> 16, c2 = c[1];
    uint32_t nlo = lo, nhi = hi;
    if (c2 >= (uint32_t)k) { nlo = sp[2]; }
    else if (c1 >= (uint32_t)k) { nlo = sp[1]; nhi = sp[2] - 1; }
    else if (c0 >= (uint32_t)k) { nlo = sp[0]; nhi = sp[1] - 1; }
    else { nhi = sp[0] - 1; }
    lo = max(nlo, lo);
    hi = nhi;
  }
  const uint32_t tau = lo;

  uint32_t gt_mask = 0, eq_mask = 0;
#pragma unroll
  for (int e = 0; e < kEPT; ++e) {
    const bool v = j0 + e < n;
    gt_mask |= (v && key[e] > tau ? 1u : 0u) << e;
    eq_mask |= (v && key[e] == tau ? 1u : 0u) << e;
  }
  const uint32_t n_gt = __popc(gt_mask), n_eq = __popc(eq_mask);
  uint32_t tot[1] = {n_gt};
  block_sums<1>(tot, s_red, parity);
  const int need = k - (int)tot[0];              // equal keys to take, lowest entries first

  // exclusive block scan of (gt | eq << 16)
  const uint32_t packed = n_gt | (n_eq << 16);
  const int lane = tid & 31, wid = tid >> 5, nw = NT >> 5;
  uint32_t x = packed;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  uint32_t* sc = s_red + 128;                   // apart from block_sums' buffers
  if (lane == 31) sc[wid] = x;
  __syncthreads();
  if (wid == 0) {
    uint32_t w = lane < nw ? sc[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) sc[lane] = w;
  }
  __syncthreads();
  const uint32_t excl = (wid > 0 ? sc[wid - 1] : 0u) + x - packed;
  const int gt_before = (int)(excl & 0xffffu);
  const int eq_before = (int)(excl >> 16);
  const int take_eq = min(max(need - eq_before, 0), (int)n_eq);
  uint32_t eq_take = 0, rest = eq_mask;
  for (int i = 0; i < take_eq; ++i) {
    const uint32_t low = rest & (0u - rest);
    eq_take |= low;
    rest ^= low;
  }
  uint32_t sel = gt_mask | eq_take;
  int pos = gt_before + min(eq_before, need);
  while (sel) {
    const int e = __ffs(sel) - 1;
    sel &= sel - 1;
    if (pos < k) {
      out[pos] = map ? map[j0 + e] : base + j0 + e;
      if (out_keys) reinterpret_cast<Bits*>(out_keys)[pos] = bits[j0 + e];
    }
    ++pos;
  }
  if (tid == 0 && cnt) *cnt = k;
}

// Direct pass: one CTA per query row (rows of at most kChunk entries).
template <typename S>
__global__ void __launch_bounds__(kNT) topk_row_kernel(
    const S* __restrict__ scores, const int32_t* __restrict__ q_pos, int m, int E, int k,
    int32_t* __restrict__ idx, int32_t* __restrict__ count) {
  __shared__ uint32_t s_red[128 + 32];
  pdl_launch_dependents();
  pdl_wait();
  const int row = blockIdx.x;
  const int ev = visible_entries(q_pos[row], m, E);
  cta_topk<S>(scores + (size_t)row * E, ev, k, nullptr, 0, idx + (size_t)row * k, count + row,
              nullptr, s_red);
}

// First pass for long rows: chunk c of row r keeps its top-k (scores and entry indices).
template <typename S>
__global__ void __launch_bounds__(kNT) topk_chunk_kernel(
    const S* __restrict__ scores, const int32_t* __restrict__ q_pos, int m, int E, int k,
    int nchunks, S* __restrict__ cand_scores, int32_t* __restrict__ cand_idx) {
  __shared__ uint32_t s_red[128 + 32];
  pdl_launch_dependents();
  pdl_wait();
  const int row = blockIdx.x / nchunks, c = blockIdx.x % nchunks;
  const int ev = visible_entries(q_pos[row], m, E);
  const int beg = c * kChunk;
  const int n = max(0, min(ev - beg, kChunk));
  const size_t slot = ((size_t)row * nchunks + c) * k;
  cta_topk<S>(scores + (size_t)row * E + beg, n, k, nullptr, beg, cand_idx + slot, nullptr,
              cand_scores + slot, s_red);
}

// Second pass: top-k of a row's nchunks * k candidates (padding slots hold the
// sentinel, whose key sits below every score, and index -1).
template <typename S>
__global__ void __launch_bounds__(kNT) topk_merge_kernel(
    const S* __restrict__ cand_scores, const int32_t* __restrict__ cand_idx,
    const int32_t* __restrict__ q_pos, int m, int E, int k, int nchunks,
    int32_t* __restrict__ idx, int32_t* __restrict__ count) {
  __shared__ uint32_t s_red[128 + 32];
  pdl_launch_dependents();
  pdl_wait();
  const int row = blockIdx.x;
  const int ev = visible_entries(q_pos[row], m, E);
  const size_t slot = (size_t)row * nchunks * k;
  if (ev <= k) {   // the first chunk already holds every visible entry, in order
    for (int j = threadIdx.x; j < k; j += blockDim.x) idx[(size_t)row * k + j] = cand_idx[slot + j];
    if (threadIdx.x == 0) count[row] = ev;
    return;
  }
  cta_topk<S>(cand_scores + slot, nchunks * k, k, cand_idx + slot, 0, idx + (size_t)row * k,
              count + row, nullptr, s_red);
}

int threads_for(int n) {
  const int nt = (n + kEPT - 1) / kEPT;
  return nt <= 128 ? 128 : (nt <= 256 ? 256 : 512);
}

}  // namespace

size_t topk_workspace_bytes(int rows, int E, int k, int score_dtype) {
  if (E <= kChunk || k > kChunk) return 0;
  const int nchunks = (E + kChunk - 1) / kChunk;
  if ((size_t)nchunks * k > (size_t)kChunk) return 0;   // candidates must fit one CTA
  const size_t es = score_dtype == CSA_BF16 ? 2 : 4;
  return (size_t)rows * nchunks * k * (es + 4) + 256;
}

// Rows of up to kChunk entries: one CTA each.  Longer rows: chunk pass + candidate
// pass (needs ws of topk_workspace_bytes), as long as all candidates fit one CTA.
csa_status launch_topk_search(const void* scores, int score_dtype, const int32_t* q_pos, int m,
                              int rows, int E, int k, int32_t* idx, int32_t* count, void* ws,
                              size_t ws_bytes, cudaStream_t st, bool pdl) {
  if (rows == 0) return CSA_OK;
  if (k > kChunk) return CSA_ERR_UNSUPPORTED;
  const bool bf = score_dtype == CSA_BF16;
  if (E <= kChunk) {
    const int nt = threads_for(E);
    const cudaError_t e =
        bf ? csa_launch(topk_row_kernel<__nv_bfloat16>, dim3(rows), dim3(nt), 0, st, pdl,
                        reinterpret_cast<const __nv_bfloat16*>(scores), q_pos, m, E, k, idx, count)
           : csa_launch(topk_row_kernel<float>, dim3(rows), dim3(nt), 0, st, pdl,
                        reinterpret_cast<const float*>(scores), q_pos, m, E, k, idx, count);
    return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
  }
  const size_t need = topk_workspace_bytes(rows, E, k, score_dtype);
  if (need == 0) return CSA_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 15)) return CSA_ERR_UNSUPPORTED;
  const int nchunks = (E + kChunk - 1) / kChunk;
  const size_t ncand = (size_t)rows * nchunks * k;
  int32_t* cand_idx = static_cast<int32_t*>(ws);
  void* cand_sc = cand_idx + ncand;
  const int nt2 = threads_for(nchunks * k);
  cudaError_t e;
  if (bf) {
    e = csa_launch(topk_chunk_kernel<__nv_bfloat16>, dim3(rows * nchunks), dim3(kNT), 0, st, pdl,
                   reinterpret_cast<const __nv_bfloat16*>(scores), q_pos, m, E, k, nchunks,
                   static_cast<__nv_bfloat16*>(cand_sc), cand_idx);
    if (e == cudaSuccess)
      e = csa_launch(topk_merge_kernel<__nv_bfloat16>, dim3(rows), dim3(nt2), 0, st, pdl,
                     static_cast<const __nv_bfloat16*>(cand_sc), (const int32_t*)cand_idx, q_pos,
                     m, E, k, nchunks, idx, count);
  } else {
    e = csa_launch(topk_chunk_kernel<float>, dim3(rows * nchunks), dim3(kNT), 0, st, pdl,
                   reinterpret_cast<const float*>(scores), q_pos, m, E, k, nchunks,
                   static_cast<float*>(cand_sc), cand_idx);
    if (e == cudaSuccess)
      e = csa_launch(topk_merge_kernel<float>, dim3(rows), dim3(nt2), 0, st, pdl,
                     static_cast<const float*>(cand_sc), (const int32_t*)cand_idx, q_pos, m, E, k,
                     nchunks, idx, count);
  }
  return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

}  // namespace csa
