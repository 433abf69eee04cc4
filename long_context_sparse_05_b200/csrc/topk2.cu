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
// Few long rows (decode: one query per sequence) spread each row over a thread-block
// cluster of 2..16 CTAs, each holding a contiguous slice, and every count is a cluster
// sum: warp 0 of each CTA pushes its counts into every CTA's shared memory with
// st.async, counted on the receiver's mbarrier, so a round costs one one-way message
// instead of a cluster barrier plus remote reads.  bf16 rows take two rounds of 256
// buckets (the top byte of the 16-bit key, then the low byte) when each thread holds 8
// keys, and the two histograms of every rank also give each CTA the keys above / equal
// to tau of the lower ranks; otherwise (fp32 rows, 32 keys per thread) the candidate
// range splits into 16 power-of-two buckets per round and those counts are exchanged
// once more at the end.  Either way the selection comes out in ascending entry order.
//
// Rows longer than a cluster holds (16 x 16384) are cut into chunks: every chunk
// keeps its own top-k (the global top-k is contained in the union, and since chunks
// are contiguous index ranges the lowest-index rule for ties carries over), and a
// second pass selects the top-k of the candidates.
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace csa {

namespace {

constexpr int kEPT = 32;            // entries per thread
constexpr int kNT = 512;            // threads of the largest CTA
constexpr int kChunk = kNT * kEPT;  // entries one CTA holds
constexpr int kMaxClusterRanks = 16;       // CTAs of the largest (non-portable) cluster

template <typename S> struct Keys;
template <> struct Keys<__nv_bfloat16> {
  using Bits = uint16_t;
  static constexpr Bits kSentinel = 0xffffu;   // pattern whose key is 0: below every score
  __device__ static __forceinline__ uint32_t key(uint32_t u) {
    if ((u & 0x7fffu) == 0) u = 0;   // -0 ties with +0
    return (u & 0x8000u) ? (~u & 0xffffu) : (u | 0x8000u);
  }
};
template <> struct Keys<float> {
  using Bits = uint32_t;
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

// ---- cluster path -----------------------------------------------------------

__device__ __forceinline__ uint32_t cl_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cl_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cl_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cl_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cl_map(const void* local, uint32_t rank) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(ra) : "r"(tc::smem_u32(local)), "r"(rank));
  return ra;
}
// 16-byte store into another CTA's shared memory, counted on that CTA's mbarrier.
__device__ __forceinline__ void st_async16(uint32_t raddr, uint4 v, uint32_t rbar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];"
      ::"r"(raddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(rbar) : "memory");
}

constexpr int kMsgWords = 8;   // one message: 8 words (16 bucket counts of 16 bits)

// Cluster exchange number `ex`: warp 0 of every CTA pushes its message (held by every
// lane of warp 0) into row `rank` of receive slot (ex & 1) of every CTA of the
// cluster; every thread then waits, bounded, for its own slot to hold all cs rows.
// Slot reuse is safe: a CTA sends exchange ex + 2 only after it received exchange
// ex + 1 from every CTA, and a CTA sends exchange ex + 1 only after a block barrier
// that follows all of its reads of exchange ex.
__device__ __forceinline__ bool cl_push(const uint4 (&msg)[2], uint32_t* s_slot, uint64_t* s_bar,
                                        int ex, uint32_t cs, uint32_t rank, int* err) {
  const int slot = ex & 1;
  uint32_t* row = s_slot + (slot * kMaxClusterRanks + rank) * kMsgWords;
  uint64_t* bar = s_bar + slot;
  if (threadIdx.x == 0) tc::mbar_arrive_expect_tx(bar, cs * kMsgWords * 4);
  if (threadIdx.x < cs) {
    const uint32_t rrow = cl_map(row, threadIdx.x), rbar = cl_map(bar, threadIdx.x);
    st_async16(rrow, msg[0], rbar);
    st_async16(rrow + 16, msg[1], rbar);
  }
  return tc::mbar_wait(bar, (ex >> 1) & 1, err);
}
// Lane l < cs of the calling warp gets row l of receive slot (ex & 1); other lanes zeros.
__device__ __forceinline__ void cl_row(const uint32_t* s_slot, int ex, uint32_t cs, uint4 (&r)[2]) {
  const uint32_t lane = threadIdx.x & 31;
  if (lane < cs) {
    const uint4* p = reinterpret_cast<const uint4*>(
        s_slot + ((ex & 1) * kMaxClusterRanks + lane) * kMsgWords);
    r[0] = p[0];
    r[1] = p[1];
  } else {
    r[0] = r[1] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// One row over a cluster: CTA `rank` holds entries [rank * per, rank * per + per) of
// the row's `ev` visible entries, EPT consecutive entries per thread.  The search
// keeps the invariant of the single-CTA search (at least k keys >= lo, fewer than k
// keys > hi) but splits [lo, hi] into 16 power-of-two buckets per round: bucket
// b(key) = min((key - lo) >> s, 15) with 16 << s covering the range, so a round
// leaves a range of at most 2^s keys and ends on the exact k-th key when s = 0.
template <typename S, int EPT>
__global__ void __launch_bounds__(kNT) topk_cluster_kernel(
    const S* __restrict__ scores, const int32_t* __restrict__ q_pos, int m, int E, int k, int per,
    int32_t* __restrict__ idx, int32_t* __restrict__ count, int* err) {
  using K = Keys<S>;
  using Bits = typename K::Bits;
  static_assert(EPT % 8 == 0, "keys are counted in groups of 8");
  __shared__ __align__(16) uint32_t s_part[kNT / 32][kMsgWords];   // warp partial sums
  __shared__ __align__(16) uint32_t s_slot[2 * kMaxClusterRanks * kMsgWords];
  __shared__ __align__(8) uint64_t s_bar[2];
  __shared__ uint32_t s_sc[32];
  const uint32_t cs = cl_size(), rank = cl_rank();
  const int tid = threadIdx.x, NT = blockDim.x;
  const int lane = tid & 31, wid = tid >> 5, nw = NT >> 5;
  if (tid == 0) {
    tc::mbar_init(&s_bar[0], 1);
    tc::mbar_init(&s_bar[1], 1);
    tc::fence_barrier_init();
  }
  cl_arrive();                                   // barriers initialised before any push
  pdl_launch_dependents();
  pdl_wait();
  const int row = blockIdx.x / cs;
  const int base = (int)rank * per;
  const Bits* bits = reinterpret_cast<const Bits*>(scores + (size_t)row * E + base);
  const int nl = max(0, min(E - base, per));     // entries of this slice in the row
  const int j0 = tid * EPT;

  // keys first (independent of the query position), then the visible count
  uint32_t key[EPT];
  const bool vec = ((reinterpret_cast<uintptr_t>(bits + j0) & 15) == 0) && j0 + EPT <= nl;
  if (vec) {
    constexpr int kPer = 16 / sizeof(Bits);
#pragma unroll
    for (int v = 0; v < EPT / kPer; ++v) {
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(bits + j0) + v);
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if constexpr (sizeof(Bits) == 2) {
          key[v * kPer + 2 * i] = w[i] & 0xffffu;
          key[v * kPer + 2 * i + 1] = w[i] >> 16;
        } else {
          key[v * kPer + i] = w[i];
        }
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < EPT; ++e) key[e] = j0 + e < nl ? bits[j0 + e] : 0u;
  }
  const int ev = visible_entries(q_pos[row], m, E);
  const int n = max(0, min(ev - base, per));     // this CTA's visible entries
#pragma unroll
  for (int e = 0; e < EPT; ++e) key[e] = j0 + e < n ? K::key(key[e]) : 0u;   // past n: key 0

  int32_t* out = idx + (size_t)row * k;
  if (ev <= k) {                                 // everything visible is kept
    for (int j = (int)rank * NT + tid; j < k; j += (int)cs * NT) out[j] = j < ev ? j : -1;
    if (rank == 0 && tid == 0) count[row] = ev;
    cl_wait();
    return;
  }

  int ex = 0;
  uint4 msg[2], r[2];
  // cluster-wide [min, max] of the valid keys
  {
    uint32_t kmin = 0xffffffffu, kmax = 0;
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      const bool v = j0 + e < n;
      kmin = v ? min(kmin, key[e]) : kmin;
      kmax = v ? max(kmax, key[e]) : kmax;
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) { s_part[wid][0] = kmin; s_part[wid][1] = kmax; }
    __syncthreads();
    if (wid == 0) {
      const uint32_t a = lane < nw ? s_part[lane][0] : 0xffffffffu;
      const uint32_t b = lane < nw ? s_part[lane][1] : 0u;
      msg[0] = make_uint4(__reduce_min_sync(0xffffffffu, a), __reduce_max_sync(0xffffffffu, b), 0u, 0u);
      msg[1] = make_uint4(0u, 0u, 0u, 0u);
    }
    cl_wait();                                   // every CTA's barriers are initialised
    cl_push(msg, s_slot, s_bar, ex, cs, rank, err);
    cl_row(s_slot, ex, cs, r);
    ++ex;
    const bool in = (uint32_t)lane < cs;
    kmin = __reduce_min_sync(0xffffffffu, in ? r[0].x : 0xffffffffu);
    kmax = __reduce_max_sync(0xffffffffu, in ? r[0].y : 0u);
    kmin = min(kmin, kmax);                      // (only a failed exchange leaves kmin > kmax)
    msg[0].x = kmin;                             // lo / hi below
    msg[0].y = kmax;
  }
  uint32_t lo = msg[0].x, hi = msg[0].y;
  int rounds = 0;
  while (lo < hi && rounds < 8) {                // 8 rounds resolve any 32-bit range
    ++rounds;
    const int p = 32 - __clz(hi - lo);           // 2^p > hi - lo
    const int sh = max(p - 4, 0);
    // bucket counts: 4-bit fields per group of 8 keys, widened to bytes, then to 16 bits
    uint32_t ev_lo = 0, od_lo = 0, ev_hi = 0, od_hi = 0;   // byte fields: even / odd buckets
#pragma unroll
    for (int g = 0; g < EPT / 8; ++g) {
      uint32_t a_lo = 0, a_hi = 0;               // buckets 0-7 / 8-15, 4 bits each
#pragma unroll
      for (int e = g * 8; e < g * 8 + 8; ++e) {
        const uint32_t kk = key[e];
        const uint32_t b = min((kk - lo) >> sh, 15u);
        const uint32_t t = 1u << ((b & 7u) << 2);
        const bool v = kk >= lo;
        a_lo += (v && b < 8u) ? t : 0u;
        a_hi += (v && b >= 8u) ? t : 0u;
      }
      ev_lo += a_lo & 0x0f0f0f0fu;
      od_lo += (a_lo >> 4) & 0x0f0f0f0fu;
      ev_hi += a_hi & 0x0f0f0f0fu;
      od_hi += (a_hi >> 4) & 0x0f0f0f0fu;
    }
    // word j holds buckets 2j (low half) and 2j + 1 (high half)
    uint32_t wv[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      wv[j] = __byte_perm(ev_lo, od_lo, 0x4440u | j | (j << 8) | 0x0) & 0x00ff00ffu;
      wv[4 + j] = __byte_perm(ev_hi, od_hi, 0x4440u | j | (j << 8)) & 0x00ff00ffu;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) wv[j] = __reduce_add_sync(0xffffffffu, wv[j]);
    if (lane == 0) {
      *reinterpret_cast<uint4*>(&s_part[wid][0]) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      *reinterpret_cast<uint4*>(&s_part[wid][4]) = make_uint4(wv[4], wv[5], wv[6], wv[7]);
    }
    __syncthreads();
    if (wid == 0) {
      uint4 a = make_uint4(0u, 0u, 0u, 0u), b = a;
      for (int w = 0; w < nw; ++w) {
        const uint4 x = *reinterpret_cast<const uint4*>(&s_part[w][0]);
        const uint4 y = *reinterpret_cast<const uint4*>(&s_part[w][4]);
        a.x += x.x; a.y += x.y; a.z += x.z; a.w += x.w;
        b.x += y.x; b.y += y.y; b.z += y.z; b.w += y.w;
      }
      msg[0] = a;
      msg[1] = b;
    }
    cl_push(msg, s_slot, s_bar, ex, cs, rank, err);
    cl_row(s_slot, ex, cs, r);
    ++ex;
    // cluster totals per bucket (16 bits per CTA, summed in 32 bits), then the highest
    // bucket whose suffix count reaches k
    const uint32_t rw[8] = {r[0].x, r[0].y, r[0].z, r[0].w, r[1].x, r[1].y, r[1].z, r[1].w};
    uint32_t suffix = 0;
    int sel = 0;
    bool found = false;
#pragma unroll
    for (int b = 15; b >= 0; --b) {
      const uint32_t h = (b & 1) ? (rw[b >> 1] >> 16) : (rw[b >> 1] & 0xffffu);
      suffix += __reduce_add_sync(0xffffffffu, h);
      if (!found && suffix >= (uint32_t)k) { sel = b; found = true; }
    }
    const uint64_t top = (uint64_t)lo + ((uint64_t)(sel + 1) << sh) - 1;
    lo = lo + ((uint32_t)sel << sh);
    hi = (uint32_t)min((uint64_t)hi, top);
  }
  const uint32_t tau = lo;

  uint32_t gt_mask = 0, eq_mask = 0;
#pragma unroll
  for (int e = 0; e < EPT; ++e) {
    const bool v = j0 + e < n;
    gt_mask |= (v && key[e] > tau ? 1u : 0u) << e;
    eq_mask |= (v && key[e] == tau ? 1u : 0u) << e;
  }
  const uint32_t n_gt = __popc(gt_mask), n_eq = __popc(eq_mask);
  const uint32_t packed = n_gt | (n_eq << 16);
  // inclusive warp scan of (gt | eq << 16); warp totals to s_sc
  uint32_t x = packed;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_sc[wid] = x;
  __syncthreads();
  if (wid == 0) {
    uint32_t w = lane < nw ? s_sc[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    const uint32_t cta = __shfl_sync(0xffffffffu, w, 31);   // this CTA's (gt | eq << 16)
    msg[0] = make_uint4(cta, 0u, 0u, 0u);
    msg[1] = make_uint4(0u, 0u, 0u, 0u);
    if (lane < nw) s_sc[lane] = w;
  }
  cl_push(msg, s_slot, s_bar, ex, cs, rank, err);
  cl_row(s_slot, ex, cs, r);
  int need, G, Q;                                // k - keys above tau; lower ranks' gt / eq
  {
    const bool lower = (uint32_t)lane < rank;
    need = k - (int)__reduce_add_sync(0xffffffffu, r[0].x & 0xffffu);
    G = (int)__reduce_add_sync(0xffffffffu, lower ? (r[0].x & 0xffffu) : 0u);
    Q = (int)__reduce_add_sync(0xffffffffu, lower ? (r[0].x >> 16) : 0u);
  }
  cl_arrive();                                   // no CTA leaves before all pushes landed

  const uint32_t excl = (wid > 0 ? s_sc[wid - 1] : 0u) + x - packed;
  const int gt_before = G + (int)(excl & 0xffffu);
  const int eq_before = Q + (int)(excl >> 16);
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
    if (pos >= 0 && pos < k) out[pos] = base + j0 + e;
    ++pos;
  }
  if (rank == 0 && tid == 0) count[row] = k;
  cl_wait();
}

// bf16 rows over a cluster, in two rounds of 256 buckets: the top byte of the 16-bit key
// over all visible keys, then the low byte over the keys whose top byte is the chosen
// one, give the exact k-th key tau.  Each round's message is a CTA's 256 bucket counts
// (16 bits each), pushed into every CTA of the cluster, so every CTA keeps every CTA's
// two histograms: the keys above / equal to tau of the lower ranks (for the ascending
// output) follow from them without a further exchange.
constexpr int kHistWords = 128;   // 256 counts of 16 bits

// Bucket counts of this warp into its own histogram s_wh (zeroed; shared atomics, so
// only lanes of one warp contend).  Round A (top < 0): bucket = key >> 8 over the
// visible keys; round B: bucket = key & 255 over the visible keys with key >> 8 == top.
template <int EPT>
__device__ __forceinline__ void hist256(const uint32_t (&key)[EPT], int j0, int n, int top,
                                        uint32_t* s_wh) {
#pragma unroll
  for (int e = 0; e < EPT; ++e) {
    const uint32_t kk = key[e];
    const bool act = j0 + e < n && (top < 0 || (int)(kk >> 8) == top);
    if (act) atomicAdd(&s_wh[top < 0 ? (kk >> 8) : (kk & 255u)], 1u);
  }
}
// CTA histogram s_hist[b] = sum over the warps' histograms, each warp's zeroed again.
__device__ __forceinline__ void sum_warp_hists(uint32_t* s_wh, uint32_t* s_hist, int nw) {
  for (int b = threadIdx.x; b < 256; b += blockDim.x) {
    uint32_t t = 0;
    for (int w = 0; w < nw; ++w) { t += s_wh[w * 256 + b]; s_wh[w * 256 + b] = 0u; }
    s_hist[b] = t;
  }
}

// Warp 0: this CTA's histogram (16-bit counts, lane l: buckets 8l .. 8l + 7) into row
// `rank` of slot `slot` of every CTA of the cluster, counted on that CTA's s_bar[slot].
__device__ __forceinline__ void push_hist(const uint32_t* s_hist, uint32_t* s_msg, uint64_t* s_bar,
                                          int slot, uint32_t cs, uint32_t rank) {
  const int lane = threadIdx.x & 31;
  const uint4 a = *reinterpret_cast<const uint4*>(s_hist + 8 * lane);
  const uint4 b = *reinterpret_cast<const uint4*>(s_hist + 8 * lane + 4);
  const uint4 v = make_uint4(a.x | (a.y << 16), a.z | (a.w << 16), b.x | (b.y << 16), b.z | (b.w << 16));
  uint32_t* row = s_msg + (slot * kMaxClusterRanks + rank) * kHistWords + 4 * lane;
  for (uint32_t r = 0; r < cs; ++r) st_async16(cl_map(row, r), v, cl_map(&s_bar[slot], r));
}

// Warp 0, after slot `slot` holds all cs histograms: the bucket B holding the krem-th
// largest key (buckets above it hold fewer than krem keys, B and above at least krem)
// and the count of keys in the buckets above B (every lane gets both).
__device__ __forceinline__ void pick_bucket(const uint32_t* s_msg, int slot, uint32_t cs,
                                            uint32_t krem, uint32_t& B, uint32_t& above_B) {
  const int lane = threadIdx.x & 31;
  uint32_t t[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  for (uint32_t r = 0; r < cs; ++r) {
    const uint4 v = *reinterpret_cast<const uint4*>(s_msg + (slot * kMaxClusterRanks + r) * kHistWords + 4 * lane);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) { t[2 * i] += w[i] & 0xffffu; t[2 * i + 1] += w[i] >> 16; }
  }
  uint32_t tot = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) tot += t[i];
  uint32_t suf = tot;                              // keys in the buckets of lanes >= this one
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, suf, o);
    if (lane + o < 32) suf += y;
  }
  const uint32_t higher = suf - tot;               // keys in the buckets of lanes above
  uint32_t b_here = 0, above_here = 0;
  const bool mine = higher < krem && suf >= krem;
  if (mine) {
    uint32_t s = higher;
#pragma unroll
    for (int i = 7; i >= 0; --i) {
      if (s + t[i] >= krem) { b_here = 8 * lane + i; above_here = s; break; }
      s += t[i];
    }
  }
  const uint32_t who = __ballot_sync(0xffffffffu, mine);
  const int src = who ? __ffs(who) - 1 : 0;
  B = __shfl_sync(0xffffffffu, b_here, src);
  above_B = __shfl_sync(0xffffffffu, above_here, src);
}

template <int EPT>
__global__ void __launch_bounds__(kNT) topk_cluster256_kernel(
    const __nv_bfloat16* __restrict__ scores, const int32_t* __restrict__ q_pos, int m, int E, int k,
    int per, int32_t* __restrict__ idx, int32_t* __restrict__ count, int* err) {
  using K = Keys<__nv_bfloat16>;
  static_assert(EPT % 8 == 0, "keys are loaded in groups of 8");
  __shared__ __align__(16) uint32_t s_hist[256];
  __shared__ __align__(16) uint32_t s_wh[kNT / 32 * 256];                     // per-warp histograms
  __shared__ __align__(16) uint32_t s_msg[2 * kMaxClusterRanks * kHistWords];
  __shared__ __align__(8) uint64_t s_bar[2];
  __shared__ uint32_t s_sc[32];
  __shared__ uint32_t s_sel[4];
  const uint32_t cs = cl_size(), rank = cl_rank();
  const int tid = threadIdx.x, NT = blockDim.x;
  const int lane = tid & 31, wid = tid >> 5, nw = NT >> 5;
  if (tid == 0) {
    // each slot is used once: both expect every rank's histogram
    tc::mbar_init(&s_bar[0], 1);
    tc::mbar_init(&s_bar[1], 1);
    tc::fence_barrier_init();
    tc::mbar_arrive_expect_tx(&s_bar[0], cs * kHistWords * 4);
    tc::mbar_arrive_expect_tx(&s_bar[1], cs * kHistWords * 4);
  }
  for (int i = tid; i < nw * 256; i += NT) s_wh[i] = 0u;
  cl_arrive();                                   // barriers initialised before any push
  pdl_launch_dependents();
  pdl_wait();
  const int row = blockIdx.x / cs;
  const int base = (int)rank * per;
  const uint16_t* bits = reinterpret_cast<const uint16_t*>(scores + (size_t)row * E + base);
  const int nl = max(0, min(E - base, per));     // entries of this slice in the row
  const int j0 = tid * EPT;

  uint32_t key[EPT];
  const bool vec = ((reinterpret_cast<uintptr_t>(bits + j0) & 15) == 0) && j0 + EPT <= nl;
  if (vec) {
#pragma unroll
    for (int v = 0; v < EPT / 8; ++v) {
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(bits + j0) + v);
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        key[v * 8 + 2 * i] = w[i] & 0xffffu;
        key[v * 8 + 2 * i + 1] = w[i] >> 16;
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < EPT; ++e) key[e] = j0 + e < nl ? bits[j0 + e] : 0u;
  }
  const int ev = visible_entries(q_pos[row], m, E);
  const int n = max(0, min(ev - base, per));     // this CTA's visible entries
#pragma unroll
  for (int e = 0; e < EPT; ++e) key[e] = j0 + e < n ? K::key(key[e]) : 0u;

  int32_t* out = idx + (size_t)row * k;
  if (ev <= k) {                                 // everything visible is kept
    for (int j = (int)rank * NT + tid; j < k; j += (int)cs * NT) out[j] = j < ev ? j : -1;
    if (rank == 0 && tid == 0) count[row] = ev;
    cl_wait();
    return;
  }

  // round A: the top byte
  __syncthreads();                               // the warp histograms are zeroed
  hist256<EPT>(key, j0, n, -1, s_wh + wid * 256);
  __syncthreads();
  sum_warp_hists(s_wh, s_hist, nw);
  __syncthreads();
  cl_wait();                                     // every CTA's barriers are initialised
  if (wid == 0) push_hist(s_hist, s_msg, s_bar, 0, cs, rank);
  if (wid == 0) {
    const bool got = tc::mbar_wait(&s_bar[0], 0, err);
    uint32_t B0, aboveA;
    pick_bucket(s_msg, 0, cs, (uint32_t)k, B0, aboveA);
    if (lane == 0) { s_sel[0] = got ? B0 : 0u; s_sel[1] = aboveA; }
  }
  __syncthreads();
  const uint32_t B0 = s_sel[0], aboveA = s_sel[1];
  // round B: the low byte among the keys with top byte B0
  hist256<EPT>(key, j0, n, (int)B0, s_wh + wid * 256);
  __syncthreads();
  sum_warp_hists(s_wh, s_hist, nw);
  __syncthreads();
  if (wid == 0) push_hist(s_hist, s_msg, s_bar, 1, cs, rank);
  if (wid == 0) {
    const bool got = tc::mbar_wait(&s_bar[1], 0, err);
    uint32_t B1, aboveB;
    pick_bucket(s_msg, 1, cs, (uint32_t)k - aboveA, B1, aboveB);
    // keys above / equal to tau of the ranks below this one, from their histograms
    uint32_t G = 0, Q = 0;
    for (uint32_t r = 0; r < rank; ++r) {
      const uint4 a = *reinterpret_cast<const uint4*>(s_msg + (0 * kMaxClusterRanks + r) * kHistWords + 4 * lane);
      const uint4 b = *reinterpret_cast<const uint4*>(s_msg + (1 * kMaxClusterRanks + r) * kHistWords + 4 * lane);
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
      uint32_t g = 0, q = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t bin = 8 * lane + i;
        const uint32_t ca = (i & 1) ? (wa[i >> 1] >> 16) : (wa[i >> 1] & 0xffffu);
        const uint32_t cb = (i & 1) ? (wb[i >> 1] >> 16) : (wb[i >> 1] & 0xffffu);
        g += (bin > B0 ? ca : 0u) + (bin > B1 ? cb : 0u);
        q += bin == B1 ? cb : 0u;
      }
      G += __reduce_add_sync(0xffffffffu, g);
      Q += __reduce_add_sync(0xffffffffu, q);
    }
    if (lane == 0) {
      s_sel[0] = got ? ((B0 << 8) | B1) : 0xffffffffu;
      s_sel[1] = aboveA + aboveB;                // keys above tau in the row
      s_sel[2] = G;
      s_sel[3] = Q;
    }
  }
  __syncthreads();
  cl_arrive();                                   // every push into this CTA has landed
  const uint32_t tau = s_sel[0];
  const int need = k - (int)s_sel[1];            // keys equal to tau to take, lowest first
  const int G = (int)s_sel[2], Q = (int)s_sel[3];

  uint32_t gt_mask = 0, eq_mask = 0;
#pragma unroll
  for (int e = 0; e < EPT; ++e) {
    const bool v = j0 + e < n;
    gt_mask |= (v && key[e] > tau ? 1u : 0u) << e;
    eq_mask |= (v && key[e] == tau ? 1u : 0u) << e;
  }
  const uint32_t n_gt = __popc(gt_mask), n_eq = __popc(eq_mask);
  const uint32_t packed = n_gt | (n_eq << 16);
  uint32_t x = packed;                           // inclusive warp scan, warp totals to s_sc
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_sc[wid] = x;
  __syncthreads();
  if (wid == 0) {
    uint32_t w = lane < nw ? s_sc[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) s_sc[lane] = w;
  }
  __syncthreads();
  const uint32_t excl = (wid > 0 ? s_sc[wid - 1] : 0u) + x - packed;
  const int gt_before = G + (int)(excl & 0xffffu);
  const int eq_before = Q + (int)(excl >> 16);
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
    if (pos >= 0 && pos < k) out[pos] = base + j0 + e;
    ++pos;
  }
  if (rank == 0 && tid == 0) count[row] = k;
  cl_wait();
}

int threads_for(int n) {
  const int nt = (n + kEPT - 1) / kEPT;
  return nt <= 128 ? 128 : (nt <= 256 ? 256 : 512);
}

constexpr int kMinPerCta = 2048;   // below this a CTA's rounds cost less than a cluster barrier

int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return sms;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

// The cluster kernel of a score type and slice: two 256-bucket rounds for bf16 slices of
// 8 keys per thread; the 16-bucket search for fp32 and for 32 keys per thread (there
// the per-warp histograms of the first round contend more than the extra rounds cost).
template <typename S, int EPT> struct ClusterKernel {
  static constexpr auto fn = topk_cluster_kernel<S, EPT>;
};
template <> struct ClusterKernel<__nv_bfloat16, 8> {
  static constexpr auto fn = topk_cluster256_kernel<8>;
};

template <typename S, int EPT>
cudaError_t prep_cluster_kernel(int cs) {
  if (cs > 8)
    return cudaFuncSetAttribute(ClusterKernel<S, EPT>::fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return cudaSuccess;
}

// Whether one cluster of `cs` CTAs of `nt` threads fits the device (cached per device).
bool cluster_fits(int cs, int nt, bool bf, int ept) {
  static int cache[16][2][2][kMaxClusterRanks + 1][5] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) return false;
  const int ti = nt <= 32 ? 0 : nt <= 64 ? 1 : nt <= 128 ? 2 : nt <= 256 ? 3 : 4;
  int& c = cache[dev][bf][ept == 32][cs][ti];
  if (c) return c > 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs);
  cfg.blockDim = dim3(nt);
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = cs;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  cudaError_t e;
  if (bf) {
    e = ept == 32 ? prep_cluster_kernel<__nv_bfloat16, 32>(cs) : prep_cluster_kernel<__nv_bfloat16, 8>(cs);
    if (e == cudaSuccess)
      e = ept == 32 ? cudaOccupancyMaxActiveClusters(&n, ClusterKernel<__nv_bfloat16, 32>::fn, &cfg)
                    : cudaOccupancyMaxActiveClusters(&n, ClusterKernel<__nv_bfloat16, 8>::fn, &cfg);
  } else {
    e = ept == 32 ? prep_cluster_kernel<float, 32>(cs) : prep_cluster_kernel<float, 8>(cs);
    if (e == cudaSuccess)
      e = ept == 32 ? cudaOccupancyMaxActiveClusters(&n, ClusterKernel<float, 32>::fn, &cfg)
                    : cudaOccupancyMaxActiveClusters(&n, ClusterKernel<float, 8>::fn, &cfg);
  }
  if (e != cudaSuccess) { cudaGetLastError(); n = 0; }
  c = n > 0 ? 2 : 1;
  return n > 0;
}

enum TopkMode { kRow, kCluster, kChunked, kNone };
struct TopkPlan {
  TopkMode mode;
  int cs, ept, per, nt;   // cluster path: CTAs per row, entries per thread / per CTA, threads
};

// Rows of up to kChunk entries with enough rows to fill the device: one CTA each.
// Fewer, longer rows: a cluster per row, as many CTAs as the device has SMs for (at
// least ceil(E / kChunk), at most 16, at least kMinPerCta entries each).  Rows beyond
// a 16-CTA cluster: chunk pass + candidate pass, if the candidates fit one CTA.
TopkPlan topk_plan(int rows, int E, int k, bool bf) {
  TopkPlan p{kNone, 1, kEPT, kChunk, kNT};
  if (k > kChunk) return p;
  const int sms = sm_count();
  int need = 1;
  while (need * kChunk < E) need *= 2;            // CTAs a row needs at the least
  int cs = 1;
  while (cs * 2 <= kMaxClusterRanks && (long long)rows * cs * 2 <= sms && (long long)E >= (long long)cs * 2 * kMinPerCta)
    cs *= 2;
  cs = max(cs, need);
  while (cs > 1 && cs <= kMaxClusterRanks) {
    const int per0 = (E + cs - 1) / cs;
    const int ept = per0 <= 4096 ? 8 : kEPT;
    const int per = (per0 + 32 * ept - 1) / (32 * ept) * (32 * ept);
    const int nt = per / ept;
    if (cluster_fits(cs, nt, bf, ept)) return TopkPlan{kCluster, cs, ept, per, nt};
    if (cs / 2 < need) break;
    cs /= 2;
  }
  if (E <= kChunk) { p.mode = kRow; return p; }
  const int nchunks = (E + kChunk - 1) / kChunk;
  if ((size_t)nchunks * k <= (size_t)kChunk) p.mode = kChunked;
  return p;
}

}  // namespace

size_t topk_workspace_bytes(int rows, int E, int k, int score_dtype) {
  const bool bf = score_dtype == CSA_BF16;
  if (topk_plan(rows, E, k, bf).mode != kChunked) return 0;
  const int nchunks = (E + kChunk - 1) / kChunk;
  const size_t es = bf ? 2 : 4;
  return (size_t)rows * nchunks * k * (es + 4) + 256;
}

csa_status launch_topk_search(const void* scores, int score_dtype, const int32_t* q_pos, int m,
                              int rows, int E, int k, int32_t* idx, int32_t* count, void* ws,
                              size_t ws_bytes, cudaStream_t st, bool pdl) {
  if (rows == 0) return CSA_OK;
  const bool bf = score_dtype == CSA_BF16;
  const TopkPlan pl = topk_plan(rows, E, k, bf);
  if (pl.mode == kNone) return CSA_ERR_UNSUPPORTED;
  if (pl.mode == kRow) {
    const int nt = threads_for(E);
    const cudaError_t e =
        bf ? csa_launch(topk_row_kernel<__nv_bfloat16>, dim3(rows), dim3(nt), 0, st, pdl,
                        reinterpret_cast<const __nv_bfloat16*>(scores), q_pos, m, E, k, idx, count)
           : csa_launch(topk_row_kernel<float>, dim3(rows), dim3(nt), 0, st, pdl,
                        reinterpret_cast<const float*>(scores), q_pos, m, E, k, idx, count);
    return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
  }
  if (pl.mode == kCluster) {
    int* err = device_error_word();
    if (!err) return CSA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(rows * pl.cs);
    cfg.blockDim = dim3(pl.nt);
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = pl.cs;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = pdl ? 2 : 1;
    cudaError_t e;
    if (bf) {
      const auto* sc = reinterpret_cast<const __nv_bfloat16*>(scores);
      e = pl.ept == 32 ? cudaLaunchKernelEx(&cfg, ClusterKernel<__nv_bfloat16, 32>::fn, sc, q_pos, m,
                                            E, k, pl.per, idx, count, err)
                       : cudaLaunchKernelEx(&cfg, ClusterKernel<__nv_bfloat16, 8>::fn, sc, q_pos, m,
                                            E, k, pl.per, idx, count, err);
    } else {
      const auto* sc = reinterpret_cast<const float*>(scores);
      e = pl.ept == 32 ? cudaLaunchKernelEx(&cfg, topk_cluster_kernel<float, 32>, sc, q_pos, m, E, k,
                                            pl.per, idx, count, err)
                       : cudaLaunchKernelEx(&cfg, topk_cluster_kernel<float, 8>, sc, q_pos, m, E, k,
                                            pl.per, idx, count, err);
    }
    return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
  }
  const size_t need = topk_workspace_bytes(rows, E, k, score_dtype);
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
