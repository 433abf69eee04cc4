// Shared-latent MQA with sliding window and sink on the tcgen05 tensor cores
// (sm_100a), for 64 heads of 512 dims in bf16.
//
// Method: "DeepSeek Technical Reports", section DSA (attention over the top-k
// entries) and section CSA (raw sliding window); "DeepSeek V4 结构速览",
// sections "CSA（c4a 路线）" (selected entries concatenated with the window
// rows; one 512-dim latent is K and V for all 64 heads) and "HCA（c128a 路线）"
// (dense over every entry; attention sink).
//
// One query's rows (selected entries, then window rows) are cut into tiles of
// 128 rows.  A tile is gathered with cp.async into shared memory as eight
// 128-byte-swizzled column blocks [128 rows x 64 dims]; the same bytes are
//   * the K-major A operand of  S^T[r, h] = KV[r] . q[h]      (M=128 rows, N=64 heads, K=512)
//   * the MN-major A operand of O^T[d, h] += V^T[d, r] P^T[r, h] (M=4x128 dims, N=64, K=128 rows)
// so every row is read from memory once.  S^T lands in TMEM with rows on lanes:
// the per-head max and sum over rows are warp transpose-reductions (62 shuffles
// for 64 heads) plus a combine in shared memory.  P^T is written to
// shared memory MN-major (row r's 64 heads are one swizzled 128-byte line).
// The running max is updated lazily (only when a tile's max exceeds it by 2^8),
// which rescales the O^T accumulator in TMEM.
//
// Work item = (query, split of its rows).  With one split the CTA writes the
// normalised output (the sink joins the denominator).  With several (CSA decode),
// the splits of one query form a thread-block cluster.  As soon as its last softmax is
// done, every split pushes its running max and sum per head to every rank (st.async
// into distributed shared memory, counted on the receiver's mbarrier), so while its PV
// still runs each rank forms the same log-sum-exp weights e^(M_j - M) / (e^sink +
// sum_i l_i e^(M_i - M)).  Each split then stages its O scaled by its own weight, as
// bf16, bulk-stores it to the workspace, the cluster synchronises (barrier.cluster,
// release / acquire), and every CTA bulk-loads one slice of the 512 output dims from
// every split and adds them, so no second kernel runs.  Dense decode (HCA, tens of
// splits) writes fp32 partials and a small merge kernel combines them.
//
// CTA (288 threads): warps 0-7 gather, read TMEM and run the softmax, two warps per
// TMEM lane quarter (warp w owns lanes 32 (w % 4).., 32 heads each); warp 8 lane 0
// issues every MMA.  Ordering uses named barriers (tile ready, P ready) and
// mbarriers signalled by tcgen05.commit (S ready; PV done per 128-dim block).  Within an
// item, the next tile is gathered column-block pair by pair as soon as the current PV
// has read that pair, and its S^T MMAs start on each pair as it lands, so the gather of
// tile j + 1 runs under the PV of tile j.
#include "kernels.h"
#include "tc_common.cuh"

#include <climits>
#include <cmath>

namespace csa {

namespace {

constexpr int kH = 64;            // heads
constexpr int kD = 512;           // head dim = latent dim
constexpr int kRows = 128;        // rows per tile (MMA M of S^T)
constexpr int kKVBlkBytes = kRows * 128;   // one column block of the KV tile: 16 KB
constexpr int kQBlkBytes = kH * 128;       // one column block of q: 8 KB
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThresh = 8.0f;     // log2 units
constexpr int kSW = 8;                     // gather / softmax warps (two per TMEM lane quarter)
constexpr int kThreadsA = 32 * kSW + 32;   // plus the MMA warp
constexpr int kST = 32 * kSW;              // softmax threads
constexpr uint32_t kWaitHintNs = 64;       // a parked mbarrier wait re-checks this often

struct AttnTc {
  const __nv_bfloat16* q; const __nv_bfloat16* kv; const int32_t* idx; const int32_t* count;
  const __nv_bfloat16* win; const int32_t* q_pos; const float* sink;
  __nv_bfloat16* out; float* lse;
  float* part_o; float* part_m; float* part_l;
  int* err;
  int T, n_w, m, k, E_cap, n, rows_total, nsplit, rps, dense;
  int cluster;   // nsplit > 1: 1 = the splits of a query are one cluster and merge inside
                 // the kernel; 0 = fp32 partials go to the workspace and attn_merge_kernel
                 // combines them
  uint8_t* part_bf;   // cluster mode: per item, the scaled O as bf16 [512][64] (swizzled rows)
  float scale_log2;
  int d_rope_out;     // inverse RoPE on the last d_rope_out output dims at the query position
  double inv_freq[kMaxOutRopePairs];   // theta^(-2j/d_rope_out)
  const int32_t* block_table;   // paged entries (see AttnArgs)
  int max_pages, num_pages, win_ring;
};

// sin / cos of the inverse-RoPE angle of output dim d at position t (identity below the
// rotary dims)
__device__ __forceinline__ void out_rope_sincos(const AttnTc& p, int d, int t, float& sn, float& cs) {
  sn = 0.f; cs = 1.f;
  const int u = d - (kD - p.d_rope_out);
  if (p.d_rope_out > 0 && u >= 0) rope_angle((double)t * p.inv_freq[u >> 1], &sn, &cs);
}

struct QInfo {
  int sb, t, nsel, w0, nrows;
};

__device__ __forceinline__ QInfo query_info(const AttnTc& p, int qrow) {
  QInfo Q;
  Q.sb = qrow / p.T;
  Q.t = min(max(p.q_pos[qrow], 0), p.n - 1);
  int ns = p.dense ? visible_entries(Q.t, p.m, p.E_cap) : p.count[qrow];
  Q.nsel = max(0, min(ns, p.dense ? p.E_cap : p.k));
  Q.w0 = max(0, Q.t - p.n_w + 1);
  Q.nrows = Q.nsel + (Q.t - Q.w0 + 1);
  return Q;
}

// Source row of list position pos, or nullptr for a padded / invalid row.
__device__ __forceinline__ const __nv_bfloat16* row_src(const AttnTc& p, const QInfo& Q, int qrow,
                                                        int pos, int e_pre = INT_MIN) {
  if (pos >= Q.nrows) return nullptr;
  if (pos < Q.nsel) {
    const int e = p.dense ? pos : e_pre != INT_MIN ? e_pre : p.idx[(size_t)qrow * p.k + pos];
    if (e < 0 || e >= p.E_cap) return nullptr;
    if (p.block_table) {
      const int pg = p.block_table[(size_t)Q.sb * p.max_pages + e / kPageEntries];
      if ((unsigned)pg >= (unsigned)p.num_pages) return nullptr;
      return p.kv + ((size_t)pg * kPageEntries + e % kPageEntries) * kD;
    }
    return p.kv + ((size_t)Q.sb * p.E_cap + e) * kD;
  }
  const int u = Q.w0 + (pos - Q.nsel);
  if (p.win_ring) return p.win + ((size_t)Q.sb * p.win_ring + u % p.win_ring) * kD;
  return p.win + ((size_t)Q.sb * p.n + u) * kD;
}

// Copy `nrows_blk` rows of 512 bf16 into the swizzled column-block layout.
// Warp w of the kSW gather warps copies rows w, w + kSW, ...; two 16-byte chunks per lane per row.
template <typename SrcFn>
__device__ __forceinline__ void gather_rows(uint8_t* dst, int blk_bytes, int nrows_blk, int gw,
                                            int lane, SrcFn src_of, const void* dummy) {
  for (int r = gw; r < nrows_blk; r += kSW) {
    const __nv_bfloat16* src = src_of(r);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = lane + 32 * h;          // 16-byte chunk 0..63 of the row
      const int cb = c >> 3, cc = c & 7;
      uint8_t* d = dst + cb * blk_bytes + r * 128 + ((cc ^ (r & 7)) << 4);
      if (src) tc::cp_async16(d, src + c * 8, 16);
      else tc::cp_async16(d, dummy, 0);
    }
  }
}

// Copy dims 128 mb .. 128 mb + 127 (column blocks 2 mb, 2 mb + 1) of the tile's rows:
// half a warp per row (256 contiguous source bytes), rows 2 w, 2 w + 1, 2 w + 16, ... for
// gather warp w.
__device__ __forceinline__ void gather_pair(uint8_t* dst, int mb, int gw, int lane,
                                            const __nv_bfloat16* const* rows, const void* dummy) {
  const int c = 16 * mb + (lane & 15);          // 16-byte chunk of the row
  const int cb = c >> 3, cc = c & 7;
  for (int r = 2 * gw + (lane >> 4); r < kRows; r += 2 * kSW) {
    const __nv_bfloat16* src = rows[r];
    uint8_t* d = dst + cb * kKVBlkBytes + r * 128 + ((cc ^ (r & 7)) << 4);
    if (src) tc::cp_async16(d, src + c * 8, 16);
    else tc::cp_async16(d, dummy, 0);
  }
}

// This thread's copies of a pair have landed: publish them to the tensor core and arrive
// at the pair's named barrier (the MMA warp syncs on it).
__device__ __forceinline__ void pair_landed(int id) {
  tc::fence_proxy_async();
  tc::tc_fence_before();
  tc::named_bar_arrive(id, kThreadsA);
}

// One halving step of the transpose-reduction: lanes with bit `OFF` set keep the
// upper half of their HALF live values, the others the lower half, and each
// combines what it keeps with what its partner sends.
template <bool kMax, int OFF, int HALF, int N>
__device__ __forceinline__ void xpose_step(float (&v)[N], int lane) {
  const bool hi = (lane & OFF) != 0;
#pragma unroll
  for (int i = 0; i < HALF; ++i) {
    const float send = hi ? v[i] : v[i + HALF];
    const float keep = hi ? v[i + HALF] : v[i];
    const float recv = __shfl_xor_sync(0xffffffffu, send, OFF);
    v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
  }
}

// Transpose-reduction of 32 values over the 32 lanes of a warp (31 shuffles):
// afterwards lane L holds the reduction of value L over the warp (v[0]).
template <bool kMax>
__device__ __forceinline__ void xpose_reduce32(float (&v)[32], int lane) {
  xpose_step<kMax, 16, 16>(v, lane);
  xpose_step<kMax, 8, 8>(v, lane);
  xpose_step<kMax, 4, 4>(v, lane);
  xpose_step<kMax, 2, 2>(v, lane);
  xpose_step<kMax, 1, 1>(v, lane);
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

constexpr int kMaxSplit = 16;         // splits of one query merged inside one cluster
constexpr int kMaxSplitGlobal = 32;   // splits of one query merged through the workspace

// Cluster merge.  Each split stores its O scaled by its log-sum-exp weight (bf16 [512
// dims][64 heads], the 16-byte chunk c of dim d's row at chunk c ^ (d & 7)) to the
// workspace with one bulk store; after a cluster barrier every rank bulk-loads, from
// every split, the rows of the dims it owns and adds them.  Shared memory (KV / query
// tile area, free once PV is done):
//   [0, 64 KB)           this split's scaled O, staged for the bulk store
//   [64 KB, 144 KB)      received slices: split j's rows of this rank's dims at slot j
constexpr int kCmRecvO = 64 * 1024;
constexpr size_t kPartB = (size_t)kD * kH * 2;   // one split's record
__device__ __forceinline__ int cm_chunk(int d, int chunk) { return chunk ^ (d & 7); }

__device__ __forceinline__ void bulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
               ::"l"(gdst), "r"(tc::smem_u32(ssrc)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Waits until this thread's committed bulk copies have completed (their writes performed).
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_load_g(void* sdst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(tc::smem_u32(sdst)), "l"(gsrc), "r"(bytes), "r"(tc::smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cl_map(const void* local, uint32_t rank) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(tc::smem_u32(local)), "r"(rank));
  return ra;
}
// 8-byte store into another CTA's shared memory, counted (bytes) on that CTA's mbarrier.
__device__ __forceinline__ void st_async8(uint32_t raddr, uint32_t a, uint32_t b, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];"
               ::"r"(raddr), "r"(a), "r"(b), "r"(rbar) : "memory");
}

// Dims of the output slice merged by cluster rank `rank`.
__device__ __forceinline__ void cm_slice(int ns, int rank, int& d0, int& d1) {
  const int dps = ((kD + ns - 1) / ns + 7) & ~7;
  d0 = min(kD, rank * dps);
  d1 = min(kD, d0 + dps);
}

// Merge of the splits of query `qrow` for output dims [d0, d1) (a multiple of 4 wide):
// out = sum_s e^{m_s} O_s / (e^{sink} + sum_s e^{m_s} l_s); every thread of the CTA joins.
// The partials are [split][dim][head] fp32; the slice of every split, and all running
// maxima and sums, are staged into shared memory with one batch of cp.async copies
// (one memory round trip), then combined there.
__device__ void merge_slice(const AttnTc& p, int qrow, int d0, int d1, bool write_lse,
                            uint8_t* stage /* >= nsplit * (d1 - d0) * 256 bytes */,
                            float* s_ml /* [2][cap][kH] */, float* s_mw /* [cap][kH] */,
                            int cap, const void* dummy) {
  const int tid = threadIdx.x;
  const int ns = p.nsplit;
  const int dsl = d1 - d0;
  const size_t it0 = (size_t)qrow * ns;
  // running maxima and sums: ns x 64 floats each, contiguous over the splits
  for (int c = tid; c < 2 * ns * 16; c += blockDim.x) {
    const int which = c / (ns * 16), cc = c % (ns * 16);
    const float* src = (which == 0 ? p.part_m : p.part_l) + it0 * kH + cc * 4;
    tc::cp_async16(s_ml + which * cap * kH + cc * 4, src, 16);
  }
  // the slice of every split: dsl x 64 floats, contiguous within a split
  const int cps = dsl * 16;                       // 16-byte chunks per split
  for (int c = tid; c < ns * cps; c += blockDim.x) {
    const int sp = c / cps, cc = c % cps;
    const float* src = p.part_o + ((it0 + sp) * kD + d0) * kH + cc * 4;
    tc::cp_async16(stage + ((size_t)sp * dsl * kH + cc * 4) * 4, dsl > 0 ? (const void*)src : dummy,
                   dsl > 0 ? 16 : 0);
  }
  tc::cp_async_wait_all();
  __syncthreads();
  if (tid < kH) {
    const int h = tid;
    const float sink2 = p.sink[h] * kLog2e;
    float M = sink2;
    for (int sp = 0; sp < ns; ++sp) M = fmaxf(M, s_ml[sp * kH + h]);
    float den = exp2f(sink2 - M);
    for (int sp = 0; sp < ns; ++sp) {
      const float ms = s_ml[sp * kH + h];
      const float e = ms == -INFINITY ? 0.f : exp2f(ms - M);
      s_mw[sp * kH + h] = e;
      den += s_ml[cap * kH + sp * kH + h] * e;
    }
    const float inv = 1.f / den;
    for (int sp = 0; sp < ns; ++sp) s_mw[sp * kH + h] *= inv;
    if (write_lse && p.lse) p.lse[(size_t)qrow * kH + h] = (M + log2f(den)) * 0.6931471805599453f;
  }
  __syncthreads();
  const float* st = reinterpret_cast<const float*>(stage);
  const int nd4 = dsl >> 2;
  for (int x = tid; x < kH * nd4; x += blockDim.x) {
    const int h = x % kH;                         // consecutive threads: consecutive heads
    const int dd = 4 * (x / kH);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int sp = 0; sp < ns; ++sp) {
      const float w = s_mw[sp * kH + h];
      if (w == 0.f) continue;   // an empty split leaves its partial O unwritten
      const float* src = st + ((size_t)sp * dsl + dd) * kH + h;
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u] = fmaf(src[u * kH], w, acc[u]);
    }
    if (p.d_rope_out > 0) {
      const int t = query_info(p, qrow).t;
#pragma unroll
      for (int u = 0; u < 4; u += 2) {
        float sn, cs;
        out_rope_sincos(p, d0 + dd + u, t, sn, cs);
        const float x0 = acc[u], x1 = acc[u + 1];
        acc[u] = inv_rope_elem(x0, x1, d0 + dd + u, kD, p.d_rope_out, sn, cs);
        acc[u + 1] = inv_rope_elem(x1, x0, d0 + dd + u + 1, kD, p.d_rope_out, sn, cs);
      }
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc[0], acc[1]);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc[2], acc[3]);
    uint2 u2;
    u2.x = *reinterpret_cast<uint32_t*>(&lo);
    u2.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(&p.out[((size_t)qrow * kH + h) * kD + d0 + dd]) = u2;
  }
}

// Cluster merge of query `qrow` (every thread of the CTA joins).  Each split bulk-stores
// its scaled O to the workspace; after the cluster barrier rank r bulk-loads, from every
// split, the rows of output dims [d0, d1) and adds them.
__device__ __forceinline__ void cluster_merge(const AttnTc& p, int qrow, int item, int rank,
                                              uint8_t* area, uint64_t* bar_r, bool ok,
                                              bool blocks_stored) {
  const int tid = threadIdx.x;
  const int ns = p.nsplit;
  int d0, d1;
  cm_slice(ns, rank, d0, d1);
  const int dsl = d1 - d0;
  const int dps = ((kD + ns - 1) / ns + 7) & ~7;
  // this split's record to the workspace (the rows were fenced for the async proxy): in
  // one copy, or already in flight as four blocks issued by threads 0 and kST / 2
  if (!blocks_stored) {
    if (tid == 0) {
      bulk_store(p.part_bf + (size_t)item * kPartB, area, kD * kH * 2);
      bulk_commit();
      bulk_wait_all();
      fence_proxy_async_global();
    }
  } else if (tid == 0 || tid == kST / 2) {
    bulk_wait_all();
    fence_proxy_async_global();
  }
  cluster_sync_all();   // every split's record is in the workspace
  if (tid == 0) {
    fence_proxy_async_global();
    tc::mbar_arrive_expect_tx(bar_r, (uint32_t)(ns * dsl * kH * 2));
    const size_t it0 = (size_t)qrow * ns;
    if (dsl > 0)
      for (int j = 0; j < ns; ++j)
        bulk_load_g(area + kCmRecvO + (size_t)j * dps * kH * 2,
                    p.part_bf + (it0 + j) * kPartB + (size_t)d0 * kH * 2, (uint32_t)(dsl * kH * 2),
                    bar_r);
  }
  // one thread waits for the slices and releases the others at a CTA barrier (threads
  // parked in an mbarrier wait resume late)
  const bool got = __syncthreads_and(tid == 0 ? tc::mbar_wait_hint(bar_r, 0, p.err, kWaitHintNs) : true);
  // thread = (chunk of 8 heads, dim); consecutive threads: consecutive dims, so each
  // split is one conflict-free 16-byte shared load per thread and each head's output
  // run is a coalesced store
  const __nv_bfloat16* recv = reinterpret_cast<const __nv_bfloat16*>(area + kCmRecvO);
  for (int x = tid; x < dsl * 8; x += blockDim.x) {
    const int c = x / dsl, dd = x - c * dsl;
    const int d = d0 + dd;
    const int off = dd * kH + cm_chunk(d, c) * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int j = 0; j < ns; ++j) {
      const uint4 v = *reinterpret_cast<const uint4*>(recv + (size_t)j * dps * kH + off);
      const uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&q[e]);
        acc[2 * e] += __low2float(b2);
        acc[2 * e + 1] += __high2float(b2);
      }
    }
    if (p.d_rope_out > 0) {
      // dims d and d ^ 1 (a rotary pair) sit in lanes x and x ^ 1, both active
      const unsigned mask = __activemask();
      float sn, cs;
      out_rope_sincos(p, d, query_info(p, qrow).t, sn, cs);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float y = __shfl_xor_sync(mask, acc[e], 1);
        acc[e] = inv_rope_elem(acc[e], y, d, kD, p.d_rope_out, sn, cs);
      }
    }
    __nv_bfloat16* o = p.out + ((size_t)qrow * kH + 8 * c) * kD + d;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      o[(size_t)e * kD] = __float2bfloat16_rn((ok && got) ? acc[e] : __int_as_float(0x7fc00000));
  }
}

// Workspace merge (dense decode with more splits than a cluster holds): CTA per
// (query, slice of 16 dims).
constexpr int kMergeDims = 16;
constexpr int kMergeThreads = 256;
__global__ void __launch_bounds__(kMergeThreads) attn_merge_kernel(AttnTc p) {
  extern __shared__ __align__(16) float mm_smem[];
  const int cap = p.nsplit;                               // shared memory sized for it
  float* s_ml = mm_smem;                                  // [2][cap][kH]
  float* s_mw = s_ml + 2 * cap * kH;                      // [cap][kH]
  uint8_t* stage = reinterpret_cast<uint8_t*>(s_mw + cap * kH);
  pdl_launch_dependents();
  pdl_wait();
  const int qrow = blockIdx.x;
  const int d0 = blockIdx.y * kMergeDims;
  merge_slice(p, qrow, d0, min(kD, d0 + kMergeDims), blockIdx.y == 0, stage, s_ml, s_mw,
              cap, p.q);
}

__global__ void __launch_bounds__(kThreadsA, 1) attn_tc_kernel(AttnTc p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sKV = base;                          // 8 x 16 KB
  uint8_t* sQ = sKV + 8 * kKVBlkBytes;          // 8 x 8 KB
  uint8_t* sP = sQ + 8 * kQBlkBytes;            // 16 KB: [128 rows][64 heads] bf16, swizzled
  float* s_red = reinterpret_cast<float*>(sP + kRows * 128);   // [4][64]
  float* s_M = s_red + 4 * kH;                  // running max (log2 units)
  float* s_Mu = s_M + kH;                       // max used for this tile
  float* s_alpha = s_Mu + kH;                   // rescale factor of this tile
  float* s_l = s_alpha + kH;                    // running sum
  int* s_flag = reinterpret_cast<int*>(s_l + kH);
  uint64_t* bar_s = reinterpret_cast<uint64_t*>(s_flag + 4);
  uint64_t* bar_pv = bar_s + 1;                 // [4]: PV of dim block mb done (3: all of O)
  uint64_t* bar_r = bar_pv + 4;                 // cluster merge: received slices
  uint64_t* bar_st = bar_r + 1;                 // cluster merge: maxima and sums received
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_st + 1);
  const __nv_bfloat16** s_rows = reinterpret_cast<const __nv_bfloat16**>(tmem_holder + 2);  // [128]
  float* s_stats = reinterpret_cast<float*>(                 // [kMaxSplit][kH][2]: (max, sum)
      (reinterpret_cast<uintptr_t>(s_rows + kRows) + 15) & ~(uintptr_t)15);
  float* s_sink2 = s_stats + kMaxSplit * kH * 2;             // [kH] sink logits, log2 units

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tid = threadIdx.x;

  pdl_launch_dependents();
  // the first item's query heads are an input of this call: fetch them before waiting
  // on the preceding kernels (selections, positions and caches come from those)
  const bool q_pre = (int)blockIdx.x < p.rows_total * p.nsplit && warp < kSW;
  if (q_pre) {
    const __nv_bfloat16* qb = p.q + (size_t)(blockIdx.x / p.nsplit) * kH * kD;
    gather_rows(sQ, kQBlkBytes, kH, warp, lane, [&](int h) { return qb + (size_t)h * kD; }, p.q);
  }
  if (tid < kH) s_sink2[tid] = p.sink[tid] * kLog2e;   // an input: read before the wait
  const int crank = p.cluster ? (int)cluster_rank() : 0;
  if (tid == 0) {
    tc::mbar_init(bar_s, 1);
    for (int i = 0; i < 4; ++i) tc::mbar_init(bar_pv + i, 1);
    tc::mbar_init(bar_r, 1);
    tc::mbar_init(bar_st, 1);
    tc::fence_barrier_init();
    // one item per CTA in cluster mode: the bytes of maxima and sums every rank pushes here
    if (p.cluster) tc::mbar_arrive_expect_tx(bar_st, (uint32_t)(p.nsplit * kH * 8));
  }
  if (warp == 0) tc::tmem_alloc(tmem_holder, 512);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  // every rank's barriers are initialised before any rank pushes into them
  if (p.cluster) cluster_sync_all();
  pdl_wait();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tS = tmem;            // columns [0, 64): S^T
  const uint32_t tO = tmem + 64;       // columns [64, 320): O^T, 4 blocks of 64

  const int items = p.rows_total * p.nsplit;
  uint32_t ns = 0;                     // commits waited on bar_s
  uint32_t npv = 0;                    // tiles whose PV commits were waited on (bar_pv)
  bool ok = true;
  bool q_ready = false;                // softmax warps: this item's query heads are on their way

  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int qrow = item / p.nsplit;
    const int split = item % p.nsplit;
    // the first tile's list entry of this thread's row is loaded alongside the query's
    // position and selection count (all three come from the preceding kernels)
    int e_pre = INT_MIN;
    if (warp < 4 && !p.dense) {
      const int pos0 = (item % p.nsplit) * p.rps + warp * 32 + lane;
      if (pos0 < p.k) e_pre = p.idx[(size_t)qrow * p.k + pos0];
    }
    const QInfo Q = query_info(p, qrow);
    // rows [rb, re) of the query's list, in sub-tiles of up to 128 rows
    const int rb = split * p.rps;
    const int re = min(rb + p.rps, Q.nrows);
    const int jb = 0;
    const int je = re > rb ? (re - rb + kRows - 1) / kRows : 0;

    if (warp == kSW) {
      // ---------------------------------------------------------------- MMA issuer
      constexpr uint32_t idS = tc::instr_desc(128, kH, 1, 1, 0, 0);   // bf16 K-major x K-major
      constexpr uint32_t idO = tc::instr_desc(128, kH, 1, 1, 1, 1);   // bf16 MN-major x MN-major
      // base descriptors; each MMA's operands are a constant byte offset from them
      const uint64_t dS_a = tc::smem_desc_sw128(tc::smem_u32(sKV), 16, 1024);
      const uint64_t dS_b = tc::smem_desc_sw128(tc::smem_u32(sQ), 16, 1024);
      const uint64_t dO_a = tc::smem_desc_sw128(tc::smem_u32(sKV), kKVBlkBytes, 1024);
      const uint64_t dO_b = tc::smem_desc_sw128(tc::smem_u32(sP), 8192, 1024);
      for (int j = jb; j < je; ++j) {
        // S^T by column-block pairs (dims 128 mb ..): the item's first tile (and q) arrives
        // whole, every later tile pair by pair as the previous tile's PV frees the pairs
        for (int mb = 0; mb < 4; ++mb) {
          if (j > jb) tc::named_bar(4 + mb, kThreadsA);
          else if (mb == 0) tc::named_bar(1, kThreadsA);
          if (lane == 0) {
            tc::tc_fence_after();
#pragma unroll
            for (int kb = 2 * mb; kb < 2 * mb + 2; ++kb) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t a = tc::desc_advance(dS_a, kb * kKVBlkBytes + kk * 32);
                const uint64_t b = tc::desc_advance(dS_b, kb * kQBlkBytes + kk * 32);
                tc::mma_f16(tS, a, b, idS, (kb | kk) != 0);
              }
            }
            if (mb == 3) tc::mma_commit(bar_s);
          }
          __syncwarp();
        }
        tc::named_bar(2, kThreadsA);                 // P^T in shared memory, O rescaled
        if (lane == 0) {
          tc::tc_fence_after();
#pragma unroll
          for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t a = tc::desc_advance(dO_a, 2 * mb * kKVBlkBytes + kk * 2048);
              const uint64_t b = tc::desc_advance(dO_b, kk * 2048);
              tc::mma_f16(tO + mb * kH, a, b, idO, (j > jb) || (kk > 0));
            }
            // every MMA so far is tracked: KV column blocks 2 mb, 2 mb + 1 are free once it fires
            tc::mma_commit(bar_pv + mb);
          }
        }
        __syncwarp();
      }
    } else {

    // ------------------------------------------------------ softmax warps 0..kSW-1
    // warps w and w + 4 share TMEM lane quarter w % 4 (tile rows); w / 4 picks the
    // 32 heads (S columns) and the two 128-dim O blocks this thread handles
    const int qd = warp & 3, hf = warp >> 2;
    const int r = qd * 32 + lane;                    // this thread's TMEM lane / tile row
    const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
    const bool have_q = (q_pre && item == (int)blockIdx.x) || q_ready;
    q_ready = false;
    if (tid < kH) { s_M[tid] = -INFINITY; s_l[tid] = 0.f; }
    if (je > jb) {
      // the item's first tile, whole (the previous item's O has been read: KV and P are free)
      if (!have_q) {
        const __nv_bfloat16* qb = p.q + (size_t)qrow * kH * kD;
        gather_rows(sQ, kQBlkBytes, kH, warp, lane,
                    [&](int h) { return qb + (size_t)h * kD; }, p.kv);
      }
      // source of every row of the tile: one coalesced pass over the index list
      if (hf == 0) {
        const int pos = rb + jb * kRows + r;
        s_rows[r] = pos < re ? row_src(p, Q, qrow, pos, e_pre) : nullptr;
      }
      tc::named_bar(3, kST);
      gather_rows(sKV, kKVBlkBytes, kRows, warp, lane, [&](int rr) { return s_rows[rr]; }, p.kv);
      tc::cp_async_wait_all();
      tc::fence_proxy_async();
      tc::tc_fence_before();
      tc::named_bar(1, kThreadsA);
    }
    for (int j = jb; j < je; ++j) {
      // the next tile's list entry of this thread's row, loaded behind this tile's S^T
      int e_nxt = INT_MIN;
      if (hf == 0 && !p.dense && j + 1 < je) {
        const int pn = rb + (j + 1) * kRows + r;
        if (pn < p.k) e_nxt = p.idx[(size_t)qrow * p.k + pn];
      }

      // logits of row r for this thread's 32 heads
      ok = ok && tc::mbar_wait_hint(bar_s, ns & 1, p.err, kWaitHintNs);
      ++ns;
      tc::tc_fence_after();
      if (j == je - 1 && p.nsplit == 1 && item + (int)gridDim.x < items) {
        // the last S^T of this item is done with the query heads: fetch the next
        // item's now, behind this tile's softmax, PV and the output (one split per
        // query only: with several, the cluster merge uses this shared memory)
        const __nv_bfloat16* qn = p.q + (size_t)(item + (int)gridDim.x) * kH * kD;
        gather_rows(sQ, kQBlkBytes, kH, warp, lane, [&](int h) { return qn + (size_t)h * kD; }, p.q);
        q_ready = true;
      }
      uint32_t lgb[32];                              // logits (float bits), log2 units
      tc::tmem_ld32(tS + lane_addr + 32 * hf, lgb);
      tc::tmem_ld_wait(lgb);
      const bool valid = s_rows[r] != nullptr;
      float v[32];
#pragma unroll
      for (int h = 0; h < 32; ++h) {
        const float l = valid ? __uint_as_float(lgb[h]) * p.scale_log2 : -INFINITY;
        lgb[h] = __float_as_uint(l);
        v[h] = l;
      }
      // After the first tile, the common case: no logit exceeds the running maximum by more
      // than the rescale threshold, so the running maximum stays this tile's reference
      // (p <= 2^8) and no maximum pass or rescale is needed; otherwise the exact pass.
      bool exact = j == jb;
      if (!exact) {
        bool big = false;
#pragma unroll
        for (int h = 0; h < 32; ++h) big |= __uint_as_float(lgb[h]) > s_M[32 * hf + h] + kRescaleThresh;
        exact = tc::bar_red_or(3, kST, big);
      }
      if (exact) {
      xpose_reduce32<true>(v, lane);
      if (tid == 0) s_flag[0] = 0;   // every read of the previous tile's flag is behind two barriers
      s_red[qd * kH + 32 * hf + lane] = v[0];
      tc::named_bar(3, kST);
      if (tid < kH) {
        const float tm = fmaxf(fmaxf(s_red[tid], s_red[kH + tid]), fmaxf(s_red[2 * kH + tid], s_red[3 * kH + tid]));
        const float Mr = s_M[tid];
        float Mu = Mr, al = 1.f;
        int resc = 0;
        if (j == jb) { Mu = tm; al = 0.f; }
        else if (tm > Mr + kRescaleThresh) { Mu = tm; al = exp2f(Mr - tm); resc = 1; }
        s_Mu[tid] = Mu == -INFINITY ? 0.f : Mu;   // an all-masked tile gives p = 0, not NaN
        s_alpha[tid] = al;
        s_M[tid] = Mu;
        if (resc) atomicOr(&s_flag[0], 1);
      }
      tc::named_bar(3, kST);
      }
      if (exact && s_flag[0] && j > jb) {
        // rescale the O^T accumulator: column h of this thread's two blocks times alpha[h]
        for (int mb = 2 * hf; mb < 2 * hf + 2; ++mb) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t o[32];
            const uint32_t ta = tO + mb * kH + half * 32 + lane_addr;
            tc::tmem_ld32(ta, o);
            tc::tmem_ld_wait(o);
#pragma unroll
            for (int h = 0; h < 32; ++h)
              o[h] = __float_as_uint(__uint_as_float(o[h]) * s_alpha[half * 32 + h]);
            tc::tmem_st32(ta, o);
          }
        }
        tc::tmem_st_wait();
      }
      // probabilities: bf16 into P^T (row r = one swizzled 128-byte line, this thread's
      // four 16-byte chunks), then their sums
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        const int cblk = 4 * hf + cb;
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h0 = cb * 8 + 2 * e;              // within this thread's 32 heads
          const float p0 = exp2f(__uint_as_float(lgb[h0]) - s_Mu[32 * hf + h0]);
          const float p1 = exp2f(__uint_as_float(lgb[h0 + 1]) - s_Mu[32 * hf + h0 + 1]);
          const __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
          w4[e] = *reinterpret_cast<const uint32_t*>(&pr);
          v[h0] = __low2float(pr);
          v[h0 + 1] = __high2float(pr);
        }
        *reinterpret_cast<uint4*>(sP + r * 128 + ((cblk ^ (r & 7)) << 4)) =
            make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      xpose_reduce32<false>(v, lane);
      tc::named_bar(3, kST);                         // everyone has read s_red (max pass)
      s_red[qd * kH + 32 * hf + lane] = v[0];
      tc::named_bar(3, kST);
      if (tid < kH) {
        const float ts = s_red[tid] + s_red[kH + tid] + s_red[2 * kH + tid] + s_red[3 * kH + tid];
        s_l[tid] = (j == jb ? 0.f : exact ? s_l[tid] * s_alpha[tid] : s_l[tid]) + ts;
      }
      tc::fence_proxy_async();
      tc::tc_fence_before();
      tc::named_bar(2, kThreadsA);
      if (j + 1 < je) {
        // the next tile, column-block pair by pair as this tile's PV frees the pairs; the
        // MMA warp starts its S^T on each pair as soon as it has landed.  Every read of
        // this tile's row table is behind the barrier above.
        if (hf == 0) {
          const int pos = rb + (j + 1) * kRows + r;
          s_rows[r] = pos < re ? row_src(p, Q, qrow, pos, e_nxt) : nullptr;
        }
        tc::named_bar(3, kST);
        for (int mb = 0; mb < 4; ++mb) {
          ok = ok && tc::mbar_wait_hint(bar_pv + mb, npv & 1, p.err, kWaitHintNs);
          tc::tc_fence_after();
          gather_pair(sKV, mb, warp, lane, s_rows, p.kv);
          tc::cp_async_commit();
        }
        ++npv;
        tc::cp_async_wait_group<3>();
        pair_landed(4);
        tc::cp_async_wait_group<2>();
        pair_landed(5);
        tc::cp_async_wait_group<1>();
        pair_landed(6);
        tc::cp_async_wait_group<0>();
        pair_landed(7);
      }
    }

    if (p.nsplit > 1 && p.cluster) {
      // this split's running maxima and sums (final after its last softmax; an empty
      // split keeps -inf and 0) to every rank while its PV still runs; with every rank's,
      // each rank forms the same log-sum-exp denominators and its own weights
      if (tid < kH) {
        const float Mv = s_M[tid], lv = s_l[tid];
        for (int j = 0; j < p.nsplit; ++j)
          st_async8(cl_map(s_stats + (crank * kH + tid) * 2, (uint32_t)j), __float_as_uint(Mv),
                    __float_as_uint(lv), cl_map(bar_st, (uint32_t)j));
        const bool got = tc::mbar_wait_hint(bar_st, 0, p.err, kWaitHintNs);
        const float sink2 = s_sink2[tid];
        float M = sink2;
        for (int j = 0; j < p.nsplit; ++j) M = fmaxf(M, s_stats[(j * kH + tid) * 2]);
        float den = exp2f(sink2 - M);
        for (int j = 0; j < p.nsplit; ++j) {
          const float mj = s_stats[(j * kH + tid) * 2];
          den = fmaf(s_stats[(j * kH + tid) * 2 + 1], mj == -INFINITY ? 0.f : exp2f(mj - M), den);
        }
        const float wme = Mv == -INFINITY ? 0.f : exp2f(Mv - M) / den;
        s_alpha[tid] = (ok && got) ? wme : __int_as_float(0x7fc00000);
        if (crank == 0 && p.lse) p.lse[(size_t)qrow * kH + tid] = (M + log2f(den)) * 0.6931471805599453f;
      }
    }

    if (je <= jb) {
      // empty split: nothing to add.  Cluster mode: its running max stays -inf (weight 0)
      // and its O is zeroed so that the merge adds 0.
      if (p.nsplit > 1 && !p.cluster && tid < kH) {
        p.part_m[(size_t)item * kH + tid] = -INFINITY;
        p.part_l[(size_t)item * kH + tid] = 0.f;
      }
      if (p.nsplit > 1 && p.cluster) {
        uint4* z = reinterpret_cast<uint4*>(sKV);
        for (int x = tid; x < kD * kH * 2 / 16; x += kST) z[x] = make_uint4(0u, 0u, 0u, 0u);
        tc::fence_proxy_async();
      }
    } else if (p.nsplit > 1 && p.cluster) {
      // O scaled by this split's weight into shared memory (bf16 record rows, dims 128 mb ..
      // at bytes 16 KB mb: the KV column block that PV block mb / 2 has already read).  Each
      // half of the warps stages its two dim blocks as soon as the PV of the block is done,
      // and one thread of the half bulk-stores the block to the workspace, so the staging and
      // the stores run under the remaining PV.
      tc::named_bar(3, kST);                         // weights (s_alpha) final
      for (int mb = 2 * hf; mb < 2 * hf + 2; ++mb) {
        ok = ok && tc::mbar_wait_hint(bar_pv + mb, npv & 1, p.err, kWaitHintNs);
        tc::tc_fence_after();
        const int d = mb * 128 + r;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t o[32];
          tc::tmem_ld32(tO + mb * kH + half * 32 + lane_addr, o);
          tc::tmem_ld_wait(o);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {    // 8 heads = one 16-byte chunk
            const float4 wa = *reinterpret_cast<const float4*>(s_alpha + half * 32 + c4 * 8);
            const float4 wb = *reinterpret_cast<const float4*>(s_alpha + half * 32 + c4 * 8 + 4);
            const float wt[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(
                  __uint_as_float(o[8 * c4 + 2 * e]) * wt[2 * e],
                  __uint_as_float(o[8 * c4 + 2 * e + 1]) * wt[2 * e + 1]);
              w4[e] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            *reinterpret_cast<uint4*>(sKV + (size_t)d * kH * 2 + cm_chunk(d, half * 4 + c4) * 16) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
        tc::fence_proxy_async();   // the bulk copy reads these rows through the async proxy
        tc::named_bar(4 + hf, kST / 2);
        if (qd == 0 && lane == 0) {
          const size_t off = (size_t)mb * 128 * kH * 2;
          bulk_store(p.part_bf + (size_t)item * kPartB + off, sKV + off, 128 * kH * 2);
          bulk_commit();
        }
      }
      ++npv;
    } else if (p.nsplit > 1) {
      // fp32 partials for the workspace merge, each 128-dim block as soon as its PV is done;
      // this thread's heads' running max and sum are its own (tid < kH) writes
      for (int mb = 2 * hf; mb < 2 * hf + 2; ++mb) {
        ok = ok && tc::mbar_wait_hint(bar_pv + mb, npv & 1, p.err, kWaitHintNs);
        tc::tc_fence_after();
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t o[32];
          tc::tmem_ld32(tO + mb * kH + half * 32 + lane_addr, o);
          tc::tmem_ld_wait(o);
          const int d = mb * 128 + r;
          float4* dst = reinterpret_cast<float4*>(&p.part_o[((size_t)item * kD + d) * kH + half * 32]);
#pragma unroll
          for (int h4 = 0; h4 < 8; ++h4) {
            float4 v = make_float4(__uint_as_float(o[4 * h4]), __uint_as_float(o[4 * h4 + 1]),
                                   __uint_as_float(o[4 * h4 + 2]), __uint_as_float(o[4 * h4 + 3]));
            if (!ok) v = make_float4(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000),
                                     __int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
            dst[h4] = v;
          }
        }
      }
      ++npv;
      if (tid < kH) {
        p.part_m[(size_t)item * kH + tid] = s_M[tid];
        p.part_l[(size_t)item * kH + tid] = s_l[tid];
      }
    } else {
      // one split: the normalised output, the sink in the denominator.  Every warp takes
      // the four 128-dim blocks of O one after another, each as soon as its PV is done
      // (the later blocks' PV still runs): thread = dim d = 128 mb + r, heads of its half hf.
      // Every read of s_alpha / s_l / s_M by the last softmax is behind its closing barrier.
      if (tid < kH) {   // one reciprocal denominator per head, where the rescale factors were
        const float den = s_l[tid] + exp2f(s_sink2[tid] - s_M[tid]);
        s_alpha[tid] = 1.f / den;
        if (p.lse) p.lse[(size_t)qrow * kH + tid] = (s_M[tid] + log2f(den)) * 0.6931471805599453f;
      }
      tc::named_bar(3, kST);
      float inv[32];                                 // this half's 32 head denominators
#pragma unroll
      for (int h = 0; h < 32; h += 4) {
        const float4 w4 = *reinterpret_cast<const float4*>(s_alpha + 32 * hf + h);
        inv[h] = w4.x; inv[h + 1] = w4.y; inv[h + 2] = w4.z; inv[h + 3] = w4.w;
      }
      for (int mb = 0; mb < 4; ++mb) {
        ok = ok && tc::mbar_wait_hint(bar_pv + mb, npv & 1, p.err, kWaitHintNs);
        tc::tc_fence_after();
        uint32_t o[32];
        tc::tmem_ld32(tO + mb * kH + 32 * hf + lane_addr, o);
        tc::tmem_ld_wait(o);
        const int d = mb * 128 + r;
        // rotary output dims: the pair partner (dim d ^ 1) is in lane ^ 1; the condition
        // is uniform over the warp's 32 dims when d_rope_out is a multiple of 32
        const bool rot = p.d_rope_out > 0 && mb * 128 + qd * 32 + 31 >= kD - p.d_rope_out;
        float sn, cs;
        out_rope_sincos(p, d, Q.t, sn, cs);
#pragma unroll
        for (int h = 0; h < 32; ++h) {
          float val = __uint_as_float(o[h]) * inv[h];
          if (rot) val = inv_rope_elem(val, __shfl_xor_sync(0xffffffffu, val, 1), d, kD,
                                       p.d_rope_out, sn, cs);
          p.out[((size_t)qrow * kH + 32 * hf + h) * kD + d] =
              __float2bfloat16_rn(ok ? val : __int_as_float(0x7fc00000));
        }
      }
      ++npv;
    }
    tc::tc_fence_before();
    tc::named_bar(3, kST);                           // s_M / s_l reads done before the next item
    }   // softmax warps

    if (p.nsplit > 1 && p.cluster) {
      // every split of this query has its O, max and sum in shared memory: merge one
      // slice of the dims, then keep this CTA's shared memory alive until all peers
      // have read it
      __syncthreads();
      cluster_merge(p, qrow, item, crank, sKV, bar_r, ok, je > jb);
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// alignment slack, KV tile, q, P^T, s_red + four per-head arrays, flag, seven mbarriers,
// TMEM holder, row-pointer table, 16-byte alignment, merge maxima / sums, sink logits
constexpr size_t kSmemBytes = 1024 + 8 * kKVBlkBytes + 8 * kQBlkBytes + kRows * 128 +
                              (4 * kH + 4 * kH) * 4 + 16 + 7 * 8 + 8 + kRows * 8 + 16 +
                              kMaxSplit * kH * 2 * 4 + kH * 4;
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");

struct Plan {
  int nsplit, rps;   // splits per query and rows per split
  int cluster;       // merge inside a cluster (else through the workspace)
};

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

// How many clusters of `cs` attention CTAs the device can hold at once (cached per device).
int max_active_clusters(int cs) {
  static int cache[64][kMaxSplit + 1] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || cs < 1 || cs > kMaxSplit) return 0;
  if (cache[dev][cs]) return cache[dev][cs] - 1;
  int n = 0;
  if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes) == cudaSuccess &&
      (cs <= 8 || cudaFuncSetAttribute(attn_tc_kernel,
                                       cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                      cudaSuccess)) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cs);
    cfg.blockDim = dim3(kThreadsA);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = cs;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, attn_tc_kernel, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();   // a refused query leaves no error behind
  cache[dev][cs] = n + 1;
  return n;
}

// Decode (one query per sequence) splits each query's rows over several CTAs, at
// most one CTA per SM over the whole grid and at least 16 rows per split.
//  - selected entries (CSA): the splits of a query form one cluster, as large as lets
//    all b clusters be resident at once (at most kMaxSplit); merged in the cluster;
//  - dense (HCA, thousands of rows per query): up to kMaxSplitGlobal splits, merged
//    through the workspace by attn_merge_kernel.
// Prefill: one split per query.
Plan plan(int k, int n_w, int b, int T, int E_cap, bool dense, int sms) {
  const long long rows_max = (long long)(dense ? E_cap : k) + n_w;
  Plan P{1, (int)std::min<long long>(rows_max, INT_MAX), 0};
  if (T == 1 && b > 0) {
    const int cap = dense ? kMaxSplitGlobal : kMaxSplit;
    int ns = std::max(1, std::min(cap, sms / b));
    ns = (int)std::min<long long>(ns, std::max<long long>(1, rows_max / 16));
    if (!dense)
      while (ns > 1 && max_active_clusters(ns) < b) --ns;
    long long rps = (rows_max + ns - 1) / ns;
    rps = (rps + 15) / 16 * 16;
    P.rps = (int)rps;
    P.nsplit = (int)((rows_max + rps - 1) / rps);
    P.cluster = !dense && P.nsplit > 1;
  }
  return P;
}

// Shared memory of attn_merge_kernel for ns splits (several CTAs fit on an SM).
size_t merge_smem_bytes(int ns) {
  return (size_t)3 * ns * kH * 4 + (size_t)ns * kMergeDims * kH * 4;
}

}  // namespace

bool attn_tc_supported(int H, int d, int dtype) {
  return H == kH && d == kD && dtype == CSA_BF16;
}

int attn_launch_count(int H, int d, int k, int n_w, int b, int T, int E_cap, int dtype) {
  if (!attn_tc_supported(H, d, dtype)) return 1;
  const Plan P = plan(k, n_w, b, T, E_cap, k <= 0, sm_count());
  return P.nsplit > 1 && !P.cluster ? 2 : 1;
}

size_t attn_tc_workspace_bytes(int H, int d, int k, int n_w, int b, int T, int E_cap, int dtype) {
  if (!attn_tc_supported(H, d, dtype) || b <= 0 || T <= 0) return 0;
  const Plan P = plan(k, n_w, b, T, E_cap, k <= 0, sm_count());
  if (P.nsplit <= 1) return 0;
  const size_t items = (size_t)b * T * P.nsplit;
  if (P.cluster) return items * kPartB + 256;
  return items * kH * kD * 4 + 2 * items * kH * 4 + 256;
}

csa_status launch_attn_tc(const AttnArgs& a, int b, int dtype, void* ws, size_t ws_bytes,
                          cudaStream_t st) {
  if (!attn_tc_supported(a.H, a.d, dtype)) return CSA_ERR_UNSUPPORTED;
  if (a.d_rope_out > 2 * kMaxOutRopePairs) return CSA_ERR_UNSUPPORTED;
  const bool dense = a.idx == nullptr;
  const int sms = sm_count();
  const Plan P = plan(dense ? 0 : a.k, a.n_w, b, a.T, a.E_cap, dense, sms);
  AttnTc p{};
  p.q = reinterpret_cast<const __nv_bfloat16*>(a.q);
  p.kv = reinterpret_cast<const __nv_bfloat16*>(a.kv ? a.kv : a.win);
  p.idx = a.idx; p.count = a.count;
  p.win = reinterpret_cast<const __nv_bfloat16*>(a.win);
  p.q_pos = a.q_pos; p.sink = a.sink;
  p.out = reinterpret_cast<__nv_bfloat16*>(a.out); p.lse = a.lse;
  p.err = device_error_word();
  if (!p.err) return CSA_ERR_CUDA;
  p.T = a.T; p.n_w = a.n_w; p.m = a.m; p.k = a.k; p.E_cap = a.kv ? a.E_cap : 0; p.n = a.n;
  p.rows_total = b * a.T; p.nsplit = P.nsplit; p.rps = P.rps; p.dense = dense ? 1 : 0;
  p.cluster = P.cluster;
  p.scale_log2 = a.scale * kLog2e;
  p.d_rope_out = a.d_rope_out;
  p.block_table = a.block_table; p.max_pages = a.max_pages; p.num_pages = a.num_pages;
  p.win_ring = a.win_ring;
  for (int j = 0; j < kMaxOutRopePairs; ++j)
    p.inv_freq[j] = 2 * j < a.d_rope_out ? std::pow(a.theta, -2.0 * j / (double)a.d_rope_out) : 0.0;
  if (P.nsplit > 1 && P.cluster) {
    const size_t items = (size_t)b * a.T * P.nsplit;
    if (!ws || ws_bytes < items * kPartB || (reinterpret_cast<uintptr_t>(ws) & 15))
      return CSA_ERR_INVALID_ARG;
    p.part_bf = static_cast<uint8_t*>(ws);
  }
  if (P.nsplit > 1 && !P.cluster) {
    const size_t items = (size_t)b * a.T * P.nsplit;
    const size_t need = items * kH * kD * 4 + 2 * items * kH * 4;
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 15)) return CSA_ERR_INVALID_ARG;
    if (P.nsplit > kMaxSplitGlobal) return CSA_ERR_UNSUPPORTED;
    p.part_o = reinterpret_cast<float*>(ws);
    p.part_m = p.part_o + items * kH * kD;
    p.part_l = p.part_m + items * kH;
  }
  if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes) != cudaSuccess)
    return CSA_ERR_CUDA;
  const long long items = (long long)b * a.T * P.nsplit;
  if (!P.cluster) {
    const int grid = (int)std::min<long long>(items, sms);
    if (csa_launch(attn_tc_kernel, dim3(grid), dim3(kThreadsA), kSmemBytes, st, a.pdl != 0, p) !=
        cudaSuccess)
      return CSA_ERR_CUDA;
    if (P.nsplit > 1) {
      const size_t msm = merge_smem_bytes(P.nsplit);
      if (cudaFuncSetAttribute(attn_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)msm) != cudaSuccess)
        return CSA_ERR_CUDA;
      if (csa_launch(attn_merge_kernel, dim3(b * a.T, kD / kMergeDims), dim3(kMergeThreads), msm, st,
                     a.pdl != 0, p) != cudaSuccess)
        return CSA_ERR_CUDA;
    }
    return CSA_OK;
  }
  // one CTA per (query, split); the splits of a query form one cluster
  if (items > 0x7fffffff) return CSA_ERR_UNSUPPORTED;
  if (P.nsplit > 8 &&
      cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
          cudaSuccess)
    return CSA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)items);
  cfg.blockDim = dim3(kThreadsA);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)P.nsplit;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = a.pdl ? 2 : 1;
  if (cudaLaunchKernelEx(&cfg, attn_tc_kernel, p) != cudaSuccess) return CSA_ERR_CUDA;
  return CSA_OK;
}

}  // namespace csa

// ---------------------------------------------------------------------------
// Allocation-free variant: the split partials live in a fixed device array of
// this file instead of a caller workspace (see csa_sparse_attn_noalloc in csa.h).
// ---------------------------------------------------------------------------
namespace csa {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[CSA_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array in the current device's context.  In host code the
// array's name is only a host-side stand-in, so the address comes from the runtime, on
// every call: a context recreated after a device reset places the array anew.
csa_status noalloc_scratch(void** out) {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return CSA_ERR_CUDA;
  *out = ptr;
  return CSA_OK;
}

}  // namespace
}  // namespace csa

extern "C" csa_status csa_sparse_attn_noalloc(const csa_attn_params* p, const void* q,
                                              const void* kv_comp, int E_cap, const int32_t* idx,
                                              const int32_t* count, const void* kv_win, int n,
                                              const int32_t* q_pos, const float* sink, int b, int T,
                                              void* out, float* lse, cudaStream_t stream) {
  if (!p) return CSA_ERR_INVALID_ARG;
  if (csa_sparse_attn_workspace_size(p, b, T, E_cap) > CSA_NOALLOC_SCRATCH_BYTES)
    return CSA_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const csa_status st = csa::noalloc_scratch(&scratch);
  if (st != CSA_OK) return st;
  return csa_sparse_attn(p, q, kv_comp, E_cap, idx, count, kv_win, n, q_pos, sink, b, T, out, lse,
                         scratch, CSA_NOALLOC_SCRATCH_BYTES, stream);
}
