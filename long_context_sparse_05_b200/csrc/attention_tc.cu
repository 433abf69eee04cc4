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
// for 64 heads) plus a 4-warp combine in shared memory.  P^T is written to
// shared memory MN-major (row r's 64 heads are one swizzled 128-byte line).
// The running max is updated lazily (only when a tile's max exceeds it by 2^8),
// which rescales the O^T accumulator in TMEM.
//
// Work item = (query, split of its tiles).  With one split the CTA writes the
// normalised output (the sink joins the denominator); with several, it writes
// an unnormalised fp32 partial (O, running max, running sum) and
// attn_merge_kernel combines the splits with the sink (log-sum-exp merge).
//
// CTA: warps 0-3 gather, read TMEM and run the softmax (warp w owns TMEM lanes
// 32w..32w+31); warp 4 lane 0 issues every MMA.  Ordering uses two named
// barriers (tile ready, P ready) and two mbarriers signalled by tcgen05.commit
// (S ready, O ready).
#include "kernels.h"
#include "tc_common.cuh"

#include <climits>
#include <mutex>

namespace csa {

namespace {

constexpr int kH = 64;            // heads
constexpr int kD = 512;           // head dim = latent dim
constexpr int kRows = 128;        // rows per tile (MMA M of S^T)
constexpr int kKVBlkBytes = kRows * 128;   // one column block of the KV tile: 16 KB
constexpr int kQBlkBytes = kH * 128;       // one column block of q: 8 KB
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThresh = 8.0f;     // log2 units

struct AttnTc {
  const __nv_bfloat16* q; const __nv_bfloat16* kv; const int32_t* idx; const int32_t* count;
  const __nv_bfloat16* win; const int32_t* q_pos; const float* sink;
  __nv_bfloat16* out; float* lse;
  float* part_o; float* part_m; float* part_l;
  int* err;
  int T, n_w, m, k, E_cap, n, rows_total, nsplit, tps, dense;
  float scale_log2;
};

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
                                                        int pos) {
  if (pos >= Q.nrows) return nullptr;
  if (pos < Q.nsel) {
    const int e = p.dense ? pos : p.idx[(size_t)qrow * p.k + pos];
    if (e < 0 || e >= p.E_cap) return nullptr;
    return p.kv + ((size_t)Q.sb * p.E_cap + e) * kD;
  }
  const int u = Q.w0 + (pos - Q.nsel);
  return p.win + ((size_t)Q.sb * p.n + u) * kD;
}

// Copy `nrows_blk` rows of 512 bf16 into the swizzled column-block layout.
// Warp w of the 4 gather warps copies rows w, w+4, ...; two 16-byte chunks per lane per row.
template <typename SrcFn>
__device__ __forceinline__ void gather_rows(uint8_t* dst, int blk_bytes, int nrows_blk, int gw,
                                            int lane, SrcFn src_of, const void* dummy) {
  for (int r = gw; r < nrows_blk; r += 4) {
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

// One halving step of the transpose-reduction: lanes with bit `OFF` set keep the
// upper half of their HALF live values, the others the lower half, and each
// combines what it keeps with what its partner sends.
template <bool kMax, int OFF, int HALF>
__device__ __forceinline__ void xpose_step(float (&v)[64], int lane) {
  const bool hi = (lane & OFF) != 0;
#pragma unroll
  for (int i = 0; i < HALF; ++i) {
    const float send = hi ? v[i] : v[i + HALF];
    const float keep = hi ? v[i + HALF] : v[i];
    const float recv = __shfl_xor_sync(0xffffffffu, send, OFF);
    v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
  }
}

// Transpose-reduction of 64 values over the 32 lanes of a warp (62 shuffles):
// afterwards lane L holds the reduction of heads 2L (v[0]) and 2L+1 (v[1]).
template <bool kMax>
__device__ __forceinline__ void xpose_reduce64(float (&v)[64], int lane) {
  xpose_step<kMax, 16, 32>(v, lane);
  xpose_step<kMax, 8, 16>(v, lane);
  xpose_step<kMax, 4, 8>(v, lane);
  xpose_step<kMax, 2, 4>(v, lane);
  xpose_step<kMax, 1, 2>(v, lane);
}

__global__ void __launch_bounds__(160, 1) attn_tc_kernel(AttnTc p) {
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
  uint64_t* bar_o = bar_s + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_o + 1);
  const __nv_bfloat16** s_rows = reinterpret_cast<const __nv_bfloat16**>(tmem_holder + 2);  // [128]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tid = threadIdx.x;

  pdl_launch_dependents();
  if (tid == 0) {
    tc::mbar_init(bar_s, 1);
    tc::mbar_init(bar_o, 1);
    tc::fence_barrier_init();
  }
  if (warp == 0) tc::tmem_alloc(tmem_holder, 512);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  pdl_wait();   // selections, positions and caches come from the preceding kernels
  const uint32_t tmem = *tmem_holder;
  const uint32_t tS = tmem;            // columns [0, 64): S^T
  const uint32_t tO = tmem + 64;       // columns [64, 320): O^T, 4 blocks of 64

  const int items = p.rows_total * p.nsplit;
  uint32_t ns = 0, no = 0;             // commits waited on bar_s / bar_o
  bool ok = true;

  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int qrow = item / p.nsplit;
    const int split = item % p.nsplit;
    const QInfo Q = query_info(p, qrow);
    const int ntiles = (Q.nrows + kRows - 1) / kRows;
    const int jb = split * p.tps;
    const int je = min(jb + p.tps, ntiles);

    if (warp == 4) {
      // ---------------------------------------------------------------- MMA issuer
      constexpr uint32_t idS = tc::instr_desc(128, kH, 1, 1, 0, 0);   // bf16 K-major x K-major
      constexpr uint32_t idO = tc::instr_desc(128, kH, 1, 1, 1, 1);   // bf16 MN-major x MN-major
      for (int j = jb; j < je; ++j) {
        tc::named_bar(1, 160);                       // tile (and q) in shared memory
        if (lane == 0) {
          tc::tc_fence_after();
          for (int kb = 0; kb < 8; ++kb) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t a = tc::smem_desc_sw128(tc::smem_u32(sKV + kb * kKVBlkBytes + kk * 32), 16, 1024);
              const uint64_t b = tc::smem_desc_sw128(tc::smem_u32(sQ + kb * kQBlkBytes + kk * 32), 16, 1024);
              tc::mma_f16(tS, a, b, idS, (kb | kk) != 0);
            }
          }
          tc::mma_commit(bar_s);
        }
        __syncwarp();
        tc::named_bar(2, 160);                       // P^T in shared memory, O rescaled
        if (lane == 0) {
          tc::tc_fence_after();
          for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t a = tc::smem_desc_sw128(
                  tc::smem_u32(sKV + 2 * mb * kKVBlkBytes + kk * 2048), kKVBlkBytes, 1024);
              const uint64_t b = tc::smem_desc_sw128(tc::smem_u32(sP + kk * 2048), 8192, 1024);
              tc::mma_f16(tO + mb * kH, a, b, idO, (j > jb) || (kk > 0));
            }
          }
          tc::mma_commit(bar_o);
        }
        __syncwarp();
      }
      continue;
    }

    // ------------------------------------------------------------------ warps 0-3
    const int r = warp * 32 + lane;                  // this thread's TMEM lane / tile row
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
    if (tid < kH) { s_M[tid] = -INFINITY; s_l[tid] = 0.f; }
    for (int j = jb; j < je; ++j) {
      if (j > jb) {                                  // previous PV done: KV, P and O are free
        ok = ok && tc::mbar_wait(bar_o, no & 1, p.err);
        ++no;
        tc::tc_fence_after();
      }
      if (j == jb) {
        const __nv_bfloat16* qb = p.q + (size_t)qrow * kH * kD;
        gather_rows(sQ, kQBlkBytes, kH, warp, lane,
                    [&](int h) { return qb + (size_t)h * kD; }, p.kv);
      }
      // source of every row of the tile: one coalesced pass over the index list
      s_rows[r] = row_src(p, Q, qrow, j * kRows + r);
      tc::named_bar(3, 128);
      gather_rows(sKV, kKVBlkBytes, kRows, warp, lane, [&](int rr) { return s_rows[rr]; }, p.kv);
      tc::cp_async_wait_all();
      tc::fence_proxy_async();
      tc::tc_fence_before();
      tc::named_bar(1, 160);

      // logits of row r for all heads
      ok = ok && tc::mbar_wait(bar_s, ns & 1, p.err);
      ++ns;
      tc::tc_fence_after();
      uint32_t ra[32], rb[32];
      tc::tmem_ld32(tS + lane_addr, ra);
      tc::tmem_ld32(tS + lane_addr + 32, rb);
      tc::tmem_ld_wait(ra);
      tc::reg_fence(rb);
      const int pos = j * kRows + r;
      const bool valid = s_rows[r] != nullptr;
      (void)pos;
      float lg[64], v[64];
#pragma unroll
      for (int h = 0; h < 32; ++h) {
        lg[h] = valid ? __uint_as_float(ra[h]) * p.scale_log2 : -INFINITY;
        lg[h + 32] = valid ? __uint_as_float(rb[h]) * p.scale_log2 : -INFINITY;
      }
#pragma unroll
      for (int h = 0; h < 64; ++h) v[h] = lg[h];
      xpose_reduce64<true>(v, lane);
      if (tid == 0) s_flag[0] = 0;   // every read of the previous tile's flag is behind two barriers
      s_red[warp * kH + 2 * lane] = v[0];
      s_red[warp * kH + 2 * lane + 1] = v[1];
      tc::named_bar(3, 128);
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
      tc::named_bar(3, 128);
      if (s_flag[0] && j > jb) {
        // rescale the O^T accumulator: column h of every block times alpha[h]
        for (int mb = 0; mb < 4; ++mb) {
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
      // probabilities: bf16 into P^T (row r = one swizzled 128-byte line), then their sums
#pragma unroll
      for (int cblk = 0; cblk < 8; ++cblk) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h0 = cblk * 8 + 2 * e;
          const float p0 = exp2f(lg[h0] - s_Mu[h0]);
          const float p1 = exp2f(lg[h0 + 1] - s_Mu[h0 + 1]);
          const __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
          w4[e] = *reinterpret_cast<const uint32_t*>(&pr);
          v[h0] = __low2float(pr);
          v[h0 + 1] = __high2float(pr);
        }
        *reinterpret_cast<uint4*>(sP + r * 128 + ((cblk ^ (r & 7)) << 4)) =
            make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      xpose_reduce64<false>(v, lane);
      tc::named_bar(3, 128);                         // everyone has read s_red (max pass)
      s_red[warp * kH + 2 * lane] = v[0];
      s_red[warp * kH + 2 * lane + 1] = v[1];
      tc::named_bar(3, 128);
      if (tid < kH) {
        const float ts = s_red[tid] + s_red[kH + tid] + s_red[2 * kH + tid] + s_red[3 * kH + tid];
        s_l[tid] = (j == jb ? 0.f : s_l[tid] * s_alpha[tid]) + ts;
      }
      tc::fence_proxy_async();
      tc::tc_fence_before();
      tc::named_bar(2, 160);
    }

    if (je <= jb) {
      // empty split: nothing to add
      if (p.nsplit > 1 && tid < kH) {
        p.part_m[(size_t)item * kH + tid] = -INFINITY;
        p.part_l[(size_t)item * kH + tid] = 0.f;
      }
      continue;
    }
    ok = ok && tc::mbar_wait(bar_o, no & 1, p.err);
    ++no;
    tc::tc_fence_after();
    tc::named_bar(3, 128);                           // s_l / s_M final
    // finalise: thread owns dims d = 128 mb + r of every head
    if (p.nsplit == 1) {
      const float* sk = p.sink;
      for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t o[32];
          tc::tmem_ld32(tO + mb * kH + half * 32 + lane_addr, o);
          tc::tmem_ld_wait(o);
          const int d = mb * 128 + r;
#pragma unroll
          for (int h = 0; h < 32; ++h) {
            const int hh = half * 32 + h;
            const float den = s_l[hh] + exp2f(sk[hh] * kLog2e - s_M[hh]);
            const float val = ok ? __uint_as_float(o[h]) / den : __int_as_float(0x7fc00000);
            p.out[((size_t)qrow * kH + hh) * kD + d] = __float2bfloat16_rn(val);
          }
        }
      }
      if (p.lse && tid < kH) {
        const float den = s_l[tid] + exp2f(sk[tid] * kLog2e - s_M[tid]);
        p.lse[(size_t)qrow * kH + tid] = (s_M[tid] + log2f(den)) * 0.6931471805599453f;
      }
    } else {
      for (int mb = 0; mb < 4; ++mb) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t o[32];
          tc::tmem_ld32(tO + mb * kH + half * 32 + lane_addr, o);
          tc::tmem_ld_wait(o);
          const int d = mb * 128 + r;
#pragma unroll
          for (int h = 0; h < 32; ++h)
            p.part_o[((size_t)item * kH + half * 32 + h) * kD + d] =
                ok ? __uint_as_float(o[h]) : __int_as_float(0x7fc00000);
        }
      }
      if (tid < kH) {
        p.part_m[(size_t)item * kH + tid] = s_M[tid];
        p.part_l[(size_t)item * kH + tid] = s_l[tid];
      }
    }    tc::tc_fence_before();
    tc::named_bar(3, 128);                           // s_M / s_l reads done before the next item
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// Combines the splits of each (query, head): out = sum_s e^{m_s} O_s / (e^{sink} + sum_s e^{m_s} l_s).
// CTA per (query, 4 heads); thread t owns dims 4t..4t+3 of the 4 heads (float4 loads).
constexpr int kMergeHeads = 4;
constexpr int kMaxSplit = 64;
__global__ void __launch_bounds__(128) attn_merge_kernel(AttnTc p) {
  __shared__ float s_m[kMaxSplit][kMergeHeads], s_l[kMaxSplit][kMergeHeads];
  __shared__ float s_w[kMaxSplit][kMergeHeads];
  pdl_launch_dependents();
  pdl_wait();
  const int qrow = blockIdx.x, h0 = blockIdx.y * kMergeHeads;
  const size_t it0 = (size_t)qrow * p.nsplit;
  for (int x = threadIdx.x; x < p.nsplit * kMergeHeads; x += blockDim.x) {
    const int s = x / kMergeHeads, hh = x % kMergeHeads;
    s_m[s][hh] = __ldcg(&p.part_m[(it0 + s) * kH + h0 + hh]);
    s_l[s][hh] = __ldcg(&p.part_l[(it0 + s) * kH + h0 + hh]);
  }
  __syncthreads();
  if (threadIdx.x < kMergeHeads) {
    const int hh = threadIdx.x;
    const float sink2 = p.sink[h0 + hh] * kLog2e;
    float M = sink2;
    for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, s_m[s][hh]);
    float den = exp2f(sink2 - M);
    for (int s = 0; s < p.nsplit; ++s) {
      const float e = s_m[s][hh] == -INFINITY ? 0.f : exp2f(s_m[s][hh] - M);
      s_w[s][hh] = e;
      den += s_l[s][hh] * e;
    }
    const float inv = 1.f / den;
    for (int s = 0; s < p.nsplit; ++s) s_w[s][hh] *= inv;
    if (p.lse) p.lse[(size_t)qrow * kH + h0 + hh] = (M + log2f(den)) * 0.6931471805599453f;
  }
  __syncthreads();
  const int d = threadIdx.x * 4;
  float4 acc[kMergeHeads];
#pragma unroll
  for (int hh = 0; hh < kMergeHeads; ++hh) acc[hh] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < p.nsplit; ++s) {
    float4 v[kMergeHeads];
#pragma unroll
    for (int hh = 0; hh < kMergeHeads; ++hh)
      v[hh] = s_w[s][hh] != 0.f
                  ? __ldcg(reinterpret_cast<const float4*>(
                        &p.part_o[((it0 + s) * kH + h0 + hh) * kD + d]))
                  : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int hh = 0; hh < kMergeHeads; ++hh) {
      const float w = s_w[s][hh];
      acc[hh].x = fmaf(v[hh].x, w, acc[hh].x); acc[hh].y = fmaf(v[hh].y, w, acc[hh].y);
      acc[hh].z = fmaf(v[hh].z, w, acc[hh].z); acc[hh].w = fmaf(v[hh].w, w, acc[hh].w);
    }
  }
#pragma unroll
  for (int hh = 0; hh < kMergeHeads; ++hh) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc[hh].x, acc[hh].y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc[hh].z, acc[hh].w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&lo);
    u.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(&p.out[((size_t)qrow * kH + h0 + hh) * kD + d]) = u;
  }
}

constexpr size_t kSmemBytes = 1024 + 8 * kKVBlkBytes + 8 * kQBlkBytes + kRows * 128 +
                              (4 * kH + 4 * kH) * 4 + 16 + 16 + 16 + kRows * 8;

struct Plan {
  int nsplit, tps;
};

Plan plan(int H, int d, int k, int n_w, int b, int T, int E_cap, bool dense, int sms) {
  Plan P{1, 1};
  const long long rows_max = (long long)(dense ? E_cap : k) + n_w;
  const int tmax = (int)((rows_max + kRows - 1) / kRows);
  P.tps = tmax;
  if (T == 1) {
    // decode: split each query's tiles so the grid covers the SMs about twice
    long long want = (2LL * sms + b - 1) / b;
    int ns = (int)std::min<long long>(std::max<long long>(1, want), tmax);
    P.tps = (tmax + ns - 1) / ns;
    P.nsplit = (tmax + P.tps - 1) / P.tps;
  }
  (void)H; (void)d;
  return P;
}

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

}  // namespace

bool attn_tc_supported(int H, int d, int dtype) {
  return H == kH && d == kD && dtype == CSA_BF16;
}

int attn_launch_count(int H, int d, int k, int n_w, int b, int T, int E_cap, int dtype) {
  if (!attn_tc_supported(H, d, dtype)) return 1;
  const Plan P = plan(H, d, k, n_w, b, T, E_cap, k <= 0, sm_count());
  return P.nsplit > 1 ? 2 : 1;
}

size_t attn_tc_workspace_bytes(int H, int d, int k, int n_w, int b, int T, int E_cap, int dtype) {
  if (!attn_tc_supported(H, d, dtype) || b <= 0 || T <= 0) return 0;
  const Plan P = plan(H, d, k, n_w, b, T, E_cap, k <= 0, sm_count());
  if (P.nsplit <= 1) return 0;
  const size_t items = (size_t)b * T * P.nsplit;
  return items * kH * kD * 4 + 2 * items * kH * 4 + 256;
}

csa_status launch_attn_tc(const AttnArgs& a, int b, int dtype, void* ws, size_t ws_bytes,
                          cudaStream_t st) {
  if (!attn_tc_supported(a.H, a.d, dtype)) return CSA_ERR_UNSUPPORTED;
  const bool dense = a.idx == nullptr;
  const int sms = sm_count();
  const Plan P = plan(a.H, a.d, dense ? 0 : a.k, a.n_w, b, a.T, a.E_cap, dense, sms);
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
  p.rows_total = b * a.T; p.nsplit = P.nsplit; p.tps = P.tps; p.dense = dense ? 1 : 0;
  p.scale_log2 = a.scale * kLog2e;
  if (P.nsplit > 1) {
    const size_t items = (size_t)b * a.T * P.nsplit;
    const size_t need = items * kH * kD * 4 + 2 * items * kH * 4;
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 15)) return CSA_ERR_INVALID_ARG;
    if (P.nsplit > kMaxSplit) return CSA_ERR_UNSUPPORTED;
    p.part_o = reinterpret_cast<float*>(ws);
    p.part_m = p.part_o + items * kH * kD;
    p.part_l = p.part_m + items * kH;
  }
  if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kSmemBytes) != cudaSuccess)
    return CSA_ERR_CUDA;
  const long long items = (long long)b * a.T * P.nsplit;
  const int grid = (int)std::min<long long>(items, sms);
  if (csa_launch(attn_tc_kernel, dim3(grid), dim3(160), kSmemBytes, st, a.pdl != 0, p) !=
      cudaSuccess)
    return CSA_ERR_CUDA;
  if (P.nsplit > 1 &&
      csa_launch(attn_merge_kernel, dim3(b * a.T, kH / kMergeHeads), dim3(128), 0, st, a.pdl != 0,
                 p) != cudaSuccess)
    return CSA_ERR_CUDA;
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

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address must come from the
// runtime; it is looked up once per device.
csa_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return CSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return CSA_ERR_CUDA;
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
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
