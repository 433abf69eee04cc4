// KV compressor (pool -> RMSNorm -> partial RoPE -> store / quantise) and the
// stand-alone index-path quantiser.
//
// Method: "DeepSeek V4 结构速览", section "C4A Compressor"; section "核心设计"
// item 1 (c4a 8 rows at stride 4, c128a 128 rows at stride 128);
// "DeepSeek-V4技术报告解读", section "Compressed Sparse Attention (CSA)".
//
// Layout of the work: one CTA per (entry, sequence).  Threads are split into
// `cols` column threads (16 bytes of channels each) x `rg` row groups; each
// row group streams every rg-th row of the 2m (or m) stacked rows with an
// online per-channel softmax in float32, then the row groups are merged
// through shared memory.  Every raw row is read exactly once per entry; the
// overlap of c4a reads C_b/Z_b for the previous block and C_a/Z_a for the
// current one, which are different tensors, so no row is read twice overall.
// The HCA decode step's one entry per sequence (128 rows) is too little work for
// one CTA to finish quickly: compress_split_kernel spreads it over an 8-CTA cluster.
#include "common.cuh"
#include "kernels.h"

#include <algorithm>
#include <cmath>

namespace csa {

template <typename InT>
struct Vec16;  // 16 bytes of InT
template <> struct Vec16<float> { static constexpr int N = 4; };
template <> struct Vec16<__nv_bfloat16> { static constexpr int N = 8; };

template <typename InT>
__device__ __forceinline__ void load16(const InT* p, float* dst) {
  uint4 v = __ldcg(reinterpret_cast<const uint4*>(p));   // L2: rings are rewritten every step
  if constexpr (sizeof(InT) == 4) {
    dst[0] = __uint_as_float(v.x); dst[1] = __uint_as_float(v.y);
    dst[2] = __uint_as_float(v.z); dst[3] = __uint_as_float(v.w);
  } else {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      dst[2 * i] = __uint_as_float(w[i] << 16);
      dst[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
}

constexpr int kUnroll = 4;

// One compressed entry (entry i of sequence s) by the whole CTA; see compress_kernel.
// U rows per thread are loaded together (one memory round trip); the decode prologue,
// which runs this code once per CTA, takes U = 2 so that less code is fetched.
template <typename InT, int U = kUnroll>
__device__ __forceinline__ void compress_body(const CompressArgs& a, int i, int s, float* smem) {
  constexpr int VEC = Vec16<InT>::N;
  const int c = a.c;
  const int cols = c / VEC;
  const int rg = blockDim.x / cols;
  const int tid = threadIdx.x;
  const int cc = tid % cols;
  const int g = tid / cols;
  const int m = a.m;
  const int R = a.overlap ? 2 * m : m;

  const size_t seq_rows = a.ring ? (size_t)a.ring : (size_t)a.n;
  const InT* Ca = reinterpret_cast<const InT*>(a.C_a) + (size_t)s * seq_rows * c;
  const InT* Za = reinterpret_cast<const InT*>(a.Z_a) + (size_t)s * seq_rows * c;
  const InT* Cb = a.overlap ? reinterpret_cast<const InT*>(a.C_b) + (size_t)s * seq_rows * c : nullptr;
  const InT* Zb = a.overlap ? reinterpret_cast<const InT*>(a.Z_b) + (size_t)s * seq_rows * c : nullptr;
  // paged state: the newest token's rows come from the step's inputs, the rest from the
  // rings; an entry is compressed only by the token that completes it, m (i + 1) - 1
  const int t_new = a.ring ? m * (i + 1) - 1 : -1;
  auto rowp = [&](const InT* base, const void* fresh, int row) -> const InT* {
    if (!a.ring) return base + (size_t)row * c;
    if (row == t_new) return reinterpret_cast<const InT*>(fresh) + (size_t)s * c;
    return base + (size_t)(row % a.ring) * c;
  };

  // paged output: an entry past the sequence's block table, or whose page is not in the
  // pool, is not written (positions are device data; the kernel does not trust them)
  if (a.block_table) {
    if (i / kPageEntries >= a.max_pages) return;
    const int pg = a.block_table[(size_t)s * a.max_pages + i / kPageEntries];
    if ((unsigned)pg >= (unsigned)a.num_pages) return;
  }

  float mx[VEC], sum[VEC], acc[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) { mx[v] = -INFINITY; sum[v] = 0.f; acc[v] = 0.f; }

  if (g < rg) {
    for (int r0 = g; r0 < R; r0 += rg * U) {
      float zv[U][VEC], cv[U][VEC], bv[U][VEC];
      bool live[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int r = r0 + u * rg;
        live[u] = r < R;
        const InT *Z = nullptr, *C = nullptr;
        const float* B = nullptr;
        int row = 0;
        if (live[u]) {
          if (a.overlap && r < m) {
            if (i == 0) { live[u] = false; }
            else { row = m * (i - 1) + r; Z = Zb; C = Cb; B = a.B_b + (size_t)r * c; }
          } else {
            const int rr = a.overlap ? r - m : r;
            row = m * i + rr; Z = Za; C = Ca; B = a.B_a + (size_t)rr * c;
          }
        }
        if (live[u]) {
          const bool cur = Z == Za;
          load16<InT>(rowp(Z, cur ? a.new_Z_a : a.new_Z_b, row) + cc * VEC, zv[u]);
          load16<InT>(rowp(C, cur ? a.new_C_a : a.new_C_b, row) + cc * VEC, cv[u]);
          if ((reinterpret_cast<uintptr_t>(B) & 15) == 0) {   // rows of c floats, c % 8 == 0
#pragma unroll
            for (int v = 0; v < VEC; v += 4) {
              const float4 b4 = __ldg(reinterpret_cast<const float4*>(B + cc * VEC + v));
              bv[u][v] = b4.x; bv[u][v + 1] = b4.y; bv[u][v + 2] = b4.z; bv[u][v + 3] = b4.w;
            }
          } else {
#pragma unroll
            for (int v = 0; v < VEC; ++v) bv[u][v] = __ldg(B + cc * VEC + v);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (!live[u]) continue;
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
          const float x = zv[u][v] + bv[u][v];
          if (x > mx[v]) {
            const float sc = expf(mx[v] - x);
            sum[v] = sum[v] * sc + 1.f;
            acc[v] = acc[v] * sc + cv[u][v];
            mx[v] = x;
          } else {
            const float e = expf(x - mx[v]);
            sum[v] += e;
            acc[v] = fmaf(e, cv[u][v], acc[v]);
          }
        }
      }
    }
  }

  // merge the row groups
  float* s_mx = smem;                 // [rg][c]
  float* s_sum = s_mx + rg * c;       // [rg][c]
  float* s_acc = s_sum + rg * c;      // [rg][c]
  float* s_x = s_acc + rg * c;        // [c]
  float* s_red = s_x + c;             // [32]
  if (g < rg) {
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
      s_mx[g * c + cc * VEC + v] = mx[v];
      s_sum[g * c + cc * VEC + v] = sum[v];
      s_acc[g * c + cc * VEC + v] = acc[v];
    }
  }
  __syncthreads();
  float ss = 0.f;
  for (int ch = tid; ch < c; ch += blockDim.x) {
    float M = -INFINITY;
    for (int q = 0; q < rg; ++q) M = fmaxf(M, s_mx[q * c + ch]);
    float S = 0.f, A = 0.f;
    for (int q = 0; q < rg; ++q) {
      const float mq = s_mx[q * c + ch];
      if (mq == -INFINITY) continue;
      const float e = expf(mq - M);
      S = fmaf(s_sum[q * c + ch], e, S);
      A = fmaf(s_acc[q * c + ch], e, A);
    }
    const float x = A / S;
    s_x[ch] = x;
    ss = fmaf(x, x, ss);
  }
  float inv = 1.f;
  if (a.apply_norm) {
    const float tot = block_sum(ss, s_red);
    inv = 1.f / sqrtf(tot / (float)c + a.eps);
  }
  __syncthreads();
  // RMSNorm + RoPE (angle in float64), result back into s_x
  const int rope0 = c - a.d_rope;
  for (int pj = tid; pj < c / 2; pj += blockDim.x) {
    const int ch = 2 * pj;
    float x0 = s_x[ch] * inv, x1 = s_x[ch + 1] * inv;
    if (ch >= rope0 && a.d_rope > 0) {
      const int j = (ch - rope0) / 2;
      const double freq = j < kMaxRopePairs ? a.inv_freq[j]
                                            : pow(a.theta, -2.0 * (double)j / (double)a.d_rope);
      float sn, cs;
      rope_angle((double)((long long)m * i) * freq, &sn, &cs);
      const float y0 = x0 * cs - x1 * sn;
      const float y1 = x0 * sn + x1 * cs;
      x0 = y0; x1 = y1;
    }
    s_x[ch] = x0; s_x[ch + 1] = x1;
  }
  __syncthreads();

  // physical output row (paged: the page of entry i from the sequence's block table; a
  // shard of the entries: row i - out_off)
  const size_t orow = a.block_table
      ? (size_t)a.block_table[(size_t)s * a.max_pages + i / kPageEntries] * kPageEntries + i % kPageEntries
      : (size_t)s * a.out_E + (i - a.out_off);
  if (a.out_dtype == CSA_F32) {
    float* o = reinterpret_cast<float*>(a.out) + orow * c;
    for (int ch = tid; ch < c; ch += blockDim.x) o[ch] = s_x[ch];
  } else if (a.out_dtype == CSA_BF16) {
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.out) + orow * c;
    for (int ch = tid; ch < c; ch += blockDim.x) o[ch] = __float2bfloat16_rn(s_x[ch]);
  } else if (a.out_dtype == CSA_FP8_E4M3) {
    float am = 0.f;
    for (int ch = tid; ch < c; ch += blockDim.x) am = fmaxf(am, fabsf(s_x[ch]));
    am = block_max(am, s_red);
    const float scale = am / 448.f;
    uint8_t* o = reinterpret_cast<uint8_t*>(a.out) + orow * c;
    for (int ch = tid; ch < c; ch += blockDim.x)
      o[ch] = scale > 0.f ? f32_to_e4m3(s_x[ch] / scale) : (uint8_t)0;
    if (tid == 0) reinterpret_cast<float*>(a.out_scales)[orow] = scale;
  } else {  // CSA_NVFP4
    uint8_t* o = reinterpret_cast<uint8_t*>(a.out) + orow * (c / 2);
    // the tiled key-scale layout of the sequence, or (paged) of all pages as one array
    uint8_t* so = reinterpret_cast<uint8_t*>(a.out_scales) +
                  (a.block_table ? (size_t)0 : (size_t)s * nvfp4_key_scale_seq_bytes(a.out_E, c));
    const long long srow = a.block_table ? (long long)orow : (long long)(i - a.out_off);
    for (int blk = tid; blk < c / 16; blk += blockDim.x) {
      float am = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) am = fmaxf(am, fabsf(s_x[blk * 16 + e]));
      const uint8_t sc = f32_to_e4m3(am / 6.f);
      const float sv = e4m3_to_f32(sc);
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        o[blk * 8 + e / 2] = sv > 0.f
            ? f32x2_to_e2m1x2(s_x[blk * 16 + e] / sv, s_x[blk * 16 + e + 1] / sv)
            : (uint8_t)0;
      }
      so[nvfp4_key_scale_offset(srow, blk, c)] = sc;
    }
  }
}

// Layout of the work: one CTA per (entry, sequence); see compress_body.  U = rows a thread
// loads at once: the rows per thread of the launch, at most kUnroll (fewer registers, more
// CTAs resident per SM when each thread has only one or two rows).
template <typename InT, int U>
__global__ void __launch_bounds__(512) compress_kernel(CompressArgs a) {
  extern __shared__ float smem[];
  compress_body<InT, U>(a, a.entry_begin + blockIdx.x, blockIdx.y, smem);
}

// One row of the index-path quantiser by one warp: FP8 (per-row scale) or NVFP4 (per-16 scale).
template <typename InT>
__device__ __forceinline__ void quantize_row(const InT* __restrict__ x, int row, int d, int out_dtype,
                                             uint8_t* __restrict__ codes, void* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const InT* xr = x + (size_t)row * d;
  float am_row = 0.f;
  for (int base = 0; base < d; base += 128) {
    const int e0 = base + lane * 4;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (e0 + e < d) am_row = fmaxf(am_row, fabsf(to_f32(xr[e0 + e])));
  }
  if (out_dtype == CSA_FP8_E4M3) {
    am_row = warp_max(am_row);
    const float scale = am_row / 448.f;
    for (int base = 0; base < d; base += 128) {
      const int e0 = base + lane * 4;
      if (e0 < d) {
        uint32_t packed = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t cde = scale > 0.f ? f32_to_e4m3(to_f32(xr[e0 + e]) / scale) : 0u;
          packed |= cde << (8 * e);
        }
        *reinterpret_cast<uint32_t*>(codes + (size_t)row * d + e0) = packed;
      }
    }
    if (lane == 0) reinterpret_cast<float*>(scales)[row] = scale;
  } else {
    // NVFP4: 4 lanes x 4 elements = one 16-element block
    for (int base = 0; base < d; base += 128) {
      const int e0 = base + lane * 4;
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      float am = 0.f;
      if (e0 < d) {
#pragma unroll
        for (int e = 0; e < 4; ++e) { v[e] = to_f32(xr[e0 + e]); am = fmaxf(am, fabsf(v[e])); }
      }
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
      const uint8_t sc = f32_to_e4m3(am / 6.f);
      const float sv = e4m3_to_f32(sc);
      if (e0 < d) {
        uint8_t p0 = sv > 0.f ? f32x2_to_e2m1x2(v[0] / sv, v[1] / sv) : (uint8_t)0;
        uint8_t p1 = sv > 0.f ? f32x2_to_e2m1x2(v[2] / sv, v[3] / sv) : (uint8_t)0;
        uint8_t* cr = codes + (size_t)row * (d / 2) + e0 / 2;
        cr[0] = p0; cr[1] = p1;
        if ((lane & 3) == 0)
          reinterpret_cast<uint8_t*>(scales)[(size_t)row * (d / 16) + e0 / 16] = sc;
      }
    }
  }
}

template <typename InT>
__global__ void quantize_kernel(const InT* __restrict__ x, int rows, int d, int out_dtype,
                                uint8_t* __restrict__ codes, void* __restrict__ scales) {
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (row >= rows) return;
  quantize_row<InT>(x, row, d, out_dtype, codes, scales);
}

// The same quantisers for bf16 rows of 128 (index queries): a warp takes kQ128Rows rows,
// loads all of them first (8 bytes per lane and row, one coalesced 256-byte row per
// instruction) and keeps them in registers for the scale and the codes, so enough bytes
// are in flight to stream at HBM speed.  Element arithmetic as in quantize_row.
constexpr int kQ128Rows = 4;
__global__ void __launch_bounds__(256) quantize128_kernel(const __nv_bfloat16* __restrict__ x,
                                                          int rows, int out_dtype,
                                                          uint8_t* __restrict__ codes,
                                                          void* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int row0 = (blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5)) * kQ128Rows;
  if (row0 >= rows) return;
  uint2 raw[kQ128Rows];
#pragma unroll
  for (int i = 0; i < kQ128Rows; ++i)
    raw[i] = row0 + i < rows ? __ldg(reinterpret_cast<const uint2*>(x + (size_t)(row0 + i) * 128) + lane)
                             : make_uint2(0u, 0u);
#pragma unroll
  for (int i = 0; i < kQ128Rows; ++i) {
    const int row = row0 + i;
    if (row >= rows) break;
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&raw[i].x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&raw[i].y);
    const float v[4] = {__low2float(lo), __high2float(lo), __low2float(hi), __high2float(hi)};
    float am = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) am = fmaxf(am, fabsf(v[e]));
    if (out_dtype == CSA_FP8_E4M3) {
      am = warp_max(am);
      const float scale = am / 448.f;
      uint32_t packed = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        packed |= (scale > 0.f ? f32_to_e4m3(v[e] / scale) : 0u) << (8 * e);
      reinterpret_cast<uint32_t*>(codes + (size_t)row * 128)[lane] = packed;
      if (lane == 0) reinterpret_cast<float*>(scales)[row] = scale;
    } else {
      // NVFP4: 4 lanes x 4 elements = one 16-element block
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
      const uint8_t sc = f32_to_e4m3(am / 6.f);
      const float sv = e4m3_to_f32(sc);
      const uint8_t p0 = sv > 0.f ? f32x2_to_e2m1x2(v[0] / sv, v[1] / sv) : (uint8_t)0;
      const uint8_t p1 = sv > 0.f ? f32x2_to_e2m1x2(v[2] / sv, v[3] / sv) : (uint8_t)0;
      reinterpret_cast<uint16_t*>(codes + (size_t)row * 64)[lane] = (uint16_t)(p0 | (p1 << 8));
      if ((lane & 3) == 0) reinterpret_cast<uint8_t*>(scales)[(size_t)row * 8 + lane / 4] = sc;
    }
  }
}

// Decode prologue in one launch: CTAs [0, b) compress the latent entry of each
// sequence, [b, 2b) its index-key entry (CSA), in paged mode the next b append the new
// token's rows to the state rings, the rest quantise the index queries (16 rows per CTA);
// CTA 0 of that range also writes the query positions.
constexpr int kQRowsPerWarp = 2;   // index-query rows quantised by one warp of the prologue

template <typename InT>
__global__ void __launch_bounds__(256) decode_prologue_kernel(PrologueArgs a) {
  extern __shared__ float smem[];
  pdl_launch_dependents();   // the indexer may start fetching the unchanged key tiles
  const int blk = blockIdx.x;
  if (blk < a.b * a.nbranch) {
    if (a.skip_compress) return;   // the split kernel that follows compresses
    const int br = blk / a.b;
    const int s = blk % a.b;
    const CompressArgs& ca = br == 0 ? a.main : a.index;
    if (!a.paged) {
      compress_body<InT, 2>(ca, ca.entry_begin, s, smem);
      return;
    }
    // paged state: the entry the newest token completes, if it completes one
    const int t = a.main.pos[s];
    if (t >= 0 && (t + 1) % ca.m == 0) compress_body<InT, 2>(ca, (t + 1) / ca.m - 1, s, smem);
    return;
  }
  if (a.paged && blk < a.b * (a.nbranch + 1)) {
    // paged state: the token's raw rows into the rings, by CTAs of their own, alongside
    // the compression (no row the compression reads sits in a slot written here: the 2m
    // rows of an entry occupy distinct slots and the newest comes from the inputs)
    const int s = blk - a.b * a.nbranch;
    const int t = a.main.pos[s];
    if (t < 0) return;
    // up to nine rows (C, Z of both blocks of both branches, the window row): every
    // thread loads all its 16-byte pieces first, then stores them (one memory round trip)
    const uint4* src[9];
    uint4* dst[9];
    int n16[9], nr = 0;
    auto add = [&](void* ring, const void* fresh, int ringlen, int slot, int c) {
      src[nr] = reinterpret_cast<const uint4*>(reinterpret_cast<const InT*>(fresh) + (size_t)s * c);
      dst[nr] = reinterpret_cast<uint4*>(reinterpret_cast<InT*>(ring) + ((size_t)s * ringlen + slot) * c);
      n16[nr] = c * (int)sizeof(InT) / 16;
      ++nr;
    };
    for (int br = 0; br < a.nbranch; ++br) {
      const CompressArgs& ca = br == 0 ? a.main : a.index;
      const int slot = t % ca.ring;
      add(const_cast<void*>(ca.C_a), ca.new_C_a, ca.ring, slot, ca.c);
      add(const_cast<void*>(ca.Z_a), ca.new_Z_a, ca.ring, slot, ca.c);
      if (ca.overlap) {
        add(const_cast<void*>(ca.C_b), ca.new_C_b, ca.ring, slot, ca.c);
        add(const_cast<void*>(ca.Z_b), ca.new_Z_b, ca.ring, slot, ca.c);
      }
    }
    add(a.win, a.new_win, a.win_ring, t % a.win_ring, a.main.c);
    int total = 0;
    for (int r = 0; r < nr; ++r) total += n16[r];
    for (int x0 = threadIdx.x; x0 < total; x0 += 4 * blockDim.x) {
      uint4 v[4];
      uint4* d[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        int x = x0 + u * blockDim.x;
        d[u] = nullptr;
        if (x >= total) continue;
        int r = 0;
        while (x >= n16[r]) { x -= n16[r]; ++r; }
        v[u] = src[r][x];
        d[u] = dst[r] + x;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (d[u]) *d[u] = v[u];
    }
    return;
  }
  const int qb = blk - a.b * (a.nbranch + (a.paged ? 1 : 0));
  if (qb == 0)
    for (int i = threadIdx.x; i < a.b; i += blockDim.x) a.qpos[i] = a.paged ? a.main.pos[i] : a.t;
  // kQRowsPerWarp rows per warp, so that the whole prologue fits in one wave of CTAs
  for (int j = 0; j < kQRowsPerWarp; ++j) {
    const int row = (qb * (blockDim.x / 32) + (threadIdx.x >> 5)) * kQRowsPerWarp + j;
    if (row < a.q_rows)
      quantize_row<InT>(reinterpret_cast<const InT*>(a.q_in), row, a.q_d, a.q_dtype, a.q_codes,
                        a.q_scales);
  }
}

// One entry of a long non-overlapped block (c128a: m = 128 rows) split over the CTAs of
// a cluster: rank r pools rows [r m / CS, (r + 1) m / CS) of the block into per-channel
// partial (max, sum, weighted sum), the ranks exchange them through distributed shared
// memory, and rank r finishes channels [r c / CS, (r + 1) c / CS): combine, RMSNorm (the
// sum of squares is exchanged once more), RoPE, store.  F32 / BF16 outputs only.
__device__ __forceinline__ uint32_t cs_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cs_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
__device__ __forceinline__ float cs_ld(const float* local, uint32_t rank) {
  uint32_t la = static_cast<uint32_t>(__cvta_generic_to_shared(local)), ra;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(la), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
  return v;
}

template <typename InT>
__global__ void __launch_bounds__(256) compress_split_kernel(CompressArgs a, int32_t* qpos, int nq,
                                                             int t) {
  extern __shared__ float smem[];
  constexpr int VEC = Vec16<InT>::N;
  const int c = a.c;
  const int cols = c / VEC;
  const int rg = blockDim.x / cols;
  const int tid = threadIdx.x;
  const int cc = tid % cols, g = tid / cols;
  const int m = a.m;
  const int CS = gridDim.x;
  const int rank = (int)cs_rank();
  const int s = blockIdx.y;
  const int rpr = m / CS;
  pdl_launch_dependents();
  // paged state: the entry the sequence's new token completes, if it completes one (the
  // same for every CTA of the cluster); the preceding kernel (ring appends, positions) is
  // waited for at the end, so that this kernel's completion implies its completion
  int i = a.entry_begin, t_new = -1;
  if (a.ring) {
    const int tp = a.pos[s];
    if (tp < 0 || (tp + 1) % m != 0) { pdl_wait(); return; }
    i = (tp + 1) / m - 1;
    t_new = tp;
    // an entry past the block table, or whose page is not in the pool, is not written
    bool bad = i / kPageEntries >= a.max_pages;
    if (!bad && a.block_table) {
      const int pg = a.block_table[(size_t)s * a.max_pages + i / kPageEntries];
      bad = (unsigned)pg >= (unsigned)a.num_pages;
    }
    if (bad) { pdl_wait(); return; }
  } else {
    pdl_wait();
  }
  if (qpos && blockIdx.x == 0 && blockIdx.y == 0)
    for (int x = tid; x < nq; x += blockDim.x) qpos[x] = t;   // query positions of the step
  const size_t seq_rows = a.ring ? (size_t)a.ring : (size_t)a.n;
  const InT* Ca = reinterpret_cast<const InT*>(a.C_a) + (size_t)s * seq_rows * c;
  const InT* Za = reinterpret_cast<const InT*>(a.Z_a) + (size_t)s * seq_rows * c;
  auto rowp = [&](const InT* base, const void* fresh, size_t row) -> const InT* {
    if (!a.ring) return base + row * c;
    if ((long long)row == t_new) return reinterpret_cast<const InT*>(fresh) + (size_t)s * c;
    return base + (row % a.ring) * c;
  };
  float mx[VEC], sum[VEC], acc[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) { mx[v] = -INFINITY; sum[v] = 0.f; acc[v] = 0.f; }
  if (g < rg) {
    for (int q0 = g; q0 < rpr; q0 += rg * kUnroll) {
      float zv[kUnroll][VEC], cv[kUnroll][VEC], bv[kUnroll][VEC];
      bool live[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int q = q0 + u * rg;
        live[u] = q < rpr;
        if (live[u]) {
          const int r = rank * rpr + q;             // row inside the block
          const size_t row = (size_t)m * i + r;
          load16<InT>(rowp(Za, a.new_Z_a, row) + cc * VEC, zv[u]);
          load16<InT>(rowp(Ca, a.new_C_a, row) + cc * VEC, cv[u]);
#pragma unroll
          for (int v = 0; v < VEC; ++v) bv[u][v] = __ldg(a.B_a + (size_t)r * c + cc * VEC + v);
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        if (!live[u]) continue;
#pragma unroll
        for (int v = 0; v < VEC; ++v) {
          const float x = zv[u][v] + bv[u][v];
          if (x > mx[v]) {
            const float sc = expf(mx[v] - x);
            sum[v] = sum[v] * sc + 1.f;
            acc[v] = acc[v] * sc + cv[u][v];
            mx[v] = x;
          } else {
            const float e = expf(x - mx[v]);
            sum[v] += e;
            acc[v] = fmaf(e, cv[u][v], acc[v]);
          }
        }
      }
    }
  }
  // this CTA's partial over its rows: merge the row groups
  float* s_mx = smem;                 // [rg][c], row group 0 ends up holding the CTA partial
  float* s_sum = s_mx + rg * c;
  float* s_acc = s_sum + rg * c;
  float* s_x = s_acc + rg * c;        // [c]
  float* s_red = s_x + c;             // [32]
  float* s_ss = s_red + 32;           // [1] this rank's sum of squares
  if (g < rg) {
#pragma unroll
    for (int v = 0; v < VEC; ++v) {
      s_mx[g * c + cc * VEC + v] = mx[v];
      s_sum[g * c + cc * VEC + v] = sum[v];
      s_acc[g * c + cc * VEC + v] = acc[v];
    }
  }
  __syncthreads();
  for (int ch = tid; ch < c; ch += blockDim.x) {
    float M = -INFINITY;
    for (int q = 0; q < rg; ++q) M = fmaxf(M, s_mx[q * c + ch]);
    float S = 0.f, A = 0.f;
    for (int q = 0; q < rg; ++q) {
      const float mq = s_mx[q * c + ch];
      if (mq == -INFINITY) continue;
      const float e = expf(mq - M);
      S = fmaf(s_sum[q * c + ch], e, S);
      A = fmaf(s_acc[q * c + ch], e, A);
    }
    s_sum[ch] = S;                 // row group 0 slots: the partial of this CTA
    s_acc[ch] = A;
    s_mx[ch] = M;
  }
  cs_sync();   // every rank's partial is in its shared memory
  // channels of this rank: combine the ranks' partials
  const int cpr = c / CS;
  const int ch0 = rank * cpr;
  float ss = 0.f;
  for (int k = tid; k < cpr; k += blockDim.x) {
    const int ch = ch0 + k;
    float Mr[16], Sr[16], Ar[16];
    float M = -INFINITY;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      if (r < CS) {
        Mr[r] = cs_ld(s_mx + ch, r); Sr[r] = cs_ld(s_sum + ch, r); Ar[r] = cs_ld(s_acc + ch, r);
        M = fmaxf(M, Mr[r]);
      }
    }
    float S = 0.f, A = 0.f;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      if (r < CS && Mr[r] != -INFINITY) {
        const float e = expf(Mr[r] - M);
        S = fmaf(Sr[r], e, S);
        A = fmaf(Ar[r], e, A);
      }
    }
    const float x = A / S;
    s_x[ch] = x;
    ss = fmaf(x, x, ss);
  }
  float inv = 1.f;
  if (a.apply_norm) {
    const float part = block_sum(ss, s_red);
    if (tid == 0) s_ss[0] = part;
    cs_sync();   // every rank's sum of squares is published
    float tot = 0.f;
    for (int r = 0; r < CS; ++r) tot += cs_ld(s_ss, r);
    inv = 1.f / sqrtf(tot / (float)c + a.eps);
  } else {
    __syncthreads();
  }
  // RMSNorm + RoPE on this rank's channels (pairs stay inside a rank: cpr is even)
  const int rope0 = c - a.d_rope;
  const size_t orow = a.block_table
      ? (size_t)a.block_table[(size_t)s * a.max_pages + i / kPageEntries] * kPageEntries + i % kPageEntries
      : (size_t)s * a.out_E + i;
  for (int pj = tid; pj < cpr / 2; pj += blockDim.x) {
    const int ch = ch0 + 2 * pj;
    float x0 = s_x[ch] * inv, x1 = s_x[ch + 1] * inv;
    if (ch >= rope0 && a.d_rope > 0) {
      const int j = (ch - rope0) / 2;
      const double freq = j < kMaxRopePairs ? a.inv_freq[j]
                                            : pow(a.theta, -2.0 * (double)j / (double)a.d_rope);
      float sn, cs;
      rope_angle((double)((long long)m * i) * freq, &sn, &cs);
      const float y0 = x0 * cs - x1 * sn;
      const float y1 = x0 * sn + x1 * cs;
      x0 = y0; x1 = y1;
    }
    if (a.out_dtype == CSA_F32) {
      float* o = reinterpret_cast<float*>(a.out) + orow * c;
      o[ch] = x0; o[ch + 1] = x1;
    } else {
      __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.out) + orow * c;
      *reinterpret_cast<__nv_bfloat162*>(o + ch) = __floats2bfloat162_rn(x0, x1);
    }
  }
  cs_sync();   // peers are done reading this CTA's shared memory
  if (a.ring) pdl_wait();
}

void fill_inv_freq(CompressArgs& a) {
  for (int j = 0; j < kMaxRopePairs; ++j)
    a.inv_freq[j] = (a.d_rope > 0 && 2 * j < a.d_rope)
                        ? std::pow(a.theta, -2.0 * (double)j / (double)a.d_rope) : 0.0;
}

size_t compress_smem_bytes(const CompressArgs& a, int in_dtype, int nt) {
  const int vec = in_dtype == CSA_F32 ? 4 : 8;
  const int cols = a.c / vec;
  return (size_t)(3 * (nt / cols) * a.c + a.c + 32) * sizeof(float);
}

// Split launch for one long non-overlapped block per sequence (c128a decode).
constexpr int kSplitCS = 8;
constexpr int kSplitThreads = 256;
size_t split_smem_bytes(const CompressArgs& a, int in_dtype) {
  const int cols = a.c / (in_dtype == CSA_F32 ? 4 : 8);
  return (size_t)(3 * (kSplitThreads / cols) * a.c + a.c + 32 + 4) * sizeof(float);
}
bool compress_split_supported(const CompressArgs& a, int in_dtype) {
  const int cols = a.c / (in_dtype == CSA_F32 ? 4 : 8);
  return cols <= kSplitThreads && a.m % kSplitCS == 0 && a.c % (2 * kSplitCS) == 0 && !a.overlap &&
         (a.out_dtype == CSA_F32 || a.out_dtype == CSA_BF16) && (a.c - a.d_rope) % 2 == 0 &&
         split_smem_bytes(a, in_dtype) <= 200 * 1024;
}

csa_status launch_compress_split(CompressArgs& a, int in_dtype, int b, int32_t* qpos, int t,
                                 cudaStream_t st, bool pdl) {
  constexpr int CS = kSplitCS;
  const int nt = kSplitThreads;
  if (!compress_split_supported(a, in_dtype)) return CSA_ERR_UNSUPPORTED;
  fill_inv_freq(a);
  const size_t smem = split_smem_bytes(a, in_dtype);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS, b);
  cfg.blockDim = dim3(nt);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = CS;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl ? 2 : 1;
  cudaError_t e;
  if (in_dtype == CSA_F32) {
    cudaFuncSetAttribute(compress_split_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    e = cudaLaunchKernelEx(&cfg, compress_split_kernel<float>, a, qpos, b, t);
  } else {
    cudaFuncSetAttribute(compress_split_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    e = cudaLaunchKernelEx(&cfg, compress_split_kernel<__nv_bfloat16>, a, qpos, b, t);
  }
  return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

csa_status launch_decode_prologue(PrologueArgs& a, int in_dtype, cudaStream_t st) {
  if (!a.paged && a.nbranch == 1 && a.q_rows == 0 && !a.main.overlap && a.main.m >= 64) {
    // c128a: the block's rows over a cluster (the query positions come from the caller)
    const csa_status r = launch_compress_split(a.main, in_dtype, a.b, a.qpos, a.t, st, false);
    if (r != CSA_ERR_UNSUPPORTED) return r;
  }
  const int nt = 256;
  const int vec = in_dtype == CSA_F32 ? 4 : 8;
  fill_inv_freq(a.main);
  size_t smem = compress_smem_bytes(a.main, in_dtype, nt);
  if (a.main.c / vec > nt) return CSA_ERR_UNSUPPORTED;
  if (a.nbranch > 1) {
    fill_inv_freq(a.index);
    if (a.index.c / vec > nt) return CSA_ERR_UNSUPPORTED;
    smem = std::max(smem, compress_smem_bytes(a.index, in_dtype, nt));
  }
  if (smem > 200 * 1024) return CSA_ERR_UNSUPPORTED;
  const int qrows_per_cta = 8 * kQRowsPerWarp;
  const int qblocks = std::max(1, (a.q_rows + qrows_per_cta - 1) / qrows_per_cta);
  const int grid = a.b * (a.nbranch + (a.paged ? 1 : 0)) + qblocks;
  if (in_dtype == CSA_F32) {
    cudaFuncSetAttribute(decode_prologue_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    decode_prologue_kernel<float><<<grid, nt, smem, st>>>(a);
  } else {
    cudaFuncSetAttribute(decode_prologue_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    decode_prologue_kernel<__nv_bfloat16><<<grid, nt, smem, st>>>(a);
  }
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

csa_status launch_compress(const CompressArgs& a_in, int in_dtype, int b, int entry_count,
                           cudaStream_t st) {
  CompressArgs a = a_in;
  fill_inv_freq(a);
  const int vec = in_dtype == CSA_F32 ? 4 : 8;
  const int cols = a.c / vec;
  const int R = a.overlap ? 2 * a.m : a.m;
  int nt = R >= 64 ? 512 : 256;
  if (cols > nt) return CSA_ERR_UNSUPPORTED;
  // as many whole row groups as fit, at most one row group per row
  int rg = nt / cols;
  if (rg > R) rg = R;
  nt = rg * cols;
  if (nt % 32) nt = ((nt + 31) / 32) * 32;   // idle tail threads take no rows (g >= rg)
  const size_t smem = (size_t)(3 * (nt / cols) * a.c + a.c + 32) * sizeof(float);
  if (smem > 200 * 1024) return CSA_ERR_UNSUPPORTED;
  dim3 grid(entry_count, b);
  const int rows_per_thread = (R + rg - 1) / rg;
  auto go = [&](auto kern) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, nt, smem, st>>>(a);
  };
  if (in_dtype == CSA_F32) {
    if (rows_per_thread <= 1) go(compress_kernel<float, 1>);
    else if (rows_per_thread <= 2) go(compress_kernel<float, 2>);
    else go(compress_kernel<float, kUnroll>);
  } else {
    if (rows_per_thread <= 1) go(compress_kernel<__nv_bfloat16, 1>);
    else if (rows_per_thread <= 2) go(compress_kernel<__nv_bfloat16, 2>);
    else go(compress_kernel<__nv_bfloat16, kUnroll>);
  }
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

csa_status launch_quantize(int in_dtype, int out_dtype, const void* x, int rows, int d,
                           void* codes, void* scales, cudaStream_t st) {
  if (rows == 0) return CSA_OK;
  const int warps = 8;
  if (in_dtype == CSA_BF16 && d == 128 && (reinterpret_cast<uintptr_t>(x) & 7) == 0 &&
      (out_dtype == CSA_FP8_E4M3 || out_dtype == CSA_NVFP4) &&
      (out_dtype != CSA_NVFP4 || (reinterpret_cast<uintptr_t>(codes) & 1) == 0) &&
      (out_dtype != CSA_FP8_E4M3 || (reinterpret_cast<uintptr_t>(codes) & 3) == 0)) {
    const int rows_per_cta = warps * kQ128Rows;
    quantize128_kernel<<<(rows + rows_per_cta - 1) / rows_per_cta, warps * 32, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(x), rows, out_dtype, reinterpret_cast<uint8_t*>(codes),
        scales);
    CSA_CHECK_LAUNCH();
    return CSA_OK;
  }
  dim3 grid((rows + warps - 1) / warps);
  if (in_dtype == CSA_F32)
    quantize_kernel<float><<<grid, warps * 32, 0, st>>>(
        reinterpret_cast<const float*>(x), rows, d, out_dtype, reinterpret_cast<uint8_t*>(codes), scales);
  else
    quantize_kernel<__nv_bfloat16><<<grid, warps * 32, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(x), rows, d, out_dtype,
        reinterpret_cast<uint8_t*>(codes), scales);
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

}  // namespace csa
