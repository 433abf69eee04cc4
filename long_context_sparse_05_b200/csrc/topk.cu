// Causal top-k by radix select on the stored score bits.
//
// Method: "DeepSeek Technical Reports", section DSA (Top-k over the index
// scores of a query); "DeepSeek V4 结构速览", sections "核心设计" item 2 and
// "Lightning Indexer" (k among the causally visible entries).
//
// One CTA per query row.  Scores are mapped to order-preserving unsigned keys
// (16 bits for bf16, 32 for f32).  Each 8-bit digit, most significant first,
// gets a shared-memory histogram over the candidates that still match the
// chosen prefix; a warp scan of the 256 bins finds the digit holding the k-th
// largest key.  After the last digit the k-th key tau is exact and `need` says
// how many keys equal to tau are taken, lowest entry first.  A final ordered
// pass compacts the selection with block-wide prefix scans, so the
// output is ascending by entry without any sort.
#include "common.cuh"

namespace csa {

template <typename S> struct KeyOf;
template <> struct KeyOf<__nv_bfloat16> {
  using K = uint32_t;
  static constexpr int kBits = 16;
  __device__ static __forceinline__ uint32_t get(const __nv_bfloat16* p, int s) {
    uint32_t u = reinterpret_cast<const uint16_t*>(p)[s];
    if ((u & 0x7fffu) == 0) u = 0;   // -0 ties with +0
    return (u & 0x8000u) ? (~u & 0xffffu) : (u | 0x8000u);
  }
};
template <> struct KeyOf<float> {
  using K = uint32_t;
  static constexpr int kBits = 32;
  __device__ static __forceinline__ uint32_t get(const float* p, int s) {
    uint32_t u = __float_as_uint(p[s]);
    if ((u & 0x7fffffffu) == 0) u = 0;   // -0 ties with +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  }
};

constexpr int kTopkThreads = 512;

// Exclusive scan of one int per thread over the block; returns the block total.
__device__ __forceinline__ int block_excl_scan(int v, int* s_warp, int& total) {
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
    if (lane < nw) s_warp[lane] = w;   // inclusive warp totals
  }
  __syncthreads();
  total = s_warp[nw - 1];
  const int before = wid > 0 ? s_warp[wid - 1] : 0;
  return before + x - v;
}

template <typename S>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(
    const S* __restrict__ scores, const int32_t* __restrict__ q_pos, int m, int E, int k,
    int32_t* __restrict__ idx, int32_t* __restrict__ count) {
  using KO = KeyOf<S>;
  __shared__ int s_hist[256];
  __shared__ int s_warp[32];
  __shared__ uint32_t s_sel[2];   // chosen digit, count of keys above it
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const S* sc = scores + (size_t)row * E;
  int32_t* out = idx + (size_t)row * k;
  const int ev = visible_entries(q_pos[row], m, E);

  if (ev <= k) {
    for (int j = tid; j < k; j += blockDim.x) out[j] = j < ev ? j : -1;
    if (tid == 0) count[row] = ev;
    return;
  }

  uint32_t prefix = 0, pmask = 0;
  int need = k;   // keys still to take at or below the current prefix
#pragma unroll 1
  for (int shift = KO::kBits - 8; shift >= 0; shift -= 8) {
    for (int j = tid; j < 256; j += blockDim.x) s_hist[j] = 0;
    __syncthreads();
    for (int s = tid; s < ev; s += blockDim.x) {
      const uint32_t key = KO::get(sc, s);
      if ((key & pmask) == prefix) atomicAdd(&s_hist[(key >> shift) & 0xff], 1);
    }
    __syncthreads();
    if (tid < 32) {
      // bins 255..0 in descending order: lane l owns bins 255-8l .. 248-8l
      int local[8], run = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) { local[q] = s_hist[255 - 8 * tid - q]; run += local[q]; }
      int incl = run;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += y;
      }
      int above = incl - run;   // keys in bins strictly above this lane's first bin
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (above < need && above + local[q] >= need) {
          s_sel[0] = 255 - 8 * tid - q;
          s_sel[1] = above;
        }
        above += local[q];
      }
    }
    __syncthreads();
    const uint32_t dsel = s_sel[0];
    need -= (int)s_sel[1];
    prefix |= dsel << shift;
    pmask |= 0xffu << shift;
    __syncthreads();
  }
  const uint32_t tau = prefix;

  // ordered compaction: key > tau always; key == tau for the first `need` of them
  int base_sel = 0, base_eq = 0;
  for (int s0 = 0; s0 < ev; s0 += blockDim.x) {
    const int s = s0 + tid;
    uint32_t key = 0;
    if (s < ev) key = KO::get(sc, s);
    const int gt = (s < ev) && key > tau;
    const int eq = (s < ev) && key == tau;
    int tot_eq;
    const int rank_eq = base_eq + block_excl_scan(eq, s_warp, tot_eq);
    const int sel = gt || (eq && rank_eq < need);
    int tot_sel;
    const int pos = base_sel + block_excl_scan(sel, s_warp, tot_sel);
    if (sel && pos < k) out[pos] = s;
    base_eq += tot_eq;
    base_sel += tot_sel;
  }
  if (tid == 0) count[row] = k;
}

csa_status launch_topk(const void* scores, int score_dtype, const int32_t* q_pos, int m, int rows,
                       int E, int k, int32_t* idx, int32_t* count, cudaStream_t st) {
  if (rows == 0) return CSA_OK;
  if (score_dtype == CSA_BF16)
    topk_kernel<__nv_bfloat16><<<rows, kTopkThreads, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(scores), q_pos, m, E, k, idx, count);
  else
    topk_kernel<float><<<rows, kTopkThreads, 0, st>>>(
        reinterpret_cast<const float*>(scores), q_pos, m, E, k, idx, count);
  CSA_CHECK_LAUNCH();
  return CSA_OK;
}

}  // namespace csa
