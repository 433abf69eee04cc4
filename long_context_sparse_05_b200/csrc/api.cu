// Host side of the C ABI declared in include/csa.h: argument checks, kernel
// selection, launches, and the fused decode / prefill drivers.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

using namespace csa;

namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t dtype_row_bytes(int dt, int d) {
  switch (dt) {
    case CSA_F32: return (size_t)d * 4;
    case CSA_BF16: return (size_t)d * 2;
    case CSA_FP8_E4M3: return (size_t)d;
    case CSA_NVFP4: return (size_t)d / 2;
  }
  return 0;
}

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Bump allocator over a caller-provided workspace.
// With a NULL base it only measures (every take() returns NULL).
struct Carve {
  char* base; size_t cap; size_t used = 0; bool ok = true;
  Carve(void* b, size_t c) : base(static_cast<char*>(b)), cap(c) {}
  void* take(size_t bytes) {
    size_t off = align256(used);
    used = off + bytes;
    if (!base) return nullptr;
    if (used > cap) { ok = false; return nullptr; }
    return base + off;
  }
};

}  // namespace

extern "C" {

const char* csa_status_string(csa_status s) {
  switch (s) {
    case CSA_OK: return "CSA_OK";
    case CSA_ERR_INVALID_ARG: return "CSA_ERR_INVALID_ARG: invalid argument";
    case CSA_ERR_UNSUPPORTED: return "CSA_ERR_UNSUPPORTED: no kernel for this combination";
    case CSA_ERR_CUDA: return "CSA_ERR_CUDA: CUDA launch error";
    case CSA_ERR_TIMEOUT: return "CSA_ERR_TIMEOUT: bounded device wait gave up";
  }
  return "CSA_ERR_UNKNOWN";
}

int csa_version(void) { return 100; }

csa_status csa_compress(const csa_compress_params* p, const void* C_a, const void* Z_a,
                        const float* B_a, const void* C_b, const void* Z_b, const float* B_b,
                        int b, int n, int entry_begin, int entry_count, int out_entries_per_seq,
                        void* out, void* out_scales, cudaStream_t stream) {
  if (!p) return CSA_ERR_INVALID_ARG;
  if (p->m < 1 || p->c < 8 || p->c % 8 || p->d_rope < 0 || p->d_rope % 2 || p->d_rope > p->c)
    return CSA_ERR_INVALID_ARG;
  if (p->in_dtype != CSA_F32 && p->in_dtype != CSA_BF16) return CSA_ERR_INVALID_ARG;
  if (p->out_dtype < CSA_F32 || p->out_dtype > CSA_NVFP4) return CSA_ERR_INVALID_ARG;
  if (p->out_dtype == CSA_NVFP4 && p->c % 64) return CSA_ERR_INVALID_ARG;   // tiled key scales
  if (p->in_dtype == CSA_F32 && p->c % 4) return CSA_ERR_INVALID_ARG;
  if (b < 0 || n < 0 || entry_begin < 0 || entry_count < 0) return CSA_ERR_INVALID_ARG;
  if ((long long)p->m * (entry_begin + entry_count) > n) return CSA_ERR_INVALID_ARG;
  const int off = p->out_entry_offset;
  if (off < 0 || entry_begin < off || entry_begin + entry_count - off > out_entries_per_seq)
    return CSA_ERR_INVALID_ARG;
  if (p->out_dtype == CSA_NVFP4 && off % 128) return CSA_ERR_INVALID_ARG;
  if (b == 0 || entry_count == 0) return CSA_OK;
  if (!C_a || !Z_a || !B_a || !out) return CSA_ERR_INVALID_ARG;
  if (p->overlap && (!C_b || !Z_b || !B_b)) return CSA_ERR_INVALID_ARG;
  if ((p->out_dtype == CSA_FP8_E4M3 || p->out_dtype == CSA_NVFP4) && !out_scales)
    return CSA_ERR_INVALID_ARG;
  if (!aligned16(C_a) || !aligned16(Z_a) || (p->overlap && (!aligned16(C_b) || !aligned16(Z_b))))
    return CSA_ERR_INVALID_ARG;
  CompressArgs a{};
  a.C_a = C_a; a.Z_a = Z_a; a.B_a = B_a; a.C_b = C_b; a.Z_b = Z_b; a.B_b = B_b;
  a.n = n; a.m = p->m; a.overlap = p->overlap ? 1 : 0; a.c = p->c; a.d_rope = p->d_rope;
  a.apply_norm = p->apply_norm; a.out_dtype = p->out_dtype; a.entry_begin = entry_begin;
  a.out_E = out_entries_per_seq; a.theta = p->rope_theta; a.eps = p->eps;
  a.out = out; a.out_scales = out_scales; a.out_off = off;
  return launch_compress(a, p->in_dtype, b, entry_count, stream);
}

csa_status csa_quantize(int in_dtype, int out_dtype, const void* x, int rows, int d, void* codes,
                        void* scales, cudaStream_t stream) {
  if (in_dtype != CSA_F32 && in_dtype != CSA_BF16) return CSA_ERR_INVALID_ARG;
  if (out_dtype != CSA_FP8_E4M3 && out_dtype != CSA_NVFP4) return CSA_ERR_INVALID_ARG;
  if (rows < 0 || d <= 0 || d % 16) return CSA_ERR_INVALID_ARG;
  if (rows == 0) return CSA_OK;
  if (!x || !codes || !scales || !aligned16(codes)) return CSA_ERR_INVALID_ARG;
  return launch_quantize(in_dtype, out_dtype, x, rows, d, codes, scales, stream);
}

}  // extern "C"

namespace {

// q_raw: bf16 index queries the FP8 tensor-core kernel quantises itself (decode, one query
// per sequence); q_I and q_scales are then unused.  There is no other kernel for it.
csa_status index_scores_impl(const csa_index_params* p, const void* q_I, const void* q_scales,
                             const float* w, const void* k_I, const void* k_scales,
                             const int32_t* q_pos, int b, int T, int E_cap, int E, void* scores,
                             cudaStream_t stream, int pdl, int all_visible, int dep_entry,
                             const void* q_raw = nullptr) {
  if (q_raw) { q_I = q_raw; q_scales = k_scales; }
  if (!p) return CSA_ERR_INVALID_ARG;
  if (p->H_I < 1 || p->d_I < 16 || p->d_I % 16 || p->m < 1) return CSA_ERR_INVALID_ARG;
  if (p->qk_dtype < CSA_F32 || p->qk_dtype > CSA_NVFP4 || p->qk_dtype == CSA_BF16)
    return CSA_ERR_INVALID_ARG;
  if (p->score_dtype != CSA_F32 && p->score_dtype != CSA_BF16) return CSA_ERR_INVALID_ARG;
  if (b < 0 || T < 0 || E < 0 || E > E_cap) return CSA_ERR_INVALID_ARG;
  if (b == 0 || T == 0 || E == 0) return CSA_OK;
  if (!q_I || !w || !k_I || !q_pos || !scores) return CSA_ERR_INVALID_ARG;
  if (p->qk_dtype != CSA_F32 && (!q_scales || !k_scales)) return CSA_ERR_INVALID_ARG;
  if (p->qk_dtype == CSA_NVFP4 && p->d_I % 64) return CSA_ERR_INVALID_ARG;   // tiled key scales
  IndexArgs a{};
  a.q = q_I; a.q_scales = q_scales; a.w = w; a.k = k_I; a.k_scales = k_scales; a.q_pos = q_pos;
  a.T = T; a.H = p->H_I; a.d = p->d_I; a.m = p->m; a.qk_dtype = p->qk_dtype;
  a.score_dtype = p->score_dtype; a.E_cap = E_cap; a.E = E; a.scores = scores;
  a.pdl = pdl; a.all_visible = all_visible; a.dep_entry = dep_entry; a.q_raw = q_raw;
  csa_status st = launch_index_scores_tc(a, b, stream);
  if (st != CSA_ERR_UNSUPPORTED || q_raw) return st;
  st = launch_index_scores_fp4_tc(a, b, stream);
  if (st != CSA_ERR_UNSUPPORTED) return st;
  return launch_index_scores_simt(a, b, stream);
}

csa_status topk_impl(const void* scores, int score_dtype, const int32_t* q_pos, int m, int b,
                     int T, int E, int k, int32_t* idx, int32_t* count, void* ws, size_t ws_bytes,
                     cudaStream_t stream, bool pdl) {
  if (score_dtype != CSA_F32 && score_dtype != CSA_BF16) return CSA_ERR_INVALID_ARG;
  if (m < 1 || b < 0 || T < 0 || E < 0 || k < 1) return CSA_ERR_INVALID_ARG;
  if (b == 0 || T == 0) return CSA_OK;
  if (!scores || !q_pos || !idx || !count) return CSA_ERR_INVALID_ARG;
  const size_t need = topk_workspace_bytes(b * T, E, k, score_dtype);
  if (need && (!ws || ws_bytes < need)) return CSA_ERR_INVALID_ARG;
  const csa_status st = launch_topk_search(scores, score_dtype, q_pos, m, b * T, E, k, idx, count,
                                           ws, ws_bytes, stream, pdl);
  if (st != CSA_ERR_UNSUPPORTED) return st;
  return launch_topk(scores, score_dtype, q_pos, m, b * T, E, k, idx, count, stream);
}

csa_status sparse_attn_impl(const csa_attn_params* p, const void* q, const void* kv_comp,
                            int E_cap, const int32_t* idx, const int32_t* count,
                            const void* kv_win, int n, const int32_t* q_pos, const float* sink,
                            int b, int T, void* out, float* lse, void* ws, size_t ws_bytes,
                            cudaStream_t stream, int pdl) {
  if (!p) return CSA_ERR_INVALID_ARG;
  if (p->H < 1 || p->d < 8 || p->d % 8 || p->n_w < 0 || p->m < 1) return CSA_ERR_INVALID_ARG;
  if (p->d_rope_out < 0 || p->d_rope_out % 2 || p->d_rope_out > p->d) return CSA_ERR_INVALID_ARG;
  if (p->d_rope_out > 0 && !(p->rope_theta > 0.0)) return CSA_ERR_INVALID_ARG;
  if (p->dtype != CSA_F32 && p->dtype != CSA_BF16) return CSA_ERR_INVALID_ARG;
  if (b < 0 || T < 0 || E_cap < 0 || n < 1) return CSA_ERR_INVALID_ARG;
  if (idx && (p->k < 1 || !count)) return CSA_ERR_INVALID_ARG;
  if (b == 0 || T == 0) return CSA_OK;
  if (!q || !kv_win || !q_pos || !sink || !out) return CSA_ERR_INVALID_ARG;
  if (E_cap > 0 && !kv_comp) return CSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv_win) || (kv_comp && !aligned16(kv_comp)) || !aligned16(out))
    return CSA_ERR_INVALID_ARG;
  AttnArgs a{};
  a.q = q; a.kv = kv_comp; a.idx = idx; a.count = count; a.win = kv_win; a.q_pos = q_pos;
  a.sink = sink; a.T = T; a.H = p->H; a.d = p->d; a.n_w = p->n_w; a.m = p->m; a.k = p->k;
  a.E_cap = E_cap; a.n = n; a.scale = p->scale; a.out = out; a.lse = lse; a.pdl = pdl;
  a.d_rope_out = p->d_rope_out; a.theta = p->rope_theta;
  csa_status st = launch_attn_tc(a, b, p->dtype, ws, ws_bytes, stream);
  if (st != CSA_ERR_UNSUPPORTED) return st;
  return launch_attn_simt(a, b, p->dtype, stream);
}

}  // namespace

extern "C" {

csa_status csa_index_scores(const csa_index_params* p, const void* q_I, const void* q_scales,
                            const float* w, const void* k_I, const void* k_scales,
                            const int32_t* q_pos, int b, int T, int E_cap, int E, void* scores,
                            cudaStream_t stream) {
  return index_scores_impl(p, q_I, q_scales, w, k_I, k_scales, q_pos, b, T, E_cap, E, scores,
                           stream, 0, 0, -1);
}

size_t csa_topk_workspace_size(int score_dtype, int b, int T, int E, int k) {
  if (b <= 0 || T <= 0 || E <= 0 || k <= 0) return 0;
  return topk_workspace_bytes(b * T, E, k, score_dtype);
}

csa_status csa_topk(const void* scores, int score_dtype, const int32_t* q_pos, int m, int b, int T,
                    int E, int k, int32_t* idx, int32_t* count, void* ws, size_t ws_bytes,
                    cudaStream_t stream) {
  return topk_impl(scores, score_dtype, q_pos, m, b, T, E, k, idx, count, ws, ws_bytes, stream,
                   false);
}

size_t csa_sparse_attn_workspace_size(const csa_attn_params* p, int b, int T, int E_cap) {
  if (!p) return 0;
  return attn_tc_workspace_bytes(p->H, p->d, p->k, p->n_w, b, T, E_cap, p->dtype);
}

csa_status csa_sparse_attn(const csa_attn_params* p, const void* q, const void* kv_comp, int E_cap,
                           const int32_t* idx, const int32_t* count, const void* kv_win, int n,
                           const int32_t* q_pos, const float* sink, int b, int T, void* out,
                           float* lse, void* ws, size_t ws_bytes, cudaStream_t stream) {
  return sparse_attn_impl(p, q, kv_comp, E_cap, idx, count, kv_win, n, q_pos, sink, b, T, out, lse,
                          ws, ws_bytes, stream, 0);
}

// ---------------------------------------------------------------------------
// hierarchical indexer: top-k within a candidate pool
// ---------------------------------------------------------------------------

namespace {

struct PoolWs {
  void* gather; void* scores; void* topk_ws; size_t topk_ws_bytes; int32_t* gpos;
};

size_t pool_layout(int fmt, int d, int rows, int P, int k, void* ws, size_t cap, PoolWs* o) {
  Carve cv(ws, cap);
  PoolWs d_{};
  size_t o_pos = 0;
  const size_t gb = pool_gather_bytes(fmt, rows, P, d, nullptr, nullptr, &o_pos);
  d_.gather = cv.take(gb);
  if (d_.gather) d_.gpos = reinterpret_cast<int32_t*>(static_cast<char*>(d_.gather) + o_pos);
  d_.scores = cv.take((size_t)rows * P * 2);
  d_.topk_ws_bytes = topk_workspace_bytes(rows, P, k, CSA_BF16);
  d_.topk_ws = cv.take(d_.topk_ws_bytes);
  if (o) *o = d_;
  return cv.ok ? align256(cv.used) : 0;
}

csa_status pool_topk_impl(const csa_index_params* p, const void* q_I, const void* q_scales,
                          const float* w, const void* k_I, const void* k_scales,
                          const int32_t* q_pos, int b, int T, int E_cap, int E,
                          const int32_t* pool, const int32_t* pool_count, int P, int k,
                          int32_t* idx, int32_t* count, void* ws, size_t ws_bytes,
                          cudaStream_t stream, bool pdl) {
  if (!p) return CSA_ERR_INVALID_ARG;
  if (p->H_I < 1 || p->d_I < 16 || p->d_I % 16 || p->m < 1) return CSA_ERR_INVALID_ARG;
  if (p->qk_dtype != CSA_F32 && p->qk_dtype != CSA_FP8_E4M3 && p->qk_dtype != CSA_NVFP4)
    return CSA_ERR_INVALID_ARG;
  if (p->qk_dtype == CSA_NVFP4 && p->d_I % 64) return CSA_ERR_INVALID_ARG;
  if (b < 0 || T < 0 || E < 0 || E > E_cap || P < 1 || k < 1) return CSA_ERR_INVALID_ARG;
  if (b == 0 || T == 0) return CSA_OK;
  if (!q_I || !w || !k_I || !q_pos || !pool || !pool_count || !idx || !count)
    return CSA_ERR_INVALID_ARG;
  if (p->qk_dtype != CSA_F32 && (!q_scales || !k_scales)) return CSA_ERR_INVALID_ARG;
  if (!aligned16(k_I)) return CSA_ERR_INVALID_ARG;
  const int rows = b * T;
  PoolWs d{};
  if (pool_layout(p->qk_dtype, p->d_I, rows, P, k, ws, ws_bytes, &d) == 0 || !ws ||
      ws_bytes < pool_layout(p->qk_dtype, p->d_I, rows, P, k, nullptr, 0, nullptr))
    return CSA_ERR_INVALID_ARG;
  csa_status st = launch_pool_gather(p->qk_dtype, pool, pool_count, q_pos, k_I, k_scales, rows, T,
                                     P, E_cap, E, p->m, p->d_I, d.gather, stream, pdl);
  if (st) return st;
  size_t o_sc = 0;
  pool_gather_bytes(p->qk_dtype, rows, P, p->d_I, &o_sc, nullptr, nullptr);
  const int P_cap = (P + 255) / 256 * 256;
  csa_index_params ip = *p;
  ip.score_dtype = CSA_BF16;
  st = index_scores_impl(&ip, q_I, q_scales, w, d.gather,
                         p->qk_dtype == CSA_F32 ? nullptr : static_cast<char*>(d.gather) + o_sc,
                         d.gpos, rows, 1, P_cap, P, d.scores, stream, 1, 0, -1);
  if (st) return st;
  st = topk_impl(d.scores, CSA_BF16, d.gpos, p->m, rows, 1, P, k, idx, count, d.topk_ws,
                 d.topk_ws_bytes, stream, true);
  if (st) return st;
  return launch_pool_map(d.gather, p->qk_dtype, rows, P, p->d_I, k, idx, count, stream, true);
}

}  // namespace

size_t csa_pool_topk_workspace_size(const csa_index_params* p, int b, int T, int P, int k) {
  if (!p || b <= 0 || T <= 0 || P <= 0 || k <= 0) return 0;
  return pool_layout(p->qk_dtype, p->d_I, b * T, P, k, nullptr, 0, nullptr);
}

csa_status csa_pool_topk(const csa_index_params* p, const void* q_I, const void* q_scales,
                         const float* w, const void* k_I, const void* k_scales,
                         const int32_t* q_pos, int b, int T, int E_cap, int E,
                         const int32_t* pool, const int32_t* pool_count, int P, int k,
                         int32_t* idx, int32_t* count, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
  return pool_topk_impl(p, q_I, q_scales, w, k_I, k_scales, q_pos, b, T, E_cap, E, pool,
                        pool_count, P, k, idx, count, ws, ws_bytes, stream, false);
}

// ---------------------------------------------------------------------------
// grouped output projection
// ---------------------------------------------------------------------------

size_t csa_out_proj_workspace_size(int T, int H, int d, int g, int d_g) {
  return out_proj_workspace_bytes(T, H, d, g, d_g);
}

csa_status csa_out_proj(const void* o, const void* W, int T, int H, int d, int g, int d_g,
                        void* y, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (T < 0 || H < 1 || d < 1 || g < 1 || d_g < 1) return CSA_ERR_INVALID_ARG;
  if (!out_proj_supported(H, d, g, d_g)) return CSA_ERR_INVALID_ARG;
  if (T == 0) return CSA_OK;
  if (!o || !W || !y || !aligned16(o) || !aligned16(W) || !aligned16(y)) return CSA_ERR_INVALID_ARG;
  return launch_out_proj(o, W, T, H, d, g, d_g, y, ws, ws_bytes, stream, false);
}

// ---------------------------------------------------------------------------
// decode
// ---------------------------------------------------------------------------

namespace {

struct DecodeWs {
  void* qI_codes; void* qI_scales; void* scores; int32_t* idx; int32_t* count; int32_t* qpos;
  void* attn_ws; size_t attn_ws_bytes; void* topk_ws; size_t topk_ws_bytes;
  void* pool_ws; size_t pool_ws_bytes;
};

size_t decode_layout(const csa_decode_params* p, void* ws, size_t cap, DecodeWs* o) {
  Carve cv(ws, cap);
  DecodeWs d{};
  const int b = p->b;
  d.qpos = static_cast<int32_t*>(cv.take((size_t)b * 4));
  if (!p->hca) {
    const int E = p->L / p->m;
    if (p->idx_dtype != CSA_F32) {
      d.qI_codes = cv.take((size_t)b * p->H_I * dtype_row_bytes(p->idx_dtype, p->c_I));
      d.qI_scales = cv.take(p->idx_dtype == CSA_FP8_E4M3 ? (size_t)b * p->H_I * 4
                                                          : (size_t)b * p->H_I * (p->c_I / 16));
    }
    d.idx = static_cast<int32_t*>(cv.take((size_t)b * p->k * 4));
    d.count = static_cast<int32_t*>(cv.take((size_t)b * 4));
    if (p->mode == CSA_MODE_FULL) {
      d.scores = cv.take((size_t)b * E * 2);
      d.topk_ws_bytes = topk_workspace_bytes(b, E, p->k, CSA_BF16);
      d.topk_ws = cv.take(d.topk_ws_bytes);
    } else if (p->mode == CSA_MODE_REINDEX) {
      d.pool_ws_bytes = pool_layout(p->idx_dtype, p->c_I, b, p->P, p->k, nullptr, 0, nullptr);
      d.pool_ws = cv.take(d.pool_ws_bytes);
    }
  }
  csa_attn_params ap{p->H, p->c, p->n_w, p->scale, p->m, p->hca ? 0 : p->k, p->kv_dtype,
                     p->inv_rope ? p->d_rope : 0, p->rope_theta};
  d.attn_ws_bytes = csa_sparse_attn_workspace_size(&ap, b, 1, p->E_cap);
  d.attn_ws = cv.take(d.attn_ws_bytes);
  if (o) *o = d;
  return cv.ok ? align256(cv.used) : 0;
}

}  // namespace

namespace {
// The FP8 tensor-core indexer quantises the bf16 index queries itself (so the prologue
// does not, and the indexer does not wait for it except for the key page it writes).
bool indexer_takes_raw_q(int hca, int idx_dtype, int kv_dtype, int H_I, int c_I) {
  return !hca && idx_dtype == CSA_FP8_E4M3 && kv_dtype == CSA_BF16 && H_I == 64 && c_I == 128;
}
}  // namespace

int csa_decode_launch_count(const csa_decode_params* p) {
  if (!p || p->b <= 0) return 0;
  int n = 1;                                   // prologue: compressors, quantiser, positions
  if (!p->hca && p->mode == CSA_MODE_FULL)
    n += 1 + (topk_workspace_bytes(p->b, p->L / p->m, p->k, CSA_BF16) ? 2 : 1);
  if (!p->hca && p->mode == CSA_MODE_REINDEX)  // gather, indexer, top-k, map
    n += 3 + (topk_workspace_bytes(p->b, p->P, p->k, CSA_BF16) ? 2 : 1);
  n += attn_launch_count(p->H, p->c, p->hca ? 0 : p->k, p->n_w, p->b, 1, p->E_cap, p->kv_dtype);
  return n;
}

size_t csa_decode_workspace_size(const csa_decode_params* p) {
  if (!p) return 0;
  return decode_layout(p, nullptr, 0, nullptr);
}

csa_status csa_decode(const csa_decode_params* p, const csa_decode_tensors* x, void* ws,
                      size_t ws_bytes, cudaStream_t stream) {
  if (!p || !x) return CSA_ERR_INVALID_ARG;
  if (p->b < 0 || p->m < 1 || p->L < p->m || p->L % p->m) return CSA_ERR_INVALID_ARG;
  const int E = p->L / p->m;
  if (E > p->E_cap) return CSA_ERR_INVALID_ARG;
  if (!p->hca && (p->k < 1 || p->c_I < 16 || p->H_I < 1)) return CSA_ERR_INVALID_ARG;
  if (p->mode != CSA_MODE_FULL && p->mode != CSA_MODE_REUSE && p->mode != CSA_MODE_REINDEX)
    return CSA_ERR_INVALID_ARG;
  if (p->hca && p->mode != CSA_MODE_FULL) return CSA_ERR_INVALID_ARG;
  if (p->mode == CSA_MODE_REINDEX && p->P < 1) return CSA_ERR_INVALID_ARG;
  if (p->b == 0) return CSA_OK;
  if (p->mode == CSA_MODE_REUSE && (!x->idx_in || !x->count_in)) return CSA_ERR_INVALID_ARG;
  if (p->mode == CSA_MODE_REINDEX && (!x->pool || !x->pool_count)) return CSA_ERR_INVALID_ARG;
  DecodeWs d{};
  const size_t need = decode_layout(p, ws, ws_bytes, &d);
  if (need == 0 || !ws || ws_bytes < csa_decode_workspace_size(p)) return CSA_ERR_INVALID_ARG;
  const int b = p->b;
  const int t = p->L - 1;
  if (!x->C_a || !x->Z_a || !x->B_a || !x->kv_cache || !x->q || !x->kv_win || !x->sink || !x->out)
    return CSA_ERR_INVALID_ARG;
  if (!p->hca && (!x->C_b || !x->Z_b || !x->B_b || !x->CI_a || !x->ZI_a || !x->BI_a || !x->CI_b ||
                  !x->ZI_b || !x->BI_b || !x->kI_cache || !x->q_I || !x->w))
    return CSA_ERR_INVALID_ARG;
  if (!p->hca && p->idx_dtype != CSA_F32 && !x->kI_scales) return CSA_ERR_INVALID_ARG;
  if (p->kv_dtype != CSA_F32 && p->kv_dtype != CSA_BF16) return CSA_ERR_INVALID_ARG;
  if (!p->hca && p->idx_dtype == CSA_F32 && p->kv_dtype != CSA_F32) return CSA_ERR_UNSUPPORTED;
  if (p->c < 8 || p->c % 8 || p->d_rope < 0 || p->d_rope % 2 || p->d_rope > p->c)
    return CSA_ERR_INVALID_ARG;
  if (!p->hca && (p->c_I % 16 || p->d_rope_I < 0 || p->d_rope_I % 2 || p->d_rope_I > p->c_I))
    return CSA_ERR_INVALID_ARG;
  if (!p->hca && p->idx_dtype == CSA_NVFP4 && p->c_I % 64) return CSA_ERR_INVALID_ARG;
  if (!aligned16(x->C_a) || !aligned16(x->Z_a) ||
      (!p->hca && (!aligned16(x->C_b) || !aligned16(x->Z_b) || !aligned16(x->CI_a) ||
                   !aligned16(x->ZI_a) || !aligned16(x->CI_b) || !aligned16(x->ZI_b))))
    return CSA_ERR_INVALID_ARG;

  // 1-2. one prologue launch: compress the entry the new token completes (latent and
  //      index key), quantise the index queries, write the query positions
  PrologueArgs pa{};
  pa.main.C_a = x->C_a; pa.main.Z_a = x->Z_a; pa.main.B_a = x->B_a;
  pa.main.C_b = x->C_b; pa.main.Z_b = x->Z_b; pa.main.B_b = x->B_b;
  pa.main.n = p->L; pa.main.m = p->m; pa.main.overlap = p->hca ? 0 : 1; pa.main.c = p->c;
  pa.main.d_rope = p->d_rope; pa.main.apply_norm = 1; pa.main.out_dtype = p->kv_dtype;
  pa.main.entry_begin = E - 1; pa.main.out_E = p->E_cap; pa.main.theta = p->rope_theta;
  pa.main.eps = p->eps; pa.main.out = x->kv_cache; pa.main.out_scales = nullptr;
  pa.nbranch = p->hca ? 1 : 2;
  pa.b = b; pa.t = t; pa.qpos = d.qpos;
  const void* qI = x->q_I;
  const void* qs = nullptr;
  const bool raw_q = p->mode == CSA_MODE_FULL &&
                     indexer_takes_raw_q(p->hca, p->idx_dtype, p->kv_dtype, p->H_I, p->c_I);
  if (!p->hca) {
    pa.index = pa.main;
    pa.index.C_a = x->CI_a; pa.index.Z_a = x->ZI_a; pa.index.B_a = x->BI_a;
    pa.index.C_b = x->CI_b; pa.index.Z_b = x->ZI_b; pa.index.B_b = x->BI_b;
    pa.index.c = p->c_I; pa.index.d_rope = p->d_rope_I; pa.index.out_dtype = p->idx_dtype;
    pa.index.out = x->kI_cache; pa.index.out_scales = x->kI_scales;
    if (p->idx_dtype != CSA_F32 && !raw_q) {
      pa.q_in = x->q_I; pa.q_rows = b * p->H_I; pa.q_d = p->c_I; pa.q_dtype = p->idx_dtype;
      pa.q_codes = static_cast<uint8_t*>(d.qI_codes); pa.q_scales = d.qI_scales;
      qI = d.qI_codes; qs = d.qI_scales;
    }
  }
  csa_status st = launch_decode_prologue(pa, p->kv_dtype, stream);
  if (st) return st;
  const int32_t* idx = nullptr;
  const int32_t* cnt = nullptr;
  if (!p->hca && p->mode == CSA_MODE_REUSE) {
    // CSA2 Reuse mode: an earlier layer's selection, no scoring
    idx = x->idx_in; cnt = x->count_in;
  } else if (!p->hca && p->mode == CSA_MODE_REINDEX) {
    // CSA2 Reindex mode with the hierarchical indexer: score the candidate pool only
    int32_t* io = x->idx_out ? x->idx_out : d.idx;
    int32_t* co = x->count_out ? x->count_out : d.count;
    csa_index_params ip{p->H_I, p->c_I, p->m, p->idx_dtype, CSA_BF16};
    st = pool_topk_impl(&ip, qI, qs, x->w, x->kI_cache, x->kI_scales, d.qpos, b, 1, p->E_cap, E,
                        x->pool, x->pool_count, p->P, p->k, io, co, d.pool_ws, d.pool_ws_bytes,
                        stream, true);
    if (st) return st;
    idx = io; cnt = co;
  } else if (!p->hca) {
    // 3. score all entries
    // (programmatic dependent launches from here on: each kernel starts while its
    //  predecessor drains and waits for it only where it reads its outputs)
    csa_index_params ip{p->H_I, p->c_I, p->m, p->idx_dtype, CSA_BF16};
    st = index_scores_impl(&ip, qI, qs, x->w, x->kI_cache, x->kI_scales, d.qpos, b, 1, p->E_cap,
                           E, d.scores, stream, 1, 1, E - 1, raw_q ? x->q_I : nullptr);
    if (st) return st;
    // 4. top-k
    int32_t* io = x->idx_out ? x->idx_out : d.idx;
    int32_t* co = x->count_out ? x->count_out : d.count;
    st = topk_impl(d.scores, CSA_BF16, d.qpos, p->m, b, 1, E, p->k, io, co, d.topk_ws,
                   d.topk_ws_bytes, stream, true);
    if (st) return st;
    idx = io; cnt = co;
  }
  // 4. attention over the selection (or all entries) plus the window
  csa_attn_params ap{p->H, p->c, p->n_w, p->scale, p->m, p->hca ? 0 : p->k, p->kv_dtype,
                     p->inv_rope ? p->d_rope : 0, p->rope_theta};
  return sparse_attn_impl(&ap, x->q, x->kv_cache, p->E_cap, idx, cnt, x->kv_win, p->L, d.qpos,
                          x->sink, b, 1, x->out, x->lse, d.attn_ws, d.attn_ws_bytes, stream, 1);
}

// ---------------------------------------------------------------------------
// paged decode: classical paged caches + per-sequence state, any positions
// ---------------------------------------------------------------------------

namespace {

struct PagedWs {
  void* qI_codes; void* qI_scales; void* scores; int32_t* idx; int32_t* count; int32_t* qpos;
  void* attn_ws; size_t attn_ws_bytes; void* topk_ws; size_t topk_ws_bytes;
};

size_t paged_layout(const csa_paged_params* p, void* ws, size_t cap, PagedWs* o) {
  Carve cv(ws, cap);
  PagedWs d{};
  const int b = p->b;
  const int E = p->L_max / p->m;
  d.qpos = static_cast<int32_t*>(cv.take((size_t)b * 4));
  if (!p->hca) {
    if (p->idx_dtype != CSA_F32) {
      d.qI_codes = cv.take((size_t)b * p->H_I * dtype_row_bytes(p->idx_dtype, p->c_I));
      d.qI_scales = cv.take(p->idx_dtype == CSA_FP8_E4M3 ? (size_t)b * p->H_I * 4
                                                          : (size_t)b * p->H_I * (p->c_I / 16));
    }
    d.idx = static_cast<int32_t*>(cv.take((size_t)b * p->k * 4));
    d.count = static_cast<int32_t*>(cv.take((size_t)b * 4));
    d.scores = cv.take((size_t)b * std::max(E, 1) * 2);
    d.topk_ws_bytes = topk_workspace_bytes(b, E, p->k, CSA_BF16);
    d.topk_ws = cv.take(d.topk_ws_bytes);
  }
  csa_attn_params ap{p->H, p->c, p->n_w, p->scale, p->m, p->hca ? 0 : p->k, p->kv_dtype,
                     p->inv_rope ? p->d_rope : 0, p->rope_theta};
  d.attn_ws_bytes = csa_sparse_attn_workspace_size(&ap, b, 1, p->max_pages * kPageEntries);
  d.attn_ws = cv.take(d.attn_ws_bytes);
  if (o) *o = d;
  return cv.ok ? align256(cv.used) : 0;
}

}  // namespace

size_t csa_decode_paged_workspace_size(const csa_paged_params* p) {
  if (!p || p->b <= 0 || p->m < 1) return 0;
  return paged_layout(p, nullptr, 0, nullptr);
}

namespace {
// Paged c128a: the entry is compressed by the cluster-split kernel after the prologue
// (which then only appends the rows and copies the positions).
bool paged_split(const csa_paged_params* p) {
  if (!p->hca) return false;
  CompressArgs a{};
  a.c = p->c; a.m = p->m; a.overlap = 0; a.out_dtype = p->kv_dtype; a.d_rope = p->d_rope;
  return compress_split_supported(a, p->kv_dtype);
}
}  // namespace

int csa_decode_paged_launch_count(const csa_paged_params* p) {
  if (!p || p->b <= 0 || p->m < 1) return 0;
  int n = 1 + (paged_split(p) ? 1 : 0);
  if (!p->hca) n += 1 + (topk_workspace_bytes(p->b, p->L_max / p->m, p->k, CSA_BF16) ? 2 : 1);
  n += attn_launch_count(p->H, p->c, p->hca ? 0 : p->k, p->n_w, p->b, 1,
                         p->max_pages * kPageEntries, p->kv_dtype);
  return n;
}

csa_status csa_decode_paged(const csa_paged_params* p, const csa_paged_tensors* x, void* ws,
                            size_t ws_bytes, cudaStream_t stream) {
  if (!p || !x) return CSA_ERR_INVALID_ARG;
  if (p->b < 0 || p->m < 1 || p->L_max < 1 || p->max_pages < 1 || p->num_pages < 1 || p->n_w < 1)
    return CSA_ERR_INVALID_ARG;
  if ((long long)p->max_pages * kPageEntries * p->m < p->L_max) return CSA_ERR_INVALID_ARG;
  if (p->kv_dtype != CSA_BF16 && p->kv_dtype != CSA_F32) return CSA_ERR_INVALID_ARG;
  if (p->c < 8 || p->c % 8 || p->d_rope < 0 || p->d_rope % 2 || p->d_rope > p->c)
    return CSA_ERR_INVALID_ARG;
  if (!p->hca && (p->k < 1 || p->c_I < 16 || p->c_I % 16 || p->H_I < 1 || p->d_rope_I < 0 ||
                  p->d_rope_I % 2 || p->d_rope_I > p->c_I))
    return CSA_ERR_INVALID_ARG;
  if (!p->hca && p->idx_dtype != CSA_FP8_E4M3 && p->idx_dtype != CSA_NVFP4)
    return CSA_ERR_UNSUPPORTED;   // the paged key cache is read by the tensor-core indexers
  if (!p->hca && p->idx_dtype == CSA_NVFP4 && p->c_I % 64) return CSA_ERR_INVALID_ARG;
  if (p->b == 0) return CSA_OK;
  PagedWs d{};
  if (paged_layout(p, ws, ws_bytes, &d) == 0 || !ws || ws_bytes < csa_decode_paged_workspace_size(p))
    return CSA_ERR_INVALID_ARG;
  if (!x->kv_pages || !x->block_table || !x->win || !x->tail_C_a || !x->tail_Z_a || !x->pos ||
      !x->new_C_a || !x->new_Z_a || !x->new_win || !x->B_a || !x->q || !x->sink || !x->out)
    return CSA_ERR_INVALID_ARG;
  if (!p->hca && (!x->tail_C_b || !x->tail_Z_b || !x->new_C_b || !x->new_Z_b || !x->B_b ||
                  !x->kI_pages || !x->kI_scales || !x->tail_CI_a || !x->tail_ZI_a ||
                  !x->tail_CI_b || !x->tail_ZI_b || !x->new_CI_a || !x->new_ZI_a ||
                  !x->new_CI_b || !x->new_ZI_b || !x->BI_a || !x->BI_b || !x->q_I || !x->w))
    return CSA_ERR_INVALID_ARG;
  const void* ptrs16[] = {x->kv_pages, x->win, x->tail_C_a, x->tail_Z_a, x->new_C_a, x->new_Z_a,
                          x->new_win, x->q, x->out};
  for (const void* q : ptrs16)
    if (!aligned16(q)) return CSA_ERR_INVALID_ARG;
  if (!p->hca) {
    const void* more[] = {x->tail_C_b, x->tail_Z_b, x->new_C_b, x->new_Z_b, x->kI_pages,
                          x->kI_scales, x->tail_CI_a, x->tail_ZI_a, x->tail_CI_b, x->tail_ZI_b,
                          x->new_CI_a, x->new_ZI_a, x->new_CI_b, x->new_ZI_b};
    for (const void* q : more)
      if (!aligned16(q)) return CSA_ERR_INVALID_ARG;
  }
  const int b = p->b;
  const int E = p->L_max / p->m;
  const int ring = p->hca ? p->m : 2 * p->m;
  const size_t eb = p->kv_dtype == CSA_F32 ? 4 : 2;
  if ((size_t)p->c * eb % 16 || (!p->hca && (size_t)p->c_I * eb % 16)) return CSA_ERR_INVALID_ARG;

  // 1. prologue: append the new token's rows to the state, compress the entries the new
  //    tokens complete into their pages, quantise the index queries, copy the positions
  PrologueArgs pa{};
  CompressArgs& mc = pa.main;
  mc.C_a = x->tail_C_a; mc.Z_a = x->tail_Z_a; mc.B_a = x->B_a;
  mc.C_b = x->tail_C_b; mc.Z_b = x->tail_Z_b; mc.B_b = x->B_b;
  mc.n = ring; mc.m = p->m; mc.overlap = p->hca ? 0 : 1; mc.c = p->c; mc.d_rope = p->d_rope;
  mc.apply_norm = 1; mc.out_dtype = p->kv_dtype; mc.entry_begin = 0;
  mc.out_E = p->max_pages * kPageEntries; mc.theta = p->rope_theta; mc.eps = p->eps;
  mc.out = x->kv_pages; mc.out_scales = nullptr;
  mc.ring = ring; mc.pos = x->pos;
  mc.new_C_a = x->new_C_a; mc.new_Z_a = x->new_Z_a; mc.new_C_b = x->new_C_b; mc.new_Z_b = x->new_Z_b;
  mc.block_table = x->block_table; mc.max_pages = p->max_pages; mc.num_pages = p->num_pages;
  pa.nbranch = p->hca ? 1 : 2;
  pa.b = b; pa.t = 0; pa.qpos = d.qpos;
  pa.paged = 1; pa.win = x->win; pa.new_win = x->new_win; pa.win_ring = p->n_w;
  const void* qI = x->q_I;
  const void* qs = nullptr;
  const bool raw_q = indexer_takes_raw_q(p->hca, p->idx_dtype, p->kv_dtype, p->H_I, p->c_I);
  if (!p->hca) {
    CompressArgs& ic = pa.index;
    ic = mc;
    ic.C_a = x->tail_CI_a; ic.Z_a = x->tail_ZI_a; ic.B_a = x->BI_a;
    ic.C_b = x->tail_CI_b; ic.Z_b = x->tail_ZI_b; ic.B_b = x->BI_b;
    ic.c = p->c_I; ic.d_rope = p->d_rope_I; ic.out_dtype = p->idx_dtype;
    ic.out = x->kI_pages; ic.out_scales = x->kI_scales;
    ic.new_C_a = x->new_CI_a; ic.new_Z_a = x->new_ZI_a; ic.new_C_b = x->new_CI_b; ic.new_Z_b = x->new_ZI_b;
    if (!raw_q) {
      pa.q_in = x->q_I; pa.q_rows = b * p->H_I; pa.q_d = p->c_I; pa.q_dtype = p->idx_dtype;
      pa.q_codes = static_cast<uint8_t*>(d.qI_codes); pa.q_scales = d.qI_scales;
      qI = d.qI_codes; qs = d.qI_scales;
    }
  }
  const bool split = paged_split(p);
  pa.skip_compress = split ? 1 : 0;
  csa_status st = launch_decode_prologue(pa, p->kv_dtype, stream);
  if (st) return st;
  if (split) {   // c128a: the block's 128 rows pooled over a cluster of CTAs
    st = launch_compress_split(pa.main, p->kv_dtype, b, nullptr, 0, stream, true);
    if (st) return st;
  }
  const int32_t* idx = nullptr;
  const int32_t* cnt = nullptr;
  if (!p->hca) {
    // 2. score the visible entries of every sequence (their pages through the block table)
    IndexArgs a{};
    a.q = raw_q ? x->q_I : qI; a.q_scales = raw_q ? x->kI_scales : qs; a.w = x->w;
    a.q_raw = raw_q ? x->q_I : nullptr;
    a.k = x->kI_pages; a.k_scales = x->kI_scales;
    a.q_pos = x->pos; a.T = 1; a.H = p->H_I; a.d = p->c_I; a.m = p->m; a.qk_dtype = p->idx_dtype;
    a.score_dtype = CSA_BF16; a.E_cap = p->max_pages * kPageEntries; a.E = std::max(E, 1);
    a.scores = d.scores; a.pdl = 1; a.all_visible = 0; a.dep_entry = -1;
    a.block_table = x->block_table; a.max_pages = p->max_pages; a.num_pages = p->num_pages;
    a.pos_input = 1;
    st = launch_index_scores_tc(a, b, stream);
    if (st == CSA_ERR_UNSUPPORTED && !raw_q) st = launch_index_scores_fp4_tc(a, b, stream);
    if (st) return st;
    // 3. top-k of each sequence's visible entries
    int32_t* io = x->idx_out ? x->idx_out : d.idx;
    int32_t* co = x->count_out ? x->count_out : d.count;
    st = topk_impl(d.scores, CSA_BF16, x->pos, p->m, b, 1, std::max(E, 1), p->k, io, co,
                   d.topk_ws, d.topk_ws_bytes, stream, true);
    if (st) return st;
    idx = io; cnt = co;
  }
  // 4. attention over the selection (or every visible entry) plus the window ring
  AttnArgs a{};
  a.q = x->q; a.kv = x->kv_pages; a.idx = idx; a.count = cnt; a.win = x->win; a.q_pos = x->pos;
  a.sink = x->sink; a.T = 1; a.H = p->H; a.d = p->c; a.n_w = p->n_w; a.m = p->m;
  a.k = p->hca ? 0 : p->k; a.E_cap = p->max_pages * kPageEntries; a.n = p->L_max;
  a.scale = p->scale; a.out = x->out; a.lse = x->lse; a.pdl = 1;
  a.d_rope_out = p->inv_rope ? p->d_rope : 0; a.theta = p->rope_theta;
  a.block_table = x->block_table; a.max_pages = p->max_pages; a.num_pages = p->num_pages;
  a.win_ring = p->n_w;
  st = launch_attn_tc(a, b, p->kv_dtype, d.attn_ws, d.attn_ws_bytes, stream);
  if (st == CSA_ERR_UNSUPPORTED) st = launch_attn_simt(a, b, p->kv_dtype, stream);
  return st;
}

// ---------------------------------------------------------------------------
// context-parallel decode (entries sharded over ranks)
// ---------------------------------------------------------------------------

csa_status csa_cp_candidates(const void* scores, int E_local, const int32_t* idx,
                             const int32_t* count, int b, int k, int entry_offset,
                             void* cand_scores, int32_t* cand_idx, cudaStream_t stream) {
  if (b < 0 || k < 1 || E_local < 0 || entry_offset < 0) return CSA_ERR_INVALID_ARG;
  if (b == 0) return CSA_OK;
  if (!scores || !idx || !count || !cand_scores || !cand_idx) return CSA_ERR_INVALID_ARG;
  return launch_cp_candidates(scores, E_local, idx, count, b, k, entry_offset, cand_scores, cand_idx,
                              stream);
}

size_t csa_cp_merge_workspace_size(int G, int b, int k) {
  if (G < 1 || b < 0 || k < 1) return 0;
  return cp_merge_bytes(G, b, k, topk_workspace_bytes(b, G * k, k, CSA_BF16)) + 256;
}

csa_status csa_cp_merge(const void* cand_scores, const int32_t* cand_idx, int G, int b, int k,
                        int32_t* idx, int32_t* count, int32_t* rows_idx, void* ws, size_t ws_bytes,
                        cudaStream_t stream) {
  if (G < 1 || b < 0 || k < 1 || (long long)G * k > (1 << 30)) return CSA_ERR_INVALID_ARG;
  if (b == 0) return CSA_OK;
  if (!cand_scores || !cand_idx || !idx || !count || !rows_idx || !ws) return CSA_ERR_INVALID_ARG;
  if (ws_bytes < csa_cp_merge_workspace_size(G, b, k) || (reinterpret_cast<uintptr_t>(ws) & 255))
    return CSA_ERR_INVALID_ARG;
  return launch_cp_merge(cand_scores, cand_idx, G, b, k, idx, count, rows_idx, ws, ws_bytes, stream);
}

csa_status csa_cp_pack_rows(const void* kv_local, int E_cap_local, int E_local, int entry_offset,
                            int c, int kv_dtype, const int32_t* idx, const int32_t* count, int b,
                            int k, void* rows, cudaStream_t stream) {
  if (b < 0 || k < 1 || c < 8 || E_local < 0 || E_local > E_cap_local || entry_offset < 0)
    return CSA_ERR_INVALID_ARG;
  if (kv_dtype != CSA_F32 && kv_dtype != CSA_BF16) return CSA_ERR_INVALID_ARG;
  const size_t row_bytes = (size_t)c * (kv_dtype == CSA_F32 ? 4 : 2);
  if (row_bytes % 16) return CSA_ERR_INVALID_ARG;
  if (b == 0) return CSA_OK;
  if (!kv_local || !idx || !count || !rows || !aligned16(kv_local) || !aligned16(rows))
    return CSA_ERR_INVALID_ARG;
  return launch_cp_pack(kv_local, E_cap_local, E_local, entry_offset, row_bytes, idx, count, b, k,
                        rows, stream);
}

// ---------------------------------------------------------------------------
// prefill
// ---------------------------------------------------------------------------

namespace {

struct PrefillWs {
  void* qI_codes; void* qI_scales; void* scores; int32_t* idx; int32_t* count; int32_t* qpos;
  void* attn_ws; size_t attn_ws_bytes; void* topk_ws; size_t topk_ws_bytes;
};

size_t prefill_layout(const csa_prefill_params* p, void* ws, size_t cap, PrefillWs* o) {
  Carve cv(ws, cap);
  PrefillWs d{};
  const size_t rows = (size_t)p->b * p->n;
  const int E = p->n / p->m;
  d.qpos = static_cast<int32_t*>(cv.take(rows * 4));
  if (p->idx_dtype != CSA_F32) {
    d.qI_codes = cv.take(rows * p->H_I * dtype_row_bytes(p->idx_dtype, p->c_I));
    d.qI_scales = cv.take(p->idx_dtype == CSA_FP8_E4M3 ? rows * p->H_I * 4
                                                        : rows * p->H_I * (p->c_I / 16));
  }
  d.scores = cv.take(rows * E * (p->score_dtype == CSA_F32 ? 4 : 2));
  d.idx = static_cast<int32_t*>(cv.take(rows * p->k * 4));
  d.count = static_cast<int32_t*>(cv.take(rows * 4));
  d.topk_ws_bytes = topk_workspace_bytes((int)rows, E, p->k, p->score_dtype);
  d.topk_ws = cv.take(d.topk_ws_bytes);
  csa_attn_params ap{p->H, p->c, p->n_w, p->scale, p->m, p->k, p->kv_dtype,
                     p->inv_rope ? p->d_rope : 0, p->rope_theta};
  d.attn_ws_bytes = csa_sparse_attn_workspace_size(&ap, p->b, p->n, E);
  d.attn_ws = cv.take(d.attn_ws_bytes);
  if (o) *o = d;
  return cv.ok ? align256(cv.used) : 0;
}

}  // namespace

int csa_prefill_launch_count(const csa_prefill_params* p) {
  if (!p || p->b <= 0) return 0;
  return 1 + 2 + (p->idx_dtype != CSA_F32 ? 1 : 0) + 1 + 1 +
         attn_launch_count(p->H, p->c, p->k, p->n_w, p->b, p->n, p->n / p->m, p->kv_dtype);
}

size_t csa_prefill_workspace_size(const csa_prefill_params* p) {
  if (!p) return 0;
  return prefill_layout(p, nullptr, 0, nullptr);
}

csa_status csa_prefill(const csa_prefill_params* p, const csa_prefill_tensors* x, void* ws,
                       size_t ws_bytes, cudaStream_t stream) {
  if (!p || !x) return CSA_ERR_INVALID_ARG;
  if (p->b < 0 || p->m < 1 || p->n < p->m || p->k < 1) return CSA_ERR_INVALID_ARG;
  if (p->b == 0) return CSA_OK;
  PrefillWs d{};
  const size_t need = prefill_layout(p, ws, ws_bytes, &d);
  if (need == 0 || !ws || ws_bytes < csa_prefill_workspace_size(p)) return CSA_ERR_INVALID_ARG;
  const int b = p->b, n = p->n, E = n / p->m;
  csa_status st = launch_iota_positions(d.qpos, b, n, stream);
  if (st) return st;
  csa_compress_params cp{p->m, 1, p->c, p->d_rope, p->rope_theta, p->eps, 1, p->kv_dtype,
                         p->kv_dtype};
  st = csa_compress(&cp, x->C_a, x->Z_a, x->B_a, x->C_b, x->Z_b, x->B_b, b, n, 0, E, E,
                    x->kv_cache, nullptr, stream);
  if (st) return st;
  csa_compress_params ci{p->m, 1, p->c_I, p->d_rope_I, p->rope_theta, p->eps, 1, p->kv_dtype,
                         p->idx_dtype};
  st = csa_compress(&ci, x->CI_a, x->ZI_a, x->BI_a, x->CI_b, x->ZI_b, x->BI_b, b, n, 0, E, E,
                    x->kI_cache, x->kI_scales, stream);
  if (st) return st;
  const void* qI = x->q_I;
  const void* qs = nullptr;
  if (p->idx_dtype != CSA_F32) {
    st = csa_quantize(p->kv_dtype, p->idx_dtype, x->q_I, b * n * p->H_I, p->c_I, d.qI_codes,
                      d.qI_scales, stream);
    if (st) return st;
    qI = d.qI_codes; qs = d.qI_scales;
  } else if (p->kv_dtype != CSA_F32) {
    return CSA_ERR_UNSUPPORTED;
  }
  csa_index_params ip{p->H_I, p->c_I, p->m, p->idx_dtype, p->score_dtype};
  st = index_scores_impl(&ip, qI, qs, x->w, x->kI_cache, x->kI_scales, d.qpos, b, n, E, E,
                         d.scores, stream, 1, 0, -1);
  if (st) return st;
  int32_t* io = x->idx_out ? x->idx_out : d.idx;
  int32_t* co = x->count_out ? x->count_out : d.count;
  st = topk_impl(d.scores, p->score_dtype, d.qpos, p->m, b, n, E, p->k, io, co, d.topk_ws,
                 d.topk_ws_bytes, stream, true);
  if (st) return st;
  csa_attn_params ap{p->H, p->c, p->n_w, p->scale, p->m, p->k, p->kv_dtype,
                     p->inv_rope ? p->d_rope : 0, p->rope_theta};
  return sparse_attn_impl(&ap, x->q, x->kv_cache, E, io, co, x->kv_win, n, d.qpos, x->sink, b, n,
                          x->out, x->lse, d.attn_ws, d.attn_ws_bytes, stream, 1);
}

}  // extern "C"
