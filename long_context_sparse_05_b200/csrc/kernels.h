// Internal launch interface between the C ABI (api.cu) and the kernel files.
#pragma once

#include "csa.h"

namespace csa {

constexpr int kMaxRopePairs = 64;   // rotary pairs with a host-built frequency table

struct CompressArgs {
  const void* C_a; const void* Z_a; const float* B_a;
  const void* C_b; const void* Z_b; const float* B_b;
  int n, m, overlap, c, d_rope, apply_norm, out_dtype, entry_begin, out_E;
  double theta;
  float eps;
  void* out;
  void* out_scales;
  double inv_freq[kMaxRopePairs];   // theta^(-2j/d_rope) in float64, filled by the launcher
  // Paged state-cache mode (ring != 0): raw row u of sequence s is slot u % ring of the
  // per-sequence ring buffers C_* / Z_* ([b][ring][c]), except the newest token's row
  // (u = pos[s]), which comes from new_* ([b][c]); entry i is written at physical row
  // block_table[s][i / kPageEntries] * kPageEntries + i % kPageEntries of out / out_scales.
  int ring;
  const int32_t* pos;
  const void *new_C_a, *new_Z_a, *new_C_b, *new_Z_b;
  const int32_t* block_table;
  int max_pages;
  // entry i goes to row i - out_off of its sequence (a shard of the entries); 0: row i
  int out_off;
  int num_pages;   // paged: pages in the pool (an entry whose page is outside it is skipped)
};

constexpr int kPageEntries = CSA_PAGE_ENTRIES;   // compressed entries per page of the paged caches

struct PrologueArgs {
  CompressArgs main, index;        // index used when nbranch == 2
  int nbranch, b, t;
  int32_t* qpos;                   // [b] <- t (or <- pos[s] in paged mode)
  const void* q_in; int q_rows, q_d, q_dtype; uint8_t* q_codes; void* q_scales;
  // paged mode: the step appends the newest token's raw rows to the state rings
  // (ring slot pos[s] % main.ring; window ring slot pos[s] % win_ring) and compresses
  // an entry only for sequences whose block the token completes
  int paged;
  void* win; const void* new_win; int win_ring;
  // paged c128a: the entries are compressed by the cluster-split kernel launched next
  int skip_compress;
};

struct IndexArgs {
  const void* q; const void* q_scales; const float* w;
  const void* k; const void* k_scales; const int32_t* q_pos;
  int T, H, d, m, qk_dtype, score_dtype, E_cap, E;
  void* scores;
  int pdl;            // launch as a programmatic dependent of the preceding kernel
  int all_visible;    // every query sees all E entries (decode at t = L-1): q_pos is not read
  int dep_entry;      // first entry the preceding kernel writes (tiles before it may be
                      // fetched before waiting on that kernel); -1: all depend
  // paged keys (one query per sequence): stage js of sequence s is page
  // block_table[s][js] of kPageEntries rows; pages outside [0, num_pages) read as page 0
  const int32_t* block_table;
  int max_pages, num_pages;
  // q_pos is an input of the call (not written by the preceding kernel): it is read
  // before waiting, and only the page of the entry the token completes, (t+1)/m - 1 when
  // (t+1) % m == 0, is written by the preceding kernel
  int pos_input;
  // FP8 tensor-core path, one query per sequence: the index queries as bf16 [rows][128],
  // quantised inside the kernel (q and q_scales unused).  An input of the call, so the
  // key stages the preceding kernel does not write are scored without waiting for it.
  const void* q_raw;
};

struct AttnArgs {
  const void* q; const void* kv; const int32_t* idx; const int32_t* count;
  const void* win; const int32_t* q_pos; const float* sink;
  int T, H, d, n_w, m, k, E_cap, n;
  float scale;
  void* out; float* lse;
  int pdl;            // launch as a programmatic dependent of the preceding kernel
  int d_rope_out;     // inverse RoPE on the last d_rope_out output dims (0: none)
  double theta;       // its RoPE base
  // paged entries: entry e of sequence s is row e % kPageEntries of page
  // block_table[s][e / kPageEntries] (pages outside [0, num_pages) are skipped);
  // win_ring > 0: window token u of sequence s is slot u % win_ring of win ([b][win_ring][d])
  const int32_t* block_table;
  int max_pages, num_pages, win_ring;
};

constexpr int kMaxOutRopePairs = 32;   // rotary pairs of the output with a host-built table

csa_status launch_compress(const CompressArgs& a, int in_dtype, int b, int entry_count,
                           cudaStream_t st);
csa_status launch_decode_prologue(PrologueArgs& a, int in_dtype, cudaStream_t st);
// One long non-overlapped block (c128a) per sequence over a cluster of CTAs.  With a.ring
// (paged state) it compresses only for sequences whose new token completes a block and
// waits for the preceding kernel at its end, so that its completion implies that kernel's.
bool compress_split_supported(const CompressArgs& a, int in_dtype);
csa_status launch_compress_split(CompressArgs& a, int in_dtype, int b, int32_t* qpos, int t,
                                 cudaStream_t st, bool pdl);
csa_status launch_quantize(int in_dtype, int out_dtype, const void* x, int rows, int d,
                           void* codes, void* scales, cudaStream_t st);
// Context-parallel decode (cp.cu): a rank's top-k as (score, global entry) candidates; the
// top-k of every rank's candidates (workspace of cp_merge_bytes); the selected rows a rank
// holds packed into their selection slots.
csa_status launch_cp_candidates(const void* scores, int E_local, const int32_t* idx,
                                const int32_t* count, int b, int k, int offset, void* cand_s,
                                int32_t* cand_i, cudaStream_t st);
size_t cp_merge_bytes(int G, int b, int k, size_t topk_ws);
csa_status launch_cp_merge(const void* cand_s, const int32_t* cand_i, int G, int b, int k,
                           int32_t* idx, int32_t* count, int32_t* rows_idx, void* ws,
                           size_t ws_bytes, cudaStream_t st);
csa_status launch_cp_pack(const void* kv, int E_cap_local, int E_local, int offset, size_t row_bytes,
                          const int32_t* idx, const int32_t* count, int b, int k, void* rows,
                          cudaStream_t st);
csa_status launch_topk_search(const void* scores, int score_dtype, const int32_t* q_pos, int m,
                              int rows, int E, int k, int32_t* idx, int32_t* count, void* ws,
                              size_t ws_bytes, cudaStream_t st, bool pdl = false);
size_t topk_workspace_bytes(int rows, int E, int k, int score_dtype);
csa_status launch_topk(const void* scores, int score_dtype, const int32_t* q_pos, int m, int rows,
                       int E, int k, int32_t* idx, int32_t* count, cudaStream_t st);

// CUDA-core kernels: any shape.
csa_status launch_index_scores_simt(const IndexArgs& a, int b, cudaStream_t st);
csa_status launch_attn_simt(const AttnArgs& a, int b, int dtype, cudaStream_t st);

// Tensor-core (tcgen05) kernels: return CSA_ERR_UNSUPPORTED for shapes they do not cover.
csa_status launch_index_scores_tc(const IndexArgs& a, int b, cudaStream_t st);
csa_status launch_index_scores_fp4_tc(const IndexArgs& a, int b, cudaStream_t st);
csa_status launch_attn_tc(const AttnArgs& a, int b, int dtype, void* ws, size_t ws_bytes,
                          cudaStream_t st);
size_t attn_tc_workspace_bytes(int H, int d, int k, int n_w, int b, int T, int E_cap, int dtype);
bool attn_tc_supported(int H, int d, int dtype);
int attn_launch_count(int H, int d, int k, int n_w, int b, int T, int E_cap, int dtype);

// Hierarchical indexer: the candidate pool of every query row gathered into a key set of
// its own (workspace of pool_gather_bytes()), and top-k positions mapped back to entries.
int pool_row_bytes(int fmt, int d);
size_t pool_gather_bytes(int fmt, int rows, int P, int d, size_t* off_scales, size_t* off_pool,
                         size_t* off_pos);
csa_status launch_pool_gather(int fmt, const int32_t* pool, const int32_t* pool_count,
                              const int32_t* q_pos, const void* k, const void* k_scales, int rows,
                              int T, int P, int E_cap, int E, int m, int d, void* ws,
                              cudaStream_t st, bool pdl);
csa_status launch_pool_map(const void* ws, int fmt, int rows, int P, int d, int k, int32_t* idx,
                           const int32_t* count, cudaStream_t st, bool pdl);

// Grouped output projection (tcgen05 bf16 GEMM per head group).
bool out_proj_supported(int H, int d, int g, int d_g);
size_t out_proj_workspace_bytes(int T, int H, int d, int g, int d_g);
int out_proj_launch_count(int T, int H, int d, int g, int d_g);
csa_status launch_out_proj(const void* o, const void* W, int T, int H, int d, int g, int d_g,
                           void* y, void* ws, size_t ws_bytes, cudaStream_t st, bool pdl);

// Small helpers.
csa_status launch_fill_i32(int32_t* p, int count, int value, cudaStream_t st);
csa_status launch_iota_positions(int32_t* p, int b, int n, cudaStream_t st);

}  // namespace csa
