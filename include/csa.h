/*
 * csa.h -- C ABI of the Compressed Sparse Attention (CSA) / Heavily Compressed
 * Attention (HCA) hot path on NVIDIA B200 (sm_100a).
 *
 * The method (DeepSeek-V4 attention, as described on the pages "DeepSeek V4
 * 结构速览", "DeepSeek Technical Reports", "DeepSeek-V4技术报告解读" and
 * "DeepSeek-V4 技术解读") has four stages, each one entry point here:
 *
 *   csa_compress      KV compressor: per-channel softmax pooling of 2m raw rows
 *                     at stride m (c4a) or m rows (c128a), RMSNorm, partial
 *                     RoPE, optional FP8 / NVFP4 quantisation of index keys.
 *   csa_index_scores  lightning indexer I[t,s] = sum_j w[t,j] ReLU(q[t,j].k[s]).
 *   csa_topk          causal top-k of the scores of each query.
 *   csa_sparse_attn   shared-latent MQA (K = V) with a per-head sink over the
 *                     selected entries plus a raw sliding window; dense over all
 *                     visible entries when no index list is given (HCA).
 *
 * plus csa_quantize (the index-path quantiser on its own) and the fused
 * drivers csa_decode and csa_prefill that chain the stages on one stream.
 *
 * Conventions for every call:
 *  - Pointers named as tensors are DEVICE pointers, allocated and owned by the
 *    caller; no call allocates device memory.  The library keeps a little state
 *    of its own for the life of the process: one device error word per device
 *    (csa_device_error), cached device properties (SM count, which cluster
 *    sizes fit) and the driver's tensor-map entry point, and the fixed scratch
 *    array of csa_sparse_attn_noalloc.  Nothing of one call's data is kept for
 *    the next.
 *  - Every call is asynchronous on the caller's stream; results are ready when
 *    the stream reaches them.  No call synchronises the device.
 *  - Layouts are row-major, batch outermost, last dimension contiguous.  Base
 *    pointers must be 16-byte aligned.
 *  - Indices are int32; -1 pads unused top-k slots.
 *  - Argument errors are detected on the host before any launch and returned
 *    as CSA_ERR_INVALID_ARG (nothing is launched); a launch failure reported
 *    by the CUDA runtime is CSA_ERR_CUDA.  No call aborts the process.
 *
 * Storage types (csa_dtype):
 *  - CSA_F32, CSA_BF16: plain element arrays.
 *  - CSA_FP8_E4M3: one byte per element (OCP E4M3FN), plus one float32 scale
 *    per row: value = decode(code) * scale, scale = amax(row) / 448.
 *  - CSA_NVFP4: two E2M1 codes per byte (element 2j in bits 0-3, 2j+1 in bits
 *    4-7), plus one UE4M3 scale byte per 16 consecutive elements:
 *    value = decode(code) * decode(scale), scale = e4m3(amax(block) / 6).
 *    Query scales (and csa_quantize output) are row-major [rows][d/16].  Key
 *    caches (csa_compress output, k_I of the indexer, kI_scales of the fused
 *    calls) keep their scales TILED, in the order the block-scaled tensor-core
 *    MMA reads them: a sequence of E_cap entries owns ceil(E_cap/128) tiles of
 *    128 * d/16 bytes (d a multiple of 64); inside a tile, the scale of block j
 *    of entry r (0..127) is at byte (j/4)*512 + (r%32)*16 + (r/32)*4 + j%4.
 *    The buffer is therefore [b][ceil(E_cap/128)*128][d/16] bytes.
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1,   /* bad shape, pointer, alignment or type; nothing launched */
  CSA_ERR_UNSUPPORTED = 2,   /* a valid combination this build has no kernel for */
  CSA_ERR_CUDA = 3,          /* the CUDA runtime reported a launch error */
  CSA_ERR_TIMEOUT = 4        /* a bounded device-side wait gave up */
} csa_status;

typedef enum {
  CSA_F32 = 0,
  CSA_BF16 = 1,
  CSA_FP8_E4M3 = 2,
  CSA_NVFP4 = 3
} csa_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* csa_status_string(csa_status s);

/* Library version as major * 10000 + minor * 100 + patch. */
int csa_version(void);

/*
 * Synchronises `stream`, then reads and clears the library's device error
 * word: CSA_OK, or CSA_ERR_TIMEOUT when a bounded device-side wait of a
 * tensor-core kernel gave up since the last call (the outputs of that launch
 * are then NaN, never silently wrong).  The word is one int per device held
 * by the library for its lifetime.
 */
int csa_device_error(cudaStream_t stream);

/*
 * Failure-detection self-test: launches one thread that waits, with a bound of
 * limit_us microseconds (1 .. 100000), on a barrier nothing ever signals.  The
 * wait gives up and sets the device error word, so a following
 * csa_device_error(stream) returns CSA_ERR_TIMEOUT; the context stays usable.
 */
csa_status csa_selftest_bounded_wait(int limit_us, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Stage 1: KV compressor                                                    */
/* ------------------------------------------------------------------------ */

/*
 * Source: "DeepSeek V4 结构速览", section "C4A Compressor" (per-channel softmax
 * over the stacked logits of the previous and the current block plus a
 * positional bias, weighted sum of the stacked contents, RMSNorm, RoPE; block
 * 0 pads its previous half with zero content and -inf logits); section
 * "核心设计" item 1 (c4a: 8 rows at stride 4; c128a: 128 rows at stride 128);
 * "DeepSeek-V4技术报告解读", section "Compressed Sparse Attention (CSA)"
 * (compression formula with bias B).
 *
 * Entry i of sequence s, channel ch (R = 2m rows with overlap, m without):
 *   rows r <  m (overlap only): logit Z_b[s][m(i-1)+r][ch] + B_b[r][ch],
 *                               content C_b[s][m(i-1)+r][ch]  (i = 0: -inf, 0)
 *   rows r >= m (or all rows without overlap):
 *                               logit Z_a[s][mi+r'][ch] + B_a[r'][ch],
 *                               content C_a[s][mi+r'][ch]     (r' = r - m or r)
 *   x[ch]  = sum_r softmax_r(logit)[r] * content[r]            (float32)
 *   x      = x / sqrt(mean(x^2) + eps)                          (if apply_norm)
 *   pairs (x[c-d_rope+2j], x[c-d_rope+2j+1]) rotated by p * theta^(-2j/d_rope),
 *   p = m * i, the angle formed in float64.
 */
typedef struct {
  int m;              /* compression rate (>= 1) */
  int overlap;        /* 1: previous block from the b-branch joins; 0: current block only */
  int c;              /* channels per entry; multiple of 8 (of 64 for NVFP4 output) */
  int d_rope;         /* rotary dims at the end of each entry; even, <= c; 0 = none */
  double rope_theta;  /* RoPE base (10000) */
  float eps;          /* RMSNorm epsilon (1e-6) */
  int apply_norm;     /* 1: RMSNorm with unit gain; 0: skip (identity checks) */
  int in_dtype;       /* CSA_F32 or CSA_BF16: type of C_* and Z_* */
  int out_dtype;      /* CSA_F32, CSA_BF16, CSA_FP8_E4M3 or CSA_NVFP4 */
  int out_entry_offset; /* entry i is written at row i - out_entry_offset of each sequence's
                           out (a shard of the entries, as in context-parallel decode); 0 for
                           a whole cache; a multiple of 128 for NVFP4 output */
} csa_compress_params;

/*
 * Compresses entries [entry_begin, entry_begin + entry_count) of each of the b
 * sequences.
 *   C_a, Z_a   [b][n][c] (in_dtype)     current-block branch
 *   C_b, Z_b   [b][n][c] (in_dtype)     previous-block branch; NULL when !overlap
 *   B_a, B_b   [m][c] float32           positional biases; B_b NULL when !overlap
 *   n          tokens per sequence; requires m * (entry_begin + entry_count) <= n
 *   out        [b][out_entries_per_seq][row] with row = c elements (F32/BF16),
 *              c bytes (FP8) or c/2 bytes (NVFP4); entry i of sequence s is
 *              written at row s * out_entries_per_seq + i (caches are updated
 *              in place, other rows untouched)
 *   out_scales FP8: float32 [b][out_entries_per_seq]; NVFP4: the tiled key-scale
 *              layout (above), [b][ceil(out_entries_per_seq/128)*128][c/16] bytes,
 *              c a multiple of 64; NULL for F32/BF16
 */
csa_status csa_compress(const csa_compress_params* p,
                        const void* C_a, const void* Z_a, const float* B_a,
                        const void* C_b, const void* Z_b, const float* B_b,
                        int b, int n, int entry_begin, int entry_count, int out_entries_per_seq,
                        void* out, void* out_scales, cudaStream_t stream);

/*
 * Index-path quantiser on its own ("DeepSeek V4 结构速览", section "Lightning
 * Indexer": the QK path of the indexer runs in FP4 end to end).  Quantises
 * `rows` rows of `d` elements of x (CSA_F32 or CSA_BF16) to out_dtype
 * CSA_FP8_E4M3 (codes [rows][d], scales float32 [rows]) or CSA_NVFP4 (codes
 * [rows][d/2], scales uint8 [rows][d/16]).  d must be a multiple of 16.  The
 * divisions are IEEE float32 and the conversions round to nearest even with
 * saturation, so results are bit-identical to any exact implementation.
 */
csa_status csa_quantize(int in_dtype, int out_dtype, const void* x, int rows, int d,
                        void* codes, void* scales, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Stage 2: lightning indexer                                                */
/* ------------------------------------------------------------------------ */

/*
 * Source: "DeepSeek Technical Reports", section DSA (I[t,s] = sum_j w[t,j] *
 * ReLU(q_I[t,j] . k_I[s])); "DeepSeek V4 结构速览", section "Lightning
 * Indexer" (FP4 QK path, ReLU, per-head weighted sum, scores kept in BF16,
 * causal range).  With quantised operands, q and k are their dequantised
 * values.  Entry s is visible to query position t iff m(s+1)-1 <= t; the
 * scores of invisible entries are -inf.
 */
typedef struct {
  int H_I;          /* indexer heads */
  int d_I;          /* index-key dim; multiple of 16 */
  int m;            /* compression rate (visibility rule) */
  int qk_dtype;     /* CSA_F32, CSA_FP8_E4M3 or CSA_NVFP4 (q_I and k_I alike) */
  int score_dtype;  /* CSA_F32 or CSA_BF16 */
} csa_index_params;

/*
 *   q_I       [b][T][H_I][row]  codes (row as in csa_compress for qk_dtype)
 *   q_scales  FP8: float32 [b][T][H_I]; NVFP4: uint8 [b][T][H_I][d_I/16]; F32: NULL
 *   w         [b][T][H_I] float32 head weights
 *   k_I       [b][E_cap][row] codes;  k_scales FP8: float32 [b][E_cap]; NVFP4: the
 *             tiled key-scale layout, [b][ceil(E_cap/128)*128][d_I/16] bytes (d_I a
 *             multiple of 64)
 *   q_pos     [b][T] int32 position t of each query
 *   scores    [b][T][E] (score_dtype), E <= E_cap entries scored per query
 *
 * The tensor-core shapes (H_I = 64, d_I = 128, FP8 or NVFP4) read their operands
 * with TMA: every pointer must be 16-byte aligned and, for FP8, E_cap a multiple
 * of 4 (whole 16-byte runs of key scales).  Otherwise the call returns
 * CSA_ERR_INVALID_ARG; it never falls back to a slower kernel for these shapes.
 */
csa_status csa_index_scores(const csa_index_params* p, const void* q_I, const void* q_scales,
                            const float* w, const void* k_I, const void* k_scales,
                            const int32_t* q_pos, int b, int T, int E_cap, int E,
                            void* scores, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Stage 3: causal top-k                                                     */
/* ------------------------------------------------------------------------ */

/*
 * Source: "DeepSeek Technical Reports", section DSA (Top-k(I[t,:]));
 * "DeepSeek V4 结构速览", sections "核心设计" item 2 and "Lightning
 * Indexer" (k = 512 / 1024 among causally visible entries).
 * For each query: the k largest scores among entries s < E(t) =
 * min(E, floor((t+1)/m)); equal scores go to the lower s; if E(t) <= k all
 * visible entries are kept.  idx [b][T][k] lists the kept entries in
 * ascending order, padded with -1; count [b][T] holds how many.  The result
 * is exact (a search over the stored score bits; scores must not be NaN).
 * Few long rows are each spread over a thread-block cluster of up to 16 CTAs
 * (up to 16 x 16384 entries a row); only rows beyond what a cluster holds
 * need scratch.
 *   scores  [b][T][E] (CSA_F32 or CSA_BF16)
 *   ws      device scratch of csa_topk_workspace_size() bytes: rows too long for
 *           one cluster keep a top-k per 16384-entry chunk there first (NULL
 *           with ws_bytes 0 when the size is 0).  The size depends on the
 *           current device (its SM count) as well as on the shape.
 */
csa_status csa_topk(const void* scores, int score_dtype, const int32_t* q_pos, int m, int b, int T,
                    int E, int k, int32_t* idx, int32_t* count, void* ws, size_t ws_bytes,
                    cudaStream_t stream);
size_t csa_topk_workspace_size(int score_dtype, int b, int T, int E, int k);

/*
 * Hierarchical sparse indexer ("DeepSeek Technical Reports", section CSA2,
 * Hierarchical Sparse Indexer): a Reindex layer scores, with its own index
 * query, only a candidate pool that an earlier full indexer produced (for
 * instance a top-P with P > k of the first layer), and keeps the k best of it.
 * For query row r: the candidates are pool[r][j], j < pool_count[r], that are
 * visible to q_pos[r] (entry < min(E, floor((t+1)/m))); each is scored exactly
 * as csa_index_scores scores it (BF16 scores); the k highest are kept, equal
 * scores going to the lower entry.  idx [b][T][k] lists the kept entries in
 * the pool's order, -1 padded; count [b][T] holds how many.
 *   pool        [b][T][P] int32 entry ids, ascending, -1 padded (a csa_topk
 *               output row is such a pool); idx is then ascending too
 *   pool_count  [b][T] int32 valid pool entries of each row
 *   q_I, q_scales, w, k_I, k_scales, q_pos, E_cap, E: as in csa_index_scores
 *   ws          device scratch of csa_pool_topk_workspace_size() bytes: each row's
 *               pool is gathered into a key set of its own (the tensor-core
 *               indexer then scores it as a sequence of P entries)
 */
size_t csa_pool_topk_workspace_size(const csa_index_params* p, int b, int T, int P, int k);
csa_status csa_pool_topk(const csa_index_params* p, const void* q_I, const void* q_scales,
                         const float* w, const void* k_I, const void* k_scales,
                         const int32_t* q_pos, int b, int T, int E_cap, int E,
                         const int32_t* pool, const int32_t* pool_count, int P, int k,
                         int32_t* idx, int32_t* count, void* ws, size_t ws_bytes,
                         cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Stage 4: shared-latent MQA over selected entries + window, with sink      */
/* ------------------------------------------------------------------------ */

/*
 * Source: "DeepSeek Technical Reports", section DSA (u_t = Attn(h_t,
 * {c_s | I[t,s] in Top-k})) and section CSA (window of n_w = 128 uncompressed
 * tokens); "DeepSeek V4 结构速览", sections "CSA（c4a 路线）" (the window
 * rows are concatenated with the selected entries; one 512-dim latent is
 * both K and V for 64 heads) and "HCA（c128a 路线）" (dense over all entries,
 * attention sink); "DeepSeek-V4 技术解读", section 2.1 (shared KV MQA).
 *
 * For query t of sequence s and head h, over the rows
 *   S = { kv_comp[s][idx[j]] : j < count }  (or all j < E(t) when idx == NULL)
 *     + { kv_win[s][u] : max(0, t-n_w+1) <= u <= t }
 *   l_r = scale * q[h] . row_r
 *   out[h] = sum_r e^{l_r} row_r / (e^{sink[h]} + sum_r e^{l_r})
 *   lse[h] = log(e^{sink[h]} + sum_r e^{l_r})
 */
typedef struct {
  int H;          /* query heads */
  int d;          /* head dim = latent dim */
  int n_w;        /* window length (raw tokens, inclusive of t) */
  float scale;    /* logit scale */
  int m;          /* compression rate (dense mode: E(t) = floor((t+1)/m)) */
  int k;          /* idx row length (ignored when idx == NULL) */
  int dtype;      /* CSA_F32 or CSA_BF16: q, kv_comp, kv_win and out */
  int d_rope_out; /* inverse RoPE on the last d_rope_out dims of every head's output, at
                     the query's position (even, <= d; 0 = none; the tensor-core path takes
                     up to 64): "DeepSeek V4 结构速览", sections "CSA（c4a 路线）" and
                     "HCA（c128a 路线）".  Each interleaved pair (o[d-r+2j], o[d-r+2j+1]) is
                     rotated by -t * rope_theta^(-2j/d_rope_out), the angle formed in
                     float64, undoing the rotation RoPE gives position t. */
  double rope_theta;
} csa_attn_params;

/*
 *   q        [b][T][H][d]
 *   kv_comp  [b][E_cap][d] compressed entries
 *   idx      [b][T][k] int32 selected entries (ascending, -1 padded) or NULL
 *   count    [b][T] int32 valid entries of each idx row (NULL iff idx NULL)
 *   kv_win   [b][n][d] raw rows for the window (n tokens per sequence)
 *   q_pos    [b][T] int32 positions; requires q_pos < n
 *   sink     [H] float32
 *   out      [b][T][H][d];  lse [b][T][H] float32 or NULL
 *   ws       device scratch of at least csa_sparse_attn_workspace_size() bytes
 */
csa_status csa_sparse_attn(const csa_attn_params* p, const void* q, const void* kv_comp, int E_cap,
                           const int32_t* idx, const int32_t* count, const void* kv_win, int n,
                           const int32_t* q_pos, const float* sink, int b, int T, void* out,
                           float* lse, void* ws, size_t ws_bytes, cudaStream_t stream);

size_t csa_sparse_attn_workspace_size(const csa_attn_params* p, int b, int T, int E_cap);

/*
 * csa_sparse_attn for callers that cannot allocate device memory.  Some
 * callers may not call cudaMalloc at all: a plugin running inside a host
 * framework that owns every byte of device memory and hands out no allocator,
 * or a latency-critical decode loop that must never hit cudaMalloc, which can
 * synchronise the device and has unbounded latency.  This entry point takes
 * the same arguments as csa_sparse_attn minus the workspace and needs no
 * allocation: the split partials live in one fixed scratch array inside the
 * library (a file-scope device array of CSA_NOALLOC_SCRATCH_BYTES), which
 * every GPU that loads the library holds until the process exits.  The
 * method on the pages has no counterpart of this; it only changes where the
 * scratch lives.
 *
 *  - Every call looks up the array's device address in the current device's
 *    context (a runtime query, no allocation), so a context recreated after
 *    cudaDeviceReset is served too.  The first call on a device may load the
 *    library's module there: make it before any stream capture.
 *  - A problem whose workspace (csa_sparse_attn_workspace_size) exceeds
 *    CSA_NOALLOC_SCRATCH_BYTES is rejected with CSA_ERR_INVALID_ARG and
 *    nothing is launched.
 *  - Every call on a device shares the one array, and the array keeps the
 *    last call's contents: calls that may overlap on the GPU (different
 *    streams, or several host threads) race on it and must be serialised by
 *    the caller.  The kernels write every scratch word before reading it, so
 *    nothing needs clearing between calls.
 *  - The call allocates nothing: no cudaMalloc, no cudaFree, no allocating
 *    library routine.
 */
#define CSA_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
csa_status csa_sparse_attn_noalloc(const csa_attn_params* p, const void* q, const void* kv_comp,
                                   int E_cap, const int32_t* idx, const int32_t* count,
                                   const void* kv_win, int n, const int32_t* q_pos,
                                   const float* sink, int b, int T, void* out, float* lse,
                                   cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Output epilogue: grouped output projection                                */
/* ------------------------------------------------------------------------ */

/*
 * Source: "DeepSeek-V4 技术解读", section 2.1 (分组输出投影: the attention output is
 * split into g groups, each projected on its own, which cuts the projection's work
 * g-fold).  Group i holds heads [i*H/g, (i+1)*H/g), concatenated into K = H/g * d
 * values; y[t][i*d_g + n] = sum_k o[t][i*K + k] * W[i][n][k] (float32 accumulation,
 * bf16 result).
 *   o   [T][H][d] bf16 (the attention output, inverse RoPE applied if wanted)
 *   W   [g][d_g][K] bf16 (row n of group i's projection, K contiguous)
 *   y   [T][g * d_g] bf16
 *   ws  device scratch of csa_out_proj_workspace_size() bytes (non-zero only when a
 *       few tokens leave SMs idle and the K dimension is split; NULL when 0)
 * Requires H % g == 0, K a multiple of 64, d_g a multiple of 256, 16-byte aligned
 * pointers; otherwise CSA_ERR_INVALID_ARG.
 */
size_t csa_out_proj_workspace_size(int T, int H, int d, int g, int d_g);
csa_status csa_out_proj(const void* o, const void* W, int T, int H, int d, int g, int d_g,
                        void* y, void* ws, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------ */
/* Fused drivers                                                             */
/* ------------------------------------------------------------------------ */

/*
 * One decode step for b sequences of L tokens each (the operator graph of
 * "DeepSeek V4 结构速览", section "CSA（c4a 路线）"; HCA per section
 * "HCA（c128a 路线）").  The new token is t = L-1; it completes entry E-1
 * (E = L/m, L a multiple of m), which the step compresses from the raw rows
 * of its block (and of the previous block for c4a) into the caches in
 * place.  CSA then quantises q_I, scores all E entries, selects k and attends
 * over them plus the window; HCA attends over all E entries plus the window.
 */
/*
 * Operating modes of a CSA decode layer ("DeepSeek Technical Reports", section
 * CSA2: cross-layer KV and index reuse):
 *   CSA_MODE_FULL     the indexer scores all E entries and top-k selects k;
 *   CSA_MODE_REUSE    no scoring: the selection of an earlier layer (idx_in,
 *                     count_in) is attended with this layer's q;
 *   CSA_MODE_REINDEX  the hierarchical indexer: only the candidate pool (pool,
 *                     pool_count, P entries a row) is scored with this layer's
 *                     q_I, and its k best are attended (csa_pool_topk).
 * The step compresses the new entry of both caches in every mode.
 */
typedef enum { CSA_MODE_FULL = 0, CSA_MODE_REUSE = 1, CSA_MODE_REINDEX = 2 } csa_decode_mode;

typedef struct {
  int b, L, m, c, H;       /* sequences, context, compression rate, latent dim, heads */
  int c_I, H_I;            /* index-key dim and indexer heads (CSA only) */
  int d_rope, d_rope_I;    /* rotary dims of latent entries and of index keys */
  double rope_theta;
  float eps;
  int k, n_w;              /* top-k (CSA) and window */
  float scale;             /* attention logit scale */
  int kv_dtype;            /* CSA_BF16 or CSA_F32 */
  int idx_dtype;           /* CSA_FP8_E4M3, CSA_NVFP4 or CSA_F32 (CSA only) */
  int hca;                 /* 1: HCA (no indexer, no previous block, dense attention) */
  int E_cap;               /* entries each cache row-block holds (>= L/m) */
  int mode;                /* csa_decode_mode (CSA only; HCA takes CSA_MODE_FULL) */
  int P;                   /* CSA_MODE_REINDEX: pool row length */
  int inv_rope;            /* 1: inverse RoPE on the last d_rope output dims (see csa_attn_params) */
} csa_decode_params;

typedef struct {
  const void *C_a, *Z_a, *C_b, *Z_b;   /* [b][L][c]; C_b/Z_b NULL for HCA */
  const float *B_a, *B_b;              /* [m][c] */
  const void *CI_a, *ZI_a, *CI_b, *ZI_b; /* [b][L][c_I] (CSA) */
  const float *BI_a, *BI_b;            /* [m][c_I] (CSA) */
  void* kv_cache;                      /* [b][E_cap][c] kv_dtype; entry E-1 written */
  void* kI_cache;                      /* [b][E_cap][row] idx_dtype codes; entry E-1 written */
  void* kI_scales;                     /* FP8: float32 [b][E_cap]; NVFP4: tiled, see above */
  const void* kv_win;                  /* [b][L][c] raw window rows */
  const void* q;                       /* [b][H][c] */
  const void* q_I;                     /* [b][H_I][c_I] unquantised (kv_dtype) */
  const float* w;                      /* [b][H_I] */
  const float* sink;                   /* [H] */
  void* out;                           /* [b][H][c] kv_dtype */
  float* lse;                          /* [b][H] or NULL */
  int32_t* idx_out;                    /* [b][k] selected entries or NULL (CSA; not written
                                          in CSA_MODE_REUSE) */
  int32_t* count_out;                  /* [b] or NULL (CSA) */
  const int32_t* idx_in;               /* CSA_MODE_REUSE: [b][k] entries to attend, -1 padded */
  const int32_t* count_in;             /* CSA_MODE_REUSE: [b] */
  const int32_t* pool;                 /* CSA_MODE_REINDEX: [b][P] candidate entries */
  const int32_t* pool_count;           /* CSA_MODE_REINDEX: [b] */
} csa_decode_tensors;

csa_status csa_decode(const csa_decode_params* p, const csa_decode_tensors* x, void* ws,
                      size_t ws_bytes, cudaStream_t stream);
/* Device workspace csa_decode needs (bytes); host only. */
size_t csa_decode_workspace_size(const csa_decode_params* p);
/* Number of kernel launches one csa_decode call makes with these parameters; host only. */
int csa_decode_launch_count(const csa_decode_params* p);

/*
 * Paged decode step for b sequences at any positions: the heterogeneous KV cache of
 * "DeepSeek-V4技术报告解读", section 3.2 (异构 KV 缓存管理): a classical cache of
 * fixed-size blocks of compressed entries per request, and a fixed-size state per
 * request holding the sliding window and the raw rows not yet compressed.
 *
 * Classical cache: pages of CSA_PAGE_ENTRIES compressed entries (latent rows, index-key
 * codes and scales share the page ids).  Entry e of sequence s lives in page
 * block_table[s][e / CSA_PAGE_ENTRIES], row e % CSA_PAGE_ENTRIES:
 *   kv_pages   [num_pages][CSA_PAGE_ENTRIES][c] kv_dtype
 *   kI_pages   [num_pages][CSA_PAGE_ENTRIES][row] idx_dtype codes
 *   kI_scales  FP8: float32 [num_pages][CSA_PAGE_ENTRIES]; NVFP4: the tiled key-scale
 *              layout over num_pages * CSA_PAGE_ENTRIES entries (two tiles per page)
 * (The pages speak of blocks covering 128 raw tokens; here a block is the
 * tensor-core indexer's 256-entry stage, so that a stage is one page.)
 * State (per sequence, fixed size, updated in place by every step):
 *   win                    [b][n_w][c]: raw window row of token u at slot u % n_w
 *   tail_C_a, tail_Z_a, ... [b][R][c]: raw rows of token u at slot u % R, R = 2m for
 *                          c4a (the previous block joins), m for c128a; tail_CI_* the
 *                          index branch [b][2m][c_I]
 * Step inputs: pos[s] = t, the new token's position (any t, sequences may differ);
 * the new token's raw rows new_* ([b][c] or [b][c_I]) and its window row new_win;
 * q, q_I, w, sink as in csa_decode.  The step appends the new rows to the state, and
 * for every sequence whose block the token completes ((t+1) % m == 0) compresses entry
 * (t+1)/m - 1 into its page (the page must be in the block table).  It then scores
 * the E(t) = floor((t+1)/m) visible entries, selects k (CSA) or takes all (HCA), and
 * attends over them plus the window max(0, t-n_w+1)..t.  L_max bounds t + 1 over the
 * batch (entries scored per sequence: floor(L_max / m)).  Page ids outside
 * [0, num_pages) are read as page 0 by the indexer and skipped by the attention.
 * The CSA index path must be FP8 or NVFP4 (tensor-core indexers); HCA has none.
 */
#define CSA_PAGE_ENTRIES 256
typedef struct {
  int b, m, c, H, c_I, H_I, d_rope, d_rope_I;
  double rope_theta;
  float eps;
  int k, n_w;
  float scale;
  int kv_dtype, idx_dtype, hca;
  int max_pages;      /* block-table row length */
  int num_pages;      /* pages in kv_pages / kI_pages */
  int L_max;          /* upper bound of pos[s] + 1 over the batch */
  int inv_rope;       /* 1: inverse RoPE on the last d_rope output dims */
} csa_paged_params;

typedef struct {
  void *kv_pages, *kI_pages, *kI_scales;
  const int32_t* block_table;                        /* [b][max_pages] */
  void* win;                                         /* [b][n_w][c] */
  void *tail_C_a, *tail_Z_a, *tail_C_b, *tail_Z_b;   /* [b][R][c]; _b NULL for HCA */
  void *tail_CI_a, *tail_ZI_a, *tail_CI_b, *tail_ZI_b; /* [b][2m][c_I] (CSA) */
  const int32_t* pos;                                /* [b] */
  const void *new_C_a, *new_Z_a, *new_C_b, *new_Z_b; /* [b][c] */
  const void *new_CI_a, *new_ZI_a, *new_CI_b, *new_ZI_b; /* [b][c_I] (CSA) */
  const void* new_win;                               /* [b][c] */
  const float *B_a, *B_b, *BI_a, *BI_b;              /* [m][c], [m][c_I] */
  const void* q;                                     /* [b][H][c] */
  const void* q_I;                                   /* [b][H_I][c_I] (CSA) */
  const float* w;                                    /* [b][H_I] (CSA) */
  const float* sink;                                 /* [H] */
  void* out;                                         /* [b][H][c] */
  float* lse;                                        /* [b][H] or NULL */
  int32_t* idx_out;                                  /* [b][k] or NULL (CSA) */
  int32_t* count_out;                                /* [b] or NULL (CSA) */
} csa_paged_tensors;

csa_status csa_decode_paged(const csa_paged_params* p, const csa_paged_tensors* x, void* ws,
                            size_t ws_bytes, cudaStream_t stream);
size_t csa_decode_paged_workspace_size(const csa_paged_params* p);
int csa_decode_paged_launch_count(const csa_paged_params* p);

/*
 * CSA prefill of b sequences of n tokens; every token t = 0..n-1 is a query.
 * Compresses all E = n/m entries (latent and index branch) into the caches,
 * quantises q_I, scores every (t, s) pair, selects k per query and attends.
 */
typedef struct {
  int b, n, m, c, H, c_I, H_I, d_rope, d_rope_I;
  double rope_theta;
  float eps;
  int k, n_w;
  float scale;
  int kv_dtype;            /* CSA_BF16 or CSA_F32 */
  int idx_dtype;           /* CSA_FP8_E4M3, CSA_NVFP4 or CSA_F32 */
  int score_dtype;         /* CSA_BF16 or CSA_F32 */
  int inv_rope;            /* 1: inverse RoPE on the last d_rope output dims (see csa_attn_params) */
} csa_prefill_params;

typedef struct {
  const void *C_a, *Z_a, *C_b, *Z_b;   /* [b][n][c] */
  const float *B_a, *B_b;              /* [m][c] */
  const void *CI_a, *ZI_a, *CI_b, *ZI_b; /* [b][n][c_I] */
  const float *BI_a, *BI_b;            /* [m][c_I] */
  const void* kv_win;                  /* [b][n][c] */
  const void* q;                       /* [b][n][H][c] */
  const void* q_I;                     /* [b][n][H_I][c_I] unquantised (kv_dtype) */
  const float* w;                      /* [b][n][H_I] */
  const float* sink;                   /* [H] */
  void* kv_cache;                      /* out: [b][n/m][c] */
  void* kI_cache;                      /* out: [b][n/m][row] */
  void* kI_scales;                     /* out: as in csa_decode_tensors with E_cap = n/m */
  void* out;                           /* [b][n][H][c] */
  float* lse;                          /* [b][n][H] or NULL */
  int32_t* idx_out;                    /* [b][n][k] or NULL */
  int32_t* count_out;                  /* [b][n] or NULL */
} csa_prefill_tensors;

csa_status csa_prefill(const csa_prefill_params* p, const csa_prefill_tensors* x, void* ws,
                       size_t ws_bytes, cudaStream_t stream);
/* Device workspace csa_prefill needs (bytes); host only. */
size_t csa_prefill_workspace_size(const csa_prefill_params* p);
/* Number of kernel launches one csa_prefill call makes with these parameters; host only. */
int csa_prefill_launch_count(const csa_prefill_params* p);

/* ------------------------------------------------------------------------ */
/* Context-parallel decode: each sequence's compressed entries sharded       */
/* ------------------------------------------------------------------------ */

/*
 * Source: "DeepSeek Technical Reports", section DSA (the k best index scores of a query
 * select the entries it attends to).  A long cache is split into contiguous shards of
 * entries, one per rank; rank r holds entries [entry_offset, entry_offset + E_local) of
 * every sequence.  A decode step then runs:
 *   1. csa_index_scores and csa_topk on the rank's shard, with the query positions
 *      shifted by -m * entry_offset (the entries visible to t are those below
 *      E(t) - entry_offset in the shard);
 *   2. csa_cp_candidates: the rank's top-k as (bf16 score, global entry) pairs;
 *   3. an all-gather of the candidates over the ranks (the caller's collective), rank r's
 *      block at index r;
 *   4. csa_cp_merge: the top-k of the gathered candidates, which is exactly the top-k of
 *      the whole cache (every entry of the global top-k is among its shard's k best under
 *      the same order: score descending, entry ascending); entries ascending, -1 padded;
 *   5. csa_cp_pack_rows: the selected rows this rank holds, into their selection slots
 *      (zeros elsewhere), then a sum over the ranks (the caller's all-reduce) gathers
 *      the selected rows on every rank;
 *   6. csa_sparse_attn over the gathered rows (E_cap = k, selection rows_idx) and the
 *      window, which every rank holds.
 * The pages speak of no context parallelism; this follows from the top-k's definition.
 * All pointers are device memory, all calls asynchronous on the stream.
 */

/* cand_scores [b][k] bf16 and cand_idx [b][k] int32 from the rank's scores ([b][E_local]
 * bf16) and its top-k (idx [b][k] local entries, count [b]): the score and the global
 * entry (entry_offset + local) of each selected entry; -inf and -1 past count. */
csa_status csa_cp_candidates(const void* scores, int E_local, const int32_t* idx,
                             const int32_t* count, int b, int k, int entry_offset,
                             void* cand_scores, int32_t* cand_idx, cudaStream_t stream);

/* Top-k of G ranks' candidates: cand_scores [G][b][k] bf16, cand_idx [G][b][k] (rank r's
 * entries all below rank r + 1's).  Writes idx [b][k] (global entries, ascending, -1
 * padded), count [b] and rows_idx [b][k] (0 .. count - 1, then -1: the selection of the
 * gathered rows).  ws: csa_cp_merge_workspace_size() bytes, 256-byte aligned. */
size_t csa_cp_merge_workspace_size(int G, int b, int k);
csa_status csa_cp_merge(const void* cand_scores, const int32_t* cand_idx, int G, int b, int k,
                        int32_t* idx, int32_t* count, int32_t* rows_idx, void* ws, size_t ws_bytes,
                        cudaStream_t stream);

/* rows [b][k][c] (kv_dtype): slot j of sequence s is row (idx[s][j] - entry_offset) of
 * the rank's shard kv_local ([b][E_cap_local][c]) when entry_offset <= idx[s][j] <
 * entry_offset + E_local and j < count[s]; zeros otherwise.  c * element size must be a
 * multiple of 16; kv_local and rows 16-byte aligned. */
csa_status csa_cp_pack_rows(const void* kv_local, int E_cap_local, int E_local, int entry_offset,
                            int c, int kv_dtype, const int32_t* idx, const int32_t* count, int b,
                            int k, void* rows, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif  /* CSA_H_ */
