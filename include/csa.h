/*
 * csa.h -- C ABI of the B200 (sm_100a) CSA / HCA compressed-attention operator.
 *
 * One attention layer of DeepSeek-V4's hybrid attention, as the explainer
 * pages describe it:
 *
 *   CSA ("compressed sparse attention"): every m consecutive raw KV rows are
 *   pooled into one compressed entry with learned per-channel gate logits and
 *   positional biases over an overlapping 2m-row window; a lightning indexer
 *   scores the causally complete entries against the query; the top-k
 *   entries plus a sliding window of the w most recent raw rows are attended
 *   by shared-KV multi-query attention with a per-head sink logit, RMSNorm on
 *   queries and entries, rotary embedding on the last 64 dims only, and the
 *   inverse rotation applied to the output.
 *     - "DeepSeek-V4: Making a Million Tokens Affordable", section "Two ways
 *       to shrink attention, interleaved" (m=4, top-k=1024, overlap 2m, sink,
 *       RMSNorm, partial RoPE, inverse RoPE on the output, 128-token window).
 *     - "DeepSeek-V4 Explained: Compressed Sparse Attention and 1M Context at
 *       10% KV", section "The attention stack, and why it is two mechanisms"
 *       (compression weights and positional biases, lightning indexer,
 *       shared-KV multi-query layout, BF16 rotary dims + FP8 remainder).
 *   HCA ("heavily compressed attention"): the same path with m'=128, no
 *   overlap, no indexer and dense attention over every visible entry.
 *     - same page, same section (m' = 128, and attention dense over all the
 *       remaining entries).
 *
 * The pages give no formula for the indexer or the gate and no storage
 * layout; the definitions this library implements are stated at each call.
 *
 * Conventions (every call):
 *   - Returns csa_status_t; CSA_OK = 0.  Argument errors are detected on the
 *     host, before any launch, and leave all buffers untouched;
 *     csa_last_error() then describes the failure (thread-local string).
 *   - Every pointer is a DEVICE pointer owned by the caller, 16-byte aligned,
 *     unless marked "host".  The library allocates nothing on the hot calls.
 *   - Calls are asynchronous on the given CUDA stream (a cudaStream_t passed
 *     as void*; NULL = legacy default stream).  Device-side faults surface at
 *     the caller's next synchronisation.  Kernels contain only bounded waits:
 *     a wait that gives up sets a bit in the workspace's device error word,
 *     read back by csa_device_error().
 *   - Workspace: csa_workspace_size() bytes of device memory, zero-filled by
 *     the caller before its FIRST use (the library leaves its counters and
 *     histograms at zero after every call; zero it again after a device
 *     error).  Concurrent calls must not share a workspace.
 *   - Positions: q_pos[b * Tq + j] (device int64) is the absolute position t
 *     of query token j of sequence b; raw row index r = t - pos0.
 *
 * Stored-row formats (kv_format), one row = one compressed entry or one
 * window row, row_bytes = csa_row_bytes():
 *   CSA_FMT_F32   D float32.
 *   CSA_FMT_BF16  D bfloat16.
 *   CSA_FMT_MIXED D+80 bytes: FP8-e4m3 codes of dims [0, D-64) at byte 0,
 *                 bfloat16 of the 64 rotary dims at byte D-64, float32 scale
 *                 sigma at byte D+64, zero padding.  value = code * sigma for
 *                 the FP8 part; sigma is the smallest power of two with
 *                 max|x| / sigma <= 448 (1 for an all-zero part), codes are
 *                 round-to-nearest-even with saturation.
 *
 * Index-key formats (idx_format), one key of d_I dims per entry:
 *   CSA_FMT_F32   d_I float32, idx_key_scale all 1.
 *   CSA_FMT_E4M3  d_I e4m3 codes; idx_key_scale[i] = the key's power-of-two scale.
 *   CSA_FMT_E2M1  d_I / 2 bytes of FP4 e2m1 codes (1 sign, 2 exponent bits with bias 1, 1 mantissa
 *                 bit; magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6), two per byte with the even dim in the
 *                 low nibble; idx_key_scale[i] holds a uint32 scale word (stored in the float
 *                 array's 4 bytes): bits 0..7 = e + 127 for the key scale sigma = 2^e, bits
 *                 8+4b..11+4b = the offset delta_b (0..7) of dims [32b, 32b+32); the value of dim d
 *                 is code * sigma * 2^-delta_b.  d_I a multiple of 32.  Index queries stay e4m3.
 *                 ("DeepSeek-V4: Making a Million Tokens Affordable", "Two ways to shrink
 *                 attention, interleaved": the indexer's attention runs in FP4.)
 *
 * Rotary convention: interleaved pairs (D-64+2u, D-64+2u+1), u < 32, angle
 * pos * base^(-2u/64) formed and reduced in float64.
 */
#ifndef CSA_B200_CSA_H_
#define CSA_B200_CSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CSA_API __attribute__((visibility("default")))
#else
#define CSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum csa_status {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1,     /* bad pointer, size, alignment or layer field */
  CSA_ERR_UNSUPPORTED = 2,     /* valid, but no kernel for this shape / format */
  CSA_ERR_WORKSPACE = 3,       /* workspace missing or smaller than csa_workspace_size() */
  CSA_ERR_CUDA = 4,            /* a CUDA runtime call failed (message in csa_last_error) */
  CSA_ERR_DEVICE_TIMEOUT = 5   /* a kernel set a bit of the device error word (csa_device_error) */
} csa_status_t;

enum {
  CSA_FMT_F32 = 0,
  CSA_FMT_BF16 = 1,
  CSA_FMT_MIXED = 2,           /* kv_format only */
  CSA_FMT_E4M3 = 3,            /* idx_format only */
  CSA_FMT_E2M1 = 4             /* idx_format only: FP4 index keys, e4m3 index queries (see below) */
};

enum { CSA_KIND_CSA = 0, CSA_KIND_HCA = 1 };

/* One layer's hyper-parameters. */
typedef struct csa_layer {
  int32_t kind;          /* CSA_KIND_CSA or CSA_KIND_HCA */
  int32_t B;             /* sequences */
  int32_t H;             /* query heads (all share the one KV head) */
  int32_t D;             /* KV / head dim; the last d_rope dims are rotary */
  int32_t d_rope;        /* must be 64 */
  int32_t m;             /* raw rows per compressed entry (4 for CSA, 128 for HCA) */
  int32_t overlap;       /* 1: entry i pools raw rows [(i-1)m, (i+1)m); 0: [im, (i+1)m) */
  int32_t top_k;         /* CSA: entries kept per query; ignored for HCA */
  int32_t window;        /* w: most recent raw rows attended uncompressed (incl. current) */
  int32_t H_I;           /* CSA: indexer heads */
  int32_t d_I;           /* CSA: indexer head dim */
  int32_t kv_format;     /* CSA_FMT_F32 | CSA_FMT_BF16 | CSA_FMT_MIXED */
  int32_t idx_format;    /* CSA_FMT_F32 | CSA_FMT_E4M3 | CSA_FMT_E2M1 (index keys; queries e4m3 for E2M1) */
  int32_t act_format;    /* CSA_FMT_F32 | CSA_FMT_BF16: queries, raw rows, gate logits, output */
  double rope_base;      /* rotary base (10000) */
  float eps;             /* RMSNorm epsilon (1e-6) */
  float softmax_scale;   /* logit scale; 0 selects 1/sqrt(D) */
  int64_t pos0;          /* absolute position of raw row 0 */
} csa_layer_t;

/* Per-layer caches (state carried across decode steps; caller-owned). */
typedef struct csa_cache {
  void* entries;          /* [B][entry_cap][row_bytes] compressed entries, entry i at slot i */
  int64_t entry_cap;      /* capacity in entries per sequence */
  void* idx_keys;         /* CSA: [B][entry_cap][d_I] index keys (e4m3 codes or float32) */
  const float* idx_key_scale; /* CSA: [B][entry_cap] per-key scale (all 1 for float32 keys) */
  void* window;           /* [B][window_cap][row_bytes]: raw row r's rotated row at slot r mod window_cap */
  int64_t window_cap;     /* >= window; >= Tq + window - 1 for a Tq-token chunk */
  void* raw;              /* [B][raw_cap][D] un-rotated raw rows (act_format); row r at slot (r - raw_base) mod raw_cap */
  void* gate;             /* [B][raw_cap][D] gate logits, same indexing as raw */
  int64_t raw_cap;        /* decode: >= (1+overlap)*m; prefill: the chunk plus overlap*m look-back rows */
  int64_t raw_base;       /* raw row stored at slot 0 (0 for a ring) */
} csa_cache_t;

/* Learned per-layer parameters. */
typedef struct csa_params {
  const float* pos_bias;  /* [(1+overlap)*m][D] positional bias per window slot and channel */
  const float* gamma_kv;  /* [D] RMSNorm weight of compressed entries, or NULL (= 1) */
  const float* gamma_q;   /* [D] RMSNorm weight of queries, or NULL (= 1) */
  const float* sinks;     /* [H] per-head sink logits */
} csa_params_t;

/* Operation selector for csa_workspace_size(). */
enum {
  CSA_OP_INDEX_TOPK = 0,
  CSA_OP_SPARSE_ATTEND = 1,
  CSA_OP_HCA_ATTEND = 2,
  CSA_OP_DECODE_STEP = 3,   /* csa_decode_step / hca_decode_step */
  CSA_OP_PREFILL = 4,       /* csa_prefill */
  CSA_OP_DECODE_STEP_INDEXED = 5  /* csa_decode_step_indexed */
};

/* Index-key stream of a CSA layer: per token one index row and one row of gate logits of d_I
 * values (act_format), kept in rings with the same slots as cache->raw / cache->gate
 * (row r at slot (r - raw_base) mod raw_cap), and the slot biases of their compression. */
typedef struct csa_index_stream {
  void* raw;              /* [B][raw_cap][d_I] index rows */
  void* gate;             /* [B][raw_cap][d_I] gate logits */
  const float* pos_bias;  /* [(1+overlap)*m][d_I] positional bias per window slot and channel */
} csa_index_stream_t;

/* Bytes of one stored row for the layer's kv_format (host). */
CSA_API size_t csa_row_bytes(const csa_layer_t* L);

/* Workspace bytes an operation needs for Tq queries per sequence and caches
 * of entry_cap entries (host; 0 if the layer is invalid). */
CSA_API size_t csa_workspace_size(const csa_layer_t* L, int32_t op, int32_t Tq, int64_t entry_cap);

/* Thread-local text of the last error returned on this thread (host). */
CSA_API const char* csa_last_error(void);

/* Library version string (host). */
CSA_API const char* csa_version(void);

/* Reads and clears the device error words (synchronises the stream): the
 * workspace's word (workspace may be NULL: then it is skipped) and the
 * library's own word on the current device, where the kernels of the calls
 * that take no workspace (csa_append, csa_compress) report.  *code gets the
 * OR of the bits kernels set (0 = none):
 *   1  a bounded wait (mbarrier / tensor-memory pipeline / cluster
 *      reduction) gave up; the results of that launch are incomplete;
 *   2  the multi-CTA top-k found its score histogram inconsistent with the
 *      scores; that row's top-k output is incomplete (padded with -1).
 * Returns CSA_ERR_DEVICE_TIMEOUT if any bit was set. */
CSA_API csa_status_t csa_device_error(void* workspace, size_t ws_bytes, void* stream, int32_t* code);

/* Test and diagnostic aids (no counterpart on the pages). */

/* Workspace segments, for csa_debug_workspace_segment. */
enum {
  CSA_SEG_ERROR_WORD = 0,      /* the int32 device error word */
  CSA_SEG_SCORES = 1,          /* indexer scores [rows][entry_cap] float32 */
  CSA_SEG_TOPK_HISTOGRAM = 2,  /* multi-CTA top-k: [rows][4096] uint32 score histogram, then
                                  [rows][4] counters, then [rows][4096] second histogram */
  CSA_SEG_TOPK = 3,            /* top-k indices of the fused calls [rows][top_k] int32 */
  CSA_SEG_PARTIALS = 4,        /* attention partials */
  CSA_SEG_INDEX_QUERY = 5,     /* csa_decode_step_indexed: the produced index query [B][H_I][d_I] */
  CSA_SEG_INDEX_QUERY_SCALE = 6  /* ... and its per-head scales [B][H_I] float32 */
};

/* Byte offset and size of one segment of the workspace that
 * csa_workspace_size(L, op, Tq, entry_cap) describes (host; *bytes = 0 when
 * the operation has no such segment).  Lets a test inject state (e.g. an
 * inconsistent score histogram) into a caller-owned workspace. */
CSA_API csa_status_t csa_debug_workspace_segment(const csa_layer_t* L, int32_t op, int32_t Tq, int64_t entry_cap,
                                                 int32_t segment, size_t* offset, size_t* bytes);

/* Launches one CTA that waits, with the library's bounded wait and a limit
 * of limit_ns nanoseconds (0 < limit_ns <= 1e9), on an mbarrier phase that
 * nothing completes; when the limit passes it sets bit 1 of the workspace's
 * error word and returns.  Nothing is in flight in the CTA when it gives up,
 * so the context stays usable.  Lets a test drive the failure-reporting path
 * (csa_device_error -> CSA_ERR_DEVICE_TIMEOUT) without a device fault. */
CSA_API csa_status_t csa_debug_wait_probe(void* workspace, size_t ws_bytes, uint64_t limit_ns, void* stream);

/* Profiling aid (no counterpart on the pages).  When ev_start and ev_stop (cudaEvent_t handles
 * created with timing enabled) are both non-NULL, every later call made from this host thread
 * records ev_start immediately before and ev_stop immediately after the launch of the indexer
 * score kernel (the dominant kernel of a CSA decode step), with the external-record flag so the
 * records become event nodes when the stream is being captured into a CUDA graph.  NULL, NULL
 * turns it off.  Host only; never fails. */
CSA_API void csa_profile_events(void* ev_start, void* ev_stop);

/* Profiling aid (no counterpart on the pages).  Arms a timeline on this host thread: later
 * calls record events[0], events[1], ... (cudaEvent_t handles with timing enabled), one just
 * before each kernel launch or memset they issue, until `capacity` events are used; the records
 * use the external flag, so they become event nodes under stream capture.  The caller records
 * one more event after the last call to close the last interval.  NULL disarms it. */
CSA_API void csa_profile_timeline(void** events, int32_t capacity);

/* Events of the armed timeline used so far. */
CSA_API int32_t csa_profile_timeline_count(void);

/* Number of kernels this process has launched through the library so far (host counter). */
CSA_API uint64_t csa_launch_count(void);

/* Append Tq new tokens per sequence: raw rows x_new[b][j] (and gate rows
 * g_new) are written into the raw / gate rings at slot (r - raw_base) mod
 * raw_cap (skipped when x_new is NULL: the rows are then already in the raw
 * buffer), and each token's window row RoPE_t(x) -- rotated at its own
 * position, not normalised -- is stored at window slot r mod window_cap.
 *   x_new, g_new: [B][Tq][D] act_format, or both NULL.
 * The sliding window is the pages' short branch over the most recent tokens,
 * kept uncompressed ("DeepSeek-V4 Explained: ...", "The attention stack, and
 * why it is two mechanisms"). */
CSA_API csa_status_t csa_append(const csa_layer_t* L, const csa_cache_t* cache,
                        const void* x_new, const void* g_new,
                        const int64_t* q_pos, int32_t Tq, void* stream);

/* Compress every entry completed by the Tq tokens at q_pos (entry i is
 * completed by raw row (i+1)m - 1).  Entry i = RoPE_{pos0 + i m}(RMSNorm(e) *
 * gamma_kv) with e_c = sum_r softmax_r(gate[r][c] + pos_bias[r - (i-ov)m][c])
 * * raw[r][c] over raw rows r in [(i-ov)m, (i+1)m) clipped at 0, written to
 * entries[b][i] in kv_format.  The raw buffer must hold those rows.
 * Pages: each group of m consecutive tokens becomes one entry, pooled with
 * learned weights and per-slot position biases ("DeepSeek-V4 Explained: ...");
 * an entry reads 2m source rows, yet the sequence still shrinks m-fold
 * ("DeepSeek-V4: Making a Million Tokens Affordable", "Two ways to shrink
 * attention"). */
CSA_API csa_status_t csa_compress(const csa_layer_t* L, const csa_cache_t* cache,
                          const csa_params_t* P, const int64_t* q_pos, int32_t Tq,
                          void* stream);

/* Lightning indexer + top-k (CSA).  For query (b, j) at position t, entry i
 * is visible iff pos0 + (i+1)m - 1 <= t; its score is
 *   s_i = sum_h head_w[h] * max(0, idx_q_scale[h] * idx_key_scale[i] * <idx_q[h], idx_key[i]>)
 * and the k highest scores are kept, ties to the smaller index, written in
 * ascending entry order to topk_idx[b][j][0..k), padded with -1 when fewer
 * than k entries are visible.
 *   idx_q:       [B][Tq][H_I][d_I] e4m3 codes or float32
 *   idx_q_scale: [B][Tq][H_I] float32;  head_w: [B][Tq][H_I] float32
 *   n_max:       entries scored per query (<= entry_cap; entries beyond the
 *                query's visible count are excluded)
 *   topk_idx:    [B][Tq][top_k] int32 (output)
 *   scores:      [B][Tq][n_max] float32 (output, optional: NULL keeps them in the workspace)
 * Pages: a cheap low-rank indexer scores the compressed entries and each query
 * attends only to its k best ("DeepSeek-V4 Explained"); the indexer uses a
 * few small FP8 heads ("DeepSeek-V4, explained.", step 3). */
CSA_API csa_status_t csa_index_topk(const csa_layer_t* L, const csa_cache_t* cache,
                            const void* idx_q, const float* idx_q_scale, const float* head_w,
                            const int64_t* q_pos, int32_t Tq, int64_t n_max,
                            int32_t* topk_idx, float* scores,
                            void* workspace, size_t ws_bytes, void* stream);

/* Sparse shared-KV multi-query attention (CSA).  For query (b, j) at t:
 *   q~_h = RoPE_t(RMSNorm(q_h) * gamma_q);   keys = values = the selected
 *   entries topk_idx[b][j][*] (-1 skipped) plus the window rows r in
 *   [max(0, r_t - w + 1), r_t];  l_j = <q~_h, k_j> * softmax_scale;
 *   o_h = sum_j e^{l_j} k_j / (e^{sink_h} + sum_j e^{l_j});  out = RoPE_{-t}(o_h).
 *   q:   [B][Tq][H][D] act_format;  out: [B][Tq][H][D] act_format.
 * Pages: an entry is both key and value, the output is rotated back by the
 * query's position, and each head has a learned sink ("DeepSeek-V4: Making a
 * Million Tokens Affordable"). */
CSA_API csa_status_t csa_sparse_attend(const csa_layer_t* L, const csa_cache_t* cache,
                               const csa_params_t* P, const void* q, const int64_t* q_pos,
                               int32_t Tq, const int32_t* topk_idx, void* out,
                               void* workspace, size_t ws_bytes, void* stream);

/* Dense attention over every visible entry i < n_visible(t) (HCA) plus the
 * window rows, otherwise as csa_sparse_attend.  n_max bounds the visible
 * entries (<= entry_cap).
 * Pages: after the heavy compression, attention stays dense, without an
 * indexer or a top-k ("DeepSeek-V4: Making a Million Tokens Affordable"). */
CSA_API csa_status_t hca_attend(const csa_layer_t* L, const csa_cache_t* cache,
                        const csa_params_t* P, const void* q, const int64_t* q_pos,
                        int32_t Tq, int64_t n_max, void* out,
                        void* workspace, size_t ws_bytes, void* stream);

/* One fused CSA decode step for token t = q_pos[b] of every sequence:
 * csa_append (x_new, g_new) -> csa_compress (when t completes a group) ->
 * csa_index_topk over entry_cap entries -> csa_sparse_attend.  Tq = 1.
 * topk_idx: [B][top_k] int32 output, or NULL (kept in the workspace).
 * The index keys are inputs, so append+compress does not feed the indexer:
 * the library runs it on an internal second stream (one per thread and
 * device, created by the first call made outside stream capture), forked
 * from and joined back into `stream` before attention.  Ordering with
 * respect to `stream` is unchanged, and the pattern is graph-capturable. */
CSA_API csa_status_t csa_decode_step(const csa_layer_t* L, const csa_cache_t* cache,
                             const csa_params_t* P, const void* q,
                             const void* idx_q, const float* idx_q_scale, const float* head_w,
                             const void* x_new, const void* g_new, const int64_t* q_pos,
                             void* out, int32_t* topk_idx,
                             void* workspace, size_t ws_bytes, void* stream);

/* Index keys produced from the index-key stream.  Appends the Tq tokens' index rows x_new / g_new
 * ([B][Tq][d_I] act_format; both NULL when the rows are already in S->raw / S->gate) to the stream's
 * rings, then writes the key of every entry the tokens complete: the entry's window rows
 * [(i-ov)m, (i+1)m) clipped at 0 pooled with a per-channel softmax of gate + S->pos_bias[slot], no
 * RMSNorm, no rotation, into cache->idx_keys[b][i] (e4m3 codes of k / sigma with sigma the smallest
 * power of two with max|k| / sigma <= 448, into cache->idx_key_scale[b][i]; float32 keys get scale 1).
 * Reading of the pages: the lightning indexer scores the compressed entries "in a low-rank way"
 * ("DeepSeek-V4 Explained: ...", "The attention stack, and why it is two mechanisms"); its keys are
 * read as compressed like the entries themselves.  Needs d_I a multiple of 32, <= 128. */
CSA_API csa_status_t csa_index_keys(const csa_layer_t* L, const csa_cache_t* cache, const csa_index_stream_t* S,
                                    const void* x_new, const void* g_new, const int64_t* q_pos, int32_t Tq,
                                    void* stream);

/* Low-rank index queries: for each of `rows` query tokens, q_h = W_h c with c [rows][rank] (bf16,
 * the query's low-rank latent) and W [H_I * d_I][rank] (bf16, row h*d_I + d of W is output dim d of
 * head h), stored as idx_q [rows][H_I][d_I] e4m3 codes of q_h / sigma_h with idx_q_scale
 * [rows][H_I] the per-head power-of-two scale (the same rule as the keys), or float32 values with
 * scale 1.  rank a multiple of 16; d_I a multiple of 32, <= 128.  Same page and section (a low-rank
 * indexer); the up-projection of a latent is this library's reading of it. */
CSA_API csa_status_t csa_index_query(const csa_layer_t* L, const void* c, const void* W, int32_t rank,
                                     int32_t rows, void* idx_q, float* idx_q_scale, void* stream);

/* csa_decode_step with the index side produced in the step: csa_index_keys for the token (its
 * index row idx_x_new / idx_g_new [B][d_I]) and csa_index_query from its latent c [B][rank] run
 * first, on `stream`, and the indexer then scores the keys and queries they wrote (the index query
 * lives in the workspace of CSA_OP_DECODE_STEP_INDEXED).  Other arguments as csa_decode_step. */
CSA_API csa_status_t csa_decode_step_indexed(const csa_layer_t* L, const csa_cache_t* cache,
                                             const csa_params_t* P, const csa_index_stream_t* S,
                                             const void* q, const void* c, const void* W, int32_t rank,
                                             const float* head_w, const void* x_new, const void* g_new,
                                             const void* idx_x_new, const void* idx_g_new,
                                             const int64_t* q_pos, void* out, int32_t* topk_idx,
                                             void* workspace, size_t ws_bytes, void* stream);

/* Context-sharded CSA decode (one sequence's entries and index keys split into contiguous shards,
 * one per rank).  A rank holding entries [entry_offset, entry_offset + n_local) at slots 0.. of its
 * cache runs, for the B decode queries:
 *   1. csa_index_topk over its shard, with a layer whose pos0 is pos0 + entry_offset * m (so each
 *      shard entry's visibility is that of its global position) and n_max = n_local;
 *   2. csa_shard_candidates: (score, global index) of its local top-k;
 *   3. an all-gather of the candidates, [shards][B][top_k] each (the caller's collective);
 *   4. csa_shard_select: the global top-k of the gathered candidates, identical on every rank;
 *   5. csa_sparse_attend_partial over the selected entries it holds (one rank also the window rows);
 *   6. an all-gather of the partials, [shards][B][H][D + 2] (the caller's collective);
 *   7. csa_attend_merge: the output, with the sink counted once and the inverse rotation.
 * The result equals csa_sparse_attend with the unsharded top-k: an entry of the global top-k is in
 * its own shard's top-k, and attention over disjoint key sets merges by log-sum-exp weights.  The
 * pages describe one layer, not its distribution; the sink and the inverse rotation are those of
 * "DeepSeek-V4: Making a Million Tokens Affordable", "Two ways to shrink attention, interleaved". */

/* Step 2.  scores: [B][n_local] float32 of the shard (csa_index_topk's optional output); topk_local:
 * [B][top_k] its local top-k (-1 padded).  Writes cand_score [B][top_k] (-inf for padding) and
 * cand_idx [B][top_k] = local index + entry_offset (-1 for padding). */
CSA_API csa_status_t csa_shard_candidates(const csa_layer_t* L, const float* scores, int64_t n_local,
                                          const int32_t* topk_local, int64_t entry_offset, float* cand_score,
                                          int32_t* cand_idx, void* stream);

/* Step 4.  cand_score / cand_idx: [shards][B][top_k], shard s's lists in ascending index order and
 * the shards in ascending entry_offset order.  Writes topk_idx [B][top_k]: the top_k largest scores,
 * ties to the smaller global index, in ascending index order, -1 padded when fewer exist.
 * shards * top_k <= 262144. */
CSA_API csa_status_t csa_shard_select(const csa_layer_t* L, int32_t shards, const float* cand_score,
                                      const int32_t* cand_idx, int32_t* topk_idx, void* stream);

/* Step 5.  topk_idx [B][top_k] holds global indices; the entries in [entry_offset, entry_offset +
 * cache->entry_cap) are attended from cache slot (index - entry_offset), the others skipped; the
 * window rows only when with_window != 0.  partial: [B][H][D + 2] float32, per (query, head) the
 * weighted mean O/l of the attended rows (before the inverse rotation), then m and l in base 2
 * (max logit * log2 e and the sum of 2^(logit * log2 e - m)); no sink.  Needs H = 128, D = 512,
 * bf16 or mixed rows, B <= 8; workspace of CSA_OP_SPARSE_ATTEND. */
CSA_API csa_status_t csa_sparse_attend_partial(const csa_layer_t* L, const csa_cache_t* cache,
                                               const csa_params_t* P, const void* q, const int64_t* q_pos,
                                               const int32_t* topk_idx, int64_t entry_offset, int32_t with_window,
                                               float* partial, void* workspace, size_t ws_bytes, void* stream);

/* Step 7.  partials: [parts][B][H][D + 2] as written by csa_sparse_attend_partial; out [B][H][D]
 * act_format. */
CSA_API csa_status_t csa_attend_merge(const csa_layer_t* L, const csa_params_t* P, const int64_t* q_pos,
                                      int32_t parts, const float* partials, void* out, void* stream);

/* Bytes of the static device scratch used by csa_decode_step_scratch. */
#define CSA_SCRATCH_BYTES ((size_t)16 << 20)

/* csa_decode_step without a caller workspace (no counterpart on the pages:
 * a convenience of this library).  The workspace is a fixed array of
 * CSA_SCRATCH_BYTES in the library's static device memory, one per device,
 * so the call allocates nothing.
 *   - Limit: csa_workspace_size(L, CSA_OP_DECODE_STEP, 1, cache->entry_cap)
 *     must be <= CSA_SCRATCH_BYTES (B = 1 covers entry_cap up to 2^18, i.e.
 *     a 1M-token context at m = 4); a larger call returns CSA_ERR_WORKSPACE
 *     and touches no device state.
 *   - The array's address is looked up (cudaGetSymbolAddress, which may load
 *     the module) on the first call on each device: make that first call
 *     outside any CUDA stream capture.
 *   - Every call on a device shares its one array: two calls whose executions
 *     overlap (different streams or threads, concurrent graph replays) race
 *     on it and give undefined results.  Serialise them.
 *   - device_error: NULL, or a host int32 that receives the device error word
 *     (see csa_device_error); non-NULL synchronises the stream (not allowed
 *     during stream capture) and, when the word is non-zero, zero-fills the
 *     scratch again and returns CSA_ERR_DEVICE_TIMEOUT.  A call with NULL
 *     leaves any bits its kernels set in the scratch's word: the next call
 *     with a non-NULL device_error reports them (with its own), so after
 *     NULL calls that report covers every call since the last non-NULL one.
 *   - After a device error the scratch's histograms may be left non-zero.
 *     Every call therefore starts with a small guard kernel that, when the
 *     scratch's error word is set, zero-fills the scratch's top-k histograms
 *     and counters (keeping the word), so later calls, NULL or not, select
 *     from clean histograms.
 * Other arguments, layouts and errors as csa_decode_step. */
CSA_API csa_status_t csa_decode_step_scratch(const csa_layer_t* L, const csa_cache_t* cache,
                             const csa_params_t* P, const void* q,
                             const void* idx_q, const float* idx_q_scale, const float* head_w,
                             const void* x_new, const void* g_new, const int64_t* q_pos,
                             void* out, int32_t* topk_idx, int32_t* device_error,
                             void* stream);

/* Test aid for csa_decode_step_scratch (no counterpart on the pages): copies `bytes` bytes between
 * `buf` (host or device memory) and the current device's static scratch at byte `offset`, in the
 * direction `to_scratch` (1: buf -> scratch, 0: scratch -> buf), on `stream`, and synchronises it.
 * Offsets of the scratch's segments are those csa_debug_workspace_segment gives for the decode step.
 * Lets a test plant a device error and dirty histograms in the scratch.  A range outside the
 * CSA_SCRATCH_BYTES array returns CSA_ERR_INVALID_ARG with no device work. */
CSA_API csa_status_t csa_debug_scratch_copy(size_t offset, void* buf, size_t bytes, int32_t to_scratch,
                                            void* stream);

/* One fused HCA decode step: csa_append -> csa_compress -> hca_attend. */
CSA_API csa_status_t hca_decode_step(const csa_layer_t* L, const csa_cache_t* cache,
                             const csa_params_t* P, const void* q,
                             const void* x_new, const void* g_new, const int64_t* q_pos,
                             void* out, void* workspace, size_t ws_bytes, void* stream);

/* Chunked prefill of Tq tokens per sequence (CSA or HCA): csa_append of the
 * chunk's window rows (raw rows already in cache->raw), csa_compress of the
 * entries the chunk completes, then per query the indexer + top-k (CSA) and
 * attention.  n_max = entries visible to the chunk's last query. */
CSA_API csa_status_t csa_prefill(const csa_layer_t* L, const csa_cache_t* cache,
                         const csa_params_t* P, const void* q,
                         const void* idx_q, const float* idx_q_scale, const float* head_w,
                         const int64_t* q_pos, int32_t Tq, int64_t n_max,
                         void* out, int32_t* topk_idx,
                         void* workspace, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif  /* CSA_B200_CSA_H_ */
