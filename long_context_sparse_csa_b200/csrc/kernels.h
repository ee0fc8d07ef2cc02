// Launch-argument structs and launchers of the CSA/HCA kernels (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace csa {

// Host-side count of kernel launches issued by the library (for launch accounting).
void note_launches(int n);
// Records the next timeline event (if a timeline is armed on this thread) just before a launch.
void profile_mark(cudaStream_t s);
// Sets this thread's csa_last_error() text and returns st (for entry points outside api.cu).
csa_status_t report_error(csa_status_t st, const char* msg);
// Raises `kernel`'s dynamic shared-memory limit to at least `bytes` on the current device (function
// attributes are per device: the setting is remembered per (device, kernel), under a lock).
cudaError_t ensure_dynamic_smem(const void* kernel, size_t bytes);
// Allows a non-portable cluster size (> 8 CTAs) for `kernel` on the current device (remembered
// per (device, kernel)).
cudaError_t ensure_nonportable_cluster(const void* kernel);

// Launches a kernel in stream order, with an optional thread-block cluster size (cluster > 0).
// (Programmatic dependent launch was measured slower on the decode chain: CTAs parked at the
// dependency wait take SM slots from the kernel still running.)
template <typename Kernel, typename... Args>
cudaError_t launch_kernel(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s, int cluster,
                          Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  int n = 0;
  if (cluster > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = (unsigned)cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  profile_mark(s);
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  note_launches(1);
  return e;
}

// Test aid: one CTA waits (bounded by limit_ns) on an mbarrier phase nothing completes, then sets
// the timeout bit of *err.
cudaError_t launch_wait_probe(int* err, uint64_t limit_ns, cudaStream_t s);

// Device address of the library's own error word on the current device: kernels of calls that take
// no workspace (csa_append, csa_compress) report there; csa_device_error reads and clears it.
cudaError_t library_error_word(int** p);

// ----------------------------------------------------------------------------- append + compress
struct AppendCompressArgs {
  LayerArgs L;
  CacheArgs C;
  const int64_t* q_pos;
  int Tq;
  const uint8_t* x_new;   // [B][Tq][D] act, or null (rows already in C.raw)
  const uint8_t* g_new;
  const float* pos_bias;  // [(1+ov)m][D]
  const float* gamma_kv;  // [D] or null
  int do_append;
  int do_compress;
  int* err;               // device error word (bounded cluster waits); never null
};
cudaError_t launch_append_compress(const AppendCompressArgs& a, int B, int Tq, cudaStream_t s);

// ----------------------------------------------------------------------------- indexer
struct IndexArgs {
  int B, Tq, H_I, d_I, m;
  int idx_fmt;
  int64_t n_max, entry_cap, pos0;
  const int64_t* q_pos;
  const uint8_t* idx_q;     // [B][Tq][H_I][d_I]
  const uint8_t* idx_k;     // [B][entry_cap][d_I]
  const float* k_scale;     // [B][entry_cap]
  const float* q_scale;     // [B][Tq][H_I]
  const float* head_w;      // [B][Tq][H_I]
  float* scores;            // [B][Tq][n_max]
  uint32_t* hist;           // decode (Tq == 1): [B][4096] histogram of the scores' top 12 key bits, or null
  int* err;
  // tensor-core path tiling
  int QN;                   // queries per MMA N-tile (N = QN * H_I)
  int tiles_per_group;      // ceil(n_max / 128)
  int groups_per_seq;       // ceil(Tq / QN)
  int64_t total_items;      // B * groups_per_seq * tiles_per_group
};
// True when the tcgen05 FP8 kernel handles this shape.
bool index_tc_supported(int idx_fmt, int H_I, int d_I);
// Decode (one query per sequence): the warp-level FP8 kernel (index_decode.cu) for these shapes.
bool index_decode_supported(int idx_fmt, int H_I, int d_I);
cudaError_t launch_index_decode(const IndexArgs& a, int num_sms, cudaStream_t s);
cudaError_t launch_index_scores(IndexArgs a, int num_sms, cudaStream_t s);

// ----------------------------------------------------------------------------- index side (keys, queries)
struct IndexPrepArgs {
  int B, Tq, H_I, d_I, m, ov, act_fmt, idx_fmt;
  int64_t pos0, entry_cap, raw_cap, raw_base;
  const int64_t* q_pos;     // [B][Tq]
  // key role: append the tokens' index rows (x_new / g_new [B][Tq][d_I], or null) to the index rings
  // and compress the index key of every entry they complete into keys / key_scale (null: no key role)
  const uint8_t* x_new;
  const uint8_t* g_new;
  uint8_t* raw;             // [B][raw_cap][d_I] index-row ring (act_fmt), KV ring slots
  uint8_t* gate;
  const float* pos_bias;    // [(1+ov)m][d_I]
  uint8_t* keys;            // [B][entry_cap][d_I] (e4m3, or float32)
  float* key_scale;         // [B][entry_cap]
  // query role: q_out [rows][H_I][d_I] = encode(W_h c_row) (c null: no query role)
  const uint8_t* c;         // [rows][rank] bf16
  const uint8_t* W;         // [H_I * d_I][rank] bf16
  int rank, rows;
  uint8_t* q_out;
  float* q_scale_out;       // [rows][H_I]
  int key_blocks;           // set by the launcher
};
cudaError_t launch_index_prep(IndexPrepArgs a, cudaStream_t s);

// ----------------------------------------------------------------------------- top-k
struct TopkArgs {
  const float* scores;      // [rows][n_max]
  int64_t n_max;
  int rows, Tq, m, k;
  int64_t pos0;
  const int64_t* q_pos;     // [rows]
  int32_t* out;             // [rows][k]
  // candidate mode (shard merge): `shards` lists of k candidates per row, laid out [shards][rows][k]
  // (scores and their global indices `map`, -1 = none); the row's candidates in shard order are in
  // ascending index order, and out[] gets their indices (ties to the smaller index, ascending)
  const int32_t* map;
  int shards;
};
cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s);

// Decode rows too long for one CTA: many CTAs per row, fed by the indexer's score histogram.
struct TopkSplitArgs {
  TopkArgs base;
  const uint32_t* hist;     // [rows][4096] (zero on entry; the kernel leaves it zeroed)
  uint32_t* counts;         // [rows][kTopkSplitMaxCtas] list length of each CTA's slice (scratch)
  uint2* list;              // [rows][n_max] (key, index) of the slice's scores at or above the threshold bin
  uint32_t* cnt;            // [rows][4] counters (zero on entry; left zeroed)
  uint32_t* hist2;          // [rows][4096] histogram of key bits 19..8 in the threshold bin (zero on entry; left zeroed)
  int G;                    // CTAs per row (<= kTopkSplitMaxCtas)
  int* err;                 // device error word
};
constexpr int kTopkSplitMaxCtas = 512;
constexpr int64_t kTopkSplitMinN = 16384;     // rows at least this long use the split kernel
constexpr int64_t kTopkSplitMaxN = 655360;    // longer rows take the one-CTA-per-row kernel
int topk_split_ctas(int rows, int64_t n_max, int num_sms);
cudaError_t launch_topk_split(const TopkSplitArgs& a, cudaStream_t s);

// ----------------------------------------------------------------------------- attention
struct AttendArgs {
  LayerArgs L;
  CacheArgs C;
  const uint8_t* q;         // [rows][H][D] act
  uint8_t* qt;              // [rows][H][D] bf16 q~ = RoPE_t(RMSNorm(q) * gamma_q) (tensor-core kernel)
  int* err;                 // device error word
  const int64_t* q_pos;     // [rows]
  int Tq, rows;
  const int32_t* topk;      // CSA: [rows][k]; null for dense (HCA)
  int64_t n_max;            // dense: entries bound
  const float* gamma_q;     // [D] or null
  const float* sinks;       // [H]
  int splits;               // slot splits per row (tcgen05: cluster pairs; mma.sync: CTAs per head group)
  float* part;              // partials (O, m, l): mma.sync [rows][H/HG][splits][HG*(D+2)] fp32;
                            // tcgen05 [rows][splits] x (bf16 O/l as [D/4][H][4], then (m, l) fp32 per head)
  uint8_t* out;             // [rows][H][D] act
  // context-sharded decode: the selected indices are global and this cache holds entries
  // [entry_offset, entry_offset + entry_limit) at slots 0.. (others are skipped); no_window leaves the
  // window rows to another shard; partial_out (non-null) receives the merged (O/l, m, l) per (row,
  // head) as [rows][H][D + 2] fp32 (m, l in base 2, no sink, no inverse rotation) instead of `out`
  int64_t entry_offset, entry_limit;
  int no_window;
  float* partial_out;
  // deferred rows (dense tcgen05 path): the attention kernel leaves out the token's own window row and
  // the entry the token completes; the combine adds them as two keys, their logits (base 2) in
  // extra [rows][2][H] (-inf for a row that does not exist)
  int defer_new;
  float* extra;
};
// Attention kernel family for a call of `rows` query rows: 2 = tcgen05 (H = 128, D = 512, bf16 or
// mixed rows, at most kTcMaxRows rows), 3 = persistent tcgen05 prefill kernel (H = 64, D = 512, bf16
// rows and activations, more than kTcMaxRows rows), 1 = mma.sync head groups, 0 = CUDA-core generic.
// `dense`: every visible entry (HCA) rather than a top-k list.
constexpr int kTcMaxRows = 8;
int attend_path(const LayerArgs& L, bool dense, int rows);
// Head-group size of the mma.sync kernel (0: not applicable).
int attend_head_group(const LayerArgs& L);
int attend_num_splits(const LayerArgs& L, bool dense, int rows, int64_t slots, int num_sms);
size_t attend_partial_bytes(const LayerArgs& L, bool dense, int rows, int splits);
// q~ for the tcgen05 kernels, decode and prefill (a no-op for the other kernels, which prepare q
// themselves); it reads only q, gamma_q and q_pos, so it may run beside compression.
cudaError_t launch_attend_qprep(const AttendArgs& a, cudaStream_t s);
cudaError_t launch_attend(const AttendArgs& a, cudaStream_t s);
bool attend_prefill_tc_supported(const LayerArgs& L, int rows);
cudaError_t launch_attend_deferred(const AttendArgs& a, cudaStream_t s);
cudaError_t launch_attend_extra_logits(const AttendArgs& a, cudaStream_t s);
cudaError_t launch_attend_combine(const AttendArgs& a, cudaStream_t s);
cudaError_t launch_attend_prefill_tc(const AttendArgs& a, cudaStream_t s);

// ----------------------------------------------------------------------------- context-sharded decode
// Candidates of one shard: (score, global index) of its local top-k, [rows][k].
cudaError_t launch_shard_candidates(const float* scores, int64_t n_local, const int32_t* topk_local, int rows,
                                    int k, int64_t entry_offset, float* cand_score, int32_t* cand_idx,
                                    cudaStream_t s);
// out[rows][H][D] = merge of `parts` partials [parts][rows][H][D + 2] with the sink and the inverse
// rotation.
cudaError_t launch_attend_merge(const LayerArgs& L, const float* sinks, const int64_t* q_pos, int rows, int parts,
                                const float* partials, uint8_t* out, cudaStream_t s);

}  // namespace csa
