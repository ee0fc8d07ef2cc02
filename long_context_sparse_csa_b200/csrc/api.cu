// C ABI of the CSA/HCA operator: argument checks, workspace layout, launches.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <climits>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "csa.h"
#include "kernels.h"

using namespace csa;

namespace {

thread_local std::string g_err;
thread_local cudaEvent_t g_prof_start = nullptr, g_prof_stop = nullptr;
thread_local cudaEvent_t* g_tl = nullptr;
thread_local int g_tl_cap = 0, g_tl_n = 0;
std::atomic<uint64_t> g_launches{0};

csa_status_t fail(csa_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

csa_status_t cuda_fail(cudaError_t e, const char* where) {
  return fail(CSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  static int cached[64] = {0};
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

// A second stream per (thread, device) for the CSA decode step's fork/join: compression does not
// feed the indexer (index keys are inputs), so append+compress runs beside indexer + top-k and
// joins before attention.  Created on first use outside stream capture; nullptr means "run in
// sequence on the caller's stream" (creation failed, the caller is capturing before the first
// eager call, or a launch timeline is armed: its intervals then stay one kernel each).
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  bool failed = false;
};
thread_local SideStream g_side[64];

SideStream* side_stream(cudaStream_t main) {
  if (g_tl) return nullptr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  SideStream& ss = g_side[dev];
  if (ss.s) return &ss;
  if (ss.failed) return nullptr;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(main, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone) {
    cudaGetLastError();
    return nullptr;
  }
  if (cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess) {
    cudaGetLastError();
    if (ss.s) cudaStreamDestroy(ss.s);
    if (ss.fork) cudaEventDestroy(ss.fork);
    if (ss.join) cudaEventDestroy(ss.join);
    ss = SideStream();
    ss.failed = true;
    return nullptr;
  }
  return &ss;
}

size_t row_bytes_of(const csa_layer_t* L) {
  switch (L->kv_format) {
    case CSA_FMT_F32: return 4 * (size_t)L->D;
    case CSA_FMT_BF16: return 2 * (size_t)L->D;
    case CSA_FMT_MIXED: return (size_t)L->D + 80;
    default: return 0;
  }
}

csa_status_t check_layer(const csa_layer_t* L) {
  if (!L) return fail(CSA_ERR_INVALID_ARG, "layer is NULL");
  if (L->kind != CSA_KIND_CSA && L->kind != CSA_KIND_HCA) return fail(CSA_ERR_INVALID_ARG, "kind %d", L->kind);
  if (L->B < 1 || L->H < 1) return fail(CSA_ERR_INVALID_ARG, "B=%d H=%d", L->B, L->H);
  if (L->D < 128 || L->D > 1024 || L->D % 128) return fail(CSA_ERR_UNSUPPORTED, "D=%d (needs a multiple of 128, <= 1024)", L->D);
  if (L->d_rope != 64) return fail(CSA_ERR_UNSUPPORTED, "d_rope=%d (only 64)", L->d_rope);
  if (L->m < 1) return fail(CSA_ERR_INVALID_ARG, "m=%d", L->m);
  if (L->overlap != 0 && L->overlap != 1) return fail(CSA_ERR_INVALID_ARG, "overlap=%d", L->overlap);
  if (L->window < 1) return fail(CSA_ERR_INVALID_ARG, "window=%d", L->window);
  if (L->kv_format != CSA_FMT_F32 && L->kv_format != CSA_FMT_BF16 && L->kv_format != CSA_FMT_MIXED)
    return fail(CSA_ERR_INVALID_ARG, "kv_format=%d", L->kv_format);
  if (L->act_format != CSA_FMT_F32 && L->act_format != CSA_FMT_BF16)
    return fail(CSA_ERR_INVALID_ARG, "act_format=%d", L->act_format);
  if (!(L->rope_base > 0)) return fail(CSA_ERR_INVALID_ARG, "rope_base must be > 0");
  if (!(L->eps >= 0)) return fail(CSA_ERR_INVALID_ARG, "eps must be >= 0");
  if (L->kind == CSA_KIND_CSA) {
    if (L->top_k < 1) return fail(CSA_ERR_INVALID_ARG, "top_k=%d", L->top_k);
    if (L->H_I < 1 || L->d_I < 1) return fail(CSA_ERR_INVALID_ARG, "H_I=%d d_I=%d", L->H_I, L->d_I);
    if (L->idx_format != CSA_FMT_F32 && L->idx_format != CSA_FMT_E4M3 && L->idx_format != CSA_FMT_E2M1)
      return fail(CSA_ERR_INVALID_ARG, "idx_format=%d", L->idx_format);
    if (L->d_I % 16) return fail(CSA_ERR_UNSUPPORTED, "d_I=%d (needs a multiple of 16)", L->d_I);
    if (L->idx_format == CSA_FMT_E2M1 && L->d_I % 32)
      return fail(CSA_ERR_UNSUPPORTED, "d_I=%d (FP4 keys need a multiple of 32)", L->d_I);
    if ((size_t)L->H_I * L->d_I * 4 > 96 * 1024) return fail(CSA_ERR_UNSUPPORTED, "H_I*d_I too large");
  }
  return CSA_OK;
}

LayerArgs layer_args(const csa_layer_t* L) {
  LayerArgs a;
  a.B = L->B; a.H = L->H; a.D = L->D; a.d_rope = L->d_rope; a.m = L->m; a.ov = L->overlap;
  a.top_k = L->top_k; a.window = L->window; a.H_I = L->H_I; a.d_I = L->d_I;
  a.kv_fmt = L->kv_format; a.idx_fmt = L->idx_format; a.act_fmt = L->act_format;
  a.row_bytes = (int)row_bytes_of(L);
  a.rope_base = L->rope_base;
  a.eps = L->eps;
  a.scale = L->softmax_scale > 0 ? L->softmax_scale : 1.0f / sqrtf((float)L->D);
  a.pos0 = L->pos0;
  for (int u = 0; u < 32; ++u)
    a.theta_pi[u] = u < L->d_rope / 2 ? std::pow(L->rope_base, -2.0 * u / (double)L->d_rope) / M_PI : 0.0;
  return a;
}

CacheArgs cache_args(const csa_cache_t* c) {
  CacheArgs a;
  a.entries = static_cast<uint8_t*>(c->entries);
  a.entry_cap = c->entry_cap;
  a.idx_keys = static_cast<const uint8_t*>(c->idx_keys);
  a.idx_key_scale = c->idx_key_scale;
  a.window = static_cast<uint8_t*>(c->window);
  a.window_cap = c->window_cap;
  a.raw = static_cast<uint8_t*>(c->raw);
  a.gate = static_cast<uint8_t*>(c->gate);
  a.raw_cap = c->raw_cap;
  a.raw_base = c->raw_base;
  return a;
}

csa_status_t need_ptr(const void* p, const char* name, size_t align = 16) {
  if (!p) return fail(CSA_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned(p, align)) return fail(CSA_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
  return CSA_OK;
}

#define CSA_TRY(x)                     \
  do {                                 \
    csa_status_t _st = (x);            \
    if (_st != CSA_OK) return _st;     \
  } while (0)

csa_status_t check_cache_attend(const csa_layer_t* L, const csa_cache_t* c) {
  if (!c) return fail(CSA_ERR_INVALID_ARG, "cache is NULL");
  CSA_TRY(need_ptr(c->entries, "cache.entries"));
  CSA_TRY(need_ptr(c->window, "cache.window"));
  if (c->entry_cap < 1) return fail(CSA_ERR_INVALID_ARG, "entry_cap=%lld", (long long)c->entry_cap);
  if (c->window_cap < L->window) return fail(CSA_ERR_INVALID_ARG, "window_cap < window");
  return CSA_OK;
}

csa_status_t check_cache_raw(const csa_layer_t* L, const csa_cache_t* c, bool need_gate) {
  CSA_TRY(need_ptr(c->raw, "cache.raw"));
  if (need_gate) CSA_TRY(need_ptr(c->gate, "cache.gate"));
  if (c->raw_cap < 1) return fail(CSA_ERR_INVALID_ARG, "raw_cap=%lld", (long long)c->raw_cap);
  (void)L;
  return CSA_OK;
}

// ----------------------------------------------------------------------------- workspace layout
constexpr size_t kAlign = 256;

// Long decode rows take the multi-CTA top-k, fed by the decode indexer's score histogram.
bool use_split_topk(const csa_layer_t* L, int32_t Tq, int64_t n_max) {
  return Tq == 1 && n_max >= kTopkSplitMinN && n_max <= kTopkSplitMaxN &&
         index_decode_supported(L->idx_format, L->H_I, L->d_I);
}
size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Workspace {
  size_t err = 0;          // int error word
  size_t hist = 0, hist_bytes = 0;      // split top-k: histogram [rows][4096], counters [rows][4], histogram 2 [rows][4096]
  size_t counts = 0, list = 0;          // split top-k scratch
  size_t scores = 0, scores_bytes = 0;
  size_t topk = 0, topk_bytes = 0;
  size_t part = 0, part_bytes = 0;
  size_t qt = 0;                        // bf16 q~ of the tcgen05 attention [rows][H][D]
  size_t extra = 0;                     // HCA decode: logits of the deferred rows [rows][2][H] fp32
  size_t idxq = 0, idxqs = 0;           // indexed decode step: produced index query and its scales
  size_t total = 0;
};

Workspace layout(const csa_layer_t* L, int op, int32_t Tq, int64_t n_max) {
  Workspace w;
  const LayerArgs la = layer_args(L);
  const size_t rows = (size_t)L->B * (size_t)(Tq > 0 ? Tq : 1);
  size_t off = up(64);
  const bool csa = L->kind == CSA_KIND_CSA;
  const bool step = op == CSA_OP_DECODE_STEP || op == CSA_OP_DECODE_STEP_INDEXED;
  if (csa && (op == CSA_OP_INDEX_TOPK || step || op == CSA_OP_PREFILL)) {
    w.scores = off; w.scores_bytes = rows * (size_t)(n_max > 0 ? n_max : 1) * 4; off = up(off + w.scores_bytes);
    if (use_split_topk(L, Tq, n_max)) {
      w.hist = off; w.hist_bytes = rows * (4096 + 4 + 4096) * 4; off = up(off + w.hist_bytes);
      w.counts = off; off = up(off + rows * (size_t)kTopkSplitMaxCtas * 4);
      w.list = off; off = up(off + rows * (size_t)n_max * 8);
    }
  }
  if (csa && (step || op == CSA_OP_PREFILL)) {
    w.topk = off; w.topk_bytes = rows * (size_t)L->top_k * 4; off = up(off + w.topk_bytes);
  }
  if (csa && op == CSA_OP_DECODE_STEP_INDEXED) {
    const size_t qb = L->idx_format == CSA_FMT_F32 ? 4 : 1;
    w.idxq = off; off = up(off + rows * (size_t)L->H_I * L->d_I * qb);
    w.idxqs = off; off = up(off + rows * (size_t)L->H_I * 4);
  }
  if (op == CSA_OP_SPARSE_ATTEND || op == CSA_OP_HCA_ATTEND || step || op == CSA_OP_PREFILL) {
    const bool dense = (op == CSA_OP_HCA_ATTEND) || !csa;
    const int64_t slots = (dense ? (n_max > 0 ? n_max : 1) : (int64_t)L->top_k) + L->window;
    const int splits = attend_num_splits(la, dense, (int)rows, slots, num_sms());
    w.part = off; w.part_bytes = attend_partial_bytes(la, dense, (int)rows, splits); off = up(off + w.part_bytes);
    const int ap = attend_path(la, dense, (int)rows);
    if (ap == 2 || ap == 3) { w.qt = off; off = up(off + rows * (size_t)L->H * L->D * 2); }
    if (attend_path(la, dense, (int)rows) == 2 && dense) {
      w.extra = off; off = up(off + rows * 2 * (size_t)L->H * 4);
    }
  }
  w.total = off;
  return w;
}

csa_status_t check_ws(const Workspace& w, void* ws, size_t ws_bytes) {
  if (!ws) return fail(CSA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", w.total);
  if (!aligned(ws, kAlign)) return fail(CSA_ERR_WORKSPACE, "workspace must be %zu-byte aligned", kAlign);
  if (ws_bytes < w.total) return fail(CSA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, w.total);
  return CSA_OK;
}

uint8_t* at(void* ws, size_t off) { return static_cast<uint8_t*>(ws) + off; }

// ----------------------------------------------------------------------------- step bodies
csa_status_t run_append_compress(const csa_layer_t* L, const csa_cache_t* cache, const csa_params_t* P,
                                 const void* x_new, const void* g_new, const int64_t* q_pos, int32_t Tq,
                                 bool do_append, bool do_compress, int* err, cudaStream_t s) {
  AppendCompressArgs a;
  a.L = layer_args(L);
  a.C = cache_args(cache);
  a.q_pos = q_pos;
  a.Tq = Tq;
  a.x_new = static_cast<const uint8_t*>(x_new);
  a.g_new = static_cast<const uint8_t*>(g_new);
  a.pos_bias = P ? P->pos_bias : nullptr;
  a.gamma_kv = P ? P->gamma_kv : nullptr;
  a.do_append = do_append;
  a.do_compress = do_compress;
  a.err = err;
  cudaError_t e = launch_append_compress(a, L->B, Tq, s);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e, "append/compress launch");
}

csa_status_t run_index_topk(const csa_layer_t* L, const csa_cache_t* cache, const void* idx_q,
                            const float* idx_q_scale, const float* head_w, const int64_t* q_pos, int32_t Tq,
                            int64_t n_max, int32_t* topk, float* scores, const Workspace& w, void* ws,
                            cudaStream_t s) {
  int* err = reinterpret_cast<int*>(at(ws, w.err));
  const bool split = use_split_topk(L, Tq, n_max);
  const int rows = L->B * Tq;
  // the split top-k leaves its histogram and counters zeroed; the caller zero-fills the workspace once
  uint32_t* hist = split ? reinterpret_cast<uint32_t*>(at(ws, w.hist)) : nullptr;
  IndexArgs a;
  memset(&a, 0, sizeof(a));
  a.B = L->B; a.Tq = Tq; a.H_I = L->H_I; a.d_I = L->d_I; a.m = L->m;
  a.idx_fmt = L->idx_format;
  a.n_max = n_max; a.entry_cap = cache->entry_cap; a.pos0 = L->pos0;
  a.q_pos = q_pos;
  a.idx_q = static_cast<const uint8_t*>(idx_q);
  a.idx_k = static_cast<const uint8_t*>(cache->idx_keys);
  a.k_scale = cache->idx_key_scale;
  a.q_scale = idx_q_scale;
  a.head_w = head_w;
  a.scores = scores;
  a.hist = hist;
  a.err = err;
  const bool prof = g_prof_start && g_prof_stop;
  if (prof) cudaEventRecordWithFlags(g_prof_start, s, cudaEventRecordExternal);
  cudaError_t e = launch_index_scores(a, num_sms(), s);
  if (prof) cudaEventRecordWithFlags(g_prof_stop, s, cudaEventRecordExternal);
  if (e != cudaSuccess) return cuda_fail(e, "index-score launch");
  TopkArgs t;
  t.scores = scores; t.n_max = n_max; t.rows = rows; t.Tq = Tq; t.m = L->m; t.k = L->top_k;
  t.pos0 = L->pos0; t.q_pos = q_pos; t.out = topk;
  t.map = nullptr; t.shards = 1;
  if (split) {
    TopkSplitArgs sa;
    sa.base = t;
    sa.hist = hist;
    sa.cnt = hist + (size_t)rows * 4096;
    sa.hist2 = sa.cnt + (size_t)rows * 4;
    sa.counts = reinterpret_cast<uint32_t*>(at(ws, w.counts));
    sa.list = reinterpret_cast<uint2*>(at(ws, w.list));
    sa.G = topk_split_ctas(rows, n_max, num_sms());
    sa.err = err;
    e = launch_topk_split(sa, s);
  } else {
    e = launch_topk(t, s);
  }
  return e == cudaSuccess ? CSA_OK : cuda_fail(e, "top-k launch");
}

csa_status_t make_attend_args(const csa_layer_t* L, const csa_cache_t* cache, const csa_params_t* P, const void* q,
                              const int64_t* q_pos, int32_t Tq, const int32_t* topk, int64_t n_max, void* out,
                              const Workspace& w, void* ws, AttendArgs& a) {
  a.L = layer_args(L);
  if (attend_path(a.L, topk == nullptr, L->B * Tq) == 0 && L->H > 32)
    return fail(CSA_ERR_UNSUPPORTED, "attention: H=%d needs D=512 with bf16/mixed rows and H%%32==0, or H<=32", L->H);
  a.C = cache_args(cache);
  a.q = static_cast<const uint8_t*>(q);
  a.q_pos = q_pos;
  a.Tq = Tq;
  a.rows = L->B * Tq;
  a.topk = topk;
  a.n_max = n_max;
  a.gamma_q = P->gamma_q;
  a.sinks = P->sinks;
  const int64_t slots = (topk ? (int64_t)L->top_k : n_max) + L->window;
  a.splits = attend_num_splits(a.L, topk == nullptr, a.rows, slots, num_sms());
  if (attend_partial_bytes(a.L, topk == nullptr, a.rows, a.splits) > w.part_bytes)
    return fail(CSA_ERR_WORKSPACE, "workspace too small for the attention partials");
  a.part = reinterpret_cast<float*>(at(ws, w.part));
  a.qt = w.qt ? at(ws, w.qt) : nullptr;
  a.err = reinterpret_cast<int*>(at(ws, w.err));
  a.out = static_cast<uint8_t*>(out);
  a.entry_offset = 0;
  a.entry_limit = cache->entry_cap;
  a.no_window = 0;
  a.partial_out = nullptr;
  a.defer_new = 0;
  a.extra = w.extra ? reinterpret_cast<float*>(at(ws, w.extra)) : nullptr;
  return CSA_OK;
}

// Attention, preceded by the q~ preparation unless the caller has launched it already (run_qprep).
csa_status_t run_attend(const csa_layer_t* L, const csa_cache_t* cache, const csa_params_t* P, const void* q,
                        const int64_t* q_pos, int32_t Tq, const int32_t* topk, int64_t n_max, void* out,
                        const Workspace& w, void* ws, cudaStream_t s, bool with_qprep = true) {
  AttendArgs a;
  CSA_TRY(make_attend_args(L, cache, P, q, q_pos, Tq, topk, n_max, out, w, ws, a));
  cudaError_t e = with_qprep ? launch_attend_qprep(a, s) : cudaSuccess;
  if (e == cudaSuccess) e = launch_attend(a, s);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e, "attention launch");
}

csa_status_t run_qprep(const csa_layer_t* L, const csa_cache_t* cache, const csa_params_t* P, const void* q,
                       const int64_t* q_pos, int32_t Tq, const int32_t* topk, int64_t n_max, const Workspace& w,
                       void* ws, cudaStream_t s) {
  AttendArgs a;
  CSA_TRY(make_attend_args(L, cache, P, q, q_pos, Tq, topk, n_max, nullptr, w, ws, a));
  const cudaError_t e = launch_attend_qprep(a, s);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e, "q preparation launch");
}

csa_status_t check_params(const csa_layer_t* L, const csa_params_t* P, bool need_bias) {
  if (!P) return fail(CSA_ERR_INVALID_ARG, "params is NULL");
  if (need_bias) CSA_TRY(need_ptr(P->pos_bias, "params.pos_bias"));
  if (!P->sinks && !need_bias) return fail(CSA_ERR_INVALID_ARG, "params.sinks is NULL");
  (void)L;
  return CSA_OK;
}

}  // namespace

namespace csa {
csa_status_t report_error(csa_status_t st, const char* msg) { return fail(st, "%s", msg); }

void note_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

namespace {
std::mutex g_attr_mu;
std::map<std::pair<int, const void*>, size_t> g_smem_attr;     // (device, kernel) -> bytes set
std::map<std::pair<int, const void*>, bool> g_cluster_attr;    // (device, kernel) -> allowed
}  // namespace

cudaError_t ensure_dynamic_smem(const void* kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  size_t& have = g_smem_attr[std::make_pair(dev, kernel)];
  if (bytes <= have) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) have = bytes;
  return e;
}

cudaError_t ensure_nonportable_cluster(const void* kernel) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  bool& ok = g_cluster_attr[std::make_pair(dev, kernel)];
  if (ok) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess) ok = true;
  return e;
}
void profile_mark(cudaStream_t s) {
  if (!g_tl || g_tl_n >= g_tl_cap) return;
  // under stream capture the record becomes an event node (external flag); on a stream that is
  // not being captured it is a plain record, ordered after the launches issued before it
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) cudaGetLastError();
  if (cap == cudaStreamCaptureStatusActive) cudaEventRecordWithFlags(g_tl[g_tl_n++], s, cudaEventRecordExternal);
  else cudaEventRecord(g_tl[g_tl_n++], s);
}
}  // namespace csa

// ============================================================================= exported
extern "C" {

size_t csa_row_bytes(const csa_layer_t* L) { return L ? row_bytes_of(L) : 0; }

size_t csa_workspace_size(const csa_layer_t* L, int32_t op, int32_t Tq, int64_t entry_cap) {
  if (check_layer(L) != CSA_OK) return 0;
  return layout(L, op, Tq, entry_cap).total;
}

const char* csa_last_error(void) { return g_err.c_str(); }

const char* csa_version(void) { return "csa-b200 0.1 (sm_100a)"; }

void csa_profile_events(void* ev_start, void* ev_stop) {
  g_prof_start = static_cast<cudaEvent_t>(ev_start);
  g_prof_stop = static_cast<cudaEvent_t>(ev_stop);
}

uint64_t csa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

void csa_profile_timeline(void** events, int32_t capacity) {
  g_tl = reinterpret_cast<cudaEvent_t*>(events);
  g_tl_cap = events ? capacity : 0;
  g_tl_n = 0;
}

int32_t csa_profile_timeline_count(void) { return g_tl_n; }

csa_status_t csa_device_error(void* workspace, size_t ws_bytes, void* stream, int32_t* code) {
  if (code) *code = 0;
  if (workspace && ws_bytes < 4) return fail(CSA_ERR_WORKSPACE, "workspace smaller than its error word");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* lib_word = nullptr;
  cudaError_t e = library_error_word(&lib_word);
  int32_t v[2] = {0, 0};
  if (e == cudaSuccess && workspace) e = cudaMemcpyAsync(&v[0], workspace, 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&v[1], lib_word, 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && v[0]) e = cudaMemsetAsync(workspace, 0, 4, s);
  if (e == cudaSuccess && v[1]) e = cudaMemsetAsync(lib_word, 0, 4, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "csa_device_error");
  const int32_t bits = v[0] | v[1];
  if (code) *code = bits;
  return bits ? fail(CSA_ERR_DEVICE_TIMEOUT, "device error word 0x%x", bits) : CSA_OK;
}

csa_status_t csa_debug_workspace_segment(const csa_layer_t* L, int32_t op, int32_t Tq, int64_t entry_cap,
                                         int32_t segment, size_t* offset, size_t* bytes) {
  CSA_TRY(check_layer(L));
  if (!offset || !bytes) return fail(CSA_ERR_INVALID_ARG, "offset or bytes is NULL");
  const Workspace w = layout(L, op, Tq, entry_cap);
  *offset = 0;
  *bytes = 0;
  switch (segment) {
    case CSA_SEG_ERROR_WORD: *offset = w.err; *bytes = 4; break;
    case CSA_SEG_SCORES: *offset = w.scores; *bytes = w.scores_bytes; break;
    case CSA_SEG_TOPK_HISTOGRAM: *offset = w.hist; *bytes = w.hist_bytes; break;
    case CSA_SEG_TOPK: *offset = w.topk; *bytes = w.topk_bytes; break;
    case CSA_SEG_PARTIALS: *offset = w.part; *bytes = w.part_bytes; break;
    case CSA_SEG_INDEX_QUERY:
      *offset = w.idxq;
      *bytes = w.idxq ? (size_t)L->B * L->H_I * L->d_I * (L->idx_format == CSA_FMT_F32 ? 4 : 1) : 0;
      break;
    case CSA_SEG_INDEX_QUERY_SCALE: *offset = w.idxqs; *bytes = w.idxqs ? (size_t)L->B * L->H_I * 4 : 0; break;
    default: return fail(CSA_ERR_INVALID_ARG, "segment %d", segment);
  }
  return CSA_OK;
}

csa_status_t csa_debug_wait_probe(void* workspace, size_t ws_bytes, uint64_t limit_ns, void* stream) {
  if (!workspace || ws_bytes < 4) return fail(CSA_ERR_WORKSPACE, "workspace is NULL");
  if (limit_ns == 0 || limit_ns > 1000000000ull) return fail(CSA_ERR_INVALID_ARG, "limit_ns outside (0, 1e9]");
  const cudaError_t e = launch_wait_probe(static_cast<int*>(workspace), limit_ns, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA_OK : cuda_fail(e, "wait probe launch");
}

csa_status_t csa_append(const csa_layer_t* L, const csa_cache_t* cache, const void* x_new, const void* g_new,
                        const int64_t* q_pos, int32_t Tq, void* stream) {
  CSA_TRY(check_layer(L));
  if (!cache) return fail(CSA_ERR_INVALID_ARG, "cache is NULL");
  CSA_TRY(need_ptr(cache->window, "cache.window"));
  CSA_TRY(check_cache_raw(L, cache, x_new != nullptr));
  CSA_TRY(need_ptr(q_pos, "q_pos", 8));
  if (Tq < 1) return fail(CSA_ERR_INVALID_ARG, "Tq=%d", Tq);
  if ((x_new == nullptr) != (g_new == nullptr)) return fail(CSA_ERR_INVALID_ARG, "x_new and g_new must both be given or both NULL");
  if (x_new) { CSA_TRY(need_ptr(x_new, "x_new")); CSA_TRY(need_ptr(g_new, "g_new")); }
  if (cache->window_cap < L->window) return fail(CSA_ERR_INVALID_ARG, "window_cap < window");
  int* err = nullptr;
  const cudaError_t e = library_error_word(&err);
  if (e != cudaSuccess) return cuda_fail(e, "library error word");
  return run_append_compress(L, cache, nullptr, x_new, g_new, q_pos, Tq, true, false, err,
                             static_cast<cudaStream_t>(stream));
}

csa_status_t csa_compress(const csa_layer_t* L, const csa_cache_t* cache, const csa_params_t* P,
                          const int64_t* q_pos, int32_t Tq, void* stream) {
  CSA_TRY(check_layer(L));
  if (!cache) return fail(CSA_ERR_INVALID_ARG, "cache is NULL");
  CSA_TRY(need_ptr(cache->entries, "cache.entries"));
  CSA_TRY(check_cache_raw(L, cache, true));
  CSA_TRY(check_params(L, P, true));
  CSA_TRY(need_ptr(q_pos, "q_pos", 8));
  if (Tq < 1) return fail(CSA_ERR_INVALID_ARG, "Tq=%d", Tq);
  int* err = nullptr;
  const cudaError_t e = library_error_word(&err);
  if (e != cudaSuccess) return cuda_fail(e, "library error word");
  return run_append_compress(L, cache, P, nullptr, nullptr, q_pos, Tq, false, true, err,
                             static_cast<cudaStream_t>(stream));
}

csa_status_t csa_index_topk(const csa_layer_t* L, const csa_cache_t* cache, const void* idx_q,
                            const float* idx_q_scale, const float* head_w, const int64_t* q_pos, int32_t Tq,
                            int64_t n_max, int32_t* topk_idx, float* scores, void* workspace, size_t ws_bytes,
                            void* stream) {
  CSA_TRY(check_layer(L));
  if (L->kind != CSA_KIND_CSA) return fail(CSA_ERR_INVALID_ARG, "csa_index_topk needs a CSA layer");
  if (!cache) return fail(CSA_ERR_INVALID_ARG, "cache is NULL");
  CSA_TRY(need_ptr(cache->idx_keys, "cache.idx_keys"));
  CSA_TRY(need_ptr(cache->idx_key_scale, "cache.idx_key_scale", 4));
  CSA_TRY(need_ptr(idx_q, "idx_q"));
  CSA_TRY(need_ptr(idx_q_scale, "idx_q_scale", 4));
  CSA_TRY(need_ptr(head_w, "head_w", 4));
  CSA_TRY(need_ptr(q_pos, "q_pos", 8));
  CSA_TRY(need_ptr(topk_idx, "topk_idx", 4));
  if (Tq < 1) return fail(CSA_ERR_INVALID_ARG, "Tq=%d", Tq);
  if (n_max < 0 || n_max > cache->entry_cap) return fail(CSA_ERR_INVALID_ARG, "n_max=%lld outside [0, entry_cap]", (long long)n_max);
  const Workspace w = layout(L, CSA_OP_INDEX_TOPK, Tq, n_max);
  CSA_TRY(check_ws(w, workspace, ws_bytes));
  if (scores) CSA_TRY(need_ptr(scores, "scores", 4));
  float* sc = scores ? scores : reinterpret_cast<float*>(at(workspace, w.scores));
  return run_index_topk(L, cache, idx_q, idx_q_scale, head_w, q_pos, Tq, n_max, topk_idx, sc, w, workspace,
                        static_cast<cudaStream_t>(stream));
}

csa_status_t csa_sparse_attend(const csa_layer_t* L, const csa_cache_t* cache, const csa_params_t* P,
                               const void* q, const int64_t* q_pos, int32_t Tq, const int32_t* topk_idx,
                               void* out, void* workspace, size_t ws_bytes, void* stream) {
  CSA_TRY(check_layer(L));
  if (L->kind != CSA_KIND_CSA) return fail(CSA_ERR_INVALID_ARG, "csa_sparse_attend needs a CSA layer");
  CSA_TRY(check_cache_attend(L, cache));
  CSA_TRY(check_params(L, P, false));
  CSA_TRY(need_ptr(P->sinks, "params.sinks", 4));
  CSA_TRY(need_ptr(q, "q"));
  CSA_TRY(need_ptr(q_pos, "q_pos", 8));
  CSA_TRY(need_ptr(topk_idx, "topk_idx", 4));
  CSA_TRY(need_ptr(out, "out"));
  if (Tq < 1) return fail(CSA_ERR_INVALID_ARG, "Tq=%d", Tq);
  const Workspace w = layout(L, CSA_OP_SPARSE_ATTEND, Tq, cache->entry_cap);
  CSA_TRY(check_ws(w, workspace, ws_bytes));
  return run_attend(L, cache, P, q, q_pos, Tq, topk_idx, cache->entry_cap, out, w, workspace,
                    static_cast<cudaStream_t>(stream));
}

csa_status_t hca_attend(const csa_layer_t* L, const csa_cache_t* cache, const csa_params_t* P, const void* q,
                        const int64_t* q_pos, int32_t Tq, int64_t n_max, void* out, void* workspace,
                        size_t ws_bytes, void* stream) {
  CSA_TRY(check_layer(L));
  CSA_TRY(check_cache_attend(L, cache));
  CSA_TRY(check_params(L, P, false));
  CSA_TRY(need_ptr(P->sinks, "params.sinks", 4));
  CSA_TRY(need_ptr(q, "q"));
  CSA_TRY(need_ptr(q_pos, "q_pos", 8));
  CSA_TRY(need_ptr(out, "out"));
  if (Tq < 1) return fail(CSA_ERR_INVALID_ARG, "Tq=%d", Tq);
  if (n_max < 0 || n_max > cache->entry_cap) return fail(CSA_ERR_INVALID_ARG, "n_max outside [0, entry_cap]");
  const Workspace w = layout(L, CSA_OP_HCA_ATTEND, Tq, n_max);
  CSA_TRY(check_ws(w, workspace, ws_bytes));
  return run_attend(L, cache, P, q, q_pos, Tq, nullptr, n_max, out, w, workspace, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// The CSA decode step after argument checks: append+compress and q preparation on the side stream;
// on the caller's stream the index-side production (when `prep` is given), the indexer and top-k;
// the two join before the attention.
csa_status_t csa_decode_step_run(const csa_layer_t* L, const csa_cache_t* cache, const csa_params_t* P,
                                 const void* q, const void* idx_q, const float* idx_q_scale, const float* head_w,
                                 const void* x_new, const void* g_new, const int64_t* q_pos, void* out,
                                 int32_t* topk_idx, const Workspace& w, void* workspace, cudaStream_t s,
                                 const IndexPrepArgs* prep) {
  int32_t* tk = topk_idx ? topk_idx : reinterpret_cast<int32_t*>(at(workspace, w.topk));
  int* ws_err = reinterpret_cast<int*>(at(workspace, w.err));
  float* scores = reinterpret_cast<float*>(at(workspace, w.scores));
  auto index_side = [&]() -> csa_status_t {
    if (prep) {
      const cudaError_t e = launch_index_prep(*prep, s);
      if (e != cudaSuccess) return cuda_fail(e, "index preparation launch");
    }
    return run_index_topk(L, cache, idx_q, idx_q_scale, head_w, q_pos, 1, cache->entry_cap, tk, scores, w,
                          workspace, s);
  };
  SideStream* ss = side_stream(s);
  if (ss) {
    // fork: append+compress on the side stream, indexer + top-k here; join before attention
    cudaError_t e = cudaEventRecord(ss->fork, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->s, ss->fork, 0);
    if (e != cudaSuccess) return cuda_fail(e, "csa_decode_step fork");
    csa_status_t sc = run_append_compress(L, cache, P, x_new, g_new, q_pos, 1, true, true, ws_err, ss->s);
    if (sc == CSA_OK) sc = run_qprep(L, cache, P, q, q_pos, 1, tk, cache->entry_cap, w, workspace, ss->s);
    const csa_status_t si = sc == CSA_OK ? index_side() : sc;
    // the join is recorded whatever happened, so a capture never ends with the side stream unjoined
    e = cudaEventRecord(ss->join, ss->s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ss->join, 0);
    if (si != CSA_OK) return si;
    if (e != cudaSuccess) return cuda_fail(e, "csa_decode_step join");
    return run_attend(L, cache, P, q, q_pos, 1, tk, cache->entry_cap, out, w, workspace, s, false);
  }
  CSA_TRY(run_append_compress(L, cache, P, x_new, g_new, q_pos, 1, true, true, ws_err, s));
  CSA_TRY(index_side());
  return run_attend(L, cache, P, q, q_pos, 1, tk, cache->entry_cap, out, w, workspace, s);
}

csa_status_t check_decode_common(const csa_layer_t* L, const csa_cache_t* cache, const csa_params_t* P,
                                 const void* q, const float* head_w, const void* x_new, const void* g_new,
                                 const int64_t* q_pos, void* out, int32_t* topk_idx, const char* who) {
  CSA_TRY(check_layer(L));
  if (L->kind != CSA_KIND_CSA) return fail(CSA_ERR_INVALID_ARG, "%s needs a CSA layer", who);
  CSA_TRY(check_cache_attend(L, cache));
  CSA_TRY(check_cache_raw(L, cache, true));
  CSA_TRY(need_ptr(cache->idx_keys, "cache.idx_keys"));
  CSA_TRY(need_ptr(cache->idx_key_scale, "cache.idx_key_scale", 4));
  CSA_TRY(check_params(L, P, true));
  CSA_TRY(need_ptr(P->sinks, "params.sinks", 4));
  CSA_TRY(need_ptr(q, "q"));
  CSA_TRY(need_ptr(head_w, "head_w", 4));
  CSA_TRY(need_ptr(x_new, "x_new"));
  CSA_TRY(need_ptr(g_new, "g_new"));
  CSA_TRY(need_ptr(q_pos, "q_pos", 8));
  CSA_TRY(need_ptr(out, "out"));
  if (topk_idx) CSA_TRY(need_ptr(topk_idx, "topk_idx", 4));
  if (cache->raw_cap < (1 + L->overlap) * (int64_t)L->m) return fail(CSA_ERR_INVALID_ARG, "raw_cap < (1+overlap)*m");
  return CSA_OK;
}

// Index-side arguments shared by csa_index_keys, csa_index_query and the indexed decode step.
csa_status_t check_index_side(const csa_layer_t* L, const void* c, const void* W, int32_t rank) {
  if (L->kind != CSA_KIND_CSA) return fail(CSA_ERR_INVALID_ARG, "the index side needs a CSA layer");
  if (L->d_I % 32 || L->d_I > 128) return fail(CSA_ERR_UNSUPPORTED, "d_I=%d (index production needs a multiple of 32, <= 128)", L->d_I);
  if (c || W) {
    CSA_TRY(need_ptr(c, "c", 4));
    CSA_TRY(need_ptr(W, "W", 4));
    if (rank < 16 || rank % 16) return fail(CSA_ERR_UNSUPPORTED, "rank=%d (needs a positive multiple of 16)", rank);
    if (L->act_format != CSA_FMT_BF16) return fail(CSA_ERR_UNSUPPORTED, "the index query needs bf16 latents and weights");
  }
  return CSA_OK;
}

IndexPrepArgs index_prep_args(const csa_layer_t* L, const csa_cache_t* cache, const csa_index_stream_t* S,
                              const int64_t* q_pos, int32_t Tq) {
  IndexPrepArgs a;
  memset(&a, 0, sizeof(a));
  a.B = L->B; a.Tq = Tq; a.H_I = L->H_I; a.d_I = L->d_I; a.m = L->m; a.ov = L->overlap;
  a.act_fmt = L->act_format; a.idx_fmt = L->idx_format;
  a.pos0 = L->pos0;
  a.entry_cap = cache ? cache->entry_cap : 0;
  a.raw_cap = cache ? cache->raw_cap : 0;
  a.raw_base = cache ? cache->raw_base : 0;
  a.q_pos = q_pos;
  if (S) {
    a.raw = static_cast<uint8_t*>(S->raw);
    a.gate = static_cast<uint8_t*>(S->gate);
    a.pos_bias = S->pos_bias;
  }
  return a;
}

csa_status_t check_index_stream(const csa_layer_t* L, const csa_cache_t* cache, const csa_index_stream_t* S) {
  if (!S) return fail(CSA_ERR_INVALID_ARG, "index stream is NULL");
  CSA_TRY(need_ptr(S->raw, "index_stream.raw"));
  CSA_TRY(need_ptr(S->gate, "index_stream.gate"));
  CSA_TRY(need_ptr(S->pos_bias, "index_stream.pos_bias", 4));
  CSA_TRY(need_ptr(cache->idx_keys, "cache.idx_keys"));
  CSA_TRY(need_ptr(cache->idx_key_scale, "cache.idx_key_scale", 4));
  if (cache->raw_cap < 1) return fail(CSA_ERR_INVALID_ARG, "raw_cap=%lld", (long long)cache->raw_cap);
  (void)L;
  return CSA_OK;
}

}  // namespace

extern "C" {

csa_status_t csa_decode_step(const csa_layer_t* L, const csa_cache_t* cache, const csa_params_t* P, const void* q,
                             const void* idx_q, const float* idx_q_scale, const float* head_w, const void* x_new,
                             const void* g_new, const int64_t* q_pos, void* out, int32_t* topk_idx,
                             void* workspace, size_t ws_bytes, void* stream) {
  CSA_TRY(check_decode_common(L, cache, P, q, head_w, x_new, g_new, q_pos, out, topk_idx, "csa_decode_step"));
  CSA_TRY(need_ptr(idx_q, "idx_q"));
  CSA_TRY(need_ptr(idx_q_scale, "idx_q_scale", 4));
  const Workspace w = layout(L, CSA_OP_DECODE_STEP, 1, cache->entry_cap);
  CSA_TRY(check_ws(w, workspace, ws_bytes));
  return csa_decode_step_run(L, cache, P, q, idx_q, idx_q_scale, head_w, x_new, g_new, q_pos, out, topk_idx, w,
                             workspace, static_cast<cudaStream_t>(stream), nullptr);
}

csa_status_t csa_index_keys(const csa_layer_t* L, const csa_cache_t* cache, const csa_index_stream_t* S,
                            const void* x_new, const void* g_new, const int64_t* q_pos, int32_t Tq, void* stream) {
  CSA_TRY(check_layer(L));
  if (!cache) return fail(CSA_ERR_INVALID_ARG, "cache is NULL");
  CSA_TRY(check_index_side(L, nullptr, nullptr, 0));
  CSA_TRY(check_index_stream(L, cache, S));
  CSA_TRY(need_ptr(q_pos, "q_pos", 8));
  if (Tq < 1) return fail(CSA_ERR_INVALID_ARG, "Tq=%d", Tq);
  if ((x_new == nullptr) != (g_new == nullptr)) return fail(CSA_ERR_INVALID_ARG, "x_new and g_new must both be given or both NULL");
  if (x_new) { CSA_TRY(need_ptr(x_new, "x_new", 4)); CSA_TRY(need_ptr(g_new, "g_new", 4)); }
  IndexPrepArgs a = index_prep_args(L, cache, S, q_pos, Tq);
  a.x_new = static_cast<const uint8_t*>(x_new);
  a.g_new = static_cast<const uint8_t*>(g_new);
  a.keys = static_cast<uint8_t*>(cache->idx_keys);
  a.key_scale = const_cast<float*>(cache->idx_key_scale);
  const cudaError_t e = launch_index_prep(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA_OK : cuda_fail(e, "index key launch");
}

csa_status_t csa_index_query(const csa_layer_t* L, const void* c, const void* W, int32_t rank, int32_t rows,
                             void* idx_q, float* idx_q_scale, void* stream) {
  CSA_TRY(check_layer(L));
  if (!c || !W) return fail(CSA_ERR_INVALID_ARG, "c and W are required");
  CSA_TRY(check_index_side(L, c, W, rank));
  CSA_TRY(need_ptr(idx_q, "idx_q", 4));
  CSA_TRY(need_ptr(idx_q_scale, "idx_q_scale", 4));
  if (rows < 1) return fail(CSA_ERR_INVALID_ARG, "rows=%d", rows);
  IndexPrepArgs a = index_prep_args(L, nullptr, nullptr, nullptr, 1);
  a.c = static_cast<const uint8_t*>(c);
  a.W = static_cast<const uint8_t*>(W);
  a.rank = rank;
  a.rows = rows;
  a.q_out = static_cast<uint8_t*>(idx_q);
  a.q_scale_out = idx_q_scale;
  const cudaError_t e = launch_index_prep(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA_OK : cuda_fail(e, "index query launch");
}

csa_status_t csa_decode_step_indexed(const csa_layer_t* L, const csa_cache_t* cache, const csa_params_t* P,
                                     const csa_index_stream_t* S, const void* q, const void* c, const void* W,
                                     int32_t rank, const float* head_w, const void* x_new, const void* g_new,
                                     const void* idx_x_new, const void* idx_g_new, const int64_t* q_pos, void* out,
                                     int32_t* topk_idx, void* workspace, size_t ws_bytes, void* stream) {
  CSA_TRY(check_decode_common(L, cache, P, q, head_w, x_new, g_new, q_pos, out, topk_idx,
                              "csa_decode_step_indexed"));
  if (!c || !W) return fail(CSA_ERR_INVALID_ARG, "c and W are required");
  CSA_TRY(check_index_side(L, c, W, rank));
  CSA_TRY(check_index_stream(L, cache, S));
  CSA_TRY(need_ptr(idx_x_new, "idx_x_new", 4));
  CSA_TRY(need_ptr(idx_g_new, "idx_g_new", 4));
  const Workspace w = layout(L, CSA_OP_DECODE_STEP_INDEXED, 1, cache->entry_cap);
  CSA_TRY(check_ws(w, workspace, ws_bytes));
  IndexPrepArgs a = index_prep_args(L, cache, S, q_pos, 1);
  a.x_new = static_cast<const uint8_t*>(idx_x_new);
  a.g_new = static_cast<const uint8_t*>(idx_g_new);
  a.keys = static_cast<uint8_t*>(cache->idx_keys);
  a.key_scale = const_cast<float*>(cache->idx_key_scale);
  a.c = static_cast<const uint8_t*>(c);
  a.W = static_cast<const uint8_t*>(W);
  a.rank = rank;
  a.rows = L->B;
  a.q_out = at(workspace, w.idxq);
  a.q_scale_out = reinterpret_cast<float*>(at(workspace, w.idxqs));
  return csa_decode_step_run(L, cache, P, q, a.q_out, a.q_scale_out, head_w, x_new, g_new, q_pos, out, topk_idx, w,
                             workspace, static_cast<cudaStream_t>(stream), &a);
}

csa_status_t hca_decode_step(const csa_layer_t* L, const csa_cache_t* cache, const csa_params_t* P, const void* q,
                             const void* x_new, const void* g_new, const int64_t* q_pos, void* out,
                             void* workspace, size_t ws_bytes, void* stream) {
  CSA_TRY(check_layer(L));
  CSA_TRY(check_cache_attend(L, cache));
  CSA_TRY(check_cache_raw(L, cache, true));
  CSA_TRY(check_params(L, P, true));
  CSA_TRY(need_ptr(P->sinks, "params.sinks", 4));
  CSA_TRY(need_ptr(q, "q"));
  CSA_TRY(need_ptr(x_new, "x_new"));
  CSA_TRY(need_ptr(g_new, "g_new"));
  CSA_TRY(need_ptr(q_pos, "q_pos", 8));
  CSA_TRY(need_ptr(out, "out"));
  if (cache->raw_cap < (1 + L->overlap) * (int64_t)L->m) return fail(CSA_ERR_INVALID_ARG, "raw_cap < (1+overlap)*m");
  const Workspace w = layout(L, CSA_OP_HCA_ATTEND, 1, cache->entry_cap);
  CSA_TRY(check_ws(w, workspace, ws_bytes));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* ws_err = reinterpret_cast<int*>(at(workspace, w.err));
  SideStream* ss = side_stream(s);
  if (ss && w.extra) {
    // append+compress on the side stream beside the attention over the earlier rows; the token's own
    // window row and the entry it completes join in the combine as two extra keys, their logits taken
    // on the side stream after append+compress
    AttendArgs a;
    CSA_TRY(make_attend_args(L, cache, P, q, q_pos, 1, nullptr, cache->entry_cap, out, w, workspace, a));
    a.defer_new = 1;
    cudaError_t e = cudaEventRecord(ss->fork, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->s, ss->fork, 0);
    if (e != cudaSuccess) return cuda_fail(e, "hca_decode_step fork");
    const csa_status_t sc = run_append_compress(L, cache, P, x_new, g_new, q_pos, 1, true, true, ws_err, ss->s);
    e = launch_attend_qprep(a, s);
    if (e == cudaSuccess) e = launch_attend_deferred(a, s);
    if (e == cudaSuccess) e = launch_attend_extra_logits(a, ss->s);
    if (e == cudaSuccess) e = cudaEventRecord(ss->join, ss->s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ss->join, 0);
    if (e == cudaSuccess) e = launch_attend_combine(a, s);
    if (sc != CSA_OK) return sc;
    return e == cudaSuccess ? CSA_OK : cuda_fail(e, "hca_decode_step launch");
  }
  if (ss) {
    // fork: the attention's query preparation on the side stream beside append+compress
    cudaError_t e = cudaEventRecord(ss->fork, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ss->s, ss->fork, 0);
    if (e != cudaSuccess) return cuda_fail(e, "hca_decode_step fork");
    const csa_status_t sq = run_qprep(L, cache, P, q, q_pos, 1, nullptr, cache->entry_cap, w, workspace, ss->s);
    const csa_status_t sc = run_append_compress(L, cache, P, x_new, g_new, q_pos, 1, true, true, ws_err, s);
    e = cudaEventRecord(ss->join, ss->s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ss->join, 0);
    if (sq != CSA_OK) return sq;
    if (sc != CSA_OK) return sc;
    if (e != cudaSuccess) return cuda_fail(e, "hca_decode_step join");
    return run_attend(L, cache, P, q, q_pos, 1, nullptr, cache->entry_cap, out, w, workspace, s, false);
  }
  CSA_TRY(run_append_compress(L, cache, P, x_new, g_new, q_pos, 1, true, true, ws_err, s));
  return run_attend(L, cache, P, q, q_pos, 1, nullptr, cache->entry_cap, out, w, workspace, s);
}

csa_status_t csa_shard_candidates(const csa_layer_t* L, const float* scores, int64_t n_local,
                                  const int32_t* topk_local, int64_t entry_offset, float* cand_score,
                                  int32_t* cand_idx, void* stream) {
  CSA_TRY(check_layer(L));
  if (L->kind != CSA_KIND_CSA) return fail(CSA_ERR_INVALID_ARG, "csa_shard_candidates needs a CSA layer");
  CSA_TRY(need_ptr(scores, "scores", 4));
  CSA_TRY(need_ptr(topk_local, "topk_local", 4));
  CSA_TRY(need_ptr(cand_score, "cand_score", 4));
  CSA_TRY(need_ptr(cand_idx, "cand_idx", 4));
  if (n_local < 0 || entry_offset < 0 || entry_offset + n_local > INT32_MAX)
    return fail(CSA_ERR_INVALID_ARG, "n_local=%lld entry_offset=%lld", (long long)n_local, (long long)entry_offset);
  const cudaError_t e = launch_shard_candidates(scores, n_local, topk_local, L->B, L->top_k, entry_offset, cand_score,
                                                cand_idx, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA_OK : cuda_fail(e, "shard candidates launch");
}

csa_status_t csa_shard_select(const csa_layer_t* L, int32_t shards, const float* cand_score, const int32_t* cand_idx,
                              int32_t* topk_idx, void* stream) {
  CSA_TRY(check_layer(L));
  if (L->kind != CSA_KIND_CSA) return fail(CSA_ERR_INVALID_ARG, "csa_shard_select needs a CSA layer");
  CSA_TRY(need_ptr(cand_score, "cand_score", 4));
  CSA_TRY(need_ptr(cand_idx, "cand_idx", 4));
  CSA_TRY(need_ptr(topk_idx, "topk_idx", 4));
  if (shards < 1 || (int64_t)shards * L->top_k > 262144) return fail(CSA_ERR_INVALID_ARG, "shards=%d", shards);
  TopkArgs t;
  memset(&t, 0, sizeof(t));
  t.scores = cand_score;
  t.n_max = (int64_t)shards * L->top_k;
  t.rows = L->B; t.Tq = 1; t.m = L->m; t.k = L->top_k; t.pos0 = L->pos0;
  t.out = topk_idx;
  t.map = cand_idx;
  t.shards = shards;
  const cudaError_t e = launch_topk(t, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA_OK : cuda_fail(e, "shard select launch");
}

csa_status_t csa_sparse_attend_partial(const csa_layer_t* L, const csa_cache_t* cache, const csa_params_t* P,
                                       const void* q, const int64_t* q_pos, const int32_t* topk_idx,
                                       int64_t entry_offset, int32_t with_window, float* partial, void* workspace,
                                       size_t ws_bytes, void* stream) {
  CSA_TRY(check_layer(L));
  if (L->kind != CSA_KIND_CSA) return fail(CSA_ERR_INVALID_ARG, "csa_sparse_attend_partial needs a CSA layer");
  CSA_TRY(check_cache_attend(L, cache));
  CSA_TRY(check_params(L, P, false));
  CSA_TRY(need_ptr(q, "q"));
  CSA_TRY(need_ptr(q_pos, "q_pos", 8));
  CSA_TRY(need_ptr(topk_idx, "topk_idx", 4));
  CSA_TRY(need_ptr(partial, "partial", 8));
  if (entry_offset < 0) return fail(CSA_ERR_INVALID_ARG, "entry_offset=%lld", (long long)entry_offset);
  if (attend_path(layer_args(L), false, L->B) != 2)
    return fail(CSA_ERR_UNSUPPORTED, "partial attention needs H=128, D=512, bf16 or mixed rows and B <= 8");
  const Workspace w = layout(L, CSA_OP_SPARSE_ATTEND, 1, cache->entry_cap);
  CSA_TRY(check_ws(w, workspace, ws_bytes));
  AttendArgs a;
  csa_params_t p = *P;
  if (!p.sinks) {
    static const float zero = 0.f;     // not read on this path (no sink in a partial)
    p.sinks = &zero;
  }
  CSA_TRY(make_attend_args(L, cache, &p, q, q_pos, 1, topk_idx, cache->entry_cap, nullptr, w, workspace, a));
  a.entry_offset = entry_offset;
  a.entry_limit = cache->entry_cap;
  a.no_window = with_window ? 0 : 1;
  a.partial_out = partial;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_attend_qprep(a, s);
  if (e == cudaSuccess) e = launch_attend(a, s);
  return e == cudaSuccess ? CSA_OK : cuda_fail(e, "partial attention launch");
}

csa_status_t csa_attend_merge(const csa_layer_t* L, const csa_params_t* P, const int64_t* q_pos, int32_t parts,
                              const float* partials, void* out, void* stream) {
  CSA_TRY(check_layer(L));
  if (!P) return fail(CSA_ERR_INVALID_ARG, "params is NULL");
  CSA_TRY(need_ptr(P->sinks, "params.sinks", 4));
  CSA_TRY(need_ptr(q_pos, "q_pos", 8));
  CSA_TRY(need_ptr(partials, "partials", 8));
  CSA_TRY(need_ptr(out, "out"));
  if (parts < 1) return fail(CSA_ERR_INVALID_ARG, "parts=%d", parts);
  const LayerArgs la = layer_args(L);
  const cudaError_t e = launch_attend_merge(la, P->sinks, q_pos, L->B, parts, partials, static_cast<uint8_t*>(out),
                                            static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA_OK : cuda_fail(e, "attention merge launch");
}

csa_status_t csa_prefill(const csa_layer_t* L, const csa_cache_t* cache, const csa_params_t* P, const void* q,
                         const void* idx_q, const float* idx_q_scale, const float* head_w, const int64_t* q_pos,
                         int32_t Tq, int64_t n_max, void* out, int32_t* topk_idx, void* workspace, size_t ws_bytes,
                         void* stream) {
  CSA_TRY(check_layer(L));
  CSA_TRY(check_cache_attend(L, cache));
  CSA_TRY(check_cache_raw(L, cache, true));
  CSA_TRY(check_params(L, P, true));
  CSA_TRY(need_ptr(P->sinks, "params.sinks", 4));
  CSA_TRY(need_ptr(q, "q"));
  CSA_TRY(need_ptr(q_pos, "q_pos", 8));
  CSA_TRY(need_ptr(out, "out"));
  if (Tq < 1) return fail(CSA_ERR_INVALID_ARG, "Tq=%d", Tq);
  if (n_max < 0 || n_max > cache->entry_cap) return fail(CSA_ERR_INVALID_ARG, "n_max outside [0, entry_cap]");
  if (cache->window_cap < (int64_t)Tq + L->window - 1)
    return fail(CSA_ERR_INVALID_ARG, "window_cap must hold Tq + window - 1 rows for a chunk");
  const bool csa = L->kind == CSA_KIND_CSA;
  if (csa) {
    CSA_TRY(need_ptr(cache->idx_keys, "cache.idx_keys"));
    CSA_TRY(need_ptr(cache->idx_key_scale, "cache.idx_key_scale", 4));
    CSA_TRY(need_ptr(idx_q, "idx_q"));
    CSA_TRY(need_ptr(idx_q_scale, "idx_q_scale", 4));
    CSA_TRY(need_ptr(head_w, "head_w", 4));
    if (topk_idx) CSA_TRY(need_ptr(topk_idx, "topk_idx", 4));
  }
  const Workspace w = layout(L, CSA_OP_PREFILL, Tq, n_max);
  CSA_TRY(check_ws(w, workspace, ws_bytes));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* ws_err = reinterpret_cast<int*>(at(workspace, w.err));
  CSA_TRY(run_append_compress(L, cache, P, nullptr, nullptr, q_pos, Tq, true, true, ws_err, s));
  int32_t* tk = nullptr;
  if (csa) {
    tk = topk_idx ? topk_idx : reinterpret_cast<int32_t*>(at(workspace, w.topk));
    CSA_TRY(run_index_topk(L, cache, idx_q, idx_q_scale, head_w, q_pos, Tq, n_max, tk,
                           reinterpret_cast<float*>(at(workspace, w.scores)), w, workspace, s));
  }
  return run_attend(L, cache, P, q, q_pos, Tq, tk, n_max, out, w, workspace, s);
}

}  // extern "C"
