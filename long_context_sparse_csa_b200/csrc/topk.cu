// Top-k selection of indexer scores: the k largest scores among a query's
// visible entries, ties to the smaller entry index, emitted in ascending
// entry order and padded with -1.  "Keep the k highest-scoring blocks"
// ("DeepSeek-V4, explained.", step 4); "a top-k selector keeps only the best
// ones for core attention" ("DeepSeek-V4: Making a Million Tokens
// Affordable", section "Two ways to shrink attention, interleaved").
//
// One 1024-thread CTA per query row runs a radix select on the
// order-preserving 32-bit image of the scores (11 + 11 + 10 bits, shared-
// memory histograms), which pins the k-th largest key T and how many keys
// equal to T are taken; a final pass over the row in index order writes the
// selection with one block-wide scan per 1024 indices, so the output order
// (ascending index) and the tie rule come out deterministic.  Rows up to
// kSmemKeys scores are staged once in shared memory.
#include "kernels.h"

namespace csa {

namespace {

constexpr int kThreads = 1024;
constexpr int kSmemKeys = 40960;     // 160 KB of keys

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// Exclusive block scan (blockDim.x a multiple of 32); *total = sum over the block.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* wsum, uint32_t* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const uint32_t inc = warp_incl_scan(v, lane);
  if (lane == 31) wsum[wid] = inc;
  __syncthreads();
  if (wid == 0) {
    uint32_t x = lane < nwarps ? wsum[lane] : 0u;
    x = warp_incl_scan(x, lane);
    wsum[lane] = x;
  }
  __syncthreads();
  const uint32_t before = wid > 0 ? wsum[wid - 1] : 0u;
  *total = wsum[nwarps - 1];
  __syncthreads();
  return before + inc - v;
}

// Among the bins nb-1 .. 0 (descending), the bin b with above(b) < need <= above(b) + hist[b],
// where above(b) counts the bins above b.  Every thread gets (bin, above).
__device__ __forceinline__ void find_bin(const uint32_t* hist, int nb, uint32_t need, uint32_t* wsum,
                                         uint32_t* s_bin, uint32_t* s_above) {
  constexpr int kMaxPer = 8;                 // nb <= 8 * blockDim.x
  const int per = (nb + blockDim.x - 1) / blockDim.x;
  uint32_t c[kMaxPer];
#pragma unroll
  for (int q = 0; q < kMaxPer; ++q) {        // all loads first (hist may live in global memory)
    const int bin = nb - 1 - per * (int)threadIdx.x - q;
    c[q] = (q < per && bin >= 0) ? hist[bin] : 0u;
  }
  uint32_t c_local = 0;
#pragma unroll
  for (int q = 0; q < kMaxPer; ++q) c_local += c[q];
  uint32_t tot;
  uint32_t above = block_excl_scan(c_local, wsum, &tot);
#pragma unroll
  for (int q = 0; q < kMaxPer; ++q) {
    const int bin = nb - 1 - per * (int)threadIdx.x - q;
    if (q < per && bin >= 0) {
      if (above < need && need <= above + c[q]) { *s_bin = (uint32_t)bin; *s_above = above; }
      above += c[q];
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads, 1) topk_rows_kernel(const __grid_constant__ TopkArgs a, int use_smem) {
  extern __shared__ uint32_t keys_sm[];
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t wsum[32];
  __shared__ uint32_t sel_bin, sel_above;

  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t t = a.q_pos[row];
  const int64_t r1 = t - a.pos0 + 1;
  int64_t nv = r1 > 0 ? r1 / a.m : 0;
  if (nv > a.n_max) nv = a.n_max;
  int32_t* out = a.out + (size_t)row * a.k;
  const float* sc = a.scores + (size_t)row * a.n_max;

  if (nv <= a.k) {
    for (int i = tid; i < a.k; i += kThreads) out[i] = i < nv ? i : -1;
    return;
  }
  const int n = (int)nv;
  if (use_smem) {
    for (int i = tid; i < n; i += kThreads) keys_sm[i] = float_key(sc[i]);
    __syncthreads();
  }
  auto key_at = [&](int i) -> uint32_t { return use_smem ? keys_sm[i] : float_key(__ldg(sc + i)); };

  // ------------------------------------------------------------------ radix select of the k-th largest key
  uint32_t prefix = 0;        // fixed high bits of T
  int fixed = 0;              // number of fixed high bits
  uint32_t remaining = (uint32_t)a.k;
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int wbits = widths[pass];
    const int shift = 32 - fixed - wbits;
    const int nb = 1 << wbits;
    for (int i = tid; i < nb; i += kThreads) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kThreads) {
      const uint32_t k = key_at(i);
      if (fixed == 0 || (k >> (32 - fixed)) == prefix) atomicAdd(&hist[(k >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    find_bin(hist, nb, remaining, wsum, &sel_bin, &sel_above);
    remaining -= sel_above;
    prefix = (prefix << wbits) | sel_bin;
    fixed += wbits;
    __syncthreads();
  }
  const uint32_t T = prefix;  // exact 32-bit key of the k-th largest score

  // ------------------------------------------------------------------ ordered emission
  uint32_t gt_run = 0, eq_run = 0;
  for (int base = 0; base < n; base += kThreads) {
    const int i = base + tid;
    uint32_t gt = 0, eq = 0;
    if (i < n) {
      const uint32_t k = key_at(i);
      gt = k > T;
      eq = k == T;
    }
    uint32_t tot;
    const uint32_t ex = block_excl_scan(gt | (eq << 16), wsum, &tot);
    const uint32_t gt_before = gt_run + (ex & 0xFFFFu);
    const uint32_t eq_before = eq_run + (ex >> 16);
    if (gt || (eq && eq_before < remaining)) {
      const uint32_t pos = gt_before + min(eq_before, remaining);
      out[pos] = i;
    }
    gt_run += tot & 0xFFFFu;
    eq_run += tot >> 16;
  }
}


// ----------------------------------------------------------------------------- split mode (long decode rows)
// Many CTAs per row.  The indexer epilogue has already histogrammed the top 12 key bits of the
// row's visible scores; every CTA finds the bin b* that holds the k-th largest key, then streams
// its slice of the row: keys above b* are certainly selected (appended to `sure`), keys in b* are
// candidates (appended to `cand`).  The last CTA of the row to finish (a ticket counter, no
// waiting) resolves the candidates with two 10-bit radix passes, marks the selection in a
// shared-memory bitmap over the row's indices, and emits it in ascending index order.
#ifdef CSA_TRACE
__device__ uint64_t g_trace_t[80][24];
#define TTRACE(slot) do { if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.x < 80) { \
    uint64_t _t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(_t) :: "memory"); g_trace_t[blockIdx.x][(slot)] = _t; } } while (0)
#else
#define TTRACE(slot) ((void)0)
#endif

constexpr int kSplitThreads = 512;
constexpr int kHistBins = 4096;
constexpr int kChunk = 4096;                  // scores per filtering chunk
constexpr int kCandCap = 4096;                // candidates staged in shared memory by the resolving CTA

__global__ void __launch_bounds__(kSplitThreads, 1) topk_split_kernel(const __grid_constant__ TopkSplitArgs a) {
  extern __shared__ uint32_t bm[];              // filtering: chunk buffers; last CTA: sel[nw] | eq[nw]
  __shared__ uint32_t h2[1024];
  __shared__ uint32_t wsum[32];
  __shared__ uint32_t s_bin, s_above, s_last, s_ns, s_nc, s_gs, s_gc;
  const TopkArgs& A = a.base;
  const int row = blockIdx.y, g = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
  const int64_t t = A.q_pos[row];
  const int64_t r1 = t - A.pos0 + 1;
  int64_t nv64 = r1 > 0 ? r1 / A.m : 0;
  if (nv64 > A.n_max) nv64 = A.n_max;
  const int nv = (int)nv64;
  const int k = A.k;
  int32_t* out = A.out + (size_t)row * k;
  uint32_t* hist_row = const_cast<uint32_t*>(a.hist) + (size_t)row * kHistBins;
  if (nv <= k) {
    if (g == 0) {
      for (int i = tid; i < k; i += kSplitThreads) out[i] = i < nv ? i : -1;
      for (int i = tid; i < kHistBins; i += kSplitThreads) hist_row[i] = 0u;   // leave it zeroed for the next call
    }
    return;
  }
  uint32_t* cnt = a.cnt + (size_t)row * 4;
  int32_t* sure = a.sure + (size_t)row * k;
  uint2* cand = a.cand + (size_t)row * A.n_max;

  TTRACE(0);
  // ---------------------------------------------------------------- 1. bin of the k-th largest key
  find_bin(a.hist + (size_t)row * kHistBins, kHistBins, (uint32_t)k, wsum, &s_bin, &s_above);
  const uint32_t bstar = s_bin;
  TTRACE(1);

  // ---------------------------------------------------------------- 2. filter this CTA's slice
  // Chunks of kChunk scores: appends go to shared-memory buffers, then one global atomic per
  // counter reserves the chunk's space in `sure` / `cand`.
  const int lo = (int)((int64_t)nv * g / gridDim.x), hi = (int)((int64_t)nv * (g + 1) / gridDim.x);
  const float* sc = A.scores + (size_t)row * A.n_max;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int32_t* b_sure = reinterpret_cast<int32_t*>(bm);             // [kChunk]
  uint2* b_cand = reinterpret_cast<uint2*>(bm + kChunk);         // [kChunk]
  for (int cb = lo; cb < hi; cb += kChunk) {
    if (tid == 0) { s_ns = 0u; s_nc = 0u; }
    __syncthreads();
    const int ce = min(cb + kChunk, hi);
    constexpr int kPer = kChunk / kSplitThreads;
    float vals[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = cb + tid * kPer + u;           // a thread's kPer consecutive scores
      vals[u] = i < ce ? __ldg(sc + i) : 0.f;
    }
    uint32_t keys[kPer], ns = 0, nc2 = 0;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = cb + tid * kPer + u;
      keys[u] = float_key(vals[u]);
      const uint32_t bin = keys[u] >> 20;
      ns += (i < ce && bin > bstar);
      nc2 += (i < ce && bin == bstar);
    }
    uint32_t tot2;
    const uint32_t ex = block_excl_scan(ns | (nc2 << 16), wsum, &tot2);
    uint32_t ps = ex & 0xFFFFu, pc = ex >> 16;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = cb + tid * kPer + u;
      const uint32_t bin = keys[u] >> 20;
      if (i < ce && bin > bstar) b_sure[ps++] = i;
      if (i < ce && bin == bstar) b_cand[pc++] = make_uint2(keys[u], (uint32_t)i);
    }
    if (tid == 0) { s_ns = tot2 & 0xFFFFu; s_nc = tot2 >> 16; }
    __syncthreads();
    if (tid == 0) {
      s_gs = s_ns ? atomicAdd(cnt + 0, s_ns) : 0u;
      s_gc = s_nc ? atomicAdd(cnt + 1, s_nc) : 0u;
      // a consistent histogram keeps every append in range; anything else is reported, not written
      if (s_gs + s_ns > (uint32_t)k || s_gc + s_nc > (uint32_t)A.n_max) {
        set_device_error(a.err, kErrTopkOverflow);
        s_ns = 0u;
        s_nc = 0u;
      }
    }
    __syncthreads();
    for (uint32_t j = tid; j < s_ns; j += kSplitThreads) sure[s_gs + j] = b_sure[j];
    for (uint32_t j = tid; j < s_nc; j += kSplitThreads) cand[s_gc + j] = b_cand[j];
    __syncthreads();
  }

  TTRACE(2);
  // ---------------------------------------------------------------- 3. last CTA of the row resolves
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    s_last = atomicAdd(cnt + 2, 1u) == gridDim.x - 1 ? 1u : 0u;
  }
  __syncthreads();
  TTRACE(3);
  if (!s_last) return;
  __threadfence();
  const uint32_t n_sure = __ldcg(cnt + 0), nc = __ldcg(cnt + 1);   // after the fence: every CTA's appends
  if (n_sure >= (uint32_t)k || nc > (uint32_t)A.n_max) {   // inconsistent histogram: report, emit nothing
    if (tid == 0) {
      set_device_error(a.err, kErrTopkOverflow);
      cnt[0] = 0u; cnt[1] = 0u; cnt[2] = 0u;
    }
    for (int i = tid; i < kHistBins; i += kSplitThreads) hist_row[i] = 0u;
    return;
  }
  uint32_t rem = (uint32_t)k - n_sure;        // >= 1: fewer than k keys lie above b*
#ifdef CSA_TRACE
  if (tid == 0 && blockIdx.x < 80) { g_trace_t[blockIdx.x][8] = n_sure; g_trace_t[blockIdx.x][9] = nc; }
#endif
  TTRACE(10);
  const int nw = (nv + 31) >> 5;
  const int nw4 = (nw + 3) & ~3;               // keeps the second bitmap 16-byte aligned
  uint32_t* sel = bm;
  uint32_t* eqm = bm + nw4;
  // candidates are read three times below: stage them in shared memory when they fit
  uint2* cs = reinterpret_cast<uint2*>(bm + 2 * ((((A.n_max + 31) >> 5) + 3) & ~(int64_t)3));
  const bool staged = nc <= (uint32_t)kCandCap;
  if (staged)
    for (uint32_t j = tid; j < nc; j += kSplitThreads) cs[j] = cand[j];
  const uint2* cv = staged ? cs : cand;
  for (int i = tid; i < 2 * nw4; i += kSplitThreads) bm[i] = 0u;
  __syncthreads();
  TTRACE(4);

  // two 10-bit radix passes over the candidates' low 20 bits pin the exact key T
  uint32_t prefix = bstar;
  int fixed = 12;
  for (int pass = 0; pass < 2; ++pass) {
    const int shift = 32 - fixed - 10;
    for (int i = tid; i < 1024; i += kSplitThreads) h2[i] = 0u;
    __syncthreads();
    for (uint32_t j = tid; j < nc; j += kSplitThreads) {
      const uint32_t key = cv[j].x;
      if ((key >> (32 - fixed)) == prefix) atomicAdd(&h2[(key >> shift) & 1023u], 1u);
    }
    __syncthreads();
    find_bin(h2, 1024, rem, wsum, &s_bin, &s_above);
    rem -= s_above;
    prefix = (prefix << 10) | s_bin;
    fixed += 10;
    __syncthreads();
  }
  const uint32_t T = prefix;                   // keys > T are taken; `rem` keys == T, smallest indices
  TTRACE(5);

  for (uint32_t j = tid; j < n_sure; j += kSplitThreads) {
    const uint32_t i = (uint32_t)sure[j];
    atomicOr(&sel[i >> 5], 1u << (i & 31));
  }
  for (uint32_t j = tid; j < nc; j += kSplitThreads) {
    const uint2 c = cv[j];
    if (c.x > T) atomicOr(&sel[c.y >> 5], 1u << (c.y & 31));
    else if (c.x == T) atomicOr(&eqm[c.y >> 5], 1u << (c.y & 31));
  }
  __syncthreads();

  TTRACE(6);
  // ordered emission.  Warp w owns words [w*CW, (w+1)*CW), CW a multiple of 256; in round i lane l
  // holds the 8 consecutive words w*CW + 256i + 8l .. +7 (two 128-bit loads, no bank conflicts),
  // and one warp scan per round orders the lanes.
  const int nwarps = kSplitThreads / 32, wid = tid >> 5;
  const int CW = ((nw + nwarps - 1) / nwarps + 255) & ~255;
  const int wbeg = wid * CW, wend = min(wbeg + CW, nw);
  auto load8 = [&](const uint32_t* bmp, int w0, uint32_t v[8]) {
    if (w0 + 8 <= nw) {
      const uint4 x = *reinterpret_cast<const uint4*>(bmp + w0), y = *reinterpret_cast<const uint4*>(bmp + w0 + 4);
      v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w; v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = (w0 + q < nw) ? bmp[w0 + q] : 0u;
    }
  };
  uint32_t eq_w = 0;
  for (int base = wbeg; base < wend; base += 256) {
    uint32_t v[8];
    load8(eqm, base + 8 * lane, v);
#pragma unroll
    for (int q = 0; q < 8; ++q) eq_w += __popc(v[q]);
  }
  eq_w = __reduce_add_sync(0xffffffffu, eq_w);
  uint32_t tot;
  uint32_t eq_before = block_excl_scan(lane == 0 ? eq_w : 0u, wsum, &tot);
  eq_before = __shfl_sync(0xffffffffu, eq_before, 0);
  TTRACE(11);
  uint32_t sel_w = 0;
  for (int base = wbeg; base < wend; base += 256) {
    const int w0 = base + 8 * lane;
    uint32_t e[8], sv[8];
    load8(eqm, w0, e);
    load8(sel, w0, sv);
    uint32_t pe = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) pe += __popc(e[q]);
    const uint32_t inc = warp_incl_scan(pe, lane);
    uint32_t before = eq_before + inc - pe;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint32_t keep = 0, ew = e[q];
      while (ew && before < rem) {
        const uint32_t low = ew & (0u - ew);
        keep |= low;
        ew ^= low;
        ++before;
      }
      before += __popc(ew);
      if (keep && w0 + q < nw) sel[w0 + q] = sv[q] | keep;
      sel_w += __popc(sv[q] | keep);
    }
    eq_before += __shfl_sync(0xffffffffu, inc, 31);
  }
  TTRACE(12);
  sel_w = __reduce_add_sync(0xffffffffu, sel_w);
  uint32_t pos0 = block_excl_scan(lane == 0 ? sel_w : 0u, wsum, &tot);
  pos0 = __shfl_sync(0xffffffffu, pos0, 0);
  TTRACE(13);
  for (int base = wbeg; base < wend; base += 256) {
    const int w0 = base + 8 * lane;
    uint32_t v[8];
    load8(sel, w0, v);
    uint32_t pb = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) pb += __popc(v[q]);
    const uint32_t inc = warp_incl_scan(pb, lane);
    uint32_t pos = pos0 + inc - pb;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint32_t bits = v[q];
      while (bits) {
        const int bit = __ffs(bits) - 1;
        bits &= bits - 1;
        out[pos++] = (w0 + q) * 32 + bit;
      }
    }
    pos0 += __shfl_sync(0xffffffffu, inc, 31);
  }
  // leave the row's histogram and counters zeroed for the next call (every CTA of the row has
  // read the histogram: each took its ticket after filtering)
  for (int i = tid; i < kHistBins; i += kSplitThreads) hist_row[i] = 0u;
  if (tid < 3) cnt[tid] = 0u;
  TTRACE(7);
}

}  // namespace

#ifdef CSA_TRACE
extern "C" __attribute__((visibility("default"))) int csa_trace_read_t(uint64_t* host) {
  return (int)cudaMemcpyFromSymbol(host, g_trace_t, sizeof(g_trace_t));
}
#endif

int topk_split_ctas(int rows, int64_t n_max, int num_sms) {
  int64_t g = (2 * (int64_t)num_sms + rows - 1) / rows;
  const int64_t by_size = (n_max + 4095) / 4096;
  if (g > by_size) g = by_size;
  if (g < 1) g = 1;
  return (int)g;
}

cudaError_t launch_topk_split(const TopkSplitArgs& a, cudaStream_t s) {
  if (a.base.rows <= 0 || a.base.k <= 0) return cudaSuccess;
  size_t smem = 2 * (size_t)((((a.base.n_max + 31) / 32) + 3) & ~(int64_t)3) * 4 + (size_t)kCandCap * 8;
  if (smem < (size_t)kChunk * 12) smem = (size_t)kChunk * 12;
  static size_t configured = 0;
  if (smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(topk_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  return launch_kernel(topk_split_kernel, dim3(a.G, a.base.rows), dim3(kSplitThreads), smem, s, 0, a);
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) {
  if (a.rows <= 0 || a.k <= 0) return cudaSuccess;
  const int use_smem = a.n_max <= kSmemKeys ? 1 : 0;
  const size_t smem = use_smem ? (size_t)a.n_max * 4 : 0;
  static size_t configured = 0;
  if (smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(topk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  return launch_kernel(topk_rows_kernel, dim3(a.rows), dim3(kThreads), smem, s, 0, a, use_smem);
}

}  // namespace csa
