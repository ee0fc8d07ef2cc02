// Top-k selection of indexer scores: the k largest scores among a query's
// visible entries, ties to the smaller entry index, emitted in ascending
// entry order and padded with -1. Only the k best-scoring entries go on to the core attention
// (step 4 of "DeepSeek-V4, explained."; "DeepSeek-V4: Making a Million Tokens Affordable", section
// "Two ways to shrink attention, interleaved").
//
// One 1024-thread CTA per query row runs a radix select on the
// order-preserving 32-bit image of the scores (11 + 11 + 10 bits, shared-
// memory histograms), which pins the k-th largest key T and how many keys
// equal to T are taken; a final pass over the row in index order writes the
// selection, so the output order (ascending index) and the tie rule come out
// deterministic.  Rows up to kSmemKeys scores are staged once in shared memory;
// their final pass gives each thread a contiguous run of indices and places
// every selection with one block-wide scan of the runs' counts (rows read from
// global memory take one scan per 1024 indices, coalesced).
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
  const bool cand = a.map != nullptr;
  int64_t nv;
  if (cand) {
    nv = (int64_t)a.shards * a.k;
  } else {
    const int64_t t = a.q_pos[row];
    const int64_t r1 = t - a.pos0 + 1;
    nv = r1 > 0 ? r1 / a.m : 0;
    if (nv > a.n_max) nv = a.n_max;
  }
  int32_t* out = a.out + (size_t)row * a.k;
  const float* sc = a.scores + (size_t)row * a.n_max;
  // candidate mode: position i of the row is candidate i % k of shard i / k, stored [shard][row][k]
  auto flat = [&](int i) -> size_t { return ((size_t)(i / a.k) * a.rows + row) * a.k + (size_t)(i % a.k); };
  auto value_at = [&](int i) -> int32_t { return cand ? a.map[flat(i)] : i; };
  // a candidate slot without an entry ranks below every score (key 0)
  auto raw_key = [&](int i) -> uint32_t {
    if (!cand) return float_key(__ldg(sc + i));
    const size_t f = flat(i);
    return a.map[f] >= 0 ? float_key(__ldg(a.scores + f)) : 0u;
  };

  if (nv <= a.k) {
    for (int i = tid; i < a.k; i += kThreads) out[i] = i < nv ? value_at(i) : -1;
    return;
  }
  const int n = (int)nv;
  if (use_smem) {
    for (int i = tid; i < n; i += kThreads) keys_sm[i] = raw_key(i);
    __syncthreads();
  }
  auto key_at = [&](int i) -> uint32_t { return use_smem ? keys_sm[i] : raw_key(i); };

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
  // candidate mode with fewer than k real candidates: the k-th key is that of the empty slots, 0:
  // take the real ones only and pad the tail with -1
  if (cand && T == 0u) remaining = 0u;

  // ------------------------------------------------------------------ ordered emission
  if (use_smem) {
    // each thread takes a contiguous run of `per` indices (odd, so the runs' shared-memory words
    // fall in distinct banks across a warp); one scan of the runs' counts places every selection
    const int per = ((n + kThreads - 1) / kThreads) | 1;
    const int lo = tid * per, hi = min(lo + per, n);
    uint32_t gt_n = 0, eq_n = 0;
    for (int i = lo; i < hi; ++i) {
      const uint32_t k = keys_sm[i];
      gt_n += k > T;
      eq_n += k == T;
    }
    uint32_t gt_tot, eq_tot;
    uint32_t gt_run = block_excl_scan(gt_n, wsum, &gt_tot);
    uint32_t eq_run = block_excl_scan(eq_n, wsum, &eq_tot);
    for (int i = lo; i < hi; ++i) {
      const uint32_t k = keys_sm[i];
      if (k > T) {
        out[gt_run + min(eq_run, remaining)] = value_at(i);
        ++gt_run;
      } else if (k == T) {
        if (eq_run < remaining) out[gt_run + eq_run] = value_at(i);
        ++eq_run;
      }
    }
    const uint32_t taken = gt_tot + min(eq_tot, remaining);
    for (uint32_t p = taken + tid; p < (uint32_t)a.k; p += kThreads) out[p] = -1;
    return;
  }
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
      out[pos] = value_at(i);
    }
    gt_run += tot & 0xFFFFu;
    eq_run += tot >> 16;
  }
  const uint32_t taken = gt_run + min(eq_run, remaining);
  for (uint32_t p = taken + tid; p < (uint32_t)a.k; p += kThreads) out[p] = -1;
}


// ----------------------------------------------------------------------------- split mode (long decode rows)
// Many CTAs per row; the indexer epilogue has already histogrammed the top 12 key bits of the
// row's visible scores (the steps are described above the kernel).
#ifdef CSA_TRACE
__device__ uint64_t g_trace_t[80][24];
#define TTRACE(slot) do { if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.x < 80) { \
    uint64_t _t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(_t) :: "memory"); g_trace_t[blockIdx.x][(slot)] = _t; } } while (0)
#define TTRACE_CYC(slot) do { if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.x < 80) \
    g_trace_t[blockIdx.x][(slot)] = (uint64_t)clock64(); } while (0)
#else
#define TTRACE(slot) ((void)0)
#define TTRACE_CYC(slot) ((void)0)
#endif

constexpr int kSplitThreads = 512;
constexpr int kHistBins = 4096;
constexpr int kPer = 8;                               // scores / list entries per thread per pass
constexpr int kChunk = kSplitThreads * kPer;          // 4096 per block pass
static_assert(kHistBins == kChunk, "one histogram bin group of 8 per thread");
static_assert(kTopkSplitMaxCtas <= kSplitThreads, "one slice count per thread");

// find_bin over the row's global 4096-bin histogram: thread t holds bins 4095-8t .. 4088-8t (two
// 128-bit loads), descending.
__device__ __forceinline__ void find_bin_hist(const uint32_t* hist, uint32_t need, uint32_t* wsum, uint32_t* s_bin,
                                              uint32_t* s_above) {
  const int top = kHistBins - kPer * (int)threadIdx.x;   // exclusive upper bin of this thread
  const uint4* p = reinterpret_cast<const uint4*>(hist + top - kPer);
  const uint4 lo4 = __ldcg(p), hi4 = __ldcg(p + 1);
  const uint32_t c[kPer] = {hi4.w, hi4.z, hi4.y, hi4.x, lo4.w, lo4.z, lo4.y, lo4.x};   // bins top-1 .. top-8
  uint32_t c_local = 0;
#pragma unroll
  for (int q = 0; q < kPer; ++q) c_local += c[q];
  uint32_t tot;
  uint32_t above = block_excl_scan(c_local, wsum, &tot);
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    if (above < need && need <= above + c[q]) { *s_bin = (uint32_t)(top - 1 - q); *s_above = above; }
    above += c[q];
  }
  __syncthreads();
}

// Multi-CTA top-k of one long row (decode).  The key of a score is its order-preserving 32-bit
// image; the k-th largest key T is pinned 12 + 12 + 8 bits at a time:
//  1. every CTA finds the bin b1 of the key's top 12 bits that holds the k-th largest key, from the
//     histogram the indexer filled while writing the scores;
//  2. CTA g filters its slice [lo_g, hi_g) of the row: it writes (key, index) of every score whose
//     top bits are >= b1 into the slice's own region of `list`, in ascending index order (a block
//     scan per 4096 scores), adds each key of bin b1 to a second histogram of key bits 19..8, and
//     stores its count;
//  3. the last CTA to finish (a ticket counter; no CTA waits for another) finds the bin b2 of the
//     second histogram, then the exact key with an 8-bit histogram of the few keys left;
//  4. it concatenates the regions in CTA order (= ascending index order) and emits the entries with
//     key > T and the first (k - #{key > T}) entries with key == T, each at its rank (one block scan
//     of packed counts): ascending index order, ties to the smaller index.
__global__ void __launch_bounds__(kSplitThreads, 1) topk_split_kernel(const __grid_constant__ TopkSplitArgs a) {
  __shared__ uint32_t h3[256];
  __shared__ uint32_t wsum[32];
  __shared__ uint32_t s_off[kTopkSplitMaxCtas + 1];
  __shared__ uint32_t s_lo[kTopkSplitMaxCtas];          // first index of each CTA's slice
  __shared__ uint32_t s_bin, s_above, s_last;
  const TopkArgs& A = a.base;
  const int row = blockIdx.y, g = blockIdx.x, tid = threadIdx.x;
  const int G = gridDim.x;
  const int64_t t = A.q_pos[row];
  const int64_t r1 = t - A.pos0 + 1;
  int64_t nv64 = r1 > 0 ? r1 / A.m : 0;
  if (nv64 > A.n_max) nv64 = A.n_max;
  const int nv = (int)nv64;
  const int k = A.k;
  int32_t* out = A.out + (size_t)row * k;
  uint32_t* hist_row = const_cast<uint32_t*>(a.hist) + (size_t)row * kHistBins;
  uint32_t* hist2_row = a.hist2 + (size_t)row * kHistBins;
  if (nv <= k) {
    if (g == 0) {
      for (int i = tid; i < k; i += kSplitThreads) out[i] = i < nv ? i : -1;
      for (int i = tid; i < kHistBins; i += kSplitThreads) hist_row[i] = 0u;   // leave it zeroed for the next call
    }
    return;
  }
  uint32_t* cnt = a.cnt + (size_t)row * 4;
  uint32_t* counts = a.counts + (size_t)row * kTopkSplitMaxCtas;
  uint2* lst = a.list + (size_t)row * A.n_max;
  auto slice_lo = [&](int gg) { return (int)((int64_t)nv * gg / G); };

  TTRACE(0);
  // the slice's first scores do not depend on the histogram: their loads overlap its reads
  const int lo = slice_lo(g), hi = slice_lo(g + 1);
  const float* sc = A.scores + (size_t)row * A.n_max;
  auto load_scores = [&](int cb, int ce, float vals[kPer]) {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = cb + tid * kPer + u;           // a thread's kPer consecutive scores
      vals[u] = i < ce ? __ldcg(sc + i) : 0.f;
    }
  };
  float vals[kPer];
  load_scores(lo, min(lo + kChunk, hi), vals);
  // ---------------------------------------------------------------- 1. bin b1 of the k-th largest key
  if (tid == 0) { s_bin = 0xFFFFFFFFu; s_above = 0u; }   // stays so if the histogram holds fewer than k
  find_bin_hist(hist_row, (uint32_t)k, wsum, &s_bin, &s_above);
  const uint32_t b1 = s_bin, n_above1 = s_above;
  TTRACE(1);

  // ---------------------------------------------------------------- 2. filter this CTA's slice
  uint32_t n_mine = 0;
  for (int cb = lo; cb < hi; cb += kChunk) {
    const int ce = min(cb + kChunk, hi);
    if (cb != lo) load_scores(cb, ce, vals);
    uint32_t keys[kPer], n = 0;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      keys[u] = float_key(vals[u]);
      n += (cb + tid * kPer + u < ce && (keys[u] >> 20) >= b1);
    }
    uint32_t tot;
    uint32_t pos = (uint32_t)lo + n_mine + block_excl_scan(n, wsum, &tot);
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = cb + tid * kPer + u;
      if (i < ce && (keys[u] >> 20) >= b1) {
        lst[pos++] = make_uint2(keys[u], (uint32_t)i);
        if ((keys[u] >> 20) == b1) atomicAdd(hist2_row + ((keys[u] >> 8) & 4095u), 1u);
      }
    }
    n_mine += tot;
  }
  if (tid == 0) counts[g] = n_mine;
  TTRACE(2);
  // ---------------------------------------------------------------- 3. last CTA of the row resolves
  __syncthreads();                   // every list entry and histogram add of this CTA is issued ...
  if (tid == 0) {
    __threadfence();                 // ... and released (cumulatively) before the ticket; the ticket
    uint32_t old;                    // acquires, and the barrier below passes that on to the CTA
    asm volatile("atom.add.acquire.gpu.u32 %0, [%1], 1;" : "=r"(old) : "l"(cnt + 2) : "memory");
    s_last = old == (uint32_t)G - 1 ? 1u : 0u;
  }
  __syncthreads();
  TTRACE(3);
  if (!s_last) return;
  TTRACE(8);
  // second level: bits 19..8 of the bin-b1 keys (its loads overlap the slice counts' below)
  uint32_t rem = (uint32_t)k - n_above1;       // >= 1 when the histogram is consistent
  if (tid == 0) { s_bin = 0xFFFFFFFFu; s_above = 0u; }
  const uint32_t c_mine = tid < G ? __ldcg(counts + tid) : 0u;
  find_bin_hist(hist2_row, rem, wsum, &s_bin, &s_above);
  TTRACE(9);
  const uint32_t b2 = s_bin;
  rem -= s_above;
  const uint32_t p24 = (b1 << 12) | b2;        // top 24 bits of T
  {
    uint32_t tot;
    const uint32_t ex = block_excl_scan(c_mine, wsum, &tot);
    if (tid < G) {
      s_off[tid] = ex;
      s_lo[tid] = (uint32_t)slice_lo(tid);
    }
    if (tid == 0) s_off[G] = tot;
    if (tid < 256) h3[tid] = 0u;
  }
  __syncthreads();
  TTRACE(10);
  const uint32_t L = s_off[G];
  // entries p = base + kPer*tid + u of the concatenation (index ~0u past the end)
  auto load_chunk = [&](uint32_t base, uint32_t kk[kPer], uint32_t ii[kPer]) {
    const uint32_t p0 = base + kPer * (uint32_t)tid;
    int gg = 0;
    if (p0 < L) {                    // the slice holding p0: largest gg with s_off[gg] <= p0
      int lo2 = 0, hi2 = G - 1;
      while (lo2 < hi2) {
        const int mid = (lo2 + hi2 + 1) >> 1;
        if (s_off[mid] <= p0) lo2 = mid; else hi2 = mid - 1;
      }
      gg = lo2;
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const uint32_t p = p0 + u;
      kk[u] = 0u;
      ii[u] = ~0u;
      if (p < L) {
        while (p >= s_off[gg + 1]) ++gg;
        const uint2 e = __ldcg(lst + s_lo[gg] + (p - s_off[gg]));
        kk[u] = e.x;
        ii[u] = e.y;
      }
    }
  };
  const bool one = L <= (uint32_t)kChunk;      // the usual case: the list stays in registers
  uint32_t kk[kPer], ii[kPer];
  if (one) load_chunk(0, kk, ii);
  // every CTA of the row read both histograms' bins before its ticket: leave them zeroed now,
  // while the list's loads are in flight
  {
    uint4* h1 = reinterpret_cast<uint4*>(hist_row);
    uint4* h2 = reinterpret_cast<uint4*>(hist2_row);
    for (int i = tid; i < kHistBins / 4; i += kSplitThreads) {
      h1[i] = make_uint4(0u, 0u, 0u, 0u);
      h2[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (tid < 3) cnt[tid] = 0u;
  }
  TTRACE(4);
#ifdef CSA_TRACE
  if (one) { uint32_t x = 0; for (int u = 0; u < kPer; ++u) x += kk[u]; if (x == 12345u) s_bin = x; }
#endif
  TTRACE(11);

  // third level: the low 8 bits of the keys whose top 24 bits are p24
  const bool lvl2 = b2 != 0xFFFFFFFFu && b1 != 0xFFFFFFFFu;
  if (lvl2) {
    for (uint32_t base = 0; base < L; base += kChunk) {
      if (!one) load_chunk(base, kk, ii);
#pragma unroll
      for (int u = 0; u < kPer; ++u)
        if (ii[u] != ~0u && (kk[u] >> 8) == p24) atomicAdd(&h3[kk[u] & 255u], 1u);
    }
  }
  __syncthreads();
  TTRACE(12);
  if (tid < 32) {
    // one warp: lane l holds bins 255-8l .. 248-8l (descending)
    uint32_t c[8], c_local = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) { c[q] = lvl2 ? h3[255 - 8 * tid - q] : 0u; c_local += c[q]; }
    uint32_t above = warp_incl_scan(c_local, tid) - c_local;
    uint32_t bin = 0xFFFFFFFFu, ab = 0u;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (above < rem && rem <= above + c[q]) { bin = (uint32_t)(255 - 8 * tid - q); ab = above; }
      above += c[q];
    }
    const uint32_t hit = __ballot_sync(0xffffffffu, bin != 0xFFFFFFFFu);
    if (tid == 0 && !hit) { s_bin = 0xFFFFFFFFu; s_above = 0u; }
    if (bin != 0xFFFFFFFFu) { s_bin = bin; s_above = ab; }
  }
  __syncthreads();
  const bool resolved = lvl2 && s_bin != 0xFFFFFFFFu;
  const uint32_t T = (p24 << 8) | (s_bin & 255u);   // every key > T is taken, and `rem` keys == T
  rem -= resolved ? s_above : 0u;
  TTRACE(5);

  // ---------------------------------------------------------------- 4. ordered emission
  uint32_t gt_run = 0, tie_run = 0;
  if (resolved) {
    for (uint32_t base = 0; base < L; base += kChunk) {
      if (!one) load_chunk(base, kk, ii);
      uint32_t ngt = 0, ntie = 0;
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        ngt += (ii[u] != ~0u && kk[u] > T);
        ntie += (ii[u] != ~0u && kk[u] == T);
      }
      uint32_t tot;
      const uint32_t ex = block_excl_scan(ngt | (ntie << 16), wsum, &tot);
      uint32_t gtb = gt_run + (ex & 0xFFFFu), tieb = tie_run + (ex >> 16);
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        if (ii[u] == ~0u) continue;
        if (kk[u] > T) {
          const uint32_t pos = gtb + min(tieb, rem);
          if (pos < (uint32_t)k) out[pos] = (int32_t)ii[u];
          ++gtb;
        } else if (kk[u] == T) {
          if (tieb < rem && gtb + tieb < (uint32_t)k) out[gtb + tieb] = (int32_t)ii[u];
          ++tieb;
        }
      }
      gt_run += tot & 0xFFFFu;
      tie_run += tot >> 16;
    }
  }
  // a consistent histogram yields exactly k; otherwise report and pad what was not written
  const uint32_t n_out = resolved ? gt_run + min(tie_run, rem) : 0u;
  if (n_out != (uint32_t)k) {
    if (tid == 0) set_device_error(a.err, kErrTopkOverflow);
    for (uint32_t i = n_out + tid; i < (uint32_t)k; i += kSplitThreads) out[i] = -1;
  }
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
  if (a.G < 1 || a.G > kTopkSplitMaxCtas) return cudaErrorInvalidValue;
  return launch_kernel(topk_split_kernel, dim3(a.G, a.base.rows), dim3(kSplitThreads), 0, s, 0, a);
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) {
  if (a.rows <= 0 || a.k <= 0) return cudaSuccess;
  const int64_t n_row = a.map ? (int64_t)a.shards * a.k : a.n_max;   // keys of a row
  const int use_smem = n_row <= kSmemKeys ? 1 : 0;
  const size_t smem = use_smem ? (size_t)n_row * 4 : 0;
  {
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(topk_rows_kernel), smem);
    if (e != cudaSuccess) return e;
  }
  return launch_kernel(topk_rows_kernel, dim3(a.rows), dim3(kThreads), smem, s, 0, a, use_smem);
}

}  // namespace csa
