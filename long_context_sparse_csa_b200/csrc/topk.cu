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

// Exclusive block scan (blockDim.x == kThreads); *total = sum over the block.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* wsum, uint32_t* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const uint32_t inc = warp_incl_scan(v, lane);
  if (lane == 31) wsum[wid] = inc;
  __syncthreads();
  if (wid == 0) {
    uint32_t x = wsum[lane];
    x = warp_incl_scan(x, lane);
    wsum[lane] = x;
  }
  __syncthreads();
  const uint32_t before = wid > 0 ? wsum[wid - 1] : 0u;
  *total = wsum[31];
  __syncthreads();
  return before + inc - v;
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
    // suffix counts: thread t owns the bins (nb-1 - per*t - q), q < per, in descending order
    const int per = nb / kThreads;             // 2 or 1
    uint32_t c_local = 0;
    for (int q = 0; q < per; ++q) c_local += hist[nb - 1 - per * tid - q];
    uint32_t tot;
    uint32_t above = block_excl_scan(c_local, wsum, &tot);
    for (int q = 0; q < per; ++q) {
      const int bin = nb - 1 - per * tid - q;
      const uint32_t h = hist[bin];
      if (above < remaining && remaining <= above + h) { sel_bin = (uint32_t)bin; sel_above = above; }
      above += h;
    }
    __syncthreads();
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

}  // namespace

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) {
  if (a.rows <= 0 || a.k <= 0) return cudaSuccess;
  const int use_smem = a.n_max <= kSmemKeys ? 1 : 0;
  const size_t smem = use_smem ? (size_t)a.n_max * 4 : 0;
  static size_t configured = 0;
  if (smem > 48 * 1024 && smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(topk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  topk_rows_kernel<<<a.rows, kThreads, smem, s>>>(a, use_smem);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace csa
