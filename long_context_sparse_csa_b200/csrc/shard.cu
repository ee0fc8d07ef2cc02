// Context-sharded CSA decode: one sequence's compressed entries and index keys split into contiguous
// shards, one per rank.  Each rank scores and selects within its shard, the ranks exchange their
// candidates, every rank picks the same global top-k from them, attends the selected entries it
// holds (one rank also the window rows), and the ranks' partial results are merged once, with the
// sink and the inverse rotation.  The exchanges are the caller's collectives (an all-gather each);
// this file holds the two small kernels around them.  The selection of the merged candidates reuses
// the one-CTA-per-row top-k in its candidate mode.
//
// The pages describe one attention layer, not its distribution.  The split is exact: the global
// top-k of the union of the shards' top-k lists is the top-k of all entries (an entry in the global
// top-k is in its own shard's top-k), and attention over a union of disjoint key sets is the merge
// of the per-set partials (m, l, O/l) by their log-sum-exp weights, with the sink counted once
// ("DeepSeek-V4: Making a Million Tokens Affordable", "Two ways to shrink attention, interleaved",
// for the sink and the inverse rotation).
#include "kernels.h"

namespace csa {

namespace {

// (score, global index) of each of the row's local top-k entries; -inf and -1 for padding.
__global__ void shard_candidates_kernel(const float* __restrict__ scores, int64_t n_local,
                                        const int32_t* __restrict__ topk_local, int k, int64_t entry_offset,
                                        float* __restrict__ cand_score, int32_t* __restrict__ cand_idx) {
  const int row = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= k) return;
  const int32_t e = topk_local[(size_t)row * k + i];
  const bool ok = e >= 0 && e < n_local;
  cand_score[(size_t)row * k + i] = ok ? scores[(size_t)row * n_local + e] : -INFINITY;
  cand_idx[(size_t)row * k + i] = ok ? (int32_t)(e + entry_offset) : -1;
}

// One (row, head) per CTA, 4 output dims per thread: o = sum_g w_g O_g / (2^(s - M) + sum_g w_g) with
// w_g = l_g 2^(m_g - M) and M the largest of the sink and the parts' maxima (base 2), then the
// inverse rotation of the last 64 dims by the query's position.
__global__ void attend_merge_kernel(const __grid_constant__ LayerArgs L, const float* __restrict__ sinks,
                                    const int64_t* __restrict__ q_pos, int rows, int parts,
                                    const float* __restrict__ partials, uint8_t* __restrict__ out) {
  const int row = blockIdx.y, h = blockIdx.x;
  const int D = L.D;
  const int d0 = 4 * threadIdx.x;
  if (d0 >= D) return;
  const size_t part_stride = (size_t)rows * L.H * (D + 2);
  const size_t off = ((size_t)row * L.H + h) * (D + 2);
  const float sk = sinks[h] * kLog2e;
  float M = sk;
  for (int g = 0; g < parts; ++g) M = fmaxf(M, partials[g * part_stride + off + D]);
  float z = exp2f(sk - M), o[4] = {0.f, 0.f, 0.f, 0.f};
  for (int g = 0; g < parts; ++g) {
    const float* p = partials + g * part_stride + off;
    const float m = p[D], l = p[D + 1];
    if (m == -INFINITY || !(l > 0.f)) continue;
    const float w = l * exp2f(m - M);
    z += w;
#pragma unroll
    for (int k = 0; k < 4; ++k) o[k] = fmaf(w, p[d0 + k], o[k]);
  }
  const float inv = 1.f / z;
#pragma unroll
  for (int k = 0; k < 4; ++k) o[k] *= inv;
  if (d0 >= D - L.d_rope) {
    const double t = (double)q_pos[row];
#pragma unroll
    for (int k = 0; k < 4; k += 2) {
      float c, s;
      rope_cos_sin(-t, (d0 + k - (D - L.d_rope)) >> 1, L, &c, &s);
      const float x0 = o[k], x1 = o[k + 1];
      o[k] = x0 * c - x1 * s;
      o[k + 1] = x0 * s + x1 * c;
    }
  }
  uint8_t* dst = out + ((size_t)row * L.H + h) * (size_t)D * act_bytes(L.act_fmt);
  store_act4(dst, L.act_fmt, d0, o);
}

}  // namespace

cudaError_t launch_shard_candidates(const float* scores, int64_t n_local, const int32_t* topk_local, int rows,
                                    int k, int64_t entry_offset, float* cand_score, int32_t* cand_idx,
                                    cudaStream_t s) {
  if (rows <= 0 || k <= 0) return cudaSuccess;
  return launch_kernel(shard_candidates_kernel, dim3((unsigned)((k + 255) / 256), (unsigned)rows), dim3(256), 0, s,
                       0, scores, n_local, topk_local, k, entry_offset, cand_score, cand_idx);
}

cudaError_t launch_attend_merge(const LayerArgs& L, const float* sinks, const int64_t* q_pos, int rows, int parts,
                                const float* partials, uint8_t* out, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  return launch_kernel(attend_merge_kernel, dim3((unsigned)L.H, (unsigned)rows), dim3((unsigned)(L.D / 4)), 0, s, 0,
                       L, sinks, q_pos, rows, parts, partials, out);
}

}  // namespace csa
