// The index side of a CSA step, produced on the device: index keys compressed from an index-key
// stream, and index queries projected from the query's low-rank latent.
//
// Index keys ("DeepSeek-V4 Explained: ...", "The attention stack, and why it is two mechanisms": the
// lightning indexer scores the compressed entries in a low-rank way).  The operator reads the key of
// entry i as the index-key stream compressed like the KV stream: every token carries an index row and
// a row of gate logits of d_I channels; the key pools the entry's window rows [(i - ov) m, (i + 1) m)
// with a per-channel softmax of gate + slot bias, with no RMSNorm and no rotation, and is stored as
// e4m3 codes with one power-of-two scale (the smallest with max|k| / scale <= 448), or as float32.
//
// Index queries: q_h = W_h c for the query's latent c of r values and the learned up-projection W
// [H_I * d_I][r] (bf16), each head stored as e4m3 codes with its own power-of-two scale.  A cluster of
// four CTAs takes 16 query rows and one head, a quarter of the head's output dims each; the warps of
// a CTA run bf16 mma.sync m16n8k16 over interleaved k-steps of the r inputs (A = the latents, B = W's
// rows read as a column-major operand, fp32 accumulation), and the cluster reduces the head's max |q|
// per row for the scale.  In decode (one row) the kernel is a stream over W: H_I * d_I * r * 2 bytes
// (4 MiB for 32 x 128 x 512), read by 4 H_I SMs with every lane's weight loads in flight.
#include "kernels.h"

namespace csa {

namespace {

constexpr int kPrepThreads = 128;

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void mma_bf16_16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float act_at(const uint8_t* row, int fmt, int c) {
  return fmt == CSA_FMT_F32 ? reinterpret_cast<const float*>(row)[c]
                            : bf16_bits_to_f(reinterpret_cast<const uint16_t*>(row)[c]);
}

__device__ __forceinline__ void act_store(uint8_t* row, int fmt, int c, float v) {
  if (fmt == CSA_FMT_F32) reinterpret_cast<float*>(row)[c] = v;
  else reinterpret_cast<uint16_t*>(row)[c] = f_to_bf16_bits(v);
}

// One token (b, j): append its index row and gate row to the index rings (when given), then, if the
// token completes a group, compress that entry's index key.  Thread c owns channel c.
__device__ void index_key_token(const IndexPrepArgs& a, int b, int j, float* red) {
  const int c = threadIdx.x;
  const int d_I = a.d_I;
  const int64_t t = a.q_pos[(int64_t)b * a.Tq + j];
  const int64_t r = t - a.pos0;
  if (r < 0) return;                                        // block-uniform
  const size_t ab = a.act_fmt == CSA_FMT_F32 ? 4 : 2;
  const size_t arow = (size_t)d_I * ab;
  float xn = 0.f, gn = 0.f;
  if (a.x_new && c < d_I) {
    xn = act_at(a.x_new + ((size_t)b * a.Tq + j) * arow, a.act_fmt, c);
    gn = act_at(a.g_new + ((size_t)b * a.Tq + j) * arow, a.act_fmt, c);
    const int64_t s = ring_slot(r, a.raw_base, a.raw_cap);
    act_store(a.raw + ((size_t)b * a.raw_cap + s) * arow, a.act_fmt, c, xn);
    act_store(a.gate + ((size_t)b * a.raw_cap + s) * arow, a.act_fmt, c, gn);
  }
  if ((r + 1) % a.m != 0) return;                           // block-uniform
  const int64_t i = (r + 1) / a.m - 1;
  if (i >= a.entry_cap) return;
  const int64_t lo = (i - a.ov) * (int64_t)a.m;
  float mx = -INFINITY, sum = 0.f, acc = 0.f;
  if (c < d_I) {
    for (int64_t rr = lo < 0 ? 0 : lo; rr <= r; ++rr) {
      float x, z;
      if (rr == r && a.x_new) {
        x = xn;
        z = gn;
      } else {
        const int64_t s = ring_slot(rr, a.raw_base, a.raw_cap);
        x = act_at(a.raw + ((size_t)b * a.raw_cap + s) * arow, a.act_fmt, c);
        z = act_at(a.gate + ((size_t)b * a.raw_cap + s) * arow, a.act_fmt, c);
      }
      z = (z + a.pos_bias[(size_t)(rr - lo) * d_I + c]) * kLog2e;
      if (z > mx) {
        const float sc = exp2f(mx - z);
        sum *= sc;
        acc *= sc;
        mx = z;
      }
      const float e = exp2f(z - mx);
      sum += e;
      acc = fmaf(e, x, acc);
    }
  }
  const float k = c < d_I ? acc / sum : 0.f;
  if (a.idx_fmt == CSA_FMT_E2M1) {
    // FP4: key scale sigma from the key's max |k| (max / sigma <= 6), per 32-channel block (one warp)
    // the largest offset delta <= 7 with max_block |k| * 2^delta / sigma <= 6, codes rounded to
    // nearest-even at sigma * 2^-delta, two per byte (even channel in the low nibble)
    const int warp = c >> 5, lane = c & 31;
    float inv;
    const float sig = pow2_scale_fp4(block_max(fabsf(k), red), &inv);
    const float bmax = warp_max(fabsf(k)) * inv;             // exact: inv is a power of two
    uint32_t delta = 0;
    while (delta < 7 && bmax * (float)(2u << delta) <= 6.f) ++delta;
    const float x = k * inv * (float)(1u << delta);
    const uint32_t mag = e2m1_rne_magnitude(fabsf(x));
    const uint32_t code = (x < 0.f && mag != 0u) ? (mag | 8u) : mag;
    const uint32_t hi = __shfl_down_sync(0xffffffffu, code, 1);
    uint8_t* dst = a.keys + ((size_t)b * a.entry_cap + (size_t)i) * (size_t)(d_I / 2);
    if (c < d_I && (c & 1) == 0) dst[c >> 1] = (uint8_t)(code | (hi << 4));
    __shared__ uint32_t deltas[8];
    if (lane == 0) deltas[warp] = delta;
    __syncthreads();
    if (c == 0) {
      int e;
      frexpf(sig, &e);                                       // sig = 2^(e - 1)
      uint32_t word = (uint32_t)(e - 1 + 127);
      for (int blk = 0; blk < d_I / 32; ++blk) word |= deltas[blk] << (8 + 4 * blk);
      reinterpret_cast<uint32_t*>(a.key_scale)[(size_t)b * a.entry_cap + (size_t)i] = word;
    }
    return;
  }
  uint8_t* dst = a.keys + ((size_t)b * a.entry_cap + (size_t)i) * (size_t)d_I * (a.idx_fmt == CSA_FMT_F32 ? 4 : 1);
  if (a.idx_fmt == CSA_FMT_F32) {
    if (c < d_I) reinterpret_cast<float*>(dst)[c] = k;
    if (c == 0) a.key_scale[(size_t)b * a.entry_cap + (size_t)i] = 1.f;
    return;
  }
  const float amax = block_max(fabsf(k), red);
  float inv;
  const float sig = pow2_scale(amax, &inv);
  if (c < d_I) dst[c] = f_to_e4m3_sat(k * inv);
  if (c == 0) a.key_scale[(size_t)b * a.entry_cap + (size_t)i] = sig;
}

// Rows [16 rt, 16 rt + 16) of head h, output dims [qd dq, qd dq + dq) with dq = d_I / 4.  The head's
// four quarters are the four CTAs of one cluster, so the head's weights W_h are read by four SMs
// at once; each CTA computes its quarter of q = W_h c, and the four exchange their per-row max |q|
// through distributed shared memory so that every quarter is encoded with the head's one scale.
// Inside the CTA the four warps split the rank's k-steps (warp w takes steps w, w + 4, ...), with
// many independent weight loads in flight per lane, and add their partial sums in shared memory.
__device__ void index_query_tile(const IndexPrepArgs& a, int rt, int h, float* part, float* qmax) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, j = lane & 3;
  const int d_I = a.d_I, r = a.rank;
  const int qd = (int)cluster_rank();
  const int dq = d_I / 4, nt = dq / 8;                      // 1..4 n-tiles of 8 dims
  const int row0 = 16 * rt + g, row1 = row0 + 8;
  const bool ok0 = row0 < a.rows, ok1 = row1 < a.rows;
  const uint16_t* C = reinterpret_cast<const uint16_t*>(a.c);
  const uint16_t* W = reinterpret_cast<const uint16_t*>(a.W) + ((size_t)h * d_I + (size_t)qd * dq) * r;
  // the cluster's first phase: arrive now, wait before the first remote store (every CTA has started)
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  float acc[4][4];
#pragma unroll
  for (int n = 0; n < 4; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  const int ksteps = r / 16;
#pragma unroll 8
  for (int st = warp; st < ksteps; st += 4) {
    const int k0 = 16 * st;
    uint32_t af[4];
    af[0] = ok0 ? __ldg(reinterpret_cast<const uint32_t*>(C + (size_t)row0 * r + k0 + 2 * j)) : 0u;
    af[1] = ok1 ? __ldg(reinterpret_cast<const uint32_t*>(C + (size_t)row1 * r + k0 + 2 * j)) : 0u;
    af[2] = ok0 ? __ldg(reinterpret_cast<const uint32_t*>(C + (size_t)row0 * r + k0 + 8 + 2 * j)) : 0u;
    af[3] = ok1 ? __ldg(reinterpret_cast<const uint32_t*>(C + (size_t)row1 * r + k0 + 8 + 2 * j)) : 0u;
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      if (n < nt) {
        const uint16_t* wr = W + (size_t)(8 * n + g) * r + k0 + 2 * j;
        mma_bf16_16816(acc[n], af, __ldg(reinterpret_cast<const uint32_t*>(wr)),
                       __ldg(reinterpret_cast<const uint32_t*>(wr + 8)));
      }
    }
  }
  // acc[n][0..1]: row g, dims 8n + 2j (+1); acc[n][2..3]: row g + 8.  Partial sums -> [warp][row][32]
#pragma unroll
  for (int n = 0; n < 4; ++n) {
    if (n < nt) {
      const int d = 8 * n + 2 * j;
      part[(warp * 16 + g) * 32 + d] = acc[n][0];
      part[(warp * 16 + g) * 32 + d + 1] = acc[n][1];
      part[(warp * 16 + g + 8) * 32 + d] = acc[n][2];
      part[(warp * 16 + g + 8) * 32 + d + 1] = acc[n][3];
    }
  }
  __syncthreads();
  // thread t: row t / 8 of the tile, dims 4 (t % 8) .. + 4 of the quarter
  const int tr = threadIdx.x >> 3, td = 4 * (threadIdx.x & 7);
  const bool mine = td < dq;                                // dq is a multiple of 8: all 4 dims or none
  float v[4], mx = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    v[e] = 0.f;
    if (mine) {
#pragma unroll
      for (int w = 0; w < 4; ++w) v[e] += part[(w * 16 + tr) * 32 + td + e];
    }
    mx = fmaxf(mx, fabsf(v[e]));
  }
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  if ((threadIdx.x & 7) == 0) {
    const uint32_t local = (uint32_t)__cvta_generic_to_shared(qmax + qd * 16 + tr);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      uint32_t remote;
      asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(p));
      asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(mx) : "memory");
    }
  }
  // release our stores to the peers, acquire theirs; no remote access follows, so a CTA may exit
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
  const float am = fmaxf(fmaxf(qmax[tr], qmax[16 + tr]), fmaxf(qmax[32 + tr], qmax[48 + tr]));
  const int row = 16 * rt + tr;
  if (row >= a.rows) return;
  const bool f32 = a.idx_fmt == CSA_FMT_F32;
  float inv = 1.f, sg = 1.f;
  if (!f32) sg = pow2_scale(am, &inv);
  uint8_t* q = a.q_out + ((size_t)row * a.H_I + h) * (size_t)d_I * (f32 ? 4 : 1);
  const int d = qd * dq + td;
  if (mine) {
    if (f32) {
#pragma unroll
      for (int e = 0; e < 4; ++e) reinterpret_cast<float*>(q)[d + e] = v[e];
    } else {
      uint32_t w = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) w |= (uint32_t)f_to_e4m3_sat(v[e] * inv) << (8 * e);
      *reinterpret_cast<uint32_t*>(q + d) = w;
    }
  }
  if (qd == 0 && td == 0) a.q_scale_out[(size_t)row * a.H_I + h] = sg;
}

// Blocks [0, key_blocks) compress index keys (one token each; the count is rounded up to whole
// clusters when queries follow); the rest project index queries, one cluster of four CTAs per
// (16-row tile, head).
__global__ void __launch_bounds__(kPrepThreads) index_prep_kernel(const __grid_constant__ IndexPrepArgs a) {
  __shared__ float red[64];
  __shared__ float part[4 * 16 * 32];
  __shared__ float qmax[4 * 16];
  const int blk = blockIdx.x;
  if (blk < a.key_blocks) {
    if (a.keys && blk < a.B * a.Tq) index_key_token(a, blk / a.Tq, blk % a.Tq, red);
    return;
  }
  const int q = (blk - a.key_blocks) >> 2;
  index_query_tile(a, q / a.H_I, q % a.H_I, part, qmax);
}

}  // namespace

cudaError_t launch_index_prep(IndexPrepArgs a, cudaStream_t s) {
  const int q_blocks = a.c ? ((a.rows + 15) / 16) * a.H_I * 4 : 0;
  a.key_blocks = a.keys ? a.B * a.Tq : 0;
  if (q_blocks) a.key_blocks = (a.key_blocks + 3) & ~3;    // whole clusters of four
  if (a.key_blocks + q_blocks == 0) return cudaSuccess;
  return launch_kernel(index_prep_kernel, dim3((unsigned)(a.key_blocks + q_blocks)), dim3(kPrepThreads), 0, s,
                       q_blocks ? 4 : 0, a);
}

}  // namespace csa
