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
// [H_I * d_I][r] (bf16), each head stored as e4m3 codes with its own power-of-two scale.  A CTA takes
// 16 query rows and one head: four warps split the head's 128 output dims, each runs bf16 mma.sync
// m16n8k16 over the r inputs (A = the latents, B = W's rows of the head read as a column-major
// operand, fp32 accumulation), then the CTA reduces the head's max |q| per row for the scale.
#include "kernels.h"

namespace csa {

namespace {

constexpr int kPrepThreads = 128;

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

// Rows [16 rt, 16 rt + 16) of head h: q = W_h c, then the head's scale per row and the codes.
__device__ void index_query_tile(const IndexPrepArgs& a, int rt, int h, float* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, j = lane & 3;
  const int d_I = a.d_I, r = a.rank;
  const int row0 = 16 * rt + g, row1 = row0 + 8;
  const int cols = d_I / 4;                                 // this warp's output dims: [warp * cols, +cols)
  const int nt = cols / 8;                                  // n-tiles of 8
  const uint16_t* C = reinterpret_cast<const uint16_t*>(a.c);
  const uint16_t* W = reinterpret_cast<const uint16_t*>(a.W) + (size_t)h * d_I * r;
  float acc[4][4];                                          // up to 4 n-tiles (d_I <= 128)
#pragma unroll
  for (int n = 0; n < 4; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  for (int k0 = 0; k0 < r; k0 += 16) {
    uint32_t af[4];
    af[0] = row0 < a.rows ? *reinterpret_cast<const uint32_t*>(C + (size_t)row0 * r + k0 + 2 * j) : 0u;
    af[1] = row1 < a.rows ? *reinterpret_cast<const uint32_t*>(C + (size_t)row1 * r + k0 + 2 * j) : 0u;
    af[2] = row0 < a.rows ? *reinterpret_cast<const uint32_t*>(C + (size_t)row0 * r + k0 + 8 + 2 * j) : 0u;
    af[3] = row1 < a.rows ? *reinterpret_cast<const uint32_t*>(C + (size_t)row1 * r + k0 + 8 + 2 * j) : 0u;
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      if (n < nt) {
        const uint16_t* wr = W + (size_t)(warp * cols + 8 * n + g) * r + k0 + 2 * j;
        mma_bf16_16816(acc[n], af, __ldg(reinterpret_cast<const uint32_t*>(wr)),
                       __ldg(reinterpret_cast<const uint32_t*>(wr + 8)));
      }
    }
  }
  // acc[n][0..1]: row0, dims warp*cols + 8n + 2j (+1); acc[n][2..3]: row1
  float m0 = 0.f, m1 = 0.f;
#pragma unroll
  for (int n = 0; n < 4; ++n)
    if (n < nt) {
      m0 = fmaxf(m0, fmaxf(fabsf(acc[n][0]), fabsf(acc[n][1])));
      m1 = fmaxf(m1, fmaxf(fabsf(acc[n][2]), fabsf(acc[n][3])));
    }
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) {
    m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
    m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
  }
  if (j == 0) {
    red[warp * 16 + g] = m0;
    red[warp * 16 + g + 8] = m1;
  }
  __syncthreads();
  const float am0 = fmaxf(fmaxf(red[g], red[16 + g]), fmaxf(red[32 + g], red[48 + g]));
  const float am1 = fmaxf(fmaxf(red[g + 8], red[16 + g + 8]), fmaxf(red[32 + g + 8], red[48 + g + 8]));
  float inv0 = 1.f, inv1 = 1.f, sg0 = 1.f, sg1 = 1.f;
  const bool f32 = a.idx_fmt == CSA_FMT_F32;
  if (!f32) {
    sg0 = pow2_scale(am0, &inv0);
    sg1 = pow2_scale(am1, &inv1);
  }
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int row = half ? row1 : row0;
    if (row >= a.rows) continue;
    const float inv = half ? inv1 : inv0;
    uint8_t* q = a.q_out + ((size_t)row * a.H_I + h) * (size_t)d_I * (f32 ? 4 : 1);
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      if (n >= nt) continue;
      const int d = warp * cols + 8 * n + 2 * j;
      const float v0 = acc[n][2 * half], v1 = acc[n][2 * half + 1];
      if (f32) {
        *reinterpret_cast<float2*>(q + 4 * (size_t)d) = make_float2(v0, v1);
      } else {
        *reinterpret_cast<uint16_t*>(q + d) =
            (uint16_t)((uint32_t)f_to_e4m3_sat(v0 * inv) | ((uint32_t)f_to_e4m3_sat(v1 * inv) << 8));
      }
    }
    if (warp == 0 && j == 0) a.q_scale_out[(size_t)row * a.H_I + h] = half ? sg1 : sg0;
  }
}

// Blocks [0, key_blocks) compress index keys (one token each); the rest project index queries
// (one (16-row tile, head) each).
__global__ void __launch_bounds__(kPrepThreads) index_prep_kernel(const __grid_constant__ IndexPrepArgs a) {
  __shared__ float red[64];
  const int blk = blockIdx.x;
  if (blk < a.key_blocks) {
    index_key_token(a, blk / a.Tq, blk % a.Tq, red);
    return;
  }
  const int q = blk - a.key_blocks;
  index_query_tile(a, q / a.H_I, q % a.H_I, red);
}

}  // namespace

cudaError_t launch_index_prep(IndexPrepArgs a, cudaStream_t s) {
  a.key_blocks = a.keys ? a.B * a.Tq : 0;
  const int q_blocks = a.c ? ((a.rows + 15) / 16) * a.H_I : 0;
  if (a.key_blocks + q_blocks == 0) return cudaSuccess;
  return launch_kernel(index_prep_kernel, dim3((unsigned)(a.key_blocks + q_blocks)), dim3(kPrepThreads), 0, s, 0, a);
}

}  // namespace csa
