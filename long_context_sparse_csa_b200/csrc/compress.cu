// Append new tokens to the caches and compress completed groups into entries.
//
// Compression follows "DeepSeek-V4: Making a Million Tokens Affordable",
// section "Two ways to shrink attention, interleaved" (each entry pools m
// tokens, drawing from 2m source rows with overlap) and "DeepSeek-V4
// Explained: ...", section "The attention stack, and why it is two
// mechanisms" (learned compression weights and positional biases): per
// channel, a softmax over the window's rows of gate logit + slot bias weights
// the raw rows; the pooled vector gets an RMSNorm and rotary embedding on its
// last 64 dims at position pos0 + i*m, and is stored in the cache format.
//
// One CTA per (token, sequence), D/4 threads, 4 consecutive channels per
// thread; raw rows are read once with 8/16-byte vector loads and the
// per-channel softmax runs online in registers.
#include "common.cuh"
#include "kernels.h"

namespace csa {

namespace {

__device__ __forceinline__ void rope4(float v[4], int c0, const LayerArgs& L, double pos) {
  const int dn = L.D - L.d_rope;
  if (c0 < dn) return;
  const int u = (c0 - dn) >> 1;
  float c, s, a, b;
  rope_cos_sin(pos, u, L, &c, &s);
  a = v[0]; b = v[1];
  v[0] = a * c - b * s; v[1] = a * s + b * c;
  rope_cos_sin(pos, u + 1, L, &c, &s);
  a = v[2]; b = v[3];
  v[2] = a * c - b * s; v[3] = a * s + b * c;
}

// Block-cooperative store of one row in the cache format.  Every thread of the block calls it
// (the FP8 scale needs a block-wide max); threads with active == false hold no channels.
__device__ __forceinline__ void pack_row(uint8_t* dst, const LayerArgs& L, int c0, const float v[4], bool active,
                                         float* scratch) {
  if (L.kv_fmt == CSA_FMT_F32) {
    if (active) *reinterpret_cast<float4*>(dst + 4 * (size_t)c0) = make_float4(v[0], v[1], v[2], v[3]);
    return;
  }
  if (L.kv_fmt == CSA_FMT_BF16) {
    if (active) store_act4(dst, CSA_FMT_BF16, c0, v);
    return;
  }
  const int dn = L.D - L.d_rope;
  float am = 0.f;
  if (active && c0 < dn) am = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
  am = block_max(am, scratch);
  float inv;
  const float sig = pow2_scale(am, &inv);
  if (!active) return;
  if (c0 < dn) {
    uint32_t w = (uint32_t)f_to_e4m3_sat(v[0] * inv) | ((uint32_t)f_to_e4m3_sat(v[1] * inv) << 8) |
                 ((uint32_t)f_to_e4m3_sat(v[2] * inv) << 16) | ((uint32_t)f_to_e4m3_sat(v[3] * inv) << 24);
    *reinterpret_cast<uint32_t*>(dst + c0) = w;
  } else {
    store_act4(dst + dn, CSA_FMT_BF16, c0 - dn, v);
  }
  if (threadIdx.x == 0) {
    *reinterpret_cast<float*>(dst + L.D + 64) = sig;
    *reinterpret_cast<uint32_t*>(dst + L.D + 68) = 0u;
    *reinterpret_cast<uint2*>(dst + L.D + 72) = make_uint2(0u, 0u);
  }
}

constexpr int kRowBatch = 8;   // rows whose loads are issued together per thread

// Block = (D/4) channel threads x RG row groups.  Row group 0 appends the new token; every row
// group pools a strided subset of the entry's source rows with an online softmax; the groups'
// partial (max, sum, weighted sum) are merged through shared memory.
__global__ void __launch_bounds__(512) append_compress_kernel(const __grid_constant__ AppendCompressArgs a) {
  __shared__ float scratch[32];
  extern __shared__ float part[];                  // [RG][3][D]
  const LayerArgs& L = a.L;
  const CacheArgs& C = a.C;
  const int j = blockIdx.x, b = blockIdx.y;
  const int CT = L.D / 4;                          // channel threads per row group
  const int RG = blockDim.x / CT;
  const int ct = threadIdx.x % CT, rg = threadIdx.x / CT;
  const int c0 = ct * 4;
  const bool lead = rg == 0;
  const int64_t t = a.q_pos[(int64_t)b * a.Tq + j];
  const int64_t r = t - L.pos0;
  if (r < 0) return;  // uniform over the block
  const size_t arow = (size_t)L.D * act_bytes(L.act_fmt);
  const bool have_new = a.x_new != nullptr;
  float x[4] = {0.f, 0.f, 0.f, 0.f}, g[4] = {0.f, 0.f, 0.f, 0.f};
  if (have_new) {
    load_act4(a.x_new + ((size_t)b * a.Tq + j) * arow, L.act_fmt, c0, x);
    load_act4(a.g_new + ((size_t)b * a.Tq + j) * arow, L.act_fmt, c0, g);
  } else if (a.do_append) {
    const int64_t s = ring_slot(r, C.raw_base, C.raw_cap);
    load_act4(C.raw + ((size_t)b * C.raw_cap + s) * arow, L.act_fmt, c0, x);
  }

  if (a.do_append) {
    if (have_new && lead) {
      const int64_t s = ring_slot(r, C.raw_base, C.raw_cap);
      store_act4(C.raw + ((size_t)b * C.raw_cap + s) * arow, L.act_fmt, c0, x);
      store_act4(C.gate + ((size_t)b * C.raw_cap + s) * arow, L.act_fmt, c0, g);
    }
    float w[4] = {x[0], x[1], x[2], x[3]};
    rope4(w, c0, L, (double)t);
    uint8_t* dst = C.window + ((size_t)b * C.window_cap + (size_t)(r % C.window_cap)) * L.row_bytes;
    pack_row(dst, L, c0, w, lead, scratch);
  }

  if (!(a.do_compress && ((r + 1) % L.m) == 0)) return;
  const int64_t i = (r + 1) / L.m - 1;
  const int64_t lo = (i - L.ov) * (int64_t)L.m;
  const int64_t r_begin = lo < 0 ? 0 : lo;
  // Online softmax in base 2 (logits pre-scaled by log2 e): per batch of rows, one max, one
  // rescale of the running sums, then one exp2 per element.  Ring slots advance incrementally.
  float mx[4], sum[4], acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) { mx[k] = -INFINITY; sum[k] = 0.f; acc[k] = 0.f; }
  const int64_t rstep = (int64_t)RG;
  int64_t slot = ring_slot(r_begin + rg, C.raw_base, C.raw_cap);
  const int64_t slot_step = rstep % C.raw_cap;
  for (int64_t rb = r_begin + rg; rb <= r; rb += rstep * kRowBatch) {
    float xv[kRowBatch][4], zv[kRowBatch][4];
#pragma unroll
    for (int u = 0; u < kRowBatch; ++u) {
      const int64_t rr = rb + (int64_t)u * rstep;
      const bool in = rr <= r;
      if (in && rr == r && have_new) {
#pragma unroll
        for (int k = 0; k < 4; ++k) { xv[u][k] = x[k]; zv[u][k] = g[k]; }
      } else if (in) {
        load_act4(C.raw + ((size_t)b * C.raw_cap + slot) * arow, L.act_fmt, c0, xv[u]);
        load_act4(C.gate + ((size_t)b * C.raw_cap + slot) * arow, L.act_fmt, c0, zv[u]);
      }
      if (in) {
        const float4 bias = __ldg(reinterpret_cast<const float4*>(a.pos_bias + (size_t)(rr - lo) * L.D + c0));
        zv[u][0] = (zv[u][0] + bias.x) * kLog2e; zv[u][1] = (zv[u][1] + bias.y) * kLog2e;
        zv[u][2] = (zv[u][2] + bias.z) * kLog2e; zv[u][3] = (zv[u][3] + bias.w) * kLog2e;
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) { xv[u][k] = 0.f; zv[u][k] = -INFINITY; }
      }
      slot += slot_step;
      if (slot >= C.raw_cap) slot -= C.raw_cap;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float bm = zv[0][k];
#pragma unroll
      for (int u = 1; u < kRowBatch; ++u) bm = fmaxf(bm, zv[u][k]);
      if (bm > mx[k]) {
        const float sc = exp2f(mx[k] - bm);
        sum[k] *= sc;
        acc[k] *= sc;
        mx[k] = bm;
      }
#pragma unroll
      for (int u = 0; u < kRowBatch; ++u) {
        const float e = exp2f(zv[u][k] - mx[k]);
        sum[k] += e;
        acc[k] = fmaf(e, xv[u][k], acc[k]);
      }
    }
  }
  // merge the row groups
  if (RG > 1) {
    float* pm = part + (size_t)rg * 3 * L.D;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      pm[c0 + k] = mx[k];
      pm[L.D + c0 + k] = sum[k];
      pm[2 * L.D + c0 + k] = acc[k];
    }
    __syncthreads();
    if (lead) {
      for (int q = 1; q < RG; ++q) {
        const float* po = part + (size_t)q * 3 * L.D;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float m2 = po[c0 + k];
          if (m2 == -INFINITY) continue;
          const float M = fmaxf(mx[k], m2);
          const float f1 = exp2f(mx[k] - M), f2 = exp2f(m2 - M);
          sum[k] = sum[k] * f1 + po[L.D + c0 + k] * f2;
          acc[k] = acc[k] * f1 + po[2 * L.D + c0 + k] * f2;
          mx[k] = M;
        }
      }
    }
  }
  float e[4] = {0.f, 0.f, 0.f, 0.f};
  float ss = 0.f;
  if (lead) {
#pragma unroll
    for (int k = 0; k < 4; ++k) { e[k] = acc[k] / sum[k]; ss += e[k] * e[k]; }
  }
  ss = block_sum(ss, scratch);
  const float rs = 1.0f / sqrtf(ss / (float)L.D + L.eps);
  const float4 gk = a.gamma_kv ? __ldg(reinterpret_cast<const float4*>(a.gamma_kv + c0)) : make_float4(1.f, 1.f, 1.f, 1.f);
  e[0] *= rs * gk.x; e[1] *= rs * gk.y; e[2] *= rs * gk.z; e[3] *= rs * gk.w;
  rope4(e, c0, L, (double)(L.pos0 + i * (int64_t)L.m));
  uint8_t* dst = C.entries + ((size_t)b * C.entry_cap + (size_t)i) * L.row_bytes;
  pack_row(dst, L, c0, e, lead, scratch);
}

}  // namespace

cudaError_t launch_append_compress(const AppendCompressArgs& a, int B, int Tq, cudaStream_t s) {
  dim3 grid(Tq, B);
  const int ct = a.L.D / 4;
  // decode: spread the entry's source rows over row groups; a chunk has parallelism across tokens
  int rg = 1;
  if (a.do_compress && Tq <= 64) {
    const int rows = (1 + a.L.ov) * a.L.m;
    rg = 512 / ct;
    while (rg > 1 && (rg / 2) * kRowBatch >= rows) rg /= 2;
  }
  const size_t smem = rg > 1 ? (size_t)rg * 3 * a.L.D * sizeof(float) : 0;
  static size_t configured = 0;
  if (smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(append_compress_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  profile_mark(s);
  append_compress_kernel<<<grid, ct * rg, smem, s>>>(a);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace csa
