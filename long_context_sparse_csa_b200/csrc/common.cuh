// Shared device helpers of the CSA/HCA kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "csa.h"

namespace csa {

constexpr float kLog2e = 1.4426950408889634f;

// ----------------------------------------------------------------------------- launch parameters
// Everything a kernel needs about one layer, flattened for __grid_constant__ use.
struct LayerArgs {
  int B, H, D, d_rope, m, ov, top_k, window, H_I, d_I;
  int kv_fmt, idx_fmt, act_fmt;
  int row_bytes;
  double rope_base;
  float eps, scale;
  int64_t pos0;
  double theta_pi[32];   // base^(-2u/d_rope) / pi, u < d_rope/2, formed on the host in float64
};

struct CacheArgs {
  uint8_t* entries;
  int64_t entry_cap;
  const uint8_t* idx_keys;
  const float* idx_key_scale;
  uint8_t* window;
  int64_t window_cap;
  uint8_t* raw;
  uint8_t* gate;
  int64_t raw_cap, raw_base;
};

// ----------------------------------------------------------------------------- scalar conversions
__device__ __forceinline__ float bf16_bits_to_f(uint32_t b) { return __uint_as_float(b << 16); }

__device__ __forceinline__ uint16_t f_to_bf16_bits(float x) {
  __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&h);
}

__device__ __forceinline__ float e4m3_to_f(uint8_t c) {
  __nv_fp8_e4m3 v;
  v.__x = c;
  return float(v);
}

// FP4 e2m1 code (low 4 bits: sign, 2 exponent bits with bias 1, 1 mantissa bit) -> float.
__device__ __forceinline__ float e2m1_to_f(uint32_t code) {
  const uint32_t e = (code >> 1) & 3u, m = code & 1u;
  const float mag = e == 0 ? 0.5f * (float)m : (1.f + 0.5f * (float)m) * (float)(1u << (e - 1));
  return (code & 8u) ? -mag : mag;
}

// Round |x| (finite) to the nearest e2m1 magnitude code 0..7, ties to the even code, saturating at 6.
// The magnitudes are 0, .5, 1, 1.5, 2, 3, 4, 6 and the midpoints between them .25, .75, 1.25, 1.75,
// 2.5, 3.5, 5: the code is the number of midpoints below |x|, moved up to the even neighbour when
// |x| sits exactly on an odd code's upper midpoint.
__device__ __forceinline__ uint32_t e2m1_rne_magnitude(float ax) {
  const float mid[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};
  uint32_t c = 0;
#pragma unroll
  for (int k = 0; k < 7; ++k) c += ax > mid[k] ? 1u : 0u;
  if (c < 7 && ax == mid[c] && (c & 1u)) ++c;
  return c;
}

__device__ __forceinline__ uint8_t f_to_e4m3_sat(float x) {
  return (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

// Smallest power of two sigma with amax / sigma <= 448 (1 for amax == 0); *inv = 1 / sigma.
// 448 = 0.875 * 2^9: with amax = f * 2^e (0.5 <= f < 1) the bound first holds at
// k = e - 9 when f <= 0.875, else at k = e - 8.
__device__ __forceinline__ float pow2_scale(float amax, float* inv) {
  if (!(amax > 0.f)) { *inv = 1.f; return 1.f; }
  int e;
  float f = frexpf(amax, &e);
  int k = (f <= 0.875f) ? e - 9 : e - 8;
  *inv = ldexpf(1.f, -k);
  return ldexpf(1.f, k);
}

// Smallest power of two sigma with amax / sigma <= 6, the FP4 maximum (1 for amax == 0); *inv = 1 /
// sigma.  6 = 0.75 * 2^3: with amax = f * 2^e (0.5 <= f < 1) the bound first holds at k = e - 3 when
// f <= 0.75, else at k = e - 2.
__device__ __forceinline__ float pow2_scale_fp4(float amax, float* inv) {
  if (!(amax > 0.f)) { *inv = 1.f; return 1.f; }
  int e;
  float f = frexpf(amax, &e);
  int k = (f <= 0.75f) ? e - 3 : e - 2;
  *inv = ldexpf(1.f, -k);
  return ldexpf(1.f, k);
}

// Rotary angle of pair u at position pos, formed in float64 as pos * theta_u; taken as
// sincospi(pos * theta_u / pi), whose argument reduction (modulo 2) is exact.  Returns float cos/sin.
__device__ __forceinline__ void rope_cos_sin(double pos, int u, const LayerArgs& L, float* c, float* s) {
  double sd, cd;
  sincospi(pos * L.theta_pi[u], &sd, &cd);
  *c = (float)cd;
  *s = (float)sd;
}

// ----------------------------------------------------------------------------- row access
// Loads 4 consecutive channels [c, c+4) of an activation row (float32 or bf16).
__device__ __forceinline__ void load_act4(const uint8_t* row, int fmt, int c, float v[4]) {
  if (fmt == CSA_FMT_F32) {
    float4 x = *reinterpret_cast<const float4*>(row + 4 * (size_t)c);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else {
    uint2 x = *reinterpret_cast<const uint2*>(row + 2 * (size_t)c);
    v[0] = bf16_bits_to_f(x.x & 0xFFFFu); v[1] = bf16_bits_to_f(x.x >> 16);
    v[2] = bf16_bits_to_f(x.y & 0xFFFFu); v[3] = bf16_bits_to_f(x.y >> 16);
  }
}

__device__ __forceinline__ void store_act4(uint8_t* row, int fmt, int c, const float v[4]) {
  if (fmt == CSA_FMT_F32) {
    *reinterpret_cast<float4*>(row + 4 * (size_t)c) = make_float4(v[0], v[1], v[2], v[3]);
  } else {
    uint2 x;
    x.x = (uint32_t)f_to_bf16_bits(v[0]) | ((uint32_t)f_to_bf16_bits(v[1]) << 16);
    x.y = (uint32_t)f_to_bf16_bits(v[2]) | ((uint32_t)f_to_bf16_bits(v[3]) << 16);
    *reinterpret_cast<uint2*>(row + 2 * (size_t)c) = x;
  }
}

__device__ __forceinline__ size_t act_bytes(int fmt) { return fmt == CSA_FMT_F32 ? 4 : 2; }

__device__ __forceinline__ int64_t ring_slot(int64_t r, int64_t base, int64_t cap) {
  int64_t s = (r - base) % cap;
  return s < 0 ? s + cap : s;
}

// ----------------------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide sum / max for blockDim.x <= 1024 (scratch: 32 floats).
__device__ __forceinline__ float block_sum(float v, float* scratch) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) scratch[wid] = v;
  __syncthreads();
  float r = (lane < nw) ? scratch[lane] : 0.f;
  return warp_sum(r);
}

__device__ __forceinline__ float block_max(float v, float* scratch) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) scratch[wid] = v;
  __syncthreads();
  float r = (lane < nw) ? scratch[lane] : -INFINITY;
  return warp_max(r);
}

// Order-preserving map of a float to uint32 (larger float -> larger key); -0 == +0.
__device__ __forceinline__ uint32_t float_key(float f) {
  f = f + 0.0f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ----------------------------------------------------------------------------- error word
enum : int {
  kErrWaitTimeout = 1,
  kErrTopkOverflow = 2,     // split top-k: appends exceeded their reserved range (inconsistent histogram)
};

__device__ __forceinline__ void set_device_error(int* err, int bits) {
  if (err) atomicOr(err, bits);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

}  // namespace csa
