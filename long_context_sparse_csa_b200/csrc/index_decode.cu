// Lightning-indexer scores for decode (one query per sequence):
//   s_i = sum_h w_h * ReLU(sigma_q,h * sigma_k,i * <q_h, k_i>)
// over every index key of the sequence, keys of 128 dims in FP8 e4m3 or in FP4 e2m1 with block
// scales, H_I = 16, 32 or 64 heads.
//
// The pages describe the indexer only in words: a cheap low-rank scorer of the compressed entries
// ("DeepSeek-V4 Explained: ...", "The attention stack, and why it is two mechanisms") made of a few
// small FP8 heads ("DeepSeek-V4, explained.", step 3) whose attention runs in FP4 ("DeepSeek-V4:
// Making a Million Tokens Affordable", "Two ways to shrink attention, interleaved").  In decode it
// reads 132 bytes per entry (68 in FP4) and does 64 FLOPs per key byte (32 heads): it is a stream
// over the key cache, built like a bandwidth kernel, with warp-level tensor-core MMAs keeping the
// FLOPs off the CUDA cores.
//
// Streaming: one producer thread per CTA copies tiles of 128 keys with the tensor memory accelerator
// into a ring of shared-memory stages (FP8: 16 KB boxes in the 128-byte swizzle; FP4: 8 KB, no
// swizzle), two CTAs per SM; each CTA takes a contiguous range of (sequence, tile) items.
//
// Scoring: four consumer warps split each tile, 32 keys each, in groups of 8.  A group is one pass of
// mma.sync m16n8k32 e4m3 -> f32 per 16 heads and 32 dims: A = the query (16 heads x 32 dims, from
// registers), B = the 8 keys (32 dims x 8 keys).  The dot product does not depend on the order of
// its 128 terms, so the MMA's k index is permuted such that lane l's share of B over the four
// k-steps is one contiguous 32-dim piece of key l/4, dims [32(l%4), 32(l%4) + 32): logical k = 4j + i
// (i < 4) of k-step t is dim 32j + 8t + i, logical k = 16 + 4j + i is dim 32j + 8t + 4 + i, for lanes
// with l%4 = j, and the query fragments are laid out with the same permutation once per sequence.
// In the 128-byte swizzle the two 16-byte pieces a lane reads fall on distinct banks across each
// quarter warp.  A lane's 32 dims are exactly one FP4 scale block, so its FP4 codes times the block's
// offset 2^-delta (delta <= 7) are exact e4m3 values: the lane converts them in registers (a byte
// permute through a table of the eight magnitudes at that offset) and the same e4m3 MMA runs; the
// key's power-of-two scale multiplies the score.
//
// Scores are written as float32 (-inf past the query's visible entries) and, for the multi-CTA
// top-k, counted into a shared 4096-bin histogram of their keys' top 12 bits, added to the
// sequence's global histogram when the CTA leaves the sequence.  Every mbarrier wait is bounded: a
// wait that gives up sets the error word and stops that warp's work, and the warp still takes every
// barrier and arrival of the schedule, so no other warp is left waiting for it.
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.h"
#include "sm100.cuh"

namespace csa {

namespace {

using namespace sm100;

constexpr int kConsumers = 4;              // consumer warps (32 keys of a tile each)
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kStages = 4;
constexpr int kTileKeys = 128;
constexpr int kDI = 128;
constexpr int kHistBins = 4096;

template <bool FP4> __host__ __device__ constexpr int tile_bytes() { return kTileKeys * (FP4 ? kDI / 2 : kDI); }
template <bool FP4> __host__ __device__ constexpr size_t smem_bytes() {
  return 1024 + (size_t)kStages * tile_bytes<FP4>() + kHistBins * 4 + 64 + 2 * kStages * 8 + 64;
}

__device__ __forceinline__ void mma_e4m3(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four FP4 codes (the low 16 bits of w, one per nibble) -> four e4m3 bytes through the table of the
// eight magnitudes at this block's offset (lut_lo: magnitudes 0..3, lut_hi: 4..7); each nibble's
// sign bit (bit 3) becomes its byte's sign bit (bit 7).
__device__ __forceinline__ uint32_t fp4x4_to_e4m3(uint32_t w, uint32_t lut_lo, uint32_t lut_hi) {
  const uint32_t mag = __byte_perm(lut_lo, lut_hi, w & 0x7777u);
  const uint32_t sgn = ((w & 0x8u) << 4) | ((w & 0x80u) << 8) | ((w & 0x800u) << 12) | ((w & 0x8000u) << 16);
  return mag | sgn;
}

// Per-sequence constants of one lane: the query's A fragments under the k permutation, and the
// scale-folded head weights of the lane's heads 16 mt + g and 16 mt + g + 8 (g = lane / 4).
template <int MT>
struct QueryFrags {
  uint32_t a[MT][4][4];      // [m-tile][k-step][a0..a3]
  float wq[MT][2];           // w_h * sigma_q,h
  bool pos;                  // every sigma_q,h >= 0 (then ReLU(qs ks v) = qs ks ReLU(v) for ks >= 0)
};

template <int MT>
__device__ __forceinline__ void load_query(const IndexArgs& a, int b, int lane, QueryFrags<MT>& f) {
  const int g = lane >> 2, j = lane & 3;
  const uint8_t* q = a.idx_q + (size_t)b * a.H_I * kDI;
  const float* qs = a.q_scale + (size_t)b * a.H_I;
  const float* w = a.head_w + (size_t)b * a.H_I;
  bool pos = true;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int h0 = 16 * mt + g, h1 = h0 + 8;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int d = 32 * j + 8 * t;
      f.a[mt][t][0] = __ldg(reinterpret_cast<const uint32_t*>(q + (size_t)h0 * kDI + d));
      f.a[mt][t][1] = __ldg(reinterpret_cast<const uint32_t*>(q + (size_t)h1 * kDI + d));
      f.a[mt][t][2] = __ldg(reinterpret_cast<const uint32_t*>(q + (size_t)h0 * kDI + d + 4));
      f.a[mt][t][3] = __ldg(reinterpret_cast<const uint32_t*>(q + (size_t)h1 * kDI + d + 4));
    }
    const float q0 = __ldg(qs + h0), q1 = __ldg(qs + h1);
    f.wq[mt][0] = __ldg(w + h0) * q0;
    f.wq[mt][1] = __ldg(w + h1) * q1;
    pos = pos && q0 >= 0.f && q1 >= 0.f;
  }
  f.pos = __all_sync(0xffffffffu, pos) != 0;
}

__device__ __forceinline__ void consumer_bar() { asm volatile("barrier.sync.aligned 1, 128;" ::: "memory"); }

// Per-lane key-side values of one tile, loaded a tile ahead: the two output keys' scales (FP8: the
// float scales; FP4: the scale words) and, for FP4, the scale word of the lane's B key.
struct TileScales {
  uint32_t ks[4][2];
  uint32_t wb[4];
};

template <int MT, bool FP4>
__global__ void __launch_bounds__(kThreads, MT == 4 ? 1 : 2)
index_score_decode_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ IndexArgs a) {
  constexpr int kTile = tile_bytes<FP4>();
  constexpr int kKeyBytes = FP4 ? kDI / 2 : kDI;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* hist = reinterpret_cast<uint32_t*>(tiles + (size_t)kStages * kTile);
  uint32_t* lut = hist + kHistBins;                             // FP4: [offset 0..7][2] e4m3 magnitude bytes
  uint64_t* full = reinterpret_cast<uint64_t*>(lut + 16);
  uint64_t* empty = full + kStages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool use_hist = a.hist != nullptr;
  const int64_t tpb = (a.n_max + kTileKeys - 1) / kTileKeys;   // tiles per sequence
  const int64_t total = (int64_t)a.B * tpb;
  const int64_t lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
  const int n = (int)(hi - lo);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);
    }
    fence_barrier_init();
    prefetch_tensormap(&kmap);
  }
  if (use_hist)
    for (int i = threadIdx.x; i < kHistBins; i += kThreads) hist[i] = 0u;
  if (FP4 && threadIdx.x < 64) {
    // e4m3 code of magnitude m of e2m1 scaled by 2^-delta: exact for every m and delta <= 7
    const float mags[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
    const int delta = threadIdx.x >> 3, m = threadIdx.x & 7;
    reinterpret_cast<uint8_t*>(lut)[threadIdx.x] = f_to_e4m3_sat(mags[m] * __uint_as_float((uint32_t)(127 - delta) << 23));
  }
  __syncthreads();

  if (warp == kConsumers) {
    // ------------------------------------------------------------------ producer (lane 0)
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      for (int it = 0; it < n; ++it) {
        const int s = it % kStages;
        if (it >= kStages) ok = mbar_wait(&empty[s], (uint32_t)(((it / kStages) - 1) & 1));
        if (!ok) break;
        const int64_t item = lo + it;
        const int64_t b = item / tpb, t = item - b * tpb;
        mbar_arrive_expect_tx(&full[s], (uint32_t)kTile);
        tma_load_2d(tiles + (size_t)s * kTile, &kmap, &full[s], 0, (int)(b * a.entry_cap + t * kTileKeys));
        issued = it + 1;
      }
      if (!ok) set_device_error(a.err, kErrWaitTimeout);
      // every copy this thread issued lands before it leaves (bounded waits): a copy never outlives
      // the CTA, whatever the consumers did
      for (int it = issued - kStages > 0 ? issued - kStages : 0; it < issued; ++it)
        mbar_wait(&full[it % kStages], (uint32_t)((it / kStages) & 1));
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int g = lane >> 2, j = lane & 3;
  bool ok = true;
  int b_cur = -1;
  QueryFrags<MT> f;
  int64_t nv = 0;
  float* out = nullptr;
  auto load_scales = [&](int it, TileScales& d) {
    const int64_t item = lo + it;
    const int64_t b = item / tpb, t = item - b * tpb;
    const uint32_t* ksb = reinterpret_cast<const uint32_t*>(a.k_scale) + (size_t)b * a.entry_cap;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int64_t e0 = t * kTileKeys + 32 * warp + 8 * q;
      const int64_t eo = e0 + 2 * j, ei = e0 + g;
      d.ks[q][0] = eo < a.n_max ? __ldg(ksb + eo) : 0u;
      d.ks[q][1] = eo + 1 < a.n_max ? __ldg(ksb + eo + 1) : 0u;
      d.wb[q] = (FP4 && ei < a.n_max) ? __ldg(ksb + ei) : 0u;
    }
  };
  auto flush = [&](int b) {
    if (!use_hist) return;
    consumer_bar();
    uint32_t* dst = a.hist + (size_t)b * kHistBins;
    for (int i = threadIdx.x; i < kHistBins; i += 32 * kConsumers) {
      const uint32_t v = hist[i];
      if (v) {
        atomicAdd(dst + i, v);
        hist[i] = 0u;
      }
    }
    consumer_bar();
  };
  TileScales nxt;
  if (n > 0) load_scales(0, nxt);
  for (int it = 0; it < n; ++it) {
    const int s = it % kStages;
    const int64_t item = lo + it;
    const int b = (int)(item / tpb);
    const int64_t t = item - (int64_t)b * tpb;
    if (b != b_cur) {                                        // same item index in every consumer warp
      if (b_cur >= 0) flush(b_cur);
      b_cur = b;
      load_query<MT>(a, b, lane, f);
      const int64_t r1 = a.q_pos[b] - a.pos0 + 1;
      nv = r1 > 0 ? r1 / a.m : 0;
      nv = nv < a.n_max ? nv : a.n_max;
      out = a.scores + (size_t)b * a.n_max;
    }
    const TileScales cur = nxt;
    if (it + 1 < n) load_scales(it + 1, nxt);
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (uint32_t)((it / kStages) & 1))) != 0;
    const uint8_t* tile = tiles + (size_t)s * kTile;
    if (ok) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int r = 32 * warp + 8 * q + g;                 // this lane's key (B column) in the tile
        uint32_t bw[8];
        float k0s, k1s;
        if (FP4) {
          const uint4 c4 = *reinterpret_cast<const uint4*>(tile + r * kKeyBytes + 16 * j);
          const uint32_t delta = (cur.wb[q] >> (8 + 4 * j)) & 7u;
          const uint32_t lut_lo = lut[2 * delta], lut_hi = lut[2 * delta + 1];
          const uint32_t cw[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            bw[2 * u] = fp4x4_to_e4m3(cw[u], lut_lo, lut_hi);
            bw[2 * u + 1] = fp4x4_to_e4m3(cw[u] >> 16, lut_lo, lut_hi);
          }
          // the two output keys' scales: the exponents of their scale words
          k0s = __uint_as_float((cur.ks[q][0] & 0xFFu) << 23);
          k1s = __uint_as_float((cur.ks[q][1] & 0xFFu) << 23);
        } else {
          // 128-byte swizzle: 16-byte piece c of row r sits at r*128 + ((c ^ (r & 7)) << 4)
          const uint4 p0 = *reinterpret_cast<const uint4*>(tile + r * 128 + (((2 * j) ^ (r & 7)) << 4));
          const uint4 p1 = *reinterpret_cast<const uint4*>(tile + r * 128 + (((2 * j + 1) ^ (r & 7)) << 4));
          bw[0] = p0.x; bw[1] = p0.y; bw[2] = p0.z; bw[3] = p0.w;
          bw[4] = p1.x; bw[5] = p1.y; bw[6] = p1.z; bw[7] = p1.w;
          k0s = __uint_as_float(cur.ks[q][0]);
          k1s = __uint_as_float(cur.ks[q][1]);
        }
        float c[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          c[mt][0] = c[mt][1] = c[mt][2] = c[mt][3] = 0.f;
#pragma unroll
          for (int tt = 0; tt < 4; ++tt) mma_e4m3(c[mt], f.a[mt][tt], bw[2 * tt], bw[2 * tt + 1]);
        }
        // c[mt][0..1]: head 16mt + g, keys 2j, 2j+1 of the group; c[mt][2..3]: head 16mt + g + 8
        float s0 = 0.f, s1 = 0.f;
        if (f.pos && k0s >= 0.f && k1s >= 0.f) {
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            s0 = fmaf(f.wq[mt][0], fmaxf(c[mt][0], 0.f), s0);
            s0 = fmaf(f.wq[mt][1], fmaxf(c[mt][2], 0.f), s0);
            s1 = fmaf(f.wq[mt][0], fmaxf(c[mt][1], 0.f), s1);
            s1 = fmaf(f.wq[mt][1], fmaxf(c[mt][3], 0.f), s1);
          }
          s0 *= k0s;
          s1 *= k1s;
        } else {
          // a negative scale somewhere: the ReLU sees qs * ks * v head by head
          const float* qs_b = a.q_scale + (size_t)b * a.H_I;
          const float* w_b = a.head_w + (size_t)b * a.H_I;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            const int h0 = 16 * mt + g, h1 = h0 + 8;
            const float w0 = __ldg(w_b + h0), w1 = __ldg(w_b + h1), q0 = __ldg(qs_b + h0), q1 = __ldg(qs_b + h1);
            s0 += w0 * fmaxf(c[mt][0] * (q0 * k0s), 0.f) + w1 * fmaxf(c[mt][2] * (q1 * k0s), 0.f);
            s1 += w0 * fmaxf(c[mt][1] * (q0 * k1s), 0.f) + w1 * fmaxf(c[mt][3] * (q1 * k1s), 0.f);
          }
        }
        // sum over the 8 lanes holding the other heads of the same keys (same j)
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          s0 += __shfl_xor_sync(0xffffffffu, s0, o);
          s1 += __shfl_xor_sync(0xffffffffu, s1, o);
        }
        if (lane < 8) {                                     // lane g*4 + j, g < 2: key 2j + g
          const int64_t e = t * kTileKeys + 32 * warp + 8 * q + 2 * j + g;
          const float v = g ? s1 : s0;
          if (e < a.n_max) {
            const bool vis = e < nv;
            out[e] = vis ? v : -INFINITY;
            if (use_hist && vis) atomicAdd(&hist[float_key(v) >> 20], 1u);
          }
        }
      }
    }
    // every shared-memory read of the stage has completed (its values went through the MMAs): hand
    // the stage back to the producer
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  if (b_cur >= 0) flush(b_cur);
  if (!ok && lane == 0) set_device_error(a.err, kErrWaitTimeout);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

bool index_decode_supported(int idx_fmt, int H_I, int d_I) {
  return (idx_fmt == CSA_FMT_E4M3 || idx_fmt == CSA_FMT_E2M1) && d_I == kDI && (H_I == 16 || H_I == 32 || H_I == 64);
}

cudaError_t launch_index_decode(const IndexArgs& a, int num_sms, cudaStream_t s) {
  if (a.n_max <= 0 || a.B <= 0) return cudaSuccess;
  if (a.H_I != 16 && a.H_I != 32 && a.H_I != 64) return cudaErrorInvalidValue;
  const bool fp4 = a.idx_fmt == CSA_FMT_E2M1;
  // keys as a 2D byte tensor [B * entry_cap][key bytes], boxes of 128 keys (rows past the end read 0)
  auto fn = encode_fn();
  if (!fn) return cudaErrorInvalidValue;
  CUtensorMap kmap;
  const cuuint64_t kb = fp4 ? kDI / 2 : kDI;
  cuuint64_t dims[2] = {kb, (cuuint64_t)a.B * (cuuint64_t)a.entry_cap};
  cuuint64_t strides[1] = {kb};
  cuuint32_t box[2] = {(cuuint32_t)kb, (cuuint32_t)kTileKeys};
  cuuint32_t es[2] = {1, 1};
  if (fn(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.idx_k), dims, strides, box, es,
         CU_TENSOR_MAP_INTERLEAVE_NONE, fp4 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int64_t items = (int64_t)a.B * ((a.n_max + kTileKeys - 1) / kTileKeys);
  int64_t grid = 2 * (int64_t)num_sms;
  if (grid > items) grid = items;
  auto kern = fp4 ? (a.H_I == 16 ? index_score_decode_kernel<1, true> : a.H_I == 32 ? index_score_decode_kernel<2, true>
                                                                                    : index_score_decode_kernel<4, true>)
                  : (a.H_I == 16 ? index_score_decode_kernel<1, false> : a.H_I == 32 ? index_score_decode_kernel<2, false>
                                                                                     : index_score_decode_kernel<4, false>);
  const size_t smem = fp4 ? smem_bytes<true>() : smem_bytes<false>();
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, dim3((unsigned)grid), dim3(kThreads), smem, s, 0, kmap, a);
}

}  // namespace csa
