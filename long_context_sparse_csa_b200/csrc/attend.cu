// Shared-KV multi-query attention over gathered KV rows with a sink logit.
//
// What it computes ("DeepSeek-V4: Making a Million Tokens Affordable", section "Two ways to
// shrink attention, interleaved"):
// - each compressed entry is both the key and the value;
// - queries and entries are RMS-normalised;
// - the output is rotated back by the query's position (RoPE at -t), so it depends only on relative
//   positions;
// - a learned per-head sink logit lets a head put part of its attention weight on nothing.
// Step 8 of "DeepSeek-V4, explained." has heads that share keys read the same contiguous rows: here
// every gathered row is loaded once per CTA and serves all of the CTA's heads.
//
// Key slots of a query at raw row r_t: [0, n_sel) are compressed entries
// (the top-k list for CSA, -1 skipped; every visible entry for HCA), then
// [n_sel, n_sel + n_win) are the window rows r_t - n_win + 1 .. r_t.
//
// Tensor-core kernel (D = 512, BF16 or mixed BF16/FP8 rows): a CTA owns one
// query, a group of HG heads (M = HG) and a contiguous range of 64-slot key
// tiles.  Each tile is gathered row by row (16-byte vector loads; FP8 codes
// times the row's power-of-two scale convert exactly to BF16) into a swizzled
// shared-memory tile, S = Q K^T and O += P V run as bf16 mma.sync with fp32
// accumulation and an online softmax.  When several CTAs split one query's
// slots, each writes (O, m, l) and a combine kernel merges the splits with
// the sink and applies the inverse rotation.
#include <cooperative_groups.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.h"
#include "sm100.cuh"

namespace cg = cooperative_groups;

namespace csa {

namespace {

constexpr int kD = 512;
constexpr int kTile = 64;
constexpr int kH128 = 128;

#ifdef CSA_TRACE
__device__ uint64_t g_trace_a[320][16];
#define ATRACE(slot) do { if (threadIdx.x == 0 && blockIdx.z == 0 && blockIdx.y == 0 && blockIdx.x < 320) { \
    uint64_t _t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(_t) :: "memory"); g_trace_a[blockIdx.x][(slot)] = _t; } } while (0)
#define ATRACE_C(thr, slot) do { if (threadIdx.x == (thr) && blockIdx.z == 0 && blockIdx.y == 0 && blockIdx.x < 320) \
    g_trace_a[blockIdx.x][(slot)] = (uint64_t)clock64(); } while (0)
#define ATRACE_T(thr, slot) do { if (threadIdx.x == (thr) && blockIdx.z == 0 && blockIdx.y == 0 && blockIdx.x < 320) { \
    uint64_t _t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(_t) :: "memory"); g_trace_a[blockIdx.x][(slot)] = _t; } } while (0)
__device__ uint64_t g_trace_cb[256][4];
#define CBTRACE(slot) do { if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.x < 256) { \
    uint64_t _t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(_t) :: "memory"); g_trace_cb[blockIdx.x][(slot)] = _t; } } while (0)
#else
#define ATRACE(slot) ((void)0)
#define ATRACE_T(thr, slot) ((void)0)
#define ATRACE_C(thr, slot) ((void)0)
#define CBTRACE(slot) ((void)0)
#endif

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg_nc_v4(const uint8_t* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack_f16x2(uint32_t w) {
  return __half22float2(*reinterpret_cast<const __half2*>(&w));
}

// 2^e as a float, for integer e in [-126, 127] (built from the exponent field: exact).
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((e + 127) << 23); }

// Two e4m3 codes (low byte first) -> two floats, via the hardware e4m3x2 -> f16x2 conversion.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t codes) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)codes, __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// Swizzled byte offset of 16-byte chunk `ch` of row `row` in a tile whose rows are `pitch` bytes.
__device__ __forceinline__ uint32_t swz(int row, int ch, int pitch) {
  return (uint32_t)(row * pitch + (((ch ^ (row & 7))) << 4));
}

struct SlotInfo {
  int64_t rt, n_sel, n_win, R;
  int64_t wlast;             // last window row attended (r_t, or r_t - 1 when deferred)
};

__device__ __forceinline__ SlotInfo slot_info(const AttendArgs& a, int64_t t) {
  SlotInfo s;
  s.rt = t - a.L.pos0;
  const int64_t r1 = s.rt + 1 > 0 ? s.rt + 1 : 0;
  const int64_t nvis = r1 / a.L.m;
  s.n_sel = a.topk ? (int64_t)a.L.top_k : (nvis < a.n_max ? nvis : a.n_max);
  s.n_win = a.no_window ? 0 : (r1 < a.L.window ? r1 : a.L.window);
  s.wlast = s.rt;
  if (a.defer_new && !a.topk) {
    // this step's own rows join in the combine: the entry the token completes, and its window row
    if (r1 > 0 && r1 % a.L.m == 0 && nvis <= a.n_max && s.n_sel > 0) s.n_sel -= 1;
    if (s.n_win > 0) {
      s.n_win -= 1;
      s.wlast = s.rt - 1;
    }
  }
  s.R = s.n_sel + s.n_win;
  return s;
}

// Stored row of key slot s, or null when the slot holds nothing (-1 or out of range).
__device__ __forceinline__ const uint8_t* slot_row(const AttendArgs& a, const SlotInfo& si, int row, int b,
                                                   int64_t s) {
  const CacheArgs& C = a.C;
  if (s < si.n_sel) {
    const int64_t e = a.topk ? (int64_t)a.topk[(size_t)row * a.L.top_k + s] - a.entry_offset : s;
    if (e < 0 || e >= a.entry_limit) return nullptr;
    return C.entries + ((size_t)b * C.entry_cap + (size_t)e) * a.L.row_bytes;
  }
  if (s < si.R) {
    const int64_t wr = si.wlast - si.n_win + 1 + (s - si.n_sel);
    return C.window + ((size_t)b * C.window_cap + (size_t)(wr % C.window_cap)) * a.L.row_bytes;
  }
  return nullptr;
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit_wait() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int HG, int FMT>
__global__ void __launch_bounds__(HG * 8, 1) attend_mma_kernel(const __grid_constant__ AttendArgs a) {
  constexpr int NW = HG / 4;          // warps
  constexpr int NT = NW * 32;         // threads
  constexpr int MT = HG / 16;         // m-tiles (16 heads each)
  constexpr int DW = kD / NW;         // output dims per warp in P*V
  constexpr int NTW = DW / 8;         // n-tiles per warp in P*V

  // bf16 rows need no conversion: they arrive by asynchronous copies into two tile buffers, the
  // next tile's copies in flight while the current tile is computed
  constexpr bool kAsync = FMT == CSA_FMT_BF16;
  constexpr int kBufs = kAsync ? 2 : 1;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* Qs = smem;                                   // [HG][1024]  bf16 q~
  uint8_t* Kbuf = Qs + HG * 1024;                       // [kBufs][64][1024]  bf16 key/value tiles
  uint8_t* Ks = Kbuf;                                   // the current tile
  uint8_t* Ps = Kbuf + kBufs * kTile * 1024;            // [HG][128]   bf16 probabilities
  float* pmax = reinterpret_cast<float*>(Ps + HG * 128);  // [4][HG]
  float* psum = pmax + 4 * HG;                          // [4][HG]
  float* m_run = psum + 4 * HG;                         // [HG]
  float* l_run = m_run + HG;                            // [HG]
  float* corr = l_run + HG;                             // [HG]
  float* cs = corr + HG;                                // [32]
  float* sn = cs + 32;                                  // [32]
  const uint8_t** rowbuf = reinterpret_cast<const uint8_t**>(sn + 32);  // [kBufs][64]
  const uint8_t** rowptr = rowbuf;                      // rows of the current tile

  const LayerArgs& L = a.L;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tq = lane & 3;
  const int row = blockIdx.z, hg = blockIdx.y, sp = blockIdx.x;
  const int b = row / a.Tq;
  const int64_t t = a.q_pos[row];
  const SlotInfo si = slot_info(a, t);
  const int64_t T = (si.R + kTile - 1) / kTile;
  const int64_t t0 = T * sp / a.splits, t1 = T * (sp + 1) / a.splits;
  const float cl2 = L.scale * kLog2e;
  ATRACE(0);

  if (tid < 32) {
    float c, s;
    rope_cos_sin((double)t, tid, L, &c, &s);
    cs[tid] = c;
    sn[tid] = s;
  }
  if (tid < HG) { m_run[tid] = -INFINITY; l_run[tid] = 0.f; }
  __syncthreads();

  // ---------------------------------------------------------------- key/value tile gather
  // gather_load issues every 16-byte load of a 64-row tile into registers; gather_store converts
  // (FP8 codes x the row's power-of-two scale -> bf16, exact) into the swizzled shared tile.  The
  // first tile's loads are issued before the query prologue so their latency is hidden by it.
  constexpr int kChunksRow = FMT == CSA_FMT_BF16 ? 64 : 36;
  constexpr int kPer = (kTile * kChunksRow + NT - 1) / NT;
  struct Gl { uint4 c[kPer]; float sig[kPer]; };
  auto gather_load = [&](Gl& g) {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int idx = tid + u * NT;
      g.c[u] = make_uint4(0u, 0u, 0u, 0u);
      g.sig[u] = 0.f;
      if (idx < kTile * kChunksRow) {
        const int rr = idx / kChunksRow, ch = idx % kChunksRow;
        const uint8_t* p = rowptr[rr];
        if (p) {
          if (FMT == CSA_FMT_BF16) {
            g.c[u] = ldg_nc_v4(p + ch * 16);
          } else {
            g.c[u] = ldg_nc_v4(p + (ch < 28 ? ch * 16 : (kD - 64) + (ch - 28) * 16));
            if (ch < 28) g.sig[u] = __ldg(reinterpret_cast<const float*>(p + kD + 64));
          }
        }
      }
    }
  };
  auto gather_store = [&](const Gl& g) {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int idx = tid + u * NT;
      if (idx >= kTile * kChunksRow) break;
      const int rr = idx / kChunksRow, ch = idx % kChunksRow;
      if (FMT == CSA_FMT_BF16) {
        *reinterpret_cast<uint4*>(Ks + swz(rr, ch, 1024)) = g.c[u];
      } else if (ch < 28) {
        const uint32_t w[4] = {g.c[u].x, g.c[u].y, g.c[u].z, g.c[u].w};
        uint32_t outw[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 lo = e4m3x2_to_float2((uint16_t)(w[q] & 0xFFFFu));
          const float2 hi = e4m3x2_to_float2((uint16_t)(w[q] >> 16));
          outw[2 * q] = pack_bf16x2(lo.x * g.sig[u], lo.y * g.sig[u]);
          outw[2 * q + 1] = pack_bf16x2(hi.x * g.sig[u], hi.y * g.sig[u]);
        }
        *reinterpret_cast<uint4*>(Ks + swz(rr, 2 * ch, 1024)) = make_uint4(outw[0], outw[1], outw[2], outw[3]);
        *reinterpret_cast<uint4*>(Ks + swz(rr, 2 * ch + 1, 1024)) = make_uint4(outw[4], outw[5], outw[6], outw[7]);
      } else {
        *reinterpret_cast<uint4*>(Ks + swz(rr, 56 + (ch - 28), 1024)) = g.c[u];
      }
    }
  };
  // kAsync: every 16-byte piece of a 64-row tile by an asynchronous copy (empty slots -> zero rows)
  auto gather_async = [&](uint8_t* dst, const uint8_t* const* rp) {
    for (int idx = tid; idx < kTile * 64; idx += NT) {
      const int rr = idx >> 6, ch = idx & 63;
      uint8_t* d = dst + swz(rr, ch, 1024);
      const uint8_t* p = rp[rr];
      if (p) cp_async16(d, p + ch * 16);
      else *reinterpret_cast<uint4*>(d) = make_uint4(0u, 0u, 0u, 0u);
    }
  };
  Gl gl;
  if (t0 < t1) {
    if (tid < kTile) rowptr[tid] = slot_row(a, si, row, b, t0 * kTile + tid);
    __syncthreads();
    if constexpr (kAsync) {
      gather_async(Kbuf, rowbuf);
      cp_async_commit();
    } else {
      gather_load(gl);
    }
  }

  // ---------------------------------------------------------------- q~ = RoPE_t(RMSNorm(q) * gamma_q), bf16
  // Each warp owns HG/NW heads; lane l holds dims [16l, 16l+16).  All of the warp's loads (its
  // heads' q values and gamma) are issued before any head is normalised.
  {
    constexpr int HPW = HG / NW;
    const size_t ab = L.act_fmt == CSA_FMT_F32 ? 4 : 2;
    float gm[16];
    if (a.gamma_q) {
#pragma unroll
      for (int k = 0; k < 16; k += 4) {
        const float4 g4 = __ldg(reinterpret_cast<const float4*>(a.gamma_q + 16 * lane + k));
        gm[k] = g4.x; gm[k + 1] = g4.y; gm[k + 2] = g4.z; gm[k + 3] = g4.w;
      }
    } else {
#pragma unroll
      for (int k = 0; k < 16; ++k) gm[k] = 1.f;
    }
    float v[HPW][16];
#pragma unroll
    for (int i = 0; i < HPW; ++i) {
      const int h = hg * HG + warp + i * NW;
      const uint8_t* qrow = a.q + ((size_t)row * L.H + h) * kD * ab;
      if (L.act_fmt == CSA_FMT_F32) {
#pragma unroll
        for (int k = 0; k < 16; k += 4) load_act4(qrow, CSA_FMT_F32, 16 * lane + k, v[i] + k);
      } else {
        const uint4 u0 = __ldg(reinterpret_cast<const uint4*>(qrow + 2 * 16 * lane));
        const uint4 u1 = __ldg(reinterpret_cast<const uint4*>(qrow + 2 * 16 * lane + 16));
        const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) { v[i][2 * k] = bf16_bits_to_f(w[k] & 0xFFFFu); v[i][2 * k + 1] = bf16_bits_to_f(w[k] >> 16); }
      }
    }
#pragma unroll
    for (int i = 0; i < HPW; ++i) {
      const int hh = warp + i * NW;
      float ss = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) ss += v[i][k] * v[i][k];
      ss = warp_sum(ss);
      const float rs = 1.0f / sqrtf(ss / (float)kD + L.eps);
#pragma unroll
      for (int k = 0; k < 16; ++k) v[i][k] *= rs * gm[k];
      if (lane >= 28) {
#pragma unroll
        for (int k = 0; k < 16; k += 2) {
          const int u = (16 * lane + k - (kD - 64)) >> 1;
          const float x0 = v[i][k], x1 = v[i][k + 1];
          v[i][k] = x0 * cs[u] - x1 * sn[u];
          v[i][k + 1] = x0 * sn[u] + x1 * cs[u];
        }
      }
      uint4 p0, p1;
      p0.x = pack_bf16x2(v[i][0], v[i][1]); p0.y = pack_bf16x2(v[i][2], v[i][3]);
      p0.z = pack_bf16x2(v[i][4], v[i][5]); p0.w = pack_bf16x2(v[i][6], v[i][7]);
      p1.x = pack_bf16x2(v[i][8], v[i][9]); p1.y = pack_bf16x2(v[i][10], v[i][11]);
      p1.z = pack_bf16x2(v[i][12], v[i][13]); p1.w = pack_bf16x2(v[i][14], v[i][15]);
      *reinterpret_cast<uint4*>(Qs + swz(hh, 2 * lane, 1024)) = p0;
      *reinterpret_cast<uint4*>(Qs + swz(hh, 2 * lane + 1, 1024)) = p1;
    }
  }

  float o[MT][NTW][4];
#pragma unroll
  for (int i = 0; i < MT; ++i)
#pragma unroll
    for (int j = 0; j < NTW; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) o[i][j][k] = 0.f;
  __syncthreads();

  const int mt = warp >> 2, np = warp & 3;   // S-phase tile of this warp: heads mt*16.., slots np*16..
  ATRACE(1);
  int ti = 0;
  for (int64_t tile = t0; tile < t1; ++tile, ++ti) {
    if constexpr (kAsync) {
      const int cur = ti & 1;
      Ks = Kbuf + cur * kTile * 1024;
      rowptr = rowbuf + cur * kTile;
      if (tile + 1 < t1) {
        // the other buffer was last read by the previous tile, which ended with a block barrier
        const uint8_t** rp = rowbuf + (cur ^ 1) * kTile;
        if (tid < kTile) rp[tid] = slot_row(a, si, row, b, (tile + 1) * kTile + tid);
        __syncthreads();
        gather_async(Kbuf + (cur ^ 1) * kTile * 1024, rp);
        cp_async_commit();
        cp_async_wait_group<1>();        // this tile's copies: the older group
      } else {
        cp_async_wait_group<0>();
      }
      __syncthreads();
    } else {
      if (tile != t0) {
        if (tid < kTile) rowptr[tid] = slot_row(a, si, row, b, tile * kTile + tid);
        __syncthreads();
        gather_load(gl);
      }
      gather_store(gl);
      __syncthreads();
    }
    if (ti < 2) ATRACE(2 + 4 * ti);

    // ------------------------------------------------------------ S = Q K^T for (heads mt*16.., slots np*16..)
    float sacc[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k) sacc[i][k] = 0.f;
    {
      const int mi = lane >> 3;
      const int qrow = mt * 16 + (lane & 7) + ((mi & 1) << 3);
      const int krow = np * 16 + (lane & 7) + ((mi >> 1) << 3);
#pragma unroll 8
      for (int ks = 0; ks < kD / 16; ++ks) {
        uint32_t af[4], b0, b1, b2, b3;
        ldsm_x4(smem_addr(Qs + swz(qrow, 2 * ks + (mi >> 1), 1024)), af[0], af[1], af[2], af[3]);
        ldsm_x4(smem_addr(Ks + swz(krow, 2 * ks + (mi & 1), 1024)), b0, b1, b2, b3);
        mma_bf16(sacc[0], af, b0, b1);
        mma_bf16(sacc[1], af, b2, b3);
      }
    }
    float pm0 = -INFINITY, pm1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int col = np * 16 + nt * 8 + 2 * tq + (i & 1);
        const float v = rowptr[col] ? sacc[nt][i] * cl2 : -INFINITY;
        sacc[nt][i] = v;
        if (i < 2) pm0 = fmaxf(pm0, v); else pm1 = fmaxf(pm1, v);
      }
    if (ti < 2) ATRACE(3 + 4 * ti);
    pm0 = fmaxf(pm0, __shfl_xor_sync(0xffffffffu, pm0, 1));
    pm0 = fmaxf(pm0, __shfl_xor_sync(0xffffffffu, pm0, 2));
    pm1 = fmaxf(pm1, __shfl_xor_sync(0xffffffffu, pm1, 1));
    pm1 = fmaxf(pm1, __shfl_xor_sync(0xffffffffu, pm1, 2));
    if (tq == 0) {
      pmax[np * HG + mt * 16 + g] = pm0;
      pmax[np * HG + mt * 16 + g + 8] = pm1;
    }
    __syncthreads();
    if (tid < HG) {
      const float tm = fmaxf(fmaxf(pmax[tid], pmax[HG + tid]), fmaxf(pmax[2 * HG + tid], pmax[3 * HG + tid]));
      const float mo = m_run[tid];
      const float mn = fmaxf(mo, tm);
      corr[tid] = (mn == -INFINITY) ? 1.f : exp2f(mo - mn);
      m_run[tid] = mn;
    }
    __syncthreads();

    // ------------------------------------------------------------ P = exp2(S - m), bf16 into shared memory
    {
      const float mn0 = m_run[mt * 16 + g], mn1 = m_run[mt * 16 + g + 8];
      float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int col = np * 16 + nt * 8 + 2 * tq;
        const float p0 = mn0 == -INFINITY ? 0.f : exp2f(sacc[nt][0] - mn0);
        const float p1 = mn0 == -INFINITY ? 0.f : exp2f(sacc[nt][1] - mn0);
        const float p2 = mn1 == -INFINITY ? 0.f : exp2f(sacc[nt][2] - mn1);
        const float p3 = mn1 == -INFINITY ? 0.f : exp2f(sacc[nt][3] - mn1);
        const uint32_t w01 = pack_bf16x2(p0, p1), w23 = pack_bf16x2(p2, p3);
        ps0 += bf16_bits_to_f(w01 & 0xFFFFu) + bf16_bits_to_f(w01 >> 16);
        ps1 += bf16_bits_to_f(w23 & 0xFFFFu) + bf16_bits_to_f(w23 >> 16);
        const int h0 = mt * 16 + g, h1 = h0 + 8;
        *reinterpret_cast<uint32_t*>(Ps + swz(h0, col >> 3, 128) + (col & 7) * 2) = w01;
        *reinterpret_cast<uint32_t*>(Ps + swz(h1, col >> 3, 128) + (col & 7) * 2) = w23;
      }
      ps0 += __shfl_xor_sync(0xffffffffu, ps0, 1);
      ps0 += __shfl_xor_sync(0xffffffffu, ps0, 2);
      ps1 += __shfl_xor_sync(0xffffffffu, ps1, 1);
      ps1 += __shfl_xor_sync(0xffffffffu, ps1, 2);
      if (tq == 0) {
        psum[np * HG + mt * 16 + g] = ps0;
        psum[np * HG + mt * 16 + g + 8] = ps1;
      }
    }
    __syncthreads();
    if (tid < HG)
      l_run[tid] = l_run[tid] * corr[tid] + (psum[tid] + psum[HG + tid]) + (psum[2 * HG + tid] + psum[3 * HG + tid]);

    if (ti < 2) ATRACE(4 + 4 * ti);
    // ------------------------------------------------------------ O = O * corr + P V (warp owns dims warp*DW..)
#pragma unroll
    for (int m2 = 0; m2 < MT; ++m2) {
      const float c0 = corr[m2 * 16 + g], c1 = corr[m2 * 16 + g + 8];
#pragma unroll
      for (int j = 0; j < NTW; ++j) {
        o[m2][j][0] *= c0; o[m2][j][1] *= c0;
        o[m2][j][2] *= c1; o[m2][j][3] *= c1;
      }
    }
    {
      const int mi = lane >> 3;
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk) {
        uint32_t pa[MT][4];
#pragma unroll
        for (int m2 = 0; m2 < MT; ++m2) {
          const int prow = m2 * 16 + (lane & 7) + ((mi & 1) << 3);
          ldsm_x4(smem_addr(Ps + swz(prow, 2 * kk + (mi >> 1), 128)), pa[m2][0], pa[m2][1], pa[m2][2], pa[m2][3]);
        }
        const int krow = kk * 16 + (lane & 7) + ((mi & 1) << 3);
#pragma unroll
        for (int n2 = 0; n2 < NTW / 2; ++n2) {
          uint32_t b0, b1, b2, b3;
          const int ch = (warp * DW + n2 * 16) / 8 + (mi >> 1);
          ldsm_x4_t(smem_addr(Ks + swz(krow, ch, 1024)), b0, b1, b2, b3);
#pragma unroll
          for (int m2 = 0; m2 < MT; ++m2) {
            mma_bf16(o[m2][2 * n2], pa[m2], b0, b1);
            mma_bf16(o[m2][2 * n2 + 1], pa[m2], b2, b3);
          }
        }
      }
    }
    __syncthreads();
  }

  ATRACE(10);
  // ---------------------------------------------------------------- epilogue
  if (a.splits > 1) {
    float* part = a.part + (((size_t)row * (L.H / HG) + hg) * a.splits + sp) * (size_t)(HG * (kD + 2));
#pragma unroll
    for (int m2 = 0; m2 < MT; ++m2)
#pragma unroll
      for (int j = 0; j < NTW; ++j) {
        const int dim = warp * DW + j * 8 + 2 * tq;
        const int h0 = m2 * 16 + g;
        *reinterpret_cast<float2*>(part + (size_t)h0 * kD + dim) = make_float2(o[m2][j][0], o[m2][j][1]);
        *reinterpret_cast<float2*>(part + (size_t)(h0 + 8) * kD + dim) = make_float2(o[m2][j][2], o[m2][j][3]);
      }
    if (tid < HG) {
      part[HG * kD + tid] = m_run[tid];
      part[HG * kD + HG + tid] = l_run[tid];
    }
    ATRACE(11);
    return;
  }
  // single split: merge the sink, normalise, rotate back by -t, store
  if (tid < HG) {
    const float sk = a.sinks[hg * HG + tid] * kLog2e;
    const float mo = m_run[tid];
    const float M = fmaxf(mo, sk);
    const float den = l_run[tid] * exp2f(mo - M) + exp2f(sk - M);
    corr[tid] = exp2f(mo - M) / den;
  }
  __syncthreads();
#pragma unroll
  for (int m2 = 0; m2 < MT; ++m2)
#pragma unroll
    for (int j = 0; j < NTW; ++j) {
      const int dim = warp * DW + j * 8 + 2 * tq;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int hl = m2 * 16 + g + half * 8;
        float x0 = o[m2][j][2 * half] * corr[hl], x1 = o[m2][j][2 * half + 1] * corr[hl];
        if (dim >= kD - 64) {
          const int u = (dim - (kD - 64)) >> 1;
          const float c = cs[u], s = sn[u];
          const float y0 = x0 * c + x1 * s, y1 = -x0 * s + x1 * c;
          x0 = y0; x1 = y1;
        }
        const size_t off = ((size_t)row * L.H + hg * HG + hl) * kD + dim;
        if (L.act_fmt == CSA_FMT_F32) {
          *reinterpret_cast<float2*>(a.out + off * 4) = make_float2(x0, x1);
        } else {
          *reinterpret_cast<uint32_t*>(a.out + off * 2) = pack_bf16x2(x0, x1);
        }
      }
    }
}

// Merge the splits of one (query, head): sink, normalisation, inverse rotation.  The split
// maxima and sums are staged in shared memory first, so every partial-output load of the
// weighted sum is independent and can be in flight together.
template <int HG>
__global__ void __launch_bounds__(512) attend_combine_kernel(const __grid_constant__ AttendArgs a) {
  constexpr int kGroups = 4;                       // split groups; 128 dim-threads each
  __shared__ float fac[1024];
  __shared__ float s_inv;
  __shared__ float4 red[kGroups - 1][kD / 4];
  const LayerArgs& L = a.L;
  const int h = blockIdx.x, row = blockIdx.y;
  const int hg = h / HG, hl = h % HG;
  const size_t pstride = (size_t)HG * (kD + 2);
  const float* base = a.part + ((size_t)row * (L.H / HG) + hg) * a.splits * pstride;
  const float sk = a.sinks[h] * kLog2e;
  const int S = a.splits;
  const int tid = threadIdx.x, grp = tid >> 7, dt = tid & 127;
  float lsum = 0.f;
  for (int s = tid; s < S; s += blockDim.x) {
    fac[s] = base[s * pstride + HG * kD + hl];
    fac[512 + s] = base[s * pstride + HG * kD + HG + hl];
  }
  __syncthreads();
  if (tid < 32) {
    float M = sk;
    for (int s = tid; s < S; s += 32) M = fmaxf(M, fac[s]);
    M = warp_max(M);
    for (int s = tid; s < S; s += 32) {
      const float f = exp2f(fac[s] - M);
      lsum += fac[512 + s] * f;
      fac[s] = f;
    }
    lsum = warp_sum(lsum) + exp2f(sk - M);
    if (tid == 0) s_inv = 1.f / lsum;
  }
  __syncthreads();
  // each split group sums every kGroups-th split, 8 loads in flight per thread
  const int d0 = dt * 4;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  const float* p = base + (size_t)hl * kD + d0;
  for (int s0 = grp; s0 < S; s0 += kGroups * 8) {
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int s = s0 + u * kGroups;
      v[u] = s < S ? *reinterpret_cast<const float4*>(p + s * pstride) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int s = s0 + u * kGroups;
      const float f = s < S ? fac[s] : 0.f;
      acc[0] += v[u].x * f; acc[1] += v[u].y * f; acc[2] += v[u].z * f; acc[3] += v[u].w * f;
    }
  }
  if (grp > 0) red[grp - 1][dt] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  __syncthreads();
  if (grp != 0) return;
#pragma unroll
  for (int q = 0; q < kGroups - 1; ++q) {
    const float4 o = red[q][dt];
    acc[0] += o.x; acc[1] += o.y; acc[2] += o.z; acc[3] += o.w;
  }
  const float inv = s_inv;
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] *= inv;
  if (d0 >= kD - 64) {
    const int64_t t = a.q_pos[row];
#pragma unroll
    for (int k = 0; k < 4; k += 2) {
      float c, s;
      rope_cos_sin(-(double)t, (d0 + k - (kD - 64)) >> 1, L, &c, &s);
      const float x0 = acc[k], x1 = acc[k + 1];
      acc[k] = x0 * c - x1 * s;
      acc[k + 1] = x0 * s + x1 * c;
    }
  }
  uint8_t* dst = a.out + ((size_t)row * L.H + h) * kD * (L.act_fmt == CSA_FMT_F32 ? 4 : 2);
  store_act4(dst, L.act_fmt, d0, acc);
}

// CUDA-core attention for other shapes / float32 rows: one warp per head, one CTA per query.
__global__ void attend_generic_kernel(const __grid_constant__ AttendArgs a) {
  const LayerArgs& L = a.L;
  const int lane = threadIdx.x & 31, h = threadIdx.x >> 5;
  const int row = blockIdx.x, b = row / a.Tq;
  const int D = L.D, dpl = D / 32, dn = D - L.d_rope;
  const int64_t t = a.q_pos[row];
  const SlotInfo si = slot_info(a, t);
  float q[32], o[32];
  const size_t ab = L.act_fmt == CSA_FMT_F32 ? 4 : 2;
  const uint8_t* qrow = a.q + ((size_t)row * L.H + h) * D * ab;
  float ss = 0.f;
  for (int k = 0; k < dpl; ++k) {
    const int d = lane * dpl + k;
    q[k] = L.act_fmt == CSA_FMT_F32 ? reinterpret_cast<const float*>(qrow)[d]
                                    : bf16_bits_to_f(reinterpret_cast<const uint16_t*>(qrow)[d]);
    ss += q[k] * q[k];
    o[k] = 0.f;
  }
  ss = warp_sum(ss);
  const float rs = 1.0f / sqrtf(ss / (float)D + L.eps);
  for (int k = 0; k < dpl; ++k) q[k] *= rs * (a.gamma_q ? a.gamma_q[lane * dpl + k] : 1.f);
  for (int k = 0; k + 1 < dpl; k += 2) {
    const int d = lane * dpl + k;
    if (d >= dn) {
      float c, s;
      rope_cos_sin((double)t, (d - dn) >> 1, L, &c, &s);
      const float x0 = q[k], x1 = q[k + 1];
      q[k] = x0 * c - x1 * s;
      q[k + 1] = x0 * s + x1 * c;
    }
  }
  float m = -INFINITY, l = 0.f;
  for (int64_t s = 0; s < si.R; ++s) {
    const uint8_t* p = slot_row(a, si, row, b, s);
    if (!p) continue;
    float kv[32];
    float sig = 1.f;
    if (L.kv_fmt == CSA_FMT_MIXED) sig = *reinterpret_cast<const float*>(p + D + 64);
    float dot = 0.f;
    for (int k = 0; k < dpl; ++k) {
      const int d = lane * dpl + k;
      float v;
      if (L.kv_fmt == CSA_FMT_F32) v = reinterpret_cast<const float*>(p)[d];
      else if (L.kv_fmt == CSA_FMT_BF16) v = bf16_bits_to_f(reinterpret_cast<const uint16_t*>(p)[d]);
      else v = d < dn ? e4m3_to_f(p[d]) * sig : bf16_bits_to_f(reinterpret_cast<const uint16_t*>(p + dn)[d - dn]);
      kv[k] = v;
      dot += q[k] * v;
    }
    dot = warp_sum(dot) * L.scale;
    if (dot > m) {
      const float c = expf(m - dot);
      l = l * c + 1.f;
      for (int k = 0; k < dpl; ++k) o[k] = o[k] * c + kv[k];
      m = dot;
    } else {
      const float pe = expf(dot - m);
      l += pe;
      for (int k = 0; k < dpl; ++k) o[k] += pe * kv[k];
    }
  }
  const float sk = a.sinks[h];
  const float M = fmaxf(m, sk);
  const float f = expf(m - M) / (l * expf(m - M) + expf(sk - M));
  for (int k = 0; k < dpl; ++k) o[k] *= f;
  for (int k = 0; k + 1 < dpl; k += 2) {
    const int d = lane * dpl + k;
    if (d >= dn) {
      float c, s;
      rope_cos_sin(-(double)t, (d - dn) >> 1, L, &c, &s);
      const float x0 = o[k], x1 = o[k + 1];
      o[k] = x0 * c - x1 * s;
      o[k + 1] = x0 * s + x1 * c;
    }
  }
  uint8_t* dst = a.out + ((size_t)row * L.H + h) * D * ab;
  for (int k = 0; k < dpl; ++k) {
    const int d = lane * dpl + k;
    if (L.act_fmt == CSA_FMT_F32) reinterpret_cast<float*>(dst)[d] = o[k];
    else reinterpret_cast<uint16_t*>(dst)[d] = f_to_bf16_bits(o[k]);
  }
}

// ----------------------------------------------------------------------------- tensor-core kernel (tcgen05)
// A cluster of two CTAs per (query, 128-slot split); CTA dh owns dims [256 dh, 256 dh + 256) of
// q~ and of the split's rows (keys and values are the same rows), all 128 heads as the MMA's M:
//   S_dh[h, s] = q~[h, half] . k_s[half]   tcgen05 kind::f16, A = q~ half (smem, by the tensor
//                                          memory accelerator), B = the half rows as bf16 (K-major),
//                                          D = TMEM cols [0, 128)
//   S = S_0 + S_1                          each thread sends its 64 partial scores to its twin in
//                                          the peer CTA through distributed shared memory
//   P = exp2(S*scale*log2e - m), bf16      one thread per (head, slot half), from registers
//   O[h, half] = P . V[:, half]            A = P (smem, K-major), B = the same bf16 half rows read
//                                          MN-major, D = TMEM cols [256, 512)
// Each CTA thus reads half of q~ and half of each row, and the q~ copy overlaps the rows' copy and
// conversion.  The CTA writes (O, m, l) of its half for the combine kernel, or, when one split
// covers the query, finishes its half of the output (sink, normalisation, inverse rotation).
constexpr int kTcN = 128;                  // key slots per CTA of a dense slot list (S columns, PV K)
constexpr int kTcNSparse = 64;             // ... of a top-k list: 18 cluster pairs for 1,152 slots
constexpr int kTcHalf = 256;               // output dims per CTA
constexpr int kTcThreads = 256;
constexpr int kTcQBlock = 128 * 128;       // one 64-dim column block of q~ (128 heads): 16 KB
constexpr int kTcHalfRow = 336;           // a half of a stored mixed-format row in X (<= 21 pieces)
constexpr size_t kTcPartBytes = (size_t)kD * kH128 * 2 + 2 * kH128 * 4;   // one split's partial: bf16 O/l, m, l
// X holds the raw half rows, then P [N / 64 blocks][128 heads][128 B]; 1024-byte multiple
__host__ __device__ constexpr int tc_x_bytes(int n) {
  const int raw = n * kTcHalfRow, p = (n / 64) * kTcQBlock;
  return ((raw > p ? raw : p) + 1023) / 1024 * 1024;
}
// the peer's partial scores: [slot half][N / 16 groups of 8][128 heads] x 16 bytes of fp16, then the
// power-of-two exponent each sending thread scaled them by: [slot half][128 heads] int32
__host__ __device__ constexpr int tc_xr_bytes(int n) { return n * 256 + 2 * 128 * 4; }
constexpr size_t tc_smem_bytes(int n) {
  return 1024 + 4 * (size_t)n * 128 + 4 * (size_t)kTcQBlock + tc_x_bytes(n) + tc_xr_bytes(n) + 64 + n * 8 +
         4 * 128 * 4 + n * 8;
}
static_assert(tc_x_bytes(kTcN) == kTcN * kTcHalfRow, "X at 128 slots: the raw half rows");
static_assert(tc_smem_bytes(kTcN) <= 227 * 1024, "tcgen05 attention shared memory");

// q~ = RoPE_t(RMSNorm(q) * gamma_q) in bf16, once per (query, head): one warp per head, lane l
// holds dims [16l, 16l+16) (the rotary pairs sit in lanes 28..31).
// q~ of one (row, head): RMSNorm, gamma, the rotation of the last 64 dims by the row's angles rcs.
__device__ __forceinline__ void qprep_head(const AttendArgs& a, int row, int h, int lane, const float2* rcs) {
  const LayerArgs& L = a.L;
  const size_t ab = L.act_fmt == CSA_FMT_F32 ? 4 : 2;
  const uint8_t* qrow = a.q + ((size_t)row * L.H + h) * kD * ab;
  float gm[16], v[16];
  if (a.gamma_q) {
#pragma unroll
    for (int k = 0; k < 16; k += 4) {
      const float4 g4 = __ldg(reinterpret_cast<const float4*>(a.gamma_q + 16 * lane + k));
      gm[k] = g4.x; gm[k + 1] = g4.y; gm[k + 2] = g4.z; gm[k + 3] = g4.w;
    }
  } else {
#pragma unroll
    for (int k = 0; k < 16; ++k) gm[k] = 1.f;
  }
  if (L.act_fmt == CSA_FMT_F32) {
#pragma unroll
    for (int k = 0; k < 16; k += 4) load_act4(qrow, CSA_FMT_F32, 16 * lane + k, v + k);
  } else {
    const uint4 u0 = __ldg(reinterpret_cast<const uint4*>(qrow + 2 * 16 * lane));
    const uint4 u1 = __ldg(reinterpret_cast<const uint4*>(qrow + 2 * 16 * lane + 16));
    const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) { v[2 * k] = bf16_bits_to_f(w[k] & 0xFFFFu); v[2 * k + 1] = bf16_bits_to_f(w[k] >> 16); }
  }
  float cs[8], sn[8];
  if (lane >= 28) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float2 r = rcs[(16 * lane + 2 * k - (kD - 64)) >> 1];
      cs[k] = r.x;
      sn[k] = r.y;
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < 16; ++k) ss += v[k] * v[k];
  ss = warp_sum(ss);
  const float rs = 1.0f / sqrtf(ss / (float)kD + L.eps);
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] *= rs * gm[k];
  if (lane >= 28) {
#pragma unroll
    for (int k = 0; k < 16; k += 2) {
      const float x0 = v[k], x1 = v[k + 1];
      v[k] = x0 * cs[k >> 1] - x1 * sn[k >> 1];
      v[k + 1] = x0 * sn[k >> 1] + x1 * cs[k >> 1];
    }
  }
  uint4 p0, p1;
  p0.x = pack_bf16x2(v[0], v[1]); p0.y = pack_bf16x2(v[2], v[3]);
  p0.z = pack_bf16x2(v[4], v[5]); p0.w = pack_bf16x2(v[6], v[7]);
  p1.x = pack_bf16x2(v[8], v[9]); p1.y = pack_bf16x2(v[10], v[11]);
  p1.z = pack_bf16x2(v[12], v[13]); p1.w = pack_bf16x2(v[14], v[15]);
  uint4* dst = reinterpret_cast<uint4*>(a.qt + (((size_t)row * L.H + h) * kD + 16 * lane) * 2);
  dst[0] = p0;
  dst[1] = p1;
}


__global__ void __launch_bounds__(128) qprep_kernel(const __grid_constant__ AttendArgs a, int hpc) {
  const LayerArgs& L = a.L;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.y;
  const int64_t t = a.q_pos[row];
  // the row's 32 rotation angles (the last 64 dims), once per CTA, one per thread
  __shared__ float2 rcs[32];
  if (threadIdx.x < 32) {
    float c, sn;
    rope_cos_sin((double)t, (int)threadIdx.x, L, &c, &sn);
    rcs[threadIdx.x] = make_float2(c, sn);
  }
  __syncthreads();
  // heads [hpc blockIdx.x, hpc blockIdx.x + hpc), one warp each in turn
  for (int hh = warp; hh < hpc; hh += 4) {
    const int h = blockIdx.x * hpc + hh;
    if (h >= L.H) break;
    qprep_head(a, row, h, lane, rcs);
  }
}

// The rows a deferred attention leaves to the combine: [0] the token's window row, [1] the entry the
// token completes (null when it completes none).
struct DeferredRows {
  const uint8_t* p[2];
};

__device__ __forceinline__ DeferredRows deferred_rows(const AttendArgs& a, int row) {
  DeferredRows d;
  d.p[0] = d.p[1] = nullptr;
  const CacheArgs& C = a.C;
  const int b = row / a.Tq;
  const int64_t rt = a.q_pos[row] - a.L.pos0;
  if (rt < 0 || a.no_window) return d;
  d.p[0] = C.window + ((size_t)b * C.window_cap + (size_t)(rt % C.window_cap)) * a.L.row_bytes;
  const int64_t r1 = rt + 1, nvis = r1 / a.L.m;
  if (r1 % a.L.m == 0 && nvis <= a.n_max)
    d.p[1] = C.entries + ((size_t)b * C.entry_cap + (size_t)(nvis - 1)) * a.L.row_bytes;
  return d;
}

// Values of dims d0..d0+3 of a stored bf16 or mixed row (codes times the row's power-of-two scale).
__device__ __forceinline__ void stored4(const uint8_t* row, const LayerArgs& L, int d0, float v[4]) {
  if (L.kv_fmt == CSA_FMT_BF16 || d0 >= kD - 64) {
    const uint8_t* p = L.kv_fmt == CSA_FMT_BF16 ? row + d0 * 2 : row + (kD - 64) + (d0 - (kD - 64)) * 2;
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    v[0] = bf16_bits_to_f(u.x & 0xFFFFu); v[1] = bf16_bits_to_f(u.x >> 16);
    v[2] = bf16_bits_to_f(u.y & 0xFFFFu); v[3] = bf16_bits_to_f(u.y >> 16);
    return;
  }
  const float sg = *reinterpret_cast<const float*>(row + kD + 64);
  const uint32_t w = *reinterpret_cast<const uint32_t*>(row + d0);
  const float2 lo = e4m3x2_to_float2((uint16_t)(w & 0xFFFFu)), hi = e4m3x2_to_float2((uint16_t)(w >> 16));
  v[0] = lo.x * sg; v[1] = lo.y * sg; v[2] = hi.x * sg; v[3] = hi.y * sg;
}

// Logits (base 2) of the deferred rows for every head: one warp per (head, row), lane l taking dims
// [16 l, 16 l + 16) of q~ and of the stored row; -inf for a row that does not exist.
__global__ void __launch_bounds__(128) attend_extra_logits_kernel(const __grid_constant__ AttendArgs a) {
  const LayerArgs& L = a.L;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.y, hk = blockIdx.x * 4 + warp;
  const int h = hk >> 1, k = hk & 1;
  if (h >= L.H) return;
  const DeferredRows dr = deferred_rows(a, row);
  float* dst = a.extra + ((size_t)row * 2 + k) * L.H + h;
  if (!dr.p[k]) {
    if (lane == 0) *dst = -INFINITY;
    return;
  }
  // q~ of the head from q itself (so this kernel waits for nothing but append+compress): RMSNorm over
  // the warp, gamma, the rotation by +t (dims 448..511 in lanes 28..31), rounded to bf16 as the
  // attention's operand is
  float qv[16], ss = 0.f;
  if (L.act_fmt == CSA_FMT_F32) {
#pragma unroll
    for (int i = 0; i < 16; i += 4) load_act4(a.q + ((size_t)row * L.H + h) * kD * 4, CSA_FMT_F32, 16 * lane + i, qv + i);
  } else {
    const uint4* qp = reinterpret_cast<const uint4*>(a.q + (((size_t)row * L.H + h) * kD + 16 * lane) * 2);
    const uint4 q0 = __ldg(qp), q1 = __ldg(qp + 1);
    const uint32_t qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      qv[2 * i] = bf16_bits_to_f(qw[i] & 0xFFFFu);
      qv[2 * i + 1] = bf16_bits_to_f(qw[i] >> 16);
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) ss = fmaf(qv[i], qv[i], ss);
  ss = warp_sum(ss);
  const float rs = 1.0f / sqrtf(ss / (float)kD + L.eps);
  const int64_t t = a.q_pos[row];
#pragma unroll
  for (int i = 0; i < 16; ++i) qv[i] *= rs * (a.gamma_q ? __ldg(a.gamma_q + 16 * lane + i) : 1.f);
  // rotary pair u's cos / sin computed by lane u (one float64 sincospi per lane), shuffled to the
  // lanes holding dims 448..511
  float cu, su;
  rope_cos_sin((double)t, lane, L, &cu, &su);
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const int u = (lane >= 28 ? 8 * (lane - 28) : 0) + (i >> 1);
    const float c = __shfl_sync(0xffffffffu, cu, u), sn = __shfl_sync(0xffffffffu, su, u);
    if (lane >= 28) {
      const float x0 = qv[i], x1 = qv[i + 1];
      qv[i] = x0 * c - x1 * sn;
      qv[i + 1] = x0 * sn + x1 * c;
    }
  }
  float dot = 0.f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float v[4];
    stored4(dr.p[k], L, 16 * lane + 4 * c, v);
#pragma unroll
    for (int e = 0; e < 4; ++e) dot = fmaf(bf16_bits_to_f(f_to_bf16_bits(qv[4 * c + e])), v[e], dot);
  }
  dot = warp_sum(dot);
  if (lane == 0) *dst = dot * (L.scale * kLog2e);
}

// Byte offset of 16-byte piece j (dims 8j..8j+7 of a 64-dim block) of row r in a 128-byte-swizzled
// K-major tile of rows.
__device__ __forceinline__ uint32_t sw128(int r, int j) { return (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4)); }

template <int FMT, int kN>
__global__ void __launch_bounds__(kTcThreads, 1) attend_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                 const __grid_constant__ AttendArgs a) {
  using namespace sm100;
  static_assert(kN == 64 || kN == 128, "64 or 128 slots per CTA");
  constexpr int kRegion = kN * 128;          // one 64-dim column block of the row tile
  constexpr int kLogN = kN == 128 ? 7 : 6;
  constexpr int kHalf = kN / 2;              // slots per softmax thread
  constexpr int kX = tc_x_bytes(kN);
  extern __shared__ uint8_t tc_smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* KV = sm;                                        // [4 blocks][128 slots][128 B] bf16: this CTA's dims
  uint8_t* Q = KV + 4 * kRegion;                           // q~ half [4][128][128 B], then the peer's S partial
  uint8_t* X = Q + 4 * kTcQBlock;                          // raw half rows, then P [N / 64][128][128 B]
  uint8_t* XR = X + kX;                                    // the peer's partial scores (received)
  uint64_t* bars = reinterpret_cast<uint64_t*>(XR + tc_xr_bytes(kN));   // S, received scores, O, q~
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  uint32_t* vbits = tmem_slot + 1;                         // [4] slot validity bitmasks
  int* valid = reinterpret_cast<int*>(tmem_slot + 8);      // [kN]
  int32_t* sidx = valid + kN;                            // [kN] entries of the selected slots (CSA)
  float* mls = reinterpret_cast<float*>(sidx + kN);      // [4][128]: max, sum of each column half, per head
  const uint8_t** rptr = reinterpret_cast<const uint8_t**>(mls + 4 * 128);   // [kN] stored row of each slot

  cg::cluster_group cluster = cg::this_cluster();
  const LayerArgs& L = a.L;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = blockIdx.z, dh = (int)cluster.block_rank(), sp = blockIdx.x >> 1;
  const int b = row / a.Tq;
  ATRACE_T(0, 0);
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
    mbar_arrive_expect_tx(&bars[1], (uint32_t)tc_xr_bytes(kN));   // the peer's scores, counted in bytes
    fence_barrier_init();
    // q~ dims [256 dh, 256 dh + 256) with the tensor memory accelerator: four 64-dim boxes of 128
    // heads, 128-byte swizzled (the K-major operand layout); in flight while the rows come in
    mbar_arrive_expect_tx(&bars[3], 4u * 128u * 128u);
#pragma unroll 1
    for (int c = 0; c < 4; ++c) tma_load_2d(Q + c * (128 * 128), &qmap, &bars[3], dh * kTcHalf + c * 64, row * kH128);
  }
  // first phase of the pair's cluster barrier: arrived now (each CTA's receive barrier is set up),
  // awaited just before the scores are sent
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  const int64_t t = a.q_pos[row];
  const SlotInfo si = slot_info(a, t);
  const int64_t s0 = (int64_t)sp * kN;
  if (a.topk)
    for (int i = tid; i < kN; i += kTcThreads) {
      const int64_t s = s0 + i;
      sidx[i] = s < si.n_sel ? a.topk[(size_t)row * L.top_k + s] : -1;
    }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  ATRACE_T(0, 1);

  // ---------------------------------------------------------------- this CTA's half of the rows -> bf16 tile
  // Compact loops throughout: this code runs once per CTA, so its instruction fetch counts.
  {
    const CacheArgs& C = a.C;
    auto row_ptr = [&](int r) -> const uint8_t* {
      const int64_t s = s0 + r;
      if (s < si.n_sel) {
        const int64_t e = a.topk ? (int64_t)sidx[r] - a.entry_offset : s;
        if (e < 0 || e >= a.entry_limit) return nullptr;
        return C.entries + ((size_t)b * C.entry_cap + (size_t)e) * L.row_bytes;
      }
      if (s < si.R) {
        const int64_t wr = si.wlast - si.n_win + 1 + (s - si.n_sel);
        return C.window + ((size_t)b * C.window_cap + (size_t)(wr % C.window_cap)) * L.row_bytes;
      }
      return nullptr;
    };
    if (tid < kN) {
      const uint8_t* p = row_ptr(tid);
      rptr[tid] = p;
      valid[tid] = p != nullptr;
    }
    __syncthreads();
    if (FMT == CSA_FMT_BF16) {
      // bf16 rows need no conversion: this half's 32 pieces of 16 bytes straight into the swizzled tile
      for (int idx = tid; idx < kN * 32; idx += kTcThreads) {     // rows fastest: distinct banks
        const int r = idx & (kN - 1), ch = idx >> kLogN;
        uint8_t* dst = KV + (ch >> 3) * kRegion + sw128(r, ch & 7);
        if (valid[r]) cp_async16(dst, rptr[r] + (dh * 32 + ch) * 16);
        else *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
      }
      cp_async_commit_wait();
    } else {
      // The stored row: 448 e4m3 codes, 64 bf16 rotary dims, the fp32 power-of-two scale (+ pad).
      // Half 0 takes codes 0..255 and the scale (17 pieces); half 1 codes 256..447, the rotary
      // dims and the scale (21 pieces), each at kTcHalfRow bytes per row of X.
      const int npc = dh ? 21 : 17;
      for (int idx = tid; idx < kN * npc; idx += kTcThreads) {
        const int r = idx / npc, pc = idx - r * npc;
        const int src = dh ? kTcHalf + 16 * pc : (pc < 16 ? 16 * pc : kD + 64);
        if (valid[r]) cp_async16(X + r * kTcHalfRow + pc * 16, rptr[r] + src);
      }
      cp_async_commit_wait();
      __syncthreads();
      ATRACE_T(0, 7);
      // codes x the row's scale -> bf16 (exact), rotary dims copied; consecutive threads take
      // consecutive rows of one piece, so their swizzled 16-byte stores fall on distinct banks
      const int ncode = dh ? 12 : 16, nit = dh ? 20 : 16;
      const int sc_off = dh ? 320 : 256;
#pragma unroll 2
      for (int idx = tid; idx < kN * nit; idx += kTcThreads) {
        const int r = idx & (kN - 1), it = idx >> kLogN;
        const bool ok = valid[r] != 0;
        const uint8_t* src = X + r * kTcHalfRow;
        if (it < ncode) {
          uint4 lo4 = make_uint4(0u, 0u, 0u, 0u), hi4 = lo4;
          if (ok) {
            const uint4 c = *reinterpret_cast<const uint4*>(src + it * 16);
            const float sg = *reinterpret_cast<const float*>(src + sc_off);
            const uint32_t w[4] = {c.x, c.y, c.z, c.w};
            uint32_t o[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float2 lo = e4m3x2_to_float2((uint16_t)(w[q] & 0xFFFFu));
              const float2 hi = e4m3x2_to_float2((uint16_t)(w[q] >> 16));
              o[2 * q] = pack_bf16x2(lo.x * sg, lo.y * sg);
              o[2 * q + 1] = pack_bf16x2(hi.x * sg, hi.y * sg);
            }
            lo4 = make_uint4(o[0], o[1], o[2], o[3]);
            hi4 = make_uint4(o[4], o[5], o[6], o[7]);
          }
          uint8_t* blk = KV + (it >> 2) * kRegion;
          const int j0 = (2 * it) & 7;
          *reinterpret_cast<uint4*>(blk + sw128(r, j0)) = lo4;
          *reinterpret_cast<uint4*>(blk + sw128(r, j0 + 1)) = hi4;
        } else {
          *reinterpret_cast<uint4*>(KV + 3 * kRegion + sw128(r, it - 12)) =
              ok ? *reinterpret_cast<const uint4*>(src + 192 + (it - 12) * 16) : make_uint4(0u, 0u, 0u, 0u);
        }
      }
    }
  }
  if (warp == 0) {                   // slot validity as bit masks for the softmax
#pragma unroll
    for (int q = 0; q < kN / 32; ++q) {
      const uint32_t m = __ballot_sync(0xffffffffu, valid[32 * q + lane] != 0);
      if (lane == 0) vbits[q] = m;
    }
  }
  fence_proxy_async_smem();
  __syncthreads();                   // X is free again; every raw row is converted
  ATRACE_T(0, 2);

  // ---------------------------------------------------------------- S partial = q~[:, half] K[:, half]^T
  const uint32_t idesc_s = instr_desc(128, kN, 1u);
  bool ok = true;
  if (tid == 0) {
    ok = mbar_wait(&bars[3], 0u);
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        const uint64_t ad = desc_kmajor_sw128(smem_u32(Q + c * (128 * 128)));
        const uint64_t bd = desc_kmajor_sw128(smem_u32(KV + c * kRegion));
#pragma unroll
        for (int k = 0; k < 4; ++k) umma_f16(tmem, ad + 2u * k, bd + 2u * k, idesc_s, (c | k) ? 1u : 0u);
      }
      umma_commit(&bars[0]);
    }
  }
  if (ok) ok = mbar_wait(&bars[0], 0u);
  tc_fence_after();
  ATRACE_T(0, 3);

  // ---------------------------------------------------------------- S = the two partials (cluster pair)
  // Warps w and w+4 read the same TMEM lanes (heads 32(w%4)..); warps 4..7 take the first half of
  // the slots, warps 0..3 the second.  Each thread sends its partial scores to the thread with the
  // same (head, slot half) in the peer CTA: st.async into the peer's receive buffer as [slot half]
  // [groups of 8][head] 16-byte pieces of fp16, the bytes counted on the peer's receive barrier (no
  // cluster barrier per exchange).  Before rounding, the thread scales its scores by 2^-e, with e
  // chosen from their largest magnitude so that it lands in [2^14, 2^15): no partial score of any
  // size overflows fp16's range, and each keeps fp16's 2^-11 relative rounding, finer than the bf16
  // of q~ it is made of.  e itself crosses as one more 4-byte st.async.
  const float cl2 = L.scale * kLog2e;
  const int h = (warp & 3) * 32 + lane;
  const int hs = warp >= 4 ? 0 : 1;                       // slot half of this warp
  const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  float s[kHalf];
#pragma unroll
  for (int c = 0; c < kHalf; c += 32) tmem_ld_32x32b_x32(lane_addr + kHalf * hs + c, s + c);
  tmem_wait_ld();
  int32_t* XE = reinterpret_cast<int32_t*>(XR + kN * 256);   // [slot half][head] exponents received
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  ATRACE_T(0, 4);
  {
    float amx = 0.f;
#pragma unroll
    for (int c = 0; c < kHalf; ++c) amx = fmaxf(amx, fabsf(s[c]));
    // floor(log2 amx) from the exponent field (amx >= 0; a subnormal or zero amx gives -127)
    int e = (int)((__float_as_uint(amx) >> 23) & 0xFFu) - 127 - 14;
    e = e < -110 ? -110 : (e > 110 ? 110 : e);
    const float sc = pow2i(-e);
    uint32_t rd, rb, re;
    const uint32_t ld = smem_u32(XR) + (uint32_t)(((size_t)hs * (kHalf / 8) * kH128 + h) * 16);
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rd) : "r"(ld), "r"(dh ^ 1));
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rb) : "r"(smem_u32(&bars[1])), "r"(dh ^ 1));
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(re) : "r"(smem_u32(XE + hs * kH128 + h)), "r"(dh ^ 1));
#pragma unroll
    for (int j = 0; j < kHalf / 8; ++j) {
      const float* v = s + 8 * j;
      asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];"
                   ::"r"(rd + (uint32_t)(j * kH128 * 16)), "r"(pack_f16x2(v[0] * sc, v[1] * sc)),
                     "r"(pack_f16x2(v[2] * sc, v[3] * sc)), "r"(pack_f16x2(v[4] * sc, v[5] * sc)),
                     "r"(pack_f16x2(v[6] * sc, v[7] * sc)), "r"(rb)
                   : "memory");
    }
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];"
                 ::"r"(re), "r"(e), "r"(rb)
                 : "memory");
  }
  if (!mbar_wait(&bars[1], 0u)) ok = false;
  // second phase: this CTA has all of its peer's scores (awaited before the CTA leaves, so neither
  // CTA of the pair exits while the other still sends to it)
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  ATRACE_T(0, 8);
  {
    const uint4* mine = reinterpret_cast<const uint4*>(XR) + (size_t)hs * (kHalf / 8) * kH128 + h;
    const float up = pow2i(XE[hs * kH128 + h]);
#pragma unroll
    for (int j = 0; j < kHalf / 8; ++j) {
      const uint4 v = mine[(size_t)j * kH128];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = unpack_f16x2(w[q]);
        s[8 * j + 2 * q] += f.x * up;
        s[8 * j + 2 * q + 1] += f.y * up;
      }
    }
  }

  // ---------------------------------------------------------------- softmax from registers
  ATRACE_C(128, 12);
  {
    float mm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int q = 0; q < kHalf / 32; ++q) {
      const uint32_t bits = vbits[(kHalf / 32) * hs + q];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float z = ((bits >> j) & 1u) ? s[32 * q + j] * cl2 : -INFINITY;
        mm[j & 3] = fmaxf(mm[j & 3], z);
      }
    }
    mls[hs * 128 + h] = fmaxf(fmaxf(mm[0], mm[1]), fmaxf(mm[2], mm[3]));
  }
  __syncthreads();
  const float m = fmaxf(mls[h], mls[128 + h]);
  const float ms = m == -INFINITY ? 0.f : m;
  ATRACE_C(128, 13);
  {
    float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q = 0; q < kHalf / 32; ++q) {
      const uint32_t cbits = vbits[(kHalf / 32) * hs + q];
      uint32_t w[16];
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const uint32_t bits = cbits >> j;
        const float p0 = exp2f(((bits & 1u) ? s[32 * q + j] * cl2 : -INFINITY) - ms);
        const float p1 = exp2f(((bits & 2u) ? s[32 * q + j + 1] * cl2 : -INFINITY) - ms);
        w[j >> 1] = pack_bf16x2(p0, p1);
        ls[(j >> 1) & 3] += bf16_bits_to_f(w[j >> 1] & 0xFFFFu) + bf16_bits_to_f(w[j >> 1] >> 16);
      }
      const int s0p = kHalf * hs + 32 * q;           // first slot of these 32
      uint8_t* blk = X + (s0p >> 6) * kTcQBlock;
      const int j0 = (s0p & 63) >> 3;
#pragma unroll
      for (int u = 0; u < 4; ++u)
        *reinterpret_cast<uint4*>(blk + sw128(h, j0 + u)) = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
    }
    mls[256 + hs * 128 + h] = (ls[0] + ls[1]) + (ls[2] + ls[3]);
  }
  ATRACE_C(128, 14);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  ATRACE_T(128, 9);
  ATRACE_C(128, 15);
  const float l = mls[256 + h] + mls[384 + h];

  // ---------------------------------------------------------------- O[:, half] = P V[:, half]
  if (tid == 0) {
    tc_fence_after();
    const uint32_t idesc_o = instr_desc(128, kTcHalf, 1u) | (1u << 16);   // B (the rows) MN-major
#pragma unroll 1
    for (int kk = 0; kk < kN / 16; ++kk) {
      const uint64_t ad = desc_kmajor_sw128(smem_u32(X + (kk >> 2) * (128 * 128))) + 2u * (kk & 3);
      const uint64_t bd = desc_mnmajor_sw128(smem_u32(KV + kk * 16 * 128), kRegion, 1024u);
      umma_f16(tmem + 256u, ad, bd, idesc_o, kk > 0 ? 1u : 0u);
    }
    umma_commit(&bars[2]);
  }
  ATRACE_T(0, 5);

  // ---------------------------------------------------------------- epilogue over all 8 warps
  // warps 4..7 take output columns 0..127 of this half, warps 0..3 columns 128..255
  if (ok) ok = mbar_wait(&bars[2], 0u);
  ATRACE_T(128, 10);
  tc_fence_after();
  const int e0 = hs * (kTcHalf / 2);
  if (a.splits > 1 || a.partial_out || a.defer_new) {
    // partial of this split: O / l in bf16 as [dim / 4][head][4] (a warp's stores are contiguous,
    // the combine reads a head's 4 dims in one 8-byte load), then (m, l) per head in fp32.  O / l
    // is a convex combination of value rows, so its bf16 rounding is no coarser than the output's.
    uint8_t* part = reinterpret_cast<uint8_t*>(a.part) + ((size_t)row * a.splits + sp) * kTcPartBytes;
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    uint2* od = reinterpret_cast<uint2*>(part);
#pragma unroll 1
    for (int c0 = e0; c0 < e0 + kTcHalf / 2; c0 += 32) {
      float v[32];
      tmem_ld_32x32b_x32(lane_addr + 256u + c0, v);
      tmem_wait_ld();
      uint2* dst = od + (size_t)((dh * kTcHalf + c0) >> 2) * kH128 + h;
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        dst[(size_t)(j >> 2) * kH128] = make_uint2(pack_bf16x2(v[j] * inv_l, v[j + 1] * inv_l),
                                                   pack_bf16x2(v[j + 2] * inv_l, v[j + 3] * inv_l));
    }
    if (dh == 0 && hs == 0)
      reinterpret_cast<float2*>(part + (size_t)kD * kH128 * 2)[h] = make_float2(m, l);
  } else {
    // one split covers the query: sink, normalisation, rotation back by -t, store
    const float sk = a.sinks[h] * kLog2e;
    const float M = fmaxf(m, sk);
    const float f = exp2f(m - M) / (l * exp2f(m - M) + exp2f(sk - M));
    const size_t ab = L.act_fmt == CSA_FMT_F32 ? 4 : 2;
    uint8_t* dst = a.out + ((size_t)row * L.H + h) * kD * ab;
#pragma unroll 1
    for (int c0 = e0; c0 < e0 + kTcHalf / 2; c0 += 32) {
      float v[32];
      tmem_ld_32x32b_x32(lane_addr + 256u + c0, v);
      tmem_wait_ld();
      const int d0 = dh * kTcHalf + c0;
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] *= f;
      if (d0 >= kD - 64) {
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          float c, s;
          rope_cos_sin((double)t, (d0 + j - (kD - 64)) >> 1, L, &c, &s);
          const float x0 = v[j], x1 = v[j + 1];
          v[j] = x0 * c + x1 * s;
          v[j + 1] = -x0 * s + x1 * c;
        }
      }
#pragma unroll
      for (int j = 0; j < 32; j += 4) store_act4(dst, L.act_fmt, d0 + j, v + j);
    }
  }
  tc_fence_before();
  ATRACE_T(128, 11);
  if (!ok && tid == 0) set_device_error(a.err, kErrWaitTimeout);
  __syncthreads();
  ATRACE_T(0, 6);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}

// Merge of the tcgen05 kernel's splits for 4 output dims of one query and all 128 heads: four
// groups of 128 threads (one per head) each take every 4th split and merge them online, 17 splits
// per step with every load of the step in flight (one 8-byte load of a head's 4 dims and one of
// its (m, l) per split, contiguous across a warp); the groups then merge through shared memory
// with the sink.  Normalisation and inverse rotation as in the single-split epilogue.
__global__ void __launch_bounds__(512) attend_tc_combine_kernel(const __grid_constant__ AttendArgs a) {
  constexpr int kU = 17;                              // splits per group and step: 68 per step in all
  __shared__ float red[4][6][kH128];
  const LayerArgs& L = a.L;
  const int h = threadIdx.x & 127, g = threadIdx.x >> 7;
  const int d0 = blockIdx.x * 4, row = blockIdx.y;
  const int S = a.splits;
  CBTRACE(0);
  const uint8_t* base = reinterpret_cast<const uint8_t*>(a.part) + (size_t)row * S * kTcPartBytes;
  float Mg = -INFINITY, lg = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s0 = g; s0 < S; s0 += 4 * kU) {
    float2 ml[kU];
    uint2 o[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int s = s0 + 4 * u;
      ml[u] = make_float2(-INFINITY, 0.f);
      o[u] = make_uint2(0u, 0u);
      if (s < S) {
        const uint8_t* ps = base + (size_t)s * kTcPartBytes;
        ml[u] = reinterpret_cast<const float2*>(ps + (size_t)kD * kH128 * 2)[h];
        o[u] = reinterpret_cast<const uint2*>(ps)[(size_t)(d0 >> 2) * kH128 + h];
      }
    }
    float mx = Mg;
#pragma unroll
    for (int u = 0; u < kU; ++u) mx = fmaxf(mx, ml[u].x);
    if (mx == -INFINITY) continue;
    const float sc = exp2f(Mg - mx);                   // 0 while nothing is merged yet
    lg *= sc;
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] *= sc;
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const float f = ml[u].y * exp2f(ml[u].x - mx);  // split weight: l_s * 2^(m_s - M)
      lg += f;
      acc[0] += f * bf16_bits_to_f(o[u].x & 0xFFFFu);
      acc[1] += f * bf16_bits_to_f(o[u].x >> 16);
      acc[2] += f * bf16_bits_to_f(o[u].y & 0xFFFFu);
      acc[3] += f * bf16_bits_to_f(o[u].y >> 16);
    }
    Mg = mx;
  }
  CBTRACE(1);
  red[g][0][h] = Mg;
  red[g][1][h] = lg;
#pragma unroll
  for (int k = 0; k < 4; ++k) red[g][2 + k][h] = acc[k];
  __syncthreads();
  if (g != 0) return;
  if (a.partial_out) {
    // a shard's partial: the splits merged without the sink, O normalised by their total weight
    float Mp = -INFINITY;
#pragma unroll
    for (int q = 0; q < 4; ++q) Mp = fmaxf(Mp, red[q][0][h]);
    float lp = 0.f, op[4] = {0.f, 0.f, 0.f, 0.f};
    if (Mp != -INFINITY) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float f = red[q][0][h] == -INFINITY ? 0.f : exp2f(red[q][0][h] - Mp);
        lp += red[q][1][h] * f;
#pragma unroll
        for (int k = 0; k < 4; ++k) op[k] += red[q][2 + k][h] * f;
      }
    }
    const float inv = lp > 0.f ? 1.f / lp : 0.f;
    float* pd = a.partial_out + ((size_t)row * L.H + h) * (kD + 2);
    for (int k = 0; k < 4; ++k) pd[d0 + k] = op[k] * inv;                 // rows of D + 2 floats: 8-byte aligned
    if (d0 == 0) {
      pd[kD] = Mp;
      pd[kD + 1] = lp;
    }
    return;
  }
  const float sk = a.sinks[h] * kLog2e;
  float M = sk;
#pragma unroll
  for (int q = 0; q < 4; ++q) M = fmaxf(M, red[q][0][h]);
  // deferred rows of this step (the token's window row, the entry it completes): one key each, with
  // its logit (base 2) from attend_extra_logits_kernel and its value read from the cache here
  float ex[2] = {-INFINITY, -INFINITY}, xv[2][4];
  if (a.defer_new) {
    const DeferredRows dr = deferred_rows(a, row);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (!dr.p[k]) continue;
      ex[k] = a.extra[((size_t)row * 2 + k) * L.H + h];
      stored4(dr.p[k], L, d0, xv[k]);
      M = fmaxf(M, ex[k]);
    }
  }
  float lsum = exp2f(sk - M), out[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float f = red[q][0][h] == -INFINITY ? 0.f : exp2f(red[q][0][h] - M);
    lsum += red[q][1][h] * f;
#pragma unroll
    for (int k = 0; k < 4; ++k) out[k] += red[q][2 + k][h] * f;
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    if (ex[k] == -INFINITY) continue;
    const float f = exp2f(ex[k] - M);
    lsum += f;
#pragma unroll
    for (int c = 0; c < 4; ++c) out[c] = fmaf(f, xv[k][c], out[c]);
  }
  const float inv = 1.f / lsum;
#pragma unroll
  for (int k = 0; k < 4; ++k) out[k] *= inv;
  if (d0 >= kD - 64) {
    const int64_t t = a.q_pos[row];
#pragma unroll
    for (int k = 0; k < 4; k += 2) {
      float c, s;
      rope_cos_sin(-(double)t, (d0 + k - (kD - 64)) >> 1, L, &c, &s);
      const float x0 = out[k], x1 = out[k + 1];
      out[k] = x0 * c - x1 * s;
      out[k + 1] = x0 * s + x1 * c;
    }
  }
  uint8_t* dst = a.out + ((size_t)row * L.H + h) * kD * (L.act_fmt == CSA_FMT_F32 ? 4 : 2);
  store_act4(dst, L.act_fmt, d0, out);
  CBTRACE(2);
}

#ifdef CSA_TRACE
extern "C" __attribute__((visibility("default"))) int csa_trace_read_cb(uint64_t* host) {
  return (int)cudaMemcpyFromSymbol(host, g_trace_cb, sizeof(g_trace_cb));
}
extern "C" __attribute__((visibility("default"))) int csa_trace_read_a(uint64_t* host) {
  return (int)cudaMemcpyFromSymbol(host, g_trace_a, sizeof(g_trace_a));
}
#endif

template <int HG, int FMT>
size_t mma_smem_bytes() {
  const size_t bufs = FMT == CSA_FMT_BF16 ? 2 : 1;
  return (size_t)HG * 1024 + bufs * kTile * 1024 + (size_t)HG * 128 + (11 * HG + 64) * sizeof(float) +
         bufs * kTile * sizeof(void*);
}

template <int HG, int FMT>
cudaError_t launch_mma(const AttendArgs& a, cudaStream_t s) {
  const size_t smem = mma_smem_bytes<HG, FMT>();
  {
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(attend_mma_kernel<HG, FMT>),
                                         smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(a.splits, a.L.H / HG, a.rows);
  cudaError_t e = launch_kernel(attend_mma_kernel<HG, FMT>, grid, dim3(HG * 8), smem, s, 0, a);
  if (e != cudaSuccess || a.splits == 1) return e;
  return launch_kernel(attend_combine_kernel<HG>, dim3(a.L.H, a.rows), dim3(512), 0, s, 0, a);
}

}  // namespace

int attend_path(const LayerArgs& L, bool dense, int rows) {
  // Decode-like calls (few query rows) with 128 heads of 512 dims take the tcgen05 kernel, dense and
  // top-k alike: a top-k list of about 1,150 slots is 18 cluster pairs of 64 slots, measured faster
  // than the mma.sync kernel over every SM and than 9 pairs of 128.  That kernel gives every query
  // one CTA pair per slot tile and a partial per tile, so calls with many query rows (chunked
  // prefill) take the mma.sync kernel, which needs no split there; so do other head counts.
  // Chunked prefill with 64 heads of bf16 rows takes the persistent tcgen05 kernel that computes the
  // transposed products (keys, then dims, as the MMA's M; attend_prefill.cu).
  (void)dense;
  if (rows <= kTcMaxRows && L.H == kH128 && L.D == kD && L.d_rope == 64 &&
      (L.kv_fmt == CSA_FMT_BF16 || L.kv_fmt == CSA_FMT_MIXED))
    return 2;
  if (attend_prefill_tc_supported(L, rows)) return 3;
  return attend_head_group(L) > 0 ? 1 : 0;
}

int attend_head_group(const LayerArgs& L) {
  if (L.D != kD || L.d_rope != 64) return 0;
  if (L.kv_fmt != CSA_FMT_BF16 && L.kv_fmt != CSA_FMT_MIXED) return 0;
  if (L.H % 64 == 0 && L.H <= 64) return 64;
  if (L.H % 32 == 0) return 32;
  return 0;
}

int attend_num_splits(const LayerArgs& L, bool dense, int rows, int64_t slots, int num_sms) {
  if (attend_path(L, dense, rows) == 3) return 1;
  if (attend_path(L, dense, rows) == 2) {
    const int n = dense ? kTcN : kTcNSparse;
    const int64_t s = (slots + n - 1) / n;
    return (int)(s < 1 ? 1 : s);
  }
  const int HG = attend_head_group(L);
  if (HG == 0) return 1;
  const int64_t pairs = (int64_t)rows * (L.H / HG);
  const int64_t tiles = (slots + kTile - 1) / kTile;
  // one CTA per SM (the kernel's registers allow no more): a single wave of CTAs
  int64_t want = ((int64_t)num_sms + pairs - 1) / pairs;
  if (want > tiles) want = tiles;
  if (want < 1) want = 1;
  return (int)want;
}

size_t attend_partial_bytes(const LayerArgs& L, bool dense, int rows, int splits) {
  if (attend_path(L, dense, rows) == 2) return splits <= 1 ? 0 : (size_t)rows * splits * kTcPartBytes;
  const int HG = attend_head_group(L);
  if (HG == 0 || splits <= 1) return 0;
  return (size_t)rows * (L.H / HG) * splits * HG * (kD + 2) * sizeof(float);
}

cudaError_t launch_attend_qprep(const AttendArgs& a, cudaStream_t s) {
  const int path = a.rows > 0 ? attend_path(a.L, a.topk == nullptr, a.rows) : 0;
  if (path != 2 && path != 3) return cudaSuccess;
  // decode (few rows): 4 heads per CTA for parallelism; chunks: 16, so each row's angles are formed
  // by fewer CTAs
  const int hpc = a.rows > kTcMaxRows ? 16 : 4;
  return launch_kernel(qprep_kernel, dim3((unsigned)((a.L.H + hpc - 1) / hpc), (unsigned)a.rows), dim3(128), 0, s, 0,
                       a, hpc);
}

PFN_cuTensorMapEncodeTiled_v12000 tma_encode_fn() {
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

// q~ [rows * 128 heads][512] bf16 as boxes of 64 dims x 128 heads, 128-byte swizzled.
bool make_qt_map(CUtensorMap* m, const void* qt, int rows) {
  auto fn = tma_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows * kH128};
  cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kH128};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(qt), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FMT, int kN>
cudaError_t launch_tc_n(const AttendArgs& a, cudaStream_t s) {
  constexpr size_t smem = tc_smem_bytes(kN);
  {
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(attend_tc_kernel<FMT, kN>),
                                         smem);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap qmap;
  if (!make_qt_map(&qmap, a.qt, a.rows)) return cudaErrorInvalidValue;
  cudaError_t e = launch_kernel(attend_tc_kernel<FMT, kN>, dim3((unsigned)(2 * a.splits), 1, (unsigned)a.rows),
                                dim3(kTcThreads), smem, s, 2, qmap, a);
  if (e != cudaSuccess || (a.splits == 1 && !a.partial_out)) return e;
  return launch_kernel(attend_tc_combine_kernel, dim3(kD / 4, a.rows), dim3(4 * kH128), 0, s, 0, a);
}

// dense slot lists take 128-slot splits; top-k lists 64-slot splits (as attend_num_splits counts them)
template <int FMT>
cudaError_t launch_tc(const AttendArgs& a, cudaStream_t s) {
  return a.topk ? launch_tc_n<FMT, kTcNSparse>(a, s) : launch_tc_n<FMT, kTcN>(a, s);
}

// The deferred-row form of the tcgen05 dense attention, in three launches that the caller orders
// around the concurrent append+compress: the attention over the earlier rows (q~ prepared first),
// the deferred rows' logits (after append+compress and q~), and the combine.
cudaError_t launch_attend_deferred(const AttendArgs& a, cudaStream_t s) {
  if (a.rows <= 0) return cudaSuccess;
  constexpr size_t smem = tc_smem_bytes(kTcN);
  auto kern = a.L.kv_fmt == CSA_FMT_MIXED ? attend_tc_kernel<CSA_FMT_MIXED, kTcN> : attend_tc_kernel<CSA_FMT_BF16, kTcN>;
  {
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return e;
  }
  CUtensorMap qmap;
  if (!make_qt_map(&qmap, a.qt, a.rows)) return cudaErrorInvalidValue;
  return launch_kernel(kern, dim3((unsigned)(2 * a.splits), 1, (unsigned)a.rows), dim3(kTcThreads), smem, s, 2,
                       qmap, a);
}

cudaError_t launch_attend_extra_logits(const AttendArgs& a, cudaStream_t s) {
  if (a.rows <= 0) return cudaSuccess;
  return launch_kernel(attend_extra_logits_kernel, dim3((unsigned)((2 * a.L.H + 3) / 4), (unsigned)a.rows), dim3(128),
                       0, s, 0, a);
}

cudaError_t launch_attend_combine(const AttendArgs& a, cudaStream_t s) {
  if (a.rows <= 0) return cudaSuccess;
  return launch_kernel(attend_tc_combine_kernel, dim3(kD / 4, a.rows), dim3(4 * kH128), 0, s, 0, a);
}

cudaError_t launch_attend(const AttendArgs& a, cudaStream_t s) {
  if (a.rows <= 0) return cudaSuccess;
  const int path = attend_path(a.L, a.topk == nullptr, a.rows);
  if (path == 2)
    return a.L.kv_fmt == CSA_FMT_MIXED ? launch_tc<CSA_FMT_MIXED>(a, s) : launch_tc<CSA_FMT_BF16>(a, s);
  if (path == 3) return launch_attend_prefill_tc(a, s);
  const int HG = attend_head_group(a.L);
  if (HG == 0) {
    return launch_kernel(attend_generic_kernel, dim3(a.rows), dim3(a.L.H * 32), 0, s, 0, a);
  }
  const bool mixed = a.L.kv_fmt == CSA_FMT_MIXED;
  if (HG == 64) return mixed ? launch_mma<64, CSA_FMT_MIXED>(a, s) : launch_mma<64, CSA_FMT_BF16>(a, s);
  return mixed ? launch_mma<32, CSA_FMT_MIXED>(a, s) : launch_mma<32, CSA_FMT_BF16>(a, s);
}

}  // namespace csa
