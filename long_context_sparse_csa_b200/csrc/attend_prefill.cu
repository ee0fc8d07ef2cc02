// Chunked-prefill attention on the tensor cores (tcgen05): many query rows, 64 query heads sharing one
// KV head of 512 dims stored in bf16.  What it computes is the shared-KV multi-query attention with a
// sink of "DeepSeek-V4: Making a Million Tokens Affordable", section "Two ways to shrink attention,
// interleaved" (keys are also the values, q~ = RoPE_t(RMSNorm(q) * gamma_q), the output rotated back
// by -t), over each query's own key slots: its top-k entries (CSA) or every visible entry (HCA), then
// its window rows.
//
// Every query gathers its own keys, so the contraction is per query: S = q~ K^T (64 heads x R keys x
// 512 dims), then O = P K.  Sixty-four heads fill only half of the 128-row MMA, so the kernel computes
// the transposes, with the keys (then the dims) as the MMA's M:
//   S^T[key, h]  = sum_d K[key, d] q~[h, d]    A = a 128-key tile of rows (K-major, 8 blocks of 64
//                                              dims), B = q~ (K-major); M = 128, N = 64; TMEM [0, 64)
//   O^T[d, h]   += sum_key K[key, d] P[key, h]  A = the same tile read dims-major (M-tile mt = dims
//                                              128 mt ..), B = P (heads-major); TMEM [256 + 64 mt, +64)
// and the online softmax over keys in between.  A softmax thread owns one key (its TMEM lane) and half
// of the heads, and holds that key's 32 head scores; the tile's per-head maxima come from a butterfly
// reduce-scatter across the warp on bf16 pairs and shared memory across the four lane quarters.  A head's
// running maximum moves only when its tile maximum exceeds it by more than 8 (in log2 units); then
// O^T's column and the partial sums are rescaled.  Exponentials are taken against the running maximum,
// so they stay below 2^8; a tile none of whose scores exceeds its head's running maximum by more than
// the margin skips the maxima altogether.  Each softmax thread keeps its key's partial sums per head;
// they are reduced once per query, in the epilogue.
//
// With N = 64 each MMA reads 6 KB of shared memory per 131 K multiply-adds, so the MMAs run at the
// shared memory's rate (about 60 % of the tensor pipe's), and a tile's MMAs share that bandwidth with
// the copies of the next tile's rows.
//
// Roles, in one persistent CTA per SM (query rows strided by the grid):
//   warp 0      the MMA issuer (one thread)
//   warps 1-8   softmax, two warps per TMEM lane quarter (32 heads each); after a tile's P they copy
//               the next tile's key rows in 16-byte cp.async pieces into the 128-byte-swizzled tile,
//               eight threads per 128-byte row segment, block by block: a 64-dim block is refilled as
//               soon as the O^T MMAs that read it are done, while the other M-tiles still run.  Per
//               query the epilogue: 1 / (l + 2^(sink - m)), the rotation by -t, the bf16 store
//   warps 9-10  q~ loaders (q~ made beforehand by the q preparation kernel), and the table of the
//               query's rotation angles for the epilogue
// Every mbarrier wait is bounded: a wait that gives up sets the device error word, and the role stops.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "kernels.h"
#include "sm100.cuh"

namespace csa {

namespace {

using namespace sm100;

constexpr int kD = 512;
constexpr int kHeads = 64;                    // query heads (MMA N)
constexpr int kKeys = 128;                    // keys per tile (MMA M of S^T)
constexpr int kBlocks = 8;                    // 64-dim column blocks of a row
constexpr int kBlockBytes = kKeys * 128;      // one block of the key tile: 16 KB
constexpr int kQBlockBytes = kHeads * 128;    // one block of q~: 8 KB
constexpr int kThreads = 352;                 // warp 0 MMA, warps 1-8 softmax, warps 9-10 loaders
constexpr int kLoaders = 64;                  // q~ loaders
constexpr int kCopiers = 256;                 // key tile copies (the softmax threads)
constexpr float kRescale = 8.f;               // log2 margin before a running maximum moves
// A head's running maximum before any key was seen: finite, so that 2^(z - m) needs no special
// case (a masked score, -inf, still gives 0) and m + kRescale stays below every finite score.
constexpr float kNoMax = -3.0e38f;

struct __align__(8) PfBars {
  uint64_t kvfull[kBlocks], kvfree[kBlocks];
  uint64_t qfull, qfree, sfull, pfull, ofull, ofree, drain;
  uint64_t ropefull[2];
  uint32_t tmem_base;
};

// shared memory: key tile 128 KB, q~ 64 KB, P 16 KB, then the small arrays
constexpr size_t kOffQ = (size_t)kBlocks * kBlockBytes;
constexpr size_t kOffP = kOffQ + (size_t)kBlocks * kQBlockBytes;
constexpr size_t kOffMx = kOffP + (size_t)kKeys * 128;
constexpr size_t kOffRope = kOffMx + (4 * kHeads + 3 * kHeads + 4) * sizeof(float);
constexpr size_t kOffBars = kOffRope + 2 * 32 * sizeof(float2);
constexpr size_t kSmemBytes = 1024 + kOffBars + sizeof(PfBars);
static_assert(kSmemBytes <= 227 * 1024, "prefill attention shared memory");

#ifdef CSA_TRACE
// Diagnostic build only: per-CTA timestamps (ns) of the first tiles and queries.
__device__ uint64_t g_trace_p[160][272];
#define PTRACE(slot) do { if (blockIdx.x < 160 && (slot) < 272) g_trace_p[blockIdx.x][(slot)] = global_timer_ns(); } while (0)
#else
#define PTRACE(slot) ((void)0)
#endif

// An empty key slot is filled from this zero row, so that every piece of a tile is a cp.async whose
// landing the block's barrier tracks.
__device__ __align__(16) uint8_t g_zero_row[kD * 2];

__device__ __forceinline__ uint32_t sw128(int r, int j) { return (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4)); }

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
// Arrives on the mbarrier (without raising its expected count) once this thread's earlier cp.async
// copies have landed.
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void softmax_bar() { asm volatile("barrier.sync.aligned 1, 256;" ::: "memory"); }
// Barrier of the 256 softmax threads that also returns whether any of them passed true.
__device__ __forceinline__ bool softmax_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "barrier.red.or.pred p, 3, 256, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

// 2^x by the MUFU approximation (ex2.approx.ftz): relative error about 2^-22, results below 2^-126
// flushed to 0.  The arguments here are at most the rescale margin, and the results are rounded to
// bf16 or summed with them.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return (uint32_t)f_to_bf16_bits(lo) | ((uint32_t)f_to_bf16_bits(hi) << 16);
}

// Key slots of the query at position t: [0, n_sel) entries, [n_sel, R) window rows.
struct Slots {
  int64_t rt, n_sel, n_win, R;
  int tiles;
};

__device__ __forceinline__ Slots slots_of(const AttendArgs& a, int64_t t) {
  Slots s;
  s.rt = t - a.L.pos0;
  const int64_t r1 = s.rt + 1 > 0 ? s.rt + 1 : 0;
  const int64_t nvis = r1 / a.L.m;
  s.n_sel = a.topk ? (int64_t)a.L.top_k : (nvis < a.n_max ? nvis : a.n_max);
  s.n_win = r1 < a.L.window ? r1 : a.L.window;
  s.R = s.n_sel + s.n_win;
  const int64_t nt = (s.R + kKeys - 1) / kKeys;
  s.tiles = nt < 1 ? 1 : (int)nt;               // at least one (all-masked) tile: every role walks it
  return s;
}

// Stored row of slot s of query `row` (sequence b), or null for an empty slot (-1, out of range).
__device__ __forceinline__ const uint8_t* slot_ptr(const AttendArgs& a, const Slots& si, int row, int b, int64_t s) {
  const CacheArgs& C = a.C;
  if (s < si.n_sel) {
    const int64_t e = a.topk ? (int64_t)__ldg(a.topk + (size_t)row * a.L.top_k + s) : s;
    if (e < 0 || e >= C.entry_cap) return nullptr;
    return C.entries + ((size_t)b * C.entry_cap + (size_t)e) * a.L.row_bytes;
  }
  if (s < si.R) {
    const int64_t wr = si.rt - si.n_win + 1 + (s - si.n_sel);
    return C.window + ((size_t)b * C.window_cap + (size_t)(wr % C.window_cap)) * a.L.row_bytes;
  }
  return nullptr;
}

// A copying thread's view of a key tile: the loads it needs (the query position and the top-k
// entries of its four rows 32 it + crow), issued early, and the row addresses formed from them later.
struct TileRaw {
  int64_t t;
  int32_t e[4];
};

__device__ __forceinline__ TileRaw tile_raw(const AttendArgs& a, int row, int i, int crow) {
  TileRaw r;
  r.t = a.q_pos[row];
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int s = i * kKeys + 32 * it + crow;
    r.e[it] = (a.topk && s < a.L.top_k) ? __ldg(a.topk + (size_t)row * a.L.top_k + s) : s;
  }
  return r;
}

struct TileSrc {
  const uint8_t* p[4];
};

// Piece `piece` of each of the four rows (an empty slot reads the zero row); the same slots as
// slot_ptr, from the loaded entries.
__device__ __forceinline__ TileSrc tile_src(const AttendArgs& a, const TileRaw& raw, int row, int i, int crow,
                                            int piece) {
  const Slots si = slots_of(a, raw.t);
  const int b = row / a.Tq;
  const CacheArgs& C = a.C;
  TileSrc r;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int64_t s = (int64_t)i * kKeys + 32 * it + crow;
    const uint8_t* sp = nullptr;
    if (s < si.n_sel) {
      const int64_t e = raw.e[it];
      if (e >= 0 && e < C.entry_cap) sp = C.entries + ((size_t)b * C.entry_cap + (size_t)e) * a.L.row_bytes;
    } else if (s < si.R) {
      const int64_t wr = si.rt - si.n_win + 1 + (s - si.n_sel);
      sp = C.window + ((size_t)b * C.window_cap + (size_t)(wr % C.window_cap)) * a.L.row_bytes;
    }
    r.p[it] = (sp ? sp : g_zero_row) + 16 * piece;
  }
  return r;
}

// Copies of tile g into the key buffer, block by block: block c once the O^T MMAs of tile g - 1 are
// done with it; each block's copies arrive on its barrier when they land.  False if a wait gave up.
__device__ __forceinline__ bool copy_tile(uint8_t* KV, PfBars* bars, const TileSrc& src, uint32_t g, int crow,
                                          int piece) {
  for (int c = 0; c < kBlocks; ++c) {
    if (!mbar_wait(&bars->kvfree[c], (g & 1u) ^ 1u)) return false;
    uint8_t* dst = KV + c * kBlockBytes;
#pragma unroll
    for (int it = 0; it < 4; ++it) cp_async16(dst + sw128(32 * it + crow, piece), src.p[it] + c * 128);
    cp_async_arrive(&bars->kvfull[c]);
  }
  return true;
}

__device__ __forceinline__ uint32_t bf16x2_max(uint32_t x, uint32_t y) {
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&x), b = *reinterpret_cast<__nv_bfloat162*>(&y);
  __nv_bfloat162 r = __hmax2(a, b);
  return *reinterpret_cast<uint32_t*>(&r);
}

__global__ void __launch_bounds__(kThreads, 1) attend_prefill_tc_kernel(const __grid_constant__ AttendArgs a) {
  extern __shared__ uint8_t pf_smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pf_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* KV = sm;                                             // [8 blocks][128 keys][128 B]
  uint8_t* Q = sm + kOffQ;                                      // [8 blocks][64 heads][128 B]
  uint8_t* P = sm + kOffP;                                      // [128 keys][64 heads] bf16, swizzled
  float* mx = reinterpret_cast<float*>(sm + kOffMx);            // [4 warps][64]: tile maxima / sums
  float* mrun = mx + 4 * kHeads;                                // [64] running maxima (log2 units)
  float* alph = mrun + kHeads;                                  // [64] rescale factors of this tile
  float* fh = alph + kHeads;                                    // [64] output factors (epilogue)
  int* flag = reinterpret_cast<int*>(fh + kHeads);              // [2] any head of a half rescaled
  float2* rope_cs = reinterpret_cast<float2*>(sm + kOffRope);  // [2 queries][32 pairs] (cos, sin)
  PfBars* bars = reinterpret_cast<PfBars*>(sm + kOffBars);

  const LayerArgs& L = a.L;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int c = 0; c < kBlocks; ++c) {
      mbar_init(&bars->kvfull[c], kCopiers);
      mbar_init(&bars->kvfree[c], 1);
    }
    mbar_init(&bars->qfull, kLoaders);
    mbar_init(&bars->qfree, 1);
    mbar_init(&bars->sfull, 1);
    mbar_init(&bars->pfull, 256);
    mbar_init(&bars->ofull, 1);
    mbar_init(&bars->ofree, 256);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->ropefull[0], 32);
    mbar_init(&bars->ropefull[1], 32);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const float cl2 = L.scale * kLog2e;
  if (tid == 0) PTRACE(95);

  if (warp == 0) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = instr_desc(kKeys, kHeads, 1u);                          // both K-major
      const uint32_t idesc_o = instr_desc(128, kHeads, 1u) | (1u << 15) | (1u << 16);  // both MN-major
      // operand descriptors of the buffers' starts; the MMAs below add constant offsets (16-byte
      // units) to these, so the issue sequence holds no address arithmetic
      const uint64_t kv_k = desc_kmajor_sw128(smem_u32(KV));
      const uint64_t q_k = desc_kmajor_sw128(smem_u32(Q));
      const uint64_t kv_mn = desc_mnmajor_sw128(smem_u32(KV), kBlockBytes, 1024u);
      const uint64_t p_mn = desc_mnmajor_sw128(smem_u32(P), kBlockBytes, 1024u);
      bool ok = true;
      uint32_t g = 0, j = 0;
      bool issued = false;
      for (int row = blockIdx.x; row < a.rows && ok; row += gridDim.x, ++j) {
        const Slots si = slots_of(a, a.q_pos[row]);
        if (!mbar_wait(&bars->qfull, j & 1u)) { ok = false; break; }
        for (int i = 0; i < si.tiles; ++i, ++g) {
          // S^T = K q~^T over the 8 blocks of this tile, as each block lands
#pragma unroll
          for (int c = 0; c < kBlocks; ++c) {
            if (!mbar_wait(&bars->kvfull[c], g & 1u)) { ok = false; break; }
            if (c == 0 && g < 16) PTRACE(256 + g);
            fence_proxy_async_smem();                 // the loaders' copies, for the tensor core
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f16(tmem, kv_k + (uint64_t)(c * (kBlockBytes >> 4) + 2 * kk),
                       q_k + (uint64_t)(c * (kQBlockBytes >> 4) + 2 * kk), idesc_s, (c | kk) ? 1u : 0u);
            issued = true;
          }
          if (!ok) break;
          umma_commit(&bars->sfull);
          if (g < 16) PTRACE(g);
          if (i + 1 == si.tiles) umma_commit(&bars->qfree);
          // O^T += K^T P once the softmax has written P (and rescaled O^T where needed); the first tile
          // of a query overwrites O^T once the previous query's epilogue has read it
          if (!mbar_wait(&bars->pfull, g & 1u)) { ok = false; break; }
          if (g < 16) PTRACE(96 + g);
          if (i == 0 && !mbar_wait(&bars->ofree, (j & 1u) ^ 1u)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
            for (int kk = 0; kk < kKeys / 16; ++kk)
              umma_f16(tmem + 256u + 64u * (uint32_t)mt, kv_mn + (uint64_t)((2 * mt * kBlockBytes + kk * 2048) >> 4),
                       p_mn + (uint64_t)((kk * 2048) >> 4), idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
            umma_commit(&bars->kvfree[2 * mt]);
            umma_commit(&bars->kvfree[2 * mt + 1]);
            if (mt == 0 && g < 16) PTRACE(112 + g);
          }
          if (g < 16) PTRACE(16 + g);
#ifdef CSA_TRACE
          // diagnostic build: completion of the first and last M-tiles as the issuer sees them
          if (g < 16) {
            mbar_wait(&bars->kvfree[1], g & 1u);
            PTRACE(176 + g);
            mbar_wait(&bars->kvfree[7], g & 1u);
            PTRACE(192 + g);
          }
#endif
        }
        if (!ok) break;
        umma_commit(&bars->ofull);
      }
      if (!ok) {
        set_device_error(a.err, kErrWaitTimeout);
      }
      // nothing of this thread is in flight when TMEM is released
      if (issued) {
        umma_commit(&bars->drain);
        mbar_wait(&bars->drain, 0u);
      }
    }
    __syncwarp();
  } else if (warp <= 8) {
    // ------------------------------------------------------------------ softmax and epilogue
    // Two warps per TMEM lane quarter: warp w takes key (or dim) 32 (w % 4) + lane and heads
    // [32 hf, 32 hf + 32), hf = (w - 1) / 4.
    const int w4 = warp & 3;                                  // TMEM lane quarter of this warp
    const int hf = (warp - 1) >> 2;                           // head half
    const int h0 = 32 * hf;
    const int key = w4 * 32 + lane;                           // key of S^T, dim of O^T's M-tile
    const uint32_t lane_addr = tmem + ((uint32_t)(w4 * 32) << 16);
    // Between a tile's P and the next tile's S^T these threads are idle, so they copy the next
    // tile's key rows, block by block as the O^T MMAs release the blocks: thread st copies piece
    // st % 8 of rows 32 it + st / 8 (it < 4), so eight threads cover a 128-byte row segment.  The
    // loads those copies need are issued before the softmax and used after it.
    const int st = tid - 32;                                  // 0..255
    const int crow = st >> 3, cpiece = st & 7;
    bool ok = true;
    uint32_t g = 0, j = 0;
    if (blockIdx.x < a.rows) {
      const TileRaw raw = tile_raw(a, blockIdx.x, 0, crow);
      ok = copy_tile(KV, bars, tile_src(a, raw, blockIdx.x, 0, crow, cpiece), 0u, crow, cpiece);
    }
    for (int row = blockIdx.x; row < a.rows && ok; row += gridDim.x, ++j) {
      const int64_t t = a.q_pos[row];
      const Slots si = slots_of(a, t);
      const int b = row / a.Tq;
      float lp[32];                                           // this key's partial sums of its heads
#pragma unroll
      for (int h = 0; h < 32; ++h) lp[h] = 0.f;
      if (hf == 0 && key < kHeads) mrun[key] = kNoMax;
      softmax_bar();
      for (int i = 0; i < si.tiles; ++i, ++g) {
        // the tile after this one: the next of this query, or the first of the CTA's next query
        const bool more = i + 1 < si.tiles || row + (int)gridDim.x < a.rows;
        const int row_n = i + 1 < si.tiles ? row : row + (int)gridDim.x;
        const int i_n = i + 1 < si.tiles ? i + 1 : 0;
        TileRaw raw_n;
        if (more) raw_n = tile_raw(a, row_n, i_n, crow);
        const int64_t s = (int64_t)i * kKeys + key;
        const bool valid = slot_ptr(a, si, row, b, s) != nullptr;
        if (!mbar_wait(&bars->sfull, g & 1u)) { ok = false; break; }
        if (tid == 32 && g < 16) PTRACE(32 + g);
        tc_fence_after();
        float z[32];
        tmem_ld_32x32b_x32(lane_addr + (uint32_t)h0, z);
        tmem_wait_ld();
        if (tid == 32 && g < 16) PTRACE(208 + g);
#pragma unroll
        for (int h = 0; h < 32; ++h) z[h] = valid ? z[h] * cl2 : -INFINITY;
        // The tile's maxima are needed only where a score exceeds its head's running maximum by more
        // than the margin (always on a query's first tile); otherwise the maxima stay as they are.
        bool over = false;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 m4 = reinterpret_cast<const float4*>(mrun + h0)[q];
          over |= (z[4 * q] > m4.x + kRescale) | (z[4 * q + 1] > m4.y + kRescale) |
                  (z[4 * q + 2] > m4.z + kRescale) | (z[4 * q + 3] > m4.w + kRescale);
        }
        bool moved = false;
        const bool any_over = softmax_any(over);
        if (tid == 32 && g < 16) PTRACE(224 + g);
        if (any_over) {
          // the tile's maxima per head: lanes (a butterfly over bf16 pairs, then the last pair's
          // neighbours), then warps
          {
            uint32_t w[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) w[q] = pack_bf16x2(z[2 * q], z[2 * q + 1]);
#pragma unroll
            for (int o = 16, n = 8; o >= 2; o >>= 1, n >>= 1) {
              const bool upper = (lane & o) != 0;
#pragma unroll
              for (int q = 0; q < n; ++q) {
                const uint32_t send = upper ? w[q] : w[q + n];
                const uint32_t keep = upper ? w[q + n] : w[q];
                w[q] = bf16x2_max(keep, __shfl_xor_sync(0xffffffffu, send, o));
              }
            }
            w[0] = bf16x2_max(w[0], __shfl_xor_sync(0xffffffffu, w[0], 1));
            // lanes 2k and 2k + 1 now hold heads h0 + 2k, h0 + 2k + 1
            if ((lane & 1) == 0) {
              mx[w4 * kHeads + h0 + lane] = bf16_bits_to_f(w[0] & 0xFFFFu);
              mx[w4 * kHeads + h0 + lane + 1] = bf16_bits_to_f(w[0] >> 16);
            }
          }
          softmax_bar();
          if (w4 == 0) {
            const int h = h0 + lane;
            const float tm = fmaxf(fmaxf(mx[h], mx[kHeads + h]), fmaxf(mx[2 * kHeads + h], mx[3 * kHeads + h]));
            const float mr = mrun[h];
            float al = 1.f;
            int mv = 0;
            if (tm > mr + kRescale) {
              al = fast_exp2(mr - tm);                // 0 on the first move
              mrun[h] = tm;
              mv = 1;
            }
            alph[h] = al;
            mv = __any_sync(0xffffffffu, mv);
            if (lane == 0) flag[hf] = mv;
          }
          softmax_bar();
          moved = (flag[0] | flag[1]) != 0;
        }
        // P = 2^(z - m) in bf16, this key's row of P (its heads' 64 bytes); the partial sums
        // (rescaled where the head's maximum moved) take the rounded values
        uint8_t* prow = P;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          uint32_t w[4];
          float mm[8], aa[8];
          *reinterpret_cast<float4*>(mm) = reinterpret_cast<const float4*>(mrun + h0)[2 * jj];
          *reinterpret_cast<float4*>(mm + 4) = reinterpret_cast<const float4*>(mrun + h0)[2 * jj + 1];
          if (moved) {
            *reinterpret_cast<float4*>(aa) = reinterpret_cast<const float4*>(alph + h0)[2 * jj];
            *reinterpret_cast<float4*>(aa + 4) = reinterpret_cast<const float4*>(alph + h0)[2 * jj + 1];
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int h = 8 * jj + 2 * q;
            const float m0 = mm[2 * q], m1 = mm[2 * q + 1];
            const float p0 = fast_exp2(z[h] - m0);
            const float p1 = fast_exp2(z[h + 1] - m1);
            w[q] = pack_bf16x2(p0, p1);
            if (moved) {
              lp[h] *= aa[2 * q];
              lp[h + 1] *= aa[2 * q + 1];
            }
            lp[h] += bf16_bits_to_f(w[q] & 0xFFFFu);
            lp[h + 1] += bf16_bits_to_f(w[q] >> 16);
          }
          *reinterpret_cast<uint4*>(prow + sw128(key, 4 * hf + jj)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        if (tid == 32 && g < 16) PTRACE(240 + g);
        // rescale O^T, the previous tiles' sum (complete, as this tile's S^T is), where a maximum moved
        if (moved && i > 0) {
#pragma unroll 1
          for (int mt = 0; mt < 4; ++mt) {
            float o[32];
            tmem_ld_32x32b_x32(lane_addr + 256u + 64u * mt + h0, o);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; ++u) o[u] *= alph[h0 + u];
            tmem_st_32x32b_x32(lane_addr + 256u + 64u * mt + h0, o);
          }
          tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars->pfull);
        if (tid == 32 && g < 16) PTRACE(48 + g);
        if (more && !copy_tile(KV, bars, tile_src(a, raw_n, row_n, i_n, crow, cpiece), g + 1, crow, cpiece)) {
          ok = false;
          break;
        }
        if (tid == 32 && g < 16) PTRACE(64 + g);
      }
      if (!ok) break;
      // ---------------------------------------------------------------- epilogue of this query
      // this warp's partial sums per head: lane l ends with head h0 + l
#pragma unroll
      for (int o = 16, n = 16; o >= 1; o >>= 1, n >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int q = 0; q < n; ++q) {
          const float send = upper ? lp[q] : lp[q + n];
          const float keep = upper ? lp[q + n] : lp[q];
          lp[q] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      mx[w4 * kHeads + h0 + lane] = lp[0];
      softmax_bar();
      if (w4 == 0) {
        const int h = h0 + lane;
        const float l = (mx[h] + mx[kHeads + h]) + (mx[2 * kHeads + h] + mx[3 * kHeads + h]);
        const float m = mrun[h];
        const float sk = a.sinks[h] * kLog2e;
        // o = O / (l + 2^(sink - m)), O and l relative to the running maximum m
        fh[h] = m == kNoMax ? 0.f : 1.f / (l + exp2f(sk - m));
      }
      softmax_bar();
      if (tid == 32 && j < 2) PTRACE(160 + 8 * j);
      if (!mbar_wait(&bars->ofull, j & 1u)) { ok = false; break; }
      if (tid == 32 && j < 2) PTRACE(161 + 8 * j);
      tc_fence_after();
      // per M-tile: this thread's dim of its 32 heads -> the warp's own [32 heads][32 dims] bf16
      // staging tile in P's buffer (free: the query's last P.V is done), then 16-byte stores of
      // its heads' 64-byte row pieces
      uint8_t* out = a.out + (size_t)row * kHeads * kD * 2;
      uint16_t* wst = reinterpret_cast<uint16_t*>(P) + (warp - 1) * 32 * 32;
      // all of this thread's O^T values, then O^T is released (the next query's first P.V may
      // overwrite it while this query's output is still being stored).  Scaled by the heads' output
      // factors on the way; M-tiles 0-2 (no rotary dims) are rounded to bf16 at once, in pairs of
      // heads, the last M-tile stays in fp32 for the rotation.
      uint32_t ob[3][16];
      float o3[32];
      {
        float o[3][32];
#pragma unroll
        for (int mt = 0; mt < 3; ++mt) tmem_ld_32x32b_x32(lane_addr + 256u + 64u * mt + h0, o[mt]);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; u += 2) {
          const float f0 = fh[h0 + u], f1 = fh[h0 + u + 1];
#pragma unroll
          for (int mt = 0; mt < 3; ++mt) ob[mt][u >> 1] = pack_bf16x2(o[mt][u] * f0, o[mt][u + 1] * f1);
        }
      }
      tmem_ld_32x32b_x32(lane_addr + 256u + 64u * 3 + h0, o3);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars->ofree);
      if (tid == 32 && j < 2) PTRACE(162 + 8 * j + 4);
#pragma unroll
      for (int u = 0; u < 32; ++u) o3[u] *= fh[h0 + u];
      if (!mbar_wait(&bars->ropefull[j & 1u], (j >> 1) & 1u)) { ok = false; break; }
      // the rotary dims (the last 64) are the upper half of the last M-tile: whole warps
      if (w4 >= 2) {
        const int d = 3 * 128 + key;
        const float2 cs = rope_cs[(j & 1u) * 32 + ((d - (kD - 64)) >> 1)];
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          // rotation by -t of the pair (d even, d + 1): partner in the neighbouring lane
          const float v = o3[u], pv = __shfl_xor_sync(0xffffffffu, v, 1);
          o3[u] = (d & 1) ? (-pv * cs.y + v * cs.x) : (v * cs.x + pv * cs.y);
        }
      }
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
        for (int u = 0; u < 32; u += 2) {
          uint32_t w2 = mt < 3 ? ob[mt < 3 ? mt : 0][u >> 1] : pack_bf16x2(o3[u], o3[u + 1]);
          wst[u * 32 + lane] = (uint16_t)(w2 & 0xFFFFu);
          wst[(u + 1) * 32 + lane] = (uint16_t)(w2 >> 16);
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int q = k * 32 + lane, u = q >> 2, part = q & 3;
          *reinterpret_cast<uint4*>(out + ((size_t)(h0 + u) * kD + mt * 128 + w4 * 32) * 2 + part * 16) =
              *reinterpret_cast<const uint4*>(wst + u * 32 + part * 8);
        }
        __syncwarp();
        if (tid == 32 && j < 2 && mt < 3) PTRACE(162 + 8 * j + mt);
      }
      if (tid == 32 && j < 8) PTRACE(80 + j);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (!ok) {
      set_device_error(a.err, kErrWaitTimeout);
    }
  } else {
    // ------------------------------------------------------------------ q~ loaders
    // Consecutive threads copy consecutive 16-byte pieces of a head's row.
    const int lt = tid - 288;                                 // 0..63
    bool ok = true;
    uint32_t j = 0;
    for (int row = blockIdx.x; row < a.rows && ok; row += gridDim.x, ++j) {
      // q~ of this query (made by the q preparation kernel, 64 KB contiguous) once the previous
      // query's S^T MMAs are done with the buffer
      if (!mbar_wait(&bars->qfree, (j & 1u) ^ 1u)) { ok = false; break; }
      {
        const uint8_t* src = a.qt + (size_t)row * kHeads * kD * 2;
#pragma unroll 8
        for (int h = 0; h < kHeads; ++h)
          cp_async16(Q + (lt >> 3) * kQBlockBytes + sw128(h, lt & 7), src + (size_t)h * kD * 2 + 16 * lt);
        // the rotation angles of this query's output (its 32 rotary pairs), while the copies land
        if (lt < 32) {
          float c, sn;
          rope_cos_sin((double)a.q_pos[row], lt, L, &c, &sn);
          rope_cs[(j & 1u) * 32 + lt] = make_float2(c, sn);
          mbar_arrive(&bars->ropefull[j & 1u]);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        fence_proxy_async_smem();
        mbar_arrive(&bars->qfull);
        if (tid == 288 && j < 8) PTRACE(88 + j);
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (!ok) {
      set_device_error(a.err, kErrWaitTimeout);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

#ifdef CSA_TRACE
}  // namespace
extern "C" __attribute__((visibility("default"))) int csa_trace_read_p(uint64_t* host) {
  return (int)cudaMemcpyFromSymbol(host, g_trace_p, sizeof(g_trace_p));
}
namespace {
#endif

int device_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  static int cached[64] = {0};
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

}  // namespace

bool attend_prefill_tc_supported(const LayerArgs& L, int rows) {
  return rows > kTcMaxRows && L.H == kHeads && L.D == kD && L.d_rope == 64 && L.kv_fmt == CSA_FMT_BF16 &&
         L.act_fmt == CSA_FMT_BF16;
}

cudaError_t launch_attend_prefill_tc(const AttendArgs& a, cudaStream_t s) {
  if (a.rows <= 0) return cudaSuccess;
  {
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(attend_prefill_tc_kernel), kSmemBytes);
    if (e != cudaSuccess) return e;
  }
  const int sms = device_sms();
  const int grid = a.rows < sms ? a.rows : sms;
  return launch_kernel(attend_prefill_tc_kernel, dim3((unsigned)grid), dim3(kThreads), kSmemBytes, s, 0, a);
}

}  // namespace csa
