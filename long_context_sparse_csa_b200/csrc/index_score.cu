// Lightning-indexer scores:  s_i = sum_h w_h * ReLU(sigma_q,h * sigma_k,i * <q_h, k_i>).
//
// The pages describe the indexer only in words. "DeepSeek-V4 Explained: ...", section "The
// attention stack, and why it is two mechanisms", calls it a cheap low-rank scorer of the
// compressed entries. Step 3 of the per-query list in "DeepSeek-V4, explained." gives it a few small
// FP8 heads that score each past entry. This file holds the multi-head ReLU-weighted dot product the
// operator defines from that.
//
// Tensor-core path (FP8 e4m3 keys, d_I = 128): the score tile of 128 entries
// x (QN queries * H_I heads) is one tcgen05 kind::f8f6f4 MMA chain (M = 128
// entries, N = QN*H_I, K = 128 in four K=32 steps) with A = index keys staged
// by TMA in the 128-byte swizzle layout and B = index queries, accumulating
// in TMEM.  Two persistent CTAs per SM each run a 3-role pipeline: warp 0
// issues TMA loads into a ring (decode 4 stages, prefill 2), warp 1 issues the
// MMAs into TMEM accumulators (decode 4 of N = 32 columns, prefill 1 of
// N = 256: the two CTAs share the SM's 512 columns), warps 2-5 read an
// accumulator back with tcgen05.ld, apply the ReLU / head-weight epilogue and
// store the fp32 scores (coalesced).
// Decode streams the keys once from HBM; it is a bandwidth-bound kernel whose
// MMA keeps the 64 FLOP/byte of 32 heads off the CUDA cores.
//
// FP4 keys (e2m1 codes with a power-of-two key scale and per-32-dim block offsets, "DeepSeek-V4:
// Making a Million Tokens Affordable", "Two ways to shrink attention, interleaved": the indexer's
// attention runs in FP4) take the same pipeline at half the key bytes.  The tensor memory
// accelerator reads a tile's packed codes (64 bytes per key) and writes them 16 codes to a 16-byte
// chunk (8 bytes of codes, 8 of gap), so the shared-memory tile has the FP8 tile's 128-byte rows and
// swizzle; a second copy brings the tile's 128 scale words.  The MMA is kind::mxf8f6f4.block_scale
// with A = e2m1 keys and B = e4m3 queries: each 32-dim block of a key carries its own E8M0 scale,
// sigma * 2^-delta_b, which is exactly the key format's block scale, so the accumulator holds
// sigma_k * <q, k> and the epilogue is the FP8 one with a key scale of 1.  The MMA warp turns the
// scale words into the block-scale matrices (one per K-block of 32 dims: key l's scale in TMEM lane
// l % 32 of every 32-lane quarter, column l / 32) in shared memory and copies them into TMEM with
// tcgen05.cp ahead of the tile's MMAs; the query side's scales are all 1 (E8M0 127).
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "kernels.h"
#include "sm100.cuh"

namespace csa {

namespace {

using namespace sm100;

constexpr int kMaxStages = 6;                 // ring depth bound: decode runs 4 stages, prefill 2 (2 CTAs per SM)
constexpr int kTileE = 128;                 // entries per tile (MMA M)
constexpr int kDI = 128;                    // index-key bytes per entry
constexpr int kTileBytes = kTileE * kDI;    // 16 KB
constexpr int kThreads = 192;               // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kSfBytes = 512;               // FP4: 128 scale words of a tile; one 32 x 16 B scale matrix
// FP4 shared memory past the key ring: [stages][128] scale words, [stages][4][512] block-scale
// matrices, the query-scale matrix (1 KB slot, keeping the query tiles 1024-byte aligned)
__host__ __device__ constexpr size_t fp4_extra_smem(int stages) { return (size_t)stages * 5 * kSfBytes + 1024; }

__device__ __forceinline__ int64_t n_visible(const IndexArgs& a, int b, int j) {
  const int64_t t = a.q_pos[(int64_t)b * a.Tq + j];
  const int64_t r1 = t - a.pos0 + 1;
  const int64_t nv = r1 > 0 ? r1 / a.m : 0;
  return nv < a.n_max ? nv : a.n_max;
}

// A work item is (group g of QN queries of one sequence, entry tile et).  Tiles of a group past
// its last visible entry are skipped; validity is monotone in et within a group.
struct Group {
  int64_t g;
  int b, j0, j1;
  int last_et;                // last tile holding a visible entry (-1: none)
};

__device__ __forceinline__ Group group_info(const IndexArgs& a, int64_t g) {
  Group G;
  G.g = g;
  G.b = (int)(g / a.groups_per_seq);
  G.j0 = (int)(g % a.groups_per_seq) * a.QN;
  G.j1 = min(G.j0 + a.QN, a.Tq);
  int64_t nv = 0;
  for (int j = G.j0; j < G.j1; ++j) nv = max(nv, n_visible(a, G.b, j));
  G.last_et = (int)((nv + kTileE - 1) / kTileE) - 1;
  return G;
}

// The work items of one CTA, in order: item k -> (group g, entry tile et).  When there are no
// more groups than CTAs (decode), the CTAs are split evenly over the groups and each takes every
// Gc-th tile of its group, so at any moment the grid streams neighbouring tiles of the key cache
// rather than CTA-sized slabs far apart.  Otherwise (prefill) each CTA takes a contiguous range
// of items, which keeps its query tile resident across consecutive items.
struct Sched {
  bool strided;
  int64_t g0, w0, count, tpg;
  int et0, step;
  __device__ __forceinline__ void at(int64_t k, int64_t* g, int* et) const {
    if (strided) { *g = g0; *et = et0 + (int)k * step; }
    else { const int64_t w = w0 + k; *g = w / tpg; *et = (int)(w - *g * tpg); }
  }
};

__device__ __forceinline__ Sched make_sched(const IndexArgs& a) {
  Sched s;
  s.tpg = a.tiles_per_group;
  const int64_t groups = a.total_items / s.tpg;
  if (groups <= (int64_t)gridDim.x) {
    const int gc = (int)(gridDim.x / groups);
    s.strided = true;
    s.g0 = blockIdx.x / gc;
    s.et0 = blockIdx.x % gc;
    s.step = gc;
    s.w0 = 0;
    s.count = s.g0 < groups ? (s.tpg - s.et0 + gc - 1) / gc : 0;
  } else {
    s.strided = false;
    s.w0 = a.total_items * blockIdx.x / gridDim.x;
    s.count = a.total_items * (blockIdx.x + 1) / gridDim.x - s.w0;
    s.g0 = 0; s.et0 = 0; s.step = 1;
  }
  return s;
}

#ifdef CSA_TRACE
// Diagnostic build only: per-CTA timestamps (ns) of the indexer pipeline.
__device__ uint64_t g_trace[320][80];
#define TRACE(slot) do { if (blockIdx.x < 320) g_trace[blockIdx.x][(slot)] = global_timer_ns(); } while (0)
#define TRACE_VAL(slot, v) do { if (blockIdx.x < 320) g_trace[blockIdx.x][(slot)] = (uint64_t)(v); } while (0)
#define CYC() clock64()
#else
#define TRACE(slot) ((void)0)
#define TRACE_VAL(slot, v) ((void)0)
#define CYC() 0ll
#endif

constexpr int kHistBins = 4096;               // top 12 bits of the order-preserving score key
constexpr int kMaxQH = 256;                   // QN * H_I

constexpr int kMaxAcc = 4;                    // TMEM accumulators (decode: 4 x N columns; N = 256: 2)

struct __align__(8) Barriers {
  uint64_t full[kMaxStages], empty[kMaxStages];
  uint64_t bfull[2], bempty[2];
  uint64_t tfull[kMaxAcc], tempty[kMaxAcc];
  uint32_t tmem_base;
};

constexpr int kKsChunk = 8;                   // key-scale prefetch distance, in work items

struct EpiSmem {
  float w[kMaxQH];            // head weights of the group's queries
  float qs[kMaxQH];           // index-query scales
  float wq[kMaxQH];           // w * qs (used when every scale is positive)
  int pos[kMaxQH / 16];       // 1 when all of the query's index-query scales are > 0
  int64_t nv[kMaxQH / 16];    // visible entries per query (QN <= 16)
  float ks[kKsChunk][kTileE]; // key scales of the current chunk of items (each thread its own entry)
  uint32_t hist[kHistBins];   // score histogram of the current group (decode only: the prefill
                              // instantiation allocates the struct without it); 16-byte aligned
};
constexpr size_t kEpiSmemNoHist = sizeof(EpiSmem) - sizeof(uint32_t) * kHistBins;

__device__ __forceinline__ void epi_bar() { asm volatile("barrier.sync.aligned 5, 128;" ::: "memory"); }
// Set-up barrier: the producer warp arrives without waiting, the other five warps wait.
__device__ __forceinline__ void setup_arrive() { asm volatile("barrier.arrive.aligned 1, 192;" ::: "memory"); }
__device__ __forceinline__ void setup_sync() { asm volatile("barrier.sync.aligned 1, 192;" ::: "memory"); }

// Schedule bounds of group g as the three roles walk it.  In the strided (decode) schedule every
// tile below n_max is streamed, so that no query-position load gates the first key copy (entries
// past a query's visibility are masked by the epilogue); otherwise tiles past the group's last
// visible entry are skipped.
__device__ __forceinline__ Group sched_group(const IndexArgs& a, int64_t g, bool strided) {
  if (!strided) return group_info(a, g);
  Group G;
  G.g = g;
  G.b = (int)(g / a.groups_per_seq);
  G.j0 = (int)(g % a.groups_per_seq) * a.QN;
  G.j1 = min(G.j0 + a.QN, a.Tq);
  G.last_et = a.tiles_per_group - 1;
  return G;
}

// A group's per-query constants, as loaded by epilogue thread te (of 128): head weight and
// index-query scale of columns te and te + 128, the visibility of query te (te < QN).
struct GroupConsts {
  float w[2], qs[2];
  int64_t nv;
};

__device__ __forceinline__ GroupConsts load_group_consts(const IndexArgs& a, int64_t g, int te) {
  GroupConsts c;
  const int b = (int)(g / a.groups_per_seq), j0 = (int)(g % a.groups_per_seq) * a.QN;
  const int QH = a.QN * a.H_I;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int i = te + 128 * r;
    c.w[r] = 0.f;
    c.qs[r] = 0.f;
    if (i < QH) {
      const int j = j0 + i / a.H_I;
      const int64_t row = (int64_t)b * a.Tq + (j < a.Tq ? j : a.Tq - 1);
      c.w[r] = __ldg(a.head_w + row * a.H_I + i % a.H_I);
      c.qs[r] = __ldg(a.q_scale + row * a.H_I + i % a.H_I);
    }
  }
  c.nv = (te < a.QN && j0 + te < a.Tq) ? n_visible(a, b, j0 + te) : 0;
  return c;
}

// Issues the key-scale loads of items [k0, k0 + kKsChunk) for entry lane e_loc (0 past the end).
// FP4 keys carry their scales into the MMA: the epilogue's key scale is 1.
template <bool kFP4>
__device__ __forceinline__ void load_key_scales(const IndexArgs& a, const Sched& sc, int64_t k0, int e_loc,
                                                float ks[kKsChunk]) {
#pragma unroll
  for (int u = 0; u < kKsChunk; ++u) {
    ks[u] = 0.f;
    if (kFP4) {
      ks[u] = 1.f;
      continue;
    }
    if (k0 + u < sc.count) {
      int64_t g;
      int et;
      sc.at(k0 + u, &g, &et);
      const int64_t e = (int64_t)et * kTileE + e_loc;
      if (e < a.n_max) ks[u] = __ldg(a.k_scale + (g / a.groups_per_seq) * a.entry_cap + e);
    }
  }
}

// kHI > 0: decode specialisation (one query per group, kHI index heads, head weights in registers);
// kHI == 0: any QN x H_I (prefill).  kFP4: e2m1 keys with block scales (smap: their scale words).
// Chunk mode: the scores of key e for the queries whose HI columns sit in v (64 accumulator columns
// starting at column c0 of the group's ncol).  v is indexed with constants only, so it stays in
// registers.
template <int HI>
__device__ __forceinline__ void chunk_scores(const IndexArgs& a, const EpiSmem* es, const Group& G, const float (&v)[64],
                                             int c0, int ncol, int64_t e, float ks, bool in_range, bool use_hist,
                                             uint32_t* hist, int lane) {
#pragma unroll
  for (int qq = 0; qq < 64 / HI; ++qq) {
    if (c0 + qq * HI >= ncol) break;
    const int q = c0 / HI + qq;
    const int64_t row = (int64_t)G.b * a.Tq + G.j0 + q;
    // positive scales: ReLU(qs * ks * v) = qs * ks * ReLU(v), so s = ks * sum_h (w*qs)_h ReLU(v_h)
    const bool fast = es->pos[q] && ks > 0.f;
    float sc = 0.f;
    if (fast) {
      const float4* wqq = reinterpret_cast<const float4*>(es->wq + q * HI);
#pragma unroll
      for (int h = 0; h < HI; h += 4) {
        const float4 w4 = wqq[h / 4];
        sc = fmaf(w4.x, fmaxf(v[qq * HI + h], 0.f), sc);
        sc = fmaf(w4.y, fmaxf(v[qq * HI + h + 1], 0.f), sc);
        sc = fmaf(w4.z, fmaxf(v[qq * HI + h + 2], 0.f), sc);
        sc = fmaf(w4.w, fmaxf(v[qq * HI + h + 3], 0.f), sc);
      }
      sc *= ks;
    } else {
      const float* wq = es->w + q * HI;
      const float* sq = es->qs + q * HI;
#pragma unroll
      for (int h = 0; h < HI; ++h) sc += wq[h] * fmaxf(v[qq * HI + h] * (sq[h] * ks), 0.f);
    }
    const bool vis = e < es->nv[q];
    if (in_range) a.scores[row * a.n_max + e] = vis ? sc : -INFINITY;
    if (use_hist) {
      // one shared-memory atomic per distinct bin in the warp
      const uint32_t bin = vis ? (float_key(sc) >> 20) : 0xFFFFFFFFu;
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (bin != 0xFFFFFFFFu && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
    }
  }
}

template <int kStages, int kHI, bool kFP4>
__global__ void __launch_bounds__(kThreads, 2)
index_score_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                      const __grid_constant__ CUtensorMap smap, const __grid_constant__ IndexArgs a, int N,
                      int nacc, uint32_t tmem_cols) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* A = smem;                                  // [kStages][kTileBytes]
  uint8_t* SFw = A + kStages * kTileBytes;            // FP4: [kStages][128] key scale words
  uint8_t* SFs = SFw + kStages * kSfBytes;            // FP4: [kStages][4 K-blocks][32 x 16 B] block scales
  uint8_t* SFq = SFs + kStages * 4 * kSfBytes;        // FP4: the query side's block scales (all 1)
  uint8_t* Bq = kFP4 ? A + kStages * kTileBytes + fp4_extra_smem(kStages) : A + kStages * kTileBytes;  // [2][N * 128]
  Barriers* bars = reinterpret_cast<Barriers*>(Bq + 2 * N * kDI);
  EpiSmem* es = reinterpret_cast<EpiSmem*>(reinterpret_cast<uint8_t*>(bars) + ((sizeof(Barriers) + 15) & ~size_t(15)));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Sched sc = make_sched(a);
  if (threadIdx.x == 0) TRACE(0);
  // Epilogue warps issue the first group's constants and the first chunk of key scales now: their
  // latency then overlaps the set-up below and the first key tile's copy.
  const int te = threadIdx.x - 64;            // epilogue thread 0..127
  const int e_loc = (warp & 3) * 32 + lane;   // epilogue: entry row = TMEM lane of this warp's quarter
  GroupConsts gc0;
  float ks_cur[kKsChunk];
  if (warp >= 2 && sc.count > 0) {
    int64_t g;
    int et;
    sc.at(0, &g, &et);
    gc0 = load_group_consts(a, g, te);
    load_key_scales<kFP4>(a, sc, 0, e_loc, ks_cur);
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&bars->full[s], 1); mbar_init(&bars->empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&bars->bfull[s], 1); mbar_init(&bars->bempty[s], 1); }
    for (int s = 0; s < kMaxAcc; ++s) { mbar_init(&bars->tfull[s], 1); mbar_init(&bars->tempty[s], 128); }
    fence_barrier_init();
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&qmap);
    if (kFP4) prefetch_tensormap(&smap);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, tmem_cols);
    tmem_relinquish();
  }
  // The producer needs neither TMEM nor the other warps: it arrives at the set-up barrier (its
  // barrier initialisation is then visible to the waiting warps) and starts copying at once.
  uint32_t tmem = 0;
  if (warp == 0) {
    __syncwarp();
    setup_arrive();
  } else {
    tc_fence_before();
    setup_sync();
    tc_fence_after();
    tmem = bars->tmem_base;
    if (threadIdx.x == 32) TRACE(71);
    if (threadIdx.x == 64) TRACE(72);
  }
  if (threadIdx.x == 0) TRACE(1);

  // The producer and MMA warps run their loops with all 32 lanes (every wait is warp-uniform) and
  // let lane 0 alone issue the bulk copies, MMAs and commits, so no warp reaches a block barrier
  // while one of its lanes is still working.
  auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity)) != 0;
  };
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    Group G;
    G.g = -1;
    int gi = -1;
    int issued_par[kStages];
    for (int s = 0; s < kStages; ++s) issued_par[s] = -1;
    int b_issued_par[2] = {-1, -1};
    bool ok = true;
    for (int64_t k = 0; k < sc.count && ok; ++k) {
      int64_t g;
      int et;
      sc.at(k, &g, &et);
      if (g != G.g) G = sched_group(a, g, sc.strided);
      if (et > G.last_et) continue;
      // validity is monotone in et, so the first item of a group in this CTA is its first valid one
      int64_t gp = -1;
      int etp;
      if (k > 0) sc.at(k - 1, &gp, &etp);
      const bool first_of_group = (k == 0) || gp != g;
      if (first_of_group) {
        ++gi;
        const int slot = gi & 1;
        const uint32_t use = (uint32_t)(gi >> 1);
        if (!wait_all(&bars->bempty[slot], (use & 1u) ^ 1u)) { ok = false; break; }
        if (lane == 0) {
          mbar_arrive_expect_tx(&bars->bfull[slot], (uint32_t)(N * kDI));
          tma_load_2d(Bq + slot * N * kDI, &qmap, &bars->bfull[slot], 0,
                      (int)(((int64_t)G.b * a.Tq + G.j0) * a.H_I));
        }
        __syncwarp();
        b_issued_par[slot] = (int)(use & 1u);
      }
      if (!wait_all(&bars->empty[stage], phase ^ 1u)) { ok = false; break; }
      if (lane == 0) {
        // FP4: the box's packed codes are half its shared-memory footprint, plus the scale words
        mbar_arrive_expect_tx(&bars->full[stage], kFP4 ? (uint32_t)(kTileBytes / 2 + kSfBytes) : (uint32_t)kTileBytes);
        tma_load_2d(A + stage * kTileBytes, &kmap, &bars->full[stage], 0,
                    (int)((int64_t)G.b * a.entry_cap + (int64_t)et * kTileE));
        if (kFP4) tma_load_2d(SFw + stage * kSfBytes, &smap, &bars->full[stage], et * kTileE, G.b);
        if (k < 16) TRACE(2 + k);
      }
      __syncwarp();
      issued_par[stage] = (int)phase;
      if (++stage == kStages) { stage = 0; phase ^= 1u; }
    }
    if (!ok && lane == 0) set_device_error(a.err, kErrWaitTimeout);
    // never leave a bulk copy in flight when the CTA exits
    for (int s = 0; s < kStages; ++s)
      if (issued_par[s] >= 0) wait_all(&bars->full[s], (uint32_t)issued_par[s]);
    for (int s = 0; s < 2; ++s)
      if (b_issued_par[s] >= 0) wait_all(&bars->bfull[s], (uint32_t)b_issued_par[s]);
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    const uint32_t idesc = kFP4 ? instr_desc_block_scaled(128, N, 5u, 0u) : instr_desc(128, N, 0u);
    // FP4: TMEM columns [sfa0 + 16 acc, + 16) hold accumulator acc's key block scales (4 columns per
    // K-block), [sfq, sfq + 4) the query side's (all 1: E8M0 127)
    const uint32_t sfa0 = ((uint32_t)(nacc * N) + 15u) & ~15u;
    const uint32_t sfq = sfa0 + 16u * (uint32_t)nacc;
    // (copied into TMEM just before the first MMA, so that every copy is followed by an MMA whose
    // completion the end of the loop waits for)
    bool sfq_copied = false;
    if (kFP4) {
      reinterpret_cast<uint4*>(SFq)[lane] = make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
      fence_proxy_async_smem();
      __syncwarp();
    }
    int stage = 0, acc = 0, gi = -1;
    uint32_t phase = 0, acc_phase = 0;
    Group G;
    G.g = -1;
    int last_acc = -1;
    uint32_t last_acc_par = 0;
    bool ok = true;
    for (int64_t k = 0; k < sc.count; ++k) {
      int64_t g;
      int et;
      sc.at(k, &g, &et);
      if (g != G.g) G = sched_group(a, g, sc.strided);
      if (et > G.last_et) continue;
      int64_t gp = -1;
      int etp;
      if (k > 0) sc.at(k - 1, &gp, &etp);
      const bool first_of_group = (k == 0) || gp != g;
      if (first_of_group) {
        ++gi;
        if (!wait_all(&bars->bfull[gi & 1], (uint32_t)((gi >> 1) & 1))) { ok = false; break; }
      }
      const int slot = gi & 1;
      if (!wait_all(&bars->full[stage], phase)) { ok = false; break; }
      if (lane == 0 && k < 16) TRACE(18 + k);
      if (!wait_all(&bars->tempty[acc], acc_phase ^ 1u)) { ok = false; break; }
      // release the query tile after the group's last valid item in this CTA
      bool last_of_group = k + 1 >= sc.count;
      if (!last_of_group) {
        int64_t gn;
        int etn;
        sc.at(k + 1, &gn, &etn);
        last_of_group = gn != g || etn > G.last_et;
      }
      uint8_t* sfs = SFs + stage * 4 * kSfBytes;
      if (kFP4) {
        // scale words of keys l, 32 + l, 64 + l, 96 + l -> row l of each K-block's block-scale matrix:
        // E8M0 of sigma * 2^-delta_kk = (exponent byte) - delta_kk
        const uint32_t* raw = reinterpret_cast<const uint32_t*>(SFw + stage * kSfBytes);
        uint32_t wv[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) wv[c] = raw[32 * c + lane];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t o[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int e8 = (int)(wv[c] & 0xFFu) - (int)((wv[c] >> (8 + 4 * kk)) & 0xFu);
            o[c] = (uint32_t)(e8 > 0 ? e8 : 0) * 0x01010101u;
          }
          reinterpret_cast<uint4*>(sfs + kk * kSfBytes)[lane] = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      if (lane == 0) {
        tc_fence_after();
        const uint64_t ad = desc_kmajor_sw128(smem_u32(A + stage * kTileBytes));
        const uint64_t bd = desc_kmajor_sw128(smem_u32(Bq + slot * N * kDI));
        if (kFP4) {
          const uint32_t sfa = tmem + sfa0 + 16u * (uint32_t)acc;
          if (!sfq_copied) {
            tmem_cp_32x128b_x4(tmem + sfq, desc_noswizzle(smem_u32(SFq), 128u));
            sfq_copied = true;
          }
#pragma unroll
          for (int kk = 0; kk < kDI / 32; ++kk)
            tmem_cp_32x128b_x4(sfa + 4u * kk, desc_noswizzle(smem_u32(sfs + kk * kSfBytes), 128u));
#pragma unroll
          for (int kk = 0; kk < kDI / 32; ++kk)
            umma_mxf8f6f4(tmem + (uint32_t)(acc * N), ad + 2u * kk, bd + 2u * kk, idesc, sfa + 4u * kk, tmem + sfq,
                          kk > 0 ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < kDI / 32; ++kk)
            umma_f8f6f4(tmem + (uint32_t)(acc * N), ad + 2u * kk, bd + 2u * kk, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->empty[stage]);
        umma_commit(&bars->tfull[acc]);
        if (last_of_group) umma_commit(&bars->bempty[slot]);
      }
      __syncwarp();
      last_acc = acc;
      last_acc_par = acc_phase;
      if (++stage == kStages) { stage = 0; phase ^= 1u; }
      if (++acc == nacc) { acc = 0; acc_phase ^= 1u; }
    }
    if (!ok && lane == 0) set_device_error(a.err, kErrWaitTimeout);
    // the accumulator must be idle before TMEM is released
    if (last_acc >= 0) wait_all(&bars->tfull[last_acc], last_acc_par);
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    // Every epilogue warp runs the same sequence of named barriers whatever happens (a wait that
    // times out only stops the warp's work), so the 128-thread barrier can never be left short.
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const bool use_hist = kHI > 0 && a.hist != nullptr && a.QN == 1;
    const int QH = a.QN * a.H_I;
    if (use_hist)
      for (int i = te; i < kHistBins; i += 128) es->hist[i] = 0u;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    Group G;
    G.g = -1;
    // decode: the group's w * qs per head, its scale positivity and visibility, in registers
    float wr[kHI > 0 ? kHI : 1];
    int pos_reg = 0;
    int64_t nv_reg = 0;
    // adds the shared histogram into the row's global one (one reduction per non-empty bin)
    auto flush_hist = [&](const Group& H, bool clear) {
      uint32_t* dst = a.hist + ((int64_t)H.b * a.Tq + H.j0) * kHistBins;
      uint4* src = reinterpret_cast<uint4*>(es->hist);
      uint4 v[kHistBins / 4 / 128];
#pragma unroll
      for (int r = 0; r < kHistBins / 4 / 128; ++r) v[r] = src[te + 128 * r];
#pragma unroll
      for (int r = 0; r < kHistBins / 4 / 128; ++r) {
        uint32_t* d = dst + 4 * (te + 128 * r);
        if (v[r].x) atomicAdd(d + 0, v[r].x);
        if (v[r].y) atomicAdd(d + 1, v[r].y);
        if (v[r].z) atomicAdd(d + 2, v[r].z);
        if (v[r].w) atomicAdd(d + 3, v[r].w);
        if (clear) src[te + 128 * r] = make_uint4(0u, 0u, 0u, 0u);
      }
    };
    auto enter_group = [&](int64_t g, const GroupConsts& c) {
      epi_bar();
      if (use_hist && G.g >= 0) flush_hist(G, true);
      G = sched_group(a, g, sc.strided);
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int i = te + 128 * r;
        if (i < QH) {
          es->w[i] = c.w[r];
          es->qs[i] = c.qs[r];
          es->wq[i] = c.w[r] * c.qs[r];
        }
      }
      if (te < a.QN) es->nv[te] = c.nv;
      epi_bar();
      if (te < a.QN) {
        int p = 1;
        for (int h = 0; h < a.H_I; ++h) p &= es->qs[te * a.H_I + h] > 0.f;
        es->pos[te] = p;
      }
      epi_bar();
      if constexpr (kHI > 0) {
#pragma unroll
        for (int h = 0; h < kHI; ++h) wr[h] = es->wq[h];
        pos_reg = es->pos[0];
        nv_reg = es->nv[0];
      }
    };
    int done = 0;
    long long cyc_wait = 0, cyc_ld = 0, cyc_st = 0, cyc_all = 0;
    float ks_nxt[kKsChunk];
    for (int64_t k0 = 0; k0 < sc.count; k0 += kKsChunk) {
      // this chunk's key scales (loaded one chunk ago) go to shared memory, the next chunk's are
      // issued now and land while this chunk is processed
#pragma unroll
      for (int u = 0; u < kKsChunk; ++u) es->ks[u][e_loc] = ks_cur[u];
      const bool more = k0 + kKsChunk < sc.count;
      if (more) load_key_scales<kFP4>(a, sc, k0 + kKsChunk, e_loc, ks_nxt);
      const int kn = (int)min((int64_t)kKsChunk, sc.count - k0);
      for (int u = 0; u < kn; ++u) {
        const int64_t k = k0 + u;
        int64_t g;
        int et;
        sc.at(k, &g, &et);
        if (g != G.g) {
          enter_group(g, G.g < 0 ? gc0 : load_group_consts(a, g, te));
          if (threadIdx.x == 64 && done == 0) TRACE(73);
        }
        if (et > G.last_et) continue;
        const int64_t e = (int64_t)et * kTileE + e_loc;
        const bool in_range = e < a.n_max;
        const float ks = es->ks[u][e_loc];
        long long c0 = CYC();
        if (ok) ok = mbar_wait(&bars->tfull[acc], acc_phase);
        long long c1 = CYC();
        if (threadIdx.x == 64 && done < 16) TRACE(34 + done);
        if (ok && kHI > 0) {
          // decode: one query, kHI columns of the accumulator
          tc_fence_after();
          float v[kHI > 0 ? kHI : 1];
          if constexpr (kHI == 16) {
            tmem_ld_32x32b_x16(lane_addr + (uint32_t)(acc * N), v);
          } else if constexpr (kHI > 0) {
#pragma unroll
            for (int hc = 0; hc < kHI; hc += 32) tmem_ld_32x32b_x32(lane_addr + (uint32_t)(acc * N + hc), v + hc);
          }
          tmem_wait_ld();
          cyc_ld += CYC() - c1;
          tc_fence_before();
          mbar_arrive(&bars->tempty[acc]);
          float s = 0.f;
          if (pos_reg && ks > 0.f) {
            // positive scales: ReLU(qs * ks * v) = qs * ks * ReLU(v)
#pragma unroll
            for (int h = 0; h < kHI; ++h) s = fmaf(wr[h], fmaxf(v[h], 0.f), s);
            s *= ks;
          } else {
#pragma unroll
            for (int h = 0; h < kHI; ++h) s += es->w[h] * fmaxf(v[h] * (es->qs[h] * ks), 0.f);
          }
          long long c2 = CYC();
          const bool vis = e < nv_reg;
          if (in_range) a.scores[((int64_t)G.b * a.Tq + G.j0) * a.n_max + e] = vis ? s : -INFINITY;
          if (use_hist && vis) atomicAdd(&es->hist[float_key(s) >> 20], 1u);
          cyc_st += CYC() - c2;
        } else if (ok) {
          // chunk mode: the group's queries j0 .. j1 - 1, H_I columns each, read 64 columns (two or four
          // queries) per TMEM wait
          tc_fence_after();
          const int nq = G.j1 - G.j0, ncol = nq * a.H_I;
          for (int c0 = 0; c0 < ncol; c0 += 64) {
            float v[64];
            tmem_ld_32x32b_x32(lane_addr + (uint32_t)(acc * N + c0), v);
            if (c0 + 32 < ncol) tmem_ld_32x32b_x32(lane_addr + (uint32_t)(acc * N + c0 + 32), v + 32);
            tmem_wait_ld();
            cyc_ld += CYC() - c1;
            if (c0 + 64 >= ncol) {
              // every column of this accumulator is in registers: hand it back to the MMA warp
              tc_fence_before();
              mbar_arrive(&bars->tempty[acc]);
            }
            long long c2 = CYC();
            if (a.H_I == 32)
              chunk_scores<32>(a, es, G, v, c0, ncol, e, ks, in_range, use_hist, es->hist, lane);
            else
              chunk_scores<16>(a, es, G, v, c0, ncol, e, ks, in_range, use_hist, es->hist, lane);
            cyc_st += CYC() - c2;
          }
        }
        cyc_wait += c1 - c0;
        cyc_all += CYC() - c0;
        if (++acc == nacc) { acc = 0; acc_phase ^= 1u; }
        if (threadIdx.x == 64 && done < 16) TRACE(50 + done);
        ++done;
      }
      if (more) {
#pragma unroll
        for (int u = 0; u < kKsChunk; ++u) ks_cur[u] = ks_nxt[u];
      }
    }
    if (threadIdx.x == 64) {
      TRACE_VAL(74, cyc_wait);
      TRACE_VAL(75, cyc_ld);
      TRACE_VAL(76, cyc_st);
      TRACE_VAL(77, cyc_all);
    }
    epi_bar();
    if (use_hist && G.g >= 0) flush_hist(G, false);
    if (!ok) set_device_error(a.err, kErrWaitTimeout);
  }

  if (threadIdx.x == 0) TRACE(68);
  if (threadIdx.x == 64) TRACE(70);
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) TRACE(66);
  if (threadIdx.x == 64) TRACE(67);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// CUDA-core path for float32 index tensors or shapes the tensor-core kernel does not take.
__global__ void index_score_generic_kernel(const __grid_constant__ IndexArgs a) {
  extern __shared__ float qv[];                      // [H_I][d_I]
  const int64_t row = blockIdx.y;
  const int b = (int)(row / a.Tq), j = (int)(row % a.Tq);
  const int nq = a.H_I * a.d_I;
  for (int i = threadIdx.x; i < nq; i += blockDim.x) {
    qv[i] = a.idx_fmt == CSA_FMT_F32 ? reinterpret_cast<const float*>(a.idx_q)[row * nq + i]
                                     : e4m3_to_f(a.idx_q[row * nq + i]);
  }
  __syncthreads();
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= a.n_max) return;
  if (e >= n_visible(a, b, j)) { a.scores[row * a.n_max + e] = -INFINITY; return; }
  const int64_t krow = (int64_t)b * a.entry_cap + e;
  // FP4 keys: the scale word holds the key scale's exponent and the 32-dim blocks' offsets
  const uint32_t word = a.idx_fmt == CSA_FMT_E2M1 ? reinterpret_cast<const uint32_t*>(a.k_scale)[krow] : 0u;
  const float ks = a.idx_fmt == CSA_FMT_E2M1 ? __uint_as_float((word & 0xFFu) << 23) : a.k_scale[krow];
  float s = 0.f;
  for (int h = 0; h < a.H_I; ++h) {
    float dot = 0.f;
    if (a.idx_fmt == CSA_FMT_F32) {
      const float* k = reinterpret_cast<const float*>(a.idx_k) + krow * a.d_I;
      for (int d = 0; d < a.d_I; ++d) dot += qv[h * a.d_I + d] * k[d];
    } else if (a.idx_fmt == CSA_FMT_E2M1) {
      const uint8_t* k = a.idx_k + krow * (a.d_I / 2);
      for (int d = 0; d < a.d_I; ++d) {
        const uint32_t code = (k[d >> 1] >> ((d & 1) * 4)) & 0xFu;
        const int delta = (int)((word >> (8 + 4 * (d >> 5))) & 0xFu);
        dot += qv[h * a.d_I + d] * (e2m1_to_f(code) * __uint_as_float((uint32_t)(127 - delta) << 23));
      }
    } else {
      const uint8_t* k = a.idx_k + krow * a.d_I;
      for (int d = 0; d < a.d_I; ++d) dot += qv[h * a.d_I + d] * e4m3_to_f(k[d]);
    }
    s += a.head_w[row * a.H_I + h] * fmaxf(dot * (a.q_scale[row * a.H_I + h] * ks), 0.f);
  }
  a.scores[row * a.n_max + e] = s;
}

// ----------------------------------------------------------------------------- host side
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

// 2D byte tensor [rows][128] with a 128-byte-swizzled box of box_rows x 128.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kDI, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kDI};
  cuuint32_t box[2] = {(cuuint32_t)kDI, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// FP4 keys [rows][64 bytes] (128 e2m1 codes each) as 128 x 128 boxes: the codes land 16 to a 16-byte
// chunk (8 bytes of codes, then 8 of gap), rows of 128 bytes in the 128-byte swizzle.  Needs a
// 32-byte aligned base.
bool make_map_fp4(CUtensorMap* m, const void* base, uint64_t rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kDI, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(kDI / 2)};
  cuuint32_t box[2] = {(cuuint32_t)kDI, (cuuint32_t)kTileE};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// FP4 scale words [B][entry_cap] (uint32) as boxes of 128 words of one sequence, zero past entry_cap.
// Needs entry_cap a multiple of 4 (16-byte row pitch) and a 16-byte aligned base.
bool make_scale_map(CUtensorMap* m, const void* base, uint64_t entry_cap, uint64_t B) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)entry_cap, (cuuint64_t)B};
  cuuint64_t strides[1] = {(cuuint64_t)(entry_cap * 4)};
  cuuint32_t box[2] = {(cuuint32_t)kTileE, 1};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

#ifdef CSA_TRACE
extern "C" __attribute__((visibility("default"))) int csa_trace_read(uint64_t* host, int n) {
  return (int)cudaMemcpyFromSymbol(host, g_trace, sizeof(uint64_t) * (size_t)n);
}
#endif

bool index_tc_supported(int idx_fmt, int H_I, int d_I) {
  return idx_fmt == CSA_FMT_E4M3 && d_I == kDI && (H_I == 16 || H_I == 32 || H_I == 64);
}

namespace {

// FP4 keys on the tensor-core kernel: d_I = 128, 16 or 32 heads (two CTAs per SM fit the extra
// shared memory), a scale-word pitch the tensor memory accelerator can step (entry_cap a multiple of
// 4), and the base alignments its boxes need.
bool index_tc_fp4_ok(const IndexArgs& a) {
  return a.idx_fmt == CSA_FMT_E2M1 && a.d_I == kDI && (a.H_I == 16 || a.H_I == 32) && a.entry_cap % 4 == 0 &&
         (reinterpret_cast<uintptr_t>(a.idx_k) & 31u) == 0 && (reinterpret_cast<uintptr_t>(a.k_scale) & 15u) == 0;
}

template <bool kFP4>
using TcKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, IndexArgs, int, int, uint32_t);

template <bool kFP4>
TcKernel<kFP4> tc_kernel(bool decode, int H_I) {
  if (!decode) return index_score_tc_kernel<2, 0, kFP4>;
  if (H_I == 16) return index_score_tc_kernel<4, 16, kFP4>;
  if constexpr (kFP4) {
    return index_score_tc_kernel<4, 32, kFP4>;            // FP4 takes 16 or 32 heads
  } else {
    if (H_I == 32) return index_score_tc_kernel<4, 32, kFP4>;
    return index_score_tc_kernel<4, 64, kFP4>;
  }
}

}  // namespace

cudaError_t launch_index_scores(IndexArgs a, int num_sms, cudaStream_t s) {
  if (a.n_max <= 0 || a.Tq <= 0 || a.B <= 0) return cudaSuccess;
  const bool fp4 = index_tc_fp4_ok(a);
  // FP4 keys the tensor-core kernel does not take: the warp-level streaming kernel in decode (it also
  // fills the top-k's histogram), else the CUDA-core kernel below
  if (a.idx_fmt == CSA_FMT_E2M1 && !fp4 && a.Tq == 1 && index_decode_supported(a.idx_fmt, a.H_I, a.d_I))
    return launch_index_decode(a, num_sms, s);
  if (!fp4 && !index_tc_supported(a.idx_fmt, a.H_I, a.d_I)) {
    dim3 grid((unsigned)((a.n_max + 127) / 128), (unsigned)(a.B * a.Tq));
    const size_t sm = (size_t)a.H_I * a.d_I * sizeof(float);
    if (sm > 0) {
      cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(index_score_generic_kernel), sm);
      if (e != cudaSuccess) return e;
    }
    return launch_kernel(index_score_generic_kernel, grid, dim3(128), sm, s, 0, a);
  }
  // FP4 prefill tiles hold at most 128 query columns, so the accumulator and the block-scale columns
  // fit the CTA's 256 TMEM columns
  a.QN = a.Tq == 1 ? 1 : min((fp4 ? 128 : 256) / a.H_I, a.Tq);
  const int N = a.QN * a.H_I;
  a.tiles_per_group = (int)((a.n_max + kTileE - 1) / kTileE);
  a.groups_per_seq = (a.Tq + a.QN - 1) / a.QN;
  a.total_items = (int64_t)a.B * a.groups_per_seq * a.tiles_per_group;
  CUtensorMap kmap, qmap, smap;
  memset(&smap, 0, sizeof(smap));
  if (fp4) {
    if (!make_map_fp4(&kmap, a.idx_k, (uint64_t)a.B * a.entry_cap)) return cudaErrorInvalidValue;
    if (!make_scale_map(&smap, a.k_scale, (uint64_t)a.entry_cap, (uint64_t)a.B)) return cudaErrorInvalidValue;
  } else if (!make_map(&kmap, a.idx_k, (uint64_t)a.B * a.entry_cap, kTileE)) {
    return cudaErrorInvalidValue;
  }
  if (!make_map(&qmap, a.idx_q, (uint64_t)a.B * a.Tq * a.H_I, (uint32_t)N)) return cudaErrorInvalidValue;
  const bool decode = a.Tq == 1;
  // two CTAs per SM in both modes (two independent pipelines, twice the epilogue warps); their TMEM
  // shares the SM's 512 columns: decode 4 accumulators of N <= 64 columns, prefill one of N = 256
  // (FP4: N <= 128, plus 16 block-scale columns per accumulator and 4 for the query side)
  const int nacc = decode ? 4 : 1;
  const uint32_t need = fp4 ? (((uint32_t)(nacc * N) + 15u) & ~15u) + 16u * (uint32_t)nacc + 4u : (uint32_t)(nacc * N);
  uint32_t cols = 32;
  while (cols < need) cols <<= 1;
  const int stages = decode ? 4 : 2;
  const size_t smem = 1024 + (size_t)stages * kTileBytes + (fp4 ? fp4_extra_smem(stages) : 0) + 2 * (size_t)N * kDI +
                      ((sizeof(Barriers) + 15) & ~size_t(15)) + (decode ? sizeof(EpiSmem) : kEpiSmemNoHist) + 64;
  const void* kern = fp4 ? reinterpret_cast<const void*>(tc_kernel<true>(decode, a.H_I))
                         : reinterpret_cast<const void*>(tc_kernel<false>(decode, a.H_I));
  {
    cudaError_t e = ensure_dynamic_smem(kern, smem);
    if (e != cudaSuccess) return e;
  }
  const int64_t ctas = 2 * (int64_t)num_sms;
  const int64_t grid = a.total_items < ctas ? a.total_items : ctas;
  if (fp4)
    return launch_kernel(tc_kernel<true>(decode, a.H_I), dim3((unsigned)grid), dim3(kThreads), smem, s, 0, kmap, qmap,
                         smap, a, N, nacc, cols);
  return launch_kernel(tc_kernel<false>(decode, a.H_I), dim3((unsigned)grid), dim3(kThreads), smem, s, 0, kmap, qmap,
                       smap, a, N, nacc, cols);
}

}  // namespace csa
