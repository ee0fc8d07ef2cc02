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
// Decode: a thread-block cluster per (token, sequence) splits the channels
// (8 CTAs, or 16 for long pooling windows); inside a CTA, threads of 4
// consecutive channels times row groups that pool strided subsets of the
// window with an online softmax in registers, merged in shared memory; the
// row-wide RMSNorm sum and FP8 amax are reduced over the cluster by mail.
// Chunked prefill: one CTA per token.  Raw rows are read once with 8/16-byte
// vector loads.
#include <cooperative_groups.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace cg = cooperative_groups;

namespace csa {

namespace {

// Error word of calls that take no workspace (csa_append, csa_compress), one per device.
__device__ int g_library_error;

#ifdef CSA_TRACE
__device__ uint64_t g_trace_c[4][16];
#define CTRACE(slot) do { if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) { \
    uint64_t _t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(_t) :: "memory"); \
    g_trace_c[(L.m == 4) ? 0 : 1][(slot)] = _t; } } while (0)
#define CTRACE_C(slot) do { if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) \
    g_trace_c[(L.m == 4) ? 0 : 1][(slot)] = (uint64_t)clock64(); } while (0)
#else
#define CTRACE(slot) ((void)0)
#define CTRACE_C(slot) ((void)0)
#endif

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

constexpr int kRowBatch = 8;   // rows whose loads are issued together per thread

// Cluster-wide reductions by mail: each CTA sends its partial to every CTA of the cluster (itself
// included) with st.async into that CTA's mailbox, the bytes counted on the receiver's mbarrier, and
// every CTA reduces the CL partials it received.  No cluster barrier per reduction: a barrier's
// release would first wait for this CTA's outstanding global stores (the window and raw rows).
// Mailbox k serves one reduction per launch: 0 the window row's FP8 amax, 1 the entry's RMSNorm
// sum and FP8 amax.
constexpr int kMailMaxCl = 16;
struct ClusterMail {
  uint64_t bar[2];
  float2 box[2][kMailMaxCl];   // box[k][sender rank]
};

__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// Threads 0..CL-1 each send v to one CTA of the cluster.
__device__ __forceinline__ void mail_send(ClusterMail* m, int k, int q, int CL, float2 v) {
  if ((int)threadIdx.x >= CL) return;
  const uint32_t to = threadIdx.x;
  uint32_t rd, rb;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rd) : "r"(sm100::smem_u32(&m->box[k][q])), "r"(to));
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rb) : "r"(sm100::smem_u32(&m->bar[k])), "r"(to));
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];"
               ::"r"(rd), "f"(v.x), "f"(v.y), "r"(rb)
               : "memory");
}

// Waits (bounded) for the CL partials of mailbox k; every thread gets (sum of .x, max of .y).  A
// wait that gives up sets the error word's timeout bit: the reduced values are then incomplete.
__device__ __forceinline__ float2 mail_reduce(ClusterMail* m, int k, int CL, int* err) {
  if (!sm100::mbar_wait(&m->bar[k], 0u)) set_device_error(err, kErrWaitTimeout);
  float x = 0.f, y = -INFINITY;
  for (int p = 0; p < CL; ++p) {
    const float2 v = m->box[k][p];
    x += v.x;
    y = fmaxf(y, v.y);
  }
  return make_float2(x, y);
}

// Block sum of s and block max of m, in thread 0 (scratch: 64 floats).
__device__ __forceinline__ float2 block_sum_max(float s, float m, float* scratch) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  s = warp_sum(s);
  m = warp_max(m);
  __syncthreads();
  if (lane == 0) { scratch[wid] = s; scratch[32 + wid] = m; }
  __syncthreads();
  float x = 0.f, y = -INFINITY;
  if (threadIdx.x < 32) {
    x = lane < nw ? scratch[lane] : 0.f;
    y = lane < nw ? scratch[32 + lane] : -INFINITY;
    x = warp_sum(x);
    y = warp_max(y);
  }
  return make_float2(x, y);
}

// Stores this CTA's channels of one row in the cache format.  `am` is the cluster-wide max |x|
// over the FP8 dims (mixed format only); threads with active == false hold no channels.
__device__ __forceinline__ void pack_slice(uint8_t* dst, const LayerArgs& L, int c0, const float v[4], bool active,
                                           float am, bool writes_scale) {
  if (L.kv_fmt == CSA_FMT_F32) {
    if (active) *reinterpret_cast<float4*>(dst + 4 * (size_t)c0) = make_float4(v[0], v[1], v[2], v[3]);
    return;
  }
  if (L.kv_fmt == CSA_FMT_BF16) {
    if (active) store_act4(dst, CSA_FMT_BF16, c0, v);
    return;
  }
  const int dn = L.D - L.d_rope;
  float inv;
  const float sig = pow2_scale(am, &inv);
  if (active) {
    if (c0 < dn) {
      uint32_t w = (uint32_t)f_to_e4m3_sat(v[0] * inv) | ((uint32_t)f_to_e4m3_sat(v[1] * inv) << 8) |
                   ((uint32_t)f_to_e4m3_sat(v[2] * inv) << 16) | ((uint32_t)f_to_e4m3_sat(v[3] * inv) << 24);
      *reinterpret_cast<uint32_t*>(dst + c0) = w;
    } else {
      store_act4(dst + dn, CSA_FMT_BF16, c0 - dn, v);
    }
  }
  if (writes_scale && threadIdx.x == 0) {
    *reinterpret_cast<float*>(dst + L.D + 64) = sig;
    *reinterpret_cast<uint32_t*>(dst + L.D + 68) = 0u;
    *reinterpret_cast<uint2*>(dst + L.D + 72) = make_uint2(0u, 0u);
  }
}

__device__ __forceinline__ float local_amax(const float v[4], int c0, int dn, bool active) {
  return (active && c0 < dn) ? fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))) : 0.f;
}

// One token per cluster of CL CTAs; CTA rank q owns channels [q*D/CL, (q+1)*D/CL).  Inside a CTA:
// (D/CL/4) channel threads x RG row groups.  Row group 0 appends the token (its window row); every
// row group pools a strided subset of the completed entry's source rows with an online softmax;
// groups merge through shared memory and the row-wide RMSNorm sum and FP8 amax are reduced over
// the cluster.  With CL = 1 (chunked prefill) the cluster reductions are plain block reductions.
__global__ void __launch_bounds__(256) append_compress_kernel(const __grid_constant__ AppendCompressArgs a, int CL) {
  __shared__ float scratch[64];
  __shared__ ClusterMail mail;
  extern __shared__ float part[];                  // [RG][3][DC]
  cg::cluster_group cluster = cg::this_cluster();
  const LayerArgs& L = a.L;
  const CacheArgs& C = a.C;
  const int q = (int)cluster.block_rank();
  const int j = blockIdx.x / CL, b = blockIdx.y;
  const int DC = L.D / CL;                         // channels of this CTA
  const int CT = DC / 4;                           // channel threads per row group
  const int RG = blockDim.x / CT;
  const int ct = threadIdx.x % CT, rg = threadIdx.x / CT;
  const int c0 = q * DC + ct * 4;                  // first channel of this thread (row-wide index)
  const bool lead = rg == 0;
  const int dn = L.D - L.d_rope;
  CTRACE(0);
  // mailboxes: each expects CL partials of 8 bytes; the cluster barrier's first phase (arrived now,
  // awaited before the first send) makes every CTA's initialisation visible to its peers
  if (threadIdx.x == 0) {
    sm100::mbar_init(&mail.bar[0], 1);
    sm100::mbar_init(&mail.bar[1], 1);
    sm100::mbar_arrive_expect_tx(&mail.bar[0], 8u * (uint32_t)CL);
    sm100::mbar_arrive_expect_tx(&mail.bar[1], 8u * (uint32_t)CL);
    sm100::fence_barrier_init();
  }
  cluster_arrive_relaxed();
  bool mail_open = false, done_mail = false;       // uniform over the cluster
  const int64_t t = a.q_pos[(int64_t)b * a.Tq + j];
  const int64_t r = t - L.pos0;
  const bool valid = r >= 0;                       // uniform over the cluster
  const size_t arow = (size_t)L.D * act_bytes(L.act_fmt);
  const bool have_new = a.x_new != nullptr;
  float x[4] = {0.f, 0.f, 0.f, 0.f}, g[4] = {0.f, 0.f, 0.f, 0.f};
  if (valid) {
    if (have_new) {
      load_act4(a.x_new + ((size_t)b * a.Tq + j) * arow, L.act_fmt, c0, x);
      load_act4(a.g_new + ((size_t)b * a.Tq + j) * arow, L.act_fmt, c0, g);
    } else if (a.do_append) {
      const int64_t s = ring_slot(r, C.raw_base, C.raw_cap);
      load_act4(C.raw + ((size_t)b * C.raw_cap + s) * arow, L.act_fmt, c0, x);
    }
  }
  CTRACE(1);
  const bool compress = valid && a.do_compress && ((r + 1) % L.m) == 0;
  // issued now, used after the pooling
  const float4 gk = (compress && a.gamma_kv) ? __ldg(reinterpret_cast<const float4*>(a.gamma_kv + c0))
                                             : make_float4(1.f, 1.f, 1.f, 1.f);

  if (valid && a.do_append) {
    if (have_new && lead) {
      const int64_t s = ring_slot(r, C.raw_base, C.raw_cap);
      store_act4(C.raw + ((size_t)b * C.raw_cap + s) * arow, L.act_fmt, c0, x);
      store_act4(C.gate + ((size_t)b * C.raw_cap + s) * arow, L.act_fmt, c0, g);
    }
    float w[4] = {x[0], x[1], x[2], x[3]};
    rope4(w, c0, L, (double)t);
    float am = 0.f;
    if (L.kv_fmt == CSA_FMT_MIXED) {
      const float bm = block_max(local_amax(w, c0, dn, lead), scratch);
      if (!mail_open) { cluster_wait(); mail_open = true; }
      mail_send(&mail, 0, q, CL, make_float2(0.f, bm));
      am = mail_reduce(&mail, 0, CL, a.err).y;
      if (!compress) { cluster_arrive_relaxed(); done_mail = true; }   // this CTA's mail is all in
    }
    uint8_t* dst = C.window + ((size_t)b * C.window_cap + (size_t)(r % C.window_cap)) * L.row_bytes;
    pack_slice(dst, L, c0, w, lead, am, q == 0);
  }
  CTRACE(2);
  CTRACE(3);
  CTRACE_C(10);

  if (compress) {
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
      // 1) issue every load of the batch (rows past r re-read a valid row and are masked below)
      float xv[kRowBatch][4], zv[kRowBatch][4];
      float4 bias[kRowBatch];
      int64_t slots[kRowBatch];
#pragma unroll
      for (int u = 0; u < kRowBatch; ++u) {
        slots[u] = slot;
        slot += slot_step;
        if (slot >= C.raw_cap) slot -= C.raw_cap;
      }
#pragma unroll
      for (int u = 0; u < kRowBatch; ++u) {
        const int64_t rr = rb + (int64_t)u * rstep;
        const int64_t sl = rr <= r ? slots[u] : slots[0];
        load_act4(C.raw + ((size_t)b * C.raw_cap + sl) * arow, L.act_fmt, c0, xv[u]);
        load_act4(C.gate + ((size_t)b * C.raw_cap + sl) * arow, L.act_fmt, c0, zv[u]);
        const int64_t br = (rr <= r ? rr : rb) - lo;
        bias[u] = __ldg(reinterpret_cast<const float4*>(a.pos_bias + (size_t)br * L.D + c0));
      }
      // 2) logits in base 2, masked rows, the just-appended row from registers
#pragma unroll
      for (int u = 0; u < kRowBatch; ++u) {
        const int64_t rr = rb + (int64_t)u * rstep;
        if (rr == r && have_new) {
#pragma unroll
          for (int k = 0; k < 4; ++k) { xv[u][k] = x[k]; zv[u][k] = g[k]; }
        }
        if (rr <= r) {
          zv[u][0] = (zv[u][0] + bias[u].x) * kLog2e; zv[u][1] = (zv[u][1] + bias[u].y) * kLog2e;
          zv[u][2] = (zv[u][2] + bias[u].z) * kLog2e; zv[u][3] = (zv[u][3] + bias[u].w) * kLog2e;
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) { xv[u][k] = 0.f; zv[u][k] = -INFINITY; }
        }
      }
      // 3) batch max, one rescale, exp2 per element
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
    CTRACE(4);
    CTRACE_C(11);
    // merge the row groups
    if (RG >= 4) {
      // two levels over all threads: thread (channel c, slice j) merges groups j, j+J, ..., then
      // the lead threads merge the J slices of their channels (max first, then independent exp2)
      float* pm = part + (size_t)rg * 3 * DC;
      const int cl0 = ct * 4;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        pm[cl0 + k] = mx[k];
        pm[DC + cl0 + k] = sum[k];
        pm[2 * DC + cl0 + k] = acc[k];
      }
      __syncthreads();
      CTRACE_C(14);
      // (every slice holds exactly 4 row groups, RG = 4 J; each level issues all of its shared-
      // memory loads before any arithmetic, so their latencies overlap)
      const int J = (int)blockDim.x / DC;            // = RG / 4 slices per channel
      const int c = threadIdx.x % DC, jj = threadIdx.x / DC;
      float m4[4], s4[4], a4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float* po = part + (size_t)(jj + u * J) * 3 * DC;
        m4[u] = po[c];
        s4[u] = po[DC + c];
        a4[u] = po[2 * DC + c];
      }
      const float M = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      float sm = 0.f, ac = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float f = m4[u] == -INFINITY ? 0.f : exp2f(m4[u] - M);
        sm += s4[u] * f;
        ac += a4[u] * f;
      }
      __syncthreads();
      float* p1 = part + (size_t)jj * 3 * DC;
      p1[c] = M;
      p1[DC + c] = sm;
      p1[2 * DC + c] = ac;
      __syncthreads();
      // level 2: one thread per channel merges the J slices; the result goes to the slot after the
      // slices (RG = 4 J > J), where the lead threads pick up their 4 channels
      float* pf = part + (size_t)J * 3 * DC;
      if ((int)threadIdx.x < DC) {
        constexpr int kMaxJ = 8;                     // RG <= 32
        const int cc = threadIdx.x;
        float mj[kMaxJ], sj[kMaxJ], aj[kMaxJ];
#pragma unroll
        for (int q2 = 0; q2 < kMaxJ; ++q2) {
          mj[q2] = -INFINITY; sj[q2] = 0.f; aj[q2] = 0.f;
          if (q2 < J) {
            const float* po = part + (size_t)q2 * 3 * DC;
            mj[q2] = po[cc];
            sj[q2] = po[DC + cc];
            aj[q2] = po[2 * DC + cc];
          }
        }
        float M2 = mj[0];
#pragma unroll
        for (int q2 = 1; q2 < kMaxJ; ++q2) M2 = fmaxf(M2, mj[q2]);
        float s2 = 0.f, a2 = 0.f;
#pragma unroll
        for (int q2 = 0; q2 < kMaxJ; ++q2) {
          const float f = mj[q2] == -INFINITY ? 0.f : exp2f(mj[q2] - M2);
          s2 += sj[q2] * f;
          a2 += aj[q2] * f;
        }
        pf[cc] = M2;
        pf[DC + cc] = s2;
        pf[2 * DC + cc] = a2;
      }
      __syncthreads();
      if (lead) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          mx[k] = pf[cl0 + k];
          sum[k] = pf[DC + cl0 + k];
          acc[k] = pf[2 * DC + cl0 + k];
        }
      }
    } else if (RG > 1) {
      float* pm = part + (size_t)rg * 3 * DC;
      const int cl0 = ct * 4;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        pm[cl0 + k] = mx[k];
        pm[DC + cl0 + k] = sum[k];
        pm[2 * DC + cl0 + k] = acc[k];
      }
      __syncthreads();
      if (lead) {
        // max over the groups first, then independent exp2 terms (no serial rescale chain)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float M = mx[k];
          for (int qq = 1; qq < RG; ++qq) M = fmaxf(M, part[(size_t)qq * 3 * DC + cl0 + k]);
          float sm = sum[k] * exp2f(mx[k] - M), ac = acc[k] * exp2f(mx[k] - M);
          for (int qq = 1; qq < RG; ++qq) {
            const float* po = part + (size_t)qq * 3 * DC;
            const float m2 = po[cl0 + k];
            const float f = m2 == -INFINITY ? 0.f : exp2f(m2 - M);
            sm += po[DC + cl0 + k] * f;
            ac += po[2 * DC + cl0 + k] * f;
          }
          sum[k] = sm;
          acc[k] = ac;
          mx[k] = M;
        }
      }
    }
    CTRACE(5);
    CTRACE_C(12);
    float e[4] = {0.f, 0.f, 0.f, 0.f};
    float ss = 0.f, eg = 0.f;
    if (lead) {
#pragma unroll
      for (int k = 0; k < 4; ++k) { e[k] = acc[k] / sum[k]; ss += e[k] * e[k]; }
      // FP8 dims are not rotated and rs > 0: max |e * rs * gamma| = rs * max |e * gamma|, so the
      // scale's amax rides on the same cluster reduction as the RMSNorm sum
      if (c0 < dn)
        eg = fmaxf(fmaxf(fabsf(e[0] * gk.x), fabsf(e[1] * gk.y)), fmaxf(fabsf(e[2] * gk.z), fabsf(e[3] * gk.w)));
    }
    const float2 bl = block_sum_max(ss, eg, scratch);
    if (!mail_open) { cluster_wait(); mail_open = true; }
    mail_send(&mail, 1, q, CL, bl);
    const float2 red2 = mail_reduce(&mail, 1, CL, a.err);
    cluster_arrive_relaxed();                      // this CTA's mail is all in
    done_mail = true;
    const float rs = 1.0f / sqrtf(red2.x / (float)L.D + L.eps);
    e[0] *= rs * gk.x; e[1] *= rs * gk.y; e[2] *= rs * gk.z; e[3] *= rs * gk.w;
    CTRACE(6);
    CTRACE_C(13);
    rope4(e, c0, L, (double)(L.pos0 + i * (int64_t)L.m));
    CTRACE(7);
    const float am = L.kv_fmt == CSA_FMT_MIXED ? red2.y * rs : 0.f;
    uint8_t* dst = C.entries + ((size_t)b * C.entry_cap + (size_t)i) * L.row_bytes;
    pack_slice(dst, L, c0, e, lead, am, q == 0);
    CTRACE(8);
    CTRACE_C(15);
  }
  // second phase of the cluster barrier: no CTA leaves before every CTA has received its mail
  if (!mail_open) cluster_wait();
  if (!done_mail) cluster_arrive_relaxed();
  cluster_wait();
}

}  // namespace

#ifdef CSA_TRACE
extern "C" __attribute__((visibility("default"))) int csa_trace_read_c(uint64_t* host) {
  return (int)cudaMemcpyFromSymbol(host, g_trace_c, sizeof(g_trace_c));
}
#endif

cudaError_t library_error_word(int** p) {
  static std::mutex mu;
  static int* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* q = nullptr;
    e = cudaGetSymbolAddress(&q, g_library_error);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<int*>(q);
  }
  *p = addr[dev];
  return cudaSuccess;
}

cudaError_t launch_append_compress(const AppendCompressArgs& a, int B, int Tq, cudaStream_t s) {
  // decode (few tokens): a cluster of CL CTAs per token splits the channels, and row groups split
  // the entry's source rows; a chunk has parallelism across tokens and runs one CTA per token.
  // A long pooling window (HCA's m' = 128 rows) takes a 16-CTA cluster (32 channels per CTA, up to
  // 32 row groups): twice the SMs issue its row loads; short windows keep 8 CTAs of 64 channels.
  const bool spread = Tq <= 64;
  const int rows = (1 + a.L.ov) * a.L.m;
  const bool wide = spread && a.do_compress && rows >= 64 && a.L.D >= 512;
  int CL = 1;
  if (spread) {
    CL = wide ? a.L.D / 32 : a.L.D / 64;
    const int cmax = wide ? 16 : 8;
    if (CL > cmax) CL = cmax;
    if (CL < 1) CL = 1;
  }
  const int ct = a.L.D / CL / 4;
  int rg = 1;
  if (spread && a.do_compress) {
    const int rg_max = wide ? 32 : 16;
    rg = rows < rg_max ? rows : rg_max;
    while (rg > 1 && ct * rg > 256) rg >>= 1;
  }
  if (CL > 8) {
    cudaError_t e = ensure_nonportable_cluster(reinterpret_cast<const void*>(append_compress_kernel));
    if (e != cudaSuccess) return e;
  }
  const size_t smem = rg > 1 ? (size_t)rg * 3 * (a.L.D / CL) * sizeof(float) : 0;
  {
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(append_compress_kernel), smem);
    if (e != cudaSuccess) return e;
  }
  return launch_kernel(append_compress_kernel, dim3((unsigned)(Tq * CL), (unsigned)B), dim3((unsigned)(ct * rg)), smem, s,
                    CL, a, CL);
}

}  // namespace csa
