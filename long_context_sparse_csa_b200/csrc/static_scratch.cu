// csa_decode_step_scratch: the fused CSA decode step with its workspace taken from a fixed device
// array compiled into the library, so that the call allocates nothing and needs no caller buffer.
// The pages have no counterpart: this is a convenience entry of the library's own.
//
// The array lives in static device memory (zero-initialised when the module loads, which is the
// zero-fill the workspace contract asks for; the kernels leave their counters and histograms at zero
// after every call).  Its address is looked up once per device with cudaGetSymbolAddress, on the
// first call made on that device.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "csa.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = CSA_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// After a device error the split top-k may leave its histograms and counters non-zero.  Run
// before every call: when the scratch's error word is set, zero those segments (the word itself is
// kept for the next call that reads it); otherwise return at once.
__global__ void __launch_bounds__(256) scratch_guard_kernel(const int* err, uint4* seg, size_t n16) {
  if (*reinterpret_cast<const volatile int*>(err) == 0) return;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (size_t)gridDim.x * blockDim.x)
    seg[i] = make_uint4(0u, 0u, 0u, 0u);
}

// Device address of g_scratch on the current device (looked up on the first call per device).
csa_status_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return csa::report_error(CSA_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return csa::report_error(CSA_ERR_INVALID_ARG, "device ordinal out of range");
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return csa::report_error(CSA_ERR_CUDA, cudaGetErrorString(e));
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return CSA_OK;
}

}  // namespace

extern "C" CSA_API csa_status_t csa_decode_step_scratch(const csa_layer_t* L, const csa_cache_t* cache,
                                                        const csa_params_t* P, const void* q, const void* idx_q,
                                                        const float* idx_q_scale, const float* head_w,
                                                        const void* x_new, const void* g_new, const int64_t* q_pos,
                                                        void* out, int32_t* topk_idx, int32_t* device_error,
                                                        void* stream) {
  if (!L || !cache) return csa::report_error(CSA_ERR_INVALID_ARG, "layer or cache is NULL");
  // size check first, on the host: an oversize call touches no device state
  const size_t need = csa_workspace_size(L, CSA_OP_DECODE_STEP, 1, cache->entry_cap);
  if (need == 0) return csa::report_error(CSA_ERR_INVALID_ARG, "invalid layer");
  if (need > kScratchBytes) {
    char msg[160];
    snprintf(msg, sizeof(msg), "decode step needs %zu workspace bytes > the %zu-byte static scratch", need,
             kScratchBytes);
    return csa::report_error(CSA_ERR_WORKSPACE, msg);
  }
  if (device_error) *device_error = 0;
  void* ws = nullptr;
  csa_status_t st = scratch_address(&ws);
  if (st != CSA_OK) return st;
  size_t err_off = 0, err_bytes = 0, seg_off = 0, seg_bytes = 0;
  st = csa_debug_workspace_segment(L, CSA_OP_DECODE_STEP, 1, cache->entry_cap, CSA_SEG_ERROR_WORD, &err_off,
                                   &err_bytes);
  if (st == CSA_OK)
    st = csa_debug_workspace_segment(L, CSA_OP_DECODE_STEP, 1, cache->entry_cap, CSA_SEG_TOPK_HISTOGRAM, &seg_off,
                                     &seg_bytes);
  if (st != CSA_OK) return st;
  if (seg_bytes > 0) {
    unsigned char* base = static_cast<unsigned char*>(ws);
    const int grid = (int)((seg_bytes / 16 + 255) / 256 < 64 ? (seg_bytes / 16 + 255) / 256 : 64);
    const cudaError_t e = csa::launch_kernel(scratch_guard_kernel, dim3(grid), dim3(256), 0,
                                             static_cast<cudaStream_t>(stream), 0,
                                             reinterpret_cast<const int*>(base + err_off),
                                             reinterpret_cast<uint4*>(base + seg_off), seg_bytes / 16);
    if (e != cudaSuccess) return csa::report_error(CSA_ERR_CUDA, cudaGetErrorString(e));
  }
  st = csa_decode_step(L, cache, P, q, idx_q, idx_q_scale, head_w, x_new, g_new, q_pos, out, topk_idx, ws,
                       kScratchBytes, stream);
  if (st != CSA_OK || !device_error) return st;
  // read back (and clear) the device error word; after an error, restore the all-zero scratch
  st = csa_device_error(ws, kScratchBytes, stream, device_error);
  if (st == CSA_ERR_DEVICE_TIMEOUT) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(ws, 0, kScratchBytes, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return csa::report_error(CSA_ERR_CUDA, cudaGetErrorString(e));
  }
  return st;
}

extern "C" CSA_API csa_status_t csa_debug_scratch_copy(size_t offset, void* buf, size_t bytes, int32_t to_scratch,
                                                       void* stream) {
  if (bytes == 0) return CSA_OK;
  if (!buf) return csa::report_error(CSA_ERR_INVALID_ARG, "buf is NULL");
  if (offset > kScratchBytes || bytes > kScratchBytes - offset)
    return csa::report_error(CSA_ERR_INVALID_ARG, "range outside the static scratch");
  void* ws = nullptr;
  csa_status_t st = scratch_address(&ws);
  if (st != CSA_OK) return st;
  unsigned char* p = static_cast<unsigned char*>(ws) + offset;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = to_scratch ? cudaMemcpyAsync(p, buf, bytes, cudaMemcpyDefault, s)
                             : cudaMemcpyAsync(buf, p, bytes, cudaMemcpyDefault, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return csa::report_error(CSA_ERR_CUDA, cudaGetErrorString(e));
  return CSA_OK;
}
