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
  void* ws = nullptr;
  csa_status_t st = scratch_address(&ws);
  if (st != CSA_OK) return st;
  st = csa_decode_step(L, cache, P, q, idx_q, idx_q_scale, head_w, x_new, g_new, q_pos, out, topk_idx, ws,
                       kScratchBytes, stream);
  if (st != CSA_OK || !device_error) return st;
  // read back (and clear) the device error word; after an error, restore the all-zero scratch
  st = csa_device_error(ws, kScratchBytes, stream, device_error);
  if (*device_error != 0) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(ws, 0, kScratchBytes, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return csa::report_error(CSA_ERR_CUDA, cudaGetErrorString(e));
  }
  return st;
}
