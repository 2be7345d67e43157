// saga_noalloc.cu - saga_decode_attn without a caller-provided workspace.
//
// For callers that cannot allocate device memory around a decode call: code
// whose device memory is owned by another allocator (a serving engine that
// reserves HBM up front and hands out fixed buffers), or code that must not
// call cudaMalloc at that point (for example while another thread captures
// a CUDA graph on the same device, where an allocation would break the
// capture).  The scratch lives in a fixed array of this library's device
// image instead.
#include <cuda_runtime.h>
#include <stdio.h>

#include <mutex>

#include "saga.h"

namespace {

// Scratch shared by every saga_decode_attn_noalloc call on a device.  It is
// part of the library's device image: every device that loads the library
// holds these bytes until the process exits.
constexpr size_t kScratchBytes = SAGA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

thread_local char g_noalloc_err[256] = "";

struct DeviceScratch {
  void* ptr = nullptr;
  bool ready = false;
};
DeviceScratch g_scratch[128];
std::mutex g_scratch_mu;

// Device address of the scratch array for the current device.  In host code
// the array's name only stands for the symbol, so the address comes from
// cudaGetSymbolAddress, once per device, with that device current.
int scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    snprintf(g_noalloc_err, sizeof(g_noalloc_err), "cudaGetDevice: %s", cudaGetErrorString(e));
    return SAGA_ERR_CUDA;
  }
  if (dev < 0 || dev >= 128) {
    snprintf(g_noalloc_err, sizeof(g_noalloc_err), "device ordinal %d out of range", dev);
    return SAGA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch[dev].ready) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
      snprintf(g_noalloc_err, sizeof(g_noalloc_err), "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
      return SAGA_ERR_CUDA;
    }
    g_scratch[dev].ptr = ptr;
    g_scratch[dev].ready = true;
  }
  *out = g_scratch[dev].ptr;
  return SAGA_OK;
}

}  // namespace

extern "C" {

size_t saga_noalloc_scratch_bytes(void) { return kScratchBytes; }

int saga_decode_attn_noalloc(const saga_shape* s, const void* q, const void* k_cache, const void* v_cache,
                             int seq_len, const int* seq_len_dev, int n_top, int refresh_interval, long long step,
                             float* tau, void* out, int out_dtype, int* sel_count, int* sel_idx, void* stream) {
  g_noalloc_err[0] = '\0';
  const size_t need = saga_workspace_bytes(s);
  if (need == 0) return saga_decode_attn(s, q, k_cache, v_cache, seq_len, seq_len_dev, n_top, refresh_interval, step,
                                         tau, out, out_dtype, sel_count, sel_idx, nullptr, 0, stream);
  if (need > kScratchBytes) {
    snprintf(g_noalloc_err, sizeof(g_noalloc_err),
             "saga_decode_attn_noalloc: this shape needs %zu bytes of scratch, the built-in scratch holds %zu; "
             "use saga_decode_attn with a workspace",
             need, kScratchBytes);
    return SAGA_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  int rc = scratch_for_current_device(&scratch);
  if (rc != SAGA_OK) return rc;
  // the status word is the only part a call reads before writing it
  cudaError_t e = cudaMemsetAsync(scratch, 0, 16, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    snprintf(g_noalloc_err, sizeof(g_noalloc_err), "cudaMemsetAsync(status): %s", cudaGetErrorString(e));
    return SAGA_ERR_CUDA;
  }
  return saga_decode_attn(s, q, k_cache, v_cache, seq_len, seq_len_dev, n_top, refresh_interval, step, tau, out,
                          out_dtype, sel_count, sel_idx, scratch, kScratchBytes, stream);
}

const char* saga_noalloc_last_error(void) {
  return g_noalloc_err[0] != '\0' ? g_noalloc_err : saga_last_error();
}

}  // extern "C"
