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

namespace saga {
int decode_attn_clearing_status(const saga_shape* s, const void* q, const void* k_cache, const void* v_cache,
                                int seq_len, const int* seq_len_dev, int n_top, int refresh_interval, long long step,
                                float* tau, void* out, int out_dtype, int* sel_count, int* sel_idx, void* workspace,
                                size_t ws_bytes, void* stream);
}

namespace {

// Scratch shared by every saga_decode_attn_noalloc call on a device.  It is
// part of the library's device image: every device that loads the library
// holds these bytes until the process exits.  Its first 16 bytes hold the
// status word (SAGA_STATUS_* bits), as at the start of a workspace.
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
// cudaGetSymbolAddress, with that device current.  It is looked up again on
// every call made outside stream capture (a cheap host query once the module
// is loaded, and correct after a cudaDeviceReset has recreated the context);
// during capture the address cached by an earlier call is used, so the first
// call on a device must come before any capture.
int scratch_for_current_device(cudaStream_t stream, void** out) {
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
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(stream, &cs);
  if (e != cudaSuccess) {
    snprintf(g_noalloc_err, sizeof(g_noalloc_err), "cudaStreamIsCapturing: %s", cudaGetErrorString(e));
    return SAGA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (cs == cudaStreamCaptureStatusNone || !g_scratch[dev].ready) {
    if (cs != cudaStreamCaptureStatusNone) {
      snprintf(g_noalloc_err, sizeof(g_noalloc_err),
               "saga_decode_attn_noalloc: first call on device %d made during stream capture; call it once before "
               "capturing",
               dev);
      return SAGA_ERR_CUDA;
    }
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
  if (need == 0)  // invalid shape: saga_decode_attn reports why, enqueueing nothing
    return saga_decode_attn(s, q, k_cache, v_cache, seq_len, seq_len_dev, n_top, refresh_interval, step, tau, out,
                            out_dtype, sel_count, sel_idx, nullptr, 0, stream);
  if (need > kScratchBytes) {
    snprintf(g_noalloc_err, sizeof(g_noalloc_err),
             "saga_decode_attn_noalloc: this shape needs %zu bytes of scratch, the built-in scratch holds %zu; "
             "use saga_decode_attn with a workspace",
             need, kScratchBytes);
    return SAGA_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  int rc = scratch_for_current_device(static_cast<cudaStream_t>(stream), &scratch);
  if (rc != SAGA_OK) return rc;
  // every argument is checked before anything is enqueued; the status word
  // (the only part of the scratch a call reads before writing it) is then
  // cleared on the stream ahead of the kernels
  return saga::decode_attn_clearing_status(s, q, k_cache, v_cache, seq_len, seq_len_dev, n_top, refresh_interval, step,
                                           tau, out, out_dtype, sel_count, sel_idx, scratch, kScratchBytes, stream);
}

int saga_noalloc_get_status(void* stream, unsigned* status) {
  g_noalloc_err[0] = '\0';
  if (status == nullptr) {
    snprintf(g_noalloc_err, sizeof(g_noalloc_err), "status is NULL");
    return SAGA_ERR_ARG;
  }
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(status, g_noalloc_scratch, sizeof(unsigned), 0, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) {
    snprintf(g_noalloc_err, sizeof(g_noalloc_err), "saga_noalloc_get_status: %s", cudaGetErrorString(e));
    return SAGA_ERR_CUDA;
  }
  return SAGA_OK;
}

const char* saga_noalloc_last_error(void) {
  return g_noalloc_err[0] != '\0' ? g_noalloc_err : saga_last_error();
}

}  // extern "C"
