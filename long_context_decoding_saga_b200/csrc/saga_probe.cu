// saga_probe.cu - the pure-read ceiling of HBM on this device: one streaming
// read of a caller buffer with 16-byte loads, four in flight per thread, a
// grid of a whole number of CTAs per SM.  The attention kernels read keys and
// values and write almost nothing, so this is the roofline they are held to
// next to the copy bandwidth (which counts a read and a write per byte).
#include <cuda_runtime.h>
#include <stdint.h>

#include "saga.h"

namespace {

constexpr int kProbeThreads = 512;
constexpr int kProbeUnroll = 4;

// Each thread XORs what it reads into one word per CTA, so no load can be
// dropped; the sink is written once per CTA.
__global__ void __launch_bounds__(kProbeThreads) saga_read_probe_kernel(const uint4* __restrict__ src, size_t n16,
                                                                         unsigned* sink) {
  const size_t stride = (size_t)gridDim.x * kProbeThreads;
  uint32_t acc = 0;
  size_t i = (size_t)blockIdx.x * kProbeThreads + threadIdx.x;
  for (; i + (kProbeUnroll - 1) * stride < n16; i += kProbeUnroll * stride) {
    uint4 v[kProbeUnroll];
#pragma unroll
    for (int u = 0; u < kProbeUnroll; ++u) v[u] = __ldcs(src + i + u * stride);  // streaming: no reuse
#pragma unroll
    for (int u = 0; u < kProbeUnroll; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = __ldcs(src + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  __shared__ uint32_t wacc[kProbeThreads / 32];
  if ((threadIdx.x & 31) == 0) wacc[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t a = 0;
    for (int w = 0; w < kProbeThreads / 32; ++w) a ^= wacc[w];
    sink[blockIdx.x] = a;
  }
}

}  // namespace

extern "C" {

size_t saga_read_probe_sink_words(void) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return (size_t)sms * 4;  // up to four CTAs per SM
}

int saga_read_probe(const void* buf, size_t bytes, unsigned* sink, void* stream) {
  if (buf == nullptr || sink == nullptr || bytes < 16 || (reinterpret_cast<uintptr_t>(buf) & 15u) != 0)
    return SAGA_ERR_ARG;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return SAGA_ERR_CUDA;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, saga_read_probe_kernel, kProbeThreads, 0) != cudaSuccess)
    return SAGA_ERR_CUDA;
  per_sm = per_sm < 1 ? 1 : (per_sm > 4 ? 4 : per_sm);
  saga_read_probe_kernel<<<sms * per_sm, kProbeThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(buf), bytes / 16, sink);
  return cudaGetLastError() == cudaSuccess ? SAGA_OK : SAGA_ERR_CUDA;
}

}  // extern "C"
