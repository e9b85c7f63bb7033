// Read-only HBM bandwidth probe (sm_100a).
//
// The roofline the attention kernels are reported against is a copy (read +
// write); a read-mostly stream such as paged decode can run a little above
// it.  This kernel streams a buffer once with 16-byte non-allocating loads and
// nothing else, so its rate is the read-only ceiling on the same GPU.  The
// loads feed an XOR of all 32-bit words (order-independent, so the result is
// exact and checkable), reduced per CTA and merged with one atomicXor.
#include "pa_device.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

constexpr int kProbeThreads = 256;
constexpr int kProbeCtasPerSm = 8;    // 2048 threads per SM, 32 registers each
constexpr int kProbeUnroll = 4;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__global__ void __launch_bounds__(kProbeThreads, kProbeCtasPerSm)
hbm_read_probe_kernel(const uint4* __restrict__ p, int64_t n16, uint32_t* sink) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kProbeThreads;
  int64_t i = static_cast<int64_t>(blockIdx.x) * kProbeThreads + threadIdx.x;
  uint32_t acc = 0;
  // kProbeUnroll independent 16-byte loads in flight per thread
  for (; i + (kProbeUnroll - 1) * stride < n16; i += kProbeUnroll * stride) {
    uint4 v[kProbeUnroll];
#pragma unroll
    for (int u = 0; u < kProbeUnroll; ++u) v[u] = ld_stream(p + i + u * stride);
#pragma unroll
    for (int u = 0; u < kProbeUnroll; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = ld_stream(p + i);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  __shared__ uint32_t s_acc[kProbeThreads / 32];
  if ((threadIdx.x & 31) == 0) s_acc[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t x = 0;
    for (int w = 0; w < kProbeThreads / 32; ++w) x ^= s_acc[w];
    atomicXor(sink, x);
  }
}

}  // namespace

cudaError_t launch_hbm_read_probe(const void* buf, int64_t bytes, uint32_t* sink,
                                  cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(sink, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) return e;
  if (bytes == 0) return cudaSuccess;
  // every SM's full complement of threads, 4 x 16 B in flight per thread
  hbm_read_probe_kernel<<<static_cast<unsigned>(kProbeCtasPerSm * sms), kProbeThreads, 0,
                          stream>>>(
      static_cast<const uint4*>(buf), bytes / 16, sink);
  return cudaGetLastError();
}

}  // namespace pa
