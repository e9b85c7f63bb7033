// Whole-block operations on the paged pool (sm_100a).
//
// copy_blocks: the device half of copy-on-write ("PagedAttention 与 Continuous
// Batching", §3.8 COW 与引用计数): when a sequence must append into a last
// block that other sequences still reference (ref_count > 1), the block
// manager allocates a fresh block, this kernel copies the shared block's K and
// V contents into it, and the sequence's table is redirected to the copy.
//
// swap_blocks: moving whole blocks between the device pool and a host pool
// for preemption by swapping (§3.9 Swap 的 IO 代价, §6.1): one asynchronous copy
// per run of consecutive blocks, bound by the host link, not by HBM.
//
// In the [num_blocks][num_kv_heads][block_size][head_dim] layout a block
// (all heads) is one contiguous run of Hkv*BS*D elements, so both are plain
// block-granular copies.
#include "pa_device.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

constexpr int kCopyThreads = 256;
constexpr int kCopyChunk = kCopyThreads * 16 * 4;   // bytes per CTA pass: 4 x 16 B per thread

// grid: (chunks of a block, pairs).  Each CTA moves one chunk of one block of
// both pools with 16-byte loads and stores.
__global__ void __launch_bounds__(kCopyThreads)
copy_blocks_kernel(uint8_t* k_cache, uint8_t* v_cache, const int64_t* __restrict__ mapping,
                   int64_t block_bytes, int32_t num_blocks) {
  const int64_t pair = blockIdx.y;
  const int64_t src = mapping[2 * pair];
  const int64_t dst = mapping[2 * pair + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report_error(kErrBlockRange);
    return;
  }
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kCopyChunk;
#pragma unroll
  for (int pool = 0; pool < 2; ++pool) {
    uint8_t* p = pool == 0 ? k_cache : v_cache;
    const uint4* s = reinterpret_cast<const uint4*>(p + src * block_bytes + base);
    uint4* d = reinterpret_cast<uint4*>(p + dst * block_bytes + base);
    const int64_t n16 = min(static_cast<int64_t>(kCopyChunk), block_bytes - base) / 16;
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = threadIdx.x + u * kCopyThreads;
      if (i < n16) v[u] = s[i];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = threadIdx.x + u * kCopyThreads;
      if (i < n16) d[i] = v[u];
    }
  }
}

// Gather/scatter of whole blocks between two pools that may live in device
// memory or in device-mapped pinned host memory: one CTA per pair and pool,
// 16-byte accesses; over the host link the many independent requests in
// flight keep it busy where one copy per scattered block would not.  The
// (src, dst) pairs travel by value in the kernel parameters (up to
// kMovePairs per launch), so the host-side mapping needs no device copy.
__global__ void __launch_bounds__(kCopyThreads)
move_blocks_kernel(uint8_t* dst_k, uint8_t* dst_v, const uint8_t* src_k, const uint8_t* src_v,
                   const __grid_constant__ MovePairs pairs, int64_t block_bytes) {
  const int pair = blockIdx.x >> 1;
  const bool v = blockIdx.x & 1;
  const int64_t src = pairs.p[2 * pair], dst = pairs.p[2 * pair + 1];
  const uint4* s = reinterpret_cast<const uint4*>((v ? src_v : src_k) + src * block_bytes);
  uint4* d = reinterpret_cast<uint4*>((v ? dst_v : dst_k) + dst * block_bytes);
  const int64_t n16 = block_bytes / 16;
  for (int64_t i = threadIdx.x; i < n16; i += 4 * kCopyThreads) {
    uint4 r[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (i + u * kCopyThreads < n16) r[u] = s[i + u * kCopyThreads];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (i + u * kCopyThreads < n16) d[i + u * kCopyThreads] = r[u];
  }
}

}  // namespace

cudaError_t launch_move_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                               const int64_t* host_mapping, int64_t num_pairs,
                               int64_t block_bytes, cudaStream_t stream) {
  for (int64_t s0 = 0; s0 < num_pairs; s0 += kMovePairs) {
    MovePairs mp;
    const int64_t n = min(static_cast<int64_t>(kMovePairs), num_pairs - s0);
    for (int64_t i = 0; i < 2 * n; ++i) mp.p[i] = host_mapping[2 * s0 + i];
    move_blocks_kernel<<<static_cast<unsigned>(2 * n), kCopyThreads, 0, stream>>>(
        static_cast<uint8_t*>(dst_k), static_cast<uint8_t*>(dst_v),
        static_cast<const uint8_t*>(src_k), static_cast<const uint8_t*>(src_v), mp, block_bytes);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_copy_blocks(void* k_cache, void* v_cache, const int64_t* mapping,
                               int64_t num_pairs, int64_t block_bytes, int32_t num_blocks,
                               cudaStream_t stream) {
  if (num_pairs <= 0) return cudaSuccess;
  if (num_pairs > 65535) {
    // more pairs than one grid dimension holds: launch in slices
    for (int64_t s = 0; s < num_pairs; s += 65535) {
      const int64_t n = min(static_cast<int64_t>(65535), num_pairs - s);
      cudaError_t e = launch_copy_blocks(k_cache, v_cache, mapping + 2 * s, n, block_bytes,
                                         num_blocks, stream);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  dim3 grid(static_cast<unsigned>((block_bytes + kCopyChunk - 1) / kCopyChunk),
            static_cast<unsigned>(num_pairs));
  copy_blocks_kernel<<<grid, kCopyThreads, 0, stream>>>(static_cast<uint8_t*>(k_cache),
                                                        static_cast<uint8_t*>(v_cache), mapping,
                                                        block_bytes, num_blocks);
  return cudaGetLastError();
}

}  // namespace pa
