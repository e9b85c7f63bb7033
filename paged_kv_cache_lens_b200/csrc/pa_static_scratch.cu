// pa_decode_static: paged decode attention for callers that cannot allocate
// device memory.
//
// pa_decode needs a caller-supplied workspace for the split-K partials (a
// running max, a running sum and an unnormalised output per partition).  Some
// callers have no way to obtain one at the point where they run attention:
// a plug-in living inside a host program that owns all device memory and
// gives the plug-in no allocator, or a latency-critical loop in which
// cudaMalloc (which may synchronise the whole device) is not acceptable.
// This entry point serves them: its scratch is a file-scope device array of
// fixed size, so the call itself allocates nothing.
//
// The array (PA_DECODE_STATIC_SCRATCH_BYTES, 32 MiB) exists once on every GPU
// that loads this library and stays allocated until the process exits.  In
// host code the array's name only denotes a host-side stand-in, not a device
// address, so the first call on each device, with that device current, looks
// up its device address with cudaGetSymbolAddress and remembers it; that
// first call should therefore come before any stream capture.  Every call on
// a device shares the one array: calls whose executions overlap on the GPU
// (different streams, or different host threads) race on it and must be
// serialised by the caller.  The kernel writes every partial it later reads,
// so nothing has to be cleared between calls.
#include "pa.h"

#include <cuda_runtime.h>

#include <mutex>

namespace {

constexpr size_t kScratchBytes = PA_DECODE_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kScratchBytes];

void* g_scratch_addr[kMaxDevices];
cudaError_t g_scratch_status[kMaxDevices];
std::once_flag g_scratch_once[kMaxDevices];

}  // namespace

extern "C" pa_status pa_decode_static(void* out, pa_dtype out_dtype, const void* q,
                                      pa_dtype q_dtype, int32_t batch, int32_t num_q_heads,
                                      const void* k_cache, const void* v_cache,
                                      const pa_cache_desc* cache, const int32_t* block_tables,
                                      int32_t max_blocks_per_seq, const int32_t* context_lens,
                                      int32_t max_context_len, float scale,
                                      int32_t partition_size, void* stream) {
  if (!cache) return PA_ERR_INVALID_ARG;
  const size_t need = pa_decode_workspace_size(batch, num_q_heads, cache->head_dim,
                                               max_context_len, partition_size);
  if (need > kScratchBytes) return PA_ERR_WORKSPACE;   // the fixed scratch is too small
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
  std::call_once(g_scratch_once[dev], [dev] {
    g_scratch_status[dev] = cudaGetSymbolAddress(&g_scratch_addr[dev], g_static_scratch);
  });
  if (g_scratch_status[dev] != cudaSuccess || !g_scratch_addr[dev]) return PA_ERR_CUDA;
  return pa_decode(out, out_dtype, q, q_dtype, batch, num_q_heads, k_cache, v_cache, cache,
                   block_tables, max_blocks_per_seq, context_lens, max_context_len, scale,
                   partition_size, g_scratch_addr[dev], kScratchBytes, stream);
}
