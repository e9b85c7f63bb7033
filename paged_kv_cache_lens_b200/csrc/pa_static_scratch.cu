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
// address, so the first call in each CUDA context (one per device, unless the
// caller makes its own), with that device current, looks up its device
// address with cudaGetSymbolAddress, checks the result and remembers it for
// that context; that first call should therefore come before any stream
// capture.  Only a successful look-up is remembered: a failed one returns
// PA_ERR_CUDA and the next call tries again.  The remembered address is keyed
// by the context's process-unique id, so after a device reset (which ends the
// context the address belonged to) the next call looks the address up again
// in the new context.  Every call on a device shares the one array: calls
// whose executions overlap on the GPU (different streams, or different host
// threads) race on it and must be serialised by the caller.  The kernel writes
// every partial it later reads, so nothing has to be cleared between calls.
#include "pa.h"
#include "pa_launch.h"

#include <cuda_runtime.h>

#include <mutex>
#include <utility>
#include <vector>

namespace {

constexpr size_t kScratchBytes = PA_DECODE_STATIC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_static_scratch[kScratchBytes];

// (context id, device address of g_static_scratch in that context)
std::mutex g_scratch_mu;
std::vector<std::pair<uint64_t, void*>> g_scratch_addr;

// The array's device address in the current context, or null on failure.
void* scratch_address() {
  const uint64_t ctx = pa::current_context_id();
  if (ctx == 0) return nullptr;
  {
    std::lock_guard<std::mutex> g(g_scratch_mu);
    for (const auto& e : g_scratch_addr)
      if (e.first == ctx) return e.second;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) {
    (void)cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> g(g_scratch_mu);
  g_scratch_addr.emplace_back(ctx, p);
  return p;
}

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
  void* scratch = scratch_address();
  if (!scratch) return PA_ERR_CUDA;
  return pa_decode(out, out_dtype, q, q_dtype, batch, num_q_heads, k_cache, v_cache, cache,
                   block_tables, max_blocks_per_seq, context_lens, max_context_len, scale,
                   partition_size, scratch, kScratchBytes, stream);
}
