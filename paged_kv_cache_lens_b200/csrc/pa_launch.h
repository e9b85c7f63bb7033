// Host-side launch descriptors shared by the C-ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace pa {

// Device error word codes (the first one reported wins until the host clears it).
enum : unsigned {
  kErrNone = 0,
  kErrBlockRange = 1,   // a block id read from a table lies outside the pool
  kErrSlotRange = 2,    // a slot lies outside the pool
  kErrTimeout = 3,      // a bounded wait gave up
  kErrLenRange = 4      // a row's key count exceeds max_context_len (cut there)
};

// Everything one attention launch needs; plain pointers and sizes.
struct AttnArgs {
  void* out;                    // [rows][Hq][D]
  const void* q;                // [rows][Hq][D]
  int out_dtype, q_dtype, kv_dtype;
  int32_t rows;                 // query rows (sequences for decode, total_q for varlen)
  int32_t num_q_heads, num_kv_heads, head_dim, group;
  int32_t head_chunks;          // decode: query heads of a group taken 8 at a time (>= 1)
  int32_t num_blocks, block_size;
  const int32_t* block_tables;  // [num_seqs][max_blocks_per_seq]
  int32_t max_blocks_per_seq;
  const int32_t* context_lens;  // decode: [rows]; varlen: nullptr
  const int32_t* row_seq;       // varlen: request of each row (workspace)
  const int32_t* row_len;       // varlen: visible keys of each row (workspace)
  const int32_t* cu_seqlens_q;  // varlen only
  const int32_t* seqlens_k;     // varlen only
  int32_t varlen_requests;      // varlen, chunk path on: row index = request, q_len 1 only
  const int2* pf_items;         // prefill work list (request, query tile)
  const int32_t* pf_count;      // number of valid items
  int32_t num_seqs;
  const float* k_scale;
  const float* v_scale;
  float scale;
  int32_t max_context_len;      // host bound; longer rows are clamped to it
  int32_t window;               // > 0: a query at position p sees keys p-window+1 .. p
  const float* alibi;           // [Hq] ALiBi slopes (bias slope * (key - p)) or nullptr
  int32_t partition_size;       // tokens per split-K partition
  int32_t max_parts;            // partitions of the longest row
  float* ws_m;                  // [rows][Hq][max_parts] running max (log2 domain)
  float* ws_l;                  // [rows][Hq][max_parts] running sum
  float* ws_o;                  // [rows][Hq][max_parts][D] unnormalised output
  const void* k_cache;
  const void* v_cache;
};

// Workspace carve-up (all offsets 256-byte aligned).
struct DecodeWorkspace {
  size_t m_off, l_off, o_off, total;
};

DecodeWorkspace decode_workspace_layout(int64_t rows, int32_t num_q_heads, int32_t head_dim,
                                        int32_t max_parts);

// Tensor maps over the pool viewed as [num_blocks*Hkv*block_size rows, D cols]
// with 128-byte boxes and the 128-byte swizzle.  Returns false on failure.
bool make_pool_tensor_map(CUtensorMap* map, const void* base, int kv_dtype, int64_t rows,
                          int32_t head_dim, int32_t box_rows);

cudaError_t launch_paged_attention(const AttnArgs& a, const CUtensorMap& kmap,
                                   const CUtensorMap& vmap, cudaStream_t stream);

// Request and visible-key count of each packed row.  With skip_chunks, rows
// of requests with q_len >= 2 get row_len = -1 (the prefill kernel owns them).
cudaError_t launch_varlen_prep(int32_t total_q, int32_t num_seqs, const int32_t* cu_seqlens_q,
                               const int32_t* seqlens_k, int32_t* row_seq, int32_t* row_len,
                               bool skip_chunks, cudaStream_t stream);

// Tensor-core prefill of the q_len >= 2 requests of a varlen step.
bool prefill_supported(int q_dtype, int kv_dtype, int32_t head_dim, int32_t group);
int prefill_query_tile(int32_t group);
int32_t prefill_item_capacity(int32_t num_seqs, int32_t total_q);
int prefill_tiles_per_item(int32_t head_dim);
// Builds the (request, pair of query tiles) list in a.pf_items / a.pf_count
// (heaviest first) and resets *unit_counter, then runs the persistent
// tensor-core prefill over it (one CTA per SM taking units through the counter).
cudaError_t launch_paged_prefill(const AttnArgs& a, const CUtensorMap& kmap,
                                 const CUtensorMap& vmap, const CUtensorMap& qmap,
                                 int32_t capacity, int32_t* unit_counter, cudaStream_t stream);

// 3-D tensor map over q [total_q][Hq][D] (16-bit), box {64, group, rows}.
bool make_q_tensor_map(CUtensorMap* map, const void* q, int64_t total_q, int32_t num_q_heads,
                       int32_t head_dim, int32_t group, int32_t rows);

cudaError_t launch_reshape_and_cache(const void* key, const void* value, int src_dtype,
                                     int64_t num_tokens, int64_t token_stride,
                                     const int64_t* slot_mapping, void* k_cache, void* v_cache,
                                     int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                                     int32_t head_dim, int kv_dtype, const float* k_scale,
                                     const float* v_scale, cudaStream_t stream);

bool attention_supported(int q_dtype, int kv_dtype, int32_t head_dim, int32_t group);

// (src, dst) block pairs passed by value to one launch (16 KiB of parameters).
constexpr int kMovePairs = 1024;
struct MovePairs {
  int64_t p[2 * kMovePairs];
};
// Whole-block moves between two device-accessible pools (device memory or
// mapped pinned host memory); the mapping is read on the host.
cudaError_t launch_move_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                               const int64_t* host_mapping, int64_t num_pairs,
                               int64_t block_bytes, cudaStream_t stream);
// Read-only HBM stream over `bytes` (a multiple of 16) at `buf` (16-byte
// aligned): *sink = XOR of all 32-bit words.
cudaError_t launch_hbm_read_probe(const void* buf, int64_t bytes, uint32_t* sink,
                                  cudaStream_t stream);
cudaError_t launch_copy_blocks(void* k_cache, void* v_cache, const int64_t* mapping,
                               int64_t num_pairs, int64_t block_bytes, int32_t num_blocks,
                               cudaStream_t stream);

unsigned int read_and_clear_error_word(cudaStream_t stream, cudaError_t* err);

// One CTA that waits, with a short poll limit, on an mbarrier nothing
// completes, then records kErrTimeout (the bounded-wait path, exercised).
cudaError_t launch_wait_timeout_selftest(cudaStream_t stream);

// Identity of the CUDA context current on the calling thread (cuCtxGetId:
// unique for the life of the process, so a context destroyed by a device
// reset and its successor differ); 0 when it cannot be had.
uint64_t current_context_id();

// cudaFuncSetAttribute(kernel, MaxDynamicSharedMemorySize, bytes), done once
// per (context, kernel): the setting belongs to the function in the current
// context and outlives the call.
cudaError_t ensure_smem_attribute(const void* kernel, int bytes);

}  // namespace pa
