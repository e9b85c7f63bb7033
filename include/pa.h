/*
 * libpa — paged KV-cache attention for NVIDIA B200 (sm_100a).
 *
 * A block-paged KV cache ("PagedAttention 与 Continuous Batching", §3.2-§3.3:
 * fixed 16-token physical blocks, one block table per request mapping logical
 * to physical blocks) and the three data-parallel steps that touch it:
 *
 *   pa_reshape_and_cache  write this step's new K/V rows into their physical
 *                         slots (§3.3 decode steps 1-2; slot_mapping from §2.5
 *                         step 4).
 *   pa_decode             one query row per sequence attends its cached
 *                         context through the block table (§3.6 PagedAttention
 *                         Kernel), query heads of a GQA group sharing each KV
 *                         block, long contexts split into partitions merged by
 *                         a log-sum-exp reduce.
 *   pa_varlen             the packed mixed prefill/decode step: query rows of
 *                         all scheduled requests packed as [total_q, H, D],
 *                         cu_seqlens marking request boundaries ("推理优化与服务：
 *                         从 PagedAttention 到分离式部署", 最新进展 on the V1
 *                         unified step), causal within each request.
 *
 * Conventions for every entry point:
 *   - Pointers named as device pointers are CUDA device memory owned by the
 *     caller; the library allocates nothing, keeps no state between calls
 *     (apart from one device error word, see pa_device_error) and never
 *     synchronises the stream.  Work is enqueued on `stream` (a cudaStream_t;
 *     NULL is the legacy default stream) and the call returns.
 *   - Arguments are validated on the host before anything is enqueued; a
 *     failed check returns PA_ERR_INVALID_ARG / PA_ERR_UNSUPPORTED /
 *     PA_ERR_WORKSPACE and enqueues nothing.  A failed launch returns
 *     PA_ERR_CUDA.  No exception crosses this interface.
 *   - KV pool layout (a reading: the pages fix no axis order): k_cache and
 *     v_cache are [num_blocks][num_kv_heads][block_size][head_dim], row-major,
 *     so each (block, head) tile is one contiguous run.  Token t of a request
 *     with block table bt lives at slot bt[t / block_size] * block_size +
 *     t % block_size.
 *   - Block-table entries at or past ceil(len / block_size) are never read.
 *     Entries that are read and fall outside [0, num_blocks) are skipped
 *     (treated as masked) and recorded in the device error word.
 *   - GQA: query head hq reads KV head hq / (num_q_heads / num_kv_heads);
 *     num_q_heads is a multiple of num_kv_heads, the group at most 128 (MHA,
 *     GQA and MQA alike).
 *   - Attention accumulates in fp32; softmax is exact up to rounding.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PA_F16 = 0,        /* IEEE binary16 */
    PA_BF16 = 1,       /* bfloat16 */
    PA_FP8_E4M3 = 2,   /* OCP FP8 E4M3 (KV pool only), with per-head fp32 scales */
    PA_F32 = 3         /* IEEE binary32 (outputs only) */
} pa_dtype;

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned buffer */
    PA_ERR_UNSUPPORTED = 2,   /* dtype / head_dim / block_size / group size not built */
    PA_ERR_WORKSPACE = 3,     /* workspace smaller than the *_workspace_size figure */
    PA_ERR_OUT_OF_RANGE = 4,  /* a kernel met a block id or slot outside the pool, or a
                                 length above the max_context_len it was promised */
    PA_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed */
    PA_ERR_TIMEOUT = 6        /* a kernel's bounded wait for its own copies expired */
} pa_status;

/* Description of one layer's KV pool (a host struct; the scale pointers in it
 * are device pointers). */
typedef struct {
    int32_t num_blocks;     /* physical blocks in the pool */
    int32_t block_size;     /* tokens per block: 8, 16 or 32 */
    int32_t num_kv_heads;
    int32_t head_dim;       /* 64, 128 or 256, for every kv_dtype */
    pa_dtype kv_dtype;      /* PA_F16, PA_BF16 or PA_FP8_E4M3 */
    const float* k_scale;   /* [num_kv_heads] device fp32, FP8 only, else NULL */
    const float* v_scale;   /* [num_kv_heads] device fp32, FP8 only, else NULL */
} pa_cache_desc;

/*
 * Human-readable name of a status code (static storage, never NULL).
 */
const char* pa_status_string(pa_status status);

/*
 * Write new K/V rows into the paged pool ("PagedAttention 与 Continuous
 * Batching", §3.3: append each new token's K/V into the last block if it has
 * room, else into a freshly allocated block; the scheduler encodes the chosen
 * slot per token in slot_mapping, §2.5 step 4).
 *
 * key, value   : device, num_tokens rows; row i starts at element
 *                i * token_stride and holds [num_kv_heads][head_dim]
 *                contiguous elements of src_dtype (PA_F16 or PA_BF16).
 *                token_stride >= num_kv_heads * head_dim lets K/V sit inside
 *                a fused QKV buffer.  Both must be 16-byte aligned, and
 *                token_stride * element size a multiple of 16 bytes.
 * slot_mapping : device int64 [num_tokens]; slot = block * block_size +
 *                offset; a negative slot skips the token (padding).  Slots
 *                must be unique within one call (duplicates race).
 * k_cache, v_cache : device pools (layout above), written in place.
 * cache        : pool description.  kv_dtype == src_dtype copies the bits;
 *                PA_FP8_E4M3 stores e4m3(round-to-nearest-even, saturating)
 *                of x / k_scale[h] (resp. v_scale[h]), the quotient taken as
 *                an IEEE fp32 division.
 * A slot beyond the pool is skipped and recorded in the device error word.
 */
pa_status pa_reshape_and_cache(const void* key, const void* value, pa_dtype src_dtype,
                               int64_t num_tokens, int64_t token_stride,
                               const int64_t* slot_mapping, void* k_cache, void* v_cache,
                               const pa_cache_desc* cache, void* stream);

/*
 * Bytes of workspace pa_decode needs for these sizes (0 when no sequence can
 * span more than one partition).  partition_size as passed to pa_decode
 * (0 = automatic, which is what this function then assumes).
 */
size_t pa_decode_workspace_size(int32_t batch, int32_t num_q_heads, int32_t head_dim,
                                int32_t max_context_len, int32_t partition_size);

/*
 * Paged decode attention ("PagedAttention 与 Continuous Batching", §3.6): for
 * every sequence b and query head hq,
 *   out[b][hq] = sum_t softmax_t(scale * <q[b][hq], K_t>) V_t
 * over the context_lens[b] cached tokens of sequence b (the current token's
 * K/V already written by pa_reshape_and_cache), K_t/V_t fetched through
 * block_tables[b].  A sequence with context_lens[b] == 0 yields zeros.
 *
 * out          : device [batch][num_q_heads][head_dim] of out_dtype
 *                (PA_F16, PA_BF16 or PA_F32; rounded to nearest even).
 * q            : device [batch][num_q_heads][head_dim] of q_dtype.  With a
 *                16-bit pool q_dtype must equal the pool dtype; with an FP8
 *                pool it may be PA_BF16 or PA_F16 (|q| must stay below 65504,
 *                the products being taken in f16).
 * block_tables : device int32 [batch][max_blocks_per_seq].
 * context_lens : device int32 [batch], each in [0, max_context_len].
 * max_context_len: host upper bound of context_lens, used to size the grid
 *                and the workspace without reading device memory.  A row
 *                whose context_lens entry exceeds it is cut to its first
 *                max_context_len keys and reported in the device error word
 *                (PA_ERR_OUT_OF_RANGE from pa_device_error).
 * partition_size: tokens per split-K partition (a multiple of 64, or 0 for
 *                an automatic choice).  Sequences longer than one partition
 *                are split; partial results (running max, sum and
 *                unnormalised output per partition) are merged with the
 *                log-sum-exp rule in a second pass.
 * workspace    : device scratch of at least pa_decode_workspace_size(...)
 *                bytes, 256-byte aligned, contents irrelevant on entry.
 *                Concurrent calls must not share a workspace.
 */
pa_status pa_decode(void* out, pa_dtype out_dtype, const void* q, pa_dtype q_dtype,
                    int32_t batch, int32_t num_q_heads, const void* k_cache,
                    const void* v_cache, const pa_cache_desc* cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* context_lens, int32_t max_context_len, float scale,
                    int32_t partition_size, void* workspace, size_t workspace_bytes,
                    void* stream);

/*
 * Optional attention variants ("PagedAttention 与 Continuous Batching", §10.8
 * FAQ: paged kernels must also cover sliding window and ALiBi).  A zeroed
 * struct (or a NULL pointer) means plain attention.
 */
typedef struct {
    int32_t window;              /* > 0: a query at absolute position p sees only
                                    keys p - window + 1 .. p; <= 0: no window */
    const float* alibi_slopes;   /* NULL, or device fp32 [num_q_heads]: adds
                                    slope[hq] * (key position - query position)
                                    to the scaled logit (a non-positive bias) */
} pa_attn_options;

/*
 * pa_decode with options (NULL = pa_decode).
 */
pa_status pa_decode_ex(void* out, pa_dtype out_dtype, const void* q, pa_dtype q_dtype,
                       int32_t batch, int32_t num_q_heads, const void* k_cache,
                       const void* v_cache, const pa_cache_desc* cache,
                       const int32_t* block_tables, int32_t max_blocks_per_seq,
                       const int32_t* context_lens, int32_t max_context_len, float scale,
                       int32_t partition_size, const pa_attn_options* options, void* workspace,
                       size_t workspace_bytes, void* stream);

/*
 * Bytes of workspace pa_varlen needs for these sizes, whichever kernels the
 * call ends up using (the worst case over both paths described below).
 */
size_t pa_varlen_workspace_size(int32_t num_seqs, int32_t total_q, int32_t num_q_heads,
                                int32_t head_dim, int32_t max_context_len);

/*
 * Infrastructure, not a step of the method: the workspace pa_varlen /
 * pa_varlen_ex need for these sizes and types, no more.  When the call's
 * prefill chunks run on the tensor-core chunk kernel (see pa_varlen) only
 * the q_len 1 requests use split-K partials, one work row per request, so
 * the partials are sized for num_seqs rows instead of total_q.  The figure
 * assumes an out pointer that is 16-byte aligned; a call whose out is not
 * needs pa_varlen_workspace_size bytes.  Returns 0 for invalid sizes.
 */
size_t pa_varlen_workspace_size_ex(int32_t num_seqs, int32_t total_q, int32_t num_q_heads,
                                   int32_t num_kv_heads, int32_t head_dim, int32_t max_q_len,
                                   int32_t max_context_len, pa_dtype q_dtype, pa_dtype kv_dtype);

/*
 * Packed mixed prefill/decode attention ("推理优化与服务：从 PagedAttention 到
 * 分离式部署", 最新进展: the unified step packs every scheduled query token
 * with cu_seqlens; "PagedAttention 与 Continuous Batching", §4.2: chunked
 * prefill shares a step with decodes).  Request r owns query rows
 * cu_seqlens_q[r] .. cu_seqlens_q[r+1]-1 (q_len_r rows) and seqlens_k[r] keys
 * (kv_len_r = cached + this step's new tokens, the new ones already written by
 * pa_reshape_and_cache).  Row i of request r sits at absolute position
 * kv_len_r - q_len_r + i and attends keys 0 .. kv_len_r - q_len_r + i
 * (causal mask aligned to the bottom right).  Rows with no visible key yield
 * zeros.  q_len 1 rows are decode rows; longer ones are prefill chunks.
 * Chunks run on the tensor-core chunk kernel when the GQA group is a power
 * of two up to 128, out is 16-byte aligned, and either the pool is bf16/f16
 * with head_dim 64, 128 or 256 and q of the pool's type, or the pool is
 * E4M3 with head_dim 128 and q f16 or bf16; otherwise every row runs on the
 * decode kernel.  Either way the result is the same attention.
 *
 * out, q       : device [total_q][num_q_heads][head_dim].
 * cu_seqlens_q : device int32 [num_seqs + 1], non-decreasing, cu[0] = 0,
 *                cu[num_seqs] = total_q.
 * seqlens_k    : device int32 [num_seqs], kv_len_r >= q_len_r.
 * max_q_len, max_context_len: host upper bounds of q_len_r and kv_len_r (a
 *                request whose kv_len_r exceeds max_context_len is cut there;
 *                rows run by the decode kernel also report it in the device
 *                error word, as for pa_decode, but a request of q_len_r >= 2
 *                taken by the chunk kernel is cut without a report).
 * block_tables : device int32 [num_seqs][max_blocks_per_seq].
 * workspace    : device scratch of at least pa_varlen_workspace_size(...)
 *                bytes (or pa_varlen_workspace_size_ex(...) for these exact
 *                types), 256-byte aligned; PA_ERR_WORKSPACE if smaller than
 *                what the path the call takes needs.
 */
pa_status pa_varlen(void* out, pa_dtype out_dtype, const void* q, pa_dtype q_dtype,
                    int32_t total_q, int32_t num_seqs, int32_t num_q_heads,
                    const int32_t* cu_seqlens_q, const int32_t* seqlens_k, int32_t max_q_len,
                    int32_t max_context_len, const void* k_cache, const void* v_cache,
                    const pa_cache_desc* cache, const int32_t* block_tables,
                    int32_t max_blocks_per_seq, float scale, void* workspace,
                    size_t workspace_bytes, void* stream);

/*
 * Size of the fixed device scratch behind pa_decode_static (per GPU).
 */
#define PA_DECODE_STATIC_SCRATCH_BYTES (32u * 1024u * 1024u)

/*
 * pa_decode without a workspace argument, for callers that cannot allocate
 * device memory (the pages describe no such call; it exists for this
 * library's users).  A plug-in inside a host program that owns all device
 * memory and exposes no allocator, or a latency-critical loop that cannot
 * afford cudaMalloc's implicit device synchronisation, still has to hand
 * pa_decode a workspace; this call instead keeps its split-K partials in a
 * file-scope device array of PA_DECODE_STATIC_SCRATCH_BYTES that every GPU
 * loading the library holds until the process exits.  It allocates nothing.
 *
 * Arguments and results are those of pa_decode minus the workspace.  Sizes
 * whose partials need more than PA_DECODE_STATIC_SCRATCH_BYTES (see
 * pa_decode_workspace_size) return PA_ERR_WORKSPACE without launching.
 * The first call in each CUDA context (normally once per device), made with
 * that device current, looks up the array's device address
 * (cudaGetSymbolAddress) and keeps it for that context; make that first call
 * before any stream capture.  A failed look-up returns PA_ERR_CUDA and is not
 * kept (the next call tries again); after a device reset the new context
 * looks the address up afresh.  All calls on one device share the array and
 * leave their partials in it: calls that overlap on the GPU (other streams,
 * other host threads) race and must be serialised by the caller.
 */
pa_status pa_decode_static(void* out, pa_dtype out_dtype, const void* q, pa_dtype q_dtype,
                           int32_t batch, int32_t num_q_heads, const void* k_cache,
                           const void* v_cache, const pa_cache_desc* cache,
                           const int32_t* block_tables, int32_t max_blocks_per_seq,
                           const int32_t* context_lens, int32_t max_context_len, float scale,
                           int32_t partition_size, void* stream);

/*
 * Copy whole blocks inside one pool, for copy-on-write ("PagedAttention 与
 * Continuous Batching", §3.8 COW 与引用计数: when a sequence must append into
 * a last block still referenced by other sequences, the block manager
 * allocates a new block, the shared block's contents are copied into it and
 * the sequence's table is redirected).
 *
 * k_cache, v_cache : device pools described by `cache`; block `dst` of both
 *                receives the contents of block `src` (all heads, all slots).
 * block_mapping: device int64 [num_pairs][2] = (src, dst) pairs.  A dst must
 *                not be another pair's src or dst (pairs run concurrently).
 *                A pair with an id outside [0, num_blocks) is skipped and
 *                recorded in the device error word.
 */
pa_status pa_copy_blocks(void* k_cache, void* v_cache, const pa_cache_desc* cache,
                         const int64_t* block_mapping, int64_t num_pairs, void* stream);

/*
 * Move whole blocks between two pools of the same geometry, typically the
 * device pool and a pinned host pool, for preemption by swapping ("PagedAttention
 * 与 Continuous Batching", §3.9 Swap 的 IO 代价): block dst of (dst_k, dst_v)
 * receives block src of (src_k, src_v).
 *
 * dst_k, dst_v, src_k, src_v : pool base addresses, device or pinned host
 *                memory (unified addressing decides the direction).
 * cache        : geometry (block_size, num_kv_heads, head_dim, kv_dtype);
 *                its num_blocks is ignored, the two pools' block counts are
 *                src_num_blocks and dst_num_blocks.
 * block_mapping: HOST int64 [num_pairs][2] = (src, dst); validated on the host
 *                (PA_ERR_INVALID_ARG for an id outside its pool).  Runs of
 *                consecutive pairs are merged into one copy each.
 */
pa_status pa_swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                         const pa_cache_desc* cache, int64_t src_num_blocks,
                         int64_t dst_num_blocks, const int64_t* block_mapping, int64_t num_pairs,
                         void* stream);

/*
 * pa_varlen with options (NULL = pa_varlen).
 */
pa_status pa_varlen_ex(void* out, pa_dtype out_dtype, const void* q, pa_dtype q_dtype,
                       int32_t total_q, int32_t num_seqs, int32_t num_q_heads,
                       const int32_t* cu_seqlens_q, const int32_t* seqlens_k, int32_t max_q_len,
                       int32_t max_context_len, const void* k_cache, const void* v_cache,
                       const pa_cache_desc* cache, const int32_t* block_tables,
                       int32_t max_blocks_per_seq, float scale, const pa_attn_options* options,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * Measurement helper, not part of the method (the pages have no counterpart):
 * stream `bytes` of device memory at `buf` once with read-only 16-byte loads,
 * the read-only bandwidth ceiling that the attention kernels' achieved GB/s
 * is reported beside (the roofline denominator itself is a measured copy).
 *
 * buf    : device memory, 16-byte aligned; bytes a multiple of 16 (0 allowed).
 * sink   : device uint32, 4-byte aligned; receives the XOR of all 32-bit
 *          words of the buffer (exact; a check that every byte was read).
 * Errors : PA_ERR_INVALID_ARG for misaligned or negative arguments,
 *          PA_ERR_CUDA if the launch fails.  Asynchronous on `stream`.
 */
pa_status pa_hbm_read_probe(const void* buf, int64_t bytes, void* sink, void* stream);

/*
 * Self-test of the failure path, not part of the method (the pages have no
 * counterpart): every wait inside this library's kernels is bounded, and a
 * wait that runs out records PA_ERR_TIMEOUT in the device error word and lets
 * its kernel return instead of hanging.  This call enqueues one small kernel
 * that waits, with a short limit (a few thousand polls), on a barrier that
 * nothing completes, so that the next pa_device_error returns
 * PA_ERR_TIMEOUT.  The CUDA context stays usable.  Asynchronous on `stream`;
 * PA_ERR_CUDA if the launch fails.
 */
pa_status pa_selftest_wait_timeout(void* stream);

/*
 * Read and clear the device error word that kernels set when they skip an
 * out-of-range block id or slot, or cut a row whose context_lens / seqlens_k
 * entry exceeds the max_context_len it was promised (PA_ERR_OUT_OF_RANGE; the
 * row's attention then covers its first max_context_len keys only; rows of a
 * pa_varlen chunk on the tensor-core path are cut without a report), or give
 * up a bounded wait (PA_ERR_TIMEOUT).  Synchronises `stream` first.  Returns PA_OK when no
 * kernel reported anything since the last call.
 */
pa_status pa_device_error(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
