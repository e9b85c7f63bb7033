// C ABI of libpa: argument validation, workspace sizing, tensor-map set-up and
// dispatch to the kernels.  See include/pa.h for the contract of every call.
#include "pa.h"
#include "pa_launch.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cstdio>
#include <cstdlib>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

namespace pa {

namespace {

constexpr int64_t kAlign = 256;

inline int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }
inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Automatic partition size: 512 tokens, halved (down to 128) while the
// launch would have fewer than ~2048 (row, head, partition) items, so short
// batches of long contexts still fill the 148 SMs.
int32_t auto_partition(int64_t rows, int32_t num_q_heads, int32_t max_context_len) {
  int32_t ps = 512;
  while (ps > 128 && rows * num_q_heads * cdiv(max_context_len, ps) < 2048) ps /= 2;
  return ps;
}

int32_t resolve_partition(int64_t rows, int32_t num_q_heads, int32_t max_context_len,
                          int32_t requested) {
  return requested > 0 ? requested : auto_partition(rows, num_q_heads, max_context_len);
}

bool valid_partition(int32_t ps) { return ps == 0 || (ps >= 64 && ps <= 1024 && ps % 64 == 0); }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once per process (the
// initialisation of a function-local static is thread-safe); null if absent.
EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(p);
    return nullptr;
  }();
  return fn;
}

template <class F>
F driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<F>(p);
  return nullptr;
}

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Encoded pool / query tensor maps, keyed by everything the encoding reads
// (base address, element type, extents, box): a hit returns the very bytes a
// fresh encode would.  A small round-robin table shared by all host threads.
struct MapKey {
  const void* base;
  int kind;            // 0: pool (esz in `a`), 1: q
  int64_t a, b, c, d, e;
  bool operator==(const MapKey& o) const {
    return base == o.base && kind == o.kind && a == o.a && b == o.b && c == o.c && d == o.d &&
           e == o.e;
  }
};
constexpr int kMapCacheSize = 32;
struct MapCache {
  std::mutex mu;
  MapKey key[kMapCacheSize];
  CUtensorMap map[kMapCacheSize];
  bool used[kMapCacheSize] = {};
  int next = 0;
};
MapCache& map_cache() {
  static MapCache c;
  return c;
}
bool map_lookup(const MapKey& k, CUtensorMap* out) {
  MapCache& c = map_cache();
  std::lock_guard<std::mutex> g(c.mu);
  for (int i = 0; i < kMapCacheSize; ++i)
    if (c.used[i] && c.key[i] == k) {
      *out = c.map[i];
      return true;
    }
  return false;
}
void map_store(const MapKey& k, const CUtensorMap& m) {
  MapCache& c = map_cache();
  std::lock_guard<std::mutex> g(c.mu);
  const int i = c.next;
  c.next = (c.next + 1) % kMapCacheSize;
  c.key[i] = k;
  c.map[i] = m;
  c.used[i] = true;
}

// With PA_DEBUG set in the environment, CUDA failures are described on stderr
// (the status code alone cannot carry the runtime's reason).
pa_status cuda_fail(cudaError_t e, const char* where) {
  if (std::getenv("PA_DEBUG"))
    std::fprintf(stderr, "libpa: %s: %s\n", where, cudaGetErrorString(e));
  return PA_ERR_CUDA;
}

pa_status map_fail(const char* which) {
  if (std::getenv("PA_DEBUG")) std::fprintf(stderr, "libpa: tensor map for %s failed\n", which);
  return PA_ERR_CUDA;
}

size_t elem_size(pa_dtype t) {
  switch (t) {
    case PA_F16: case PA_BF16: return 2;
    case PA_FP8_E4M3: return 1;
    case PA_F32: return 4;
  }
  return 0;
}

pa_status check_cache(const pa_cache_desc* c) {
  if (!c) return PA_ERR_INVALID_ARG;
  if (c->num_blocks <= 0 || c->num_kv_heads <= 0 || c->head_dim <= 0) return PA_ERR_INVALID_ARG;
  if (c->block_size != 8 && c->block_size != 16 && c->block_size != 32) return PA_ERR_UNSUPPORTED;
  if (c->kv_dtype != PA_F16 && c->kv_dtype != PA_BF16 && c->kv_dtype != PA_FP8_E4M3)
    return PA_ERR_UNSUPPORTED;
  if (c->kv_dtype == PA_FP8_E4M3 && (!c->k_scale || !c->v_scale)) return PA_ERR_INVALID_ARG;
  // TMA row coordinates are 32-bit
  if (static_cast<int64_t>(c->num_blocks) * c->num_kv_heads * c->block_size > INT_MAX)
    return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

}  // namespace

DecodeWorkspace decode_workspace_layout(int64_t rows, int32_t num_q_heads, int32_t head_dim,
                                        int32_t max_parts) {
  DecodeWorkspace w{0, 0, 0, 0};
  if (max_parts <= 1) return w;
  const int64_t n = rows * num_q_heads * max_parts;
  w.m_off = 0;
  w.l_off = align_up(n * 4, kAlign);
  w.o_off = w.l_off + align_up(n * 4, kAlign);
  w.total = w.o_off + align_up(n * head_dim * 4, kAlign);
  return w;
}

uint64_t current_context_id() {
  static const CtxGetCurrentFn get_cur = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_cur || !get_id) return 0;
  CUcontext c = nullptr;
  if (get_cur(&c) != CUDA_SUCCESS || !c) {
    // nothing current yet: the runtime makes the device's primary context
    // current when asked to use the device
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return 0;
    if (get_cur(&c) != CUDA_SUCCESS || !c) return 0;
  }
  unsigned long long id = 0;
  if (get_id(c, &id) != CUDA_SUCCESS) return 0;
  return static_cast<uint64_t>(id) + 1;   // 0 stays "unknown"
}

cudaError_t ensure_smem_attribute(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::vector<std::pair<uint64_t, const void*>> done;
  const uint64_t ctx = current_context_id();
  if (ctx) {
    std::lock_guard<std::mutex> g(mu);
    for (const auto& d : done)
      if (d.first == ctx && d.second == kernel) return cudaSuccess;
  }
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && ctx) {
    std::lock_guard<std::mutex> g(mu);
    done.emplace_back(ctx, kernel);
  }
  return e;
}

bool make_pool_tensor_map(CUtensorMap* map, const void* base, int kv_dtype, int64_t rows,
                          int32_t head_dim, int32_t box_rows) {
  const int esz = (kv_dtype == PA_FP8_E4M3) ? 1 : 2;
  const MapKey key{base, 0, esz, rows, head_dim, box_rows, 0};
  if (map_lookup(key, map)) return true;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(head_dim) * esz};
  // rows of 128 bytes or more: 128-byte boxes, 128-byte swizzle; narrower rows
  // (E4M3 at head_dim 64) as one unswizzled box per row
  const bool narrow = static_cast<int64_t>(head_dim) * esz < 128;
  cuuint32_t box[2] = {static_cast<cuuint32_t>(narrow ? head_dim : 128 / esz),
                       static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, esz == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16,
                   2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   narrow ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS && std::getenv("PA_DEBUG"))
    std::fprintf(stderr, "libpa: pool tensor map: CUresult %d\n", static_cast<int>(r));
  if (r == CUDA_SUCCESS) map_store(key, *map);
  return r == CUDA_SUCCESS;
}

bool make_q_tensor_map(CUtensorMap* map, const void* q, int64_t total_q, int32_t num_q_heads,
                       int32_t head_dim, int32_t group, int32_t rows) {
  const MapKey key{q, 1, total_q, num_q_heads, head_dim, group, rows};
  if (map_lookup(key, map)) return true;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_q_heads),
                        static_cast<cuuint64_t>(total_q)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                           static_cast<cuuint64_t>(num_q_heads) * head_dim * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(q), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS && std::getenv("PA_DEBUG"))
    std::fprintf(stderr, "libpa: q tensor map: CUresult %d\n", static_cast<int>(r));
  if (r == CUDA_SUCCESS) map_store(key, *map);
  return r == CUDA_SUCCESS;
}

}  // namespace pa

using namespace pa;

extern "C" {

const char* pa_status_string(pa_status status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG: invalid argument";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: configuration not supported";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE: workspace too small";
    case PA_ERR_OUT_OF_RANGE: return "PA_ERR_OUT_OF_RANGE: block id or slot outside the pool, or length above max_context_len";
    case PA_ERR_CUDA: return "PA_ERR_CUDA: CUDA runtime or launch failure";
    case PA_ERR_TIMEOUT: return "PA_ERR_TIMEOUT: a kernel gave up a bounded wait";
  }
  return "PA_ERR_UNKNOWN";
}

pa_status pa_reshape_and_cache(const void* key, const void* value, pa_dtype src_dtype,
                               int64_t num_tokens, int64_t token_stride,
                               const int64_t* slot_mapping, void* k_cache, void* v_cache,
                               const pa_cache_desc* cache, void* stream) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (num_tokens < 0) return PA_ERR_INVALID_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !slot_mapping || !k_cache || !v_cache) return PA_ERR_INVALID_ARG;
  if (src_dtype != PA_F16 && src_dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (cache->kv_dtype != PA_FP8_E4M3 && cache->kv_dtype != src_dtype) return PA_ERR_UNSUPPORTED;
  if (cache->head_dim % 8 != 0) return PA_ERR_UNSUPPORTED;
  const int64_t row = static_cast<int64_t>(cache->num_kv_heads) * cache->head_dim;
  if (token_stride < row) return PA_ERR_INVALID_ARG;
  if ((token_stride * 2) % 16 != 0) return PA_ERR_INVALID_ARG;
  const uintptr_t pool_align = cache->kv_dtype == PA_FP8_E4M3 ? 8 : 16;
  if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_cache, pool_align) ||
      !aligned(v_cache, pool_align) || !aligned(slot_mapping, 8))
    return PA_ERR_INVALID_ARG;
  cudaError_t e = launch_reshape_and_cache(
      key, value, src_dtype, num_tokens, token_stride, slot_mapping, k_cache, v_cache,
      cache->num_blocks, cache->block_size, cache->num_kv_heads, cache->head_dim,
      cache->kv_dtype, cache->k_scale, cache->v_scale, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "reshape_and_cache launch");
}

size_t pa_decode_workspace_size(int32_t batch, int32_t num_q_heads, int32_t head_dim,
                                int32_t max_context_len, int32_t partition_size) {
  if (batch <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len <= 0) return 0;
  if (!valid_partition(partition_size)) return 0;
  const int32_t ps = resolve_partition(batch, num_q_heads, max_context_len, partition_size);
  const int32_t parts = static_cast<int32_t>(cdiv(max_context_len, ps));
  return decode_workspace_layout(batch, num_q_heads, head_dim, parts).total;
}

// Varlen workspace: [row_seq | row_len] int32 [total_q] each, the prefill
// work list (int2 [capacity] + a count and a unit counter), then the split-K
// partials.  With the chunk path the decode kernel sees one work row per
// request (num_seqs rows); without it one per packed query row (total_q).
static int64_t varlen_head_bytes(int32_t num_seqs, int32_t total_q) {
  const int64_t maps = 2 * align_up(static_cast<int64_t>(total_q) * 4, kAlign);
  const int64_t items =
      align_up(static_cast<int64_t>(prefill_item_capacity(num_seqs, total_q)) * 8, kAlign) +
      kAlign;
  return maps + items;
}

static int64_t varlen_partials(int64_t rows, int32_t num_q_heads, int32_t head_dim,
                               int32_t max_context_len) {
  if (max_context_len <= 0) return 0;
  const int32_t ps = auto_partition(rows, num_q_heads, max_context_len);
  const int32_t parts = static_cast<int32_t>(cdiv(max_context_len, ps));
  return static_cast<int64_t>(decode_workspace_layout(rows, num_q_heads, head_dim, parts).total);
}

size_t pa_varlen_workspace_size(int32_t num_seqs, int32_t total_q, int32_t num_q_heads,
                                int32_t head_dim, int32_t max_context_len) {
  if (num_seqs <= 0 || total_q <= 0 || num_q_heads <= 0 || head_dim <= 0) return 0;
  const int64_t a = varlen_partials(total_q, num_q_heads, head_dim, max_context_len);
  const int64_t b = varlen_partials(num_seqs, num_q_heads, head_dim, max_context_len);
  return static_cast<size_t>(varlen_head_bytes(num_seqs, total_q) + (a > b ? a : b));
}

// Whether pa_varlen runs the q_len >= 2 requests on the chunk kernel.
static bool varlen_chunk_path(int32_t max_q_len, pa_dtype q_dtype, pa_dtype kv_dtype,
                              int32_t head_dim, int32_t group, const void* out) {
  return max_q_len >= 2 && (out == nullptr || aligned(out, 16)) &&
         prefill_supported(q_dtype, kv_dtype, head_dim, group);
}

size_t pa_varlen_workspace_size_ex(int32_t num_seqs, int32_t total_q, int32_t num_q_heads,
                                   int32_t num_kv_heads, int32_t head_dim, int32_t max_q_len,
                                   int32_t max_context_len, pa_dtype q_dtype, pa_dtype kv_dtype) {
  if (num_seqs <= 0 || total_q <= 0 || num_q_heads <= 0 || head_dim <= 0 || num_kv_heads <= 0 ||
      num_q_heads % num_kv_heads != 0)
    return 0;
  const bool chunks = varlen_chunk_path(max_q_len, q_dtype, kv_dtype, head_dim,
                                        num_q_heads / num_kv_heads, nullptr);
  return static_cast<size_t>(
      varlen_head_bytes(num_seqs, total_q) +
      varlen_partials(chunks ? num_seqs : total_q, num_q_heads, head_dim, max_context_len));
}

static pa_status check_attention(void* out, pa_dtype out_dtype, const void* q, pa_dtype q_dtype,
                                 int32_t num_q_heads, const void* k_cache, const void* v_cache,
                                 const pa_cache_desc* cache, const int32_t* block_tables,
                                 int32_t max_blocks_per_seq, int32_t max_context_len) {
  pa_status st = check_cache(cache);
  if (st != PA_OK) return st;
  if (!out || !q || !k_cache || !v_cache || !block_tables) return PA_ERR_INVALID_ARG;
  if (num_q_heads <= 0 || num_q_heads % cache->num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  if (max_context_len < 0 || max_blocks_per_seq < 0) return PA_ERR_INVALID_ARG;
  if (cdiv(max_context_len, cache->block_size) > max_blocks_per_seq) return PA_ERR_INVALID_ARG;
  if (out_dtype != PA_F16 && out_dtype != PA_BF16 && out_dtype != PA_F32)
    return PA_ERR_UNSUPPORTED;
  const int32_t group = num_q_heads / cache->num_kv_heads;
  if (!attention_supported(q_dtype, cache->kv_dtype, cache->head_dim, group))
    return PA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(out, elem_size(out_dtype)) || !aligned(block_tables, 4))
    return PA_ERR_INVALID_ARG;
  return PA_OK;
}

static pa_status run_attention(AttnArgs& a, const pa_cache_desc* cache, int32_t max_context_len,
                               int32_t ps, float* ws_base, size_t ws_bytes, size_t ws_needed,
                               cudaStream_t stream) {
  a.partition_size = ps;
  a.max_context_len = max_context_len;
  a.max_parts = static_cast<int32_t>(cdiv(max_context_len > 0 ? max_context_len : 1, ps));
  if (a.max_parts > 1) {
    if (!ws_base || ws_bytes < ws_needed) return PA_ERR_WORKSPACE;
    if (!aligned(ws_base, 256)) return PA_ERR_INVALID_ARG;
    DecodeWorkspace w = decode_workspace_layout(a.rows, a.num_q_heads, a.head_dim, a.max_parts);
    auto* b = reinterpret_cast<uint8_t*>(ws_base);
    a.ws_m = reinterpret_cast<float*>(b + w.m_off);
    a.ws_l = reinterpret_cast<float*>(b + w.l_off);
    a.ws_o = reinterpret_cast<float*>(b + w.o_off);
  } else {
    a.ws_m = a.ws_l = a.ws_o = nullptr;
  }
  const int64_t pool_rows = static_cast<int64_t>(cache->num_blocks) * cache->num_kv_heads *
                            cache->block_size;
  const int32_t box_rows = cache->block_size < 16 ? cache->block_size : 16;
  CUtensorMap kmap, vmap;
  if (!make_pool_tensor_map(&kmap, a.k_cache, cache->kv_dtype, pool_rows, cache->head_dim,
                            box_rows) ||
      !make_pool_tensor_map(&vmap, a.v_cache, cache->kv_dtype, pool_rows, cache->head_dim,
                            box_rows))
    return map_fail("the KV pool");
  cudaError_t e = launch_paged_attention(a, kmap, vmap, stream);
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "attention launch");
}

static void fill_common(AttnArgs& a, void* out, pa_dtype out_dtype, const void* q,
                        pa_dtype q_dtype, int32_t num_q_heads, const void* k_cache,
                        const void* v_cache, const pa_cache_desc* cache,
                        const int32_t* block_tables, int32_t max_blocks_per_seq, float scale) {
  std::memset(&a, 0, sizeof(a));
  a.out = out;
  a.q = q;
  a.out_dtype = out_dtype;
  a.q_dtype = q_dtype;
  a.kv_dtype = cache->kv_dtype;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = cache->num_kv_heads;
  a.head_dim = cache->head_dim;
  a.group = num_q_heads / cache->num_kv_heads;
  a.head_chunks = a.group > 8 ? (a.group + 7) / 8 : 1;
  a.num_blocks = cache->num_blocks;
  a.block_size = cache->block_size;
  a.block_tables = block_tables;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.k_scale = cache->k_scale;
  a.v_scale = cache->v_scale;
  a.scale = scale;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
}

static pa_status apply_options(AttnArgs& a, const pa_attn_options* o) {
  a.window = 0;
  a.alibi = nullptr;
  if (!o) return PA_OK;
  if (o->alibi_slopes && !aligned(o->alibi_slopes, 4)) return PA_ERR_INVALID_ARG;
  a.window = o->window > 0 ? o->window : 0;
  a.alibi = o->alibi_slopes;
  return PA_OK;
}

pa_status pa_decode(void* out, pa_dtype out_dtype, const void* q, pa_dtype q_dtype,
                    int32_t batch, int32_t num_q_heads, const void* k_cache,
                    const void* v_cache, const pa_cache_desc* cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* context_lens, int32_t max_context_len, float scale,
                    int32_t partition_size, void* workspace, size_t workspace_bytes,
                    void* stream) {
  return pa_decode_ex(out, out_dtype, q, q_dtype, batch, num_q_heads, k_cache, v_cache, cache,
                      block_tables, max_blocks_per_seq, context_lens, max_context_len, scale,
                      partition_size, nullptr, workspace, workspace_bytes, stream);
}

pa_status pa_decode_ex(void* out, pa_dtype out_dtype, const void* q, pa_dtype q_dtype,
                       int32_t batch, int32_t num_q_heads, const void* k_cache,
                       const void* v_cache, const pa_cache_desc* cache,
                       const int32_t* block_tables, int32_t max_blocks_per_seq,
                       const int32_t* context_lens, int32_t max_context_len, float scale,
                       int32_t partition_size, const pa_attn_options* options, void* workspace,
                       size_t workspace_bytes, void* stream) {
  if (batch < 0) return PA_ERR_INVALID_ARG;
  pa_status st = check_attention(out, out_dtype, q, q_dtype, num_q_heads, k_cache, v_cache,
                                 cache, block_tables, max_blocks_per_seq, max_context_len);
  if (st != PA_OK) return st;
  if (!context_lens) return PA_ERR_INVALID_ARG;
  if (!valid_partition(partition_size)) return PA_ERR_INVALID_ARG;
  if (batch == 0) return PA_OK;
  AttnArgs a;
  fill_common(a, out, out_dtype, q, q_dtype, num_q_heads, k_cache, v_cache, cache, block_tables,
              max_blocks_per_seq, scale);
  a.rows = batch;
  a.num_seqs = batch;
  a.context_lens = context_lens;
  st = apply_options(a, options);
  if (st != PA_OK) return st;
  const int32_t ps = resolve_partition(batch, num_q_heads, max_context_len, partition_size);
  const size_t need =
      pa_decode_workspace_size(batch, num_q_heads, cache->head_dim, max_context_len, ps);
  return run_attention(a, cache, max_context_len, ps, static_cast<float*>(workspace),
                       workspace_bytes, need, static_cast<cudaStream_t>(stream));
}

pa_status pa_varlen(void* out, pa_dtype out_dtype, const void* q, pa_dtype q_dtype,
                    int32_t total_q, int32_t num_seqs, int32_t num_q_heads,
                    const int32_t* cu_seqlens_q, const int32_t* seqlens_k, int32_t max_q_len,
                    int32_t max_context_len, const void* k_cache, const void* v_cache,
                    const pa_cache_desc* cache, const int32_t* block_tables,
                    int32_t max_blocks_per_seq, float scale, void* workspace,
                    size_t workspace_bytes, void* stream) {
  return pa_varlen_ex(out, out_dtype, q, q_dtype, total_q, num_seqs, num_q_heads, cu_seqlens_q,
                      seqlens_k, max_q_len, max_context_len, k_cache, v_cache, cache,
                      block_tables, max_blocks_per_seq, scale, nullptr, workspace,
                      workspace_bytes, stream);
}

pa_status pa_varlen_ex(void* out, pa_dtype out_dtype, const void* q, pa_dtype q_dtype,
                       int32_t total_q, int32_t num_seqs, int32_t num_q_heads,
                       const int32_t* cu_seqlens_q, const int32_t* seqlens_k, int32_t max_q_len,
                       int32_t max_context_len, const void* k_cache, const void* v_cache,
                       const pa_cache_desc* cache, const int32_t* block_tables,
                       int32_t max_blocks_per_seq, float scale, const pa_attn_options* options,
                       void* workspace, size_t workspace_bytes, void* stream) {
  if (total_q < 0 || num_seqs < 0 || max_q_len < 0) return PA_ERR_INVALID_ARG;
  pa_status st = check_attention(out, out_dtype, q, q_dtype, num_q_heads, k_cache, v_cache,
                                 cache, block_tables, max_blocks_per_seq, max_context_len);
  if (st != PA_OK) return st;
  if (!cu_seqlens_q || !seqlens_k) return PA_ERR_INVALID_ARG;
  if (max_q_len > max_context_len) return PA_ERR_INVALID_ARG;
  if (total_q == 0) return PA_OK;
  if (num_seqs == 0) return PA_ERR_INVALID_ARG;
  const int32_t group = num_q_heads / cache->num_kv_heads;
  const bool chunks = varlen_chunk_path(max_q_len, q_dtype, cache->kv_dtype, cache->head_dim,
                                        group, out);
  const int64_t rows = chunks ? num_seqs : total_q;
  const size_t need = static_cast<size_t>(
      varlen_head_bytes(num_seqs, total_q) +
      varlen_partials(rows, num_q_heads, cache->head_dim, max_context_len));
  if (!workspace || workspace_bytes < need) return PA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return PA_ERR_INVALID_ARG;
  auto* b = static_cast<uint8_t*>(workspace);
  const int64_t map_bytes = align_up(static_cast<int64_t>(total_q) * 4, kAlign);
  const int32_t capacity = prefill_item_capacity(num_seqs, total_q);
  const int64_t item_bytes = align_up(static_cast<int64_t>(capacity) * 8, kAlign) + kAlign;
  int32_t* row_seq = reinterpret_cast<int32_t*>(b);
  int32_t* row_len = reinterpret_cast<int32_t*>(b + map_bytes);
  int2* items = reinterpret_cast<int2*>(b + 2 * map_bytes);
  int32_t* item_count = reinterpret_cast<int32_t*>(b + 2 * map_bytes + item_bytes - kAlign);
  uint8_t* partials = b + 2 * map_bytes + item_bytes;
  const size_t head = static_cast<size_t>(2 * map_bytes + item_bytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  AttnArgs a;
  fill_common(a, out, out_dtype, q, q_dtype, num_q_heads, k_cache, v_cache, cache, block_tables,
              max_blocks_per_seq, scale);
  st = apply_options(a, options);
  if (st != PA_OK) return st;
  a.num_seqs = num_seqs;
  a.cu_seqlens_q = cu_seqlens_q;
  a.seqlens_k = seqlens_k;
  if (chunks) {
    // q_len >= 2 requests: the tensor-core prefill over a compact work list;
    // q_len == 1 requests: the decode kernel, one work row per request.
    const int64_t pool_rows =
        static_cast<int64_t>(cache->num_blocks) * cache->num_kv_heads * cache->block_size;
    const int32_t box_rows = cache->block_size < 16 ? cache->block_size : 16;
    CUtensorMap kmap, vmap, qmap;
    if (!make_pool_tensor_map(&kmap, k_cache, cache->kv_dtype, pool_rows, cache->head_dim,
                              box_rows) ||
        !make_pool_tensor_map(&vmap, v_cache, cache->kv_dtype, pool_rows, cache->head_dim,
                              box_rows) ||
        !make_q_tensor_map(&qmap, q, total_q, num_q_heads, cache->head_dim, group,
                           prefill_query_tile(group)))
      return map_fail("the prefill operands");
    AttnArgs p = a;
    p.max_context_len = max_context_len;
    p.pf_items = items;
    p.pf_count = item_count;
    cudaError_t fe = launch_paged_prefill(p, kmap, vmap, qmap, capacity, item_count + 1, s);
    if (fe != cudaSuccess) return cuda_fail(fe, "prefill launch");
    a.rows = num_seqs;
    a.varlen_requests = 1;
  } else {
    cudaError_t pe = launch_varlen_prep(total_q, num_seqs, cu_seqlens_q, seqlens_k, row_seq,
                                        row_len, false, s);
    if (pe != cudaSuccess) return cuda_fail(pe, "varlen row map launch");
    a.rows = total_q;
    a.row_seq = row_seq;
    a.row_len = row_len;
  }
  const int32_t ps = auto_partition(rows, num_q_heads, max_context_len > 0 ? max_context_len : 1);
  const size_t part_need =
      static_cast<size_t>(varlen_partials(rows, num_q_heads, cache->head_dim, max_context_len));
  return run_attention(a, cache, max_context_len, ps, reinterpret_cast<float*>(partials),
                       workspace_bytes - head, part_need, s);
}

static int64_t block_bytes_of(const pa_cache_desc* c) {
  return static_cast<int64_t>(c->num_kv_heads) * c->block_size * c->head_dim *
         static_cast<int64_t>(elem_size(c->kv_dtype));
}

pa_status pa_copy_blocks(void* k_cache, void* v_cache, const pa_cache_desc* cache,
                         const int64_t* block_mapping, int64_t num_pairs, void* stream) {
  // geometry only: copying bytes needs no FP8 scales
  if (!cache || cache->num_blocks <= 0 || cache->num_kv_heads <= 0 || cache->head_dim <= 0 ||
      cache->block_size <= 0)
    return PA_ERR_INVALID_ARG;
  if (!elem_size(cache->kv_dtype) || cache->kv_dtype == PA_F32) return PA_ERR_UNSUPPORTED;
  if (num_pairs < 0) return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (!k_cache || !v_cache || !block_mapping) return PA_ERR_INVALID_ARG;
  const int64_t bb = block_bytes_of(cache);
  if (bb % 16 != 0 || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_mapping, 8))
    return PA_ERR_INVALID_ARG;
  cudaError_t e = launch_copy_blocks(k_cache, v_cache, block_mapping, num_pairs, bb,
                                     cache->num_blocks, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "copy_blocks launch");
}

pa_status pa_swap_blocks(void* dst_k, void* dst_v, const void* src_k, const void* src_v,
                         const pa_cache_desc* cache, int64_t src_num_blocks,
                         int64_t dst_num_blocks, const int64_t* block_mapping, int64_t num_pairs,
                         void* stream) {
  if (!cache || cache->num_kv_heads <= 0 || cache->head_dim <= 0 || cache->block_size <= 0)
    return PA_ERR_INVALID_ARG;
  if (!elem_size(cache->kv_dtype) || cache->kv_dtype == PA_F32) return PA_ERR_UNSUPPORTED;
  if (num_pairs < 0 || src_num_blocks < 0 || dst_num_blocks < 0) return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (!dst_k || !dst_v || !src_k || !src_v || !block_mapping) return PA_ERR_INVALID_ARG;
  for (int64_t i = 0; i < num_pairs; ++i) {
    const int64_t s = block_mapping[2 * i], d = block_mapping[2 * i + 1];
    if (s < 0 || s >= src_num_blocks || d < 0 || d >= dst_num_blocks) return PA_ERR_INVALID_ARG;
  }
  const int64_t bb = block_bytes_of(cache);
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  // Pools the GPU can address (device memory, mapped pinned host memory):
  // one gather/scatter kernel per 1024 pairs.  Otherwise one copy per run.
  auto addressable = [](const void* p) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
      (void)cudaGetLastError();
      return false;
    }
    return at.type == cudaMemoryTypeDevice ||
           (at.type == cudaMemoryTypeHost && at.devicePointer == p);
  };
  if (bb % 16 == 0 && addressable(dst_k) && addressable(dst_v) && addressable(src_k) &&
      addressable(src_v) && aligned(dst_k, 16) && aligned(dst_v, 16) && aligned(src_k, 16) &&
      aligned(src_v, 16)) {
    cudaError_t e =
        launch_move_blocks(dst_k, dst_v, src_k, src_v, block_mapping, num_pairs, bb, strm);
    return e == cudaSuccess ? PA_OK : cuda_fail(e, "swap_blocks launch");
  }
  int64_t i = 0;
  while (i < num_pairs) {
    const int64_t s0 = block_mapping[2 * i], d0 = block_mapping[2 * i + 1];
    int64_t n = 1;
    while (i + n < num_pairs && block_mapping[2 * (i + n)] == s0 + n &&
           block_mapping[2 * (i + n) + 1] == d0 + n)
      ++n;
    const size_t bytes = static_cast<size_t>(n * bb);
    cudaError_t e = cudaMemcpyAsync(static_cast<uint8_t*>(dst_k) + d0 * bb,
                                    static_cast<const uint8_t*>(src_k) + s0 * bb, bytes,
                                    cudaMemcpyDefault, strm);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(static_cast<uint8_t*>(dst_v) + d0 * bb,
                          static_cast<const uint8_t*>(src_v) + s0 * bb, bytes, cudaMemcpyDefault,
                          strm);
    if (e != cudaSuccess) return cuda_fail(e, "swap_blocks copy");
    i += n;
  }
  return PA_OK;
}

pa_status pa_hbm_read_probe(const void* buf, int64_t bytes, void* sink, void* stream) {
  if (bytes < 0 || bytes % 16 != 0 || !sink || !aligned(sink, 4)) return PA_ERR_INVALID_ARG;
  if (bytes > 0 && (!buf || !aligned(buf, 16))) return PA_ERR_INVALID_ARG;
  cudaError_t e = launch_hbm_read_probe(buf, bytes, static_cast<uint32_t*>(sink),
                                        static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "hbm_read_probe launch");
}

pa_status pa_selftest_wait_timeout(void* stream) {
  cudaError_t e = launch_wait_timeout_selftest(static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PA_OK : cuda_fail(e, "wait-timeout self-test launch");
}

pa_status pa_device_error(void* stream) {
  cudaError_t e;
  unsigned v = read_and_clear_error_word(static_cast<cudaStream_t>(stream), &e);
  if (e != cudaSuccess) return PA_ERR_CUDA;
  if (v == kErrTimeout) return PA_ERR_TIMEOUT;
  if (v != 0) return PA_ERR_OUT_OF_RANGE;
  return PA_OK;
}

}  // extern "C"
