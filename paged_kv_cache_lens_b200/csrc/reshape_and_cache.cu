// Cache write for the paged KV pool (sm_100a).
//
// "PagedAttention 与 Continuous Batching", §3.3 (数据结构): each decode step
// computes the new token's K/V and appends it to the sequence's last block, or
// to a freshly allocated block when the last one is full; §2.5 step 4 hands
// the chosen physical slot of every token to the forward pass as slot_mapping.
// This kernel performs that scatter: row i of K/V ([Hkv][D]) goes to
// pool[slot / 16][h][slot % 16][:] for every head h.
//
// One thread moves 8 consecutive elements (a 16-byte load); consecutive
// threads cover consecutive elements of a token row, so both the read and the
// write of a (token, head) row are coalesced 16-byte accesses.  The FP8 E4M3
// variant divides by the per-head scale (IEEE fp32 division) and rounds to
// nearest even with saturation.
#include "pa_device.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

template <int MODE>  // 0: 16-bit copy, 1: bf16 -> e4m3, 2: f16 -> e4m3
__global__ void __launch_bounds__(256)
reshape_and_cache_kernel(const uint16_t* __restrict__ key, const uint16_t* __restrict__ value,
                         int64_t num_tokens, int64_t token_stride,
                         const int64_t* __restrict__ slot_mapping, void* k_cache, void* v_cache,
                         int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                         int32_t head_dim, const float* __restrict__ k_scale,
                         const float* __restrict__ v_scale) {
  const int chunks_per_row = head_dim >> 3;
  const int64_t per_token = static_cast<int64_t>(num_kv_heads) * chunks_per_row;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= num_tokens * per_token) return;
  const int64_t i = gid / per_token;
  const int rem = static_cast<int>(gid - i * per_token);
  const int h = rem / chunks_per_row;
  const int ch = rem - h * chunks_per_row;
  const int64_t slot = slot_mapping[i];
  if (slot < 0) return;
  const int64_t blk = slot / block_size;
  const int64_t off = slot - blk * block_size;
  if (blk >= num_blocks) {
    report_error(kErrSlotRange);
    return;
  }
  const int64_t src = i * token_stride + static_cast<int64_t>(h) * head_dim + ch * 8;
  const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim + ch * 8;
  const uint4 kv = *reinterpret_cast<const uint4*>(key + src);
  const uint4 vv = *reinterpret_cast<const uint4*>(value + src);
  if constexpr (MODE == 0) {
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(k_cache) + dst) = kv;
    *reinterpret_cast<uint4*>(static_cast<uint16_t*>(v_cache) + dst) = vv;
  } else {
    const float ks = k_scale[h], vs = v_scale[h];
    auto quant8 = [&](const uint4 w, float sc) -> uint2 {
      const uint32_t in[4] = {w.x, w.y, w.z, w.w};
      uint32_t outw[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        uint32_t packed = 0;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const uint32_t word = in[2 * j + e];
          float lo, hi;
          if constexpr (MODE == 1) {
            lo = __uint_as_float(word << 16);
            hi = __uint_as_float(word & 0xFFFF0000u);
          } else {
            lo = __half2float(__ushort_as_half(static_cast<unsigned short>(word & 0xFFFF)));
            hi = __half2float(__ushort_as_half(static_cast<unsigned short>(word >> 16)));
          }
          const float qlo = __fdiv_rn(lo, sc);
          const float qhi = __fdiv_rn(hi, sc);
          uint16_t two;
          asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(two) : "f"(qhi), "f"(qlo));
          packed |= static_cast<uint32_t>(two) << (16 * e);
        }
        outw[j] = packed;
      }
      return make_uint2(outw[0], outw[1]);
    };
    *reinterpret_cast<uint2*>(static_cast<uint8_t*>(k_cache) + dst) = quant8(kv, ks);
    *reinterpret_cast<uint2*>(static_cast<uint8_t*>(v_cache) + dst) = quant8(vv, vs);
  }
}

}  // namespace

cudaError_t launch_reshape_and_cache(const void* key, const void* value, int src_dtype,
                                     int64_t num_tokens, int64_t token_stride,
                                     const int64_t* slot_mapping, void* k_cache, void* v_cache,
                                     int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                                     int32_t head_dim, int kv_dtype, const float* k_scale,
                                     const float* v_scale, cudaStream_t stream) {
  const int64_t total = num_tokens * num_kv_heads * (head_dim / 8);
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (total + threads - 1) / threads;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  const auto* k = static_cast<const uint16_t*>(key);
  const auto* v = static_cast<const uint16_t*>(value);
  if (kv_dtype == 2) {
    if (src_dtype == 1)
      reshape_and_cache_kernel<1><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
          k, v, num_tokens, token_stride, slot_mapping, k_cache, v_cache, num_blocks, block_size,
          num_kv_heads, head_dim, k_scale, v_scale);
    else
      reshape_and_cache_kernel<2><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
          k, v, num_tokens, token_stride, slot_mapping, k_cache, v_cache, num_blocks, block_size,
          num_kv_heads, head_dim, k_scale, v_scale);
  } else {
    reshape_and_cache_kernel<0><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
        k, v, num_tokens, token_stride, slot_mapping, k_cache, v_cache, num_blocks, block_size,
        num_kv_heads, head_dim, k_scale, v_scale);
  }
  return cudaGetLastError();
}

}  // namespace pa
