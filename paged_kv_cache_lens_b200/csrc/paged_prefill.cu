// Prefill chunks of the packed varlen step on the 5th-generation tensor cores
// (tcgen05 + TMEM + TMA), sm_100a.
//
// What is computed ("推理优化与服务：从 PagedAttention 到分离式部署", 最新进展: the
// V1 step packs every scheduled query token as [total_q, H, D] with
// cu_seqlens; "PagedAttention 与 Continuous Batching", §4.2: chunked prefill
// mixes prompt chunks with decodes): for a request with q_len > 1 rows over
// kv_len keys (cached context + this chunk, already in the paged pool), row i
// attends keys 0 .. kv_len - q_len + i through the request's block table.
//
// One CTA = (request, KV head, tile of 128/G query positions); the G query
// heads of the GQA group are stacked so the Q tile is a dense 128-row operand
// and every K/V tile is read once for the whole group.  Per 128-key tile:
//   S = Q K^T        tcgen05.mma kind::f16, A = Q and B = K from shared memory
//                    (128-byte swizzle, K-major), D = S in TMEM (fp32);
//   P = softmax row  one thread per row reads its TMEM lane, writes P as
//                    bf16/f16 hi + lo halves back into the same TMEM columns;
//   O += P V         tcgen05.mma with A = P straight from TMEM and B = V from
//                    shared memory (MN-major), D = O in TMEM.
// Softmax is taken in two passes over the keys (pass 1: row max and sum; pass
// 2: normalised P), so O never needs rescaling.  Warp roles: warps 0-3 own
// the 128 rows (TMEM lanes), warp 4 issues the TMA loads (paged K/V tiles are
// gathered block by block: 8 boxes of 16 tokens per 128-key tile), warp 5
// allocates TMEM and issues the MMAs from one thread.  S/P live in two TMEM
// buffers so the MMA of tile j+1 overlaps the softmax of tile j.
#include "pa_device.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

constexpr int kPfThreads = 192;          // 4 softmax warps, 1 TMA warp, 1 MMA warp
constexpr int kBN = 128;                 // keys per tile
constexpr int kHalf = 128 * 128;         // one 64-column (128-byte) half of a 128-row tile
constexpr int kQBytes = 2 * kHalf;
constexpr int kKVBytes = 2 * kHalf;
constexpr int kStageBytes = 2 * kKVBytes;
constexpr int kStages = 2;
constexpr int kBarBase = kQBytes + kStages * kStageBytes;
constexpr int kNumBars = 12;
constexpr int kSmemBytes = kBarBase + kNumBars * 8 + 16 + 1024;
constexpr uint32_t kTmemCols = 512;      // S/P buffer 0 at col 0, buffer 1 at 128, O at 256
constexpr uint32_t kWaitLimit = 1u << 20;
constexpr float kLog2eF = 1.4426950408889634f;

enum { B_Q = 0, B_KVF = 1, B_KVE = 3, B_SF = 5, B_PF = 7, B_PVD = 9, B_O = 11 };

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023) == 1023 && *abort_flag) return false;
  }
  *abort_flag = 1;
  report_error(kErrTimeout);
  return false;
}

template <bool BF16, int G>
__global__ void __launch_bounds__(kPfThreads, 1)
paged_prefill_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap,
                     const __grid_constant__ CUtensorMap qmap) {
  constexpr int TQ = 128 / G;             // query positions per tile
  constexpr uint32_t kIdescS = idesc_f16(BF16, 128, kBN, false);
  constexpr uint32_t kIdescPV = idesc_f16(BF16, 128, 128, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarBase);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarBase + kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: (request, KV head, query tile); heavier (later) tiles first
  const int nqt = a.max_parts;            // query tiles per request (host: ceil(max_q_len/TQ))
  int64_t bid = blockIdx.x;
  const int qt = nqt - 1 - static_cast<int>(bid % nqt);
  bid /= nqt;
  const int h = static_cast<int>(bid % a.num_kv_heads);
  const int r = static_cast<int>(bid / a.num_kv_heads);
  const int cu0 = a.cu_seqlens_q[r];
  const int q_len = a.cu_seqlens_q[r + 1] - cu0;
  if (q_len < 2 || qt * TQ >= q_len) return;        // decode rows and empty tiles
  const int kv_len = min(a.seqlens_k[r], a.max_context_len);
  const int rows_valid = min(TQ, q_len - qt * TQ);
  const int pos0 = kv_len - q_len + qt * TQ;        // absolute position of tile row 0
  const int last_pos = pos0 + rows_valid - 1;
  if (last_pos < 0) return;
  const int nkv = last_pos / kBN + 1;
  const int n_iter = 2 * nkv;
  const int hq0 = h * G;

  if (threadIdx.x == 0) {
    mbar_init(&bars[B_Q], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[B_KVF + s], 1);
      mbar_init(&bars[B_KVE + s], 1);
      mbar_init(&bars[B_SF + s], 1);
      mbar_init(&bars[B_PF + s], 128);
      mbar_init(&bars[B_PVD + s], 1);
    }
    mbar_init(&bars[B_O], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ================================================================ TMA producer
    if (lane == 0) {
      const int oob_row = a.num_blocks * a.num_kv_heads * 16;
      const int32_t* bt = a.block_tables + static_cast<int64_t>(r) * a.max_blocks_per_seq;
      mbar_arrive_expect_tx(&bars[B_Q], kQBytes);
      tma_load_3d(sQ, &qmap, 0, hq0, cu0 + qt * TQ, &bars[B_Q]);
      tma_load_3d(sQ + kHalf, &qmap, 64, hq0, cu0 + qt * TQ, &bars[B_Q]);
      const uint64_t pol = l2_policy_evict_last();
      uint32_t ph_empty[2] = {0, 0};
      int issued = 0;
      for (int it = 0; it < n_iter && !*abort_flag; ++it) {
        const int st = it & 1;
        if (it >= 2) {
          if (!wait_or_abort(&bars[B_KVE + st], ph_empty[st], abort_flag)) break;
          ph_empty[st] ^= 1;
        }
        const bool pass2 = it >= nkv;
        const int j = pass2 ? it - nkv : it;
        uint8_t* sK = smem + kQBytes + st * kStageBytes;
        uint8_t* sV = sK + kKVBytes;
        mbar_arrive_expect_tx(&bars[B_KVF + st], pass2 ? kStageBytes : kKVBytes);
        int ys[8];
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          const int key0 = j * kBN + b * 16;
          int y = oob_row;
          if (key0 < kv_len) {
            const int phys = __ldg(bt + key0 / 16);
            if (static_cast<unsigned>(phys) < static_cast<unsigned>(a.num_blocks))
              y = (phys * a.num_kv_heads + h) * 16;
            else
              report_error(kErrBlockRange);
          }
          ys[b] = y;
        }
#pragma unroll
        for (int b = 0; b < 8; ++b) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            tma_load_2d(sK + half * kHalf + b * 2048, &kmap, half * 64, ys[b], &bars[B_KVF + st],
                        pol);
            if (pass2)
              tma_load_2d(sV + half * kHalf + b * 2048, &vmap, half * 64, ys[b],
                          &bars[B_KVF + st], pol);
          }
        }
        issued = it + 1;
      }
      // the last copies into each stage have landed before the CTA may exit
      for (int it = issued - 1; it >= 0 && it >= issued - 2; --it)
        (void)mbar_wait_bounded(&bars[B_KVF + (it & 1)], (it >> 1) & 1);
      (void)mbar_wait_bounded(&bars[B_Q], 0);
    }
  } else if (warp == 5) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      uint32_t ph_full[2] = {0, 0}, ph_pf[2] = {0, 0}, ph_pvd[2] = {0, 0};
      bool ok = wait_or_abort(&bars[B_Q], 0, abort_flag);
      const uint32_t q_addr = smem_u32(sQ);
      bool first_pv = true;
      auto issue_s = [&](int it) -> bool {
        const int st = it & 1;
        if (!wait_or_abort(&bars[B_KVF + st], ph_full[st], abort_flag)) return false;
        ph_full[st] ^= 1;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(smem + kQBytes + st * kStageBytes);
        const uint32_t d = tmem + static_cast<uint32_t>((it & 1) * 128);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
          tc_mma_ss(d, smem_desc_sw128(q_addr + off, 16, 1024),
                    smem_desc_sw128(k_addr + off, 16, 1024), kIdescS, ks > 0 ? 1u : 0u);
        }
        tc_commit(&bars[B_SF + (it & 1)]);
        if (it < nkv) tc_commit(&bars[B_KVE + st]);     // pass 1 only needs K
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int it = 0; ok && it < n_iter; ++it) {
        const int b = it & 1;
        // S of the next tile into the other buffer, once that buffer is free
        if (it + 1 < n_iter) {
          const int pb = (it + 1) & 1;
          if (it >= 1) {
            if (it - 1 < nkv) {            // softmax finished reading S(it-1)
              if (!(ok = wait_or_abort(&bars[B_PF + pb], ph_pf[pb], abort_flag))) break;
              ph_pf[pb] ^= 1;
            } else {                       // PV(it-1) finished reading P(it-1)
              if (!(ok = wait_or_abort(&bars[B_PVD + pb], ph_pvd[pb], abort_flag))) break;
              ph_pvd[pb] ^= 1;
            }
          }
          if (!(ok = issue_s(it + 1))) break;
        }
        if (it >= nkv) {
          // O += P V once the softmax warps have written P(it)
          if (!(ok = wait_or_abort(&bars[B_PF + b], ph_pf[b], abort_flag))) break;
          ph_pf[b] ^= 1;
          tc_fence_after();
          const int st = it & 1;
          const uint32_t v_addr = smem_u32(smem + kQBytes + st * kStageBytes + kKVBytes);
          const uint32_t p_base = tmem + static_cast<uint32_t>(b * 128);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t vd = smem_desc_sw128(v_addr + ks * 2048, kHalf, 1024);
            tc_mma_ts(tmem + 256, p_base + ks * 8, vd, kIdescPV, first_pv ? 0u : 1u);
            first_pv = false;
            tc_mma_ts(tmem + 256, p_base + 64 + ks * 8, vd, kIdescPV, 1u);
          }
          tc_commit(&bars[B_KVE + st]);
          tc_commit(&bars[B_PVD + b]);
        }
      }
      tc_commit(&bars[B_O]);                 // every MMA issued above is complete
      if (!ok) (void)wait_or_abort(&bars[B_O], 0, abort_flag);
    }
  } else {
    // ================================================================ softmax / epilogue
    const int t = threadIdx.x;                 // row of the tile == TMEM lane
    const int i = t / G, g = t % G;
    const bool row_ok = i < rows_valid;
    const int pos = pos0 + i;
    const float c = a.scale * kLog2eF;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float m = -INFINITY, l = 0.f, inv_l = 0.f;
    uint32_t ph_sf[2] = {0, 0};
    bool ok = true;
    for (int it = 0; it < n_iter; ++it) {
      const int b = it & 1;
      if (!wait_or_abort(&bars[B_SF + b], ph_sf[b], abort_flag)) { ok = false; break; }
      ph_sf[b] ^= 1;
      tc_fence_after();
      const bool pass2 = it >= nkv;
      const int j = pass2 ? it - nkv : it;
      uint32_t raw[128];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t (&chunk)[32] = *reinterpret_cast<uint32_t (*)[32]>(raw + 32 * q4);
        tmem_ld32(lane_base + b * 128 + 32 * q4, chunk);
      }
      tmem_wait_ld();
      const int key0 = j * kBN;
      const int lim = row_ok ? pos - key0 : -1;     // columns n <= lim are visible
      if (!pass2) {
        float tm = -INFINITY;
#pragma unroll
        for (int n = 0; n < 128; ++n)
          if (n <= lim) tm = fmaxf(tm, __uint_as_float(raw[n]) * c);
        const float m_new = fmaxf(m, tm);
        if (m_new != -INFINITY) {
          float sum = 0.f;
#pragma unroll
          for (int n = 0; n < 128; ++n)
            if (n <= lim) sum += exp2f(__uint_as_float(raw[n]) * c - m_new);
          l = l * exp2f(m - m_new) + sum;
          m = m_new;
        }
        tc_fence_before();
        mbar_arrive(&bars[B_PF + b]);
      } else {
        if (it == nkv) inv_l = l > 0.f ? 1.f / l : 0.f;
        uint32_t hi[64], lo[64];
#pragma unroll
        for (int n2 = 0; n2 < 64; ++n2) {
          const int n = 2 * n2;
          const float p0 = (n <= lim) ? exp2f(__uint_as_float(raw[n]) * c - m) * inv_l : 0.f;
          const float p1 =
              (n + 1 <= lim) ? exp2f(__uint_as_float(raw[n + 1]) * c - m) * inv_l : 0.f;
          const uint32_t hw = pack2<BF16>(p0, p1);
          hi[n2] = hw;
          lo[n2] = pack2<BF16>(p0 - lo_half_to_float<BF16>(hw),
                               p1 - lo_half_to_float<BF16>(hw >> 16));
        }
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
          tmem_st32(lane_base + b * 128 + 32 * q2,
                    *reinterpret_cast<const uint32_t (*)[32]>(hi + 32 * q2));
          tmem_st32(lane_base + b * 128 + 64 + 32 * q2,
                    *reinterpret_cast<const uint32_t (*)[32]>(lo + 32 * q2));
        }
        // Keys of the context's partial last block that lie past kv_len hold
        // whatever the slot held; P is 0 there but 0 * NaN is NaN: clear them.
        const int stale0 = kv_len, stale1 = min((kv_len + 15) & ~15, key0 + kBN);
        if (stale0 < stale1 && stale0 >= key0) {
          const int st = it & 1;
          if (wait_or_abort(&bars[B_KVF + st], (it >> 1) & 1, abort_flag)) {
            uint8_t* sV = smem + kQBytes + st * kStageBytes + kKVBytes;
            const int nrows = stale1 - stale0;
            for (int idx = t; idx < nrows * 16; idx += 128) {
              const int row = stale0 - key0 + idx / 16;
              const int c16 = idx % 16;
              *reinterpret_cast<uint4*>(sV + (c16 >> 3) * kHalf + row * 128 + (c16 & 7) * 16) =
                  make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[B_PF + b]);
      }
    }
    // ---- epilogue: O row -> out
    if (ok && wait_or_abort(&bars[B_O], 0, abort_flag)) {
      tc_fence_after();
      uint32_t o[128];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
        tmem_ld32(lane_base + 256 + 32 * q4, *reinterpret_cast<uint32_t (*)[32]>(o + 32 * q4));
      tmem_wait_ld();
      if (row_ok) {
        const int64_t orow =
            (static_cast<int64_t>(cu0 + qt * TQ + i) * a.num_q_heads + hq0 + g) * 128;
        if (a.out_dtype == 3) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow);
#pragma unroll
          for (int k = 0; k < 32; ++k)
            dst[k] = make_float4(__uint_as_float(o[4 * k]), __uint_as_float(o[4 * k + 1]),
                                 __uint_as_float(o[4 * k + 2]), __uint_as_float(o[4 * k + 3]));
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + orow);
          const bool ob = (a.out_dtype == 1);
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = __uint_as_float(o[8 * k + 2 * e]);
              const float x1 = __uint_as_float(o[8 * k + 2 * e + 1]);
              w[e] = ob ? pack2<true>(x0, x1) : pack2<false>(x0, x1);
            }
            dst[k] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
  }

  // ---- teardown: every MMA and copy of this CTA has completed (or been
  // given a bounded chance to) before TMEM is released.
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <bool BF16, int G>
cudaError_t launch_prefill_typed(const AttnArgs& a, const CUtensorMap& k, const CUtensorMap& v,
                                 const CUtensorMap& q, int nqt, cudaStream_t s) {
  auto kern = paged_prefill_kernel<BF16, G>;
  static bool configured = false;   // one flag per instantiation
  if (!configured) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  AttnArgs b = a;
  b.max_parts = nqt;
  const int64_t grid = static_cast<int64_t>(a.num_seqs) * a.num_kv_heads * nqt;
  if (grid == 0) return cudaSuccess;
  kern<<<static_cast<unsigned>(grid), kPfThreads, kSmemBytes, s>>>(b, k, v, q);
  return cudaGetLastError();
}

template <bool BF16>
cudaError_t launch_prefill_g(const AttnArgs& a, const CUtensorMap& k, const CUtensorMap& v,
                             const CUtensorMap& q, int nqt, cudaStream_t s) {
  switch (a.group) {
    case 1: return launch_prefill_typed<BF16, 1>(a, k, v, q, nqt, s);
    case 2: return launch_prefill_typed<BF16, 2>(a, k, v, q, nqt, s);
    case 4: return launch_prefill_typed<BF16, 4>(a, k, v, q, nqt, s);
    case 8: return launch_prefill_typed<BF16, 8>(a, k, v, q, nqt, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool prefill_supported(int q_dtype, int kv_dtype, int32_t head_dim, int32_t group) {
  if (head_dim != 128) return false;
  if (!(kv_dtype == 0 || kv_dtype == 1) || q_dtype != kv_dtype) return false;
  return group == 1 || group == 2 || group == 4 || group == 8;
}

int prefill_query_tile(int32_t group) { return 128 / group; }

cudaError_t launch_paged_prefill(const AttnArgs& a, const CUtensorMap& kmap,
                                 const CUtensorMap& vmap, const CUtensorMap& qmap,
                                 int32_t max_q_len, cudaStream_t stream) {
  const int tq = 128 / a.group;
  const int nqt = (max_q_len + tq - 1) / tq;
  if (nqt <= 0) return cudaSuccess;
  return a.kv_dtype == 1 ? launch_prefill_g<true>(a, kmap, vmap, qmap, nqt, stream)
                         : launch_prefill_g<false>(a, kmap, vmap, qmap, nqt, stream);
}

}  // namespace pa
