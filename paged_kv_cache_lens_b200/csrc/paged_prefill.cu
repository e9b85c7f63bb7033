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
//                    bf16/f16 hi + lo halves back over the S columns it has read;
//   O += P V         tcgen05.mma with A = P straight from TMEM and B = V from
//                    shared memory (MN-major), D = O in TMEM.
// Softmax is online in one pass: P is taken against a running row maximum
// that is only raised (and O, l rescaled in TMEM / registers) when a tile's
// maximum exceeds it by more than 2^8, so P <= 256 and rescaling is rare.
// Warp roles: 8 softmax warps in two groups of four that take alternate key
// tiles (one thread per tile row, all 128 columns); a group passes the row
// maxima it used to the other through shared memory, so the exponentials of
// one group overlap the TMEM loads, maxima and stores of the other.  2 TMA
// producer warps (K and V; paged tiles gathered 16 tokens at a time), 1 warp
// that allocates TMEM and issues the MMAs (one lane elected per instruction).
// S/P live in three TMEM buffers: S runs up to two tiles ahead of PV.
#include "pa_device.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

constexpr int kSoftmaxWarps = 8;         // two groups of four: even and odd key tiles
constexpr int kSoftmaxThreads = kSoftmaxWarps * 32;
constexpr int kGroupThreads = kSoftmaxThreads / 2;
constexpr int kProducerWarps = 2;        // one streams K tiles, one V tiles
constexpr int kProducerWarp0 = 8;
constexpr int kMmaWarp = kProducerWarp0 + kProducerWarps;
constexpr int kPfThreads = (kMmaWarp + 1) * 32;
constexpr int kBN = 128;                 // keys per tile
constexpr int kHalf = 128 * 128;         // one 64-column (128-byte) half of a 128-row tile
constexpr int kQBytes = 2 * kHalf;
constexpr int kTileBytes = 2 * kHalf;    // one K or V tile: 128 keys x 128 dims
constexpr int kKStages = 3;              // K is freed as soon as S is computed
constexpr int kVStages = 2;              // V is freed when PV has run
constexpr int kSBufs = 3;                // S/P buffers in TMEM
constexpr int kKOff = kQBytes;
constexpr int kVOff = kKOff + kKStages * kTileBytes;
constexpr int kTblMax = 2048;            // block-table entries cached in shared memory
constexpr int kTblOff = kVOff + kVStages * kTileBytes;
constexpr int kRedOff = kTblOff + kTblMax * 4;   // [2 slots][128] maxima, [2 groups][128] sums
constexpr int kBarBase = kRedOff + 4 * 128 * 4;
constexpr float kRescaleGap = 8.f;       // raise the running max when exceeded by 2^8
// barriers: Q | K full x3 | K empty x3 | V full x2 | V empty x2 | S full x3 | P full x3 |
//           PV done x3 | O | row maxima published [2 slots][4 lane quarters]
enum { B_Q = 0, B_KF = 1, B_KE = 4, B_VF = 7, B_VE = 9, B_SF = 11, B_PF = 14, B_PVD = 17,
       B_O = 20, B_MX = 21, kNumBars = 29 };
constexpr int kSmemBytes = kBarBase + kNumBars * 8 + 16 + 1024;
constexpr uint32_t kTmemCols = 512;      // S/P buffers at columns 0, 128, 256; O at 384
constexpr uint32_t kOCol = 384;
constexpr uint32_t kWaitLimit = 1u << 20;
constexpr float kLog2eF = 1.4426950408889634f;

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
  int32_t* tbl = reinterpret_cast<int32_t*>(smem + kTblOff);
  float* red = reinterpret_cast<float*>(smem + kRedOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarBase);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarBase + kNumBars * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item from the compact list: (request, query tile) x KV head
  const int item = blockIdx.x / a.num_kv_heads;
  const int h = blockIdx.x - item * a.num_kv_heads;
  if (item >= *a.pf_count) return;
  const int2 rq = a.pf_items[item];
  const int r = rq.x, qt = rq.y;
  const int cu0 = a.cu_seqlens_q[r];
  const int q_len = a.cu_seqlens_q[r + 1] - cu0;
  const int kv_len = min(a.seqlens_k[r], a.max_context_len);
  const int rows_valid = min(TQ, q_len - qt * TQ);
  const int pos0 = kv_len - q_len + qt * TQ;        // absolute position of tile row 0
  const int last_pos = pos0 + rows_valid - 1;
  if (rows_valid <= 0 || last_pos < 0) return;
  const int nkv = last_pos / kBN + 1;
  // sliding window: key tiles before the first key any row of the tile sees
  // are skipped (tiles jlo .. nkv-1 are visited, ntile of them)
  const int jlo = a.window > 0 ? max(0, pos0 - a.window + 1) / kBN : 0;
  const int ntile = nkv - jlo;
  const int n_iter = ntile;
  const int hq0 = h * G;

  if (threadIdx.x == 0) {
    mbar_init(&bars[B_Q], 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bars[B_KF + s], 1);
      mbar_init(&bars[B_KE + s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bars[B_VF + s], 1);
      mbar_init(&bars[B_VE + s], 1);
    }
    for (int s = 0; s < kSBufs; ++s) {
      mbar_init(&bars[B_SF + s], 1);
      mbar_init(&bars[B_PF + s], kGroupThreads);
      mbar_init(&bars[B_PVD + s], 1);
    }
    mbar_init(&bars[B_O], 1);
    for (int s = 0; s < 8; ++s) mbar_init(&bars[B_MX + s], 32);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= kProducerWarp0 && warp < kMmaWarp) {
    // ================================================================ TMA producers
    // One warp streams K tiles, one V tiles.  Lane 0 waits for a free stage
    // and arms its barrier with the tile's bytes; lanes 0-7 then each fetch
    // one 16-key sub-tile (both 64-column halves) through the block table.
    const int pw = warp - kProducerWarp0;
    const bool is_v = pw == 1;
    const int32_t* bt = a.block_tables + static_cast<int64_t>(r) * a.max_blocks_per_seq;
    const int bs = a.block_size;
    const int nblk = last_pos / bs + 1;               // blocks holding visible keys
    const int ncache = min(nblk, kTblMax);
    for (int i = pw * 32 + lane; i < ncache; i += kProducerWarps * 32) tbl[i] = __ldg(bt + i);
    named_bar(2, kProducerWarps * 32);
    const int oob_row = a.num_blocks * a.num_kv_heads * bs;
    if (pw == 0 && lane == 0) {
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&vmap);
      mbar_arrive_expect_tx(&bars[B_Q], kQBytes);
      tma_load_3d(sQ, &qmap, 0, hq0, cu0 + qt * TQ, &bars[B_Q]);
      tma_load_3d(sQ + kHalf, &qmap, 64, hq0, cu0 + qt * TQ, &bars[B_Q]);
    }
    const uint64_t pol = l2_policy_evict_last();
    const int nstage = is_v ? kVStages : kKStages;
    uint64_t* full = &bars[is_v ? B_VF : B_KF];
    uint64_t* empty = &bars[is_v ? B_VE : B_KE];
    const CUtensorMap* map = is_v ? &vmap : &kmap;
    uint8_t* ring = smem + (is_v ? kVOff : kKOff);
    int issued = 0;
    for (int u = 0; u < ntile; ++u) {
      const int j = jlo + u;                              // key tile
      const int st = u % nstage;
      int go = 1;
      if (lane == 0) {
        go = !*abort_flag;
        if (go && u >= nstage) go = wait_or_abort(&empty[st], (u / nstage - 1) & 1, abort_flag);
        if (go) mbar_arrive_expect_tx(&full[st], kTileBytes);
      }
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
      if (lane < 8) {
        // sub-tile `lane` of key tile j: one box of 16 rows (two of 8 rows
        // for 8-token blocks); past the visible keys the box starts past the
        // pool and is zero filled
        const int sti = j * 8 + lane;
        int y0 = oob_row, y1 = bs == 8 ? oob_row : -1;
        if (sti * 16 <= last_pos) {
          const int32_t* src = (sti + 1) * 16 / bs + 1 < kTblMax ? tbl : bt;
          int r0, r1;
          if (tile_rows(src, sti, bs, nblk, a.num_blocks, a.num_kv_heads, h, oob_row, r0, r1)) {
            y0 = r0;
            y1 = r1;
          } else {
            report_error(kErrBlockRange);
          }
        }
        uint8_t* box = ring + st * kTileBytes + lane * 2048;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          tma_load_2d(box + half * kHalf, map, half * 64, y0, &full[st], pol);
          if (y1 >= 0) tma_load_2d(box + half * kHalf + 1024, map, half * 64, y1, &full[st], pol);
        }
      }
      issued = u + 1;
    }
    // the last copies into each stage have landed before the CTA may exit
    if (lane == 0) {
      for (int u = issued - 1; u >= 0 && u >= issued - nstage; --u)
        (void)mbar_wait_bounded(&full[u % nstage], (u / nstage) & 1);
      if (pw == 0) (void)mbar_wait_bounded(&bars[B_Q], 0);
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    // The whole warp runs this loop converged (every wait is taken by all
    // lanes, and agreed on); one elected lane issues each MMA and commit.
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, wait_or_abort(bar, parity, abort_flag));
    };
    bool ok = wait_all(&bars[B_Q], 0);
    // descriptors of the first 16-column slice of Q, K stage 0 and V stage 0;
    // a slice or stage is an offset added to the start-address field (byte
    // address / 16, which stays below 2^14 for any shared-memory address)
    const uint64_t q_desc = smem_desc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t k_desc = smem_desc_sw128(smem_u32(smem + kKOff), 16, 1024);
    const uint64_t v_desc = smem_desc_sw128(smem_u32(smem + kVOff), kHalf, 1024);
    int next_s = 0;
    for (int it = 0; ok && it < n_iter; ++it) {
      // S runs up to two tiles ahead of PV, so both softmax groups have a
      // tile to work on; buffer reuse waits for PV(next_s - 3) only
      while (ok && next_s < n_iter && next_s <= it + 2) {
        const int sb = next_s % kSBufs;
        if (next_s >= kSBufs && !(ok = wait_all(&bars[B_PVD + sb], (next_s / kSBufs - 1) & 1)))
          break;
        const int ks = next_s % kKStages;
        if (!(ok = wait_all(&bars[B_KF + ks], (next_s / kKStages) & 1))) break;
        tc_fence_after();
        const uint64_t kd = k_desc + static_cast<uint64_t>((ks * kTileBytes) >> 4);
        const uint32_t d = tmem + static_cast<uint32_t>(sb * 128);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kHalf + (kk & 3) * 32) >> 4);
          tc_mma_ss_warp(d, q_desc + off, kd + off, kIdescS, kk > 0 ? 1u : 0u);
        }
        tc_commit_warp(&bars[B_SF + sb]);
        tc_commit_warp(&bars[B_KE + ks]);       // S is the only reader of K
        ++next_s;
      }
      if (!ok) break;
      // O += P V once the softmax group has written P(it) (and rescaled O)
      const int b = it % kSBufs;
      if (!(ok = wait_all(&bars[B_PF + b], (it / kSBufs) & 1))) break;
      const int vs = it % kVStages;
      if (!(ok = wait_all(&bars[B_VF + vs], (it / kVStages) & 1))) break;
      tc_fence_after();
      const uint64_t vd = v_desc + static_cast<uint64_t>((vs * kTileBytes) >> 4);
      const uint32_t p_base = tmem + static_cast<uint32_t>(b * 128);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        // keys 16kk .. 16kk+15: chunk kk/2 of 32 keys holds 16 hi columns
        // then 16 lo columns, 8 columns (16 packed values) per half chunk
        const uint32_t pc = p_base + 32 * (kk >> 1) + 8 * (kk & 1);
        const uint64_t vk = vd + static_cast<uint64_t>((kk * 2048) >> 4);
        tc_mma_ts_warp(tmem + kOCol, pc, vk, kIdescPV, (it == 0 && kk == 0) ? 0u : 1u);
        tc_mma_ts_warp(tmem + kOCol, pc + 16, vk, kIdescPV, 1u);
      }
      tc_commit_warp(&bars[B_VE + vs]);
      tc_commit_warp(&bars[B_PVD + b]);
    }
    tc_commit_warp(&bars[B_O]);              // every MMA issued above is complete
    if (!ok) (void)wait_all(&bars[B_O], 0);
  } else {
    // ================================================================ softmax / epilogue
    // Group grp (warps 4*grp ..) takes key tiles grp, grp + 2, ...; warp w's
    // 32 threads own tile rows (= TMEM lanes) 32*(w%4).., all 128 columns.
    const int quarter = warp & 3, grp = warp >> 2;
    const int t = quarter * 32 + lane;         // tile row == TMEM lane
    const int i = t / G, g = t % G;
    const bool row_ok = i < rows_valid;
    const int pos = pos0 + i;
    const float c = a.scale * kLog2eF;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    bool ok = true;
    // Row visibility: keys lo_row .. pos (lo_row from the sliding window);
    // logits in the log2 domain x = s*scale*log2e + slope*log2e*(key - pos).
    const int lo_row = a.window > 0 ? pos - a.window + 1 : 0;
    const float slope = a.alibi ? a.alibi[hq0 + g] * kLog2eF : 0.f;
    // without ALiBi (and with scale > 0) the max is taken on the raw scores
    // and the scale folds into the exponent's FFMA
    const bool direct = a.alibi == nullptr && c > 0.f;
    const float cc = direct ? c : 1.f;
    // a tile every row sees in full needs no mask
    auto tile_full = [&](int j) {
      return j * kBN + kBN - 1 <= pos0 && (a.window <= 0 || j * kBN >= last_pos - a.window + 1);
    };
    // 32 columns of S (column0 = k0 .. k0 + 31 of the tile) -> logits in place
    auto logits = [&](uint32_t (&v)[32], int col0, int nlo, int nhi, bool full, float b0) {
      if (!direct) {
#pragma unroll
        for (int n = 0; n < 32; ++n)
          v[n] = __float_as_uint(
              fmaf(__uint_as_float(v[n]), c, fmaf(slope, static_cast<float>(col0 + n), b0)));
      }
      if (!full) {
#pragma unroll
        for (int n = 0; n < 32; ++n)
          if (col0 + n < nlo || col0 + n > nhi) v[n] = __float_as_uint(-INFINITY);
      }
    };
    float* m_pub = red;                        // [slot = tile & 1][row]: maximum used
    float l_part = 0.f;                        // this group's share of the row sum,
    float m_l = -INFINITY;                     // relative to 2^m_l
    for (int it = grp; ok && it < n_iter; it += 2) {
      const int b = it % kSBufs;
      if (!wait_or_abort(&bars[B_SF + b], (it / kSBufs) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const int j = jlo + it;
      const int key0 = j * kBN;
      const bool full = tile_full(j);
      // keys outside lo_row .. pos of this row (every key of a padding row)
      // are masked; stale slots past kv_len always fall in a masked tile
      const int nlo = full ? 0 : (row_ok ? lo_row - key0 : kBN);
      const int nhi = full ? kBN - 1 : (row_ok ? pos - key0 : -1);
      const float b0 = slope * static_cast<float>(key0 - pos);
      const uint32_t s_col = lane_base + b * 128;
      // ---- the row of S (128 columns) in registers, one TMEM round trip;
      // the tile's row maximum (log2 domain) in four independent chains
      uint32_t v[4][32];
#pragma unroll
      for (int k = 0; k < 4; ++k) tmem_ld32(s_col + 32 * k, v[k]);
      tmem_wait_ld();
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        logits(v[k], 32 * k, nlo, nhi, full, b0);
#pragma unroll
        for (int n2 = 0; n2 < 16; ++n2)
          m4[n2 & 3] = fmax3(m4[n2 & 3], __uint_as_float(v[k][2 * n2]), __uint_as_float(v[k][2 * n2 + 1]));
      }
      float m_tile = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      if (direct) m_tile *= c;                 // scale > 0: the maximum commutes with it
      // ---- the running maximum before this tile, from the group that ran
      // tile it - 1; raise it only when this tile exceeds it by 2^8
      float m_prev = -INFINITY;
      if (it > 0) {
        const int sp = (it - 1) & 1;
        if (!wait_or_abort(&bars[B_MX + 4 * sp + quarter], ((it - 1) >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        m_prev = m_pub[sp * 128 + t];
      }
      const bool raise = (m_prev == -INFINITY) ? (m_tile != -INFINITY)
                                               : (m_tile > m_prev + kRescaleGap);
      const float m_new = raise ? m_tile : m_prev;
      m_pub[(it & 1) * 128 + t] = m_new;
      mbar_arrive(&bars[B_MX + 4 * (it & 1) + quarter]);
      if (m_new != m_l) {                      // rescale this group's partial sum
        l_part = (m_l == -INFINITY) ? 0.f : l_part * fast_exp2(m_l - m_new);
        m_l = m_new;
      }
      // ---- p = 2^(x - m_new) per 32-column chunk, written back over the
      // chunk's S columns as 16 hi then 16 lo columns of packed pairs
      const float nmu = (m_new == -INFINITY) ? 0.f : -m_new;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int n2 = 0; n2 < 16; ++n2) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(v[k][2 * n2]), cc, nmu));   // 2^-inf = 0
          const float p1 = fast_exp2(fmaf(__uint_as_float(v[k][2 * n2 + 1]), cc, nmu));
          ls[n2 & 3] += p0 + p1;
          const uint32_t hw = pack2<BF16>(p0, p1);
          hi[n2] = hw;
          lo[n2] = pack2<BF16>(p0 - lo_half_to_float<BF16>(hw), p1 - lo_half_to_float<BF16>(hw >> 16));
        }
        tmem_st16(s_col + 32 * k, hi);
        tmem_st16(s_col + 32 * k + 16, lo);
      }
      l_part += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      if (it > 0 && __any_sync(0xffffffffu, raise)) {
        // O holds PV of tiles < it: wait for PV(it - 1), then scale the rows
        // that raised their maximum (alpha = 1 elsewhere, 0 for a row whose
        // earlier keys were all masked)
        const float alpha = !raise ? 1.f : (m_prev == -INFINITY ? 0.f : fast_exp2(m_prev - m_new));
        if (!wait_or_abort(&bars[B_PVD + (it - 1) % kSBufs], ((it - 1) / kSBufs) & 1,
                           abort_flag)) {
          ok = false;
        }
        tc_fence_after();
#pragma unroll 1
        for (int q2 = 0; q2 < 4; ++q2) {
          uint32_t o[32];
          tmem_ld32(lane_base + kOCol + 32 * q2, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(lane_base + kOCol + 32 * q2, o);
        }
      }
      // Keys of the context's partial last block that lie past kv_len hold
      // whatever the slot held; P is 0 there but 0 * NaN is NaN: clear them.
      const int stale0 = kv_len, stale1 = min((kv_len + 15) & ~15, key0 + kBN);
      if (stale0 < stale1 && stale0 >= key0) {
        const int vs = it % kVStages;
        if (wait_or_abort(&bars[B_VF + vs], (it / kVStages) & 1, abort_flag)) {
          uint8_t* sV = smem + kVOff + vs * kTileBytes;
          const int nrows = stale1 - stale0;
          for (int idx = t; idx < nrows * 16; idx += kGroupThreads) {
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
    // -------- epilogue: O row / l -> out (group grp writes dims 64*grp ..)
    named_bar(1, kSoftmaxThreads);             // every tile's maximum is published
    const float m_fin = n_iter > 0 ? m_pub[((n_iter - 1) & 1) * 128 + t] : -INFINITY;
    red[256 + grp * 128 + t] =
        (m_l == -INFINITY || m_fin == -INFINITY) ? 0.f : l_part * fast_exp2(m_l - m_fin);
    named_bar(1, kSoftmaxThreads);
    const float l_row = red[256 + t] + red[384 + t];
    const float inv_l = l_row > 0.f ? 1.f / l_row : 0.f;
    const int half = grp;
    if (ok && wait_or_abort(&bars[B_O], 0, abort_flag)) {
      tc_fence_after();
      uint32_t o[64];
      tmem_ld32(lane_base + kOCol + half * 64, *reinterpret_cast<uint32_t (*)[32]>(o));
      tmem_ld32(lane_base + kOCol + half * 64 + 32, *reinterpret_cast<uint32_t (*)[32]>(o + 32));
      tmem_wait_ld();
      if (row_ok) {
        const int64_t orow =
            (static_cast<int64_t>(cu0 + qt * TQ + i) * a.num_q_heads + hq0 + g) * 128 + half * 64;
        if (a.out_dtype == 3) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow);
#pragma unroll
          for (int k = 0; k < 16; ++k)
            dst[k] = make_float4(__uint_as_float(o[4 * k]) * inv_l,
                                 __uint_as_float(o[4 * k + 1]) * inv_l,
                                 __uint_as_float(o[4 * k + 2]) * inv_l,
                                 __uint_as_float(o[4 * k + 3]) * inv_l);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + orow);
          const bool ob = (a.out_dtype == 1);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = __uint_as_float(o[8 * k + 2 * e]) * inv_l;
              const float x1 = __uint_as_float(o[8 * k + 2 * e + 1]) * inv_l;
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
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Compact list of (request, query tile) items of the q_len >= 2 requests,
// ordered by the number of key tiles each visits, most first (longest
// processing time first: the heavy CTAs start in the first wave instead of
// forming the grid's tail).  One CTA: a histogram of item weights in shared
// memory, a descending exclusive scan over it, then each item takes a slot in
// its weight's range (order within one weight is arbitrary; every item
// writes its own output rows, so the result does not depend on it).
constexpr int kItemThreads = 1024;
constexpr int kWeightBuckets = 4096;     // weights past the last bucket share it

__device__ __forceinline__ int item_weight(const int32_t* cu, const int32_t* seqlens_k,
                                           int32_t max_context_len, int32_t window, int tq,
                                           int r, int qt) {
  const int q_len = cu[r + 1] - cu[r];
  const int kv_len = min(seqlens_k[r], max_context_len);
  const int rows = min(tq, q_len - qt * tq);
  const int pos0 = kv_len - q_len + qt * tq;
  const int last = pos0 + rows - 1;
  if (rows <= 0 || last < 0) return 0;
  const int jlo = window > 0 ? max(0, pos0 - window + 1) / kBN : 0;
  return min(last / kBN + 1 - jlo, kWeightBuckets - 1);
}

__global__ void __launch_bounds__(kItemThreads)
prefill_items_kernel(int32_t num_seqs, const int32_t* cu, const int32_t* seqlens_k,
                     int32_t max_context_len, int32_t window, int tq, int2* items,
                     int32_t* count, int32_t capacity) {
  __shared__ int s_hist[kWeightBuckets];
  __shared__ int s_part[kItemThreads];
  for (int i = threadIdx.x; i < kWeightBuckets; i += kItemThreads) s_hist[i] = 0;
  __syncthreads();
  // ---- histogram of item weights
  for (int r = threadIdx.x; r < num_seqs; r += kItemThreads) {
    const int ql = cu[r + 1] - cu[r];
    if (ql < 2) continue;
    for (int qt = 0; qt < (ql + tq - 1) / tq; ++qt)
      atomicAdd(&s_hist[item_weight(cu, seqlens_k, max_context_len, window, tq, r, qt)], 1);
  }
  __syncthreads();
  // ---- descending exclusive scan: bucket w starts after every heavier item.
  // Thread t owns buckets kWeightBuckets-1-4t .. -3 (4 per thread, heaviest first).
  constexpr int kPer = kWeightBuckets / kItemThreads;
  int mine[kPer], sum = 0;
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    mine[k] = s_hist[kWeightBuckets - 1 - (kPer * threadIdx.x + k)];
    sum += mine[k];
  }
  s_part[threadIdx.x] = sum;
  __syncthreads();
  for (int off = 1; off < kItemThreads; off <<= 1) {      // inclusive Hillis-Steele scan
    const int v = threadIdx.x >= off ? s_part[threadIdx.x - off] : 0;
    __syncthreads();
    s_part[threadIdx.x] += v;
    __syncthreads();
  }
  int base = s_part[threadIdx.x] - sum;
  const int total = s_part[kItemThreads - 1];
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    s_hist[kWeightBuckets - 1 - (kPer * threadIdx.x + k)] = base;   // next free slot
    base += mine[k];
  }
  __syncthreads();
  // ---- scatter
  for (int r = threadIdx.x; r < num_seqs; r += kItemThreads) {
    const int ql = cu[r + 1] - cu[r];
    if (ql < 2) continue;
    for (int qt = 0; qt < (ql + tq - 1) / tq; ++qt) {
      const int slot =
          atomicAdd(&s_hist[item_weight(cu, seqlens_k, max_context_len, window, tq, r, qt)], 1);
      if (slot < capacity) items[slot] = make_int2(r, qt);
    }
  }
  if (threadIdx.x == 0) *count = min(total, capacity);
}

template <bool BF16, int G>
cudaError_t launch_prefill_typed(const AttnArgs& a, const CUtensorMap& k, const CUtensorMap& v,
                                 const CUtensorMap& q, int capacity, cudaStream_t s) {
  auto kern = paged_prefill_kernel<BF16, G>;
  const int64_t grid = static_cast<int64_t>(capacity) * a.num_kv_heads;
  if (grid == 0) return cudaSuccess;
  // the shared-memory limit is a per-device setting of the function: set it
  // for the current device on every launch (a host-side call)
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<static_cast<unsigned>(grid), kPfThreads, kSmemBytes, s>>>(a, k, v, q);
  return cudaGetLastError();
}

template <bool BF16>
cudaError_t launch_prefill_g(const AttnArgs& a, const CUtensorMap& k, const CUtensorMap& v,
                             const CUtensorMap& q, int capacity, cudaStream_t s) {
  switch (a.group) {
    case 1: return launch_prefill_typed<BF16, 1>(a, k, v, q, capacity, s);
    case 2: return launch_prefill_typed<BF16, 2>(a, k, v, q, capacity, s);
    case 4: return launch_prefill_typed<BF16, 4>(a, k, v, q, capacity, s);
    case 8: return launch_prefill_typed<BF16, 8>(a, k, v, q, capacity, s);
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

int32_t prefill_item_capacity(int32_t num_seqs, int32_t total_q) {
  // sum_r ceil(q_len_r / tq) over requests with q_len_r >= 2, tq >= 16
  return total_q / 16 + (num_seqs < total_q / 2 ? num_seqs : total_q / 2) + 1;
}

cudaError_t launch_paged_prefill(const AttnArgs& a, const CUtensorMap& kmap,
                                 const CUtensorMap& vmap, const CUtensorMap& qmap,
                                 int32_t capacity, cudaStream_t stream) {
  const int tq = 128 / a.group;
  prefill_items_kernel<<<1, kItemThreads, 0, stream>>>(
      a.num_seqs, a.cu_seqlens_q, a.seqlens_k, a.max_context_len, a.window, tq,
      const_cast<int2*>(a.pf_items), const_cast<int32_t*>(a.pf_count), capacity);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return a.kv_dtype == 1 ? launch_prefill_g<true>(a, kmap, vmap, qmap, capacity, stream)
                         : launch_prefill_g<false>(a, kmap, vmap, qmap, capacity, stream);
}

}  // namespace pa
