// Paged attention kernels for sm_100a: split-K decode over a block-paged KV
// cache, the log-sum-exp merge of partitions, and the row map of the packed
// varlen step.
//
// What is computed ("PagedAttention 与 Continuous Batching", §3.6
// PagedAttention Kernel): for each query row, walk the request's block table,
// fetch each 16-token physical block of K and V, and accumulate softmax(QK^T)V
// with a running max and sum (online softmax).  The per-row context is cut
// into partitions of partition_size tokens (one CTA each); partitions of one
// row are merged with M = max_p m_p, L = sum_p l_p 2^(m_p - M),
// out = sum_p 2^(m_p - M) o_p / L.
//
// How it maps onto the B200:
//   * one CTA = (query row, KV head, partition); its 4 warps take the
//     partition's blocks round-robin, each with a private online-softmax state
//     and a private ring of NSTAGE shared-memory stages;
//   * each block's K and V tiles ([16 tokens][D], contiguous in the pool) are
//     fetched by 2-D TMA loads (128-byte boxes, 128-byte swizzle) issued by one
//     lane, completion tracked by an mbarrier with a bounded wait;
//   * QK^T and PV run on the tensor cores as warp-level m16n8k16 MMAs with
//     the 16 tokens of a block as M and the GQA query-head group as N, so the
//     group shares every K/V tile it reads; P enters the PV product as a
//     hi + lo pair of 16-bit values (p = hi + lo to ~2^-17), which for groups
//     of up to 4 heads fills the otherwise idle half of the N = 8 columns;
//   * the running max is raised only when a block's maximum passes it by
//     more than 2^8 (so P <= 256): most blocks skip the rescale of O;
//   * FP8 E4M3 tiles are widened to f16 in registers (exact), the per-head
//     scales folded into the logit multiplier and the output; P is one f16
//     value there (the pools' 5e-2 bound).
#include "pa_device.cuh"
#include "pa_launch.h"

#include <cstdio>

namespace pa {

__device__ unsigned int g_error_word = 0;

namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kBlockTokens = 16;
constexpr int kMaxPartitionBlocks = 128;  // partition_size <= 1024 tokens, blocks >= 8 tokens
constexpr int kMaxGroup = 128;            // query heads per KV head
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazyRaise = 8.f;         // raise the running max when passed by 2^8

enum { KV_F16 = 0, KV_BF16 = 1, KV_FP8 = 2 };

template <int KVT, int D>
struct Geo {
  static constexpr int kElemBytes = (KVT == KV_FP8) ? 1 : 2;
  static constexpr int kRowBytes = D * kElemBytes;
  // rows of 128 bytes or more travel as 128-byte boxes with the 128-byte
  // swizzle; narrower rows (E4M3 at head_dim 64: 64 bytes) as one unswizzled box
  static constexpr bool kNarrow = kRowBytes < 128;
  static constexpr int kPitch = kNarrow ? kRowBytes : 128;   // bytes per box row
  static constexpr int kBoxBytes = kBlockTokens * kPitch;
  static constexpr int kBoxes = kRowBytes / kPitch;
  static constexpr int kBoxElems = kPitch / kElemBytes;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;
  static_assert(kRowBytes % kPitch == 0, "rows must be whole boxes");
  static_assert(!kNarrow || KVT == KV_FP8, "narrow rows only for E4M3 pools");
};

template <int KVT, int D, int GT, int NSTAGE>
struct Smem {
  using G = Geo<KVT, D>;
  static constexpr int kNT = GT / 4;                                  // PV n-tiles
  static constexpr int kTiles = kWarps * NSTAGE * 2 * G::kTileBytes;  // K,V rings
  static constexpr int kPT = kWarps * kNT * 8 * kBlockTokens * 2;      // P^T per warp
  static constexpr int kBars = kWarps * NSTAGE * 8;
  static constexpr int kTbl = kMaxPartitionBlocks * 4;
  static constexpr int kMerge = kWarps * (GT * D + 2 * GT) * 4;
  static_assert(kMerge <= kTiles, "merge area reuses the rings");
  static constexpr int kTotal = kTiles + kPT + kBars + kTbl + 1024;   // + alignment slack
};

__device__ __forceinline__ int swz(int row, int chunk) {  // 128-byte swizzle
  return row * 128 + ((chunk ^ (row & 7)) << 4);
}

// The sequence, visible-key count and packed query row behind work row `row`:
// decode (row = sequence), varlen rows mapped by the row-map kernel, or varlen
// requests with the chunk path on (row = request; only q_len-1 requests here,
// L = -1 marks the others, which the prefill kernel owns).
__device__ __forceinline__ void resolve_row(const AttnArgs& a, int row, int& seq, int& L,
                                            int& qrow) {
  if (a.row_seq) {
    seq = a.row_seq[row];
    L = a.row_len[row];
    qrow = row;
  } else if (a.varlen_requests) {
    seq = row;
    const int c0 = a.cu_seqlens_q[row];
    qrow = c0;
    L = (a.cu_seqlens_q[row + 1] - c0 == 1) ? a.seqlens_k[row] : -1;
  } else {
    seq = row;
    L = a.context_lens[row];
    qrow = row;
  }
}

template <int KVT, bool Q_BF16, int D, int GT, int NSTAGE>
__global__ void __launch_bounds__(kThreads)
paged_attn_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap kmap,
                  const __grid_constant__ CUtensorMap vmap) {
  constexpr bool kFP8 = (KVT == KV_FP8);
  constexpr bool kMmaBF16 = (KVT == KV_BF16);
  using G = Geo<KVT, D>;
  using S = Smem<KVT, D, GT, NSTAGE>;
  constexpr int kNT = S::kNT;
  constexpr int kNTPV = kFP8 ? 1 : kNT;   // n-tiles holding P (E4M3 pools: hi only)
  constexpr int kKSteps = D / 16;
  constexpr int kMTiles = D / 16;
  constexpr int kTB = G::kTileBytes;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  uint16_t* pt_all = reinterpret_cast<uint16_t*>(smem + S::kTiles);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kTiles + S::kPT);
  int32_t* tbl = reinterpret_cast<int32_t*>(smem + S::kTiles + S::kPT + S::kBars);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int r = lane >> 2;
  const int c = lane & 3;

  // ---- work item: (row, kv head, partition, chunk of at most 8 query heads);
  // the chunks of one (row, head, partition) are adjacent blocks, so a group
  // larger than 8 reads each K/V tile from HBM once and from L2 after that
  int64_t bid = blockIdx.x;
  const int chunk = static_cast<int>(bid % a.head_chunks);
  bid /= a.head_chunks;
  const int part = static_cast<int>(bid % a.max_parts);
  bid /= a.max_parts;
  const int h = static_cast<int>(bid % a.num_kv_heads);
  const int row = static_cast<int>(bid / a.num_kv_heads);
  int seq, L, qrow;
  resolve_row(a, row, seq, L, qrow);
  if (L < 0) return;               // a varlen row owned by the prefill kernel
  if (L > a.max_context_len) {     // a row longer than the promised bound is cut there
    if (part == 0 && h == 0 && threadIdx.x == 0) report_error(kErrLenRange);
    L = a.max_context_len;
  }
  const int group = min(a.group - chunk * GT, GT);   // query heads of this chunk
  const int hq0 = h * a.group + chunk * GT;
  const int Hq = a.num_q_heads;
  if (L <= 0) {
    if (part == 0)
      for (int i = threadIdx.x; i < group * D; i += kThreads)
        store_out(a.out, (static_cast<int64_t>(qrow) * Hq + hq0) * D + i, a.out_dtype, 0.f);
    return;
  }
  const int PS = a.partition_size;
  const int nparts = (L + PS - 1) / PS;
  if (part >= nparts) return;
  const int tok0 = part * PS;
  const int ntok = min(PS, L - tok0);
  // sliding window: visible keys are lo .. L-1 (the query sits at L-1)
  const int lo = a.window > 0 ? max(0, L - a.window) : 0;
  const int t_lo = max(0, lo - tok0);                  // first visible token of the partition
  const int first_tile = t_lo / kBlockTokens;
  const int nblk = (ntok + kBlockTokens - 1) / kBlockTokens;   // 16-token tiles
  const int bs = a.block_size;
  const int npblk = (ntok + bs - 1) / bs;                          // pool blocks

  const int32_t* bt = a.block_tables + static_cast<int64_t>(seq) * a.max_blocks_per_seq +
                      tok0 / bs;
  for (int i = threadIdx.x; i < npblk; i += kThreads) tbl[i] = bt[i];
  if constexpr (kFP8) {
    // one f16 P: the lo columns of P^T are never written and stay zero
    uint32_t* z = reinterpret_cast<uint32_t*>(pt_all);
    for (int i = threadIdx.x; i < S::kPT / 4; i += kThreads) z[i] = 0;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kWarps * NSTAGE; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
  }
  __syncthreads();

  // ---- per-warp pipeline
  uint8_t* wt = tiles + warp * NSTAGE * 2 * kTB;
  uint64_t* wb = bars + warp * NSTAGE;
  uint16_t* pt = pt_all + warp * kNT * 8 * kBlockTokens;
  const int ntiles = nblk - first_tile;                // tiles holding visible keys
  const int my_blocks = ntiles > warp ? (ntiles - warp + kWarps - 1) / kWarps : 0;
  const uint64_t policy = l2_policy_evict_first();
  const int num_blocks = a.num_blocks;

  const int oob_row = num_blocks * a.num_kv_heads * bs;
  auto issue = [&](int k) {
    const int i = first_tile + warp + k * kWarps;
    const int s = k % NSTAGE;
    uint64_t* bar = wb + s;
    int y0, y1;
    if (!tile_rows(tbl, i, bs, npblk, num_blocks, a.num_kv_heads, h, oob_row, y0, y1)) {
      report_error(kErrBlockRange);
      mbar_arrive(bar);
      return;
    }
    mbar_arrive_expect_tx(bar, 2 * kTB);
    uint8_t* kt = wt + s * 2 * kTB;
#pragma unroll
    for (int b = 0; b < G::kBoxes; ++b) {
      tma_load_2d(kt + b * G::kBoxBytes, &kmap, b * G::kBoxElems, y0, bar, policy);
      tma_load_2d(kt + kTB + b * G::kBoxBytes, &vmap, b * G::kBoxElems, y0, bar, policy);
      if (y1 >= 0) {          // 8-token blocks: rows 8..15 of the tile from the next block
        tma_load_2d(kt + b * G::kBoxBytes + 8 * G::kPitch, &kmap, b * G::kBoxElems, y1, bar,
                    policy);
        tma_load_2d(kt + kTB + b * G::kBoxBytes + 8 * G::kPitch, &vmap, b * G::kBoxElems, y1,
                    bar, policy);
      }
    }
  };
  if (lane == 0)
    for (int k = 0; k < NSTAGE && k < my_blocks; ++k) issue(k);

  // ---- Q as the B operand of QK^T: column n = lane/4 is head hq0 + n
  uint32_t qf[kKSteps][2];
  {
    const int n = r;
    const bool live = n < group && n < GT;
    const uint16_t* qptr = static_cast<const uint16_t*>(a.q) +
                           (static_cast<int64_t>(qrow) * Hq + hq0 + (live ? n : 0)) * D;
    if constexpr (!kFP8) {
#pragma unroll
      for (int p = 0; p < D / 32; ++p) {
        const int base = (p >> 1) * 64 + 8 * (2 * c + (p & 1));
        uint4 w = live ? *reinterpret_cast<const uint4*>(qptr + base) : make_uint4(0, 0, 0, 0);
        qf[2 * p][0] = w.x;
        qf[2 * p][1] = w.y;
        qf[2 * p + 1][0] = w.z;
        qf[2 * p + 1][1] = w.w;
      }
    } else {
#pragma unroll
      for (int p = 0; p < D / 64; ++p) {
        const int base = G::kNarrow ? 16 * c : (p >> 1) * 128 + 16 * (2 * c + (p & 1));
        uint4 w0 = make_uint4(0, 0, 0, 0), w1 = w0;
        if (live) {
          w0 = *reinterpret_cast<const uint4*>(qptr + base);
          w1 = *reinterpret_cast<const uint4*>(qptr + base + 8);
        }
        uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          uint32_t lo = wv[2 * hh], hi = wv[2 * hh + 1];
          if constexpr (Q_BF16) {
            lo = bf16x2_to_f16x2(lo);
            hi = bf16x2_to_f16x2(hi);
          }
          qf[4 * p + hh][0] = lo;
          qf[4 * p + hh][1] = hi;
        }
      }
    }
  }

  float qk_mul = a.scale * kLog2e;
  float v_mul = 1.f;
  if constexpr (kFP8) {
    qk_mul *= a.k_scale[h];
    v_mul = a.v_scale[h];
  }
  // ALiBi slopes of this lane's two score columns (query heads hq0 + 2c + j),
  // in the log2 domain; the bias of key t is slope * (t - (L - 1))
  float alibi[2] = {0.f, 0.f};
  if (a.alibi) {
#pragma unroll
    for (int j = 0; j < 2; ++j)
      if (2 * c + j < group && 2 * c + j < GT) alibi[j] = a.alibi[hq0 + 2 * c + j] * kLog2e;
  }
  const int key_base = tok0 - (L - 1);                 // key position - query position

  // ---- online-softmax state (columns 2c, 2c+1 of this lane) and output
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  float acc[kNT][kMTiles][4];
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
    for (int mt = 0; mt < kMTiles; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][mt][e] = 0.f;

  bool dead = false;
  int k = 0;
  for (; k < my_blocks; ++k) {
    const int i = first_tile + warp + k * kWarps;
    const int s = k % NSTAGE;
    const uint32_t parity = (k / NSTAGE) & 1;
    bool ok = mbar_wait_bounded(wb + s, parity);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) {
      if (lane == 0) report_error(kErrTimeout);
      dead = true;
      break;
    }
    int y0_, y1_;
    const bool valid_blk =
        tile_rows(tbl, i, bs, npblk, num_blocks, a.num_kv_heads, h, oob_row, y0_, y1_);
    const int valid = valid_blk ? min(kBlockTokens, ntok - i * kBlockTokens) : 0;
    const uint8_t* kt = wt + s * 2 * kTB;
    const uint8_t* vt = kt + kTB;
    const uint32_t kt_s = smem_u32(kt), vt_s = smem_u32(vt);

    if (valid > 0 && valid < kBlockTokens) {
      // Rows past the context may hold anything (stale or never-written
      // slots); P is 0 there but 0 * NaN is NaN, so clear those V rows.
      uint8_t* vz = wt + s * 2 * kTB + kTB;
      const int dead_rows = kBlockTokens - valid;
      constexpr int kChunks = G::kPitch / 16;               // 16-byte chunks per box row
      for (int idx = lane; idx < dead_rows * G::kBoxes * kChunks; idx += 32) {
        const int chunk = idx % kChunks;
        const int rb = idx / kChunks;
        const int box = rb / dead_rows;
        const int rw = valid + (rb - box * dead_rows);
        *reinterpret_cast<uint4*>(vz + box * G::kBoxBytes + rw * G::kPitch + chunk * 16) =
            make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();   // order these writes before the next TMA into the stage
      __syncwarp();
    }
    if (valid > 0) {
      // ---- S^T = K Q^T : [16 tokens] x [8 heads]
      float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      if constexpr (!kFP8) {
#pragma unroll
        for (int p = 0; p < D / 32; ++p) {
          const int box = p >> 1;
          const int ch = 2 * c + (p & 1);
          const uint4 R0 = lds128(kt_s + box * G::kBoxBytes + swz(r, ch));
          const uint4 R8 = lds128(kt_s + box * G::kBoxBytes + swz(r + 8, ch));
          mma16816<kMmaBF16>(sacc[0], R0.x, R8.x, R0.y, R8.y, qf[2 * p][0], qf[2 * p][1]);
          mma16816<kMmaBF16>(sacc[1], R0.z, R8.z, R0.w, R8.w, qf[2 * p + 1][0],
                             qf[2 * p + 1][1]);
        }
      } else {
#pragma unroll
        for (int p = 0; p < D / 64; ++p) {
          const int box = p >> 1;
          const int ch = 2 * c + (p & 1);
          const uint4 R0 = G::kNarrow ? lds128(kt_s + r * G::kPitch + 16 * c)
                                      : lds128(kt_s + box * G::kBoxBytes + swz(r, ch));
          const uint4 R8 = G::kNarrow ? lds128(kt_s + (r + 8) * G::kPitch + 16 * c)
                                      : lds128(kt_s + box * G::kBoxBytes + swz(r + 8, ch));
          const uint32_t w0[4] = {R0.x, R0.y, R0.z, R0.w};
          const uint32_t w8[4] = {R8.x, R8.y, R8.z, R8.w};
#pragma unroll
          for (int hh = 0; hh < 4; ++hh) {
            mma16816<false>(sacc[hh & 1], e4m3x2_to_f16x2(w0[hh]), e4m3x2_to_f16x2(w8[hh]),
                            e4m3x2_to_f16x2(w0[hh] >> 16), e4m3x2_to_f16x2(w8[hh] >> 16),
                            qf[4 * p + hh][0], qf[4 * p + hh][1]);
          }
        }
      }
      // s[0]:(t=r,col 2c) s[1]:(r,2c+1) s[2]:(r+8,2c) s[3]:(r+8,2c+1), log2 domain
      float sv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = r + ((e >> 1) << 3);
        const int trel = i * kBlockTokens + t;         // token within the partition
        sv[e] = (t < valid && trel >= t_lo)
                    ? (sacc[0][e] + sacc[1][e]) * qk_mul +
                          alibi[e & 1] * static_cast<float>(key_base + trel)
                    : -INFINITY;
      }
      // the running max is raised (and O, l rescaled) only when a block's
      // maximum passes it by more than 2^8, so P <= 256 and most blocks skip
      // the rescale (the decision is warp-uniform)
      float bmx[2];
      bool need = false;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float bm = fmaxf(sv[j], sv[j + 2]);
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
        bmx[j] = bm;
        need |= bm > m_run[j] + kLazyRaise;
      }
      const bool raise = __any_sync(0xffffffffu, need);
      float alpha[2] = {1.f, 1.f}, pv[4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        if (raise) {
          const float m_new = fmaxf(m_run[j], bmx[j]);
          alpha[j] = fast_exp2(m_run[j] - ((m_new == -INFINITY) ? 0.f : m_new));
          m_run[j] = m_new;
        }
        const float m_use = (m_run[j] == -INFINITY) ? 0.f : m_run[j];
        pv[j] = fast_exp2(sv[j] - m_use);
        pv[j + 2] = fast_exp2(sv[j + 2] - m_use);
        l_run[j] = l_run[j] * alpha[j] + pv[j] + pv[j + 2];
      }
      // ---- P^T (hi, lo) to shared memory: pt[col][token].  E4M3 pools
      // (5e-2 bound) take one f16 P; their lo columns stay zero.
      const bool writer = (kNT == 2) || (c < 2);
      if (writer) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = r + ((e >> 1) << 3);
          const int col = 2 * c + (e & 1);
          const float p = pv[e];
          if constexpr (kFP8) {
            pt[col * kBlockTokens + t] = __half_as_ushort(__float2half_rn(p));
          } else {
            uint16_t hi, lo;
            if constexpr (kMmaBF16) {
              const __nv_bfloat16 hb = __float2bfloat16_rn(p);
              hi = __bfloat16_as_ushort(hb);
              lo = __bfloat16_as_ushort(__float2bfloat16_rn(p - __bfloat162float(hb)));
            } else {
              const __half hh = __float2half_rn(p);
              hi = __half_as_ushort(hh);
              lo = __half_as_ushort(__float2half_rn(p - __half2float(hh)));
            }
            const int lo_col = (kNT == 2) ? col + 8 : col + 4;
            pt[col * kBlockTokens + t] = hi;
            pt[lo_col * kBlockTokens + t] = lo;
          }
        }
      }
      __syncwarp();
      const uint32_t* pt32 = reinterpret_cast<const uint32_t*>(pt);
      uint32_t pb[kNT][2];
#pragma unroll
      for (int nt = 0; nt < kNTPV; ++nt) {
        pb[nt][0] = pt32[(nt * 8 + r) * 8 + c];
        pb[nt][1] = pt32[(nt * 8 + r) * 8 + 4 + c];
      }
      // ---- rescale the running output (when raised), then O^T += V^T P^T
      if (raise) {
        float al0 = alpha[0], al1 = alpha[1];
        if constexpr (kNT == 1) {
          const float o0 = __shfl_xor_sync(0xffffffffu, al0, 2);
          const float o1 = __shfl_xor_sync(0xffffffffu, al1, 2);
          if (c >= 2) {
            al0 = o0;
            al1 = o1;
          }
        }
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
          for (int mt = 0; mt < kMTiles; ++mt) {
            acc[nt][mt][0] *= al0;
            acc[nt][mt][1] *= al1;
            acc[nt][mt][2] *= al0;
            acc[nt][mt][3] *= al1;
          }
      }
      if constexpr (!kFP8) {
        const int mi = lane >> 3, rr = lane & 7;
        const int t = rr + ((mi >> 1) << 3);
#pragma unroll
        for (int mt = 0; mt < kMTiles; ++mt) {
          const int box = mt >> 2;
          const int ch = 2 * (mt & 3) + (mi & 1);
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4_trans(vt_s + box * G::kBoxBytes + swz(t, ch), a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt)
            mma16816<kMmaBF16>(acc[nt][mt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
        }
      } else if constexpr (G::kNarrow) {
        // 64-byte rows: lane (r, c) reads 16 dims (chunk r % 4) of tokens 2c,
        // 2c+1, 2c+8, 2c+9 and takes the 8 starting at 8 (r / 4); m-tile t
        // row r (r + 8) is dim 16 (r % 4) + 8 (r / 4) + 2t (+ 1)
        const int ch = r & 3, hv = r >> 2;
        const uint4 W0 = lds128(vt_s + (2 * c) * G::kPitch + 16 * ch);
        const uint4 W1 = lds128(vt_s + (2 * c + 1) * G::kPitch + 16 * ch);
        const uint4 W2 = lds128(vt_s + (2 * c + 8) * G::kPitch + 16 * ch);
        const uint4 W3 = lds128(vt_s + (2 * c + 9) * G::kPitch + 16 * ch);
        const uint32_t x0[2] = {hv ? W0.z : W0.x, hv ? W0.w : W0.y};
        const uint32_t x1[2] = {hv ? W1.z : W1.x, hv ? W1.w : W1.y};
        const uint32_t x2[2] = {hv ? W2.z : W2.x, hv ? W2.w : W2.y};
        const uint32_t x3[2] = {hv ? W3.z : W3.x, hv ? W3.w : W3.y};
#pragma unroll
        for (int t = 0; t < kMTiles; ++t) {
          const uint32_t sel = (t & 1) ? 0x7362u : 0x5140u;
          const uint32_t lo01 = __byte_perm(x0[t >> 1], x1[t >> 1], sel);
          const uint32_t lo23 = __byte_perm(x2[t >> 1], x3[t >> 1], sel);
          const uint32_t a0 = e4m3x2_to_f16x2(lo01), a1 = e4m3x2_to_f16x2(lo01 >> 16);
          const uint32_t a2 = e4m3x2_to_f16x2(lo23), a3 = e4m3x2_to_f16x2(lo23 >> 16);
#pragma unroll
          for (int nt = 0; nt < kNTPV; ++nt)
            mma16816<false>(acc[nt][t], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
        }
      } else {
#pragma unroll
        for (int box = 0; box < G::kBoxes; ++box) {
          const uint32_t vb = vt_s + box * G::kBoxBytes;
          const uint4 W0 = lds128(vb + swz(2 * c, r));
          const uint4 W1 = lds128(vb + swz(2 * c + 1, r));
          const uint4 W2 = lds128(vb + swz(2 * c + 8, r));
          const uint4 W3 = lds128(vb + swz(2 * c + 9, r));
          const uint32_t x0[4] = {W0.x, W0.y, W0.z, W0.w};
          const uint32_t x1[4] = {W1.x, W1.y, W1.z, W1.w};
          const uint32_t x2[4] = {W2.x, W2.y, W2.z, W2.w};
          const uint32_t x3[4] = {W3.x, W3.y, W3.z, W3.w};
#pragma unroll
          for (int mm = 0; mm < 8; ++mm) {
            // bytes (k of token t, k of token t+1, k+1 of t, k+1 of t+1)
            const uint32_t sel = (mm & 1) ? 0x7362u : 0x5140u;
            const uint32_t lo01 = __byte_perm(x0[mm >> 1], x1[mm >> 1], sel);
            const uint32_t lo23 = __byte_perm(x2[mm >> 1], x3[mm >> 1], sel);
            const uint32_t a0 = e4m3x2_to_f16x2(lo01), a1 = e4m3x2_to_f16x2(lo01 >> 16);
            const uint32_t a2 = e4m3x2_to_f16x2(lo23), a3 = e4m3x2_to_f16x2(lo23 >> 16);
#pragma unroll
            for (int nt = 0; nt < kNTPV; ++nt)
              mma16816<false>(acc[nt][box * 8 + mm], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0 && k + NSTAGE < my_blocks) issue(k + NSTAGE);
  }
  if (dead) {
    // give every copy this warp still has in flight a bounded chance to land
    for (int kk = k + 1; kk < my_blocks && kk < k + NSTAGE; ++kk)
      (void)mbar_wait_bounded(wb + (kk % NSTAGE), (kk / NSTAGE) & 1);
  }
  const bool any_dead = __syncthreads_or(dead);
  if (any_dead) return;

  // ---- finish this warp: full row sums, hi + lo halves of the output
  float l_tot[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    float v = l_run[j];
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 16);
    l_tot[j] = v;
  }
  if constexpr (kNT == 1) {
#pragma unroll
    for (int mt = 0; mt < kMTiles; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[0][mt][e] += __shfl_xor_sync(0xffffffffu, acc[0][mt][e], 2);
  } else {
#pragma unroll
    for (int mt = 0; mt < kMTiles; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[0][mt][e] += acc[1][mt][e];
  }

  // ---- cross-warp merge through shared memory (rings are idle now)
  float* mg = reinterpret_cast<float*>(tiles);
  float* mg_o = mg + warp * (GT * D + 2 * GT);
  float* mg_m = mg_o + GT * D;
  float* mg_l = mg_m + GT;
  const bool owner = (kNT == 2) || (c < 2);
  if (owner) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int g = 2 * c + j;
      if (r == 0) {
        mg_m[g] = m_run[j];
        mg_l[g] = l_tot[j];
      }
#pragma unroll
      for (int mt = 0; mt < kMTiles; ++mt) {
        int d0, d1;
        if constexpr (!kFP8) {
          d0 = 16 * mt + r;
          d1 = d0 + 8;
        } else if constexpr (G::kNarrow) {
          d0 = 16 * (r & 3) + 8 * (r >> 2) + 2 * mt;
          d1 = d0 + 1;
        } else {
          d0 = (mt >> 3) * 128 + 16 * r + 2 * (mt & 7);
          d1 = d0 + 1;
        }
        mg_o[g * D + d0] = acc[0][mt][j];
        mg_o[g * D + d1] = acc[0][mt][2 + j];
      }
    }
  }
  __syncthreads();
  const int stride_w = GT * D + 2 * GT;
  const bool single = (nparts == 1);
  for (int idx = threadIdx.x; idx < group * D; idx += kThreads) {
    const int g = idx / D;
    const int d = idx - g * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mg[w * stride_w + GT * D + g]);
    const float Mu = (M == -INFINITY) ? 0.f : M;
    float lsum = 0.f, o = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float f = fast_exp2(mg[w * stride_w + GT * D + g] - Mu);
      lsum += f * mg[w * stride_w + GT * D + GT + g];
      o += f * mg[w * stride_w + g * D + d];
    }
    if (single) {
      const int64_t oq = static_cast<int64_t>(qrow) * Hq + hq0 + g;
      store_out(a.out, oq * D + d, a.out_dtype, lsum > 0.f ? o * v_mul / lsum : 0.f);
    } else {
      const int64_t hq = static_cast<int64_t>(row) * Hq + hq0 + g;
      const int64_t pidx = hq * a.max_parts + part;
      a.ws_o[pidx * D + d] = o;
      if (d == 0) {
        a.ws_m[pidx] = M;
        a.ws_l[pidx] = lsum;
      }
    }
  }
}

// Merge the partitions of every (row, KV head) whose context spans more than
// one partition.
__global__ void __launch_bounds__(kThreads) lse_reduce_kernel(const __grid_constant__ AttnArgs a) {
  const int h = blockIdx.x % a.num_kv_heads;
  const int row = blockIdx.x / a.num_kv_heads;
  int seq, L, qrow;
  resolve_row(a, row, seq, L, qrow);
  L = min(L, a.max_context_len);
  const int PS = a.partition_size;
  const int nparts = (L + PS - 1) / PS;
  if (nparts <= 1) return;
  const int group = a.group, D = a.head_dim, Hq = a.num_q_heads;
  const int hq0 = h * group;
  __shared__ float s_M[kMaxGroup], s_inv[kMaxGroup];
  const float vm = (a.kv_dtype == KV_FP8) ? a.v_scale[h] : 1.f;
  for (int g = threadIdx.x; g < group; g += blockDim.x) {
    const int64_t base = (static_cast<int64_t>(row) * Hq + hq0 + g) * a.max_parts;
    float M = -INFINITY;
    for (int p = 0; p < nparts; ++p) M = fmaxf(M, a.ws_m[base + p]);
    const float Mu = (M == -INFINITY) ? 0.f : M;
    float lsum = 0.f;
    for (int p = 0; p < nparts; ++p) lsum += fast_exp2(a.ws_m[base + p] - Mu) * a.ws_l[base + p];
    s_M[g] = Mu;
    s_inv[g] = lsum > 0.f ? vm / lsum : 0.f;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < group * D; idx += blockDim.x) {
    const int g = idx / D, d = idx - g * D;
    const int64_t hq = static_cast<int64_t>(row) * Hq + hq0 + g;
    const int64_t base = hq * a.max_parts;
    float o = 0.f;
    for (int p = 0; p < nparts; ++p)
      o += fast_exp2(a.ws_m[base + p] - s_M[g]) * a.ws_o[(base + p) * D + d];
    const int64_t oq = static_cast<int64_t>(qrow) * Hq + hq0 + g;
    store_out(a.out, oq * D + d, a.out_dtype, o * s_inv[g]);
  }
}

// Request index and visible-key count of every packed query row.
__global__ void varlen_prep_kernel(int32_t total_q, int32_t num_seqs, const int32_t* cu,
                                   const int32_t* seqlens_k, int32_t* row_seq,
                                   int32_t* row_len, bool skip_chunks) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total_q) return;
  int lo = 0, hi = num_seqs;            // first r with cu[r] > i, minus one
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (cu[mid] <= i) lo = mid + 1; else hi = mid;
  }
  int r = lo - 1;
  if (r < 0) r = 0;
  if (r > num_seqs - 1) r = num_seqs - 1;
  const int q_len = cu[r + 1] - cu[r];
  const int kv = seqlens_k[r];
  int n = kv - q_len + (i - cu[r]) + 1;
  n = n < 0 ? 0 : (n > kv ? kv : n);
  row_seq[i] = r;
  row_len[i] = (skip_chunks && q_len >= 2) ? -1 : n;
}

template <int KVT, bool Q_BF16, int D, int GT>
cudaError_t launch_typed(const AttnArgs& a, const CUtensorMap& kmap, const CUtensorMap& vmap,
                         cudaStream_t stream) {
  constexpr int NSTAGE = 2;
  using S = Smem<KVT, D, GT, NSTAGE>;
  auto kern = paged_attn_kernel<KVT, Q_BF16, D, GT, NSTAGE>;
  const int64_t grid =
      static_cast<int64_t>(a.rows) * a.num_kv_heads * a.max_parts * a.head_chunks;
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  if (grid == 0) return cudaSuccess;
  // the shared-memory limit is a setting of the function in the current
  // context: made once per context
  cudaError_t se = ensure_smem_attribute(reinterpret_cast<const void*>(kern), S::kTotal);
  if (se != cudaSuccess) return se;
  kern<<<static_cast<unsigned>(grid), kThreads, S::kTotal, stream>>>(a, kmap, vmap);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.max_parts > 1) {
    lse_reduce_kernel<<<static_cast<unsigned>(static_cast<int64_t>(a.rows) * a.num_kv_heads),
                        kThreads, 0, stream>>>(a);
    e = cudaGetLastError();
  }
  return e;
}

template <int KVT, bool Q_BF16, int D>
cudaError_t launch_group(const AttnArgs& a, const CUtensorMap& k, const CUtensorMap& v,
                         cudaStream_t s) {
  if (a.group <= 4) return launch_typed<KVT, Q_BF16, D, 4>(a, k, v, s);
  return launch_typed<KVT, Q_BF16, D, 8>(a, k, v, s);
}

template <int KVT, bool Q_BF16>
cudaError_t launch_dim(const AttnArgs& a, const CUtensorMap& k, const CUtensorMap& v,
                       cudaStream_t s) {
  switch (a.head_dim) {
    case 64: return launch_group<KVT, Q_BF16, 64>(a, k, v, s);
    case 128: return launch_group<KVT, Q_BF16, 128>(a, k, v, s);
    case 256: return launch_group<KVT, Q_BF16, 256>(a, k, v, s);
    default: break;
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool attention_supported(int q_dtype, int kv_dtype, int32_t head_dim, int32_t group) {
  if (group < 1 || group > kMaxGroup) return false;
  if (kv_dtype == KV_F16 || kv_dtype == KV_BF16) {
    if (q_dtype != kv_dtype) return false;
    return head_dim == 64 || head_dim == 128 || head_dim == 256;
  }
  if (kv_dtype == KV_FP8) {
    if (q_dtype != KV_F16 && q_dtype != KV_BF16) return false;
    return head_dim == 64 || head_dim == 128 || head_dim == 256;
  }
  return false;
}

cudaError_t launch_paged_attention(const AttnArgs& a, const CUtensorMap& kmap,
                                   const CUtensorMap& vmap, cudaStream_t stream) {
  switch (a.kv_dtype) {
    case KV_F16: return launch_dim<KV_F16, false>(a, kmap, vmap, stream);
    case KV_BF16: return launch_dim<KV_BF16, true>(a, kmap, vmap, stream);
    case KV_FP8:
      return a.q_dtype == KV_BF16 ? launch_dim<KV_FP8, true>(a, kmap, vmap, stream)
                                  : launch_dim<KV_FP8, false>(a, kmap, vmap, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_varlen_prep(int32_t total_q, int32_t num_seqs, const int32_t* cu_seqlens_q,
                               const int32_t* seqlens_k, int32_t* row_seq, int32_t* row_len,
                               bool skip_chunks, cudaStream_t stream) {
  if (total_q <= 0) return cudaSuccess;
  const int threads = 256;
  varlen_prep_kernel<<<(total_q + threads - 1) / threads, threads, 0, stream>>>(
      total_q, num_seqs, cu_seqlens_q, seqlens_k, row_seq, row_len, skip_chunks);
  return cudaGetLastError();
}

unsigned int read_and_clear_error_word(cudaStream_t stream, cudaError_t* err) {
  unsigned int v = 0, zero = 0;
  *err = cudaStreamSynchronize(stream);
  if (*err != cudaSuccess) return 0;
  *err = cudaMemcpyFromSymbol(&v, g_error_word, sizeof(v));
  if (*err != cudaSuccess) return 0;
  if (v) *err = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
  return v;
}

}  // namespace pa
