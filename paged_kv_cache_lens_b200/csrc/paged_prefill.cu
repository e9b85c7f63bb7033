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
// Work unit = (request, pair of query tiles, KV head).  A query tile is
// 128/G consecutive positions x the G query heads of the GQA group, stacked
// into a dense 128-row operand, so every K/V tile is read once for the whole
// group and shared by both query tiles of the pair (one for head_dim 256).
// Per 64-key tile and query tile i:
//   S_i = Q_i K^T    tcgen05.mma kind::f16, A = Q_i and B = K from shared
//                    memory (128-byte swizzle, K-major), D = S_i in TMEM (fp32);
//   P_i = softmax    one thread per row reads its TMEM lane of S_i and writes
//                    P_i (a separate TMEM region) as 16-bit hi + lo halves;
//   O_i += P_i V     tcgen05.mma with A = P_i from TMEM and B = V from shared
//                    memory (MN-major), D = O_i in TMEM.
// Softmax is online in one pass: P is taken against a running row maximum
// that is only raised (and O_i, l rescaled) when a tile's maximum exceeds it
// by more than 2^8, so P <= 256 and rescaling is rare.
//
// Warp roles: one softmax group of 4 warps per query tile (each owns its
// tile's rows, running maximum, sum and O, so the groups never wait on each
// other); a K and a V producer warp (paged tiles gathered 16 tokens at a time
// by TMA through the block table); one MMA-issuing warp per query tile, which
// issues S_i(j+1) while softmax i still works on tile j and PV_i(j) once P_i(j)
// is written.  S_i and P_i are separate TMEM regions: S_i(j+1) can be
// computed while PV_i(j) still reads P_i(j).
//
// CTAs are persistent (one per SM): each takes units from a heaviest-first
// list through an atomic counter until the list is exhausted.
#include "pa_device.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

constexpr int kBN = 64;                  // keys per tile
constexpr int kTblMax = 2048;            // block-table entries cached in shared memory
constexpr uint32_t kWaitLimit = 1u << 21;
constexpr float kRescaleGap = 8.f;       // raise the running max when exceeded by 2^8
constexpr float kLog2eF = 1.4426950408889634f;
constexpr uint32_t kTmemCols = 512;

template <int D, bool FP8 = false>
struct Cfg {
  static constexpr int NQ = (D == 256) ? 1 : 2;            // query tiles per unit
  static constexpr int kCB = D / 64;                       // 128-byte column blocks
  static constexpr int kQCB = 128 * 128;                   // bytes of a query tile column block
  static constexpr int kQBytes = kCB * kQCB;
  static constexpr int kKVCB = kBN * 128;                  // bytes of a K/V tile column block
  static constexpr int kKVBytes = kCB * kKVCB;
  static constexpr int kKSt = (D == 256) ? 2 : (FP8 ? 3 : 4);
  static constexpr int kVSt = (D == 256) ? 2 : (FP8 ? 3 : 4);
  // E4M3 pools: tiles land in a byte staging ring and are widened to f16
  // into the operand rings by their producer
  static constexpr int kSt8 = FP8 ? 2 : 0;
  static constexpr int kStage8Bytes = kBN * D;             // one E4M3 tile (128-byte rows)
  static constexpr int kSoftmaxWarps = 4 * NQ;
  static constexpr int kKWarp = kSoftmaxWarps;             // K producer
  static constexpr int kVWarp = kSoftmaxWarps + 1;         // V producer
  static constexpr int kMmaWarp0 = kSoftmaxWarps + 2;      // MMA warp i issues for query tile i
  static constexpr int kThreads = (kMmaWarp0 + NQ) * 32;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = NQ * kQBytes;
  static constexpr int kVOff = kKOff + kKSt * kKVBytes;
  static constexpr int kK8Off = kVOff + kVSt * kKVBytes;
  static constexpr int kV8Off = kK8Off + kSt8 * kStage8Bytes;
  static constexpr int kTblOff = kV8Off + kSt8 * kStage8Bytes;
  static constexpr int kBarOff = kTblOff + kTblMax * 4;
  // barriers: Q full [NQ] | K full, empty [kKSt] | V full, empty [kVSt] |
  //           S full, S free, P full, PV done [NQ] | drain [NQ] | V fixed |
  //           Q ready [NQ] | K, V staging full [kSt8] (E4M3 pools)
  static constexpr int B_Q = 0, B_KF = NQ, B_KE = B_KF + kKSt, B_VF = B_KE + kKSt,
                       B_VE = B_VF + kVSt, B_SF = B_VE + kVSt, B_SE = B_SF + NQ,
                       B_PF = B_SE + NQ, B_PVD = B_PF + NQ, B_DR = B_PVD + NQ,
                       B_VX = B_DR + NQ, B_QR = B_VX + 1, B_K8 = B_QR + NQ,
                       B_V8 = B_K8 + kSt8, kBars = B_V8 + kSt8;
  static constexpr int kMiscOff = kBarOff + kBars * 8;     // tmem base, abort, unit slots
  // + alignment slack; at least 116 KiB so that two CTAs never share an SM
  // (each allocates all 512 TMEM columns)
  static constexpr int kSmem = (kMiscOff + 64 + 1024) > 116 * 1024 ? (kMiscOff + 64 + 1024)
                                                                    : 116 * 1024;
  // TMEM columns: S_i at 64 i, P_i at 128 + 64 i, O_i at 256 + D i
  static constexpr uint32_t kSCol = 0, kPCol = 128, kOCol = 256;
  static_assert(kOCol + NQ * D <= kTmemCols, "TMEM budget");
  static_assert(kSmem <= 227 * 1024, "shared-memory budget");
};

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

// Geometry of query tile i of a unit: its rows, positions and the 64-key tiles
// it visits (jlo .. nkv-1; none when rows <= 0).
struct QTile {
  int rows, pos0, last, jlo, nkv;
  __device__ __forceinline__ bool active(int j) const { return rows > 0 && j >= jlo && j < nkv; }
  __device__ __forceinline__ int count() const { return rows > 0 ? nkv - jlo : 0; }
};

__device__ __forceinline__ QTile qtile(int q_len, int kv_len, int tq, int qt, int window) {
  QTile t;
  t.rows = min(tq, q_len - qt * tq);
  t.pos0 = kv_len - q_len + qt * tq;
  t.last = t.pos0 + t.rows - 1;
  if (t.rows <= 0 || t.last < 0) {
    t.rows = 0;
    t.jlo = t.nkv = 0;
    return t;
  }
  t.nkv = t.last / kBN + 1;
  t.jlo = window > 0 ? max(0, t.pos0 - window + 1) / kBN : 0;
  return t;
}

// Everything every role needs to know about one unit.
template <int NQ>
struct Unit {
  int r, pair, h, cu0, q_len, kv_len, tq;
  QTile qt[NQ];
  int j0, nu;     // key tiles j0 .. j0 + nu - 1 are loaded (the union of the tiles' ranges)
  int last_all;   // last position any row of the unit sees
  // the last loaded tile holds slots past kv_len (the rest of the context's
  // last 16-key block): the V producer clears them before the PVs read it
  bool stale;
};

template <int NQ>
__device__ __forceinline__ Unit<NQ> make_unit(const AttnArgs& a, int idx, int tq) {
  Unit<NQ> u;
  const int item = idx / a.num_kv_heads;
  u.h = idx - item * a.num_kv_heads;
  const int2 rp = a.pf_items[item];
  u.r = rp.x;
  u.pair = rp.y;
  u.tq = tq;
  u.cu0 = a.cu_seqlens_q[u.r];
  u.q_len = a.cu_seqlens_q[u.r + 1] - u.cu0;
  u.kv_len = min(a.seqlens_k[u.r], a.max_context_len);
  u.j0 = 0x7fffffff;
  int jend = 0;
#pragma unroll
  for (int i = 0; i < NQ; ++i) {
    u.qt[i] = qtile(u.q_len, u.kv_len, tq, NQ * u.pair + i, a.window);
    if (u.qt[i].rows > 0) {
      u.j0 = min(u.j0, u.qt[i].jlo);
      jend = max(jend, u.qt[i].nkv);
    }
  }
  u.nu = jend > 0 ? jend - u.j0 : 0;
  if (u.nu == 0) u.j0 = 0;
  u.last_all = -1;
#pragma unroll
  for (int i = 0; i < NQ; ++i)
    if (u.qt[i].rows > 0) u.last_all = max(u.last_all, u.qt[i].last);
  u.stale = u.nu > 0 && (u.kv_len % 16) != 0 && u.last_all >= ((u.kv_len - 1) & ~15);
  return u;
}

// E4M3 pool tile staging -> f16 operand tile: 16 bytes (16 dims) of row r at
// 128-byte-swizzled chunk c become 32 bytes (two 8-dim chunks) of the f16
// tile's column block c / 4, also 128-byte swizzled.
template <int D>
__device__ __forceinline__ void widen_e4m3_tile(const uint8_t* src, uint8_t* dst, int lane) {
  constexpr int kChunks = D / 16;                  // 16-byte chunks per E4M3 row
  for (int ix = lane; ix < kBN * kChunks; ix += 32) {
    const int r = ix / kChunks, c = ix % kChunks;
    const int sw = r & 7;
    const uint4 w = *reinterpret_cast<const uint4*>(src + (c >> 3) * (kBN * 128) + r * 128 +
                                                    (((c & 7) ^ sw) << 4));
    const uint4 lo = make_uint4(e4m3x2_to_f16x2(w.x), e4m3x2_to_f16x2(w.x >> 16),
                                e4m3x2_to_f16x2(w.y), e4m3x2_to_f16x2(w.y >> 16));
    const uint4 hi = make_uint4(e4m3x2_to_f16x2(w.z), e4m3x2_to_f16x2(w.z >> 16),
                                e4m3x2_to_f16x2(w.w), e4m3x2_to_f16x2(w.w >> 16));
    uint8_t* row = dst + (c >> 2) * (kBN * 128) + r * 128;
    *reinterpret_cast<uint4*>(row + (((2 * (c & 3)) ^ sw) << 4)) = lo;
    *reinterpret_cast<uint4*>(row + (((2 * (c & 3) + 1) ^ sw) << 4)) = hi;
  }
}

// bf16 query tile -> f16, in place (128-byte rows, the swizzle is a
// permutation of whole 16-byte chunks within a row, so it is kept).
template <int D>
__device__ __forceinline__ void q_bf16_to_f16(uint8_t* q, int lane) {
  for (int ix = lane; ix < 128 * D / 8; ix += 32) {
    uint4* p = reinterpret_cast<uint4*>(q) + ix;
    uint4 w = *p;
    w.x = bf16x2_to_f16x2(w.x);
    w.y = bf16x2_to_f16x2(w.y);
    w.z = bf16x2_to_f16x2(w.z);
    w.w = bf16x2_to_f16x2(w.w);
    *p = w;
  }
}

// P = 2^(x - m) for the PV product as two 16-bit values per key.
//  bf16 pools: hi = p truncated to bf16 (the upper half of its fp32 bits),
//    lo = (p - hi) truncated the same way: p - (hi + lo) < 2^-14 p, no
//    conversion instruction (the exponentials already keep the conversion
//    pipe busy);
//  f16 pools: hi = f16(p), lo = f16(p - hi), nearest even;
//  E4M3 pools (5e-2 tolerance): hi = f16(p) alone, lo unused.
template <int KVT>
__device__ __forceinline__ void pack_p(float p0, float p1, uint32_t& hi, uint32_t& lo) {
  if constexpr (KVT == 1) {
    const uint32_t b0 = __float_as_uint(p0), b1 = __float_as_uint(p1);
    hi = __byte_perm(b0, b1, 0x7632);
    const float r0 = p0 - __uint_as_float(b0 & 0xFFFF0000u);
    const float r1 = p1 - __uint_as_float(b1 & 0xFFFF0000u);
    lo = __byte_perm(__float_as_uint(r0), __float_as_uint(r1), 0x7632);
  } else if constexpr (KVT == 0) {
    hi = pack2<false>(p0, p1);
    lo = pack2<false>(p0 - lo_half_to_float<false>(hi), p1 - lo_half_to_float<false>(hi >> 16));
  } else {
    hi = pack2<false>(p0, p1);
    lo = 0;
  }
}

// KVT: 0 f16 pool, 1 bf16 pool, 2 E4M3 pool (widened to f16; the query is
// bf16 when Q_BF16, converted to f16 in shared memory).
template <int KVT, bool Q_BF16, int D>
__global__ void __launch_bounds__(Cfg<D, KVT == 2>::kThreads, 1)
paged_prefill_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap,
                     const __grid_constant__ CUtensorMap qmap, int log2g, int32_t* unit_counter) {
  constexpr bool FP8 = (KVT == 2);
  constexpr bool BF16 = (KVT == 1);                // the MMA operand type
  using C = Cfg<D, FP8>;
  constexpr int NQ = C::NQ;
  constexpr uint32_t kIdescS = idesc_f16(BF16, 128, kBN, false);
  constexpr uint32_t kIdescPV = idesc_f16(BF16, 128, D, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  int32_t* tbl = reinterpret_cast<int32_t*>(smem + C::kTblOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  volatile int* unit_slot = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 8);  // [2]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = 1 << log2g;
  const int tq = 128 >> log2g;              // query positions per tile
  const int total_units = *a.pf_count * a.num_kv_heads;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NQ; ++i) {
      mbar_init(&bars[C::B_Q + i], 1);
      mbar_init(&bars[C::B_SF + i], 1);
      mbar_init(&bars[C::B_SE + i], 128);
      mbar_init(&bars[C::B_PF + i], 128);
      mbar_init(&bars[C::B_PVD + i], 1);
    }
    // a K or V stage is free once every MMA warp's readers of it are done
    for (int s = 0; s < C::kKSt; ++s) {
      mbar_init(&bars[C::B_KF + s], 1);
      mbar_init(&bars[C::B_KE + s], NQ);
    }
    for (int s = 0; s < C::kVSt; ++s) {
      mbar_init(&bars[C::B_VF + s], 1);
      mbar_init(&bars[C::B_VE + s], NQ);
    }
    for (int i = 0; i < NQ; ++i) {
      mbar_init(&bars[C::B_DR + i], 1);
      mbar_init(&bars[C::B_QR + i], 1);
    }
    mbar_init(&bars[C::B_VX], 1);
    for (int s = 0; s < C::kSt8; ++s) {
      mbar_init(&bars[C::B_K8 + s], 1);
      mbar_init(&bars[C::B_V8 + s], 1);
    }
    *abort_flag = 0;
    unit_slot[0] = atomicAdd(unit_counter, 1);
    fence_barrier_init();
  }
  if (warp == C::kMmaWarp0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Running counts of every barrier's completed phases, kept across units by
  // the roles that wait on them (parity = count & 1).
  uint32_t kcnt = 0, vcnt = 0;             // K / V tiles loaded (producers) or passed (others)
  uint32_t c8 = 0;                         // producers (E4M3): tiles staged
  uint32_t qc8[NQ];                        // K producer (E4M3): loads of each query tile
#pragma unroll
  for (int i = 0; i < NQ; ++i) qc8[i] = 0;
  uint32_t mq = 0, ms = 0, mp = 0, mx = 0; // MMA warp: its Q loads, S tiles, PV batches, V fixes
  uint32_t sm_s = 0, sm_p = 0;             // softmax group: its tile's S tiles and PV batches

  int k = 0;
  for (;; ++k) {
    const int idx = unit_slot[k & 1];
    if (idx >= total_units || *abort_flag) break;
    const Unit<NQ> U = make_unit<NQ>(a, idx, tq);
    const int hq0 = U.h * G;

    if (warp == C::kKWarp || warp == C::kVWarp) {
      // ============================================================ TMA producers
      const bool is_v = warp == C::kVWarp;
      const int32_t* bt = a.block_tables + static_cast<int64_t>(U.r) * a.max_blocks_per_seq;
      const int bs = a.block_size;
      const int last_all = U.last_all;
      const int nblk = last_all / bs + 1;
      const int ncache = min(nblk, kTblMax);
      for (int i = (is_v ? 32 : 0) + lane; i < ncache; i += 64) tbl[i] = __ldg(bt + i);
      named_bar(2, 64);
      const int oob_row = a.num_blocks * a.num_kv_heads * bs;
      if (!is_v && lane == 0) {
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
          if (U.qt[i].rows <= 0) continue;
          uint64_t* qb = &bars[C::B_Q + i];
          mbar_arrive_expect_tx(qb, C::kQBytes);
          uint8_t* sq = smem + C::kQOff + i * C::kQBytes;
          const int row0 = U.cu0 + (NQ * U.pair + i) * tq;
#pragma unroll
          for (int cb = 0; cb < C::kCB; ++cb)
            tma_load_3d(sq + cb * C::kQCB, &qmap, cb * 64, hq0, row0, qb);
        }
      }
      const uint64_t pol = l2_policy_evict_last();
      const int nst = is_v ? C::kVSt : C::kKSt;
      uint64_t* full = &bars[is_v ? C::B_VF : C::B_KF];
      uint64_t* empty = &bars[is_v ? C::B_VE : C::B_KE];
      const CUtensorMap* map = is_v ? &vmap : &kmap;
      uint8_t* ring = smem + (is_v ? C::kVOff : C::kKOff);
      uint32_t& cnt = is_v ? vcnt : kcnt;
      if constexpr (FP8) {
        // ---- E4M3 pool: TMA into the byte staging ring, widen to f16 into
        // the operand ring, then release the operand stage
        uint64_t* sfull = &bars[is_v ? C::B_V8 : C::B_K8];
        uint8_t* stage = smem + (is_v ? C::kV8Off : C::kK8Off);
        auto stage_tile = [&](int u) {         // lane 0 arms, lanes 0-3 load
          const uint32_t s8 = (c8 + u) % C::kSt8;
          if (lane == 0) mbar_arrive_expect_tx(&sfull[s8], C::kStage8Bytes);
          __syncwarp();
          if (lane < kBN / 16) {
            const int sti = (U.j0 + u) * (kBN / 16) + lane;
            int y0 = oob_row, y1 = bs == 8 ? oob_row : -1;
            if (sti * 16 <= last_all) {
              const int32_t* src = (sti + 1) * 16 / bs + 1 < kTblMax ? tbl : bt;
              int r0, r1;
              if (tile_rows(src, sti, bs, nblk, a.num_blocks, a.num_kv_heads, U.h, oob_row, r0,
                            r1)) {
                y0 = r0;
                y1 = r1;
              } else {
                report_error(kErrBlockRange);
              }
            }
            uint8_t* box = stage + s8 * C::kStage8Bytes + lane * 2048;
#pragma unroll
            for (int cb = 0; cb < D / 128; ++cb) {
              tma_load_2d(box + cb * (kBN * 128), map, cb * 128, y0, &sfull[s8], pol);
              if (y1 >= 0)
                tma_load_2d(box + cb * (kBN * 128) + 1024, map, cb * 128, y1, &sfull[s8], pol);
            }
          }
        };
        for (int u = 0; u < C::kSt8 && u < U.nu; ++u) stage_tile(u);
        if (!is_v) {
          // the query tiles: f16 in shared memory before the MMA warps read them
#pragma unroll
          for (int i = 0; i < NQ; ++i) {
            if (U.qt[i].rows <= 0) continue;
            if (__all_sync(0xffffffffu,
                           wait_or_abort(&bars[C::B_Q + i], qc8[i] & 1, abort_flag))) {
              if constexpr (Q_BF16) q_bf16_to_f16<D>(smem + C::kQOff + i * C::kQBytes, lane);
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bars[C::B_QR + i]);
            }
            ++qc8[i];
          }
        }
        for (int u = 0; u < U.nu; ++u) {
          const uint32_t s8 = (c8 + u) % C::kSt8;
          const uint32_t st = cnt % nst;
          bool go = __all_sync(0xffffffffu, wait_or_abort(&sfull[s8], ((c8 + u) / C::kSt8) & 1,
                                                            abort_flag));
          if (go && cnt >= static_cast<uint32_t>(nst))
            go = __all_sync(0xffffffffu,
                            wait_or_abort(&empty[st], ((cnt / nst) - 1) & 1, abort_flag));
          if (!go) break;
          uint8_t* dst = ring + st * C::kKVBytes;
          widen_e4m3_tile<D>(stage + s8 * C::kStage8Bytes, dst, lane);
          if (is_v && U.stale && u == U.nu - 1) {
            // rows of the context's last 16-key block past kv_len: zero
            const int jl = U.j0 + U.nu - 1;
            const int r0 = U.kv_len - jl * kBN;
            const int r1 = ((U.kv_len + 15) & ~15) - jl * kBN;
            for (int ix = lane; ix < (r1 - r0) * 8 * C::kCB; ix += 32) {
              const int rr = r0 + ix / (8 * C::kCB);
              const int rem = ix % (8 * C::kCB);
              *reinterpret_cast<uint4*>(dst + (rem >> 3) * C::kKVCB + rr * 128 + (rem & 7) * 16) =
                  make_uint4(0, 0, 0, 0);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[st]);
          ++cnt;
          __syncwarp();
          if (u + C::kSt8 < U.nu) stage_tile(u + C::kSt8);
        }
        c8 += U.nu;
        if (is_v && U.stale && lane == 0) mbar_arrive(&bars[C::B_VX]);
        __syncwarp();
      } else
      for (int u = 0; u < U.nu; ++u) {
        const int j = U.j0 + u;
        const uint32_t st = cnt % nst;
        int go = 1;
        if (lane == 0) {
          go = !*abort_flag;
          if (go && cnt >= static_cast<uint32_t>(nst))
            go = wait_or_abort(&empty[st], ((cnt / nst) - 1) & 1, abort_flag);
          if (go) mbar_arrive_expect_tx(&full[st], C::kKVBytes);
        }
        if (!__shfl_sync(0xffffffffu, go, 0)) break;
        if (lane < kBN / 16) {
          // 16-key sub-tile `lane` of key tile j; past the keys any row sees
          // the box starts past the pool and is zero filled
          const int sti = j * (kBN / 16) + lane;
          int y0 = oob_row, y1 = bs == 8 ? oob_row : -1;
          if (sti * 16 <= last_all) {
            const int32_t* src = (sti + 1) * 16 / bs + 1 < kTblMax ? tbl : bt;
            int r0, r1;
            if (tile_rows(src, sti, bs, nblk, a.num_blocks, a.num_kv_heads, U.h, oob_row, r0,
                          r1)) {
              y0 = r0;
              y1 = r1;
            } else {
              report_error(kErrBlockRange);
            }
          }
          uint8_t* box = ring + st * C::kKVBytes + lane * 2048;
#pragma unroll
          for (int cb = 0; cb < C::kCB; ++cb) {
            tma_load_2d(box + cb * C::kKVCB, map, cb * 64, y0, &full[st], pol);
            if (y1 >= 0)
              tma_load_2d(box + cb * C::kKVCB + 1024, map, cb * 64, y1, &full[st], pol);
          }
        }
        ++cnt;
      }
      if (!FP8 && is_v && U.stale && !*abort_flag) {
        // V rows of the context's last 16-key block past kv_len hold whatever
        // the slots held; P is 0 there but 0 * NaN is NaN: once the unit's
        // last V tile (which holds them) has landed, clear them, then let
        // the MMA warps at it
        const uint32_t lt = cnt - 1;
        const bool landed = __all_sync(
            0xffffffffu, wait_or_abort(&full[lt % nst], (lt / nst) & 1, abort_flag));
        if (landed) {
          uint8_t* sv = ring + (lt % nst) * C::kKVBytes;
          const int jl = U.j0 + U.nu - 1;
          const int r0 = U.kv_len - jl * kBN;
          const int r1 = ((U.kv_len + 15) & ~15) - jl * kBN;
          for (int ix = lane; ix < (r1 - r0) * 8 * C::kCB; ix += 32) {
            const int rr = r0 + ix / (8 * C::kCB);
            const int rem = ix % (8 * C::kCB);
            *reinterpret_cast<uint4*>(sv + (rem >> 3) * C::kKVCB + rr * 128 + (rem & 7) * 16) =
                make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[C::B_VX]);
        }
      }
      __syncwarp();
    } else if (warp >= C::kMmaWarp0) {
      // ============================================================ MMA issuers
      // Warp kMmaWarp0 + i issues every MMA of query tile i, converged, one
      // elected lane per instruction: S_i(j) as soon as softmax i has read
      // S_i(j-1) and K(j) has landed, then PV_i(j-1) once P_i(j-1) is
      // written.  Its commits track only its own MMAs, so the two query
      // tiles never wait on each other's softmax.
      const int i = warp - C::kMmaWarp0;
      const QTile T = (NQ == 2 && i == 1) ? U.qt[NQ - 1] : U.qt[0];
      auto wait_all = [&](uint64_t* bar, uint32_t parity) {
        return __all_sync(0xffffffffu, wait_or_abort(bar, parity, abort_flag));
      };
      bool ok = true;
      const uint64_t qdesc =
          smem_desc_sw128(smem_u32(smem + C::kQOff + i * C::kQBytes), 16, 1024);
      if (T.rows > 0) {
        ok = wait_all(&bars[FP8 ? C::B_QR + i : C::B_Q + i], mq & 1);
        ++mq;
      }
      const uint64_t kdesc0 = smem_desc_sw128(smem_u32(smem + C::kKOff), 16, 1024);
      const uint64_t vdesc0 = smem_desc_sw128(smem_u32(smem + C::kVOff), C::kKVCB, 1024);
      const uint32_t d_s = tmem + C::kSCol + 64 * i;
      const uint32_t d_o = tmem + C::kOCol + D * i;
      const uint32_t a_p = tmem + C::kPCol + 64 * i;
      bool first_pv = true;
      for (int u = 0; ok && u <= U.nu; ++u) {
        const int j = U.j0 + u;
        if (u < U.nu) {
          // K(j) is waited for even when this tile does not need it, so that
          // this warp's release of the stage never runs ahead of the load
          const uint32_t ks = kcnt % C::kKSt;
          if (!(ok = wait_all(&bars[C::B_KF + ks], (kcnt / C::kKSt) & 1))) break;
          if (T.active(j)) {
            // ---- S_i(j) = Q_i K(j)^T
            if (ms > 0 && !(ok = wait_all(&bars[C::B_SE + i], (ms - 1) & 1))) break;
            tc_fence_after();
            const uint64_t kd = kdesc0 + static_cast<uint64_t>((ks * C::kKVBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t qo = static_cast<uint64_t>(((kk >> 2) * C::kQCB + (kk & 3) * 32) >> 4);
              const uint64_t ko = static_cast<uint64_t>(((kk >> 2) * C::kKVCB + (kk & 3) * 32) >> 4);
              tc_mma_ss_warp(d_s, qdesc + qo, kd + ko, kIdescS, kk > 0 ? 1u : 0u);
            }
            tc_commit_warp(&bars[C::B_SF + i]);
            ++ms;
          }
          tc_commit_warp(&bars[C::B_KE + ks]);   // this warp's reads of K(j) are done
          ++kcnt;
        }
        if (u >= 1) {
          const uint32_t vs = vcnt % C::kVSt;
          if (!(ok = wait_all(&bars[C::B_VF + vs], (vcnt / C::kVSt) & 1))) break;
          if (U.stale && u == U.nu) {     // the unit's last V tile, cleared by its producer
            if (!(ok = wait_all(&bars[C::B_VX], mx & 1))) break;
            ++mx;
          }
          if (T.active(j - 1)) {
            // ---- O_i += P_i(j-1) V(j-1)
            if (!(ok = wait_all(&bars[C::B_PF + i], mp & 1))) break;
            tc_fence_after();
            const uint64_t vd = vdesc0 + static_cast<uint64_t>((vs * C::kKVBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk) {
              // keys 16kk .. 16kk+15: 8 columns of hi pairs, then 8 of lo pairs
              const uint64_t vk = vd + static_cast<uint64_t>((kk * 2048) >> 4);
              tc_mma_ts_warp(d_o, a_p + 16 * kk, vk, kIdescPV, (first_pv && kk == 0) ? 0u : 1u);
              if constexpr (!FP8) tc_mma_ts_warp(d_o, a_p + 16 * kk + 8, vk, kIdescPV, 1u);
            }
            first_pv = false;
            tc_commit_warp(&bars[C::B_PVD + i]);
            ++mp;
          }
          tc_commit_warp(&bars[C::B_VE + vs]);   // this warp's reads of V(j-1) are done
          ++vcnt;
        }
      }
      if (!ok) *abort_flag = 1;
    } else {
      // ============================================================ softmax / epilogue
      const int qi = warp >> 2;                  // query tile of this group
      const QTile T = (NQ == 2 && qi == 1) ? U.qt[NQ - 1] : U.qt[0];
      const int quarter = warp & 3;
      const int t = quarter * 32 + lane;         // tile row == TMEM lane
      const int row = t >> log2g, g = t & (G - 1);
      const bool row_ok = row < T.rows;
      const int pos = T.pos0 + row;
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
      const uint32_t s_col = lane_base + C::kSCol + 64 * qi;
      const uint32_t p_col = lane_base + C::kPCol + 64 * qi;
      const uint32_t o_col = lane_base + C::kOCol + D * qi;
      const float c = a.scale * kLog2eF * (FP8 ? a.k_scale[U.h] : 1.f);
      const int lo_row = a.window > 0 ? pos - a.window + 1 : 0;
      const float slope = a.alibi ? a.alibi[hq0 + g] * kLog2eF : 0.f;
      // without ALiBi (and with scale > 0) the maximum is taken on the raw
      // scores and the scale folds into the exponent's FFMA
      const bool direct = a.alibi == nullptr && c > 0.f;
      const float cc = direct ? c : 1.f;
      bool ok = true;
      float m_run = -INFINITY, l_run = 0.f;
      const int n = T.count();
      for (int cix = 0; ok && cix < n; ++cix) {
        const int j = T.jlo + cix;
        ok = __all_sync(0xffffffffu, wait_or_abort(&bars[C::B_SF + qi], sm_s & 1, abort_flag));
        if (!ok) break;
        ++sm_s;
        tc_fence_after();
        uint32_t v[2][32];
        tmem_ld32(s_col, v[0]);
        tmem_ld32(s_col + 32, v[1]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars[C::B_SE + qi]);      // S_i may be overwritten now
        const int key0 = j * kBN;
        const bool full = key0 + kBN - 1 <= T.pos0 &&
                          (a.window <= 0 || key0 >= T.last - a.window + 1);
        const int nlo = full ? 0 : (row_ok ? lo_row - key0 : kBN);
        const int nhi = full ? kBN - 1 : (row_ok ? pos - key0 : -1);
        const float b0 = slope * static_cast<float>(key0 - pos);
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          if (!direct) {
#pragma unroll
            for (int x = 0; x < 32; ++x)
              v[h2][x] = __float_as_uint(fmaf(__uint_as_float(v[h2][x]), c,
                                              fmaf(slope, static_cast<float>(32 * h2 + x), b0)));
          }
          if (!full) {
#pragma unroll
            for (int x = 0; x < 32; ++x)
              if (32 * h2 + x < nlo || 32 * h2 + x > nhi) v[h2][x] = __float_as_uint(-INFINITY);
          }
#pragma unroll
          for (int x2 = 0; x2 < 16; ++x2)
            m4[x2 & 3] = fmax3(m4[x2 & 3], __uint_as_float(v[h2][2 * x2]),
                               __uint_as_float(v[h2][2 * x2 + 1]));
        }
        float m_tile = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        if (direct) m_tile *= c;                 // scale > 0: the maximum commutes with it
        const bool raise = (m_run == -INFINITY) ? (m_tile != -INFINITY)
                                                : (m_tile > m_run + kRescaleGap);
        const float m_new = raise ? m_tile : m_run;
        const float alpha = (!raise || m_run == -INFINITY) ? 1.f : fast_exp2(m_run - m_new);
        l_run *= alpha;
        const float nmu = (m_new == -INFINITY) ? 0.f : -m_new;
        // p = 2^(x - m_new) as 16-bit hi + lo pairs: for each 16 keys, 8
        // columns of hi pairs then 8 of lo pairs
        uint32_t pk[2][32];
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
          for (int x2 = 0; x2 < 16; ++x2) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(v[h2][2 * x2]), cc, nmu));
            const float p1 = fast_exp2(fmaf(__uint_as_float(v[h2][2 * x2 + 1]), cc, nmu));
            ls[x2 & 3] += p0 + p1;
            const int grp = x2 >> 3, w = x2 & 7;   // 16-key group within the half, pair
            pack_p<KVT>(p0, p1, pk[h2][16 * grp + w], pk[h2][16 * grp + 8 + w]);
          }
        }
        l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        m_run = m_new;
        if (cix > 0) {
          // P_i and O_i are free once PV_i of the previous tile has completed
          ok = __all_sync(0xffffffffu, wait_or_abort(&bars[C::B_PVD + qi], sm_p & 1, abort_flag));
          if (!ok) break;
          ++sm_p;
          tc_fence_after();
          if (__any_sync(0xffffffffu, raise && alpha != 1.f)) {
#pragma unroll 1
            for (int q2 = 0; q2 < D / 32; ++q2) {
              uint32_t o[32];
              tmem_ld32(o_col + 32 * q2, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(o_col + 32 * q2, o);
            }
          }
        }
        tmem_st32(p_col, pk[0]);
        tmem_st32(p_col + 32, pk[1]);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[C::B_PF + qi]);
      }
      // -------- epilogue: O_i row / l -> out
      if (n > 0) {
        const bool have = __all_sync(
            0xffffffffu, ok && wait_or_abort(&bars[C::B_PVD + qi], sm_p & 1, abort_flag));
        ++sm_p;
        if (have) {
          tc_fence_after();
          const float inv_l =
              l_run > 0.f ? (FP8 ? a.v_scale[U.h] : 1.f) / l_run : 0.f;
          const int64_t orow = (static_cast<int64_t>(U.cu0 + (NQ * U.pair + qi) * tq + row) *
                                    a.num_q_heads + hq0 + g) * D;
#pragma unroll 1
          for (int q2 = 0; q2 < D / 32; ++q2) {
            uint32_t o[32];
            tmem_ld32(o_col + 32 * q2, o);
            tmem_wait_ld();
            if (!row_ok) continue;
            if (a.out_dtype == 3) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow + 32 * q2);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                dst[e] = make_float4(__uint_as_float(o[4 * e]) * inv_l,
                                     __uint_as_float(o[4 * e + 1]) * inv_l,
                                     __uint_as_float(o[4 * e + 2]) * inv_l,
                                     __uint_as_float(o[4 * e + 3]) * inv_l);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + orow + 32 * q2);
              const bool ob = (a.out_dtype == 1);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                uint32_t w[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                  const float x0 = __uint_as_float(o[8 * e + 2 * x]) * inv_l;
                  const float x1 = __uint_as_float(o[8 * e + 2 * x + 1]) * inv_l;
                  w[x] = ob ? pack2<true>(x0, x1) : pack2<false>(x0, x1);
                }
                dst[e] = make_uint4(w[0], w[1], w[2], w[3]);
              }
            }
          }
        }
      }
    }
    // ---- the V tiles every role counted for this unit

    // ---- next unit: thread 0 takes it before the CTA-wide hand-over
    if (threadIdx.x == 0) unit_slot[(k + 1) & 1] = atomicAdd(unit_counter, 1);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  // ---- teardown: every MMA and copy of this CTA has completed (or been
  // given a bounded chance to) before TMEM is released.
  if (warp >= C::kMmaWarp0) {
    tc_commit_warp(&bars[C::B_DR + (warp - C::kMmaWarp0)]);
    (void)mbar_wait_bounded(&bars[C::B_DR + (warp - C::kMmaWarp0)], 0);
  }
  if ((warp == C::kKWarp || warp == C::kVWarp) && lane == 0 && *abort_flag) {
    const bool is_v = warp == C::kVWarp;
    const int nst = is_v ? C::kVSt : C::kKSt;
    uint64_t* full = &bars[is_v ? C::B_VF : C::B_KF];
    const uint32_t cnt = is_v ? vcnt : kcnt;
    for (uint32_t s = 0; s < static_cast<uint32_t>(nst) && s < cnt; ++s)
      (void)mbar_wait_bounded(&full[(cnt - 1 - s) % nst], ((cnt - 1 - s) / nst) & 1, 1u << 16);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == C::kMmaWarp0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Compact list of (request, pair of query tiles) items of the q_len >= 2
// requests, ordered by the number of key tiles the pair visits, most first
// (longest processing time first: the heavy units are taken first instead of
// forming the tail).  One CTA: a histogram of item weights in shared memory, a
// descending exclusive scan over it, then each item takes a slot in its
// weight's range (order within one weight is arbitrary; every item writes its
// own output rows, so the result does not depend on it).  Also resets the
// persistent kernel's unit counter.
constexpr int kItemThreads = 1024;
constexpr int kWeightBuckets = 4096;     // weights past the last bucket share it

__device__ __forceinline__ int item_weight(const int32_t* cu, const int32_t* seqlens_k,
                                           int32_t max_context_len, int32_t window, int tq,
                                           int nq, int r, int pair) {
  const int q_len = cu[r + 1] - cu[r];
  const int kv_len = min(seqlens_k[r], max_context_len);
  int w = 0;
  for (int i = 0; i < nq; ++i) w += qtile(q_len, kv_len, tq, nq * pair + i, window).count();
  return min(w, kWeightBuckets - 1);
}

__global__ void __launch_bounds__(kItemThreads)
prefill_items_kernel(int32_t num_seqs, const int32_t* cu, const int32_t* seqlens_k,
                     int32_t max_context_len, int32_t window, int tq, int nq, int2* items,
                     int32_t* count, int32_t capacity, int32_t* unit_counter) {
  __shared__ int s_hist[kWeightBuckets];
  __shared__ int s_part[kItemThreads];
  for (int i = threadIdx.x; i < kWeightBuckets; i += kItemThreads) s_hist[i] = 0;
  __syncthreads();
  const int span = tq * nq;                // query positions per item
  // ---- histogram of item weights
  for (int r = threadIdx.x; r < num_seqs; r += kItemThreads) {
    const int ql = cu[r + 1] - cu[r];
    if (ql < 2) continue;
    for (int p = 0; p < (ql + span - 1) / span; ++p)
      atomicAdd(&s_hist[item_weight(cu, seqlens_k, max_context_len, window, tq, nq, r, p)], 1);
  }
  __syncthreads();
  // ---- descending exclusive scan: bucket w starts after every heavier item.
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
    for (int p = 0; p < (ql + span - 1) / span; ++p) {
      const int slot = atomicAdd(
          &s_hist[item_weight(cu, seqlens_k, max_context_len, window, tq, nq, r, p)], 1);
      if (slot < capacity) items[slot] = make_int2(r, p);
    }
  }
  if (threadIdx.x == 0) {
    *count = min(total, capacity);
    *unit_counter = 0;
  }
}

int g_num_sms[64];

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (g_num_sms[dev] <= 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_num_sms[dev] = n;
  }
  return g_num_sms[dev];
}

int ilog2(int x) {
  int l = 0;
  while ((1 << l) < x) ++l;
  return l;
}

template <int KVT, bool Q_BF16, int D>
cudaError_t launch_prefill_typed(const AttnArgs& a, const CUtensorMap& k, const CUtensorMap& v,
                                 const CUtensorMap& q, int capacity, int32_t* unit_counter,
                                 cudaStream_t s) {
  using C = Cfg<D, KVT == 2>;
  auto kern = paged_prefill_kernel<KVT, Q_BF16, D>;
  const int64_t units = static_cast<int64_t>(capacity) * a.num_kv_heads;
  if (units == 0) return cudaSuccess;
  cudaError_t e = ensure_smem_attribute(reinterpret_cast<const void*>(kern), C::kSmem);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(units < num_sms() ? units : num_sms());
  kern<<<grid, C::kThreads, C::kSmem, s>>>(a, k, v, q, ilog2(a.group), unit_counter);
  return cudaGetLastError();
}

template <int KVT>
cudaError_t launch_prefill_d(const AttnArgs& a, const CUtensorMap& k, const CUtensorMap& v,
                             const CUtensorMap& q, int capacity, int32_t* ctr, cudaStream_t s) {
  constexpr bool QB = (KVT == 1);
  switch (a.head_dim) {
    case 64: return launch_prefill_typed<KVT, QB, 64>(a, k, v, q, capacity, ctr, s);
    case 128: return launch_prefill_typed<KVT, QB, 128>(a, k, v, q, capacity, ctr, s);
    case 256: return launch_prefill_typed<KVT, QB, 256>(a, k, v, q, capacity, ctr, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_prefill_fp8(const AttnArgs& a, const CUtensorMap& k, const CUtensorMap& v,
                               const CUtensorMap& q, int capacity, int32_t* ctr, cudaStream_t s) {
  if (a.head_dim != 128) return cudaErrorInvalidValue;
  return a.q_dtype == 1 ? launch_prefill_typed<2, true, 128>(a, k, v, q, capacity, ctr, s)
                        : launch_prefill_typed<2, false, 128>(a, k, v, q, capacity, ctr, s);
}

}  // namespace

bool prefill_supported(int q_dtype, int kv_dtype, int32_t head_dim, int32_t group) {
  if (group < 1 || group > 128 || (group & (group - 1)) != 0) return false;
  if (kv_dtype == 2)   // E4M3 pool, widened to f16 in shared memory: head_dim 128
    return head_dim == 128 && (q_dtype == 0 || q_dtype == 1);
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return false;
  return (kv_dtype == 0 || kv_dtype == 1) && q_dtype == kv_dtype;
}

int prefill_query_tile(int32_t group) { return 128 / group; }

int prefill_tiles_per_item(int32_t head_dim) { return head_dim == 256 ? 1 : 2; }

int32_t prefill_item_capacity(int32_t num_seqs, int32_t total_q) {
  // every item holds at least one query row of a request with q_len >= 2
  (void)num_seqs;
  return total_q;
}

cudaError_t launch_paged_prefill(const AttnArgs& a, const CUtensorMap& kmap,
                                 const CUtensorMap& vmap, const CUtensorMap& qmap,
                                 int32_t capacity, int32_t* unit_counter, cudaStream_t stream) {
  const int tq = 128 / a.group;
  const int nq = prefill_tiles_per_item(a.head_dim);
  prefill_items_kernel<<<1, kItemThreads, 0, stream>>>(
      a.num_seqs, a.cu_seqlens_q, a.seqlens_k, a.max_context_len, a.window, tq, nq,
      const_cast<int2*>(a.pf_items), const_cast<int32_t*>(a.pf_count), capacity, unit_counter);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.kv_dtype == 2) return launch_prefill_fp8(a, kmap, vmap, qmap, capacity, unit_counter, stream);
  return a.kv_dtype == 1 ? launch_prefill_d<1>(a, kmap, vmap, qmap, capacity, unit_counter, stream)
                         : launch_prefill_d<0>(a, kmap, vmap, qmap, capacity, unit_counter, stream);
}

}  // namespace pa
