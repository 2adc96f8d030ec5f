// decode_tc_kernel.cuh — split-KV GQA decode for d = 128 on the tcgen05 tensor cores.
//
// Same result and workspace layout as fa_decode_split_kernel (decode_kernel.cuh): per
// (sequence, query head, KV split) a normalised partial O row and its log2-domain LSE,
// merged afterwards by fa_decode_combine_kernel. What changes is how a split is computed.
// The decode is bound by device-memory bandwidth (page "Empreinte mémoire et calcul des
// couches Transformer": the KV cache is read in full for every generated token); done on
// CUDA cores its per-row arithmetic (bf16 unpacking, fp32 dot products, lane reductions)
// costs more issue slots than the memory time allows. Here the two contractions per
// 128-token tile run on the tensor core and the threads only do the softmax:
//     S^T[tokens x heads] = K_tile[128 x d] . Q^T        (M = 128 tokens, N = 16, K = d)
//     O^T[d x heads]     += V_tile^T . P^T                (M = d = 128, N = 16, K = 128)
// Q holds up to 16 query heads of one KV head (rows past the group are never stored).
//
// Persistent CTAs (one per SM), scheduled dynamically. A work unit is one split (up to
// split_tokens tokens) of one (sequence, KV-head tile); the units that exist (splits
// before kv_len) are numbered in (sequence, head tile, split) order. CTA c starts with
// unit c; each further unit is a ticket from an atomic counter in the workspace, so a
// CTA that streams slower simply takes fewer units. The counter is zeroed by a one-thread
// kernel that this one depends on programmatically: the CTAs start at once, and the
// ticket taker waits (griddepcontrol.wait) for the zeroing only before its first ticket. The K
// producer takes the tickets and hands each unit to the other roles through a 4-deep
// shared-memory ring of unit descriptors. Warps:
//   0-3  softmax: thread t owns token t of the tile (TMEM lane t of S^T) and row d = t
//        of O^T; warp-level max, cross-warp max through shared memory + an mbarrier,
//        lazy rescale of O^T (threshold 2^8), P^T written to shared memory in the
//        canonical K-major 128-byte-swizzle layout. The epilogue of unit k (normalised
//        partial row + LSE) runs after unit k + 1's first P^T: unit k accumulates in
//        O^T[k & 1], so its last P.V completes while the next unit already streams.
//   4    K producer: the unit's query rows (TMA, double-buffered) and K tiles.
//   5    TMEM allocator and single-thread tcgen05.mma issuer. S^T of tile j+1 is issued
//        before P.V of tile j, so scores are ready when the softmax warps need them.
//   6    V producer: V tiles.
// K and V have separate ring barriers: a K slot is refilled as soon as its S^T MMA is
// done, a tile before the V slot frees. Tokens of a tile past the split's end are masked
// to -inf and their V rows zeroed in shared memory (rows of the cache past kv_len are never
// used, whatever they hold).
//
// PAGED = true reads the cache from a page pool (PagedKV in sm100.cuh): a 128-token tile
// is one box of a page of >= 128 tokens, or 128 / page_size boxes of smaller pages, each
// landing at its row offset of the swizzled tile (page_size >= 16 keeps every box on a
// 1 KB swizzle-atom boundary). Each producer then runs as a whole warp, lane i handling
// page i of a tile. A box wholly past the split's end is aimed past the pool and reads
// zeros, so table entries beyond the sequence are never read.
#pragma once

#include <cuda.h>
#include <math_constants.h>

#include "sm100.cuh"

namespace fa {

constexpr int kTcD = 128;
constexpr int kTcTile = 128;                 // tokens per tile (MMA M for S^T)
constexpr int kTcStages = 3;
constexpr int kTcThreads = 224;
constexpr int kTcWarpKProd = 4;
constexpr int kTcWarpMma = 5;
constexpr int kTcWarpVProd = 6;
constexpr int kTcN = 16;                     // padded head count (MMA N)
constexpr int kTcChunk = kTcTile * 128;      // 128 rows x 128 bytes
constexpr int kTcTileBytes = kTcTile * kTcD * 2;          // 32 KB (K or V)
constexpr int kTcStageBytes = 2 * kTcTileBytes;           // K then V
constexpr int kTcQBytes = kTcN * kTcD * 2;                // 4 KB: 2 chunks of 16 x 128 B
constexpr int kTcPBytes = kTcN * kTcTile * 2;             // 4 KB: 2 chunks of 16 x 128 B
constexpr int kTcSmallChunk = kTcN * 128;                 // 2 KB
constexpr int kTcOffQ = kTcStages * kTcStageBytes;        // Q[2]
constexpr int kTcOffP = kTcOffQ + 2 * kTcQBytes;          // P[2]
constexpr int kTcOffRed = kTcOffP + 2 * kTcPBytes;        // float [2][4 warps][16]
constexpr int kTcOffBar = kTcOffRed + 2 * 4 * kTcN * 4;
// barriers: kfull[3] kempty[3] vfull[3] vempty[3] qfull[2] qempty[2] s[2] p[2] o[2] x pv drain
// + unit ring: ufull[4] uempty[4]
constexpr int kTcUnitRing = 4;
constexpr int kTcNBars = 4 * kTcStages + 13 + 2 * kTcUnitRing;
constexpr int kTcOffMisc = (kTcOffBar + kTcNBars * 8 + 15) / 16 * 16;
constexpr int kTcOffSched = kTcOffMisc + 16;              // TcStart (8-byte fields)
constexpr int kTcOffRing = kTcOffSched + 64;               // unit descriptors (int4 each)
constexpr int kTcSmemBytes = kTcOffRing + 16 * kTcUnitRing + 1024;
static_assert(kTcOffQ % 1024 == 0 && kTcOffP % 1024 == 0, "128-byte-swizzle operands need 1 KB alignment");
static_assert(kTcOffRed % 16 == 0 && kTcOffBar % 8 == 0, "reduction / barrier alignment");
static_assert(kTcOffMisc % 16 == 0 && kTcOffSched % 16 == 0 && kTcOffRing % 16 == 0,
              "16-byte shared accesses (descriptor ring, TcStart) need 16-byte alignment");
constexpr uint32_t kTcTmemCols = 64;                      // S^T x2 [0,32), O^T x2 [32,64)
static_assert(kTcSmemBytes <= 227 * 1024, "shared memory budget");


struct DecodeTcParams {
  const int* kv_lens;     // [B]
  unsigned* tickets;      // unit counter, zero at launch
  float* ws_o;            // [B, Hq, n_split, 128]
  float* ws_lse;          // [B, Hq, n_split]
  int B, Hq, Hkv, G, GT;  // GT = heads per tile (<= 16), n_gt tiles per KV head
  int n_gt;
  int max_len, split_tokens, n_split;
  float scale_log2;
  uint64_t timeout_ns;
  int skip_q_load;        // test hook: the Q tiles are never loaded
  PagedKV pk;             // PAGED kernels only
};

struct TcUnit {
  int b, kvh, g0, split, t0, t1;
};

__device__ __forceinline__ int tc_seq_len(const DecodeTcParams& p, int b) {
  const int len = p.kv_lens[b];
  return len < 0 ? 0 : (len > p.max_len ? p.max_len : len);
}

// Position of a unit in the numbering: sequence b (length len, ns splits) whose first unit
// is number base; unit base + hg * ns + s is split s of head tile hg.
struct TcCursor {
  int b, len, ns;
  long long base;
  // Move forward to unit k (k >= base, k below the total) and decode it.
  __device__ __forceinline__ void locate(const DecodeTcParams& p, long long k, TcUnit& w) {
    const int HT = p.Hkv * p.n_gt;
    while (k >= base + static_cast<long long>(HT) * ns) {
      base += static_cast<long long>(HT) * ns;
      ++b;
      len = tc_seq_len(p, b);
      ns = (len + p.split_tokens - 1) / p.split_tokens;
    }
    const int r = static_cast<int>(k - base);
    const int hg = r / ns, sp = r - hg * ns;
    w.b = b;
    w.kvh = hg / p.n_gt;
    w.g0 = (hg - w.kvh * p.n_gt) * p.GT;
    w.split = sp;
    w.t0 = sp * p.split_tokens;
    w.t1 = min(len, w.t0 + p.split_tokens);
  }
};

struct TcStart {
  TcCursor cur;           // positioned at or before unit blockIdx.x
  long long total;        // units that exist
};

// Total unit count and a cursor at sequence 0 (executed by one full warp).
__device__ __forceinline__ TcStart tc_start(const DecodeTcParams& p) {
  const int lane = threadIdx.x & 31;
  long long total = 0;
  for (int b0 = 0; b0 < p.B; b0 += 32) {
    const int len = (b0 + lane < p.B) ? tc_seq_len(p, b0 + lane) : 0;
    long long v = (len + p.split_tokens - 1) / p.split_tokens;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    total += v;
  }
  TcStart st;
  st.total = total * p.Hkv * p.n_gt;
  st.cur.b = 0;
  st.cur.len = tc_seq_len(p, 0);
  st.cur.ns = (st.cur.len + p.split_tokens - 1) / p.split_tokens;
  st.cur.base = 0;
  return st;
}

// Unit descriptor passed from the K producer to the other roles (b < 0: no more units).
struct TcDesc {
  int b, kvh, g0, split;
};

// The tiles (128 tokens from t0 to t1) of one unit.
struct TcTiles {
  TcUnit w;
  int t;
  __device__ __forceinline__ bool unit_first() const { return t == w.t0; }
  __device__ __forceinline__ bool unit_last() const { return t + kTcTile >= w.t1; }
};

__device__ __forceinline__ void tc_unit_from(const DecodeTcParams& p, const TcDesc& d, TcUnit& w) {
  w.b = d.b;
  w.kvh = d.kvh;
  w.g0 = d.g0;
  w.split = d.split;
  w.t0 = d.split * p.split_tokens;
  w.t1 = min(tc_seq_len(p, d.b), w.t0 + p.split_tokens);
}

// Zeroes the unit counter of one decode call. The split kernel is its programmatic
// dependent: it may start once this has begun and waits for the store only before its
// first ticket.
__global__ void __launch_bounds__(32) fa_decode_ticket_reset_kernel(unsigned* tickets) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) *tickets = 0u;
}

template <bool BF16, int GT, bool PAGED>
__global__ void __launch_bounds__(kTcThreads, 1)
fa_decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmQ, const DecodeTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t bar0 = base + kTcOffBar;
  auto bar_kfull = [&](int s) { return bar0 + 8u * s; };
  auto bar_kempty = [&](int s) { return bar0 + 8u * (kTcStages + s); };
  auto bar_vfull = [&](int s) { return bar0 + 8u * (2 * kTcStages + s); };
  auto bar_vempty = [&](int s) { return bar0 + 8u * (3 * kTcStages + s); };
  auto bar_qfull = [&](int b) { return bar0 + 8u * (4 * kTcStages + b); };
  auto bar_qempty = [&](int b) { return bar0 + 8u * (4 * kTcStages + 2 + b); };
  auto bar_s = [&](int b) { return bar0 + 8u * (4 * kTcStages + 4 + b); };   // S^T[b] ready
  auto bar_p = [&](int b) { return bar0 + 8u * (4 * kTcStages + 6 + b); };   // P^T[b] written
  // O^T[b] of a unit complete (unit k of the CTA accumulates in O^T[k & 1])
  auto bar_o = [&](int b) { return bar0 + 8u * (4 * kTcStages + 8 + b); };
  const uint32_t bar_x = bar0 + 8u * (4 * kTcStages + 10);   // cross-warp exchange (4)
  const uint32_t bar_pv = bar0 + 8u * (4 * kTcStages + 11);  // each P.V done
  const uint32_t bar_drain = bar0 + 8u * (4 * kTcStages + 12);
  // Unit ring: slot n % 4 holds the descriptor of the CTA's n-th unit.
  auto bar_ufull = [&](int n) { return bar0 + 8u * (4 * kTcStages + 13 + (n & (kTcUnitRing - 1))); };
  auto bar_uempty = [&](int n) {
    return bar0 + 8u * (4 * kTcStages + 13 + kTcUnitRing + (n & (kTcUnitRing - 1)));
  };
  // Plain shared accesses: mbarrier arrive / wait (asm with memory clobbers) order them.
  int4* ring = reinterpret_cast<int4*>(sbase + kTcOffRing);
  // Readers of each descriptor: V producer, MMA thread, 4 softmax warps.
  constexpr int kTcRingReaders = 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + kTcOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + kTcOffMisc + 4);
  float* red = reinterpret_cast<float*>(sbase + kTcOffRed);  // [2][4][16]

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(bar_kfull(s), 1);
      mbar_init(bar_kempty(s), 1);
      mbar_init(bar_vfull(s), 1);
      mbar_init(bar_vempty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_qfull(b), 1);
      mbar_init(bar_qempty(b), 1);
      mbar_init(bar_s(b), 1);
      mbar_init(bar_p(b), 128);
    }
    mbar_init(bar_o(0), 1);
    mbar_init(bar_o(1), 1);
    mbar_init(bar_x, 4);
    mbar_init(bar_pv, 1);
    mbar_init(bar_drain, 1);
    for (int n = 0; n < kTcUnitRing; ++n) {
      mbar_init(bar_ufull(n), 1);
      mbar_init(bar_uempty(n), kTcRingReaders);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  // P^T buffers start at zero: rows past the head tile stay zero for the whole kernel.
  for (int i = threadIdx.x; i < (2 * kTcPBytes) / 16; i += kTcThreads)
    reinterpret_cast<uint4*>(sbase + kTcOffP)[i] = make_uint4(0, 0, 0, 0);
  TcStart* start0 = reinterpret_cast<TcStart*>(sbase + kTcOffSched);
  if (warp == 0) {
    const TcStart st = tc_start(p);
    if (lane == 0) *start0 = st;
  }
  if (warp == kTcWarpMma) tmem_alloc(smem_u32(tmem_slot), kTcTmemCols);
  if (warp == kTcWarpKProd && lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmQ);
  }
  if (warp == kTcWarpVProd && lane == 0) prefetch_tmap(&tmV);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, &g_fa_status, p.timeout_ns};
  // Reader side of the unit ring: the n-th unit's descriptor (false if the wait ran out).
  auto ring_read = [&](int n, TcDesc& d) -> bool {
    if (!mbar_wait(bar_ufull(n), (n / kTcUnitRing) & 1, wc)) return false;
    const int4 v = ring[n & (kTcUnitRing - 1)];
    d.b = v.x;
    d.kvh = v.y;
    d.g0 = v.z;
    d.split = v.w;
    return true;
  };

  if (warp == kTcWarpKProd || warp == kTcWarpVProd) {
    // ---------------------------------------------------------------- TMA producers
    if constexpr (!PAGED) {
    if (lane == 0) {
      const bool is_k = warp == kTcWarpKProd;
      const CUtensorMap* tm = is_k ? &tmK : &tmV;
      int jg = 0, uc = 0, n = 0;
      bool ok = true, counter_ready = false;
      const TcStart st = *start0;
      TcCursor cursor = st.cur;
      long long ticket = blockIdx.x;                 // unit of the CTA's first ticket
      while (ok) {
        TcUnit w;
        if (is_k) {
          // Publish unit n (or the end) to the other roles.
          const bool have = ticket < st.total;
          if (have) cursor.locate(p, ticket, w);
          if (n >= kTcUnitRing && !mbar_wait(bar_uempty(n), (n / kTcUnitRing - 1) & 1, wc)) {
            ok = false;
            break;
          }
          ring[n & (kTcUnitRing - 1)] = have ? make_int4(w.b, w.kvh, w.g0, w.split) : make_int4(-1, 0, 0, 0);
          mbar_arrive(bar_ufull(n));
          ++n;
          if (!have) break;
          // Query rows of the unit: 16 rows from head (b, kvh*G + g0) on (rows past the
          // head tile are loaded but never used); Q buffer uc % 2.
          const int qb = uc & 1;
          if (uc >= 2 && !mbar_wait(bar_qempty(qb), ((uc >> 1) - 1) & 1, wc)) { ok = false; break; }
          mbar_arrive_expect_tx(bar_qfull(qb), kTcQBytes);
          const int row0 = w.b * p.Hq + w.kvh * p.G + w.g0;
          for (int ch = 0; ch < 2 && !p.skip_q_load; ++ch)
            tma_load_3d(base + kTcOffQ + qb * kTcQBytes + ch * kTcSmallChunk, &tmQ, bar_qfull(qb),
                        ch * 64, row0, 0);
          ++uc;
        } else {
          TcDesc d;
          if (!ring_read(n, d)) { ok = false; break; }
          mbar_arrive(bar_uempty(n));
          ++n;
          if (d.b < 0) break;
          tc_unit_from(p, d, w);
        }
        unsigned next_ticket = 0;
        bool asked = false;
        const int bhkv = w.b * p.Hkv + w.kvh;
        for (int t = w.t0; t < w.t1; t += kTcTile, ++jg) {
          // The next ticket is drawn two tiles before this unit's loads end: late enough to
          // balance, early enough that its latency hides behind these loads.
          if (is_k && !asked && t + 2 * kTcTile >= w.t1) {
            if (!counter_ready) {   // the counter is zeroed by the launch this one depends on
              asm volatile("griddepcontrol.wait;" ::: "memory");
              counter_ready = true;
            }
            next_ticket = atomicAdd(p.tickets, 1u);
            asked = true;
          }
          const int stg = jg % kTcStages;
          const uint32_t empty = is_k ? bar_kempty(stg) : bar_vempty(stg);
          const uint32_t full = is_k ? bar_kfull(stg) : bar_vfull(stg);
          if (jg >= kTcStages && !mbar_wait(empty, ((jg / kTcStages) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full, kTcTileBytes);
          const uint32_t dst = base + stg * kTcStageBytes + (is_k ? 0 : kTcTileBytes);
          for (int ch = 0; ch < 2; ++ch) tma_load_3d(dst + ch * kTcChunk, tm, full, ch * 64, t, bhkv);
        }
        if (is_k) ticket = static_cast<long long>(gridDim.x) + next_ticket;
      }
      if (!ok || *abort_flag) {
        // Loads still in flight must land before the CTA exits.
        for (int k = max(0, jg - kTcStages); k < jg; ++k)
          mbar_wait_drain(is_k ? bar_kfull(k % kTcStages) : bar_vfull(k % kTcStages),
                          (k / kTcStages) & 1, kDrainNs);
        if (is_k)
          for (int k = max(0, uc - 2); k < uc; ++k) mbar_wait_drain(bar_qfull(k & 1), (k >> 1) & 1, kDrainNs);
      }
    }
    } else {
    // Paged pool: the whole warp walks the units. Lane 0 does what the contiguous path's
    // producer does (unit ring, tickets, Q, ring barriers); lane i reads the table entry of
    // page i of each tile and issues that page's two boxes.
    const bool leader = lane == 0;
    const bool is_k = warp == kTcWarpKProd;
    const CUtensorMap* tm = is_k ? &tmK : &tmV;
    const int ps = 1 << p.pk.page_shift;
    const int rows = min(kTcTile, ps);
    const bool mine = lane * rows < kTcTile;
    int jg = 0, uc = 0, n = 0;
    bool ok = true, counter_ready = false;
    const TcStart st = *start0;
    TcCursor cursor = st.cur;
    long long ticket = blockIdx.x;                   // unit of the CTA's first ticket
    while (ok) {
      TcUnit w;
      if (is_k) {
        // Publish unit n (or the end) to the other roles.
        const bool have = ticket < st.total;
        if (have) cursor.locate(p, ticket, w);
        if (leader) {
          if (n >= kTcUnitRing && !mbar_wait(bar_uempty(n), (n / kTcUnitRing - 1) & 1, wc)) {
            ok = false;
          } else {
            ring[n & (kTcUnitRing - 1)] =
                have ? make_int4(w.b, w.kvh, w.g0, w.split) : make_int4(-1, 0, 0, 0);
            mbar_arrive(bar_ufull(n));
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        ++n;
        if (!have) break;
        // Query rows of the unit (as in the contiguous path), Q buffer uc % 2.
        const int qb = uc & 1;
        if (leader) {
          if (uc >= 2 && !mbar_wait(bar_qempty(qb), ((uc >> 1) - 1) & 1, wc)) {
            ok = false;
          } else {
            mbar_arrive_expect_tx(bar_qfull(qb), kTcQBytes);
            const int row0 = w.b * p.Hq + w.kvh * p.G + w.g0;
            for (int ch = 0; ch < 2 && !p.skip_q_load; ++ch)
              tma_load_3d(base + kTcOffQ + qb * kTcQBytes + ch * kTcSmallChunk, &tmQ, bar_qfull(qb),
                          ch * 64, row0, 0);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        ++uc;
      } else {
        TcDesc d{0, 0, 0, 0};
        int got = 1;
        if (leader) {
          got = ring_read(n, d) ? 1 : 0;
          if (got) mbar_arrive(bar_uempty(n));
        }
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) { ok = false; break; }
        d.b = __shfl_sync(0xffffffffu, d.b, 0);
        d.kvh = __shfl_sync(0xffffffffu, d.kvh, 0);
        d.g0 = __shfl_sync(0xffffffffu, d.g0, 0);
        d.split = __shfl_sync(0xffffffffu, d.split, 0);
        ++n;
        if (d.b < 0) break;
        tc_unit_from(p, d, w);
      }
      unsigned next_ticket = 0;
      bool asked = false;
      for (int t = w.t0; t < w.t1; t += kTcTile, ++jg) {
        // The next ticket is drawn two tiles before this unit's loads end.
        if (is_k && !asked && t + 2 * kTcTile >= w.t1) {
          if (leader) {
            if (!counter_ready) {   // the counter is zeroed by the launch this one depends on
              asm volatile("griddepcontrol.wait;" ::: "memory");
              counter_ready = true;
            }
            next_ticket = atomicAdd(p.tickets, 1u);
          }
          asked = true;
        }
        const int stg = jg % kTcStages;
        const uint32_t empty = is_k ? bar_kempty(stg) : bar_vempty(stg);
        const uint32_t full = is_k ? bar_kfull(stg) : bar_vfull(stg);
        // This lane's page: read before the slot wait so that its latency hides behind it.
        // A page wholly past the split's end is aimed past the pool (zeros).
        const int tok = t + lane * rows;
        const bool used = mine && tok < w.t1;
        const int entry = used ? paged_entry(p.pk, w.b, tok) : 0;
        if (leader) {
          if (jg >= kTcStages && !mbar_wait(empty, ((jg / kTcStages) - 1) & 1, wc))
            ok = false;
          else
            mbar_arrive_expect_tx(full, kTcTileBytes);
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (mine) {
          const uint32_t dst = base + stg * kTcStageBytes + (is_k ? 0 : kTcTileBytes);
          const int z = used ? paged_z(p.pk, entry, w.kvh) : paged_z_oob(p.pk);
          const int y = t & (ps - 1) & ~(kTcTile - 1);   // 0 for pages of <= 128 tokens
          for (int ch = 0; ch < 2; ++ch)
            tma_load_3d(dst + ch * kTcChunk + lane * rows * 128, tm, full, ch * 64, y, z);
        }
      }
      if (is_k) ticket = static_cast<long long>(gridDim.x) + __shfl_sync(0xffffffffu, next_ticket, 0);
    }
    if (leader && (!ok || *abort_flag)) {
      // Loads still in flight must land before the CTA exits.
      for (int k = max(0, jg - kTcStages); k < jg; ++k)
        mbar_wait_drain(is_k ? bar_kfull(k % kTcStages) : bar_vfull(k % kTcStages),
                        (k / kTcStages) & 1, kDrainNs);
      if (is_k)
        for (int k = max(0, uc - 2); k < uc; ++k) mbar_wait_drain(bar_qfull(k & 1), (k >> 1) & 1, kDrainNs);
    }
    }
  } else if (warp == kTcWarpMma) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t FMT = BF16 ? 1u : 0u;
      constexpr uint32_t IDESC_S = idesc_f16(kTcTile, kTcN, FMT, 0u, 0u);   // K-major A, B
      constexpr uint32_t IDESC_O = idesc_f16(kTcD, kTcN, FMT, 1u, 0u);      // A = V^T, MN-major
      bool ok = true, issued = false;
      int uc = -1;                                   // unit of the S side (Q buffer uc % 2)
      int uo = 0;                                    // unit of the P.V side (O^T buffer uo % 2)
      // S^T for tile j (K slot j % 3) with the current unit's Q; frees the K slot (and, on the
      // unit's last tile, the Q buffer) when it completes.
      auto issue_s = [&](int j, bool last_of_unit) {
        const uint32_t ka = base + (j % kTcStages) * kTcStageBytes;
        const uint32_t qa = base + kTcOffQ + (uc & 1) * kTcQBytes;
#pragma unroll
        for (int kk = 0; kk < kTcD / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;
          mma_f16_ss(tmem + 16 * (j & 1), sdesc_k_sw128(ka + (kk >> 2) * kTcChunk + off),
                     sdesc_k_sw128(qa + (kk >> 2) * kTcSmallChunk + off), IDESC_S,
                     kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_s(j & 1));
        mma_commit(bar_kempty(j % kTcStages));
        if (last_of_unit) mma_commit(bar_qempty(uc & 1));
      };
      auto wait_s_inputs = [&](int j, const TcTiles& it) -> bool {
        if (it.unit_first()) {
          ++uc;
          if (!mbar_wait(bar_qfull(uc & 1), (uc >> 1) & 1, wc)) return false;
        }
        if (!mbar_wait(bar_kfull(j % kTcStages), (j / kTcStages) & 1, wc)) return false;
        tc_fence_after();
        return true;
      };
      // Next tile of the unit stream: 1 = a tile, 0 = no more units, -1 = a wait ran out.
      int nu = 0;
      auto advance = [&](TcTiles& it, bool first) -> int {
        if (!first) {
          it.t += kTcTile;
          if (it.t < it.w.t1) return 1;
        }
        TcDesc d;
        if (!ring_read(nu, d)) return -1;
        mbar_arrive(bar_uempty(nu));
        ++nu;
        if (d.b < 0) return 0;
        tc_unit_from(p, d, it.w);
        it.t = it.w.t0;
        return 1;
      };
      TcTiles cur;
      const int r0 = advance(cur, true);
      bool have = r0 == 1;
      if (r0 < 0) ok = false;
      if (have) {
        ok = wait_s_inputs(0, cur);
        if (ok) {
          issue_s(0, cur.unit_last());
          issued = true;
        }
      }
      for (int j = 0; have && ok; ++j) {
        TcTiles nxt = cur;
        const int rn = advance(nxt, false);
        if (rn < 0) { ok = false; break; }
        const bool have_next = rn == 1;
        if (have_next) {
          if (!wait_s_inputs(j + 1, nxt)) { ok = false; break; }
          issue_s(j + 1, nxt.unit_last());
        }
        if (!mbar_wait(bar_p(j & 1), (j >> 1) & 1, wc)) { ok = false; break; }
        if (!mbar_wait(bar_vfull(j % kTcStages), (j / kTcStages) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t va = base + (j % kTcStages) * kTcStageBytes + kTcTileBytes;
        const uint32_t pa = base + kTcOffP + (j & 1) * kTcPBytes;
        const bool acc0 = !cur.unit_first();
#pragma unroll
        for (int kk = 0; kk < kTcTile / 16; ++kk) {
          mma_f16_ss(tmem + 32 + 16 * (uo & 1), sdesc_mn_sw128(va + kk * 2048, kTcChunk),
                     sdesc_k_sw128(pa + (kk >> 2) * kTcSmallChunk + (kk & 3) * 32), IDESC_O,
                     (acc0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar_vempty(j % kTcStages));
        mma_commit(bar_pv);
        if (cur.unit_last()) {
          mma_commit(bar_o(uo & 1));
          ++uo;
        }
        cur = nxt;
        have = have_next;
      }
      if (issued) {
        mma_commit(bar_drain);
        mbar_wait_drain(bar_drain, 0, kDrainNs);
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax warps 0-3
    const int t = threadIdx.x;                       // token of the tile / row d of O^T
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_base;            // S^T[b] at column 16 * b
    const uint32_t tO0 = tmem + lane_base + 32;      // O^T[b] at column 32 + 16 b
    const float c = p.scale_log2;
    uint8_t* pbuf = sbase + kTcOffP;
    int jg = 0, uc = 0, xc = 0;
    bool ok = true;

    // Warp maxima/sums of the GT head values -> combined over the 4 warps (bounded wait).
    auto exchange = [&](float (&v)[GT], bool is_max) -> bool {
#pragma unroll
      for (int h = 0; h < GT; ++h) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float y = __shfl_xor_sync(0xffffffffu, v[h], o);
          v[h] = is_max ? fmaxf(v[h], y) : v[h] + y;
        }
      }
      float* slot = red + (xc & 1) * (4 * kTcN);
      if (lane == 0) {
#pragma unroll
        for (int h = 0; h < GT; ++h) slot[warp * kTcN + h] = v[h];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_x);
      bool got = true;
      if (lane == 0) got = mbar_wait(bar_x, xc & 1, wc);
      got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
      ++xc;
      if (!got) return false;
#pragma unroll
      for (int h = 0; h < GT; ++h) {
        const float a = slot[h], b2 = slot[kTcN + h], c2 = slot[2 * kTcN + h], d2 = slot[3 * kTcN + h];
        v[h] = is_max ? fmaxf(fmaxf(a, b2), fmaxf(c2, d2)) : (a + b2) + (c2 + d2);
      }
      return true;
    };

    // The epilogue of unit k runs after the first P of unit k + 1 (or at the end), so the
    // softmax warps never idle on unit k's last P.V: that product accumulates in O^T[k & 1]
    // while unit k + 1 starts in O^T[(k + 1) & 1].
    TcUnit w_prev;
    float m_prev[GT], l_prev[GT];
    bool have_prev = false;
    auto epilogue = [&]() -> bool {
      const int b = uc & 1;
      bool got = true;
      if (lane == 0) got = mbar_wait(bar_o(b), (uc >> 1) & 1, wc);
      got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
      ++uc;
      have_prev = false;
      if (!got) return false;
      tc_fence_after();
      uint32_t ov[kTcN];
      tmem_ld32x32b_x16(tO0 + 16 * b, ov);           // row d = t of O^T
      float L[GT];
#pragma unroll
      for (int h = 0; h < GT; ++h) L[h] = l_prev[h];
      if (!exchange(L, false)) return false;
#pragma unroll
      for (int h = 0; h < GT; ++h) {
        if (w_prev.g0 + h >= p.G) break;
        const int hq = w_prev.kvh * p.G + w_prev.g0 + h;
        const size_t row = (static_cast<size_t>(w_prev.b) * p.Hq + hq) * p.n_split + w_prev.split;
        p.ws_o[row * kTcD + t] = __uint_as_float(ov[h]) / L[h];
        if (t == 0) p.ws_lse[row] = m_prev[h] + __log2f(L[h]);
      }
      return true;
    };
    int nu = 0;                                      // descriptors read
    for (int uk = 0; ok; ++uk) {                     // uk: units started (O^T buffer uk % 2)
      TcDesc d;
      bool got_d = true;
      if (lane == 0) got_d = ring_read(nu, d);
      if (!__shfl_sync(0xffffffffu, got_d ? 1 : 0, 0)) { ok = false; break; }
      d.b = __shfl_sync(0xffffffffu, d.b, 0);
      d.kvh = __shfl_sync(0xffffffffu, d.kvh, 0);
      d.g0 = __shfl_sync(0xffffffffu, d.g0, 0);
      d.split = __shfl_sync(0xffffffffu, d.split, 0);
      if (lane == 0) mbar_arrive(bar_uempty(nu));
      ++nu;
      if (d.b < 0) break;
      TcUnit w;
      tc_unit_from(p, d, w);
      const uint32_t tO = tO0 + 16 * (uk & 1);
      float m[GT], l[GT];
#pragma unroll
      for (int h = 0; h < GT; ++h) { m[h] = -CUDART_INF_F; l[h] = 0.f; }
      int tile = 0;
      for (int t0 = w.t0; t0 < w.t1; t0 += kTcTile, ++jg, ++tile) {
        bool got = true;
        if (lane == 0) got = mbar_wait(bar_s(jg & 1), (jg >> 1) & 1, wc);
        got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
        if (!got) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[kTcN];
        tmem_ld32x32b_x16(tS + 16 * (jg & 1), sr);
        const bool valid = t0 + t < w.t1;
        float x[GT], mt[GT];
#pragma unroll
        for (int h = 0; h < GT; ++h) {
          x[h] = valid ? __uint_as_float(sr[h]) * c : -CUDART_INF_F;
          mt[h] = x[h];
        }
        if (!exchange(mt, true)) { ok = false; break; }
        bool need = false;
        float alpha[kTcN];
#pragma unroll
        for (int h = 0; h < kTcN; ++h) alpha[h] = 1.f;
#pragma unroll
        for (int h = 0; h < GT; ++h) {
          if (mt[h] > m[h] + 8.0f) {                 // uniform over the CTA
            alpha[h] = (m[h] == -CUDART_INF_F) ? 0.f : ex2_approx(m[h] - mt[h]);
            l[h] *= alpha[h];
            m[h] = mt[h];
            need = need || tile > 0;
          }
        }
        if (need) {                                  // O^T holds earlier tiles of the unit
          // S^T of this tile was issued before P.V of the previous one: wait for that.
          got = true;
          if (lane == 0) got = mbar_wait(bar_pv, (jg - 1) & 1, wc);
          got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
          if (!got) { ok = false; break; }
          tc_fence_after();
          uint32_t ov[kTcN];
          tmem_ld32x32b_x16(tO, ov);
#pragma unroll
          for (int h = 0; h < kTcN; ++h) ov[h] = __float_as_uint(__uint_as_float(ov[h]) * alpha[h]);
          tmem_st32x32b_x16(tO, ov);
          tmem_st_wait();
        }
        // P^T[h][t] (16-bit) into the K-major swizzled P buffer; token t is element t%64
        // of chunk t/64, 16-byte unit (t%64)/8.
        const int ch = t >> 6, e = t & 63, u16 = e >> 3;
        uint8_t* pb = pbuf + (jg & 1) * kTcPBytes;
#pragma unroll
        for (int h = 0; h < GT; ++h) {
          const float mref = (m[h] == -CUDART_INF_F) ? 0.f : m[h];
          const float pr = valid ? ex2_approx(x[h] - mref) : 0.f;
          l[h] += pr;
          const uint32_t pw = pack_half2(pr, 0.f, BF16);
          *reinterpret_cast<uint16_t*>(pb + ch * kTcSmallChunk + h * 128 + ((u16 ^ (h & 7)) << 4) +
                                       (e & 7) * 2) = static_cast<uint16_t>(pw & 0xFFFFu);
        }
        if (__any_sync(0xffffffffu, !valid)) {        // warp-uniform
          // Zero V rows past the split. The V producer may still be filling this slot:
          // wait for it first so the zeros land after the copy.
          got = true;
          if (lane == 0) got = mbar_wait(bar_vfull(jg % kTcStages), (jg / kTcStages) & 1, wc);
          got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
          if (!got) { ok = false; break; }
          if (!valid) {
            uint8_t* vrow = sbase + (jg % kTcStages) * kTcStageBytes + kTcTileBytes + t * 128;
#pragma unroll
            for (int cch = 0; cch < 2; ++cch)
#pragma unroll
              for (int k = 0; k < 8; ++k)
                *reinterpret_cast<uint4*>(vrow + cch * kTcChunk + k * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar_p(jg & 1));
        if (tile == 0 && have_prev && !epilogue()) { ok = false; break; }
      }
      if (!ok) break;
      w_prev = w;
#pragma unroll
      for (int h = 0; h < GT; ++h) { m_prev[h] = m[h]; l_prev[h] = l[h]; }
      have_prev = true;
    }
    if (ok && have_prev) epilogue();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kTcWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcTmemCols);
  }
}

}  // namespace fa
