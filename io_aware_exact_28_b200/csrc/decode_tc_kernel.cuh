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
// Persistent CTAs (one per SM). A work unit is one split (up to split_tokens tokens) of
// one (sequence, KV-head tile); its weight is 4 per 128-token tile plus 1 for its fixed
// work (query load, epilogue). Units are ordered (sequence, head tile, split), splits past
// kv_len do not exist, and CTA c takes the units whose weight prefix starts in
// [c W / grid, (c+1) W / grid), W the total: each CTA gets a contiguous run of units within
// one unit's weight of the average, whatever the kv_len mix. Warp 0 locates the run's
// first unit with a scan over the sequences' weights (a closed form per kv_len) and every
// role walks the same run (TcSched). Warps:
//   0-3  softmax: thread t owns token t of the tile (TMEM lane t of S^T) and row d = t
//        of O^T; warp-level max, cross-warp max through shared memory + an mbarrier,
//        lazy rescale of O^T (threshold 2^8), P^T written to shared memory in the
//        canonical K-major 128-byte-swizzle layout; per-unit epilogue writes the partial.
//   4    K producer: the unit's query rows (TMA, double-buffered) and K tiles.
//   5    TMEM allocator and single-thread tcgen05.mma issuer. S^T of tile j+1 is issued
//        before P.V of tile j, so scores are ready when the softmax warps need them.
//   6    V producer: V tiles.
// K and V have separate ring barriers: a K slot is refilled as soon as its S^T MMA is
// done, a tile before the V slot frees. Tokens of a tile past the split's end are masked
// to -inf and their V rows zeroed in shared memory (rows of the cache past kv_len are never
// used, whatever they hold).
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
// barriers: kfull[3] kempty[3] vfull[3] vempty[3] qfull[2] qempty[2] s[2] p[2] o x pv drain
constexpr int kTcNBars = 4 * kTcStages + 12;
constexpr int kTcOffMisc = kTcOffBar + kTcNBars * 8;
constexpr int kTcOffSched = kTcOffMisc + 16;              // the CTA's first unit (TcSched)
constexpr int kTcSmemBytes = kTcOffSched + 48 + 1024;
constexpr uint32_t kTcTmemCols = 64;                      // S^T x2 [0,32), O^T [32,48)
static_assert(kTcSmemBytes <= 227 * 1024, "shared memory budget");

// Debug builds only (-DFA_TC_TRACE): CTA 0 records clock64() at pipeline events of its
// first 1024 tiles into g_fa_tc_trace[event][tile], read back with fa_debug_tc_trace().
#ifdef FA_TC_TRACE
__device__ long long g_fa_tc_trace[8][1024];
#define FA_TC_EVENT(ev, idx) \
  do { if (blockIdx.x == 0 && (idx) < 1024) g_fa_tc_trace[ev][idx] = clock64(); } while (0)
#else
#define FA_TC_EVENT(ev, idx) do {} while (0)
#endif

struct DecodeTcParams {
  const int* kv_lens;     // [B]
  float* ws_o;            // [B, Hq, n_split, 128]
  float* ws_lse;          // [B, Hq, n_split]
  int B, Hq, Hkv, G, GT;  // GT = heads per tile (<= 16), n_gt tiles per KV head
  int n_gt;
  int max_len, split_tokens, n_split;
  float scale_log2;
  uint64_t timeout_ns;
};

struct TcUnit {
  int b, kvh, g0, split, t0, t1;
};

__device__ __forceinline__ int tc_seq_len(const DecodeTcParams& p, int b) {
  const int len = p.kv_lens[b];
  return len < 0 ? 0 : (len > p.max_len ? p.max_len : len);
}

// Weight of split s of a sequence of length len (0 if the split does not exist).
__device__ __forceinline__ int tc_split_weight(const DecodeTcParams& p, int len, int s) {
  const int t0 = s * p.split_tokens;
  const int n = min(len, t0 + p.split_tokens) - t0;
  return n > 0 ? 4 * ((n + kTcTile - 1) / kTcTile) + 1 : 0;
}

// Weight of all splits of one (sequence, head tile).
__device__ __forceinline__ long long tc_seq_weight(const DecodeTcParams& p, int len) {
  const int full = len / p.split_tokens;
  const long long wf = 4 * (p.split_tokens / kTcTile) + 1;
  return full * wf + tc_split_weight(p, len, full);
}

// Position in this CTA's run of units: sequence b, head tile hg (KV head hg / n_gt), split
// s; pre = weight prefix at the unit's start; the run ends at the first unit with pre >= hi.
struct TcSched {
  int b, hg, s, len;
  long long pre, hi;
  __device__ __forceinline__ bool valid(const DecodeTcParams& p) const { return b < p.B && pre < hi; }
  __device__ __forceinline__ void advance(const DecodeTcParams& p) {
    pre += tc_split_weight(p, len, s);
    if (++s * p.split_tokens < len) return;
    s = 0;
    if (++hg < p.Hkv * p.n_gt) return;
    hg = 0;
    for (++b; b < p.B; ++b) {
      len = tc_seq_len(p, b);
      if (len > 0) break;
    }
  }
  __device__ __forceinline__ void unit(const DecodeTcParams& p, TcUnit& w) const {
    w.b = b;
    w.kvh = hg / p.n_gt;
    w.g0 = (hg - w.kvh * p.n_gt) * p.GT;
    w.split = s;
    w.t0 = s * p.split_tokens;
    w.t1 = min(len, w.t0 + p.split_tokens);
  }
};

// The first unit of CTA blockIdx.x's run (executed by one full warp; lane 0's result).
__device__ __forceinline__ TcSched tc_sched_start(const DecodeTcParams& p) {
  const int lane = threadIdx.x & 31;
  const long long HT = static_cast<long long>(p.Hkv) * p.n_gt;
  long long total = 0;
  for (int b0 = 0; b0 < p.B; b0 += 32) {
    long long v = (b0 + lane < p.B) ? tc_seq_weight(p, tc_seq_len(p, b0 + lane)) : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    total += v;
  }
  total *= HT;
  const long long lo = total * blockIdx.x / gridDim.x;
  TcSched sc;
  sc.b = p.B;
  sc.hg = sc.s = sc.len = 0;
  sc.pre = total;
  sc.hi = total * (blockIdx.x + 1) / gridDim.x;
  long long run = 0;                                   // weight before sequence b0
  for (int b0 = 0; b0 < p.B; b0 += 32) {
    const int b = b0 + lane;
    const int len = b < p.B ? tc_seq_len(p, b) : 0;
    const long long wb = b < p.B ? tc_seq_weight(p, len) * HT : 0;
    long long incl = wb;                               // inclusive scan over the lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, wb > 0 && run + incl > lo);
    if (hit) {
      const int src = __ffs(hit) - 1;
      const long long before = run + __shfl_sync(0xffffffffu, incl - wb, src);
      const int len_b = __shfl_sync(0xffffffffu, len, src);
      const long long w1 = tc_seq_weight(p, len_b);    // one head tile's splits
      const long long q = lo - before;
      sc.b = b0 + src;
      sc.len = len_b;
      sc.hg = static_cast<int>(q / w1);
      const long long r = q - sc.hg * w1;
      const long long wf = 4 * (p.split_tokens / kTcTile) + 1;
      sc.s = static_cast<int>(r / wf);
      sc.pre = before + sc.hg * w1 + sc.s * wf;
      if (sc.pre < lo) sc.advance(p);                  // starts in the previous CTA's share
      break;
    }
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  return sc;
}

// Walks the tiles (128 tokens from t0 to t1) of the units of this CTA's run.
struct TcTiles {
  TcSched sc;
  int t;
  TcUnit w;
  __device__ __forceinline__ bool first(const DecodeTcParams& p, const TcSched& start) {
    sc = start;
    if (!sc.valid(p)) return false;
    sc.unit(p, w);
    t = w.t0;
    return true;
  }
  __device__ __forceinline__ bool next(const DecodeTcParams& p) {
    t += kTcTile;
    if (t < w.t1) return true;
    sc.advance(p);
    if (!sc.valid(p)) return false;
    sc.unit(p, w);
    t = w.t0;
    return true;
  }
  __device__ __forceinline__ bool unit_first() const { return t == w.t0; }
  __device__ __forceinline__ bool unit_last() const { return t + kTcTile >= w.t1; }
};

template <bool BF16, int GT>
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
  const uint32_t bar_o = bar0 + 8u * (4 * kTcStages + 8);    // O^T of a unit complete
  const uint32_t bar_x = bar0 + 8u * (4 * kTcStages + 9);    // cross-warp exchange (4)
  const uint32_t bar_pv = bar0 + 8u * (4 * kTcStages + 10);  // each P.V done
  const uint32_t bar_drain = bar0 + 8u * (4 * kTcStages + 11);
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
    mbar_init(bar_o, 1);
    mbar_init(bar_x, 4);
    mbar_init(bar_pv, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  // P^T buffers start at zero: rows past the head tile stay zero for the whole kernel.
  for (int i = threadIdx.x; i < (2 * kTcPBytes) / 16; i += kTcThreads)
    reinterpret_cast<uint4*>(sbase + kTcOffP)[i] = make_uint4(0, 0, 0, 0);
  TcSched* sched0 = reinterpret_cast<TcSched*>(sbase + kTcOffSched);
  if (warp == 0) {
    const TcSched sc = tc_sched_start(p);
    if (lane == 0) *sched0 = sc;
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
  const TcSched start = *sched0;

  if (warp == kTcWarpKProd || warp == kTcWarpVProd) {
    // ---------------------------------------------------------------- TMA producers
    if (lane == 0) {
      const bool is_k = warp == kTcWarpKProd;
      const CUtensorMap* tm = is_k ? &tmK : &tmV;
      TcTiles cur;
      bool have = cur.first(p, start);
      int jg = 0, uc = 0;
      bool ok = true;
      for (; have && ok; ++jg) {
        if (is_k && cur.unit_first()) {
          // Query rows of the unit: 16 rows from head (b, kvh*G + g0) on (rows past the
          // head tile are loaded but never used); Q buffer uc % 2.
          const int qb = uc & 1;
          if (uc >= 2 && !mbar_wait(bar_qempty(qb), ((uc >> 1) - 1) & 1, wc)) { ok = false; break; }
          mbar_arrive_expect_tx(bar_qfull(qb), kTcQBytes);
          const int row0 = cur.w.b * p.Hq + cur.w.kvh * p.G + cur.w.g0;
          for (int ch = 0; ch < 2; ++ch)
            tma_load_3d(base + kTcOffQ + qb * kTcQBytes + ch * kTcSmallChunk, &tmQ, bar_qfull(qb),
                        ch * 64, row0, 0);
          ++uc;
        }
        const int st = jg % kTcStages;
        const uint32_t empty = is_k ? bar_kempty(st) : bar_vempty(st);
        const uint32_t full = is_k ? bar_kfull(st) : bar_vfull(st);
        if (jg >= kTcStages && !mbar_wait(empty, ((jg / kTcStages) - 1) & 1, wc)) {
          ok = false;
          break;
        }
        if (is_k) FA_TC_EVENT(0, jg);
        mbar_arrive_expect_tx(full, kTcTileBytes);
        const uint32_t dst = base + st * kTcStageBytes + (is_k ? 0 : kTcTileBytes);
        const int bhkv = cur.w.b * p.Hkv + cur.w.kvh;
        for (int ch = 0; ch < 2; ++ch) tma_load_3d(dst + ch * kTcChunk, tm, full, ch * 64, cur.t, bhkv);
        have = cur.next(p);
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
  } else if (warp == kTcWarpMma) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t FMT = BF16 ? 1u : 0u;
      constexpr uint32_t IDESC_S = idesc_f16(kTcTile, kTcN, FMT, 0u, 0u);   // K-major A, B
      constexpr uint32_t IDESC_O = idesc_f16(kTcD, kTcN, FMT, 1u, 0u);      // A = V^T, MN-major
      bool ok = true, issued = false;
      int uc = -1;                                   // unit counter (Q buffer uc % 2)
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
      TcTiles cur;
      bool have = cur.first(p, start);
      if (have) {
        ok = wait_s_inputs(0, cur);
        if (ok) {
          issue_s(0, cur.unit_last());
          issued = true;
        }
      }
      for (int j = 0; have && ok; ++j) {
        TcTiles nxt = cur;
        const bool have_next = nxt.next(p);
        if (have_next) {
          if (!wait_s_inputs(j + 1, nxt)) { ok = false; break; }
          FA_TC_EVENT(1, j + 1);
          issue_s(j + 1, nxt.unit_last());
        }
        if (!mbar_wait(bar_p(j & 1), (j >> 1) & 1, wc)) { ok = false; break; }
        FA_TC_EVENT(2, j);
        if (!mbar_wait(bar_vfull(j % kTcStages), (j / kTcStages) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t va = base + (j % kTcStages) * kTcStageBytes + kTcTileBytes;
        const uint32_t pa = base + kTcOffP + (j & 1) * kTcPBytes;
        const bool acc0 = !cur.unit_first();
#pragma unroll
        for (int kk = 0; kk < kTcTile / 16; ++kk) {
          mma_f16_ss(tmem + 32, sdesc_mn_sw128(va + kk * 2048, kTcChunk),
                     sdesc_k_sw128(pa + (kk >> 2) * kTcSmallChunk + (kk & 3) * 32), IDESC_O,
                     (acc0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar_vempty(j % kTcStages));
        mma_commit(bar_pv);
        if (cur.unit_last()) mma_commit(bar_o);
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
    const uint32_t tO = tmem + lane_base + 32;
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

    for (TcSched sc = start; sc.valid(p) && ok; sc.advance(p)) {
      TcUnit w;
      sc.unit(p, w);
      float m[GT], l[GT];
#pragma unroll
      for (int h = 0; h < GT; ++h) { m[h] = -CUDART_INF_F; l[h] = 0.f; }
      int tile = 0;
      for (int t0 = w.t0; t0 < w.t1; t0 += kTcTile, ++jg, ++tile) {
        bool got = true;
        if (lane == 0) got = mbar_wait(bar_s(jg & 1), (jg >> 1) & 1, wc);
        if (t == 0) FA_TC_EVENT(3, jg);
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
        if (t == 0) FA_TC_EVENT(4, jg);
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
        if (t == 0) FA_TC_EVENT(5, jg);
      }
      if (!ok) break;
      // ------------------------------------------------------------ unit epilogue
      bool got = true;
      if (lane == 0) got = mbar_wait(bar_o, uc & 1, wc);
      got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
      ++uc;
      if (!got) { ok = false; break; }
      tc_fence_after();
      uint32_t ov[kTcN];
      tmem_ld32x32b_x16(tO, ov);                     // row d = t of O^T
      float L[GT];
#pragma unroll
      for (int h = 0; h < GT; ++h) L[h] = l[h];
      if (!exchange(L, false)) { ok = false; break; }
#pragma unroll
      for (int h = 0; h < GT; ++h) {
        if (w.g0 + h >= p.G) break;
        const int hq = w.kvh * p.G + w.g0 + h;
        const size_t row = (static_cast<size_t>(w.b) * p.Hq + hq) * p.n_split + w.split;
        p.ws_o[row * kTcD + t] = __uint_as_float(ov[h]) / L[h];
        if (t == 0) p.ws_lse[row] = m[h] + __log2f(L[h]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kTcWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcTmemCols);
  }
}

}  // namespace fa
