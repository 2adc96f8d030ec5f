// bwd_kernel.cuh — gradients of exact attention (dQ, dK, dV) for sm_100a, by recomputation.
//
// The backward pass keeps no score matrix either: it recomputes the scores tile by tile
// from Q, K and the forward's per-row statistic L (page "Flash Attention" (zh), "IO 感知的
// 算法设计", tiling plus recomputation; page "Flash Attention ... IO-aware exact" (fr), the
// pseudo-code's second output L). With P_ij = exp(scale * q_i . k_j - L_i) recomputed and
// D_i = sum_d dO_id O_id:
//     dV = P^T dO      dP = dO V^T      dS = P * (dP - D)
//     dQ = scale * dS K                  dK = scale * dS^T Q
// Two kernels: fa_bwd_preprocess_kernel, then fa_bwd_fused_kernel, whose grid holds the
// CTAs of both gradient passes (independent of each other):
//   fa_bwd_preprocess_kernel  D and L * log2(e) per query row, padded to whole 128-row
//                             tiles; rows without a visible key and rows past Nq get
//                             +inf, so their P is exactly 0 in both passes below.
//   dQ pass (bwd_dq_tile)     one CTA per 128-row query tile: per key tile j,
//                             S = Q K_j^T and dP = dO V_j^T (tcgen05, TMEM; two dP
//                             buffers), then the elementwise warps form dS and
//                             dQ += dS K_j (A = dS in TMEM); dP(j+1), and dQ(j) once
//                             S(j+1) is issued, run beside the elementwise work.
//   dK/dV pass (bwd_dkdv_tile) one CTA per 128-row key tile of a KV head: per query tile i
//                             of every query head of its group, S^T = K Q_i^T and
//                             dP^T = V dO_i^T; the elementwise warps form P^T, then dS^T,
//                             each released on its own barrier to dV += P^T dO_i and
//                             dK += dS^T Q_i (A operands in TMEM), so that the next step's
//                             P^T pass runs beside dK and the next dP^T. The group's query
//                             heads are summed in TMEM, so no atomics are needed.
// Causal masking is bottom-right aligned as in the forward: key j is visible to query i
// iff j <= i + (Nk - Nq).
#pragma once

#include <cuda.h>
#include <math_constants.h>

#include "sm100.cuh"

namespace fa {

constexpr int kBwdTile = 128;          // query rows and key rows per tile

// Packed fp32 product of two pairs (sm_100 mul.f32x2), beside f2_fma / f2_sub.
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// TMEM column of the 16-bit operand that one 16-element K step kk of a P.X product reads.
// With G elementwise groups, group g owns the streamed columns [g*TN/G, (g+1)*TN/G) of S
// and dP and packs its share of P (or dS) at the start of that range, so K step kk lies in
// the range of group (16 kk) / (TN/G), at packed column (16 kk - g*TN/G) / 2 past its start.
template <int TN, int G>
__device__ __forceinline__ uint32_t packed_col(int kk) {
  const int g = (16 * kk) / (TN / G);
  return static_cast<uint32_t>(g * (TN / G) + (16 * kk - g * (TN / G)) / 2);
}

struct BwdParams {
  const float* lse2;      // [B*Hq, Nq_pad] L * log2(e), +inf where P must be 0
  const float* dsum;      // [B*Hq, Nq_pad] D
  void* out;              // dq [B*Hq, Nq, D] (dQ kernel) or dk [B*Hkv, Nk, D] (dK/dV kernel)
  void* out2;             // dv [B*Hkv, Nk, D] (dK/dV kernel)
  int Hq, Hkv, group;
  int Nq, Nk, Nq_pad;
  int causal_offset;      // Nk - Nq
  float scale, scale_log2;
  uint64_t timeout_ns;
  int skip_resident_load;   // test hook: the resident tiles are never loaded
};

// ------------------------------------------------------------------------------------
// D_i = sum_d dO_id O_id and L_i * log2(e), padded per head to Nq_pad rows.
// D/8 threads per row, each loading 16 bytes (8 elements) of O and of dO; the row's
// partial sums meet by shuffles within its group of lanes. The grid covers
// BH * Nq_pad * (D/8) threads; lanes past the end only take part in the shuffles.
template <int D, bool BF16>
__global__ void __launch_bounds__(256)
fa_bwd_preprocess_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
                         const float* __restrict__ lse, float* __restrict__ lse2,
                         float* __restrict__ dsum, int BH, int Nq, int Nq_pad) {
  constexpr int TPR = D / 8;                          // threads per row (8 or 16)
  const long long gt = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long rowid = gt / TPR;
  const int sub = static_cast<int>(gt - rowid * TPR);
  const bool valid = rowid < static_cast<long long>(BH) * Nq_pad;
  const int bh = valid ? static_cast<int>(rowid / Nq_pad) : 0;
  const int row = valid ? static_cast<int>(rowid - static_cast<long long>(bh) * Nq_pad) : 0;
  float acc = 0.f;
  if (valid && row < Nq) {
    const size_t off = (static_cast<size_t>(bh) * Nq + row) * D + sub * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(o + off);
    const uint4 g = *reinterpret_cast<const uint4*>(dout + off);
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float o0, o1, g0, g1;
      unpack_half2(av[e], o0, o1, BF16);
      unpack_half2(gv[e], g0, g1, BF16);
      acc = fmaf(o0, g0, fmaf(o1, g1, acc));
    }
  }
#pragma unroll
  for (int m = TPR / 2; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  if (valid && sub == 0) {
    const float l = row < Nq ? lse[static_cast<size_t>(bh) * Nq + row] : -CUDART_INF_F;
    lse2[static_cast<size_t>(bh) * Nq_pad + row] =
        (l == -CUDART_INF_F) ? CUDART_INF_F : l * 1.4426950408889634f;
    dsum[static_cast<size_t>(bh) * Nq_pad + row] = acc;
  }
}

// Per head-dimension configuration. Each CTA keeps one 128-row tile resident (Q and dO
// in the dQ pass, K and V in the dK/dV pass) and streams the other side in tiles of TN
// rows. d = 64 streams 64-row tiles, so that TMEM (S | dP | accumulators | second dP)
// fits in 256 columns and shared memory in half an SM, two CTAs per SM; d = 128 streams
// 128-row tiles, one CTA per SM. Within a CTA the products of one step overlap the
// elementwise work of another (see the two passes below).
template <int D>
struct BwdCfg {
  static constexpr int TN = (D == 64) ? 64 : 128;    // rows of a streamed tile
  static constexpr int CTAS = (D == 64) ? 2 : 1;     // resident CTAs per SM
  // Elementwise groups of 4 warps (128 rows each), each taking TN/G streamed columns:
  // two at d = 128 (one CTA per SM), one at d = 64, where a second group measured slower
  // (two CTAs already share the SM, and registers are capped at 96 per thread).
  static constexpr int G = (D == 64) ? 1 : 2;
  static constexpr int EW_THREADS = 128 * G;
  static constexpr int WARP_PROD = 4 * G;
  static constexpr int WARP_MMA = 4 * G + 1;
  static constexpr int THREADS = 32 * (4 * G + 2);
  static constexpr int NCH = D / 64;                 // 128-byte swizzle chunks along d
  static constexpr int CHUNK = kBwdTile * 128;       // resident tile: 128 rows x 128 bytes
  static constexpr int SCHUNK = TN * 128;            // streamed tile: TN rows x 128 bytes
  static constexpr int TILE_BYTES = kBwdTile * D * 2;
  static constexpr int STILE_BYTES = TN * D * 2;
  static constexpr int NS = (D == 64) ? 8 : 4;       // ring items (one streamed tile each)
  static constexpr int A_OFF = 0;                    // dQ: Q, dO;  dK/dV: K, V
  static constexpr int RING_OFF = 2 * TILE_BYTES;
  static constexpr int VEC_OFF = RING_OFF + NS * STILE_BYTES;  // dK/dV: L and D per ring pair
  static constexpr int BAR_OFF = VEC_OFF + (NS / 2) * 2 * TN * 4;
  static constexpr int NBARS = 1 + 2 * NS + 6;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = (D == 64) ? 256 : 512;
  static constexpr uint32_t P_COL = TN;              // dP (dQ kernel) / dP^T (dK/dV kernel)
  static constexpr uint32_t ACC_COL = 2 * TN;        // dQ, or dV then dK
  static constexpr uint32_t DP1_COL = ACC_COL + D;   // dQ kernel: dP of odd key tiles
  static_assert(SMEM_BYTES * CTAS <= 227 * 1024, "shared memory budget");
  static_assert(ACC_COL + 2 * D <= TMEM_COLS, "TMEM budget");
  static_assert(DP1_COL + TN <= TMEM_COLS, "TMEM budget (second dP buffer)");
};

// ------------------------------------------------------------------------------------
// dQ: CTA (query tile qt, head bh), key tiles of TN rows. TMEM: S [0,TN), dP of even key
// tiles [TN,2TN), dQ [2TN, 2TN+D), dP of odd key tiles [2TN+D, 3TN+D); dS(j) is packed
// over the first TN/2 columns of its step's dP buffer. Once step j's elementwise work is
// done the tensor core computes S(j+1), which is all step j+1 waits for (its dP was
// computed earlier), then dQ += dS(j) K_j and dP(j+2) into the buffer dS(j) leaves, both
// beside step j+1's elementwise work. The producer loads V ahead of K (order K_0, V_0,
// V_1, K_1, V_2, K_2, ...), so that each V tile's ring slot, freed by the dP two steps
// back, is filled before it is needed.
template <int D, bool BF16, bool CAUSAL>
__device__ __forceinline__ void bwd_dq_tile(const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                            const CUtensorMap& tmV, const CUtensorMap& tmDO,
                                            const BwdParams& p, const int tile, const int bh) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = bh / p.Hq, h = bh - b * p.Hq;
  const int bh_kv = b * p.Hkv + h / p.group;
  constexpr int TN = C::TN;
  const int q0 = tile * kBwdTile;
  const int n_kv_total = (p.Nk + TN - 1) / TN;
  int n_kv = n_kv_total;
  if (CAUSAL) {
    const int kmax = min(q0 + kBwdTile - 1, p.Nq - 1) + p.causal_offset;
    n_kv = kmax < 0 ? 0 : min(n_kv_total, kmax / TN + 1);
  }

  const uint32_t bar0 = base + C::BAR_OFF;
  const uint32_t bar_a = bar0;                                       // Q and dO landed
  auto bar_full = [&](int i) { return bar0 + 8u * (1 + i); };
  auto bar_empty = [&](int i) { return bar0 + 8u * (1 + C::NS + i); };
  const uint32_t bar_s = bar0 + 8u * (1 + 2 * C::NS);                // S and dP ready
  const uint32_t bar_ds = bar0 + 8u * (2 + 2 * C::NS);               // dS in TMEM (128 rows)
  const uint32_t bar_done = bar0 + 8u * (3 + 2 * C::NS);             // every MMA done
  const uint32_t bar_drain = bar0 + 8u * (4 + 2 * C::NS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + C::MISC_OFF + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar_a, 1);
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(bar_full(i), 1);
      mbar_init(bar_empty(i), 1);
    }
    mbar_init(bar_s, 1);
    mbar_init(bar_ds, C::EW_THREADS);
    mbar_init(bar_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == C::WARP_MMA) tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, &g_fa_status, p.timeout_ns};

  if (warp == C::WARP_PROD) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && n_kv > 0) {
      mbar_arrive_expect_tx(bar_a, 2 * C::TILE_BYTES);
      for (int ch = 0; ch < C::NCH && !p.skip_resident_load; ++ch) {
        tma_load_3d(base + C::A_OFF + ch * C::CHUNK, &tmQ, bar_a, ch * 64, q0, bh);
        tma_load_3d(base + C::A_OFF + C::TILE_BYTES + ch * C::CHUNK, &tmDO, bar_a, ch * 64, q0, bh);
      }
      int it = 0;
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        for (int x = 0; x < 2; ++x) {                   // K_0, V_0; then V_j, K_j
          const int kv = (j == 0) ? x : 1 - x;
          const int slot = it % C::NS, round = it / C::NS;
          if (round > 0 && !mbar_wait(bar_empty(slot), (round - 1) & 1, wc)) { ok = false; break; }
          mbar_arrive_expect_tx(bar_full(slot), C::STILE_BYTES);
          for (int ch = 0; ch < C::NCH; ++ch)
            tma_load_3d(base + C::RING_OFF + slot * C::STILE_BYTES + ch * C::SCHUNK, kv ? &tmV : &tmK,
                        bar_full(slot), ch * 64, j * TN, bh_kv);
          ++it;
        }
      }
      if (!ok || *abort_flag) {
        for (int i = max(0, it - C::NS); i < it; ++i)
          mbar_wait_drain(bar_full(i % C::NS), (i / C::NS) & 1, kDrainNs);
        mbar_wait_drain(bar_a, 0, kDrainNs);
      }
    }
  } else if (warp == C::WARP_MMA) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t IDESC_S = idesc_f16(kBwdTile, TN, BF16 ? 1u : 0u, 0u, 0u);
      constexpr uint32_t IDESC_Q = idesc_f16(kBwdTile, D, BF16 ? 1u : 0u, 0u, 1u);
      // X[cols col, +TN) = A[128 x D] B[TN x D]^T, both K-major (d contiguous).
      auto issue_abt = [&](uint32_t col, uint32_t a, uint32_t bt) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;
          mma_f16_ss(tmem + col, sdesc_k_sw128(a + (kk >> 2) * C::CHUNK + koff),
                     sdesc_k_sw128(bt + (kk >> 2) * C::SCHUNK + koff), IDESC_S, kk > 0 ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(bar_a, 0, wc);
      bool issued = false;
      tc_fence_after();
      const uint32_t qa = base + C::A_OFF, doa = base + C::A_OFF + C::TILE_BYTES;
      // Ring items in load order: K_0 = 0, V_0 = 1, then V_j = 2j, K_j = 2j + 1.
      auto k_item = [](int j) { return j == 0 ? 0 : 2 * j + 1; };
      auto v_item = [](int j) { return j == 0 ? 1 : 2 * j; };
      auto item_addr = [&](int it) { return base + C::RING_OFF + (it % C::NS) * C::STILE_BYTES; };
      auto wait_item = [&](int it) { return mbar_wait(bar_full(it % C::NS), (it / C::NS) & 1, wc); };
      auto dp_col = [](int j) { return (j & 1) ? C::DP1_COL : C::P_COL; };
      // Steps 0 and 1: S(0), dP(0), then dP(1) into the other buffer.
      if (ok && wait_item(k_item(0)) && wait_item(v_item(0))) {
        tc_fence_after();
        issue_abt(0, qa, item_addr(k_item(0)));                 // S = Q K_0^T
        issue_abt(dp_col(0), doa, item_addr(v_item(0)));        // dP = dO V_0^T
        issued = true;
        mma_commit(bar_s);
        mma_commit(bar_empty(v_item(0) % C::NS));               // V_0 no longer needed
        if (n_kv > 1) {
          if (wait_item(v_item(1))) {
            tc_fence_after();
            issue_abt(dp_col(1), doa, item_addr(v_item(1)));
            mma_commit(bar_empty(v_item(1) % C::NS));
          } else {
            ok = false;
          }
        }
      } else {
        ok = false;
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        // Step j's elementwise work done: S is free, dS(j) is packed over dP buffer j & 1.
        if (!mbar_wait(bar_ds, j & 1, wc)) { ok = false; break; }
        tc_fence_after();
        if (j + 1 < n_kv) {                                     // S(j+1): step j+1 ready
          if (!wait_item(k_item(j + 1))) { ok = false; break; }
          tc_fence_after();
          issue_abt(0, qa, item_addr(k_item(j + 1)));
          mma_commit(bar_s);
        }
        // dQ += dS K_j: A = dS (packed 16-bit in TMEM, per elementwise group), B = K_j MN-major.
        const uint32_t ka = item_addr(k_item(j));
#pragma unroll
        for (int kk = 0; kk < TN / 16; ++kk)
          mma_f16_ts(tmem + C::ACC_COL, tmem + dp_col(j) + packed_col<TN, C::G>(kk),
                     sdesc_mn_sw128(ka + kk * 2048, C::SCHUNK), IDESC_Q, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar_empty(k_item(j) % C::NS));
        if (j + 2 < n_kv) {                                     // dP(j+2), after dQ(j) read dS(j)
          if (!wait_item(v_item(j + 2))) { ok = false; break; }
          tc_fence_after();
          issue_abt(dp_col(j + 2), doa, item_addr(v_item(j + 2)));
          mma_commit(bar_empty(v_item(j + 2) % C::NS));
        }
      }
      if (issued) mma_commit(ok ? bar_done : bar_drain);
      if (issued && !ok) mbar_wait_drain(bar_drain, 0, kDrainNs);
    }
  } else {
    // ------------------------------------------------------------------ elementwise + epilogue
    // Group g = warp / 4 takes key columns [g*TN/G, (g+1)*TN/G) of every row; warp w reads
    // TMEM lanes 32*(w % 4) .. +31, i.e. rows r of the tile.
    constexpr int G = C::G;
    const int g = (G == 1) ? 0 : (warp >> 2);
    const int r = (warp & 3) * 32 + lane;                   // query row of the tile
    const int row = q0 + r;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + g * (TN / G);
    const uint32_t tQ = tmem + lane_base + C::ACC_COL + g * (D / G);
    const float lse2 = p.lse2[static_cast<size_t>(bh) * p.Nq_pad + row];
    const float dsum = p.dsum[static_cast<size_t>(bh) * p.Nq_pad + row];
    const int lim = CAUSAL ? min(row + p.causal_offset, p.Nk - 1) : p.Nk - 1;
    const int lim_min = CAUSAL ? min(q0 + p.causal_offset, p.Nk - 1) : p.Nk - 1;
    const float c = p.scale_log2;
    const uint64_t c2 = f2_pack(c, c), nl2 = f2_pack(-lse2, -lse2), dsum2 = f2_pack(dsum, dsum);
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(bar_s, j & 1, wc))) { ok = false; break; }
      tc_fence_after();
      const int key0 = j * TN + g * (TN / G);                // first key of this group's columns
      const bool masked = key0 + TN / G - 1 > lim_min;       // warp-uniform per CTA
      const uint32_t tP = tS + ((j & 1) ? C::DP1_COL : C::P_COL);   // this step's dP buffer
#pragma unroll
      for (int cc = 0; cc < TN / (32 * G); ++cc) {
        uint32_t s[32], dp[32];
        tmem_ld32x32b_x32(tS + 32 * cc, s);
        tmem_ld32x32b_x32(tP + 32 * cc, dp);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          // Pair (2i, 2i+1) in packed fp32: P = 2^(s*c - L), dS = P (dP - D).
          const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1])),
                                     c2, nl2);
          float x0, x1;
          f2_unpack(x2, x0, x1);
          float pv[2] = {ex2_approx(x0), ex2_approx(x1)};
#pragma unroll
          for (int e = 0; e < 2; ++e)
            if (masked && key0 + 32 * cc + 2 * i + e > lim) pv[e] = 0.f;
          const uint64_t d2 = f2_mul(f2_pack(pv[0], pv[1]),
                                     f2_sub(f2_pack(__uint_as_float(dp[2 * i]), __uint_as_float(dp[2 * i + 1])),
                                            dsum2));
          float d0, d1;
          f2_unpack(d2, d0, d1);
          pk[i] = pack_half2(d0, d1, BF16);
        }
        tmem_st32x32b_x16(tP + 16 * cc, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_ds);
    }
    if (ok && n_kv > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_done, 0, wc));
    if (ok) {
      tc_fence_after();
      // dQ = scale * (dS K), rows past Nq skipped; a tile without keys writes zeros. Group g
      // writes columns [g*D/G, (g+1)*D/G) of the row.
      const bool row_ok = row < p.Nq;
      uint16_t* orow = static_cast<uint16_t*>(p.out) +
                       (static_cast<size_t>(bh) * p.Nq + (row_ok ? row : 0)) * D + g * (D / G);
#pragma unroll
      for (int ch = 0; ch < D / (32 * G); ++ch) {
        uint32_t a[32];
        if (n_kv > 0) {
          tmem_ld32x32b_x32(tQ + 32 * ch, a);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = 0u;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 w;
          w.x = pack_half2(__uint_as_float(a[8 * u + 0]) * p.scale, __uint_as_float(a[8 * u + 1]) * p.scale, BF16);
          w.y = pack_half2(__uint_as_float(a[8 * u + 2]) * p.scale, __uint_as_float(a[8 * u + 3]) * p.scale, BF16);
          w.z = pack_half2(__uint_as_float(a[8 * u + 4]) * p.scale, __uint_as_float(a[8 * u + 5]) * p.scale, BF16);
          w.w = pack_half2(__uint_as_float(a[8 * u + 6]) * p.scale, __uint_as_float(a[8 * u + 7]) * p.scale, BF16);
          if (row_ok) *reinterpret_cast<uint4*>(orow + 32 * ch + 8 * u) = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------------
// dK, dV: CTA (key tile kt, KV head bh_kv). K and V are loaded once; each step brings
// Q_i and dO_i of one TN-row query tile of one query head of the group (a 2-item ring
// pair) plus that tile's L * log2(e) and D vectors. TMEM: S^T [0,TN) (P^T packed over its
// first TN/2 columns), dP^T [TN,2TN) (dS^T packed over its first TN/2), dV [2TN, 2TN+D),
// dK [2TN+D, 2TN+2D). Barriers per step: S^T ready, dP^T ready (MMA -> elementwise);
// P^T written, dS^T written (elementwise -> MMA). Products in the order dV(s), S^T(s+1)
// over P^T(s), dK(s), dP^T(s+1) over dS^T(s).
template <int D, bool BF16, bool CAUSAL>
__device__ __forceinline__ void bwd_dkdv_tile(const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                              const CUtensorMap& tmV, const CUtensorMap& tmDO,
                                              const BwdParams& p, const int tile, const int bh_kv) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = bh_kv / p.Hkv, hk = bh_kv - b * p.Hkv;
  constexpr int TN = C::TN;
  const int k0 = tile * kBwdTile;
  const int n_q = (p.Nq + TN - 1) / TN;
  // Query tiles that see any key of this tile: queries i with k0 <= i + offset.
  int q_first = 0;
  if (CAUSAL) {
    const int need = k0 - p.causal_offset;                  // smallest visible query row
    q_first = need <= 0 ? 0 : min(n_q, need / TN);
  }
  const int per_head = n_q - q_first;
  const int n_steps = per_head * p.group;                   // (head of the group, tile)
  auto step_of = [&](int s, int& h, int& q0) {
    const int g = s / max(per_head, 1);
    h = hk * p.group + g;
    q0 = (q_first + (s - g * per_head)) * TN;
  };

  const uint32_t bar0 = base + C::BAR_OFF;
  const uint32_t bar_a = bar0;                                       // K and V landed
  auto bar_full = [&](int i) { return bar0 + 8u * (1 + i); };        // pair slot i (Q, dO, vecs)
  auto bar_empty = [&](int i) { return bar0 + 8u * (1 + C::NS + i); };
  const uint32_t bar_s = bar0 + 8u * (1 + 2 * C::NS);                // S^T ready
  const uint32_t bar_ps = bar0 + 8u * (2 + 2 * C::NS);               // dS^T in TMEM (128 rows)
  const uint32_t bar_done = bar0 + 8u * (3 + 2 * C::NS);
  const uint32_t bar_drain = bar0 + 8u * (4 + 2 * C::NS);
  const uint32_t bar_pp = bar0 + 8u * (5 + 2 * C::NS);               // P^T in TMEM (128 rows)
  const uint32_t bar_dp = bar0 + 8u * (6 + 2 * C::NS);               // dP^T ready
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + C::MISC_OFF + 4);
  constexpr int NP = C::NS / 2;                                      // ring pairs

  if (threadIdx.x == 0) {
    mbar_init(bar_a, 1);
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(bar_full(i), 1);
      mbar_init(bar_empty(i), 1);
    }
    mbar_init(bar_s, 1);
    mbar_init(bar_ps, C::EW_THREADS);
    mbar_init(bar_pp, C::EW_THREADS);
    mbar_init(bar_dp, 1);
    mbar_init(bar_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == C::WARP_MMA) tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, &g_fa_status, p.timeout_ns};
  auto q_tile = [&](int slot) { return base + C::RING_OFF + (2 * slot) * C::STILE_BYTES; };
  auto do_tile = [&](int slot) { return base + C::RING_OFF + (2 * slot + 1) * C::STILE_BYTES; };
  auto vec = [&](int slot) { return sbase + C::VEC_OFF + slot * 2 * TN * 4; };

  if (warp == C::WARP_PROD) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && n_steps > 0) {
      mbar_arrive_expect_tx(bar_a, 2 * C::TILE_BYTES);
      for (int ch = 0; ch < C::NCH && !p.skip_resident_load; ++ch) {
        tma_load_3d(base + C::A_OFF + ch * C::CHUNK, &tmK, bar_a, ch * 64, k0, bh_kv);
        tma_load_3d(base + C::A_OFF + C::TILE_BYTES + ch * C::CHUNK, &tmV, bar_a, ch * 64, k0, bh_kv);
      }
      bool ok = true;
      int s = 0;
      for (; s < n_steps && ok; ++s) {
        const int slot = s % NP, round = s / NP;
        if (round > 0 && !mbar_wait(bar_empty(slot), (round - 1) & 1, wc)) { ok = false; break; }
        int h, q0;
        step_of(s, h, q0);
        const int bhq = b * p.Hq + h;
        mbar_arrive_expect_tx(bar_full(slot), 2 * C::STILE_BYTES + 2 * TN * 4);
        for (int ch = 0; ch < C::NCH; ++ch) {
          tma_load_3d(q_tile(slot) + ch * C::SCHUNK, &tmQ, bar_full(slot), ch * 64, q0, bhq);
          tma_load_3d(do_tile(slot) + ch * C::SCHUNK, &tmDO, bar_full(slot), ch * 64, q0, bhq);
        }
        const size_t vrow = static_cast<size_t>(bhq) * p.Nq_pad + q0;
        bulk_load(smem_u32(vec(slot)), p.lse2 + vrow, TN * 4, bar_full(slot));
        bulk_load(smem_u32(vec(slot) + TN * 4), p.dsum + vrow, TN * 4, bar_full(slot));
      }
      if (!ok || *abort_flag) {
        for (int i = max(0, s - NP); i < s; ++i)
          mbar_wait_drain(bar_full(i % NP), (i / NP) & 1, kDrainNs);
        mbar_wait_drain(bar_a, 0, kDrainNs);
      }
    }
  } else if (warp == C::WARP_MMA) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_steps > 0) {
      constexpr uint32_t IDESC_S = idesc_f16(kBwdTile, TN, BF16 ? 1u : 0u, 0u, 0u);
      constexpr uint32_t IDESC_G = idesc_f16(kBwdTile, D, BF16 ? 1u : 0u, 0u, 1u);
      // X[cols col, +TN) = A[128 x D] (resident) B[TN x D]^T (streamed), both K-major.
      auto issue_abt = [&](uint32_t col, uint32_t a, uint32_t bt) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;
          mma_f16_ss(tmem + col, sdesc_k_sw128(a + (kk >> 2) * C::CHUNK + koff),
                     sdesc_k_sw128(bt + (kk >> 2) * C::SCHUNK + koff), IDESC_S, kk > 0 ? 1u : 0u);
        }
      };
      // X[acc] += A[128 x TN] (packed 16-bit in TMEM from col a, per elementwise group)
      // B[TN x D] (streamed, MN-major).
      auto issue_tb = [&](uint32_t acc, uint32_t a, uint32_t bmn, bool acc0) {
#pragma unroll
        for (int kk = 0; kk < TN / 16; ++kk)
          mma_f16_ts(tmem + acc, tmem + a + packed_col<TN, C::G>(kk), sdesc_mn_sw128(bmn + kk * 2048, C::SCHUNK),
                     IDESC_G, (acc0 || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(bar_a, 0, wc);
      bool issued = false;
      tc_fence_after();
      const uint32_t ka = base + C::A_OFF, va = base + C::A_OFF + C::TILE_BYTES;
      // Order: S^T(0), dP^T(0); then per step s: dV(s) once P^T(s) is written, S^T(s+1)
      // over it; dK(s) once dS^T(s) is written, dP^T(s+1) over it. The elementwise warps'
      // P^T pass of step s+1 then runs beside dK(s) and dP^T(s+1).
      if (ok && mbar_wait(bar_full(0), 0, wc)) {
        tc_fence_after();
        issue_abt(0, ka, q_tile(0));                    // S^T = K Q_0^T
        issued = true;
        mma_commit(bar_s);
        issue_abt(C::P_COL, va, do_tile(0));            // dP^T = V dO_0^T
        mma_commit(bar_dp);
      } else {
        ok = false;
      }
      for (int s = 0; s < n_steps && ok; ++s) {
        const int slot = s % NP, nslot = (s + 1) % NP;
        const bool next = s + 1 < n_steps;
        if (!mbar_wait(bar_pp, s & 1, wc)) { ok = false; break; }
        tc_fence_after();
        issue_tb(C::ACC_COL, 0, do_tile(slot), s > 0);          // dV += P^T dO_i
        if (next) {
          if (!mbar_wait(bar_full(nslot), ((s + 1) / NP) & 1, wc)) { ok = false; break; }
          tc_fence_after();
          issue_abt(0, ka, q_tile(nslot));                      // S^T(s+1), after dV(s)
          mma_commit(bar_s);
        }
        if (!mbar_wait(bar_ps, s & 1, wc)) { ok = false; break; }
        tc_fence_after();
        issue_tb(C::ACC_COL + D, C::P_COL, q_tile(slot), s > 0);  // dK += dS^T Q_i
        mma_commit(bar_empty(slot));
        if (next) {
          issue_abt(C::P_COL, va, do_tile(nslot));              // dP^T(s+1), after dK(s)
          mma_commit(bar_dp);
        }
      }
      if (issued) mma_commit(ok ? bar_done : bar_drain);
      if (issued && !ok) mbar_wait_drain(bar_drain, 0, kDrainNs);
    }
  } else {
    // ------------------------------------------------------------------ elementwise + epilogue
    // Group g = warp / 4 takes query columns [g*TN/G, (g+1)*TN/G) of every key row; warp w
    // reads TMEM lanes 32*(w % 4) .. +31. In the epilogue, with two groups group 0 writes
    // dV and group 1 dK; a single group writes both.
    constexpr int G = C::G;
    const int g = (G == 1) ? 0 : (warp >> 2);
    const int r = (warp & 3) * 32 + lane;                   // key row of the tile
    const int key = k0 + r;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + g * (TN / G), tP = tS + C::P_COL;
    const uint32_t tV = tmem + lane_base + C::ACC_COL, tK = tV + D;
    const float c = p.scale_log2;
    const uint64_t c2 = f2_pack(c, c);
    bool ok = true;
    for (int s = 0; s < n_steps; ++s) {
      const int slot = s % NP;
      // The vectors of this step landed with its Q tile (the MMA warp waited for them too).
      if (!__all_sync(0xffffffffu, mbar_wait(bar_full(slot), (s / NP) & 1, wc))) { ok = false; break; }
      if (!__all_sync(0xffffffffu, mbar_wait(bar_s, s & 1, wc))) { ok = false; break; }
      tc_fence_after();
      int h, q0;
      step_of(s, h, q0);
      const float* lv = reinterpret_cast<const float*>(vec(slot));
      const float* dv = lv + TN;
      // Key `key` is visible to query q0 + col iff key <= q0 + col + offset.
      const int first_vis = key - p.causal_offset - q0;     // smallest visible column
      const bool masked = CAUSAL && __any_sync(0xffffffffu, first_vis > 0);
      // Pass 1: P^T = 2^(S^T c - L) for this group's TN/G columns, kept in fp32 for pass 2
      // and stored packed over S^T's columns, then released to the dV product.
      constexpr int NCOL = TN / G;
      float pf[NCOL];
#pragma unroll
      for (int cc = 0; cc < NCOL / 32; ++cc) {
        uint32_t st[32];
        tmem_ld32x32b_x32(tS + 32 * cc, st);
        uint32_t pk[16];
        // This chunk's 32 columns of L, read as 16-byte shared-memory loads (the same address
        // in every lane: one broadcast each), four columns (two pairs) per load.
        const float4* l4 = reinterpret_cast<const float4*>(lv + g * NCOL + 32 * cc);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 lq = l4[q];
          const float lcol[4] = {lq.x, lq.y, lq.z, lq.w};
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int i = 2 * q + hh;
            // Pair (2i, 2i+1) in packed fp32: x = s*c - L, P = 2^x.
            const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(st[2 * i]), __uint_as_float(st[2 * i + 1])),
                                       c2, f2_pack(-lcol[2 * hh], -lcol[2 * hh + 1]));
            float x0, x1;
            f2_unpack(x2, x0, x1);
            float pv[2] = {ex2_approx(x0), ex2_approx(x1)};
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int col = g * NCOL + 32 * cc + 2 * i + e;
              if (masked && col < first_vis) pv[e] = 0.f;
              pf[32 * cc + 2 * i + e] = pv[e];
            }
            pk[i] = pack_half2(pv[0], pv[1], BF16);
          }
        }
        tmem_st32x32b_x16(tS + 16 * cc, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_pp);
      // Pass 2: dS^T = P^T (dP^T - D), stored packed over dP^T's columns.
      if (!__all_sync(0xffffffffu, mbar_wait(bar_dp, s & 1, wc))) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < NCOL / 32; ++cc) {
        uint32_t dpt[32];
        tmem_ld32x32b_x32(tP + 32 * cc, dpt);
        uint32_t dk[16];
        const float4* d4 = reinterpret_cast<const float4*>(dv + g * NCOL + 32 * cc);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 dq = d4[q];
          const float dcol[4] = {dq.x, dq.y, dq.z, dq.w};
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int i = 2 * q + hh;
            const uint64_t ds2 = f2_mul(f2_pack(pf[32 * cc + 2 * i], pf[32 * cc + 2 * i + 1]),
                                        f2_sub(f2_pack(__uint_as_float(dpt[2 * i]),
                                                       __uint_as_float(dpt[2 * i + 1])),
                                               f2_pack(dcol[2 * hh], dcol[2 * hh + 1])));
            float ds0, ds1;
            f2_unpack(ds2, ds0, ds1);
            dk[i] = pack_half2(ds0, ds1, BF16);
          }
        }
        tmem_st32x32b_x16(tP + 16 * cc, dk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_ps);
    }
    if (ok && n_steps > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_done, 0, wc));
    if (ok) {
      tc_fence_after();
      const bool row_ok = key < p.Nk;
      const size_t orow = (static_cast<size_t>(bh_kv) * p.Nk + (row_ok ? key : 0)) * D;
#pragma unroll
      for (int which = g; which < 2; which += G) {          // dV, then dK (times scale)
        uint16_t* dst = static_cast<uint16_t*>(which ? p.out : p.out2) + orow;
        const float f = which ? p.scale : 1.0f;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t a[32];
          if (n_steps > 0) {
            tmem_ld32x32b_x32((which ? tK : tV) + 32 * ch, a);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) a[i] = 0u;
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 w;
            w.x = pack_half2(__uint_as_float(a[8 * u + 0]) * f, __uint_as_float(a[8 * u + 1]) * f, BF16);
            w.y = pack_half2(__uint_as_float(a[8 * u + 2]) * f, __uint_as_float(a[8 * u + 3]) * f, BF16);
            w.z = pack_half2(__uint_as_float(a[8 * u + 4]) * f, __uint_as_float(a[8 * u + 5]) * f, BF16);
            w.w = pack_half2(__uint_as_float(a[8 * u + 6]) * f, __uint_as_float(a[8 * u + 7]) * f, BF16);
            if (row_ok) *reinterpret_cast<uint4*>(dst + 32 * ch + 8 * u) = w;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Both gradient passes in one grid: the dK/dV CTAs first, then the dQ CTAs, each set
// heaviest causal tile first (key tile 0 sees the most queries; the last query tile the
// most keys), so that dQ work fills the SMs the last dK/dV wave leaves idle. The two
// passes are independent: both read only Q, K, V, dO and the preprocessed L and D.
template <int D, bool BF16, bool CAUSAL>
__global__ void __launch_bounds__(BwdCfg<D>::THREADS, BwdCfg<D>::CTAS)
fa_bwd_fused_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKs,
                    const __grid_constant__ CUtensorMap tmVs, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmQs, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDOs,
                    const BwdParams pq, const BwdParams pk, const int n_k, const int n_q,
                    const int BHkv, const int BH) {
  const int bid = blockIdx.x;
  const int n_kv_blocks = n_k * BHkv;
  if (bid < n_kv_blocks) {
    const int kt = bid / BHkv;
    bwd_dkdv_tile<D, BF16, CAUSAL>(tmQs, tmK, tmV, tmDOs, pk, kt, bid - kt * BHkv);
  } else {
    const int c = bid - n_kv_blocks;
    const int r = c / BH;
    bwd_dq_tile<D, BF16, CAUSAL>(tmQ, tmKs, tmVs, tmDO, pq, n_q - 1 - r, c - r * BH);
  }
}

}  // namespace fa
