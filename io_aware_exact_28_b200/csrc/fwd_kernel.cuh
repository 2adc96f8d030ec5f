// fwd_kernel.cuh — exact attention forward (prefill) for sm_100a.
//
// One CTA owns 256 query rows of one (batch, query head): two 128-row Q tiles that
// take turns on the tensor core. Per K/V tile j (BN keys: 128 at d = 128, 64 at d = 64)
// and Q tile t:
//     S_t = Q_t K_j^T                    tcgen05.mma, fp32 accumulator in TMEM
//     softmax warps: mask, row max, lazy rescale of O_t, P_t = exp2(S*c - m) -> TMEM
//     O_t += P_t V_j                     tcgen05.mma with A read from TMEM
// so the 128x128 score tile lives only in tensor memory and registers and never reaches
// device memory. This is the tiling + online-softmax scheme of page "Kotaemon
// FlashAttention" (algorithm bullets: Q split into row blocks, K_j/V_j blocks streamed
// through on-chip memory, running max and normaliser, result identical to the untiled
// formula) and page "Flash Attention ... IO-aware exact" (fr), tiling pseudo-code (Q_i
// read once, K_j/V_j per block, O_i and L written once at the end).
//
// Warp roles (FwdCfg::THREADS: 384 at d = 128, 320 at d = 64):
//   warps 0-3  softmax + epilogue for Q tile 0 (thread r owns row r = TMEM lane r)
//   warps 4-7  softmax + epilogue for Q tile 1
//   warp  8    TMA producer: Q tiles once, then K_j, V_j through an NS-stage ring
//   warp  9    TMEM allocator and single-thread tcgen05.mma issuer
//   warps 10-11 (d = 128 only) idle: they complete warpgroup 2 for the register re-split
//
// Tensor memory (FwdCfg::TMEM_COLS): S_t at columns [t*BN, (t+1)*BN) (fp32); P_t
// overwrites the first BN/2 of those columns as packed 16-bit pairs; O_t at
// [2*BN + t*D, 2*BN + (t+1)*D).
//
// Lazy rescaling: the running maximum m used in the exponent is only raised when a new
// tile maximum exceeds it by more than 8 (log2 units). O and l are both accumulated
// against the same m, so the final O/l and LSE = (m + log2 l) ln 2 are exact in real
// arithmetic whatever m is; the bound keeps P <= 2^8.
#pragma once

#include <cuda.h>
#include <math_constants.h>

#include "sm100.cuh"

namespace fa {

constexpr int kBM = 128;           // query rows per Q tile (one TMEM lane per row)
constexpr int kQTiles = 2;         // Q tiles per CTA
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;

// Polynomial-exp2 pair masks (see FwdCfg::kEmuPairs); off by default: measured slower on
// B200 at both head dimensions, because the softmax is latency-bound, not MUFU-bound.
#ifndef FA_EMU_PAIRS_D64
#define FA_EMU_PAIRS_D64 0u
#endif
#ifndef FA_EMU_PAIRS_D128
#define FA_EMU_PAIRS_D128 0u
#endif
#ifndef FA_REGSPLIT
#define FA_REGSPLIT 1
#endif

// Per head-dimension configuration.
//  d = 128: 128-key tiles, one CTA per SM, TMEM S 2x128 + O 2x128 = 512 columns.
//  d = 64:  64-key tiles, two CTAs per SM (TMEM S 2x64 + O 2x64 = 256 columns each), so
//           four Q tiles are in flight per SM and one CTA's prologue/epilogue overlaps the
//           other's main loop: at d = 64 the per-tile softmax <-> MMA round trip, not any
//           one pipe, is the limit.
template <int D>
struct FwdCfg {
  static constexpr int BN = (D == 64) ? 64 : 128;     // keys per K/V tile
  static constexpr int CTAS = (D == 64) ? 2 : 1;      // resident CTAs per SM
  // d = 128: 3 warpgroups (warps 10-11 idle) so the register re-split below can apply;
  // d = 64: 10 warps, two CTAs per SM share the register file (96 registers per thread).
  static constexpr int THREADS = (D == 64) ? 320 : 384;
  static constexpr bool REGSPLIT = (D == 128) && FA_REGSPLIT;
  static constexpr int NCH = D / 64;                  // 128-byte swizzle chunks along d
  static constexpr int Q_CHUNK = kBM * 128;           // 128 rows x 128 bytes
  static constexpr int KV_CHUNK = BN * 128;
  static constexpr int Q_TILE_BYTES = kBM * D * 2;    // one 128-row tile of Q or O
  static constexpr int KV_TILE_BYTES = BN * D * 2;
  static constexpr int NS = (D == 64) ? 8 : 4;        // K/V ring stages
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = kQTiles * Q_TILE_BYTES;
  static constexpr int BAR_OFF = KV_OFF + NS * KV_TILE_BYTES;
  static constexpr int NBARS = 1 + 2 * NS + 2 * kQTiles + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;   // + slack for 1 KB alignment
  static constexpr uint32_t TMEM_COLS = (D == 64) ? 256 : 512;
  static constexpr uint32_t S_COL = 0;                // S_t at t * BN
  static constexpr uint32_t O_COL = kQTiles * BN;     // O_t at O_COL + t * D
  // Registers per thread: the launch allocation (65536 / (threads * CTAS), rounded down
  // to 8) is re-split so that warpgroup 2 (producer, MMA, 2 idle warps) keeps REGS_OTHER
  // and the two softmax warpgroups get REGS_SOFTMAX; the split uses exactly the launch
  // allocation (checked on the host against the compiled register count).
  static constexpr uint32_t REGS_LAUNCH = (D == 64) ? 96 : 168;
  static constexpr uint32_t REGS_OTHER = 72;
  static constexpr uint32_t REGS_SOFTMAX = 216;
  static_assert(!REGSPLIT || 128 * REGS_OTHER + 256 * REGS_SOFTMAX <= THREADS * REGS_LAUNCH,
                "register split");
  static_assert(THREADS * REGS_LAUNCH * CTAS <= 65536, "register file");
  // Which of every 8 consecutive P column pairs use the polynomial exp2 (bit i = pair i).
  static constexpr uint32_t kEmuPairs = (D == 64) ? FA_EMU_PAIRS_D64 : FA_EMU_PAIRS_D128;
  static_assert(O_COL + kQTiles * D <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES * CTAS <= 227 * 1024, "shared memory budget");
};

struct FwdParams {
  float* lse;           // [B*Hq, Nq] or nullptr
  int Hq, Hkv, group;   // group = Hq / Hkv
  int Nq, Nk;
  int causal_offset;    // Nk - Nq (bottom-right alignment)
  float scale_log2;     // scale * log2(e)
  uint64_t timeout_ns;
  int skip_q_load;      // test hook
};

template <int D>
__device__ __forceinline__ void rescale_o_row(uint32_t tO, float alpha) {
#pragma unroll
  for (int c = 0; c < D; c += 32) {
    uint32_t v[32];
    tmem_ld32x32b_x32(tO + c, v);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
    tmem_st32x32b_x32(tO + c, v);
  }
  tmem_st_wait();
}

template <int D, bool BF16, bool CAUSAL>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, FwdCfg<D>::CTAS)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
              const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x;                        // b * Hq + h
  const int b = bh / p.Hq;
  const int h = bh - b * p.Hq;
  const int bh_kv = b * p.Hkv + h / p.group;
  const int qb = gridDim.y - 1 - blockIdx.y;        // heaviest (causal) blocks launch first
  const int q0 = qb * (kQTiles * kBM);

  constexpr int kBN = C::BN;
  const int n_kv_total = (p.Nk + kBN - 1) / kBN;
  // Key tiles each query tile visits: a tile past the last query row visits none, and
  // under the causal mask a tile stops at the key tile holding its last row's diagonal.
  int n_kv_t[kQTiles];
#pragma unroll
  for (int t = 0; t < kQTiles; ++t) {
    const int row_first = q0 + t * kBM;
    int n = row_first < p.Nq ? n_kv_total : 0;
    if (CAUSAL && n > 0) {
      const int kmax = min(row_first + kBM - 1, p.Nq - 1) + p.causal_offset;
      n = kmax < 0 ? 0 : min(n_kv_total, kmax / kBN + 1);
    }
    n_kv_t[t] = n;
  }
  int n_kv = 0;                                     // key tiles the CTA loads
#pragma unroll
  for (int t = 0; t < kQTiles; ++t) n_kv = max(n_kv, n_kv_t[t]);

  const uint32_t bar0 = base + C::BAR_OFF;
  auto bar_q = [&]() { return bar0; };
  auto bar_full = [&](int i) { return bar0 + 8u * (1 + i); };
  auto bar_empty = [&](int i) { return bar0 + 8u * (1 + C::NS + i); };
  auto bar_s = [&](int t) { return bar0 + 8u * (1 + 2 * C::NS + t); };
  auto bar_p = [&](int t) { return bar0 + 8u * (1 + 2 * C::NS + kQTiles + t); };
  const uint32_t bar_drain = bar0 + 8u * (1 + 2 * C::NS + 2 * kQTiles);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + C::MISC_OFF + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar_q(), 1);
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(bar_full(i), 1);
      mbar_init(bar_empty(i), 1);
    }
    for (int t = 0; t < kQTiles; ++t) {
      mbar_init(bar_s(t), 1);
      mbar_init(bar_p(t), kBM);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kWarpMma) tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
  if (warp == kWarpProducer && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, &g_fa_status, p.timeout_ns};

  // Each role's code sits inside the branch that set its register budget.
  if (warp >= 2 * 4) {
    if constexpr (C::REGSPLIT) setmaxnreg_dec<C::REGS_OTHER>();
    if (warp == kWarpProducer) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      bool q_issued = false;
      // A query tile with no visible key tile writes zeros from its softmax warps straight
      // into its Q buffer, so that buffer must not be loaded.
      if (!p.skip_q_load && n_kv > 0) {
        int q_tiles = 0;
#pragma unroll
        for (int t = 0; t < kQTiles; ++t) q_tiles += n_kv_t[t] > 0 ? 1 : 0;
        mbar_arrive_expect_tx(bar_q(), q_tiles * C::Q_TILE_BYTES);
#pragma unroll
        for (int t = 0; t < kQTiles; ++t) {
          if (n_kv_t[t] == 0) continue;
          for (int ch = 0; ch < C::NCH; ++ch)
            tma_load_3d(base + C::Q_OFF + t * C::Q_TILE_BYTES + ch * C::Q_CHUNK, &tmQ, bar_q(),
                        ch * 64, q0 + t * kBM, bh);
        }
        q_issued = true;
      }
      int it = 0;
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        for (int kv = 0; kv < 2; ++kv) {
          const int slot = it % C::NS;
          const int round = it / C::NS;
          if (round > 0 && !mbar_wait(bar_empty(slot), (round - 1) & 1, wc)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar_full(slot), C::KV_TILE_BYTES);
          const CUtensorMap* tm = kv ? &tmV : &tmK;
          for (int ch = 0; ch < C::NCH; ++ch)
            tma_load_3d(base + C::KV_OFF + slot * C::KV_TILE_BYTES + ch * C::KV_CHUNK, tm,
                        bar_full(slot), ch * 64, j * kBN, bh_kv);
          ++it;
        }
      }
      if (!ok || *abort_flag) {
        // Loads still in flight must land before the CTA exits.
        for (int k = max(0, it - C::NS); k < it; ++k)
          mbar_wait_drain(bar_full(k % C::NS), (k / C::NS) & 1, kDrainNs);
        if (q_issued) mbar_wait_drain(bar_q(), 0, kDrainNs);
      }
    }
    } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t IDESC_S = idesc_f16(kBM, kBN, BF16 ? 1u : 0u, 0u, 0u);
      constexpr uint32_t IDESC_O = idesc_f16(kBM, D, BF16 ? 1u : 0u, 0u, 1u);
      auto issue_s = [&](int t, int kslot) {
        const uint32_t qa = base + C::Q_OFF + t * C::Q_TILE_BYTES;
        const uint32_t ka = base + C::KV_OFF + kslot * C::KV_TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;
          mma_f16_ss(tmem + C::S_COL + t * kBN, sdesc_k_sw128(qa + (kk >> 2) * C::Q_CHUNK + koff),
                     sdesc_k_sw128(ka + (kk >> 2) * C::KV_CHUNK + koff),
                     IDESC_S, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, int vslot, bool acc0) {
        const uint32_t va = base + C::KV_OFF + vslot * C::KV_TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          mma_f16_ts(tmem + C::O_COL + t * D, tmem + C::S_COL + t * kBN + kk * 8,
                     sdesc_mn_sw128(va + kk * 2048, C::KV_CHUNK), IDESC_O,
                     (acc0 || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(bar_q(), 0, wc);
      bool issued = false;
      tc_fence_after();
      // Commits on bar_s(t): one per S_t(j), j < n_kv_t[t], then one after the last PV_t
      // (O_t complete). A tile that stops early gets its last PV in the next iteration.
      for (int j = 0; j < n_kv && ok; ++j) {
        const int kit = 2 * j, kslot = kit % C::NS;
        const int vit = 2 * j - 1, vslot = (vit + C::NS) % C::NS;   // V_{j-1}
        if (!mbar_wait(bar_full(kslot), (kit / C::NS) & 1, wc)) { ok = false; break; }
        if (j > 0 && !mbar_wait(bar_full(vslot), (vit / C::NS) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        for (int t = 0; t < kQTiles; ++t) {
          if (j > 0 && j - 1 < n_kv_t[t]) {
            if (!mbar_wait(bar_p(t), (j - 1) & 1, wc)) { ok = false; break; }
            tc_fence_after();
            issue_pv(t, vslot, j - 1 > 0);
            if (j == n_kv_t[t]) mma_commit(bar_s(t));   // final phase: O_t complete
          }
          if (j < n_kv_t[t]) {
            issue_s(t, kslot);
            issued = true;
            mma_commit(bar_s(t));
          }
        }
        if (!ok) break;
        if (j > 0) mma_commit(bar_empty(vslot));
        mma_commit(bar_empty(kslot));
      }
      if (ok) {
        const int vit = 2 * n_kv - 1, vslot = vit % C::NS;
        ok = mbar_wait(bar_full(vslot), (vit / C::NS) & 1, wc);
        for (int t = 0; t < kQTiles && ok; ++t) {
          if (n_kv_t[t] != n_kv) continue;
          if (!mbar_wait(bar_p(t), (n_kv - 1) & 1, wc)) { ok = false; break; }
          tc_fence_after();
          issue_pv(t, vslot, n_kv - 1 > 0);
          mma_commit(bar_s(t));   // final phase: O_t complete
        }
        if (ok) mma_commit(bar_empty(vslot));
      }
      if (issued) {
        // Every MMA must have finished before TMEM is released.
        mma_commit(bar_drain);
        mbar_wait_drain(bar_drain, 0, kDrainNs);
      }
    }
    }   // warps 10-11: idle, straight to the final barrier
  } else {
    if constexpr (C::REGSPLIT) setmaxnreg_inc<C::REGS_SOFTMAX>();
    // ------------------------------------------------------------------ softmax + epilogue
    const int t = warp >> 2;
    const int r = threadIdx.x & (kBM - 1);
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::S_COL + t * kBN;
    const uint32_t tO = tmem + lane_base + C::O_COL + t * D;
    const int row = q0 + t * kBM + r;
    const int row_min = q0 + t * kBM;
    const int lim = CAUSAL ? min(row + p.causal_offset, p.Nk - 1) : p.Nk - 1;
    const int lim_min = CAUSAL ? min(row_min + p.causal_offset, p.Nk - 1) : p.Nk - 1;
    const float c = p.scale_log2;

    const int n_t = t == 0 ? n_kv_t[0] : n_kv_t[kQTiles - 1];
    float m_used = -CUDART_INF_F;
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_t; ++j) {
      if (!mbar_wait(bar_s(t), j & 1, wc)) { ok = false; break; }
      tc_fence_after();
      const int key0 = j * kBN;
      const bool masked_tile = key0 + kBN - 1 > lim_min;   // tile-uniform: diagonal or ragged
      // Scores of a 32-column chunk cc, with masked keys set to -inf.
      auto mask_chunk = [&](uint32_t (&v)[32], int cc) {
        if (masked_tile) {
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (key0 + 32 * cc + k > lim) v[k] = __float_as_uint(-CUDART_INF_F);
        }
      };
      // Row maximum over 8 independent chains (short dependency chains).
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = -CUDART_INF_F;
      auto max_chunk = [&](const uint32_t (&v)[32]) {
#pragma unroll
        for (int k = 0; k < 32; ++k) mx8[k & 7] = fmaxf(mx8[k & 7], __uint_as_float(v[k]));
      };
      // d = 128 keeps the whole 128-score row in registers; d = 64 (two CTAs per SM, 96
      // registers) reads its 64-score row from TMEM twice: once for the max, once for P.
      constexpr bool kResident = (kBN == 128);
      uint32_t sr[kResident ? kBN : 32];
      if constexpr (kResident) {
        tmem_ld32x32b_x128(tS, sr);
#pragma unroll
        for (int cc = 0; cc < kBN / 32; ++cc) {
          uint32_t (&v)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * cc]);
          mask_chunk(v, cc);
          max_chunk(v);
        }
      } else {
#pragma unroll
        for (int cc = 0; cc < kBN / 32; ++cc) {
          tmem_ld32x32b_x32(tS + 32 * cc, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
          mask_chunk(*reinterpret_cast<uint32_t(*)[32]>(&sr[0]), cc);
          max_chunk(*reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        }
      }
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * c;
      if (mx > m_used + 8.0f) {                      // scale > 0: -inf stays -inf
        if (m_used != -CUDART_INF_F) {               // O_t and l hold earlier tiles
          const float alpha = ex2_approx(m_used - mx);
          l *= alpha;
          rescale_o_row<D>(tO, alpha);
        }
        m_used = mx;
      }
      const float mref = (m_used == -CUDART_INF_F) ? 0.f : m_used;
      // P = 2^(s*c - m) in 32-column chunks, each stored to TMEM as 16 packed columns
      // (P_t occupies S_t columns [0, BN/2); chunk cc only overwrites columns already read).
      // In tiles without masked scores, the pairs selected by kEmuPairs are evaluated
      // with the FMA-pipe polynomial instead of MUFU.EX2. The argument s*c - m and the
      // row sum use packed f32x2 arithmetic.
      const uint64_t c2 = f2_pack(c, c);
      const uint64_t nm2 = f2_pack(-mref, -mref);
      uint64_t l2a = f2_pack(0.f, 0.f), l2b = l2a;
#pragma unroll
      for (int cc = 0; cc < kBN / 32; ++cc) {
        if constexpr (!kResident) {
          tmem_ld32x32b_x32(tS + 32 * cc, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
          mask_chunk(*reinterpret_cast<uint32_t(*)[32]>(&sr[0]), cc);
        }
        const uint32_t* v = kResident ? &sr[32 * cc] : &sr[0];
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint64_t x2 =
              f2_fma(f2_pack(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), c2, nm2);
          uint64_t p2;
          if (!masked_tile && ((FwdCfg<D>::kEmuPairs >> (i & 7)) & 1u)) {
            p2 = exp2_poly_f2(x2);
          } else {
            float x0, x1;
            f2_unpack(x2, x0, x1);
            p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
          }
          if (i & 1) l2b = f2_add(l2b, p2); else l2a = f2_add(l2a, p2);
          float p0, p1;
          f2_unpack(p2, p0, p1);
          pk[i] = pack_half2(p0, p1, BF16);
        }
        tmem_st32x32b_x16(tS + cc * 16, pk);
      }
      {
        float la, lb, lc, ld;
        f2_unpack(l2a, la, lb);
        f2_unpack(l2b, lc, ld);
        l += (la + lb) + (lc + ld);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_p(t));
    }
    if (ok && n_t > 0) {
      ok = mbar_wait(bar_s(t), n_t & 1, wc);        // final PV of this tile done
      tc_fence_after();
    }
    uint8_t* otile = sbase + C::Q_OFF + t * C::Q_TILE_BYTES;   // Q_t no longer read
    if (ok) {
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
      for (int ch = 0; ch < C::NCH; ++ch) {
        uint32_t o[64];
        if (n_t > 0) {
          uint32_t (&o_lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&o[0]);
          uint32_t (&o_hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&o[32]);
          tmem_ld32x32b_x32(tO + ch * 64, o_lo);
          tmem_ld32x32b_x32(tO + ch * 64 + 32, o_hi);
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i) o[i] = 0u;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint4 w;
          w.x = pack_half2(__uint_as_float(o[8 * u + 0]) * inv_l, __uint_as_float(o[8 * u + 1]) * inv_l, BF16);
          w.y = pack_half2(__uint_as_float(o[8 * u + 2]) * inv_l, __uint_as_float(o[8 * u + 3]) * inv_l, BF16);
          w.z = pack_half2(__uint_as_float(o[8 * u + 4]) * inv_l, __uint_as_float(o[8 * u + 5]) * inv_l, BF16);
          w.w = pack_half2(__uint_as_float(o[8 * u + 6]) * inv_l, __uint_as_float(o[8 * u + 7]) * inv_l, BF16);
          // 128-byte swizzle: 16-byte unit u of row r sits at unit u ^ (r mod 8)
          *reinterpret_cast<uint4*>(otile + ch * C::Q_CHUNK + r * 128 + ((u ^ (r & 7)) << 4)) = w;
        }
      }
      if (p.lse != nullptr && row < p.Nq) {
        p.lse[static_cast<size_t>(bh) * p.Nq + row] =
            (l > 0.f) ? (m_used + __log2f(l)) * 0.69314718055994530942f : -CUDART_INF_F;
      }
      fence_proxy_async_smem();
    }
    named_barrier_sync(1 + t, kBM);
    if (r == 0 && ok && !*abort_flag && row_min < p.Nq) {
      for (int ch = 0; ch < C::NCH; ++ch)
        tma_store_3d(&tmO, smem_u32(otile + ch * C::Q_CHUNK), ch * 64, q0 + t * kBM, bh);
      tma_store_commit_and_wait_read();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
