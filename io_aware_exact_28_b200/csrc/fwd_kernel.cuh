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
// PAGED = true reads K and V from a page pool (PagedKV in sm100.cuh) through two map
// pairs over [num_pages * Hkv, rows, d]: tmK/tmV with rows = page_size, and tmKt/tmVt
// with rows = the used rows of the sequence's last page, so that pool rows past Nk read
// as zero exactly as the rows past Nk of a contiguous map do. A key tile is one box of a
// page of >= BN tokens or BN / page_size boxes of smaller pages; a box wholly past Nk is
// aimed past the pool (zeros) and its table entry is never read.
//
// Lazy rescaling: the running maximum m used in the exponent is only raised when a new
// tile maximum exceeds it by more than 8 (log2 units). O and l are both accumulated
// against the same m, so the final O/l and LSE = (m + log2 l) ln 2 are exact in real
// arithmetic whatever m is; the bound keeps P <= 2^8.
#pragma once

#include <cuda.h>
#include <math_constants.h>

#include <type_traits>

#include "sm100.cuh"

namespace fa {

constexpr int kBM = 128;           // query rows per Q tile (one TMEM lane per row)
struct EmptyBase {};

// Keys per K/V tile at d = 64 (64: two CTAs per SM; 128: the d = 128 structure, one CTA
// per SM, measured slower on the mha2k workload).
#ifndef FA_D64_BN
#define FA_D64_BN 64
#endif
// 64-key tiles: exponential pairs, of the 16 in each 32-score chunk, evaluated on the FMA
// pipe (exp2_emu) instead of the MUFU unit (0, 1, 2 or 4). A 64-key tile's softmax needs
// twice the MUFU time of its two products; 128-key tiles (16-bit or E4M3) are faster with
// every exponential on the MUFU unit.
#ifndef FA_EXP2_EMU_D64
#define FA_EXP2_EMU_D64 2
#endif

// Per head-dimension configuration.
//  d = 128: 128-key tiles, one CTA per SM, TMEM S 2x128 + O 2x128 = 512 columns.
//  d = 64:  64-key tiles, two CTAs per SM (TMEM S 2x64 + O 2x64 = 256 columns each), so
//           four Q tiles are in flight per SM and one CTA's prologue/epilogue overlaps the
//           other's main loop: at d = 64 the per-tile softmax <-> MMA round trip, not any
//           one pipe, is the limit.
//  FP8 (d = 128 only): E4M3 Q, K, V; a row is 128 bytes, so the shared-memory tiles have
//           the d = 64 geometry (one 128-byte swizzle chunk) and the ring is 8 stages deep;
//           TMEM, threads and registers are those of d = 128.
template <int D, bool FP8 = false>
struct FwdCfg {
  static constexpr int ELEM = FP8 ? 1 : 2;            // bytes per Q/K/V element
  static constexpr int ROWB = D * ELEM;               // bytes per Q/K/V row
  static constexpr int BN = (D == 64) ? FA_D64_BN : 128;   // keys per K/V tile
  static constexpr int QT = 2;                         // 128-row Q tiles per CTA
  static constexpr bool NARROW = (BN == 64);          // 64-key tiles, two CTAs per SM
  static constexpr int CTAS = NARROW ? 2 : 1;         // resident CTAs per SM
  // 128-key tiles: 3 warpgroups (warps 10-11 idle) so the register re-split below can
  // apply; 64-key tiles: 10 warps, two CTAs per SM share the register file (96 each).
  static constexpr int THREADS = NARROW ? 320 : 384;
  static constexpr int WARP_PRODUCER = 4 * QT;        // TMA producer warp
  static constexpr int WARP_MMA = 4 * QT + 1;         // TMEM allocator and MMA issuer
  static constexpr bool REGSPLIT = !NARROW;            // warpgroup register re-split
  // Pairs i (0-15) of a 32-score chunk whose 2^x comes from exp2_emu.
  static constexpr int EMU_PAIRS = NARROW ? FA_EXP2_EMU_D64 : 0;
  static_assert(EMU_PAIRS == 0 || EMU_PAIRS == 1 || EMU_PAIRS == 2 || EMU_PAIRS == 4,
                "exp2 emulation: 0, 1, 2 or 4 pairs of 16");
  static constexpr uint32_t EMU_MASK = EMU_PAIRS == 1 ? 0x0008u
                                       : EMU_PAIRS == 2 ? 0x0808u
                                       : EMU_PAIRS == 4 ? 0x8888u : 0u;
  static constexpr int NCH = ROWB / 128;              // 128-byte swizzle chunks along d
  static constexpr int OCH = D / 64;                  // 64-column chunks of an O row
  static constexpr int Q_CHUNK = kBM * 128;           // 128 rows x 128 bytes
  static constexpr int KV_CHUNK = BN * 128;
  static constexpr int Q_TILE_BYTES = kBM * ROWB;     // one 128-row tile of Q
  static constexpr int KV_TILE_BYTES = BN * ROWB;
  static constexpr int NS = (ROWB == 128) ? 8 : 4;    // K/V ring stages
  // Keys per P.V instruction (32 bytes of K) and TMEM columns of P per 32 scores.
  static constexpr int KPI = 32 / ELEM;
  static constexpr int P_COLS32 = 8 * ELEM;
  // Lazy-rescale threshold (log2 units) and exponent offset: P = 2^(s*c - m + OFF) stays
  // in (0, 2^(TAU+OFF)]. FP8 keeps P in [2^-6, 2^8] (normal E4M3) for every score within
  // 10 of the running max, and the offset cancels in O / l.
  static constexpr float TAU = FP8 ? 4.f : 8.f;
  static constexpr float OFF = FP8 ? 4.f : 0.f;
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = QT * Q_TILE_BYTES;
  static constexpr int BAR_OFF = KV_OFF + NS * KV_TILE_BYTES;
  // q, full[NS], empty[NS], s[2], p[2], o[2], qempty, clc_full[2], clc_empty[2], drain, tail
  static constexpr int NBARS = 1 + 2 * NS + 3 * QT + 1 + 4 + 1 + 1;
  static constexpr int CLC_OFF = BAR_OFF + ((NBARS * 8 + 15) / 16) * 16;   // 2 x 16-byte responses
  static constexpr int MISC_OFF = CLC_OFF + 32;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;   // + slack for 1 KB alignment
  static constexpr uint32_t TMEM_COLS = NARROW ? 256 : 512;
  static constexpr uint32_t S_COL = 0;                // S_t at t * BN
  static constexpr uint32_t O_COL = QT * BN;          // O_t at O_COL + t * D
  // Registers per thread: the launch allocation (65536 / (threads * CTAS), rounded down
  // to 8) is re-split so that warpgroup 2 (producer, MMA, 2 idle warps) keeps REGS_OTHER
  // and the two softmax warpgroups get REGS_SOFTMAX; the split uses exactly the launch
  // allocation (checked on the host against the compiled register count).
  static constexpr uint32_t REGS_LAUNCH = NARROW ? 96 : 168;
  static constexpr uint32_t REGS_OTHER = 72;
  static constexpr uint32_t REGS_SOFTMAX = 216;
  static_assert(!REGSPLIT || 128 * REGS_OTHER + 256 * REGS_SOFTMAX <= THREADS * REGS_LAUNCH,
                "register split");
  static_assert(THREADS * REGS_LAUNCH * CTAS <= 65536, "register file");
  static_assert(O_COL + QT * D <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES * CTAS <= 227 * 1024, "shared memory budget");
};

struct FwdParams {
  void* o;              // [B*Hq, Nq, D], 16-bit
  float* lse;           // [B*Hq, Nq] or nullptr
  int BH;               // B * Hq
  int n_qb;             // query blocks of QT * kBM rows per (batch, head)
  int Hq, Hkv, group;   // group = Hq / Hkv
  int Nq, Nk;
  int causal_offset;    // Nk - Nq (bottom-right alignment)
  float scale_log2;     // scale * log2(e)
  uint64_t timeout_ns;
  int skip_q_load;      // test hook
  PagedKV pk;           // PAGED kernels only
  int last_page;        // PAGED: page index (t / page_size) of key Nk - 1
  float o_scale;        // FP8 kernels: multiplies O (the descale of V)
  const int* q_lens;    // VARLEN: [B] query rows of each sequence (nullptr: Nq for all)
  const int* kv_lens;   // VARLEN: [B] keys of each sequence (nullptr: Nk for all)
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

// Multiply 16 TMEM columns of packed 16-bit P pairs (32 values of this row) by alpha.
template <bool BF16>
__device__ __forceinline__ void rescale_p_cols(uint32_t taddr, float alpha) {
  uint32_t v[16];
  tmem_ld32x32b_x16(taddr, v);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float lo, hi;
    unpack_half2(v[i], lo, hi, BF16);
    v[i] = pack_half2(lo * alpha, hi * alpha, BF16);
  }
  tmem_st32x32b_x16(taddr, v);
  tmem_st_wait();
}

template <int D, bool BF16, bool CAUSAL, bool PAGED, bool FP8 = false, bool VARLEN = false,
          bool KVMAJOR = false>
__global__ void __launch_bounds__(FwdCfg<D, FP8>::THREADS, FwdCfg<D, FP8>::CTAS)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKt,
              const __grid_constant__ CUtensorMap tmVt, const FwdParams p) {
  using C = FwdCfg<D, FP8>;
  static_assert(!FP8 || (D == 128 && !PAGED && !VARLEN), "FP8: d = 128, contiguous K/V");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int kBN = C::BN;

  // Work unit u covers query block qb of (batch, head) bh; units are numbered heaviest
  // causal block first, which is also the order in which the hardware starts CTAs and
  // hands out not-yet-started CTAs to running ones.
  // n_t[t]: key tiles query tile t visits. A tile past the last query row visits none,
  // and under the causal mask a tile stops at the key tile of its last row's diagonal.
  // Lengths of the unit's sequence: query rows nq and keys nk (Nq and Nk, unless VARLEN
  // gives per-sequence lengths, clamped to [0, Nq] and [0, Nk]); off = nk - nq aligns the
  // causal mask to the end of the sequence. Only VARLEN units carry them; the others read
  // the kernel parameters, so that no role keeps three more registers live.
  const int n_kv_all = (p.Nk + kBN - 1) / kBN;   // key tiles of a sequence of Nk keys
  struct Lens {
    int nq, nk;
  };
  struct Unit : std::conditional_t<VARLEN, Lens, EmptyBase> {
    int bh, bh_kv, q0;
    int n_t[C::QT];
    int n_kv;           // key tiles the unit loads: max over its query tiles
  };
  auto u_nq = [&](const Unit& w) -> int {
    if constexpr (VARLEN) return w.nq; else return p.Nq;
  };
  auto u_nk = [&](const Unit& w) -> int {
    if constexpr (VARLEN) return w.nk; else return p.Nk;
  };
  auto u_off = [&](const Unit& w) -> int {
    if constexpr (VARLEN) return w.nk - w.nq; else return p.causal_offset;
  };
  auto decode_unit = [&](int u) {
    Unit w;
    // KVMAJOR (grouped-query calls whose K/V would not stay in L2): the units of one KV
    // head (every query block, heaviest first, of each query head that reads it) are
    // numbered together, so that the CTAs running at any time stream one or two KV heads
    // and each K/V tile is read from DRAM about once. Otherwise query block by query
    // block, heaviest first, all heads of a block together.
    int qb;
    if constexpr (KVMAJOR) {
      const int per_kv = p.n_qb * p.group;
      const int kv = u / per_kv;
      const int r = u - kv * per_kv;
      qb = p.n_qb - 1 - r / p.group;
      const int g = r - (r / p.group) * p.group;
      w.bh_kv = kv;
      w.bh = (kv / p.Hkv) * p.Hq + (kv - (kv / p.Hkv) * p.Hkv) * p.group + g;
    } else {
      qb = p.n_qb - 1 - u / p.BH;
      w.bh = u - (u / p.BH) * p.BH;
      w.bh_kv = (w.bh / p.Hq) * p.Hkv + (w.bh % p.Hq) / p.group;
    }
    w.q0 = qb * (C::QT * kBM);
    w.n_kv = 0;
    if constexpr (VARLEN) {
      const int b = w.bh / p.Hq;
      w.nq = p.q_lens ? min(max(__ldg(p.q_lens + b), 0), p.Nq) : p.Nq;
      w.nk = p.kv_lens ? min(max(__ldg(p.kv_lens + b), 0), p.Nk) : p.Nk;
    }
    const int n_kv_total = VARLEN ? (u_nk(w) + kBN - 1) / kBN : n_kv_all;
#pragma unroll
    for (int t = 0; t < C::QT; ++t) {
      const int row_first = w.q0 + t * kBM;
      int n = row_first < u_nq(w) ? n_kv_total : 0;
      if (CAUSAL && n > 0) {
        const int kmax = min(row_first + kBM - 1, u_nq(w) - 1) + u_off(w);
        n = kmax < 0 ? 0 : min(n_kv_total, kmax / kBN + 1);
      }
      w.n_t[t] = n;
      w.n_kv = max(w.n_kv, n);
    }
    return w;
  };

  const uint32_t bar0 = base + C::BAR_OFF;
  auto bar_q = [&]() { return bar0; };
  auto bar_full = [&](int i) { return bar0 + 8u * (1 + i); };
  auto bar_empty = [&](int i) { return bar0 + 8u * (1 + C::NS + i); };
  auto bar_s = [&](int t) { return bar0 + 8u * (1 + 2 * C::NS + t); };
  auto bar_p = [&](int t) { return bar0 + 8u * (1 + 2 * C::NS + C::QT + t); };
  auto bar_o = [&](int t) { return bar0 + 8u * (1 + 2 * C::NS + 2 * C::QT + t); };
  const uint32_t bar_qempty = bar0 + 8u * (1 + 2 * C::NS + 3 * C::QT);
  auto bar_clc_full = [&](int i) { return bar0 + 8u * (2 + 2 * C::NS + 3 * C::QT + i); };
  auto bar_clc_empty = [&](int i) { return bar0 + 8u * (4 + 2 * C::NS + 3 * C::QT + i); };
  const uint32_t bar_drain = bar0 + 8u * (6 + 2 * C::NS + 3 * C::QT);
  const uint32_t bar_tail = bar0 + 8u * (7 + 2 * C::NS + 3 * C::QT);   // VARLEN: ragged V tile
  auto clc_resp = [&](int i) { return base + C::CLC_OFF + 16u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sbase + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + C::MISC_OFF + 4);
  // Readers of each scheduling response: the MMA thread and the 8 softmax warps.
  constexpr int kClcReaders = 1 + 4 * C::QT;

  if (threadIdx.x == 0) {
    mbar_init(bar_q(), 1);
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(bar_full(i), 1);
      mbar_init(bar_empty(i), 1);
    }
    for (int t = 0; t < C::QT; ++t) {
      mbar_init(bar_s(t), 1);
      mbar_init(bar_p(t), kBM);
      mbar_init(bar_o(t), 1);
    }
    mbar_init(bar_qempty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_clc_full(i), 1);
      mbar_init(bar_clc_empty(i), kClcReaders);
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_tail, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == C::WARP_MMA) tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
  if (warp == C::WARP_PRODUCER && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    if (PAGED) {
      prefetch_tmap(&tmKt);
      prefetch_tmap(&tmVt);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, &g_fa_status, p.timeout_ns};

  // Each role's code sits inside the branch that set its register budget. Every role
  // walks the same unit sequence: its own blockIdx.x, then the CTAs the producer takes
  // over, published through clc_resp[k & 1] (k = units finished).
  if (warp >= 4 * C::QT) {
    if constexpr (C::REGSPLIT) setmaxnreg_dec<C::REGS_OTHER>();
    if (warp == C::WARP_PRODUCER) {
    // ------------------------------------------------------------------ TMA producer
    // Contiguous K/V of one length: lane 0 alone issues every copy (one box per 64 columns
    // of a tile).
    if constexpr (!PAGED && !VARLEN) {
    if (lane == 0) {
      int unit = blockIdx.x, k = 0, it = 0, q_loads = 0;
      bool ok = true, clc_pending = false;
      while (true) {
        const Unit w = decode_unit(unit);
        // A query tile with no visible key writes zeros and needs no Q.
        if (!p.skip_q_load && w.n_kv > 0) {
          // Q is reloaded once the previous unit's S products have all read it.
          if (q_loads > 0 && !mbar_wait(bar_qempty, (q_loads - 1) & 1, wc)) { ok = false; break; }
          int q_tiles = 0;
#pragma unroll
          for (int t = 0; t < C::QT; ++t) q_tiles += w.n_t[t] > 0 ? 1 : 0;
          mbar_arrive_expect_tx(bar_q(), q_tiles * C::Q_TILE_BYTES);
#pragma unroll
          for (int t = 0; t < C::QT; ++t) {
            if (w.n_t[t] == 0) continue;
            for (int ch = 0; ch < C::NCH; ++ch)
              tma_load_3d(base + C::Q_OFF + t * C::Q_TILE_BYTES + ch * C::Q_CHUNK, &tmQ, bar_q(),
                          ch * 64, w.q0 + t * kBM, w.bh);
          }
          ++q_loads;
        }
        for (int j = 0; j < w.n_kv && ok; ++j) {
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
                          bar_full(slot), ch * 64, j * kBN, w.bh_kv);
            ++it;
          }
        }
        if (!ok) break;
        // All loads of this unit are issued: take over the next CTA that has not started.
        const int sl = k & 1;
        if (k >= 2 && !mbar_wait(bar_clc_empty(sl), ((k >> 1) - 1) & 1, wc)) { ok = false; break; }
        mbar_arrive_expect_tx(bar_clc_full(sl), 16);
        clc_try_cancel(clc_resp(sl), bar_clc_full(sl));
        clc_pending = true;
        if (!mbar_wait(bar_clc_full(sl), (k >> 1) & 1, wc)) { ok = false; break; }
        clc_pending = false;
        uint32_t next;
        const bool more = clc_query(clc_resp(sl), next);
        ++k;
        if (!more) break;
        unit = static_cast<int>(next);
      }
      if (!ok || *abort_flag) {
        // Copies still in flight must land before the CTA exits.
        for (int i = max(0, it - C::NS); i < it; ++i)
          mbar_wait_drain(bar_full(i % C::NS), (i / C::NS) & 1, kDrainNs);
        if (q_loads > 0) mbar_wait_drain(bar_q(), (q_loads - 1) & 1, kDrainNs);
        if (clc_pending) mbar_wait_drain(bar_clc_full(k & 1), (k >> 1) & 1, kDrainNs);
      }
    }
    } else {
    // The whole warp walks the units. Lane 0 waits on the ring, arms the barriers, loads Q
    // and takes over CTAs; its decisions reach the other lanes through shuffles. Paged:
    // lane i reads the table entry of page i of a key tile and issues that page's boxes,
    // so a tile of small pages costs one table read and NCH boxes per lane. VARLEN: the V
    // tile that holds a sequence's last key lands on bar_tail first; the warp then zeroes
    // its rows past that key (whatever the cache holds there, P = 0 multiplies zeros) and
    // only then completes the ring slot.
    const bool leader = lane == 0;
    int unit = blockIdx.x, k = 0, it = 0, q_loads = 0, tail_uses = 0;
    bool ok = true, clc_pending = false, tail_pending = false;
    while (true) {
      const Unit w = decode_unit(unit);
      // A query tile with no visible key writes zeros and needs no Q.
      if (!p.skip_q_load && w.n_kv > 0) {
        if (leader) {
          // Q is reloaded once the previous unit's S products have all read it.
          if (q_loads > 0 && !mbar_wait(bar_qempty, (q_loads - 1) & 1, wc)) {
            ok = false;
          } else {
            int q_tiles = 0;
#pragma unroll
            for (int t = 0; t < C::QT; ++t) q_tiles += w.n_t[t] > 0 ? 1 : 0;
            mbar_arrive_expect_tx(bar_q(), q_tiles * C::Q_TILE_BYTES);
#pragma unroll
            for (int t = 0; t < C::QT; ++t) {
              if (w.n_t[t] == 0) continue;
              for (int ch = 0; ch < C::NCH; ++ch)
                tma_load_3d(base + C::Q_OFF + t * C::Q_TILE_BYTES + ch * C::Q_CHUNK, &tmQ, bar_q(),
                            ch * 64, w.q0 + t * kBM, w.bh);
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        ++q_loads;
      }
      for (int j = 0; j < w.n_kv && ok; ++j) {
        // Paged: box `lane` of key tile j holds keys [j*BN + lane*rows, +rows). The table
        // entry is read here and checked after the slot wait, so its latency hides there.
        int rows = kBN, y = 0, entry = 0, z = 0;
        bool have = false;
        if constexpr (PAGED) {
          const int ps = 1 << p.pk.page_shift;
          rows = min(kBN, ps);
          y = (j * kBN) & (ps - 1) & ~(kBN - 1);   // row of the tile in a large page
          const int b = w.bh_kv / p.Hkv;
          const int tok = j * kBN + lane * rows;
          have = lane * rows < kBN && tok < u_nk(w);
          if (have) entry = paged_entry(p.pk, b, tok);
        }
        for (int kv = 0; kv < 2; ++kv) {
          const int slot = it % C::NS;
          const int round = it / C::NS;
          const bool zero_tail = VARLEN && kv == 1 && (j + 1) * kBN > u_nk(w);
          const uint32_t land = zero_tail ? bar_tail : bar_full(slot);
          if (leader) {
            if (round > 0 && !mbar_wait(bar_empty(slot), (round - 1) & 1, wc))
              ok = false;
            else
              mbar_arrive_expect_tx(land, C::KV_TILE_BYTES);
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
          const uint32_t dst = base + C::KV_OFF + slot * C::KV_TILE_BYTES;
          if constexpr (PAGED) {
            if (lane * rows < kBN) {
              const int tok = j * kBN + lane * rows;
              if (kv == 0) {   // the page's head index, shared by the K and V boxes
                const int kvh = w.bh_kv - (w.bh_kv / p.Hkv) * p.Hkv;
                z = have ? paged_z(p.pk, entry, kvh) : paged_z_oob(p.pk);
              }
              const bool tail = !VARLEN && have && (tok >> p.pk.page_shift) == p.last_page;
              const CUtensorMap* tm = kv ? (tail ? &tmVt : &tmV) : (tail ? &tmKt : &tmK);
              for (int ch = 0; ch < C::NCH; ++ch)
                tma_load_3d(dst + ch * C::KV_CHUNK + lane * rows * 128, tm, land, ch * 64, y, z);
            }
          } else if (leader) {
            const CUtensorMap* tm = kv ? &tmV : &tmK;
            for (int ch = 0; ch < C::NCH; ++ch)
              tma_load_3d(dst + ch * C::KV_CHUNK, tm, land, ch * 64, j * kBN, w.bh_kv);
          }
          if (zero_tail) {
            // Rows [nk - j*BN, BN) of the landed V tile: 128 bytes per row and swizzle chunk
            // (the swizzle permutes 16-byte pieces within a row, so whole rows stay whole).
            tail_pending = true;
            if (leader && !mbar_wait(bar_tail, tail_uses & 1, wc)) ok = false;
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            tail_pending = false;
            ++tail_uses;
            const int r0 = u_nk(w) - j * kBN;
            const int n16 = (kBN - r0) * 8;                  // 16-byte pieces per chunk
            const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
            for (int ch = 0; ch < C::NCH; ++ch)
              for (int i = lane; i < n16; i += 32)
                *reinterpret_cast<uint4*>(sbase + C::KV_OFF + slot * C::KV_TILE_BYTES +
                                          ch * C::KV_CHUNK + r0 * 128 + i * 16) = zero;
            fence_proxy_async_smem();
            __syncwarp();
            if (leader) mbar_arrive(bar_full(slot));
          }
          ++it;
        }
      }
      if (!ok) break;
      // All loads of this unit are issued: take over the next CTA that has not started.
      const int sl = k & 1;
      int more = 0;
      uint32_t next = 0;
      if (leader) {
        if (k >= 2 && !mbar_wait(bar_clc_empty(sl), ((k >> 1) - 1) & 1, wc)) {
          ok = false;
        } else {
          mbar_arrive_expect_tx(bar_clc_full(sl), 16);
          clc_try_cancel(clc_resp(sl), bar_clc_full(sl));
          clc_pending = true;
          if (!mbar_wait(bar_clc_full(sl), (k >> 1) & 1, wc)) {
            ok = false;
          } else {
            clc_pending = false;
            more = clc_query(clc_resp(sl), next) ? 1 : 0;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      more = __shfl_sync(0xffffffffu, more, 0);
      next = __shfl_sync(0xffffffffu, next, 0);
      if (!ok) break;
      ++k;
      if (!more) break;
      unit = static_cast<int>(next);
    }
    if (leader && (!ok || *abort_flag)) {
      // Copies still in flight must land before the CTA exits (copies issued by any lane
      // complete on the same ring barriers, or on bar_tail).
      for (int i = max(0, it - C::NS); i < it; ++i)
        mbar_wait_drain(bar_full(i % C::NS), (i / C::NS) & 1, kDrainNs);
      if (tail_pending) mbar_wait_drain(bar_tail, tail_uses & 1, kDrainNs);
      if (q_loads > 0) mbar_wait_drain(bar_q(), (q_loads - 1) & 1, kDrainNs);
      if (clc_pending) mbar_wait_drain(bar_clc_full(k & 1), (k >> 1) & 1, kDrainNs);
    }
    }
    } else if (warp == C::WARP_MMA) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Format code: fp16 0 / bf16 1 under kind::f16; E4M3 is code 0 under kind::f8f6f4.
      constexpr uint32_t FMT = (!FP8 && BF16) ? 1u : 0u;
      constexpr uint32_t IDESC_S = idesc_f16(kBM, kBN, FMT, 0u, 0u);
      constexpr uint32_t IDESC_O = idesc_f16(kBM, D, FMT, 0u, 1u);
      // 32 bytes of K per instruction: d/16 (16-bit) or d/32 (E4M3) instructions per S.
      auto issue_s = [&](int t, int kslot) {
        const uint32_t qa = base + C::Q_OFF + t * C::Q_TILE_BYTES;
        const uint32_t ka = base + C::KV_OFF + kslot * C::KV_TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::ROWB / 32; ++kk) {
          const uint32_t koff = (kk & 3) * 32;
          const uint64_t da = sdesc_k_sw128(qa + (kk >> 2) * C::Q_CHUNK + koff);
          const uint64_t db = sdesc_k_sw128(ka + (kk >> 2) * C::KV_CHUNK + koff);
          if constexpr (FP8) mma_f8_ss(tmem + C::S_COL + t * kBN, da, db, IDESC_S, kk > 0 ? 1u : 0u);
          else mma_f16_ss(tmem + C::S_COL + t * kBN, da, db, IDESC_S, kk > 0 ? 1u : 0u);
        }
      };
      // P from TMEM (8 columns = KPI keys per instruction), V rows MN-major from SMEM.
      auto issue_pv = [&](int t, int vslot, bool acc0) {
        const uint32_t va = base + C::KV_OFF + vslot * C::KV_TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < kBN / C::KPI; ++kk) {
          const uint64_t db = sdesc_mn_sw128(va + kk * C::KPI * 128, C::KV_CHUNK);
          if constexpr (FP8)
            mma_f8_ts(tmem + C::O_COL + t * D, tmem + C::S_COL + t * kBN + kk * 8, db, IDESC_O,
                      (acc0 || kk > 0) ? 1u : 0u);
          else
            mma_f16_ts(tmem + C::O_COL + t * D, tmem + C::S_COL + t * kBN + kk * 8, db, IDESC_O,
                       (acc0 || kk > 0) ? 1u : 0u);
        }
      };
      int unit = blockIdx.x, k = 0, it = 0, q_uses = 0;
      int p_seen[C::QT];
#pragma unroll
      for (int t = 0; t < C::QT; ++t) p_seen[t] = 0;
      bool ok = true, issued = false;
      while (ok) {
        const Unit w = decode_unit(unit);
        if (w.n_kv > 0) {
          ok = mbar_wait(bar_q(), q_uses & 1, wc);
          ++q_uses;
          tc_fence_after();
          // Per key tile j and query tile t: the PV of tile j-1 (its last one completes
          // O_t: commit bar_o), then S_t(j) (commit bar_s). MMAs of one thread run in
          // order, so S_t(j) never overwrites P_t(j-1) before that PV has read it.
          for (int j = 0; j < w.n_kv && ok; ++j) {
            const int kit = it + 2 * j, kslot = kit % C::NS;
            const int vit = kit - 1, vslot = (vit + C::NS) % C::NS;   // V_{j-1}
            if (!mbar_wait(bar_full(kslot), (kit / C::NS) & 1, wc)) { ok = false; break; }
            if (j > 0 && !mbar_wait(bar_full(vslot), (vit / C::NS) & 1, wc)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int t = 0; t < C::QT; ++t) {
              if (j > 0 && j - 1 < w.n_t[t]) {
                if (!mbar_wait(bar_p(t), p_seen[t] & 1, wc)) { ok = false; break; }
                ++p_seen[t];
                tc_fence_after();
                issue_pv(t, vslot, j - 1 > 0);
                if (j == w.n_t[t]) mma_commit(bar_o(t));
              }
              if (j < w.n_t[t]) {
                issue_s(t, kslot);
                issued = true;
                mma_commit(bar_s(t));
              }
            }
            if (!ok) break;
            if (j == w.n_kv - 1) mma_commit(bar_qempty);    // every S of the unit issued
            if (j > 0) mma_commit(bar_empty(vslot));
            mma_commit(bar_empty(kslot));
          }
          if (ok) {
            const int vit = it + 2 * w.n_kv - 1, vslot = vit % C::NS;
            ok = mbar_wait(bar_full(vslot), (vit / C::NS) & 1, wc);
#pragma unroll
            for (int t = 0; t < C::QT; ++t) {
              if (!ok || w.n_t[t] != w.n_kv) continue;
              if (!mbar_wait(bar_p(t), p_seen[t] & 1, wc)) { ok = false; break; }
              ++p_seen[t];
              tc_fence_after();
              issue_pv(t, vslot, w.n_kv - 1 > 0);
              mma_commit(bar_o(t));
            }
            if (ok) mma_commit(bar_empty(vslot));
          }
          it += 2 * w.n_kv;
        }
        if (!ok) break;
        const int sl = k & 1;
        if (!mbar_wait(bar_clc_full(sl), (k >> 1) & 1, wc)) { ok = false; break; }
        uint32_t next;
        const bool more = clc_query(clc_resp(sl), next);
        mbar_arrive(bar_clc_empty(sl));
        ++k;
        if (!more) break;
        unit = static_cast<int>(next);
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
    const float c = p.scale_log2;
    int unit = blockIdx.x, k = 0, s_seen = 0, o_seen = 0;
    bool ok = true;
    while (true) {
      const Unit w = decode_unit(unit);
      int n_t = 0;   // this warp's tile, selected with static indices (no local memory)
#pragma unroll
      for (int tt = 0; tt < C::QT; ++tt)
        if (tt == t) n_t = w.n_t[tt];
      const int row = w.q0 + t * kBM + r;
      const int row_min = w.q0 + t * kBM;
      const int lim = CAUSAL ? min(row + u_off(w), u_nk(w) - 1) : u_nk(w) - 1;
      const int lim_min = CAUSAL ? min(row_min + u_off(w), u_nk(w) - 1) : u_nk(w) - 1;

      float m_used = -CUDART_INF_F;
      float l = 0.f;
      for (int j = 0; j < n_t; ++j) {
        // Wait results are made warp-uniform: the TMEM loads and stores below are
        // warp-collective, so a warp must never split on an aborted wait.
        if (!__all_sync(0xffffffffu, mbar_wait(bar_s(t), s_seen & 1, wc))) { ok = false; break; }
        ++s_seen;
        tc_fence_after();
        const int key0 = j * kBN;
        const bool masked_tile = key0 + kBN - 1 > lim_min;   // tile-uniform: diagonal or ragged
        // Scores of a 32-column chunk cc, with masked keys set to -inf.
        auto mask_chunk = [&](uint32_t (&v)[32], int cc) {
          if (masked_tile) {
#pragma unroll
            for (int kk = 0; kk < 32; ++kk)
              if (key0 + 32 * cc + kk > lim) v[kk] = __float_as_uint(-CUDART_INF_F);
          }
        };
        // Row maximum over 8 independent chains (short dependency chains).
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = -CUDART_INF_F;
        auto max_chunk = [&](const uint32_t (&v)[32]) {
#pragma unroll
          for (int kk = 0; kk < 32; kk += 2)
            mx8[(kk >> 1) & 7] = fmax3(mx8[(kk >> 1) & 7], __uint_as_float(v[kk]), __uint_as_float(v[kk + 1]));
        };
        // d = 128 keeps the whole 128-score row in registers; d = 64 (two CTAs per SM, 96
        // registers) reads its 64-score row from TMEM twice: once for the max, once for P.
        constexpr bool kResident = (kBN == 128);
        uint32_t sr[kResident ? kBN : 32];
        const uint64_t c2 = f2_pack(c, c);
        // P = 2^(s*c - mref) in 32-column chunks, each stored to TMEM as 16 packed columns
        // (P_t occupies S_t columns [0, BN/2); chunk cc only overwrites columns already
        // read); returns the row sum of the unrounded fp32 P. With track, the row maximum
        // of the scores is gathered in mx8 on the way.
        // P of one 32-column chunk v (scores of keys 32 cc ..) against mref, stored as 16
        // packed columns at tS + 16 cc; returns its row sum (unrounded fp32 P). With track,
        // the scores' maximum is gathered in mx8 on the way.
        // 2^x of pair i of a chunk: MUFU ex2, or exp2_emu for the pairs EMU_MASK names (i is
        // a compile-time index once the loops are unrolled).
        auto exp2_pair = [&](uint64_t x2, int i) -> uint64_t {
          float x0, x1;
          f2_unpack(x2, x0, x1);
          if ((C::EMU_MASK >> i) & 1u) return f2_pack(exp2_emu(x0), exp2_emu(x1));
          return f2_pack(ex2_approx(x0), ex2_approx(x1));
        };
        auto chunk_p = [&](const uint32_t* v, int cc, float mref, bool track) -> float {
          const float nm = FP8 ? C::OFF - mref : -mref;
          const uint64_t nm2 = f2_pack(nm, nm);
          uint64_t l2a = f2_pack(0.f, 0.f), l2b = l2a;
          if constexpr (FP8) {
            // 32 scores -> 8 columns of four E4M3 values, one store.
            uint32_t pk[8];
            float pp[2];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              if (track)
                mx8[i & 7] = fmax3(mx8[i & 7], __uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
              const uint64_t x2 =
                  f2_fma(f2_pack(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), c2, nm2);
              const uint64_t p2 = exp2_pair(x2, i);
              if (i & 1) l2b = f2_add(l2b, p2); else l2a = f2_add(l2a, p2);
              float p0, p1;
              f2_unpack(p2, p0, p1);
              if (i & 1) pk[i >> 1] = pack_e4m3x4(pp[0], pp[1], p0, p1);
              else { pp[0] = p0; pp[1] = p1; }
            }
            tmem_st32x32b_x8(tS + cc * C::P_COLS32, pk);
            float la, lb, lc, ld;
            f2_unpack(l2a, la, lb);
            f2_unpack(l2b, lc, ld);
            return (la + lb) + (lc + ld);
          }
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {               // 8 packed columns per store
            uint32_t pk[8];
#pragma unroll
            for (int ii = 0; ii < 8; ++ii) {
              const int i = 8 * hh + ii;
              if (track)
                mx8[i & 7] = fmax3(mx8[i & 7], __uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
              const uint64_t x2 =
                  f2_fma(f2_pack(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), c2, nm2);
              const uint64_t p2 = exp2_pair(x2, i);
              if (i & 1) l2b = f2_add(l2b, p2); else l2a = f2_add(l2a, p2);
              float p0, p1;
              f2_unpack(p2, p0, p1);
              pk[ii] = pack_half2(p0, p1, BF16);
            }
            tmem_st32x32b_x8(tS + cc * 16 + hh * 8, pk);
          }
          float la, lb, lc, ld;
          f2_unpack(l2a, la, lb);
          f2_unpack(l2b, lc, ld);
          return (la + lb) + (lc + ld);
        };
        // P of the whole row (all chunks; d = 64 loads each chunk from TMEM here).
        // d = 64: a 32-key chunk past every row limit of the warp (causal diagonal) has
        // P = 0, stored without loading its scores or evaluating its exponentials
        // (warp-uniform test). The resident d = 128 path keeps its straight-line chunk
        // loop: the branch cost it more than the skipped exponentials saved.
        auto dead_chunk = [&](int cc) -> bool {
          return masked_tile && __all_sync(0xffffffffu, key0 + 32 * cc > lim);
        };
        auto store_zero_p = [&](int cc) {
          const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
          for (int hh = 0; hh < C::P_COLS32 / 8; ++hh) tmem_st32x32b_x8(tS + cc * C::P_COLS32 + hh * 8, z);
        };
        auto p_pass = [&](float mref, bool track) -> float {
          float sum = 0.f;
#pragma unroll
          for (int cc = 0; cc < kBN / 32; ++cc) {
            if constexpr (!kResident) {
              tmem_ld32x32b_x32(tS + 32 * cc, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
              mask_chunk(*reinterpret_cast<uint32_t(*)[32]>(&sr[0]), cc);
            }
            sum += chunk_p(kResident ? &sr[32 * cc] : &sr[0], cc, mref, track);
          }
          return sum;
        };
        // Raise m only when the tile max exceeds it by more than 8 (scale > 0: -inf stays
        // -inf). Rows that already hold earlier tiles rescale O_t and l. The TMEM rescale
        // is warp-collective: the warp runs it if any row needs it, with factor 1 elsewhere.
        auto raise_max = [&]() -> bool {
          const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                                 fmaxf(mx8[6], mx8[7])) * c;
          const bool grow = mx > m_used + C::TAU;
          const bool rescale = grow && m_used != -CUDART_INF_F;
          if (__any_sync(0xffffffffu, rescale)) {
            const float alpha = rescale ? ex2_approx(m_used - mx) : 1.0f;
            l *= alpha;
            rescale_o_row<D>(tO, alpha);
          }
          if (grow) m_used = mx;
          return __any_sync(0xffffffffu, grow);
        };
        if constexpr (kResident) {
          tmem_ld32x32b_x128(tS, sr);
#pragma unroll
          for (int cc = 0; cc < kBN / 32; ++cc) mask_chunk(*reinterpret_cast<uint32_t(*)[32]>(&sr[32 * cc]), cc);
          if (__all_sync(0xffffffffu, m_used != -CUDART_INF_F)) {
            // Every row already has a running max: compute P against it while gathering the
            // tile max; only if some row's max grew past the lazy threshold (rare after the
            // first tiles) is P recomputed, from the scores still in registers.
            float lsum = p_pass(m_used, true);
            if (raise_max()) lsum = p_pass(m_used, false);
            l += lsum;
          } else {
#pragma unroll
            for (int cc = 0; cc < kBN / 32; ++cc) max_chunk(*reinterpret_cast<uint32_t(*)[32]>(&sr[32 * cc]));
            raise_max();
            l += p_pass((m_used == -CUDART_INF_F) ? 0.f : m_used, false);
          }
        } else {
          // d = 64: one TMEM load per 32-column chunk. The chunk's max comes from registers;
          // a row whose max grows past the lazy threshold (every row on its first tile,
          // rarely later) raises m, and rows that already hold P (earlier tiles in O and l,
          // earlier chunks in TMEM) rescale them; then P of the chunk is computed and stored.
          uint32_t (&v)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
          float lsum = 0.f;
#pragma unroll
          for (int cc = 0; cc < kBN / 32; ++cc) {
            if (dead_chunk(cc)) {
              store_zero_p(cc);
              continue;
            }
            tmem_ld32x32b_x32(tS + 32 * cc, v);
            mask_chunk(v, cc);
#pragma unroll
            for (int i = 0; i < 8; ++i) mx8[i] = -CUDART_INF_F;
            max_chunk(v);
            const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                                   fmaxf(mx8[6], mx8[7])) * c;
            const bool grow = mx > m_used + C::TAU;
            const bool rescale = grow && m_used != -CUDART_INF_F;
            if (__any_sync(0xffffffffu, rescale)) {
              const float alpha = rescale ? ex2_approx(m_used - mx) : 1.0f;
              l *= alpha;
              lsum *= alpha;
              rescale_o_row<D>(tO, alpha);
              if (cc > 0) {
                tmem_st_wait();                            // stored P chunks, read back below
#pragma unroll
                for (int c0 = 0; c0 < cc; ++c0) rescale_p_cols<BF16>(tS + 16 * c0, alpha);
              }
              // Reload the chunk (its columns are untouched: P goes below 16 cc) instead of
              // keeping 32 scores live across the rescale.
              tmem_ld32x32b_x32(tS + 32 * cc, v);
              mask_chunk(v, cc);
            }
            if (grow) m_used = mx;
            lsum += chunk_p(v, cc, (m_used == -CUDART_INF_F) ? 0.f : m_used, false);
          }
          l += lsum;
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar_p(t));
      }
      if (ok && n_t > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_o(t), o_seen & 1, wc));   // last PV done
        ++o_seen;
        tc_fence_after();
      }
      if (!ok) break;
      // Epilogue: O / l straight from registers to global memory (one 2*D-byte row per
      // thread), then LSE = (m + log2 l) ln 2. A tile that saw no key writes zeros / -inf.
      // Every lane loads from TMEM (warp-collective); rows past Nq store nothing.
      {
        const bool row_ok = row < u_nq(w);
        uint16_t* orow = static_cast<uint16_t*>(p.o) +
                         (static_cast<size_t>(w.bh) * p.Nq + (row_ok ? row : 0)) * D;
        float inv_l = (l > 0.f) ? 1.f / l : 0.f;
        if constexpr (FP8) inv_l *= p.o_scale;
#pragma unroll
        for (int ch = 0; ch < C::OCH; ++ch) {
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
            uint4 v4;
            v4.x = pack_half2(__uint_as_float(o[8 * u + 0]) * inv_l, __uint_as_float(o[8 * u + 1]) * inv_l, BF16);
            v4.y = pack_half2(__uint_as_float(o[8 * u + 2]) * inv_l, __uint_as_float(o[8 * u + 3]) * inv_l, BF16);
            v4.z = pack_half2(__uint_as_float(o[8 * u + 4]) * inv_l, __uint_as_float(o[8 * u + 5]) * inv_l, BF16);
            v4.w = pack_half2(__uint_as_float(o[8 * u + 6]) * inv_l, __uint_as_float(o[8 * u + 7]) * inv_l, BF16);
            if (row_ok) *reinterpret_cast<uint4*>(orow + ch * 64 + u * 8) = v4;
          }
        }
        if (row_ok && p.lse != nullptr) {
          p.lse[static_cast<size_t>(w.bh) * p.Nq + row] =
              (l > 0.f) ? (m_used - C::OFF + __log2f(l)) * 0.69314718055994530942f : -CUDART_INF_F;
        }
      }
      // The next unit: every lane reads the response, then one arrival per warp.
      const int sl = k & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_clc_full(sl), (k >> 1) & 1, wc))) { ok = false; break; }
      uint32_t next;
      const bool more = clc_query(clc_resp(sl), next);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_clc_empty(sl));
      ++k;
      if (!more) break;
      unit = static_cast<int>(next);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
