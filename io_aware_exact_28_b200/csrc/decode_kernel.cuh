// decode_kernel.cuh — single-token attention over a grouped-query KV cache, split-KV.
//
// Decode reads every valid K and V row of the cache once per step, so it is bound by
// device-memory bandwidth (page "Empreinte mémoire et calcul des couches Transformer":
// KV-cache size per token and the memory-bound character of cache access). The split
// kernel therefore
//   * streams each split's K and V rows into a shared-memory ring with bulk TMA copies
//     (the rows of one split are contiguous, so one copy per tensor per stage), keeping
//     many bytes in flight without spending registers on them;
//   * reads each K/V row once for all G = Hq/Hkv query heads that share it;
//   * computes in fp32, two lanes of math per instruction (f32x2 FMA).
//
// Split kernel: grid (split, kv head x head tile, sequence), 128 threads (4 warps). A
// split covers up to `split_tokens` consecutive cache rows in stages of 32 tokens. Each
// token row is read from shared memory by LPT lanes (DPL = D/LPT elements per lane), the
// LPT partial dot products are summed with xor-shuffles, and each warp runs its own online
// softmax over its tokens (running max with the lazy-rescale rule of the prefill kernel).
// The four warps merge through shared memory and the CTA writes, per query head, a
// normalised partial O row and its log2-domain logsumexp.
//
// PAGED = true reads the rows from a page pool (PagedKV in sm100.cuh). Pages hold a power
// of two >= 16 tokens and stages start at multiples of 32, so a stage is one copy per
// tensor from one page, or two from two 16-token pages. A table entry outside the pool is
// recorded in the status word and its rows are not copied.
//
// Combine kernel: grid (sequence x query head), D threads, launched as a programmatic
// dependent of the split kernel. It merges the valid splits with weights 2^(lse_s - max)
// (the online-softmax rescaling identity, page "Kotaemon FlashAttention", running max and
// normaliser bullet) and writes O (16-bit) and the natural-log LSE.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include "sm100.cuh"

namespace fa {

constexpr int kDecThreads = 128;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecStageTok = 32;     // tokens per ring stage
constexpr int kDecStages = 4;        // ring depth

struct DecodeParams {
  const uint16_t* q;      // [B, Hq, D]
  const uint16_t* kc;     // [B, Hkv, max_len, D]
  const uint16_t* vc;
  const int* kv_lens;     // [B]
  float* ws_o;            // [B, Hq, n_split, D]
  float* ws_lse;          // [B, Hq, n_split]  (log2 domain)
  int Hq, Hkv, G;         // G = Hq / Hkv
  int max_len, split_tokens, n_split;
  float scale_log2;
  uint64_t timeout_ns;
  int skip_kv_load;       // test hook: the ring stages are armed but never filled
  PagedKV pk;             // PAGED kernels only (kc, vc are then the page pools)
};

__device__ __forceinline__ int clamp_len(int n, int max_len) {
  return n < 0 ? 0 : (n > max_len ? max_len : n);
}

// 16-byte shared-memory load.
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// A pair of fp32 values in one packed f32x2 register pair.
using pair_t = uint64_t;
__device__ __forceinline__ pair_t pmake(float a, float b) { return f2_pack(a, b); }
__device__ __forceinline__ void psplit(pair_t v, float& a, float& b) { f2_unpack(v, a, b); }
__device__ __forceinline__ pair_t pfma(pair_t a, pair_t b, pair_t c) { return f2_fma(a, b, c); }

// Two 16-bit values in one 32-bit word -> a pair (low element first).
template <bool BF16>
__device__ __forceinline__ pair_t half2_to_pair(uint32_t w) {
  if (BF16) return pmake(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&w));
  return pmake(x.x, x.y);
}

template <int D, int GT>
struct DecCfg {
  // Lanes per token row: 8 while GT*D/8 registers of q and of the accumulator stay <= 64
  // per lane, otherwise 16.
#ifdef FA_DEC_LPT
  static constexpr int LPT = FA_DEC_LPT;
#else
  static constexpr int LPT = (GT * (D / 8) <= 64) ? 8 : 16;
#endif
  static constexpr int DPL = D / LPT;                 // elements per lane (8 or 16)
  static constexpr int NV = DPL / 8;                  // 16-byte loads per lane per row
  static constexpr int TPI = 32 / LPT;                // tokens per warp instruction
  static constexpr int TPW = kDecStageTok / kDecWarps;  // tokens per warp per stage
  static constexpr int GROUPS = TPW / TPI;            // token groups per warp per stage
  static constexpr int ROW = D * 2;                   // bytes per token row
  static constexpr int STAGE_BYTES = kDecStageTok * ROW;
  static constexpr int SMEM_BYTES = 2 * kDecStages * STAGE_BYTES + 2 * kDecStages * 8 + 16;
  // Three CTAs per SM (<= 168 registers) where the head tile allows it without spills.
  static constexpr int MIN_BLOCKS = (GT == 8) ? 2 : 3;
  static_assert(GROUPS >= 1 && TPW % TPI == 0, "stage split");
};

template <int D, int GT, bool BF16, bool PAGED>
__global__ void __launch_bounds__(kDecThreads, DecCfg<D, GT>::MIN_BLOCKS)
fa_decode_split_kernel(const DecodeParams p) {
  using C = DecCfg<D, GT>;
  extern __shared__ __align__(128) uint8_t dsmem[];

  // Let the dependent combine kernel launch as soon as every split CTA has started; it
  // waits for this grid to finish before reading anything.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int split = blockIdx.x;
  const int n_gt = (p.G + GT - 1) / GT;
  const int kvh = blockIdx.y / n_gt;
  const int g0 = (blockIdx.y - kvh * n_gt) * GT;      // first query head of the group tile
  const int b = blockIdx.z;
  const int len = clamp_len(p.kv_lens[b], p.max_len);
  const int t0 = split * p.split_tokens;
  if (t0 >= len) return;                               // this split is never merged
  const int t1 = min(len, t0 + p.split_tokens);
  const int n_stages = (t1 - t0 + kDecStageTok - 1) / kDecStageTok;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane / C::LPT;                       // token of the instruction
  const int li = lane % C::LPT;                        // lane within the token's group

  const uint32_t sK = smem_u32(dsmem);
  const uint32_t sV = sK + kDecStages * C::STAGE_BYTES;
  const uint32_t bar_full = sV + kDecStages * C::STAGE_BYTES;   // kDecStages x 8 bytes
  const uint32_t bar_empty = bar_full + kDecStages * 8;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(dsmem + 2 * kDecStages * C::STAGE_BYTES +
                                                             2 * kDecStages * 8);
  const WaitCtl wc{abort_flag, &g_fa_status, p.timeout_ns};

  const size_t kv_base = (static_cast<size_t>(b) * p.Hkv + kvh) * p.max_len * D;
  const uint16_t* kg = p.kc + kv_base + static_cast<size_t>(t0) * D;
  const uint16_t* vg = p.vc + kv_base + static_cast<size_t>(t0) * D;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, kDecWarps);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();

  auto issue = [&](int st) {               // thread 0: fill ring slot st % kDecStages
    const int slot = st % kDecStages;
    const int tok0 = t0 + st * kDecStageTok;
    const int n = min(kDecStageTok, t1 - tok0);
    if constexpr (PAGED) {
      // Tokens [tok0, tok0 + n0) from one page, [tok0 + n0, tok0 + n) from the next.
      const int ps = 1 << p.pk.page_shift;
      const int n0 = min(n, ps - (tok0 & (ps - 1)));
      const int n1 = n - n0;
      const int e0 = paged_entry(p.pk, b, tok0);
      const int e1 = n1 > 0 ? paged_entry(p.pk, b, tok0 + n0) : 0;
      const bool ok0 = static_cast<unsigned>(e0) < static_cast<unsigned>(p.pk.num_pages);
      const bool ok1 = n1 > 0 && static_cast<unsigned>(e1) < static_cast<unsigned>(p.pk.num_pages);
      if (!ok0 || (n1 > 0 && !ok1)) atomicCAS(&g_fa_status, 0, kStatusBadPage);
      const uint32_t b0 = ok0 ? static_cast<uint32_t>(n0) * C::ROW : 0u;
      const uint32_t b1 = ok1 ? static_cast<uint32_t>(n1) * C::ROW : 0u;
      mbar_arrive_expect_tx(bar_full + 8 * slot, 2 * (b0 + b1));
      if (p.skip_kv_load) return;
      const size_t page_elems = static_cast<size_t>(ps) * D;
      if (ok0) {
        const size_t off = (static_cast<size_t>(e0) * p.Hkv + kvh) * page_elems +
                           static_cast<size_t>(tok0 & (ps - 1)) * D;
        bulk_load(sK + slot * C::STAGE_BYTES, p.kc + off, b0, bar_full + 8 * slot);
        bulk_load(sV + slot * C::STAGE_BYTES, p.vc + off, b0, bar_full + 8 * slot);
      }
      if (ok1) {
        const size_t off = (static_cast<size_t>(e1) * p.Hkv + kvh) * page_elems;
        bulk_load(sK + slot * C::STAGE_BYTES + n0 * C::ROW, p.kc + off, b1, bar_full + 8 * slot);
        bulk_load(sV + slot * C::STAGE_BYTES + n0 * C::ROW, p.vc + off, b1, bar_full + 8 * slot);
      }
    } else {
      const uint32_t bytes = static_cast<uint32_t>(n) * C::ROW;
      mbar_arrive_expect_tx(bar_full + 8 * slot, 2 * bytes);
      if (p.skip_kv_load) return;
      bulk_load(sK + slot * C::STAGE_BYTES, kg + static_cast<size_t>(st) * kDecStageTok * D, bytes,
                bar_full + 8 * slot);
      bulk_load(sV + slot * C::STAGE_BYTES, vg + static_cast<size_t>(st) * kDecStageTok * D, bytes,
                bar_full + 8 * slot);
    }
  };
  int issued = 0;
  if (threadIdx.x == 0) {
    for (; issued < min(kDecStages, n_stages); ++issued) issue(issued);
  }

  // This lane's slice of the query rows (pre-multiplied by scale*log2(e)) as f32x2 pairs:
  // elements [8*li, 8*li+8) (+64 for the second half when DPL = 16).
  pair_t q2[GT][C::DPL / 2];
#pragma unroll
  for (int g = 0; g < GT; ++g) {
    const bool hv = g0 + g < p.G;
    const int h = kvh * p.G + g0 + g;
#pragma unroll
    for (int nv = 0; nv < C::NV; ++nv) {
      uint4 w = make_uint4(0, 0, 0, 0);
      if (hv) w = *reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(b) * p.Hq + h) * D +
                                                  nv * (D / 2) + li * 8);
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float a, c;
        psplit(half2_to_pair<BF16>(u[e]), a, c);
        q2[g][nv * 4 + e] = pmake(a * p.scale_log2, c * p.scale_log2);
      }
    }
  }

  float m[GT], l[GT];
  pair_t acc[GT][C::DPL / 2];
#pragma unroll
  for (int g = 0; g < GT; ++g) {
    m[g] = -CUDART_INF_F;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < C::DPL / 2; ++e) acc[g][e] = pmake(0.f, 0.f);
  }

  bool ok = true;
  for (int st = 0; st < n_stages; ++st) {
    const int slot = st % kDecStages;
    if (lane == 0) ok = mbar_wait(bar_full + 8 * slot, (st / kDecStages) & 1, wc);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (!ok) break;
    const int base_tok = t0 + st * kDecStageTok + warp * C::TPW;   // first token of this warp
    const uint32_t kst = sK + slot * C::STAGE_BYTES + (warp * C::TPW) * C::ROW;
    const uint32_t vst = sV + slot * C::STAGE_BYTES + (warp * C::TPW) * C::ROW;

    float s[C::GROUPS][GT];
    bool valid[C::GROUPS];
#pragma unroll
    for (int u = 0; u < C::GROUPS; ++u) {
      const int tl = u * C::TPI + sub;                 // token within the warp's slice
      valid[u] = base_tok + tl < t1;
      uint32_t kw[C::DPL / 2];
#pragma unroll
      for (int nv = 0; nv < C::NV; ++nv) {
        const uint4 w = lds128(kst + tl * C::ROW + nv * (C::ROW / 2) + li * 16);
        kw[nv * 4 + 0] = w.x; kw[nv * 4 + 1] = w.y; kw[nv * 4 + 2] = w.z; kw[nv * 4 + 3] = w.w;
      }
#pragma unroll
      for (int g = 0; g < GT; ++g) {
        pair_t a2 = pmake(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < C::DPL / 2; ++e) a2 = pfma(q2[g][e], half2_to_pair<BF16>(kw[e]), a2);
        float x, y;
        psplit(a2, x, y);
        s[u][g] = x + y;
      }
    }
    // Sum the partial dot products over the LPT lanes of each token.
#pragma unroll
    for (int o = 1; o < C::LPT; o <<= 1) {
#pragma unroll
      for (int u = 0; u < C::GROUPS; ++u)
#pragma unroll
        for (int g = 0; g < GT; ++g) s[u][g] += __shfl_xor_sync(0xffffffffu, s[u][g], o);
    }
    // Online softmax over the warp's tokens of this stage (lazy rescale, threshold 2^8).
#pragma unroll
    for (int g = 0; g < GT; ++g) {
      float mb = -CUDART_INF_F;
#pragma unroll
      for (int u = 0; u < C::GROUPS; ++u) {
        if (!valid[u]) s[u][g] = -CUDART_INF_F;
        mb = fmaxf(mb, s[u][g]);
      }
#pragma unroll
      for (int o = C::LPT; o < 32; o <<= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
      if (mb > m[g] + 8.0f) {                          // warp-uniform
        const float alpha = (m[g] == -CUDART_INF_F) ? 0.f : ex2_approx(m[g] - mb);
        l[g] *= alpha;
        const pair_t a2 = pmake(alpha, alpha);
#pragma unroll
        for (int e = 0; e < C::DPL / 2; ++e) acc[g][e] = pfma(acc[g][e], a2, pmake(0.f, 0.f));
        m[g] = mb;
      }
    }
#pragma unroll
    for (int u = 0; u < C::GROUPS; ++u) {
      const int tl = u * C::TPI + sub;
      uint32_t vw[C::DPL / 2];
#pragma unroll
      for (int nv = 0; nv < C::NV; ++nv) {
        uint4 w = lds128(vst + tl * C::ROW + nv * (C::ROW / 2) + li * 16);
        if (!valid[u]) w = make_uint4(0, 0, 0, 0);     // slot bytes past the split: never used
        vw[nv * 4 + 0] = w.x; vw[nv * 4 + 1] = w.y; vw[nv * 4 + 2] = w.z; vw[nv * 4 + 3] = w.w;
      }
#pragma unroll
      for (int g = 0; g < GT; ++g) {
        // A warp whose tokens were all past the end still has m = -inf: use 0 there.
        const float mref = (m[g] == -CUDART_INF_F) ? 0.f : m[g];
        const float pr = ex2_approx(s[u][g] - mref);   // 0 for invalid tokens (s = -inf)
        l[g] += pr;
        const pair_t p2 = pmake(pr, pr);
#pragma unroll
        for (int e = 0; e < C::DPL / 2; ++e) acc[g][e] = pfma(p2, half2_to_pair<BF16>(vw[e]), acc[g][e]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_empty + 8 * slot);
    // Refill the slot the whole CTA has finished with.
    if (threadIdx.x == 0 && issued < n_stages) {
      const int rs = issued % kDecStages;              // == slot of stage issued - kDecStages
      if (mbar_wait(bar_empty + 8 * rs, ((issued / kDecStages) - 1) & 1, wc)) {
        issue(issued);
        ++issued;
      }
    }
  }
  if (threadIdx.x == 0 && *abort_flag) {
    // Copies still in flight must land before the CTA exits.
    for (int k = max(0, issued - kDecStages); k < issued; ++k)
      mbar_wait_drain(bar_full + 8 * (k % kDecStages), (k / kDecStages) & 1, 200000000ull);
  }

  // Merge the token sub-groups of the warp (they share m).
#pragma unroll
  for (int o = C::LPT; o < 32; o <<= 1) {
#pragma unroll
    for (int g = 0; g < GT; ++g) {
      l[g] += __shfl_xor_sync(0xffffffffu, l[g], o);
#pragma unroll
      for (int e = 0; e < C::DPL / 2; ++e) {
        float x, y;
        psplit(acc[g][e], x, y);
        x += __shfl_xor_sync(0xffffffffu, x, o);
        y += __shfl_xor_sync(0xffffffffu, y, o);
        acc[g][e] = pmake(x, y);
      }
    }
  }

  // Cross-warp merge through shared memory (the K ring is free now).
  __syncthreads();
  float* sm_acc = reinterpret_cast<float*>(dsmem);                      // [warps][GT][D]
  float* sm_m = sm_acc + kDecWarps * GT * D;                            // [warps][GT]
  float* sm_l = sm_m + kDecWarps * GT;
  if (lane < C::LPT) {
#pragma unroll
    for (int g = 0; g < GT; ++g)
#pragma unroll
      for (int nv = 0; nv < C::NV; ++nv)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float x, y;
          psplit(acc[g][nv * 4 + e], x, y);
          const int d0 = nv * (D / 2) + li * 8 + 2 * e;
          sm_acc[(warp * GT + g) * D + d0] = x;
          sm_acc[(warp * GT + g) * D + d0 + 1] = y;
        }
  }
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < GT; ++g) {
      sm_m[warp * GT + g] = m[g];
      sm_l[warp * GT + g] = l[g];
    }
  }
  __syncthreads();
  if (!ok || *abort_flag) return;

  for (int idx = threadIdx.x; idx < GT * D; idx += kDecThreads) {
    const int g = idx / D;
    const int e = idx - g * D;
    if (g0 + g >= p.G) continue;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, sm_m[w * GT + g]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      const float mw = sm_m[w * GT + g];
      const float wt = (mw == -CUDART_INF_F) ? 0.f : ex2_approx(mw - M);
      L = fmaf(wt, sm_l[w * GT + g], L);
      O = fmaf(wt, sm_acc[(w * GT + g) * D + e], O);
    }
    const int h = kvh * p.G + g0 + g;
    const size_t row = (static_cast<size_t>(b) * p.Hq + h) * p.n_split + split;
    p.ws_o[row * D + e] = O / L;
    if (e == 0) p.ws_lse[row] = M + __log2f(L);
  }
}

struct CombineParams {
  const float* ws_o;
  const float* ws_lse;
  const int* kv_lens;
  uint16_t* o;            // [B, Hq, D]
  float* lse;             // [B, Hq] or nullptr
  int Hq, max_len, split_tokens, n_split;
};

template <int D, bool BF16>
__global__ void __launch_bounds__(D)
fa_decode_combine_kernel(const CombineParams p) {
  const int bh = blockIdx.x;
  const int b = bh / p.Hq;
  const int e = threadIdx.x;
  // kv_lens is an input, not a result of the split kernel: read it before the wait.
  const int len = clamp_len(p.kv_lens[b], p.max_len);
  const int ns = (len + p.split_tokens - 1) / p.split_tokens;
  const float* lse_s = p.ws_lse + static_cast<size_t>(bh) * p.n_split;
  const float* o_s = p.ws_o + static_cast<size_t>(bh) * p.n_split * D;
  // Launched as a programmatic dependent of the split kernel: wait until it has finished
  // and its writes are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // The first kU splits' LSE and partial rows are all requested before any is used (one
  // round trip); longer split lists continue in a loop.
  constexpr int kU = 8;
  float ls[kU], ov[kU];
#pragma unroll
  for (int s = 0; s < kU; ++s) {
    ls[s] = s < ns ? lse_s[s] : -CUDART_INF_F;
    ov[s] = s < ns ? o_s[static_cast<size_t>(s) * D + e] : 0.f;
  }
  float M = -CUDART_INF_F;
#pragma unroll
  for (int s = 0; s < kU; ++s) M = fmaxf(M, ls[s]);
  for (int s = kU; s < ns; ++s) M = fmaxf(M, lse_s[s]);
  float L = 0.f, O = 0.f;
#pragma unroll
  for (int s = 0; s < kU; ++s) {
    if (s < ns) {
      const float w = ex2_approx(ls[s] - M);
      L += w;
      O = fmaf(w, ov[s], O);
    }
  }
  for (int s = kU; s < ns; ++s) {
    const float w = ex2_approx(lse_s[s] - M);
    L += w;
    O = fmaf(w, o_s[static_cast<size_t>(s) * D + e], O);
  }
  const float out = (ns > 0) ? O / L : 0.f;
  if (BF16) {
    const __nv_bfloat16 x = __float2bfloat16_rn(out);
    p.o[static_cast<size_t>(bh) * D + e] = *reinterpret_cast<const uint16_t*>(&x);
  } else {
    const __half x = __float2half_rn(out);
    p.o[static_cast<size_t>(bh) * D + e] = *reinterpret_cast<const uint16_t*>(&x);
  }
  if (e == 0 && p.lse != nullptr)
    p.lse[bh] = (ns > 0) ? (M + __log2f(L)) * 0.69314718055994530942f : -CUDART_INF_F;
}

}  // namespace fa
