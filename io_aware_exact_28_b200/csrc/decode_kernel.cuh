// decode_kernel.cuh — single-token attention over a grouped-query KV cache, split-KV.
//
// Decode reads every valid K and V row of the cache once per step, so it is bound by
// device-memory bandwidth (page "Empreinte mémoire et calcul des couches Transformer":
// KV-cache size per token and the memory-bound character of cache access). The kernel
// therefore streams the cache with coalesced 128-bit loads, reads each K/V row once for
// all G = Hq/Hkv query heads that share it, and keeps the math in fp32 registers.
//
// Split kernel: grid (split, kv head x head tile, sequence), 128 threads. A split covers
// up to `split_tokens` consecutive cache rows. Each token row is read by D/8 lanes (8
// elements = 16 bytes per lane); each warp runs its own online softmax over its tokens
// (running max with the same lazy-rescale rule as the prefill kernel), the four warps
// merge through shared memory, and the CTA writes a normalised partial O row and its
// log2-domain logsumexp per query head.
//
// Combine kernel: grid (sequence x query head), D threads. Merges the valid splits with
// weights 2^(lse_s - max) (the online-softmax rescaling identity, page "Kotaemon
// FlashAttention", running max and normaliser bullet) and writes O (16-bit) and the
// natural-log LSE.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include "sm100.cuh"

namespace fa {

constexpr int kDecThreads = 128;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecUnroll = 4;       // token groups per warp per batch (loads in flight)

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
};

__device__ __forceinline__ uint4 ld_stream_u4(const void* ptr) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(ptr));
  return v;
}

template <bool BF16>
__device__ __forceinline__ void unpack8(const uint4& w, float (&f)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (BF16) {
      f[2 * i] = __uint_as_float(u[i] << 16);
      f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    } else {
      const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&u[i]));
      f[2 * i] = x.x;
      f[2 * i + 1] = x.y;
    }
  }
}

__device__ __forceinline__ int clamp_len(int n, int max_len) {
  return n < 0 ? 0 : (n > max_len ? max_len : n);
}

template <int D, int GT, bool BF16>
__global__ void __launch_bounds__(kDecThreads)
fa_decode_split_kernel(const DecodeParams p) {
  constexpr int LPT = D / 8;           // lanes per token row
  constexpr int TPI = 32 / LPT;        // tokens per warp per load instruction
  constexpr int TOK_PER_BATCH = kDecUnroll * kDecWarps * TPI;

  const int split = blockIdx.x;
  const int n_gt = (p.G + GT - 1) / GT;
  const int kvh = blockIdx.y / n_gt;
  const int g0 = (blockIdx.y - kvh * n_gt) * GT;      // first query head of the group tile
  const int b = blockIdx.z;
  const int len = clamp_len(p.kv_lens[b], p.max_len);
  const int t0 = split * p.split_tokens;
  if (t0 >= len) return;                               // this split is never merged
  const int t1 = min(len, t0 + p.split_tokens);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPT;                          // which token of the instruction
  const int dofs = (lane % LPT) * 8;

  const size_t kv_base = (static_cast<size_t>(b) * p.Hkv + kvh) * p.max_len * D;
  const uint16_t* kp = p.kc + kv_base + dofs;
  const uint16_t* vp = p.vc + kv_base + dofs;

  // This lane's slice of the query rows, pre-multiplied by scale*log2(e).
  float qf[GT][8];
#pragma unroll
  for (int g = 0; g < GT; ++g) {
    const int h = kvh * p.G + g0 + g;
    if (g0 + g < p.G) {
      const uint4 w = *reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(b) * p.Hq + h) * D + dofs);
      unpack8<BF16>(w, qf[g]);
#pragma unroll
      for (int e = 0; e < 8; ++e) qf[g][e] *= p.scale_log2;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) qf[g][e] = 0.f;
    }
  }

  float m[GT], l[GT], acc[GT][8];
#pragma unroll
  for (int g = 0; g < GT; ++g) {
    m[g] = -CUDART_INF_F;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
  }

  for (int base = t0; base < t1; base += TOK_PER_BATCH) {
    uint4 kw[kDecUnroll], vw[kDecUnroll];
    bool valid[kDecUnroll];
#pragma unroll
    for (int u = 0; u < kDecUnroll; ++u) {
      const int tok = base + (u * kDecWarps + warp) * TPI + sub;
      valid[u] = tok < t1;
      if (valid[u]) {
        kw[u] = ld_stream_u4(kp + static_cast<size_t>(tok) * D);
        vw[u] = ld_stream_u4(vp + static_cast<size_t>(tok) * D);
      } else {
        kw[u] = make_uint4(0, 0, 0, 0);
        vw[u] = make_uint4(0, 0, 0, 0);
      }
    }
    float s[kDecUnroll][GT];
#pragma unroll
    for (int u = 0; u < kDecUnroll; ++u) {
      float kf[8];
      unpack8<BF16>(kw[u], kf);
#pragma unroll
      for (int g = 0; g < GT; ++g) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaf(qf[g][e], kf[e], a);
        s[u][g] = a;
      }
    }
    // Sum the partial dot products over the LPT lanes that share a token.
#pragma unroll
    for (int o = 1; o < LPT; o <<= 1) {
#pragma unroll
      for (int u = 0; u < kDecUnroll; ++u)
#pragma unroll
        for (int g = 0; g < GT; ++g) s[u][g] += __shfl_xor_sync(0xffffffffu, s[u][g], o);
    }
#pragma unroll
    for (int g = 0; g < GT; ++g) {
      float mb = -CUDART_INF_F;
#pragma unroll
      for (int u = 0; u < kDecUnroll; ++u) {
        if (!valid[u]) s[u][g] = -CUDART_INF_F;
        mb = fmaxf(mb, s[u][g]);
      }
#pragma unroll
      for (int o = LPT; o < 32; o <<= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
      if (mb > m[g] + 8.0f) {                          // warp-uniform lazy rescale
        const float alpha = (m[g] == -CUDART_INF_F) ? 0.f : ex2_approx(m[g] - mb);
        l[g] *= alpha;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[g][e] *= alpha;
        m[g] = mb;
      }
    }
#pragma unroll
    for (int u = 0; u < kDecUnroll; ++u) {
      float vf[8];
      unpack8<BF16>(vw[u], vf);
#pragma unroll
      for (int g = 0; g < GT; ++g) {
        // A warp whose tokens were all past the end still has m = -inf: use 0 there.
        const float mref = (m[g] == -CUDART_INF_F) ? 0.f : m[g];
        const float pr = ex2_approx(s[u][g] - mref);   // 0 for invalid tokens (s = -inf)
        l[g] += pr;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(pr, vf[e], acc[g][e]);
      }
    }
  }

  // Merge the token sub-groups of the warp (they share m).
#pragma unroll
  for (int o = LPT; o < 32; o <<= 1) {
#pragma unroll
    for (int g = 0; g < GT; ++g) {
      l[g] += __shfl_xor_sync(0xffffffffu, l[g], o);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], o);
    }
  }

  __shared__ float sm_m[kDecWarps][GT];
  __shared__ float sm_l[kDecWarps][GT];
  __shared__ __align__(16) float sm_acc[kDecWarps][GT][D];
  if (lane < LPT) {
#pragma unroll
    for (int g = 0; g < GT; ++g) {
#pragma unroll
      for (int e = 0; e < 8; ++e) sm_acc[warp][g][dofs + e] = acc[g][e];
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < GT; ++g) {
      sm_m[warp][g] = m[g];
      sm_l[warp][g] = l[g];
    }
  }
  __syncthreads();

  for (int idx = threadIdx.x; idx < GT * D; idx += kDecThreads) {
    const int g = idx / D;
    const int e = idx - g * D;
    if (g0 + g >= p.G) continue;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, sm_m[w][g]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      const float wt = (sm_m[w][g] == -CUDART_INF_F) ? 0.f : ex2_approx(sm_m[w][g] - M);
      L = fmaf(wt, sm_l[w][g], L);
      O = fmaf(wt, sm_acc[w][g][e], O);
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
  const int len = clamp_len(p.kv_lens[b], p.max_len);
  const int ns = (len + p.split_tokens - 1) / p.split_tokens;
  const float* lse_s = p.ws_lse + static_cast<size_t>(bh) * p.n_split;
  const float* o_s = p.ws_o + static_cast<size_t>(bh) * p.n_split * D;
  float M = -CUDART_INF_F;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, lse_s[s]);
  float L = 0.f, O = 0.f;
  for (int s = 0; s < ns; ++s) {
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
