// fa_api.cu — host side of the C ABI declared in include/fa.h: argument checks, TMA
// descriptors, launch configuration and status reporting. Compiled for sm_100a only.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "fa.h"
#include "decode_kernel.cuh"
#include "decode_tc_kernel.cuh"
#include "fwd_kernel.cuh"
#include "bwd_kernel.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;   // 2 s

// Test hooks, set by fa_set_wait_timeout_ns / fa_debug_skip_q_load and read by every
// launch; atomics, since the setters may run on another host thread.
std::atomic<uint64_t> g_timeout_ns{kDefaultTimeoutNs};
std::atomic<int> g_skip_q_load{0};

// ---------------------------------------------------------------------------------------
// Device checks (cached per device)
// ---------------------------------------------------------------------------------------
enum DevState : int { kUnknown = 0, kSupported = 1, kUnsupported = 2 };
int g_dev_state[kMaxDevices];
std::mutex g_mu;

fa_status check_device(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  *dev_out = dev;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_dev_state[dev] == kUnknown) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return FA_ERR_CUDA;
    g_dev_state[dev] = (major == 10 && minor == 0) ? kSupported : kUnsupported;
  }
  return g_dev_state[dev] == kSupported ? FA_OK : FA_ERR_UNSUPPORTED;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------------------------------
// TMA descriptors through the driver entry point (no link-time dependency on libcuda)
// ---------------------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [heads, rows, d] 16-bit view whose heads start head_rows rows apart in memory
// (head_rows >= rows; 0 means rows). Box = 64 columns (128 bytes) x box_rows rows x 1
// head, 128-byte swizzle; rows past `rows` read as zero and are clipped on store.
bool make_tile_map(CUtensorMap* m, const void* ptr, int d, int rows, long long heads, bool bf16,
                   int box_rows, long long head_rows = 0) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(head_rows > 0 ? head_rows : rows) * d * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
             const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [heads, rows, d] 8-bit (E4M3) view: box = 128 columns (128 bytes) x box_rows rows x 1
// head, 128-byte swizzle; rows past `rows` read as zero.
bool make_tile_map8(CUtensorMap* m, const void* ptr, int d, int rows, long long heads,
                    int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d),
                                 static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(d)};
  const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------------------
// Backward launch: D and L * log2(e), then one grid for dK / dV and dQ (stream-ordered).
// ---------------------------------------------------------------------------------------
template <typename K>
bool set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
         cudaSuccess;
}

// Tensor maps of the backward pass: 128-row boxes for the tile a CTA keeps resident and
// TN-row boxes (BwdCfg<D>::TN) for the tiles it streams.
struct BwdMaps {
  CUtensorMap q, dout, k, v;          // 128-row boxes
  CUtensorMap q_s, dout_s, k_s, v_s;  // TN-row boxes
};

template <int D, bool BF16>
fa_status launch_bwd(int dev, const BwdMaps& m, const void* o, const void* dout, const float* lse,
                     void* dq, void* dk, void* dv, fa::BwdParams prm, long long BH, long long BHkv,
                     int n_q, int n_k, int causal, cudaStream_t st) {
  using C = fa::BwdCfg<D>;
  auto fused_c = fa::fa_bwd_fused_kernel<D, BF16, true>;
  auto fused_n = fa::fa_bwd_fused_kernel<D, BF16, false>;
  static int ready[kMaxDevices];
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!ready[dev]) {
      if (!set_smem(fused_c, C::SMEM_BYTES) || !set_smem(fused_n, C::SMEM_BYTES)) return FA_ERR_CUDA;
      ready[dev] = 1;
    }
  }
  const long long threads = BH * prm.Nq_pad * (D / 8);
  fa::fa_bwd_preprocess_kernel<D, BF16><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(
      static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout), lse,
      const_cast<float*>(prm.lse2), const_cast<float*>(prm.dsum), static_cast<int>(BH), prm.Nq,
      prm.Nq_pad);
  fa::BwdParams pq = prm, pk = prm;
  pq.out = dq;
  pq.out2 = nullptr;
  pk.out = dk;
  pk.out2 = dv;
  const unsigned nb = static_cast<unsigned>(n_k * BHkv + n_q * BH);
  if (causal)
    fused_c<<<nb, C::THREADS, C::SMEM_BYTES, st>>>(m.q, m.k_s, m.v_s, m.dout, m.q_s, m.k, m.v,
                                                    m.dout_s, pq, pk, n_k, n_q, static_cast<int>(BHkv),
                                                    static_cast<int>(BH));
  else
    fused_n<<<nb, C::THREADS, C::SMEM_BYTES, st>>>(m.q, m.k_s, m.v_s, m.dout, m.q_s, m.k, m.v,
                                                    m.dout_s, pq, pk, n_k, n_q, static_cast<int>(BHkv),
                                                    static_cast<int>(BH));
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------
// Forward launch
// ---------------------------------------------------------------------------------------
// K/V maps of one call: the whole cache, and (paged) the last page's used rows.
struct KVMaps {
  CUtensorMap k, v, kt, vt;
};

template <int D, bool BF16, bool CAUSAL, bool PAGED, bool FP8 = false, bool VARLEN = false,
          bool KVMAJOR = false>
fa_status launch_fwd(int dev, const CUtensorMap& mq, const KVMaps& kv, const fa::FwdParams& prm,
                     cudaStream_t stream) {
  using C = fa::FwdCfg<D, FP8>;
  auto kernel = fa::fa_fwd_kernel<D, BF16, CAUSAL, PAGED, FP8, VARLEN, KVMAJOR>;
  static int attr_state[kMaxDevices];   // 0 unknown, 1 ready, 2 unusable build
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (attr_state[dev] == 0) {
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared) != cudaSuccess)
        return FA_ERR_CUDA;
      // The in-kernel register re-split hands out exactly the launch allocation; a build
      // whose compiled register count differs would make it wait forever, so refuse it.
      cudaFuncAttributes fattr;
      if (cudaFuncGetAttributes(&fattr, kernel) != cudaSuccess) return FA_ERR_CUDA;
      attr_state[dev] =
          (!C::REGSPLIT || static_cast<uint32_t>(fattr.numRegs) == C::REGS_LAUNCH) ? 1 : 2;
    }
    if (attr_state[dev] != 1) return FA_ERR_UNSUPPORTED;
  }
  // One CTA per work unit (C::QT Q tiles of a (batch, head)); running CTAs take over the
  // ones that have not started, so the grid size only bounds the work, not the residency.
  fa::FwdParams p = prm;
  const long long n_qb = (p.Nq + C::QT * fa::kBM - 1) / (C::QT * fa::kBM);
  if (static_cast<long long>(p.BH) * n_qb >= (1LL << 31)) return FA_ERR_INVALID_ARG;
  p.n_qb = static_cast<int>(n_qb);
  const unsigned n_units = static_cast<unsigned>(p.BH) * static_cast<unsigned>(p.n_qb);
  kernel<<<n_units, C::THREADS, C::SMEM_BYTES, stream>>>(mq, kv.k, kv.v, kv.kt, kv.vt, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D, bool BF16, bool VARLEN>
fa_status dispatch_causal(int causal, bool paged, int dev, const CUtensorMap& mq, const KVMaps& kv,
                          const fa::FwdParams& prm, cudaStream_t st, bool kv_major) {
  if constexpr (!VARLEN) {
    if (!paged && kv_major)
      return causal ? launch_fwd<D, BF16, true, false, false, false, true>(dev, mq, kv, prm, st)
                    : launch_fwd<D, BF16, false, false, false, false, true>(dev, mq, kv, prm, st);
  }
  if (paged)
    return causal ? launch_fwd<D, BF16, true, true, false, VARLEN>(dev, mq, kv, prm, st)
                  : launch_fwd<D, BF16, false, true, false, VARLEN>(dev, mq, kv, prm, st);
  return causal ? launch_fwd<D, BF16, true, false, false, VARLEN>(dev, mq, kv, prm, st)
                : launch_fwd<D, BF16, false, false, false, VARLEN>(dev, mq, kv, prm, st);
}

template <int D, bool BF16>
fa_status dispatch_varlen(bool varlen, int causal, bool paged, int dev, const CUtensorMap& mq,
                          const KVMaps& kv, const fa::FwdParams& prm, cudaStream_t st,
                          bool kv_major) {
  return varlen ? dispatch_causal<D, BF16, true>(causal, paged, dev, mq, kv, prm, st, false)
                : dispatch_causal<D, BF16, false>(causal, paged, dev, mq, kv, prm, st, kv_major);
}

// ---------------------------------------------------------------------------------------
// Decode sizing: the split length depends only on (B, Hq, max_kv_len) so that the
// workspace query and the launch always agree.
// ---------------------------------------------------------------------------------------
// Build define FA_DECODE_SPLIT_TOKENS (a power of two in [32, 4096]) overrides the choice
// (0: the sizing below).
#ifndef FA_DECODE_SPLIT_TOKENS
#define FA_DECODE_SPLIT_TOKENS 0
#endif
static_assert(FA_DECODE_SPLIT_TOKENS == 0 ||
                  (FA_DECODE_SPLIT_TOKENS >= 32 && FA_DECODE_SPLIT_TOKENS <= 4096 &&
                   (FA_DECODE_SPLIT_TOKENS & (FA_DECODE_SPLIT_TOKENS - 1)) == 0),
              "FA_DECODE_SPLIT_TOKENS: a power of two in [32, 4096], or 0");
constexpr int split_tokens_override() { return FA_DECODE_SPLIT_TOKENS; }

int decode_split_tokens(int B, int Hq, int max_len) {
  if (split_tokens_override()) return split_tokens_override();
  const long long units = static_cast<long long>(B) * (Hq >= 4 ? Hq / 4 : 1);
  int s = 256;
  while (s > 64 && units * ((max_len + s - 1) / s) < 148LL * 8) s >>= 1;
  return s;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct DecodeLayout {
  int split_tokens, n_split;
  size_t o_bytes, lse_off, ticket_off, total;
};

// d = 128 decodes on the tensor cores in 128-token tiles (decode_tc_kernel.cuh) unless the
// build define FA_DECODE_CUDA_CORES=1 selects the CUDA-core kernel (decode_kernel.cuh).
#ifndef FA_DECODE_CUDA_CORES
#define FA_DECODE_CUDA_CORES 0
#endif
bool use_tc_decode(int d) { return d == fa::kTcD && !FA_DECODE_CUDA_CORES; }

bool decode_layout(int B, int Hq, int max_len, int d, DecodeLayout* L) {
  if (B <= 0 || Hq <= 0 || max_len <= 0 || d <= 0) return false;
  if (use_tc_decode(d)) {
    // Splits of whole 128-token tiles; 1024 tokens (8 tiles) unless overridden (measured
    // best on the 4096-token-cache workload: fewer unit boundaries per CTA).
    const int o = split_tokens_override();
    L->split_tokens = o ? ((o + fa::kTcTile - 1) / fa::kTcTile) * fa::kTcTile : 8 * fa::kTcTile;
  } else {
    L->split_tokens = decode_split_tokens(B, Hq, max_len);
  }
  L->n_split = (max_len + L->split_tokens - 1) / L->split_tokens;
  const size_t rows = static_cast<size_t>(B) * Hq * L->n_split;
  L->o_bytes = align_up(rows * d * sizeof(float), 256);
  L->lse_off = L->o_bytes;
  L->ticket_off = L->lse_off + align_up(rows * sizeof(float), 256);   // tensor-core unit counter
  L->total = L->ticket_off + 256;
  return true;
}

// The combine is a programmatic dependent launch: it is scheduled while the split
// kernel's last CTAs run and waits (griddepcontrol.wait) for its results.
template <int D, bool BF16>
fa_status launch_combine_pdl(const fa::CombineParams& cp, int B, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(B * cp.Hq, 1, 1);
  cfg.blockDim = dim3(D, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, fa::fa_decode_combine_kernel<D, BF16>, cp) != cudaSuccess)
    return FA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D, int GT, bool BF16, bool PAGED>
fa_status launch_decode_t(int dev, const fa::DecodeParams& dp, const fa::CombineParams& cp,
                          int B, int Hkv, int G, cudaStream_t st) {
  using C = fa::DecCfg<D, GT>;
  auto split_kernel = fa::fa_decode_split_kernel<D, GT, BF16, PAGED>;
  static bool attr_set[kMaxDevices];
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!attr_set[dev]) {
      if (cudaFuncSetAttribute(split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               C::SMEM_BYTES) != cudaSuccess)
        return FA_ERR_CUDA;
      attr_set[dev] = true;
    }
  }
  const int n_gt = (G + GT - 1) / GT;
  dim3 grid(dp.n_split, Hkv * n_gt, B);
  split_kernel<<<grid, fa::kDecThreads, C::SMEM_BYTES, st>>>(dp);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  return launch_combine_pdl<D, BF16>(cp, B, st);
}

template <int D, bool BF16, bool PAGED>
fa_status launch_decode_g(int dev, const fa::DecodeParams& dp, const fa::CombineParams& cp,
                          int B, int Hkv, int G, cudaStream_t st) {
  if (G <= 1) return launch_decode_t<D, 1, BF16, PAGED>(dev, dp, cp, B, Hkv, G, st);
  if (G <= 2) return launch_decode_t<D, 2, BF16, PAGED>(dev, dp, cp, B, Hkv, G, st);
  if (G <= 4) return launch_decode_t<D, 4, BF16, PAGED>(dev, dp, cp, B, Hkv, G, st);
  return launch_decode_t<D, 8, BF16, PAGED>(dev, dp, cp, B, Hkv, G, st);
}

// Paged-cache arguments of one call (host side); see include/fa.h.
struct PagedArgs {
  const int* table;
  int num_pages, page_size, max_pages;
  fa::PagedKV device(int Hkv) const {
    fa::PagedKV pk;
    pk.table = table;
    pk.max_pages = max_pages;
    pk.page_shift = 0;
    while ((1 << pk.page_shift) < page_size) ++pk.page_shift;
    pk.num_pages = num_pages;
    pk.Hkv = Hkv;
    return pk;
  }
};

fa_status check_paged(const PagedArgs& pg, int Hkv) {
  if (!pg.table || pg.num_pages <= 0 || pg.max_pages <= 0 || pg.page_size <= 0)
    return FA_ERR_INVALID_ARG;
  if (pg.page_size < 16 || (pg.page_size & (pg.page_size - 1)) != 0) return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(pg.max_pages) * pg.page_size >= (1LL << 31) ||
      static_cast<long long>(pg.num_pages) * Hkv >= (1LL << 31) - 1)
    return FA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(pg.table) & 3u) return FA_ERR_ALIGNMENT;
  return FA_OK;
}

template <bool BF16, int GT, bool PAGED>
fa_status launch_decode_tc_t(int dev, const void* q, const void* kc, const void* vc,
                           const int* kv_lens, uint8_t* ws, const DecodeLayout& L, int B, int Hq,
                           int Hkv, int max_len, float scale, const fa::CombineParams& cp,
                           const PagedArgs* pg, cudaStream_t st) {
  auto kernel = fa::fa_decode_tc_kernel<BF16, GT, PAGED>;
  static int sm_count[kMaxDevices];
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (sm_count[dev] == 0) {
      int n = 0;
      if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
          cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               fa::kTcSmemBytes) != cudaSuccess)
        return FA_ERR_CUDA;
      sm_count[dev] = n;
    }
  }
  CUtensorMap mk, mv, mq;
  const long long BHkv = static_cast<long long>(B) * Hkv;
  // q as [1, B*Hq, 128]: 16-row boxes, one per work unit (rows past B*Hq read as zero).
  // Paged pools as [num_pages*Hkv, page_size, 128] with boxes of min(page_size, 128) rows.
  if (PAGED) {
    const long long heads = static_cast<long long>(pg->num_pages) * Hkv;
    const int box = pg->page_size < fa::kTcTile ? pg->page_size : fa::kTcTile;
    if (!make_tile_map(&mk, kc, fa::kTcD, pg->page_size, heads, BF16, box) ||
        !make_tile_map(&mv, vc, fa::kTcD, pg->page_size, heads, BF16, box))
      return FA_ERR_CUDA;
  } else if (!make_tile_map(&mk, kc, fa::kTcD, max_len, BHkv, BF16, fa::kTcTile) ||
             !make_tile_map(&mv, vc, fa::kTcD, max_len, BHkv, BF16, fa::kTcTile)) {
    return FA_ERR_CUDA;
  }
  if (!make_tile_map(&mq, q, fa::kTcD, B * Hq, 1, BF16, fa::kTcN)) return FA_ERR_CUDA;
  fa::DecodeTcParams tp;
  tp.kv_lens = kv_lens;
  tp.tickets = reinterpret_cast<unsigned*>(ws + L.ticket_off);
  tp.ws_o = reinterpret_cast<float*>(ws);
  tp.ws_lse = reinterpret_cast<float*>(ws + L.lse_off);
  tp.B = B;
  tp.Hq = Hq;
  tp.Hkv = Hkv;
  tp.G = Hq / Hkv;
  tp.GT = GT;
  tp.n_gt = (tp.G + tp.GT - 1) / tp.GT;
  tp.max_len = max_len;
  tp.split_tokens = L.split_tokens;
  tp.n_split = L.n_split;
  tp.scale_log2 = scale * 1.4426950408889634f;
  tp.timeout_ns = g_timeout_ns.load(std::memory_order_relaxed);
  tp.skip_q_load = g_skip_q_load.load(std::memory_order_relaxed);
  tp.pk = PAGED ? pg->device(Hkv) : fa::PagedKV{};
  const long long n_units = static_cast<long long>(L.n_split) * B * Hkv * tp.n_gt;
  if (n_units >= (1LL << 31)) return FA_ERR_INVALID_ARG;
  const int grid = static_cast<int>(n_units < sm_count[dev] ? n_units : sm_count[dev]);
  // The unit counter starts at zero on every call: a one-thread kernel stores the zero,
  // and the split kernel, its programmatic dependent, overlaps its own start with it.
  fa::fa_decode_ticket_reset_kernel<<<1, 32, 0, st>>>(tp.tickets);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(fa::kTcThreads, 1, 1);
  cfg.dynamicSmemBytes = fa::kTcSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, mk, mv, mq, tp) != cudaSuccess) return FA_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  return launch_combine_pdl<fa::kTcD, BF16>(cp, B, st);
}

// Head tile = the smallest of 1, 2, 4, 8, 16 that holds G (16 tiles larger groups).
template <bool BF16, bool PAGED>
fa_status launch_decode_tc(int dev, const void* q, const void* kc, const void* vc,
                           const int* kv_lens, uint8_t* ws, const DecodeLayout& L, int B, int Hq,
                           int Hkv, int max_len, float scale, const fa::CombineParams& cp,
                           const PagedArgs* pg, cudaStream_t st) {
  const int G = Hq / Hkv;
#define FA_TC_CASE(GT_)                                                                           \
  return launch_decode_tc_t<BF16, GT_, PAGED>(dev, q, kc, vc, kv_lens, ws, L, B, Hq, Hkv, max_len, \
                                              scale, cp, pg, st)
  if (G <= 1) FA_TC_CASE(1);
  if (G <= 2) FA_TC_CASE(2);
  if (G <= 4) FA_TC_CASE(4);
  if (G <= 8) FA_TC_CASE(8);
  FA_TC_CASE(16);
#undef FA_TC_CASE
}

fa_status common_checks(int B, int Hq, int Hkv, int d, float scale, int dtype) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// Prefill unit order of the uniform 16-bit kernels: KV head by KV head when the call's K
// and V (all heads, Nk keys) exceed half of the 126 MB L2, so that they would not stay
// resident while every KV head streams at once; measured on B200, gqa32k (134 MB): DRAM
// reads 1.89 -> 0.40 GB at the same speed; gqa8k (34 MB, resident either way): 4% slower,
// so it keeps query-block order. (Paged, per-sequence-length and E4M3 calls keep it too.)
int kv_major_order(int B, int Hq, int Hkv, int Nk, int d, int elem_bytes) {
  if (Hq == Hkv) return 0;
  const long long kv_bytes = 2LL * B * Hkv * static_cast<long long>(Nk) * d * elem_bytes;
  return kv_bytes > (63LL << 20) ? 1 : 0;
}

// fa_fwd, fa_fwd_kvcache and fa_fwd_paged: K/V heads hold kv_rows rows in memory, of which
// Nk are used; pg != nullptr reads them from a page pool instead. q_lens / kv_lens (device,
// may be null) give each sequence its own query rows (<= Nq) and keys (<= Nk).
fa_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                   int Hkv, int Nq, int Nk, long long kv_rows, int d, int causal, float scale,
                   fa_dtype dtype, const PagedArgs* pg, void* stream, const int* q_lens = nullptr,
                   const int* kv_lens = nullptr) {
  if (!q || !k || !v || !o) return FA_ERR_INVALID_ARG;
  if (Nq <= 0 || Nk <= 0 || (causal != 0 && causal != 1)) return FA_ERR_INVALID_ARG;
  fa_status s = common_checks(B, Hq, Hkv, d, scale, dtype);
  if (s != FA_OK) return s;
  if (pg) {
    s = check_paged(*pg, Hkv);
    if (s != FA_OK) return s;
    if (static_cast<long long>(pg->max_pages) * pg->page_size < Nk) return FA_ERR_INVALID_ARG;
  }
  const long long BH = static_cast<long long>(B) * Hq;
  const long long BHkv = static_cast<long long>(B) * Hkv;
  if (BH >= (1LL << 31)) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FA_ERR_ALIGNMENT;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FA_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(q_lens) & 3u) || (reinterpret_cast<uintptr_t>(kv_lens) & 3u))
    return FA_ERR_ALIGNMENT;
  int dev = 0;
  s = check_device(&dev);
  if (s != FA_OK) return s;

  const bool bf16 = dtype == FA_BF16;
  const bool varlen = q_lens != nullptr || kv_lens != nullptr;
  CUtensorMap mq;
  KVMaps kv;
  const int kv_box = (d == 64) ? fa::FwdCfg<64>::BN : fa::FwdCfg<128>::BN;
  if (!make_tile_map(&mq, q, d, Nq, BH, bf16, fa::kBM)) return FA_ERR_CUDA;
  if (pg) {
    // [num_pages*Hkv, page_size, d] views; the tail maps end at the last page's used rows.
    const long long heads = static_cast<long long>(pg->num_pages) * Hkv;
    const int box = pg->page_size < kv_box ? pg->page_size : kv_box;
    // (Per-sequence lengths do without tail maps: the kernel zeroes V rows past each
    // sequence's last key in shared memory.)
    const int tail_rows = Nk - ((Nk - 1) / pg->page_size) * pg->page_size;
    if (!make_tile_map(&kv.k, k, d, pg->page_size, heads, bf16, box) ||
        !make_tile_map(&kv.v, v, d, pg->page_size, heads, bf16, box) ||
        !make_tile_map(&kv.kt, k, d, tail_rows, heads, bf16, box, pg->page_size) ||
        !make_tile_map(&kv.vt, v, d, tail_rows, heads, bf16, box, pg->page_size))
      return FA_ERR_CUDA;
  } else {
    if (!make_tile_map(&kv.k, k, d, Nk, BHkv, bf16, kv_box, kv_rows) ||
        !make_tile_map(&kv.v, v, d, Nk, BHkv, bf16, kv_box, kv_rows))
      return FA_ERR_CUDA;
    kv.kt = kv.k;
    kv.vt = kv.v;
  }

  fa::FwdParams prm;
  prm.o = o;
  prm.lse = lse;
  prm.BH = static_cast<int>(BH);
  prm.n_qb = 0;   // set per configuration at launch
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.group = Hq / Hkv;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.causal_offset = Nk - Nq;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.timeout_ns = g_timeout_ns.load(std::memory_order_relaxed);
  prm.skip_q_load = g_skip_q_load.load(std::memory_order_relaxed);
  prm.o_scale = 1.f;
  prm.pk = pg ? pg->device(Hkv) : fa::PagedKV{};
  prm.last_page = pg ? (Nk - 1) / pg->page_size : 0;
  prm.q_lens = q_lens;
  prm.kv_lens = kv_lens;
  const bool kvm = kv_major_order(B, Hq, Hkv, Nk, d, 2);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool paged = pg != nullptr;
  if (d == 64)
    return bf16 ? dispatch_varlen<64, true>(varlen, causal, paged, dev, mq, kv, prm, st, kvm)
                : dispatch_varlen<64, false>(varlen, causal, paged, dev, mq, kv, prm, st, kvm);
  return bf16 ? dispatch_varlen<128, true>(varlen, causal, paged, dev, mq, kv, prm, st, kvm)
              : dispatch_varlen<128, false>(varlen, causal, paged, dev, mq, kv, prm, st, kvm);
}
}  // namespace

extern "C" {

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                 int Hkv, int Nq, int Nk, int d, int causal, float scale, fa_dtype dtype,
                 void* stream) {
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, Nk, d, causal, scale, dtype, nullptr, stream);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq,
                 int Nk, int d, int causal, float scale, fa_dtype dtype, void* workspace,
                 size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (Nq <= 0 || Nk <= 0 || (causal != 0 && causal != 1)) return FA_ERR_INVALID_ARG;
  fa_status s = common_checks(B, Hq, Hkv, d, scale, dtype);
  if (s != FA_OK) return s;
  const long long BH = static_cast<long long>(B) * Hq;
  const long long BHkv = static_cast<long long>(B) * Hkv;
  const int n_q = (Nq + fa::kBwdTile - 1) / fa::kBwdTile;
  const int n_k = (Nk + fa::kBwdTile - 1) / fa::kBwdTile;
  if (BH >= 65536 || BHkv >= 65536 || BH * n_q * fa::kBwdTile * 32 >= (1LL << 31))
    return FA_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, o, dout, static_cast<const void*>(dq), static_cast<const void*>(dk),
                          static_cast<const void*>(dv)})
    if (!aligned16(ptr)) return FA_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return FA_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < fa_bwd_workspace_bytes(B, Hq, Nq)) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_ALIGNMENT;
  int dev = 0;
  s = check_device(&dev);
  if (s != FA_OK) return s;

  const bool bf16 = dtype == FA_BF16;
  const int nq_pad = n_q * fa::kBwdTile;
  float* lse2 = static_cast<float*>(workspace);
  float* dsum = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                         fa_bwd_workspace_bytes(B, Hq, Nq) / 2);
  BwdMaps mp;
  const int tn = (d == 64) ? fa::BwdCfg<64>::TN : fa::BwdCfg<128>::TN;
  if (!make_tile_map(&mp.q, q, d, Nq, BH, bf16, fa::kBwdTile) ||
      !make_tile_map(&mp.dout, dout, d, Nq, BH, bf16, fa::kBwdTile) ||
      !make_tile_map(&mp.k, k, d, Nk, BHkv, bf16, fa::kBwdTile) ||
      !make_tile_map(&mp.v, v, d, Nk, BHkv, bf16, fa::kBwdTile) ||
      !make_tile_map(&mp.q_s, q, d, Nq, BH, bf16, tn) ||
      !make_tile_map(&mp.dout_s, dout, d, Nq, BH, bf16, tn) ||
      !make_tile_map(&mp.k_s, k, d, Nk, BHkv, bf16, tn) ||
      !make_tile_map(&mp.v_s, v, d, Nk, BHkv, bf16, tn))
    return FA_ERR_CUDA;
  fa::BwdParams prm;
  prm.lse2 = lse2;
  prm.dsum = dsum;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.group = Hq / Hkv;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.Nq_pad = nq_pad;
  prm.causal_offset = Nk - Nq;
  prm.scale = scale;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.timeout_ns = g_timeout_ns.load(std::memory_order_relaxed);
  prm.skip_resident_load = g_skip_q_load.load(std::memory_order_relaxed);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 64)
    return bf16 ? launch_bwd<64, true>(dev, mp, o, dout, lse, dq, dk, dv, prm, BH, BHkv, n_q, n_k, causal, st)
                : launch_bwd<64, false>(dev, mp, o, dout, lse, dq, dk, dv, prm, BH, BHkv, n_q, n_k, causal, st);
  return bf16 ? launch_bwd<128, true>(dev, mp, o, dout, lse, dq, dk, dv, prm, BH, BHkv, n_q, n_k, causal, st)
              : launch_bwd<128, false>(dev, mp, o, dout, lse, dq, dk, dv, prm, BH, BHkv, n_q, n_k, causal, st);
}

fa_status fa_fwd_kvcache(const void* q, const void* kcache, const void* vcache,
                         const int* q_lens, const int* kv_lens, void* o, float* lse, int B,
                         int Hq, int Hkv, int Nq, int Nk, int cache_len, int d, int causal,
                         float scale, fa_dtype dtype, void* stream) {
  if (cache_len < Nk || cache_len <= 0) return FA_ERR_INVALID_ARG;
  return fwd_impl(q, kcache, vcache, o, lse, B, Hq, Hkv, Nq, Nk, cache_len, d, causal, scale,
                  dtype, nullptr, stream, q_lens, kv_lens);
}

fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                     float q_descale, float k_descale, float v_descale, void* stream) {
  if (!q || !k || !v || !o) return FA_ERR_INVALID_ARG;
  if (Nq <= 0 || Nk <= 0 || (causal != 0 && causal != 1)) return FA_ERR_INVALID_ARG;
  fa_status s = common_checks(B, Hq, Hkv, d, scale, FA_BF16);
  if (s != FA_OK) return s;
  for (float x : {q_descale, k_descale, v_descale})
    if (!std::isfinite(x) || !(x > 0.f)) return FA_ERR_INVALID_ARG;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(B) * Hq;
  const long long BHkv = static_cast<long long>(B) * Hkv;
  if (BH >= (1LL << 31)) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FA_ERR_ALIGNMENT;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FA_ERR_ALIGNMENT;
  int dev = 0;
  s = check_device(&dev);
  if (s != FA_OK) return s;

  using C8 = fa::FwdCfg<128, true>;
  CUtensorMap mq;
  KVMaps kv;
  if (!make_tile_map8(&mq, q, d, Nq, BH, fa::kBM) ||
      !make_tile_map8(&kv.k, k, d, Nk, BHkv, C8::BN) ||
      !make_tile_map8(&kv.v, v, d, Nk, BHkv, C8::BN))
    return FA_ERR_CUDA;
  kv.kt = kv.k;
  kv.vt = kv.v;
  fa::FwdParams prm;
  prm.o = o;
  prm.lse = lse;
  prm.BH = static_cast<int>(BH);
  prm.n_qb = 0;   // set per configuration at launch
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.group = Hq / Hkv;
  prm.Nq = Nq;
  prm.Nk = Nk;
  prm.causal_offset = Nk - Nq;
  // Scores of the stored values carry the Q and K descales; O carries V's.
  prm.scale_log2 = scale * q_descale * k_descale * 1.4426950408889634f;
  prm.timeout_ns = g_timeout_ns.load(std::memory_order_relaxed);
  prm.skip_q_load = g_skip_q_load.load(std::memory_order_relaxed);
  prm.pk = fa::PagedKV{};
  prm.last_page = 0;
  prm.o_scale = v_descale;
  prm.q_lens = nullptr;
  prm.kv_lens = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return causal ? launch_fwd<128, true, true, false, true>(dev, mq, kv, prm, st)
                : launch_fwd<128, true, false, false, true>(dev, mq, kv, prm, st);
}

fa_status fa_fwd_paged(const void* q, const void* kpool, const void* vpool, const int* block_table,
                       const int* q_lens, const int* kv_lens, void* o, float* lse, int B, int Hq,
                       int Hkv, int Nq, int Nk, int num_pages, int page_size,
                       int max_pages_per_seq, int d, int causal, float scale, fa_dtype dtype,
                       void* stream) {
  const PagedArgs pg{block_table, num_pages, page_size, max_pages_per_seq};
  return fwd_impl(q, kpool, vpool, o, lse, B, Hq, Hkv, Nq, Nk, 0, d, causal, scale, dtype, &pg,
                  stream, q_lens, kv_lens);
}

size_t fa_bwd_workspace_bytes(int B, int Hq, int Nq) {
  if (B <= 0 || Hq <= 0 || Nq <= 0) return 0;
  const size_t nq_pad = static_cast<size_t>((Nq + fa::kBwdTile - 1) / fa::kBwdTile) * fa::kBwdTile;
  return 2 * align_up(static_cast<size_t>(B) * Hq * nq_pad * sizeof(float), 256);
}

size_t fa_decode_workspace_bytes(int B, int Hq, int max_kv_len, int d) {
  DecodeLayout L;
  if (!decode_layout(B, Hq, max_kv_len, d, &L)) return 0;
  return L.total;
}

}  // extern "C"

namespace {
// fa_decode and fa_decode_paged; pg != nullptr reads the cache from a page pool, whose
// sequences hold at most max_kv_len = max_pages * page_size tokens.
fa_status decode_impl(const void* q, const void* kcache, const void* vcache, const int* kv_lens,
                      void* o, float* lse, int B, int Hq, int Hkv, int max_kv_len, int d,
                      float scale, fa_dtype dtype, void* workspace, size_t workspace_bytes,
                      const PagedArgs* pg, void* stream) {
  if (!q || !kcache || !vcache || !kv_lens || !o) return FA_ERR_INVALID_ARG;
  if (max_kv_len <= 0) return FA_ERR_INVALID_ARG;
  fa_status s = common_checks(B, Hq, Hkv, d, scale, dtype);
  if (s != FA_OK) return s;
  if (pg) {
    s = check_paged(*pg, Hkv);
    if (s != FA_OK) return s;
  }
  if (B > 65535 || static_cast<long long>(B) * Hq >= (1LL << 31)) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(o))
    return FA_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(kv_lens) & 3u) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FA_ERR_ALIGNMENT;
  DecodeLayout L;
  decode_layout(B, Hq, max_kv_len, d, &L);
  if (!workspace || workspace_bytes < L.total) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_ALIGNMENT;
  const int G = Hq / Hkv;
  if (static_cast<long long>(Hkv) * ((G + 7) / 8) > 65535) return FA_ERR_INVALID_ARG;
  int dev = 0;
  s = check_device(&dev);
  if (s != FA_OK) return s;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool bf16 = dtype == FA_BF16;
  fa::CombineParams cp;
  cp.ws_o = reinterpret_cast<float*>(ws);
  cp.ws_lse = reinterpret_cast<float*>(ws + L.lse_off);
  cp.kv_lens = kv_lens;
  cp.o = static_cast<uint16_t*>(o);
  cp.lse = lse;
  cp.Hq = Hq;
  cp.max_len = max_kv_len;
  cp.split_tokens = L.split_tokens;
  cp.n_split = L.n_split;
  if (use_tc_decode(d)) {
    if (pg)
      return bf16 ? launch_decode_tc<true, true>(dev, q, kcache, vcache, kv_lens, ws, L, B, Hq, Hkv,
                                                 max_kv_len, scale, cp, pg, st)
                  : launch_decode_tc<false, true>(dev, q, kcache, vcache, kv_lens, ws, L, B, Hq,
                                                  Hkv, max_kv_len, scale, cp, pg, st);
    return bf16 ? launch_decode_tc<true, false>(dev, q, kcache, vcache, kv_lens, ws, L, B, Hq, Hkv,
                                                max_kv_len, scale, cp, nullptr, st)
                : launch_decode_tc<false, false>(dev, q, kcache, vcache, kv_lens, ws, L, B, Hq, Hkv,
                                                 max_kv_len, scale, cp, nullptr, st);
  }
  fa::DecodeParams dp;
  dp.q = static_cast<const uint16_t*>(q);
  dp.kc = static_cast<const uint16_t*>(kcache);
  dp.vc = static_cast<const uint16_t*>(vcache);
  dp.kv_lens = kv_lens;
  dp.ws_o = reinterpret_cast<float*>(ws);
  dp.ws_lse = reinterpret_cast<float*>(ws + L.lse_off);
  dp.Hq = Hq;
  dp.Hkv = Hkv;
  dp.G = G;
  dp.max_len = max_kv_len;
  dp.split_tokens = L.split_tokens;
  dp.n_split = L.n_split;
  dp.scale_log2 = scale * 1.4426950408889634f;
  dp.timeout_ns = g_timeout_ns.load(std::memory_order_relaxed);
  dp.skip_kv_load = g_skip_q_load.load(std::memory_order_relaxed);
  dp.pk = pg ? pg->device(Hkv) : fa::PagedKV{};
#define FA_DEC_CASE(D_, BF_)                                                         \
  return pg ? launch_decode_g<D_, BF_, true>(dev, dp, cp, B, Hkv, G, st)             \
            : launch_decode_g<D_, BF_, false>(dev, dp, cp, B, Hkv, G, st)
  if (d == 64) {
    if (bf16) FA_DEC_CASE(64, true);
    FA_DEC_CASE(64, false);
  }
  if (bf16) FA_DEC_CASE(128, true);
  FA_DEC_CASE(128, false);
#undef FA_DEC_CASE
}
}  // namespace

extern "C" {

fa_status fa_decode(const void* q, const void* kcache, const void* vcache, const int* kv_lens,
                    void* o, float* lse, int B, int Hq, int Hkv, int max_kv_len, int d,
                    float scale, fa_dtype dtype, void* workspace, size_t workspace_bytes,
                    void* stream) {
  return decode_impl(q, kcache, vcache, kv_lens, o, lse, B, Hq, Hkv, max_kv_len, d, scale, dtype,
                     workspace, workspace_bytes, nullptr, stream);
}

fa_status fa_decode_paged(const void* q, const void* kpool, const void* vpool,
                          const int* block_table, const int* kv_lens, void* o, float* lse, int B,
                          int Hq, int Hkv, int num_pages, int page_size, int max_pages_per_seq,
                          int d, float scale, fa_dtype dtype, void* workspace,
                          size_t workspace_bytes, void* stream) {
  const PagedArgs pg{block_table, num_pages, page_size, max_pages_per_seq};
  const long long max_len = static_cast<long long>(max_pages_per_seq) * page_size;
  if (max_pages_per_seq <= 0 || page_size <= 0 || max_len >= (1LL << 31)) return FA_ERR_INVALID_ARG;
  return decode_impl(q, kpool, vpool, kv_lens, o, lse, B, Hq, Hkv, static_cast<int>(max_len), d,
                     scale, dtype, workspace, workspace_bytes, &pg, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Allocation-free decode: split-KV scratch in a fixed device array of this file. In host
// code `g_decode_noalloc_scratch` names a host-side stand-in, not device memory, so its
// device address is looked up once per device with cudaGetSymbolAddress (with that device
// current) and only that address is handed to the kernels.
// ---------------------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_decode_noalloc_scratch[FA_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {
void* g_noalloc_scratch_ptr[kMaxDevices];

fa_status noalloc_scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_noalloc_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_noalloc_scratch) != cudaSuccess || p == nullptr)
      return FA_ERR_CUDA;
    g_noalloc_scratch_ptr[dev] = p;
  }
  *out = g_noalloc_scratch_ptr[dev];
  return FA_OK;
}
}  // namespace

extern "C" {

fa_status fa_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                            const int* kv_lens, void* o, float* lse, int B, int Hq, int Hkv,
                            int max_kv_len, int d, float scale, fa_dtype dtype, void* stream) {
  const size_t need = fa_decode_workspace_bytes(B, Hq, max_kv_len, d);
  if (need == 0)   // invalid sizes: let fa_decode report them without touching CUDA
    return fa_decode(q, kcache, vcache, kv_lens, o, lse, B, Hq, Hkv, max_kv_len, d, scale,
                     dtype, nullptr, 0, stream);
  if (need > FA_DECODE_NOALLOC_SCRATCH_BYTES) return FA_ERR_WORKSPACE;
  int dev = 0;
  fa_status s = check_device(&dev);
  if (s != FA_OK) return s;
  void* scratch = nullptr;
  s = noalloc_scratch_address(dev, &scratch);
  if (s != FA_OK) return s;
  return fa_decode(q, kcache, vcache, kv_lens, o, lse, B, Hq, Hkv, max_kv_len, d, scale, dtype,
                   scratch, FA_DECODE_NOALLOC_SCRATCH_BYTES, stream);
}

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_ALIGNMENT: return "FA_ERR_ALIGNMENT";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
  }
  return "FA_ERR_UNKNOWN";
}

fa_status fa_device_status(int clear) {
  if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_fa_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (clear && v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(fa::g_fa_status, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  }
  return v == 0 ? FA_OK : static_cast<fa_status>(v);
}

void fa_set_wait_timeout_ns(uint64_t ns) {
  g_timeout_ns.store(ns ? ns : kDefaultTimeoutNs, std::memory_order_relaxed);
}

void fa_debug_skip_q_load(int enable) { g_skip_q_load.store(enable ? 1 : 0, std::memory_order_relaxed); }

const char* fa_build_info(void) { return "libfa_b200 0.1 sm_100a (tcgen05/TMA prefill, split-KV decode)"; }

}  // extern "C"
