/*
 * fa.h — C ABI of the B200 exact-attention library (libfa_b200.so).
 *
 * The library computes exact scaled-dot-product attention
 *     O = softmax(scale * Q K^T) V,    LSE_i = log(sum_j exp(scale * q_i . k_j))
 * tile by tile with an online softmax, so the score matrix never reaches device memory.
 * Sources: page "Kotaemon FlashAttention" (attention formula; algorithm bullets: Q row
 * blocks, K_j/V_j blocks streamed through on-chip memory, running max and normaliser,
 * result identical to the untiled formula); page "Flash Attention ... IO-aware exact"
 * (fr), tiling pseudo-code (returns O and the per-row statistic L) and PyTorch section
 * (is_causal); page "Flash Attention" (zh), online-softmax bullet and the O(N) memory
 * claim.
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller. The library allocates
 *    no device memory and keeps no per-call state; work is enqueued asynchronously on
 *    `stream` (a cudaStream_t passed as void*; NULL = the legacy default stream).
 *  - Tensors are contiguous, row-major, 16-bit (fp16 or bf16 per `dtype`); LSE is fp32.
 *  - `scale` multiplies Q.K^T before the softmax (every workload passes 1/sqrt(d)).
 *  - Grouped-query attention: query head h reads KV head h / (Hq / Hkv).
 *  - Causal masking is bottom-right aligned: key j is visible to query i iff
 *    j <= i + (Nk - Nq) (page "Flash Attention ... IO-aware exact" (fr), manual chunking
 *    example). A row with no visible key gets O = 0 and LSE = -inf.
 *  - Errors are returned as fa_status; nothing is thrown across the ABI. Host-side
 *    argument checks run before any CUDA call, so FA_ERR_INVALID_ARG /
 *    FA_ERR_UNSUPPORTED / FA_ERR_ALIGNMENT leave the stream untouched.
 *  - Device-side waits are bounded. A wait that runs out sets a device status word that
 *    fa_device_status() reads (FA_ERR_DEVICE_TIMEOUT); the kernel then returns early.
 */
#ifndef FA_B200_FA_H_
#define FA_B200_FA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { FA_FP16 = 0, FA_BF16 = 1 } fa_dtype;

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,     /* null pointer, non-positive size, Hq % Hkv != 0, bad scale */
  FA_ERR_UNSUPPORTED = 2,     /* d not in {64,128}, unknown dtype, device is not sm_100 */
  FA_ERR_ALIGNMENT = 3,       /* a tensor pointer is not 16-byte aligned */
  FA_ERR_CUDA = 4,            /* a CUDA runtime/driver call or a launch failed */
  FA_ERR_DEVICE_TIMEOUT = 5,  /* a bounded device-side wait ran out (see fa_device_status) */
  FA_ERR_WORKSPACE = 6        /* decode workspace missing or smaller than required */
} fa_status;

/*
 * fa_fwd — prefill / forward attention, O and per-row LSE.
 *
 * Defined by: page "Kotaemon FlashAttention", attention formula and algorithm bullets;
 * page "Flash Attention ... IO-aware exact" (fr), tiling pseudo-code (outputs O and L)
 * and the PyTorch section (causal flag).
 *
 *   q    [B, Hq,  Nq, d]  fp16/bf16
 *   k, v [B, Hkv, Nk, d]  fp16/bf16
 *   o    [B, Hq,  Nq, d]  same dtype as q (written, rounded to nearest even)
 *   lse  [B, Hq,  Nq]     fp32, natural log of the row normaliser of the scaled scores;
 *                         may be NULL (then not written)
 *   causal  0 or 1 (bottom-right aligned when Nq != Nk)
 *   scale   finite, > 0
 *
 * Requirements: B, Hq, Hkv, Nq, Nk >= 1; Hq % Hkv == 0; d in {64, 128}; q, k, v, o
 * 16-byte aligned, lse 4-byte aligned; sm_100 device; B*Hq and B*Hkv < 2^31.
 * Returns FA_OK once the kernel is enqueued on `stream`.
 */
FA_API fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int Hq, int Hkv, int Nq, int Nk, int d,
                 int causal, float scale, fa_dtype dtype, void* stream);

/*
 * fa_fwd_kvcache — fa_fwd for a chunk of queries against the first Nk rows of a KV cache
 * whose capacity per head is cache_len >= Nk (chunked prefill: the newest Nq tokens
 * attend to the whole prefix, causally aligned to its end), optionally with lengths that
 * differ per sequence.
 *
 * Defined by: page "Flash Attention ... IO-aware exact" (fr), "Erreurs courantes et
 * solutions" (the manual chunking example: a chunk of queries attends to every key up to
 * the chunk's end) and "Optimisation avancée : KV Cache et persistent attention" (keys and
 * values cached per session, each session with its own length); the result for sequence
 * b is fa_fwd's with q = its first nq_b query rows and k, v = its cache's first nk_b rows.
 *
 *   q, o, lse           as fa_fwd, [B, Hq, Nq, d] / [B, Hq, Nq]: Nq is the row capacity
 *   kcache, vcache      [B, Hkv, cache_len, d]
 *   q_lens              NULL (every sequence has nq_b = Nq query rows) or [B] int32 in
 *                       device memory, 4-byte aligned: nq_b = q_lens[b] clamped to [0, Nq]
 *   kv_lens             NULL (nk_b = Nk keys each) or [B] int32 in device memory, 4-byte
 *                       aligned: nk_b = kv_lens[b] clamped to [0, Nk]
 *   causal              0 or 1; query row i of sequence b sees key j iff j <= i + nk_b - nq_b
 *                       (the chunk is the last nq_b of the sequence's nk_b tokens)
 *
 * Rows [0, nk_b) of each head of sequence b are used; rows [nk_b, cache_len) and query
 * rows [nq_b, Nq) may hold anything (NaN included) and never affect a written value.
 * Output rows [nq_b, Nq) of o and lse are not written. A row with no visible key
 * (nk_b = 0, or nq_b > nk_b causal) gets O = 0 and LSE = -inf.
 *
 * Requirements: those of fa_fwd, plus 1 <= Nk <= cache_len. Same errors and ownership.
 */
FA_API fa_status fa_fwd_kvcache(const void* q, const void* kcache, const void* vcache,
                         const int* q_lens, const int* kv_lens, void* o, float* lse, int B,
                         int Hq, int Hkv, int Nq, int Nk, int cache_len, int d, int causal,
                         float scale, fa_dtype dtype, void* stream);

/*
 * Paged KV cache (fa_fwd_paged, fa_decode_paged).
 *
 * Defined by: page "Flash Attention ... IO-aware exact" (fr), "Optimisation avancée : KV
 * Cache et persistent attention": keys and values are cached per session, extended as
 * tokens arrive and released per session. Here the cache is one pool of fixed-size pages
 * shared by all sequences: a sequence owns a list of pages (its block-table row), so a
 * sequence is grown or released without moving any other sequence's data. The result is
 * the one fa_fwd / fa_decode give on the sequence's tokens gathered in order.
 *
 *   kpool, vpool  [num_pages, Hkv, page_size, d] fp16/bf16, 16-byte aligned: page p of KV
 *                 head h holds page_size consecutive tokens of one sequence
 *   block_table   [B, max_pages_per_seq] int32, device memory, 4-byte aligned: token t of
 *                 sequence b sits in page block_table[b][t / page_size], row
 *                 t % page_size. Only the entries that cover the sequence's tokens are
 *                 read (the others may hold anything, e.g. -1).
 *   page_size     a power of two >= 16 (FA_ERR_UNSUPPORTED otherwise)
 *   num_pages     pool size; num_pages * Hkv < 2^31 - 1, max_pages_per_seq * page_size < 2^31
 *
 * Pool rows that hold no token of the sequence (a page's rows past the sequence's end,
 * pages of other sequences, unused pages) never affect the result, whatever they hold.
 * A table entry that is read and lies outside [0, num_pages) is never dereferenced: the
 * kernel records FA_ERR_INVALID_ARG in the device status word (fa_device_status) and the
 * result of that sequence is unspecified.
 */

/*
 * fa_fwd_paged — fa_fwd_kvcache with the keys and values in a paged pool: each of the B
 * sequences attends to its first nk_b tokens, found through its block-table row.
 *
 * Defined by: the per-session cache of page "Flash Attention ... IO-aware exact" (fr),
 * "Optimisation avancée : KV Cache et persistent attention", laid out as the paged pool
 * above; the attention itself is fa_fwd_kvcache's.
 *
 *   q, o, lse         as fa_fwd, [B, Hq, Nq, d] / [B, Hq, Nq]: Nq is the row capacity
 *   q_lens, kv_lens   as fa_fwd_kvcache (NULL: Nq rows and Nk keys for every sequence;
 *                     otherwise per-sequence values clamped to [0, Nq] and [0, Nk])
 *   causal            0 or 1, bottom-right aligned per sequence (the chunk is the last
 *                     nq_b of the sequence's nk_b tokens)
 *
 * Only the table entries that cover tokens [0, nk_b) of sequence b are read; output rows
 * [nq_b, Nq) are not written.
 *
 * Requirements: those of fa_fwd and of the paged cache above, plus
 * Nk <= max_pages_per_seq * page_size.
 */
FA_API fa_status fa_fwd_paged(const void* q, const void* kpool, const void* vpool,
                       const int* block_table, const int* q_lens, const int* kv_lens, void* o,
                       float* lse, int B, int Hq, int Hkv, int Nq, int Nk, int num_pages,
                       int page_size, int max_pages_per_seq, int d, int causal, float scale,
                       fa_dtype dtype, void* stream);

/*
 * fa_fwd_fp8 — fa_fwd with 8-bit (E4M3) Q, K and V and per-tensor descale factors: the
 * attention of the real-valued tensors q_descale*Q, k_descale*K, v_descale*V.
 *
 * Not on the pages as a kernel: the pages discuss lowering precision by quantisation
 * (page "Empreinte mémoire et calcul des couches Transformer", quantisation bullet: 16 to
 * 8 bits halves the memory; page "Kotaemon FlashAttention", engineering notes on
 * quantisation); this applies it to the attention inputs. The method is fa_fwd's, with both products on the 8-bit tensor-core
 * path and P rounded to E4M3 before P.V (its row sum is taken before rounding).
 *
 *   q    [B, Hq,  Nq, d]  E4M3 bytes (OCP FP8 E4M3: bias 7, no infinities, max 448)
 *   k, v [B, Hkv, Nk, d]  E4M3 bytes
 *   o    [B, Hq,  Nq, d]  bf16 (written)
 *   lse  [B, Hq,  Nq]     fp32, natural log, of the descaled scores; may be NULL
 *   scale, causal         as fa_fwd; q_descale, k_descale, v_descale finite and > 0
 *
 * Requirements: those of fa_fwd, with d = 128 only (FA_ERR_UNSUPPORTED otherwise).
 */
FA_API fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                     float q_descale, float k_descale, float v_descale, void* stream);

/*
 * fa_bwd_workspace_bytes — bytes of scratch that fa_bwd needs for these sizes.
 *
 * Not an operation of the pages: a size query for fa_bwd's per-row scratch (the LSE in
 * log2 units and D_i = sum_d dO_id O_id, one fp32 each per padded query row). Pure host
 * arithmetic; returns 0 for invalid sizes.
 */
FA_API size_t fa_bwd_workspace_bytes(int B, int Hq, int Nq);

/*
 * fa_bwd — gradients of fa_fwd: dQ, dK, dV for an upstream gradient dO, recomputing the
 * scores tile by tile from Q, K and the forward's LSE (no N x N matrix is stored).
 *
 * Defined by: the derivative of fa_fwd's result (page "Kotaemon FlashAttention",
 * attention formula); the recomputation from the saved per-row statistic follows page
 * "Flash Attention" (zh), "IO 感知的算法设计" (tiling plus recomputation) and the L output of
 * page "Flash Attention ... IO-aware exact" (fr), tiling pseudo-code.
 *
 *   q, o, dout    [B, Hq,  Nq, d]  fp16/bf16; o and lse are fa_fwd's outputs for q, k, v
 *   k, v          [B, Hkv, Nk, d]
 *   lse           [B, Hq,  Nq]     fp32 (natural log, as fa_fwd writes it)
 *   dq            [B, Hq,  Nq, d]  written
 *   dk, dv        [B, Hkv, Nk, d]  written; a KV head sums the gradients of all query heads
 *                                  that read it
 *   causal, scale as passed to fa_fwd
 *   workspace     device scratch of at least fa_bwd_workspace_bytes(B, Hq, Nq) bytes,
 *                 16-byte aligned, owned by the caller, no initialisation needed
 *
 * Requirements: those of fa_fwd, plus every listed pointer non-NULL (lse included) and
 * 16-byte aligned (lse 4-byte), workspace_bytes large enough (FA_ERR_WORKSPACE).
 */
FA_API fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o,
                 const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                 int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                 fa_dtype dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_decode_workspace_bytes — bytes of scratch that fa_decode needs for these sizes.
 *
 * Not an operation of the pages: a size query (pure host arithmetic) for fa_decode's
 * split-KV scratch.
 *
 * The split-KV decode writes, per (sequence, query head, KV split), a partial output
 * row (d fp32) and its logsumexp (fp32), then merges them. max_kv_len is the cache
 * capacity (its row stride), which bounds the number of splits. Returns 0 for invalid
 * sizes.
 */
FA_API size_t fa_decode_workspace_bytes(int B, int Hq, int max_kv_len, int d);

/*
 * fa_decode — single-token decode over a grouped-query KV cache (split-KV).
 *
 * Defined by: the attention formula (page "Kotaemon FlashAttention") with one query row
 * per sequence, non-causal over the cache's valid rows; KV-cache use and its per-token
 * size with 8 KV heads of dimension 128 (page "Empreinte mémoire et calcul des couches
 * Transformer", KV-cache paragraph). The merge of the per-split partial results uses the
 * same rescaling identity as the online softmax (page "Kotaemon FlashAttention", running
 * max and normaliser).
 *
 *   q         [B, Hq, d]               fp16/bf16
 *   kcache,
 *   vcache    [B, Hkv, max_kv_len, d]  fp16/bf16; rows >= kv_lens[b] never affect the
 *                                      result, whatever they hold (the d = 128 kernel may
 *                                      fetch them as part of a 128-row tile, then masks them)
 *   kv_lens   [B] int32, device memory; values are clamped to [0, max_kv_len]
 *   o         [B, Hq, d]               same dtype as q
 *   lse       [B, Hq] fp32, may be NULL
 *   workspace device scratch of at least fa_decode_workspace_bytes(B, Hq, max_kv_len, d)
 *             bytes, 16-byte aligned, owned by the caller; contents need no initialisation
 *             and are meaningless after the call. Two decodes that may run at the same
 *             time need separate workspaces.
 *
 * A sequence with kv_lens[b] == 0 gets O = 0 and LSE = -inf.
 * Requirements: as fa_fwd, plus workspace_bytes >= the required size
 * (FA_ERR_WORKSPACE otherwise).
 */
FA_API fa_status fa_decode(const void* q, const void* kcache, const void* vcache,
                    const int* kv_lens, void* o, float* lse,
                    int B, int Hq, int Hkv, int max_kv_len, int d,
                    float scale, fa_dtype dtype, void* workspace, size_t workspace_bytes,
                    void* stream);

/*
 * fa_decode_paged — fa_decode over a paged pool (see "Paged KV cache" above): sequence b
 * attends to its first kv_lens[b] tokens, found through its block-table row.
 *
 * Defined by: the per-session cache of page "Flash Attention ... IO-aware exact" (fr),
 * "Optimisation avancée : KV Cache et persistent attention", laid out as the paged pool
 * above; the decode itself is fa_decode's.
 *
 *   q, o, lse, kv_lens   as fa_decode; kv_lens are clamped to
 *                        [0, max_pages_per_seq * page_size]
 *   workspace            at least fa_decode_workspace_bytes(B, Hq,
 *                        max_pages_per_seq * page_size, d) bytes, as for fa_decode
 *
 * Requirements: those of fa_decode and of the paged cache.
 */
FA_API fa_status fa_decode_paged(const void* q, const void* kpool, const void* vpool,
                          const int* block_table, const int* kv_lens, void* o, float* lse,
                          int B, int Hq, int Hkv, int num_pages, int page_size,
                          int max_pages_per_seq, int d, float scale, fa_dtype dtype,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_decode_noalloc — fa_decode for callers that cannot allocate device memory.
 *
 * Not from the pages (they have no counterpart): a convenience form of fa_decode whose
 * split-KV scratch is a fixed array compiled into this library instead of a
 * caller-provided workspace. Some callers cannot call cudaMalloc at the point where they
 * decode: an inference server that has handed almost all device memory to its own pool
 * and KV cache up front (a fresh cudaMalloc would fail or fragment that pool), a plugin
 * that is given tensors but no allocator, or a latency-critical decode loop that must not
 * pay cudaMalloc/cudaFree's cost and implicit device-wide synchronisation. This entry
 * point needs nothing beyond the inputs and outputs, and it calls no allocating routine.
 *
 * Arguments, layouts, ownership and results are those of fa_decode, minus the workspace.
 * Limits and behaviour:
 *  - the scratch is FA_DECODE_NOALLOC_SCRATCH_BYTES (32 MiB) of device memory per GPU,
 *    reserved when the library's device code is loaded on that GPU and held until the
 *    process exits; calls whose fa_decode_workspace_bytes(B, Hq, max_kv_len, d) exceeds
 *    it return FA_ERR_WORKSPACE without launching anything;
 *  - the first call on each device looks up the scratch's device address (with that
 *    device current) and keeps it for the life of the process; make that first call
 *    before any stream capture. A cudaDeviceReset (or any other teardown of the device's
 *    primary context) unloads the array, so the kept address is stale afterwards: do not
 *    call fa_decode_noalloc on a device after resetting it in the same process;
 *  - every call on a device shares the one scratch array, which keeps the previous call's
 *    contents (the kernels overwrite every slot they later read, so nothing needs
 *    clearing); two calls whose kernels may overlap on the GPU (different streams, or
 *    different host threads) race on it and give wrong results. Serialise them, or use
 *    fa_decode with separate workspaces.
 */
#define FA_DECODE_NOALLOC_SCRATCH_BYTES (32u << 20)
FA_API fa_status fa_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                                   const int* kv_lens, void* o, float* lse,
                                   int B, int Hq, int Hkv, int max_kv_len, int d,
                                   float scale, fa_dtype dtype, void* stream);

/* fa_status_string — static, human-readable name of a status code (never NULL). Not an
 * operation of the pages: error reporting. */
FA_API const char* fa_status_string(fa_status s);

/*
 * Not operations of the pages: error reporting and the test hooks of the bounded waits.
 *
 * fa_device_status — synchronises the current device, then returns FA_OK or the first
 * error a kernel of this library recorded on it (FA_ERR_DEVICE_TIMEOUT, or
 * FA_ERR_INVALID_ARG for a paged-cache table entry outside the pool). If `clear` is
 * non-zero the recorded error is reset afterwards. FA_ERR_CUDA if the synchronisation
 * itself fails.
 */
FA_API fa_status fa_device_status(int clear);

/*
 * Not an operation of the pages.
 *
 * fa_set_wait_timeout_ns — upper bound, in nanoseconds, on every device-side barrier wait
 * of kernels launched afterwards from this process (default 2e9, i.e. 2 s). 0 restores
 * the default. Test hook for the timeout path; normal callers never need it.
 */
FA_API void fa_set_wait_timeout_ns(uint64_t ns);

/*
 * Not an operation of the pages.
 *
 * fa_debug_skip_q_load — test hook for the bounded-wait path: when non-zero, fa_fwd
 * kernels launched afterwards never issue the Q-tile load, the d = 128 decode kernels
 * never load their query rows, the other decode kernels never fill their K/V stages, and
 * fa_bwd kernels never issue the loads of their resident tiles (Q and dO, or K and V), so
 * the barriers that wait for them are never completed and every wait that depends on them
 * runs out. The kernel records
 * FA_ERR_DEVICE_TIMEOUT and returns; the outputs are then unspecified. 0 restores normal
 * operation.
 */
FA_API void fa_debug_skip_q_load(int enable);

/* fa_build_info — static string: library version and the GPU architecture it targets.
 * Not an operation of the pages. */
FA_API const char* fa_build_info(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_FA_H_ */
