/*
 * jetlong.h -- C ABI of libjetlong: dynamic bifocal RoPE attention on B200
 * (sm_100a).
 *
 * The method (Jet-Long, "Efficient long-context extension with dynamic bifocal
 * RoPE"):
 *   - G = max(1, ceil(L / w_pretrained)) is recomputed from the current length L
 *     (bittide paper summary §3.1, group-size equation; techwalker explainer §二).
 *   - f(x) = floor(x / G) maps remote positions back onto the pretrained grid
 *     (bittide summary §3.1, position-map equation).
 *   - A causal pair (query q, key k <= q) with q - k < w_local is LOCAL and uses
 *     standard RoPE at (q, k); every other pair is REMOTE and uses RoPE at
 *     (f(q), f(k)) (techwalker §二, bittide §3.2).  G = 1 is exactly plain
 *     causal RoPE attention.
 *   - Prefill merges the two windows with LogSumExp weights (techwalker §四,
 *     bittide §3.2); decode keeps the cache at original positions and applies the
 *     corrections dq = f(q) - q and dk = f(k) - k in registers (techwalker §三,
 *     bittide §3.3).
 *
 * Conventions for every entry point
 *   - RoPE pairs are rotate-half: (x_i, x_{i+D/2}) rotated by pos * theta_i with
 *     theta_i = rope_base^(-2i/D).  q and k passed to prefill are PRE-RoPE.
 *   - Softmax scale defaults to 1/sqrt(D).  lse is the natural log of
 *     sum_k exp(scale * score_k), in fp32.
 *   - All tensor pointers are caller-owned DEVICE memory, contiguous, 16-byte
 *     aligned.  The library writes only `out`, `lse` and the workspace (the
 *     decode and the three-call prefill take one; the fused prefill and the
 *     chunked prefill rotate their keys inside the kernels and need none).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  No entry point synchronises the host with the device except the
 *     first call that builds or grows a library-owned table (see below) and
 *     jl_check_device_status.
 *   - Arguments are validated before anything is launched.  A rejected call
 *     returns JL_ERR_INVALID_ARG or JL_ERR_UNSUPPORTED, launches nothing and
 *     leaves a message for jl_last_error().  No C++ exception crosses the ABI
 *     and no kernel traps.
 *   - Library-owned device memory: per device, a cos/sin table of the RoPE
 *     angles (fp64 sincos rounded to fp32, [positions][D/2] pairs) grown on
 *     demand, and a 4-byte device status word.  A table that is replaced by a
 *     larger one stays allocated (launches in flight may read it) until
 *     jl_finalize, which releases them all.  The first call that creates or
 *     grows the table allocates and synchronises its stream, so make it before
 *     any stream capture.  The library holds no per-call scratch: calls on
 *     different streams may overlap on the GPU.
 */
#ifndef JETLONG_H
#define JETLONG_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st *jl_stream_t;

typedef enum {
  JL_OK = 0,
  JL_ERR_INVALID_ARG = 1, /* a null/misaligned pointer, a bad size or shape */
  JL_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. head dim) */
  JL_ERR_CUDA = 3,        /* a CUDA runtime/driver call or launch failed */
  JL_ERR_TIMEOUT = 4      /* a kernel's bounded wait expired (device status) */
} jl_status;

typedef enum { JL_BF16 = 0, JL_F32 = 1 } jl_dtype;

enum {
  /* Run the same kernels with the bifocal rule switched off: every pair takes
   * standard RoPE at its original positions (plain causal RoPE attention).
   * This is the overhead baseline; with G = 1 the bifocal call takes exactly
   * this path. */
  JL_FLAG_NO_BIFOCAL = 1u << 0,
  /* jl_bifocal_decode_batched / jl_bifocal_decode_paged: `pos` is a DEVICE
   * array of B int32 positions (4-byte aligned), read on `stream` when the call
   * runs.  The plan is then made on the device (no host data, no host
   * synchronisation), so the call can be captured in a CUDA graph and replayed
   * with new positions; positions are checked on the device (out of range:
   * the status word is raised, see jl_check_device_status, and the sequence is
   * decoded as if at position 0).  The cos/sin table and the tensor maps then
   * cover the whole cache (cache_capacity, or max_pages_per_seq * page_size),
   * so make one call before capturing (it may build or grow the table). */
  JL_FLAG_DEVICE_POS = 1u << 1,
  /* jl_bifocal_prefill_ex, bf16: rotate the keys once per call instead of in
   * the attention kernel.  A first pass writes both rotated copies of every
   * key, R(l) k and R(floor(l / G)) k, into the caller's workspace (at least
   * jl_bifocal_prefill_rotated_keys_bytes() bytes, 256-byte aligned,
   * required), and the attention kernel then streams the copy of each pass's
   * class instead of rotating each K tile in shared memory.  Faster at long
   * lengths, at the cost of that memory (512 MiB for B = 1, L = 131072,
   * Hkv = 8, D = 128); the result is the same computation, rounded the same
   * way up to the order of the fp32 operations that form each rotated key.
   * Ignored for JL_F32 (that kernel always rotates in place). */
  JL_FLAG_ROTATE_KEYS_ONCE = 1u << 2,
  /* TEST ONLY (jl_bifocal_decode): exercises the kernels' bounded waits.  The
   * decode kernel's TMA producer withholds its first arrival, so the consumer
   * warps' wait on the first K/V block expires after about one second; they
   * raise the device status word and every warp of the kernel returns without
   * a copy in flight.  The call itself returns JL_OK (the launch succeeded),
   * out and lse are invalid, and the next jl_check_device_status returns
   * JL_ERR_TIMEOUT and clears the word, after which the library works as
   * before.  Accepted only where the tensor-core decode kernel runs (D = 128,
   * Hkv <= 8, Hq / Hkv <= 8), JL_ERR_UNSUPPORTED otherwise; every other
   * entry point rejects it as an unknown flag. */
  JL_FLAG_DEBUG_SKIP_ARRIVE = 1u << 31
};

/* G = max(1, ceil(L / w_pretrained)) (bittide summary §3.1).  Returns -1 when
 * L < 1 or w_pretrained < 1.  Host-only. */
long long jl_group_size(long long L, long long w_pretrained);

/*
 * Bifocal prefill, bf16 (techwalker §四; bittide §3.2, §3.4).
 *   q    [B, L, Hq, D]  bf16, pre-RoPE, query at position l is row l
 *   k, v [B, L, Hkv, D] bf16, k pre-RoPE; Hq % Hkv == 0 (grouped-query heads:
 *                       query head h reads kv head h / (Hq / Hkv))
 *   out  [B, L, Hq, D]  bf16 (written)
 *   lse  [B, Hq, L]     fp32 (written)
 *   D == 128.  w_local >= 0 (0 = every pair remote), w_pretrained >= 1,
 *   rope_base > 1.  Queries and keys are rotated inside the attention kernel
 *   (keys tile by tile in shared memory, to R(k) for the local passes and to
 *   R(f(k)) for the remote ones), so the call needs no memory beyond its
 *   arguments.
 */
jl_status jl_bifocal_prefill(const void *q, const void *k, const void *v,
                             void *out, float *lse, int B, int L, int Hq,
                             int Hkv, int D, int w_local, int w_pretrained,
                             double rope_base, jl_stream_t stream);

/* Bytes of caller workspace jl_bifocal_prefill_ex needs: 0 for every size and
 * dtype (the keys are rotated inside the kernels). */
size_t jl_bifocal_prefill_workspace_size(int B, int L, int Hkv, int D,
                                         jl_dtype dtype);

/* Bytes of workspace jl_bifocal_prefill_ex needs with JL_FLAG_ROTATE_KEYS_ONCE:
 * two bf16 copies of the keys, 2 * B * L * Hkv * D * 2 bytes, each rounded up
 * to 256.  0 for sizes below 1. */
size_t jl_bifocal_prefill_rotated_keys_bytes(int B, int L, int Hkv, int D);

/*
 * Bifocal prefill with every option.  dtype JL_BF16 (D == 128, tensor cores)
 * or JL_F32 (D in {64, 128}, fp32 CUDA-core kernel; out is fp32).
 * softmax_scale <= 0 selects 1/sqrt(D).  flags: JL_FLAG_NO_BIFOCAL,
 * JL_FLAG_ROTATE_KEYS_ONCE.
 * workspace, workspace_bytes: used only with JL_FLAG_ROTATE_KEYS_ONCE (the
 * rotated keys; at least jl_bifocal_prefill_rotated_keys_bytes() bytes,
 * 256-byte aligned, JL_ERR_INVALID_ARG otherwise).  Without the flag no
 * workspace is needed: any value, NULL and 0 included, is accepted and
 * nothing is written there.
 */
jl_status jl_bifocal_prefill_ex(const void *q, const void *k, const void *v,
                                void *out, float *lse, int B, int L, int Hq,
                                int Hkv, int D, int w_local, int w_pretrained,
                                double rope_base, jl_dtype dtype,
                                float softmax_scale, unsigned flags,
                                void *workspace, size_t workspace_bytes,
                                jl_stream_t stream);

/*
 * The same bifocal prefill through the pages' unfused formulation, kept to
 * measure the fused kernel against it and as a second GPU check of the
 * inclusion-exclusion identity (bittide paper summary §3.2; techwalker
 * explainer §四): three attention calls and a LogSumExp merge,
 *   A = causal attention with every pair at remapped positions (f(q), f(k)),
 *   B = the local window (0 <= q - k < w_local) at original positions,
 *   C = the same window at remapped positions,
 *   out = (e^lse_A O_A + e^lse_B O_B - e^lse_C O_C) / (e^lse_A + e^lse_B - e^lse_C),
 *   lse = ln(e^lse_A + e^lse_B - e^lse_C).
 * Arguments, layouts and results are those of jl_bifocal_prefill (bf16,
 * D == 128; flags: JL_FLAG_NO_BIFOCAL).  A is written to out / lse and merged
 * in place; O_B, O_C (bf16) and their lse live in the workspace, so the merge
 * sees outputs rounded to bf16 (the fused kernel has no such step).
 * workspace: device memory of at least
 * jl_bifocal_prefill_3pass_workspace_size() bytes, 256-byte aligned
 * (required).  With w_local = 0 the window is empty and out = A.
 */
size_t jl_bifocal_prefill_3pass_workspace_size(int B, int L, int Hq, int Hkv, int D);
jl_status jl_bifocal_prefill_3pass(const void *q, const void *k, const void *v,
                                   void *out, float *lse, int B, int L, int Hq,
                                   int Hkv, int D, int w_local, int w_pretrained,
                                   double rope_base, unsigned flags,
                                   void *workspace, size_t workspace_bytes,
                                   jl_stream_t stream);

/*
 * Chunked prefill against a cache: Lq new tokens attend to a cached prefix and
 * to themselves (a long prompt processed in pieces, or text appended to a long
 * context; techwalker §三 for the cache at original positions).
 *   q              [B, Lq, Hq, D] bf16, pre-RoPE; row r is the token at position
 *                  q_offset + r
 *   k_cache_roped  [B, cache_capacity, Hkv, D] bf16, keys rotated by standard
 *                  RoPE at their original positions (the decode cache layout);
 *                  slots 0 .. q_offset + Lq - 1 valid (the prefix and this
 *                  chunk, written by the caller)
 *   v_cache        [B, cache_capacity, Hkv, D] bf16, the same slots valid
 *   out [B, Lq, Hq, D] bf16 and lse [B, Hq, Lq] fp32 (written)
 * G = max(1, ceil((q_offset + Lq) / w_pretrained)) from the total length, and
 * the local/remote rule of jl_bifocal_prefill over keys [0, q_offset + Lq): the
 * result is rows q_offset .. q_offset + Lq - 1 of jl_bifocal_prefill over the
 * whole sequence (up to the bf16 rounding of the cached keys).  Keys at
 * remapped positions are formed from the cache as R(f(k) - k) k_cache, tile by
 * tile inside the kernel; the cache is only read.
 * q_offset a multiple of 128 (JL_ERR_UNSUPPORTED otherwise), q_offset + Lq <=
 * cache_capacity, D == 128, flags: JL_FLAG_NO_BIFOCAL.
 * workspace, workspace_bytes: not used (no workspace is needed; the size
 * query returns 0); any value, NULL and 0 included, is accepted.
 */
size_t jl_bifocal_prefill_chunk_workspace_size(int B, int q_offset, int Lq, int Hkv,
                                               int D);
jl_status jl_bifocal_prefill_chunk(const void *q, const void *k_cache_roped,
                                   const void *v_cache, int q_offset, int cache_capacity,
                                   void *out, float *lse, int B, int Lq, int Hq, int Hkv,
                                   int D, int w_local, int w_pretrained, double rope_base,
                                   unsigned flags, void *workspace, size_t workspace_bytes,
                                   jl_stream_t stream);

/* Bytes of workspace jl_bifocal_decode needs for these sizes. */
size_t jl_bifocal_decode_workspace_size(int B, int Hq, int Hkv, int D, int pos);

/*
 * Single-token bifocal decode, bf16 (techwalker §三; bittide §3.3).
 *   q_new          [B, Hq, D] bf16, pre-RoPE, the token at position `pos`
 *   k_cache_roped  [B, cache_capacity, Hkv, D] bf16, keys already rotated by
 *                  standard RoPE at their original positions; slots 0..pos are
 *                  valid and slot pos holds the new token's key
 *   v_cache        [B, cache_capacity, Hkv, D] bf16
 *   out [B, Hq, D] bf16 and lse [B, Hq] fp32 (written)
 *   G is computed from L = pos + 1.  Keys with pos - k < w_local take no
 *   correction; farther keys are rotated by dk = f(k) - k in registers, and the
 *   query by dq = f(pos) - pos.  The caches are never written.
 *   workspace: device memory of at least jl_bifocal_decode_workspace_size()
 *   bytes, 16-byte aligned (split-KV partial results).
 *   D == 128, 0 <= pos < cache_capacity, Hq % Hkv == 0.
 *   flags: JL_FLAG_NO_BIFOCAL; JL_FLAG_DEBUG_SKIP_ARRIVE (tests only).
 */
jl_status jl_bifocal_decode(const void *q_new, const void *k_cache_roped,
                            const void *v_cache, int pos, int cache_capacity,
                            void *out, float *lse, void *workspace,
                            size_t workspace_bytes, int B, int Hq, int Hkv,
                            int D, int w_local, int w_pretrained,
                            double rope_base, unsigned flags,
                            jl_stream_t stream);

/*
 * jl_bifocal_decode_noalloc -- the same single-token decode as
 * jl_bifocal_decode, for callers that cannot allocate device memory: for
 * example a host engine whose memory pool owns every device byte and forbids
 * other allocations, or a latency-critical decode loop that cannot accept the
 * implicit synchronisation an allocation brings.  This entry point has no
 * counterpart in the paper; it is a packaging variant of the decode path.
 *
 *   Arguments, layouts and results are those of jl_bifocal_decode, without
 *   the workspace.  It calls no cudaMalloc, cudaFree or other allocating
 *   routine, and does not touch the library-owned angle table or status word:
 *   the kernel evaluates its rotation angles itself (fp64 sincos rounded to
 *   fp32, as the table holds them).
 *   Split partials go to a fixed array compiled into the library:
 *   1,048,576 floats (4 MiB), present on every GPU that loads the library until
 *   the process exits.  Sizes are accepted while
 *   B * Hq * n_splits * (D + 4) fits it (n_splits about 75 for B=1, Hq=32 at
 *   pos = 131071); larger sizes return JL_ERR_UNSUPPORTED with a message.
 *   The first call on each device looks up that array's device address (with
 *   that device current) and caches it; make that first call before any stream
 *   capture.  jl_finalize drops the cached addresses: after a device reset
 *   (cudaDeviceReset), call jl_finalize before the next call, which then looks
 *   the address up again.  Every call shares the array and it keeps the last call's
 *   partials; each call writes every entry it reads before reading it.  Calls
 *   whose executions overlap on the GPU (other streams, other threads) race on
 *   the array: serialise them.
 */
jl_status jl_bifocal_decode_noalloc(const void *q_new, const void *k_cache_roped,
                                    const void *v_cache, int pos, int cache_capacity,
                                    void *out, float *lse, int B, int Hq, int Hkv, int D,
                                    int w_local, int w_pretrained, double rope_base,
                                    unsigned flags, jl_stream_t stream);

/*
 * Batched single-token decode, one position per sequence (the batch-size > 1,
 * ragged case of jl_bifocal_decode; techwalker §三, bittide §3.3).
 *   pos   HOST array of B positions (a DEVICE array with JL_FLAG_DEVICE_POS),
 *         0 <= pos[b] < cache_capacity; sequence b decodes its token at pos[b]
 *         over cache slots 0..pos[b], with its own
 *         G = max(1, ceil((pos[b] + 1) / w_pretrained)) and window.
 *   q_new [B, Hq, D], caches [B, cache_capacity, Hkv, D], out [B, Hq, D],
 *   lse [B, Hq]: as jl_bifocal_decode.  Cache slots past pos[b] are never
 *   used (any contents).
 *   workspace: at least jl_bifocal_decode_batched_workspace_size() bytes,
 *   256-byte aligned.  The library plans one wave of CTAs over all sequences'
 *   keys on the host and copies the plan (a few KiB, from pageable memory)
 *   into the workspace on `stream` before the kernels; such a call is not
 *   capturable in a CUDA graph.  With JL_FLAG_DEVICE_POS, pos is a device
 *   array and the same plan is made on the device (capturable, bit for bit
 *   the same result).
 *   D == 128, Hkv <= 8, Hq / Hkv <= 8 (JL_ERR_UNSUPPORTED otherwise).
 *   flags: JL_FLAG_NO_BIFOCAL, JL_FLAG_DEVICE_POS.
 */
size_t jl_bifocal_decode_batched_workspace_size(int B, int Hq, int Hkv, int D);
jl_status jl_bifocal_decode_batched(const void *q_new, const void *k_cache_roped,
                                    const void *v_cache, const int *pos,
                                    int cache_capacity, void *out, float *lse,
                                    void *workspace, size_t workspace_bytes, int B,
                                    int Hq, int Hkv, int D, int w_local,
                                    int w_pretrained, double rope_base,
                                    unsigned flags, jl_stream_t stream);

/*
 * Batched single-token decode over a PAGED cache (the paged form of
 * jl_bifocal_decode_batched; techwalker §三, bittide §3.3).  Keys and values
 * live in a shared pool of fixed-size pages; a per-sequence block table lists
 * the pages of each sequence in key order.
 *   k_pages, v_pages  DEVICE pools [num_pages, page_size, Hkv, D] bf16; keys
 *         rotated at their ORIGINAL positions, as in jl_bifocal_decode.
 *   page_size  keys per page: a positive multiple of 16 (else
 *         JL_ERR_INVALID_ARG); num_pages * page_size <= 2^31 - 1.
 *   block_table  DEVICE int32 [B, max_pages_per_seq], 4-byte aligned: key k of
 *         sequence b is row k % page_size of page
 *         block_table[b * max_pages_per_seq + k / page_size].  Only the
 *         entries covering keys 0..pos[b] are read.  An entry outside
 *         [0, num_pages) is not followed: the kernel reads page 0 instead and
 *         raises the device status word, so out and lse are invalid and the
 *         next jl_check_device_status returns JL_ERR_INVALID_ARG.
 *   pos   HOST array of B positions, 0 <= pos[b] < max_pages_per_seq *
 *         page_size; the token of sequence b is at pos[b] and already stored
 *         (a DEVICE array with JL_FLAG_DEVICE_POS).
 *   q_new, out, lse, workspace, flags: as jl_bifocal_decode_batched (the same
 *         workspace size; capturable in a CUDA graph with JL_FLAG_DEVICE_POS).
 *   Rows of a page past pos[b] are never used (any contents).  For the same
 *   keys the result is bit for bit that of jl_bifocal_decode_batched.
 */
jl_status jl_bifocal_decode_paged(const void *q_new, const void *k_pages, const void *v_pages,
                                  int num_pages, int page_size, const int *block_table,
                                  int max_pages_per_seq, const int *pos, void *out, float *lse,
                                  void *workspace, size_t workspace_bytes, int B, int Hq,
                                  int Hkv, int D, int w_local, int w_pretrained,
                                  double rope_base, unsigned flags, jl_stream_t stream);

/* Message for the last non-OK status returned on this thread ("" if none). */
const char *jl_last_error(void);

/*
 * Synchronises `stream`, then reads and clears the current device's status
 * word.  Returns JL_ERR_TIMEOUT if a kernel gave up a bounded wait since the
 * last check, JL_ERR_INVALID_ARG if a kernel refused an out-of-range index (a
 * block-table entry of jl_bifocal_decode_paged); the outputs of that call are
 * then invalid.  JL_ERR_CUDA on a CUDA error, JL_OK otherwise.
 */
jl_status jl_check_device_status(jl_stream_t stream);

/* Releases every library-owned device buffer on every device (synchronises
 * each device first) and forgets the cached device address of
 * jl_bifocal_decode_noalloc's fixed array.  Later calls re-create them.  Call it
 * after a device reset, before the library's next call. */
void jl_finalize(void);

#ifdef __cplusplus
}
#endif

#endif /* JETLONG_H */
