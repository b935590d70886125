/*
 * ropeattn — causal attention with rotary position embedding (RoPE) applied at
 * remapped position indices, for NVIDIA B200 (sm_100a).
 *
 * Plain C ABI: pointers, sizes and one parameter struct. Every device pointer
 * must point to memory of the current CUDA device. Streams are passed as
 * `void*` holding a cudaStream_t (NULL = legacy default stream). All compute
 * calls are asynchronous and stream-ordered; the host returns after launch.
 *
 * What is computed (the passages that define it):
 *   RoPE frequencies theta_i = base^(-2i/d) and the block-diagonal rotation
 *   R_p on coordinate pairs (2i, 2i+1): "Periodic RoPE for Infinite Context
 *   LLMs", §3.1 Eq. 1-2. Position interpolation by a factor s uses angle
 *   (p/s)*theta_i: "Jet-Long: Efficient Long-Context Extension with Dynamic
 *   Bifocal RoPE", §2.2. The softmax scale is 1/sqrt(d) (Periodic RoPE §3.3
 *   Eq. 6) unless softmax_scale > 0 is given.
 *
 * Layouts (row-major, contiguous, 16-byte aligned base pointers):
 *   prefill q [B, S, Hq, D] bf16; k, v [B, S, Hkv, D] bf16 (unrotated);
 *           out [B, S, Hq, D] fp32; lse [B, Hq, S] fp32 (natural log of the
 *           sum of exp of the scaled scores).
 *   decode  q [B, Hq, D] bf16 (unrotated, the token at position n-1);
 *           k_cache [B, n, Hkv, D] bf16 already rotated at each key's own
 *           position; v_cache [B, n, Hkv, D] bf16; out [B, Hq, D] fp32;
 *           lse [B, Hq] fp32.
 *   GQA: query head h reads key/value head h / (Hq / Hkv).
 *   Supported: D in {64, 128, 256} (the prefill runs D = 256 with one
 *   128-row query tile per CTA and 64-key tiles);
 *   Hq % Hkv == 0; decode also needs Hq / Hkv <= 16; the backward needs
 *   D = 64 or 128.
 *   Half-split pairing (params.pairing = ROPEATTN_PAIR_HALF): q, k and v are
 *   given in their own order; the rotation pairs coordinates (i, i + D/2),
 *   and key caches hold each rotated key in adjacent order instead (element
 *   2i = coordinate i, element 2i+1 = coordinate i + D/2), as
 *   ropeattn_cache_write stores them. Value caches and outputs keep the
 *   values' order.
 *
 * Errors: every entry point returns ROPEATTN_OK (0) or a negative code and
 * sets a thread-local message readable with ropeattn_last_error(). Argument
 * errors are reported before any launch and leave all buffers untouched.
 */
#ifndef ROPEATTN_H_
#define ROPEATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ROPEATTN_OK                      0
#define ROPEATTN_ERR_INVALID_ARG        -1  /* null/misaligned pointer, bad shape or parameter */
#define ROPEATTN_ERR_UNSUPPORTED_DEVICE -2  /* current device is not sm_100 */
#define ROPEATTN_ERR_WORKSPACE          -3  /* workspace missing or smaller than required */
#define ROPEATTN_ERR_CUDA               -4  /* a CUDA runtime call or launch failed */
#define ROPEATTN_ERR_TIMEOUT            -5  /* a kernel's bounded wait ran out (see ropeattn_status) */

/* Position-map kinds. */
typedef enum {
  /* p(t) = t. Periodic RoPE §3.1. */
  ROPEATTN_STANDARD  = 0,
  /* EndPrompt two segments: p(t) = t for t < seg1_len, else
   * term_start + (t - seg1_len); angles use p / interp (position
   * interpolation). "EndPrompt: Efficient Long-Context Extension via
   * Terminal Anchoring", abstract. */
  ROPEATTN_ENDPROMPT = 1,
  /* p(t) = t mod window inside causal sliding-window attention over the
   * `window` keys {t-window+1 .. t}. Periodic RoPE §3.2 Eq. 4-5. */
  ROPEATTN_PERIODIC  = 2,
  /* No rotation, full causal attention. Periodic RoPE §3.3 Eq. 6. */
  ROPEATTN_NOPE      = 3,
  /* Jet-Long bifocal: keys with t - s <= w0 use RoPE at (t, s); the others
   * use RoPE at (f(t), f(s)), f(x) = floor(x / G),
   * G = max(1, ceil(L / w_pretrained)), L = the sequence length (prefill: S;
   * decode: n). Jet-Long §3 Eq. 1, §3.1 Eq. 2-3. */
  ROPEATTN_BIFOCAL   = 4
} ropeattn_kind;

/* Which coordinates the rotation pairs. Periodic RoPE §3.1 Eq. 2 writes the
 * rotation block-diagonally on (2i, 2i+1); the half-split form pairs
 * (i, i + D/2) with the same angle p * theta_i. The two differ only by a
 * fixed permutation of the head dimensions, applied to q and k alike. NOPE
 * rotates nothing and ignores the field. */
typedef enum {
  ROPEATTN_PAIR_ADJACENT = 0,   /* (2i, 2i+1) */
  ROPEATTN_PAIR_HALF     = 1    /* (i, i + D/2) */
} ropeattn_pairing;

/* Parameters of the position map. Fields a kind does not use are ignored,
 * except the reserved ones, which must be zero. */
typedef struct ropeattn_params {
  int32_t kind;           /* ropeattn_kind */
  int32_t fixed_group;    /* BIFOCAL: 0 -> G = max(1, ceil(L / w_pretrained)) (Jet-Long
                             Eq. 2, the dynamic schedule); > 0 -> this G for every L (a
                             single group size fixed up front, as the grouped-window
                             baselines Jet-Long contrasts itself with). Others: 0. */
  double  rope_base;      /* Theta > 1 (e.g. 1e4, 5e5, 1e6) */
  double  interp;         /* ENDPROMPT: interpolation factor s >= 1 (others: ignored) */
  int64_t seg1_len;       /* ENDPROMPT: n1 >= 0, length of the intact first segment */
  int64_t term_start;     /* ENDPROMPT: first position of the terminal segment, >= 0 */
  int64_t window;         /* PERIODIC: W >= 1 (window length = period) */
  int64_t w0;             /* BIFOCAL: local window, >= 0 (0 = the token itself only) */
  int64_t w_pretrained;   /* BIFOCAL: pretrained context window, >= 1 (unused with fixed_group) */
  float   softmax_scale;  /* > 0 to override; 0 -> 1/sqrt(D) */
  int32_t pairing;        /* ropeattn_pairing (0 = adjacent) */
  int32_t reserved[2];    /* must be 0 */
} ropeattn_params;

/* Position map of a sequence of length L (Periodic RoPE §3.2 Eq. 4; Jet-Long
 * §3.1 Eq. 2-3; EndPrompt abstract).
 *   d_pos_local  [L] int32, device: the position RoPE uses for each token
 *                (BIFOCAL: the exact position t; NOPE: 0).
 *   d_pos_remote [L] int32, device, may be NULL; required for BIFOCAL:
 *                f(t) = floor(t / G). Written as t for other kinds when given.
 *   h_G          host int32, may be NULL: receives G (1 unless BIFOCAL).
 * Asynchronous on `stream` (h_G is written before return). L == 0 is a no-op.
 * Errors: INVALID_ARG (L < 0, L >= 2^31, a position >= 2^31, null
 * d_pos_local with L > 0, null d_pos_remote for BIFOCAL), CUDA. */
int ropeattn_posmap(const ropeattn_params* params, int64_t L,
                    int32_t* d_pos_local, int32_t* d_pos_remote, int32_t* h_G,
                    void* stream);

/* Writes tokens into a decode cache (Jet-Long §3.2 Eq. 4: each key is stored
 * rotated at its own position, so the cache is never rewritten when the
 * bifocal group size G changes as the sequence grows):
 *   k_cache[b, start + i, h, :] = R(p(start + i)) k[b, i, h, :]  (bf16, RNE)
 *   v_cache[b, start + i, h, :] = v[b, i, h, :]
 * for i < count, p the kind's primary position of the absolute token index
 * (t for STANDARD and BIFOCAL, EndPrompt's two segments, t mod W for
 * PERIODIC; NOPE stores keys unrotated). Angles p * theta_i in double
 * precision, rotation in fp32, as the prefill's key pre-pass does. With
 * ROPEATTN_PAIR_HALF the key is rotated on pairs (i, i + D/2) and stored in
 * adjacent order (element 2i = rotated coordinate i, 2i+1 = rotated
 * coordinate i + D/2), the order every cache reader of this library expects
 * for half-split params; values are copied as given.
 *   k, v:             [B, count, Hkv, D] bf16, device, 16-byte aligned
 *   k_cache, v_cache: [B, cache_len, Hkv, D] bf16, device, 16-byte aligned;
 *                     caller-owned
 *   v, v_cache:       both NULL to write keys only
 *   start + count <= cache_len. A prefill of S tokens emits its cache with
 *   start = 0, count = S; a decode step appends its token with start = n-1
 *   before ropeattn_decode reads the first n rows.
 * count == 0 or B == 0 is a no-op. Errors: INVALID_ARG, UNSUPPORTED_DEVICE,
 * CUDA. */
int ropeattn_cache_write(const void* k, const void* v, void* k_cache, void* v_cache,
                         int64_t B, int64_t start, int64_t count, int64_t cache_len,
                         int32_t Hkv, int32_t D, const ropeattn_params* params, void* stream);

/* Bytes of device workspace ropeattn_prefill needs for these shapes:
 * rotated keys (one copy per position map the kind uses), the query angle
 * tables and, for half-split pairing, a copy of q in adjacent order. 0 for
 * NOPE. */
size_t ropeattn_prefill_workspace_size(const ropeattn_params* params, int64_t B,
                                       int64_t S, int32_t Hq, int32_t Hkv, int32_t D);

/* Causal prefill attention with RoPE at remapped positions, L = S.
 * One pre-pass rotates the keys into `workspace` (and writes the query angle
 * tables); the attention kernel rotates each query tile inside its TMA-staged
 * load, runs QK^T and PV on the tensor cores (tcgen05, TMEM accumulators),
 * keeps an online softmax per row, and for BIFOCAL merges the local and
 * remote partials by their log-sum-exp (Jet-Long §3.3 Eq. 7) before writing.
 * Tensor-core operands are bf16: the rotated q and k are rounded to bf16
 * (round to nearest even); scores, softmax and outputs are fp32. With
 * ROPEATTN_PAIR_HALF the key pre-pass reads k on pairs (i, i + D/2) and
 * writes adjacent order, and one streaming pass first copies q into the
 * workspace in adjacent order; the attention kernel is the same.
 *   workspace: device, 256-byte aligned, >= ropeattn_prefill_workspace_size
 *              bytes (may be NULL when that size is 0). Caller-owned; the
 *              call overwrites it; calls sharing it must be stream-ordered.
 * S == 0 or B == 0 is a no-op.
 * Errors: INVALID_ARG, UNSUPPORTED_DEVICE, WORKSPACE, CUDA. */
int ropeattn_prefill(const void* q, const void* k, const void* v,
                     float* out, float* lse,
                     int64_t B, int64_t S, int32_t Hq, int32_t Hkv, int32_t D,
                     const ropeattn_params* params,
                     void* workspace, size_t workspace_bytes, void* stream);

/* The two halves of ropeattn_prefill, for callers that reuse the rotated
 * keys (several query blocks against the same keys) or time the stages:
 *   ropeattn_prefill_prepare writes the rotated keys and the query angle
 *   tables into `workspace` (reads k only; no-op for NOPE);
 *   ropeattn_prefill_attend runs the attention kernel on a workspace that a
 *   prepare call with the same params and shapes filled earlier on the same
 *   stream (k is read directly only for NOPE).
 * ropeattn_prefill(...) == prepare(...) followed by attend(...).
 * Same arguments, layouts and errors as ropeattn_prefill. */
int ropeattn_prefill_prepare(const void* k, int64_t B, int64_t S, int32_t Hq, int32_t Hkv, int32_t D,
                             const ropeattn_params* params, void* workspace, size_t workspace_bytes,
                             void* stream);
int ropeattn_prefill_attend(const void* q, const void* k, const void* v, float* out, float* lse,
                            int64_t B, int64_t S, int32_t Hq, int32_t Hkv, int32_t D,
                            const ropeattn_params* params,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes of ropeattn_prefill_backward: per position map the rotated
 * queries and keys (bf16) and the angle table, plus the log-sum-exp in log2
 * units and Delta (fp32, rows padded to a multiple of 64). 0 for arguments
 * the backward rejects (head_dim other than 64 and 128 among them) and for
 * an empty problem. */
size_t ropeattn_prefill_backward_workspace_size(const ropeattn_params* params, int64_t B, int64_t S,
                                                int32_t Hq, int32_t Hkv, int32_t D);

/* Gradients of the prefill: given the forward's inputs, its out and lse, and
 * the upstream gradient dout of out, writes dq, dk and dv. With P the row
 * softmax of scale * score(t,s), score(t,s) = <R_a q_t, R_b k_s> at the
 * kind's positions (Periodic RoPE §3.1 Eq. 2, §3.2 Eq. 4; Jet-Long §3 Eq. 1
 * and §3.1 Eq. 2-3; EndPrompt abstract), Delta_t = dout_t . out_t and
 * dS = P (dout . v - Delta):
 *   dv_s = sum_t P(t,s) dout_t,   dk_s = scale R_b^T sum_t dS(t,s) R_a q_t,
 *   dq_t = scale R_a^T sum_s dS(t,s) R_b k_s,
 * each bifocal sum split into its local (exact positions) and remote (f
 * positions) parts. P is recomputed from lse (no softmax state is saved).
 * Two tensor-core kernels (tcgen05, TMEM accumulators, no atomics: results
 * are bitwise reproducible): one per 128-key tile for dk and dv (summing the
 * query heads of each GQA group), one per 128-row query tile for dq. The
 * rotated q and k, P and dS are bf16 operands; accumulation is fp32.
 *   q, k, v, params: as for ropeattn_prefill (same kind, positions, scale,
 *                    pairing); D = 64 or 128.
 *   out [B, S, Hq, D] fp32, lse [B, Hq, S] fp32: ropeattn_prefill's results.
 *   dout [B, S, Hq, D] bf16, device.
 *   dq [B, S, Hq, D], dk, dv [B, S, Hkv, D]: fp32, device, caller-owned;
 *                    every element is written (nothing is accumulated into
 *                    them). With ROPEATTN_PAIR_HALF dq and dk are in the
 *                    heads' own order, like q and k.
 *   workspace: device, 256-byte aligned, >= the size above.
 * S == 0 or B == 0 is a no-op.
 * Errors: INVALID_ARG (also D not 64 or 128), UNSUPPORTED_DEVICE, WORKSPACE,
 * CUDA. */
int ropeattn_prefill_backward(const void* q, const void* k, const void* v, const float* out,
                              const float* lse, const void* dout, float* dq, float* dk, float* dv,
                              int64_t B, int64_t S, int32_t Hq, int32_t Hkv, int32_t D,
                              const ropeattn_params* params, void* workspace, size_t workspace_bytes,
                              void* stream);

/* Prefill of a chunk of `count` new tokens, at positions start..L-1 with
 * L = start + count, against a decode cache that already holds all L keys
 * and values (rows 0..L-1 written by ropeattn_cache_write, the chunk's own
 * tokens included): the last `count` rows of a prefill of length L, for
 * chunked prefill and for extending a cached context. Keys are read as
 * stored (Jet-Long §3.2 Eq. 4); for BIFOCAL a pre-pass writes the remote
 * keys R(Delta s) k_cache[s], Delta s = f(s) - s with G = G(L) (Eq. 5-6),
 * into `workspace`, and the remote pass reads them. Queries are rotated in
 * the attention kernel as in ropeattn_prefill. Tensor-core operands are
 * bf16 (the remote keys are rounded to bf16 after the correction). With
 * ROPEATTN_PAIR_HALF the key cache is in adjacent order (as
 * ropeattn_cache_write stores it) and q is copied into the workspace in
 * adjacent order first.
 *   q:      [B, count, Hq, D] bf16, unrotated
 *   k_cache, v_cache: [B, L, Hkv, D] bf16 (contiguous, L rows)
 *   out:    [B, count, Hq, D] fp32;  lse: [B, Hq, count] fp32 (natural log)
 *   workspace: >= ropeattn_prefill_chunk_workspace_size bytes, 256-byte
 *              aligned (may be NULL when that size is 0).
 * count == 0 or B == 0 is a no-op. With start = 0 this is a whole prefill
 * from a cache. Errors: INVALID_ARG, UNSUPPORTED_DEVICE, WORKSPACE, CUDA. */
size_t ropeattn_prefill_chunk_workspace_size(const ropeattn_params* params, int64_t B, int64_t start,
                                             int64_t count, int32_t Hq, int32_t Hkv, int32_t D);
int ropeattn_prefill_chunk(const void* q, const void* k_cache, const void* v_cache,
                           float* out, float* lse,
                           int64_t B, int64_t start, int64_t count, int32_t Hq, int32_t Hkv, int32_t D,
                           const ropeattn_params* params, void* workspace, size_t workspace_bytes,
                           void* stream);
/* ropeattn_prefill_chunk over caches with spare rows: k_cache and v_cache
 * are [B, cache_len, Hkv, D] with cache_len >= start + count (rows of each
 * batch entry allocated for the sequence to grow into); the first
 * start + count rows are used. ropeattn_prefill_chunk is this call with
 * cache_len = start + count; the workspace size is the same. */
int ropeattn_prefill_chunk_cache(const void* q, const void* k_cache, const void* v_cache,
                                 float* out, float* lse,
                                 int64_t B, int64_t start, int64_t count, int64_t cache_len,
                                 int32_t Hq, int32_t Hkv, int32_t D,
                                 const ropeattn_params* params, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* Comparator: the literal three-call bifocal prefill of Jet-Long §3.3 with a
 * separate merge kernel, on the same attention kernel: (A) sliding window
 * w0 at exact positions, (B) full causal at remote positions, (C) sliding
 * window w0 at remote positions, each writing its normalised output and
 * LSE, then O = (W_A O_A + W_B O_B - W_C O_C) / (W_A + W_B - W_C) with
 * W_X = exp(l_X - M), M = max l_X (Eq. 7), in fp32. Same result as
 * ropeattn_prefill up to rounding; exists to time the fused kernel against
 * the unfused route on the same GPU. Needs an effective bifocal map (G > 1
 * and w0 < S-1), else INVALID_ARG. Arguments and layouts as ropeattn_prefill;
 * the workspace also holds O_A, O_C and their LSEs (2 (B S Hq D + B Hq S)
 * floats more). Errors: INVALID_ARG, UNSUPPORTED_DEVICE, WORKSPACE, CUDA. */
size_t ropeattn_prefill_three_call_workspace_size(const ropeattn_params* params, int64_t B, int64_t S,
                                                  int32_t Hq, int32_t Hkv, int32_t D);
int ropeattn_prefill_three_call(const void* q, const void* k, const void* v, float* out, float* lse,
                                int64_t B, int64_t S, int32_t Hq, int32_t Hkv, int32_t D,
                                const ropeattn_params* params, void* workspace, size_t workspace_bytes,
                                void* stream);

/* Bytes of device workspace ropeattn_decode needs (split-KV partials and
 * per-head arrival counters). Depends on the current device's SM count. */
size_t ropeattn_decode_workspace_size(int64_t B, int64_t n, int32_t Hq,
                                      int32_t Hkv, int32_t D);

/* One decode step: the query token at position n-1 against a cache of n keys
 * (its own key included, stored last), L = n. Jet-Long §3.2 Eq. 4-6: the
 * cache is never rewritten; for BIFOCAL the query is rotated to p = n-1 and
 * corrected by Delta q = f(n-1) - (n-1), and each cached key with
 * (n-1) - k > w0 is corrected on the fly by Delta k = f(k) - k, in fp32
 * registers. Other kinds: the query is rotated to its position p(n-1) and
 * the cache is read as stored (PERIODIC reads only the last `window` keys).
 * Split-KV: each CTA streams a contiguous key range of one KV head through
 * a shared-memory ring filled by TMA, and the last CTA of each head merges
 * the partials by their log-sum-exp in a fixed order (deterministic). With
 * ROPEATTN_PAIR_HALF the key cache is in adjacent order (as
 * ropeattn_cache_write stores it) and the query is first copied into the
 * workspace in adjacent order.
 *   workspace: device, >= ropeattn_decode_workspace_size bytes (the size
 *              covers either pairing). The call clears its counters with
 *              cudaMemsetAsync on `stream` first; calls sharing a workspace
 *              must be stream-ordered.
 * n == 0 or B == 0 is a no-op.
 * Errors: INVALID_ARG, UNSUPPORTED_DEVICE, WORKSPACE, CUDA. */
int ropeattn_decode(const void* q, const void* k_cache, const void* v_cache,
                    float* out, float* lse,
                    int64_t B, int64_t n, int32_t Hq, int32_t Hkv, int32_t D,
                    const ropeattn_params* params,
                    void* workspace, size_t workspace_bytes, void* stream);

/* ropeattn_decode for callers that cannot allocate device memory when they
 * call: for example a plug-in running inside an engine that owns every device
 * allocation, or a latency-critical serving loop where a cudaMalloc (which can
 * synchronize the device) is not acceptable. The pages have no counterpart:
 * this is a library convenience, not part of the method.
 * Same arguments, layouts, results and errors as ropeattn_decode, without the
 * workspace: the split-KV scratch lives in a 4 MiB array inside the library
 * (a file-scope __device__ array that every GPU loading the library holds
 * until process exit). Shapes whose ropeattn_decode_workspace_size exceeds
 * 4 MiB are rejected with ROPEATTN_ERR_WORKSPACE before any launch.
 * Every call looks up the array's device address on the current device (a
 * table lookup that allocates nothing, so an address never outlives a device
 * reset); the first call on a device may load the library's device code, so
 * make that first call before any stream capture. The call allocates
 * nothing: it clears the scratch counters with cudaMemsetAsync on `stream`
 * and launches the decode kernel.
 * All calls share the one array: calls that may overlap on the GPU (different
 * streams without ordering, or different host threads) race and must not be
 * issued; calls on one stream are safe. */
int ropeattn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                            float* out, float* lse,
                            int64_t B, int64_t n, int32_t Hq, int32_t Hkv, int32_t D,
                            const ropeattn_params* params, void* stream);

/* Failure-detection self-test: launches one CTA whose mbarrier wait nothing
 * completes, bounded by limit_ns (1e3..1e9 ns), through the same bounded
 * wait every kernel uses. When the wait runs out the kernel sets the device
 * status word and returns; *d_result (device int32) receives 0 (gave up) or
 * 1 (completed, which cannot happen). The next ropeattn_status() reports
 * ROPEATTN_ERR_TIMEOUT; the context stays usable. No fault is involved.
 * Errors: INVALID_ARG, UNSUPPORTED_DEVICE, CUDA. */
int ropeattn_wait_selftest(int64_t limit_ns, int32_t* d_result, void* stream);

/* ropeattn_decode over caches with spare rows: k_cache and v_cache are
 * [B, cache_len, Hkv, D] (cache_len >= n, the rows of each batch entry
 * allocated for the sequence to grow into, as ropeattn_cache_write fills
 * them); the first n rows of each batch entry are attended. Otherwise
 * identical to ropeattn_decode (which is this call with cache_len = n). */
int ropeattn_decode_cache(const void* q, const void* k_cache, const void* v_cache,
                          float* out, float* lse,
                          int64_t B, int64_t n, int64_t cache_len, int32_t Hq, int32_t Hkv, int32_t D,
                          const ropeattn_params* params, void* workspace, size_t workspace_bytes,
                          void* stream);

/* Comparator: decode with the correction rotation unfused. A separate pass
 * writes a copy of the key cache in `workspace` in which every remote key
 * (t - s > w0) is turned by Delta s - Delta q (Jet-Long Eq. 5-6; then
 * q_local . copy[s] = q_remote . R(Delta s) k_cache[s]) and every local key
 * is copied as is, then a standard-RoPE ropeattn_decode reads the copy. Same
 * result as ropeattn_decode up to rounding (the copy is rounded to bf16); it
 * exists to time the fused decode against the unfused route. Needs an
 * effective bifocal map, else INVALID_ARG. Arguments and layouts as
 * ropeattn_decode; workspace >= ropeattn_decode_unfused_workspace_size.
 * Errors: INVALID_ARG, UNSUPPORTED_DEVICE, WORKSPACE, CUDA. */
size_t ropeattn_decode_unfused_workspace_size(int64_t B, int64_t n, int32_t Hq, int32_t Hkv, int32_t D);
int ropeattn_decode_unfused(const void* q, const void* k_cache, const void* v_cache,
                            float* out, float* lse,
                            int64_t B, int64_t n, int32_t Hq, int32_t Hkv, int32_t D,
                            const ropeattn_params* params, void* workspace, size_t workspace_bytes,
                            void* stream);

/* Reads and clears the device status word of the current device (waits for
 * the device to be idle first). Returns ROPEATTN_OK, or ROPEATTN_ERR_TIMEOUT
 * if any kernel since the last call gave up on a bounded wait (its outputs
 * are then invalid), or ROPEATTN_ERR_CUDA. */
int ropeattn_status(void);

/* Message for the last error on this host thread ("" if none). */
const char* ropeattn_last_error(void);

/* Library version as major*10000 + minor*100 + patch. */
int ropeattn_version(void);

#ifdef __cplusplus
}
#endif

#endif  /* ROPEATTN_H_ */
