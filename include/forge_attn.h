/*
 * forge_attn.h -- C ABI of the B200 (sm_100a) fused causal attention library
 * (libforge_attn.so): forward and backward of causal multi-head attention with
 * GQA head mapping, an optional sliding window and an optional attention-logit
 * softcap.
 *
 * What the operation is (Forge pages):
 *   S_ij  = scale * (q_i . k_j)
 *   s_ij  = softcap * tanh(S_ij / softcap)      if softcap > 0, else S_ij
 *           (the cap applies tanh to the scores before the softmax:
 *            src/nn/attention.h commit log, Wave 2 (attention kernels);
 *            ARCHITECTURES.md "Vague 2" item 9)
 *   key j is visible to query i iff  i - window < j <= i   (window = 0: j <= i)
 *           (ARCHITECTURES.md "Vague 2" item 8; sliding_window(0) default,
 *            forge-studio RESEARCH.md section 2)
 *   P_i   = softmax over the visible j of s_ij,   o_i = sum_j P_ij v_j,
 *   lse_i = log sum_j exp(s_ij)  (natural log)
 *   Query head hq reads KV head hq / (Hq / Hkv) (GQA; Hq % Hkv == 0 is the
 *   config rule n_heads % n_kv_heads == 0, RESEARCH.md section 2).
 *   The backward is the exact gradient of o with respect to q, k, v, including
 *   the tanh' factor of the cap (every backward on the pages differentiates
 *   through the cap exactly).
 *   A per-layer pattern (sliding_global_every) is chosen by the caller: a global
 *   layer passes window = 0.
 *
 * Layouts (all row-major, contiguous, device memory, 16-byte aligned):
 *   q, o, dO, dq : [B][Hq][T][D]      k, v, dk, dv : [B][Hkv][T][D]
 *   lse          : [B][Hq][T] float32
 *   `dtype` gives the element type of q, k, v, o, dO, dq, dk, dv.
 *   FORGE_DTYPE_BF16 runs the tensor-core kernels (bf16 operands, f32
 *   accumulation, P and dS rounded to bf16 before their products);
 *   FORGE_DTYPE_F32 runs f32 CUDA-core kernels (f32 arithmetic throughout).
 *   Supported head dims: 64, 128, 256 (d_k != d_v: forge_attn_fwd_dkv).
 *
 * Sizes (checked before any launch; FORGE_ERR_INVALID_ARG otherwise):
 *   B, Hq, Hkv, T >= 1 (an empty problem is an error, not a no-op);
 *   Hq % Hkv == 0; D even; B * Hq <= 2^24; T <= 2^30; B * Hq * T * D <= 2^40
 *   elements; (T / 128 rounded up) * B * Hq < 2^31 (the grid). A D that passes
 *   these but has no kernel returns FORGE_ERR_UNSUPPORTED.
 *
 * Ownership and behaviour:
 *   The caller allocates and frees every buffer, including the backward
 *   workspace. The library never allocates, frees or synchronises (except
 *   forge_attn_check, which synchronises the stream it is given), and launches
 *   only on `stream` (a cudaStream_t; NULL is the legacy default stream).
 *   Calls are asynchronous; outputs are fully overwritten (dq, dk, dv are not
 *   accumulated into). Errors are returned, never thrown or aborted.
 *   Every wait inside a kernel is bounded; a wait that runs out records
 *   FORGE_ERR_TIMEOUT in a device status word that forge_attn_check reports.
 */
#ifndef FORGE_ATTN_H
#define FORGE_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FORGE_OK = 0,
    FORGE_ERR_INVALID_ARG = 1, /* null or misaligned pointer, bad size, bad scalar */
    FORGE_ERR_UNSUPPORTED = 2, /* valid but no kernel built for it (e.g. a head dim, a (d_k, d_v) pair, a decode group size) */
    FORGE_ERR_WORKSPACE = 3,   /* backward workspace missing, misaligned or too small */
    FORGE_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
    FORGE_ERR_TIMEOUT = 5      /* a bounded wait inside a kernel ran out */
} forge_status;

typedef enum { FORGE_DTYPE_F32 = 0, FORGE_DTYPE_BF16 = 1 } forge_dtype;

/*
 * Forward. Writes o and lse (lse is kept for the backward).
 * scale: finite, > 0 (usually 1/sqrt(D)); window: >= 0, 0 = off, >= T acts as
 * off; softcap: finite, >= 0, 0 = off.
 * Returns FORGE_OK or an error; on error nothing is launched.
 */
forge_status forge_attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                            int B, int Hq, int Hkv, int T, int D, float scale, int window,
                            float softcap, forge_dtype dtype, void *stream);

/*
 * Forward with two optional extras (either pointer may be NULL; with both NULL
 * this is forge_attn_fwd):
 *  - sink [Hq] f32 (device): a learned logit per query head that joins every
 *    row's softmax denominator and has no value vector (attention sinks:
 *    ARCHITECTURES.md family table, GPT-OSS row, a per-head bias added to the
 *    softmax denominator; "Vague 2" item 10, which starts the online softmax's
 *    (max, sum) from it). In the units of the scores the softmax sees (after
 *    scale and cap; the sink itself is not capped). P_ij = exp(s_ij) /
 *    (exp(sink[hq]) + sum_j exp(s_ij)); lse includes it.
 *  - max_logit [B][Hq] f32 (device, written): per (batch, query head) the
 *    maximum over the allowed (i, j) of the score the softmax sees, the sink not
 *    included: the per-head maximum attention logit that QK-Clip monitors
 *    ("Vague 3" item 12; family table, Kimi K2 row). The call first sets it to
 *    -inf, then the kernels raise it with atomic maxima.
 * Both 4-byte aligned. Same errors as forge_attn_fwd.
 */
forge_status forge_attn_fwd_ext(const void *q, const void *k, const void *v, void *o, float *lse,
                                int B, int Hq, int Hkv, int T, int D, float scale, int window,
                                float softcap, const float *sink, float *max_logit, forge_dtype dtype,
                                void *stream);

/*
 * Bytes of device workspace forge_attn_bwd needs for these sizes (0 on invalid
 * sizes). Holds rowsum(dO * o) as f32 and, for bf16, an f32 dq accumulator.
 */
size_t forge_attn_bwd_workspace_size(int B, int Hq, int Hkv, int T, int D, forge_dtype dtype);

/*
 * Backward. Given q, k, v, the o and lse of the matching forward call and the
 * upstream gradient dO, writes dq, dk, dv. `workspace` is caller-owned device
 * memory of at least forge_attn_bwd_workspace_size(...) bytes, 256-byte
 * aligned; its contents on entry do not matter and are overwritten.
 * Launches three kernels in order: forge_attn_bwd_preprocess,
 * forge_attn_bwd_main, forge_attn_bwd_finalize (below), on `stream`.
 */
forge_status forge_attn_bwd(const void *q, const void *k, const void *v, const void *o,
                            const float *lse, const void *dO, void *dq, void *dk, void *dv,
                            int B, int Hq, int Hkv, int T, int D, float scale, int window,
                            float softcap, forge_dtype dtype, void *workspace,
                            size_t workspace_bytes, void *stream);

/*
 * Backward of forge_attn_fwd_ext. `lse` (from that forward) already includes the
 * sink, which is all dq, dk and dv need of it. dsink [Hq] f32 (device, written;
 * NULL = not wanted; then sink may be NULL too) receives the gradient of the
 * loss with respect to sink[hq]: -sum over b and rows t of
 * exp(sink[hq] - lse[b][hq][t]) * Delta[b][hq][t], Delta = rowsum(dO * o) (the
 * sink's softmax column times (0 - Delta), the sink having no value vector).
 * With dsink non-NULL, sink must be non-NULL. Otherwise as forge_attn_bwd.
 */
forge_status forge_attn_bwd_ext(const void *q, const void *k, const void *v, const void *o,
                                const float *lse, const void *dO, void *dq, void *dk, void *dv,
                                int B, int Hq, int Hkv, int T, int D, float scale, int window,
                                float softcap, const float *sink, float *dsink, forge_dtype dtype,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * Backward for callers that cannot allocate device memory (no counterpart on
 * the Forge pages: it exists for callers, not for the method). Some hosts only
 * receive device buffers from another runtime and have no device allocator of
 * their own, or run in a process whose memory pool owns the whole device; they
 * cannot provide the workspace forge_attn_bwd needs. This entry point takes the
 * same arguments as forge_attn_bwd minus the workspace and uses scratch that
 * lives in a fixed 32 MiB device array inside the library instead (held by
 * every GPU that loads the library until the process exits). It allocates and
 * frees nothing.
 *  - Limit: forge_attn_bwd_workspace_size(B, Hq, Hkv, T, D, dtype) must be at
 *    most 32 MiB (33554432 bytes); larger problems return FORGE_ERR_WORKSPACE
 *    (forge_attn_last_cuda_error says why) and launch nothing.
 *  - The array's device address is looked up the first time the entry point is
 *    called with a given device current, and again on the first call after the
 *    device's context has changed (after a cudaDeviceReset, say), since the
 *    array moves with the context; make the first call on each device, and the
 *    first call after a reset, before any stream capture.
 *  - All calls share the one array per device. It keeps the previous call's
 *    contents; the call clears what must start at zero itself. Calls whose work
 *    overlaps on the GPU (other streams, other host threads) race on the array:
 *    serialise them.
 */
forge_status forge_attn_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                                    const float *lse, const void *dO, void *dq, void *dk, void *dv,
                                    int B, int Hq, int Hkv, int T, int D, float scale, int window,
                                    float softcap, forge_dtype dtype, void *stream);

/*
 * The three stages of forge_attn_bwd, callable one by one on the same stream
 * with the same arguments and workspace (used to time the stages separately).
 *  preprocess: Delta_i = sum_d dO_id o_id into the workspace (f32) and, for
 *              bf16, zeroes the dq accumulator;
 *  main:       recomputes P from q, k and lse, and produces dk, dv (written
 *              out) and dq (accumulated in the workspace for bf16; written
 *              out for f32);
 *  finalize:   bf16 only, converts the dq accumulator to dq (no-op for f32).
 */
forge_status forge_attn_bwd_preprocess(const void *o, const void *dO, int B, int Hq, int Hkv,
                                       int T, int D, forge_dtype dtype, void *workspace,
                                       size_t workspace_bytes, void *stream);
forge_status forge_attn_bwd_main(const void *q, const void *k, const void *v, const float *lse,
                                 const void *dO, void *dq, void *dk, void *dv, int B, int Hq,
                                 int Hkv, int T, int D, float scale, int window, float softcap,
                                 forge_dtype dtype, void *workspace, size_t workspace_bytes,
                                 void *stream);
forge_status forge_attn_bwd_finalize(void *dq, int B, int Hq, int Hkv, int T, int D,
                                     forge_dtype dtype, void *workspace, size_t workspace_bytes,
                                     void *stream);

/*
 * Forward and backward with separate head dims for q, k (Dk) and v, o (Dv):
 * decompressed multi-head latent attention (ARCHITECTURES.md "Vague 3" item 13;
 * family table, DeepSeek V3 row: q.k over nope 128 + rope 64 = 192, values 128,
 * scale 1/sqrt(192) chosen by the caller). Layouts as above with D = Dk for q,
 * k, dq, dk and D = Dv for v, o, dO, dv. With Dk == Dv these are forge_attn_fwd /
 * forge_attn_bwd. Otherwise only (Dk, Dv) = (192, 128) is built, forward and
 * backward, in bf16 (tensor cores) and f32 (CUDA cores); any other pair returns
 * FORGE_ERR_UNSUPPORTED. The workspace of the backward holds Delta only
 * (forge_attn_bwd_workspace_size_dkv bytes): both dtypes write dq directly. The
 * bf16 backward runs a dK/dV kernel (one CTA per key tile and KV head) and a dQ
 * kernel (one CTA per query tile and query head), each recomputing P.
 */
forge_status forge_attn_fwd_dkv(const void *q, const void *k, const void *v, void *o, float *lse,
                                int B, int Hq, int Hkv, int T, int Dk, int Dv, float scale, int window,
                                float softcap, forge_dtype dtype, void *stream);
size_t forge_attn_bwd_workspace_size_dkv(int B, int Hq, int Hkv, int T, int Dk, int Dv,
                                         forge_dtype dtype);
forge_status forge_attn_bwd_dkv(const void *q, const void *k, const void *v, const void *o,
                                const float *lse, const void *dO, void *dq, void *dk, void *dv,
                                int B, int Hq, int Hkv, int T, int Dk, int Dv, float scale,
                                int window, float softcap, forge_dtype dtype, void *workspace,
                                size_t workspace_bytes, void *stream);

/*
 * Decode: one new query per (batch entry, query head) against a KV cache
 * (INFERENCE_RESEARCH.md section 2: the cache is pre-allocated to the maximum
 * length, laid out [layer][head][seq][d], and decoding gets a dedicated kernel
 * with one query, split along the cache for long contexts).
 *   q, o               : [B][Hq][D] (dtype), the new token's queries / outputs
 *   k_cache, v_cache   : [B][Hkv][Tmax][D] (dtype), one layer's cache
 *   lse                : [B][Hq] f32 (may be NULL)
 *   seq_lens           : [B] int32 (device, may be NULL): entry b holds
 *                        seq_lens[b] valid positions, 1 <= seq_lens[b] <= T; NULL
 *                        means every entry holds T. Entry b's query sits at
 *                        position len - 1 and sees keys [len - window, len - 1]
 *                        clipped at 0 (window 0: all len), capped and scaled as in
 *                        the forward; sink (may be NULL) as in forge_attn_fwd_ext.
 *                        A length outside [1, T] is reported as
 *                        FORGE_ERR_INVALID_ARG by the next forge_attn_check.
 *   T <= Tmax; Hq / Hkv <= 16; D in {64, 128, 256}; dtype bf16 or f32.
 * workspace: device memory of at least forge_attn_decode_workspace_size(B, Hq,
 * Hkv, T, D) bytes, 16-byte aligned (per-chunk partial results), overwritten.
 * Two kernels on `stream`: the split pass (one CTA per key chunk, batch entry and
 * KV head, all of the group's query heads at once) and the combine pass.
 */
size_t forge_attn_decode_workspace_size(int B, int Hq, int Hkv, int T, int D);
forge_status forge_attn_decode(const void *q, const void *k_cache, const void *v_cache, void *o,
                               float *lse, const int *seq_lens, int B, int Hq, int Hkv, int T,
                               int Tmax, int D, float scale, int window, float softcap,
                               const float *sink, forge_dtype dtype, void *workspace,
                               size_t workspace_bytes, void *stream);

/*
 * Synchronises `stream`, then reports (and clears) the error a kernel of this
 * library recorded on the current device since the last check, or FORGE_OK:
 *   FORGE_ERR_TIMEOUT      a bounded wait inside a kernel ran out;
 *   FORGE_ERR_INVALID_ARG  a decode length outside [1, T] (forge_attn_decode);
 *   FORGE_ERR_UNSUPPORTED  the backward's shared-memory layout did not fit the
 *                          dynamic shared-memory base it was given (nothing written);
 *   FORGE_ERR_CUDA         an asynchronous CUDA error (forge_attn_last_cuda_error).
 */
forge_status forge_attn_check(void *stream);

/*
 * Text of the last CUDA runtime error that a call made on this host thread ran
 * into (the detail behind a FORGE_ERR_CUDA return); "no error" if none.
 * Static storage, never NULL.
 */
const char *forge_attn_last_cuda_error(void);

/*
 * Where the first bounded wait that ran out (FORGE_ERR_TIMEOUT) gave up, for
 * diagnosis, then cleared: info4[0] = 1 + the barrier's shared-memory address
 * (0 if no wait ran out), [1] = block index, [2] = thread index, [3] = (threads
 * per block << 20) | blocks in the grid. Host array of 4; synchronous.
 */
forge_status forge_attn_timeout_info(unsigned int *info4);

/* Human-readable name of a status code (static storage, never NULL). */
const char *forge_attn_status_string(forge_status s);

/*
 * Self-test of the bounded-wait machinery: launches one tiny kernel that waits
 * on a barrier nothing will ever complete, with a wait limit of `limit_us`
 * microseconds (1..2000000). The wait runs out, the kernel records
 * FORGE_ERR_TIMEOUT and returns normally, leaving the context usable; the next
 * forge_attn_check reports it. Used by the tests of failure detection.
 */
forge_status forge_attn_selftest_timeout(unsigned int limit_us, void *stream);

/*
 * Self-test of the FMA-pipe exponential the kernels use for part of their
 * exp2 work (Cody-Waite reduction + degree-4 minimax polynomial): for each of
 * the n device floats x[i], writes that exp2 to y[i] and CUDA's exp2f(x[i]) to
 * y_ref[i]. Device pointers, asynchronous on `stream`. Used by the tests.
 */
forge_status forge_attn_selftest_exp2(const float *x, float *y, float *y_ref, int n, void *stream);

/* Library version, e.g. "forge_attn 0.1.0 sm_100a". */
const char *forge_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FORGE_ATTN_H */
