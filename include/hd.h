/*
 * hd.h - C ABI of the Hidden Decoding hot-path library (B200, sm_100a).
 *
 * The method (page "微信WeLM提出Hidden Decoding：大模型推理新范式", tahou.com):
 *   - section "隐式序列缩放的技术细节", step 1: each token is expanded into n
 *     streams; stream k of token i takes its input from the k-th of n embedding
 *     tables and sits at physical position (i-1)n+k of an nL-long sequence.
 *     0-based throughout this library: p = t*n + s, token(p) = p / n,
 *     stream(p) = p % n.
 *   - step 2: the expanded sequence runs through the unchanged Transformer with
 *     causal attention and continuous positions: the position encoding runs
 *     over the physical position p (hd_rope_expanded applies rotary encoding
 *     there).
 *   - section "规模化落地的工程优化": Stream-Factorized Attention. Intra-stream
 *     layers see only earlier positions of the same stream; cross-stream layers
 *     keep the base model's full-causal or sliding-window attention over the
 *     whole expanded sequence. KV-mirror: only the final stream's queries pass
 *     through the mirror layers and read K/V built for all n streams.
 *   - section "实验效果与成本分析": at decode the n streams of a new token are
 *     computed in one parallel step; the cache keeps K/V for every stream
 *     (page "WeLM ...", aiflownews.com, "Latent computation scaling and Hidden
 *     Decoding").
 *
 * Visibility rule (query at position p, key at position p'):
 *   HD_INTRA        p' <= p  and  p' % n == p % n        (self included)
 *   HD_CROSS_FULL   p' <= p
 *   HD_CROSS_WINDOW p' <= p  and  p - p' < n * W_tokens  (W counted in tokens)
 *
 * Conventions shared by every entry point
 *   - Every pointer is DEVICE memory owned by the caller; tensors are dense and
 *     row-major in the layouts stated below. "bf16" buffers hold IEEE bfloat16
 *     bit patterns (2 bytes each). Pointers must be 16-byte aligned.
 *   - The library allocates no memory and keeps no per-call state; scratch
 *     space ("workspace") is passed in by the caller, sized by the matching
 *     *_workspace_bytes() function.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream). Every call only enqueues work on that stream and returns.
 *   - Argument errors are reported (HD_ERR_INVALID_ARG / HD_ERR_UNSUPPORTED)
 *     before anything is launched. A failed launch returns HD_ERR_CUDA.
 *     Errors found on the device (a token id, label, sequence length or token
 *     offset out of range, a bounded wait that gave up) are recorded in a
 *     per-device status word, read and cleared with hd_device_status();
 *     kernels never trap.
 */
#ifndef HD_H_
#define HD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HD_OK = 0,
  HD_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad mode, ... */
  HD_ERR_UNSUPPORTED = 2, /* valid arguments this build does not cover (e.g. D not in {64,128}) */
  HD_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  HD_ERR_TIMEOUT = 4,     /* device status: a bounded wait inside a kernel gave up */
  HD_ERR_DEVICE_INDEX = 5 /* device status: an index read on the device was out of range (a token
                             id, seqlen, label or offset; in the checked build also a computed
                             load/store index) */
} hd_status;

typedef enum { HD_INTRA = 0, HD_CROSS_FULL = 1, HD_CROSS_WINDOW = 2 } hd_mode;

/* Human-readable name of a status code (static string, never NULL). */
const char* hd_status_string(int status);

/* Library ABI version: (major << 16) | minor. Minor 1 added RoPE, the
 * final-stream readout, the LM-head cross-entropy and its gradients,
 * final-stream-only decode and the bounded-wait self-test; minor 2 added
 * hd_build_flags. */
int hd_version(void);

/* How this copy of the library was built (no counterpart on the pages), a bit
 * mask: HD_BUILD_CHECK_BOUNDS is set in the checked build (libhd_checked.so,
 * compiled with HD_CHECK_BOUNDS), whose kernels test every computed index of a
 * plain (non-TMA) load or store against the size of its buffer. An index out
 * of range records HD_ERR_DEVICE_INDEX in the device status word and its access
 * is skipped; nothing traps. The normal build (libhd.so) has no such checks. */
#define HD_BUILD_CHECK_BOUNDS 1
int hd_build_flags(void);

/*
 * hd_expand_embed - interleaved n-table embedding gather.
 * Source: tahou.com page, "隐式序列缩放的技术细节" step 1; aiflownews.com page,
 * "Latent computation scaling and Hidden Decoding" (one table per stream).
 *
 *   out[b, t*n + s, :] = tables[s, ids[b, t], :]      (exact copy of the bytes)
 *
 *   ids     int32 [B, L]           token ids, must lie in [0, V)
 *   tables  [n, V, d] elements of `elem_bytes` bytes (fp32: 4, bf16/fp16: 2)
 *   out     [B, L*n, d] same element type
 * An id outside [0, V) leaves its n output rows zero and records
 * HD_ERR_DEVICE_INDEX in the device status word.
 */
int hd_expand_embed(const int32_t* ids, const void* tables, void* out, int B, int L, int n,
                    int V, int d, int elem_bytes, void* stream);

/*
 * hd_rope_expanded - rotary position embedding at the physical positions.
 * Source: tahou.com page, "隐式序列缩放的技术细节" step 2 (the expanded
 * sequence keeps continuous position encoding). The page does not name the
 * encoding; this is the rotary form with rotate-half pairing:
 *
 *   w_i = base^(-2i/D),  i = 0 .. D/2-1,  angle = p * w_i
 *   x[i]       <- x[i] cos(angle) - x[i + D/2] sin(angle)
 *   x[i + D/2] <- x[i + D/2] cos(angle) + x[i] sin(angle)
 *
 * applied IN PLACE to every head of the rows of q and k, where p is the
 * row's physical position: with t0 = token_offset[b] (0 if token_offset is
 * NULL), row r of k (and of q) is at p = t0*n + r; with
 * final_stream_queries_only, q row t is at p = (t0 + t)*n + n-1.
 *
 *   q            bf16 [B, S, Hq, D] (S = n*L), or [B, L, Hq, D] with
 *                final_stream_queries_only; NULL skips q
 *   k            bf16 [B, S, Hkv, D]; NULL skips k (not both NULL)
 *   token_offset int32 [B] on the device, or NULL: tokens of sequence b that
 *                precede this call (a decode step passes L = 1 and the
 *                cached token count). A negative entry leaves that
 *                sequence's rows unchanged and records HD_ERR_DEVICE_INDEX.
 *   base         > 1 (10000 in most models)
 * Supported: D in {16, 32, 64, 128, 256}. The angle is formed and reduced in
 * fp64, its sine and cosine taken in fp32; the product is rounded to bf16.
 */
int hd_rope_expanded(void* q, void* k, const int32_t* token_offset, int B, int L, int n, int Hq,
                     int Hkv, int D, int final_stream_queries_only, double base, void* stream);

/*
 * hd_final_readout - the final stream's rows of the expanded sequence.
 * Source: tahou.com page, "隐式序列缩放的技术细节" step 3 (the loss is taken
 * only on the last stream of every token).
 *
 *   out[b, t, :] = x[b, t*n + n-1, :]        (exact copy of the bytes)
 *
 *   x    [B, n*L, d] elements of `elem_bytes` bytes; out [B, L, d]
 * Supported: d * elem_bytes a multiple of 16.
 */
int hd_final_readout(const void* x, void* out, int B, int L, int n, int d, int elem_bytes,
                     void* stream);

/* Bytes of workspace hd_lm_head_ce needs (0 on invalid sizes). */
size_t hd_lm_head_ce_workspace_bytes(int B, int L, int V);

/*
 * hd_lm_head_ce - LM-head cross-entropy on the final stream, fused.
 * Source: tahou.com page, "隐式序列缩放的技术细节" step 3: only each token's
 * last stream is supervised with the next-token loss; streams 0..n-2 get no
 * direct supervision. The page gives no formula; this is the plain linear
 * head and softmax cross-entropy:
 *
 *   h_r    = x[b, t*n + n-1, :]           (r = b*L + t; read in place)
 *   lse_r  = ln sum_v exp(h_r . w_v)
 *   loss_r = lse_r - h_r . w_{labels[r]}
 *
 *   x       bf16 [B, n*L, d]: hidden states of the expanded sequence
 *   w       bf16 [V, d]: the LM head (no bias)
 *   labels  int32 [B, L]: target of each token, already shifted by the caller;
 *           a negative label marks a token without a target (loss 0). A
 *           label >= V gives loss 0 and records HD_ERR_DEVICE_INDEX.
 *   loss    fp32 [B, L]; lse fp32 [B, L] or NULL
 * The logits are never written to memory: products are accumulated in fp32
 * on the tensor cores and reduced to (max, sum of exp) per 256-wide
 * vocabulary tile. Supported: d a multiple of 64.
 * `workspace` must hold hd_lm_head_ce_workspace_bytes(B, L, V) bytes.
 */
int hd_lm_head_ce(const void* x, const void* w, const int32_t* labels, float* loss, float* lse,
                  int B, int L, int n, int d, int V, void* workspace, size_t workspace_bytes,
                  void* stream);

/* Bytes of workspace hd_lm_head_ce_bwd needs (0 on invalid sizes). */
size_t hd_lm_head_ce_bwd_workspace_bytes(int B, int L, int V);

/*
 * hd_lm_head_ce_bwd - gradients of the final-stream LM-head cross-entropy.
 * Source: as hd_lm_head_ce (tahou.com page, "隐式序列缩放的技术细节" step 3).
 *
 * For the summed loss sum_r loss_r (tokens without a target contribute
 * nothing), with G_r = softmax(h_r W^T) - onehot(labels[r]) (G_r = 0 when
 * labels[r] < 0):
 *
 *   dh = grad_scale * G W      bf16 [B, L, d]: gradient w.r.t. the final-
 *                              stream rows h (dX[b, t*n+n-1] = dh[b, t]; the
 *                              other streams' rows of dX are zero)
 *   dw = grad_scale * G^T h    fp32 [V, d]
 *
 *   x, w, labels  as hd_lm_head_ce; lse fp32 [B, L] from that call
 *   grad_scale    e.g. 1 / (number of supervised tokens) for a mean loss
 * G is recomputed from x and w (its logits on the tensor cores, fp32) and
 * stored once as bf16 in the workspace; the two products accumulate in fp32.
 * Supported: d a multiple of 64. `workspace` must hold
 * hd_lm_head_ce_bwd_workspace_bytes(B, L, V) bytes (B*L rows of G, V rounded
 * up to 256 columns).
 */
int hd_lm_head_ce_bwd(const void* x, const void* w, const int32_t* labels, const float* lse,
                      float grad_scale, void* dh, float* dw, int B, int L, int n, int d, int V,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * hd_attn_fwd - Stream-Factorized attention forward.
 * Source: tahou.com page, "规模化落地的工程优化" (intra / cross-stream bullets,
 * KV-mirror paragraph); "隐式序列缩放的技术细节" step 2 (causal attention).
 *
 *   O[p] = sum_{p' visible from p} softmax_p'(scale * q_p . k_p') v_p'
 *   lse[p] = ln sum_{p' visible} exp(scale * q_p . k_p')
 *
 *   q    bf16 [B, S, Hq, D]   (S = n*L); with final_stream_queries_only:
 *        bf16 [B, L, Hq, D], row t is the query at position t*n + n-1
 *   k, v bf16 [B, S, Hkv, D]  (Hq % Hkv == 0; query head h reads KV head
 *        h / (Hq/Hkv))
 *   out  bf16, same shape as q
 *   lse  fp32 [B, Hq, S] or [B, Hq, L] with final_stream_queries_only
 *   mode hd_mode; W_tokens is the window in tokens (used by HD_CROSS_WINDOW
 *        only, must be >= 1 there); scale is the softmax scale (> 0).
 * Supported: D in {64, 128}. Accumulation is fp32; out is rounded to bf16.
 */
int hd_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int L,
                int n, int Hq, int Hkv, int D, int mode, int W_tokens,
                int final_stream_queries_only, float scale, void* stream);

/* Bytes of workspace hd_attn_bwd needs for these sizes (0 on invalid sizes). */
size_t hd_attn_bwd_workspace_bytes(int B, int L, int n, int Hq, int Hkv, int D,
                                   int final_stream_queries_only);

/*
 * hd_attn_bwd - gradients of Stream-Factorized attention.
 * Same source and arguments as hd_attn_fwd; out and lse are that call's
 * outputs, dout has out's shape. Writes
 *   dq (q's shape), dk, dv (k's shape), all bf16:
 *   D_i = sum_d dO_id O_id, dP = dO V^T, dS = P * (dP - D),
 *   dQ = scale dS K, dK = scale sum_{group} dS^T Q, dV = sum_{group} P^T dO.
 * `workspace` must hold hd_attn_bwd_workspace_bytes(...) bytes of device
 * memory (fp32 dQ accumulator and the D vector); its contents on entry do
 * not matter and are overwritten.
 */
int hd_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                const void* dout, void* dq, void* dk, void* dv, int B, int L, int n, int Hq,
                int Hkv, int D, int mode, int W_tokens, int final_stream_queries_only,
                float scale, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace hd_decode_attn needs for these sizes (0 on invalid sizes). */
size_t hd_decode_workspace_bytes(int B, int n, int Tcap, int Hq, int Hkv, int D);

/*
 * hd_decode_attn - one decode step of the n streams of a new token.
 * Source: tahou.com page, "实验效果与成本分析" (the n streams are computed in
 * one parallel forward; decode is bandwidth-bound at small batch) and
 * "中间流的作用验证" (each stream keeps its own KV state).
 *
 *   q        bf16 [B, n, Hq, D]: the new token's n stream queries
 *   k_cache, v_cache bf16 [B, Tcap*n, Hkv, D]: the expanded sequence in
 *            position order. PRECONDITION: the new token's n K/V rows are
 *            already written at positions T*n .. T*n+n-1, T = seqlen[b]-1.
 *   seqlen   int32 [B] tokens per sequence INCLUDING the new one,
 *            1 <= seqlen[b] <= Tcap (read on the device)
 *   out      bf16 [B, n, Hq, D]; lse fp32 [B, Hq, n]
 * Query s of sequence b sits at p = T*n + s and reads the cache positions
 * the mode's visibility rule allows.
 * `workspace` must hold hd_decode_workspace_bytes(...) bytes.
 * A seqlen outside [1, Tcap] leaves that sequence's rows zero and records
 * HD_ERR_DEVICE_INDEX in the device status word.
 */
int hd_decode_attn(const void* q, const void* k_cache, const void* v_cache, const int32_t* seqlen,
                   void* out, float* lse, int B, int n, int Tcap, int Hq, int Hkv, int D, int mode,
                   int W_tokens, float scale, void* workspace, size_t workspace_bytes,
                   void* stream);

/* Bytes of workspace hd_decode_attn_final needs for these sizes, whatever the
 * mode (0 on invalid sizes). */
size_t hd_decode_final_workspace_bytes(int B, int n, int Tcap, int Hq, int Hkv, int D);

/*
 * hd_decode_attn_final - final-stream-only decode (KV-mirror layers).
 * Source: tahou.com page, "规模化落地的工程优化", KV-mirror paragraph (only the
 * last stream passes through the mirror layers, which read K/V built for all
 * streams).
 *
 * As hd_decode_attn, with one query per sequence: stream n-1 of the new
 * token, at p = T*n + n-1.
 *   q    bf16 [B, 1, Hq, D] (equivalently [B, Hq, D])
 *   out  bf16 [B, 1, Hq, D]; lse fp32 [B, Hq] (= [B, Hq, 1])
 *   k_cache, v_cache, seqlen, mode, W_tokens, scale: as hd_decode_attn
 *        (same precondition: the new token's n K/V rows are in the cache).
 * Under HD_INTRA only the final stream's cache rows (positions n-1, 2n-1, ...)
 * are read. `workspace` must hold hd_decode_final_workspace_bytes(...) bytes.
 */
int hd_decode_attn_final(const void* q, const void* k_cache, const void* v_cache,
                         const int32_t* seqlen, void* out, float* lse, int B, int n, int Tcap,
                         int Hq, int Hkv, int D, int mode, int W_tokens, float scale,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * hd_decode_attn_noalloc - hd_decode_attn for callers that cannot allocate.
 * The pages have no counterpart: this is a deployment convenience.
 *
 * Some callers may not allocate device memory while they decode (a host
 * framework that owns all GPU memory through its own pool, or a latency-bound
 * loop that must not enter cudaMalloc, which can synchronise the device).
 * This entry point takes the same arguments as hd_decode_attn minus the
 * workspace, computes the same result, and keeps its split-K scratch in a
 * fixed array of HD_DECODE_NOALLOC_SCRATCH_BYTES compiled into the library
 * (held by every GPU that loads the library until the process exits). It
 * allocates nothing and calls no allocating routine.
 *   - Sizes whose hd_decode_workspace_bytes(...) exceeds
 *     HD_DECODE_NOALLOC_SCRATCH_BYTES are rejected with HD_ERR_UNSUPPORTED.
 *   - Every call looks up the array's device address on the calling device
 *     (cudaGetSymbolAddress, which allocates nothing) before it launches. The
 *     first call on a device may also load the library's device code there:
 *     make that first call before any stream capture.
 *   - All calls on a device share the array, which keeps the last call's
 *     contents; nothing in it needs to start at zero. Calls that overlap on
 *     the GPU (two streams, or unordered host threads) race on it: order them.
 */
#define HD_DECODE_NOALLOC_SCRATCH_BYTES (16u << 20)
int hd_decode_attn_noalloc(const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* seqlen, void* out, float* lse, int B, int n, int Tcap,
                           int Hq, int Hkv, int D, int mode, int W_tokens, float scale,
                           void* stream);

/*
 * hd_selftest_wait_timeout - test the bounded-wait failure path (no fault).
 * Launches one thread that waits, through the same bounded wait the
 * tensor-core kernels use, on a barrier nothing will complete, giving up after
 * `limit_cycles` SM cycles (1 .. 2^33). Afterwards the device status word reads
 * HD_ERR_TIMEOUT (hd_device_status), and until it is cleared the tensor-core
 * kernels (hd_attn_fwd, hd_attn_bwd, hd_lm_head_ce) return without doing their
 * work, as they would after a real timeout.
 */
int hd_selftest_wait_timeout(long long limit_cycles, void* stream);

/*
 * Read (and, if `clear` is non-zero, reset) the device status word of the
 * current device. Synchronizes `stream` first. Returns HD_OK when no kernel
 * recorded an error since the last clear, else the first recorded code.
 */
int hd_device_status(void* stream, int clear);

#ifdef __cplusplus
}
#endif

#endif /* HD_H_ */
