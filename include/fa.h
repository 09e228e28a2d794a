/*
 * fa.h -- exact IO-aware attention for NVIDIA B200 (sm_100a).  C ABI.
 *
 * Every call computes exact scaled-dot-product attention
 *
 *     O = softmax(Q K^T * scale + mask) V ,    LSE = log sum_j exp(s_ij)
 *
 * ("What attention costs", samanvya.dev "Attention Is the Bottleneck": the
 * one-line definition softmax(QK^T/sqrt d)V, with 1/sqrt(d) generalised to
 * `scale` and an additive mask that is 0 on the allowed keys and -inf
 * elsewhere), tile by tile with an online softmax so the N x N score matrix
 * never reaches device memory ("FlashAttention: same math, different IO").
 * Results equal the plain definition up to floating-point rounding order.
 *
 * Conventions shared by every call
 *   - q, k, v, o, caches: bf16 (o optionally fp32), innermost dimension
 *     contiguous, token-major:  dense [B, N, H, d], packed [total, H, d],
 *     cache [num_pages, page_size, Hkv, d].  The FP8 calls
 *     (fa_decode_paged_fp8, fa_fp8_prepare, fa_fwd_fp8) take E4M3 codes with
 *     fp32 scales instead; their comments give the layouts.
 *   - GQA ("MQA and GQA"): query head h reads KV head h / (Hq / Hkv);
 *     Hq must be a multiple of Hkv; Hkv == 1 is MQA.
 *   - Masks: causal (key j visible from query i iff j <= i; "every token can
 *     see every earlier token"), sliding window W > 0 (with causal only: keys
 *     i-W+1 .. i, i.e. W keys ending at the query itself;
 *     "Sliding windows and local:global layers").  window <= 0: no window.
 *   - LSE is natural-log, in units of scaled scores; a row with no visible
 *     key (only possible for an empty sequence) has O = 0 and LSE = -inf.
 *   - head dim d in {64, 128}.
 *   - Every device pointer must be 16-byte aligned (TMA requirement);
 *     row strides are implied by the shapes.
 *   - Ownership: the caller owns every buffer.  No call allocates device
 *     memory or keeps per-call state, and calls are thread-safe (see
 *     fa_decode_paged_noalloc for its one fixed, library-owned scratch array).
 *     All calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and do not synchronise.
 *   - Errors: the return value is FA_OK (0) or a negative FA_ERR_* code.  On
 *     an argument error nothing is launched.  FA_ERR_CUDA reports a launch
 *     error (cudaGetLastError).  There is no CPU fallback: host pointers are
 *     not detected and passing them is undefined behaviour.
 *   - Device-side watchdog: every wait inside a kernel is bounded (about a
 *     second).  A wait that runs out records an error word and the kernel
 *     returns early; fa_check_device_error() reads and clears that word.
 */
#ifndef FA_SM100_H
#define FA_SM100_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

enum fa_status {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = -1,  /* null pointer, bad shape, Hq % Hkv != 0, ... */
    FA_ERR_UNSUPPORTED = -2,  /* valid but not implemented: d, page size, window without causal */
    FA_ERR_ALIGNMENT = -3,    /* a pointer is not 16-byte aligned */
    FA_ERR_WORKSPACE = -4,    /* workspace missing or smaller than required */
    FA_ERR_CUDA = -5,         /* the CUDA runtime reported an error */
    FA_ERR_TIMEOUT = -6       /* a device-side wait ran out (fa_check_device_error) */
};

enum fa_out_dtype { FA_OUT_BF16 = 0, FA_OUT_FP32 = 1 };

/*
 * Dense prefill ("FlashAttention: same math, different IO": a Q tile stays
 * on chip while K/V tiles stream past it; "FlashAttention-2": parallel over
 * sequence blocks too, normalise once at the end; "FlashAttention-4":
 * conditional rescaling, tensor memory).
 *   q      [B, N, Hq, d]  bf16, device
 *   k, v   [B, N, Hkv, d] bf16, device
 *   o      [B, N, Hq, d]  bf16 (o_dtype = FA_OUT_BF16) or fp32, device, written
 *   lse    [B, Hq, N]     fp32, device, written; may be NULL
 *   causal 0/1; window as above (requires causal); scale > 0 finite.
 * N == 0 or B == 0 is a no-op returning FA_OK.
 */
int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
           int B, int Hq, int Hkv, int N, int d, int causal, int window,
           float scale, int o_dtype, void *stream);

/*
 * Packed variable-length prefill: num_seqs sequences concatenated along the
 * token axis; each sequence attends only to itself (a document mask,
 * "FlexAttention" on the Ales Analytics kernels page).
 *   q          [total_tokens, Hq, d]  bf16, device
 *   k, v       [total_tokens, Hkv, d] bf16, device
 *   o          [total_tokens, Hq, d]  bf16 or fp32, device, written
 *   lse        [Hq, total_tokens]     fp32, device, written; may be NULL
 *   cu_seqlens [num_seqs + 1] int32, device: 0 = cu[0] <= cu[1] <= ... =
 *              total_tokens (prefix sums of the lengths).  Empty sequences are
 *              allowed and write nothing.
 *   max_seqlen >= every sequence length (sizes the launch).
 * Device-side input errors: a sequence longer than max_seqlen, or one that
 * does not lie inside [0, total_tokens) (offsets not ascending, or past the
 * end), is skipped -- none of its rows is read or written -- and reported
 * through fa_check_device_error as FA_ERR_INVALID_ARG.  The other sequences
 * are computed as usual.
 */
int fa_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                  const int *cu_seqlens, int num_seqs, int total_tokens,
                  int max_seqlen, int Hq, int Hkv, int d, int causal, int window,
                  float scale, int o_dtype, void *stream);

/*
 * Chunked prefill over a paged cache (zenaique's FlashAttention serving
 * explainer, "Real-world examples": serving engines run long prompts in chunks
 * over a paged KV cache with this kernel).  Sequence s has seq_lens_k[s] tokens in its pages -- the earlier
 * context plus this chunk, whose K/V the caller has already written -- and
 * its L_q = cu_seqlens_q[s+1] - cu_seqlens_q[s] queries are the LAST L_q of
 * them: query i of the chunk sits at position seq_lens_k[s] - L_q + i and,
 * with causal, sees keys 0 .. seq_lens_k[s] - L_q + i (window W: the last W
 * of those).  L_q = 1 is the decode; L_q = seq_lens_k is a plain prefill.
 *   q            [total_q, Hq, d] bf16, device (chunks packed by cu_seqlens_q)
 *   k_cache,
 *   v_cache      [num_pages, page_size, Hkv, d] bf16, device
 *   block_table  [num_seqs, max_pages_per_seq] int32, device (as fa_decode_paged)
 *   cu_seqlens_q [num_seqs + 1] int32, device; seq_lens_k [num_seqs] int32,
 *                device, with L_q <= seq_lens_k[s] <= max_pages_per_seq * 16
 *                (a sequence that breaks this is skipped, its rows left
 *                unwritten, and fa_check_device_error reports
 *                FA_ERR_INVALID_ARG)
 *   o            [total_q, Hq, d] bf16 or fp32, written; lse [Hq, total_q] or NULL
 *   sinks        [Hq] fp32 learned sink logits, or NULL (as fa_fwd_sinks)
 *   page_size    16.  max_seqlen_q >= every L_q.
 * Cache slots past seq_lens_k may hold anything, NaN included.
 */
int fa_fwd_paged(const void *q, const void *k_cache, const void *v_cache,
                 const int *block_table, const int *cu_seqlens_q, const int *seq_lens_k,
                 void *o, float *lse, const float *sinks, int num_seqs, int total_q,
                 int max_seqlen_q, int num_pages, int Hq, int Hkv, int d, int page_size,
                 int max_pages_per_seq, int causal, int window, float scale, int o_dtype,
                 void *stream);

/*
 * Bytes of workspace fa_bwd / fa_bwd_varlen need for total_tokens tokens
 * (B * N for a dense batch): an fp32 dQ accumulator [total, Hq, d] and the
 * row terms D_i = dO_i . O_i.  0 for an unsupported combination (d not 64
 * or 128).
 */
size_t fa_bwd_workspace_bytes(int total_tokens, int Hq, int d);

/*
 * fa_fwd with a document mask in any form ("FlexAttention" on the Ales
 * Analytics kernels page: document masks among the attention variants).
 *   doc_ids [B, N] int32, device: a document id per token; key j is visible
 *           from query i only if doc_ids[b][i] == doc_ids[b][j], on top of the
 *           causal / window rule.  A document's tokens need not be contiguous
 *           (for contiguous documents fa_fwd_varlen does less work: here every
 *           key block the causal / window rule admits is computed).
 * Other arguments, layouts and errors as for fa_fwd; doc_ids non-NULL and
 * 4-byte aligned.
 */
int fa_fwd_doc(const void *q, const void *k, const void *v, void *o, float *lse,
               const int *doc_ids, int B, int Hq, int Hkv, int N, int d, int causal,
               int window, float scale, int o_dtype, void *stream);

/*
 * fa_fwd / fa_fwd_varlen with a learned attention sink per query head
 * ("Sliding windows and local:global layers": gpt-oss builds one into every
 * head).  sinks [Hq] fp32, device, in units of scaled scores: z_h joins every
 * row's softmax denominator as the score of one extra key whose value is
 * zero, so O_i = sum_j e^(s_ij) V_j / (e^(z_h) + sum_j e^(s_ij)) and LSE
 * includes the e^(z_h) term.  -INFINITY for a head means no sink.  Other
 * arguments, layouts and errors as for fa_fwd / fa_fwd_varlen; sinks must be
 * non-NULL and 4-byte aligned.  fa_bwd accepts the LSE these calls write (the
 * sink enters the gradients of Q, K, V only through it).
 */
int fa_fwd_sinks(const void *q, const void *k, const void *v, void *o, float *lse,
                 const float *sinks, int B, int Hq, int Hkv, int N, int d, int causal,
                 int window, float scale, int o_dtype, void *stream);
int fa_fwd_varlen_sinks(const void *q, const void *k, const void *v, void *o, float *lse,
                        const float *sinks, const int *cu_seqlens, int num_seqs,
                        int total_tokens, int max_seqlen, int Hq, int Hkv, int d, int causal,
                        int window, float scale, int o_dtype, void *stream);

/*
 * Backward of dense prefill: the gradients of sum(dO * O) with respect to Q,
 * K and V, for O = fa_fwd(q, k, v, ...) with the same mask and scale.  The
 * attention matrix is recomputed tile by tile from Q, K and the LSE the
 * forward saved, never stored (samanvya.dev "Attention Is the Bottleneck",
 * "FlashAttention: same math, different IO": the backward rebuilds the
 * matrix rather than keeping it).  With grouped heads, dK and dV of a KV head sum
 * over the query heads that read it.
 *   q, o, dout [B, N, Hq, d]  bf16, device (o as written by fa_fwd)
 *   k, v       [B, N, Hkv, d] bf16, device
 *   lse        [B, Hq, N]     fp32, device: the forward's LSE (natural log)
 *   dq         [B, N, Hq, d]  bf16, device, written
 *   dk, dv     [B, N, Hkv, d] bf16, device, written
 *   workspace  device scratch of at least fa_bwd_workspace_bytes(B * N, Hq, d)
 *              bytes, 256-byte aligned; contents on entry do not matter; not
 *              to be shared by calls that may overlap on the GPU.
 *   causal, window, scale as for fa_fwd.  d = 64 or 128 (a head dim of 64 is
 *   computed on 128-wide tiles with zero padding, at the cost of 128).
 *   N == 0 or B == 0 is a no-op returning FA_OK.
 * dQ is accumulated in fp32 with atomic adds, so its last bits may differ
 * from run to run; dK and dV are deterministic.
 */
int fa_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
           const float *lse, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int N,
           int d, int causal, int window, float scale, void *workspace,
           size_t workspace_bytes, void *stream);

/*
 * fa_bwd / fa_bwd_varlen for a forward run with learned sinks (fa_fwd_sinks,
 * fa_fwd_varlen_sinks): lse is that forward's LSE (it includes the sink
 * term), so dQ, dK, dV follow as without sinks; additionally
 * dsinks [Hq] fp32, device, written = d Loss / d z_h = sum over the rows of
 * head h of exp(z_h - LSE_i) * (0 - D_i), D_i = dO_i . O_i (the sink is one
 * more score with a zero value).  sinks and dsinks must be non-NULL and
 * 4-byte aligned; other arguments as for fa_bwd / fa_bwd_varlen.
 */
int fa_bwd_sinks(const void *q, const void *k, const void *v, const void *o, const void *dout,
                 const float *lse, const float *sinks, void *dq, void *dk, void *dv,
                 float *dsinks, int B, int Hq, int Hkv, int N, int d, int causal, int window,
                 float scale, void *workspace, size_t workspace_bytes, void *stream);
int fa_bwd_varlen_sinks(const void *q, const void *k, const void *v, const void *o,
                        const void *dout, const float *lse, const float *sinks, void *dq,
                        void *dk, void *dv, float *dsinks, const int *cu_seqlens, int num_seqs,
                        int total_tokens, int max_seqlen, int Hq, int Hkv, int d, int causal,
                        int window, float scale, void *workspace, size_t workspace_bytes,
                        void *stream);

/*
 * Backward of packed variable-length prefill (fa_fwd_varlen's layouts: q, o,
 * dout, dq [total, Hq, d]; k, v, dk, dv [total, Hkv, d]; lse [Hq, total];
 * cu_seqlens as there).  Workspace: fa_bwd_workspace_bytes(total_tokens, Hq, d).
 * A sequence longer than max_seqlen or outside [0, total_tokens) is skipped
 * (its dK, dV rows unwritten, no dQ contribution) and reported through
 * fa_check_device_error as FA_ERR_INVALID_ARG, as for fa_fwd_varlen.
 */
int fa_bwd_varlen(const void *q, const void *k, const void *v, const void *o,
                  const void *dout, const float *lse, void *dq, void *dk, void *dv,
                  const int *cu_seqlens, int num_seqs, int total_tokens, int max_seqlen,
                  int Hq, int Hkv, int d, int causal, int window, float scale,
                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * Bytes of workspace fa_decode_paged needs for these sizes (split-KV
 * partial outputs and their log-sum-exps).  0 for an invalid combination.
 */
size_t fa_decode_workspace_bytes(int num_seqs, int Hq, int d, int page_size,
                                 int max_pages_per_seq);

/*
 * Paged split-KV decode: one query token per sequence, at position
 * seq_len - 1, attending to all seq_len cached keys ("Flash-Decoding": split
 * the cache along the sequence, attend to the chunks in parallel, merge the
 * partial results with log-sum-exp; "Paging and prefix sharing": the cache
 * lives in fixed-size pages reached through a block table).
 *   q           [num_seqs, Hq, d] bf16, device
 *   k_cache,
 *   v_cache     [num_pages, page_size, Hkv, d] bf16, device
 *   block_table [num_seqs, max_pages_per_seq] int32, device; entry p of
 *               sequence s is the page holding its tokens p*page_size ..
 *               p*page_size + page_size-1; entries past ceil(seq_len /
 *               page_size) are never read.  Every read entry must lie in
 *               [0, num_pages).
 *   seq_lens    [num_seqs] int32, device; 0 <= seq_len <= max_pages_per_seq *
 *               page_size.  Cache slots past seq_len are never used in the
 *               result (they may hold anything, NaN included).
 *   o           [num_seqs, Hq, d] bf16, device, written
 *   lse         [num_seqs, Hq] fp32, device, written; may be NULL
 *   workspace   device scratch of at least fa_decode_workspace_bytes(...)
 *               bytes, 256-byte aligned; contents on entry do not matter;
 *               it must not be shared by calls that may overlap on the GPU.
 *   page_size   16 (others return FA_ERR_UNSUPPORTED).
 */
int fa_decode_paged(const void *q, const void *k_cache, const void *v_cache,
                    const int *block_table, const int *seq_lens, void *o,
                    float *lse, int num_seqs, int num_pages, int Hq, int Hkv,
                    int d, int page_size, int max_pages_per_seq, float scale,
                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * fa_decode_paged with a learned attention sink per query head (sinks [Hq]
 * fp32, device; meaning as for fa_fwd_sinks).  A sequence of length 0 then
 * gets O = 0 and LSE = z_h.
 */
int fa_decode_paged_sinks(const void *q, const void *k_cache, const void *v_cache,
                          const int *block_table, const int *seq_lens, void *o, float *lse,
                          const float *sinks, int num_seqs, int num_pages, int Hq, int Hkv,
                          int d, int page_size, int max_pages_per_seq, float scale,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * fa_decode_paged over an FP8 cache ("FP8 KV cache": the post's cache-size
 * paragraphs before "Paging and prefix sharing" -- fewer bits per cached
 * value).  k_cache/v_cache [num_pages, page_size, Hkv, d] hold OCP FP8 E4M3
 * codes (the "fn" variant, one byte each); the cached value is
 * e4m3(code) * scale with k_scale/v_scale [num_pages, Hkv] fp32, device (one
 * scale per page and KV head; a per-head scale is the case of equal page
 * scales).  sinks [Hq] or NULL (as fa_decode_paged_sinks).  Halves the bytes
 * read per token.  Other arguments, the workspace and errors as for
 * fa_decode_paged; codes of unused slots may hold anything, NaN included.
 */
int fa_decode_paged_fp8(const void *q, const void *k_cache, const void *v_cache,
                        const float *k_scale, const float *v_scale, const int *block_table,
                        const int *seq_lens, void *o, float *lse, const float *sinks,
                        int num_seqs, int num_pages, int Hq, int Hkv, int d, int page_size,
                        int max_pages_per_seq, float scale, void *workspace,
                        size_t workspace_bytes, void *stream);

/*
 * Causal sliding-window prefill that keeps the first n_sink tokens of every
 * sequence visible (samanvya.dev "Attention Is the Bottleneck", "Sliding
 * windows and local:global layers": StreamingLLM's sink tokens plus a recent
 * window).  Key j is visible from query i if j <= i and (j > i - window or
 * j < n_sink).  Dense batches as fa_fwd, always causal; window >= 1 (else
 * FA_ERR_INVALID_ARG), n_sink >= 0 (0: fa_fwd with the window).  Arguments,
 * layouts, alignment and errors as fa_fwd.
 */
int fa_fwd_sink_tokens(const void *q, const void *k, const void *v, void *o, float *lse,
                       int B, int Hq, int Hkv, int N, int d, int window, int n_sink,
                       float scale, int o_dtype, void *stream);

/* The same for packed sequences (layouts as fa_fwd_varlen); the sink tokens
 * are the first n_sink tokens of each sequence. */
int fa_fwd_varlen_sink_tokens(const void *q, const void *k, const void *v, void *o, float *lse,
                              const int *cu_seqlens, int num_seqs, int total_tokens,
                              int max_seqlen, int Hq, int Hkv, int d, int window, int n_sink,
                              float scale, int o_dtype, void *stream);

/*
 * FP8 prefill with incoherent processing ("FlashAttention-3" in samanvya.dev
 * "Attention Is the Bottleneck", "FlashAttention: same math, different IO":
 * Q and K multiplied by a random orthogonal Hadamard matrix before FP8
 * quantisation; Ales Analytics "Attention and matrix kernels", "How it
 * works": FP8 GEMMs carry a scale per block).  Two
 * calls: fa_fp8_prepare makes the E4M3 operands from bf16 Q, K, V, and
 * fa_fwd_fp8 runs the attention on them.  Dense batches, d = 128.
 *
 * fa_fp8_prepare:
 *   q [B*N, Hq, 128], k and v [B*N, Hkv, 128] bf16 (token-major, as fa_fwd)
 *   signs [128] fp32, each +1 or -1 (a random draw the caller makes once and
 *     keeps), or NULL for no rotation (plain FP8)
 *   -> q8 [B*N, Hq, 128] and k8 [B*N, Hkv, 128] E4M3 codes of
 *        Q' = Q diag(signs) H / sqrt(128), K' likewise (H the Sylvester
 *        Hadamard matrix, entry (i, k) = (-1)^popcount(i & k)), so that
 *        Q' K'^T = Q K^T;
 *      q_scale [B, Hq, nblk], k_scale [B, Hkv, nblk] fp32, nblk = ceil(N/128):
 *        one scale per (batch, head, block of 128 tokens);
 *      vt8 [B, Hkv, 128, vt_stride] E4M3 codes of V transposed (row c of
 *        (b, h) holds channel c of keys 0..N-1; vt_stride = N rounded up to a
 *        multiple of 16; bytes N..vt_stride-1 of each row are not written);
 *      v_scale [B, Hkv] fp32: one scale per (batch, KV head).
 *   A scale is the smallest power of two 2^k (k >= -126) with amax / 2^k <=
 *   448 over its block (1 for an all-zero block); a code is x / scale (exact)
 *   rounded to the nearest E4M3 value (ties to even), saturated at +-448.  workspace: fa_fp8_workspace_bytes(B, N, Hkv) bytes of device
 *   memory, 4-byte aligned (scratch; contents need no initialisation).
 *   Alignment: q, k, v, q8, k8, vt8 and signs 16 bytes; scales 4 bytes.
 *   Errors: FA_ERR_UNSUPPORTED for d != 128; FA_ERR_WORKSPACE if the
 *   workspace is missing or small; otherwise as fa_fwd.
 *
 * fa_fwd_fp8:
 *   The outputs of fa_fp8_prepare in; O [B*N, Hq, 128] (bf16 or fp32) and
 *   LSE [B, Hq, N] out, for softmax(Q'K'^T * scale + mask) V with every
 *   operand read as code * scale.  P is rounded to E4M3 for the P V product
 *   (so the result is that of FP8 attention, not bit-close to fa_fwd); the
 *   softmax statistics stay fp32.  Masks, scale, o_dtype, alignment and
 *   errors as fa_fwd (q8, k8, vt8: 16 bytes; scales: 4 bytes).
 */
size_t fa_fp8_workspace_bytes(int B, int N, int Hkv);
int fa_fp8_prepare(const void *q, const void *k, const void *v, const float *signs,
                   void *q8, void *k8, void *vt8, float *q_scale, float *k_scale,
                   float *v_scale, int B, int N, int Hq, int Hkv, int d, void *workspace,
                   size_t workspace_bytes, void *stream);
int fa_fwd_fp8(const void *q8, const void *k8, const void *vt8, const float *q_scale,
               const float *k_scale, const float *v_scale, void *o, float *lse, int B,
               int Hq, int Hkv, int N, int d, int causal, int window, float scale,
               int o_dtype, void *stream);

/*
 * fa_decode_paged without a workspace argument, for callers that cannot
 * allocate device memory: code running under a host framework whose memory
 * pool owns the device and forbids raw cudaMalloc, latency-critical serving
 * paths where cudaMalloc's implicit synchronisation is not allowed, or
 * embedded callers with a memory budget fixed at load time.  (The pages have
 * no counterpart; this is an interface convenience, computing exactly what
 * fa_decode_paged computes.)
 *
 * The split-KV scratch comes from a fixed 32 MiB array in the library's own
 * device memory, which every GPU that loads the library holds until the
 * process exits.  The arguments are checked as by fa_decode_paged; then
 * sizes whose workspace (fa_decode_workspace_bytes) exceeds 32 MiB are
 * refused with FA_ERR_WORKSPACE, before any CUDA call.  The first call on
 * each device looks up the array's device address (with that device current),
 * and a call looks it up again when the device's current context has changed
 * since (for example after cudaDeviceReset); make that first call before any
 * stream capture.  All calls share
 * the array and it keeps the last call's contents (nothing in it needs to
 * start at zero); calls that may overlap on the GPU race on it, so the caller
 * must order them.  Allocates nothing.  Other arguments, results and errors
 * as for fa_decode_paged.
 */
int fa_decode_paged_noalloc(const void *q, const void *k_cache, const void *v_cache,
                            const int *block_table, const int *seq_lens, void *o,
                            float *lse, int num_seqs, int num_pages, int Hq, int Hkv,
                            int d, int page_size, int max_pages_per_seq, float scale,
                            void *stream);

/* Human-readable text of a status code (static storage). */
const char *fa_status_string(int status);

/*
 * Synchronises `stream`, then reads and clears the device error word that a
 * kernel sets when one of its bounded waits runs out or it meets an input it
 * cannot honour.  Returns FA_OK, FA_ERR_TIMEOUT, FA_ERR_INVALID_ARG or
 * FA_ERR_CUDA.
 */
int fa_check_device_error(void *stream);

/*
 * Diagnostic: launches a one-warp kernel whose wait on a barrier never
 * completes, so the device-side watchdog must end it: after about a second
 * the wait gives up, the error word is set and the kernel returns.  A later
 * fa_check_device_error() then reports FA_ERR_TIMEOUT and the CUDA context
 * stays usable.  Returns FA_OK once launched (asynchronous on `stream`).
 */
int fa_selftest_watchdog(void *stream);

/* Library version, major * 10000 + minor * 100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_SM100_H */
