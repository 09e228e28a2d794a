/*
 * oracle.c -- plain, slow fp64 CPU definition of exact attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the tests, the smoke check and the bench's CPU-baseline
 * leg use it.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes (the definition, not the tiled algorithm):
 *   "What attention costs" (samanvya.dev, attention optimisation post):
 *       Attention(Q, K, V) = softmax(Q K^T / sqrt(d)) V
 *   generalised to a caller-given `scale` in place of 1/sqrt(d) and an
 *   additive mask that is 0 on the allowed key set A(i) and -inf elsewhere.
 *   The softmax is taken in the textbook two-pass order the same post lists
 *   for the naive three-kernel flow: all scores of a row, then their max,
 *   then the exponentials and their sum, then the weighted sum of V rows.
 *   The score row is materialised in full, one query row at a time.
 *
 *   LSE_i = M_i + log(l_i) in natural log, M_i = max_j S_ij,
 *   l_i = sum_j exp(S_ij - M_i): the per-row softmax statistics the same post
 *   says the backward keeps instead of the matrix.
 *
 * Allowed key sets A(i) (readings of the pages, each stated once here):
 *   non-causal : every key of the same sequence;
 *   causal     : keys j <= i (full causal attention: each token attends to
 *                all tokens before it, "Attending to fewer tokens");
 *   window W>0 : causal and j > i - W, i.e. the W keys ending at the
 *                token itself ("Sliding windows and local:global layers");
 *   decode     : the one query is the sequence's last token and sees all of
 *                its seq_len keys, gathered page by page through the block
 *                table ("Paging and prefix sharing").
 *   A row whose allowed set is empty gets O = 0 and LSE = -inf.
 *   GQA: query head h reads KV head h / (Hq / Hkv) ("MQA and GQA").
 *
 * Split-KV combine ("Flash-Decoding"): partial results over disjoint key
 * sets are merged with the log-sum-exp rule
 *   M = max_s lse_s, w_s = exp(lse_s - M), lse = M + log(sum_s w_s),
 *   O = sum_s w_s O_s / sum_s w_s.
 *
 * Further functions, each with its reading stated where it is defined:
 *   - oracle_attn_bwd_varlen (+ _sinks, _dq_rows, _dkv_rows): the gradients dQ, dK, dV
 *     (and of the sink logits) by the chain rule through the definition;
 *   - the learned sink logit per head (the _sinks variants): one more score
 *     in the denominator with a zero value;
 *   - oracle_decode_paged_fp8: the decode over an FP8 E4M3 cache with a scale
 *     per (page, KV head);
 *   - oracle_prefill_paged: a chunk of new queries over a paged cache, the
 *     chunk holding each sequence's last positions;
 *   - oracle_attn_varlen_rows_doc: a document mask by per-token ids;
 *   - oracle_attn_varlen_rows_sink_tokens: a sliding window that keeps the
 *     first tokens of each sequence visible;
 *   - oracle_hadamard_rotate, oracle_e4m3_encode, oracle_quantize_e4m3_blocks,
 *     oracle_attn_fp8: the FP8 prefill with incoherent processing (rotation
 *     of Q and K, block-scaled E4M3 codes, attention over the codes).
 *
 * Inputs are bf16 bit patterns (uint16); each is widened exactly to double.
 * All sums run in a fixed sequential order, so results do not depend on the
 * OpenMP thread count.  libm exp/log in double; build without -ffast-math.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 is the upper 16 bits of an IEEE binary32; widening is exact. */
static double widen(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Is key j (0-based, in the sequence) visible from query i? */
static int allowed(int64_t i, int64_t j, int causal, int window)
{
    if (!causal) return 1;
    if (j > i) return 0;
    if (window > 0 && j <= i - window) return 0;
    return 1;
}

/*
 * One output row.  keys[j] / vals[j] point at the d-vector of key / value j;
 * vis[j] says whether key j is in A(i).  s is scratch of length nkeys.
 * `sink` is a per-head logit that joins the softmax denominator as the score
 * of one extra key whose value is zero (-INFINITY: no sink).
 * Writes o[0..d) and *lse; optionally the probability row p[0..nkeys).
 */
static void attend_row_sink(const double *q, int d, int64_t nkeys,
                            const uint16_t *const *keys, const uint16_t *const *vals,
                            const unsigned char *vis, double scale, double sink,
                            double *s, double *o, double *lse, double *p)
{
    int64_t j;
    int c;
    double m = -INFINITY, l = 0.0;
    int any = 0;

    /* 1. scores of the allowed keys */
    for (j = 0; j < nkeys; ++j) {
        if (!vis[j]) { s[j] = -INFINITY; continue; }
        double acc = 0.0;
        for (c = 0; c < d; ++c) acc += q[c] * widen(keys[j][c]);
        s[j] = scale * acc;
        any = 1;
    }
    for (c = 0; c < d; ++c) o[c] = 0.0;
    if (!any && sink == -INFINITY) {
        *lse = -INFINITY;
        if (p) for (j = 0; j < nkeys; ++j) p[j] = 0.0;
        return;
    }
    /* 2. row max (the sink counts as a score), then the denominator */
    for (j = 0; j < nkeys; ++j)
        if (vis[j] && s[j] > m) m = s[j];
    if (sink > m) m = sink;
    for (j = 0; j < nkeys; ++j)
        if (vis[j]) l += exp(s[j] - m);
    if (sink != -INFINITY) l += exp(sink - m);
    /* 3. probabilities times values (the sink's value is zero) */
    for (j = 0; j < nkeys; ++j) {
        double pj = vis[j] ? exp(s[j] - m) / l : 0.0;
        if (p) p[j] = pj;
        if (!vis[j]) continue;
        for (c = 0; c < d; ++c) o[c] += pj * widen(vals[j][c]);
    }
    /* 4. log-sum-exp */
    *lse = m + log(l);
}

static void attend_row(const double *q, int d, int64_t nkeys,
                       const uint16_t *const *keys, const uint16_t *const *vals,
                       const unsigned char *vis, double scale,
                       double *s, double *o, double *lse, double *p)
{
    attend_row_sink(q, d, nkeys, keys, vals, vis, scale, -INFINITY, s, o, lse, p);
}

/*
 * Packed-sequence attention, optionally on a subset of query tokens.
 *   q [total, Hq, d], k/v [total, Hkv, d] (bf16 bits), sequences given by
 *   cu_seqlens[0..num_seqs] (prefix sums of the lengths).
 *   rows: global token indices to compute (NULL = all `total` tokens, in order)
 *   o   [nrows, Hq, d]  lse [nrows, Hq]   (fp64)
 * Returns 0, or -1 on a bad argument (a row outside every sequence, Hq not a
 * multiple of Hkv, ...).
 */
static int attn_varlen_rows_sinks(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                  const int32_t *cu_seqlens, int num_seqs,
                                  int Hq, int Hkv, int d, int causal, int window,
                                  double scale, const double *sinks, const int32_t *doc,
                                  int n_sink_tokens,
                                  const int64_t *rows, int64_t nrows, double *o, double *lse)
{
    if (Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0 || num_seqs < 0) return -1;
    const int group = Hq / Hkv;
    const int64_t total = cu_seqlens[num_seqs];
    if (!rows) nrows = total;
    int64_t maxlen = 0;
    for (int s = 0; s < num_seqs; ++s) {
        int64_t L = (int64_t)cu_seqlens[s + 1] - cu_seqlens[s];
        if (L < 0) return -1;
        if (L > maxlen) maxlen = L;
    }
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t t = rows ? rows[r] : r;
        if (t < 0 || t >= total) return -1;
    }
    int bad = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(maxlen > 0 ? maxlen : 1));
        double *qd = (double *)malloc(sizeof(double) * (size_t)d);
        const uint16_t **kp = (const uint16_t **)malloc(sizeof(void *) * (size_t)(maxlen > 0 ? maxlen : 1));
        const uint16_t **vp = (const uint16_t **)malloc(sizeof(void *) * (size_t)(maxlen > 0 ? maxlen : 1));
        unsigned char *vis = (unsigned char *)malloc((size_t)(maxlen > 0 ? maxlen : 1));
        if (!s || !qd || !kp || !vp || !vis) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t task = 0; task < nrows * (int64_t)Hq; ++task) {
                int64_t r = task / Hq;
                int h = (int)(task % Hq);
                int64_t t = rows ? rows[r] : r;
                /* which sequence holds token t */
                int seq = 0;
                while (seq < num_seqs && cu_seqlens[seq + 1] <= t) ++seq;
                int64_t start = cu_seqlens[seq];
                int64_t L = (int64_t)cu_seqlens[seq + 1] - start;
                int64_t i = t - start;
                int g = h / group;
                for (int c = 0; c < d; ++c)
                    qd[c] = widen(q[(t * Hq + h) * (int64_t)d + c]);
                for (int64_t j = 0; j < L; ++j) {
                    kp[j] = k + ((start + j) * Hkv + g) * (int64_t)d;
                    vp[j] = v + ((start + j) * Hkv + g) * (int64_t)d;
                    vis[j] = (unsigned char)((allowed(i, j, causal, window) ||
                                              (causal && j <= i && j < n_sink_tokens)) &&
                                             (!doc || doc[start + i] == doc[start + j]));
                }
                attend_row_sink(qd, d, L, kp, vp, vis, scale, sinks ? sinks[h] : -INFINITY, s,
                                o + (r * Hq + h) * (int64_t)d, lse + r * Hq + h, NULL);
            }
        }
        free(s); free(qd); free(kp); free(vp); free(vis);
    }
    return bad ? -2 : 0;
}

int oracle_attn_varlen_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            const int32_t *cu_seqlens, int num_seqs,
                            int Hq, int Hkv, int d, int causal, int window,
                            double scale, const int64_t *rows, int64_t nrows,
                            double *o, double *lse)
{
    return attn_varlen_rows_sinks(q, k, v, cu_seqlens, num_seqs, Hq, Hkv, d, causal, window,
                                  scale, NULL, NULL, 0, rows, nrows, o, lse);
}

/*
 * The same with a learned sink logit per query head, sinks[Hq] (in units of
 * scaled scores), joining every row's softmax denominator as the score of
 * one extra key with a zero value ("Sliding windows and local:global
 * layers": gpt-oss builds a learned sink into every head).  LSE includes the
 * sink's term.
 */
int oracle_attn_varlen_rows_sinks(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                  const int32_t *cu_seqlens, int num_seqs,
                                  int Hq, int Hkv, int d, int causal, int window,
                                  double scale, const double *sinks, const int64_t *rows,
                                  int64_t nrows, double *o, double *lse)
{
    if (!sinks) return -1;
    return attn_varlen_rows_sinks(q, k, v, cu_seqlens, num_seqs, Hq, Hkv, d, causal, window,
                                  scale, sinks, NULL, 0, rows, nrows, o, lse);
}

/*
 * Packed sequences with a document mask in any form ("FlexAttention":
 * document masks among the attention variants, Ales Analytics kernels page):
 * doc[total] holds a document id per token, and key j is visible from query
 * i only if both carry the same id (on top of the causal / window rule), so
 * a document's tokens need not be contiguous.  rows as for
 * oracle_attn_varlen_rows.
 */
int oracle_attn_varlen_rows_doc(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                const int32_t *cu_seqlens, int num_seqs,
                                int Hq, int Hkv, int d, int causal, int window,
                                double scale, const int32_t *doc, const int64_t *rows,
                                int64_t nrows, double *o, double *lse)
{
    if (!doc) return -1;
    return attn_varlen_rows_sinks(q, k, v, cu_seqlens, num_seqs, Hq, Hkv, d, causal, window,
                                  scale, NULL, doc, 0, rows, nrows, o, lse);
}

/*
 * Sink tokens with a sliding window ("Sliding windows and local:global
 * layers": StreamingLLM retains the first few tokens as sinks beside the
 * recent window): with causal and window W > 0, key j is visible from query i if
 * j <= i and (j > i - W or j < n_sink) -- the first n_sink tokens of each
 * sequence stay visible to every later query.  Otherwise as
 * oracle_attn_varlen_rows.
 */
int oracle_attn_varlen_rows_sink_tokens(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                        const int32_t *cu_seqlens, int num_seqs, int Hq,
                                        int Hkv, int d, int window, int n_sink, double scale,
                                        const int64_t *rows, int64_t nrows, double *o,
                                        double *lse)
{
    if (window <= 0 || n_sink < 0) return -1;
    return attn_varlen_rows_sinks(q, k, v, cu_seqlens, num_seqs, Hq, Hkv, d, 1, window,
                                  scale, NULL, NULL, n_sink, rows, nrows, o, lse);
}

/* Dense batch: q [B,N,Hq,d], k/v [B,N,Hkv,d]; o [B,N,Hq,d]; lse [B,Hq,N]. */
int oracle_attn(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                int B, int Hq, int Hkv, int N, int d, int causal, int window,
                double scale, double *o, double *lse)
{
    if (B < 0 || N < 0) return -1;
    int32_t *cu = (int32_t *)malloc(sizeof(int32_t) * (size_t)(B + 1));
    double *lse_t = (double *)malloc(sizeof(double) * (size_t)((int64_t)B * N * Hq + 1));
    if (!cu || !lse_t) { free(cu); free(lse_t); return -2; }
    for (int b = 0; b <= B; ++b) cu[b] = b * N;
    int rc = oracle_attn_varlen_rows(q, k, v, cu, B, Hq, Hkv, d, causal, window,
                                     scale, NULL, 0, o, lse_t);
    if (rc == 0) {
        /* token-major [B*N, Hq] -> [B, Hq, N] */
        for (int b = 0; b < B; ++b)
            for (int h = 0; h < Hq; ++h)
                for (int i = 0; i < N; ++i)
                    lse[((int64_t)b * Hq + h) * N + i] = lse_t[((int64_t)b * N + i) * Hq + h];
    }
    free(cu); free(lse_t);
    return rc;
}

/*
 * The probability matrix of one (sequence, head) -- for invariant checks on
 * small cases.  p [L, L] for the sequence `seq` of a packed batch.
 */
int oracle_probs(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                 const int32_t *cu_seqlens, int num_seqs, int seq, int h,
                 int Hq, int Hkv, int d, int causal, int window, double scale,
                 double *p)
{
    if (seq < 0 || seq >= num_seqs || h < 0 || h >= Hq || Hq % Hkv) return -1;
    int64_t start = cu_seqlens[seq], L = (int64_t)cu_seqlens[seq + 1] - start;
    int g = h / (Hq / Hkv);
    double *s = (double *)malloc(sizeof(double) * (size_t)(L + 1));
    double *qd = (double *)malloc(sizeof(double) * (size_t)d);
    double *o = (double *)malloc(sizeof(double) * (size_t)d);
    const uint16_t **kp = (const uint16_t **)malloc(sizeof(void *) * (size_t)(L + 1));
    const uint16_t **vp = (const uint16_t **)malloc(sizeof(void *) * (size_t)(L + 1));
    unsigned char *vis = (unsigned char *)malloc((size_t)(L + 1));
    int rc = (s && qd && o && kp && vp && vis) ? 0 : -2;
    for (int64_t i = 0; rc == 0 && i < L; ++i) {
        double lse;
        for (int c = 0; c < d; ++c) qd[c] = widen(q[((start + i) * Hq + h) * (int64_t)d + c]);
        for (int64_t j = 0; j < L; ++j) {
            kp[j] = k + ((start + j) * Hkv + g) * (int64_t)d;
            vp[j] = v + ((start + j) * Hkv + g) * (int64_t)d;
            vis[j] = (unsigned char)allowed(i, j, causal, window);
        }
        attend_row(qd, d, L, kp, vp, vis, scale, s, o, &lse, p + i * L);
    }
    free(s); free(qd); free(o); free(kp); free(vp); free(vis);
    return rc;
}

/*
 * Paged decode: one query token per sequence, at position seq_len - 1, seeing
 * all seq_len cached keys.  Key j of sequence s lives in page
 * block_table[s * max_pages + j / page_size], slot j % page_size.
 *   q [S, Hq, d]; k_cache/v_cache [num_pages, page_size, Hkv, d]
 *   o [S, Hq, d]; lse [S, Hq]
 */
static int decode_paged_sinks(const uint16_t *q, const uint16_t *k_cache,
                              const uint16_t *v_cache, const int32_t *block_table,
                              const int32_t *seq_lens, int S, int Hq, int Hkv, int d,
                              int page_size, int max_pages, int64_t num_pages,
                              double scale, const double *sinks, double *o, double *lse)
{
    if (S < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || page_size <= 0) return -1;
    int64_t maxlen = 0;
    for (int s = 0; s < S; ++s) {
        if (seq_lens[s] < 0 || seq_lens[s] > (int64_t)max_pages * page_size) return -1;
        if (seq_lens[s] > maxlen) maxlen = seq_lens[s];
        for (int64_t p = 0; p < ((int64_t)seq_lens[s] + page_size - 1) / page_size; ++p) {
            int32_t pg = block_table[(int64_t)s * max_pages + p];
            if (pg < 0 || pg >= num_pages) return -1;
        }
    }
    const int group = Hq / Hkv;
    int bad = 0;
#pragma omp parallel
    {
        size_t n = (size_t)(maxlen > 0 ? maxlen : 1);
        double *sb = (double *)malloc(sizeof(double) * n);
        double *qd = (double *)malloc(sizeof(double) * (size_t)d);
        const uint16_t **kp = (const uint16_t **)malloc(sizeof(void *) * n);
        const uint16_t **vp = (const uint16_t **)malloc(sizeof(void *) * n);
        unsigned char *vis = (unsigned char *)malloc(n);
        if (!sb || !qd || !kp || !vp || !vis) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t task = 0; task < (int64_t)S * Hq; ++task) {
                int s = (int)(task / Hq), h = (int)(task % Hq), g = h / group;
                int64_t L = seq_lens[s];
                for (int c = 0; c < d; ++c) qd[c] = widen(q[((int64_t)s * Hq + h) * d + c]);
                for (int64_t j = 0; j < L; ++j) {
                    int64_t pg = block_table[(int64_t)s * max_pages + j / page_size];
                    int64_t slot = j % page_size;
                    kp[j] = k_cache + ((pg * page_size + slot) * Hkv + g) * (int64_t)d;
                    vp[j] = v_cache + ((pg * page_size + slot) * Hkv + g) * (int64_t)d;
                    vis[j] = (unsigned char)allowed(L - 1, j, 1, 0);
                }
                attend_row_sink(qd, d, L, kp, vp, vis, scale, sinks ? sinks[h] : -INFINITY,
                                sb, o + task * d, lse + task, NULL);
            }
        }
        free(sb); free(qd); free(kp); free(vp); free(vis);
    }
    return bad ? -2 : 0;
}

int oracle_decode_paged(const uint16_t *q, const uint16_t *k_cache,
                        const uint16_t *v_cache, const int32_t *block_table,
                        const int32_t *seq_lens, int S, int Hq, int Hkv, int d,
                        int page_size, int max_pages, int64_t num_pages,
                        double scale, double *o, double *lse)
{
    return decode_paged_sinks(q, k_cache, v_cache, block_table, seq_lens, S, Hq, Hkv, d,
                              page_size, max_pages, num_pages, scale, NULL, o, lse);
}

/* Paged decode with a learned sink logit per query head (sinks[Hq]). */
int oracle_decode_paged_sinks(const uint16_t *q, const uint16_t *k_cache,
                              const uint16_t *v_cache, const int32_t *block_table,
                              const int32_t *seq_lens, int S, int Hq, int Hkv, int d,
                              int page_size, int max_pages, int64_t num_pages,
                              double scale, const double *sinks, double *o, double *lse)
{
    if (!sinks) return -1;
    return decode_paged_sinks(q, k_cache, v_cache, block_table, seq_lens, S, Hq, Hkv, d,
                              page_size, max_pages, num_pages, scale, sinks, o, lse);
}

/*
 * Log-sum-exp merge of partial results over disjoint key sets.
 *   o_parts [nparts, rows, d], lse_parts [nparts, rows] -> o [rows, d], lse [rows]
 * A part with lse = -inf carries no weight; if every part is -inf the row is
 * O = 0, LSE = -inf.
 */
int oracle_lse_combine(const double *o_parts, const double *lse_parts,
                       int nparts, int64_t rows, int d, double *o, double *lse)
{
    if (nparts < 0 || rows < 0 || d <= 0) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        double m = -INFINITY, wsum = 0.0;
        int c, s;
        for (s = 0; s < nparts; ++s)
            if (lse_parts[(int64_t)s * rows + r] > m) m = lse_parts[(int64_t)s * rows + r];
        for (c = 0; c < d; ++c) o[r * d + c] = 0.0;
        if (m == -INFINITY) { lse[r] = -INFINITY; continue; }
        for (s = 0; s < nparts; ++s) {
            double w = exp(lse_parts[(int64_t)s * rows + r] - m);
            wsum += w;
            for (c = 0; c < d; ++c) o[r * d + c] += w * o_parts[((int64_t)s * rows + r) * d + c];
        }
        for (c = 0; c < d; ++c) o[r * d + c] /= wsum;
        lse[r] = m + log(wsum);
    }
    return 0;
}

/*
 * Backward of packed-sequence attention (the backward rebuilds the attention
 * matrix from the inputs and the forward's row statistics rather than
 * storing it: "FlashAttention: same math, different IO").  The
 * pages give no formulas; these are the chain rule through the definition
 * above, with the upstream gradient dO = dLoss/dO:
 *   P_ij  = softmax_j(S_ij) over A(i)           (two-pass, as attend_row)
 *   dV_j  = sum_i P_ij dO_i
 *   dP_ij = dO_i . V_j
 *   D_i   = sum_j P_ij dP_ij                    (softmax Jacobian term)
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale sum_j dS_ij K_j
 *   dK_j  = scale sum_i dS_ij Q_i
 * With GQA, dK and dV of KV head g sum over the query heads that read g.
 *   q, dout [total, Hq, d]; k, v [total, Hkv, d] (bf16 bits)
 *   dq [total, Hq, d]; dk, dv [total, Hkv, d] (fp64)
 * Each (sequence, KV head) is one task that owns its dK/dV rows; sums run in
 * a fixed order (query head, then row, ascending), independent of threads.
 */
/*
 * One query row of the backward: given q_i, dO_i and the key/value rows of
 * its sequence, fills p[j] = P_ij and ds[j] = dS_ij (0 outside A(i)) and
 * dq[c] = scale sum_j dS_ij K_j[c].  Scratch: sc, dp (length nkeys), orow (d).
 */
static void bwd_row(const double *qd, const double *dod, int d, int64_t nkeys,
                    const uint16_t *const *kp, const uint16_t *const *vp,
                    const unsigned char *vis, double scale, double sink, double *sc,
                    double *p, double *dp, double *ds, double *orow, double *dq,
                    double *lse_out, double *D_out)
{
    double lse_i, D = 0.0;
    attend_row_sink(qd, d, nkeys, kp, vp, vis, scale, sink, sc, orow, &lse_i, p);
    /* dP and the Jacobian term D_i */
    for (int64_t j = 0; j < nkeys; ++j) {
        dp[j] = 0.0;
        if (!vis[j]) continue;
        for (int c = 0; c < d; ++c) dp[j] += dod[c] * widen(vp[j][c]);
        D += p[j] * dp[j];
    }
    for (int c = 0; c < d; ++c) dq[c] = 0.0;
    for (int64_t j = 0; j < nkeys; ++j) {
        ds[j] = vis[j] ? p[j] * (dp[j] - D) : 0.0;
        if (!vis[j]) continue;
        for (int c = 0; c < d; ++c) dq[c] += scale * ds[j] * widen(kp[j][c]);
    }
    if (lse_out) *lse_out = lse_i;
    if (D_out) *D_out = D;
}

static int attn_bwd_varlen_sinks(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                 const uint16_t *dout, const int32_t *cu_seqlens, int num_seqs,
                                 int Hq, int Hkv, int d, int causal, int window, double scale,
                                 const double *sinks, double *dq, double *dk, double *dv,
                                 double *dsinks)
{
    if (Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0 || num_seqs < 0) return -1;
    const int group = Hq / Hkv;
    int64_t maxlen = 0;
    for (int s = 0; s < num_seqs; ++s) {
        int64_t L = (int64_t)cu_seqlens[s + 1] - cu_seqlens[s];
        if (L < 0) return -1;
        if (L > maxlen) maxlen = L;
    }
    /* per-(sequence, KV head) partial sums of the sink gradient, summed in
       a fixed order afterwards so the result does not depend on threads */
    double *part = NULL;
    if (dsinks) {
        part = (double *)calloc((size_t)num_seqs * Hq + 1, sizeof(double));
        if (!part) return -2;
    }
    int bad = 0;
#pragma omp parallel
    {
        size_t n = (size_t)(maxlen > 0 ? maxlen : 1);
        double *sc = (double *)malloc(sizeof(double) * n);
        double *p = (double *)malloc(sizeof(double) * n);
        double *dp = (double *)malloc(sizeof(double) * n);
        double *ds = (double *)malloc(sizeof(double) * n);
        double *qd = (double *)malloc(sizeof(double) * (size_t)d);
        double *dod = (double *)malloc(sizeof(double) * (size_t)d);
        double *orow = (double *)malloc(sizeof(double) * (size_t)d);
        const uint16_t **kp = (const uint16_t **)malloc(sizeof(void *) * n);
        const uint16_t **vp = (const uint16_t **)malloc(sizeof(void *) * n);
        unsigned char *vis = (unsigned char *)malloc(n);
        if (!sc || !p || !dp || !ds || !qd || !dod || !orow || !kp || !vp || !vis) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t task = 0; task < (int64_t)num_seqs * Hkv; ++task) {
                int seq = (int)(task / Hkv), g = (int)(task % Hkv);
                int64_t start = cu_seqlens[seq];
                int64_t L = (int64_t)cu_seqlens[seq + 1] - start;
                for (int64_t j = 0; j < L; ++j) {
                    kp[j] = k + ((start + j) * Hkv + g) * (int64_t)d;
                    vp[j] = v + ((start + j) * Hkv + g) * (int64_t)d;
                    for (int c = 0; c < d; ++c) {
                        dk[((start + j) * Hkv + g) * (int64_t)d + c] = 0.0;
                        dv[((start + j) * Hkv + g) * (int64_t)d + c] = 0.0;
                    }
                }
                for (int h = g * group; h < (g + 1) * group; ++h) {
                    for (int64_t i = 0; i < L; ++i) {
                        const int64_t row = ((start + i) * Hq + h) * (int64_t)d;
                        for (int c = 0; c < d; ++c) {
                            qd[c] = widen(q[row + c]);
                            dod[c] = widen(dout[row + c]);
                        }
                        for (int64_t j = 0; j < L; ++j)
                            vis[j] = (unsigned char)allowed(i, j, causal, window);
                        double lse_i, D_i;
                        const double z = sinks ? sinks[h] : -INFINITY;
                        bwd_row(qd, dod, d, L, kp, vp, vis, scale, z, sc, p, dp, ds, orow,
                                dq + row, &lse_i, &D_i);
                        /* the sink's weight exp(z - LSE_i) times (0 - D_i) */
                        if (part && z != -INFINITY)
                            part[task * group + (h - g * group)] -= exp(z - lse_i) * D_i;
                        for (int64_t j = 0; j < L; ++j) {
                            if (!vis[j]) continue;
                            double *dkj = dk + ((start + j) * Hkv + g) * (int64_t)d;
                            double *dvj = dv + ((start + j) * Hkv + g) * (int64_t)d;
                            for (int c = 0; c < d; ++c) {
                                dkj[c] += scale * ds[j] * qd[c];
                                dvj[c] += p[j] * dod[c];
                            }
                        }
                    }
                }
            }
        }
        free(sc); free(p); free(dp); free(ds); free(qd); free(dod); free(orow);
        free(kp); free(vp); free(vis);
    }
    if (dsinks) {
        for (int h = 0; h < Hq; ++h) {
            double acc = 0.0;
            for (int seq = 0; seq < num_seqs; ++seq)
                acc += part[((int64_t)seq * Hkv + h / group) * group + h % group];
            dsinks[h] = acc;
        }
        free(part);
    }
    return bad ? -2 : 0;
}

int oracle_attn_bwd_varlen(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                           const uint16_t *dout, const int32_t *cu_seqlens, int num_seqs,
                           int Hq, int Hkv, int d, int causal, int window, double scale,
                           double *dq, double *dk, double *dv)
{
    return attn_bwd_varlen_sinks(q, k, v, dout, cu_seqlens, num_seqs, Hq, Hkv, d, causal,
                                 window, scale, NULL, dq, dk, dv, NULL);
}

/*
 * The same with a learned sink logit per query head (sinks[Hq]): P is the
 * softmax with the sink in its denominator, and dsinks[h] = d Loss / d z_h =
 * sum over rows of head h of exp(z_h - LSE_i) * (0 - D_i) (the sink's value
 * is zero, so its dP is 0).
 */
int oracle_attn_bwd_varlen_sinks(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                 const uint16_t *dout, const int32_t *cu_seqlens, int num_seqs,
                                 int Hq, int Hkv, int d, int causal, int window, double scale,
                                 const double *sinks, double *dq, double *dk, double *dv,
                                 double *dsinks)
{
    if (!sinks || !dsinks) return -1;
    return attn_bwd_varlen_sinks(q, k, v, dout, cu_seqlens, num_seqs, Hq, Hkv, d, causal,
                                 window, scale, sinks, dq, dk, dv, dsinks);
}

/*
 * dQ of selected query tokens only (every query head): rows[r] is a packed
 * token index; dq [nrows, Hq, d].  Each row needs only its own row of P, so
 * this stays cheap at any sequence length.
 */
int oracle_attn_bwd_dq_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            const uint16_t *dout, const int32_t *cu_seqlens, int num_seqs,
                            int Hq, int Hkv, int d, int causal, int window, double scale,
                            const int64_t *rows, int64_t nrows, double *dq)
{
    if (Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0 || num_seqs < 0 || nrows < 0) return -1;
    const int group = Hq / Hkv;
    const int64_t total = cu_seqlens[num_seqs];
    int64_t maxlen = 0;
    for (int s = 0; s < num_seqs; ++s) {
        int64_t L = (int64_t)cu_seqlens[s + 1] - cu_seqlens[s];
        if (L < 0) return -1;
        if (L > maxlen) maxlen = L;
    }
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= total) return -1;
    int bad = 0;
#pragma omp parallel
    {
        size_t n = (size_t)(maxlen > 0 ? maxlen : 1);
        double *sc = (double *)malloc(sizeof(double) * n);
        double *p = (double *)malloc(sizeof(double) * n);
        double *dp = (double *)malloc(sizeof(double) * n);
        double *ds = (double *)malloc(sizeof(double) * n);
        double *qd = (double *)malloc(sizeof(double) * (size_t)d);
        double *dod = (double *)malloc(sizeof(double) * (size_t)d);
        double *orow = (double *)malloc(sizeof(double) * (size_t)d);
        const uint16_t **kp = (const uint16_t **)malloc(sizeof(void *) * n);
        const uint16_t **vp = (const uint16_t **)malloc(sizeof(void *) * n);
        unsigned char *vis = (unsigned char *)malloc(n);
        if (!sc || !p || !dp || !ds || !qd || !dod || !orow || !kp || !vp || !vis) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t task = 0; task < nrows * (int64_t)Hq; ++task) {
                int64_t r = task / Hq, t = rows[r];
                int h = (int)(task % Hq), g = h / group;
                int seq = 0;
                while (seq < num_seqs && cu_seqlens[seq + 1] <= t) ++seq;
                int64_t start = cu_seqlens[seq];
                int64_t L = (int64_t)cu_seqlens[seq + 1] - start, i = t - start;
                const int64_t row = (t * Hq + h) * (int64_t)d;
                for (int c = 0; c < d; ++c) {
                    qd[c] = widen(q[row + c]);
                    dod[c] = widen(dout[row + c]);
                }
                for (int64_t j = 0; j < L; ++j) {
                    kp[j] = k + ((start + j) * Hkv + g) * (int64_t)d;
                    vp[j] = v + ((start + j) * Hkv + g) * (int64_t)d;
                    vis[j] = (unsigned char)allowed(i, j, causal, window);
                }
                bwd_row(qd, dod, d, L, kp, vp, vis, scale, -INFINITY, sc, p, dp, ds, orow,
                        dq + (r * Hq + h) * (int64_t)d, NULL, NULL);
            }
        }
        free(sc); free(p); free(dp); free(ds); free(qd); free(dod); free(orow);
        free(kp); free(vp); free(vis);
    }
    return bad ? -2 : 0;
}

/*
 * dK and dV of selected key tokens only (every KV head): rows[r] is a packed
 * token index; dk, dv [nrows, Hkv, d].  The same chain rule as the full
 * backward, summed per key instead of scattered per query:
 *   dV_j = sum_{h in group} sum_{i : j in A(i)} P_ij dO_i,
 *   dK_j = scale sum_{h in group} sum_{i : j in A(i)} dS_ij Q_i,
 *   P_ij = exp(S_ij - LSE_i),  dS_ij = P_ij (dO_i . V_j - D_i),
 * with LSE_i and D_i = sum_j P_ij (dO_i . V_j) of every query row (token,
 * query head) taken first from bwd_row over the row's whole allowed set.
 * The second pass sums over query heads, then query rows, in ascending order.
 */
int oracle_attn_bwd_dkv_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                             const uint16_t *dout, const int32_t *cu_seqlens, int num_seqs,
                             int Hq, int Hkv, int d, int causal, int window, double scale,
                             const int64_t *rows, int64_t nrows, double *dk, double *dv)
{
    if (Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv != 0 || num_seqs < 0 || nrows < 0) return -1;
    const int group = Hq / Hkv;
    const int64_t total = cu_seqlens[num_seqs];
    int64_t maxlen = 0;
    for (int s = 0; s < num_seqs; ++s) {
        int64_t L = (int64_t)cu_seqlens[s + 1] - cu_seqlens[s];
        if (L < 0) return -1;
        if (L > maxlen) maxlen = L;
    }
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= total) return -1;
    /* row statistics of every (token, query head) */
    double *lse = (double *)malloc(sizeof(double) * (size_t)(total > 0 ? total : 1) * Hq);
    double *Dr = (double *)malloc(sizeof(double) * (size_t)(total > 0 ? total : 1) * Hq);
    if (!lse || !Dr) {
        free(lse); free(Dr);
        return -2;
    }
    int bad = 0;
#pragma omp parallel
    {
        size_t n = (size_t)(maxlen > 0 ? maxlen : 1);
        double *sc = (double *)malloc(sizeof(double) * n);
        double *p = (double *)malloc(sizeof(double) * n);
        double *dp = (double *)malloc(sizeof(double) * n);
        double *ds = (double *)malloc(sizeof(double) * n);
        double *qd = (double *)malloc(sizeof(double) * (size_t)d);
        double *dod = (double *)malloc(sizeof(double) * (size_t)d);
        double *orow = (double *)malloc(sizeof(double) * (size_t)d);
        double *dqs = (double *)malloc(sizeof(double) * (size_t)d);
        const uint16_t **kp = (const uint16_t **)malloc(sizeof(void *) * n);
        const uint16_t **vp = (const uint16_t **)malloc(sizeof(void *) * n);
        unsigned char *vis = (unsigned char *)malloc(n);
        if (!sc || !p || !dp || !ds || !qd || !dod || !orow || !dqs || !kp || !vp || !vis) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t task = 0; task < total * (int64_t)Hq; ++task) {
                int64_t t = task / Hq;
                int h = (int)(task % Hq), g = h / group;
                int seq = 0;
                while (seq < num_seqs && cu_seqlens[seq + 1] <= t) ++seq;
                int64_t start = cu_seqlens[seq];
                int64_t L = (int64_t)cu_seqlens[seq + 1] - start, i = t - start;
                const int64_t row = (t * Hq + h) * (int64_t)d;
                for (int c = 0; c < d; ++c) {
                    qd[c] = widen(q[row + c]);
                    dod[c] = widen(dout[row + c]);
                }
                for (int64_t j = 0; j < L; ++j) {
                    kp[j] = k + ((start + j) * Hkv + g) * (int64_t)d;
                    vp[j] = v + ((start + j) * Hkv + g) * (int64_t)d;
                    vis[j] = (unsigned char)allowed(i, j, causal, window);
                }
                bwd_row(qd, dod, d, L, kp, vp, vis, scale, -INFINITY, sc, p, dp, ds, orow,
                        dqs, lse + task, Dr + task);
            }
        }
        free(sc); free(p); free(dp); free(ds); free(qd); free(dod); free(orow); free(dqs);
        free(kp); free(vp); free(vis);
    }
    if (bad) {
        free(lse); free(Dr);
        return -2;
    }
    /* per selected key token and KV head: the sums over the rows that see it */
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t task = 0; task < nrows * (int64_t)Hkv; ++task) {
        int64_t r = task / Hkv, t = rows[r];
        int g = (int)(task % Hkv);
        int seq = 0;
        while (seq < num_seqs && cu_seqlens[seq + 1] <= t) ++seq;
        int64_t start = cu_seqlens[seq];
        int64_t L = (int64_t)cu_seqlens[seq + 1] - start, j = t - start;
        const uint16_t *kj = k + (t * Hkv + g) * (int64_t)d;
        const uint16_t *vj = v + (t * Hkv + g) * (int64_t)d;
        double *dkr = dk + (r * Hkv + g) * (int64_t)d;
        double *dvr = dv + (r * Hkv + g) * (int64_t)d;
        for (int c = 0; c < d; ++c) dkr[c] = dvr[c] = 0.0;
        for (int h = g * group; h < (g + 1) * group; ++h) {
            for (int64_t i = 0; i < L; ++i) {
                if (!allowed(i, j, causal, window)) continue;
                const int64_t ti = start + i;
                const uint16_t *qi = q + (ti * Hq + h) * (int64_t)d;
                const uint16_t *doi = dout + (ti * Hq + h) * (int64_t)d;
                double s_ij = 0.0, dp_ij = 0.0;
                for (int c = 0; c < d; ++c) {
                    s_ij += widen(qi[c]) * widen(kj[c]);
                    dp_ij += widen(doi[c]) * widen(vj[c]);
                }
                const double p_ij = exp(scale * s_ij - lse[ti * Hq + h]);
                const double ds_ij = p_ij * (dp_ij - Dr[ti * Hq + h]);
                for (int c = 0; c < d; ++c) {
                    dvr[c] += p_ij * widen(doi[c]);
                    dkr[c] += scale * ds_ij * widen(qi[c]);
                }
            }
        }
    }
    free(lse); free(Dr);
    return 0;
}

/*
 * FP8 KV cache ("Quantize what's left" in the same post: serving engines
 * commonly store the cache in 8 bits).
 * Codes are OCP FP8 E4M3 in its "fn" form (no infinities): sign bit, 4
 * exponent bits with bias 7, 3 mantissa bits; exponent field 0 holds the
 * subnormals m/8 * 2^-6; S.1111.111 is NaN.  A cached value is
 * e4m3(code) * scale, with one fp32 scale per (page, KV head).
 */
double oracle_e4m3_value(uint8_t code)
{
    const int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/*
 * One row over FP8 keys and values: keys[j]/vals[j] point at d codes,
 * ks[j]/vs[j] are their dequantisation scales.  Same steps as
 * attend_row_sink with K_j = e4m3(code) * ks[j], V_j = e4m3(code) * vs[j].
 */
static void attend_row_fp8(const double *q, int d, int64_t nkeys,
                           const uint8_t *const *keys, const uint8_t *const *vals,
                           const double *ks, const double *vs, double scale, double sink,
                           double *s, double *o, double *lse)
{
    int64_t j;
    int c;
    double m = -INFINITY, l = 0.0;
    for (c = 0; c < d; ++c) o[c] = 0.0;
    for (j = 0; j < nkeys; ++j) {
        double acc = 0.0;
        for (c = 0; c < d; ++c) acc += q[c] * (oracle_e4m3_value(keys[j][c]) * ks[j]);
        s[j] = scale * acc;
    }
    if (nkeys == 0 && sink == -INFINITY) { *lse = -INFINITY; return; }
    for (j = 0; j < nkeys; ++j)
        if (s[j] > m) m = s[j];
    if (sink > m) m = sink;
    for (j = 0; j < nkeys; ++j) l += exp(s[j] - m);
    if (sink != -INFINITY) l += exp(sink - m);
    for (j = 0; j < nkeys; ++j) {
        const double pj = exp(s[j] - m) / l;
        for (c = 0; c < d; ++c) o[c] += pj * (oracle_e4m3_value(vals[j][c]) * vs[j]);
    }
    *lse = m + log(l);
}

/*
 * Paged decode over an FP8 cache: k_cache/v_cache [num_pages, page_size,
 * Hkv, d] E4M3 codes; k_scale/v_scale [num_pages, Hkv] fp32; sinks [Hq] or
 * NULL.  Otherwise as oracle_decode_paged.
 */
int oracle_decode_paged_fp8(const uint16_t *q, const uint8_t *k_cache, const uint8_t *v_cache,
                            const float *k_scale, const float *v_scale,
                            const int32_t *block_table, const int32_t *seq_lens, int S,
                            int Hq, int Hkv, int d, int page_size, int max_pages,
                            int64_t num_pages, double scale, const double *sinks, double *o,
                            double *lse)
{
    if (S < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || page_size <= 0) return -1;
    int64_t maxlen = 0;
    for (int s = 0; s < S; ++s) {
        if (seq_lens[s] < 0 || seq_lens[s] > (int64_t)max_pages * page_size) return -1;
        if (seq_lens[s] > maxlen) maxlen = seq_lens[s];
        for (int64_t p = 0; p < ((int64_t)seq_lens[s] + page_size - 1) / page_size; ++p) {
            int32_t pg = block_table[(int64_t)s * max_pages + p];
            if (pg < 0 || pg >= num_pages) return -1;
        }
    }
    const int group = Hq / Hkv;
    int bad = 0;
#pragma omp parallel
    {
        size_t n = (size_t)(maxlen > 0 ? maxlen : 1);
        double *sb = (double *)malloc(sizeof(double) * n);
        double *ksr = (double *)malloc(sizeof(double) * n);
        double *vsr = (double *)malloc(sizeof(double) * n);
        double *qd = (double *)malloc(sizeof(double) * (size_t)d);
        const uint8_t **kp = (const uint8_t **)malloc(sizeof(void *) * n);
        const uint8_t **vp = (const uint8_t **)malloc(sizeof(void *) * n);
        if (!sb || !ksr || !vsr || !qd || !kp || !vp) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t task = 0; task < (int64_t)S * Hq; ++task) {
                int s = (int)(task / Hq), h = (int)(task % Hq), g = h / group;
                int64_t L = seq_lens[s];
                for (int c = 0; c < d; ++c) qd[c] = widen(q[((int64_t)s * Hq + h) * d + c]);
                for (int64_t j = 0; j < L; ++j) {
                    int64_t pg = block_table[(int64_t)s * max_pages + j / page_size];
                    int64_t slot = j % page_size;
                    kp[j] = k_cache + ((pg * page_size + slot) * Hkv + g) * (int64_t)d;
                    vp[j] = v_cache + ((pg * page_size + slot) * Hkv + g) * (int64_t)d;
                    ksr[j] = (double)k_scale[pg * Hkv + g];
                    vsr[j] = (double)v_scale[pg * Hkv + g];
                }
                attend_row_fp8(qd, d, L, kp, vp, ksr, vsr, scale,
                               sinks ? sinks[h] : -INFINITY, sb, o + task * d, lse + task);
            }
        }
        free(sb); free(ksr); free(vsr); free(qd); free(kp); free(vp);
    }
    return bad ? -2 : 0;
}

/*
 * Chunked prefill over a paged cache (zenaique's FlashAttention serving
 * explainer, "Real-world examples": serving engines run long prompts in
 * chunks over a paged KV cache): sequence s has seq_lens_k[s] tokens in its pages (earlier
 * context plus this chunk's own keys), and its L_q = cu_seqlens_q[s+1] -
 * cu_seqlens_q[s] new query tokens are the last L_q of them: query i of the
 * chunk sits at position seq_lens_k[s] - L_q + i (the causal reading that
 * makes L_q = 1 the decode case and L_q = seq_lens_k the plain prefill).
 *   q [total_q, Hq, d]; k_cache/v_cache [num_pages, page_size, Hkv, d]
 *   block_table [S, max_pages]; sinks [Hq] or NULL
 *   o [total_q, Hq, d]; lse [total_q, Hq]
 * Returns -1 if some L_q > seq_lens_k or a used table entry is out of range.
 */
int oracle_prefill_paged(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                         const int32_t *block_table, const int32_t *cu_seqlens_q,
                         const int32_t *seq_lens_k, int S, int Hq, int Hkv, int d,
                         int page_size, int max_pages, int64_t num_pages, int causal,
                         int window, double scale, const double *sinks, double *o,
                         double *lse)
{
    if (S < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || page_size <= 0) return -1;
    int64_t maxlen = 0;
    for (int s = 0; s < S; ++s) {
        const int64_t Lq = (int64_t)cu_seqlens_q[s + 1] - cu_seqlens_q[s];
        const int64_t Lk = seq_lens_k[s];
        if (Lq < 0 || Lk < Lq || Lk > (int64_t)max_pages * page_size) return -1;
        if (Lk > maxlen) maxlen = Lk;
        for (int64_t p = 0; p < (Lk + page_size - 1) / page_size; ++p) {
            int32_t pg = block_table[(int64_t)s * max_pages + p];
            if (pg < 0 || pg >= num_pages) return -1;
        }
    }
    const int group = Hq / Hkv;
    const int64_t total_q = cu_seqlens_q[S];
    int bad = 0;
#pragma omp parallel
    {
        size_t n = (size_t)(maxlen > 0 ? maxlen : 1);
        double *sb = (double *)malloc(sizeof(double) * n);
        double *qd = (double *)malloc(sizeof(double) * (size_t)d);
        const uint16_t **kp = (const uint16_t **)malloc(sizeof(void *) * n);
        const uint16_t **vp = (const uint16_t **)malloc(sizeof(void *) * n);
        unsigned char *vis = (unsigned char *)malloc(n);
        if (!sb || !qd || !kp || !vp || !vis) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t task = 0; task < total_q * (int64_t)Hq; ++task) {
                const int64_t t = task / Hq;
                const int h = (int)(task % Hq), g = h / group;
                int s = 0;
                while (s < S && cu_seqlens_q[s + 1] <= t) ++s;
                const int64_t Lq = (int64_t)cu_seqlens_q[s + 1] - cu_seqlens_q[s];
                const int64_t Lk = seq_lens_k[s];
                const int64_t pos = Lk - Lq + (t - cu_seqlens_q[s]);
                for (int c = 0; c < d; ++c) qd[c] = widen(q[(t * Hq + h) * (int64_t)d + c]);
                for (int64_t j = 0; j < Lk; ++j) {
                    const int64_t pg = block_table[(int64_t)s * max_pages + j / page_size];
                    const int64_t slot = j % page_size;
                    kp[j] = k_cache + ((pg * page_size + slot) * Hkv + g) * (int64_t)d;
                    vp[j] = v_cache + ((pg * page_size + slot) * Hkv + g) * (int64_t)d;
                    vis[j] = (unsigned char)allowed(pos, j, causal, window);
                }
                attend_row_sink(qd, d, Lk, kp, vp, vis, scale, sinks ? sinks[h] : -INFINITY,
                                sb, o + task * (int64_t)d, lse + task, NULL);
            }
        }
        free(sb); free(qd); free(kp); free(vp); free(vis);
    }
    return bad ? -2 : 0;
}

/*
 * FP8 prefill with incoherent processing ("FlashAttention-3" in the
 * "FlashAttention: same math, different IO" part of samanvya.dev's post: a
 * random orthogonal Hadamard transform of Q and K ahead of E4M3 quantisation
 * spreads outlier channels over all dimensions; Ales Analytics "Attention and
 * matrix kernels", "How it works": FP8 GEMMs carry a scale per block).
 * Readings, where the pages leave the step open:
 *   - the orthogonal matrix is M = D H / sqrt(d): D = diag(signs), a random
 *     +-1 per channel drawn by the caller, H the Sylvester Hadamard matrix of
 *     order d (a power of two), entry (k, c) = (-1)^popcount(k & c).  Both Q
 *     and K are rotated by the same M, so (Q M)(K M)^T = Q K^T exactly;
 *   - Q and K get one scale per (batch, head, block of 128 tokens), V (not
 *     rotated) one per (batch, KV head): V's contraction runs over all keys,
 *     so its scale has to factor out of the whole sum;
 *   - the pages do not say how a block's scale is chosen: here it is the
 *     smallest power of two 2^k with amax / 2^k <= 448 (448 = largest finite
 *     E4M3; k >= -126 so that 1 / scale is a finite fp32), 1 for an all-zero
 *     block -- the power-of-two scales of the OCP microscaling formats.  Then
 *     x / scale is exact and the code is decided on the exact value: the
 *     E4M3 value nearest to x / scale, ties to the even code, saturated to
 *     +-448.
 * The attention is then the plain definition applied to the dequantised
 * values code * scale.
 */

/* Sylvester Hadamard entry of order 2^k: (-1)^popcount(k & c). */
static int hadamard_sign(int k, int c)
{
    unsigned x = (unsigned)(k & c);
    int par = 0;
    while (x) { par ^= 1; x &= x - 1; }
    return par ? -1 : 1;
}

/*
 * y[r][c] = sum_k signs[k] * x[r][k] * H[k][c] / sqrt(d) for rows of d bf16
 * values (signs NULL: y = x, no rotation).  d must be a power of two.
 */
int oracle_hadamard_rotate(const uint16_t *x, int64_t rows, int d, const double *signs,
                           double *y)
{
    if (d <= 0 || (d & (d - 1)) || rows < 0) return -1;
    const double inv = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *xr = x + r * d;
        double *yr = y + r * d;
        if (!signs) {
            for (int c = 0; c < d; ++c) yr[c] = widen(xr[c]);
            continue;
        }
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int k = 0; k < d; ++k)
                acc += signs[k] * widen(xr[k]) * (double)hadamard_sign(k, c);
            yr[c] = acc * inv;
        }
    }
    return 0;
}

/*
 * The E4M3 code nearest to y (ties to the even code), saturating at +-448.
 * The grid: spacing 2^(e-3) on [2^e, 2^(e+1)) for e >= -6, and the
 * subnormals m * 2^-9 below 2^-6.
 */
uint8_t oracle_e4m3_encode(double y)
{
    if (isnan(y)) return 0x7F;
    const int sign = signbit(y) ? 1 : 0;
    const double a = fabs(y);
    if (a >= 448.0) return (uint8_t)((sign << 7) | 0x7E);
    int e = -6;
    if (a >= ldexp(1.0, -6)) {
        frexp(a, &e);   /* a = f * 2^e, f in [0.5, 1) */
        e -= 1;         /* a in [2^e, 2^(e+1)) */
    }
    const double r = rint(ldexp(a, 3 - e));   /* units of the spacing; ties to even */
    int field, mant;
    if (e == -6 && r < 8.0) {
        field = 0;
        mant = (int)r;
    } else if (r >= 16.0) {
        field = e + 1 + 7;
        mant = 0;
    } else {
        field = e + 7;
        mant = (int)r - 8;
    }
    if (field > 15 || (field == 15 && mant == 7)) return (uint8_t)((sign << 7) | 0x7E);
    return (uint8_t)((sign << 7) | (field << 3) | mant);
}

/* The scale of a block whose largest magnitude is amax (see above). */
float oracle_e4m3_block_scale(double amax)
{
    if (!(amax > 0.0)) return 1.0f;
    int e;
    const double f = frexp(amax, &e);          /* amax = f * 2^e, f in [0.5, 1) */
    int k = (f <= 0.875) ? e - 9 : e - 8;       /* 448 = 0.875 * 2^9 */
    if (k < -126) k = -126;
    return (float)ldexp(1.0, k);
}

/*
 * Block-scaled E4M3 quantisation of x [B, N, H, d] (fp64): one scale per
 * (b, h, block of `block` tokens), scales [B, H, ceil(N / block)] fp32.
 */
int oracle_quantize_e4m3_blocks(const double *x, int B, int N, int H, int d, int block,
                                uint8_t *codes, float *scales)
{
    if (B < 0 || N < 0 || H <= 0 || d <= 0 || block <= 0) return -1;
    const int nblk = (N + block - 1) / block;
#pragma omp parallel for schedule(static)
    for (int64_t task = 0; task < (int64_t)B * H * nblk; ++task) {
        const int b = (int)(task / ((int64_t)H * nblk));
        const int h = (int)((task / nblk) % H);
        const int blk = (int)(task % nblk);
        const int n0 = blk * block, n1 = (n0 + block < N) ? n0 + block : N;
        double amax = 0.0;
        for (int n = n0; n < n1; ++n)
            for (int c = 0; c < d; ++c) {
                const double v = fabs(x[(((int64_t)b * N + n) * H + h) * d + c]);
                if (v > amax) amax = v;
            }
        const float sc = oracle_e4m3_block_scale(amax);
        scales[((int64_t)b * H + h) * nblk + blk] = sc;
        for (int n = n0; n < n1; ++n)
            for (int c = 0; c < d; ++c) {
                const int64_t i = (((int64_t)b * N + n) * H + h) * d + c;
                codes[i] = oracle_e4m3_encode(x[i] / (double)sc);
            }
    }
    return 0;
}

/*
 * Attention over E4M3 codes: q8 [B, N, Hq, d] with q_scale [B, Hq, ceil(N /
 * qblock)], k8 [B, N, Hkv, d] with k_scale [B, Hkv, ceil(N / kblock)], v8
 * [B, N, Hkv, d] with v_scale [B, Hkv].  Each value is code * its scale;
 * then the definition with causal / window masks as in oracle_attn.
 *   rows: the query positions to compute in every batch (NULL = all N, in order)
 *   o [B, nrows, Hq, d], lse [B, Hq, nrows] (fp64)
 */
int oracle_attn_fp8(const uint8_t *q8, const float *q_scale, int qblock,
                    const uint8_t *k8, const float *k_scale, int kblock,
                    const uint8_t *v8, const float *v_scale,
                    int B, int N, int Hq, int Hkv, int d, int causal, int window,
                    double scale, const int64_t *rows, int64_t nrows, double *o, double *lse)
{
    if (B < 0 || N < 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Hq % Hkv || qblock <= 0 ||
        kblock <= 0)
        return -1;
    if (!rows) nrows = N;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows && (rows[r] < 0 || rows[r] >= N)) return -1;
    const int group = Hq / Hkv;
    const int nbq = (N + qblock - 1) / qblock, nbk = (N + kblock - 1) / kblock;
    int bad = 0;
#pragma omp parallel
    {
        size_t n = (size_t)(N > 0 ? N : 1);
        double *sb = (double *)malloc(sizeof(double) * n);
        double *ksr = (double *)malloc(sizeof(double) * n);
        double *vsr = (double *)malloc(sizeof(double) * n);
        double *qd = (double *)malloc(sizeof(double) * (size_t)d);
        double *orow = (double *)malloc(sizeof(double) * (size_t)d);
        const uint8_t **kp = (const uint8_t **)malloc(sizeof(void *) * n);
        const uint8_t **vp = (const uint8_t **)malloc(sizeof(void *) * n);
        if (!sb || !ksr || !vsr || !qd || !orow || !kp || !vp) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t task = 0; task < (int64_t)B * nrows * Hq; ++task) {
                const int b = (int)(task / (nrows * Hq));
                const int64_t r = (task / Hq) % nrows;
                const int i = (int)(rows ? rows[r] : r);
                const int h = (int)(task % Hq), g = h / group;
                const double qs = (double)q_scale[((int64_t)b * Hq + h) * nbq + i / qblock];
                for (int c = 0; c < d; ++c)
                    qd[c] = oracle_e4m3_value(q8[(((int64_t)b * N + i) * Hq + h) * d + c]) * qs;
                /* the allowed keys are one contiguous range */
                int j0 = 0, j1 = N;
                if (causal) {
                    j1 = i + 1;
                    if (window > 0 && i - window + 1 > 0) j0 = i - window + 1;
                }
                int nk = 0;
                for (int j = j0; j < j1; ++j, ++nk) {
                    kp[nk] = k8 + (((int64_t)b * N + j) * Hkv + g) * d;
                    vp[nk] = v8 + (((int64_t)b * N + j) * Hkv + g) * d;
                    ksr[nk] = (double)k_scale[((int64_t)b * Hkv + g) * nbk + j / kblock];
                    vsr[nk] = (double)v_scale[(int64_t)b * Hkv + g];
                }
                double l;
                attend_row_fp8(qd, d, nk, kp, vp, ksr, vsr, scale, -INFINITY, sb, orow, &l);
                for (int c = 0; c < d; ++c) o[task * d + c] = orow[c];
                lse[((int64_t)b * Hq + h) * nrows + r] = l;
            }
        }
        free(sb); free(ksr); free(vsr); free(qd); free(orow); free(kp); free(vp);
    }
    return bad ? -2 : 0;
}
