/*
 * attn_oracle.c -- plain fp64 CPU oracle for the exact attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; it exists so that tests, the smoke check and the CPU baseline leg
 * of the benchmark can compare the CUDA kernels against a slow, obviously
 * correct definition.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes (pages: "FlashAttention common interfaces" (xllm-io blog),
 * sections 3.1 flash_attn_func, 3.2 flash_attn_varlen_func, 3.3
 * flash_attn_with_kvcache, 3.4 flash_attn_combine, 4.2 GQA, 4.3 sliding
 * window, 5.1 ALiBi, 5.2 softcap; and the flash-attn changelog post
 * (framerc.cn), items "causal mask aligned bottom-right since v2.1",
 * "v2.2 split-kv", "v2.5 paged KV cache", "v2.6 softcapping"):
 *
 *   for every sequence b, query head h, query row i:
 *     hk   = h / (H / Hkv)                       (GQA: contiguous head groups)
 *     off  = Sk_b - Sq_b                         (bottom-right alignment)
 *     s_j  = scale * <q_i, k_j>                  for every key j in [0, Sk_b)
 *     s_j  = softcap * tanh(s_j / softcap)       if softcap > 0
 *     s_j -= slope_h * |i + off - j|             if ALiBi slopes are given
 *     key j is allowed iff
 *        (!causal || j <= i + off) &&
 *        (left  < 0 || j >= i + off - left) &&
 *        (right < 0 || j <= i + off + right)
 *     no allowed key:  O = 0, LSE = -inf
 *     otherwise:       M = max allowed s_j, LSE = M + ln sum exp(s_j - M),
 *                      O = sum exp(s_j - LSE) * v_j      (allowed j only)
 *
 * The score row is materialised in full and the softmax takes two passes
 * (max, then sum); there is no blocking, no online rescaling, no fusion.
 *
 * Combine (section 3.4): LSE = M + ln sum_s exp(lse_s - M) with M = max_s lse_s,
 * O = sum_s exp(lse_s - LSE) * O_s; all lse_s = -inf gives O = 0, LSE = -inf.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* One (sequence, head) problem: query rows, key/value row pointers. */
static void attend_head(const double *q, long q_row_stride,       /* q rows for this seq+head */
                        const double *const *krow, const double *const *vrow,
                        double *out, long o_row_stride, double *lse, long lse_stride,
                        long Sq, long Sk, int d, double scale, int causal, int wl,
                        int wr, double softcap, double slope, int has_alibi,
                        double *s /* scratch [Sk] */, unsigned char *ok /* scratch [Sk] */)
{
    const long off = Sk - Sq;
    for (long i = 0; i < Sq; ++i) {
        const double *qi = q + i * q_row_stride;
        double *oi = out + i * o_row_stride;
        /* pass 0: full score row and its mask */
        long n_ok = 0;
        for (long j = 0; j < Sk; ++j) {
            const double *kj = krow[j];
            double acc = 0.0;
            for (int t = 0; t < d; ++t) acc += qi[t] * kj[t];
            double sj = scale * acc;
            if (softcap > 0.0) sj = softcap * tanh(sj / softcap);
            if (has_alibi) sj -= slope * fabs((double)(i + off - j));
            s[j] = sj;
            const long c = i + off;
            int a = 1;
            if (causal && j > c) a = 0;
            if (wl >= 0 && j < c - wl) a = 0;
            if (wr >= 0 && j > c + wr) a = 0;
            ok[j] = (unsigned char)a;
            n_ok += a;
        }
        if (n_ok == 0) {
            for (int t = 0; t < d; ++t) oi[t] = 0.0;
            lse[i * lse_stride] = -INFINITY;
            continue;
        }
        /* pass 1: max over allowed keys */
        double M = -INFINITY;
        for (long j = 0; j < Sk; ++j)
            if (ok[j] && s[j] > M) M = s[j];
        /* pass 2: normaliser */
        double Z = 0.0;
        for (long j = 0; j < Sk; ++j)
            if (ok[j]) Z += exp(s[j] - M);
        const double L = M + log(Z);
        lse[i * lse_stride] = L;
        /* output: probability-weighted sum of value rows */
        for (int t = 0; t < d; ++t) oi[t] = 0.0;
        for (long j = 0; j < Sk; ++j) {
            if (!ok[j]) continue;
            const double p = exp(s[j] - L);
            const double *vj = vrow[j];
            for (int t = 0; t < d; ++t) oi[t] += p * vj[t];
        }
    }
}

/*
 * Dense or varlen attention.  Packed layout:
 *   q   [total_q][H][d], k, v [total_k][Hkv][d], out [total_q][H][d],
 *   lse [total_q][H]
 * Sequence b owns query rows cu_q[b] .. cu_q[b+1]-1 and key rows
 * cu_k[b] .. cu_k[b+1]-1.  A dense batch is the special case cu = b * S.
 * slopes: NULL or [H].  Returns 0, or -1 on a bad argument.
 */
int oracle_attention(const double *q, const double *k, const double *v, double *out,
                     double *lse, int nseq, const int64_t *cu_q, const int64_t *cu_k,
                     int H, int Hkv, int d, double scale, int causal, int wl, int wr,
                     double softcap, const double *slopes, int nthreads)
{
    if (H <= 0 || Hkv <= 0 || H % Hkv != 0 || d <= 0 || nseq < 0) return -1;
    const int G = H / Hkv;
    const long n_items = (long)nseq * H;
    long max_sk = 0;
    for (int b = 0; b < nseq; ++b) {
        long sk = cu_k[b + 1] - cu_k[b];
        if (sk > max_sk) max_sk = sk;
        if (sk < 0 || cu_q[b + 1] - cu_q[b] < 0) return -1;
    }
    (void)nthreads;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(max_sk + 1));
        unsigned char *okm = (unsigned char *)malloc((size_t)(max_sk + 1));
        const double **kr = (const double **)malloc(sizeof(double *) * (size_t)(max_sk + 1));
        const double **vr = (const double **)malloc(sizeof(double *) * (size_t)(max_sk + 1));
#pragma omp for schedule(dynamic, 1)
        for (long it = 0; it < n_items; ++it) {
            const int b = (int)(it / H), h = (int)(it % H), hk = h / G;
            const long q0 = cu_q[b], Sq = cu_q[b + 1] - cu_q[b];
            const long k0 = cu_k[b], Sk = cu_k[b + 1] - cu_k[b];
            for (long j = 0; j < Sk; ++j) {
                kr[j] = k + ((k0 + j) * Hkv + hk) * (long)d;
                vr[j] = v + ((k0 + j) * Hkv + hk) * (long)d;
            }
            attend_head(q + (q0 * H + h) * (long)d, (long)H * d, kr, vr,
                        out + (q0 * H + h) * (long)d, (long)H * d, lse + q0 * H + h, H, Sq, Sk,
                        d, scale, causal, wl, wr, softcap, slopes ? slopes[h] : 0.0,
                        slopes != NULL, s, okm);
        }
        free(s);
        free(okm);
        free(kr);
        free(vr);
    }
    return 0;
}

/*
 * Attention against a paged KV cache (changelog v2.5: a block_table maps each
 * sequence's logical pages to physical pages of a shared pool).
 *   q    [B][Sq][H][d], out [B][Sq][H][d], lse [B][Sq][H]
 *   kpool, vpool [num_blocks][page][Hkv][d]
 *   block_table [B][max_blocks] (entry p of sequence b is the pool block that
 *   holds its keys p*page .. p*page+page-1), cache_seqlens [B] = number of keys
 *   sequence b attends (Sk_b).  Query row i of sequence b sits at key position
 *   i + Sk_b - Sq (bottom-right alignment).
 */
int oracle_attention_paged(const double *q, const double *kpool, const double *vpool,
                           double *out, double *lse, int B, int Sq, int H, int Hkv, int d,
                           const int32_t *block_table, int max_blocks, int page,
                           long num_blocks, const int32_t *cache_seqlens, double scale,
                           int causal, int wl, int wr, double softcap, const double *slopes,
                           int nthreads)
{
    if (H <= 0 || Hkv <= 0 || H % Hkv != 0 || d <= 0 || B < 0 || page <= 0) return -1;
    const int G = H / Hkv;
    long max_sk = 0;
    for (int b = 0; b < B; ++b) {
        long sk = cache_seqlens[b];
        if (sk < 0 || (sk + page - 1) / page > max_blocks) return -1;
        for (long p = 0; p < (sk + page - 1) / page; ++p) {
            int32_t blk = block_table[(long)b * max_blocks + p];
            if (blk < 0 || blk >= num_blocks) return -1;
        }
        if (sk > max_sk) max_sk = sk;
    }
    const long n_items = (long)B * H;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(max_sk + 1));
        unsigned char *okm = (unsigned char *)malloc((size_t)(max_sk + 1));
        const double **kr = (const double **)malloc(sizeof(double *) * (size_t)(max_sk + 1));
        const double **vr = (const double **)malloc(sizeof(double *) * (size_t)(max_sk + 1));
#pragma omp for schedule(dynamic, 1)
        for (long it = 0; it < n_items; ++it) {
            const int b = (int)(it / H), h = (int)(it % H), hk = h / G;
            const long Sk = cache_seqlens[b];
            for (long j = 0; j < Sk; ++j) {
                const long blk = block_table[(long)b * max_blocks + j / page];
                const long row = blk * page + j % page;
                kr[j] = kpool + (row * Hkv + hk) * (long)d;
                vr[j] = vpool + (row * Hkv + hk) * (long)d;
            }
            const long qoff = ((long)b * Sq * H + h) * (long)d;
            attend_head(q + qoff, (long)H * d, kr, vr, out + qoff, (long)H * d,
                        lse + (long)b * Sq * H + h, H, Sq, Sk, d, scale, causal, wl, wr,
                        softcap, slopes ? slopes[h] : 0.0, slopes != NULL, s, okm);
        }
        free(s);
        free(okm);
        free(kr);
        free(vr);
    }
    return 0;
}

/*
 * LSE-weighted combine of split partials (section 3.4 flash_attn_combine).
 *   out_partial [rows][d][splits], lse_partial [rows][splits] (the pages' layout
 *   with (batch, seqlen, heads) flattened into rows); out [rows][d], lse [rows].
 */
int oracle_combine(const double *out_partial, const double *lse_partial, double *out,
                   double *lse, long rows, int d, int splits)
{
    if (rows < 0 || d <= 0 || splits <= 0) return -1;
    for (long r = 0; r < rows; ++r) {
        const double *lp = lse_partial + r * splits;
        double M = -INFINITY;
        for (int s = 0; s < splits; ++s)
            if (lp[s] > M) M = lp[s];
        double *o = out + r * d;
        if (M == -INFINITY) {
            for (int t = 0; t < d; ++t) o[t] = 0.0;
            lse[r] = -INFINITY;
            continue;
        }
        double Z = 0.0;
        for (int s = 0; s < splits; ++s) Z += exp(lp[s] - M);
        const double L = M + log(Z);
        lse[r] = L;
        for (int t = 0; t < d; ++t) {
            double acc = 0.0;
            for (int s = 0; s < splits; ++s) {
                if (lp[s] == -INFINITY) continue;
                acc += exp(lp[s] - L) * out_partial[(r * d + t) * splits + s];
            }
            o[t] = acc;
        }
    }
    return 0;
}
