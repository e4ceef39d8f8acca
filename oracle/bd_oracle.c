/*
 * Block-diffusion attention: plain fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
 * definition the CUDA path is checked against.  Only the tests, the smoke
 * check and the CPU-baseline leg of the benchmark may load it; the library
 * never calls it and shares no code, header or table with it.
 *
 * What it computes, and where each part comes from:
 *
 *  - Training/prefill form.  The query/key sequence of one (batch, head) is
 *    [x_t ; x_0]: rows 0..L-1 are the L noisy tokens, rows L..2L-1 the L clean
 *    ones, each half cut into blocks of b tokens (so L must be a multiple of
 *    b: the number of blocks is K = L_total / L_B in the BDLM objective of
 *    "LLaDA2.0-Uni" (discuss.pytorch.kr), section "Training objective and loss
 *    function", eq. L_BDLM).  The mask has the three parts named in
 *    "Nemotron-Labs-Diffusion-8B-Base 3x decoding speed-up" (doido.pw),
 *    section 1 "Block Diffusion Attention":
 *        M_BD  : a noisy token sees every noisy token of its own block;
 *        M_OBC : a noisy token of block k sees the clean tokens of blocks < k;
 *        M_BC  : a clean token of block k sees the clean tokens of blocks <= k.
 *    Clean tokens see no noisy token.  This is the reading that matches the
 *    BDLM conditioning p(x_{0,k} | x_{0,<k}, x_{t,k}) of the same eq. L_BDLM.
 *
 *  - Block-decode form.  A block of b noisy queries attends to the cached
 *    clean prefix (positions 0..cache_len-1) and to its own block, whose keys
 *    the caller has placed at cache positions cache_len..cache_len+b-1.
 *    Inside the block the attention is bidirectional for diffusion denoising
 *    (mode 0) or causal for self-speculative verification (mode 1): the
 *    "draft bidirectionally, verify causally over the same KV cache" flow of
 *    the same article, section 2 "Linear Speculative Decoding", and of
 *    "Nemotron-Labs-Diffusion-VLM-8B", section "Multi-mode decoding".
 *    Mode 2 is cross-attention only: the block rows are the canvas of an
 *    encoder-decoder model and see the encoder's cache positions
 *    0..cache_len-1 and nothing of the canvas ("DiffusionGemma" pipeline
 *    page, introduction and pipeline class description); with cache_len = 0
 *    such a row has no visible key.
 *
 *  - Sparse prefix retention (SPRINT, "LLaDA2.0-Uni", section "SPRINT:
 *    training-free inference acceleration", paragraph "Sparse Prefix
 *    Retention"): at the start of a block the cached prefix is pruned once.
 *    Position i gets the score s_i = alpha * I_i + (1 - alpha) * c_i, where
 *    I_i = |k_i|_2 / mean_j |k_j|_2 is its mean-normalised key norm and c_i
 *    the caller's top-1 confidence; each modality keeps its best-scoring
 *    fraction (images r_img = 0.8, text r_text = 1.0 on the page).
 *
 *  - For each query row: gather its visible key list, s_c = scale * q.k_c,
 *    m = max s, Z = sum exp(s_c - m), out = sum exp(s_c - m) / Z * v_c,
 *    lse = m + ln Z (natural log; the scale is inside).  A row with no
 *    visible key (never produced by valid inputs) gets out = 0, lse = -inf.
 *
 *  - Grouped-query attention: q-head h reads kv-head h / (Hq / Hkv).
 *
 * Inputs are the bf16 bit patterns the GPU receives; each is widened to fp64
 * exactly.  Every sum is a plain left-to-right fp64 loop.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Widen one bf16 bit pattern to double (exact: bf16 is the top half of an
 * IEEE binary32). */
static double bf16_bits_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int bdo_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Visibility predicate of the training/prefill mask for a sequence
 * [x_t ; x_0] of 2L positions cut into blocks of b: does query row r see key
 * position c?  Returns 1 or 0. */
int bdo_fwd_sees(int L, int b, int r, int c)
{
    int r_noisy = r < L;
    int c_noisy = c < L;
    int k_r = (r_noisy ? r : r - L) / b; /* block index of the query */
    int k_c = (c_noisy ? c : c - L) / b; /* block index of the key */
    if (r_noisy && c_noisy)
        return k_c == k_r; /* M_BD: own noisy block, bidirectional */
    if (r_noisy && !c_noisy)
        return k_c < k_r; /* M_OBC: strictly earlier clean blocks */
    if (!r_noisy && !c_noisy)
        return k_c <= k_r; /* M_BC: clean blocks up to its own */
    return 0;              /* clean queries never see noisy keys */
}

/* Visibility predicate of the block-decode form: does block row j (0 <= j < b)
 * see cache position c, given cache_len clean positions before the block?
 * mode 0: the block sees itself bidirectionally (denoising a draft);
 * mode 1: causally (verifying it); mode 2: not at all -- the rows are a
 * decoder canvas that cross-attends to an encoder's cache only ("Diffusion-
 * Gemma" pipeline page: a bidirectional decoder cross-attends to the KV
 * cache the causal encoder wrote, to denoise a canvas of canvas_length
 * tokens). */
int bdo_decode_sees(int cache_len, int b, int mode, int j, int c)
{
    if (c < 0)
        return 0;
    if (c < cache_len)
        return 1; /* the whole clean prefix */
    if (mode == 2)
        return 0; /* cross-attention only: nothing of the canvas itself */
    if (c < cache_len + b) {
        int jc = c - cache_len; /* row of the block that key c belongs to */
        return mode == 0 ? 1 : (jc <= j);
    }
    return 0;
}

/* The training/prefill mask as a dense [2L][2L] 0/1 matrix, cell (r, c) =
 * bdo_fwd_sees(L, b, r, c).  Returns 0, or -1 on a bad argument. */
int bdo_fwd_mask(int L, int b, uint8_t *mask)
{
    if (L <= 0 || b <= 0 || L % b != 0)
        return -1;
    const int N = 2 * L;
    int r, c;
    for (r = 0; r < N; ++r)
        for (c = 0; c < N; ++c)
            mask[(int64_t)r * N + c] = (uint8_t)bdo_fwd_sees(L, b, r, c);
    return 0;
}

/* Softmax attention of one query row over an explicit list of key rows.
 * q: d bf16 values; kbase/vbase: key/value rows of this kv-head (row stride d);
 * idx: the n visible key rows.  Writes out[d] and *lse.  s: scratch of n. */
static void attend_row(const uint16_t *q, const uint16_t *kbase,
                       const uint16_t *vbase, const int64_t *idx, int64_t n,
                       int d, double scale, double *s, double *out,
                       double *lse)
{
    int64_t j;
    int t;
    for (t = 0; t < d; ++t)
        out[t] = 0.0;
    if (n == 0) {
        *lse = -INFINITY;
        return;
    }
    for (j = 0; j < n; ++j) {
        const uint16_t *kr = kbase + idx[j] * (int64_t)d;
        double acc = 0.0;
        for (t = 0; t < d; ++t)
            acc += bf16_bits_to_double(q[t]) * bf16_bits_to_double(kr[t]);
        s[j] = scale * acc;
    }
    double m = s[0];
    for (j = 1; j < n; ++j)
        if (s[j] > m)
            m = s[j];
    double Z = 0.0;
    for (j = 0; j < n; ++j)
        Z += exp(s[j] - m);
    for (j = 0; j < n; ++j) {
        double p = exp(s[j] - m) / Z;
        const uint16_t *vr = vbase + idx[j] * (int64_t)d;
        for (t = 0; t < d; ++t)
            out[t] += p * bf16_bits_to_double(vr[t]);
    }
    *lse = m + log(Z);
}

/* Training/prefill form.
 * q: [B, Hq, 2L, d], k, v: [B, Hkv, 2L, d], all bf16 bit patterns, row-major.
 * rows: flat query-row ids ((batch * Hq + h) * 2L + r) to compute, or NULL for
 * every row in that order; nrows: their number.
 * out: [nrows, d] fp64, lse: [nrows] fp64.
 * Returns 0, or -1 on a bad argument. */
int bdo_fwd_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                 int B, int Hq, int Hkv, int L, int b, int d, double scale,
                 const int64_t *rows, int64_t nrows, double *out, double *lse)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || b <= 0 || d <= 0)
        return -1;
    if (Hq % Hkv != 0 || L % b != 0)
        return -1;
    const int64_t N = 2 * (int64_t)L;
    const int64_t total = (int64_t)B * Hq * N;
    if (rows == NULL)
        nrows = total;
    int64_t i;
    int bad = 0;
    for (i = 0; rows != NULL && i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= total)
            bad = 1;
    if (bad)
        return -1;
    const int group = Hq / Hkv;

#pragma omp parallel
    {
        int64_t *idx = (int64_t *)malloc(sizeof(int64_t) * N);
        double *s = (double *)malloc(sizeof(double) * N);
        int64_t ii;
#pragma omp for schedule(dynamic, 8)
        for (ii = 0; ii < nrows; ++ii) {
            int64_t id = rows ? rows[ii] : ii;
            int r = (int)(id % N);
            int64_t bh = id / N;
            int h = (int)(bh % Hq);
            int64_t bi = bh / Hq;
            int g = h / group;
            const uint16_t *qr = q + id * (int64_t)d;
            const uint16_t *kb = k + ((bi * Hkv + g) * N) * (int64_t)d;
            const uint16_t *vb = v + ((bi * Hkv + g) * N) * (int64_t)d;
            int64_t n = 0;
            int c;
            for (c = 0; c < N; ++c)
                if (bdo_fwd_sees(L, b, r, c))
                    idx[n++] = c;
            attend_row(qr, kb, vb, idx, n, d, scale, s, out + ii * (int64_t)d,
                       lse + ii);
        }
        free(idx);
        free(s);
    }
    return 0;
}

/* Block-decode form.
 * q_blk: [B, Hq, b, d]; k_cache, v_cache: [B, Hkv, S_cap, d] (bf16 bits);
 * cache_len: [B]; the block's own keys sit at cache_len[i]..cache_len[i]+b-1.
 * mode: 0 bidirectional inside the block, 1 causal, 2 prefix only.
 * rows: flat ids ((batch * Hq + h) * b + j) or NULL for all; out: [nrows, d],
 * lse: [nrows].  Returns 0, or -1 on a bad argument (including
 * cache_len[i] + b > S_cap in modes 0 and 1, cache_len[i] > S_cap in mode 2). */
int bdo_decode_rows(const uint16_t *q_blk, const uint16_t *k_cache,
                    const uint16_t *v_cache, const int32_t *cache_len, int B,
                    int Hq, int Hkv, int b, int d, int S_cap, int mode,
                    double scale, const int64_t *rows, int64_t nrows,
                    double *out, double *lse)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || b <= 0 || d <= 0 || S_cap <= 0)
        return -1;
    if (Hq % Hkv != 0 || mode < 0 || mode > 2)
        return -1;
    int i;
    /* modes 0 and 1 read the block's own keys after the prefix; mode 2 reads
     * the prefix only */
    const int own = (mode == 2) ? 0 : b;
    for (i = 0; i < B; ++i)
        if (cache_len[i] < 0 || (int64_t)cache_len[i] + own > S_cap)
            return -1;
    const int64_t total = (int64_t)B * Hq * b;
    if (rows == NULL)
        nrows = total;
    int64_t ii;
    for (ii = 0; rows != NULL && ii < nrows; ++ii)
        if (rows[ii] < 0 || rows[ii] >= total)
            return -1;
    const int group = Hq / Hkv;

#pragma omp parallel
    {
        int64_t *idx = (int64_t *)malloc(sizeof(int64_t) * S_cap);
        double *s = (double *)malloc(sizeof(double) * S_cap);
        int64_t jj;
#pragma omp for schedule(dynamic, 4)
        for (jj = 0; jj < nrows; ++jj) {
            int64_t id = rows ? rows[jj] : jj;
            int j = (int)(id % b);
            int64_t bh = id / b;
            int h = (int)(bh % Hq);
            int64_t bi = bh / Hq;
            int g = h / group;
            int len = cache_len[bi];
            const uint16_t *qr = q_blk + id * (int64_t)d;
            const uint16_t *kb = k_cache + ((bi * Hkv + g) * (int64_t)S_cap) * d;
            const uint16_t *vb = v_cache + ((bi * Hkv + g) * (int64_t)S_cap) * d;
            int64_t n = 0;
            int c;
            for (c = 0; c < S_cap; ++c)
                if (bdo_decode_sees(len, b, mode, j, c))
                    idx[n++] = c;
            attend_row(qr, kb, vb, idx, n, d, scale, s, out + jj * (int64_t)d,
                       lse + jj);
        }
        free(idx);
        free(s);
    }
    return 0;
}

/* Attention probabilities of one training/prefill query row over all 2L key
 * positions (0 for invisible keys).  row: flat query-row id as above.
 * p: [2L] fp64.  Returns 0, or -1 on a bad argument. */
int bdo_fwd_row_probs(const uint16_t *q, const uint16_t *k, int B, int Hq,
                      int Hkv, int L, int b, int d, double scale, int64_t row,
                      double *p)
{
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || b <= 0 || d <= 0)
        return -1;
    if (Hq % Hkv != 0 || L % b != 0)
        return -1;
    const int64_t N = 2 * (int64_t)L;
    if (row < 0 || row >= (int64_t)B * Hq * N)
        return -1;
    int r = (int)(row % N);
    int64_t bh = row / N;
    int h = (int)(bh % Hq);
    int64_t bi = bh / Hq;
    int g = h / (Hq / Hkv);
    const uint16_t *qr = q + row * (int64_t)d;
    const uint16_t *kb = k + ((bi * Hkv + g) * N) * (int64_t)d;
    double m = -INFINITY;
    int c, t;
    for (c = 0; c < N; ++c) {
        p[c] = -INFINITY;
        if (!bdo_fwd_sees(L, b, r, c))
            continue;
        double acc = 0.0;
        for (t = 0; t < d; ++t)
            acc += bf16_bits_to_double(qr[t]) *
                   bf16_bits_to_double(kb[(int64_t)c * d + t]);
        p[c] = scale * acc;
        if (p[c] > m)
            m = p[c];
    }
    double Z = 0.0;
    for (c = 0; c < N; ++c)
        if (p[c] != -INFINITY)
            Z += exp(p[c] - m);
    for (c = 0; c < N; ++c)
        p[c] = (p[c] == -INFINITY) ? 0.0 : exp(p[c] - m) / Z;
    return 0;
}

/* Merge partial attention results over a partition of one row's visible keys
 * into the result over their union: lse = ln sum_s exp(lse_s), out =
 * sum_s exp(lse_s - lse) * o_s.  Parts with lse_s = -inf are empty and skipped.
 * o_s: [nparts, d], lse_s: [nparts]; out: [d], lse: [1]. */
void bdo_combine(int nparts, int d, const double *o_s, const double *lse_s,
                 double *out, double *lse)
{
    int s, t;
    double m = -INFINITY;
    for (s = 0; s < nparts; ++s)
        if (lse_s[s] > m)
            m = lse_s[s];
    for (t = 0; t < d; ++t)
        out[t] = 0.0;
    if (m == -INFINITY) {
        *lse = -INFINITY;
        return;
    }
    double Z = 0.0;
    for (s = 0; s < nparts; ++s)
        if (lse_s[s] != -INFINITY)
            Z += exp(lse_s[s] - m);
    *lse = m + log(Z);
    for (s = 0; s < nparts; ++s) {
        if (lse_s[s] == -INFINITY)
            continue;
        double w = exp(lse_s[s] - *lse);
        for (t = 0; t < d; ++t)
            out[t] += w * o_s[(int64_t)s * d + t];
    }
}

/* ------------------------------------------------------------------------
 * Sparse prefix retention (SPRINT).
 *
 * Readings where the page is silent (stated once here, used below):
 *  - k_i is the key of position i in this cache across all its kv-heads,
 *    so |k_i|_2 = sqrt(sum over heads h and dims t of k[h][i][t]^2);
 *  - the mean in I_i runs over the prefix positions 0..cache_len-1 (the L of
 *    the page's formula); if it is 0 (an all-zero prefix) every I_i is 0;
 *  - alpha and the keep ratios r are single-precision numbers; modality 0
 *    is text, any other value image; a modality with n prefix positions
 *    keeps floor(r * n + 1/2) of them (r widened to double),
 *    clamped to [0, n]: the best scores, ties broken by the lower position;
 *  - the kept positions stay in their original order (stable compaction)
 *    and become the new prefix.
 */

typedef struct {
    double s;
    int p;
} bdo_scored;

/* higher score first; equal scores: lower position first */
static int bdo_scored_cmp(const void *a, const void *b)
{
    const bdo_scored *x = (const bdo_scored *)a, *y = (const bdo_scored *)b;
    if (x->s > y->s)
        return -1;
    if (x->s < y->s)
        return 1;
    return (x->p > y->p) - (x->p < y->p);
}

/* Scores and kept positions of the prefix of every sequence.
 * k_cache: [B, Hkv, S_cap, d] bf16 bits; cache_len: [B];
 * conf: [B, S_cap] fp32 top-1 confidences; modality: [B, S_cap] (0 text,
 * else image).  Writes score: [B, S_cap] fp64 (0 beyond the prefix),
 * kept: [B, S_cap] int32, the kept positions in increasing order followed by
 * -1, and new_len: [B], their number.  Returns 0, or -1 on a bad argument. */
int bdo_sprint_select(const uint16_t *k_cache, const int32_t *cache_len,
                      const float *conf, const uint8_t *modality, int B,
                      int Hkv, int d, int S_cap, float alpha_f,
                      float keep_text_f, float keep_image_f, double *score,
                      int32_t *kept, int32_t *new_len)
{
    /* alpha and the keep ratios are single-precision inputs, widened */
    const double alpha = alpha_f, keep_text = keep_text_f, keep_image = keep_image_f;
    if (B <= 0 || Hkv <= 0 || d <= 0 || S_cap <= 0)
        return -1;
    if (!(alpha >= 0.0 && alpha <= 1.0) || !(keep_text >= 0.0 && keep_text <= 1.0) ||
        !(keep_image >= 0.0 && keep_image <= 1.0))
        return -1;
    int i;
    for (i = 0; i < B; ++i)
        if (cache_len[i] < 0 || cache_len[i] > S_cap)
            return -1;
    for (i = 0; i < B; ++i) {
        const int n = cache_len[i];
        double *sc = score + (int64_t)i * S_cap;
        int32_t *kp = kept + (int64_t)i * S_cap;
        int p, h, t, m;
        /* key norms, then their mean over the prefix */
        double mean = 0.0;
        for (p = 0; p < S_cap; ++p)
            sc[p] = 0.0;
        for (p = 0; p < n; ++p) {
            double ss = 0.0;
            for (h = 0; h < Hkv; ++h) {
                const uint16_t *row = k_cache + (((int64_t)i * Hkv + h) * S_cap + p) * d;
                for (t = 0; t < d; ++t) {
                    double x = bf16_bits_to_double(row[t]);
                    ss += x * x;
                }
            }
            sc[p] = sqrt(ss); /* |k_p|_2 for now */
            mean += sc[p];
        }
        if (n > 0)
            mean /= n;
        /* composite score */
        for (p = 0; p < n; ++p) {
            double inorm = mean > 0.0 ? sc[p] / mean : 0.0;
            sc[p] = alpha * inorm + (1.0 - alpha) * (double)conf[(int64_t)i * S_cap + p];
        }
        /* per modality: keep the best floor(r n + 1/2) */
        char *keep = (char *)calloc((size_t)(n > 0 ? n : 1), 1);
        bdo_scored *lst = (bdo_scored *)malloc(sizeof(bdo_scored) * (size_t)(n > 0 ? n : 1));
        for (m = 0; m < 2; ++m) {
            int cnt = 0;
            for (p = 0; p < n; ++p) {
                int is_img = modality[(int64_t)i * S_cap + p] != 0;
                if (is_img == m) {
                    lst[cnt].s = sc[p];
                    lst[cnt].p = p;
                    ++cnt;
                }
            }
            double r = (m == 0) ? keep_text : keep_image;
            int64_t want = (int64_t)floor(r * (double)cnt + 0.5);
            if (want < 0)
                want = 0;
            if (want > cnt)
                want = cnt;
            qsort(lst, (size_t)cnt, sizeof(bdo_scored), bdo_scored_cmp);
            for (p = 0; p < want; ++p)
                keep[lst[p].p] = 1;
        }
        int nk = 0;
        for (p = 0; p < n; ++p)
            if (keep[p])
                kp[nk++] = p;
        for (p = nk; p < S_cap; ++p)
            kp[p] = -1;
        new_len[i] = nk;
        free(keep);
        free(lst);
    }
    return 0;
}
