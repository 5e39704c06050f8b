/*
 * attn_oracle.c -- fp64 CPU oracle for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the package's smoke check
 * and the benchmark's CPU-baseline leg may load this library. The product
 * path (the CUDA library and its Python binding) never calls it and shares
 * no code, header, table or helper with it.
 *
 * What it computes is the plain definition of attention that the pages state
 * as the standard algorithm ("FlashAttention及变种改进", section 二.1
 * "标准自注意力的计算瓶颈": build the score matrix S from Q and K, take
 * P = softmax(S) row by row, then O = P V; the pages' formula itself is lost
 * in extraction, so the textbook form is used). FlashAttention reaches the
 * same result exactly, only faster ("IO感知技术革命", section
 * "在线Softmax的现金流优化"; "FlashAttention深度解析", section
 * "重新定义注意力计算"), so this oracle materialises each row of S and P
 * explicitly and runs no tiling and no online recurrence.
 *
 * Per output row i of head h, for every key j (all in fp64):
 *   s_ij  = scale * sum_c q_ic k_jc
 *   s_ij  = softcap * tanh(s_ij / softcap)           if softcap > 0
 *   s_ij += -slope_h * |(i + Nk - Nq) - j|           if ALiBi slopes given
 *   s_ij  = -inf                                     if key j is masked
 *   m_i   = max_j s_ij
 *   P_ij  = exp(s_ij - m_i) / sum_j exp(s_ij - m_i)
 *   O_i   = sum_j P_ij v_j
 *   LSE_i = m_i + ln sum_j exp(s_ij - m_i)
 * A row whose keys are all masked gets O_i = 0 and LSE_i = -inf (the empty
 * sum).
 *
 * Readings taken where the pages are silent (each is listed with its reason
 * in the design notes of the repository):
 *   - causal masking is aligned bottom-right ("Flash-Attention v2.0 到 v2.7",
 *     opening paragraph: since v2.1 the mask is anchored at the bottom-right
 *     corner, so one decode query sees all N+1 keys): query i sits at key
 *     position pos_i = i + Nk - Nq and sees key j only if j <= pos_i;
 *   - the sliding window (same page, section v2.3) keeps keys with
 *     pos_i - window_left <= j <= pos_i + window_right, a negative bound
 *     meaning unbounded on that side;
 *   - ALiBi (section v2.4) adds -slope_h * |pos_i - j| after softcapping;
 *   - softcapping (section v2.6) is c * tanh(s / c) on the scaled score;
 *   - the paged cache (section v2.5) stores token t of sequence b at row
 *     t % page_size of page block_table[b][t / page_size];
 *   - a split-KV partial (section v2.2) is this same definition restricted
 *     to one contiguous key range of the sequence, and the merge of the
 *     partials is lse = ln sum_s exp(lse_s), O = sum_s exp(lse_s - lse) O_s.
 *
 * Inputs may be given as fp16, bf16, fp8 E4M3 or fp8 E5M2 storage (the
 * already-rounded values the GPU sees; they are widened to fp64 exactly) or
 * as fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <omp.h>

#define ORACLE_F16 0
#define ORACLE_BF16 1
#define ORACLE_F64 2
#define ORACLE_E4M3 3
#define ORACLE_E5M2 4

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
static double widen_f16(uint16_t bits)
{
    int sign = (bits >> 15) & 1;
    int expo = (bits >> 10) & 0x1f;
    int frac = bits & 0x3ff;
    double mag;
    if (expo == 0)
        mag = ldexp((double)frac, -24);              /* subnormal: frac * 2^-24 */
    else if (expo == 31)
        mag = frac ? NAN : INFINITY;
    else
        mag = ldexp((double)(1024 + frac), expo - 25); /* (1.frac) * 2^(e-15) */
    return sign ? -mag : mag;
}

/* bfloat16 is the upper half of an IEEE binary32. */
static double widen_bf16(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* 8-bit floats (the FP8 forward that "FlashAttention深度解析" names, section
 * 未来展望). E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 fraction bits; no
 * infinities, exponent and fraction all ones is NaN, so the largest value is
 * 1.75 * 2^8 = 448. */
static double widen_e4m3(uint8_t bits)
{
    int sign = bits >> 7;
    int expo = (bits >> 3) & 0xf;
    int frac = bits & 0x7;
    double mag;
    if (expo == 15 && frac == 7)
        return NAN;
    if (expo == 0)
        mag = ldexp((double)frac, -9);               /* subnormal: (frac / 8) * 2^(1-7) */
    else
        mag = ldexp((double)(8 + frac), expo - 10);  /* (1.frac) * 2^(e-7) */
    return sign ? -mag : mag;
}

/* E5M2: 1 sign bit, 5 exponent bits (bias 15), 2 fraction bits, IEEE-style
 * infinities and NaNs at exponent 31. */
static double widen_e5m2(uint8_t bits)
{
    int sign = bits >> 7;
    int expo = (bits >> 2) & 0x1f;
    int frac = bits & 0x3;
    double mag;
    if (expo == 31)
        mag = frac ? NAN : INFINITY;
    else if (expo == 0)
        mag = ldexp((double)frac, -16);              /* subnormal: (frac / 4) * 2^(1-15) */
    else
        mag = ldexp((double)(4 + frac), expo - 17);  /* (1.frac) * 2^(e-15) */
    return sign ? -mag : mag;
}

static double load_elem(const void *base, long idx, int dtype)
{
    if (dtype == ORACLE_F64)
        return ((const double *)base)[idx];
    if (dtype == ORACLE_E4M3)
        return widen_e4m3(((const uint8_t *)base)[idx]);
    if (dtype == ORACLE_E5M2)
        return widen_e5m2(((const uint8_t *)base)[idx]);
    uint16_t bits = ((const uint16_t *)base)[idx];
    return dtype == ORACLE_BF16 ? widen_bf16(bits) : widen_f16(bits);
}

/* Widens n stored elements to fp64 (exposed so tests can pin the decoders). */
int oracle_widen(const void *src, int dtype, double *dst, long n)
{
    if (dtype < 0 || dtype > 4)
        return 1;
    for (long i = 0; i < n; ++i)
        dst[i] = load_elem(src, i, dtype);
    return 0;
}

/* Masking rule: is key j visible to the query that sits at key position pos? */
static int key_visible(long pos, long j, long nkeys, int causal, long wl, long wr)
{
    if (j < 0 || j >= nkeys)
        return 0;
    if (causal && j > pos)
        return 0;
    if (wl >= 0 && j < pos - wl)
        return 0;
    if (wr >= 0 && j > pos + wr)
        return 0;
    return 1;
}

/* Everything one output row needs. Keys are addressed through per-key element
 * offsets so the same routine serves the contiguous and the paged layouts. */
typedef struct {
    const void *q; long q_off;
    const void *k; const long *k_off;
    const void *v; const long *v_off;
    long nkeys;          /* keys 0 .. nkeys-1 exist */
    long key_lo, key_hi; /* only keys in [key_lo, key_hi) take part (split-KV partials) */
    int d, dtype;
    double scale, softcap, slope;
    int has_alibi, causal;
    long pos, wl, wr;
} row_spec;

/* One row of the plain definition. s and e are scratch rows of nkeys doubles;
 * p_out (nkeys doubles) receives the probability row if not NULL. */
static void attend_row(const row_spec *r, double *s, double *e, double *o, double *lse,
                       double *p_out)
{
    const int d = r->d;
    /* 1. scores */
    for (long j = 0; j < r->nkeys; ++j) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c)
            dot += load_elem(r->q, r->q_off + c, r->dtype) * load_elem(r->k, r->k_off[j] + c, r->dtype);
        double sj = r->scale * dot;
        if (r->softcap > 0.0)
            sj = r->softcap * tanh(sj / r->softcap);
        if (r->has_alibi)
            sj += -r->slope * fabs((double)(r->pos - j));
        int vis = key_visible(r->pos, j, r->nkeys, r->causal, r->wl, r->wr) &&
                  j >= r->key_lo && j < r->key_hi;
        s[j] = vis ? sj : -INFINITY;
    }
    /* 2. row max */
    double m = -INFINITY;
    for (long j = 0; j < r->nkeys; ++j)
        if (s[j] > m)
            m = s[j];
    if (m == -INFINITY) { /* every key masked: empty sum */
        for (int c = 0; c < d; ++c)
            o[c] = 0.0;
        *lse = -INFINITY;
        if (p_out)
            for (long j = 0; j < r->nkeys; ++j)
                p_out[j] = 0.0;
        return;
    }
    /* 3. probabilities */
    double sum = 0.0;
    for (long j = 0; j < r->nkeys; ++j) {
        e[j] = exp(s[j] - m); /* exp(-inf) = 0 for masked keys */
        sum += e[j];
    }
    for (long j = 0; j < r->nkeys; ++j)
        e[j] /= sum;
    if (p_out)
        memcpy(p_out, e, sizeof(double) * (size_t)r->nkeys);
    /* 4. O = P V */
    for (int c = 0; c < d; ++c)
        o[c] = 0.0;
    for (long j = 0; j < r->nkeys; ++j) {
        if (e[j] == 0.0)
            continue;
        for (int c = 0; c < d; ++c)
            o[c] += e[j] * load_elem(r->v, r->v_off[j] + c, r->dtype);
    }
    /* 5. log-sum-exp */
    *lse = m + log(sum);
}

static void set_threads(int num_threads)
{
    if (num_threads > 0)
        omp_set_num_threads(num_threads);
}

/*
 * Contiguous forward. q is [B, Nq, H, d]; k, v are [B, Nk, H, d]; all in
 * storage type dtype. rows (n_rows entries, or NULL for all Nq rows) selects
 * the query rows to compute. Outputs: o [B, n_rows, H, d], lse [B, H, n_rows],
 * and if p_out is not NULL the probabilities [B, H, n_rows, Nk].
 * Returns 0, or nonzero on a bad argument.
 */
int oracle_attn_fwd(const void *q, const void *k, const void *v, int dtype,
                    double *o, double *lse, double *p_out,
                    int B, int H, int Nq, int Nk, int d, double scale, int causal,
                    int window_left, int window_right, const double *alibi_slopes,
                    double softcap, const int *rows, int n_rows, int num_threads)
{
    if (!q || !k || !v || !o || !lse || B < 0 || H < 0 || Nq < 0 || Nk < 0 || d <= 0)
        return 1;
    if (dtype < 0 || dtype > 4)
        return 1;
    if (!rows)
        n_rows = Nq;
    for (int r = 0; rows && r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= Nq)
            return 2;
    set_threads(num_threads);
    const long delta = (long)Nk - (long)Nq;
    long n_units = (long)B * H * n_rows;
    int failed = 0;
#pragma omp parallel
    {
        double *s = malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
        double *e = malloc(sizeof(double) * (size_t)(Nk > 0 ? Nk : 1));
        long *koff = malloc(sizeof(long) * (size_t)(Nk > 0 ? Nk : 1));
        if (!s || !e || !koff) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (long u = 0; u < n_units; ++u) {
                int r = (int)(u % n_rows);
                int h = (int)((u / n_rows) % H);
                int b = (int)(u / ((long)n_rows * H));
                int i = rows ? rows[r] : r;
                for (long j = 0; j < Nk; ++j)
                    koff[j] = (((long)b * Nk + j) * H + h) * d;
                row_spec rs = {
                    .q = q, .q_off = (((long)b * Nq + i) * H + h) * d,
                    .k = k, .k_off = koff, .v = v, .v_off = koff,
                    .nkeys = Nk, .key_lo = 0, .key_hi = Nk,
                    .d = d, .dtype = dtype, .scale = scale, .softcap = softcap,
                    .slope = alibi_slopes ? alibi_slopes[h] : 0.0,
                    .has_alibi = alibi_slopes != NULL, .causal = causal,
                    .pos = i + delta, .wl = window_left, .wr = window_right,
                };
                double *orow = o + (((long)b * n_rows + r) * H + h) * d;
                double *lrow = lse + ((long)b * H + h) * n_rows + r;
                double *prow = p_out ? p_out + (((long)b * H + h) * n_rows + r) * (long)Nk : NULL;
                attend_row(&rs, s, e, orow, lrow, prow);
            }
        }
        free(s);
        free(e);
        free(koff);
    }
    return failed ? 3 : 0;
}

/* Key range [lo, hi) of split `split` out of `num_splits` for a sequence whose
 * visible keys are [vis_lo, vis_hi): near-equal contiguous chunks, each a
 * whole number of pages long. */
static void split_range(long vis_lo, long vis_hi, int num_splits, int split, int page_size,
                        long *lo, long *hi)
{
    long n = vis_hi - vis_lo;
    if (n <= 0) {
        *lo = *hi = vis_hi;
        return;
    }
    long chunk = (n + num_splits - 1) / num_splits;
    chunk = (chunk + page_size - 1) / page_size * page_size;
    long a = vis_lo + (long)split * chunk;
    long b = a + chunk;
    if (a > vis_hi)
        a = vis_hi;
    if (b > vis_hi)
        b = vis_hi;
    *lo = a;
    *hi = b;
}

/*
 * Paged decode (one query per sequence, causal, bottom-right aligned so the
 * query sits at position cache_seqlens[b] - 1 and sees every cached key).
 * q is [B, 1, H, d]; k_cache, v_cache are [num_pages, page_size, H, d];
 * block_table is [B, max_blocks]; cache_seqlens is [B]. batch (n_batch
 * entries, or NULL for all B) selects sequences. If num_splits <= 1 the
 * outputs are o [n_batch, 1, H, d] and lse [n_batch, H, 1]. If num_splits > 1
 * the outputs are the split partials o [num_splits, n_batch, H, d] and
 * lse [num_splits, n_batch, H].
 * Returns 0, 2 for a bad index in batch, 4 for a block-table entry or
 * sequence length out of range, 1 for other bad arguments.
 */
int oracle_attn_decode_paged(const void *q, const void *k_cache, const void *v_cache, int dtype,
                             const int *block_table, const int *cache_seqlens,
                             double *o, double *lse,
                             int B, int H, int d, int num_pages, int page_size, int max_blocks,
                             double scale, int window_left, const double *alibi_slopes,
                             double softcap, const int *batch, int n_batch, int num_splits,
                             int num_threads)
{
    if (!q || !k_cache || !v_cache || !block_table || !cache_seqlens || !o || !lse)
        return 1;
    if (B < 0 || H <= 0 || d <= 0 || page_size <= 0 || max_blocks < 0 || dtype < 0 || dtype > 4)
        return 1;
    if (!batch)
        n_batch = B;
    int S = num_splits > 1 ? num_splits : 1;
    for (int r = 0; r < n_batch; ++r) {
        int b = batch ? batch[r] : r;
        if (b < 0 || b >= B)
            return 2;
        long L = cache_seqlens[b];
        if (L < 0 || L > (long)max_blocks * page_size)
            return 4;
        for (long blk = 0; blk < (L + page_size - 1) / page_size; ++blk) {
            int pg = block_table[(long)b * max_blocks + blk];
            if (pg < 0 || pg >= num_pages)
                return 4;
        }
    }
    set_threads(num_threads);
    long n_units = (long)S * n_batch * H;
    long maxL = (long)max_blocks * page_size;
    int failed = 0;
#pragma omp parallel
    {
        double *s = malloc(sizeof(double) * (size_t)(maxL > 0 ? maxL : 1));
        double *e = malloc(sizeof(double) * (size_t)(maxL > 0 ? maxL : 1));
        long *off = malloc(sizeof(long) * (size_t)(maxL > 0 ? maxL : 1));
        if (!s || !e || !off) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long u = 0; u < n_units; ++u) {
                int h = (int)(u % H);
                int r = (int)((u / H) % n_batch);
                int sp = (int)(u / ((long)H * n_batch));
                int b = batch ? batch[r] : r;
                long L = cache_seqlens[b];
                /* gather the sequence's keys through the block table */
                for (long t = 0; t < L; ++t) {
                    long pg = block_table[(long)b * max_blocks + t / page_size];
                    off[t] = ((pg * page_size + t % page_size) * H + h) * d;
                }
                long pos = L - 1;
                long lo = 0, hi = L;
                if (S > 1) {
                    long vis_lo = window_left >= 0 ? pos - window_left : 0;
                    if (vis_lo < 0)
                        vis_lo = 0;
                    split_range(vis_lo, L, S, sp, page_size, &lo, &hi);
                }
                row_spec rs = {
                    .q = q, .q_off = ((long)b * H + h) * d,
                    .k = k_cache, .k_off = off, .v = v_cache, .v_off = off,
                    .nkeys = L, .key_lo = lo, .key_hi = hi,
                    .d = d, .dtype = dtype, .scale = scale, .softcap = softcap,
                    .slope = alibi_slopes ? alibi_slopes[h] : 0.0,
                    .has_alibi = alibi_slopes != NULL, .causal = 1,
                    .pos = pos, .wl = window_left, .wr = -1,
                };
                double *orow = o + (((long)sp * n_batch + r) * H + h) * d;
                double *lrow = lse + ((long)sp * n_batch + r) * H + h;
                attend_row(&rs, s, e, orow, lrow, NULL);
            }
        }
        free(s);
        free(e);
        free(off);
    }
    return failed ? 3 : 0;
}

/*
 * Merge of split-KV partials: for each of n rows, given num_splits partial
 * outputs o_part [num_splits, n, d] and lse_part [num_splits, n], computes
 * lse = ln sum_s exp(lse_s) and O = sum_s exp(lse_s - lse) O_s. Splits with
 * lse_s = -inf carry no keys and get weight 0; if every split is empty the
 * row is empty (O = 0, lse = -inf).
 */
int oracle_combine_splits(const double *o_part, const double *lse_part, int num_splits, long n,
                          int d, double *o, double *lse)
{
    if (!o_part || !lse_part || !o || !lse || num_splits <= 0 || n < 0 || d <= 0)
        return 1;
    for (long r = 0; r < n; ++r) {
        double m = -INFINITY;
        for (int sp = 0; sp < num_splits; ++sp)
            if (lse_part[(long)sp * n + r] > m)
                m = lse_part[(long)sp * n + r];
        for (int c = 0; c < d; ++c)
            o[r * d + c] = 0.0;
        if (m == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double sum = 0.0;
        for (int sp = 0; sp < num_splits; ++sp)
            sum += exp(lse_part[(long)sp * n + r] - m);
        double total = m + log(sum);
        for (int sp = 0; sp < num_splits; ++sp) {
            double w = exp(lse_part[(long)sp * n + r] - total);
            for (int c = 0; c < d; ++c)
                o[r * d + c] += w * o_part[((long)sp * n + r) * d + c];
        }
        lse[r] = total;
    }
    return 0;
}

int oracle_max_threads(void)
{
    return omp_get_max_threads();
}
