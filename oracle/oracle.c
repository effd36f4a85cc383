/*
 * oracle.c -- plain single-threaded fp32 CPU reference of the greedy decode
 * step (see oracle.h for the sources and the precision rules).
 *
 * TEST INFRASTRUCTURE ONLY: tests, the smoke check and the benchmark's
 * CPU-baseline leg are the only users.  Nothing here is shared with the GPU
 * library.  Every function is the plain definition, computed directly:
 * no blocking, no fusion, no reordering of sums.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- formats */

/* IEEE 754 binary16: s | 5-bit exponent (bias 15) | 10-bit fraction. */
float or_fp16_to_f32(uint16_t h)
{
    int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
    float v;
    if (e == 0)
        v = ldexpf((float)m, -24);                /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexpf((float)(m + 1024), e - 25);    /* (1 + m/1024) * 2^(e-15) */
    return s ? -v : v;
}

/* binary32 -> binary16, round to nearest, ties to even; overflow -> inf. */
uint16_t or_f32_to_fp16(float f)
{
    uint32_t x;
    memcpy(&x, &f, 4);
    uint32_t sign = (x >> 16) & 0x8000u;
    uint32_t ax = x & 0x7fffffffu;
    if (ax >= 0x7f800000u)                         /* inf or NaN */
        return (uint16_t)(sign | (ax > 0x7f800000u ? 0x7e00u : 0x7c00u));
    if (ax >= 0x477ff000u)                         /* >= 65520 rounds to inf */
        return (uint16_t)(sign | 0x7c00u);
    int e = (int)(ax >> 23) - 127;
    if (e >= -14) {                                /* normal binary16 */
        uint32_t mant = ax & 0x7fffffu;
        uint32_t h = ((uint32_t)(e + 15) << 10) | (mant >> 13);
        uint32_t rem = mant & 0x1fffu;
        if (rem > 0x1000u || (rem == 0x1000u && (h & 1u)))
            h++;
        return (uint16_t)(sign | h);
    }
    /* subnormal binary16: count units of 2^-24 */
    int shift = -(e + 1);                          /* >= 14 */
    if (shift > 24)
        return (uint16_t)sign;
    uint32_t M = (ax & 0x7fffffu) | 0x800000u;     /* value = M * 2^(e-23) */
    uint32_t m = M >> shift;
    uint32_t rem = M & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1);
    if (rem > half || (rem == half && (m & 1u)))
        m++;
    return (uint16_t)(sign | m);
}

/* OCP 8-bit E4M3 ("fn"): s | 4-bit exponent (bias 7) | 3-bit mantissa,
 * no infinities, S.1111.111 is NaN, subnormals m * 2^-9. */
float or_e4m3_to_f32(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    float v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexpf((float)m, -9);
    else
        v = ldexpf((float)(8 + m), e - 10);        /* (1 + m/8) * 2^(e-7) */
    return s ? -v : v;
}

/* binary32 -> E4M3 "fn": the representable magnitudes are k * 2^-9 for
 * k < 8 (subnormals) and (8 + m) * 2^(e-10) for e = 1..15, m = 0..7 (except
 * e = 15, m = 7, which is NaN); 448 is the largest.  Round to nearest, ties to
 * the even code; a magnitude that rounds past 448 saturates to 448. */
uint8_t or_f32_to_e4m3(float f)
{
    if (f != f)
        return 0x7Fu;
    uint8_t sign = signbit(f) ? 0x80u : 0u;
    double a = fabs((double)f);
    if (a >= 464.0)                          /* halfway to the next step (480): saturate */
        return (uint8_t)(sign | 0x7Eu);
    /* scan the 127 non-negative finite codes in order for the nearest value */
    uint8_t best = 0;
    double bestd = a;                        /* code 0 stands for 0 */
    for (int c = 1; c <= 0x7E; c++) {
        double v = (double)or_e4m3_to_f32((uint8_t)c);
        double d = fabs(v - a);
        if (d < bestd || (d == bestd && (c & 1) == 0)) {
            best = (uint8_t)c;
            bestd = d;
        }
    }
    return (uint8_t)(sign | best);
}

/* OCP 4-bit E2M1: s | 2-bit exponent (bias 1) | 1-bit mantissa;
 * magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
float or_e2m1_to_f32(uint8_t c)
{
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    float v = (e == 0) ? 0.5f * (float)m : ldexpf((float)(2 + m), e - 2);
    return s ? -v : v;
}

/* ------------------------------------------------------------ dequantize */

void or_dequant_row(const or_qmat *w, int n, float *out)
{
    const int K = w->K;
    if (w->fmt == OR_FMT_Q4_0) {
        /* w = d * (q - 8); d is the block's fp16 scale */
        const uint8_t *row = w->q + (size_t)n * (size_t)(K / 32) * 18u;
        for (int b = 0; b < K / 32; b++) {
            const uint8_t *blk = row + (size_t)b * 18u;
            float d = or_fp16_to_f32((uint16_t)(blk[0] | (blk[1] << 8)));
            for (int j = 0; j < 16; j++) {
                int lo = blk[2 + j] & 15;
                int hi = blk[2 + j] >> 4;
                out[b * 32 + j] = d * (float)(lo - 8);
                out[b * 32 + j + 16] = d * (float)(hi - 8);
            }
        }
    } else {
        /* w = (e2m1(q) * e4m3(s)) * ts.  The 16 E2M1 values are the decoder's
         * own outputs, looked up; each block's E4M3 scale is decoded once. */
        float e2m1[16];
        for (int c = 0; c < 16; c++)
            e2m1[c] = or_e2m1_to_f32((uint8_t)c);
        const uint8_t *row = w->q + (size_t)n * (size_t)(K / 2);
        const uint8_t *sc = w->s + (size_t)n * (size_t)(K / 16);
        for (int b = 0; b < K / 16; b++) {
            float blk_scale = or_e4m3_to_f32(sc[b]);
            for (int j = 0; j < 16; j++) {
                int k = b * 16 + j;
                uint8_t byte = row[k / 2];
                uint8_t code = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
                out[k] = (e2m1[code] * blk_scale) * w->ts;
            }
        }
    }
}

void or_matvec(const or_qmat *w, const float *x, float *y)
{
    float *row = (float *)malloc(sizeof(float) * (size_t)w->K);
    for (int n = 0; n < w->N; n++) {
        or_dequant_row(w, n, row);
        float acc = 0.0f;
        for (int k = 0; k < w->K; k++)
            acc += row[k] * x[k];
        y[n] = acc;
    }
    free(row);
}

/* ------------------------------------------------------------ elementwise */

void or_rmsnorm(const float *x, const float *gamma, int H, float eps, float *y)
{
    float ss = 0.0f;
    for (int i = 0; i < H; i++)
        ss += x[i] * x[i];
    float r = 1.0f / sqrtf(ss / (float)H + eps);
    for (int i = 0; i < H; i++)
        y[i] = (x[i] * r) * gamma[i];
}

/* Rotate-half RoPE: dimension pairs (i, i + hd/2) rotate by pos * theta^(-2i/hd).
 * The angle, cosine and sine are evaluated in double, then rounded to fp32. */
void or_rope(float *v, int hd, int pos, float theta)
{
    int half = hd / 2;
    for (int i = 0; i < half; i++) {
        double inv_freq = pow((double)theta, -2.0 * (double)i / (double)hd);
        double ang = (double)pos * inv_freq;
        float c = (float)cos(ang);
        float s = (float)sin(ang);
        float a = v[i], b = v[i + half];
        v[i] = a * c - b * s;
        v[i + half] = b * c + a * s;
    }
}

float or_silu(float z)
{
    return z / (1.0f + expf(-z));
}

/* --------------------------------------------------------------- attention */

static const uint16_t *kv_row(const uint16_t *pool, const or_kv *kv, int b, int nkv,
                              int kvh, int hd, int pos)
{
    if (pos < 0 || pos / kv->page_tokens >= kv->max_pages)
        return NULL;        /* outside the page table: no row */
    int32_t page = kv->page_table[(size_t)b * (size_t)kv->max_pages + (size_t)(pos / kv->page_tokens)];
    if (page < 0 || page >= kv->n_pages)
        return NULL;
    size_t off = (((size_t)page * (size_t)nkv + (size_t)kvh) * (size_t)kv->page_tokens +
                  (size_t)(pos % kv->page_tokens)) * (size_t)hd;
    return pool + off;
}

void or_attend_head(const float *q, const uint16_t *kpool, const uint16_t *vpool,
                    const or_kv *kv, int b, int nkv, int kvh, int hd, int len, float *out)
{
    float scale = 1.0f / sqrtf((float)hd);
    float *s = (float *)malloc(sizeof(float) * (size_t)len);
    for (int j = 0; j < len; j++) {
        const uint16_t *kr = kv_row(kpool, kv, b, nkv, kvh, hd, j);
        if (!kr) {
            for (int d = 0; d < hd; d++)
                out[d] = NAN;
            free(s);
            return;
        }
        float dot = 0.0f;
        for (int d = 0; d < hd; d++)
            dot += q[d] * or_fp16_to_f32(kr[d]);
        s[j] = dot * scale;
    }
    /* softmax in two passes: maximum, then exponentials and their sum */
    float m = s[0];
    for (int j = 1; j < len; j++)
        if (s[j] > m)
            m = s[j];
    float l = 0.0f;
    for (int j = 0; j < len; j++) {
        s[j] = expf(s[j] - m);
        l += s[j];
    }
    for (int d = 0; d < hd; d++) {
        float acc = 0.0f;
        for (int j = 0; j < len; j++) {
            const uint16_t *vr = kv_row(vpool, kv, b, nkv, kvh, hd, j);
            acc += s[j] * or_fp16_to_f32(vr[d]);
        }
        out[d] = acc / l;
    }
    free(s);
}

/* Element offset of the row of (b, kvh, pos) in a layer pool, or -1 when its
 * page-table entry is outside the pool or pos is outside the table. */
static long kv_row_off(const or_kv *kv, int b, int nkv, int kvh, int hd, int pos)
{
    if (pos < 0 || pos / kv->page_tokens >= kv->max_pages)
        return -1;
    int32_t page = kv->page_table[(size_t)b * (size_t)kv->max_pages + (size_t)(pos / kv->page_tokens)];
    if (page < 0 || page >= kv->n_pages)
        return -1;
    return (long)((((size_t)page * (size_t)nkv + (size_t)kvh) * (size_t)kv->page_tokens +
                   (size_t)(pos % kv->page_tokens)) * (size_t)hd);
}

void or_attend_head_e4m3(const float *q, const uint8_t *kpool, const uint8_t *vpool, float k_scale,
                         float v_scale, const or_kv *kv, int b, int nkv, int kvh, int hd, int len,
                         float *out)
{
    float scale = 1.0f / sqrtf((float)hd);
    float *s = (float *)malloc(sizeof(float) * (size_t)len);
    for (int j = 0; j < len; j++) {
        long off = kv_row_off(kv, b, nkv, kvh, hd, j);
        if (off < 0) {
            for (int d = 0; d < hd; d++)
                out[d] = NAN;
            free(s);
            return;
        }
        float dot = 0.0f;
        for (int d = 0; d < hd; d++)
            dot += q[d] * (or_e4m3_to_f32(kpool[off + d]) * k_scale);
        s[j] = dot * scale;
    }
    float m = s[0];
    for (int j = 1; j < len; j++)
        if (s[j] > m)
            m = s[j];
    float l = 0.0f;
    for (int j = 0; j < len; j++) {
        s[j] = expf(s[j] - m);
        l += s[j];
    }
    for (int d = 0; d < hd; d++) {
        float acc = 0.0f;
        for (int j = 0; j < len; j++) {
            long off = kv_row_off(kv, b, nkv, kvh, hd, j);
            acc += s[j] * (or_e4m3_to_f32(vpool[off + d]) * v_scale);
        }
        out[d] = acc / l;
    }
    free(s);
}

/* ------------------------------------------------------------ MoE + argmax */

void or_topk_softmax(const float *r, int E, int k, int32_t *idx, float *w)
{
    char *used = (char *)calloc((size_t)E, 1);
    for (int t = 0; t < k; t++) {
        int best = -1;
        for (int e = 0; e < E; e++) {
            if (used[e])
                continue;
            if (best < 0 || r[e] > r[best])   /* strict: the lower index wins ties */
                best = e;
        }
        idx[t] = best;
        used[best] = 1;
    }
    float m = r[idx[0]];
    float sum = 0.0f;
    for (int t = 0; t < k; t++) {
        w[t] = expf(r[idx[t]] - m);
        sum += w[t];
    }
    for (int t = 0; t < k; t++)
        w[t] = w[t] / sum;
    free(used);
}

int32_t or_argmax(const float *v, int n, float *margin)
{
    int best = 0;
    for (int i = 1; i < n; i++)
        if (v[i] > v[best])
            best = i;
    if (margin) {
        float second = -INFINITY;
        for (int i = 0; i < n; i++)
            if (i != best && v[i] > second)
                second = v[i];
        *margin = v[best] - second;
    }
    return best;
}

int32_t or_spec_accept(const int32_t *rows, const int32_t *greedy, int n_rows, int32_t *next)
{
    int32_t n = 0;
    for (int i = 1; i < n_rows; i++) {
        if (rows[i] != greedy[i - 1])
            break;          /* first rejected draft: nothing after it stands */
        n++;
    }
    *next = greedy[n];
    return n;
}

/* ------------------------------------------------------------ draft head */

int32_t or_draft_token(const or_qmat *embed, const or_qmat *w_draft, const float *gamma, float eps,
                       const float *h, int32_t tok, float *g_out, float *z_out)
{
    const int H = embed->K;
    float *x = (float *)malloc(sizeof(float) * (size_t)H);
    float *z = z_out ? z_out : (float *)malloc(sizeof(float) * (size_t)w_draft->N);
    or_dequant_row(embed, tok, x);
    for (int i = 0; i < H; i++)
        x[i] = h[i] + x[i];
    or_rmsnorm(x, gamma, H, eps, g_out);
    or_matvec(w_draft, g_out, z);
    int32_t d = or_argmax(z, w_draft->N, NULL);
    free(x);
    if (!z_out)
        free(z);
    return d;
}

/* ------------------------------------------------------------- decode step */

/* SwiGLU feed-forward: Wd (silu(Wg y) * (Wu y)) */
static void ffn(const or_qmat *wg, const or_qmat *wu, const or_qmat *wd, const float *y, float *out)
{
    int F = wg->N;
    float *g = (float *)malloc(sizeof(float) * (size_t)F);
    float *u = (float *)malloc(sizeof(float) * (size_t)F);
    or_matvec(wg, y, g);
    or_matvec(wu, y, u);
    for (int i = 0; i < F; i++)
        g[i] = or_silu(g[i]) * u[i];
    or_matvec(wd, g, out);
    free(g);
    free(u);
}

int32_t or_decode_token(const or_model *m, or_kv *kv, int b, int32_t token, int pos,
                        int moe_dense, float *logits, float *hidden, int32_t *moe_idx,
                        float *margin, float *moe_logits)
{
    const int H = m->H, hd = m->hd, nq = m->nq, nkv = m->nkv;
    const int nqkv = (nq + 2 * nkv) * hd;
    float *x = (float *)malloc(sizeof(float) * (size_t)H);
    float *y = (float *)malloc(sizeof(float) * (size_t)H);
    float *t = (float *)malloc(sizeof(float) * (size_t)H);
    float *qkv = (float *)malloc(sizeof(float) * (size_t)nqkv);
    float *o = (float *)malloc(sizeof(float) * (size_t)(nq * hd));
    float *lg = logits ? logits : (float *)malloc(sizeof(float) * (size_t)m->V);

    or_dequant_row(&m->embed, token, x);
    if (hidden)
        memcpy(hidden, x, sizeof(float) * (size_t)H);

    for (int l = 0; l < m->L; l++) {
        const or_layer *ly = &m->layers[l];
        /* attention block */
        or_rmsnorm(x, ly->attn_norm, H, m->eps, y);
        or_matvec(&ly->wqkv, y, qkv);
        float *q = qkv, *k = qkv + nq * hd, *v = qkv + (nq + nkv) * hd;
        for (int h = 0; h < nq; h++)
            or_rope(q + h * hd, hd, pos, m->theta);
        for (int h = 0; h < nkv; h++)
            or_rope(k + h * hd, hd, pos, m->theta);
        for (int h = 0; h < nkv; h++) {
            if (kv->kv_fmt == 1) {
                long off = kv_row_off(kv, b, nkv, h, hd, pos);
                if (off < 0)
                    continue;   /* bad page: the attention below reports NaN */
                uint8_t *kr = (uint8_t *)kv->k[l] + off, *vr = (uint8_t *)kv->v[l] + off;
                for (int d = 0; d < hd; d++) {
                    kr[d] = or_f32_to_e4m3(k[h * hd + d] / kv->k_scale[l]);
                    vr[d] = or_f32_to_e4m3(v[h * hd + d] / kv->v_scale[l]);
                }
                continue;
            }
            uint16_t *kr = (uint16_t *)kv_row(kv->k[l], kv, b, nkv, h, hd, pos);
            uint16_t *vr = (uint16_t *)kv_row(kv->v[l], kv, b, nkv, h, hd, pos);
            if (!kr || !vr)
                continue;   /* bad page: the attention below reports NaN */
            for (int d = 0; d < hd; d++) {
                kr[d] = or_f32_to_fp16(k[h * hd + d]);
                vr[d] = or_f32_to_fp16(v[h * hd + d]);
            }
        }
        for (int h = 0; h < nq; h++) {
            int kvh = h / (nq / nkv);
            if (kv->kv_fmt == 1)
                or_attend_head_e4m3(q + h * hd, (const uint8_t *)kv->k[l], (const uint8_t *)kv->v[l],
                                    kv->k_scale[l], kv->v_scale[l], kv, b, nkv, kvh, hd, pos + 1, o + h * hd);
            else
                or_attend_head(q + h * hd, kv->k[l], kv->v[l], kv, b, nkv, kvh, hd, pos + 1, o + h * hd);
        }
        or_matvec(&ly->wo, o, t);
        for (int i = 0; i < H; i++)
            x[i] += t[i];

        /* feed-forward block */
        or_rmsnorm(x, ly->ffn_norm, H, m->eps, y);
        if (m->n_experts == 0) {
            ffn(&ly->wg, &ly->wu, &ly->wd, y, t);
            for (int i = 0; i < H; i++)
                x[i] += t[i];
        } else {
            const int E = m->n_experts, K = m->topk;
            float *r = (float *)malloc(sizeof(float) * (size_t)E);
            int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)K);
            float *w = (float *)malloc(sizeof(float) * (size_t)K);
            float *acc = (float *)calloc((size_t)H, sizeof(float));
            /* router: fp32 weights, r = Wr y */
            for (int e = 0; e < E; e++) {
                float a = 0.0f;
                for (int i = 0; i < H; i++)
                    a += ly->router[(size_t)e * (size_t)H + (size_t)i] * y[i];
                r[e] = a;
            }
            if (moe_logits)
                memcpy(moe_logits + (size_t)l * (size_t)E, r, sizeof(float) * (size_t)E);
            or_topk_softmax(r, E, K, sel, w);
            if (moe_idx)
                memcpy(moe_idx + (size_t)l * (size_t)K, sel, sizeof(int32_t) * (size_t)K);
            if (moe_dense) {
                float *all = (float *)malloc(sizeof(float) * (size_t)E * (size_t)H);
                for (int e = 0; e < E; e++)
                    ffn(&ly->eg[e], &ly->eu[e], &ly->ed[e], y, all + (size_t)e * (size_t)H);
                for (int s = 0; s < K; s++)
                    for (int i = 0; i < H; i++)
                        acc[i] += w[s] * all[(size_t)sel[s] * (size_t)H + (size_t)i];
                free(all);
            } else {
                for (int s = 0; s < K; s++) {
                    ffn(&ly->eg[sel[s]], &ly->eu[sel[s]], &ly->ed[sel[s]], y, t);
                    for (int i = 0; i < H; i++)
                        acc[i] += w[s] * t[i];
                }
            }
            ffn(&ly->sg, &ly->su, &ly->sd, y, t);   /* shared expert, weight 1 */
            for (int i = 0; i < H; i++)
                acc[i] += t[i];
            for (int i = 0; i < H; i++)
                x[i] += acc[i];
            free(r);
            free(sel);
            free(w);
            free(acc);
        }
        if (hidden)
            memcpy(hidden + (size_t)(l + 1) * (size_t)H, x, sizeof(float) * (size_t)H);
    }

    or_rmsnorm(x, m->final_norm, H, m->eps, y);
    or_matvec(&m->lm_head, y, lg);
    int32_t tok = or_argmax(lg, m->V, margin);

    free(x);
    free(y);
    free(t);
    free(qkv);
    free(o);
    if (!logits)
        free(lg);
    return tok;
}
