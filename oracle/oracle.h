/*
 * oracle.h -- plain, slow, single-threaded fp32 CPU reference of one greedy
 * decode step of a pre-norm transformer over 4-bit block-quantized weights.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or helper with the GPU library; the only thing both sides
 * share is the seeded input bytes they are handed.
 *
 * What the pages fix and what is read into them (sources, by page):
 *  - "bw24" deep-dive page (10100.com, "深入解析 bw24 ..."), section 1
 *    (project overview): greedy (argmax) decoding is the correctness gate;
 *    speculative (MTP) verification must reproduce token-by-token argmax
 *    decoding exactly; NVFP4 is a native weight format.
 *  - same page, section 6 ("Paged Cache"): logical sequence positions map to
 *    physical pages through a page table.
 *  - same page, section 5, stage 4 (MTP core logic): the verify pass expands
 *    K candidate tokens along the sequence dimension over one shared KV cache.
 *  - "Rust+CUDA ... bw24 ... llama.cpp" page (devpress), section 2.1: every new
 *    token reads the whole KV cache; section 2.2: SiLU / normalisation fused
 *    with the linear layers.
 *  - The block formats themselves (GGUF-style Q4_0: 32-weight blocks with an
 *    fp16 scale d and w = d*(q-8); NVFP4: 16-element E2M1 blocks, an E4M3 block
 *    scale and an fp32 tensor scale) are the workload definition that the
 *    pages only name ("Q4", "GGUF", "NVFP4").
 *
 * Precision: every floating-point step is IEEE binary32 with round-to-nearest
 * even, no FMA contraction (built with -ffp-contract=off), sums taken
 * sequentially in increasing index order.  K and V are rounded to fp16 when
 * written into the cache, because an fp16 cache is part of the workload.
 */
#ifndef BW_ORACLE_H
#define BW_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define OR_FMT_Q4_0 0
#define OR_FMT_NVFP4 1

/* One quantized weight matrix W[N][K] (row-major, y = W x) in its canonical
 * (file) layout.
 *  Q4_0 : q = N*(K/32) blocks of 18 bytes each, row-major; a block is the fp16
 *         scale d (little-endian) followed by 16 bytes qs; element j (0..15) of
 *         the block is the low nibble of qs[j], element j+16 the high nibble.
 *         s is unused, ts is unused.
 *  NVFP4: q = N*K/2 bytes of E2M1 codes, element 2i in the low nibble of byte
 *         i of its row; s = N*K/16 E4M3 block scales; ts = fp32 tensor scale. */
typedef struct {
    int fmt;
    int N;
    int K;
    const uint8_t *q;
    const uint8_t *s;
    float ts;
} or_qmat;

typedef struct {
    const float *attn_norm;   /* gamma [H] */
    const float *ffn_norm;    /* gamma [H] */
    or_qmat wqkv;             /* [(nq + 2 nkv) hd][H]: q rows, then k, then v */
    or_qmat wo;               /* [H][nq hd] */
    /* dense FFN */
    or_qmat wg, wu;           /* [F][H] */
    or_qmat wd;               /* [H][F] */
    /* MoE FFN (n_experts > 0) */
    const float *router;      /* fp32 [E][H] */
    const or_qmat *eg, *eu;   /* E matrices [Fe][H] */
    const or_qmat *ed;        /* E matrices [H][Fe] */
    or_qmat sg, su, sd;       /* shared expert, weight 1 */
} or_layer;

typedef struct {
    int L, H, nq, nkv, hd, F, V;
    int n_experts, topk, F_exp;   /* n_experts == 0: dense model */
    float eps, theta;
    or_qmat embed;                /* [V][H] */
    or_qmat lm_head;              /* [V][H] */
    const float *final_norm;      /* [H] */
    const or_layer *layers;       /* L entries */
} or_model;

/* Paged KV cache: k[l] and v[l] point at the pool of layer l, laid out
 * [n_pages][nkv][page_tokens][hd].  The page table maps logical page j of
 * sequence b to physical page page_table[b*max_pages + j]; all layers use the
 * same physical page index.
 *  kv_fmt 0: fp16 bit patterns (the workload's cache format);
 *  kv_fmt 1: E4M3 bytes with per-layer fp32 scales k_scale[l], v_scale[l]
 *            (the FP8 variant: a value x is written as e4m3(x / scale) and
 *            read as e4m3(code) * scale). */
typedef struct {
    uint16_t **k;
    uint16_t **v;
    int n_pages;
    int page_tokens;
    const int32_t *page_table;
    int max_pages;
    int kv_fmt;
    const float *k_scale;
    const float *v_scale;
} or_kv;

/* scalar decoders (IEEE-754 binary16; OCP 8-bit E4M3 "fn"; OCP 4-bit E2M1) */
float or_fp16_to_f32(uint16_t h);
uint16_t or_f32_to_fp16(float f);          /* round to nearest even */
float or_e4m3_to_f32(uint8_t c);
float or_e2m1_to_f32(uint8_t c);
/* binary32 -> E4M3 "fn", round to nearest, ties to even; magnitudes that
 * round above 448 saturate to 448 (a KV cache never stores NaN); NaN -> 0x7F. */
uint8_t or_f32_to_e4m3(float f);

/* dequantize row n of W into out[K] */
void or_dequant_row(const or_qmat *w, int n, float *out);
/* y[n] = sum_k W[n][k] x[k], sequential fp32 */
void or_matvec(const or_qmat *w, const float *x, float *y);
/* y = x * rsqrt(mean(x^2) + eps) * gamma */
void or_rmsnorm(const float *x, const float *gamma, int H, float eps, float *y);
/* rotate-half RoPE of one head vector at position pos */
void or_rope(float *v, int hd, int pos, float theta);
float or_silu(float z);
/* one query head attending over logical positions 0..len-1 of sequence b,
 * kv head kvh of layer pool (kpool, vpool); out[hd] */
void or_attend_head(const float *q, const uint16_t *kpool, const uint16_t *vpool,
                    const or_kv *kv, int b, int nkv, int kvh, int hd, int len, float *out);
/* The same head over an E4M3 cache (the FP8 KV variant; one fp32 scale per
 * layer for K and one for V): a stored code c stands for e4m3(c) * scale,
 * the scale applied to each decoded element; pools are bytes
 * [n_pages][nkv][page_tokens][hd] behind kv's page table.  Otherwise
 * identical to or_attend_head. */
void or_attend_head_e4m3(const float *q, const uint8_t *kpool, const uint8_t *vpool, float k_scale,
                         float v_scale, const or_kv *kv, int b, int nkv, int kvh, int hd, int len,
                         float *out);
/* top-k of r[E]: value descending, lower index first on ties; softmax weights
 * over the selected values */
void or_topk_softmax(const float *r, int E, int k, int32_t *idx, float *w);
/* lowest index of the maximum; *margin = max - second largest value */
int32_t or_argmax(const float *v, int n, float *margin);
/* Speculative verify acceptance ("bw24" deep-dive page, section 5, stage 4;
 * section 1: speculative output == greedy output).  rows[0..n_rows) are the
 * tokens the verify pass ran (the last accepted token, then the drafts);
 * greedy[r] is the greedy token after row r.  Returns the number of drafts
 * accepted, n: drafts are taken in order while each one equals the greedy
 * token of the row before it.  *next = greedy[n]. */
int32_t or_spec_accept(const int32_t *rows, const int32_t *greedy, int n_rows, int32_t *next);

/* Speculative draft head (the deep-dive page, section 7: a light draft head
 * that shares the main model's embedding, with its output vocabulary pruned
 * to a fraction of the full one).  The pages fix no further detail; the
 * reading taken here:
 *   g = rmsnorm(h + deq(E)[tok]) * gamma     (h: the main model's residual
 *                                             stream after its last layer)
 *   z = deq(W_draft) g                       (W_draft: V_draft x H, the first
 *                                             V_draft token ids)
 *   draft = lowest index of max z; g_out[H] <- g, the h of the next draft.
 * z_out [V_draft] may be NULL. */
int32_t or_draft_token(const or_qmat *embed, const or_qmat *w_draft, const float *gamma, float eps,
                       const float *h, int32_t tok, float *g_out, float *z_out);

/* One greedy decode token of sequence b at position pos (writes its K/V into
 * the cache, attends over positions 0..pos).  logits [V] may be NULL;
 * hidden [(L+1)*H] (residual stream after the embedding and after each layer)
 * may be NULL; moe_idx [L*topk] (selected experts) and moe_logits [L*E]
 * (each layer's router logits) may be NULL.
 * moe_dense != 0 evaluates every expert and then combines the selected ones
 * (identical result; a self-check of the sparse path).  Returns the argmax
 * token; *margin receives the top-2 logit margin when non-NULL. */
int32_t or_decode_token(const or_model *m, or_kv *kv, int b, int32_t token, int pos,
                        int moe_dense, float *logits, float *hidden, int32_t *moe_idx,
                        float *margin, float *moe_logits);

#ifdef __cplusplus
}
#endif
#endif
