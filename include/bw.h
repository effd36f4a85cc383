/*
 * bw.h -- C ABI of the B200 (sm_100a) decode hot path.
 *
 * One call = one piece of one greedy decode step, run asynchronously on a CUDA
 * stream over caller-owned device memory.  What each call computes, and where
 * the pages define it:
 *
 *   bw_gemv_q4_0 / bw_gemv_nvfp4 -- y = W x over 4-bit block-quantized W, with
 *       an RMSNorm prologue, residual-add / SiLU-gate epilogues and an argmax
 *       reduction fused in.  "Rust+CUDA ... bw24 vs llama.cpp" page (devpress),
 *       section 2.2: linear layer, bias and activation fused in one kernel so
 *       intermediates stay in registers / shared memory; "bw24" deep-dive page
 *       (10100.com), section 7 (comparison table): Q4 GGUF weights and native
 *       NVFP4.  Block formats: GGUF-style Q4_0 (32 weights, fp16 d,
 *       w = d*(q-8)) and NVFP4 (16 E2M1 codes, E4M3 block scale, fp32 tensor
 *       scale, w = e2m1*e4m3*ts).
 *   bw_rmsnorm_fused -- x += add; y = x * rsqrt(mean(x^2) + eps) * gamma.
 *   bw_paged_attn_decode -- RoPE of the new rows' q and k, fp16 K/V write into
 *       the paged cache, GQA attention over the cache.  Deep-dive page,
 *       section 6 ("Paged Cache": logical positions -> physical pages through
 *       a page table) and section 5, stage 4 (the verify pass expands the K
 *       draft tokens along the sequence dimension over one shared cache);
 *       devpress page, section 2.1 (every token reads the whole cache).
 *   bw_moe_route_gemv -- router GEMV, top-k softmax, grouped expert SwiGLU
 *       GEMVs and the shared expert.  Deep-dive page, section 7: router
 *       ordering and expert parallelism without warp divergence.
 *   bw_argmax -- greedy sampling: the lowest index of the maximum.  Deep-dive
 *       page, section 1: the argmax token sequence is the correctness gate.
 *   bw_spec_accept -- the accepted draft count after a verify pass.
 *   bw_decode_step -- the whole step (embedding .. argmax) for B sequences of
 *       n_rows consecutive tokens each (n_rows = 1: decode; n_rows = K+1:
 *       speculative verify).  Deep-dive page, section 4: an engine facade
 *       exposing prefill and decode.
 *
 * Conventions (all entry points):
 *  - Pointers are DEVICE pointers owned by the caller unless a comment says
 *    "host".  The library never allocates, frees or synchronizes on these
 *    paths (bw_read_error is the one call that synchronizes).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *    kernel call is asynchronous on it.
 *  - Host threads may call the entry points concurrently (each with its own
 *    workspace): the library's host-side caches (SM counts, kernel
 *    attributes, tensor maps) are guarded by locks.
 *  - Arguments are validated on the host before any launch; a failed check
 *    returns BW_ERR_INVALID_ARG or BW_ERR_UNSUPPORTED_SHAPE and launches
 *    nothing.  A launch failure returns BW_ERR_CUDA.  Conditions only the
 *    device can see (a page-table entry outside the pool) set a bit in the
 *    error word at the start of the workspace; read it with bw_read_error
 *    after the stream has drained.  No exception crosses the ABI.
 *  - Workspace: scratch device memory of at least the queried size, 256-byte
 *    aligned (any other address returns BW_ERR_INVALID_ARG), zero-filled
 *    ONCE before first use (bw_workspace_init).  Kernels
 *    leave their counters at zero on return, so the same workspace serves
 *    any number of later calls and CUDA-graph replays on one stream.  Calls
 *    sharing a workspace must not run concurrently.
 *  - Kernels start early (programmatic dependent launch): they may read
 *    model data -- weights, scales, norm gains, router, RoPE table -- while
 *    the previous kernel on the stream is still running, and wait for it
 *    only before reading activations, KV or token inputs.  Model data must
 *    therefore not be written by work still in flight on the stream.
 *  - Weights live in the tiled GPU layout written by bw_repack_q4_0 /
 *    bw_repack_nvfp4 from the canonical (file) layout.  W[N][K] is cut into
 *    tiles of 128 rows x 512 columns (N padded to a multiple of 128 rows and
 *    K to a multiple of 512 columns, with zeros); tiles follow each other in
 *    (row block, column tile) order:
 *      q : per tile 32 KB: row r at r*256 bytes, 32-column chunk c of that
 *          row in the 16-byte slot c ^ (r & 7) (the chunk's 16 code bytes in
 *          the canonical nibble order of the format)
 *      s : per tile 4 KB: 8-row group g at g*256 bytes, chunk c at +c*16:
 *          the 8 rows' fp16 d (Q4_0) or 8 x 2 E4M3 block scales (NVFP4)
 *    so every tile is two contiguous blocks (streamed with plain bulk
 *    copies).  Sizes: bw_repack_bytes.  Gate/up matrices are interleaved in
 *    groups of 4 rows (rows 8g..8g+3 are gate rows 4g..4g+3, rows 8g+4..8g+7
 *    the matching up rows).
 */
#ifndef BW_H
#define BW_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BW_ABI_VERSION 1

typedef int bw_status;
#define BW_OK 0
#define BW_ERR_INVALID_ARG 1
#define BW_ERR_UNSUPPORTED_SHAPE 2
#define BW_ERR_CUDA 3
#define BW_ERR_DEVICE_TIMEOUT 4
#define BW_ERR_BAD_PAGE_INDEX 5

/* bits of the device error word (first 4 bytes of a workspace) */
#define BW_DEVERR_BAD_PAGE 1u
#define BW_DEVERR_TIMEOUT 2u
#define BW_DEVERR_BAD_TOKEN 4u
#define BW_DEVERR_BAD_POS 8u      /* position outside the page table or the RoPE table */

#define BW_FMT_Q4_0 0
#define BW_FMT_NVFP4 1

#define BW_KV_FP16 0
#define BW_KV_E4M3 1

/* GEMV flags */
#define BW_GEMV_RMSNORM 1u    /* prologue: each row of x -> rmsnorm(x) * gamma */
#define BW_GEMV_RESIDUAL 2u   /* epilogue: y = residual + W x (residual may alias y) */
#define BW_GEMV_SILU_GATE 4u  /* rows interleaved gate/up: y[m][i] = silu(g_i) * u_i, N/2 outputs */
#define BW_GEMV_ARGMAX 8u     /* also argmax_out[m] = lowest index of max_n (W x)[m][n] */

/* decode-step flags */
#define BW_STEP_ADVANCE 1u    /* after the step: tokens_in <- tokens_out, pos += n_rows */
#define BW_STEP_VALIDATE_ONLY 2u  /* validate descriptors and arguments on the host; launch nothing */
#define BW_STEP_PERSISTENT 4u /* batch-1 dense step as one persistent kernel (else: the per-layer chain) */
#define BW_MAX_VERIFY_ROWS 8  /* n_rows limit of a verify pass (the last token + up to 7 drafts) */

/* Human-readable name of a status code (static string, never NULL). */
const char *bw_status_string(bw_status s);
/* BW_ABI_VERSION of the loaded library. */
int bw_abi_version(void);

/* ------------------------------------------------------------- workspace */

/* Zero-fill `bytes` of workspace on `stream` (once, before first use). */
bw_status bw_workspace_init(void *ws, size_t bytes, void *stream);
/* Synchronize `stream`, then copy the device error word of `ws` into
 * *err_out (host) and clear it on the device.  ws == NULL reads the error word
 * of bw_gemv_q4_0_noalloc's fixed scratch on the current device instead. */
bw_status bw_read_error(void *ws, uint32_t *err_out, void *stream);
/* Asynchronous form of bw_read_error: enqueue on `stream`, after everything
 * already queued there, one tiny kernel that ORs the device error word of `ws`
 * (NULL: bw_gemv_q4_0_noalloc's fixed scratch on the current device) into
 * *dst and clears the word.  dst is DEVICE memory (4-byte aligned) owned by
 * the caller; nothing synchronizes, so the call can be captured in a CUDA
 * graph -- e.g. after every step of a multi-step graph, with one copy of
 * *dst to the host at the end.  Returns BW_ERR_INVALID_ARG (nothing queued)
 * for a NULL or misaligned dst or a misaligned ws. */
bw_status bw_drain_error(void *ws, uint32_t *dst, void *stream);

/* ---------------------------------------------------------------- layout */

/* Bytes of the tiled codes (*q_bytes) and scales (*s_bytes) of a matrix of
 * `rows` rows (2N for gate/up) and K columns in the GPU layout. */
bw_status bw_repack_bytes(int rows, int K, size_t *q_bytes, size_t *s_bytes);
/* Canonical Q4_0 (N x K/32 blocks of 18 bytes) -> tiled GPU layout.
 * blocks_up != NULL: gate/up interleave of two N x K matrices; the output
 * then has 2N rows.  q_out / s_out: bw_repack_bytes() each, 16-byte aligned
 * (the padding is zero-filled).  Requires K % 32 == 0, rows % 8 == 0
 * (N % 4 == 0 for gate/up). */
bw_status bw_repack_q4_0(const void *blocks, const void *blocks_up, int N, int K,
                         void *q_out, void *s_out, void *stream);
/* Canonical NVFP4 (codes [N][K/2], E4M3 scales [N][K/16]) -> tiled GPU
 * layout; q_up/s_up != NULL: gate/up interleave as above. */
bw_status bw_repack_nvfp4(const void *q, const void *s, const void *q_up, const void *s_up,
                          int N, int K, void *q_out, void *s_out, void *stream);

/* ------------------------------------------------------------------ GEMV */

/* y[m][n] = sum_k W[n][k] x'[m][k] for m < M, with x' = x or, with
 * BW_GEMV_RMSNORM, x' = x * rsqrt(mean(x^2) + eps) * gamma.
 *   x: fp32 [M][K]; y: fp32 [M][N] ([M][N/2] with SILU_GATE; may be NULL
 *   with ARGMAX); residual: fp32 [M][N] or NULL; argmax_out: int32 [M] or NULL;
 *   gamma: fp32 [K] or NULL.
 * Shapes: N % 8 == 0, K % 32 == 0, M >= 1 (Q4_0 runs in passes of up to 4
 * rows on the CUDA cores; NVFP4 with M > 4 runs on the tensor cores in passes
 * of up to 32 rows, with fp16-rounded activations).  Pointers 16-byte
 * aligned; fmt-specific shape limits return BW_ERR_UNSUPPORTED_SHAPE.
 * ws must hold bw_gemv_workspace_bytes(N, K, M, flags). */
bw_status bw_gemv_q4_0(const void *w_q, const void *w_d, int N, int K,
                       const float *x, int M, const float *gamma, float eps,
                       const float *residual, float *y, int32_t *argmax_out,
                       unsigned flags, void *ws, size_t ws_bytes, void *stream);
/* Same contract; ts is the tensor scale of all rows, or of the gate rows
 * with SILU_GATE, in which case ts_up scales the up rows. */
bw_status bw_gemv_nvfp4(const void *w_q, const void *w_s, float ts, float ts_up, int N, int K,
                        const float *x, int M, const float *gamma, float eps,
                        const float *residual, float *y, int32_t *argmax_out,
                        unsigned flags, void *ws, size_t ws_bytes, void *stream);
size_t bw_gemv_workspace_bytes(int N, int K, int M, unsigned flags);

/* Size of the fixed device scratch behind bw_gemv_q4_0_noalloc (1 MiB). */
#define BW_GEMV_NOALLOC_SCRATCH_BYTES (1u << 20)
/* bw_gemv_q4_0 without a workspace argument, for callers that cannot allocate
 * device memory (a host framework that owns every allocation and passes a
 * library only inputs and outputs, or a path where cudaMalloc's implicit
 * synchronization is not acceptable).  No counterpart in the pages: a
 * library-interface addition.
 *   Same arguments, layout and results as bw_gemv_q4_0 (the same kernel and
 *   split plan, so the outputs are bit-identical).  The scratch is a
 *   file-scope __device__ array of BW_GEMV_NOALLOC_SCRATCH_BYTES that every
 *   GPU loading the library holds until process exit; nothing is allocated
 *   or freed (it issues one cudaMemsetAsync to clear its counters, after
 *   every argument check has passed).
 *   Device-side conditions (a bounded wait that ran out) set bits in the
 *   array's error word, which calls do not clear: read and clear it with
 *   bw_read_error(NULL, &err, stream).
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.
 *   All calls share the one array: calls that overlap on the GPU (other
 *   streams, other host threads) race and must be serialized by the caller.
 *   A shape whose split-K scratch exceeds the array returns
 *   BW_ERR_UNSUPPORTED_SHAPE without launching. */
bw_status bw_gemv_q4_0_noalloc(const void *w_q, const void *w_d, int N, int K,
                               const float *x, int M, const float *gamma, float eps,
                               const float *residual, float *y, int32_t *argmax_out,
                               unsigned flags, void *stream);

/* -------------------------------------------------------- small kernels */

/* x [M][H] fp32 in place: x += add (if add != NULL); y = rmsnorm(x) * gamma,
 * written as fp32 (y_fp16 == 0) or fp16 (y_fp16 != 0) [M][H].  y may be NULL. */
bw_status bw_rmsnorm_fused(float *x, const float *add, const float *gamma, int M, int H,
                           float eps, void *y, int y_fp16, void *stream);

/* x[m][:] = dequantized row tokens[m] of the embedding matrix (tiled GPU layout,
 * e_q / e_s 16-byte aligned).  A token outside [0, V) sets BW_DEVERR_BAD_TOKEN
 * in ws's error word (ws optional; when given, a workspace as above) and
 * writes zeros. */
bw_status bw_embed(int fmt, const void *e_q, const void *e_s, float ts, int V, int H,
                   const int32_t *tokens, int M, float *x, void *ws, void *stream);

/* cos/sin of pos * theta^(-2i/hd), evaluated in fp64 and rounded to fp32:
 * [max_pos][hd/2] each. */
bw_status bw_rope_table(float theta, int hd, int max_pos, float *cos_out, float *sin_out,
                        void *stream);

/* idx_out[m] = lowest index of the maximum of logits[m][0..V); margin_out[m]
 * (optional) = max - second largest value. */
bw_status bw_argmax(const float *logits, int M, int V, int32_t *idx_out, float *margin_out,
                    void *stream);

/* ------------------------------------------------------------- attention */

/* Paged GQA decode attention for B sequences x n_rows consecutive query rows.
 *   qkv: fp32 [B*n_rows][(nq + 2 nkv) hd] raw projections (q heads, k heads,
 *        v heads); row b*n_rows + r sits at position pos[b] + r.
 *   rope_cos/rope_sin: fp32 [rope_max_pos][hd/2] (bw_rope_table).
 *   k_pool/v_pool: fp16 [n_pages][nkv][16][hd] of this layer.  The RoPE'd k
 *        and the v of every row are rounded to fp16 and written at logical
 *        position pos[b] + r (physical page page_table[b][pos/16], slot pos%16).
 *   page_table: int32 [B][max_pages]; pos: int32 [B].
 *   out: fp32 [B*n_rows][nq hd]; row r of sequence b attends over positions
 *        0 .. pos[b] + r (causal within the rows); query head h reads kv head
 *        h / (nq / nkv); scale 1/sqrt(hd); fp32 softmax.
 * Requires hd == 128 or 64, nq % nkv == 0, (nq/nkv) * n_rows <= 32,
 * n_rows <= 8, max_pages <= 8192 (else BW_ERR_UNSUPPORTED_SHAPE); qkv, out,
 * k_pool and v_pool 16-byte aligned (else BW_ERR_INVALID_ARG).
 * A page-table entry outside [0, n_pages) sets BW_DEVERR_BAD_PAGE; the page
 * is neither read nor written. */
bw_status bw_paged_attn_decode(const float *qkv, const float *rope_cos, const float *rope_sin,
                               int rope_max_pos, void *k_pool, void *v_pool,
                               const int32_t *page_table, int max_pages, int n_pages,
                               const int32_t *pos, int B, int n_rows, int nq, int nkv, int hd,
                               float *out, void *ws, size_t ws_bytes, void *stream);
/* The same over an E4M3 cache (bw_kv, kv_fmt BW_KV_E4M3): k_pool / v_pool are
 * byte pools in the fp16 pools' layout; k_scale, v_scale > 0 the layer's
 * scales.  The new rows are written as E4M3 codes of value / scale. */
bw_status bw_paged_attn_decode_fp8(const float *qkv, const float *rope_cos, const float *rope_sin,
                                   int rope_max_pos, void *k_pool, void *v_pool, float k_scale, float v_scale,
                                   const int32_t *page_table, int max_pages, int n_pages,
                                   const int32_t *pos, int B, int n_rows, int nq, int nkv, int hd,
                                   float *out, void *ws, size_t ws_bytes, void *stream);
size_t bw_attn_workspace_bytes(int B, int n_rows, int nq, int nkv, int hd, int max_pages);

/* ------------------------------------------------------------ whole step */

/* (bw_qweight, bw_layer, bw_model, bw_kv are declared below.) */
struct bw_model;
struct bw_layer;

typedef struct bw_qweight {
    int fmt;         /* BW_FMT_Q4_0 or BW_FMT_NVFP4 */
    int N, K;        /* rows in the GPU layout (2F for gate/up) and columns */
    const void *q;   /* GPU-layout nibbles */
    const void *s;   /* GPU-layout scales */
    float ts;        /* NVFP4 tensor scale (gate half for gate/up) */
    float ts_up;     /* NVFP4 tensor scale of the up half (gate/up); else ignored */
} bw_qweight;

typedef struct bw_layer {
    const float *attn_norm;  /* gamma [H] */
    const float *ffn_norm;   /* gamma [H] */
    bw_qweight wqkv;         /* [(nq + 2 nkv) hd][H] */
    bw_qweight wo;           /* [H][nq hd] */
    bw_qweight wgu;          /* dense: gate/up interleaved [2F][H] */
    bw_qweight wd;           /* dense: [H][F] */
    /* MoE (n_experts > 0) */
    const float *router;     /* fp32 [E][H] */
    const void *egu_q, *egu_s;  /* experts' gate/up, E matrices [2Fe][H] back to back */
    const void *ed_q, *ed_s;    /* experts' down, E matrices [H][Fe] back to back */
    const float *egu_ts;     /* fp32 [E][2]: gate and up tensor scales per expert */
    const float *ed_ts;      /* fp32 [E] */
    bw_qweight sgu, sd;      /* shared expert (weight 1) */
} bw_layer;

typedef struct bw_model {
    int L, H, nq, nkv, hd, F, V;
    int n_experts, topk, F_exp;  /* n_experts == 0: dense FFN */
    float eps;
    bw_qweight embed;            /* [V][H] */
    bw_qweight lm_head;          /* [V][H] */
    const float *final_norm;     /* [H] */
    const float *rope_cos, *rope_sin;
    int rope_max_pos;
    const bw_layer *layers;      /* HOST array of L layers */
} bw_model;

typedef struct bw_kv {
    void *const *k;              /* HOST array of L device pointers: fp16 [n_pages][nkv][16][hd] */
    void *const *v;
    int n_pages;
    int max_pages;
    const int32_t *page_table;   /* device int32 [B][max_pages] */
    /* BW_KV_FP16 (0), or BW_KV_E4M3 (1): the pools hold one byte per element in
     * the same layout, an OCP E4M3 code c standing for e4m3(c) * scale with one
     * fp32 scale per layer for K and one for V; a new row x is stored as the
     * E4M3 code of x / scale, rounded to nearest even and saturated to +-448.
     * The pages name FP8 on Blackwell (deep-dive page, section 7) without a
     * scheme; this per-layer scaling is the plainest one. */
    int kv_fmt;
    const float *k_scale;        /* HOST array of L fp32 scales (kv_fmt 1), each > 0 */
    const float *v_scale;
} bw_kv;

/* Mixture-of-experts feed-forward block of one layer for R token rows, in place:
 *   y = rmsnorm(x) * ffn_norm;  r = Wr y (router, fp32 [E][H]);
 *   top-k experts by logit (ties: the lower index); w = softmax over the k
 *   selected logits;  x += sum_k w_k FFN_{e_k}(y) + FFN_shared(y), where
 *   FFN(y) = Wd (silu(Wg y) * (Wu y)).
 *   x: fp32 [R][H]; topk_idx: int32 [R][topk] and topk_w: fp32 [R][topk]
 *   (optional outputs, in selection order).
 * Expert weights: m->layers-style bw_layer fields egu_* / ed_* (E matrices
 * back to back in the GPU layout) and sgu / sd (shared expert), all 16-byte
 * aligned and in one format.  Limits: E <= 1024, topk <= 16, R <= 256,
 * H % 32 == 0, F_exp % 32 == 0 (else BW_ERR_UNSUPPORTED_SHAPE).
 * ws must hold bw_moe_workspace_bytes(m, R). */
bw_status bw_moe_route_gemv(const struct bw_model *m, const struct bw_layer *ly, float *x, int R,
                            int32_t *topk_idx, float *topk_w, void *ws, size_t ws_bytes, void *stream);
size_t bw_moe_workspace_bytes(const struct bw_model *m, int R);

/* One greedy decode step for B sequences of n_rows tokens each.
 * The step runs as a chain of kernels (about five per layer).  With
 * BW_STEP_PERSISTENT a batch-1 step (B == 1, n_rows == 1) of a dense model runs
 * instead as ONE persistent cooperative kernel with a CTA per SM (streaming
 * every layer's weights and KV pages through a shared-memory ring, phases
 * ordered by device-side counters); both give the same results within the
 * tolerance of fp32 summation order.
 *   tokens_in: int32 [B*n_rows]; pos: int32 [B] (position of each sequence's
 *   first row); tokens_out: int32 [B*n_rows] (argmax after each row);
 *   logits: fp32 [B*n_rows][V] or NULL.
 * flags: BW_STEP_ADVANCE (n_rows == 1 only); BW_STEP_VALIDATE_ONLY runs every
 *   host-side check of the step (descriptor shapes and alignment, every
 *   launch's limits) and returns without touching the device -- the same
 *   checks a normal call makes before its first launch, so a rejected call
 *   never leaves a partial step queued.
 * ws must hold bw_decode_workspace_bytes(m, kv, B, n_rows). */
bw_status bw_decode_step(const bw_model *m, const bw_kv *kv, int32_t *tokens_in, int32_t *pos,
                         int B, int n_rows, int32_t *tokens_out, float *logits, unsigned flags,
                         void *ws, size_t ws_bytes, void *stream);
size_t bw_decode_workspace_bytes(const bw_model *m, const bw_kv *kv, int B, int n_rows);
/* Device address, inside ws, of the step's residual stream: fp32
 * [B*n_rows][H].  After bw_decode_step it holds each row's hidden state after
 * the last layer (the LM head's input before its RMSNorm) until the next call
 * on ws -- what a speculative draft head starts from.  Host arithmetic only;
 * NULL for arguments bw_decode_workspace_bytes would not size. */
const float *bw_decode_hidden(const bw_model *m, const bw_kv *kv, int B, int n_rows, const void *ws);
/* Device addresses, inside ws, of the expert choice of the last MoE layer the
 * latest bw_decode_step on ws ran: *idx = int32 [B*n_rows][topk] expert ids in
 * selection order (logit descending, ties to the lower id), *w = fp32
 * [B*n_rows][topk] their softmax weights.  Deep-dive page, section 7 (the
 * router's ordering of expert choices).  Host arithmetic only; valid until
 * the next call on ws.  BW_ERR_UNSUPPORTED_SHAPE for a dense model. */
bw_status bw_decode_moe_route(const bw_model *m, const bw_kv *kv, int B, int n_rows, const void *ws,
                              const int32_t **idx, const float **w);

/* Chunked prefill of one sequence: the prompt tokens[0..n-1] at positions
 * pos0 .. pos0 + n - 1.  "bw24" deep-dive page (10100.com), section 5, stage 3:
 * the prompt goes through in chunks, one after another; each chunk updates
 * the KV cache and only the last one returns logits.  Each chunk of up to
 * `chunk` tokens runs as one bw_decode_step with n_rows = the chunk's tokens
 * (rows causal within the chunk, each row's K/V written at its position), so
 * the cache and the result equal decoding the prompt one token at a time, up
 * to fp32 summation order.
 *   kv: its page table's FIRST row is the sequence (for sequence b of a
 *       batched cache, pass a bw_kv whose page_table points at row b);
 *   tokens: device int32 [n]; next_token: device int32 [1], the greedy token
 *   after the last prompt token; logits: device fp32 [V] of that last row, or
 *   NULL.
 * 1 <= chunk <= BW_MAX_VERIFY_ROWS, and the decode step's limits for n_rows =
 * chunk (nq / nkv * chunk <= 32) -- else BW_ERR_UNSUPPORTED_SHAPE;
 * pos0 + n <= min(16 * max_pages, rope_max_pos) -- else BW_ERR_INVALID_ARG.
 * Every chunk's checks run before the first launch.  Launches: one position
 * fill, then ceil(n / chunk) decode steps, then two device copies; graph
 * capturable.  ws must hold bw_prefill_workspace_bytes(m, kv, chunk) (the
 * decode step's workspace for n_rows = chunk comes first). */
bw_status bw_prefill(const bw_model *m, const bw_kv *kv, const int32_t *tokens, int n, int pos0, int chunk,
                     int32_t *next_token, float *logits, void *ws, size_t ws_bytes, void *stream);
size_t bw_prefill_workspace_bytes(const bw_model *m, const bw_kv *kv, int chunk);

/* Speculative draft head: K draft tokens for the next verify pass.  "bw24"
 * deep-dive page (10100.com), section 7 (a light MTP draft head sharing the
 * main model's embedding, its output vocabulary pruned to the first ids) and
 * section 5, stage 4 (the drafts become the rows of one verify pass).  The
 * page gives no formula; draft i = 1..K is
 *     x = h + E[t];  g = rmsnorm(x) * norm;  d_i = lowest index of max (w g)
 * with h <- g and t <- d_i for the next draft.  The first draft starts from
 * row *row (row == NULL: row 0) of `hidden` and t = tokens[0].
 *   hidden: fp32 [n_rows][H], the residual stream of the last step
 *           (bw_decode_hidden: a verify pass's rows, or a plain step's row);
 *   row:    optional int32 [1] on the device -- e.g. bw_spec_accept's n_accept
 *           of the pass that produced `hidden`, the row whose greedy token is
 *           tokens[0];
 *   tokens: int32 [K + 1]: tokens[0] in (the last emitted token); tokens[1..K]
 *           out (the drafts) -- the token row of the next verify pass.
 * B = 1; 1 <= K <= BW_MAX_VERIFY_ROWS - 1; H <= 12288.  A token or row outside
 * its range sets BW_DEVERR_BAD_TOKEN.  2K launches; graph capturable.
 * ws must hold bw_mtp_workspace_bytes(m, dh). */
typedef struct bw_draft_head {
    const float *norm;           /* gamma [H] */
    bw_qweight w;                /* [V_draft][H] over token ids 0 .. V_draft-1, in the model's format */
} bw_draft_head;
bw_status bw_mtp_draft(const bw_model *m, const bw_draft_head *dh, const float *hidden, int n_rows,
                       const int32_t *row, int32_t *tokens, int K, void *ws, size_t ws_bytes, void *stream);
size_t bw_mtp_workspace_bytes(const bw_model *m, const bw_draft_head *dh);

/* Acceptance after a speculative verify pass.  "bw24" deep-dive page
 * (10100.com), section 5, stage 4 (the verify kernel unrolls the drafts as
 * sequence rows and masks every row after the first mismatch) and section 1
 * (the speculative output equals plain greedy decoding token for token).
 *   tokens_in:  int32 [B*n_rows], the rows the pass ran: t0, d1 .. dK;
 *   tokens_out: int32 [B*n_rows], its greedy token a_r after each row r.
 *   n_accept:   int32 [B] out: n = the largest count with d_i == a_{i-1} for
 *               every i <= n.  The pass has then produced d1..dn, a_n.
 *   next_out:   optional; next_out[b*next_stride] = a_n (the next pass's t0).
 *               It may be tokens_in itself with stride n_rows.
 *   pos:        optional int32 [B]; pos[b] += n + 1 (KV rows past the accepted
 *               ones are stale and are overwritten by later passes).
 * Requires 1 <= n_rows <= BW_MAX_VERIFY_ROWS.  Device pointers; asynchronous
 * on stream; graph capturable. */
bw_status bw_spec_accept(const int32_t *tokens_in, const int32_t *tokens_out, int B, int n_rows,
                         int32_t *n_accept, int32_t *next_out, int next_stride, int32_t *pos,
                         void *stream);

#ifdef __cplusplus
}
#endif
#endif /* BW_H */
