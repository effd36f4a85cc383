// decode.cu -- one greedy decode step (embedding .. argmax) of a pre-norm
// transformer, as a chain of libbw kernels on one stream (sm_100a).
//
// Per layer: QKV GEMV (RMSNorm prologue) -> paged attention (RoPE + KV write)
// -> O GEMV (+ residual) -> gate/up GEMV (RMSNorm prologue, SiLU-gate
// epilogue) -> down GEMV (+ residual); then the LM-head GEMV with the final
// RMSNorm prologue and the greedy argmax fused in.  Every kernel is launched
// with programmatic dependent launch, so the next kernel's CTAs start
// streaming their weights while the previous one drains.  The chain is
// capturable in a CUDA graph; with BW_STEP_ADVANCE the argmax kernel also
// feeds the next step (token in, position + 1), so a graph of many steps
// decodes autoregressively without the host.
//
// With BW_STEP_PERSISTENT, a batch-1 step of a dense model runs instead as one
// persistent kernel (step_persistent.cu).
//
// The deep-dive page (10100.com), section 4, describes the engine facade that
// exposes prefill and decode; this is its decode call on device memory.
#include "bw_common.cuh"

namespace bw {

bw_status moe_ffn_launch(const bw_model *m, const bw_layer *ly, float *x, int R, const Scratch &sc,
                         char *moe_base, cudaStream_t st);
bw_status moe_check(const bw_model *m, const bw_layer *ly, int R);
size_t moe_scratch_bytes(const bw_model *m, int R);
void moe_route_buffers(const bw_model *m, int R, char *base, int32_t **sel, float **wts);
bool persistent_step_applies(const bw_model *m, int B, int n_rows);
size_t persistent_scratch_bytes(const bw_model *m);
bw_status persistent_step_launch(const bw_model *m, const bw_kv *kv, int32_t *tokens_in, int32_t *pos,
                                 int32_t *tokens_out, float *logits, bool advance, float *x, float *qkv, float *attn,
                                 float *act, char *scratch, const Scratch &sc, cudaStream_t st);

struct StepBuffers {
    float *x, *qkv, *attn, *act;
    char *moe;
    char *pk;       // scratch of the persistent batch-1 step (when it applies)
    Scratch kern;   // scratch shared by the kernels of the step
};

static size_t kernel_scratch_bytes(const bw_model *m, const bw_kv *kv, int B, int n_rows) {
    const int R = B * n_rows;
    const int nqkv = (m->nq + 2 * m->nkv) * m->hd;
    size_t s = attn_scratch_bytes(B, n_rows, m->nq, m->nkv, m->hd, kv->max_pages);
    s = max(s, gemv_scratch_bytes(nqkv, m->H, R));
    s = max(s, gemv_scratch_bytes(m->H, m->nq * m->hd, R));
    if (m->n_experts == 0) {
        s = max(s, gemv_scratch_bytes(2 * m->F, m->H, R));
        s = max(s, gemv_scratch_bytes(m->H, m->F, R));
    }
    s = max(s, gemv_scratch_bytes(m->V, m->H, R));
    return s;
}

static size_t step_bytes(const bw_model *m, const bw_kv *kv, int B, int n_rows, StepBuffers *bufs,
                         void *ws) {
    const int R = B * n_rows;
    const size_t nqkv = static_cast<size_t>(m->nq + 2 * m->nkv) * m->hd;
    Carver cv(ws ? static_cast<char *>(ws) + BW_WS_HDR_BYTES : nullptr);
    float *x = cv.take<float>(static_cast<size_t>(R) * m->H);
    float *qkv = cv.take<float>(R * nqkv);
    float *attn = cv.take<float>(static_cast<size_t>(R) * m->nq * m->hd);
    float *act = cv.take<float>(static_cast<size_t>(R) * max(m->F, 1));
    char *moe = m->n_experts ? cv.take<char>(moe_scratch_bytes(m, R)) : nullptr;
    char *pk = persistent_step_applies(m, B, n_rows) ? cv.take<char>(persistent_scratch_bytes(m)) : nullptr;
    const size_t kb = kernel_scratch_bytes(m, kv, B, n_rows);
    char *kbase = cv.take<char>(kb);
    if (bufs) {
        bufs->x = x;
        bufs->qkv = qkv;
        bufs->attn = attn;
        bufs->act = act;
        bufs->moe = moe;
        bufs->pk = pk;
        bufs->kern.err = ws ? ws_error_word(ws) : nullptr;
        bufs->kern.cnt = ws ? ws_counters(ws) : nullptr;
        bufs->kern.base = kbase;
        bufs->kern.bytes = kb;
    }
    return BW_WS_HDR_BYTES + cv.off;
}

static bool qw_ok(const bw_qweight &w, int N, int K, int fmt) {
    return w.q && w.s && w.N == N && w.K == K && w.fmt == fmt;
}

// Every launch of the step validated before the first is queued, with the
// arguments the launches below pass (same order, same buffers).
static bw_status step_check(const bw_model *m, const bw_kv *kv, const int32_t *tokens_in, const int32_t *pos, int B,
                            int n_rows, const int32_t *tokens_out, const float *logits, const StepBuffers &bf) {
    const int fmt = m->embed.fmt;
    const int R = B * n_rows;
    const int nqkv = (m->nq + 2 * m->nkv) * m->hd;
    bw_status s = embed_check(fmt, m->embed.q, m->embed.s, m->V, m->H, tokens_in, R, bf.x);
    for (int l = 0; l < m->L && s == BW_OK; l++) {
        const bw_layer &ly = m->layers[l];
        s = gemv_check(fmt, ly.wqkv.q, ly.wqkv.s, nqkv, m->H, bf.x, R, ly.attn_norm, nullptr, bf.qkv, nullptr,
                       BW_GEMV_RMSNORM, bf.kern);
        if (s == BW_OK)
            s = attn_check(bf.qkv, m->rope_cos, m->rope_sin, m->rope_max_pos, kv->k[l], kv->v[l], kv->page_table,
                           kv->max_pages, kv->n_pages, pos, B, n_rows, m->nq, m->nkv, m->hd, bf.attn, bf.kern);
        if (s == BW_OK)
            s = gemv_check(fmt, ly.wo.q, ly.wo.s, m->H, m->nq * m->hd, bf.attn, R, nullptr, bf.x, bf.x, nullptr,
                           BW_GEMV_RESIDUAL, bf.kern);
        if (s != BW_OK) break;
        if (m->n_experts == 0) {
            s = gemv_check(fmt, ly.wgu.q, ly.wgu.s, 2 * m->F, m->H, bf.x, R, ly.ffn_norm, nullptr, bf.act, nullptr,
                           BW_GEMV_RMSNORM | BW_GEMV_SILU_GATE, bf.kern);
            if (s == BW_OK)
                s = gemv_check(fmt, ly.wd.q, ly.wd.s, m->H, m->F, bf.act, R, nullptr, bf.x, bf.x, nullptr,
                               BW_GEMV_RESIDUAL, bf.kern);
        } else {
            s = moe_check(m, &ly, R);
            if (s == BW_OK && ly.sgu.fmt != fmt) s = BW_ERR_INVALID_ARG;
        }
    }
    if (s == BW_OK)
        s = gemv_check(fmt, m->lm_head.q, m->lm_head.s, m->V, m->H, bf.x, R, m->final_norm, nullptr, logits,
                       tokens_out, BW_GEMV_RMSNORM | BW_GEMV_ARGMAX, bf.kern);
    return s;
}

}  // namespace bw

extern "C" {

const float *bw_decode_hidden(const bw_model *m, const bw_kv *kv, int B, int n_rows, const void *ws) {
    if (!m || !kv || !ws || B <= 0 || n_rows <= 0) return nullptr;
    bw::StepBuffers bf;
    bw::step_bytes(m, kv, B, n_rows, &bf, const_cast<void *>(ws));
    return bf.x;
}

bw_status bw_decode_moe_route(const bw_model *m, const bw_kv *kv, int B, int n_rows, const void *ws,
                              const int32_t **idx, const float **w) {
    if (!m || !kv || !ws || B <= 0 || n_rows <= 0 || !idx || !w) return BW_ERR_INVALID_ARG;
    if (m->n_experts <= 0) return BW_ERR_UNSUPPORTED_SHAPE;
    bw::StepBuffers bf;
    bw::step_bytes(m, kv, B, n_rows, &bf, const_cast<void *>(ws));
    int32_t *sel = nullptr;
    float *wts = nullptr;
    bw::moe_route_buffers(m, B * n_rows, bf.moe, &sel, &wts);
    *idx = sel;
    *w = wts;
    return BW_OK;
}

size_t bw_decode_workspace_bytes(const bw_model *m, const bw_kv *kv, int B, int n_rows) {
    if (!m || !kv || B <= 0 || n_rows <= 0) return BW_WS_HDR_BYTES;
    return bw::step_bytes(m, kv, B, n_rows, nullptr, nullptr);
}

bw_status bw_decode_step(const bw_model *m, const bw_kv *kv, int32_t *tokens_in, int32_t *pos, int B,
                         int n_rows, int32_t *tokens_out, float *logits, unsigned flags, void *ws,
                         size_t ws_bytes, void *stream) {
    using namespace bw;
    if (!m || !kv || !tokens_in || !pos || !tokens_out || !ws_ok(ws) || B <= 0 || n_rows <= 0)
        return BW_ERR_INVALID_ARG;
    if (!m->layers || !kv->k || !kv->v || !kv->page_table || !m->rope_cos || !m->rope_sin ||
        !m->final_norm)
        return BW_ERR_INVALID_ARG;
    if ((flags & BW_STEP_ADVANCE) && n_rows != 1) return BW_ERR_INVALID_ARG;
    if (kv->kv_fmt != 0 && kv->kv_fmt != 1) return BW_ERR_INVALID_ARG;
    if (kv->kv_fmt == 1) {
        if (!kv->k_scale || !kv->v_scale) return BW_ERR_INVALID_ARG;
        for (int l = 0; l < m->L; l++)
            if (!(kv->k_scale[l] > 0.0f && kv->v_scale[l] > 0.0f && isfinite(kv->k_scale[l]) &&
                  isfinite(kv->v_scale[l])))
                return BW_ERR_INVALID_ARG;
    }
    const int fmt = m->embed.fmt;
    const int nqkv = (m->nq + 2 * m->nkv) * m->hd;
    if (!qw_ok(m->embed, m->V, m->H, fmt) || !qw_ok(m->lm_head, m->V, m->H, fmt))
        return BW_ERR_INVALID_ARG;
    for (int l = 0; l < m->L; l++) {
        const bw_layer &ly = m->layers[l];
        if (!ly.attn_norm || !ly.ffn_norm || !qw_ok(ly.wqkv, nqkv, m->H, fmt) ||
            !qw_ok(ly.wo, m->H, m->nq * m->hd, fmt) || !kv->k[l] || !kv->v[l])
            return BW_ERR_INVALID_ARG;
        if (m->n_experts == 0 &&
            (!qw_ok(ly.wgu, 2 * m->F, m->H, fmt) || !qw_ok(ly.wd, m->H, m->F, fmt)))
            return BW_ERR_INVALID_ARG;
    }
    StepBuffers bf;
    if (ws_bytes < step_bytes(m, kv, B, n_rows, &bf, ws)) return BW_ERR_INVALID_ARG;
    bw_status s = step_check(m, kv, tokens_in, pos, B, n_rows, tokens_out, logits, bf);
    if (s != BW_OK || (flags & BW_STEP_VALIDATE_ONLY)) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int R = B * n_rows;
    if (bf.pk && (flags & BW_STEP_PERSISTENT) && kv->kv_fmt == 0)
        return persistent_step_launch(m, kv, tokens_in, pos, tokens_out, logits, (flags & BW_STEP_ADVANCE) != 0,
                                      bf.x, bf.qkv, bf.attn, bf.act, bf.pk, bf.kern, st);

    s = embed_launch(fmt, m->embed.q, m->embed.s, m->embed.ts, m->V, m->H, tokens_in, R, bf.x,
                     bf.kern.err, st);
    if (s != BW_OK) return s;
    for (int l = 0; l < m->L; l++) {
        const bw_layer &ly = m->layers[l];
        s = gemv_launch(fmt, ly.wqkv.q, ly.wqkv.s, ly.wqkv.ts, ly.wqkv.ts, nqkv, m->H, bf.x, R,
                        ly.attn_norm, m->eps, nullptr, bf.qkv, nullptr, BW_GEMV_RMSNORM, bf.kern, st);
        if (s != BW_OK) return s;
        s = attn_launch(bf.qkv, m->rope_cos, m->rope_sin, m->rope_max_pos, kv->k[l], kv->v[l],
                        kv->page_table, kv->max_pages, kv->n_pages, pos, B, n_rows, m->nq, m->nkv, m->hd,
                        bf.attn, bf.kern, st, kv->kv_fmt, kv->kv_fmt ? kv->k_scale[l] : 1.0f,
                        kv->kv_fmt ? kv->v_scale[l] : 1.0f, /*early=*/true);
        if (s != BW_OK) return s;
        s = gemv_launch(fmt, ly.wo.q, ly.wo.s, ly.wo.ts, ly.wo.ts, m->H, m->nq * m->hd, bf.attn, R,
                        nullptr, m->eps, bf.x, bf.x, nullptr, BW_GEMV_RESIDUAL, bf.kern, st);
        if (s != BW_OK) return s;
        if (m->n_experts == 0) {
            s = gemv_launch(fmt, ly.wgu.q, ly.wgu.s, ly.wgu.ts, ly.wgu.ts_up, 2 * m->F, m->H, bf.x, R,
                            ly.ffn_norm, m->eps, nullptr, bf.act, nullptr,
                            BW_GEMV_RMSNORM | BW_GEMV_SILU_GATE, bf.kern, st);
            if (s != BW_OK) return s;
            s = gemv_launch(fmt, ly.wd.q, ly.wd.s, ly.wd.ts, ly.wd.ts, m->H, m->F, bf.act, R, nullptr,
                            m->eps, bf.x, bf.x, nullptr, BW_GEMV_RESIDUAL, bf.kern, st);
        } else {
            s = moe_ffn_launch(m, &ly, bf.x, R, bf.kern, bf.moe, st);
        }
        if (s != BW_OK) return s;
    }
    const bool adv = flags & BW_STEP_ADVANCE;
    s = gemv_launch(fmt, m->lm_head.q, m->lm_head.s, m->lm_head.ts, m->lm_head.ts, m->V, m->H, bf.x, R,
                    m->final_norm, m->eps, nullptr, logits, tokens_out, BW_GEMV_RMSNORM | BW_GEMV_ARGMAX,
                    bf.kern, st, adv ? tokens_in : nullptr, adv ? pos : nullptr);
    return s;
}

}  // extern "C"
