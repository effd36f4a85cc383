// mtp.cu -- the speculative draft head: K draft tokens for the next verify
// pass (sm_100a).
//
// The "bw24" deep-dive page (10100.com), section 7, describes the MTP draft
// head: light, sharing the main model's embedding, its output vocabulary pruned
// to the first ids; section 5, stage 4, runs its K drafts through one verify
// pass; section 1 puts the speculative decoder's output equal to plain greedy
// decoding.  The page gives no formula.  Draft i (i = 1..K) is
//     x = h + E[t],  g = rmsnorm(x) * gamma_d,  d_i = argmax (W_d g),
// then h <- g and t <- d_i; the first draft starts from the main model's
// residual stream after its last layer at the row whose greedy token is t.
// Each draft is two launches: a one-CTA prologue (row select, embedding
// dequant, add, RMSNorm) and the library's dequant GEMV with the argmax
// epilogue writing d_i straight into the verify pass's token row.
#include "gemv_core.cuh"

namespace bw {

constexpr int MTP_THREADS = 512;

// g = rmsnorm(h + E[tokens[i]]) * gamma, h = hidden row (*row, or 0) for the
// first draft (h_prev == nullptr), else h_prev.
__global__ void __launch_bounds__(MTP_THREADS) mtp_prologue_kernel(int fmt, const uint8_t *eq, const uint8_t *es,
                                                                   float ts, int V, int H, const int32_t *tokens,
                                                                   int i, const float *hidden, const int32_t *row,
                                                                   int n_rows, const float *h_prev,
                                                                   const float *gamma, float eps, float *g,
                                                                   uint32_t *err) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ float mp_x[];
    __shared__ float red[MTP_THREADS / 32];
    __shared__ float s_r;
    const int tok = tokens[i];
    const bool ok = tok >= 0 && tok < V;
    int r = row ? *row : 0;
    if (r < 0 || r >= n_rows) {
        if (threadIdx.x == 0) set_error(err, BW_DEVERR_BAD_TOKEN);
        r = 0;
    }
    if (!ok && threadIdx.x == 0) set_error(err, BW_DEVERR_BAD_TOKEN);
    const float *h = h_prev ? h_prev : hidden + static_cast<size_t>(r) * H;
    const int KT = gv_col_tiles(H);
    float ss = 0.0f;
    for (int k = threadIdx.x; k < H; k += MTP_THREADS) {
        float w = 0.0f;
        if (ok) {
            // the embedding row in the tiled layout (see gemv_core.cuh)
            const int c = k >> 5, e = k & 31;
            const size_t tile = static_cast<size_t>(tok / GV_TR) * KT + c / GV_TC;
            const int rr = tok % GV_TR;
            const size_t qo = tile * GV_NIB_BYTES + static_cast<size_t>(rr) * (GV_TC * 16) + (((c % GV_TC) ^ (rr % 8)) * 16);
            const size_t so = tile * GV_SC_BYTES + static_cast<size_t>(rr / 8) * (GV_TC * 16) + (c % GV_TC) * 16 + (rr % 8) * 2;
            if (fmt == BW_FMT_Q4_0) {
                const uint8_t byte = eq[qo + (e & 15)];
                const int q = (e >> 4) ? (byte >> 4) : (byte & 15);
                w = __fmul_rn(half_bits_to_f(*reinterpret_cast<const uint16_t *>(es + so)), static_cast<float>(q - 8));
            } else {
                const uint8_t byte = eq[qo + (e >> 1)];
                const float2 v2 = e2m1x2_to_f2(byte);
                w = __fmul_rn(__fmul_rn((e & 1) ? v2.y : v2.x, e4m3_to_f(es[so + (e >> 4)])), ts);
            }
        }
        const float x = __fadd_rn(h[k], w);
        mp_x[k] = x;
        ss = fmaf(x, x, ss);
    }
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.0f;
        for (int w2 = 0; w2 < MTP_THREADS / 32; w2++) t += red[w2];
        s_r = 1.0f / sqrtf(t / static_cast<float>(H) + eps);
    }
    __syncthreads();
    for (int k = threadIdx.x; k < H; k += MTP_THREADS) g[k] = __fmul_rn(__fmul_rn(mp_x[k], s_r), gamma[k]);
}

struct MtpBuffers {
    float *g[2];
    Scratch kern;
};

static size_t mtp_bytes(const bw_model *m, const bw_draft_head *dh, MtpBuffers *b, void *ws) {
    Carver cv(ws ? static_cast<char *>(ws) + BW_WS_HDR_BYTES : nullptr);
    float *g0 = cv.take<float>(m->H);
    float *g1 = cv.take<float>(m->H);
    const size_t kb = gemv_scratch_bytes(dh->w.N, m->H, 1);
    char *kbase = cv.take<char>(kb);
    if (b) {
        b->g[0] = g0;
        b->g[1] = g1;
        b->kern.err = ws ? ws_error_word(ws) : nullptr;
        b->kern.cnt = ws ? ws_counters(ws) : nullptr;
        b->kern.base = kbase;
        b->kern.bytes = kb;
    }
    return BW_WS_HDR_BYTES + cv.off;
}

}  // namespace bw

extern "C" {

size_t bw_mtp_workspace_bytes(const bw_model *m, const bw_draft_head *dh) {
    if (!m || !dh || m->H <= 0 || dh->w.N <= 0) return BW_WS_HDR_BYTES;
    return bw::mtp_bytes(m, dh, nullptr, nullptr);
}

bw_status bw_mtp_draft(const bw_model *m, const bw_draft_head *dh, const float *hidden, int n_rows,
                       const int32_t *row, int32_t *tokens, int K, void *ws, size_t ws_bytes, void *stream) {
    using namespace bw;
    if (!m || !dh || !hidden || !tokens || !ws_ok(ws) || n_rows <= 0) return BW_ERR_INVALID_ARG;
    if (K < 1 || K > BW_MAX_VERIFY_ROWS - 1) return BW_ERR_INVALID_ARG;
    const int fmt = m->embed.fmt;
    if (!m->embed.q || !m->embed.s || m->embed.N != m->V || m->embed.K != m->H) return BW_ERR_INVALID_ARG;
    if (!dh->norm || !dh->w.q || !dh->w.s || dh->w.K != m->H || dh->w.fmt != fmt || dh->w.N <= 0 || dh->w.N > m->V)
        return BW_ERR_INVALID_ARG;
    if (m->H % 32 || m->H > 12288) return BW_ERR_UNSUPPORTED_SHAPE;   // the row fits 48 KB of shared memory
    if (!aligned16(m->embed.q) || !aligned16(m->embed.s)) return BW_ERR_INVALID_ARG;
    MtpBuffers b;
    if (ws_bytes < mtp_bytes(m, dh, &b, ws)) return BW_ERR_INVALID_ARG;
    // every GEMV launch's checks before the first launch
    bw_status s = gemv_check(fmt, dh->w.q, dh->w.s, dh->w.N, m->H, b.g[0], 1, nullptr, nullptr, nullptr, tokens,
                             BW_GEMV_ARGMAX, b.kern);
    if (s != BW_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t smem = static_cast<size_t>(m->H) * 4;
    for (int i = 0; i < K; i++) {
        float *g = b.g[i & 1];
        s = launch_pdl(mtp_prologue_kernel, dim3(1), dim3(MTP_THREADS), smem, st, fmt,
                       static_cast<const uint8_t *>(m->embed.q), static_cast<const uint8_t *>(m->embed.s), m->embed.ts,
                       m->V, m->H, static_cast<const int32_t *>(tokens), i, hidden, row, n_rows,
                       static_cast<const float *>(i == 0 ? nullptr : b.g[(i - 1) & 1]), dh->norm, m->eps, g,
                       b.kern.err);
        if (s != BW_OK) return s;
        s = gemv_launch(fmt, dh->w.q, dh->w.s, dh->w.ts, dh->w.ts, dh->w.N, m->H, g, 1, nullptr, m->eps, nullptr,
                        nullptr, tokens + i + 1, BW_GEMV_ARGMAX, b.kern, st, nullptr, nullptr);
        if (s != BW_OK) return s;
    }
    return BW_OK;
}

}  // extern "C"
