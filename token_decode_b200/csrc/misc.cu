// misc.cu -- layout repack, embedding gather, RoPE table, argmax and RMSNorm
// kernels of libbw (sm_100a).
#include <math.h>

#include "gemv_core.cuh"

namespace bw {

// ------------------------------------------------------------------ repack

// out row R of an interleaved gate/up matrix: rows 8g..8g+3 are gate rows
// 4g..4g+3, rows 8g+4..8g+7 the matching up rows.
__device__ __forceinline__ void src_row(int R, bool inter, int &row, int &which) {
    if (!inter) {
        row = R;
        which = 0;
        return;
    }
    const int g = R >> 3, i = R & 7;
    row = 4 * g + (i & 3);
    which = i >> 2;
}

// Tiled layout offsets (see gemv_core.cuh): codes of (row R, chunk c) and the
// byte offset of row R's scale slot for chunk c.
__device__ __forceinline__ size_t tile_code_off(int R, int c, int KT) {
    const size_t tile = static_cast<size_t>(R / GV_TR) * KT + c / GV_TC;
    return tile * GV_NIB_BYTES + static_cast<size_t>(R % GV_TR) * (GV_TC * 16) + ((c % GV_TC) ^ (R % 8)) * 16;
}
__device__ __forceinline__ size_t tile_scale_off(int R, int c, int KT) {
    const size_t tile = static_cast<size_t>(R / GV_TR) * KT + c / GV_TC;
    return tile * GV_SC_BYTES + static_cast<size_t>((R % GV_TR) / 8) * (GV_TC * 16) + (c % GV_TC) * 16 + (R % 8) * 2;
}

__global__ void repack_q4_0_kernel(const uint8_t *blocks, const uint8_t *blocks_up, int rows, int NC, int KT,
                                   uint8_t *q_out, uint8_t *s_out) {
    const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= static_cast<size_t>(rows) * NC) return;
    const int R = static_cast<int>(i / NC), c = static_cast<int>(i % NC);
    int row, which;
    src_row(R, blocks_up != nullptr, row, which);
    const uint8_t *src = (which ? blocks_up : blocks) + (static_cast<size_t>(row) * NC + c) * 18;
    const uint16_t *s16 = reinterpret_cast<const uint16_t *>(src);   // 18-byte blocks: 2-byte aligned
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; k++) w[k] = static_cast<uint32_t>(s16[1 + 2 * k]) | (static_cast<uint32_t>(s16[2 + 2 * k]) << 16);
    *reinterpret_cast<uint4 *>(q_out + tile_code_off(R, c, KT)) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint16_t *>(s_out + tile_scale_off(R, c, KT)) = s16[0];
}

__global__ void repack_nvfp4_kernel(const uint8_t *q, const uint8_t *s, const uint8_t *q_up,
                                    const uint8_t *s_up, int rows, int NC, int KT, uint8_t *q_out, uint8_t *s_out) {
    const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= static_cast<size_t>(rows) * NC) return;
    const int R = static_cast<int>(i / NC), c = static_cast<int>(i % NC);
    int row, which;
    src_row(R, q_up != nullptr, row, which);
    const uint8_t *qs = which ? q_up : q;
    const uint8_t *ss = which ? s_up : s;
    *reinterpret_cast<uint4 *>(q_out + tile_code_off(R, c, KT)) =
        *reinterpret_cast<const uint4 *>(qs + static_cast<size_t>(row) * NC * 16 + static_cast<size_t>(c) * 16);
    uint8_t *d = s_out + tile_scale_off(R, c, KT);
    d[0] = ss[static_cast<size_t>(row) * NC * 2 + 2 * c];
    d[1] = ss[static_cast<size_t>(row) * NC * 2 + 2 * c + 1];
}

// --------------------------------------------------------------- embedding

// Dequantize rows tokens[m] of a GPU-layout matrix: Q4_0 w = d * (q - 8);
// NVFP4 w = (e2m1 * e4m3) * ts -- each one fp32 rounding, like the format's
// definition.
__global__ void embed_kernel(int fmt, const uint8_t *eq, const uint8_t *es, float ts, int V, int H,
                             const int32_t *tokens, float *x, uint32_t *err) {
    pdl_trigger();
    pdl_wait();
    const int m = blockIdx.x;
    const int tok = tokens[m];
    const bool ok = tok >= 0 && tok < V;
    if (!ok && threadIdx.x == 0) set_error(err, BW_DEVERR_BAD_TOKEN);
    const int KT = gv_col_tiles(H);
    for (int k = threadIdx.x; k < H; k += blockDim.x) {
        float w = 0.0f;
        if (ok) {
            const int c = k >> 5, e = k & 31;
            const size_t qo = tile_code_off(tok, c, KT), so = tile_scale_off(tok, c, KT);
            if (fmt == BW_FMT_Q4_0) {
                const uint8_t byte = eq[qo + (e & 15)];
                const int q = (e >> 4) ? (byte >> 4) : (byte & 15);
                const uint16_t dh = *reinterpret_cast<const uint16_t *>(es + so);
                w = __fmul_rn(half_bits_to_f(dh), static_cast<float>(q - 8));
            } else {
                const uint8_t byte = eq[qo + (e >> 1)];
                const float2 v2 = e2m1x2_to_f2(byte);
                const float ev = (e & 1) ? v2.y : v2.x;
                const float sv = e4m3_to_f(es[so + (e >> 4)]);
                w = __fmul_rn(__fmul_rn(ev, sv), ts);
            }
        }
        x[static_cast<size_t>(m) * H + k] = w;
    }
}

// ---------------------------------------------------------------- RoPE table

__global__ void rope_table_kernel(double theta, int hd, int max_pos, float *cs, float *sn) {
    const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int half = hd / 2;
    if (i >= static_cast<size_t>(max_pos) * half) return;
    const int p = static_cast<int>(i / half), d = static_cast<int>(i % half);
    const double inv_freq = pow(theta, -2.0 * static_cast<double>(d) / static_cast<double>(hd));
    const double ang = static_cast<double>(p) * inv_freq;
    cs[i] = static_cast<float>(cos(ang));
    sn[i] = static_cast<float>(sin(ang));
}

// ------------------------------------------------------------------ argmax

struct Top2 {
    float v;
    int i;
    float v2;
};

__device__ __forceinline__ Top2 merge(Top2 a, Top2 b) {
    if (better(b.v, b.i, a.v, a.i)) return {b.v, b.i, fmaxf(a.v, b.v2)};
    return {a.v, a.i, fmaxf(a.v2, b.v)};
}

__global__ void argmax_kernel(const float *logits, int V, int32_t *idx, float *margin) {
    pdl_trigger();
    pdl_wait();
    __shared__ Top2 red[32];
    const int m = blockIdx.x;
    const float *row = logits + static_cast<size_t>(m) * V;
    Top2 t = {-INFINITY, 0x7fffffff, -INFINITY};
    for (int i = threadIdx.x; i < V; i += blockDim.x) {
        const float v = row[i];
        if (better(v, i, t.v, t.i)) {
            t.v2 = fmaxf(t.v2, t.v);
            t.v = v;
            t.i = i;
        } else {
            t.v2 = fmaxf(t.v2, v);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        Top2 u;
        u.v = __shfl_xor_sync(0xffffffffu, t.v, o);
        u.i = __shfl_xor_sync(0xffffffffu, t.i, o);
        u.v2 = __shfl_xor_sync(0xffffffffu, t.v2, o);
        t = merge(t, u);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = t;
    __syncthreads();
    if (threadIdx.x == 0) {
        Top2 a = red[0];
        for (int w = 1; w < static_cast<int>(blockDim.x >> 5); w++) a = merge(a, red[w]);
        idx[m] = (a.i == 0x7fffffff) ? 0 : a.i;
        if (margin) margin[m] = a.v - a.v2;
    }
}

// ----------------------------------------------------------------- RMSNorm

__global__ void rmsnorm_kernel(float *x, const float *add, const float *gamma, int H, float eps, void *y,
                               int y_fp16) {
    pdl_trigger();
    pdl_wait();
    __shared__ float red[32];
    __shared__ float s_r;
    const int m = blockIdx.x;
    float *xr = x + static_cast<size_t>(m) * H;
    float ss = 0.0f;
    for (int i = threadIdx.x; i < H; i += blockDim.x) {
        float v = xr[i];
        if (add) {
            v = v + add[static_cast<size_t>(m) * H + i];
            xr[i] = v;
        }
        ss = fmaf(v, v, ss);
    }
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.0f;
        for (int w = 0; w < static_cast<int>(blockDim.x >> 5); w++) t += red[w];
        s_r = 1.0f / sqrtf(t / static_cast<float>(H) + eps);
    }
    __syncthreads();
    if (!y) return;
    for (int i = threadIdx.x; i < H; i += blockDim.x) {
        const float v = __fmul_rn(__fmul_rn(xr[i], s_r), gamma[i]);
        if (y_fp16)
            static_cast<__half *>(y)[static_cast<size_t>(m) * H + i] = __float2half_rn(v);
        else
            static_cast<float *>(y)[static_cast<size_t>(m) * H + i] = v;
    }
}

bw_status embed_check(int fmt, const void *e_q, const void *e_s, int V, int H, const int32_t *tokens, int M,
                      const float *x) {
    if (!e_q || !e_s || !tokens || !x || V <= 0 || H <= 0 || M <= 0) return BW_ERR_INVALID_ARG;
    if (H % 32) return BW_ERR_UNSUPPORTED_SHAPE;
    if (fmt != BW_FMT_Q4_0 && fmt != BW_FMT_NVFP4) return BW_ERR_INVALID_ARG;
    if (!aligned16(e_q) || !aligned16(e_s)) return BW_ERR_INVALID_ARG;   // the tiled layout's alignment
    return BW_OK;
}

bw_status embed_launch(int fmt, const void *e_q, const void *e_s, float ts, int V, int H,
                       const int32_t *tokens, int M, float *x, uint32_t *err, cudaStream_t st) {
    const bw_status chk = embed_check(fmt, e_q, e_s, V, H, tokens, M, x);
    if (chk != BW_OK) return chk;
    return launch_pdl(embed_kernel, dim3(M), dim3(256), 0, st, fmt, static_cast<const uint8_t *>(e_q),
                      static_cast<const uint8_t *>(e_s), ts, V, H, tokens, x, err);
}

bw_status rmsnorm_launch(float *x, const float *add, const float *gamma, int M, int H, float eps, void *y,
                         int y_fp16, cudaStream_t st) {
    if (!x || M <= 0 || H <= 0 || (y && !gamma)) return BW_ERR_INVALID_ARG;
    return launch_pdl(rmsnorm_kernel, dim3(M), dim3(256), 0, st, x, add, gamma, H, eps, y, y_fp16);
}

}  // namespace bw

extern "C" {

bw_status bw_repack_bytes(int rows, int K, size_t *q_bytes, size_t *s_bytes) {
    if (rows <= 0 || K <= 0 || K % 32 || !q_bytes || !s_bytes) return BW_ERR_INVALID_ARG;
    const size_t tiles = static_cast<size_t>(bw::gv_row_blocks(rows)) * bw::gv_col_tiles(K);
    *q_bytes = tiles * bw::GV_NIB_BYTES;
    *s_bytes = tiles * bw::GV_SC_BYTES;
    return BW_OK;
}

bw_status bw_repack_q4_0(const void *blocks, const void *blocks_up, int N, int K, void *q_out, void *s_out,
                         void *stream) {
    if (!blocks || !q_out || !s_out || N <= 0 || K <= 0) return BW_ERR_INVALID_ARG;
    const int rows = blocks_up ? 2 * N : N;
    if (K % 32 || rows % 8 || (blocks_up && N % 4)) return BW_ERR_UNSUPPORTED_SHAPE;
    if (!bw::aligned16(q_out) || !bw::aligned16(s_out) || (reinterpret_cast<uintptr_t>(blocks) & 1) ||
        (blocks_up && (reinterpret_cast<uintptr_t>(blocks_up) & 1)))
        return BW_ERR_INVALID_ARG;
    const int NC = K / 32, KT = bw::gv_col_tiles(K);
    size_t qb = 0, sb = 0;
    bw_repack_bytes(rows, K, &qb, &sb);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(q_out, 0, qb, st) != cudaSuccess || cudaMemsetAsync(s_out, 0, sb, st) != cudaSuccess) {
        (void)cudaGetLastError();
        return BW_ERR_CUDA;
    }
    const size_t n = static_cast<size_t>(rows) * NC;
    bw::repack_q4_0_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(
        static_cast<const uint8_t *>(blocks), static_cast<const uint8_t *>(blocks_up), rows, NC, KT,
        static_cast<uint8_t *>(q_out), static_cast<uint8_t *>(s_out));
    return bw::launch_status();
}

bw_status bw_repack_nvfp4(const void *q, const void *s, const void *q_up, const void *s_up, int N, int K,
                          void *q_out, void *s_out, void *stream) {
    if (!q || !s || !q_out || !s_out || N <= 0 || K <= 0 || (!q_up) != (!s_up)) return BW_ERR_INVALID_ARG;
    const int rows = q_up ? 2 * N : N;
    if (K % 32 || rows % 8 || (q_up && N % 4)) return BW_ERR_UNSUPPORTED_SHAPE;
    if (!bw::aligned16(q) || !bw::aligned16(q_out) || !bw::aligned16(s_out) || (q_up && !bw::aligned16(q_up)))
        return BW_ERR_INVALID_ARG;
    const int NC = K / 32, KT = bw::gv_col_tiles(K);
    size_t qb = 0, sb = 0;
    bw_repack_bytes(rows, K, &qb, &sb);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(q_out, 0, qb, st) != cudaSuccess || cudaMemsetAsync(s_out, 0, sb, st) != cudaSuccess) {
        (void)cudaGetLastError();
        return BW_ERR_CUDA;
    }
    const size_t n = static_cast<size_t>(rows) * NC;
    bw::repack_nvfp4_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(
        static_cast<const uint8_t *>(q), static_cast<const uint8_t *>(s), static_cast<const uint8_t *>(q_up),
        static_cast<const uint8_t *>(s_up), rows, NC, KT, static_cast<uint8_t *>(q_out), static_cast<uint8_t *>(s_out));
    return bw::launch_status();
}

bw_status bw_embed(int fmt, const void *e_q, const void *e_s, float ts, int V, int H, const int32_t *tokens,
                   int M, float *x, void *ws, void *stream) {
    if (ws && !bw::ws_ok(ws)) return BW_ERR_INVALID_ARG;
    return bw::embed_launch(fmt, e_q, e_s, ts, V, H, tokens, M, x, ws ? bw::ws_error_word(ws) : nullptr,
                            static_cast<cudaStream_t>(stream));
}

bw_status bw_rope_table(float theta, int hd, int max_pos, float *cos_out, float *sin_out, void *stream) {
    if (!cos_out || !sin_out || hd <= 0 || hd % 2 || max_pos <= 0 || !(theta > 0.0f)) return BW_ERR_INVALID_ARG;
    const size_t n = static_cast<size_t>(max_pos) * (hd / 2);
    bw::rope_table_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<double>(theta), hd, max_pos, cos_out, sin_out);
    return bw::launch_status();
}

bw_status bw_argmax(const float *logits, int M, int V, int32_t *idx_out, float *margin_out, void *stream) {
    if (!logits || !idx_out || M <= 0 || V <= 0) return BW_ERR_INVALID_ARG;
    return bw::launch_pdl(bw::argmax_kernel, dim3(M), dim3(1024), 0, static_cast<cudaStream_t>(stream), logits,
                          V, idx_out, margin_out);
}

bw_status bw_rmsnorm_fused(float *x, const float *add, const float *gamma, int M, int H, float eps, void *y,
                           int y_fp16, void *stream) {
    return bw::rmsnorm_launch(x, add, gamma, M, H, eps, y, y_fp16, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
