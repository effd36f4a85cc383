// moe.cu -- mixture-of-experts feed-forward block for a batch of token rows
// (sm_100a): router GEMV, top-k softmax, per-expert bucketing, grouped expert
// SwiGLU GEMVs over the union of the selected experts, shared expert and the
// weighted combine.
//
// The deep-dive page (10100.com), section 7, credits the MoE speed to
// ordering the router's choices and running experts in parallel without warp
// divergence.  Here: every (expert, token) assignment is bucketed by expert
// in index order and rows in row order (one small kernel, deterministic);
// then one grouped GEMV launch covers every selected expert at once -- grid.y
// is the expert group, grid.x the 64-row block of that expert's matrix -- so
// a warp only ever runs one expert's weights over that expert's tokens, and
// each selected expert's weights stream from HBM once per step however many
// tokens chose it.  The shared expert is the last group (all rows).
//
//   y = rmsnorm(x) * ffn_norm;  r = Wr y;  top-k by (value desc, index asc);
//   w = softmax over the selected logits;
//   x += sum_k w_k * Wd_e (silu(Wg_e y) * Wu_e y) + shared(y)
#include <math.h>

#include "gemv_core.cuh"

namespace bw {

bw_status rmsnorm_launch(float *x, const float *add, const float *gamma, int M, int H, float eps, void *y,
                         int y_fp16, cudaStream_t st);

constexpr int MOE_RMAX = 256;     // token rows per call
constexpr int MOE_KMAX = 16;      // experts per token
constexpr int MOE_EMAX = 1024;    // experts
constexpr int MOE_M = 4;          // token rows per pass of the grouped GEMV

// ------------------------------------------------------------------ router

// logits[r][e] = sum_k Wr[e][k] y[r][k]; one warp per expert, the rows of y
// staged in shared memory 128 columns at a time (rows rb..rb+31).
__global__ void __launch_bounds__(256) moe_router_kernel(const float *y, const float *wr, int R, int H, int E,
                                                         float *logits) {
    pdl_trigger();
    pdl_wait();
    __shared__ __align__(16) float ys[32][128];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 8 + warp;
    const int r0 = blockIdx.y * 32;
    const int nr = min(32, R - r0);
    float acc[32];
#pragma unroll
    for (int r = 0; r < 32; r++) acc[r] = 0.0f;
    for (int k0 = 0; k0 < H; k0 += 128) {
        __syncthreads();
        for (int i = threadIdx.x; i < 32 * 128; i += 256) {
            const int r = i >> 7, c = i & 127;
            ys[r][c] = (r < nr && k0 + c < H) ? y[static_cast<size_t>(r0 + r) * H + k0 + c] : 0.0f;
        }
        __syncthreads();
        if (e < E) {
            const int k = k0 + lane * 4;
            float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
            if (k < H) w = *reinterpret_cast<const float4 *>(wr + static_cast<size_t>(e) * H + k);
#pragma unroll
            for (int r = 0; r < 32; r++) {
                if (r < nr) {
                    const float4 v = *reinterpret_cast<const float4 *>(&ys[r][lane * 4]);
                    float a = acc[r];
                    a = fmaf(w.x, v.x, a);
                    a = fmaf(w.y, v.y, a);
                    a = fmaf(w.z, v.z, a);
                    a = fmaf(w.w, v.w, a);
                    acc[r] = a;
                }
            }
        }
    }
    if (e >= E) return;
#pragma unroll
    for (int r = 0; r < 32; r++) {
        if (r < nr) {
            const float v = warp_sum(acc[r]);
            if (lane == 0) logits[static_cast<size_t>(r0 + r) * E + e] = v;
        }
    }
}

// --------------------------------------------------- top-k + bucketing

struct Routing {
    int *grp_n;        // [1]   groups = selected experts + the shared expert
    int *grp_expert;   // [E+1] expert of each group in index order; -1 = shared
    int *grp_off;      // [E+2] assignment offsets
    int *asg_row;      // [R*K + R] token row of each assignment
    int *inv;          // [R*K] assignment index of (row, slot)
};

// One CTA.  Warp w selects the top-k of rows w, w+32, ...: repeated warp-wide
// argmax (value descending, lower expert index on ties) over the experts not
// yet chosen; softmax over the chosen logits in selection order.  Then the
// assignments are bucketed by expert (index order) and, within an expert, by
// row (row order) -- deterministic.
__global__ void __launch_bounds__(1024) moe_topk_kernel(const float *logits, int R, int E, int K, int32_t *sel_out,
                                                        float *w_out, Routing rt) {
    pdl_trigger();
    pdl_wait();
    __shared__ int s_sel[MOE_RMAX][MOE_KMAX];
    __shared__ int s_cnt[MOE_EMAX];
    __shared__ int s_off[MOE_EMAX];
    __shared__ int s_sh_off;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per_lane = (E + 31) / 32;
    for (int i = threadIdx.x; i < R * K; i += blockDim.x) rt.inv[i] = -1;
    for (int r = warp; r < R; r += 32) {
        const float *lr = logits + static_cast<size_t>(r) * E;
        uint32_t used = 0;
        float sv[MOE_KMAX];
        for (int t = 0; t < K; t++) {
            float bv = -INFINITY;
            int be = 0x7fffffff;
            for (int j = 0; j < per_lane; j++) {
                const int e = lane + 32 * j;
                if (e < E && !(used & (1u << j))) {
                    const float v = lr[e];
                    if (better(v, e, bv, be)) {
                        bv = v;
                        be = e;
                    }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oe = __shfl_xor_sync(0xffffffffu, be, o);
                if (better(ov, oe, bv, be)) {
                    bv = ov;
                    be = oe;
                }
            }
            if (be != 0x7fffffff && (be & 31) == lane) used |= 1u << (be >> 5);
            if (lane == 0) s_sel[r][t] = be;
            sv[t] = bv;
        }
        if (lane == 0) {
            const float m = sv[0];
            float w[MOE_KMAX];
            float sum = 0.0f;
            for (int t = 0; t < K; t++) {
                w[t] = expf(sv[t] - m);
                sum += w[t];
            }
            for (int t = 0; t < K; t++) {
                w_out[static_cast<size_t>(r) * K + t] = w[t] / sum;
                sel_out[static_cast<size_t>(r) * K + t] = s_sel[r][t];
            }
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int c = 0;
        for (int r = 0; r < R; r++)
            for (int t = 0; t < K; t++) c += (s_sel[r][t] == e);
        s_cnt[e] = c;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int off = 0, g = 0;
        for (int e = 0; e < E; e++) {
            s_off[e] = off;
            if (s_cnt[e] > 0) {
                rt.grp_expert[g] = e;
                rt.grp_off[g] = off;
                off += s_cnt[e];
                g++;
            }
        }
        rt.grp_expert[g] = -1;           // shared expert: every row
        rt.grp_off[g] = off;
        rt.grp_off[g + 1] = off + R;
        *rt.grp_n = g + 1;
        s_sh_off = off;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        if (s_cnt[e] == 0) continue;
        int j = s_off[e];
        for (int r = 0; r < R; r++)
            for (int t = 0; t < K; t++)
                if (s_sel[r][t] == e) {
                    rt.asg_row[j] = r;
                    rt.inv[r * K + t] = j;
                    j++;
                }
    }
    for (int r = threadIdx.x; r < R; r += blockDim.x) rt.asg_row[s_sh_off + r] = r;
}

// ------------------------------------------------------- grouped GEMV

struct GroupedParams {
    const uint8_t *eq, *es;    // expert stack (tiled layout, experts back to back)
    const uint8_t *shq, *shs;  // shared expert (tiled layout)
    size_t q_stride, s_stride; // bytes per expert matrix
    int N, K, NC, RG, KT;      // one expert matrix: rows (GPU layout), columns
    const int *grp_n, *grp_expert, *grp_off, *asg_row;
    const float *x;            // source activations
    int gather;                // 1: row asg_row[j] of x, 0: row j of x
    float *y;                  // [assignments][N or N/2]
    int silu;                  // gate/up interleaved rows -> silu(g) * u
    const float *ts_tab;       // NVFP4 tensor scales: [E][2] (gate/up) or [E]
    float ts_sh, ts_sh_up;     // shared expert
    int nst;
    uint32_t *err;
};

// One CTA per (128-row block, group); the group's tokens are processed MOE_M
// rows at a time, the expert's tiles streamed for each pass (after the first
// pass they come from L2).
template <int FMT>
__global__ void __launch_bounds__(GV_THREADS, 1) moe_grouped_gemv_kernel(const GroupedParams p) {
    constexpr int M = MOE_M;
    extern __shared__ __align__(128) unsigned char gg_smem[];
    const int nst = p.nst;
    const int CS = p.KT * GV_TC;
    unsigned char *stages = gg_smem;
    float *xs = reinterpret_cast<float *>(gg_smem + static_cast<size_t>(nst) * GV_STAGE_BYTES);  // [M][CS][32]
    float *ct = xs + static_cast<size_t>(M) * CS * 32;                                            // [M][CS]
    uint64_t *full = reinterpret_cast<uint64_t *>(ct + ((static_cast<size_t>(M) * CS + 1) & ~static_cast<size_t>(1)));
    uint64_t *empty = full + nst;
    const uint32_t stages_a = smem_u32(stages), xs_a = smem_u32(xs), ct_a = smem_u32(ct);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], GV_CW);
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_trigger();
    pdl_wait();   // the routing tables come from the previous kernel
    const int g = blockIdx.y;
    if (g >= *p.grp_n) return;
    const int expert = p.grp_expert[g];
    const int off = p.grp_off[g];
    const int cnt = p.grp_off[g + 1] - off;
    const int rb = blockIdx.x;
    const int ntb = (cnt + M - 1) / M;
    const int T = p.KT;
    const int n_steps = ntb * T;
    const uint8_t *bq = expert >= 0 ? p.eq + static_cast<size_t>(expert) * p.q_stride : p.shq;
    const uint8_t *bs = expert >= 0 ? p.es + static_cast<size_t>(expert) * p.s_stride : p.shs;

    if (warp == GV_CW) {
        if (lane == 0) {
            for (int step = 0; step < n_steps; step++) {
                const int s = step % nst;
                if (step >= nst) mbar_wait(&empty[s], static_cast<uint32_t>((step / nst - 1) & 1), p.err);
                const size_t tile = static_cast<size_t>(rb) * p.KT + step % T;
                unsigned char *st = stages + static_cast<size_t>(s) * GV_STAGE_BYTES;
                mbar_arrive_tx_relaxed(&full[s], GV_STAGE_BYTES);
                bulk_g2s(st, bq + tile * GV_NIB_BYTES, GV_NIB_BYTES, &full[s]);
                bulk_g2s(st + GV_NIB_BYTES, bs + tile * GV_SC_BYTES, GV_SC_BYTES, &full[s]);
            }
        }
        return;
    }

    float ts = 1.0f, ts_up = 1.0f;
    if constexpr (FMT == BW_FMT_NVFP4) {
        if (expert >= 0) {
            ts = p.silu ? p.ts_tab[2 * expert] : p.ts_tab[expert];
            ts_up = p.silu ? p.ts_tab[2 * expert + 1] : ts;
        } else {
            ts = p.ts_sh;
            ts_up = p.ts_sh_up;
        }
    }
    const int rg = rb * (GV_TR / 8) + 2 * warp + (lane >> 4);
    const int nc = p.NC;
    int step = 0;
    for (int tb = 0; tb < ntb; tb++) {
        const int mcnt = min(M, cnt - tb * M);
        consumer_sync();   // the previous pass is done with the staged activations
        // pass 1: the tokens' activation rows in natural order, loads back to back
#pragma unroll
        for (int m = 0; m < M; m++) {
            const float *xr = nullptr;
            if (m < mcnt) {
                const int j = off + tb * M + m;
                xr = p.x + static_cast<size_t>(p.gather ? p.asg_row[j] : j) * p.K;
            }
#pragma unroll 4
            for (int e = threadIdx.x; e < nc * 32; e += GV_CW * 32)
                xs[static_cast<size_t>(m) * CS * 32 + e] = xr ? xr[e] : 0.0f;
        }
        consumer_sync();
        stage_pass2<FMT, M>(xs, ct, nullptr, nullptr, CS, nc, warp, lane);
        consumer_sync();
        float acc[8][M];
#pragma unroll
        for (int r = 0; r < 8; r++)
#pragma unroll
            for (int m = 0; m < M; m++) acc[r][m] = 0.0f;
        for (int kt = 0; kt < T; kt++, step++) {
            const int s = step % nst;
            mbar_wait(&full[s], static_cast<uint32_t>((step / nst) & 1), p.err);
            const int cl = kt * GV_TC + (lane & 15);
            if (cl < nc)
                stage_chunk<FMT, M>(stages_a + static_cast<uint32_t>(s) * GV_STAGE_BYTES, warp, lane, xs_a, ct_a, cl,
                                    CS, acc);
            __syncwarp();
            if (lane == 0) mbar_arrive_relaxed(&empty[s]);
        }
        float tot[M];
        reduce_rows16<M>(acc, lane, tot);
        const int r = (lane >> 1) & 7;
        float val[M];
#pragma unroll
        for (int m = 0; m < M; m++) {
            float v = tot[m];
            if constexpr (FMT == BW_FMT_Q4_0) {
                v *= 281474976710656.0f;   // 2^48
            } else {
                v *= (p.silu && r >= 4) ? ts_up : ts;
            }
            val[m] = v;
        }
        const bool act = (lane & 1) == 0 && rg < p.RG;
        if (p.silu) {
#pragma unroll
            for (int m = 0; m < M; m++) {
                const float up = __shfl_down_sync(0xffffffffu, val[m], 8);
                if (act && r < 4 && m < mcnt) {
                    const float gt = val[m];
                    const size_t j = static_cast<size_t>(off + tb * M + m);
                    p.y[j * (p.N / 2) + rg * 4 + r] = (gt / (1.0f + expf(-gt))) * up;
                }
            }
        } else if (act) {
#pragma unroll
            for (int m = 0; m < M; m++)
                if (m < mcnt) p.y[static_cast<size_t>(off + tb * M + m) * p.N + rg * 8 + r] = val[m];
        }
    }
}

// ----------------------------------------------------------------- combine

// x[r] += (sum_k w[r][k] * out[assignment of (r, k)]) + out[shared assignment of r],
// summed in selection order.
__global__ void moe_combine_kernel(float *x, const float *dout, const float *w, const int *inv, const int *grp_n,
                                   const int *grp_off, int R, int H, int K) {
    pdl_trigger();
    pdl_wait();
    const int sh = grp_off[*grp_n - 1];
    const size_t n = static_cast<size_t>(R) * H;
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const int r = static_cast<int>(i / H), h = static_cast<int>(i % H);
        float acc = 0.0f;
        for (int t = 0; t < K; t++) {
            const int j = inv[r * K + t];   // -1 only if the router row had no finite logit
            if (j >= 0) acc = fmaf(w[r * K + t], dout[static_cast<size_t>(j) * H + h], acc);
        }
        acc += dout[static_cast<size_t>(sh + r) * H + h];
        x[i] += acc;
    }
}

// -------------------------------------------------------------------- host

struct MoeScratch {
    float *y, *logits, *wts, *act, *dout;
    int32_t *sel;
    Routing rt;
};

static size_t moe_carve(const bw_model *m, int R, char *base, MoeScratch *ms) {
    const int E = m->n_experts, K = m->topk, H = m->H, Fe = m->F_exp;
    const size_t nasg = static_cast<size_t>(R) * K + R;
    Carver cv(base);
    MoeScratch s;
    s.y = cv.take<float>(static_cast<size_t>(R) * H);
    s.logits = cv.take<float>(static_cast<size_t>(R) * E);
    s.wts = cv.take<float>(static_cast<size_t>(R) * K);
    s.sel = cv.take<int32_t>(static_cast<size_t>(R) * K);
    s.rt.grp_n = cv.take<int>(1);
    s.rt.grp_expert = cv.take<int>(E + 1);
    s.rt.grp_off = cv.take<int>(E + 2);
    s.rt.asg_row = cv.take<int>(nasg);
    s.rt.inv = cv.take<int>(static_cast<size_t>(R) * K);
    s.act = cv.take<float>(nasg * Fe);
    s.dout = cv.take<float>(nasg * H);
    if (ms) *ms = s;
    return cv.off;
}

size_t moe_scratch_bytes(const bw_model *m, int R) { return moe_carve(m, R, nullptr, nullptr); }

template <int FMT>
static bw_status grouped_go(const GroupedParams &p, int RB, int groups, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(p.nst) * GV_STAGE_BYTES +
                        static_cast<size_t>(MOE_M) * p.KT * GV_TC * 33 * 4 + 16 + 2 * static_cast<size_t>(p.nst) * 8;
    static size_t attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return BW_ERR_CUDA;
    if (attr_set[dev] < smem) {
        if (cudaFuncSetAttribute(moe_grouped_gemv_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess) {
            (void)cudaGetLastError();
            return BW_ERR_CUDA;
        }
        attr_set[dev] = smem;
    }
    return launch_pdl(moe_grouped_gemv_kernel<FMT>, dim3(RB, groups), dim3(GV_THREADS), smem, st, p);
}

bw_status moe_ffn_launch(const bw_model *m, const bw_layer *ly, float *x, int R, const Scratch &sc, char *moe_base,
                         cudaStream_t st, int32_t *topk_idx, float *topk_w);

bw_status moe_ffn_launch(const bw_model *m, const bw_layer *ly, float *x, int R, const Scratch &sc, char *moe_base,
                         cudaStream_t st) {
    return moe_ffn_launch(m, ly, x, R, sc, moe_base, st, nullptr, nullptr);
}

bw_status moe_ffn_launch(const bw_model *m, const bw_layer *ly, float *x, int R, const Scratch &sc, char *moe_base,
                         cudaStream_t st, int32_t *topk_idx, float *topk_w) {
    const int E = m->n_experts, K = m->topk, H = m->H, Fe = m->F_exp;
    const int fmt = ly->sgu.fmt;
    if (E <= 0 || E > MOE_EMAX || K <= 0 || K > MOE_KMAX || K > E || R <= 0 || R > MOE_RMAX)
        return BW_ERR_UNSUPPORTED_SHAPE;
    if (H % 32 || Fe % 32 || H % 4) return BW_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<size_t>(MOE_M) * gv_col_tiles(H) * GV_TC * 33 * 4 > 66 * 1024) return BW_ERR_UNSUPPORTED_SHAPE;
    if (!ly->router || !ly->egu_q || !ly->egu_s || !ly->ed_q || !ly->ed_s || !ly->ffn_norm || !ly->sgu.q ||
        !ly->sgu.s || !ly->sd.q || !ly->sd.s || !x || !moe_base)
        return BW_ERR_INVALID_ARG;
    if (fmt == BW_FMT_NVFP4 && (!ly->egu_ts || !ly->ed_ts)) return BW_ERR_INVALID_ARG;
    if (ly->sgu.N != 2 * Fe || ly->sgu.K != H || ly->sd.N != H || ly->sd.K != Fe || ly->sd.fmt != fmt)
        return BW_ERR_INVALID_ARG;
    MoeScratch ms;
    moe_carve(m, R, moe_base, &ms);
    bw_status s = rmsnorm_launch(x, nullptr, ly->ffn_norm, R, H, m->eps, ms.y, 0, st);
    if (s != BW_OK) return s;
    s = launch_pdl(moe_router_kernel, dim3((E + 7) / 8, (R + 31) / 32), dim3(256), 0, st,
                   static_cast<const float *>(ms.y), ly->router, R, H, E, ms.logits);
    if (s != BW_OK) return s;
    int32_t *sel = topk_idx ? topk_idx : ms.sel;
    float *wts = topk_w ? topk_w : ms.wts;
    s = launch_pdl(moe_topk_kernel, dim3(1), dim3(1024), 0, st, static_cast<const float *>(ms.logits), R, E, K, sel,
                   wts, ms.rt);
    if (s != BW_OK) return s;
    GroupedParams gp;
    gp.grp_n = ms.rt.grp_n;
    gp.grp_expert = ms.rt.grp_expert;
    gp.grp_off = ms.rt.grp_off;
    gp.asg_row = ms.rt.asg_row;
    gp.nst = 3;
    gp.err = sc.err;
    size_t qb = 0, sb = 0;
    // gate/up: rows of y gathered per assignment -> act[assignment][Fe]
    bw_repack_bytes(2 * Fe, H, &qb, &sb);
    gp.eq = static_cast<const uint8_t *>(ly->egu_q);
    gp.es = static_cast<const uint8_t *>(ly->egu_s);
    gp.shq = static_cast<const uint8_t *>(ly->sgu.q);
    gp.shs = static_cast<const uint8_t *>(ly->sgu.s);
    gp.q_stride = qb;
    gp.s_stride = sb;
    gp.N = 2 * Fe;
    gp.K = H;
    gp.NC = H / 32;
    gp.RG = gp.N / 8;
    gp.KT = gv_col_tiles(H);
    gp.x = ms.y;
    gp.gather = 1;
    gp.y = ms.act;
    gp.silu = 1;
    gp.ts_tab = ly->egu_ts;
    gp.ts_sh = ly->sgu.ts;
    gp.ts_sh_up = ly->sgu.ts_up;
    s = fmt == BW_FMT_Q4_0 ? grouped_go<BW_FMT_Q4_0>(gp, gv_row_blocks(gp.N), E + 1, st)
                           : grouped_go<BW_FMT_NVFP4>(gp, gv_row_blocks(gp.N), E + 1, st);
    if (s != BW_OK) return s;
    // down: act[assignment] -> dout[assignment][H]
    bw_repack_bytes(H, Fe, &qb, &sb);
    gp.eq = static_cast<const uint8_t *>(ly->ed_q);
    gp.es = static_cast<const uint8_t *>(ly->ed_s);
    gp.shq = static_cast<const uint8_t *>(ly->sd.q);
    gp.shs = static_cast<const uint8_t *>(ly->sd.s);
    gp.q_stride = qb;
    gp.s_stride = sb;
    gp.N = H;
    gp.K = Fe;
    gp.NC = Fe / 32;
    gp.RG = H / 8;
    gp.KT = gv_col_tiles(Fe);
    gp.x = ms.act;
    gp.gather = 0;
    gp.y = ms.dout;
    gp.silu = 0;
    gp.ts_tab = ly->ed_ts;
    gp.ts_sh = ly->sd.ts;
    gp.ts_sh_up = ly->sd.ts;
    s = fmt == BW_FMT_Q4_0 ? grouped_go<BW_FMT_Q4_0>(gp, gv_row_blocks(H), E + 1, st)
                           : grouped_go<BW_FMT_NVFP4>(gp, gv_row_blocks(H), E + 1, st);
    if (s != BW_OK) return s;
    const size_t nblk = (static_cast<size_t>(R) * H + 255) / 256;
    const int blocks = static_cast<int>(nblk < 4096 ? nblk : 4096);
    return launch_pdl(moe_combine_kernel, dim3(blocks), dim3(256), 0, st, x, static_cast<const float *>(ms.dout),
                      static_cast<const float *>(wts), static_cast<const int *>(ms.rt.inv),
                      static_cast<const int *>(ms.rt.grp_n), static_cast<const int *>(ms.rt.grp_off), R, H, K);
}

}  // namespace bw

extern "C" {

bw_status bw_moe_route_gemv(const bw_model *m, const bw_layer *ly, float *x, int R, int32_t *topk_idx,
                            float *topk_w, void *ws, size_t ws_bytes, void *stream) {
    if (!m || !ly || !ws) return BW_ERR_INVALID_ARG;
    if (ws_bytes < bw_moe_workspace_bytes(m, R)) return BW_ERR_INVALID_ARG;
    bw::Scratch sc = bw::scratch_of(ws, ws_bytes);
    return bw::moe_ffn_launch(m, ly, x, R, sc, sc.base, static_cast<cudaStream_t>(stream), topk_idx, topk_w);
}

size_t bw_moe_workspace_bytes(const bw_model *m, int R) {
    if (!m || R <= 0 || m->n_experts <= 0) return BW_WS_HDR_BYTES;
    return BW_WS_HDR_BYTES + bw::moe_scratch_bytes(m, R);
}

}  // extern "C"
