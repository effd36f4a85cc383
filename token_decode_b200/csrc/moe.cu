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

// Partial router logits over one 512-column slice of H:
//   part[slice][r][e] = sum_{k in slice} Wr[e][k] y[r][k]
// CTA = (8 experts, one slice, 32 rows).  The slice of y is staged once,
// transposed ([k][row], padded), and the 8 experts' weight slices beside it;
// lane = row, so each thread sums its own dot product (no reductions).  The
// top-k kernel adds the slices in slice order.
constexpr int MOE_KS = 512;

__global__ void __launch_bounds__(256) moe_router_kernel(const float *y, const float *wr, int R, int H, int E,
                                                         float *part) {
    pdl_trigger();
    extern __shared__ __align__(16) float rt_sm[];
    float *ys = rt_sm;                        // [MOE_KS][33]
    float *wsm = rt_sm + MOE_KS * 33;         // [8][MOE_KS]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e0 = blockIdx.x * 8, k0 = blockIdx.y * MOE_KS, r0 = blockIdx.z * 32;
    const int kn = min(MOE_KS, H - k0), nr = min(32, R - r0);
    // the router weights are constant: stage them before the dependency wait
    // (16-byte loads; H is a multiple of 32, so kn and every row start are too)
    constexpr int K4 = MOE_KS / 4;
    {
        constexpr int NW = 8 * K4 / 256;
        float4 v[NW];
#pragma unroll
        for (int u = 0; u < NW; u++) {
            const int i = threadIdx.x + u * 256, w = i / K4, k4 = i - w * K4;
            v[u] = (e0 + w < E && 4 * k4 < kn)
                       ? *reinterpret_cast<const float4 *>(wr + static_cast<size_t>(e0 + w) * H + k0 + 4 * k4)
                       : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
#pragma unroll
        for (int u = 0; u < NW; u++) reinterpret_cast<float4 *>(wsm)[threadIdx.x + u * 256] = v[u];
    }
    pdl_wait();
    {
        // the rows' slice: every load in flight at once, then stored transposed
        constexpr int NY = 32 * K4 / 256;
        float4 v[NY];
#pragma unroll
        for (int u = 0; u < NY; u++) {
            const int i = threadIdx.x + u * 256, r = i / K4, k4 = i - r * K4;
            v[u] = (r < nr && 4 * k4 < kn)
                       ? *reinterpret_cast<const float4 *>(y + static_cast<size_t>(r0 + r) * H + k0 + 4 * k4)
                       : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
#pragma unroll
        for (int u = 0; u < NY; u++) {
            const int i = threadIdx.x + u * 256, r = i / K4, k = 4 * (i - r * K4);
            ys[k * 33 + r] = v[u].x;
            ys[(k + 1) * 33 + r] = v[u].y;
            ys[(k + 2) * 33 + r] = v[u].z;
            ys[(k + 3) * 33 + r] = v[u].w;
        }
    }
    __syncthreads();
    const int e = e0 + warp;
    const float *wv = wsm + warp * MOE_KS;
    float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
    for (int k = 0; k < kn; k += 4) {
        a0 = fmaf(wv[k], ys[k * 33 + lane], a0);
        a1 = fmaf(wv[k + 1], ys[(k + 1) * 33 + lane], a1);
        a2 = fmaf(wv[k + 2], ys[(k + 2) * 33 + lane], a2);
        a3 = fmaf(wv[k + 3], ys[(k + 3) * 33 + lane], a3);
    }
    if (e < E && lane < nr) part[(static_cast<size_t>(blockIdx.y) * R + r0 + lane) * E + e] = (a0 + a1) + (a2 + a3);
}

// --------------------------------------------------- top-k + bucketing

struct Routing {
    int *n_items;      // [1]   work items of the grouped GEMVs (one pass over a row-block chunk)
    int *grp_item;     // [E+2] first item of each group
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
// row (row order) -- deterministic: per-expert counts (shared-memory atomics,
// order-free), one block-wide exclusive scan over the experts for the bucket
// offsets, group indices and work items, then for each selected expert a warp
// walks the rows 32 at a time and places them with a ballot prefix.
constexpr int MOE_NRC = 4;   // row-block chunks per expert matrix (work items per pass)
constexpr int MOE_SLB = 4;   // router slices loaded per batch (up to 256 experts)

template <int LV>   // logits per lane: ceil(E / 32) <= LV
__global__ void __launch_bounds__(1024) moe_topk_kernel(const float *part, int n_slices, int R, int E, int K,
                                                        int32_t *sel_out, float *w_out, Routing rt) {
    pdl_trigger();
    pdl_wait();
    __shared__ int s_sel[MOE_RMAX][MOE_KMAX];
    __shared__ int s_cnt[MOE_EMAX];
    __shared__ int s_off[MOE_EMAX];
    __shared__ int s_wsum[3][32];
    __shared__ int s_tot[3];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int per_lane = (E + 31) / 32;
    for (int e = tid; e < MOE_EMAX; e += blockDim.x) s_cnt[e] = 0;
    for (int i = tid; i < R * K; i += blockDim.x) rt.inv[i] = -1;
    __syncthreads();
    for (int r = warp; r < R; r += 32) {
        // this row's logits in registers: lane holds experts lane + 32 j, the
        // router slices added in slice order, a batch of slices' loads in flight
        constexpr int SB = LV <= 8 ? MOE_SLB : 1;
        float lv[LV];
#pragma unroll
        for (int j = 0; j < LV; j++) lv[j] = 0.0f;
        for (int sl0 = 0; sl0 < n_slices; sl0 += SB) {
            float t[SB][LV];
#pragma unroll
            for (int b = 0; b < SB; b++)
#pragma unroll
                for (int j = 0; j < LV; j++) {
                    const int e = lane + 32 * j;
                    t[b][j] = (sl0 + b < n_slices && j < per_lane && e < E)
                                  ? part[(static_cast<size_t>(sl0 + b) * R + r) * E + e]
                                  : 0.0f;
                }
#pragma unroll
            for (int b = 0; b < SB; b++)
#pragma unroll
                for (int j = 0; j < LV; j++) {
                    if (sl0 + b == 0)
                        lv[j] = t[b][j];
                    else if (sl0 + b < n_slices)
                        lv[j] += t[b][j];
                }
        }
#pragma unroll
        for (int j = 0; j < LV; j++)
            if (!(j < per_lane && lane + 32 * j < E)) lv[j] = -INFINITY;
        uint32_t used = 0;
        float sv[MOE_KMAX];
        for (int t = 0; t < K; t++) {
            float bv = -INFINITY;
            int be = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < LV; j++) {
                const int e = lane + 32 * j;
                if (j < per_lane && e < E && !(used & (1u << j))) {
                    const float v = lv[j];
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
            if (lane == 0) {
                s_sel[r][t] = be;
                if (be != 0x7fffffff) atomicAdd(&s_cnt[be], 1);
            }
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
    // exclusive scan over the experts (thread = expert) of: assignments,
    // "selected" (the group index) and work items
    {
        const int e = tid;
        const int c = e < E ? s_cnt[e] : 0;
        int v[3] = {c, c > 0 ? 1 : 0, c > 0 ? MOE_NRC * ((c + MOE_M - 1) / MOE_M) : 0};
        int inc[3] = {v[0], v[1], v[2]};
#pragma unroll
        for (int o = 1; o < 32; o <<= 1)
#pragma unroll
            for (int q = 0; q < 3; q++) {
                const int u = __shfl_up_sync(0xffffffffu, inc[q], o);
                if (lane >= o) inc[q] += u;
            }
        if (lane == 31)
#pragma unroll
            for (int q = 0; q < 3; q++) s_wsum[q][warp] = inc[q];
        __syncthreads();
        if (warp == 0) {
            const int nw = blockDim.x >> 5;
#pragma unroll
            for (int q = 0; q < 3; q++) {
                const int x = lane < nw ? s_wsum[q][lane] : 0;
                int y = x;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int u = __shfl_up_sync(0xffffffffu, y, o);
                    if (lane >= o) y += u;
                }
                if (lane < nw) s_wsum[q][lane] = y - x;   // exclusive warp prefix
                if (lane == 31) s_tot[q] = y;
            }
        }
        __syncthreads();
        int ex[3];
#pragma unroll
        for (int q = 0; q < 3; q++) ex[q] = inc[q] - v[q] + s_wsum[q][warp];
        if (e < MOE_EMAX) s_off[e] = ex[0];
        if (c > 0) {
            rt.grp_expert[ex[1]] = e;
            rt.grp_off[ex[1]] = ex[0];
            rt.grp_item[ex[1]] = ex[2];
        }
        if (tid == 0) {
            const int g = s_tot[1], sh = s_tot[0], it = s_tot[2];
            rt.grp_expert[g] = -1;   // shared expert: every row
            rt.grp_off[g] = sh;
            rt.grp_off[g + 1] = sh + R;
            *rt.grp_n = g + 1;
            rt.grp_item[g] = it;
            const int it2 = it + MOE_NRC * ((R + MOE_M - 1) / MOE_M);
            rt.grp_item[g + 1] = it2;
            *rt.n_items = it2;
        }
    }
    __syncthreads();   // s_off
    // each selected expert's assignments, rows in order: a warp walks the rows
    // 32 at a time (lane = row) and places the ones that chose the expert
    for (int e = warp; e < E; e += blockDim.x >> 5) {
        if (s_cnt[e] == 0) continue;
        int j0 = s_off[e];
        for (int r0 = 0; r0 < R; r0 += 32) {
            const int r = r0 + lane;
            int slot = -1;
            if (r < R)
                for (int t = 0; t < K; t++)
                    if (s_sel[r][t] == e) slot = t;
            const uint32_t m = __ballot_sync(0xffffffffu, slot >= 0);
            if (slot >= 0) {
                const int j = j0 + __popc(m & ((1u << lane) - 1u));
                rt.asg_row[j] = r;
                rt.inv[r * K + slot] = j;
            }
            j0 += __popc(m);
        }
    }
    for (int r = tid; r < R; r += blockDim.x) rt.asg_row[s_tot[0] + r] = r;
}

// ------------------------------------------------------- grouped GEMV

struct GroupedParams {
    const uint8_t *eq, *es;    // expert stack (tiled layout, experts back to back)
    const uint8_t *shq, *shs;  // shared expert (tiled layout)
    size_t q_stride, s_stride; // bytes per expert matrix
    int N, K, NC, RG, KT;      // one expert matrix: rows (GPU layout), columns
    const int *grp_n, *grp_expert, *grp_off, *asg_row, *grp_item, *n_items;
    int RB, RBC;               // row blocks of one matrix, row blocks per work item
    const float *x;            // source activations
    int gather;                // 1: row asg_row[j] of x, 0: row j of x
    float *y;                  // [assignments][N or N/2]
    int silu;                  // gate/up interleaved rows -> silu(g) * u
    const float *ts_tab;       // NVFP4 tensor scales: [E][2] (gate/up) or [E]
    float ts_sh, ts_sh_up;     // shared expert
    int nst;
    uint32_t *err;
};

// Persistent CTAs over the work items: item = (group, pass of up to MOE_M of
// the group's rows, chunk of RBC row blocks of the expert's matrix); CTA c
// takes items c, c + grid, ...  The producer warp streams the same item
// sequence (the routing comes from the previous kernel, so it waits for it
// first) and runs ahead across items; the consumers stage each item's
// activation rows, then consume its RBC x KT tiles, with the epilogue of each
// 128-row block.  Items are independent: results do not depend on the grid.
struct MoeItem {
    int expert, off, mcnt, rb0, rb1;
};

__device__ __forceinline__ MoeItem moe_item(const GroupedParams &p, int i) {
    // group of item i: grp_item is ascending (binary search)
    int lo = 0, hi = *p.grp_n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.grp_item[mid] <= i) lo = mid; else hi = mid - 1;
    }
    const int g = lo;
    const int local = i - p.grp_item[g];
    const int tb = local / MOE_NRC, rc = local - tb * MOE_NRC;
    const int cnt = p.grp_off[g + 1] - p.grp_off[g];
    MoeItem it;
    it.expert = p.grp_expert[g];
    it.off = p.grp_off[g] + tb * MOE_M;
    it.mcnt = min(MOE_M, cnt - tb * MOE_M);
    it.rb0 = min(p.RB, rc * p.RBC);
    it.rb1 = min(p.RB, it.rb0 + p.RBC);
    return it;
}

// One-pass staging of up to MR activation rows (rows mcnt..MR-1 staged as
// zeros) in the staged form of stage_x: every row's 16-byte loads of a batch
// in flight together, the 8 lanes that loaded a chunk exchanging halves with
// the lane 4 apart (Q4_0 granules) and adding up its sum; chunks never
// straddle rows (a row is a multiple of 8 elements).  Row m lands at xs + m * CS * 32, its chunk terms at ct + m * CS.
template <int FMT, int MR>
__device__ __forceinline__ void stage_rows_t(const float4 *const (&src)[MR], int mcnt, int n4, float *xs, float *ct,
                                             int CS, int tid) {
    constexpr int U = 8, STEP = GV_CW * 32;
    const int j = tid & 7, tot = MR * n4;
    for (int b = 0; b < tot; b += U * STEP) {
        float4 v[U];
#pragma unroll
        for (int u = 0; u < U; u++) {
            const int i = b + u * STEP + tid;
            const int m = i / n4, e = i - m * n4;
            const float4 *row = src[0];
#pragma unroll
            for (int mm = 1; mm < MR; mm++)
                if (m == mm) row = src[mm];
            v[u] = (i < tot && m < mcnt) ? row[e] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
#pragma unroll
        for (int u = 0; u < U; u++) {
            if (b + u * STEP >= tot) break;   // uniform
            const int i = b + u * STEP + tid;
            const bool keep = i < tot;
            const int m = keep ? i / n4 : 0, d = keep ? i - m * n4 : 0;
            const float4 w = v[u];
            const int c = d >> 3;
            float *xm = xs + static_cast<size_t>(m) * CS * 32;
            if constexpr (FMT == BW_FMT_Q4_0) {
                const float4 o = make_float4(__shfl_xor_sync(0xffffffffu, w.x, 4), __shfl_xor_sync(0xffffffffu, w.y, 4),
                                             __shfl_xor_sync(0xffffffffu, w.z, 4), __shfl_xor_sync(0xffffffffu, w.w, 4));
                const bool low = j < 4;
                const float4 A = low ? w : o, B = low ? o : w;
                const int G = low ? 2 * j : 2 * (j - 4) + 1;
                const float4 gr = low ? make_float4(A.x, B.x, A.y, B.y) : make_float4(A.z, B.z, A.w, B.w);
                float cs = (w.x + w.y) + (w.z + w.w);
                cs += __shfl_xor_sync(0xffffffffu, cs, 1);
                cs += __shfl_xor_sync(0xffffffffu, cs, 2);
                cs += __shfl_xor_sync(0xffffffffu, cs, 4);
                if (keep) {
                    *reinterpret_cast<float4 *>(xm + c * 32 + 4 * (G ^ (c & 7))) =
                        make_float4(gr.x * __int_as_float((127 + 101) << 23), gr.y * __int_as_float((127 + 97) << 23),
                                    gr.z * __int_as_float((127 + 93) << 23), gr.w * __int_as_float((127 + 89) << 23));
                    if (j == 0) ct[static_cast<size_t>(m) * CS + c] = cs * -2.8421709430404007e-14f;   // -8 * 2^-48
                }
            } else {
                if (keep) *reinterpret_cast<float4 *>(xm + c * 32 + 4 * (j ^ (c & 7))) = w;
            }
        }
    }
}

// One item's row blocks with MR activation rows: the item's rows are staged
// (pre-scaled and swizzled as they are loaded), then each row block's KT
// tiles are consumed and its outputs written.  `step` counts the ring stages (shared with the producer).
template <int FMT, int MR>
__device__ __forceinline__ void moe_item_rows(const GroupedParams &p, const MoeItem &it, const float4 *const (&xr)[MOE_M],
                                              float *xs, float *ct, int CS, int nc, int warp, int lane,
                                              uint32_t stages_a, uint32_t xs_a, uint32_t ct_a, uint64_t *full,
                                              uint64_t *empty, int &step, float ts, float ts_up) {
    const int nst = p.nst, T = p.KT;
    const float4 *rows[MR];
#pragma unroll
    for (int m = 0; m < MR; m++) rows[m] = xr[m];
    stage_rows_t<FMT, MR>(rows, it.mcnt, nc * 8, xs, ct, CS, static_cast<int>(threadIdx.x));
    consumer_sync();
    for (int rb = it.rb0; rb < it.rb1; rb++) {
        const int rg = rb * (GV_TR / 8) + 2 * warp + (lane >> 4);
        float acc[8][MR];
#pragma unroll
        for (int r = 0; r < 8; r++)
#pragma unroll
            for (int m = 0; m < MR; m++) acc[r][m] = 0.0f;
        const ChunkLane cn = chunk_lane(warp, lane);
        for (int kt = 0; kt < T; kt++, step++) {
            const int s = step % nst;
            mbar_wait(&full[s], static_cast<uint32_t>((step / nst) & 1), p.err);
            const int cl = kt * GV_TC + (lane & 15);
            if (cl < nc)
                stage_chunk<FMT, MR>(stages_a + static_cast<uint32_t>(s) * GV_STAGE_BYTES, cn, xs_a, ct_a, cl, CS,
                                     acc);
            __syncwarp();
            if (lane == 0) mbar_arrive_relaxed(&empty[s]);
        }
        float tot[MR];
        reduce_rows16<MR>(acc, lane, tot);
        const int r = (lane >> 1) & 7;
        float val[MR];
#pragma unroll
        for (int m = 0; m < MR; m++) {
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
            for (int m = 0; m < MR; m++) {
                const float up = __shfl_down_sync(0xffffffffu, val[m], 8);
                if (act && r < 4 && m < it.mcnt) {
                    const float gt = val[m];
                    const size_t j = static_cast<size_t>(it.off + m);
                    p.y[j * (p.N / 2) + rg * 4 + r] = (gt / (1.0f + expf(-gt))) * up;
                }
            }
        } else if (act) {
#pragma unroll
            for (int m = 0; m < MR; m++)
                if (m < it.mcnt) p.y[static_cast<size_t>(it.off + m) * p.N + rg * 8 + r] = val[m];
        }
    }
}

template <int FMT>
__global__ void __launch_bounds__(GV_THREADS, 1) moe_grouped_gemv_kernel(const GroupedParams p) {
    constexpr int M = MOE_M;
    extern __shared__ __align__(1024) unsigned char gg_smem[];
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
    const int n_items = *p.n_items;
    const int T = p.KT;

    if (warp == GV_CW) {
        if (lane == 0) {
            int step = 0;
            for (int i = blockIdx.x; i < n_items; i += gridDim.x) {
                const MoeItem it = moe_item(p, i);
                const uint8_t *bq = it.expert >= 0 ? p.eq + static_cast<size_t>(it.expert) * p.q_stride : p.shq;
                const uint8_t *bs = it.expert >= 0 ? p.es + static_cast<size_t>(it.expert) * p.s_stride : p.shs;
                for (int rb = it.rb0; rb < it.rb1; rb++)
                    for (int kt = 0; kt < T; kt++, step++) {
                        const int s = step % nst;
                        if (step >= nst) mbar_wait(&empty[s], static_cast<uint32_t>((step / nst - 1) & 1), p.err);
                        const size_t tile = static_cast<size_t>(rb) * p.KT + kt;
                        unsigned char *st = stages + static_cast<size_t>(s) * GV_STAGE_BYTES;
                        mbar_arrive_tx_relaxed(&full[s], GV_STAGE_BYTES);
                        bulk_g2s(st, bq + tile * GV_NIB_BYTES, GV_NIB_BYTES, &full[s]);
                        bulk_g2s(st + GV_NIB_BYTES, bs + tile * GV_SC_BYTES, GV_SC_BYTES, &full[s]);
                    }
            }
        }
        return;
    }

    const int nc = p.NC;
    int step = 0;
    for (int i = blockIdx.x; i < n_items; i += gridDim.x) {
        const MoeItem it = moe_item(p, i);
        float ts = 1.0f, ts_up = 1.0f;
        if constexpr (FMT == BW_FMT_NVFP4) {
            if (it.expert >= 0) {
                ts = p.silu ? p.ts_tab[2 * it.expert] : p.ts_tab[it.expert];
                ts_up = p.silu ? p.ts_tab[2 * it.expert + 1] : ts;
            } else {
                ts = p.ts_sh;
                ts_up = p.ts_sh_up;
            }
        }
        consumer_sync();   // the previous item is done with the staged activations
        const float4 *xr[M];
#pragma unroll
        for (int m = 0; m < M; m++) {
            xr[m] = reinterpret_cast<const float4 *>(p.x);
            if (m < it.mcnt) {
                const int j = it.off + m;
                xr[m] = reinterpret_cast<const float4 *>(p.x + static_cast<size_t>(p.gather ? p.asg_row[j] : j) * p.K);
            }
        }
        // the inner loop for the item's actual row count (1, 2 or up to 4)
        if (it.mcnt == 1)
            moe_item_rows<FMT, 1>(p, it, xr, xs, ct, CS, nc, warp, lane, stages_a, xs_a, ct_a, full, empty, step, ts, ts_up);
        else if (it.mcnt == 2)
            moe_item_rows<FMT, 2>(p, it, xr, xs, ct, CS, nc, warp, lane, stages_a, xs_a, ct_a, full, empty, step, ts, ts_up);
        else
            moe_item_rows<FMT, M>(p, it, xr, xs, ct, CS, nc, warp, lane, stages_a, xs_a, ct_a, full, empty, step, ts, ts_up);
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
    s.logits = cv.take<float>(static_cast<size_t>((H + MOE_KS - 1) / MOE_KS) * R * E);   // router slice partials
    s.wts = cv.take<float>(static_cast<size_t>(R) * K);
    s.sel = cv.take<int32_t>(static_cast<size_t>(R) * K);
    s.rt.n_items = cv.take<int>(1);
    s.rt.grp_item = cv.take<int>(E + 2);
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

// Where, inside a MoE scratch region at `base`, the top-k kernel leaves the
// selected experts and their weights (when the caller passes no outputs).
void moe_route_buffers(const bw_model *m, int R, char *base, int32_t **sel, float **wts) {
    MoeScratch ms;
    moe_carve(m, R, base, &ms);
    *sel = ms.sel;
    *wts = ms.wts;
}

template <int FMT>
static bw_status grouped_go(const GroupedParams &p, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(p.nst) * GV_STAGE_BYTES +
                        static_cast<size_t>(MOE_M) * p.KT * GV_TC * 33 * 4 + 16 + 2 * static_cast<size_t>(p.nst) * 8;
    static size_t attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return BW_ERR_CUDA;
    {
        static std::mutex mu;   // host threads may call the library concurrently
        std::lock_guard<std::mutex> lk(mu);
        if (attr_set[dev] < smem) {
            if (cudaFuncSetAttribute(moe_grouped_gemv_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem)) != cudaSuccess) {
                (void)cudaGetLastError();
                return BW_ERR_CUDA;
            }
            attr_set[dev] = smem;
        }
    }
    // persistent: one CTA per SM, items assigned round robin
    return launch_pdl(moe_grouped_gemv_kernel<FMT>, dim3(sm_count()), dim3(GV_THREADS), smem, st, p);
}

bw_status moe_ffn_launch(const bw_model *m, const bw_layer *ly, float *x, int R, const Scratch &sc, char *moe_base,
                         cudaStream_t st, int32_t *topk_idx, float *topk_w);

bw_status moe_ffn_launch(const bw_model *m, const bw_layer *ly, float *x, int R, const Scratch &sc, char *moe_base,
                         cudaStream_t st) {
    return moe_ffn_launch(m, ly, x, R, sc, moe_base, st, nullptr, nullptr);
}

bw_status moe_check(const bw_model *m, const bw_layer *ly, int R) {
    if (!m || !ly) return BW_ERR_INVALID_ARG;
    const int E = m->n_experts, K = m->topk, H = m->H, Fe = m->F_exp;
    const int fmt = ly->sgu.fmt;
    if (E <= 0 || E > MOE_EMAX || K <= 0 || K > MOE_KMAX || K > E || R <= 0 || R > MOE_RMAX)
        return BW_ERR_UNSUPPORTED_SHAPE;
    if (H <= 0 || Fe <= 0 || H % 32 || Fe % 32) return BW_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<size_t>(MOE_M) * gv_col_tiles(H) * GV_TC * 33 * 4 > 66 * 1024) return BW_ERR_UNSUPPORTED_SHAPE;
    if (!ly->router || !ly->egu_q || !ly->egu_s || !ly->ed_q || !ly->ed_s || !ly->ffn_norm || !ly->sgu.q ||
        !ly->sgu.s || !ly->sd.q || !ly->sd.s)
        return BW_ERR_INVALID_ARG;
    if (fmt != BW_FMT_Q4_0 && fmt != BW_FMT_NVFP4) return BW_ERR_INVALID_ARG;
    if (fmt == BW_FMT_NVFP4 && (!ly->egu_ts || !ly->ed_ts)) return BW_ERR_INVALID_ARG;
    if (ly->sgu.N != 2 * Fe || ly->sgu.K != H || ly->sd.N != H || ly->sd.K != Fe || ly->sd.fmt != fmt)
        return BW_ERR_INVALID_ARG;
    // the grouped GEMVs stream every expert matrix with bulk copies
    if (!aligned16(ly->egu_q) || !aligned16(ly->egu_s) || !aligned16(ly->ed_q) || !aligned16(ly->ed_s) ||
        !aligned16(ly->sgu.q) || !aligned16(ly->sgu.s) || !aligned16(ly->sd.q) || !aligned16(ly->sd.s))
        return BW_ERR_INVALID_ARG;
    return BW_OK;
}

bw_status moe_ffn_launch(const bw_model *m, const bw_layer *ly, float *x, int R, const Scratch &sc, char *moe_base,
                         cudaStream_t st, int32_t *topk_idx, float *topk_w) {
    const bw_status chk = moe_check(m, ly, R);
    if (chk != BW_OK) return chk;
    if (!x || !moe_base) return BW_ERR_INVALID_ARG;
    const int E = m->n_experts, K = m->topk, H = m->H, Fe = m->F_exp;
    const int fmt = ly->sgu.fmt;
    MoeScratch ms;
    moe_carve(m, R, moe_base, &ms);
    bw_status s = rmsnorm_launch(x, nullptr, ly->ffn_norm, R, H, m->eps, ms.y, 0, st);
    if (s != BW_OK) return s;
    const int n_slices = (H + MOE_KS - 1) / MOE_KS;
    {
        const size_t rsm = (static_cast<size_t>(MOE_KS) * 33 + 8 * MOE_KS) * 4;
        static bool attr_set[64] = {};
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev < 0 || dev >= 64) return BW_ERR_CUDA;
        static std::mutex mu;   // host threads may call the library concurrently
        std::unique_lock<std::mutex> lk(mu);
        if (!attr_set[dev]) {
            if (cudaFuncSetAttribute(moe_router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(rsm)) != cudaSuccess) {
                (void)cudaGetLastError();
                return BW_ERR_CUDA;
            }
            attr_set[dev] = true;
        }
        lk.unlock();
        s = launch_pdl(moe_router_kernel, dim3((E + 7) / 8, n_slices, (R + 31) / 32), dim3(256), rsm, st,
                       static_cast<const float *>(ms.y), ly->router, R, H, E, ms.logits);
    }
    if (s != BW_OK) return s;
    int32_t *sel = topk_idx ? topk_idx : ms.sel;
    float *wts = topk_w ? topk_w : ms.wts;
    s = E <= 256 ? launch_pdl(moe_topk_kernel<8>, dim3(1), dim3(1024), 0, st, static_cast<const float *>(ms.logits),
                              n_slices, R, E, K, sel, wts, ms.rt)
                 : launch_pdl(moe_topk_kernel<MOE_EMAX / 32>, dim3(1), dim3(1024), 0, st,
                              static_cast<const float *>(ms.logits), n_slices, R, E, K, sel, wts, ms.rt);
    if (s != BW_OK) return s;
    GroupedParams gp;
    gp.grp_n = ms.rt.grp_n;
    gp.grp_expert = ms.rt.grp_expert;
    gp.grp_off = ms.rt.grp_off;
    gp.asg_row = ms.rt.asg_row;
    gp.grp_item = ms.rt.grp_item;
    gp.n_items = ms.rt.n_items;
    gp.nst = 4;
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
    gp.RB = gv_row_blocks(gp.N);
    gp.RBC = (gp.RB + MOE_NRC - 1) / MOE_NRC;
    gp.x = ms.y;
    gp.gather = 1;
    gp.y = ms.act;
    gp.silu = 1;
    gp.ts_tab = ly->egu_ts;
    gp.ts_sh = ly->sgu.ts;
    gp.ts_sh_up = ly->sgu.ts_up;
    s = fmt == BW_FMT_Q4_0 ? grouped_go<BW_FMT_Q4_0>(gp, st) : grouped_go<BW_FMT_NVFP4>(gp, st);
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
    gp.RB = gv_row_blocks(H);
    gp.RBC = (gp.RB + MOE_NRC - 1) / MOE_NRC;
    gp.x = ms.act;
    gp.gather = 0;
    gp.y = ms.dout;
    gp.silu = 0;
    gp.ts_tab = ly->ed_ts;
    gp.ts_sh = ly->sd.ts;
    gp.ts_sh_up = ly->sd.ts;
    s = fmt == BW_FMT_Q4_0 ? grouped_go<BW_FMT_Q4_0>(gp, st) : grouped_go<BW_FMT_NVFP4>(gp, st);
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
    if (!m || !ly || !bw::ws_ok(ws)) return BW_ERR_INVALID_ARG;
    if (ws_bytes < bw_moe_workspace_bytes(m, R)) return BW_ERR_INVALID_ARG;
    bw::Scratch sc = bw::scratch_of(ws, ws_bytes);
    return bw::moe_ffn_launch(m, ly, x, R, sc, sc.base, static_cast<cudaStream_t>(stream), topk_idx, topk_w);
}

size_t bw_moe_workspace_bytes(const bw_model *m, int R) {
    if (!m || R <= 0 || m->n_experts <= 0) return BW_WS_HDR_BYTES;
    return BW_WS_HDR_BYTES + bw::moe_scratch_bytes(m, R);
}

}  // extern "C"
