// gemv.cu -- fused dequant-GEMV over 4-bit block-quantized weights (sm_100a).
//
// y = W x for 1..4 activation rows, W in Q4_0 or NVFP4 (GPU layout, see
// bw.h).  Fused: RMSNorm prologue, residual-add / SiLU-gate epilogues, greedy
// argmax over the outputs.  The fusion follows the devpress bw24 page,
// section 2.2 (linear + activation in one kernel, intermediates in registers
// and shared memory).
//
// Work decomposition.  Rows come in groups of 8 ("row groups", rg); the K
// axis in 32-element chunks.  K is cut into S slices so that RG*S work items
// cover ~2 CTAs x 8 warps per SM; one warp owns one (rg, slice) item at a
// time and each lane streams whole chunks of that item: 8 rows x 16 bytes of
// nibbles + 16 bytes of scales per chunk, with every warp-wide load
// instruction covering 512 contiguous bytes.  The activation slice is staged
// once per CTA in shared memory (16-byte granules XOR-swizzled by chunk so
// the 32 lanes of a warp hit distinct banks).  Items with S > 1 leave their
// partial sums in the workspace; the last warp to finish a row group (atomic
// counter, no waiting) adds the slices in slice order, so results are
// deterministic run to run.
//
// Q4_0 arithmetic without integer->float conversions: a nibble q masked in
// place into the low bits of an fp32 word is the denormal q * 2^(4p-149)
// (p = its nibble slot within a 16-bit half).  The activation is pre-scaled
// by 2^(101-4p), so the product is exactly q*x*2^-48 and the FMA accumulates
// it in the normal fp32 range.  The -8 offset enters once per chunk through
// the activation's chunk sum.  With one-hot x the result is exactly d*(q-8),
// i.e. the dequantized weight, bit for bit.
//
// NVFP4: the sm_100a e2m1x2 -> f16x2 conversion gives exact values; the E4M3
// block scale multiplies each 16-element block dot, the tensor scale the
// final sum.
//
// Programmatic dependent launch: weights are constant, so every warp issues
// the loads of its first chunk before griddepcontrol.wait; only the
// activations and the outputs depend on the previous kernel.
#include <math.h>
#include <stdio.h>

#include "bw_common.cuh"

namespace bw {

constexpr int GEMV_THREADS = 256;
constexpr int GEMV_WARPS = GEMV_THREADS / 32;
constexpr int GEMV_MAX_M = 4;

struct GemvParams {
    const uint8_t *q;      // [N][K/2]
    const uint4 *s;        // [N/8][K/32] x 16 bytes
    int N, K, M;
    int NC, RG;            // chunks per row, row groups
    int S, CS;             // slices, chunks per slice
    int grid_rg;           // CTAs per slice
    const float *x;        // [M][K]
    const float *gamma;    // [K] or null
    float eps;
    const float *residual; // [M][N] or null
    float *y;              // [M][N] ([M][N/2] with SILU_GATE) or null
    int32_t *argmax_out;   // [M] or null
    unsigned flags;
    float ts, ts_up;
    float *partial;        // [S][RG][8][M]
    uint32_t *rg_cnt;      // [RG]
    float *am_val;         // [grid][M]
    int *am_idx;           // [grid][M]
    uint32_t *am_cnt;      // [1]
    int32_t *adv_tokens;   // [M] or null: also receives the argmax (next step's input)
    int32_t *adv_pos;      // [M] or null: incremented after the argmax
};

// x'[m][e] for element e of chunk c lives at granule (g ^ (c & 7)) of the
// chunk, g = idx / 4, idx = position of e in the kernel's consumption order.
__device__ __forceinline__ int q4_order(int e) {
    // byte j = e % 16 of the block: word j/4, nibble 2*(j%4) (+1 for the high half)
    const int j = e & 15;
    return 8 * (j >> 2) + 2 * (j & 3) + (e >> 4);
}

__device__ __forceinline__ float4 ld_gran(const float *xs_chunk, int g, int c) {
    return *reinterpret_cast<const float4 *>(xs_chunk + 4 * (g ^ (c & 7)));
}

template <int FMT>
__device__ __forceinline__ void load_chunk(const GemvParams &p, int rg, int kc, uint4 (&w)[9]) {
    const uint8_t *base = p.q + static_cast<size_t>(rg) * 8u * static_cast<size_t>(p.K / 2) +
                          static_cast<size_t>(kc) * 16u;
    const size_t rs = static_cast<size_t>(p.K / 2);
#pragma unroll
    for (int r = 0; r < 8; r++) w[r] = ld_stream16(base + r * rs);
    w[8] = ld_stream16(p.s + static_cast<size_t>(rg) * p.NC + kc);
}

__device__ __forceinline__ uint32_t u4_get(const uint4 &v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// acc[r][m] += dot(row r of this chunk, x'[m] of this chunk)
template <int FMT, int M>
__device__ __forceinline__ void compute_chunk(const uint4 (&w)[9], const float *xs, const float *ct,
                                              int cl, int chunk_stride, float (&acc)[8][M]) {
    if constexpr (FMT == BW_FMT_Q4_0) {
        float bd[8][M];
#pragma unroll
        for (int r = 0; r < 8; r++)
#pragma unroll
            for (int m = 0; m < M; m++) bd[r][m] = ct[m * chunk_stride];
#pragma unroll
        for (int wd = 0; wd < 4; wd++) {
            float4 xa[M], xb[M];
#pragma unroll
            for (int m = 0; m < M; m++) {
                const float *xc = xs + static_cast<size_t>(m) * chunk_stride * 32 + cl * 32;
                xa[m] = ld_gran(xc, 2 * wd, cl);
                xb[m] = ld_gran(xc, 2 * wd + 1, cl);
            }
#pragma unroll
            for (int r = 0; r < 8; r++) {
                const uint32_t v = u4_get(w[r], wd);
                const uint32_t h = v >> 16;
                const float f0 = __uint_as_float(v & 0xfu), f1 = __uint_as_float(v & 0xf0u);
                const float f2 = __uint_as_float(v & 0xf00u), f3 = __uint_as_float(v & 0xf000u);
                const float f4 = __uint_as_float(h & 0xfu), f5 = __uint_as_float(h & 0xf0u);
                const float f6 = __uint_as_float(h & 0xf00u), f7 = __uint_as_float(h & 0xf000u);
#pragma unroll
                for (int m = 0; m < M; m++) {
                    float b = bd[r][m];
                    b = fma_rn(f0, xa[m].x, b);
                    b = fma_rn(f1, xa[m].y, b);
                    b = fma_rn(f2, xa[m].z, b);
                    b = fma_rn(f3, xa[m].w, b);
                    b = fma_rn(f4, xb[m].x, b);
                    b = fma_rn(f5, xb[m].y, b);
                    b = fma_rn(f6, xb[m].z, b);
                    b = fma_rn(f7, xb[m].w, b);
                    bd[r][m] = b;
                }
            }
        }
#pragma unroll
        for (int r = 0; r < 8; r++) {
            const float d = half_bits_to_f((u4_get(w[8], r >> 1) >> (16 * (r & 1))) & 0xffffu);
#pragma unroll
            for (int m = 0; m < M; m++) acc[r][m] = fma_rn(d, bd[r][m], acc[r][m]);
        }
    } else {
#pragma unroll
        for (int half = 0; half < 2; half++) {
            float bd[8][M];
#pragma unroll
            for (int r = 0; r < 8; r++)
#pragma unroll
                for (int m = 0; m < M; m++) bd[r][m] = 0.0f;
#pragma unroll
            for (int wd = 2 * half; wd < 2 * half + 2; wd++) {
                float4 xa[M], xb[M];
#pragma unroll
                for (int m = 0; m < M; m++) {
                    const float *xc = xs + static_cast<size_t>(m) * chunk_stride * 32 + cl * 32;
                    xa[m] = ld_gran(xc, 2 * wd, cl);
                    xb[m] = ld_gran(xc, 2 * wd + 1, cl);
                }
#pragma unroll
                for (int r = 0; r < 8; r++) {
                    const uint32_t v = u4_get(w[r], wd);
                    const float2 e0 = e2m1x2_to_f2(v & 0xffu);
                    const float2 e1 = e2m1x2_to_f2((v >> 8) & 0xffu);
                    const float2 e2 = e2m1x2_to_f2((v >> 16) & 0xffu);
                    const float2 e3 = e2m1x2_to_f2(v >> 24);
#pragma unroll
                    for (int m = 0; m < M; m++) {
                        float b = bd[r][m];
                        b = fma_rn(e0.x, xa[m].x, b);
                        b = fma_rn(e0.y, xa[m].y, b);
                        b = fma_rn(e1.x, xa[m].z, b);
                        b = fma_rn(e1.y, xa[m].w, b);
                        b = fma_rn(e2.x, xb[m].x, b);
                        b = fma_rn(e2.y, xb[m].y, b);
                        b = fma_rn(e3.x, xb[m].z, b);
                        b = fma_rn(e3.y, xb[m].w, b);
                        bd[r][m] = b;
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < 8; r++) {
                const uint32_t two = (u4_get(w[8], r >> 1) >> (16 * (r & 1))) & 0xffffu;
                const float2 sc = e4m3x2_to_f2(two);
                const float s = half ? sc.y : sc.x;
#pragma unroll
                for (int m = 0; m < M; m++) acc[r][m] = fma_rn(s, bd[r][m], acc[r][m]);
            }
        }
    }
}

// Reduce acc[8][M] over the 32 lanes.  Afterwards lane l with (l & 3) == 0
// holds the totals of row (l >> 2) in out[m].
template <int M>
__device__ __forceinline__ void reduce_rows(float (&acc)[8][M], int lane, float (&out)[M]) {
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
#pragma unroll
    for (int m = 0; m < M; m++) {
        float b[4], c[2];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float send = b4 ? acc[i][m] : acc[i + 4][m];
            const float keep = b4 ? acc[i + 4][m] : acc[i][m];
            b[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
#pragma unroll
        for (int i = 0; i < 2; i++) {
            const float send = b3 ? b[i] : b[i + 2];
            const float keep = b3 ? b[i + 2] : b[i];
            c[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
        const float send = b2 ? c[0] : c[1];
        const float keep = b2 ? c[1] : c[0];
        float d = keep + __shfl_xor_sync(0xffffffffu, send, 4);
        d += __shfl_xor_sync(0xffffffffu, d, 2);
        d += __shfl_xor_sync(0xffffffffu, d, 1);
        out[m] = d;
    }
}

// Final values of row group rg (lanes with (lane & 3) == 0 hold row lane>>2):
// scale, epilogue, outputs, argmax tracking.
template <int FMT, int M>
__device__ __forceinline__ void epilogue(const GemvParams &p, int rg, int lane, const float (&tot)[M],
                                         float (&bestv)[M], int (&besti)[M]) {
    const int r = lane >> 2;
    const bool gu = p.flags & BW_GEMV_SILU_GATE;
    float val[M];
#pragma unroll
    for (int m = 0; m < M; m++) {
        float v = tot[m];
        if constexpr (FMT == BW_FMT_Q4_0) {
            v = v * 281474976710656.0f;   // 2^48 undoes the activation pre-scale
        } else {
            v = v * ((gu && r >= 4) ? p.ts_up : p.ts);
        }
        val[m] = v;
    }
    if (gu) {
        // gate row r (< 4) pairs with up row r + 4, held by lane + 16
#pragma unroll
        for (int m = 0; m < M; m++) {
            const float up = __shfl_down_sync(0xffffffffu, val[m], 16);
            if ((lane & 3) == 0 && r < 4 && m < p.M) {
                const float g = val[m];
                const float a = (g / (1.0f + expf(-g))) * up;
                p.y[static_cast<size_t>(m) * (p.N / 2) + rg * 4 + r] = a;
            }
        }
        return;
    }
    if ((lane & 3) != 0) return;
    const int n = rg * 8 + r;
#pragma unroll
    for (int m = 0; m < M; m++) {
        if (m >= p.M) break;
        float v = val[m];
        const size_t o = static_cast<size_t>(m) * p.N + n;
        if (p.flags & BW_GEMV_RESIDUAL) v = p.residual[o] + v;
        if (p.y) p.y[o] = v;
        if (better(v, n, bestv[m], besti[m])) {
            bestv[m] = v;
            besti[m] = n;
        }
    }
}

// CTAs resident per SM the launch plan assumes (register budget 128 at M = 1)
template <int M>
constexpr int gemv_ctas_per_sm() { return M == 1 ? 2 : 1; }

template <int FMT, int M>
__global__ void __launch_bounds__(GEMV_THREADS, gemv_ctas_per_sm<M>()) gemv_kernel(const GemvParams p) {
    extern __shared__ float4 smem4[];
    float *xs = reinterpret_cast<float *>(smem4);      // [M][CS][32] swizzled
    float *ct = xs + static_cast<size_t>(M) * p.CS * 32; // [M][CS] chunk terms (Q4_0)
    __shared__ float s_red[GEMV_WARPS][M];
    __shared__ float s_rnorm[M];
    __shared__ float s_bv[GEMV_WARPS][M];
    __shared__ int s_bi[GEMV_WARPS][M];
    __shared__ bool s_last;

    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slice = blockIdx.x % p.S;
    const int cta_in_slice = blockIdx.x / p.S;
    const int c0 = slice * p.CS;
    const int nc = min(p.CS, p.NC - c0);
    const int u = (nc + 31) >> 5;
    const int rg_stride = p.grid_rg * GEMV_WARPS;

    // ---- prefetch the first chunk of this warp's first item (constant data)
    int rg = cta_in_slice * GEMV_WARPS + warp;
    int j = 0;
    uint4 cur[9];
    if (rg < p.RG && lane < nc) load_chunk<FMT>(p, rg, c0 + lane, cur);

    pdl_wait();

    // ---- prologue: activations of this slice into shared memory
    if (p.flags & BW_GEMV_RMSNORM) {
        float ss[M];
#pragma unroll
        for (int m = 0; m < M; m++) ss[m] = 0.0f;
        for (int k = threadIdx.x; k < p.K; k += GEMV_THREADS)
#pragma unroll
            for (int m = 0; m < M; m++)
                if (m < p.M) {
                    const float v = p.x[static_cast<size_t>(m) * p.K + k];
                    ss[m] = fma_rn(v, v, ss[m]);
                }
#pragma unroll
        for (int m = 0; m < M; m++) {
            ss[m] = warp_sum(ss[m]);
            if (lane == 0) s_red[warp][m] = ss[m];
        }
        __syncthreads();
        if (threadIdx.x < M) {
            float t = 0.0f;
            for (int w2 = 0; w2 < GEMV_WARPS; w2++) t += s_red[w2][threadIdx.x];
            s_rnorm[threadIdx.x] = 1.0f / sqrtf(t / static_cast<float>(p.K) + p.eps);
        }
        __syncthreads();
    }
    for (int pair = warp; pair < M * nc; pair += GEMV_WARPS) {
        const int m = pair / nc, cl = pair - m * nc;
        const int e = lane;
        const int k = (c0 + cl) * 32 + e;
        float v = 0.0f;
        if (m < p.M) {
            v = p.x[static_cast<size_t>(m) * p.K + k];
            if (p.flags & BW_GEMV_RMSNORM) v = (v * s_rnorm[m]) * p.gamma[k];
        }
        float *xc = xs + static_cast<size_t>(m) * p.CS * 32 + cl * 32;
        if constexpr (FMT == BW_FMT_Q4_0) {
            const int idx = q4_order(e);
            const float scale = __int_as_float((127 + 101 - 4 * (idx & 3)) << 23);
            xc[4 * ((idx >> 2) ^ (cl & 7)) + (idx & 3)] = v * scale;
            const float sum = warp_sum(v);
            if (lane == 0) ct[m * p.CS + cl] = sum * -2.8421709430404007e-14f;  // -8 * 2^-48
        } else {
            xc[4 * ((e >> 2) ^ (cl & 7)) + (e & 3)] = v;
        }
    }
    __syncthreads();

    // ---- main loop over (item, chunk) steps with a one-step prefetch
    float acc[8][M];
#pragma unroll
    for (int r = 0; r < 8; r++)
#pragma unroll
        for (int m = 0; m < M; m++) acc[r][m] = 0.0f;
    float bestv[M];
    int besti[M];
#pragma unroll
    for (int m = 0; m < M; m++) {
        bestv[m] = -INFINITY;
        besti[m] = 0x7fffffff;
    }

    while (rg < p.RG) {
        int nrg = rg, nj = j + 1;
        if (nj == u) {
            nj = 0;
            nrg = rg + rg_stride;
        }
        uint4 nxt[9];
        const int ncl = lane + 32 * nj;
        if (nrg < p.RG && ncl < nc) load_chunk<FMT>(p, nrg, c0 + ncl, nxt);
        const int cl = lane + 32 * j;
        if (cl < nc) compute_chunk<FMT, M>(cur, xs, ct + cl, cl, p.CS, acc);
        if (j == u - 1) {
            float tot[M];
            reduce_rows<M>(acc, lane, tot);
#pragma unroll
            for (int r = 0; r < 8; r++)
#pragma unroll
                for (int m = 0; m < M; m++) acc[r][m] = 0.0f;
            if (p.S == 1) {
                epilogue<FMT, M>(p, rg, lane, tot, bestv, besti);
            } else {
                const int r = lane >> 2;
                if ((lane & 3) == 0) {
                    float *dst = p.partial + ((static_cast<size_t>(slice) * p.RG + rg) * 8 + r) * M;
#pragma unroll
                    for (int m = 0; m < M; m++) __stcg(dst + m, tot[m]);
                }
                __threadfence();
                __syncwarp();
                uint32_t old = 0;
                if (lane == 0) old = atomicAdd(p.rg_cnt + rg, 1u);
                old = __shfl_sync(0xffffffffu, old, 0);
                if (old == static_cast<uint32_t>(p.S - 1)) {
                    __threadfence();
                    float sum[M];
#pragma unroll
                    for (int m = 0; m < M; m++) sum[m] = 0.0f;
                    if ((lane & 3) == 0)
                        for (int s2 = 0; s2 < p.S; s2++) {
                            const float *src = p.partial + ((static_cast<size_t>(s2) * p.RG + rg) * 8 + r) * M;
#pragma unroll
                            for (int m = 0; m < M; m++) sum[m] += ld_cg(src + m);
                        }
                    epilogue<FMT, M>(p, rg, lane, sum, bestv, besti);
                    if (lane == 0) p.rg_cnt[rg] = 0u;
                }
            }
        }
        rg = nrg;
        j = nj;
#pragma unroll
        for (int i = 0; i < 9; i++) cur[i] = nxt[i];
    }

    // ---- greedy argmax over all outputs
    if (p.flags & BW_GEMV_ARGMAX) {
#pragma unroll
        for (int m = 0; m < M; m++) {
            float v = bestv[m];
            int i = besti[m];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, v, o);
                const int oi = __shfl_xor_sync(0xffffffffu, i, o);
                if (better(ov, oi, v, i)) {
                    v = ov;
                    i = oi;
                }
            }
            if (lane == 0) {
                s_bv[warp][m] = v;
                s_bi[warp][m] = i;
            }
        }
        __syncthreads();
        if (threadIdx.x < M) {
            const int m = threadIdx.x;
            float v = s_bv[0][m];
            int i = s_bi[0][m];
            for (int w2 = 1; w2 < GEMV_WARPS; w2++)
                if (better(s_bv[w2][m], s_bi[w2][m], v, i)) {
                    v = s_bv[w2][m];
                    i = s_bi[w2][m];
                }
            __stcg(p.am_val + blockIdx.x * M + m, v);
            __stcg(p.am_idx + blockIdx.x * M + m, i);
        }
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) s_last = atomicAdd(p.am_cnt, 1u) == gridDim.x - 1;
        __syncthreads();
        if (s_last) {
            __threadfence();
            for (int m = warp; m < p.M; m += GEMV_WARPS) {
                float v = -INFINITY;
                int i = 0x7fffffff;
                for (int b = lane; b < static_cast<int>(gridDim.x); b += 32) {
                    const float bv = ld_cg(p.am_val + b * M + m);
                    const int bi = __ldcg(p.am_idx + b * M + m);
                    if (better(bv, bi, v, i)) {
                        v = bv;
                        i = bi;
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, v, o);
                    const int oi = __shfl_xor_sync(0xffffffffu, i, o);
                    if (better(ov, oi, v, i)) {
                        v = ov;
                        i = oi;
                    }
                }
                if (lane == 0) {
                    const int tok = (i == 0x7fffffff) ? 0 : i;
                    p.argmax_out[m] = tok;
                    if (p.adv_tokens) p.adv_tokens[m] = tok;
                    if (p.adv_pos) p.adv_pos[m] += 1;
                }
            }
            if (threadIdx.x == 0) *p.am_cnt = 0u;
        }
    }
}

// ------------------------------------------------------------------- host

struct GemvPlan {
    int S, CS, grid_rg, grid;
    size_t smem;
    size_t partial_floats;
};

static GemvPlan plan_gemv(int N, int K, int Mk) {
    GemvPlan pl;
    const int RG = N / 8, NC = K / 32;
    const int per_sm = Mk == 1 ? gemv_ctas_per_sm<1>() : gemv_ctas_per_sm<2>();
    const int target_warps = sm_count() * per_sm * GEMV_WARPS;
    int S = 1;
    if (RG < target_warps) {
        S = (target_warps + RG / 2) / RG;
        S = max(1, min(S, max(1, NC / 16)));
    }
    int CS = (NC + S - 1) / S;
    S = (NC + CS - 1) / CS;
    // keep the staged activations within 96 KB
    while (static_cast<size_t>(Mk) * CS * 33 * 4 > 96u * 1024u && CS > 32) {
        S++;
        CS = (NC + S - 1) / S;
        S = (NC + CS - 1) / CS;
    }
    const int target_ctas = sm_count() * per_sm;
    int grid_rg = (RG + GEMV_WARPS - 1) / GEMV_WARPS;
    grid_rg = max(1, min(grid_rg, target_ctas / S));
    pl.S = S;
    pl.CS = CS;
    pl.grid_rg = grid_rg;
    pl.grid = S * grid_rg;
    pl.smem = static_cast<size_t>(Mk) * CS * 32 * 4 + static_cast<size_t>(Mk) * CS * 4;
    pl.partial_floats = S > 1 ? static_cast<size_t>(S) * RG * 8 * Mk : 0;
    return pl;
}

static int kernel_m(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : 4; }

size_t gemv_scratch_bytes(int N, int K, int M) {
    size_t tot = 0;
    for (int m0 = 0; m0 < M; m0 += GEMV_MAX_M) {
        const int Mk = kernel_m(min(GEMV_MAX_M, M - m0));
        const GemvPlan pl = plan_gemv(N, K, Mk);
        size_t b = align_up(pl.partial_floats * 4, BW_WS_ALIGN) +
                   2 * align_up(static_cast<size_t>(pl.grid) * Mk * 4, BW_WS_ALIGN);
        tot = max(tot, b);
    }
    return tot;
}

template <int FMT, int M>
static bw_status launch_gemv_m(const GemvParams &p0, const GemvPlan &pl, cudaStream_t st) {
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return BW_ERR_CUDA;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(gemv_kernel<FMT, M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 100 * 1024) != cudaSuccess)
            return BW_ERR_CUDA;
        attr_set[dev] = true;
    }
    return launch_pdl(gemv_kernel<FMT, M>, dim3(pl.grid), dim3(GEMV_THREADS), pl.smem, st, p0);
}

bw_status gemv_launch(int fmt, const void *wq, const void *ws_scales, float ts, float ts_up, int N,
                      int K, const float *x, int M, const float *gamma, float eps,
                      const float *residual, float *y, int32_t *argmax_out, unsigned flags,
                      const Scratch &sc, cudaStream_t st, int32_t *adv_tokens, int32_t *adv_pos) {
    if (!wq || !ws_scales || !x || !sc.cnt || N <= 0 || K <= 0 || M <= 0) return BW_ERR_INVALID_ARG;
    if (N % 8 || K % 32) return BW_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(wq) || !aligned16(ws_scales) || !aligned16(x)) return BW_ERR_INVALID_ARG;
    if ((flags & BW_GEMV_RMSNORM) && !gamma) return BW_ERR_INVALID_ARG;
    if ((flags & BW_GEMV_RESIDUAL) && !residual) return BW_ERR_INVALID_ARG;
    if ((flags & BW_GEMV_ARGMAX) && !argmax_out) return BW_ERR_INVALID_ARG;
    if ((flags & BW_GEMV_SILU_GATE) && (flags & (BW_GEMV_RESIDUAL | BW_GEMV_ARGMAX)))
        return BW_ERR_INVALID_ARG;
    if (!(flags & BW_GEMV_ARGMAX) && !y) return BW_ERR_INVALID_ARG;
    if (sc.bytes < gemv_scratch_bytes(N, K, M)) return BW_ERR_INVALID_ARG;
    const int ncols = (flags & BW_GEMV_SILU_GATE) ? N / 2 : N;
    for (int m0 = 0; m0 < M; m0 += GEMV_MAX_M) {
        const int Mr = min(GEMV_MAX_M, M - m0);
        const int Mk = kernel_m(Mr);
        const GemvPlan pl = plan_gemv(N, K, Mk);
        Carver cv(sc.base);
        GemvParams p;
        p.q = static_cast<const uint8_t *>(wq);
        p.s = static_cast<const uint4 *>(ws_scales);
        p.N = N;
        p.K = K;
        p.M = Mr;
        p.NC = K / 32;
        p.RG = N / 8;
        p.S = pl.S;
        p.CS = pl.CS;
        p.grid_rg = pl.grid_rg;
        p.x = x + static_cast<size_t>(m0) * K;
        p.gamma = gamma;
        p.eps = eps;
        p.residual = residual ? residual + static_cast<size_t>(m0) * N : nullptr;
        p.y = y ? y + static_cast<size_t>(m0) * ncols : nullptr;
        p.argmax_out = argmax_out ? argmax_out + m0 : nullptr;
        p.flags = flags;
        p.ts = ts;
        p.ts_up = ts_up;
        p.partial = cv.take<float>(pl.partial_floats);
        p.am_val = cv.take<float>(static_cast<size_t>(pl.grid) * Mk);
        p.am_idx = cv.take<int>(static_cast<size_t>(pl.grid) * Mk);
        p.rg_cnt = sc.cnt + CNT_GEMV_RG;
        p.am_cnt = sc.cnt + CNT_ARGMAX;
        p.adv_tokens = adv_tokens ? adv_tokens + m0 : nullptr;
        p.adv_pos = adv_pos ? adv_pos + m0 : nullptr;
        if (pl.S > 1 && p.RG + CNT_GEMV_RG > CNT_ATTN) return BW_ERR_UNSUPPORTED_SHAPE;
        bw_status stt;
        if (fmt == BW_FMT_Q4_0) {
            stt = Mk == 1 ? launch_gemv_m<BW_FMT_Q4_0, 1>(p, pl, st)
                : Mk == 2 ? launch_gemv_m<BW_FMT_Q4_0, 2>(p, pl, st)
                          : launch_gemv_m<BW_FMT_Q4_0, 4>(p, pl, st);
        } else {
            stt = Mk == 1 ? launch_gemv_m<BW_FMT_NVFP4, 1>(p, pl, st)
                : Mk == 2 ? launch_gemv_m<BW_FMT_NVFP4, 2>(p, pl, st)
                          : launch_gemv_m<BW_FMT_NVFP4, 4>(p, pl, st);
        }
        if (stt != BW_OK) return stt;
    }
    return BW_OK;
}

}  // namespace bw

extern "C" {

bw_status bw_gemv_q4_0(const void *w_q, const void *w_d, int N, int K, const float *x, int M,
                       const float *gamma, float eps, const float *residual, float *y,
                       int32_t *argmax_out, unsigned flags, void *ws, size_t ws_bytes,
                       void *stream) {
    if (!ws) return BW_ERR_INVALID_ARG;
    return bw::gemv_launch(BW_FMT_Q4_0, w_q, w_d, 1.0f, 1.0f, N, K, x, M, gamma, eps, residual, y,
                           argmax_out, flags, bw::scratch_of(ws, ws_bytes),
                           static_cast<cudaStream_t>(stream));
}

bw_status bw_gemv_nvfp4(const void *w_q, const void *w_s, float ts, float ts_up, int N, int K,
                        const float *x, int M, const float *gamma, float eps,
                        const float *residual, float *y, int32_t *argmax_out, unsigned flags,
                        void *ws, size_t ws_bytes, void *stream) {
    if (!ws) return BW_ERR_INVALID_ARG;
    return bw::gemv_launch(BW_FMT_NVFP4, w_q, w_s, ts, ts_up, N, K, x, M, gamma, eps, residual, y,
                           argmax_out, flags, bw::scratch_of(ws, ws_bytes),
                           static_cast<cudaStream_t>(stream));
}

size_t bw_gemv_workspace_bytes(int N, int K, int M, unsigned flags) {
    (void)flags;
    if (N <= 0 || K <= 0 || M <= 0) return BW_WS_HDR_BYTES;
    return BW_WS_HDR_BYTES + bw::gemv_scratch_bytes(N, K, M);
}

}  // extern "C"
