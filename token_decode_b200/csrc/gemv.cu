// gemv.cu -- fused dequant-GEMV over 4-bit block-quantized weights (sm_100a).
//
// y = W x for 1..4 activation rows, W in Q4_0 or NVFP4 (GPU layout, see
// bw.h).  Fused: RMSNorm prologue, residual-add / SiLU-gate epilogues, greedy
// argmax over the outputs.  The fusion follows the devpress bw24 page,
// section 2.2 (linear + activation in one kernel, intermediates in registers
// and shared memory); the TMA staging follows the deep-dive page, section 2
// (asynchronous global->shared prefetch while computing).
//
// Warp-specialized CTA: a producer warp streams weight tiles of 128 rows x
// 512 columns -- in the tiled layout each is one contiguous 32 KB block of
// codes plus one 4 KB block of scales, i.e. two plain bulk copies
// (cp.async.bulk) -- into a ring of shared-memory stages (mbarrier
// full/empty pairs); eight consumer warps each own two 8-row groups of the
// tile (one per half-warp), one 32-column chunk per lane.  The producer
// touches only constant weights, so it starts streaming before
// griddepcontrol.wait, while the previous kernel drains.
//
// Work decomposition: 128-row blocks x K slices.  The slice count S is chosen
// on the host by a makespan search over the SM count; slices leave partial
// sums in the workspace and the last warp to finish a row group (atomic
// counter, no waiting) adds them in slice order, so results are
// deterministic.  The activation slice of a CTA is staged once in shared
// memory (16-byte granules XOR-swizzled by chunk, conflict-free per warp),
// transformed as it is loaded; with the RMSNorm prologue the staged values
// are x * gamma and the scalar 1/rms of each row multiplies the dot products
// in the epilogue.
//
// Q4_0 arithmetic without integer->float conversions: a nibble q masked in
// place into the low bits of an fp32 word is the denormal q * 2^(4p-149)
// (p = its nibble slot within a 16-bit half).  The activation is pre-scaled
// by 2^(101-4p), so each product is exactly q*x*2^-48 and packed fp32x2 FMAs
// accumulate in the normal range.  The -8 offset enters once per chunk
// through the activation's chunk sum.  With one-hot x the result is exactly
// d*(q-8), the dequantized weight.
//
// NVFP4: the sm_100a e2m1x2 -> f16x2 conversion gives exact values; the E4M3
// block scale multiplies each 16-element block dot, the tensor scale the
// final sum.
#include "gemv_core.cuh"

namespace bw {

// Largest dynamic shared memory a CTA may request (the static arrays take the rest).
constexpr size_t GV_SMEM_LIMIT = 227 * 1024 - 2048;

// One activation row: a CTA is half an SM (2 stages, <= 32 KB of staged
// activations, <= 113 registers), so two CTAs share an SM -- two of this
// kernel, or this one and the next kernel on the stream starting early.
// More rows need the registers of a whole SM.
template <int M>
__host__ __device__ constexpr int gv_ctas_per_sm() { return M == 1 ? 2 : 1; }
__host__ __device__ constexpr int gv_stages(int M) { return M == 1 ? 2 : 3; }
__host__ __device__ constexpr size_t gv_xs_limit(int M) { return M == 1 ? 38 * 1024 : 66 * 1024; }

struct GemvParams {
    const uint8_t *q;      // tiled codes
    const uint8_t *s;      // tiled scales
    int N, K, M;
    int NC, RG, RB, KT;    // chunks per row, row groups, row blocks, column tiles
    int S, CT;             // slices, column tiles per slice
    int per_slice;         // CTAs per slice
    int nst;               // pipeline stages
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
    uint32_t *err;
};

// The residual values of row group rg that this lane's epilogue adds
// (zeros where it adds none), loaded early so the load overlaps other work.
template <int M>
__device__ __forceinline__ void load_residual(const GemvParams &p, int rg, int lane, float (&res)[M]) {
#pragma unroll
    for (int m = 0; m < M; m++) res[m] = 0.0f;
    if (!(p.flags & BW_GEMV_RESIDUAL) || (lane & 1) != 0 || rg >= p.RG) return;
    const int n = rg * 8 + ((lane >> 1) & 7);
#pragma unroll
    for (int m = 0; m < M; m++)
        if (m < p.M) res[m] = p.residual[static_cast<size_t>(m) * p.N + n];
}

// Final values of row group rg (lanes with (lane & 1) == 0 hold row
// (lane >> 1) & 7): scale (rs: the RMSNorm factor of each activation row, or
// 1), epilogue (res: the residual to add), outputs,
// argmax tracking.  All lanes must call it (it shuffles); `act` gates the
// stores.
template <int FMT, int M>
__device__ __forceinline__ void epilogue(const GemvParams &p, int rg, int lane, const float (&tot)[M],
                                         const float (&rs)[M], const float (&res)[M], float (&bestv)[M],
                                         int (&besti)[M], bool act) {
    const int r = (lane >> 1) & 7;
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
        val[m] = v * rs[m];
    }
    if (gu) {
        // gate row r (< 4) pairs with up row r + 4, held by lane + 8
#pragma unroll
        for (int m = 0; m < M; m++) {
            const float up = __shfl_down_sync(0xffffffffu, val[m], 8);
            if (act && (lane & 1) == 0 && r < 4 && m < p.M && rg < p.RG) {
                const float g = val[m];
                const float a = (g / (1.0f + expf(-g))) * up;
                p.y[static_cast<size_t>(m) * (p.N / 2) + rg * 4 + r] = a;
            }
        }
        return;
    }
    if (!act || (lane & 1) != 0 || rg >= p.RG) return;
    const int n = rg * 8 + r;
#pragma unroll
    for (int m = 0; m < M; m++) {
        if (m >= p.M) break;
        float v = val[m];
        const size_t o = static_cast<size_t>(m) * p.N + n;
        if (p.flags & BW_GEMV_RESIDUAL) v = res[m] + v;
        if (p.y) p.y[o] = v;
        if (better(v, n, bestv[m], besti[m])) {
            bestv[m] = v;
            besti[m] = n;
        }
    }
}

template <int FMT, int M>
__global__ void __launch_bounds__(GV_THREADS, gv_ctas_per_sm<M>()) gemv_kernel(const GemvParams p) {
    extern __shared__ __align__(1024) unsigned char gv_smem[];
    const int nst = p.nst;
    unsigned char *stages = gv_smem;                                                     // nst x 36 KB
    float *xs = reinterpret_cast<float *>(gv_smem + static_cast<size_t>(nst) * GV_STAGE_BYTES);  // [M][CS][32]
    const int CS = p.CT * GV_TC;                                                          // chunks per slice
    float *ct = xs + static_cast<size_t>(M) * CS * 32;                                   // [M][CS]
    float *gt = ct + ((static_cast<size_t>(M) * CS + 3) & ~static_cast<size_t>(3));      // [CS*32] gains (RMSNorm)
    uint64_t *full = reinterpret_cast<uint64_t *>(gt + ((p.flags & BW_GEMV_RMSNORM) ? CS * 32 : 0));
    uint64_t *empty = full + nst;
    const uint32_t stages_a = smem_u32(stages), xs_a = smem_u32(xs), ct_a = smem_u32(ct);
    __shared__ float s_red[GV_CW][M];
    __shared__ float s_bv[GV_CW][M];
    __shared__ int s_bi[GV_CW][M];
    __shared__ bool s_last;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slice = blockIdx.x % p.S;
    const int j0 = blockIdx.x / p.S;
    const int kt0 = slice * p.CT;
    const int T = min(p.CT, p.KT - kt0);                  // column tiles of this slice
    const int c0 = kt0 * GV_TC;
    const int nc = min(T * GV_TC, p.NC - c0);             // real chunks of this slice
    const int n_items = j0 < p.RB ? (p.RB - 1 - j0) / p.per_slice + 1 : 0;
    const int n_steps = n_items * T;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], GV_CW);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == GV_CW) {
        // ---- producer: constant weights only, so no dependency wait
        if (lane == 0) {
            RingPos rp = {0, 0u};
            for (int step = 0; step < n_steps; step++, ring_next(rp, nst)) {
                const int s = rp.s;
                if (step >= nst) mbar_wait(&empty[s], rp.ph ^ 1u, p.err);
                const int item = step / T, kt = kt0 + (step - item * T);
                const int rb = j0 + item * p.per_slice;
                const size_t tile = static_cast<size_t>(rb) * p.KT + kt;
                unsigned char *st = stages + static_cast<size_t>(s) * GV_STAGE_BYTES;
                mbar_arrive_tx_relaxed(&full[s], GV_STAGE_BYTES);
                bulk_g2s(st, p.q + tile * GV_NIB_BYTES, GV_NIB_BYTES, &full[s]);
                bulk_g2s(st + GV_NIB_BYTES, p.s + tile * GV_SC_BYTES, GV_SC_BYTES, &full[s]);
            }
        }
        return;
    }

    // ---- consumers
    const int ctid = threadIdx.x;   // 0 .. 255
    const bool norm = p.flags & BW_GEMV_RMSNORM;
    const int ne = nc * 32;
    // the slice's RMSNorm gains are model data like the weights: staged
    // before the dependency wait
    if (norm) {
        (void)stage_row4(reinterpret_cast<const float4 *>(p.gamma + c0 * 32), ne / 4, reinterpret_cast<float4 *>(gt),
                         0, ne / 4, ctid);
        consumer_sync();
    }
    pdl_wait();
    // dependents launch only once this kernel's own dependency is met (the
    // producer warp never signals): a kernel that starts after this one may
    // read, before its own wait, whatever the launches before this one wrote
    pdl_trigger();
    // the slice's activations, one batch of independent 16-byte loads per
    // thread, stored straight in the staged form (times the gains); with
    // RMSNorm over a K slice the whole row is read in the same batch, for the
    // sum of squares.  The norm's 1/rms factor is a scalar per row: the
    // epilogue applies it to the dot products.
    float ss[M];
#pragma unroll
    for (int m = 0; m < M; m++) {
        float *xm = xs + static_cast<size_t>(m) * CS * 32;
        float *ctm = ct + static_cast<size_t>(m) * CS;
        if (m >= p.M) {
            float4 *xm4 = reinterpret_cast<float4 *>(xm);
            for (int e = ctid; e < ne / 4; e += GV_CW * 32) xm4[e] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            for (int e = ctid; e < nc; e += GV_CW * 32) ctm[e] = 0.0f;
            ss[m] = 0.0f;
            continue;
        }
        const float4 *xr4 = reinterpret_cast<const float4 *>(p.x + static_cast<size_t>(m) * p.K);
        const float4 *gt4 = norm ? reinterpret_cast<const float4 *>(gt) : nullptr;
        if (norm && p.S > 1)
            ss[m] = stage_row_t<FMT>(xr4, p.K / 4, xm, ctm, gt4, c0 * 8, ne / 4, ctid);
        else
            ss[m] = stage_row_t<FMT>(xr4 + c0 * 8, ne / 4, xm, ctm, gt4, 0, ne / 4, ctid);
    }
    if (norm) {
#pragma unroll
        for (int m = 0; m < M; m++) {
            ss[m] = warp_sum(ss[m]);
            if (lane == 0) s_red[warp][m] = ss[m];
        }
    }
    consumer_sync();
    // per-row output factor: 1/rms with RMSNorm (every thread adds the warps'
    // sums in the same order)
    float rs[M];
#pragma unroll
    for (int m = 0; m < M; m++) {
        rs[m] = 1.0f;
        if (norm) {
            float t = 0.0f;
#pragma unroll
            for (int w2 = 0; w2 < GV_CW; w2++) t += s_red[w2][m];
            rs[m] = 1.0f / sqrtf(t / static_cast<float>(p.K) + p.eps);
        }
    }

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

    const ChunkLane cn = chunk_lane(warp, lane);
    RingPos rp = {0, 0u};
    for (int item = 0; item < n_items; item++) {
        const int rb = j0 + item * p.per_slice;
        const int rg = rb * (GV_TR / 8) + 2 * warp + (lane >> 4);
        for (int kt = 0; kt < T; kt++, ring_next(rp, nst)) {
            const int s = rp.s;
            mbar_wait(&full[s], rp.ph, p.err);
            const int cl = kt * GV_TC + (lane & 15);
            if (cl < nc)
                stage_chunk<FMT, M>(stages_a + static_cast<uint32_t>(s) * GV_STAGE_BYTES, cn, xs_a, ct_a, cl, CS, acc);
            __syncwarp();
            if (lane == 0) mbar_arrive_relaxed(&empty[s]);
        }
        float res[M];
        load_residual<M>(p, rg, lane, res);
        float tot[M];
        reduce_rows16<M>(acc, lane, tot);
#pragma unroll
        for (int r = 0; r < 8; r++)
#pragma unroll
            for (int m = 0; m < M; m++) acc[r][m] = 0.0f;
        if (p.S == 1) {
            epilogue<FMT, M>(p, rg, lane, tot, rs, res, bestv, besti, true);
        } else {
            // split K: leave the partial sums; the last slice to finish a row
            // group (per half-warp) adds them in slice order and runs the epilogue
            const int r = (lane >> 1) & 7;
            const bool real = rg < p.RG;
            if ((lane & 1) == 0 && real) {
                float *dst = p.partial + ((static_cast<size_t>(slice) * p.RG + rg) * 8 + r) * M;
#pragma unroll
                for (int m = 0; m < M; m++) __stcg(dst + m, tot[m]);
            }
            fence_acq_rel_gpu();
            __syncwarp();
            uint32_t old = 0;
            if ((lane & 15) == 0 && real) old = atomicAdd(p.rg_cnt + rg, 1u);
            old = __shfl_sync(0xffffffffu, old, lane & 16);
            const bool last = real && old == static_cast<uint32_t>(p.S - 1);
            float sum[M];
#pragma unroll
            for (int m = 0; m < M; m++) sum[m] = 0.0f;
            if (last) {
                fence_acq_rel_gpu();
                if ((lane & 1) == 0)
                    // batches of 8 slices' loads in flight, added in slice order
                    for (int s0 = 0; s0 < p.S; s0 += 8) {
                        float v[8][M];
#pragma unroll
                        for (int u = 0; u < 8; u++) {
                            const float *src = p.partial + ((static_cast<size_t>(s0 + u) * p.RG + rg) * 8 + r) * M;
#pragma unroll
                            for (int m = 0; m < M; m++) v[u][m] = s0 + u < p.S ? ld_cg(src + m) : 0.0f;
                        }
#pragma unroll
                        for (int u = 0; u < 8; u++)
                            if (s0 + u < p.S)
#pragma unroll
                                for (int m = 0; m < M; m++) sum[m] += v[u][m];
                    }
            }
            epilogue<FMT, M>(p, rg, lane, sum, rs, res, bestv, besti, last);
            if (last && (lane & 15) == 0) p.rg_cnt[rg] = 0u;
        }
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
        consumer_sync();
        if (ctid < M) {
            const int m = ctid;
            float v = s_bv[0][m];
            int i = s_bi[0][m];
            for (int w2 = 1; w2 < GV_CW; w2++)
                if (better(s_bv[w2][m], s_bi[w2][m], v, i)) {
                    v = s_bv[w2][m];
                    i = s_bi[w2][m];
                }
            __stcg(p.am_val + blockIdx.x * M + m, v);
            __stcg(p.am_idx + blockIdx.x * M + m, i);
        }
        __threadfence();
        consumer_sync();
        if (ctid == 0) s_last = atomicAdd(p.am_cnt, 1u) == gridDim.x - 1;
        consumer_sync();
        if (s_last) {
            __threadfence();
            for (int m = warp; m < p.M; m += GV_CW) {
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
            if (ctid == 0) *p.am_cnt = 0u;
        }
    }
}

// ------------------------------------------------------------------- host

struct GemvPlan {
    int S, CT, per_slice, grid, nst;
    size_t smem;
    size_t partial_floats;
};

static int kernel_m(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : 4; }

// Slices: minimise (rounds of items over the CTA slots) x (column tiles per
// item), with a small cost per extra slice (the partial-sum pass), subject to
// the staged activations fitting in shared memory.
static GemvPlan plan_gemv(int N, int K, int Mk, bool norm) {
    GemvPlan pl;
    const int RB = gv_row_blocks(N), KT = gv_col_tiles(K), RG = N / 8;
    const int G = sm_count() * (Mk == 1 ? gv_ctas_per_sm<1>() : gv_ctas_per_sm<2>());
    int bestS = 1, bestCT = KT;
    double best = 1e30;
    for (int S = 1; S <= min(64, KT); S++) {
        const int CT = (KT + S - 1) / S;
        if ((KT + CT - 1) / CT != S) continue;
        if (static_cast<size_t>(Mk) * CT * GV_TC * 33 * 4 + (norm ? static_cast<size_t>(CT) * GV_TC * 32 * 4 : 0) >
            gv_xs_limit(Mk))
            continue;
        const int per_slice = max(1, min(RB, G / S));
        const int rounds = (RB + per_slice - 1) / per_slice;
        // an item costs its column tiles plus its epilogue (more with split K:
        // partial sums, a fence and a counter per row group)
        const double cost = static_cast<double>(rounds) * (CT + (S > 1 ? 1.5 : 0.5));
        if (cost < best - 1e-9) {
            best = cost;
            bestS = S;
            bestCT = CT;
        }
    }
    pl.S = bestS;
    pl.CT = bestCT;
    pl.per_slice = max(1, min(RB, G / bestS));
    pl.grid = pl.S * pl.per_slice;
    pl.nst = gv_stages(Mk);
    pl.smem = static_cast<size_t>(pl.nst) * GV_STAGE_BYTES + static_cast<size_t>(Mk) * bestCT * GV_TC * 33 * 4 + 16 +
              (norm ? static_cast<size_t>(bestCT) * GV_TC * 32 * 4 : 0) + 2 * static_cast<size_t>(pl.nst) * 8;
    pl.partial_floats = pl.S > 1 ? static_cast<size_t>(pl.S) * RG * 8 * Mk : 0;
    return pl;
}

// NVFP4 with more rows than a CUDA-core pass takes goes to the tensor cores
static bool use_mma(int fmt, int M) { return fmt == BW_FMT_NVFP4 && M > GV_MAX_M; }

size_t gemv_scratch_bytes(int N, int K, int M) {
    size_t tot = M > GV_MAX_M ? mma_scratch_bytes(N, K, M) : 0;
    for (int m0 = 0; m0 < M; m0 += GV_MAX_M) {
        const int Mk = kernel_m(min(GV_MAX_M, M - m0));
        for (int norm = 0; norm < 2; norm++) {
        const GemvPlan pl = plan_gemv(N, K, Mk, norm != 0);
        size_t b = align_up(pl.partial_floats * 4, BW_WS_ALIGN) +
                   2 * align_up(static_cast<size_t>(pl.grid) * Mk * 4, BW_WS_ALIGN);
        tot = max(tot, b);
        }
    }
    return tot;
}

template <int FMT, int M>
static bw_status launch_gemv_m(const GemvParams &p0, const GemvPlan &pl, cudaStream_t st) {
    // raise the kernel's dynamic shared-memory limit to what this plan needs
    static size_t attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return BW_ERR_CUDA;
    {
        static std::mutex mu;   // host threads may call the library concurrently
        std::lock_guard<std::mutex> lk(mu);
        if (attr_set[dev] < pl.smem) {
            if (cudaFuncSetAttribute(gemv_kernel<FMT, M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(pl.smem)) != cudaSuccess) {
                (void)cudaGetLastError();
                return BW_ERR_CUDA;
            }
            attr_set[dev] = pl.smem;
        }
    }
    return launch_pdl(gemv_kernel<FMT, M>, dim3(pl.grid), dim3(GV_THREADS), pl.smem, st, p0);
}

bw_status gemv_check(int fmt, const void *wq, const void *ws_scales, int N, int K, const float *x, int M,
                     const float *gamma, const float *residual, const float *y, const int32_t *argmax_out,
                     unsigned flags, const Scratch &sc) {
    if (!wq || !ws_scales || !x || !sc.cnt || N <= 0 || K <= 0 || M <= 0) return BW_ERR_INVALID_ARG;
    if (fmt != BW_FMT_Q4_0 && fmt != BW_FMT_NVFP4) return BW_ERR_INVALID_ARG;
    if (N % 8 || K % 32) return BW_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(wq) || !aligned16(ws_scales) || !aligned16(x)) return BW_ERR_INVALID_ARG;
    if ((flags & BW_GEMV_RMSNORM) && (!gamma || !aligned16(gamma))) return BW_ERR_INVALID_ARG;
    if ((flags & BW_GEMV_RESIDUAL) && !residual) return BW_ERR_INVALID_ARG;
    if ((flags & BW_GEMV_ARGMAX) && !argmax_out) return BW_ERR_INVALID_ARG;
    if ((flags & BW_GEMV_SILU_GATE) && (flags & (BW_GEMV_RESIDUAL | BW_GEMV_ARGMAX)))
        return BW_ERR_INVALID_ARG;
    if (!(flags & BW_GEMV_ARGMAX) && !y) return BW_ERR_INVALID_ARG;
    if (sc.bytes < gemv_scratch_bytes(N, K, M)) return BW_ERR_INVALID_ARG;
    if (use_mma(fmt, M)) return mma_check(N, K, M);
    for (int m0 = 0; m0 < M; m0 += GV_MAX_M) {
        const GemvPlan pl = plan_gemv(N, K, kernel_m(min(GV_MAX_M, M - m0)), (flags & BW_GEMV_RMSNORM) != 0);
        if (pl.smem > GV_SMEM_LIMIT) return BW_ERR_UNSUPPORTED_SHAPE;
        if (pl.S > 1 && N / 8 + CNT_GEMV_RG > CNT_ATTN) return BW_ERR_UNSUPPORTED_SHAPE;
    }
    return BW_OK;
}

bw_status gemv_launch(int fmt, const void *wq, const void *ws_scales, float ts, float ts_up, int N,
                      int K, const float *x, int M, const float *gamma, float eps,
                      const float *residual, float *y, int32_t *argmax_out, unsigned flags,
                      const Scratch &sc, cudaStream_t st, int32_t *adv_tokens, int32_t *adv_pos) {
    const bw_status chk = gemv_check(fmt, wq, ws_scales, N, K, x, M, gamma, residual, y, argmax_out, flags, sc);
    if (chk != BW_OK) return chk;
    if (use_mma(fmt, M))
        return mma_gemm_launch(wq, ws_scales, ts, ts_up, N, K, x, M, gamma, eps, residual, y, argmax_out, flags, sc,
                               st, adv_tokens, adv_pos);
    const int ncols = (flags & BW_GEMV_SILU_GATE) ? N / 2 : N;
    for (int m0 = 0; m0 < M; m0 += GV_MAX_M) {
        const int Mr = min(GV_MAX_M, M - m0);
        const int Mk = kernel_m(Mr);
        const GemvPlan pl = plan_gemv(N, K, Mk, (flags & BW_GEMV_RMSNORM) != 0);
        Carver cv(sc.base);
        GemvParams p;
        p.q = static_cast<const uint8_t *>(wq);
        p.s = static_cast<const uint8_t *>(ws_scales);
        p.N = N;
        p.K = K;
        p.M = Mr;
        p.NC = K / 32;
        p.RG = N / 8;
        p.RB = gv_row_blocks(N);
        p.KT = gv_col_tiles(K);
        p.S = pl.S;
        p.CT = pl.CT;
        p.per_slice = pl.per_slice;
        p.nst = pl.nst;
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
        p.err = sc.err;
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
    if (!bw::ws_ok(ws)) return BW_ERR_INVALID_ARG;
    return bw::gemv_launch(BW_FMT_Q4_0, w_q, w_d, 1.0f, 1.0f, N, K, x, M, gamma, eps, residual, y,
                           argmax_out, flags, bw::scratch_of(ws, ws_bytes),
                           static_cast<cudaStream_t>(stream));
}

bw_status bw_gemv_nvfp4(const void *w_q, const void *w_s, float ts, float ts_up, int N, int K,
                        const float *x, int M, const float *gamma, float eps,
                        const float *residual, float *y, int32_t *argmax_out, unsigned flags,
                        void *ws, size_t ws_bytes, void *stream) {
    if (!bw::ws_ok(ws)) return BW_ERR_INVALID_ARG;
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
