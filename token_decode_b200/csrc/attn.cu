// attn.cu -- paged fp16-KV GQA decode attention with fused RoPE and KV write
// (sm_100a).
//
// One CTA per (split, kv head, sequence).  The split owns a contiguous range
// of whole pages of the sequence's logical positions (split-KV, so a batch-1
// step still fills every SM); it
//   1. ropes the G = nq/nkv query heads of its kv head for each of the n_rows
//      query rows (positions pos..pos+n_rows-1),
//   2. if one of those positions falls in its range, ropes that row's k,
//      rounds k and v to fp16 and writes them into the paged pool (the
//      deep-dive page, section 6: positions map to physical pages through
//      the page table; section 5, stage 4: the K draft rows of a verify pass
//      share one cache, causally masked),
//   3. streams its pages through shared memory in 32-token tiles (cp.async,
//      double-buffered) with an online softmax in fp32,
//   4. leaves (max, sum, unnormalised output) per query in the workspace; the
//      last CTA of the (sequence, kv head) -- atomic counter, no waiting --
//      combines the splits in split order, so results are deterministic and
//      independent of the physical page order.
// The K tile is stored with its 16-byte granules XOR-swizzled by token so the
// lane-per-token score loop reads shared memory without bank conflicts.
#include <math.h>

#include "bw_common.cuh"

namespace bw {

constexpr int ATT_THREADS = 128;
constexpr int ATT_WARPS = ATT_THREADS / 32;
constexpr int ATT_TT = 32;          // tokens per tile (two pages)
constexpr int ATT_MAXQ = 32;        // query vectors per CTA (G * n_rows)

struct AttnParams {
    const float *qkv;
    const float *rope_cos, *rope_sin;
    int rope_max_pos;
    __half *k_pool, *v_pool;
    const int32_t *page_table;
    int max_pages, n_pages;
    const int32_t *pos;
    int B, R, nq, nkv, G, Q, n_split;
    float scale;
    float *out;
    float *part_m, *part_l, *part_o;   // [B][nkv][n_split][Q] (+ [hd])
    uint32_t *cnt;                     // [B][nkv]
    uint32_t *err;
};

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// rotate-half RoPE of one pair, rounding each product like the plain formula
__device__ __forceinline__ void rope_pair(float a, float b, float c, float s, float &ra, float &rb) {
    ra = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
    rb = __fadd_rn(__fmul_rn(b, c), __fmul_rn(a, s));
}

template <int HD, int QMAX>
__global__ void __launch_bounds__(ATT_THREADS) attn_kernel(const AttnParams p) {
    constexpr int NG = HD / 8;   // 16-byte granules per row
    extern __shared__ float4 att_smem[];
    __half (*sk)[ATT_TT * HD] = reinterpret_cast<__half (*)[ATT_TT * HD]>(att_smem);
    __half (*sv)[ATT_TT * HD] = reinterpret_cast<__half (*)[ATT_TT * HD]>(sk + 2);
    float *sq = reinterpret_cast<float *>(sv + 2);                       // [QMAX][HD]
    float (*sp)[ATT_TT] = reinterpret_cast<float (*)[ATT_TT]>(sq + QMAX * HD);  // [QMAX][TT]
    __shared__ float s_m[ATT_MAXQ], s_l[ATT_MAXQ], s_corr[ATT_MAXQ];
    __shared__ int s_page[2][ATT_TT / 16];
    __shared__ bool s_last;

    pdl_trigger();
    const int sp_idx = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_wait();

    const int p0 = p.pos[b];
    int len = p0 + p.R;
    if (p0 < 0 || len > p.max_pages * 16 || len > p.rope_max_pos) {
        if (tid == 0) set_error(p.err, BW_DEVERR_BAD_POS);
        len = max(0, min(len, min(p.max_pages * 16, p.rope_max_pos)));
    }
    const int n_pg = (len + 15) / 16;
    const int pps = (n_pg + p.n_split - 1) / p.n_split;
    const int pg0 = min(n_pg, sp_idx * pps), pg1 = min(n_pg, pg0 + pps);
    const int t0 = pg0 * 16, t1 = min(len, pg1 * 16);
    const int32_t *pt = p.page_table + static_cast<size_t>(b) * p.max_pages;
    const size_t row_stride = static_cast<size_t>(p.nq + 2 * p.nkv) * HD;

    // ---- 1. roped, unscaled queries into shared memory
    for (int i = tid; i < p.Q * (HD / 2); i += ATT_THREADS) {
        const int qi = i / (HD / 2), d = i - qi * (HD / 2);
        const int r = qi / p.G, g = qi - r * p.G;
        const int h = kvh * p.G + g;
        const int ppos = max(0, min(p0 + r, p.rope_max_pos - 1));
        const float *src = p.qkv + (static_cast<size_t>(b) * p.R + r) * row_stride + static_cast<size_t>(h) * HD;
        const float c = p.rope_cos[static_cast<size_t>(ppos) * (HD / 2) + d];
        const float s = p.rope_sin[static_cast<size_t>(ppos) * (HD / 2) + d];
        float ra, rb;
        rope_pair(src[d], src[d + HD / 2], c, s, ra, rb);
        sq[qi * HD + d] = ra;
        sq[qi * HD + d + HD / 2] = rb;
    }
    if (tid < ATT_MAXQ) {
        s_m[tid] = -INFINITY;
        s_l[tid] = 0.0f;
    }

    // ---- 2. the new rows' k (roped) and v, rounded to fp16, into the pool
    for (int r = 0; r < p.R; r++) {
        const int ppos = p0 + r;
        if (ppos < t0 || ppos >= t1) continue;   // t1 <= max_pages * 16
        const int page = pt[ppos / 16];
        if (page < 0 || page >= p.n_pages) {
            if (tid == 0) set_error(p.err, BW_DEVERR_BAD_PAGE);
            continue;
        }
        const size_t off = ((static_cast<size_t>(page) * p.nkv + kvh) * 16 + (ppos & 15)) * HD;
        const float *krow = p.qkv + (static_cast<size_t>(b) * p.R + r) * row_stride +
                            static_cast<size_t>(p.nq + kvh) * HD;
        const float *vrow = krow + static_cast<size_t>(p.nkv) * HD;
        const int rp = ppos;
        for (int d = tid; d < HD / 2; d += ATT_THREADS) {
            const float c = p.rope_cos[static_cast<size_t>(rp) * (HD / 2) + d];
            const float s = p.rope_sin[static_cast<size_t>(rp) * (HD / 2) + d];
            float ra, rb;
            rope_pair(krow[d], krow[d + HD / 2], c, s, ra, rb);
            p.k_pool[off + d] = __float2half_rn(ra);
            p.k_pool[off + d + HD / 2] = __float2half_rn(rb);
        }
        for (int d = tid; d < HD; d += ATT_THREADS) p.v_pool[off + d] = __float2half_rn(vrow[d]);
    }
    __syncthreads();

    // ---- 3. tiles of 32 tokens: scores, online softmax, P.V
    const int n_tiles = (t1 - t0 + ATT_TT - 1) / ATT_TT;
    auto issue_tile = [&](int tile, int buf) {
        const int tb = t0 + tile * ATT_TT;
        if (tid < ATT_TT / 16) {
            const int lp = tb / 16 + tid;
            int page = -1;
            if (lp * 16 < t1) {
                page = pt[lp];
                if (page < 0 || page >= p.n_pages) {
                    set_error(p.err, BW_DEVERR_BAD_PAGE);
                    page = -1;
                }
            }
            s_page[buf][tid] = page;
        }
        __syncthreads();
        for (int i = tid; i < ATT_TT * NG; i += ATT_THREADS) {
            const int t = i / NG, g = i - t * NG;
            const int page = s_page[buf][t / 16];
            if (page < 0) continue;
            const size_t off = ((static_cast<size_t>(page) * p.nkv + kvh) * 16 + (t & 15)) * HD + g * 8;
            cp_async16(&sk[buf][t * HD + 8 * (g ^ (t & 7))], p.k_pool + off);
            cp_async16(&sv[buf][t * HD + 8 * g], p.v_pool + off);
        }
        cp_async_commit();
    };

    // thread -> output dims: HD == 128: one dim per thread for every query;
    // HD == 64: dim tid % 64 for the queries of parity tid / 64
    constexpr int QSTEP = ATT_THREADS / HD;            // 1 or 2
    constexpr int NACC = QMAX / QSTEP;
    float acc[NACC];
#pragma unroll
    for (int i = 0; i < NACC; i++) acc[i] = 0.0f;
    const int od = tid % HD, oq0 = tid / HD;

    if (n_tiles > 0) issue_tile(0, 0);
    for (int tile = 0; tile < n_tiles; tile++) {
        const int buf = tile & 1;
        if (tile + 1 < n_tiles) {
            issue_tile(tile + 1, buf ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const int tb = t0 + tile * ATT_TT;
        // scores: lane = token, warp strides over queries
        {
            const int t = lane;
            const int tpos = tb + t;
            const bool tok_ok = tpos < t1 && s_page[buf][t / 16] >= 0;
            uint4 kr[NG];
            if (tok_ok) {
#pragma unroll
                for (int g = 0; g < NG; g++)
                    kr[g] = *reinterpret_cast<const uint4 *>(&sk[buf][t * HD + 8 * (g ^ (t & 7))]);
            }
            for (int qi = warp; qi < p.Q; qi += ATT_WARPS) {
                const int r = qi / p.G;
                float s = -INFINITY;
                if (tok_ok && tpos <= p0 + r) {
                    float dot = 0.0f;
#pragma unroll
                    for (int g = 0; g < NG; g++) {
                        const float4 qa = *reinterpret_cast<const float4 *>(&sq[qi * HD + 8 * g]);
                        const float4 qb = *reinterpret_cast<const float4 *>(&sq[qi * HD + 8 * g + 4]);
                        const float2 k0 = __half22float2(*reinterpret_cast<const __half2 *>(&kr[g].x));
                        const float2 k1 = __half22float2(*reinterpret_cast<const __half2 *>(&kr[g].y));
                        const float2 k2 = __half22float2(*reinterpret_cast<const __half2 *>(&kr[g].z));
                        const float2 k3 = __half22float2(*reinterpret_cast<const __half2 *>(&kr[g].w));
                        dot = fmaf(qa.x, k0.x, dot);
                        dot = fmaf(qa.y, k0.y, dot);
                        dot = fmaf(qa.z, k1.x, dot);
                        dot = fmaf(qa.w, k1.y, dot);
                        dot = fmaf(qb.x, k2.x, dot);
                        dot = fmaf(qb.y, k2.y, dot);
                        dot = fmaf(qb.z, k3.x, dot);
                        dot = fmaf(qb.w, k3.y, dot);
                    }
                    s = dot * p.scale;
                }
                // online softmax update of this query (one warp owns it)
                const float m_old = s_m[qi];
                const float m_new = fmaxf(m_old, warp_max(s));
                const float pr = (s == -INFINITY) ? 0.0f : expf(s - m_new);
                const float lsum = warp_sum(pr);
                sp[qi][t] = pr;
                if (lane == 0) {
                    const float corr = (m_old == -INFINITY) ? 0.0f : expf(m_old - m_new);
                    s_corr[qi] = corr;
                    s_l[qi] = s_l[qi] * corr + lsum;
                    s_m[qi] = m_new;
                }
            }
        }
        __syncthreads();
        // P.V: thread owns dim od for queries oq0, oq0 + QSTEP, ...
#pragma unroll
        for (int i = 0; i < NACC; i++) {
            const int qi = oq0 + i * QSTEP;
            if (qi < p.Q) acc[i] *= s_corr[qi];
        }
        {
            const int nt = min(ATT_TT, t1 - tb);
            for (int pg = 0; pg < ATT_TT / 16; pg++) {
                if (s_page[buf][pg] < 0) continue;
                const int te = min(nt, pg * 16 + 16);
                for (int t = pg * 16; t < te; t++) {
                    const float v = __half2float(sv[buf][t * HD + od]);
#pragma unroll
                    for (int i = 0; i < NACC; i++) {
                        const int qi = oq0 + i * QSTEP;
                        if (qi < p.Q) acc[i] = fmaf(sp[qi][t], v, acc[i]);
                    }
                }
            }
        }
        __syncthreads();
    }

    // ---- 4. partial results, then the last CTA combines the splits
    const size_t grp = static_cast<size_t>(b) * p.nkv + kvh;
    if (p.n_split == 1) {
#pragma unroll
        for (int i = 0; i < NACC; i++) {
            const int qi = oq0 + i * QSTEP;
            if (qi < p.Q) {
                const int r = qi / p.G, g = qi - r * p.G;
                const float l = s_l[qi];
                p.out[(static_cast<size_t>(b) * p.R + r) * (static_cast<size_t>(p.nq) * HD) +
                      static_cast<size_t>(kvh * p.G + g) * HD + od] = acc[i] / l;
            }
        }
        return;
    }
    const size_t pbase = (grp * p.n_split + sp_idx) * p.Q;
#pragma unroll
    for (int i = 0; i < NACC; i++) {
        const int qi = oq0 + i * QSTEP;
        if (qi < p.Q) __stcg(p.part_o + (pbase + qi) * HD + od, acc[i]);
    }
    if (tid < p.Q) {
        __stcg(p.part_m + pbase + tid, s_m[tid]);
        __stcg(p.part_l + pbase + tid, s_l[tid]);
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(p.cnt + grp, 1u) == static_cast<uint32_t>(p.n_split - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // combine the splits: gather every split's (max, sum) into shared memory
    // (the K/V tile buffers are free now), then one coefficient per (split,
    // query), then each thread sums its output dim over the splits in order.
    const int nsq = p.n_split * p.Q;
    float *cm = reinterpret_cast<float *>(att_smem);      // [n_split][Q] maxima -> coefficients
    float *cl = cm + nsq;                                  // [n_split][Q] sums
    const size_t gbase = grp * p.n_split * p.Q;
    for (int i = tid; i < nsq; i += ATT_THREADS) {
        cm[i] = ld_cg(p.part_m + gbase + i);
        cl[i] = ld_cg(p.part_l + gbase + i);
    }
    __syncthreads();
    if (tid < p.Q) {
        float M = -INFINITY;
        for (int s2 = 0; s2 < p.n_split; s2++) M = fmaxf(M, cm[s2 * p.Q + tid]);
        float L = 0.0f;
        for (int s2 = 0; s2 < p.n_split; s2++) {
            const float ms = cm[s2 * p.Q + tid];
            const float w = (ms == -INFINITY) ? 0.0f : expf(ms - M);
            L = fmaf(cl[s2 * p.Q + tid], w, L);
            cm[s2 * p.Q + tid] = w;
        }
        s_l[tid] = L;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < NACC; i++) {
        const int qi = oq0 + i * QSTEP;
        if (qi >= p.Q) continue;
        float O = 0.0f;
        const float *po = p.part_o + (gbase + qi) * HD + od;
        const size_t sstride = static_cast<size_t>(p.Q) * HD;
#pragma unroll 8
        for (int s2 = 0; s2 < p.n_split; s2++) O = fmaf(ld_cg(po + s2 * sstride), cm[s2 * p.Q + qi], O);
        const int r = qi / p.G, g = qi - r * p.G;
        p.out[(static_cast<size_t>(b) * p.R + r) * (static_cast<size_t>(p.nq) * HD) +
              static_cast<size_t>(kvh * p.G + g) * HD + od] = O / s_l[qi];
    }
    if (tid == 0) p.cnt[grp] = 0u;
}

template <int HD, int QMAX>
static bw_status attn_go(dim3 grid, cudaStream_t st, const AttnParams &p) {
    const size_t smem = 4u * ATT_TT * HD * sizeof(__half) + static_cast<size_t>(QMAX) * HD * 4 +
                        static_cast<size_t>(QMAX) * ATT_TT * 4;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return BW_ERR_CUDA;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(attn_kernel<HD, QMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return BW_ERR_CUDA;
        attr_set[dev] = true;
    }
    return launch_pdl(attn_kernel<HD, QMAX>, grid, dim3(ATT_THREADS), smem, st, p);
}

// Splits per (sequence, kv head): enough CTAs to cover every SM about once,
// at least ~4 pages per split, at most 64 splits (the combine keeps
// n_split * 32 floats of statistics in shared memory).
static int attn_splits(int B, int nkv, int max_pages) {
    const int groups = B * nkv;
    int ns = (sm_count() + groups - 1) / groups;
    ns = max(1, min(ns, (max_pages + 3) / 4));
    ns = min(ns, 64);
    return ns;
}

size_t attn_scratch_bytes(int B, int R, int nq, int nkv, int hd, int max_pages) {
    const int ns = attn_splits(B, nkv, max_pages);
    const size_t Q = static_cast<size_t>(nq / nkv) * R;
    const size_t n = static_cast<size_t>(B) * nkv * ns * Q;
    return 2 * align_up(n * 4, BW_WS_ALIGN) + align_up(n * hd * 4, BW_WS_ALIGN);
}

bw_status attn_launch(const float *qkv, const float *rope_cos, const float *rope_sin, int rope_max_pos,
                      void *k_pool, void *v_pool, const int32_t *page_table, int max_pages,
                      int n_pages, const int32_t *pos, int B, int R, int nq, int nkv, int hd,
                      float *out, const Scratch &sc, cudaStream_t st) {
    if (!qkv || !rope_cos || !rope_sin || !k_pool || !v_pool || !page_table || !pos || !out || !sc.cnt)
        return BW_ERR_INVALID_ARG;
    if (B <= 0 || R <= 0 || nq <= 0 || nkv <= 0 || max_pages <= 0 || n_pages <= 0 || rope_max_pos <= 0)
        return BW_ERR_INVALID_ARG;
    if ((hd != 128 && hd != 64) || nq % nkv || (nq / nkv) * R > ATT_MAXQ) return BW_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(k_pool) || !aligned16(v_pool) || !aligned16(qkv)) return BW_ERR_INVALID_ARG;
    if (B * nkv + CNT_ATTN > BW_WS_COUNTERS) return BW_ERR_UNSUPPORTED_SHAPE;
    if (sc.bytes < attn_scratch_bytes(B, R, nq, nkv, hd, max_pages)) return BW_ERR_INVALID_ARG;
    AttnParams p;
    p.qkv = qkv;
    p.rope_cos = rope_cos;
    p.rope_sin = rope_sin;
    p.rope_max_pos = rope_max_pos;
    p.k_pool = static_cast<__half *>(k_pool);
    p.v_pool = static_cast<__half *>(v_pool);
    p.page_table = page_table;
    p.max_pages = max_pages;
    p.n_pages = n_pages;
    p.pos = pos;
    p.B = B;
    p.R = R;
    p.nq = nq;
    p.nkv = nkv;
    p.G = nq / nkv;
    p.Q = p.G * R;
    p.n_split = attn_splits(B, nkv, max_pages);
    p.scale = 1.0f / sqrtf(static_cast<float>(hd));
    p.out = out;
    const size_t n = static_cast<size_t>(B) * nkv * p.n_split * p.Q;
    Carver cv(sc.base);
    p.part_m = cv.take<float>(n);
    p.part_l = cv.take<float>(n);
    p.part_o = cv.take<float>(n * hd);
    p.cnt = sc.cnt + CNT_ATTN;
    p.err = sc.err;
    dim3 grid(p.n_split, nkv, B);
    if (hd == 128) {
        if (p.Q <= 4) return attn_go<128, 4>(grid, st, p);
        if (p.Q <= 8) return attn_go<128, 8>(grid, st, p);
        if (p.Q <= 16) return attn_go<128, 16>(grid, st, p);
        return attn_go<128, 32>(grid, st, p);
    }
    if (p.Q <= 8) return attn_go<64, 8>(grid, st, p);
    return attn_go<64, 32>(grid, st, p);
}

}  // namespace bw

extern "C" {

bw_status bw_paged_attn_decode(const float *qkv, const float *rope_cos, const float *rope_sin,
                               int rope_max_pos, void *k_pool, void *v_pool,
                               const int32_t *page_table, int max_pages, int n_pages,
                               const int32_t *pos, int B, int n_rows, int nq, int nkv, int hd,
                               float *out, void *ws, size_t ws_bytes, void *stream) {
    if (!ws) return BW_ERR_INVALID_ARG;
    return bw::attn_launch(qkv, rope_cos, rope_sin, rope_max_pos, k_pool, v_pool, page_table,
                           max_pages, n_pages, pos, B, n_rows, nq, nkv, hd, out,
                           bw::scratch_of(ws, ws_bytes), static_cast<cudaStream_t>(stream));
}

size_t bw_attn_workspace_bytes(int B, int n_rows, int nq, int nkv, int hd, int max_pages) {
    if (B <= 0 || n_rows <= 0 || nq <= 0 || nkv <= 0 || hd <= 0 || max_pages <= 0 || nq % nkv)
        return BW_WS_HDR_BYTES;
    return BW_WS_HDR_BYTES + bw::attn_scratch_bytes(B, n_rows, nq, nkv, hd, max_pages);
}

}  // extern "C"
