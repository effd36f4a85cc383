// attn.cu -- paged fp16-KV GQA decode attention with fused RoPE and KV write
// (sm_100a).
//
// One CTA per (split, kv head, sequence); the splits of one (sequence, kv
// head) form a thread-block cluster.  Each CTA
//   1. ropes the G = nq/nkv query heads of its kv head for each of the n_rows
//      query rows (positions pos..pos+n_rows-1),
//   2. ropes the new rows' k, rounds k and v to fp16 and writes them into the
//      paged pool when their position falls in its page range (the deep-dive
//      page, section 6: logical positions map to physical pages through the
//      page table; section 5, stage 4: the draft rows of a verify pass share
//      one cache, causally masked),
//   3. streams its pages into a ring of shared-memory stages with 1-D bulk
//      copies (cp.async.bulk, completion on an mbarrier; two pages = 32
//      tokens per stage) and runs an fp32 online softmax over them,
//   4. combines the splits through distributed shared memory: after a
//      cluster barrier every CTA reads the others' (max, sum, partial output)
//      and writes a slice of the final output, in split order, so results are
//      deterministic and independent of the physical page order.
// K rows are read with a per-lane rotation of their 16-byte granules (lane t
// starts at granule t), which keeps the linear bulk-copied layout free of
// shared-memory bank conflicts; the query is stored split in two float4
// planes so its rotated reads are conflict-free too.
#include <cooperative_groups.h>
#include <math.h>

#include "bw_common.cuh"

namespace cg = cooperative_groups;

namespace bw {

constexpr int ATT_THREADS = 256;
constexpr int ATT_WARPS = ATT_THREADS / 32;
constexpr int ATT_TT = 32;          // tokens per stage (two pages)
constexpr int ATT_MAXQ = 32;        // query vectors per CTA (G * n_rows)
constexpr int ATT_MAXR = 8;         // query rows per sequence (1 + draft tokens)
constexpr int ATT_MAXNS = 16;       // splits (cluster size) per (sequence, kv head)

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
    uint32_t *err;
};

template <int HD>
__host__ __device__ constexpr int att_stages() { return HD == 128 ? 4 : 6; }

template <int HD, int QMAX>
constexpr size_t att_smem_bytes() {
    return static_cast<size_t>(att_stages<HD>()) * 2 * ATT_TT * HD * 2   // K/V ring (fp16)
           + static_cast<size_t>(QMAX) * HD * 4                          // query planes (fp32)
           + static_cast<size_t>(QMAX) * ATT_TT * 4                      // probabilities
           + 2 * static_cast<size_t>(ATT_MAXR) * HD * 2                  // new k, v rows (fp16)
           + static_cast<size_t>(att_stages<HD>()) * 8;                  // mbarriers
}

// rotate-half RoPE of one pair, rounding each product like the plain formula
__device__ __forceinline__ void rope_pair(float a, float b, float c, float s, float &ra, float &rb) {
    ra = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
    rb = __fadd_rn(__fmul_rn(b, c), __fmul_rn(a, s));
}

__device__ __forceinline__ float dot8(const float4 lo, const float4 hi, const uint4 k) {
    const float2 k0 = __half22float2(*reinterpret_cast<const __half2 *>(&k.x));
    const float2 k1 = __half22float2(*reinterpret_cast<const __half2 *>(&k.y));
    const float2 k2 = __half22float2(*reinterpret_cast<const __half2 *>(&k.z));
    const float2 k3 = __half22float2(*reinterpret_cast<const __half2 *>(&k.w));
    float d = lo.x * k0.x;
    d = fmaf(lo.y, k0.y, d);
    d = fmaf(lo.z, k1.x, d);
    d = fmaf(lo.w, k1.y, d);
    d = fmaf(hi.x, k2.x, d);
    d = fmaf(hi.y, k2.y, d);
    d = fmaf(hi.z, k3.x, d);
    d = fmaf(hi.w, k3.y, d);
    return d;
}

template <int HD, int QMAX>
__global__ void __launch_bounds__(ATT_THREADS) attn_kernel(const AttnParams p) {
    constexpr int NG = HD / 8;              // 16-byte granules per K/V row
    constexpr int NST = att_stages<HD>();
    constexpr int SH = ATT_TT * HD;         // halves per K (or V) stage
    constexpr int TG = ATT_THREADS / HD;    // P.V token groups: 2 (HD 128) or 4 (HD 64)
    constexpr int TPG = ATT_TT / TG;        // tokens per group and stage (16 or 8)
    constexpr int NACC = QMAX;
    constexpr int QPW = (QMAX + ATT_WARPS - 1) / ATT_WARPS;   // queries owned per warp
    extern __shared__ __align__(128) unsigned char att_sm[];
    __half *ring = reinterpret_cast<__half *>(att_sm);                       // [NST][K|V][SH]
    float4 *q_lo = reinterpret_cast<float4 *>(ring + static_cast<size_t>(NST) * 2 * SH);  // [QMAX][NG]
    float4 *q_hi = q_lo + QMAX * NG;                                        // [QMAX][NG]
    float *P = reinterpret_cast<float *>(q_hi + QMAX * NG);                 // [QMAX][TT]
    __half *newk = reinterpret_cast<__half *>(P + QMAX * ATT_TT);           // [MAXR][HD]
    __half *newv = newk + ATT_MAXR * HD;
    uint64_t *bar = reinterpret_cast<uint64_t *>(newv + ATT_MAXR * HD);     // [NST]
    __shared__ float s_m[ATT_MAXQ], s_l[ATT_MAXQ], s_corr[ATT_MAXQ];
    __shared__ int s_page[NST][2];

    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_trigger();
    if (tid == 0) {
        for (int s = 0; s < NST; s++) mbar_init(&bar[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();

    const int p0 = p.pos[b];
    int len = p0 + p.R;
    if (p0 < 0 || len > p.max_pages * 16 || len > p.rope_max_pos) {
        if (tid == 0) set_error(p.err, BW_DEVERR_BAD_POS);
        len = max(0, min(len, min(p.max_pages * 16, p.rope_max_pos)));
    }
    const int n_pg = (len + 15) / 16;
    const int pps = (n_pg + p.n_split - 1) / p.n_split;
    const int pg0 = min(n_pg, split * pps), pg1 = min(n_pg, pg0 + pps);
    const int t1 = min(len, pg1 * 16);
    const int n_tiles = (pg1 - pg0 + 1) / 2;
    const int32_t *pt = p.page_table + static_cast<size_t>(b) * p.max_pages;
    const size_t row_stride = static_cast<size_t>(p.nq + 2 * p.nkv) * HD;
    constexpr uint32_t PAGE_BYTES = 16 * HD * 2;

    // one thread streams pages: expect the bytes, then issue the bulk copies
    auto issue = [&](int tile) {
        const int st = tile % NST;
        int pages[2];
        uint32_t bytes = 0;
        for (int j = 0; j < 2; j++) {
            const int lp = pg0 + 2 * tile + j;
            int page = -1;
            if (lp < pg1) {
                page = pt[lp];
                if (page < 0 || page >= p.n_pages) {
                    set_error(p.err, BW_DEVERR_BAD_PAGE);
                    page = -1;
                }
            }
            pages[j] = page;
            s_page[st][j] = page;
            if (page >= 0) bytes += 2 * PAGE_BYTES;
        }
        mbar_arrive_tx(&bar[st], bytes);
        __half *sk = ring + static_cast<size_t>(st) * 2 * SH;
        for (int j = 0; j < 2; j++) {
            if (pages[j] < 0) continue;
            const size_t off = (static_cast<size_t>(pages[j]) * p.nkv + kvh) * 16 * HD;
            bulk_g2s(sk + j * 16 * HD, p.k_pool + off, PAGE_BYTES, &bar[st]);
            bulk_g2s(sk + SH + j * 16 * HD, p.v_pool + off, PAGE_BYTES, &bar[st]);
        }
    };
    if (tid == 0)
        for (int t = 0; t < min(NST, n_tiles); t++) issue(t);

    // ---- 1. roped queries, split into two float4 planes per 8-dim granule
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
        float *lo = reinterpret_cast<float *>(q_lo + qi * NG);
        float *hi = reinterpret_cast<float *>(q_hi + qi * NG);
        const int da = d, db = d + HD / 2;
        ((da & 7) < 4 ? lo : hi)[(da >> 3) * 4 + (da & 3)] = ra;
        ((db & 7) < 4 ? lo : hi)[(db >> 3) * 4 + (db & 3)] = rb;
    }

    // ---- 2. the new rows' k (roped) and v, rounded to fp16: kept for this
    //         CTA's stages and written into the pool
    for (int r = 0; r < p.R; r++) {
        const int ppos = p0 + r;
        if (ppos < pg0 * 16 || ppos >= t1) continue;
        const int page = pt[ppos / 16];
        const bool ok = page >= 0 && page < p.n_pages;
        if (!ok && tid == 0) set_error(p.err, BW_DEVERR_BAD_PAGE);
        const size_t off = ((static_cast<size_t>(ok ? page : 0) * p.nkv + kvh) * 16 + (ppos & 15)) * HD;
        const float *krow = p.qkv + (static_cast<size_t>(b) * p.R + r) * row_stride +
                            static_cast<size_t>(p.nq + kvh) * HD;
        const float *vrow = krow + static_cast<size_t>(p.nkv) * HD;
        for (int d = tid; d < HD / 2; d += ATT_THREADS) {
            const float c = p.rope_cos[static_cast<size_t>(ppos) * (HD / 2) + d];
            const float s = p.rope_sin[static_cast<size_t>(ppos) * (HD / 2) + d];
            float ra, rb;
            rope_pair(krow[d], krow[d + HD / 2], c, s, ra, rb);
            const __half ha = __float2half_rn(ra), hb = __float2half_rn(rb);
            newk[r * HD + d] = ha;
            newk[r * HD + d + HD / 2] = hb;
            if (ok) {
                p.k_pool[off + d] = ha;
                p.k_pool[off + d + HD / 2] = hb;
            }
        }
        for (int d = tid; d < HD; d += ATT_THREADS) {
            const __half hv = __float2half_rn(vrow[d]);
            newv[r * HD + d] = hv;
            if (ok) p.v_pool[off + d] = hv;
        }
    }
    __syncthreads();

    // ---- 3. stages of 32 tokens: scores, online softmax, P.V
    float m_run[QPW], l_run[QPW];
#pragma unroll
    for (int j = 0; j < QPW; j++) {
        m_run[j] = -INFINITY;
        l_run[j] = 0.0f;
    }
    float acc[NACC];
#pragma unroll
    for (int i = 0; i < NACC; i++) acc[i] = 0.0f;
    const int od = tid % HD, tq = tid / HD;   // output dim, token group

    for (int tile = 0; tile < n_tiles; tile++) {
        const int st = tile % NST;
        mbar_wait(&bar[st], static_cast<uint32_t>((tile / NST) & 1), p.err);
        __half *sk = ring + static_cast<size_t>(st) * 2 * SH;
        __half *sv = sk + SH;
        const int tb = (pg0 + 2 * tile) * 16;
        // the rows written by this step replace what the copy brought
        for (int r = 0; r < p.R; r++) {
            const int slot = p0 + r - tb;
            if (slot < 0 || slot >= ATT_TT || p0 + r >= t1 || s_page[st][slot >> 4] < 0) continue;
            for (int d = tid; d < HD; d += ATT_THREADS) {
                sk[slot * HD + d] = newk[r * HD + d];
                sv[slot * HD + d] = newv[r * HD + d];
            }
        }
        __syncthreads();
        // scores: lane = token, warp w owns queries w, w + 4, ...
        {
            const int t = lane;
            const int tpos = tb + t;
            const bool tok_ok = tpos < t1 && s_page[st][t >> 4] >= 0;
            uint4 kr[NG];
#pragma unroll
            for (int g = 0; g < NG; g++) {
                const int g2 = (g + t) & (NG - 1);
                kr[g] = *reinterpret_cast<const uint4 *>(sk + t * HD + g2 * 8);
            }
#pragma unroll
            for (int j = 0; j < QPW; j++) {
                const int qi = warp + ATT_WARPS * j;
                if (qi >= p.Q) break;
                const int r = qi / p.G;
                float s = -INFINITY;
                if (tok_ok && tpos <= p0 + r) {
                    float dot = 0.0f;
#pragma unroll
                    for (int g = 0; g < NG; g++) {
                        const int g2 = (g + t) & (NG - 1);
                        dot += dot8(q_lo[qi * NG + g2], q_hi[qi * NG + g2], kr[g]);
                    }
                    s = dot * p.scale;
                }
                const float m_new = fmaxf(m_run[j], warp_max(s));
                const float pr = (s == -INFINITY) ? 0.0f : expf(s - m_new);
                const float lsum = warp_sum(pr);
                const float corr = (m_run[j] == -INFINITY) ? 0.0f : expf(m_run[j] - m_new);
                l_run[j] = l_run[j] * corr + lsum;
                m_run[j] = m_new;
                P[qi * ATT_TT + t] = pr;
                if (lane == 0) s_corr[qi] = corr;
            }
        }
        __syncthreads();
        // P.V: thread (od, tq) sums tokens [tq*TPG, tq*TPG + TPG) of the stage
#pragma unroll
        for (int i = 0; i < NACC; i++)
            if (i < p.Q) acc[i] *= s_corr[i];
        {
            const int nt = min(ATT_TT, t1 - tb);
            const int ta = tq * TPG;
            const int te = min(nt, ta + TPG);
            if (ta < te && s_page[st][ta >> 4] >= 0) {
                for (int t4 = ta; t4 < te; t4 += 4) {
                    float v[4];
#pragma unroll
                    for (int u = 0; u < 4; u++)
                        v[u] = (t4 + u < te) ? __half2float(sv[(t4 + u) * HD + od]) : 0.0f;
#pragma unroll
                    for (int i = 0; i < NACC; i++) {
                        if (i < p.Q) {
                            const float4 pr = *reinterpret_cast<const float4 *>(&P[i * ATT_TT + t4]);
                            float a = acc[i];
                            a = fmaf(pr.x, v[0], a);
                            a = fmaf(pr.y, v[1], a);
                            a = fmaf(pr.z, v[2], a);
                            a = fmaf(pr.w, v[3], a);
                            acc[i] = a;
                        }
                    }
                }
            }
        }
        __syncthreads();
        if (tid == 0 && tile + NST < n_tiles) issue(tile + NST);
    }
    if (lane == 0) {
#pragma unroll
        for (int j = 0; j < QPW; j++) {
            const int qi = warp + ATT_WARPS * j;
            if (qi < p.Q) {
                s_m[qi] = m_run[j];
                s_l[qi] = l_run[j];
            }
        }
    }
    __syncthreads();

    // ---- 4. outputs: merge the token groups (in group order), then write
    //         directly or combine across the cluster's splits
    float *s_o = reinterpret_cast<float *>(att_sm);   // [TG][Q][HD]: the ring is drained
#pragma unroll
    for (int i = 0; i < NACC; i++)
        if (i < p.Q) s_o[(tq * QMAX + i) * HD + od] = acc[i];
    __syncthreads();
    for (int e = tid; e < p.Q * HD; e += ATT_THREADS) {
        const int qi = e / HD, d = e - qi * HD;
        float o = s_o[qi * HD + d];
#pragma unroll
        for (int g = 1; g < TG; g++) o += s_o[(g * QMAX + qi) * HD + d];
        if (p.n_split == 1) {
            const int r = qi / p.G, gq = qi - r * p.G;
            p.out[(static_cast<size_t>(b) * p.R + r) * (static_cast<size_t>(p.nq) * HD) +
                  static_cast<size_t>(kvh * p.G + gq) * HD + d] = o / s_l[qi];
        } else {
            s_o[(TG * QMAX) * HD + e] = o;   // merged partial after the group planes
        }
    }
    if (p.n_split == 1) return;
    float *s_om = s_o + (TG * QMAX) * HD;
    __syncthreads();
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int ns = p.n_split;
    for (int e = split * ATT_THREADS + tid; e < p.Q * HD; e += ns * ATT_THREADS) {
        const int qi = e / HD, d = e - qi * HD;
        float ms[ATT_MAXNS];
        float M = -INFINITY;
        for (int r2 = 0; r2 < ns; r2++) {
            ms[r2] = cluster.map_shared_rank(s_m, r2)[qi];
            M = fmaxf(M, ms[r2]);
        }
        float L = 0.0f, O = 0.0f;
        for (int r2 = 0; r2 < ns; r2++) {
            if (ms[r2] == -INFINITY) continue;
            const float w = expf(ms[r2] - M);
            L = fmaf(cluster.map_shared_rank(s_l, r2)[qi], w, L);
            O = fmaf(cluster.map_shared_rank(s_om, r2)[qi * HD + d], w, O);
        }
        const int r = qi / p.G, g = qi - r * p.G;
        p.out[(static_cast<size_t>(b) * p.R + r) * (static_cast<size_t>(p.nq) * HD) +
              static_cast<size_t>(kvh * p.G + g) * HD + d] = O / L;
    }
    cluster.sync();   // keep this CTA's shared memory alive until every reader is done
}

// Splits per (sequence, kv head) = cluster size: about one CTA per SM in
// total, at least one stage (two pages) each, at most 16.
static int attn_splits(int B, int nkv, int max_pages) {
    const int groups = B * nkv;
    int ns = (sm_count() + groups / 2) / groups;
    ns = max(1, min(ns, ATT_MAXNS));
    ns = min(ns, max(1, (max_pages + 1) / 2));
    return ns;
}

size_t attn_scratch_bytes(int B, int R, int nq, int nkv, int hd, int max_pages) {
    (void)B; (void)R; (void)nq; (void)nkv; (void)hd; (void)max_pages;
    return 0;
}

template <int HD, int QMAX>
static bw_status attn_go(int ns, int nkv, int B, cudaStream_t st, const AttnParams &p) {
    constexpr size_t smem = att_smem_bytes<HD, QMAX>();
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return BW_ERR_CUDA;
    if (!attr_set[dev]) {
        if (cudaFuncSetAttribute(attn_kernel<HD, QMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess ||
            cudaFuncSetAttribute(attn_kernel<HD, QMAX>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess) {
            (void)cudaGetLastError();
            return BW_ERR_CUDA;
        }
        attr_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ns, nkv, B);
    cfg.blockDim = dim3(ATT_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = ns;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    AttnParams q = p;
    q.n_split = ns;
    cudaError_t e = cudaLaunchKernelEx(&cfg, attn_kernel<HD, QMAX>, q);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return BW_ERR_CUDA;
    }
    return BW_OK;
}

bw_status attn_launch(const float *qkv, const float *rope_cos, const float *rope_sin, int rope_max_pos,
                      void *k_pool, void *v_pool, const int32_t *page_table, int max_pages,
                      int n_pages, const int32_t *pos, int B, int R, int nq, int nkv, int hd,
                      float *out, const Scratch &sc, cudaStream_t st) {
    if (!qkv || !rope_cos || !rope_sin || !k_pool || !v_pool || !page_table || !pos || !out)
        return BW_ERR_INVALID_ARG;
    if (B <= 0 || R <= 0 || nq <= 0 || nkv <= 0 || max_pages <= 0 || n_pages <= 0 || rope_max_pos <= 0)
        return BW_ERR_INVALID_ARG;
    if ((hd != 128 && hd != 64) || nq % nkv || (nq / nkv) * R > ATT_MAXQ || R > ATT_MAXR)
        return BW_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(k_pool) || !aligned16(v_pool) || !aligned16(qkv)) return BW_ERR_INVALID_ARG;
    if (nkv > 65535 || B > 65535) return BW_ERR_UNSUPPORTED_SHAPE;
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
    p.scale = 1.0f / sqrtf(static_cast<float>(hd));
    p.out = out;
    p.err = sc.err;
    const int ns = attn_splits(B, nkv, max_pages);
    if (hd == 128) {
        if (p.Q <= 4) return attn_go<128, 4>(ns, nkv, B, st, p);
        if (p.Q <= 8) return attn_go<128, 8>(ns, nkv, B, st, p);
        if (p.Q <= 16) return attn_go<128, 16>(ns, nkv, B, st, p);
        return attn_go<128, 32>(ns, nkv, B, st, p);
    }
    if (p.Q <= 8) return attn_go<64, 8>(ns, nkv, B, st, p);
    return attn_go<64, 32>(ns, nkv, B, st, p);
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
