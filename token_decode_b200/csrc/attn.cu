// attn.cu -- paged fp16-KV GQA decode attention with fused RoPE and KV write
// (sm_100a).
//
// One CTA per (split, kv head, sequence).  A split is a contiguous range of
// the sequence's logical pages.  Each CTA
//   1. ropes the G = nq/nkv query heads of its kv head for each of the n_rows
//      query rows (positions pos..pos+n_rows-1),
//   2. ropes the new rows' k, rounds k and v to fp16 and writes them into the
//      paged pool when their position falls in its page range (the deep-dive
//      page, section 6: logical positions map to physical pages through the
//      page table; section 5, stage 4: the draft rows of a verify pass share
//      one cache, causally masked),
//   3. streams its pages into a ring of shared-memory stages: a producer warp
//      issues TMA tile loads (cp.async.bulk.tensor, boxes of 16 tokens x 64
//      dims with the 128-byte swizzle, completion on a "full" mbarrier) and
//      refills a stage when the consumer warps have released it (an "empty"
//      mbarrier), so the ring needs no block-wide barrier; the swizzle makes
//      the 8x8 fragment loads of K and V free of bank conflicts;
//   4. runs the scores and P.V of each 64-token stage on the tensor cores
//      (warp-level mma.m16n8k16, fp32 accumulate): the query rows are padded
//      to 16 (or 32); q and the probabilities are split into fp16 hi + lo
//      parts (hi + lo reproduces an fp32 value to ~22 bits) and multiplied by
//      the exact fp16 K and V in two MMAs each, so the products keep fp32
//      accuracy; the online softmax keeps one running max and sum per query
//      row, exchanged between warps through shared memory (two barriers per
//      stage, double-buffered);
//   5. writes the output (one split) or leaves (max, sum, partial output) in
//      the workspace; the last CTA of a
//      (sequence, kv head) to finish -- an atomic counter, no waiting --
//      combines the splits in split order.  Results are therefore
//      deterministic and independent of the physical page order.
// The q and P planes have padded rows, so their 8x8 fragment loads are free
// of shared-memory bank conflicts.
#include <cooperative_groups.h>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include <cuda_fp8.h>

#include "bw_common.cuh"

namespace cg = cooperative_groups;

namespace bw {

constexpr int ATT_CW = 8;                       // consumer warps
constexpr int ATT_THREADS = (ATT_CW + 1) * 32;  // + one producer warp
constexpr int ATT_CT = ATT_CW * 32;             // consumer threads
constexpr int ATT_MAXQ = 32;                    // query vectors per CTA (G * n_rows)
constexpr int ATT_MAXR = 8;                     // query rows per sequence (1 + draft tokens)
constexpr int ATT_MAXNS = 64;                   // splits per (sequence, kv head)
constexpr int ATT_MAXCL = 16;                   // splits merged inside one thread-block cluster
constexpr int ATT_MAXPAGES = 8192;              // page-table width the CTA's page list holds
constexpr int ATT_ST = 64;                      // tokens per stage: 4 pages, 8 per consumer warp
constexpr int ATT_PPS = ATT_ST / 16;
constexpr int ATT_PST = ATT_ST + 8;             // padded row of the probability planes (halves)
constexpr int ATT_PT_U = 2;                     // page-table entries per thread loaded with the position

struct AttnParams {
    const float *qkv;
    const float *rope_cos, *rope_sin;
    int rope_max_pos;
    __half *k_pool, *v_pool;  // fp16 pools, or E4M3 byte pools (same layout) with FP8 KV
    const int32_t *page_table;
    int max_pages, n_pages;
    const int32_t *pos;
    int B, R, nq, nkv, G, Q, n_split;
    int cluster;          // 1: the splits of a (sequence, kv head) are one cluster and merge through DSMEM
    int early;            // 1: pos and the page table are complete before this launch (see attn_launch)
    float scale;          // 1/sqrt(hd), times the K scale with FP8 KV
    float scale2;         // scale * log2(e) (base-2 softmax)
    float kscale, vscale; // FP8 KV: a stored code c stands for e4m3(c) * scale (1 for fp16)
    float *out;
    float *part_o;        // [B][nkv][n_split][Q][HD]
    float *part_ml;       // [B][nkv][n_split][Q][2]
    uint32_t *cnt;        // [B][nkv] arrival counters (zero between launches)
    uint32_t *err;
    // the layer's K and V pools as 2-D tensors [n_pages*nkv*16 rows][hd],
    // loaded in boxes of 16 rows x 64 dims with the 128-byte swizzle
    CUtensorMap tmk, tmv;
};

// shared memory: K/V ring, q hi/lo planes, P hi/lo planes (double buffered),
// row max / row sum exchange (double buffered), new k/v rows, barriers, and
// with FP8 KV the E4M3 landing ring the copies fill
template <int HD, int MT, int NST, int F8 = 0>
__host__ __device__ constexpr size_t att_smem_fixed() {
    return static_cast<size_t>(F8 ? 1 : NST) * 2 * ATT_ST * HD * 2       // K/V ring (fp16)
           + static_cast<size_t>(F8) * NST * 2 * ATT_ST * HD              // E4M3 landing ring
           + 2 * static_cast<size_t>(16 * MT) * (HD + 8) * 2              // q hi, lo
           + 2 * 2 * static_cast<size_t>(16 * MT) * ATT_PST * 2           // P hi, lo x 2 buffers
           + 2 * 2 * static_cast<size_t>(ATT_CW) * (16 * MT) * 4          // row max, row sum x 2 buffers
           + 2 * static_cast<size_t>(ATT_MAXR) * HD * 2                   // new k, v rows
           + 2 * static_cast<size_t>(NST) * 8                             // mbarriers
           + 1024;                                                        // ring alignment
}

// rotate-half RoPE of one pair, rounding each product like the plain formula
__device__ __forceinline__ void rope_pair(float a, float b, float c, float s, float &ra, float &rb) {
    ra = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
    rb = __fadd_rn(__fmul_rn(b, c), __fmul_rn(a, s));
}

__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(ATT_CT) : "memory"); }

// TMA tile load of one 2-D box (no multicast), completion on `bar`
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *tmap, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Byte offset of (token T of a stage, dim d) in a K or V stage: page T/16 is
// hd/64 boxes of 16 rows x 128 bytes; the 128-byte swizzle puts 16-byte chunk
// c of box row t at chunk c ^ (t & 7).
template <int HD>
__device__ __forceinline__ uint32_t kv_off(int T, int d) {
    const int t = T & 15, c = (d & 63) >> 3;
    return static_cast<uint32_t>((((T >> 4) * (HD / 64) + (d >> 6)) << 11) + (t << 7) + ((c ^ (t & 7)) << 4) +
                                 ((d & 7) << 1));
}

// Byte offset of (token T of a stage, code d) in an E4M3 landing stage: rows
// of HD bytes, one tensor box of 16 rows per page, with the copy's 128-byte
// (HD 128) or 64-byte (HD 64) swizzle moving 16-byte chunk c of row T to
// c ^ (T & 7) or c ^ ((T >> 1) & 3).
template <int HD>
__device__ __forceinline__ uint32_t land_off(int T, int d) {
    const int sw = HD == 128 ? (T & 7) : ((T >> 1) & 3);
    return static_cast<uint32_t>(T * HD + ((((d >> 4) ^ sw)) << 4) + (d & 15));
}

// four E4M3 codes (bytes of w, lowest first) -> two fp16x2 words; exact, since
// every E4M3 value is an fp16 value
__device__ __forceinline__ void e4m3x4_to_h4(uint32_t w, uint32_t &lo, uint32_t &hi) {
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.rn.f16x2.e4m3x2 %0, a;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

// warp-level tensor-core MMA (m16n8k16, f16 inputs, f32 accumulate) and the
// 8x8 shared-memory matrix loads that feed it
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t &r0, uint32_t &r1, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t &r0, uint32_t &r1, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

// Splits a value into fp16 hi + lo: hi + lo reproduces v to ~22 bits, so two
// MMAs (hi and lo) against exact fp16 K/V give products at fp32-level accuracy.
__device__ __forceinline__ void split_f16(float v, __half &hi, __half &lo) {
    hi = __float2half_rn(v);
    lo = __float2half_rn(v - __half2float(hi));
}

// NST: ring stages -- 2 when two CTAs share an SM, 4 when each CTA has an SM
// to itself (a short split then has all its pages in flight at once).
//
// F8 = 1: the pools hold E4M3 codes with per-layer K and V scales (the FP8 KV
// cache).  The copies bring a stage's codes into a landing ring; the consumers
// turn them into fp16 (exact: every E4M3 value is an fp16 value) in the fp16
// ring's layout and release the landing slot at once, so the tensor-core code
// below runs unchanged on the codes' values; the K scale is folded into the
// score scale and the V scale multiplies the output.
template <int HD, int MT, int NST, int F8>
__global__ void __launch_bounds__(ATT_THREADS, NST == 2 ? 2 : 1) attn_kernel(const __grid_constant__ AttnParams p) {
    constexpr int ATT_NST = NST;
    // fp16 ring stages: with FP8 KV one, since each warp converts into it only
    // what it reads itself (the landing ring is the one the copies run ahead in)
    constexpr int RS = F8 ? 1 : NST;
    constexpr int QM = 16 * MT;             // query rows of the MMA tiles (padded)
    constexpr int QS = HD + 8;              // padded q row (halves)
    constexpr int NKS = HD / 16;            // k-steps of the score MMA
    constexpr int WD = HD / ATT_CW;         // output dims per warp in P.V
    constexpr int NT = WD / 8;              // n-tiles per warp in P.V
    constexpr int SH = ATT_ST * HD;         // halves per K (or V) stage
    constexpr uint32_t PAGE_BYTES = 16 * HD * 2;
    // the cluster merge's partials and weights live in the drained ring
    static_assert(NST != 4 || (static_cast<size_t>(ATT_MAXQ) * HD + 3 * ATT_MAXQ + 2 * ATT_MAXCL * ATT_MAXQ) * 4 <=
                                  static_cast<size_t>(RS) * 2 * SH * 2,
                  "cluster merge scratch exceeds the ring");
    extern __shared__ __align__(1024) unsigned char att_sm_raw[];
    // the swizzle pattern follows address bits, so the ring starts on 1024 bytes
    unsigned char *att_sm = att_sm_raw + ((1024u - (smem_u32(att_sm_raw) & 1023u)) & 1023u);
    __half *ring = reinterpret_cast<__half *>(att_sm);                                  // [RS][K|V][SH]
    // E4M3 landing ring [NST][K|V][ATT_ST][HD] (FP8 KV only): 1024-byte aligned,
    // right after the fp16 ring, as tensor copies need
    unsigned char *land = reinterpret_cast<unsigned char *>(ring + static_cast<size_t>(RS) * 2 * SH);
    __half *qh = reinterpret_cast<__half *>(land + static_cast<size_t>(F8) * ATT_NST * 2 * ATT_ST * HD);  // [QM][QS]
    __half *ql = qh + QM * QS;
    __half *Ph = ql + QM * QS;                                                        // [2][QM][PST]
    __half *Pl = Ph + 2 * QM * ATT_PST;
    float *rmax = reinterpret_cast<float *>(Pl + 2 * QM * ATT_PST);                   // [2][CW][QM]
    float *rsum = rmax + 2 * ATT_CW * QM;
    __half *newk = reinterpret_cast<__half *>(rsum + 2 * ATT_CW * QM);                // [MAXR][HD]
    __half *newv = newk + ATT_MAXR * HD;
    uint64_t *full = reinterpret_cast<uint64_t *>(newv + ATT_MAXR * HD);              // [NST]
    uint64_t *empty = full + ATT_NST;                                                 // [NST]
    int *pages = reinterpret_cast<int *>(empty + ATT_NST);                            // this split's pages
    __shared__ bool s_last;

    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < ATT_NST; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], ATT_CW);
        }
        fence_mbar_init();
    }
    pdl_trigger();
    pdl_wait();

    // a page-table row of up to ATT_PT_U * ATT_THREADS entries is loaded
    // together with the position, so the split's page list does not cost a
    // second dependent round trip
    const int32_t *pt = p.page_table + static_cast<size_t>(b) * p.max_pages;
    const bool pt_pre = p.max_pages <= ATT_PT_U * ATT_THREADS;
    int pte[ATT_PT_U];
#pragma unroll
    for (int u = 0; u < ATT_PT_U; u++) {
        const int i = tid + u * ATT_THREADS;
        pte[u] = (pt_pre && i < p.max_pages) ? pt[i] : -1;
    }
    const int p0 = p.pos[b];
    int len = p0 + p.R;
    if (p0 < 0 || len > p.max_pages * 16 || len > p.rope_max_pos) {
        if (tid == 0) set_error(p.err, BW_DEVERR_BAD_POS);
        len = max(0, min(len, min(p.max_pages * 16, p.rope_max_pos)));
    }
    const int n_pg = (len + 15) / 16;
    const int pps = (n_pg + p.n_split - 1) / p.n_split;
    const int pg0 = min(n_pg, split * pps), pg1 = min(n_pg, pg0 + pps);
    const int npl = pg1 - pg0;                          // pages of this split
    const int t1 = min(len, pg1 * 16);
    const int n_stages = (npl + ATT_PPS - 1) / ATT_PPS;
    const size_t row_stride = static_cast<size_t>(p.nq + 2 * p.nkv) * HD;

    // the split's physical pages, validated once, in parallel
    if (pt_pre) {
#pragma unroll
        for (int u = 0; u < ATT_PT_U; u++) {
            const int i = tid + u * ATT_THREADS;
            if (i >= pg0 && i < pg1) {
                int page = pte[u];
                if (page < 0 || page >= p.n_pages) {
                    set_error(p.err, BW_DEVERR_BAD_PAGE);
                    page = -1;
                }
                pages[i - pg0] = page;
            }
        }
    } else {
        for (int i = tid; i < npl; i += ATT_THREADS) {
            int page = pt[pg0 + i];
            if (page < 0 || page >= p.n_pages) {
                set_error(p.err, BW_DEVERR_BAD_PAGE);
                page = -1;
            }
            pages[i] = page;
        }
    }
    __syncthreads();

    if (warp == ATT_CW) {
        // ---- producer: one lane streams the stages
        if (lane == 0) {
            for (int s = 0; s < n_stages; s++) {
                const int st = s % ATT_NST;
                if (s >= ATT_NST) mbar_wait(&empty[st], static_cast<uint32_t>((s / ATT_NST - 1) & 1), p.err);
                constexpr uint32_t PB = F8 ? 16 * HD : PAGE_BYTES;   // bytes of one page of K (or V)
                uint32_t bytes = 0;
                for (int j = 0; j < ATT_PPS; j++) {
                    const int lp = s * ATT_PPS + j;
                    if (lp < npl && pages[lp] >= 0) bytes += 2 * PB;
                }
                mbar_arrive_tx(&full[st], bytes);
                unsigned char *sk = F8 ? land + static_cast<size_t>(st) * 2 * ATT_ST * HD
                                       : reinterpret_cast<unsigned char *>(ring + static_cast<size_t>(st) * 2 * SH);
                for (int j = 0; j < ATT_PPS; j++) {
                    const int lp = s * ATT_PPS + j;
                    if (lp >= npl || pages[lp] < 0) continue;
                    const int y = (pages[lp] * p.nkv + kvh) * 16;     // first row of this page
                    if constexpr (F8) {
                        // one box of 16 rows x HD bytes per page, tokens back to back
                        // (swizzled, see land_off)
                        tma_load_2d(sk + j * PB, &p.tmk, 0, y, &full[st]);
                        tma_load_2d(sk + ATT_ST * HD + j * PB, &p.tmv, 0, y, &full[st]);
                    } else {
#pragma unroll
                        for (int h = 0; h < HD / 64; h++) {
                            const int box = (j * (HD / 64) + h) << 11;
                            tma_load_2d(sk + box, &p.tmk, h * 64, y, &full[st]);
                            tma_load_2d(sk + SH * 2 + box, &p.tmv, h * 64, y, &full[st]);
                        }
                    }
                }
            }
        }
        return;
    }

    // ---- 1. roped queries as fp16 hi/lo planes (padding rows are zero)
    for (int i = tid; i < QM * (HD / 2); i += ATT_CT) {
        const int qi = i / (HD / 2), d = i - qi * (HD / 2);
        float ra = 0.0f, rb = 0.0f;
        if (qi < p.Q) {
            const int r = qi / p.G, g = qi - r * p.G;
            const int h = kvh * p.G + g;
            const int ppos = max(0, min(p0 + r, p.rope_max_pos - 1));
            const float *src = p.qkv + (static_cast<size_t>(b) * p.R + r) * row_stride + static_cast<size_t>(h) * HD;
            const float c = p.rope_cos[static_cast<size_t>(ppos) * (HD / 2) + d];
            const float s = p.rope_sin[static_cast<size_t>(ppos) * (HD / 2) + d];
            rope_pair(src[d], src[d + HD / 2], c, s, ra, rb);
        }
        __half h0, l0, h1, l1;
        split_f16(ra, h0, l0);
        split_f16(rb, h1, l1);
        qh[qi * QS + d] = h0;
        ql[qi * QS + d] = l0;
        qh[qi * QS + d + HD / 2] = h1;
        ql[qi * QS + d + HD / 2] = l1;
    }

    // ---- 2. the new rows' k (roped) and v, rounded to fp16: kept for this
    //         CTA's stages and written into the pool
    for (int r = 0; r < p.R; r++) {
        const int ppos = p0 + r;
        if (ppos < pg0 * 16 || ppos >= t1) continue;
        const int page = pages[ppos / 16 - pg0];
        const bool ok = page >= 0;
        const size_t off = ((static_cast<size_t>(ok ? page : 0) * p.nkv + kvh) * 16 + (ppos & 15)) * HD;
        const float *krow = p.qkv + (static_cast<size_t>(b) * p.R + r) * row_stride +
                            static_cast<size_t>(p.nq + kvh) * HD;
        const float *vrow = krow + static_cast<size_t>(p.nkv) * HD;
        for (int d = tid; d < HD / 2; d += ATT_CT) {
            const float c = p.rope_cos[static_cast<size_t>(ppos) * (HD / 2) + d];
            const float s = p.rope_sin[static_cast<size_t>(ppos) * (HD / 2) + d];
            float ra, rb;
            rope_pair(krow[d], krow[d + HD / 2], c, s, ra, rb);
            if constexpr (F8) {
                // E4M3 of value / scale, round to nearest even, saturating to +-448
                const __nv_fp8_storage_t ca = __nv_cvt_float_to_fp8(__fdiv_rn(ra, p.kscale), __NV_SATFINITE, __NV_E4M3);
                const __nv_fp8_storage_t cb = __nv_cvt_float_to_fp8(__fdiv_rn(rb, p.kscale), __NV_SATFINITE, __NV_E4M3);
                newk[r * HD + d] = __float2half_rn(e4m3_to_f(ca));
                newk[r * HD + d + HD / 2] = __float2half_rn(e4m3_to_f(cb));
                if (ok) {
                    reinterpret_cast<uint8_t *>(p.k_pool)[off + d] = ca;
                    reinterpret_cast<uint8_t *>(p.k_pool)[off + d + HD / 2] = cb;
                }
            } else {
                const __half ha = __float2half_rn(ra), hb = __float2half_rn(rb);
                newk[r * HD + d] = ha;
                newk[r * HD + d + HD / 2] = hb;
                if (ok) {
                    p.k_pool[off + d] = ha;
                    p.k_pool[off + d + HD / 2] = hb;
                }
            }
        }
        for (int d = tid; d < HD; d += ATT_CT) {
            if constexpr (F8) {
                const __nv_fp8_storage_t cv = __nv_cvt_float_to_fp8(__fdiv_rn(vrow[d], p.vscale), __NV_SATFINITE, __NV_E4M3);
                newv[r * HD + d] = __float2half_rn(e4m3_to_f(cv));
                if (ok) reinterpret_cast<uint8_t *>(p.v_pool)[off + d] = cv;
            } else {
                const __half hv = __float2half_rn(vrow[d]);
                newv[r * HD + d] = hv;
                if (ok) p.v_pool[off + d] = hv;
            }
        }
    }
    consumers_sync();

    // ---- 3. stages of 64 tokens on the tensor cores
    const int gid = lane >> 2, tig = lane & 3;          // fragment row group / thread in group
    const uint32_t qh_a = smem_u32(qh), ql_a = smem_u32(ql);
    float m_run[MT][2], l_run[MT][2];
    float o[MT][NT][4];
#pragma unroll
    for (int mt = 0; mt < MT; mt++) {
#pragma unroll
        for (int h = 0; h < 2; h++) {
            m_run[mt][h] = -INFINITY;
            l_run[mt][h] = 0.0f;
        }
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
#pragma unroll
            for (int i = 0; i < 4; i++) o[mt][nt][i] = 0.0f;
    }

    for (int s = 0; s < n_stages; s++) {
        const int st = s % ATT_NST, buf = s & 1;
        mbar_wait(&full[st], static_cast<uint32_t>((s / ATT_NST) & 1), p.err);
        __half *sk = ring + static_cast<size_t>(F8 ? 0 : st) * 2 * SH;
        __half *sv = sk + SH;
        if constexpr (F8) {
            // E4M3 codes -> fp16 values in the ring's layout.  Each warp converts
            // exactly what it reads below -- K of its 8 tokens (all dims), V of
            // its WD dims (all tokens) -- so no CTA barrier is needed; the
            // landing slot goes back to the producer once every warp is done.
            const unsigned char *lk = land + static_cast<size_t>(st) * 2 * ATT_ST * HD;
            const unsigned char *lv = lk + ATT_ST * HD;
            unsigned char *skb = reinterpret_cast<unsigned char *>(sk), *svb = reinterpret_cast<unsigned char *>(sv);
            constexpr int KC = HD / 16;                 // 16-code chunks of a token
#pragma unroll
            for (int i = lane; i < 8 * KC; i += 32) {
                const int T = warp * 8 + i / KC, d0 = (i % KC) * 16;
                const uint4 c = *reinterpret_cast<const uint4 *>(lk + land_off<HD>(T, d0));
                uint32_t h[8];
                e4m3x4_to_h4(c.x, h[0], h[1]);
                e4m3x4_to_h4(c.y, h[2], h[3]);
                e4m3x4_to_h4(c.z, h[4], h[5]);
                e4m3x4_to_h4(c.w, h[6], h[7]);
                *reinterpret_cast<uint4 *>(skb + kv_off<HD>(T, d0)) = make_uint4(h[0], h[1], h[2], h[3]);
                *reinterpret_cast<uint4 *>(skb + kv_off<HD>(T, d0 + 8)) = make_uint4(h[4], h[5], h[6], h[7]);
            }
            const int vd0 = warp * WD;
#pragma unroll
            for (int T = lane; T < ATT_ST; T += 32) {
                if constexpr (WD == 16) {
                    const uint4 c = *reinterpret_cast<const uint4 *>(lv + land_off<HD>(T, vd0));
                    uint32_t h[8];
                    e4m3x4_to_h4(c.x, h[0], h[1]);
                    e4m3x4_to_h4(c.y, h[2], h[3]);
                    e4m3x4_to_h4(c.z, h[4], h[5]);
                    e4m3x4_to_h4(c.w, h[6], h[7]);
                    *reinterpret_cast<uint4 *>(svb + kv_off<HD>(T, vd0)) = make_uint4(h[0], h[1], h[2], h[3]);
                    *reinterpret_cast<uint4 *>(svb + kv_off<HD>(T, vd0 + 8)) = make_uint4(h[4], h[5], h[6], h[7]);
                } else {
                    const uint2 c = *reinterpret_cast<const uint2 *>(lv + land_off<HD>(T, vd0));
                    uint32_t h[4];
                    e4m3x4_to_h4(c.x, h[0], h[1]);
                    e4m3x4_to_h4(c.y, h[2], h[3]);
                    *reinterpret_cast<uint4 *>(svb + kv_off<HD>(T, vd0)) = make_uint4(h[0], h[1], h[2], h[3]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        const int tb = (pg0 + s * ATT_PPS) * 16;       // position of the stage's first token
        const int nvalid = min(ATT_ST, t1 - tb);
        bool missing = false;
        for (int j = 0; j < ATT_PPS; j++) {
            const int lp = s * ATT_PPS + j;
            if (lp < npl && pages[lp] < 0) missing = true;
        }
        const bool fix_new = p0 + p.R > tb && p0 < tb + ATT_ST;
        if (fix_new || missing || nvalid < ATT_ST) {
            // rows written by this step replace what the copy brought; V rows the
            // copy did not fill are zeroed (their probability is 0, 0 * stale could be NaN)
            if constexpr (F8) consumers_sync();   // every warp's conversion of the stage is done
            unsigned char *skb = reinterpret_cast<unsigned char *>(sk), *svb = reinterpret_cast<unsigned char *>(sv);
            for (int r = 0; r < p.R; r++) {
                const int slot = p0 + r - tb;
                if (slot < 0 || slot >= nvalid || pages[s * ATT_PPS + (slot >> 4)] < 0) continue;
                for (int d = tid; d < HD; d += ATT_CT) {
                    *reinterpret_cast<__half *>(skb + kv_off<HD>(slot, d)) = newk[r * HD + d];
                    *reinterpret_cast<__half *>(svb + kv_off<HD>(slot, d)) = newv[r * HD + d];
                }
            }
            // a token's 128-byte box rows hold only its own dims: zero them whole
            for (int e = tid; e < ATT_ST * (HD / 64) * 8; e += ATT_CT) {
                const int T = e / ((HD / 64) * 8), rem = e - T * ((HD / 64) * 8);
                const bool hole = T >= nvalid || pages[s * ATT_PPS + (T >> 4)] < 0;
                if (hole) {
                    const uint32_t row = static_cast<uint32_t>((((T >> 4) * (HD / 64) + (rem >> 3)) << 11) + ((T & 15) << 7));
                    *reinterpret_cast<uint4 *>(svb + row + ((rem & 7) << 4)) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            fence_async_smem();   // the next TMA load into this stage comes after these writes
            consumers_sync();
        }
        // scores: warp w takes tokens 8w .. 8w+7 (one n-tile) for every query row
        const int t0 = warp * 8;
        float sc[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; mt++)
#pragma unroll
            for (int i = 0; i < 4; i++) sc[mt][i] = 0.0f;
        {
            const uint32_t k_a = smem_u32(sk);
            const int ktok = t0 + (lane & 7), khalf = ((lane >> 3) & 1) * 8;
            const int arow = (lane & 7) + ((lane >> 3) & 1) * 8, acol = (lane >> 4) * 8;
#pragma unroll
            for (int kk = 0; kk < NKS; kk++) {
                uint32_t b0, b1;
                ldsm_x2(b0, b1, k_a + kv_off<HD>(ktok, kk * 16 + khalf));
#pragma unroll
                for (int mt = 0; mt < MT; mt++) {
                    const uint32_t off = static_cast<uint32_t>(((mt * 16 + arow) * QS + kk * 16 + acol) * 2);
                    uint32_t a[4];
                    ldsm_x4(a, qh_a + off);
                    mma16816(sc[mt], a, b0, b1);
                    ldsm_x4(a, ql_a + off);
                    mma16816(sc[mt], a, b0, b1);
                }
            }
        }
        // mask, row maxima over this warp's 8 tokens
        const int tok0 = t0 + tig * 2;                  // tokens of fragment columns 0, 1
#pragma unroll
        for (int mt = 0; mt < MT; mt++) {
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const int qi = mt * 16 + gid + 8 * h;
                const int lim = (qi < p.Q) ? min(t1, p0 + qi / p.G + 1) : 0;   // causal limit (exclusive)
#pragma unroll
                for (int c = 0; c < 2; c++) {
                    const int t = tok0 + c;
                    const bool ok = tb + t < lim && pages[s * ATT_PPS + (t >> 4)] >= 0;
                    sc[mt][2 * h + c] = ok ? sc[mt][2 * h + c] * p.scale : -INFINITY;
                }
                float mx = fmaxf(sc[mt][2 * h], sc[mt][2 * h + 1]);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                if (tig == 0) rmax[(buf * ATT_CW + warp) * QM + qi] = mx;
            }
        }
        consumers_sync();
        // probabilities against the new running max; row sums
        float corr[MT][2];
        __half *ph = Ph + buf * QM * ATT_PST, *pl = Pl + buf * QM * ATT_PST;
#pragma unroll
        for (int mt = 0; mt < MT; mt++) {
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const int qi = mt * 16 + gid + 8 * h;
                float ms = -INFINITY;
#pragma unroll
                for (int w2 = 0; w2 < ATT_CW; w2++) ms = fmaxf(ms, rmax[(buf * ATT_CW + w2) * QM + qi]);
                const float m_new = fmaxf(m_run[mt][h], ms);
                corr[mt][h] = (m_run[mt][h] == -INFINITY) ? 0.0f : expf(m_run[mt][h] - m_new);
                m_run[mt][h] = m_new;
                float sum = 0.0f;
#pragma unroll
                for (int c = 0; c < 2; c++) {
                    const float v = sc[mt][2 * h + c];
                    const float pr = (v == -INFINITY) ? 0.0f : expf(v - m_new);
                    sum += pr;
                    __half hi, lo;
                    split_f16(pr, hi, lo);
                    ph[qi * ATT_PST + tok0 + c] = hi;
                    pl[qi * ATT_PST + tok0 + c] = lo;
                }
                sum += __shfl_xor_sync(0xffffffffu, sum, 1);
                sum += __shfl_xor_sync(0xffffffffu, sum, 2);
                if (tig == 0) rsum[(buf * ATT_CW + warp) * QM + qi] = sum;
            }
        }
        consumers_sync();
#pragma unroll
        for (int mt = 0; mt < MT; mt++) {
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const int qi = mt * 16 + gid + 8 * h;
                float ss = 0.0f;
#pragma unroll
                for (int w2 = 0; w2 < ATT_CW; w2++) ss += rsum[(buf * ATT_CW + w2) * QM + qi];
                l_run[mt][h] = l_run[mt][h] * corr[mt][h] + ss;
#pragma unroll
                for (int nt = 0; nt < NT; nt++) {
                    o[mt][nt][2 * h] *= corr[mt][h];
                    o[mt][nt][2 * h + 1] *= corr[mt][h];
                }
            }
        }
        // P.V: warp w produces output dims w*WD .. w*WD + WD - 1 for every query row
        {
            const uint32_t ph_a = smem_u32(ph), pl_a = smem_u32(pl);
            const int arow = (lane & 7) + ((lane >> 3) & 1) * 8, acol = (lane >> 4) * 8;
            // V^T fragments: matrix i of the x4 load = tokens (i & 1) * 8 .., dims (i >> 1) * 8 ..
            const int vi = lane >> 3;
            const uint32_t v_a = smem_u32(sv);
            const int vtok = (lane & 7) + (vi & 1) * 8, vdim = warp * WD + (vi >> 1) * 8;
#pragma unroll
            for (int kk = 0; kk < ATT_ST / 16; kk++) {
                uint32_t bv[4];
                if constexpr (NT == 2) {
                    ldsm_x4_t(bv, v_a + kv_off<HD>(kk * 16 + vtok, vdim));
                } else {
                    ldsm_x2_t(bv[0], bv[1], v_a + kv_off<HD>(kk * 16 + vtok, vdim));
                }
#pragma unroll
                for (int mt = 0; mt < MT; mt++) {
                    const uint32_t off = static_cast<uint32_t>(((mt * 16 + arow) * ATT_PST + kk * 16 + acol) * 2);
                    uint32_t a[4];
                    ldsm_x4(a, ph_a + off);
#pragma unroll
                    for (int nt = 0; nt < NT; nt++) mma16816(o[mt][nt], a, bv[2 * nt], bv[2 * nt + 1]);
                    ldsm_x4(a, pl_a + off);
#pragma unroll
                    for (int nt = 0; nt < NT; nt++) mma16816(o[mt][nt], a, bv[2 * nt], bv[2 * nt + 1]);
                }
            }
        }
        // this warp is done with the stage: release it to the producer
        if constexpr (!F8) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
    }

    // ---- 4. the output, or a partial for the split combine
    if (p.cluster) {
        // the splits form one thread-block cluster: partials stay in shared
        // memory (the drained ring), each CTA merges a slice of the outputs
        // from every split's shared memory, in split order.  The partials
        // overwrite the ring, which slower warps may still be reading (V of
        // the last stage): all consumers finish first.
        consumers_sync();
        float *s_o = reinterpret_cast<float *>(att_sm);           // [Q][HD] unnormalized output
        float *s_m = s_o + ATT_MAXQ * HD;                           // [Q]
        float *s_l = s_m + ATT_MAXQ;                                // [Q]
#pragma unroll
        for (int mt = 0; mt < MT; mt++) {
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const int qi = mt * 16 + gid + 8 * h;
                if (qi >= p.Q) continue;
#pragma unroll
                for (int nt = 0; nt < NT; nt++) {
                    const int d = warp * WD + nt * 8 + tig * 2;
                    s_o[qi * HD + d] = o[mt][nt][2 * h];
                    s_o[qi * HD + d + 1] = o[mt][nt][2 * h + 1];
                }
                if (warp == 0 && tig == 0) {
                    s_m[qi] = m_run[mt][h];
                    s_l[qi] = l_run[mt][h];
                }
            }
        }
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        const int ns = p.n_split;
        // every split's (max, sum) in one parallel pass of remote loads, the
        // merge weights once per query row, then one pass of independent
        // remote loads of the partial outputs, summed in split order
        float *s_w = s_l + ATT_MAXQ;                  // [ns][Q] max, then weight (local only)
        float *s_sl = s_w + ATT_MAXCL * ATT_MAXQ;     // [ns][Q] sums
        float *s_L = s_sl + ATT_MAXCL * ATT_MAXQ;     // [Q]
        for (int e = tid; e < ns * p.Q; e += ATT_CT) {
            const int r2 = e / p.Q, qi = e - r2 * p.Q;
            s_w[e] = cluster.map_shared_rank(s_m, r2)[qi];
            s_sl[e] = cluster.map_shared_rank(s_l, r2)[qi];
        }
        consumers_sync();
        if (tid < p.Q) {
            const int qi = tid;
            float M = -INFINITY;
            for (int r2 = 0; r2 < ns; r2++) M = fmaxf(M, s_w[r2 * p.Q + qi]);
            float L = 0.0f;
            for (int r2 = 0; r2 < ns; r2++) {
                const float m2 = s_w[r2 * p.Q + qi];
                const float w = (m2 == -INFINITY) ? 0.0f : expf(m2 - M);
                s_w[r2 * p.Q + qi] = w;
                L = fmaf(s_sl[r2 * p.Q + qi], w, L);
            }
            s_L[qi] = L;
        }
        consumers_sync();
        const int per = (p.Q * HD + ns - 1) / ns;
        for (int e = split * per + tid; e < min(p.Q * HD, (split + 1) * per); e += ATT_CT) {
            const int qi = e / HD, d = e - qi * HD;
            float ov[ATT_MAXCL];
#pragma unroll
            for (int r2 = 0; r2 < ATT_MAXCL; r2++)
                ov[r2] = r2 < ns ? cluster.map_shared_rank(s_o, min(r2, ns - 1))[qi * HD + d] : 0.0f;
            float O = 0.0f;
#pragma unroll
            for (int r2 = 0; r2 < ATT_MAXCL; r2++)
                if (r2 < ns) O = fmaf(ov[r2], s_w[r2 * p.Q + qi], O);
            const int r = qi / p.G, gq = qi - r * p.G;
            p.out[(static_cast<size_t>(b) * p.R + r) * (static_cast<size_t>(p.nq) * HD) +
                  static_cast<size_t>(kvh * p.G + gq) * HD + d] = (O * p.vscale) / s_L[qi];
        }
        cluster.sync();   // keep this CTA's shared memory alive until every reader is done
        return;
    }
    const size_t pbase = (static_cast<size_t>(b) * p.nkv + kvh) * p.n_split;
#pragma unroll
    for (int mt = 0; mt < MT; mt++) {
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const int qi = mt * 16 + gid + 8 * h;
            if (qi >= p.Q) continue;
            const int r = qi / p.G, gq = qi - r * p.G;
#pragma unroll
            for (int nt = 0; nt < NT; nt++) {
                const int d = warp * WD + nt * 8 + tig * 2;
                const float o0 = o[mt][nt][2 * h], o1 = o[mt][nt][2 * h + 1];
                if (p.n_split == 1) {
                    float *dst = p.out + (static_cast<size_t>(b) * p.R + r) * (static_cast<size_t>(p.nq) * HD) +
                                 static_cast<size_t>(kvh * p.G + gq) * HD + d;
                    dst[0] = (o0 * p.vscale) / l_run[mt][h];
                    dst[1] = (o1 * p.vscale) / l_run[mt][h];
                } else {
                    __stcg(reinterpret_cast<float2 *>(p.part_o + ((pbase + split) * p.Q + qi) * HD + d),
                           make_float2(o0, o1));
                }
            }
            if (p.n_split > 1 && warp == 0 && tig == 0)
                __stcg(reinterpret_cast<float2 *>(p.part_ml + ((pbase + split) * p.Q + qi) * 2),
                       make_float2(m_run[mt][h], l_run[mt][h]));
        }
    }
    if (p.n_split == 1) return;
    // the last split of this (sequence, kv head) to finish combines all of them
    __threadfence();
    consumers_sync();
    uint32_t *cnt = p.cnt + static_cast<size_t>(b) * p.nkv + kvh;
    if (tid == 0) s_last = atomicAdd(cnt, 1u) == static_cast<uint32_t>(p.n_split - 1);
    consumers_sync();
    if (!s_last) return;
    __threadfence();
    const int ns = p.n_split;
    // every split's (max, sum) in one parallel pass, the weights from shared
    // memory, then one pass of independent float4 loads of the partial outputs
    float *s_w = reinterpret_cast<float *>(att_sm);        // [ns][Q] max, then weight (the ring is free)
    float *s_sl = s_w + ATT_MAXNS * ATT_MAXQ;              // [ns][Q] sums
    float *s_L = s_sl + ATT_MAXNS * ATT_MAXQ;              // [Q]
    for (int e = tid; e < ns * p.Q; e += ATT_CT) {
        const float2 ml = __ldcg(reinterpret_cast<const float2 *>(p.part_ml + (pbase * p.Q + e) * 2));
        s_w[e] = ml.x;
        s_sl[e] = ml.y;
    }
    consumers_sync();
    if (tid < p.Q) {
        const int qi = tid;
        float M = -INFINITY;
        for (int r2 = 0; r2 < ns; r2++) M = fmaxf(M, s_w[r2 * p.Q + qi]);
        float L = 0.0f;
        for (int r2 = 0; r2 < ns; r2++) {
            const float m2 = s_w[r2 * p.Q + qi];
            const float w = (m2 == -INFINITY) ? 0.0f : expf(m2 - M);
            s_w[r2 * p.Q + qi] = w;
            L = fmaf(s_sl[r2 * p.Q + qi], w, L);
        }
        s_L[qi] = L;
    }
    consumers_sync();
    for (int e = tid; e < p.Q * (HD / 4); e += ATT_CT) {
        const int qi = e / (HD / 4), d = (e - qi * (HD / 4)) * 4;
        const float4 *src = reinterpret_cast<const float4 *>(p.part_o + (pbase * p.Q + qi) * HD + d);
        const size_t stride = static_cast<size_t>(p.Q) * HD / 4;
        float4 O = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll 16
        for (int r2 = 0; r2 < ns; r2++) {
            const float4 v = __ldcg(src + r2 * stride);
            const float w = s_w[r2 * p.Q + qi];
            O.x = fmaf(v.x, w, O.x);
            O.y = fmaf(v.y, w, O.y);
            O.z = fmaf(v.z, w, O.z);
            O.w = fmaf(v.w, w, O.w);
        }
        const int r = qi / p.G, gq = qi - r * p.G;
        const float L = s_L[qi];
        float *dst = p.out + (static_cast<size_t>(b) * p.R + r) * (static_cast<size_t>(p.nq) * HD) +
                     static_cast<size_t>(kvh * p.G + gq) * HD + d;
        const float vs = p.vscale;
        *reinterpret_cast<float4 *>(dst) = make_float4((O.x * vs) / L, (O.y * vs) / L, (O.z * vs) / L, (O.w * vs) / L);
    }
    consumers_sync();
    if (tid == 0) *cnt = 0u;
}

// ---------------------------------------------------------------------------
// Grouped-query decode attention with the tokens on the MMA's M side, for up
// to 8 query rows per (sequence, kv head).
//
// The kv head's G * R roped query rows, split into fp16 hi and lo parts, are
// the N = 8 (up to 4 rows) or 16 (up to 8 rows) columns of the MMA, and 16
// tokens are its M rows:
//     S^T [16 tokens x cols]  = K [16 tokens x hd] . Q^T [hd x cols]
//     O^T [hd x cols]        += V^T [hd x 16 tokens] . P^T [16 tokens x cols]
// so no MMA row is padding and the hi / lo products cost no second MMA.  Each
// consumer warp owns 16 tokens (one page) of every stage:
// its own running max and sum per query row and its own O^T; nothing crosses
// warps inside the stage loop.  The hi and lo columns are added, and the warps
// merged, once at the end.
//
// With an E4M3 cache the MMA fragments are built straight from the codes in
// shared memory (cvt.rn.f16x2.e4m3x2, exact): K's dims (the score MMA's k) and
// V's tokens (the output MMA's k) are taken in an order that puts a lane's
// codes in whole 32-bit words -- any order of k gives the same sums, as long
// as Q and P are written in the same order -- and O^T's rows (dims) in an
// order that lets one word of V feed two m-tiles.
//
// Softmax in base 2: the scores are scaled by log2(e) / sqrt(hd) and
// exponentiated with exp2f; the merges use the same units.
//
// Splits of a (sequence, kv head) that fit one thread-block cluster (2..16)
// combine in the leader (rank 0): every other split writes its partial --
// unnormalized O, then (max, sum) per query row -- straight from registers
// into a receive slot in the leader's shared memory with st.async, whose
// bytes count down a transaction barrier the leader armed for all of them at
// start; the leader adds the partials in split order and releases the others
// (a remote arrive on a barrier of theirs, so that none exits while its
// stores are in flight).  One cluster barrier, split into an arrive at start
// and a wait before the first remote access, orders the barriers'
// initialisation.  More splits combine through the workspace (last arriver).
//
// Inside a decode step (AttnParams::early) the page list, the position and the
// first K/V copies do not wait for the previous kernel (the projection), only
// the query rows and the new k/v row do.
constexpr int AG_PST = 24;                        // padded P^T row (halves): conflict-free ldmatrix
constexpr int AG_MAXQ = 8;                        // query rows per (sequence, kv head)

template <int CT>
__device__ __forceinline__ void ag_sync() { asm volatile("bar.sync 1, %0;" ::"n"(CT) : "memory"); }

__device__ __forceinline__ uint32_t ag_prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// E4M3 K: MMA k-index of dim d.  Lane group t (lane & 3) reads bytes 16t ..
// 16t + 15 of each 64 dims: word j of them is k-step 4g + j, its bytes the
// k positions 2t, 2t + 1, 2t + 8, 2t + 9 of that step.
__device__ __forceinline__ int ag_kidx_f8(int d) {
    const int g = d >> 6, r = d & 63, t = r >> 4, j = (r >> 2) & 3, e = r & 3;
    return (4 * g + j) * 16 + 2 * t + (e & 1) + 8 * (e >> 1);
}
// E4M3 V: MMA k-index of token tau (0..15) of a warp's page.  Lane group t
// reads tokens 4t .. 4t + 3: k positions 2t, 2t + 1, 2t + 8, 2t + 9.
__device__ __forceinline__ int ag_tidx_f8(int tau) {
    const int t = tau >> 2, e = tau & 3;
    return 2 * t + (e & 1) + 8 * (e >> 1);
}

// a stage is one page (16 tokens) per consumer warp, K and V
template <int HD, int F8, int CW>
__host__ __device__ constexpr size_t ag_stage_bytes() {
    return static_cast<size_t>(2) * 16 * CW * HD * (F8 ? 1 : 2);
}

// byte offset of the per-warp merge scratch in the drained ring: after the
// split merge's partials, maxima, sums and weights
template <int HD>
__host__ __device__ constexpr size_t ag_scratch_off() {
    return ((static_cast<size_t>(ATT_MAXQ) * HD + 3 * ATT_MAXQ + 2 * ATT_MAXCL * ATT_MAXQ) * 4 + 15) / 16 * 16;
}

template <int HD, int NQT, int NST, int F8, int CW>
__host__ __device__ constexpr size_t ag_smem_fixed() {
    return static_cast<size_t>(NST) * ag_stage_bytes<HD, F8, CW>()             // K/V ring
           + static_cast<size_t>(8 * NQT) * (HD + 8) * 2                       // Q^T [cols][dims]
           + static_cast<size_t>(CW) * 8 * NQT * AG_PST * 2                    // P^T per warp [cols][tokens]
           + 2 * static_cast<size_t>(ATT_MAXR) * HD * (F8 ? 1 : 2)            // new k, v rows
           + 2 * static_cast<size_t>(CW) * AG_MAXQ * 4                        // warp maxima, sums
           + (2 * static_cast<size_t>(NST) + 2) * 8                           // mbarriers
           + 1024;                                                            // ring alignment
}

// Cluster merge: each non-leader split writes its partial -- O [Q][HD]
// (unnormalized), then (max, sum) per query row -- into slot rank - 1 of the
// leader's receive area, which follows the page list.
__host__ __device__ constexpr int ag_slot_floats(int Q, int HD) { return (Q * HD + 2 * Q + 3) / 4 * 4; }
__host__ __device__ constexpr uint32_t ag_push_bytes(int Q, int HD) { return static_cast<uint32_t>(Q * HD + 2 * Q) * 4; }
__host__ __device__ constexpr size_t ag_recv_bytes(int ns, int Q, int HD) {
    return ns > 1 ? 16 + static_cast<size_t>(ns - 1) * ag_slot_floats(Q, HD) * 4 : 0;
}

__device__ __forceinline__ void cluster_arrive_rel() { asm volatile("barrier.cluster.arrive.release;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait_acq() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }
// this CTA's shared address `a` as seen in cluster rank `rank`'s shared memory
__device__ __forceinline__ uint32_t ag_mapa(uint32_t a, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}
// stores into another CTA's shared memory that complete_tx on its mbarrier
__device__ __forceinline__ void st_async_v4(uint32_t addr, float4 v, uint32_t mbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(addr),
                 "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(mbar)
                 : "memory");
}
__device__ __forceinline__ void st_async_v2(uint32_t addr, float a, float b, uint32_t mbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(addr), "f"(a),
                 "f"(b), "r"(mbar)
                 : "memory");
}
// arrive on an mbarrier in another CTA of the cluster
__device__ __forceinline__ void mbar_arrive_remote(uint32_t mbar) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(mbar) : "memory");
}

// CW consumer warps: 4 (two CTAs share an SM) or 8 (a CTA has an SM to itself)
template <int HD, int NQT, int NST, int F8, int CW>
__global__ void __launch_bounds__((CW + 1) * 32, CW == 4 ? 2 : 1) attn_g_kernel(const __grid_constant__ AttnParams p) {
    constexpr int AG_CW = CW;                   // consumer warps
    constexpr int AG_CT = CW * 32;              // consumer threads
    constexpr int AG_THREADS = AG_CT + 32;      // + the producer warp
    constexpr int AG_ST = 16 * CW;              // tokens per stage: one page per consumer warp
    constexpr int AG_PPS = CW;
    constexpr int NC = 8 * NQT;                 // MMA columns
    constexpr int QP = 4 * NQT;                 // query rows per part (hi, lo)
    constexpr int QSS = HD + 8;                 // padded Q^T row (halves)
    constexpr int NKS = HD / 16;                // k-steps of the score MMA
    constexpr int NMT = HD / 16;                // m-tiles of O^T
    constexpr size_t STB = ag_stage_bytes<HD, F8, CW>();
    constexpr uint32_t PB = 16 * HD * (F8 ? 1 : 2);   // bytes of one page of K (or V)
    constexpr int EB = F8 ? 1 : 2;              // bytes of a stored element
    static_assert(ag_scratch_off<HD>() + static_cast<size_t>(AG_CW) * QP * HD * 4 <= NST * STB,
                  "merge scratch exceeds the ring");
    extern __shared__ __align__(1024) unsigned char ag_sm_raw[];
    // the swizzle pattern follows address bits, so the ring starts on 1024 bytes
    unsigned char *sm = ag_sm_raw + ((1024u - (smem_u32(ag_sm_raw) & 1023u)) & 1023u);
    unsigned char *ring = sm;                                                   // [NST][K|V]
    __half *qs = reinterpret_cast<__half *>(ring + NST * STB);                  // [NC][QSS]
    __half *ps = qs + NC * QSS;                                                 // [CW][NC][PST]
    unsigned char *newk = reinterpret_cast<unsigned char *>(ps + AG_CW * NC * AG_PST);   // [MAXR][HD]
    unsigned char *newv = newk + ATT_MAXR * HD * EB;
    float *s_mw = reinterpret_cast<float *>(newv + ATT_MAXR * HD * EB);        // [CW][MAXQ]
    float *s_lw = s_mw + AG_CW * AG_MAXQ;
    uint64_t *full = reinterpret_cast<uint64_t *>(s_lw + AG_CW * AG_MAXQ);     // [NST]
    uint64_t *empty = full + NST;                                              // [NST]
    uint64_t *mrecv = empty + NST;             // leader: the other splits' partials have landed
    uint64_t *mack = mrecv + 1;                // non-leader: the leader has all of this split's partial
    int *pages = reinterpret_cast<int *>(mack + 1);                            // this split's pages
    float *rcv = reinterpret_cast<float *>(sm + (reinterpret_cast<uintptr_t>(pages + p.max_pages) -
                                                 reinterpret_cast<uintptr_t>(sm) + 15) / 16 * 16);   // [ns-1][slot]
    __shared__ bool s_last;

    const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < NST; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], AG_CW);
        }
        if (p.cluster) {
            mbar_init(mrecv, 1);
            mbar_init(mack, 1);
        }
        fence_mbar_init();
        // the leader expects every other split's partial before any can arrive
        if (p.cluster && split == 0) mbar_arrive_tx(mrecv, (p.n_split - 1) * ag_push_bytes(p.Q, HD));
    }
    // every thread: this CTA's barriers exist (released to the cluster)
    if (p.cluster) cluster_arrive_rel();
    // With p.early the launch that precedes this one signalled its dependents
    // only after its own dependency wait, so every launch before that one --
    // and with them pos and the page table -- is complete: the page list and
    // the first K/V copies need not wait for the previous kernel (L2 loads).
    if (!p.early) pdl_wait();

    const int32_t *pt = p.page_table + static_cast<size_t>(b) * p.max_pages;
    const bool pt_pre = p.max_pages <= ATT_PT_U * AG_THREADS;
    int pte[ATT_PT_U];
#pragma unroll
    for (int u = 0; u < ATT_PT_U; u++) {
        const int i = tid + u * AG_THREADS;
        pte[u] = (pt_pre && i < p.max_pages) ? __ldcg(pt + i) : -1;
    }
    const int p0 = __ldcg(p.pos + b);
    int len = p0 + p.R;
    if (p0 < 0 || len > p.max_pages * 16 || len > p.rope_max_pos) {
        if (tid == 0) set_error(p.err, BW_DEVERR_BAD_POS);
        len = max(0, min(len, min(p.max_pages * 16, p.rope_max_pos)));
    }
    const int n_pg = (len + 15) / 16;
    const int pps = (n_pg + p.n_split - 1) / p.n_split;
    const int pg0 = min(n_pg, split * pps), pg1 = min(n_pg, pg0 + pps);
    const int npl = pg1 - pg0;                          // pages of this split
    const int t1 = min(len, pg1 * 16);
    const int n_stages = (npl + AG_PPS - 1) / AG_PPS;
    const size_t row_stride = static_cast<size_t>(p.nq + 2 * p.nkv) * HD;

    if (pt_pre) {
#pragma unroll
        for (int u = 0; u < ATT_PT_U; u++) {
            const int i = tid + u * AG_THREADS;
            if (i >= pg0 && i < pg1) {
                int page = pte[u];
                if (page < 0 || page >= p.n_pages) {
                    set_error(p.err, BW_DEVERR_BAD_PAGE);
                    page = -1;
                }
                pages[i - pg0] = page;
            }
        }
    } else {
        for (int i = tid; i < npl; i += AG_THREADS) {
            int page = __ldcg(pt + pg0 + i);
            if (page < 0 || page >= p.n_pages) {
                set_error(p.err, BW_DEVERR_BAD_PAGE);
                page = -1;
            }
            pages[i] = page;
        }
    }
    __syncthreads();

    if (warp == AG_CW) {
        // ---- producer: one lane streams the stages
        if (lane == 0) {
            for (int s = 0; s < n_stages; s++) {
                const int st = s % NST;
                if (s >= NST) mbar_wait(&empty[st], static_cast<uint32_t>((s / NST - 1) & 1), p.err);
                uint32_t bytes = 0;
                for (int j = 0; j < AG_PPS; j++) {
                    const int lp = s * AG_PPS + j;
                    if (lp < npl && pages[lp] >= 0) bytes += 2 * PB;
                }
                mbar_arrive_tx(&full[st], bytes);
                unsigned char *sk = ring + static_cast<size_t>(st) * STB;
                for (int j = 0; j < AG_PPS; j++) {
                    const int lp = s * AG_PPS + j;
                    if (lp >= npl || pages[lp] < 0) continue;
                    const int y = (pages[lp] * p.nkv + kvh) * 16;     // first row of this page
                    if constexpr (F8) {
                        // one box of 16 rows x HD bytes per page (swizzled, see land_off)
                        tma_load_2d(sk + j * PB, &p.tmk, 0, y, &full[st]);
                        tma_load_2d(sk + STB / 2 + j * PB, &p.tmv, 0, y, &full[st]);
                    } else {
#pragma unroll
                        for (int h = 0; h < HD / 64; h++) {
                            const int box = (j * (HD / 64) + h) << 11;
                            tma_load_2d(sk + box, &p.tmk, h * 64, y, &full[st]);
                            tma_load_2d(sk + STB / 2 + box, &p.tmv, h * 64, y, &full[st]);
                        }
                    }
                }
            }
        }
        if (p.cluster) cluster_wait_acq();   // pairs this warp's arrive
        return;
    }

    if (p.early) pdl_wait();   // the query rows and new k/v come from the previous kernel

    // ---- 1. Q^T: the roped query rows as fp16 hi (columns 0..QP-1) and lo
    //         (QP..2QP-1) parts, in the MMA's k order; padding rows are zero.
    //         Their loads are issued first, so that they are in flight with
    //         the new rows' loads (one round trip for both).
    constexpr int NQI = (QP * (HD / 2) + AG_CT - 1) / AG_CT;
    float qx[NQI], qy[NQI], qc[NQI], qn[NQI];
#pragma unroll
    for (int u = 0; u < NQI; u++) {
        const int i = tid + u * AG_CT;
        const int qi = i / (HD / 2), d = i - qi * (HD / 2);
        qx[u] = 0.0f;
        qy[u] = 0.0f;
        qc[u] = 0.0f;
        qn[u] = 0.0f;
        if (i < QP * (HD / 2) && qi < p.Q) {
            const int r = qi / p.G, g = qi - r * p.G;
            const int h = kvh * p.G + g;
            const int ppos = max(0, min(p0 + r, p.rope_max_pos - 1));
            const float *src = p.qkv + (static_cast<size_t>(b) * p.R + r) * row_stride + static_cast<size_t>(h) * HD;
            qx[u] = src[d];
            qy[u] = src[d + HD / 2];
            qc[u] = p.rope_cos[static_cast<size_t>(ppos) * (HD / 2) + d];
            qn[u] = p.rope_sin[static_cast<size_t>(ppos) * (HD / 2) + d];
        }
    }

    // ---- 2. the new rows' k (roped) and v as stored (fp16, or E4M3 codes of
    //         value / scale): kept for this CTA's stages and written into the pool
    for (int r = 0; r < p.R; r++) {
        const int ppos = p0 + r;
        if (ppos < pg0 * 16 || ppos >= t1) continue;
        const int page = pages[ppos / 16 - pg0];
        const bool ok = page >= 0;
        const size_t off = ((static_cast<size_t>(ok ? page : 0) * p.nkv + kvh) * 16 + (ppos & 15)) * HD;
        const float *krow = p.qkv + (static_cast<size_t>(b) * p.R + r) * row_stride +
                            static_cast<size_t>(p.nq + kvh) * HD;
        const float *vrow = krow + static_cast<size_t>(p.nkv) * HD;
        for (int d = tid; d < HD / 2; d += AG_CT) {
            const float c = p.rope_cos[static_cast<size_t>(ppos) * (HD / 2) + d];
            const float s = p.rope_sin[static_cast<size_t>(ppos) * (HD / 2) + d];
            float ra, rb;
            rope_pair(krow[d], krow[d + HD / 2], c, s, ra, rb);
            if constexpr (F8) {
                // E4M3 of value / scale, round to nearest even, saturating to +-448
                const __nv_fp8_storage_t ca = __nv_cvt_float_to_fp8(__fdiv_rn(ra, p.kscale), __NV_SATFINITE, __NV_E4M3);
                const __nv_fp8_storage_t cb = __nv_cvt_float_to_fp8(__fdiv_rn(rb, p.kscale), __NV_SATFINITE, __NV_E4M3);
                newk[r * HD + d] = ca;
                newk[r * HD + d + HD / 2] = cb;
                if (ok) {
                    reinterpret_cast<uint8_t *>(p.k_pool)[off + d] = ca;
                    reinterpret_cast<uint8_t *>(p.k_pool)[off + d + HD / 2] = cb;
                }
            } else {
                const __half ha = __float2half_rn(ra), hb = __float2half_rn(rb);
                reinterpret_cast<__half *>(newk)[r * HD + d] = ha;
                reinterpret_cast<__half *>(newk)[r * HD + d + HD / 2] = hb;
                if (ok) {
                    p.k_pool[off + d] = ha;
                    p.k_pool[off + d + HD / 2] = hb;
                }
            }
        }
        for (int d = tid; d < HD; d += AG_CT) {
            if constexpr (F8) {
                const __nv_fp8_storage_t cv = __nv_cvt_float_to_fp8(__fdiv_rn(vrow[d], p.vscale), __NV_SATFINITE, __NV_E4M3);
                newv[r * HD + d] = cv;
                if (ok) reinterpret_cast<uint8_t *>(p.v_pool)[off + d] = cv;
            } else {
                const __half hv = __float2half_rn(vrow[d]);
                reinterpret_cast<__half *>(newv)[r * HD + d] = hv;
                if (ok) p.v_pool[off + d] = hv;
            }
        }
    }
#pragma unroll
    for (int u = 0; u < NQI; u++) {
        const int i = tid + u * AG_CT;
        if (i < QP * (HD / 2)) {
            const int qi = i / (HD / 2), d = i - qi * (HD / 2);
            float ra = 0.0f, rb = 0.0f;
            if (qi < p.Q) rope_pair(qx[u], qy[u], qc[u], qn[u], ra, rb);
            __half h0, l0, h1, l1;
            split_f16(ra, h0, l0);
            split_f16(rb, h1, l1);
            const int ka = F8 ? ag_kidx_f8(d) : d, kb = F8 ? ag_kidx_f8(d + HD / 2) : d + HD / 2;
            qs[qi * QSS + ka] = h0;
            qs[(QP + qi) * QSS + ka] = l0;
            qs[qi * QSS + kb] = h1;
            qs[(QP + qi) * QSS + kb] = l1;
        }
    }
    ag_sync<AG_CT>();

    // ---- 3. stages of one page per warp
    const int gid = lane >> 2, tig = lane & 3;          // fragment row group / thread in group
    // this lane's query rows qa, qa + 1 (score and output columns 2 tig, 2 tig + 1)
    const int qa = NQT == 1 ? 2 * (tig & 1) : 2 * tig;
    uint32_t qb[NKS][NQT][2];                           // Q^T fragments, held for every stage
    {
        const int l8 = lane & 7, kh = ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int kk = 0; kk < NKS; kk++)
#pragma unroll
            for (int nt = 0; nt < NQT; nt++)
                ldsm_x2(qb[kk][nt][0], qb[kk][nt][1], smem_u32(qs + (nt * 8 + l8) * QSS + kk * 16 + kh));
    }
    const int tw = warp * 16;                           // this warp's tokens in a stage
    __half *pw = ps + warp * NC * AG_PST;               // this warp's P^T
    float m_q[2] = {-INFINITY, -INFINITY}, l_q[2] = {0.0f, 0.0f};
    float ot[NMT][NQT][4];
#pragma unroll
    for (int mt = 0; mt < NMT; mt++)
#pragma unroll
        for (int nt = 0; nt < NQT; nt++)
#pragma unroll
            for (int i = 0; i < 4; i++) ot[mt][nt][i] = 0.0f;

    for (int s = 0; s < n_stages; s++) {
        const int st = s % NST;
        mbar_wait(&full[st], static_cast<uint32_t>((s / NST) & 1), p.err);
        // the next kernel (it streams only its weights before its wait) starts
        // once this CTA's first K/V stage has landed, so that its copies do not
        // compete with the first stage
        if (s == 0) pdl_trigger();
        unsigned char *sk = ring + static_cast<size_t>(st) * STB;
        unsigned char *sv = sk + STB / 2;
        const int tb = (pg0 + s * AG_PPS) * 16;       // position of the stage's first token
        const int nvalid = min(AG_ST, t1 - tb);
        const bool page_ok = s * AG_PPS + warp < npl && pages[s * AG_PPS + warp] >= 0;   // this warp's page
        const bool fix_new = p0 + p.R > tb + tw && p0 < tb + tw + 16;
        if (fix_new || !page_ok || nvalid < tw + 16) {
            // this warp's rows written by this step replace what the copy
            // brought; its V rows the copy did not fill are zeroed (their
            // probability is 0, and 0 * stale could be NaN)
            for (int r = 0; r < p.R; r++) {
                const int slot = p0 + r - tb;
                if (slot < tw || slot >= tw + 16 || slot >= nvalid || !page_ok) continue;
                for (int d = lane; d < HD; d += 32) {
                    if constexpr (F8) {
                        sk[land_off<HD>(slot, d)] = newk[r * HD + d];
                        sv[land_off<HD>(slot, d)] = newv[r * HD + d];
                    } else {
                        *reinterpret_cast<__half *>(sk + kv_off<HD>(slot, d)) = reinterpret_cast<__half *>(newk)[r * HD + d];
                        *reinterpret_cast<__half *>(sv + kv_off<HD>(slot, d)) = reinterpret_cast<__half *>(newv)[r * HD + d];
                    }
                }
            }
            // a token's row is HD / 16 (E4M3) or HD / 8 (fp16) 16-byte chunks: zero them whole
            constexpr int RC = HD * EB / 16;
            for (int e = lane; e < 16 * RC; e += 32) {
                const int T = tw + e / RC, c = e % RC;
                if (T >= nvalid || !page_ok) {
                    const uint32_t o16 = F8 ? static_cast<uint32_t>(T * HD + c * 16)
                                            : static_cast<uint32_t>((((T >> 4) * (HD / 64) + (c >> 3)) << 11) +
                                                                    ((T & 15) << 7) + ((c & 7) << 4));
                    *reinterpret_cast<uint4 *>(sv + o16) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            fence_async_smem();   // a later copy into this stage comes after these writes
            __syncwarp();
        }
        // scores S^T: 16 tokens x NC columns, even and odd k-steps in separate
        // accumulators (two shorter MMA chains)
        float c[2][NQT][4];
#pragma unroll
        for (int e = 0; e < 2; e++)
#pragma unroll
            for (int nt = 0; nt < NQT; nt++)
#pragma unroll
                for (int i = 0; i < 4; i++) c[e][nt][i] = 0.0f;
        if constexpr (F8) {
#pragma unroll
            for (int g = 0; g < HD / 64; g++) {
                const uint4 w0 = *reinterpret_cast<const uint4 *>(sk + land_off<HD>(tw + gid, g * 64 + tig * 16));
                const uint4 w1 = *reinterpret_cast<const uint4 *>(sk + land_off<HD>(tw + gid + 8, g * 64 + tig * 16));
                const uint32_t r0[4] = {w0.x, w0.y, w0.z, w0.w}, r1[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    uint32_t a[4];
                    e4m3x4_to_h4(r0[j], a[0], a[2]);
                    e4m3x4_to_h4(r1[j], a[1], a[3]);
#pragma unroll
                    for (int nt = 0; nt < NQT; nt++) mma16816(c[j & 1][nt], a, qb[4 * g + j][nt][0], qb[4 * g + j][nt][1]);
                }
            }
        } else {
            const uint32_t k_a = smem_u32(sk);
            const int ktok = tw + (lane & 7) + ((lane >> 3) & 1) * 8, kd = (lane >> 4) * 8;
#pragma unroll
            for (int kk = 0; kk < NKS; kk++) {
                uint32_t a[4];
                ldsm_x4(a, k_a + kv_off<HD>(ktok, kk * 16 + kd));
#pragma unroll
                for (int nt = 0; nt < NQT; nt++) mma16816(c[kk & 1][nt], a, qb[kk][nt][0], qb[kk][nt][1]);
            }
        }
        // hi + lo columns: this lane's scores of tokens gid (0, 1) and gid + 8
        // (2, 3) for query rows qa, qa + 1
        float sc[4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float c0 = c[0][0][i] + c[1][0][i], c1 = c[0][NQT - 1][i] + c[1][NQT - 1][i];
            sc[i] = NQT == 1 ? c0 + __shfl_xor_sync(0xffffffffu, c0, 2) : c0 + c1;
        }
        const int tokA = tw + gid, tokB = tokA + 8;
        float corr[2], pr[4];
#pragma unroll
        for (int j = 0; j < 2; j++) {
            const int qi = qa + j;
            const int lim = (qi < p.Q && page_ok) ? min(t1, p0 + qi / p.G + 1) : 0;   // causal limit (exclusive)
            const float vA = tb + tokA < lim ? sc[j] * p.scale2 : -INFINITY;
            const float vB = tb + tokB < lim ? sc[2 + j] * p.scale2 : -INFINITY;
            float mx = fmaxf(vA, vB);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float m_new = fmaxf(m_q[j], mx);
            corr[j] = (m_q[j] == -INFINITY) ? 0.0f : exp2f(m_q[j] - m_new);
            m_q[j] = m_new;
            pr[j] = (vA == -INFINITY) ? 0.0f : exp2f(vA - m_new);
            pr[2 + j] = (vB == -INFINITY) ? 0.0f : exp2f(vB - m_new);
            l_q[j] = l_q[j] * corr[j] + (pr[j] + pr[2 + j]);
        }
        if (__any_sync(0xffffffffu, corr[0] != 1.0f || corr[1] != 1.0f)) {
#pragma unroll
            for (int mt = 0; mt < NMT; mt++)
#pragma unroll
                for (int nt = 0; nt < NQT; nt++) {
                    ot[mt][nt][0] *= corr[0];
                    ot[mt][nt][1] *= corr[1];
                    ot[mt][nt][2] *= corr[0];
                    ot[mt][nt][3] *= corr[1];
                }
        }
        // P^T [cols][k] as fp16 hi and lo parts (one part per lane when NQT is
        // 1: lanes tig and tig ^ 2 hold the same probabilities)
        {
            const int kA = F8 ? ag_tidx_f8(gid) : gid, kB = F8 ? ag_tidx_f8(gid + 8) : gid + 8;
#pragma unroll
            for (int j = 0; j < 2; j++) {
                __half hA, lA, hB, lB;
                split_f16(pr[j], hA, lA);
                split_f16(pr[2 + j], hB, lB);
                if constexpr (NQT == 1) {
                    const bool lo = tig >= 2;
                    __half *row = pw + ((lo ? QP : 0) + qa + j) * AG_PST;
                    row[kA] = lo ? lA : hA;
                    row[kB] = lo ? lB : hB;
                } else {
                    pw[(qa + j) * AG_PST + kA] = hA;
                    pw[(qa + j) * AG_PST + kB] = hB;
                    pw[(QP + qa + j) * AG_PST + kA] = lA;
                    pw[(QP + qa + j) * AG_PST + kB] = lB;
                }
            }
        }
        __syncwarp();
        uint32_t pb[NQT][2];
        {
            const int l8 = lane & 7, i4 = lane >> 3;
            if constexpr (NQT == 1) {
                ldsm_x2(pb[0][0], pb[0][1], smem_u32(pw + l8 * AG_PST + (i4 & 1) * 8));
            } else {
                uint32_t r4[4];
                ldsm_x4(r4, smem_u32(pw + ((i4 >> 1) * 8 + l8) * AG_PST + (i4 & 1) * 8));
                pb[0][0] = r4[0];
                pb[0][1] = r4[1];
                pb[NQT - 1][0] = r4[2];
                pb[NQT - 1][1] = r4[3];
            }
        }
        // O^T += V^T P^T over this warp's 16 tokens
        if constexpr (F8) {
#pragma unroll
            for (int u = 0; u < HD / 32; u++) {
                uint32_t W[4];
#pragma unroll
                for (int j = 0; j < 4; j++)
                    W[j] = *reinterpret_cast<const uint32_t *>(sv + land_off<HD>(tw + 4 * tig + j, u * 32 + 4 * gid));
                // bytes (dim 4 gid + i) of tokens 4 tig + j: m-tile 2u takes dims
                // i = 0 (row gid) and 1 (row gid + 8), m-tile 2u + 1 dims 2 and 3
                const uint32_t x01 = ag_prmt(W[0], W[1], 0x5140u), y01 = ag_prmt(W[0], W[1], 0x7362u);
                const uint32_t x23 = ag_prmt(W[2], W[3], 0x5140u), y23 = ag_prmt(W[2], W[3], 0x7362u);
                uint32_t a[4];
                e4m3x4_to_h4(x01, a[0], a[1]);
                e4m3x4_to_h4(x23, a[2], a[3]);
#pragma unroll
                for (int nt = 0; nt < NQT; nt++) mma16816(ot[2 * u][nt], a, pb[nt][0], pb[nt][1]);
                e4m3x4_to_h4(y01, a[0], a[1]);
                e4m3x4_to_h4(y23, a[2], a[3]);
#pragma unroll
                for (int nt = 0; nt < NQT; nt++) mma16816(ot[2 * u + 1][nt], a, pb[nt][0], pb[nt][1]);
            }
        } else {
            const uint32_t v_a = smem_u32(sv);
            const int vtok = tw + (lane & 7) + ((lane >> 4) & 1) * 8, vd = ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int mt = 0; mt < NMT; mt++) {
                uint32_t a[4];
                ldsm_x4_t(a, v_a + kv_off<HD>(vtok, mt * 16 + vd));
#pragma unroll
                for (int nt = 0; nt < NQT; nt++) mma16816(ot[mt][nt], a, pb[nt][0], pb[nt][1]);
            }
        }
        // this warp is done with the stage: release it to the producer
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
    }

    // ---- 4. merge the warps: hi + lo columns, sums over the warp's tokens,
    //         then every warp's output weighted by exp(m_w - M) into the drained
    //         ring and summed in warp order into s_o [Q][HD], s_m, s_l
#pragma unroll
    for (int j = 0; j < 2; j++) {
        l_q[j] += __shfl_xor_sync(0xffffffffu, l_q[j], 4);
        l_q[j] += __shfl_xor_sync(0xffffffffu, l_q[j], 8);
        l_q[j] += __shfl_xor_sync(0xffffffffu, l_q[j], 16);
    }
    float o2[NMT][4];
#pragma unroll
    for (int mt = 0; mt < NMT; mt++)
#pragma unroll
        for (int i = 0; i < 4; i++)
            o2[mt][i] = NQT == 1 ? ot[mt][0][i] + __shfl_xor_sync(0xffffffffu, ot[mt][0][i], 2)
                                 : ot[mt][0][i] + ot[mt][NQT - 1][i];
    const bool writer = NQT == 2 || tig < 2;            // one lane per (row, query) pair
    if (writer && gid == 0) {
#pragma unroll
        for (int j = 0; j < 2; j++) {
            s_mw[warp * AG_MAXQ + qa + j] = m_q[j];
            s_lw[warp * AG_MAXQ + qa + j] = l_q[j];
        }
    }
    ag_sync<AG_CT>();   // also: every warp is done with the ring
    float *s_o = reinterpret_cast<float *>(sm);         // [Q][HD] unnormalized output
    float *s_m = s_o + ATT_MAXQ * HD;                   // [Q]
    float *s_l = s_m + ATT_MAXQ;                        // [Q]
    float *scr = reinterpret_cast<float *>(sm + ag_scratch_off<HD>());   // [CW][QP][HD]
    if (writer) {
        float wgt[2];
#pragma unroll
        for (int j = 0; j < 2; j++) {
            float M = -INFINITY;
#pragma unroll
            for (int w2 = 0; w2 < AG_CW; w2++) M = fmaxf(M, s_mw[w2 * AG_MAXQ + qa + j]);
            wgt[j] = (m_q[j] == -INFINITY) ? 0.0f : exp2f(m_q[j] - M);
        }
#pragma unroll
        for (int mt = 0; mt < NMT; mt++)
#pragma unroll
            for (int h = 0; h < 2; h++) {
                // O^T row gid + 8h of m-tile mt is dim d
                const int d = F8 ? (mt >> 1) * 32 + 4 * gid + 2 * (mt & 1) + h : mt * 16 + gid + 8 * h;
#pragma unroll
                for (int j = 0; j < 2; j++) scr[(warp * QP + qa + j) * HD + d] = o2[mt][2 * h + j] * wgt[j];
            }
    }
    ag_sync<AG_CT>();
    // a non-leader split of a cluster writes its partial straight into the
    // leader's receive slot (stores that count down the leader's barrier)
    const bool pusher = p.cluster && split != 0;
    uint32_t slot_a = 0, mrecv_a = 0;
    if (p.cluster) cluster_wait_acq();   // every CTA of the cluster has its barriers
    if (pusher) {
        slot_a = ag_mapa(smem_u32(rcv + (split - 1) * ag_slot_floats(p.Q, HD)), 0);
        mrecv_a = ag_mapa(smem_u32(mrecv), 0);
    }
    for (int e4 = tid; e4 < p.Q * (HD / 4); e4 += AG_CT) {
        const int qi = e4 / (HD / 4), d = (e4 - qi * (HD / 4)) * 4;
        float4 o = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
        for (int w2 = 0; w2 < AG_CW; w2++) {
            const float4 v = *reinterpret_cast<const float4 *>(scr + (w2 * QP + qi) * HD + d);
            o.x += v.x;
            o.y += v.y;
            o.z += v.z;
            o.w += v.w;
        }
        if (pusher)
            st_async_v4(slot_a + static_cast<uint32_t>(e4) * 16, o, mrecv_a);
        else
            *reinterpret_cast<float4 *>(s_o + qi * HD + d) = o;
    }
    if (tid < p.Q) {
        float M = -INFINITY;
#pragma unroll
        for (int w2 = 0; w2 < AG_CW; w2++) M = fmaxf(M, s_mw[w2 * AG_MAXQ + tid]);
        float L = 0.0f;
#pragma unroll
        for (int w2 = 0; w2 < AG_CW; w2++) {
            const float m2 = s_mw[w2 * AG_MAXQ + tid];
            L += (m2 == -INFINITY) ? 0.0f : s_lw[w2 * AG_MAXQ + tid] * exp2f(m2 - M);
        }
        if (pusher) {
            st_async_v2(slot_a + static_cast<uint32_t>(p.Q * HD + 2 * tid) * 4, M, L, mrecv_a);
        } else {
            s_m[tid] = M;
            s_l[tid] = L;
        }
    }
    if (pusher) {
        // stay (with the stores in flight) until the leader holds all of them
        mbar_wait(mack, 0, p.err);
        return;
    }
    ag_sync<AG_CT>();

    // ---- 5. the output, or a partial for the split combine
    if (p.cluster) {
        // the cluster's leader: every split's partial is in shared memory
        // (its own in s_o, s_m, s_l; the others in the receive slots); the
        // splits are combined in split order
        const int ns = p.n_split, SF = ag_slot_floats(p.Q, HD);
        mbar_wait(mrecv, 0, p.err);
        {
            // the other splits may leave: their partials are all here
            const int r = tid - (AG_CT - 32);
            if (r >= 1 && r < ns) mbar_arrive_remote(ag_mapa(smem_u32(mack), static_cast<uint32_t>(r)));
        }
        // split r's (max, sum) of query row qi
        auto m_of = [&](int r, int qi) { return r == 0 ? s_m[qi] : rcv[(r - 1) * SF + p.Q * HD + 2 * qi]; };
        auto l_of = [&](int r, int qi) { return r == 0 ? s_l[qi] : rcv[(r - 1) * SF + p.Q * HD + 2 * qi + 1]; };
        float *s_w = s_l + ATT_MAXQ;                  // [ns][Q] weights 2^(m_r - M)
        if (tid < ns * p.Q) {
            const int r = tid / p.Q, qi = tid - r * p.Q;
            float M = -INFINITY;
#pragma unroll
            for (int r2 = 0; r2 < ATT_MAXCL; r2++)
                if (r2 < ns) M = fmaxf(M, m_of(r2, qi));
            const float m = m_of(r, qi);
            s_w[tid] = (m == -INFINITY) ? 0.0f : exp2f(m - M);
        }
        ag_sync<AG_CT>();
        // four dims of one query row per thread; sums in split order
        const float4 *rcv4 = reinterpret_cast<const float4 *>(rcv);
        for (int e4 = tid; e4 < p.Q * (HD / 4); e4 += AG_CT) {
            const int qi = e4 / (HD / 4), d = (e4 - qi * (HD / 4)) * 4;
            float L = 0.0f;
            float4 O = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            for (int r0 = 0; r0 < ns; r0 += 4) {
                // four splits' loads in flight, then their terms in order
                float wv[4], lv[4];
                float4 ov[4];
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const int r2 = r0 + u;
                    if (r2 < ns) {
                        wv[u] = s_w[r2 * p.Q + qi];
                        lv[u] = l_of(r2, qi);
                        ov[u] = r2 == 0 ? *reinterpret_cast<const float4 *>(s_o + qi * HD + d)
                                        : rcv4[((r2 - 1) * SF) / 4 + e4];
                    }
                }
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    if (r0 + u < ns) {
                        L = fmaf(lv[u], wv[u], L);
                        O.x = fmaf(ov[u].x, wv[u], O.x);
                        O.y = fmaf(ov[u].y, wv[u], O.y);
                        O.z = fmaf(ov[u].z, wv[u], O.z);
                        O.w = fmaf(ov[u].w, wv[u], O.w);
                    }
                }
            }
            const int r = qi / p.G, gq = qi - r * p.G;
            const float vs = p.vscale;
            *reinterpret_cast<float4 *>(p.out + (static_cast<size_t>(b) * p.R + r) * (static_cast<size_t>(p.nq) * HD) +
                                        static_cast<size_t>(kvh * p.G + gq) * HD + d) =
                make_float4((O.x * vs) / L, (O.y * vs) / L, (O.z * vs) / L, (O.w * vs) / L);
        }
        return;
    }
    const size_t pbase = (static_cast<size_t>(b) * p.nkv + kvh) * p.n_split;
    if (p.n_split == 1) {
        for (int e = tid; e < p.Q * (HD / 4); e += AG_CT) {
            const int qi = e / (HD / 4), d = (e - qi * (HD / 4)) * 4;
            const int r = qi / p.G, gq = qi - r * p.G;
            const float4 o = *reinterpret_cast<const float4 *>(s_o + qi * HD + d);
            const float L = s_l[qi], vs = p.vscale;
            *reinterpret_cast<float4 *>(p.out + (static_cast<size_t>(b) * p.R + r) * (static_cast<size_t>(p.nq) * HD) +
                                        static_cast<size_t>(kvh * p.G + gq) * HD + d) =
                make_float4((o.x * vs) / L, (o.y * vs) / L, (o.z * vs) / L, (o.w * vs) / L);
        }
        return;
    }
    for (int e = tid; e < p.Q * (HD / 4); e += AG_CT) {
        const int qi = e / (HD / 4), d = (e - qi * (HD / 4)) * 4;
        __stcg(reinterpret_cast<float4 *>(p.part_o + ((pbase + split) * p.Q + qi) * HD + d),
               *reinterpret_cast<const float4 *>(s_o + qi * HD + d));
    }
    if (tid < p.Q)
        __stcg(reinterpret_cast<float2 *>(p.part_ml + ((pbase + split) * p.Q + tid) * 2), make_float2(s_m[tid], s_l[tid]));
    // the last split of this (sequence, kv head) to finish combines all of them
    fence_acq_rel_gpu();
    ag_sync<AG_CT>();
    uint32_t *cnt = p.cnt + static_cast<size_t>(b) * p.nkv + kvh;
    if (tid == 0) s_last = atomicAdd(cnt, 1u) == static_cast<uint32_t>(p.n_split - 1);
    ag_sync<AG_CT>();
    if (!s_last) return;
    fence_acq_rel_gpu();
    const int ns = p.n_split;
    float *s_w = reinterpret_cast<float *>(sm);            // [ns][Q] max, then weight (the ring is free)
    float *s_sl = s_w + ATT_MAXNS * ATT_MAXQ;              // [ns][Q] sums
    float *s_L = s_sl + ATT_MAXNS * ATT_MAXQ;              // [Q]
    for (int e = tid; e < ns * p.Q; e += AG_CT) {
        const float2 ml = __ldcg(reinterpret_cast<const float2 *>(p.part_ml + (pbase * p.Q + e) * 2));
        s_w[e] = ml.x;
        s_sl[e] = ml.y;
    }
    ag_sync<AG_CT>();
    if (tid < p.Q) {
        const int qi = tid;
        float M = -INFINITY;
        for (int r2 = 0; r2 < ns; r2++) M = fmaxf(M, s_w[r2 * p.Q + qi]);
        float L = 0.0f;
        for (int r2 = 0; r2 < ns; r2++) {
            const float m2 = s_w[r2 * p.Q + qi];
            const float w = (m2 == -INFINITY) ? 0.0f : exp2f(m2 - M);
            s_w[r2 * p.Q + qi] = w;
            L = fmaf(s_sl[r2 * p.Q + qi], w, L);
        }
        s_L[qi] = L;
    }
    ag_sync<AG_CT>();
    for (int e = tid; e < p.Q * (HD / 4); e += AG_CT) {
        const int qi = e / (HD / 4), d = (e - qi * (HD / 4)) * 4;
        const float4 *src = reinterpret_cast<const float4 *>(p.part_o + (pbase * p.Q + qi) * HD + d);
        const size_t stride = static_cast<size_t>(p.Q) * HD / 4;
        float4 O = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll 16
        for (int r2 = 0; r2 < ns; r2++) {
            const float4 v = __ldcg(src + r2 * stride);
            const float w = s_w[r2 * p.Q + qi];
            O.x = fmaf(v.x, w, O.x);
            O.y = fmaf(v.y, w, O.y);
            O.z = fmaf(v.z, w, O.z);
            O.w = fmaf(v.w, w, O.w);
        }
        const int r = qi / p.G, gq = qi - r * p.G;
        const float L = s_L[qi];
        float *dst = p.out + (static_cast<size_t>(b) * p.R + r) * (static_cast<size_t>(p.nq) * HD) +
                     static_cast<size_t>(kvh * p.G + gq) * HD + d;
        const float vs = p.vscale;
        *reinterpret_cast<float4 *>(dst) = make_float4((O.x * vs) / L, (O.y * vs) / L, (O.z * vs) / L, (O.w * vs) / L);
    }
    ag_sync<AG_CT>();
    if (tid == 0) *cnt = 0u;
}

// Splits per (sequence, kv head).  Many (sequence, kv head) groups: one
// split, the grid already fills the GPU.  Few: about sqrt(pages) splits --
// a split streams pages/ns pages, the merge reads ns partials -- bounded so
// that every CTA has an SM (and a deep ring) to itself.
static int attn_splits(int B, int nkv, int max_pages) {
    const int groups = B * nkv;
    if (groups >= sm_count()) return 1;
    int ns = static_cast<int>(sqrt(static_cast<double>(max_pages)) + 0.5);
    ns = min(ns, sm_count() / groups);
    ns = min(ns, max(1, max_pages / 4));
    return max(1, min(ns, ATT_MAXNS));
}

size_t attn_scratch_bytes(int B, int R, int nq, int nkv, int hd, int max_pages) {
    const int ns = attn_splits(B, nkv, max_pages);
    if (ns == 1) return 0;
    const size_t Q = static_cast<size_t>(nq / max(1, nkv)) * R;
    return align_up(static_cast<size_t>(B) * nkv * ns * Q * hd * 4, BW_WS_ALIGN) +
           align_up(static_cast<size_t>(B) * nkv * ns * Q * 2 * 4, BW_WS_ALIGN);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// dependency on the driver library); encoded maps are cached per pool.
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::mutex mu;   // host threads may call the library concurrently
    std::lock_guard<std::mutex> lk(mu);
    if (!fn) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            (void)cudaGetLastError();
            return nullptr;
        }
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

// fp16 pools: boxes of 16 rows x 64 dims with the 128-byte swizzle; E4M3
// pools (f8): boxes of 16 rows x hd bytes with the hd-byte swizzle (128 or 64).
static bool kv_tensor_map(CUtensorMap *out, void *pool, int n_pages, int nkv, int hd, bool f8) {
    struct Entry {
        void *pool;
        int rows, hd;
        bool f8;
        CUtensorMap map;
    };
    static Entry cache[512];
    static int n_cache = 0, next = 0;
    static std::mutex mu;   // host threads may call the library concurrently
    std::lock_guard<std::mutex> lk(mu);
    const int rows = n_pages * nkv * 16;
    for (int i = 0; i < n_cache; i++)
        if (cache[i].pool == pool && cache[i].rows == rows && cache[i].hd == hd && cache[i].f8 == f8) {
            *out = cache[i].map;
            return true;
        }
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(hd), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(hd) * (f8 ? 1 : 2)};
    const cuuint32_t box[2] = {f8 ? static_cast<cuuint32_t>(hd) : 64u, 16};
    const cuuint32_t estr[2] = {1, 1};
    CUtensorMap m;
    if (fn(&m, f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, pool, dims, strides, box,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, (f8 && hd == 64) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    Entry &e = cache[n_cache < 512 ? n_cache++ : (next++ % 512)];
    e.pool = pool;
    e.rows = rows;
    e.hd = hd;
    e.f8 = f8;
    e.map = m;
    *out = m;
    return true;
}

template <int HD, int MT, int NST, int F8>
static bw_status attn_go(int ns, int nkv, int B, cudaStream_t st, const AttnParams &p) {
    const size_t smem = att_smem_fixed<HD, MT, NST, F8>() + static_cast<size_t>(p.max_pages) * 4;
    static size_t attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return BW_ERR_CUDA;
    AttnParams q = p;
    q.n_split = ns;
    q.cluster = (ns > 1 && ns <= ATT_MAXCL && NST == 4) ? 1 : 0;
    {
        static bool cl_set[64] = {};
        static std::mutex mu;   // host threads may call the library concurrently
        std::lock_guard<std::mutex> lk(mu);
        if (attr_set[dev] < smem) {
            if (cudaFuncSetAttribute(attn_kernel<HD, MT, NST, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem)) != cudaSuccess) {
                (void)cudaGetLastError();
                return BW_ERR_CUDA;
            }
            attr_set[dev] = smem;
        }
        if (q.cluster && !cl_set[dev]) {
            if (cudaFuncSetAttribute(attn_kernel<HD, MT, NST, F8>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                cudaSuccess) {
                (void)cudaGetLastError();
                return BW_ERR_CUDA;
            }
            cl_set[dev] = true;
        }
    }
    if (!q.cluster) return launch_pdl(attn_kernel<HD, MT, NST, F8>, dim3(ns, nkv, B), dim3(ATT_THREADS), smem, st, q);
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
    if (cudaLaunchKernelEx(&cfg, attn_kernel<HD, MT, NST, F8>, q) != cudaSuccess) {
        (void)cudaGetLastError();
        return BW_ERR_CUDA;
    }
    return BW_OK;
}

template <int HD, int MT, int F8>
static bw_status attn_go_st(int ns, int nkv, int B, cudaStream_t st, const AttnParams &p) {
    // a grid that fits one CTA per SM gets the deep ring, where it fits shared memory
    const bool fits = att_smem_fixed<HD, MT, 4, F8>() + static_cast<size_t>(p.max_pages) * 4 <= 227 * 1024 - 1024;
    return static_cast<long>(ns) * nkv * B <= sm_count() && fits ? attn_go<HD, MT, 4, F8>(ns, nkv, B, st, p)
                                                                 : attn_go<HD, MT, 2, F8>(ns, nkv, B, st, p);
}

template <int HD, int NQT, int NST, int F8, int CW>
static bw_status attn_g_go(int ns, int nkv, int B, bool cl, cudaStream_t st, const AttnParams &p) {
    const size_t base = ag_smem_fixed<HD, NQT, NST, F8, CW>() + static_cast<size_t>(p.max_pages) * 4;
    // the cluster leader's receive area must fit next to the ring; otherwise
    // the splits combine through the workspace
    if (cl && base + ag_recv_bytes(ns, p.Q, HD) > 227 * 1024) cl = false;
    const size_t smem = base + (cl ? ag_recv_bytes(ns, p.Q, HD) : 0);
    if (smem > 227 * 1024) return BW_ERR_UNSUPPORTED_SHAPE;
    static size_t attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return BW_ERR_CUDA;
    AttnParams q = p;
    q.n_split = ns;
    q.cluster = cl ? 1 : 0;
    {
        static bool cl_set[64] = {};
        static std::mutex mu;   // host threads may call the library concurrently
        std::lock_guard<std::mutex> lk(mu);
        if (attr_set[dev] < smem) {
            if (cudaFuncSetAttribute(attn_g_kernel<HD, NQT, NST, F8, CW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem)) != cudaSuccess) {
                (void)cudaGetLastError();
                return BW_ERR_CUDA;
            }
            attr_set[dev] = smem;
        }
        if (cl && !cl_set[dev]) {
            if (cudaFuncSetAttribute(attn_g_kernel<HD, NQT, NST, F8, CW>, cudaFuncAttributeNonPortableClusterSizeAllowed,
                                     1) != cudaSuccess) {
                (void)cudaGetLastError();
                return BW_ERR_CUDA;
            }
            cl_set[dev] = true;
        }
    }
    if (!cl) return launch_pdl(attn_g_kernel<HD, NQT, NST, F8, CW>, dim3(ns, nkv, B), dim3((CW + 1) * 32), smem, st, q);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ns, nkv, B);
    cfg.blockDim = dim3((CW + 1) * 32);
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
    if (cudaLaunchKernelEx(&cfg, attn_g_kernel<HD, NQT, NST, F8, CW>, q) != cudaSuccess) {
        (void)cudaGetLastError();
        return BW_ERR_CUDA;
    }
    return BW_OK;
}

// Shape of the token-on-M kernel.  When every CTA has an SM to itself: 8
// consumer warps (stages of 8 pages) and, for 2..16 splits, a cluster merge;
// otherwise 4 consumer warps and two CTAs per SM.  Ring: 2 stages of fp16,
// or 4 of E4M3 (half the bytes).
template <int HD, int NQT, int F8>
static bw_status attn_g_st(int ns, int nkv, int B, cudaStream_t st, const AttnParams &p) {
    const bool deep = static_cast<long>(ns) * nkv * B <= sm_count();
    const bool cl = deep && ns > 1 && ns <= ATT_MAXCL;
    constexpr int NST = F8 ? 4 : 2;
    return deep ? attn_g_go<HD, NQT, NST, F8, 8>(ns, nkv, B, cl, st, p)
                : attn_g_go<HD, NQT, NST, F8, 4>(ns, nkv, B, cl, st, p);
}

bw_status attn_check(const float *qkv, const float *rope_cos, const float *rope_sin, int rope_max_pos,
                     const void *k_pool, const void *v_pool, const int32_t *page_table, int max_pages, int n_pages,
                     const int32_t *pos, int B, int R, int nq, int nkv, int hd, const float *out, const Scratch &sc) {
    if (!qkv || !rope_cos || !rope_sin || !k_pool || !v_pool || !page_table || !pos || !out || !sc.cnt)
        return BW_ERR_INVALID_ARG;
    if (B <= 0 || R <= 0 || nq <= 0 || nkv <= 0 || max_pages <= 0 || n_pages <= 0 || rope_max_pos <= 0)
        return BW_ERR_INVALID_ARG;
    if ((hd != 128 && hd != 64) || nq % nkv || (nq / nkv) * R > ATT_MAXQ || R > ATT_MAXR)
        return BW_ERR_UNSUPPORTED_SHAPE;
    if (max_pages > ATT_MAXPAGES) return BW_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(k_pool) || !aligned16(v_pool) || !aligned16(qkv) || !aligned16(out)) return BW_ERR_INVALID_ARG;
    if (nkv > 65535 || B > 65535) return BW_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<size_t>(B) * nkv > 65536 - CNT_ATTN - 16) return BW_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<long long>(n_pages) * nkv * 16 > 0xffffffffLL) return BW_ERR_UNSUPPORTED_SHAPE;
    if (sc.bytes < attn_scratch_bytes(B, R, nq, nkv, hd, max_pages)) return BW_ERR_INVALID_ARG;
    return BW_OK;
}

bw_status attn_launch(const float *qkv, const float *rope_cos, const float *rope_sin, int rope_max_pos,
                      void *k_pool, void *v_pool, const int32_t *page_table, int max_pages,
                      int n_pages, const int32_t *pos, int B, int R, int nq, int nkv, int hd,
                      float *out, const Scratch &sc, cudaStream_t st, int kv_fmt, float kscale, float vscale,
                      bool early) {
    if (kv_fmt != 0 && kv_fmt != 1) return BW_ERR_INVALID_ARG;
    if (kv_fmt == 1 && !(kscale > 0.0f && vscale > 0.0f && isfinite(kscale) && isfinite(vscale)))
        return BW_ERR_INVALID_ARG;
    const bool f8 = kv_fmt == 1;
    const bw_status chk = attn_check(qkv, rope_cos, rope_sin, rope_max_pos, k_pool, v_pool, page_table, max_pages,
                                     n_pages, pos, B, R, nq, nkv, hd, out, sc);
    if (chk != BW_OK) return chk;
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
    p.kscale = f8 ? kscale : 1.0f;
    p.vscale = f8 ? vscale : 1.0f;
    if (f8) p.scale = p.scale * kscale;
    // the token-on-M kernel's softmax runs in base 2: scores times log2(e)
    p.scale2 = static_cast<float>(static_cast<double>(p.scale) * 1.4426950408889634);
    p.out = out;
    p.err = sc.err;
    p.cnt = sc.cnt + CNT_ATTN;
    p.cluster = 0;
    p.early = early ? 1 : 0;
    if (!kv_tensor_map(&p.tmk, k_pool, n_pages, nkv, hd, f8) || !kv_tensor_map(&p.tmv, v_pool, n_pages, nkv, hd, f8))
        return BW_ERR_CUDA;
    const int ns = attn_splits(B, nkv, max_pages);
    Carver cv(sc.base);
    p.part_o = ns > 1 ? cv.take<float>(static_cast<size_t>(B) * nkv * ns * p.Q * hd) : nullptr;
    p.part_ml = ns > 1 ? cv.take<float>(static_cast<size_t>(B) * nkv * ns * p.Q * 2) : nullptr;
    if (p.Q <= AG_MAXQ) {
        // up to 8 query rows: the token-on-M kernel
        if (f8) {
            if (hd == 128)
                return p.Q <= 4 ? attn_g_st<128, 1, 1>(ns, nkv, B, st, p) : attn_g_st<128, 2, 1>(ns, nkv, B, st, p);
            return p.Q <= 4 ? attn_g_st<64, 1, 1>(ns, nkv, B, st, p) : attn_g_st<64, 2, 1>(ns, nkv, B, st, p);
        }
        if (hd == 128)
            return p.Q <= 4 ? attn_g_st<128, 1, 0>(ns, nkv, B, st, p) : attn_g_st<128, 2, 0>(ns, nkv, B, st, p);
        return p.Q <= 4 ? attn_g_st<64, 1, 0>(ns, nkv, B, st, p) : attn_g_st<64, 2, 0>(ns, nkv, B, st, p);
    }
    if (f8) {
        if (hd == 128)
            return p.Q <= 16 ? attn_go_st<128, 1, 1>(ns, nkv, B, st, p) : attn_go_st<128, 2, 1>(ns, nkv, B, st, p);
        return p.Q <= 16 ? attn_go_st<64, 1, 1>(ns, nkv, B, st, p) : attn_go_st<64, 2, 1>(ns, nkv, B, st, p);
    }
    if (hd == 128) return p.Q <= 16 ? attn_go_st<128, 1, 0>(ns, nkv, B, st, p) : attn_go_st<128, 2, 0>(ns, nkv, B, st, p);
    return p.Q <= 16 ? attn_go_st<64, 1, 0>(ns, nkv, B, st, p) : attn_go_st<64, 2, 0>(ns, nkv, B, st, p);
}

}  // namespace bw

extern "C" {

bw_status bw_paged_attn_decode(const float *qkv, const float *rope_cos, const float *rope_sin,
                               int rope_max_pos, void *k_pool, void *v_pool,
                               const int32_t *page_table, int max_pages, int n_pages,
                               const int32_t *pos, int B, int n_rows, int nq, int nkv, int hd,
                               float *out, void *ws, size_t ws_bytes, void *stream) {
    if (!bw::ws_ok(ws)) return BW_ERR_INVALID_ARG;
    return bw::attn_launch(qkv, rope_cos, rope_sin, rope_max_pos, k_pool, v_pool, page_table,
                           max_pages, n_pages, pos, B, n_rows, nq, nkv, hd, out,
                           bw::scratch_of(ws, ws_bytes), static_cast<cudaStream_t>(stream), 0, 1.0f, 1.0f);
}

bw_status bw_paged_attn_decode_fp8(const float *qkv, const float *rope_cos, const float *rope_sin,
                                   int rope_max_pos, void *k_pool, void *v_pool, float k_scale, float v_scale,
                                   const int32_t *page_table, int max_pages, int n_pages,
                                   const int32_t *pos, int B, int n_rows, int nq, int nkv, int hd,
                                   float *out, void *ws, size_t ws_bytes, void *stream) {
    if (!bw::ws_ok(ws)) return BW_ERR_INVALID_ARG;
    return bw::attn_launch(qkv, rope_cos, rope_sin, rope_max_pos, k_pool, v_pool, page_table,
                           max_pages, n_pages, pos, B, n_rows, nq, nkv, hd, out,
                           bw::scratch_of(ws, ws_bytes), static_cast<cudaStream_t>(stream), 1, k_scale, v_scale);
}

size_t bw_attn_workspace_bytes(int B, int n_rows, int nq, int nkv, int hd, int max_pages) {
    if (B <= 0 || n_rows <= 0 || nq <= 0 || nkv <= 0 || hd <= 0 || max_pages <= 0 || nq % nkv)
        return BW_WS_HDR_BYTES;
    return BW_WS_HDR_BYTES + bw::attn_scratch_bytes(B, n_rows, nq, nkv, hd, max_pages);
}

}  // extern "C"
