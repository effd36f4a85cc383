// gemv_core.cuh -- device core shared by the dense and the grouped-expert
// dequant-GEMV kernels (sm_100a): the tiled weight layout, the stage
// pipeline helpers, the 4-bit dequant-dot inner loop and the lane
// reduction.
//
// Tiled GPU layout (written by the repack kernels).  A matrix W[N][K] is cut
// into tiles of 128 rows x 512 columns (16 chunks of 32 columns); N is padded
// to a multiple of 128 rows and K to a multiple of 512 columns with zeros.
// Tile (rb, kt) of the codes is one contiguous 32 KB block: row r of the tile
// at r*256 bytes, chunk c of that row in 16-byte slot c ^ (r & 7) (the 16
// code bytes of the chunk in the canonical nibble order).  The XOR keeps both
// access patterns free of shared-memory bank conflicts: 16 lanes reading the
// 16 chunks of one row, and 8 lanes reading one chunk of 8 consecutive rows.  Tile (rb, kt) of the scales is one
// contiguous 4 KB block: row group g (rows 8g..8g+7 of the tile) at g*256,
// chunk c at +c*16: the 8 rows' fp16 d (Q4_0) or 8 x 2 E4M3 block scales
// (NVFP4).  Tiles follow each other in (rb, kt) order.  Every pipeline stage
// is therefore two plain contiguous bulk copies that stream at full HBM
// rate.
#pragma once

#include <math.h>

#include "bw_common.cuh"

namespace bw {

constexpr int GV_CW = 8;                          // consumer warps
constexpr int GV_THREADS = (GV_CW + 1) * 32;      // + one producer warp
constexpr int GV_MAX_M = 4;
constexpr int GV_TR = 128;                        // tile rows (16 row groups)
constexpr int GV_TC = 16;                         // tile chunks (of 32 columns)
constexpr uint32_t GV_NIB_BYTES = GV_TR * GV_TC * 16;        // 32 KB
constexpr uint32_t GV_SC_BYTES = (GV_TR / 8) * GV_TC * 16;   // 4 KB
constexpr uint32_t GV_STAGE_BYTES = GV_NIB_BYTES + GV_SC_BYTES;

__host__ __device__ constexpr int gv_row_blocks(int N) { return (N + GV_TR - 1) / GV_TR; }
__host__ __device__ constexpr int gv_col_tiles(int K) { return (K / 32 + GV_TC - 1) / GV_TC; }

// Producer arrival that only announces the bytes its bulk copies will
// deliver; it publishes no data of its own, so it needs no release fence.
__device__ __forceinline__ void mbar_arrive_tx_relaxed(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.relaxed.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Consumer release of a stage.  Relaxed: every shared-memory load of the
// stage has already been consumed by the arithmetic before this point, so
// the loads are complete and no release fence is needed.
__device__ __forceinline__ void mbar_arrive_relaxed(uint64_t *bar) {
    asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(GV_CW * 32) : "memory");
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// Position of element e (0..31) of a Q4_0 chunk in the kernel's consumption
// order: byte j = e % 16 is word j/4, nibble 2*(j%4), +1 for the high half.
__device__ __forceinline__ int q4_order(int e) {
    const int j = e & 15;
    return 8 * (j >> 2) + 2 * (j & 3) + (e >> 4);
}

// Explicit shared-memory loads (32-bit shared addresses).  Volatile so they
// stay after the mbarrier wait that publishes the stage they read.
__device__ __forceinline__ uint4 lds_u4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ float4 lds_f4(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ float lds_f(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
    return v;
}

// Loads the 16-byte elements [0, n4) of a row, a batch of 8 independent
// loads per thread in flight before the first is used; elements
// [lo, lo + n_keep) are also stored to dst[e - lo].  Returns this thread's
// sum of squares over every element it loaded.
__device__ __forceinline__ float stage_row4(const float4 *src, int n4, float4 *dst, int lo, int n_keep, int tid) {
    constexpr int U = 8, STEP = GV_CW * 32;
    float ss = 0.0f;
    for (int b = 0; b < n4; b += U * STEP) {
        float4 v[U];
#pragma unroll
        for (int u = 0; u < U; u++) {
            const int e = b + u * STEP + tid;
            v[u] = e < n4 ? src[e] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
#pragma unroll
        for (int u = 0; u < U; u++) {
            const int d = b + u * STEP + tid - lo;
            if (d >= 0 && d < n_keep) dst[d] = v[u];
            ss = fma_rn(v[u].x, v[u].x, ss);
            ss = fma_rn(v[u].y, v[u].y, ss);
            ss = fma_rn(v[u].z, v[u].z, ss);
            ss = fma_rn(v[u].w, v[u].w, ss);
        }
    }
    return ss;
}

// One-pass staging: loads the 16-byte elements [0, n4) of a row (a batch of
// 8 independent loads per thread in flight) and stores elements
// [lo, lo + n_keep) -- times the gains gt4[e - lo] when gt4 is given -- in the
// staged form of stage_x below: chunk c (8 elements of 16 bytes) at
// xs + 32 c, granules XOR-swizzled by c, Q4_0 values pre-scaled per nibble
// slot and the chunk's -8 term in ct[c].  The 8 elements of a chunk are
// loaded by 8 consecutive lanes (lo is a multiple of 8), which exchange
// halves with the lane 4 apart to form the Q4_0 granules and add up the
// chunk sum.  Returns this thread's sum of squares over every element it
// loaded (before the gains).
template <int FMT>
__device__ __forceinline__ float stage_row_t(const float4 *src, int n4, float *xs, float *ct, const float4 *gt4, int lo,
                                             int n_keep, int tid) {
    constexpr int U = 8, STEP = GV_CW * 32;
    const int j = tid & 7;
    float ss = 0.0f;
    for (int b = 0; b < n4; b += U * STEP) {
        float4 v[U];
#pragma unroll
        for (int u = 0; u < U; u++) {
            const int e = b + u * STEP + tid;
            v[u] = e < n4 ? src[e] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
#pragma unroll
        for (int u = 0; u < U; u++) {
            if (b + u * STEP >= n4) break;   // no lane of the CTA has this element (uniform)
            ss = fma_rn(v[u].x, v[u].x, ss);
            ss = fma_rn(v[u].y, v[u].y, ss);
            ss = fma_rn(v[u].z, v[u].z, ss);
            ss = fma_rn(v[u].w, v[u].w, ss);
            const int d = b + u * STEP + tid - lo;
            const bool keep = d >= 0 && d < n_keep;
            float4 w = keep ? v[u] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (gt4 && keep) {
                const float4 g = gt4[d];
                w = make_float4(w.x * g.x, w.y * g.y, w.z * g.z, w.w * g.w);
            }
            const int c = keep ? d >> 3 : 0;
            if constexpr (FMT == BW_FMT_Q4_0) {
                // lanes j < 4 hold elements 4j .. 4j+3 of the chunk, lanes j >= 4
                // elements 16 + 4(j-4) ..: granule 2j takes (A.x, B.x, A.y, B.y),
                // granule 2j+1 (A.z, B.z, A.w, B.w), A from lane j, B from lane j+4
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
                    // 2^(101 - 4p) for granule slot p
                    *reinterpret_cast<float4 *>(xs + c * 32 + 4 * (G ^ (c & 7))) =
                        make_float4(gr.x * __int_as_float((127 + 101) << 23), gr.y * __int_as_float((127 + 97) << 23),
                                    gr.z * __int_as_float((127 + 93) << 23), gr.w * __int_as_float((127 + 89) << 23));
                    if (j == 0) ct[c] = cs * -2.8421709430404007e-14f;   // -8 * 2^-48
                }
            } else {
                if (keep) *reinterpret_cast<float4 *>(xs + c * 32 + 4 * (j ^ (c & 7))) = w;
            }
        }
    }
    return ss;
}

// Staged activations: chunk c of row m at (m*chunk_stride + c)*128 bytes; its
// 16-byte granule g is stored at granule (g ^ (c & 7)), so 8 lanes reading
// granule g of 8 consecutive chunks hit 8 different bank groups.
__device__ __forceinline__ uint32_t gran_addr(uint32_t chunk_a, int g, int c) {
    return chunk_a + 16u * static_cast<uint32_t>(g ^ (c & 7));
}

// Writes activation value v of element e of local chunk cl (row m) into the
// staged layout: Q4_0 pre-scaled per nibble slot, plus the chunk's -8 term.
template <int FMT>
__device__ __forceinline__ void stage_x(float *xs, float *ct, int chunk_stride, int m, int cl, int lane, float v) {
    float *xc = xs + static_cast<size_t>(m * chunk_stride + cl) * 32;
    if constexpr (FMT == BW_FMT_Q4_0) {
        const int idx = q4_order(lane);
        const float scale = __int_as_float((127 + 101 - 4 * (idx & 3)) << 23);   // 2^(101-4p)
        xc[4 * ((idx >> 2) ^ (cl & 7)) + (idx & 3)] = v * scale;
        const float sum = warp_sum(v);
        if (lane == 0) ct[m * chunk_stride + cl] = sum * -2.8421709430404007e-14f;   // -8 * 2^-48
    } else {
        xc[4 * ((lane >> 2) ^ (cl & 7)) + (lane & 3)] = v;
    }
}

// Second staging pass: the slice's activations sit in natural order at the
// start of each chunk's slot (first pass: one wide burst of independent
// global loads); each warp turns its chunks into the swizzled, pre-scaled
// form in place, applying the RMSNorm (x * rnorm) * gamma when gt != null.
// Two chunks per iteration, so that their loads and lane sums overlap.
template <int FMT, int M>
__device__ __forceinline__ void stage_pass2(float *xs, float *ct, const float *gt, const float *rnorm, int CS,
                                            int nc, int warp, int lane) {
    const int np = M * nc;
    for (int pair = warp; pair < np; pair += 2 * GV_CW) {
        const int pair2 = pair + GV_CW;
        const bool two = pair2 < np;
        const int m = pair / nc, cl = pair - m * nc;
        const int m2 = two ? pair2 / nc : m, cl2 = two ? pair2 - m2 * nc : cl;
        float v = xs[static_cast<size_t>(m * CS + cl) * 32 + lane];
        float v2 = xs[static_cast<size_t>(m2 * CS + cl2) * 32 + lane];
        if (gt) {
            v = (v * rnorm[m]) * gt[cl * 32 + lane];
            v2 = (v2 * rnorm[m2]) * gt[cl2 * 32 + lane];
        }
        __syncwarp();
        stage_x<FMT>(xs, ct, CS, m, cl, lane, v);
        if (two) stage_x<FMT>(xs, ct, CS, m2, cl2, lane, v2);
    }
}

__device__ __forceinline__ uint32_t u4_get(const uint4 &v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// 64-bit helpers: the f32x2 FMA takes register pairs; building every operand
// pair in one 64-bit register (masks applied to {v, v}, activations loaded as
// 64-bit words, accumulators kept as pairs) leaves nothing to re-pair.
__device__ __forceinline__ uint64_t and_pair(uint32_t v, uint64_t mask) {
    uint64_t r;
    asm("{\n\t.reg .b64 vv;\n\tmov.b64 vv, {%1, %1};\n\tand.b64 %0, vv, %2;\n\t}" : "=l"(r) : "r"(v), "l"(mask));
    return r;
}
__device__ __forceinline__ uint64_t ffma2_64(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ void lds_2x64(uint32_t a, uint64_t &lo, uint64_t &hi) {
    asm volatile("ld.shared.v2.u64 {%0, %1}, [%2];" : "=l"(lo), "=l"(hi) : "r"(a));
}
__device__ __forceinline__ uint64_t pair_f(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float pair_sum(uint64_t p) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
    return lo + hi;
}
// E2M1 codes of one byte (low nibble -> low half) as an fp32 pair (exact)
__device__ __forceinline__ uint64_t e2m1x2_pair(uint32_t byte) {
    uint64_t r;
    asm("{\n\t.reg .b8 b;\n\t.reg .b32 p;\n\t.reg .b16 h0, h1;\n\t.reg .f32 f0, f1;\n\t"
        "cvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 p, b;\n\tmov.b32 {h0, h1}, p;\n\t"
        "cvt.f32.f16 f0, h0;\n\tcvt.f32.f16 f1, h1;\n\tmov.b64 %0, {f0, f1};\n\t}"
        : "=l"(r) : "r"(byte));
    return r;
}

// acc[r][m] += dot(row r of this chunk, x'[m] of this chunk).
//   w: 8 rows x 16 bytes of codes + 16 bytes of scales (this lane's chunk)
//   xs_a: shared address of the staged activations [M][chunk_stride][32]
//         (128-byte aligned); x7 = 16 * (cl & 7), the chunk's granule swizzle,
//         so granule g of a chunk sits at (chunk address + x7) ^ (16 g)
//   ctv[m]: the chunk's -8 * 2^-48 * sum(x) term (Q4_0)
template <int FMT, int M>
__device__ __forceinline__ void compute_chunk(const uint4 (&w)[9], uint32_t xs_a, uint32_t x7, const float (&ctv)[M],
                                              int cl, int chunk_stride, float (&acc)[8][M]) {
    if constexpr (FMT == BW_FMT_Q4_0) {
        uint64_t bd[8][M];
#pragma unroll
        for (int m = 0; m < M; m++) {
            const uint64_t init = pair_f(ctv[m], 0.0f);
#pragma unroll
            for (int r = 0; r < 8; r++) bd[r][m] = init;
        }
#pragma unroll
        for (int wd = 0; wd < 4; wd++) {
            uint64_t x01[M], x23[M], x45[M], x67[M];
#pragma unroll
            for (int m = 0; m < M; m++) {
                const uint32_t xc = xs_a + 128u * static_cast<uint32_t>(m * chunk_stride + cl) + x7;
                lds_2x64(xc ^ (32u * wd), x01[m], x23[m]);
                lds_2x64(xc ^ (32u * wd + 16u), x45[m], x67[m]);
            }
#pragma unroll
            for (int r = 0; r < 8; r++) {
                const uint32_t v = u4_get(w[r], wd);
                const uint32_t h = v >> 16;
                // nibble slots 0..3 of each 16-bit half, masked in place: (slot 0, slot 1), (slot 2, slot 3)
                const uint64_t f01 = and_pair(v, 0x000000F00000000Full);
                const uint64_t f23 = and_pair(v, 0x0000F00000000F00ull);
                const uint64_t f45 = and_pair(h, 0x000000F00000000Full);
                const uint64_t f67 = and_pair(h, 0x0000F00000000F00ull);
#pragma unroll
                for (int m = 0; m < M; m++) {
                    uint64_t b = bd[r][m];
                    b = ffma2_64(f01, x01[m], b);
                    b = ffma2_64(f23, x23[m], b);
                    b = ffma2_64(f45, x45[m], b);
                    b = ffma2_64(f67, x67[m], b);
                    bd[r][m] = b;
                }
            }
        }
#pragma unroll
        for (int r2 = 0; r2 < 4; r2++) {
            const float2 d = __half22float2(*reinterpret_cast<const __half2 *>(&(r2 == 0 ? w[8].x : r2 == 1 ? w[8].y
                                                                                  : r2 == 2 ? w[8].z : w[8].w)));
#pragma unroll
            for (int m = 0; m < M; m++) {
                acc[2 * r2][m] = fma_rn(d.x, pair_sum(bd[2 * r2][m]), acc[2 * r2][m]);
                acc[2 * r2 + 1][m] = fma_rn(d.y, pair_sum(bd[2 * r2 + 1][m]), acc[2 * r2 + 1][m]);
            }
        }
    } else {
#pragma unroll
        for (int half = 0; half < 2; half++) {
            uint64_t bd[8][M];
#pragma unroll
            for (int r = 0; r < 8; r++)
#pragma unroll
                for (int m = 0; m < M; m++) bd[r][m] = 0ull;
#pragma unroll
            for (int wd = 2 * half; wd < 2 * half + 2; wd++) {
                uint64_t x01[M], x23[M], x45[M], x67[M];
#pragma unroll
                for (int m = 0; m < M; m++) {
                    const uint32_t xc = xs_a + 128u * static_cast<uint32_t>(m * chunk_stride + cl) + x7;
                    lds_2x64(xc ^ (32u * wd), x01[m], x23[m]);
                    lds_2x64(xc ^ (32u * wd + 16u), x45[m], x67[m]);
                }
#pragma unroll
                for (int r = 0; r < 8; r++) {
                    const uint32_t v = u4_get(w[r], wd);
                    const uint64_t e0 = e2m1x2_pair(v);
                    const uint64_t e1 = e2m1x2_pair(v >> 8);
                    const uint64_t e2 = e2m1x2_pair(v >> 16);
                    const uint64_t e3 = e2m1x2_pair(v >> 24);
#pragma unroll
                    for (int m = 0; m < M; m++) {
                        uint64_t b = bd[r][m];
                        b = ffma2_64(e0, x01[m], b);
                        b = ffma2_64(e1, x23[m], b);
                        b = ffma2_64(e2, x45[m], b);
                        b = ffma2_64(e3, x67[m], b);
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
                for (int m = 0; m < M; m++) acc[r][m] = fma_rn(s, pair_sum(bd[r][m]), acc[r][m]);
            }
        }
    }
}

// The lane-constant part of a stage's shared-memory addresses (callers hoist
// it out of their stage loops).  Warp w owns row groups 2w (lanes 0..15) and
// 2w+1 (lanes 16..31) of the 128-row tile; lane & 15 is the chunk.
struct ChunkLane {
    uint32_t w;    // row 8g's chunk c before the XOR swizzle: g * 2048 + c * 16
    uint32_t s;    // the chunk's scales: 32 KB + g * 256 + c * 16
    uint32_t x7;   // 16 * (c & 7), the activation granule swizzle
};
__device__ __forceinline__ ChunkLane chunk_lane(int warp, int lane) {
    const uint32_t g = 2 * warp + (lane >> 4), c = lane & 15;
    return {g * (8u * GV_TC * 16u) + c * 16u, GV_NIB_BYTES + g * (GV_TC * 16u) + c * 16u, 16u * (c & 7u)};
}

// Ring position of a stage stream: slot and the parity of its full barrier.
struct RingPos {
    int s;
    uint32_t ph;
};
__device__ __forceinline__ void ring_next(RingPos &r, int nst) {
    if (++r.s == nst) {
        r.s = 0;
        r.ph ^= 1u;
    }
}

// One lane's chunk of one stage (stage_a 256-byte aligned, so row r's slot
// c ^ r of row group g sits at (stage_a + g*2048 + c*16) ^ (16 r), + 256 r).
template <int FMT, int M>
__device__ __forceinline__ void stage_chunk(uint32_t stage_a, const ChunkLane &cn, uint32_t xs_a, uint32_t ct_a,
                                            int cl, int chunk_stride, float (&acc)[8][M]) {
    const uint32_t wb = stage_a + cn.w;
    uint4 w[9];
#pragma unroll
    for (int r = 0; r < 8; r++) w[r] = lds_u4((wb ^ (16u * r)) + 256u * r);
    w[8] = lds_u4(stage_a + cn.s);
    float ctv[M];
#pragma unroll
    for (int m = 0; m < M; m++)
        ctv[m] = (FMT == BW_FMT_Q4_0) ? lds_f(ct_a + 4u * static_cast<uint32_t>(m * chunk_stride + cl)) : 0.0f;
    compute_chunk<FMT, M>(w, xs_a, cn.x7, ctv, cl, chunk_stride, acc);
}

// Reduce acc[8][M] over each half-warp (16 lanes, one row group each).
// Afterwards lane l with (l & 1) == 0 holds the totals of row ((l >> 1) & 7)
// of its half's row group in out[m].
template <int M>
__device__ __forceinline__ void reduce_rows16(float (&acc)[8][M], int lane, float (&out)[M]) {
    const bool b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
#pragma unroll
    for (int m = 0; m < M; m++) {
        float b[4], c[2];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const float send = b3 ? acc[i][m] : acc[i + 4][m];
            const float keep = b3 ? acc[i + 4][m] : acc[i][m];
            b[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
#pragma unroll
        for (int i = 0; i < 2; i++) {
            const float send = b2 ? b[i] : b[i + 2];
            const float keep = b2 ? b[i + 2] : b[i];
            c[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
        }
        const float send = b1 ? c[0] : c[1];
        const float keep = b1 ? c[1] : c[0];
        float d = keep + __shfl_xor_sync(0xffffffffu, send, 2);
        d += __shfl_xor_sync(0xffffffffu, d, 1);
        out[m] = d;
    }
}

}  // namespace bw
