// gemm_mma.cu -- small-M GEMM over NVFP4 weights on the sm_100a tensor cores
// (tcgen05), for the batched-decode and speculative-verify passes that carry
// 5..32 activation rows.
//
// The deep-dive page (10100.com), section 7, lists native NVFP4 weights and
// tensor-core decode on Blackwell; section 5, stage 4 turns the verify pass
// into a few-row contraction.  With M rows the 4-bit weight tile is reused M
// times, so past a handful of rows the CUDA-core dot products stop keeping up
// with HBM while the tensor cores still do.
//
// Numerics.  An NVFP4 weight is e2m1 * e4m3 * ts.  The first product has at
// most 6 significant bits and lies in [2^-10, 2688], so it is EXACT in fp16:
// the A operand carries the exact block-scaled weights, the tensor scale ts
// multiplies the fp32 accumulator in the epilogue.  Activations are rounded
// to fp16 (RNE) for the B operand -- the only rounding beyond fp32
// reordering, graded by tolerance.
//
// One CTA per SM, 10 warps:
//   warp 0     producer: streams weight tiles (32 KB codes + 4 KB scales, the
//              tiled layout of bw.h) into a ring of shared-memory stages with
//              plain bulk copies (no multicast);
//   warp 1     owns the tensor memory (alloc/dealloc); lane 0 issues the MMAs;
//   warps 2..5 dequantize (one weight row per thread: TMEM lane = row) into
//              A slots in tensor memory with tcgen05.st;
//   warps 6..9 run each row block's epilogue from its accumulator (tcgen05.ld):
//              once it is in registers the next row block's MMAs start, and the
//              rest of the epilogue (split-K partial sums, residual, SiLU gate,
//              argmax) overlaps them.
// A tcgen05.mma of M = 128, K = 16 costs the issuing thread about 150-200
// cycles whatever N (16..256) and wherever A lives (measured on a B200), so at
// N = 32 the MMA issue sets the pace (one 64-column A slot = 4 MMAs); the
// dequant of a slot takes less, and the epilogue must not stall it.
// MMA: kind::f16, M = 128 weight rows, N = the activation rows padded to 16
// or 32, K = 16 per instruction; A from tensor memory, B from shared memory
// in the canonical K-major layout without swizzle.  The activations are
// packed into that layout once per GEMM (act_pack_kernel, with the RMSNorm
// fused) and each CTA fetches its K slice with one bulk copy; fp32 accumulators in tensor memory, double
// buffered so the next row block's MMAs overlap the epilogue.
// Work split: 128-row blocks x K slices (as the CUDA-core GEMV); slices
// leave partial sums, the last CTA of a row block adds them in slice order.
#include "gemv_core.cuh"

#include <cuda_fp16.h>

namespace bw {

constexpr int MM_THREADS = 320;
constexpr int MM_DW = 4;                 // dequant / epilogue warps (warps 2..5)
constexpr int MM_NA = 4;                 // A slots in tensor memory, 64 columns of K each
constexpr int MM_SLOT_COLS = 32;         // 64 fp16 per row = 32 x 32-bit columns
constexpr int MM_TMEM_COLS = 256;        // 4 A slots (128) + 2 accumulators (<= 64), power of two
constexpr int MM_ACC_COL = MM_NA * MM_SLOT_COLS;
constexpr int MM_MAXM = 32;
constexpr int MM_NST = 3;
constexpr size_t MM_SMEM_LIMIT = 227 * 1024 - 2048;   // dynamic part; static arrays take the rest

struct MmaParams {
    const uint8_t *q, *s;
    int N, K, M, Mp;                     // Mp: rows padded to 16 or 32 (the MMA's N)
    int RB, KT, S, CT, per_slice;
    const uint8_t *bpk;                  // activations, fp16, packed (act_pack_kernel)
    const float *residual;
    float *y;
    int32_t *argmax_out;
    unsigned flags;
    float ts, ts_up;
    float *partial;                      // [S][RB*128][Mp]
    uint32_t *rb_cnt;                    // [RB]
    float *am_val;                       // [grid][Mp]
    int *am_idx;
    uint32_t *am_cnt;
    int32_t *adv_tokens, *adv_pos;
    uint32_t *err;
};

// ------------------------------------------------------------ tcgen05 PTX

__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// arrive (once) on `bar` when every MMA this thread issued so far has completed
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// D[128 x N] (+)= A[128 x 16] (tensor memory) * B[N x 16]^T (shared memory), f16 in, f32 accumulate
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// this warp's 32 lanes x 32 consecutive 32-bit columns
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
        "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
        "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]),
          "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]),
          "=r"(v[30]), "=r"(v[31])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 16; i < 32; i++) v[i] = 0u;
}
// wait for the loads above; the values pass through so no use moves ahead of the wait
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.wait::ld.sync.aligned;"
        : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
          "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]),
          "+r"(v[16]), "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]), "+r"(v[22]),
          "+r"(v[23]), "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]), "+r"(v[29]),
          "+r"(v[30]), "+r"(v[31])
        :
        : "memory");
}
// atomic add with acquire-release semantics at GPU scope (the split-K
// arrival counter: it publishes this CTA's partial sums and, for the last
// arriver, acquires everyone else's)
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t *addr, uint32_t v) {
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
    return old;
}
// the four epilogue warps' barrier
__device__ __forceinline__ void ep_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Shared-memory matrix descriptor, K-major canonical layout without swizzle:
// 8-row x 16-byte core matrices, `lbo` bytes between the two core matrices
// along K, `sbo` bytes between 8-row groups.
__device__ __forceinline__ uint64_t smem_desc_kmajor(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;   // descriptor version of sm_100
    return d;                              // base offset 0, relative LBO, no swizzle
}

// Instruction descriptor of kind::f16: f16 A and B, both K-major, f32 D,
// M = 128, N = n.
__host__ __device__ constexpr uint32_t mma_idesc_f16(int n) {
    return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

// two e2m1 codes (one byte, element 2i low) -> f16x2 {2i, 2i+1}
__device__ __forceinline__ uint32_t e2m1x2_h2(uint32_t byte) {
    uint32_t h2;
    asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(h2) : "r"(byte));
    return h2;
}
__device__ __forceinline__ uint32_t e4m3x2_h2(uint32_t two) {
    uint32_t h2;
    asm("{\n\t.reg .b16 s;\n\tcvt.u16.u32 s, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, s;\n\t}" : "=r"(h2) : "r"(two));
    return h2;
}
__device__ __forceinline__ uint32_t hmul2_u(uint32_t a, uint32_t b) {
    __half2 r = __hmul2(*reinterpret_cast<__half2 *>(&a), *reinterpret_cast<__half2 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
}

// One chunk (32 weights) of one row: 16 code bytes + the two E4M3 block
// scales -> 16 f16x2 words {w[2i], w[2i+1]} = e2m1 * e4m3, exact.
__device__ __forceinline__ void dequant_chunk(uint4 c, uint32_t sc2, uint32_t *out) {
    const uint32_t s = e4m3x2_h2(sc2);
    const uint32_t s0 = __byte_perm(s, s, 0x1010), s1 = __byte_perm(s, s, 0x3232);
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int j = 0; j < 4; j++)
#pragma unroll
        for (int b = 0; b < 4; b++) out[j * 4 + b] = hmul2_u(e2m1x2_h2((w[j] >> (8 * b)) & 0xffu), j < 2 ? s0 : s1);
}

// ----------------------------------------------------------------- kernel

__global__ void __launch_bounds__(MM_THREADS, 1) mma_gemm_kernel(const MmaParams p) {
    extern __shared__ __align__(1024) unsigned char mm_smem[];
    unsigned char *stages = mm_smem;                                             // MM_NST x 36 KB
    unsigned char *bsm = mm_smem + static_cast<size_t>(MM_NST) * GV_STAGE_BYTES;   // B: [CS*4 core cols][Mp/8][128 B]
    const int CS = p.CT * GV_TC;                                                 // chunks per slice
    const size_t b_bytes = static_cast<size_t>(CS) * 4 * (p.Mp / 8) * 128;
    uint64_t *bars = reinterpret_cast<uint64_t *>(bsm + b_bytes);
    uint64_t *full = bars, *empty = bars + MM_NST;
    uint64_t *afull = empty + MM_NST, *aempty = afull + MM_NA;
    uint64_t *dfull = aempty + MM_NA, *dread = dfull + 2;
    uint64_t *bfull = dread + 1;
    __shared__ uint32_t s_tmem;
    __shared__ float s_bv[MM_DW][MM_MAXM];
    __shared__ int s_bi[MM_DW][MM_MAXM];
    __shared__ bool s_last;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slice = blockIdx.x % p.S;
    const int j0 = blockIdx.x / p.S;
    const int kt0 = slice * p.CT;
    const int T = min(p.CT, p.KT - kt0);
    const int n_items = j0 < p.RB ? (p.RB - 1 - j0) / p.per_slice + 1 : 0;
    const int n_tiles = n_items * T;

    if (threadIdx.x == 0) {
        for (int i = 0; i < MM_NST; i++) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], MM_DW);
        }
        for (int i = 0; i < MM_NA; i++) {
            mbar_init(&afull[i], MM_DW);
            mbar_init(&aempty[i], 1);
        }
        for (int i = 0; i < 2; i++) mbar_init(&dfull[i], 1);
        mbar_init(dread, MM_DW);
        mbar_init(bfull, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&s_tmem, MM_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    if (warp == 0) {
        // ---- producer: the first stages of constant weights before the
        //      dependency wait, then this slice's packed activations (one
        //      contiguous block), then the rest of the weights
        if (lane == 0) {
            auto issue = [&](int t) {
                const int s = t % MM_NST;
                if (t >= MM_NST) mbar_wait(&empty[s], static_cast<uint32_t>((t / MM_NST - 1) & 1), p.err);
                const int item = t / T, kt = kt0 + (t - item * T);
                const int rb = j0 + item * p.per_slice;
                const size_t tile = static_cast<size_t>(rb) * p.KT + kt;
                unsigned char *st = stages + static_cast<size_t>(s) * GV_STAGE_BYTES;
                mbar_arrive_tx(&full[s], GV_STAGE_BYTES);
                bulk_g2s(st, p.q + tile * GV_NIB_BYTES, GV_NIB_BYTES, &full[s]);
                bulk_g2s(st + GV_NIB_BYTES, p.s + tile * GV_SC_BYTES, GV_SC_BYTES, &full[s]);
            };
            const int pre = min(MM_NST, n_tiles);
            for (int t = 0; t < pre; t++) issue(t);
            pdl_wait();
            // dependents launch only once this kernel's dependency is met:
            // a kernel after this one may read, before its own wait, what
            // the launches before this one wrote
            pdl_trigger();
            if (n_tiles > 0) {
                const uint32_t col_bytes = static_cast<uint32_t>(GV_TC * 4 * (p.Mp / 8) * 128);   // one column tile
                mbar_arrive_tx(bfull, static_cast<uint32_t>(T) * col_bytes);
                bulk_g2s(bsm, p.bpk + static_cast<size_t>(kt0) * col_bytes, static_cast<uint32_t>(T) * col_bytes, bfull);
            }
            for (int t = pre; t < n_tiles; t++) issue(t);
        }
    } else if (warp == 1) {
        // ---- MMA issuer
        if (lane == 0 && n_items > 0) {
            const uint32_t idesc = mma_idesc_f16(p.Mp);
            const uint32_t b_a = smem_u32(bsm);
            const uint32_t lbo = static_cast<uint32_t>(p.Mp / 8) * 128u, sbo = 128u;
            // the slice's activations have landed in shared memory
            mbar_wait(bfull, 0u, p.err);
            tc_fence_after();
            int g = 0;   // A-slot step
            for (int item = 0; item < n_items; item++) {
                const int db = item & 1;
                // the previous row block's accumulator is in the epilogue warps'
                // registers: MMAs running while another warp reads tensor memory
                // with tcgen05.ld corrupted lanes of that read on a B200 (even
                // with the two accumulators 64 columns apart), so they never overlap
                if (item >= 1) mbar_wait(dread, static_cast<uint32_t>((item - 1) & 1), p.err);
                tc_fence_after();
                const uint32_t d_t = tmem + MM_ACC_COL + static_cast<uint32_t>(db * p.Mp);
                for (int kt = 0; kt < T; kt++) {
                    for (int st8 = 0; st8 < 8; st8++, g++) {
                        const int a = g % MM_NA;
                        mbar_wait(&afull[a], static_cast<uint32_t>((g / MM_NA) & 1), p.err);
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 4; kk++) {
                            // K offset inside the slice, in 8-element core columns
                            const int kc = (kt * 512 + st8 * 64 + kk * 16) / 8;
                            const uint64_t bd = smem_desc_kmajor(b_a + static_cast<uint32_t>(kc) * lbo, lbo, sbo);
                            tc_mma_ts(d_t, tmem + static_cast<uint32_t>(a * MM_SLOT_COLS + kk * 8), bd, idesc,
                                      (kt | st8 | kk) != 0);
                        }
                        tc_commit(&aempty[a]);
                    }
                }
                tc_commit(&dfull[db]);
            }
        }
        __syncwarp();
    } else if (warp < 2 + MM_DW) {
        // ---- dequant warps: quarter qd of the tile rows into the A slots
        const int qd = warp & 3;                  // tensor-memory lane quarter this warp may access
        const int r = qd * 32 + lane;             // tile row = tensor-memory lane
        const uint32_t t_row = tmem + (static_cast<uint32_t>(qd * 32) << 16);
        int g = 0, t = 0;
        for (int item = 0; item < n_items; item++) {
            for (int kt = 0; kt < T; kt++, t++) {
                const int s = t % MM_NST;
                mbar_wait(&full[s], static_cast<uint32_t>((t / MM_NST) & 1), p.err);
                const uint32_t st_a = smem_u32(stages) + static_cast<uint32_t>(s) * GV_STAGE_BYTES;
                const uint32_t row_a = st_a + static_cast<uint32_t>(r) * (GV_TC * 16);
                const uint32_t sc_a = st_a + GV_NIB_BYTES + static_cast<uint32_t>(r >> 3) * (GV_TC * 16) + (r & 7) * 2;
                for (int st8 = 0; st8 < 8; st8++, g++) {
                    const int a = g % MM_NA;
                    const int c0 = 2 * st8;
                    const uint4 w0 = lds_u4(row_a + static_cast<uint32_t>((c0 ^ (r & 7)) * 16));
                    const uint4 w1 = lds_u4(row_a + static_cast<uint32_t>(((c0 + 1) ^ (r & 7)) * 16));
                    uint32_t sc0, sc1;
                    asm volatile("ld.shared.u16 %0, [%1];" : "=r"(sc0) : "r"(sc_a + c0 * 16));
                    asm volatile("ld.shared.u16 %0, [%1];" : "=r"(sc1) : "r"(sc_a + (c0 + 1) * 16));
                    if (st8 == 7) {
                        // every code of this stage is in registers: release it
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&empty[s]);
                    }
                    uint32_t h[32];
                    dequant_chunk(w0, sc0, h);
                    dequant_chunk(w1, sc1, h + 16);
                    if (g >= MM_NA) mbar_wait(&aempty[a], static_cast<uint32_t>((g / MM_NA - 1) & 1), p.err);
                    tc_fence_after();
                    tmem_st32(t_row + static_cast<uint32_t>(a * MM_SLOT_COLS), h);
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&afull[a]);
                }
            }
        }
    } else {
        // ---- epilogue warps: each row block's accumulator (quarter qd of its
        //      rows) while the next row block's MMAs run
        const int ew = warp - 2 - MM_DW;          // 0..3 (arrival bookkeeping)
        const int qd = warp & 3;                  // tensor-memory lane quarter this warp may access
        const int r = qd * 32 + lane;             // tile row = tensor-memory lane
        const int dtid = ew * 32 + lane;          // 0..127
        const uint32_t t_row = tmem + (static_cast<uint32_t>(qd * 32) << 16);
        const float tsc = ((p.flags & BW_GEMV_SILU_GATE) && (r & 7) >= 4) ? p.ts_up : p.ts;
        float bestv[MM_MAXM];
        int besti[MM_MAXM];
#pragma unroll
        for (int m = 0; m < MM_MAXM; m++) {
            bestv[m] = -INFINITY;
            besti[m] = 0x7fffffff;
        }
        for (int item = 0; item < n_items; item++) {
            const int rb = j0 + item * p.per_slice;
            // ---- accumulator of this row block (the epilogue reads what earlier
            //      kernels wrote: wait for them once)
            if (item == 0) pdl_wait();
            const int db = item & 1;
            mbar_wait(&dfull[db], static_cast<uint32_t>((item >> 1) & 1), p.err);
            tc_fence_after();
            uint32_t acc_u[32];
            if (p.Mp == 32)
                tmem_ld32(t_row + MM_ACC_COL + static_cast<uint32_t>(db * p.Mp), acc_u);
            else
                tmem_ld16(t_row + MM_ACC_COL + static_cast<uint32_t>(db * p.Mp), acc_u);
            tmem_ld_wait(acc_u);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dread);
            float v[MM_MAXM];
#pragma unroll
            for (int m = 0; m < MM_MAXM; m++) v[m] = __uint_as_float(acc_u[m]);

            const int n = rb * GV_TR + r;
            // the residual rows of this output row, all loads issued at once
            // (y may be the residual itself, so they cannot wait for the
            // stores), before the split-K hand-off whose round trip they overlap
            float res[MM_MAXM];
            if ((p.flags & BW_GEMV_RESIDUAL) && n < p.N) {
#pragma unroll
                for (int m = 0; m < MM_MAXM; m++)
                    res[m] = m < p.M ? __ldcg(p.residual + static_cast<size_t>(m) * p.N + n) : 0.0f;
            }
            bool act = true;
            if (p.S > 1) {
                float *dst = p.partial + (static_cast<size_t>(slice) * p.RB * GV_TR + n) * p.Mp;
#pragma unroll
                for (int m = 0; m < MM_MAXM; m += 4)
                    if (m < p.Mp)
                        __stcg(reinterpret_cast<float4 *>(dst + m), make_float4(v[m], v[m + 1], v[m + 2], v[m + 3]));
                // every lane's partial sums are written (barrier), then one thread
                // publishes them and counts this slice's arrival: a GPU-scope
                // fence after the barrier covers the other lanes' stores
                ep_sync();
                if (dtid == 0) {
                    __threadfence();
                    s_last = atom_add_acq_rel(p.rb_cnt + rb, 1u) == static_cast<uint32_t>(p.S - 1);
                    if (s_last) __threadfence();
                }
                ep_sync();
                act = s_last;
                if (act) {
#pragma unroll
                    for (int m = 0; m < MM_MAXM; m++) v[m] = 0.0f;
                    for (int s2 = 0; s2 < p.S; s2++) {
                        const float *src = p.partial + (static_cast<size_t>(s2) * p.RB * GV_TR + n) * p.Mp;
#pragma unroll
                        for (int m = 0; m < MM_MAXM; m += 4) {
                            if (m >= p.Mp) break;
                            const float4 q4 = __ldcg(reinterpret_cast<const float4 *>(src + m));
                            v[m] += q4.x;
                            v[m + 1] += q4.y;
                            v[m + 2] += q4.z;
                            v[m + 3] += q4.w;
                        }
                    }
                    if (dtid == 0) p.rb_cnt[rb] = 0u;
                }
            }
            // epilogue (all lanes take part in the shuffle)
#pragma unroll
            for (int m = 0; m < MM_MAXM; m++) v[m] *= tsc;
            if (p.flags & BW_GEMV_SILU_GATE) {
#pragma unroll
                for (int m = 0; m < MM_MAXM; m++) {
                    const float up = __shfl_down_sync(0xffffffffu, v[m], 4);
                    if (act && (r & 7) < 4 && m < p.M && n < p.N) {
                        const float gt = v[m];
                        p.y[static_cast<size_t>(m) * (p.N / 2) + (n >> 3) * 4 + (r & 7)] = (gt / (1.0f + expf(-gt))) * up;
                    }
                }
            } else if (act && n < p.N) {
#pragma unroll
                for (int m = 0; m < MM_MAXM; m++) {
                    if (m >= p.M) break;
                    float val = v[m];
                    const size_t o = static_cast<size_t>(m) * p.N + n;
                    if (p.flags & BW_GEMV_RESIDUAL) val = res[m] + val;
                    if (p.y) p.y[o] = val;
                    if (better(val, n, bestv[m], besti[m])) {
                        bestv[m] = val;
                        besti[m] = n;
                    }
                }
            }
        }

        pdl_wait();   // (already done by the first epilogue when this CTA had work)
        // ---- greedy argmax: CTA partials, the last CTA reduces
        if (p.flags & BW_GEMV_ARGMAX) {
#pragma unroll
            for (int m = 0; m < MM_MAXM; m++) {
                float bv = bestv[m];
                int bi = besti[m];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                    if (better(ov, oi, bv, bi)) {
                        bv = ov;
                        bi = oi;
                    }
                }
                if (lane == 0) {
                    s_bv[ew][m] = bv;
                    s_bi[ew][m] = bi;
                }
            }
            ep_sync();
            if (dtid < p.M) {
                const int m = dtid;
                float bv = s_bv[0][m];
                int bi = s_bi[0][m];
                for (int w2 = 1; w2 < MM_DW; w2++)
                    if (better(s_bv[w2][m], s_bi[w2][m], bv, bi)) {
                        bv = s_bv[w2][m];
                        bi = s_bi[w2][m];
                    }
                __stcg(p.am_val + blockIdx.x * p.Mp + m, bv);
                __stcg(p.am_idx + blockIdx.x * p.Mp + m, bi);
            }
            __threadfence();
            ep_sync();
            if (dtid == 0) s_last = atomicAdd(p.am_cnt, 1u) == gridDim.x - 1;
            ep_sync();
            if (s_last) {
                __threadfence();
                for (int m = ew; m < p.M; m += MM_DW) {
                    float bv = -INFINITY;
                    int bi = 0x7fffffff;
                    for (int b = lane; b < static_cast<int>(gridDim.x); b += 32) {
                        const float ov = __ldcg(p.am_val + b * p.Mp + m);
                        const int oi = __ldcg(p.am_idx + b * p.Mp + m);
                        if (better(ov, oi, bv, bi)) {
                            bv = ov;
                            bi = oi;
                        }
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                        if (better(ov, oi, bv, bi)) {
                            bv = ov;
                            bi = oi;
                        }
                    }
                    if (lane == 0) {
                        const int tok = (bi == 0x7fffffff) ? 0 : bi;
                        p.argmax_out[m] = tok;
                        if (p.adv_tokens) p.adv_tokens[m] = tok;
                        if (p.adv_pos) p.adv_pos[m] += 1;
                    }
                }
                if (dtid == 0) *p.am_cnt = 0u;
            }
        }
    }

    // every tensor-memory access of the CTA is done: free it
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, MM_TMEM_COLS);
    }
}

// Activations -> fp16 B operand in the canonical K-major layout of the MMA:
// core column kc (8 consecutive k) of row m at ((kc * Mp/8 + m/8) * 8 + m%8)
// * 16 bytes; the column tiles of K are therefore contiguous blocks.  Rows
// M..Mp-1 and columns K..KT*512-1 are zero.  With gamma, the row is
// normalized first: (x * r) * gamma, r = 1 / sqrt(mean(x^2) + eps).
// Grid (Mp, KT): each CTA packs one 512-column tile of one row (and sums the
// squares of the whole row for its norm -- a few KB from L2).
__global__ void act_pack_kernel(const float *x, int M, int Mp, int K, int KT, const float *gamma, float eps,
                                uint8_t *out) {
    pdl_trigger();
    pdl_wait();
    __shared__ float red[32];
    __shared__ float s_rn;
    const int m = blockIdx.x;
    const bool real = m < M;
    const float *xr = x + static_cast<size_t>(real ? m : 0) * K;
    if (gamma && real) {
        float ss = 0.0f;
        for (int k = threadIdx.x; k < K; k += blockDim.x) ss = fma_rn(xr[k], xr[k], ss);
        ss = warp_sum(ss);
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
        __syncthreads();
        if (threadIdx.x == 0) {
            float t = 0.0f;
            for (int w = 0; w < static_cast<int>(blockDim.x >> 5); w++) t += red[w];
            s_rn = 1.0f / sqrtf(t / static_cast<float>(K) + eps);
        }
        __syncthreads();
    }
    const float rn = (gamma && real) ? s_rn : 1.0f;
    // this CTA's column tile: 64 core columns of 8
    const int kc1 = (blockIdx.y + 1) * 64;
    for (int kc = blockIdx.y * 64 + threadIdx.x; kc < kc1; kc += blockDim.x) {
        const int k = kc * 8;
        uint32_t h[4] = {0u, 0u, 0u, 0u};
        if (real && k < K) {
            const float4 a0 = *reinterpret_cast<const float4 *>(xr + k);
            const float4 a1 = *reinterpret_cast<const float4 *>(xr + k + 4);
            float v[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            if (gamma) {
                const float4 g0 = *reinterpret_cast<const float4 *>(gamma + k);
                const float4 g1 = *reinterpret_cast<const float4 *>(gamma + k + 4);
                const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
                for (int i = 0; i < 8; i++) v[i] = __fmul_rn(__fmul_rn(v[i], rn), gg[i]);
            }
#pragma unroll
            for (int i = 0; i < 4; i++) {
                __half2 hh = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
                h[i] = *reinterpret_cast<uint32_t *>(&hh);
            }
        }
        *reinterpret_cast<uint4 *>(out + (static_cast<size_t>(kc) * (Mp / 8) + (m >> 3)) * 128 + (m & 7) * 16) =
            make_uint4(h[0], h[1], h[2], h[3]);
    }
}

// ------------------------------------------------------------------- host

struct MmaPlan {
    int S, CT, per_slice, grid;
    size_t smem, partial_floats;
};

static size_t mma_b_bytes(int Mp, int CT) { return static_cast<size_t>(CT) * GV_TC * 4 * (Mp / 8) * 128; }

static MmaPlan plan_mma(int N, int K, int Mp) {
    MmaPlan pl;
    const int RB = gv_row_blocks(N), KT = gv_col_tiles(K);
    const int G = sm_count();
    const size_t fixed = static_cast<size_t>(MM_NST) * GV_STAGE_BYTES + 24 * 8 + 1024;   // + mbarriers, slack
    int bestS = KT, bestCT = 1;
    double best = 1e30;
    for (int S = 1; S <= min(64, KT); S++) {
        const int CT = (KT + S - 1) / S;
        if ((KT + CT - 1) / CT != S) continue;
        if (fixed + mma_b_bytes(Mp, CT) > MM_SMEM_LIMIT) continue;
        const int per_slice = max(1, min(RB, G / S));
        const int rounds = (RB + per_slice - 1) / per_slice;
        // the MMAs of a CTA's tiles are the critical path (the epilogue warps
        // overlap them); split K adds an item's fp32 partial sums, 128 x Mp x 4
        // bytes against a tile's 36 KB, that go back to memory
        const double part = S > 1 ? 128.0 * Mp * 4 / GV_STAGE_BYTES : 0.0;
        const double cost = static_cast<double>(rounds) * (CT + part) + 0.01 * S;
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
    pl.smem = fixed + mma_b_bytes(Mp, bestCT);
    pl.partial_floats = pl.S > 1 ? static_cast<size_t>(pl.S) * RB * GV_TR * Mp : 0;
    return pl;
}

static int mma_rows_padded(int M) { return M <= 16 ? 16 : 32; }

size_t mma_scratch_bytes(int N, int K, int M) {
    size_t tot = 0;
    for (int m0 = 0; m0 < M; m0 += MM_MAXM) {
        const int Mp = mma_rows_padded(min(MM_MAXM, M - m0));
        const MmaPlan pl = plan_mma(N, K, Mp);
        const size_t b = align_up(pl.partial_floats * 4, BW_WS_ALIGN) +
                         2 * align_up(static_cast<size_t>(pl.grid) * Mp * 4, BW_WS_ALIGN) +
                         align_up(static_cast<size_t>(gv_col_tiles(K)) * 512 * Mp * 2, BW_WS_ALIGN);
        tot = max(tot, b);
    }
    return tot;
}

bw_status mma_check(int N, int K, int M) {
    if (N <= 0 || K <= 0 || M <= 0) return BW_ERR_INVALID_ARG;
    if (K % 8) return BW_ERR_UNSUPPORTED_SHAPE;
    for (int m0 = 0; m0 < M; m0 += MM_MAXM) {
        const MmaPlan pl = plan_mma(N, K, mma_rows_padded(min(MM_MAXM, M - m0)));
        if (pl.smem > MM_SMEM_LIMIT) return BW_ERR_UNSUPPORTED_SHAPE;
        if (pl.S > 1 && gv_row_blocks(N) + CNT_GEMV_RG > CNT_ATTN) return BW_ERR_UNSUPPORTED_SHAPE;
    }
    return BW_OK;
}

bw_status mma_gemm_launch(const void *wq, const void *ws_scales, float ts, float ts_up, int N, int K,
                          const float *x, int M, const float *gamma, float eps, const float *residual, float *y,
                          int32_t *argmax_out, unsigned flags, const Scratch &sc, cudaStream_t st,
                          int32_t *adv_tokens, int32_t *adv_pos) {
    if (sc.bytes < mma_scratch_bytes(N, K, M)) return BW_ERR_INVALID_ARG;
    if (!aligned16(gamma) && (flags & BW_GEMV_RMSNORM)) return BW_ERR_INVALID_ARG;
    const bw_status chk = mma_check(N, K, M);
    if (chk != BW_OK) return chk;
    const int ncols = (flags & BW_GEMV_SILU_GATE) ? N / 2 : N;
    static size_t attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return BW_ERR_CUDA;
    for (int m0 = 0; m0 < M; m0 += MM_MAXM) {
        const int Mr = min(MM_MAXM, M - m0);
        const int Mp = mma_rows_padded(Mr);
        const MmaPlan pl = plan_mma(N, K, Mp);
        if (pl.smem > MM_SMEM_LIMIT) return BW_ERR_UNSUPPORTED_SHAPE;
        if (pl.S > 1 && gv_row_blocks(N) + CNT_GEMV_RG > CNT_ATTN) return BW_ERR_UNSUPPORTED_SHAPE;
        Carver cv(sc.base);
        MmaParams p;
        p.q = static_cast<const uint8_t *>(wq);
        p.s = static_cast<const uint8_t *>(ws_scales);
        p.N = N;
        p.K = K;
        p.M = Mr;
        p.Mp = Mp;
        p.RB = gv_row_blocks(N);
        p.KT = gv_col_tiles(K);
        p.S = pl.S;
        p.CT = pl.CT;
        p.per_slice = pl.per_slice;
        p.residual = residual ? residual + static_cast<size_t>(m0) * N : nullptr;
        p.y = y ? y + static_cast<size_t>(m0) * ncols : nullptr;
        p.argmax_out = argmax_out ? argmax_out + m0 : nullptr;
        p.flags = flags;
        p.ts = ts;
        p.ts_up = ts_up;
        p.partial = cv.take<float>(pl.partial_floats);
        p.am_val = cv.take<float>(static_cast<size_t>(pl.grid) * Mp);
        p.am_idx = cv.take<int>(static_cast<size_t>(pl.grid) * Mp);
        uint8_t *bpk = cv.take<uint8_t>(static_cast<size_t>(p.KT) * 512 * Mp * 2);
        p.bpk = bpk;
        p.rb_cnt = sc.cnt + CNT_GEMV_RG;
        p.am_cnt = sc.cnt + CNT_ARGMAX;
        p.adv_tokens = adv_tokens ? adv_tokens + m0 : nullptr;
        p.adv_pos = adv_pos ? adv_pos + m0 : nullptr;
        p.err = sc.err;
        const bw_status s0 = launch_pdl(act_pack_kernel, dim3(Mp, p.KT), dim3(256), 0, st, x + static_cast<size_t>(m0) * K,
                                        Mr, Mp, K, p.KT, (flags & BW_GEMV_RMSNORM) ? gamma : nullptr, eps, bpk);
        if (s0 != BW_OK) return s0;
        {
            static std::mutex mu;   // host threads may call the library concurrently
            std::lock_guard<std::mutex> lk(mu);
            if (attr_set[dev] < pl.smem) {
                if (cudaFuncSetAttribute(mma_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(pl.smem)) != cudaSuccess) {
                    (void)cudaGetLastError();
                    return BW_ERR_CUDA;
                }
                attr_set[dev] = pl.smem;
            }
        }
        const bw_status s1 = launch_pdl(mma_gemm_kernel, dim3(pl.grid), dim3(MM_THREADS), pl.smem, st, p);
        if (s1 != BW_OK) return s1;
    }
    return BW_OK;
}

}  // namespace bw
