// step_persistent.cu -- the whole batch-1 decode step of a dense model as ONE
// persistent kernel (sm_100a).
//
// The layer-by-layer chain launches about five kernels per layer; at batch 1
// each of them moves only a few MB, so the chain spends much of its time in
// launch latency, dependency waits and ramp-up instead of streaming weights.
// This kernel keeps one CTA resident on every SM for the whole step (a
// cooperative launch, so all CTAs are co-resident and may wait for each
// other) and walks the same sequence of phases in every CTA:
//
//   embedding -> for each layer: QKV -> attention -> O -> gate/up -> down
//   -> final norm + LM head + argmax
//
// The devpress bw24 page, section 2.3, describes the same aim (lean
// scheduling without host round trips) and section 2.4 tuning the launch to
// the SM count; this is that idea on one B200: the scheduling is static and
// on the device.
//
// Weight streaming never waits for activations.  Each CTA owns a fixed,
// contiguous range of every matrix's 36 KB tiles (the tiled layout of
// gemv_core.cuh, in (row block, column tile) order) and of every layer's KV
// pages, known at launch.  A producer warp streams all of them, phase after
// phase, through a ring of shared-memory stages (plain bulk copies,
// mbarrier full/empty pairs) and is held back only by free ring slots -- it
// runs ahead across phase and layer boundaries while the consumers wait for
// their inputs.  Weights, norm gains and the KV rows of earlier positions are
// constant during the step, which is what makes this legal.
//
// Sixteen consumer warps form two groups of eight that take alternate ring
// stages; each group runs the dequant-dot of gemv_core.cuh on its tiles (a
// half-warp per 8-row group, a lane per 32-column chunk) and the two groups'
// sums are added in a fixed order at the end of every row block segment.
// Split-K: a row block whose column tiles span several CTAs leaves one
// partial sum per CTA; the last CTA to arrive (an atomic counter per 8-row
// group, no waiting) adds them in column order and runs the epilogue, so
// results are deterministic.  A phase's consumers wait for the previous
// phase's output through monotonic completion counters (bounded spins that
// set BW_DEVERR_TIMEOUT and abort the step rather than hang).
//
// Attention: every kv head gets S = (CTAs / nkv) CTAs, each a contiguous
// range of the sequence's pages (the last one also holds the new token,
// whose RoPE'd k and v it writes into the cache in fp16); every CTA keeps an
// online softmax per query head of its group on the CUDA cores, then the S
// CTAs of a head merge the partial results together, each a slice of the
// outputs.  The deep-dive page, section 6: logical positions map to physical
// pages through the page table.
#include <math.h>

#include "gemv_core.cuh"

namespace bw {

constexpr int PK_GRP = 2;                      // consumer groups
constexpr int PK_CW = GV_CW * PK_GRP;          // consumer warps
constexpr int PK_CT = PK_CW * 32;              // consumer threads
constexpr int PK_THREADS = PK_CT + 32;         // + one producer warp
constexpr int PK_MAXG = 8;                     // query heads per kv head
constexpr int PK_MAXSLOTS = 16;                // staged column tiles of a phase
constexpr uint32_t PK_SPIN = 1u << 22;         // polls of a dependency wait before it gives up

// counters of the persistent step, uint32 indices into Scratch::cnt (zero
// between launches; the last CTA to leave resets them)
constexpr unsigned PKC_BASE = 8;
enum : unsigned { PKC_X = 0, PKC_QKV, PKC_ATT, PKC_O, PKC_GU, PKC_AM, PKC_EXIT, PKC_ABORT, PKC_ARRIVE = 8 };
constexpr int PK_MAXKV = 64 - PKC_BASE - PKC_ARRIVE;   // arrival counters of the kv heads
constexpr unsigned PKC_RG = CNT_GEMV_RG;       // split-K counters, one per 8-row group

struct PkLayer {
    const uint8_t *qkv_q, *qkv_s, *o_q, *o_s, *gu_q, *gu_s, *d_q, *d_s;
    const float *attn_norm, *ffn_norm;
    __half *k_pool, *v_pool;
    float ts_qkv, ts_o, ts_g, ts_u, ts_d;
};

constexpr int PK_MAXL = 96;

struct PkParams {
    int L, H, nq, nkv, hd, F, V, G;
    float eps, scale;
    const uint8_t *emb_q, *emb_s;
    float emb_ts;
    const uint8_t *lm_q, *lm_s;
    float lm_ts;
    const float *final_norm;
    const float *rope_cos, *rope_sin;
    int rope_max_pos;
    const int32_t *page_table;
    int max_pages, n_pages;
    int32_t *tokens_in, *pos, *tokens_out;
    float *logits;
    int advance;
    float *x, *qkv, *attn, *act;     // activations (workspace)
    float *part;                     // [grid][2][128] split-K partial sums
    float *att_ml;                   // [grid][PK_MAXG][2] attention (max, sum) per split
    float *att_o;                    // [grid][PK_MAXG][hd] unnormalised attention outputs
    float *am_val;                   // [grid]
    int *am_idx;                     // [grid]
    uint32_t *cnt;                   // Scratch::cnt
    uint32_t *err;
    int nst, S, nslots;              // ring stages, attention CTAs per kv head, staged tiles per phase
    PkLayer layer[PK_MAXL];
};

// one GEMV phase: the matrix and what goes in and out
struct PkMat {
    const uint8_t *q, *s;
    int N, K, RB, KT, T;
    float ts, ts_up;
};

enum : int { PH_QKV = 0, PH_ATT, PH_O, PH_GU, PH_DOWN, PH_LM };

__device__ __forceinline__ PkMat pk_mat(const PkParams &p, int kind, int l) {
    PkMat m;
    const PkLayer &ly = p.layer[l < p.L ? l : 0];
    if (kind == PH_QKV) {
        m.q = ly.qkv_q; m.s = ly.qkv_s; m.N = (p.nq + 2 * p.nkv) * p.hd; m.K = p.H;
        m.ts = m.ts_up = ly.ts_qkv;
    } else if (kind == PH_O) {
        m.q = ly.o_q; m.s = ly.o_s; m.N = p.H; m.K = p.nq * p.hd;
        m.ts = m.ts_up = ly.ts_o;
    } else if (kind == PH_GU) {
        m.q = ly.gu_q; m.s = ly.gu_s; m.N = 2 * p.F; m.K = p.H;
        m.ts = ly.ts_g; m.ts_up = ly.ts_u;
    } else if (kind == PH_DOWN) {
        m.q = ly.d_q; m.s = ly.d_s; m.N = p.H; m.K = p.F;
        m.ts = m.ts_up = ly.ts_d;
    } else {
        m.q = p.lm_q; m.s = p.lm_s; m.N = p.V; m.K = p.H;
        m.ts = m.ts_up = p.lm_ts;
    }
    m.RB = gv_row_blocks(m.N);
    m.KT = gv_col_tiles(m.K);
    m.T = m.RB * m.KT;
    return m;
}

// First tile of CTA c's range.  Ranges are contiguous and balanced to +-1
// tile over min(T, G) CTAs, so every CTA that has a range has at least one
// tile; CTAs c >= T (a matrix with fewer tiles than CTAs) get none.
__device__ __forceinline__ int pk_start(int T, int c, int G) {
    const int ge = min(T, G);
    return c >= ge ? T : static_cast<int>(static_cast<long long>(T) * c / ge);
}
// the CTA whose range holds tile t
__device__ __forceinline__ int pk_owner(int T, int t, int G) {
    const int ge = min(T, G);
    int c = static_cast<int>((static_cast<long long>(t) * ge) / T);
    while (c + 1 < ge && pk_start(T, c + 1, G) <= t) c++;
    while (c > 0 && pk_start(T, c, G) > t) c--;
    return c;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void pk_sync() { asm volatile("bar.sync 1, %0;" ::"n"(PK_CT) : "memory"); }

__device__ __forceinline__ bool pk_aborted(const PkParams &p) {
    return ld_acquire_u32(p.cnt + PKC_BASE + PKC_ABORT) != 0;
}
__device__ __forceinline__ void pk_abort(const PkParams &p) {
    set_error(p.err, BW_DEVERR_TIMEOUT);
    atomicExch(p.cnt + PKC_BASE + PKC_ABORT, 1u);
}

// Consumer-wide wait until counter >= target (thread 0 polls, the others wait
// at the barrier).  Returns false when the step was aborted.
__device__ bool pk_wait(const PkParams &p, unsigned which, uint32_t target, int ctid, int *s_ok) {
    if (ctid == 0) {
        const uint32_t *c = p.cnt + PKC_BASE + which;
        int ok = 1;
        uint32_t i = 0;
        while (ld_acquire_u32(c) < target) {
            if ((++i & 63) == 0 && pk_aborted(p)) {
                ok = 0;
                break;
            }
            if (i >= PK_SPIN) {
                pk_abort(p);
                ok = 0;
                break;
            }
        }
        *s_ok = ok;
    }
    pk_sync();
    return *s_ok != 0;
}

// Bounded mbarrier wait that also gives up when the step was aborted.
__device__ bool pk_mbar_wait(const PkParams &p, uint64_t *bar, uint32_t parity) {
    for (uint32_t i = 0; i < PK_SPIN; i++) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63) == 63 && pk_aborted(p)) return false;
    }
    pk_abort(p);
    return false;
}

// consumer-wide completion: every consumer's global writes, then one atomic
__device__ __forceinline__ void pk_signal(const PkParams &p, unsigned which, uint32_t add, int ctid) {
    pk_sync();
    if (ctid == 0 && add) {
        __threadfence();
        atomicAdd(p.cnt + PKC_BASE + which, add);
    }
}

// ------------------------------------------------------------- producer

// Position in the CTA's stage stream: index, ring slot, parity of the slot's
// full barrier (advanced incrementally: no division by the ring depth).
struct PkStream {
    uint32_t i;
    int s;
    uint32_t ph;
    __device__ __forceinline__ void adv(int nst) {
        i++;
        if (++s == nst) {
            s = 0;
            ph ^= 1u;
        }
    }
    __device__ __forceinline__ void skip(int n, int nst) {
        for (int k = 0; k < n; k++) adv(nst);
    }
};

struct PkRing {
    unsigned char *stages;
    uint64_t *full, *empty;
    int nst;
};

__device__ __forceinline__ bool pk_slot(const PkParams &p, const PkRing &r, const PkStream &st, unsigned char *&dst,
                                        uint64_t *&bar) {
    if (st.i >= static_cast<uint32_t>(r.nst) && !pk_mbar_wait(p, &r.empty[st.s], st.ph ^ 1u)) return false;
    dst = r.stages + static_cast<size_t>(st.s) * GV_STAGE_BYTES;
    bar = &r.full[st.s];
    return true;
}

// The pages [p0, p1) of the sequence that attention CTA c reads (false when
// the position is outside the page table or the RoPE table: no pages).
__device__ __forceinline__ bool pk_att_range(const PkParams &p, int c, int pos, int &p0, int &p1) {
    const int np = pos / 16 + 1;
    const bool ok = pos >= 0 && pos < p.rope_max_pos && np <= p.max_pages;
    const int s = c % p.S;
    p0 = ok ? static_cast<int>(static_cast<long long>(np) * s / p.S) : 0;
    p1 = ok ? static_cast<int>(static_cast<long long>(np) * (s + 1) / p.S) : 0;
    return ok;
}

// Pages [p0, p1) of kv head kvh: tokens of page j of a stage at j * 2 * PB (K)
// and j * 2 * PB + PB (V), PB = 16 * hd * 2 bytes.
__device__ __forceinline__ int pk_pages_per_stage(int hd) { return static_cast<int>(32768 / (2 * 16 * hd * 2)); }

__device__ void pk_producer(const PkParams &p, const PkRing &r, int c, int G, int lane, int pos) {
    PkStream stream = {0u, 0, 0u};
    bool live = true;
    const int PB = 16 * p.hd * 2;
    const int PPS = pk_pages_per_stage(p.hd);
    const int natt = p.S * p.nkv;
    for (int l = 0; l <= p.L && live; l++) {
        for (int kind = (l < p.L ? PH_QKV : PH_LM); kind <= (l < p.L ? PH_DOWN : PH_LM) && live; kind++) {
            if (kind == PH_ATT) {
                int p0, p1;
                if (c >= natt || !pk_att_range(p, c, pos, p0, p1)) continue;
                const int kvh = c / p.S;
                const __half *kp = p.layer[l].k_pool, *vp = p.layer[l].v_pool;
                for (int j0 = p0; j0 < p1 && live; j0 += PPS) {
                    const int n = min(PPS, p1 - j0);
                    const int pg = lane < n ? __ldg(p.page_table + j0 + lane) : -1;
                    const bool okp = lane < n && pg >= 0 && pg < p.n_pages;
                    const unsigned good = __ballot_sync(0xffffffffu, okp);
                    int lv = 1;
                    if (lane == 0) {
                        unsigned char *dst;
                        uint64_t *bar;
                        lv = pk_slot(p, r, stream, dst, bar) ? 1 : 0;
                        if (lv) mbar_arrive_tx_relaxed(bar, static_cast<uint32_t>(__popc(good)) * 2u * PB);
                    }
                    live = __shfl_sync(0xffffffffu, lv, 0) != 0;
                    // every lane with a page issues its two copies (after the expect-tx above)
                    if (live && okp) {
                        const size_t off = (static_cast<size_t>(pg) * p.nkv + kvh) * 16 * p.hd;
                        unsigned char *dst = r.stages + static_cast<size_t>(stream.s) * GV_STAGE_BYTES +
                                             static_cast<size_t>(lane) * 2 * PB;
                        bulk_g2s(dst, kp + off, PB, &r.full[stream.s]);
                        bulk_g2s(dst + PB, vp + off, PB, &r.full[stream.s]);
                    }
                    if (live) stream.adv(r.nst);
                }
                continue;
            }
            const PkMat m = pk_mat(p, kind, l);
            const int a = pk_start(m.T, c, G), b = pk_start(m.T, c + 1, G);
            if (lane == 0) {
                for (int t = a; t < b && live; t++, stream.adv(r.nst)) {
                    unsigned char *dst;
                    uint64_t *bar;
                    live = pk_slot(p, r, stream, dst, bar);
                    if (!live) break;
                    mbar_arrive_tx_relaxed(bar, GV_STAGE_BYTES);
                    bulk_g2s(dst, m.q + static_cast<size_t>(t) * GV_NIB_BYTES, GV_NIB_BYTES, bar);
                    bulk_g2s(dst + GV_NIB_BYTES, m.s + static_cast<size_t>(t) * GV_SC_BYTES, GV_SC_BYTES, bar);
                }
            }
            stream.i = __shfl_sync(0xffffffffu, stream.i, 0);
            stream.s = __shfl_sync(0xffffffffu, stream.s, 0);
            stream.ph = __shfl_sync(0xffffffffu, stream.ph, 0);
            live = __shfl_sync(0xffffffffu, live, 0);
        }
    }
    // no copy may still be landing in shared memory when the CTA exits
    if (lane == 0) {
        const uint32_t first = stream.i > static_cast<uint32_t>(r.nst) ? stream.i - r.nst : 0u;
        for (uint32_t i = first; i < stream.i; i++)
            (void)mbar_wait(&r.full[i % r.nst], static_cast<uint32_t>((i / r.nst) & 1), p.err);
    }
}

// ------------------------------------------------------------- consumers

// floats of the attention-merge scratch (a multiple of 4, so what follows stays 16-byte aligned)
__host__ __device__ constexpr int pk_mrg_floats(int S, int hd) {
    return (2 * PK_MAXG * S + PK_MAXG + S * (PK_MAXG * hd / S + 2) + 64 + 3) & ~3;
}

struct PkSmem {
    float *xs, *ct, *gt;     // staged activations, chunk terms, RMSNorm gains
    float *red;              // [2][8 warps][32] group-1 row sums
    float *att;              // [PK_MAXG][hd + 2] group-1 attention state
    float *mrg;              // merge scratch
    int *misc;               // [0] wait flag, [1] finalised count, [2..] argmax
    float *amv;              // [8]
    int *ami;                // [8]
};

// Stages the phase's input columns: slot i holds column tile (kt_a + i) % KT.
// With RMSNorm the whole row is read for the sum of squares.  Pass 1 stores
// natural order, pass 2 swizzles / pre-scales (gemv_core.cuh).
template <int FMT>
__device__ void pk_stage(const PkParams &p, const float *xin, const float *gamma, int K, int KT, int kt_a, int nslots,
                         const PkSmem &sm, int ctid, int warp, int lane) {
    const int CS = nslots * GV_TC;
    float4 *xs4 = reinterpret_cast<float4 *>(sm.xs);
    float4 *gt4 = reinterpret_cast<float4 *>(sm.gt);
    const float4 *x4 = reinterpret_cast<const float4 *>(xin);
    const bool norm = gamma != nullptr;
    float ss = 0.0f;
    if (norm) {
        // whole row (sum of squares), keeping the staged columns
        const int n4 = K / 4;
        for (int b0 = 0; b0 < n4; b0 += 8 * PK_CT) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; u++) {
                const int e = b0 + u * PK_CT + ctid;
                v[u] = e < n4 ? __ldcg(x4 + e) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            }
#pragma unroll
            for (int u = 0; u < 8; u++) {
                const int e = b0 + u * PK_CT + ctid;
                ss = fma_rn(v[u].x, v[u].x, ss);
                ss = fma_rn(v[u].y, v[u].y, ss);
                ss = fma_rn(v[u].z, v[u].z, ss);
                ss = fma_rn(v[u].w, v[u].w, ss);
                if (e < n4) {
                    const int kt = e / 128;
                    const int slot = (kt - kt_a + KT) % KT;
                    if (slot < nslots) xs4[slot * 128 + (e & 127)] = v[u];
                }
            }
        }
        // the staged columns' gains, and zeros past K
        for (int j0 = 0; j0 < nslots * 128; j0 += 8 * PK_CT) {
            float4 g[8];
#pragma unroll
            for (int u = 0; u < 8; u++) {
                const int j = j0 + u * PK_CT + ctid;
                const int e = ((kt_a + j / 128) % KT) * 128 + (j & 127);
                g[u] = (j < nslots * 128 && e < n4) ? __ldg(reinterpret_cast<const float4 *>(gamma) + e)
                                                     : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            }
#pragma unroll
            for (int u = 0; u < 8; u++) {
                const int j = j0 + u * PK_CT + ctid;
                if (j < nslots * 128) {
                    gt4[j] = g[u];
                    const int e = ((kt_a + j / 128) % KT) * 128 + (j & 127);
                    if (e >= n4) xs4[j] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                }
            }
        }
    } else {
        const int n4 = K / 4;
        for (int j0 = 0; j0 < nslots * 128; j0 += 8 * PK_CT) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; u++) {
                const int j = j0 + u * PK_CT + ctid;
                const int e = ((kt_a + j / 128) % KT) * 128 + (j & 127);
                v[u] = (j < nslots * 128 && e < n4) ? __ldcg(x4 + e) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            }
#pragma unroll
            for (int u = 0; u < 8; u++) {
                const int j = j0 + u * PK_CT + ctid;
                if (j < nslots * 128) xs4[j] = v[u];
            }
        }
    }
    float rnorm = 0.0f;
    if (norm) {
        ss = warp_sum(ss);
        if (lane == 0) sm.mrg[warp] = ss;
        pk_sync();
        float t = 0.0f;
        for (int w = 0; w < PK_CW; w++) t += sm.mrg[w];
        rnorm = 1.0f / sqrtf(t / static_cast<float>(K) + p.eps);
    }
    pk_sync();
    // pass 2: a warp per chunk, in place
    for (int cl = warp; cl < CS; cl += PK_CW) {
        float v = sm.xs[cl * 32 + lane];
        if (norm) v = (v * rnorm) * sm.gt[cl * 32 + lane];
        __syncwarp();
        stage_x<FMT>(sm.xs, sm.ct, CS, 0, cl, lane, v);
    }
    pk_sync();
}

// Epilogue of one finalised 8-row group (all lanes of the half-warp's warp
// call it; lanes with (lane & 1) == 0 hold row (lane >> 1) & 7).
template <int FMT>
__device__ __forceinline__ void pk_epilogue(const PkParams &p, int kind, const PkMat &m, int rg, int lane, float tot,
                                            bool act, float &bestv, int &besti) {
    const int r = (lane >> 1) & 7;
    const bool gu = kind == PH_GU;
    float v = tot;
    if constexpr (FMT == BW_FMT_Q4_0) v = v * 281474976710656.0f;   // 2^48 undoes the activation pre-scale
    else v = v * ((gu && r >= 4) ? m.ts_up : m.ts);
    const int RG = m.N / 8;
    if (gu) {
        const float up = __shfl_down_sync(0xffffffffu, v, 8);
        if (act && (lane & 1) == 0 && r < 4 && rg < RG) p.act[rg * 4 + r] = (v / (1.0f + expf(-v))) * up;
        return;
    }
    if (!act || (lane & 1) != 0 || rg >= RG) return;
    const int n = rg * 8 + r;
    if (kind == PH_QKV) {
        p.qkv[n] = v;
    } else if (kind == PH_O || kind == PH_DOWN) {
        p.x[n] = __ldcg(p.x + n) + v;
    } else {
        if (p.logits) p.logits[n] = v;
        if (better(v, n, bestv, besti)) {
            bestv = v;
            besti = n;
        }
    }
}

template <int FMT>
__device__ void pk_gemv_phase(const PkParams &p, int kind, int l, const PkRing &rg_ring, const PkSmem &sm,
                              PkStream &stream, int &par, int c, int G, int ctid, int warp, int lane,
                              float &bestv, int &besti) {
    const PkMat m = pk_mat(p, kind, l);
    const int a = pk_start(m.T, c, G), b = pk_start(m.T, c + 1, G);
    const int gid = warp >> 3, wig = warp & 7;
    if (a >= b) return;
    // wait for the input
    unsigned wc;
    uint32_t target;
    const float *xin;
    const float *gamma = nullptr;
    if (kind == PH_QKV) {
        wc = PKC_X; target = p.H / 32 + l * (p.H / 8); xin = p.x; gamma = p.layer[l].attn_norm;
    } else if (kind == PH_O) {
        wc = PKC_ATT; target = (l + 1) * p.S * p.nkv; xin = p.attn;
    } else if (kind == PH_GU) {
        wc = PKC_O; target = (l + 1) * (p.H / 8); xin = p.x; gamma = p.layer[l].ffn_norm;
    } else if (kind == PH_DOWN) {
        wc = PKC_GU; target = (l + 1) * (2 * p.F / 8); xin = p.act;
    } else {
        wc = PKC_X; target = p.H / 32 + p.L * (p.H / 8); xin = p.x; gamma = p.final_norm;
    }
    if (!pk_wait(p, wc, target, ctid, sm.misc)) {
        stream.skip(b - a, rg_ring.nst);
        return;
    }
    const int kt_a = a % m.KT;
    const int nslots = min(b - a, m.KT);
    pk_stage<FMT>(p, xin, gamma, m.K, m.KT, kt_a, nslots, sm, ctid, warp, lane);
    const int CS = nslots * GV_TC;
    const uint32_t stages_a = smem_u32(rg_ring.stages), xs_a = smem_u32(sm.xs), ct_a = smem_u32(sm.ct);
    if (ctid == 0) sm.misc[1] = 0;
    float acc[8][1];
#pragma unroll
    for (int r = 0; r < 8; r++) acc[r][0] = 0.0f;
    const int RG = m.N / 8;
    const int rb_first = a / m.KT;
    const ChunkLane cn = chunk_lane(wig, lane);
    for (int t = a; t < b; t++, stream.adv(rg_ring.nst)) {
        const int rb = t / m.KT, kt = t - rb * m.KT;
        if (static_cast<int>(stream.i & 1) == gid) {
            const int s = stream.s;
            (void)pk_mbar_wait(p, &rg_ring.full[s], stream.ph);
            const int slot = (kt - kt_a + m.KT) % m.KT;
            stage_chunk<FMT, 1>(stages_a + static_cast<uint32_t>(s) * GV_STAGE_BYTES, cn, xs_a, ct_a,
                                slot * GV_TC + (lane & 15), CS, acc);
            __syncwarp();
            if (lane == 0) mbar_arrive_relaxed(&rg_ring.empty[s]);
        }
        if (kt != m.KT - 1 && t != b - 1) continue;
        // end of this CTA's segment of row block rb
        float tot[1];
        reduce_rows16<1>(acc, lane, tot);
#pragma unroll
        for (int r = 0; r < 8; r++) acc[r][0] = 0.0f;
        float *red = sm.red + (par * 8 + wig) * 32;
        if (gid == 1) red[lane] = tot[0];
        pk_sync();
        par ^= 1;
        if (gid == 1) continue;
        const float v0 = tot[0] + red[lane];
        const int rg = rb * 16 + 2 * wig + (lane >> 4);
        const int c_lo = pk_owner(m.T, rb * m.KT, G), c_hi = pk_owner(m.T, rb * m.KT + m.KT - 1, G);
        const int r8 = (lane >> 1) & 7;
        const int row = (2 * wig + (lane >> 4)) * 8 + r8;   // row within the 128-row block
        if (c_lo == c_hi) {
            pk_epilogue<FMT>(p, kind, m, rg, lane, v0, true, bestv, besti);
            if ((lane & 15) == 0 && rg < RG) atomicAdd(sm.misc + 1, 1);
            continue;
        }
        // split K: leave this CTA's partial; the last to arrive adds them in column order
        const int myslot = rb == rb_first ? 0 : 1;
        if ((lane & 1) == 0 && rg < RG) __stcg(p.part + (static_cast<size_t>(c) * 2 + myslot) * 128 + row, v0);
        __threadfence();
        __syncwarp();
        uint32_t old = 0;
        if ((lane & 15) == 0 && rg < RG) old = atomicAdd(p.cnt + PKC_RG + rg, 1u);
        old = __shfl_sync(0xffffffffu, old, lane & 16);
        const bool last = rg < RG && old == static_cast<uint32_t>(c_hi - c_lo);
        float sum = 0.0f;
        if (last) {
            __threadfence();
            if ((lane & 1) == 0) {
                for (int c2 = c_lo; c2 <= c_hi; c2++) {
                    const int sl = (rb == pk_start(m.T, c2, G) / m.KT) ? 0 : 1;
                    sum += __ldcg(p.part + (static_cast<size_t>(c2) * 2 + sl) * 128 + row);
                }
            }
        }
        pk_epilogue<FMT>(p, kind, m, rg, lane, sum, last, bestv, besti);
        if (last && (lane & 15) == 0) {
            p.cnt[PKC_RG + rg] = 0u;
            atomicAdd(sm.misc + 1, 1);
        }
    }
    // phase completion: the row groups this CTA finalised
    pk_sync();
    const int fin = sm.misc[1];
    unsigned done = kind == PH_QKV ? PKC_QKV : kind == PH_O ? PKC_O : kind == PH_GU ? PKC_GU
                  : kind == PH_DOWN ? PKC_X : PKC_AM;
    if (kind != PH_LM) pk_signal(p, done, static_cast<uint32_t>(fin), ctid);
}

// scores of 8 tokens: every lane holds its dims' partial dot per token; returns
// all 8 totals in every lane (transposed butterfly, then a broadcast)
__device__ __forceinline__ void pk_dot8(float (&v)[8], float (&out)[8], int lane) {
    float t4[4], t2[2];
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float send = b4 ? v[i] : v[i + 4];
        const float keep = b4 ? v[i + 4] : v[i];
        t4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 2; i++) {
        const float send = b3 ? t4[i] : t4[i + 2];
        const float keep = b3 ? t4[i + 2] : t4[i];
        t2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    float t1;
    {
        const float send = b2 ? t2[0] : t2[1];
        const float keep = b2 ? t2[1] : t2[0];
        t1 = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    t1 += __shfl_xor_sync(0xffffffffu, t1, 2);
    t1 += __shfl_xor_sync(0xffffffffu, t1, 1);
    // lane l now holds the total of token (l >> 2) & 7
#pragma unroll
    for (int j = 0; j < 8; j++) out[j] = __shfl_sync(0xffffffffu, t1, j << 2);
}

// online softmax state of one query head in one warp: lane holds DPL dims
template <int DPL>
struct PkAtt {
    float m, l;
    float o[DPL];
};

template <int DPL>
__device__ __forceinline__ void pk_att_update(PkAtt<DPL> &st, const float (&s)[8], const float (&vv)[8][DPL]) {
    float mb = s[0];
#pragma unroll
    for (int j = 1; j < 8; j++) mb = fmaxf(mb, s[j]);
    const float mn = fmaxf(st.m, mb);
    if (mn == -INFINITY) return;   // nothing valid yet
    const float corr = st.m == -INFINITY ? 0.0f : expf(st.m - mn);
    float pj[8], ps = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; j++) {
        pj[j] = s[j] == -INFINITY ? 0.0f : expf(s[j] - mn);
        ps += pj[j];
    }
    st.l = fmaf(st.l, corr, ps);
#pragma unroll
    for (int d = 0; d < DPL; d++) {
        float o = st.o[d] * corr;
#pragma unroll
        for (int j = 0; j < 8; j++) o = fmaf(pj[j], vv[j][d], o);
        st.o[d] = o;
    }
    st.m = mn;
}

__device__ __forceinline__ void ld_half_dims(const unsigned char *row, int lane, float *out, int dpl) {
    if (dpl == 4) {
        const uint2 u = *reinterpret_cast<const uint2 *>(row + lane * 8);
        const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&u.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&u.y));
        out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
    } else {
        const uint32_t u = *reinterpret_cast<const uint32_t *>(row + lane * 4);
        const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&u));
        out[0] = a.x; out[1] = a.y;
    }
}

// RoPE'd values of this lane's dims of one head vector h (hd dims) at `pos`
template <int DPL>
__device__ __forceinline__ void pk_rope(const PkParams &p, const float *h, int pos, int lane, float (&out)[DPL]) {
    const int hd = p.hd, half = hd / 2;
#pragma unroll
    for (int k = 0; k < DPL; k++) {
        const int d = lane * DPL + k;
        const int i = d < half ? d : d - half;
        const float a = __ldcg(h + i), b = __ldcg(h + i + half);
        const float cs = __ldg(p.rope_cos + static_cast<size_t>(pos) * half + i);
        const float sn = __ldg(p.rope_sin + static_cast<size_t>(pos) * half + i);
        out[k] = d < half ? __fsub_rn(__fmul_rn(a, cs), __fmul_rn(b, sn)) : __fadd_rn(__fmul_rn(b, cs), __fmul_rn(a, sn));
    }
}

template <int DPL>
__device__ void pk_att_phase(const PkParams &p, int l, const PkRing &ring, const PkSmem &sm, PkStream &stream, int c,
                             int ctid, int warp, int lane, int pos) {
    const int natt = p.S * p.nkv;
    if (c >= natt) return;
    const int hd = p.hd, G = p.G;
    const int kvh = c / p.S, s = c % p.S;
    const int np = pos / 16 + 1;
    const int PB = 16 * hd * 2, PPS = pk_pages_per_stage(hd);
    int p0, p1;
    const bool pos_ok = pk_att_range(p, c, pos, p0, p1);
    const int nstg = (p1 - p0 + PPS - 1) / PPS;
    const int gid = warp >> 3, wig = warp & 7;
    if (!pk_wait(p, PKC_QKV, (l + 1) * ((p.nq + 2 * p.nkv) * hd / 8), ctid, sm.misc)) {
        stream.skip(nstg, ring.nst);
        return;
    }
    if (!pos_ok && ctid == 0) set_error(p.err, BW_DEVERR_BAD_POS);
    const int g = wig;
    const bool head = g < G;
    PkAtt<DPL> st;
    st.m = -INFINITY;
    st.l = 0.0f;
#pragma unroll
    for (int d = 0; d < DPL; d++) st.o[d] = 0.0f;
    float q[DPL];
    if (head && pos_ok) pk_rope<DPL>(p, p.qkv + static_cast<size_t>(kvh * G + g) * hd, pos, lane, q);
    const int last_slot = pos % 16;   // slot of the new token in the last page (not yet in the pool)
    for (int i = 0; i < nstg; i++, stream.adv(ring.nst)) {
        if (static_cast<int>(stream.i & 1) != gid) continue;
        const int sidx = stream.s;
        (void)pk_mbar_wait(p, &ring.full[sidx], stream.ph);
        if (head && pos_ok) {
            const unsigned char *stg = ring.stages + static_cast<size_t>(sidx) * GV_STAGE_BYTES;
            const int j0 = p0 + i * PPS, n = min(PPS, p1 - j0);
            for (int j = 0; j < n; j++) {
                const int pg = __ldg(p.page_table + j0 + j);
                const bool okp = pg >= 0 && pg < p.n_pages;
                const int nvalid = !okp ? 0 : (j0 + j == np - 1 ? last_slot : 16);
                const unsigned char *kb = stg + static_cast<size_t>(j) * 2 * PB, *vb = kb + PB;
#pragma unroll
                for (int half = 0; half < 2; half++) {
                    float pd[8], sc[8], vv[8][DPL];
#pragma unroll
                    for (int t = 0; t < 8; t++) {
                        const int tok = half * 8 + t;
                        float kd[DPL];
                        ld_half_dims(kb + tok * hd * 2, lane, kd, DPL);
                        ld_half_dims(vb + tok * hd * 2, lane, vv[t], DPL);
                        float a = 0.0f;
#pragma unroll
                        for (int d = 0; d < DPL; d++) a = fmaf(q[d], kd[d], a);
                        pd[t] = a;
                    }
                    pk_dot8(pd, sc, lane);
#pragma unroll
                    for (int t = 0; t < 8; t++) {
                        const int tok = half * 8 + t;
                        sc[t] = tok < nvalid ? sc[t] * p.scale : -INFINITY;
                        if (tok >= nvalid) {
#pragma unroll
                            for (int d = 0; d < DPL; d++) vv[t][d] = 0.0f;   // stale slots may hold NaN
                        }
                    }
                    pk_att_update<DPL>(st, sc, vv);
                }
                if (!okp && lane == 0 && g == 0) set_error(p.err, BW_DEVERR_BAD_PAGE);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_relaxed(&ring.empty[sidx]);
    }
    // group 1 hands its state to group 0
    float *gs = sm.att + static_cast<size_t>(g) * (hd + 2);
    if (gid == 1 && head) {
#pragma unroll
        for (int d = 0; d < DPL; d++) gs[lane * DPL + d] = st.o[d];
        if (lane == 0) {
            gs[hd] = st.m;
            gs[hd + 1] = st.l;
        }
    }
    pk_sync();
    if (gid == 0 && head) {
        const float m2 = gs[hd], l2 = gs[hd + 1];
        const float mn = fmaxf(st.m, m2);
        if (mn != -INFINITY) {
            const float c1 = st.m == -INFINITY ? 0.0f : expf(st.m - mn);
            const float c2 = m2 == -INFINITY ? 0.0f : expf(m2 - mn);
            st.l = st.l * c1 + l2 * c2;
#pragma unroll
            for (int d = 0; d < DPL; d++) st.o[d] = st.o[d] * c1 + gs[lane * DPL + d] * c2;
            st.m = mn;
        }
        if (s == p.S - 1 && pos_ok) {
            // the new token: RoPE'd k and v rounded to fp16 (the cache format), written to the pool
            const float *kin = p.qkv + static_cast<size_t>(p.nq) * hd + static_cast<size_t>(kvh) * hd;
            const float *vin = p.qkv + static_cast<size_t>(p.nq + p.nkv) * hd + static_cast<size_t>(kvh) * hd;
            float kr[DPL], kn[DPL], vn[DPL];
            pk_rope<DPL>(p, kin, pos, lane, kr);
#pragma unroll
            for (int d = 0; d < DPL; d++) {
                kn[d] = __half2float(__float2half_rn(kr[d]));
                vn[d] = __half2float(__float2half_rn(__ldcg(vin + lane * DPL + d)));
            }
            const int pg = __ldg(p.page_table + np - 1);
            const bool okp = pg >= 0 && pg < p.n_pages;
            if (g == 0 && okp) {
                const size_t off = ((static_cast<size_t>(pg) * p.nkv + kvh) * 16 + last_slot) * hd + lane * DPL;
#pragma unroll
                for (int d = 0; d < DPL; d++) {
                    p.layer[l].k_pool[off + d] = __float2half_rn(kn[d]);
                    p.layer[l].v_pool[off + d] = __float2half_rn(vn[d]);
                }
            }
            float a = 0.0f;
#pragma unroll
            for (int d = 0; d < DPL; d++) a = fmaf(q[d], kn[d], a);
            const float sc = warp_sum(a) * p.scale;
            const float mn2 = fmaxf(st.m, sc);
            const float c1 = st.m == -INFINITY ? 0.0f : expf(st.m - mn2);
            const float pn = expf(sc - mn2);
            st.l = fmaf(st.l, c1, pn);
#pragma unroll
            for (int d = 0; d < DPL; d++) st.o[d] = fmaf(pn, vn[d], st.o[d] * c1);
            st.m = mn2;
        }
        float *po = p.att_o + (static_cast<size_t>(c) * PK_MAXG + g) * hd;
#pragma unroll
        for (int d = 0; d < DPL; d++) __stcg(po + lane * DPL + d, st.o[d]);
        if (lane == 0) {
            __stcg(p.att_ml + (static_cast<size_t>(c) * PK_MAXG + g) * 2, st.m);
            __stcg(p.att_ml + (static_cast<size_t>(c) * PK_MAXG + g) * 2 + 1, st.l);
        }
    }
    // all S splits of this kv head done -> each merges a slice of the head's outputs
    pk_signal(p, PKC_ARRIVE + kvh, 1, ctid);
    if (!pk_wait(p, PKC_ARRIVE + kvh, (l + 1) * p.S, ctid, sm.misc)) return;
    const int E = G * hd;
    const int e0 = static_cast<int>(static_cast<long long>(E) * s / p.S);
    const int e1 = static_cast<int>(static_cast<long long>(E) * (s + 1) / p.S);
    if (e0 < e1) {
        const int g_lo = e0 / hd, g_hi = (e1 - 1) / hd, ng = g_hi - g_lo + 1;
        const int S = p.S;
        float *wm = sm.mrg;                          // [ng][S] max, then weight
        float *wl = wm + ng * S;                     // [ng][S] sums
        float *hl = wl + ng * S;                     // [ng] total sum
        float *prod = hl + ng;                       // [S][e1 - e0]
        const int c0 = kvh * S;
        for (int i = ctid; i < ng * S; i += PK_CT) {
            const int gg = g_lo + i / S, s2 = i % S;
            wm[i] = __ldcg(p.att_ml + (static_cast<size_t>(c0 + s2) * PK_MAXG + gg) * 2);
            wl[i] = __ldcg(p.att_ml + (static_cast<size_t>(c0 + s2) * PK_MAXG + gg) * 2 + 1);
        }
        pk_sync();
        if (ctid < ng) {
            float M = -INFINITY;
            for (int s2 = 0; s2 < S; s2++) M = fmaxf(M, wm[ctid * S + s2]);
            float L = 0.0f;
            for (int s2 = 0; s2 < S; s2++) {
                const float mm = wm[ctid * S + s2];
                const float w = mm == -INFINITY ? 0.0f : expf(mm - M);
                wm[ctid * S + s2] = w;
                L = fmaf(wl[ctid * S + s2], w, L);
            }
            hl[ctid] = L;
        }
        pk_sync();
        const int ne = e1 - e0;
        for (int i = ctid; i < ne * S; i += PK_CT) {
            const int s2 = i / ne, e = e0 + i % ne;
            const int gg = e / hd, d = e % hd;
            const float w = wm[(gg - g_lo) * S + s2];
            prod[i] = w == 0.0f ? 0.0f : w * __ldcg(p.att_o + (static_cast<size_t>(c0 + s2) * PK_MAXG + gg) * hd + d);
        }
        pk_sync();
        for (int i = ctid; i < ne; i += PK_CT) {
            const int e = e0 + i, gg = e / hd;
            float O = 0.0f;
            for (int s2 = 0; s2 < S; s2++) O += prod[s2 * ne + i];
            p.attn[static_cast<size_t>(kvh) * E + e] = O / hl[gg - g_lo];
        }
    }
    pk_signal(p, PKC_ATT, 1, ctid);
}

template <int FMT, int DPL>
__global__ void __launch_bounds__(PK_THREADS, 1) step_persistent_kernel(const __grid_constant__ PkParams p) {
    extern __shared__ __align__(1024) unsigned char pk_smem[];
    const int c = blockIdx.x, G = gridDim.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    PkRing ring;
    ring.nst = p.nst;
    ring.stages = pk_smem;
    unsigned char *tail = pk_smem + static_cast<size_t>(p.nst) * GV_STAGE_BYTES;
    PkSmem sm;
    sm.xs = reinterpret_cast<float *>(tail);
    tail += static_cast<size_t>(p.nslots) * GV_TC * 32 * 4;
    sm.ct = reinterpret_cast<float *>(tail);
    tail += static_cast<size_t>(p.nslots) * GV_TC * 4;
    sm.gt = reinterpret_cast<float *>(tail);
    tail += static_cast<size_t>(p.nslots) * GV_TC * 32 * 4;
    sm.red = reinterpret_cast<float *>(tail);
    tail += 2 * 8 * 32 * 4;
    sm.att = reinterpret_cast<float *>(tail);
    tail += static_cast<size_t>(PK_MAXG) * (p.hd + 2) * 4;
    sm.mrg = reinterpret_cast<float *>(tail);
    tail += static_cast<size_t>(pk_mrg_floats(p.S, p.hd)) * 4;
    sm.misc = reinterpret_cast<int *>(tail);
    tail += 64 * 4;
    ring.full = reinterpret_cast<uint64_t *>(tail);
    ring.empty = ring.full + p.nst;
    sm.amv = reinterpret_cast<float *>(sm.misc + 16);
    sm.ami = sm.misc + 32;

    __shared__ int s_in[2];   // position and token of this step, read once
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.nst; s++) {
            mbar_init(&ring.full[s], 1);
            mbar_init(&ring.empty[s], GV_CW);
        }
        fence_mbar_init();
        s_in[0] = *p.pos;
        s_in[1] = *p.tokens_in;
    }
    __syncthreads();
    const int pos = s_in[0];

    if (warp == PK_CW) {
        pk_producer(p, ring, c, G, lane, pos);
    } else {
        const int ctid = threadIdx.x;
        PkStream stream = {0u, 0, 0u};
        int par = 0;
        // embedding: x = dequantized row tokens_in[0], 32 columns per CTA and round
        {
            const int tok = s_in[1];
            const bool ok = tok >= 0 && tok < p.V;
            if (!ok && c == 0 && ctid == 0) set_error(p.err, BW_DEVERR_BAD_TOKEN);
            const int KT = gv_col_tiles(p.H), nch = p.H / 32;
            int mine = 0;
            for (int ch = c; ch < nch; ch += G) {
                mine++;
                if (ctid < 32) {
                    float w = 0.0f;
                    if (ok) {
                        const int e = ctid;
                        const size_t tile = static_cast<size_t>(tok / GV_TR) * KT + ch / GV_TC;
                        const int r = tok % GV_TR;
                        const size_t qo = tile * GV_NIB_BYTES + static_cast<size_t>(r) * (GV_TC * 16) +
                                          (((ch % GV_TC) ^ (r % 8)) * 16);
                        const size_t so = tile * GV_SC_BYTES + static_cast<size_t>(r / 8) * (GV_TC * 16) +
                                          (ch % GV_TC) * 16 + (r % 8) * 2;
                        if constexpr (FMT == BW_FMT_Q4_0) {
                            const uint8_t byte = p.emb_q[qo + (e & 15)];
                            const int q = (e >> 4) ? (byte >> 4) : (byte & 15);
                            const uint16_t dh = *reinterpret_cast<const uint16_t *>(p.emb_s + so);
                            w = __fmul_rn(half_bits_to_f(dh), static_cast<float>(q - 8));
                        } else {
                            const uint8_t byte = p.emb_q[qo + (e >> 1)];
                            const float2 v2 = e2m1x2_to_f2(byte);
                            const float ev = (e & 1) ? v2.y : v2.x;
                            const float sv = e4m3_to_f(p.emb_s[so + (e >> 4)]);
                            w = __fmul_rn(__fmul_rn(ev, sv), p.emb_ts);
                        }
                    }
                    p.x[ch * 32 + ctid] = w;
                }
            }
            pk_signal(p, PKC_X, static_cast<uint32_t>(mine), ctid);
        }
        float bestv = -INFINITY;
        int besti = 0x7fffffff;
        for (int l = 0; l < p.L; l++) {
            pk_gemv_phase<FMT>(p, PH_QKV, l, ring, sm, stream, par, c, G, ctid, warp, lane, bestv, besti);
            pk_att_phase<DPL>(p, l, ring, sm, stream, c, ctid, warp, lane, pos);
            pk_gemv_phase<FMT>(p, PH_O, l, ring, sm, stream, par, c, G, ctid, warp, lane, bestv, besti);
            pk_gemv_phase<FMT>(p, PH_GU, l, ring, sm, stream, par, c, G, ctid, warp, lane, bestv, besti);
            pk_gemv_phase<FMT>(p, PH_DOWN, l, ring, sm, stream, par, c, G, ctid, warp, lane, bestv, besti);
        }
        pk_gemv_phase<FMT>(p, PH_LM, p.L, ring, sm, stream, par, c, G, ctid, warp, lane, bestv, besti);
        // greedy argmax: this CTA's best, then the last CTA reduces
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bestv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, besti, o);
            if (better(ov, oi, bestv, besti)) {
                bestv = ov;
                besti = oi;
            }
        }
        if (lane == 0 && warp < 8) {
            sm.amv[warp] = bestv;
            sm.ami[warp] = besti;
        }
        pk_sync();
        if (ctid == 0) {
            float v = sm.amv[0];
            int i = sm.ami[0];
            for (int w = 1; w < 8; w++)
                if (better(sm.amv[w], sm.ami[w], v, i)) {
                    v = sm.amv[w];
                    i = sm.ami[w];
                }
            __stcg(p.am_val + c, v);
            __stcg(p.am_idx + c, i);
            __threadfence();
            const bool last = atomicAdd(p.cnt + PKC_BASE + PKC_AM, 1u) == static_cast<uint32_t>(G - 1);
            if (last) {
                __threadfence();
                float bv = -INFINITY;
                int bi = 0x7fffffff;
                for (int b = 0; b < G; b++) {
                    const float vv = __ldcg(p.am_val + b);
                    const int ii = __ldcg(p.am_idx + b);
                    if (better(vv, ii, bv, bi)) {
                        bv = vv;
                        bi = ii;
                    }
                }
                const int tok = bi == 0x7fffffff ? 0 : bi;
                p.tokens_out[0] = tok;
                if (p.advance) {
                    p.tokens_in[0] = tok;
                    p.pos[0] = pos + 1;
                }
            }
        }
    }
    // leave: the last CTA out resets the step's counters
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const bool last = atomicAdd(p.cnt + PKC_BASE + PKC_EXIT, 1u) == static_cast<uint32_t>(G - 1);
        if (last) {
            __threadfence();
            const bool aborted = p.cnt[PKC_BASE + PKC_ABORT] != 0;
            for (unsigned i = 0; i < PKC_ARRIVE + PK_MAXKV; i++) p.cnt[PKC_BASE + i] = 0u;
            if (aborted) {
                // counters a cut-short phase may have left behind
                const int maxrg = max(max((p.nq + 2 * p.nkv) * p.hd, 2 * p.F), max(p.H, p.V)) / 8;
                for (int i = 0; i < maxrg; i++) p.cnt[PKC_RG + i] = 0u;
            }
        }
    }
}

// ------------------------------------------------------------------- host

static size_t pk_smem_bytes(int nst, int nslots, int hd, int S) {
    return static_cast<size_t>(nst) * GV_STAGE_BYTES + static_cast<size_t>(nslots) * GV_TC * 32 * 4 * 2 +
           static_cast<size_t>(nslots) * GV_TC * 4 + 2 * 8 * 32 * 4 + static_cast<size_t>(PK_MAXG) * (hd + 2) * 4 +
           static_cast<size_t>(pk_mrg_floats(S, hd)) * 4 + 64 * 4 +
           2 * static_cast<size_t>(nst) * 8;
}

struct PkPlan {
    int grid, S, nslots, nst;
    size_t smem;
};

static int pk_max_slots(const bw_model *m, int grid) {
    auto slots = [&](int N, int K) {
        const int RB = gv_row_blocks(N), KT = gv_col_tiles(K);
        const long long T = static_cast<long long>(RB) * KT;
        const int per = static_cast<int>((T + grid - 1) / grid);
        return min(per, KT);
    };
    int s = slots((m->nq + 2 * m->nkv) * m->hd, m->H);
    s = max(s, slots(m->H, m->nq * m->hd));
    s = max(s, slots(2 * m->F, m->H));
    s = max(s, slots(m->H, m->F));
    s = max(s, slots(m->V, m->H));
    return s;
}

// Whether the persistent step applies, and its launch shape.
static bool pk_plan(const bw_model *m, PkPlan *pl) {
    if (m->n_experts != 0 || m->L > PK_MAXL || m->L <= 0) return false;
    if (m->hd != 128 && m->hd != 64) return false;
    if (m->nq % m->nkv || m->nq / m->nkv > PK_MAXG || m->nkv > PK_MAXKV) return false;
    if (m->H % 512 != 0 && m->H % 32 != 0) return false;
    const int grid = sm_count();
    if (grid / m->nkv < 1) return false;
    if (m->V / 8 + static_cast<int>(PKC_RG) > static_cast<int>(CNT_ATTN)) return false;
    if (max(max((m->nq + 2 * m->nkv) * m->hd, 2 * m->F), m->H) / 8 + static_cast<int>(PKC_RG) >
        static_cast<int>(CNT_ATTN))
        return false;
    const int S = grid / m->nkv;
    const int ns = pk_max_slots(m, grid);
    if (ns > PK_MAXSLOTS) return false;
    int nst = 0;
    for (int n = 6; n >= 3; n--)
        if (pk_smem_bytes(n, ns, m->hd, S) <= 227 * 1024 - 1024) {
            nst = n;
            break;
        }
    if (!nst) return false;
    pl->grid = grid;
    pl->S = S;
    pl->nslots = ns;
    pl->nst = nst;
    pl->smem = pk_smem_bytes(nst, ns, m->hd, S);
    return true;
}

bool persistent_step_applies(const bw_model *m, int B, int n_rows) {
    PkPlan pl;
    return B == 1 && n_rows == 1 && pk_plan(m, &pl);
}

size_t persistent_scratch_bytes(const bw_model *m) {
    PkPlan pl;
    if (!pk_plan(m, &pl)) return 0;
    return align_up(static_cast<size_t>(pl.grid) * 2 * 128 * 4, BW_WS_ALIGN) +
           align_up(static_cast<size_t>(pl.grid) * PK_MAXG * 2 * 4, BW_WS_ALIGN) +
           align_up(static_cast<size_t>(pl.grid) * PK_MAXG * m->hd * 4, BW_WS_ALIGN) +
           2 * align_up(static_cast<size_t>(pl.grid) * 4, BW_WS_ALIGN);
}

template <int FMT, int DPL>
static bw_status pk_go(const PkParams &p, const PkPlan &pl, cudaStream_t st) {
    static size_t attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return BW_ERR_CUDA;
    {
        static std::mutex mu;   // host threads may call the library concurrently
        std::lock_guard<std::mutex> lk(mu);
        if (attr_set[dev] < pl.smem) {
            if (cudaFuncSetAttribute(step_persistent_kernel<FMT, DPL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(pl.smem)) != cudaSuccess) {
                (void)cudaGetLastError();
                return BW_ERR_CUDA;
            }
            attr_set[dev] = pl.smem;
        }
    }
    // every CTA must be resident at once (they wait for each other)
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, step_persistent_kernel<FMT, DPL>, PK_THREADS,
                                                      pl.smem) != cudaSuccess ||
        per_sm < 1) {
        (void)cudaGetLastError();
        return BW_ERR_UNSUPPORTED_SHAPE;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.grid);
    cfg.blockDim = dim3(PK_THREADS);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, step_persistent_kernel<FMT, DPL>, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return BW_ERR_CUDA;
    }
    return BW_OK;
}

bw_status persistent_step_launch(const bw_model *m, const bw_kv *kv, int32_t *tokens_in, int32_t *pos,
                                 int32_t *tokens_out, float *logits, bool advance, float *x, float *qkv, float *attn,
                                 float *act, char *scratch, const Scratch &sc, cudaStream_t st) {
    PkPlan pl;
    if (!pk_plan(m, &pl)) return BW_ERR_UNSUPPORTED_SHAPE;
    PkParams p;
    memset(&p, 0, sizeof(p));
    p.L = m->L;
    p.H = m->H;
    p.nq = m->nq;
    p.nkv = m->nkv;
    p.hd = m->hd;
    p.F = m->F;
    p.V = m->V;
    p.G = m->nq / m->nkv;
    p.eps = m->eps;
    p.scale = 1.0f / sqrtf(static_cast<float>(m->hd));
    p.emb_q = static_cast<const uint8_t *>(m->embed.q);
    p.emb_s = static_cast<const uint8_t *>(m->embed.s);
    p.emb_ts = m->embed.ts;
    p.lm_q = static_cast<const uint8_t *>(m->lm_head.q);
    p.lm_s = static_cast<const uint8_t *>(m->lm_head.s);
    p.lm_ts = m->lm_head.ts;
    p.final_norm = m->final_norm;
    p.rope_cos = m->rope_cos;
    p.rope_sin = m->rope_sin;
    p.rope_max_pos = m->rope_max_pos;
    p.page_table = kv->page_table;
    p.max_pages = kv->max_pages;
    p.n_pages = kv->n_pages;
    p.tokens_in = tokens_in;
    p.pos = pos;
    p.tokens_out = tokens_out;
    p.logits = logits;
    p.advance = advance ? 1 : 0;
    p.x = x;
    p.qkv = qkv;
    p.attn = attn;
    p.act = act;
    Carver cv(scratch);
    p.part = cv.take<float>(static_cast<size_t>(pl.grid) * 2 * 128);
    p.att_ml = cv.take<float>(static_cast<size_t>(pl.grid) * PK_MAXG * 2);
    p.att_o = cv.take<float>(static_cast<size_t>(pl.grid) * PK_MAXG * m->hd);
    p.am_val = cv.take<float>(pl.grid);
    p.am_idx = cv.take<int>(pl.grid);
    p.cnt = sc.cnt;
    p.err = sc.err;
    p.nst = pl.nst;
    p.S = pl.S;
    p.nslots = pl.nslots;
    for (int l = 0; l < m->L; l++) {
        const bw_layer &ly = m->layers[l];
        PkLayer &d = p.layer[l];
        d.qkv_q = static_cast<const uint8_t *>(ly.wqkv.q);
        d.qkv_s = static_cast<const uint8_t *>(ly.wqkv.s);
        d.o_q = static_cast<const uint8_t *>(ly.wo.q);
        d.o_s = static_cast<const uint8_t *>(ly.wo.s);
        d.gu_q = static_cast<const uint8_t *>(ly.wgu.q);
        d.gu_s = static_cast<const uint8_t *>(ly.wgu.s);
        d.d_q = static_cast<const uint8_t *>(ly.wd.q);
        d.d_s = static_cast<const uint8_t *>(ly.wd.s);
        d.attn_norm = ly.attn_norm;
        d.ffn_norm = ly.ffn_norm;
        d.k_pool = static_cast<__half *>(kv->k[l]);
        d.v_pool = static_cast<__half *>(kv->v[l]);
        d.ts_qkv = ly.wqkv.ts;
        d.ts_o = ly.wo.ts;
        d.ts_g = ly.wgu.ts;
        d.ts_u = ly.wgu.ts_up;
        d.ts_d = ly.wd.ts;
    }
    const int fmt = m->embed.fmt;
    if (fmt == BW_FMT_Q4_0)
        return m->hd == 128 ? pk_go<BW_FMT_Q4_0, 4>(p, pl, st) : pk_go<BW_FMT_Q4_0, 2>(p, pl, st);
    return m->hd == 128 ? pk_go<BW_FMT_NVFP4, 4>(p, pl, st) : pk_go<BW_FMT_NVFP4, 2>(p, pl, st);
}

}  // namespace bw
