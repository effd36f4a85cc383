// bw_common.cuh -- device helpers shared by the sm_100a kernels of libbw.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/bw.h"

#define BW_WS_HDR_BYTES (1u << 18)     // error word + counters at the start of a workspace
#define BW_WS_COUNTERS 65000u          // uint32 counters after the error word
#define BW_WS_ALIGN 256u

namespace bw {

// ------------------------------------------------------------ host side

int sm_count();                         // multiprocessors of the current device (cached)
bw_status launch_status();              // BW_OK or BW_ERR_CUDA after a launch

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// A workspace as the ABI requires it: non-null and BW_WS_ALIGN-byte aligned
// (the kernels' scratch regions inherit that alignment).
inline bool ws_ok(const void *ws) { return ws && (reinterpret_cast<uintptr_t>(ws) & (BW_WS_ALIGN - 1)) == 0; }

inline uint32_t *ws_error_word(void *ws) { return static_cast<uint32_t *>(ws); }
inline uint32_t *ws_counters(void *ws) { return static_cast<uint32_t *>(ws) + 16; }

// What a kernel launcher may use of a workspace: the device error word, the
// self-resetting counters, and `bytes` of scratch at `base`.
struct Scratch {
    uint32_t *err;
    uint32_t *cnt;
    char *base;
    size_t bytes;
};

inline Scratch scratch_of(void *ws, size_t ws_bytes) {
    Scratch s;
    s.err = ws_error_word(ws);
    s.cnt = ws_counters(ws);
    s.base = static_cast<char *>(ws) + BW_WS_HDR_BYTES;
    s.bytes = ws_bytes > BW_WS_HDR_BYTES ? ws_bytes - BW_WS_HDR_BYTES : 0;
    return s;
}

// Carves consecutive 256-byte aligned regions out of a scratch area.
struct Carver {
    char *base;
    size_t off;
    explicit Carver(char *b) : base(b), off(0) {}
    template <class T>
    T *take(size_t count) {
        T *p = reinterpret_cast<T *>(base ? base + off : nullptr);
        off = align_up(off + count * sizeof(T), BW_WS_ALIGN);
        return p;
    }
};

// counter regions (uint32 indices into Scratch::cnt)
constexpr unsigned CNT_ARGMAX = 1;
constexpr unsigned CNT_GEMV_RG = 64;
constexpr unsigned CNT_ATTN = 32768;

// internal launchers (host), shared by the single-op entry points and the step.
// Each *_check validates exactly what its launcher would reject, without
// launching, so that a caller composing several launches (the decode step)
// can reject bad arguments before the first one is queued.
size_t gemv_scratch_bytes(int N, int K, int M);
bw_status gemv_check(int fmt, const void *wq, const void *wscales, int N, int K, const float *x, int M,
                     const float *gamma, const float *residual, const float *y, const int32_t *argmax_out,
                     unsigned flags, const Scratch &sc);
bw_status mma_check(int N, int K, int M);
bw_status attn_check(const float *qkv, const float *rope_cos, const float *rope_sin, int rope_max_pos,
                     const void *k_pool, const void *v_pool, const int32_t *page_table, int max_pages, int n_pages,
                     const int32_t *pos, int B, int R, int nq, int nkv, int hd, const float *out, const Scratch &sc);
bw_status embed_check(int fmt, const void *e_q, const void *e_s, int V, int H, const int32_t *tokens, int M,
                      const float *x);
bw_status gemv_launch(int fmt, const void *wq, const void *wscales, float ts, float ts_up, int N, int K,
                      const float *x, int M, const float *gamma, float eps, const float *residual,
                      float *y, int32_t *argmax_out, unsigned flags, const Scratch &sc,
                      cudaStream_t st, int32_t *adv_tokens = nullptr, int32_t *adv_pos = nullptr);
size_t mma_scratch_bytes(int N, int K, int M);
bw_status mma_gemm_launch(const void *wq, const void *wscales, float ts, float ts_up, int N, int K,
                          const float *x, int M, const float *gamma, float eps, const float *residual,
                          float *y, int32_t *argmax_out, unsigned flags, const Scratch &sc, cudaStream_t st,
                          int32_t *adv_tokens, int32_t *adv_pos);
size_t attn_scratch_bytes(int B, int R, int nq, int nkv, int hd, int max_pages);
// early: pos and page_table were written before the launch that precedes
// this one, and that launch (one of this library's projection kernels)
// signals its dependents only after its own dependency wait; the kernel then
// reads them, and starts the K/V copies, before its own wait.
bw_status attn_launch(const float *qkv, const float *rope_cos, const float *rope_sin, int rope_max_pos,
                      void *k_pool, void *v_pool, const int32_t *page_table, int max_pages, int n_pages,
                      const int32_t *pos, int B, int R, int nq, int nkv, int hd, float *out,
                      const Scratch &sc, cudaStream_t st, int kv_fmt = 0, float kscale = 1.0f,
                      float vscale = 1.0f, bool early = false);
bw_status embed_launch(int fmt, const void *e_q, const void *e_s, float ts, int V, int H,
                       const int32_t *tokens, int M, float *x, uint32_t *err, cudaStream_t st);

// Launches `kernel` with programmatic dependent launch enabled, so that its
// CTAs may start (and stream constant weights) while the previous kernel on
// the stream drains; the kernel calls pdl_wait() before touching anything
// the previous kernels wrote.
template <typename... KArgs, typename... Args>
bw_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return BW_ERR_CUDA;
    }
    return BW_OK;
}

// ---------------------------------------------------------- device side

__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// 16-byte streaming load of read-only data that is used once (weights).
__device__ __forceinline__ uint4 ld_stream16(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Plain coherent loads/stores through L2 (data written by other CTAs of the
// same grid).
__device__ __forceinline__ float ld_cg(const float *p) { return __ldcg(p); }

__device__ __forceinline__ float fma_rn(float a, float b, float c) {
    float d;
    asm("fma.rn.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// (value, index) pair that prefers the larger value and, on equal values, the
// lower index (greedy argmax tie rule).
__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
    return v > bv || (v == bv && i < bi);
}

// Two E2M1 codes (low nibble -> .x, high nibble -> .y) to two floats, via the
// sm_100a e2m1x2 -> f16x2 conversion (exact).
__device__ __forceinline__ float2 e2m1x2_to_f2(uint32_t byte) {
    uint32_t h2;
    asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}"
        : "=r"(h2) : "r"(byte));
    __half2 h = *reinterpret_cast<__half2 *>(&h2);
    return __half22float2(h);
}

// Two E4M3 codes (low byte -> .x, high byte -> .y) to two floats (exact).
__device__ __forceinline__ float2 e4m3x2_to_f2(uint32_t two_bytes) {
    uint32_t h2;
    asm("{\n\t.reg .b16 s;\n\tcvt.u16.u32 s, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, s;\n\t}"
        : "=r"(h2) : "r"(two_bytes));
    __half2 h = *reinterpret_cast<__half2 *>(&h2);
    return __half22float2(h);
}

__device__ __forceinline__ float e4m3_to_f(uint32_t byte) { return e4m3x2_to_f2(byte & 0xffu).x; }

__device__ __forceinline__ float half_bits_to_f(uint32_t h) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h)));
}

// Release/acquire fence at GPU scope: with a relaxed atomic after it (writer)
// or before it (reader), orders plain global accesses across CTAs (lighter
// than the sequentially consistent __threadfence).
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

__device__ __forceinline__ void set_error(uint32_t *err, uint32_t bit) {
    if (err) atomicOr(err, bit);
}

// ------------------------------------------------ mbarrier + bulk copies

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: gives up after `limit` polls (each poll may itself suspend
// for a while), records BW_DEVERR_TIMEOUT and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t *err,
                                          uint32_t limit = 1u << 22) {
    for (uint32_t i = 0; i < limit; i++)
        if (mbar_try_wait(bar, parity)) return true;
    set_error(err, BW_DEVERR_TIMEOUT);
    return false;
}
// orders this thread's generic-proxy shared-memory writes before later
// async-proxy accesses (TMA, bulk copies, tensor-core operand reads)
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`
// (16-byte aligned addresses, size a multiple of 16).  No multicast.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

}  // namespace bw
