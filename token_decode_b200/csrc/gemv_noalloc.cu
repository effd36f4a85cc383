// gemv_noalloc.cu -- the Q4_0 GEMV for callers that cannot allocate device
// memory.
//
// bw_gemv_q4_0 needs a caller-provided workspace (split-K partial sums,
// self-resetting counters, argmax partials).  Some callers have no way to
// provide one: a host framework that owns every device allocation and hands
// a library only its inputs and outputs, or a code path where cudaMalloc's
// implicit device-wide synchronization is not acceptable.  For them this
// entry point runs the very same kernel with its scratch in a fixed,
// file-scope device array of BW_GEMV_NOALLOC_SCRATCH_BYTES, which every GPU
// that loads the library keeps until the process exits.
#include "bw_common.cuh"

namespace bw {
namespace {

// error word + counters (the first BW_WS_HDR_BYTES), then the kernel scratch
static __device__ __align__(256) unsigned char g_noalloc_scratch[BW_GEMV_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch, looked up once per device.  In host
// code the array's name is only a host-side stand-in, so the address must
// come from cudaGetSymbolAddress with that device current.
void *g_noalloc_ptr[64] = {};
std::mutex g_noalloc_mu;   // host threads may call the library concurrently

}  // namespace

// The scratch array's device address on the current device (looked up on
// first use).  Also used by bw_read_error(NULL, ...), which reads and clears
// the array's error word.
bw_status noalloc_scratch(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        (void)cudaGetLastError();
        return BW_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            (void)cudaGetLastError();
            return BW_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return BW_OK;
}

}  // namespace bw

extern "C" bw_status bw_gemv_q4_0_noalloc(const void *w_q, const void *w_d, int N, int K, const float *x,
                                          int M, const float *gamma, float eps, const float *residual,
                                          float *y, int32_t *argmax_out, unsigned flags, void *stream) {
    if (N <= 0 || K <= 0 || M <= 0) return BW_ERR_INVALID_ARG;
    if (N % 8 || K % 32) return BW_ERR_UNSUPPORTED_SHAPE;
    // the shape must fit the fixed scratch: refuse it rather than overrun
    if (bw::gemv_scratch_bytes(N, K, M) > BW_GEMV_NOALLOC_SCRATCH_BYTES - BW_WS_HDR_BYTES ||
        N / 8 + bw::CNT_GEMV_RG > bw::CNT_ATTN)
        return BW_ERR_UNSUPPORTED_SHAPE;
    void *ws = nullptr;
    bw_status s = bw::noalloc_scratch(&ws);
    if (s != BW_OK) return s;
    const bw::Scratch sc = bw::scratch_of(ws, BW_GEMV_NOALLOC_SCRATCH_BYTES);
    // every argument check runs before anything is queued
    s = bw::gemv_check(BW_FMT_Q4_0, w_q, w_d, N, K, x, M, gamma, residual, y, argmax_out, flags, sc);
    if (s != BW_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // The array keeps whatever the previous call left.  The counters this
    // launch can use must start at zero: clear them (a call cut short by a
    // device-side timeout may have left some behind).  The error word before
    // them is left alone, so a timeout stays visible to bw_read_error(NULL).
    const size_t clear = (16u + bw::CNT_GEMV_RG + static_cast<size_t>(N / 8)) * sizeof(uint32_t);
    if (cudaMemsetAsync(static_cast<char *>(ws) + sizeof(uint32_t), 0, clear - sizeof(uint32_t), st) !=
        cudaSuccess) {
        (void)cudaGetLastError();
        return BW_ERR_CUDA;
    }
    return bw::gemv_launch(BW_FMT_Q4_0, w_q, w_d, 1.0f, 1.0f, N, K, x, M, gamma, eps, residual, y, argmax_out,
                           flags, sc, st);
}
