// abi.cu -- status strings, device properties, workspace helpers of libbw.
#include <stdio.h>

#include "bw_common.cuh"

namespace bw {

bw_status noalloc_scratch(void **out);   // gemv_noalloc.cu

int sm_count() {
    static int cached[64] = {};
    static std::mutex mu;   // host threads may call the library concurrently
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lk(mu);
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

// one thread: the error word moves into the caller's accumulator
__global__ void drain_error_kernel(uint32_t *err, uint32_t *dst) {
    if (threadIdx.x == 0) {
        const uint32_t v = atomicExch(err, 0u);
        if (v) atomicOr(dst, v);
    }
}

bw_status launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? BW_OK : BW_ERR_CUDA;
}

}  // namespace bw

extern "C" {

const char *bw_status_string(bw_status s) {
    switch (s) {
        case BW_OK: return "ok";
        case BW_ERR_INVALID_ARG: return "invalid argument";
        case BW_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case BW_ERR_CUDA: return "CUDA error";
        case BW_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case BW_ERR_BAD_PAGE_INDEX: return "page-table entry outside the KV pool";
        default: return "unknown status";
    }
}

int bw_abi_version(void) { return BW_ABI_VERSION; }

bw_status bw_workspace_init(void *ws, size_t bytes, void *stream) {
    if (!bw::ws_ok(ws) || bytes < BW_WS_HDR_BYTES) return BW_ERR_INVALID_ARG;
    if (cudaMemsetAsync(ws, 0, bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        (void)cudaGetLastError();
        return BW_ERR_CUDA;
    }
    return BW_OK;
}

bw_status bw_read_error(void *ws, uint32_t *err_out, void *stream) {
    if (!err_out) return BW_ERR_INVALID_ARG;
    if (!ws) {
        // the error word of bw_gemv_q4_0_noalloc's fixed scratch on this device
        const bw_status s = bw::noalloc_scratch(&ws);
        if (s != BW_OK) return s;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) {
        (void)cudaGetLastError();
        return BW_ERR_CUDA;
    }
    uint32_t v = 0;
    if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemset(ws, 0, sizeof(v)) != cudaSuccess) {
        (void)cudaGetLastError();
        return BW_ERR_CUDA;
    }
    *err_out = v;
    return BW_OK;
}

bw_status bw_drain_error(void *ws, uint32_t *dst, void *stream) {
    if (!dst || (reinterpret_cast<uintptr_t>(dst) & 3u)) return BW_ERR_INVALID_ARG;
    if (ws && !bw::ws_ok(ws)) return BW_ERR_INVALID_ARG;
    if (!ws) {
        const bw_status s = bw::noalloc_scratch(&ws);
        if (s != BW_OK) return s;
    }
    // a plain launch: ordered after all the stream's earlier work
    bw::drain_error_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t *>(ws), dst);
    return bw::launch_status();
}

}  // extern "C"
