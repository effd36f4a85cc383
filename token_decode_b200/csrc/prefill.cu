// prefill.cu -- chunked prefill of one sequence (sm_100a).
//
// The "bw24" deep-dive page (10100.com), section 5, stage 3, pushes a long
// prompt through the engine in chunks, one after another: every chunk
// updates the KV cache, and only the last chunk returns logits.  Here a chunk
// of up to `chunk` prompt tokens is one multi-row step of the decode path:
// its rows sit at consecutive positions, each row attends causally to the
// cache and to the rows before it in the chunk, and writes its own K/V row at
// its own position -- so a prefill computes what decoding the prompt one
// token at a time computes (up to fp32 summation order).
#include <algorithm>

#include "bw_common.cuh"

namespace bw {

// positions of the chunks' first rows: pos0, pos0 + chunk, ...
__global__ void prefill_pos_kernel(int32_t *pos, int pos0, int chunk, int n_chunks) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n_chunks) pos[i] = pos0 + i * chunk;
}

struct PrefillBuffers {
    size_t step;     // bytes of the step workspace at the start of ws
    int32_t *pos;    // [max chunks] first position of every chunk
    int32_t *tok;    // [chunk] greedy tokens of the latest chunk
    float *lg;       // [chunk][V] logits of the last chunk
};

// workspace: the step workspace -- the largest any chunk size 1..chunk needs
// (a one-row step also holds the persistent step's scratch) -- then the
// buffers above
static size_t prefill_bytes(const bw_model *m, const bw_kv *kv, int chunk, PrefillBuffers *pb, void *ws) {
    size_t step = 0;
    for (int r = 1; r <= chunk; r++) step = std::max(step, bw_decode_workspace_bytes(m, kv, 1, r));
    const size_t max_chunks = (static_cast<size_t>(kv->max_pages) * 16 + chunk - 1) / chunk;
    size_t off = align_up(step, BW_WS_ALIGN);
    const size_t pos_off = off;
    off = align_up(off + max_chunks * 4, BW_WS_ALIGN);
    const size_t tok_off = off;
    off = align_up(off + static_cast<size_t>(chunk) * 4, BW_WS_ALIGN);
    const size_t lg_off = off;
    off += static_cast<size_t>(chunk) * m->V * 4;
    if (pb) {
        char *w = static_cast<char *>(ws);
        pb->step = step;
        pb->pos = reinterpret_cast<int32_t *>(w + pos_off);
        pb->tok = reinterpret_cast<int32_t *>(w + tok_off);
        pb->lg = reinterpret_cast<float *>(w + lg_off);
    }
    return off;
}

}  // namespace bw

extern "C" {

size_t bw_prefill_workspace_bytes(const bw_model *m, const bw_kv *kv, int chunk) {
    if (!m || !kv || chunk < 1 || chunk > BW_MAX_VERIFY_ROWS || kv->max_pages <= 0 || m->V <= 0)
        return BW_WS_HDR_BYTES;
    return bw::prefill_bytes(m, kv, chunk, nullptr, nullptr);
}

bw_status bw_prefill(const bw_model *m, const bw_kv *kv, const int32_t *tokens, int n, int pos0, int chunk,
                     int32_t *next_token, float *logits, void *ws, size_t ws_bytes, void *stream) {
    using namespace bw;
    if (!m || !kv || !tokens || !next_token || !ws_ok(ws) || n <= 0 || pos0 < 0) return BW_ERR_INVALID_ARG;
    if (chunk < 1 || chunk > BW_MAX_VERIFY_ROWS) return BW_ERR_UNSUPPORTED_SHAPE;
    if (kv->max_pages <= 0 || m->V <= 0) return BW_ERR_INVALID_ARG;
    if (static_cast<long long>(pos0) + n > static_cast<long long>(kv->max_pages) * 16 ||
        static_cast<long long>(pos0) + n > m->rope_max_pos)
        return BW_ERR_INVALID_ARG;
    PrefillBuffers pb;
    if (ws_bytes < prefill_bytes(m, kv, chunk, &pb, ws)) return BW_ERR_INVALID_ARG;
    const int n_chunks = (n + chunk - 1) / chunk;
    const int last = n - (n_chunks - 1) * chunk;   // rows of the last chunk
    int32_t *tok_in = const_cast<int32_t *>(tokens);   // read only: no BW_STEP_ADVANCE
    // every step's host-side checks before the first launch
    bw_status s = bw_decode_step(m, kv, tok_in, pb.pos, 1, n_chunks > 1 ? chunk : last, pb.tok,
                                 n_chunks == 1 && logits ? pb.lg : nullptr, BW_STEP_VALIDATE_ONLY, ws, pb.step, stream);
    if (s != BW_OK) return s;
    if (n_chunks > 1 && last != chunk) {
        s = bw_decode_step(m, kv, tok_in, pb.pos, 1, last, pb.tok, logits ? pb.lg : nullptr, BW_STEP_VALIDATE_ONLY,
                           ws, pb.step, stream);
        if (s != BW_OK) return s;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    prefill_pos_kernel<<<(n_chunks + 255) / 256, 256, 0, st>>>(pb.pos, pos0, chunk, n_chunks);
    if (cudaGetLastError() != cudaSuccess) return BW_ERR_CUDA;
    for (int c = 0; c < n_chunks; c++) {
        const bool fin = c == n_chunks - 1;
        s = bw_decode_step(m, kv, tok_in + static_cast<size_t>(c) * chunk, pb.pos + c, 1, fin ? last : chunk, pb.tok,
                           fin && logits ? pb.lg : nullptr, 0, ws, pb.step, stream);
        if (s != BW_OK) return s;
    }
    // the last prompt token's greedy successor (and its logits)
    if (cudaMemcpyAsync(next_token, pb.tok + (last - 1), 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return BW_ERR_CUDA;
    if (logits && cudaMemcpyAsync(logits, pb.lg + static_cast<size_t>(last - 1) * m->V,
                                  static_cast<size_t>(m->V) * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return BW_ERR_CUDA;
    return BW_OK;
}

}  // extern "C"
