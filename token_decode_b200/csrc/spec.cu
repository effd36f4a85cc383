// spec.cu -- acceptance step of a speculative verify pass (sm_100a).
//
// The verify pass (bw_decode_step with n_rows = K + 1) runs the last accepted
// token t0 and the K draft tokens d1..dK of each sequence as consecutive rows
// sharing one KV cache, and returns the greedy token a_r after every row r.
// The "bw24" deep-dive page (10100.com), section 5, stage 4, describes that
// verify kernel: from the first draft that does not match, the later rows are
// masked out.  Section 1 of the same page fixes what that must preserve: the
// speculative output is token for token the plain greedy output.  So draft
// d_i stands while d_1..d_i all equal the greedy token of the row before
// (d_i == a_{i-1}); with n drafts standing, the pass has produced n + 1 new
// tokens, d_1..d_n followed by a_n.
#include "bw_common.cuh"

namespace bw {

__global__ void spec_accept_kernel(const int32_t *rows, const int32_t *am, int B, int n_rows,
                                   int32_t *n_accept, int32_t *next, int next_stride, int32_t *pos) {
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B) return;
    const int32_t *r = rows + static_cast<size_t>(b) * n_rows;
    const int32_t *a = am + static_cast<size_t>(b) * n_rows;
    int n = 0;
    while (n + 1 < n_rows && r[n + 1] == a[n]) n++;
    const int32_t nxt = a[n];   // read every row of b before a possibly aliased write
    n_accept[b] = n;
    if (next) next[static_cast<size_t>(b) * next_stride] = nxt;
    if (pos) pos[b] += n + 1;
}

}  // namespace bw

extern "C" {

bw_status bw_spec_accept(const int32_t *tokens_in, const int32_t *tokens_out, int B, int n_rows,
                         int32_t *n_accept, int32_t *next_out, int next_stride, int32_t *pos,
                         void *stream) {
    if (!tokens_in || !tokens_out || !n_accept || B <= 0 || n_rows <= 0 || n_rows > BW_MAX_VERIFY_ROWS)
        return BW_ERR_INVALID_ARG;
    if (next_out && next_stride < 1) return BW_ERR_INVALID_ARG;
    const int threads = 128;
    return bw::launch_pdl(bw::spec_accept_kernel, dim3((B + threads - 1) / threads), dim3(threads), 0,
                          static_cast<cudaStream_t>(stream), tokens_in, tokens_out, B, n_rows, n_accept,
                          next_out, next_stride, pos);
}

}  // extern "C"
