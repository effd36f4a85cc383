// moe.cu -- mixture-of-experts FFN (placeholder until the routed path lands).
#include "bw_common.cuh"

namespace bw {

size_t moe_scratch_bytes(const bw_model *m, int R) {
    (void)m;
    (void)R;
    return 0;
}

bw_status moe_ffn_launch(const bw_model *m, const bw_layer *ly, float *x, int R, const Scratch &sc,
                         char *moe_base, cudaStream_t st) {
    (void)m; (void)ly; (void)x; (void)R; (void)sc; (void)moe_base; (void)st;
    return BW_ERR_UNSUPPORTED_SHAPE;
}

}  // namespace bw

extern "C" {

bw_status bw_moe_route_gemv(const bw_model *m, const bw_layer *ly, float *x, int R, int32_t *topk_idx,
                            float *topk_w, void *ws, size_t ws_bytes, void *stream) {
    (void)m; (void)ly; (void)x; (void)R; (void)topk_idx; (void)topk_w; (void)ws; (void)ws_bytes;
    (void)stream;
    return BW_ERR_UNSUPPORTED_SHAPE;
}

size_t bw_moe_workspace_bytes(const bw_model *m, int R) {
    (void)m;
    (void)R;
    return BW_WS_HDR_BYTES;
}

}  // extern "C"
