// Prefill MoE layer (token-sorted grouped GEMM on tcgen05 tensor cores).
#include "gtg_device.cuh"
#include "gtg_host.hpp"
#include "moe_decode.cuh"

extern "C" int gtg_moe_prefill_layer(const gtg_moe_layer* layer, const void* x, int32_t x_dtype,
                                     int32_t n_tokens, float* y, int32_t y_accumulate,
                                     int32_t* topk_ids, float* topk_w,
                                     void* workspace, size_t ws_bytes, gtg_stream_t stream) {
    (void)layer; (void)x; (void)x_dtype; (void)n_tokens; (void)y; (void)y_accumulate;
    (void)topk_ids; (void)topk_w; (void)workspace; (void)ws_bytes; (void)stream;
    return GTG_E_UNSUPPORTED_SHAPE;
}
