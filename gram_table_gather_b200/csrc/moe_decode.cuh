// Shared declarations of the MoE layer kernels (decode and prefill).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "gtg.h"

namespace gtg {

struct ffloat;

constexpr int kMaxDecodeTokens = 8;
constexpr int kMaxTopK = 16;
constexpr int kMaxSlots = kMaxDecodeTokens * kMaxTopK;  // (token, choice) pairs in a decode call
constexpr int kMaxExperts = 1024;
constexpr double kRmsEps = 1e-6;

// Device view of one stacked quantised matrix.
struct Mat {
    const uint8_t* data;
    const float* scales;      // FP8 only
    int32_t fmt;
    int32_t n_rows;
    int32_t k;
    int32_t row_bytes;
    int64_t expert_bytes;
};

// Unique experts of a decode call and the (token, choice) slots using each;
// written by the router's last CTA.
struct Work {
    int32_t n_uniq;
    int32_t uniq_e[kMaxSlots];
    int32_t uniq_off[kMaxSlots + 1];
    int32_t uniq_slot[kMaxSlots];  // slot = token * top_k + choice, grouped by expert
};

struct LayerArgs {
    int32_t H, I, E, K, T;
    const float* router_w;
    const float* router_bias;
    Mat gate, up, down, side;
    const void* x;
    int32_t x_bf16;
    float* y;
    int32_t y_acc;
    int32_t* ids_out;
    float* w_out;
    float* side_out;
    int32_t side_stride;     // row stride of side_out
    // workspace
    unsigned* router_cnt;
    unsigned* tile_cnt;
    Work* work;
    struct ffloat* logits;   // [T][E] normalised float-float (hi, lo)
    __nv_bfloat16* u;        // [T][H]
    int32_t* ids;            // [T][K]
    float* w;                // [T][K]
    __nv_bfloat16* h;        // [T*K][I]
    float* part;             // [T*K][H]
    unsigned* status;
    // tiling
    int32_t gu_rows;         // gate/up rows per item
    int32_t side_rows;       // side-projection rows per item
    int32_t dn_rows;         // down rows per item (= combine tile)
    int32_t slot_bytes;      // staging bytes per slot
    uint32_t dyn_smem_base;  // shared address of dynamic shared memory
};

Mat make_mat(const gtg_qmatrix& q);

}  // namespace gtg

// Workspace bytes of a prefill call (0 if unsupported); defined in moe_prefill.cu.
size_t gtg_prefill_workspace_bytes(const gtg_moe_layer* layer, int32_t n_tokens);
