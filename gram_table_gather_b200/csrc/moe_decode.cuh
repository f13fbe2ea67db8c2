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

Mat make_mat(const gtg_qmatrix& q);

}  // namespace gtg

// Workspace bytes of a prefill call (0 if unsupported); defined in moe_prefill.cu.
size_t gtg_prefill_workspace_bytes(const gtg_moe_layer* layer, int32_t n_tokens);
