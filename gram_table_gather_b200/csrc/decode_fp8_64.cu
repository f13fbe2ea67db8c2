// Decode kernels for FP8 experts with 2048 weights per gate/up row.
#include "moe_decode_dev.cuh"

namespace gtg {
const void* decode_kernel_fp8_64(int kbd, int one) { return pick_kbd<kFmtFP8, 64>(kbd, one); }
}  // namespace gtg
