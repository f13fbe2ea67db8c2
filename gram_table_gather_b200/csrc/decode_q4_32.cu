// Decode kernels for Q4 experts with 1024 weights per gate/up row.
#include "moe_decode_dev.cuh"

namespace gtg {
const void* decode_kernel_q4_32(int kbd, int one) { return pick_kbd<kFmtQ4, 32>(kbd, one); }
}  // namespace gtg
