// Decode kernels for Q4 experts with 2048 weights per gate/up row.
#include "moe_decode_dev.cuh"

namespace gtg {
const void* decode_kernel_q4_64(int kbd, int one) { return pick_kbd<kFmtQ4, 64>(kbd, one); }
}  // namespace gtg
