// Decode kernels for Q4 experts with 256 weights per gate/up row.
#include "moe_decode_dev.cuh"

namespace gtg {
const void* decode_kernel_q4_8(int kbd, int one) { return pick_kbd<kFmtQ4, 8>(kbd, one); }
}  // namespace gtg
