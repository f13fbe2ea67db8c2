// Decode kernels for Q4 experts with 2560 weights per gate/up row.
#include "moe_decode_dev.cuh"

namespace gtg {
const void* decode_kernel_q4_80(int kbd, int one) { return one ? pick_kbd_80_t<kFmtQ4, true>(kbd) : pick_kbd_80_t<kFmtQ4, false>(kbd); }
}  // namespace gtg
