// decode_x_d256.cu -- decode kernel instances for head dimension 256 with affine
// codes stored 2, 3, 5 or 6 bits wide (transcoded per block to 4-bit codes
// for 2 and 3 bits, to 8-bit codes for 5 and 6 bits).
#include "decode_dispatch.cuh"

namespace qkv {
bool decode_ops_x_d256(int bits, int gs, int nc, bool f32, DecodeOps* ops) {
  return decode_ops_x_for<256>(bits, gs, nc, f32, ops);
}
}  // namespace qkv
