// decode_d128.cu -- decode kernel instances for head dimension 128.
#include "decode_dispatch.cuh"

namespace qkv {
bool decode_ops_d128(int bits, int gs, bool q8, int nc, bool f32, int var, DecodeOps* ops) {
  return decode_ops_for<128>(bits, gs, q8, nc, f32, var, ops);
}
}  // namespace qkv
