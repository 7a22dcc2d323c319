// dequantize.cu -- materialize rows [0, L) of a quantized cache as fp16.
//
// The prompt path of llama.cpp #25556 converts the Q8_0 K/V cache to fp16 and
// runs dense attention on it; this kernel is that conversion, for A/B
// comparisons of "materialize, then dense attention" against the fused
// kernels (bench rows materialize_*).  Each output is the correctly rounded
// fp16 of scale * code + bias (Q8_0: scale * code): the product and the sum
// are exact in fp64 (11- and 8-bit operands), so the one rounding is the
// final one -- the same value the CPU oracle's exact dequantization rounds to.
//
// Grid: x = chunks of 8 outputs (16 bytes) over the L rows of one slab,
// y = (batch, kv head) slab; one thread per chunk.
#include "qkv_common.cuh"
#include "qkv_internal.h"

namespace qkv {

struct DequantParams {
  const uint32_t* codes;
  const uint16_t* scales;
  const uint16_t* biases;
  uint16_t* out;            // [B * Hkv, L, D] fp16 bits
  int64_t Lcap;
  int64_t L;
  int D;
  int cshift;               // log2(D / 8): chunks per row
};

template <int BITS, int GS, bool Q8>
__global__ void __launch_bounds__(256) qkv_dequantize_kernel(const __grid_constant__ DequantParams p) {
  const int64_t chunk = (int64_t)blockIdx.x * 256 + threadIdx.x;
  const int64_t j = chunk >> p.cshift;              // row within the slab
  if (j >= p.L) return;
  const int c8 = (int)(chunk & ((1 << p.cshift) - 1));
  const int64_t slab = blockIdx.y;
  const int64_t crow = slab * p.Lcap + j;
  const int ng = p.D / GS;
  const int g = (c8 * 8) / GS;
  const double s = (double)half_bits_to_float(p.scales[crow * ng + g]);
  const double b = Q8 ? 0.0 : (double)half_bits_to_float(p.biases[crow * ng + g]);
  uint32_t w[2];
  uint64_t stream = 0;                              // 2, 3, 5, 6 bits: the chunk's 8 codes
  if constexpr (BITS == 4) {
    w[0] = p.codes[crow * (p.D / 8) + c8];
  } else if constexpr (BITS == 8) {
    const uint2 v = reinterpret_cast<const uint2*>(p.codes + crow * (p.D / 4))[c8];
    w[0] = v.x; w[1] = v.y;
  } else {
    // one little-endian bit stream per row: the chunk's 8 BITS bits from its
    // (at most three) words, none past the row
    const uint32_t* row = p.codes + crow * (p.D * BITS / 32);
    const int pos = c8 * 8 * BITS, wi = pos >> 5, sh = pos & 31;
    const uint32_t w0 = row[wi];
    const uint32_t w1 = sh + 8 * BITS > 32 ? row[wi + 1] : 0u;
    const uint32_t w2 = sh + 8 * BITS > 64 ? row[wi + 2] : 0u;
    stream = ((uint64_t)__funnelshift_r(w1, w2, sh) << 32) | __funnelshift_r(w0, w1, sh);
  }
  uint32_t o[4];
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    double x[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      int code;
      if constexpr (BITS == 4) code = (int)((w[0] >> (4 * (e + k))) & 0xfu);
      else if constexpr (Q8) code = (int)(int8_t)((w[(e + k) >> 2] >> (8 * ((e + k) & 3))) & 0xffu);
      else if constexpr (BITS == 8) code = (int)((w[(e + k) >> 2] >> (8 * ((e + k) & 3))) & 0xffu);
      else code = (int)((stream >> (BITS * (e + k))) & ((1u << BITS) - 1u));
      x[k] = s * (double)code + b;
    }
    const uint32_t lo = __half_as_ushort(__double2half(x[0]));
    const uint32_t hi = __half_as_ushort(__double2half(x[1]));
    o[e >> 1] = lo | (hi << 16);
  }
  reinterpret_cast<uint4*>(p.out + (slab * p.L + j) * p.D)[c8] = make_uint4(o[0], o[1], o[2], o[3]);
}

cudaError_t launch_dequantize(const qkv_cache* c, int B, int Hkv, int D, int64_t L, void* out,
                              cudaStream_t stream) {
  DequantParams p;
  p.codes = c->codes;
  p.scales = c->scales;
  p.biases = c->biases;
  p.out = static_cast<uint16_t*>(out);
  p.Lcap = c->Lcap;
  p.L = L;
  p.D = D;
  int shift = 0;
  while ((8 << shift) < D) ++shift;
  p.cshift = shift;
  const int64_t slabs = (int64_t)B * Hkv;
  if (slabs > 65535 || (8 << shift) != D) return cudaErrorInvalidValue;
  const int64_t chunks = L << shift;
  dim3 grid((unsigned)((chunks + 255) / 256), (unsigned)slabs, 1);
  const int bits = c->fmt == QKV_Q8_0 ? 8 : c->bits, gs = c->fmt == QKV_Q8_0 ? 32 : c->group_size;
#define QKV_DQ(BITS, GS, Q8) qkv_dequantize_kernel<BITS, GS, Q8><<<grid, 256, 0, stream>>>(p)
  if (c->fmt == QKV_Q8_0) QKV_DQ(8, 32, true);
  else if (bits == 4 && gs == 32) QKV_DQ(4, 32, false);
  else if (bits == 4 && gs == 64) QKV_DQ(4, 64, false);
  else if (bits == 4 && gs == 128) QKV_DQ(4, 128, false);
  else if (bits == 8 && gs == 32) QKV_DQ(8, 32, false);
  else if (bits == 8 && gs == 64) QKV_DQ(8, 64, false);
  else if (bits == 8 && gs == 128) QKV_DQ(8, 128, false);
  else if (bits == 2 && gs == 32) QKV_DQ(2, 32, false);
  else if (bits == 2 && gs == 64) QKV_DQ(2, 64, false);
  else if (bits == 2 && gs == 128) QKV_DQ(2, 128, false);
  else if (bits == 3 && gs == 32) QKV_DQ(3, 32, false);
  else if (bits == 3 && gs == 64) QKV_DQ(3, 64, false);
  else if (bits == 3 && gs == 128) QKV_DQ(3, 128, false);
  else if (bits == 5 && gs == 32) QKV_DQ(5, 32, false);
  else if (bits == 5 && gs == 64) QKV_DQ(5, 64, false);
  else if (bits == 5 && gs == 128) QKV_DQ(5, 128, false);
  else if (bits == 6 && gs == 32) QKV_DQ(6, 32, false);
  else if (bits == 6 && gs == 64) QKV_DQ(6, 64, false);
  else if (bits == 6 && gs == 128) QKV_DQ(6, 128, false);
  else return cudaErrorInvalidValue;
#undef QKV_DQ
  return cudaGetLastError();
}

}  // namespace qkv
