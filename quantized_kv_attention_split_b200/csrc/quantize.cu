// quantize.cu -- quantize-and-append of new K/V tokens into the cache.
//
// Follows MLX compare "v0.19.3...quantized-kv-update" (quantized.h kv_update:
// each new row is quantized group by group and written at token `offset` of
// the cache; affine_quantize_impl: eps = 1e-7 on the scale) and, for Q8_0,
// llama.cpp PR #25556 (blocks of 32 int8 with one fp16 scale).  The
// quantizer body is not printed on the pages; the reading used (and matched
// bit for bit by the CPU oracle) is, per group, in fp32 IEEE arithmetic:
//   affine: s = max((max-min)/(2^bits-1), 1e-7); scale = fp16(s);
//           bias = fp16(min); code = clamp(rint((x - bias) / scale))
//   Q8_0:   scale = fp16(max|x| / 127); code = clamp(rint(x / scale), +-127)
//
// Design: one thread owns 8 consecutive elements (one 16-byte load), the
// gs/8 lanes of a group reduce min/max with shuffles, each thread packs its 8
// codes into one (4-bit) or two (8-bit) words and stores them; the first lane
// of a group stores the fp16 scale (and bias).  Grid: x = blocks of tokens
// (256 / (D/8) tokens per block), y = (batch, kv head) slab, z = K or V (one
// launch when both caches have the same format), so no thread divides.
#include <algorithm>

#include "qkv_common.cuh"
#include "qkv_internal.h"

namespace qkv {

struct QuantSide {
  const uint16_t* src;      // [B * Hkv * Lnew, D] fp16/bf16 bits
  uint32_t* codes;          // cache codes base
  uint16_t* scales;
  uint16_t* biases;
  int64_t Lcap;
};

struct QuantParams {
  QuantSide side[2];
  int D;
  int row_shift;            // log2(D / 8): threads per token row
  int Lnew;
  int64_t offset;
};

template <bool BF16>
__device__ __forceinline__ float in_to_float(uint16_t b) {
  if constexpr (BF16) return __uint_as_float((uint32_t)b << 16);
  else return __half2float(__ushort_as_half(b));
}

// rint(RN(d / s)) -- the code decision of the quantizer -- without a division
// in the common case.  With r = RN(1/s), q0 = RN(d * r) is within 2^-14 of
// RN(d / s) whenever |q0| < 2^9 (two roundings of relative error 2^-24 each),
// so both round to the same integer unless q0 lies within 2^-13 of a
// half-integer; that rare case, and any |q0| >= 2^9 or non-finite value, takes
// the correctly rounded division, so the result is always identical to it.
__device__ __forceinline__ int div_rint(float d, float s, float r) {
  const float q0 = __fmul_rn(d, r);
  const float n = rintf(q0);
  if (!(fabsf(q0) < 512.f) || fabsf(fabsf(__fsub_rn(q0, n)) - 0.5f) < 0x1p-13f)
    return __float2int_rn(__fdiv_rn(d, s));
  return (int)n;
}

template <int LANES>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
  for (int off = 1; off < LANES; off <<= 1) v = fmaxf(v, __shfl_xor_sync(~0u, v, off));
  return v;
}
template <int LANES>
__device__ __forceinline__ float group_min(float v) {
#pragma unroll
  for (int off = 1; off < LANES; off <<= 1) v = fminf(v, __shfl_xor_sync(~0u, v, off));
  return v;
}

template <int GS, int BITS, bool Q8, bool BF16>
__global__ void __launch_bounds__(256) qkv_quantize_kernel(const QuantParams p, int side0) {
  constexpr int LANES = GS / 8;
  const QuantSide& s = (side0 + (int)blockIdx.z) ? p.side[1] : p.side[0];
  const int per_row = p.D >> 3;
  const int tok = blockIdx.x * (256 >> p.row_shift) + (threadIdx.x >> p.row_shift);
  const int c8 = threadIdx.x & (per_row - 1);        // which 8-element slice of the row
  const bool active = tok < p.Lnew;                 // inactive lanes still join the shuffles
  const int64_t slab = blockIdx.y;                  // b * Hkv + kv head
  const int64_t srow = slab * p.Lnew + (active ? tok : 0);
  const int64_t crow = slab * s.Lcap + p.offset + tok;
  float x[8];
  if (active) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(s.src + srow * p.D + c8 * 8));
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = in_to_float<BF16>((uint16_t)(w[i] & 0xffff));
      x[2 * i + 1] = in_to_float<BF16>((uint16_t)(w[i] >> 16));
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = 0.f;
  }
  const int grp = (c8 * 8) / GS;
  const bool leader = ((c8 * 8) % GS) == 0;
  const int ng = p.D / GS;
  if constexpr (Q8) {
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(x[i]));
    a = group_max<LANES>(a);
    const float d = __fdiv_rn(a, 127.f);
    const __half d16 = __float2half_rn(d);
    const float df = __half2float(d16);
    const float rd = __frcp_rn(df);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int q = 0;
      if (df != 0.f) {
        q = div_rint(x[i], df, rd);
        q = q < -127 ? -127 : (q > 127 ? 127 : q);
      }
      w[i >> 2] |= (uint32_t)(q & 0xff) << ((i & 3) * 8);
    }
    if (active) {
      uint2* dst = reinterpret_cast<uint2*>(s.codes + crow * (p.D / 4) + c8 * 2);
      *dst = make_uint2(w[0], w[1]);
      if (leader) s.scales[crow * ng + grp] = __half_as_ushort(d16);
    }
  } else {
    float mn = x[0], mx = x[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) { mn = fminf(mn, x[i]); mx = fmaxf(mx, x[i]); }
    mn = group_min<LANES>(mn);
    mx = group_max<LANES>(mx);
    constexpr float levels = (float)((1 << BITS) - 1);
    float sc = __fdiv_rn(__fsub_rn(mx, mn), levels);
    sc = fmaxf(sc, 1e-7f);
    const __half s16 = __float2half_rn(sc);
    const __half b16 = __float2half_rn(mn);
    const float sf = __half2float(s16), bf = __half2float(b16);
    const float rs = __frcp_rn(sf);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int q = div_rint(__fsub_rn(x[i], bf), sf, rs);
      q = q < 0 ? 0 : (q > (1 << BITS) - 1 ? (1 << BITS) - 1 : q);
      if constexpr (BITS == 4) w[0] |= (uint32_t)q << (i * 4);
      else w[i >> 2] |= (uint32_t)q << ((i & 3) * 8);
    }
    if (active) {
      if constexpr (BITS == 4) {
        s.codes[crow * (p.D / 8) + c8] = w[0];
      } else {
        *reinterpret_cast<uint2*>(s.codes + crow * (p.D / 4) + c8 * 2) = make_uint2(w[0], w[1]);
      }
      if (leader) {
        s.scales[crow * ng + grp] = __half_as_ushort(s16);
        s.biases[crow * ng + grp] = __half_as_ushort(b16);
      }
    }
  }
}

namespace {

template <bool BF16>
cudaError_t launch_q(int fmt, int bits, int gs, const QuantParams& p, int side0, int nsides,
                     dim3 grid, cudaStream_t stream) {
  grid.z = nsides;
#define QKV_QLAUNCH(GS, BITS, Q8) \
  qkv_quantize_kernel<GS, BITS, Q8, BF16><<<grid, 256, 0, stream>>>(p, side0)
  if (fmt == QKV_Q8_0) QKV_QLAUNCH(32, 8, true);
  else if (bits == 4 && gs == 32) QKV_QLAUNCH(32, 4, false);
  else if (bits == 4 && gs == 64) QKV_QLAUNCH(64, 4, false);
  else if (bits == 4 && gs == 128) QKV_QLAUNCH(128, 4, false);
  else if (bits == 8 && gs == 32) QKV_QLAUNCH(32, 8, false);
  else if (bits == 8 && gs == 64) QKV_QLAUNCH(64, 8, false);
  else if (bits == 8 && gs == 128) QKV_QLAUNCH(128, 8, false);
  else return cudaErrorInvalidValue;
#undef QKV_QLAUNCH
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const void* new_k, const void* new_v, int in_dtype, int B, int Hkv,
                            int Lnew, int D, const qkv_cache* k, const qkv_cache* v,
                            int64_t offset, cudaStream_t stream) {
  QuantParams p;
  const qkv_cache* c[2] = {k, v};
  const void* src[2] = {new_k, new_v};
  int fmt[2], bits[2], gs[2];
  for (int i = 0; i < 2; ++i) {
    p.side[i].src = static_cast<const uint16_t*>(src[i]);
    p.side[i].codes = c[i]->codes;
    p.side[i].scales = c[i]->scales;
    p.side[i].biases = c[i]->biases;
    p.side[i].Lcap = c[i]->Lcap;
    fmt[i] = c[i]->fmt;
    bits[i] = c[i]->fmt == QKV_Q8_0 ? 8 : c[i]->bits;
    gs[i] = c[i]->fmt == QKV_Q8_0 ? 32 : c[i]->group_size;
  }
  int shift = 0;
  while ((8 << shift) < D) ++shift;                 // D / 8 = 2^shift threads per token
  p.D = D;
  p.row_shift = shift;
  p.Lnew = Lnew;
  p.offset = offset;
  const int64_t slabs = (int64_t)B * Hkv;
  if (slabs > 65535 || (8 << shift) != D) return cudaErrorInvalidValue;
  const int tpb = 256 >> shift;                     // tokens per block
  dim3 grid((unsigned)((Lnew + tpb - 1) / tpb), (unsigned)slabs, 1);
  const bool same = fmt[0] == fmt[1] && bits[0] == bits[1] && gs[0] == gs[1];
  const bool bf16 = in_dtype == QKV_BF16;
  for (int side0 = 0; side0 < 2; side0 += same ? 2 : 1) {
    const int n = same ? 2 : 1;
    cudaError_t e = bf16 ? launch_q<true>(fmt[side0], bits[side0], gs[side0], p, side0, n, grid, stream)
                         : launch_q<false>(fmt[side0], bits[side0], gs[side0], p, side0, n, grid, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace qkv
