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
// Design: one thread owns 16 consecutive elements (two 16-byte loads), the
// gs/16 lanes of a group reduce min/max with shuffles, each thread packs its
// 16 codes into two (4-bit) or four (8-bit) words and stores them; the first
// lane of a group stores the fp16 scale (and bias).  Grid: x = blocks of
// tokens (256 / (D/16) tokens per block), y = (batch, kv head) slab, z = K or
// V (one launch when both caches have the same format), so no thread divides.
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
// half-integer.  `exact` is set for that rare case and for any |q0| >= 2^9 or
// non-finite value; the caller then redoes the row with the correctly rounded
// division, so the result is always identical to it.
__device__ __forceinline__ int fast_rint_div(float d, float r, bool& exact) {
  const float q0 = __fmul_rn(d, r);
  const float n = rintf(q0);
  exact |= !(fabsf(q0) < 512.f) | (fabsf(fabsf(__fsub_rn(q0, n)) - 0.5f) < 0x1p-13f);
  return (int)fminf(fmaxf(n, -512.f), 512.f);
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

constexpr int kQEpt = 16;   // elements per thread (two 16-byte loads)

template <int GS, int BITS, bool Q8, bool BF16>
__global__ void __launch_bounds__(256) qkv_quantize_kernel(const QuantParams p, int side0) {
  constexpr int LANES = GS / kQEpt;                 // threads per group
  const QuantSide& s = (side0 + (int)blockIdx.z) ? p.side[1] : p.side[0];
  const int per_row = p.D / kQEpt;
  const int tok = blockIdx.x * (256 >> p.row_shift) + (threadIdx.x >> p.row_shift);
  const int c16 = threadIdx.x & (per_row - 1);      // which 16-element slice of the row
  const bool active = tok < p.Lnew;                 // inactive lanes still join the shuffles
  const int64_t slab = blockIdx.y;                  // b * Hkv + kv head
  const int64_t srow = slab * p.Lnew + (active ? tok : 0);
  const int64_t crow = slab * s.Lcap + p.offset + tok;
  float x[kQEpt];
  if (active) {
    const uint4* src = reinterpret_cast<const uint4*>(s.src + srow * p.D + c16 * kQEpt);
    const uint4 r0 = __ldg(src), r1 = __ldg(src + 1);
    const uint32_t w[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      x[2 * i] = in_to_float<BF16>((uint16_t)(w[i] & 0xffff));
      x[2 * i + 1] = in_to_float<BF16>((uint16_t)(w[i] >> 16));
    }
  } else {
#pragma unroll
    for (int i = 0; i < kQEpt; ++i) x[i] = 0.f;
  }
  const int grp = (c16 * kQEpt) / GS;
  const bool leader = ((c16 * kQEpt) % GS) == 0;
  const int ng = p.D / GS;
  int q[kQEpt];
  uint16_t sbits, bbits = 0;
  if constexpr (Q8) {
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < kQEpt; ++i) a = fmaxf(a, fabsf(x[i]));
    a = group_max<LANES>(a);
    const float d = __fdiv_rn(a, 127.f);
    const __half d16 = __float2half_rn(d);
    const float df = __half2float(d16);
    sbits = __half_as_ushort(d16);
    const float rd = __frcp_rn(df);
    bool exact = false;
#pragma unroll
    for (int i = 0; i < kQEpt; ++i) q[i] = fast_rint_div(x[i], rd, exact);
    if (exact) {
#pragma unroll
      for (int i = 0; i < kQEpt; ++i) q[i] = __float2int_rn(__fdiv_rn(x[i], df));
    }
#pragma unroll
    for (int i = 0; i < kQEpt; ++i) q[i] = df == 0.f ? 0 : (q[i] < -127 ? -127 : (q[i] > 127 ? 127 : q[i]));
  } else {
    float mn = x[0], mx = x[0];
#pragma unroll
    for (int i = 1; i < kQEpt; ++i) { mn = fminf(mn, x[i]); mx = fmaxf(mx, x[i]); }
    mn = group_min<LANES>(mn);
    mx = group_max<LANES>(mx);
    constexpr float levels = (float)((1 << BITS) - 1);
    float sc = __fdiv_rn(__fsub_rn(mx, mn), levels);
    sc = fmaxf(sc, 1e-7f);
    const __half s16 = __float2half_rn(sc);
    const __half b16 = __float2half_rn(mn);
    const float sf = __half2float(s16), bf = __half2float(b16);
    sbits = __half_as_ushort(s16);
    bbits = __half_as_ushort(b16);
    const float rs = __frcp_rn(sf);
    bool exact = false;
#pragma unroll
    for (int i = 0; i < kQEpt; ++i) q[i] = fast_rint_div(__fsub_rn(x[i], bf), rs, exact);
    if (exact) {
#pragma unroll
      for (int i = 0; i < kQEpt; ++i) q[i] = __float2int_rn(__fdiv_rn(__fsub_rn(x[i], bf), sf));
    }
#pragma unroll
    for (int i = 0; i < kQEpt; ++i) q[i] = q[i] < 0 ? 0 : (q[i] > (1 << BITS) - 1 ? (1 << BITS) - 1 : q[i]);
  }
  if (active) {
    if constexpr (BITS == 4) {
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < kQEpt; ++i) w[i >> 3] |= (uint32_t)q[i] << ((i & 7) * 4);
      *reinterpret_cast<uint2*>(s.codes + crow * (p.D / 8) + c16 * 2) = make_uint2(w[0], w[1]);
    } else {
      uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int i = 0; i < kQEpt; ++i) w[i >> 2] |= (uint32_t)(q[i] & 0xff) << ((i & 3) * 8);
      *reinterpret_cast<uint4*>(s.codes + crow * (p.D / 4) + c16 * 4) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (leader) {
      s.scales[crow * ng + grp] = sbits;
      if constexpr (!Q8) s.biases[crow * ng + grp] = bbits;
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
  while ((kQEpt << shift) < D) ++shift;             // D / 16 = 2^shift threads per token
  p.D = D;
  p.row_shift = shift;
  p.Lnew = Lnew;
  p.offset = offset;
  const int64_t slabs = (int64_t)B * Hkv;
  if (slabs > 65535 || (kQEpt << shift) != D) return cudaErrorInvalidValue;
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
