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
// of a group stores the fp16 scale (and bias).  K and V are handled by the two
// halves of the grid's y dimension.
#include <algorithm>

#include "qkv_common.cuh"
#include "qkv_internal.h"

namespace qkv {

struct QuantSide {
  const uint16_t* src;      // [rows, D] fp16/bf16 bits
  uint32_t* codes;          // cache codes base
  uint16_t* scales;
  uint16_t* biases;
  int fmt, bits, gs;
};

struct QuantParams {
  QuantSide side[2];
  int in_dtype;
  int D;
  int64_t rows;             // B * Hkv * Lnew
  int Lnew;
  int64_t Lcap, offset;
};

__device__ __forceinline__ float load_in(const uint16_t* p, int dtype, int64_t i) {
  return dtype == QKV_F16 ? __half2float(__ushort_as_half(p[i]))
                          : __bfloat162float(__ushort_as_bfloat16(p[i]));
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

template <int GS, int BITS, bool Q8>
__device__ __forceinline__ void quantize_item(const QuantParams& p, const QuantSide& s,
                                              int64_t item, bool active) {
  constexpr int LANES = GS / 8;
  const int per_row = p.D / 8;
  const int64_t r = item / per_row;
  const int c8 = (int)(item - r * per_row);        // which 8-element slice of the row
  float x[8];
  if (active) {
    const uint4 raw = *reinterpret_cast<const uint4*>(s.src + r * p.D + c8 * 8);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint16_t lo = (uint16_t)(w[i] & 0xffff), hi = (uint16_t)(w[i] >> 16);
      x[2 * i] = load_in(&lo, p.in_dtype, 0);
      x[2 * i + 1] = load_in(&hi, p.in_dtype, 0);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = 0.f;
  }
  const int64_t crow = (r / p.Lnew) * p.Lcap + p.offset + (r % p.Lnew);
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
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int q = 0;
      if (df != 0.f) {
        q = __float2int_rn(__fdiv_rn(x[i], df));
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
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int q = __float2int_rn(__fdiv_rn(__fsub_rn(x[i], bf), sf));
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

template <int GS, int BITS, bool Q8>
__global__ void __launch_bounds__(256) qkv_quantize_kernel(const QuantParams p, int side_idx) {
  const QuantSide& s = p.side[side_idx];
  const int64_t items = p.rows * (p.D / 8);
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  // the loop bound is rounded up to whole warps so every lane takes part in
  // the group shuffles; lanes past the end are inactive
  const int64_t items_w = (items + 31) / 32 * 32;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items_w; it += stride) {
    quantize_item<GS, BITS, Q8>(p, s, it < items ? it : 0, it < items);
  }
}

cudaError_t launch_quantize_side(const QuantParams& p, int side_idx, cudaStream_t stream) {
  const QuantSide& s = p.side[side_idx];
  const int64_t items = p.rows * (p.D / 8);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (items + 255) / 256;
  const int grid = (int)std::min<int64_t>(want, (int64_t)sms * 16);
  if (grid <= 0) return cudaSuccess;
#define QKV_QLAUNCH(GS, BITS, Q8) \
  qkv_quantize_kernel<GS, BITS, Q8><<<grid, 256, 0, stream>>>(p, side_idx)
  if (s.fmt == QKV_Q8_0) QKV_QLAUNCH(32, 8, true);
  else if (s.bits == 4 && s.gs == 32) QKV_QLAUNCH(32, 4, false);
  else if (s.bits == 4 && s.gs == 64) QKV_QLAUNCH(64, 4, false);
  else if (s.bits == 4 && s.gs == 128) QKV_QLAUNCH(128, 4, false);
  else if (s.bits == 8 && s.gs == 32) QKV_QLAUNCH(32, 8, false);
  else if (s.bits == 8 && s.gs == 64) QKV_QLAUNCH(64, 8, false);
  else if (s.bits == 8 && s.gs == 128) QKV_QLAUNCH(128, 8, false);
  else return cudaErrorInvalidValue;
#undef QKV_QLAUNCH
  return cudaGetLastError();
}

cudaError_t launch_quantize(const void* new_k, const void* new_v, int in_dtype, int B, int Hkv,
                            int Lnew, int D, const qkv_cache* k, const qkv_cache* v,
                            int64_t offset, cudaStream_t stream) {
  QuantParams p;
  const qkv_cache* c[2] = {k, v};
  const void* src[2] = {new_k, new_v};
  for (int i = 0; i < 2; ++i) {
    p.side[i].src = static_cast<const uint16_t*>(src[i]);
    p.side[i].codes = c[i]->codes;
    p.side[i].scales = c[i]->scales;
    p.side[i].biases = c[i]->biases;
    p.side[i].fmt = c[i]->fmt;
    p.side[i].bits = c[i]->fmt == QKV_Q8_0 ? 8 : c[i]->bits;
    p.side[i].gs = c[i]->fmt == QKV_Q8_0 ? 32 : c[i]->group_size;
  }
  p.in_dtype = in_dtype;
  p.D = D;
  p.rows = (int64_t)B * Hkv * Lnew;
  p.Lnew = Lnew;
  p.Lcap = k->Lcap;
  p.offset = offset;
  cudaError_t e = launch_quantize_side(p, 0, stream);
  if (e != cudaSuccess) return e;
  p.Lcap = v->Lcap;
  return launch_quantize_side(p, 1, stream);
}

}  // namespace qkv
