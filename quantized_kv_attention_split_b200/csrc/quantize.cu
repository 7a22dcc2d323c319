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
// Design: one thread owns 16 consecutive elements (two 16-byte loads) and
// takes their min / max (or largest magnitude) on the packed 16-bit pairs;
// the gs/16 lanes of a group reduce with shuffles, each thread packs its
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
  int row_shift;            // log2(D / 32): threads per token row
  int Lnew;
  int64_t offset;
};

// Packed pairs of 16-bit inputs (fp16 or bf16): elementwise min / max
// (exact: a selection), magnitudes, and the conversion of a pair to fp32.
template <bool BF16>
__device__ __forceinline__ uint32_t pmin(uint32_t a, uint32_t b) {
  uint32_t r;
  if constexpr (BF16) {
    const __nv_bfloat162 v = __hmin2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                                     *reinterpret_cast<const __nv_bfloat162*>(&b));
    r = *reinterpret_cast<const uint32_t*>(&v);
  } else {
    const __half2 v = __hmin2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
    r = *reinterpret_cast<const uint32_t*>(&v);
  }
  return r;
}
template <bool BF16>
__device__ __forceinline__ uint32_t pmax(uint32_t a, uint32_t b) {
  uint32_t r;
  if constexpr (BF16) {
    const __nv_bfloat162 v = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                                     *reinterpret_cast<const __nv_bfloat162*>(&b));
    r = *reinterpret_cast<const uint32_t*>(&v);
  } else {
    const __half2 v = __hmax2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
    r = *reinterpret_cast<const uint32_t*>(&v);
  }
  return r;
}
template <bool BF16>
__device__ __forceinline__ float2 to_f2(uint32_t w) {
  if constexpr (BF16) return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  else return __half22float2(*reinterpret_cast<const __half2*>(&w));
}

// rint(RN(d / s)) -- the code decision of the quantizer -- without a division
// or a conversion instruction in the common case.  With r = RN(1/s),
// q0 = RN(d * r) differs from RN(d / s) by less than 2^-14 whenever
// |q0| < 2^9 (two roundings of relative error 2^-24 each), so both round to
// the same integer unless q0 lies within 2^-13 of a half-integer.  The integer
// is taken by adding 1.5 * 2^23 (the sum's unit in the last place is 1, so the
// addition rounds q0 to the nearest integer, ties to even, for |q0| < 2^22)
// and reading the sum's low bits.  `exact` is set for a near-tie or a
// non-finite q0; the caller then redoes the row with the correctly rounded
// division, so the result is always identical to it.  For |q0| >= 2^9 the
// result may be off, but then both it and the true code lie beyond the code
// range on the same side (the read-back integer is monotone in q0 and keeps
// its sign), so the caller's clamp gives the same code.
constexpr float kRoundMagic = 12582912.f;            // 1.5 * 2^23
constexpr int kRoundMagicBits = 0x4B400000;
__device__ __forceinline__ int fast_rint_div(float d, float r, bool& exact) {
  const float q0 = __fmul_rn(d, r);
  const float y = __fadd_rn(q0, kRoundMagic);
  exact |= !(fabsf(__fsub_rn(q0, __fsub_rn(y, kRoundMagic))) <= 0.5f - 0x1p-13f);
  return __float_as_int(y) - kRoundMagicBits;
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

constexpr int kQEpt = 32;   // elements per thread (four 16-byte loads)
constexpr int kQWords = kQEpt / 2;

template <int GS, int BITS, bool Q8, bool BF16>
__global__ void __launch_bounds__(256, 6) qkv_quantize_kernel(const __grid_constant__ QuantParams p, int side0) {
  constexpr int LANES = GS / kQEpt;                 // threads per group
  const QuantSide& s = (side0 + (int)blockIdx.z) ? p.side[1] : p.side[0];
  const int per_row = p.D / kQEpt;
  const int tok = blockIdx.x * (256 >> p.row_shift) + (threadIdx.x >> p.row_shift);
  const int cs = threadIdx.x & (per_row - 1);       // which 32-element slice of the row
  const bool active = tok < p.Lnew;                 // inactive lanes still join the shuffles
  const int64_t slab = blockIdx.y;                  // b * Hkv + kv head
  const int64_t srow = slab * p.Lnew + (active ? tok : 0);
  const int64_t crow = slab * s.Lcap + p.offset + tok;
  uint32_t w[kQWords];                              // 32 raw 16-bit inputs, two per word
  if (active) {
    const uint4* src = reinterpret_cast<const uint4*>(s.src + srow * p.D + cs * kQEpt);
#pragma unroll
    for (int k = 0; k < kQWords / 4; ++k) {
      const uint4 r = __ldg(src + k);
      w[4 * k] = r.x; w[4 * k + 1] = r.y; w[4 * k + 2] = r.z; w[4 * k + 3] = r.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < kQWords; ++i) w[i] = 0u;
  }
  const int grp = (cs * kQEpt) / GS;
  const bool leader = ((cs * kQEpt) % GS) == 0;
  const int ng = p.D / GS;
  // per group: the value subtracted (bias; 0 for Q8_0), the fp16 scale as
  // float and its reciprocal; `inside` when every code of the group is known
  // to fall inside the code range before clamping (then the clamp is skipped)
  uint16_t sbits, bbits = 0;
  float bf = 0.f, sf;
  bool inside;
  constexpr int QLO = Q8 ? -127 : 0, QHI = Q8 ? 127 : (1 << BITS) - 1;
  if constexpr (Q8) {
    uint32_t a2 = w[0] & 0x7fff7fffu;
#pragma unroll
    for (int i = 1; i < kQWords; ++i) a2 = pmax<BF16>(a2, w[i] & 0x7fff7fffu);
    const float2 af = to_f2<BF16>(a2);
    const float a = group_max<LANES>(fmaxf(af.x, af.y));
    const __half d16 = __float2half_rn(__fdiv_rn(a, 127.f));
    sf = __half2float(d16);
    sbits = __half_as_ushort(d16);
    // |x| / d <= a / d; below 127.25 every code lies in [-127, 127]
    inside = sf > 0.f && a < 127.25f * sf;
  } else {
    uint32_t mn2 = w[0], mx2 = w[0];
#pragma unroll
    for (int i = 1; i < kQWords; ++i) { mn2 = pmin<BF16>(mn2, w[i]); mx2 = pmax<BF16>(mx2, w[i]); }
    const float2 fmn = to_f2<BF16>(mn2), fmx = to_f2<BF16>(mx2);
    const float mn = group_min<LANES>(fminf(fmn.x, fmn.y));
    const float mx = group_max<LANES>(fmaxf(fmx.x, fmx.y));
    constexpr float levels = (float)QHI;
    const float sc = fmaxf(__fdiv_rn(__fsub_rn(mx, mn), levels), 1e-7f);
    const __half s16 = __float2half_rn(sc);
    const __half b16 = __float2half_rn(mn);
    sf = __half2float(s16);
    bf = __half2float(b16);
    sbits = __half_as_ushort(s16);
    bbits = __half_as_ushort(b16);
    // (x - bias) / scale lies within [(mn - bias) / scale, (mx - bias) / scale];
    // with margins of a quarter step both ends round into [0, levels]
    inside = __fsub_rn(mn, bf) > -0.25f * sf && __fsub_rn(mx, bf) < (levels + 0.25f) * sf;
  }
  const float rs = __frcp_rn(sf);
  // Codes two at a time straight from the packed inputs, packed as they come;
  // a second pass with the correctly rounded division in the rare case that
  // flags it.  Q8_0 with a zero scale gives zero codes.
  constexpr int CPW = 32 / BITS;                    // codes per output word
  uint32_t o[kQEpt / CPW];
  auto emit = [&](int i, int c, bool clamp) {       // code of element i
    if (clamp) c = min(max(c, QLO), QHI);
    if constexpr (Q8) {
      // signed codes: their low bytes, four per word
      c = sf == 0.f ? 0 : c;
      const uint32_t sel = (i % 4) == 0 ? 0x3210u : (i % 4) == 1 ? 0x3240u : (i % 4) == 2 ? 0x3410u : 0x4210u;
      o[i / 4] = (i % 4) == 0 ? (uint32_t)c & 0xffu : __byte_perm(o[i / 4], (uint32_t)c, sel);
    } else {
      // codes in [0, levels]: place them by multiplication, no masking
      const uint32_t u = (uint32_t)c * (1u << ((i % CPW) * BITS));
      o[i / CPW] = (i % CPW) == 0 ? u : o[i / CPW] + u;
    }
  };
  bool exact = false;
  if (__all_sync(~0u, inside)) {
#pragma unroll
    for (int i = 0; i < kQWords; ++i) {
      const float2 f = to_f2<BF16>(w[i]);
      emit(2 * i, fast_rint_div(__fsub_rn(f.x, bf), rs, exact), false);
      emit(2 * i + 1, fast_rint_div(__fsub_rn(f.y, bf), rs, exact), false);
    }
  } else {
#pragma unroll
    for (int i = 0; i < kQWords; ++i) {
      const float2 f = to_f2<BF16>(w[i]);
      emit(2 * i, fast_rint_div(__fsub_rn(f.x, bf), rs, exact), true);
      emit(2 * i + 1, fast_rint_div(__fsub_rn(f.y, bf), rs, exact), true);
    }
  }
  if (exact) {
#pragma unroll
    for (int i = 0; i < kQWords; ++i) {
      const float2 f = to_f2<BF16>(w[i]);
      emit(2 * i, __float2int_rn(__fdiv_rn(__fsub_rn(f.x, bf), sf)), true);
      emit(2 * i + 1, __float2int_rn(__fdiv_rn(__fsub_rn(f.y, bf), sf)), true);
    }
  }
  if (active) {
    uint4* dst = reinterpret_cast<uint4*>(s.codes + crow * (p.D * BITS / 32) + cs * (kQEpt * BITS / 32));
#pragma unroll
    for (int k = 0; k < kQEpt * BITS / 128; ++k)
      dst[k] = make_uint4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
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
  while ((kQEpt << shift) < D) ++shift;             // D / 32 = 2^shift threads per token
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
