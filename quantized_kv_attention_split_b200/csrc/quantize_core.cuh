// quantize_core.cuh -- the arithmetic of the KV-update quantizer, shared by
// the quantize-and-append kernel and the fused update + decode kernel, so both
// write the same bytes.
//
// Follows MLX compare "v0.19.3...quantized-kv-update" (quantized.h kv_update;
// affine_quantize_impl: eps = 1e-7 on the scale) and, for Q8_0, llama.cpp PR
// #25556 (blocks of 32 int8 with one fp16 scale).  The quantizer body is not
// printed on the pages; the reading used (and matched bit for bit by the CPU
// oracle) is, per group, in fp32 IEEE arithmetic:
//   affine: s = max((max-min)/(2^bits-1), 1e-7); scale = fp16(s);
//           bias = fp16(min); code = clamp(rint((x - bias) / scale))
//   Q8_0:   scale = fp16(max|x| / 127); code = clamp(rint(x / scale), +-127)
#pragma once

#include "qkv_common.cuh"

namespace qkv {

constexpr int kQEpt = 32;   // elements per thread (four 16-byte loads)
constexpr int kQWords = kQEpt / 2;

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


// The quantizer of one thread's 32 consecutive elements of a row (16 words
// of packed 16-bit inputs, zeros for a thread without a row): the GS/32
// threads of a group (adjacent lanes; every lane of the warp takes part in
// the shuffles) agree on the group's fp16 scale (and bias), and the thread's
// codes come out packed, low bits first, in kQEpt * BITS / 32 = BITS words.
// For widths that do not divide 32 (3, 5, 6 bits) the row is one
// little-endian bit stream, element i at bits [i BITS, (i + 1) BITS), so a
// code may straddle two words; 32 codes fill exactly BITS words, so every
// code stays inside its thread's words.
template <int GS, int BITS, bool Q8, bool BF16>
__device__ __forceinline__ void quantize_slice(const uint32_t (&w)[kQWords], uint32_t* o,
                                               uint16_t& sbits, uint16_t& bbits) {
  constexpr int LANES = GS / kQEpt;                 // threads per group
  bbits = 0;
  // per group: the value subtracted (bias; 0 for Q8_0), the fp16 scale as
  // float and its reciprocal; `inside` when every code of the group is known
  // to fall inside the code range before clamping (then the clamp is skipped)
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
  constexpr bool STREAM = !Q8 && (32 % BITS) != 0;  // codes straddle words
  auto emit = [&](int i, int c, bool clamp) {       // code of element i
    if (clamp) c = min(max(c, QLO), QHI);
    if constexpr (Q8) {
      // signed codes: their low bytes, four per word
      c = sf == 0.f ? 0 : c;
      const uint32_t sel = (i % 4) == 0 ? 0x3210u : (i % 4) == 1 ? 0x3240u : (i % 4) == 2 ? 0x3410u : 0x4210u;
      o[i / 4] = (i % 4) == 0 ? (uint32_t)c & 0xffu : __byte_perm(o[i / 4], (uint32_t)c, sel);
    } else if constexpr (STREAM) {
      // codes in [0, levels] at bit i * BITS of the stream (words zeroed first)
      const int pos = i * BITS, wd = pos / 32, sh = pos % 32;
      o[wd] |= (uint32_t)c << sh;
      if (sh + BITS > 32) o[wd + 1] |= (uint32_t)c >> (32 - sh);
    } else {
      // codes in [0, levels]: place them by multiplication, no masking
      const uint32_t u = (uint32_t)c * (1u << ((i % CPW) * BITS));
      o[i / CPW] = (i % CPW) == 0 ? u : o[i / CPW] + u;
    }
  };
  auto clear = [&]() {
    if constexpr (STREAM) {
#pragma unroll
      for (int k = 0; k < BITS; ++k) o[k] = 0u;
    }
  };
  clear();
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
    clear();
#pragma unroll
    for (int i = 0; i < kQWords; ++i) {
      const float2 f = to_f2<BF16>(w[i]);
      emit(2 * i, __float2int_rn(__fdiv_rn(__fsub_rn(f.x, bf), sf)), true);
      emit(2 * i + 1, __float2int_rn(__fdiv_rn(__fsub_rn(f.y, bf), sf)), true);
    }
  }
}

}  // namespace qkv
