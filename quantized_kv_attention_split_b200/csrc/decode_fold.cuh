// decode_fold.cuh -- the log-sum-exp fold of a split unit's per-CTA partials
// (m_i, l_i, o_i) into its output,
//   M = max_i m_i,  l = sum_i l_i 2^(m_i - M),  out = sum_i o_i 2^(m_i - M) / l
// (base-2 logits), the same rule the online softmax applies within a CTA; a
// head's attention-sink logit s, when given, joins as l += 2^(s - M).
#pragma once

#include "qkv_common.cuh"
#include "qkv_internal.h"

namespace qkv {

// ---------------------------------------------------------------------------
// Where the partials of unit u are: n parts, part 0 in slot slot0, part pp > 0
// in slot 2 * (cfirst + pp) (a CTA holds two slots: its first segment's and
// its last's).
struct UnitParts {
  int64_t cfirst, slot0;
  int n;
};
__device__ __forceinline__ UnitParts unit_parts(const DecodeParams& p, int64_t u, int64_t nC) {
  const int64_t S = p.stages_per_unit, T = p.total_stages;
  UnitParts r;
  if (p.pieces > 0) {
    // every CTA covered one piece of one unit: CTAs u*pieces ... in order
    r.cfirst = u * p.pieces;
    r.n = p.pieces;
    r.slot0 = 2 * r.cfirst;
  } else {
    // CTA c covered blocks [c*T/nC, (c+1)*T/nC): the unit's first and last CTA
    r.cfirst = udiv64((u * S + 1) * nC - 1, T);
    const int64_t clast = udiv64((u + 1) * S * nC - 1, T);
    r.n = (int)(clast - r.cfirst + 1);
    // the first CTA used its second slot if its range began in an earlier unit
    r.slot0 = 2 * r.cfirst + (udiv64(udiv64(r.cfirst * T, nC), S) == u ? 0 : 1);
  }
  return r;
}

constexpr int kMergeBatch = 8;   // parts whose loads a thread has in flight

// Log-sum-exp fold of 4 consecutive outputs (row R, dims 4 e4 .. 4 e4 + 3) of
// a split unit over its parts, shared by `lanes` adjacent threads (a power of
// two; lane `sub` takes every lanes-th part), combined by shuffles; lane 0
// writes the normalized output (with the head's sink logit, if any, in the
// denominator).  Every thread of the warp calls it (inactive ones with
// active = false), since the combine is a warp shuffle.
template <int D, int HPC>
__device__ __forceinline__ void merge_item(const DecodeParams& p, const UnitParts& up, int64_t uh,
                                           int head, int R, int e4, int sub, int lanes,
                                           bool active) {
  float M = -INFINITY, Ls = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j0 = 0; active && sub + lanes * j0 < up.n; j0 += kMergeBatch) {
    float4 o[kMergeBatch];
    float2 v[kMergeBatch];
#pragma unroll
    for (int k = 0; k < kMergeBatch; ++k) {
      const int pp = sub + lanes * (j0 + k);
      if (pp < up.n) {
        const int64_t sx = pp == 0 ? up.slot0 : 2 * (up.cfirst + pp);
        o[k] = __ldcg(reinterpret_cast<const float4*>(p.part_o + (sx * HPC + R) * D) + e4);
        v[k] = __ldcg(reinterpret_cast<const float2*>(p.part_ml + (sx * HPC + R) * 2));
      } else {
        o[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        v[k] = make_float2(-INFINITY, 0.f);
      }
    }
    float Mb = M;
#pragma unroll
    for (int k = 0; k < kMergeBatch; ++k) Mb = fmaxf(Mb, v[k].x);
    if (Mb != M) {
      const float f = M == -INFINITY ? 0.f : ex2(M - Mb);
      Ls *= f; acc.x *= f; acc.y *= f; acc.z *= f; acc.w *= f;
      M = Mb;
    }
#pragma unroll
    for (int k = 0; k < kMergeBatch; ++k) {
      const float w = v[k].x == -INFINITY ? 0.f : ex2(v[k].x - M);
      Ls = fmaf(w, v[k].y, Ls);
      acc.x = fmaf(w, o[k].x, acc.x);
      acc.y = fmaf(w, o[k].y, acc.y);
      acc.z = fmaf(w, o[k].z, acc.z);
      acc.w = fmaf(w, o[k].w, acc.w);
    }
  }
  for (int off = 1; off < lanes; off <<= 1) {
    const float M2 = __shfl_xor_sync(~0u, M, off), L2 = __shfl_xor_sync(~0u, Ls, off);
    const float x2 = __shfl_xor_sync(~0u, acc.x, off), y2 = __shfl_xor_sync(~0u, acc.y, off);
    const float z2 = __shfl_xor_sync(~0u, acc.z, off), w2 = __shfl_xor_sync(~0u, acc.w, off);
    const float Mn = fmaxf(M, M2);
    const float f1 = M == -INFINITY ? 0.f : ex2(M - Mn), f2 = M2 == -INFINITY ? 0.f : ex2(M2 - Mn);
    Ls = Ls * f1 + L2 * f2;
    acc.x = acc.x * f1 + x2 * f2; acc.y = acc.y * f1 + y2 * f2;
    acc.z = acc.z * f1 + z2 * f2; acc.w = acc.w * f1 + w2 * f2;
    M = Mn;
  }
  if (!active || sub != 0) return;
  float fo = 1.f;
  if (p.sinks != nullptr && Ls > 0.f) {
    // the head's sink logit joins the denominator: (M, l) -> (max(M, s), l 2^(M - M') + 2^(s - M'))
    const int hkv = (int)(uh - udiv64(uh, p.Hkv) * p.Hkv);
    const float s2 = kLog2e * p.sinks[hkv * p.Gq + head / p.Lq];
    const float Mn = fmaxf(M, s2);
    fo = ex2(M - Mn);
    Ls = Ls * fo + ex2(s2 - Mn);
  }
  const float inv = Ls > 0.f ? fo / Ls : 0.f;
  const int64_t oi = (uh * p.G + head) * D + e4 * 4;
  store4_from_float(p.out, p.out_dtype, oi,
                    make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv));
}

}  // namespace qkv
