// decode_kernel.cuh -- split-K flash-decode over a group-quantized KV cache.
//
// What it computes (MLX compare "v0.19.3...quantized-kv-update", mlx/fast.cpp
// quantized_scaled_dot_product_attention and sdpa_vector.h quant_sdpa_vector):
//   out[b,h] = softmax_j(q[b,h]*scale . Khat[b,h/G,j] + mask) . Vhat[b,h/G,:]
// with Khat/Vhat = scale*code + bias per group of GS along D (affine) or
// scale*code (Q8_0, llama.cpp PR #25556), for one query per head.
//
// How (B200 design; the Metal kernel on the pages walks every key of one head
// with one threadgroup and has no split, no GQA sharing and no tensor cores):
//  * Work: units (batch, kv-head, chunk-group of <=32 query heads) x stages of
//    TK keys, flattened and cut evenly over the grid, so every SM gets the
//    same number of stages.  A CTA touches at most two units partially; a
//    partial result (running max m, sum l, unnormalized o) goes to workspace
//    and the last CTA of a unit to finish (atomic ticket) merges them
//    (log-sum-exp rescaling) -- one launch, no waiting.
//  * Staging: all 256 threads stream codes and scales with 16-byte cp.async
//    (zero-filled past L) into an NSTAGE-deep shared-memory ring.  Code tiles
//    are XOR-swizzled per 128-byte line so both fragment read patterns below
//    are bank-conflict-free.
//  * Scores: one m16n8k16 tensor op per 16 keys x 8 query heads x 16 dims.
//    Codes enter the tensor core EXACTLY as fp16 subnormals (a mask of the
//    packed word leaves code*2^-24 or code*2^-20); the query is prescaled by a
//    power of two (and by 1/16 for the 2^-20 positions).  The per-group key
//    scale and the bias term (bias * sum of q over the group, the identity the
//    Metal kernel uses with its query_sum) are applied in fp32 afterwards.
//    Q8_0 codes are offset by 128 (xor 0x80) and corrected the same way.
//  * Online softmax in base 2 with warp shuffles over the 16 keys.
//  * Values: O^T[e,h] += V^T[e,j] (P[j,h]*s_v[j]*2^tau): V codes are the A
//    operand (pairs of keys per register, built with byte permutes), the
//    probabilities times the per-key value scale are the B operand, moved
//    from the score fragment layout with movmatrix.trans.  tau normalizes each
//    16-key block so the fp16 operand never over- or underflows; the block
//    result is folded into fp32 accumulators.  The value bias term
//    sum_j P[j,h]*b_v[j] is accumulated in fp32.  With fp32 output the B
//    operand is split into fp16 hi + lo parts (two tensor ops).
#pragma once

#include "qkv_common.cuh"
#include "qkv_internal.h"

namespace qkv {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecStageBudget = 96 * 1024;

// XOR coefficients (3 bits each, for line bits 0..3) of the 16-byte-unit
// swizzle inside each 128-byte line of a staged code tile, found by exhaustive
// search so that the K-fragment and V-fragment read patterns are free of bank
// conflicts for every supported (D, bits, group size).
__host__ __device__ constexpr uint32_t swz_pack(int c0, int c1, int c2, int c3) {
  return (uint32_t)(c0 | (c1 << 3) | (c2 << 6) | (c3 << 9));
}
__host__ __device__ constexpr uint32_t swizzle_coeffs(int D, int bits, int gs) {
  return D == 64 ? (bits == 4 ? (gs == 32 ? swz_pack(1, 0, 0, 0) : swz_pack(2, 0, 0, 0))
                              : swz_pack(2, 4, 0, 0))
       : D == 128 ? (bits == 4 ? (gs == 32 ? swz_pack(1, 2, 0, 0) : swz_pack(2, 4, 0, 0))
                               : (gs == 32 ? swz_pack(2, 4, 2, 0)
                                  : gs == 64 ? swz_pack(4, 2, 4, 0) : swz_pack(1, 2, 4, 0)))
       : (bits == 4 ? (gs == 32 ? swz_pack(1, 2, 4, 0)
                       : gs == 64 ? swz_pack(2, 4, 2, 0) : swz_pack(4, 2, 4, 0))
                    : (gs == 32 ? swz_pack(0, 2, 4, 2)
                       : gs == 64 ? swz_pack(0, 4, 2, 4) : swz_pack(0, 1, 2, 4)));
}

template <uint32_t SWZ>
__device__ __forceinline__ int swz_offset(int lin) {
  const int line = lin >> 7;
  int f = 0;
  if (line & 1) f ^= (SWZ & 7);
  if (line & 2) f ^= ((SWZ >> 3) & 7);
  if (line & 4) f ^= ((SWZ >> 6) & 7);
  if (line & 8) f ^= ((SWZ >> 9) & 7);
  return (lin & ~0x7f) | ((((lin >> 4) & 7) ^ f) << 4) | (lin & 15);
}

template <int D, int BITS, int GS, bool Q8, int NC>
struct DecCfg {
  static constexpr int RB = D * BITS / 8;      // bytes per code row
  static constexpr int UPR = RB / 16;          // 16-byte units per row
  static constexpr int NG = D / GS;            // groups per row
  static constexpr int GB = GS * BITS / 8;     // bytes per group per row
  static constexpr int NW = GS * BITS / 128;   // K-fragment words per thread per (row, group)
  static constexpr int KPG = GS / 16;          // k-steps per group == V m-tiles per group
  static constexpr int KSTEPS = D / 16;
  static constexpr int MT = D / 16;
  static constexpr int CB = GS * BITS / 64;    // V chunk bytes per thread per (key, group)
  static constexpr int CW = CB >= 4 ? CB / 4 : 1;
  static constexpr int NMETA = Q8 ? 2 : 4;
  static constexpr int MROW = NG * 2;          // meta bytes per key per array
  static constexpr int WPC = kDecWarps / NC;   // warps per head chunk
  static constexpr int TK = 16 * WPC;          // keys per stage
  static constexpr int CODES = TK * RB;
  static constexpr int META = ((TK * MROW + 127) / 128) * 128;
  static constexpr int META_UNITS = TK * MROW / 16;
  static constexpr int STAGE = 2 * CODES + NMETA * META;
  static constexpr int NSTAGE = kDecStageBudget / STAGE > 6 ? 6
                              : (kDecStageBudget / STAGE < 2 ? 2 : kDecStageBudget / STAGE);
  static constexpr int EPI = kDecWarps * (8 * D + 16) * 4;
  static constexpr int SMEM = NSTAGE * STAGE > EPI ? NSTAGE * STAGE : EPI;
  static constexpr uint32_t SWZ = swizzle_coeffs(D, BITS, GS);
  static_assert(D % GS == 0, "D must be a multiple of the group size");
  static_assert(NG <= 8, "at most 8 groups per row");
  static_assert(RB % 16 == 0, "code rows must be whole 16-byte units");
};

// Vector shared-memory loads of N 32-bit words (N in 1, 2, 4).
template <int N>
__device__ __forceinline__ void lds_words(const uint8_t* p, uint32_t* w) {
  if constexpr (N == 1) {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  } else if constexpr (N == 2) {
    uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x; w[1] = v.y;
  } else {
    uint4 v = *reinterpret_cast<const uint4*>(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  }
}

// NG half values (raw bits) of one key's metadata row.
template <int NG>
__device__ __forceinline__ void lds_meta(const uint8_t* p, uint16_t* h) {
  if constexpr (NG == 1) {
    h[0] = *reinterpret_cast<const uint16_t*>(p);
  } else {
    uint32_t w[NG / 2];
    lds_words<NG / 2 == 3 ? 2 : NG / 2>(p, w);
#pragma unroll
    for (int i = 0; i < NG / 2; ++i) { h[2 * i] = w[i] & 0xffff; h[2 * i + 1] = w[i] >> 16; }
  }
}

template <int D, int BITS, int GS, bool Q8, int NC, bool F32OUT>
__global__ void __launch_bounds__(kDecThreads, 1)
qsdpa_decode_kernel(const DecodeParams p) {
  using C = DecCfg<D, BITS, GS, Q8, NC>;
  constexpr int NG = C::NG, KPG = C::KPG, MT = C::MT, TK = C::TK, NSTAGE = C::NSTAGE;
  constexpr int HPC = NC * 8;
  extern __shared__ __align__(128) uint8_t smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int chunk = warp / C::WPC, sub = warp % C::WPC;
  const int64_t S = p.stages_per_unit, T = p.total_stages;
  const int64_t nC = gridDim.x;
  const int64_t lo = (int64_t)blockIdx.x * T / nC, hi = ((int64_t)blockIdx.x + 1) * T / nC;
  const int64_t first_unit = lo / S;
  __shared__ int s_flag;

  for (int64_t x = lo; x < hi;) {
    const int64_t u = x / S;
    const int s0 = (int)(x - u * S);
    const int s1 = (int)(min(hi, (u + 1) * S) - u * S);
    x = u * S + s1;

    const int cg = (int)(u % p.ncg);
    const int hkv = (int)((u / p.ncg) % p.Hkv);
    const int b = (int)(u / ((int64_t)p.ncg * p.Hkv));
    const int64_t row0 = ((int64_t)b * p.Hkv + hkv) * p.Lcap;   // first cache row of this head
    const int hbase = cg * HPC;                                  // first local head of the CTA
    const int myhead = hbase + chunk * 8 + g;                    // head whose q this lane loads
    const bool head_ok = myhead < p.G;

    // ---------------- query fragments (B operand of the score MMA) ----------
    uint32_t bq[C::KSTEPS][2];
    float qsc[NG][2];
    float scaleK;
    {
      const int64_t qrow = (((int64_t)b * p.Hkv + hkv) * p.G + myhead) * D;
      float qv[C::KSTEPS][4];
      float qs[NG];
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) qs[gg] = 0.f;
      float qmax = 0.f;
#pragma unroll
      for (int s = 0; s < C::KSTEPS; ++s) {
        const int G = s / KPG, ks = s % KPG;
        int e[4];
        if constexpr (BITS == 4) {
          const int m = ks >> 1, hi2 = (ks & 1) * 2;
          const int e0 = G * GS + (t * C::NW + m) * 8 + hi2;
          e[0] = e0; e[1] = e0 + 4; e[2] = e0 + 1; e[3] = e0 + 5;
        } else {
          const int e0 = G * GS + (t * C::NW + ks) * 4;
          e[0] = e0; e[1] = e0 + 2; e[2] = e0 + 1; e[3] = e0 + 3;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          qv[s][i] = head_ok ? load_as_float(p.q, p.q_dtype, qrow + e[i]) : 0.f;
          qs[G] += qv[s][i];
          qmax = fmaxf(qmax, fabsf(qv[s][i]));
        }
      }
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) qmax = fmaxf(qmax, __shfl_xor_sync(~0u, qmax, off));
      // prescale q by 2^sigma so that max|q'| lies in [2^14, 2^15)
      int sigma = qmax > 0.f ? 14 - (int)(((__float_as_uint(qmax) >> 23) & 0xff) - 127) : 0;
      sigma = max(-96, min(96, sigma));
      const float qscale = exp2i(sigma);
      const float qscale16 = exp2i(sigma - 4);
#pragma unroll
      for (int s = 0; s < C::KSTEPS; ++s) {
        if constexpr (BITS == 4) {
          bq[s][0] = pack_half2(qv[s][0] * qscale, qv[s][1] * qscale);
          bq[s][1] = pack_half2(qv[s][2] * qscale16, qv[s][3] * qscale16);
        } else {
          bq[s][0] = pack_half2(qv[s][0] * qscale, qv[s][1] * qscale);
          bq[s][1] = pack_half2(qv[s][2] * qscale, qv[s][3] * qscale);
        }
      }
      // group sums: reduce over t, then hand heads 2t, 2t+1 to every lane
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
        qs[gg] += __shfl_xor_sync(~0u, qs[gg], 1);
        qs[gg] += __shfl_xor_sync(~0u, qs[gg], 2);
        qsc[gg][0] = __shfl_sync(~0u, qs[gg], (2 * t) * 4) * p.scale_log2e;
        qsc[gg][1] = __shfl_sync(~0u, qs[gg], (2 * t + 1) * 4) * p.scale_log2e;
      }
      scaleK = p.scale_log2e * exp2i(24 - sigma);
    }

    // ---------------- running state ----------------------------------------
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float beta[2][NG];
    float O[MT][4];
#pragma unroll
    for (int gg = 0; gg < NG; ++gg) { beta[0][gg] = 0.f; beta[1][gg] = 0.f; }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) { O[mt][0] = O[mt][1] = O[mt][2] = O[mt][3] = 0.f; }

    const uint8_t* gK = p.kc + row0 * C::RB;
    const uint8_t* gV = p.vc + row0 * C::RB;
    const uint8_t* gKs = reinterpret_cast<const uint8_t*>(p.ks + row0 * NG);
    const uint8_t* gKb = Q8 ? gKs : reinterpret_cast<const uint8_t*>(p.kb + row0 * NG);
    const uint8_t* gVs = reinterpret_cast<const uint8_t*>(p.vs + row0 * NG);
    const uint8_t* gVb = Q8 ? gVs : reinterpret_cast<const uint8_t*>(p.vb + row0 * NG);
    const int64_t L = p.L;

    auto issue_stage = [&](int stage, int buf) {
      uint8_t* sb = smem + buf * C::STAGE;
      const int64_t key0 = (int64_t)stage * TK;
      constexpr int CU = TK * C::UPR;
#pragma unroll 4
      for (int i = tid; i < 2 * CU; i += kDecThreads) {
        const int which = i >= CU;
        const int j = which ? i - CU : i;
        const int row = j / C::UPR, cu = j - row * C::UPR;
        const int64_t key = key0 + row;
        const uint8_t* base = which ? gV : gK;
        const bool ok = key < L;
        const uint8_t* src = ok ? base + key * C::RB + cu * 16 : base;
        const int lin = row * C::RB + cu * 16;
        cp_async16(smem_u32(sb + which * C::CODES + swz_offset<C::SWZ>(lin)), src, ok ? 16 : 0);
      }
      for (int i = tid; i < C::NMETA * C::META_UNITS; i += kDecThreads) {
        const int arr = i / C::META_UNITS, j = i - arr * C::META_UNITS;
        // affine: K scales, K biases, V scales, V biases; Q8_0: K scales, V scales
        const uint8_t* gm = Q8 ? (arr == 0 ? gKs : gVs)
                               : (arr == 0 ? gKs : arr == 1 ? gKb : arr == 2 ? gVs : gVb);
        const int64_t kfirst = key0 + (j * 16) / C::MROW;
        const bool ok = kfirst < L;
        const uint8_t* src = ok ? gm + key0 * C::MROW + j * 16 : gm;
        cp_async16(smem_u32(sb + 2 * C::CODES + arr * C::META + j * 16), src, ok ? 16 : 0);
      }
    };

    const int nst = s1 - s0;
#pragma unroll
    for (int i = 0; i < NSTAGE - 1; ++i) {
      if (i < nst) issue_stage(s0 + i, i);
      cp_async_commit();
    }

    for (int it = 0; it < nst; ++it) {
      cp_async_wait<NSTAGE - 2>();
      __syncthreads();
      {
        const int nx = it + NSTAGE - 1;
        if (nx < nst) issue_stage(s0 + nx, nx % NSTAGE);
        cp_async_commit();
      }
      uint8_t* sb = smem + (it % NSTAGE) * C::STAGE;
      const int64_t key0 = (int64_t)(s0 + it) * TK;
      if (key0 + TK > L) {
        // keys past L: clear their (possibly stale) scales and biases
        const int first_bad = (int)(L - key0);
        uint16_t* meta = reinterpret_cast<uint16_t*>(sb + 2 * C::CODES);
        for (int i = tid; i < C::NMETA * TK * NG; i += kDecThreads) {
          const int arr = i / (TK * NG), r = i - arr * TK * NG;
          if (r / NG >= first_bad) meta[arr * (C::META / 2) + r] = 0;
        }
        __syncthreads();
      }

      const int k0 = sub * 16;
      const int64_t kg0 = key0 + k0;
      if (kg0 >= L) continue;                      // warp-uniform: whole block past L
      const uint8_t* sK = sb;
      const uint8_t* sV = sb + C::CODES;
      const uint8_t* sMeta = sb + 2 * C::CODES;

      // metadata of keys k0+g (row 0) and k0+g+8 (row 1)
      uint16_t ks0[NG], ks1[NG], kb0[NG], kb1[NG], vs0[NG], vs1[NG], vb0[NG], vb1[NG];
      {
        const int r0 = k0 + g, r1 = r0 + 8;
        if constexpr (Q8) {
          lds_meta<NG>(sMeta + r0 * C::MROW, ks0);
          lds_meta<NG>(sMeta + r1 * C::MROW, ks1);
          lds_meta<NG>(sMeta + C::META + r0 * C::MROW, vs0);
          lds_meta<NG>(sMeta + C::META + r1 * C::MROW, vs1);
        } else {
          lds_meta<NG>(sMeta + r0 * C::MROW, ks0);
          lds_meta<NG>(sMeta + r1 * C::MROW, ks1);
          lds_meta<NG>(sMeta + C::META + r0 * C::MROW, kb0);
          lds_meta<NG>(sMeta + C::META + r1 * C::MROW, kb1);
          lds_meta<NG>(sMeta + 2 * C::META + r0 * C::MROW, vs0);
          lds_meta<NG>(sMeta + 2 * C::META + r1 * C::MROW, vs1);
          lds_meta<NG>(sMeta + 3 * C::META + r0 * C::MROW, vb0);
          lds_meta<NG>(sMeta + 3 * C::META + r1 * C::MROW, vb1);
        }
      }

      // ---------------- scores S[key][head] (base-2 logits) ------------------
      float S[4] = {0.f, 0.f, 0.f, 0.f};
      {
        const int r0 = k0 + g, r1 = r0 + 8;
        int s = 0;
#pragma unroll
        for (int G = 0; G < NG; ++G) {
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
          uint32_t w0[C::NW], w1[C::NW];
          const int byte = G * C::GB + t * C::NW * 4;
#pragma unroll
          for (int part = 0; part < (C::NW + 3) / 4; ++part) {
            constexpr int PW = C::NW < 4 ? C::NW : 4;
            lds_words<PW>(sK + swz_offset<C::SWZ>(r0 * C::RB + byte + part * 16), w0 + part * 4);
            lds_words<PW>(sK + swz_offset<C::SWZ>(r1 * C::RB + byte + part * 16), w1 + part * 4);
          }
#pragma unroll
          for (int m = 0; m < C::NW; ++m) {
            if constexpr (BITS == 4) {
              uint32_t a[4] = {w0[m] & 0x000F000Fu, w1[m] & 0x000F000Fu,
                               w0[m] & 0x00F000F0u, w1[m] & 0x00F000F0u};
              mma_f16(acc, a, bq[s][0], bq[s][1], acc);
              ++s;
              const uint32_t y0 = w0[m] >> 8, y1 = w1[m] >> 8;
              uint32_t a2[4] = {y0 & 0x000F000Fu, y1 & 0x000F000Fu,
                                y0 & 0x00F000F0u, y1 & 0x00F000F0u};
              mma_f16(acc, a2, bq[s][0], bq[s][1], acc);
              ++s;
            } else {
              const uint32_t x0 = Q8 ? (w0[m] ^ 0x80808080u) : w0[m];
              const uint32_t x1 = Q8 ? (w1[m] ^ 0x80808080u) : w1[m];
              uint32_t a[4] = {x0 & 0x00FF00FFu, x1 & 0x00FF00FFu,
                               prmt(x0, 0u, 0x4341u), prmt(x1, 0u, 0x4341u)};
              mma_f16(acc, a, bq[s][0], bq[s][1], acc);
              ++s;
            }
          }
          const float sk0 = half_bits_to_float(ks0[G]), sk1 = half_bits_to_float(ks1[G]);
          const float bb0 = Q8 ? -128.f * sk0 : half_bits_to_float(kb0[G]);
          const float bb1 = Q8 ? -128.f * sk1 : half_bits_to_float(kb1[G]);
          const float c0 = sk0 * scaleK, c1 = sk1 * scaleK;
          S[0] = fmaf(c0, acc[0], fmaf(bb0, qsc[G][0], S[0]));
          S[1] = fmaf(c0, acc[1], fmaf(bb0, qsc[G][1], S[1]));
          S[2] = fmaf(c1, acc[2], fmaf(bb1, qsc[G][0], S[2]));
          S[3] = fmaf(c1, acc[3], fmaf(bb1, qsc[G][1], S[3]));
        }
      }
      if (kg0 + 16 > L) {
        if (kg0 + g >= L) { S[0] = -INFINITY; S[1] = -INFINITY; }
        if (kg0 + g + 8 >= L) { S[2] = -INFINITY; S[3] = -INFINITY; }
      }
      if (p.mask_kind != QKV_MASK_NONE) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int vh = hbase + chunk * 8 + 2 * t + j;     // row = head * Lq + query
          if (vh < p.G) {
            const int hr = vh / p.Lq, qi = vh - hr * p.Lq;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const int64_t key = kg0 + g + 8 * r;
              if (key >= L) continue;
              if (p.mask_kind == QKV_MASK_CAUSAL) {
                if (key > L - p.Lq + qi) S[2 * r + j] = -INFINITY;
              } else {
                const int64_t mi = (int64_t)b * p.msb + ((int64_t)hkv * p.Gq + hr) * p.msh +
                                   (int64_t)qi * p.msq + key;
                S[2 * r + j] += kLog2e * load_as_float(p.mask, p.mask_dtype, mi);
              }
            }
          }
        }
      }

      // ---------------- online softmax ----------------------------------------
      float t0 = fmaxf(S[0], S[2]), t1 = fmaxf(S[1], S[3]);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        t0 = fmaxf(t0, __shfl_xor_sync(~0u, t0, off));
        t1 = fmaxf(t1, __shfl_xor_sync(~0u, t1, off));
      }
      const float n0 = fmaxf(m0, t0), n1 = fmaxf(m1, t1);
      const float u0 = n0 == -INFINITY ? 0.f : n0, u1 = n1 == -INFINITY ? 0.f : n1;
      const float al0 = ex2(m0 - u0), al1 = ex2(m1 - u1);
      const float p0 = ex2(S[0] - u0), p1 = ex2(S[1] - u1);
      const float p2 = ex2(S[2] - u0), p3 = ex2(S[3] - u1);
      m0 = n0; m1 = n1;
      l0 = fmaf(l0, al0, p0 + p2);
      l1 = fmaf(l1, al1, p1 + p3);
      if (__any_sync(~0u, (al0 != 1.f) || (al1 != 1.f))) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          O[mt][0] *= al0; O[mt][1] *= al1; O[mt][2] *= al0; O[mt][3] *= al1;
        }
#pragma unroll
        for (int G = 0; G < NG; ++G) { beta[0][G] *= al0; beta[1][G] *= al1; }
      }
      if constexpr (!Q8) {
#pragma unroll
        for (int G = 0; G < NG; ++G) {
          const float vb0f = half_bits_to_float(vb0[G]), vb1f = half_bits_to_float(vb1[G]);
          beta[0][G] = fmaf(p0, vb0f, fmaf(p2, vb1f, beta[0][G]));
          beta[1][G] = fmaf(p1, vb0f, fmaf(p3, vb1f, beta[1][G]));
        }
      }

      // ---------------- values --------------------------------------------------
#pragma unroll
      for (int G = 0; G < NG; ++G) {
        uint32_t mx = max((uint32_t)vs0[G], (uint32_t)vs1[G]);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) mx = max(mx, __shfl_xor_sync(~0u, mx, off));
        const int E = (int)((mx >> 10) & 31);
        const int tau = mx == 0 ? 0 : 14 - (E == 0 ? -15 : E - 15);
        const float up = exp2i(tau);
        const float sv0 = half_bits_to_float(vs0[G]) * up, sv1 = half_bits_to_float(vs1[G]) * up;
        const float x00 = p0 * sv0, x01 = p1 * sv0, x10 = p2 * sv1, x11 = p3 * sv1;
        const uint32_t top = pack_half2(x00, x01), bot = pack_half2(x10, x11);
        const uint32_t b0 = movmatrix_trans(top), b1 = movmatrix_trans(bot);
        uint32_t b0l = 0, b1l = 0;
        if constexpr (F32OUT) {
          const float2 ft = unpack_half2(top), fb = unpack_half2(bot);
          b0l = movmatrix_trans(pack_half2(x00 - ft.x, x01 - ft.y));
          b1l = movmatrix_trans(pack_half2(x10 - fb.x, x11 - fb.y));
        }
        // codes of keys 2t, 2t+1, 2t+8, 2t+9 for this lane's chunk of group G
        uint32_t wa[C::CW], wb[C::CW], wc[C::CW], wd[C::CW];
        {
          const int byte = G * C::GB + g * C::CB;
          const int ra = k0 + 2 * t;
          if constexpr (C::CB == 2) {
            wa[0] = *reinterpret_cast<const uint16_t*>(sV + swz_offset<C::SWZ>(ra * C::RB + byte));
            wb[0] = *reinterpret_cast<const uint16_t*>(sV + swz_offset<C::SWZ>((ra + 1) * C::RB + byte));
            wc[0] = *reinterpret_cast<const uint16_t*>(sV + swz_offset<C::SWZ>((ra + 8) * C::RB + byte));
            wd[0] = *reinterpret_cast<const uint16_t*>(sV + swz_offset<C::SWZ>((ra + 9) * C::RB + byte));
          } else {
            lds_words<C::CW>(sV + swz_offset<C::SWZ>(ra * C::RB + byte), wa);
            lds_words<C::CW>(sV + swz_offset<C::SWZ>((ra + 1) * C::RB + byte), wb);
            lds_words<C::CW>(sV + swz_offset<C::SWZ>((ra + 8) * C::RB + byte), wc);
            lds_words<C::CW>(sV + swz_offset<C::SWZ>((ra + 9) * C::RB + byte), wd);
          }
          if constexpr (Q8) {
#pragma unroll
            for (int i = 0; i < C::CW; ++i) {
              wa[i] ^= 0x80808080u; wb[i] ^= 0x80808080u; wc[i] ^= 0x80808080u; wd[i] ^= 0x80808080u;
            }
          }
        }
        // fp32 factor undoing tau and the subnormal code scaling
        const float f_lo = exp2i((Q8 ? 0 : 24) - tau);
        const float f_hi = exp2i((Q8 ? 0 : (BITS == 4 ? 20 : 24)) - tau);
#pragma unroll
        for (int i = 0; i < KPG; ++i) {
          uint32_t a[4];
          if constexpr (BITS == 4) {
            const int w = i >> 2;
            const uint32_t sel = ((4u + (i & 3)) << 8) | (uint32_t)(i & 3);
            const uint32_t xv = prmt(wa[w], wb[w], sel), yv = prmt(wc[w], wd[w], sel);
            a[0] = xv & 0x000F000Fu; a[1] = xv & 0x00F000F0u;
            a[2] = yv & 0x000F000Fu; a[3] = yv & 0x00F000F0u;
          } else {
            const int w = i >> 1;
            const uint32_t mA = wa[w] & 0x00FF00FFu, mB = wb[w] & 0x00FF00FFu;
            const uint32_t nA = wa[w] & 0xFF00FF00u, nB = wb[w] & 0xFF00FF00u;
            const uint32_t mC = wc[w] & 0x00FF00FFu, mD = wd[w] & 0x00FF00FFu;
            const uint32_t nC2 = wc[w] & 0xFF00FF00u, nD = wd[w] & 0xFF00FF00u;
            const uint32_t selm = (i & 1) ? 0x7632u : 0x5410u;
            const uint32_t seln = (i & 1) ? 0x6723u : 0x4501u;
            a[0] = prmt(mA, mB, selm); a[1] = prmt(nA, nB, seln);
            a[2] = prmt(mC, mD, selm); a[3] = prmt(nC2, nD, seln);
            if constexpr (Q8) {
              // exact signed codes: (1024 + u) - 1152 with u = code + 128
              const __half2 off = __float2half2_rn(1152.f);
#pragma unroll
              for (int r = 0; r < 4; ++r) {
                uint32_t v = a[r] | 0x64006400u;
                __half2 hv = __hsub2(*reinterpret_cast<__half2*>(&v), off);
                a[r] = *reinterpret_cast<uint32_t*>(&hv);
              }
            }
          }
          float d[4];
          const float z[4] = {0.f, 0.f, 0.f, 0.f};
          mma_f16(d, a, b0, b1, z);
          if constexpr (F32OUT) mma_f16(d, a, b0l, b1l, d);
          const int mt = G * KPG + i;
          O[mt][0] = fmaf(d[0], f_lo, O[mt][0]);
          O[mt][1] = fmaf(d[1], f_lo, O[mt][1]);
          O[mt][2] = fmaf(d[2], f_hi, O[mt][2]);
          O[mt][3] = fmaf(d[3], f_hi, O[mt][3]);
        }
      }
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---------------- epilogue: combine the warps of each head chunk ----------
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(~0u, l0, off);
      l1 += __shfl_xor_sync(~0u, l1, off);
#pragma unroll
      for (int G = 0; G < NG; ++G) {
        beta[0][G] += __shfl_xor_sync(~0u, beta[0][G], off);
        beta[1][G] += __shfl_xor_sync(~0u, beta[1][G], off);
      }
    }
    float* ws = reinterpret_cast<float*>(smem) + warp * (8 * D + 16);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int G = mt / KPG, i = mt % KPG;
      const int e = G * GS + g * (GS / 8) + 2 * i;
      ws[(2 * t) * D + e] = O[mt][0] + beta[0][G];
      ws[(2 * t + 1) * D + e] = O[mt][1] + beta[1][G];
      ws[(2 * t) * D + e + 1] = O[mt][2] + beta[0][G];
      ws[(2 * t + 1) * D + e + 1] = O[mt][3] + beta[1][G];
    }
    if (g == 0) {
      ws[8 * D + 2 * t] = m0; ws[8 * D + 2 * t + 1] = m1;
      ws[8 * D + 8 + 2 * t] = l0; ws[8 * D + 8 + 2 * t + 1] = l1;
    }
    __syncthreads();

    const bool complete = (s0 == 0) && (s1 == (int)S);
    const int64_t slot = 2 * (int64_t)blockIdx.x + (u == first_unit ? 0 : 1);
    const float* wsf = reinterpret_cast<const float*>(smem);
    for (int idx = tid; idx < HPC * D; idx += kDecThreads) {
      const int hl = idx / D, e = idx - hl * D;       // hl: head within the chunk-group
      const int c = hl >> 3, hh = hl & 7;
      const int head = hbase + hl;
      if (head >= p.G) continue;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < C::WPC; ++w) M = fmaxf(M, wsf[(c * C::WPC + w) * (8 * D + 16) + 8 * D + hh]);
      float o = 0.f, l = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < C::WPC; ++w) {
          const float* wp = wsf + (c * C::WPC + w) * (8 * D + 16);
          const float mw = wp[8 * D + hh];
          if (mw == -INFINITY) continue;
          const float sc = ex2(mw - M);
          o = fmaf(sc, wp[hh * D + e], o);
          l = fmaf(sc, wp[8 * D + 8 + hh], l);
        }
      }
      if (complete) {
        const int64_t oi = (((int64_t)b * p.Hkv + hkv) * p.G + head) * D + e;
        store_from_float(p.out, p.out_dtype, oi, l > 0.f ? o / l : 0.f);
      } else {
        p.part_o[(slot * HPC + hl) * D + e] = o;
        if (e == 0) {
          p.part_ml[(slot * HPC + hl) * 2 + 0] = M;
          p.part_ml[(slot * HPC + hl) * 2 + 1] = l;
        }
      }
    }

    if (!complete) {
      // last CTA of this unit to arrive merges all partial results
      __threadfence();
      __syncthreads();
      const int64_t cfirst = ((u * S + 1) * nC - 1) / T;
      const int64_t clast = (((u + 1) * S) * nC - 1) / T;
      if (tid == 0) {
        const unsigned nparts = (unsigned)(clast - cfirst + 1);
        const unsigned prev = atomicAdd(&p.tickets[u], 1u);
        const int last = prev == nparts - 1;
        if (last) p.tickets[u] = 0u;
        s_flag = last;
      }
      __syncthreads();
      if (s_flag) {
        __threadfence();
        for (int idx = tid; idx < HPC * D; idx += kDecThreads) {
          const int hl = idx / D, e = idx - hl * D;
          const int head = hbase + hl;
          if (head >= p.G) continue;
          float M = -INFINITY, l = 0.f, o = 0.f;
          for (int64_t c = cfirst; c <= clast; ++c) {
            const int64_t clo = c * T / nC;
            const int64_t sl = 2 * c + ((clo / S) == u ? 0 : 1);
            const float mp = __ldcg(&p.part_ml[(sl * HPC + hl) * 2 + 0]);
            if (mp == -INFINITY) continue;
            const float lp = __ldcg(&p.part_ml[(sl * HPC + hl) * 2 + 1]);
            const float op = __ldcg(&p.part_o[(sl * HPC + hl) * D + e]);
            if (mp > M) {
              const float sc = ex2(M - mp);     // M = -inf -> 0
              o *= sc; l *= sc; M = mp;
            }
            const float sc = ex2(mp - M);
            o = fmaf(sc, op, o);
            l = fmaf(sc, lp, l);
          }
          const int64_t oi = (((int64_t)b * p.Hkv + hkv) * p.G + head) * D + e;
          store_from_float(p.out, p.out_dtype, oi, l > 0.f ? o / l : 0.f);
        }
      }
    }
    __syncthreads();
  }
}

// Host-side helpers for one instance.
template <int D, int BITS, int GS, bool Q8, int NC, bool F32OUT>
struct DecodeInstance {
  using C = DecCfg<D, BITS, GS, Q8, NC>;
  static int max_ctas_per_sm() {
    static int cached = -1;
    if (cached < 0) {
      auto k = qsdpa_decode_kernel<D, BITS, GS, Q8, NC, F32OUT>;
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
        return 0;
      int n = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kDecThreads, C::SMEM) != cudaSuccess)
        return 0;
      cached = n;
    }
    return cached;
  }
  static cudaError_t launch(const DecodePlan& plan, const DecodeParams& p, cudaStream_t s) {
    auto k = qsdpa_decode_kernel<D, BITS, GS, Q8, NC, F32OUT>;
    k<<<plan.grid, kDecThreads, C::SMEM, s>>>(p);
    return cudaGetLastError();
  }
};

}  // namespace qkv
