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

// 8 warps per CTA; two CTAs per SM for D <= 128 (independent CTAs overlap
// each other's stage boundaries), one for D = 256 (more registers per thread).
__host__ __device__ constexpr int dec_warps(int) { return 8; }
constexpr int kDecWarpsMax = 8;
__host__ __device__ constexpr int dec_ctas_per_sm(int D) { return D <= 128 ? 2 : 1; }

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

// XOR coefficients of the value tile's swizzle: the value fragments are read
// with ldmatrix, 8 key rows x one 16-byte unit per matrix, and these make the
// 8 rows hit 8 different bank groups (exhaustive search over the same family).
__host__ __device__ constexpr uint32_t vswizzle_coeffs(int rb) {
  return rb == 32 ? swz_pack(1, 0, 0, 0) : rb == 64 ? swz_pack(1, 2, 0, 0)
       : rb == 128 ? swz_pack(1, 2, 4, 0) : swz_pack(0, 1, 2, 4);
}

// XOR pattern (already shifted to bits 4..6) of 128-byte line `line`.
template <uint32_t SWZ>
__host__ __device__ __forceinline__ constexpr int swz_line(int line) {
  return (((line & 1) ? (SWZ & 7) : 0) ^ ((line & 2) ? ((SWZ >> 3) & 7) : 0) ^
          ((line & 4) ? ((SWZ >> 6) & 7) : 0) ^ ((line & 8) ? ((SWZ >> 9) & 7) : 0)) << 4;
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
  static constexpr int NWARP = dec_warps(D);
  static constexpr int NTHR = 32 * NWARP;
  static constexpr int WPC = NWARP / NC;       // warps per head chunk
  // ring budget per CTA (228 KB per SM holds two CTAs of 108 KB plus their
  // reserved 1 KB each)
  static constexpr int BUDGET = D <= 128 ? 110592 : 224 * 1024;
  // 16-key blocks per warp per stage: two when three such stages fit, else one
  static constexpr int STAGE2 = 2 * (32 * WPC) * RB + NMETA * (((32 * WPC * MROW + 127) / 128) * 128);
  static constexpr int SUB = 3 * STAGE2 <= BUDGET ? 2 : 1;
  static constexpr int TK = 16 * SUB * WPC;      // keys per stage
  static constexpr int CODES = TK * RB;
  static constexpr int META = ((TK * MROW + 127) / 128) * 128;
  static constexpr int META_UNITS = TK * MROW / 16;
  static constexpr int STAGE = 2 * CODES + NMETA * META;
  static constexpr int NSTAGE = BUDGET / STAGE > 6 ? 6 : (BUDGET / STAGE < 2 ? 2 : BUDGET / STAGE);
  // epilogue: per-warp partial rows
  static constexpr int EPI = NWARP * (8 * D + 16) * 4;
  static constexpr int RING = NSTAGE * STAGE > EPI ? NSTAGE * STAGE : EPI;
  static constexpr int QSB = NC * 8 * D * 4;            // fp32 query rows (in the last ring slot)
  static constexpr int SMEM = RING > (NSTAGE - 1) * STAGE + QSB ? RING : (NSTAGE - 1) * STAGE + QSB;
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t SWZ = swizzle_coeffs(D, BITS, GS);   // key tile
  static constexpr uint32_t SWZV = vswizzle_coeffs(RB);          // value tile
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

// a / b for non-negative 64-bit values, in 32-bit arithmetic when both fit
// (the common case; 64-bit division costs several times more instructions).
__device__ __forceinline__ int64_t udiv64(int64_t a, int64_t b) {
  if (((uint64_t)a | (uint64_t)b) >> 32 == 0) return (int64_t)((uint32_t)a / (uint32_t)b);
  return a / b;
}

constexpr int kMergeBatch = 10;   // parts whose loads one merging thread has in flight
constexpr int kMergeGroup = 8;    // parts per first-level merge when a unit merges in two levels
constexpr int64_t kMergeFlat = 1 << 15;   // largest parts x rows x D merged by one CTA in one level

// Combines n partial results (m, l, o) of one unit by log-sum-exp rescaling.
// Part i lives in slot 2 * (c0 + i * step), except part 0, which is in slot0.
// Writes either the nrows normalized rows starting at element out_base
// (dst_o == nullptr) or one combined partial (dst_ml, dst_o).  A thread owns 4
// consecutive outputs of one row and every tpi-th part; it loads (m, l) and o
// of a batch of parts at once and folds them in online, then the tpi threads
// of an output (adjacent lanes) combine with shuffles: one round trip per
// batch and no barrier.
template <int D, int HPC>
__device__ __noinline__ void merge_unit(const float* ml, const float* po, int n, int64_t slot0,
                                        int64_t c0, int step, int tid, int nthreads, int nrows,
                                        void* out, int out_dtype, int64_t out_base, float* dst_ml,
                                        float* dst_o) {
  constexpr int V4 = D / 4;
  const int items = nrows * V4;
  int tpi = 1;
  while (tpi < 32 && items * tpi * 2 <= nthreads) tpi *= 2;
  const int ipp = nthreads / tpi;                                 // items per pass
  const int sub = tid & (tpi - 1);
  for (int i0 = 0; i0 < items; i0 += ipp) {
    const int item = i0 + tid / tpi;
    const bool active = item < items;
    const int hl = active ? item / V4 : 0, e4 = active ? item - hl * V4 : 0;
    float M = -INFINITY, Ls = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int jb = 0; sub + tpi * jb < n; jb += kMergeBatch) {
      float4 o[kMergeBatch];
      float2 v[kMergeBatch];
#pragma unroll
      for (int k = 0; k < kMergeBatch; ++k) {
        const int pp = sub + tpi * (jb + k);
        if (active && pp < n) {
          const int64_t sx = pp == 0 ? slot0 : 2 * (c0 + (int64_t)pp * step);
          o[k] = __ldcg(reinterpret_cast<const float4*>(po + (sx * HPC + hl) * D) + e4);
          v[k] = __ldcg(reinterpret_cast<const float2*>(ml + (sx * HPC + hl) * 2));
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
    for (int off = 1; off < tpi; off <<= 1) {
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
    if (active && sub == 0) {
      if (dst_o != nullptr) {
        *reinterpret_cast<float4*>(dst_o + hl * D + e4 * 4) = acc;
        if (e4 == 0) { dst_ml[hl * 2] = M; dst_ml[hl * 2 + 1] = Ls; }
      } else {
        const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
        const int64_t oi = out_base + (int64_t)hl * D + e4 * 4;
        store_from_float(out, out_dtype, oi, acc.x * inv);
        store_from_float(out, out_dtype, oi + 1, acc.y * inv);
        store_from_float(out, out_dtype, oi + 2, acc.z * inv);
        store_from_float(out, out_dtype, oi + 3, acc.w * inv);
      }
    }
  }
}

// Transposing shared-memory matrix loads (8x8 of 16-bit elements per matrix).
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];\n"
               : "=r"(r0), "=r"(r1) : "r"(addr) : "memory");
}

// Raw fp16 bits of group G's scale (or bias) of row r in a staged meta array.
template <int NG>
__device__ __forceinline__ uint16_t meta_half(const uint8_t* base, int r, int G) {
  return reinterpret_cast<const uint16_t*>(base)[r * NG + G];
}

// Group G's value (as float) of a metadata row held as 32-bit words.
template <int NG>
__device__ __forceinline__ float meta_f(const uint32_t* w, int G) {
  if constexpr (NG == 1) {
    return half_bits_to_float((uint16_t)w[0]);
  } else {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[G >> 1]));
    return (G & 1) ? f.y : f.x;
  }
}
// Group G's 16-bit value of a metadata row held as 32-bit words.
template <int NG>
__device__ __forceinline__ uint32_t meta_bits(const uint32_t* w, int G) {
  if constexpr (NG == 1) return w[0] & 0xffffu;
  else return (G & 1) ? (w[G >> 1] >> 16) : (w[G >> 1] & 0xffffu);
}
// A key's NG metadata halves as 32-bit words.
template <int NG>
__device__ __forceinline__ void meta_row(const uint8_t* base, int r, uint32_t* w) {
  if constexpr (NG == 1) {
    w[0] = reinterpret_cast<const uint16_t*>(base)[r];
  } else {
    lds_words<NG / 2>(base + r * NG * 2, w);
  }
}

template <int D, int BITS, int GS, bool Q8, int NC, bool F32OUT>
__global__ void __launch_bounds__(32 * dec_warps(D), dec_ctas_per_sm(D))
qsdpa_decode_kernel(const DecodeParams p) {
  using C = DecCfg<D, BITS, GS, Q8, NC>;
  constexpr int NG = C::NG, KPG = C::KPG, MT = C::MT, TK = C::TK, NSTAGE = C::NSTAGE;
  constexpr int HPC = NC * 8;
  constexpr int MW = NG == 1 ? 1 : NG / 2;     // 32-bit words of one key's metadata row
  extern __shared__ __align__(128) uint8_t smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int chunk = warp / C::WPC, sub = warp % C::WPC;
  const int64_t S = p.stages_per_unit, T = p.total_stages;
  const int64_t nC = gridDim.x;
  const int64_t lo = udiv64((int64_t)blockIdx.x * T, nC), hi = udiv64(((int64_t)blockIdx.x + 1) * T, nC);
  const int64_t first_unit = udiv64(lo, S);
  __shared__ int s_flag;

  for (int64_t x = lo; x < hi;) {
    const int64_t u = udiv64(x, S);
    const int s0 = (int)(x - u * S);
    const int s1 = (int)(min(hi, (u + 1) * S) - u * S);
    x = u * S + s1;

    const int64_t uh = udiv64(u, p.ncg);                 // (batch, kv head)
    const int cg = (int)(u - uh * p.ncg);
    const int b = (int)udiv64(uh, p.Hkv);
    const int hkv = (int)(uh - (int64_t)b * p.Hkv);
    const int64_t row0 = ((int64_t)b * p.Hkv + hkv) * p.Lcap;   // first cache row of this head
    const int hbase = cg * HPC;                                  // first local row of the CTA

    const uint8_t* gK = p.kc + row0 * C::RB;
    const uint8_t* gV = p.vc + row0 * C::RB;
    const uint8_t* gKs = reinterpret_cast<const uint8_t*>(p.ks + row0 * NG);
    const uint8_t* gKb = Q8 ? gKs : reinterpret_cast<const uint8_t*>(p.kb + row0 * NG);
    const uint8_t* gVs = reinterpret_cast<const uint8_t*>(p.vs + row0 * NG);
    const uint8_t* gVb = Q8 ? gVs : reinterpret_cast<const uint8_t*>(p.vb + row0 * NG);
    const int64_t L = p.L;

    // copy plan: 16-byte unit i of a stage is row (i mod CU) / UPR of the K
    // tile (i < CU) or of the V tile.  When CU is a multiple of the thread
    // count every unit of a thread lies in a line with the same swizzle.
    constexpr int CU = TK * C::UPR;
    constexpr int NU = (2 * CU + C::NTHR - 1) / C::NTHR;
    const int fx_tid = swz_line<C::SWZ>((tid >> 3) & 15);
    const int fx_tid_v = swz_line<C::SWZV>((tid >> 3) & 15);

    constexpr bool META1 = C::NMETA * C::META_UNITS <= C::NTHR;   // one metadata unit per thread
    auto issue_stage = [&](int stage, int buf) {
      const uint32_t sbase = smem_u32(smem + buf * C::STAGE);
      const int64_t key0 = (int64_t)stage * TK;
      const int nvalid = (int)(L - key0 < (int64_t)TK ? L - key0 : (int64_t)TK);      // rows of this stage below L
      if (CU % C::NTHR == 0 && META1 && nvalid == TK) {
        // a full stage: fixed per-thread offsets, no per-unit tests.  Unit
        // tid + k * NTHR lies k * NTHR * 16 bytes further in both the source
        // and (the swizzle acts on bits below that) the stage.
        const uint8_t* ks = gK + key0 * C::RB + tid * 16;
        const uint8_t* vs = gV + key0 * C::RB + tid * 16;
        const uint32_t d0 = sbase + ((tid * 16) ^ fx_tid);
        const uint32_t d0v = sbase + C::CODES + ((tid * 16) ^ fx_tid_v);
#pragma unroll
        for (int k = 0; k < CU / C::NTHR; ++k) {
          cp_async16(d0 + k * C::NTHR * 16, ks + k * C::NTHR * 16, 16);
          cp_async16(d0v + k * C::NTHR * 16, vs + k * C::NTHR * 16, 16);
        }
        if (tid < C::NMETA * C::META_UNITS) {
          const int marr = tid / C::META_UNITS, mj = tid - marr * C::META_UNITS;
          const uint8_t* gm = Q8 ? (marr == 0 ? gKs : gVs)
                                 : (marr == 0 ? gKs : marr == 1 ? gKb : marr == 2 ? gVs : gVb);
          cp_async16(sbase + 2 * C::CODES + marr * C::META + mj * 16, gm + key0 * C::MROW + mj * 16, 16);
        }
        return;
      }
      const uint8_t* kb0 = gK + key0 * C::RB;
      const uint8_t* vb0 = gV + key0 * C::RB;
#pragma unroll
      for (int k = 0; k < NU; ++k) {
        const int i = tid + k * C::NTHR;
        if ((2 * CU) % C::NTHR == 0 || i < 2 * CU) {
          const int which = i >= CU, j = which ? i - CU : i;
          const bool ok = (j / C::UPR) < nvalid;
          const uint8_t* src = (which ? vb0 : kb0) + (ok ? j * 16 : 0);
          const int dst = (CU % C::NTHR == 0)
                              ? which * C::CODES + ((j * 16) ^ (which ? fx_tid_v : fx_tid))
                              : which * C::CODES + (which ? swz_offset<C::SWZV>(j * 16)
                                                          : swz_offset<C::SWZ>(j * 16));
          cp_async16(sbase + dst, src, ok ? 16 : 0);
        }
      }
      for (int i = tid; i < C::NMETA * C::META_UNITS; i += C::NTHR) {
        const int arr = i / C::META_UNITS, j = i - arr * C::META_UNITS;
        // affine: K scales, K biases, V scales, V biases; Q8_0: K scales, V scales
        const uint8_t* gm = Q8 ? (arr == 0 ? gKs : gVs)
                               : (arr == 0 ? gKs : arr == 1 ? gKb : arr == 2 ? gVs : gVb);
        const bool ok = (j * 16) / C::MROW < nvalid;
        const uint8_t* src = gm + (ok ? key0 * C::MROW + j * 16 : 0);
        cp_async16(sbase + 2 * C::CODES + arr * C::META + j * 16, src, ok ? 16 : 0);
      }
    };

    // fragment offsets inside a stage (fixed per lane).  The swizzle is
    // linear in the line bits and a group never straddles a line, so it splits
    // into a per-row part (computed once here), a per-group constant and, for
    // the second 16-key block, the constant of a 16-row shift.
    const int k0 = sub * 16 * C::SUB;
    auto row_x = [&](int r) { return swz_line<C::SWZ>((r * C::RB) >> 7); };
    const int xk0 = row_x(k0 + g), xk1 = row_x(k0 + g + 8);
    // value fragments: ldmatrix rows.  Lane l addresses row l % 8 of matrix
    // l / 8; matrices 0/1 hold keys 0-7, 2/3 keys 8-15 of the 16-key block, and
    // matrices 0/2 the first, 1/3 the second 16-byte unit of a unit pair (x2
    // loads for 4-bit groups of 32: matrix 0 keys 0-7, matrix 1 keys 8-15).
    constexpr bool VX2 = BITS == 4 && GS == 32;
    const int vkey = k0 + (lane & 7) + (VX2 ? ((lane >> 3) & 1) * 8 : ((lane >> 4) & 1) * 8);
    const int vunit = VX2 ? 0 : ((lane >> 3) & 1);
    auto koff = [&](int r, int x, int st, int G, int part) {
      return ((r * C::RB + G * C::GB + t * C::NW * 4 + part * 16) ^ x) ^
             swz_line<C::SWZ>((G * C::GB) >> 7) ^ swz_line<C::SWZ>((st * 16 * C::RB) >> 7);
    };

    const int nst = s1 - s0;
    // query rows: their (small) loads go out first, then the copies of the
    // first stages; the rows are staged as fp32 in the ring's last slot, which
    // the first NSTAGE-1 stages do not use
    float* qst = reinterpret_cast<float*>(smem + (NSTAGE - 1) * C::STAGE);
    constexpr int QCH = HPC * D / 8;                      // 16-byte query chunks
    constexpr int QPT = (QCH + C::NTHR - 1) / C::NTHR;
    // Value-scale bound for this CTA's keys of the unit: tau (per group) is
    // fixed so that P * s_v * 2^tau < 2^15 for every key (P <= 1), i.e.
    // tau = 29 - the largest exponent field of the group's value scales.  The
    // scales are loaded here, with the query, before the stages' copies
    // (which then find them in L2).
    __shared__ int s_vexp[kDecWarpsMax * 8];
    int vexp[NG];
    {
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) vexp[gg] = 0;
      const int64_t klo = (int64_t)s0 * TK;
      const int64_t khi = (int64_t)s1 * TK < L ? (int64_t)s1 * TK : L;
      const uint16_t* vsg = p.vs + (row0 + klo) * NG;
      const int nh = (int)((khi - klo) * NG);      // halves; whole 16-byte units stay in the slab
      constexpr int VB = 4;                        // 16-byte loads in flight per thread
      for (int c0 = tid * 8; c0 < nh; c0 += VB * C::NTHR * 8) {
        uint4 w4[VB];
#pragma unroll
        for (int k = 0; k < VB; ++k) {
          const int c = c0 + k * C::NTHR * 8;
          w4[k] = c < nh ? __ldg(reinterpret_cast<const uint4*>(vsg + c)) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int k = 0; k < VB; ++k) {
          const int c = c0 + k * C::NTHR * 8;
          const uint32_t w[4] = {w4[k].x, w4[k].y, w4[k].z, w4[k].w};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int e = (int)((w[j >> 1] >> (16 * (j & 1) + 10)) & 31);
            if (c + j < nh) vexp[j % NG] = max(vexp[j % NG], e);
          }
        }
      }
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) vexp[gg] = max(vexp[gg], __shfl_xor_sync(~0u, vexp[gg], off));
        if (lane == 0) s_vexp[warp * 8 + gg] = vexp[gg];
      }
    }
    uint4 qraw[QPT];
    {
      const int64_t qbase = (((int64_t)b * p.Hkv + hkv) * p.G + hbase) * D;
      const int nrows = min(HPC, p.G - hbase);
#pragma unroll
      for (int k = 0; k < QPT; ++k) {
        const int i = tid + k * C::NTHR;
        const int hl = i / (D / 8), c = i - hl * (D / 8);
        qraw[k] = make_uint4(0u, 0u, 0u, 0u);
        if (i < QCH && hl < nrows)
          qraw[k] = __ldg(reinterpret_cast<const uint4*>(
              reinterpret_cast<const uint16_t*>(p.q) + qbase + (int64_t)hl * D + c * 8));
      }
    }
#pragma unroll
    for (int i = 0; i < NSTAGE - 1; ++i) {
      if (i < nst) issue_stage(s0 + i, i);
      cp_async_commit();
    }
#pragma unroll
    for (int k = 0; k < QPT; ++k) {
      const int i = tid + k * C::NTHR;
      if (QCH % C::NTHR == 0 || i < QCH) {
        const uint32_t w[4] = {qraw[k].x, qraw[k].y, qraw[k].z, qraw[k].w};
        float v[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (p.q_dtype == QKV_F16) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
            v[2 * j] = f.x; v[2 * j + 1] = f.y;
          } else {
            v[2 * j] = __uint_as_float(w[j] << 16);
            v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
          }
        }
        float4* dst = reinterpret_cast<float4*>(qst + i * 8);
        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
      }
    }
    __syncthreads();

    // ---------------- query fragments (B operand of the score MMA) ----------
    uint32_t bq[C::KSTEPS][2];
    float qsc[NG][2];
    float scaleK;
    {
      const float* qr = qst + (chunk * 8 + g) * D;
      float qs[NG];
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) qs[gg] = 0.f;
      float qmax = 0.f;
      float qv[C::KSTEPS][4];
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
          qv[s][i] = qr[e[i]];
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
        const float sc2 = BITS == 4 ? qscale16 : qscale;
        bq[s][0] = pack_half2(qv[s][0] * qscale, qv[s][1] * qscale);
        bq[s][1] = pack_half2(qv[s][2] * sc2, qv[s][3] * sc2);
      }
      // group sums: reduce over t, then hand rows 2t, 2t+1 to every lane
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
    int tau[NG];          // per group: the value operand carries 2^tau
#pragma unroll
    for (int gg = 0; gg < NG; ++gg) {
      beta[0][gg] = 0.f; beta[1][gg] = 0.f;
      int e = 0;
#pragma unroll
      for (int w = 0; w < C::NWARP; ++w) e = max(e, s_vexp[w * 8 + gg]);
      tau[gg] = 29 - e;
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) { O[mt][0] = O[mt][1] = O[mt][2] = O[mt][3] = 0.f; }

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
      const int kvalid = (int)(L - key0 < (int64_t)TK ? L - key0 : (int64_t)TK);   // valid keys of this stage
      if (kvalid < TK) {
        // keys past L: clear their (possibly stale) scales and biases
        uint16_t* meta = reinterpret_cast<uint16_t*>(sb + 2 * C::CODES);
        for (int i = tid; i < C::NMETA * TK * NG; i += C::NTHR) {
          const int arr = i / (TK * NG), r = i - arr * TK * NG;
          if (r / NG >= kvalid) meta[arr * (C::META / 2) + r] = 0;
        }
        __syncthreads();
      }
      if (k0 >= kvalid) continue;                  // warp-uniform: whole block past L
      const uint8_t* sK = sb;
      const uint8_t* sV = sb + C::CODES;
      const uint8_t* sMeta = sb + 2 * C::CODES;

      // ---------------- scores S[block][key][row] (base-2 logits) -------------
      float Sv[C::SUB][4];
#pragma unroll
      for (int st = 0; st < C::SUB; ++st) {
        const int r0 = k0 + 16 * st + g, r1 = r0 + 8;
        float* Sx = Sv[st];
        Sx[0] = Sx[1] = Sx[2] = Sx[3] = 0.f;
        uint32_t ks0[MW], ks1[MW], kb0[MW], kb1[MW];
        meta_row<NG>(sMeta, r0, ks0);
        meta_row<NG>(sMeta, r1, ks1);
        if constexpr (!Q8) {
          meta_row<NG>(sMeta + C::META, r0, kb0);
          meta_row<NG>(sMeta + C::META, r1, kb1);
        }
        int s = 0;
#pragma unroll
        for (int G = 0; G < NG; ++G) {
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
          uint32_t w0[C::NW], w1[C::NW];
#pragma unroll
          for (int part = 0; part < (C::NW + 3) / 4; ++part) {
            constexpr int PW = C::NW < 4 ? C::NW : 4;
            lds_words<PW>(sK + koff(r0, xk0, st, G, part), w0 + part * 4);
            lds_words<PW>(sK + koff(r1, xk1, st, G, part), w1 + part * 4);
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
          const float sk0 = meta_f<NG>(ks0, G), sk1 = meta_f<NG>(ks1, G);
          const float bb0 = Q8 ? -128.f * sk0 : meta_f<NG>(kb0, G);
          const float bb1 = Q8 ? -128.f * sk1 : meta_f<NG>(kb1, G);
          const float c0 = sk0 * scaleK, c1 = sk1 * scaleK;
          Sx[0] = fmaf(c0, acc[0], fmaf(bb0, qsc[G][0], Sx[0]));
          Sx[1] = fmaf(c0, acc[1], fmaf(bb0, qsc[G][1], Sx[1]));
          Sx[2] = fmaf(c1, acc[2], fmaf(bb1, qsc[G][0], Sx[2]));
          Sx[3] = fmaf(c1, acc[3], fmaf(bb1, qsc[G][1], Sx[3]));
        }
        const int kr0 = 16 * st + k0 + g;                 // key index within the stage
        if (kvalid < TK) {                                // only a stage that reaches L
          if (kr0 >= kvalid) { Sx[0] = -INFINITY; Sx[1] = -INFINITY; }
          if (kr0 + 8 >= kvalid) { Sx[2] = -INFINITY; Sx[3] = -INFINITY; }
        }
        if (p.mask_kind != QKV_MASK_NONE) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int vh = hbase + chunk * 8 + 2 * t + j;     // row = head * Lq + query
            if (vh < p.G) {
              const int hr = vh / p.Lq, qi = vh - hr * p.Lq;
#pragma unroll
              for (int r = 0; r < 2; ++r) {
                const int64_t key = key0 + kr0 + 8 * r;
                if (key >= L) continue;
                if (p.mask_kind == QKV_MASK_CAUSAL) {
                  if (key > L - p.Lq + qi) Sx[2 * r + j] = -INFINITY;
                } else {
                  const int64_t mi = (int64_t)b * p.msb + ((int64_t)hkv * p.Gq + hr) * p.msh +
                                     (int64_t)qi * p.msq + key;
                  Sx[2 * r + j] += kLog2e * load_as_float(p.mask, p.mask_dtype, mi);
                }
              }
            }
          }
        }
      }

      // ---------------- online softmax over the warp's 32 keys -----------------
      float t0 = -INFINITY, t1 = -INFINITY;
#pragma unroll
      for (int st = 0; st < C::SUB; ++st) {
        t0 = fmaxf(t0, fmaxf(Sv[st][0], Sv[st][2]));
        t1 = fmaxf(t1, fmaxf(Sv[st][1], Sv[st][3]));
      }
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        t0 = fmaxf(t0, __shfl_xor_sync(~0u, t0, off));
        t1 = fmaxf(t1, __shfl_xor_sync(~0u, t1, off));
      }
      const float n0 = fmaxf(m0, t0), n1 = fmaxf(m1, t1);
      const float u0 = n0 == -INFINITY ? 0.f : n0, u1 = n1 == -INFINITY ? 0.f : n1;
      const float al0 = ex2(m0 - u0), al1 = ex2(m1 - u1);
      float P[C::SUB][4];
#pragma unroll
      for (int st = 0; st < C::SUB; ++st) {
        P[st][0] = ex2(Sv[st][0] - u0); P[st][1] = ex2(Sv[st][1] - u1);
        P[st][2] = ex2(Sv[st][2] - u0); P[st][3] = ex2(Sv[st][3] - u1);
      }
      m0 = n0; m1 = n1;
      float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
      for (int st = 0; st < C::SUB; ++st) { ps0 += P[st][0] + P[st][2]; ps1 += P[st][1] + P[st][3]; }
      l0 = fmaf(l0, al0, ps0);
      l1 = fmaf(l1, al1, ps1);
      if (__any_sync(~0u, (al0 != 1.f) || (al1 != 1.f))) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          O[mt][0] *= al0; O[mt][1] *= al1; O[mt][2] *= al0; O[mt][3] *= al1;
        }
#pragma unroll
        for (int G = 0; G < NG; ++G) { beta[0][G] *= al0; beta[1][G] *= al1; }
      }

      // ---------------- values --------------------------------------------------
      uint32_t vsw[C::SUB][2][MW], vbw[C::SUB][2][MW];
#pragma unroll
      for (int st = 0; st < C::SUB; ++st) {
        const int r0 = k0 + 16 * st + g;
        meta_row<NG>(sMeta + (Q8 ? 1 : 2) * C::META, r0, vsw[st][0]);
        meta_row<NG>(sMeta + (Q8 ? 1 : 2) * C::META, r0 + 8, vsw[st][1]);
        if constexpr (!Q8) {
          meta_row<NG>(sMeta + 3 * C::META, r0, vbw[st][0]);
          meta_row<NG>(sMeta + 3 * C::META, r0 + 8, vbw[st][1]);
        }
      }
#pragma unroll
      for (int G = 0; G < NG; ++G) {
        if constexpr (!Q8) {
#pragma unroll
          for (int st = 0; st < C::SUB; ++st) {
            const float vb0f = meta_f<NG>(vbw[st][0], G), vb1f = meta_f<NG>(vbw[st][1], G);
            beta[0][G] = fmaf(P[st][0], vb0f, fmaf(P[st][2], vb1f, beta[0][G]));
            beta[1][G] = fmaf(P[st][1], vb0f, fmaf(P[st][3], vb1f, beta[1][G]));
          }
        }
        const float up = exp2i(tau[G]);
#pragma unroll
        for (int st = 0; st < C::SUB; ++st) {
          const float sv0 = meta_f<NG>(vsw[st][0], G) * up, sv1 = meta_f<NG>(vsw[st][1], G) * up;
          const float x00 = P[st][0] * sv0, x01 = P[st][1] * sv0;
          const float x10 = P[st][2] * sv1, x11 = P[st][3] * sv1;
          const uint32_t top = pack_half2(x00, x01), bot = pack_half2(x10, x11);
          const uint32_t b0 = movmatrix_trans(top), b1 = movmatrix_trans(bot);
          uint32_t b0l = 0, b1l = 0;
          if constexpr (F32OUT) {
            const float2 ft = unpack_half2(top), fb = unpack_half2(bot);
            b0l = movmatrix_trans(pack_half2(x00 - ft.x, x01 - ft.y));
            b1l = movmatrix_trans(pack_half2(x10 - fb.x, x11 - fb.y));
          }
          // value codes of the block: ldmatrix .trans gives lane (g, t) one
          // 16-bit unit of keys 2t and 2t+1 (and of 2t+8, 2t+9) per register:
          // the key pairs of the A operand, one unit (4 or 2 dims) per register
          constexpr int PAIRS = VX2 ? 1 : (BITS == 4 ? GS / 64 : GS / 32);   // unit pairs per group
#pragma unroll
          for (int pr = 0; pr < PAIRS; ++pr) {
            const int lin = (vkey + 16 * st) * C::RB + G * C::GB + (2 * pr + vunit) * 16;
            const uint32_t va = smem_u32(sV) + swz_offset<C::SWZV>(lin);
            uint32_t R[4];
            if constexpr (VX2) {
              ldsm_x2_trans(va, R[0], R[2]);
              R[1] = R[0]; R[3] = R[2];
            } else {
              ldsm_x4_trans(va, R[0], R[1], R[2], R[3]);
            }
            if constexpr (Q8) {
#pragma unroll
              for (int r = 0; r < 4; ++r) R[r] ^= 0x80808080u;
            }
            constexpr int MPP = VX2 ? 2 : (BITS == 4 ? 4 : 2);       // m-tiles per pair
#pragma unroll
            for (int c = 0; c < MPP; ++c) {
              uint32_t a[4];
              if constexpr (BITS == 4) {
                // nibble c of each unit (x2: nibbles c and c + 2 for the two row halves)
                const int clo = c, chi = VX2 ? c + 2 : c;
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                  const int cc = (r & 1) ? chi : clo;
                  const uint32_t y = (cc >= 2) ? (R[r] >> 8) : R[r];
                  a[r] = y & ((cc & 1) ? 0x00F000F0u : 0x000F000Fu);
                }
              } else {
#pragma unroll
                for (int r = 0; r < 4; ++r) a[r] = (c ? (R[r] >> 8) : R[r]) & 0x00FF00FFu;
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
              const int mt = G * KPG + pr * MPP + c;
              mma_f16(O[mt], a, b0, b1, O[mt]);
              if constexpr (F32OUT) mma_f16(O[mt], a, b0l, b1l, O[mt]);
            }
          }
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
      // rows g / g+8 of value m-tile i of group G (the ldmatrix unit layout):
      //  4-bit, groups >= 64: unit pair i/4, nibble c = i%4 -> dims 64(i/4)+4g+c, +32
      //  4-bit, groups of 32: nibble c = i -> dims 4g+c and 4g+c+2
      //  8-bit: unit pair i/2, byte c = i%2 -> dims 32(i/2)+2g+c, +16
      int dlo, dhi;
      bool x16 = false;                          // odd nibbles carry code * 2^-20
      if constexpr (BITS == 4 && GS == 32) {
        dlo = G * GS + 4 * g + i; dhi = dlo + 2; x16 = (i & 1) != 0;
      } else if constexpr (BITS == 4) {
        dlo = G * GS + 64 * (i >> 2) + 4 * g + (i & 3); dhi = dlo + 32; x16 = (i & 1) != 0;
      } else {
        dlo = G * GS + 32 * (i >> 1) + 2 * g + (i & 1); dhi = dlo + 16;
      }
      // codes entered as code*2^-24 (Q8_0: exact codes); O of group G carries 2^tau
      const float f = exp2i((Q8 ? 0 : (x16 ? 20 : 24)) - tau[G]);
      ws[(2 * t) * D + dlo] = fmaf(O[mt][0], f, beta[0][G]);
      ws[(2 * t + 1) * D + dlo] = fmaf(O[mt][1], f, beta[1][G]);
      ws[(2 * t) * D + dhi] = fmaf(O[mt][2], f, beta[0][G]);
      ws[(2 * t + 1) * D + dhi] = fmaf(O[mt][3], f, beta[1][G]);
    }
    if (g == 0) {
      ws[8 * D + 2 * t] = m0; ws[8 * D + 2 * t + 1] = m1;
      ws[8 * D + 8 + 2 * t] = l0; ws[8 * D + 8 + 2 * t + 1] = l1;
    }
    __syncthreads();

    const bool complete = (s0 == 0) && (s1 == (int)S);
    const int64_t slot = 2 * (int64_t)blockIdx.x + (u == first_unit ? 0 : 1);
    const float* wsf = reinterpret_cast<const float*>(smem);
    for (int idx = tid; idx < HPC * D; idx += C::NTHR) {
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
      // The unit's partials are merged by the last of its CTAs to finish
      // (atomic ticket), in one level when their volume is small, else in two:
      // the last CTA of each group of kMergeGroup consecutive CTAs merges the
      // group into a second-level partial and the last group merger merges
      // those.  Nobody waits on anybody.
      __threadfence();
      __syncthreads();
      const int64_t cfirst = udiv64((u * S + 1) * nC - 1, T);
      const int64_t clast = udiv64(((u + 1) * S) * nC - 1, T);
      const int nparts = (int)(clast - cfirst + 1);
      const int nrows = min(HPC, p.G - hbase);
      // slot of the unit's first CTA: its second slot if it began in an
      // earlier unit; every later CTA of the unit began in this one
      const int64_t slot0 = 2 * cfirst + (udiv64(udiv64(cfirst * T, nC), S) == u ? 0 : 1);
      auto slot_of = [&](int64_t c) -> int64_t { return c == cfirst ? slot0 : 2 * c; };
      const int64_t out_base = (((int64_t)b * p.Hkv + hkv) * p.G + hbase) * D;
      if ((int64_t)nparts * nrows * D <= kMergeFlat) {
        if (tid == 0) {
          const unsigned prev = atomicAdd(&p.tickets[u], 1u);
          const int last = prev == (unsigned)nparts - 1;
          if (last) p.tickets[u] = 0u;
          s_flag = last;
        }
        __syncthreads();
        if (s_flag) {
          __threadfence();
          merge_unit<D, HPC>(p.part_ml, p.part_o, nparts, slot0, cfirst, 1, tid, C::NTHR, nrows,
                             p.out, p.out_dtype, out_base, nullptr, nullptr);
        }
      } else {
        const int ngroups = (nparts + kMergeGroup - 1) / kMergeGroup;
        const int gi = (int)((int64_t)blockIdx.x - cfirst) / kMergeGroup;
        const int64_t c0 = cfirst + (int64_t)gi * kMergeGroup;
        const int64_t lead = slot_of(c0);                       // the group's second-level slot
        const int gsz = min(kMergeGroup, nparts - gi * kMergeGroup);
        if (tid == 0) {
          const unsigned prev = atomicAdd(&p.tickets1[lead], 1u);
          const int last = prev == (unsigned)gsz - 1;
          if (last) p.tickets1[lead] = 0u;
          s_flag = last;
        }
        __syncthreads();
        if (s_flag) {
          __threadfence();
          merge_unit<D, HPC>(p.part_ml, p.part_o, gsz, lead, c0, 1, tid, C::NTHR, nrows,
                             nullptr, 0, 0, p.part2_ml + lead * HPC * 2, p.part2_o + lead * HPC * D);
          __threadfence();
          __syncthreads();
          if (tid == 0) {
            const unsigned prev = atomicAdd(&p.tickets[u], 1u);
            const int last = prev == (unsigned)ngroups - 1;
            if (last) p.tickets[u] = 0u;
            s_flag = last;
          }
          __syncthreads();
          if (s_flag) {
            __threadfence();
            merge_unit<D, HPC>(p.part2_ml, p.part2_o, ngroups, slot0, cfirst, kMergeGroup, tid,
                               C::NTHR, nrows, p.out, p.out_dtype, out_base, nullptr, nullptr);
          }
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
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, C::NTHR, C::SMEM) != cudaSuccess)
        return 0;
      cached = n;
    }
    return cached;
  }
  static cudaError_t launch(const DecodePlan& plan, const DecodeParams& p, cudaStream_t s) {
    auto k = qsdpa_decode_kernel<D, BITS, GS, Q8, NC, F32OUT>;
    k<<<plan.grid, C::NTHR, C::SMEM, s>>>(p);
    return cudaGetLastError();
  }
};

}  // namespace qkv
