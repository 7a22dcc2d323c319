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
//  * Work: units (batch, kv-head, chunk-group of <=32 query heads) x blocks
//    of BK (16 or 32) keys, flattened and cut evenly over one CTA per SM.  A
//    CTA touches at most two units partially; a partial result (running max
//    m, sum l, unnormalized o) goes to workspace and a second kernel
//    (decode_merge.cuh) merges the partials of split units (log-sum-exp
//    rescaling).  Both are programmatic dependent launches: a kernel's
//    set-up overlaps the previous kernel of the stream.
//  * Teams: the warps of a CTA form teams (one warp per 8-row head chunk).
//    A team streams its own blocks -- handed out in order through a shared
//    counter, so fast teams take more -- with 16-byte cp.async (zero-filled
//    past L) into its own NSTAGE-deep shared-memory ring and meets only its
//    own warps; there is no CTA-wide barrier until the epilogue.  Code tiles
//    are XOR-swizzled per 128-byte line so both fragment read patterns below
//    are bank-conflict-free.
//  * Scores: one m16n8k16 tensor op per 16 keys x 8 query heads x 16 dims.
//    Codes enter the tensor core EXACTLY as fp16 subnormals (a mask of the
//    packed word leaves code*2^-24 or code*2^-20); the query is prescaled by a
//    power of two (and by 1/16 for the 2^-20 positions).  The per-group key
//    scale and the bias term (bias * sum of q over the group, the identity the
//    Metal kernel uses with its query_sum) are applied in fp32 afterwards.
//    Q8_0 codes are offset by 128 (xor 0x80) and corrected the same way.
//  * Online softmax in base 2 with warp shuffles over the block's keys.
//  * Values: O^T[e,h] += V^T[e,j] (P[j,h]*s_v[j]*2^tau): V codes are the A
//    operand (transposing ldmatrix loads hand every lane a key pair per
//    register), the probabilities times the per-key value scale are the B
//    operand, moved from the score fragment layout with movmatrix.trans.
//    tau (per warp and group, lowered when a larger value scale appears, with
//    an exact power-of-two rescale of O) keeps the fp16 operand below 2^15.
//    The value bias term sum_j P[j,h]*b_v[j] is accumulated in fp32.  With
//    fp32 output the B operand is split into fp16 hi + lo parts (two tensor
//    ops).
#pragma once

#include "qkv_common.cuh"
#include "qkv_internal.h"
#include "quantize_core.cuh"

namespace qkv {

// 16 warps per CTA for D <= 128, 8 for D = 256 (about 250 registers per
// thread); one CTA per SM.  The warps form teams of NC, one warp per 8-row head
// chunk; every team streams its own blocks of keys through its own
// shared-memory ring, so the main loop has no CTA-wide barrier and warps that
// are ahead never wait for warps that are behind.
__host__ __device__ constexpr int dec_warps(int D) { return D <= 128 ? 16 : 8; }
constexpr int kDecWarpsMax = 16;
__host__ __device__ constexpr int dec_ctas_per_sm(int) { return 1; }

// XOR coefficients (3 bits each, for line bits 0..3) of the 16-byte-unit
// swizzle inside each 128-byte line of a staged code tile, found by exhaustive
// search so that the K-fragment and V-fragment read patterns are free of bank
// conflicts for every supported (D, bits, group size).
__host__ __device__ constexpr uint32_t swz_pack(int c0, int c1, int c2, int c3) {
  return (uint32_t)(c0 | (c1 << 3) | (c2 << 6) | (c3 << 9));
}
__host__ __device__ constexpr uint32_t swizzle_coeffs(int D, int bits, int gs) {
  return bits == 2 ? (D == 64 ? swz_pack(0, 0, 0, 0) : D == 128 ? swz_pack(1, 0, 0, 0)
                      : (gs == 64 ? swz_pack(2, 1, 0, 0) : swz_pack(2, 0, 0, 0)))
       : D == 64 ? (bits == 4 ? (gs == 32 ? swz_pack(1, 0, 0, 0) : swz_pack(2, 0, 0, 0))
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

// Swizzled offset of byte offset `lin` (lin with its unit bits XORed by the
// pattern of its line); linear over XOR of offsets.
template <uint32_t SWZ>
__host__ __device__ __forceinline__ constexpr int swz_xor(int lin) {
  return lin ^ swz_line<SWZ>((lin >> 7) & 15);
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

// SB: the width of the codes as stored in the cache.  BITS (2, 4 or 8) is the
// width the fragment code computes with (2: groups of 64 or 128 only, one or
// two whole words per lane and row); SB != BITS (affine 2-bit codes in groups
// of 32 and 3-bit codes, computed as 4-bit; 5 or 6-bit codes, computed as
// 8-bit) stages each block's
// packed rows as they are (one little-endian bit stream per row; rows
// straddle 16-byte units) and the team transcodes them into a tile of its own
// before the block's math.
template <int D, int BITS, int GS, bool Q8, int NC, int SB = BITS>
struct DecCfg {
  static constexpr bool XC = SB != BITS;       // transcoded from SB-bit codes
  static constexpr int RB = D * BITS / 8;      // bytes per code row (compute width)
  static constexpr int RBS = D * SB / 8;       // bytes per code row as stored
  static constexpr int UPR = RB / 16;          // 16-byte units per row
  static constexpr int NG = D / GS;            // groups per row
  static constexpr int GB = GS * BITS / 8;     // bytes per group per row
  static constexpr int NW = GS * BITS / 128;   // K-fragment words per thread per (row, group)
  static constexpr int KPG = GS / 16;          // k-steps per group == V m-tiles per group
  static constexpr int KSTEPS = D / 16;
  static constexpr int MT = D / 16;
  static constexpr int NMETA = Q8 ? 2 : 4;
  static constexpr int MROW = NG * 2;          // meta bytes per key per array
  static constexpr int NWARP = dec_warps(D);
  static constexpr int NTHR = 32 * NWARP;
  static constexpr int NTEAM = NWARP / NC;     // teams; each has one warp per head chunk
  static constexpr int TTHR = 32 * NC;         // threads per team
  static constexpr int WPC = NTEAM;            // warps per head chunk
  static constexpr int QROW = 2 * D + 4;       // staged query row: raw 16-bit values + 4 bytes of padding
  static constexpr int QSB = ((NC * 8 * QROW + 127) / 128) * 128;
  // dynamic shared memory of the one CTA of an SM (227 KB less static data)
  static constexpr int BUDGET = 227 * 1024 - 2048;
  static constexpr int r16(int x) { return (x + 15) / 16 * 16; }
  static constexpr int r128(int x) { return (x + 127) / 128 * 128; }
  // staged codes of one tile (K or V): the compute tile, or the packed rows
  static constexpr int scodes(int sub) { return XC ? r16(16 * sub * RBS) : 16 * sub * RB; }
  static constexpr int stage_bytes(int sub) { return r128(2 * scodes(sub) + NMETA * r16(16 * sub * MROW)); }
  // a team's K and V compute tiles (transcoded blocks only)
  static constexpr int xtile_bytes(int sub) { return XC ? 2 * 16 * sub * RB : 0; }
  // 16-key sub-blocks per block: two when three such stages per team fit
  // (D = 256 keeps one: its register budget is spent)
  // fused update: the new token's raw K and V rows (16-bit inputs)
  static constexpr int NEWB = 4 * D;
  static constexpr int SUB = (D <= 128 && NTEAM * (3 * stage_bytes(2) + xtile_bytes(2)) + QSB + NEWB <= BUDGET) ? 2 : 1;
  static constexpr int BK = 16 * SUB;          // keys per block
  static constexpr int TK = BK;
  static constexpr int CODES = BK * RB;        // one compute tile
  static constexpr int SCODES = scodes(SUB);   // one staged tile
  static constexpr int MOFF = 2 * SCODES;      // metadata arrays in a stage
  static constexpr int KUS = SCODES / 16;      // 16-byte units of a staged packed tile
  static constexpr int XT = xtile_bytes(SUB);
  static constexpr int META = r16(BK * MROW);
  static constexpr int META_UNITS = BK * MROW / 16;
  static constexpr int KU = BK * UPR;          // 16-byte code units per tile
  static constexpr int MU = NMETA * META_UNITS;
  static constexpr int STAGE = stage_bytes(SUB);
  static constexpr int NS_FIT = (BUDGET - QSB - NEWB - NTEAM * XT) / (NTEAM * STAGE);
  static constexpr int NSTAGE = NS_FIT > 6 ? 6 : NS_FIT;
  static constexpr int XTOFF = NSTAGE * STAGE;          // the team's compute tiles after its ring
  static constexpr int TRING = NSTAGE * STAGE + XT;     // one team's region
  static constexpr int QOFF = NTEAM * TRING;            // query rows after the rings
  // epilogue (after every ring is drained): per-warp partial rows, then the
  // per-(row, warp) combine weights and per-row (m, l)
  static constexpr int WSW = 8 * D + 16;               // floats per warp
  static constexpr int EPI_W = NWARP * WSW * 4;
  static constexpr int EPI = EPI_W + NC * 8 * (NTEAM + 1) * 4 + NC * 8 * 2 * 4;
  static constexpr int NEWOFF = QOFF + QSB;
  static constexpr int SMEM = NEWOFF + NEWB > EPI ? NEWOFF + NEWB : EPI;
  // three stages per team (two for transcoded blocks, whose compute tiles take
  // the room of the third: the copy of the next block still overlaps the
  // math of the current one)
  static_assert(NSTAGE >= (XC ? 2 : 3), "stages per team");
  static_assert(SMEM <= BUDGET, "shared memory budget");
  static_assert(META_UNITS * 16 == BK * MROW, "metadata rows must fill 16-byte units");
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

// Fused update, by one warp of the team that got the block of key L - 1:
// quantize the new token's K and V rows (raw 16-bit values staged at s_new)
// with the quantizer's arithmetic -- lanes [0, D/32) take K's 32-element
// slices, the next D/32 lanes V's -- write codes and metadata to cache row
// crow and into row r of the staged block at sb.  Out of line: it runs once
// per unit and keeps its registers out of the main loop.
template <int D, int BITS, int GS, bool Q8>
__device__ __noinline__ void fused_quantize_patch(const DecodeParams& p, const uint8_t* s_new,
                                                  uint8_t* sb, int64_t crow, int r, int lane) {
  using C = DecCfg<D, BITS, GS, Q8, 1>;
  constexpr int NG = C::NG;
  constexpr int SL = D / kQEpt;
  constexpr int OW = kQEpt * BITS / 32;                // code words of a slice
  const bool isv = lane >= SL, act = lane < 2 * SL;
  const int cs = isv ? lane - SL : lane;
  uint32_t w[kQWords];
#pragma unroll
  for (int k = 0; k < kQWords / 4; ++k) {
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (act) v = *reinterpret_cast<const uint4*>(s_new + isv * 2 * D + cs * 64 + k * 16);
    w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
  }
  uint32_t o[OW];
  uint16_t sbits, bbits;
  if (p.new_bf16) quantize_slice<GS, BITS, Q8, true>(w, o, sbits, bbits);
  else quantize_slice<GS, BITS, Q8, false>(w, o, sbits, bbits);
  if (!act) return;
  uint32_t* codes = const_cast<uint32_t*>(reinterpret_cast<const uint32_t*>(isv ? p.vc : p.kc));
  uint4* dst = reinterpret_cast<uint4*>(codes + crow * (C::RB / 4) + cs * OW);
#pragma unroll
  for (int k = 0; k < OW / 4; ++k) {
    const uint4 v = make_uint4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
    dst[k] = v;
    // the slice's 16-byte units in the staged (swizzled) row
    const int lin = r * C::RB + cs * OW * 4 + k * 16;
    *reinterpret_cast<uint4*>(sb + (isv ? C::CODES + swz_xor<C::SWZV>(lin) : swz_xor<C::SWZ>(lin))) = v;
  }
  if ((cs * kQEpt) % GS == 0) {
    // metadata arrays in stage order: affine K scales, K biases, V scales, V
    // biases; Q8_0 K scales, V scales
    const int gq = (cs * kQEpt) / GS;
    uint16_t* sc = const_cast<uint16_t*>(isv ? p.vs : p.ks);
    sc[crow * NG + gq] = sbits;
    reinterpret_cast<uint16_t*>(sb + 2 * C::CODES + (Q8 ? isv : 2 * isv) * C::META)[r * NG + gq] = sbits;
    if constexpr (!Q8) {
      uint16_t* bi = const_cast<uint16_t*>(isv ? p.vb : p.kb);
      bi[crow * NG + gq] = bbits;
      reinterpret_cast<uint16_t*>(sb + 2 * C::CODES + (2 * isv + 1) * C::META)[r * NG + gq] = bbits;
    }
  }
}

// Additive-mask values of a lane's row for the keys 16 st + 8 r (relative to
// m) of one block, st < SUB, r < 2; keys at or past nk read nothing (0).  No
// branch around the loads, so they are in flight together.
template <int SUB, typename T>
__device__ __forceinline__ void dec_mask_vals(const T* m, int nk, float (&mv)[SUB][2]) {
#pragma unroll
  for (int st = 0; st < SUB; ++st)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int k = 16 * st + 8 * r;
      mv[st][r] = k < nk ? to_float_ld(m + k) : 0.f;
    }
}

// Masks of the field-spreading step below: N codes form blocks of 2H codes,
// block b starting at bit 2 H b BITS, each block's codes still packed SB bits
// apart; LO selects every block's lower H codes, HI its upper H codes.
__host__ __device__ constexpr uint32_t spread_mask(int N, int H, int SB, int BITS, bool hi) {
  uint32_t m = 0u;
  for (int b = 0; b < N / (2 * H); ++b)
    for (int i = hi ? H * SB : 0; i < (hi ? 2 * H * SB : H * SB); ++i) m |= 1u << (2 * H * b * BITS + i);
  return m;
}

// N codes of SB bits packed from bit 0 -> the same codes BITS bits apart
// (BITS > SB): halving steps, each moving the upper half of every block up
// into the zero gap above it (two ANDs, a shift and an OR per step).
template <int N, int SB, int BITS, int H = N / 2>
__device__ __forceinline__ uint32_t spread_codes(uint32_t f) {
  if constexpr (H == 0) {
    return f;
  } else {
    constexpr uint32_t LO = spread_mask(N, H, SB, BITS, false), HI = spread_mask(N, H, SB, BITS, true);
    return spread_codes<N, SB, BITS, H / 2>((f & LO) | ((f & HI) << (H * (BITS - SB))));
  }
}

// A team's transcode of one staged block of SB-bit codes (K rows, then V
// rows SCODES bytes later; each row one little-endian bit stream, element e
// at bits [e SB, (e + 1) SB)) into its K and V tiles of BITS-bit codes at xt
// (4-bit for 2- and 3-bit codes, 8-bit for 5- and 6-bit ones), laid out and
// swizzled exactly as staged codes of that width are.  A thread takes one
// 16-byte unit of the tile: U = 128 / BITS codes, whose U SB stream bits
// start at a word boundary (at bit 16 of a word for odd units of 5-bit
// codes); each output word is one field of 32 / BITS codes, spread.  Reads
// stay inside the stage (the V rows and the metadata follow the K rows; the
// metadata follow the V rows).
template <class C, int D, int SB, int BITS>
__device__ __forceinline__ void transcode_block(const uint8_t* raw, uint8_t* xt, int ttid) {
  constexpr int U = 128 / BITS;                    // codes per 16-byte unit of the tile
  constexpr int F = 32 / BITS;                     // codes per output word
  constexpr int UPR = C::RB / 16;                  // units per row
  constexpr int ITEMS = 2 * C::BK * UPR;
  constexpr bool ALIGNED = (U * SB) % 32 == 0;     // every unit starts at a word
  constexpr int NIN = ALIGNED ? U * SB / 32 : (U * SB + 16 + 31) / 32;   // input words read
  constexpr uint32_t FMASK = F * SB == 32 ? ~0u : (1u << (F * SB)) - 1u;
  static_assert((D * SB) % 32 == 0, "rows start at a word");
  static_assert(ALIGNED || SB == 5, "unaligned units only for 5-bit codes (offset 0 or 16)");
  const uint32_t* rw = reinterpret_cast<const uint32_t*>(raw);
#pragma unroll 2
  for (int it = ttid; it < ITEMS; it += C::TTHR) {
    const int which = it >= C::BK * UPR;
    const int rem = which ? it - C::BK * UPR : it;
    const int r = rem / UPR, j = rem - r * UPR;
    const int p0 = (r * D + U * j) * SB;           // stream bit of the unit's first code
    const uint32_t* src = rw + which * (C::SCODES / 4) + (p0 >> 5);
    uint32_t w[NIN + 1];
#pragma unroll
    for (int k = 0; k < NIN; ++k) w[k] = src[k];
    w[NIN] = 0u;
    if constexpr (!ALIGNED) {
      const int sh = p0 & 31;                      // 0 or 16
#pragma unroll
      for (int k = 0; k < NIN; ++k) w[k] = __funnelshift_r(w[k], w[k + 1], sh);
    }
    uint32_t out[4];
#pragma unroll
    for (int o = 0; o < 4; ++o) {
      constexpr int FB = F * SB;                   // field bits
      const int bit = o * FB, wi = bit >> 5, sh = bit & 31;
      const uint32_t f = (sh == 0 ? w[wi] : __funnelshift_r(w[wi], w[wi + 1], sh)) & FMASK;
      out[o] = spread_codes<F, SB, BITS>(f);
    }
    const int lin = r * C::RB + 16 * j;
    *reinterpret_cast<uint4*>(xt + (which ? C::CODES + swz_xor<C::SWZV>(lin) : swz_xor<C::SWZ>(lin))) =
        make_uint4(out[0], out[1], out[2], out[3]);
  }
}

template <int D, int BITS, int GS, bool Q8, int NC, bool F32OUT, int VAR, int SB = BITS>
__global__ void __launch_bounds__(32 * dec_warps(D), 1)
qsdpa_decode_kernel(const __grid_constant__ DecodeParams p) {
  constexpr bool FUSED = VAR == kDecFused;     // also quantizes the new token into row L - 1
  constexpr bool EXT = VAR == kDecExt;         // logit softcap, mask slopes, sinks
  constexpr bool ADDMASK = VAR != kDecPlain;   // additive masks (plain: none, or causal)
  using C = DecCfg<D, BITS, GS, Q8, NC, SB>;
  static_assert(!C::XC || (!Q8 && VAR == kDecPlain && ((BITS == 4 && SB < 4) || (BITS == 8 && SB > 4 && SB < 8))),
                "2- and 3-bit codes compute as 4-bit, 5- and 6-bit codes as 8-bit");
  static_assert(BITS != 2 || (!Q8 && VAR == kDecPlain && GS >= 64),
                "2-bit fragments: affine codes in groups of 64 or 128, plain variant");
  constexpr int NG = C::NG, KPG = C::KPG, MT = C::MT, BK = C::BK, NSTAGE = C::NSTAGE;
  constexpr int NTEAM = C::NTEAM, TTHR = C::TTHR;
  constexpr int HPC = NC * 8;
  constexpr int MW = NG == 1 ? 1 : NG / 2;     // 32-bit words of one key's metadata row
  extern __shared__ __align__(128) uint8_t smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int team = warp / NC, chunk = warp - team * NC;
  const int ttid = tid - team * TTHR;          // thread index within the team
  uint8_t* const ring = smem + team * C::TRING;
  uint8_t* const qst = smem + C::QOFF;
  const int64_t S = p.stages_per_unit, T = p.total_stages;   // blocks of BK keys
  const int64_t nC = gridDim.x;
  const int64_t lo = udiv64((int64_t)blockIdx.x * T, nC), hi = udiv64(((int64_t)blockIdx.x + 1) * T, nC);
  const int64_t first_unit = udiv64(lo, S);
  __shared__ int s_next;                 // next block of the segment to hand out
  __shared__ int s_grab[NTEAM][2];       // a team's next block, double-buffered

  // The launch's parameters sit in constant-bank lines that no SM has cached
  // yet: touch every line from a different warp so that the misses overlap
  // instead of following each other through the first instructions.
  if (lane == 0 && warp * 64 < (int)sizeof(DecodeParams)) {
    const uint32_t v = reinterpret_cast<const uint32_t*>(&p)[warp * 16];
    asm volatile("" :: "r"(v));
  }
  if (tid == 0) s_next = NTEAM * (NSTAGE - 1);
  __syncthreads();

  // the threads of one team meet here (one warp: a warp barrier)
  auto team_sync = [&]() {
    if constexpr (NC == 1) __syncwarp();
    else asm volatile("bar.sync %0, %1;\n" :: "r"(1 + team), "n"(TTHR) : "memory");
  };

  // A CTA's range [lo, hi) of (unit, block) pairs is walked as segments, one
  // per unit it touches; the teams share a segment's blocks through s_next.
  for (int64_t x = lo; x < hi;) {
    const int64_t u = udiv64(x, S);
    const int s0 = (int)(x - u * S);
    const int s1 = (int)(min(hi, (u + 1) * S) - u * S);
    x = u * S + s1;
    const int nblk = s1 - s0;

    const int64_t uh = udiv64(u, p.ncg);                 // (batch, kv head)
    const int cg = (int)(u - uh * p.ncg);
    const int b = (int)udiv64(uh, p.Hkv);
    const int hkv = (int)(uh - (int64_t)b * p.Hkv);
    const int64_t row0 = ((int64_t)b * p.Hkv + hkv) * p.Lcap;   // first cache row of this head
    const int hbase = cg * HPC;                                  // first local row of the CTA

    const int64_t L = p.L;
    // Fused update: the segment that holds the unit's last block (key L - 1,
    // the new token) has the team that gets that block fetch the new K and V
    // rows with the block's copies, quantize them with the quantizer's own
    // arithmetic, write them to the cache and patch its staged copy of the row
    // (which may predate that write); see fused_quantize_patch.
    const bool newtok = FUSED && s1 == (int)S;
    uint8_t* const s_new = smem + C::NEWOFF;

    // Copy plan of one block (by its team): 16-byte unit i is row i / UPR of
    // the K tile (i < KU) or of the V tile, then the metadata arrays.  Unit
    // ttid + k * TTHR of a tile lies in line (ttid / 8) + k * TTHR / 8, and
    // the swizzle is linear in the line bits, so it splits into a per-thread
    // part and a per-k constant.
    const int fx = swz_line<C::SWZ>((ttid >> 3) & 15);
    const int fxv = swz_line<C::SWZV>((ttid >> 3) & 15);
    // a lane's metadata unit when every lane copies at most one: unit ttid is
    // 16-byte unit ttid % META_UNITS of array ttid / META_UNITS (lanes past
    // the last unit copy nothing)
    const uint8_t* mlane;
    {
      const int marr = ttid / C::META_UNITS, mj16 = (ttid - marr * C::META_UNITS) * 16;
      const uint16_t* arr = Q8 ? (marr == 0 ? p.ks : p.vs)
                               : (marr == 0 ? p.ks : marr == 1 ? p.kb : marr == 2 ? p.vs : p.vb);
      mlane = reinterpret_cast<const uint8_t*>(arr) + mj16;
    }
    auto issue_block = [&](int blk, int slot) {
      const uint32_t sbase = smem_u32(ring + slot * C::STAGE);
      const int64_t key0 = (int64_t)(s0 + blk) * BK;
      const int nvalid = (int)(L - key0 < (int64_t)BK ? L - key0 : (int64_t)BK);
      // global addresses are formed from the launch parameters each time
      // (constant operands) rather than kept live across the loop
      const int64_t grow = row0 + key0;                        // cache row of the block's first key
      const uint8_t* kb0 = p.kc + grow * C::RB;
      const uint8_t* vb0 = p.vc + grow * C::RB;
      if constexpr (C::XC) {
        // packed rows as they are, flat: a 16-byte unit that holds a byte of
        // a valid row is copied whole (its tail lies below the next multiple
        // of 8 rows, inside the cache); later units are zero-filled
        const uint8_t* ks0 = p.kc + grow * C::RBS;
        const uint8_t* vs0 = p.vc + grow * C::RBS;
        const int vbytes = nvalid * C::RBS;
        constexpr int NU = (2 * C::KUS + TTHR - 1) / TTHR;
#pragma unroll
        for (int k = 0; k < NU; ++k) {
          const int i = ttid + k * TTHR;
          if ((2 * C::KUS) % TTHR == 0 || i < 2 * C::KUS) {
            const int which = i >= C::KUS, j = which ? i - C::KUS : i;
            const bool ok = j * 16 < vbytes;
            cp_async16(sbase + which * C::SCODES + j * 16, (which ? vs0 : ks0) + (ok ? j * 16 : 0),
                       ok ? 16 : 0);
          }
        }
      } else if (C::KU % TTHR == 0 && nvalid == BK) {
        const uint8_t* ks = kb0 + ttid * 16;
        const uint8_t* vs = vb0 + ttid * 16;
        const uint32_t dk = sbase + ((ttid * 16) ^ fx);
        const uint32_t dv = sbase + C::CODES + ((ttid * 16) ^ fxv);
#pragma unroll
        for (int k = 0; k < C::KU / TTHR; ++k) {
          const int kx = swz_line<C::SWZ>((k * TTHR / 8) & 15);
          const int kxv = swz_line<C::SWZV>((k * TTHR / 8) & 15);
          cp_async16((dk ^ kx) + k * TTHR * 16, ks + k * TTHR * 16, 16);
          cp_async16((dv ^ kxv) + k * TTHR * 16, vs + k * TTHR * 16, 16);
        }
      } else {
        constexpr int NU = (2 * C::KU + TTHR - 1) / TTHR;
#pragma unroll
        for (int k = 0; k < NU; ++k) {
          const int i = ttid + k * TTHR;
          if ((2 * C::KU) % TTHR == 0 || i < 2 * C::KU) {
            const int which = i >= C::KU, j = which ? i - C::KU : i;
            const bool ok = (j / C::UPR) < nvalid;
            const uint8_t* src = (which ? vb0 : kb0) + (ok ? j * 16 : 0);
            const int dst = which ? C::CODES + swz_offset<C::SWZV>(j * 16) : swz_offset<C::SWZ>(j * 16);
            cp_async16(sbase + dst, src, ok ? 16 : 0);
          }
        }
      }
      // metadata: affine K scales, K biases, V scales, V biases; Q8_0 K and V scales
      if constexpr (FUSED) {
        if (newtok && blk == nblk - 1) {
          // the new token's raw K and V rows (D 16-bit values each), 4D bytes
          for (int i = ttid; i < D / 4; i += TTHR) {
            const int isv = i >= D / 8, j = isv ? i - D / 8 : i;
            cp_async16(smem_u32(s_new) + i * 16,
                       reinterpret_cast<const uint8_t*>((isv ? p.new_v : p.new_k) + uh * D) + j * 16, 16);
          }
        }
      }
      if constexpr (C::MU <= TTHR) {
        // one unit per lane: its array and offset were chosen once (mlane)
        if (C::MU == TTHR || ttid < C::MU) {
          const int marr = ttid / C::META_UNITS, mj16 = (ttid - marr * C::META_UNITS) * 16;
          const bool ok = mj16 / C::MROW < nvalid;
          cp_async16(sbase + C::MOFF + marr * C::META + mj16,
                     mlane + grow * C::MROW - (ok ? 0 : mj16), ok ? 16 : 0);
        }
        return;
      }
#pragma unroll
      for (int k = 0; k < (C::MU + TTHR - 1) / TTHR; ++k) {
        const int i = ttid + k * TTHR;
        if (C::MU % TTHR == 0 || i < C::MU) {
          const int arr = i / C::META_UNITS, j = i - arr * C::META_UNITS;
          const uint16_t* gm = Q8 ? (arr == 0 ? p.ks : p.vs)
                                  : (arr == 0 ? p.ks : arr == 1 ? p.kb : arr == 2 ? p.vs : p.vb);
          const bool ok = (j * 16) / C::MROW < nvalid;
          const uint8_t* src = reinterpret_cast<const uint8_t*>(gm + grow * NG) + (ok ? j * 16 : 0);
          cp_async16(sbase + C::MOFF + arr * C::META + j * 16, src, ok ? 16 : 0);
        }
      }
    };

    // Fragment offsets inside a tile.  A fragment address is a per-lane part
    // plus a compile-time part (sub-block, group, unit) whose bits do not
    // overlap, so the sum is an XOR, and the swizzle is linear over XOR: the
    // swizzled offset is the swizzled lane part XOR the swizzled constant.
    //  key fragments: row g (or g + 8) of the sub-block, the lane's words t
    const int kl0 = swz_xor<C::SWZ>(g * C::RB + t * C::NW * 4);
    const int kl1 = swz_xor<C::SWZ>((g + 8) * C::RB + t * C::NW * 4);
    auto kconst = [](int st, int G, int part) {
      return swz_xor<C::SWZ>(st * 16 * C::RB + G * C::GB + part * 16);
    };
    //  value fragments: ldmatrix rows.  Lane l addresses row l % 8 of matrix
    //  l / 8; matrices 0/1 hold keys 0-7, 2/3 keys 8-15 of the 16-key block,
    //  and matrices 0/2 the first, 1/3 the second 16-byte unit of a unit pair
    //  (x2 loads for 4-bit groups of 32: matrix 0 keys 0-7, matrix 1 keys 8-15).
    // (x2 loads: a group of one 16-byte unit -- 4-bit codes in groups of 32,
    // 2-bit codes in groups of 64)
    constexpr bool VX2 = (BITS == 4 && GS == 32) || (BITS == 2 && GS == 64);
    const int vkey = (lane & 7) + (VX2 ? ((lane >> 3) & 1) * 8 : ((lane >> 4) & 1) * 8);
    const int vunit = VX2 ? 0 : ((lane >> 3) & 1);
    const int vl = swz_xor<C::SWZV>(vkey * C::RB + vunit * 16);

    // ---------------- prologue ----------------------------------------------
    // The query rows go out first, then every team's first NSTAGE-1 blocks,
    // so that the small loads do not queue behind the copies.  The rows are
    // staged as raw 16-bit values in rows padded by 4 bytes, which keeps the
    // fragment reads below free of bank conflicts.
    constexpr int QCH = HPC * D / 8;                      // 16-byte query chunks
    constexpr int QPT = (QCH + C::NTHR - 1) / C::NTHR;
    // Everything above touched only parameters and shared memory; inputs are
    // read, and the workspace written, only once the previous kernel of the
    // stream has completed (this launch may start early, overlapping its
    // set-up with that kernel's tail).  Before waiting, one lane per team
    // asks L2 for the team's first blocks (a prefetch reads no data into the
    // CTA and L2 stays coherent with writes of the previous kernel, so it is
    // safe to issue early): their copies then start from L2.
    if (lane == 0 && chunk == 0) {
#pragma unroll
      for (int i = 0; i < NSTAGE - 1; ++i) {
        const int blk = team + NTEAM * i;
        if (blk >= nblk) break;
        const int64_t key0 = (int64_t)(s0 + blk) * BK;
        const int rows = (int)(p.Lcap - key0 < (int64_t)BK ? p.Lcap - key0 : (int64_t)BK);   // inside the cache
        const int64_t grow = row0 + key0;
        prefetch_l2_bulk(p.kc + grow * C::RBS, (uint32_t)(rows * C::RBS + 15) & ~15u);
        prefetch_l2_bulk(p.vc + grow * C::RBS, (uint32_t)(rows * C::RBS + 15) & ~15u);
      }
    }
    grid_dep_wait();
    uint4 qraw[QPT];
    {
      const int64_t qbase = (uh * p.G + hbase) * D;
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
      const int blk = team + NTEAM * i;
      if (blk < nblk) issue_block(blk, i);
      cp_async_commit();
    }
#pragma unroll
    for (int k = 0; k < QPT; ++k) {
      const int i = tid + k * C::NTHR;
      if (QCH % C::NTHR == 0 || i < QCH) {
        const int hl = i / (D / 8), c = i - hl * (D / 8);
        uint32_t* dst = reinterpret_cast<uint32_t*>(qst + hl * C::QROW + c * 16);
        dst[0] = qraw[k].x; dst[1] = qraw[k].y; dst[2] = qraw[k].z; dst[3] = qraw[k].w;
      }
    }
    __syncthreads();
    if (ttid == 0) s_grab[team][0] = atomicAdd(&s_next, 1);

    // ---------------- query fragments (B operand of the score MMA) ----------
    uint32_t bq[C::KSTEPS][2];
    float qsc[NG][2];
    float scaleK;
    {
      const uint16_t* qr = reinterpret_cast<const uint16_t*>(qst + (chunk * 8 + g) * C::QROW);
      const bool qf16 = p.q_dtype == QKV_F16;
      float qs[NG];
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) qs[gg] = 0.f;
      float qmax = 0.f;
      float qv[C::KSTEPS][4];
#pragma unroll
      for (int s = 0; s < C::KSTEPS; ++s) {
        const int G = s / KPG, ks = s % KPG;
        int e[4];
        if constexpr (BITS == 2) {
          // word m of the lane's words, code positions (2j, 2j+8) and
          // (2j+1, 2j+9) (after a shift by 8 for j >= 2)
          const int m = ks >> 2, j = ks & 3;
          const int e0 = G * GS + (t * C::NW + m) * 16 + 2 * j;
          e[0] = e0; e[1] = e0 + 8; e[2] = e0 + 1; e[3] = e0 + 9;
        } else if constexpr (BITS == 4) {
          const int m = ks >> 1, hi2 = (ks & 1) * 2;
          const int e0 = G * GS + (t * C::NW + m) * 8 + hi2;
          e[0] = e0; e[1] = e0 + 4; e[2] = e0 + 1; e[3] = e0 + 5;
        } else {
          const int e0 = G * GS + (t * C::NW + ks) * 4;
          e[0] = e0; e[1] = e0 + 2; e[2] = e0 + 1; e[3] = e0 + 3;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint16_t h = qr[e[i]];
          qv[s][i] = qf16 ? __half2float(__ushort_as_half(h)) : __uint_as_float((uint32_t)h << 16);
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
        // the query at a code position that the masked word holds 2^k times
        // too large carries 2^-k: 4-bit, odd nibbles x16; 2-bit, positions
        // 2j, 2j+1 of a byte pair x4^(2j mod 4), x4^(2j+1 mod 4)
        float sc1 = qscale, sc2 = BITS == 4 ? qscale16 : qscale;
        if constexpr (BITS == 2) {
          const bool odd = ((s % KPG) & 1) != 0;
          sc1 = odd ? exp2i(sigma - 4) : qscale;
          sc2 = odd ? exp2i(sigma - 6) : exp2i(sigma - 2);
        }
        bq[s][0] = pack_half2(qv[s][0] * sc1, qv[s][1] * sc1);
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
    // Per group, the value operand carries 2^tau, with tau = 21 - the largest
    // exponent field of the group's value scales seen so far, so that
    // P * s_v * 2^tau < 2^15 for every key (P <= 2^8, the lazy max below).  vbound holds those
    // largest scales (magnitudes, as fp16 bits, two groups per word); tau
    // only decreases, and O is rescaled by the exact power of two when it does.
    int tau[NG];
    uint32_t vbound[MW];
#pragma unroll
    for (int gg = 0; gg < NG; ++gg) { beta[0][gg] = 0.f; beta[1][gg] = 0.f; tau[gg] = 21; }
#pragma unroll
    for (int w = 0; w < MW; ++w) vbound[w] = 0u;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) { O[mt][0] = O[mt][1] = O[mt][2] = O[mt][3] = 0.f; }


    // ---------------- main loop: the team's blocks ---------------------------
    // pend[] holds the blocks in flight, oldest first; blocks are handed out in
    // increasing order, so once a team sees a block past the segment it has
    // nothing left.
    int pend[NSTAGE - 1];
#pragma unroll
    for (int i = 0; i < NSTAGE - 1; ++i) pend[i] = team + NTEAM * i;
    int slot = 0;
    for (int it = 0; pend[0] < nblk; ++it) {
      cp_async_wait<NSTAGE - 2>();
      team_sync();
      const int cur = pend[0];
      uint8_t* sb = ring + slot * C::STAGE;
      {
        // the slot read in the previous iteration takes the next block
        const int nb = s_grab[team][it & 1];
        if (ttid == 0) s_grab[team][(it + 1) & 1] = atomicAdd(&s_next, 1);
        if (nb < nblk) issue_block(nb, slot == 0 ? NSTAGE - 1 : slot - 1);
        cp_async_commit();
#pragma unroll
        for (int i = 0; i < NSTAGE - 2; ++i) pend[i] = pend[i + 1];
        pend[NSTAGE - 2] = nb;
        slot = slot + 1 == NSTAGE ? 0 : slot + 1;
      }
      const int64_t key0 = (int64_t)(s0 + cur) * BK;
      const int kvalid = (int)(L - key0 < (int64_t)BK ? L - key0 : (int64_t)BK);   // valid keys of this block
      if constexpr (FUSED) {
        if (newtok && key0 + kvalid == L) {
          if (chunk == 0)
            fused_quantize_patch<D, BITS, GS, Q8>(p, s_new, sb, row0 + L - 1, kvalid - 1, lane);
          team_sync();
        }
      }
      const uint8_t* sK = sb;
      const uint8_t* sV = sb + C::CODES;
      const uint8_t* sMeta = sb + C::MOFF;
      if constexpr (C::XC) {
        // the team's warps are past the previous block (team_sync above), so
        // its compute tiles are free
        uint8_t* xt = ring + C::XTOFF;
        transcode_block<C, D, SB, BITS>(sb, xt, ttid);
        team_sync();
        sK = xt;
        sV = xt + C::CODES;
      }

      // ---------------- scores S[block][key][row] (base-2 logits) -------------
      float Sv[C::SUB][4];
#pragma unroll
      for (int st = 0; st < C::SUB; ++st) {
        const int r0 = 16 * st + g, r1 = r0 + 8;
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
            lds_words<PW>(sK + (kl0 ^ kconst(st, G, part)), w0 + part * 4);
            lds_words<PW>(sK + (kl1 ^ kconst(st, G, part)), w1 + part * 4);
          }
#pragma unroll
          for (int m = 0; m < C::NW; ++m) {
            if constexpr (BITS == 2) {
              // 16 codes per word: masks leave code * 4^k * 2^-24 (k = 0..3)
              // in each half, exact fp16 subnormals; the shifted word gives
              // the upper 8 positions of each half
#pragma unroll
              for (int hb = 0; hb < 2; ++hb) {
                const uint32_t y0 = hb ? w0[m] >> 8 : w0[m], y1 = hb ? w1[m] >> 8 : w1[m];
                uint32_t a[4] = {y0 & 0x00030003u, y1 & 0x00030003u, y0 & 0x000C000Cu, y1 & 0x000C000Cu};
                mma_f16(acc, a, bq[s][0], bq[s][1], acc);
                ++s;
                uint32_t a2[4] = {y0 & 0x00300030u, y1 & 0x00300030u, y0 & 0x00C000C0u, y1 & 0x00C000C0u};
                mma_f16(acc, a2, bq[s][0], bq[s][1], acc);
                ++s;
              }
            } else if constexpr (BITS == 4) {
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
        if (EXT && p.cap_a > 0.f) {                       // logit softcap (before the mask)
#pragma unroll
          for (int i = 0; i < 4; ++i) Sx[i] = softcap_log2(Sx[i], p.cap_a, p.cap_k);
        }
        const int kr0 = 16 * st + g;                      // key index within the block
        if (kvalid < BK) {                                // only a block that reaches L
          if (kr0 >= kvalid) { Sx[0] = -INFINITY; Sx[1] = -INFINITY; }
          if (kr0 + 8 >= kvalid) { Sx[2] = -INFINITY; Sx[3] = -INFINITY; }
        }
      }
      if (p.mask_kind != QKV_MASK_NONE) {
        // the lane's rows 2t, 2t+1 of its chunk against keys 16 st + g (+ 8):
        // per row one division, then the block's mask values read together
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int vh = hbase + chunk * 8 + 2 * t + j;         // row = head * Lq + query
          const bool rv = vh < p.G;
          const int hr = rv ? vh / p.Lq : 0, qi = rv ? vh - hr * p.Lq : 0;
          // the plain variant is never launched with an additive mask
          if (!ADDMASK || p.mask_kind == QKV_MASK_CAUSAL) {
            const int64_t last = L - p.Lq + qi - key0 - g;      // last visible key, block-relative
#pragma unroll
            for (int st = 0; st < C::SUB; ++st) {
              if (16 * st > last) Sv[st][j] = -INFINITY;
              if (16 * st + 8 > last) Sv[st][2 + j] = -INFINITY;
            }
          } else if constexpr (ADDMASK) {
            const float slope = kLog2e * (EXT && p.slopes != nullptr && rv
                                              ? p.slopes[hkv * p.Gq + hr] : 1.f);
            const int64_t mrow = (int64_t)b * p.msb + ((int64_t)hkv * p.Gq + hr) * p.msh +
                                 (int64_t)qi * p.msq + key0 + g;
            const int nk = rv ? (int)(L - key0 - g < (int64_t)BK ? L - key0 - g : (int64_t)BK) : 0;
            float mv[C::SUB][2];
            if (p.mask_dtype == QKV_F32)
              dec_mask_vals<C::SUB>(reinterpret_cast<const float*>(p.mask) + mrow, nk, mv);
            else if (p.mask_dtype == QKV_F16)
              dec_mask_vals<C::SUB>(reinterpret_cast<const __half*>(p.mask) + mrow, nk, mv);
            else
              dec_mask_vals<C::SUB>(reinterpret_cast<const __nv_bfloat16*>(p.mask) + mrow, nk, mv);
#pragma unroll
            for (int st = 0; st < C::SUB; ++st)
#pragma unroll
              for (int r = 0; r < 2; ++r) {
                float& x = Sv[st][2 * r + j];
                x = mv[st][r] == -INFINITY ? -INFINITY : fmaf(slope, mv[st][r], x);
              }
          }
        }
      }

      // ---------------- online softmax over the warp's keys ---------------------
      // The running max moves lazily: only when a score exceeds it by more
      // than 8 (base 2) does the warp agree on a new per-row max and rescale;
      // otherwise P = 2^(S - m) <= 2^8, which tau leaves room for.
      float t0 = -INFINITY, t1 = -INFINITY;
#pragma unroll
      for (int st = 0; st < C::SUB; ++st) {
        t0 = fmaxf(t0, fmaxf(Sv[st][0], Sv[st][2]));
        t1 = fmaxf(t1, fmaxf(Sv[st][1], Sv[st][3]));
      }
      if (__any_sync(~0u, (t0 > m0 + 8.f) || (t1 > m1 + 8.f))) {
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          t0 = fmaxf(t0, __shfl_xor_sync(~0u, t0, off));
          t1 = fmaxf(t1, __shfl_xor_sync(~0u, t1, off));
        }
        const float n0 = fmaxf(m0, t0), n1 = fmaxf(m1, t1);
        const float al0 = ex2(m0 - (n0 == -INFINITY ? 0.f : n0));
        const float al1 = ex2(m1 - (n1 == -INFINITY ? 0.f : n1));
        m0 = n0; m1 = n1;
        l0 *= al0; l1 *= al1;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          O[mt][0] *= al0; O[mt][1] *= al1; O[mt][2] *= al0; O[mt][3] *= al1;
        }
#pragma unroll
        for (int G = 0; G < NG; ++G) { beta[0][G] *= al0; beta[1][G] *= al1; }
      }
      const float u0 = m0 == -INFINITY ? 0.f : m0, u1 = m1 == -INFINITY ? 0.f : m1;
      float P[C::SUB][4];
#pragma unroll
      for (int st = 0; st < C::SUB; ++st) {
        P[st][0] = ex2(Sv[st][0] - u0); P[st][1] = ex2(Sv[st][1] - u1);
        P[st][2] = ex2(Sv[st][2] - u0); P[st][3] = ex2(Sv[st][3] - u1);
      }
      float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
      for (int st = 0; st < C::SUB; ++st) { ps0 += P[st][0] + P[st][2]; ps1 += P[st][1] + P[st][3]; }
      l0 += ps0;
      l1 += ps1;

      // ---------------- values --------------------------------------------------
      uint32_t vsw[C::SUB][2][MW], vbw[C::SUB][2][MW];
#pragma unroll
      for (int st = 0; st < C::SUB; ++st) {
        const int r0 = 16 * st + g;
        meta_row<NG>(sMeta + (Q8 ? 1 : 2) * C::META, r0, vsw[st][0]);
        meta_row<NG>(sMeta + (Q8 ? 1 : 2) * C::META, r0 + 8, vsw[st][1]);
        if constexpr (!Q8) {
          meta_row<NG>(sMeta + 3 * C::META, r0, vbw[st][0]);
          meta_row<NG>(sMeta + 3 * C::META, r0 + 8, vbw[st][1]);
        }
        if (kvalid < BK) {
          // keys past L: a metadata unit that starts below L is copied whole
#pragma unroll
          for (int w = 0; w < MW; ++w) {
            if (r0 >= kvalid) { vsw[st][0][w] = 0u; vbw[st][0][w] = 0u; }
            if (r0 + 8 >= kvalid) { vsw[st][1][w] = 0u; vbw[st][1][w] = 0u; }
          }
        }
      }
      {
        // largest value scale of the block per group (fp16 bits of non-negative
        // magnitudes order like the values); a rare warp-wide step when it
        // exceeds the bound
        uint32_t vm[MW];
        bool grow = false;
#pragma unroll
        for (int w = 0; w < MW; ++w) {
          vm[w] = __vmaxu2(vsw[0][0][w] & 0x7fff7fffu, vsw[0][1][w] & 0x7fff7fffu);
#pragma unroll
          for (int st = 1; st < C::SUB; ++st)
            vm[w] = __vmaxu2(vm[w], __vmaxu2(vsw[st][0][w] & 0x7fff7fffu, vsw[st][1][w] & 0x7fff7fffu));
          grow |= __vmaxu2(vm[w], vbound[w]) != vbound[w];
        }
        if (__any_sync(~0u, grow)) {
#pragma unroll
          for (int w = 0; w < MW; ++w) {
            vm[w] = __vmaxu2(vm[w], vbound[w]);
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) vm[w] = __vmaxu2(vm[w], __shfl_xor_sync(~0u, vm[w], off));
            vbound[w] = vm[w];
          }
#pragma unroll
          for (int G = 0; G < NG; ++G) {
            const int e = (int)((vbound[G >> 1] >> (16 * (G & 1) + 10)) & 31);
            const int nt = 21 - e;
            if (nt < tau[G]) {
              const float f = exp2i(nt - tau[G]);
#pragma unroll
              for (int i = 0; i < KPG; ++i) {
                O[G * KPG + i][0] *= f; O[G * KPG + i][1] *= f;
                O[G * KPG + i][2] *= f; O[G * KPG + i][3] *= f;
              }
              tau[G] = nt;
            }
          }
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
          constexpr int PAIRS = VX2 ? 1 : (BITS == 2 ? GS / 128 : BITS == 4 ? GS / 64 : GS / 32);   // unit pairs per group
#pragma unroll
          for (int pr = 0; pr < PAIRS; ++pr) {
            const uint32_t va = smem_u32(sV) + (vl ^ swz_xor<C::SWZV>(16 * st * C::RB + G * C::GB + 2 * pr * 16));
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
            constexpr int MPP = BITS == 2 ? (VX2 ? 4 : 8) : VX2 ? 2 : (BITS == 4 ? 4 : 2);   // m-tiles per pair
#pragma unroll
            for (int c = 0; c < MPP; ++c) {
              uint32_t a[4];
              if constexpr (BITS == 2) {
                // code position k of each 16-bit unit: mask 3 << 2k leaves
                // code * 4^k * 2^-24 (k = c mod 4), the upper positions after
                // a shift by 8 (x2: the second row half; x4: m-tiles 4..7)
                constexpr uint32_t kM[4] = {0x00030003u, 0x000C000Cu, 0x00300030u, 0x00C000C0u};
                const uint32_t msk = kM[c & 3];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                  const bool up = VX2 ? (r & 1) != 0 : c >= 4;
                  a[r] = (up ? (R[r] >> 8) : R[r]) & msk;
                }
              } else if constexpr (BITS == 4) {
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
    cp_async_wait<0>();          // only empty groups can still be pending
    __syncthreads();             // every team is done with its ring
    grid_dep_launch();           // the next kernel may start its set-up

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
    // Per warp, its accumulators in fragment order (one float4 per m-tile and
    // lane, stores free of bank conflicts), then (m, l) of its 8 rows.
    float* ws = reinterpret_cast<float*>(smem) + warp * C::WSW;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int G = mt / KPG, i = mt % KPG;
      // codes entered as code*2^-24 (odd nibbles: code*2^-20; Q8_0: exact
      // codes); O of group G carries 2^tau
      const bool x16 = BITS == 4 && (i & 1) != 0;
      // 2-bit: m-tile i holds code position i mod 4 of its units, x4^(i mod 4)
      const int x4 = BITS == 2 ? 2 * (i & 3) : 0;
      const float f = exp2i((Q8 ? 0 : (x16 ? 20 : 24 - x4)) - tau[G]);
      reinterpret_cast<float4*>(ws)[mt * 32 + lane] =
          make_float4(fmaf(O[mt][0], f, beta[0][G]), fmaf(O[mt][1], f, beta[1][G]),
                      fmaf(O[mt][2], f, beta[0][G]), fmaf(O[mt][3], f, beta[1][G]));
    }
    if (g == 0) {
      ws[8 * D + 2 * t] = m0; ws[8 * D + 2 * t + 1] = m1;
      ws[8 * D + 8 + 2 * t] = l0; ws[8 * D + 8 + 2 * t + 1] = l1;
    }
    __syncthreads();

    const bool complete = (s0 == 0) && (s1 == (int)S);
    const float* wsf = reinterpret_cast<const float*>(smem);
    constexpr int WST = NTEAM + 1;                               // padded weight row
    float* wgt = reinterpret_cast<float*>(smem + C::EPI_W);     // [HPC][WST] combine weights
    float* rml = wgt + HPC * WST;                                // [HPC][2] (m, l) of the CTA
    // weights: thread (row R, team k) of the first HPC * NTEAM threads; the
    // NTEAM teams of a row are adjacent lanes
    if (tid < HPC * NTEAM) {
      const int R = tid / NTEAM, k = tid - R * NTEAM;
      const int c = R >> 3, hh = R & 7;
      const float* wp = wsf + (k * NC + c) * C::WSW;
      const float mw = wp[8 * D + hh], lw = wp[8 * D + 8 + hh];
      float M = mw;
#pragma unroll
      for (int off = 1; off < NTEAM; off <<= 1) M = fmaxf(M, __shfl_xor_sync(~0u, M, off));
      const float w = mw == -INFINITY ? 0.f : ex2(mw - M);
      float Ls = w * lw;
#pragma unroll
      for (int off = 1; off < NTEAM; off <<= 1) Ls += __shfl_xor_sync(~0u, Ls, off);
      float wk = w;
      if (complete) {
        // a CTA that covered its whole unit normalizes here; the head's sink
        // logit (if any) joins the denominator (a split unit's sink is added
        // by the merge, once)
        float Lt = Ls;
        if (EXT && p.sinks != nullptr && hbase + R < p.G) {
          const float s2 = kLog2e * p.sinks[hkv * p.Gq + (hbase + R) / p.Lq];
          const float Mn = fmaxf(M, s2);
          if (Mn != -INFINITY) {
            const float f = M == -INFINITY ? 0.f : ex2(M - Mn);
            Lt = Ls * f + ex2(s2 - Mn);
            wk = w * f;
          }
        }
        wk = (Ls > 0.f && Lt > 0.f) ? wk / Lt : 0.f;
      }
      wgt[R * WST + k] = wk;
      if (k == 0) { rml[2 * R] = M; rml[2 * R + 1] = Ls; }
    }
    __syncthreads();
    const int64_t pslot = 2 * (int64_t)blockIdx.x + (u == first_unit ? 0 : 1);
    // element (chunk c, m-tile mt, lane (gl, tl), j) of the fragment order is
    // row c*8 + 2*tl + (j & 1) and the dim of m-tile mt's row gl (j < 2) or
    // gl + 8 (j >= 2):
    //  4-bit, groups >= 64: unit pair i/4, nibble i%4 -> dims 64(i/4)+4g+i%4, +32
    //  4-bit, groups of 32: nibble i -> dims 4g+i and 4g+i+2
    //  8-bit: unit pair i/2, byte i%2 -> dims 32(i/2)+2g+i%2, +16
    // A thread takes 4 consecutive elements (j = 0..3 of one lane's m-tile):
    // rows R0 = c*8 + 2*tl and R0 + 1, dims dim and dim + dj; one float4 read
    // per team and four independent sums.
    for (int q4 = tid; q4 < HPC * D / 4; q4 += C::NTHR) {
      const int idx = 4 * q4;
      const int c = idx / (8 * D), r = idx - c * 8 * D;
      const int mt = r >> 7, lj = r & 127, gl = lj >> 4, tl = (lj >> 2) & 3;
      const int R0 = c * 8 + 2 * tl;
      const int head = hbase + R0;
      if (head >= p.G) continue;
      const bool v1 = head + 1 < p.G;
      const int G = mt / KPG, i = mt % KPG;
      int dim, dj;
      if constexpr (BITS == 2 && GS == 64) { dim = G * GS + 8 * gl + i; dj = 4; }
      else if constexpr (BITS == 2) { dim = G * GS + 8 * gl + i; dj = 64; }
      else if constexpr (BITS == 4 && GS == 32) { dim = G * GS + 4 * gl + i; dj = 2; }
      else if constexpr (BITS == 4) { dim = G * GS + 64 * (i >> 2) + 4 * gl + (i & 3); dj = 32; }
      else { dim = G * GS + 32 * (i >> 1) + 2 * gl + (i & 1); dj = 16; }
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < NTEAM; ++k) {
        const float4 x = *reinterpret_cast<const float4*>(wsf + (k * NC + c) * C::WSW + r);
        const float w0 = wgt[R0 * WST + k], w1 = wgt[(R0 + 1) * WST + k];
        o.x = fmaf(w0, x.x, o.x); o.y = fmaf(w1, x.y, o.y);
        o.z = fmaf(w0, x.z, o.z); o.w = fmaf(w1, x.w, o.w);
      }
      if (complete) {
        const int64_t oi = (uh * p.G + head) * D + dim;
        store_from_float(p.out, p.out_dtype, oi, o.x);
        store_from_float(p.out, p.out_dtype, oi + dj, o.z);
        if (v1) {
          store_from_float(p.out, p.out_dtype, oi + D, o.y);
          store_from_float(p.out, p.out_dtype, oi + D + dj, o.w);
        }
      } else {
        float* po = p.part_o + (pslot * HPC + R0) * D + dim;
        po[0] = o.x; po[dj] = o.z;
        if (v1) { po[D] = o.y; po[D + dj] = o.w; }
        if (dim == 0) {
          float* pm = p.part_ml + (pslot * HPC + R0) * 2;
          pm[0] = rml[2 * R0]; pm[1] = rml[2 * R0 + 1];
          if (v1) { pm[2] = rml[2 * R0 + 2]; pm[3] = rml[2 * R0 + 3]; }
        }
      }
    }
    if (tid == 0) s_next = NTEAM * (NSTAGE - 1);                 // for the next segment
    __syncthreads();             // the next segment reuses the shared memory
  }

}

}  // namespace qkv
