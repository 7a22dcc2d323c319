// kview.cu -- attention whose values are a view of the keys: K rows of
// Dk = 576 elements in one quantized cache, V = the first Dv = 512 elements of
// every K row (the MLA shape of the llama.cpp PR's follow-up tests, "576/512
// MLA", whose dequantization skips V when V is a view of K; llama.cpp #25556,
// merged follow-up).  One cache stream serves both operands: each block of
// keys is dequantized once.
//
//   out[b, h, i, :] = softmax_j(q[b, h, i] * scale . Khat[b, h / G, j] (+ causal))
//                     . Khat[b, h / G, j, :Dv]
//
// Work: units = (batch, kv head, tile of 64 (head, query) rows, row = head *
// Lq + query), each split over `pieces` CTAs along L in blocks of 64 keys.
// A CTA (16 warps):
//  * stages the packed K rows and their scales (and biases) of the next block
//    by cp.async into one raw slot while it computes on the current one; all
//    threads dequantize a block once into an fp16 tile [64 keys][576] (rows
//    padded by 16 bytes, so the fragment loads below are free of bank
//    conflicts): fp16(scale*code+bias), one rounding, as the tcgen05 prefill
//    dequantizes its tiles;
//  * S^T[key][row] = K q^T on the m16n8k16 tensor op: warp w takes keys
//    16 (w % 4) .. +16 and rows 16 (w / 4) .. +16 over the 36 k-steps (four
//    independent accumulator chains), K from the tile (ldmatrix), q from an
//    fp16 tile prescaled per row by a power of two (exact for normal values);
//  * the block maximum of each row (shuffles, then across the 4 key warps in
//    shared memory) moves the running maximum; P = 2^(S - m) in fp16 goes to a
//    [row][key] tile;
//  * O^T[dim][row] += V^T P: warp w owns dims 32 w .. +32 of all 64 rows, V^T
//    read from the same K tile with the transposing ldmatrix (the view costs
//    nothing), after rescaling its accumulators by the rows' factors.
// One dequantized block thus serves 64 rows (all 64 heads of a kv head's
// tile), and the tensor ops of both products run 16 and 8 independent chains
// per warp.  A CTA that covered its whole unit writes the normalized output;
// otherwise (m, l, O) go to the workspace in the split-K decode's partial
// layout and the decode's merge kernel (decode_merge.cuh, 512-wide rows)
// folds them.
#include <algorithm>

#include "decode_merge.cuh"

namespace qkv {

namespace {

constexpr int kKvDk = 576, kKvDv = 512;
constexpr int kKvBN = 64;                       // keys per block
constexpr int kKvRows = 64;                     // (head, query) rows per CTA
constexpr int kKvWarps = 16;
constexpr int kKvThreads = 32 * kKvWarps;
constexpr int kKvRowBytes = kKvDk * 2 + 16;     // padded fp16 row of the K and q tiles
constexpr int kKvPRowBytes = kKvBN * 2 + 16;    // padded fp16 row of the P tile
constexpr int kKvMaxGrid = 160;                 // CTAs whose partials the workspace holds (two slots each)

template <bool Q8, int BITS, int GS>
struct KvCfg {
  static constexpr int RB = kKvDk * BITS / 8;   // packed bytes per key
  static constexpr int NG = kKvDk / GS;         // groups per key
  static constexpr int CODES = kKvBN * RB;      // packed codes of a block
  static constexpr int META = kKvBN * NG * 2;   // one metadata array of a block
  static constexpr int NMETA = Q8 ? 1 : 2;      // scales (and biases)
  static constexpr int RAW = (CODES + NMETA * META + 127) / 128 * 128;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + kKvRows * kKvRowBytes;
  static constexpr int P_OFF = K_OFF + kKvBN * kKvRowBytes;
  static constexpr int RED_OFF = P_OFF + kKvRows * kKvPRowBytes;      // [4][64] floats
  static constexpr int STAT_OFF = RED_OFF + 4 * kKvRows * 4;          // rowscale, m, alpha: [3][64]
  static constexpr int RAW_OFF = (STAT_OFF + 3 * kKvRows * 4 + 127) / 128 * 128;
  static constexpr int SMEM = RAW_OFF + RAW;    // one raw slot: the next block lands during the math
  static constexpr int CPR = RB / 16;            // 16-byte code chunks per key
  static_assert(CODES % 16 == 0 && META % 16 == 0, "whole 16-byte units");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];\n"
               : "=r"(r0), "=r"(r1) : "r"(addr) : "memory");
}

// One 16-byte chunk of packed codes (16 8-bit or 32 4-bit codes of key row
// `key`, all in one group) -> fp16 scale * code + bias at dims e0 .. of the
// tile row, in natural order.
template <bool Q8, int BITS>
__device__ __forceinline__ void kv_convert(uint4 w4, __half2 s2, __half2 b2, uint8_t* row, int e0) {
  const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
  const __half2 off = __float2half2_rn(Q8 ? 1152.f : 1024.f);   // Q8_0 codes enter as code + 128
  constexpr int N = BITS == 8 ? 16 : 32;
  uint32_t o[N / 2];
#pragma unroll
  for (int k = 0; k < N / 2; ++k) {
    uint32_t c0, c1;
    if constexpr (BITS == 8) {
      const uint32_t x = Q8 ? (wv[k >> 1] ^ 0x80808080u) : wv[k >> 1];
      c0 = (x >> (16 * (k & 1))) & 0xffu;
      c1 = (x >> (16 * (k & 1) + 8)) & 0xffu;
    } else {
      c0 = (wv[k >> 2] >> (8 * (k & 3))) & 0xfu;
      c1 = (wv[k >> 2] >> (8 * (k & 3) + 4)) & 0xfu;
    }
    const uint32_t h = (c0 | (c1 << 16)) | 0x64006400u;              // 1024 + code, exact
    const __half2 v = __hfma2(__hsub2(*reinterpret_cast<const __half2*>(&h), off), s2, b2);
    o[k] = *reinterpret_cast<const uint32_t*>(&v);
  }
#pragma unroll
  for (int k = 0; k < N / 8; ++k)
    *reinterpret_cast<uint4*>(row + (e0 + 8 * k) * 2) = make_uint4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
}

template <bool Q8, int BITS, int GS>
__global__ void __launch_bounds__(kKvThreads, 1) qsdpa_kview_kernel(const __grid_constant__ DecodeParams p) {
  using C = KvCfg<Q8, BITS, GS>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  uint8_t* const qt = smem + C::Q_OFF;
  uint8_t* const kt = smem + C::K_OFF;
  uint8_t* const pt = smem + C::P_OFF;
  uint8_t* const raw = smem + C::RAW_OFF;
  float* const red = reinterpret_cast<float*>(smem + C::RED_OFF);     // [4 key warps][64 rows]
  float* const rsc = reinterpret_cast<float*>(smem + C::STAT_OFF);    // per-row logit scale
  float* const rm = rsc + kKvRows;                                    // running maximum
  float* const ral = rm + kKvRows;                                    // this block's factor

  // this CTA's unit and blocks: units x pieces CTAs, piece k of unit u
  const int64_t S = p.stages_per_unit;
  const int64_t u = blockIdx.x / p.pieces;
  const int piece = (int)(blockIdx.x - u * p.pieces);
  const int64_t blo = S * piece / p.pieces, bhi = S * (piece + 1) / p.pieces;
  const int64_t uh = u / p.ncg;                          // (batch, kv head)
  const int cg = (int)(u - uh * p.ncg);
  const int b = (int)(uh / p.Hkv), hkv = (int)(uh - (int64_t)b * p.Hkv);
  const int64_t row0 = uh * p.Lcap;                      // first cache row of this head
  const int rbase = cg * kKvRows;                        // first (head, query) row of the tile
  const int64_t L = p.L;

  auto issue = [&](int64_t blk) {
    const int64_t key0 = blk * kKvBN;
    const int nvalid = (int)min((int64_t)kKvBN, L - key0);
    const uint32_t dst = smem_u32(raw);
    const uint8_t* src = p.kc + (row0 + key0) * C::RB;
    const int cbytes = nvalid * C::RB, mbytes = nvalid * C::NG * 2;
    for (int i = tid; i < C::CODES / 16; i += kKvThreads) {
      const bool ok = i * 16 < cbytes;
      cp_async16(dst + i * 16, src + (ok ? i * 16 : 0), ok ? 16 : 0);
    }
    // metadata rows straddle 16-byte units: a unit holding a byte of a valid
    // row is copied whole (its tail stays below the next multiple of 8 rows,
    // inside the cache); rows past L get scale 0 in the conversion anyway
    for (int i = tid; i < C::NMETA * C::META / 16; i += kKvThreads) {
      const int arr = i / (C::META / 16), j = i - arr * (C::META / 16);
      const bool ok = j * 16 < mbytes;
      const uint16_t* m = arr == 0 ? p.ks : p.kb;
      cp_async16(dst + C::CODES + arr * C::META + j * 16,
                 reinterpret_cast<const uint8_t*>(m + (row0 + key0) * C::NG) + (ok ? j * 16 : 0),
                 ok ? 16 : 0);
    }
  };

  grid_dep_wait();
  if (blo < bhi) issue(blo);
  cp_async_commit();

  // q rows -> fp16, each row prescaled by a power of two so that its largest
  // magnitude lies in [2^14, 2^15) (exact for normal values); the logit scale
  // of row r becomes scale log2(e) 2^-sigma_r.  8 threads per row.
  {
    constexpr int TPR = kKvThreads / kKvRows;           // threads per row
    const int r = tid / TPR, sub = tid % TPR;
    const int row = rbase + r;
    const bool ok = row < p.G;
    const int hl = ok ? row / p.Lq : 0, qi = ok ? row - hl * p.Lq : 0;
    const uint16_t* qr = reinterpret_cast<const uint16_t*>(p.q) +
                         (((int64_t)b * p.Hq + (int64_t)hkv * p.Gq + hl) * p.Lq + qi) * kKvDk;
    float mx = 0.f;
    for (int e = sub * 2; e < kKvDk; e += 2 * TPR) {
      const uint32_t w = ok ? *reinterpret_cast<const uint32_t*>(qr + e) : 0u;
      const float a = p.q_dtype == QKV_F16 ? half_bits_to_float((uint16_t)(w & 0xffff)) : __uint_as_float(w << 16);
      const float c = p.q_dtype == QKV_F16 ? half_bits_to_float((uint16_t)(w >> 16)) : __uint_as_float(w & 0xffff0000u);
      mx = fmaxf(mx, fmaxf(fabsf(a), fabsf(c)));
    }
#pragma unroll
    for (int off = 1; off < TPR; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(~0u, mx, off));
    int sigma = mx > 0.f ? 14 - (int)(((__float_as_uint(mx) >> 23) & 0xff) - 127) : 0;
    sigma = max(-96, min(96, sigma));
    const float up = exp2i(sigma);
    for (int e = sub * 2; e < kKvDk; e += 2 * TPR) {
      const uint32_t w = ok ? *reinterpret_cast<const uint32_t*>(qr + e) : 0u;
      const float a = p.q_dtype == QKV_F16 ? half_bits_to_float((uint16_t)(w & 0xffff)) : __uint_as_float(w << 16);
      const float c = p.q_dtype == QKV_F16 ? half_bits_to_float((uint16_t)(w >> 16)) : __uint_as_float(w & 0xffff0000u);
      *reinterpret_cast<uint32_t*>(qt + r * kKvRowBytes + e * 2) = pack_half2(a * up, c * up);
    }
    if (sub == 0) {
      rsc[r] = p.scale_log2e * exp2i(-sigma);
      rm[r] = -INFINITY;
    }
  }

  // running state: the O^T fragments of dims 32 warp .. +32 (2 m-tiles) of
  // all 8 row n-tiles; the row sums l (kept by threads 0..63)
  float O[2][8][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) O[mt][nt][0] = O[mt][nt][1] = O[mt][nt][2] = O[mt][nt][3] = 0.f;
  float lsum = 0.f;                                      // row tid (tid < 64)
  const int km = warp & 3, rn = warp >> 2;               // score tile: keys 16 km, rows 16 rn
  const uint32_t qbase = smem_u32(qt), kbase = smem_u32(kt), pbase = smem_u32(pt);

  for (int64_t blk = blo; blk < bhi; ++blk) {
    const int64_t key0 = blk * kKvBN;
    const int nvalid = (int)min((int64_t)kKvBN, L - key0);
    cp_async_wait<0>();
    __syncthreads();                                     // block landed; last block's tiles are free
    // ---- dequantize the block into the fp16 K tile --------------------------
    {
      const uint16_t* sc = reinterpret_cast<const uint16_t*>(raw + C::CODES);
      const uint16_t* bi = reinterpret_cast<const uint16_t*>(raw + C::CODES + C::META);
      for (int i = tid; i < kKvBN * C::CPR; i += kKvThreads) {
        const int key = i / C::CPR, ch = i - key * C::CPR;
        const int e0 = ch * (128 / BITS), grp = e0 / GS;
        const bool live = key < nvalid;
        const __half2 s2 = __half2half2(__ushort_as_half(live ? sc[key * C::NG + grp] : (uint16_t)0));
        const __half2 b2 = Q8 ? __float2half2_rn(0.f)
                              : __half2half2(__ushort_as_half(live ? bi[key * C::NG + grp] : (uint16_t)0));
        kv_convert<Q8, BITS>(*reinterpret_cast<const uint4*>(raw + i * 16), s2, b2,
                             kt + key * kKvRowBytes, e0);
      }
    }
    __syncthreads();                                     // tile written; raw slot free
    if (blk + 1 < bhi) issue(blk + 1);                   // lands during this block's math
    cp_async_commit();

    // ---- scores of keys 16 km .. +16, rows 16 rn .. +16 ----------------------
    // two n-tiles of 8 rows, even and odd k-steps in separate accumulators
    float s[2][2][4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) s[h][nt][0] = s[h][nt][1] = s[h][nt][2] = s[h][nt][3] = 0.f;
    {
      const uint32_t aaddr = kbase + (16 * km + (lane & 15)) * kKvRowBytes + 8 * (lane >> 4) * 2;
      const uint32_t baddr = qbase + (16 * rn + 8 * (lane >> 4) + (lane & 7)) * kKvRowBytes +
                             8 * ((lane >> 3) & 1) * 2;
#pragma unroll 6
      for (int ks = 0; ks < kKvDk / 16; ks += 2) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t a[4], bq[4];
          ldsm_x4(aaddr + (ks + h) * 32, a);
          ldsm_x4(baddr + (ks + h) * 32, bq);
          mma_f16(s[h][0], a, bq[0], bq[1], s[h][0]);
          mma_f16(s[h][1], a, bq[2], bq[3], s[h][1]);
        }
      }
    }
    // base-2 logits; keys past L, and past each row's causal limit, are -inf.
    // lg[nt][i]: key 16 km + g + 8 (i >> 1), row 16 rn + 8 nt + 2 t + (i & 1)
    float lg[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = 16 * rn + 8 * nt + 2 * t + (i & 1);
        const int key = 16 * km + g + 8 * (i >> 1);
        bool vis = key < nvalid;
        if (p.mask_kind == QKV_MASK_CAUSAL) {
          const int row = rbase + r;
          const int qi = row - (row / p.Lq) * p.Lq;
          vis = vis && key0 + key <= L - p.Lq + qi;
        }
        lg[nt][i] = vis ? (s[0][nt][i] + s[1][nt][i]) * rsc[r] : -INFINITY;
      }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float m0 = fmaxf(lg[nt][0], lg[nt][2]), m1 = fmaxf(lg[nt][1], lg[nt][3]);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(~0u, m0, off));
        m1 = fmaxf(m1, __shfl_xor_sync(~0u, m1, off));
      }
      const int r0 = 16 * rn + 8 * nt + 2 * t;
      if (g == 0) { red[km * kKvRows + r0] = m0; red[km * kKvRows + r0 + 1] = m1; }
    }
    __syncthreads();
    if (tid < kKvRows) {
      const float bm = fmaxf(fmaxf(red[tid], red[kKvRows + tid]), fmaxf(red[2 * kKvRows + tid], red[3 * kKvRows + tid]));
      const float mo = rm[tid], mn = fmaxf(mo, bm);
      ral[tid] = mn == -INFINITY ? 1.f : ex2(mo - mn);   // mo = -inf: nothing accumulated yet
      rm[tid] = mn;
    }
    __syncthreads();
    // ---- P = 2^(S - m) in fp16 to the [row][key] tile; partial row sums -----
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int r0 = 16 * rn + 8 * nt + 2 * t;
      const float mr0 = rm[r0], mr1 = rm[r0 + 1];
      float p4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float m = (i & 1) ? mr1 : mr0;
        p4[i] = lg[nt][i] == -INFINITY ? 0.f : ex2(lg[nt][i] - m);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = r0 + (i & 1), key = 16 * km + g + 8 * (i >> 1);
        *reinterpret_cast<__half*>(pt + r * kKvPRowBytes + key * 2) = __float2half_rn(p4[i]);
      }
      // the row sums are taken over the fp16 values the tensor op will use
      float s0 = __half2float(__float2half_rn(p4[0])) + __half2float(__float2half_rn(p4[2]));
      float s1 = __half2float(__float2half_rn(p4[1])) + __half2float(__float2half_rn(p4[3]));
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        s0 += __shfl_xor_sync(~0u, s0, off);
        s1 += __shfl_xor_sync(~0u, s1, off);
      }
      if (g == 0) { red[km * kKvRows + r0] = s0; red[km * kKvRows + r0 + 1] = s1; }
    }
    __syncthreads();
    if (tid < kKvRows)
      lsum = lsum * ral[tid] + ((red[tid] + red[kKvRows + tid]) + (red[2 * kKvRows + tid] + red[3 * kKvRows + tid]));
    // ---- O^T[dims 32 warp ..][rows] += V^T P, V = the tile's first 512 dims ---
    {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float a0 = ral[8 * nt + 2 * t], a1 = ral[8 * nt + 2 * t + 1];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          O[mt][nt][0] *= a0; O[mt][nt][1] *= a1;
          O[mt][nt][2] *= a0; O[mt][nt][3] *= a1;
        }
      }
      const int mi = lane >> 3, mj = lane & 7;           // ldmatrix: matrix, row
#pragma unroll
      for (int kk = 0; kk < kKvBN / 16; ++kk) {
        uint32_t a[2][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const int d0 = 32 * warp + 16 * mt;
          ldsm_x4_t(kbase + (16 * kk + mj + 8 * (mi >> 1)) * kKvRowBytes + (d0 + 8 * (mi & 1)) * 2, a[mt]);
        }
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t bp[4];                                // n-tiles 2 np and 2 np + 1
          ldsm_x4(pbase + (16 * np + 8 * (lane >> 4) + (lane & 7)) * kKvPRowBytes +
                      (16 * kk + 8 * ((lane >> 3) & 1)) * 2,
                  bp);
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            mma_f16(O[mt][2 * np], a[mt], bp[0], bp[1], O[mt][2 * np]);
            mma_f16(O[mt][2 * np + 1], a[mt], bp[2], bp[3], O[mt][2 * np + 1]);
          }
        }
      }
    }
  }
  cp_async_wait<0>();
  if (tid < kKvRows) red[tid] = lsum;                    // final row sums
  __syncthreads();
  grid_dep_launch();

  // ---- output: O / l (whole unit) or the partial (m, l, O) ---------------------
  const bool complete = p.pieces == 1;
  const int64_t slot = 2 * (int64_t)blockIdx.x;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int r = 8 * nt + 2 * t + j, row = rbase + r;
      if (row >= p.G) continue;
      const float l = red[r];
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
          const int dim = 32 * warp + 16 * mt + g + 8 * hi;
          const float o = O[mt][nt][2 * hi + j];
          if (complete) store_from_float(p.out, p.out_dtype, (uh * p.G + row) * kKvDv + dim, o * inv);
          else p.part_o[(slot * kKvRows + r) * kKvDv + dim] = o;
        }
    }
  if (!complete && tid < kKvRows) {
    p.part_ml[(slot * kKvRows + tid) * 2] = rm[tid];
    p.part_ml[(slot * kKvRows + tid) * 2 + 1] = red[tid];
  }
}

template <bool Q8, int BITS, int GS>
cudaError_t launch_kv(DecodeParams& p, int64_t units, int pieces, cudaStream_t s) {
  using C = KvCfg<Q8, BITS, GS>;
  auto k = qsdpa_kview_kernel<Q8, BITS, GS>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(units * pieces));
  cfg.blockDim = dim3(kKvThreads);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k, p);
  if (e != cudaSuccess || pieces == 1) return e;
  // merge of the split units: the decode's merge kernel on 512-wide rows
  int lanes = 1;
  while (lanes < 4 && lanes * kMergeBatch < pieces) lanes *= 2;
  const int64_t threads = units * kKvRows * (kKvDv / 4) * lanes;
  cfg.gridDim = dim3((unsigned)((threads + kMergeThreads - 1) / kMergeThreads));
  cfg.blockDim = dim3(kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&cfg, qsdpa_merge_kernel<kKvDv, kKvRows>, p, units * pieces, lanes);
}

int kv_sm_count() {
  static int cached[64] = {};
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

}  // namespace

size_t kview_workspace_bytes() {
  return (size_t)2 * kKvMaxGrid * kKvRows * (kKvDv + 2) * 4;
}

// Plans and launches the view attention: every unit split over the same
// number of CTAs (one CTA per SM in all, at most the workspace's slots, at
// least two blocks of keys per CTA).
cudaError_t launch_kview(int bits, int gs, int fmt, DecodeParams& p, cudaStream_t s) {
  const int64_t rows = p.G;
  p.ncg = (int)((rows + kKvRows - 1) / kKvRows);
  const int64_t units = (int64_t)p.B * p.Hkv * p.ncg;
  const int64_t S = (p.L + kKvBN - 1) / kKvBN;
  int64_t pieces = std::max<int64_t>(1, std::min<int64_t>(kv_sm_count() / std::max<int64_t>(1, units),
                                                          (S + 1) / 2));
  pieces = std::min<int64_t>(pieces, std::max<int64_t>(1, kKvMaxGrid / units));
  if (units * pieces > kKvMaxGrid && pieces > 1) pieces = 1;
  if (units > 0x7fffffff / pieces) return cudaErrorInvalidValue;
  p.stages_per_unit = S;
  p.total_stages = units * S;
  p.pieces = (int)pieces;
  // the merge kernel's partial layout: o [slot][64][512], (m, l) [slot][64][2]
  float* part = p.part_o;
  p.part_ml = part + (size_t)2 * kKvMaxGrid * kKvRows * kKvDv;
  const bool q8 = fmt == QKV_Q8_0;
  if (q8) return launch_kv<true, 8, 32>(p, units, (int)pieces, s);
  if (bits == 8 && gs == 32) return launch_kv<false, 8, 32>(p, units, (int)pieces, s);
  if (bits == 8 && gs == 64) return launch_kv<false, 8, 64>(p, units, (int)pieces, s);
  if (bits == 4 && gs == 32) return launch_kv<false, 4, 32>(p, units, (int)pieces, s);
  if (bits == 4 && gs == 64) return launch_kv<false, 4, 64>(p, units, (int)pieces, s);
  return cudaErrorInvalidValue;
}

}  // namespace qkv
