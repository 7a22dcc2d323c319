// prefill_kernel.cuh -- multi-query attention over a group-quantized KV cache
// on the 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// What it computes (MLX compare "v0.19.3...quantized-kv-update", mlx/fast.cpp
// quantized_scaled_dot_product_attention, the Lq > 1 fallback:
// quantized_matmul(q, K^T) -> + mask -> softmax -> quantized_matmul(P, V)), in
// one fused pass per tile, for the KV formats of the decode kernel.  The
// dequantize-tiles-to-16-bit-then-MMA pattern follows the MLX CUDA work-in-
// progress page (SharedTile::load_quantized feeding the tensor cores); the
// 5th-generation MMA, TMEM, the warp roles and the layouts are this kernel's.
//
// One CTA owns 128 rows (TMEM lanes) of one kv head; a row is a (query, head)
// pair, r = query * G + head, so the G heads that share a KV head share every
// dequantized K/V tile and a tile's rows span few query positions (tight
// causal bound).  Three warp roles work on 32-key tiles, double-buffered:
//   * dequant warps (4): cp.async the packed codes and scales of tile t+2 into
//     a two-slot ring while dequantizing tile t into fp16 K [key][d] and
//     V [d][key] in the tensor core's K-major swizzled layouts;
//   * MMA warp (1): S(t) = Q K(t)^T into TMEM (M=128, N=32, K=16 per op), and
//     once the softmax warps hand over P(t-1), O += P(t-1) V(t-1) (M=128,
//     N=D); completion is signalled with tcgen05.commit on mbarriers;
//   * softmax warps (4, one TMEM lane = one row per thread): scale and mask
//     S, online softmax with a lazily moved maximum (moved only when it grows
//     by more than 2^8, so the O accumulator in TMEM is rarely rescaled), P as
//     fp16 into shared memory; finally O / l to the output.
// Every mbarrier wait is bounded: a time-out records an error in the status
// word and makes every later wait return at once, so all roles finish the
// tile loop, release TMEM and return.
#pragma once

#include "qkv_common.cuh"
#include "qkv_internal.h"

namespace qkv {

constexpr int kPfBM = 128;        // rows per CTA
constexpr int kPfBN = 32;         // keys per tile
constexpr int kPfSoftWarps = 4;
constexpr int kPfDqWarps = 4;
constexpr int kPfMmaWarp = kPfSoftWarps + kPfDqWarps;
constexpr int kPfThreads = 32 * (kPfMmaWarp + 1);
constexpr unsigned kPfWaitLimit = 1u << 21;   // try_wait rounds (<= 1 us each) before giving up

struct PrefillParams {
  const void* q;            // [B, Hq, Lq, D]
  int q_dtype;
  void* out;                // [B, Hq, Lq, D]
  int out_dtype;
  const uint8_t* kc;
  const uint16_t* ks;
  const uint16_t* kb;
  const uint8_t* vc;
  const uint16_t* vs;
  const uint16_t* vb;
  int64_t Lcap, L;
  int B, Hq, Hkv, G, Lq;
  int mtiles;               // 128-row tiles per kv head
  float scale_log2e;
  int mask_kind;
  const void* mask;
  int mask_dtype;
  int64_t msb, msh, msq;
  unsigned* status;         // nonzero after a tensor-core wait timed out
};

template <int D, int BITS, int GS, bool Q8>
struct PfCfg {
  static constexpr int RB = D * BITS / 8;            // bytes per code row
  static constexpr int UPR = RB / 16;
  static constexpr int NG = D / GS;
  static constexpr int NMETA = Q8 ? 2 : 4;
  static constexpr int META_BYTES = ((kPfBN * NG * 2 + 127) / 128) * 128;
  // operands (1024-byte aligned): Q, K[2], V[2], P[2]
  static constexpr int Q_OFF = 0;
  static constexpr int Q_BYTES = kPfBM * D * 2;      // SW128: D/64 blocks of [128][64]
  static constexpr int K_BYTES = kPfBN * D * 2;      // SW128: D/64 blocks of [32][64]
  static constexpr int K_OFF = Q_OFF + Q_BYTES;
  static constexpr int V_BYTES = D * kPfBN * 2;      // SW64: [D][32]
  static constexpr int V_OFF = K_OFF + 2 * K_BYTES;
  static constexpr int P_BYTES = kPfBM * kPfBN * 2;  // SW64: [128][32]
  static constexpr int P_OFF = V_OFF + 2 * V_BYTES;
  // raw ring slots: K codes, V codes, metadata arrays
  static constexpr int RAW_BYTES = 2 * kPfBN * RB + NMETA * META_BYTES;
  static constexpr int RAW_OFF = P_OFF + 2 * P_BYTES;
  static constexpr int BAR_OFF = RAW_OFF + 2 * RAW_BYTES;
  static constexpr int SMEM = BAR_OFF + 128 + 1024;  // + barriers, TMEM slot, alignment slack
  static constexpr int TMEM_COLS = D + 2 * kPfBN <= 128 ? 128 : (D + 2 * kPfBN <= 256 ? 256 : 512);
  static_assert(D + 2 * kPfBN <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

// ---- tcgen05 / mbarrier wrappers -------------------------------------------
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_init(uint32_t addr, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" :: "r"(addr), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t addr) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}\n"
               :: "r"(addr) : "memory");
}
// Bounded wait for the phase with the given parity.  Returns at once (false)
// if the CTA has already given up; on a time-out it records the error and
// makes the CTA give up.
__device__ __forceinline__ bool mbar_wait(uint32_t addr, uint32_t parity, volatile int* abort_flag,
                                          unsigned* status, unsigned code) {
  for (unsigned i = 0; i < kPfWaitLimit; ++i) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done) : "r"(addr), "r"(parity), "r"(1000u) : "memory");
    if (done) return true;
    if (*abort_flag) return false;
  }
  *abort_flag = 1;
  atomicOr(status, code);
  return false;
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n"
               :: "r"(bar) : "memory");
}
// D(tmem) (+)= A(smem desc) * B(smem desc), kind::f16 with fp32 accumulate.
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
      :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate),
         "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
// Shared-memory matrix descriptor of a K-major operand with 8-row groups
// `sbo` bytes apart; swizzle 2 = 128-byte rows (64 16-bit elements), 4 =
// 64-byte rows (32 elements).
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t sbo, uint32_t swizzle) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3fff);          // start address
  d |= (uint64_t)1 << 16;                          // leading byte offset (unused, 16 B)
  d |= (uint64_t)((sbo >> 4) & 0x3fff) << 32;      // stride byte offset
  d |= (uint64_t)1 << 46;                          // descriptor version (sm_100)
  d |= (uint64_t)swizzle << 61;
  return d;
}
// Instruction descriptor: f16 x f16 -> f32, both operands K-major, M x N.
__host__ __device__ constexpr uint32_t f16_idesc(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// 32 consecutive fp32 columns of this thread's TMEM lane (warp-collective).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n"
      :: "r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
         "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])),
         "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
         "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
         "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
         "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
         "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
         "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
         "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
         "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
         "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;\n" :: "r"(id), "r"(nthreads) : "memory");
}

// Byte offset of 16-bit element (row, col) in a K-major operand with
// 128-byte swizzled rows (64 columns per block, `rows` rows per block).
__device__ __forceinline__ int sw128_off(int row, int col, int rows) {
  const int blk = col >> 6, chunk = (col >> 3) & 7;
  return blk * rows * 128 + row * 128 + ((chunk ^ (row & 7)) << 4) + (col & 7) * 2;
}
// Same for 64-byte swizzled rows (32 columns).
__device__ __forceinline__ int sw64_off(int row, int col) {
  const int chunk = (col >> 3) & 3;
  return row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4) + (col & 7) * 2;
}

// Position of head-dimension element e inside a K-major row.  The 4-bit codes
// of a 32-bit word come out of the mask-and-magic conversion as the pairs
// (0,4), (1,5), (2,6), (3,7); Q is stored with the same permutation so Q K^T is
// unchanged.  8-bit codes come out in natural order.
template <int BITS>
__device__ __forceinline__ int k_pos(int e) {
  if constexpr (BITS == 4) {
    const int j = e & 7;
    return (e & ~7) | ((j & 3) << 1) | (j >> 2);
  } else {
    return e;
  }
}

// Low bytes of lanes 0/2 of a word -> fp16 pair (1024 + b0, 1024 + b2): the
// magic exponent 0x64 makes the fp16 value 1024 + byte exactly.
__device__ __forceinline__ __half2 u8pair_plus1024(uint32_t w) {
  const uint32_t x = (w & 0x00FF00FFu) | 0x64006400u;
  return *reinterpret_cast<const __half2*>(&x);
}

// Raw V rows are stored with their 16-byte units XOR-swizzled by (row / 8)
// so the transposing reads below (8 rows x 8 word positions per warp) spread
// over all banks.
template <int UPR>
__device__ __forceinline__ int rawv_unit(int row, int unit) {
  constexpr int M = UPR >= 8 ? 7 : UPR - 1;
  return unit ^ ((row >> 3) & M);
}

// Dequantizes one staged tile (raw slot `raw`) into K (fp16 [key][d], SW128)
// and V (fp16 [d][key], SW64); value = scale * code + bias rounded once.
template <int D, int BITS, int GS, bool Q8>
__device__ __forceinline__ void dequant_tile(const uint8_t* raw, uint8_t* kdst, uint8_t* vdst,
                                             int dq) {
  using C = PfCfg<D, BITS, GS, Q8>;
  constexpr int NG = C::NG;
  constexpr int NT = 32 * kPfDqWarps;
  const uint8_t* rk = raw;
  const uint8_t* rv = raw + kPfBN * C::RB;
  const uint8_t* meta = raw + 2 * kPfBN * C::RB;
  const uint16_t* mks = reinterpret_cast<const uint16_t*>(meta);
  const uint16_t* mkb = reinterpret_cast<const uint16_t*>(meta + C::META_BYTES);
  const uint16_t* mvs = reinterpret_cast<const uint16_t*>(meta + (Q8 ? 1 : 2) * C::META_BYTES);
  const uint16_t* mvb = reinterpret_cast<const uint16_t*>(meta + 3 * C::META_BYTES);
  const __half2 off = __float2half2_rn(Q8 ? 1152.f : 1024.f);   // Q8 codes are stored +128

  // K: one 16-byte output chunk (8 elements of one key) per step
  constexpr int KCH = D / 8;
  for (int ci = dq; ci < kPfBN * KCH; ci += NT) {
    const int j = ci / KCH, c = ci - j * KCH;
    const int G = (c * 8) / GS;
    const __half2 s2 = __half2half2(__ushort_as_half(mks[j * NG + G]));
    const __half2 b2 = Q8 ? __float2half2_rn(0.f) : __half2half2(__ushort_as_half(mkb[j * NG + G]));
    __half2 h[4];
    if constexpr (BITS == 8) {
      const uint2 w = *reinterpret_cast<const uint2*>(rk + j * C::RB + c * 8);
      const uint32_t w0 = Q8 ? (w.x ^ 0x80808080u) : w.x, w1 = Q8 ? (w.y ^ 0x80808080u) : w.y;
      h[0] = u8pair_plus1024(prmt(w0, 0u, 0x4140u));
      h[1] = u8pair_plus1024(prmt(w0, 0u, 0x4342u));
      h[2] = u8pair_plus1024(prmt(w1, 0u, 0x4140u));
      h[3] = u8pair_plus1024(prmt(w1, 0u, 0x4342u));
    } else {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(rk + j * C::RB + c * 4);
#pragma unroll
      for (int k = 0; k < 4; ++k) {      // nibbles (k, k+4) -> positions (2k, 2k+1)
        const uint32_t x = ((w >> (4 * k)) & 0x000F000Fu) | 0x64006400u;
        h[k] = *reinterpret_cast<const __half2*>(&x);
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 v = __hfma2(__hsub2(h[i], off), s2, b2);
      o[i] = *reinterpret_cast<const uint32_t*>(&v);
    }
    *reinterpret_cast<uint4*>(kdst + sw128_off(j, c * 8, kPfBN)) = make_uint4(o[0], o[1], o[2], o[3]);
  }

  // V: a task = one 32-bit code word position (EPW dims) x 8 keys, transposed
  // in registers into EPW output chunks (one per dim) of 8 keys each
  constexpr int EPW = 32 / BITS;                 // dims per word
  constexpr int WPR = D / EPW;                   // words per key row
  constexpr int KB8 = kPfBN / 8;                 // 8-key blocks per tile
  for (int task = dq; task < WPR * KB8; task += NT) {
    const int kb8 = task % KB8, wi = task / KB8;
    const int e0 = wi * EPW, j0 = kb8 * 8;
    const int G = e0 / GS;
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = j0 + i;
      const int unit = rawv_unit<C::UPR>(r, (wi * 4) >> 4);
      w[i] = *reinterpret_cast<const uint32_t*>(rv + r * C::RB + unit * 16 + ((wi * 4) & 15));
      if (Q8) w[i] ^= 0x80808080u;
    }
    __half2 s2[4], b2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      s2[i] = __halves2half2(__ushort_as_half(mvs[(j0 + 2 * i) * NG + G]),
                             __ushort_as_half(mvs[(j0 + 2 * i + 1) * NG + G]));
      b2[i] = Q8 ? __float2half2_rn(0.f)
                 : __halves2half2(__ushort_as_half(mvb[(j0 + 2 * i) * NG + G]),
                                  __ushort_as_half(mvb[(j0 + 2 * i + 1) * NG + G]));
    }
#pragma unroll
    for (int d = 0; d < EPW; ++d) {
      uint32_t hv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        __half2 c;
        if constexpr (BITS == 8) {
          // byte d of the words of keys j0+2i and j0+2i+1 -> lanes 0 and 2
          c = __hsub2(u8pair_plus1024(prmt(w[2 * i], w[2 * i + 1], (uint32_t)(d | ((4 + d) << 8)))), off);
        } else {
          const int sh = 4 * d;
          const uint32_t x = ((w[2 * i] >> sh) & 0xFu) | (((w[2 * i + 1] >> sh) & 0xFu) << 16) |
                             0x64006400u;
          c = __hsub2(*reinterpret_cast<const __half2*>(&x), off);
        }
        const __half2 v = __hfma2(c, s2[i], b2[i]);
        hv[i] = *reinterpret_cast<const uint32_t*>(&v);
      }
      *reinterpret_cast<uint4*>(vdst + sw64_off(e0 + d, j0)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
    }
  }
}

template <int D, int BITS, int GS, bool Q8>
__global__ void __launch_bounds__(kPfThreads, 1) qsdpa_prefill_tc_kernel(const PrefillParams p) {
  using C = PfCfg<D, BITS, GS, Q8>;
  constexpr int NG = C::NG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // mbarriers: kv_ready[2], s_full[2], p_ready[2], pv_done[2]
  const uint32_t bar0 = sbase + C::BAR_OFF;
  auto kv_ready = [&](int i) { return bar0 + 8 * i; };
  auto s_full = [&](int i) { return bar0 + 16 + 8 * i; };
  auto p_ready = [&](int i) { return bar0 + 32 + 8 * i; };
  auto pv_done = [&](int i) { return bar0 + 48 + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::BAR_OFF + 64);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::BAR_OFF + 68);

  const int mt = blockIdx.x % p.mtiles;
  const int hkv = (blockIdx.x / p.mtiles) % p.Hkv;
  const int b = blockIdx.x / (p.mtiles * p.Hkv);
  const int R = p.G * p.Lq;                       // rows of this kv head
  const int64_t L = p.L;
  int64_t kend = L;                               // causal rows see keys <= L - Lq + query
  if (p.mask_kind == QKV_MASK_CAUSAL) {
    const int last_row = min(R, (mt + 1) * kPfBM) - 1;
    kend = min(L, L - p.Lq + last_row / p.G + 1);
  }
  const int ntiles = kend > 0 ? (int)((kend + kPfBN - 1) / kPfBN) : 0;

  if (warp == kPfMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n"
                 :: "r"(smem_u32(tmem_slot)), "r"(C::TMEM_COLS) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(kv_ready(i), 32 * kPfDqWarps);
      mbar_init(s_full(i), 1);
      mbar_init(p_ready(i), 32 * kPfSoftWarps);
      mbar_init(pv_done(i), 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    *abort_flag = 0;
  }

  // ---- Q rows -> fp16 (per-row power-of-two prescale), swizzled K-major ----
  const int r = mt * kPfBM + tid;                 // softmax threads: this thread's row
  const bool row_ok = tid < kPfBM && r < R;
  const int qi = row_ok ? r / p.G : 0;
  const int hh = row_ok ? r - qi * p.G : 0;
  const int64_t qrow = (((int64_t)b * p.Hq + (int64_t)hkv * p.G + hh) * p.Lq + qi) * D;
  float rowscale = 0.f;
  if (tid < kPfBM) {
    float mx = 0.f;
    if (row_ok) {
      for (int e = 0; e < D; e += 8) {
        const uint4 raw = *reinterpret_cast<const uint4*>(
            reinterpret_cast<const uint16_t*>(p.q) + qrow + e);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float a = p.q_dtype == QKV_F16 ? __half2float(__ushort_as_half((uint16_t)(w[k] & 0xffff)))
                                               : __uint_as_float(w[k] << 16);
          const float c = p.q_dtype == QKV_F16 ? __half2float(__ushort_as_half((uint16_t)(w[k] >> 16)))
                                               : __uint_as_float(w[k] & 0xffff0000u);
          mx = fmaxf(mx, fmaxf(fabsf(a), fabsf(c)));
        }
      }
    }
    int sigma = mx > 0.f ? 14 - (int)(((__float_as_uint(mx) >> 23) & 0xff) - 127) : 0;
    sigma = max(-96, min(96, sigma));
    const float up = exp2i(sigma);
    rowscale = p.scale_log2e * exp2i(-sigma);
    uint16_t* qs = reinterpret_cast<uint16_t*>(smem + C::Q_OFF);
    for (int e = 0; e < D; e += 8) {
      uint32_t w[4] = {0u, 0u, 0u, 0u};
      if (row_ok) {
        const uint4 raw = *reinterpret_cast<const uint4*>(
            reinterpret_cast<const uint16_t*>(p.q) + qrow + e);
        w[0] = raw.x; w[1] = raw.y; w[2] = raw.z; w[3] = raw.w;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint16_t bits = (uint16_t)(w[k >> 1] >> (16 * (k & 1)));
        const float v = p.q_dtype == QKV_F16 ? __half2float(__ushort_as_half(bits))
                                             : __uint_as_float((uint32_t)bits << 16);
        qs[sw128_off(tid, k_pos<BITS>(e + k), kPfBM) / 2] = __half_as_ushort(__float2half_rn(v * up));
      }
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int64_t row0 = ((int64_t)b * p.Hkv + hkv) * p.Lcap;
  constexpr uint32_t kS_COL = D;                   // S[2] after O

  if (warp >= kPfSoftWarps && warp < kPfMmaWarp) {
    // ======================= dequant warps =====================================
    const int dq = tid - 32 * kPfSoftWarps;
    constexpr int NT = 32 * kPfDqWarps;
    const uint8_t* gK = p.kc + row0 * C::RB;
    const uint8_t* gV = p.vc + row0 * C::RB;
    const uint8_t* gKs = reinterpret_cast<const uint8_t*>(p.ks + row0 * NG);
    const uint8_t* gKb = Q8 ? gKs : reinterpret_cast<const uint8_t*>(p.kb + row0 * NG);
    const uint8_t* gVs = reinterpret_cast<const uint8_t*>(p.vs + row0 * NG);
    const uint8_t* gVb = Q8 ? gVs : reinterpret_cast<const uint8_t*>(p.vb + row0 * NG);
    auto issue = [&](int t) {
      const uint32_t slot = sbase + C::RAW_OFF + (t & 1) * C::RAW_BYTES;
      const int64_t key0 = (int64_t)t * kPfBN;
      const int64_t nvalid = L - key0;
      constexpr int CU = kPfBN * C::UPR;
      for (int i = dq; i < 2 * CU; i += NT) {
        const int which = i >= CU, j = which ? i - CU : i;
        const int row = j / C::UPR, unit = j - row * C::UPR;
        const bool ok = row < nvalid;
        const uint8_t* src = (which ? gV : gK) + (ok ? (key0 + row) * C::RB + unit * 16 : 0);
        const int dst = which ? kPfBN * C::RB + row * C::RB + rawv_unit<C::UPR>(row, unit) * 16
                              : j * 16;
        cp_async16(slot + dst, src, ok ? 16 : 0);
      }
      constexpr int MU = kPfBN * NG * 2 / 16;
      for (int i = dq; i < C::NMETA * MU; i += NT) {
        const int arr = i / MU, j = i - arr * MU;
        const uint8_t* gm = Q8 ? (arr == 0 ? gKs : gVs)
                               : (arr == 0 ? gKs : arr == 1 ? gKb : arr == 2 ? gVs : gVb);
        const bool ok = (j * 16) / (NG * 2) < nvalid;
        cp_async16(slot + 2 * kPfBN * C::RB + arr * C::META_BYTES + j * 16,
                   ok ? gm + key0 * NG * 2 + j * 16 : gm, ok ? 16 : 0);
      }
    };
    if (ntiles > 0) issue(0);
    cp_async_commit();
    if (ntiles > 1) issue(1);
    cp_async_commit();
    for (int t = 0; t < ntiles; ++t) {
      const int s = t & 1;
      cp_async_wait<1>();
      named_sync(1, NT);
      uint8_t* raw = smem + C::RAW_OFF + s * C::RAW_BYTES;
      const int64_t nvalid = L - (int64_t)t * kPfBN;
      if (nvalid < kPfBN) {          // clear stale scales/biases of keys past L
        uint16_t* meta = reinterpret_cast<uint16_t*>(raw + 2 * kPfBN * C::RB);
        for (int i = dq; i < C::NMETA * kPfBN * NG; i += NT) {
          const int arr = i / (kPfBN * NG), rr = i - arr * kPfBN * NG;
          if (rr / NG >= nvalid) meta[arr * (C::META_BYTES / 2) + rr] = 0;
        }
        named_sync(1, NT);
      }
      if (t >= 2) {                  // operand slot s free once P V of tile t-2 is done
        mbar_wait(pv_done(s), ((t - 2) >> 1) & 1, abort_flag, p.status, 1u);
        tc_fence_after();
      }
      dequant_tile<D, BITS, GS, Q8>(raw, smem + C::K_OFF + s * C::K_BYTES,
                                    smem + C::V_OFF + s * C::V_BYTES, dq);
      fence_async_smem();
      mbar_arrive(kv_ready(s));
      named_sync(1, NT);             // everyone is done reading raw slot s
      if (t + 2 < ntiles) issue(t + 2);
      cp_async_commit();
    }
    cp_async_wait<0>();
  } else if (warp == kPfMmaWarp) {
    // ======================= MMA warp ==========================================
    constexpr uint32_t idesc_s = f16_idesc(kPfBM, kPfBN);
    constexpr uint32_t idesc_o = f16_idesc(kPfBM, D);
    auto issue_s = [&](int t) {
      const int s = t & 1;
      mbar_wait(kv_ready(s), (t >> 1) & 1, abort_flag, p.status, 2u);
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const int blk = k >> 2, sub = (k & 3) * 32;
          const uint64_t a = umma_desc(sbase + C::Q_OFF + blk * kPfBM * 128 + sub, 1024, 2);
          const uint64_t bd = umma_desc(sbase + C::K_OFF + s * C::K_BYTES + blk * kPfBN * 128 + sub,
                                        1024, 2);
          tc_mma(tmem + kS_COL + s * kPfBN, a, bd, idesc_s, k > 0 ? 1u : 0u);
        }
        tc_commit(s_full(s));
      }
      __syncwarp();
    };
    auto issue_pv = [&](int t) {
      const int s = t & 1;
      mbar_wait(p_ready(s), (t >> 1) & 1, abort_flag, p.status, 4u);
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int k = 0; k < kPfBN / 16; ++k) {
          const uint64_t a = umma_desc(sbase + C::P_OFF + s * C::P_BYTES + k * 32, 512, 4);
          const uint64_t bd = umma_desc(sbase + C::V_OFF + s * C::V_BYTES + k * 32, 512, 4);
          tc_mma(tmem, a, bd, idesc_o, (t > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(pv_done(s));
      }
      __syncwarp();
    };
    if (ntiles > 0) issue_s(0);
    for (int t = 0; t < ntiles; ++t) {
      if (t + 1 < ntiles) issue_s(t + 1);   // overlaps the softmax of tile t
      issue_pv(t);
    }
  } else {
    // ======================= softmax warps (one row per thread) =================
    const uint32_t tmem_row = tmem + ((uint32_t)(warp * 32) << 16);
    const int64_t causal_lim = L - p.Lq + qi;    // last visible key of this row
    float m_used = -INFINITY, lsum = 0.f;
    for (int t = 0; t < ntiles; ++t) {
      const int s = t & 1;
      const int64_t key0 = (int64_t)t * kPfBN;
      mbar_wait(s_full(s), (t >> 1) & 1, abort_flag, p.status, 8u);
      tc_fence_after();
      float sv[kPfBN];
      tmem_ld32(tmem_row + kS_COL + s * kPfBN, sv);
      tmem_wait_ld();
      float tmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < kPfBN; ++j) {
        const int64_t key = key0 + j;
        float v = sv[j] * rowscale;
        bool vis = row_ok && key < kend;
        if (p.mask_kind == QKV_MASK_CAUSAL) vis = vis && key <= causal_lim;
        if (vis && p.mask_kind == QKV_MASK_ADDITIVE) {
          const int64_t mi = (int64_t)b * p.msb + ((int64_t)hkv * p.G + hh) * p.msh +
                             (int64_t)qi * p.msq + key;
          v += kLog2e * load_as_float(p.mask, p.mask_dtype, mi);
        }
        sv[j] = vis ? v : -INFINITY;
        tmax = fmaxf(tmax, sv[j]);
      }
      float alpha = 1.f;
      if (tmax > m_used + 8.f || (m_used == -INFINITY && tmax != -INFINITY)) {
        alpha = m_used == -INFINITY ? 0.f : ex2(m_used - tmax);
        m_used = tmax;
      }
      const float mref = m_used == -INFINITY ? 0.f : m_used;
      // P slot s is free once the P V product of tile t-2 is done; the O
      // rescale needs the product of tile t-1 done (both are rare waits)
      if (t >= 2) mbar_wait(pv_done(s), ((t - 2) >> 1) & 1, abort_flag, p.status, 16u);
      const bool rescale = t > 0 && __any_sync(~0u, alpha != 1.f);
      if (rescale) {
        mbar_wait(pv_done(s ^ 1), ((t - 1) >> 1) & 1, abort_flag, p.status, 32u);
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          float o[32];
          tmem_ld32(tmem_row + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(tmem_row + c, o);
        }
        tmem_wait_st();
      }
      float rs = 0.f;
      uint8_t* ps = smem + C::P_OFF + s * C::P_BYTES;
#pragma unroll
      for (int j = 0; j < kPfBN; j += 8) {
        uint32_t pk[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float a = ex2(sv[j + 2 * i] - mref), c = ex2(sv[j + 2 * i + 1] - mref);
          rs += a + c;
          pk[i] = pack_half2(a, c);
        }
        *reinterpret_cast<uint4*>(ps + sw64_off(tid, j)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      lsum = lsum * alpha + rs;
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(p_ready(s));
    }
    // ---- epilogue: O / l -> out --------------------------------------------
    bool have = ntiles > 0;
    if (have) {
      have = mbar_wait(pv_done((ntiles - 1) & 1), ((ntiles - 1) >> 1) & 1, abort_flag, p.status, 64u);
      tc_fence_after();
    }
    have = __all_sync(~0u, have) && !*abort_flag;
    const float inv = (lsum > 0.f && have) ? 1.f / lsum : 0.f;
    for (int c = 0; c < D; c += 32) {
      float o[32];
      if (have) {
        tmem_ld32(tmem_row + c, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0.f;
      }
      if (row_ok) {
        if (p.out_dtype == QKV_BF16 || p.out_dtype == QKV_F16) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint32_t pk[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float a = o[i + 2 * k] * inv, cc = o[i + 2 * k + 1] * inv;
              if (p.out_dtype == QKV_F16) {
                pk[k] = pack_half2(a, cc);
              } else {
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(a, cc);
                pk[k] = *reinterpret_cast<const uint32_t*>(&h2);
              }
            }
            *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) + qrow + c + i) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) store_from_float(p.out, p.out_dtype, qrow + c + i, o[i] * inv);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kPfMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n"
                 :: "r"(tmem), "r"(C::TMEM_COLS) : "memory");
  }
}

}  // namespace qkv
