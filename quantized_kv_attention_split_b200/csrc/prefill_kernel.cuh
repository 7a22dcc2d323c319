// prefill_kernel.cuh -- multi-query attention over a group-quantized KV cache
// on the 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// What it computes (MLX compare "v0.19.3...quantized-kv-update", mlx/fast.cpp
// quantized_scaled_dot_product_attention, the Lq > 1 fallback:
// quantized_matmul(q, K^T) -> + mask -> softmax -> quantized_matmul(P, V)), in
// one fused pass per tile, for the KV formats of the decode kernel.  The
// dequantize-tiles-to-16-bit-then-MMA pattern follows the MLX CUDA work-in-
// progress page (SharedTile::load_quantized feeding the tensor cores); the
// 5th-generation MMA, TMEM residency, the warp roles and the layouts are this
// kernel's.
//
// One CTA owns 128 rows (TMEM lanes) of one kv head; a row is a (query, head)
// pair, r = query * G + head, so the G heads that share a KV head share every
// dequantized K/V tile and a tile's rows span few query positions (tight
// causal bound).  Work goes in 32-key tiles through three warp roles:
//   * producer warp (1): bulk copies (cp.async.bulk, one per contiguous array)
//     of the packed codes and scales of 32-key half tiles into a four-slot
//     ring, refilled as soon as the dequant warps release a tile's slots;
//   * dequant warps (10): turn tile t into fp16 K and V, both stored
//     [key][d] with 128-byte swizzled rows (K is the K-major B operand of
//     S = Q K^T, V the MN-major B operand of O += P V), two K slots and three
//     V slots so dequantization runs ahead of the tensor cores;
//   * MMA warp (1): S(t) = Q K(t)^T and O += P(t-1) V(t-1) with Q and P read
//     from TMEM (the A operand), so shared memory only streams K and V;
//     completion is signalled with tcgen05.commit on mbarriers;
//   * softmax warps (4, one TMEM lane = one row per thread): stage the
//     prescaled Q into TMEM, then per tile: scale and mask S, online softmax
//     with a lazily moved maximum (moved only when it grows by more than 2^8,
//     so O in TMEM is rarely rescaled), P as fp16 into TMEM; finally O / l to
//     the output.
// Range: the fp16 tiles hold scale * code + bias, which leaves the fp16 range
// for caches of large values (bf16 inputs, or fp16 ones near its maximum).
// The magnitudes are bounded from the scales and biases (read straight from
// global memory, off the
// tiles' critical path).  A call launches a check of every scale and bias in
// rows [0, L) (qkv_range_check_kernel, ~1 MB for the 512-query prompt at
// depth 20K), which raises a flag in the workspace when some value can reach
// 2^15, then two instances of this kernel.  The first (RANGE false) is the
// kernel described above and runs when the flag is down.  The second (RANGE
// true) runs when it is up: the producer publishes powers of two per tile,
// 2^eK for the tile's K (S of the tile is scaled back by 2^eK in the softmax)
// and 2^eV for V, the largest needed so far (O in TMEM is rescaled exactly
// when it grows, and scaled back by 2^eV at the end); its last CTA lowers the
// flag.  The instance that does not run exits at once.
// Every mbarrier wait is bounded: a time-out records an error in the status
// word and makes every later wait return at once, so all roles finish the
// tile loop; before exit the CTA waits (bounded) for its own bulk copies and
// tensor-core work in flight, then releases TMEM.
#pragma once

#include "qkv_common.cuh"
#include "qkv_internal.h"

namespace qkv {

constexpr int kPfBM = 128;        // rows per CTA
constexpr int kPfBN = 64;         // keys per tile (S = Q K^T is 128 x 64)
constexpr int kPfRawKeys = 32;    // keys per packed half tile (one bulk-copy slot)
constexpr int kPfSoftWarps = 4;   // one thread per row (TMEM lane)
constexpr int kPfSoftThreads = 32 * kPfSoftWarps;
constexpr int kPfDqWarps = 10;   // 16 warps in all: 128 registers per thread
constexpr int kPfDqThreads = 32 * kPfDqWarps;
constexpr int kPfMmaWarp = kPfSoftWarps + kPfDqWarps;
constexpr int kPfProdWarp = kPfMmaWarp + 1;     // issues the bulk copies
constexpr int kPfThreads = 32 * (kPfProdWarp + 1);
constexpr int kPfKSlots = 2;      // fp16 K tiles (slot free once S of the tile is done)
constexpr int kPfVSlots = 2;      // fp16 V tiles (slot free once P V of the tile is done)
constexpr int kPfRawSlots = 4;    // packed half tiles in flight
// A wait on a barrier gives up after this long (ns; PrefillParams.wait_ns
// overrides it): a tile's waits normally end within microseconds and a whole
// 512-query prompt at depth 20K takes about half a millisecond, so 200 ms
// leaves room for a GPU shared with other work while a CTA that can never
// proceed still reports within a fraction of a second.
constexpr uint64_t kPfWaitNs = 200000000ull;

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
  float cap_a, cap_k;       // logit softcap (cap_a == 0: off), as in DecodeParams
  const float* slopes;      // per-head additive-mask slopes, fp32 [Hq] or null
  const float* sinks;       // per-head sink logits, fp32 [Hq] or null
  unsigned* status;         // nonzero after a tensor-core wait timed out
  uint64_t wait_ns;         // time limit of a wait (0: kPfWaitNs)
  int stall_half;           // test hook: the producer never copies this half tile (-1: none)
  unsigned* range;          // [2]: a tile reaches 2^15 (set by the first instance),
                            // CTAs of the second instance done (its last zeroes both)
};

// Lane -> chunk map of the dequant warps (a GF(2)-linear map given by the
// chunk offset each lane bit adds), chosen per layout so that each 8-lane
// phase of the 16-byte packed-tile reads and of the 16-byte swizzled fp16
// writes touches eight different bank groups.
__host__ __device__ constexpr int pf_lane_col(int D, int bits, int b) {
  return (D == 128 && bits == 4 && b == 1) ? 10
       : (D == 128 && bits == 8 && b == 2) ? 12
       : (D == 256 && bits == 4 && b == 1) ? 10
       : (D == 256 && bits == 4 && b == 2) ? 20
       : (D == 256 && bits == 8 && b == 2) ? 20
       : (1 << b);
}

template <int D, int BITS, int GS, bool Q8>
struct PfCfg {
  static constexpr int RB = D * BITS / 8;            // bytes per code row
  static constexpr int UPR = RB / 16;                // 16-byte chunks per code row
  static constexpr int CPC = 128 / BITS;             // codes per 16-byte chunk
  static constexpr int NG = D / GS;
  static constexpr int NMETA = Q8 ? 2 : 4;           // scale (and bias) arrays of K and V
  static constexpr int META_BYTES = ((kPfRawKeys * NG * 2 + 127) / 128) * 128;
  // shared memory (1024-byte aligned operand slots)
  static constexpr int KV_BYTES = kPfBN * D * 2;     // D/64 blocks of [64 keys][128 B]
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + kPfKSlots * KV_BYTES;
  static constexpr int RAW_CODES = kPfRawKeys * RB;
  static constexpr int RAW_BYTES = 2 * RAW_CODES + NMETA * META_BYTES;
  static constexpr int RAW_OFF = V_OFF + kPfVSlots * KV_BYTES;
  static constexpr int BAR_OFF = RAW_OFF + kPfRawSlots * RAW_BYTES;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;  // + barriers, TMEM slot, alignment slack
  // TMEM columns: O, S[2] (P of a tile overwrites the first half of its S), Q (fp16 pairs)
  static constexpr int O_COL = 0;
  static constexpr int S_COL = D;
  static constexpr int Q_COL = S_COL + 2 * kPfBN;
  static constexpr int COLS = Q_COL + D / 2;
  static constexpr int TMEM_COLS = COLS <= 128 ? 128 : (COLS <= 256 ? 256 : 512);
  static_assert(COLS <= 512, "TMEM budget");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(RAW_BYTES % 128 == 0 && KV_BYTES % 1024 == 0, "slot alignment");
  static_assert((kPfRawKeys * UPR) % 32 == 0, "whole warps of chunks");
};

// ---- tcgen05 / mbarrier / bulk-copy wrappers -------------------------------
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
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t addr, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}\n"
               :: "r"(addr), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t addr, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(done) : "r"(addr), "r"(parity) : "memory");
  return done != 0;
}
__device__ __forceinline__ uint64_t pf_now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait for the phase with the given parity (at most limit_ns of the
// global timer).  Returns at once (false) if the CTA has already given up; on
// a time-out it records the error and makes the CTA give up.
__device__ __forceinline__ bool mbar_wait(uint32_t addr, uint32_t parity, volatile int* abort_flag,
                                          unsigned* status, unsigned code, uint64_t limit_ns) {
  if (mbar_try(addr, parity)) return true;
  const uint64_t t0 = pf_now_ns();
  for (;;) {
    if (mbar_try(addr, parity)) return true;
    if (*abort_flag) return false;
    if (pf_now_ns() - t0 > limit_ns) break;
  }
  *abort_flag = 1;
  atomicOr(status, code);
  return false;
}
// Bounded wait that ignores an earlier give-up: used before exit for the
// CTA's own asynchronous work still in flight.
__device__ __forceinline__ void mbar_drain(uint32_t addr, uint32_t parity, unsigned* status,
                                           uint64_t limit_ns) {
  const uint64_t t0 = pf_now_ns();
  for (;;) {
    if (mbar_try(addr, parity)) return;
    if (pf_now_ns() - t0 > limit_ns) break;
  }
  atomicOr(status, 128u);
}
// Per-tile range exponents, published by the producer warp in a ring of 8
// words of shared memory: ((t + 1) << 10) | (eK << 5) | eV for tile t.  The
// tag makes every entry self-identifying (no phase to track); the producer is
// never more than a few tiles ahead of the slowest reader.  Bounded wait that
// returns -1 on a give-up (and records a time-out like mbar_wait).
constexpr int kPfRangeRing = 8;
__device__ __forceinline__ int pf_range_get(const volatile uint32_t* ring, int t,
                                            volatile int* abort_flag, unsigned* status,
                                            uint64_t limit_ns) {
  const uint32_t want = (uint32_t)(t + 1) & 0x3fffffu;
  uint64_t t0 = 0;
  for (unsigned i = 0;; ++i) {
    const uint32_t v = ring[t & (kPfRangeRing - 1)];
    if ((v >> 10) == want) return (int)(v & 1023u);
    if (*abort_flag) return -1;
    if (i == 256) t0 = pf_now_ns();            // normally published a tile ahead: rare
    if (i >= 256) {
      __nanosleep(64);
      if (pf_now_ns() - t0 > limit_ns) break;
    }
  }
  *abort_flag = 1;
  atomicOr(status, 256u);
  return -1;
}
// Exponent e >= 0 such that a tile whose values are bounded by `bound` fits
// below 2^15 once multiplied by 2^-e (0 for bounds below 2^15).
__device__ __forceinline__ int pf_range_exp(float bound) {
  const int ex = (int)((__float_as_uint(bound) >> 23) & 0xff) - 127;   // floor(log2 bound)
  return min(31, max(0, ex - 14));
}

// Cache-line prefetches of global memory (no data returned, no fault).
__device__ __forceinline__ void prefetch_l1(const void* a) {
  asm volatile("prefetch.global.L1 [%0];\n" :: "l"(a));
}
__device__ __forceinline__ void prefetch_l2(const void* a) {
  asm volatile("prefetch.global.L2 [%0];\n" :: "l"(a));
}

// One contiguous global -> shared copy completing on an mbarrier (no multicast).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
      :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n"
               :: "r"(bar) : "memory");
}
// D(tmem) (+)= A(tmem) * B(smem desc), kind::f16 with fp32 accumulate.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}\n"
      :: "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate),
         "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
// Shared-memory matrix descriptor with 128-byte swizzled rows: `sbo` = bytes
// between 8-row groups, `lbo` = bytes between 64-element column blocks (used
// by MN-major operands only).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3fff);          // start address
  d |= (uint64_t)((lbo >> 4) & 0x3fff) << 16;      // leading byte offset
  d |= (uint64_t)((sbo >> 4) & 0x3fff) << 32;      // stride byte offset
  d |= (uint64_t)1 << 46;                          // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                          // 128-byte swizzle
  return d;
}
// Instruction descriptor: f16 x f16 -> f32, A K-major, B K-major (or MN-major
// with b_mn), M x N.
__host__ __device__ constexpr uint32_t f16_idesc(int M, int N, bool b_mn) {
  return (1u << 4) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// 32 consecutive 32-bit columns of this thread's TMEM lane (warp-collective).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n"
      :: "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]),
         "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]),
         "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]),
         "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]),
         "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};\n"
      :: "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]),
         "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]),
         "r"(v[13]), "r"(v[14]), "r"(v[15])
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

// Byte offset of 16-bit element (row, col) in a tile of 64-row blocks with
// 128-byte swizzled rows (64 columns per block).
__device__ __forceinline__ int sw128_off(int row, int col) {
  const int blk = col >> 6, chunk = (col >> 3) & 7;
  return blk * kPfBN * 128 + row * 128 + ((chunk ^ (row & 7)) << 4) + (col & 7) * 2;
}

// Position of head-dimension element e inside a K/V row.  The 4-bit codes of
// a 32-bit word come out of the mask-and-magic conversion as the pairs (0,4),
// (1,5), (2,6), (3,7); Q is stored with the same permutation so Q K^T is
// unchanged, and the output columns of P V are put back in the epilogue.
// 8-bit codes come out in natural order.
template <int BITS>
__host__ __device__ constexpr int k_pos(int e) {
  if constexpr (BITS == 4) {
    return (e & ~7) | ((e & 3) << 1) | ((e & 7) >> 2);
  } else {
    return e;
  }
}

// Converts one 16-byte chunk of codes (16 codes of 8 bits or 32 of 4 bits,
// all in one group) of key row `row`, chunk index u of the row, to fp16 in the
// 128-byte swizzled [key][d] tile: value = scale * code + bias rounded once.
template <int D, int BITS, int GS, bool Q8>
__device__ __forceinline__ void pf_convert_chunk(uint4 w4, __half2 s2, __half2 b2, uint8_t* dst,
                                                 int row, int u) {
  const __half2 off = __float2half2_rn(Q8 ? 1152.f : 1024.f);   // Q8 codes are stored +128
  const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
  if constexpr (BITS == 8) {
    uint32_t o[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t x = Q8 ? (wv[k] ^ 0x80808080u) : wv[k];
      const uint32_t h0 = prmt(x, 0x64646464u, 0x4140u);   // (1024 + byte0, 1024 + byte1)
      const uint32_t h1 = prmt(x, 0x64646464u, 0x4342u);
      const __half2 v0 = __hfma2(__hsub2(*reinterpret_cast<const __half2*>(&h0), off), s2, b2);
      const __half2 v1 = __hfma2(__hsub2(*reinterpret_cast<const __half2*>(&h1), off), s2, b2);
      o[2 * k] = *reinterpret_cast<const uint32_t*>(&v0);
      o[2 * k + 1] = *reinterpret_cast<const uint32_t*>(&v1);
    }
    *reinterpret_cast<uint4*>(dst + sw128_off(row, u * 16)) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4*>(dst + sw128_off(row, u * 16 + 8)) = make_uint4(o[4], o[5], o[6], o[7]);
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) {      // word k: d = 32u + 8k .. +7, nibbles (j, j+4) -> (2j, 2j+1)
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t x = ((wv[k] >> (4 * j)) & 0x000F000Fu) | 0x64006400u;
        const __half2 v = __hfma2(__hsub2(*reinterpret_cast<const __half2*>(&x), off), s2, b2);
        o[j] = *reinterpret_cast<const uint32_t*>(&v);
      }
      *reinterpret_cast<uint4*>(dst + sw128_off(row, u * 32 + 8 * k)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// A thread's share of one 64-key operand tile (K or V): its 16-byte code
// chunks of both packed half tiles with their scale and bias, loaded from the
// raw ring ahead of the conversion.  raw[h]: the half tile's slot; codes at
// +codes_off, scales at +sc_off, biases at +bi_off; rows at or past nv[h]
// (keys past L) get scale and bias 0, hence zeros.
template <int D, int BITS, int GS, bool Q8>
struct PfChunks {
  using C = PfCfg<D, BITS, GS, Q8>;
  static constexpr int NCH = kPfRawKeys * C::UPR;
  static constexpr int ITERS = (NCH + kPfDqThreads - 1) / kPfDqThreads;
  uint4 w[2][ITERS];
  __half2 s2[2][ITERS], b2[2][ITERS];

  __device__ __forceinline__ static bool has(int chunk0, int it) {
    return NCH % kPfDqThreads == 0 || chunk0 + it * kPfDqThreads < NCH;   // whole warps
  }
  // e > 0: scale and bias multiplied by 2^-e (exact power of two), so the
  // converted values stay below 2^15 (see the range note above)
  __device__ __forceinline__ void load(const uint8_t* const raw[2], int codes_off, int sc_off,
                                       int bi_off, const int nv[2], int chunk0, int e) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int it = 0; it < ITERS; ++it) {
        if (!has(chunk0, it)) continue;
        const int i = chunk0 + it * kPfDqThreads;
        const int key = i / C::UPR, u = i - key * C::UPR;
        const int g = (u * C::CPC) / GS;
        const bool live = key < nv[h];
        const uint16_t* sc = reinterpret_cast<const uint16_t*>(raw[h] + sc_off);
        const uint16_t* bi = reinterpret_cast<const uint16_t*>(raw[h] + bi_off);
        w[h][it] = *reinterpret_cast<const uint4*>(raw[h] + codes_off + i * 16);
        s2[h][it] = __half2half2(__ushort_as_half(live ? sc[key * C::NG + g] : (uint16_t)0));
        b2[h][it] = Q8 ? __float2half2_rn(0.f)
                       : __half2half2(__ushort_as_half(live ? bi[key * C::NG + g] : (uint16_t)0));
      }
    }
    if (e != 0) {
      const __half2 f = __float2half2_rn(exp2i(-e));
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int it = 0; it < ITERS; ++it) {
          s2[h][it] = __hmul2(s2[h][it], f);
          b2[h][it] = __hmul2(b2[h][it], f);
        }
    }
  }
  __device__ __forceinline__ void store(uint8_t* dst, int chunk0) const {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int it = 0; it < ITERS; ++it) {
        if (!has(chunk0, it)) continue;
        const int i = chunk0 + it * kPfDqThreads;
        const int key = i / C::UPR, u = i - key * C::UPR;
        pf_convert_chunk<D, BITS, GS, Q8>(w[h][it], s2[h][it], b2[h][it], dst, h * kPfRawKeys + key, u);
      }
    }
  }
};

// Adds slope * mask[j] to the base-2 logits sv[j] of one tile row for j < lim
// (the others are -inf already and read nothing); a -inf mask entry hides the
// key.  Each thread reads its own row, so the reads go 16 bytes at a time when
// the row is 16-byte aligned (scalar reads for the row's ragged end and for
// unaligned rows), without branches around them; they go out 16 elements at a
// time (the compiler barrier between the groups keeps it from hoisting all of
// them, which would not fit the registers next to the tile).
__device__ __forceinline__ void pf_unpack(uint4 r, const float*, float* o) {
  o[0] = __uint_as_float(r.x); o[1] = __uint_as_float(r.y);
  o[2] = __uint_as_float(r.z); o[3] = __uint_as_float(r.w);
}
__device__ __forceinline__ void pf_unpack(uint4 r, const __half*, float* o) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = unpack_half2(w[i]);
    o[2 * i] = f.x; o[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void pf_unpack(uint4 r, const __nv_bfloat16*, float* o) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = __uint_as_float(w[i] << 16);
    o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// The common case of pf_add_mask (mask instance), taken when every key of the
// tile is visible to every row of the warp and the slope is positive: sv[j]
// (raw products) becomes rs * sv[j] + slope * mask[j] in two operations, with
// no per-key selects (a -inf mask entry still gives -inf: slope * -inf is
// -inf and the products are finite).
template <typename T>
__device__ __forceinline__ void pf_scale_add_mask(float (&sv)[kPfBN], const T* m, float rs, float slope) {
  constexpr int EPV = 16 / (int)sizeof(T);              // elements per 16-byte read
  const bool vec = (reinterpret_cast<uintptr_t>(m) & 15u) == 0;
#pragma unroll
  for (int c = 0; c < kPfBN; c += 16) {
#pragma unroll
    for (int v = c; v < c + 16; v += EPV) {
      float mv[EPV];
      if (vec) {
        pf_unpack(__ldg(reinterpret_cast<const uint4*>(m + v)), m, mv);
      } else {
#pragma unroll
        for (int e = 0; e < EPV; ++e) mv[e] = to_float_ld(m + v + e);
      }
#pragma unroll
      for (int e = 0; e < EPV; ++e) sv[v + e] = fmaf(sv[v + e], rs, slope * mv[e]);
    }
    asm volatile("" ::: "memory");
  }
}

template <typename T>
__device__ __forceinline__ void pf_add_mask(float (&sv)[kPfBN], const T* m, int lim, float slope) {
  constexpr int EPV = 16 / (int)sizeof(T);              // elements per 16-byte read
  const bool vec = (reinterpret_cast<uintptr_t>(m) & 15u) == 0;
#pragma unroll
  for (int c = 0; c < kPfBN; c += 16) {
#pragma unroll
    for (int v = c; v < c + 16; v += EPV) {
      float mv[EPV];
      if (vec && v + EPV <= lim) {
        pf_unpack(__ldg(reinterpret_cast<const uint4*>(m + v)), m, mv);
      } else {
#pragma unroll
        for (int e = 0; e < EPV; ++e) mv[e] = v + e < lim ? to_float_ld(m + v + e) : 0.f;
      }
#pragma unroll
      for (int e = 0; e < EPV; ++e)
        sv[v + e] = mv[e] == -INFINITY ? -INFINITY : fmaf(slope, mv[e], sv[v + e]);
    }
    asm volatile("" ::: "memory");
  }
}

// VAR: kPfPlain; kPfExt, the instance with the attention extensions (logit
// softcap, additive-mask slopes, sinks), which the plain instance carries no
// code for; kPfMask, the one for additive masks (with or without slopes) and
// no other extension, which reads each tile's mask in one pass with the
// scaling of S and fetches the next tiles' entries ahead.  RANGE: the second
// instance of a call (see the range note above).
enum : int { kPfPlain = 0, kPfExt = 1, kPfMask = 2 };
template <int D, int BITS, int GS, bool Q8, int VAR, bool RANGE>
__global__ void __launch_bounds__(kPfThreads, 1) qsdpa_prefill_tc_kernel(const PrefillParams p) {
  constexpr bool EXT = VAR == kPfExt;
  constexpr bool AMASK = VAR == kPfMask;
  using C = PfCfg<D, BITS, GS, Q8>;
  constexpr int NG = C::NG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint64_t wait_ns = p.wait_ns != 0 ? p.wait_ns : kPfWaitNs;
  const uint32_t bar0 = sbase + C::BAR_OFF;
  constexpr uint32_t RO = 8 * kPfRawSlots;                    // barriers after the raw ones
  auto raw_full = [&](int i) { return bar0 + 8 * i; };        // [raw slots] packed half tile landed
  auto k_ready = [&](int i) { return bar0 + RO + 8 * i; };    // [2] fp16 K written
  auto v_ready = [&](int i) { return bar0 + RO + 16 + 8 * i; };   // [2] fp16 V written
  auto s_full = [&](int i) { return bar0 + RO + 32 + 8 * i; };    // [2] S in TMEM
  auto p_ready = [&](int i) { return bar0 + RO + 48 + 8 * i; };   // [2] P in TMEM
  auto pv_done = [&](int i) { return bar0 + RO + 64 + 8 * i; };   // [2] P V product done
  const uint32_t mma_done = bar0 + RO + 80;                   // all tensor-core work done
  auto raw_free = [&](int i) { return bar0 + RO + 88 + 8 * i; };  // [2] a tile's raw slots released
  {
    // the range flag was written by the range check kernel, two kernels
    // earlier in the stream: the first instance runs when it is down, the
    // second when it is up.  Every CTA of the second instance counts itself
    // done at exit; the last one lowers the flag and the count for the next
    // call.
    __shared__ int s_run;
    if (tid == 0) s_run = (*reinterpret_cast<volatile unsigned*>(p.range) != 0u) == RANGE;
    __syncthreads();
    const bool run = s_run != 0;
    __syncthreads();
    if (!run) {
      if (RANGE && tid == 0 && atomicAdd(p.range + 1, 1u) + 1 == gridDim.x) {
        p.range[1] = 0u;
        p.range[0] = 0u;
      }
      return;
    }
  }
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::BAR_OFF + RO + 112);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::BAR_OFF + RO + 116);
  volatile uint32_t* range_ring = reinterpret_cast<volatile uint32_t*>(smem + C::BAR_OFF + RO + 128);
  static_assert(8 * kPfRawSlots + 128 + 4 * kPfRangeRing <= 256, "barrier area");

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
  const int nhalves = kend > 0 ? (int)((kend + kPfRawKeys - 1) / kPfRawKeys) : 0;

  if (warp == kPfMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n"
                 :: "r"(smem_u32(tmem_slot)), "r"(C::TMEM_COLS) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  if (tid == 0) {
    for (int i = 0; i < kPfRawSlots; ++i) mbar_init(raw_full(i), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(k_ready(i), kPfDqThreads);
      mbar_init(v_ready(i), kPfDqThreads);
      mbar_init(s_full(i), 1);
      mbar_init(p_ready(i), kPfSoftThreads);
      mbar_init(pv_done(i), 1);
    }
    mbar_init(mma_done, 1);
    mbar_init(raw_free(0), kPfDqThreads);
    mbar_init(raw_free(1), kPfDqThreads);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    *abort_flag = 0;
    for (int i = 0; i < kPfRangeRing; ++i) range_ring[i] = 0u;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t row0 = ((int64_t)b * p.Hkv + hkv) * p.Lcap;

  // softmax threads: row r = TMEM lane
  const int quarter = warp & 3;
  const int r = mt * kPfBM + quarter * 32 + lane;
  const bool row_ok = warp < kPfSoftWarps && r < R;
  const int qi = row_ok ? r / p.G : 0;
  const int hh = row_ok ? r - qi * p.G : 0;
  const int64_t qrow = (((int64_t)b * p.Hq + (int64_t)hkv * p.G + hh) * p.Lq + qi) * D;
  const uint32_t tmem_row = tmem + ((uint32_t)(quarter * 32) << 16);

  // dequant warps: packed half-tile sources
  const int dq = tid - kPfSoftThreads;
  const uint8_t* gK = p.kc + row0 * C::RB;
  const uint8_t* gV = p.vc + row0 * C::RB;
  int issued = 0;                                // half tiles whose bulk copies were issued
  // The bulk copies of half tiles i0 .. i0+n-1 (n <= 2), issued by the 32
  // lanes of the producer warp: lane 0 first registers the byte counts on
  // the slots' mbarriers, then every lane issues at most one copy.
  constexpr int CPH = 2 + C::NMETA;              // copies per half tile
  auto issue_raw = [&](int i0, int n) {
    issued += n;
    if (lane == 0) {
      for (int k = 0; k < n; ++k) {
        const int i = i0 + k;
        if (i == p.stall_half) continue;         // test hook: this half tile never lands
        const int64_t key0 = (int64_t)i * kPfRawKeys;
        const int nv = L - key0 < kPfRawKeys ? (int)(L - key0) : kPfRawKeys;
        const int nv8 = (nv + 7) & ~7;           // scale rows in whole 16-byte units
        mbar_arrive_expect_tx(raw_full(i % kPfRawSlots),
                              (uint32_t)(2 * nv * C::RB + C::NMETA * nv8 * NG * 2));
      }
    }
    __syncwarp();
    if (lane < n * CPH && i0 + lane / CPH != p.stall_half) {
      const int i = i0 + lane / CPH, which = lane % CPH;
      const int slot = i % kPfRawSlots;
      const int64_t key0 = (int64_t)i * kPfRawKeys;
      const int nv = L - key0 < kPfRawKeys ? (int)(L - key0) : kPfRawKeys;
      const int nv8 = (nv + 7) & ~7;
      const uint32_t cb = (uint32_t)(nv * C::RB), mb = (uint32_t)(nv8 * NG * 2);
      const uint32_t bar = raw_full(slot);
      const uint32_t dst = sbase + C::RAW_OFF + slot * C::RAW_BYTES;
      const int64_t m0 = (row0 + key0) * NG;
      if (which == 0) bulk_g2s(dst, gK + key0 * C::RB, cb, bar);
      else if (which == 1) bulk_g2s(dst + C::RAW_CODES, gV + key0 * C::RB, cb, bar);
      else {
        // metadata arrays in order: K scales, (K biases,) V scales, (V biases)
        const int arr = which - 2;
        const uint16_t* src = Q8 ? (arr == 0 ? p.ks : p.vs)
                                 : (arr == 0 ? p.ks : arr == 1 ? p.kb : arr == 2 ? p.vs : p.vb);
        bulk_g2s(dst + 2 * C::RAW_CODES + arr * C::META_BYTES, src + m0, mb, bar);
      }
    }
  };
  if (warp == kPfProdWarp) {
    const int n0 = nhalves < kPfRawSlots ? nhalves : kPfRawSlots;
    for (int i0 = 0; i0 < n0; i0 += 2) issue_raw(i0, n0 - i0 < 2 ? n0 - i0 : 2);
  }

  // ---- Q rows -> fp16 (per-row power-of-two prescale) in TMEM ----------------
  float rowscale = 0.f;
  if (warp < kPfSoftWarps) {
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
    {
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 64) {       // 64 elements = 32 TMEM columns
        uint32_t qw[32];
#pragma unroll
        for (int e8 = 0; e8 < 64; e8 += 8) {
          uint32_t w[4] = {0u, 0u, 0u, 0u};
          if (row_ok) {
            const uint4 raw = *reinterpret_cast<const uint4*>(
                reinterpret_cast<const uint16_t*>(p.q) + qrow + c0 + e8);
            w[0] = raw.x; w[1] = raw.y; w[2] = raw.z; w[3] = raw.w;
          }
          float v[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint16_t bits = (uint16_t)(w[k >> 1] >> (16 * (k & 1)));
            v[k] = (p.q_dtype == QKV_F16 ? __half2float(__ushort_as_half(bits))
                                         : __uint_as_float((uint32_t)bits << 16)) * up;
          }
          float sq[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) sq[k_pos<BITS>(k)] = v[k];
#pragma unroll
          for (int k = 0; k < 4; ++k) qw[e8 / 2 + k] = pack_half2(sq[2 * k], sq[2 * k + 1]);
        }
        tmem_st32(tmem_row + C::Q_COL + c0 / 2, qw);
      }
      tmem_wait_st();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp >= kPfSoftWarps && warp < kPfMmaWarp) {
    // ======================= dequant warps =====================================
    int cl = 0;
#pragma unroll
    for (int bt = 0; bt < 5; ++bt)
      if ((lane >> bt) & 1) cl ^= pf_lane_col(D, BITS, bt);
    const int chunk0 = (dq >> 5) * 32 + cl;
    // the tile's two packed half tiles; a half tile past the last one gives
    // zeros (its keys are never visible)
    for (int t = 0; t < ntiles; ++t) {
      const int s = t & 1;
      const uint8_t* raw[2];
      int nv[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int i = 2 * t + h;
        const bool present = i < nhalves;
        const int slot = i % kPfRawSlots;
        if (present) mbar_wait(raw_full(slot), (i / kPfRawSlots) & 1, abort_flag, p.status, 1u, wait_ns);
        raw[h] = smem + C::RAW_OFF + slot * C::RAW_BYTES;
        const int64_t key0 = (int64_t)i * kPfRawKeys;
        nv[h] = !present ? 0 : (L - key0 < kPfRawKeys ? (int)(L - key0) : kPfRawKeys);
      }
      // the tile's range exponents (second instance only)
      int eK = 0, eV = 0;
      if constexpr (RANGE) {
        const int rg = pf_range_get(range_ring, t, abort_flag, p.status, wait_ns);
        eK = rg < 0 ? 0 : rg >> 5;
        eV = rg < 0 ? 0 : rg & 31;
      }
      // K and V chunks of this thread come in together; V converts after K
      PfChunks<D, BITS, GS, Q8> kch, vch;
      kch.load(raw, 0, 2 * C::RAW_CODES, 2 * C::RAW_CODES + C::META_BYTES, nv, chunk0, eK);
      vch.load(raw, C::RAW_CODES, 2 * C::RAW_CODES + (Q8 ? 1 : 2) * C::META_BYTES,
               2 * C::RAW_CODES + 3 * C::META_BYTES, nv, chunk0, eV);
      if (t >= kPfKSlots)                        // K slot free once S of tile t-2 is done
        mbar_wait(s_full(s), ((t - 2) >> 1) & 1, abort_flag, p.status, 1u, wait_ns);
      kch.store(smem + C::K_OFF + s * C::KV_BYTES, chunk0);
      fence_async_smem();
      mbar_arrive(k_ready(s));
      mbar_arrive(raw_free(s));                  // this thread is done with the raw slots
      if (t >= kPfVSlots)                        // V slot free once P V of tile t-2 is done
        mbar_wait(pv_done(s), ((t - 2) >> 1) & 1, abort_flag, p.status, 1u, wait_ns);
      vch.store(smem + C::V_OFF + s * C::KV_BYTES, chunk0);
      fence_async_smem();
      mbar_arrive(v_ready(s));
    }
  } else if (warp == kPfProdWarp) {
    // ======================= producer warp =====================================
    if constexpr (!RANGE) {
    for (int t = 0; t + 2 < ntiles || 2 * t + kPfRawSlots < nhalves; ++t) {
      const int i0 = 2 * t + kPfRawSlots;
      if (i0 >= nhalves) break;
      mbar_wait(raw_free(t & 1), (t >> 1) & 1, abort_flag, p.status, 1u, wait_ns);
      // warp-uniform decision (issue_raw synchronizes the warp)
      if (__shfl_sync(~0u, (int)*abort_flag, 0) != 0) break;
      issue_raw(i0, nhalves - i0 < 2 ? nhalves - i0 : 2);
    }
    } else {
    // Range exponents: the warp reads tile t + 2's scales (and biases)
    // straight from global memory while it waits to refill the raw slots of
    // tile t, and publishes the tile's exponents after that refill -- a tile
    // and more before the dequant warps need them -- then starts the reads
    // for tile t + 3.  Tiles 0 and 1 are published before the loop.
    constexpr float kCodeMax = Q8 ? 128.f : (float)((1 << BITS) - 1);   // largest |code|
    constexpr int U4 = kPfBN * NG * 2 / 16;      // 16-byte units of one metadata array of a tile
    constexpr int PER = (U4 + 31) / 32;          // per lane
    uint4 fm[C::NMETA][PER];                     // metadata of the tile in flight
    int eV = 0;                                  // largest V exponent so far
    auto fetch = [&](int t) {
      const int64_t key0 = (int64_t)t * kPfBN;
      const int nvt = L - key0 < kPfBN ? (int)(L - key0) : kPfBN;
#pragma unroll
      for (int a = 0; a < C::NMETA; ++a) {
        // arrays in stage order: K scales, (K biases,) V scales, (V biases)
        const uint16_t* m = Q8 ? (a == 0 ? p.ks : p.vs)
                               : (a == 0 ? p.ks : a == 1 ? p.kb : a == 2 ? p.vs : p.vb);
        const uint4* src = reinterpret_cast<const uint4*>(m + (row0 + key0) * NG);
#pragma unroll
        for (int k = 0; k < PER; ++k) {
          const int i = lane + 32 * k;             // unit i holds keys from i * 8 / NG on
          fm[a][k] = (i < U4 && i * 8 / NG < nvt) ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
        }
      }
    };
    auto finish = [&](int t) {
      const int64_t key0 = (int64_t)t * kPfBN;
      const int nvt = L - key0 < kPfBN ? (int)(L - key0) : kPfBN;
      float bk = 0.f, bv = 0.f;                  // bounds of |scale * code + bias|
#pragma unroll
      for (int k = 0; k < PER; ++k) {
        const int i = lane + 32 * k;
        const uint32_t* ks = reinterpret_cast<const uint32_t*>(&fm[0][k]);
        const uint32_t* vs = reinterpret_cast<const uint32_t*>(&fm[Q8 ? 1 : 2][k]);
        const uint32_t* kb = reinterpret_cast<const uint32_t*>(&fm[Q8 ? 0 : 1][k]);
        const uint32_t* vb = reinterpret_cast<const uint32_t*>(&fm[Q8 ? 1 : 3][k]);
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          if (i >= U4 || (i * 8 + h) / NG >= nvt) continue;
          const int sh = 16 * (h & 1);
          const float sk = fabsf(half_bits_to_float((uint16_t)(ks[h >> 1] >> sh)));
          const float sv = fabsf(half_bits_to_float((uint16_t)(vs[h >> 1] >> sh)));
          const float ak = Q8 ? 0.f : fabsf(half_bits_to_float((uint16_t)(kb[h >> 1] >> sh)));
          const float av = Q8 ? 0.f : fabsf(half_bits_to_float((uint16_t)(vb[h >> 1] >> sh)));
          bk = fmaxf(bk, fmaf(sk, kCodeMax, ak));
          bv = fmaxf(bv, fmaf(sv, kCodeMax, av));
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        bk = fmaxf(bk, __shfl_xor_sync(~0u, bk, off));
        bv = fmaxf(bv, __shfl_xor_sync(~0u, bv, off));
      }
      eV = max(eV, pf_range_exp(bv));
      if (lane == 0)
        range_ring[t & (kPfRangeRing - 1)] =
            (((uint32_t)(t + 1) & 0x3fffffu) << 10) | ((uint32_t)pf_range_exp(bk) << 5) | (uint32_t)eV;
    };
    for (int t = 0; t < 2 && t < ntiles; ++t) { fetch(t); finish(t); }
    if (2 < ntiles) fetch(2);
    for (int t = 0; t < ntiles; ++t) {
      const int i0 = 2 * t + kPfRawSlots;
      if (i0 < nhalves) {
        mbar_wait(raw_free(t & 1), (t >> 1) & 1, abort_flag, p.status, 1u, wait_ns);
        // warp-uniform decision (issue_raw synchronizes the warp)
        if (__shfl_sync(~0u, (int)*abort_flag, 0) != 0) break;
        issue_raw(i0, nhalves - i0 < 2 ? nhalves - i0 : 2);
      }
      // tile t + 2's metadata was fetched before the wait above: no stall here
      if (t + 2 < ntiles) finish(t + 2);
      if (t + 3 < ntiles) fetch(t + 3);
    }
    }
    if (lane == 0) {                             // own bulk copies still in flight (after a give-up)
      for (int i = max(0, issued - kPfRawSlots); i < issued; ++i)
        mbar_drain(raw_full(i % kPfRawSlots), (i / kPfRawSlots) & 1, p.status, wait_ns);
    }
    __syncwarp();
  } else if (warp == kPfMmaWarp) {
    // ======================= MMA warp ==========================================
    constexpr uint32_t idesc_s = f16_idesc(kPfBM, kPfBN, false);
    constexpr uint32_t idesc_o = f16_idesc(kPfBM, D, true);
    auto issue_s = [&](int t) {
      const int s = t & 1;
      mbar_wait(k_ready(s), (t >> 1) & 1, abort_flag, p.status, 2u, wait_ns);
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint64_t bd = umma_desc_sw128(
              sbase + C::K_OFF + s * C::KV_BYTES + (k >> 2) * kPfBN * 128 + (k & 3) * 32, 16, 1024);
          tc_mma_ts(tmem + C::S_COL + s * kPfBN, tmem + C::Q_COL + k * 8, bd, idesc_s,
                    k > 0 ? 1u : 0u);
        }
        tc_commit(s_full(s));
      }
      __syncwarp();
    };
    auto issue_pv = [&](int t) {
      const int s = t & 1;
      mbar_wait(v_ready(s), (t >> 1) & 1, abort_flag, p.status, 4u, wait_ns);
      mbar_wait(p_ready(s), (t >> 1) & 1, abort_flag, p.status, 4u, wait_ns);
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int k = 0; k < kPfBN / 16; ++k) {
          const uint64_t bd = umma_desc_sw128(sbase + C::V_OFF + s * C::KV_BYTES + k * 16 * 128,
                                              kPfBN * 128, 1024);
          // P of tile t: fp16 pairs in the first half of its S columns
          tc_mma_ts(tmem + C::O_COL, tmem + C::S_COL + s * kPfBN + k * 8, bd, idesc_o,
                    (t > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(pv_done(s));
      }
      __syncwarp();
    };
    // S(t+2) reuses the columns of S(t) and P(t): it is issued after P V of
    // tile t, and the tensor core executes one thread's operations in order
    if (ntiles > 0) issue_s(0);
    if (ntiles > 1) issue_s(1);
    for (int t = 0; t < ntiles; ++t) {
      issue_pv(t);
      if (t + 2 < ntiles) issue_s(t + 2);
    }
    if (lane == 0) {                             // every MMA issued above has completed
      tc_commit(mma_done);
      mbar_drain(mma_done, 0, p.status, wait_ns);
    }
    __syncwarp();
  } else {
    // ======================= softmax warps (one row per thread) =================
    const int64_t causal_lim = L - p.Lq + qi;    // last visible key of this row
    const bool causal = p.mask_kind == QKV_MASK_CAUSAL;
    const bool additive = p.mask_kind == QKV_MASK_ADDITIVE;
    const bool capped = EXT && p.cap_a > 0.f;    // logit softcap
    const float slope = kLog2e * ((EXT || AMASK) && additive && p.slopes != nullptr && row_ok
                                      ? p.slopes[hkv * p.G + hh] : 1.f);
    float m_used = -INFINITY, lsum = 0.f;
    // additive mask: this row's entries, mbase + key (elements of esz bytes)
    const int64_t mbase = (int64_t)b * p.msb + ((int64_t)hkv * p.G + hh) * p.msh + (int64_t)qi * p.msq;
    for (int t = 0; t < ntiles; ++t) {
      const int s = t & 1;
      const int64_t key0 = (int64_t)t * kPfBN;
      if constexpr (AMASK) {
        if (additive && row_ok) {
          // the row's mask entries of the next tile into L1 and of the one
          // after into L2 while this tile's S is computed (keys below L only,
          // so every address lies in the row)
          const int esz = p.mask_dtype == QKV_F32 ? 4 : 2;
          const char* mr = static_cast<const char*>(p.mask) + (mbase + key0) * esz;
          if (key0 + kPfBN < kend) prefetch_l1(mr + kPfBN * esz);
          if (key0 + kPfBN + 128 / esz < kend) prefetch_l1(mr + kPfBN * esz + 128);
          if (key0 + 2 * kPfBN < kend) prefetch_l2(mr + 2 * kPfBN * esz);
          if (key0 + 2 * kPfBN + 128 / esz < kend) prefetch_l2(mr + 2 * kPfBN * esz + 128);
        }
      }
      mbar_wait(s_full(s), (t >> 1) & 1, abort_flag, p.status, 8u, wait_ns);
      tc_fence_after();
      // second instance: S of this tile was computed from K * 2^-eK: scale it
      // back (the ring still holds tile t - 1's entry: the producer is never
      // more than a few tiles ahead of this role)
      int eK = 0, dV = 0;
      if constexpr (RANGE) {
        const int rg = pf_range_get(range_ring, t, abort_flag, p.status, wait_ns);
        eK = rg < 0 ? 0 : rg >> 5;
        dV = rg < 0 || t == 0 ? 0 : (rg & 31) - (int)(range_ring[(t - 1) & (kPfRangeRing - 1)] & 31u);
      }
      const float rs = eK == 0 ? rowscale : rowscale * exp2i(eK);
      float sv[kPfBN];
      tmem_ld32(tmem_row + C::S_COL + s * kPfBN, reinterpret_cast<uint32_t*>(sv));
      tmem_ld32(tmem_row + C::S_COL + s * kPfBN + 32, reinterpret_cast<uint32_t*>(sv + 32));
      tmem_wait_ld();
      // a tile without masked keys for any row of the warp takes the short path
      // (the tile maximum is taken over the raw products, which needs rowscale >= 0)
      const bool full = __all_sync(~0u, row_ok && !additive && rowscale >= 0.f &&
                                            key0 + kPfBN <= kend &&
                                            (!causal || key0 + kPfBN - 1 <= causal_lim));
      float tmax;
      if (full) {
        float m0 = fmaxf(sv[0], sv[1]), m1 = fmaxf(sv[2], sv[3]);
#pragma unroll
        for (int j = 4; j < kPfBN; j += 4) {
          m0 = fmaxf(m0, fmaxf(sv[j], sv[j + 1]));
          m1 = fmaxf(m1, fmaxf(sv[j + 2], sv[j + 3]));
        }
        tmax = fmaxf(m0, m1) * rs;
        if (capped) tmax = softcap_log2(tmax, p.cap_a, p.cap_k);   // the cap is increasing
      } else {
        // per-element path: keys j < lim of the tile are visible (below L and the
        // causal limit); then the additive mask, its loads all issued together
        int64_t nv = kend - key0;
        if (causal && causal_lim - key0 + 1 < nv) nv = causal_lim - key0 + 1;
        const int lim = !row_ok || nv <= 0 ? 0 : nv >= kPfBN ? kPfBN : (int)nv;
        if (AMASK && additive && __all_sync(~0u, lim == kPfBN && slope > 0.f)) {
          // every key visible to every row of the warp: scale and mask in one pass
          const int64_t mrow = mbase + key0;
          if (p.mask_dtype == QKV_F32)
            pf_scale_add_mask(sv, reinterpret_cast<const float*>(p.mask) + mrow, rs, slope);
          else if (p.mask_dtype == QKV_F16)
            pf_scale_add_mask(sv, reinterpret_cast<const __half*>(p.mask) + mrow, rs, slope);
          else
            pf_scale_add_mask(sv, reinterpret_cast<const __nv_bfloat16*>(p.mask) + mrow, rs, slope);
        } else {
#pragma unroll
        for (int j = 0; j < kPfBN; ++j) {
          float v = sv[j] * rs;
          if (capped) v = softcap_log2(v, p.cap_a, p.cap_k);
          sv[j] = j < lim ? v : -INFINITY;
        }
        if (additive) {
          const int64_t mrow = mbase + key0;
          if (p.mask_dtype == QKV_F32)
            pf_add_mask(sv, reinterpret_cast<const float*>(p.mask) + mrow, lim, slope);
          else if (p.mask_dtype == QKV_F16)
            pf_add_mask(sv, reinterpret_cast<const __half*>(p.mask) + mrow, lim, slope);
          else
            pf_add_mask(sv, reinterpret_cast<const __nv_bfloat16*>(p.mask) + mrow, lim, slope);
        }
        }
        float m0 = sv[0], m1 = sv[1];
#pragma unroll
        for (int j = 2; j < kPfBN; j += 2) { m0 = fmaxf(m0, sv[j]); m1 = fmaxf(m1, sv[j + 1]); }
        tmax = fmaxf(m0, m1);
      }
      float alpha = 1.f;
      if (tmax > m_used + 8.f) {
        // no earlier key was visible: O and l are still zero, nothing to rescale
        alpha = m_used == -INFINITY ? 1.f : ex2(m_used - tmax);
        m_used = tmax;
      }
      const float mref = m_used == -INFINITY ? 0.f : m_used;
      // O also takes the growth of the V exponent (its P V terms from here on
      // are computed from V * 2^-eV of this tile)
      const float alpha_o = dV > 0 ? alpha * exp2i(-dV) : alpha;
      const bool rescale = t > 0 && __any_sync(~0u, alpha_o != 1.f);
      if (rescale) {                             // needs P V of tile t-1 done (rare)
        mbar_wait(pv_done((t - 1) & 1), ((t - 1) >> 1) & 1, abort_flag, p.status, 32u, wait_ns);
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_ld32(tmem_row + C::O_COL + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha_o);
          tmem_st32(tmem_row + C::O_COL + c, o);
        }
      }
      // P (fp16 pairs) over the first half of this tile's S columns, which
      // this thread has already read
      float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t pk[16];
        if (full && capped) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a = ex2(softcap_log2(sv[32 * hf + 2 * i] * rs, p.cap_a, p.cap_k) - mref);
            const float c = ex2(softcap_log2(sv[32 * hf + 2 * i + 1] * rs, p.cap_a, p.cap_k) - mref);
            rs0 += a; rs1 += c;
            pk[i] = pack_half2(a, c);
          }
        } else if (full) {
          const float nm = -mref;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a = ex2(fmaf(sv[32 * hf + 2 * i], rs, nm));
            const float c = ex2(fmaf(sv[32 * hf + 2 * i + 1], rs, nm));
            rs0 += a; rs1 += c;
            pk[i] = pack_half2(a, c);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a = ex2(sv[32 * hf + 2 * i] - mref), c = ex2(sv[32 * hf + 2 * i + 1] - mref);
            rs0 += a; rs1 += c;
            pk[i] = pack_half2(a, c);
          }
        }
        tmem_st16(tmem_row + C::S_COL + s * kPfBN + 16 * hf, pk);
      }
      tmem_wait_st();
      lsum = lsum * alpha + (rs0 + rs1);
      tc_fence_before();
      mbar_arrive(p_ready(s));
    }
    // ---- epilogue: O / l -> out --------------------------------------------
    bool have = ntiles > 0;
    if (have) {
      have = mbar_wait(pv_done((ntiles - 1) & 1), ((ntiles - 1) >> 1) & 1, abort_flag, p.status, 64u, wait_ns);
      tc_fence_after();
    }
    have = __all_sync(~0u, have) && !*abort_flag;
    float fo = 1.f;
    if (EXT && p.sinks != nullptr && row_ok && lsum > 0.f) {
      // the head's sink logit joins the denominator (P, l and O are relative to m_used)
      const float s2 = kLog2e * p.sinks[hkv * p.G + hh];
      const float Mn = fmaxf(m_used, s2);
      fo = ex2(m_used - Mn);
      lsum = lsum * fo + ex2(s2 - Mn);
    }
    // O carries 2^-eV of the last tile (the largest V exponent)
    const int eVend = RANGE && ntiles > 0 ? (int)(range_ring[(ntiles - 1) & (kPfRangeRing - 1)] & 31u) : 0;
    const float inv = (lsum > 0.f && have) ? fo / lsum * exp2i(eVend) : 0.f;
#pragma unroll 1
    for (int c = 0; c < D; c += 32) {
      uint32_t ob[32];
      if (have) {
        tmem_ld32(tmem_row + C::O_COL + c, ob);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) ob[i] = 0u;
      }
      float o[32];                               // output order (undo the 4-bit pairing)
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = __uint_as_float(ob[k_pos<BITS>(i)]) * inv;
      if (row_ok) {
        if (p.out_dtype == QKV_BF16 || p.out_dtype == QKV_F16) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint32_t pq[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              if (p.out_dtype == QKV_F16) {
                pq[k] = pack_half2(o[i + 2 * k], o[i + 2 * k + 1]);
              } else {
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(o[i + 2 * k], o[i + 2 * k + 1]);
                pq[k] = *reinterpret_cast<const uint32_t*>(&h2);
              }
            }
            *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.out) + qrow + c + i) =
                make_uint4(pq[0], pq[1], pq[2], pq[3]);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) store_from_float(p.out, p.out_dtype, qrow + c + i, o[i]);
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
  if constexpr (RANGE) {
    if (tid == 0 && atomicAdd(p.range + 1, 1u) + 1 == gridDim.x) { p.range[1] = 0u; p.range[0] = 0u; }
  }
}

// The range check that precedes the prefill kernel's instances: every
// 16-byte unit of the K and V metadata rows [0, L) of every (batch, kv head)
// slab (8 fp16 values; the values of rows at or past L ignored); if some
// |scale| * (largest code) + |bias| reaches 2^15, the flag goes up.
template <bool Q8, int BITS>
__global__ void __launch_bounds__(256) qkv_range_check_kernel(const PrefillParams p, int ng) {
  constexpr float kCodeMax = Q8 ? 128.f : (float)((1 << BITS) - 1);
  const int64_t units = (p.L * ng + 7) / 8;                   // per slab and array
  const int64_t slab = blockIdx.y;
  const int64_t base = slab * p.Lcap * ng;                    // first element of the slab
  float bound = 0.f;
  for (int64_t u = (int64_t)blockIdx.x * 256 + threadIdx.x; u < units; u += (int64_t)gridDim.x * 256) {
    uint4 v[4];
    const uint16_t* arr[4] = {p.ks, Q8 ? p.ks : p.kb, p.vs, Q8 ? p.vs : p.vb};
#pragma unroll
    for (int a = 0; a < 4; ++a) v[a] = __ldg(reinterpret_cast<const uint4*>(arr[a] + base) + u);
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      if ((u * 8 + h) / ng >= p.L) break;
      const int sh = 16 * (h & 1);
      const uint32_t* w0 = reinterpret_cast<const uint32_t*>(&v[0]);
      const uint32_t* w1 = reinterpret_cast<const uint32_t*>(&v[1]);
      const uint32_t* w2 = reinterpret_cast<const uint32_t*>(&v[2]);
      const uint32_t* w3 = reinterpret_cast<const uint32_t*>(&v[3]);
      const float sk = fabsf(half_bits_to_float((uint16_t)(w0[h >> 1] >> sh)));
      const float sv = fabsf(half_bits_to_float((uint16_t)(w2[h >> 1] >> sh)));
      const float bk = Q8 ? 0.f : fabsf(half_bits_to_float((uint16_t)(w1[h >> 1] >> sh)));
      const float bv = Q8 ? 0.f : fabsf(half_bits_to_float((uint16_t)(w3[h >> 1] >> sh)));
      bound = fmaxf(bound, fmaxf(fmaf(sk, kCodeMax, bk), fmaf(sv, kCodeMax, bv)));
    }
  }
  // NaN counts as out of range too (the scaled path takes it like the rest)
  if (__any_sync(~0u, !(bound < 32768.f)) && (threadIdx.x & 31) == 0) atomicOr(p.range, 1u);
}

}  // namespace qkv
