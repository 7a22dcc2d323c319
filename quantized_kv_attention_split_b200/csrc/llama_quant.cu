// llama_quant.cu -- llama.cpp's Q4_0 / Q4_1 / Q5_0 / Q5_1 KV blocks written on
// the GPU: new tokens quantized into blocks (or straight into the affine cache
// rows that hold the same values), and affine cache rows written back out as
// blocks.
//
// The llama.cpp PR's follow-up extends its KV conversion to these block types
// (llama.cpp #25556, merged follow-up: "Q8_0/Q4_0/Q4_1/Q5_0/Q5_1"); the pages
// show neither their bytes nor their quantizers.  Bytes: the GGUF blocks of 32
// elements -- little-endian fp16 d (then fp16 m for the _1 types), then for Q5
// the 32 fifth bits qh (bit e for element e), then qs[16] with element j < 16
// in the low and element j + 16 in the high nibble of qs[j].  Quantizers: the
// published reference ones, per block of 32 in fp32:
//   _0: m = the element of largest magnitude (the first such), d = m / -8 (Q4)
//       or m / -16 (Q5), id = 1/d (0 if d == 0), q = min(15 | 31,
//       trunc(x id + 8.5 | 16.5));
//   _1: lo, hi = min, max; d = (hi - lo) / 15 (or 31), id = 1/d (0 if d == 0),
//       q = min(15 | 31, trunc((x - lo) id + 0.5)), m = lo;
// d (and m) stored as fp16 (round to nearest even), the codes computed from
// the fp32 d.  Each operation below is one IEEE fp32 operation with
// round-to-nearest (explicit intrinsics: no contraction into fused
// multiply-adds), in that order, so the blocks are bit-identical to the CPU
// oracle's.  One thread per block of 32 elements.
#include "qkv_common.cuh"
#include "qkv_internal.h"

namespace qkv {

struct LlamaQuantParams {
  const uint16_t* x;           // [B, Hkv, L, D] f16 / bf16 (quantize)
  int bf16;
  uint8_t* blocks;             // block bytes (quantize to blocks; export)
  int64_t sb, sh, sl;          // their byte strides (b, kv head, token)
  uint32_t* codes;             // affine cache (quantize into it; export from it)
  uint16_t* scales;
  uint16_t* biases;
  int64_t Lcap, offset;        // cache rows [offset, offset + L)
  int64_t L;
  int Hkv, nb;                 // kv heads, blocks per row (D / 32)
  int64_t total;               // B * Hkv * L * nb
};

__device__ __forceinline__ void llama_coords(const LlamaQuantParams& p, int64_t i, int nbytes,
                                             int64_t* xrow, int64_t* crow, int64_t* boff,
                                             int* g) {
  const int64_t rest = i / p.nb;
  *g = (int)(i - rest * p.nb);
  const int64_t bh = rest / p.L;
  const int64_t l = rest - bh * p.L;
  const int64_t b = bh / p.Hkv, h = bh - b * p.Hkv;
  *xrow = rest;                                          // row of x: (b, h, l)
  *crow = bh * p.Lcap + p.offset + l;                    // cache row
  *boff = b * p.sb + h * p.sh + l * p.sl + (int64_t)*g * nbytes;
}

// Reference quantizer of one block of 32 fp32 values: fp16 d and m bits and
// the 32 codes (OFF = 8 or 16 for the _0 types, 0 for the _1 types; TOP = 15
// or 31).
template <int OFF, int TOP>
__device__ __forceinline__ void llama_quantize32(const float (&x)[32], uint16_t* d16, uint16_t* m16,
                                                 uint32_t (&q)[32]) {
  float d, lo = 0.f;
  if constexpr (OFF != 0) {
    float amax = fabsf(x[0]), mval = x[0];
#pragma unroll
    for (int e = 1; e < 32; ++e) {
      const float a = fabsf(x[e]);
      if (a > amax) { amax = a; mval = x[e]; }            // first element of largest magnitude
    }
    d = __fdiv_rn(mval, -(float)OFF);
  } else {
    float hi = x[0];
    lo = x[0];
#pragma unroll
    for (int e = 1; e < 32; ++e) { lo = fminf(lo, x[e]); hi = fmaxf(hi, x[e]); }
    d = __fdiv_rn(__fsub_rn(hi, lo), (float)TOP);
  }
  const float id = d != 0.f ? __fdiv_rn(1.f, d) : 0.f;
  constexpr float kAdd = OFF != 0 ? (float)OFF + 0.5f : 0.5f;
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const float v = OFF != 0 ? x[e] : __fsub_rn(x[e], lo);
    const float t = __fadd_rn(__fmul_rn(v, id), kAdd);
    const uint32_t c = __float2uint_rz(t);                   // trunc of a non-negative value
    q[e] = c < (uint32_t)TOP ? c : (uint32_t)TOP;
  }
  *d16 = __half_as_ushort(__float2half_rn(d));
  *m16 = __half_as_ushort(__float2half_rn(lo));
}

// Writes one block's bytes (2-byte aligned) as 16-bit units.
template <int NBYTES, bool HAS_M, bool HAS_QH>
__device__ __forceinline__ void llama_store_block(uint8_t* dst8, uint16_t d16, uint16_t m16,
                                                  const uint32_t (&q)[32]) {
  uint16_t* dst = reinterpret_cast<uint16_t*>(dst8);
  int u = 0;
  dst[u++] = d16;
  if constexpr (HAS_M) dst[u++] = m16;
  if constexpr (HAS_QH) {
    uint32_t qh = 0u;
#pragma unroll
    for (int e = 0; e < 32; ++e) qh |= ((q[e] >> 4) & 1u) << e;
    dst[u++] = (uint16_t)(qh & 0xffffu);
    dst[u++] = (uint16_t)(qh >> 16);
  }
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    const uint32_t b0 = (q[j] & 0xfu) | ((q[j + 16] & 0xfu) << 4);
    const uint32_t b1 = (q[j + 1] & 0xfu) | ((q[j + 17] & 0xfu) << 4);
    dst[u++] = (uint16_t)(b0 | (b1 << 8));
  }
}

// TO_CACHE false: new rows of x -> blocks.  TO_CACHE true: new rows of x ->
// affine cache rows that hold the blocks' values exactly (scale d, bias m or
// -OFF d rounded to fp16 from the fp16 d, as the block import writes them;
// 4-bit codes for Q4, 8-bit codes for Q5).
template <int NBYTES, bool HAS_M, bool HAS_QH, int OFF, int BITS, bool TO_CACHE>
__global__ void __launch_bounds__(256) qkv_llama_quantize_kernel(const __grid_constant__ LlamaQuantParams p) {
  constexpr int TOP = HAS_QH ? 31 : 15;
  const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (i >= p.total) return;
  int64_t xrow, crow, boff;
  int g;
  llama_coords(p, i, NBYTES, &xrow, &crow, &boff, &g);
  const uint4* src = reinterpret_cast<const uint4*>(p.x + (xrow * p.nb + g) * 32);
  float x[32];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint4 v = __ldg(src + k);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo16 = w[j] & 0xffffu, hi16 = w[j] >> 16;
      x[8 * k + 2 * j] = p.bf16 ? __uint_as_float(lo16 << 16) : half_bits_to_float((uint16_t)lo16);
      x[8 * k + 2 * j + 1] = p.bf16 ? __uint_as_float(hi16 << 16) : half_bits_to_float((uint16_t)hi16);
    }
  }
  uint16_t d16, m16;
  uint32_t q[32];
  llama_quantize32<OFF, TOP>(x, &d16, &m16, q);
  if constexpr (!TO_CACHE) {
    llama_store_block<NBYTES, HAS_M, HAS_QH>(p.blocks + boff, d16, m16, q);
  } else {
    constexpr int PER = 32 / BITS, NW = 32 / PER;          // codes per word, words per block
    uint32_t w[NW];
#pragma unroll
    for (int k = 0; k < NW; ++k) {
      w[k] = 0u;
#pragma unroll
      for (int e = 0; e < PER; ++e) w[k] |= q[k * PER + e] << (BITS * e);
    }
    uint4* dst = reinterpret_cast<uint4*>(p.codes + crow * (p.nb * NW) + g * NW);
#pragma unroll
    for (int k = 0; k < NW / 4; ++k) dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
    const uint16_t bias = HAS_M ? m16
                                : __half_as_ushort(__float2half_rn(-(float)OFF * half_bits_to_float(d16)));
    p.scales[crow * p.nb + g] = d16;
    p.biases[crow * p.nb + g] = bias;
  }
}

// Affine cache rows (groups of 32) -> blocks: d = the scale, m = the bias (_1
// types), the codes' low 4 bits and (Q5) fifth bits.  The block holds the
// group's values when the group is one such a block can hold (codes below 16
// or 32; for the _0 types, bias == -8d or -16d) -- the groups that the import
// and the block quantizer write.
template <int NBYTES, bool HAS_M, bool HAS_QH, int BITS>
__global__ void __launch_bounds__(256) qkv_llama_export_kernel(const __grid_constant__ LlamaQuantParams p) {
  const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (i >= p.total) return;
  int64_t xrow, crow, boff;
  int g;
  llama_coords(p, i, NBYTES, &xrow, &crow, &boff, &g);
  constexpr int PER = 32 / BITS, NW = 32 / PER;
  const uint4* src = reinterpret_cast<const uint4*>(p.codes + crow * (p.nb * NW) + g * NW);
  uint32_t w[NW];
#pragma unroll
  for (int k = 0; k < NW / 4; ++k) {
    const uint4 v = __ldg(src + k);
    w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
  }
  uint32_t q[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) q[e] = (w[e / PER] >> (BITS * (e % PER))) & ((1u << BITS) - 1u);
  const uint16_t d16 = __ldg(reinterpret_cast<const unsigned short*>(p.scales) + crow * p.nb + g);
  const uint16_t m16 = HAS_M ? __ldg(reinterpret_cast<const unsigned short*>(p.biases) + crow * p.nb + g)
                             : (uint16_t)0;
  llama_store_block<NBYTES, HAS_M, HAS_QH>(p.blocks + boff, d16, m16, q);
}

template <bool TO_CACHE>
cudaError_t launch_llama_quantize_t(int kind, const LlamaQuantParams& p, int64_t grid, cudaStream_t s) {
  switch (kind) {
    case QKV_BLOCKS_Q4_0: qkv_llama_quantize_kernel<18, false, false, 8, 4, TO_CACHE><<<(unsigned)grid, 256, 0, s>>>(p); break;
    case QKV_BLOCKS_Q4_1: qkv_llama_quantize_kernel<20, true, false, 0, 4, TO_CACHE><<<(unsigned)grid, 256, 0, s>>>(p); break;
    case QKV_BLOCKS_Q5_0: qkv_llama_quantize_kernel<22, false, true, 16, 8, TO_CACHE><<<(unsigned)grid, 256, 0, s>>>(p); break;
    case QKV_BLOCKS_Q5_1: qkv_llama_quantize_kernel<24, true, true, 0, 8, TO_CACHE><<<(unsigned)grid, 256, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// x [B, Hkv, L, D] -> blocks (c == nullptr) or into rows [offset, offset + L)
// of the affine cache c.
cudaError_t launch_llama_quantize(int kind, const void* x, int in_dtype, int B, int Hkv, int D,
                                  int64_t L, void* blocks, int64_t sb, int64_t sh, int64_t sl,
                                  const qkv_cache* c, int64_t offset, cudaStream_t stream) {
  LlamaQuantParams p = {};
  p.x = static_cast<const uint16_t*>(x);
  p.bf16 = in_dtype == QKV_BF16;
  p.blocks = static_cast<uint8_t*>(blocks);
  p.sb = sb; p.sh = sh; p.sl = sl;
  if (c != nullptr) {
    p.codes = c->codes; p.scales = c->scales; p.biases = c->biases; p.Lcap = c->Lcap;
  }
  p.offset = offset;
  p.L = L;
  p.Hkv = Hkv;
  p.nb = D / 32;
  p.total = (int64_t)B * Hkv * L * p.nb;
  const int64_t grid = (p.total + 255) / 256;
  if (grid > 0x7fffffff) return cudaErrorInvalidValue;
  return c != nullptr ? launch_llama_quantize_t<true>(kind, p, grid, stream)
                      : launch_llama_quantize_t<false>(kind, p, grid, stream);
}

// Rows [offset, offset + L) of the affine cache c -> blocks.
cudaError_t launch_llama_export(int kind, const qkv_cache* c, int B, int Hkv, int D, int64_t offset,
                                int64_t L, void* blocks, int64_t sb, int64_t sh, int64_t sl,
                                cudaStream_t stream) {
  LlamaQuantParams p = {};
  p.blocks = static_cast<uint8_t*>(blocks);
  p.sb = sb; p.sh = sh; p.sl = sl;
  p.codes = c->codes; p.scales = c->scales; p.biases = c->biases; p.Lcap = c->Lcap;
  p.offset = offset;
  p.L = L;
  p.Hkv = Hkv;
  p.nb = D / 32;
  p.total = (int64_t)B * Hkv * L * p.nb;
  const int64_t grid = (p.total + 255) / 256;
  if (grid > 0x7fffffff) return cudaErrorInvalidValue;
  switch (kind) {
    case QKV_BLOCKS_Q4_0: qkv_llama_export_kernel<18, false, false, 4><<<(unsigned)grid, 256, 0, stream>>>(p); break;
    case QKV_BLOCKS_Q4_1: qkv_llama_export_kernel<20, true, false, 4><<<(unsigned)grid, 256, 0, stream>>>(p); break;
    case QKV_BLOCKS_Q5_0: qkv_llama_export_kernel<22, false, true, 8><<<(unsigned)grid, 256, 0, stream>>>(p); break;
    case QKV_BLOCKS_Q5_1: qkv_llama_export_kernel<24, true, true, 8><<<(unsigned)grid, 256, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace qkv
