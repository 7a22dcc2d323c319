// blocks.cu -- conversion between llama.cpp-style interleaved Q8_0 blocks and
// the library's Q8_0 planes.
//
// llama.cpp #25556 keeps its KV cache as Q8_0 blocks; its byte layout is the
// GGUF Q8_0 block: 34 bytes, the fp16 scale first (little-endian), then the 32
// int8 codes in element order.  This library stores a codes plane (element e
// in byte e%4 of 32-bit word e/4, i.e. the same byte order) and a scales
// plane, so a block is 17 little-endian 16-bit units: unit 0 is the scale,
// units 1..16 are the codes two at a time, and code word w of the block is
// unit 1+2w | unit 2+2w << 16.  Data movement only, bit for bit.
//
// One thread per block, whose 16-bit units are read (or written) one by one,
// since 34-byte blocks are only 2-byte aligned in general; when the block
// array and its strides are 4-byte aligned (as llama.cpp's are: D/32 is even,
// so a row of blocks is a multiple of 68 bytes), the write to blocks takes one
// thread per pair of blocks instead: 68 bytes starting 4-byte aligned, written
// as 17 32-bit words.  The plane side moves 16-byte code chunks and the scales.
#include "qkv_common.cuh"
#include "qkv_internal.h"

namespace qkv {

struct BlocksParams {
  const uint8_t* src_blocks;   // from_blocks: source blocks
  uint8_t* dst_blocks;         // to_blocks: destination blocks
  uint32_t* codes;             // the cache planes (read by to_blocks, written by from_blocks)
  uint16_t* scales;
  uint16_t* biases;            // affine destination (llama.cpp Q4/Q5 blocks)
  int64_t Lcap, offset, L;
  int Hkv, nb;                 // kv heads, blocks per row (D / 32)
  int64_t sb, sh, sl;          // byte strides of a block row (b, kv head, token)
  int64_t total;               // B * Hkv * L * nb (blocks), or half of it (pairs)
};

__device__ __forceinline__ void block_coords(const BlocksParams& p, int64_t i, int64_t* crow,
                                             int64_t* boff, int* g, int block_bytes = 34) {
  const int64_t rest = i / p.nb;
  *g = (int)(i - rest * p.nb);
  const int64_t bh = rest / p.L;
  const int64_t l = rest - bh * p.L;
  const int64_t b = bh / p.Hkv, h = bh - b * p.Hkv;
  *crow = bh * p.Lcap + p.offset + l;                      // cache row
  *boff = b * p.sb + h * p.sh + l * p.sl + (int64_t)*g * block_bytes;
}

__global__ void __launch_bounds__(256) qkv_q8_0_from_blocks_kernel(const __grid_constant__ BlocksParams p) {
  const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (i >= p.total) return;
  int64_t crow, boff;
  int g;
  block_coords(p, i, &crow, &boff, &g);
  const uint16_t* src = reinterpret_cast<const uint16_t*>(p.src_blocks + boff);
  uint32_t u[17];
#pragma unroll
  for (int k = 0; k < 17; ++k) u[k] = __ldg(src + k);
  uint4* dst = reinterpret_cast<uint4*>(p.codes + crow * (p.nb * 8) + g * 8);
  dst[0] = make_uint4(u[1] | (u[2] << 16), u[3] | (u[4] << 16), u[5] | (u[6] << 16), u[7] | (u[8] << 16));
  dst[1] = make_uint4(u[9] | (u[10] << 16), u[11] | (u[12] << 16), u[13] | (u[14] << 16),
                      u[15] | (u[16] << 16));
  p.scales[crow * p.nb + g] = (uint16_t)u[0];
}

__global__ void __launch_bounds__(256) qkv_q8_0_to_blocks_kernel(const __grid_constant__ BlocksParams p) {
  const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (i >= p.total) return;
  int64_t crow, boff;
  int g;
  block_coords(p, i, &crow, &boff, &g);
  const uint4* src = reinterpret_cast<const uint4*>(p.codes + crow * (p.nb * 8) + g * 8);
  const uint4 a = __ldg(src), c = __ldg(src + 1);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
  uint16_t* dst = reinterpret_cast<uint16_t*>(p.dst_blocks + boff);
  dst[0] = __ldg(reinterpret_cast<const unsigned short*>(p.scales) + crow * p.nb + g);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    dst[1 + 2 * k] = (uint16_t)(w[k] & 0xffffu);
    dst[2 + 2 * k] = (uint16_t)(w[k] >> 16);
  }
}

// Pair form of the write to blocks: thread i writes blocks 2i and 2i+1 (nb is
// even, so a pair never straddles two rows).  Words of the 68 bytes: the first
// block's scale and first code half, then its code words shifted by 16 bits,
// then the last code half with the second block's scale, then the second
// block's code words.
__global__ void __launch_bounds__(256) qkv_q8_0_to_block_pairs_kernel(const __grid_constant__ BlocksParams p) {
  const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (i >= p.total) return;
  int64_t crow, boff;
  int g;
  block_coords(p, 2 * i, &crow, &boff, &g);
  const uint4* src = reinterpret_cast<const uint4*>(p.codes + crow * (p.nb * 8) + g * 8);
  const uint4 a = __ldg(src), c = __ldg(src + 1), d = __ldg(src + 2), e = __ldg(src + 3);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
  const uint32_t s0 = __ldg(reinterpret_cast<const unsigned short*>(p.scales) + crow * p.nb + g);
  const uint32_t s1 = __ldg(reinterpret_cast<const unsigned short*>(p.scales) + crow * p.nb + g + 1);
  uint32_t* dst = reinterpret_cast<uint32_t*>(p.dst_blocks + boff);
  dst[0] = s0 | (w[0] << 16);
#pragma unroll
  for (int k = 1; k < 8; ++k) dst[k] = __byte_perm(w[k - 1], w[k], 0x5432);
  dst[8] = (w[7] >> 16) | (s1 << 16);
  dst[9] = d.x; dst[10] = d.y; dst[11] = d.z; dst[12] = d.w;
  dst[13] = e.x; dst[14] = e.y; dst[15] = e.z; dst[16] = e.w;
}

// llama.cpp's Q4_0 / Q4_1 / Q5_0 / Q5_1 blocks of 32 (NBYTES bytes: fp16 d,
// then fp16 m (HAS_M), then the 32 fifth bits qh (HAS_QH, bit e for element
// e), then qs[16]: element j < 16 in the low nibble of qs[j], element j + 16
// in the high one) into an affine cache with groups of 32 holding the same
// values: scale d, bias m or -OFF * d (a power-of-two multiple of an fp16
// value: exact while |OFF * d| <= 65504, i.e. |d| <= 8188 for Q4_0 and 4094
// for Q5_0; a larger d gives a block whose values leave the fp16 range, and
// its bias rounds to +-inf), codes BITS wide in the library's packing (element e at bits
// BITS*(e % (32/BITS)) of word e / (32/BITS)).  One thread per block.
template <int NBYTES, bool HAS_M, bool HAS_QH, int OFF, int BITS>
__global__ void __launch_bounds__(256) qkv_llama_blocks_kernel(const __grid_constant__ BlocksParams p) {
  const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (i >= p.total) return;
  int64_t crow, boff;
  int g;
  block_coords(p, i, &crow, &boff, &g, NBYTES);
  const uint16_t* src = reinterpret_cast<const uint16_t*>(p.src_blocks + boff);
  constexpr int NU = NBYTES / 2;
  uint32_t u[NU];
#pragma unroll
  for (int k = 0; k < NU; ++k) u[k] = __ldg(src + k);
  constexpr int QH = HAS_M ? 2 : 1;                  // unit of qh
  constexpr int QS = QH + (HAS_QH ? 2 : 0);          // first unit of qs
  const uint32_t qh = HAS_QH ? (u[QH] | (u[QH + 1] << 16)) : 0u;
  uint32_t q[32];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t byte = (u[QS + j / 2] >> (8 * (j & 1))) & 0xffu;
    q[j] = byte & 0xfu;
    q[j + 16] = byte >> 4;
  }
  if constexpr (HAS_QH) {
#pragma unroll
    for (int e = 0; e < 32; ++e) q[e] |= ((qh >> e) & 1u) << 4;
  }
  constexpr int PER = 32 / BITS;                      // codes per word
  constexpr int NW = 32 / PER;                        // words per block
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
  const uint16_t d = (uint16_t)u[0];
  uint16_t m;
  if constexpr (HAS_M) m = (uint16_t)u[1];
  else m = __half_as_ushort(__float2half_rn(-(float)OFF * __half2float(__ushort_as_half(d))));
  p.scales[crow * p.nb + g] = d;
  p.biases[crow * p.nb + g] = m;
}

cudaError_t launch_llama_blocks(int kind, const void* src_blocks, const qkv_cache* c, int B, int Hkv,
                                int D, int64_t offset, int64_t L, int64_t sb, int64_t sh,
                                int64_t sl, cudaStream_t stream) {
  BlocksParams p;
  p.src_blocks = static_cast<const uint8_t*>(src_blocks);
  p.dst_blocks = nullptr;
  p.codes = c->codes;
  p.scales = c->scales;
  p.biases = c->biases;
  p.Lcap = c->Lcap;
  p.offset = offset;
  p.L = L;
  p.Hkv = Hkv;
  p.nb = D / 32;
  p.sb = sb; p.sh = sh; p.sl = sl;
  p.total = (int64_t)B * Hkv * L * p.nb;
  const int64_t grid = (p.total + 255) / 256;
  if (grid > 0x7fffffff) return cudaErrorInvalidValue;
  switch (kind) {
    case QKV_BLOCKS_Q4_0: qkv_llama_blocks_kernel<18, false, false, 8, 4><<<(unsigned)grid, 256, 0, stream>>>(p); break;
    case QKV_BLOCKS_Q4_1: qkv_llama_blocks_kernel<20, true, false, 0, 4><<<(unsigned)grid, 256, 0, stream>>>(p); break;
    case QKV_BLOCKS_Q5_0: qkv_llama_blocks_kernel<22, false, true, 16, 8><<<(unsigned)grid, 256, 0, stream>>>(p); break;
    case QKV_BLOCKS_Q5_1: qkv_llama_blocks_kernel<24, true, true, 0, 8><<<(unsigned)grid, 256, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_q8_0_blocks(bool to_blocks, const void* src_blocks, void* dst_blocks,
                               const qkv_cache* c, int B, int Hkv, int D, int64_t offset, int64_t L,
                               int64_t sb, int64_t sh, int64_t sl, cudaStream_t stream) {
  BlocksParams p;
  p.src_blocks = static_cast<const uint8_t*>(src_blocks);
  p.dst_blocks = static_cast<uint8_t*>(dst_blocks);
  p.codes = c->codes;
  p.scales = c->scales;
  p.biases = nullptr;
  p.Lcap = c->Lcap;
  p.offset = offset;
  p.L = L;
  p.Hkv = Hkv;
  p.nb = D / 32;
  p.sb = sb; p.sh = sh; p.sl = sl;
  const uintptr_t base = reinterpret_cast<uintptr_t>(to_blocks ? dst_blocks : src_blocks);
  // 16-bit reads measured faster than the pair form's 32-bit ones for the
  // read from blocks (both through L1); the write to blocks gains from pairs
  const bool pairs = to_blocks &&
                     ((base | (uintptr_t)sb | (uintptr_t)sh | (uintptr_t)sl) & 3u) == 0 && p.nb % 2 == 0;
  p.total = (int64_t)B * Hkv * L * p.nb / (pairs ? 2 : 1);
  const int64_t grid = (p.total + 255) / 256;
  if (grid > 0x7fffffff) return cudaErrorInvalidValue;
  if (pairs) {
    qkv_q8_0_to_block_pairs_kernel<<<(unsigned)grid, 256, 0, stream>>>(p);
  } else {
    if (to_blocks) qkv_q8_0_to_blocks_kernel<<<(unsigned)grid, 256, 0, stream>>>(p);
    else qkv_q8_0_from_blocks_kernel<<<(unsigned)grid, 256, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace qkv
