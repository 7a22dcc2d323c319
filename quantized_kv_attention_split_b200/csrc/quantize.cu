// quantize.cu -- quantize-and-append of new K/V tokens into the cache.
//
// The quantizer's arithmetic is in quantize_core.cuh (shared with the fused
// update + decode kernel).
//
// Design: one thread owns 32 consecutive elements (four 16-byte loads) and
// takes their min / max (or largest magnitude) on the packed 16-bit pairs;
// the gs/32 lanes of a group reduce with shuffles, each thread packs its
// codes into words and stores them; the first lane of a group stores the
// fp16 scale (and bias).  Grid: x = blocks of tokens (256 / (D/32) tokens
// per block), y = (batch, kv head) slab, z = K or V (one launch when both
// caches have the same format).
#include <algorithm>

#include "qkv_common.cuh"
#include "qkv_internal.h"
#include "quantize_core.cuh"

namespace qkv {

struct QuantSide {
  const uint16_t* src;      // [B * Hkv * Lnew, D] fp16/bf16 bits
  uint32_t* codes;          // cache codes base
  uint16_t* scales;
  uint16_t* biases;
  int64_t Lcap;
};

struct QuantParams {
  QuantSide side[2];
  int D;
  int per_row;              // D / 32: threads per token row
  int tpb;                  // tokens per 256-thread block
  int Lnew;
  int64_t offset;
};

template <int GS, int BITS, bool Q8, bool BF16>
__global__ void __launch_bounds__(256, 6) qkv_quantize_kernel(const __grid_constant__ QuantParams p, int side0) {
  const QuantSide& s = (side0 + (int)blockIdx.z) ? p.side[1] : p.side[0];
  // rows of D / 32 threads back to back (a row starts on an even lane, so the
  // 1, 2 or 4 lanes of a group are adjacent and aligned for the shuffles)
  const int lt = threadIdx.x / p.per_row;           // token within the block
  const int cs = threadIdx.x - lt * p.per_row;      // which 32-element slice of the row
  const int tok = blockIdx.x * p.tpb + lt;
  const bool active = lt < p.tpb && tok < p.Lnew;   // inactive lanes still join the shuffles
  const int64_t slab = blockIdx.y;                  // b * Hkv + kv head
  const int64_t srow = slab * p.Lnew + (active ? tok : 0);
  const int64_t crow = slab * s.Lcap + p.offset + tok;
  uint32_t w[kQWords];                              // 32 raw 16-bit inputs, two per word
  if (active) {
    const uint4* src = reinterpret_cast<const uint4*>(s.src + srow * p.D + cs * kQEpt);
#pragma unroll
    for (int k = 0; k < kQWords / 4; ++k) {
      const uint4 r = __ldg(src + k);
      w[4 * k] = r.x; w[4 * k + 1] = r.y; w[4 * k + 2] = r.z; w[4 * k + 3] = r.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < kQWords; ++i) w[i] = 0u;
  }
  const int grp = (cs * kQEpt) / GS;
  const bool leader = ((cs * kQEpt) % GS) == 0;
  const int ng = p.D / GS;
  uint32_t o[kQEpt * BITS / 32];
  uint16_t sbits, bbits;
  quantize_slice<GS, BITS, Q8, BF16>(w, o, sbits, bbits);
  if (active) {
    // the thread's BITS words: 16-byte stores for 4 and 8 bits, 8-byte ones
    // for 2 and 6 (their offsets are 8-byte aligned), words for 3 and 5
    uint32_t* dw = s.codes + crow * (p.D * BITS / 32) + cs * (kQEpt * BITS / 32);
    if constexpr (BITS % 4 == 0) {
#pragma unroll
      for (int k = 0; k < BITS / 4; ++k)
        reinterpret_cast<uint4*>(dw)[k] = make_uint4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
    } else if constexpr (BITS % 2 == 0) {
#pragma unroll
      for (int k = 0; k < BITS / 2; ++k) reinterpret_cast<uint2*>(dw)[k] = make_uint2(o[2 * k], o[2 * k + 1]);
    } else {
#pragma unroll
      for (int k = 0; k < BITS; ++k) dw[k] = o[k];
    }
    if (leader) {
      s.scales[crow * ng + grp] = sbits;
      if constexpr (!Q8) s.biases[crow * ng + grp] = bbits;
    }
  }
}

namespace {

template <bool BF16>
cudaError_t launch_q(int fmt, int bits, int gs, const QuantParams& p, int side0, int nsides,
                     dim3 grid, cudaStream_t stream) {
  grid.z = nsides;
#define QKV_QLAUNCH(GS, BITS, Q8) \
  qkv_quantize_kernel<GS, BITS, Q8, BF16><<<grid, 256, 0, stream>>>(p, side0)
  if (fmt == QKV_Q8_0) QKV_QLAUNCH(32, 8, true);
  else if (bits == 4 && gs == 32) QKV_QLAUNCH(32, 4, false);
  else if (bits == 4 && gs == 64) QKV_QLAUNCH(64, 4, false);
  else if (bits == 4 && gs == 128) QKV_QLAUNCH(128, 4, false);
  else if (bits == 8 && gs == 32) QKV_QLAUNCH(32, 8, false);
  else if (bits == 8 && gs == 64) QKV_QLAUNCH(64, 8, false);
  else if (bits == 8 && gs == 128) QKV_QLAUNCH(128, 8, false);
  else if (bits == 2 && gs == 32) QKV_QLAUNCH(32, 2, false);
  else if (bits == 2 && gs == 64) QKV_QLAUNCH(64, 2, false);
  else if (bits == 2 && gs == 128) QKV_QLAUNCH(128, 2, false);
  else if (bits == 3 && gs == 32) QKV_QLAUNCH(32, 3, false);
  else if (bits == 3 && gs == 64) QKV_QLAUNCH(64, 3, false);
  else if (bits == 3 && gs == 128) QKV_QLAUNCH(128, 3, false);
  else if (bits == 5 && gs == 32) QKV_QLAUNCH(32, 5, false);
  else if (bits == 5 && gs == 64) QKV_QLAUNCH(64, 5, false);
  else if (bits == 5 && gs == 128) QKV_QLAUNCH(128, 5, false);
  else if (bits == 6 && gs == 32) QKV_QLAUNCH(32, 6, false);
  else if (bits == 6 && gs == 64) QKV_QLAUNCH(64, 6, false);
  else if (bits == 6 && gs == 128) QKV_QLAUNCH(128, 6, false);
  else return cudaErrorInvalidValue;
#undef QKV_QLAUNCH
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const void* new_k, const void* new_v, int in_dtype, int B, int Hkv,
                            int Lnew, int D, const qkv_cache* k, const qkv_cache* v,
                            int64_t offset, cudaStream_t stream) {
  QuantParams p;
  const qkv_cache* c[2] = {k, v};
  const void* src[2] = {new_k, new_v};
  int fmt[2], bits[2], gs[2];
  for (int i = 0; i < 2; ++i) {
    p.side[i].src = static_cast<const uint16_t*>(src[i]);
    p.side[i].codes = c[i]->codes;
    p.side[i].scales = c[i]->scales;
    p.side[i].biases = c[i]->biases;
    p.side[i].Lcap = c[i]->Lcap;
    fmt[i] = c[i]->fmt;
    bits[i] = c[i]->fmt == QKV_Q8_0 ? 8 : c[i]->bits;
    gs[i] = c[i]->fmt == QKV_Q8_0 ? 32 : c[i]->group_size;
  }
  p.D = D;
  p.per_row = D / kQEpt;
  p.Lnew = Lnew;
  p.offset = offset;
  const int64_t slabs = (int64_t)B * Hkv;
  if (slabs > 65535 || D % kQEpt != 0 || p.per_row > 256 || p.per_row % 2 != 0)
    return cudaErrorInvalidValue;
  const int tpb = 256 / p.per_row;                  // tokens per block
  p.tpb = tpb;
  dim3 grid((unsigned)((Lnew + tpb - 1) / tpb), (unsigned)slabs, 1);
  const bool same = fmt[0] == fmt[1] && bits[0] == bits[1] && gs[0] == gs[1];
  const bool bf16 = in_dtype == QKV_BF16;
  for (int side0 = 0; side0 < 2; side0 += same ? 2 : 1) {
    const int n = same ? 2 : 1;
    cudaError_t e = bf16 ? launch_q<true>(fmt[side0], bits[side0], gs[side0], p, side0, n, grid, stream)
                         : launch_q<false>(fmt[side0], bits[side0], gs[side0], p, side0, n, grid, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace qkv
