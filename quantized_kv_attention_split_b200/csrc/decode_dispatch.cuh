// decode_dispatch.cuh -- compile-time instance table for the decode kernel.
// Each decode_*.cu translation unit instantiates the kernels of one head
// dimension; decode_plan.cu picks one at run time.
#pragma once

#include "decode_kernel.cuh"
#include "decode_merge.cuh"

namespace qkv {

// Host-side helpers for one instance.
template <int D, int BITS, int GS, bool Q8, int NC, bool F32OUT, int VAR, int SB = BITS>
struct DecodeInstance {
  using C = DecCfg<D, BITS, GS, Q8, NC, SB>;
  static int max_ctas_per_sm() {
    static int cached = -1;
    if (cached < 0) {
      auto k = qsdpa_decode_kernel<D, BITS, GS, Q8, NC, F32OUT, VAR, SB>;
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
        return 0;
      int n = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, C::NTHR, C::SMEM) != cudaSuccess)
        return 0;
      cached = n;
    }
    return cached;
  }
  // Both kernels are launched with programmatic stream serialization: the
  // set-up before a kernel's grid_dep_wait() overlaps the previous kernel.
  static cudaError_t launch(const DecodePlan& plan, const DecodeParams& p, cudaStream_t s) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)plan.grid);
    cfg.blockDim = dim3(C::NTHR);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, qsdpa_decode_kernel<D, BITS, GS, Q8, NC, F32OUT, VAR, SB>, p);
    if (e != cudaSuccess || !plan.merge) return e;
    // parts per unit: at most the CTAs that share one unit
    const int64_t parts = plan.pieces > 0 ? plan.pieces : (plan.grid + plan.units - 1) / plan.units + 1;
    int lanes = 1;
    while (lanes < 4 && lanes * kMergeBatch < parts) lanes *= 2;
    const int64_t threads = plan.units * (NC * 8) * (D / 4) * lanes;
    cfg.gridDim = dim3((unsigned)((threads + kMergeThreads - 1) / kMergeThreads));
    cfg.blockDim = dim3(kMergeThreads);
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, qsdpa_merge_kernel<D, NC * 8>, p, (int64_t)plan.grid, lanes);
  }
};


struct DecodeOps {
  int (*occupancy)();
  cudaError_t (*launch)(const DecodePlan&, const DecodeParams&, cudaStream_t);
  int tk;      // keys per block
  int nc;
  int teams;   // teams of warps per CTA, each streaming its own blocks
  size_t smem;
};

template <int D, int BITS, int GS, bool Q8, int NC, bool F32, int VAR, int SB = BITS>
DecodeOps make_decode_ops() {
  using I = DecodeInstance<D, BITS, GS, Q8, NC, F32, VAR, SB>;
  return DecodeOps{&I::max_ctas_per_sm, &I::launch, I::C::TK, NC, I::C::NTEAM, (size_t)I::C::SMEM};
}

// The six variants of one format and chunking: f32 selects the
// split-precision value operand used for fp32 output; var the plain kernel,
// the one that also quantizes the new token into the cache, or the one with
// the attention extensions (kept apart so the others carry none of their
// registers).
template <int D, int BITS, int GS, bool Q8, int NC>
DecodeOps pick_decode_ops(bool f32, int var) {
  if (var == kDecFused) return f32 ? make_decode_ops<D, BITS, GS, Q8, NC, true, kDecFused>()
                                   : make_decode_ops<D, BITS, GS, Q8, NC, false, kDecFused>();
  if (var == kDecExt) return f32 ? make_decode_ops<D, BITS, GS, Q8, NC, true, kDecExt>()
                                 : make_decode_ops<D, BITS, GS, Q8, NC, false, kDecExt>();
  return f32 ? make_decode_ops<D, BITS, GS, Q8, NC, true, kDecPlain>()
             : make_decode_ops<D, BITS, GS, Q8, NC, false, kDecPlain>();
}

// Instances of one head dimension; nc in {1, 2, 4}.
template <int D>
bool decode_ops_for(int bits, int gs, bool q8, int nc, bool f32, int var, DecodeOps* ops) {
#define QKV_DEC_NC(BITS, GS, Q8)                                                   \
  do {                                                                             \
    if (nc == 1) *ops = pick_decode_ops<D, BITS, GS, Q8, 1>(f32, var);             \
    else if (nc == 2) *ops = pick_decode_ops<D, BITS, GS, Q8, 2>(f32, var);        \
    else *ops = pick_decode_ops<D, BITS, GS, Q8, 4>(f32, var);                     \
    return true;                                                                   \
  } while (0)
  if (q8) {
    QKV_DEC_NC(8, 32, true);
  }
  if (bits == 4) {
    if (gs == 32) QKV_DEC_NC(4, 32, false);
    if (gs == 64) QKV_DEC_NC(4, 64, false);
    if constexpr (D >= 128) { if (gs == 128) QKV_DEC_NC(4, 128, false); }
  } else if (bits == 8) {
    if (gs == 32) QKV_DEC_NC(8, 32, false);
    if (gs == 64) QKV_DEC_NC(8, 64, false);
    if constexpr (D >= 128) { if (gs == 128) QKV_DEC_NC(8, 128, false); }
  }
#undef QKV_DEC_NC
  return false;
}

// Affine codes stored 2, 3, 5 or 6 bits wide: the plain kernel (no additive
// mask, no extensions, no fused update); 2-bit codes in groups of 64 or 128
// computed as they are, the others transcoding each block to the 4-bit tile
// (2-bit codes in groups of 32, 3-bit codes) or the 8-bit tile (5- and 6-bit
// codes).
template <int D>
bool decode_ops_x_for(int bits, int gs, int nc, bool f32, DecodeOps* ops) {
#define QKV_DEC_X(SB, GS)                                                                      \
  do {                                                                                         \
    constexpr int CB = SB < 4 ? 4 : 8;                                                         \
    if (nc == 1) *ops = f32 ? make_decode_ops<D, CB, GS, false, 1, true, kDecPlain, SB>()      \
                            : make_decode_ops<D, CB, GS, false, 1, false, kDecPlain, SB>();    \
    else if (nc == 2) *ops = f32 ? make_decode_ops<D, CB, GS, false, 2, true, kDecPlain, SB>() \
                                 : make_decode_ops<D, CB, GS, false, 2, false, kDecPlain, SB>(); \
    else *ops = f32 ? make_decode_ops<D, CB, GS, false, 4, true, kDecPlain, SB>()              \
                    : make_decode_ops<D, CB, GS, false, 4, false, kDecPlain, SB>();            \
    return true;                                                                               \
  } while (0)
#define QKV_DEC_XB(SB)                                      \
  do {                                                      \
    if (gs == 32) QKV_DEC_X(SB, 32);                        \
    if (gs == 64) QKV_DEC_X(SB, 64);                        \
    if constexpr (D >= 128) { if (gs == 128) QKV_DEC_X(SB, 128); } \
  } while (0)
  if (bits == 2) {
    // groups of 64 or 128: the 2-bit fragments themselves (whole words per
    // lane); groups of 32: transcoded to 4-bit
#define QKV_DEC_N2(GS)                                                                         \
  do {                                                                                         \
    if (nc == 1) *ops = f32 ? make_decode_ops<D, 2, GS, false, 1, true, kDecPlain>()           \
                            : make_decode_ops<D, 2, GS, false, 1, false, kDecPlain>();         \
    else if (nc == 2) *ops = f32 ? make_decode_ops<D, 2, GS, false, 2, true, kDecPlain>()      \
                                 : make_decode_ops<D, 2, GS, false, 2, false, kDecPlain>();    \
    else *ops = f32 ? make_decode_ops<D, 2, GS, false, 4, true, kDecPlain>()                   \
                    : make_decode_ops<D, 2, GS, false, 4, false, kDecPlain>();                 \
    return true;                                                                               \
  } while (0)
    if (gs == 64) QKV_DEC_N2(64);
    if constexpr (D >= 128) { if (gs == 128) QKV_DEC_N2(128); }
#undef QKV_DEC_N2
    QKV_DEC_XB(2);
  }
  if (bits == 3) QKV_DEC_XB(3);
  if (bits == 5) QKV_DEC_XB(5);
  if (bits == 6) QKV_DEC_XB(6);
#undef QKV_DEC_XB
#undef QKV_DEC_X
  return false;
}

bool decode_ops_d64(int bits, int gs, bool q8, int nc, bool f32, int var, DecodeOps* ops);
bool decode_ops_d128(int bits, int gs, bool q8, int nc, bool f32, int var, DecodeOps* ops);
bool decode_ops_d256(int bits, int gs, bool q8, int nc, bool f32, int var, DecodeOps* ops);
bool decode_ops_x_d64(int bits, int gs, int nc, bool f32, DecodeOps* ops);
bool decode_ops_x_d128(int bits, int gs, int nc, bool f32, DecodeOps* ops);
bool decode_ops_x_d256(int bits, int gs, int nc, bool f32, DecodeOps* ops);

}  // namespace qkv
