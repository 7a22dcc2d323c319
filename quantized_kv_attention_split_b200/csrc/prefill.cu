// prefill.cu -- host side of the tcgen05 multi-query kernel: instance table
// and launch.
#include <algorithm>

#include "prefill_kernel.cuh"

namespace qkv {

namespace {

template <int D, int BITS, int GS, bool Q8, int VAR, bool RANGE>
cudaError_t launch_pf_r(const PrefillParams& p, int grid, cudaStream_t s) {
  using C = PfCfg<D, BITS, GS, Q8>;
  auto k = qsdpa_prefill_tc_kernel<D, BITS, GS, Q8, VAR, RANGE>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  k<<<grid, kPfThreads, C::SMEM, s>>>(p);
  return cudaGetLastError();
}

// A call: the range check of the cache's scales and biases, then the kernel
// and its range-scaled instance (one of the two runs, the other exits at
// once).
template <int D, int BITS, int GS, bool Q8, int VAR>
cudaError_t launch_pf_v(const PrefillParams& p, int grid, cudaStream_t s) {
  const int ng = D / GS;
  const int64_t units = (p.L * ng + 7) / 8;
  const int64_t slabs = (int64_t)p.B * p.Hkv;
  if (slabs > 65535) return cudaErrorInvalidValue;
  const unsigned cx = (unsigned)std::min<int64_t>(std::max<int64_t>(1, (units + 255) / 256), 148);
  qkv_range_check_kernel<Q8, BITS><<<dim3(cx, (unsigned)slabs), 256, 0, s>>>(p, ng);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_pf_r<D, BITS, GS, Q8, VAR, false>(p, grid, s);
  if (e != cudaSuccess) return e;
  return launch_pf_r<D, BITS, GS, Q8, VAR, true>(p, grid, s);
}

// the extension instance only when an extension is in use; additive masks
// (with or without slopes) and no softcap or sinks: the mask instance
template <int D, int BITS, int GS, bool Q8>
cudaError_t launch_pf(const PrefillParams& p, int grid, cudaStream_t s) {
  if (p.mask_kind == QKV_MASK_ADDITIVE && !(p.cap_a > 0.f) && p.sinks == nullptr)
    return launch_pf_v<D, BITS, GS, Q8, kPfMask>(p, grid, s);
  if (p.cap_a > 0.f || p.slopes != nullptr || p.sinks != nullptr)
    return launch_pf_v<D, BITS, GS, Q8, kPfExt>(p, grid, s);
  return launch_pf_v<D, BITS, GS, Q8, kPfPlain>(p, grid, s);
}

template <int D>
cudaError_t launch_pf_d(int bits, int gs, bool q8, const PrefillParams& p, int grid,
                        cudaStream_t s) {
  if (q8) return launch_pf<D, 8, 32, true>(p, grid, s);
  if (bits == 4) {
    if (gs == 32) return launch_pf<D, 4, 32, false>(p, grid, s);
    if (gs == 64) return launch_pf<D, 4, 64, false>(p, grid, s);
    if constexpr (D >= 128) { if (gs == 128) return launch_pf<D, 4, 128, false>(p, grid, s); }
  } else {
    if (gs == 32) return launch_pf<D, 8, 32, false>(p, grid, s);
    if (gs == 64) return launch_pf<D, 8, 64, false>(p, grid, s);
    if constexpr (D >= 128) { if (gs == 128) return launch_pf<D, 8, 128, false>(p, grid, s); }
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_prefill_tc(int D, int bits, int gs, int fmt, PrefillParams& p, cudaStream_t s) {
  const int R = p.G * p.Lq;
  p.mtiles = (R + kPfBM - 1) / kPfBM;
  const int64_t grid = (int64_t)p.B * p.Hkv * p.mtiles;
  if (grid <= 0 || grid > (1ll << 31) - 1) return cudaErrorInvalidValue;
  const bool q8 = fmt == QKV_Q8_0;
  if (D == 64) return launch_pf_d<64>(bits, gs, q8, p, (int)grid, s);
  if (D == 128) return launch_pf_d<128>(bits, gs, q8, p, (int)grid, s);
  if (D == 256) return launch_pf_d<256>(bits, gs, q8, p, (int)grid, s);
  return cudaErrorInvalidValue;
}

}  // namespace qkv
