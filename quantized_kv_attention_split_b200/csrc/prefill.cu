// prefill.cu -- host side of the tcgen05 multi-query kernel: instance table
// and launch.
#include "prefill_kernel.cuh"

namespace qkv {

namespace {

template <int D, int BITS, int GS, bool Q8, bool EXT>
cudaError_t launch_pf_v(const PrefillParams& p, int grid, cudaStream_t s) {
  using C = PfCfg<D, BITS, GS, Q8>;
  auto k = qsdpa_prefill_tc_kernel<D, BITS, GS, Q8, EXT>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  k<<<grid, kPfThreads, C::SMEM, s>>>(p);
  return cudaGetLastError();
}

// the extension instance only when an extension is in use
template <int D, int BITS, int GS, bool Q8>
cudaError_t launch_pf(const PrefillParams& p, int grid, cudaStream_t s) {
  if (p.cap_a > 0.f || p.slopes != nullptr || p.sinks != nullptr)
    return launch_pf_v<D, BITS, GS, Q8, true>(p, grid, s);
  return launch_pf_v<D, BITS, GS, Q8, false>(p, grid, s);
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
