// api.cu -- extern "C" entry points of libqkv.so: argument validation, work
// planning and kernel launch.  Declarations and contracts: include/qkv.h.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "qkv_internal.h"

namespace qkv {
cudaError_t launch_quantize(const void* new_k, const void* new_v, int in_dtype, int B, int Hkv,
                            int Lnew, int D, const qkv_cache* k, const qkv_cache* v,
                            int64_t offset, cudaStream_t stream);
size_t decode_workspace_bound(int B, int Hq, int Hkv, int D);
size_t decode_workspace_zero_bytes(int B, int Hq, int Hkv);
void decode_chunking(int G, int* nc, int* ncg);
struct PrefillParams;
}  // namespace qkv
#include "prefill_kernel.cuh"
namespace qkv {
cudaError_t launch_prefill_tc(int D, int bits, int gs, int fmt, PrefillParams& p, cudaStream_t s);
}  // namespace qkv

namespace {

thread_local char g_last_error[512] = "";

// Multi-query calls with at least this many (head, query) rows per kv head run
// on the tcgen05 kernel; smaller ones, and fp32 output (whose 1e-4 accuracy
// needs the split-precision value operand), on the split-K kernel.
constexpr int kTensorPrefillMinRows = 64;

qkv_status fail(qkv_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

qkv_status ok() {
  g_last_error[0] = '\0';
  return QKV_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates one cache description for head dimension D (kview: also the
// 576-element key rows of the view attention, which the quantizer writes).
qkv_status check_cache(const char* name, const qkv_cache* c, int D, bool kview = false) {
  if (c == nullptr) return fail(QKV_ERR_INVALID_ARG, "%s: cache descriptor is NULL", name);
  if (c->fmt != QKV_AFFINE && c->fmt != QKV_Q8_0)
    return fail(QKV_ERR_INVALID_ARG, "%s: unknown format %d", name, c->fmt);
  if (c->fmt == QKV_AFFINE) {
    if (c->bits != 2 && c->bits != 3 && c->bits != 4 && c->bits != 5 && c->bits != 6 && c->bits != 8)
      return fail(QKV_ERR_UNSUPPORTED, "%s: affine bits must be 2, 3, 4, 5, 6 or 8 (got %d)", name,
                  c->bits);
    if (c->group_size != 32 && c->group_size != 64 && c->group_size != 128)
      return fail(QKV_ERR_UNSUPPORTED, "%s: group_size must be 32, 64 or 128 (got %d)", name,
                  c->group_size);
    if (c->biases == nullptr) return fail(QKV_ERR_INVALID_ARG, "%s: affine cache needs biases", name);
  } else {
    if (c->bits != 8 || c->group_size != 32)
      return fail(QKV_ERR_INVALID_ARG, "%s: Q8_0 needs bits 8 and group_size 32", name);
  }
  if (D != 64 && D != 128 && D != 256 && !(kview && D == 576))
    return fail(QKV_ERR_UNSUPPORTED, "head dimension must be 64, 128 or 256%s (got %d)",
                kview ? " (or 576)" : "", D);
  if (D % c->group_size != 0)
    return fail(QKV_ERR_UNSUPPORTED, "%s: D=%d is not a multiple of group_size=%d", name, D,
                c->group_size);
  if (c->codes == nullptr || c->scales == nullptr)
    return fail(QKV_ERR_INVALID_ARG, "%s: codes and scales must be non-NULL", name);
  if (c->Lcap <= 0) return fail(QKV_ERR_INVALID_ARG, "%s: Lcap must be positive", name);
  if (c->Lcap % 8 != 0)
    return fail(QKV_ERR_ALIGNMENT, "%s: Lcap must be a multiple of 8 (got %lld)", name,
                (long long)c->Lcap);
  if (!aligned16(c->codes) || !aligned16(c->scales) ||
      (c->fmt == QKV_AFFINE && !aligned16(c->biases)))
    return fail(QKV_ERR_ALIGNMENT, "%s: codes, scales and biases must be 16-byte aligned", name);
  return QKV_OK;
}

// Where q or out of an attention call lives.  Device (or managed) memory, or
// page-locked host memory that the device reads and writes at the same
// address (cudaHostAlloc / cudaMallocHost, and cudaHostRegister where the
// mapping is the identity, as with unified addressing on 64-bit hosts): the
// split-K kernels then move those bytes over the host link themselves.
// Anything else -- pageable host memory, an unknown address -- is refused
// before a launch, since no kernel could touch it.
enum class Where { kDevice, kHost };
qkv_status where_is(const char* name, const void* ptr, Where* w) {
  cudaPointerAttributes a;
  const cudaError_t e = cudaPointerGetAttributes(&a, ptr);
  if (e != cudaSuccess) {
    cudaGetLastError();
    if (e == cudaErrorInvalidValue)
      return fail(QKV_ERR_INVALID_ARG, "%s: not an address the device can use", name);
    return fail(QKV_ERR_CUDA, "cudaPointerGetAttributes(%s): %s", name, cudaGetErrorString(e));
  }
  if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) {
    *w = Where::kDevice;
    return QKV_OK;
  }
  if (a.type == cudaMemoryTypeHost && a.devicePointer == ptr) {
    *w = Where::kHost;
    return QKV_OK;
  }
  return fail(QKV_ERR_INVALID_ARG,
              "%s must be device memory or page-locked host memory mapped at the same address", name);
}

qkv_status check_dtype(const char* name, int dt, bool allow_f32) {
  if (dt == QKV_F16 || dt == QKV_BF16 || (allow_f32 && dt == QKV_F32)) return QKV_OK;
  return fail(QKV_ERR_INVALID_ARG, "%s: unsupported dtype %d", name, dt);
}

// new_k / new_v (non-null only for Lq == 1): fused update -- the new token
// is quantized into cache row L - 1 by the decode kernel itself.
qkv_status attention(const void* q, int q_dtype, int B, int Hq, int Hkv, int Lq, int D,
                     const qkv_cache* k, const qkv_cache* v, int64_t L, float scale,
                     const qkv_mask* mask, void* out, int out_dtype, void* workspace,
                     size_t workspace_bytes, void* stream, const void* new_k = nullptr,
                     const void* new_v = nullptr, int in_dtype = QKV_F16,
                     const qkv_attn_ext* ext = nullptr) {
  qkv_status st;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0)
    return fail(QKV_ERR_INVALID_ARG, "B, Hq, Hkv and Lq must be positive");
  if (Hq % Hkv != 0) return fail(QKV_ERR_INVALID_ARG, "Hq=%d is not a multiple of Hkv=%d", Hq, Hkv);
  if ((st = check_cache("k", k, D)) != QKV_OK) return st;
  if ((st = check_cache("v", v, D)) != QKV_OK) return st;
  if (k->fmt != v->fmt || k->bits != v->bits || k->group_size != v->group_size)
    return fail(QKV_ERR_UNSUPPORTED, "k and v must use the same format, bits and group_size");
  if (k->Lcap != v->Lcap) return fail(QKV_ERR_INVALID_ARG, "k and v must have the same Lcap");
  if (L < 0 || L > k->Lcap) return fail(QKV_ERR_INVALID_ARG, "L=%lld outside [0, Lcap]", (long long)L);
  if ((st = check_dtype("q", q_dtype, false)) != QKV_OK) return st;
  if ((st = check_dtype("out", out_dtype, true)) != QKV_OK) return st;
  if (q == nullptr || out == nullptr) return fail(QKV_ERR_INVALID_ARG, "q and out must be non-NULL");
  if (!aligned16(q) || !aligned16(out))
    return fail(QKV_ERR_ALIGNMENT, "q and out must be 16-byte aligned");
  if (!(scale == scale)) return fail(QKV_ERR_INVALID_ARG, "scale is NaN");
  int mkind = QKV_MASK_NONE;
  if (mask != nullptr) {
    mkind = mask->kind;
    if (mkind != QKV_MASK_NONE && mkind != QKV_MASK_CAUSAL && mkind != QKV_MASK_ADDITIVE)
      return fail(QKV_ERR_INVALID_ARG, "unknown mask kind %d", mkind);
    if (mkind == QKV_MASK_ADDITIVE) {
      if (mask->add == nullptr) return fail(QKV_ERR_INVALID_ARG, "additive mask pointer is NULL");
      if ((st = check_dtype("mask", mask->add_dtype, true)) != QKV_OK) return st;
      if (mask->stride_b < 0 || mask->stride_h < 0 || mask->stride_q < 0)
        return fail(QKV_ERR_INVALID_ARG, "mask strides must be non-negative");
    }
  }
  if ((int64_t)Hq * Lq > (int64_t)1 << 30)
    return fail(QKV_ERR_INVALID_ARG, "Hq * Lq too large");
  float cap_a = 0.f, cap_k = 0.f;
  const float* slopes = nullptr;
  const float* sinks = nullptr;
  if (ext != nullptr) {
    if (!(ext->softcap >= 0.f) || std::isinf(ext->softcap))
      return fail(QKV_ERR_INVALID_ARG, "softcap must be finite and >= 0");
    if (ext->softcap > 0.f) {
      cap_a = ext->softcap * 1.4426950408889634f;
      cap_k = 2.f / ext->softcap;
    }
    if ((reinterpret_cast<uintptr_t>(ext->mask_slopes) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(ext->sinks) & 3u) != 0)
      return fail(QKV_ERR_ALIGNMENT, "mask_slopes and sinks must be 4-byte aligned");
    if (mkind == QKV_MASK_ADDITIVE) slopes = ext->mask_slopes;
    sinks = ext->sinks;
  }

  Where q_at, out_at;
  if ((st = where_is("q", q, &q_at)) != QKV_OK) return st;
  if ((st = where_is("out", out, &out_at)) != QKV_OK) return st;
  const bool host_io = q_at == Where::kHost || out_at == Where::kHost;

  const size_t elems = (size_t)B * Hq * Lq * D;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (L == 0) {
    const size_t esz = out_dtype == QKV_F32 ? 4 : 2;
    if (cudaMemsetAsync(out, 0, elems * esz, s) != cudaSuccess)
      return fail(QKV_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(cudaGetLastError()));
    return ok();
  }

  const int G = Hq / Hkv;
  const int rows = G * Lq;                 // rows of one kv head: (head, query) pairs
  // the tcgen05 kernel dequantizes 4- and 8-bit codes and takes q and out
  // from device memory; other widths, and q or out in host memory, take the
  // split-K kernel
  const bool tc_codes = k->fmt == QKV_Q8_0 || k->bits == 4 || k->bits == 8;
  if (Lq > 1 && rows >= kTensorPrefillMinRows && out_dtype != QKV_F32 && tc_codes && !host_io) {
    // many query rows per kv head: the tcgen05 kernel (whole 128-row tiles)
    const size_t need = qsdpa_workspace_size(B, Hq, Hkv, Lq, D, L);
    if (workspace == nullptr || workspace_bytes < need)
      return fail(QKV_ERR_WORKSPACE, "workspace of %zu bytes required (got %zu)", need,
                  workspace_bytes);
    qkv::PrefillParams pp;
    std::memset(&pp, 0, sizeof(pp));
    pp.q = q; pp.q_dtype = q_dtype; pp.out = out; pp.out_dtype = out_dtype;
    pp.kc = reinterpret_cast<const uint8_t*>(k->codes); pp.ks = k->scales; pp.kb = k->biases;
    pp.vc = reinterpret_cast<const uint8_t*>(v->codes); pp.vs = v->scales; pp.vb = v->biases;
    pp.Lcap = k->Lcap; pp.L = L;
    pp.B = B; pp.Hq = Hq; pp.Hkv = Hkv; pp.G = G; pp.Lq = Lq;
    pp.scale_log2e = scale * 1.4426950408889634f;
    pp.mask_kind = mkind;
    if (mkind == QKV_MASK_ADDITIVE) {
      pp.mask = mask->add; pp.mask_dtype = mask->add_dtype;
      pp.msb = mask->stride_b; pp.msh = mask->stride_h; pp.msq = mask->stride_q;
    }
    pp.cap_a = cap_a; pp.cap_k = cap_k; pp.slopes = slopes; pp.sinks = sinks;
    pp.status = static_cast<unsigned*>(workspace);
    // time limit of the kernel's waits, and a test hook that withholds the copy
    // of one half tile so that a wait runs out (environment, read per call)
    pp.wait_ns = 0;
    pp.stall_half = -1;
    if (const char* e = std::getenv("QKV_PREFILL_WAIT_NS")) pp.wait_ns = std::strtoull(e, nullptr, 10);
    if (const char* e = std::getenv("QKV_PREFILL_STALL_HALF")) pp.stall_half = std::atoi(e);
    pp.range = static_cast<unsigned*>(workspace) + 1;   // words 1 and 2 of the zeroed header
    cudaError_t e = qkv::launch_prefill_tc(D, k->bits, k->group_size, k->fmt, pp, s);
    if (e != cudaSuccess) return fail(QKV_ERR_CUDA, "prefill launch: %s", cudaGetErrorString(e));
    return ok();
  }
  qkv::DecodePlan plan;
  const bool fused = new_k != nullptr;
  const bool extended = cap_a > 0.f || slopes != nullptr || sinks != nullptr;
  if (fused && extended)
    return fail(QKV_ERR_UNSUPPORTED, "the fused update step takes no attention extensions");
  // additive masks run on the extension variant (the plain one carries no
  // code for them); the fused variant has its own
  const int var = fused ? qkv::kDecFused
                        : (extended || mkind == QKV_MASK_ADDITIVE) ? qkv::kDecExt : qkv::kDecPlain;
  if (!qkv::plan_decode(D, k->bits, k->group_size, k->fmt, out_dtype == QKV_F32, var, B,
                        Hkv * rows, Hkv, L, &plan))
    return fail(QKV_ERR_UNSUPPORTED,
                "no kernel for D=%d bits=%d group_size=%d%s", D, k->bits, k->group_size,
                (k->bits == 4 || k->bits == 8 || k->fmt == QKV_Q8_0)
                    ? "" : " (2/3/5/6-bit codes: no additive mask, extensions or fused update)");
  if (plan.ws_total > 0) {
    if (workspace == nullptr || workspace_bytes < plan.ws_total)
      return fail(QKV_ERR_WORKSPACE, "workspace of %zu bytes required (got %zu)", plan.ws_total,
                  workspace_bytes);
    if (!aligned16(workspace)) return fail(QKV_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  }
  qkv::DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = q; p.q_dtype = q_dtype; p.out = out; p.out_dtype = out_dtype;
  p.kc = reinterpret_cast<const uint8_t*>(k->codes); p.ks = k->scales; p.kb = k->biases;
  p.vc = reinterpret_cast<const uint8_t*>(v->codes); p.vs = v->scales; p.vb = v->biases;
  p.Lcap = k->Lcap; p.L = L;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.G = rows; p.Gq = G; p.Lq = Lq;
  p.scale_log2e = scale * 1.4426950408889634f;
  p.mask_kind = mkind;
  if (mkind == QKV_MASK_ADDITIVE) {
    p.mask = mask->add; p.mask_dtype = mask->add_dtype;
    p.msb = mask->stride_b; p.msh = mask->stride_h; p.msq = mask->stride_q;
  }
  if (mkind == QKV_MASK_CAUSAL && Lq == 1) p.mask_kind = QKV_MASK_NONE;  // all keys visible
  p.cap_a = cap_a; p.cap_k = cap_k; p.slopes = slopes; p.sinks = sinks;
  if (fused) {
    p.new_k = static_cast<const uint16_t*>(new_k);
    p.new_v = static_cast<const uint16_t*>(new_v);
    p.new_bf16 = in_dtype == QKV_BF16;
  }
  uint8_t* parts = static_cast<uint8_t*>(workspace) + plan.ws_header;
  p.part_o = reinterpret_cast<float*>(parts);
  p.part_ml = reinterpret_cast<float*>(parts + plan.ws_part_o);
  cudaError_t e = qkv::launch_decode(D, k->bits, k->group_size, k->fmt, out_dtype == QKV_F32,
                                     plan, p, s);
  if (e != cudaSuccess) return fail(QKV_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
  return ok();
}

qkv_status check_blocks_args(const qkv_cache* c, int B, int Hkv, int D, int64_t offset, int64_t L,
                             const void* blocks, int64_t sb, int64_t sh, int64_t sl,
                             int want_fmt = QKV_Q8_0, int want_bits = 8) {
  qkv_status st;
  if ((st = check_cache("cache", c, D)) != QKV_OK) return st;
  if (want_fmt == QKV_Q8_0 && c->fmt != QKV_Q8_0)
    return fail(QKV_ERR_UNSUPPORTED, "Q8_0 block conversion needs a Q8_0 cache");
  if (want_fmt == QKV_AFFINE && (c->fmt != QKV_AFFINE || c->group_size != 32 || c->bits != want_bits))
    return fail(QKV_ERR_UNSUPPORTED, "these blocks need an affine cache with group_size 32 and %d-bit codes",
                want_bits);
  if (B <= 0 || Hkv <= 0) return fail(QKV_ERR_INVALID_ARG, "B and Hkv must be positive");
  if (offset < 0 || L < 0 || offset + L > c->Lcap)
    return fail(QKV_ERR_INVALID_ARG, "rows [%lld, %lld) outside [0, Lcap]", (long long)offset,
                (long long)(offset + L));
  if (blocks == nullptr) return fail(QKV_ERR_INVALID_ARG, "blocks must be non-NULL");
  if (sb < 0 || sh < 0 || sl < 0) return fail(QKV_ERR_INVALID_ARG, "block strides must be non-negative");
  if ((reinterpret_cast<uintptr_t>(blocks) & 1u) != 0 || ((sb | sh | sl) & 1) != 0)
    return fail(QKV_ERR_ALIGNMENT, "blocks and their strides must be 2-byte aligned");
  return QKV_OK;
}

}  // namespace

extern "C" {

const char* qkv_status_string(int status) {
  switch (status) {
    case QKV_OK: return "ok";
    case QKV_ERR_INVALID_ARG: return "invalid argument";
    case QKV_ERR_UNSUPPORTED: return "unsupported";
    case QKV_ERR_ALIGNMENT: return "alignment";
    case QKV_ERR_WORKSPACE: return "workspace too small";
    case QKV_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

const char* qkv_last_error(void) { return g_last_error; }

size_t qsdpa_workspace_size(int B, int Hq, int Hkv, int Lq, int D, int64_t L) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0 || Hq % Hkv || L < 0) return 0;
  if (D != 64 && D != 128 && D != 256) return 0;
  return qkv::decode_workspace_bound(B, Hq * Lq, Hkv, D);
}

size_t qsdpa_workspace_zero_bytes(int B, int Hq, int Hkv, int Lq, int D, int64_t L) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0 || Hq % Hkv || L < 0) return 0;
  (void)D;
  return qkv::decode_workspace_zero_bytes(B, Hq * Lq, Hkv);
}

qkv_status qkv_quantize_update(const void* new_k, const void* new_v, int in_dtype, int B, int Hkv,
                               int Lnew, int D, const qkv_cache* k, const qkv_cache* v,
                               int64_t offset, void* stream) {
  qkv_status st;
  if (B <= 0 || Hkv <= 0 || Lnew < 0) return fail(QKV_ERR_INVALID_ARG, "B, Hkv must be positive, Lnew >= 0");
  if ((st = check_cache("k", k, D, true)) != QKV_OK) return st;
  if ((st = check_cache("v", v, D, true)) != QKV_OK) return st;
  if (in_dtype != QKV_F16 && in_dtype != QKV_BF16)
    return fail(QKV_ERR_INVALID_ARG, "new tokens must be f16 or bf16 (got %d)", in_dtype);
  if ((int64_t)B * Hkv > 65535)
    return fail(QKV_ERR_UNSUPPORTED, "B * Hkv must be at most 65535 (got %lld)", (long long)B * Hkv);
  if (Lnew == 0) return ok();
  if (new_k == nullptr || new_v == nullptr)
    return fail(QKV_ERR_INVALID_ARG, "new_k and new_v must be non-NULL");
  if (!aligned16(new_k) || !aligned16(new_v))
    return fail(QKV_ERR_ALIGNMENT, "new_k and new_v must be 16-byte aligned");
  if (offset < 0 || offset + Lnew > k->Lcap || offset + Lnew > v->Lcap)
    return fail(QKV_ERR_INVALID_ARG, "offset=%lld with Lnew=%d exceeds Lcap", (long long)offset, Lnew);
  cudaError_t e = qkv::launch_quantize(new_k, new_v, in_dtype, B, Hkv, Lnew, D, k, v, offset,
                                       static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(QKV_ERR_CUDA, "quantize launch: %s", cudaGetErrorString(e));
  return ok();
}

qkv_status qkv_dequantize(const qkv_cache* c, int B, int Hkv, int D, int64_t L, void* out,
                          void* stream) {
  qkv_status st;
  if ((st = check_cache("cache", c, D)) != QKV_OK) return st;
  if (B <= 0 || Hkv <= 0) return fail(QKV_ERR_INVALID_ARG, "B and Hkv must be positive");
  if ((int64_t)B * Hkv > 65535)
    return fail(QKV_ERR_UNSUPPORTED, "B * Hkv must be at most 65535 (got %lld)", (long long)B * Hkv);
  if (L < 0 || L > c->Lcap) return fail(QKV_ERR_INVALID_ARG, "L=%lld outside [0, Lcap]", (long long)L);
  if (L == 0) return ok();
  if (out == nullptr) return fail(QKV_ERR_INVALID_ARG, "out must be non-NULL");
  if (!aligned16(out)) return fail(QKV_ERR_ALIGNMENT, "out must be 16-byte aligned");
  cudaError_t e = qkv::launch_dequantize(c, B, Hkv, D, L, out, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(QKV_ERR_CUDA, "dequantize launch: %s", cudaGetErrorString(e));
  return ok();
}


qkv_status qkv_q8_0_from_blocks(const void* blocks, int B, int Hkv, int D, int64_t L,
                                int64_t stride_b, int64_t stride_h, int64_t stride_l,
                                const qkv_cache* dst, int64_t offset, void* stream) {
  qkv_status st = check_blocks_args(dst, B, Hkv, D, offset, L, blocks, stride_b, stride_h, stride_l);
  if (st != QKV_OK) return st;
  if (L == 0) return ok();
  cudaError_t e = qkv::launch_q8_0_blocks(false, blocks, nullptr, dst, B, Hkv, D, offset, L, stride_b,
                                          stride_h, stride_l, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(QKV_ERR_CUDA, "block conversion launch: %s", cudaGetErrorString(e));
  return ok();
}

qkv_status qkv_llama_blocks_to_cache(int kind, const void* blocks, int B, int Hkv, int D,
                                     int64_t L, int64_t stride_b, int64_t stride_h,
                                     int64_t stride_l, const qkv_cache* dst, int64_t offset,
                                     void* stream) {
  if (kind < QKV_BLOCKS_Q4_0 || kind > QKV_BLOCKS_Q5_1)
    return fail(QKV_ERR_INVALID_ARG, "unknown block kind %d", kind);
  const int bits = (kind == QKV_BLOCKS_Q4_0 || kind == QKV_BLOCKS_Q4_1) ? 4 : 8;
  qkv_status st = check_blocks_args(dst, B, Hkv, D, offset, L, blocks, stride_b, stride_h, stride_l,
                                    QKV_AFFINE, bits);
  if (st != QKV_OK) return st;
  if (L == 0) return ok();
  cudaError_t e = qkv::launch_llama_blocks(kind, blocks, dst, B, Hkv, D, offset, L, stride_b, stride_h,
                                           stride_l, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(QKV_ERR_CUDA, "block conversion launch: %s", cudaGetErrorString(e));
  return ok();
}

qkv_status qkv_llama_quantize_blocks(int kind, const void* x, int in_dtype, int B, int Hkv, int D,
                                     int64_t L, void* blocks, int64_t stride_b, int64_t stride_h,
                                     int64_t stride_l, void* stream) {
  if (kind < QKV_BLOCKS_Q4_0 || kind > QKV_BLOCKS_Q5_1)
    return fail(QKV_ERR_INVALID_ARG, "unknown block kind %d", kind);
  if (B <= 0 || Hkv <= 0 || L < 0) return fail(QKV_ERR_INVALID_ARG, "B, Hkv must be positive, L >= 0");
  if (D != 64 && D != 128 && D != 256)
    return fail(QKV_ERR_UNSUPPORTED, "head dimension must be 64, 128 or 256 (got %d)", D);
  if (in_dtype != QKV_F16 && in_dtype != QKV_BF16)
    return fail(QKV_ERR_INVALID_ARG, "x must be f16 or bf16 (got %d)", in_dtype);
  if (L == 0) return ok();
  if (x == nullptr || blocks == nullptr) return fail(QKV_ERR_INVALID_ARG, "x and blocks must be non-NULL");
  if (!aligned16(x)) return fail(QKV_ERR_ALIGNMENT, "x must be 16-byte aligned");
  if (stride_b < 0 || stride_h < 0 || stride_l < 0)
    return fail(QKV_ERR_INVALID_ARG, "block strides must be non-negative");
  if ((reinterpret_cast<uintptr_t>(blocks) & 1u) != 0 || ((stride_b | stride_h | stride_l) & 1) != 0)
    return fail(QKV_ERR_ALIGNMENT, "blocks and their strides must be 2-byte aligned");
  cudaError_t e = qkv::launch_llama_quantize(kind, x, in_dtype, B, Hkv, D, L, blocks, stride_b,
                                             stride_h, stride_l, nullptr, 0,
                                             static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(QKV_ERR_CUDA, "block quantize launch: %s", cudaGetErrorString(e));
  return ok();
}

qkv_status qkv_llama_quantize_update(int kind, const void* new_k, const void* new_v, int in_dtype,
                                     int B, int Hkv, int Lnew, int D, const qkv_cache* k,
                                     const qkv_cache* v, int64_t offset, void* stream) {
  if (kind < QKV_BLOCKS_Q4_0 || kind > QKV_BLOCKS_Q5_1)
    return fail(QKV_ERR_INVALID_ARG, "unknown block kind %d", kind);
  const int bits = (kind == QKV_BLOCKS_Q4_0 || kind == QKV_BLOCKS_Q4_1) ? 4 : 8;
  if (B <= 0 || Hkv <= 0 || Lnew < 0) return fail(QKV_ERR_INVALID_ARG, "B, Hkv must be positive, Lnew >= 0");
  qkv_status st;
  for (const qkv_cache* c : {k, v}) {
    if ((st = check_cache(c == k ? "k" : "v", c, D)) != QKV_OK) return st;
    if (c->fmt != QKV_AFFINE || c->group_size != 32 || c->bits != bits)
      return fail(QKV_ERR_UNSUPPORTED,
                  "these blocks need an affine cache with group_size 32 and %d-bit codes", bits);
  }
  if (in_dtype != QKV_F16 && in_dtype != QKV_BF16)
    return fail(QKV_ERR_INVALID_ARG, "new tokens must be f16 or bf16 (got %d)", in_dtype);
  if (offset < 0 || offset + Lnew > k->Lcap || offset + Lnew > v->Lcap)
    return fail(QKV_ERR_INVALID_ARG, "offset=%lld with Lnew=%d exceeds Lcap", (long long)offset, Lnew);
  if (Lnew == 0) return ok();
  if (new_k == nullptr || new_v == nullptr)
    return fail(QKV_ERR_INVALID_ARG, "new_k and new_v must be non-NULL");
  if (!aligned16(new_k) || !aligned16(new_v))
    return fail(QKV_ERR_ALIGNMENT, "new_k and new_v must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = qkv::launch_llama_quantize(kind, new_k, in_dtype, B, Hkv, D, Lnew, nullptr, 0, 0, 0,
                                             k, offset, s);
  if (e == cudaSuccess)
    e = qkv::launch_llama_quantize(kind, new_v, in_dtype, B, Hkv, D, Lnew, nullptr, 0, 0, 0, v,
                                   offset, s);
  if (e != cudaSuccess) return fail(QKV_ERR_CUDA, "block quantize launch: %s", cudaGetErrorString(e));
  return ok();
}

qkv_status qkv_llama_cache_to_blocks(int kind, const qkv_cache* src, int B, int Hkv, int D,
                                     int64_t offset, int64_t L, void* blocks, int64_t stride_b,
                                     int64_t stride_h, int64_t stride_l, void* stream) {
  if (kind < QKV_BLOCKS_Q4_0 || kind > QKV_BLOCKS_Q5_1)
    return fail(QKV_ERR_INVALID_ARG, "unknown block kind %d", kind);
  const int bits = (kind == QKV_BLOCKS_Q4_0 || kind == QKV_BLOCKS_Q4_1) ? 4 : 8;
  qkv_status st = check_blocks_args(src, B, Hkv, D, offset, L, blocks, stride_b, stride_h, stride_l,
                                    QKV_AFFINE, bits);
  if (st != QKV_OK) return st;
  if (L == 0) return ok();
  cudaError_t e = qkv::launch_llama_export(kind, src, B, Hkv, D, offset, L, blocks, stride_b,
                                           stride_h, stride_l, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(QKV_ERR_CUDA, "block export launch: %s", cudaGetErrorString(e));
  return ok();
}

qkv_status qkv_q8_0_to_blocks(const qkv_cache* src, int B, int Hkv, int D, int64_t offset, int64_t L,
                              void* blocks, int64_t stride_b, int64_t stride_h, int64_t stride_l,
                              void* stream) {
  qkv_status st = check_blocks_args(src, B, Hkv, D, offset, L, blocks, stride_b, stride_h, stride_l);
  if (st != QKV_OK) return st;
  if (L == 0) return ok();
  cudaError_t e = qkv::launch_q8_0_blocks(true, nullptr, blocks, src, B, Hkv, D, offset, L, stride_b,
                                          stride_h, stride_l, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(QKV_ERR_CUDA, "block conversion launch: %s", cudaGetErrorString(e));
  return ok();
}

qkv_status qsdpa_decode(const void* q, int q_dtype, int B, int Hq, int Hkv, int D,
                        const qkv_cache* k, const qkv_cache* v, int64_t L, float scale,
                        const qkv_mask* mask, void* out, int out_dtype, void* workspace,
                        size_t workspace_bytes, void* stream) {
  return attention(q, q_dtype, B, Hq, Hkv, 1, D, k, v, L, scale, mask, out, out_dtype, workspace,
                   workspace_bytes, stream);
}

qkv_status qsdpa_decode_update(const void* q, int q_dtype, const void* new_k, const void* new_v,
                               int in_dtype, int B, int Hq, int Hkv, int D, const qkv_cache* k,
                               const qkv_cache* v, int64_t L_old, float scale,
                               const qkv_mask* mask, void* out, int out_dtype, void* workspace,
                               size_t workspace_bytes, void* stream) {
  qkv_status st;
  if ((st = check_cache("k", k, D)) != QKV_OK) return st;
  if ((st = check_cache("v", v, D)) != QKV_OK) return st;
  if (in_dtype != QKV_F16 && in_dtype != QKV_BF16)
    return fail(QKV_ERR_INVALID_ARG, "new tokens must be f16 or bf16 (got %d)", in_dtype);
  if (new_k == nullptr || new_v == nullptr)
    return fail(QKV_ERR_INVALID_ARG, "new_k and new_v must be non-NULL");
  if (!aligned16(new_k) || !aligned16(new_v))
    return fail(QKV_ERR_ALIGNMENT, "new_k and new_v must be 16-byte aligned");
  if (L_old < 0 || L_old + 1 > k->Lcap || L_old + 1 > v->Lcap)
    return fail(QKV_ERR_INVALID_ARG, "L_old=%lld: the new token does not fit Lcap", (long long)L_old);
  return attention(q, q_dtype, B, Hq, Hkv, 1, D, k, v, L_old + 1, scale, mask, out, out_dtype,
                   workspace, workspace_bytes, stream, new_k, new_v, in_dtype);
}

qkv_status qsdpa_prefill(const void* q, int q_dtype, int B, int Hq, int Hkv, int Lq, int D,
                         const qkv_cache* k, const qkv_cache* v, int64_t L, float scale,
                         const qkv_mask* mask, void* out, int out_dtype, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return attention(q, q_dtype, B, Hq, Hkv, Lq, D, k, v, L, scale, mask, out, out_dtype, workspace,
                   workspace_bytes, stream);
}

size_t qsdpa_kview_workspace_size(int B, int Hq, int Hkv, int Lq, int Dk, int Dv, int64_t L) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0 || Hq % Hkv || L < 0) return 0;
  if (Dk != 576 || Dv != 512) return 0;
  return qkv::kview_workspace_bytes();
}

qkv_status qsdpa_attention_kview(const void* q, int q_dtype, int B, int Hq, int Hkv, int Lq, int Dk,
                                 int Dv, const qkv_cache* k, int64_t L, float scale,
                                 const qkv_mask* mask, void* out, int out_dtype, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0)
    return fail(QKV_ERR_INVALID_ARG, "B, Hq, Hkv and Lq must be positive");
  if (Hq % Hkv != 0) return fail(QKV_ERR_INVALID_ARG, "Hq=%d is not a multiple of Hkv=%d", Hq, Hkv);
  if (Dk != 576 || Dv != 512)
    return fail(QKV_ERR_UNSUPPORTED, "values as a view of the keys: Dk=576, Dv=512 (got %d/%d)", Dk, Dv);
  if (k == nullptr) return fail(QKV_ERR_INVALID_ARG, "k: cache descriptor is NULL");
  if (k->fmt == QKV_Q8_0) {
    if (k->bits != 8 || k->group_size != 32)
      return fail(QKV_ERR_INVALID_ARG, "k: Q8_0 needs bits 8 and group_size 32");
  } else if (k->fmt == QKV_AFFINE) {
    if ((k->bits != 4 && k->bits != 8) || (k->group_size != 32 && k->group_size != 64))
      return fail(QKV_ERR_UNSUPPORTED, "k: the view kernel takes affine 4- or 8-bit codes in groups "
                  "of 32 or 64 (got %d bits, group %d)", k->bits, k->group_size);
    if (k->biases == nullptr) return fail(QKV_ERR_INVALID_ARG, "k: affine cache needs biases");
  } else {
    return fail(QKV_ERR_INVALID_ARG, "k: unknown format %d", k->fmt);
  }
  if (k->codes == nullptr || k->scales == nullptr)
    return fail(QKV_ERR_INVALID_ARG, "k: codes and scales must be non-NULL");
  if (k->Lcap <= 0 || k->Lcap % 8 != 0)
    return fail(k->Lcap <= 0 ? QKV_ERR_INVALID_ARG : QKV_ERR_ALIGNMENT,
                "k: Lcap must be a positive multiple of 8 (got %lld)", (long long)k->Lcap);
  if (!aligned16(k->codes) || !aligned16(k->scales) || (k->fmt == QKV_AFFINE && !aligned16(k->biases)))
    return fail(QKV_ERR_ALIGNMENT, "k: codes, scales and biases must be 16-byte aligned");
  if (L < 0 || L > k->Lcap) return fail(QKV_ERR_INVALID_ARG, "L=%lld outside [0, Lcap]", (long long)L);
  qkv_status st;
  if ((st = check_dtype("q", q_dtype, false)) != QKV_OK) return st;
  if (out_dtype != QKV_F16 && out_dtype != QKV_BF16)
    return fail(out_dtype == QKV_F32 ? QKV_ERR_UNSUPPORTED : QKV_ERR_INVALID_ARG,
                "out: f16 or bf16 (the view kernel's tiles are fp16: no fp32-accurate output)");
  if (q == nullptr || out == nullptr) return fail(QKV_ERR_INVALID_ARG, "q and out must be non-NULL");
  if (!aligned16(q) || !aligned16(out)) return fail(QKV_ERR_ALIGNMENT, "q and out must be 16-byte aligned");
  if (!(scale == scale)) return fail(QKV_ERR_INVALID_ARG, "scale is NaN");
  int mkind = mask == nullptr ? QKV_MASK_NONE : mask->kind;
  if (mkind == QKV_MASK_ADDITIVE)
    return fail(QKV_ERR_UNSUPPORTED, "the view kernel takes no additive mask (none or causal)");
  if (mkind != QKV_MASK_NONE && mkind != QKV_MASK_CAUSAL)
    return fail(QKV_ERR_INVALID_ARG, "unknown mask kind %d", mkind);
  if ((int64_t)Hq * Lq > (int64_t)1 << 30) return fail(QKV_ERR_INVALID_ARG, "Hq * Lq too large");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (L == 0) {
    if (cudaMemsetAsync(out, 0, (size_t)B * Hq * Lq * Dv * 2, s) != cudaSuccess)
      return fail(QKV_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(cudaGetLastError()));
    return ok();
  }
  const size_t need = qkv::kview_workspace_bytes();
  if (workspace == nullptr || workspace_bytes < need)
    return fail(QKV_ERR_WORKSPACE, "workspace of %zu bytes required (got %zu)", need, workspace_bytes);
  if (!aligned16(workspace)) return fail(QKV_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  qkv::DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = q; p.q_dtype = q_dtype; p.out = out; p.out_dtype = out_dtype;
  p.kc = reinterpret_cast<const uint8_t*>(k->codes); p.ks = k->scales; p.kb = k->biases;
  p.Lcap = k->Lcap; p.L = L;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Gq = Hq / Hkv; p.Lq = Lq; p.G = (Hq / Hkv) * Lq;
  p.scale_log2e = scale * 1.4426950408889634f;
  p.mask_kind = (mkind == QKV_MASK_CAUSAL && Lq > 1) ? QKV_MASK_CAUSAL : QKV_MASK_NONE;
  p.part_o = static_cast<float*>(workspace);
  cudaError_t e = qkv::launch_kview(k->bits, k->group_size, k->fmt, p, s);
  if (e != cudaSuccess) return fail(QKV_ERR_CUDA, "view attention launch: %s", cudaGetErrorString(e));
  return ok();
}

qkv_status qsdpa_decode_ext(const void* q, int q_dtype, int B, int Hq, int Hkv, int D,
                            const qkv_cache* k, const qkv_cache* v, int64_t L, float scale,
                            const qkv_mask* mask, const qkv_attn_ext* ext, void* out,
                            int out_dtype, void* workspace, size_t workspace_bytes,
                            void* stream) {
  return attention(q, q_dtype, B, Hq, Hkv, 1, D, k, v, L, scale, mask, out, out_dtype, workspace,
                   workspace_bytes, stream, nullptr, nullptr, QKV_F16, ext);
}

qkv_status qsdpa_prefill_ext(const void* q, int q_dtype, int B, int Hq, int Hkv, int Lq, int D,
                             const qkv_cache* k, const qkv_cache* v, int64_t L, float scale,
                             const qkv_mask* mask, const qkv_attn_ext* ext, void* out,
                             int out_dtype, void* workspace, size_t workspace_bytes,
                             void* stream) {
  return attention(q, q_dtype, B, Hq, Hkv, Lq, D, k, v, L, scale, mask, out, out_dtype, workspace,
                   workspace_bytes, stream, nullptr, nullptr, QKV_F16, ext);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free decode entry point.
//
// Some callers cannot allocate device memory at the point where they decode:
// code running inside a memory pool that forbids cudaMalloc/cudaFree, hosts
// that pre-plan every buffer before serving starts, or plug-in interfaces that
// only hand over input and output pointers.  For them, qsdpa_decode_noalloc
// runs the same decode kernel as qsdpa_decode but keeps its scratch (the
// partial results of the split over L) in a
// fixed-size array that lives in this library's device image.  Every GPU that
// loads the library holds that array until the process exits.
// ---------------------------------------------------------------------------
#include <mutex>

namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;    // 8 MiB per device
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of the scratch array for the current device.  Taken once per
// device with that device current (the host-side symbol is only a stand-in and
// must never be handed to a kernel).
qkv_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(QKV_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return fail(QKV_ERR_UNSUPPORTED, "device %d beyond the %d devices supported", dev,
                kNoAllocMaxDevices);
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(QKV_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return QKV_OK;
}

}  // namespace

extern "C" qkv_status qsdpa_decode_noalloc(const void* q, int q_dtype, int B, int Hq, int Hkv,
                                           int D, const qkv_cache* k, const qkv_cache* v,
                                           int64_t L, float scale, const qkv_mask* mask,
                                           void* out, int out_dtype, void* stream) {
  // the checks qsdpa_decode makes first, in its order, so that both entry
  // points return the same status for a shape neither can run
  if (B <= 0 || Hq <= 0 || Hkv <= 0)
    return fail(QKV_ERR_INVALID_ARG, "B, Hq, Hkv and Lq must be positive");
  if (Hq % Hkv != 0) return fail(QKV_ERR_INVALID_ARG, "Hq=%d is not a multiple of Hkv=%d", Hq, Hkv);
  qkv_status st;
  if ((st = check_cache("k", k, D)) != QKV_OK) return st;
  if ((st = check_cache("v", v, D)) != QKV_OK) return st;
  if (L < 0 || L > k->Lcap) return fail(QKV_ERR_INVALID_ARG, "L=%lld outside [0, Lcap]", (long long)L);
  const size_t need = qsdpa_workspace_size(B, Hq, Hkv, 1, D, L);
  if (need == 0) return fail(QKV_ERR_INVALID_ARG, "invalid decode shape (D=%d, L=%lld)", D,
                             (long long)L);
  if (need > kNoAllocScratchBytes)
    return fail(QKV_ERR_WORKSPACE,
                "qsdpa_decode_noalloc: this shape needs %zu bytes of scratch, more than the "
                "%zu bytes built into the library; use qsdpa_decode with a caller workspace",
                need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != QKV_OK) return st;
  // decode keeps no state in its scratch between calls (the header that
  // qsdpa_workspace_zero_bytes covers is the prefill's), so nothing to clear
  return qsdpa_decode(q, q_dtype, B, Hq, Hkv, D, k, v, L, scale, mask, out, out_dtype, scratch,
                      kNoAllocScratchBytes, stream);
}
