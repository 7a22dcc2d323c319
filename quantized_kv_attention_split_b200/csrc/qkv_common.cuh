// qkv_common.cuh -- small device helpers shared by the libqkv kernels
// (sm_100a).  Inline PTX wrappers for cp.async staging, the m16n8k16 tensor
// instruction, the 8x8 fragment transpose, byte permutes and exp2.
#pragma once

#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/qkv.h"

namespace qkv {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global->shared copy; src_bytes 0 fills the destination with zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n"
               :: "r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" :: "n"(N) : "memory");
}

// D = A(16x16, f16, row) * B(16x8, f16, col) + C, fp32 accumulate.
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4],
                                        uint32_t b0, uint32_t b1, const float (&c)[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1),
        "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]));
}

// Transpose of an 8x8 matrix of 16-bit values held one row-pair per thread
// (thread l holds row l/4, columns 2*(l%4), 2*(l%4)+1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// Logit softcap applied to a base-2 logit S = log2(e) x: returns
// log2(e) c tanh(x / c).  From tanh(y) = 1 - 2 / (1 + e^(2y)) with y = x / c:
// e^(2y) = 2^(S k) for k = 2 / c, so the result is a - 2a / (1 + 2^(S k)) with
// a = c log2(e).  The exponent is clamped at 64 (the quotient is then below
// 2^-60 a) so no infinity enters the division; the absolute error is a few
// units of a * 2^-23, from ex2.approx and the approximate division.
__device__ __forceinline__ float softcap_log2(float S, float a, float k) {
  return a - __fdividef(2.f * a, 1.f + ex2(fminf(S * k, 64.f)));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  return __byte_perm(a, b, sel);
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_half2(uint32_t x) {
  __half2 h = *reinterpret_cast<__half2*>(&x);
  return __half22float2(h);
}
__device__ __forceinline__ float half_bits_to_float(uint16_t b) {
  return __half2float(__ushort_as_half(b));
}

// Load element i of a 16-bit (f16/bf16) or fp32 tensor as float.
__device__ __forceinline__ float load_as_float(const void* p, int dtype, int64_t i) {
  if (dtype == QKV_F16) return __half2float(reinterpret_cast<const __half*>(p)[i]);
  if (dtype == QKV_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  return reinterpret_cast<const float*>(p)[i];
}
// Read-only loads of one mask element as fp32.
__device__ __forceinline__ float to_float_ld(const float* p) { return __ldg(p); }
__device__ __forceinline__ float to_float_ld(const __half* p) { return __half2float(__ldg(p)); }
__device__ __forceinline__ float to_float_ld(const __nv_bfloat16* p) {
  return __bfloat162float(__ldg(p));
}
__device__ __forceinline__ void store_from_float(void* p, int dtype, int64_t i, float v) {
  if (dtype == QKV_F16) reinterpret_cast<__half*>(p)[i] = __float2half_rn(v);
  else if (dtype == QKV_BF16) reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else reinterpret_cast<float*>(p)[i] = v;
}

// Four consecutive outputs i..i+3 (i a multiple of 4, the buffer 16-byte
// aligned) in one 8- or 16-byte store: fewer, wider writes, which matters
// most when out is host memory written over the host link.
__device__ __forceinline__ void store4_from_float(void* p, int dtype, int64_t i, float4 v) {
  if (dtype == QKV_F32) {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(p) + i) = v;
    return;
  }
  uint2 w;
  if (dtype == QKV_F16) {
    const __half2 a = __floats2half2_rn(v.x, v.y), b = __floats2half2_rn(v.z, v.w);
    w = make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
  } else {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    w = make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
  }
  *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(p) + i) = w;
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel of the stream is still
// running; grid_dep_wait() returns once that kernel has completed and its
// memory operations are visible, and grid_dep_launch() lets the next kernel
// of the stream start early (it still waits in its own grid_dep_wait()).
// Both are no-ops for a normal launch.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// Bulk prefetch of [a, a + bytes) into L2 (a 16-byte aligned, bytes a multiple
// of 16; no data returned, no fault).
__device__ __forceinline__ void prefetch_l2_bulk(const void* a, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" :: "l"(a), "r"(bytes) : "memory");
}

// a / b for non-negative 64-bit values, in 32-bit arithmetic when both fit
// (the common case; 64-bit division costs several times more instructions).
__device__ __forceinline__ int64_t udiv64(int64_t a, int64_t b) {
  if (((uint64_t)a | (uint64_t)b) >> 32 == 0) return (int64_t)((uint32_t)a / (uint32_t)b);
  return a / b;
}

// 2^k as float for integer k in [-126, 127].
__device__ __forceinline__ float exp2i(int k) {
  return __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
}

}  // namespace qkv
