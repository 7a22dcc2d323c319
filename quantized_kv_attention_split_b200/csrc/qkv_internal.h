// qkv_internal.h -- parameter blocks and launcher declarations shared between
// the C-ABI front end (api.cu) and the kernel translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/qkv.h"

namespace qkv {

// Everything one decode launch needs (device pointers and sizes).
// Decode kernel variants: the plain kernel (no mask, or causal), the fused
// update step (also quantizes the new token into cache row L - 1; any mask)
// and the one for additive masks and the attention extensions (logit softcap,
// additive-mask slopes, sinks).
enum : int { kDecPlain = 0, kDecFused = 1, kDecExt = 2 };

struct DecodeParams {
  const void* q;            // [B, Hq, 1, D]
  int q_dtype;
  void* out;                // [B, Hq, 1, D]
  int out_dtype;
  const uint8_t* kc;        // K codes, bytes
  const uint16_t* ks;       // K scales
  const uint16_t* kb;       // K biases (affine)
  const uint8_t* vc;
  const uint16_t* vs;
  const uint16_t* vb;
  int64_t Lcap;
  int64_t L;
  int B, Hq, Hkv;
  int G;                    // rows per kv head: (query heads per kv head) * Lq
  int Gq;                   // query heads per kv head
  int Lq;                   // queries per head (row r = head * Lq + query)
  int ncg;                  // row chunk-groups (of up to 32 rows) per kv head
  float scale_log2e;        // softmax scale times log2(e)
  // mask: kind 0 none, 1 causal (bottom-right aligned), 2 additive
  int mask_kind;
  const void* mask;
  int mask_dtype;
  int64_t msb, msh, msq;
  // extensions: softcap of the base-2 logit S -> cap_a - 2 cap_a / (1 + 2^(S cap_k))
  // (cap_a = softcap * log2(e), cap_k = 2 / softcap; cap_a == 0: off), per-head
  // additive-mask slopes and sink logits (fp32 [Hq], may be null)
  float cap_a, cap_k;
  const float* slopes;
  const float* sinks;
  // work split: units (b, kv-head, chunk-group) x blocks of TK keys, divided
  // evenly over gridDim.x CTAs
  int64_t stages_per_unit;
  int64_t total_stages;
  int pieces;               // CTAs per unit when every CTA covers one piece of one unit, else 0
  // fused update: the new token of every (batch, kv head), [B * Hkv, D]
  // fp16/bf16 bits, is quantized into cache row L - 1 (null: plain decode)
  const uint16_t* new_k;
  const uint16_t* new_v;
  int new_bf16;
  float* part_o;            // [2 * nCTA][HPC][D]   per-CTA partials
  float* part_ml;           // [2 * nCTA][HPC][2]
};

struct DecodePlan {
  int tk;                   // keys per stage
  int nc;                   // head chunks (of 8) per CTA
  int hpc;                  // heads per chunk-group slot (nc * 8)
  int ncg;
  int64_t units;
  int64_t stages_per_unit;
  int64_t total_stages;
  int grid;
  int var;                  // kDecPlain, kDecFused or kDecExt
  int pieces;               // CTAs per unit when the grid cuts every unit alike, else 0
  bool merge;               // some unit is split over several CTAs: merge kernel after
  size_t smem;
  size_t ws_header;         // bytes before the partials (zero between calls)
  size_t ws_part_o;         // bytes of one partial array
  size_t ws_part_ml;        // bytes
  size_t ws_total;
};

// Plans a decode launch for the current device; returns false if the shape
// has no kernel instance.
bool plan_decode(int D, int bits, int gs, int fmt, int out_f32, int var, int B, int Hq,
                 int Hkv, int64_t L, DecodePlan* plan);
cudaError_t launch_decode(int D, int bits, int gs, int fmt, int out_f32,
                          const DecodePlan& plan, DecodeParams& p, cudaStream_t stream);

// Rows [0, L) of a cache as fp16 [B * Hkv, L, D] (dequantize.cu).
cudaError_t launch_dequantize(const qkv_cache* c, int B, int Hkv, int D, int64_t L, void* out,
                              cudaStream_t stream);
cudaError_t launch_llama_blocks(int kind, const void* src_blocks, const qkv_cache* c, int B, int Hkv,
                                int D, int64_t offset, int64_t L, int64_t sb, int64_t sh,
                                int64_t sl, cudaStream_t stream);
// Attention whose values are the first 512 elements of 576-element keys
// (kview.cu): plans the split and launches (p: the decode parameters with the
// key cache, G = rows per kv head, part_o = the workspace).
cudaError_t launch_kview(int bits, int gs, int fmt, DecodeParams& p, cudaStream_t s);
size_t kview_workspace_bytes();

cudaError_t launch_llama_quantize(int kind, const void* x, int in_dtype, int B, int Hkv, int D,
                                  int64_t L, void* blocks, int64_t sb, int64_t sh, int64_t sl,
                                  const qkv_cache* c, int64_t offset, cudaStream_t stream);
cudaError_t launch_llama_export(int kind, const qkv_cache* c, int B, int Hkv, int D, int64_t offset,
                                int64_t L, void* blocks, int64_t sb, int64_t sh, int64_t sl,
                                cudaStream_t stream);
cudaError_t launch_q8_0_blocks(bool to_blocks, const void* src_blocks, void* dst_blocks,
                               const qkv_cache* c, int B, int Hkv, int D, int64_t offset, int64_t L,
                               int64_t sb, int64_t sh, int64_t sl, cudaStream_t stream);

}  // namespace qkv
