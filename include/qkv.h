/*
 * qkv.h -- C ABI of libqkv.so: scaled-dot-product attention over a
 * group-quantized KV cache, and the quantizer that appends tokens to it,
 * for NVIDIA B200 (sm_100a).
 *
 * Sources the operations follow (web pages, by title and section):
 *  - MLX compare "v0.19.3...quantized-kv-update" ("add
 *    fast::quantized_kv_update"): mlx/fast.h declarations of
 *    quantized_scaled_dot_product_attention(q, k, k_scales, k_biases, v,
 *    v_scales, v_biases, scale, mask, group_size, bits) and kv_update(...);
 *    mlx/fast.cpp (the fallback defines the math); sdpa_vector.h
 *    quant_sdpa_vector (packing, dequant, GQA mapping); quantized.h kv_update
 *    and affine_quantize_impl (eps 1e-7).
 *  - llama.cpp PR #25556 "Metal: Optimize q8_0 KV": the Q8_0 KV format; its
 *    merged follow-up: the attention variants its tests cover (sinks, ALiBi,
 *    logit softcap) and the other KV block types (Q4_0, Q4_1, Q5_0, Q5_1).
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller, with one
 *    exception: q and out of the attention calls (qsdpa_decode, _ext,
 *    _update, _noalloc, qsdpa_prefill, _ext) may instead point to page-locked
 *    host memory that the device addresses at the same pointer (cudaHostAlloc
 *    or cudaMallocHost memory, or cudaHostRegister'ed memory, on a host with
 *    unified addressing).  The split-K kernels then read q and write out over
 *    the host link themselves, with no separate copy, and a multi-query call
 *    with such a q or out runs on the split-K kernel.  Any other host address
 *    (pageable memory) returns QKV_ERR_INVALID_ARG before anything is
 *    launched.  The library never allocates device memory and never
 *    synchronizes: work is enqueued on `stream` (a cudaStream_t; NULL =
 *    legacy default stream).
 *  - Half-precision values are passed as their 16-bit patterns.
 *  - Arguments are validated before anything is launched.  On any error the
 *    call returns a status other than QKV_OK, launches nothing, and
 *    qkv_last_error() (per host thread) describes the problem.  Errors
 *    reported by the CUDA runtime at launch return QKV_ERR_CUDA.
 *  - No exception crosses this interface and nothing is printed.
 *
 * Cache layout (qkv_cache): one struct describes one of K or V.
 *  - codes  uint32 [B, Hkv, Lcap, D*bits/32], row-major.  Element e of a row
 *           is stored at bits [(e % (32/bits))*bits, ...+bits) of word
 *           e / (32/bits): low bits first (the pages' load_keys order).
 *           Affine codes are unsigned; Q8_0 codes are two's-complement int8.
 *  - scales fp16 [B, Hkv, Lcap, D/group_size]
 *  - biases fp16 [B, Hkv, Lcap, D/group_size] (affine only; NULL for Q8_0)
 *  - dequantized value = scale * code + bias (affine) or scale * code (Q8_0).
 *  - Lcap is the row capacity per (batch, kv-head); a call uses rows [0, L).
 *    Lcap must be a multiple of 8 and every pointer 16-byte aligned
 *    (QKV_ERR_ALIGNMENT otherwise).
 *  - Supported: affine bits 2, 3, 4, 5, 6 or 8 with group_size 32, 64 or
 *    128; Q8_0 (bits 8, group_size 32); D in {64, 128, 256} with
 *    D % group_size == 0 (and D = 576 for qsdpa_attention_kview and the
 *    quantizer).  Codes of 3, 5 and 6 bits straddle words (the rule above
 *    read as one little-endian bit stream per row: element e at bits
 *    [e*bits, (e+1)*bits)).  With 2, 3, 5 or 6-bit codes the attention
 *    calls take no additive mask, no extensions and no fused update
 *    (QKV_ERR_UNSUPPORTED), and multi-query calls run on the split-K kernel.
 */
#ifndef QKV_H_
#define QKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QKV_OK = 0,
  QKV_ERR_INVALID_ARG = 1,   /* bad shape, NULL pointer, out-of-range value   */
  QKV_ERR_UNSUPPORTED = 2,   /* valid request this build does not implement   */
  QKV_ERR_ALIGNMENT = 3,     /* pointer or Lcap alignment requirement not met */
  QKV_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required    */
  QKV_ERR_CUDA = 5           /* the CUDA runtime reported an error            */
} qkv_status;

typedef enum { QKV_F16 = 0, QKV_BF16 = 1, QKV_F32 = 2 } qkv_dtype;
typedef enum { QKV_AFFINE = 0, QKV_Q8_0 = 1 } qkv_format;
typedef enum { QKV_MASK_NONE = 0, QKV_MASK_CAUSAL = 1, QKV_MASK_ADDITIVE = 2 } qkv_mask_kind;

typedef struct {
  int fmt;              /* qkv_format                                         */
  int bits;             /* affine: 2, 3, 4, 5, 6 or 8; Q8_0: 8                */
  int group_size;       /* affine: 32, 64 or 128; Q8_0: 32                    */
  uint32_t* codes;      /* [B, Hkv, Lcap, D*bits/32]                          */
  uint16_t* scales;     /* fp16 [B, Hkv, Lcap, D/group_size]                  */
  uint16_t* biases;     /* fp16, same shape; NULL for Q8_0                    */
  int64_t Lcap;         /* rows per (batch, kv-head); multiple of 8           */
} qkv_cache;

/* Optional mask (pass NULL for none).
 *  - QKV_MASK_CAUSAL: query i of Lq sees key j iff j <= L - Lq + i (aligned to
 *    the bottom-right, i.e. the queries are the last Lq positions).
 *  - QKV_MASK_ADDITIVE: logit(b,h,i,j) += add[b*stride_b + h*stride_h +
 *    i*stride_q + j] (element strides; 0 broadcasts), dtype add_dtype; -inf
 *    hides a key.  The mask is added after `scale` (the pages' fallback adds
 *    it to q*scale . K^T).
 * A query row that sees no key returns zeros. */
typedef struct {
  int kind;             /* qkv_mask_kind */
  const void* add;
  int add_dtype;        /* qkv_dtype */
  int64_t stride_b, stride_h, stride_q;
} qkv_mask;

/* Optional attention extensions (pass NULL for none).  The llama.cpp PR's
 * tests cover these variants of flash attention (sinks, ALiBi, logit
 * softcap); the pages print no formula, so this library takes the usual
 * definitions (the CPU oracle states the same):
 *  softcap > 0:  the scaled logit x = scale * q.k becomes softcap*tanh(x/softcap),
 *                before the mask is added (Gemma-2 style logit capping);
 *                0 = off.  Must be finite and >= 0.
 *  mask_slopes:  device fp32 [Hq] or NULL: with an additive mask, query head h
 *                adds mask_slopes[h] * mask (a -inf entry still hides the key;
 *                ignored without an additive mask).  ALiBi is this with a mask
 *                holding minus the query-key distance and the slopes of
 *                Press et al. (2^(-8(h+1)/Hq) for a power-of-two Hq).
 *  sinks:        device fp32 [Hq] or NULL: a per-head logit s_h that joins the
 *                softmax denominator with no value row (gpt-oss style
 *                attention sinks): out = sum_j e^(x_j - M) v_j /
 *                (sum_j e^(x_j - M) + e^(s_h - M)), M = max(max_j x_j, s_h).
 *                A query row with no visible key still returns zeros.
 * Both arrays must be 4-byte aligned and stay valid until the call's kernels
 * have run.  They cost the kernels nothing when absent; softcap adds one
 * exp2 and one division per logit. */
typedef struct {
  float softcap;
  const float* mask_slopes;
  const float* sinks;
} qkv_attn_ext;

/* Quantize Lnew new tokens per (batch, kv-head) and write them into rows
 * [offset, offset+Lnew) of the K and V caches, in place (MLX kv_update /
 * KVUpdate::eval_gpu; the pages copy the whole cache first, this library
 * updates the caller's buffers in place).
 *  new_k, new_v: [B, Hkv, Lnew, D] contiguous, dtype in_dtype (f16 or bf16).
 *  Per group of group_size elements along D (fp32 IEEE, this order):
 *   affine: mn, mx = min, max; s = (mx-mn)/(2^bits-1); s = max(s, 1e-7);
 *           scale = fp16_rne(s); bias = fp16_rne(mn);
 *           code = clamp(rint((x - bias)/scale), 0, 2^bits-1)
 *   Q8_0:   d = max|x|/127; scale = fp16_rne(d);
 *           code = scale == 0 ? 0 : clamp(rint(x/scale), -127, 127)
 *  The result is bit-identical to the CPU oracle.  D is 64, 128, 256 or 576
 *  (the key rows of qsdpa_attention_kview).  Requires
 *  0 <= offset <= Lcap - Lnew and B*Hkv <= 65535 (QKV_ERR_UNSUPPORTED
 *  otherwise).  k and v may use different formats (then K and V are two
 *  launches, else one). */
qkv_status qkv_quantize_update(const void* new_k, const void* new_v, int in_dtype,
                               int B, int Hkv, int Lnew, int D,
                               const qkv_cache* k, const qkv_cache* v,
                               int64_t offset, void* stream);

/* Single-query attention (Lq = 1): out = softmax(q*scale . K^T + mask) V over
 * keys [0, L) of the dequantized cache (MLX quant_sdpa_vector semantics, plus
 * GQA, masks and a split over L).
 *  q:   [B, Hq, 1, D] contiguous, q_dtype f16 or bf16.
 *  out: [B, Hq, 1, D] contiguous, out_dtype f16, bf16 or f32.
 *  Hq % Hkv == 0; query head h reads kv-head h / (Hq/Hkv).
 *  workspace: device scratch of at least qsdpa_workspace_size(...) bytes,
 *  16-byte aligned; decode keeps no state in it between calls.  Calls that
 *  share a workspace must not overlap on the GPU.  One kernel launch, or two
 *  when the keys of a (batch, kv-head) are split over several CTAs (the
 *  second merges their partial results); both are programmatic dependent
 *  launches, whose set-up may overlap the previous kernel of the stream (they
 *  read no input and write nothing before that kernel has completed).
 *  L == 0 writes zeros.  Accuracy: max-abs error vs fp64 <= 2e-3 for f16/bf16
 *  out, <= 1e-4 for f32 out (values of order one). */
qkv_status qsdpa_decode(const void* q, int q_dtype, int B, int Hq, int Hkv, int D,
                        const qkv_cache* k, const qkv_cache* v, int64_t L,
                        float scale, const qkv_mask* mask, void* out, int out_dtype,
                        void* workspace, size_t workspace_bytes, void* stream);

/* Fused decode step (the pages' two calls -- the cache update of the new
 * token, then single-query attention -- in one decode launch; the pages have
 * no fused form).  The new token of every (batch, kv head), new_k / new_v
 * [B, Hkv, 1, D] contiguous in in_dtype (f16 or bf16, 16-byte aligned), is
 * quantized into cache row L_old exactly as qkv_quantize_update(.., Lnew = 1,
 * offset = L_old) would write it, and out is qsdpa_decode over the
 * L_old + 1 keys [0, L_old] that then hold.  Requires L_old + 1 <= Lcap.
 * Same workspace rules, launches and accuracy as qsdpa_decode; the cache row
 * is written by the decode kernel, so it must not be read by another kernel
 * that runs concurrently on the GPU. */
qkv_status qsdpa_decode_update(const void* q, int q_dtype, const void* new_k, const void* new_v,
                               int in_dtype, int B, int Hq, int Hkv, int D, const qkv_cache* k,
                               const qkv_cache* v, int64_t L_old, float scale,
                               const qkv_mask* mask, void* out, int out_dtype, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Multi-query attention (any Lq >= 1) over keys [0, L) with an optional mask
 * (the pages' Lq > 1 fallback: quantized_matmul -> softmax -> quantized_matmul,
 * computed here in one fused pass).  q/out: [B, Hq, Lq, D] contiguous.
 * Same workspace rules as qsdpa_decode, and the first
 * qsdpa_workspace_zero_bytes(...) bytes must be zero before the first call
 * (the kernels leave them zero).  With at least 64 (head, query) rows
 * per kv head and f16/bf16 output the call runs on the tcgen05 tensor-core
 * kernel (K and V tiles dequantized to fp16, fp32 accumulation in TMEM);
 * otherwise, and always for f32 output, on the split-K kernel.  The tcgen05
 * kernel bounds its waits on the tensor core (200 ms each; the environment
 * variable QKV_PREFILL_WAIT_NS sets another limit in ns, and
 * QKV_PREFILL_STALL_HALF=i, a test hook, withholds the copy of the i-th
 * 32-key block so that a wait runs out): if one ever times out it sets
 * the first 32-bit word of the workspace nonzero (the output is then invalid)
 * and the kernel still returns; that word must be zeroed again before the
 * workspace is reused.  Its fp16
 * tiles hold scale * code + bias: a small kernel first checks every scale and
 * bias of rows [0, L), and when some value can reach 2^15 the call runs a
 * second instance of the tcgen05 kernel that scales each tile by a power of
 * two and undoes it exactly (values up to the largest the fp16 scales and
 * biases can express are computed correctly); words 1 and 2 of the workspace
 * carry that decision and are zero again after the call. */
qkv_status qsdpa_prefill(const void* q, int q_dtype, int B, int Hq, int Hkv, int Lq,
                         int D, const qkv_cache* k, const qkv_cache* v, int64_t L,
                         float scale, const qkv_mask* mask, void* out, int out_dtype,
                         void* workspace, size_t workspace_bytes, void* stream);

/* qsdpa_decode / qsdpa_prefill with the attention extensions above (ext may
 * be NULL, which is the plain call).  Same arguments, rules and accuracy
 * otherwise. */
qkv_status qsdpa_decode_ext(const void* q, int q_dtype, int B, int Hq, int Hkv, int D,
                            const qkv_cache* k, const qkv_cache* v, int64_t L,
                            float scale, const qkv_mask* mask, const qkv_attn_ext* ext,
                            void* out, int out_dtype, void* workspace,
                            size_t workspace_bytes, void* stream);
qkv_status qsdpa_prefill_ext(const void* q, int q_dtype, int B, int Hq, int Hkv, int Lq,
                             int D, const qkv_cache* k, const qkv_cache* v, int64_t L,
                             float scale, const qkv_mask* mask, const qkv_attn_ext* ext,
                             void* out, int out_dtype, void* workspace,
                             size_t workspace_bytes, void* stream);

/* Rows [0, L) of one quantized cache materialized as fp16:
 * out[b, h, j, e] = fp16(scale * code + bias) (Q8_0: scale * code), the
 * correctly rounded value of the exact dequantization.  The prompt path of
 * llama.cpp #25556 converts a Q8_0 cache to fp16 and runs dense attention on
 * it; this is that conversion, for comparisons of "materialize, then dense
 * attention" with the fused kernels.  out: [B, Hkv, L, D] contiguous fp16,
 * 16-byte aligned, caller-owned.  One launch. */
qkv_status qkv_dequantize(const qkv_cache* c, int B, int Hkv, int D, int64_t L, void* out,
                          void* stream);

/* Conversion between llama.cpp-style interleaved Q8_0 blocks and this
 * library's Q8_0 planes, bit for bit (llama.cpp #25556 keeps its KV cache in
 * Q8_0 blocks; their byte layout, not shown on the pages, is the GGUF Q8_0
 * block: 34 bytes, the fp16 scale first (little-endian), then the 32 int8
 * codes in element order).  A row of D elements (b, kv head, token l) is D/32
 * consecutive blocks starting at byte b*stride_b + h*stride_h + l*stride_l of
 * `blocks` (llama.cpp's token-major K cache: stride_l = Hkv*D/32*34,
 * stride_h = D/32*34).  blocks and the strides must be 2-byte aligned.
 *  qkv_q8_0_from_blocks: writes tokens [0, L) of the blocks into cache rows
 *    [offset, offset + L) of dst (a Q8_0 qkv_cache); 0 <= offset, offset + L <= Lcap.
 *  qkv_q8_0_to_blocks: writes cache rows [offset, offset + L) of src into
 *    tokens [0, L) of the blocks; destination rows must not overlap.
 * One launch each; L == 0 does nothing. */
qkv_status qkv_q8_0_from_blocks(const void* blocks, int B, int Hkv, int D, int64_t L,
                                int64_t stride_b, int64_t stride_h, int64_t stride_l,
                                const qkv_cache* dst, int64_t offset, void* stream);
qkv_status qkv_q8_0_to_blocks(const qkv_cache* src, int B, int Hkv, int D, int64_t offset,
                              int64_t L, void* blocks, int64_t stride_b, int64_t stride_h,
                              int64_t stride_l, void* stream);

/* llama.cpp's other KV block formats into an affine cache with groups of 32
 * that holds exactly the same values (the PR's follow-up extends its KV
 * conversion to these types; their bytes, not on the pages, are the GGUF
 * blocks of 32 elements, little-endian fp16 fields first):
 *   QKV_BLOCKS_Q4_0  18 bytes: d, qs[16]            x = d (q - 8)   -> 4-bit cache, bias -8d
 *   QKV_BLOCKS_Q4_1  20 bytes: d, m, qs[16]         x = d q + m     -> 4-bit cache, bias m
 *   QKV_BLOCKS_Q5_0  22 bytes: d, qh[4], qs[16]     x = d (q - 16)  -> 8-bit cache, bias -16d
 *   QKV_BLOCKS_Q5_1  24 bytes: d, m, qh[4], qs[16]  x = d q + m     -> 8-bit cache, bias m
 * (element j < 16 in the low nibble of qs[j], element j + 16 in its high
 * nibble; the fifth bit of element e is bit e of qh).  dst: affine, group_size
 * 32, bits 4 for Q4 and 8 for Q5.  Rows, strides, offset and alignment as for
 * qkv_q8_0_from_blocks (with the block sizes above).  The decode and prefill
 * calls then read the cache like any affine cache.  One launch.
 * Range: the bias -8d (Q4_0) or -16d (Q5_0) is exact in fp16 for |d| <= 8188
 * (Q4_0) or |d| <= 4094 (Q5_0); a block with a larger d holds values outside
 * the fp16 range, its bias is stored as +-inf and attention over it returns
 * non-finite values (the conversion itself reports no error). */
typedef enum { QKV_BLOCKS_Q4_0 = 0, QKV_BLOCKS_Q4_1 = 1, QKV_BLOCKS_Q5_0 = 2,
               QKV_BLOCKS_Q5_1 = 3 } qkv_block_kind;
qkv_status qkv_llama_blocks_to_cache(int kind, const void* blocks, int B, int Hkv, int D,
                                     int64_t L, int64_t stride_b, int64_t stride_h,
                                     int64_t stride_l, const qkv_cache* dst, int64_t offset,
                                     void* stream);

/* The same block formats written on the GPU (the PR's follow-up keeps the KV
 * cache in these types, so a cache imported from llama.cpp is extended in its
 * own format).  The quantizer is llama.cpp's published reference one (not on
 * the pages), per block of 32 elements in fp32 IEEE operations in this order:
 *   Q4_0 / Q5_0: m = the element of largest magnitude (the first such),
 *                d = m / -8 (Q5_0: m / -16), id = d == 0 ? 0 : 1/d,
 *                q = min(15 (31), trunc(x*id + 8.5 (16.5)))
 *   Q4_1 / Q5_1: lo, hi = min, max, d = (hi - lo) / 15 (31),
 *                id = d == 0 ? 0 : 1/d, q = min(15 (31), trunc((x - lo)*id + 0.5)),
 *                m = lo
 * with d and m stored as fp16 (round to nearest even) and the codes computed
 * from the fp32 d; bit-identical to the CPU oracle.
 *  qkv_llama_quantize_blocks: x [B, Hkv, L, D] contiguous, f16 or bf16,
 *    16-byte aligned -> the blocks of tokens [0, L), placed by the byte
 *    strides as for qkv_q8_0_from_blocks (blocks and strides 2-byte aligned;
 *    offset the blocks pointer to append).  D in {64, 128, 256}.
 *  qkv_llama_quantize_update: new_k / new_v [B, Hkv, Lnew, D] (f16 or bf16,
 *    16-byte aligned) quantized the same way and written into rows
 *    [offset, offset + Lnew) of affine caches with group_size 32 (4-bit codes
 *    for Q4, 8-bit for Q5) exactly as qkv_llama_blocks_to_cache would import
 *    the resulting blocks (scale d, bias m, or -8d / -16d rounded to fp16 from
 *    the fp16 d).  Two launches (K, then V).
 *  qkv_llama_cache_to_blocks: rows [offset, offset + L) of such an affine
 *    cache -> blocks (d = scale, m = bias, the codes' low bits).  The blocks
 *    hold the rows' values exactly for groups that blocks of that kind can
 *    hold -- codes below 16 (Q4) or 32 (Q5), and for Q4_0 / Q5_0 a bias of
 *    -8 (-16) times the scale: the groups written by the import and the
 *    quantizers above.  One launch.
 * L == 0 / Lnew == 0 do nothing. */
qkv_status qkv_llama_quantize_blocks(int kind, const void* x, int in_dtype, int B, int Hkv, int D,
                                     int64_t L, void* blocks, int64_t stride_b, int64_t stride_h,
                                     int64_t stride_l, void* stream);
qkv_status qkv_llama_quantize_update(int kind, const void* new_k, const void* new_v, int in_dtype,
                                     int B, int Hkv, int Lnew, int D, const qkv_cache* k,
                                     const qkv_cache* v, int64_t offset, void* stream);
qkv_status qkv_llama_cache_to_blocks(int kind, const qkv_cache* src, int B, int Hkv, int D,
                                     int64_t offset, int64_t L, void* blocks, int64_t stride_b,
                                     int64_t stride_h, int64_t stride_l, void* stream);

/* Attention whose values are a view of the keys (the "576/512 MLA" shape of
 * the llama.cpp PR's follow-up tests: K rows of Dk = 576 elements, V = the
 * first Dv = 512 elements of every K row, so the cache holds K only and one
 * stream serves both):
 *   out[b,h,i,:] = softmax_j(q[b,h,i]*scale . Khat[b,h/G,j] (+ causal)) . Khat[b,h/G,j,:512]
 *  q:   [B, Hq, Lq, 576] contiguous, f16 or bf16.
 *  out: [B, Hq, Lq, 512] contiguous, f16 or bf16 (fp32 output is refused:
 *       the kernel dequantizes to fp16 tiles, max-abs error <= 2e-3 for
 *       values of order one).
 *  k:   Q8_0, or affine 4- or 8-bit codes in groups of 32 or 64; rows of 576.
 *  mask: NULL, none or causal (bottom-right); no additive mask.
 *  workspace: at least qsdpa_kview_workspace_size(...) bytes, 16-byte aligned
 *  (partial results of the split over L; no state between calls).  One
 *  launch, or two when the keys of a (batch, kv head, 64-row tile) are split
 *  over several CTAs (the second is the decode's merge kernel).  Any Lq >= 1
 *  (decode and prefill).  L == 0 writes zeros. */
qkv_status qsdpa_attention_kview(const void* q, int q_dtype, int B, int Hq, int Hkv, int Lq, int Dk,
                                 int Dv, const qkv_cache* k, int64_t L, float scale,
                                 const qkv_mask* mask, void* out, int out_dtype, void* workspace,
                                 size_t workspace_bytes, void* stream);
size_t qsdpa_kview_workspace_size(int B, int Hq, int Hkv, int Lq, int Dk, int Dv, int64_t L);

/* Allocation-free variant of qsdpa_decode (the pages have no counterpart:
 * MLX and llama.cpp allocate their temporaries through their own allocators).
 * For callers that cannot allocate device memory when they decode -- code
 * that runs under an allocator which forbids cudaMalloc/cudaFree, services
 * that fix every buffer before they start, or plug-in interfaces that hand
 * over only inputs and outputs.  Same arguments and results as qsdpa_decode,
 * without the workspace: its scratch (partial results) lives in a
 * 8 MiB array built into this library, which every GPU that loads the
 * library keeps until the process exits.  Shapes whose workspace
 * (qsdpa_workspace_size) exceeds 8 MiB are rejected with QKV_ERR_WORKSPACE.
 * The first call on a device looks up that device's address of the array;
 * make that first call before any stream capture.  Every call reuses the same
 * array, so calls that may overlap on the GPU (other streams, other host
 * threads on the same device) race: order them on one stream. */
qkv_status qsdpa_decode_noalloc(const void* q, int q_dtype, int B, int Hq, int Hkv, int D,
                                const qkv_cache* k, const qkv_cache* v, int64_t L,
                                float scale, const qkv_mask* mask, void* out, int out_dtype,
                                void* stream);

/* Workspace bytes needed by qsdpa_decode (Lq = 1) or qsdpa_prefill for this
 * problem on the CURRENT device, and how many leading bytes must be zero
 * before the first qsdpa_prefill call.  0 on invalid arguments. */
size_t qsdpa_workspace_size(int B, int Hq, int Hkv, int Lq, int D, int64_t L);
size_t qsdpa_workspace_zero_bytes(int B, int Hq, int Hkv, int Lq, int D, int64_t L);

/* Human-readable text of a status code, and the detail of this host thread's
 * most recent error (empty string if none). */
const char* qkv_status_string(int status);
const char* qkv_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* QKV_H_ */
