// qkv_oracle.cpp -- plain, slow, CPU-only statement of what the quantized-KV
// attention path computes.  TEST INFRASTRUCTURE ONLY: the CUDA library never
// links, includes or calls this file; only the test-suite, the smoke check and
// the CPU-baseline leg of the benchmark load it.  It shares no source with the
// GPU path (its own half-precision conversions, its own packing, its own
// attention).
//
// Sources (web pages; cited by page title and the file/section shown on it):
//  [MLX-KV]  MLX compare "v0.19.3...quantized-kv-update" (commit "add
//            fast::quantized_kv_update"):
//              - mlx/fast.cpp, quantized_scaled_dot_product_attention: the
//                fallback that defines the math (q*scale, GQA reshape,
//                quantized_matmul(q, K^T), + additive mask, precise softmax,
//                quantized_matmul(P, V)).
//              - mlx/backend/metal/kernels/sdpa_vector.h, quant_sdpa_vector /
//                load_keys / load_values: packing order (element j of a
//                32-bit word sits at bits [j*bits, (j+1)*bits)), dequant
//                w = scale*code + bias, kv_head = q_head / gqa_factor.
//              - mlx/backend/metal/kernels/quantized.h, affine_quantize_impl:
//                eps = 1e-7 for the scale; affine dequantize "scale*d + bias".
//              - mlx/fast.cpp, kv_update and KVUpdate::eval_gpu: new rows are
//                quantized and written at token `offset` of the cache.
//  [MLX-WIP] MLX compare "v0.30.0...6c60bd1" ("Fixed mma and working
//            dequant"), SharedTile::load_quantized: ((w >> (j*bits)) & MASK)
//            * s + b, the same packing and dequant.
//  [LCPP]    llama.cpp PR #25556 "Metal: Optimize q8_0 KV" and its merged
//            follow-up: the Q8_0 KV cache format (blocks of 32 int8 codes
//            with one fp16 scale).
//
// Readings where the pages are silent (each also listed in the design notes):
//  * affine quantizer body is not printed: min-max asymmetric quantization,
//    scale = (max-min)/(2^bits-1) clamped below by eps, bias = group minimum,
//    both stored as fp16 (RNE), codes = round-half-even((x-bias)/scale) with
//    the STORED fp16 scale and bias, clamped to [0, 2^bits-1].  All fp32 IEEE
//    operations in this fixed order so that a GPU quantizer can match bit for
//    bit.
//  * Q8_0 quantizer formula is not printed: d = absmax/127 (fp32), stored as
//    fp16 (RNE); codes = round-half-even(x / stored d) clamped to [-127, 127];
//    d == 0 gives all-zero codes.  Layout is struct-of-arrays: codes as int8
//    (element e in byte e%4 of 32-bit word e/4), scales in a separate plane.
//  * mask: additive (fp16/bf16/fp32) or causal aligned to the bottom-right
//    (query i of Lq sees key j iff j <= L - Lq + i); a row with no visible key
//    returns zeros.
//  * attention math in fp64 after exact dequantization.
//  * parity unpinned: agreement with MLX's or llama.cpp's OWN quantizer
//    outputs (their rounding choices) -- the pages print neither the
//    quantizer bodies nor a worked example; the quantizers here are pinned
//    only by what their definitions fix (error bound, per-element optimality,
//    min-max structure, hand-derived fixtures).
//  * extensions that the llama.cpp PR's test coverage lists (sinks, ALiBi,
//    logit softcap; the pages give no formula for them), in their usual
//    definitions:
//      - logit softcap c > 0: the scaled logit x = scale*q.k becomes
//        c*tanh(x/c), before the mask is added;
//      - ALiBi as a per-head slope on the additive mask: head h adds
//        slope[h]*mask (a -inf entry hides the key whatever the slope);
//      - attention sink: a per-head logit sink[h] that joins the softmax
//        denominator (exp(sink - M)) with no value row, so the weights of
//        the keys sum to less than 1; a row with no visible key still
//        returns zeros.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <thread>
#include <vector>
#include <limits>

namespace {

// ---------------------------------------------------------------------------
// IEEE-754 half (binary16) and bfloat16 conversions, written from the format
// definitions.  Round-to-nearest-even on narrowing.
// ---------------------------------------------------------------------------
float bits_to_f32(uint32_t u) { float f; std::memcpy(&f, &u, 4); return f; }
uint32_t f32_to_bits(float f) { uint32_t u; std::memcpy(&u, &f, 4); return u; }

float half_to_float(uint16_t h) {
  const uint32_t sign = (uint32_t)(h >> 15) & 1u;
  const int exp = (h >> 10) & 0x1f;
  const uint32_t man = h & 0x3ffu;
  double mag;
  if (exp == 0) {
    mag = std::ldexp((double)man, -24);             // subnormal: man * 2^-24
  } else if (exp == 31) {
    if (man) return std::numeric_limits<float>::quiet_NaN();
    mag = std::numeric_limits<double>::infinity();
  } else {
    mag = std::ldexp((double)(1024 + man), exp - 25);  // (1.man) * 2^(exp-15)
  }
  return (float)(sign ? -mag : mag);  // exact: every half is a float
}

// Round a finite, non-negative double `a` (exactly representable as float) to
// binary16 magnitude bits with round-half-even; overflow -> infinity.
uint16_t half_mag_from_double(double a) {
  if (a == 0.0) return 0;
  // smallest normal half = 2^-14; subnormal quantum = 2^-24
  int e;
  std::frexp(a, &e);             // a = f * 2^e, f in [0.5, 1)
  int exp_unbiased = e - 1;      // a = 1.xxx * 2^(e-1)
  if (exp_unbiased < -14) {
    // subnormal range: quantum 2^-24
    double q = a * 16777216.0;   // a / 2^-24 (exact scaling by power of two)
    double r = std::nearbyint(q);  // round-half-even (default rounding mode)
    // r may reach 1024 -> becomes smallest normal; bit pattern still works
    return (uint16_t)r;
  }
  // normal: quantum 2^(exp_unbiased-10)
  double scale = std::ldexp(1.0, 10 - exp_unbiased);
  double m = std::nearbyint(a * scale);          // in [1024, 2048]
  int ex = exp_unbiased;
  if (m >= 2048.0) { m /= 2.0; ex += 1; }        // carried into next binade
  if (ex > 15) return 0x7c00;                    // overflow -> inf
  return (uint16_t)(((ex + 15) << 10) | ((int)m - 1024));
}

uint16_t float_to_half_rne(float f) {
  const uint32_t u = f32_to_bits(f);
  const uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  if (std::isnan(f)) return (uint16_t)(sign | 0x7e00);
  if (std::isinf(f)) return (uint16_t)(sign | 0x7c00);
  return (uint16_t)(sign | half_mag_from_double(std::fabs((double)f)));
}

float bf16_to_float(uint16_t b) { return bits_to_f32((uint32_t)b << 16); }

uint16_t float_to_bf16_rne(float f) {
  uint32_t u = f32_to_bits(f);
  if (std::isnan(f)) return (uint16_t)((u >> 16) | 0x40);
  // keep the upper 16 bits, rounding the dropped 16 to nearest, ties to even
  uint32_t lower = u & 0xffffu;
  uint32_t upper = u >> 16;
  if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1;
  return (uint16_t)upper;
}

enum Dtype { DT_F16 = 0, DT_BF16 = 1, DT_F32 = 2 };

float load_elem(const void* p, int dtype, int64_t i) {
  switch (dtype) {
    case DT_F16: return half_to_float(((const uint16_t*)p)[i]);
    case DT_BF16: return bf16_to_float(((const uint16_t*)p)[i]);
    default: return ((const float*)p)[i];
  }
}

// ---------------------------------------------------------------------------
// Code packing.  A row's codes form one little-endian bit stream: element e
// occupies bits [e*bits, (e+1)*bits), bit i of the stream being bit i%32 of
// 32-bit word i/32.  For 2, 4 and 8 bits this is "element j of a word at bits
// [j*bits, (j+1)*bits)" ([MLX-KV] sdpa_vector.h); for 3 and 5 bits it packs 8
// codes in 3 or 5 bytes and for 6 bits 4 codes in 3 bytes, the pack sizes
// that [MLX-WIP] mlx/backend/cuda/quantized/quantized_utils.cuh
// (get_pack_factor, get_bytes_per_pack) states -- reading: within a pack, the
// same little-endian order (the pages print no 3/5/6-bit pack layout).
// ---------------------------------------------------------------------------
void put_code(uint32_t* row, int e, int bits, uint32_t q) {
  const int64_t pos = (int64_t)e * bits;
  const int w = (int)(pos / 32), sh = (int)(pos % 32);
  row[w] |= q << sh;
  if (sh + bits > 32) row[w + 1] |= q >> (32 - sh);     // the code straddles two words
}

uint32_t get_code(const uint32_t* row, int e, int bits) {
  const int64_t pos = (int64_t)e * bits;
  const int w = (int)(pos / 32), sh = (int)(pos % 32);
  uint64_t v = row[w] >> sh;
  if (sh + bits > 32) v |= (uint64_t)row[w + 1] << (32 - sh);
  return (uint32_t)(v & ((1u << bits) - 1u));
}

// ---------------------------------------------------------------------------
// Quantizers ([MLX-KV] quantized.h affine_quantize_impl / kv_update; [LCPP]).
// ---------------------------------------------------------------------------
void quantize_affine_group(const float* x, int gs, int bits,
                           uint32_t* codes_row, int first_elem,
                           uint16_t* scale_out, uint16_t* bias_out) {
  float mn = x[0], mx = x[0];
  for (int i = 1; i < gs; ++i) { mn = std::min(mn, x[i]); mx = std::max(mx, x[i]); }
  const float levels = (float)((1 << bits) - 1);
  float s = (mx - mn) / levels;
  if (!(s >= 1e-7f)) s = 1e-7f;                 // eps from affine_quantize_impl
  const uint16_t s16 = float_to_half_rne(s);
  const uint16_t b16 = float_to_half_rne(mn);
  const float sf = half_to_float(s16);
  const float bf = half_to_float(b16);
  const int qmax = (1 << bits) - 1;
  for (int i = 0; i < gs; ++i) {
    float t = (x[i] - bf) / sf;
    float r = std::nearbyint(t);
    int q = (int)r;
    if (q < 0) q = 0;
    if (q > qmax) q = qmax;
    put_code(codes_row, first_elem + i, bits, (uint32_t)q);   // element index within the row
  }
  *scale_out = s16;
  *bias_out = b16;
}

void quantize_q8_0_group(const float* x, uint32_t* codes_row, int first_elem,
                         uint16_t* scale_out) {
  float a = 0.0f;
  for (int i = 0; i < 32; ++i) a = std::max(a, std::fabs(x[i]));
  const float d = a / 127.0f;
  const uint16_t d16 = float_to_half_rne(d);
  const float df = half_to_float(d16);
  for (int i = 0; i < 32; ++i) {
    int q = 0;
    if (df != 0.0f) {
      float r = std::nearbyint(x[i] / df);
      q = (int)r;
      if (q < -127) q = -127;
      if (q > 127) q = 127;
    }
    const int e = first_elem + i;
    codes_row[e / 4] |= (uint32_t)(uint8_t)(int8_t)q << ((e % 4) * 8);
  }
  *scale_out = d16;
}

// ---------------------------------------------------------------------------
// Dequantization of one cache row into fp64 ([MLX-KV] load_keys/load_values,
// affine dequantize; [MLX-WIP] load_quantized).
// ---------------------------------------------------------------------------
struct Cache {
  int fmt;              // 0 affine, 1 Q8_0
  int bits;
  int gs;
  const uint32_t* codes;
  const uint16_t* scales;
  const uint16_t* biases;
  int64_t Lcap;
};

void dequant_row(const Cache& c, int D, int64_t row, double* out) {
  const int words = D * c.bits / 32;
  const int ng = D / c.gs;
  const uint32_t* w = c.codes + row * words;
  const uint16_t* sc = c.scales + row * ng;
  const uint16_t* bi = c.fmt == 0 ? c.biases + row * ng : nullptr;
  for (int e = 0; e < D; ++e) {
    const uint32_t field = get_code(w, e, c.bits);
    const int g = e / c.gs;
    const double s = (double)half_to_float(sc[g]);
    if (c.fmt == 0) {
      out[e] = s * (double)field + (double)half_to_float(bi[g]);
    } else {
      out[e] = s * (double)(int8_t)(uint8_t)field;   // Q8_0: signed code
    }
  }
}

// ---------------------------------------------------------------------------
// Attention ([MLX-KV] fast.cpp fallback): O = softmax(q*scale . K^T + mask) V
// with K, V dequantized, computed in fp64.
// ---------------------------------------------------------------------------
struct Mask {
  int kind;             // 0 none, 1 causal (bottom-right), 2 additive
  const void* add;
  int add_dtype;
  int64_t sb, sh, sq;   // element strides of the additive mask (row = keys)
};

struct Problem {
  const double* q;      // [B,Hq,Lq,D] already converted to fp64
  int B, Hq, Hkv, Lq, D;
  int Dv;               // output / value width: D, or fewer when V is a view of K's first Dv
  Cache k, v;
  int64_t L;
  double scale;
  Mask mask;
  double softcap;       // 0: off
  const double* sinks;  // [Hq] or null
  const double* slopes; // [Hq] or null (additive mask multiplier)
};

// Logit of key j for query row (b,h,i); returns false if the key is invisible.
bool logit(const Problem& p, int b, int h, int i, int64_t j,
           const std::vector<double>& kh, double* out) {
  const double* qr = p.q + (((int64_t)b * p.Hq + h) * p.Lq + i) * p.D;
  double s = 0.0;
  for (int e = 0; e < p.D; ++e) s += (qr[e] * p.scale) * kh[e];
  if (p.softcap > 0.0) s = p.softcap * std::tanh(s / p.softcap);
  if (p.mask.kind == 1) {
    if (j > p.L - p.Lq + i) return false;
  } else if (p.mask.kind == 2) {
    const int64_t idx = b * p.mask.sb + h * p.mask.sh + i * p.mask.sq + j;
    const double m = (double)load_elem(p.mask.add, p.mask.add_dtype, idx);
    if (std::isinf(m) && m < 0) return false;
    s += (p.slopes ? p.slopes[h] : 1.0) * m;
  }
  *out = s;
  return true;
}

// Two-pass form: all logits, max, exp, normalize, weighted sum of V.
void attend_two_pass(const Problem& p, int b, int h, int i, double* o,
                     double* probs /* nullable, [L] */) {
  const int G = p.Hq / p.Hkv;
  const int kvh = h / G;                                     // GQA mapping
  const int64_t base = ((int64_t)b * p.Hkv + kvh) * p.k.Lcap;
  std::vector<double> kh(p.D), vh(p.D);
  std::vector<double> s(p.L);
  std::vector<char> vis(p.L, 0);
  double mx = -std::numeric_limits<double>::infinity();
  for (int64_t j = 0; j < p.L; ++j) {
    dequant_row(p.k, p.D, base + j, kh.data());
    if (logit(p, b, h, i, j, kh, &s[j])) { vis[j] = 1; mx = std::max(mx, s[j]); }
  }
  for (int e = 0; e < p.Dv; ++e) o[e] = 0.0;
  if (probs) for (int64_t j = 0; j < p.L; ++j) probs[j] = 0.0;
  if (!(mx > -std::numeric_limits<double>::infinity())) return;  // none visible
  double l = 0.0;
  if (p.sinks) {                                             // the sink joins the max and the sum
    mx = std::max(mx, p.sinks[h]);
    l += std::exp(p.sinks[h] - mx);
  }
  for (int64_t j = 0; j < p.L; ++j) if (vis[j]) { s[j] = std::exp(s[j] - mx); l += s[j]; }
  const int64_t vbase = ((int64_t)b * p.Hkv + kvh) * p.v.Lcap;
  for (int64_t j = 0; j < p.L; ++j) {
    if (!vis[j]) continue;
    const double pj = s[j] / l;
    if (probs) probs[j] = pj;
    dequant_row(p.v, p.D, vbase + j, vh.data());
    for (int e = 0; e < p.Dv; ++e) o[e] += pj * vh[e];
  }
}

// Online form over [j0, j1): running max m, running sum l, unnormalized o.
void attend_online_range(const Problem& p, int b, int h, int i, int64_t j0,
                         int64_t j1, double* m_out, double* l_out, double* o) {
  const int G = p.Hq / p.Hkv;
  const int kvh = h / G;
  const int64_t kb = ((int64_t)b * p.Hkv + kvh) * p.k.Lcap;
  const int64_t vb = ((int64_t)b * p.Hkv + kvh) * p.v.Lcap;
  std::vector<double> kh(p.D), vh(p.D);
  double m = -std::numeric_limits<double>::infinity(), l = 0.0;
  for (int e = 0; e < p.Dv; ++e) o[e] = 0.0;
  for (int64_t j = j0; j < j1; ++j) {
    dequant_row(p.k, p.D, kb + j, kh.data());
    double sj;
    if (!logit(p, b, h, i, j, kh, &sj)) continue;
    const double mn = std::max(m, sj);
    const double alpha = (m == -std::numeric_limits<double>::infinity()) ? 0.0 : std::exp(m - mn);
    const double pj = std::exp(sj - mn);
    dequant_row(p.v, p.D, vb + j, vh.data());
    l = l * alpha + pj;
    for (int e = 0; e < p.Dv; ++e) o[e] = o[e] * alpha + pj * vh[e];
    m = mn;
  }
  *m_out = m;
  *l_out = l;
}

// Final normalization of an online/merged (m, l, o): o / l, with the head's
// sink (if any) folded into the denominator; no visible key gives zeros.
void finish_row(const Problem& p, int h, double m, double l, double* o) {
  if (!(l > 0.0)) { for (int e = 0; e < p.Dv; ++e) o[e] = 0.0; return; }
  double w = 1.0;
  if (p.sinks) {
    const double M = std::max(m, p.sinks[h]);
    w = std::exp(m - M);
    l = l * w + std::exp(p.sinks[h] - M);
  }
  for (int e = 0; e < p.Dv; ++e) o[e] = o[e] * w / l;
}

// Split form: partition keys into `nsplit` contiguous chunks, run the online
// form on each, then merge the partial (m, l, o) by log-sum-exp rescaling.
void attend_split(const Problem& p, int b, int h, int i, int nsplit, double* o) {
  const double ninf = -std::numeric_limits<double>::infinity();
  std::vector<double> ms(nsplit), ls(nsplit), os((size_t)nsplit * p.Dv);
  for (int sidx = 0; sidx < nsplit; ++sidx) {
    const int64_t j0 = p.L * sidx / nsplit, j1 = p.L * (sidx + 1) / nsplit;
    attend_online_range(p, b, h, i, j0, j1, &ms[sidx], &ls[sidx], &os[(size_t)sidx * p.Dv]);
  }
  double M = ninf;
  for (double m : ms) M = std::max(M, m);
  for (int e = 0; e < p.Dv; ++e) o[e] = 0.0;
  if (M == ninf) return;
  double l = 0.0;
  for (int sidx = 0; sidx < nsplit; ++sidx) {
    if (ms[sidx] == ninf) continue;
    const double w = std::exp(ms[sidx] - M);
    l += w * ls[sidx];
    for (int e = 0; e < p.Dv; ++e) o[e] += w * os[(size_t)sidx * p.Dv + e];
  }
  finish_row(p, h, M, l, o);
}

template <class F>
void parallel_rows(int64_t n, int nthreads, F f) {
  if (nthreads <= 1 || n <= 1) { for (int64_t r = 0; r < n; ++r) f(r); return; }
  nthreads = (int)std::min<int64_t>(nthreads, n);
  std::vector<std::thread> ts;
  for (int t = 0; t < nthreads; ++t) {
    ts.emplace_back([&, t]() { for (int64_t r = t; r < n; r += nthreads) f(r); });
  }
  for (auto& th : ts) th.join();
}

// Every requested row (b, h, i) of the output, in one of the three evaluation
// orders; row id ((b*Hq)+h)*Lq+i, output rows of p.Dv values.
void run_rows(const Problem& p, int mode, int nsplit, const int64_t* rows, int64_t total,
              double* out, int nthreads) {
  parallel_rows(total, nthreads, [&](int64_t r) {
    const int64_t id = rows ? rows[r] : r;
    const int i = (int)(id % p.Lq);
    const int h = (int)((id / p.Lq) % p.Hq);
    const int b = (int)(id / ((int64_t)p.Lq * p.Hq));
    double* o = out + id * p.Dv;
    if (mode == 0) {
      attend_two_pass(p, b, h, i, o, nullptr);
    } else if (mode == 1) {
      double m, l;
      attend_online_range(p, b, h, i, 0, p.L, &m, &l, o);
      finish_row(p, h, m, l, o);
    } else {
      attend_split(p, b, h, i, nsplit < 1 ? 1 : nsplit, o);
    }
  });
}

Cache make_cache(int fmt, int bits, int gs, const uint32_t* codes,
                 const uint16_t* scales, const uint16_t* biases, int64_t Lcap) {
  Cache c;
  c.fmt = fmt; c.bits = bits; c.gs = gs; c.codes = codes; c.scales = scales;
  c.biases = biases; c.Lcap = Lcap;
  return c;
}

}  // namespace

extern "C" {

// --- conversions (exposed so tests can pin them against a library routine) --
void orc_f32_to_f16(const float* x, uint16_t* y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = float_to_half_rne(x[i]);
}
void orc_f16_to_f32(const uint16_t* x, float* y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = half_to_float(x[i]);
}
void orc_f32_to_bf16(const float* x, uint16_t* y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = float_to_bf16_rne(x[i]);
}
void orc_bf16_to_f32(const uint16_t* x, float* y, int64_t n) {
  for (int64_t i = 0; i < n; ++i) y[i] = bf16_to_float(x[i]);
}

// --- quantize `rows` rows of D elements (fp16 / bf16 / fp32 input) ----------
// codes: [rows, D*bits/32] uint32 (zeroed here), scales/biases: [rows, D/gs].
// fmt 0 = affine (bits 2, 3, 4, 5, 6 or 8; gs | D; D*bits a multiple of 32),
// fmt 1 = Q8_0 (gs 32).
int orc_quantize(int fmt, const void* x, int in_dtype, int64_t rows, int D,
                 int gs, int bits, uint32_t* codes, uint16_t* scales,
                 uint16_t* biases, int nthreads) {
  if (fmt == 1) { bits = 8; gs = 32; }
  if (D % gs != 0 || bits < 2 || bits > 8 || bits == 7 || (D * bits) % 32 != 0) return 1;
  const int words = D * bits / 32, ng = D / gs;
  parallel_rows(rows, nthreads, [&](int64_t r) {
    std::vector<float> xr(D);
    for (int e = 0; e < D; ++e) xr[e] = load_elem(x, in_dtype, r * D + e);
    uint32_t* cr = codes + r * words;
    for (int w = 0; w < words; ++w) cr[w] = 0u;
    for (int g = 0; g < ng; ++g) {
      if (fmt == 0)
        quantize_affine_group(&xr[g * gs], gs, bits, cr, g * gs, &scales[r * ng + g],
                              &biases[r * ng + g]);
      else
        quantize_q8_0_group(&xr[g * gs], cr, g * gs, &scales[r * ng + g]);
    }
  });
  return 0;
}

// --- dequantize `rows` rows into fp64 ---------------------------------------
int orc_dequantize(int fmt, int bits, int gs, const uint32_t* codes,
                   const uint16_t* scales, const uint16_t* biases, int64_t rows,
                   int D, double* out) {
  if (fmt == 1) { bits = 8; gs = 32; }
  Cache c = make_cache(fmt, bits, gs, codes, scales, biases, rows);
  for (int64_t r = 0; r < rows; ++r) dequant_row(c, D, r, out + r * D);
  return 0;
}

// --- attention ---------------------------------------------------------------
// q: fp64 [B,Hq,Lq,D].  K/V caches: codes [B,Hkv,Lcap,D*bits/32], scales and
// biases [B,Hkv,Lcap,D/gs] (biases ignored for Q8_0).  L valid keys.
// mode: 0 two-pass, 1 online, 2 split into `nsplit` chunks then merged.
// rows: optional list of nrows (b,h,i) triples (flattened row ids
// ((b*Hq)+h)*Lq+i); when null every row is computed.  out: fp64 [B,Hq,Lq,D]
// (only the requested rows are written).
int orc_attention(const double* q, int B, int Hq, int Hkv, int Lq, int D,
                  int kfmt, int kbits, int kgs, const uint32_t* kcodes,
                  const uint16_t* kscales, const uint16_t* kbiases,
                  int vfmt, int vbits, int vgs, const uint32_t* vcodes,
                  const uint16_t* vscales, const uint16_t* vbiases,
                  int64_t Lcap, int64_t L, double scale, int mask_kind,
                  const void* mask_add, int mask_dtype, int64_t msb,
                  int64_t msh, int64_t msq, double softcap,
                  const double* sinks, const double* slopes, int mode, int nsplit,
                  const int64_t* rows, int64_t nrows, double* out,
                  int nthreads) {
  if (Hkv <= 0 || Hq % Hkv != 0 || L < 0 || L > Lcap) return 1;
  if (kfmt == 1) { kbits = 8; kgs = 32; }
  if (vfmt == 1) { vbits = 8; vgs = 32; }
  Problem p;
  p.q = q; p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lq = Lq; p.D = D; p.Dv = D;
  p.k = make_cache(kfmt, kbits, kgs, kcodes, kscales, kbiases, Lcap);
  p.v = make_cache(vfmt, vbits, vgs, vcodes, vscales, vbiases, Lcap);
  p.L = L; p.scale = scale;
  p.mask.kind = mask_kind; p.mask.add = mask_add; p.mask.add_dtype = mask_dtype;
  p.mask.sb = msb; p.mask.sh = msh; p.mask.sq = msq;
  p.softcap = softcap; p.sinks = sinks; p.slopes = slopes;
  const int64_t total = rows ? nrows : (int64_t)B * Hq * Lq;
  run_rows(p, mode, nsplit, rows, total, out, nthreads);
  return 0;
}

// --- attention whose values are a view of the keys ---------------------------
// (the MLA shape of the llama.cpp PR's follow-up: K rows of Dk elements, V the
// first Dv of each K row).  One cache; out: fp64 [B,Hq,Lq,Dv].
int orc_attention_kview(const double* q, int B, int Hq, int Hkv, int Lq, int Dk, int Dv,
                        int kfmt, int kbits, int kgs, const uint32_t* kcodes,
                        const uint16_t* kscales, const uint16_t* kbiases,
                        int64_t Lcap, int64_t L, double scale, int mask_kind,
                        const void* mask_add, int mask_dtype, int64_t msb,
                        int64_t msh, int64_t msq, double softcap,
                        const double* sinks, const double* slopes, int mode, int nsplit,
                        const int64_t* rows, int64_t nrows, double* out,
                        int nthreads) {
  if (Hkv <= 0 || Hq % Hkv != 0 || L < 0 || L > Lcap || Dv <= 0 || Dv > Dk) return 1;
  if (kfmt == 1) { kbits = 8; kgs = 32; }
  Problem p;
  p.q = q; p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lq = Lq; p.D = Dk; p.Dv = Dv;
  p.k = make_cache(kfmt, kbits, kgs, kcodes, kscales, kbiases, Lcap);
  p.v = p.k;                                            // values: the key rows themselves
  p.L = L; p.scale = scale;
  p.mask.kind = mask_kind; p.mask.add = mask_add; p.mask.add_dtype = mask_dtype;
  p.mask.sb = msb; p.mask.sh = msh; p.mask.sq = msq;
  p.softcap = softcap; p.sinks = sinks; p.slopes = slopes;
  const int64_t total = rows ? nrows : (int64_t)B * Hq * Lq;
  run_rows(p, mode, nsplit, rows, total, out, nthreads);
  return 0;
}

// Softmax probabilities of one query row (b,h,i) over the L keys (two-pass).
int orc_attention_probs(const double* q, int B, int Hq, int Hkv, int Lq, int D,
                        int kfmt, int kbits, int kgs, const uint32_t* kcodes,
                        const uint16_t* kscales, const uint16_t* kbiases,
                        int vfmt, int vbits, int vgs, const uint32_t* vcodes,
                        const uint16_t* vscales, const uint16_t* vbiases,
                        int64_t Lcap, int64_t L, double scale, int mask_kind,
                        const void* mask_add, int mask_dtype, int64_t msb,
                        int64_t msh, int64_t msq, double softcap,
                        const double* sinks, const double* slopes, int b, int h, int i,
                        double* probs, double* o) {
  if (Hkv <= 0 || Hq % Hkv != 0 || L < 0 || L > Lcap) return 1;
  if (kfmt == 1) { kbits = 8; kgs = 32; }
  if (vfmt == 1) { vbits = 8; vgs = 32; }
  Problem p;
  p.q = q; p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lq = Lq; p.D = D; p.Dv = D;
  p.k = make_cache(kfmt, kbits, kgs, kcodes, kscales, kbiases, Lcap);
  p.v = make_cache(vfmt, vbits, vgs, vcodes, vscales, vbiases, Lcap);
  p.L = L; p.scale = scale;
  p.mask.kind = mask_kind; p.mask.add = mask_add; p.mask.add_dtype = mask_dtype;
  p.mask.sb = msb; p.mask.sh = msh; p.mask.sq = msq;
  p.softcap = softcap; p.sinks = sinks; p.slopes = slopes;
  attend_two_pass(p, b, h, i, o, probs);
  return 0;
}

}  // extern "C"
