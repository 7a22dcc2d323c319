// decode_plan.cu -- chooses the decode kernel instance and its work split.
#include <algorithm>

#include "decode_dispatch.cuh"

namespace qkv {

namespace {

// Grid cap per SM used both for planning and for the workspace bound, so that
// qsdpa_workspace_size() does not depend on the kernel instance.
int max_ctas_per_sm(int D) { return dec_ctas_per_sm(D); }
// Largest grid (the workspace holds two partial slots per CTA).
constexpr int64_t kMaxGrid = 8 * 48;
// Partials of at least this many floats count as large (16 rows x D = 256 do).
constexpr int64_t kBigPartial = 2048;
constexpr int64_t kBigPartMinStages = 2;   // blocks per team
// With large partials, at most this many CTAs share a unit: the merge reads
// every partial, and beyond this the longer merge costs more than the shorter
// loop gains (Q8_0, D = 256, 16 rows, 10K and 20K keys: 64 measured best of
// 32, 48 and 64 since the epilogue combines four elements per thread).
constexpr int64_t kBigPartMaxPieces = 64;

// SM count of the current device, queried once per device (every decode call
// plans its grid with it).
int sm_count() {
  constexpr int kMaxDevices = 64;
  static int cached[kMaxDevices] = {};
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kMaxDevices && cached[dev] > 0) return cached[dev];
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kMaxDevices) cached[dev] = n;
  return n;
}

bool get_ops(int D, int bits, int gs, int fmt, int nc, bool f32, int var, DecodeOps* ops) {
  const bool q8 = fmt == QKV_Q8_0;
  if (!q8 && bits != 4 && bits != 8) {
    // codes stored 2, 3, 5 or 6 bits wide: the plain kernel only
    if (var != kDecPlain) return false;
    if (D == 64) return decode_ops_x_d64(bits, gs, nc, f32, ops);
    if (D == 128) return decode_ops_x_d128(bits, gs, nc, f32, ops);
    if (D == 256) return decode_ops_x_d256(bits, gs, nc, f32, ops);
    return false;
  }
  if (D == 64) return decode_ops_d64(bits, gs, q8, nc, f32, var, ops);
  if (D == 128) return decode_ops_d128(bits, gs, q8, nc, f32, var, ops);
  if (D == 256) return decode_ops_d256(bits, gs, q8, nc, f32, var, ops);
  return false;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

size_t max_grid(int D) {
  return (size_t)std::min<int64_t>((int64_t)std::max(1, sm_count()) * max_ctas_per_sm(D), kMaxGrid);
}

}  // namespace

void decode_chunking(int G, int* nc, int* ncg) {
  const int chunks = (G + 7) / 8;
  *nc = chunks <= 1 ? 1 : (chunks <= 2 ? 2 : 4);
  *ncg = (chunks + *nc - 1) / *nc;
}

// Workspace layout: a 256-byte header that is zero between calls (its first
// word is the prefill's status word; decode leaves it alone), then two
// partial slots per CTA: o, then (m, l).
constexpr size_t kWsHeader = 256;
void decode_ws_layout(size_t hpc, int D, size_t maxgrid, DecodePlan* plan) {
  plan->ws_header = kWsHeader;
  plan->ws_part_o = round_up(2 * maxgrid * hpc * D * 4, 256);
  plan->ws_part_ml = round_up(2 * maxgrid * hpc * 2 * 4, 256);
  plan->ws_total = plan->ws_header + plan->ws_part_o + plan->ws_part_ml;
}

size_t decode_workspace_bound(int B, int Hq, int Hkv, int D) {
  if (B <= 0 || Hkv <= 0 || Hq % Hkv) return 0;
  int nc, ncg;
  decode_chunking(Hq / Hkv, &nc, &ncg);
  (void)ncg;
  DecodePlan plan;
  decode_ws_layout((size_t)nc * 8, D, max_grid(D), &plan);
  return plan.ws_total;
}

size_t decode_workspace_zero_bytes(int B, int Hq, int Hkv) {
  if (B <= 0 || Hkv <= 0 || Hq % Hkv) return 0;
  return kWsHeader;
}

bool plan_decode(int D, int bits, int gs, int fmt, int out_f32, int var, int B, int Hq,
                 int Hkv, int64_t L, DecodePlan* plan) {
  int nc, ncg;
  decode_chunking(Hq / Hkv, &nc, &ncg);
  DecodeOps ops;
  if (!get_ops(D, bits, gs, fmt, nc, out_f32 != 0, var, &ops)) return false;
  plan->var = var;
  const int sms = std::max(1, sm_count());
  const int occ = std::min(max_ctas_per_sm(D), std::max(1, ops.occupancy()));
  plan->tk = ops.tk;
  plan->nc = nc;
  plan->hpc = nc * 8;
  plan->ncg = ncg;
  plan->units = (int64_t)B * Hkv * ncg;
  plan->stages_per_unit = (L + ops.tk - 1) / ops.tk;
  plan->total_stages = plan->units * plan->stages_per_unit;
  // One CTA per SM, each a contiguous equal share of the (unit, block) range.
  int64_t cap = (int64_t)sms * occ;
  cap = std::min<int64_t>(cap, plan->total_stages);
  cap = std::min<int64_t>(cap, kMaxGrid);              // partial slots in the workspace
  // A CTA's partial (rows x D fp32) is written, read back and merged; when it
  // is large (many query rows per KV head, wide heads) give every team of
  // every CTA several blocks, so that partials stay a small fraction of the
  // bytes streamed.
  if ((int64_t)plan->hpc * D >= kBigPartial) {
    const int64_t per = (int64_t)ops.teams * kBigPartMinStages;
    cap = std::min<int64_t>(cap, std::max<int64_t>(1, plan->total_stages / per));
  }
  int64_t grid = std::max<int64_t>(1, cap);
  // When the units are few, cut every unit into the same number of pieces (no
  // CTA then covers parts of two units, which would cost it a second prologue
  // and epilogue), as long as that leaves at most 15% of the grid idle; no
  // more pieces than give every team a block (short caches: fewer partials).
  if (plan->units <= grid) {
    int64_t per_unit = std::min<int64_t>(grid / plan->units,
                                         (plan->stages_per_unit + ops.teams - 1) / ops.teams);
    bool capped = false;
    if ((int64_t)plan->hpc * D >= kBigPartial && per_unit > kBigPartMaxPieces) {
      per_unit = kBigPartMaxPieces;
      capped = true;
    }
    if (capped || per_unit * plan->units * 100 >= grid * 85 || per_unit * ops.teams >= plan->stages_per_unit)
      grid = std::max<int64_t>(1, per_unit) * plan->units;
  }
  plan->grid = (int)std::max<int64_t>(1, grid);
  plan->smem = ops.smem;
  // a merge kernel runs after the decode kernel when some unit is split over
  // several CTAs, i.e. some CTA boundary falls inside a unit
  plan->merge = false;
  for (int64_t c = 1; c < plan->grid && !plan->merge; ++c)
    plan->merge = (c * plan->total_stages / plan->grid) % plan->stages_per_unit != 0;
  plan->pieces = plan->grid % plan->units == 0 ? (int)(plan->grid / plan->units) : 0;
  decode_ws_layout((size_t)plan->hpc, D, max_grid(D), plan);
  return true;
}

cudaError_t launch_decode(int D, int bits, int gs, int fmt, int out_f32, const DecodePlan& plan,
                          DecodeParams& p, cudaStream_t stream) {
  DecodeOps ops;
  if (!get_ops(D, bits, gs, fmt, plan.nc, out_f32 != 0, plan.var, &ops)) return cudaErrorInvalidValue;
  p.ncg = plan.ncg;
  p.stages_per_unit = plan.stages_per_unit;
  p.total_stages = plan.total_stages;
  p.pieces = plan.pieces;
  return ops.launch(plan, p, stream);
}

}  // namespace qkv
