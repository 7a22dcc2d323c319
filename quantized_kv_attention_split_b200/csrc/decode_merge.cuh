// decode_merge.cuh -- second pass of the split-K decode, as its own kernel:
// the log-sum-exp merge (decode_fold.cuh) of the per-CTA partials of every
// split unit.
#pragma once

#include "qkv_common.cuh"
#include "qkv_internal.h"
#include "decode_fold.cuh"

namespace qkv {

// ---------------------------------------------------------------------------
// Merge of split units: after the decode grid has completed, `lanes`
// adjacent threads (a power of two up to 4, chosen so that a thread's share of
// the parts fits one batch of loads) per (unit, row, 4 consecutive outputs)
// fold the unit's partials.  A unit that one CTA covered whole was written by
// that CTA.  (Folding in the decode kernel instead -- the last CTA of a unit,
// found with an atomic count, folds the others' partials -- measured slower:
// the count's round trip and the fold sit on the grid's critical path.)
constexpr int kMergeThreads = 128;

template <int D, int HPC>
__global__ void __launch_bounds__(kMergeThreads)
qsdpa_merge_kernel(const __grid_constant__ DecodeParams p, int64_t nC, int lanes) {
  grid_dep_launch();             // the next kernel may take SMs as this one's CTAs finish
  grid_dep_wait();               // the decode grid's partials are complete and visible
  constexpr int V4 = D / 4;
  const int64_t S = p.stages_per_unit, T = p.total_stages;
  const int gt = blockIdx.x * kMergeThreads + threadIdx.x;
  const int sub = gt & (lanes - 1);
  const int item = gt >> (31 - __clz(lanes));
  const int u = item / (HPC * V4);
  const int r = item - u * (HPC * V4), R = r / V4, e4 = r - R * V4;
  const int uh = p.ncg == 1 ? u : u / p.ncg;
  const int head = (u - uh * p.ncg) * HPC + R;
  const int units = (int)udiv64(T, S);
  bool active = u < units && head < p.G;
  UnitParts up;
  up.cfirst = 0; up.slot0 = 0; up.n = 0;
  if (active) up = unit_parts(p, u, nC);
  active = active && up.n > 1;
  merge_item<D, HPC>(p, up, uh, head, R, e4, sub, lanes, active);
}

}  // namespace qkv
