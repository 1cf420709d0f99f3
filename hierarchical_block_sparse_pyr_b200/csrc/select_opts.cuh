// Selection variants shared by the three walk kernels (tensor-core prefill,
// CUDA-core prefill, decode): the PHAROS page's budget allocation (DBA),
// confidence fallback (FCF) and cross-level guidance (RCG), and the trace of
// the nodes kept at each level.
//   DBA  level 0 keeps budget[unit] blocks (clamped to [0, topk]); without a
//        budget array, topk - fcf_extra.
//   FCF  the confidence is the smallest margin (last kept - first dropped)
//        over the levels above 0 and at the level-0 budget boundary; below
//        fcf_tau, level 0 keeps min(budget + fcf_extra, topk) blocks.
//   RCG  candidates rank by R = S + rcg_lambda * R(parent) (R = S at the start
//        level); margins and the gap are taken on R.
//   gap  the smallest margin of any decision taken: each level's margin at
//        the boundary it used, and |confidence - fcf_tau| when the fallback
//        could change the result.
#pragma once

#include "pyr_common.cuh"

namespace pyr {

struct SelOpts {
  const int32_t* budget;  // [B * Hkv] or null
  float fcf_tau;
  int fcf_extra;          // 0: no fallback
  float rcg_lambda;       // 0: no guidance
  int32_t* trace;         // [B * Hkv][nqb][s0 + 1][tw] or null
  int tw;                 // trace entries per level: max(cap / 2, topk)
};

// Level-0 budget of a unit before any fallback.
__device__ __forceinline__ int sel_base_budget(const SelOpts& o, const Geo& g, int unit) {
  const int b = o.budget ? o.budget[unit] : g.topk - o.fcf_extra;
  return min(max(b, 0), g.topk);
}

// Level-0 keep count with the fallback on, from the n candidates' ranking
// scores by rank (sbr[r], best first) and the confidence of the levels above.
// *decision_margin: |c - fcf_tau| when keeping more would change the result,
// +inf otherwise.
__device__ __forceinline__ int sel_fcf_keep(const SelOpts& o, const Geo& g, int base, int n, const float* sbr,
                                            float conf, float* decision_margin) {
  const int kb = min(base, n);
  float c = conf;
  if (kb > 0 && kb < n) c = fminf(c, sbr[kb - 1] - sbr[kb]);
  const int wide = min(min(base + o.fcf_extra, g.topk), n);
  *decision_margin = wide != kb ? fabsf(c - o.fcf_tau) : __int_as_float(0x7f800000);
  return c < o.fcf_tau ? wide : kb;
}

// The trace row of level l for (unit, query block qb).
__device__ __forceinline__ int32_t* sel_trace_row(const SelOpts& o, const Geo& g, int unit, int qb, int l) {
  return o.trace + (((size_t)unit * g.nqb + qb) * (g.s0 + 1) + (g.s0 - l)) * o.tw;
}

}  // namespace pyr
