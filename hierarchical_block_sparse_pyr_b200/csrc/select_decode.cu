// Coarse-to-fine LogSumExp top-K key-block selection for decode (one query
// row per head): the PISA walk (start at the coarsest level, score a bounded
// candidate set with LogSumExp, pass the survivors' children on) for the
// block that holds the new token, routes to strictly preceding blocks with -1
// padding (PHBA A.1.2).
//
// A decode walk scores at most `cap` nodes per level against only G query
// rows, so it is a short latency chain: one 128-thread CTA per (batch, kv
// head), TPC threads per candidate (TPC = 128 / cap slots: 2 for cap <= 64,
// 1 for cap <= 128), each taking d / TPC elements of the node mean from its
// (hi, lo) pair in fp32 and of all G query rows (held in shared memory,
// pre-scaled by log2(e) / sqrt(d)). Per level: the thread's 16-byte loads of
// the candidate's (hi, lo) row, all issued before the first is used (one memory
// round trip), FMAs, a shuffle between the candidate's threads, the LogSumExp over the G
// rows, a rank count over packed keys (ties to the lower node index), and
// the kept node of rank r writes its children to slots 2r, 2r+1. The node
// that straddles the query block uses the exact mean of its part before the
// block, precomputed for every level from the binary decomposition of
// [m 2^l, i) into whole finer nodes. fp32 throughout.
// The PHAROS variants and the trace follow select_opts.cuh: guidance adds the
// parent's ranking score, the level-0 keep count comes from the budget and,
// with the fallback, from the scores by rank after one more barrier.
#include "pyr_common.cuh"
#include "select_opts.cuh"

namespace pyr {

namespace {

constexpr int kThreads = 128;
constexpr int kMaxCap = 128;
constexpr int kMaxG = 8;
constexpr int kMaxLevels = 24;

__device__ __forceinline__ float key_score_d(unsigned long long k) {
  const uint32_t u = (uint32_t)(k >> 32);
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; k++) {
    f[2 * k] = __uint_as_float(w[k] << 16);
    f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}

template <typename T, int D, int TPC>
__global__ void __launch_bounds__(kThreads) select_decode_kernel(const T* __restrict__ Q,
                                                                 const __nv_bfloat16* __restrict__ pyr,
                                                                 int32_t* __restrict__ idx, float* __restrict__ gap_out,
                                                                 Geo g, SelOpts o) {
  constexpr int DPT = D / TPC;  // elements of d per thread
  __shared__ __align__(16) float q_s[kMaxG * D];
  __shared__ __align__(16) float part[kMaxLevels * D];
  __shared__ __align__(16) unsigned long long keys[kMaxCap + 8];
  __shared__ int cand[kMaxCap];
  __shared__ int kept[kMaxCap];
  __shared__ float s_edge[2];
  __shared__ float s_gap;
  __shared__ float s_conf;
  __shared__ float sbr[kMaxCap];  // level-0 ranking scores by rank (fallback decision)
  __shared__ float psc[kMaxCap];  // parent's ranking score per candidate slot (guidance)

  const int tid = threadIdx.x;
  const int unit = blockIdx.x;
  const int bi = unit / g.Hkv, hk = unit % g.Hkv;
  const int G = g.G;
  const int p = g.q_offset;  // the query's position (Nq == 1)
  const int i = p / g.b;
  const __nv_bfloat16* pu = pyr + (size_t)unit * g.P * 2 * D;
  const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
  auto straddler = [&](int l) { return (l > 0 && (i & ((1 << l) - 1)) != 0) ? (i >> l) : -1; };

  // the G query rows, scaled so that dot products come out in log2 units
  for (int x = tid; x < G * D; x += kThreads) {
    const int gg = x / D, e = x - gg * D;
    q_s[x] = to_f32(Q[((size_t)bi * g.Hq + hk * G + gg) * g.Nq * D + e]) * sl2;
  }
  // exact means of the straddling nodes' parts before i, levels 1..s0
  for (int e = tid; e < D; e += kThreads) {
    float acc = 0.f;
    for (int l = 1; l <= g.s0; l++) {
      if ((i >> (l - 1)) & 1)
        acc += split_load(pu + (size_t)(g.lvl_off[l - 1] + (i >> (l - 1)) - 1) * 2 * D, D, e) *
               (float)(g.b << (l - 1));
      const int cnt = i - ((i >> l) << l);
      part[l * D + e] = cnt > 0 ? acc / (float)(cnt * g.b) : 0.f;
    }
  }
  if (tid == 0) s_gap = s_conf = __int_as_float(0x7f800000);
  __syncthreads();
  const int base = sel_base_budget(o, g, unit);
  const bool rcg = o.rcg_lambda != 0.f;

  const int my_c = tid / TPC, my_h = tid % TPC;  // scoring: candidate slot, part of d
  int nc = min(g.lvl_n[g.s0], (i + (1 << g.s0) - 1) >> g.s0);
  int32_t* out = idx + (size_t)unit * g.topk;

  for (int l = g.s0; l >= 0; l--) {
    const bool start = (l == g.s0);
    const int ms = straddler(l);
    const int slot_m = tid < nc ? (start ? tid : cand[tid]) : -1;
    // ---- score: this thread's share of q_g . kbar_m for every row g
    const int m = my_c < nc ? (start ? my_c : cand[my_c]) : -1;
    float acc[kMaxG];
#pragma unroll
    for (int gg = 0; gg < kMaxG; gg++) acc[gg] = 0.f;
    if (m >= 0) {
      const int e0 = my_h * DPT;
      if (m == ms) {
        const float* pr = part + l * D + e0;
        for (int e = 0; e < DPT; e += 4) {
          const float4 kv = *reinterpret_cast<const float4*>(pr + e);
#pragma unroll
          for (int gg = 0; gg < kMaxG; gg++) {
            if (gg < G) {
              const float4 qa = *reinterpret_cast<const float4*>(q_s + gg * D + e0 + e);
              acc[gg] = fmaf(qa.x, kv.x, fmaf(qa.y, kv.y, fmaf(qa.z, kv.z, fmaf(qa.w, kv.w, acc[gg]))));
            }
          }
        }
      } else {
        const __nv_bfloat16* row = pu + (size_t)(g.lvl_off[l] + m) * 2 * D;
        const uint4* hi4 = reinterpret_cast<const uint4*>(row + e0);
        const uint4* lo4 = reinterpret_cast<const uint4*>(row + D + e0);
        // every 16-byte load of this thread's share first: one memory round trip per level
        uint4 hv[DPT / 8], lv[DPT / 8];
#pragma unroll
        for (int v = 0; v < DPT / 8; v++) {
          hv[v] = __ldg(hi4 + v);
          lv[v] = __ldg(lo4 + v);
        }
#pragma unroll
        for (int v = 0; v < DPT / 8; v++) {
          float hf[8], lf[8], kv[8];
          bf16x8_to_f32(hv[v], hf);
          bf16x8_to_f32(lv[v], lf);
#pragma unroll
          for (int k = 0; k < 8; k++) kv[k] = hf[k] + lf[k];
          const int e = e0 + v * 8;
#pragma unroll
          for (int gg = 0; gg < kMaxG; gg++) {
            if (gg < G) {
              // the 8 query elements of row gg as two 16-byte loads (the same for every candidate: broadcast)
              const float4 qa = *reinterpret_cast<const float4*>(q_s + gg * D + e);
              const float4 qb = *reinterpret_cast<const float4*>(q_s + gg * D + e + 4);
              float a = acc[gg];
              a = fmaf(qa.x, kv[0], a);
              a = fmaf(qa.y, kv[1], a);
              a = fmaf(qa.z, kv[2], a);
              a = fmaf(qa.w, kv[3], a);
              a = fmaf(qb.x, kv[4], a);
              a = fmaf(qb.y, kv[5], a);
              a = fmaf(qb.z, kv[6], a);
              a = fmaf(qb.w, kv[7], a);
              acc[gg] = a;
            }
          }
        }
      }
    }
    if (TPC == 2) {
#pragma unroll
      for (int gg = 0; gg < kMaxG; gg++) acc[gg] += __shfl_xor_sync(0xffffffffu, acc[gg], 1);
    }
    // ---- LogSumExp over the G rows (log2 units), key of the candidate
    if (my_h == 0 && my_c < nc) {
      unsigned long long key = 0ull;  // empty slots rank below every node
      if (m >= 0) {
        float mx = acc[0];
#pragma unroll
        for (int gg = 1; gg < kMaxG; gg++)
          if (gg < G) mx = fmaxf(mx, acc[gg]);
        float s = 0.f;
#pragma unroll
        for (int gg = 0; gg < kMaxG; gg++)
          if (gg < G) s += exp2f(acc[gg] - mx);
        const int j0 = m << l;
        const int j1 = min(min((m + 1) << l, g.nb), i);
        const float nval = (float)(min((int64_t)j1 * g.b, (int64_t)g.N) - (int64_t)j0 * g.b);
        float sc = (mx + __log2f(s)) * 0.6931471805599453f + __logf(nval);
        if (rcg && !start) sc = fmaf(o.rcg_lambda, psc[my_c], sc);
        key = ((unsigned long long)float_order_key(sc) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)m);
      }
      keys[my_c] = key;
    }
    const int nc8 = (nc + 7) & ~7;
    if (tid >= nc && tid < nc8) keys[tid] = 0ull;
    const int n_valid = __syncthreads_count(slot_m >= 0);
    // ---- keep the best; a kept node of rank r puts its children in slots 2r, 2r + 1
    const int keep_lo = min(l > 0 ? g.cap / 2 : base, n_valid);
    int32_t* trow = o.trace ? sel_trace_row(o, g, unit, 0, l) : nullptr;
    int my_rank = -1;
    unsigned long long my_key = 0ull;
    if (slot_m >= 0) {
      my_key = keys[tid];
      int rank = 0;
      const ulonglong2* k2 = reinterpret_cast<const ulonglong2*>(keys);
      for (int c = 0; c < nc8 / 2; c += 4) {
        const ulonglong2 a0 = k2[c], a1 = k2[c + 1], a2 = k2[c + 2], a3 = k2[c + 3];
        rank += (a0.x > my_key) + (a0.y > my_key) + (a1.x > my_key) + (a1.y > my_key) + (a2.x > my_key) +
                (a2.y > my_key) + (a3.x > my_key) + (a3.y > my_key);
      }
      my_rank = rank;
    }
    int keep = keep_lo;
    float decision_margin = __int_as_float(0x7f800000);
    if (l == 0 && o.fcf_extra > 0 && keep_lo < n_valid) {  // block-uniform
      if (my_rank >= 0) sbr[my_rank] = key_score_d(my_key);
      __syncthreads();
      keep = sel_fcf_keep(o, g, base, n_valid, sbr, s_conf, &decision_margin);
    }
    if (my_rank >= 0) {
      if (my_rank < keep) {
        if (l > 0) {
          const int c1 = 2 * slot_m + 1;
          cand[2 * my_rank] = 2 * slot_m;
          cand[2 * my_rank + 1] = (c1 < g.lvl_n[l - 1] && (c1 << (l - 1)) < i) ? c1 : -1;
          if (rcg) psc[2 * my_rank] = psc[2 * my_rank + 1] = key_score_d(my_key);
        } else {
          kept[my_rank] = slot_m;
        }
        if (trow) trow[my_rank] = slot_m;
      }
      if (my_rank == keep - 1) s_edge[0] = key_score_d(my_key);
      if (my_rank == keep) s_edge[1] = key_score_d(my_key);
    }
    if (trow && tid >= keep && tid < o.tw) trow[tid] = -1;
    __syncthreads();
    if (tid == 0) {
      if (keep < n_valid && keep > 0) {
        const float mg = s_edge[0] - s_edge[1];
        s_gap = fminf(s_gap, mg);
        if (l > 0) s_conf = fminf(s_conf, mg);
      }
      s_gap = fminf(s_gap, decision_margin);
    }
    nc = 2 * keep;
    if (l == 0) {
      for (int k = tid; k < g.topk; k += kThreads) {
        if (k < keep) {
          const int mk = kept[k];
          int pos = 0;
          for (int k2 = 0; k2 < keep; k2++) pos += kept[k2] < mk;
          out[pos] = mk;
        } else {
          out[k] = -1;
        }
      }
      __syncthreads();
      if (gap_out && tid == 0) gap_out[unit] = s_gap;
    }
  }
}

template <typename T, int D>
cudaError_t launch_dec(const Geo& g, const void* Q, const __nv_bfloat16* pyr, int32_t* idx, float* gap,
                       const SelOpts& o, cudaStream_t st) {
  if (g.cap <= 64)
    select_decode_kernel<T, D, 2><<<g.B * g.Hkv, kThreads, 0, st>>>(static_cast<const T*>(Q), pyr, idx, gap, g, o);
  else
    select_decode_kernel<T, D, 1><<<g.B * g.Hkv, kThreads, 0, st>>>(static_cast<const T*>(Q), pyr, idx, gap, g, o);
  return cudaGetLastError();
}

}  // namespace

bool select_decode_supported(const Geo& g) {
  return g.Nq == 1 && g.G <= kMaxG && g.cap <= kMaxCap && g.s0 < kMaxLevels && (g.d == 64 || g.d == 128);
}

cudaError_t launch_select_decode(const Geo& g, const void* Q, const __nv_bfloat16* pyr, int32_t* idx, float* gap,
                                 const SelOpts& o, cudaStream_t st) {
  if (g.dtype == PYR_F32) {
    if (g.d == 64) return launch_dec<float, 64>(g, Q, pyr, idx, gap, o, st);
    return launch_dec<float, 128>(g, Q, pyr, idx, gap, o, st);
  }
  if (g.d == 64) return launch_dec<__nv_bfloat16, 64>(g, Q, pyr, idx, gap, o, st);
  return launch_dec<__nv_bfloat16, 128>(g, Q, pyr, idx, gap, o, st);
}

}  // namespace pyr
