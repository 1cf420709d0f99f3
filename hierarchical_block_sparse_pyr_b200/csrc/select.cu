// Coarse-to-fine LogSumExp top-K key-block selection (PISA abstract: start
// at the coarsest level, score a bounded candidate set with LogSumExp, pass
// the survivors' children to the next finer level; routes only to strictly
// preceding blocks with -1 padding, PHBA A.1.2).
//
// One CTA per (batch, kv head, query block i). The CTA stages the G*b query
// rows of the block once, then walks the levels s0 .. 0. Per level:
//   gather   <= cap candidate node means (the node that straddles block i
//            uses the exact mean of its part before i, built from the
//            binary decomposition of [m 2^l, i) into whole finer nodes);
//   score    x_rc = q_r . kbar_c / sqrt(d) as a register-tiled GEMM-let
//            (64x64 output tiles, 4x4 per thread), then per column an
//            online max / sum-exp over the rows and S_c = LSE + ln n_valid;
//   select   bitonic sort of packed 64-bit keys (order-preserving score bits
//            over the inverted node index, so ties go to the lower index),
//            keep cap/2 (levels > 0) or topk (level 0), expand children.
// fp32 throughout; the score matrix never leaves shared memory.
// The PHAROS variants and the trace follow select_opts.cuh (guidance adds the
// parent's ranking score; the level-0 keep count comes from the budget and the
// fallback; the trace lists the kept nodes of every level).
#include "pyr_common.cuh"
#include "select_opts.cuh"

namespace pyr {

namespace {

constexpr int kThreads = 256;
constexpr int kTile = 64;      // output tile edge (rows and columns)
constexpr int kMaxCap = 128;
constexpr int kMaxLevels = 24;

struct SelSmem {
  // offsets in bytes into dynamic shared memory
  size_t q, mt, st, colm, cols, keys, cand, nval, part, pcnt, psc, total;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~(size_t)15; }

// Row pitch (floats) of the transposed candidate tile: a multiple of 4 so that
// float4 loads stay 16-byte aligned, plus 4 to spread the banks.
__host__ __device__ inline int cand_pitch(int cap) { return ((cap + 3) & ~3) + 4; }

__host__ __device__ inline SelSmem sel_layout(int R, int d, int elt, int cap) {
  SelSmem s;
  const int CP = cand_pitch(cap);
  size_t o = 0;
  s.q = o;    o = align16(o + (size_t)d * R * elt);
  s.mt = o;   o = align16(o + (size_t)d * CP * 4);
  s.st = o;   o = align16(o + (size_t)kTile * (kTile + 1) * 4);
  s.colm = o; o = align16(o + (size_t)kMaxCap * 4);
  s.cols = o; o = align16(o + (size_t)kMaxCap * 4);
  s.keys = o; o = align16(o + (size_t)kMaxCap * 8);
  s.cand = o; o = align16(o + (size_t)2 * kMaxCap * 4);
  s.nval = o; o = align16(o + (size_t)kMaxCap * 4);
  s.part = o; o = align16(o + (size_t)kMaxLevels * d * 4);
  s.pcnt = o; o = align16(o + (size_t)kMaxLevels * 4);
  s.psc = o;  o = align16(o + (size_t)2 * kMaxCap * 4);
  s.total = o;
  return s;
}

__device__ __forceinline__ float key_to_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Descending bitonic sort of n_pow2 64-bit keys in shared memory.
__device__ void bitonic_desc(unsigned long long* key, int n_pow2) {
  for (int k = 2; k <= n_pow2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int t = threadIdx.x; t < n_pow2; t += kThreads) {
        const int p = t ^ j;
        if (p > t) {
          const unsigned long long a = key[t], b = key[p];
          const bool desc = (t & k) == 0;
          if (desc ? (a < b) : (a > b)) {
            key[t] = b;
            key[p] = a;
          }
        }
      }
      __syncthreads();
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) select_kernel(const T* __restrict__ Q, const __nv_bfloat16* __restrict__ pyr,
                                                          int32_t* __restrict__ idx, float* __restrict__ gap_out,
                                                          int* status, Geo g, SelOpts o) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int qb = blockIdx.x;
  const int unit = blockIdx.y;
  const int bi = unit / g.Hkv, hk = unit % g.Hkv;
  const int i = g.i0 + qb;
  const int d = g.d;
  const int CP = cand_pitch(g.cap);

  // query rows of block i over the group's heads
  const int p0 = max(i * g.b, g.q_offset);
  const int p1 = min((i + 1) * g.b, g.q_offset + g.Nq);
  const int rb = p1 - p0;
  const int R = g.G * rb;
  const SelSmem L = sel_layout(g.G * min(g.b, g.Nq), d, (int)sizeof(T), g.cap);
  T* Qs = reinterpret_cast<T*>(smem + L.q);              // [d][R]
  float* Mt = reinterpret_cast<float*>(smem + L.mt);     // [d][CP]
  float* St = reinterpret_cast<float*>(smem + L.st);     // [64][65]
  float* colm = reinterpret_cast<float*>(smem + L.colm);
  float* cols = reinterpret_cast<float*>(smem + L.cols);
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(smem + L.keys);
  int* cand = reinterpret_cast<int*>(smem + L.cand);
  float* nval = reinterpret_cast<float*>(smem + L.nval);
  float* part = reinterpret_cast<float*>(smem + L.part);  // [s0+1][d] partial means
  float* pcnt = reinterpret_cast<float*>(smem + L.pcnt);
  float* psc = reinterpret_cast<float*>(smem + L.psc);  // parent's ranking score per candidate [2][kMaxCap]
  __shared__ int s_nc;
  __shared__ float s_gap;
  __shared__ float s_conf;
  const int base = sel_base_budget(o, g, unit);
  const bool rcg = o.rcg_lambda != 0.f;

  for (int x = threadIdx.x; x < R * d; x += kThreads) {
    const int r = x / d, e = x - r * d;
    const int gg = r / rb, t = p0 - g.q_offset + (r - gg * rb);
    const int hq = hk * g.G + gg;
    Qs[(size_t)e * R + r] = Q[(((size_t)bi * g.Hq + hq) * g.Nq + t) * d + e];
  }
  const __nv_bfloat16* pu = pyr + (size_t)unit * g.P * 2 * d;
  // exact means of the straddling node's valid part, levels 1..s0
  for (int e = threadIdx.x; e < d; e += kThreads) {
    float acc = 0.f;
    part[e] = 0.f;
    for (int l = 1; l <= g.s0 && l < kMaxLevels; l++) {
      if ((i >> (l - 1)) & 1) {
        const int m = (i >> (l - 1)) - 1;  // whole left sibling at level l-1
        acc += split_load(pu + (size_t)(g.lvl_off[l - 1] + m) * 2 * d, d, e) * (float)((int64_t)g.b << (l - 1));
      }
      const int cnt_blocks = i - ((i >> l) << l);
      part[l * d + e] = cnt_blocks > 0 ? acc / (float)((int64_t)cnt_blocks * g.b) : 0.f;
    }
  }
  if (threadIdx.x == 0) {
    int nc = 0;
    for (int m = 0; m < g.lvl_n[g.s0]; m++)
      if ((m << g.s0) < i) cand[nc++] = m;
    s_nc = nc;
    s_gap = s_conf = __int_as_float(0x7f800000);  // +inf
    for (int l = 0; l <= g.s0 && l < kMaxLevels; l++) pcnt[l] = (float)((int64_t)(i - ((i >> l) << l)) * g.b);
  }
  __syncthreads();

  const float scale = rsqrtf((float)d);
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;

  for (int l = g.s0; l >= 0; l--) {
    const int nc = s_nc;
    // gather candidate means (transposed) and valid token counts
    for (int x = threadIdx.x; x < nc * d; x += kThreads) {
      const int c = x / d, e = x - c * d;
      const int m = cand[c];
      const int j0 = m << l;
      const bool straddle = ((m + 1) << l) > i && j0 < i && l > 0;
      Mt[(size_t)e * CP + c] = straddle ? part[l * d + e] : split_load(pu + (size_t)(g.lvl_off[l] + m) * 2 * d, d, e);
    }
    for (int c = threadIdx.x; c < nc; c += kThreads) {
      const int m = cand[c];
      const int j0 = m << l;
      const int j1 = min(min((m + 1) << l, g.nb), i);
      const int64_t t1 = min((int64_t)j1 * g.b, (int64_t)g.N);
      nval[c] = (float)(t1 - (int64_t)j0 * g.b);
      colm[c] = -INFINITY;
      cols[c] = 0.f;
    }
    __syncthreads();

    for (int c0 = 0; c0 < nc; c0 += kTile) {
      for (int r0 = 0; r0 < R; r0 += kTile) {
        float acc[4][4];
#pragma unroll
        for (int a = 0; a < 4; a++)
#pragma unroll
          for (int bb = 0; bb < 4; bb++) acc[a][bb] = 0.f;
        const int rr = r0 + ty * 4, cc = c0 + tx * 4;
        if (rr < R && cc < nc) {
          for (int e = 0; e < d; e++) {
            float qv[4];
#pragma unroll
            for (int a = 0; a < 4; a++) qv[a] = (rr + a < R) ? to_f32(Qs[(size_t)e * R + rr + a]) : 0.f;
            const float4 mv = *reinterpret_cast<const float4*>(Mt + (size_t)e * CP + cc);
#pragma unroll
            for (int a = 0; a < 4; a++) {
              acc[a][0] = fmaf(qv[a], mv.x, acc[a][0]);
              acc[a][1] = fmaf(qv[a], mv.y, acc[a][1]);
              acc[a][2] = fmaf(qv[a], mv.z, acc[a][2]);
              acc[a][3] = fmaf(qv[a], mv.w, acc[a][3]);
            }
          }
        }
#pragma unroll
        for (int a = 0; a < 4; a++)
#pragma unroll
          for (int bb = 0; bb < 4; bb++) St[(ty * 4 + a) * (kTile + 1) + tx * 4 + bb] = acc[a][bb] * scale;
        __syncthreads();
        // online column LSE over this row tile: 4 threads per column
        {
          const int c = threadIdx.x / 4, part4 = threadIdx.x % 4;
          const int rows = min(kTile, R - r0);
          float m = -INFINITY, s = 0.f;
          if (c0 + c < nc) {
            for (int r = part4; r < rows; r += 4) m = fmaxf(m, St[r * (kTile + 1) + c]);
            for (int r = part4; r < rows; r += 4) s += expf(St[r * (kTile + 1) + c] - m);
          }
#pragma unroll
          for (int off = 1; off < 4; off <<= 1) {
            const float mo = __shfl_xor_sync(0xffffffffu, m, off);
            const float so = __shfl_xor_sync(0xffffffffu, s, off);
            const float mn = fmaxf(m, mo);
            s = (mn == -INFINITY) ? 0.f : s * expf(m - mn) + so * expf(mo - mn);
            m = mn;
          }
          if (part4 == 0 && c0 + c < nc) {
            const float mo = colm[c0 + c], so = cols[c0 + c];
            const float mn = fmaxf(m, mo);
            cols[c0 + c] = s * expf(m - mn) + ((mo == -INFINITY) ? 0.f : so * expf(mo - mn));
            colm[c0 + c] = mn;
          }
        }
        __syncthreads();
      }
    }

    // scores -> packed keys, padded to a power of two
    int np2 = 1;
    while (np2 < nc) np2 <<= 1;
    for (int c = threadIdx.x; c < np2; c += kThreads) {
      unsigned long long k = 0ull;
      if (c < nc) {
        float sc = colm[c] + logf(cols[c]) + logf(nval[c]);
        if (rcg && l < g.s0) sc = fmaf(o.rcg_lambda, psc[c], sc);
        k = ((unsigned long long)float_order_key(sc) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)cand[c]);
      }
      keys[c] = k;
    }
    __syncthreads();
    bitonic_desc(keys, np2);

    const int keep_lo = min(l > 0 ? g.cap / 2 : base, nc);
    int keep = keep_lo;
    float decision_margin = __int_as_float(0x7f800000);
    if (l == 0 && o.fcf_extra > 0 && keep_lo < nc) {
      // the scores by rank, from the sorted keys (colm is free once the keys are made)
      for (int c = threadIdx.x; c < nc; c += kThreads) colm[c] = key_to_float((uint32_t)(keys[c] >> 32));
      __syncthreads();
      keep = sel_fcf_keep(o, g, base, nc, colm, s_conf, &decision_margin);
    }
    if (o.trace) {
      int32_t* trow = sel_trace_row(o, g, unit, qb, l);
      for (int k = threadIdx.x; k < o.tw; k += kThreads)
        trow[k] = k < keep ? (int)(0xFFFFFFFFu - (uint32_t)(keys[k] & 0xFFFFFFFFull)) : -1;
    }
    if (threadIdx.x == 0) {
      if (keep < nc && keep > 0) {
        const float a = key_to_float((uint32_t)(keys[keep - 1] >> 32));
        const float b = key_to_float((uint32_t)(keys[keep] >> 32));
        s_gap = fminf(s_gap, a - b);
        if (l > 0) s_conf = fminf(s_conf, a - b);
      }
      s_gap = fminf(s_gap, decision_margin);
      if (l > 0) {
        int nn = 0;
        int* next = cand + kMaxCap;
        float* next_p = psc + kMaxCap;
        for (int k = 0; k < keep; k++) {
          const int m = (int)(0xFFFFFFFFu - (uint32_t)(keys[k] & 0xFFFFFFFFull));
          const float r = key_to_float((uint32_t)(keys[k] >> 32));
          for (int ch = 2 * m; ch <= 2 * m + 1; ch++)
            if (ch < g.lvl_n[l - 1] && (ch << (l - 1)) < i) {
              next_p[nn] = r;
              next[nn++] = ch;
            }
        }
        for (int k = 0; k < nn; k++) {
          cand[k] = next[k];
          psc[k] = next_p[k];
        }
        s_nc = nn;
      }
    }
    __syncthreads();
    if (l == 0) {
      // kept blocks in ascending order, then -1
      int32_t* out = idx + ((size_t)unit * g.nqb + qb) * g.topk;
      for (int k = threadIdx.x; k < g.topk; k += kThreads) {
        if (k < keep) {
          const int m = (int)(0xFFFFFFFFu - (uint32_t)(keys[k] & 0xFFFFFFFFull));
          int rank = 0;
          for (int k2 = 0; k2 < keep; k2++) {
            const int m2 = (int)(0xFFFFFFFFu - (uint32_t)(keys[k2] & 0xFFFFFFFFull));
            rank += (m2 < m);
          }
          out[rank] = m;
        } else {
          out[k] = -1;
        }
      }
      if (gap_out && threadIdx.x == 0) gap_out[(size_t)unit * g.nqb + qb] = s_gap;
    }
  }
  (void)status;
}

template <typename T>
cudaError_t launch_t(const Geo& g, const void* Q, const __nv_bfloat16* pyr, int32_t* idx, float* gap, int* status,
                     const SelOpts& o, cudaStream_t st) {
  const SelSmem L = sel_layout(g.G * min(g.b, g.Nq), g.d, (int)sizeof(T), g.cap);
  auto kern = select_kernel<T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  dim3 grid(g.nqb, g.B * g.Hkv);
  kern<<<grid, kThreads, L.total, st>>>(reinterpret_cast<const T*>(Q), pyr, idx, gap, status, g, o);
  return cudaGetLastError();
}

}  // namespace

size_t select_smem_bytes(const Geo& g) {
  const int elt = g.dtype == PYR_BF16 ? 2 : 4;
  return sel_layout(g.G * min(g.b, g.Nq), g.d, elt, g.cap).total;
}

cudaError_t launch_select(const Geo& g, const void* Q, const __nv_bfloat16* pyr, int32_t* idx, float* gap, int* status,
                          const SelOpts& o, cudaStream_t st) {
  if (g.dtype == PYR_BF16) return launch_t<__nv_bfloat16>(g, Q, pyr, idx, gap, status, o, st);
  return launch_t<float>(g, Q, pyr, idx, gap, status, o, st);
}

}  // namespace pyr
