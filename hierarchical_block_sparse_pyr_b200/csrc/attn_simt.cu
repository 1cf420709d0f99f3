// Causal block-sparse attention on the CUDA cores, fp32 arithmetic (PHBA
// 3.1/3.3/A.1.3: routed blocks plus the current block under one online
// softmax; output and log-sum-exp written, no N x N matrix).
//
// One CTA per (batch, kv head, query block, chunk of 64 query rows). The rows
// of a chunk may come from several heads of the kv group (grouped-query
// attention shares the selection), so every K/V tile the CTA stages serves
// all of them. Keys are processed in 32-key sub-tiles: lane l of a warp owns
// key l for the scores and d/32 output columns for the P.V update; a warp
// owns 16 query rows. This kernel serves fp32 inputs (where the tolerance
// leaves no room for reduced-precision tensor-core operands) and is the
// general fallback for shapes the tensor-core kernels do not take.
// With PHBA prefix states (M > 0; PHBA summary 3.3 and A.1.3) the same online
// softmax continues over the M slots of the current block's state and of the
// state aligned with each routed block (blocks >= 1), scored with the
// state-branch query against the state keys; the slots carry no causal mask.
#include "pyr_common.cuh"

namespace pyr {

namespace {

constexpr int kRows = 64;      // query rows per CTA
constexpr int kWarps = 4;      // 16 rows per warp
constexpr int kKeys = 32;      // keys per sub-tile

template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) attn_simt_kernel(const T* __restrict__ Q, const T* __restrict__ K,
                                                                const T* __restrict__ V,
                                                                const int32_t* __restrict__ idx, int dense,
                                                                T* __restrict__ O, float* __restrict__ lse,
                                                                int* status, Geo g, const T* __restrict__ Qst,
                                                                const T* __restrict__ PK, const T* __restrict__ PV,
                                                                int M) {
  constexpr int CPL = D / 32;  // output columns per lane
  extern __shared__ __align__(16) float sm[];
  float* Qs = sm;                          // [64][D]
  float* Ks = Qs + kRows * D;              // [32][D+1]
  float* Vs = Ks + kKeys * (D + 1);        // [32][D]
  float* Ps = Vs + kKeys * D;              // [4 warps][16][32]
  __shared__ int s_blocks[130];
  __shared__ int s_nblk;

  const int qb = blockIdx.x, unit = blockIdx.y, chunk = blockIdx.z;
  const int bi = unit / g.Hkv, hk = unit % g.Hkv;
  const int i = g.i0 + qb;
  const int p0 = max(i * g.b, g.q_offset);
  const int p1 = min((i + 1) * g.b, g.q_offset + g.Nq);
  const int rb = p1 - p0;
  const int R = g.G * rb;
  const int r_begin = chunk * kRows;
  if (r_begin >= R) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float scale_log2 = rsqrtf((float)D) * 1.4426950408889634f;

  // stage the chunk's query rows
  for (int x = threadIdx.x; x < kRows * D; x += kWarps * 32) {
    const int r = x / D, e = x - r * D;
    const int ra = r_begin + r;
    float v = 0.f;
    if (ra < R) {
      const int gg = ra / rb, t = p0 - g.q_offset + (ra - gg * rb);
      v = to_f32(Q[(((size_t)bi * g.Hq + hk * g.G + gg) * g.Nq + t) * D + e]);
    }
    Qs[x] = v;
  }
  // the list of key blocks: selected (validated) then the diagonal
  if (threadIdx.x == 0) {
    int n = 0;
    if (!dense) {
      const int32_t* row = idx + ((size_t)unit * g.nqb + qb) * g.topk;
      int prev = -1;
      for (int k = 0; k < g.topk; k++) {
        const int j = row[k];
        if (j < 0) continue;
        if (j >= i || j <= prev) {
          report(status, PYR_EBADIDX);
          continue;
        }
        prev = j;
        s_blocks[n++] = j;
      }
    }
    s_blocks[n++] = i;
    s_nblk = n;
  }
  __syncthreads();

  // per-row state (warp rows r = warp*16 + rr)
  float m_run[16], l_run[16], acc[16][CPL];
  int pos[16];
#pragma unroll
  for (int rr = 0; rr < 16; rr++) {
    m_run[rr] = -INFINITY;
    l_run[rr] = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; c++) acc[rr][c] = 0.f;
    const int ra = r_begin + warp * 16 + rr;
    pos[rr] = -1;
    if (ra < R) {
      const int gg = ra / rb;
      pos[rr] = p0 + (ra - gg * rb);
    }
  }
  float* Pw = Ps + warp * 16 * kKeys;
  const T* Ku = K + (size_t)unit * g.N * D;
  const T* Vu = V + (size_t)unit * g.N * D;
  const int nblk = dense ? (i + 1) : s_nblk;

  // one staged sub-tile of up to 32 keys: scores, online softmax, P.V. Lane `lane` owns key `lane`
  // of the tile, valid when lane < n_keys and, with causal_first >= 0, when its position
  // causal_first + lane is at most the row's position
  auto consume_tile = [&](int n_keys, int causal_first) {
    float s[16];
#pragma unroll
    for (int rr = 0; rr < 16; rr++) s[rr] = 0.f;
    const float* Qw = Qs + warp * 16 * D;
    for (int e = 0; e < D; e++) {
      const float kv = Ks[lane * (D + 1) + e];
#pragma unroll
      for (int rr = 0; rr < 16; rr++) s[rr] = fmaf(Qw[rr * D + e], kv, s[rr]);
    }
#pragma unroll
    for (int rr = 0; rr < 16; rr++) {
      const bool ok = pos[rr] >= 0 && lane < n_keys && (causal_first < 0 || causal_first + lane <= pos[rr]);
      const float x = ok ? s[rr] * scale_log2 : -INFINITY;  // log2 domain
      float mx = x;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m_run[rr], mx);
      const float p = (m_new == -INFINITY) ? 0.f : exp2f(x - m_new);
      float ps = p;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      const float corr = (m_run[rr] == -INFINITY) ? 0.f : exp2f(m_run[rr] - m_new);
      l_run[rr] = l_run[rr] * corr + ps;
      m_run[rr] = m_new;
#pragma unroll
      for (int c = 0; c < CPL; c++) acc[rr][c] *= corr;
      Pw[rr * kKeys + lane] = p;
    }
    __syncwarp();
    for (int k = 0; k < kKeys; k++) {
      float vv[CPL];
#pragma unroll
      for (int c = 0; c < CPL; c++) vv[c] = Vs[k * D + lane + 32 * c];
#pragma unroll
      for (int rr = 0; rr < 16; rr++) {
        const float p = Pw[rr * kKeys + k];
#pragma unroll
        for (int c = 0; c < CPL; c++) acc[rr][c] = fmaf(p, vv[c], acc[rr][c]);
      }
    }
    __syncwarp();
  };
  // stage rows [r0, r0 + n) of K-like and V-like tensors (zeros past n)
  auto stage = [&](const T* Kt, const T* Vt, int n) {
    __syncthreads();  // previous sub-tile fully consumed
    for (int x = threadIdx.x; x < kKeys * D; x += kWarps * 32) {
      const int k = x / D, e = x - k * D;
      float kv = 0.f, vv = 0.f;
      if (k < n) {
        kv = to_f32(Kt[(size_t)k * D + e]);
        vv = to_f32(Vt[(size_t)k * D + e]);
      }
      Ks[k * (D + 1) + e] = kv;
      Vs[k * D + e] = vv;
    }
    __syncthreads();
  };

  for (int bk = 0; bk < nblk; bk++) {
    const int j = dense ? (bk < i ? bk : i) : s_blocks[bk];
    const int kb0 = j * g.b;
    const int kb1 = min(kb0 + g.b, g.N);
    for (int t0 = kb0; t0 < kb1; t0 += kKeys) {
      const int n = min(kKeys, kb1 - t0);
      stage(Ku + (size_t)t0 * D, Vu + (size_t)t0 * D, n);
      consume_tile(n, j < i ? -1 : t0);
    }
  }

  if (M > 0 && !dense) {
    // prefix-state slots: the state-branch query replaces the token query in shared memory
    if (Qst != Q) {
      __syncthreads();
      for (int x = threadIdx.x; x < kRows * D; x += kWarps * 32) {
        const int r = x / D, e = x - r * D;
        const int ra = r_begin + r;
        float v = 0.f;
        if (ra < R) {
          const int gg = ra / rb, t = p0 - g.q_offset + (ra - gg * rb);
          v = to_f32(Qst[(((size_t)bi * g.Hq + hk * g.G + gg) * g.Nq + t) * D + e]);
        }
        Qs[x] = v;
      }
    }
    const T* PKu = PK + (size_t)unit * g.nb * M * D;
    const T* PVu = PV + (size_t)unit * g.nb * M * D;
    for (int bk = 0; bk < nblk; bk++) {
      const int j = s_blocks[bk];  // routed blocks, then the current block
      if (j < 1) continue;         // block 0 has an empty prefix: no state
      for (int c0 = 0; c0 < M; c0 += kKeys) {
        const int n = min(kKeys, M - c0);
        stage(PKu + ((size_t)j * M + c0) * D, PVu + ((size_t)j * M + c0) * D, n);
        consume_tile(n, -1);
      }
    }
  }

#pragma unroll
  for (int rr = 0; rr < 16; rr++) {
    const int ra = r_begin + warp * 16 + rr;
    if (ra >= R) continue;
    const int gg = ra / rb, t = p0 - g.q_offset + (ra - gg * rb);
    const size_t row = ((size_t)bi * g.Hq + hk * g.G + gg) * g.Nq + t;
    const float inv = 1.f / l_run[rr];
#pragma unroll
    for (int c = 0; c < CPL; c++) {
      const float o = acc[rr][c] * inv;
      if constexpr (sizeof(T) == 4)
        O[row * D + lane + 32 * c] = o;
      else
        O[row * D + lane + 32 * c] = __float2bfloat16_rn(o);
    }
    if (lse && lane == 0) lse[row] = (m_run[rr] + log2f(l_run[rr])) * 0.6931471805599453f;
  }
}

template <typename T, int D>
cudaError_t launch_t(const Geo& g, const void* Q, const void* K, const void* V, const int32_t* idx, int dense,
                     void* O, float* lse, int* status, cudaStream_t st, const void* Qst, const void* PK,
                     const void* PV, int M) {
  const size_t smem = sizeof(float) * ((size_t)kRows * D + kKeys * (D + 1) + kKeys * D + kWarps * 16 * kKeys);
  auto kern = attn_simt_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int rows = g.G * min(g.b, g.Nq);
  dim3 grid(g.nqb, g.B * g.Hkv, ceil_div(rows, kRows));
  kern<<<grid, kWarps * 32, smem, st>>>(reinterpret_cast<const T*>(Q), reinterpret_cast<const T*>(K),
                                         reinterpret_cast<const T*>(V), idx, dense, reinterpret_cast<T*>(O), lse,
                                         status, g, reinterpret_cast<const T*>(Qst ? Qst : Q),
                                         reinterpret_cast<const T*>(PK), reinterpret_cast<const T*>(PV), M);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_simt(const Geo& g, const void* Q, const void* K, const void* V, const int32_t* idx,
                             int dense, void* O, float* lse, int* status, cudaStream_t st, const void* Qst,
                             const void* PK, const void* PV, int M) {
  if (g.dtype == PYR_BF16)
    return g.d == 128 ? launch_t<__nv_bfloat16, 128>(g, Q, K, V, idx, dense, O, lse, status, st, Qst, PK, PV, M)
                      : launch_t<__nv_bfloat16, 64>(g, Q, K, V, idx, dense, O, lse, status, st, Qst, PK, PV, M);
  return g.d == 128 ? launch_t<float, 128>(g, Q, K, V, idx, dense, O, lse, status, st, Qst, PK, PV, M)
                    : launch_t<float, 64>(g, Q, K, V, idx, dense, O, lse, status, st, Qst, PK, PV, M);
}

}  // namespace pyr
