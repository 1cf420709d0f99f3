// Backward pass of causal block-sparse attention (PHBA summary, A.1.2
// "Routing metadata kernels" and A.1.4 "Sparse backward kernel").
//
// Route inversion: the query-centric routes idx[u][qb][*] are re-expressed per
// key block, as A.1.2 describes: count the assignments of every key block,
// prefix-sum the counts into contiguous ranges (offset), scatter the query
// block ids into them (rho). The scatter claims slots with atomics, so a last
// pass sorts each range: the output does not depend on thread timing.
//   route_count_kernel   one thread per idx row: offset[u][j] += 1 per route
//   route_scan_kernel    one CTA per unit: in-place inclusive scan, so that
//                        offset[u][j] is the end of j's range; offset[u][nb]
//                        = total; rho's unused tail = -1
//   route_scatter_kernel one thread per idx row: pos = --offset[u][j]; after
//                        it offset[u][j] is the start of j's range
//   route_sort_kernel    one CTA per (key block, unit): rank by counting, or a
//                        bitmap of the range's query blocks for long ranges
//
// Gradients (the SIMT path: fp32 on the CUDA cores, every dtype and shape the
// library takes). P is recomputed from the saved log-sum-exp as A.1.4 states;
// D_t = dO_t . O_t is computed once per row into the caller's workspace.
//   bwd_delta_kernel  one warp per query row: D_t (bf16 rows of 128: the
//                     vectorised bwd_delta_bf16_d128_kernel)
//   bwd_dq_kernel     one warp per query row: walks the row's routed blocks
//                     and its own block, dQ_t = sum_k dS_tk k_k / sqrt(d)
//   bwd_dkdv_kernel   one warp per key: walks the query blocks that route to
//                     the key's block (the block-major ranges) and the key's
//                     own block, dK_k = sum_t dS_tk q_t / sqrt(d),
//                     dV_k = sum_t P_tk dO_t over the G heads of the group
// No atomics touch the gradients: every output element has one owner.
#include <algorithm>

#include "pyr_common.cuh"

namespace pyr {

namespace {

constexpr int kEntryThreads = 256;
constexpr int kScanThreads = 1024;
constexpr int kWarpsPerCta = 4;

// Walks the routes of one idx row of query block i in slot order with the rule
// the forward kernels apply: an entry is used only if it is >= 0, < i and
// greater than the last used entry; any other non-negative entry is skipped
// and reported. f(j) is called for every used entry.
template <typename F>
__device__ __forceinline__ void for_routes(const int32_t* row, int topk, int i, int* status, F f) {
  int prev = -1;
  for (int k = 0; k < topk; k++) {
    const int j = row[k];
    if (j < 0) continue;
    if (j >= i || j <= prev) {
      if (status) report(status, PYR_EBADIDX);
      continue;
    }
    prev = j;
    f(j);
  }
}

// one thread per idx row
__global__ void route_count_kernel(const int32_t* __restrict__ idx, int32_t* offset, int* status, Geo g) {
  const int64_t n = (int64_t)g.B * g.Hkv * g.nqb;
  for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < n; r += (int64_t)gridDim.x * blockDim.x) {
    const int qb = (int)(r % g.nqb), u = (int)(r / g.nqb);
    int32_t* off = offset + (int64_t)u * (g.nb + 1);
    for_routes(idx + r * g.topk, g.topk, g.i0 + qb, status, [&](int j) { atomicAdd(off + j, 1); });
  }
}

__global__ void __launch_bounds__(kScanThreads) route_scan_kernel(int32_t* offset, int32_t* rho, Geo g) {
  __shared__ int warp_sums[kScanThreads / 32];
  const int u = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  int32_t* off = offset + (int64_t)u * (g.nb + 1);
  const int per = (g.nb + kScanThreads - 1) / kScanThreads;
  const int j0 = min(t * per, g.nb), j1 = min(j0 + per, g.nb);
  int local = 0;
  for (int j = j0; j < j1; j++) local += off[j];
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  int run = incl - local + (warp > 0 ? warp_sums[warp - 1] : 0);
  for (int j = j0; j < j1; j++) {
    run += off[j];
    off[j] = run;
  }
  const int total = warp_sums[kScanThreads / 32 - 1];
  if (t == 0) off[g.nb] = total;
  int32_t* r = rho + (int64_t)u * g.nqb * g.topk;
  for (int x = total + t; x < g.nqb * g.topk; x += kScanThreads) r[x] = -1;
}

__global__ void route_scatter_kernel(const int32_t* __restrict__ idx, int32_t* offset, int32_t* rho, Geo g) {
  const int64_t n = (int64_t)g.B * g.Hkv * g.nqb;
  for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < n; r += (int64_t)gridDim.x * blockDim.x) {
    const int qb = (int)(r % g.nqb), u = (int)(r / g.nqb);
    int32_t* off = offset + (int64_t)u * (g.nb + 1);
    int32_t* dst = rho + (int64_t)u * g.nqb * g.topk;
    for_routes(idx + r * g.topk, g.topk, g.i0 + qb, nullptr, [&](int j) { dst[atomicSub(off + j, 1) - 1] = qb; });
  }
}

// One CTA per (key block j, unit) puts j's range in ascending order. The
// entries of a range are distinct query blocks (a row routes a block at most
// once). Up to kSortThreads entries: each thread ranks its entry by counting
// the smaller ones. Longer ranges: a bitmap over the query blocks, then each
// thread emits the set bits of its run of words after a block-wide prefix
// count. Either way the work is linear in the range (plus nqb / 32 words).
constexpr int kSortThreads = 128;

__global__ void __launch_bounds__(kSortThreads) route_sort_kernel(const int32_t* __restrict__ offset, int32_t* rho,
                                                                 Geo g) {
  extern __shared__ uint32_t bits[];  // ceil(nqb / 32) words
  __shared__ int32_t vals[kSortThreads];
  __shared__ int warp_tot[kSortThreads / 32];
  const int u = blockIdx.y, j = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int32_t* off = offset + (int64_t)u * (g.nb + 1);
  int32_t* r = rho + (int64_t)u * g.nqb * g.topk;
  const int a = off[j], n = off[j + 1] - a;
  if (n <= 1) return;
  if (n <= kSortThreads) {
    const int v = t < n ? r[a + t] : 0;
    vals[t] = v;
    __syncthreads();  // every entry is read before any is written
    if (t < n) {
      int rank = 0;
      for (int k = 0; k < n; k++) rank += vals[k] < v;
      r[a + rank] = v;
    }
    return;
  }
  const int words = (g.nqb + 31) >> 5;
  for (int w = t; w < words; w += kSortThreads) bits[w] = 0;
  __syncthreads();
  for (int k = t; k < n; k += kSortThreads) {
    const int v = r[a + k];
    atomicOr(&bits[v >> 5], 1u << (v & 31));
  }
  __syncthreads();
  const int per = (words + kSortThreads - 1) / kSortThreads;
  const int w0 = min(words, t * per), w1 = min(words, w0 + per);
  int cnt = 0;
  for (int w = w0; w < w1; w++) cnt += __popc(bits[w]);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int pos = a + incl - cnt;
  for (int w = 0; w < warp; w++) pos += warp_tot[w];
  for (int w = w0; w < w1; w++) {
    uint32_t m = bits[w];
    while (m) {
      r[pos++] = (w << 5) + __ffs(m) - 1;
      m &= m - 1;
    }
  }
}

// ---------------------------------------------------------------- gradients

template <typename T, int DPL>
__device__ __forceinline__ void load_row(const T* p, int lane, float* v) {
#pragma unroll
  for (int c = 0; c < DPL; c++) v[c] = to_f32(p[lane * DPL + c]);
}

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

template <typename T, int DPL>
__device__ __forceinline__ void store_row(T* p, int lane, const float* v, float scale) {
#pragma unroll
  for (int c = 0; c < DPL; c++) p[lane * DPL + c] = from_f32<T>(v[c] * scale);
}

__device__ __forceinline__ void warp_sum2(float* a, float* b) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    *a += __shfl_xor_sync(0xffffffffu, *a, o);
    *b += __shfl_xor_sync(0xffffffffu, *b, o);
  }
}

template <typename T, int DPL>
__global__ void __launch_bounds__(kWarpsPerCta * 32) bwd_delta_kernel(const T* __restrict__ O, const T* __restrict__ dO,
                                                                   float* __restrict__ delta, Geo g) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (row >= (int64_t)g.B * g.Hq * g.Nq) return;
  float o[DPL], d[DPL];
  load_row<T, DPL>(O + row * g.d, lane, o);
  load_row<T, DPL>(dO + row * g.d, lane, d);
  float a = 0.f, z = 0.f;
#pragma unroll
  for (int c = 0; c < DPL; c++) a += o[c] * d[c];
  warp_sum2(&a, &z);
  if (lane == 0) delta[row] = a;
}

// D_t for bf16 rows of 128: 16 lanes per row (16 bytes of O and of dO each),
// and each warp has 8 rows (4 per half-warp) of loads in flight per iteration.
__device__ __forceinline__ float dot_bf16x8(uint4 a, uint4 b) {
  const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&b);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 4; i++) {
    const float2 u = __bfloat1622float2(x[i]), v = __bfloat1622float2(y[i]);
    s = fmaf(u.x, v.x, s);
    s = fmaf(u.y, v.y, s);
  }
  return s;
}

__global__ void __launch_bounds__(256) bwd_delta_bf16_d128_kernel(const __nv_bfloat16* __restrict__ O,
                                                                  const __nv_bfloat16* __restrict__ dO,
                                                                  float* __restrict__ delta, int64_t rows) {
  const int lane = threadIdx.x & 31, half = lane >> 4, sub = lane & 15;
  const int64_t warp_id = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t r0 = warp_id * 8; r0 < rows; r0 += nwarps * 8) {  // the same trip count for the whole warp
    uint4 a[4], b[4];
#pragma unroll
    for (int k = 0; k < 4; k++) {
      const int64_t r = r0 + half * 4 + k;
      a[k] = b[k] = make_uint4(0u, 0u, 0u, 0u);
      if (r < rows) {
        a[k] = __ldg(reinterpret_cast<const uint4*>(O + r * 128) + sub);
        b[k] = __ldg(reinterpret_cast<const uint4*>(dO + r * 128) + sub);
      }
    }
    float s[4];
#pragma unroll
    for (int k = 0; k < 4; k++) s[k] = dot_bf16x8(a[k], b[k]);
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1)
#pragma unroll
      for (int k = 0; k < 4; k++) s[k] += __shfl_xor_sync(0xffffffffu, s[k], o);
    const int64_t r = r0 + half * 4 + sub;
    if (sub < 4 && r < rows) delta[r] = sub == 0 ? s[0] : sub == 1 ? s[1] : sub == 2 ? s[2] : s[3];
  }
}

template <typename T, int DPL>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
    bwd_dq_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V, const T* __restrict__ dO,
                  const float* __restrict__ lse, const float* __restrict__ delta, const int32_t* __restrict__ idx,
                  T* __restrict__ dQ, Geo g) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (row >= (int64_t)g.B * g.Hq * g.Nq) return;
  const int t = (int)(row % g.Nq);
  const int64_t bh = row / g.Nq;
  const int bi = (int)(bh / g.Hq), hq = (int)(bh % g.Hq), hk = hq / g.G;
  const int unit = bi * g.Hkv + hk;
  const int p = g.q_offset + t, i = p / g.b, qb = i - g.i0;
  const float sl2 = rsqrtf((float)g.d) * 1.4426950408889634f;
  const float lse2 = lse[row] * 1.4426950408889634f, D = delta[row];
  float q[DPL], d[DPL], acc[DPL];
  load_row<T, DPL>(Q + row * g.d, lane, q);
  load_row<T, DPL>(dO + row * g.d, lane, d);
#pragma unroll
  for (int c = 0; c < DPL; c++) acc[c] = 0.f;
  const T* Ku = K + (int64_t)unit * g.N * g.d;
  const T* Vu = V + (int64_t)unit * g.N * g.d;
  auto visit = [&](int x) {
    float k[DPL], v[DPL];
    load_row<T, DPL>(Ku + (int64_t)x * g.d, lane, k);
    load_row<T, DPL>(Vu + (int64_t)x * g.d, lane, v);
    float s = 0.f, dp = 0.f;
#pragma unroll
    for (int c = 0; c < DPL; c++) {
      s += q[c] * k[c];
      dp += d[c] * v[c];
    }
    warp_sum2(&s, &dp);
    const float P = exp2f(s * sl2 - lse2);
    const float dS = P * (dp - D);
#pragma unroll
    for (int c = 0; c < DPL; c++) acc[c] += dS * k[c];
  };
  for_routes(idx + ((int64_t)unit * g.nqb + qb) * g.topk, g.topk, i, nullptr, [&](int j) {
    const int x1 = min((j + 1) * g.b, g.N);
    for (int x = j * g.b; x < x1; x++) visit(x);
  });
  for (int x = i * g.b; x <= p; x++) visit(x);
  store_row<T, DPL>(dQ + row * g.d, lane, acc, rsqrtf((float)g.d));
}

template <typename T, int DPL>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
    bwd_dkdv_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
                    const T* __restrict__ dO, const float* __restrict__ lse, const float* __restrict__ delta,
                    const int32_t* __restrict__ offset, const int32_t* __restrict__ rho, T* __restrict__ dK,
                    T* __restrict__ dV, Geo g) {
  const int lane = threadIdx.x & 31;
  const int64_t key = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  if (key >= (int64_t)g.B * g.Hkv * g.N) return;
  const int unit = (int)(key / g.N), x = (int)(key % g.N), j = x / g.b;
  const int bi = unit / g.Hkv, hk = unit % g.Hkv;
  const float sl2 = rsqrtf((float)g.d) * 1.4426950408889634f;
  float k[DPL], v[DPL], gk[DPL], gv[DPL];
  load_row<T, DPL>(K + key * g.d, lane, k);
  load_row<T, DPL>(V + key * g.d, lane, v);
#pragma unroll
  for (int c = 0; c < DPL; c++) gk[c] = gv[c] = 0.f;
  // every row of query block qb, in every head of the group; the key's own block only from
  // the key's position on (causal)
  auto rows_of = [&](int qb, int p_from) {
    const int i = g.i0 + qb;
    const int pa = max(max(i * g.b, g.q_offset), p_from), pz = min((i + 1) * g.b, g.q_offset + g.Nq);
    for (int gg = 0; gg < g.G; gg++) {
      const int64_t row0 = ((int64_t)bi * g.Hq + hk * g.G + gg) * g.Nq - g.q_offset;
      for (int p = pa; p < pz; p++) {
        const int64_t row = row0 + p;
        float q[DPL], d[DPL];
        load_row<T, DPL>(Q + row * g.d, lane, q);
        load_row<T, DPL>(dO + row * g.d, lane, d);
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int c = 0; c < DPL; c++) {
          s += q[c] * k[c];
          dp += d[c] * v[c];
        }
        warp_sum2(&s, &dp);
        const float P = exp2f(s * sl2 - lse[row] * 1.4426950408889634f);
        const float dS = P * (dp - delta[row]);
#pragma unroll
        for (int c = 0; c < DPL; c++) {
          gk[c] += dS * q[c];
          gv[c] += P * d[c];
        }
      }
    }
  };
  const int32_t* off = offset + (int64_t)unit * (g.nb + 1);
  const int32_t* r = rho + (int64_t)unit * g.nqb * g.topk;
  for (int e = off[j]; e < off[j + 1]; e++) rows_of(r[e], 0);
  if (j >= g.i0 && j < g.i0 + g.nqb) rows_of(j - g.i0, x);
  store_row<T, DPL>(dK + key * g.d, lane, gk, rsqrtf((float)g.d));
  store_row<T, DPL>(dV + key * g.d, lane, gv, 1.f);
}

inline int grid_for(int64_t n, int threads) {
  const int64_t b = (n + threads - 1) / threads;
  return (int)(b < 148 * 16 ? (b > 0 ? b : 1) : 148 * 16);
}

template <typename T, int DPL>
cudaError_t launch_grads(const Geo& g, const void* Q, const void* K, const void* V, const void* O, const float* lse,
                         const void* dO, const int32_t* idx, const int32_t* offset, const int32_t* rho, float* delta,
                         void* dQ, void* dK, void* dV, int parts, cudaStream_t st) {
  const int64_t rows = (int64_t)g.B * g.Hq * g.Nq, keys = (int64_t)g.B * g.Hkv * g.N;
  const unsigned rgrid = (unsigned)((rows + kWarpsPerCta - 1) / kWarpsPerCta);
  const unsigned kgrid = (unsigned)((keys + kWarpsPerCta - 1) / kWarpsPerCta);
  const T* q = static_cast<const T*>(Q);
  const T* k = static_cast<const T*>(K);
  const T* v = static_cast<const T*>(V);
  const T* d = static_cast<const T*>(dO);
  if ((parts & kBwdDelta) && sizeof(T) == 2 && g.d == 128) {
    const unsigned grid = (unsigned)std::min<int64_t>((rows + 63) / 64, 148 * 16);  // 8 warps x 8 rows per CTA pass
    bwd_delta_bf16_d128_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(O),
                                                     reinterpret_cast<const __nv_bfloat16*>(dO), delta, rows);
  } else if (parts & kBwdDelta) {
    bwd_delta_kernel<T, DPL><<<rgrid, kWarpsPerCta * 32, 0, st>>>(static_cast<const T*>(O), d, delta, g);
  }
  if (parts & kBwdDq)
    bwd_dq_kernel<T, DPL><<<rgrid, kWarpsPerCta * 32, 0, st>>>(q, k, v, d, lse, delta, idx, static_cast<T*>(dQ), g);
  if (parts & kBwdDkdv)
    bwd_dkdv_kernel<T, DPL><<<kgrid, kWarpsPerCta * 32, 0, st>>>(q, k, v, d, lse, delta, offset, rho,
                                                                 static_cast<T*>(dK), static_cast<T*>(dV), g);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route_invert(const Geo& g, const int32_t* idx, int32_t* offset, int32_t* rho, int* status,
                                cudaStream_t st) {
  const int64_t rows = (int64_t)g.B * g.Hkv * g.nqb;
  cudaError_t e = cudaMemsetAsync(offset, 0, sizeof(int32_t) * (size_t)g.B * g.Hkv * (g.nb + 1), st);
  if (e != cudaSuccess) return e;
  route_count_kernel<<<grid_for(rows, kEntryThreads), kEntryThreads, 0, st>>>(idx, offset, status, g);
  route_scan_kernel<<<g.B * g.Hkv, kScanThreads, 0, st>>>(offset, rho, g);
  route_scatter_kernel<<<grid_for(rows, kEntryThreads), kEntryThreads, 0, st>>>(idx, offset, rho, g);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t bitmap = sizeof(uint32_t) * (size_t)((g.nqb + 31) / 32);
  if (bitmap > 48 * 1024) {
    e = cudaFuncSetAttribute(route_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bitmap);
    if (e != cudaSuccess) return e;
  }
  route_sort_kernel<<<dim3(g.nb, g.B * g.Hkv), kSortThreads, bitmap, st>>>(offset, rho, g);
  return cudaGetLastError();
}

cudaError_t launch_backward_simt(const Geo& g, const void* Q, const void* K, const void* V, const void* O,
                                 const float* lse, const void* dO, const int32_t* idx, const int32_t* offset,
                                 const int32_t* rho, float* delta, void* dQ, void* dK, void* dV, int parts,
                                 cudaStream_t st) {
  if (g.dtype == PYR_F32) {
    if (g.d == 64)
      return launch_grads<float, 2>(g, Q, K, V, O, lse, dO, idx, offset, rho, delta, dQ, dK, dV, parts, st);
    return launch_grads<float, 4>(g, Q, K, V, O, lse, dO, idx, offset, rho, delta, dQ, dK, dV, parts, st);
  }
  if (g.d == 64)
    return launch_grads<__nv_bfloat16, 2>(g, Q, K, V, O, lse, dO, idx, offset, rho, delta, dQ, dK, dV, parts, st);
  return launch_grads<__nv_bfloat16, 4>(g, Q, K, V, O, lse, dO, idx, offset, rho, delta, dQ, dK, dV, parts, st);
}

}  // namespace pyr
