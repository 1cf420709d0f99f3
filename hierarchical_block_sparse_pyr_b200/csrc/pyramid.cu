// Key pyramid: level 0 = mean key of each block, level l = mean of the keys
// under node (l, m) (PISA abstract: pooling builds the coarse-to-fine key
// hierarchy; PHBA A.1.2: centroids average the block's key rows in fp32).
//
// HBM-bound: K is read exactly once with 16-byte loads and the pyramid
// (about 2 nb nodes of 4 d bytes per head) is written once. Means are
// accumulated in fp32 and stored as bf16 (hi, lo) pairs; every level is
// computed from fp32 sums, so the pair rounding never compounds.
//   pyr_chunk_kernel  one CTA per chunk of CB consecutive key blocks of one
//                     (batch, kv head): one warp streams one block at a time
//                     (lanes split the row into 16-byte vectors, the rest of
//                     the warp splits rows), reduces with shuffles, and the
//                     CTA then pools the chunk's subtree in shared memory.
//   pyr_top_kernel    the levels above the chunk level, one CTA per
//                     (unit, 16-element slice of d), entirely in shared memory;
//                     launched as a programmatic dependent of the chunk kernel,
//                     so its CTAs are resident before the chunk kernel ends and
//                     wait (griddepcontrol.wait) for the chunk kernel's writes.
#include <algorithm>

#include "pyr_common.cuh"

namespace pyr {

namespace {

constexpr int kChunkThreads = 256;
constexpr int kTopSlice = 16;
constexpr int kTopThreads = 256;

__device__ __forceinline__ int64_t tokens_in(int j0, int j1, int b, int N) {
  int64_t t0 = (int64_t)j0 * b, t1 = (int64_t)j1 * b;
  if (t1 > N) t1 = N;
  return t1 > t0 ? t1 - t0 : 0;
}

template <typename T>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int E = 4;
  __device__ static void add(float* acc, uint4 v) {
    acc[0] += __uint_as_float(v.x);
    acc[1] += __uint_as_float(v.y);
    acc[2] += __uint_as_float(v.z);
    acc[3] += __uint_as_float(v.w);
  }
};
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int E = 8;
  __device__ static void add(float* acc, uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; k++) {
      acc[2 * k] += __uint_as_float(w[k] << 16);
      acc[2 * k + 1] += __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
};

__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// smem: two ping-pong level buffers of CB x D floats.
template <typename T, int D>
__global__ void __launch_bounds__(kChunkThreads) pyr_chunk_kernel(const T* __restrict__ K, __nv_bfloat16* __restrict__ pyr,
                                                                  Geo g, int CB, int t_levels) {
  constexpr int E = Vec<T>::E;
  constexpr int VPR = D / E;        // 16-byte vectors per key row
  constexpr int RLW = 32 / VPR;     // rows one warp instruction covers
  static_assert(VPR <= 32 && 32 % VPR == 0, "row must fit a warp");
  extern __shared__ float smem[];
  float* cur = smem;
  float* nxt = smem + (size_t)CB * D;

  const int unit = blockIdx.y;
  const int chunk = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = lane % VPR, rl = lane / VPR;
  const int j_begin = chunk * CB;
  const T* Ku = K + (size_t)unit * g.N * D;
  __nv_bfloat16* pu = pyr + (size_t)unit * g.P * 2 * D;

  // level 0: warp w handles blocks w, w + 8, ...
  for (int jl = warp; jl < CB; jl += kChunkThreads / 32) {
    const int j = j_begin + jl;
    float acc[E];
#pragma unroll
    for (int k = 0; k < E; k++) acc[k] = 0.f;
    int cnt = 0;
    if (j < g.nb) {
      const int t0 = j * g.b;
      const int t1 = min(t0 + g.b, g.N);
      cnt = t1 - t0;
      const uint4* base = reinterpret_cast<const uint4*>(Ku + (size_t)t0 * D) + c;
      int r = rl;
      // 8 independent loads in flight per lane
      for (; r + 7 * RLW < cnt; r += 8 * RLW) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; u++) v[u] = ldg_stream(base + (size_t)(r + u * RLW) * VPR);
#pragma unroll
        for (int u = 0; u < 8; u++) Vec<T>::add(acc, v[u]);
      }
      for (; r < cnt; r += RLW) Vec<T>::add(acc, ldg_stream(base + (size_t)r * VPR));
    }
#pragma unroll
    for (int off = VPR; off < 32; off <<= 1)
#pragma unroll
      for (int k = 0; k < E; k++) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], off);
    if (rl == 0) {
      float* dst = cur + (size_t)jl * D + c * E;
#pragma unroll
      for (int k = 0; k < E; k++) dst[k] = acc[k];
      if (j < g.nb) {
        const float inv = 1.f / (float)cnt;
        uint32_t wh[E / 2], wl[E / 2];
#pragma unroll
        for (int k = 0; k < E / 2; k++) {
          const float x0 = acc[2 * k] * inv, x1 = acc[2 * k + 1] * inv;
          const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
          const float2 hf = __bfloat1622float2(h);
          const __nv_bfloat162 lo = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
          wh[k] = *reinterpret_cast<const uint32_t*>(&h);
          wl[k] = *reinterpret_cast<const uint32_t*>(&lo);
        }
        __nv_bfloat16* row = pu + (size_t)j * 2 * D + c * E;
        if constexpr (E == 8) {
          *reinterpret_cast<uint4*>(row) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
          *reinterpret_cast<uint4*>(row + D) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
        } else {
          *reinterpret_cast<uint2*>(row) = make_uint2(wh[0], wh[1]);
          *reinterpret_cast<uint2*>(row + D) = make_uint2(wl[0], wl[1]);
        }
      }
    }
  }
  __syncthreads();

  // levels 1 .. t_levels inside the chunk
  int n_loc = CB;
  for (int l = 1; l <= t_levels; l++) {
    n_loc >>= 1;
    const int m0 = chunk * n_loc;
    for (int x = threadIdx.x; x < n_loc * D; x += kChunkThreads) {
      const int ml = x / D, e = x - ml * D;
      const float s = cur[(size_t)(2 * ml) * D + e] + cur[(size_t)(2 * ml + 1) * D + e];
      nxt[(size_t)ml * D + e] = s;
      const int m = m0 + ml;
      if (m < g.lvl_n[l]) {
        const int j0 = m << l;
        const int j1 = min((m + 1) << l, g.nb);
        split_store(pu + (size_t)(g.lvl_off[l] + m) * 2 * D, D, e, s / (float)tokens_in(j0, j1, g.b, g.N));
      }
    }
    __syncthreads();
    float* t = cur;
    cur = nxt;
    nxt = t;
  }
  // this CTA's nodes are written: the top-level kernel may start launching
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Levels t+1 .. L from level t, for one unit and a 16-wide slice of d.
__global__ void __launch_bounds__(kTopThreads) pyr_top_kernel(__nv_bfloat16* __restrict__ pyr, Geo g, int t) {
  extern __shared__ float sm[];
  const int unit = blockIdx.y;
  const int e0 = blockIdx.x * kTopSlice;
  __nv_bfloat16* pu = pyr + (size_t)unit * g.P * 2 * g.d;
  const int nt = g.lvl_n[t];
  float* cur = sm;
  float* nxt = sm + (size_t)nt * kTopSlice;
  // the chunk kernel's level-t nodes are complete and visible past this point
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // load level t as sums
  for (int x = threadIdx.x; x < nt * kTopSlice; x += kTopThreads) {
    const int m = x / kTopSlice, e = x - m * kTopSlice;
    const int j0 = m << t, j1 = min((m + 1) << t, g.nb);
    cur[x] = split_load(pu + (size_t)(g.lvl_off[t] + m) * 2 * g.d, g.d, e0 + e) * (float)tokens_in(j0, j1, g.b, g.N);
  }
  __syncthreads();
  int n_prev = nt;
  for (int l = t + 1; l <= g.L; l++) {
    const int n = g.lvl_n[l];
    for (int x = threadIdx.x; x < n * kTopSlice; x += kTopThreads) {
      const int m = x / kTopSlice, e = x - m * kTopSlice;
      float s = cur[(size_t)(2 * m) * kTopSlice + e];
      if (2 * m + 1 < n_prev) s += cur[(size_t)(2 * m + 1) * kTopSlice + e];
      nxt[x] = s;
      const int j0 = m << l, j1 = min((m + 1) << l, g.nb);
      split_store(pu + (size_t)(g.lvl_off[l] + m) * 2 * g.d, g.d, e0 + e, s / (float)tokens_in(j0, j1, g.b, g.N));
    }
    __syncthreads();
    float* tmp = cur;
    cur = nxt;
    nxt = tmp;
    n_prev = n;
  }
}

// Incremental update after the keys at positions >= from_pos (same shape)
// were rewritten, e.g. a decoded token written into the last slot: every
// node whose key range reaches such a position is recomputed, one CTA per
// (batch, kv head), thread e owning element e of d. Changed nodes are carried
// level to level as fp32 sums in shared memory (at most 32 per level);
// unchanged siblings are read back from their (hi, lo) pairs.
constexpr int kUpdMax = 32;

template <typename T>
__global__ void __launch_bounds__(128) pyr_update_kernel(const T* __restrict__ K, __nv_bfloat16* __restrict__ pyr,
                                                         Geo g, int j_first) {
  __shared__ float sums[2][kUpdMax][128];
  const int unit = blockIdx.x;
  const int e = threadIdx.x;
  if (e >= g.d) return;
  const T* Ku = K + (size_t)unit * g.N * g.d;
  __nv_bfloat16* pu = pyr + (size_t)unit * g.P * 2 * g.d;
  int cur = 0;
  // level 0: the changed blocks, straight from K
  for (int j = j_first; j < g.nb; j++) {
    const int t0 = j * g.b, t1 = min(t0 + g.b, g.N);
    float acc = 0.f;
    for (int t = t0; t < t1; t++) acc += to_f32(Ku[(size_t)t * g.d + e]);
    sums[cur][j - j_first][e] = acc;
    split_store(pu + (size_t)j * 2 * g.d, g.d, e, acc / (float)(t1 - t0));
  }
  for (int l = 1; l <= g.L; l++) {
    const int m0 = j_first >> l, c0 = j_first >> (l - 1);  // first changed node, first changed child
    for (int m = m0; m < g.lvl_n[l]; m++) {
      float s = 0.f;
      for (int ch = 2 * m; ch <= 2 * m + 1 && ch < g.lvl_n[l - 1]; ch++) {
        if (ch >= c0) {
          s += sums[cur][ch - c0][e];
        } else {
          const int cj0 = ch << (l - 1), cj1 = min((ch + 1) << (l - 1), g.nb);
          s += split_load(pu + (size_t)(g.lvl_off[l - 1] + ch) * 2 * g.d, g.d, e) *
               (float)tokens_in(cj0, cj1, g.b, g.N);
        }
      }
      sums[cur ^ 1][m - m0][e] = s;
      const int j0 = m << l, j1 = min((m + 1) << l, g.nb);
      split_store(pu + (size_t)(g.lvl_off[l] + m) * 2 * g.d, g.d, e, s / (float)tokens_in(j0, j1, g.b, g.N));
    }
    cur ^= 1;
  }
}

template <typename T, int D>
cudaError_t launch_chunks(const Geo& g, const void* K, __nv_bfloat16* pyr, int CB, int t, cudaStream_t st) {
  const size_t smem = (size_t)2 * CB * D * sizeof(float);
  auto kern = pyr_chunk_kernel<T, D>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(ceil_div(g.nb, CB), g.B * g.Hkv);
  kern<<<grid, kChunkThreads, smem, st>>>(reinterpret_cast<const T*>(K), pyr, g, CB, t);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pyramid_update(const Geo& g, const void* K, __nv_bfloat16* pyr, int from_pos, int* status,
                                  cudaStream_t st) {
  const int j_first = from_pos / g.b;
  if (g.nb - j_first > kUpdMax) return launch_pyramid(g, K, pyr, status, st);
  if (g.dtype == PYR_BF16)
    pyr_update_kernel<__nv_bfloat16><<<g.B * g.Hkv, 128, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(K), pyr, g,
                                                                   j_first);
  else
    pyr_update_kernel<float><<<g.B * g.Hkv, 128, 0, st>>>(reinterpret_cast<const float*>(K), pyr, g, j_first);
  return cudaGetLastError();
}

namespace {

// means[n][e] = hi + lo for every node n of every unit: a streaming pass, 8 elements per thread
__global__ void __launch_bounds__(256) pyr_means_kernel(const __nv_bfloat16* __restrict__ pyr,
                                                         float* __restrict__ means, int64_t nodes, int d) {
  const int64_t per_node = d / 8;  // 8-element groups per node
  const int64_t total = nodes * per_node;
  for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < total; x += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = x / per_node, e8 = (x - n * per_node) * 8;
    const uint4 hv = *reinterpret_cast<const uint4*>(pyr + (n * 2) * d + e8);
    const uint4 lv = *reinterpret_cast<const uint4*>(pyr + (n * 2 + 1) * d + e8);
    const uint32_t h[4] = {hv.x, hv.y, hv.z, hv.w}, lo[4] = {lv.x, lv.y, lv.z, lv.w};
    float out[8];
#pragma unroll
    for (int k = 0; k < 4; k++) {
      out[2 * k] = __uint_as_float(h[k] << 16) + __uint_as_float(lo[k] << 16);
      out[2 * k + 1] = __uint_as_float(h[k] & 0xFFFF0000u) + __uint_as_float(lo[k] & 0xFFFF0000u);
    }
    float* dst = means + n * d + e8;
    if ((reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
      reinterpret_cast<float4*>(dst)[0] = make_float4(out[0], out[1], out[2], out[3]);
      reinterpret_cast<float4*>(dst)[1] = make_float4(out[4], out[5], out[6], out[7]);
    } else {
#pragma unroll
      for (int k = 0; k < 8; k++) dst[k] = out[k];
    }
  }
}

}  // namespace

cudaError_t launch_pyramid_means(const Geo& g, const __nv_bfloat16* pyr, float* means, cudaStream_t st) {
  const int64_t nodes = (int64_t)g.B * g.Hkv * g.P;
  const int64_t groups = nodes * (g.d / 8);
  const int blocks = (int)std::min<int64_t>((groups + 255) / 256, 148 * 16);
  if (blocks <= 0) return cudaSuccess;
  pyr_means_kernel<<<blocks, 256, 0, st>>>(pyr, means, nodes, g.d);
  return cudaGetLastError();
}

cudaError_t launch_pyramid(const Geo& g, const void* K, __nv_bfloat16* pyr, int* status, cudaStream_t st) {
  (void)status;
  // Chunk: ~1024 key rows per CTA, and at most 1024 level-t nodes left for the top kernel.
  int CB = 1;
  while (CB * g.b < 1024) CB <<= 1;
  while ((int64_t)CB * 1024 < g.nb) CB <<= 1;
  int t = 0;
  while ((1 << t) < CB) t++;
  if (t > g.L) {  // the whole pyramid fits one chunk
    t = g.L;
    CB = 1 << t;
  }
  cudaError_t e;
  if (g.dtype == PYR_BF16)
    e = g.d == 128 ? launch_chunks<__nv_bfloat16, 128>(g, K, pyr, CB, t, st)
                   : launch_chunks<__nv_bfloat16, 64>(g, K, pyr, CB, t, st);
  else
    e = g.d == 128 ? launch_chunks<float, 128>(g, K, pyr, CB, t, st) : launch_chunks<float, 64>(g, K, pyr, CB, t, st);
  if (e != cudaSuccess || t >= g.L) return e;
  const size_t smem = (size_t)2 * g.lvl_n[t] * kTopSlice * sizeof(float);
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(pyr_top_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(g.d / kTopSlice, g.B * g.Hkv, 1);
  cfg.blockDim = dim3(kTopThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, pyr_top_kernel, pyr, g, t);
}

}  // namespace pyr
