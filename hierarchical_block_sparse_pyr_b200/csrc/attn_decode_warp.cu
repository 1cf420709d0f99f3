// Decode attention with one warp per 64-key tile: one new query row per head
// (Nq == 1) against a long key / value context (PHBA 3.1 / A.1.3 semantics:
// the routed blocks plus the current block, one softmax, output and
// log-sum-exp). HBM-bound: every routed block's keys and values are read once.
//
// A cluster of kCluster CTAs per (batch, kv head) splits the unit's 64-key
// tiles (routed blocks and the current block; a 128-key block is two tiles);
// within a CTA each of kWarps warps takes whole tiles and runs each by itself,
// with no block-wide barrier in the loop (the other warps' tiles overlap one
// warp's loads: two stages per warp with 32-key tiles measured slower, 0.146
// against 0.117 ms, the per-tile work not amortising over half the keys):
//   load   lane 0 issues a TMA load of the K tile (two 64 d x 64 key boxes,
//          128-byte swizzle) and a 1-D bulk copy of the V tile into the warp's
//          stage, completing on the warp's mbarrier;
//   score  lane l owns keys l and l + 32: for each 8-element chunk of d it reads
//          the chunk of both keys (the swizzle puts the chunks of 8 consecutive
//          keys in 8 different bank groups) and the same chunk of every query
//          row (one address for the whole warp: a broadcast), fp32 FMAs;
//   softmax per query row, max and sum over the warp by shuffles; the warp's
//          running max / sum / output are rescaled lazily per tile;
//   P.V    lane l owns d-elements 4l .. 4l + 3; probabilities go through the
//          warp's shared-memory row, values are read as one 256-byte row per key.
// At the end the warps' partial states merge in shared memory, and CTA 0 of
// the cluster merges the CTAs' through distributed shared memory. Every
// mbarrier wait is bounded; an abort still reaches both cluster barriers.
#include <cooperative_groups.h>

#include "pyr_common.cuh"
#include "tc_util.cuh"
#include "tile_list.cuh"

namespace pyr {

namespace {

using namespace tc;

constexpr int kWarps = 6;            // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kTileKeys = 64;        // keys per tile
constexpr int kStages = 1;           // stages per warp
constexpr int kCluster = 2;          // CTAs per (batch, kv head)
constexpr int kMaxGw = 8;            // query rows per kv head
constexpr int kMaxListW = 130;

struct WPlan {
  // per warp and stage: K tile [2 halves][64 keys][128 B] (16 KB), then V tile [64 keys][256 B] (16 KB)
  static constexpr int kStageBytes = 32768;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kWarps * kStages * kStageBytes;  // (end of the stages)
  static constexpr int kQ = kV;                            // [kMaxGw][128] fp32, scaled to log2 units
  static constexpr int kP = kQ + kMaxGw * 128 * 4;         // per warp: [kMaxGw][32] fp32 probabilities
  static constexpr int kML = kP + kWarps * kMaxGw * kTileKeys * 4;  // per warp: [kMaxGw] max, [kMaxGw] sum
  static constexpr int kCta = kML + kWarps * 2 * kMaxGw * 4;  // CTA partial: [kMaxGw] max, sum, 1/sum...
  static constexpr int kPo = kCta + 4 * kMaxGw * 4;        // CTA partial output [kMaxGw][128] fp32
  static constexpr int kW = kPo + kMaxGw * 128 * 4;        // merge weights [kMaxGw][kCluster]
  static constexpr int kList = kW + kMaxGw * kCluster * 4;  // the unit's block list
  static constexpr int kBar = kList + kMaxListW * 4 + 8;   // kWarps mbarriers (8-byte aligned)
  static constexpr int kBytes = kBar + kWarps * kStages * 8 + 16 + 1024;  // + alignment slack
};

__device__ __forceinline__ void bulk_load_w(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void cluster_sync_w() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_rank_w() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// bf16 pairs of a 16-byte chunk to 8 floats
__device__ __forceinline__ void cvt8(const uint4& v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; k++) {
    f[2 * k] = __uint_as_float(w[k] << 16);
    f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}

template <int GM>  // query rows per kv head, rounded up (G <= GM <= 8)
__global__ void __launch_bounds__(kThreads, 1)
    attn_decode_warp_kernel(const __grid_constant__ CUtensorMap tmK, const __nv_bfloat16* __restrict__ Q,
                            const __nv_bfloat16* __restrict__ V, const int32_t* __restrict__ idx, int dense,
                            __nv_bfloat16* __restrict__ O, float* __restrict__ lse, int* status, Geo g) {
  constexpr int D = 128;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_align<1024>(smem_raw);
  float* qs = reinterpret_cast<float*>(smem + WPlan::kQ);
  int* list = reinterpret_cast<int*>(smem + WPlan::kList);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + WPlan::kBar);
  __shared__ int tl_scratch[kTileListScratch];
  __shared__ int tl_entries[kTileListPitch];
  __shared__ int s_n;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank_w();
  const int CS = gridDim.x;
  const int unit = blockIdx.y;
  const int bi = unit / g.Hkv, hk = unit % g.Hkv;
  const int G = g.G;
  const int pos = g.q_offset;  // the query's position
  const int i = pos / g.b;     // its (current) block

  if (tid == 0) {
    s_abort = 0;
    for (int w = 0; w < kWarps * kStages; w++) mbar_init(bars + w, 1);
    fence_mbar_init();
  }
  // the unit's blocks: routed (ascending, validated), then the current block
  if (!dense) {
    // every thread of the CTA takes part (the helper has block-wide barriers); rank 0 alone reports
    // bad routes, the cluster's other CTAs see the same ones
    const int n = build_tile_list<1>(idx + (size_t)unit * g.nqb * g.topk, g.topk, i, 1, tl_scratch, tl_entries,
                                     rank == 0 ? status : nullptr);
    if (warp == 0) {
      for (int e = lane; e < n; e += 32) list[e] = tl_entries[e] >> 4;
      if (lane == 0) s_n = n;
    }
  } else if (tid == 0) {
    s_n = i + 1;
  }
  const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
  for (int x = tid; x < G * D; x += kThreads) {
    const int gg = x / D, e = x - gg * D;
    qs[x] = __bfloat162float(Q[((size_t)bi * g.Hq + hk * G + gg) * g.Nq * D + e]) * sl2;
  }
  __syncthreads();

  const int tpb = g.b / kTileKeys;  // tiles per block
  const int n_tiles = s_n * tpb;
  const int per = (n_tiles + CS - 1) / CS;
  const int t_begin = min(n_tiles, (int)rank * per), t_end = min(n_tiles, t_begin + per);
  unsigned char* stage0 = smem + WPlan::kK + warp * kStages * WPlan::kStageBytes;
  float* sP = reinterpret_cast<float*>(smem + WPlan::kP) + warp * kMaxGw * kTileKeys;
  uint64_t* wbar = bars + warp * kStages;
  const __nv_bfloat16* Vu = V + (size_t)unit * g.N * D;
  // this warp's tiles: t_begin + warp + kWarps * k, k = 0 .. n_mine - 1
  const int n_mine = t_begin + warp < t_end ? (t_end - 1 - (t_begin + warp)) / kWarps + 1 : 0;
  auto tile_of = [&](int k, int* j, int* key0, int* nk) {
    const int t = t_begin + warp + kWarps * k;
    *j = dense ? t / tpb : list[t / tpb];
    *key0 = *j * g.b + (t % tpb) * kTileKeys;
    *nk = max(0, min(kTileKeys, g.N - *key0));
  };
  auto issue = [&](int k) {  // lane 0: tile k into stage k % kStages
    int j, key0, nk;
    tile_of(k, &j, &key0, &nk);
    unsigned char* st = stage0 + (k % kStages) * WPlan::kStageBytes;
    uint64_t* bar = wbar + (k % kStages);
    // the K boxes always move 16 KB (keys past N arrive as zeros); V moves its nk rows
    mbar_expect_tx(bar, 16384 + (uint32_t)nk * D * 2);
    tma_load_3d(st, &tmK, 0, key0, unit, bar);
    tma_load_3d(st + 8192, &tmK, 64, key0, unit, bar);
    if (nk > 0) bulk_load_w(st + 16384, Vu + (size_t)key0 * D, (uint32_t)nk * D * 2, bar);
  };
  if (lane == 0)
    for (int k = 0; k < min(kStages, n_mine); k++) issue(k);

  float m_run[GM], l_run[GM], acc[GM][4];
#pragma unroll
  for (int r = 0; r < GM; r++) {
    m_run[r] = -INFINITY;
    l_run[r] = 0.f;
#pragma unroll
    for (int c = 0; c < 4; c++) acc[r][c] = 0.f;
  }
  bool ok = true;
  int k = 0;
  for (; k < n_mine; k++) {
    ok = mbar_wait(wbar + (k % kStages), (k / kStages) & 1, (volatile int*)&s_abort);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    int j, key0, nk;
    tile_of(k, &j, &key0, &nk);
    const unsigned char* sK = stage0 + (k % kStages) * WPlan::kStageBytes;
    const __nv_bfloat16* sV = reinterpret_cast<const __nv_bfloat16*>(sK + 16384);

    // ---- scores of keys lane and lane + 32 against every query row (log2 units)
    float s0[GM], s1[GM];
#pragma unroll
    for (int r = 0; r < GM; r++) s0[r] = s1[r] = 0.f;
#pragma unroll 2
    for (int cc = 0; cc < 16; cc++) {
      const int h = cc >> 3, c = cc & 7;
      const int off = h * 8192 + lane * 128 + ((c ^ (lane & 7)) << 4);
      float k0[8], k1[8];
      cvt8(*reinterpret_cast<const uint4*>(sK + off), k0);
      cvt8(*reinterpret_cast<const uint4*>(sK + off + 32 * 128), k1);
#pragma unroll
      for (int r = 0; r < GM; r++) {
        if (r < G) {
          const float4 qa = *reinterpret_cast<const float4*>(qs + r * D + cc * 8);
          const float4 qb = *reinterpret_cast<const float4*>(qs + r * D + cc * 8 + 4);
          float a = s0[r], b = s1[r];
          a = fmaf(qa.x, k0[0], a); b = fmaf(qa.x, k1[0], b);
          a = fmaf(qa.y, k0[1], a); b = fmaf(qa.y, k1[1], b);
          a = fmaf(qa.z, k0[2], a); b = fmaf(qa.z, k1[2], b);
          a = fmaf(qa.w, k0[3], a); b = fmaf(qa.w, k1[3], b);
          a = fmaf(qb.x, k0[4], a); b = fmaf(qb.x, k1[4], b);
          a = fmaf(qb.y, k0[5], a); b = fmaf(qb.y, k1[5], b);
          a = fmaf(qb.z, k0[6], a); b = fmaf(qb.z, k1[6], b);
          a = fmaf(qb.w, k0[7], a); b = fmaf(qb.w, k1[7], b);
          s0[r] = a;
          s1[r] = b;
        }
      }
    }
    // ---- online softmax per row: keys past N or past the query's position are masked
    const bool v0 = lane < nk && (j < i || key0 + lane <= pos);
    const bool v1 = lane + 32 < nk && (j < i || key0 + lane + 32 <= pos);
#pragma unroll
    for (int r = 0; r < GM; r++) {
      if (r < G) {
        const float a = v0 ? s0[r] : -INFINITY, b = v1 ? s1[r] : -INFINITY;
        float mx = fmaxf(a, b);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float m_new = fmaxf(m_run[r], mx);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float p0 = ex2(a - m_use), p1 = ex2(b - m_use);
        float sum = p0 + p1;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float corr = m_run[r] == -INFINITY ? 0.f : ex2(m_run[r] - m_use);
        l_run[r] = l_run[r] * corr + sum;
        m_run[r] = m_new;
#pragma unroll
        for (int c = 0; c < 4; c++) acc[r][c] *= corr;
        sP[r * kTileKeys + lane] = p0;
        sP[r * kTileKeys + lane + 32] = p1;
      }
    }
    __syncwarp();
    // ---- P.V: lane owns d-elements 4 lane .. 4 lane + 3
#pragma unroll 4
    for (int key = 0; key < nk; key++) {
      const uint2 w = *reinterpret_cast<const uint2*>(sV + (size_t)key * D + lane * 4);
      const float x0 = __uint_as_float(w.x << 16), x1 = __uint_as_float(w.x & 0xFFFF0000u);
      const float x2 = __uint_as_float(w.y << 16), x3 = __uint_as_float(w.y & 0xFFFF0000u);
#pragma unroll
      for (int r = 0; r < GM; r++) {
        if (r < G) {
          const float p = sP[r * kTileKeys + key];
          acc[r][0] = fmaf(p, x0, acc[r][0]);
          acc[r][1] = fmaf(p, x1, acc[r][1]);
          acc[r][2] = fmaf(p, x2, acc[r][2]);
          acc[r][3] = fmaf(p, x3, acc[r][3]);
        }
      }
    }
    __syncwarp();  // the stage and the probabilities are free again
    if (lane == 0 && k + kStages < n_mine) issue(k + kStages);
  }
  if (!ok) {
    // drain: this warp's copies still in flight (issued for tiles k .. k + kStages - 1)
    if (lane == 0) {
      volatile int no_abort = 0;
      for (int u = k; u < min(n_mine, k + kStages); u++) mbar_wait(wbar + (u % kStages), (u / kStages) & 1, &no_abort);
      report(status, PYR_ETIMEOUT);
    }
  }
  __syncthreads();  // every warp done with its stages: they hold the warps' partial outputs now

  // ---- merge the warps: per row the max, the rescaled sums and outputs
  float* wml = reinterpret_cast<float*>(smem + WPlan::kML);    // [warp][2][kMaxGw]
  float* wacc = reinterpret_cast<float*>(smem + WPlan::kK);    // [warp][kMaxGw][128], over the stages
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < GM; r++) {
      wml[(warp * 2) * kMaxGw + r] = m_run[r];
      wml[(warp * 2 + 1) * kMaxGw + r] = l_run[r];
    }
  }
#pragma unroll
  for (int r = 0; r < GM; r++)
    if (r < G)
      *reinterpret_cast<float4*>(wacc + ((size_t)warp * kMaxGw + r) * D + lane * 4) =
          make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
  __syncthreads();
  float* cml = reinterpret_cast<float*>(smem + WPlan::kCta);  // [0]: max, [kMaxGw]: sum
  float* po = reinterpret_cast<float*>(smem + WPlan::kPo);
  for (int x = tid; x < G * D; x += kThreads) {
    const int r = x / D, e = x - r * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; w++) M = fmaxf(M, wml[(w * 2) * kMaxGw + r]);
    float L = 0.f, a = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; w++) {
      const float mw = wml[(w * 2) * kMaxGw + r];
      const float sc = mw == -INFINITY ? 0.f : ex2(mw - M);
      L += sc * wml[(w * 2 + 1) * kMaxGw + r];
      a += sc * wacc[((size_t)w * kMaxGw + r) * D + e];
    }
    po[x] = a;
    if (e == 0) {
      cml[r] = M;
      cml[kMaxGw + r] = L;
    }
  }
  __syncthreads();
  cluster_sync_w();
  if (rank == 0) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    float* wts = reinterpret_cast<float*>(smem + WPlan::kW);  // [kMaxGw][kCluster], then 1/L in cml
    for (int r = tid; r < G; r += kThreads) {
      float mr[kCluster], lr[kCluster], M = -INFINITY;
#pragma unroll
      for (int c = 0; c < kCluster; c++) {
        mr[c] = c < CS ? *cluster.map_shared_rank(cml + r, c) : -INFINITY;
        lr[c] = c < CS ? *cluster.map_shared_rank(cml + kMaxGw + r, c) : 0.f;
        M = fmaxf(M, mr[c]);
      }
      float L = 0.f;
#pragma unroll
      for (int c = 0; c < kCluster; c++) {
        const float w = mr[c] == -INFINITY ? 0.f : ex2(mr[c] - M);
        wts[r * kCluster + c] = w;
        L += w * lr[c];
      }
      cml[2 * kMaxGw + r] = L > 0.f ? 1.f / L : 0.f;
      const size_t orow = ((size_t)bi * g.Hq + hk * G + r) * g.Nq;
      if (lse) lse[orow] = (M + log2f(L)) * 0.6931471805599453f;
    }
    __syncthreads();
    for (int x = tid; x < G * D; x += kThreads) {
      const int r = x / D;
      float a = 0.f;
#pragma unroll
      for (int c = 0; c < kCluster; c++)
        if (c < CS) a += wts[r * kCluster + c] * *cluster.map_shared_rank(po + x, c);
      const size_t orow = ((size_t)bi * g.Hq + hk * G + r) * g.Nq;
      O[orow * D + (x - r * D)] = __float2bfloat16_rn(a * cml[2 * kMaxGw + r]);
    }
  }
  cluster_sync_w();  // no CTA leaves while CTA 0 still reads its shared memory
}

template <int GM>
cudaError_t launch_gm(const Geo& g, const CUtensorMap& mk, const void* Q, const void* V, const int32_t* idx, int dense,
                      void* O, float* lse, int* status, cudaStream_t st) {
  auto kern = attn_decode_warp_kernel<GM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, WPlan::kBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kCluster, g.B * g.Hkv, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = WPlan::kBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mk, reinterpret_cast<const __nv_bfloat16*>(Q),
                            reinterpret_cast<const __nv_bfloat16*>(V), idx, dense,
                            reinterpret_cast<__nv_bfloat16*>(O), lse, status, g);
}

}  // namespace

bool attn_decode_warp_supported(const Geo& g) {
  return g.Nq == 1 && g.dtype == PYR_BF16 && g.d == 128 && (g.b == 64 || g.b == 128) && g.G <= kMaxGw &&
         g.topk + 1 <= kMaxListW;
}

cudaError_t launch_attn_decode_warp(const Geo& g, const void* Q, const void* K, const void* V, const int32_t* idx,
                                    int dense, void* O, float* lse, int* status, cudaStream_t st) {
  CUtensorMap mk;
  if (!make_tmap_bf16_3d(&mk, K, g.d, g.N, g.B * g.Hkv, kTileKeys)) return cudaErrorInvalidValue;
  if (g.G <= 4) return launch_gm<4>(g, mk, Q, V, idx, dense, O, lse, status, st);
  return launch_gm<8>(g, mk, Q, V, idx, dense, O, lse, status, st);
}

}  // namespace pyr
