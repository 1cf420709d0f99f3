// Decode attention: one new query row per head (Nq == 1) against a long key /
// value context (PHBA 3.1 / A.1.3 semantics: the routed blocks plus the
// current block, one softmax, output and log-sum-exp). HBM-bound: every routed
// block's keys and values are read once.
//
// One thread-block cluster of CS CTAs per (batch, kv head). The block list
// (routed blocks + the current block) is split evenly over the cluster; each
// CTA streams its whole blocks (contiguous b x d slabs of K and V) through a
// two-stage shared-memory ring with 1-D bulk async copies, and keeps an
// online softmax for the G query rows of the kv group (grouped-query attention
// shares the routes). The CTAs' partial (max, sum, output) states are merged by
// CTA 0 through distributed shared memory, so nothing is written to global
// memory except O and lse. All mbarrier waits are bounded; every CTA still
// reaches both cluster barriers, so an abort never strands the cluster.
#include <cooperative_groups.h>

#include "pyr_common.cuh"
#include "tc_util.cuh"
#include "tile_list.cuh"

namespace pyr {

namespace {

using namespace tc;

constexpr int kThreads = 128;
constexpr int kMaxCluster = 4;
constexpr int kMaxG = 32;
constexpr int kMaxList = 130;

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

template <int BK, int GM>  // keys per block; query rows per kv head (rounded up)
struct DecPlan {
  static constexpr int kStage = 2 * BK * 128 * 2;       // K and V of one block, bf16, d = 128
  static constexpr int kRing = 0;
  static constexpr int kQ = kRing + 2 * kStage;         // [GM][128] fp32
  static constexpr int kS = kQ + GM * 128 * 4;          // [GM][BK] fp32 scores / probabilities
  static constexpr int kO = kS + GM * BK * 4;           // [GM][128] fp32 partial output
  static constexpr int kM = kO + GM * 128 * 4;          // [GM] max, [GM] sum, [GM] correction
  static constexpr int kW = kM + 3 * GM * 4;            // [GM][kMaxCluster] merge weights, [GM] 1/sum
  static constexpr int kList = kW + GM * (kMaxCluster + 1) * 4;  // block list
  static constexpr int kBar = kList + kMaxList * 4 + 8;  // 2 mbarriers (8-byte aligned)
  static constexpr int kBytes = ((kBar + 16 + 127) / 128) * 128 + 128;
};

template <int BK, int GM>  // keys per block; query rows per kv head rounded up (G <= GM)
__global__ void __launch_bounds__(kThreads) attn_decode_kernel(const __nv_bfloat16* __restrict__ Q,
                                                               const __nv_bfloat16* __restrict__ K,
                                                               const __nv_bfloat16* __restrict__ V,
                                                               const int32_t* __restrict__ idx, int dense,
                                                               __nv_bfloat16* __restrict__ O, float* __restrict__ lse,
                                                               int* status, Geo g) {
  using PL = DecPlan<BK, GM>;
  constexpr int D = 128;
  constexpr int PARTS = kThreads / BK;  // threads per key in the score phase
  constexpr int DP = D / PARTS;         // d-elements per thread per key
  extern __shared__ unsigned char smem_raw[];
  // the base is aligned through an integer: measured faster here than the shared-space form
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~(uintptr_t)127);
  float* qs = reinterpret_cast<float*>(smem + PL::kQ);
  float* sc = reinterpret_cast<float*>(smem + PL::kS);
  float* po = reinterpret_cast<float*>(smem + PL::kO);
  float* m_run = reinterpret_cast<float*>(smem + PL::kM);
  float* l_run = m_run + GM;
  float* corr = l_run + GM;
  float* wts = reinterpret_cast<float*>(smem + PL::kW);  // [GM][kMaxCluster], then [GM] 1/sum
  int* list = reinterpret_cast<int*>(smem + PL::kList);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PL::kBar);
  __shared__ int s_n;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const int CS = gridDim.x;
  const int unit = blockIdx.y;
  const int bi = unit / g.Hkv, hk = unit % g.Hkv;
  const int G = g.G;
  const int pos = g.q_offset;  // the single query row's position
  const int i = pos / g.b;     // its (diagonal) block

  // ---- block list: routed blocks (ascending, validated), then the diagonal block; built by the
  // whole CTA (one warp loads and compacts the idx row)
  __shared__ int tl_scratch[kTileListScratch];
  __shared__ int tl_entries[kTileListPitch];
  if (tid == 0) {
    s_abort = 0;
    mbar_init(bars + 0, 1);
    mbar_init(bars + 1, 1);
    fence_mbar_init();
  }
  if (!dense) {
    // nqb == 1 in decode; the cluster's other CTAs see the same routes, so only rank 0 reports
    const int n = build_tile_list<1>(idx + (size_t)unit * g.nqb * g.topk, g.topk, i, 1, tl_scratch, tl_entries,
                                     rank == 0 ? status : nullptr);
    for (int e = tid; e < n; e += kThreads) list[e] = tl_entries[e] >> 4;
    if (tid == 0) s_n = n;
  } else if (tid == 0) {
    s_n = i + 1;
  }
  for (int x = tid; x < G * D; x += kThreads) {
    const int gg = x / D, e = x - gg * D;
    qs[x] = __bfloat162float(Q[((size_t)bi * g.Hq + hk * G + gg) * g.Nq * D + e]);
  }
  for (int x = tid; x < G; x += kThreads) {
    m_run[x] = -INFINITY;
    l_run[x] = 0.f;
  }
  for (int x = tid; x < G * D; x += kThreads) po[x] = 0.f;
  __syncthreads();

  const int n = s_n;
  const int per = (n + CS - 1) / CS;
  const int e_begin = min(n, (int)rank * per), e_end = min(n, e_begin + per);
  const int nmine = e_end - e_begin;
  auto block_of = [&](int e) { return dense ? e : list[e]; };
  const __nv_bfloat16* Ku = K + (size_t)unit * g.N * D;
  const __nv_bfloat16* Vu = V + (size_t)unit * g.N * D;
  unsigned char* ring = smem + PL::kRing;
  auto issue = [&](int k) {  // local block k into stage k & 1
    const int j = block_of(e_begin + k);
    const int nk = min(g.b, g.N - j * g.b);
    const uint32_t bytes = (uint32_t)nk * D * 2;
    unsigned char* st = ring + (k & 1) * PL::kStage;
    mbar_expect_tx(bars + (k & 1), 2 * bytes);
    bulk_load(st, Ku + (size_t)j * g.b * D, bytes, bars + (k & 1));
    bulk_load(st + BK * D * 2, Vu + (size_t)j * g.b * D, bytes, bars + (k & 1));
  };
  if (tid == 0) {
    if (nmine > 0) issue(0);
    if (nmine > 1) issue(1);
  }
  const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
  // P.V ownership: 4 consecutive d-elements (c4) for rows rg, rg + 4, ...
  const int c4 = tid & 31, rg = tid >> 5;
  float acc[GM / 4][4];
#pragma unroll
  for (int a = 0; a < GM / 4; a++)
#pragma unroll
    for (int b = 0; b < 4; b++) acc[a][b] = 0.f;

  bool ok = true;
  int k = 0;
  for (; k < nmine; k++) {
    if (tid == 0) ok = mbar_wait(bars + (k & 1), (k >> 1) & 1, (volatile int*)&s_abort);
    ok = __syncthreads_and(ok);
    if (!ok) break;
    const int j = block_of(e_begin + k);
    const int nk = min(g.b, g.N - j * g.b);
    const __nv_bfloat16* Ks = reinterpret_cast<const __nv_bfloat16*>(ring + (k & 1) * PL::kStage);
    const __nv_bfloat16* Vs = Ks + BK * D;
    // ---- scores: thread -> (key, part of d); parts combine through shuffles
    {
      const int key = tid / PARTS, pp = tid % PARTS;
      float dot[GM];
#pragma unroll
      for (int gg = 0; gg < GM; gg++) dot[gg] = 0.f;
      if (key < nk) {
        const __nv_bfloat16* kr = Ks + (size_t)key * D + pp * DP;
#pragma unroll
        for (int c = 0; c < DP / 8; c++) {
          const int cc = (c + key + pp * 4) % (DP / 8);  // stagger 16-byte chunks: no bank conflicts
          const uint4 w = *reinterpret_cast<const uint4*>(kr + cc * 8);
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
          float kf[8];
#pragma unroll
          for (int h = 0; h < 4; h++) {
            kf[2 * h] = __uint_as_float(ws[h] << 16);
            kf[2 * h + 1] = __uint_as_float(ws[h] & 0xFFFF0000u);
          }
          const int e = pp * DP + cc * 8;
#pragma unroll
          for (int gg = 0; gg < GM; gg++) {
            if (gg < G) {
              const float4 qa = *reinterpret_cast<const float4*>(qs + gg * D + e);
              const float4 qb = *reinterpret_cast<const float4*>(qs + gg * D + e + 4);
              float d0 = dot[gg];
              d0 = fmaf(qa.x, kf[0], d0);
              d0 = fmaf(qa.y, kf[1], d0);
              d0 = fmaf(qa.z, kf[2], d0);
              d0 = fmaf(qa.w, kf[3], d0);
              d0 = fmaf(qb.x, kf[4], d0);
              d0 = fmaf(qb.y, kf[5], d0);
              d0 = fmaf(qb.z, kf[6], d0);
              d0 = fmaf(qb.w, kf[7], d0);
              dot[gg] = d0;
            }
          }
        }
      }
#pragma unroll
      for (int off = 1; off < PARTS; off <<= 1)
#pragma unroll
        for (int gg = 0; gg < GM; gg++)
          if (gg < G) dot[gg] += __shfl_xor_sync(0xffffffffu, dot[gg], off);
      if (pp == 0) {
        const int kp = j * g.b + key;
        const bool valid = key < nk && (j < i || kp <= pos);
#pragma unroll
        for (int gg = 0; gg < GM; gg++)
          if (gg < G) sc[gg * BK + key] = valid ? dot[gg] * sl2 : -INFINITY;
      }
    }
    __syncthreads();
    // ---- per-row block max, running state update, probabilities (warp w: rows w, w + 4, ...)
    for (int gg = warp; gg < G; gg += 4) {
      float mx = -INFINITY;
      for (int c = lane; c < BK; c += 32) mx = fmaxf(mx, sc[gg * BK + c]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_old = m_run[gg];
      const float m_new = fmaxf(m_old, mx);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      float sum = 0.f;
      for (int c = lane; c < BK; c += 32) {
        const float pr = ex2(sc[gg * BK + c] - m_use);
        sc[gg * BK + c] = pr;
        sum += pr;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      if (lane == 0) {
        const float cr = m_old == -INFINITY ? 0.f : ex2(m_old - m_use);
        corr[gg] = cr;
        l_run[gg] = l_run[gg] * cr + sum;
        m_run[gg] = m_new;
      }
    }
    __syncthreads();
    // ---- O = O * corr + P V
#pragma unroll
    for (int a = 0; a < GM / 4; a++) {
      const int gg = rg + 4 * a;
      if (gg < G) {
        const float cr = corr[gg];
#pragma unroll
        for (int b = 0; b < 4; b++) acc[a][b] *= cr;
      }
    }
    for (int key = 0; key < nk; key++) {
      const uint2 w = *reinterpret_cast<const uint2*>(Vs + (size_t)key * D + c4 * 4);
      const float v0 = __uint_as_float(w.x << 16), v1 = __uint_as_float(w.x & 0xFFFF0000u);
      const float v2 = __uint_as_float(w.y << 16), v3 = __uint_as_float(w.y & 0xFFFF0000u);
#pragma unroll
      for (int a = 0; a < GM / 4; a++) {
        const int gg = rg + 4 * a;
        if (gg < G) {
          const float pr = sc[gg * BK + key];
          acc[a][0] = fmaf(pr, v0, acc[a][0]);
          acc[a][1] = fmaf(pr, v1, acc[a][1]);
          acc[a][2] = fmaf(pr, v2, acc[a][2]);
          acc[a][3] = fmaf(pr, v3, acc[a][3]);
        }
      }
    }
    __syncthreads();  // the stage and the scores are free again
    if (tid == 0 && k + 2 < nmine) issue(k + 2);
  }
  // drain this CTA's copies after an abort, before the cluster can finish
  if (!ok && tid == 0) {
    volatile int no_abort = 0;
    for (int u = k; u < min(nmine, k + 2); u++) mbar_wait(bars + (u & 1), (u >> 1) & 1, &no_abort);
  }
  // ---- partial state to shared memory, merged by CTA 0 through distributed shared memory
#pragma unroll
  for (int a = 0; a < GM / 4; a++) {
    const int gg = rg + 4 * a;
    if (gg < G) *reinterpret_cast<float4*>(po + gg * D + c4 * 4) = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
  }
  if (!ok && tid == 0) report(status, PYR_ETIMEOUT);
  __syncthreads();
  cluster_sync();
  if (rank == 0) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    // per row: the global max, the weights 2^(m_r - M) of the CTAs' partial states, 1 / sum
    for (int gg = tid; gg < G; gg += kThreads) {
      float mr[kMaxCluster], lr[kMaxCluster], M = -INFINITY;
#pragma unroll
      for (int r = 0; r < kMaxCluster; r++) {
        mr[r] = r < CS ? *cluster.map_shared_rank(m_run + gg, r) : -INFINITY;
        lr[r] = r < CS ? *cluster.map_shared_rank(l_run + gg, r) : 0.f;
      }
#pragma unroll
      for (int r = 0; r < kMaxCluster; r++) M = fmaxf(M, mr[r]);
      float L = 0.f;
#pragma unroll
      for (int r = 0; r < kMaxCluster; r++) {
        const float w = mr[r] == -INFINITY ? 0.f : ex2(mr[r] - M);
        wts[gg * kMaxCluster + r] = w;
        L += w * lr[r];
      }
      wts[GM * kMaxCluster + gg] = L > 0.f ? 1.f / L : 0.f;
      const size_t orow = ((size_t)bi * g.Hq + hk * G + gg) * g.Nq;
      if (lse) lse[orow] = (M + log2f(L)) * 0.6931471805599453f;
    }
    __syncthreads();
    for (int x = tid; x < G * D; x += kThreads) {
      const int gg = x / D;
      float part[kMaxCluster];
#pragma unroll
      for (int r = 0; r < kMaxCluster; r++) part[r] = r < CS ? *cluster.map_shared_rank(po + x, r) : 0.f;
      float a = 0.f;
#pragma unroll
      for (int r = 0; r < kMaxCluster; r++) a += r < CS ? wts[gg * kMaxCluster + r] * part[r] : 0.f;
      const size_t orow = ((size_t)bi * g.Hq + hk * G + gg) * g.Nq;
      O[orow * D + (x - gg * D)] = __float2bfloat16_rn(a * wts[GM * kMaxCluster + gg]);
    }
  }
  cluster_sync();  // no CTA leaves while CTA 0 still reads its shared memory
}

template <int BK, int GM>
cudaError_t launch_bk(const Geo& g, const void* Q, const void* K, const void* V, const int32_t* idx, int dense,
                      void* O, float* lse, int* status, cudaStream_t st) {
  auto kern = attn_decode_kernel<BK, GM>;
  const int bytes = DecPlan<BK, GM>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  const int nblk = dense ? g.i0 + 1 : min(g.topk, g.i0) + 1;
  const int CS = max(1, min(kMaxCluster, nblk));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS, g.B * g.Hkv, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, reinterpret_cast<const __nv_bfloat16*>(Q),
                            reinterpret_cast<const __nv_bfloat16*>(K), reinterpret_cast<const __nv_bfloat16*>(V), idx,
                            dense, reinterpret_cast<__nv_bfloat16*>(O), lse, status, g);
}

template <int BK>
cudaError_t launch_g(const Geo& g, const void* Q, const void* K, const void* V, const int32_t* idx, int dense,
                     void* O, float* lse, int* status, cudaStream_t st) {
  if (g.G <= 4) return launch_bk<BK, 4>(g, Q, K, V, idx, dense, O, lse, status, st);
  if (g.G <= 8) return launch_bk<BK, 8>(g, Q, K, V, idx, dense, O, lse, status, st);
  if (g.G <= 16) return launch_bk<BK, 16>(g, Q, K, V, idx, dense, O, lse, status, st);
  return launch_bk<BK, 32>(g, Q, K, V, idx, dense, O, lse, status, st);
}

}  // namespace

bool attn_decode_supported(const Geo& g) {
  return g.Nq == 1 && g.dtype == PYR_BF16 && g.d == 128 && (g.b == 64 || g.b == 128) && g.G <= kMaxG &&
         g.topk + 1 <= kMaxList;
}

cudaError_t launch_attn_decode(const Geo& g, const void* Q, const void* K, const void* V, const int32_t* idx,
                               int dense, void* O, float* lse, int* status, cudaStream_t st) {
  if (g.b == 64) return launch_g<64>(g, Q, K, V, idx, dense, O, lse, status, st);
  return launch_g<128>(g, Q, K, V, idx, dense, O, lse, status, st);
}

}  // namespace pyr
