// Decode attention with one warp per 64-key tile: one new query row per head
// (Nq == 1) against a long key / value context (PHBA 3.1 / A.1.3 semantics:
// the routed blocks plus the current block, one softmax, output and
// log-sum-exp). HBM-bound: every routed block's keys and values are read once.
//
// One CTA per (batch, kv head) takes the unit's 64-key tiles (routed blocks
// and the current block; a 128-key block is two tiles); each of kWarps warps
// takes whole tiles and runs each by itself, with no block-wide barrier in
// the loop (the other warps' tiles overlap one warp's loads):
//   load   lane 0 issues TMA loads of the K and V tiles (two 64 d x 64 key
//          boxes each, 128-byte swizzle) into the warp's stage, completing on
//          the warp's mbarrier;
//   score  S^T = K q^T per tile on the warp's tensor-core MMAs (m16n8k16, bf16
//          operands, fp32 accumulation): keys are the M dimension (four
//          16-key row tiles), the G <= 8 query rows of the kv group the N
//          dimension, d the K dimension; K fragments come from the swizzled
//          tile by ldmatrix, q^T fragments stay in registers for the whole
//          unit (q is used exactly, as bf16);
//   softmax per query row over the tile's keys: each lane holds 8 keys of two
//          rows, max and the rescaling by shuffles across the 8 lanes that
//          share a row; exponentials on the MUFU unit;
//   P.V    O^T += V^T P^T: V^T fragments by transposing ldmatrix from the
//          swizzled V tile, P^T fragments by an in-register 8x8 transpose
//          (movmatrix) of the bf16 probabilities.
// At the end the warps' partial states (row max, sum, O) merge in shared
// memory. Every mbarrier wait is bounded; a warp that times out drains its
// copies in flight and the CTA reports PYR_ETIMEOUT.
// Why warp MMAs in an HBM-bound kernel: with CUDA-core FMAs (the same loop as
// packed fp32 FMAs) the tile's G x 64 x 128 products and the matching P.V cost
// about 2,000 instructions per warp, and with six warps per SM the issue rate,
// not HBM, set the time (0.104 ms on the 128K GQA decode workload, 40% of
// HBM); as m16n8k16 MMAs they are 64 MMAs and 64 ldmatrix per tile (0.055 ms,
// 76%). The tile is a warp-sized product that one warp owns end to end; the
// CTA-wide tcgen05 path (single-thread issue, accumulators in TMEM lanes that
// only their own warp can read) would put block-wide synchronisation back in
// the loop. Splitting each unit over a cluster of 2 or 4 CTAs was slower
// (0.115 and 0.160 ms with the CUDA-core loop): per-CTA setup and the merge
// outweigh the extra parallelism.
#include "pyr_common.cuh"
#include "tc_util.cuh"
#include "tile_list.cuh"

namespace pyr {

namespace {

using namespace tc;

constexpr int kWarps = 6;            // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kTileKeys = 64;        // keys per tile
constexpr int kMaxGw = 8;            // query rows per kv head (the N = 8 of the MMAs)
constexpr int kMaxListW = 130;

struct WPlan {
  // per warp: K tile [2 d-halves][64 keys][128 B] (16 KB), then V tile, same layout (16 KB)
  static constexpr int kStageBytes = 32768;
  static constexpr int kK = 0;
  static constexpr int kML = kK + kWarps * kStageBytes;        // per warp: [kMaxGw] max, [kMaxGw] sum
  static constexpr int kList = kML + kWarps * 2 * kMaxGw * 4;   // the unit's block list
  static constexpr int kBar = kList + kMaxListW * 4 + 8;        // kWarps mbarriers (8-byte aligned)
  static constexpr int kBytes = kBar + kWarps * 8 + 16 + 1024;  // + alignment slack
};

// byte offset of 16-byte chunk `ch` (8 d-elements, 0..15) of key row `key` in a tile
// loaded as two 64 d x 64 key TMA boxes with the 128-byte swizzle
__device__ __forceinline__ uint32_t tile_off(int key, int ch) {
  return (uint32_t)((ch >> 3) * 8192 + key * 128 + (((ch & 7) ^ (key & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D += A B for one m16n8k16 tile: A 16 x 16 bf16 (4 registers), B 16 x 8 bf16 (2), D 16 x 8 fp32
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// transpose of an 8 x 8 matrix of 16-bit elements held one row pair per lane
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_decode_warp_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                            const __nv_bfloat16* __restrict__ Q, const int32_t* __restrict__ idx, int dense,
                            __nv_bfloat16* __restrict__ O, float* __restrict__ lse, int* status, Geo g) {
  constexpr int D = 128;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_align<1024>(smem_raw);
  int* list = reinterpret_cast<int*>(smem + WPlan::kList);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + WPlan::kBar);
  __shared__ int tl_scratch[kTileListScratch];
  __shared__ int tl_entries[kTileListPitch];
  __shared__ int s_n;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.x;
  const int bi = unit / g.Hkv, hk = unit % g.Hkv;
  const int G = g.G;
  const int pos = g.q_offset;  // the query's position
  const int i = pos / g.b;     // its (current) block
  const int gq = lane >> 2;    // fragment row group: lanes 4gq .. 4gq + 3
  const int cq = 2 * (lane & 3);  // fragment column pair: the query rows cq, cq + 1 of the accumulators

  if (tid == 0) {
    s_abort = 0;
    for (int w = 0; w < kWarps; w++) mbar_init(bars + w, 1);
    fence_mbar_init();
  }
  // the unit's blocks: routed (ascending, validated), then the current block
  if (!dense) {
    // every thread of the CTA takes part (the helper has block-wide barriers)
    const int n = build_tile_list<1>(idx + (size_t)unit * g.nqb * g.topk, g.topk, i, 1, tl_scratch, tl_entries,
                                     status);
    if (warp == 0) {
      for (int e = lane; e < n; e += 32) list[e] = tl_entries[e] >> 4;
      if (lane == 0) s_n = n;
    }
  } else if (tid == 0) {
    s_n = i + 1;
  }
  // q^T as the B operand of the score MMAs (k = d, n = query row), for the whole unit: lane holds
  // rows gq (zero past G), d pairs 16 kc + cq .. + 1 (b0) and 16 kc + 8 + cq .. + 1 (b1)
  uint32_t qb[8][2];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(Q + ((size_t)bi * g.Hq + hk * G + gq) * g.Nq * D);
#pragma unroll
    for (int kc = 0; kc < 8; kc++) {
      qb[kc][0] = gq < G ? __ldg(qrow + (16 * kc + cq) / 2) : 0u;
      qb[kc][1] = gq < G ? __ldg(qrow + (16 * kc + 8 + cq) / 2) : 0u;
    }
  }
  __syncthreads();

  const int tpb = g.b / kTileKeys;  // tiles per block
  const int n_tiles = s_n * tpb;
  unsigned char* stage = smem + WPlan::kK + warp * WPlan::kStageBytes;
  uint64_t* wbar = bars + warp;
  // this warp's tiles: warp + kWarps * k, k = 0 .. n_mine - 1
  const int n_mine = warp < n_tiles ? (n_tiles - 1 - warp) / kWarps + 1 : 0;
  auto tile_of = [&](int k, int* j, int* key0, int* nk) {
    const int t = warp + kWarps * k;
    *j = dense ? t / tpb : list[t / tpb];
    *key0 = *j * g.b + (t % tpb) * kTileKeys;
    *nk = max(0, min(kTileKeys, g.N - *key0));
  };
  auto issue = [&](int k) {  // lane 0: tile k into the warp's stage; keys past N arrive as zeros
    int j, key0, nk;
    tile_of(k, &j, &key0, &nk);
    mbar_expect_tx(wbar, 32768);
    tma_load_3d(stage, &tmK, 0, key0, unit, wbar);
    tma_load_3d(stage + 8192, &tmK, 64, key0, unit, wbar);
    tma_load_3d(stage + 16384, &tmV, 0, key0, unit, wbar);
    tma_load_3d(stage + 24576, &tmV, 64, key0, unit, wbar);
  };
  if (lane == 0 && n_mine > 0) issue(0);

  // ldmatrix row addresses. K (A operand of the scores, m = key, k = d): matrix lane / 8 of a
  // 16 x 16 fragment is keys + 8 (lane & 8), d-chunk + (lane >> 4). V^T (A operand of P.V,
  // m = d, k = key, transposing load of V rows): keys + 8 (lane >> 4), d-chunk + ((lane >> 3) & 1).
  const uint32_t sK = smem_u32(stage), sV = smem_u32(stage + 16384);
  const int k_key = (lane & 7) + (lane & 8), k_ch = lane >> 4;
  const int v_key = (lane & 7) + ((lane >> 4) << 3), v_ch = (lane >> 3) & 1;

  const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float o[8][4];  // O^T: d rows 16 md + gq (+ 8 in [2], [3]), query rows cq, cq + 1
#pragma unroll
  for (int md = 0; md < 8; md++)
#pragma unroll
    for (int c = 0; c < 4; c++) o[md][c] = 0.f;
  bool ok = true;
  int k = 0;
  for (; k < n_mine; k++) {
    ok = mbar_wait(wbar, k & 1, (volatile int*)&s_abort);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    int j, key0, nk;
    tile_of(k, &j, &key0, &nk);

    // ---- S^T = K q^T: four 16-key row tiles, eight 16-wide d steps
    float sc[4][4];
#pragma unroll
    for (int mt = 0; mt < 4; mt++) {
#pragma unroll
      for (int c = 0; c < 4; c++) sc[mt][c] = 0.f;
#pragma unroll
      for (int kc = 0; kc < 8; kc++) {
        uint32_t a[4];
        ldsm_x4(sK + tile_off(16 * mt + k_key, 2 * kc + k_ch), a);
        mma16816(sc[mt], a, qb[kc][0], qb[kc][1]);
      }
    }
    // ---- online softmax per query row (lane: rows cq + e, keys 16 mt + gq (+ 8)); masked keys:
    // past N, or past the query's position in its own block
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int mt = 0; mt < 4; mt++)
#pragma unroll
      for (int c = 0; c < 4; c++) {
        const int key = 16 * mt + gq + ((c >> 1) << 3);
        const bool valid = key < nk && (j < i || key0 + key <= pos);
        sc[mt][c] = valid ? sc[mt][c] * sl2 : -INFINITY;
        mx[c & 1] = fmaxf(mx[c & 1], sc[mt][c]);
      }
    float corr[2], m_use[2];
#pragma unroll
    for (int e = 0; e < 2; e++) {
#pragma unroll
      for (int sh = 4; sh < 32; sh <<= 1) mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], sh));
      const float m_new = fmaxf(m_run[e], mx[e]);
      m_use[e] = m_new == -INFINITY ? 0.f : m_new;
      corr[e] = m_run[e] == -INFINITY ? 0.f : ex2(m_run[e] - m_use[e]);
      m_run[e] = m_new;
    }
    float ls[2] = {0.f, 0.f};
    uint32_t pb[4][2];  // P^T as the B operand of P.V (k = key, n = query row), per 16-key step
#pragma unroll
    for (int mt = 0; mt < 4; mt++) {
      const float p0 = ex2(sc[mt][0] - m_use[0]), p1 = ex2(sc[mt][1] - m_use[1]);
      const float p2 = ex2(sc[mt][2] - m_use[0]), p3 = ex2(sc[mt][3] - m_use[1]);
      ls[0] += p0 + p2;
      ls[1] += p1 + p3;
      // lane holds (key gq, rows cq, cq + 1): the transpose gives (row gq, keys cq, cq + 1)
      pb[mt][0] = movmatrix_t(pack_bf16x2(p0, p1));
      pb[mt][1] = movmatrix_t(pack_bf16x2(p2, p3));
    }
#pragma unroll
    for (int e = 0; e < 2; e++) l_run[e] = l_run[e] * corr[e] + ls[e];
    if (__any_sync(0xffffffffu, corr[0] != 1.f || corr[1] != 1.f)) {
#pragma unroll
      for (int md = 0; md < 8; md++) {
        o[md][0] *= corr[0];
        o[md][1] *= corr[1];
        o[md][2] *= corr[0];
        o[md][3] *= corr[1];
      }
    }
    // ---- O^T += V^T P^T: eight 16-wide d row tiles, four 16-key steps
#pragma unroll
    for (int md = 0; md < 8; md++)
#pragma unroll
      for (int kk = 0; kk < 4; kk++) {
        uint32_t a[4];
        ldsm_x4_t(sV + tile_off(16 * kk + v_key, 2 * md + v_ch), a);
        mma16816(o[md], a, pb[kk][0], pb[kk][1]);
      }
    __syncwarp();  // every lane's reads of the stage are done before it is refilled
    if (lane == 0 && k + 1 < n_mine) issue(k + 1);
  }
  if (!ok && lane == 0) {
    // drain: this warp's copy still in flight (issued for tile k)
    volatile int no_abort = 0;
    mbar_wait(wbar, k & 1, &no_abort);
    report(status, PYR_ETIMEOUT);
  }
  // the row sums: lanes gq = 0 .. 7 hold parts of the same rows
#pragma unroll
  for (int e = 0; e < 2; e++)
#pragma unroll
    for (int sh = 4; sh < 32; sh <<= 1) l_run[e] += __shfl_xor_sync(0xffffffffu, l_run[e], sh);
  __syncthreads();  // every warp done with its stage: the stages hold the warps' partial outputs now

  // ---- merge the warps: per row the max, the rescaled sums and outputs
  float* wml = reinterpret_cast<float*>(smem + WPlan::kML);  // [warp][2][kMaxGw]
  float* wacc = reinterpret_cast<float*>(smem + WPlan::kK);  // [warp][kMaxGw][128], over the stages
  if (gq == 0) {
#pragma unroll
    for (int e = 0; e < 2; e++) {
      wml[(warp * 2) * kMaxGw + cq + e] = m_run[e];
      wml[(warp * 2 + 1) * kMaxGw + cq + e] = l_run[e];
    }
  }
#pragma unroll
  for (int md = 0; md < 8; md++)
#pragma unroll
    for (int c = 0; c < 4; c++) {
      const int r = cq + (c & 1), d = 16 * md + gq + ((c >> 1) << 3);
      wacc[((size_t)warp * kMaxGw + r) * D + d] = o[md][c];
    }
  __syncthreads();
  for (int x = tid; x < G * D; x += kThreads) {
    const int r = x / D, e = x - r * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; w++) M = fmaxf(M, wml[(w * 2) * kMaxGw + r]);
    float L = 0.f, a = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; w++) {
      const float mw = wml[(w * 2) * kMaxGw + r];
      const float scl = mw == -INFINITY ? 0.f : ex2(mw - M);
      L += scl * wml[(w * 2 + 1) * kMaxGw + r];
      a += scl * wacc[((size_t)w * kMaxGw + r) * D + e];
    }
    const size_t orow = ((size_t)bi * g.Hq + hk * G + r) * g.Nq;
    O[orow * D + e] = __float2bfloat16_rn(L > 0.f ? a / L : 0.f);
    if (e == 0 && lse) lse[orow] = (M + log2f(L)) * 0.6931471805599453f;
  }
}

}  // namespace

bool attn_decode_warp_supported(const Geo& g) {
  return g.Nq == 1 && g.dtype == PYR_BF16 && g.d == 128 && (g.b == 64 || g.b == 128) && g.G <= kMaxGw &&
         g.topk + 1 <= kMaxListW;
}

cudaError_t launch_attn_decode_warp(const Geo& g, const void* Q, const void* K, const void* V, const int32_t* idx,
                                    int dense, void* O, float* lse, int* status, cudaStream_t st) {
  CUtensorMap mk, mv;
  if (!make_tmap_bf16_3d(&mk, K, g.d, g.N, g.B * g.Hkv, kTileKeys) ||
      !make_tmap_bf16_3d(&mv, V, g.d, g.N, g.B * g.Hkv, kTileKeys))
    return cudaErrorInvalidValue;
  auto kern = attn_decode_warp_kernel;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, WPlan::kBytes);
  if (e != cudaSuccess) return e;
  kern<<<g.B * g.Hkv, kThreads, WPlan::kBytes, st>>>(mk, mv, reinterpret_cast<const __nv_bfloat16*>(Q), idx, dense,
                                                     reinterpret_cast<__nv_bfloat16*>(O), lse, status, g);
  return cudaGetLastError();
}

}  // namespace pyr
