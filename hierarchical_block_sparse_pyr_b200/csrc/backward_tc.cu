// Backward pass of causal block-sparse attention on the tcgen05 tensor cores
// (bf16 operands, fp32 accumulation in tensor memory), PHBA summary A.1.4:
// scores and probabilities are recomputed on chip from the saved log-sum-exp,
// never stored. With the routes fixed and D_t = dO_t . O_t (precomputed per
// row), every attended (row t, key k) pair gives
//   P = exp(q_t . k_k / sqrt(d) - lse_t),  dS = P (dO_t . v_k - D_t).
//
// bwd_dq_tc_kernel: one CTA per 128 query rows of one (batch, kv head), the
// query-side mirror of the forward kernel. The K/V tile list is the forward's:
// the union of the tile's query blocks' routed blocks and their own blocks,
// with a mode per query block (skip / full / causal). Per 64-key tile:
//   S  = Q K^T   and  dP = dO V^T   into tensor memory (double-buffered);
//   one thread per row: P and dS = P (dP - D), written back as bf16 over S;
//   dQ += dS K   with dS read from tensor memory and K (the same shared-memory
//                tile as in S) described as an MN-major operand.
// Warp roles: warps 0-3 one thread per row; warp 4 TMA producer of Q, dO and
// the K tiles (3-stage ring: a K tile lives until its dQ MMA has run); warp 5
// MMA issuer; warp 6 TMA producer of the V tiles (2 stages). MMAs of one
// thread run in issue order, so the S/dP buffers of tile t+2 are only
// overwritten after the dQ MMA of tile t has read dS from them. Every wait is
// bounded; an abort drains in-flight copies and MMAs and frees tensor memory.
//
// bwd_dkdv_tc_kernel: one CTA per 128 keys of one (batch, kv head) (two
// 64-key blocks paired, or one 128-key block), the key-side mirror. The
// block-major schedule of A.1.4: the CTA walks the ascending union of the
// query blocks that attend its key blocks (each block's own query block,
// causal, then the query blocks whose routes list it, from offset/rho), each
// entry with a mode per key block. For every 64-row chunk (one head's rows of
// a visited query block):
//   S^T = K Q^T   and  dP^T = V dO^T   into tensor memory (keys on the lanes);
//   one thread per key: P^T and dS^T = P^T (dP^T - D), bf16, over S^T / dP^T;
//   dV += P^T dO  and  dK += dS^T Q  with the A operand read from tensor memory
//                 and the Q / dO chunk (the tile used above) as MN-major B.
// K and V stay in shared memory for the whole CTA; Q, dO and the chunk's lse
// and D stream through a 3-stage ring. Warps 0-3 one thread per key; warp 4
// producer (TMA for Q and dO, plain loads for lse and D); warp 5 MMA issuer.
#include <cudaTypedefs.h>

#include "pyr_common.cuh"
#include "tc_util.cuh"
#include "tile_list.cuh"

namespace pyr {

namespace {

using namespace tc;

constexpr int kKeys = 64;       // keys per K/V tile
constexpr int kMaxTiles = 264;  // >= 2 * (topk + 1) blocks of b / 64 tiles, topk <= 128

struct DqPlan {
  static constexpr int kQ = 0;                  // [2 halves][128 rows][128 B]
  static constexpr int kDO = kQ + 32768;        // same layout
  static constexpr int kK = kDO + 32768;        // 3 x [2][64][128 B]
  static constexpr int kV = kK + 3 * 16384;     // 2 x [2][64][128 B]
  static constexpr int kBar = kV + 2 * 16384;
  static constexpr int kNumBars = 1 + 6 + 4 + 2 + 2 + 1 + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kTiles = kMisc + 16;
  static constexpr int kEnd = kTiles + kMaxTiles * 4;
  static constexpr int kBytes = kEnd + 1024;
  static constexpr int kThreads = 7 * 32;
  static constexpr int kTmemCols = 512;  // S[2] 0..127, dP[2] 128..255, dQ 256..383
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int QB, int KB>
__global__ void __launch_bounds__(DqPlan::kThreads, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                     const float* __restrict__ lse, const float* __restrict__ delta, const int32_t* __restrict__ idx,
                     __nv_bfloat16* __restrict__ dQ, int* status, Geo g) {
  using PL = DqPlan;
  constexpr int TPB = KB / kKeys;  // tiles per key block
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_align<1024>(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PL::kBar);
  uint64_t* bar_q = bars;               // Q and dO landed
  uint64_t* bar_k_full = bars + 1;      // [3]
  uint64_t* bar_k_free = bars + 4;      // [3]
  uint64_t* bar_v_full = bars + 7;      // [2]
  uint64_t* bar_v_free = bars + 9;      // [2]
  uint64_t* bar_s_full = bars + 11;     // [2] S and dP of a tile in tensor memory
  uint64_t* bar_p_full = bars + 13;     // [2] dS of a tile written back (4 warps)
  uint64_t* bar_dq = bars + 15;         // every dQ MMA done
  uint64_t* bar_drain = bars + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + PL::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + PL::kMisc + 4);
  int* tiles = reinterpret_cast<int*>(smem + PL::kTiles);
  unsigned char* sQ = smem + PL::kQ;
  unsigned char* sDO = smem + PL::kDO;
  unsigned char* sK = smem + PL::kK;
  unsigned char* sV = smem + PL::kV;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.y;
  const int bi = unit / g.Hkv, hk = unit % g.Hkv;
  const int GB = g.G * g.b;                     // rows of one query block (all heads of the group)
  const int subs = max(1, QB * GB / 128);       // 128-row tiles per query group
  const int grp = blockIdx.x / subs, sub = blockIdx.x % subs;
  const int qb0 = grp * QB;
  const int i_first = g.i0 + qb0;
  const int nq_here = min(QB, g.nqb - qb0);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < 3; s++) {
      mbar_init(bar_k_full + s, 1);
      mbar_init(bar_k_free + s, 1);
    }
    for (int s = 0; s < 2; s++) {
      mbar_init(bar_v_full + s, 1);
      mbar_init(bar_v_free + s, 1);
      mbar_init(bar_s_full + s, 1);
      mbar_init(bar_p_full + s, 4);
    }
    mbar_init(bar_dq, 1);
    mbar_init(bar_drain, 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  // the tile's key-block list, built in the K ring before any copy lands there
  const int n_entries = build_tile_list<QB>(idx + ((size_t)unit * g.nqb + qb0) * g.topk, g.topk, i_first, nq_here,
                                            reinterpret_cast<int*>(sK), tiles, status);
  if (warp == 5) {
    tmem_alloc(tmem_slot, PL::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tP = tmem + 128, tDQ = tmem + 256;
  const int T = n_entries * TPB;

  auto tile_info = [&](int t, int* key0, int* mode) {
    const int e = t / TPB, h = t - e * TPB;
    *key0 = (tiles[e] >> 4) * KB + h * kKeys;
    *mode = tiles[e] & 15;
  };

  if (warp == 4 || warp == 6) {
    // ------------------------------------------------------------ producers
    const bool is_k = (warp == 4);
    if (lane == 0) {
      bool ok = true;
      if (is_k) {
        mbar_expect_tx(bar_q, 65536);
        for (int c = 0; c < 2; c++) {
          const int rr = sub * 128 + c * 64;
          const int qsub = rr / GB, within = rr % GB;
          const int gq = within / g.b, off = within % g.b;
          const int row = (i_first + qsub) * g.b + off - g.q_offset;
          const int head = bi * g.Hq + hk * g.G + gq;
          for (int h = 0; h < 2; h++) {
            tma_load_3d(sQ + h * 16384 + c * 8192, &tmQ, h * 64, row, head, bar_q);
            tma_load_3d(sDO + h * 16384 + c * 8192, &tmDO, h * 64, row, head, bar_q);
          }
        }
      }
      const int NS = is_k ? 3 : 2;
      uint64_t* full = is_k ? bar_k_full : bar_v_full;
      uint64_t* fre = is_k ? bar_k_free : bar_v_free;
      unsigned char* ring = is_k ? sK : sV;
      const CUtensorMap* map = is_k ? &tmK : &tmV;
      int t = 0;
      for (; t < T && ok; t++) {
        const int s = t % NS, k = t / NS;
        if (k > 0) ok = mbar_wait(fre + s, (k - 1) & 1, abort_flag);
        if (!ok) break;
        int key0, mode;
        tile_info(t, &key0, &mode);
        mbar_expect_tx(full + s, 16384);
        for (int h = 0; h < 2; h++) tma_load_3d(ring + s * 16384 + h * 8192, map, h * 64, key0, unit, full + s);
      }
      volatile int no_abort = 0;
      if (is_k) mbar_wait(bar_q, 0, &no_abort);
      for (int u = max(0, t - NS); u < t; u++) mbar_wait(full + (u % NS), (u / NS) & 1, &no_abort);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, kKeys, 0, 0);
      constexpr uint32_t idesc_q = idesc_bf16_f32(128, 128, 0, 1);
      const uint32_t aQ = smem_u32(sQ), aDO = smem_u32(sDO), aK = smem_u32(sK), aV = smem_u32(sV);
      bool ok = mbar_wait(bar_q, 0, abort_flag);
      int issued = 0;
      for (int t = 0; t <= T && ok; t++) {
        if (t < T) {
          const int sk = t % 3, sv = t % 2, sb = t & 1;
          ok = mbar_wait(bar_k_full + sk, (t / 3) & 1, abort_flag);
          if (ok) ok = mbar_wait(bar_v_full + sv, (t / 2) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; kk++) {
            const uint32_t oq = (kk >> 2) * 16384 + (kk & 3) * 32, ok_ = (kk >> 2) * 8192 + (kk & 3) * 32;
            umma_bf16(tS + sb * 64, sdesc_sw128(aQ + oq, 16, 1024), sdesc_sw128(aK + sk * 16384 + ok_, 16, 1024),
                      idesc_s, kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < 8; kk++) {
            const uint32_t oq = (kk >> 2) * 16384 + (kk & 3) * 32, ov = (kk >> 2) * 8192 + (kk & 3) * 32;
            umma_bf16(tP + sb * 64, sdesc_sw128(aDO + oq, 16, 1024), sdesc_sw128(aV + sv * 16384 + ov, 16, 1024),
                      idesc_s, kk > 0);
          }
          umma_commit(bar_s_full + sb);
          umma_commit(bar_v_free + sv);
          issued++;
        }
        if (t >= 1) {
          const int u = t - 1, sk = u % 3, pb = u & 1;
          ok = mbar_wait(bar_p_full + pb, (u >> 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; kk++)
            umma_bf16_ts(tDQ, tS + pb * 64 + kk * 8, sdesc_sw128(aK + sk * 16384 + kk * 2048, 8192, 1024), idesc_q,
                         (u > 0 || kk > 0) ? 1u : 0u);
          umma_commit(bar_k_free + sk);
          issued++;
        }
      }
      if (ok) umma_commit(bar_dq);
      if (issued > 0) {
        umma_commit(bar_drain);
        volatile int no_abort = 0;
        mbar_wait(bar_drain, 0, &no_abort);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ one thread per row
    const int r = warp * 32 + lane;
    const int rr = sub * 128 + r;
    const int qsub = rr / GB, within = rr % GB;
    const int gq = within / g.b, off = within % g.b;
    const int iq = i_first + qsub;
    const int p = iq * g.b + off;
    const bool row_ok = qsub < nq_here && p >= g.q_offset && p < g.q_offset + g.Nq;
    const size_t orow = ((size_t)bi * g.Hq + hk * g.G + gq) * g.Nq + (size_t)(p - g.q_offset);
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float sl2 = rsqrtf((float)g.d) * 1.4426950408889634f;
    const float lse2 = row_ok ? lse[orow] * 1.4426950408889634f : 0.f;
    const float D = row_ok ? delta[orow] : 0.f;
    bool ok = true;
    float s[kKeys], dp[kKeys];
    for (int t = 0; t < T; t++) {
      const int sb = t & 1;
      ok = warp_wait(bar_s_full + sb, (t >> 1) & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      tmem_ld32(tS + lane_base + sb * 64, s);
      tmem_ld32(tS + lane_base + sb * 64 + 32, s + 32);
      tmem_ld32(tP + lane_base + sb * 64, dp);
      tmem_ld32(tP + lane_base + sb * 64 + 32, dp + 32);
      tmem_wait_ld();
      int key0, mode;
      tile_info(t, &key0, &mode);
      const int md = row_ok ? (mode >> (2 * qsub)) & 3 : 0;
      const int lim = md == 0 ? 0 : (md == 1 ? min(kKeys, g.N - key0) : min(kKeys, p - key0 + 1));
      uint32_t pk[32];
      const float2 scl = make_float2(sl2, sl2), offs = make_float2(-lse2, -lse2), dd = make_float2(-D, -D);
#pragma unroll
      for (int c = 0; c < 32; c++) {
        const float2 x = __ffma2_rn(make_float2(s[2 * c], s[2 * c + 1]), scl, offs);
        const float p0 = 2 * c < lim ? ex2(x.x) : 0.f, p1 = 2 * c + 1 < lim ? ex2(x.y) : 0.f;
        const float2 y = __fadd2_rn(make_float2(dp[2 * c], dp[2 * c + 1]), dd);
        pk[c] = pack_bf16(p0 * y.x, p1 * y.y);
      }
      tmem_st32u(tS + lane_base + sb * 64, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p_full + sb);
    }
    if (ok) ok = warp_wait(bar_dq, 0, abort_flag);
    if (ok) {
      tc_fence_after();
      const float scale = rsqrtf((float)g.d);
      float o[32];
#pragma unroll 1
      for (int c = 0; c < 128; c += 32) {
        tmem_ld32(tDQ + lane_base + c, o);
        tmem_wait_ld();
        if (row_ok && T > 0) {
          uint4* dst = reinterpret_cast<uint4*>(dQ + orow * 128 + c);
#pragma unroll
          for (int k = 0; k < 4; k++) {
            uint4 v;
            v.x = pack_bf16(o[8 * k + 0] * scale, o[8 * k + 1] * scale);
            v.y = pack_bf16(o[8 * k + 2] * scale, o[8 * k + 3] * scale);
            v.z = pack_bf16(o[8 * k + 4] * scale, o[8 * k + 5] * scale);
            v.w = pack_bf16(o[8 * k + 6] * scale, o[8 * k + 7] * scale);
            dst[k] = v;
          }
        }
      }
    }
  }

  // ---- teardown ----
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) report(status, PYR_ETIMEOUT);
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, PL::kTmemCols);
  }
}

template <int QB, int KB>
cudaError_t launch_dq(const Geo& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                      const CUtensorMap& mdo, const float* lse, const float* delta, const int32_t* idx, void* dQ,
                      int* status, cudaStream_t st) {
  auto kern = bwd_dq_tc_kernel<QB, KB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, DqPlan::kBytes);
  if (e != cudaSuccess) return e;
  const int subs = QB * g.G * g.b >= 256 ? QB * g.G * g.b / 128 : 1;
  dim3 grid(((g.nqb + QB - 1) / QB) * subs, g.B * g.Hkv);
  kern<<<grid, DqPlan::kThreads, DqPlan::kBytes, st>>>(mq, mk, mv, mdo, lse, delta, idx,
                                                        reinterpret_cast<__nv_bfloat16*>(dQ), status, g);
  return cudaGetLastError();
}


// ---------------------------------------------------------------------------- dK, dV

constexpr int kKvStages = 3;

struct KvPlan {
  static constexpr int kK = 0;                              // [2 halves][128 keys][128 B]
  static constexpr int kV = 32768;
  static constexpr int kStage = 65536;                      // stages: Q chunk, dO chunk, lse, D
  static constexpr int kStageBytes = 16384 + 16384 + 256 + 256;
  static constexpr int kBar = kStage + kKvStages * kStageBytes;
  static constexpr int kNumBars = 1 + 2 * kKvStages + 2 + 2 + 1 + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kEnd = kMisc + 16;
  static constexpr int kBytes = kEnd + 1024;
  static constexpr int kThreads = 6 * 32;
  static constexpr int kTmemCols = 512;  // S^T[2] 0..127, dP^T[2] 128..255, dV 256..383, dK 384..511
};

// The visits of a 128-key tile: the ascending union, over its TPB key blocks
// jj, of [jj (own block, causal)] + rho[offset[jj] .. offset[jj+1]) (routed,
// all > jj), as (query block, 2 mode bits per key block: 1 full, 2 causal).
template <int TPB>
struct Visits {
  const int32_t* r[TPB];
  int n[TPB], pos[TPB], own[TPB];  // own: the key block's own query block, -1 once visited
  __device__ void init(const int32_t* offset, const int32_t* rho, int j0, int nb) {
    for (int h = 0; h < TPB; h++) {
      const int jj = j0 + h;
      if (jj < nb) {
        r[h] = rho + offset[jj];
        n[h] = offset[jj + 1] - offset[jj];
        own[h] = jj;
      } else {
        r[h] = rho;
        n[h] = 0;
        own[h] = -1;
      }
      pos[h] = 0;
    }
  }
  __device__ bool next(int* qb, int* mode) {
    int cand[TPB];
    int best = 0x7fffffff;
    for (int h = 0; h < TPB; h++) {
      cand[h] = own[h] >= 0 ? own[h] : (pos[h] < n[h] ? r[h][pos[h]] : 0x7fffffff);
      best = min(best, cand[h]);
    }
    if (best == 0x7fffffff) return false;
    int m = 0;
    for (int h = 0; h < TPB; h++) {
      if (cand[h] != best) continue;
      if (own[h] >= 0) {
        m |= 2 << (2 * h);
        own[h] = -1;
      } else {
        m |= 1 << (2 * h);
        pos[h]++;
      }
    }
    *qb = best;
    *mode = m;
    return true;
  }
};

template <int KB>
__global__ void __launch_bounds__(KvPlan::kThreads, 1)
    bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                       const float* __restrict__ lse, const float* __restrict__ delta,
                       const int32_t* __restrict__ offset, const int32_t* __restrict__ rho,
                       __nv_bfloat16* __restrict__ dK, __nv_bfloat16* __restrict__ dV, int* status, Geo g) {
  using PL = KvPlan;
  constexpr int TPB = 128 / KB;  // key blocks per tile
  constexpr int NS = kKvStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_align<1024>(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PL::kBar);
  uint64_t* bar_kv = bars;                   // K and V landed
  uint64_t* bar_full = bars + 1;             // [NS] a chunk's Q, dO, lse, D landed
  uint64_t* bar_free = bars + 1 + NS;        // [NS] the chunk's last MMA finished
  uint64_t* bar_s_full = bars + 1 + 2 * NS;  // [2] S^T, dP^T in tensor memory
  uint64_t* bar_p_full = bar_s_full + 2;     // [2] P^T, dS^T written back (4 warps)
  uint64_t* bar_done = bar_p_full + 2;
  uint64_t* bar_drain = bar_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + PL::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + PL::kMisc + 4);
  int* s_nvisits = reinterpret_cast<int*>(smem + PL::kMisc + 8);
  unsigned char* sK = smem + PL::kK;
  unsigned char* sV = smem + PL::kV;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.y;
  const int bi = unit / g.Hkv, hk = unit % g.Hkv;
  const int x0 = blockIdx.x * 128;  // first key of the tile
  const int j0 = x0 / KB;
  const int32_t* off_u = offset + (size_t)unit * (g.nb + 1);
  const int32_t* rho_u = rho + (size_t)unit * g.nqb * g.topk;
  const int CPV = g.G * g.b / 64;  // 64-row chunks per visited query block

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < NS; s++) {
      mbar_init(bar_full + s, 1);
      mbar_init(bar_free + s, 1);
    }
    for (int s = 0; s < 2; s++) {
      mbar_init(bar_s_full + s, 1);
      mbar_init(bar_p_full + s, 4);
    }
    mbar_init(bar_done, 1);
    mbar_init(bar_drain, 1);
    fence_mbar_init();
    *abort_flag = 0;
    Visits<TPB> vis;
    vis.init(off_u, rho_u, j0, g.nb);
    int n = 0, qb, mode;
    while (vis.next(&qb, &mode)) n++;
    *s_nvisits = n;
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, PL::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tP = tmem + 128, tDV = tmem + 256, tDK = tmem + 384;
  const int T = *s_nvisits * CPV;  // chunks

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    bool ok = true;
    if (lane == 0) {
      mbar_expect_tx(bar_kv, 65536);
      for (int c = 0; c < 2; c++)
        for (int h = 0; h < 2; h++) {
          tma_load_3d(sK + h * 16384 + c * 8192, &tmK, h * 64, x0 + c * 64, unit, bar_kv);
          tma_load_3d(sV + h * 16384 + c * 8192, &tmV, h * 64, x0 + c * 64, unit, bar_kv);
        }
    }
    Visits<TPB> vis;
    vis.init(off_u, rho_u, j0, g.nb);
    int qb = 0, mode = 0, t = 0;
    for (; t < T && ok; t++) {
      const int ch = t % CPV;
      if (ch == 0) vis.next(&qb, &mode);
      const int s = t % NS, k = t / NS;
      if (k > 0) {
        bool w = true;
        if (lane == 0) w = mbar_wait(bar_free + s, (k - 1) & 1, abort_flag);
        ok = __shfl_sync(0xffffffffu, w, 0);
        if (!ok) break;
      }
      const int r0 = ch * 64;  // first row of the chunk within the query block's G*b rows
      const int gq = r0 / g.b, offr = r0 % g.b;
      const int head = bi * g.Hq + hk * g.G + gq;
      const int p0 = qb * g.b + offr;  // position of the chunk's first row (q_offset = 0)
      unsigned char* st = smem + PL::kStage + s * PL::kStageBytes;
      float* s_lse = reinterpret_cast<float*>(st + 32768);
      float* s_del = s_lse + 64;
      for (int e = lane; e < 64; e += 32) {
        const int p = p0 + e;
        const size_t row = (size_t)head * g.Nq + p;
        s_lse[e] = p < g.Nq ? lse[row] * 1.4426950408889634f : 0.f;
        s_del[e] = p < g.Nq ? delta[row] : 0.f;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_expect_tx(bar_full + s, 32768);
        for (int h = 0; h < 2; h++) {
          tma_load_3d(st + h * 8192, &tmQ, h * 64, p0, head, bar_full + s);
          tma_load_3d(st + 16384 + h * 8192, &tmDO, h * 64, p0, head, bar_full + s);
        }
      }
      __syncwarp();
    }
    if (lane == 0) {
      volatile int no_abort = 0;
      mbar_wait(bar_kv, 0, &no_abort);
      for (int u = max(0, t - NS); u < t; u++) mbar_wait(bar_full + (u % NS), (u / NS) & 1, &no_abort);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t idesc_g = idesc_bf16_f32(128, 128, 0, 1);
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aSt = smem_u32(smem + PL::kStage);
      bool ok = mbar_wait(bar_kv, 0, abort_flag);
      int issued = 0;
      for (int t = 0; t <= T && ok; t++) {
        if (t < T) {
          const int s = t % NS, sb = t & 1;
          ok = mbar_wait(bar_full + s, (t / NS) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t aQ = aSt + s * PL::kStageBytes, aDO = aQ + 16384;
#pragma unroll
          for (int kk = 0; kk < 8; kk++) {
            const uint32_t oa = (kk >> 2) * 16384 + (kk & 3) * 32, ob = (kk >> 2) * 8192 + (kk & 3) * 32;
            umma_bf16(tS + sb * 64, sdesc_sw128(aK + oa, 16, 1024), sdesc_sw128(aQ + ob, 16, 1024), idesc_s,
                      kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < 8; kk++) {
            const uint32_t oa = (kk >> 2) * 16384 + (kk & 3) * 32, ob = (kk >> 2) * 8192 + (kk & 3) * 32;
            umma_bf16(tP + sb * 64, sdesc_sw128(aV + oa, 16, 1024), sdesc_sw128(aDO + ob, 16, 1024), idesc_s,
                      kk > 0);
          }
          umma_commit(bar_s_full + sb);
          issued++;
        }
        if (t >= 1) {
          const int u = t - 1, s = u % NS, pb = u & 1;
          ok = mbar_wait(bar_p_full + pb, (u >> 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t aQ = aSt + s * PL::kStageBytes, aDO = aQ + 16384;
#pragma unroll
          for (int kk = 0; kk < 4; kk++) {
            umma_bf16_ts(tDV, tS + pb * 64 + kk * 8, sdesc_sw128(aDO + kk * 2048, 8192, 1024), idesc_g,
                         (u > 0 || kk > 0) ? 1u : 0u);
            umma_bf16_ts(tDK, tP + pb * 64 + kk * 8, sdesc_sw128(aQ + kk * 2048, 8192, 1024), idesc_g,
                         (u > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(bar_free + s);
          issued++;
        }
      }
      if (ok) umma_commit(bar_done);
      if (issued > 0) {
        umma_commit(bar_drain);
        volatile int no_abort = 0;
        mbar_wait(bar_drain, 0, &no_abort);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ one thread per key
    const int r = warp * 32 + lane;
    const int x = x0 + r;  // this thread's key position
    const int h = r / KB;  // its key block within the tile
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float sl2 = rsqrtf((float)g.d) * 1.4426950408889634f;
    Visits<TPB> vis;
    vis.init(off_u, rho_u, j0, g.nb);
    int qb = 0, mode = 0;
    bool ok = true;
    float sv[64], dp[64];
    for (int t = 0; t < T; t++) {
      const int ch = t % CPV, s = t % NS, sb = t & 1;
      if (ch == 0) vis.next(&qb, &mode);
      ok = warp_wait(bar_s_full + sb, (t >> 1) & 1, abort_flag);
      if (ok) ok = warp_wait(bar_full + s, (t / NS) & 1, abort_flag);  // lse, D of the chunk
      if (!ok) break;
      tc_fence_after();
      tmem_ld32(tS + lane_base + sb * 64, sv);
      tmem_ld32(tS + lane_base + sb * 64 + 32, sv + 32);
      tmem_ld32(tP + lane_base + sb * 64, dp);
      tmem_ld32(tP + lane_base + sb * 64 + 32, dp + 32);
      tmem_wait_ld();
      const float* s_lse = reinterpret_cast<const float*>(smem + PL::kStage + s * PL::kStageBytes + 32768);
      const float* s_del = s_lse + 64;
      const int md = x < g.N ? (mode >> (2 * h)) & 3 : 0;
      const int p0 = qb * g.b + (ch * 64) % g.b;  // position of column 0
      // valid columns: rows with positions < N; for the own block only rows at or after the key
      const int c_lo = md == 2 ? max(0, x - p0) : (md == 1 ? 0 : 64);
      const int c_hi = min(64, g.N - p0);
      uint32_t pk[32], dk[32];
#pragma unroll
      for (int c = 0; c < 32; c++) {
        const float2 l2 = *reinterpret_cast<const float2*>(s_lse + 2 * c);
        const float2 dd = *reinterpret_cast<const float2*>(s_del + 2 * c);
        const float2 y = __ffma2_rn(make_float2(sv[2 * c], sv[2 * c + 1]), make_float2(sl2, sl2),
                                    make_float2(-l2.x, -l2.y));
        const bool v0 = 2 * c >= c_lo && 2 * c < c_hi, v1 = 2 * c + 1 >= c_lo && 2 * c + 1 < c_hi;
        const float q0 = v0 ? ex2(y.x) : 0.f, q1 = v1 ? ex2(y.y) : 0.f;
        pk[c] = pack_bf16(q0, q1);
        dk[c] = pack_bf16(q0 * (dp[2 * c] - dd.x), q1 * (dp[2 * c + 1] - dd.y));
      }
      tmem_st32u(tS + lane_base + sb * 64, pk);
      tmem_st32u(tP + lane_base + sb * 64, dk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p_full + sb);
    }
    if (ok) ok = warp_wait(bar_done, 0, abort_flag);
    if (ok) {
      tc_fence_after();
      const float scale = rsqrtf((float)g.d);
      float o[32];
      for (int which = 0; which < 2; which++) {
        __nv_bfloat16* dst_base = (which ? dK : dV) + ((size_t)unit * g.N + x) * 128;
        const float sc = which ? scale : 1.f;
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          tmem_ld32((which ? tDK : tDV) + lane_base + c, o);
          tmem_wait_ld();
          if (x < g.N) {
            uint4* dst = reinterpret_cast<uint4*>(dst_base + c);
#pragma unroll
            for (int k = 0; k < 4; k++) {
              uint4 v;
              v.x = pack_bf16(o[8 * k + 0] * sc, o[8 * k + 1] * sc);
              v.y = pack_bf16(o[8 * k + 2] * sc, o[8 * k + 3] * sc);
              v.z = pack_bf16(o[8 * k + 4] * sc, o[8 * k + 5] * sc);
              v.w = pack_bf16(o[8 * k + 6] * sc, o[8 * k + 7] * sc);
              dst[k] = v;
            }
          }
        }
      }
    }
  }

  // ---- teardown ----
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) report(status, PYR_ETIMEOUT);
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, PL::kTmemCols);
  }
}

template <int KB>
cudaError_t launch_dkdv(const Geo& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        const CUtensorMap& mdo, const float* lse, const float* delta, const int32_t* offset,
                        const int32_t* rho, void* dK, void* dV, int* status, cudaStream_t st) {
  auto kern = bwd_dkdv_tc_kernel<KB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, KvPlan::kBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((g.N + 127) / 128, g.B * g.Hkv);
  kern<<<grid, KvPlan::kThreads, KvPlan::kBytes, st>>>(mq, mk, mv, mdo, lse, delta, offset, rho,
                                                        reinterpret_cast<__nv_bfloat16*>(dK),
                                                        reinterpret_cast<__nv_bfloat16*>(dV), status, g);
  return cudaGetLastError();
}

}  // namespace

// 64-row MHA blocks (backward_pair.cu): products transposed so that one block's own list fills M = 128
bool backward_pair_supported(const Geo& g);
cudaError_t launch_backward_dq_pair(const Geo& g, const CUtensorMap& mq, const CUtensorMap& mk,
                                    const CUtensorMap& mv, const CUtensorMap& mdo, const float* lse,
                                    const float* delta, const int32_t* idx, void* dQ, int* status, cudaStream_t st);
cudaError_t launch_backward_dkdv_pair(const Geo& g, const CUtensorMap& mq, const CUtensorMap& mk,
                                      const CUtensorMap& mv, const CUtensorMap& mdo, const float* lse,
                                      const float* delta, const int32_t* offset, const int32_t* rho, void* dK,
                                      void* dV, void* scratch, int* status, cudaStream_t st);

bool backward_tc_supported(const Geo& g) {
  if (g.dtype != PYR_BF16 || g.d != 128) return false;
  if (g.b != 64 && g.b != 128) return false;
  if (g.q_offset != 0 || g.Nq != g.N) return false;
  const int rows = g.G * g.b;
  return rows == 64 || rows == 128 || rows == 256;
}

cudaError_t launch_backward_dq_tc(const Geo& g, const void* Q, const void* K, const void* V, const void* dO,
                                  const float* lse, const float* delta, const int32_t* idx, void* dQ, int* status,
                                  cudaStream_t st) {
  CUtensorMap mq, mk, mv, mdo;
  if (!make_tmap_bf16_3d(&mq, Q, g.d, g.Nq, g.B * g.Hq) || !make_tmap_bf16_3d(&mk, K, g.d, g.N, g.B * g.Hkv) ||
      !make_tmap_bf16_3d(&mv, V, g.d, g.N, g.B * g.Hkv) || !make_tmap_bf16_3d(&mdo, dO, g.d, g.Nq, g.B * g.Hq))
    return cudaErrorInvalidValue;
  if (backward_pair_supported(g))
    return launch_backward_dq_pair(g, mq, mk, mv, mdo, lse, delta, idx, dQ, status, st);
  const int rows = g.G * g.b;
  if (g.b == 64) {
    if (rows == 64) return launch_dq<2, 64>(g, mq, mk, mv, mdo, lse, delta, idx, dQ, status, st);
    return launch_dq<1, 64>(g, mq, mk, mv, mdo, lse, delta, idx, dQ, status, st);
  }
  return launch_dq<1, 128>(g, mq, mk, mv, mdo, lse, delta, idx, dQ, status, st);
}

}  // namespace pyr

namespace pyr {
cudaError_t launch_backward_dkdv_tc(const Geo& g, const void* Q, const void* K, const void* V, const void* dO,
                                    const float* lse, const float* delta, const int32_t* offset, const int32_t* rho,
                                    void* dK, void* dV, void* scratch, int* status, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mdo;
  if (!tc::make_tmap_bf16_3d(&mq, Q, g.d, g.Nq, g.B * g.Hq) || !tc::make_tmap_bf16_3d(&mk, K, g.d, g.N, g.B * g.Hkv) ||
      !tc::make_tmap_bf16_3d(&mv, V, g.d, g.N, g.B * g.Hkv) || !tc::make_tmap_bf16_3d(&mdo, dO, g.d, g.Nq, g.B * g.Hq))
    return cudaErrorInvalidValue;
  if (backward_pair_supported(g))
    return launch_backward_dkdv_pair(g, mq, mk, mv, mdo, lse, delta, offset, rho, dK, dV, scratch, status, st);
  if (g.b == 64) return launch_dkdv<64>(g, mq, mk, mv, mdo, lse, delta, offset, rho, dK, dV, status, st);
  return launch_dkdv<128>(g, mq, mk, mv, mdo, lse, delta, offset, rho, dK, dV, status, st);
}
}  // namespace pyr
