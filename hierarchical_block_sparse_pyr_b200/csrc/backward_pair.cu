// Backward pass of causal block-sparse attention for 64-row MHA query blocks
// (bf16, d = 128, b = 64, one query head per kv head) on the tcgen05 tensor
// cores, PHBA summary A.1.4: P and dS are recomputed from the saved
// log-sum-exp, never stored.
//
// A 64-row block fills half of an M = 128 MMA, and an M = 64 MMA takes as long
// as an M = 128 one. Pairing two blocks in one 128-row tile over the union of
// their lists (the general kernels of backward_tc.cu) pays a full step for
// every union entry, even where only one half attends it. These kernels put
// on the M side of every MMA 128 rows that ONE block's own list supplies, two
// list entries at a time, and transpose the products to match, so no union is
// formed:
//
// bwd_dq_pair_kernel: one CTA per (query block i, unit). Its key tiles (the
// accepted routes of row i, ascending, then block i itself) are taken two at a
// time, 128 keys per step:
//   S^T = K2 Q^T,  dP^T = V2 dO^T      (M = 128 keys, N = 64 rows, K = d)
//   one thread per key: P^T = exp(S^T / sqrt(d) - lse), dS^T = P^T (dP^T - D),
//   bf16, written to shared memory over the V tiles (dP^T no longer needs them)
//   dQ^T += K2^T dS^T                   (M = d, N = 64 rows, K = 128 keys)
//
// bwd_dkdv_pair_kernel: one CTA per (key block j, unit). The query blocks that
// attend j (j itself, causal, then the block-major list offset/rho, all > j)
// are taken two at a time, 128 rows per step:
//   S = Q2 K^T,  dP = dO2 V^T          (M = 128 rows, N = 64 keys, K = d)
//   one thread per row: P, then dS = P (dP - D), bf16, through one buffer
//   dV^T += dO2^T P,  dK^T += Q2^T dS  (M = d, N = 64 keys, K = 128 rows)
//
// An odd list pads its last step with a second copy of its last block whose
// half is masked to zero (the operands stay finite, so 0 * operand = 0).
// Operands transposed for the second product are read from the same
// shared-memory tiles as MN-major descriptors. Each CTA holds 256 tensor-memory
// columns and at most 112 KB of shared memory, so two CTAs share an SM and
// one's loads and softmax run under the other's MMAs. Warps 0-3: one thread
// per tensor-memory lane; warp 4: TMA producer; warp 5: MMA issuer. Every wait
// is bounded; an abort drains in-flight copies and MMAs and frees tensor
// memory.
#include <cudaTypedefs.h>

#include "pyr_common.cuh"
#include "tc_util.cuh"
#include "tile_list.cuh"

namespace pyr {

namespace {

using namespace tc;

constexpr float kLog2e = 1.4426950408889634f;

// Shared memory is laid out from the dynamic window's start, which the
// kernels require to be 1024-byte aligned (the 128-byte swizzle atoms are
// 1024 bytes); they check it and report PYR_EINVAL otherwise.
struct DqPairPlan {
  static constexpr int kQ = 0;          // [2 d-halves][64 rows][128 B]
  static constexpr int kDO = 16384;     // same
  static constexpr int kK = 32768;      // [2 d-halves][128 keys][128 B]
  static constexpr int kV = 65536;      // same; dS^T [128 keys][64 rows] bf16 over its first 16 KB
  static constexpr int kRow = 98304;    // lse * log2(e) [64], D [64] of the block's rows
  static constexpr int kBar = kRow + 512;
  static constexpr int kNumBars = 7;
  static constexpr int kMisc = kBar + kNumBars * 8;  // tensor-memory base, abort flag
  static constexpr int kList = kMisc + 16;          // route compaction scratch
  static constexpr int kBytes = kList + kTileListScratch * 4;
  static constexpr int kThreads = 6 * 32;
  static constexpr int kTmemCols = 256;  // S^T 0..63, dP^T 64..127, dQ^T 128..191
};

struct KvPairPlan {
  static constexpr int kK = 0;        // [2 d-halves][64 keys][128 B]
  static constexpr int kV = 16384;    // same
  static constexpr int kQ = 32768;    // [2 d-halves][128 rows][128 B]
  static constexpr int kDO = 65536;   // same
  static constexpr int kPS = 98304;   // P, then dS: [128 rows][64 keys] bf16
  static constexpr int kBar = 114688;
  static constexpr int kNumBars = 9;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kThreads = 6 * 32;
  static constexpr int kTmemCols = 256;  // S 0..63, dP 64..127, dV^T 128..191, dK^T 192..255
};
static_assert(2 * (KvPairPlan::kBytes + 1024) <= 228 * 1024, "two dK/dV CTAs per SM");
static_assert(2 * (DqPairPlan::kBytes + 1024) <= 228 * 1024, "two dQ CTAs per SM");

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Row r of a [128][64] bf16 MN-major operand with 128-byte swizzle (row = the
// K index, 64 contiguous N elements): 16-byte chunk c sits at chunk c ^ (r % 8).
__device__ __forceinline__ void store_row_sw128(unsigned char* base, int r, const uint32_t* v) {
  unsigned char* row = base + r * 128;
#pragma unroll
  for (int c = 0; c < 8; c++)
    *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
}

// The four shared-memory descriptors of one K = 16 slice kk (0..7):
//  K-major, 128 rows of 128 B per d-half, d-halves `half` bytes apart
__device__ __forceinline__ uint64_t kmajor(uint32_t base, int kk, uint32_t half) {
  return sdesc_sw128(base + (kk >> 2) * half + (kk & 3) * 32, 16, 1024);
}
//  MN-major, rows = the K index (16 rows per slice), 64-element chunks `chunk` bytes apart
__device__ __forceinline__ uint64_t mnmajor(uint32_t base, int kk, uint32_t chunk) {
  return sdesc_sw128(base + kk * 2048, chunk, 1024);
}

// ---------------------------------------------------------------------------- dQ

__global__ void __launch_bounds__(DqPairPlan::kThreads, 2)
    bwd_dq_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                       const float* __restrict__ lse, const float* __restrict__ delta,
                       const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ dQ, int* status, Geo g) {
  using PL = DqPairPlan;
  extern __shared__ __align__(1024) unsigned char smem[];
  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0) report(status, PYR_EINVAL);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PL::kBar);
  uint64_t* bar_q = bars;         // Q, dO landed (and the rows' lse, D written)
  uint64_t* bar_kv = bars + 1;    // a step's K and V tiles landed
  uint64_t* bar_s = bars + 2;     // S^T, dP^T of the step in tensor memory
  uint64_t* bar_p = bars + 3;     // dS^T of the step written (4 warps)
  uint64_t* bar_free = bars + 4;  // the step's dQ MMAs done: K, V and dS^T reusable
  uint64_t* bar_dq = bars + 5;    // every dQ MMA done
  uint64_t* bar_drain = bars + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + PL::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + PL::kMisc + 4);
  int* list = reinterpret_cast<int*>(smem + PL::kList);
  unsigned char* sQ = smem + PL::kQ;
  unsigned char* sDO = smem + PL::kDO;
  unsigned char* sK = smem + PL::kK;
  unsigned char* sV = smem + PL::kV;
  float* s_row = reinterpret_cast<float*>(smem + PL::kRow);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.y;  // (batch, kv head) = (batch, query head): one query head per kv head
  const int iq = g.i0 + blockIdx.x;
  const int p0 = iq * 64 - g.q_offset;  // first row of the block (q_offset = 0 here)
  const int rows = min(64, g.Nq - p0);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_kv, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_p, 4);
    mbar_init(bar_free, 1);
    mbar_init(bar_dq, 1);
    mbar_init(bar_drain, 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  // the block's key tiles: accepted routes, ascending, then block iq (ends with a CTA barrier)
  compact_routes(idx + ((size_t)unit * g.nqb + blockIdx.x) * g.topk, g.topk, iq, 1, list, status);
  const int T = list[4 * kTileListPitch];
  const int steps = (T + 1) >> 1;
  if (warp == 5) {
    tmem_alloc(tmem_slot, PL::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tP = tmem + 64, tDQ = tmem + 128;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    for (int e = lane; e < 64; e += 32) {
      const bool in = e < rows;
      const size_t row = (size_t)unit * g.Nq + p0 + e;
      s_row[e] = in ? lse[row] * kLog2e : 0.f;
      s_row[64 + e] = in ? delta[row] : 0.f;
    }
    __syncwarp();
    if (lane == 0) {
      mbar_expect_tx(bar_q, 32768);
      for (int h = 0; h < 2; h++) {
        tma_load_3d(sQ + h * 8192, &tmQ, h * 64, p0, unit, bar_q);
        tma_load_3d(sDO + h * 8192, &tmDO, h * 64, p0, unit, bar_q);
      }
      int u = 0;
      for (; u < steps; u++) {
        if (u > 0 && !mbar_wait(bar_free, (u - 1) & 1, abort_flag)) break;
        mbar_expect_tx(bar_kv, 65536);
        for (int c = 0; c < 2; c++) {
          const int key0 = list[min(2 * u + c, T - 1)] * 64;
          for (int h = 0; h < 2; h++) {
            tma_load_3d(sK + h * 16384 + c * 8192, &tmK, h * 64, key0, unit, bar_kv);
            tma_load_3d(sV + h * 16384 + c * 8192, &tmV, h * 64, key0, unit, bar_kv);
          }
        }
      }
      // copies still in flight land before the CTA can exit
      volatile int no_abort = 0;
      mbar_wait(bar_q, 0, &no_abort);
      if (u > 0) mbar_wait(bar_kv, (u - 1) & 1, &no_abort);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);  // keys x rows, both K-major
      constexpr uint32_t idesc_q = idesc_bf16_f32(128, 64, 1, 1);  // d x rows, both MN-major
      const uint32_t aQ = smem_u32(sQ), aDO = smem_u32(sDO), aK = smem_u32(sK), aV = smem_u32(sV);
      bool ok = mbar_wait(bar_q, 0, abort_flag);
      int issued = 0;
      for (int u = 0; u < steps && ok; u++) {
        ok = mbar_wait(bar_kv, u & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; kk++) umma_bf16(tS, kmajor(aK, kk, 16384), kmajor(aQ, kk, 8192), idesc_s, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; kk++) umma_bf16(tP, kmajor(aV, kk, 16384), kmajor(aDO, kk, 8192), idesc_s, kk > 0);
        umma_commit(bar_s);
        issued++;
        ok = mbar_wait(bar_p, u & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; kk++)
          umma_bf16(tDQ, mnmajor(aK, kk, 16384), mnmajor(aV, kk, 8192), idesc_q, (u > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar_free);
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
    // ------------------------------------------------------------ one thread per key (lane)
    const int r = warp * 32 + lane;  // key r % 64 of the step's tile r / 64
    const int half = r >> 6, kr = r & 63;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float sl2 = rsqrtf((float)g.d) * kLog2e;
    bool ok = warp_wait(bar_q, 0, abort_flag);  // the rows' lse and D
    for (int u = 0; u < steps && ok; u++) {
      const int t = 2 * u + half;
      const int x = list[min(t, T - 1)] * 64 + kr;  // this thread's key position
      // rows that attend the key: [c_lo, c_hi); none in a padding half or past the keys;
      // in block iq itself (the last tile) only rows at or after the key
      const int c_lo = t == T - 1 ? kr : 0;
      const int c_hi = (t < T && x < g.N) ? rows : 0;
      ok = warp_wait(bar_s, u & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      float s[64], dp[64];
      tmem_ld32(tS + lane_base, s);
      tmem_ld32(tS + lane_base + 32, s + 32);
      tmem_ld32(tP + lane_base, dp);
      tmem_ld32(tP + lane_base + 32, dp + 32);
      tmem_wait_ld();
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 64; c += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(s_row + c);
        const float4 d4 = *reinterpret_cast<const float4*>(s_row + 64 + c);
        const float2 y0 = __ffma2_rn(make_float2(s[c], s[c + 1]), make_float2(sl2, sl2), make_float2(-l4.x, -l4.y));
        const float2 y1 =
            __ffma2_rn(make_float2(s[c + 2], s[c + 3]), make_float2(sl2, sl2), make_float2(-l4.z, -l4.w));
        const float e0 = (c >= c_lo && c < c_hi) ? ex2(y0.x) : 0.f;
        const float e1 = (c + 1 >= c_lo && c + 1 < c_hi) ? ex2(y0.y) : 0.f;
        const float e2 = (c + 2 >= c_lo && c + 2 < c_hi) ? ex2(y1.x) : 0.f;
        const float e3 = (c + 3 >= c_lo && c + 3 < c_hi) ? ex2(y1.y) : 0.f;
        pk[c / 2] = pack_bf16(e0 * (dp[c] - d4.x), e1 * (dp[c + 1] - d4.y));
        pk[c / 2 + 1] = pack_bf16(e2 * (dp[c + 2] - d4.z), e3 * (dp[c + 3] - d4.w));
      }
      // dS^T over the V tiles: the step's dP^T MMAs (committed with bar_s) have read them
      store_row_sw128(sV, r, pk);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p);
    }
    if (ok) ok = warp_wait(bar_dq, 0, abort_flag);
    if (ok) {
      tc_fence_after();
      float o[64];
      tmem_ld32(tDQ + lane_base, o);
      tmem_ld32(tDQ + lane_base + 32, o + 32);
      tmem_wait_ld();
      const float scale = rsqrtf((float)g.d);
      // lane r of dQ^T is feature r: column c is row p0 + c
      __nv_bfloat16* dst = dQ + ((size_t)unit * g.Nq + p0) * 128 + r;
#pragma unroll
      for (int c = 0; c < 64; c++)
        if (c < rows) dst[(size_t)c * 128] = __float2bfloat16_rn(o[c] * scale);
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

// ---------------------------------------------------------------------------- dK, dV

__global__ void __launch_bounds__(KvPairPlan::kThreads, 2)
    bwd_dkdv_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                         const float* __restrict__ lse, const float* __restrict__ delta,
                         const int32_t* __restrict__ offset, const int32_t* __restrict__ rho,
                         __nv_bfloat16* __restrict__ dK, __nv_bfloat16* __restrict__ dV, int* status, Geo g) {
  using PL = KvPairPlan;
  extern __shared__ __align__(1024) unsigned char smem[];
  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0) report(status, PYR_EINVAL);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PL::kBar);
  uint64_t* bar_kv = bars;        // the block's K and V landed
  uint64_t* bar_ld = bars + 1;    // a step's Q2, dO2 landed
  uint64_t* bar_s = bars + 2;     // S, dP of the step in tensor memory
  uint64_t* bar_p = bars + 3;     // P written (4 warps)
  uint64_t* bar_pv = bars + 4;    // the step's dV MMAs done: the buffer takes dS
  uint64_t* bar_ds = bars + 5;    // dS written (4 warps)
  uint64_t* bar_free = bars + 6;  // the step's dK MMAs done: Q2, dO2 and the buffer reusable
  uint64_t* bar_done = bars + 7;  // every MMA done
  uint64_t* bar_drain = bars + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + PL::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + PL::kMisc + 4);
  unsigned char* sK = smem + PL::kK;
  unsigned char* sV = smem + PL::kV;
  unsigned char* sQ = smem + PL::kQ;
  unsigned char* sDO = smem + PL::kDO;
  unsigned char* sPS = smem + PL::kPS;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.y;
  const int j = blockIdx.x;  // key block
  const int x0 = j * 64;
  // query blocks attending j: j itself (entry 0), then rho[offset[j] ..) (all > j, ascending)
  const int32_t* off_u = offset + (size_t)unit * (g.nb + 1);
  const int32_t* vis = rho + (size_t)unit * g.nqb * g.topk + off_u[j];
  const int T = 1 + off_u[j + 1] - off_u[j];
  const int steps = (T + 1) >> 1;
  auto qblock = [&](int t) { return t == 0 ? j : vis[t - 1]; };

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    mbar_init(bar_ld, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_p, 4);
    mbar_init(bar_pv, 1);
    mbar_init(bar_ds, 4);
    mbar_init(bar_free, 1);
    mbar_init(bar_done, 1);
    mbar_init(bar_drain, 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, PL::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tP = tmem + 64, tDV = tmem + 128, tDK = tmem + 192;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_expect_tx(bar_kv, 32768);
      for (int h = 0; h < 2; h++) {
        tma_load_3d(sK + h * 8192, &tmK, h * 64, x0, unit, bar_kv);
        tma_load_3d(sV + h * 8192, &tmV, h * 64, x0, unit, bar_kv);
      }
      int u = 0;
      for (; u < steps; u++) {
        if (u > 0 && !mbar_wait(bar_free, (u - 1) & 1, abort_flag)) break;
        mbar_expect_tx(bar_ld, 65536);
        for (int c = 0; c < 2; c++) {
          const int row0 = qblock(min(2 * u + c, T - 1)) * 64;
          for (int h = 0; h < 2; h++) {
            tma_load_3d(sQ + h * 16384 + c * 8192, &tmQ, h * 64, row0, unit, bar_ld);
            tma_load_3d(sDO + h * 16384 + c * 8192, &tmDO, h * 64, row0, unit, bar_ld);
          }
        }
      }
      volatile int no_abort = 0;
      mbar_wait(bar_kv, 0, &no_abort);
      if (u > 0) mbar_wait(bar_ld, (u - 1) & 1, &no_abort);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);  // rows x keys, both K-major
      constexpr uint32_t idesc_g = idesc_bf16_f32(128, 64, 1, 1);  // d x keys, both MN-major
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ), aDO = smem_u32(sDO);
      const uint32_t aPS = smem_u32(sPS);
      bool ok = mbar_wait(bar_kv, 0, abort_flag);
      int issued = 0;
      for (int u = 0; u < steps && ok; u++) {
        ok = mbar_wait(bar_ld, u & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; kk++) umma_bf16(tS, kmajor(aQ, kk, 16384), kmajor(aK, kk, 8192), idesc_s, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; kk++) umma_bf16(tP, kmajor(aDO, kk, 16384), kmajor(aV, kk, 8192), idesc_s, kk > 0);
        umma_commit(bar_s);
        issued++;
        ok = mbar_wait(bar_p, u & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; kk++)
          umma_bf16(tDV, mnmajor(aDO, kk, 16384), mnmajor(aPS, kk, 8192), idesc_g, (u > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar_pv);
        ok = mbar_wait(bar_ds, u & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; kk++)
          umma_bf16(tDK, mnmajor(aQ, kk, 16384), mnmajor(aPS, kk, 8192), idesc_g, (u > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar_free);
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
    // ------------------------------------------------------------ one thread per row (lane)
    const int r = warp * 32 + lane;  // row r % 64 of the step's query block r / 64
    const int half = r >> 6, rr = r & 63;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const float sl2 = rsqrtf((float)g.d) * kLog2e;
    const int keys = min(64, g.N - x0);
    bool ok = true;
    for (int u = 0; u < steps && ok; u++) {
      const int t = 2 * u + half;
      const int p = qblock(min(t, T - 1)) * 64 + rr;  // this thread's row position
      const bool in = t < T && p < g.Nq;
      // keys the row attends: [0, c_hi); in block j itself (entry 0) only keys up to the row
      const int c_hi = in ? (t == 0 ? min(keys, rr + 1) : keys) : 0;
      const size_t row = (size_t)unit * g.Nq + min(p, g.Nq - 1);
      const float lse2 = lse[row] * kLog2e, D = delta[row];
      ok = warp_wait(bar_s, u & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      float s[64], dp[64];
      tmem_ld32(tS + lane_base, s);
      tmem_ld32(tS + lane_base + 32, s + 32);
      tmem_ld32(tP + lane_base, dp);
      tmem_ld32(tP + lane_base + 32, dp + 32);
      tmem_wait_ld();
      uint32_t pk[32], dk[32];
      const float2 scl = make_float2(sl2, sl2), offs = make_float2(-lse2, -lse2), dd = make_float2(-D, -D);
#pragma unroll
      for (int c = 0; c < 32; c++) {
        const float2 y = __ffma2_rn(make_float2(s[2 * c], s[2 * c + 1]), scl, offs);
        const float e0 = 2 * c < c_hi ? ex2(y.x) : 0.f, e1 = 2 * c + 1 < c_hi ? ex2(y.y) : 0.f;
        const float2 z = __fadd2_rn(make_float2(dp[2 * c], dp[2 * c + 1]), dd);
        pk[c] = pack_bf16(e0, e1);
        dk[c] = pack_bf16(e0 * z.x, e1 * z.y);
      }
      // the buffer is free: bar_s was committed after the previous step's dK MMAs
      store_row_sw128(sPS, r, pk);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p);
      ok = warp_wait(bar_pv, u & 1, abort_flag);  // dV has read P
      if (!ok) break;
      store_row_sw128(sPS, r, dk);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_ds);
    }
    if (ok) ok = warp_wait(bar_done, 0, abort_flag);
    if (ok) {
      tc_fence_after();
      const float scale = rsqrtf((float)g.d);
      float o[64];
      for (int which = 0; which < 2; which++) {
        tmem_ld32((which ? tDK : tDV) + lane_base, o);
        tmem_ld32((which ? tDK : tDV) + lane_base + 32, o + 32);
        tmem_wait_ld();
        const float sc = which ? scale : 1.f;
        // lane r of dV^T / dK^T is feature r: column c is key x0 + c
        __nv_bfloat16* dst = (which ? dK : dV) + ((size_t)unit * g.N + x0) * 128 + r;
#pragma unroll
        for (int c = 0; c < 64; c++)
          if (c < keys) dst[(size_t)c * 128] = __float2bfloat16_rn(o[c] * sc);
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

}  // namespace

bool backward_pair_supported(const Geo& g) {
  return g.dtype == PYR_BF16 && g.d == 128 && g.b == 64 && g.G == 1 && g.q_offset == 0 && g.Nq == g.N;
}

cudaError_t launch_backward_dq_pair(const Geo& g, const CUtensorMap& mq, const CUtensorMap& mk,
                                    const CUtensorMap& mv, const CUtensorMap& mdo, const float* lse,
                                    const float* delta, const int32_t* idx, void* dQ, int* status, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       DqPairPlan::kBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(g.nqb, g.B * g.Hkv);
  bwd_dq_pair_kernel<<<grid, DqPairPlan::kThreads, DqPairPlan::kBytes, st>>>(
      mq, mk, mv, mdo, lse, delta, idx, reinterpret_cast<__nv_bfloat16*>(dQ), status, g);
  return cudaGetLastError();
}

cudaError_t launch_backward_dkdv_pair(const Geo& g, const CUtensorMap& mq, const CUtensorMap& mk,
                                      const CUtensorMap& mv, const CUtensorMap& mdo, const float* lse,
                                      const float* delta, const int32_t* offset, const int32_t* rho, void* dK,
                                      void* dV, int* status, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       KvPairPlan::kBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(g.nb, g.B * g.Hkv);
  bwd_dkdv_pair_kernel<<<grid, KvPairPlan::kThreads, KvPairPlan::kBytes, st>>>(
      mq, mk, mv, mdo, lse, delta, offset, rho, reinterpret_cast<__nv_bfloat16*>(dK),
      reinterpret_cast<__nv_bfloat16*>(dV), status, g);
  return cudaGetLastError();
}

}  // namespace pyr
