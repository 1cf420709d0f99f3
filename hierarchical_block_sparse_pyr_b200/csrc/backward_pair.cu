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
// list entries per step, and transpose the products to match, so no union is
// formed:
//
// bwd_dq_pair_kernel, per query block i: its key tiles (the accepted routes of
// row i, ascending, then block i itself), 128 keys per step:
//   S^T = K2 Q^T,  dP^T = V2 dO^T      (M = 128 keys, N = 64 rows, K = d)
//   one thread per key: P^T = exp(S^T / sqrt(d) - lse), dS^T = P^T (dP^T - D),
//   bf16, written to shared memory over the V tiles (dP^T no longer needs them)
//   dQ^T += K2^T dS^T                   (M = d, N = 64 rows, K = 128 keys)
//
// bwd_dkdv_pair_kernel, per key block j: the query blocks that attend j (j
// itself, causal, then the block-major list offset/rho, all > j), 128 rows
// per step:
//   S = Q2 K^T,  dP = dO2 V^T          (M = 128 rows, N = 64 keys, K = d)
//   one thread per row: P and dS = P (dP - D), bf16, into shared memory
//   dV^T += dO2^T P,  dK^T += Q2^T dS  (M = d, N = 64 keys, K = 128 rows)
//
// An odd list pads its last step with a second copy of its last block whose
// half is masked to zero (the operands stay finite, so 0 * operand = 0).
// Operands transposed for the second product are read from the same
// shared-memory tiles through MN-major descriptors.
//
// Both kernels are persistent, one CTA per SM, and software-pipelined across
// steps and blocks: two stages of the streamed operands (K2/V2, or Q2/dO2),
// two stages of the per-block operands, two S/dP buffers and two accumulators
// in tensor memory (512 columns). Step u's S and dP are issued while step
// u-1's gradient MMAs wait for its softmax, so the softmax of u-1 runs under
// the S and dP of u, and a block's epilogue under the next block's steps. dQ
// CTAs walk query blocks blockIdx.x + k gridDim.x (every list holds at most
// topk + 1 tiles). dK/dV lists range from one block to every later query
// block (a block that every query routes to), so dK/dV CTAs take key blocks
// from an atomic work counter, the long lists first, and the longest list
// starts at the beginning. Warps 0-7: softmax, warps w and w + 4 on
// tensor-memory lanes 32 (w % 4) .. + 31 with 32 columns each (two warps per
// scheduler, so one's tensor-memory loads overlap the other's math); warp 8:
// producer (route lists, TMA); warps 9, 10, 11: MMA issuers (dQ: S, dP, dQ;
// dK/dV: S and dP, dV, dK). A thread issues one MMA about every 65
// cycles (measured), while an N = 64 MMA runs in about 32, so a single
// issuer would leave the tensor pipe idle half the time. Every wait is
// bounded; an abort drains in-flight copies and MMAs and frees tensor memory.
#include <cudaTypedefs.h>

#include <algorithm>

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
// dQ: one persistent CTA per SM walks its query blocks w = blockIdx.x + k gridDim.x.
struct DqPairPlan {
  static constexpr int kStages = 3;     // K2/V2 stages
  static constexpr int kQ = 0;          // {Q, dO} of the current block: [2 d-halves][64 rows][128 B] each
  static constexpr int kKV = 32768;     // kStages x {K2, V2}: [2 d-halves][128 keys][128 B] each;
                                        //   dS^T [128 keys][64 rows] bf16 over the first 16 KB of V2
  static constexpr int kRow = kKV + kStages * 65536;  // 2 blocks x {lse * log2(e) [64], D [64]}
  static constexpr int kInfo = kRow + 1024;           // kStages x StepInfo
  static constexpr int kBar = kInfo + 64;
  static constexpr int kNumBars = 25;
  static constexpr int kMisc = kBar + kNumBars * 8;  // tensor-memory base, abort flag
  static constexpr int kList = kMisc + 16;          // the producer's route list
  static constexpr int kBytes = kList + kTileListPitch * 4;
  static constexpr int kThreads = 12 * 32;
  static constexpr int kTmemCols = 512;  // S^T, dP^T of 2 steps at 128 s (+64); dQ^T of 2 blocks at 256 + 64 b
};

// One step (two blocks on the M side), written by the producer before the step's copies.
struct StepInfo {
  int a, b;   // the two blocks: key blocks (dQ) or query blocks (dK, dV)
  int flags;  // kFirst / kLast (of the work item's list), kEnd (of the CTA), own / padding tiles
  int w;      // work item: unit * nqb + query block (dQ) or unit * nb + key block (dK, dV)
};
constexpr int kFirst = 1, kLast = 2, kEnd = 4, kOwnA = 8, kOwnB = 16, kPadB = 32;

// dK, dV: one persistent CTA per SM takes key blocks from a work counter, long lists first.
struct KvPairPlan {
  static constexpr int kKV = 0;        // 2 stages x {K, V}: [2 d-halves][64 keys][128 B] each
  static constexpr int kQ = 65536;     // 2 stages x {Q2, dO2}: [2 d-halves][128 rows][128 B] each
  static constexpr int kP = 196608;    // P  [128 rows][64 keys] bf16, MN-major operand
  static constexpr int kDS = 212992;   // dS [128 rows][64 keys] bf16, MN-major operand
  static constexpr int kInfo = 229376;  // 2 stages x StepInfo
  static constexpr int kBar = kInfo + 64;
  static constexpr int kNumBars = 23;
  static constexpr int kMisc = kBar + kNumBars * 8;  // tensor-memory base, abort flag, first work item
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kThreads = 12 * 32;
  static constexpr int kTmemCols = 512;  // S, dP of 2 steps at 128 s (+64); dV^T, dK^T of 2 blocks at 256 + 128 b (+64)
};
// Key blocks whose lists hold more query blocks than this are scheduled first.
constexpr int kLongList = 64;
static_assert(KvPairPlan::kBytes <= 227 * 1024, "dK/dV shared memory");
static_assert(DqPairPlan::kBytes <= 227 * 1024, "dQ shared memory");

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Half h (16-byte chunks 4h .. 4h + 3, N elements 32h .. 32h + 31) of row r of a
// [128][64] bf16 MN-major operand with 128-byte swizzle (row = the K index, 64
// contiguous N elements): chunk c of a row sits at chunk c ^ (r % 8).
__device__ __forceinline__ void store_row_half_sw128(unsigned char* base, int r, int h, const uint32_t* v) {
  unsigned char* row = base + r * 128;
#pragma unroll
  for (int c = 0; c < 4; c++)
    *reinterpret_cast<uint4*>(row + (((4 * h + c) ^ (r & 7)) << 4)) =
        make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
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

__global__ void __launch_bounds__(DqPairPlan::kThreads, 1)
    bwd_dq_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                       const float* __restrict__ lse, const float* __restrict__ delta,
                       const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ dQ, int* status, Geo g) {
  using PL = DqPairPlan;
  constexpr int NS = PL::kStages;
  extern __shared__ __align__(1024) unsigned char smem[];
  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0) report(status, PYR_EINVAL);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PL::kBar);
  uint64_t* q_full = bars;              // a block's Q, dO landed
  uint64_t* q_free = bars + 1;          // the block's last S^T, dP^T MMAs done (2 issuers)
  uint64_t* row_full = bars + 2;        // [2] a block's lse, D written
  uint64_t* row_free = bars + 4;        // [2] ... read (8 softmax warps)
  uint64_t* kv_full = bars + 6;         // [NS] a step's K2, V2 landed, its StepInfo written
  uint64_t* kv_free = kv_full + NS;     // [NS] the step's dQ MMAs done: K2, V2 and dS^T reusable
  uint64_t* s_full = kv_free + NS;      // [2] S^T, dP^T of a step in tensor memory (2 issuers)
  uint64_t* s_free = s_full + 2;        // [2] ... read into registers (8 softmax warps)
  uint64_t* p_full = s_free + 2;        // [2] dS^T of a step written (8 softmax warps)
  uint64_t* dq_full = p_full + 2;       // [2] a block's dQ^T complete
  uint64_t* dq_free = dq_full + 2;      // [2] ... read into registers (8 softmax warps)
  uint64_t* bar_drain = dq_free + 2;    // [3] each issuer's MMAs done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + PL::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + PL::kMisc + 4);
  StepInfo* info = reinterpret_cast<StepInfo*>(smem + PL::kInfo);
  int* list = reinterpret_cast<int*>(smem + PL::kList);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = g.nqb * g.B * g.Hkv;  // work items: (unit, query block)

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_free, 2);
    for (int s = 0; s < 2; s++) {
      mbar_init(row_full + s, 1);
      mbar_init(row_free + s, 8);
      mbar_init(s_full + s, 2);
      mbar_init(s_free + s, 8);
      mbar_init(p_full + s, 8);
      mbar_init(dq_full + s, 1);
      mbar_init(dq_free + s, 8);
    }
    for (int s = 0; s < NS; s++) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_free + s, 1);
    }
    for (int k = 0; k < 3; k++) mbar_init(bar_drain + k, 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, PL::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    int u = 0, nq = 0;  // steps and blocks whose copies were issued
    bool ok = true;
    // a block's idx row and its rows' lse and D, loaded one block ahead into registers
    int nidx[4];
    float nl[2], nd[2];
    auto fetch = [&](int w) {
      if (w >= total) return;
      const int32_t* row = idx + (size_t)w * g.topk;
#pragma unroll
      for (int c = 0; c < 4; c++) nidx[c] = 32 * c + lane < g.topk ? row[32 * c + lane] : -1;
      const int unit = w / g.nqb, p0 = (g.i0 + w % g.nqb) * 64 - g.q_offset, rows = min(64, g.Nq - p0);
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const int e = lane + 32 * h;
        const size_t r = (size_t)unit * g.Nq + p0 + min(e, rows - 1);
        nl[h] = e < rows ? lse[r] * kLog2e : 0.f;
        nd[h] = e < rows ? delta[r] : 0.f;
      }
    };
    fetch(blockIdx.x);
    for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
      const int unit = w / g.nqb, iq = g.i0 + w % g.nqb;
      const int p0 = iq * 64 - g.q_offset;
      const int rs = nq & 1;
      if (nq >= 2) {
        bool f = true;
        if (lane == 0) f = mbar_wait(row_free + rs, ((nq >> 1) - 1) & 1, abort_flag);
        ok = __shfl_sync(0xffffffffu, f, 0);
        if (!ok) break;
      }
      // key tiles: accepted routes, ascending, then block iq
      const int T = compact_route_row_with([&](int c) { return nidx[c]; }, g.topk, iq, list, status);
      float* s_row = reinterpret_cast<float*>(smem + PL::kRow + rs * 512);
      s_row[lane] = nl[0];
      s_row[lane + 32] = nl[1];
      s_row[64 + lane] = nd[0];
      s_row[96 + lane] = nd[1];
      __syncwarp();
      fetch(w + (int)gridDim.x);  // in flight while this block's copies are issued
      const int steps = (T + 1) >> 1;
      const bool last_w = w + (int)gridDim.x >= total;
      if (lane == 0) {
        mbar_arrive(row_full + rs);
        for (int t = 0; t < steps; t++, u++) {
          const int s = u % NS;
          if (u >= NS && !mbar_wait(kv_free + s, ((u / NS) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const int ta = 2 * t, tb = 2 * t + 1;
          StepInfo si;
          si.a = list[ta];
          si.b = list[min(tb, T - 1)];
          si.w = w;
          si.flags = (t == 0 ? kFirst : 0) | (t == steps - 1 ? kLast : 0) | (t == steps - 1 && last_w ? kEnd : 0) |
                     (ta == T - 1 ? kOwnA : 0) | (tb == T - 1 ? kOwnB : 0) | (tb >= T ? kPadB : 0);
          info[s] = si;
          unsigned char* skv = smem + PL::kKV + s * 65536;
          mbar_expect_tx(kv_full + s, 65536);
          for (int c = 0; c < 2; c++) {
            const int key0 = (c ? si.b : si.a) * 64;
            for (int h = 0; h < 2; h++) {
              tma_load_3d(skv + h * 16384 + c * 8192, &tmK, h * 64, key0, unit, kv_full + s);
              tma_load_3d(skv + 32768 + h * 16384 + c * 8192, &tmV, h * 64, key0, unit, kv_full + s);
            }
          }
          if (t == 0) {
            // Q, dO after the first step's tiles: the previous block's last S^T, dP^T must be done
            if (nq >= 1 && !mbar_wait(q_free, (nq - 1) & 1, abort_flag)) {
              ok = false;
              u++;
              break;
            }
            mbar_expect_tx(q_full, 32768);
            for (int h = 0; h < 2; h++) {
              tma_load_3d(smem + PL::kQ + h * 8192, &tmQ, h * 64, p0, unit, q_full);
              tma_load_3d(smem + PL::kQ + 16384 + h * 8192, &tmDO, h * 64, p0, unit, q_full);
            }
            nq++;
            // the next block's Q and dO (first read here, so from DRAM) into L2: its load waits for
            // this block's last S^T, dP^T and then stalls the next block's first step
            if (!last_w) {
              const int wn = w + (int)gridDim.x;
              const int pn = (g.i0 + wn % g.nqb) * 64 - g.q_offset;
              for (int h = 0; h < 2; h++) {
                tma_prefetch_3d(&tmQ, h * 64, pn, wn / g.nqb);
                tma_prefetch_3d(&tmDO, h * 64, pn, wn / g.nqb);
              }
            }
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      u = __shfl_sync(0xffffffffu, u, 0);
      nq = __shfl_sync(0xffffffffu, nq, 0);
    }
    // copies still in flight land before the CTA can exit
    if (lane == 0) {
      volatile int no_abort = 0;
      for (int v = max(0, u - NS); v < u; v++) mbar_wait(kv_full + (v % NS), (v / NS) & 1, &no_abort);
      if (nq > 0) mbar_wait(q_full, (nq - 1) & 1, &no_abort);
    }
    __syncwarp();
  } else if (warp == 9 || warp == 10) {
    // ------------------------------------------------------------ S^T (warp 9) and dP^T (warp 10) issuers
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);  // keys x rows, both K-major
      const bool is_s = warp == 9;
      const uint32_t a0 = smem_u32(smem), aB = a0 + PL::kQ + (is_s ? 0 : 16384);  // Q or dO
      int issued = 0, u = 0, n = 0;
      while (true) {
        const int s = u % NS;
        if (!mbar_wait(kv_full + s, (u / NS) & 1, abort_flag)) break;
        const int flags = info[s].flags;
        if ((flags & kFirst) && !mbar_wait(q_full, n & 1, abort_flag)) break;
        if (u >= 2 && !mbar_wait(s_free + (u & 1), ((u >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t aA = a0 + PL::kKV + s * 65536 + (is_s ? 0 : 32768);  // K2 or V2
        const uint32_t tD = tmem + (u & 1) * 128 + (is_s ? 0 : 64);
#pragma unroll
        for (int kk = 0; kk < 8; kk++) umma_bf16(tD, kmajor(aA, kk, 16384), kmajor(aB, kk, 8192), idesc_s, kk > 0);
        umma_commit(s_full + (u & 1));
        issued++;
        if (flags & kLast) {
          umma_commit(q_free);
          n++;
        }
        if (flags & kEnd) break;
        u++;
      }
      if (issued > 0) {
        umma_commit(bar_drain + warp - 9);
        volatile int no_abort = 0;
        mbar_wait(bar_drain + warp - 9, 0, &no_abort);
      }
    }
    __syncwarp();
  } else if (warp == 11) {
    // ------------------------------------------------------------ dQ issuer
    if (lane == 0) {
      constexpr uint32_t idesc_q = idesc_bf16_f32(128, 64, 1, 1);  // d x rows, both MN-major
      const uint32_t a0 = smem_u32(smem);
      int issued = 0, u = 0, n = 0;
      while (true) {
        const int s = u % NS, b = n & 1;
        // the step's StepInfo (its stage is refilled only after this thread's kv_free commit)
        if (!mbar_wait(kv_full + s, (u / NS) & 1, abort_flag)) break;
        const int flags = info[s].flags;
        if (!mbar_wait(p_full + (u & 1), (u >> 1) & 1, abort_flag)) break;
        if ((flags & kFirst) && n >= 2 && !mbar_wait(dq_free + b, ((n >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        // dQ^T of the block += K2^T dS^T of the step
        const uint32_t aK = a0 + PL::kKV + s * 65536, aDS = aK + 32768;
        const uint32_t tDQ = tmem + 256 + b * 64;
#pragma unroll
        for (int kk = 0; kk < 8; kk++)
          umma_bf16(tDQ, mnmajor(aK, kk, 16384), mnmajor(aDS, kk, 8192), idesc_q,
                    ((flags & kFirst) && kk == 0) ? 0u : 1u);
        umma_commit(kv_free + s);
        issued++;
        if (flags & kLast) {
          umma_commit(dq_full + b);
          n++;
        }
        if (flags & kEnd) break;
        u++;
      }
      if (issued > 0) {
        umma_commit(bar_drain + 2);
        volatile int no_abort = 0;
        mbar_wait(bar_drain + 2, 0, &no_abort);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax: warps w and w + 4 share
    // tensor-memory lanes 32 (w % 4) .. + 31 (one key each) and take columns (rows) 0-31 / 32-63
    const int q4 = warp & 3, c0 = (warp >> 2) * 32;
    const int r = q4 * 32 + lane;  // key r % 64 of the step's tile r / 64
    const int half = r >> 6, kr = r & 63;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const float sl2 = rsqrtf((float)g.d) * kLog2e, scale = rsqrtf((float)g.d);
    int u = 0, n = 0;
    while (true) {
      const int s = u % NS, b = n & 1;
      if (!warp_wait(kv_full + s, (u / NS) & 1, abort_flag)) break;  // the step's StepInfo
      const StepInfo si = info[s];
      if ((si.flags & kFirst) && !warp_wait(row_full + b, (n >> 1) & 1, abort_flag)) break;  // lse, D
      if (!warp_wait(s_full + (u & 1), (u >> 1) & 1, abort_flag)) break;
      tc_fence_after();
      float sv[32], dp[32];
      const uint32_t tS = tmem + (u & 1) * 128 + lane_base + c0;
      tmem_ld32(tS, sv);
      tmem_ld32(tS + 64, dp);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free + (u & 1));
      const int unit = si.w / g.nqb;
      const int p0 = (g.i0 + si.w % g.nqb) * 64 - g.q_offset, rows = min(64, g.Nq - p0);
      const int x = (half ? si.b : si.a) * 64 + kr;  // this thread's key position
      // rows that attend the key: [c_lo, c_hi) (columns c0 + c); none in a padding half or past the
      // keys; in the block's own tile only rows at or after the key
      const int c_lo = ((si.flags & (half ? kOwnB : kOwnA)) ? kr : 0) - c0;
      const int c_hi = (((half && (si.flags & kPadB)) || x >= g.N) ? 0 : rows) - c0;
      const float* s_row = reinterpret_cast<const float*>(smem + PL::kRow + b * 512) + c0;
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 32; c += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(s_row + c);
        const float4 d4 = *reinterpret_cast<const float4*>(s_row + 64 + c);
        const float2 y0 = __ffma2_rn(make_float2(sv[c], sv[c + 1]), make_float2(sl2, sl2), make_float2(-l4.x, -l4.y));
        const float2 y1 =
            __ffma2_rn(make_float2(sv[c + 2], sv[c + 3]), make_float2(sl2, sl2), make_float2(-l4.z, -l4.w));
        const float e0 = (c >= c_lo && c < c_hi) ? ex2(y0.x) : 0.f;
        const float e1 = (c + 1 >= c_lo && c + 1 < c_hi) ? ex2(y0.y) : 0.f;
        const float e2 = (c + 2 >= c_lo && c + 2 < c_hi) ? ex2(y1.x) : 0.f;
        const float e3 = (c + 3 >= c_lo && c + 3 < c_hi) ? ex2(y1.y) : 0.f;
        pk[c / 2] = pack_bf16(e0 * (dp[c] - d4.x), e1 * (dp[c + 1] - d4.y));
        pk[c / 2 + 1] = pack_bf16(e2 * (dp[c + 2] - d4.z), e3 * (dp[c + 3] - d4.w));
      }
      // dS^T over the V tiles: the step's dP^T MMAs (committed with s_full) have read them
      store_row_half_sw128(smem + PL::kKV + s * 65536 + 32768, r, c0 >> 5, pk);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + (u & 1));
      if (si.flags & kLast) {
        if (lane == 0) mbar_arrive(row_free + b);  // the block's lse and D are read
        if (!warp_wait(dq_full + b, (n >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        float o[32];
        tmem_ld32(tmem + 256 + b * 64 + lane_base + c0, o);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dq_free + b);
        // lane r of dQ^T is feature r: column c0 + c is row p0 + c0 + c
        __nv_bfloat16* dst = dQ + ((size_t)unit * g.Nq + p0 + c0) * 128 + r;
#pragma unroll
        for (int c = 0; c < 32; c++)
          if (c0 + c < rows) dst[(size_t)c * 128] = __float2bfloat16_rn(o[c] * scale);
        n++;
      }
      if (si.flags & kEnd) break;
      u++;
    }
  }

  // ---- teardown ----
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) report(status, PYR_ETIMEOUT);
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, PL::kTmemCols);
  }
}

// ---------------------------------------------------------------------------- dK, dV

// Work order of the dK/dV kernel: items (unit * nb + key block) whose list is
// longer than kLongList go to `list` first (any order: each item's result does
// not depend on when it runs); ctr[0] counts them, ctr[1] is the work counter.
__global__ void bwd_long_items_kernel(const int32_t* __restrict__ offset, int* ctr, int* list, Geo g) {
  const int total = g.nb * g.B * g.Hkv;
  for (int w = blockIdx.x * blockDim.x + threadIdx.x; w < total; w += gridDim.x * blockDim.x) {
    const int32_t* off = offset + (size_t)(w / g.nb) * (g.nb + 1) + w % g.nb;
    if (off[1] - off[0] + 1 > kLongList) list[atomicAdd(ctr, 1)] = w;
  }
}

// The next work item of the calling CTA, or -1: long items first, then the
// others in index order.
__device__ __forceinline__ int grab_item(int* ctr, const int* list, const int32_t* __restrict__ offset, const Geo& g) {
  const int total = g.nb * g.B * g.Hkv, nlong = ctr[0];
  for (;;) {
    const int t = atomicAdd(ctr + 1, 1);
    if (t < nlong) return list[t];
    const int w = t - nlong;
    if (w >= total) return -1;
    const int32_t* off = offset + (size_t)(w / g.nb) * (g.nb + 1) + w % g.nb;
    if (off[1] - off[0] + 1 <= kLongList) return w;
  }
}

__global__ void __launch_bounds__(KvPairPlan::kThreads, 1)
    bwd_dkdv_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                         const float* __restrict__ lse, const float* __restrict__ delta,
                         const int32_t* __restrict__ offset, const int32_t* __restrict__ rho, int* ctr,
                         const int* long_list, __nv_bfloat16* __restrict__ dK, __nv_bfloat16* __restrict__ dV,
                         int* status, Geo g) {
  using PL = KvPairPlan;
  extern __shared__ __align__(1024) unsigned char smem[];
  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0) report(status, PYR_EINVAL);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PL::kBar);
  uint64_t* kv_full = bars;        // [2] a key block's K, V landed
  uint64_t* kv_free = bars + 2;    // [2] its last S, dP MMAs done
  uint64_t* ld_full = bars + 4;    // [2] a step's Q2, dO2 landed, its StepInfo written
  uint64_t* ld_free = bars + 6;    // [2] the step's dV and dK MMAs done (2 issuers): Q2, dO2 reusable
  uint64_t* s_full = bars + 8;     // [2] S, dP of a step in tensor memory
  uint64_t* s_free = bars + 10;    // [2] ... read into registers (8 softmax warps)
  uint64_t* acc_full = bars + 12;  // [2] a key block's dV^T, dK^T complete (2 issuers)
  uint64_t* acc_free = bars + 14;  // [2] ... read into registers (8 softmax warps)
  uint64_t* p_full = bars + 16;    // P written (8 softmax warps)
  uint64_t* p_free = bars + 17;    // the dV MMAs that read P done
  uint64_t* ds_full = bars + 18;   // dS written (8 softmax warps)
  uint64_t* ds_free = bars + 19;   // the dK MMAs that read dS done
  uint64_t* bar_drain = bars + 20;  // [3] each issuer's MMAs done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + PL::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + PL::kMisc + 4);
  int* first_item = reinterpret_cast<int*>(smem + PL::kMisc + 8);
  StepInfo* info = reinterpret_cast<StepInfo*>(smem + PL::kInfo);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; s++) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_free + s, 1);
      mbar_init(ld_full + s, 1);
      mbar_init(ld_free + s, 2);
      mbar_init(s_full + s, 1);
      mbar_init(s_free + s, 8);
      mbar_init(acc_full + s, 2);
      mbar_init(acc_free + s, 8);
    }
    mbar_init(p_full, 8);
    mbar_init(p_free, 1);
    mbar_init(ds_full, 8);
    mbar_init(ds_free, 1);
    for (int k = 0; k < 3; k++) mbar_init(bar_drain + k, 1);
    fence_mbar_init();
    *abort_flag = 0;
    *first_item = grab_item(ctr, long_list, offset, g);
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, PL::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool has_work = *first_item >= 0;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int u = 0, n = 0;  // steps and key blocks whose copies were issued
      bool ok = true;
      int item = *first_item;
      while (item >= 0 && ok) {
        const int next = grab_item(ctr, long_list, offset, g);
        const int unit = item / g.nb, j = item % g.nb;
        const int32_t* off = offset + (size_t)unit * (g.nb + 1) + j;
        const int32_t* vis = rho + (size_t)unit * g.nqb * g.topk + off[0];
        const int T = 1 + off[1] - off[0];  // j itself, then the query blocks that route to j
        const int ks = n & 1;
        if (n >= 2 && !(ok = mbar_wait(kv_free + ks, ((n >> 1) - 1) & 1, abort_flag))) break;
        unsigned char* skv = smem + PL::kKV + ks * 32768;
        mbar_expect_tx(kv_full + ks, 32768);
        for (int h = 0; h < 2; h++) {
          tma_load_3d(skv + h * 8192, &tmK, h * 64, j * 64, unit, kv_full + ks);
          tma_load_3d(skv + 16384 + h * 8192, &tmV, h * 64, j * 64, unit, kv_full + ks);
        }
        n++;
        const int steps = (T + 1) >> 1;
        for (int t = 0; t < steps; t++, u++) {
          const int s = u & 1;
          if (u >= 2 && !(ok = mbar_wait(ld_free + s, ((u >> 1) - 1) & 1, abort_flag))) break;
          const int ta = 2 * t, tb = 2 * t + 1;
          StepInfo si;
          si.a = ta == 0 ? j : vis[ta - 1];
          si.b = tb < T ? vis[tb - 1] : si.a;
          si.w = item;
          si.flags = (t == 0 ? kFirst : 0) | (t == steps - 1 ? kLast : 0) | (t == steps - 1 && next < 0 ? kEnd : 0) |
                     (ta == 0 ? kOwnA : 0) | (tb >= T ? kPadB : 0);
          info[s] = si;
          unsigned char* sq = smem + PL::kQ + s * 65536;
          mbar_expect_tx(ld_full + s, 65536);
          for (int c = 0; c < 2; c++) {
            const int row0 = (c ? si.b : si.a) * 64;
            for (int h = 0; h < 2; h++) {
              tma_load_3d(sq + h * 16384 + c * 8192, &tmQ, h * 64, row0, unit, ld_full + s);
              tma_load_3d(sq + 32768 + h * 16384 + c * 8192, &tmDO, h * 64, row0, unit, ld_full + s);
            }
          }
        }
        item = next;
      }
      // copies still in flight land before the CTA can exit
      volatile int no_abort = 0;
      for (int v = max(0, u - 2); v < u; v++) mbar_wait(ld_full + (v & 1), (v >> 1) & 1, &no_abort);
      for (int m = max(0, n - 2); m < n; m++) mbar_wait(kv_full + (m & 1), (m >> 1) & 1, &no_abort);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ S, dP issuer
    if (lane == 0 && has_work) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);  // rows x keys, both K-major
      const uint32_t a0 = smem_u32(smem);
      int issued = 0, u = 0, n = 0;
      while (true) {
        const int s = u & 1, ks = n & 1;
        if (!mbar_wait(ld_full + s, (u >> 1) & 1, abort_flag)) break;
        const int flags = info[s].flags;
        if ((flags & kFirst) && !mbar_wait(kv_full + ks, (n >> 1) & 1, abort_flag)) break;
        if (u >= 2 && !mbar_wait(s_free + s, ((u >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t aQ = a0 + PL::kQ + s * 65536, aDO = aQ + 32768;
        const uint32_t aK = a0 + PL::kKV + ks * 32768, aV = aK + 16384;
        const uint32_t tS = tmem + s * 128, tP = tS + 64;
#pragma unroll
        for (int kk = 0; kk < 8; kk++) umma_bf16(tS, kmajor(aQ, kk, 16384), kmajor(aK, kk, 8192), idesc_s, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; kk++) umma_bf16(tP, kmajor(aDO, kk, 16384), kmajor(aV, kk, 8192), idesc_s, kk > 0);
        umma_commit(s_full + s);
        issued++;
        if (flags & kLast) {
          umma_commit(kv_free + ks);
          n++;
        }
        if (flags & kEnd) break;
        u++;
      }
      if (issued > 0) {
        umma_commit(bar_drain);
        volatile int no_abort = 0;
        mbar_wait(bar_drain, 0, &no_abort);
      }
    }
    __syncwarp();
  } else if (warp == 10 || warp == 11) {
    // ------------------------------------------------------------ dV (warp 10) and dK (warp 11) issuers
    if (lane == 0 && has_work) {
      constexpr uint32_t idesc_g = idesc_bf16_f32(128, 64, 1, 1);  // d x keys, both MN-major
      const bool is_v = warp == 10;
      uint64_t* in_full = is_v ? p_full : ds_full;    // P or dS written
      uint64_t* in_free = is_v ? p_free : ds_free;    // ... read by this issuer's MMAs
      const uint32_t a0 = smem_u32(smem), aB = a0 + (is_v ? PL::kP : PL::kDS);
      int issued = 0, u = 0, n = 0;
      while (true) {
        const int s = u & 1, b = n & 1;
        // the step's StepInfo (its stage is refilled only after this thread's ld_free commit)
        if (!mbar_wait(ld_full + s, (u >> 1) & 1, abort_flag)) break;
        const int flags = info[s].flags;
        if (!mbar_wait(in_full, u & 1, abort_flag)) break;
        if ((flags & kFirst) && n >= 2 && !mbar_wait(acc_free + b, ((n >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        // dV^T += dO2^T P, or dK^T += Q2^T dS, of the key block
        const uint32_t aA = a0 + PL::kQ + s * 65536 + (is_v ? 32768 : 0);
        const uint32_t tD = tmem + 256 + b * 128 + (is_v ? 0 : 64);
#pragma unroll
        for (int kk = 0; kk < 8; kk++)
          umma_bf16(tD, mnmajor(aA, kk, 16384), mnmajor(aB, kk, 8192), idesc_g, ((flags & kFirst) && kk == 0) ? 0u : 1u);
        umma_commit(in_free);
        // Q2, dO2 reusable once both issuers are done: this step's S and dP were complete
        // before its softmax wrote P
        umma_commit(ld_free + s);
        issued++;
        if (flags & kLast) {
          umma_commit(acc_full + b);
          n++;
        }
        if (flags & kEnd) break;
        u++;
      }
      if (issued > 0) {
        umma_commit(bar_drain + warp - 9);
        volatile int no_abort = 0;
        mbar_wait(bar_drain + warp - 9, 0, &no_abort);
      }
    }
    __syncwarp();
  } else if (has_work) {
    // ------------------------------------------------------------ softmax: warps w and w + 4 share
    // tensor-memory lanes 32 (w % 4) .. + 31 (one row each) and take columns (keys) 0-31 / 32-63
    const int q4 = warp & 3, c0 = (warp >> 2) * 32;
    const int r = q4 * 32 + lane;  // row r % 64 of the step's query block r / 64
    const int half = r >> 6, rr = r & 63;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const float sl2 = rsqrtf((float)g.d) * kLog2e, scale = rsqrtf((float)g.d);
    int u = 0, n = 0;
    while (true) {
      const int s = u & 1, b = n & 1;
      if (!warp_wait(ld_full + s, (u >> 1) & 1, abort_flag)) break;  // the step's StepInfo
      const StepInfo si = info[s];
      const int unit = si.w / g.nb, x0 = (si.w % g.nb) * 64, keys = min(64, g.N - x0);
      const int p = (half ? si.b : si.a) * 64 + rr;  // this thread's row position
      // keys the row attends: [0, c_hi) (columns c0 + c); none in a padding half or past the rows;
      // in the key block's own query block only keys up to the row
      const bool in = !(half && (si.flags & kPadB)) && p < g.Nq;
      const int c_hi = (in ? ((!half && (si.flags & kOwnA)) ? min(keys, rr + 1) : keys) : 0) - c0;
      const size_t row = (size_t)unit * g.Nq + min(p, g.Nq - 1);
      const float lse2 = lse[row] * kLog2e, D = delta[row];
      if (!warp_wait(s_full + s, (u >> 1) & 1, abort_flag)) break;
      tc_fence_after();
      float sv[32], dp[32];
      const uint32_t tS = tmem + s * 128 + lane_base + c0;
      tmem_ld32(tS, sv);
      tmem_ld32(tS + 64, dp);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free + s);
      uint32_t pk[16], dk[16];
      const float2 scl = make_float2(sl2, sl2), offs = make_float2(-lse2, -lse2), dd = make_float2(-D, -D);
#pragma unroll
      for (int c = 0; c < 16; c++) {
        const float2 y = __ffma2_rn(make_float2(sv[2 * c], sv[2 * c + 1]), scl, offs);
        const float e0 = 2 * c < c_hi ? ex2(y.x) : 0.f, e1 = 2 * c + 1 < c_hi ? ex2(y.y) : 0.f;
        const float2 z = __fadd2_rn(make_float2(dp[2 * c], dp[2 * c + 1]), dd);
        pk[c] = pack_bf16(e0, e1);
        dk[c] = pack_bf16(e0 * z.x, e1 * z.y);
      }
      if (u >= 1 && !warp_wait(p_free, (u - 1) & 1, abort_flag)) break;  // the previous dV MMAs read P
      store_row_half_sw128(smem + PL::kP, r, c0 >> 5, pk);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      if (u >= 1 && !warp_wait(ds_free, (u - 1) & 1, abort_flag)) break;  // the previous dK MMAs read dS
      store_row_half_sw128(smem + PL::kDS, r, c0 >> 5, dk);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_full);
      if (si.flags & kLast) {
        if (!warp_wait(acc_full + b, (n >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        // lane r of dV^T / dK^T is feature r: column c0 + c is key x0 + c0 + c
        const uint32_t tDV = tmem + 256 + b * 128 + lane_base + c0;
        float o[32];
        tmem_ld32(tDV, o);
        tmem_wait_ld();
        __nv_bfloat16* dst = dV + ((size_t)unit * g.N + x0 + c0) * 128 + r;
#pragma unroll
        for (int c = 0; c < 32; c++)
          if (c0 + c < keys) dst[(size_t)c * 128] = __float2bfloat16_rn(o[c]);
        tmem_ld32(tDV + 64, o);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_free + b);
        dst = dK + ((size_t)unit * g.N + x0 + c0) * 128 + r;
#pragma unroll
        for (int c = 0; c < 32; c++)
          if (c0 + c < keys) dst[(size_t)c * 128] = __float2bfloat16_rn(o[c] * scale);
        n++;
      }
      if (si.flags & kEnd) break;
      u++;
    }
  }

  // ---- teardown ----
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) report(status, PYR_ETIMEOUT);
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, PL::kTmemCols);
  }
}

}  // namespace

bool backward_pair_supported(const Geo& g) {
  return g.dtype == PYR_BF16 && g.d == 128 && g.b == 64 && g.G == 1 && g.q_offset == 0 && g.Nq == g.N &&
         g.topk <= 128;
}

cudaError_t launch_backward_dq_pair(const Geo& g, const CUtensorMap& mq, const CUtensorMap& mk,
                                    const CUtensorMap& mv, const CUtensorMap& mdo, const float* lse,
                                    const float* delta, const int32_t* idx, void* dQ, int* status, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       DqPairPlan::kBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int total = g.nqb * g.B * g.Hkv;  // persistent: one CTA per SM walks its share of the query blocks
  bwd_dq_pair_kernel<<<std::min(total, sms), DqPairPlan::kThreads, DqPairPlan::kBytes, st>>>(
      mq, mk, mv, mdo, lse, delta, idx, reinterpret_cast<__nv_bfloat16*>(dQ), status, g);
  return cudaGetLastError();
}

cudaError_t launch_backward_dkdv_pair(const Geo& g, const CUtensorMap& mq, const CUtensorMap& mk,
                                      const CUtensorMap& mv, const CUtensorMap& mdo, const float* lse,
                                      const float* delta, const int32_t* offset, const int32_t* rho, void* dK,
                                      void* dV, void* scratch, int* status, cudaStream_t st) {
  // scratch (>= 8 + 4 * items bytes, free until this kernel ends): the work counters, then the long items
  int* ctr = static_cast<int*>(scratch);
  int* list = ctr + 2;
  const int total = g.nb * g.B * g.Hkv;
  cudaError_t e = cudaMemsetAsync(ctr, 0, 2 * sizeof(int), st);
  if (e != cudaSuccess) return e;
  bwd_long_items_kernel<<<std::min((total + 255) / 256, 1024), 256, 0, st>>>(offset, ctr, list, g);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dkdv_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, KvPairPlan::kBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  bwd_dkdv_pair_kernel<<<std::min(total, sms), KvPairPlan::kThreads, KvPairPlan::kBytes, st>>>(
      mq, mk, mv, mdo, lse, delta, offset, rho, ctr, list, reinterpret_cast<__nv_bfloat16*>(dK),
      reinterpret_cast<__nv_bfloat16*>(dV), status, g);
  return cudaGetLastError();
}

}  // namespace pyr
