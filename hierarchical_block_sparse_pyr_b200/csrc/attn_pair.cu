// Causal block-sparse attention for 64-row query blocks of one head (MHA,
// b = 64) on the tcgen05 tensor cores: two query blocks per CTA, each walking
// its own key-block list (PHBA 3.1 / A.1.3: the routed blocks plus the
// block's own, one online softmax, output and log-sum-exp).
//
// A 128-row tile over the union of two blocks' routes (the general kernel)
// spends MMAs and softmax steps on every block that either one routes: for
// independent routes the union is ~1.8x one block's list. Here the two blocks
// are two M = 64 halves that advance in lockstep over their OWN lists: step k
// takes the k-th entry of each list. The halves share the tensor-memory
// columns and use the two halves of every 32-lane TMEM sub-partition: an
// M = 64 accumulator occupies lanes 0..15 of each sub-partition, and a second
// one at lane offset 16 fills lanes 16..31. So one softmax warp (32 lanes)
// reads the same columns for 16 rows of block A (lanes 0..15) and 16 rows of
// block B (lanes 16..31) with one load.
//   S slot sb (columns 64 sb .. 64 sb + 63): S_A at lane offset 0, S_B at 16;
//   O (columns 128..255): O_A at lane offset 0, O_B at 16.
//   P_A goes back into tensor memory over S_A and feeds the P.V MMA from there
//   (A operand in TMEM, at the same lanes as its accumulator); P_B goes to
//   shared memory (a 128B-swizzled K-major operand) and feeds an SS MMA.
// Routed attention only: dense attention (every block for both query blocks)
// keeps the general kernel, whose union is then exactly one block list. With
// PHBA prefix states (M > 0, a multiple of 64; PHBA summary 3.3 and A.1.3:
// one softmax over tokens and state slots) each half's state tiles follow its
// token tiles: every entry j >= 1 of its list brings the M-slot state stored
// before block j (its own block's state for the diagonal, the aligned state
// for a routed block) as M / 64 tiles with no mask; block 0 has no state.
// Warp roles (as in the general kernel): warps 0..3 softmax, one thread per
// row (lanes 0..15 of warp w: rows 16w .. 16w + 15 of A; lanes 16..31: the
// same rows of B); warp 4 TMA producer of Q and of the step's
// K tiles (one per half); warp 5 MMA issuer; warp 6 TMA producer of the step's
// V tiles. Every mbarrier wait is bounded; a wait that runs out aborts the CTA
// (PYR_ETIMEOUT), which still drains its copies and MMAs and frees its tensor
// memory before it exits.
#include <cudaTypedefs.h>

#include "pyr_common.cuh"
#include "tc_util.cuh"
#include "tile_list.cuh"

namespace pyr {

namespace {

using namespace tc;

constexpr int kKeys = 64;           // keys per tile = rows per query block
constexpr float kRescale = 8.0f;    // lazy rescale threshold (log2 units)
constexpr int kThreads = 7 * 32;
constexpr uint32_t kHalfB = 16u << 16;  // TMEM lane offset of block B's accumulators

struct PairPlan {
  static constexpr int kQ = 0;              // [2 d-halves][128 rows][128 B]: rows 0-63 block A, 64-127 block B
  static constexpr int kK = kQ + 32768;     // [A, B][2 d-halves][64 keys][128 B]
  static constexpr int kV = kK + 32768;     // same
  static constexpr int kPB = kV + 32768;    // P of block B: [64 rows][64 keys] bf16, 128B-swizzled, K-major
  static constexpr int kBar = kPB + 8192;
  static constexpr int kNumBars = 14;       // q, k full/free, v full/free, s_full[2], p_full[2], pb_free, o, done, drain
  static constexpr int kMisc = kBar + kNumBars * 8;  // tmem slot, abort flag
  static constexpr int kLists = kMisc + 16;          // the two route lists (compact_routes scratch)
  static constexpr int kEnd = kLists + kTileListScratch * 4;
  static constexpr int kBytes = kEnd + 1024;  // + alignment slack
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <bool kStates>  // PHBA state tiles after the token tiles (M > 0)
__global__ void __launch_bounds__(kThreads, 2)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ idx,
                     __nv_bfloat16* __restrict__ O, float* __restrict__ lse, int* status, Geo g,
                     const __grid_constant__ CUtensorMap tmPK, const __grid_constant__ CUtensorMap tmPV, int M) {
  using PL = PairPlan;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_align<1024>(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PL::kBar);
  uint64_t* bar_q = bars;
  uint64_t* bar_k_full = bars + 1;
  uint64_t* bar_k_free = bars + 2;
  uint64_t* bar_v_full = bars + 3;
  uint64_t* bar_v_free = bars + 4;
  uint64_t* bar_s_full = bars + 5;  // [2]
  uint64_t* bar_p_full = bars + 7;  // [2]
  uint64_t* bar_pb_free = bars + 9;
  uint64_t* bar_o = bars + 10;
  uint64_t* bar_done = bars + 11;
  uint64_t* bar_drain = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + PL::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + PL::kMisc + 4);
  int* lists = reinterpret_cast<int*>(smem + PL::kLists);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.y;
  const int bi = unit / g.Hkv, hk = unit % g.Hkv;
  const int head = bi * g.Hq + hk;  // one query head per kv head
  const int i_first = g.i0 + 2 * blockIdx.x;
  const int nq_here = min(2, g.nqb - 2 * blockIdx.x);

  if (threadIdx.x == 0) {
    for (int b = 0; b < PL::kNumBars; b++) mbar_init(bars + b, b == 7 || b == 8 ? 4 : 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  compact_routes(idx + ((size_t)unit * g.nqb + 2 * blockIdx.x) * g.topk, g.topk, i_first, nq_here, lists, status);
  if (warp == 5) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;        // S slot sb at column 64 sb; P_A over its first 32 columns
  const uint32_t tO = tmem + 128;  // O at columns 128..255

  // tiles per half: the routed blocks, then the block itself, then (with states) M / 64 tiles of the
  // state of every listed block j >= 1 (the list is ascending, so only its first entry can be block 0)
  const int SPB = M / kKeys;
  int T[2], Ttok[2], sfirst[2];
#pragma unroll
  for (int h = 0; h < 2; h++) {
    Ttok[h] = h < nq_here ? lists[4 * kTileListPitch + h] : 0;
    sfirst[h] = (Ttok[h] > 0 && lists[h * kTileListPitch] == 0) ? 1 : 0;
    T[h] = Ttok[h] + (kStates ? (Ttok[h] - sfirst[h]) * SPB : 0);
  }
  const int Tmax = max(T[0], T[1]);
  // tile k of half h: its first key row (in K / V, or in the [nb * M] state rows) and whether it is a state tile
  auto tile_of = [&](int h, int k, int* key0) -> bool {
    if (!kStates || k < Ttok[h]) {
      *key0 = lists[h * kTileListPitch + k] * kKeys;
      return false;
    }
    const int u = k - Ttok[h], e = sfirst[h] + u / SPB;
    *key0 = lists[h * kTileListPitch + e] * M + (u % SPB) * kKeys;
    return true;
  };

  unsigned char* sQ = smem + PL::kQ;
  unsigned char* sK = smem + PL::kK;
  unsigned char* sV = smem + PL::kV;
  unsigned char* sPB = smem + PL::kPB;

  if (warp == 4 || warp == 6) {
    // ------------------------------------------------------------ producers (K + Q, V)
    const bool is_k = (warp == 4);
    if (lane == 0) {
      if (is_k) {
        mbar_expect_tx(bar_q, 32768);
        for (int h = 0; h < 2; h++) {
          const int row = (i_first + h) * kKeys - g.q_offset;  // rows past the end read as zeros
          for (int dh = 0; dh < 2; dh++) tma_load_3d(sQ + dh * 16384 + h * 8192, &tmQ, dh * 64, row, head, bar_q);
        }
      }
      uint64_t* full = is_k ? bar_k_full : bar_v_full;
      uint64_t* fre = is_k ? bar_k_free : bar_v_free;
      unsigned char* ring = is_k ? sK : sV;
      const CUtensorMap* map = is_k ? &tmK : &tmV;
      bool ok = true;
      int k = 0;
      for (; k < Tmax && ok; k++) {
        if (k > 0) ok = mbar_wait(fre, (k - 1) & 1, abort_flag);
        if (!ok) break;
        const int nt = (k < T[0] ? 1 : 0) + (k < T[1] ? 1 : 0);
        mbar_expect_tx(full, nt * 16384);
        for (int h = 0; h < 2; h++) {
          if (k >= T[h]) continue;
          int key0;
          const bool state = tile_of(h, k, &key0);
          const CUtensorMap* mp = state ? (is_k ? &tmPK : &tmPV) : map;
          for (int dh = 0; dh < 2; dh++) tma_load_3d(ring + h * 16384 + dh * 8192, mp, dh * 64, key0, unit, full);
        }
      }
      // drain: wait (bounded) for every copy issued so far before the CTA may exit
      volatile int no_abort = 0;
      if (is_k) mbar_wait(bar_q, 0, &no_abort);
      if (k > 0) mbar_wait(full, (k - 1) & 1, &no_abort);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(64, kKeys, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(64, 128, 0, 1);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aPB = smem_u32(sPB);
      bool ok = mbar_wait(bar_q, 0, abort_flag);
      int issued = 0;
      for (int k = 0; k <= Tmax && ok; k++) {
        if (k < Tmax) {
          const int sb = k & 1;
          ok = mbar_wait(bar_k_full, k & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          for (int h = 0; h < 2; h++) {
            if (k >= T[h]) continue;
            for (int kk = 0; kk < 8; kk++) {
              const uint64_t a = sdesc_sw128(aQ + (kk >> 2) * 16384 + h * 8192 + (kk & 3) * 32, 16, 1024);
              const uint64_t b = sdesc_sw128(aK + h * 16384 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
              umma_bf16(tS + sb * 64 + (h ? kHalfB : 0u), a, b, idesc_qk, kk > 0);
            }
          }
          umma_commit(bar_s_full + sb);
          umma_commit(bar_k_free);
          issued++;
        }
        if (k >= 1) {
          const int u = k - 1, pb = u & 1;
          ok = mbar_wait(bar_p_full + pb, (u >> 1) & 1, abort_flag);
          if (ok) ok = mbar_wait(bar_v_full, u & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          if (u < T[0])
            for (int kk = 0; kk < 4; kk++) {
              const uint64_t b = sdesc_sw128(aV + kk * 2048, 8192, 1024);
              umma_bf16_ts(tO, tS + pb * 64 + kk * 8, b, idesc_pv, (u > 0 || kk > 0) ? 1u : 0u);
            }
          if (u < T[1])
            for (int kk = 0; kk < 4; kk++) {
              const uint64_t a = sdesc_sw128(aPB + kk * 32, 16, 1024);
              const uint64_t b = sdesc_sw128(aV + 16384 + kk * 2048, 8192, 1024);
              umma_bf16(tO + kHalfB, a, b, idesc_pv, (u > 0 || kk > 0) ? 1u : 0u);
            }
          umma_commit(bar_v_free);
          umma_commit(bar_pb_free);
          umma_commit(bar_o);
          issued++;
        }
      }
      if (ok) umma_commit(bar_done);  // after the last P.V: the epilogue may read O
      if (issued > 0) {
        // every MMA issued so far must finish before the CTA frees its tensor memory
        umma_commit(bar_drain);
        volatile int no_abort = 0;
        mbar_wait(bar_drain, 0, &no_abort);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int h = lane >> 4;                  // 0: block A (lanes 0..15), 1: block B (lanes 16..31)
    const int rr = 16 * warp + (lane & 15);   // row within the block
    const int iq = i_first + h;
    const int p = iq * kKeys + rr;            // position of this row
    const bool row_ok = h < nq_here && p >= g.q_offset && p < g.q_offset + g.Nq;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t tS_row = tS + lane_base;
    const uint32_t tO_row = tO + lane_base;
    const float sl2 = rsqrtf((float)g.d) * 1.4426950408889634f;
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    float s[kKeys];
    for (int k = 0; k < Tmax; k++) {
      const int sb = k & 1;
      // this row's tile at step k: full (routed: every key < N), causal (its own block), state slots (all
      // of them), or none
      int md = 0, key0 = 0, lim = 0;
      if (row_ok && k < T[h]) {
        if (tile_of(h, k, &key0)) {
          md = 1;
          lim = kKeys;
        } else {
          md = key0 == iq * kKeys ? 2 : 1;
          lim = md == 1 ? min(kKeys, g.N - key0) : min(kKeys, p - key0 + 1);
        }
      }
      ok = warp_wait(bar_s_full + sb, (k >> 1) & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      tmem_ld32(tS_row + sb * 64, s);
      tmem_ld32(tS_row + sb * 64 + 32, s + 32);
      tmem_wait_ld();
      if (lim < kKeys) {
#pragma unroll
        for (int c = 0; c < kKeys; c++) s[c] = c < lim ? s[c] : -INFINITY;
      }
      // row max of the raw scores (the positive scale commutes with max): 3-input tree
      float mx;
      {
        float a[22];
#pragma unroll
        for (int c = 0; c < 21; c++) a[c] = fmax3(s[3 * c], s[3 * c + 1], s[3 * c + 2]);
        a[21] = s[63];
        float b2[8];
#pragma unroll
        for (int c = 0; c < 7; c++) b2[c] = fmax3(a[3 * c], a[3 * c + 1], a[3 * c + 2]);
        b2[7] = a[21];
        mx = fmax3(fmax3(b2[0], b2[1], b2[2]), fmax3(b2[3], b2[4], b2[5]), fmaxf(b2[6], b2[7]));
      }
      const float m_new = fmaxf(m_ref, mx * sl2);
      const bool need = (m_ref != -INFINITY) && (m_new > m_ref + kRescale);
      float factor = 1.f;
      if (need) {
        factor = ex2(m_ref - m_new);
        l_sum *= factor;
        m_ref = m_new;
      } else if (m_ref == -INFINITY) {
        m_ref = m_new;
      }
      if (__any_sync(0xffffffffu, need)) {
        // O holds P.V of the steps before k: wait for the last of them, then rescale this lane's row
        ok = warp_wait(bar_o, (k - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        float o[32];
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          tmem_ld32(tO_row + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e++) o[e] *= factor;
          tmem_st32(tO_row + c, o);
        }
      }
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      // p = 2^(s * sl2 - m): packed FMA, exponentials on the MUFU unit; four packed partial sums
      uint32_t pk[32];
      const float2 scl = make_float2(sl2, sl2), off = make_float2(-m_use, -m_use);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 32; c++) {
        const float2 x = __ffma2_rn(make_float2(s[2 * c], s[2 * c + 1]), scl, off);
        const float2 e = make_float2(ex2(x.x), ex2(x.y));
        acc[c & 3] = __fadd2_rn(acc[c & 3], e);
        pk[c] = pack_bf16(e.x, e.y);
      }
      const float2 s01 = __fadd2_rn(acc[0], acc[1]), s23 = __fadd2_rn(acc[2], acc[3]);
      const float2 sall = __fadd2_rn(s01, s23);
      l_sum += sall.x + sall.y;
      // P_A: into tensor memory over S_A (lanes 0..15 of the warp's sub-partition; the same store
      // leaves P_B in lanes 16..31, unused); P_B: into the shared-memory operand
      tmem_st32u(tS_row + sb * 64, pk);
      tmem_wait_st();
      if (h == 1) {
        if (k > 0) ok = mbar_wait(bar_pb_free, (k - 1) & 1, abort_flag);  // P.V of step k-1 read P_B
        if (ok) {
#pragma unroll
          for (int c = 0; c < 8; c++)
            *reinterpret_cast<uint4*>(sPB + rr * 128 + ((c ^ (rr & 7)) << 4)) =
                make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          fence_proxy_async_smem();
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p_full + sb);
    }
    // ---- epilogue: the one-phase barrier after the last P.V (bar_o's parity could alias)
    if (ok) ok = warp_wait(bar_done, 0, abort_flag);
    if (ok) {
      tc_fence_after();
      const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
      const size_t orow = (size_t)head * g.Nq + (size_t)(p - g.q_offset);
      float o[32];
#pragma unroll 1
      for (int c = 0; c < 128; c += 32) {
        tmem_ld32(tO_row + c, o);
        tmem_wait_ld();
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(O + orow * 128 + c);
#pragma unroll
          for (int e = 0; e < 4; e++) {
            uint4 v;
            v.x = pack_bf16(o[8 * e + 0] * inv, o[8 * e + 1] * inv);
            v.y = pack_bf16(o[8 * e + 2] * inv, o[8 * e + 3] * inv);
            v.z = pack_bf16(o[8 * e + 4] * inv, o[8 * e + 5] * inv);
            v.w = pack_bf16(o[8 * e + 6] * inv, o[8 * e + 7] * inv);
            dst[e] = v;
          }
        }
      }
      if (row_ok && lse) lse[orow] = (m_ref + log2f(l_sum)) * 0.6931471805599453f;
    }
  }

  // ---- teardown ----
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) report(status, PYR_ETIMEOUT);
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

bool attn_pair_supported(const Geo& g) {
  return g.dtype == PYR_BF16 && g.d == 128 && g.b == kKeys && g.G == 1 && g.Nq > 1 && g.topk + 1 <= kTileListPitch;
}

cudaError_t launch_attn_pair(const Geo& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                             const int32_t* idx, void* O, float* lse, int* status, cudaStream_t st,
                             const CUtensorMap& mpk, const CUtensorMap& mpv, int M) {
  auto kern = M > 0 ? attn_pair_kernel<true> : attn_pair_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PairPlan::kBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((g.nqb + 1) / 2, g.B * g.Hkv);
  kern<<<grid, kThreads, PairPlan::kBytes, st>>>(mq, mk, mv, idx, reinterpret_cast<__nv_bfloat16*>(O), lse, status, g,
                                                 mpk, mpv, M);
  return cudaGetLastError();
}

}  // namespace pyr
