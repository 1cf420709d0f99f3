// Causal block-sparse attention on the tcgen05 tensor cores (bf16 operands,
// fp32 accumulation in tensor memory). PHBA 3.1 / 3.3 / A.1.3: each query tile
// attends to its routed key blocks plus its own block, one online-softmax merge
// over all of them, output and log-sum-exp written; PHBA A.1.3 also lets one
// loaded key block serve every row of the query tile that routes to it, which
// is how a CTA here shares K/V tiles across the G heads of a kv group and, for
// 64-row query blocks, across two consecutive query blocks.
//
// CTA = one query tile of 128*MT rows of one (batch, kv head):
//   MT = 1 or 2 M-tiles of 128 rows; QB = 1 or 2 query blocks per tile.
//   Row r -> query block i0 + r / (G*b), head r % (G*b) / b, offset r % b.
// Warp roles:
//   warps 0 .. 4*MT-1   softmax: one thread per row (TMEM lane); scale, mask,
//                       lazily rescaled online softmax; P (bf16) is written
//                       back into tensor memory over the S tile it came from;
//                       epilogue;
//   warp 4*MT           TMA producer of Q (once) and of the K tiles (64 keys);
//   warp 4*MT+1         MMA issuer of S = Q K^T into TMEM (two S buffers);
//   warp 4*MT+2         TMA producer of the V tiles;
//   warp 4*MT+3         MMA issuer of O += P V, P read from TMEM, V from
//                       shared memory.
// One thread issues an MMA about every 65 cycles, while an M = 128, N = 64
// MMA runs in about 32, so the two products get an issuing thread each.
// K and V have separate rings: a K tile is released as soon as its QK MMA has
// finished, so the next K loads run one tile ahead of the late PV use of V.
// S buffer reuse: QK of tile t+2 writes the S slot that holds P of tile t, so
// its issuer first waits for the commit of PV t (bar_s_free); the softmax of
// tile t+2 starts only once the commit of QK t+2 (hence PV t) has landed.
// The K/V tile list is the union of the query blocks' routed blocks and their
// diagonal blocks, ascending; each entry carries a mode per query block
// (skip / full / causal). With PHBA prefix states (M > 0; PHBA summary 3.3 and
// A.1.3: one softmax over tokens and state slots) the tiles of the M-slot
// states follow the token tiles: each entry j >= 1 of the list brings the
// state stored before block j (the current block's state for the diagonal,
// the aligned state for a routed block), with the entry's modes and no causal
// mask; block 0 has an empty prefix and no state. The state slots are scored
// with the same Q tile as the tokens. Every mbarrier wait is bounded; a wait that runs out
// aborts the CTA (PYR_ETIMEOUT), and the CTA still drains its in-flight
// copies and MMAs and frees its tensor memory before it exits.
#include <cudaTypedefs.h>

#include "pyr_common.cuh"
#include "tc_util.cuh"
#include "tile_list.cuh"

namespace pyr {

namespace {

using namespace tc;

constexpr int kKeys = 64;         // keys per K/V tile
constexpr int kMaxTiles = 264;    // >= 2 * (topk + 1) for topk <= 128
constexpr float kRescale = 8.0f;  // lazy rescale threshold (log2 units)

template <int MT, int NS>
struct Plan {
  static constexpr int kQ = 0;                         // MT x [2 halves][128 rows][128 B]
  static constexpr int kKV = kQ + MT * 32768;          // K ring: NS x [2][64][128 B], then V ring
  static constexpr int kV = kKV + NS * 16384;
  static constexpr int kBar = kV + NS * 16384;         // mbarriers
  static constexpr int kNumBars = 1 + 4 * NS + 2 + 2 + 3 + 3;
  static constexpr int kMisc = kBar + kNumBars * 8;    // tmem slot, abort flag, tile count
  static constexpr int kTiles = kMisc + 16;            // tile entries: (block << 4) | modes
  static constexpr int kEnd = kTiles + kMaxTiles * 4;
  static constexpr int kBytes = kEnd + 1024;           // + alignment slack
  static constexpr int kThreads = (4 * MT + 4) * 32;
  static constexpr int kTmemCols = MT == 1 ? 256 : 512;
  static constexpr int kMinBlocks = kBytes <= 113 * 1024 ? 2 : 1;
};

// A wait whose outcome the whole warp shares, so that a timeout never leaves
// the warp diverged in front of a .sync.aligned instruction.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int MT, int QB, int KB, int NS>
__global__ void __launch_bounds__(Plan<MT, NS>::kThreads, Plan<MT, NS>::kMinBlocks)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ idx, int dense,
                   __nv_bfloat16* __restrict__ O, float* __restrict__ lse, int* status, Geo g,
                   const __grid_constant__ CUtensorMap tmPK, const __grid_constant__ CUtensorMap tmPV, int M) {
  using PL = Plan<MT, NS>;
  constexpr int TPB = KB / kKeys;  // tiles per key block
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_align<1024>(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PL::kBar);
  uint64_t* bar_q = bars;
  uint64_t* bar_k_full = bars + 1;
  uint64_t* bar_k_free = bar_k_full + NS;
  uint64_t* bar_v_full = bar_k_free + NS;
  uint64_t* bar_v_free = bar_v_full + NS;
  uint64_t* bar_s_full = bar_v_free + NS;   // [2]
  uint64_t* bar_p_full = bar_s_full + 2;    // [2]
  uint64_t* bar_o = bar_p_full + 2;
  uint64_t* bar_drain = bar_o + 1;
  uint64_t* bar_done = bar_drain + 1;  // every MMA of the CTA finished (one phase)
  uint64_t* bar_drain2 = bar_done + 1;  // the P.V issuer's MMAs finished
  uint64_t* bar_s_free = bar_drain2 + 1;  // [2] the P.V MMAs that read P from an S slot done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + PL::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + PL::kMisc + 4);
  int* tiles = reinterpret_cast<int*>(smem + PL::kTiles);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.y;
  const int bi = unit / g.Hkv, hk = unit % g.Hkv;
  const int qb0 = blockIdx.x * QB;
  const int i_first = g.i0 + qb0;
  const int nq_here = min(QB, g.nqb - qb0);  // query blocks present in this tile

  // ---- setup: barriers; the tile's key-block list (built in the K ring, before any copy) ----
  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < NS; s++) {
      mbar_init(bar_k_full + s, 1);
      mbar_init(bar_k_free + s, 1);
      mbar_init(bar_v_full + s, 1);
      mbar_init(bar_v_free + s, 1);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(bar_s_full + b, 1);
      mbar_init(bar_p_full + b, 4 * MT);
    }
    mbar_init(bar_o, 1);
    mbar_init(bar_drain, 1);
    mbar_init(bar_done, 1);
    mbar_init(bar_drain2, 1);
    mbar_init(bar_s_free, 1);
    mbar_init(bar_s_free + 1, 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  int n_entries = 0;
  if (!dense)
    n_entries = build_tile_list<QB>(idx + ((size_t)unit * g.nqb + qb0) * g.topk, g.topk, i_first, nq_here,
                                    reinterpret_cast<int*>(smem + PL::kKV), tiles, status);
  const int softmax_warps = 4 * MT;
  if (warp == softmax_warps + 1) {
    tmem_alloc(tmem_slot, PL::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;             // S[mt][sb] at column (mt*2 + sb)*64; P over its first 32
  const uint32_t tO = tmem + 128 * MT;  // O[mt] at column 128*MT + mt*128
  const int nblk = dense ? (i_first + nq_here) : n_entries;  // dense: blocks 0 .. last diagonal
  const int T_tok = nblk * TPB;
  // state tiles: the entries j >= 1 (the list is ascending, so only its first entry can be block 0)
  const int st_first = (n_entries > 0 && (tiles[0] >> 4) == 0) ? 1 : 0;
  const int SPB = M / kKeys;  // tiles per state
  const int T = T_tok + ((M > 0 && !dense) ? (n_entries - st_first) * SPB : 0);

  // tile t -> (first key row, modes); state tiles: the row in the [nb * M] state rows, full modes
  auto tile_info = [&](int t, int* key0, int* mode) {
    if (t >= T_tok) {
      const int k = (t - T_tok) / SPB, h = (t - T_tok) - k * SPB;
      const int ent = tiles[st_first + k];
      const int m = ent & 15;
      *key0 = (ent >> 4) * M + h * kKeys;
      *mode = (m | (m >> 1)) & 5;  // causal (2) -> full (1) in each query block's two bits
      return;
    }
    const int e = t / TPB, h = t - e * TPB;
    int j, m;
    if (dense) {
      j = e;
      m = 0;
      for (int q = 0; q < nq_here; q++) {
        const int iq = i_first + q;
        m |= (j < iq ? 1 : (j == iq ? 2 : 0)) << (2 * q);
      }
    } else {
      j = tiles[e] >> 4;
      m = tiles[e] & 15;
    }
    *key0 = j * KB + h * kKeys;
    *mode = m;
  };

  unsigned char* sQ = smem + PL::kQ;
  unsigned char* sK = smem + PL::kKV;
  unsigned char* sV = smem + PL::kV;

  if (warp == softmax_warps || warp == softmax_warps + 2) {
    // ------------------------------------------------------------ producers (K + Q, V)
    const bool is_k = (warp == softmax_warps);
    if (lane == 0) {
      bool ok = true;
      if (is_k) {
        mbar_expect_tx(bar_q, MT * 32768);
        for (int mt = 0; mt < MT; mt++)
          for (int c = 0; c < 2; c++) {
            const int r0 = mt * 128 + c * 64;
            const int qsub = r0 / (g.G * g.b), within = r0 % (g.G * g.b);
            const int gq = within / g.b, off = within % g.b;
            const int row = (i_first + qsub) * g.b + off - g.q_offset;
            const int head = bi * g.Hq + hk * g.G + gq;
            for (int h = 0; h < 2; h++)
              tma_load_3d(sQ + mt * 32768 + h * 16384 + c * 8192, &tmQ, h * 64, row, head, bar_q);
          }
      }
      uint64_t* full = is_k ? bar_k_full : bar_v_full;
      uint64_t* fre = is_k ? bar_k_free : bar_v_free;
      unsigned char* ring = is_k ? sK : sV;
      int t = 0;
      for (; t < T && ok; t++) {
        const int s = t % NS, k = t / NS;
        if (k > 0) ok = mbar_wait(fre + s, (k - 1) & 1, abort_flag);
        if (!ok) break;
        int key0, mode;
        tile_info(t, &key0, &mode);
        unsigned char* st = ring + s * 16384;
        const CUtensorMap* map = t < T_tok ? (is_k ? &tmK : &tmV) : (is_k ? &tmPK : &tmPV);
        mbar_expect_tx(full + s, 16384);
        for (int h = 0; h < 2; h++) tma_load_3d(st + h * 8192, map, h * 64, key0, unit, full + s);
      }
      // drain: wait (bounded) for every copy issued so far before the CTA may exit
      volatile int no_abort = 0;
      if (is_k) mbar_wait(bar_q, 0, &no_abort);
      for (int u = max(0, t - NS); u < t; u++) mbar_wait(full + (u % NS), (u / NS) & 1, &no_abort);
    }
    __syncwarp();
  } else if (warp == softmax_warps + 1) {
    // ------------------------------------------------------------ Q.K^T issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kKeys, 0, 0);
      // operand descriptors: the base of each operand once; a stage and a K step add offsets to the
      // start-address field (16-byte units, no carry: shared addresses stay below 2^18 bytes)
      const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024), dK = sdesc_sw128(smem_u32(sK), 16, 1024);
      bool ok = mbar_wait(bar_q, 0, abort_flag);
      int issued = 0;
      for (int t = 0; t < T && ok; t++) {
        const int s = t % NS, sb = t & 1;
        ok = mbar_wait(bar_k_full + s, (t / NS) & 1, abort_flag);
        // S slot sb held P of tile t - 2 until that tile's P.V MMAs were done
        if (ok && t >= 2) ok = mbar_wait(bar_s_free + sb, ((t >> 1) - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dKs = dK + (uint64_t)(s * (16384 >> 4));
#pragma unroll
        for (int mt = 0; mt < MT; mt++)
#pragma unroll
          for (int kk = 0; kk < 8; kk++)
            umma_bf16(tS + (mt * 2 + sb) * 64, dQ + (uint64_t)((mt * 32768 + (kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                      dKs + (uint64_t)(((kk >> 2) * 8192 + (kk & 3) * 32) >> 4), idesc_qk, kk > 0);
        umma_commit(bar_s_full + sb);
        umma_commit(bar_k_free + s);
        issued++;
      }
      if (issued > 0) {
        // every MMA issued so far must finish before the CTA frees its tensor memory
        umma_commit(bar_drain);
        volatile int no_abort = 0;
        mbar_wait(bar_drain, 0, &no_abort);
      }
    }
    __syncwarp();
  } else if (warp == softmax_warps + 3) {
    // ------------------------------------------------------------ P.V issuer
    if (lane == 0) {
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
      const uint64_t dV = sdesc_sw128(smem_u32(sV), 8192, 1024);
      bool ok = true;
      int issued = 0;
      for (int u = 0; u < T && ok; u++) {
        const int s = u % NS, pb = u & 1;
        ok = mbar_wait(bar_p_full + pb, (u >> 1) & 1, abort_flag);
        if (ok) ok = mbar_wait(bar_v_full + s, (u / NS) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dVs = dV + (uint64_t)(s * (16384 >> 4));
        const uint32_t acc0 = u > 0 ? 1u : 0u;
#pragma unroll
        for (int mt = 0; mt < MT; mt++)
#pragma unroll
          for (int kk = 0; kk < 4; kk++)
            umma_bf16_ts(tO + mt * 128, tS + (mt * 2 + pb) * 64 + kk * 8, dVs + (uint64_t)((kk * 2048) >> 4), idesc_pv,
                         kk > 0 ? 1u : acc0);
        umma_commit(bar_v_free + s);
        umma_commit(bar_o);
        umma_commit(bar_s_free + pb);
        issued++;
      }
      if (ok) umma_commit(bar_done);  // after the last P.V: the epilogue may read O
      if (issued > 0) {
        umma_commit(bar_drain2);
        volatile int no_abort = 0;
        mbar_wait(bar_drain2, 0, &no_abort);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int mt = warp >> 2, wq = warp & 3;
    const int r = mt * 128 + wq * 32 + lane;
    const int qsub = r / (g.G * g.b), within = r % (g.G * g.b);
    const int gq = within / g.b, off = within % g.b;
    const int iq = i_first + qsub;
    const int p = iq * g.b + off;  // position of this row
    const bool row_ok = qsub < nq_here && p >= g.q_offset && p < g.q_offset + g.Nq;
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const uint32_t tS_row = tS + lane_base + (mt * 2) * 64;
    const uint32_t tO_row = tO + lane_base + mt * 128;
    const float sl2 = rsqrtf((float)g.d) * 1.4426950408889634f;
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    float s[kKeys];
    for (int t = 0; t < T; t++) {
      const int sb = t & 1;
      int key0, mode;
      tile_info(t, &key0, &mode);
      const int md = row_ok ? (mode >> (2 * qsub)) & 3 : 0;
      ok = warp_wait(bar_s_full + sb, (t >> 1) & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      if (__all_sync(0xffffffffu, md == 0)) {
        // no row of this warp attends the tile (with two query blocks per CTA, the tile may be
        // routed for the other block only): P = 0, without reading S or touching the softmax state
        uint32_t zero[32];
#pragma unroll
        for (int c = 0; c < 32; c++) zero[c] = 0u;
        tmem_st32u(tS_row + sb * 64, zero);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_p_full + sb);
        continue;
      }
      tmem_ld32(tS_row + sb * 64, s);
      tmem_ld32(tS_row + sb * 64 + 32, s + 32);
      tmem_wait_ld();

      // valid keys: full -> every key < N; causal -> keys <= p; state slots -> all of them
      const int lim = md == 0 ? 0
                              : (t >= T_tok ? kKeys : (md == 1 ? min(kKeys, g.N - key0) : min(kKeys, p - key0 + 1)));
      if (lim < kKeys) {
#pragma unroll
        for (int c = 0; c < kKeys; c++) s[c] = c < lim ? s[c] : -INFINITY;
      }
      // row max of the raw scores (the positive scale commutes with max): 3-input tree
      float mx;
      {
        float a[22];
#pragma unroll
        for (int k = 0; k < 21; k++) a[k] = fmax3(s[3 * k], s[3 * k + 1], s[3 * k + 2]);
        a[21] = s[63];
        float b2[8];
#pragma unroll
        for (int k = 0; k < 7; k++) b2[k] = fmax3(a[3 * k], a[3 * k + 1], a[3 * k + 2]);
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
        // O holds P.V of the tiles before t: wait for the last of them, then rescale this warp's rows
        ok = warp_wait(bar_o, (t - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        float o[32];
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          tmem_ld32(tO_row + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; k++) o[k] *= factor;
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
        // every exponential on the MUFU unit: the softmax is issue-bound, and a polynomial on the
        // FMA pipe costs more issue slots than it saves (measured)
        const float2 e = make_float2(ex2(x.x), ex2(x.y));
        acc[c & 3] = __fadd2_rn(acc[c & 3], e);
        pk[c] = pack_bf16(e.x, e.y);
      }
      const float2 s01 = __fadd2_rn(acc[0], acc[1]), s23 = __fadd2_rn(acc[2], acc[3]);
      const float2 sall = __fadd2_rn(s01, s23);
      l_sum += sall.x + sall.y;
      tmem_st32u(tS_row + sb * 64, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p_full + sb);
    }
    // ---- epilogue ----
    // the last P.V: wait on the one-phase barrier, not on bar_o, whose parity can alias when the
    // P.V of tile T-2 is still in flight (s_full of tile T-1 only guarantees P.V of tile T-3)
    if (ok) ok = warp_wait(bar_done, 0, abort_flag);
    if (ok) {
      tc_fence_after();
      const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
      const size_t orow = ((size_t)bi * g.Hq + hk * g.G + gq) * g.Nq + (size_t)(p - g.q_offset);
      float o[32];
#pragma unroll 1
      for (int c = 0; c < 128; c += 32) {
        tmem_ld32(tO_row + c, o);
        tmem_wait_ld();
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(O + orow * 128 + c);
#pragma unroll
          for (int k = 0; k < 4; k++) {
            uint4 v;
            v.x = pack_bf16(o[8 * k + 0] * inv, o[8 * k + 1] * inv);
            v.y = pack_bf16(o[8 * k + 2] * inv, o[8 * k + 3] * inv);
            v.z = pack_bf16(o[8 * k + 4] * inv, o[8 * k + 5] * inv);
            v.w = pack_bf16(o[8 * k + 6] * inv, o[8 * k + 7] * inv);
            dst[k] = v;
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
  if (warp == softmax_warps + 1) {
    tc_fence_after();
    tmem_dealloc(tmem, PL::kTmemCols);
  }
}

// ---- host side -------------------------------------------------------------

template <int MT, int QB, int KB, int NS>
cudaError_t launch_cfg(const Geo& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const int32_t* idx, int dense, void* O, float* lse, int* status, cudaStream_t st,
                       const CUtensorMap& mpk, const CUtensorMap& mpv, int M) {
  using PL = Plan<MT, NS>;
  auto kern = attn_tc_kernel<MT, QB, KB, NS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PL::kBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((g.nqb + QB - 1) / QB, g.B * g.Hkv);
  kern<<<grid, PL::kThreads, PL::kBytes, st>>>(mq, mk, mv, idx, dense, reinterpret_cast<__nv_bfloat16*>(O), lse,
                                                status, g, mpk, mpv, M);
  return cudaGetLastError();
}

}  // namespace

// two 64-row query blocks of one head per CTA, each over its own block list (attn_pair.cu)
bool attn_pair_supported(const Geo& g);
cudaError_t launch_attn_pair(const Geo& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                             const int32_t* idx, void* O, float* lse, int* status, cudaStream_t st,
                             const CUtensorMap& mpk, const CUtensorMap& mpv, int M);

bool attn_tc_supported(const Geo& g) {
  if (g.dtype != PYR_BF16 || g.d != 128) return false;
  if (g.b != 64 && g.b != 128) return false;
  if (g.Nq == 1) return false;  // decode has its own kernel
  const int rows = g.G * g.b;
  // the tile list holds QB * (topk + 1) blocks of b / 64 tiles each: <= kMaxTiles for topk <= 128
  return rows == 64 || rows == 128 || rows == 256;
}

cudaError_t launch_attn_tc(const Geo& g, const void* Q, const void* K, const void* V, const int32_t* idx, int dense,
                           void* O, float* lse, int* status, cudaStream_t st, const void* PK, const void* PV,
                           int M) {
  CUtensorMap mq, mk, mv, mpk, mpv;
  if (!make_tmap_bf16_3d(&mq, Q, g.d, g.Nq, g.B * g.Hq) || !make_tmap_bf16_3d(&mk, K, g.d, g.N, g.B * g.Hkv) ||
      !make_tmap_bf16_3d(&mv, V, g.d, g.N, g.B * g.Hkv))
    return cudaErrorInvalidValue;
  if (M > 0) {
    // states [B * Hkv][nb * M][d]: a tile of 64 slots is a 64-row box like a K tile
    if (M % kKeys || !make_tmap_bf16_3d(&mpk, PK, g.d, g.nb * M, g.B * g.Hkv) ||
        !make_tmap_bf16_3d(&mpv, PV, g.d, g.nb * M, g.B * g.Hkv))
      return cudaErrorInvalidValue;
  } else {
    mpk = mk;  // unused
    mpv = mv;
  }
  const int rows = g.G * g.b;
  if (!dense && attn_pair_supported(g))
    return launch_attn_pair(g, mq, mk, mv, idx, O, lse, status, st, mpk, mpv, M);
  if (g.b == 64) {
    if (rows == 64) return launch_cfg<1, 2, 64, 2>(g, mq, mk, mv, idx, dense, O, lse, status, st, mpk, mpv, M);
    if (rows == 128) return launch_cfg<1, 1, 64, 2>(g, mq, mk, mv, idx, dense, O, lse, status, st, mpk, mpv, M);
    return launch_cfg<2, 1, 64, 3>(g, mq, mk, mv, idx, dense, O, lse, status, st, mpk, mpv, M);
  }
  if (rows == 128) return launch_cfg<1, 1, 128, 2>(g, mq, mk, mv, idx, dense, O, lse, status, st, mpk, mpv, M);
  return launch_cfg<2, 1, 128, 3>(g, mq, mk, mv, idx, dense, O, lse, status, st, mpk, mpv, M);
}

namespace tc {

// looked up once per process; the initialisation of a function-local static is thread-safe
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    return cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
                   q == cudaDriverEntryPointSuccess
               ? reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p)
               : nullptr;
  }();
  return fn;
}

bool make_tmap_bf16_3d(CUtensorMap* m, const void* base, int inner, int rows, int heads, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)rows * inner * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_f32_3d(CUtensorMap* m, const void* base, int inner, int rows, int heads, int box_inner, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)inner * 4, (cuuint64_t)rows * inner * 4};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc

}  // namespace pyr
