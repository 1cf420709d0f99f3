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
//                       lazy-rescaled online softmax, P (bf16) to shared
//                       memory in the 128B-swizzled K-major layout, epilogue;
//   warp 4*MT           TMA producer: Q once, then K and V tiles of 64 keys;
//   warp 4*MT+1         MMA issuer: S = Q K^T into TMEM (double buffered),
//                       O += P V into TMEM.
// The K/V tile list is the union of the query blocks' routed blocks and their
// diagonal blocks, ascending; each tile carries a mode per query block
// (skip / full / causal). Every mbarrier wait is bounded; a wait that runs out
// aborts the CTA (PYR_ETIMEOUT), and the CTA still drains its in-flight
// copies and frees its tensor memory before it exits.
#include <cudaTypedefs.h>

#include "pyr_common.cuh"
#include "tc_util.cuh"

namespace pyr {

namespace {

using namespace tc;

constexpr int kKeys = 64;         // keys per K/V tile
constexpr int kMaxTiles = 264;    // (topk + 1) * 2 for topk <= 128
constexpr float kRescale = 8.0f;  // lazy rescale threshold (log2 units)

template <int MT, int NS, int NPB>
struct Plan {
  static constexpr int kQ = 0;                           // MT x [2 halves][128 rows][128 B]
  static constexpr int kKV = kQ + MT * 32768;            // NS x (K [2][64][128 B], V [2][64][128 B])
  static constexpr int kP = kKV + NS * 32768;            // NPB x MT x [128 rows][128 B]
  static constexpr int kBar = kP + NPB * MT * 16384;     // mbarriers
  static constexpr int kNumBars = 1 + 2 * NS + 4 + 2 * NPB + 2;
  static constexpr int kMisc = kBar + kNumBars * 8;      // tmem slot, abort flag, tile count
  static constexpr int kTiles = kMisc + 16;              // tile key offsets, then modes
  static constexpr int kEnd = kTiles + kMaxTiles * 8;
  static constexpr int kBytes = kEnd + 1024;             // + alignment slack
  static constexpr int kThreads = (4 * MT + 2) * 32;
  static constexpr int kTmemCols = MT == 1 ? 256 : 512;
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

template <int MT, int QB, int KB, int NS, int NPB>
__global__ void __launch_bounds__(Plan<MT, NS, NPB>::kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ idx, int dense,
                   __nv_bfloat16* __restrict__ O, float* __restrict__ lse, int* status, Geo g) {
  using PL = Plan<MT, NS, NPB>;
  constexpr int TPB = KB / kKeys;  // tiles per key block
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PL::kBar);
  uint64_t* bar_q = bars;
  uint64_t* bar_kv_full = bars + 1;
  uint64_t* bar_kv_free = bar_kv_full + NS;
  uint64_t* bar_s_full = bar_kv_free + NS;  // [2]
  uint64_t* bar_s_free = bar_s_full + 2;    // [2]
  uint64_t* bar_p_full = bar_s_free + 2;    // [NPB]
  uint64_t* bar_p_free = bar_p_full + NPB;  // [NPB]
  uint64_t* bar_o = bar_p_free + NPB;
  uint64_t* bar_drain = bar_o + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + PL::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + PL::kMisc + 4);
  int* s_ntiles = reinterpret_cast<int*>(smem + PL::kMisc + 8);
  int* tile_key = reinterpret_cast<int*>(smem + PL::kTiles);
  int* tile_mode = tile_key + kMaxTiles;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.y;
  const int bi = unit / g.Hkv, hk = unit % g.Hkv;
  const int qb0 = blockIdx.x * QB;
  const int i_first = g.i0 + qb0;
  const int nq_here = min(QB, g.nqb - qb0);  // query blocks present in this tile

  // ---- setup: barriers, tile list ----
  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < NS; s++) {
      mbar_init(bar_kv_full + s, 1);
      mbar_init(bar_kv_free + s, 1);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(bar_s_full + b, 1);
      mbar_init(bar_s_free + b, 4 * MT);
    }
    for (int b = 0; b < NPB; b++) {
      mbar_init(bar_p_full + b, 4 * MT);
      mbar_init(bar_p_free + b, 1);
    }
    mbar_init(bar_o, 1);
    mbar_init(bar_drain, 1);
    fence_mbar_init();
    *abort_flag = 0;
    int n = 0;
    if (!dense) {
      // merge the ascending lists sel(i_q) + [i_q] of the query blocks of the tile
      int pos[QB], prev[QB];
      const int32_t* row[QB];
      for (int q = 0; q < QB; q++) {
        pos[q] = 0;
        prev[q] = -1;
        row[q] = idx + ((size_t)unit * g.nqb + (qb0 + q)) * g.topk;
      }
      while (n < kMaxTiles / TPB) {
        // next valid candidate of each query block (the diagonal comes last)
        int cand[QB];
        int best = 0x7fffffff;
        for (int q = 0; q < QB; q++) {
          cand[q] = 0x7fffffff;
          if (q >= nq_here) continue;
          const int iq = i_first + q;
          while (pos[q] < g.topk) {
            const int j = row[q][pos[q]];
            if (j < 0) {
              pos[q]++;
              continue;
            }
            if (j >= iq || j <= prev[q]) {
              report(status, PYR_EBADIDX);
              pos[q]++;
              continue;
            }
            break;
          }
          if (pos[q] < g.topk) cand[q] = row[q][pos[q]];
          else if (pos[q] == g.topk) cand[q] = iq;  // the diagonal block
          best = min(best, cand[q]);
        }
        if (best == 0x7fffffff) break;
        int mode = 0;
        for (int q = 0; q < QB; q++) {
          if (cand[q] == best) {
            mode |= (pos[q] == g.topk ? 2 : 1) << (2 * q);
            prev[q] = best;
            pos[q]++;
          }
        }
        tile_key[n] = best;
        tile_mode[n] = mode;
        n++;
      }
    }
    *s_ntiles = n;
  }
  __syncthreads();
  const int nblk = dense ? (i_first + nq_here) : *s_ntiles;  // dense: blocks 0 .. last diagonal
  const int T = nblk * TPB;

  // block list entry -> (key offset, modes)
  auto tile_info = [&](int t, int* key0, int* mode) {
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
      j = tile_key[e];
      m = tile_mode[e];
    }
    *key0 = j * KB + h * kKeys;
    *mode = m;
  };

  const int softmax_warps = 4 * MT;
  if (warp == softmax_warps + 1) {
    tmem_alloc(tmem_slot, PL::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;                 // S[mt][sb] at column (mt*2 + sb)*64
  const uint32_t tO = tmem + 128 * MT;      // O[mt] at column 128*MT + mt*128

  unsigned char* sQ = smem + PL::kQ;
  unsigned char* sKV = smem + PL::kKV;
  unsigned char* sP = smem + PL::kP;

  if (warp == softmax_warps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
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
      int t = 0;
      for (; t < T && ok; t++) {
        const int s = t % NS, k = t / NS;
        if (k > 0) ok = mbar_wait(bar_kv_free + s, (k - 1) & 1, abort_flag);
        if (!ok) break;
        int key0, mode;
        tile_info(t, &key0, &mode);
        unsigned char* st = sKV + s * 32768;
        mbar_expect_tx(bar_kv_full + s, 32768);
        for (int h = 0; h < 2; h++) {
          tma_load_3d(st + h * 8192, &tmK, h * 64, key0, unit, bar_kv_full + s);
          tma_load_3d(st + 16384 + h * 8192, &tmV, h * 64, key0, unit, bar_kv_full + s);
        }
      }
      // drain: wait (bounded) for every copy issued so far before the CTA may exit
      volatile int no_abort = 0;
      mbar_wait(bar_q, 0, &no_abort);
      for (int u = max(0, t - NS); u < t; u++) mbar_wait(bar_kv_full + (u % NS), (u / NS) & 1, &no_abort);
    }
    __syncwarp();
  } else if (warp == softmax_warps + 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kKeys, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
      const uint32_t aQ = smem_u32(sQ), aKV = smem_u32(sKV), aP = smem_u32(sP);
      bool ok = mbar_wait(bar_q, 0, abort_flag);
      int issued = 0;
      for (int t = 0; t <= T && ok; t++) {
        if (t < T) {
          const int s = t % NS, sb = t & 1;
          ok = mbar_wait(bar_kv_full + s, (t / NS) & 1, abort_flag);
          if (ok && t >= 2) ok = mbar_wait(bar_s_free + sb, ((t >> 1) - 1) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          for (int mt = 0; mt < MT; mt++)
            for (int kk = 0; kk < 8; kk++) {
              const uint64_t a = sdesc_sw128(aQ + mt * 32768 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
              const uint64_t b = sdesc_sw128(aKV + s * 32768 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
              umma_bf16(tS + (mt * 2 + sb) * 64, a, b, idesc_qk, kk > 0);
            }
          umma_commit(bar_s_full + sb);
          issued++;
        }
        if (t >= 1) {
          const int u = t - 1, s = u % NS, pb = u % NPB;
          ok = mbar_wait(bar_p_full + pb, (u / NPB) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          for (int mt = 0; mt < MT; mt++)
            for (int kk = 0; kk < 4; kk++) {
              const uint64_t a = sdesc_sw128(aP + (pb * MT + mt) * 16384 + kk * 32, 16, 1024);
              const uint64_t b = sdesc_sw128(aKV + s * 32768 + 16384 + kk * 2048, 8192, 1024);
              umma_bf16(tO + mt * 128, a, b, idesc_pv, (u > 0 || kk > 0) ? 1u : 0u);
            }
          umma_commit(bar_p_free + pb);
          umma_commit(bar_kv_free + s);
          umma_commit(bar_o);
          issued++;
        }
      }
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
    const int rsw = (wq * 32 + lane) & 7;  // swizzle phase of this row
    unsigned char* p_row_base = sP + mt * 16384 + ((wq * 32 + lane) >> 3) * 1024 + rsw * 128;
    float s[kKeys];
    for (int t = 0; t < T; t++) {
      const int sb = t & 1;
      ok = warp_wait(bar_s_full + sb, (t >> 1) & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      tmem_ld32(tS_row + sb * 64, s);
      tmem_ld32(tS_row + sb * 64 + 32, s + 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_s_free + sb);

      int key0, mode;
      tile_info(t, &key0, &mode);
      const int md = row_ok ? (mode >> (2 * qsub)) & 3 : 0;
      // valid keys: full -> all keys < N; causal -> keys <= p
      const int lim = md == 0 ? 0 : (md == 1 ? min(kKeys, g.N - key0) : min(kKeys, p - key0 + 1));
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kKeys; c++) {
        s[c] = c < lim ? s[c] * sl2 : -INFINITY;
        mx = fmaxf(mx, s[c]);
      }
      const float m_new = fmaxf(m_ref, mx);
      const bool need = (m_ref != -INFINITY) && (m_new > m_ref + kRescale);
      float factor = 1.f;
      if (need) {
        factor = exp2f(m_ref - m_new);
        l_sum *= factor;
        m_ref = m_new;
      } else if (m_ref == -INFINITY) {
        m_ref = m_new;
      }
      if (__any_sync(0xffffffffu, need)) {
        // O holds P.V of tiles < t: wait for the last of them, then rescale this warp's rows
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
        tmem_wait_st();
      }
      const int pb = t % NPB;
      if (t >= NPB) {
        ok = warp_wait(bar_p_free + pb, ((t / NPB) - 1) & 1, abort_flag);
        if (!ok) break;
      }
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      unsigned char* prow = p_row_base + pb * MT * 16384;
      float part = 0.f;
#pragma unroll
      for (int c8 = 0; c8 < 8; c8++) {
        float e[8];
#pragma unroll
        for (int k = 0; k < 8; k++) {
          e[k] = exp2f(s[c8 * 8 + k] - m_use);
          part += e[k];
        }
        uint4 v;
        v.x = pack_bf16(e[0], e[1]);
        v.y = pack_bf16(e[2], e[3]);
        v.z = pack_bf16(e[4], e[5]);
        v.w = pack_bf16(e[6], e[7]);
        *reinterpret_cast<uint4*>(prow + ((c8 ^ rsw) << 4)) = v;
      }
      l_sum += part;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p_full + pb);
    }
    // ---- epilogue ----
    if (ok) ok = warp_wait(bar_o, (T - 1) & 1, abort_flag);
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

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D map over a [heads][rows][d] bf16 tensor; box = 64 d-elements x 64 rows x 1 head, 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, int d, int rows, int heads) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows * d * 2};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MT, int QB, int KB, int NS, int NPB>
cudaError_t launch_cfg(const Geo& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const int32_t* idx, int dense, void* O, float* lse, int* status, cudaStream_t st) {
  using PL = Plan<MT, NS, NPB>;
  auto kern = attn_tc_kernel<MT, QB, KB, NS, NPB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PL::kBytes);
  if (e != cudaSuccess) return e;
  dim3 grid((g.nqb + QB - 1) / QB, g.B * g.Hkv);
  kern<<<grid, PL::kThreads, PL::kBytes, st>>>(mq, mk, mv, idx, dense, reinterpret_cast<__nv_bfloat16*>(O), lse,
                                                status, g);
  return cudaGetLastError();
}

}  // namespace

bool attn_tc_supported(const Geo& g) {
  if (g.dtype != PYR_BF16 || g.d != 128) return false;
  if (g.b != 64 && g.b != 128) return false;
  if (g.Nq == 1) return false;  // decode has its own kernel
  const int rows = g.G * g.b;
  if (rows != 64 && rows != 128 && rows != 256) return false;
  // the tile list holds QB * (topk + 1) blocks of b / 64 tiles each: <= kMaxTiles for topk <= 128
  return true;
}

cudaError_t launch_attn_tc(const Geo& g, const void* Q, const void* K, const void* V, const int32_t* idx, int dense,
                           void* O, float* lse, int* status, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, Q, g.d, g.Nq, g.B * g.Hq) || !make_map(&mk, K, g.d, g.N, g.B * g.Hkv) ||
      !make_map(&mv, V, g.d, g.N, g.B * g.Hkv))
    return cudaErrorInvalidValue;
  const int rows = g.G * g.b;
  if (g.b == 64) {
    if (rows == 64) return launch_cfg<1, 2, 64, 3, 2>(g, mq, mk, mv, idx, dense, O, lse, status, st);
    if (rows == 128) return launch_cfg<1, 1, 64, 3, 2>(g, mq, mk, mv, idx, dense, O, lse, status, st);
    return launch_cfg<2, 1, 64, 2, 2>(g, mq, mk, mv, idx, dense, O, lse, status, st);
  }
  if (rows == 128) return launch_cfg<1, 1, 128, 3, 2>(g, mq, mk, mv, idx, dense, O, lse, status, st);
  return launch_cfg<2, 1, 128, 2, 2>(g, mq, mk, mv, idx, dense, O, lse, status, st);
}

}  // namespace pyr
