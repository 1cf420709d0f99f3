// Coarse-to-fine LogSumExp top-K key-block selection with the scoring GEMM on
// the tcgen05 tensor cores (PISA abstract: start at the coarsest level, score
// a bounded candidate set with LogSumExp, pass the survivors' children to the
// next finer level; routes only to strictly preceding blocks, -1 padding,
// PHBA A.1.2).
//
// One CTA (4 warps) per (batch, kv head, query block i). Per level:
//   gather   the <= cap candidate node rows are copied (cp.async, 16 bytes
//            per thread) straight from the pyramid, which already stores every
//            mean as a bf16 (hi, lo) pair, to their places in the 128B-swizzled
//            K-major A operands; the one node that straddles block i
//            uses the exact mean of its part before i, from the binary
//            decomposition of [m 2^l, i) into whole finer nodes, split by a
//            thread into hi + lo;
//   score    D[candidate][row] = kbar . q_row on the tensor cores, as
//            A_hi * Q^T + A_lo * Q^T (M = candidates: 64 or 128, N = the
//            G*b query rows staged once by TMA, K = d), fp32 accumulation in
//            tensor memory. Each TMEM lane then holds one candidate's dot
//            products with every query row, so the LogSumExp over rows is a
//            per-thread reduction; S = LSE(q.kbar / sqrt(d)) + ln n_valid;
//   select   a parallel rank count over packed 64-bit keys (order-preserving
//            score bits over the inverted node index: ties go to the lower
//            index), keep cap/2 (levels > 0) or topk (level 0), and a warp
//            scan compacts the surviving nodes' valid children.
// q is exactly representable in bf16, so the only rounding beyond fp32
// accumulation is the hi/lo split of the means.
#include "pyr_common.cuh"
#include "tc_util.cuh"

namespace pyr {

namespace {

using namespace tc;

constexpr int kThreads = 128;
constexpr int kMaxCap = 128;

struct SelPlan {
  int q, a_hi, a_lo, part, keys, cand, kept, misc, bars, total;
};

// R: query rows (N of the MMA); MC: candidate rows (M of the MMA); levels: s0 + 1.
__host__ __device__ inline SelPlan sel_plan(int R, int MC, int levels, int d) {
  SelPlan p;
  int o = 0;
  p.q = o;     o += R * d * 2;           // [2 halves][R][128 B]
  p.a_hi = o;  o += MC * d * 2;          // [2 halves][MC][128 B]
  p.a_lo = o;  o += MC * d * 2;
  p.part = o;  o += levels * d * 4;      // straddling-node means, fp32
  p.keys = o;  o += kMaxCap * 8;
  p.cand = o;  o += kMaxCap * 4;
  p.kept = o;  o += kMaxCap * 4;
  p.misc = o;  o += 64;                  // nc, gap, tmem slot, abort flag, boundary scores
  p.bars = o;  o += 16;                  // q_full, mma_done
  p.total = o + 1024;                    // + alignment slack
  return p;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float key_score(unsigned long long k) {
  const uint32_t u = (uint32_t)(k >> 32);
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

template <int MC>
__global__ void __launch_bounds__(kThreads, MC == 64 ? 4 : 2) select_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                             const __nv_bfloat16* __restrict__ pyr, int32_t* __restrict__ idx,
                                                             float* __restrict__ gap_out, int* status, Geo g) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int R = g.G * g.b;  // query rows of a full block (N of the MMA)
  const SelPlan L = sel_plan(R, MC, g.s0 + 1, 128);
  unsigned char* sQ = smem + L.q;
  unsigned char* sAh = smem + L.a_hi;
  unsigned char* sAl = smem + L.a_lo;
  float* part = reinterpret_cast<float*>(smem + L.part);
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(smem + L.keys);
  int* cand = reinterpret_cast<int*>(smem + L.cand);
  int* kept = reinterpret_cast<int*>(smem + L.kept);
  int* s_nc = reinterpret_cast<int*>(smem + L.misc);
  float* s_gap = reinterpret_cast<float*>(smem + L.misc + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 12);
  float* s_edge = reinterpret_cast<float*>(smem + L.misc + 16);  // [0]: last kept, [1]: first dropped
  uint64_t* bar_q = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* bar_mma = bar_q + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x, unit = blockIdx.y;
  const int bi = unit / g.Hkv, hk = unit % g.Hkv;
  const int i = g.i0 + qb;
  const int p0 = max(i * g.b, g.q_offset);
  const int rb = min((i + 1) * g.b, g.q_offset + g.Nq) - p0;  // valid rows per head
  const int tcols = R <= 64 ? 64 : (R <= 128 ? 128 : 256);
  // this thread's candidate (TMEM lane): M=128 -> lane t; M=64 -> rows 16w..16w+15 in lanes 32w..32w+15
  const int my_c = MC == 128 ? threadIdx.x : (lane < 16 ? warp * 16 + lane : -1);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    *abort_flag = 0;
    *s_gap = __int_as_float(0x7f800000);
    // start level: every node of level s0 that begins before block i
    *s_nc = min(g.lvl_n[g.s0], (i + (1 << g.s0) - 1) >> g.s0);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // the G*b query rows: per head, b/64 boxes of 64 rows x 64 d per d-half
    mbar_expect_tx(bar_q, R * 256);
    for (int gg = 0; gg < g.G; gg++)
      for (int c = 0; c < g.b / 64; c++) {
        const int row = i * g.b + c * 64 - g.q_offset;
        const int head = bi * g.Hq + hk * g.G + gg;
        for (int h = 0; h < 2; h++)
          tma_load_3d(sQ + h * (R * 128) + (gg * g.b + c * 64) * 128, &tmQ, h * 64, row, head, bar_q);
      }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tcols);
    tmem_relinquish();
  }
  // exact means of the straddling node's part before i, levels 1..s0
  const __nv_bfloat16* pu = pyr + (size_t)unit * g.P * 256;
  for (int e = threadIdx.x; e < 128; e += kThreads) {
    float acc = 0.f;
    part[e] = 0.f;
    for (int l = 1; l <= g.s0; l++) {
      if ((i >> (l - 1)) & 1)
        acc += split_load(pu + (size_t)(g.lvl_off[l - 1] + (i >> (l - 1)) - 1) * 256, 128, e) * (float)(g.b << (l - 1));
      const int cnt = i - ((i >> l) << l);
      part[l * 128 + e] = cnt > 0 ? acc / (float)(cnt * g.b) : 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tD = *tmem_slot;
  const uint32_t my_lane_addr = tD + ((uint32_t)(warp * 32) << 16);
  const float sl2 = rsqrtf((float)g.d) * 1.4426950408889634f;
  const uint32_t idesc = idesc_bf16_f32(MC, R, 0, 0);
  bool ok = true;
  if (threadIdx.x == 0) ok = mbar_wait(bar_q, 0, abort_flag);
  ok = __syncthreads_and(ok);
  int nphase = 0;
  int32_t* out = idx + ((size_t)unit * g.nqb + qb) * g.topk;

  for (int l = g.s0; l >= 0 && ok; l--) {
    const int nc = *s_nc;
    const bool start = (l == g.s0);
    // ---- gather: every thread copies 16-byte chunks of the candidates' (hi, lo) rows with
    // cp.async straight to their swizzled places in the A operands (consecutive threads take
    // consecutive chunks of a row: coalesced, all copies in flight together); the straddling
    // node's row (at most one per level) is written by warp 1 from the exact partial mean.
    const int ms = (l > 0 && (i & ((1 << l) - 1)) != 0) ? (i >> l) : -1;  // the straddling node
    for (int x = threadIdx.x; x < nc * 32; x += kThreads) {
      const int c = x >> 5, q = x & 31;  // chunk q: 8 elements; 0..15 hi, 16..31 lo
      const int m = start ? c : cand[c];
      if (m == ms) continue;
      const int h = (q >> 3) & 1, c8 = q & 7;
      unsigned char* dst = ((q < 16) ? sAh : sAl) + h * (MC * 128) + (c >> 3) * 1024 + (c & 7) * 128 + ((c8 ^ (c & 7)) << 4);
      cp_async16(dst, pu + (size_t)(g.lvl_off[l] + m) * 256 + q * 8);
    }
    cp_async_wait_all();
    if (warp == 1 && ms >= 0) {
      for (int c = 0; c < nc; c++) {
        if ((start ? c : cand[c]) != ms) continue;
        const float4 v = *reinterpret_cast<const float4*>(part + l * 128 + lane * 4);
        const float x[4] = {v.x, v.y, v.z, v.w};
        float hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
          hi[e] = __bfloat162float(__float2bfloat16_rn(x[e]));
          lo[e] = x[e] - hi[e];
        }
        const int h = lane >> 4, c8 = (lane & 15) >> 1, half8 = (lane & 1) * 8;
        const int off = h * (MC * 128) + (c >> 3) * 1024 + (c & 7) * 128 + ((c8 ^ (c & 7)) << 4) + half8;
        *reinterpret_cast<uint2*>(sAh + off) = make_uint2(pack_bf16x2(hi[0], hi[1]), pack_bf16x2(hi[2], hi[3]));
        *reinterpret_cast<uint2*>(sAl + off) = make_uint2(pack_bf16x2(lo[0], lo[1]), pack_bf16x2(lo[2], lo[3]));
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    // ---- score on the tensor cores
    if (threadIdx.x == 0) {
      tc_fence_after();
      const uint32_t aQ = smem_u32(sQ), aH = smem_u32(sAh), aL = smem_u32(sAl);
      for (int kk = 0; kk < 8; kk++) {
        const uint64_t b = sdesc_sw128(aQ + (kk >> 2) * (R * 128) + (kk & 3) * 32, 16, 1024);
        const uint64_t ah = sdesc_sw128(aH + (kk >> 2) * (MC * 128) + (kk & 3) * 32, 16, 1024);
        const uint64_t al = sdesc_sw128(aL + (kk >> 2) * (MC * 128) + (kk & 3) * 32, 16, 1024);
        umma_bf16(tD, ah, b, idesc, kk > 0);
        umma_bf16(tD, al, b, idesc, 1);
      }
      umma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, nphase & 1, abort_flag);
    ok = __syncthreads_and(ok);  // block-uniform: the loop below has block-wide barriers
    nphase++;
    if (!ok) break;
    tc_fence_after();
    // ---- LogSumExp over the valid query rows, one candidate per thread: pass 1 takes the
    // max of the raw dot products (the positive scale commutes with max), pass 2 re-reads
    // TMEM and sums 2^(x * scale - max) with packed FMAs and four independent partial sums.
    float m2 = -INFINITY, s2 = 0.f;
    const bool warp_has = MC == 128 ? (warp * 32 < nc) : (warp * 16 < nc);
    if (warp_has) {
      const bool full = (rb == g.b);
      float v[32];
      float mx = -INFINITY;
      for (int c0 = 0; c0 < R; c0 += 32) {
        tmem_ld32(my_lane_addr + c0, v);
        tmem_wait_ld();
        if (!full) {
#pragma unroll
          for (int k = 0; k < 32; k++) v[k] = ((c0 + k) % g.b) < rb ? v[k] : -INFINITY;
        }
        float a[11];
#pragma unroll
        for (int k = 0; k < 10; k++) a[k] = fmax3(v[3 * k], v[3 * k + 1], v[3 * k + 2]);
        a[10] = fmaxf(v[30], v[31]);
        mx = fmax3(mx, fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), fmax3(a[6], a[7], a[8])),
                   fmaxf(a[9], a[10]));
      }
      m2 = mx * sl2;
      const float2 scl = make_float2(sl2, sl2), off = make_float2(-m2, -m2);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      for (int c0 = 0; c0 < R; c0 += 32) {
        tmem_ld32(my_lane_addr + c0, v);
        tmem_wait_ld();
        if (!full) {
#pragma unroll
          for (int k = 0; k < 32; k++) v[k] = ((c0 + k) % g.b) < rb ? v[k] : -INFINITY;
        }
#pragma unroll
        for (int k = 0; k < 16; k++) {
          const float2 x = __ffma2_rn(make_float2(v[2 * k], v[2 * k + 1]), scl, off);
          acc[k & 3] = __fadd2_rn(acc[k & 3], make_float2(ex2(x.x), ex2(x.y)));
        }
      }
      const float2 t = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
      s2 = t.x + t.y;
    }
    tc_fence_before();
    if (my_c >= 0 && my_c < nc) {
      const int m = start ? my_c : cand[my_c];
      const int j0 = m << l;
      const int j1 = min(min((m + 1) << l, g.nb), i);
      const float nval = (float)(min((int64_t)j1 * g.b, (int64_t)g.N) - (int64_t)j0 * g.b);
      const float sc = (m2 + __log2f(s2)) * 0.6931471805599453f + __logf(nval);
      keys[my_c] = ((unsigned long long)float_order_key(sc) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)m);
    }
    __syncthreads();
    // ---- keep the best: rank = number of strictly larger keys
    const int want = l > 0 ? g.cap / 2 : g.topk;
    const int keep = min(want, nc);
    if (my_c >= 0 && my_c < nc) {
      const unsigned long long k = keys[my_c];
      int rank = 0;
      for (int c = 0; c < nc; c++) rank += keys[c] > k;
      if (rank < keep) kept[rank] = (int)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull));
      if (rank == keep - 1) s_edge[0] = key_score(k);
      if (rank == keep) s_edge[1] = key_score(k);
    }
    __syncthreads();
    if (l > 0) {
      // children of the kept nodes that exist and start before block i, compacted by warp 0
      if (warp == 0) {
        if (lane == 0 && keep < nc && keep > 0) *s_gap = fminf(*s_gap, s_edge[0] - s_edge[1]);
        int base = 0;
        for (int k0 = 0; k0 < keep; k0 += 32) {
          const int k = k0 + lane;
          int m = -1, cnt = 0;
          if (k < keep) {
            m = kept[k];
            cnt = 1 + ((2 * m + 1 < g.lvl_n[l - 1] && ((2 * m + 1) << (l - 1)) < i) ? 1 : 0);
          }
          int incl = cnt;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          const int pos = base + incl - cnt;
          if (cnt > 0) cand[pos] = 2 * m;
          if (cnt > 1) cand[pos + 1] = 2 * m + 1;
          base += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) *s_nc = base;
      }
      __syncthreads();
    } else {
      // the kept blocks in ascending order, then -1
      if (threadIdx.x == 0 && keep < nc && keep > 0) *s_gap = fminf(*s_gap, s_edge[0] - s_edge[1]);
      for (int k = threadIdx.x; k < g.topk; k += kThreads) {
        if (k < keep) {
          const int m = kept[k];
          int pos = 0;
          for (int k2 = 0; k2 < keep; k2++) pos += kept[k2] < m;
          out[pos] = m;
        } else {
          out[k] = -1;
        }
      }
      __syncthreads();
      if (gap_out && threadIdx.x == 0) gap_out[(size_t)unit * g.nqb + qb] = *s_gap;
    }
  }

  // ---- teardown
  if (threadIdx.x == 0 && nphase > 0 && !ok) {
    // the last MMA batch may still be in flight after an abort: let it finish
    umma_commit(bar_mma);
    volatile int no_abort = 0;
    mbar_wait(bar_mma, nphase & 1, &no_abort);
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) report(status, PYR_ETIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tD, tcols);
  }
}

template <int MC>
cudaError_t launch_mc(const Geo& g, const CUtensorMap& mq, const __nv_bfloat16* pyr, int32_t* idx, float* gap,
                      int* status, cudaStream_t st) {
  const SelPlan L = sel_plan(g.G * g.b, MC, g.s0 + 1, 128);
  auto kern = select_tc_kernel<MC>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
  if (e != cudaSuccess) return e;
  dim3 grid(g.nqb, g.B * g.Hkv);
  kern<<<grid, kThreads, L.total, st>>>(mq, pyr, idx, gap, status, g);
  return cudaGetLastError();
}

}  // namespace

bool select_tc_supported(const Geo& g) {
  if (g.dtype != PYR_BF16 || g.d != 128 || g.Nq == 1) return false;
  if (g.b % 64 != 0) return false;
  const int R = g.G * g.b;
  if (R != 64 && R != 128 && R != 256) return false;
  if (g.q_offset % g.b != 0) return false;
  const int MC = g.cap <= 64 ? 64 : 128;
  return sel_plan(R, MC, g.s0 + 1, 128).total <= 227 * 1024;
}

cudaError_t launch_select_tc(const Geo& g, const void* Q, const __nv_bfloat16* pyr, int32_t* idx, float* gap,
                             int* status, cudaStream_t st) {
  CUtensorMap mq;
  if (!tc::make_tmap_bf16_3d(&mq, Q, g.d, g.Nq, g.B * g.Hq)) return cudaErrorInvalidValue;
  if (g.cap <= 64) return launch_mc<64>(g, mq, pyr, idx, gap, status, st);
  return launch_mc<128>(g, mq, pyr, idx, gap, status, st);
}

}  // namespace pyr
