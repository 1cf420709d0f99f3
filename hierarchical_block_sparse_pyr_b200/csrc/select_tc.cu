// Coarse-to-fine LogSumExp top-K key-block selection with the scoring GEMM on
// the tcgen05 tensor cores (PISA abstract: start at the coarsest level, score
// a bounded candidate set with LogSumExp, pass the survivors' children to the
// next finer level; routes only to strictly preceding blocks, -1 padding,
// PHBA A.1.2).
//
// One CTA (4 warps) per (batch, kv head, query block i). The walk is a chain
// of dependent levels, so the kernel is built for latency: per level it takes
// five block-wide barriers and one batch of MMAs. A level that has no more
// valid candidates than it keeps (cap/2, or topk at level 0) passes all of
// them on whatever their scores, so it skips gather, score and LogSumExp and
// ranks the candidates by node index (three barriers).
//   prologue the G*b query rows are staged once by TMA (the N operand); the
//            start level's candidates are requested at once; the nodes that
//            straddle block i (one per level) get the exact means of their
//            parts before i, from the binary decomposition of [m 2^l, i) into
//            whole finer nodes, stored as (hi, lo) rows in shared memory;
//   gather   the <= cap candidate rows are copied (cp.async, 16 bytes per
//            thread) straight from the pyramid, which already stores every
//            mean as a bf16 (hi, lo) pair, to their places in the
//            128B-swizzled K-major A operands (the straddling node's row from
//            shared memory);
//   score    D[candidate][row] = kbar . q_row on the tensor cores, as
//            A_hi * Q^T + A_lo * Q^T (M = candidate slots: 64 or 128, N = G*b,
//            K = d), fp32 accumulation in tensor memory. Each TMEM lane holds
//            one candidate's dot products with every query row, so the
//            LogSumExp over rows is a per-thread reduction (one pass, online
//            max); S = LSE(q.kbar / sqrt(d)) + ln n_valid;
//   select   a parallel rank count over packed 64-bit keys (order-preserving
//            score bits over the inverted node index: ties go to the lower
//            index) keeps cap/2 (levels > 0) or topk (level 0); the kept node
//            of rank r writes its children to candidate slots 2r and 2r + 1
//            (-1 for a child that does not exist or starts at or after block i).
// q is exactly representable in bf16, so the only rounding beyond fp32
// accumulation is the hi/lo split of the means.
// The PHAROS variants (select_opts.cuh) change only the ranking score (RCG:
// the parent's ranking score is added), the level-0 keep count (DBA budget,
// FCF fallback: level 0 then publishes the scores by rank and takes one more
// barrier to decide) and, with a trace, what is written per level.
#include "pyr_common.cuh"
#include "select_opts.cuh"
#include "tc_util.cuh"

namespace pyr {

namespace {

using namespace tc;

constexpr int kThreads = 128;
constexpr int kMaxCap = 128;
constexpr int kMaxLevels = 16;  // scored levels: s0 + 1 <= 16 (nb <= 2^15 * cap)

// Candidate rows of the scoring MMA. A candidate's mean is the pair (hi, lo).
// STACK: both rows go into one A operand, in the same quarter of the M rows (so in the
//   same warp's TMEM lanes): quarter q holds H = MC/8 candidates, their hi rows first, then
//   their lo rows; one tile of MC rows scores CPT = MC/2 candidates, and the lane pair adds
//   hi + lo with a shuffle. For caps that leave M rows empty otherwise (cap <= MC/2).
// !STACK: hi rows and lo rows are two A operands with the candidate at the same row, both
//   MMAs accumulate into one D; one tile scores CPT = MC candidates (cap = MC).
template <int MC, int NT, bool STACK>
struct SelCfg {
  static constexpr int CPT = STACK ? MC / 2 : MC;       // candidates per tile
  static constexpr int H = STACK ? MC / 8 : MC / 4;     // candidates per TMEM warp quarter
  static constexpr int kAOp = MC * 256;                 // one operand: [2 d-halves][MC rows][128 B]
  static constexpr int kATile = STACK ? kAOp : 2 * kAOp;
  static constexpr int kMinBlocks = MC == 64 ? 5 : 2;
};

struct SelPlan {
  int q, a, ppair, keys, cand, kept, sbr, psc, misc, bars, total;
};

// R: query rows (N of the MMA); a_bytes: the A tiles; levels: s0 + 1.
__host__ __device__ inline SelPlan sel_plan(int R, int a_bytes, int levels, int d) {
  SelPlan p;
  int o = 0;
  p.q = o;     o += R * d * 2;           // [2 halves][R][128 B]
  p.a = o;     o += a_bytes;             // NT x [2 halves][MC][128 B]
  p.ppair = o; o += levels * d * 4;      // straddling-node means as (hi, lo) rows, [level][2][d] bf16
  p.keys = o;  o += (kMaxCap + 8) * 8;
  p.cand = o;  o += kMaxCap * 4;
  p.kept = o;  o += kMaxCap * 4;
  p.sbr = o;   o += kMaxCap * 4;         // level-0 ranking scores by rank (fallback decision)
  p.psc = o;   o += kMaxCap * 4;         // parent's ranking score per candidate slot (guidance)
  p.misc = o;  o += 64;                  // gap, tmem slot, abort flag, boundary scores, confidence
  p.bars = o;  o += 16;                  // q_full, mma_done
  p.total = o + 1024;                    // + alignment slack
  return p;
}

__device__ __forceinline__ float key_score(unsigned long long k) {
  const uint32_t u = (uint32_t)(k >> 32);
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

// Byte offset, inside the A tiles, of 16-byte chunk q (0..15: hi elements 8q..8q+7;
// 16..31: the same elements of lo) of candidate slot c (128B-swizzled, K-major).
template <int MC, int NT, bool STACK>
__device__ __forceinline__ int a_chunk_off(int c, int q) {
  using C = SelCfg<MC, NT, STACK>;
  const int t = c / C::CPT, cc = c - t * C::CPT;
  int row, op;
  if (STACK) {
    const int quarter = cc / C::H, w = cc - quarter * C::H;
    row = quarter * (MC / 4) + (q >= 16 ? C::H : 0) + w;
    op = 0;
  } else {
    row = cc;
    op = q >= 16 ? C::kAOp : 0;
  }
  const int q16 = q & 15, h = q16 >> 3, c8 = q16 & 7;
  return t * C::kATile + op + h * (MC * 128) + (row >> 3) * 1024 + (row & 7) * 128 + ((c8 ^ (row & 7)) << 4);
}

template <int MC, int NT, bool STACK>
__global__ void __launch_bounds__(kThreads, SelCfg<MC, NT, STACK>::kMinBlocks)
    select_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __nv_bfloat16* __restrict__ pyr,
                     int32_t* __restrict__ idx, float* __restrict__ gap_out, int* status, Geo g, SelOpts o) {
  using C = SelCfg<MC, NT, STACK>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_align<1024>(smem_raw);
  const int R = g.G * g.b;  // query rows of a full block (N of the MMA)
  const SelPlan L = sel_plan(R, NT * C::kATile, g.s0 + 1, 128);
  unsigned char* sQ = smem + L.q;
  unsigned char* sA = smem + L.a;
  unsigned char* ppair = smem + L.ppair;
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(smem + L.keys);
  int* cand = reinterpret_cast<int*>(smem + L.cand);
  int* kept = reinterpret_cast<int*>(smem + L.kept);
  float* s_gap = reinterpret_cast<float*>(smem + L.misc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 8);
  float* s_edge = reinterpret_cast<float*>(smem + L.misc + 16);  // [0]: last kept, [1]: first dropped
  float* s_conf = reinterpret_cast<float*>(smem + L.misc + 32);  // smallest margin above level 0
  float* sbr = reinterpret_cast<float*>(smem + L.sbr);
  float* psc = reinterpret_cast<float*>(smem + L.psc);
  uint64_t* bar_q = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* bar_mma = bar_q + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qb = blockIdx.x, unit = blockIdx.y;
  const int bi = unit / g.Hkv, hk = unit % g.Hkv;
  const int i = g.i0 + qb;
  const int p0 = max(i * g.b, g.q_offset);
  const int rb = min((i + 1) * g.b, g.q_offset + g.Nq) - p0;  // valid rows per head
  const int tcols = NT * R <= 64 ? 64 : (NT * R <= 128 ? 128 : (NT * R <= 256 ? 256 : 512));
  // scoring role of this thread: TMEM lane `lane` of warp `warp` holds, in each tile t, the hi
  // (role 0) or lo (role 1) dot products of candidate t*CPT + warp*H + (lane % H) (STACK), or
  // their sum for candidate t*CPT + warp*32 + lane (!STACK, role 0)
  const bool scorer = STACK ? lane < 2 * C::H : true;
  const int role = STACK ? (lane / C::H) & 1 : 0;
  const int my_cq = warp * C::H + (lane % C::H);  // candidate within a tile
  const __nv_bfloat16* pu = pyr + (size_t)unit * g.P * 256;
  auto straddler = [&](int l) { return (l > 0 && (i & ((1 << l) - 1)) != 0) ? (i >> l) : -1; };

  if (tid == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    *abort_flag = 0;
    *s_gap = __int_as_float(0x7f800000);
    *s_conf = __int_as_float(0x7f800000);
  }
  const int base = sel_base_budget(o, g, unit);  // level-0 budget before any fallback
  const bool rcg = o.rcg_lambda != 0.f;
  // gather targets: thread tid copies 16-byte chunk q = lane of candidate slots c = warp + 4k; with
  // stacked operands (at most 64 slots) the swizzled destinations depend only on (c, q) and are
  // computed once here instead of at every level
  constexpr int kPer = STACK ? NT * C::CPT / 4 : 1;
  int goff[kPer];
  if (STACK) {
#pragma unroll
    for (int k = 0; k < kPer; k++) goff[k] = a_chunk_off<MC, NT, STACK>(warp + 4 * k, lane);
  }
  // separate hi / lo operands (one tile of MC rows): slot c = warp + 4k is row c, so its destination is
  // a per-thread base + (k / 2) 8-row groups + one of two in-group offsets (row & 7 = warp + 4 (k & 1))
  int ns_base = 0, ns_par0 = 0, ns_par1 = 0;
  if (!STACK) {
    const int q16 = lane & 15, c8 = q16 & 7;
    ns_base = (lane >= 16 ? C::kAOp : 0) + (q16 >> 3) * (MC * 128);
    ns_par0 = warp * 128 + ((c8 ^ warp) << 4);
    ns_par1 = (warp + 4) * 128 + ((c8 ^ (warp + 4)) << 4);
  }
  // start level s0: every node that begins before block i, node m in slot m
  int nc = min(g.lvl_n[g.s0], (i + (1 << g.s0) - 1) >> g.s0);
  {
    const int ms = straddler(g.s0);
    if (STACK) {
      const __nv_bfloat16* src = pu + (size_t)g.lvl_off[g.s0] * 256 + lane * 8;
#pragma unroll
      for (int k = 0; k < kPer; k++) {
        const int c = warp + 4 * k;
        if (c < nc && c != ms) cp_async16(sA + goff[k], src + (size_t)c * 256);
      }
    } else {
      const __nv_bfloat16* src = pu + (size_t)g.lvl_off[g.s0] * 256 + lane * 8;
#pragma unroll 4
      for (int k = 0; k < MC / 4; k++) {
        const int c = warp + 4 * k;
        if (c >= nc) break;
        if (c != ms) cp_async16(sA + ns_base + (k >> 1) * 1024 + ((k & 1) ? ns_par1 : ns_par0), src + (size_t)c * 256);
      }
    }
  }
  __syncthreads();  // barrier init visible before the TMA uses it
  if (tid == 0) {
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
  // exact means of the straddling nodes' parts before i, levels 1..s0, stored as (hi, lo)
  // rows: [m 2^l, i) is the union of the whole level-(l'-1) nodes (i >> (l'-1)) - 1 for the
  // set bits l'-1 < l of i; all their loads are issued before any is used
  {
    const int e = tid;  // d = 128 = kThreads: one element per thread
    float v[kMaxLevels];
#pragma unroll
    for (int l = 1; l < kMaxLevels; l++)
      v[l] = (l <= g.s0 && ((i >> (l - 1)) & 1))
                 ? split_load(pu + (size_t)(g.lvl_off[l - 1] + (i >> (l - 1)) - 1) * 256, 128, e) * (float)(g.b << (l - 1))
                 : 0.f;
    float acc = 0.f;
    __nv_bfloat16* pp = reinterpret_cast<__nv_bfloat16*>(ppair);
#pragma unroll
    for (int l = 1; l < kMaxLevels; l++) {
      if (l > g.s0) break;
      acc += v[l];
      const int cnt = i - ((i >> l) << l);
      const float x = cnt > 0 ? acc / (float)(cnt * g.b) : 0.f;
      const __nv_bfloat16 hi = __float2bfloat16_rn(x);
      pp[l * 256 + e] = hi;
      pp[l * 256 + 128 + e] = __float2bfloat16_rn(x - __bfloat162float(hi));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  {
    // the start level's straddling node (slot = its index) from its (hi, lo) row
    const int ms = straddler(g.s0);
    if (ms >= 0 && ms < nc && tid < 32)
      *reinterpret_cast<uint4*>(sA + a_chunk_off<MC, NT, STACK>(ms, tid)) =
          *reinterpret_cast<const uint4*>(ppair + g.s0 * 512 + tid * 16);
  }
  const uint32_t tD = *tmem_slot;
  const uint32_t my_lane_addr = tD + ((uint32_t)(warp * 32) << 16);
  const float sl2 = rsqrtf((float)g.d) * 1.4426950408889634f;
  const uint32_t idesc = idesc_bf16_f32(MC, R, 0, 0);
  // shared-memory descriptors of the operands' first K step; the K steps add fixed offsets
  const uint64_t dQ0 = sdesc_sw128(smem_u32(sQ), 16, 1024), dA0 = sdesc_sw128(smem_u32(sA), 16, 1024);
  const uint32_t q_half = (uint32_t)R * 8;  // a d-half of Q, in 16-byte units
  bool ok = true;
  if (tid == 0) ok = mbar_wait(bar_q, 0, abort_flag);
  ok = __syncthreads_and(ok);
  int nphase = 0;
  int32_t* out = idx + ((size_t)unit * g.nqb + qb) * g.topk;

  // valid candidate slots of the level about to run: every start-level node begins before block i;
  // below, every kept node's left child does, and the rank step counts the valid right children
  int n_valid_next = nc;
  for (int l = g.s0; l >= 0 && ok; l--) {
    const bool start = (l == g.s0);
    // this thread's slot (rank phase: slot = tid) and its node; with at most 32 slots (M = 64,
    // stacked rows) four threads share slot tid / 4 in the rank count
    // stacked operands hold at most CPT = 32 or 64 slots: TPS = 4 or 2 threads share a slot in the rank
    constexpr int TPS = STACK ? kThreads / C::CPT : 1;
    constexpr bool kSplit = TPS > 1;
    const int slot_m = tid < nc ? (start ? tid : cand[tid]) : -1;
    const int split_m = (kSplit && tid / TPS < nc) ? (start ? tid / TPS : cand[tid / TPS]) : -1;
    const int n_valid = n_valid_next;
    // keep count, except at level 0 with the fallback on, where it can grow after scoring
    const int keep_lo = min(l > 0 ? g.cap / 2 : base, n_valid);
    int32_t* trow = o.trace ? sel_trace_row(o, g, unit, qb, l) : nullptr;
    if (keep_lo == n_valid && !rcg) {
      // every valid candidate survives this level whatever its score: no scoring. Keys that
      // rank the candidates by node index (a fixed score, index tie-break) hand the same set on
      for (int c = tid; c < nc; c += kThreads) {
        const int m = start ? c : cand[c];
        keys[c] = m >= 0 ? (0x80000000ull << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)m) : 0ull;
      }
      cp_async_wait_all();  // the start level's gather, if this is the start level
    } else {
    // ---- gather (levels below the start): every thread copies 16-byte chunks of the
    // candidates' (hi, lo) rows with cp.async straight to their swizzled places in the A
    // operand; the straddling node's row comes from shared memory instead; empty slots (-1)
    // are left as they are: their D rows are never read
    if (!start) {
      const int ms = straddler(l);
      if (STACK) {
        const __nv_bfloat16* src = pu + (size_t)g.lvl_off[l] * 256 + lane * 8;
        const uint4 strad = *reinterpret_cast<const uint4*>(ppair + l * 512 + lane * 16);
#pragma unroll
        for (int k = 0; k < kPer; k++) {
          const int c = warp + 4 * k;
          const int m = c < nc ? cand[c] : -1;
          if (m < 0) continue;
          if (m == ms)
            *reinterpret_cast<uint4*>(sA + goff[k]) = strad;
          else
            cp_async16(sA + goff[k], src + (size_t)m * 256);
        }
      } else {
        const __nv_bfloat16* src = pu + (size_t)g.lvl_off[l] * 256 + lane * 8;
        const uint4 strad = *reinterpret_cast<const uint4*>(ppair + l * 512 + lane * 16);
#pragma unroll 4
        for (int k = 0; k < MC / 4; k++) {
          const int c = warp + 4 * k;
          if (c >= nc) break;
          const int m = cand[c];
          if (m < 0) continue;
          unsigned char* dst = sA + ns_base + (k >> 1) * 1024 + ((k & 1) ? ns_par1 : ns_par0);
          if (m == ms)
            *reinterpret_cast<uint4*>(dst) = strad;
          else
            cp_async16(dst, src + (size_t)m * 256);
        }
      }
    }
    cp_async_wait_all();
    fence_proxy_async_smem();
    __syncthreads();
    const int ntiles = (nc + C::CPT - 1) / C::CPT;  // tiles holding at least one candidate
    // ---- score on the tensor cores: D_t = A_t Q^T (hi and lo rows of the candidates of
    // tile t), 8 K steps of 16 per tile
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int t = 0; t < NT; t++) {
        if (t >= ntiles) break;
#pragma unroll
        for (int kk = 0; kk < 8; kk++) {
          const uint32_t oq = (kk >> 2) * q_half + (kk & 3) * 2;
          const uint32_t oa = (t * C::kATile + (kk >> 2) * (MC * 128)) / 16 + (kk & 3) * 2;
          umma_bf16(tD + t * R, dA0 + oa, dQ0 + oq, idesc, kk > 0);
          if (!STACK) umma_bf16(tD + t * R, dA0 + oa + C::kAOp / 16, dQ0 + oq, idesc, 1);
        }
      }
      umma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, nphase & 1, abort_flag);
    ok = __syncthreads_and(ok);  // block-uniform: the loop below has block-wide barriers
    nphase++;
    if (!ok) break;
    tc_fence_after();
    // ---- LogSumExp over the valid query rows. The two lanes of a candidate (hi, lo) swap
    // halves of every 64-column batch with one shuffle each, so that each holds hi + lo for 32
    // columns; each keeps an online max and sum over its columns, and the pair merges at the end
    const bool full = (rb == g.b);
    if constexpr (STACK && MC == 64) {
      // M = 64 stacked rows: an M = 64 accumulator fills lanes 0-15 of each warp's TMEM sub-partition,
      // 8 candidates' hi rows in lanes 0-7 and their lo rows in lanes 8-15. The 16-lane TMEM load hands
      // thread t the hi row (lane t/4) and the lo row (lane t/4 + 8) of one candidate at the same two
      // columns of every eight, so hi + lo is thread-local and four threads split the candidate's query
      // rows. (The same load over the M = 128 stacked layout, two 16-lane groups per warp with the rows
      // regrouped to match, measured slower at 64K than the 32-lane load with a shuffle: 1.386 -> 1.457 ms.)
      const int cb = 2 * (lane & 3);
      {
        const int c = warp * C::H + (lane >> 2);
        const uint32_t grp_addr = my_lane_addr;
        float m2 = -INFINITY, s2 = 0.f;
        if (ntiles > 0 && __any_sync(0xffffffffu, c < nc)) {  // warp-uniform
#pragma unroll 1
          for (int c0 = 0; c0 < R; c0 += 64) {
            uint32_t r[32];
            tmem_ld16x256b_x8(grp_addr + c0, r);
            tmem_wait_ld();
            float x[16];
#pragma unroll
            for (int k = 0; k < 8; k++) {
              x[2 * k] = __uint_as_float(r[4 * k]) + __uint_as_float(r[4 * k + 2]);
              x[2 * k + 1] = __uint_as_float(r[4 * k + 1]) + __uint_as_float(r[4 * k + 3]);
            }
            if (!full) {
#pragma unroll
              for (int k = 0; k < 16; k++) x[k] = ((c0 + 8 * (k >> 1) + cb + (k & 1)) % g.b) < rb ? x[k] : -INFINITY;
            }
            float a[6];
#pragma unroll
            for (int k = 0; k < 5; k++) a[k] = fmax3(x[3 * k], x[3 * k + 1], x[3 * k + 2]);
            a[5] = x[15];
            const float bm = fmax3(fmax3(a[0], a[1], a[2]), a[3], fmaxf(a[4], a[5])) * sl2;
            const float mn = fmaxf(m2, bm);
            if (mn != -INFINITY) {
              s2 *= ex2(m2 - mn);  // 0 on the first valid batch (m2 = -inf)
              m2 = mn;
              const float2 scl = make_float2(sl2, sl2), off = make_float2(-m2, -m2);
              float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
              for (int k = 0; k < 8; k++) {
                const float2 y = __ffma2_rn(make_float2(x[2 * k], x[2 * k + 1]), scl, off);
                acc[k & 1] = __fadd2_rn(acc[k & 1], make_float2(ex2(y.x), ex2(y.y)));
              }
              const float2 sum = __fadd2_rn(acc[0], acc[1]);
              s2 += sum.x + sum.y;
            }
          }
        }
        // merge the four threads of the candidate
#pragma unroll
        for (int sh = 1; sh <= 2; sh <<= 1) {
          const float mo = __shfl_xor_sync(0xffffffffu, m2, sh), so = __shfl_xor_sync(0xffffffffu, s2, sh);
          const float M = fmaxf(m2, mo);
          s2 = (m2 == -INFINITY ? 0.f : s2 * ex2(m2 - M)) + (mo == -INFINITY ? 0.f : so * ex2(mo - M));
          m2 = M;
        }
        if ((lane & 3) == 0 && c < nc) {
          const int m = start ? c : cand[c];
          unsigned long long key = 0ull;  // empty slots rank below every node
          if (m >= 0) {
            const int j0 = m << l;
            const int j1 = min(min((m + 1) << l, g.nb), i);
            const float nval = (float)(min((int64_t)j1 * g.b, (int64_t)g.N) - (int64_t)j0 * g.b);
            float sc = (m2 + __log2f(s2)) * 0.6931471805599453f + __logf(nval);
            if (rcg && !start) sc = fmaf(o.rcg_lambda, psc[c], sc);
            key = ((unsigned long long)float_order_key(sc) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)m);
          }
          keys[c] = key;
        }
      }
    } else
#pragma unroll 1
    for (int t = 0; t < ntiles; t++) {
      const int c = t * C::CPT + my_cq;
      if (!__any_sync(0xffffffffu, scorer && c < nc)) continue;  // warp-uniform
      float m2 = -INFINITY, s2 = 0.f;
      float v[64];
      constexpr int NX = STACK ? 32 : 64;  // columns of a 64-column batch that this lane reduces
      for (int c0 = 0; c0 < R; c0 += 64) {
        tmem_ld32(my_lane_addr + t * R + c0, v);
        tmem_ld32(my_lane_addr + t * R + c0 + 32, v + 32);
        tmem_wait_ld();
        if (STACK) {
#pragma unroll
          for (int k = 0; k < 32; k++) {
            const float send = role ? v[k] : v[32 + k];
            const float recv = __shfl_xor_sync(0xffffffffu, send, C::H);
            v[k] = (role ? v[32 + k] : v[k]) + recv;
          }
        }
        const int colb = c0 + role * 32;  // first column of this lane's columns
        if (!full) {
#pragma unroll
          for (int k = 0; k < NX; k++) v[k] = ((colb + k) % g.b) < rb ? v[k] : -INFINITY;
        }
        float a[NX / 3 + 1];
#pragma unroll
        for (int k = 0; k < NX / 3; k++) a[k] = fmax3(v[3 * k], v[3 * k + 1], v[3 * k + 2]);
        a[NX / 3] = NX % 3 == 2 ? fmaxf(v[NX - 2], v[NX - 1]) : v[NX - 1];
        float bm = a[0];
#pragma unroll
        for (int k = 1; k < NX / 3 + 1; k++) bm = fmaxf(bm, a[k]);
        bm *= sl2;
        const float mn = fmaxf(m2, bm);
        if (mn == -INFINITY) continue;  // nothing valid yet in this lane's columns
        s2 *= ex2(m2 - mn);             // 0 on the first valid batch (m2 = -inf)
        m2 = mn;
        const float2 scl = make_float2(sl2, sl2), off = make_float2(-m2, -m2);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int k = 0; k < NX / 2; k++) {
          const float2 y = __ffma2_rn(make_float2(v[2 * k], v[2 * k + 1]), scl, off);
          acc[k & 3] = __fadd2_rn(acc[k & 3], make_float2(ex2(y.x), ex2(y.y)));
        }
        const float2 sum = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
        s2 += sum.x + sum.y;
      }
      // merge the pair's (max, sum)
      float M = m2, S = s2;
      if (STACK) {
        const float mo = __shfl_xor_sync(0xffffffffu, m2, C::H), so = __shfl_xor_sync(0xffffffffu, s2, C::H);
        M = fmaxf(m2, mo);
        S = (m2 == -INFINITY ? 0.f : s2 * ex2(m2 - M)) + (mo == -INFINITY ? 0.f : so * ex2(mo - M));
      }
      if (scorer && role == 0 && c < nc) {
        const int m = start ? c : cand[c];
        unsigned long long key = 0ull;  // empty slots rank below every node
        if (m >= 0) {
          const int j0 = m << l;
          const int j1 = min(min((m + 1) << l, g.nb), i);
          const float nval = (float)(min((int64_t)j1 * g.b, (int64_t)g.N) - (int64_t)j0 * g.b);
          float sc = (M + __log2f(S)) * 0.6931471805599453f + __logf(nval);
          if (rcg && !start) sc = fmaf(o.rcg_lambda, psc[c], sc);
          key = ((unsigned long long)float_order_key(sc) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)m);
        }
        keys[c] = key;
      }
    }
    }  // scored level
    tc_fence_before();
    const int nc8 = (nc + 7) & ~7;
    if (tid >= nc && tid < (kSplit ? C::CPT : nc8)) keys[tid] = 0ull;  // zero pad for the 8-wide reads
    __syncthreads();
    // ---- keep the best: rank = number of strictly larger keys (keys are distinct: they hold the
    // node index); a kept node of rank r puts its children (those that exist and start before
    // block i; -1 otherwise) in slots 2r, 2r + 1
    int my_rank = -1, my_node = -1;
    unsigned long long my_key = 0ull;
    if (kSplit) {
      // slot tid / TPS: each of its TPS threads counts the larger keys among CPT / TPS of the CPT
      constexpr int KPP = C::CPT / TPS;
      const int sl = tid / TPS, part = tid % TPS;
      const unsigned long long k_sl = keys[sl];
      const ulonglong2* k2 = reinterpret_cast<const ulonglong2*>(keys) + part * (KPP / 2);
      int rank = 0;
#pragma unroll
      for (int u = 0; u < KPP / 2; u++) {
        const ulonglong2 a = k2[u];
        rank += (a.x > k_sl) + (a.y > k_sl);
      }
      if (split_m < 0) rank = 0;
#pragma unroll
      for (int sh = 1; sh < TPS; sh <<= 1) rank += __shfl_xor_sync(0xffffffffu, rank, sh);
      if (split_m >= 0 && part == 0) {
        my_rank = rank;
        my_node = split_m;
        my_key = k_sl;
      }
    } else if (slot_m >= 0) {
      my_key = keys[tid];
      int rank = 0;
      const ulonglong2* k2 = reinterpret_cast<const ulonglong2*>(keys);
      for (int c = 0; c < nc8 / 2; c += 4) {
        const ulonglong2 a0 = k2[c], a1 = k2[c + 1], a2 = k2[c + 2], a3 = k2[c + 3];
        rank += (a0.x > my_key) + (a0.y > my_key) + (a1.x > my_key) + (a1.y > my_key) + (a2.x > my_key) +
                (a2.y > my_key) + (a3.x > my_key) + (a3.y > my_key);
      }
      my_rank = rank;
      my_node = slot_m;
    }
    int keep = keep_lo;
    float decision_margin = __int_as_float(0x7f800000);
    if (l == 0 && o.fcf_extra > 0 && keep_lo < n_valid) {  // block-uniform
      if (my_rank >= 0) sbr[my_rank] = key_score(my_key);
      __syncthreads();
      keep = sel_fcf_keep(o, g, base, n_valid, sbr, *s_conf, &decision_margin);
    }
    bool right_valid = false;
    if (my_rank >= 0) {
      if (my_rank < keep) {
        if (l > 0) {
          const int c1 = 2 * my_node + 1;
          right_valid = c1 < g.lvl_n[l - 1] && (c1 << (l - 1)) < i;
          cand[2 * my_rank] = 2 * my_node;
          cand[2 * my_rank + 1] = right_valid ? c1 : -1;
          if (rcg) psc[2 * my_rank] = psc[2 * my_rank + 1] = key_score(my_key);
        } else {
          kept[my_rank] = my_node;
        }
        if (trow) trow[my_rank] = my_node;
      }
      if (my_rank == keep - 1) s_edge[0] = key_score(my_key);
      if (my_rank == keep) s_edge[1] = key_score(my_key);
    }
    if (trow && tid >= keep && tid < o.tw) trow[tid] = -1;
    n_valid_next = keep + __syncthreads_count(right_valid);  // also the barrier before the next level
    if (tid == 0) {
      if (keep < n_valid && keep > 0) {
        const float mg = s_edge[0] - s_edge[1];
        *s_gap = fminf(*s_gap, mg);
        if (l > 0) *s_conf = fminf(*s_conf, mg);
      }
      *s_gap = fminf(*s_gap, decision_margin);
    }
    nc = 2 * keep;
    if (l == 0) {
      // the kept blocks in ascending order, then -1
      for (int k = tid; k < g.topk; k += kThreads) {
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
      if (gap_out && tid == 0) gap_out[(size_t)unit * g.nqb + qb] = *s_gap;
    }
  }

  // ---- teardown
  if (tid == 0 && nphase > 0 && !ok) {
    // the last MMA batch may still be in flight after an abort: let it finish
    umma_commit(bar_mma);
    volatile int no_abort = 0;
    mbar_wait(bar_mma, nphase & 1, &no_abort);
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && tid == 0) report(status, PYR_ETIMEOUT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tD, tcols);
  }
}

template <int MC, int NT, bool STACK>
cudaError_t launch_mc(const Geo& g, const CUtensorMap& mq, const __nv_bfloat16* pyr, int32_t* idx, float* gap,
                      int* status, const SelOpts& o, cudaStream_t st) {
  const SelPlan L = sel_plan(g.G * g.b, NT * SelCfg<MC, NT, STACK>::kATile, g.s0 + 1, 128);
  auto kern = select_tc_kernel<MC, NT, STACK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
  if (e != cudaSuccess) return e;
  dim3 grid(g.nqb, g.B * g.Hkv);
  kern<<<grid, kThreads, L.total, st>>>(mq, pyr, idx, gap, status, g, o);
  return cudaGetLastError();
}

// the A operand bytes for a cap: stacked M=64 (cap <= 32), stacked M=128 (cap <= 64), or
// separate hi and lo M=128 operands (cap <= 128)
inline int sel_a_bytes(int cap) { return cap <= 32 ? 64 * 256 : (cap <= 64 ? 128 * 256 : 2 * 128 * 256); }

}  // namespace

bool select_tc_supported(const Geo& g) {
  if (g.dtype != PYR_BF16 || g.d != 128 || g.Nq == 1) return false;
  if (g.b % 64 != 0) return false;
  const int R = g.G * g.b;
  if (R != 64 && R != 128 && R != 256) return false;
  if (g.q_offset % g.b != 0) return false;
  if (g.s0 >= kMaxLevels) return false;
  return sel_plan(R, sel_a_bytes(g.cap), g.s0 + 1, 128).total <= 227 * 1024;
}

cudaError_t launch_select_tc(const Geo& g, const void* Q, const __nv_bfloat16* pyr, int32_t* idx, float* gap,
                             int* status, const SelOpts& o, cudaStream_t st) {
  CUtensorMap mq;
  if (!tc::make_tmap_bf16_3d(&mq, Q, g.d, g.Nq, g.B * g.Hq)) return cudaErrorInvalidValue;
  if (g.cap <= 32) return launch_mc<64, 1, true>(g, mq, pyr, idx, gap, status, o, st);
  if (g.cap <= 64) return launch_mc<128, 1, true>(g, mq, pyr, idx, gap, status, o, st);
  return launch_mc<128, 1, false>(g, mq, pyr, idx, gap, status, o, st);
}

}  // namespace pyr
