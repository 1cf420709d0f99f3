// PHBA prefix states (PHBA summary, 2.2 "Gated slot memory", 3.2 "Prefix-state
// construction", A.1.1 "Chunkwise parallel prefix-state memory construction").
//
// Per (batch, kv head) unit, M-slot key and value states follow
//   S[s] <- a_t[s] S[s] + w_t[s] x_t        (x = the state-branch key, or V)
// from zero, and the state of key block j is S after the tokens before j b.
// The chunkwise form the summary describes (only boundary states are carried
// from chunk to chunk; within a chunk the writes are a matrix product, with
// log-A sums for stability) is what runs here, with the chunk = one key block:
//   pass A, one CTA per (block j, unit), all blocks in parallel:
//     R_t[s] = sum_{t' > t in the block} log a_t'[s]   (log-A suffix sums)
//     U_j[s][e] = sum_t w_t[s] exp(R_t[s]) x_t[e]      (for x = K and x = V)
//     D_j[s] = exp(sum over the block of log a_t[s])    (the block's decay)
//   pass B, one thread per (unit, slot, element), over the blocks in order:
//     P_0 = 0,  P_{j+1} = D_j P_j + U_j,  P_j written in the input dtype.
// A zero retention gives log 0 = -inf and exp(-inf) = 0, so no infinity is ever
// subtracted from another. Arithmetic is fp32; U and D live in a caller-owned
// workspace.
// With bf16 inputs, d = 128, b = 64 and M a multiple of 32, a single kernel
// replaces both passes (phba_carry_tc_kernel below): each CTA carries its part
// of the state through the blocks in order, the block products run on the
// tcgen05 tensor cores, and U and D never leave the chip (no workspace
// traffic, which in the two-pass form was 2 x 4 bytes per state element).
#include "pyr_common.cuh"
#include "tc_util.cuh"

namespace pyr {

namespace {

constexpr int kThreads = 256;
constexpr int kSlotGroup = 64;  // slots per pass of a pass-A CTA

struct PhbaWs {
  size_t u_bytes, d_bytes, total;
};

__host__ __device__ inline PhbaWs phba_ws(int units, int nb, int M, int D) {
  PhbaWs w;
  w.u_bytes = (size_t)units * nb * 2 * M * D * sizeof(float);
  w.d_bytes = (size_t)units * nb * M * sizeof(float);
  w.total = w.u_bytes + w.d_bytes;
  return w;
}

// Pass A. Shared memory: coef [b][kSlotGroup] fp32 and x [b][D] fp32.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) phba_chunk_kernel(const T* __restrict__ Ks, const T* __restrict__ V,
                                                              const float* __restrict__ A,
                                                              const float* __restrict__ W, int M,
                                                              float* __restrict__ U, float* __restrict__ Dj, Geo g) {
  extern __shared__ __align__(16) float sm[];
  float* coef = sm;                       // [b][kSlotGroup]
  float* xs = coef + g.b * kSlotGroup;    // [b][D]
  const int j = blockIdx.x, unit = blockIdx.y;
  const int t0 = j * g.b, n = min(g.b, g.N - t0);  // tokens of the block
  constexpr int TX = D / 4;                          // threads across d (4 elements each)
  constexpr int TY = kThreads / TX;                  // slot lanes
  const int tx = threadIdx.x % TX, ty = threadIdx.x / TX;
  const float* Au = A + ((size_t)unit * g.N + t0) * M;
  const float* Wu = W + ((size_t)unit * g.N + t0) * M;
  float* Uj = U + ((size_t)unit * g.nb + j) * 2 * M * D;

  for (int s0 = 0; s0 < M; s0 += kSlotGroup) {
    const int ns = min(kSlotGroup, M - s0);
    __syncthreads();  // the previous group's coefficients are consumed
    // log-A suffix sums of the group's slots, one thread per slot walking the block backwards
    if (threadIdx.x < ns) {
      const int s = s0 + threadIdx.x;
      float r = 0.f;  // sum of log a over the tokens after t
      for (int t = n - 1; t >= 0; t--) {
        coef[t * kSlotGroup + threadIdx.x] = Wu[(size_t)t * M + s] * __expf(r);
        r += __logf(Au[(size_t)t * M + s]);
      }
      Dj[((size_t)unit * g.nb + j) * M + s] = __expf(r);
    }
    for (int which = 0; which < 2; which++) {
      const T* X = (which == 0 ? Ks : V) + ((size_t)unit * g.N + t0) * D;
      __syncthreads();  // coef written; xs free
      for (int x = threadIdx.x; x < n * D; x += kThreads) xs[x] = to_f32(X[x]);
      __syncthreads();
      // U[s][4 tx .. 4 tx + 3] for the slots s = s0 + ty + TY k of the group
      constexpr int KS = kSlotGroup / TY;
      float acc[KS][4];
#pragma unroll
      for (int k = 0; k < KS; k++)
#pragma unroll
        for (int c = 0; c < 4; c++) acc[k][c] = 0.f;
      for (int t = 0; t < n; t++) {
        const float4 xv = *reinterpret_cast<const float4*>(xs + t * D + 4 * tx);
#pragma unroll
        for (int k = 0; k < KS; k++) {
          const float c = coef[t * kSlotGroup + ty + TY * k];
          acc[k][0] = fmaf(c, xv.x, acc[k][0]);
          acc[k][1] = fmaf(c, xv.y, acc[k][1]);
          acc[k][2] = fmaf(c, xv.z, acc[k][2]);
          acc[k][3] = fmaf(c, xv.w, acc[k][3]);
        }
      }
#pragma unroll
      for (int k = 0; k < KS; k++) {
        const int sl = ty + TY * k;
        if (sl < ns)
          *reinterpret_cast<float4*>(Uj + ((size_t)which * M + s0 + sl) * D + 4 * tx) =
              make_float4(acc[k][0], acc[k][1], acc[k][2], acc[k][3]);
      }
    }
  }
}

// Pass B: one thread per (slot, element) of one unit, carrying the key and the value state.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) phba_scan_kernel(const float* __restrict__ U,
                                                             const float* __restrict__ Dj, int M,
                                                             T* __restrict__ PK, T* __restrict__ PV, Geo g) {
  const int unit = blockIdx.y;
  const int x = blockIdx.x * kThreads + threadIdx.x;  // s * D + e
  if (x >= M * D) return;
  const int s = x / D;
  float sk = 0.f, sv = 0.f;
  const size_t per = (size_t)M * D;
  const float* Uu = U + (size_t)unit * g.nb * 2 * per;
  const float* Du = Dj + (size_t)unit * g.nb * M;
  T* pk = PK + (size_t)unit * g.nb * per + x;
  T* pv = PV + (size_t)unit * g.nb * per + x;
#pragma unroll 4
  for (int j = 0; j < g.nb; j++) {
    const float uk = Uu[(size_t)j * 2 * per + x], uv = Uu[(size_t)j * 2 * per + per + x];
    const float dj = Du[(size_t)j * M + s];
    if constexpr (sizeof(T) == 4) {
      pk[(size_t)j * per] = sk;
      pv[(size_t)j * per] = sv;
    } else {
      pk[(size_t)j * per] = __float2bfloat16_rn(sk);
      pv[(size_t)j * per] = __float2bfloat16_rn(sv);
    }
    sk = fmaf(dj, sk, uk);
    sv = fmaf(dj, sv, uv);
  }
}

// One pass on the tensor cores, no workspace (bf16, d = 128, b = 64, M a multiple of 32): one CTA per
// (unit, state: keys or values, tile of 32 slots) walks the blocks in order and carries its part of the
// state, P^T [128 d][32 slots] fp32, in registers (thread e of the carry warps holds row e). Per block j:
//   C^T[s][t] = w_t[s] prod_{t' > t in the block} a_t'[s]  (products, not log sums: a zero retention
//               gives an exact 0 either way), D_j[s] = prod_t a_t[s], split into bf16 hi + lo rows;
//   U_j^T = X_j^T C_j^T  on the tensor cores (M = 128 d, N = 32 slots, K = 64 tokens; X_j, the block's
//               keys or values, arrives by TMA as an MN-major A operand), hi and lo into one fp32 result;
//   state j = P (written in the input dtype), then P <- D_j P + U_j.
// Warp roles, each walking the blocks in order, up to kBufs blocks apart:
//   warps 0-3  coefficients: warp q takes tokens 16q .. 16q + 15, lane s slot s; C_j and D_j go to
//              buffer j % kBufs once the carry has released it;
//   warps 4-7  carry: thread e = TMEM lane e; stores state j, reads U_j, updates P;
//   warp 8     producer: gates and X of block j into a kStages-deep ring (TMA);
//   warp 9     MMA issuer: U_j into tensor-memory buffer j % kBufs.
// The carry is the only sequential chain; the buffers let the coefficients and the MMAs of the next
// blocks run while it works (two buffers measured 0.441 ms on the 32K workload with 128 slots, four
// buffers and four stages the figure in the design notes).
struct CarryPlan {
  static constexpr int kStages = 4;
  static constexpr int kBufs = 4;                  // coefficient / U / decay buffers
  static constexpr int kA = 0;                     // per stage: retention gates [64 tokens][32 slots] fp32
  static constexpr int kW = 8192;                  //            write gates, same layout
  static constexpr int kX = 16384;                 //            X [2 d-halves][64 tokens][128 B], 128B swizzle
  static constexpr int kStage = 32768;
  static constexpr int kC = kStages * kStage;      // [buffer][hi, lo][32 slots][64 tokens] bf16, K-major
  static constexpr int kDec = kC + kBufs * 8192;   // [buffer][32] block decays
  static constexpr int kPart = kDec + kBufs * 32 * 4;  // [4 quarters][32] products of a quarter's retentions
  static constexpr int kBar = kPart + 4 * 32 * 4;  // full, free [stage]; c_full, u_full, u_free [buffer]; drain
  static constexpr int kNumBars = 2 * kStages + 3 * kBufs + 1;
  static constexpr int kMisc = kBar + kNumBars * 8;  // tmem slot, abort flag
  static constexpr int kBytes = kMisc + 16 + 1024;   // + alignment slack
  static constexpr int kThreads = 10 * 32;
};

// A bounded mbarrier wait that sleeps 32 ns between polls: the roles of the carry kernel wait on one
// another for most of their time, and polling warps take issue slots from the ones that work (same-box
// A/B at 32K with 128 slots: 0.401 -> 0.383 ms; the same back-off slowed the attention kernel, whose
// waits sit on its critical path, so it is local to this kernel).
__device__ __forceinline__ bool mbar_wait_backoff(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  using namespace tc;
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    __nanosleep(32);
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

// Named barrier 1 over the four coefficient warps, with an AND over their predicates: a wait's outcome
// becomes the same for all of them before their next named barrier, so an abort never strands a warp.
__device__ __forceinline__ bool bar_and_128(bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)p)
      : "memory");
  return r != 0;
}

template <typename T>
__global__ void __launch_bounds__(CarryPlan::kThreads, 1)
    phba_carry_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                         const __grid_constant__ CUtensorMap tmKs, const __grid_constant__ CUtensorMap tmV,
                         T* __restrict__ PK, T* __restrict__ PV, int M, int* status, Geo g) {
  using namespace tc;
  using PL = CarryPlan;
  constexpr int D = 128, BT = 64, NS = 32, NST = PL::kStages, NB = PL::kBufs;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_align<1024>(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PL::kBar);
  uint64_t* bar_full = bars;              // [stage] gates and X landed
  uint64_t* bar_free = bars + NST;        // [stage] the stage's MMA has run
  uint64_t* bar_c_full = bars + 2 * NST;  // [buffer] coefficients written (4 warp arrivals)
  uint64_t* bar_u_full = bar_c_full + NB; // [buffer] U in tensor memory
  uint64_t* bar_u_free = bar_u_full + NB; // [buffer] the carry has read U and D (4 warp arrivals)
  uint64_t* bar_drain = bar_u_free + NB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + PL::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + PL::kMisc + 4);
  float* sdec = reinterpret_cast<float*>(smem + PL::kDec);
  float* spart = reinterpret_cast<float*>(smem + PL::kPart);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int which = blockIdx.x & 1, s0 = (blockIdx.x >> 1) * NS, unit = blockIdx.y;
  const int nb = g.nb;

  if (tid == 0) {
    for (int b = 0; b < PL::kNumBars; b++) mbar_init(bars + b, 1);
    for (int b = 0; b < NB; b++) {
      mbar_init(bar_c_full + b, 4);
      mbar_init(bar_u_free + b, 4);
    }
    fence_mbar_init();
    *abort_flag = 0;
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 32 * NB);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tU = *tmem_slot;  // U_j^T in columns 32 (j % NB) .. + 31, lane = d

  if (warp < 4) {
    // ------------------------------------------------------------ coefficients
    const int q = warp;
    for (int j = 0; j < nb; j++) {
      const int st = j % NST, b = j % NB;
      bool ok = mbar_wait_backoff(bar_full + st, (j / NST) & 1, abort_flag);
      if (ok && j >= NB) ok = mbar_wait_backoff(bar_u_free + b, (j / NB - 1) & 1, abort_flag);  // buffer b is free
      if (!bar_and_128(ok)) break;
      const float* ga = reinterpret_cast<const float*>(smem + st * PL::kStage + PL::kA);
      const float* gw = reinterpret_cast<const float*>(smem + st * PL::kStage + PL::kW);
      const int n = min(BT, g.N - j * BT);  // tokens of the block (the rest arrive as zeros)
      float c[16];
      float r = 1.f;
#pragma unroll
      for (int t = 15; t >= 0; t--) {
        const int tt = 16 * q + t;
        const float a = tt < n ? ga[tt * NS + lane] : 1.f;
        const float w = tt < n ? gw[tt * NS + lane] : 0.f;
        c[t] = w * r;
        r *= a;
      }
      spart[q * NS + lane] = r;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      float later = 1.f;  // the retentions of the quarters after this one
      for (int q2 = q + 1; q2 < 4; q2++) later *= spart[q2 * NS + lane];
      if (q == 0) sdec[b * NS + lane] = r * later;
      unsigned char* cb = smem + PL::kC + b * 8192;
#pragma unroll
      for (int h = 0; h < 2; h++) {  // 16-byte chunk 2q + h holds tokens 16q + 8h .. + 7
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
          const float x0 = c[8 * h + 2 * e] * later, x1 = c[8 * h + 2 * e + 1] * later;
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(x0, x1);
          const __nv_bfloat162 l2 = __floats2bfloat162_rn(x0 - __bfloat162float(h2.x), x1 - __bfloat162float(h2.y));
          hi[e] = *reinterpret_cast<const uint32_t*>(&h2);
          lo[e] = *reinterpret_cast<const uint32_t*>(&l2);
        }
        const int off = lane * 128 + (((2 * q + h) ^ (lane & 7)) << 4);
        *reinterpret_cast<uint4*>(cb + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(cb + 4096 + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      fence_proxy_async_smem();  // the coefficient rows are read by the tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_c_full + b);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ carry
    const int e = tid - 128;  // TMEM lane = row d of the state
    const uint32_t lane_addr = tU + ((uint32_t)((warp - 4) * 32) << 16);
    T* out = (which ? PV : PK) + (size_t)unit * nb * M * D + (size_t)s0 * D + e;
    float P[NS];  // the state rows d = e of the slots s0 .. s0 + 31, before block j
#pragma unroll
    for (int k = 0; k < NS; k++) P[k] = 0.f;
    for (int j = 0; j < nb; j++) {
      const int b = j % NB;
      T* row = out + (size_t)j * M * D;
#pragma unroll
      for (int k = 0; k < NS; k++) {
        if constexpr (sizeof(T) == 4) row[(size_t)k * D] = P[k];
        else row[(size_t)k * D] = __float2bfloat16_rn(P[k]);
      }
      // U_j is in tensor memory; the wait on the coefficient barrier makes D_j, which the coefficient
      // warps wrote before their arrival, visible here
      bool ok = mbar_wait_backoff(bar_u_full + b, (j / NB) & 1, abort_flag);
      if (ok) ok = mbar_wait_backoff(bar_c_full + b, (j / NB) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      float u[NS];
      tmem_ld32(lane_addr + b * 32, u);
      tmem_wait_ld();
      const float* dec = sdec + b * NS;
#pragma unroll
      for (int k = 0; k < NS; k++) P[k] = fmaf(dec[k], P[k], u[k]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_u_free + b);
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ producer: gates and X of block j
    if (lane == 0) {
      const CUtensorMap* tmX = which ? &tmV : &tmKs;
      bool ok = true;
      int j = 0;
      for (; j < nb && ok; j++) {
        const int st = j % NST;
        if (j >= NST) ok = mbar_wait_backoff(bar_free + st, (j / NST - 1) & 1, abort_flag);
        if (!ok) break;
        unsigned char* sb = smem + st * PL::kStage;
        mbar_expect_tx(bar_full + st, 32768);
        tma_load_3d(sb + PL::kA, &tmA, s0, j * BT, unit, bar_full + st);
        tma_load_3d(sb + PL::kW, &tmW, s0, j * BT, unit, bar_full + st);
        tma_load_3d(sb + PL::kX, tmX, 0, j * BT, unit, bar_full + st);
        tma_load_3d(sb + PL::kX + 8192, tmX, 64, j * BT, unit, bar_full + st);
      }
      // drain: the copies of the last (up to) three blocks issued
      volatile int no_abort = 0;
      for (int u = max(0, j - NST); u < j; u++) mbar_wait(bar_full + u % NST, (u / NST) & 1, &no_abort);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, NS, 1, 0);  // A = X^T MN-major, B = C^T K-major
      int issued = 0;
      for (int j = 0; j < nb; j++) {
        const int st = j % NST, b = j % NB;
        bool ok = mbar_wait_backoff(bar_c_full + b, (j / NB) & 1, abort_flag);  // implies the carry freed buffer b
        if (ok) ok = mbar_wait_backoff(bar_full + st, (j / NST) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dX = sdesc_sw128(smem_u32(smem + st * PL::kStage + PL::kX), 8192, 1024);
        const uint64_t dH = sdesc_sw128(smem_u32(smem + PL::kC + b * 8192), 16, 1024);
        const uint64_t dL = sdesc_sw128(smem_u32(smem + PL::kC + b * 8192 + 4096), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; kk++) {  // 16 tokens per step
          umma_bf16(tU + b * 32, dX + (uint64_t)((kk * 2048) >> 4), dH + (uint64_t)((kk * 32) >> 4), idesc, kk > 0);
          umma_bf16(tU + b * 32, dX + (uint64_t)((kk * 2048) >> 4), dL + (uint64_t)((kk * 32) >> 4), idesc, 1);
        }
        umma_commit(bar_u_full + b);
        umma_commit(bar_free + st);
        issued++;
      }
      if (issued > 0) {
        // every MMA issued must finish before tensor memory is freed
        umma_commit(bar_drain);
        volatile int no_abort = 0;
        mbar_wait(bar_drain, 0, &no_abort);
      }
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && tid == 0) report(status, PYR_ETIMEOUT);
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tU, 32 * NB);
  }
}

template <typename T, int D>
cudaError_t launch_t(const Geo& g, int M, const void* Ks, const void* V, const float* A, const float* W, void* PK,
                     void* PV, void* ws, int* status, cudaStream_t st) {
  const PhbaWs L = phba_ws(g.B * g.Hkv, g.nb, M, D);
  float* U = static_cast<float*>(ws);
  float* Dj = reinterpret_cast<float*>(static_cast<char*>(ws) + L.u_bytes);
  cudaError_t e;
  if constexpr (sizeof(T) == 2 && D == 128) {
    if (M % 32 == 0 && g.b == 64) {
      // one pass, no workspace
      CUtensorMap ma, mw, mk, mv;
      if (!tc::make_tmap_f32_3d(&ma, A, M, g.N, g.B * g.Hkv, 32, 64) ||
          !tc::make_tmap_f32_3d(&mw, W, M, g.N, g.B * g.Hkv, 32, 64) ||
          !tc::make_tmap_bf16_3d(&mk, Ks, D, g.N, g.B * g.Hkv) || !tc::make_tmap_bf16_3d(&mv, V, D, g.N, g.B * g.Hkv))
        return cudaErrorInvalidValue;
      auto kc = phba_carry_tc_kernel<T>;
      e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, CarryPlan::kBytes);
      if (e != cudaSuccess) return e;
      kc<<<dim3(2 * (M / 32), g.B * g.Hkv), CarryPlan::kThreads, CarryPlan::kBytes, st>>>(ma, mw, mk, mv, static_cast<T*>(PK),
                                                                           static_cast<T*>(PV), M, status, g);
      return cudaGetLastError();
    }
  }
  const size_t smem = sizeof(float) * ((size_t)g.b * kSlotGroup + (size_t)g.b * D);
  auto ka = phba_chunk_kernel<T, D>;
  e = cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ka<<<dim3(g.nb, g.B * g.Hkv), kThreads, smem, st>>>(static_cast<const T*>(Ks), static_cast<const T*>(V), A, W,
                                                       M, U, Dj, g);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  phba_scan_kernel<T, D><<<dim3(ceil_div((int64_t)M * D, kThreads), g.B * g.Hkv), kThreads, 0, st>>>(
      U, Dj, M, static_cast<T*>(PK), static_cast<T*>(PV), g);
  return cudaGetLastError();
}

}  // namespace

size_t phba_workspace_bytes(const Geo& g, int M) { return phba_ws(g.B * g.Hkv, g.nb, M, g.d).total; }

cudaError_t launch_phba_states(const Geo& g, int M, const void* Ks, const void* V, const float* A, const float* W,
                               void* PK, void* PV, void* ws, int* status, cudaStream_t st) {
  if (g.dtype == PYR_BF16)
    return g.d == 128 ? launch_t<__nv_bfloat16, 128>(g, M, Ks, V, A, W, PK, PV, ws, status, st)
                      : launch_t<__nv_bfloat16, 64>(g, M, Ks, V, A, W, PK, PV, ws, status, st);
  return g.d == 128 ? launch_t<float, 128>(g, M, Ks, V, A, W, PK, PV, ws, status, st)
                    : launch_t<float, 64>(g, M, Ks, V, A, W, PK, PV, ws, status, st);
}

}  // namespace pyr
