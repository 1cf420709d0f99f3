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
// With bf16 inputs, d = 128 and M = 128, pass A runs on the tcgen05 tensor
// cores: thread s builds slot s's coefficient row w_t[s] exp(R_t[s]) over the
// block's 64 tokens, split into bf16 hi + lo rows (the pair carries fp32 to
// about 2^-17), which form the K-major A operands [128 slots][64 tokens]; the
// block's state keys and values arrive by TMA as MN-major B operands [64 tokens]
// [128 d]; U_K and U_V accumulate in tensor memory (hi and lo MMAs into one
// fp32 result) and each thread writes its slot's rows out.
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

// Pass A on the tensor cores (bf16, d = 128, M = 128, b = 64: one 64-token box per block).
struct TcPlan {
  static constexpr int kXK = 0;               // [2 d-halves][64 tokens][128 B], 128-byte swizzle
  static constexpr int kXV = 16384;
  static constexpr int kChi = 32768;          // [128 slots][64 tokens] bf16, K-major, 128-byte swizzle
  static constexpr int kClo = 49152;
  static constexpr int kBar = 65536;          // x_full, mma_done
  static constexpr int kMisc = kBar + 16;     // tmem slot, abort flag
  static constexpr int kBytes = kMisc + 16 + 1024;  // + alignment slack
};

__global__ void __launch_bounds__(128) phba_chunk_tc_kernel(const __grid_constant__ CUtensorMap tmKs,
                                                            const __grid_constant__ CUtensorMap tmV,
                                                            const float* __restrict__ A, const float* __restrict__ W,
                                                            float* __restrict__ U, float* __restrict__ Dj,
                                                            int* status, Geo g) {
  using namespace tc;
  constexpr int M = 128, D = 128, BT = 64;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_align<1024>(smem_raw);
  uint64_t* bar_x = reinterpret_cast<uint64_t*>(smem + TcPlan::kBar);
  uint64_t* bar_mma = bar_x + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + TcPlan::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + TcPlan::kMisc + 4);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int j = blockIdx.x, unit = blockIdx.y;
  const int t0 = j * g.b, n = min(g.b, g.N - t0);

  if (tid == 0) {
    mbar_init(bar_x, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    *abort_flag = 0;
  }
  __syncthreads();
  if (tid == 0) {
    // the block's state keys and values; rows past N arrive as zeros
    mbar_expect_tx(bar_x, 32768);
    for (int h = 0; h < 2; h++) {
      tma_load_3d(smem + TcPlan::kXK + h * 8192, &tmKs, h * 64, t0, unit, bar_x);
      tma_load_3d(smem + TcPlan::kXV + h * 8192, &tmV, h * 64, t0, unit, bar_x);
    }
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  // slot tid's coefficients over the block's tokens, from the log-A suffix sums (tokens past the
  // block's end get 0), as bf16 hi + lo rows. Every gate is loaded first, so that all the loads are
  // in flight together; the scan then runs on registers (c takes the write gates' place)
  {
    const int s = tid;
    const float* As = A + ((size_t)unit * g.N + t0) * M + s;
    const float* Ws = W + ((size_t)unit * g.N + t0) * M + s;
    float a[BT], c[BT];
#pragma unroll
    for (int t = 0; t < BT; t++) {
      a[t] = t < n ? __ldg(As + (size_t)t * M) : 1.f;
      c[t] = t < n ? __ldg(Ws + (size_t)t * M) : 0.f;
    }
    float r = 0.f;
#pragma unroll
    for (int t = BT - 1; t >= 0; t--) {
      c[t] *= __expf(r);
      r += __logf(a[t]);
    }
    Dj[((size_t)unit * g.nb + j) * M + s] = __expf(r);
#pragma unroll
    for (int ch = 0; ch < 8; ch++) {  // 16-byte chunk ch holds tokens 8 ch .. 8 ch + 7
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int q = 0; q < 4; q++) {
        const float a = c[8 * ch + 2 * q], b = c[8 * ch + 2 * q + 1];
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(a, b);
        const __nv_bfloat162 l2 =
            __floats2bfloat162_rn(a - __bfloat162float(h2.x), b - __bfloat162float(h2.y));
        hi[q] = *reinterpret_cast<const uint32_t*>(&h2);
        lo[q] = *reinterpret_cast<const uint32_t*>(&l2);
      }
      const int off = s * 128 + ((ch ^ (s & 7)) << 4);
      *reinterpret_cast<uint4*>(smem + TcPlan::kChi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(smem + TcPlan::kClo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  }
  fence_proxy_async_smem();  // the coefficient rows are read by the tensor cores
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tD = *tmem_slot;
  bool issued = false;
  if (tid == 0) {
    bool ok = mbar_wait(bar_x, 0, abort_flag);
    if (ok) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 1);  // A K-major, B MN-major
      const uint32_t aH = smem_u32(smem + TcPlan::kChi), aL = smem_u32(smem + TcPlan::kClo);
      const uint32_t bK = smem_u32(smem + TcPlan::kXK), bV = smem_u32(smem + TcPlan::kXV);
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; kk++) {  // 16 tokens per step
        const uint64_t dh = sdesc_sw128(aH + kk * 32, 16, 1024), dl = sdesc_sw128(aL + kk * 32, 16, 1024);
        const uint64_t dk = sdesc_sw128(bK + kk * 2048, 8192, 1024), dv = sdesc_sw128(bV + kk * 2048, 8192, 1024);
        umma_bf16(tD, dh, dk, idesc, kk > 0);
        umma_bf16(tD, dl, dk, idesc, 1);
        umma_bf16(tD + 128, dh, dv, idesc, kk > 0);
        umma_bf16(tD + 128, dl, dv, idesc, 1);
      }
      umma_commit(bar_mma);
      issued = true;
    } else {
      volatile int no_abort = 0;
      mbar_wait(bar_x, 0, &no_abort);  // the copies still land in this CTA's shared memory
    }
  }
  issued = __syncthreads_or(issued);
  bool ok = issued && mbar_wait(bar_mma, 0, abort_flag);
  ok = __syncthreads_and(ok);
  if (ok) {
    tc_fence_after();
    // thread s holds TMEM lane s: its slot's rows of U_K (columns 0..127) and U_V (128..255)
    const uint32_t lane_addr = tD + ((uint32_t)(warp * 32) << 16);
    float* Us = U + ((size_t)unit * g.nb + j) * 2 * M * D;
    float v[32];
    for (int which = 0; which < 2; which++) {
      float* row = Us + ((size_t)which * M + tid) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        tmem_ld32(lane_addr + which * 128 + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 8; q++)
          *reinterpret_cast<float4*>(row + c0 + 4 * q) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      }
    }
  } else if (tid == 0 && issued) {
    // the MMAs may still be in flight after an abort: let them finish before freeing tensor memory
    umma_commit(bar_mma);
    volatile int no_abort = 0;
    mbar_wait(bar_mma, 0, &no_abort);
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && tid == 0) report(status, PYR_ETIMEOUT);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tD, 256);
  }
}

template <typename T, int D>
cudaError_t launch_t(const Geo& g, int M, const void* Ks, const void* V, const float* A, const float* W, void* PK,
                     void* PV, void* ws, int* status, cudaStream_t st) {
  const PhbaWs L = phba_ws(g.B * g.Hkv, g.nb, M, D);
  float* U = static_cast<float*>(ws);
  float* Dj = reinterpret_cast<float*>(static_cast<char*>(ws) + L.u_bytes);
  cudaError_t e;
  if (sizeof(T) == 2 && D == 128 && M == 128 && g.b == 64) {
    CUtensorMap mk, mv;
    if (!tc::make_tmap_bf16_3d(&mk, Ks, D, g.N, g.B * g.Hkv) || !tc::make_tmap_bf16_3d(&mv, V, D, g.N, g.B * g.Hkv))
      return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(phba_chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TcPlan::kBytes);
    if (e != cudaSuccess) return e;
    phba_chunk_tc_kernel<<<dim3(g.nb, g.B * g.Hkv), 128, TcPlan::kBytes, st>>>(mk, mv, A, W, U, Dj, status, g);
  } else {
    const size_t smem = sizeof(float) * ((size_t)g.b * kSlotGroup + (size_t)g.b * D);
    auto ka = phba_chunk_kernel<T, D>;
    e = cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    ka<<<dim3(g.nb, g.B * g.Hkv), kThreads, smem, st>>>(static_cast<const T*>(Ks), static_cast<const T*>(V), A, W,
                                                         M, U, Dj, g);
  }
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
