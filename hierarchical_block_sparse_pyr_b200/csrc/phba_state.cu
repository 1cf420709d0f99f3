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
#include "pyr_common.cuh"

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

template <typename T, int D>
cudaError_t launch_t(const Geo& g, int M, const void* Ks, const void* V, const float* A, const float* W, void* PK,
                     void* PV, void* ws, cudaStream_t st) {
  const PhbaWs L = phba_ws(g.B * g.Hkv, g.nb, M, D);
  float* U = static_cast<float*>(ws);
  float* Dj = reinterpret_cast<float*>(static_cast<char*>(ws) + L.u_bytes);
  const size_t smem = sizeof(float) * ((size_t)g.b * kSlotGroup + (size_t)g.b * D);
  auto ka = phba_chunk_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ka<<<dim3(g.nb, g.B * g.Hkv), kThreads, smem, st>>>(static_cast<const T*>(Ks), static_cast<const T*>(V), A, W, M,
                                                       U, Dj, g);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  phba_scan_kernel<T, D><<<dim3(ceil_div((int64_t)M * D, kThreads), g.B * g.Hkv), kThreads, 0, st>>>(
      U, Dj, M, static_cast<T*>(PK), static_cast<T*>(PV), g);
  return cudaGetLastError();
}

}  // namespace

size_t phba_workspace_bytes(const Geo& g, int M) { return phba_ws(g.B * g.Hkv, g.nb, M, g.d).total; }

cudaError_t launch_phba_states(const Geo& g, int M, const void* Ks, const void* V, const float* A, const float* W,
                               void* PK, void* PV, void* ws, cudaStream_t st) {
  if (g.dtype == PYR_BF16)
    return g.d == 128 ? launch_t<__nv_bfloat16, 128>(g, M, Ks, V, A, W, PK, PV, ws, st)
                      : launch_t<__nv_bfloat16, 64>(g, M, Ks, V, A, W, PK, PV, ws, st);
  return g.d == 128 ? launch_t<float, 128>(g, M, Ks, V, A, W, PK, PV, ws, st)
                    : launch_t<float, 64>(g, M, Ks, V, A, W, PK, PV, ws, st);
}

}  // namespace pyr
