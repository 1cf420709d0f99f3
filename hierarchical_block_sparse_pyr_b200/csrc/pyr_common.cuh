// Shared device helpers and the internal launch interface of libpyr.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pyr.h"

namespace pyr {

// Geometry derived from a validated pyr_shape.
struct Geo {
  int B, Hq, Hkv, G, N, Nq, q_offset, d, b, topk, cap, dtype;
  int nb;       // key blocks
  int L;        // top level (levels 0..L)
  int nqb;      // query blocks per (batch, kv head)
  int i0;       // first query block
  int s0;       // first scored level: the finest with <= cap nodes
  int64_t P;    // pyramid nodes per (batch, kv head)
  int lvl_off[32];  // node offset of each level
  int lvl_n[32];    // nodes of each level
};

inline int ceil_div(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

// Dynamic shared memory rounded up to an A-byte boundary of the shared address
// (A a power of two). The offset is added to the __shared__ array itself, so
// the compiler still knows the result points to shared memory and accesses it
// with shared-memory instructions; a round trip through an integer would turn
// every access through it into a generic one.
template <int A>
__device__ __forceinline__ unsigned char* smem_align(unsigned char* raw) {
  const uint32_t s = (uint32_t)__cvta_generic_to_shared(raw);
  return raw + ((A - (s & (A - 1))) & (A - 1));
}

// Device status word: the first error wins.
__device__ __forceinline__ void report(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Pyramid node storage: a node mean x is kept as the unevaluated bf16 pair
// hi = RN(x), lo = RN(x - hi) (|x - hi - lo| <= 2^-17 |x|), in a row of 2d
// bf16: [hi_0 .. hi_{d-1} | lo_0 .. lo_{d-1}]. This is exactly the operand
// format the tensor-core scoring consumes, so selection copies node rows
// straight into its MMA operands.
__device__ __forceinline__ void split_store(__nv_bfloat16* row, int d, int e, float x) {
  const __nv_bfloat16 hi = __float2bfloat16_rn(x);
  row[e] = hi;
  row[d + e] = __float2bfloat16_rn(x - __bfloat162float(hi));
}
__device__ __forceinline__ float split_load(const __nv_bfloat16* row, int d, int e) {
  return __bfloat162float(row[e]) + __bfloat162float(row[d + e]);
}

// Order-preserving map of a float to uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_order_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Host-side shape check of every entry point: PYR_OK or the error code the
// entry points return for this shape.
int validate_shape(const pyr_shape* s);

// Unique id (for the life of the process) of the CUDA context current on the
// calling thread; when no context is current, the current device's primary
// context is made current first, as any runtime call would. Device addresses of
// __device__ variables, streams and events belong to one context, so caches of
// them are keyed by this id rather than by device ordinal. False on failure.
bool current_context_id(unsigned long long* id);

// Launchers (one per kernel family). Each returns cudaSuccess or the launch error.
cudaError_t launch_pyramid(const Geo& g, const void* K, __nv_bfloat16* pyr, int* status, cudaStream_t st);
cudaError_t launch_pyramid_update(const Geo& g, const void* K, __nv_bfloat16* pyr, int from_pos, int* status,
                                  cudaStream_t st);
// fp32 node means (hi + lo) of a pyramid, [B * Hkv][P][d]
cudaError_t launch_pyramid_means(const Geo& g, const __nv_bfloat16* pyr, float* means, cudaStream_t st);
bool attn_decode_supported(const Geo& g);
bool attn_decode_warp_supported(const Geo& g);  // one warp per 64-key tile, G <= 8
cudaError_t launch_attn_decode_warp(const Geo& g, const void* Q, const void* K, const void* V, const int32_t* idx,
                                    int dense, void* O, float* lse, int* status, cudaStream_t st);
cudaError_t launch_attn_decode(const Geo& g, const void* Q, const void* K, const void* V, const int32_t* idx,
                               int dense, void* O, float* lse, int* status, cudaStream_t st);
struct SelOpts;  // selection variants and trace (select_opts.cuh)
cudaError_t launch_select(const Geo& g, const void* Q, const __nv_bfloat16* pyr, int32_t* idx, float* gap, int* status,
                          const SelOpts& o, cudaStream_t st);
bool select_tc_supported(const Geo& g);
bool select_decode_supported(const Geo& g);
cudaError_t launch_select_decode(const Geo& g, const void* Q, const __nv_bfloat16* pyr, int32_t* idx, float* gap,
                                 const SelOpts& o, cudaStream_t st);
cudaError_t launch_select_tc(const Geo& g, const void* Q, const __nv_bfloat16* pyr, int32_t* idx, float* gap, int* status,
                             const SelOpts& o, cudaStream_t st);
bool attn_tc_supported(const Geo& g);
// PK, PV: PHBA prefix states [B * Hkv][nb][M][d] (M = 0: none; M % 64 == 0 here)
cudaError_t launch_attn_tc(const Geo& g, const void* Q, const void* K, const void* V, const int32_t* idx, int dense,
                           void* O, float* lse, int* status, cudaStream_t st, const void* PK = nullptr,
                           const void* PV = nullptr, int M = 0);
cudaError_t launch_route_invert(const Geo& g, const int32_t* idx, int32_t* offset, int32_t* rho, int* status,
                                cudaStream_t st);
// parts of the SIMT backward to launch (bit mask)
constexpr int kBwdDelta = 1, kBwdDq = 2, kBwdDkdv = 4;
cudaError_t launch_backward_simt(const Geo& g, const void* Q, const void* K, const void* V, const void* O,
                                 const float* lse, const void* dO, const int32_t* idx, const int32_t* offset,
                                 const int32_t* rho, float* delta, void* dQ, void* dK, void* dV, int parts,
                                 cudaStream_t st);
bool backward_tc_supported(const Geo& g);
// scratch: device memory of at least 8 + 4 * B * Hkv * nb bytes that no other operand uses and that
// nothing reads until this launch ends (bsa_backward passes dQ, written afterwards)
cudaError_t launch_backward_dkdv_tc(const Geo& g, const void* Q, const void* K, const void* V, const void* dO,
                                    const float* lse, const float* delta, const int32_t* offset, const int32_t* rho,
                                    void* dK, void* dV, void* scratch, int* status, cudaStream_t st);
cudaError_t launch_backward_dq_tc(const Geo& g, const void* Q, const void* K, const void* V, const void* dO,
                                  const float* lse, const float* delta, const int32_t* idx, void* dQ, int* status,
                                  cudaStream_t st);
// Qst: the state branch's query (null: Q); PK, PV, M as for launch_attn_tc (any M)
cudaError_t launch_attn_simt(const Geo& g, const void* Q, const void* K, const void* V, const int32_t* idx,
                             int dense, void* O, float* lse, int* status, cudaStream_t st, const void* Qst = nullptr,
                             const void* PK = nullptr, const void* PV = nullptr, int M = 0);
// PHBA prefix states: pass A (chunk-local products) and pass B (carry across blocks)
size_t phba_workspace_bytes(const Geo& g, int M);
cudaError_t launch_phba_states(const Geo& g, int M, const void* Ks, const void* V, const float* A, const float* W,
                               void* PK, void* PV, void* ws, int* status, cudaStream_t st);

}  // namespace pyr
