// C ABI of libpyr: argument validation, geometry, dispatch to the kernels.
// Every entry point validates on the host, enqueues on the caller's stream
// and returns; nothing here allocates device memory or synchronises.
#include <cuda.h>
#include <stdint.h>

#include "pyr_common.cuh"
#include "select_opts.cuh"

namespace pyr {
size_t select_smem_bytes(const Geo& g);
}

using pyr::Geo;

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

constexpr int kPhbaMaxSlots = 256;  // prefix-state slots per state

// Shape checks shared by every entry point. Returns PYR_OK and fills g.
int make_geo(const pyr_shape* s, Geo* g) {
  if (!s) return PYR_EINVAL;
  if (s->B <= 0 || s->Hq <= 0 || s->Hkv <= 0 || s->Hq % s->Hkv || s->N <= 0 || s->Nq <= 0 || s->q_offset < 0 ||
      (int64_t)s->q_offset + s->Nq > s->N || s->b <= 0 || s->d <= 0 || s->topk < 1 || s->cap < 2 || s->cap % 2 ||
      s->topk > s->cap)
    return PYR_EINVAL;
  if (s->dtype != PYR_F32 && s->dtype != PYR_BF16) return PYR_EUNSUPPORTED;
  if (s->d != 64 && s->d != 128) return PYR_EUNSUPPORTED;
  if (s->b != 16 && s->b != 32 && s->b != 64 && s->b != 128) return PYR_EUNSUPPORTED;
  if (s->cap > 128) return PYR_EUNSUPPORTED;
  if (!(s->Nq == 1 || s->q_offset % s->b == 0)) return PYR_EUNSUPPORTED;
  if ((int64_t)s->B * s->Hkv > 65535) return PYR_EUNSUPPORTED;
  g->B = s->B;
  g->Hq = s->Hq;
  g->Hkv = s->Hkv;
  g->G = s->Hq / s->Hkv;
  g->N = s->N;
  g->Nq = s->Nq;
  g->q_offset = s->q_offset;
  g->d = s->d;
  g->b = s->b;
  g->topk = s->topk;
  g->cap = s->cap;
  g->dtype = s->dtype;
  g->nb = (int)(((int64_t)s->N + s->b - 1) / s->b);
  int L = 0;
  while (((int64_t)1 << L) < g->nb) L++;
  if (L >= 31) return PYR_EUNSUPPORTED;
  g->L = L;
  int64_t off = 0;
  for (int l = 0; l < 32; l++) {
    g->lvl_n[l] = l <= L ? (int)((g->nb + ((int64_t)1 << l) - 1) >> l) : 0;
    g->lvl_off[l] = (int)off;
    off += g->lvl_n[l];
  }
  g->P = off;
  g->i0 = s->q_offset / s->b;
  g->nqb = (s->q_offset + s->Nq - 1) / s->b - g->i0 + 1;
  int s0 = 0;
  while (g->lvl_n[s0] > s->cap) s0++;
  g->s0 = s0;
  if (s0 >= 24) return PYR_EUNSUPPORTED;  // the selection kernel keeps partial means for 24 levels
  if ((int64_t)g->G * (s->Nq < s->b ? s->Nq : s->b) > 1024) return PYR_EUNSUPPORTED;
  return PYR_OK;
}

int launch_status(cudaError_t e) { return e == cudaSuccess ? PYR_OK : PYR_ECUDA; }

}  // namespace

int pyr::validate_shape(const pyr_shape* s) {
  Geo g;
  return make_geo(s, &g);
}

namespace {

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

}  // namespace

bool pyr::current_context_id(unsigned long long* id) {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id || !id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) {
    // no context bound to this thread yet: bind the current device's primary context, as the
    // first runtime call on the thread would
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return false;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  }
  return get_id(ctx, id) == CUDA_SUCCESS;
}

extern "C" {

int pyr_num_levels(const pyr_shape* s) {
  Geo g;
  return make_geo(s, &g) == PYR_OK ? g.L + 1 : 0;
}

int64_t pyr_num_nodes(const pyr_shape* s) {
  Geo g;
  return make_geo(s, &g) == PYR_OK ? g.P : 0;
}

int64_t pyr_num_qblocks(const pyr_shape* s) {
  Geo g;
  return make_geo(s, &g) == PYR_OK ? g.nqb : 0;
}

size_t pyr_pyramid_elems(const pyr_shape* s) {
  Geo g;
  return make_geo(s, &g) == PYR_OK ? (size_t)s->B * s->Hkv * (size_t)g.P * 2 * s->d : 0;
}

int pyr_build(const pyr_shape* s, const void* K, void* pyr, int* dev_status, void* stream) {
  Geo g;
  int rc = make_geo(s, &g);
  if (rc) return rc;
  if (!K || !pyr || !aligned16(K) || !aligned16(pyr)) return PYR_EINVAL;
  return launch_status(pyr::launch_pyramid(g, K, static_cast<__nv_bfloat16*>(pyr), dev_status, (cudaStream_t)stream));
}

int pyr_means(const pyr_shape* s, const void* pyr, float* means, int* dev_status, void* stream) {
  Geo g;
  int rc = make_geo(s, &g);
  if (rc) return rc;
  if (!pyr || !means || !aligned16(pyr) || (reinterpret_cast<uintptr_t>(means) & 3)) return PYR_EINVAL;
  (void)dev_status;
  return launch_status(
      pyr::launch_pyramid_means(g, static_cast<const __nv_bfloat16*>(pyr), means, (cudaStream_t)stream));
}

int pyr_update(const pyr_shape* s, const void* K, void* pyr, int from_pos, int* dev_status, void* stream) {
  Geo g;
  int rc = make_geo(s, &g);
  if (rc) return rc;
  if (!K || !pyr || !aligned16(K) || !aligned16(pyr)) return PYR_EINVAL;
  if (from_pos < 0 || from_pos >= s->N) return PYR_EINVAL;
  return launch_status(
      pyr::launch_pyramid_update(g, K, static_cast<__nv_bfloat16*>(pyr), from_pos, dev_status, (cudaStream_t)stream));
}

int pyr_select_trace_levels(const pyr_shape* s) {
  Geo g;
  return make_geo(s, &g) == PYR_OK ? g.s0 + 1 : 0;
}

int pyr_select_trace_width(const pyr_shape* s) {
  Geo g;
  return make_geo(s, &g) == PYR_OK ? (s->cap / 2 > s->topk ? s->cap / 2 : s->topk) : 0;
}

int pyr_select_ex(const pyr_shape* s, const void* Q, const void* pyr_v, const pyr_select_opts* opts, int32_t* idx,
                  float* gap, int* dev_status, void* stream) {
  Geo g;
  int rc = make_geo(s, &g);
  if (rc) return rc;
  const __nv_bfloat16* pyr = static_cast<const __nv_bfloat16*>(pyr_v);
  if (!Q || !pyr || !idx || !aligned16(Q) || !aligned16(pyr) || !aligned16(idx)) return PYR_EINVAL;
  pyr::SelOpts o = {nullptr, 0.f, 0, 0.f, nullptr, 0};
  if (opts) {
    // NaN or infinite guidance weights and NaN thresholds have no meaning; tau may be +-inf
    if (opts->fcf_extra < 0 || opts->fcf_tau != opts->fcf_tau || !(fabsf(opts->rcg_lambda) < INFINITY))
      return PYR_EINVAL;
    if (((uintptr_t)opts->budget & 3u) || ((uintptr_t)opts->trace & 3u)) return PYR_EINVAL;
    o.budget = opts->budget;
    o.fcf_tau = opts->fcf_tau;
    o.fcf_extra = opts->fcf_extra;
    o.rcg_lambda = opts->rcg_lambda;
    o.trace = opts->trace;
    o.tw = s->cap / 2 > s->topk ? s->cap / 2 : s->topk;
  }
  const cudaStream_t st = (cudaStream_t)stream;
  if (pyr::select_tc_supported(g)) return launch_status(pyr::launch_select_tc(g, Q, pyr, idx, gap, dev_status, o, st));
  if (pyr::select_decode_supported(g)) return launch_status(pyr::launch_select_decode(g, Q, pyr, idx, gap, o, st));
  if (pyr::select_smem_bytes(g) > 227 * 1024) return PYR_EUNSUPPORTED;
  return launch_status(pyr::launch_select(g, Q, pyr, idx, gap, dev_status, o, st));
}

int pyr_select(const pyr_shape* s, const void* Q, const void* pyr, int32_t* idx, float* gap, int* dev_status,
               void* stream) {
  return pyr_select_ex(s, Q, pyr, nullptr, idx, gap, dev_status, stream);
}

int bsa_forward(const pyr_shape* s, const void* Q, const void* K, const void* V, const int32_t* idx, void* O,
                float* lse, int* dev_status, void* stream) {
  Geo g;
  int rc = make_geo(s, &g);
  if (rc) return rc;
  if (!Q || !K || !V || !idx || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return PYR_EINVAL;
  if (pyr::attn_tc_supported(g))
    return launch_status(pyr::launch_attn_tc(g, Q, K, V, idx, 0, O, lse, dev_status, (cudaStream_t)stream));
  if (pyr::attn_decode_warp_supported(g))
    return launch_status(pyr::launch_attn_decode_warp(g, Q, K, V, idx, 0, O, lse, dev_status, (cudaStream_t)stream));
  if (pyr::attn_decode_supported(g))
    return launch_status(pyr::launch_attn_decode(g, Q, K, V, idx, 0, O, lse, dev_status, (cudaStream_t)stream));
  return launch_status(pyr::launch_attn_simt(g, Q, K, V, idx, 0, O, lse, dev_status, (cudaStream_t)stream));
}

size_t phba_state_elems(const pyr_shape* s, int M) {
  Geo g;
  if (make_geo(s, &g) != PYR_OK || M < 1 || M > kPhbaMaxSlots) return 0;
  return (size_t)s->B * s->Hkv * g.nb * M * s->d;
}

size_t phba_state_workspace_bytes(const pyr_shape* s, int M) {
  Geo g;
  if (make_geo(s, &g) != PYR_OK || M < 1 || M > kPhbaMaxSlots) return 0;
  return pyr::phba_workspace_bytes(g, M);
}

int phba_state_build(const pyr_shape* s, int M, const void* Ks, const void* V, const float* A, const float* W,
                     void* PK, void* PV, void* workspace, size_t workspace_bytes, int* dev_status, void* stream) {
  Geo g;
  int rc = make_geo(s, &g);
  if (rc) return rc;
  if (M < 1 || M > kPhbaMaxSlots) return PYR_EUNSUPPORTED;
  if (!Ks || !V || !A || !W || !PK || !PV || !workspace || !aligned16(Ks) || !aligned16(V) || !aligned16(A) ||
      !aligned16(W) || !aligned16(PK) || !aligned16(PV) || !aligned16(workspace))
    return PYR_EINVAL;
  if (workspace_bytes < pyr::phba_workspace_bytes(g, M)) return PYR_EINVAL;
  return launch_status(
      pyr::launch_phba_states(g, M, Ks, V, A, W, PK, PV, workspace, dev_status, (cudaStream_t)stream));
}

int phba_forward(const pyr_shape* s, const void* Q, const void* K, const void* V, const int32_t* idx, const void* Qs,
                 int M, const void* PK, const void* PV, void* O, float* lse, int* dev_status, void* stream) {
  Geo g;
  int rc = make_geo(s, &g);
  if (rc) return rc;
  if (M < 0 || M > kPhbaMaxSlots) return PYR_EUNSUPPORTED;
  if (!Q || !K || !V || !idx || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) ||
      (Qs && !aligned16(Qs)))
    return PYR_EINVAL;
  if (M > 0 && (!PK || !PV || !aligned16(PK) || !aligned16(PV))) return PYR_EINVAL;
  const cudaStream_t st = (cudaStream_t)stream;
  // the tensor-core kernel scores the state slots with its Q tile: it takes the states when the
  // state branch's query is Q and the states come in whole 64-slot tiles
  if (pyr::attn_tc_supported(g) && (M == 0 || ((Qs == nullptr || Qs == Q) && M % 64 == 0)))
    return launch_status(pyr::launch_attn_tc(g, Q, K, V, idx, 0, O, lse, dev_status, st, PK, PV, M));
  if (M == 0 && pyr::attn_decode_warp_supported(g))
    return launch_status(pyr::launch_attn_decode_warp(g, Q, K, V, idx, 0, O, lse, dev_status, st));
  if (M == 0 && pyr::attn_decode_supported(g))
    return launch_status(pyr::launch_attn_decode(g, Q, K, V, idx, 0, O, lse, dev_status, st));
  return launch_status(pyr::launch_attn_simt(g, Q, K, V, idx, 0, O, lse, dev_status, st, Qs, PK, PV, M));
}

int dense_forward(const pyr_shape* s, const void* Q, const void* K, const void* V, void* O, float* lse,
                  int* dev_status, void* stream) {
  Geo g;
  int rc = make_geo(s, &g);
  if (rc) return rc;
  if (!Q || !K || !V || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return PYR_EINVAL;
  if (pyr::attn_tc_supported(g))
    return launch_status(pyr::launch_attn_tc(g, Q, K, V, nullptr, 1, O, lse, dev_status, (cudaStream_t)stream));
  if (pyr::attn_decode_warp_supported(g))
    return launch_status(pyr::launch_attn_decode_warp(g, Q, K, V, nullptr, 1, O, lse, dev_status, (cudaStream_t)stream));
  if (pyr::attn_decode_supported(g))
    return launch_status(pyr::launch_attn_decode(g, Q, K, V, nullptr, 1, O, lse, dev_status, (cudaStream_t)stream));
  return launch_status(pyr::launch_attn_simt(g, Q, K, V, nullptr, 1, O, lse, dev_status, (cudaStream_t)stream));
}

int bsa_route_invert(const pyr_shape* s, const int32_t* idx, int32_t* offset, int32_t* rho, int* dev_status,
                     void* stream) {
  Geo g;
  int rc = make_geo(s, &g);
  if (rc) return rc;
  if (!idx || !offset || !rho || !aligned16(idx) || ((uintptr_t)offset & 3u) || ((uintptr_t)rho & 3u))
    return PYR_EINVAL;
  return launch_status(pyr::launch_route_invert(g, idx, offset, rho, dev_status, (cudaStream_t)stream));
}

int bsa_backward(const pyr_shape* s, const void* Q, const void* K, const void* V, const void* O, const float* lse,
                 const void* dO, const int32_t* idx, const int32_t* offset, const int32_t* rho, float* delta,
                 void* dQ, void* dK, void* dV, int* dev_status, void* stream) {
  Geo g;
  int rc = make_geo(s, &g);
  if (rc) return rc;
  const void* need[] = {Q, K, V, O, lse, dO, idx, offset, rho, delta, dQ, dK, dV};
  for (const void* p : need)
    if (!p) return PYR_EINVAL;
  const void* vec[] = {Q, K, V, O, dO, dQ, dK, dV, idx};
  for (const void* p : vec)
    if (!aligned16(p)) return PYR_EINVAL;
  if (((uintptr_t)lse & 3u) || ((uintptr_t)delta & 3u) || ((uintptr_t)offset & 3u) || ((uintptr_t)rho & 3u))
    return PYR_EINVAL;
  if (s->q_offset != 0 || s->Nq != s->N) return PYR_EUNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  if (pyr::backward_tc_supported(g)) {
    cudaError_t e = pyr::launch_backward_simt(g, Q, K, V, O, lse, dO, idx, offset, rho, delta, dQ, dK, dV,
                                              pyr::kBwdDelta, st);
    // dK, dV first: until the dQ kernel writes it, dQ serves the dK/dV kernel as its work-list scratch
    if (e == cudaSuccess)
      e = pyr::launch_backward_dkdv_tc(g, Q, K, V, dO, lse, delta, offset, rho, dK, dV, dQ, dev_status, st);
    if (e == cudaSuccess) e = pyr::launch_backward_dq_tc(g, Q, K, V, dO, lse, delta, idx, dQ, dev_status, st);
    return launch_status(e);
  }
  return launch_status(pyr::launch_backward_simt(g, Q, K, V, O, lse, dO, idx, offset, rho, delta, dQ, dK, dV,
                                                 pyr::kBwdDelta | pyr::kBwdDq | pyr::kBwdDkdv, st));
}

const char* pyr_strerror(int code) {
  switch (code) {
    case PYR_OK: return "ok";
    case PYR_EINVAL: return "invalid argument (null or misaligned pointer, or inconsistent shape)";
    case PYR_EUNSUPPORTED: return "unsupported shape or dtype";
    case PYR_ECUDA: return "CUDA launch failed";
    case PYR_ETIMEOUT: return "a bounded device wait ran out";
    case PYR_EBADIDX: return "idx lists a block that is not strictly before its query block, or not ascending";
    default: return "unknown status";
  }
}

}  // extern "C"
