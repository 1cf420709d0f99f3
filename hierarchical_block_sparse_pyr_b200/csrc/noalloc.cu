// bsa_backward_noalloc: the backward pass for callers that cannot allocate
// device memory.
//
// bsa_backward needs a workspace of one fp32 per query row (D_t = dO_t . O_t),
// which its caller allocates. Some callers cannot: plugins whose host framework
// owns every byte of device memory and hands out only the tensors it knows
// about, and serving or real-time loops that must never call cudaMalloc (it can
// synchronise the device and block on the allocator). This entry point
// keeps that workspace in a fixed array in the library's own device memory
// instead, so the caller passes only inputs and outputs.
//
// The array is a file-scope __device__ variable of kMaxRows floats (16 MiB):
// every GPU that loads the library holds it until the process exits. Host
// code must not pass the array's name to a kernel (on the host that name is a
// stand-in, not a device address). Its device address belongs to the CUDA
// context the library's module is loaded in, so it is looked up with
// cudaGetSymbolAddress on the first call made in each context (the primary
// context of a device, or a context the caller made current with the driver
// API), with that context current, and cached under the context's unique id;
// a context made after a cudaDeviceReset gets a lookup of its own.
#include <map>
#include <mutex>

#include "pyr_common.cuh"

namespace pyr {
namespace {

constexpr int64_t kMaxRows = 4 * 1024 * 1024;  // B * Hq * Nq query rows

static __device__ __align__(256) float g_delta_scratch[kMaxRows];

std::mutex g_scratch_mu;
std::map<unsigned long long, float*> g_scratch_ptr;  // context id -> address of g_delta_scratch

// The device address of g_delta_scratch in the current context, or nullptr.
float* scratch_for_current_context() {
  unsigned long long ctx = 0;
  if (!current_context_id(&ctx)) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const auto it = g_scratch_ptr.find(ctx);
  if (it != g_scratch_ptr.end()) return it->second;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_delta_scratch) != cudaSuccess || p == nullptr) return nullptr;
  g_scratch_ptr[ctx] = static_cast<float*>(p);
  return static_cast<float*>(p);
}

}  // namespace
}  // namespace pyr

extern "C" int bsa_backward_noalloc(const pyr_shape* s, const void* Q, const void* K, const void* V, const void* O,
                                    const float* lse, const void* dO, const int32_t* idx, const int32_t* offset,
                                    const int32_t* rho, void* dQ, void* dK, void* dV, int* dev_status,
                                    void* stream) {
  // a malformed shape is reported as such before the limit check and before any CUDA call
  const int rc = pyr::validate_shape(s);
  if (rc != PYR_OK) return rc;
  const int64_t rows = (int64_t)s->B * s->Hq * s->Nq;
  if (rows > pyr::kMaxRows) return PYR_EUNSUPPORTED;  // beyond the fixed workspace
  float* delta = pyr::scratch_for_current_context();
  if (!delta) return PYR_ECUDA;
  // the workspace is written in full (one value per query row) before it is read, so it needs no
  // clearing between calls
  return bsa_backward(s, Q, K, V, O, lse, dO, idx, offset, rho, delta, dQ, dK, dV, dev_status, stream);
}
