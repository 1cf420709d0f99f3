// bsa_forward_host: the forward path for inputs and outputs in host memory.
//
// The (batch, kv head) units are independent through all three steps (pyramid,
// selection, attention), so they stream through the device in chunks of
// consecutive units: while chunk c is computed on the caller's stream, chunk
// c + 1 is copied in on one copy stream and chunk c - 1's output is copied out
// on another. PCIe moves data in both directions at once, so a step costs
// about the host-to-device copy of Q, K and V plus the compute and copy-out
// of the last chunk, instead of the sum of all three.
//
// A chunk of n consecutive units is itself a valid shape: B = n, Hq = G,
// Hkv = 1. Unit u = bi * Hkv + hk owns query heads hk G .. hk G + G - 1 of
// batch bi, which lie next to each other in [B][Hq][Nq][d], so unit u's query
// rows start at u G Nq d and its keys at u N d. Every kernel computes a unit
// the same way whatever the other units of its launch are, so the result is
// bit-identical to pyr_build + pyr_select + bsa_forward over the whole batch.
//
// Device workspace (caller-owned): two slots of {Q, K, V, O, lse} for one
// chunk each, and one pyramid and one idx array for a chunk (the compute
// stream is in order, so those are reused chunk after chunk). Each part
// starts on a 256-byte boundary relative to the workspace base.
#include <map>
#include <memory>
#include <mutex>
#include <vector>

#include "pyr_common.cuh"

namespace {

constexpr int kSlots = 2;
constexpr size_t kAlign = 256;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct ChunkLayout {
  size_t q, kv, o, lse, pyr, idx;  // bytes of each part for one chunk, rounded up
  size_t slot;                     // q + 2 kv + o + lse
  size_t total;                    // kSlots * slot + pyr + idx
};

ChunkLayout layout_for(const pyr_shape* s, int64_t P, int64_t nqb, int upc, bool with_lse) {
  const size_t elt = s->dtype == PYR_F32 ? 4 : 2;
  const size_t G = (size_t)(s->Hq / s->Hkv);
  ChunkLayout c;
  c.q = round_up((size_t)upc * G * s->Nq * s->d * elt);
  c.kv = round_up((size_t)upc * s->N * s->d * elt);
  c.o = c.q;
  c.lse = with_lse ? round_up((size_t)upc * G * s->Nq * sizeof(float)) : 0;
  c.pyr = round_up((size_t)upc * P * 2 * s->d * 2);
  c.idx = round_up((size_t)upc * nqb * s->topk * sizeof(int32_t));
  c.slot = c.q + 2 * c.kv + c.o + c.lse;
  c.total = kSlots * c.slot + c.pyr + c.idx;
  return c;
}

// Chunk sizes when the caller passes 0. Every chunk costs a fixed overhead (its
// copies and launches), and the last chunk's compute and copy-out are not
// hidden, so the chunks shrink towards the end: chunks of `cap` units first,
// then cap/2, ..., 2, 1, 1 (measured at 32K, 16 one-unit chunks take 8.7 ms
// per step and 8 two-unit chunks 8.4 ms, against 7.6 ms for the copies alone).
// cap: a quarter of the units, and at most 96 MiB of inputs per chunk.
int auto_cap(const pyr_shape* s) {
  const int U = s->B * s->Hkv;
  const size_t elt = s->dtype == PYR_F32 ? 4 : 2;
  const size_t in_unit = (size_t)(s->Hq / s->Hkv) * s->Nq * s->d * elt + 2 * (size_t)s->N * s->d * elt;
  const size_t by_bytes = (96u << 20) / (in_unit ? in_unit : 1);
  size_t cap = (size_t)(U / 4);
  if (cap > by_bytes) cap = by_bytes;
  return cap < 1 ? 1 : (int)cap;
}

// The chunk sizes of a call (in order), summing to U: uniform chunks of upc
// units (the last one possibly smaller), or with upc == 0 the shrinking
// schedule above. Returns the largest chunk, which sizes the device slots.
int chunk_schedule(const pyr_shape* s, int upc, std::vector<int>* sizes) {
  const int U = s->B * s->Hkv;
  sizes->clear();
  if (upc > 0) {
    if (upc > U) upc = U;
    for (int u0 = 0; u0 < U; u0 += upc) sizes->push_back(U - u0 < upc ? U - u0 : upc);
    return upc;
  }
  const int cap = auto_cap(s);
  std::vector<int> tail = {1, 1};  // the end of the call, last chunk last
  int sum = 2;
  for (int n = 2; n < cap && sum + n <= U; n *= 2) {
    tail.insert(tail.begin(), n);
    sum += n;
  }
  if (sum > U) {  // too few units for the tail: one unit per chunk
    sizes->assign(U, 1);
    return 1;
  }
  const int rest = U - sum;
  if (rest % cap) sizes->push_back(rest % cap);
  for (int k = 0; k < rest / cap; k++) sizes->push_back(cap);
  sizes->insert(sizes->end(), tail.begin(), tail.end());
  int mx = 1;
  for (int n : *sizes) mx = n > mx ? n : mx;
  return mx;
}

// Two copy streams and the events that order the slots, made once per CUDA
// context (streams and events belong to the context they were made in, so the
// primary context of a device, a context the caller made current with the
// driver API and a context made after a cudaDeviceReset each get their own)
// and kept until the process exits. The mutex serialises the enqueueing of
// calls in one context, so that an event is re-recorded only after every wait
// on its previous record has been enqueued.
struct DeviceStreams {
  std::mutex mu;
  bool ready = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t entry, in_done[kSlots], compute_done[kSlots], out_done[kSlots], h2d_exit, d2h_exit;
};

std::mutex g_dev_mu;
std::map<unsigned long long, std::unique_ptr<DeviceStreams>> g_dev;  // context id -> its streams

DeviceStreams* streams_for_current_context() {
  unsigned long long ctx = 0;
  if (!pyr::current_context_id(&ctx)) return nullptr;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  std::unique_ptr<DeviceStreams>& ds = g_dev[ctx];
  if (!ds) ds.reset(new DeviceStreams);
  return ds.get();
}

cudaError_t init_streams(DeviceStreams& ds) {
  if (ds.ready) return cudaSuccess;
  cudaError_t e = cudaStreamCreateWithFlags(&ds.h2d, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&ds.d2h, cudaStreamNonBlocking);
  cudaEvent_t* evs[] = {&ds.entry, &ds.h2d_exit, &ds.d2h_exit};
  for (cudaEvent_t* ev : evs)
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  for (int k = 0; k < kSlots && e == cudaSuccess; k++) {
    e = cudaEventCreateWithFlags(&ds.in_done[k], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ds.compute_done[k], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ds.out_done[k], cudaEventDisableTiming);
  }
  // on failure the streams and events made so far are kept and the next call
  // makes the rest again; a failure here means the device is unusable anyway
  if (e == cudaSuccess) ds.ready = true;
  return e;
}

int status_of(cudaError_t e) { return e == cudaSuccess ? PYR_OK : PYR_ECUDA; }

}  // namespace

extern "C" size_t pyr_host_workspace_bytes(const pyr_shape* s, int units_per_chunk, int with_lse) {
  if (units_per_chunk < 0 || pyr::validate_shape(s) != PYR_OK) return 0;
  const int64_t P = pyr_num_nodes(s), nqb = pyr_num_qblocks(s);
  std::vector<int> sizes;
  const int upc = chunk_schedule(s, units_per_chunk, &sizes);
  return layout_for(s, P, nqb, upc, with_lse != 0).total;
}

extern "C" int bsa_forward_host(const pyr_shape* s, const void* Q, const void* K, const void* V, void* O, float* lse,
                                int units_per_chunk, void* workspace, size_t workspace_bytes, int* dev_status,
                                void* stream) {
  const int rc0 = pyr::validate_shape(s);
  if (rc0 != PYR_OK) return rc0;
  const int64_t P = pyr_num_nodes(s), nqb = pyr_num_qblocks(s);
  if (!Q || !K || !V || !O || !workspace || ((uintptr_t)workspace & 15u) || units_per_chunk < 0) return PYR_EINVAL;
  std::vector<int> sizes;
  const int upc = chunk_schedule(s, units_per_chunk, &sizes);
  const ChunkLayout c = layout_for(s, P, nqb, upc, lse != nullptr);
  if (workspace_bytes < c.total) return PYR_EINVAL;

  DeviceStreams* dsp = streams_for_current_context();
  if (!dsp) return PYR_ECUDA;
  DeviceStreams& ds = *dsp;
  std::lock_guard<std::mutex> lock(ds.mu);
  if (init_streams(ds) != cudaSuccess) return PYR_ECUDA;

  const cudaStream_t st = (cudaStream_t)stream;
  const size_t elt = s->dtype == PYR_F32 ? 4 : 2;
  const int G = s->Hq / s->Hkv;
  const size_t q_unit = (size_t)G * s->Nq * s->d * elt, kv_unit = (size_t)s->N * s->d * elt;
  const size_t lse_unit = (size_t)G * s->Nq * sizeof(float);
  char* base = static_cast<char*>(workspace);
  char* pyr = base + kSlots * c.slot;
  int32_t* idx = reinterpret_cast<int32_t*>(pyr + c.pyr);

  // nothing on the copy streams may start before the caller's earlier work on
  // its stream (which may still be using the workspace)
  cudaError_t e = cudaEventRecord(ds.entry, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(ds.h2d, ds.entry, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(ds.d2h, ds.entry, 0);
  int rc = status_of(e);

  const int nchunks = (int)sizes.size();
  for (int ch = 0, u0 = 0; ch < nchunks && rc == PYR_OK; u0 += sizes[ch], ch++) {
    const int n = sizes[ch];
    const int k = ch % kSlots;
    char* slot = base + k * c.slot;
    char *dq = slot, *dk = slot + c.q, *dv = dk + c.kv, *dout = dv + c.kv;
    float* dlse = lse ? reinterpret_cast<float*>(dout + c.o) : nullptr;
    pyr_shape cs = *s;
    cs.B = n;
    cs.Hq = G;
    cs.Hkv = 1;

    // in: the slot's inputs are free once the chunk that used it two chunks ago has been computed
    if (ch >= kSlots) e = cudaStreamWaitEvent(ds.h2d, ds.compute_done[k], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(dq, static_cast<const char*>(Q) + u0 * q_unit, n * q_unit, cudaMemcpyHostToDevice, ds.h2d);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(dk, static_cast<const char*>(K) + u0 * kv_unit, n * kv_unit, cudaMemcpyHostToDevice,
                          ds.h2d);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(dv, static_cast<const char*>(V) + u0 * kv_unit, n * kv_unit, cudaMemcpyHostToDevice,
                          ds.h2d);
    if (e == cudaSuccess) e = cudaEventRecord(ds.in_done[k], ds.h2d);
    // compute: after the inputs arrived and the slot's previous output left
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ds.in_done[k], 0);
    if (e == cudaSuccess && ch >= kSlots) e = cudaStreamWaitEvent(st, ds.out_done[k], 0);
    rc = status_of(e);
    if (rc == PYR_OK) rc = pyr_build(&cs, dk, pyr, dev_status, st);
    if (rc == PYR_OK) rc = pyr_select(&cs, dq, pyr, idx, nullptr, dev_status, st);
    if (rc == PYR_OK) rc = bsa_forward(&cs, dq, dk, dv, idx, dout, dlse, dev_status, st);
    if (rc != PYR_OK) break;
    e = cudaEventRecord(ds.compute_done[k], st);
    // out
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ds.d2h, ds.compute_done[k], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(static_cast<char*>(O) + u0 * q_unit, dout, n * q_unit, cudaMemcpyDeviceToHost, ds.d2h);
    if (e == cudaSuccess && lse)
      e = cudaMemcpyAsync(lse + (size_t)u0 * (lse_unit / sizeof(float)), dlse, n * lse_unit, cudaMemcpyDeviceToHost,
                          ds.d2h);
    if (e == cudaSuccess) e = cudaEventRecord(ds.out_done[k], ds.d2h);
    rc = status_of(e);
  }

  // the caller's stream ends after everything enqueued above, on error too:
  // its later work may free or reuse the workspace and the host buffers
  cudaError_t e2 = cudaEventRecord(ds.h2d_exit, ds.h2d);
  if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(st, ds.h2d_exit, 0);
  if (e2 == cudaSuccess) e2 = cudaEventRecord(ds.d2h_exit, ds.d2h);
  if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(st, ds.d2h_exit, 0);
  if (rc == PYR_OK) rc = status_of(e2);
  return rc;
}
