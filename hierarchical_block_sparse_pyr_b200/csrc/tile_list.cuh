// The key-block list of a query tile: the ascending union of the key blocks
// that QB (1 or 2) consecutive query blocks attend (PHBA summary, A.1.3: one
// loaded block serves every row of the tile that routes to it). Query block
// i attends its routed blocks (its idx row) and its own block. Entries are
// (block << 4) | modes, 2 bits per query block q at bit 2q: 1 routed (every
// key), 2 own block (keys up to the row's position), 0 not attended.
//
// A route of row i is used only if it is >= 0, < i and greater than every
// earlier in-range route of the row (the rule every kernel of the library
// applies); other non-negative entries are skipped and reported as
// PYR_EBADIDX. Built by the whole CTA in parallel: one warp per query block
// compacts its row (a prefix-max scan reproduces the sequential rule), then
// every element finds its place in the union by binary search, duplicates
// (blocks routed by both query blocks) folded into one entry.
#pragma once

#include "pyr_common.cuh"

namespace pyr {

constexpr int kTileListPitch = 132;  // >= topk + 1 for topk <= 128, multiple of 4
// shared-memory ints build_tile_list needs as scratch: two lists, the duplicate
// flags and their prefix counts, two counts
constexpr int kTileListScratch = 4 * kTileListPitch + 4;

__device__ __forceinline__ int lower_bound_smem(const int* a, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < v) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// Warp-level compaction of one idx row (query block iq, in slot order, by the
// rule above) into L: the accepted routes, ascending, then iq itself. Lane l
// reads slot 32 c + l as get(c) (topk <= 128: at most 4 chunks). Returns the
// length on every lane; L is complete (and visible to the warp) on return.
template <typename Get>
__device__ inline int compact_route_row_with(Get get, int topk, int iq, int* L, int* status) {
  const int lane = threadIdx.x & 31;
  int base = 0, pmax = -1;
#pragma unroll
  for (int c = 0; c < 4; c++) {
    const int k0 = 32 * c;
    if (k0 >= topk) break;
    const int j = k0 + lane < topk ? get(c) : -1;
    const bool in_range = j >= 0 && j < iq;
    int incl = in_range ? j : -1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl = max(incl, y);
    }
    int before = __shfl_up_sync(0xffffffffu, incl, 1);
    before = max(lane == 0 ? -1 : before, pmax);
    const bool acc = in_range && j > before;
    if (j >= 0 && !acc) report(status, PYR_EBADIDX);
    const unsigned m = __ballot_sync(0xffffffffu, acc);
    if (acc) L[base + __popc(m & ((1u << lane) - 1u))] = j;
    base += __popc(m);
    pmax = max(pmax, __shfl_sync(0xffffffffu, incl, 31));
  }
  if (lane == 0) L[base] = iq;
  __syncwarp();
  return base + 1;
}

// The same, reading the row from global memory.
__device__ inline int compact_route_row(const int32_t* __restrict__ row, int topk, int iq, int* L, int* status) {
  const int lane = threadIdx.x & 31;
  return compact_route_row_with([&](int c) { return row[32 * c + lane]; }, topk, iq, L, status);
}

// Compaction of the routes of nq (1..2) consecutive query blocks, one warp per
// block: list q (at scratch + q * kTileListPitch) holds row q's accepted routes,
// ascending, then the block's own index; its length is at
// scratch[4 * kTileListPitch + q]. Call from every thread of the CTA (it ends
// with a block-wide barrier).
__device__ inline void compact_routes(const int32_t* __restrict__ rows, int topk, int i_first, int nq, int* scratch,
                                      int* status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp < nq) {
    const int n = compact_route_row(rows + (size_t)warp * topk, topk, i_first + warp,
                                    scratch + warp * kTileListPitch, status);
    if (lane == 0) scratch[4 * kTileListPitch + warp] = n;
  }
  __syncthreads();
}

// Call from every thread of the CTA (it contains block-wide barriers).
// rows: the QB idx rows in global memory (row q = query block i_first + q);
// nq: query blocks present (1..QB). Returns the number of entries in tiles.
template <int QB>
__device__ int build_tile_list(const int32_t* __restrict__ rows, int topk, int i_first, int nq, int* scratch,
                               int* tiles, int* status) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int* cnt = scratch + 4 * kTileListPitch;  // [0], [1]: list lengths
  compact_routes(rows, topk, i_first, nq, scratch, status);
  const int na = cnt[0];
  const int* A = scratch;
  if (QB == 1 || nq == 1) {
    for (int k = tid; k < na; k += blockDim.x) tiles[k] = (A[k] << 4) | (k == na - 1 ? 2 : 1);
    __syncthreads();
    return na;
  }
  const int nb = cnt[1];
  const int* B = scratch + kTileListPitch;
  int* inA = scratch + 2 * kTileListPitch;  // [k]: B[k] is also in A
  int* dup = scratch + 3 * kTileListPitch;  // [k]: duplicates among B[0 .. k-1]
  if (warp == 0) {
    int run = 0;
    for (int k0 = 0; k0 <= nb; k0 += 32) {
      const int k = k0 + lane;
      int f = 0;
      if (k < nb) {
        const int la = lower_bound_smem(A, na, B[k]);
        f = (la < na && A[la] == B[k]) ? 1 : 0;
        inA[k] = f;
      }
      int incl = f;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (k <= nb) dup[k] = run + incl - f;  // exclusive
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  __syncthreads();
  for (int k = tid; k < na; k += blockDim.x) {
    const int a = A[k];
    const int lb = lower_bound_smem(B, nb, a);
    const bool inB = lb < nb && B[lb] == a;
    const int mode = (k == na - 1 ? 2 : 1) | (inB ? (lb == nb - 1 ? 2 : 1) << 2 : 0);
    tiles[k + lb - dup[lb]] = (a << 4) | mode;
  }
  for (int k = tid; k < nb; k += blockDim.x) {
    if (inA[k]) continue;
    const int b = B[k];
    const int la = lower_bound_smem(A, na, b);
    tiles[la + k - dup[k]] = (b << 4) | ((k == nb - 1 ? 2 : 1) << 2);
  }
  const int n = na + nb - dup[nb];
  __syncthreads();
  return n;
}

}  // namespace pyr
