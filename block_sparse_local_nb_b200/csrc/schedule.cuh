// Work order of the persistent attention kernels.
//
// A work item is one 128-row tile of one (sequence, head).  Tiles that lie
// entirely past their sequence's length carry no work (only zero outputs), so
// a plain round-robin over all tiles leaves some SMs with many more real tiles
// than others when lengths vary.  The kernels instead walk the list of
// non-empty tiles round-robin (every SM gets the same number, +-1), then the
// list of empty tiles, whose outputs are zero-filled (none when every sequence
// is full length).  The list is implicit: a
// prefix table over sequences, pre[b] = number of non-empty tiles (all heads)
// of sequences before b, built once per CTA in shared memory and searched per
// item.  The clamped lengths sit beside it, so that decoding an item reads
// shared memory only (a global load there would stall every role of the CTA
// at each item boundary).  Batches larger than kMaxSchedBatch fall back to a
// round-robin over all tiles, with the lengths read from global memory.
#pragma once

#include "nb_internal.h"

namespace nb {

constexpr int kMaxSchedBatch = 1024;
// pre[0..batch], then the clamped lengths len[0..batch) from pre + kMaxSchedBatch + 1
constexpr int kSchedBytes = (2 * kMaxSchedBatch + 1) * 4;

// Warp-cooperative: fills pre[0..batch] and len[0..batch) (call with one full
// warp, then sync the CTA).
__device__ __forceinline__ void sched_build(int* pre, const AttnArgs& a, int rows_per_tile,
                                            int lane) {
  if (a.batch > kMaxSchedBatch) return;
  int carry = 0;
  for (int b0 = 0; b0 < a.batch; b0 += 32) {
    const int b = b0 + lane;
    int v = 0;
    if (b < a.batch) {
      int L = a.lengths ? a.lengths[b] : a.n;
      L = min(max(L, 0), a.n);
      pre[kMaxSchedBatch + 1 + b] = L;
      v = a.heads * ((L + rows_per_tile - 1) / rows_per_tile);
    }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += t;
    }
    if (b < a.batch) pre[b + 1] = carry + v;
    carry += __shfl_sync(0xffffffffu, v, 31);
  }
  if (lane == 0) pre[0] = 0;
}

struct Sched {
  const int* pre;
  const int* len;  // clamped lengths (balanced only)
  bool balanced;   // walk the non-empty list (else every tile, round-robin)
  int count;       // items of the first pass
};

__device__ __forceinline__ Sched sched_view(const int* pre, const AttnArgs& a, int all_items) {
  Sched s;
  s.pre = pre;
  s.len = pre + kMaxSchedBatch + 1;
  s.balanced = a.batch <= kMaxSchedBatch;
  s.count = s.balanced ? pre[a.batch] : all_items;
  return s;
}

// Length of sequence b clamped to [0, n].
__device__ __forceinline__ int sched_length(const Sched& s, const AttnArgs& a, int b) {
  if (s.balanced) return s.len[b];
  const int L = a.lengths ? a.lengths[b] : a.n;
  return min(max(L, 0), a.n);
}

// (sequence, head, tile) of item k of the non-empty list.
__device__ __forceinline__ void sched_nonempty(const Sched& s, int batch, int heads, int k, int& b,
                                               int& h, int& tile) {
  int lo = 0, hi = batch - 1;  // largest b with pre[b] <= k
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s.pre[mid] <= k) lo = mid; else hi = mid - 1;
  }
  b = lo;
  const int T = (s.pre[b + 1] - s.pre[b]) / heads;
  const int rem = k - s.pre[b];
  h = rem / T;
  tile = rem - h * T;
}

// (sequence, head, tile) of item e of the empty list: the tiles of sequence b
// from ceil(L_b / rows) on, for every head.  Before sequence b there are
// b * heads * ntiles - pre[b] of them.
__device__ __forceinline__ void sched_empty(const Sched& s, int batch, int heads, int ntiles, int e,
                                            int& b, int& h, int& tile) {
  int lo = 0, hi = batch - 1;  // largest b with epre(b) <= e
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (mid * heads * ntiles - s.pre[mid] <= e) lo = mid; else hi = mid - 1;
  }
  b = lo;
  const int T = (s.pre[b + 1] - s.pre[b]) / heads;  // non-empty tiles per head
  const int rem = e - (b * heads * ntiles - s.pre[b]);
  h = rem / (ntiles - T);
  tile = T + (rem - h * (ntiles - T));
}

}  // namespace nb
