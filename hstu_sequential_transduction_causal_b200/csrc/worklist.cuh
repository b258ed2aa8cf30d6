// worklist.cuh - the jagged tile work list of a batch of at most 32 sequences, computed by one warp
// ("4.4 Scaling Recommendation Models", Efficiency tricks: kernels over variable-length sequences).
// Lane b owns sequence b. The items (b, query tile t) are written tile index by tile index, tiles
// with more causal key tiles first, ties by increasing b; the key-tile list mirrors it. Short
// sequences share a tile (pack): a run of consecutive sequences of at most kPackMaxLen tokens each
// (empty ones included) whose rows add up to at most 128 becomes one item (b, -k), greedily in batch
// order. Also validates the offsets (offsets[0] == 0, lengths in [0, max_len], offsets[B] == T); a
// violation records kDevBadInput and empties the lists so no later kernel reads out of bounds.
// Used by the work-list kernel and, for the layer forward, by an idle warp of the f1 GEMM launch.
#pragma once

#include <stdint.h>

#include "hstu_internal.h"
#include "sm100_ptx.cuh"

namespace hstu {
namespace {

constexpr int kPackMaxLen = 64;

// Unit records of the persistent attention forward, one per work item p: {b, tile, row0, n, pair0,
// 0, 0, 0} (int32): the item, the first row and row count its tiles cover (a pack's rows for a pack),
// and the index of its query tile's first causal pair. Run by threads [tid, tid + nthreads) after
// items, count and pair_base are written and visible to them.
__device__ void write_unit_records(const int64_t* __restrict__ off, const int32_t* items, int count,
                                   const long long* pair_base, int32_t* urec, int tid, int nthreads) {
  for (int p = tid; p < count; p += nthreads) {
    const int b = items[2 * p], t = items[2 * p + 1];
    const int k = t < 0 ? -t : 1;
    const int qt = t < 0 ? 0 : t;
    int4 r0, r1;
    r0.x = b;
    r0.y = t;
    r0.z = static_cast<int>(off[b]);
    r0.w = static_cast<int>(off[b + k] - off[b]);
    r1.x = static_cast<int>(pair_base[b] + static_cast<long long>(qt) * (qt + 1) / 2);
    r1.y = r1.z = r1.w = 0;
    reinterpret_cast<int4*>(urec)[2 * p] = r0;
    reinterpret_cast<int4*>(urec)[2 * p + 1] = r1;
  }
}

// The whole list from one full warp (B <= 32; the caller checks). Every lane's length is loaded
// once; the packing walks the lengths by shuffles (uniform control flow), not by dependent loads.
__device__ void worklist_warp(const WorklistArgs& w) {
  const int lane = threadIdx.x & 31;
  const int B = w.B;
  if (lane == 0) {   // the persistent attention kernels' unit (and finished-CTA) counters
    if (w.sched) w.sched[0] = 0;
    if (w.sched2) w.sched2[0] = w.sched2[1] = 0;
  }
  const bool mine = lane < B;
  long long n = 0;
  if (mine) n = w.off[lane + 1] - w.off[lane];
  bool bad = (B < 0 || B > 32 || w.off[0] != 0 || w.off[B > 0 ? B : 0] != w.T || (mine && (n < 0 || n > w.max_len)));
  bad = __any_sync(0xffffffffu, bad);
  if (bad) {
    if (lane == 0) {
      *w.count = 0;
      if (w.kcount) *w.kcount = 0;
      report_error(w.status, kDevBadInput);
      if (w.pair_base) w.pair_base[B > 0 && B <= 32 ? B : 0] = 0;
    }
    return;
  }
  const int nt_all = mine ? static_cast<int>((n + kQTile - 1) / kQTile) : 0;
  // pack[b]: k >= 2 for the first sequence of a pack of k, 0 for the other members, 1 on its own
  int pk = 1;
  if (w.pack) {
    for (int i = 0; i < B;) {
      const long long ni = __shfl_sync(0xffffffffu, n, i);
      if (ni <= 0 || ni > kPackMaxLen) {
        ++i;
        continue;
      }
      long long total = ni;
      int k = 1;
      while (i + k < B) {
        const long long m = __shfl_sync(0xffffffffu, n, i + k);
        if (m > kPackMaxLen || total + m > kQTile) break;
        total += m;
        ++k;
      }
      if (lane == i) pk = k;
      else if (lane > i && lane < i + k) pk = 0;
      i += k;
    }
    if (mine) w.pack[lane] = pk;
  }
  const int nt = pk == 0 ? 0 : nt_all;   // a pack member's rows are in its pack's tile
  int max_tiles = nt;
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) max_tiles = max(max_tiles, __shfl_xor_sync(0xffffffffu, max_tiles, d));
  int base = 0;
  for (int t = max_tiles - 1; t >= 0; --t) {
    const bool flag = nt > t;
    const unsigned m = __ballot_sync(0xffffffffu, flag);
    if (flag) {
      const int pos = base + __popc(m & ((1u << lane) - 1u));
      w.items[2 * pos] = lane;
      w.items[2 * pos + 1] = pk >= 2 ? -pk : t;
      if (w.kitems) {
        w.kitems[2 * pos] = lane;
        w.kitems[2 * pos + 1] = pk >= 2 ? -pk : nt - 1 - t;
      }
    }
    base += __popc(m);
  }
  if (lane == 0) {
    *w.count = base;
    if (w.kcount) *w.kcount = base;
  }
  if (!w.pair_base) return;
  // pair_base[b] = sum_{b' < b} nt_b' (nt_b' + 1) / 2: index of sequence b's first causal
  // (query tile, key tile) pair; pair_base[B] is the total.
  const long long v = static_cast<long long>(nt_all) * (nt_all + 1) / 2;
  long long inc = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, inc, d);
    if (lane >= d) inc += y;
  }
  if (mine) w.pair_base[lane] = inc - v;
  const long long total = __shfl_sync(0xffffffffu, inc, 31);
  if (lane == 0) w.pair_base[B] = total;
  if (!w.urec) return;
  __syncwarp();
  write_unit_records(w.off, w.items, base, w.pair_base, w.urec, lane, 32);
}

}  // namespace
}  // namespace hstu
