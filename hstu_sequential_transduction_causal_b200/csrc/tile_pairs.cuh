// tile_pairs.cuh - numbering of the causal (query tile, key tile) pairs of a jagged batch.
// Sequence b with nt_b = ceil(n_b / 128) tiles owns pairs [pair_base[b], pair_base[b+1]) with
// pair_base[b] = sum_{b' < b} nt_b' (nt_b' + 1) / 2; inside it, pair (qt, kt <= qt) is number
// qt (qt + 1) / 2 + kt. Bias tiles are stored in this order.
#pragma once

#include <stdint.h>

namespace hstu {

// Decodes pair p into (b, qt, kt); false when p is past the batch's last pair.
__device__ __forceinline__ bool decode_tile_pair(long long p, const long long* __restrict__ pair_base, int B, int* b,
                                                 int* qt, int* kt) {
  if (B <= 0 || p >= pair_base[B]) return false;
  int lo = 0, hi = B;   // invariant: pair_base[lo] <= p < pair_base[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (pair_base[mid] <= p) lo = mid;
    else hi = mid;
  }
  const long long l = p - pair_base[lo];
  int q = static_cast<int>((sqrt(8.0 * static_cast<double>(l) + 1.0) - 1.0) * 0.5);
  while (static_cast<long long>(q + 1) * (q + 2) / 2 <= l) ++q;
  while (q > 0 && static_cast<long long>(q) * (q + 1) / 2 > l) --q;
  *b = lo;
  *qt = q;
  *kt = static_cast<int>(l - static_cast<long long>(q) * (q + 1) / 2);
  return true;
}

// Rows covered by the tiles of causal pair (b, qt, kt): sequence b (from row seq0, n rows), or,
// for the only pair of the first sequence of a pack of k >= 2 short sequences (pack[b] = k), the
// pack's rows. False for the pair of a pack member, which no tile uses.
__device__ __forceinline__ bool pair_rows(const int64_t* __restrict__ offsets, const int32_t* __restrict__ pack,
                                          int b, long long* seq0, int* n) {
  *seq0 = offsets[b];
  int k = 1;
  if (pack) {
    k = pack[b];
    if (k == 0) return false;
  }
  *n = static_cast<int>(offsets[b + k] - *seq0);
  return true;
}

}  // namespace hstu
