// bias_tile.cuh - the relative half-bias of one causal (query tile, key tile) pair, computed by one
// block of 256 threads:
//   bias(i, j) = 0.5 (rab_pos[clamp(i - j)] + rab_time[bucket(t_i - t_j)])
// ("HSTU: The First Exploration of the Scaling Law", 7.1.4 Innovation 2: position and time bias;
// the buckets of time_bucket_dev.cuh). The bias does not depend on the head, so a pair's tile is
// computed once and read by every head.
//
// Thread t takes the column pairs 2 (t % 16) + 32 e, e < 4, of the rows t / 16 + 16 p, p < 8: 64
// elements, 4-byte half-bias (and 2-byte bucket) stores. TRANSPOSED: rows are keys and columns
// queries (the backward's [key][query] tiles); otherwise rows are queries. Timestamps past
// the sequence end are clamped to its last token (those elements are masked by the attention).
// When every difference of the tile fits in int32 (spans under 68 years of seconds) the bucket
// arithmetic is 32-bit.
#pragma once

#include <stdint.h>

#include "hstu_internal.h"
#include "sm100_ptx.cuh"
#include "tile_pairs.cuh"
#include "time_bucket_dev.cuh"

namespace hstu {
namespace {

constexpr int kBiasThreads = 256;

__device__ __forceinline__ int bias_pos_index(long long r, int L) {
  r = r > L - 1 ? L - 1 : r;
  r = r < -(L - 1) ? -(L - 1) : r;
  return static_cast<int>(r) + L - 1;
}

template <bool TRANSPOSED, bool BUCKETS>
__device__ __forceinline__ void bias_tile_block(const AttnArgs& a, long long pair, uint16_t* __restrict__ tile,
                                                uint8_t* __restrict__ btile) {
  __shared__ long long s_ts[256];          // [0,128): query timestamps, [128,256): key timestamps
  __shared__ int s_ts32[256];              // the same minus the tile minimum (fast path)
  __shared__ long long s_tau[kTauEntries];
  __shared__ int s_tau32[kTauEntries];
  __shared__ float s_win[256], s_rt[128];
  __shared__ long long s_red[16];
  int b, qt, kt;
  if (!decode_tile_pair(pair, a.pair_base, a.B, &b, &qt, &kt)) return;
  const long long seq0 = a.offsets[b];
  const int n = static_cast<int>(a.offsets[b + 1] - seq0);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  {
    const int idx = (tid < 128 ? qt : kt) * kQTile + (tid & 127);
    const long long t = a.ts[seq0 + (idx < n ? idx : n - 1)];
    s_ts[tid] = t;
    long long mn = t, mx = t;
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) {
      mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, d));
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, d));
    }
    if (lane == 0) {
      s_red[warp] = mn;
      s_red[8 + warp] = mx;
    }
  }
  if (tid < a.n_buckets) s_rt[tid] = 0.5f * a.rab_time[tid];
  if (tid < 255) s_win[tid] = 0.5f * a.rab_pos[bias_pos_index(static_cast<long long>(qt - kt) * kQTile - 127 + tid,
                                                               a.pos_max_len)];
  for (int e = tid; e < kTauEntries; e += kBiasThreads) {
    s_tau[e] = c_time_taus[e];
    s_tau32[e] = c_time_taus32[e];
  }
  __syncthreads();
  long long lo = s_red[0], hi = s_red[8];
#pragma unroll
  for (int w = 1; w < 8; ++w) {
    lo = min(lo, s_red[w]);
    hi = max(hi, s_red[8 + w]);
  }
  const bool fast = hi - lo < 0x7fffffffLL;
  if (fast) s_ts32[tid] = static_cast<int>(s_ts[tid] - lo);
  __syncthreads();
  const int nb = a.n_buckets;
  // thread: column pairs c = 2 (tid % 16) + 32 e + x (e < 4, x < 2) of rows r = tid / 16 + 16 p (p < 8).
  // The 16 lanes of a half-warp read 32 consecutive diagonals of the rab_pos window (no bank
  // conflicts) and store 64 contiguous bytes of one row.
  const int cl = 2 * (tid & 15), rr = tid >> 4;
  // the query / key timestamp arrays of rows and columns
  const int row_base = TRANSPOSED ? 128 : 0, col_base = TRANSPOSED ? 0 : 128;
  if (fast) {
    int tc[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      tc[2 * e] = s_ts32[col_base + cl + 32 * e];
      tc[2 * e + 1] = s_ts32[col_base + cl + 32 * e + 1];
    }
#pragma unroll 2
    for (int p = 0; p < 8; ++p) {
      const int r = rr + 16 * p;
      const int tr = s_ts32[row_base + r];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v2[2];
        uint32_t bw = 0u;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int c = cl + 32 * e + x;
          const int dt = TRANSPOSED ? tc[2 * e + x] - tr : tr - tc[2 * e + x];   // t_query - t_key
          const int bkt = time_bucket32(dt, s_tau32, nb);
          v2[x] = s_win[TRANSPOSED ? c - r + 127 : r - c + 127] + s_rt[bkt];
          bw |= static_cast<uint32_t>(bkt) << (8 * x);
        }
        *reinterpret_cast<uint32_t*>(tile + r * kQTile + cl + 32 * e) = pack_f16x2(v2[0], v2[1]);
        if (BUCKETS) *reinterpret_cast<uint16_t*>(btile + r * kQTile + cl + 32 * e) = static_cast<uint16_t>(bw);
      }
    }
  } else {
#pragma unroll 1
    for (int p = 0; p < 8; ++p) {
      const int r = rr + 16 * p;
      const long long tr = s_ts[row_base + r];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v2[2];
        uint32_t bw = 0u;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int c = cl + 32 * e + x;
          const long long tcv = s_ts[col_base + c];
          const int bkt = time_bucket_dev(TRANSPOSED ? tcv - tr : tr - tcv, s_tau, nb);
          v2[x] = s_win[TRANSPOSED ? c - r + 127 : r - c + 127] + s_rt[bkt];
          bw |= static_cast<uint32_t>(bkt) << (8 * x);
        }
        *reinterpret_cast<uint32_t*>(tile + r * kQTile + cl + 32 * e) = pack_f16x2(v2[0], v2[1]);
        if (BUCKETS) *reinterpret_cast<uint16_t*>(btile + r * kQTile + cl + 32 * e) = static_cast<uint16_t>(bw);
      }
    }
  }
}

}  // namespace
}  // namespace hstu
