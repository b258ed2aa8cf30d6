// stochastic_length.cu - Stochastic Length subsampling of jagged sequences ("HSTU: The First
// Exploration of the Scaling Law", 7.1.5 Stochastic Length): a history of n tokens keeps
// L = min(n, floor(n^(alpha/2) + 1/2)) of them, the L tokens with the smallest random keys (ties by
// position), in their original order. The random keys are inputs (one int64 per raw token).
//
//  sl_lengths_kernel: one block; L_b per sequence and their exclusive prefix (the new offsets).
//  sl_select_kernel:  one block per sequence; a radix select over the 64-bit keys finds the L-th
//                     smallest key k* and the rank r of the last kept token among those equal to k*;
//                     then block-wide scans keep, in position order, every token with key < k* and
//                     the first r + 1 tokens with key == k*, and write their global indices, their
//                     timestamps and their rows of X.
#include <cuda_runtime.h>
#include <stdint.h>

#include "hstu_internal.h"
#include "sm100_ptx.cuh"

namespace hstu {

namespace {

constexpr int kSlThreads = 1024;
constexpr int kSlWarps = kSlThreads / 32;

__device__ __forceinline__ long long keep_count(long long n, double half_alpha) {
  if (n <= 0) return 0;
  const long long L = static_cast<long long>(floor(pow(static_cast<double>(n), half_alpha) + 0.5));
  return L < n ? (L < 0 ? 0 : L) : n;
}

// Exclusive block-wide prefix of one int per thread; returns the block total in *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, d);
    if (lane >= d) inc += y;
  }
  if (lane == 31) s_warp[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const int w = s_warp[lane];
    int winc = w;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, winc, d);
      if (lane >= d) winc += y;
    }
    s_warp[lane] = winc - w;
    if (lane == 31) s_warp[32] = winc;
  }
  __syncthreads();
  const int excl = s_warp[warp] + inc - v;
  *total = s_warp[32];
  __syncthreads();
  return excl;
}

__global__ void __launch_bounds__(kSlThreads)
sl_lengths_kernel(const int64_t* __restrict__ off, int B, double half_alpha, int64_t* __restrict__ new_off,
                  int* status) {
  __shared__ long long s_wsum[kSlWarps];
  __shared__ long long s_run;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    s_run = 0;
    if (off[0] != 0) report_error(status, kDevBadInput);
  }
  __syncthreads();
  for (int c0 = 0; c0 < B; c0 += kSlThreads) {
    const int b = c0 + tid;
    long long v = 0;
    if (b < B) {
      const long long n = off[b + 1] - off[b];
      if (n < 0) report_error(status, kDevBadInput);
      v = keep_count(n, half_alpha);
    }
    long long inc = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, inc, d);
      if (lane >= d) inc += y;
    }
    if (lane == 31) s_wsum[warp] = inc;
    __syncthreads();
    if (warp == 0) {
      const long long w = s_wsum[lane];
      long long winc = w;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, winc, d);
        if (lane >= d) winc += y;
      }
      s_wsum[lane] = winc - w;
    }
    __syncthreads();
    const long long excl = s_run + s_wsum[warp] + inc - v;
    if (b < B) new_off[b] = excl;
    __syncthreads();
    if (tid == kSlThreads - 1) s_run = excl + v;
    __syncthreads();
  }
  if (tid == 0) new_off[B] = s_run;
}

__global__ void __launch_bounds__(kSlThreads)
sl_select_kernel(const int64_t* __restrict__ off, const int64_t* __restrict__ ts, const int64_t* __restrict__ keys,
                 const int64_t* __restrict__ new_off, const uint8_t* __restrict__ x, int64_t row_bytes,
                 int64_t* __restrict__ kept, uint8_t* __restrict__ x_out, int64_t* __restrict__ ts_out,
                 int* status) {
  __shared__ unsigned int s_hist[256];
  __shared__ int s_warp[33];
  __shared__ unsigned long long s_prefix;
  __shared__ long long s_rank;
  const int tid = threadIdx.x;
  const int b = blockIdx.x;
  const long long s0 = off[b];
  const long long n = off[b + 1] - s0;
  const long long o0 = new_off[b];
  const long long L = new_off[b + 1] - o0;
  if (L <= 0 || n <= 0) return;
  if (L > n) {   // offsets not produced by sl_lengths for this batch: nothing is written
    if (tid == 0) report_error(status, kDevBadInput);
    return;
  }
  auto ukey = [&](long long i) {
    return static_cast<unsigned long long>(keys[s0 + i]) ^ 0x8000000000000000ull;   // signed -> unsigned order
  };
  unsigned long long kstar = ~0ull;
  long long rstar = n;           // every token with key == kstar and equal-rank <= rstar is kept
  if (L < n) {
    // radix select of the element of rank L - 1 (0-based, ascending)
    unsigned long long prefix = 0, mask = 0;
    long long r = L - 1;
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = 56 - 8 * pass;
      for (int d = tid; d < 256; d += kSlThreads) s_hist[d] = 0;
      __syncthreads();
      for (long long i = tid; i < n; i += kSlThreads) {
        const unsigned long long u = ukey(i);
        if ((u & mask) == prefix) atomicAdd(&s_hist[(u >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (tid == 0) {
        long long cum = 0;
        int sel = 255;
        for (int d = 0; d < 256; ++d) {
          if (cum + s_hist[d] > r) {
            sel = d;
            break;
          }
          cum += s_hist[d];
        }
        s_prefix = prefix | (static_cast<unsigned long long>(sel) << shift);
        s_rank = r - cum;
      }
      __syncthreads();
      prefix = s_prefix;
      r = s_rank;
      mask |= 255ull << shift;
      __syncthreads();
    }
    kstar = prefix;
    rstar = r;
  }
  // keep in position order: key < kstar, or key == kstar with equal-rank <= rstar
  long long eq_base = 0, out_base = 0;
  for (long long c0 = 0; c0 < n; c0 += kSlThreads) {
    const long long i = c0 + tid;
    const bool in = i < n;
    const unsigned long long u = in ? ukey(i) : ~0ull;
    const bool eq = in && L < n && u == kstar;
    int eq_total = 0;
    const int eq_rank = block_exclusive_scan(eq ? 1 : 0, s_warp, &eq_total);
    const bool keep = in && (L == n || u < kstar || (eq && eq_base + eq_rank <= rstar));
    int keep_total = 0;
    const int pos = block_exclusive_scan(keep ? 1 : 0, s_warp, &keep_total);
    if (keep) {
      const long long o = o0 + out_base + pos;
      kept[o] = s0 + i;
      if (ts_out) ts_out[o] = ts[s0 + i];
    }
    eq_base += eq_total;
    out_base += keep_total;
  }
  if (!x_out) return;
  __syncthreads();   // kept[] of this sequence is written (global memory, same block)
  // rows: one warp per kept token, 16-byte vectors
  const int lane = tid & 31, warp = tid >> 5;
  const long long vecs = row_bytes / 16;
  for (long long o = warp; o < L; o += kSlWarps) {
    const long long src = kept[o0 + o];
    const uint4* sp = reinterpret_cast<const uint4*>(x + src * row_bytes);
    uint4* dp = reinterpret_cast<uint4*>(x_out + (o0 + o) * row_bytes);
    for (long long v = lane; v < vecs; v += 32) dp[v] = sp[v];
  }
}

}  // namespace

cudaError_t launch_sl_lengths(const int64_t* offsets, int B, double alpha, int64_t* new_offsets, int* status,
                              cudaStream_t st) {
  sl_lengths_kernel<<<1, kSlThreads, 0, st>>>(offsets, B, 0.5 * alpha, new_offsets, status);
  return cudaGetLastError();
}

cudaError_t launch_sl_select(const int64_t* offsets, int B, const int64_t* ts, const int64_t* keys,
                             const int64_t* new_offsets, const void* x, int64_t row_bytes, int64_t* kept, void* x_out,
                             int64_t* ts_out, int* status, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  sl_select_kernel<<<B, kSlThreads, 0, st>>>(offsets, ts, keys, new_offsets, static_cast<const uint8_t*>(x), row_bytes,
                                             kept, static_cast<uint8_t*>(x_out), ts_out, status);
  return cudaGetLastError();
}

}  // namespace hstu
