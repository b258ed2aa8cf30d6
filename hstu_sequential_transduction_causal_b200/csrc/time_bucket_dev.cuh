// time_bucket_dev.cuh - device evaluation of the relative-time bucket
//   bucket(dt) = min(nb - 1, floor(ln(max(dt, 1)) / 0.301)) = min(nb - 1, #{k >= 1 : tau_k <= dt})
// from the exact integer thresholds tau_k = ceil(exp(0.301 k)) of time_bucket_table.h. A float
// estimate of ln(dt) / 0.301 (error about 1e-5, so its integer part is at most one away from the
// exact count) is corrected by one integer comparison on each side: the result is exact for every
// int64 dt. The table is staged as tau[0..128] with tau_0 = INT64_MIN and tau_128 = INT64_MAX
// sentinels. Each translation unit holds its own constant copy.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "time_bucket_table.h"

namespace hstu {
namespace {

constexpr int kTauEntries = 129;
__constant__ long long c_time_taus[kTauEntries];

__device__ __forceinline__ int time_bucket_dev(long long dt, const long long* tau, int nb) {
  if (dt <= 1) return 0;
  constexpr float kLn2Over0301 = 0.693147180559945f / 0.301f;
  const float lf = __log2f(__ll2float_rn(dt)) * kLn2Over0301;   // >= 2.3 for dt >= 2
  int k = min(static_cast<int>(lf), 126);
  k += (dt >= tau[k + 1] ? 1 : 0) - (dt < tau[k] ? 1 : 0);
  return min(k, nb - 1);
}

// bucket(t_q - t_k) for any two int64 timestamps. The difference is formed in unsigned 64-bit
// arithmetic, so it never overflows: t_q <= t_k gives bucket 0, and a difference above INT64_MAX
// exceeds every threshold (all are below 2^63), which gives the last bucket.
__device__ __forceinline__ int time_bucket_pair64(long long tq, long long tk, const long long* tau, int nb) {
  if (tq <= tk) return 0;
  const unsigned long long u = static_cast<unsigned long long>(tq) - static_cast<unsigned long long>(tk);
  if (u > 0x7fffffffffffffffULL) return nb - 1;
  return time_bucket_dev(static_cast<long long>(u), tau, nb);
}

// The same for a difference known to fit in int32 (timestamps of a tile within 2^31 of each other):
// tau32 holds tau_k saturated to INT32_MAX (tau_72 > 2^31 > every int32 dt, so no bucket past 71 is
// reached) and tau32[0] = INT32_MIN; all arithmetic is 32-bit.
__constant__ int c_time_taus32[kTauEntries];

// Branch-free: dt <= 1 is clamped to 1, whose estimate is 0 and whose corrections are both 0
// (tau[1] = 2 > 1, tau[0] = INT32_MIN), so bucket 0 falls out of the general path. The estimate is
// integer arithmetic (one leading-zero count, no conversions or logarithm on the special-function
// unit): log2(v) is replaced by its chord on each octave, e + f with e the position of the leading
// one and f the bits below it read as a fraction, which lies at most 0.0861 below log2(v); in 8.24
// fixed point times 590 / 256 (for 1 / (0.301 log2 e) = 2.30284) the estimate of ln(v) / 0.301 is
// within (-0.2, +0.06) of it for v < 2^31, so its floor is at most one bucket off and the two
// threshold comparisons make the result exact.
__device__ __forceinline__ int time_bucket32(int dt, const int* tau, int nb) {
  const int v = max(dt, 1);
  const unsigned u = static_cast<unsigned>(v);
  const int lz = __clz(v);
  const unsigned fx = (static_cast<unsigned>(31 - lz) << 24) | (((u << lz) << 1) >> 8);
  int k = min(static_cast<int>(__umulhi(fx, 590u)), 126);
  k += (v >= tau[k + 1] ? 1 : 0) - (v < tau[k] ? 1 : 0);
  return min(k, nb - 1);
}

// The same tables in global memory, for kernels that stage them into shared memory: a warp reads 32
// consecutive entries in one request, where reads of different constant-bank entries by the lanes of
// a warp are serialised (and, on an SM's first touch, each one misses the constant cache).
__device__ long long g_time_taus[kTauEntries];
__device__ int g_time_taus32[kTauEntries];

// Copies tau_0..tau_128 to this translation unit's constant bank and global mirrors, once per device. The copies are
// synchronous, so the first call on a device must come before any stream capture. Safe to call from
// several host threads: the upload is serialised and later calls only read a flag.
inline cudaError_t upload_time_taus() {
  static std::atomic<bool> done[64];
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool tracked = dev >= 0 && dev < 64;
  if (tracked && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  std::lock_guard<std::mutex> lock(mu);
  if (tracked && done[dev].load(std::memory_order_relaxed)) return cudaSuccess;
  long long taus[kTauEntries];
  taus[0] = -0x7fffffffffffffffLL - 1;
  for (int k = 1; k <= HSTU_TB_NUM_THRESHOLDS; ++k) taus[k] = kHstuTimeThresholds[k - 1];
  for (int k = HSTU_TB_NUM_THRESHOLDS + 1; k < kTauEntries; ++k) taus[k] = 0x7fffffffffffffffLL;
  e = cudaMemcpyToSymbol(c_time_taus, taus, sizeof(taus));
  int taus32[kTauEntries];
  for (int k = 0; k < kTauEntries; ++k)
    taus32[k] = k == 0 ? (-0x7fffffff - 1) : (taus[k] > 0x7fffffffLL ? 0x7fffffff : static_cast<int>(taus[k]));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(c_time_taus32, taus32, sizeof(taus32));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_time_taus, taus, sizeof(taus));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_time_taus32, taus32, sizeof(taus32));
  if (e == cudaSuccess && tracked) done[dev].store(true, std::memory_order_release);
  return e;
}

}  // namespace
}  // namespace hstu
