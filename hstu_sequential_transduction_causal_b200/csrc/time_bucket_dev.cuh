// time_bucket_dev.cuh - device evaluation of the relative-time bucket
//   bucket(dt) = min(nb - 1, floor(ln(max(dt, 1)) / 0.301))
// from the exact integer thresholds of time_bucket_table.h: o = floor(log2 dt) selects an octave,
// whose base count plus up to three comparisons give the bucket. No floating point is involved,
// so the result is exact for every int64 dt. Each translation unit holds its own constant copy.
#pragma once

#include <cuda_runtime.h>

#include "time_bucket_table.h"

namespace hstu {
namespace {

__constant__ long long c_time_octaves[63][4];

__device__ __forceinline__ int time_bucket_dev(long long dt, const long long (*oct)[4], int nb) {
  int b = 0;
  if (dt > 1) {
    const int o = 63 - __clzll(dt);
    b = static_cast<int>(oct[o][3]) + (dt >= oct[o][0]) + (dt >= oct[o][1]) + (dt >= oct[o][2]);
  }
  return min(b, nb - 1);
}

// Copies the octave table to this translation unit's constant bank, once per device.
inline cudaError_t upload_time_octaves() {
  static bool done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
  e = cudaMemcpyToSymbol(c_time_octaves, kHstuTimeOctaves, sizeof(kHstuTimeOctaves));
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
  return e;
}

}  // namespace
}  // namespace hstu
