// falcon_append.cu - row movement of the M-FALCON prefix append ("HSTU: The First Exploration of the
// Scaling Law", 7.1.5 M-FALCON: the history's K, V cache is reused across requests).
//
// A user's cached prefix of n_old tokens grows by a new actions. In the combined prefix (user u owns
// rows [new_off[u], new_off[u + 1]), n_old + a of them) the first n_old rows keep their cached K, V
// (a causal layer's K, V of a token do not depend on later tokens), and the a appended rows get the K,
// V their own layer input gives. append_scatter_kernel builds one layer of the combined cache and the
// combined query buffer (the appended rows' Q at their combined rows, zeros elsewhere);
// append_gather_kernel brings the attention output of the appended rows back to their own order.
// One warp per row, 16-byte copies. A combined length other than n_old + a is reported as bad input
// and the user's rows are left untouched.
#include <cuda_runtime.h>
#include <stdint.h>

#include "hstu_internal.h"
#include "sm100_ptx.cuh"

namespace hstu {
namespace {

// The sequence owning row r of a batch with offsets off[0..B] (off[b] <= r < off[b + 1]).
__device__ __forceinline__ int owner_of(const int64_t* __restrict__ off, int B, long long r) {
  int lo = 0, hi = B;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (off[mid] <= r) lo = mid;
    else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ void copy16(const uint8_t* src, uint8_t* dst, int bytes, int lane) {
  for (int o = lane * 16; o < bytes; o += 32 * 16)
    *reinterpret_cast<uint4*>(dst + o) = *reinterpret_cast<const uint4*>(src + o);
}

__device__ __forceinline__ void zero16(uint8_t* dst, int bytes, int lane) {
  for (int o = lane * 16; o < bytes; o += 32 * 16) *reinterpret_cast<uint4*>(dst + o) = make_uint4(0, 0, 0, 0);
}

// cache rows are [K | V], 2D fp16; uvqk rows [U | V | Q | K], 4D fp16; q rows D fp16
__global__ void __launch_bounds__(256)
append_scatter_kernel(const int64_t* __restrict__ old_off, const int64_t* __restrict__ app_off,
                      const int64_t* __restrict__ new_off, int users, int64_t T_new, int D,
                      const uint16_t* __restrict__ old_cache, const uint16_t* __restrict__ uvqk, uint16_t* new_cache,
                      uint16_t* qbuf, int* status) {
  pdl_enter();
  const long long r = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= T_new) return;
  const int u = owner_of(new_off, users, r);
  const long long j = r - new_off[u];
  const long long n_old = old_off[u + 1] - old_off[u], n_app = app_off[u + 1] - app_off[u];
  if (n_old + n_app != new_off[u + 1] - new_off[u]) {
    if (j == 0 && lane == 0) report_error(status, kDevBadInput);
    return;
  }
  uint8_t* cache_row = reinterpret_cast<uint8_t*>(new_cache + r * 2 * D);
  uint8_t* q_row = reinterpret_cast<uint8_t*>(qbuf + r * D);
  if (j < n_old) {
    copy16(reinterpret_cast<const uint8_t*>(old_cache + (old_off[u] + j) * 2 * D), cache_row, 4 * D, lane);
    zero16(q_row, 2 * D, lane);
  } else {
    const uint8_t* src = reinterpret_cast<const uint8_t*>(uvqk + (app_off[u] + (j - n_old)) * 4 * D);
    copy16(src + 6 * D, cache_row, 2 * D, lane);          // K
    copy16(src + 2 * D, cache_row + 2 * D, 2 * D, lane);  // V
    copy16(src + 4 * D, q_row, 2 * D, lane);              // Q
  }
}

// o_app[i] = o_comb[combined row of appended row i], fp32 rows of D
__global__ void __launch_bounds__(256)
append_gather_kernel(const int64_t* __restrict__ old_off, const int64_t* __restrict__ app_off,
                     const int64_t* __restrict__ new_off, int users, int64_t A, int D,
                     const float* __restrict__ o_comb, float* o_app) {
  pdl_enter();
  const long long i = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (i >= A) return;
  const int u = owner_of(app_off, users, i);
  const long long r = new_off[u] + (old_off[u + 1] - old_off[u]) + (i - app_off[u]);
  if (r >= new_off[u + 1]) return;   // inconsistent lengths, reported by the scatter
  copy16(reinterpret_cast<const uint8_t*>(o_comb + r * D), reinterpret_cast<uint8_t*>(o_app + i * D), 4 * D, lane);
}

}  // namespace

cudaError_t falcon_append_scatter(const int64_t* old_off, const int64_t* app_off, const int64_t* new_off, int users,
                                  int64_t T_new, int D, const uint16_t* old_cache, const uint16_t* uvqk,
                                  uint16_t* new_cache, uint16_t* qbuf, int* status, cudaStream_t st) {
  if (T_new == 0) return cudaSuccess;
  return launch_pdl(append_scatter_kernel, dim3(static_cast<unsigned>((T_new + 7) / 8)), dim3(256), 0, st, old_off,
                    app_off, new_off, users, T_new, D, old_cache, uvqk, new_cache, qbuf, status);
}

cudaError_t falcon_append_gather(const int64_t* old_off, const int64_t* app_off, const int64_t* new_off, int users,
                                 int64_t A, int D, const float* o_comb, float* o_app, cudaStream_t st) {
  if (A == 0) return cudaSuccess;
  return launch_pdl(append_gather_kernel, dim3(static_cast<unsigned>((A + 7) / 8)), dim3(256), 0, st, old_off,
                    app_off, new_off, users, A, D, o_comb, o_app);
}

}  // namespace hstu
