// vec_io.cuh - per-thread vector loads/stores of VPT consecutive elements of an fp32, bf16 or
// fp16 row (16-byte accesses where VPT allows), converting to/from fp32 registers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "sm100_ptx.cuh"

namespace hstu {

template <int VPT, int DT>
__device__ __forceinline__ void load_vec(const void* base, int64_t idx, float* v) {
  if constexpr (DT == kDtOne) {
#pragma unroll
    for (int e = 0; e < VPT; ++e) v[e] = 1.0f;
  } else if constexpr (VPT == 1) {
    if constexpr (DT == kDtF32) v[0] = reinterpret_cast<const float*>(base)[idx];
    else if constexpr (DT == kDtBF16) v[0] = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[idx]);
    else v[0] = __half2float(reinterpret_cast<const __half*>(base)[idx]);
  } else if constexpr (DT == kDtF32) {
    const float* p = reinterpret_cast<const float*>(base) + idx;
    if constexpr (VPT % 4 == 0) {
#pragma unroll
      for (int q = 0; q < VPT / 4; ++q) {
        const float4 t = reinterpret_cast<const float4*>(p)[q];
        v[4 * q] = t.x; v[4 * q + 1] = t.y; v[4 * q + 2] = t.z; v[4 * q + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < VPT; ++e) v[e] = p[e];
    }
  } else {
    const uint16_t* p = reinterpret_cast<const uint16_t*>(base) + idx;
    if constexpr (VPT % 8 == 0) {
#pragma unroll
      for (int q = 0; q < VPT / 8; ++q) {
        const uint4 t = reinterpret_cast<const uint4*>(p)[q];
        const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = DT == kDtBF16 ? unpack_bf16x2(w[e]) : unpack_f16x2(w[e]);
          v[8 * q + 2 * e] = f.x;
          v[8 * q + 2 * e + 1] = f.y;
        }
      }
    } else if constexpr (VPT == 4) {   // one 8-byte load
      const uint2 t = *reinterpret_cast<const uint2*>(p);
      const float2 f0 = DT == kDtBF16 ? unpack_bf16x2(t.x) : unpack_f16x2(t.x);
      const float2 f1 = DT == kDtBF16 ? unpack_bf16x2(t.y) : unpack_f16x2(t.y);
      v[0] = f0.x; v[1] = f0.y; v[2] = f1.x; v[3] = f1.y;
    } else {
#pragma unroll
      for (int e = 0; e < VPT; e += 2) {
        const uint32_t w = reinterpret_cast<const uint32_t*>(p)[e / 2];
        const float2 f = DT == kDtBF16 ? unpack_bf16x2(w) : unpack_f16x2(w);
        v[e] = f.x;
        v[e + 1] = f.y;
      }
    }
  }
}

template <int VPT, int DT>
__device__ __forceinline__ void store_vec(void* base, int64_t idx, const float* v) {
  if constexpr (DT == kDtF32) {
    float* p = reinterpret_cast<float*>(base) + idx;
    if constexpr (VPT % 4 == 0) {
#pragma unroll
      for (int q = 0; q < VPT / 4; ++q)
        reinterpret_cast<float4*>(p)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
#pragma unroll
      for (int e = 0; e < VPT; ++e) p[e] = v[e];
    }
  } else {
    uint16_t* p = reinterpret_cast<uint16_t*>(base) + idx;
    auto pk = [](float a, float b) { return DT == kDtBF16 ? pack_bf16x2(a, b) : pack_f16x2(a, b); };
    if constexpr (VPT % 8 == 0) {
#pragma unroll
      for (int q = 0; q < VPT / 8; ++q)
        reinterpret_cast<uint4*>(p)[q] = make_uint4(pk(v[8 * q], v[8 * q + 1]), pk(v[8 * q + 2], v[8 * q + 3]),
                                                    pk(v[8 * q + 4], v[8 * q + 5]), pk(v[8 * q + 6], v[8 * q + 7]));
    } else if constexpr (VPT == 4) {   // one 8-byte store
      *reinterpret_cast<uint2*>(p) = make_uint2(pk(v[0], v[1]), pk(v[2], v[3]));
    } else {
#pragma unroll
      for (int e = 0; e < VPT; e += 2) reinterpret_cast<uint32_t*>(p)[e / 2] = pk(v[e], v[e + 1]);
    }
  }
}

}  // namespace hstu
