// gemm_sm100.cu - the layer's projection GEMMs on the 5th-generation tensor cores.
//
// C[M, N] = A[M, K] * B[N, K]^T with bf16 operands and fp32 accumulation in tensor memory.
// Each operand is either K-major (row-major [rows, K]) or MN-major (row-major [K, rows]), so the
// forward projections (X W1^T, G W2^T) and the backward ones (dY W2, dZ W1, dY^T G, dZ^T X)
// share one kernel. Operand tiles arrive by TMA (128-byte swizzle) into a STAGES-deep ring; one
// thread issues tcgen05.mma (M=128, N=BN, K=16) into TMEM; four warps run the fused epilogue:
//   SILU:   Z = acc + b;  out0 = SiLU(Z) (the U|V|Q|K activations), out1 = Z (optional)
//   LINEAR: Y = acc (+ b) (+ R);  out0 = Y, out1 = bf16 copy of Y (optional)
//   ATOMIC: out0 += acc (fp32 reductions for split-K weight gradients)
// ("4.4 Scaling Recommendation Models", Generative Recommenders and HSTU: f1 with phi1 = SiLU
// and the split into U, V, Q, K; f2 followed by the residual of the "Code" sketch.)
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hstu_internal.h"
#include "sm100_ptx.cuh"

namespace hstu {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kThreads = 192;   // warps 0-3 epilogue, warp 4 TMA, warp 5 MMA

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr int kABytes = kBM * kBK * 2;      // 16 KB
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTileBytes = STAGES * kStageBytes;
  static constexpr int kBarOff = kTileBytes;
  static constexpr int kTotal = kTileBytes + 256 + 1024;   // barriers + alignment slack
};

__host__ __device__ __forceinline__ int dt_size(int dt) { return dt == kDtF32 ? 4 : 2; }

// 32 consecutive values of one row, stored as fp32, bf16 or fp16 (16-byte vector stores).
__device__ __forceinline__ void store_row32(void* out, int dt, const float* v) {
  if (dt == kDtF32) {
    float4* o = reinterpret_cast<float4*>(out);
#pragma unroll
    for (int q = 0; q < 8; ++q) o[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  } else {
    uint4* o = reinterpret_cast<uint4*>(out);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        w[e] = dt == kDtBF16 ? pack_bf16x2(v[8 * q + 2 * e], v[8 * q + 2 * e + 1])
                             : pack_f16x2(v[8 * q + 2 * e], v[8 * q + 2 * e + 1]);
      o[q] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

__device__ __forceinline__ void load_row32(const void* in, int dt, float* v) {
  if (dt == kDtF32) {
    const float4* p = reinterpret_cast<const float4*>(in);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float4 t = p[q];
      v[4 * q] = t.x; v[4 * q + 1] = t.y; v[4 * q + 2] = t.z; v[4 * q + 3] = t.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(in);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 t = p[q];
      const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = dt == kDtBF16 ? unpack_bf16x2(w[e]) : unpack_f16x2(w[e]);
        v[8 * q + 2 * e] = f.x;
        v[8 * q + 2 * e + 1] = f.y;
      }
    }
  }
}

__device__ __forceinline__ void store_one(void* base, int dt, int64_t idx, float v) {
  if (dt == kDtF32) reinterpret_cast<float*>(base)[idx] = v;
  else if (dt == kDtBF16) reinterpret_cast<__nv_bfloat16*>(base)[idx] = __float2bfloat16_rn(v);
  else reinterpret_cast<__half*>(base)[idx] = __float2half_rn(v);
}

__device__ __forceinline__ float load_one(const void* base, int dt, int64_t idx) {
  if (dt == kDtF32) return reinterpret_cast<const float*>(base)[idx];
  if (dt == kDtBF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[idx]);
  return __half2float(reinterpret_cast<const __half*>(base)[idx]);
}

template <int BN, int STAGES, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    int M, int N, int num_kb, int kb_per_split, uint32_t idesc, GemmEpilogue epi, WaitCtl ctl) {
  using L = GemmSmem<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  // bars[0..STAGES): full, [STAGES..2*STAGES): empty, [2*STAGES]: accumulator ready
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN;
  const int m0 = blockIdx.y * kBM;
  const int kb_begin = blockIdx.z * kb_per_split;
  const int kb_end = min(num_kb, kb_begin + kb_per_split);
  const int nkb = max(0, kb_end - kb_begin);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * STAGES + 1; ++i) mbar_init(smem_u32(&bars[i]), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      for (int i = 0; i < nkb; ++i) {
        const int s = i % STAGES;
        if (i >= STAGES && !mbar_wait(smem_u32(&bars[STAGES + s]), ((i / STAGES) - 1) & 1, abort_flag, ctl)) break;
        const uint32_t full = smem_u32(&bars[s]);
        const uint32_t sa = smem_u32(smem + s * L::kStageBytes);
        const uint32_t sb = sa + L::kABytes;
        const int kx = (kb_begin + i) * kBK;
        mbar_arrive_expect_tx(full, L::kStageBytes);
        if (!A_MN) {
          tma_load_2d(sa, &tmA, full, kx, m0);
        } else {
          tma_load_2d(sa, &tmA, full, m0, kx);
          tma_load_2d(sa + 8192, &tmA, full, m0 + 64, kx);
        }
        if (!B_MN) {
          tma_load_2d(sb, &tmB, full, kx, n0);
        } else {
#pragma unroll
          for (int c = 0; c < BN / 64; ++c) tma_load_2d(sb + c * 8192, &tmB, full, n0 + 64 * c, kx);
        }
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(smem_u32(&bars[s]), (i / STAGES) & 1, abort_flag, ctl)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * L::kStageBytes);
        const uint32_t sb = sa + L::kABytes;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = A_MN ? make_sdesc_sw128(sa + kk * 2048, 8192, 1024)
                                   : make_sdesc_sw128(sa + kk * 32, 16, 1024);
          const uint64_t bd = B_MN ? make_sdesc_sw128(sb + kk * 2048, 8192, 1024)
                                   : make_sdesc_sw128(sb + kk * 32, 16, 1024);
          umma_f16_ss(tmem_acc, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(smem_u32(&bars[STAGES + s]));
      }
      if (ok) umma_commit(smem_u32(&bars[2 * STAGES]));
    }
  } else {
    // epilogue warps 0-3: thread owns output row m0 + 32*warp + lane
    bool have_acc = nkb > 0;
    if (have_acc) have_acc = mbar_wait(smem_u32(&bars[2 * STAGES]), 0, abort_flag, ctl);
    if (have_acc || nkb == 0) {
      tc_fence_after();
      const int row = m0 + warp * 32 + lane;
      const bool row_ok = row < M;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        if (nkb > 0) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem_acc + (static_cast<uint32_t>(warp * 32) << 16) + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.0f;
        }
        const int n = n0 + c * 32;
        if (!row_ok || n >= N) continue;
        if (epi.kind == kEpiAtomic) {
          float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(epi.out0) +
                                                static_cast<int64_t>(row) * epi.ld_out0 + n);
#pragma unroll
          for (int j = 0; j < 8; ++j) atomicAdd(o + j, make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
          continue;
        }
        if (epi.bias) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] += __ldg(epi.bias + n + j);
        }
        if (epi.kind == kEpiSilu) {
          if (epi.out1) {
            uint8_t* o1 = reinterpret_cast<uint8_t*>(epi.out1) +
                          (static_cast<int64_t>(row) * epi.ld_out1 + n) * dt_size(epi.out1_dt);
            store_row32(o1, epi.out1_dt, v);
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = silu_fast(v[j]);
        } else if (epi.resid) {
          float rv[32];
          const uint8_t* rp = reinterpret_cast<const uint8_t*>(epi.resid) +
                              (static_cast<int64_t>(row) * epi.ld_resid + n) * dt_size(epi.resid_dt);
          load_row32(rp, epi.resid_dt, rv);
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] += rv[j];
        }
        uint8_t* o0 = reinterpret_cast<uint8_t*>(epi.out0) +
                      (static_cast<int64_t>(row) * epi.ld_out0 + n) * dt_size(epi.out0_dt);
        store_row32(o0, epi.out0_dt, v);
        if (epi.kind == kEpiLinear && epi.out1) {
          uint8_t* o1 = reinterpret_cast<uint8_t*>(epi.out1) +
                        (static_cast<int64_t>(row) * epi.ld_out1 + n) * dt_size(epi.out1_dt);
          store_row32(o1, epi.out1_dt, v);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_acc, BN);
  }
}

// ----------------------------------------------------------------------------------------------
// fp32 CUDA-core GEMM (the exact fp32 mode; small shapes only)
// ----------------------------------------------------------------------------------------------

__global__ void __launch_bounds__(256)
gemm_f32_simt_kernel(const float* __restrict__ A, int64_t sam, int64_t sak, const float* __restrict__ B,
                     int64_t sbn, int64_t sbk, int M, int N, int K, GemmEpilogue epi) {
  __shared__ float As[16][64 + 1];
  __shared__ float Bs[16][64 + 1];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int e = threadIdx.x; e < 16 * 64; e += 256) {
      const int kk = e / 64, mm = e % 64;
      const int m = m0 + mm, k = k0 + kk;
      As[kk][mm] = (m < M && k < K) ? A[m * sam + k * sak] : 0.0f;
      const int n = n0 + mm;
      Bs[kk][mm] = (n < N && k < K) ? B[n * sbn + k * sbk] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j];
      if (epi.kind == kEpiAtomic) {
        atomicAdd(reinterpret_cast<float*>(epi.out0) + m * epi.ld_out0 + n, v);
        continue;
      }
      if (epi.bias) v += epi.bias[n];
      if (epi.kind == kEpiSilu) {
        if (epi.out1) store_one(epi.out1, epi.out1_dt, static_cast<int64_t>(m) * epi.ld_out1 + n, v);
        v = v / (1.0f + expf(-v));
      } else if (epi.resid) {
        v += load_one(epi.resid, epi.resid_dt, static_cast<int64_t>(m) * epi.ld_resid + n);
      }
      store_one(epi.out0, epi.out0_dt, static_cast<int64_t>(m) * epi.ld_out0 + n, v);
      if (epi.kind == kEpiLinear && epi.out1)
        store_one(epi.out1, epi.out1_dt, static_cast<int64_t>(m) * epi.ld_out1 + n, v);
    }
  }
}

template <int BN, int STAGES, bool A_MN, bool B_MN>
cudaError_t launch_tc(const GemmArgs& g, cudaStream_t st) {
  using L = GemmSmem<BN, STAGES>;
  CUtensorMap tmA, tmB;
  // A: K-major -> [M rows, K] box {64, 128}; MN-major -> [K rows, M] box {64, 64}
  if (!A_MN) {
    if (!encode_tmap_2d_bf16(&tmA, g.A, g.K, g.M, g.lda, 64, kBM, g.f16)) return cudaErrorInvalidValue;
  } else {
    if (!encode_tmap_2d_bf16(&tmA, g.A, g.M, g.K, g.lda, 64, 64, g.f16)) return cudaErrorInvalidValue;
  }
  if (!B_MN) {
    if (!encode_tmap_2d_bf16(&tmB, g.B, g.K, g.N, g.ldb, 64, BN, g.f16)) return cudaErrorInvalidValue;
  } else {
    if (!encode_tmap_2d_bf16(&tmB, g.B, g.N, g.K, g.ldb, 64, 64, g.f16)) return cudaErrorInvalidValue;
  }
  auto kern = gemm_bf16_tc_kernel<BN, STAGES, A_MN, B_MN>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), L::kTotal);
  if (e != cudaSuccess) return e;
  const int num_kb = static_cast<int>((g.K + kBK - 1) / kBK);
  const int splits = g.splits < 1 ? 1 : g.splits;
  const int kb_per = (num_kb + splits - 1) / splits;
  const int zdim = (num_kb + kb_per - 1) / kb_per;
  dim3 grid(static_cast<unsigned>((g.N + BN - 1) / BN), static_cast<unsigned>((g.M + kBM - 1) / kBM),
            static_cast<unsigned>(zdim < 1 ? 1 : zdim));
  const uint32_t idesc = make_idesc_f16kind(kBM, BN, A_MN ? 1 : 0, B_MN ? 1 : 0, g.f16);
  kern<<<grid, kThreads, L::kTotal, st>>>(tmA, tmB, static_cast<int>(g.M), static_cast<int>(g.N), num_kb,
                                          kb_per, idesc, g.epi, wait_ctl(g.status));
  return cudaGetLastError();
}

template <int BN, int STAGES>
cudaError_t dispatch_major(const GemmArgs& g, cudaStream_t st) {
  if (!g.a_mn && !g.b_mn) return launch_tc<BN, STAGES, false, false>(g, st);
  if (!g.a_mn && g.b_mn) return launch_tc<BN, STAGES, false, true>(g, st);
  if (g.a_mn && !g.b_mn) return launch_tc<BN, STAGES, true, false>(g, st);
  return launch_tc<BN, STAGES, true, true>(g, st);
}

}  // namespace

cudaError_t gemm_bf16(const GemmArgs& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  if (g.N % 256 == 0 && g.N >= 1024) return dispatch_major<256, 4>(g, st);
  return dispatch_major<128, 4>(g, st);
}

cudaError_t gemm_f32(const GemmArgs& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0) return cudaSuccess;
  // A(m, k): K-major -> A[m*lda + k]; MN-major -> A[k*lda + m]
  const int64_t sam = g.a_mn ? 1 : g.lda, sak = g.a_mn ? g.lda : 1;
  const int64_t sbn = g.b_mn ? 1 : g.ldb, sbk = g.b_mn ? g.ldb : 1;
  dim3 grid(static_cast<unsigned>((g.N + 63) / 64), static_cast<unsigned>((g.M + 63) / 64));
  gemm_f32_simt_kernel<<<grid, 256, 0, st>>>(static_cast<const float*>(g.A), sam, sak,
                                             static_cast<const float*>(g.B), sbn, sbk, static_cast<int>(g.M),
                                             static_cast<int>(g.N), static_cast<int>(g.K), g.epi);
  return cudaGetLastError();
}

}  // namespace hstu
