// gemm_sm100.cu - the layer's projection GEMMs on the 5th-generation tensor cores.
//
// C[M, N] = A[M, K] * B[N, K]^T with 16-bit operands (both bf16 or both fp16) and fp32 accumulation
// in tensor memory.
// Each operand is either K-major (row-major [rows, K]) or MN-major (row-major [K, rows]), so the
// forward projections (X W1^T, G W2^T) and the backward ones (dY W2, dZ W1, dY^T G, dZ^T X)
// share one kernel. Operand tiles arrive by TMA (128-byte swizzle) into a STAGES-deep ring; one
// thread issues tcgen05.mma (M=128, N=BN, K=16) into TMEM; four warps run the fused epilogue:
//   SILU:   Z = acc + b;  out0 = SiLU(Z) (the U|V|Q|K activations), out1 = Z (optional)
//   LINEAR: Y = acc (+ b) (+ R);  out0 = Y, out1 = a second copy of Y in out1's dtype (optional;
//           the fp16 copy a stacked layer's f1 reads)
//   ATOMIC: out0 += acc (fp32 reductions for split-K weight gradients)
// ("4.4 Scaling Recommendation Models", Generative Recommenders and HSTU: f1 with phi1 = SiLU
// and the split into U, V, Q, K; f2 followed by the residual of the "Code" sketch.)
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "hstu_internal.h"
#include "sm100_ptx.cuh"

namespace hstu {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kEpiWarps = 8;    // 2 per TMEM lane quadrant, each on half of the tile's columns
constexpr int kThreads = 32 * (kEpiWarps + 2);   // warps 0-7 epilogue, warp 8 TMA, warp 9 MMA
constexpr int kBoxBytes = 4096; // one epilogue staging box: 32 rows x 128 bytes

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr int kABytes = kBM * kBK * 2;      // 16 KB
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTileBytes = STAGES * kStageBytes;
  static constexpr int kOut = kTileBytes;            // 8 epilogue warps x 2 staging boxes
  static constexpr int kBarOff = kOut + kEpiWarps * 2 * kBoxBytes;
  static constexpr int kTotal = kBarOff + 256 + 1024;   // barriers + alignment slack
};

__host__ __device__ __forceinline__ int dt_size(int dt) { return dt == kDtF32 ? 4 : 2; }

struct GemmParams {
  int M, N, num_kb, kb_per, tiles_n, splits, total;
  uint32_t idesc;
  GemmEpilogue epi;
};

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

// Per-warp epilogue staging: boxes of 32 rows x 128 bytes in the 128-byte swizzled layout of the
// output tensor maps, written row-per-lane (16-byte units XOR-ed with the row: conflict-free) and
// sent by TMA (store or fp32 reduce-add), two boxes in flight per warp. Box slot i is sent by lane i
// (a thread keeps about one bulk copy in flight, so the two slots' copies overlap).
struct EpiStage {
  uint8_t* base;   // this warp's 2 boxes
  int slot;
  __device__ __forceinline__ void emit(const CUtensorMap* map, bool reduce, int x, int y, const uint32_t* w) {
    const int lane = threadIdx.x & 31;
    if (lane == slot) bulk_wait_group_read<0>();   // this slot's previous box has been read
    __syncwarp();
    uint8_t* box = base + slot * kBoxBytes;
    uint8_t* row = box + lane * 128;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      *reinterpret_cast<uint4*>(row + ((u ^ (lane & 7)) << 4)) = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == slot) {
      if (reduce) tma_reduce_add_2d(map, smem_u32(box), x, y);
      else tma_store_2d(map, smem_u32(box), x, y);
      bulk_commit_group();
    }
    slot ^= 1;
  }
};

// 64 values of one row -> the output's boxes: one 64-column box for 2-byte types, two 32-column
// boxes for fp32.
__device__ __forceinline__ void emit64(EpiStage& es, const CUtensorMap* map, int dt, bool reduce, int x, int y,
                                       const float* v, int xlim) {
  uint32_t w[32];
  if (dt == kDtF32) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (x + 32 * h >= xlim) break;   // (warp-uniform) a box wholly past the last column
#pragma unroll
      for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(v[32 * h + j]);
      es.emit(map, reduce, x + 32 * h, y, w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      w[j] = dt == kDtBF16 ? pack_bf16x2(v[2 * j], v[2 * j + 1]) : pack_f16x2(v[2 * j], v[2 * j + 1]);
    es.emit(map, false, x, y, w);
  }
}

// Persistent tensor-core GEMM: CTAs stride over (m tile, n tile, k split) work items; the
// accumulator is double-buffered in TMEM so the epilogue of one tile overlaps the next tile's
// mainloop.
template <int BN, int STAGES, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmO0, const __grid_constant__ CUtensorMap tmO1,
                    GemmParams P, WaitCtl ctl) {
  pdl_enter();
  using L = GemmSmem<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  // [0, STAGES) full | [STAGES, 2 STAGES) empty | 2 STAGES + b: accumulator b full | + 2: empty
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto acc_full = [&](int b) { return smem_u32(&bars[2 * STAGES + b]); };
  auto acc_empty = [&](int b) { return smem_u32(&bars[2 * STAGES + 2 + b]); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * STAGES; ++i) mbar_init(smem_u32(&bars[i]), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full(b), 1);
      mbar_init(acc_empty(b), 32 * kEpiWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kEpiWarps && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_slot;

  auto decode = [&](int t, int& m0, int& n0, int& kb0, int& kb1) {
    const int ks = t % P.splits;
    const int rest = t / P.splits;
    n0 = (rest % P.tiles_n) * BN;
    m0 = (rest / P.tiles_n) * kBM;
    kb0 = ks * P.kb_per;
    kb1 = min(P.num_kb, kb0 + P.kb_per);
  };

  if (warp == kEpiWarps) {
    // TMA producer. A thread keeps about one tile load in flight (measured: one 16 KB box per
    // ~550 cycles per issuing thread, 3x that from 4 lanes), so the boxes of a stage are issued by
    // different lanes: box i of stage s by lane s * boxes + i (A: 1 K-major box or 2 MN-major halves;
    // B: 1 K-major box or BN / 64 MN-major boxes). Lane 0 waits for the stage and registers the
    // bytes first.
    constexpr int kABoxes = A_MN ? 2 : 1;
    constexpr int kBoxes = kABoxes + (B_MN ? BN / 64 : 1);
    static_assert(kBoxes * STAGES <= 32, "one lane per box of every stage");
    int g = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < P.total; t += gridDim.x) {
      int m0, n0, kb0, kb1;
      decode(t, m0, n0, kb0, kb1);
      for (int kb = kb0; kb < kb1; ++kb, ++g) {
        const int s = g % STAGES;
        bool free_ok = true;   // lane 0 waits; the result is made warp-uniform
        if (lane == 0 && g >= STAGES)
          free_ok = mbar_wait(smem_u32(&bars[STAGES + s]), ((g / STAGES) - 1) & 1, abort_flag, ctl);
        if (!__shfl_sync(0xffffffffu, free_ok ? 1 : 0, 0)) {
          ok = false;
          break;
        }
        const uint32_t full = smem_u32(&bars[s]);
        const uint32_t sa = smem_u32(smem + s * L::kStageBytes);
        const uint32_t sb = sa + L::kABytes;
        const int kx = kb * kBK;
        if (lane == 0) mbar_arrive_expect_tx(full, L::kStageBytes);
        __syncwarp();
        // stage s's boxes come from lanes [s * kBoxes, (s + 1) * kBoxes): consecutive stages are in
        // flight from different threads
        const int bx = lane - s * kBoxes;
        if (bx >= 0 && bx < kABoxes) {
          if (!A_MN) tma_load_2d(sa, &tmA, full, kx, m0);
          else tma_load_2d(sa + bx * 8192, &tmA, full, m0 + 64 * bx, kx);
        } else if (bx >= kABoxes && bx < kBoxes) {
          const int c = bx - kABoxes;
          if (!B_MN) tma_load_2d(sb, &tmB, full, kx, n0);
          else tma_load_2d(sb + c * 8192, &tmB, full, n0 + 64 * c, kx);
        }
      }
    }
  } else if (warp == kEpiWarps + 1) {
    if (lane == 0) {
      // descriptors of stage 0's A and B tiles; stages and K steps are offsets from them
      const uint32_t sa0 = smem_u32(smem), sb0 = sa0 + L::kABytes;
      const uint64_t a_desc0 = A_MN ? make_sdesc_sw128(sa0, 8192, 1024) : make_sdesc_sw128(sa0, 16, 1024);
      const uint64_t b_desc0 = B_MN ? make_sdesc_sw128(sb0, 8192, 1024) : make_sdesc_sw128(sb0, 16, 1024);
      int g = 0, it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < P.total; t += gridDim.x, ++it) {
        int m0, n0, kb0, kb1;
        decode(t, m0, n0, kb0, kb1);
        const int buf = it & 1;
        if (it >= 2 && !mbar_wait(acc_empty(buf), ((it >> 1) - 1) & 1, abort_flag, ctl)) { ok = false; break; }
        tc_fence_after();
        const uint32_t acc = tmem_acc + buf * BN;
        for (int kb = kb0; kb < kb1; ++kb, ++g) {
          const int s = g % STAGES;
          if (!mbar_wait(smem_u32(&bars[s]), (g / STAGES) & 1, abort_flag, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad0 = sdesc_add(a_desc0, s * L::kStageBytes);
          const uint64_t bd0 = sdesc_add(b_desc0, s * L::kStageBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_f16_ss(acc, sdesc_add(ad0, A_MN ? kk * 2048 : kk * 32), sdesc_add(bd0, B_MN ? kk * 2048 : kk * 32),
                        P.idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          umma_commit(smem_u32(&bars[STAGES + s]));
        }
        if (ok) umma_commit(acc_full(buf));
      }
    }
  } else {
    // epilogue warps 0-7: TMEM lanes 32 (warp % 4) .. +31 = output rows m0 + 32 (warp % 4) + lane,
    // columns [BN/2 (warp / 4), +BN/2)
    const GemmEpilogue& epi = P.epi;
    const int quad = warp & 3, chalf = warp >> 2;
    EpiStage es{smem + L::kOut + warp * 2 * kBoxBytes, 0};
    int it = 0;
    for (int t = blockIdx.x; t < P.total; t += gridDim.x, ++it) {
      int m0, n0, kb0, kb1;
      decode(t, m0, n0, kb0, kb1);
      const int buf = it & 1;
      if (!mbar_wait(acc_full(buf), (it >> 1) & 1, abort_flag, ctl)) break;
      tc_fence_after();
      const int row = m0 + quad * 32 + lane;
      const bool row_ok = row < P.M;
      const int ybox = m0 + quad * 32;
      constexpr int kChunks = BN / 128;   // 64-column chunks per warp
#pragma unroll 1
      for (int c = 0; c < kChunks; ++c) {
        const int col = chalf * (BN / 2) + c * 64;   // within the tile
        const int n = n0 + col;
        float v[64];
        {
          uint32_t r[32];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            tmem_ld_32x32b_x32(tmem_acc + buf * BN + (static_cast<uint32_t>(quad * 32) << 16) + col + 32 * h, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[32 * h + j] = __uint_as_float(r[j]);
          }
        }
        if (c == kChunks - 1) {   // this warp's part of the accumulator is in registers: release it
          tc_fence_before();
          mbar_arrive(acc_empty(buf));
        }
        if (n >= P.N) continue;
        if (epi.kind == kEpiAtomic) {
          emit64(es, &tmO0, kDtF32, true, n, ybox, v, P.N);
          continue;
        }
        if (epi.bias) {
          const float4* bp = reinterpret_cast<const float4*>(epi.bias + n);
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float4 b4 = (n + 4 * q < P.N) ? __ldg(bp + q) : make_float4(0.f, 0.f, 0.f, 0.f);
            v[4 * q] += b4.x; v[4 * q + 1] += b4.y; v[4 * q + 2] += b4.z; v[4 * q + 3] += b4.w;
          }
        }
        if (epi.kind == kEpiSilu) {
          // Z and SiLU(Z) stored in fp16: a pre-activation outside the fp16 range (or NaN) is reported
          // (HSTU_ERR_DEVICE) instead of becoming inf silently
          if (row_ok && (epi.out0_dt == kDtF16 || epi.out1_dt == kDtF16)) {
            bool in_range = true;
#pragma unroll
            for (int j = 0; j < 64; ++j) in_range &= fabsf(v[j]) <= 65504.0f;
            if (!in_range) report_error(ctl.status, kDevBadInput);
          }
          if (epi.out1) emit64(es, &tmO1, epi.out1_dt, false, n, ybox, v, P.N);
#pragma unroll
          for (int j = 0; j < 64; ++j) v[j] = silu_tanh(v[j]);
        } else if (epi.resid) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float rv[32];
            if (row_ok && n + 32 * h < P.N) {
              const uint8_t* rp = reinterpret_cast<const uint8_t*>(epi.resid) +
                                  (static_cast<int64_t>(row) * epi.ld_resid + n + 32 * h) * dt_size(epi.resid_dt);
              load_row32(rp, epi.resid_dt, rv);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) rv[j] = 0.0f;
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) v[32 * h + j] += rv[j];
          }
        }
        emit64(es, &tmO0, epi.out0_dt, false, n, ybox, v, P.N);
        if (epi.kind == kEpiLinear && epi.out1) emit64(es, &tmO1, epi.out1_dt, false, n, ybox, v, P.N);
      }
    }
    if (lane < 2) bulk_wait_group_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_acc, 2 * BN);
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
  CUtensorMap tmA, tmB, tmO0, tmO1;
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
  // outputs: boxes of 32 rows x 128 bytes
  const int dt0 = g.epi.kind == kEpiAtomic ? kDtF32 : g.epi.out0_dt;
  if (!encode_tmap_2d_out(&tmO0, g.epi.out0, dt0, g.N, g.M, g.epi.ld_out0, 128 / dt_size(dt0), 32))
    return cudaErrorInvalidValue;
  if (g.epi.out1) {
    if (!encode_tmap_2d_out(&tmO1, g.epi.out1, g.epi.out1_dt, g.N, g.M, g.epi.ld_out1, 128 / dt_size(g.epi.out1_dt), 32))
      return cudaErrorInvalidValue;
  } else {
    tmO1 = tmO0;
  }
  auto kern = gemm_bf16_tc_kernel<BN, STAGES, A_MN, B_MN>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), L::kTotal);
  if (e != cudaSuccess) return e;
  GemmParams P{};
  P.M = static_cast<int>(g.M);
  P.N = static_cast<int>(g.N);
  P.num_kb = static_cast<int>((g.K + kBK - 1) / kBK);
  const int splits = g.splits < 1 ? 1 : g.splits;
  P.kb_per = (P.num_kb + splits - 1) / splits;
  P.splits = (P.num_kb + P.kb_per - 1) / P.kb_per;
  P.tiles_n = static_cast<int>((g.N + BN - 1) / BN);
  const int tiles_m = static_cast<int>((g.M + kBM - 1) / kBM);
  P.total = tiles_m * P.tiles_n * P.splits;
  P.idesc = make_idesc_f16kind(kBM, BN, A_MN ? 1 : 0, B_MN ? 1 : 0, g.f16);
  P.epi = g.epi;
  const int grid = P.total < sm_count() ? P.total : sm_count();
  return launch_pdl(kern, dim3(grid), dim3(kThreads), L::kTotal, st, tmA, tmB, tmO0, tmO1, P, wait_ctl(g.status));
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
  if (g.K <= 0) return cudaErrorInvalidValue;
  if (g.N % 256 == 0 && g.N >= 1024) return dispatch_major<256, 3>(g, st);
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
