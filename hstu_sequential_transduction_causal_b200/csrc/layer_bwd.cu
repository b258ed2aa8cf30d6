// layer_bwd.cu - elementwise and reduction kernels of the layer backward (the GEMMs and the
// attention backward live in their own files).
//
// Derived from the layer forward of "4.4 Scaling Recommendation Models", Generative Recommenders
// and HSTU (Y = f2(LN(O) (.) U) + X with U, V, Q, K = Split(SiLU(f1(X)))):
//   norm-gate backward: with xhat = (O - mu) rstd, Ln = gamma xhat + beta,
//     dLn = dG (.) U,  dU = dG (.) Ln,  dxhat = dLn (.) gamma,
//     dO = rstd (dxhat - mean(dxhat) - xhat mean(dxhat xhat)),
//     dgamma = sum_t dLn (.) xhat,  dbeta = sum_t dLn;
//   SiLU backward: dZ = dS (.) SiLU'(Z), SiLU'(z) = s(z)(1 + z(1 - s(z))), s = logistic;
//   column sums for the bias gradients.
#include <algorithm>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hstu_internal.h"
#include "sm100_ptx.cuh"
#include "vec_io.cuh"

namespace hstu {

namespace {

// One warp per token row (grid-stride over rows); lane l holds features 128 k + 4 l + i (k < VPT / 4,
// i < 4): every load and store of the warp covers 128 consecutive features (coalesced). gamma and
// beta are staged in shared memory (registers for two blocks per SM).
// Writes dO (act dtype), dZ_U = dU (.) SiLU'(Z_U) (fp16, row stride ld_dz) and per-block partial
// sums of dgamma | dbeta into partial[blockIdx.x][0 .. 2D).
template <int VPT, int AT>
__global__ void __launch_bounds__(256, 2)
norm_gate_bwd_kernel(int64_t T, const float* __restrict__ dg, const float* __restrict__ o, const void* __restrict__ u,
                     const void* __restrict__ zu, int64_t ld_act, const float* __restrict__ gamma,
                     const float* __restrict__ beta, const float* __restrict__ mu, const float* __restrict__ rstd,
                     void* __restrict__ d_o, void* __restrict__ dz, int64_t ld_dz, float* __restrict__ partial) {
  constexpr int D = VPT * 32;
  constexpr int KG = VPT / 4;   // groups of 4 features per lane
  __shared__ __align__(16) float s_gb[2 * D];
  __shared__ float s_red[8][2][D];
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    s_gb[c] = gamma[c];
    s_gb[D + c] = beta[c];
  }
  pdl_enter();
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float gacc[VPT], bacc[VPT];
#pragma unroll
  for (int e = 0; e < VPT; ++e) gacc[e] = bacc[e] = 0.0f;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + warp; row < T; row += static_cast<int64_t>(gridDim.x) * 8) {
    float g[VPT], x[VPT], uu[VPT], z[VPT];
#pragma unroll
    for (int k = 0; k < KG; ++k) {
      const int c = 128 * k + 4 * lane;
      load_vec<4, kDtF32>(dg, row * D + c, g + 4 * k);
      load_vec<4, kDtF32>(o, row * D + c, x + 4 * k);
      load_vec<4, AT>(u, row * ld_act + c, uu + 4 * k);
      load_vec<4, AT>(zu, row * ld_act + c, z + 4 * k);
    }
    const float m = mu[row], rs = rstd[row];
    float s1 = 0.0f, s2 = 0.0f;
#pragma unroll
    for (int k = 0; k < KG; ++k) {
      const int c = 128 * k + 4 * lane;
      float gm[4], bt[4];
      load_vec<4, kDtF32>(s_gb, c, gm);
      load_vec<4, kDtF32>(s_gb + D, c, bt);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = 4 * k + i;
        const float xh = (x[e] - m) * rs;
        const float dln = g[e] * uu[e];
        const float dxh = dln * gm[i];
        gacc[e] = fmaf(dln, xh, gacc[e]);
        bacc[e] += dln;
        s1 += dxh;
        s2 = fmaf(dxh, xh, s2);
        const float du = g[e] * fmaf(gm[i], xh, bt[i]);
        z[e] = du * silu_grad(z[e]);        // dZ_U
        x[e] = xh;                          // keep xhat
        g[e] = dxh;                         // keep dxhat
      }
      store_vec<4, kDtF16>(dz, row * ld_dz + c, z + 4 * k);
    }
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) {
      s1 += __shfl_xor_sync(0xffffffffu, s1, k);
      s2 += __shfl_xor_sync(0xffffffffu, s2, k);
    }
    const float m1 = s1 * (1.0f / D), m2 = s2 * (1.0f / D);
#pragma unroll
    for (int e = 0; e < VPT; ++e) g[e] = rs * (g[e] - m1 - x[e] * m2);
#pragma unroll
    for (int k = 0; k < KG; ++k) store_vec<4, AT>(d_o, row * D + 128 * k + 4 * lane, g + 4 * k);
  }
#pragma unroll
  for (int e = 0; e < VPT; ++e) {
    const int f = 128 * (e >> 2) + 4 * lane + (e & 3);
    s_red[warp][0][f] = gacc[e];
    s_red[warp][1][f] = bacc[e];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < 2 * D; c += 256) {
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += s_red[w][c / D][c % D];
    partial[static_cast<int64_t>(blockIdx.x) * 2 * D + c] = s;
  }
}

// Row slots per warp of the staged backward below.
constexpr int kNgbSlots = 2;

// Threads of the fused conversion + column-sum kernel (rows_to_f16_colsum_kernel).
constexpr int kTailThreads = 256;

// The same backward with the rows staged by bulk copies (dG, O as fp32, then U and Z_U of the act
// type): a persistent grid whose warps each own kNgbSlots row slots in shared memory and rows gw,
// gw + W, ... (gw = the warp's global index, W = all warps); lane 0 refills a slot as soon as the
// warp has read it. xhat and dxhat are recomputed from the slot after the row reductions instead of
// being held in registers. The slot memory holds the block's dgamma | dbeta sums at the end.
template <int VPT, int AT>
__global__ void __launch_bounds__(256, 2)
norm_gate_bwd_staged_kernel(int64_t T, const float* __restrict__ dg, const float* __restrict__ o,
                            const void* __restrict__ u, const void* __restrict__ zu, int64_t ld_act,
                            const float* __restrict__ gamma, const float* __restrict__ beta,
                            const float* __restrict__ mu, const float* __restrict__ rstd, void* __restrict__ d_o,
                            void* __restrict__ dz, int64_t ld_dz, float* __restrict__ partial, WaitCtl ctl) {
  constexpr int D = VPT * 32, KG = VPT / 4;
  constexpr int GB = D * 4, OB = D * 4, AB = D * 2, SLOT = GB + OB + 2 * AB, S = kNgbSlots;
  static_assert(VPT % 4 == 0, "groups of four features per lane");
  static_assert(8 * S * SLOT >= 8 * 2 * D * 4, "the slots hold the block's partial sums at the end");
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t s_bar[8 * S];
  __shared__ int s_abort;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 8 * S; ++i) mbar_init(smem_u32(&s_bar[i]), 1);
    s_abort = 0;
    fence_barrier_init();
  }
  float gm[VPT], bt[VPT];
#pragma unroll
  for (int k = 0; k < KG; ++k) {
    load_vec<4, kDtF32>(gamma, 128 * k + 4 * lane, gm + 4 * k);
    load_vec<4, kDtF32>(beta, 128 * k + 4 * lane, bt + 4 * k);
  }
  pdl_enter();
  __syncthreads();
  const long long W = static_cast<long long>(gridDim.x) * 8, gw = static_cast<long long>(blockIdx.x) * 8 + warp;
  uint8_t* wslots = smem + static_cast<size_t>(warp) * S * SLOT;
  auto issue = [&](long long i) {   // lane 0: row i of this warp into slot i % S
    const long long row = gw + i * W;
    if (row >= T) return;
    const int sl = static_cast<int>(i % S);
    const uint32_t bar = smem_u32(&s_bar[warp * S + sl]);
    const uint32_t dst = smem_u32(wslots + sl * SLOT);
    mbar_arrive_expect_tx(bar, SLOT);
    bulk_load(dst, dg + row * D, GB, bar);
    bulk_load(dst + GB, o + row * D, OB, bar);
    bulk_load(dst + GB + OB, static_cast<const uint16_t*>(u) + row * ld_act, AB, bar);
    bulk_load(dst + GB + OB + AB, static_cast<const uint16_t*>(zu) + row * ld_act, AB, bar);
  };
  if (lane == 0)
    for (int i = 0; i < S; ++i) issue(i);
  float gacc[VPT], bacc[VPT];
#pragma unroll
  for (int e = 0; e < VPT; ++e) gacc[e] = bacc[e] = 0.0f;
  for (long long i = 0;; ++i) {
    const long long row = gw + i * W;
    if (row >= T) break;
    const int sl = static_cast<int>(i % S);
    if (!mbar_wait_warp(smem_u32(&s_bar[warp * S + sl]), static_cast<uint32_t>((i / S) & 1), &s_abort, ctl)) break;
    const uint8_t* sg = wslots + sl * SLOT;
    const uint8_t *so = sg + GB, *su = so + OB, *sz = su + AB;
    const float m = mu[row], rs = rstd[row];
    float s1 = 0.0f, s2 = 0.0f;
#pragma unroll
    for (int k = 0; k < KG; ++k) {
      const int c = 128 * k + 4 * lane;
      float g4[4], x4[4], u4[4], z4[4];
      load_vec<4, kDtF32>(sg, c, g4);
      load_vec<4, kDtF32>(so, c, x4);
      load_vec<4, AT>(su, c, u4);
      load_vec<4, AT>(sz, c, z4);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int e = 4 * k + q;
        const float xh = (x4[q] - m) * rs;
        const float dln = g4[q] * u4[q];
        const float dxh = dln * gm[e];
        gacc[e] = fmaf(dln, xh, gacc[e]);
        bacc[e] += dln;
        s1 += dxh;
        s2 = fmaf(dxh, xh, s2);
        z4[q] = g4[q] * fmaf(gm[e], xh, bt[e]) * silu_grad(z4[q]);   // dZ_U
      }
      store_vec<4, kDtF16>(dz, row * ld_dz + c, z4);
    }
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) {
      s1 += __shfl_xor_sync(0xffffffffu, s1, k);
      s2 += __shfl_xor_sync(0xffffffffu, s2, k);
    }
    const float m1 = s1 * (1.0f / D), m2 = s2 * (1.0f / D);
#pragma unroll
    for (int k = 0; k < KG; ++k) {
      const int c = 128 * k + 4 * lane;
      float g4[4], x4[4], u4[4];
      load_vec<4, kDtF32>(sg, c, g4);
      load_vec<4, kDtF32>(so, c, x4);
      load_vec<4, AT>(su, c, u4);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float xh = (x4[q] - m) * rs;
        const float dxh = g4[q] * u4[q] * gm[4 * k + q];
        g4[q] = rs * (dxh - m1 - xh * m2);
      }
      store_vec<4, AT>(d_o, row * D + c, g4);
    }
    // every lane has read the slot: refill it (generic reads before the copy engine's writes)
    __syncwarp();
    if (lane == 0) {
      fence_proxy_async_smem();
      issue(i + S);
    }
  }
  // the block's partial sums, through the slot memory once every copy has landed and been read (a
  // failed wait set s_abort, so every thread of the block takes the same branch)
  __syncthreads();
  if (s_abort) return;
  float* s_red = reinterpret_cast<float*>(smem);   // [8][2][D]
#pragma unroll
  for (int e = 0; e < VPT; ++e) {
    const int f = 128 * (e >> 2) + 4 * lane + (e & 3);
    s_red[(warp * 2 + 0) * D + f] = gacc[e];
    s_red[(warp * 2 + 1) * D + f] = bacc[e];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < 2 * D; c += 256) {
    float t = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += s_red[(w * 2 + c / D) * D + c % D];
    partial[static_cast<int64_t>(blockIdx.x) * 2 * D + c] = t;
  }
}

// Block blk of a batch of column-sum finishes (job j sums parts rows, row stride ld, of its partial
// buffer into out[0 .. cols)): 32 columns of one job, each summed over its partial rows by the 8
// warps (rows p = warp mod 8) and then across warps through s_part.
__device__ __forceinline__ void colsum_finish_block(const ColsumJobs& jobs, int blk, float (*s_part)[33]) {
  int j = 0;
  while (j + 1 < jobs.njobs && blk >= jobs.first_block[j + 1]) ++j;
  const ColsumJob& jb = jobs.job[j];
  const int cl = threadIdx.x & 31, slice = threadIdx.x >> 5;
  const int c = (blk - jobs.first_block[j]) * 32 + cl;
  float s0 = 0.0f, s1 = 0.0f;
  if (c < jb.cols) {
    int p = slice;
    for (; p + 8 < jb.parts; p += 16) {
      s0 += jb.partial[static_cast<int64_t>(p) * jb.ld + c];
      s1 += jb.partial[static_cast<int64_t>(p + 8) * jb.ld + c];
    }
    if (p < jb.parts) s0 += jb.partial[static_cast<int64_t>(p) * jb.ld + c];
  }
  s_part[slice][cl] = s0 + s1;
  __syncthreads();
  if (slice == 0 && c < jb.cols) {
    float t = 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) t += s_part[k][cl];
    jb.out[c] = t;
  }
}

// dZ[:, D:4D] = [dV | dQ | dK] (.) SiLU'(Z[:, D:4D]) in fp16 (g* are fp32 [T, D]), together with the
// column sums of all of dZ (the db1 of f1's bias). After the first fin_blocks blocks (column-sum
// finishes of earlier launches), a block covers 32 rows x 64 columns of dZ: warp w takes rows
// 4w .. 4w+3, lane l row 4w + l / 8 and columns 8 (l % 8) .. +7, so each row's 64 columns are one
// coalesced access. Columns [0, D) (dZ_U, written by the LayerNorm backward) are only read back for
// their sums, and so are dZ_V and dZ_K when dv and dk are null (the attention backward wrote them).
// The block's 32 rows are summed by shuffles (the 4 rows of a warp) and shared memory (the 8 warps)
// into partial[row block][cols] and / or by fp32 atomics into db1; the sums are of the fp16 values
// stored. Block b covers column block b % (4D / 64) of row block b / (4D / 64).
template <int AT>
__global__ void __launch_bounds__(256)
dz_assemble_kernel(int64_t T, int D, const float* __restrict__ dv, const float* __restrict__ dq,
                   const float* __restrict__ dk, const void* __restrict__ z, int64_t ld_z, void* __restrict__ dz,
                   int64_t ld_dz, float* __restrict__ partial, float* __restrict__ db1, ColsumJobs fin,
                   int fin_blocks) {
  __shared__ float s_red[8][64];
  __shared__ float s_fin[8][33];
  pdl_enter();
  if (static_cast<int>(blockIdx.x) < fin_blocks) {   // (block-uniform) a finish of an earlier launch's sums
    colsum_finish_block(fin, static_cast<int>(blockIdx.x), s_fin);
    return;
  }
  const int blk = static_cast<int>(blockIdx.x) - fin_blocks;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ncb = 4 * D / 64;
  const int cb = blk % ncb;
  const int64_t rb = blk / ncb;
  const int c = 64 * cb + 8 * (lane & 7);   // column of dZ, in [0, 4D)
  const int64_t row = 32 * rb + 4 * warp + (lane >> 3);
  float v[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = 0.0f;
  if (row < T) {
    const int blk = c < D ? -1 : (c - D) / D;
    const float* g = blk == 0 ? dv : (blk == 1 ? dq : (blk == 2 ? dk : nullptr));
    if (!g) {   // written by an earlier kernel (dZ_U; dZ_V and dZ_K when dv, dk are null): its sums only
      load_vec<8, kDtF16>(dz, row * ld_dz + c, v);
    } else {
      const int cc = (c - D) - blk * D;
      float zv[8];
      load_vec<8, kDtF32>(g, row * D + cc, v);
      load_vec<8, AT>(z, row * ld_z + c, zv);
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = __half2float(__float2half_rn(v[e] * silu_grad(zv[e])));
      store_vec<8, kDtF16>(dz, row * ld_dz + c, v);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    v[e] += __shfl_xor_sync(0xffffffffu, v[e], 8);
    v[e] += __shfl_xor_sync(0xffffffffu, v[e], 16);
  }
  if (lane < 8)
#pragma unroll
    for (int e = 0; e < 8; ++e) s_red[warp][8 * lane + e] = v[e];
  __syncthreads();
  if (threadIdx.x < 64) {
    float t = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += s_red[w][threadIdx.x];
    if (partial) partial[rb * 4 * D + 64 * cb + threadIdx.x] = t;
    if (db1) atomicAdd(db1 + 64 * cb + threadIdx.x, t);
  }
}

struct ConvertBatch {
  ConvertJob job[kMaxConvertJobs];
  int first_block[kMaxConvertJobs + 1];   // block b runs job j with first_block[j] <= b < first_block[j + 1]
  int njobs;
};

// Block blk of a batch of conversions to fp16 (and zero fills): it finds its job, then 8 elements
// per thread.
__device__ __forceinline__ void convert_block(const ConvertBatch& cb, int blk) {
  int j = 0;
  while (j + 1 < cb.njobs && blk >= cb.first_block[j + 1]) ++j;
  const ConvertJob& jb = cb.job[j];
  const int64_t i = (static_cast<int64_t>(blk - cb.first_block[j]) * blockDim.x + threadIdx.x) * 8;
  if (i >= jb.n) return;
  const int cnt = jb.n - i >= 8 ? 8 : static_cast<int>(jb.n - i);
  if (!jb.in) {   // zero fill: 32-byte stores where out is 16-byte aligned, else word by word
    float* o = static_cast<float*>(jb.out) + i;
    if (cnt == 8 && (reinterpret_cast<uintptr_t>(jb.out) & 15) == 0) {
      reinterpret_cast<float4*>(o)[0] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      reinterpret_cast<float4*>(o)[1] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    } else {
      for (int k = 0; k < cnt; ++k) o[k] = 0.0f;
    }
    return;
  }
  float v[8];
  if (cnt == 8) {
    if (jb.in_dt == kDtF32) load_vec<8, kDtF32>(jb.in, i, v);
    else if (jb.in_dt == kDtBF16) load_vec<8, kDtBF16>(jb.in, i, v);
    else load_vec<8, kDtF16>(jb.in, i, v);
    store_vec<8, kDtF16>(jb.out, i, v);
  } else {
    for (int k = 0; k < cnt; ++k) {
      if (jb.in_dt == kDtF32) load_vec<1, kDtF32>(jb.in, i + k, &v[0]);
      else if (jb.in_dt == kDtBF16) load_vec<1, kDtBF16>(jb.in, i + k, &v[0]);
      else load_vec<1, kDtF16>(jb.in, i + k, &v[0]);
      reinterpret_cast<__half*>(jb.out)[i + k] = __float2half_rn(v[0]);
    }
  }
}

// The backward's first launch, two independent jobs over one grid:
// - blocks [0, col_blocks): dY converted to fp16 (out, may be null when the caller holds an fp16
//   copy) and the partial column sums of dY (the db2 of f2's bias): block b sums rows [b R, (b+1) R)
//   into partial[b][0 .. D); its threads own 8 columns each (D / 8 per row, 256 / (D / 8) rows side
//   by side) and keep four rows' loads in flight each;
// - the rest: the fp16 copies of the other GEMM operands and zero fills of the outputs later
//   launches accumulate into (cb).
template <int D, int IT>
__global__ void __launch_bounds__(kTailThreads)
rows_to_f16_colsum_kernel(int64_t T, const void* __restrict__ in, void* __restrict__ out, int64_t rows_per,
                          float* __restrict__ partial, int col_blocks, ConvertBatch cb) {
  constexpr int TPR = D / 8, RP = kTailThreads / TPR, U = 4;
  static_assert(RP >= 1 && kTailThreads % TPR == 0, "whole rows per block");
  __shared__ float s_red[RP > 1 ? RP - 1 : 1][D];
  pdl_enter();
  if (static_cast<int>(blockIdx.x) >= col_blocks) {   // (block-uniform)
    convert_block(cb, static_cast<int>(blockIdx.x) - col_blocks);
    return;
  }
  const int g = threadIdx.x % TPR, rp = threadIdx.x / TPR;
  const int c = 8 * g;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * rows_per;
  const int64_t r1 = r0 + rows_per < T ? r0 + rows_per : T;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
  for (int64_t row = r0 + rp; row < r1; row += U * RP) {
    float v[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t r = row + static_cast<int64_t>(u) * RP;
      if (r < r1) load_vec<8, IT>(in, r * D + c, v[u]);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t r = row + static_cast<int64_t>(u) * RP;
      if (r >= r1) continue;
      if (out) store_vec<8, kDtF16>(out, r * D + c, v[u]);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += v[u][e];
    }
  }
  if constexpr (RP > 1) {
    if (rp > 0)
#pragma unroll
      for (int e = 0; e < 8; ++e) s_red[rp - 1][c + e] = acc[e];
    __syncthreads();
    if (rp == 0)
      for (int q = 1; q < RP; ++q)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += s_red[q - 1][c + e];
  }
  if (rp == 0)
#pragma unroll
    for (int e = 0; e < 8; ++e) partial[static_cast<int64_t>(blockIdx.x) * D + c + e] = acc[e];
}

// partial[y][c] = sum over rows [y R, (y+1) R) of in[row][c]; one thread per column.
template <int DT>
__global__ void __launch_bounds__(256)
colsum_partial_kernel(const void* __restrict__ in, int64_t rows, int cols, int64_t ld, int64_t rows_per,
                      float* __restrict__ partial) {
  pdl_enter();
  const int c = blockIdx.x * 256 + threadIdx.x;
  if (c >= cols) return;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per;
  const int64_t r1 = r0 + rows_per < rows ? r0 + rows_per : rows;
  // four independent accumulators: four loads in flight per thread
  float s[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  int64_t r = r0;
  for (; r + 4 <= r1; r += 4) {
    float v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) load_vec<1, DT>(in, (r + q) * ld + c, &v[q]);
#pragma unroll
    for (int q = 0; q < 4; ++q) s[q] += v[q];
  }
  for (; r < r1; ++r) {
    float v;
    load_vec<1, DT>(in, r * ld + c, &v);
    s[0] += v;
  }
  partial[static_cast<int64_t>(blockIdx.y) * cols + c] = (s[0] + s[1]) + (s[2] + s[3]);
}

// out[i] = in[i] converted between fp32 / bf16 / fp16, 8 elements per thread (scalar tail).
template <int IT, int OT>
__global__ void __launch_bounds__(256)
convert_kernel(const void* __restrict__ in, void* __restrict__ out, int64_t n) {
  pdl_enter();
  const int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  if (i + 8 <= n) {
    float v[8];
    load_vec<8, IT>(in, i, v);
    store_vec<8, OT>(out, i, v);
  } else {
    for (int64_t k = i; k < n; ++k) {
      float v;
      load_vec<1, IT>(in, k, &v);
      if constexpr (OT == kDtF32) reinterpret_cast<float*>(out)[k] = v;
      else if constexpr (OT == kDtBF16) reinterpret_cast<__nv_bfloat16*>(out)[k] = __float2bfloat16_rn(v);
      else reinterpret_cast<__half*>(out)[k] = __float2half_rn(v);
    }
  }
}

// Sums `parts` partial rows: block of 256 threads = 32 columns x 8 interleaved slices of the rows,
// then a shared-memory sum of the slices (the loads are independent and coalesced per warp).
__global__ void __launch_bounds__(256)
colsum_final_kernel(const float* __restrict__ partial, int parts, int cols, float* __restrict__ out) {
  pdl_enter();
  __shared__ float s_part[8][33];
  const int cl = threadIdx.x & 31, slice = threadIdx.x >> 5;
  const int c = blockIdx.x * 32 + cl;
  float s0 = 0.0f, s1 = 0.0f;
  if (c < cols) {
    int p = slice;
    for (; p + 8 < parts; p += 16) {
      s0 += partial[static_cast<int64_t>(p) * cols + c];
      s1 += partial[static_cast<int64_t>(p + 8) * cols + c];
    }
    if (p < parts) s0 += partial[static_cast<int64_t>(p) * cols + c];
  }
  s_part[slice][cl] = s0 + s1;
  __syncthreads();
  if (slice == 0 && c < cols) {
    float t = 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) t += s_part[k][cl];
    out[c] = t;
  }
}

}  // namespace

// Two blocks of eight rows per SM of a 148-SM part (at most); one block per eight rows below that.
int norm_gate_bwd_blocks(int64_t T) {
  const int64_t b = (T + 7) / 8;
  return static_cast<int>(b < 296 ? (b > 0 ? b : 1) : 296);
}

cudaError_t norm_gate_bwd(int64_t T, int D, int act_dt, const float* dg, const float* o, const void* u,
                          const void* zu, int64_t ld_act, const float* gamma, const float* beta, const float* mu,
                          const float* rstd, void* d_o, void* dz, int64_t ld_dz, float* partial, int* parts_out,
                          cudaStream_t st, int* status) {
  *parts_out = 0;
  if (T == 0) return cudaSuccess;
  const int G = norm_gate_bwd_blocks(T);
  cudaError_t e = prof_record(kProfNormBwd, false, st);
  if (e != cudaSuccess) return e;
  // the staged kernel copies whole rows: 16-byte aligned row starts for U and Z_U (dG, O and the
  // fp32 rows are [T, D] with D a multiple of 128)
  const bool staged = (((reinterpret_cast<uintptr_t>(u) | reinterpret_cast<uintptr_t>(zu) |
                         reinterpret_cast<uintptr_t>(dg) | reinterpret_cast<uintptr_t>(o) |
                         static_cast<uintptr_t>(ld_act * 2)) & 15) == 0);
  const int gs = static_cast<int>(std::min<int64_t>((T + 7) / 8, 2ll * sm_count()));
  int parts = G;   // partial rows written
#define HSTU_NGB_ONE(VPT, AT)                                                                                    \
  if (staged && gs <= G) {                                                                                       \
    constexpr int kSmem = 8 * kNgbSlots * VPT * 32 * 12;                                                         \
    auto kern = norm_gate_bwd_staged_kernel<VPT, AT>;                                                            \
    e = ensure_smem_attr(reinterpret_cast<const void*>(kern), kSmem);                                            \
    if (e == cudaSuccess)                                                                                        \
      e = launch_pdl(kern, dim3(gs), dim3(256), kSmem, st, T, dg, o, u, zu, ld_act, gamma, beta, mu, rstd, d_o, dz, \
                     ld_dz, partial, wait_ctl(status));                                                           \
    parts = gs;                                                                                                  \
  } else {                                                                                                       \
    e = launch_pdl(norm_gate_bwd_kernel<VPT, AT>, dim3(G), dim3(256), 0, st, T, dg, o, u, zu, ld_act, gamma, beta, \
                   mu, rstd, d_o, dz, ld_dz, partial);                                                            \
  }
#define HSTU_NGB(VPT)                                                                                            \
  if (act_dt == kDtF16) {                                                                                        \
    HSTU_NGB_ONE(VPT, kDtF16)                                                                                    \
  } else if (act_dt == kDtBF16) {                                                                                \
    HSTU_NGB_ONE(VPT, kDtBF16)                                                                                   \
  } else {                                                                                                       \
    return cudaErrorInvalidValue;                                                                                \
  }
  switch (D) {
    case 256: HSTU_NGB(8); break;
    case 512: HSTU_NGB(16); break;
    default: return cudaErrorInvalidValue;
  }
#undef HSTU_NGB
#undef HSTU_NGB_ONE
  if (e == cudaSuccess) e = prof_record(kProfNormBwd, true, st);
  *parts_out = parts;
  return e;
}

namespace {
// Partial rows of the fused column sum: blocks of at least 16 rows, at most kTailParts of them.
int tail_parts(int64_t T, int64_t* rows_per) {
  int64_t g = (T + 15) / 16;
  g = g < 1 ? 1 : (g > kTailParts ? kTailParts : g);
  *rows_per = (T + g - 1) / g;
  return static_cast<int>((T + *rows_per - 1) / *rows_per);
}
}  // namespace

namespace {
// Packs up to four column-sum finishes (32 columns a block); returns the block count.
int pack_colsum_jobs(const ColsumJob* jobs, int njobs, ColsumJobs* cj) {
  *cj = ColsumJobs{};
  int nb = 0, k = 0;
  for (int j = 0; j < njobs && j < 4; ++j) {
    if (jobs[j].cols <= 0) continue;
    cj->job[k] = jobs[j];
    cj->first_block[k] = nb;
    nb += (jobs[j].cols + 31) / 32;
    ++k;
  }
  cj->first_block[k] = nb;
  cj->njobs = k;
  return nb;
}
}  // namespace

cudaError_t dz_assemble(int64_t T, int D, int act_dt, const float* dv, const float* dq, const float* dk,
                        const void* z, int64_t ld_z, void* dz, int64_t ld_dz, float* partial, int* parts,
                        cudaStream_t st, float* db1, const ColsumJob* fin, int nfin) {
  *parts = static_cast<int>((T + 31) / 32);
  if (T == 0) return cudaSuccess;
  if (D % 64 || nfin > 4) return cudaErrorInvalidValue;
  const int64_t blocks = static_cast<int64_t>(4 * D / 64) * *parts;
  ColsumJobs cj;
  const int fin_blocks = pack_colsum_jobs(fin, fin ? nfin : 0, &cj);
  if (blocks + fin_blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(blocks + fin_blocks));
  if (act_dt != kDtF16 && act_dt != kDtBF16) return cudaErrorInvalidValue;
  cudaError_t e = prof_record(kProfDz, false, st);
  if (e == cudaSuccess)
    e = act_dt == kDtF16 ? launch_pdl(dz_assemble_kernel<kDtF16>, grid, dim3(256), 0, st, T, D, dv, dq, dk, z, ld_z,
                                      dz, ld_dz, partial, db1, cj, fin_blocks)
                         : launch_pdl(dz_assemble_kernel<kDtBF16>, grid, dim3(256), 0, st, T, D, dv, dq, dk, z, ld_z,
                                      dz, ld_dz, partial, db1, cj, fin_blocks);
  if (e == cudaSuccess) e = prof_record(kProfDz, true, st);
  return e;
}

cudaError_t rows_to_f16_colsum(int64_t T, int D, int in_dt, const void* in, void* out, float* partial, int* parts,
                               const ConvertJob* jobs, int njobs, cudaStream_t st) {
  *parts = 0;
  ConvertBatch cb{};
  int nb = 0, k = 0;
  if (njobs > kMaxConvertJobs) return cudaErrorInvalidValue;
  for (int j = 0; j < njobs; ++j) {
    if (jobs[j].n <= 0) continue;
    if (!jobs[j].out) return cudaErrorInvalidValue;
    if (jobs[j].in && jobs[j].in_dt != kDtF32 && jobs[j].in_dt != kDtBF16 && jobs[j].in_dt != kDtF16)
      return cudaErrorInvalidValue;
    cb.job[k] = jobs[j];
    cb.first_block[k] = nb;
    const int64_t blocks = ((jobs[j].n + 7) / 8 + 255) / 256;
    if (nb + blocks > 0x3fffffffLL) return cudaErrorInvalidValue;
    nb += static_cast<int>(blocks);
    ++k;
  }
  cb.first_block[k] = nb;
  cb.njobs = k;
  int64_t rows_per = 1;
  const int g = T > 0 ? tail_parts(T, &rows_per) : 0;
  *parts = g;
  if (g + nb == 0) return cudaSuccess;
#define HSTU_RC(DD, IT)                                                                                          \
  if (D == DD && in_dt == IT)                                                                                    \
    return launch_pdl(rows_to_f16_colsum_kernel<DD, IT>, dim3(g + nb), dim3(kTailThreads), 0, st, T, in, out,    \
                      rows_per, partial, g, cb);
  HSTU_RC(256, kDtF32)
  HSTU_RC(512, kDtF32)
  HSTU_RC(256, kDtBF16)
  HSTU_RC(512, kDtBF16)
  HSTU_RC(256, kDtF16)
  HSTU_RC(512, kDtF16)
#undef HSTU_RC
  return cudaErrorInvalidValue;
}


cudaError_t convert_dtype(const void* in, int in_dt, void* out, int out_dt, int64_t n, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>(((n + 7) / 8 + 255) / 256);
#define HSTU_CV(I, O) \
  if (in_dt == I && out_dt == O) return launch_pdl(convert_kernel<I, O>, dim3(blocks), dim3(256), 0, st, in, out, n);
  HSTU_CV(kDtBF16, kDtF16)
  HSTU_CV(kDtF32, kDtF16)
  HSTU_CV(kDtF32, kDtBF16)
  HSTU_CV(kDtF16, kDtBF16)
  HSTU_CV(kDtBF16, kDtF32)
  HSTU_CV(kDtF16, kDtF32)
#undef HSTU_CV
  return cudaErrorInvalidValue;
}

constexpr int kColsumParts = 256;   // most row slices of a column sum (the partial buffer's height)

size_t colsum_partial_floats(int cols) { return static_cast<size_t>(kColsumParts) * cols; }

cudaError_t column_sum(const void* in, int dt, int64_t rows, int cols, int64_t ld, float* partial, float* out,
                       cudaStream_t st) {
  if (cols == 0) return cudaSuccess;
  // about four blocks per SM: more row slices when there are few column blocks
  const int col_blocks = (cols + 255) / 256;
  int want = (4 * 148 + col_blocks - 1) / col_blocks;
  want = want < 32 ? 32 : (want > kColsumParts ? kColsumParts : want);
  const int64_t rows_per = (rows + want - 1) / want;
  const int parts = rows == 0 ? 1 : static_cast<int>((rows + rows_per - 1) / rows_per);
  if (rows == 0) return cudaMemsetAsync(out, 0, sizeof(float) * cols, st);
  dim3 grid((cols + 255) / 256, parts);
  cudaError_t e;
  if (dt == kDtF32) e = launch_pdl(colsum_partial_kernel<kDtF32>, grid, dim3(256), 0, st, in, rows, cols, ld, rows_per, partial);
  else if (dt == kDtBF16)
    e = launch_pdl(colsum_partial_kernel<kDtBF16>, grid, dim3(256), 0, st, in, rows, cols, ld, rows_per, partial);
  else e = launch_pdl(colsum_partial_kernel<kDtF16>, grid, dim3(256), 0, st, in, rows, cols, ld, rows_per, partial);
  if (e != cudaSuccess) return e;
  return launch_pdl(colsum_final_kernel, dim3((cols + 31) / 32), dim3(256), 0, st, static_cast<const float*>(partial), parts,
                    cols, out);
}

}  // namespace hstu
