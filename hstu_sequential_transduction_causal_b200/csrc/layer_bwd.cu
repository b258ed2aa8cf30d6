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

__device__ __forceinline__ float silu_grad(float z) {
  const float s = 1.0f / (1.0f + __expf(fminf(-z, 80.0f)));
  return s * (1.0f + z * (1.0f - s));
}

// One warp per token row (grid-stride over rows); lane l holds features 128 k + 4 l + i (k < VPT / 4,
// i < 4): every load and store of the warp covers 128 consecutive features (coalesced).
// Writes dO (act dtype), dZ_U = dU (.) SiLU'(Z_U) (fp16, row stride ld_dz) and per-block partial
// sums of dgamma | dbeta into partial[blockIdx.x][0 .. 2D).
template <int VPT, int AT>
__global__ void __launch_bounds__(256)
norm_gate_bwd_kernel(int64_t T, const float* __restrict__ dg, const float* __restrict__ o, const void* __restrict__ u,
                     const void* __restrict__ zu, int64_t ld_act, const float* __restrict__ gamma,
                     const float* __restrict__ beta, const float* __restrict__ mu, const float* __restrict__ rstd,
                     void* __restrict__ d_o, void* __restrict__ dz, int64_t ld_dz, float* __restrict__ partial) {
  pdl_enter();
  constexpr int D = VPT * 32;
  constexpr int KG = VPT / 4;   // groups of 4 features per lane
  __shared__ float s_red[8][2][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  auto feat = [&](int e) { return 128 * (e >> 2) + 4 * lane + (e & 3); };
  float gacc[VPT], bacc[VPT];
#pragma unroll
  for (int e = 0; e < VPT; ++e) gacc[e] = bacc[e] = 0.0f;
  float gm[VPT], bt[VPT];
#pragma unroll
  for (int k = 0; k < KG; ++k) {
    load_vec<4, kDtF32>(gamma, 128 * k + 4 * lane, gm + 4 * k);
    load_vec<4, kDtF32>(beta, 128 * k + 4 * lane, bt + 4 * k);
  }
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
    for (int e = 0; e < VPT; ++e) {
      const float xh = (x[e] - m) * rs;
      const float dln = g[e] * uu[e];
      const float dxh = dln * gm[e];
      gacc[e] = fmaf(dln, xh, gacc[e]);
      bacc[e] += dln;
      s1 += dxh;
      s2 = fmaf(dxh, xh, s2);
      const float du = g[e] * fmaf(gm[e], xh, bt[e]);
      z[e] = du * silu_grad(z[e]);        // dZ_U
      x[e] = xh;                          // keep xhat
      g[e] = dxh;                         // keep dxhat
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
    for (int k = 0; k < KG; ++k) {
      const int c = 128 * k + 4 * lane;
      store_vec<4, AT>(d_o, row * D + c, g + 4 * k);
      store_vec<4, kDtF16>(dz, row * ld_dz + c, z + 4 * k);
    }
  }
#pragma unroll
  for (int e = 0; e < VPT; ++e) {
    s_red[warp][0][feat(e)] = gacc[e];
    s_red[warp][1][feat(e)] = bacc[e];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < 2 * D; c += 256) {
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += s_red[w][c / D][c % D];
    partial[static_cast<int64_t>(blockIdx.x) * 2 * D + c] = s;
  }
}

// dZ[:, D:4D] = [dV | dQ | dK] (.) SiLU'(Z[:, D:4D]) in fp16; g* are fp32 [T, D].
template <int AT>
__global__ void __launch_bounds__(256)
dz_assemble_kernel(int64_t T, int D, const float* __restrict__ dv, const float* __restrict__ dq,
                   const float* __restrict__ dk, const void* __restrict__ z, int64_t ld_z, void* __restrict__ dz,
                   int64_t ld_dz) {
  pdl_enter();
  const int64_t idx = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 8;   // over T x 3D
  const int64_t per_row = 3ll * D;
  if (idx >= T * per_row) return;
  const int64_t row = idx / per_row;
  const int c = static_cast<int>(idx - row * per_row);   // multiple of 8, block of 8 inside one of V|Q|K
  const int blk = c / D, cc = c - blk * D;
  const float* g = blk == 0 ? dv : (blk == 1 ? dq : dk);
  float gv[8], zv[8];
  load_vec<8, kDtF32>(g, row * D + cc, gv);
  load_vec<8, AT>(z, row * ld_z + D + c, zv);
#pragma unroll
  for (int e = 0; e < 8; ++e) gv[e] *= silu_grad(zv[e]);
  store_vec<8, kDtF16>(dz, row * ld_dz + D + c, gv);
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

int norm_gate_bwd_blocks(int64_t T) {
  const int64_t b = (T + 7) / 8;
  return static_cast<int>(b < 296 ? (b > 0 ? b : 1) : 296);
}

cudaError_t norm_gate_bwd(int64_t T, int D, int act_dt, const float* dg, const float* o, const void* u,
                          const void* zu, int64_t ld_act, const float* gamma, const float* beta, const float* mu,
                          const float* rstd, void* d_o, void* dz, int64_t ld_dz, float* partial,
                          float* dgamma_dbeta_out, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int G = norm_gate_bwd_blocks(T);
  cudaError_t e = prof_record(kProfNormBwd, false, st);
  if (e != cudaSuccess) return e;
#define HSTU_NGB(VPT)                                                                                            \
  if (act_dt == kDtF16)                                                                                          \
    e = launch_pdl(norm_gate_bwd_kernel<VPT, kDtF16>, dim3(G), dim3(256), 0, st, T, dg, o, u, zu, ld_act, gamma,   \
                   beta, mu, rstd, d_o, dz, ld_dz, partial);                                                      \
  else if (act_dt == kDtBF16)                                                                                    \
    e = launch_pdl(norm_gate_bwd_kernel<VPT, kDtBF16>, dim3(G), dim3(256), 0, st, T, dg, o, u, zu, ld_act, gamma,  \
                   beta, mu, rstd, d_o, dz, ld_dz, partial);                                                      \
  else                                                                                                           \
    return cudaErrorInvalidValue;
  switch (D) {
    case 256: HSTU_NGB(8); break;
    case 512: HSTU_NGB(16); break;
    default: return cudaErrorInvalidValue;
  }
#undef HSTU_NGB
  if (e == cudaSuccess) e = prof_record(kProfNormBwd, true, st);
  if (e != cudaSuccess) return e;
  return launch_pdl(colsum_final_kernel, dim3((2 * D + 31) / 32), dim3(256), 0, st, static_cast<const float*>(partial), G,
                    2 * D, dgamma_dbeta_out);
}

cudaError_t dz_assemble(int64_t T, int D, int act_dt, const float* dv, const float* dq, const float* dk,
                        const void* z, int64_t ld_z, void* dz, int64_t ld_dz, cudaStream_t st) {
  const int64_t threads = T * 3ll * D / 8;
  if (threads == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
  if (act_dt == kDtF16)
    return launch_pdl(dz_assemble_kernel<kDtF16>, dim3(blocks), dim3(256), 0, st, T, D, dv, dq, dk, z, ld_z, dz, ld_dz);
  if (act_dt == kDtBF16)
    return launch_pdl(dz_assemble_kernel<kDtBF16>, dim3(blocks), dim3(256), 0, st, T, D, dv, dq, dk, z, ld_z, dz, ld_dz);
  return cudaErrorInvalidValue;
}

struct ConvertBatch {
  ConvertJob job[4];
  int first_block[5];   // block b converts job j with first_block[j] <= b < first_block[j + 1]
  int njobs;
};

// Several tensors converted to fp16 by one launch: each block finds its job, then 8 elements per
// thread as in convert_kernel.
__global__ void __launch_bounds__(256)
convert_many_kernel(ConvertBatch cb) {
  pdl_enter();
  int j = 0;
  while (j + 1 < cb.njobs && static_cast<int>(blockIdx.x) >= cb.first_block[j + 1]) ++j;
  const ConvertJob& jb = cb.job[j];
  const int64_t i = (static_cast<int64_t>(blockIdx.x - cb.first_block[j]) * blockDim.x + threadIdx.x) * 8;
  if (i >= jb.n) return;
  const int cnt = jb.n - i >= 8 ? 8 : static_cast<int>(jb.n - i);
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

cudaError_t convert_many_to_f16(const ConvertJob* jobs, int njobs, cudaStream_t st) {
  ConvertBatch cb{};
  int nb = 0, k = 0;
  for (int j = 0; j < njobs && j < 4; ++j) {
    if (jobs[j].n <= 0) continue;
    if (jobs[j].in_dt != kDtF32 && jobs[j].in_dt != kDtBF16 && jobs[j].in_dt != kDtF16) return cudaErrorInvalidValue;
    cb.job[k] = jobs[j];
    cb.first_block[k] = nb;
    const int64_t blocks = ((jobs[j].n + 7) / 8 + 255) / 256;
    if (nb + blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    nb += static_cast<int>(blocks);
    ++k;
  }
  if (k == 0) return cudaSuccess;
  cb.first_block[k] = nb;
  cb.njobs = k;
  return launch_pdl(convert_many_kernel, dim3(static_cast<unsigned>(nb)), dim3(256), 0, st, cb);
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
