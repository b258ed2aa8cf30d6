// norm_in.cu - backward of the input LayerNorm of the norm_in layer variant (the first page's "Code"
// sketch normalises the layer input before f1: Xn = LayerNorm_in(X), the residual adds X).
//
// Given d Xn (fp32, the f1 backward's dZ W1), per token with xhat = (x - mu) rstd and g = d Xn gamma:
//   dX = dY + rstd (g - mean(g) - xhat mean(g xhat))          (mean over the D features of the token)
// and, summed over tokens, dgamma = sum d Xn xhat, dbeta = sum d Xn. One warp per token (lane l holds
// the 4-feature groups 4 l + 128 k as in the forward); a fixed grid of blocks strides over the tokens
// and leaves per-block partial sums of dgamma | dbeta, added up by a second kernel.
#include <cuda_runtime.h>
#include <stdint.h>

#include "hstu_internal.h"
#include "sm100_ptx.cuh"
#include "vec_io.cuh"

namespace hstu {
namespace {

constexpr int kLnBlocks = 296;

template <int VPT, int XT, int YT>
__global__ void __launch_bounds__(256)
ln_in_bwd_kernel(int64_t T, const float* __restrict__ dxn, const void* __restrict__ x, const void* __restrict__ dy,
                 const float* __restrict__ gamma, const float* __restrict__ mu, const float* __restrict__ rstd,
                 void* __restrict__ dx, void* __restrict__ dx_f16, float* __restrict__ partial) {
  pdl_enter();
  constexpr int D = VPT * 32;
  constexpr bool kGrouped = VPT % 4 == 0;
  constexpr int KG = kGrouped ? VPT / 4 : 1, W = kGrouped ? 4 : VPT;
  __shared__ float s_acc[8][2 * D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  auto col = [&](int k) { return kGrouped ? 128 * k + 4 * lane : lane * VPT; };
  float gm[VPT], accg[VPT], accb[VPT];
#pragma unroll
  for (int k = 0; k < KG; ++k) load_vec<W, kDtF32>(gamma, col(k), gm + W * k);
#pragma unroll
  for (int e = 0; e < VPT; ++e) accg[e] = accb[e] = 0.0f;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + warp; row < T; row += static_cast<int64_t>(gridDim.x) * 8) {
    float d[VPT], xv[VPT];
#pragma unroll
    for (int k = 0; k < KG; ++k) {
      load_vec<W, kDtF32>(dxn, row * D + col(k), d + W * k);
      load_vec<W, XT>(x, row * D + col(k), xv + W * k);
    }
    const float m = mu[row], r = rstd[row];
    float sg = 0.0f, sgx = 0.0f;
#pragma unroll
    for (int e = 0; e < VPT; ++e) {
      xv[e] = (xv[e] - m) * r;               // xhat
      const float g = d[e] * gm[e];
      sg += g;
      sgx = fmaf(g, xv[e], sgx);
      accg[e] = fmaf(d[e], xv[e], accg[e]);
      accb[e] += d[e];
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) {
      sg += __shfl_xor_sync(0xffffffffu, sg, s);
      sgx += __shfl_xor_sync(0xffffffffu, sgx, s);
    }
    const float mg = sg * (1.0f / D), mgx = sgx * (1.0f / D);
    float out[VPT];
#pragma unroll
    for (int k = 0; k < KG; ++k) load_vec<W, YT>(dy, row * D + col(k), out + W * k);
#pragma unroll
    for (int e = 0; e < VPT; ++e) out[e] += r * (d[e] * gm[e] - mg - xv[e] * mgx);
#pragma unroll
    for (int k = 0; k < KG; ++k) {
      store_vec<W, XT>(dx, row * D + col(k), out + W * k);
      if (dx_f16) store_vec<W, kDtF16>(dx_f16, row * D + col(k), out + W * k);
    }
  }
#pragma unroll
  for (int k = 0; k < KG; ++k)
#pragma unroll
    for (int i = 0; i < W; ++i) {
      s_acc[warp][col(k) + i] = accg[W * k + i];
      s_acc[warp][D + col(k) + i] = accb[W * k + i];
    }
  __syncthreads();
  for (int c = threadIdx.x; c < 2 * D; c += 256) {
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += s_acc[w][c];
    partial[static_cast<int64_t>(blockIdx.x) * 2 * D + c] = v;
  }
}

__global__ void __launch_bounds__(256)
ln_in_bwd_finish_kernel(const float* __restrict__ partial, int parts, int D, float* __restrict__ dgamma,
                        float* __restrict__ dbeta) {
  pdl_enter();
  const int c = blockIdx.x * 256 + threadIdx.x;
  if (c >= 2 * D) return;
  float v = 0.0f;
  for (int p = 0; p < parts; ++p) v += partial[static_cast<int64_t>(p) * 2 * D + c];
  if (c < D) dgamma[c] = v;
  else dbeta[c - D] = v;
}

}  // namespace

size_t ln_in_bwd_partial_floats(int D) { return static_cast<size_t>(kLnBlocks) * 2 * D; }

cudaError_t ln_in_bwd(int64_t T, int D, int x_dt, int y_dt, const float* dxn, const void* x, const void* dy,
                      const float* gamma, const float* mu, const float* rstd, void* dx, void* dx_f16, float* partial,
                      float* dgamma, float* dbeta, cudaStream_t st) {
  const int64_t want = (T + 7) / 8;
  const int G = static_cast<int>(want < kLnBlocks ? (want > 0 ? want : 1) : kLnBlocks);
  cudaError_t e = cudaErrorInvalidValue;
#define HSTU_LNB(VPT)                                                                                              \
  if (x_dt == kDtF32 && y_dt == kDtF32)                                                                            \
    e = launch_pdl(ln_in_bwd_kernel<VPT, kDtF32, kDtF32>, dim3(G), dim3(256), 0, st, T, dxn, x, dy, gamma, mu, rstd, \
                   dx, dx_f16, partial);                                                                            \
  else if (x_dt == kDtBF16 && y_dt == kDtBF16)                                                                     \
    e = launch_pdl(ln_in_bwd_kernel<VPT, kDtBF16, kDtBF16>, dim3(G), dim3(256), 0, st, T, dxn, x, dy, gamma, mu,     \
                   rstd, dx, dx_f16, partial);                                                                      \
  else                                                                                                             \
    return cudaErrorInvalidValue;
  switch (D) {
    case 256: HSTU_LNB(8); break;
    case 512: HSTU_LNB(16); break;
    default: return cudaErrorInvalidValue;
  }
#undef HSTU_LNB
  if (e != cudaSuccess) return e;
  return launch_pdl(ln_in_bwd_finish_kernel, dim3((2 * D + 255) / 256), dim3(256), 0, st,
                    static_cast<const float*>(partial), G, D, dgamma, dbeta);
}

}  // namespace hstu
