// attn_fwd_sm100.cu - jagged causal pointwise attention, forward.
//
// O_i = sum_{j <= i, same sequence} SiLU(q_i . k_j + rab_pos[i-j] + rab_time[bucket(t_i - t_j)])
//       * inv_N * v_j   per head.
// ("4.4 Scaling Recommendation Models", Generative Recommenders and HSTU: second equation and the
// pointwise-aggregation bullet; "HSTU: The First Exploration of the Scaling Law", 7.1.4
// Innovation 1 (SiLU, no softmax, no 1/sqrt(d) scale) and Innovation 2 (position and time bias).)
//
// Tensor-core kernel (bf16 or fp16 operands, fp32 accumulation), one CTA per (sequence, 128-row query tile, head) from the jagged work
// list (longest causal rows first). Only key tiles 0..t of the query tile's own sequence are
// visited (causal tile skipping; padding never exists in the jagged layout).
//   warp 4  : TMA producer (Q once, K/V double-buffered, 128-byte swizzle)
//   warp 5  : tcgen05 issuer: S = Q K^T into a double-buffered TMEM tile, O += P V in TMEM
//   warps 0-3: one query row per thread: S from TMEM, + bias, SiLU, causal mask, bf16 P into
//             swizzled shared memory (the A operand of the P V MMA)
// 1/N is applied once to the fp32 accumulator in the epilogue.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hstu_internal.h"
#include "sm100_ptx.cuh"
#include "time_bucket_dev.cuh"

namespace hstu {

namespace {

constexpr int kThreads = 192;
constexpr int kD = 64;

struct AttnSmem {
  static constexpr int kQ = 0;
  static constexpr int kK = 16384;            // 2 stages
  static constexpr int kV = kK + 2 * 16384;   // 2 stages
  static constexpr int kP = kV + 2 * 16384;   // 2 buffers of 32 KB (two 64-key chunks)
  static constexpr int kRabTime = kP + 2 * 32768;
  static constexpr int kOct = kRabTime + 512;
  static constexpr int kKts = kOct + 63 * 32 + 32;   // 2 x 128 int64
  static constexpr int kPos = kKts + 2 * 128 * 8;    // 2 x 256 float
  static constexpr int kBar = kPos + 2 * 256 * 4;
  static constexpr int kTotal = kBar + 256 + 1024;
};

__device__ __forceinline__ int pos_index(long long r, int L) {
  r = r > L - 1 ? L - 1 : r;
  r = r < -(L - 1) ? -(L - 1) : r;
  return static_cast<int>(r) + L - 1;
}

template <bool F16>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, AttnArgs a, WaitCtl ctl) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int H = a.H;
  const int item = blockIdx.x / H;
  const int h = blockIdx.x - item * H;
  if (item >= *a.count) return;
  const int b = a.items[2 * item];
  const int qt = a.items[2 * item + 1];
  const long long seq0 = a.offsets[b];
  const int n = static_cast<int>(a.offsets[b + 1] - seq0);
  const int nkt = qt + 1;

  float* s_rab_time = reinterpret_cast<float*>(smem + AttnSmem::kRabTime);
  long long* s_tau = reinterpret_cast<long long*>(smem + AttnSmem::kOct);
  long long* s_kts = reinterpret_cast<long long*>(smem + AttnSmem::kKts);
  float* s_pos = reinterpret_cast<float*>(smem + AttnSmem::kPos);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AttnSmem::kBar);
  // 0 q_full | 1,2 kv_full | 3,4 kv_empty | 5,6 s_full | 7,8 s_free | 9,10 p_full | 11,12 p_empty
  // 13 o_full | 14 staging barrier of the 128 SiLU threads (a bounded replacement of bar.sync)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t bar_q = smem_u32(&bars[0]);
  auto bar_kv_full = [&](int s) { return smem_u32(&bars[1 + s]); };
  auto bar_kv_empty = [&](int s) { return smem_u32(&bars[3 + s]); };
  auto bar_s_full = [&](int s) { return smem_u32(&bars[5 + s]); };
  auto bar_s_free = [&](int s) { return smem_u32(&bars[7 + s]); };
  auto bar_p_full = [&](int s) { return smem_u32(&bars[9 + s]); };
  auto bar_p_empty = [&](int s) { return smem_u32(&bars[11 + s]); };
  const uint32_t bar_o = smem_u32(&bars[13]);
  const uint32_t bar_stage = smem_u32(&bars[14]);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tid = threadIdx.x;

  if (tid == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_kv_full(s), 1);
      mbar_init(bar_kv_empty(s), 1);
      mbar_init(bar_s_full(s), 1);
      mbar_init(bar_s_free(s), 128);
      mbar_init(bar_p_full(s), 128);
      mbar_init(bar_p_empty(s), 1);
    }
    mbar_init(bar_o, 1);
    mbar_init(bar_stage, 128);
    *abort_flag = 0;
    fence_barrier_init();
  }
  for (int e = tid; e < a.n_buckets && e < 128; e += kThreads) s_rab_time[e] = a.rab_time[e];
  for (int e = tid; e < kTauEntries; e += kThreads) s_tau[e] = g_time_taus[e];
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;           // S0: cols [0,128), S1: [128,256), O: [256,320)
  const uint32_t tmem_o = tmem + 256;

  const uint32_t sQ = smem_u32(smem + AttnSmem::kQ);
  const uint32_t sK0 = smem_u32(smem + AttnSmem::kK);
  const uint32_t sV0 = smem_u32(smem + AttnSmem::kV);
  const uint32_t sP0 = smem_u32(smem + AttnSmem::kP);
  const int qrow0 = static_cast<int>(seq0) + qt * kQTile;

  if (warp == 4) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, 16384);
      tma_load_2d(sQ, &tmQ, bar_q, h * kD, qrow0);
      for (int kt = 0; kt < nkt; ++kt) {
        const int s = kt & 1;
        if (kt >= 2 && !mbar_wait(bar_kv_empty(s), ((kt >> 1) & 1) ^ 1, abort_flag, ctl)) break;
        mbar_arrive_expect_tx(bar_kv_full(s), 32768);
        const int krow = static_cast<int>(seq0) + kt * kQTile;
        tma_load_2d(sK0 + s * 16384, &tmK, bar_kv_full(s), h * kD, krow);
        tma_load_2d(sV0 + s * 16384, &tmV, bar_kv_full(s), h * kD, krow);
      }
    }
  } else if (warp == 5) {
    // ---------------- tcgen05 issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc_f16kind(128, 128, 0, 0, F16);
      constexpr uint32_t idesc_pv = make_idesc_f16kind(128, 64, 0, 1, F16);
      bool ok = mbar_wait(bar_q, 0, abort_flag, ctl);
      auto issue_pv = [&](int t) -> bool {
        const int s = t & 1;
        if (!mbar_wait(bar_p_full(s), (t >> 1) & 1, abort_flag, ctl)) return false;
        tc_fence_after();
        const uint32_t p = sP0 + s * 32768;
        const uint32_t v = sV0 + s * 16384;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = make_sdesc_sw128(p + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = make_sdesc_sw128(v + kk * 2048, 16384, 1024);
          umma_f16_ss(tmem_o, ad, bd, idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar_kv_empty(s));
        umma_commit(bar_p_empty(s));
        return true;
      };
      for (int kt = 0; ok && kt < nkt; ++kt) {
        const int s = kt & 1;
        if (!mbar_wait(bar_kv_full(s), (kt >> 1) & 1, abort_flag, ctl)) { ok = false; break; }
        if (kt >= 2 && !mbar_wait(bar_s_free(s), ((kt >> 1) & 1) ^ 1, abort_flag, ctl)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kb = sK0 + s * 16384;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          umma_f16_ss(tmem + s * 128, make_sdesc_sw128(sQ + kk * 32, 16, 1024),
                      make_sdesc_sw128(kb + kk * 32, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar_s_full(s));
        if (kt >= 1 && !issue_pv(kt - 1)) { ok = false; break; }
      }
      if (ok && issue_pv(nkt - 1)) umma_commit(bar_o);
    }
  } else {
    // ---------------- SiLU warps: thread = query row ----------------
    const int r = tid;                       // 0..127, TMEM lane
    const int qi = qt * kQTile + r;          // local query index
    const long long gi = seq0 + (qi < n ? qi : (n > 0 ? n - 1 : 0));
    const long long t_i = a.ts[gi];
    const int L = a.pos_max_len;
    const int nb = a.n_buckets;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    bool ok = true;
    uint32_t stage_phase = 0;
    for (int kt = 0; kt < nkt; ++kt) {
      const int s = kt & 1;
      // stage this key tile's timestamps and the rab_pos window for i - j in
      // [128 (qt - kt) - 127, 128 (qt - kt) + 127]
      {
        const long long kj = seq0 + static_cast<long long>(kt) * kQTile + r;
        s_kts[s * 128 + r] = kj < a.T ? a.ts[kj] : 0;
        const long long rel0 = static_cast<long long>(qt - kt) * kQTile - 127;
        s_pos[s * 256 + r] = a.rab_pos[pos_index(rel0 + r, L)];
        if (r < 127) s_pos[s * 256 + 128 + r] = a.rab_pos[pos_index(rel0 + 128 + r, L)];
      }
      mbar_arrive(bar_stage);
      if (!mbar_wait(bar_stage, stage_phase, abort_flag, ctl)) { ok = false; break; }
      stage_phase ^= 1;
      if (!mbar_wait(bar_s_full(s), (kt >> 1) & 1, abort_flag, ctl)) { ok = false; break; }
      tc_fence_after();
      if (kt >= 2 && !mbar_wait(bar_p_empty(s), ((kt >> 1) & 1) ^ 1, abort_flag, ctl)) { ok = false; break; }
      const bool diag = (kt == qt);
      uint8_t* prow = smem + AttnSmem::kP + s * 32768 + r * 128;
      const float* pw = s_pos + s * 256 + r + 127;     // pw[-col] = rab_pos for (r, col)
      const long long* kts = s_kts + s * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t sv[32];
        tmem_ld_32x32b_x32(tmem + lane_base + s * 128 + c * 32, sv);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          float y[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int col = c * 32 + j + e;
            const int bkt = time_bucket_pair64(t_i, kts[col], s_tau, nb);
            const float x = __uint_as_float(sv[j + e]) + pw[-col] + s_rab_time[bkt];
            y[e] = (!diag || col <= r) ? silu_fast(x) : 0.0f;
          }
          pk[j / 2] = F16 ? pack_f16x2(y[0], y[1]) : pack_bf16x2(y[0], y[1]);
        }
        uint8_t* chunk = prow + (c >> 1) * 16384;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int u = (c & 1) * 4 + q;
          *reinterpret_cast<uint4*>(chunk + ((u ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar_s_free(s));
      fence_proxy_async_smem();
      mbar_arrive(bar_p_full(s));
    }
    if (ok && mbar_wait(bar_o, 0, abort_flag, ctl)) {
      tc_fence_after();
      uint32_t o0[32], o1[32];
      tmem_ld_32x32b_x32(tmem_o + lane_base, o0);
      tmem_ld_32x32b_x32(tmem_o + lane_base + 32, o1);
      tmem_ld_wait();
      if (qi < n) {
        const float sc = a.inv_N;
        if (a.o_f32) {
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.o) + (seq0 + qi) * a.ld_o + h * kD);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(__uint_as_float(o0[4 * q]) * sc, __uint_as_float(o0[4 * q + 1]) * sc,
                                 __uint_as_float(o0[4 * q + 2]) * sc, __uint_as_float(o0[4 * q + 3]) * sc);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[8 + q] = make_float4(__uint_as_float(o1[4 * q]) * sc, __uint_as_float(o1[4 * q + 1]) * sc,
                                     __uint_as_float(o1[4 * q + 2]) * sc, __uint_as_float(o1[4 * q + 3]) * sc);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) + (seq0 + qi) * a.ld_o + h * kD);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pack_bf16x2(__uint_as_float(o0[8 * q]) * sc, __uint_as_float(o0[8 * q + 1]) * sc),
                                pack_bf16x2(__uint_as_float(o0[8 * q + 2]) * sc, __uint_as_float(o0[8 * q + 3]) * sc),
                                pack_bf16x2(__uint_as_float(o0[8 * q + 4]) * sc, __uint_as_float(o0[8 * q + 5]) * sc),
                                pack_bf16x2(__uint_as_float(o0[8 * q + 6]) * sc, __uint_as_float(o0[8 * q + 7]) * sc));
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[4 + q] = make_uint4(pack_bf16x2(__uint_as_float(o1[8 * q]) * sc, __uint_as_float(o1[8 * q + 1]) * sc),
                                    pack_bf16x2(__uint_as_float(o1[8 * q + 2]) * sc, __uint_as_float(o1[8 * q + 3]) * sc),
                                    pack_bf16x2(__uint_as_float(o1[8 * q + 4]) * sc, __uint_as_float(o1[8 * q + 5]) * sc),
                                    pack_bf16x2(__uint_as_float(o1[8 * q + 6]) * sc, __uint_as_float(o1[8 * q + 7]) * sc));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------------------------------------------
// fp32 CUDA-core kernel (exact fp32 mode): one warp per (query row, head); lanes hold features.
// ----------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128)
attn_fwd_f32_kernel(AttnArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long wid = static_cast<long long>(blockIdx.x) * 4 + warp;
  if (wid >= a.T * a.H) return;
  const long long i = wid / a.H;
  const int h = static_cast<int>(wid - i * a.H);
  // sequence of row i: last b with offsets[b] <= i (binary search over non-decreasing offsets)
  int lo = 0, hi = a.B;   // invariant offsets[lo] <= i < offsets[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (a.offsets[mid] <= i) lo = mid; else hi = mid;
  }
  const long long s0 = a.offsets[lo];
  const float* q = reinterpret_cast<const float*>(a.q) + i * a.ld_q + h * a.dqk;
  const float q0 = lane < a.dqk ? q[lane] : 0.0f;
  const float q1 = lane + 32 < a.dqk ? q[lane + 32] : 0.0f;
  float acc0 = 0.0f, acc1 = 0.0f;
  const long long t_i = a.ts[i];
  const int L = a.pos_max_len;
  for (long long j = s0; j <= i; ++j) {
    const float* kr = reinterpret_cast<const float*>(a.k) + j * a.ld_k + h * a.dqk;
    float part = (lane < a.dqk ? q0 * kr[lane] : 0.0f) + (lane + 32 < a.dqk ? q1 * kr[lane + 32] : 0.0f);
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) part += __shfl_xor_sync(0xffffffffu, part, m);
    const int bkt = time_bucket_pair64(t_i, a.ts[j], c_time_taus, a.n_buckets);
    const float x = part + a.rab_pos[pos_index(i - j, L)] + a.rab_time[bkt];
    const float w = x / (1.0f + expf(-x)) * a.inv_N;
    const float* vr = reinterpret_cast<const float*>(a.v) + j * a.ld_v + h * a.dv;
    if (lane < a.dv) acc0 = fmaf(w, vr[lane], acc0);
    if (lane + 32 < a.dv) acc1 = fmaf(w, vr[lane + 32], acc1);
  }
  float* o = reinterpret_cast<float*>(a.o) + i * a.ld_o + h * a.dv;
  if (lane < a.dv) o[lane] = acc0;
  if (lane + 32 < a.dv) o[lane + 32] = acc1;
}

}  // namespace

cudaError_t attn_fwd_bf16_tc(const AttnArgs& a, cudaStream_t st) {
  cudaError_t e = upload_time_taus();
  if (e != cudaSuccess) return e;
  if (a.T == 0 || a.capacity == 0) return cudaSuccess;
  CUtensorMap tq, tk, tv;
  const bool f16 = a.in_f16 != 0;
  if (!encode_tmap_2d_bf16(&tq, a.q, static_cast<int64_t>(a.H) * kD, a.T, a.ld_q, 64, 128, f16) ||
      !encode_tmap_2d_bf16(&tk, a.k, static_cast<int64_t>(a.H) * kD, a.T, a.ld_k, 64, 128, f16) ||
      !encode_tmap_2d_bf16(&tv, a.v, static_cast<int64_t>(a.H) * kD, a.T, a.ld_v, 64, 128, f16))
    return cudaErrorInvalidValue;
  auto kern = f16 ? attn_fwd_tc_kernel<true> : attn_fwd_tc_kernel<false>;
  e = ensure_smem_attr(reinterpret_cast<const void*>(kern), AttnSmem::kTotal);
  if (e != cudaSuccess) return e;
  const long long blocks = a.capacity * a.H;
  kern<<<static_cast<unsigned>(blocks), kThreads, AttnSmem::kTotal, st>>>(tq, tk, tv, a, wait_ctl(a.status));
  return cudaGetLastError();
}

cudaError_t attn_fwd_f32_simt(const AttnArgs& a, cudaStream_t st) {
  cudaError_t e = upload_time_taus();
  if (e != cudaSuccess) return e;
  const long long warps = a.T * a.H;
  if (warps == 0) return cudaSuccess;
  attn_fwd_f32_kernel<<<static_cast<unsigned>((warps + 3) / 4), 128, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace hstu
