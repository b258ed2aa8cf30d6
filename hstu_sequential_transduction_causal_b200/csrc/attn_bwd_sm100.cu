// attn_bwd_sm100.cu - jagged causal pointwise attention, backward.
//
// With x_ij = q_i.k_j + rab(i, j), A_ij = SiLU(x_ij) inv_N on causal pairs (j <= i) and 0 elsewhere,
// O = A V (per head). Given dO:
//   dV = A^T dO,  dA = dO V^T,  dX = dA (.) SiLU'(x) inv_N (causal pairs),
//   dQ = dX K,  dK = dX^T Q,  d rab_pos[idx(i-j)] += sum_h dX_ij,  d rab_time[bucket(t_i - t_j)] += sum_h dX_ij
// (derived from the forward of "4.4 Scaling Recommendation Models", Generative Recommenders and HSTU,
// second equation, and the bias of "HSTU: The First Exploration of the Scaling Law", 7.1.4
// Innovation 2).
//
// attn_bias_t_kernel: per causal (query tile, key tile) pair, the transposed fp16 half-bias tile
// [key][query] and the u8 time-bucket tile [key][query] (head independent, computed once).
// attn_bwd_tc_kernel<F16>: one CTA per (sequence, 128-key tile, head), key tiles that visit the
// most query tiles first; it walks the query tiles t >= its key tile:
//   warp 8   : TMA: K, V once; Q and dO of each query tile (2 stages); the half-bias tile.
//   warp 9   : tcgen05: S^T = K Q^T and dA^T = V dO^T into TMEM; after the elementwise step
//              dV += P^T dO (P^T from TMEM), dK += dX^T Q and dQ_tile = dX K (dX^T from shared
//              memory, read K-major for dK and MN-major for dQ).
//   warp 10  : TMA store of each tile's dX^T (16-bit, from shared memory) to the workspace.
//   warps 0-7: key row = TMEM lane (warp & 3), query half (warp >> 2): x = s + bias,
//              P^T = SiLU(x), dX^T = dA SiLU'(x) inv_N in fp32, causal and length masks;
//              dQ_tile added to the fp32 dQ by vector atomics.
// attn_table_grad_kernel<F16>: per causal tile pair, sums the H heads' dX^T tiles and adds them to
// d rab_pos (by diagonal) and d rab_time (by bucket): the tables are shared by the heads, so the
// head sum comes first and each table entry takes one atomic per tile pair.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hstu_internal.h"
#include "sm100_ptx.cuh"
#include "tile_pairs.cuh"
#include "time_bucket_dev.cuh"

namespace hstu {

namespace {

constexpr int kD = 64;
constexpr int kSiluWarpsB = 8;
constexpr int kThreadsB = 32 * (kSiluWarpsB + 3);   // + TMA producer, MMA issuer, dX^T store warp
constexpr int kSiluThreadsB = 32 * kSiluWarpsB;

__device__ __forceinline__ int pos_index_b(long long r, int L) {
  r = r > L - 1 ? L - 1 : r;
  r = r < -(L - 1) ? -(L - 1) : r;
  return static_cast<int>(r) + L - 1;
}

// ----------------------------------------------------------------------------------------------
// transposed bias and bucket tiles
// ----------------------------------------------------------------------------------------------
// Four blocks per causal tile pair, 32 key rows each. Thread t writes 8 consecutive queries
// [8 (t % 16), +8) of key rows 32 y + t / 16 + 16 p, p = 0, 1: 16-byte half-bias and 8-byte bucket
// stores. Differences within a tile that fit in int32 take 32-bit bucket arithmetic.
__global__ void __launch_bounds__(256)
attn_bias_t_kernel(AttnBwdArgs A) {
  const AttnArgs& a = A.f;
  int b, qt, kt;
  if (!decode_tile_pair(blockIdx.x, a.pair_base, a.B, &b, &qt, &kt)) return;
  const long long seq0 = a.offsets[b];
  const int n = static_cast<int>(a.offsets[b + 1] - seq0);
  __shared__ long long s_qts[128], s_kts[128], s_tau[kTauEntries], s_red[16];
  __shared__ int s_tau32[kTauEntries];
  __shared__ float s_win[256], s_rt[128];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int L = a.pos_max_len;
  const int nb = a.n_buckets;
  long long t;
  if (tid < 128) {
    const int qi = qt * kQTile + tid;
    t = a.ts[seq0 + (qi < n ? qi : n - 1)];
    s_qts[tid] = t;
  } else {
    const int kj = kt * kQTile + tid - 128;
    t = a.ts[seq0 + (kj < n ? kj : n - 1)];
    s_kts[tid - 128] = t;
  }
  if (tid < nb) s_rt[tid] = 0.5f * a.rab_time[tid];
  if (tid < 255) s_win[tid] = 0.5f * a.rab_pos[pos_index_b(static_cast<long long>(qt - kt) * kQTile - 127 + tid, L)];
  for (int e = tid; e < kTauEntries; e += 256) {
    s_tau[e] = c_time_taus[e];
    s_tau32[e] = c_time_taus32[e];
  }
  long long mn = t, mx = t;
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) {
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, d));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, d));
  }
  if (lane == 0) {
    s_red[warp] = mn;
    s_red[8 + warp] = mx;
  }
  __syncthreads();
  long long lo = s_red[0], hi = s_red[8];
#pragma unroll
  for (int w = 1; w < 8; ++w) {
    lo = min(lo, s_red[w]);
    hi = max(hi, s_red[8 + w]);
  }
  const bool fast = hi - lo < 0x7fffffffLL;
  const int c0 = 8 * (tid & 15);
  const long long tile0 = blockIdx.x * static_cast<long long>(kQTile * kQTile);
  uint16_t* tile = reinterpret_cast<uint16_t*>(A.bias_t) + tile0;
  uint8_t* btile = reinterpret_cast<uint8_t*>(A.bucket_t) + tile0;
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int j = 32 * blockIdx.y + (tid >> 4) + 16 * pass;   // key row within the tile
    uint32_t w[4], bw[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float v2[2];
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const int col = c0 + 2 * e + x;     // query column
        const int bkt = fast ? time_bucket32(static_cast<int>(s_qts[col] - lo) - static_cast<int>(s_kts[j] - lo),
                                             s_tau32, nb)
                             : time_bucket_dev(s_qts[col] - s_kts[j], s_tau, nb);
        v2[x] = s_win[col - j + 127] + s_rt[bkt];
        bw[e >> 1] |= static_cast<uint32_t>(bkt) << (8 * (2 * (e & 1) + x));
      }
      w[e] = pack_f16x2(v2[0], v2[1]);
    }
    *reinterpret_cast<uint4*>(tile + j * kQTile + c0) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint2*>(btile + j * kQTile + c0) = make_uint2(bw[0], bw[1]);
  }
}

// ----------------------------------------------------------------------------------------------
// backward kernel
// ----------------------------------------------------------------------------------------------
struct BwdSmem {
  static constexpr int kK = 0;                  // K tile of the CTA (16 KB)
  static constexpr int kV = 16384;              // V tile (16 KB)
  static constexpr int kQ0 = 32768;             // stage st: Q at kQ0 + st * 32768, dO at +16384
  static constexpr int kBT0 = kQ0 + 2 * 32768;  // stage st: half-bias^T, overwritten in place by dX^T
  static constexpr int kBar = kBT0 + 2 * 32768;
  static constexpr int kTotal = kBar + 256 + 1024;
};
static_assert(BwdSmem::kTotal <= 232448, "shared memory of the backward kernel");

template <bool F16>
__global__ void __launch_bounds__(kThreadsB, 1)
attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                   const __grid_constant__ CUtensorMap tmBT, const __grid_constant__ CUtensorMap tmDX,
                   AttnBwdArgs A, WaitCtl ctl) {
  using Lb = BwdSmem;
  const AttnArgs& a = A.f;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int item = blockIdx.x / a.H;
  const int h = blockIdx.x - item * a.H;
  if (item >= *A.kcount) return;
  const int b = A.kitems[2 * item];
  const int kt = A.kitems[2 * item + 1];
  const long long seq0 = a.offsets[b];
  const int n = static_cast<int>(a.offsets[b + 1] - seq0);
  const int nt = (n + kQTile - 1) / kQTile;
  const int nsteps = nt - kt;              // query tiles kt .. nt-1
  const long long pbase = a.pair_base[b];

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lb::kBar);
  // 0 kv_full | 1,2 qdo_full | 3,4 qdo_empty | 5,6 bb_full | 7,8 bb_empty | 9,10 s_full (query half
  // a, b) | 11,12 p_ready (half a, b) | 13 dq_full | 14 fin | 15,16 dx_full (stage)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 17);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t bar0 = smem_u32(bars);
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tid = threadIdx.x;

  if (tid == 0) {
    mbar_init(BAR(0), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(1 + s), 1);
      mbar_init(BAR(3 + s), 1);
      mbar_init(BAR(5 + s), 1);
      mbar_init(BAR(7 + s), 2);   // bias/dX stage free: the MMAs read dX^T and the store warp sent it
      mbar_init(BAR(15 + s), kSiluThreadsB);   // both query halves of dX^T written
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(BAR(9 + h), 1);
      mbar_init(BAR(11 + h), kSiluThreadsB / 2);
    }
    mbar_init(BAR(13), 1);
    mbar_init(BAR(14), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kSiluWarpsB && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmDO);
    tma_prefetch_desc(&tmBT);
    tma_prefetch_desc(&tmDX);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // query half h: S^T_h at columns [128 h, 128 h + 64) (P^T_h packed over its first 32), dA^T_h at
  // [128 h + 64, 128 h + 128); accumulators dV, dK and the dQ tile of one query tile
  const uint32_t tDV = tmem + 256, tDK = tmem + 320, tDQ = tmem + 384;

  const uint32_t sK = smem_u32(smem + Lb::kK), sV = smem_u32(smem + Lb::kV);
  const uint32_t sQ0 = smem_u32(smem + Lb::kQ0);
  const uint32_t sBT0 = smem_u32(smem + Lb::kBT0);
  const int krow = static_cast<int>(seq0) + kt * kQTile;

  if (warp == kSiluWarpsB) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      mbar_arrive_expect_tx(BAR(0), 32768);
      tma_load_2d(sK, &tmK, BAR(0), h * kD, krow);
      tma_load_2d(sV, &tmV, BAR(0), h * kD, krow);
      for (int s = 0; s < nsteps; ++s) {
        const int qt = kt + s, st = s & 1;
        const uint32_t ph_free = ((s >> 1) & 1) ^ 1;
        if (s >= 2 && !mbar_wait(BAR(3 + st), ph_free, abort_flag, ctl)) break;
        const int qrow = static_cast<int>(seq0) + qt * kQTile;
        mbar_arrive_expect_tx(BAR(1 + st), 32768);
        tma_load_2d(sQ0 + st * 32768, &tmQ, BAR(1 + st), h * kD, qrow);
        tma_load_2d(sQ0 + st * 32768 + 16384, &tmDO, BAR(1 + st), h * kD, qrow);
        if (s >= 2 && !mbar_wait(BAR(7 + st), ph_free, abort_flag, ctl)) break;
        const int prow = static_cast<int>((pbase + static_cast<long long>(qt) * (qt + 1) / 2 + kt) * kQTile);
        mbar_arrive_expect_tx(BAR(5 + st), 32768);
        tma_load_2d(sBT0 + st * 32768, &tmBT, BAR(5 + st), 0, prow);
        tma_load_2d(sBT0 + st * 32768 + 16384, &tmBT, BAR(5 + st), 64, prow);
      }
    }
  } else if (warp == kSiluWarpsB + 1) {
    // ---------------- tcgen05 issuer ----------------
    // Per query tile s, in two halves of 64 queries: S^T_h = K Q_h^T and dA^T_h = V dO_h^T, then,
    // once the elementwise warps of half h have written P^T_h (TMEM) and dX^T_h (shared memory),
    // dV += P^T_h dO_h and dK += dX^T_h Q_h; after half b also dQ_tile = dX K. The next tile's half a
    // is issued between the two halves, so each half's elementwise work overlaps MMAs.
    if (lane == 0) {
      constexpr uint32_t id_s = make_idesc_f16kind(128, 64, 0, 0, F16);
      constexpr uint32_t id_kmn = make_idesc_f16kind(128, 64, 0, 1, F16);
      constexpr uint32_t id_mnmn = make_idesc_f16kind(128, 64, 1, 1, F16);
      bool ok = mbar_wait(BAR(0), 0, abort_flag, ctl);
      auto issue_s = [&](int s, int h) -> bool {
        const int st = s & 1;
        if (h == 0 && !mbar_wait(BAR(1 + st), (s >> 1) & 1, abort_flag, ctl)) return false;
        tc_fence_after();
        const uint32_t sQ = sQ0 + st * 32768 + 8192 * h, sDO = sQ0 + st * 32768 + 16384 + 8192 * h;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_f16_ss(tmem + 128 * h, make_sdesc_sw128(sK + kk * 32, 16, 1024),
                      make_sdesc_sw128(sQ + kk * 32, 16, 1024), id_s, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_f16_ss(tmem + 128 * h + 64, make_sdesc_sw128(sV + kk * 32, 16, 1024),
                      make_sdesc_sw128(sDO + kk * 32, 16, 1024), id_s, kk > 0 ? 1u : 0u);
        umma_commit(BAR(9 + h));
        return true;
      };
      auto issue_grad = [&](int s, int h) -> bool {
        if (!mbar_wait(BAR(11 + h), s & 1, abort_flag, ctl)) return false;
        tc_fence_after();
        const int st = s & 1;
        const uint32_t sQ = sQ0 + st * 32768, sDO = sQ + 16384, sDX = sBT0 + st * 32768;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4)   // dV += P^T_h dO_h
          umma_f16_ts(tDV, tmem + 128 * h + 8 * k4, make_sdesc_sw128(sDO + (4 * h + k4) * 2048, 16384, 1024),
                      id_kmn, (s > 0 || h > 0 || k4 > 0) ? 1u : 0u);
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4)   // dK += dX^T_h Q_h
          umma_f16_ss(tDK, make_sdesc_sw128(sDX + h * 16384 + k4 * 32, 16, 1024),
                      make_sdesc_sw128(sQ + (4 * h + k4) * 2048, 16384, 1024), id_kmn,
                      (s > 0 || h > 0 || k4 > 0) ? 1u : 0u);
        return true;
      };
      if (ok && nsteps > 0) ok = issue_s(0, 0) && issue_s(0, 1);
      for (int s = 0; ok && s < nsteps; ++s) {
        const int st = s & 1;
        if (!issue_grad(s, 0) || (s + 1 < nsteps && !issue_s(s + 1, 0)) || !issue_grad(s, 1)) {
          ok = false;
          break;
        }
        const uint32_t sDX = sBT0 + st * 32768;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)   // dQ_tile = dX K
          umma_f16_ss(tDQ, make_sdesc_sw128(sDX + kk * 2048, 16384, 1024),
                      make_sdesc_sw128(sK + kk * 2048, 16384, 1024), id_mnmn, kk > 0 ? 1u : 0u);
        umma_commit(BAR(13));
        umma_commit(BAR(3 + st));
        umma_commit(BAR(7 + st));
        if (s + 1 < nsteps && !issue_s(s + 1, 1)) { ok = false; break; }
      }
      if (ok) umma_commit(BAR(14));
    }
  } else if (warp == kSiluWarpsB + 2) {
    // ---------------- dX^T store ----------------
    // Once both query halves of tile s are done, dX^T (the fp16 operand of dK and dQ, in the stage's
    // bias slot) goes to the workspace; the table gradients are summed from there over the heads.
    if (lane == 0) {
      for (int s = 0; s < nsteps; ++s) {
        const int st = s & 1;
        if (!mbar_wait(BAR(15 + st), (s >> 1) & 1, abort_flag, ctl)) break;
        const int qt = kt + s;
        const long long pair = pbase + static_cast<long long>(qt) * (qt + 1) / 2 + kt;
        const int y = static_cast<int>((pair * a.H + h) * kQTile);
        tma_store_2d(&tmDX, sBT0 + st * 32768, 0, y);
        tma_store_2d(&tmDX, sBT0 + st * 32768 + 16384, 64, y);
        bulk_commit_group();
        bulk_wait_group_read<0>();
        mbar_arrive(BAR(7 + st));
      }
      bulk_wait_group_all();
    }
  } else {
    // ---------------- elementwise warps ----------------
    const int quad = warp & 3;
    const int hq = warp >> 2;             // queries [64 hq, 64 hq + 64)
    const int rj = quad * 32 + lane;      // key row == TMEM lane of S^T, dA^T, dV, dK
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const bool key_ok = kt * kQTile + rj < n;
    const float inv_N = a.inv_N;
    bool ok = true;
    auto flush_dq = [&](int s_prev) {
      // (half-b warps) dQ tile of query tile kt + s_prev: TMEM lane = query row, all 64 columns
      const int qi = (kt + s_prev) * kQTile + quad * 32 + lane;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tDQ + lane_base + 32 * c, v);
        tmem_ld_wait();
        if (qi < n) {
          float4* dst = reinterpret_cast<float4*>(A.dq + (seq0 + qi) * A.ld_g + h * kD + 32 * c);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            atomicAdd(dst + q, make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                           __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3])));
        }
      }
    };
    for (int s = 0; ok && s < nsteps; ++s) {
      const int qt = kt + s, st = s & 1;
      if (!mbar_wait(BAR(5 + st), (s >> 1) & 1, abort_flag, ctl) ||
          !mbar_wait(BAR(9 + hq), s & 1, abort_flag, ctl)) {
        ok = false;
        break;
      }
      // half b starts after the MMAs of the previous tile's dQ: flushing it here costs no wait
      if (hq == 1 && s >= 1) {
        if (!mbar_wait(BAR(13), (s - 1) & 1, abort_flag, ctl)) { ok = false; break; }
        tc_fence_after();
        flush_dq(s - 1);
      }
      tc_fence_after();
      // masks: the diagonal tile keeps queries >= key; the last query tile keeps queries < n; a key
      // row past n keeps nothing (it only occurs in the diagonal tile of the last key tile)
      const bool need_mask = (s == 0) || (qt == nt - 1);
      const int lo_col = (s == 0) ? rj : 0;
      const int hi_col = key_ok ? min(kQTile, n - qt * kQTile) : 0;
      uint8_t* bt_row = smem + Lb::kBT0 + st * 32768 + hq * 16384 + rj * 128;
#pragma unroll 1
      for (int hc = 0; hc < 2; ++hc) {
        const int c0 = 64 * hq + 32 * hc;   // first query column of the chunk
        uint32_t sv[32], dav[32];
        tmem_ld_32x32b_x32(tmem + lane_base + 128 * hq + 32 * hc, sv);
        tmem_ld_32x32b_x32(tmem + lane_base + 128 * hq + 64 + 32 * hc, dav);
        uint32_t hb[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 w = *reinterpret_cast<const uint4*>(bt_row + (((4 * hc + q) ^ (rj & 7)) << 4));
          hb[4 * q] = w.x; hb[4 * q + 1] = w.y; hb[4 * q + 2] = w.z; hb[4 * q + 3] = w.w;
        }
        tmem_ld_wait();
        // per query, in fp32: x = s + bias, sigma(x) = (1 + tanh(x/2)) / 2, P = SiLU(x) = x sigma,
        // dX = dA inv_N SiLU'(x) with SiLU' = sigma + P (1 - sigma); P and dX are rounded once to the
        // MMA operand type. (A packed-fp16 evaluation of SiLU' quantises 1 - sigma near x = 8 and
        // biases the table-gradient sums.)
        uint32_t pp[16], dxp[16];
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
          uint32_t m = 0xFFFFFFFFu;
          if (need_mask) {
            const int col = c0 + 2 * e2;
            m = ((col >= lo_col && col < hi_col) ? 0x0000FFFFu : 0u) |
                ((col + 1 >= lo_col && col + 1 < hi_col) ? 0xFFFF0000u : 0u);
          }
          const float2 hbf = unpack_f16x2(hb[e2]);
          float pv[2], dv2[2];
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const float xs = __uint_as_float(sv[2 * e2 + x]) + 2.0f * (x ? hbf.y : hbf.x);
            const float sg = fmaf(0.5f, tanh_f32_approx(0.5f * xs), 0.5f);
            const float av = xs * sg;
            const bool keep = (m >> (16 * x)) & 1u;
            pv[x] = keep ? av : 0.0f;
            dv2[x] = keep ? __uint_as_float(dav[2 * e2 + x]) * inv_N * fmaf(av, 1.0f - sg, sg) : 0.0f;
          }
          if (F16) {
            pp[e2] = pack_f16x2(pv[0], pv[1]);
            dxp[e2] = pack_f16x2(dv2[0], dv2[1]);
          } else {   // the MMAs take A and B of one type: P and dX as bf16 next to bf16 dO, Q, K
            pp[e2] = pack_bf16x2(pv[0], pv[1]);
            dxp[e2] = pack_bf16x2(dv2[0], dv2[1]);
          }
        }
        tmem_st_32x32b_x16(tmem + lane_base + 128 * hq + 16 * hc, pp);
        // dX^T replaces the half-bias just read: same row, same swizzled 16-byte units
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(bt_row + (((4 * hc + q) ^ (rj & 7)) << 4)) =
              make_uint4(dxp[4 * q], dxp[4 * q + 1], dxp[4 * q + 2], dxp[4 * q + 3]);
      }
      tmem_st_wait();
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(BAR(11 + hq));    // P^T_h in TMEM, dX^T_h in shared memory
      mbar_arrive(BAR(15 + st));
    }
    if (ok && hq == 1 && nsteps > 0 && mbar_wait(BAR(13), (nsteps - 1) & 1, abort_flag, ctl)) {
      tc_fence_after();
      flush_dq(nsteps - 1);
    }
    if (ok && mbar_wait(BAR(14), 0, abort_flag, ctl)) {
      tc_fence_after();
      uint32_t vk[32], vv[32];
      tmem_ld_32x32b_x32(tDK + lane_base + 32 * hq, vk);
      tmem_ld_32x32b_x32(tDV + lane_base + 32 * hq, vv);
      tmem_ld_wait();
      if (key_ok) {
        const long long row = seq0 + kt * kQTile + rj;
        float4* dk = reinterpret_cast<float4*>(A.dk + row * A.ld_g + h * kD + 32 * hq);
        float4* dvp = reinterpret_cast<float4*>(A.dv + row * A.ld_g + h * kD + 32 * hq);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          dk[q] = make_float4(__uint_as_float(vk[4 * q]), __uint_as_float(vk[4 * q + 1]),
                              __uint_as_float(vk[4 * q + 2]), __uint_as_float(vk[4 * q + 3]));
          dvp[q] = make_float4(__uint_as_float(vv[4 * q]) * inv_N, __uint_as_float(vv[4 * q + 1]) * inv_N,
                               __uint_as_float(vv[4 * q + 2]) * inv_N, __uint_as_float(vv[4 * q + 3]) * inv_N);
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
// table gradients from the per-head dX^T tiles
// ----------------------------------------------------------------------------------------------
// Two blocks per causal tile pair, 64 key rows each. Thread (warp w, lane l) holds the fp32 head
// sum of key rows j_k = 64 y + 8 w + 2 k + l / 16 (k < 4), queries [c0, c0 + 8), c0 = 8 (l % 16).
//  d rab_pos: element (j, i) of the tile lies on diagonal i - j + 127 (relative position
//   128 (qt - kt) + i - j). A thread's 32 elements fall on 14 diagonals (e - 2k = const), summed in
//   registers first; in each of the 14 steps the 32 lanes of a warp touch 32 distinct diagonals, so
//   every warp adds into its own window without atomics. The 8 windows are summed and added to
//   the table, one atomic per diagonal.
//  d rab_time: each thread's elements in row-major order form runs of equal bucket (along a key
//   row the bucket only grows when timestamps are sorted); a run is added to column l of a
//   [bucket][lane] shared histogram, whose rows are then summed and added to the table.
constexpr int kTgThreads = 256;

template <bool F16>
__global__ void __launch_bounds__(kTgThreads)
attn_table_grad_kernel(AttnBwdArgs A) {
  const AttnArgs& a = A.f;
  int b, qt, kt;
  if (!decode_tile_pair(blockIdx.x, a.pair_base, a.B, &b, &qt, &kt)) return;
  __shared__ float s_win[8][256];
  __shared__ float s_hist[128][32];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int e = tid; e < 8 * 256; e += kTgThreads) (&s_win[0][0])[e] = 0.0f;
  for (int e = tid; e < 128 * 32; e += kTgThreads) (&s_hist[0][0])[e] = 0.0f;
  const int g = lane >> 4, c0 = 8 * (lane & 15);
  const int j0 = 64 * static_cast<int>(blockIdx.y) + 8 * w + g;   // row of k = 0; row k is j0 + 2k
  const long long pair = blockIdx.x;
  const uint16_t* src = reinterpret_cast<const uint16_t*>(A.dxt) + pair * a.H * (kQTile * kQTile) +
                        static_cast<long long>(j0) * kQTile + c0;
  float acc[4][8];
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[k][e] = 0.0f;
  auto add = [&](int k, const uint4& v) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float2 f;
      if (F16) {
        f = unpack_f16x2(u[q]);
      } else {
        f = make_float2(__uint_as_float(u[q] << 16), __uint_as_float(u[q] & 0xFFFF0000u));
      }
      acc[k][2 * q] += f.x;
      acc[k][2 * q + 1] += f.y;
    }
  };
  int h = 0;
  for (; h + 2 <= a.H; h += 2) {
    uint4 v0[4], v1[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v0[k] = __ldg(reinterpret_cast<const uint4*>(src + (static_cast<long long>(h) * kQTile + 2 * k) * kQTile));
      v1[k] = __ldg(reinterpret_cast<const uint4*>(src + (static_cast<long long>(h + 1) * kQTile + 2 * k) * kQTile));
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      add(k, v0[k]);
      add(k, v1[k]);
    }
  }
  if (h < a.H) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      add(k, __ldg(reinterpret_cast<const uint4*>(src + (static_cast<long long>(h) * kQTile + 2 * k) * kQTile)));
  }
  // buckets of the same 32 elements
  const uint8_t* bsrc = reinterpret_cast<const uint8_t*>(A.bucket_t) + pair * (kQTile * kQTile) +
                        static_cast<long long>(j0) * kQTile + c0;
  uint32_t bk[4][2];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(bsrc + 2 * k * kQTile));
    bk[k][0] = v.x;
    bk[k][1] = v.y;
  }
  __syncthreads();   // windows and histogram zeroed
  // d rab_pos: diagonal of (k, e) is c0 - j0 + 127 + (e - 2k)
  float pd[14];
#pragma unroll
  for (int m = 0; m < 14; ++m) pd[m] = 0.0f;
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int e = 0; e < 8; ++e) pd[e - 2 * k + 6] += acc[k][e];
  const int dbase = c0 - j0 + 127 - 6;   // diagonal of slot 0, in [-6, 254 - 13]
#pragma unroll
  for (int m = 0; m < 14; ++m) {
    const int d = dbase + m;
    if (d >= 0 && d < 255) s_win[w][d] += pd[m];
    __syncwarp();
  }
  // d rab_time: runs of equal bucket, in row-major order
  {
    int cur = static_cast<int>(bk[0][0] & 0x7Fu);
    float run = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int bb = static_cast<int>((bk[k][e >> 2] >> (8 * (e & 3))) & 0x7Fu);   // buckets < 128
        if (bb != cur) {
          if (run != 0.0f) atomicAdd(&s_hist[cur][lane], run);
          cur = bb;
          run = 0.0f;
        }
        run += acc[k][e];
      }
    if (run != 0.0f) atomicAdd(&s_hist[cur][lane], run);
  }
  __syncthreads();
  const int L = a.pos_max_len;
  if (tid < 255) {
    float v = 0.0f;
#pragma unroll
    for (int ww = 0; ww < 8; ++ww) v += s_win[ww][tid];
    if (v != 0.0f)
      atomicAdd(A.drab_pos + pos_index_b(static_cast<long long>(qt - kt) * kQTile + tid - 127, L), v);
  }
  if (tid < a.n_buckets) {
    float v = 0.0f;
#pragma unroll 8
    for (int l = 0; l < 32; ++l) v += s_hist[tid][(l + tid) & 31];
    if (v != 0.0f) atomicAdd(A.drab_time + tid, v);
  }
}

}  // namespace

cudaError_t attn_bwd_tc(const AttnBwdArgs& A, cudaStream_t st) {
  const AttnArgs& a = A.f;
  cudaError_t e = upload_time_taus();
  if (e != cudaSuccess) return e;
  if (a.T == 0 || a.capacity == 0) return cudaSuccess;
  const int mt = (a.max_len + kQTile - 1) / kQTile;
  if (mt == 0) return cudaSuccess;
  attn_bias_t_kernel<<<dim3(static_cast<unsigned>(a.max_pairs), 4), 256, 0, st>>>(A);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // TMA row coordinates of the bias and dX^T tiles are 32-bit
  if (a.max_pairs * a.H * kQTile > 0x7fffffffLL) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv, tdo, tbt, tdx;
  const bool f16 = a.in_f16 != 0;
  const int64_t W = static_cast<int64_t>(a.H) * kD;
  if (!encode_tmap_2d_bf16(&tq, a.q, W, a.T, a.ld_q, 64, 128, f16) ||
      !encode_tmap_2d_bf16(&tk, a.k, W, a.T, a.ld_k, 64, 128, f16) ||
      !encode_tmap_2d_bf16(&tv, a.v, W, a.T, a.ld_v, 64, 128, f16) ||
      !encode_tmap_2d_bf16(&tdo, A.dout, W, a.T, A.ld_do, 64, 128, f16) ||
      !encode_tmap_2d_bf16(&tbt, A.bias_t, kQTile, a.max_pairs * kQTile, kQTile, 64, 128, true) ||
      !encode_tmap_2d_bf16(&tdx, A.dxt, kQTile, a.max_pairs * a.H * kQTile, kQTile, 64, 128, f16))
    return cudaErrorInvalidValue;
  auto kern = f16 ? attn_bwd_tc_kernel<true> : attn_bwd_tc_kernel<false>;
  e = ensure_smem_attr(reinterpret_cast<const void*>(kern), BwdSmem::kTotal);
  if (e != cudaSuccess) return e;
  const long long blocks = a.capacity * a.H;
  kern<<<static_cast<unsigned>(blocks), kThreadsB, BwdSmem::kTotal, st>>>(tq, tk, tv, tdo, tbt, tdx, A,
                                                                          wait_ctl(a.status));
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  auto tg = f16 ? attn_table_grad_kernel<true> : attn_table_grad_kernel<false>;
  tg<<<dim3(static_cast<unsigned>(a.max_pairs), 2), kTgThreads, 0, st>>>(A);
  return cudaGetLastError();
}

}  // namespace hstu
