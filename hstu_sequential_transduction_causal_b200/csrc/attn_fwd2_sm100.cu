// attn_fwd2_sm100.cu - jagged causal pointwise attention forward, tensor-core kernel.
//
//   O_i = sum_{j <= i, same sequence} SiLU(q_i . k_j + rab_pos[i-j] + rab_time[bucket(t_i - t_j)])
//         * inv_N * v_j                                                   (per head)
// ("4.4 Scaling Recommendation Models", Generative Recommenders and HSTU: second equation and the
// pointwise-aggregation bullet; "HSTU: The First Exploration of the Scaling Law", 7.1.4
// Innovation 1 (SiLU instead of softmax, no 1/sqrt(d)) and Innovation 2 (position and time bias).)
//
// Two kernels:
//  1. attn_bias_kernel: for every causal (query tile, key tile) pair of every sequence, the
//     relative bias 0.5 * (rab_pos[i-j] + rab_time[bucket(t_i - t_j)]) as an fp16 128x128 tile in
//     the workspace. The bias does not depend on the head, so it is computed once per pair
//     instead of once per pair and head; buckets are exact integer evaluations.
//  2. attn_fwd_tc2_kernel<F16, G>: one CTA per (sequence, 128-row query tile, group of G heads),
//     longest causal rows first; only key tiles 0..t of the tile's own sequence are visited.
//       K/V warp : TMA producer: Q of the G heads once; per (key tile, head) K and V in separate
//                  rings: a K stage is free once its S MMA has run and a V stage once its P V MMA
//                  has, so K loads run several tiles ahead of the (later) V loads and TMA latency
//                  stays hidden; all 128-byte swizzled.
//       bias warp: TMA producer of the bias tiles (one per key tile), so that waiting for a bias
//                  stage (freed by the SiLU warps) never delays a K or V load.
//       MMA warps: two tcgen05 issuing threads. One issues S = Q K^T into one of three TMEM tiles
//                  (the tile of unit s - 3 once its P V has completed), the other O_h += P V with
//                  the A operand P read from TMEM (P overwrites the S tile it came from); neither
//                  waits behind the other's barriers, so the S MMAs of later units overlap SiLU.
//       SiLU warps (8 per group, NG groups, numbered first; then the K/V, MMA and bias warps):
//                  TMEM lane quadrant (warp & 3), key half (warp >> 2) & 1. Per element, in packed
//                  fp16: h = 0.5 s + 0.5 bias, P = h + h tanh(h) = SiLU(s + bias); causal mask on
//                  the diagonal tile only; P back into TMEM.
//     1/N is applied to the fp32 accumulator in the epilogue; O is written in fp32 (or bf16).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "hstu_internal.h"
#include "sm100_ptx.cuh"
#include "tile_pairs.cuh"
#include "time_bucket_dev.cuh"
#include "bias_tile.cuh"

namespace hstu {

namespace {

constexpr int kD = 64;
constexpr int kSiluWarps = 8;     // one group of SiLU warps: 4 TMEM lane quadrants x 2 key halves
__host__ __device__ constexpr int threads2(int ng) { return 32 * (kSiluWarps * ng + 4); }
constexpr uint32_t kHalf2Half = 0x38003800u;   // (0.5, 0.5) in fp16

// ----------------------------------------------------------------------------------------------
// 1. bias tiles
// ----------------------------------------------------------------------------------------------
// Four blocks per causal tile pair (blocks past the batch's last pair exit at once): the [query][key]
// half-bias tile of bias_tile.cuh.
__global__ void __launch_bounds__(kBiasThreads)
attn_bias_kernel(AttnArgs a) {
  bias_tiles<false, false>(a, reinterpret_cast<uint16_t*>(a.bias), nullptr);
}

// ----------------------------------------------------------------------------------------------
// 2. attention
// ----------------------------------------------------------------------------------------------
template <int G>
struct Smem2 {
  static constexpr int kBS = G == 1 ? 3 : 2;   // bias stages (one head per CTA: a bias tile per unit)
  static constexpr int kNK = G == 1 ? 4 : 3;   // K stages (16 KB)
  static constexpr int kNV = 3;                // V stages (16 KB)
  static constexpr int kQ = 0;
  static constexpr int kK = G * 16384;
  static constexpr int kV = kK + kNK * 16384;
  static constexpr int kBias = kV + kNV * 16384;
  static constexpr int kBar = kBias + kBS * 32768;
  static constexpr int kTotal = kBar + 256 + 1024;
};
static_assert(Smem2<1>::kTotal <= 232448 && Smem2<2>::kTotal <= 232448, "shared memory of the attention kernel");

// NG = 2 (one head per CTA only): two groups of SiLU warps take alternate key tiles, so one group's
// SiLU of tile t overlaps the other's of tile t + 1 (each group owns one S buffer and one bias stage).
template <bool F16, int G, bool FALCON, int NG>
__global__ void __launch_bounds__(threads2(NG), 1)
attn_fwd_tc2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmB, AttnArgs a,
                    WaitCtl ctl) {
  pdl_enter();
  using L = Smem2<G>;
  static_assert(NG == 1 || G == 1, "two SiLU groups need one head per CTA");
  constexpr int kTmaWarp = kSiluWarps * NG, kMmaWarp = kTmaWarp + 1, kBiasWarp = kTmaWarp + 2;
  constexpr int kPvWarp = kTmaWarp + 3;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int HG = a.H / G;
  const int item = blockIdx.x / HG;
  const int hg = blockIdx.x - item * HG;
  int b, qt;
  if constexpr (FALCON) {
    // (user, candidate tile): every tile of a user visits all of the user's prefix key tiles
    const int qpu = (a.cand_rows + kQTile - 1) / kQTile;
    if (qpu == 0 || item >= a.B * qpu) return;
    b = item / qpu;
    qt = item - b * qpu;
  } else {
    if (item >= *a.count) return;
    b = a.items[2 * item];
    qt = a.items[2 * item + 1];
  }
  const long long seq0 = a.offsets[b];
  const int n = static_cast<int>(a.offsets[b + 1] - seq0);
  // FALCON: keys past the bias row (a prefix longer than its contract allows) are not visited
  const int nkt = FALCON ? max(0, min((n + kQTile - 1) / kQTile, static_cast<int>(a.kbias_ld / kQTile))) : qt + 1;
  const int nsteps = nkt * G;
  const long long pair0 = FALCON ? 0 : a.pair_base[b] + static_cast<long long>(qt) * (qt + 1) / 2;

  constexpr int BS = L::kBS, NK = L::kNK, NV = L::kNV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  // 0 q_full | k_full [NK] | k_empty [NK] | v_full [NV] | v_empty [NV] | b_full [BS] | b_empty [BS] |
  // s_full [3] | p_full [3] | o_full
  constexpr int kBarK = 1, kBarV = kBarK + 2 * NK, kBarB = kBarV + 2 * NV, kBarS = kBarB + 2 * BS;
  constexpr int kBarP = kBarS + 3, kBarO = kBarP + 3, kBarPv = kBarO + 1, kNumBars = kBarPv + 3;
  static_assert(kNumBars * 8 + 8 <= 256, "barrier region");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t bar0 = smem_u32(bars);
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  const uint32_t bar_q = BAR(0), bar_o = BAR(kBarO);
  auto bar_pv_done = [&](int b) { return BAR(kBarPv + b); };   // P V of the unit in TMEM tile b done
  auto bar_k_full = [&](int s) { return BAR(kBarK + s); };
  auto bar_k_empty = [&](int s) { return BAR(kBarK + NK + s); };
  auto bar_v_full = [&](int s) { return BAR(kBarV + s); };
  auto bar_v_empty = [&](int s) { return BAR(kBarV + NV + s); };
  auto bar_b_full = [&](int s) { return BAR(kBarB + s); };
  auto bar_b_empty = [&](int s) { return BAR(kBarB + BS + s); };
  auto bar_s_full = [&](int s) { return BAR(kBarS + s); };
  auto bar_p_full = [&](int s) { return BAR(kBarP + s); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int kSiluThreads = 32 * kSiluWarps;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < NK; ++s) {
      mbar_init(bar_k_full(s), 1);
      mbar_init(bar_k_empty(s), 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(bar_v_full(s), 1);
      mbar_init(bar_v_empty(s), 1);
    }
    for (int s = 0; s < BS; ++s) {
      mbar_init(bar_b_full(s), 1);
      mbar_init(bar_b_empty(s), kSiluThreads);
    }
    for (int s = 0; s < 3; ++s) {
      mbar_init(bar_s_full(s), 1);
      mbar_init(bar_p_full(s), kSiluThreads);
    }
    mbar_init(bar_o, 1);
    for (int b3 = 0; b3 < 3; ++b3) mbar_init(bar_pv_done(b3), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if (!FALCON) tma_prefetch_desc(&tmB);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // S / P tiles of units s = 0, 1, 2 (mod 3) at columns [128 (s % 3), +128): with three of them the S
  // MMA of unit s is issued before the P V MMA of unit s - 2; O_h at [384 + 64 h, +64)
  const uint32_t tmem = *tmem_slot;
  constexpr uint32_t kOCol = 384;

  const uint32_t sQ = smem_u32(smem + L::kQ);
  const uint32_t sK = smem_u32(smem + L::kK), sV = smem_u32(smem + L::kV);
  const uint32_t sB = smem_u32(smem + L::kBias);
  const int qrow0 = FALCON ? b * a.cand_rows + qt * kQTile : static_cast<int>(seq0) + qt * kQTile;

  if (warp == kTmaWarp) {
    // ---------------- TMA producer: K stage st from lane st, V stage st from lane 8 + st ----------------
    if (lane == 0) mbar_arrive_expect_tx(bar_q, G * 16384);
    __syncwarp();
    if (lane < G) tma_load_2d(sQ + lane * 16384, &tmQ, bar_q, (hg * G + lane) * kD, qrow0);
    // unit s = (key tile s / G, head s % G): K(s) first, V(s - 1) after it, so waiting for a V
    // stage (freed late, by a P V MMA) never delays a K load
    auto load_v = [&](int s) -> bool {
      const int st = s % NV;
      if (s >= NV && !mbar_wait_warp(bar_v_empty(st), ((s / NV) - 1) & 1, abort_flag, ctl)) return false;
      if (lane == 8 + st) {
        mbar_arrive_expect_tx(bar_v_full(st), 16384);
        tma_load_2d(sV + st * 16384, &tmV, bar_v_full(st), (hg * G + s % G) * kD,
                    static_cast<int>(seq0) + (s / G) * kQTile);
      }
      return true;
    };
    bool ok = true;
    for (int s = 0; ok && s < nsteps; ++s) {
      const int kt = s / G, h = s % G;
      const int st = s % NK;
      if (s >= NK && !mbar_wait_warp(bar_k_empty(st), ((s / NK) - 1) & 1, abort_flag, ctl)) break;
      if (lane == st) {
        mbar_arrive_expect_tx(bar_k_full(st), 16384);
        tma_load_2d(sK + st * 16384, &tmK, bar_k_full(st), (hg * G + h) * kD, static_cast<int>(seq0) + kt * kQTile);
      }
      if (s >= 1) ok = load_v(s - 1);
    }
    if (ok && nsteps > 0) load_v(nsteps - 1);
  } else if (warp == kBiasWarp) {
    // ---------------- bias tiles (stage bs: its two 64-column halves from lanes 2 bs, 2 bs + 1) ----
    if (!FALCON) {
      for (int kt = 0; kt < nkt; ++kt) {
        const int bs = kt % BS;
        if (kt >= BS && !mbar_wait_warp(bar_b_empty(bs), ((kt / BS) - 1) & 1, abort_flag, ctl)) break;
        const int brow = static_cast<int>((pair0 + kt) * kQTile);
        if (lane == 0) mbar_arrive_expect_tx(bar_b_full(bs), 32768);
        __syncwarp();
        const int hx = lane - 2 * bs;
        if (hx == 0 || hx == 1) tma_load_2d(sB + bs * 32768 + hx * 16384, &tmB, bar_b_full(bs), 64 * hx, brow);
      }
    }
  } else if (warp == kMmaWarp || warp == kPvWarp) {
    // ---------------- tcgen05 issuers: S = Q K^T (one thread), O_h += P V (another) ----------------
    // Two issuing threads keep the tensor pipe fed: neither waits behind the other's barrier. S of
    // unit s reuses the TMEM tile of unit s - 3, so it waits for that unit's P V to have completed.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = make_idesc_f16kind(128, 128, 0, 0, F16);
      constexpr uint32_t idesc_pv = make_idesc_f16kind(128, 64, 0, 1, F16);
      bool ok = true;
      if (warp == kMmaWarp) {
        ok = mbar_wait(bar_q, 0, abort_flag, ctl);
        const uint64_t q_desc0 = make_sdesc_sw128(sQ, 16, 1024), k_desc0 = make_sdesc_sw128(sK, 16, 1024);
        for (int s = 0; ok && s < nsteps; ++s) {
          const int buf = s % 3, st = s % NK, h = s % G;
          if (!mbar_wait(bar_k_full(st), (s / NK) & 1, abort_flag, ctl) ||
              (s >= 3 && !mbar_wait(bar_pv_done(buf), ((s / 3) - 1) & 1, abort_flag, ctl))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t qd = sdesc_add(q_desc0, h * 16384), kd = sdesc_add(k_desc0, st * 16384);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f16_ss(tmem + buf * 128, sdesc_add(qd, kk * 32), sdesc_add(kd, kk * 32), idesc_qk, kk > 0 ? 1u : 0u);
          umma_commit(bar_s_full(buf));
          umma_commit(bar_k_empty(st));
        }
      } else {
        const uint64_t v_desc0 = make_sdesc_sw128(sV, 16384, 1024);
        for (int t = 0; ok && t < nsteps; ++t) {
          const int buf = t % 3, st = t % NV, h = t % G;
          if (!mbar_wait(bar_p_full(buf), (t / 3) & 1, abort_flag, ctl) ||
              !mbar_wait(bar_v_full(st), (t / NV) & 1, abort_flag, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t vd = sdesc_add(v_desc0, st * 16384);
          const uint32_t a_tmem = tmem + buf * 128, o_tmem = tmem + kOCol + 64 * h;
          const uint32_t acc0 = t >= G ? 1u : 0u;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_f16_ts(o_tmem, a_tmem + 64 * (kk >> 2) + 8 * (kk & 3), sdesc_add(vd, kk * 2048), idesc_pv,
                        kk > 0 ? 1u : acc0);
          umma_commit(bar_v_empty(st));
          umma_commit(bar_pv_done(buf));
        }
        if (ok && nsteps > 0) umma_commit(bar_o);
      }
    }
  } else {
    // ---------------- SiLU warps ----------------
    const int grp = warp / kSiluWarps;   // NG == 2: group g takes key tiles g, g + 2, ...
    const int quad = warp & 3;
    const int half = (warp >> 2) & 1;    // keys [64 half, 64 half + 64)
    const int r = quad * 32 + lane;      // query row within the tile == TMEM lane
    const int qi = qt * kQTile + r;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    bool ok = true;
    for (int kt = grp; ok && kt < nkt; kt += NG) {
      const int bs = kt % BS;
      if constexpr (!FALCON) {
        if (!mbar_wait(bar_b_full(bs), (kt / BS) & 1, abort_flag, ctl)) { ok = false; break; }
      }
      // FALCON: keys past the user's prefix (last tile) are masked; causal: the diagonal tile
      const int key_lim = FALCON ? n - kt * kQTile : 0;
      const bool diag = FALCON ? key_lim < kQTile : (kt == qt);
      for (int h = 0; h < G; ++h) {
        const int s = kt * G + h;
        const int buf = s % 3;
        if (!mbar_wait(bar_s_full(buf), (s / 3) & 1, abort_flag, ctl)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
          uint32_t sv[32];
          tmem_ld_32x32b_x32(tmem + lane_base + buf * 128 + 64 * half + 32 * hc, sv);
          uint32_t hb[16];   // half-bias of keys [64 half + 32 hc, +32)
          if constexpr (FALCON) {
            // the bias depends on the key only: one row shared by every query row
            const uint4* src =
                reinterpret_cast<const uint4*>(a.kbias + b * a.kbias_ld + kt * kQTile + 64 * half + 32 * hc);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint4 v = __ldg(src + u);
              hb[4 * u] = v.x; hb[4 * u + 1] = v.y; hb[4 * u + 2] = v.z; hb[4 * u + 3] = v.w;
            }
          } else {
            const uint8_t* brow = smem + L::kBias + bs * 32768 + half * 16384 + r * 128;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint4 v = *reinterpret_cast<const uint4*>(brow + (((4 * hc + u) ^ (r & 7)) << 4));
              hb[4 * u] = v.x; hb[4 * u + 1] = v.y; hb[4 * u + 2] = v.z; hb[4 * u + 3] = v.w;
            }
            // one head: the bias stage is free once both halves of its row are in registers
            if (G == 1 && hc == 1) mbar_arrive(bar_b_empty(bs));
          }
          tmem_ld_wait();
          uint32_t p[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const uint32_t s2 = pack_f16x2(__uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1]));
            const uint32_t h2 = hfma2_u32(s2, kHalf2Half, hb[j]);
            const uint32_t t2 = tanh_f16x2(h2);
            uint32_t y2 = hfma2_u32(h2, t2, h2);
            if (!F16) {   // the P V MMA takes A and B of one type: P as bf16 next to bf16 V
              const float2 f = unpack_f16x2(y2);
              y2 = pack_bf16x2(f.x, f.y);
            }
            if (diag) {
              const int col = 64 * half + 32 * hc + 2 * j;
              const int lim = FALCON ? key_lim - 1 : r;    // last key column kept
              const uint32_t m = (col + 1 <= lim) ? 0xFFFFFFFFu : ((col <= lim) ? 0x0000FFFFu : 0u);
              y2 &= m;
            }
            p[j] = y2;
          }
          // P of these 32 keys packed into 16 columns over S chunk 0 (already read)
          tmem_st_32x32b_x16(tmem + lane_base + buf * 128 + 64 * half + 16 * hc, p);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar_p_full(buf));
      }
      if constexpr (!FALCON && G > 1) mbar_arrive(bar_b_empty(bs));
    }
    if (grp > 0) ok = false;   // the epilogue is group 0's
    if (ok && (nkt == 0 || mbar_wait(bar_o, 0, abort_flag, ctl))) {
      tc_fence_after();
      // G == 1: both key halves split head 0's 64 columns; G >= 2: half c handles heads c, c+2, ...
      constexpr int kHeadsPerWarp = G == 1 ? 1 : G / 2;
      constexpr int kCols = G == 1 ? 32 : 64;
      const float sc = a.inv_N;
      const bool row_ok = FALCON ? qi < a.cand_rows : qi < n;
      const long long orow = FALCON ? static_cast<long long>(b) * a.cand_rows + qi : seq0 + qi;
#pragma unroll 1
      for (int e = 0; e < kHeadsPerWarp; ++e) {
        const int h = G == 1 ? 0 : half + 2 * e;
        const int col0 = G == 1 ? 32 * half : 0;
        float self_a = 0.0f;    // FALCON: SiLU(q_c.k_c + self bias), the candidate's own weight
        if (FALCON && row_ok) {
          const int hc0 = (hg * G + h) * kD;
          const uint4* qp = reinterpret_cast<const uint4*>(
              static_cast<const uint16_t*>(a.q) + orow * a.ld_q + hc0);
          const uint4* kp = reinterpret_cast<const uint4*>(
              static_cast<const uint16_t*>(a.kc) + orow * a.ld_c + hc0);
          float dot = 0.0f;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint4 qv = qp[u], kv = kp[u];
            const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w}, kw[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
            for (int w2 = 0; w2 < 4; ++w2) {
              const float2 qf = F16 ? unpack_f16x2(qw[w2]) : unpack_bf16x2(qw[w2]);
              const float2 kf = F16 ? unpack_f16x2(kw[w2]) : unpack_bf16x2(kw[w2]);
              dot = fmaf(qf.x, kf.x, dot);
              dot = fmaf(qf.y, kf.y, dot);
            }
          }
          const float xs = dot + *a.self_bias;
          self_a = xs / (1.0f + __expf(-xs));
        }
#pragma unroll 1
        for (int cc = 0; cc < kCols; cc += 32) {
          uint32_t ov[32];
          if (nkt > 0) {
            tmem_ld_32x32b_x32(tmem + lane_base + kOCol + 64 * h + col0 + cc, ov);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) ov[q] = 0u;
          }
          if (row_ok) {
            const int ocol = (hg * G + h) * kD + col0 + cc;
            if (FALCON) {   // + SiLU(self) v_c
              const uint4* vp = reinterpret_cast<const uint4*>(
                  static_cast<const uint16_t*>(a.vc) + orow * a.ld_c + ocol);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const uint4 vv = vp[u];
                const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
                for (int w2 = 0; w2 < 4; ++w2) {
                  const float2 vf = F16 ? unpack_f16x2(vw[w2]) : unpack_bf16x2(vw[w2]);
                  ov[8 * u + 2 * w2] = __float_as_uint(fmaf(self_a, vf.x, __uint_as_float(ov[8 * u + 2 * w2])));
                  ov[8 * u + 2 * w2 + 1] =
                      __float_as_uint(fmaf(self_a, vf.y, __uint_as_float(ov[8 * u + 2 * w2 + 1])));
                }
              }
            }
            if (a.o_f32) {
              float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.o) + orow * a.ld_o + ocol);
#pragma unroll
              for (int q = 0; q < 8; ++q)
                dst[q] = make_float4(__uint_as_float(ov[4 * q]) * sc, __uint_as_float(ov[4 * q + 1]) * sc,
                                     __uint_as_float(ov[4 * q + 2]) * sc, __uint_as_float(ov[4 * q + 3]) * sc);
            } else {
              uint4* dst =
                  reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) + orow * a.ld_o + ocol);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                dst[q] = make_uint4(
                    pack_bf16x2(__uint_as_float(ov[8 * q]) * sc, __uint_as_float(ov[8 * q + 1]) * sc),
                    pack_bf16x2(__uint_as_float(ov[8 * q + 2]) * sc, __uint_as_float(ov[8 * q + 3]) * sc),
                    pack_bf16x2(__uint_as_float(ov[8 * q + 4]) * sc, __uint_as_float(ov[8 * q + 5]) * sc),
                    pack_bf16x2(__uint_as_float(ov[8 * q + 6]) * sc, __uint_as_float(ov[8 * q + 7]) * sc));
            }
          }
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
// 3. persistent attention: one CTA per SM pulling (work item, head) units, longest first
// ----------------------------------------------------------------------------------------------
// Unit u = (work item u / H, head u % H): query tile qt of sequence b against key tiles 0..qt. CTAs
// take units from a global counter in list order, so the longest causal rows go first and a CTA that
// finishes early takes the next unit (list scheduling). Every ring below is indexed by the CTA's
// running step count s (one step = one key tile of one unit), so the pipelines run across unit
// boundaries: the next unit's Q and K loads and its first S MMAs are issued while the current
// unit's last tiles are still in SiLU or P V, and the epilogue of a unit (O from TMEM, scaled by
// 1/N) overlaps the next unit's MMAs through a second O accumulator.
//   warps 0-15 : SiLU, two groups of 8 taking alternate steps (group s % 2); each warp one TMEM lane
//                quadrant (warp & 3) and one key half ((warp >> 2) & 1). The group that runs a
//                unit's last step also writes its output.
//   warp 16    : scheduler (lane 0 takes the next unit, publishes it in a two-slot ring) and TMA
//                producer of Q (two buffers) and K (three stages); it takes the next unit as soon as
//                it has issued the current unit's last K load, so the next unit's loads start while
//                the current one computes.
//   warp 17    : tcgen05 issuer of S = Q K^T into three TMEM tiles.
//   warp 18    : TMA producer of the bias tiles and of V (three stages each), per step the bias then
//                V, so that waiting for a V stage (freed by a P V MMA) never holds back a K load or
//                the next unit.
//   warp 19    : tcgen05 issuer of O += P V, P read from TMEM, into two alternating O accumulators.
// (20 warps: five per SM sub-partition leave 96 registers a thread.)
// Every tile is loaded as 8 KB boxes of 64 rows from separate lanes: a thread keeps about one TMA
// copy in flight, and tile loads take thousands of cycles when every SM is loading.
struct Smem3 {
  static constexpr int kNQ = 2, kNK = 3, kNV = 3, kBS = 3;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kNQ * 16384;
  static constexpr int kV = kK + kNK * 16384;
  static constexpr int kBias = kV + kNV * 16384;
  static constexpr int kBar = kBias + kBS * 32768;
  static constexpr int kTotal = kBar + 512 + 1024;
};
static_assert(Smem3::kTotal <= 232448, "shared memory of the persistent attention kernel");

constexpr int kThreads3 = 32 * (2 * kSiluWarps + 4);
constexpr int kUnitConsumers = 2 * kSiluWarps + 3;   // SiLU warps, S issuer, bias / V warp, P V issuer

// A unit as the scheduler publishes it, with everything the other roles need about it (reading
// offsets, pair_base or the pack array from global memory inside the pipeline stalled it by thousands
// of cycles): sequence b, query tile qt (-k for a pack of k short sequences), head h, first row and
// row count of the sequence (or pack), its first causal pair, and the first query row to write.
struct UnitRec {
  int b, qt, h, valid;
  int row0, n, pair0, q_lo;
};

template <bool F16>
__global__ void __launch_bounds__(kThreads3, 1)
attn_fwd_persistent_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmB,
                           AttnArgs a, WaitCtl ctl) {
  // set-up below reads nothing an earlier grid writes: it overlaps that grid's tail
  pdl_trigger();
  using L = Smem3;
  constexpr int NK = L::kNK, NV = L::kNV, BS = L::kBS;
  static_assert(NK == 3 && NV == 3 && BS == 3, "the rings share the step index modulo 3");
  constexpr int kTmaWarp = 2 * kSiluWarps, kSWarp = kTmaWarp + 1, kBiasWarp = kTmaWarp + 2, kPvWarp = kTmaWarp + 3;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  // 0 u_full[2] | 2 u_empty[2] | 4 q_full[2] | 6 q_empty[2] | 8 k_full[3] | 11 k_empty[3] | 14 v_full[3] |
  // 17 v_empty[3] | 20 b_full[3] | 23 b_empty[3] | 26 s_full[3] | 29 p_full[3] | 32 pv_done[3] | 35 o_full[2] |
  // 37 o_empty[2]
  constexpr int kNumBars = 39;
  UnitRec* ring = reinterpret_cast<UnitRec*>(smem + L::kBar + 320);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + 384);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kBar + 388);
  const uint32_t bar0 = smem_u32(bars);
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  auto u_full = [&](int i) { return BAR(0 + i); };
  auto u_empty = [&](int i) { return BAR(2 + i); };
  auto q_full = [&](int i) { return BAR(4 + i); };
  auto q_empty = [&](int i) { return BAR(6 + i); };
  auto k_full = [&](int i) { return BAR(8 + i); };
  auto k_empty = [&](int i) { return BAR(11 + i); };
  auto v_full = [&](int i) { return BAR(14 + i); };
  auto v_empty = [&](int i) { return BAR(17 + i); };
  auto b_full = [&](int i) { return BAR(20 + i); };
  auto b_empty = [&](int i) { return BAR(23 + i); };
  auto s_full = [&](int i) { return BAR(26 + i); };
  auto p_full = [&](int i) { return BAR(29 + i); };
  auto pv_done = [&](int i) { return BAR(32 + i); };
  auto o_full = [&](int i) { return BAR(35 + i); };
  auto o_empty = [&](int i) { return BAR(37 + i); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int kGroupThreads = 32 * kSiluWarps;
  // a unit's query tile and key-tile count: a pack of short sequences (qt = -k) is one diagonal tile
  auto unit_qt = [](int qt) { return qt < 0 ? 0 : qt; };
  auto unit_nkt = [](int qt) { return qt < 0 ? 1 : qt + 1; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(u_full(i), 1);
      mbar_init(u_empty(i), kUnitConsumers);
      mbar_init(q_full(i), 1);
      mbar_init(q_empty(i), 1);
      mbar_init(o_full(i), 1);
      mbar_init(o_empty(i), kGroupThreads);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(k_full(i), 1);
      mbar_init(k_empty(i), 1);
      mbar_init(v_full(i), 1);
      mbar_init(v_empty(i), 1);
      mbar_init(b_full(i), 1);
      mbar_init(b_empty(i), kGroupThreads);
      mbar_init(s_full(i), 1);
      mbar_init(p_full(i), kGroupThreads);
      mbar_init(pv_done(i), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  static_assert(kNumBars * 8 <= 320, "barrier region");
  if (warp == kTmaWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  // S / P tiles of steps s = 0, 1, 2 (mod 3) at columns [128 (s % 3), +128); O of units 0, 1 (mod 2) at
  // [384 + 64 (u % 2), +64)
  const uint32_t tmem = *tmem_slot;
  constexpr uint32_t kOCol = 384;
  const uint32_t sQ = smem_u32(smem + L::kQ), sK = smem_u32(smem + L::kK), sV = smem_u32(smem + L::kV);
  const uint32_t sB = smem_u32(smem + L::kBias);

  // The unit published in ring slot uc % 2 (consumers): lane 0 waits and reads, the warp gets it by
  // shuffles, lane 0 then frees the slot.
  auto take_unit = [&](int uc, UnitRec& r) -> bool {
    const int slot = uc & 1;
    if (!mbar_wait_warp(u_full(slot), (uc >> 1) & 1, abort_flag, ctl)) return false;
    int v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (lane == 0) {
      const UnitRec x = ring[slot];
      v[0] = x.b; v[1] = x.qt; v[2] = x.h; v[3] = x.valid; v[4] = x.row0; v[5] = x.n; v[6] = x.pair0; v[7] = x.q_lo;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __shfl_sync(0xffffffffu, v[i], 0);
    r.b = v[0]; r.qt = v[1]; r.h = v[2]; r.valid = v[3]; r.row0 = v[4]; r.n = v[5]; r.pair0 = v[6]; r.q_lo = v[7];
    __syncwarp();
    if (lane == 0) mbar_arrive(u_empty(slot));
    return true;
  };

  if (warp == kTmaWarp) {
    // ---------------- scheduler + Q / K producer ----------------
    // Units u = item * H + h in work-list order: CTA x starts with unit x, later ones come from the
    // counter (offset by the grid size). One 32-byte record per item (written by the work list)
    // describes the unit; the first record is read together with the item count.
    long long total = 0;
    int4 first0 = make_int4(0, 0, 0, 0), first1 = first0;
    if (lane == 0) {
      const int4* rec = reinterpret_cast<const int4*>(a.urec) + 2 * (blockIdx.x / a.H);
      first0 = rec[0];
      first1 = rec[1];
      total = static_cast<long long>(*a.count) * a.H;
    }
    int sg = 0;
    bool ok = true;
    for (int uc = 0; ok; ++uc) {
      const int slot = uc & 1;
      if (uc >= 2 && !mbar_wait_warp(u_empty(slot), ((uc >> 1) - 1) & 1, abort_flag, ctl)) break;
      int v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (lane == 0) {
        for (bool first = uc == 0;; first = false) {
          const long long u = first ? static_cast<long long>(blockIdx.x)
                                    : static_cast<long long>(gridDim.x) + atomicAdd(a.unit_counter, 1);
          if (u >= total) break;
          const int item = static_cast<int>(u / a.H);
          int4 r0 = first0, r1 = first1;
          if (!first) {
            const int4* rec = reinterpret_cast<const int4*>(a.urec) + 2 * item;
            r0 = rec[0];
            r1 = rec[1];
          }
          const int b = r0.x, qt = r0.y;
          // prefix append: a query tile wholly inside the old prefix has nothing to write
          const long long q_lo = a.q_from ? a.q_from[b + 1] - a.q_from[b] : 0;
          if (static_cast<long long>(unit_qt(qt) + 1) * kQTile <= q_lo) continue;
          v[0] = b;
          v[1] = qt;
          v[2] = static_cast<int>(u - static_cast<long long>(item) * a.H);
          v[3] = 1;
          v[4] = r0.z;
          v[5] = r0.w;
          v[6] = r1.x;
          v[7] = static_cast<int>(q_lo);
          break;
        }
        ring[slot] = UnitRec{v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]};
        mbar_arrive(u_full(slot));
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = __shfl_sync(0xffffffffu, v[i], 0);
      if (!v[3]) break;
      const int qt = unit_qt(v[1]), h = v[2];
      const int row0 = v[4];
      const int nkt = unit_nkt(v[1]);
      const int qb = uc & 1;
      if (uc >= 2 && !mbar_wait_warp(q_empty(qb), ((uc >> 1) - 1) & 1, abort_flag, ctl)) break;
      if (lane == 0) mbar_arrive_expect_tx(q_full(qb), 16384);
      __syncwarp();
      if (lane == 16 + 2 * qb || lane == 17 + 2 * qb) {
        const int ry = lane & 1;
        tma_load_2d(sQ + qb * 16384 + ry * 8192, &tmQ, q_full(qb), h * kD, row0 + qt * kQTile + 64 * ry);
      }
      for (int kt = 0; kt < nkt; ++kt) {
        const int s = sg + kt, st = s % NK;
        if (s >= NK && !mbar_wait_warp(k_empty(st), ((s / NK) - 1) & 1, abort_flag, ctl)) { ok = false; break; }
        if (lane == 0) mbar_arrive_expect_tx(k_full(st), 16384);
        __syncwarp();
        if (lane == 2 * st || lane == 2 * st + 1) {
          const int ry = lane & 1;
          tma_load_2d(sK + st * 16384 + ry * 8192, &tmK, k_full(st), h * kD, row0 + kt * kQTile + 64 * ry);
        }
      }
      sg += nkt;
    }
  } else if (warp == kBiasWarp) {
    // ---------------- bias tiles and V (bias stage: four 8 KB boxes from lanes 4 bs .. 4 bs + 3; V
    // stage: two from lanes 12 + 2 st, 13 + 2 st) ----------------
    int sg = 0;
    bool ok = true;
    UnitRec r;
    for (int uc = 0; ok && take_unit(uc, r) && r.valid; ++uc) {
      const long long pair0 = r.pair0;
      const int nkt = unit_nkt(r.qt);
      const int hb = a.bias_heads > 1 ? r.h : 0;
      const int row0 = r.row0;
      for (int kt = 0; kt < nkt; ++kt) {
        const int s = sg + kt, bs = s % BS;
        if (s >= BS && !mbar_wait_warp(b_empty(bs), ((s / BS) - 1) & 1, abort_flag, ctl)) { ok = false; break; }
        const int brow = static_cast<int>(((pair0 + kt) * a.bias_heads + hb) * kQTile);
        if (lane == 0) mbar_arrive_expect_tx(b_full(bs), 32768);
        __syncwarp();
        const int part = lane - 4 * bs;   // column half part >> 1, row half part & 1
        if (part >= 0 && part < 4)
          tma_load_2d(sB + bs * 32768 + (part >> 1) * 16384 + (part & 1) * 8192, &tmB, b_full(bs), 64 * (part >> 1),
                      brow + 64 * (part & 1));
        const int st = s % NV;
        if (s >= NV && !mbar_wait_warp(v_empty(st), ((s / NV) - 1) & 1, abort_flag, ctl)) { ok = false; break; }
        if (lane == 0) mbar_arrive_expect_tx(v_full(st), 16384);
        __syncwarp();
        if (lane == 12 + 2 * st || lane == 13 + 2 * st) {
          const int ry = lane & 1;
          tma_load_2d(sV + st * 16384 + ry * 8192, &tmV, v_full(st), r.h * kD, row0 + kt * kQTile + 64 * ry);
        }
      }
      sg += nkt;
    }
  } else if (warp == kSWarp) {
    // ---------------- S = Q K^T ----------------
    constexpr uint32_t idesc_qk = make_idesc_f16kind(128, 128, 0, 0, F16);
    const uint64_t q_desc0 = make_sdesc_sw128(sQ, 16, 1024), k_desc0 = make_sdesc_sw128(sK, 16, 1024);
    int sg = 0;
    bool ok = true;
    UnitRec r;
    for (int uc = 0; ok && take_unit(uc, r) && r.valid; ++uc) {
      if (lane == 0) {
        const int qb = uc & 1, nkt = unit_nkt(r.qt);
        ok = mbar_wait(q_full(qb), (uc >> 1) & 1, abort_flag, ctl);
        const uint64_t qd = sdesc_add(q_desc0, qb * 16384);
        for (int kt = 0; ok && kt < nkt; ++kt) {
          const int s = sg + kt, buf = s % 3;
          if (!mbar_wait(k_full(buf), (s / 3) & 1, abort_flag, ctl) ||
              (s >= 3 && !mbar_wait(pv_done(buf), ((s / 3) - 1) & 1, abort_flag, ctl))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t kd = sdesc_add(k_desc0, buf * 16384);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f16_ss(tmem + buf * 128, sdesc_add(qd, kk * 32), sdesc_add(kd, kk * 32), idesc_qk, kk > 0 ? 1u : 0u);
          umma_commit(s_full(buf));
          umma_commit(k_empty(buf));
        }
        if (ok) umma_commit(q_empty(qb));
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      sg += unit_nkt(r.qt);
    }
  } else if (warp == kPvWarp) {
    // ---------------- O += P V ----------------
    constexpr uint32_t idesc_pv = make_idesc_f16kind(128, 64, 0, 1, F16);
    const uint64_t v_desc0 = make_sdesc_sw128(sV, 16384, 1024);
    int sg = 0;
    bool ok = true;
    UnitRec r;
    for (int uc = 0; ok && take_unit(uc, r) && r.valid; ++uc) {
      if (lane == 0) {
        const int ob = uc & 1, nkt = unit_nkt(r.qt);
        if (uc >= 2) ok = mbar_wait(o_empty(ob), ((uc >> 1) - 1) & 1, abort_flag, ctl);
        const uint32_t o_tmem = tmem + kOCol + 64 * ob;
        for (int kt = 0; ok && kt < nkt; ++kt) {
          const int s = sg + kt, buf = s % 3;
          if (!mbar_wait(p_full(buf), (s / 3) & 1, abort_flag, ctl) ||
              !mbar_wait(v_full(buf), (s / 3) & 1, abort_flag, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t vd = sdesc_add(v_desc0, buf * 16384);
          const uint32_t a_tmem = tmem + buf * 128;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_f16_ts(o_tmem, a_tmem + 64 * (kk >> 2) + 8 * (kk & 3), sdesc_add(vd, kk * 2048), idesc_pv,
                        (kk > 0 || kt > 0) ? 1u : 0u);
          umma_commit(v_empty(buf));
          umma_commit(pv_done(buf));
        }
        if (ok) umma_commit(o_full(ob));
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      sg += unit_nkt(r.qt);
    }
  } else {
    // ---------------- SiLU warps ----------------
    const int grp = warp / kSiluWarps;   // takes the steps s with s % 2 == grp
    const int quad = warp & 3;
    const int half = (warp >> 2) & 1;    // keys [64 half, 64 half + 64)
    const int r = quad * 32 + lane;      // query row within the tile == TMEM lane
    // fp32 output rows written as 32-byte stores when the base and the row stride allow them
    const bool o_v8 = ((reinterpret_cast<uintptr_t>(a.o) | static_cast<uintptr_t>(a.ld_o * 4)) & 31) == 0;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int sg = 0;
    bool ok = true;
    UnitRec u;
    for (int uc = 0; ok && take_unit(uc, u) && u.valid; ++uc) {
      const int nkt = unit_nkt(u.qt), qt = unit_qt(u.qt);
      // first key column this row may see: its own sequence's start inside a pack, else 0
      int lo = 0;
      if (u.qt < 0) {
        const long long g = static_cast<long long>(u.row0) + r;
        int s0 = u.b, s1 = u.b - u.qt;   // pack members b .. b + k - 1
        while (s1 - s0 > 1) {
          const int mid = (s0 + s1) >> 1;
          if (a.offsets[mid] <= g) s0 = mid;
          else s1 = mid;
        }
        lo = static_cast<int>(a.offsets[s0] - u.row0);
      }
      for (int kt = (sg & 1) == grp ? 0 : 1; ok && kt < nkt; kt += 2) {
        const int s = sg + kt, buf = s % 3;
        if (!mbar_wait(b_full(buf), (s / 3) & 1, abort_flag, ctl) ||
            !mbar_wait(s_full(buf), (s / 3) & 1, abort_flag, ctl)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const bool diag = kt == qt;
        // four chunks of 16 keys: [64 half + 16 hc, +16)
#pragma unroll
        for (int hc = 0; hc < 4; ++hc) {
          uint32_t sv[16];
          tmem_ld_32x32b_x16(tmem + lane_base + buf * 128 + 64 * half + 16 * hc, sv);
          uint32_t hb[8];   // half-bias of these keys
          const uint8_t* brow = smem + L::kBias + buf * 32768 + half * 16384 + r * 128;
#pragma unroll
          for (int q2 = 0; q2 < 2; ++q2) {
            const uint4 v = *reinterpret_cast<const uint4*>(brow + (((2 * hc + q2) ^ (r & 7)) << 4));
            hb[4 * q2] = v.x; hb[4 * q2 + 1] = v.y; hb[4 * q2 + 2] = v.z; hb[4 * q2 + 3] = v.w;
          }
          // the bias stage is free once the whole row is in registers
          if (hc == 3) mbar_arrive(b_empty(buf));
          tmem_ld_wait();
          uint32_t p[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t s2 = pack_f16x2(__uint_as_float(sv[2 * j]), __uint_as_float(sv[2 * j + 1]));
            const uint32_t h2 = hfma2_u32(s2, kHalf2Half, hb[j]);
            const uint32_t t2 = tanh_f16x2(h2);
            uint32_t y2 = hfma2_u32(h2, t2, h2);
            if (!F16) {   // the P V MMA takes A and B of one type: P as bf16 next to bf16 V
              const float2 f = unpack_f16x2(y2);
              y2 = pack_bf16x2(f.x, f.y);
            }
            if (diag) {   // keys lo <= col <= r
              const int col = 64 * half + 16 * hc + 2 * j;
              const uint32_t m = ((col <= r && col >= lo) ? 0x0000FFFFu : 0u) |
                                 ((col + 1 <= r && col + 1 >= lo) ? 0xFFFF0000u : 0u);
              y2 &= m;
            }
            p[j] = y2;
          }
          // P of these 16 keys packed into 8 columns over S columns already read
          tmem_st_32x32b_x8(tmem + lane_base + buf * 128 + 64 * half + 8 * hc, p);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full(buf));
      }
      // the group that ran the unit's last step writes its output: rows of this quadrant, columns
      // [32 half, +32) of the head, times 1/N
      if (ok && ((sg + nkt - 1) & 1) == grp) {
        const int ob = uc & 1;
        if (!mbar_wait(o_full(ob), (uc >> 1) & 1, abort_flag, ctl)) {
          ok = false;
        } else {
          tc_fence_after();
          const int qi = qt * kQTile + r;
          const bool row_ok = qi < u.n && qi >= u.q_lo;
          const float sc = a.inv_N;
          const long long orow = static_cast<long long>(u.row0) + qi;
          // columns [32 half + 16 c, +16) of the head, two chunks
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t ov[16];
            tmem_ld_32x32b_x16(tmem + lane_base + kOCol + 64 * ob + 32 * half + 16 * c, ov);
            tmem_ld_wait();
            if (c == 1) {
              tc_fence_before();
              mbar_arrive(o_empty(ob));
            }
            // P and the half-bias are fp16: a score beyond the fp16 range turns O non-finite, which
            // is reported (HSTU_ERR_DEVICE) instead of passing silently
            if (row_ok) {
              bool finite = true;
#pragma unroll
              for (int e = 0; e < 16; ++e) finite &= isfinite(__uint_as_float(ov[e]));
              if (!finite) report_error(a.status, kDevBadInput);
            }
            if (row_ok && HSTU_DCHECK(orow >= 0 && orow < a.T, a.status)) {
              const int ocol = u.h * kD + 32 * half + 16 * c;
              if (a.o_f32 && o_v8) {
                float* dst = reinterpret_cast<float*>(a.o) + orow * a.ld_o + ocol;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                  float f[8];
#pragma unroll
                  for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(ov[8 * q + e]) * sc;
                  st_global_v8(dst + 8 * q, f);
                }
              } else if (a.o_f32) {
                float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.o) + orow * a.ld_o + ocol);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  dst[q] = make_float4(__uint_as_float(ov[4 * q]) * sc, __uint_as_float(ov[4 * q + 1]) * sc,
                                       __uint_as_float(ov[4 * q + 2]) * sc, __uint_as_float(ov[4 * q + 3]) * sc);
              } else {
                uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) + orow * a.ld_o + ocol);
#pragma unroll
                for (int q = 0; q < 2; ++q)
                  dst[q] = make_uint4(
                      pack_bf16x2(__uint_as_float(ov[8 * q]) * sc, __uint_as_float(ov[8 * q + 1]) * sc),
                      pack_bf16x2(__uint_as_float(ov[8 * q + 2]) * sc, __uint_as_float(ov[8 * q + 3]) * sc),
                      pack_bf16x2(__uint_as_float(ov[8 * q + 4]) * sc, __uint_as_float(ov[8 * q + 5]) * sc),
                      pack_bf16x2(__uint_as_float(ov[8 * q + 6]) * sc, __uint_as_float(ov[8 * q + 7]) * sc));
              }
            }
          }
        }
      }
      sg += nkt;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// M-FALCON per-key half-bias: kbias[u * ld + j] = 0.5 (rab_pos[idx(n_u - j)] +
// rab_time[bucket(request_ts[u] - t_j)]) for j < n_u, 0 up to ld. A prefix longer than ld is a
// contract violation: recorded in the status word (the attention then stops at ld keys).
__global__ void __launch_bounds__(256)
falcon_key_bias_kernel(const int64_t* __restrict__ off, const int64_t* __restrict__ ts, const int64_t* __restrict__ req,
                       const float* __restrict__ rab_pos, const float* __restrict__ rab_time, int L, int nb,
                       uint16_t* kbias, int64_t ld, float* self_bias, int* status) {
  __shared__ long long s_tau[kTauEntries];
  for (int e = threadIdx.x; e < kTauEntries; e += blockDim.x) s_tau[e] = g_time_taus[e];
  __syncthreads();
  const int u = blockIdx.y;
  if (u == 0 && blockIdx.x == 0 && threadIdx.x == 0) *self_bias = rab_pos[L - 1] + rab_time[0];
  const long long s0 = off[u];
  const long long n = off[u + 1] - s0;
  if (n > ld || n < 0) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report_error(status, kDevBadInput);
  }
  const long long treq = req[u];
  for (long long j = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; j < ld;
       j += static_cast<long long>(gridDim.x) * blockDim.x) {
    float v = 0.0f;
    if (j < n) {
      const int bkt = time_bucket_pair64(treq, ts[s0 + j], s_tau, nb);
      v = 0.5f * (rab_pos[bias_pos_index(n - j, L)] + rab_time[bkt]);
    }
    kbias[u * ld + j] = __half_as_ushort(__float2half_rn(v));
  }
}

template <bool F16, int G, bool FALCON>
cudaError_t launch_attn2(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tb,
                         const AttnArgs& a, cudaStream_t st) {
  constexpr int NG = G == 1 ? 2 : 1;
  auto kern = attn_fwd_tc2_kernel<F16, G, FALCON, NG>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), Smem2<G>::kTotal);
  if (e != cudaSuccess) return e;
  const long long blocks =
      (FALCON ? static_cast<long long>(a.B) * ((a.cand_rows + kQTile - 1) / kQTile) : a.capacity) * (a.H / G);
  if (blocks == 0) return cudaSuccess;
  return launch_pdl(kern, dim3(static_cast<unsigned>(blocks)), dim3(threads2(NG)), Smem2<G>::kTotal, st, tq, tk, tv, tb,
                    a, wait_ctl(a.status));
}

}  // namespace

// Pairs the bias-tile grids cover at once (they loop over the rest): eight 256-thread blocks per SM
// across the 4 row blocks and the head slices.
int64_t bias_tile_grid(int64_t max_pairs, int bias_heads) {
  const int64_t fit = (4ll * sm_count()) / (bias_heads > 0 ? bias_heads : 1);
  const int64_t g = fit < 1 ? 1 : fit;
  return max_pairs < g ? max_pairs : g;
}

int64_t bias_grid_pairs(int64_t max_pairs, int bias_heads) {
  const int64_t fit = (8ll * sm_count()) / (4ll * (bias_heads > 0 ? bias_heads : 1));
  const int64_t g = fit < 1 ? 1 : fit;
  return max_pairs < g ? max_pairs : g;
}

int64_t attn_max_pairs(int64_t capacity, int max_len) {
  const int64_t mt = (static_cast<int64_t>(max_len) + kQTile - 1) / kQTile;
  return capacity * (mt + 1) / 2;
}

int sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  const bool tracked = dev >= 0 && dev < 64;
  int n = tracked ? cache[dev].load(std::memory_order_relaxed) : 0;
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (tracked) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

template <bool F16>
cudaError_t launch_attn_persistent(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                   const CUtensorMap& tb, const AttnArgs& a, cudaStream_t st) {
  auto kern = attn_fwd_persistent_kernel<F16>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), Smem3::kTotal);
  if (e != cudaSuccess) return e;
  const long long units = a.capacity * a.H;
  const long long blocks = units < sm_count() ? units : sm_count();
  if (blocks == 0) return cudaSuccess;
  e = prof_record(kProfAttnFwd, false, st);
  if (e == cudaSuccess)
    e = launch_pdl(kern, dim3(static_cast<unsigned>(blocks)), dim3(kThreads3), Smem3::kTotal, st, tq, tk, tv, tb, a,
                   wait_ctl(a.status));
  if (e == cudaSuccess) e = prof_record(kProfAttnFwd, true, st);
  return e;
}

cudaError_t attn_fwd_tc2(const AttnArgs& a_in, cudaStream_t st) {
  AttnArgs a = a_in;
  cudaError_t e = upload_time_taus();
  if (e != cudaSuccess) return e;
  if (a.T == 0 || a.capacity == 0) return cudaSuccess;
  const int mt = (a.max_len + kQTile - 1) / kQTile;
  if (mt == 0) return cudaSuccess;
  // with the layer's bias cache the kernel stages the backward's key-major tiles in dynamic shared memory
  const int bias_dyn = a.bias_t_out ? kBiasStageBytes : 0;
  if (bias_dyn) {
    e = ensure_smem_attr(reinterpret_cast<const void*>(attn_bias_kernel), bias_dyn);
    if (e != cudaSuccess) return e;
  }
  a.bias_blocks = bias_tile_grid(a.max_pairs, a.bias_heads);
  const int64_t cvt_blocks = a.cvt_n > 0 ? (a.cvt_n + 8 * kBiasThreads - 1) / (8 * kBiasThreads) : 0;
  if (a.bias_blocks + cvt_blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  e = prof_record(kProfBias, false, st);
  if (e == cudaSuccess)
    e = launch_pdl(attn_bias_kernel,
                   dim3(static_cast<unsigned>(a.bias_blocks + cvt_blocks), static_cast<unsigned>(a.bias_heads)),
                   dim3(kBiasThreads), bias_dyn, st, a);
  if (e == cudaSuccess) e = prof_record(kProfBias, true, st);
  if (e != cudaSuccess) return e;
  const bool f16 = a.in_f16 != 0;
  // the persistent kernel's unit counter lives in the workspace header (reset by the work list), its
  // unit records next to the work list; it loads every tile as 64-row boxes
  if (!a.unit_counter || !a.urec) return cudaErrorInvalidValue;
  CUtensorMap pq, pk, pv, pb;
  if (!encode_tmap_2d_bf16(&pq, a.q, static_cast<int64_t>(a.H) * kD, a.T, a.ld_q, 64, 64, f16) ||
      !encode_tmap_2d_bf16(&pk, a.k, static_cast<int64_t>(a.H) * kD, a.T, a.ld_k, 64, 64, f16) ||
      !encode_tmap_2d_bf16(&pv, a.v, static_cast<int64_t>(a.H) * kD, a.T, a.ld_v, 64, 64, f16) ||
      !encode_tmap_2d_bf16(&pb, a.bias, kQTile, a.max_pairs * a.bias_heads * kQTile, kQTile, 64, 64, true))
    return cudaErrorInvalidValue;
  return f16 ? launch_attn_persistent<true>(pq, pk, pv, pb, a, st) : launch_attn_persistent<false>(pq, pk, pv, pb, a, st);
}

cudaError_t falcon_key_bias(const int64_t* offsets, const int64_t* ts, int users, int max_len,
                            const int64_t* request_ts, const float* rab_pos, const float* rab_time, int pos_max_len,
                            int n_buckets, uint16_t* kbias, int64_t kbias_ld, float* self_bias, int* status,
                            cudaStream_t st) {
  cudaError_t e = upload_time_taus();
  if (e != cudaSuccess || users == 0) return e;
  int64_t blocks = (kbias_ld + 255) / 256;
  blocks = blocks < 1 ? 1 : (blocks > 64 ? 64 : blocks);
  const unsigned gx = static_cast<unsigned>(blocks);
  falcon_key_bias_kernel<<<dim3(gx, static_cast<unsigned>(users)), 256, 0, st>>>(
      offsets, ts, request_ts, rab_pos, rab_time, pos_max_len, n_buckets, kbias, kbias_ld, self_bias, status);
  (void)max_len;
  return cudaGetLastError();
}

cudaError_t attn_falcon_tc(const AttnArgs& a, cudaStream_t st) {
  if (a.B == 0 || a.cand_rows == 0 || a.q_rows == 0) return cudaSuccess;
  CUtensorMap tq, tk, tv;
  const bool f16 = a.in_f16 != 0;
  const int64_t W = static_cast<int64_t>(a.H) * kD;
  // an empty prefix batch still needs valid K/V maps: they are never loaded from (no key tiles)
  const int64_t kv_rows = a.T > 0 ? a.T : 1;
  if (!encode_tmap_2d_bf16(&tq, a.q, W, a.q_rows, a.ld_q, 64, 128, f16) ||
      !encode_tmap_2d_bf16(&tk, a.k, W, kv_rows, a.ld_k, 64, 128, f16) ||
      !encode_tmap_2d_bf16(&tv, a.v, W, kv_rows, a.ld_v, 64, 128, f16))
    return cudaErrorInvalidValue;
  // two heads per CTA only when that still leaves about two CTAs per SM
  const long long tiles = static_cast<long long>(a.B) * ((a.cand_rows + kQTile - 1) / kQTile);
  const int G = (a.H % 2 == 0 && tiles * (a.H / 2) >= 2 * 148) ? 2 : 1;
  if (f16)
    return G == 2 ? launch_attn2<true, 2, true>(tq, tk, tv, tq, a, st) : launch_attn2<true, 1, true>(tq, tk, tv, tq, a, st);
  return G == 2 ? launch_attn2<false, 2, true>(tq, tk, tv, tq, a, st)
                : launch_attn2<false, 1, true>(tq, tk, tv, tq, a, st);
}

}  // namespace hstu
