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
// attn_bwd_tc_kernel<F16>: persistent, one CTA per SM taking (sequence, 128-key tile, head) units
// from a counter, key tiles that visit the most query tiles first; a unit walks the query tiles
// t >= its key tile:
//   warp 16  : TMA: K, V once; Q and dO of each query tile (3 stages); the half-bias tile (2).
//   warp 17  : tcgen05: S^T = K Q^T and dA^T = V dO^T into TMEM (N = 128, the whole query tile);
//              after the elementwise step, the next tile's S^T / dA^T first, then dV += P^T dO
//              (P^T from TMEM), dK += dX^T Q and dQ_tile = dX K (dX^T from shared memory, read
//              K-major for dK and MN-major for dQ). Warp 19 idles.
//   warp 18  : TMA stores: each dQ tile (staged in shared memory) reduce-added into the fp32 dQ,
//              each tile's dX^T (16-bit, from shared memory) to the workspace.
//   warps 0-15: key row = TMEM lane (warp & 3), query half (warp >> 2) & 1, 32 of its 64 queries
//              (warp >> 3): x = s + bias, P^T = SiLU(x), dX^T = dA SiLU'(x) inv_N in fp32, causal
//              and length masks; the half-b warps also stage the previous tile's dQ.
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
#include "bias_tile.cuh"

namespace hstu {

namespace {

constexpr int kD = 64;
constexpr int kSiluWarpsB = 16;
constexpr int kThreadsB = 32 * (kSiluWarpsB + 4);   // + TMA producer, 2 MMA issuers, TMA store warp
constexpr int kSiluThreadsB = 32 * kSiluWarpsB;

// ----------------------------------------------------------------------------------------------
// transposed bias and bucket tiles
// ----------------------------------------------------------------------------------------------
// One block per causal tile pair (grid-stride): the [key][query] half-bias and u8 bucket tiles of
// bias_tile.cuh.
__global__ void __launch_bounds__(kBiasThreads)
attn_bias_t_kernel(AttnBwdArgs A) {
  bias_tiles<true, true>(A.f, reinterpret_cast<uint16_t*>(A.bias_t), reinterpret_cast<uint8_t*>(A.bucket_t));
}

// ----------------------------------------------------------------------------------------------
// backward kernel
// ----------------------------------------------------------------------------------------------
struct BwdSmem {
  static constexpr int kK = 0;                  // K tile of the CTA (16 KB)
  static constexpr int kV = 16384;              // V tile (16 KB)
  static constexpr int kQ0 = 32768;             // stage st (of 3): Q at kQ0 + st * 32768, dO at +16384
  static constexpr int kBT0 = kQ0 + 3 * 32768;  // stage st (of 2): half-bias^T, overwritten in place by dX^T
  static constexpr int kDQ = kBT0 + 2 * 32768;  // dQ tile staging for the TMA reduce-add: 2 x [128][32] fp32
  static constexpr int kBar = kDQ + 32768;
  static constexpr int kTotal = kBar + 512 + 1024;   // barriers, TMEM slot, abort flag, unit ring; alignment
};
static_assert(BwdSmem::kTotal <= 232448, "shared memory of the backward kernel");

// One (key tile, head) unit of the persistent backward: the work-list item and head of unit u.
struct BwdUnit {
  int b, kt, kt_item, h, n, nt, nsteps;
  bool packed;
  long long seq0, pbase;
};

// What the scheduler warp publishes for a unit (its global lookups resolved while the CTA's current
// unit still runs, so the other roles start the next unit without a chain of dependent loads).
struct BwdRec {
  int u, b, kt_item, n;
  long long seq0, pbase;
};

__device__ __forceinline__ BwdRec bwd_rec(const AttnBwdArgs& A, int u) {
  const AttnArgs& a = A.f;
  BwdRec r{u, 0, 0, 0, 0, 0};
  const int item = u / a.H;
  r.b = A.kitems[2 * item];
  r.kt_item = A.kitems[2 * item + 1];
  pair_rows(a.offsets, a.pack, r.b, &r.seq0, &r.n);
  r.pbase = a.pair_base[r.b];
  return r;
}

__device__ __forceinline__ BwdUnit bwd_unit(const BwdRec& r, int H) {
  BwdUnit w;
  const int item = r.u / H;
  w.h = r.u - item * H;
  w.b = r.b;
  w.kt_item = r.kt_item;
  w.packed = w.kt_item < 0;   // a pack of -kt_item short sequences: one diagonal tile
  w.kt = w.packed ? 0 : w.kt_item;
  w.seq0 = r.seq0;
  w.n = r.n;
  w.nt = (w.n + kQTile - 1) / kQTile;
  w.nsteps = w.nt - w.kt;     // query tiles kt .. nt-1
  w.pbase = r.pbase;
  return w;
}

constexpr int kRingB = 4;                        // unit ring between the scheduler warp and the others
constexpr int kRingReadersB = kSiluWarpsB + 3;   // producer, MMA issuer, store warp, elementwise warps

// Persistent: one CTA per SM takes (key tile, head) units, longest key tiles first, from a counter
// the work list zeroes; barrier phases run on per-CTA counters of units (i) and query-tile steps (G).
template <bool F16>
__global__ void __launch_bounds__(kThreadsB, 1)
attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                   const __grid_constant__ CUtensorMap tmBT, const __grid_constant__ CUtensorMap tmDX,
                   const __grid_constant__ CUtensorMap tmDQ, AttnBwdArgs A, WaitCtl ctl) {
  pdl_enter();
  using Lb = BwdSmem;
  const AttnArgs& a = A.f;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int total = *A.kcount * a.H;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lb::kBar);
  // 0 kv_full | 1,2 qdo_full | 3,4 qdo_empty | 5,6 bb_full | 7,8 bb_empty | 9,10 s_full (query half
  // a, b) | 11,12 p_ready (half a, b) | 13 dq_full | 14 fin (every MMA of the unit done) | 15,16
  // dx_full (stage) | 17 dq_staged | 18 dq_stage_free | 19,20 p_free (half a, b: the dV MMA has read
  // P^T_h) | 21 qdo_full, 22 qdo_empty of the third Q/dO stage | 23 dkdv_free (the unit's dK, dV
  // are out of TMEM) | 24.. ring_full, ring_empty, ring_got (kRingB each)
  constexpr int kNumBars = 24 + 3 * kRingB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile BwdRec* ring = reinterpret_cast<volatile BwdRec*>(tmem_slot + 2);   // kRingB records
  static_assert(8 * kNumBars + 8 + kRingB * sizeof(BwdRec) <= 512 && (8 * kNumBars + 8) % 8 == 0, "barrier region");
  const uint32_t bar0 = smem_u32(bars);
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  auto qdo_full = [&](int sq) { return sq < 2 ? BAR(1 + sq) : BAR(21); };
  auto qdo_empty = [&](int sq) { return sq < 2 ? BAR(3 + sq) : BAR(22); };
  auto ring_full = [&](int r) { return BAR(24 + r); };
  auto ring_empty = [&](int r) { return BAR(24 + kRingB + r); };
  auto ring_got = [&](int r) { return BAR(24 + 2 * kRingB + r); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tid = threadIdx.x;

  if (tid == 0) {
    mbar_init(BAR(0), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(1 + s), 1);
      mbar_init(BAR(3 + s), 2);   // Q/dO stage free: after S^T / dA^T and after the gradient MMAs
      mbar_init(BAR(5 + s), 1);
      mbar_init(BAR(7 + s), 2);   // bias/dX stage free: the MMAs read dX^T and the store warp sent it
      mbar_init(BAR(15 + s), kSiluThreadsB);   // both query halves of dX^T written
    }
    for (int hh = 0; hh < 2; ++hh) {
      mbar_init(BAR(9 + hh), 1);
      mbar_init(BAR(11 + hh), kSiluThreadsB / 2);
      mbar_init(BAR(19 + hh), 1);
    }
    mbar_init(BAR(13), 1);
    mbar_init(BAR(14), 1);
    mbar_init(BAR(21), 1);
    mbar_init(BAR(22), 2);
    mbar_init(BAR(17), kSiluThreadsB / 2);     // the half-b warps staged a dQ tile
    mbar_init(BAR(18), 1);                     // the store warp's reduce-add has read the staging
    mbar_init(BAR(23), kSiluThreadsB);
    for (int r = 0; r < kRingB; ++r) {
      mbar_init(ring_full(r), 1);
      mbar_init(ring_empty(r), kRingReadersB);
      mbar_init(ring_got(r), 1);
    }
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
    tma_prefetch_desc(&tmDQ);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // query q of the tile: S^T at column q, dA^T at column 128 + q;
  // accumulators dV, dK and the dQ tile of one query tile; P^T_h packed two per column at
  // [448 + 32 h, 448 + 32 h + 32)
  const uint32_t tDV = tmem + 256, tDK = tmem + 320, tDQ = tmem + 384, tP = tmem + 448;

  const uint32_t sK = smem_u32(smem + Lb::kK), sV = smem_u32(smem + Lb::kV);
  const uint32_t sQ0 = smem_u32(smem + Lb::kQ0);
  const uint32_t sBT0 = smem_u32(smem + Lb::kBT0);
  const uint32_t sDQ = smem_u32(smem + Lb::kDQ);

  // Unit i of this CTA for one reading thread (false: the wait gave up); u >= total ends the
  // sequence. The reader frees the ring slot once it holds the record.
  auto take_unit = [&](int i, BwdRec& rec) -> bool {
    const int r = i % kRingB;
    if (!mbar_wait(ring_full(r), (i / kRingB) & 1, abort_flag, ctl)) return false;
    rec.u = ring[r].u;
    rec.b = ring[r].b;
    rec.kt_item = ring[r].kt_item;
    rec.n = ring[r].n;
    rec.seq0 = ring[r].seq0;
    rec.pbase = ring[r].pbase;
    mbar_arrive(ring_empty(r));
    return true;
  };
  auto take_unit_warp = [&](int i, BwdRec& rec) -> bool {
    BwdRec v{0, 0, 0, 0, 0, 0};
    bool ok = true;
    if (lane == 0) ok = take_unit(i, v);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    rec.u = __shfl_sync(0xffffffffu, v.u, 0);
    rec.b = __shfl_sync(0xffffffffu, v.b, 0);
    rec.kt_item = __shfl_sync(0xffffffffu, v.kt_item, 0);
    rec.n = __shfl_sync(0xffffffffu, v.n, 0);
    rec.seq0 = __shfl_sync(0xffffffffu, v.seq0, 0);
    rec.pbase = __shfl_sync(0xffffffffu, v.pbase, 0);
    return ok;
  };

  if (warp == kSiluWarpsB) {
    // ---------------- TMA producer ----------------
    // Per unit: Q and dO of step g (counted over the CTA's units) into stage g % 3 from lanes 2 sq,
    // 2 sq + 1; K and V (lanes 0, 1) once every MMA of the previous unit has completed; the bias
    // halves of step g into stage g % 2 from lanes 8 + 2 st, 9 + 2 st, one step behind its Q / dO
    // (waiting for a bias stage never delays the next Q / dO load).
    int G = 0;
    bool ok = true;
    for (int i = 0; ok; ++i) {
      BwdRec rec;
      if (!take_unit_warp(i, rec) || rec.u >= total) break;
      const BwdUnit w = bwd_unit(rec, a.H);
      const int krow = static_cast<int>(w.seq0) + w.kt * kQTile;
      // K and V (read by this unit alone, so usually from DRAM) and the first bias tile into L2 now:
      // their loads wait until the previous unit's last MMAs have completed
      if (i >= 1 && lane == 0 && w.nsteps > 0) {
        tma_prefetch_l2_2d(&tmK, w.h * kD, krow);
        tma_prefetch_l2_2d(&tmV, w.h * kD, krow);
        const long long pair0 = w.pbase + static_cast<long long>(w.kt) * (w.kt + 1) / 2 + w.kt;
        const int prow0 = static_cast<int>((pair0 * a.bias_heads + (a.bias_heads > 1 ? w.h : 0)) * kQTile);
        tma_prefetch_l2_2d(&tmBT, 0, prow0);
        tma_prefetch_l2_2d(&tmBT, 64, prow0);
      }
      auto load_bias = [&](int s) -> bool {
        const int gs = G + s, st = gs & 1, qt = w.kt + s;
        if (gs >= 2 && !mbar_wait_warp(BAR(7 + st), ((gs >> 1) & 1) ^ 1, abort_flag, ctl)) return false;
        const long long pair = w.pbase + static_cast<long long>(qt) * (qt + 1) / 2 + w.kt;
        const int prow = static_cast<int>((pair * a.bias_heads + (a.bias_heads > 1 ? w.h : 0)) * kQTile);
        if (lane == 0) mbar_arrive_expect_tx(BAR(5 + st), 32768);
        __syncwarp();
        const int hx = lane - 8 - 2 * st;
        if (hx == 0 || hx == 1) tma_load_2d(sBT0 + st * 32768 + hx * 16384, &tmBT, BAR(5 + st), 64 * hx, prow);
        return true;
      };
      for (int s = 0; ok && s < w.nsteps; ++s) {
        const int gs = G + s, qt = w.kt + s, sq = gs % 3;
        if (gs >= 3 && !mbar_wait_warp(qdo_empty(sq), ((gs / 3) & 1) ^ 1, abort_flag, ctl)) {
          ok = false;
          break;
        }
        const int qrow = static_cast<int>(w.seq0) + qt * kQTile;
        if (lane == 0) mbar_arrive_expect_tx(qdo_full(sq), 32768);
        __syncwarp();
        if (lane == 2 * sq) tma_load_2d(sQ0 + sq * 32768, &tmQ, qdo_full(sq), w.h * kD, qrow);
        if (lane == 2 * sq + 1) tma_load_2d(sQ0 + sq * 32768 + 16384, &tmDO, qdo_full(sq), w.h * kD, qrow);
        if (s == 0) {
          if (i >= 1 && !mbar_wait_warp(BAR(14), (i - 1) & 1, abort_flag, ctl)) {
            ok = false;
            break;
          }
          if (lane == 0) mbar_arrive_expect_tx(BAR(0), 32768);
          __syncwarp();
          if (lane == 0) tma_load_2d(sK, &tmK, BAR(0), w.h * kD, krow);
          if (lane == 1) tma_load_2d(sV, &tmV, BAR(0), w.h * kD, krow);
        }
        if (s >= 1) ok = load_bias(s - 1);
      }
      if (ok && w.nsteps > 0) ok = load_bias(w.nsteps - 1);
      // every load of the unit is issued (its last steps are still to run): time to take the next
      if (ok && lane == 0) mbar_arrive(ring_got(i % kRingB));
      G += w.nsteps;
    }
  } else if (warp == kSiluWarpsB + 1) {
    // ---------------- tcgen05 issuer (warp 17) ----------------
    // Per query tile: S^T = K Q^T and dA^T = V dO^T over the whole tile (N = 128: a tcgen05.mma
    // costs the same issue time at N = 64 and 128, so two 64-query halves would double it); once
    // both query halves' elementwise warps have written P^T (TMEM) and dX^T (shared memory), first
    // the next tile's S^T / dA^T (so that its elementwise work overlaps the gradient MMAs), then
    // dV += P^T_h dO_h and dK += dX^T_h Q_h for both halves and dQ_tile = dX K. The Q / dO stage
    // is freed by two commits: after S^T / dA^T and after the gradient MMAs. A unit's first
    // gradient MMAs (which overwrite dV and dK) wait until the previous unit's dV and dK are out of
    // TMEM; its end is committed to `fin`.
    if (lane == 0) {
      constexpr uint32_t id_s = make_idesc_f16kind(128, 128, 0, 0, F16);
      constexpr uint32_t id_kmn = make_idesc_f16kind(128, 64, 0, 1, F16);
      constexpr uint32_t id_mnmn = make_idesc_f16kind(128, 64, 1, 1, F16);
      // base descriptors: K-major (lbo 16) and MN-major (lbo 16384, the 64-element block stride)
      const uint64_t k_km = make_sdesc_sw128(sK, 16, 1024), v_km = make_sdesc_sw128(sV, 16, 1024);
      const uint64_t k_mn = make_sdesc_sw128(sK, 16384, 1024);
      const uint64_t q_km = make_sdesc_sw128(sQ0, 16, 1024), q_mn = make_sdesc_sw128(sQ0, 16384, 1024);
      const uint64_t x_km = make_sdesc_sw128(sBT0, 16, 1024), x_mn = make_sdesc_sw128(sBT0, 16384, 1024);
      auto issue_s = [&](int gs) -> bool {
        const int sq = gs % 3;
        if (!mbar_wait(qdo_full(sq), (gs / 3) & 1, abort_flag, ctl)) return false;
        tc_fence_after();
        const uint64_t qd = sdesc_add(q_km, sq * 32768), dod = sdesc_add(qd, 16384);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_f16_ss(tmem, sdesc_add(k_km, kk * 32), sdesc_add(qd, kk * 32), id_s, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_f16_ss(tmem + 128, sdesc_add(v_km, kk * 32), sdesc_add(dod, kk * 32), id_s, kk > 0 ? 1u : 0u);
        umma_commit(BAR(9));
        umma_commit(BAR(10));
        umma_commit(qdo_empty(sq));
        return true;
      };
      auto issue_grad = [&](int gs, bool first, int hh) {
        const int st = gs & 1, sq = gs % 3;
        const uint64_t qd = sdesc_add(q_mn, sq * 32768 + hh * 8192), dod = sdesc_add(qd, 16384);
        const uint64_t xd = sdesc_add(x_km, st * 32768 + hh * 16384);
        const uint32_t acc0 = (!first || hh > 0) ? 1u : 0u;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4)   // dV += P^T_h dO_h
          umma_f16_ts(tDV, tP + 32 * hh + 8 * k4, sdesc_add(dod, k4 * 2048), id_kmn, k4 > 0 ? 1u : acc0);
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4)   // dK += dX^T_h Q_h
          umma_f16_ss(tDK, sdesc_add(xd, k4 * 32), sdesc_add(qd, k4 * 2048), id_kmn, k4 > 0 ? 1u : acc0);
        umma_commit(BAR(19 + hh));
      };
      int G = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        BwdRec rec;
        if (!take_unit(i, rec) || rec.u >= total) break;
        const BwdUnit w = bwd_unit(rec, a.H);
        if (!mbar_wait(BAR(0), i & 1, abort_flag, ctl) || !issue_s(G)) break;
        for (int s = 0; ok && s < w.nsteps; ++s) {
          const int gs = G + s, st = gs & 1;
          ok = mbar_wait(BAR(11), gs & 1, abort_flag, ctl) && mbar_wait(BAR(12), gs & 1, abort_flag, ctl);
          if (!ok) break;
          tc_fence_after();
          if (s + 1 < w.nsteps && !issue_s(gs + 1)) {
            ok = false;
            break;
          }
          if (s == 0 && i >= 1) {   // dV, dK of the previous unit read out of TMEM
            if (!mbar_wait(BAR(23), (i - 1) & 1, abort_flag, ctl)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          issue_grad(gs, s == 0, 0);
          issue_grad(gs, s == 0, 1);
          const uint64_t xd = sdesc_add(x_mn, st * 32768);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)   // dQ_tile = dX K
            umma_f16_ss(tDQ, sdesc_add(xd, kk * 2048), sdesc_add(k_mn, kk * 2048), id_mnmn, kk > 0 ? 1u : 0u);
          umma_commit(BAR(13));
          umma_commit(qdo_empty(gs % 3));
          umma_commit(BAR(7 + st));
        }
        if (ok) umma_commit(BAR(14));
        G += w.nsteps;
      }
    }
  } else if (warp == kSiluWarpsB + 2) {
    // ---------------- TMA stores ----------------
    // dQ tile j (staged in shared memory by the half-b warps) is added to the fp32 dQ with one
    // TMA reduce-add per 32 columns; once both query halves of tile s are done, dX^T (the 16-bit
    // operand of dK and dQ, in the stage's bias slot) goes to the workspace, from which the table
    // gradients are summed over the heads.
    // dQ reduce-adds from lanes 0 and 1, dX^T stores from lanes 2 and 3 (each lane waits for its own
    // bulk group; lane 0 then signals the barrier)
    int G = 0;
    bool ok = true;
    for (int i = 0; ok; ++i) {
      BwdRec rec;
      if (!take_unit_warp(i, rec) || rec.u >= total) break;
      const BwdUnit w = bwd_unit(rec, a.H);
      auto reduce_dq = [&](int gj, int qt) -> bool {
        if (!mbar_wait_warp(BAR(17), gj & 1, abort_flag, ctl)) return false;
        if (lane < 2) {
          const int y = static_cast<int>(w.seq0) + qt * kQTile;
          tma_reduce_add_2d(&tmDQ, sDQ + lane * 16384, w.h * kD + 32 * lane, y);
          bulk_commit_group();
          bulk_wait_group_read<0>();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(18));
        return true;
      };
      for (int s = 0; ok && s < w.nsteps; ++s) {
        const int gs = G + s, st = gs & 1;
        if (s >= 1 && !reduce_dq(gs - 1, w.kt + s - 1)) {
          ok = false;
          break;
        }
        if (!mbar_wait_warp(BAR(15 + st), (gs >> 1) & 1, abort_flag, ctl)) {
          ok = false;
          break;
        }
        if (lane == 2 || lane == 3) {
          const int qt = w.kt + s;
          const long long pair = w.pbase + static_cast<long long>(qt) * (qt + 1) / 2 + w.kt;
          const int y = static_cast<int>((pair * a.H + w.h) * kQTile);
          tma_store_2d(&tmDX, sBT0 + st * 32768 + (lane - 2) * 16384, 64 * (lane - 2), y);
          bulk_commit_group();
          bulk_wait_group_read<0>();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(7 + st));
      }
      if (ok && w.nsteps > 0) ok = reduce_dq(G + w.nsteps - 1, w.kt + w.nsteps - 1);
      G += w.nsteps;
    }
    bulk_wait_group_all();
  } else if (warp == kSiluWarpsB + 3) {
    // ---------------- unit scheduler ----------------
    // unit 0 is blockIdx.x, later ones come from the counter, each taken once the producer has
    // issued every load of the one before: a CTA claims its next unit a few steps before it can
    // start it, so the units (longest first) go to the CTAs that come free first
    if (lane == 0) {
      for (int i = 0;; ++i) {
        const int r = i % kRingB;
        if (i >= 1 && !mbar_wait(ring_got((i - 1) % kRingB), ((i - 1) / kRingB) & 1, abort_flag, ctl)) break;
        const int u = i == 0 ? static_cast<int>(blockIdx.x) : static_cast<int>(gridDim.x) + atomicAdd(A.sched, 1);
        const BwdRec rec = u < total ? bwd_rec(A, u) : BwdRec{u, 0, 0, 0, 0, 0};
        if (i >= kRingB && !mbar_wait(ring_empty(r), ((i / kRingB) - 1) & 1, abort_flag, ctl)) break;
        ring[r].u = rec.u;
        ring[r].b = rec.b;
        ring[r].kt_item = rec.kt_item;
        ring[r].n = rec.n;
        ring[r].seq0 = rec.seq0;
        ring[r].pbase = rec.pbase;
        mbar_arrive(ring_full(r));
        if (u >= total) break;
      }
    }
  } else if (warp < kSiluWarpsB) {
    // ---------------- elementwise warps ----------------
    // warp w: key rows [32 (w & 3), +32) (TMEM lane quadrant), query half hq = (w >> 2) & 1,
    // queries [64 hq + 32 sub, +32) with sub = w >> 3
    const int quad = warp & 3;
    const int hq = (warp >> 2) & 1;
    const int sub = warp >> 3;
    const int rj = quad * 32 + lane;      // key row == TMEM lane of S^T, dA^T, dV, dK
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const float inv_N = a.inv_N;
    const float cN = 0.5f * inv_N;
    bool ok = true;
    // (half-b warps) dQ tile j: TMEM lane = query row, columns [32 sub, +32) staged as box sub of
    // the reduce-add, 128-byte swizzled rows
    auto stage_dq = [&](int j) -> bool {
      if (!mbar_wait(BAR(13), j & 1, abort_flag, ctl)) return false;
      if (j >= 1 && !mbar_wait(BAR(18), (j - 1) & 1, abort_flag, ctl)) return false;
      tc_fence_after();
      uint32_t v[32];
      tmem_ld_32x32b_x32(tDQ + lane_base + 32 * sub, v);
      tmem_ld_wait();
      uint8_t* row = smem + Lb::kDQ + sub * 16384 + rj * 128;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        *reinterpret_cast<uint4*>(row + ((u ^ (rj & 7)) << 4)) = make_uint4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
      fence_proxy_async_smem();
      mbar_arrive(BAR(17));
      return true;
    };
    // one 16-query piece: x = s + bias, sigma(x) = (1 + tanh(x/2)) / 2, P = SiLU(x) = x sigma,
    // dX = dA inv_N SiLU'(x) = dA (inv_N sigma + P inv_N (1 - sigma)), all in fp32; P and dX are
    // rounded once to the MMA operand type. (A packed-fp16 evaluation of SiLU' quantises 1 - sigma
    // near x = 8 and biases the table-gradient sums.)
    auto piece = [&](const uint32_t (&sv)[16], const uint32_t (&dav)[16], const uint32_t* hb, uint32_t* pp,
                     uint32_t* dxp, bool masked, int col0, int lo_col, int hi_col) {
#pragma unroll
      for (int e2 = 0; e2 < 8; ++e2) {
        const float2 hbf = unpack_f16x2(hb[e2]);
        float pv[2], dv2[2];
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const float hx = fmaf(__uint_as_float(sv[2 * e2 + x]), 0.5f, x ? hbf.y : hbf.x);
          const float t = tanh_f32_approx(hx);
          const float av = fmaf(hx, t, hx);
          const float sgN = fmaf(cN, t, cN);
          const float w = fmaf(av, inv_N - sgN, sgN);
          float dxv = __uint_as_float(dav[2 * e2 + x]) * w;
          float pvv = av;
          if (masked) {
            const int col = col0 + 2 * e2 + x;
            const bool keep = col >= lo_col && col < hi_col;
            pvv = keep ? pvv : 0.0f;
            dxv = keep ? dxv : 0.0f;
          }
          pv[x] = pvv;
          dv2[x] = dxv;
        }
        if (F16) {
          pp[e2] = pack_f16x2(pv[0], pv[1]);
          dxp[e2] = pack_f16x2(dv2[0], dv2[1]);
        } else {   // the MMAs take A and B of one type: P and dX as bf16 next to bf16 dO, Q, K
          pp[e2] = pack_bf16x2(pv[0], pv[1]);
          dxp[e2] = pack_bf16x2(dv2[0], dv2[1]);
        }
      }
    };
    int G = 0;
    for (int i = 0; ok; ++i) {
      BwdRec rec;
      if (!take_unit_warp(i, rec) || rec.u >= total) break;
      const BwdUnit w = bwd_unit(rec, a.H);
      const int kt = w.kt, n = w.n, nt = w.nt, nsteps = w.nsteps;
      const long long seq0 = w.seq0;
      // in a pack, queries past the end of the key row's own sequence are masked
      int seg_end = n;
      if (w.packed && rj < n) {
        const long long g = seq0 + rj;
        int s0 = w.b, s1 = w.b - w.kt_item;
        while (s1 - s0 > 1) {
          const int mid = (s0 + s1) >> 1;
          if (a.offsets[mid] <= g) s0 = mid;
          else s1 = mid;
        }
        seg_end = static_cast<int>(a.offsets[s0 + 1] - seq0);
      }
    for (int s = 0; ok && s < nsteps; ++s) {
      const int gs = G + s, qt = kt + s, st = gs & 1;
      if (!mbar_wait(BAR(5 + st), (gs >> 1) & 1, abort_flag, ctl) ||
          !mbar_wait(BAR(9 + hq), gs & 1, abort_flag, ctl)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // masks: the diagonal tile keeps queries >= key; the last query tile keeps queries < n; a key
      // row past n keeps nothing (it only occurs in the diagonal tile of the last key tile)
      const bool need_mask = (s == 0) || (qt == nt - 1);
      const int lo_col = (s == 0) ? rj : 0;
      const int hi_col = (kt * kQTile + rj < n) ? min(kQTile, seg_end - qt * kQTile) : 0;
      uint8_t* bt_row = smem + Lb::kBT0 + st * 32768 + hq * 16384 + rj * 128;
#pragma unroll
      for (int pc = 0; pc < 2; ++pc) {
        const int c0 = 64 * hq + 32 * sub + 16 * pc;   // first query column of the piece
        uint32_t sv[16], dav[16];
        tmem_ld_32x32b_x16(tmem + lane_base + 64 * hq + 32 * sub + 16 * pc, sv);
        tmem_ld_32x32b_x16(tmem + lane_base + 128 + 64 * hq + 32 * sub + 16 * pc, dav);
        const int u0 = 4 * sub + 2 * pc;   // first 16-byte unit of the piece in the bias row
        uint32_t hb[8];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint4 w = *reinterpret_cast<const uint4*>(bt_row + (((u0 + q) ^ (rj & 7)) << 4));
          hb[4 * q] = w.x; hb[4 * q + 1] = w.y; hb[4 * q + 2] = w.z; hb[4 * q + 3] = w.w;
        }
        tmem_ld_wait();
        uint32_t pp[8], dxp[8];
        if (need_mask) piece(sv, dav, hb, pp, dxp, true, c0, lo_col, hi_col);
        else piece(sv, dav, hb, pp, dxp, false, c0, lo_col, hi_col);
        if (pc == 0 && gs >= 1) {   // the previous tile's dV MMA has read P^T_h
          if (!mbar_wait(BAR(19 + hq), (gs - 1) & 1, abort_flag, ctl)) { ok = false; break; }
          tc_fence_after();
        }
        tmem_st_32x32b_x8(tP + lane_base + 32 * hq + 16 * sub + 8 * pc, pp);
        // dX^T replaces the half-bias just read: same row, same swizzled 16-byte units
#pragma unroll
        for (int q = 0; q < 2; ++q)
          *reinterpret_cast<uint4*>(bt_row + (((u0 + q) ^ (rj & 7)) << 4)) =
              make_uint4(dxp[4 * q], dxp[4 * q + 1], dxp[4 * q + 2], dxp[4 * q + 3]);
      }
      if (!ok) break;
      // (half b) the previous tile's dQ: its MMAs were issued after this tile's S^T_b
      if (hq == 1 && s >= 1 && !stage_dq(gs - 1)) { ok = false; break; }
      tmem_st_wait();
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(BAR(11 + hq));    // P^T_h in TMEM, dX^T_h in shared memory
      mbar_arrive(BAR(15 + st));
    }
    if (ok && hq == 1 && nsteps > 0 && !stage_dq(G + nsteps - 1)) ok = false;
    // dK, dV: key row = TMEM lane, columns [16 (2 hq + sub), +16) of the head
    const int cc = 16 * (2 * hq + sub);
    const bool row_in = kt * kQTile + rj < n;
    const long long row = seq0 + kt * kQTile + rj;
    // (layer backward) the Z_K, Z_V values of those columns, loaded while the unit's last MMAs drain
    uint4 zk4[2] = {}, zv4[2] = {};
    if (A.dz_k && ok && row_in) {
      const long long zo = row * A.ld_z + w.h * kD + cc;
      const uint4* zkp = reinterpret_cast<const uint4*>(static_cast<const __half*>(A.z_k) + zo);
      const uint4* zvp = reinterpret_cast<const uint4*>(static_cast<const __half*>(A.z_v) + zo);
      zk4[0] = zkp[0]; zk4[1] = zkp[1];
      zv4[0] = zvp[0]; zv4[1] = zvp[1];
    }
    if (ok && !mbar_wait(BAR(14), i & 1, abort_flag, ctl)) ok = false;
    if (ok) {
      tc_fence_after();
      uint32_t vk[16], vv[16];
      tmem_ld_32x32b_x16(tDK + lane_base + cc, vk);
      tmem_ld_32x32b_x16(tDV + lane_base + cc, vv);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(BAR(23));   // the accumulators are free for the next unit
      const int h = w.h;
      if (row_in && A.dz_k) {
        // dZ_K = dK (.) SiLU'(Z_K), dZ_V = (dV inv_N) (.) SiLU'(Z_V), rounded once to fp16
        uint32_t ok2[8], ov2[8];
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) {
          const uint32_t zkw = e2 < 4 ? (&zk4[0].x)[e2] : (&zk4[1].x)[e2 - 4];
          const uint32_t zvw = e2 < 4 ? (&zv4[0].x)[e2] : (&zv4[1].x)[e2 - 4];
          const float2 zk = unpack_f16x2(zkw), zv = unpack_f16x2(zvw);
          ok2[e2] = pack_f16x2(__uint_as_float(vk[2 * e2]) * silu_grad(zk.x),
                               __uint_as_float(vk[2 * e2 + 1]) * silu_grad(zk.y));
          ov2[e2] = pack_f16x2((__uint_as_float(vv[2 * e2]) * inv_N) * silu_grad(zv.x),
                               (__uint_as_float(vv[2 * e2 + 1]) * inv_N) * silu_grad(zv.y));
        }
        const long long zo = row * A.ld_z + h * kD + cc;
        uint4* dzk = reinterpret_cast<uint4*>(static_cast<__half*>(A.dz_k) + zo);
        uint4* dzv = reinterpret_cast<uint4*>(static_cast<__half*>(A.dz_v) + zo);
        dzk[0] = make_uint4(ok2[0], ok2[1], ok2[2], ok2[3]);
        dzk[1] = make_uint4(ok2[4], ok2[5], ok2[6], ok2[7]);
        dzv[0] = make_uint4(ov2[0], ov2[1], ov2[2], ov2[3]);
        dzv[1] = make_uint4(ov2[4], ov2[5], ov2[6], ov2[7]);
      } else if (row_in) {
        float4* dk = reinterpret_cast<float4*>(A.dk + row * A.ld_g + h * kD + cc);
        float4* dvp = reinterpret_cast<float4*>(A.dv + row * A.ld_g + h * kD + cc);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          dk[q] = make_float4(__uint_as_float(vk[4 * q]), __uint_as_float(vk[4 * q + 1]),
                              __uint_as_float(vk[4 * q + 2]), __uint_as_float(vk[4 * q + 3]));
          dvp[q] = make_float4(__uint_as_float(vv[4 * q]) * inv_N, __uint_as_float(vv[4 * q + 1]) * inv_N,
                               __uint_as_float(vv[4 * q + 2]) * inv_N, __uint_as_float(vv[4 * q + 3]) * inv_N);
        }
      }
    }
    G += nsteps;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // Every unit this CTA will take is taken: the last CTA to get here puts the unit counter and the
  // finished-CTA counter back to zero, so a later launch over the same work list (a second backward
  // after one forward) starts from unit 0 without a work-list launch of its own.
  if (warp == kSiluWarpsB + 3 && lane == 0) {
    __threadfence();
    if (atomicAdd(A.sched + 1, 1) == static_cast<int>(gridDim.x) - 1) {
      atomicExch(A.sched, 0);
      atomicExch(A.sched + 1, 0);
    }
  }
}

// ----------------------------------------------------------------------------------------------
// table gradients from the per-head dX^T tiles
// ----------------------------------------------------------------------------------------------
// Two blocks per causal tile pair, 64 key rows each. Thread (warp w, lane l) holds the fp32 head
// sum of key rows j_k = 64 y + 8 w + 2 k + l / 16 (k < 4), queries [c0, c0 + 8), c0 = 8 (l % 16).
//  d rab_pos: element (j, i) of the tile lies on diagonal i - j + 127 (relative position
//   128 (qt - kt) + i - j). A thread's 32 elements fall on 14 diagonals (e - 2k = const), summed in

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

// One causal tile pair (row block yblk, table slice hb) of attn_table_grad_kernel; false when `pair`
// is past the batch's last pair.
template <bool F16>
__device__ __forceinline__ bool table_grad_pair(const AttnBwdArgs& A, long long pair, int yblk, int hb) {
  const AttnArgs& a = A.f;
  int b, qt, kt;
  if (!decode_tile_pair(pair, a.pair_base, a.B, &b, &qt, &kt)) return false;
  if (a.pack && a.pack[b] == 0) return true;   // a packed sequence's own pair: its pack's tile holds its rows
  __shared__ float s_win[8][256];
  __shared__ float s_hist[128][32];
  __shared__ float s_thist[16 * 16];
  __shared__ int s_ty[256];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  // table slice hb: with tables shared by the heads (bias_heads 1) the block sums all H heads, with
  // per-head tables only head hb
  const int h_lo = a.bias_heads > 1 ? hb : 0, h_hi = a.bias_heads > 1 ? hb + 1 : a.H;
  const int nt = a.n_types;
  for (int e = tid; e < 8 * 256; e += kTgThreads) (&s_win[0][0])[e] = 0.0f;
  for (int e = tid; e < 128 * 32; e += kTgThreads) (&s_hist[0][0])[e] = 0.0f;
  if (nt > 0) {
    s_thist[tid] = 0.0f;   // 256 threads, 16 x 16 entries
    long long seq0;
    int n;
    if (pair_rows(a.offsets, a.pack, b, &seq0, &n))
      tile_types_load(s_ty, a.token_type, seq0, n, qt * kQTile, kt * kQTile, nt, nullptr);
  }
  const int g = lane >> 4, c0 = 8 * (lane & 15);
  const int j0 = 64 * yblk + 8 * w + g;   // row of k = 0; row k is j0 + 2k
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
  int h = h_lo;
  for (; h + 2 <= h_hi; h += 2) {
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
  if (h < h_hi) {
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
  // d rab_type[type_query][type_key]: element (key row j_k, query c0 + e)
  if (nt > 0) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int tk = s_ty[128 + j0 + 2 * k];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (acc[k][e] != 0.0f) atomicAdd(&s_thist[s_ty[c0 + e] * nt + tk], acc[k][e]);
    }
  }
  __syncthreads();
  const int L = a.pos_max_len;
  float* drab_pos = A.drab_pos + static_cast<long long>(hb) * (2 * L - 1);
  float* drab_time = A.drab_time + static_cast<long long>(hb) * a.n_buckets;
  if (tid < 255) {
    float v = 0.0f;
#pragma unroll
    for (int ww = 0; ww < 8; ++ww) v += s_win[ww][tid];
    if (v != 0.0f)
      atomicAdd(drab_pos + bias_pos_index(static_cast<long long>(qt - kt) * kQTile + tid - 127, L), v);
  }
  if (tid < a.n_buckets) {
    float v = 0.0f;
#pragma unroll 8
    for (int l = 0; l < 32; ++l) v += s_hist[tid][(l + tid) & 31];
    if (v != 0.0f) atomicAdd(drab_time + tid, v);
  }
  if (nt > 0 && tid < nt * nt && s_thist[tid] != 0.0f)
    atomicAdd(A.drab_type + static_cast<long long>(hb) * nt * nt + tid, s_thist[tid]);
  return true;
}

// Pairs blockIdx.x, + gridDim.x, ... up to the batch's last one (the grid is sized for the SMs).
template <bool F16>
__global__ void __launch_bounds__(kTgThreads)
attn_table_grad_kernel(AttnBwdArgs A) {
  pdl_enter();
  for (long long p = blockIdx.x; p < A.f.max_pairs; p += gridDim.x) {
    if (!table_grad_pair<F16>(A, p, static_cast<int>(blockIdx.y), static_cast<int>(blockIdx.z))) break;
    __syncthreads();   // the shared windows and histograms are reused by the next pair
  }
}

}  // namespace

cudaError_t attn_bwd_tc(const AttnBwdArgs& A, cudaStream_t st, const SideLaunch* side) {
  const AttnArgs& a = A.f;
  cudaError_t e = upload_time_taus();
  if (e != cudaSuccess) return e;
  if (a.T == 0 || a.capacity == 0) return cudaSuccess;
  const int mt = (a.max_len + kQTile - 1) / kQTile;
  if (mt == 0) return cudaSuccess;
  if (!A.bias_cached) {
    e = launch_pdl(attn_bias_t_kernel,
                   dim3(static_cast<unsigned>(bias_tile_grid(a.max_pairs, a.bias_heads)), static_cast<unsigned>(a.bias_heads)),
                   dim3(kBiasThreads), 0, st, A);
    if (e != cudaSuccess) return e;
  }
  // TMA row coordinates of the bias and dX^T tiles are 32-bit
  if (a.max_pairs * a.H * kQTile > 0x7fffffffLL) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv, tdo, tbt, tdx, tdq;
  const bool f16 = a.in_f16 != 0;
  const int64_t W = static_cast<int64_t>(a.H) * kD;
  if (!encode_tmap_2d_bf16(&tq, a.q, W, a.T, a.ld_q, 64, 128, f16) ||
      !encode_tmap_2d_bf16(&tk, a.k, W, a.T, a.ld_k, 64, 128, f16) ||
      !encode_tmap_2d_bf16(&tv, a.v, W, a.T, a.ld_v, 64, 128, f16) ||
      !encode_tmap_2d_bf16(&tdo, A.dout, W, a.T, A.ld_do, 64, 128, f16) ||
      !encode_tmap_2d_bf16(&tbt, A.bias_t, kQTile, a.max_pairs * a.bias_heads * kQTile, kQTile, 64, 128, true) ||
      !encode_tmap_2d_bf16(&tdx, A.dxt, kQTile, a.max_pairs * a.H * kQTile, kQTile, 64, 128, f16) ||
      !encode_tmap_2d_out(&tdq, A.dq, kDtF32, W, a.T, A.ld_g, 32, 128))
    return cudaErrorInvalidValue;
  auto kern = f16 ? attn_bwd_tc_kernel<true> : attn_bwd_tc_kernel<false>;
  e = ensure_smem_attr(reinterpret_cast<const void*>(kern), BwdSmem::kTotal);
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM (the units beyond the grid come from the work list's counter)
  const long long units = a.capacity * a.H;
  const long long blocks = units < sm_count() ? units : sm_count();
  if (!A.sched) return cudaErrorInvalidValue;
  e = prof_record(kProfAttnBwd, false, st);
  if (e == cudaSuccess)
    e = launch_pdl(kern, dim3(static_cast<unsigned>(blocks)), dim3(kThreadsB), BwdSmem::kTotal, st, tq, tk, tv, tdo,
                   tbt, tdx, tdq, A, wait_ctl(a.status));
  if (e == cudaSuccess) e = prof_record(kProfAttnBwd, true, st);
  if (e != cudaSuccess) return e;
  auto tg = f16 ? attn_table_grad_kernel<true> : attn_table_grad_kernel<false>;
  cudaStream_t ts = st;
  if (side) {   // fork: the table gradients overlap what the caller launches next on st
    e = cudaEventRecord(side->fork, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side->stream, side->fork, 0);
    if (e != cudaSuccess) return e;
    ts = side->stream;
  }
  e = prof_record(kProfTableGrad, false, ts);
  if (e == cudaSuccess)
    e = launch_pdl(tg, dim3(static_cast<unsigned>(bias_grid_pairs(a.max_pairs, a.bias_heads) * 2), 2,
                            static_cast<unsigned>(a.bias_heads)),
                   dim3(kTgThreads), 0, ts, A);
  if (e == cudaSuccess) e = prof_record(kProfTableGrad, true, ts);
  return e;
}

}  // namespace hstu
