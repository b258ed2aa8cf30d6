// gemm_sm100.cu - the layer's projection GEMMs on the 5th-generation tensor cores.
//
// C[M, N] = A[M, K] * B[N, K]^T with 16-bit operands (both bf16 or both fp16) and fp32 accumulation
// in tensor memory.
// Each operand is either K-major (row-major [rows, K]) or MN-major (row-major [K, rows]), so the
// forward projections (X W1^T, G W2^T) and the backward ones (dY W2, dZ W1, dY^T G, dZ^T X)
// share one kernel. Operand tiles arrive by TMA (128-byte swizzle) into a 4-deep ring; one thread
// issues tcgen05.mma (M=128, N=256, K=16) into TMEM; eight warps run the fused epilogue:
//   SILU:   Z = acc + b;  out0 = SiLU(Z) (the U|V|Q|K activations), out1 = Z (optional)
//   LINEAR: Y = acc (+ b) (+ R);  out0 = Y, out1 = a second copy of Y in out1's dtype (optional;
//           the fp16 copy a stacked layer's f1 reads)
//   ATOMIC: out0 += acc (fp32 reductions for split-K weight gradients)
// ("4.4 Scaling Recommendation Models", Generative Recommenders and HSTU: f1 with phi1 = SiLU
// and the split into U, V, Q, K; f2 followed by the residual of the "Code" sketch.)
// One launch can run two independent products (the backward's dY W2 with dY^T G, and dZ W1 with
// dZ^T X): their work units share the persistent CTAs, taken largest first from a global counter,
// so neither product's last partial wave leaves SMs idle.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "hstu_internal.h"
#include "sm100_ptx.cuh"
#include "worklist.cuh"

namespace hstu {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;        // every tile is 128 x 256: one tcgen05.mma (M=128, K=16) costs the
                                // same issue time at N = 64, 128 or 256, so N = 256 is the only
                                // width that runs the tensor pipe at full rate
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kEpiWarps = 8;    // 2 per TMEM lane quadrant, each on half of the tile's columns
constexpr int kProdWarps = 2;                    // warps 8, 9: TMA producers of alternate stage slots
constexpr int kProdWarp0 = kEpiWarps;
constexpr int kMmaWarp = kProdWarp0 + kProdWarps;   // warp 10: MMA issue
constexpr int kSchedWarp = kMmaWarp + 1;            // warp 11: work-unit scheduler
constexpr int kThreads = 32 * (kSchedWarp + 1);     // 12 warps: 168 registers a thread
static_assert(kStages % kProdWarps == 0, "each producer warp owns whole stage slots");
constexpr int kBoxBytes = 4096; // one epilogue staging box: 32 rows x 128 bytes
constexpr int kRing = 8;        // work-unit ring between the scheduler and the other roles
constexpr int kRingReaders = kProdWarps + 1 + kEpiWarps;

struct GemmSmem {
  static constexpr int kABytes = kBM * kBK * 2;      // 16 KB
  static constexpr int kBBytes = kBN * kBK * 2;      // 32 KB
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kOut = kStages * kStageBytes;  // one staging box per epilogue warp
  static constexpr int kBarOff = kOut + kEpiWarps * kBoxBytes;
  // full[S] | empty[S] | acc_full[2] | acc_empty[2] | ring_full[R] | ring_empty[R] | ring_got[R]
  static constexpr int kNumBars = 2 * kStages + 4 + 3 * kRing;
  static constexpr int kMiscOff = kBarOff + 8 * kNumBars;   // tmem slot, abort flag, ring[R]
  static constexpr int kTotal = kMiscOff + 8 + 4 * kRing + 1024;   // + alignment slack
};
static_assert(GemmSmem::kTotal <= 232448, "shared memory per CTA");

__host__ __device__ __forceinline__ int dt_size(int dt) { return dt == kDtF32 ? 4 : 2; }

// One GEMM of a launch. Its work units are (m tile, n tile, k split) triples, k split fastest.
struct GemmProb {
  int M, N, num_kb, kb_per, tiles_n, splits, units;
  int a_mn, b_mn;
  uint32_t idesc;
  GemmEpilogue epi;
};

// The tensor maps of one problem (TMA reads them from kernel parameter space).
struct GemmMaps {
  CUtensorMap a, b, o0, o1;
};

// A launch runs one or two independent GEMMs: units [0, p[0].units) are the first problem's,
// the rest the second's. With `sched` the CTAs take units from a global counter (largest units
// should come first); without it CTA c runs units c, c + grid, c + 2 grid, ...
struct GemmLaunch {
  GemmProb p[2];
  int nprob, total;
  int* sched;   // [0] next unit, [1] CTAs finished; zero between launches (the last CTA resets them)
  int has_wl;   // static launches: the last CTA's scheduler warp (idle then) computes this work list
  WorklistArgs wl;
};

struct Unit {
  int prob, m0, n0, kb0, kb1;
};

__device__ __forceinline__ Unit decode_unit(const GemmLaunch& L, int u) {
  Unit w;
  w.prob = (L.nprob > 1 && u >= L.p[0].units) ? 1 : 0;
  const GemmProb& q = L.p[w.prob];
  const int t = w.prob ? u - L.p[0].units : u;
  const int ks = t % q.splits;
  const int rest = t / q.splits;
  w.n0 = (rest % q.tiles_n) * kBN;
  w.m0 = (rest / q.tiles_n) * kBM;
  w.kb0 = ks * q.kb_per;
  w.kb1 = min(q.num_kb, w.kb0 + q.kb_per);
  return w;
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

// Per-warp epilogue staging: one box of 32 rows x 128 bytes in the 128-byte swizzled layout of the
// output tensor maps, written row-per-lane (16-byte units XOR-ed with the row: conflict-free) and
// sent by TMA (store or fp32 reduce-add) from lane 0, which first waits until its previous box has
// been read out of shared memory.
struct EpiStage {
  uint8_t* box;
  __device__ __forceinline__ void emit(const CUtensorMap* map, bool reduce, int x, int y, const uint32_t* w) {
    const int lane = threadIdx.x & 31;
    if (lane == 0) bulk_wait_group_read<0>();
    __syncwarp();
    uint8_t* row = box + lane * 128;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      *reinterpret_cast<uint4*>(row + ((u ^ (lane & 7)) << 4)) = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (reduce) tma_reduce_add_2d(map, smem_u32(box), x, y);
      else tma_store_2d(map, smem_u32(box), x, y);
      bulk_commit_group();
    }
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

// Persistent tensor-core GEMM over the work units of one or two problems. Roles of a CTA:
//   warps 0-7   epilogue: TMEM -> registers -> fused epilogue -> TMA stores
//   warps 8, 9  TMA producers, warp 8 + p filling the stage slots s with s % 2 == p (an issuing warp
//               keeps about one stage's copies in flight; two warps stay ahead of the MMAs of
//               128 x 256 x 64 k-blocks)
//   warp 10     one thread issues tcgen05.mma (M=128, N=256, K=16) into a double-buffered TMEM
//               accumulator, so the epilogue of one unit overlaps the next unit's mainloop
//   warp 11     scheduler (dynamic mode): takes the CTA's next unit from the global counter one unit
//               ahead of the producers and publishes it to the other roles through a ring
__global__ void __launch_bounds__(kThreads, 1)
gemm_bf16_tc_kernel(const __grid_constant__ GemmMaps m0, const __grid_constant__ GemmMaps m1,
                    const __grid_constant__ GemmLaunch L, WaitCtl ctl) {
  pdl_enter();
  using S = GemmSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  auto full = [&](int s) { return smem_u32(&bars[s]); };
  auto empty = [&](int s) { return smem_u32(&bars[kStages + s]); };
  auto acc_full = [&](int b) { return smem_u32(&bars[2 * kStages + b]); };
  auto acc_empty = [&](int b) { return smem_u32(&bars[2 * kStages + 2 + b]); };
  auto ring_full = [&](int r) { return smem_u32(&bars[2 * kStages + 4 + r]); };
  auto ring_empty = [&](int r) { return smem_u32(&bars[2 * kStages + 4 + kRing + r]); };
  auto ring_got = [&](int r) { return smem_u32(&bars[2 * kStages + 4 + 2 * kRing + r]); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ring = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool dynamic = L.sched != nullptr;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(full(i), 1);
      mbar_init(empty(i), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full(b), 1);
      mbar_init(acc_empty(b), 32 * kEpiWarps);
    }
    for (int r = 0; r < kRing; ++r) {
      mbar_init(ring_full(r), 1);
      mbar_init(ring_empty(r), kRingReaders);
      mbar_init(ring_got(r), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kProdWarp0 && lane == 0) {
    tma_prefetch_desc(&m0.a);
    tma_prefetch_desc(&m0.b);
    if (L.nprob > 1) {
      tma_prefetch_desc(&m1.a);
      tma_prefetch_desc(&m1.b);
    }
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 2 * kBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_slot;

  // Unit i of this CTA, for one reading thread (false: the wait gave up). In dynamic mode the
  // reader frees the ring slot as soon as it holds the value; producer warp 0 also tells the
  // scheduler that it started the unit, which paces the next take from the global counter.
  auto take_unit = [&](int i, int& u) -> bool {
    if (!dynamic) {
      u = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
      return true;
    }
    const int r = i % kRing;
    if (!mbar_wait(ring_full(r), (i / kRing) & 1, abort_flag, ctl)) return false;
    u = ring[r];
    mbar_arrive(ring_empty(r));
    if (warp == kProdWarp0) mbar_arrive(ring_got(r));
    return true;
  };
  // the same for a whole warp (lane 0 reads, every lane gets the result)
  auto take_unit_warp = [&](int i, int& u) -> bool {
    int v = 0;
    bool ok = true;
    if (lane == 0) ok = take_unit(i, v);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    u = __shfl_sync(0xffffffffu, v, 0);
    return ok;
  };

  if (warp >= kProdWarp0 && warp < kMmaWarp) {
    // producer p: the CTA's k-blocks g (counted over all its units) with g % 2 == p, stage slot g % S
    const int p = warp - kProdWarp0;
    int g = 0;
    for (int i = 0;; ++i) {
      int u;
      if (!take_unit_warp(i, u) || u >= L.total) break;
      const Unit w = decode_unit(L, u);
      const GemmProb& q = L.p[w.prob];
      const GemmMaps& mp = w.prob ? m1 : m0;
      const int nkb = w.kb1 - w.kb0;
      const int a_boxes = q.a_mn ? 2 : 1;                 // A: 1 K-major box or 2 MN-major halves
      const int boxes = a_boxes + (q.b_mn ? kBN / 64 : 1);   // B: 1 K-major box or 4 MN-major boxes
      bool ok = true;
      for (int j = (p - g % kProdWarps + kProdWarps) % kProdWarps; j < nkb; j += kProdWarps) {
        const int gg = g + j;
        const int s = gg % kStages;
        bool free_ok = true;   // lane 0 waits; the result is made warp-uniform
        if (lane == 0 && gg >= kStages) free_ok = mbar_wait(empty(s), ((gg / kStages) - 1) & 1, abort_flag, ctl);
        if (!__shfl_sync(0xffffffffu, free_ok ? 1 : 0, 0)) {
          ok = false;
          break;
        }
        const uint32_t sa = smem_u32(smem + s * S::kStageBytes);
        const uint32_t sb = sa + S::kABytes;
        const int kx = (w.kb0 + j) * kBK;
        if (lane == 0) mbar_arrive_expect_tx(full(s), S::kStageBytes);
        __syncwarp();
        if (lane < a_boxes) {
          if (!q.a_mn) tma_load_2d(sa, &mp.a, full(s), kx, w.m0);
          else tma_load_2d(sa + lane * 8192, &mp.a, full(s), w.m0 + 64 * lane, kx);
        } else if (lane < boxes) {
          const int c = lane - a_boxes;
          if (!q.b_mn) tma_load_2d(sb, &mp.b, full(s), kx, w.n0);
          else tma_load_2d(sb + c * 8192, &mp.b, full(s), w.n0 + 64 * c, kx);
        }
      }
      if (!ok) break;
      g += nkb;
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t sa0 = smem_u32(smem), sb0 = sa0 + S::kABytes;
      int g = 0;
      for (int i = 0;; ++i) {
        int u;
        if (!take_unit(i, u) || u >= L.total) break;
        const Unit w = decode_unit(L, u);
        const GemmProb& q = L.p[w.prob];
        // descriptors of stage 0's A and B tiles; stages and K steps are offsets from them
        const uint64_t a_desc0 = q.a_mn ? make_sdesc_sw128(sa0, 8192, 1024) : make_sdesc_sw128(sa0, 16, 1024);
        const uint64_t b_desc0 = q.b_mn ? make_sdesc_sw128(sb0, 8192, 1024) : make_sdesc_sw128(sb0, 16, 1024);
        const uint32_t a_kstep = q.a_mn ? 2048 : 32, b_kstep = q.b_mn ? 2048 : 32;
        const int buf = i & 1;
        if (i >= 2 && !mbar_wait(acc_empty(buf), ((i >> 1) - 1) & 1, abort_flag, ctl)) break;
        tc_fence_after();
        const uint32_t acc = tmem_acc + buf * kBN;
        bool ok = true;
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++g) {
          const int s = g % kStages;
          if (!mbar_wait(full(s), (g / kStages) & 1, abort_flag, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad0 = sdesc_add(a_desc0, s * S::kStageBytes);
          const uint64_t bd0 = sdesc_add(b_desc0, s * S::kStageBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_f16_ss(acc, sdesc_add(ad0, kk * a_kstep), sdesc_add(bd0, kk * b_kstep), q.idesc,
                        (kb > w.kb0 || kk > 0) ? 1u : 0u);
          umma_commit(empty(s));
        }
        if (!ok) break;
        umma_commit(acc_full(buf));
      }
    }
  } else if (warp == kSchedWarp) {
    if (dynamic && lane == 0) {
      for (int i = 0;; ++i) {
        const int r = i % kRing;
        // pace: take unit i once the producers have started unit i - 1
        if (i >= 1 && !mbar_wait(ring_got((i - 1) % kRing), ((i - 1) / kRing) & 1, abort_flag, ctl)) break;
        const int u = i == 0 ? static_cast<int>(blockIdx.x) : static_cast<int>(gridDim.x) + atomicAdd(L.sched, 1);
        if (i >= kRing && !mbar_wait(ring_empty(r), ((i / kRing) - 1) & 1, abort_flag, ctl)) break;
        ring[r] = u;
        mbar_arrive(ring_full(r));
        if (u >= L.total) break;
      }
    } else if (L.has_wl && blockIdx.x == gridDim.x - 1) {
      worklist_warp(L.wl);   // the CTA with the fewest units of the stride (whole warp)
    }
  } else {
    // epilogue warps 0-7: TMEM lanes 32 (warp % 4) .. +31 = output rows m0 + 32 (warp % 4) + lane,
    // columns [128 (warp / 4), +128) of the tile
    const int quad = warp & 3, chalf = warp >> 2;
    EpiStage es{smem + S::kOut + warp * kBoxBytes};
    for (int i = 0;; ++i) {
      int u;
      if (!take_unit_warp(i, u) || u >= L.total) break;
      const Unit w = decode_unit(L, u);
      const GemmProb& q = L.p[w.prob];
      const GemmEpilogue& epi = q.epi;
      const GemmMaps& mp = w.prob ? m1 : m0;
      const int buf = i & 1;
      if (!mbar_wait(acc_full(buf), (i >> 1) & 1, abort_flag, ctl)) break;
      tc_fence_after();
      const int row = w.m0 + quad * 32 + lane;
      const bool row_ok = row < q.M;
      const int ybox = w.m0 + quad * 32;
      constexpr int kChunks = kBN / 128;   // 64-column chunks per warp
#pragma unroll 1
      for (int c = 0; c < kChunks; ++c) {
        const int col = chalf * (kBN / 2) + c * 64;   // within the tile
        const int n = w.n0 + col;
        float v[64];
        {
          uint32_t r[32];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            tmem_ld_32x32b_x32(tmem_acc + buf * kBN + (static_cast<uint32_t>(quad * 32) << 16) + col + 32 * h, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[32 * h + j] = __uint_as_float(r[j]);
          }
        }
        if (c == kChunks - 1) {   // this warp's part of the accumulator is in registers: release it
          tc_fence_before();
          mbar_arrive(acc_empty(buf));
        }
        if (n >= q.N) continue;
        if (epi.kind == kEpiAtomic) {
          emit64(es, &mp.o0, kDtF32, true, n, ybox, v, q.N);
          continue;
        }
        if (epi.bias) {
          const float4* bp = reinterpret_cast<const float4*>(epi.bias + n);
#pragma unroll
          for (int k4 = 0; k4 < 16; ++k4) {
            const float4 b4 = (n + 4 * k4 < q.N) ? __ldg(bp + k4) : make_float4(0.f, 0.f, 0.f, 0.f);
            v[4 * k4] += b4.x; v[4 * k4 + 1] += b4.y; v[4 * k4 + 2] += b4.z; v[4 * k4 + 3] += b4.w;
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
          if (epi.out1) emit64(es, &mp.o1, epi.out1_dt, false, n, ybox, v, q.N);
#pragma unroll
          for (int j = 0; j < 64; ++j) v[j] = silu_tanh(v[j]);
        } else if (epi.resid) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float rv[32];
            if (row_ok && n + 32 * h < q.N) {
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
        emit64(es, &mp.o0, epi.out0_dt, false, n, ybox, v, q.N);
        if (epi.kind == kEpiLinear && epi.out1) emit64(es, &mp.o1, epi.out1_dt, false, n, ybox, v, q.N);
      }
    }
    if (lane == 0) bulk_wait_group_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_acc, 2 * kBN);
  }
  if (dynamic && threadIdx.x == 0) {
    // every take from the counter of this launch happened before its CTA got here: the last CTA
    // leaves both counters at zero for the next launch that uses them
    __threadfence();
    if (atomicAdd(L.sched + 1, 1) == static_cast<int>(gridDim.x) - 1) {
      atomicExch(L.sched, 0);
      atomicExch(L.sched + 1, 0);
    }
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

bool encode_problem(const GemmArgs& g, GemmMaps& m) {
  // A: K-major -> [M rows, K] box {64, 128}; MN-major -> [K rows, M] box {64, 64}
  if (!g.a_mn) {
    if (!encode_tmap_2d_bf16(&m.a, g.A, g.K, g.M, g.lda, 64, kBM, g.f16)) return false;
  } else if (!encode_tmap_2d_bf16(&m.a, g.A, g.M, g.K, g.lda, 64, 64, g.f16)) {
    return false;
  }
  // B: K-major -> [N rows, K] box {64, 256}; MN-major -> [K rows, N] box {64, 64}
  if (!g.b_mn) {
    if (!encode_tmap_2d_bf16(&m.b, g.B, g.K, g.N, g.ldb, 64, kBN, g.f16)) return false;
  } else if (!encode_tmap_2d_bf16(&m.b, g.B, g.N, g.K, g.ldb, 64, 64, g.f16)) {
    return false;
  }
  // outputs: boxes of 32 rows x 128 bytes
  const int dt0 = g.epi.kind == kEpiAtomic ? kDtF32 : g.epi.out0_dt;
  if (!encode_tmap_2d_out(&m.o0, g.epi.out0, dt0, g.N, g.M, g.epi.ld_out0, 128 / dt_size(dt0), 32)) return false;
  if (g.epi.out1) {
    if (!encode_tmap_2d_out(&m.o1, g.epi.out1, g.epi.out1_dt, g.N, g.M, g.epi.ld_out1, 128 / dt_size(g.epi.out1_dt), 32))
      return false;
  } else {
    m.o1 = m.o0;
  }
  return true;
}

GemmProb make_prob(const GemmArgs& g) {
  GemmProb P{};
  P.M = static_cast<int>(g.M);
  P.N = static_cast<int>(g.N);
  P.num_kb = static_cast<int>((g.K + kBK - 1) / kBK);
  const int splits = g.splits < 1 ? 1 : g.splits;
  P.kb_per = (P.num_kb + splits - 1) / splits;
  P.splits = (P.num_kb + P.kb_per - 1) / P.kb_per;
  P.tiles_n = static_cast<int>((g.N + kBN - 1) / kBN);
  const int tiles_m = static_cast<int>((g.M + kBM - 1) / kBM);
  P.units = tiles_m * P.tiles_n * P.splits;
  P.a_mn = g.a_mn ? 1 : 0;
  P.b_mn = g.b_mn ? 1 : 0;
  P.idesc = make_idesc_f16kind(kBM, kBN, P.a_mn, P.b_mn, g.f16);
  P.epi = g.epi;
  return P;
}

}  // namespace

cudaError_t gemm_bf16_group(const GemmArgs* gs, int n, int* sched, cudaStream_t st, const WorklistArgs* side) {
  if (!gs || n < 1 || n > 2) return cudaErrorInvalidValue;
  if (side && (sched || side->B < 0 || side->B > 32)) return cudaErrorInvalidValue;
  GemmMaps maps[2];
  GemmLaunch L{};
  int k = 0;
  int* status = nullptr;
  for (int i = 0; i < n; ++i) {
    const GemmArgs& g = gs[i];
    if (g.M <= 0 || g.N <= 0) continue;   // an empty product: nothing to compute
    if (g.K <= 0 || (g.splits > 1 && g.epi.kind != kEpiAtomic)) return cudaErrorInvalidValue;
    if (!encode_problem(g, maps[k])) return cudaErrorInvalidValue;
    L.p[k] = make_prob(g);
    if (!status) status = g.status;
    ++k;
  }
  if (k == 0) return side ? cudaErrorInvalidValue : cudaSuccess;
  if (k == 1) maps[1] = maps[0];
  L.nprob = k;
  const int64_t total = static_cast<int64_t>(L.p[0].units) + (k > 1 ? L.p[1].units : 0);
  if (total >= (1ll << 30)) return cudaErrorInvalidValue;
  L.total = static_cast<int>(total);
  L.sched = sched;
  if (side) {
    L.has_wl = 1;
    L.wl = *side;
  }
  auto kern = gemm_bf16_tc_kernel;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), GemmSmem::kTotal);
  if (e != cudaSuccess) return e;
  const int grid = L.total < sm_count() ? L.total : sm_count();
  return launch_pdl(kern, dim3(grid), dim3(kThreads), GemmSmem::kTotal, st, maps[0], maps[1], L, wait_ctl(status));
}

cudaError_t gemm_bf16(const GemmArgs& g, cudaStream_t st, const WorklistArgs* side) {
  if (g.M <= 0 || g.N <= 0) return side ? cudaErrorInvalidValue : cudaSuccess;
  if (g.K <= 0) return cudaErrorInvalidValue;
  return gemm_bf16_group(&g, 1, nullptr, st, side);
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
