// jagged_norm.cu - HBM-bound kernels: jagged work list, time-bucket debug output, LayerNorm (.) U
// gating, dtype conversion, and the timeout probe of the failure path.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hstu_internal.h"
#include "sm100_ptx.cuh"
#include "time_bucket_dev.cuh"
#include "bias_tile.cuh"
#include "vec_io.cuh"
#include "worklist.cuh"

namespace hstu {

namespace {

// Short sequences share a tile (worklist.cuh: pack): greedy in batch order inside chunks of 32
// sequences (chunks are packed independently, so a block packs them in parallel).
__device__ void pack_chunk(const int64_t* __restrict__ off, int b0, int b1, int32_t* pack) {
  int i = b0;
  while (i < b1) {
    const long long n = off[i + 1] - off[i];
    if (n <= 0 || n > kPackMaxLen) {
      pack[i++] = 1;
      continue;
    }
    long long total = n;
    int k = 1;
    while (i + k < b1) {
      const long long m = off[i + k + 1] - off[i + k];
      if (m > kPackMaxLen || total + m > kQTile) break;
      total += m;
      ++k;
    }
    pack[i] = k;
    for (int j = 1; j < k; ++j) pack[i + j] = 0;
    i += k;
  }
}

// ----------------------------------------------------------------------------------------------
// Jagged tile work list ("4.4 Scaling Recommendation Models", Efficiency tricks: kernels over
// variable-length sequences). One block: emits (b, t) for every query tile t of every sequence,
// tiles with more causal key tiles first, ties by increasing b; with `pack`, a pack of k >= 2 short
// sequences is one item (b, -k) among the one-tile items. Also validates the offsets:
// offsets[0] == 0, non-decreasing, every length <= max_len, offsets[B] == T; a violation records
// kDevBadInput and empties the list so no later kernel reads out of bounds.
// ----------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(1024)
worklist_kernel(const int64_t* __restrict__ off, int B, int64_t T, int max_len, int32_t* items,
                int32_t* count, int* status, long long* pair_base, int32_t* kitems, int32_t* kcount,
                int32_t* sched, int32_t* pack, int32_t* urec, int32_t* sched2) {
  pdl_enter();
  if (threadIdx.x == 0) {   // the persistent attention kernels' unit (and finished-CTA) counters
    if (sched) sched[0] = 0;
    if (sched2) sched2[0] = sched2[1] = 0;
  }
  __shared__ int s_warp[32];
  __shared__ int s_max_tiles;
  __shared__ int s_bad;
  __shared__ int s_base;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    s_max_tiles = 0;
    s_bad = (B < 0 || off[0] != 0 || off[B] != T) ? 1 : 0;
    s_base = 0;
  }
  __syncthreads();
  for (int b = tid; b < B; b += blockDim.x) {
    const int64_t n = off[b + 1] - off[b];
    if (n < 0 || n > max_len) atomicOr(&s_bad, 1);
    else atomicMax(&s_max_tiles, static_cast<int>((n + kQTile - 1) / kQTile));
  }
  __syncthreads();
  if (s_bad) {
    if (tid == 0) {
      *count = 0;
      if (kcount) *kcount = 0;
      report_error(status, kDevBadInput);
      if (pair_base) pair_base[B > 0 ? B : 0] = 0;
    }
    return;
  }
  const int max_tiles = s_max_tiles;
  constexpr int kStageSeqs = 8192, kStageTiles = 256;
  __shared__ int s_nt[kStageSeqs];
  __shared__ int s_start[kStageTiles];
  if (B <= kStageSeqs && max_tiles <= kStageTiles) {
    // Fast path. Tile counts staged in shared memory (0 for a pack member, whose rows the pack's
    // first sequence covers); warp w owns the tile indices t = w, w+32, ...
    if (pack) {
      for (int c = tid; c * 32 < B; c += blockDim.x) pack_chunk(off, 32 * c, min(B, 32 * c + 32), pack);
      __syncthreads();
    }
    for (int b = tid; b < B; b += blockDim.x)
      s_nt[b] = (pack && pack[b] == 0) ? 0 : static_cast<int>((off[b + 1] - off[b] + kQTile - 1) / kQTile);
    __syncthreads();
    for (int t = warp; t < max_tiles; t += 32) {
      int c = 0;
      for (int b0 = 0; b0 < B; b0 += 32) {
        const int b = b0 + lane;
        c += __popc(__ballot_sync(0xffffffffu, b < B && s_nt[b] > t));
      }
      if (lane == 0) s_start[t] = c;
    }
    __syncthreads();
    if (tid == 0) {   // exclusive prefix in decreasing t (longest tiles first)
      int run = 0;
      for (int t = max_tiles - 1; t >= 0; --t) {
        const int c = s_start[t];
        s_start[t] = run;
        run += c;
      }
      s_base = run;
    }
    __syncthreads();
    for (int t = warp; t < max_tiles; t += 32) {
      int pos = s_start[t];
      for (int b0 = 0; b0 < B; b0 += 32) {
        const int b = b0 + lane;
        const bool flag = b < B && s_nt[b] > t;
        const unsigned m = __ballot_sync(0xffffffffu, flag);
        if (flag) {
          const int p = pos + __popc(m & ((1u << lane) - 1u));
          const int pk = pack ? pack[b] : 1;
          items[2 * p] = b;
          items[2 * p + 1] = pk >= 2 ? -pk : t;
          if (kitems) {   // the key tile that visits t + 1 query tiles: the same cost order
            kitems[2 * p] = b;
            kitems[2 * p + 1] = pk >= 2 ? -pk : s_nt[b] - 1 - t;
          }
        }
        pos += __popc(m);
      }
    }
    __syncthreads();
  } else for (int t = max_tiles - 1; t >= 0; --t) {
    // (large batches: no packing)
    if (pack && t == max_tiles - 1)
      for (int b = tid; b < B; b += blockDim.x) pack[b] = 1;
    for (int c0 = 0; c0 < B; c0 += blockDim.x) {
      const int b = c0 + tid;
      bool flag = false;
      if (b < B) flag = (off[b + 1] - off[b] + kQTile - 1) / kQTile > t;
      const unsigned m = __ballot_sync(0xffffffffu, flag);
      if (lane == 0) s_warp[warp] = __popc(m);
      __syncthreads();
      if (warp == 0) {
        const int v = s_warp[lane];
        int inc = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, inc, d);
          if (lane >= d) inc += y;
        }
        s_warp[lane] = inc - v;   // exclusive prefix over warps
      }
      __syncthreads();
      const int pos = s_base + s_warp[warp] + __popc(m & ((1u << lane) - 1u));
      if (flag) {
        items[2 * pos] = b;
        items[2 * pos + 1] = t;
        if (kitems) {
          kitems[2 * pos] = b;
          kitems[2 * pos + 1] = static_cast<int>((off[b + 1] - off[b] + kQTile - 1) / kQTile) - 1 - t;
        }
      }
      __syncthreads();
      if (tid == blockDim.x - 1) s_base = pos + (flag ? 1 : 0);
      __syncthreads();
    }
  }
  if (tid == 0) {
    *count = s_base;
    if (kcount) *kcount = s_base;
  }
  if (!pair_base) return;
  // pair_base[b] = sum_{b' < b} nt_b' (nt_b' + 1) / 2: index of sequence b's first causal
  // (query tile, key tile) pair; pair_base[B] is the total.
  __shared__ long long s_wsum[32];
  __shared__ long long s_run;
  if (tid == 0) s_run = 0;
  __syncthreads();
  for (int c0 = 0; c0 < B; c0 += blockDim.x) {
    const int b = c0 + tid;
    long long v = 0;
    if (b < B) {
      const long long nt = (off[b + 1] - off[b] + kQTile - 1) / kQTile;
      v = nt * (nt + 1) / 2;
    }
    long long inc = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, inc, d);
      if (lane >= d) inc += y;
    }
    if (lane == 31) s_wsum[warp] = inc;
    __syncthreads();
    if (warp == 0) {
      const long long w = s_wsum[lane];
      long long winc = w;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, winc, d);
        if (lane >= d) winc += y;
      }
      s_wsum[lane] = winc - w;
    }
    __syncthreads();
    const long long excl = s_run + s_wsum[warp] + inc - v;
    if (b < B) pair_base[b] = excl;
    __syncthreads();
    if (tid == blockDim.x - 1) s_run = excl + v;
    __syncthreads();
  }
  if (tid == 0) pair_base[B] = s_run;
  if (!urec) return;
  __syncthreads();
  write_unit_records(off, items, s_base, pair_base, urec, tid, blockDim.x);
}

// The same lists for batches of at most 32 sequences, from a single warp (worklist.cuh).
__global__ void __launch_bounds__(32)
worklist_warp_kernel(const int64_t* __restrict__ off, int B, int64_t T, int max_len, int32_t* items, int32_t* count,
                     int* status, long long* pair_base, int32_t* kitems, int32_t* kcount, int32_t* sched,
                     int32_t* pack, int32_t* urec, int32_t* sched2) {
  pdl_enter();
  worklist_warp(WorklistArgs{off, B, T, max_len, items, count, status, pair_base, kitems, kcount, sched, pack, urec,
                             sched2});
}

// Test surface of the attention's time-bucket index: block (x = qt * mt + kt, y = b) writes
// bucket(t_i - t_j) of every query i of tile qt and key j of tile kt of sequence b (all tiles, not
// only causal ones) into the n_b x n_b matrix at out + sq_off[b]. It stages the tile's timestamps,
// takes the 32-bit or 64-bit path and evaluates each element with exactly the functions the
// attention's bias tiles use (bias_tile.cuh), so a bit-exact check of this output checks theirs.
__global__ void __launch_bounds__(kBiasThreads)
time_bucket_tile_kernel(const int64_t* __restrict__ off, const int64_t* __restrict__ ts, int nb, int mt,
                        const int64_t* __restrict__ sq_off, uint8_t* __restrict__ out) {
  __shared__ TileTimes s_t;
  __shared__ long long s_tau[kTauEntries];
  __shared__ int s_tau32[kTauEntries];
  const int b = blockIdx.y;
  const int qt = blockIdx.x / mt, kt = blockIdx.x - qt * mt;
  const long long seq0 = off[b];
  const long long n = off[b + 1] - seq0;
  if (static_cast<long long>(qt) * kQTile >= n || static_cast<long long>(kt) * kQTile >= n) return;
  tile_times_load(s_t, ts, seq0, static_cast<int>(n), qt * kQTile, kt * kQTile);
  for (int e = threadIdx.x; e < kTauEntries; e += kBiasThreads) {
    s_tau[e] = g_time_taus[e];
    s_tau32[e] = g_time_taus32[e];
  }
  __syncthreads();
  const bool fast = tile_times_finish(s_t);
  uint8_t* dst = out + sq_off[b];
  for (int e = threadIdx.x; e < kQTile * kQTile; e += kBiasThreads) {
    const int r = e >> 7, c = e & 127;
    const long long i = static_cast<long long>(qt) * kQTile + r, j = static_cast<long long>(kt) * kQTile + c;
    if (i < n && j < n) dst[i * n + j] = static_cast<uint8_t>(tile_bucket<false>(s_t, fast, r, c, s_tau, s_tau32, nb));
  }
}

// ----------------------------------------------------------------------------------------------
// LayerNorm (.) U ("4.4 Scaling Recommendation Models", Generative Recommenders and HSTU, third
// equation Norm(AV) (.) U; "HSTU: The First Exploration of the Scaling Law", 7.1.4 Innovation 3):
// one warp per token (lane l holds 4-feature groups 4 l + 128 k, or [l VPT, (l+1) VPT) for small D);
// mean and variance by warp shuffles (two passes over registers), fp32 statistics stored for the
// backward.
// ----------------------------------------------------------------------------------------------
template <int VPT, int OT, int UT, int GT>
__global__ void __launch_bounds__(256, VPT <= 16 ? 4 : 2)
norm_gate_kernel(int64_t T, const void* __restrict__ o, int64_t ld_o, const void* __restrict__ u,
                 int64_t ld_u, const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
                 void* __restrict__ g, float* __restrict__ mu_out, float* __restrict__ rstd_out) {
  constexpr int D = VPT * 32;
  // gamma | beta staged once per block (they are parameters, not written by an earlier grid)
  __shared__ __align__(16) float s_gb[2 * D];
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    s_gb[c] = gamma[c];
    s_gb[D + c] = beta[c];
  }
  pdl_enter();
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= T) return;
  // D >= 128: lane l holds features 128 k + 4 l + i (every warp access covers 128 consecutive
  // features); smaller D: features [l VPT, (l+1) VPT)
  constexpr bool kGrouped = VPT % 4 == 0;
  auto col = [&](int k) { return kGrouped ? 128 * k + 4 * lane : lane * VPT; };
  constexpr int KG = kGrouped ? VPT / 4 : 1, W = kGrouped ? 4 : VPT;
  float x[VPT], uu[VPT];
#pragma unroll
  for (int k = 0; k < KG; ++k) {
    load_vec<W, OT>(o, row * ld_o + col(k), x + W * k);
    load_vec<W, UT>(u, row * ld_u + col(k), uu + W * k);
  }
  float s = 0.0f;
#pragma unroll
  for (int e = 0; e < VPT; ++e) s += x[e];
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
  const float mean = s * (1.0f / D);
  float q = 0.0f;
#pragma unroll
  for (int e = 0; e < VPT; ++e) {
    const float d = x[e] - mean;
    q = fmaf(d, d, q);
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) q += __shfl_xor_sync(0xffffffffu, q, m);
  const float rstd = rsqrtf(q * (1.0f / D) + eps);
#pragma unroll
  for (int k = 0; k < KG; ++k) {
    float gm[W], bt[W];
    load_vec<W, kDtF32>(s_gb, col(k), gm);
    load_vec<W, kDtF32>(s_gb + D, col(k), bt);
#pragma unroll
    for (int e = 0; e < W; ++e) x[W * k + e] = fmaf((x[W * k + e] - mean) * rstd, gm[e], bt[e]) * uu[W * k + e];
  }
#pragma unroll
  for (int k = 0; k < KG; ++k) store_vec<W, GT>(g, row * D + col(k), x + W * k);
  if (lane == 0) {
    if (mu_out) mu_out[row] = mean;
    if (rstd_out) rstd_out[row] = rstd;
  }
}

// Bytes of one element of a kDt* type in memory (kDtOne: none).
__host__ __device__ constexpr int dt_bytes(int dt) { return dt == kDtF32 ? 4 : (dt == kDtOne ? 0 : 2); }

// Row slots per warp of the staged kernel below.
constexpr int kNgSlots = 4;

// The same LayerNorm (.) U for D >= 128 with the rows staged by bulk copies: a persistent grid whose
// warps each own kNgSlots row slots in shared memory (O row, then U row) and rows gw, gw + W, ...
// (gw = the warp's global index, W = all warps); lane 0 keeps kNgSlots rows in flight, refilling a
// slot as soon as the warp has read it, so the whole batch is requested at the speed the copy
// engines take it instead of one round trip per warp. Every wait is bounded (ctl).
template <int VPT, int OT, int UT, int GT>
__global__ void __launch_bounds__(256)
norm_gate_staged_kernel(int64_t T, const void* __restrict__ o, int64_t ld_o, const void* __restrict__ u,
                        int64_t ld_u, const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
                        void* __restrict__ g, float* __restrict__ mu_out, float* __restrict__ rstd_out, WaitCtl ctl) {
  constexpr int D = VPT * 32, KG = VPT / 4;
  constexpr int OB = D * dt_bytes(OT), UB = D * dt_bytes(UT), SLOT = OB + UB, S = kNgSlots;
  static_assert(VPT % 4 == 0 && OB % 16 == 0 && UB % 16 == 0, "rows of whole 16-byte chunks");
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t s_bar[8 * S];
  __shared__ int s_abort;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 8 * S; ++i) mbar_init(smem_u32(&s_bar[i]), 1);
    s_abort = 0;
    fence_barrier_init();
  }
  float gm[VPT], bt[VPT];   // parameters: read before the wait for the earlier grid
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
    mbar_arrive_expect_tx(bar, SLOT);
    bulk_load(smem_u32(wslots + sl * SLOT), static_cast<const uint8_t*>(o) + row * ld_o * dt_bytes(OT), OB, bar);
    if constexpr (UB > 0)
      bulk_load(smem_u32(wslots + sl * SLOT + OB), static_cast<const uint8_t*>(u) + row * ld_u * dt_bytes(UT), UB, bar);
  };
  if (lane == 0)
    for (int i = 0; i < S; ++i) issue(i);
  for (long long i = 0;; ++i) {
    const long long row = gw + i * W;
    if (row >= T) break;
    const int sl = static_cast<int>(i % S);
    if (!mbar_wait_warp(smem_u32(&s_bar[warp * S + sl]), static_cast<uint32_t>((i / S) & 1), &s_abort, ctl)) break;
    const uint8_t* so = wslots + sl * SLOT;
    float x[VPT], uu[VPT];
#pragma unroll
    for (int k = 0; k < KG; ++k) {
      load_vec<4, OT>(so, 128 * k + 4 * lane, x + 4 * k);
      load_vec<4, UT>(so + OB, 128 * k + 4 * lane, uu + 4 * k);
    }
    // every lane has read the slot: refill it (generic reads before the copy engine's writes)
    __syncwarp();
    if (lane == 0) {
      fence_proxy_async_smem();
      issue(i + S);
    }
    float s = 0.0f;
#pragma unroll
    for (int e = 0; e < VPT; ++e) s += x[e];
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
    const float mean = s * (1.0f / D);
    float q = 0.0f;
#pragma unroll
    for (int e = 0; e < VPT; ++e) {
      const float d = x[e] - mean;
      q = fmaf(d, d, q);
    }
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) q += __shfl_xor_sync(0xffffffffu, q, m);
    const float rstd = rsqrtf(q * (1.0f / D) + eps);
#pragma unroll
    for (int e = 0; e < VPT; ++e) x[e] = fmaf((x[e] - mean) * rstd, gm[e], bt[e]) * uu[e];
#pragma unroll
    for (int k = 0; k < KG; ++k) store_vec<4, GT>(g, row * D + 128 * k + 4 * lane, x + 4 * k);
    if (lane == 0) {
      if (mu_out) mu_out[row] = mean;
      if (rstd_out) rstd_out[row] = rstd;
    }
  }
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ in, uint16_t* __restrict__ out, int64_t n) {
  const int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i + 3 < n) {
    const float4 v = *reinterpret_cast<const float4*>(in + i);
    *reinterpret_cast<uint2*>(out + i) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  } else {
    for (int64_t k = i; k < n; ++k) {
      __nv_bfloat16 b = __float2bfloat16_rn(in[k]);
      out[k] = *reinterpret_cast<uint16_t*>(&b);
    }
  }
}

// Waits on an mbarrier that nothing arrives at; the bounded wait records kDevTimeout.
__global__ void timeout_probe_kernel(WaitCtl ctl) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, ctl);
  __syncthreads();
}

template <int VPT, int OT, int UT, int GT>
cudaError_t launch_ng(int64_t T, const void* o, int64_t ld_o, const void* u, int64_t ld_u, const float* gamma,
                      const float* beta, float eps, void* g, float* mu, float* rstd, cudaStream_t st, int* status) {
  const int64_t rows8 = (T + 7) / 8;
  cudaError_t e = prof_record(kProfNormFwd, false, st);
  if (e != cudaSuccess) return e;
  // staged rows (D >= 128) need 16-byte aligned row starts; their sizes are whole 16-byte chunks
  bool staged = false;
  if constexpr (VPT % 4 == 0) {
    const auto al16 = [](const void* p, int64_t ld, int bytes) {
      return bytes == 0 || ((reinterpret_cast<uintptr_t>(p) | static_cast<uintptr_t>(ld * bytes)) & 15) == 0;
    };
    if (al16(o, ld_o, dt_bytes(OT)) && al16(u, ld_u, dt_bytes(UT))) {
      staged = true;
      constexpr int kSmem = 8 * kNgSlots * VPT * 32 * (dt_bytes(OT) + dt_bytes(UT));
      auto kern = norm_gate_staged_kernel<VPT, OT, UT, GT>;
      e = ensure_smem_attr(reinterpret_cast<const void*>(kern), kSmem);
      if (e != cudaSuccess) return e;
      const int per_sm = kSmem <= 100 * 1024 ? 2 : 1;
      const int64_t cap = static_cast<int64_t>(sm_count()) * per_sm;
      const int64_t blocks = rows8 < cap ? rows8 : cap;
      e = launch_pdl(kern, dim3(static_cast<unsigned>(blocks)), dim3(256), kSmem, st, T, o, ld_o, u, ld_u, gamma,
                     beta, eps, g, mu, rstd, wait_ctl(status));
    }
  }
  if (!staged)
    e = launch_pdl(norm_gate_kernel<VPT, OT, UT, GT>, dim3(static_cast<unsigned>(rows8)), dim3(256), 0, st, T, o,
                   ld_o, u, ld_u, gamma, beta, eps, g, mu, rstd);
  if (e == cudaSuccess) e = prof_record(kProfNormFwd, true, st);
  return e;
}

}  // namespace

cudaError_t launch_worklist(const int64_t* offsets, int B, int64_t T, int max_len, int32_t* items,
                            int32_t* count, int* status, cudaStream_t st, long long* pair_base, int32_t* kitems,
                            int32_t* kcount, int32_t* sched, int32_t* pack, int32_t* urec, int32_t* sched2) {
  if (urec && !pair_base) return cudaErrorInvalidValue;
  if (B >= 0 && B <= 32)
    return launch_pdl(worklist_warp_kernel, dim3(1), dim3(32), 0, st, offsets, B, T, max_len, items, count, status,
                      pair_base, kitems, kcount, sched, pack, urec, sched2);
  return launch_pdl(worklist_kernel, dim3(1), dim3(1024), 0, st, offsets, B, T, max_len, items, count, status,
                    pair_base, kitems, kcount, sched, pack, urec, sched2);
}

cudaError_t launch_time_buckets(const int64_t* offsets, const int64_t* ts, int B, int64_t T, int max_len,
                                int n_buckets, const int64_t* sq_offsets, uint8_t* out, cudaStream_t st) {
  if (T == 0 || B == 0) return cudaSuccess;
  cudaError_t e = upload_time_taus();
  if (e != cudaSuccess) return e;
  const int mt = (max_len + kQTile - 1) / kQTile;
  if (mt == 0) return cudaSuccess;
  time_bucket_tile_kernel<<<dim3(static_cast<unsigned>(mt * mt), static_cast<unsigned>(B)), kBiasThreads, 0, st>>>(
      offsets, ts, n_buckets, mt, sq_offsets, out);
  return cudaGetLastError();
}

cudaError_t norm_gate_fwd(int64_t T, int D, int o_dt, int u_dt, int g_dt, const void* o, int64_t ld_o, const void* u,
                          int64_t ld_u, const float* gamma, const float* beta, float eps, void* g, float* mu,
                          float* rstd, cudaStream_t st, int* status) {
  if (T == 0) return cudaSuccess;
  // supported (o, u, g) combinations: exact fp32; fp32 O with fp16 U and fp16 G (tensor-core
  // layer); fp32 O with fp16 or bf16 U and bf16 G; all bf16; fp32 or bf16 O without a gate and fp16
  // G (the input LayerNorm of the norm_in layer variant).
#define HSTU_NG(VPT)                                                                                     \
  if (o_dt == kDtF32 && u_dt == kDtF32 && g_dt == kDtF32)                                               \
    return launch_ng<VPT, kDtF32, kDtF32, kDtF32>(T, o, ld_o, u, ld_u, gamma, beta, eps, g, mu, rstd, st, status); \
  if (o_dt == kDtF32 && u_dt == kDtF16 && g_dt == kDtF16)                                               \
    return launch_ng<VPT, kDtF32, kDtF16, kDtF16>(T, o, ld_o, u, ld_u, gamma, beta, eps, g, mu, rstd, st, status); \
  if (o_dt == kDtF32 && u_dt == kDtF16 && g_dt == kDtBF16)                                              \
    return launch_ng<VPT, kDtF32, kDtF16, kDtBF16>(T, o, ld_o, u, ld_u, gamma, beta, eps, g, mu, rstd, st, status); \
  if (o_dt == kDtF32 && u_dt == kDtBF16 && g_dt == kDtBF16)                                             \
    return launch_ng<VPT, kDtF32, kDtBF16, kDtBF16>(T, o, ld_o, u, ld_u, gamma, beta, eps, g, mu, rstd, st, status); \
  if (o_dt == kDtBF16 && u_dt == kDtBF16 && g_dt == kDtBF16)                                            \
    return launch_ng<VPT, kDtBF16, kDtBF16, kDtBF16>(T, o, ld_o, u, ld_u, gamma, beta, eps, g, mu, rstd, st, status); \
  if (o_dt == kDtF32 && u_dt == kDtOne && g_dt == kDtF16)                                               \
    return launch_ng<VPT, kDtF32, kDtOne, kDtF16>(T, o, ld_o, u, ld_u, gamma, beta, eps, g, mu, rstd, st, status);  \
  if (o_dt == kDtBF16 && u_dt == kDtOne && g_dt == kDtF16)                                              \
    return launch_ng<VPT, kDtBF16, kDtOne, kDtF16>(T, o, ld_o, u, ld_u, gamma, beta, eps, g, mu, rstd, st, status); \
  return cudaErrorInvalidValue
  switch (D) {
    case 64: HSTU_NG(2);
    case 128: HSTU_NG(4);
    case 256: HSTU_NG(8);
    case 512: HSTU_NG(16);
    case 1024: HSTU_NG(32);
    default: return cudaErrorInvalidValue;
  }
#undef HSTU_NG
}

cudaError_t convert_f32_to_bf16(const float* in, void* out, int64_t n, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const int64_t threads = (n + 3) / 4;
  f32_to_bf16_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(in, static_cast<uint16_t*>(out), n);
  return cudaGetLastError();
}

cudaError_t launch_timeout_probe(int* status, cudaStream_t st) {
  timeout_probe_kernel<<<1, 32, 0, st>>>(wait_ctl(status));
  return cudaGetLastError();
}

}  // namespace hstu
