// bias_tile.cuh - the relative half-bias of one causal (query tile, key tile) pair, computed by one
// block of 256 threads:
//   bias(i, j) = 0.5 (rab_pos[clamp(i - j)] + rab_time[bucket(t_i - t_j)])
// ("HSTU: The First Exploration of the Scaling Law", 7.1.4 Innovation 2: position and time bias;
// the buckets of time_bucket_dev.cuh). The bias does not depend on the head, so a pair's tile is
// computed once and read by every head.
//
// Thread t takes the column pairs 2 (t % 16) + 32 e, e < 4, of the rows t / 16 + 16 p, p < 8: 64
// elements, 4-byte half-bias (and 2-byte bucket) stores. TRANSPOSED: rows are keys and columns
// queries (the backward's [key][query] tiles); otherwise rows are queries. Timestamps past
// the sequence end are clamped to its last token (those elements are masked by the attention).
// When every difference of the tile fits in int32 (spans under 68 years of seconds) the bucket
// arithmetic is 32-bit; otherwise each difference is formed without overflow in 64 bits.
#pragma once

#include <stdint.h>

#include "hstu_internal.h"
#include "sm100_ptx.cuh"
#include "tile_pairs.cuh"
#include "time_bucket_dev.cuh"
#include "vec_io.cuh"

namespace hstu {
namespace {

constexpr int kBiasThreads = 256;

template <bool V>
struct BoolTag {
  static constexpr bool value = V;
};

__device__ __forceinline__ int bias_pos_index(long long r, int L) {
  r = r > L - 1 ? L - 1 : r;
  r = r < -(L - 1) ? -(L - 1) : r;
  return static_cast<int>(r) + L - 1;
}

// Timestamps of one (query tile, key tile) in shared memory, staged by all 256 threads of a block:
// ts[0, 128) the query rows q0.., ts[128, 256) the key rows k0.. of a sequence of n tokens starting at
// global row seq0 (rows past the end clamped to its last token; those elements are masked by the
// attention). `fast` says whether every difference of the tile fits in int32: the span hi - lo is
// formed in unsigned 64-bit arithmetic (no signed overflow for any int64 timestamps) and must stay
// below 2^31 - 1; then ts32 = ts - lo and every difference is a 32-bit subtraction. The same
// staging and the same two bucket functions (time_bucket32 on ts32 differences, time_bucket_pair64
// otherwise) serve the attention's bias tiles and the time-bucket test surface.
struct TileTimes {
  long long ts[256];
  int ts32[256];
  long long red[16];
  int fast;
};

// Phase 1: every thread loads its timestamp and the per-warp minimum / maximum.
__device__ __forceinline__ void tile_times_load(TileTimes& s, const int64_t* __restrict__ ts, long long seq0, int n,
                                                int q0, int k0) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int idx = (tid < 128 ? q0 : k0) + (tid & 127);
  const long long t = ts[seq0 + (idx < n ? idx : n - 1)];
  s.ts[tid] = t;
  long long mn = t, mx = t;
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) {
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, d));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, d));
  }
  if (lane == 0) {
    s.red[warp] = mn;
    s.red[8 + warp] = mx;
  }
}

// Phase 2, after a __syncthreads: the span test and the 32-bit copies; ends with a __syncthreads.
__device__ __forceinline__ bool tile_times_finish(TileTimes& s) {
  const int tid = threadIdx.x;
  long long lo = s.red[0], hi = s.red[8];
#pragma unroll
  for (int w = 1; w < 8; ++w) {
    lo = min(lo, s.red[w]);
    hi = max(hi, s.red[8 + w]);
  }
  const bool fast = static_cast<unsigned long long>(hi) - static_cast<unsigned long long>(lo) < 0x7fffffffULL;
  if (fast) s.ts32[tid] = static_cast<int>(static_cast<unsigned long long>(s.ts[tid]) - static_cast<unsigned long long>(lo));
  __syncthreads();
  return fast;
}

// bucket(t_row - t_col) of tile element (r, c) of a staged tile: rows are queries and columns keys,
// or (transposed) rows keys and columns queries.
template <bool TRANSPOSED>
__device__ __forceinline__ int tile_bucket(const TileTimes& s, bool fast, int r, int c, const long long* tau,
                                           const int* tau32, int nb) {
  const int qi = TRANSPOSED ? c : r, kj = TRANSPOSED ? r : c;
  return fast ? time_bucket32(s.ts32[qi] - s.ts32[128 + kj], tau32, nb)
              : time_bucket_pair64(s.ts[qi], s.ts[128 + kj], tau, nb);
}

// Token types of a staged tile, clamped into [0, nt) (a type outside it is reported): ty[0, 128) the
// query rows, ty[128, 256) the key rows, like TileTimes.
__device__ __forceinline__ void tile_types_load(int* ty, const int32_t* __restrict__ types, long long seq0, int n,
                                                int q0, int k0, int nt, int* status) {
  const int tid = threadIdx.x;
  const int idx = (tid < 128 ? q0 : k0) + (tid & 127);
  int t = types[seq0 + (idx < n ? idx : n - 1)];
  if (t < 0 || t >= nt) {
    if (idx < n) report_error(status, kDevBadInput);
    t = t < 0 ? 0 : nt - 1;
  }
  ty[tid] = t;
}

// The constant part of a block's bias work, staged once per block: the bucket thresholds and the
// head slice's halved rab_time (n_buckets <= 128) and rab_type (n_types <= 16) tables. These are
// inputs of the call, never written by the kernels before it, so a kernel may stage them before its
// programmatic-dependency wait.
struct BiasConst {
  long long tau[kTauEntries];
  int tau32[kTauEntries];
  float rt[128];
  float tt[16 * 16];
};

__device__ __forceinline__ void bias_const_load(BiasConst& c, const AttnArgs& a, int hb) {
  const int tid = threadIdx.x;
  for (int e = tid; e < kTauEntries; e += kBiasThreads) {
    c.tau[e] = g_time_taus[e];
    c.tau32[e] = g_time_taus32[e];
  }
  if (tid < a.n_buckets) c.rt[tid] = 0.5f * a.rab_time[static_cast<long long>(hb) * a.n_buckets + tid];
  const int nt = a.n_types;
  if (nt > 0 && tid < nt * nt) c.tt[tid] = 0.5f * a.rab_type[static_cast<long long>(hb) * nt * nt + tid];
}

// The batch's pair numbering, offsets and packing, read by every tile's decode: staged in shared
// memory for batches of up to kSeqStage sequences (one round of loads instead of a binary search of
// dependent global loads per tile), else the global arrays.
constexpr int kSeqStage = 512;
struct SeqTables {
  const long long* pair_base;
  const int64_t* offsets;
  const int32_t* pack;
};

__device__ __forceinline__ SeqTables stage_seq_tables(const AttnArgs& a, long long* s_pb, int64_t* s_off,
                                                      int32_t* s_pack) {
  if (a.B > kSeqStage) return SeqTables{a.pair_base, a.offsets, a.pack};
  for (int i = threadIdx.x; i <= a.B; i += kBiasThreads) {
    s_pb[i] = a.pair_base[i];
    s_off[i] = a.offsets[i];
    if (a.pack && i < a.B) s_pack[i] = a.pack[i];
  }
  return SeqTables{s_pb, s_off, a.pack ? s_pack : nullptr};
}

// The whole tile of causal pair `pair` for bias head slice hb, by one block of kBiasThreads threads
// (c staged and synchronised before). With per-head tables (bias_heads = H) every head has its own
// tile; with a type term each element also adds rab_type[type_query][type_key]. BUCKETS: also the u8
// bucket tile (head-independent, written by the hb = 0 blocks). False when `pair` is past the batch's
// last pair. A block that calls it again must synchronise first (the staging arrays are reused).
// Key-major staging of a query-major pass that also produces the backward's tiles: the fp16 tile
// with rows of 130 halfs and the buckets with rows of 132 bytes (odd word strides: the transposed
// stores of a half-warp fall in distinct banks).
constexpr int kTStride = 130, kBStride = 132;
constexpr int kBiasStageBytes = kQTile * kTStride * 2 + kQTile * kBStride;   // 50,176

template <bool TRANSPOSED, bool BUCKETS>
__device__ __forceinline__ bool bias_tile_block(const AttnArgs& a, const BiasConst& cst, const SeqTables& sq,
                                                long long pair, int hb, uint16_t* __restrict__ tile,
                                                uint8_t* __restrict__ btile, uint16_t* __restrict__ tile_t,
                                                uint8_t* __restrict__ btile_t, uint16_t* __restrict__ s_tt,
                                                uint8_t* __restrict__ s_tb) {
  __shared__ TileTimes s_t;
  __shared__ float s_win[256];
  __shared__ int s_ty[256];
  int b, qt, kt, n;
  long long seq0;
  if (!decode_tile_pair(pair, sq.pair_base, a.B, &b, &qt, &kt)) return false;
  if (!pair_rows(sq.offsets, sq.pack, b, &seq0, &n)) return true;   // a packed sequence's own pair: unused
  const int tid = threadIdx.x;
  const int L = a.pos_max_len, nt = a.n_types;
  const float* rab_pos = a.rab_pos + static_cast<long long>(hb) * (2 * L - 1);
  tile_times_load(s_t, a.ts, seq0, n, qt * kQTile, kt * kQTile);
  if (tid < 255) {
    const int pi = bias_pos_index(static_cast<long long>(qt - kt) * kQTile - 127 + tid, L);
    if (HSTU_DCHECK(pi >= 0 && pi < 2 * L - 1, a.status)) s_win[tid] = 0.5f * rab_pos[pi];
  }
  if (nt > 0) tile_types_load(s_ty, a.token_type, seq0, n, qt * kQTile, kt * kQTile, nt, a.status);
  __syncthreads();
  const bool fast = tile_times_finish(s_t);
  const int nb = a.n_buckets;
  // thread: column pairs c = 2 (tid % 16) + 32 e + x (e < 4, x < 2) of rows r = tid / 16 + 16 p
  // (p < 8). The 16 lanes of a half-warp read 32 consecutive diagonals of the rab_pos window (no bank
  // conflicts) and store 64 contiguous bytes of one row.
  const int cl = 2 * (tid & 15), rr = tid >> 4;
  // one pass over the tile: query-major (KEY_MAJOR false) or key-major; bout (nullable) receives the
  // buckets in the same layout
  // stage (nullable): also write each element, key-major, into s_tt / s_tb
  auto row_pass = [&](auto fast_tag, auto key_major_tag, uint16_t* __restrict__ out, uint8_t* __restrict__ bout,
                      bool stage) {
    constexpr bool kFast = decltype(fast_tag)::value;
    constexpr bool kTr = decltype(key_major_tag)::value;
    // staging index of a row / column token: queries at [0, 128), keys at [128, 256)
    constexpr int kRowBase = kTr ? 128 : 0, kColBase = kTr ? 0 : 128;
    int tcol[8];   // (fast path) the 32-bit times of this thread's 8 columns
    if (kFast) {
#pragma unroll
      for (int j = 0; j < 8; ++j) tcol[j] = s_t.ts32[kColBase + cl + 32 * (j >> 1) + (j & 1)];
    }
#pragma unroll 2
    for (int p = 0; p < 8; ++p) {
      const int r = rr + 16 * p;
      const int trow = kFast ? s_t.ts32[kRowBase + r] : 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v2[2];
        uint32_t bw = 0u;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int c = cl + 32 * e + x;
          // bucket(t_query - t_key)
          const int bkt = kFast ? time_bucket32(kTr ? tcol[2 * e + x] - trow : trow - tcol[2 * e + x], cst.tau32, nb)
                                : tile_bucket<kTr>(s_t, false, r, c, cst.tau, cst.tau32, nb);
          const int wi = kTr ? c - r + 127 : r - c + 127;
          float v = 0.0f;
          if (HSTU_DCHECK(bkt >= 0 && bkt < nb && wi >= 0 && wi < 255, a.status)) v = s_win[wi] + cst.rt[bkt];
          if (nt > 0) {
            const int ti = s_ty[kTr ? c : r] * nt + s_ty[128 + (kTr ? r : c)];
            if (HSTU_DCHECK(ti >= 0 && ti < nt * nt, a.status)) v += cst.tt[ti];
          }
          v2[x] = v;
          bw |= static_cast<uint32_t>(bkt) << (8 * x);
          if (stage) {
            s_tt[c * kTStride + r] = __half_as_ushort(__float2half_rn(v));
            s_tb[c * kBStride + r] = static_cast<uint8_t>(bkt);
          }
        }
        *reinterpret_cast<uint32_t*>(out + r * kQTile + cl + 32 * e) = pack_f16x2(v2[0], v2[1]);
        if (bout) *reinterpret_cast<uint16_t*>(bout + r * kQTile + cl + 32 * e) = static_cast<uint16_t>(bw);
      }
    }
  };
  // the backward's key-major tile and buckets as well (a forward that caches them for its backward):
  // staged transposed in shared memory by the same pass, then copied out row by row
  const bool stage = !TRANSPOSED && tile_t && s_tt && s_tb;
  if (fast) row_pass(BoolTag<true>{}, BoolTag<TRANSPOSED>{}, tile, BUCKETS && hb == 0 ? btile : nullptr, stage);
  else row_pass(BoolTag<false>{}, BoolTag<TRANSPOSED>{}, tile, BUCKETS && hb == 0 ? btile : nullptr, stage);
  if (stage) {
    __syncthreads();
    const uint32_t* st32 = reinterpret_cast<const uint32_t*>(s_tt);
    uint32_t* gt = reinterpret_cast<uint32_t*>(tile_t);
    for (int idx = tid; idx < kQTile * kQTile / 2; idx += kBiasThreads)
      gt[idx] = st32[(idx >> 6) * (kTStride / 2) + (idx & 63)];
    if (hb == 0 && btile_t) {
      const uint32_t* sb32 = reinterpret_cast<const uint32_t*>(s_tb);
      uint32_t* gb = reinterpret_cast<uint32_t*>(btile_t);
      for (int idx = tid; idx < kQTile * kQTile / 4; idx += kBiasThreads)
        gb[idx] = sb32[(idx >> 5) * (kBStride / 4) + (idx & 31)];
    }
  }
  return true;
}

// Grid-stride loop of a bias kernel: block (x, hb = blockIdx.y) stages its constants, waits for the
// kernels before it (the pair numbering and packing come from the work list) and stages the sequence
// tables, then computes the tiles of pairs x, x + gridDim.x, ... (tiles[pair * bias_heads + hb],
// btiles[pair]; with a.bias_t_out / a.bucket_t_out also the key-major tiles and buckets there).
template <bool TRANSPOSED, bool BUCKETS>
__device__ __forceinline__ void bias_tiles(const AttnArgs& a, uint16_t* __restrict__ tiles,
                                           uint8_t* __restrict__ btiles) {
  __shared__ BiasConst s_c;
  __shared__ long long s_pb[kSeqStage + 1];
  __shared__ int64_t s_off[kSeqStage + 1];
  __shared__ int32_t s_pack[kSeqStage];
  const int hb = blockIdx.y;
  const long long tile_blocks = a.bias_blocks > 0 ? a.bias_blocks : gridDim.x;
  if (static_cast<long long>(blockIdx.x) >= tile_blocks) {   // an extra block: bf16 -> fp16 conversion
    pdl_trigger();
    pdl_wait();      // cvt_out may still be read by an earlier kernel (a previous layer's f2)
    if (hb == 0) {
      const int64_t i = ((static_cast<int64_t>(blockIdx.x) - tile_blocks) * kBiasThreads + threadIdx.x) * 8;
      if (i + 8 <= a.cvt_n) {
        float v[8];
        load_vec<8, kDtBF16>(a.cvt_in, i, v);
        store_vec<8, kDtF16>(a.cvt_out, i, v);
      } else {
        for (int64_t k = i; k < a.cvt_n; ++k) {
          float f;
          load_vec<1, kDtBF16>(a.cvt_in, k, &f);
          reinterpret_cast<__half*>(a.cvt_out)[k] = __float2half_rn(f);
        }
      }
    }
    return;
  }
  pdl_trigger();
  bias_const_load(s_c, a, hb);
  pdl_wait();
  const SeqTables sq = stage_seq_tables(a, s_pb, s_off, s_pack);
  // the query-major kernel that also writes the backward's tiles is launched with kBiasStageBytes of
  // dynamic shared memory for their staging
  extern __shared__ __align__(16) uint8_t bias_stage_dyn[];
  uint16_t* stt = nullptr;
  uint8_t* stb = nullptr;
  if (!TRANSPOSED && a.bias_t_out) {
    stt = reinterpret_cast<uint16_t*>(bias_stage_dyn);
    stb = bias_stage_dyn + kQTile * kTStride * 2;
  }
  __syncthreads();
  for (long long p = blockIdx.x; p < a.max_pairs; p += tile_blocks) {
    uint16_t* tile = tiles + (p * a.bias_heads + hb) * (kQTile * kQTile);
    uint8_t* btile = BUCKETS ? btiles + p * (kQTile * kQTile) : nullptr;
    uint16_t* tile_t = a.bias_t_out ? static_cast<uint16_t*>(a.bias_t_out) + (p * a.bias_heads + hb) * (kQTile * kQTile)
                                    : nullptr;
    uint8_t* btile_t = a.bucket_t_out ? static_cast<uint8_t*>(a.bucket_t_out) + p * (kQTile * kQTile) : nullptr;
    if (!bias_tile_block<TRANSPOSED, BUCKETS>(a, s_c, sq, p, hb, tile, btile, tile_t, btile_t, stt, stb)) break;
    __syncthreads();
  }
}

}  // namespace
}  // namespace hstu
