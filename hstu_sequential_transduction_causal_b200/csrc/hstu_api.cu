// hstu_api.cu - the extern "C" entry points of libhstu.so: argument validation, workspace
// layout, tensor-map encoding and kernel dispatch on the caller's stream. No allocation, no
// synchronisation (except hstu_sync_status, whose job it is).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "../../include/hstu.h"
#include "hstu_internal.h"

namespace hstu {

namespace {

thread_local int32_t g_last_cuda_error = 0;
thread_local cudaEvent_t g_prof_events[kProfKernels][2] = {};
thread_local cudaEvent_t g_ready_events[2] = {};   // hstu_layer_bwd_ready_events: early, w1
// The layer backward's second stream, per host thread and device (created by the first call, which
// runs outside any capture): the table gradients run there while the dZ assembly and the dX / dW1
// GEMM run on the caller's stream, which joins it back before the call returns.
struct SideRes {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr, dz = nullptr;
};
thread_local SideRes g_side[64];
std::atomic<unsigned long long> g_wait_limit{1ull << 31};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up on first use (again after a failed lookup).
EncodeTiledFn get_encode_fn() {
  static std::atomic<EncodeTiledFn> cache{nullptr};
  EncodeTiledFn fn = cache.load(std::memory_order_acquire);
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFn>(p);
      cache.store(fn, std::memory_order_release);
    }
  }
  return fn;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hstu_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return HSTU_OK;
  g_last_cuda_error = static_cast<int32_t>(e);
  return e == cudaErrorInvalidValue ? HSTU_ERR_UNSUPPORTED : HSTU_ERR_CUDA;
}

int* ws_status(void* ws) { return static_cast<int*>(ws); }

// attention workspace: [0,256) status | [256,512) count | [512, ...) items (int32 x 2 x capacity)
int64_t capacity_of(const hstu_jagged_t* j) { return static_cast<int64_t>(j->B) + (j->T + kQTile - 1) / kQTile; }

// attention workspace: [0,256) status | [256,512) work-list counts (256: forward items, 260: backward
// items, 272: the persistent forward's unit counter) | items (int32 x 2 x capacity) |
// pair_base (int64 x (B+1)) | pack (int32 x B: short sequences sharing a tile) | fp16 bias tiles
// (32 KB per causal tile pair and bias slice, 1024-aligned)
struct AttnWs {
  size_t items, pairs, pack, urec, bias, items_end, total;
  int64_t max_pairs;
};

// hb: bias tiles per causal pair (1, or H for per-head bias tables)
AttnWs attn_ws_layout(const hstu_jagged_t* j, int hb = 1) {
  AttnWs w{};
  const int64_t cap = capacity_of(j);
  w.items = kWsHeader + 256;
  w.items_end = w.items + align_up(static_cast<size_t>(cap) * 8, 256);
  w.pairs = w.items_end;
  w.pack = w.pairs + align_up(static_cast<size_t>(j->B + 1) * 8, 256);
  w.urec = w.pack + align_up(static_cast<size_t>(j->B) * 4, 256);
  w.bias = align_up(w.urec + static_cast<size_t>(cap) * 32, 1024);
  w.max_pairs = attn_max_pairs(cap, j->max_len);
  w.total = w.bias + static_cast<size_t>(w.max_pairs) * hb * kQTile * kQTile * 2;
  return w;
}

size_t attn_ws_bytes(const hstu_jagged_t* j) { return attn_ws_layout(j).total; }

// The tile-pair kernels address their per-pair tiles by 32-bit TMA row coordinates: the forward's
// bias tiles span max_pairs * 128 rows, the backward's dX^T tiles max_pairs * H * 128. A batch
// beyond that (hundreds of GB of workspace) is refused on the host, before any size is computed
// in size_t or anything is enqueued.
constexpr int64_t kMaxTmaRows = 0x7fffffffLL;
bool fwd_pairs_fit(const hstu_jagged_t* j, int hb = 1) {
  return attn_ws_layout(j).max_pairs <= kMaxTmaRows / (static_cast<int64_t>(hb) * kQTile);
}
bool bwd_pairs_fit(const hstu_jagged_t* j, int H) {
  return H > 0 && attn_ws_layout(j).max_pairs <= kMaxTmaRows / (static_cast<int64_t>(H) * kQTile);
}

// hstu_layer_saved_t.attn_bias: the backward's key-major fp16 half-bias tiles (32 KB per causal
// pair), then the u8 bucket tiles (16 KB per pair), in the layout of the attention backward's own;
// then the batch's metadata the forward's work list writes for the backward: a 256-byte header
// (int32 key-tile item count at 0, the persistent backward's unit and finished-CTA counters at 4
// and 8), the key-tile work list, pair_base and the pack array.
struct BiasCache {
  size_t bucket, meta, kitems, pairs, pack, total;
};
BiasCache bias_cache_layout(const hstu_jagged_t* j) {
  const int64_t mp = attn_ws_layout(j).max_pairs;
  const int64_t cap = capacity_of(j);
  BiasCache c{};
  c.bucket = align_up(static_cast<size_t>(mp) * kQTile * kQTile * 2, 256);
  c.meta = c.bucket + align_up(static_cast<size_t>(mp) * kQTile * kQTile, 256);
  c.kitems = c.meta + 256;
  c.pairs = c.kitems + align_up(static_cast<size_t>(cap) * 8, 256);
  c.pack = c.pairs + align_up(static_cast<size_t>(j->B + 1) * 8, 256);
  c.total = c.pack + align_up(static_cast<size_t>(j->B) * 4, 256);
  return c;
}

// attention-backward workspace: the forward layout up to pair_base, then the key-tile work list,
// the transposed fp16 bias tiles (32 KB per pair), the u8 bucket tiles (16 KB per pair) and the fp16
// dX^T tiles of every (pair, head) (32 KB each) the table gradients are summed from.
struct AttnBwdWs {
  AttnWs f;
  size_t kitems, bias_t, bucket_t, dxt, total;
};

AttnBwdWs attn_bwd_ws_layout(const hstu_jagged_t* j, int H, int hb = 1) {
  AttnBwdWs w{};
  w.f = attn_ws_layout(j);
  const int64_t cap = capacity_of(j);
  const size_t tile = static_cast<size_t>(kQTile) * kQTile;
  w.kitems = w.f.bias;   // the forward bias region is not used by the backward
  w.bias_t = align_up(w.kitems + align_up(static_cast<size_t>(cap) * 8, 256), 1024);
  w.bucket_t = w.bias_t + static_cast<size_t>(w.f.max_pairs) * hb * tile * 2;
  w.dxt = align_up(w.bucket_t + static_cast<size_t>(w.f.max_pairs) * tile, 1024);
  w.total = w.dxt + static_cast<size_t>(w.f.max_pairs) * (H > 0 ? H : 0) * tile * 2;
  return w;
}

// layer-backward workspace: the attention-backward layout, then dG (fp32), dO (fp16), dq (fp32; the
// attention backward writes dZ_K and dZ_V itself), dZ (fp16 [T, 4D]), reduction partials,
// dgamma | dbeta, and the fp16 GEMM operands: copies of dy, x, W1 and W2 (both MMA operands share
// a type; G and dZ are fp16).
struct LayerBwdWs {
  size_t dg, dO, dq, dz, part_dy, part_ln, dy_f16, x_f16, w1_f16, w2_f16, total;
};

LayerBwdWs layer_bwd_layout(const hstu_layer_desc_t* d, const hstu_jagged_t* j) {
  LayerBwdWs w{};
  const size_t T = static_cast<size_t>(j->T), D = static_cast<size_t>(d->D);
  size_t off = align_up(attn_bwd_ws_layout(j, d->H).total, 1024);
  auto take = [&](size_t bytes) { const size_t o = off; off = align_up(off + bytes, 1024); return o; };
  w.dg = take(T * D * 4);
  w.dO = take(T * D * 2);
  w.dq = take(T * D * 4);
  w.dz = take(T * 4 * D * 2);
  // partial column sums: db2 (from the fp16 copy of dY), dgamma | dbeta (LayerNorm backward); db1 is
  // added up by atomics
  w.part_dy = take(static_cast<size_t>(kTailParts) * D * 4);
  w.part_ln = take(static_cast<size_t>(norm_gate_bwd_blocks(j->T)) * 2 * D * 4);
  w.dy_f16 = take(T * D * 2);
  w.x_f16 = take(T * D * 2);
  w.w1_f16 = take(4 * D * D * 2);
  w.w2_f16 = take(D * D * 2);
  w.total = off;
  return w;
}

// The layer backward's fused dK / dV epilogue: Z_K, Z_V read and dZ_K, dZ_V written (fp16, row
// stride ld) instead of fp32 dk / dv.
struct DzKV {
  const void* z_k;
  const void* z_v;
  void* dz_k;
  void* dz_v;
  int64_t ld;
};

// Attention backward on the caller's stream; dq / dk / dv fp32 with row stride ld_g. Zeroes the
// accumulated outputs (dq, the table gradients) first.
hstu_status_t run_attn_bwd(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag, const void* q, const void* k,
                           const void* v, const void* d_out, const float* rab_pos, const float* rab_time, float* dq,
                           float* dk, float* dv, int64_t ld_g, float* d_rab_pos, float* d_rab_time, void* ws,
                           cudaStream_t st, const hstu_rab_ext_t* ext = nullptr, float* d_rab_type = nullptr,
                           void* bias_cache = nullptr, bool zeroed = false, const DzKV* dzkv = nullptr,
                           const SideLaunch* side = nullptr) {
  // zeroed: an earlier launch of the call already cleared d_rab_pos, d_rab_time and dq (T > 0)
  const int hb = ext && ext->per_head ? desc->H : 1;
  const int nt = ext ? ext->n_types : 0;
  const AttnBwdWs lay = attn_bwd_ws_layout(jag, desc->H, hb);
  cudaError_t e = cudaSuccess;
  if (!zeroed || jag->T == 0) {
    e = cudaMemsetAsync(d_rab_pos, 0, sizeof(float) * hb * (2 * static_cast<size_t>(desc->pos_max_len) - 1), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(d_rab_time, 0, sizeof(float) * hb * desc->n_time_buckets, st);
    if (e == cudaSuccess && nt > 0) e = cudaMemsetAsync(d_rab_type, 0, sizeof(float) * hb * nt * nt, st);
    if (e != cudaSuccess) return cuda_status(e);
  }
  if (jag->T == 0) return HSTU_OK;
  if (!zeroed) e = cudaMemsetAsync(dq, 0, sizeof(float) * static_cast<size_t>(jag->T) * ld_g, st);
  if (e != cudaSuccess) return cuda_status(e);
  uint8_t* w = static_cast<uint8_t*>(ws);
  AttnBwdArgs A{};
  AttnArgs& a = A.f;
  int32_t* count = reinterpret_cast<int32_t*>(w + kWsHeader);
  int32_t* kcount = count + 1;
  int32_t* items = reinterpret_cast<int32_t*>(w + lay.f.items);
  a.B = jag->B; a.T = jag->T; a.max_len = jag->max_len; a.offsets = jag->offsets; a.ts = jag->timestamps;
  a.H = desc->H; a.dqk = desc->d_qk; a.dv = desc->d_v; a.inv_N = desc->inv_N; a.pos_max_len = desc->pos_max_len;
  a.n_buckets = desc->n_time_buckets;
  a.q = q; a.ld_q = desc->ld_q; a.k = k; a.ld_k = desc->ld_k; a.v = v; a.ld_v = desc->ld_v;
  a.in_f16 = desc->dtype == HSTU_F16;
  a.rab_pos = rab_pos; a.rab_time = rab_time; a.items = items; a.count = count; a.capacity = capacity_of(jag);
  a.status = ws_status(ws);
  a.pair_base = reinterpret_cast<const long long*>(w + lay.f.pairs);
  a.max_pairs = lay.f.max_pairs;
  A.dout = d_out; A.ld_do = desc->ld_o;
  A.dq = dq; A.dk = dk; A.dv = dv; A.ld_g = ld_g;
  A.drab_pos = d_rab_pos; A.drab_time = d_rab_time; A.drab_type = d_rab_type;
  a.bias_heads = hb; a.n_types = nt;
  if (nt > 0) { a.token_type = ext->token_type; a.rab_type = ext->rab_type; }
  A.bias_t = w + lay.bias_t; A.bucket_t = w + lay.bucket_t; A.dxt = w + lay.dxt;
  A.kitems = reinterpret_cast<int32_t*>(w + lay.kitems); A.kcount = kcount;
  A.sched = count + 5;   // [276, 284) of the workspace header region
  if (dzkv) {
    A.z_k = dzkv->z_k; A.z_v = dzkv->z_v; A.dz_k = dzkv->dz_k; A.dz_v = dzkv->dz_v; A.ld_z = dzkv->ld;
  }
  a.pack = reinterpret_cast<const int32_t*>(w + lay.f.pack);
  if (bias_cache && hb == 1) {   // tiles and work list written by this batch's forward (shared tables only)
    const BiasCache bc = bias_cache_layout(jag);
    uint8_t* c = static_cast<uint8_t*>(bias_cache);
    A.bias_t = bias_cache;
    A.bucket_t = c + bc.bucket;
    A.bias_cached = 1;
    A.kitems = reinterpret_cast<const int32_t*>(c + bc.kitems);
    A.kcount = reinterpret_cast<const int32_t*>(c + bc.meta);
    A.sched = reinterpret_cast<int32_t*>(c + bc.meta) + 1;
    a.pair_base = reinterpret_cast<const long long*>(c + bc.pairs);
    a.pack = reinterpret_cast<const int32_t*>(c + bc.pack);
  } else {
    e = launch_worklist(jag->offsets, jag->B, jag->T, jag->max_len, items, count, a.status, st,
                        reinterpret_cast<long long*>(w + lay.f.pairs), reinterpret_cast<int32_t*>(w + lay.kitems),
                        kcount, nullptr, reinterpret_cast<int32_t*>(w + lay.f.pack), nullptr, A.sched);
  }
  if (e == cudaSuccess) e = attn_bwd_tc(A, st, side);
  return cuda_status(e);
}

cudaError_t side_res(SideRes** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  SideRes& r = g_side[dev];
  if (!r.s) {
    e = cudaStreamCreateWithFlags(&r.s, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r.join, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r.dz, cudaEventDisableTiming);
    if (e != cudaSuccess) return e;
  }
  *out = &r;
  return cudaSuccess;
}

hstu_status_t check_jagged(const hstu_jagged_t* j) {
  if (!j || j->B < 0 || j->T < 0 || j->max_len < 0) return HSTU_ERR_INVALID_ARG;
  if (!j->offsets) return HSTU_ERR_INVALID_ARG;
  if (j->T > 0 && !j->timestamps) return HSTU_ERR_INVALID_ARG;
  if (j->T >= (1ll << 31)) return HSTU_ERR_UNSUPPORTED;   // row coordinates of the tensor maps are int32
  return HSTU_OK;
}

bool is_tc_dtype(int dt) { return dt == HSTU_BF16 || dt == HSTU_F16; }

hstu_status_t check_attn(const hstu_attn_desc_t* d, const hstu_jagged_t* j) {
  hstu_status_t s = check_jagged(j);
  if (s != HSTU_OK) return s;
  if (!d || d->H <= 0 || d->d_qk <= 0 || d->d_v <= 0 || d->pos_max_len <= 0) return HSTU_ERR_INVALID_ARG;
  if (d->n_time_buckets < 1 || d->n_time_buckets > 128) return HSTU_ERR_UNSUPPORTED;
  if (!isfinite(d->inv_N)) return HSTU_ERR_INVALID_ARG;
  if (d->o_dtype != HSTU_F32 && d->o_dtype != HSTU_BF16) return HSTU_ERR_UNSUPPORTED;
  if (is_tc_dtype(d->dtype)) {
    if (d->d_qk != 64 || d->d_v != 64) return HSTU_ERR_UNSUPPORTED;
    if (d->ld_q % 8 || d->ld_k % 8 || d->ld_v % 8 || d->ld_o % 8) return HSTU_ERR_UNSUPPORTED;
  } else if (d->dtype == HSTU_F32) {
    if (d->d_qk > 64 || d->d_v > 64 || d->o_dtype != HSTU_F32) return HSTU_ERR_UNSUPPORTED;
  } else {
    return HSTU_ERR_UNSUPPORTED;
  }
  if (d->ld_q < static_cast<int64_t>(d->H) * d->d_qk || d->ld_k < static_cast<int64_t>(d->H) * d->d_qk ||
      d->ld_v < static_cast<int64_t>(d->H) * d->d_v || d->ld_o < static_cast<int64_t>(d->H) * d->d_v)
    return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

// An attention forward's kernel arguments and the work list they read (host values only).
struct AttnFwdPlan {
  AttnArgs a;
  WorklistArgs wl;
  bool pairs, tc;
};

// tile_pairs: the workspace has the full attn_ws_layout (bias tiles); otherwise only the work list
// fits and the tensor-core path runs the kernel that evaluates the bias per element and head.
AttnFwdPlan plan_attn_fwd(const hstu_attn_desc_t* d, const hstu_jagged_t* j, const void* q, const void* k,
                          const void* v, const float* rab_pos, const float* rab_time, void* out, void* ws,
                          bool tile_pairs = true, const hstu_rab_ext_t* ext = nullptr, const int64_t* q_from = nullptr,
                          void* bias_cache = nullptr, const void* cvt_in = nullptr, void* cvt_out = nullptr,
                          int64_t cvt_n = 0) {
  const int64_t cap = capacity_of(j);
  const int hb = ext && ext->per_head ? d->H : 1;
  const AttnWs lay = attn_ws_layout(j, hb);
  uint8_t* w = static_cast<uint8_t*>(ws);
  int32_t* count = reinterpret_cast<int32_t*>(w + kWsHeader);
  int32_t* items = reinterpret_cast<int32_t*>(w + lay.items);
  AttnArgs a{};
  a.B = j->B; a.T = j->T; a.max_len = j->max_len; a.offsets = j->offsets; a.ts = j->timestamps;
  a.H = d->H; a.dqk = d->d_qk; a.dv = d->d_v; a.inv_N = d->inv_N; a.pos_max_len = d->pos_max_len;
  a.n_buckets = d->n_time_buckets;
  a.q = q; a.ld_q = d->ld_q; a.k = k; a.ld_k = d->ld_k; a.v = v; a.ld_v = d->ld_v;
  a.o = out; a.ld_o = d->ld_o; a.o_f32 = d->o_dtype == HSTU_F32;
  a.in_f16 = d->dtype == HSTU_F16;
  a.rab_pos = rab_pos; a.rab_time = rab_time; a.items = items; a.count = count; a.capacity = cap;
  a.status = ws_status(ws);
  a.bias_heads = hb;
  a.q_from = q_from;
  if (ext && ext->n_types > 0) {
    a.n_types = ext->n_types; a.token_type = ext->token_type; a.rab_type = ext->rab_type;
  }
  const bool pairs = tile_pairs && is_tc_dtype(d->dtype);
  int32_t* cache_kitems = nullptr;   // with the layer's bias cache: the backward's work list
  int32_t* cache_meta = nullptr;
  if (pairs) {
    a.pair_base = reinterpret_cast<const long long*>(w + lay.pairs);
    a.bias = w + lay.bias;
    a.max_pairs = lay.max_pairs;
    a.unit_counter = count + 4;   // [272, 276) of the workspace header region
    a.urec = reinterpret_cast<const int32_t*>(w + lay.urec);
    // short sequences share tiles, except in a prefix append (whose rows start mid-sequence)
    if (!q_from) a.pack = reinterpret_cast<const int32_t*>(w + lay.pack);
    if (bias_cache && hb == 1 && !q_from) {   // the backward's tiles and work list too
      const BiasCache bc = bias_cache_layout(j);
      uint8_t* c = static_cast<uint8_t*>(bias_cache);
      a.bias_t_out = bias_cache;
      a.bucket_t_out = c + bc.bucket;
      a.pair_base = reinterpret_cast<const long long*>(c + bc.pairs);
      a.pack = reinterpret_cast<const int32_t*>(c + bc.pack);
      cache_kitems = reinterpret_cast<int32_t*>(c + bc.kitems);
      cache_meta = reinterpret_cast<int32_t*>(c + bc.meta);
    }
    if (cvt_n > 0) {   // a bf16 -> fp16 copy rides on the bias kernel's launch
      a.cvt_in = cvt_in;
      a.cvt_out = cvt_out;
      a.cvt_n = cvt_n;
    }
  }
  AttnFwdPlan p{};
  p.a = a;
  p.pairs = pairs;
  p.tc = is_tc_dtype(d->dtype);
  p.wl = WorklistArgs{j->offsets, j->B, j->T, j->max_len, items, count, a.status,
                      pairs ? const_cast<long long*>(a.pair_base) : nullptr, cache_kitems, cache_meta,
                      pairs ? a.unit_counter : nullptr, const_cast<int32_t*>(a.pack), const_cast<int32_t*>(a.urec),
                      cache_meta ? cache_meta + 1 : nullptr};
  return p;
}

// wl_done: an earlier launch of the call already computed the plan's work list.
hstu_status_t launch_attn_fwd(const AttnFwdPlan& p, cudaStream_t st, bool wl_done = false) {
  const WorklistArgs& l = p.wl;
  cudaError_t e = cudaSuccess;
  if (!wl_done)
    e = launch_worklist(l.off, l.B, l.T, l.max_len, l.items, l.count, l.status, st, l.pair_base, l.kitems, l.kcount,
                        l.sched, l.pack, l.urec, l.sched2);
  if (e != cudaSuccess) return cuda_status(e);
  if (l.T == 0) return HSTU_OK;
  if (!p.tc) e = attn_fwd_f32_simt(p.a, st);
  else e = p.pairs ? attn_fwd_tc2(p.a, st) : attn_fwd_bf16_tc(p.a, st);
  return cuda_status(e);
}

hstu_status_t run_attn_fwd(const hstu_attn_desc_t* d, const hstu_jagged_t* j, const void* q, const void* k,
                           const void* v, const float* rab_pos, const float* rab_time, void* out, void* ws,
                           cudaStream_t st, bool tile_pairs = true, const hstu_rab_ext_t* ext = nullptr,
                           const int64_t* q_from = nullptr) {
  return launch_attn_fwd(plan_attn_fwd(d, j, q, k, v, rab_pos, rab_time, out, ws, tile_pairs, ext, q_from), st);
}

// f1: operands x, W1 of `dtype` (BF16 tensor cores or F32 CUDA cores); uvqk / z of act_dtype.
// f16_ops: x and W1 are fp16 copies (the fp32-residual path) instead of bf16.
hstu_status_t run_uvqk(int64_t T, int32_t D, hstu_dtype_t dtype, hstu_dtype_t act_dtype, const void* x, int64_t ld_x,
                       const void* W1, const float* b1, void* uvqk, void* z, int* status, cudaStream_t st,
                       bool f16_ops = false, const WorklistArgs* side = nullptr) {
  GemmArgs g{};
  g.A = x; g.lda = ld_x; g.a_mn = false;
  g.B = W1; g.ldb = D; g.b_mn = false; g.f16 = f16_ops;
  g.M = T; g.N = 4ll * D; g.K = D; g.splits = 1;
  g.epi.kind = kEpiSilu; g.epi.bias = b1;
  g.epi.out0 = uvqk; g.epi.out0_dt = act_dtype; g.epi.ld_out0 = 4ll * D;
  g.epi.out1 = z; g.epi.out1_dt = act_dtype; g.epi.ld_out1 = 4ll * D;
  g.status = status;
  return cuda_status(dtype == HSTU_BF16 ? gemm_bf16(g, st, side) : gemm_f32(g, st));
}

// g_dtype F16: W2 is read through an fp16 copy written to w2_f16 ([D, D]) first.
hstu_status_t run_out_proj(int64_t T, int32_t D, hstu_dtype_t dtype, hstu_dtype_t g_dtype, const void* g_in,
                           const void* W2, const float* b2, const void* x, hstu_dtype_t x_dtype, void* y,
                           hstu_dtype_t y_dtype, void* y_f16, int* status, cudaStream_t st, void* w2_f16,
                           bool w2_ready = false) {
  const bool f16 = g_dtype == HSTU_F16;
  if (f16 && !w2_ready) {
    cudaError_t e = convert_dtype(W2, kDtBF16, w2_f16, kDtF16, static_cast<int64_t>(D) * D, st);
    if (e != cudaSuccess) return cuda_status(e);
  }
  GemmArgs g{};
  g.A = g_in; g.lda = D; g.a_mn = false;
  g.B = f16 ? w2_f16 : W2; g.ldb = D; g.b_mn = false; g.f16 = f16;
  g.M = T; g.N = D; g.K = D; g.splits = 1;
  g.epi.kind = kEpiLinear; g.epi.bias = b2;
  g.epi.resid = x; g.epi.resid_dt = x_dtype; g.epi.ld_resid = D;
  g.epi.out0 = y; g.epi.out0_dt = y_dtype; g.epi.ld_out0 = D;
  g.epi.out1 = y_f16; g.epi.out1_dt = kDtF16; g.epi.ld_out1 = D;
  g.status = status;
  return cuda_status(dtype == HSTU_BF16 ? gemm_bf16(g, st) : gemm_f32(g, st));
}

// Split-K factor of an accumulating GEMM run alone: about two work units per SM (128 x 256 tiles),
// each of at least 4 k-blocks of 64.
int auto_splits(int64_t M, int64_t N, int64_t K) {
  const int64_t tiles = ((M + 127) / 128) * ((N + 255) / 256);
  const int64_t nkb = (K + 63) / 64;
  int64_t s = (296 + tiles - 1) / tiles;
  const int64_t s_max = (nkb + 3) / 4;
  if (s > s_max) s = s_max;
  return static_cast<int>(s < 1 ? 1 : s);
}

// Split-K factor that cuts K into work units of about `unit_kb` k-blocks of 64 (an accumulating
// GEMM sharing a launch with a product whose units are larger).
int splits_for_unit(int64_t K, int64_t unit_kb) {
  const int64_t nkb = (K + 63) / 64;
  if (unit_kb < 1) unit_kb = 1;
  const int64_t s = (nkb + unit_kb - 1) / unit_kb;
  return static_cast<int>(s < 1 ? 1 : s);
}

// The two scheduling counters of the grouped backward GEMMs: bytes [64, 72) of the workspace header.
int* gemm_sched(void* ws) { return static_cast<int*>(ws) + 16; }

hstu_status_t check_dense(int64_t T, int32_t D, hstu_dtype_t dtype) {
  if (T < 0 || D <= 0) return HSTU_ERR_INVALID_ARG;
  if (dtype != HSTU_BF16 && dtype != HSTU_F32) return HSTU_ERR_UNSUPPORTED;
  if (dtype == HSTU_BF16 && D % 64) return HSTU_ERR_UNSUPPORTED;
  if (T >= (1ll << 31)) return HSTU_ERR_UNSUPPORTED;
  return HSTU_OK;
}

}  // namespace

WaitCtl wait_ctl(int* status) { return WaitCtl{status, g_wait_limit.load(std::memory_order_relaxed)}; }

cudaError_t prof_record(int kernel, bool stop, cudaStream_t st) {
  if (kernel < 0 || kernel >= kProfKernels) return cudaSuccess;
  cudaEvent_t ev = g_prof_events[kernel][stop ? 1 : 0];
  if (!ev) return cudaSuccess;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(st, &cs);
  if (e != cudaSuccess) return e;
  return cs == cudaStreamCaptureStatusNone ? cudaEventRecord(ev, st) : cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
}

bool encode_tmap_2d_bf16(CUtensorMap* map, const void* base, int64_t inner, int64_t outer, int64_t ld_elems,
                         int box_inner, int box_outer, bool f16) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn || !aligned16(base) || inner <= 0 || outer <= 0 || (ld_elems * 2) % 16) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_elems) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_2d_out(CUtensorMap* map, const void* base, int dt, int64_t inner, int64_t outer, int64_t ld_elems,
                        int box_inner, int box_outer) {
  EncodeTiledFn fn = get_encode_fn();
  const int64_t es = dt == kDtF32 ? 4 : 2;
  if (!fn || !aligned16(base) || inner <= 0 || outer <= 0 || (ld_elems * es) % 16) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_elems * es)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType t = dt == kDtF32    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                : dt == kDtF16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                               : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = fn(map, t, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_2d_u8(CUtensorMap* map, const void* base, int64_t inner, int64_t outer, int64_t ld_bytes,
                       int box_inner, int box_outer) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn || !aligned16(base) || inner <= 0 || outer <= 0 || ld_bytes % 16) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t ensure_smem_attr(const void* kernel, int bytes) {
  static std::mutex mu;
  static const void* done[256];
  static int done_dev[256];
  static int n_done = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_done; ++i)
    if (done[i] == kernel && done_dev[i] == dev) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  // the whole unified L1 / shared array as shared memory, so that the blocks per SM the kernel was
  // sized for (two 96 KB blocks for the staged LayerNorm kernels) are resident together
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e == cudaSuccess && n_done < 256) {
    done[n_done] = kernel;
    done_dev[n_done] = dev;
    ++n_done;
  }
  return e;
}

}  // namespace hstu

using namespace hstu;

extern "C" {

int32_t hstu_abi_version(void) { return HSTU_ABI_VERSION; }

const char* hstu_status_string(hstu_status_t s) {
  switch (s) {
    case HSTU_OK: return "HSTU_OK";
    case HSTU_ERR_INVALID_ARG: return "HSTU_ERR_INVALID_ARG";
    case HSTU_ERR_UNSUPPORTED: return "HSTU_ERR_UNSUPPORTED";
    case HSTU_ERR_WORKSPACE: return "HSTU_ERR_WORKSPACE";
    case HSTU_ERR_CUDA: return "HSTU_ERR_CUDA";
    case HSTU_ERR_TIMEOUT: return "HSTU_ERR_TIMEOUT";
    case HSTU_ERR_DEVICE: return "HSTU_ERR_DEVICE";
  }
  return "HSTU_ERR_UNKNOWN";
}

int32_t hstu_last_cuda_error(void) { return g_last_cuda_error; }

void hstu_set_wait_limit(uint64_t cycles) {
  g_wait_limit.store(cycles ? cycles : (1ull << 31), std::memory_order_relaxed);
}

hstu_status_t hstu_sync_status(void* ws, hstu_stream_t stream, int32_t* device_status) {
  if (!ws || !device_status) return HSTU_ERR_INVALID_ARG;
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(int32_t), stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_status(e);
  *device_status = v;
  return HSTU_OK;
}

hstu_status_t hstu_profile_events(int32_t kernel, void* start, void* stop) {
  if (kernel < 0 || kernel >= kProfKernels || (start == nullptr) != (stop == nullptr)) return HSTU_ERR_INVALID_ARG;
  g_prof_events[kernel][0] = static_cast<cudaEvent_t>(start);
  g_prof_events[kernel][1] = static_cast<cudaEvent_t>(stop);
  return HSTU_OK;
}

hstu_status_t hstu_layer_bwd_ready_events(void* early, void* w1) {
  if ((early == nullptr) != (w1 == nullptr)) return HSTU_ERR_INVALID_ARG;
  g_ready_events[0] = static_cast<cudaEvent_t>(early);
  g_ready_events[1] = static_cast<cudaEvent_t>(w1);
  return HSTU_OK;
}

hstu_status_t hstu_debug_timeout_probe(void* ws, size_t ws_bytes, hstu_stream_t stream) {
  if (!ws) return HSTU_ERR_INVALID_ARG;
  if (ws_bytes < kWsHeader) return HSTU_ERR_WORKSPACE;
  return cuda_status(launch_timeout_probe(ws_status(ws), stream));
}

int64_t hstu_worklist_capacity(const hstu_jagged_t* jag) {
  if (check_jagged(jag) != HSTU_OK) return -1;
  return capacity_of(jag);
}

hstu_status_t hstu_jagged_worklist(const hstu_jagged_t* jag, int32_t* items, int32_t* count, hstu_stream_t stream) {
  hstu_status_t s = check_jagged(jag);
  if (s != HSTU_OK) return s;
  if (!items || !count) return HSTU_ERR_INVALID_ARG;
  return cuda_status(launch_worklist(jag->offsets, jag->B, jag->T, jag->max_len, items, count, nullptr, stream));
}

hstu_status_t hstu_time_buckets(const hstu_jagged_t* jag, int32_t n_buckets, const int64_t* sq_offsets, uint8_t* out,
                                hstu_stream_t stream) {
  hstu_status_t s = check_jagged(jag);
  if (s != HSTU_OK) return s;
  if (n_buckets < 1 || n_buckets > 128) return HSTU_ERR_UNSUPPORTED;
  if (jag->T > 0 && (!sq_offsets || !out)) return HSTU_ERR_INVALID_ARG;
  // one block per (query tile, key tile) of each sequence: grid (mt^2, B)
  const int64_t mt = (static_cast<int64_t>(jag->max_len) + kQTile - 1) / kQTile;
  if (jag->B > 65535 || mt * mt > 0x7fffffffLL) return HSTU_ERR_UNSUPPORTED;
  return cuda_status(launch_time_buckets(jag->offsets, jag->timestamps, jag->B, jag->T, jag->max_len, n_buckets,
                                         sq_offsets, out, stream));
}

hstu_status_t hstu_uvqk_fwd(int64_t T, int32_t D, hstu_dtype_t dtype, hstu_dtype_t act_dtype, const void* x,
                            int64_t ld_x, const void* W1, const float* b1, void* uvqk, void* z, void* ws,
                            size_t ws_bytes, hstu_stream_t stream) {
  hstu_status_t s = check_dense(T, D, dtype);
  if (s != HSTU_OK) return s;
  if (dtype == HSTU_F32 ? act_dtype != HSTU_F32 : !is_tc_dtype(act_dtype)) return HSTU_ERR_UNSUPPORTED;
  if (!ws) return HSTU_ERR_INVALID_ARG;
  if (ws_bytes < kWsHeader) return HSTU_ERR_WORKSPACE;
  if (T == 0) return HSTU_OK;
  if (!x || !W1 || !uvqk || ld_x < D) return HSTU_ERR_INVALID_ARG;
  if (dtype == HSTU_BF16 && (ld_x % 8 || !aligned16(x) || !aligned16(W1) || !aligned16(uvqk) || (z && !aligned16(z)) ||
                             (b1 && !aligned16(b1))))
    return HSTU_ERR_UNSUPPORTED;
  return run_uvqk(T, D, dtype, act_dtype, x, ld_x, W1, b1, uvqk, z, ws_status(ws), stream);
}

size_t hstu_attn_workspace_size(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag) {
  if (check_jagged(jag) != HSTU_OK || !fwd_pairs_fit(jag)) return 0;
  (void)desc;
  return attn_ws_bytes(jag);
}

hstu_status_t hstu_attn_fwd(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag, const void* q, const void* k,
                            const void* v, const float* rab_pos, const float* rab_time, void* out, void* ws,
                            size_t ws_bytes, hstu_stream_t stream) {
  hstu_status_t s = check_attn(desc, jag);
  if (s != HSTU_OK) return s;
  if (!fwd_pairs_fit(jag)) return HSTU_ERR_UNSUPPORTED;
  if (!ws) return HSTU_ERR_INVALID_ARG;
  if (ws_bytes < attn_ws_bytes(jag)) return HSTU_ERR_WORKSPACE;
  if (jag->T > 0 && (!q || !k || !v || !rab_pos || !rab_time || !out)) return HSTU_ERR_INVALID_ARG;
  if (is_tc_dtype(desc->dtype) && jag->T > 0 && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)))
    return HSTU_ERR_UNSUPPORTED;
  return run_attn_fwd(desc, jag, q, k, v, rab_pos, rab_time, out, ws, stream);
}

// ext: per_head 0 or 1, n_types 0..16 with its pointers when T > 0; tensor-core dtypes only
hstu_status_t check_rab_ext(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag, const hstu_rab_ext_t* ext) {
  if (!ext || (ext->per_head != 0 && ext->per_head != 1) || ext->n_types < 0) return HSTU_ERR_INVALID_ARG;
  if (ext->n_types > 16) return HSTU_ERR_UNSUPPORTED;
  if (ext->n_types > 0 && jag->T > 0 && (!ext->token_type || !ext->rab_type)) return HSTU_ERR_INVALID_ARG;
  if (!is_tc_dtype(desc->dtype)) return HSTU_ERR_UNSUPPORTED;
  return HSTU_OK;
}

size_t hstu_attn_ext_workspace_size(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag, const hstu_rab_ext_t* ext) {
  if (!desc || !ext || check_jagged(jag) != HSTU_OK || desc->H <= 0) return 0;
  const int hb = ext->per_head ? desc->H : 1;
  if (!fwd_pairs_fit(jag, hb)) return 0;
  return attn_ws_layout(jag, hb).total;
}

hstu_status_t hstu_attn_fwd_ext(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag, const hstu_rab_ext_t* ext,
                                const void* q, const void* k, const void* v, const float* rab_pos,
                                const float* rab_time, void* out, void* ws, size_t ws_bytes, hstu_stream_t stream) {
  hstu_status_t s = check_attn(desc, jag);
  if (s != HSTU_OK) return s;
  s = check_rab_ext(desc, jag, ext);
  if (s != HSTU_OK) return s;
  const int hb = ext->per_head ? desc->H : 1;
  if (!fwd_pairs_fit(jag, hb)) return HSTU_ERR_UNSUPPORTED;
  if (!ws) return HSTU_ERR_INVALID_ARG;
  if (ws_bytes < attn_ws_layout(jag, hb).total) return HSTU_ERR_WORKSPACE;
  if (jag->T > 0 && (!q || !k || !v || !rab_pos || !rab_time || !out)) return HSTU_ERR_INVALID_ARG;
  if (jag->T > 0 && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))) return HSTU_ERR_UNSUPPORTED;
  return run_attn_fwd(desc, jag, q, k, v, rab_pos, rab_time, out, ws, stream, true, ext);
}

size_t hstu_attn_bwd_ext_workspace_size(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag,
                                        const hstu_rab_ext_t* ext) {
  if (!desc || !ext || check_jagged(jag) != HSTU_OK || !bwd_pairs_fit(jag, desc->H)) return 0;
  return attn_bwd_ws_layout(jag, desc->H, ext->per_head ? desc->H : 1).total;
}

hstu_status_t hstu_attn_bwd_ext(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag, const hstu_rab_ext_t* ext,
                                const void* q, const void* k, const void* v, const void* d_out,
                                const float* rab_pos, const float* rab_time, float* dq, float* dk, float* dv,
                                float* d_rab_pos, float* d_rab_time, float* d_rab_type, void* ws,
                                size_t ws_bytes, hstu_stream_t stream) {
  hstu_status_t s = check_attn(desc, jag);
  if (s != HSTU_OK) return s;
  s = check_rab_ext(desc, jag, ext);
  if (s != HSTU_OK) return s;
  if (!bwd_pairs_fit(jag, desc->H)) return HSTU_ERR_UNSUPPORTED;
  if (!ws) return HSTU_ERR_INVALID_ARG;
  if (ws_bytes < attn_bwd_ws_layout(jag, desc->H, ext->per_head ? desc->H : 1).total) return HSTU_ERR_WORKSPACE;
  if (!d_rab_pos || !d_rab_time || (ext->n_types > 0 && !d_rab_type)) return HSTU_ERR_INVALID_ARG;
  if (jag->T > 0) {
    if (!q || !k || !v || !d_out || !rab_pos || !rab_time || !dq || !dk || !dv) return HSTU_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(d_out) || !aligned16(dq) || !aligned16(dk) ||
        !aligned16(dv))
      return HSTU_ERR_UNSUPPORTED;
  }
  const int64_t W = static_cast<int64_t>(desc->H) * desc->d_qk;
  return run_attn_bwd(desc, jag, q, k, v, d_out, rab_pos, rab_time, dq, dk, dv, W, d_rab_pos, d_rab_time, ws, stream,
                      ext, d_rab_type);
}

size_t hstu_attn_bwd_workspace_size(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag) {
  if (!desc || check_jagged(jag) != HSTU_OK || !bwd_pairs_fit(jag, desc->H)) return 0;
  return attn_bwd_ws_layout(jag, desc->H).total;
}

hstu_status_t hstu_attn_bwd(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag, const void* q, const void* k,
                            const void* v, const void* d_out, const float* rab_pos, const float* rab_time, float* dq,
                            float* dk, float* dv, float* d_rab_pos, float* d_rab_time, void* ws, size_t ws_bytes,
                            hstu_stream_t stream) {
  hstu_status_t s = check_attn(desc, jag);
  if (s != HSTU_OK) return s;
  if (!is_tc_dtype(desc->dtype)) return HSTU_ERR_UNSUPPORTED;
  if (!bwd_pairs_fit(jag, desc->H)) return HSTU_ERR_UNSUPPORTED;
  if (!ws) return HSTU_ERR_INVALID_ARG;
  if (ws_bytes < attn_bwd_ws_layout(jag, desc->H).total) return HSTU_ERR_WORKSPACE;
  if (!d_rab_pos || !d_rab_time) return HSTU_ERR_INVALID_ARG;
  if (jag->T > 0) {
    if (!q || !k || !v || !d_out || !rab_pos || !rab_time || !dq || !dk || !dv) return HSTU_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(d_out) || !aligned16(dq) || !aligned16(dk) ||
        !aligned16(dv))
      return HSTU_ERR_UNSUPPORTED;
  }
  const int64_t W = static_cast<int64_t>(desc->H) * desc->d_qk;
  return run_attn_bwd(desc, jag, q, k, v, d_out, rab_pos, rab_time, dq, dk, dv, W, d_rab_pos, d_rab_time, ws, stream);
}

hstu_status_t hstu_norm_gate_fwd(int64_t T, int32_t D, hstu_dtype_t o_dtype, hstu_dtype_t u_dtype,
                                 hstu_dtype_t g_dtype, const void* o, int64_t ld_o, const void* u, int64_t ld_u,
                                 const float* gamma, const float* beta, float eps, void* g, float* mu, float* rstd,
                                 hstu_stream_t stream) {
  if (T < 0) return HSTU_ERR_INVALID_ARG;
  const bool combo = (o_dtype == HSTU_F32 && u_dtype == HSTU_F32 && g_dtype == HSTU_F32) ||
                     (o_dtype == HSTU_F32 && is_tc_dtype(u_dtype) && g_dtype == HSTU_BF16) ||
                     (o_dtype == HSTU_F32 && u_dtype == HSTU_F16 && g_dtype == HSTU_F16) ||
                     (o_dtype == HSTU_BF16 && u_dtype == HSTU_BF16 && g_dtype == HSTU_BF16);
  if (!combo) return HSTU_ERR_UNSUPPORTED;
  if (D != 64 && D != 128 && D != 256 && D != 512 && D != 1024) return HSTU_ERR_UNSUPPORTED;
  if (T == 0) return HSTU_OK;
  if (!o || !u || !gamma || !beta || !g || ld_o < D || ld_u < D) return HSTU_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(u) || !aligned16(g) || !aligned16(gamma) || !aligned16(beta) || ld_o % 8 ||
      ld_u % 8)
    return HSTU_ERR_UNSUPPORTED;
  return cuda_status(norm_gate_fwd(T, D, o_dtype, u_dtype, g_dtype, o, ld_o, u, ld_u, gamma, beta, eps, g, mu, rstd,
                                   stream));
}

size_t hstu_out_proj_workspace_size(int32_t D, hstu_dtype_t g_dtype) {
  if (D <= 0) return 0;
  return kWsHeader + (g_dtype == HSTU_F16 ? align_up(static_cast<size_t>(D) * D * 2, 256) : 0);
}

hstu_status_t hstu_out_proj_fwd(int64_t T, int32_t D, hstu_dtype_t dtype, hstu_dtype_t g_dtype, const void* g,
                                const void* W2, const float* b2, const void* x, hstu_dtype_t x_dtype, void* y,
                                hstu_dtype_t y_dtype, void* y_f16, void* ws, size_t ws_bytes, hstu_stream_t stream) {
  hstu_status_t s = check_dense(T, D, dtype);
  if (s != HSTU_OK) return s;
  if (!ws) return HSTU_ERR_INVALID_ARG;
  const bool g_ok = dtype == HSTU_F32 ? g_dtype == HSTU_F32 : (g_dtype == HSTU_BF16 || g_dtype == HSTU_F16);
  if (!g_ok) return HSTU_ERR_UNSUPPORTED;
  if (ws_bytes < hstu_out_proj_workspace_size(D, g_dtype)) return HSTU_ERR_WORKSPACE;
  if ((x_dtype != HSTU_F32 && x_dtype != HSTU_BF16) || (y_dtype != HSTU_F32 && y_dtype != HSTU_BF16))
    return HSTU_ERR_UNSUPPORTED;
  if (dtype == HSTU_F32 && (x_dtype != HSTU_F32 || y_dtype != HSTU_F32 || y_f16)) return HSTU_ERR_UNSUPPORTED;
  if (T == 0) return HSTU_OK;
  if (!g || !W2 || !x || !y) return HSTU_ERR_INVALID_ARG;
  if (!aligned16(g) || !aligned16(W2) || !aligned16(x) || !aligned16(y) || (y_f16 && !aligned16(y_f16)) ||
      (dtype == HSTU_BF16 && b2 && !aligned16(b2)))
    return HSTU_ERR_UNSUPPORTED;
  return run_out_proj(T, D, dtype, g_dtype, g, W2, b2, x, x_dtype, y, y_dtype, y_f16, ws_status(ws), stream,
                      static_cast<uint8_t*>(ws) + kWsHeader);
}

// layer-forward workspace: the attention workspace, then (BF16 compute) the fp16 copy of W2 and,
// for an fp32 X, fp16 copies of X and W1 (the f1 operands).
struct LayerFwdWs {
  size_t w2_f16, x_f16, w1_f16, total;
};

LayerFwdWs layer_fwd_layout(const hstu_layer_desc_t* d, const hstu_jagged_t* j) {
  LayerFwdWs w{};
  const size_t T = static_cast<size_t>(j->T), D = static_cast<size_t>(d->D);
  size_t off = align_up(attn_ws_bytes(j), 1024);
  auto take = [&](size_t bytes) { const size_t o = off; off = align_up(off + bytes, 1024); return o; };
  if (d->dtype == HSTU_BF16) {
    w.w2_f16 = take(D * D * 2);
    if (d->x_dtype == HSTU_F32) {
      w.x_f16 = take(T * D * 2);
      w.w1_f16 = take(4 * D * D * 2);
    }
  }
  w.total = off;
  return w;
}

size_t hstu_layer_workspace_size(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag) {
  if (!desc || check_jagged(jag) != HSTU_OK || desc->D <= 0 || !fwd_pairs_fit(jag)) return 0;
  return layer_fwd_layout(desc, jag).total;
}

}  // extern "C"

namespace hstu {
namespace {

// The layer forward. resid_dtype: the dtype of x as the residual (desc->x_dtype, except for the
// norm_in variant, which passes an F32 descriptor so that f1 reads x_f16 = Xn, with a bf16 or fp32 X).
hstu_status_t run_layer_fwd(const hstu_layer_desc_t* desc, hstu_dtype_t resid_dtype, const hstu_jagged_t* jag,
                            const hstu_layer_weights_t* w, const void* x, const void* x_f16, void* y, void* y_f16,
                            const hstu_layer_saved_t* saved, void* ws, size_t ws_bytes, hstu_stream_t stream) {
  if (!desc || !w || !saved) return HSTU_ERR_INVALID_ARG;
  hstu_status_t s = check_jagged(jag);
  if (s != HSTU_OK) return s;
  const int32_t D = desc->D, H = desc->H;
  if (H <= 0 || D <= 0 || D % H) return HSTU_ERR_INVALID_ARG;
  s = check_dense(jag->T, D, desc->dtype);
  if (s != HSTU_OK) return s;
  hstu_attn_desc_t ad{};
  ad.H = H; ad.d_qk = D / H; ad.d_v = D / H; ad.inv_N = desc->inv_N; ad.pos_max_len = desc->pos_max_len;
  ad.n_time_buckets = desc->n_time_buckets; ad.dtype = desc->dtype; ad.o_dtype = HSTU_F32;
  ad.ld_q = ad.ld_k = ad.ld_v = 4ll * D; ad.ld_o = D;
  s = check_attn(&ad, jag);
  if (s != HSTU_OK) return s;
  if (!fwd_pairs_fit(jag)) return HSTU_ERR_UNSUPPORTED;
  if (desc->dtype == HSTU_F32 && (desc->x_dtype != HSTU_F32 || desc->y_dtype != HSTU_F32 || y_f16))
    return HSTU_ERR_UNSUPPORTED;
  if (!ws) return HSTU_ERR_INVALID_ARG;
  if (ws_bytes < hstu_layer_workspace_size(desc, jag)) return HSTU_ERR_WORKSPACE;
  const int64_t T = jag->T;
  if (T == 0) return HSTU_OK;
  if (!x || !y || !w->W1 || !w->b1 || !w->W2 || !w->b2 || !w->gamma || !w->beta || !w->rab_pos || !w->rab_time ||
      !saved->uvqk || !saved->o || !saved->g || !saved->mu || !saved->rstd)
    return HSTU_ERR_INVALID_ARG;
  if (!aligned16(w->gamma) || !aligned16(w->beta)) return HSTU_ERR_UNSUPPORTED;   // vector loads in both modes
  if (desc->dtype == HSTU_BF16) {   // 16-byte vector and TMA access
    const void* v16[] = {x, x_f16, y, y_f16, saved->uvqk, saved->z, saved->o, saved->g, w->W1, w->W2, w->b1, w->b2};
    for (const void* p : v16)
      if (p && !aligned16(p)) return HSTU_ERR_UNSUPPORTED;
    if (saved->attn_bias && reinterpret_cast<uintptr_t>(saved->attn_bias) % 256) return HSTU_ERR_UNSUPPORTED;
  }
  cudaStream_t st = stream;
  int* status = ws_status(ws);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  const LayerFwdWs lay = layer_fwd_layout(desc, jag);
  // f1 operands: bf16 X with bf16 W1 as given; an fp32 X (residual stream) through fp16 copies of
  // X and W1, 8x finer than bf16 at the same MMA rate
  const bool x32 = desc->dtype == HSTU_BF16 && desc->x_dtype == HSTU_F32;
  const void* x_op = x;
  const void* w1_op = w->W1;
  if (x32) {
    cudaError_t e = cudaSuccess;
    if (!x_f16) e = convert_dtype(x, kDtF32, wsb + lay.x_f16, kDtF16, T * D, st);
    if (e == cudaSuccess) e = convert_dtype(w->W1, kDtBF16, wsb + lay.w1_f16, kDtF16, 4ll * D * D, st);
    if (e != cudaSuccess) return cuda_status(e);
    x_op = x_f16 ? x_f16 : wsb + lay.x_f16;
    w1_op = wsb + lay.w1_f16;
  }
  // tensor-core mode keeps U|V|Q|K (and Z) in fp16: same MMA rate as bf16, 8x finer rounding of
  // the attention operands, whose errors LayerNorm(O) would otherwise amplify
  const hstu_dtype_t act = desc->dtype == HSTU_BF16 ? HSTU_F16 : HSTU_F32;
  ad.dtype = act;
  const size_t es = act == HSTU_F32 ? 4 : 2;
  const uint8_t* uvqk = static_cast<const uint8_t*>(saved->uvqk);
  // BF16 mode: the fp16 copy of W2 that f2 reads is written by extra blocks of the attention's bias
  // kernel (one launch fewer)
  const bool w2_early = desc->dtype == HSTU_BF16;
  const AttnFwdPlan plan = plan_attn_fwd(&ad, jag, uvqk + 2 * D * es, uvqk + 3 * D * es, uvqk + 1 * D * es, w->rab_pos,
                                         w->rab_time, saved->o, ws, true, nullptr, nullptr, saved->attn_bias, w->W2,
                                         wsb + lay.w2_f16, w2_early ? static_cast<int64_t>(D) * D : 0);
  // BF16 mode, up to 32 sequences: the attention's work list is computed inside the f1 launch
  const bool wl_in_f1 = desc->dtype == HSTU_BF16 && jag->B <= 32;
  s = run_uvqk(T, D, desc->dtype, act, x_op, D, w1_op, w->b1, saved->uvqk, saved->z, status, st, x32,
               wl_in_f1 ? &plan.wl : nullptr);
  if (s != HSTU_OK) return s;
  s = launch_attn_fwd(plan, st, wl_in_f1);
  if (s != HSTU_OK) return s;
  // G in fp16 (BF16 mode): f2 then reads an fp16 copy of W2
  const hstu_dtype_t g_dt = desc->dtype == HSTU_BF16 ? HSTU_F16 : HSTU_F32;
  cudaError_t e = norm_gate_fwd(T, D, kDtF32, act, g_dt, saved->o, D, uvqk, 4ll * D, w->gamma, w->beta,
                                desc->ln_eps, saved->g, saved->mu, saved->rstd, st, status);
  if (e != cudaSuccess) return cuda_status(e);
  return run_out_proj(T, D, desc->dtype, g_dt, saved->g, w->W2, w->b2, x, resid_dtype, y, desc->y_dtype, y_f16,
                      status, st, wsb + lay.w2_f16, w2_early);
}

}  // namespace
}  // namespace hstu

extern "C" {

hstu_status_t hstu_layer_fwd(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag, const hstu_layer_weights_t* w,
                             const void* x, const void* x_f16, void* y, void* y_f16, const hstu_layer_saved_t* saved,
                             void* ws, size_t ws_bytes, hstu_stream_t stream) {
  return run_layer_fwd(desc, desc ? desc->x_dtype : HSTU_F32, jag, w, x, x_f16, y, y_f16, saved, ws, ws_bytes, stream);
}

hstu_status_t hstu_linear_bf16(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda, int32_t a_mn,
                               const void* B, int64_t ldb, int32_t b_mn, const float* bias, const void* resid,
                               hstu_dtype_t resid_dtype, int64_t ld_resid, void* out, hstu_dtype_t out_dtype,
                               int64_t ld_out, int32_t accumulate, void* ws, size_t ws_bytes, hstu_stream_t stream) {
  if (M < 0 || N < 0 || K < 0 || !ws) return HSTU_ERR_INVALID_ARG;
  if (ws_bytes < kWsHeader) return HSTU_ERR_WORKSPACE;
  if (M == 0 || N == 0) return HSTU_OK;
  if (!A || !B || !out) return HSTU_ERR_INVALID_ARG;
  if (N % 32 || lda % 8 || ldb % 8 || !aligned16(A) || !aligned16(B) || !aligned16(out)) return HSTU_ERR_UNSUPPORTED;
  if (M >= (1ll << 31) || N >= (1ll << 31) || K >= (1ll << 31)) return HSTU_ERR_UNSUPPORTED;
  if (out_dtype != HSTU_F32 && out_dtype != HSTU_BF16 && out_dtype != HSTU_F16) return HSTU_ERR_UNSUPPORTED;
  if (accumulate && (out_dtype != HSTU_F32 || bias || resid)) return HSTU_ERR_UNSUPPORTED;
  if (lda < (a_mn ? M : K) || ldb < (b_mn ? N : K) || ld_out < N) return HSTU_ERR_INVALID_ARG;
  if (bias && !aligned16(bias)) return HSTU_ERR_UNSUPPORTED;   // 16-byte vector loads in the epilogue
  if (resid) {
    if (resid_dtype != HSTU_F32 && resid_dtype != HSTU_BF16 && resid_dtype != HSTU_F16) return HSTU_ERR_UNSUPPORTED;
    if (ld_resid < N) return HSTU_ERR_INVALID_ARG;
    // residual rows are read 32 elements at a time by 16-byte vector loads
    if (!aligned16(resid) || (ld_resid * (resid_dtype == HSTU_F32 ? 4 : 2)) % 16) return HSTU_ERR_UNSUPPORTED;
  }
  GemmArgs g{};
  g.A = A; g.lda = lda; g.a_mn = a_mn != 0;
  g.B = B; g.ldb = ldb; g.b_mn = b_mn != 0; g.f16 = false;
  g.M = M; g.N = N; g.K = K;
  g.splits = accumulate ? auto_splits(M, N, K) : 1;
  g.epi.kind = accumulate ? kEpiAtomic : kEpiLinear;
  g.epi.bias = bias;
  g.epi.resid = resid; g.epi.resid_dt = resid_dtype; g.epi.ld_resid = ld_resid;
  g.epi.out0 = out; g.epi.out0_dt = out_dtype; g.epi.ld_out0 = ld_out;
  g.status = ws_status(ws);
  return cuda_status(gemm_bf16(g, stream));
}

size_t hstu_layer_bwd_workspace_size(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag) {
  if (!desc || check_jagged(jag) != HSTU_OK || !bwd_pairs_fit(jag, desc->H)) return 0;
  return layer_bwd_layout(desc, jag).total;
}

size_t hstu_layer_bias_cache_size(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag) {
  if (!desc || check_jagged(jag) != HSTU_OK || !bwd_pairs_fit(jag, desc->H)) return 0;
  return bias_cache_layout(jag).total;
}

}  // extern "C"

namespace hstu {
namespace {

// The layer backward; with nin (the norm_in variant) dW1 reads the saved Xn and the last GEMM writes
// dXn = dZ W1 (fp32, no residual) after the layer workspace, from which the input LayerNorm's
// backward forms dX = dY + LN_in^T(dXn), dgamma_in and dbeta_in.
hstu_status_t run_layer_bwd(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag, const hstu_layer_weights_t* w,
                            const void* x, const void* x_f16, const hstu_layer_saved_t* saved, const void* dy,
                            const void* dy_f16, void* dx, void* dx_f16, const hstu_layer_grads_t* gr, void* ws,
                            size_t ws_bytes, hstu_stream_t stream, const hstu_norm_in_t* nin) {
  if (!desc || !w || !saved || !gr) return HSTU_ERR_INVALID_ARG;
  hstu_status_t s = check_jagged(jag);
  if (s != HSTU_OK) return s;
  const int32_t D = desc->D, H = desc->H;
  if (H <= 0 || D <= 0 || D % H) return HSTU_ERR_INVALID_ARG;
  if (desc->dtype != HSTU_BF16) return HSTU_ERR_UNSUPPORTED;
  if (D != 256 && D != 512) return HSTU_ERR_UNSUPPORTED;
  hstu_attn_desc_t ad{};
  ad.H = H; ad.d_qk = D / H; ad.d_v = D / H; ad.inv_N = desc->inv_N; ad.pos_max_len = desc->pos_max_len;
  ad.n_time_buckets = desc->n_time_buckets; ad.dtype = HSTU_F16; ad.o_dtype = HSTU_F32;
  ad.ld_q = ad.ld_k = ad.ld_v = 4ll * D; ad.ld_o = D;
  s = check_attn(&ad, jag);
  if (s != HSTU_OK) return s;
  if (!bwd_pairs_fit(jag, H)) return HSTU_ERR_UNSUPPORTED;
  if ((desc->x_dtype != HSTU_F32 && desc->x_dtype != HSTU_BF16) || (desc->y_dtype != HSTU_F32 && desc->y_dtype != HSTU_BF16))
    return HSTU_ERR_UNSUPPORTED;
  if (!ws) return HSTU_ERR_INVALID_ARG;
  const LayerBwdWs lay = layer_bwd_layout(desc, jag);
  const size_t nin_dxn = lay.total;
  const size_t nin_part = align_up(nin_dxn + static_cast<size_t>(jag->T) * D * 4, 1024);
  if (ws_bytes < (nin ? nin_part + ln_in_bwd_partial_floats(D) * 4 : lay.total)) return HSTU_ERR_WORKSPACE;
  if (!gr->dW1 || !gr->db1 || !gr->dW2 || !gr->db2 || !gr->dgamma || !gr->dbeta || !gr->drab_pos || !gr->drab_time)
    return HSTU_ERR_INVALID_ARG;
  const int64_t T = jag->T;
  cudaStream_t st = stream;
  cudaError_t e = cudaSuccess;
  if (T == 0) {
    const size_t zs[8] = {4ull * D * D * 4, 4ull * D * 4, 1ull * D * D * 4, 1ull * D * 4, 1ull * D * 4, 1ull * D * 4,
                          (2ull * desc->pos_max_len - 1) * 4, 1ull * desc->n_time_buckets * 4};
    float* ps[8] = {gr->dW1, gr->db1, gr->dW2, gr->db2, gr->dgamma, gr->dbeta, gr->drab_pos, gr->drab_time};
    for (int i = 0; i < 8 && e == cudaSuccess; ++i) e = cudaMemsetAsync(ps[i], 0, zs[i], st);
    if (nin && e == cudaSuccess) e = cudaMemsetAsync(nin->dgamma, 0, 4ull * D, st);
    if (nin && e == cudaSuccess) e = cudaMemsetAsync(nin->dbeta, 0, 4ull * D, st);
    return cuda_status(e);
  }
  if (!x || !dy || !dx || !saved->uvqk || !saved->z || !saved->o || !saved->g || !saved->mu || !saved->rstd)
    return HSTU_ERR_INVALID_ARG;
  // the weights the backward reads (b1 and b2 are not needed: Z and Y already hold them)
  if (!w->W1 || !w->W2 || !w->gamma || !w->beta || !w->rab_pos || !w->rab_time) return HSTU_ERR_INVALID_ARG;
  // 16-byte vector loads, stores and atomics (dW1 and dW2 are accumulated by float4 atomics)
  {
    const void* v16[] = {x, x_f16, dy, dy_f16, dx, dx_f16, saved->uvqk, saved->z, saved->o, saved->g,
                         w->W1, w->W2, w->gamma, w->beta, gr->dW1, gr->dW2};
    for (const void* p : v16)
      if (p && !aligned16(p)) return HSTU_ERR_UNSUPPORTED;
    if (saved->attn_bias && reinterpret_cast<uintptr_t>(saved->attn_bias) % 256) return HSTU_ERR_UNSUPPORTED;
  }
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  int* status = ws_status(ws);
  // fp16 operands: dy (of dG and dW2, next to fp16 G and W2), x (of dW1, next to fp16 dZ), W1, W2
  const int x_dt = desc->x_dtype == HSTU_F32 ? kDtF32 : kDtBF16;
  const int y_dt = desc->y_dtype == HSTU_F32 ? kDtF32 : kDtBF16;
  const void* dy_op = dy_f16 ? dy_f16 : wsb + lay.dy_f16;
  if (nin) x_f16 = nin->xn;   // f1 read Xn: dW1 = dZ^T Xn
  const void* x_op = x_f16 ? x_f16 : wsb + lay.x_f16;
  void* w1_f16 = wsb + lay.w1_f16;
  void* w2_f16 = wsb + lay.w2_f16;
  float* part_dy = reinterpret_cast<float*>(wsb + lay.part_dy);
  float* part_ln = reinterpret_cast<float*>(wsb + lay.part_ln);
  int parts_dy = 0, parts_ln = 0;
  float* dG = reinterpret_cast<float*>(wsb + lay.dg);
  void* dO = wsb + lay.dO;
  float* dq = reinterpret_cast<float*>(wsb + lay.dq);
  void* dz = wsb + lay.dz;
  {   // one launch: the fp16 copy of dY (unless the caller passed one) with the partial sums of db2,
      // the other fp16 GEMM operand copies, and zeros in every output a later launch accumulates
      // into (dW2, dW1, dQ and the table gradients)
    ConvertJob jobs[kMaxConvertJobs];
    int nj = 0;
    if (!x_f16) jobs[nj++] = ConvertJob{x, wsb + lay.x_f16, T * D, x_dt};
    jobs[nj++] = ConvertJob{w->W1, w1_f16, 4ll * D * D, kDtBF16};
    jobs[nj++] = ConvertJob{w->W2, w2_f16, 1ll * D * D, kDtBF16};
    jobs[nj++] = ConvertJob{nullptr, gr->dW2, 1ll * D * D, kDtF32};
    jobs[nj++] = ConvertJob{nullptr, gr->dW1, 4ll * D * D, kDtF32};
    jobs[nj++] = ConvertJob{nullptr, gr->db1, 4ll * D, kDtF32};
    jobs[nj++] = ConvertJob{nullptr, dq, T * D, kDtF32};
    jobs[nj++] = ConvertJob{nullptr, gr->drab_pos, 2ll * desc->pos_max_len - 1, kDtF32};
    jobs[nj++] = ConvertJob{nullptr, gr->drab_time, desc->n_time_buckets, kDtF32};
    e = rows_to_f16_colsum(T, D, y_dt, dy, dy_f16 ? nullptr : wsb + lay.dy_f16, part_dy, &parts_dy, jobs, nj, st);
  }
  if (e != cudaSuccess) return cuda_status(e);
  // 1. f2 backward: dG = dY W2 and dW2 = dY^T G in one launch (dW2 split over K = T into units of
  //    about half a dG unit, reduced into the zeroed dW2); db2 = sum_t dY
  {
    GemmArgs gg[2] = {};
    GemmArgs& g = gg[0];
    g.A = dy_op; g.lda = D; g.a_mn = false; g.B = w2_f16; g.ldb = D; g.b_mn = true; g.f16 = true;
    g.M = T; g.N = D; g.K = D; g.splits = 1;
    g.epi.kind = kEpiLinear; g.epi.out0 = dG; g.epi.out0_dt = kDtF32; g.epi.ld_out0 = D; g.status = status;
    GemmArgs& g2 = gg[1];
    g2.A = dy_op; g2.lda = D; g2.a_mn = true; g2.B = saved->g; g2.ldb = D; g2.b_mn = true; g2.f16 = true;
    g2.M = D; g2.N = D; g2.K = T; g2.splits = splits_for_unit(T, std::max<int64_t>(4, D / 128));
    g2.epi.kind = kEpiAtomic; g2.epi.out0 = gr->dW2; g2.epi.out0_dt = kDtF32; g2.epi.ld_out0 = D; g2.status = status;
    e = gemm_bf16_group(gg, 2, gemm_sched(ws), st);
  }
  // 2. norm-gate backward: dO (fp16), dZ_U (fp16), partial dgamma | dbeta (finished with db2 and db1
  // after the dZ assembly)
  if (e == cudaSuccess)
    e = norm_gate_bwd(T, D, kDtF16, dG, static_cast<const float*>(saved->o), saved->uvqk, saved->z, 4ll * D, w->gamma,
                      w->beta, saved->mu, saved->rstd, dO, dz, 4ll * D, part_ln, &parts_ln, st, status);
  if (e != cudaSuccess) return cuda_status(e);
  // 3. attention backward
  const uint8_t* uvqk = static_cast<const uint8_t*>(saved->uvqk);
  // (the attention backward writes dZ_V and dZ_K itself, from Z, instead of fp32 dV and dK)
  uint8_t* dzb = static_cast<uint8_t*>(dz);
  const uint8_t* zb = static_cast<const uint8_t*>(saved->z);
  const DzKV dzkv{zb + 3 * D * 2, zb + 1 * D * 2, dzb + 3 * D * 2, dzb + 1 * D * 2, 4ll * D};
  SideRes* sr = nullptr;
  e = side_res(&sr);
  if (e != cudaSuccess) return cuda_status(e);
  const SideLaunch sl{sr->s, sr->fork};
  s = run_attn_bwd(&ad, jag, uvqk + 2 * D * 2, uvqk + 3 * D * 2, uvqk + 1 * D * 2, dO, w->rab_pos, w->rab_time, dq,
                   nullptr, nullptr, D, gr->drab_pos, gr->drab_time, ws, st, nullptr, nullptr, saved->attn_bias, true,
                   &dzkv, &sl);
  if (s != HSTU_OK) return s;
  // 4. SiLU backward into dZ[:, D:4D], with db1 = sum_t dZ added up by atomics (zeroed by the first
  // launch); the first blocks of the same launch finish db2, dgamma and dbeta, all straight into the
  // caller's buffers
  int parts_dz = 0;
  {
    const ColsumJob fin[3] = {{part_dy, D, parts_dy, D, gr->db2},
                              {part_ln, 2ll * D, parts_ln, D, gr->dgamma},
                              {part_ln + D, 2ll * D, parts_ln, D, gr->dbeta}};
    e = dz_assemble(T, D, kDtF16, nullptr, dq, nullptr, saved->z, 4ll * D, dz, 4ll * D, nullptr, &parts_dz, st,
                    gr->db1, fin, 3);
  }
  // dW2, db2, dgamma, dbeta, db1 (the caller's stream) and the table gradients (the second stream)
  // are final: the early event is recorded on the second stream once it has also seen the former
  if (e == cudaSuccess && g_ready_events[0]) {
    e = cudaEventRecord(sr->dz, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sr->s, sr->dz, 0);
    if (e == cudaSuccess) e = cudaEventRecord(g_ready_events[0], sr->s);
  }
  // 5. f1 backward in one launch: dX = dY + dZ W1 and dW1 = dZ^T X (fp16 dZ, x and W1; dW1 split
  //    over K = T into units of about a third of a dX unit, reduced into the zeroed dW1)
  if (e == cudaSuccess) {
    GemmArgs gg[2] = {};
    GemmArgs& g3 = gg[1];
    g3.A = dz; g3.lda = 4ll * D; g3.a_mn = true; g3.B = x_op; g3.ldb = D; g3.b_mn = true; g3.f16 = true;
    g3.M = 4ll * D; g3.N = D; g3.K = T; g3.splits = splits_for_unit(T, std::max<int64_t>(4, D / 48));
    g3.epi.kind = kEpiAtomic; g3.epi.out0 = gr->dW1; g3.epi.out0_dt = kDtF32; g3.epi.ld_out0 = D; g3.status = status;
    GemmArgs& g4 = gg[0];
    g4.A = dz; g4.lda = 4ll * D; g4.a_mn = false; g4.B = w1_f16; g4.ldb = D; g4.b_mn = true; g4.f16 = true;
    g4.M = T; g4.N = D; g4.K = 4ll * D; g4.splits = 1;
    g4.epi.kind = kEpiLinear;
    if (nin) {   // dXn = dZ W1, then through the input LayerNorm
      g4.epi.out0 = wsb + nin_dxn; g4.epi.out0_dt = kDtF32; g4.epi.ld_out0 = D;
    } else {
      g4.epi.resid = dy; g4.epi.resid_dt = desc->y_dtype; g4.epi.ld_resid = D;
      g4.epi.out0 = dx; g4.epi.out0_dt = desc->x_dtype; g4.epi.ld_out0 = D;
      g4.epi.out1 = dx_f16; g4.epi.out1_dt = kDtF16; g4.epi.ld_out1 = D;
    }
    g4.status = status;
    e = gemm_bf16_group(gg, 2, gemm_sched(ws), st);
  }
  if (e == cudaSuccess && g_ready_events[1]) e = cudaEventRecord(g_ready_events[1], st);   // dW1 final
  if (nin && e == cudaSuccess)
    e = ln_in_bwd(T, D, desc->x_dtype == HSTU_F32 ? kDtF32 : kDtBF16, desc->y_dtype == HSTU_F32 ? kDtF32 : kDtBF16,
                  reinterpret_cast<const float*>(wsb + nin_dxn), x, dy, nin->gamma, nin->mu, nin->rstd, dx, dx_f16,
                  reinterpret_cast<float*>(wsb + nin_part), nin->dgamma, nin->dbeta, st);
  // join: the caller's stream waits for the table gradients
  cudaError_t ej = cudaEventRecord(sr->join, sr->s);
  if (ej == cudaSuccess) ej = cudaStreamWaitEvent(st, sr->join, 0);
  return cuda_status(e != cudaSuccess ? e : ej);
}

}  // namespace
}  // namespace hstu

extern "C" {

hstu_status_t hstu_layer_bwd(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag, const hstu_layer_weights_t* w,
                             const void* x, const void* x_f16, const hstu_layer_saved_t* saved, const void* dy,
                             const void* dy_f16, void* dx, void* dx_f16, const hstu_layer_grads_t* grads, void* ws,
                             size_t ws_bytes, hstu_stream_t stream) {
  return run_layer_bwd(desc, jag, w, x, x_f16, saved, dy, dy_f16, dx, dx_f16, grads, ws, ws_bytes, stream, nullptr);
}

size_t hstu_layer_norm_in_workspace_size(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag) {
  if (!desc || desc->D <= 0 || desc->H <= 0) return 0;
  hstu_layer_desc_t d32 = *desc;   // the forward's fp16 W1 copy region
  d32.x_dtype = HSTU_F32;
  const size_t f = hstu_layer_workspace_size(&d32, jag);
  const size_t b = hstu_layer_bwd_workspace_size(desc, jag);
  if (f == 0 || b == 0) return 0;
  const size_t nb = align_up(align_up(b, 1024) + static_cast<size_t>(jag->T) * desc->D * 4, 1024) +
                    ln_in_bwd_partial_floats(desc->D) * 4;
  return f > nb ? f : nb;
}

hstu_status_t hstu_layer_fwd_norm_in(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag,
                                     const hstu_layer_weights_t* w, const hstu_norm_in_t* nin, const void* x, void* y,
                                     void* y_f16, const hstu_layer_saved_t* saved, void* ws, size_t ws_bytes,
                                     hstu_stream_t stream) {
  if (!desc || !w || !saved || !nin) return HSTU_ERR_INVALID_ARG;
  hstu_status_t s = check_jagged(jag);
  if (s != HSTU_OK) return s;
  if (desc->dtype != HSTU_BF16) return HSTU_ERR_UNSUPPORTED;
  if (desc->D != 256 && desc->D != 512) return HSTU_ERR_UNSUPPORTED;
  if (desc->x_dtype != HSTU_F32 && desc->x_dtype != HSTU_BF16) return HSTU_ERR_UNSUPPORTED;
  if (!ws) return HSTU_ERR_INVALID_ARG;
  if (ws_bytes < hstu_layer_norm_in_workspace_size(desc, jag)) return HSTU_ERR_WORKSPACE;
  if (jag->T == 0) return HSTU_OK;
  if (!x || !nin->gamma || !nin->beta || !nin->xn || !nin->mu || !nin->rstd) return HSTU_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(nin->gamma) || !aligned16(nin->beta) || !aligned16(nin->xn))
    return HSTU_ERR_UNSUPPORTED;
  // Xn = LayerNorm_in(X) in fp16: f1 reads it (with an fp16 copy of W1), the residual adds X itself
  cudaError_t e = norm_gate_fwd(jag->T, desc->D, desc->x_dtype == HSTU_F32 ? kDtF32 : kDtBF16, kDtOne, kDtF16, x,
                                desc->D, nullptr, 0, nin->gamma, nin->beta, desc->ln_eps, nin->xn, nin->mu, nin->rstd,
                                stream);
  if (e != cudaSuccess) return cuda_status(e);
  hstu_layer_desc_t d32 = *desc;
  d32.x_dtype = HSTU_F32;
  return run_layer_fwd(&d32, desc->x_dtype, jag, w, x, nin->xn, y, y_f16, saved, ws, ws_bytes, stream);
}

hstu_status_t hstu_layer_bwd_norm_in(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag,
                                     const hstu_layer_weights_t* w, const hstu_norm_in_t* nin, const void* x,
                                     const hstu_layer_saved_t* saved, const void* dy, void* dx, void* dx_f16,
                                     const hstu_layer_grads_t* grads, void* ws, size_t ws_bytes,
                                     hstu_stream_t stream) {
  if (!nin || !desc) return HSTU_ERR_INVALID_ARG;
  if (jag && jag->T > 0 && (!nin->gamma || !nin->xn || !nin->mu || !nin->rstd)) return HSTU_ERR_INVALID_ARG;
  if (!nin->dgamma || !nin->dbeta) return HSTU_ERR_INVALID_ARG;
  if (nin->xn && !aligned16(nin->xn)) return HSTU_ERR_UNSUPPORTED;
  if (ws_bytes < hstu_layer_norm_in_workspace_size(desc, jag)) return HSTU_ERR_WORKSPACE;
  return run_layer_bwd(desc, jag, w, x, nullptr, saved, dy, nullptr, dx, dx_f16, grads, ws, ws_bytes, stream, nin);
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// Attention forward without a caller workspace.
//
// Some callers cannot hand the library any device memory of their own: a serving process that
// reserved its whole memory budget at start-up and forbids allocation on the request path, or a
// plain C host program that has no device allocator to carve a workspace from. For them the
// attention forward's scratch (status word, work-list count and the (sequence, tile) items) lives
// in a fixed array compiled into the library. Every GPU that loads the library holds this array
// until the process exits.
// ---------------------------------------------------------------------------------------------
namespace hstu {
namespace {

constexpr size_t kNoAllocScratchBytes = kWsHeader + 256 + 8ull * HSTU_NOALLOC_MAX_ITEMS;   // 524,800 bytes
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch per device. In host code the array's name is only a
// host-side stand-in, so the address must be asked for once per device, with that device current.
struct NoAllocSlot {
  bool ready;
  void* ptr;
};
NoAllocSlot g_noalloc_slots[64];
std::mutex g_noalloc_mutex;

hstu_status_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e);
  if (dev < 0 || dev >= 64) return HSTU_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_slots[dev].ready) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_status(e);
    g_noalloc_slots[dev].ptr = p;
    g_noalloc_slots[dev].ready = true;
  }
  *out = g_noalloc_slots[dev].ptr;
  return HSTU_OK;
}

}  // namespace
}  // namespace hstu

extern "C" hstu_status_t hstu_attn_fwd_noalloc(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag, const void* q,
                                               const void* k, const void* v, const float* rab_pos,
                                               const float* rab_time, void* out, hstu_stream_t stream) {
  hstu_status_t s = check_attn(desc, jag);
  if (s != HSTU_OK) return s;
  if (capacity_of(jag) > HSTU_NOALLOC_MAX_ITEMS) return HSTU_ERR_WORKSPACE;
  if (jag->T > 0 && (!q || !k || !v || !rab_pos || !rab_time || !out)) return HSTU_ERR_INVALID_ARG;
  if (is_tc_dtype(desc->dtype) && jag->T > 0 && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)))
    return HSTU_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != HSTU_OK) return s;
  // the status word must start at zero for this call (kernels record only the first error);
  // the work list is rewritten completely by every call
  cudaError_t e = cudaMemsetAsync(scratch, 0, kWsHeader, stream);
  if (e != cudaSuccess) return cuda_status(e);
  return run_attn_fwd(desc, jag, q, k, v, rab_pos, rab_time, out, scratch, stream, false);
}

extern "C" hstu_status_t hstu_attn_fwd_noalloc_status(hstu_stream_t stream, int32_t* device_status) {
  if (!device_status) return HSTU_ERR_INVALID_ARG;
  void* scratch = nullptr;
  hstu_status_t s = noalloc_scratch(&scratch);
  if (s != HSTU_OK) return s;
  return hstu_sync_status(scratch, stream, device_status);
}

// ---------------------------------------------------------------------------------------------
// M-FALCON ("HSTU: The First Exploration of the Scaling Law", 7.1.5 M-FALCON)
// ---------------------------------------------------------------------------------------------
namespace hstu {
namespace {

// Layer 0 reads the bf16 inputs; every later layer reads the fp32 residual stream.
hstu_layer_desc_t falcon_layer_desc(const hstu_falcon_desc_t* d, bool first) {
  hstu_layer_desc_t l{};
  l.D = d->D; l.H = d->H; l.inv_N = d->inv_N; l.pos_max_len = d->pos_max_len;
  l.n_time_buckets = d->n_time_buckets; l.ln_eps = d->ln_eps;
  l.dtype = HSTU_BF16; l.x_dtype = first ? HSTU_BF16 : HSTU_F32; l.y_dtype = HSTU_F32;
  return l;
}

// Workspace: the prefix layer's workspace first (its status word is the call's status word), then
// the prefix activations of one layer, the fp32 prefix stream (two buffers) and its fp16 copy, the
// per-layer key bias rows (+ the self bias), and one candidate micro-batch of
// R = users * min(b_m, m) rows: its bf16 input rows, fp32 stream (two buffers) and fp16 copy,
// U|V|Q|K, O, G, mu, rstd, and the fp16 copies of W1 and W2 of the candidate pass.
struct FalconWs {
  size_t p_uvqk, p_o, p_g, p_mu, p_rstd, p_x0, p_x1, p_x16, kbias, self_bias, c_in, c_x0, c_x1, c_x16, c_uvqk, c_o,
      c_g, c_mu, c_rstd, w1_f16, w2_f16, total;
  int64_t kbias_ld, R;
};

FalconWs falcon_layout(const hstu_falcon_desc_t* d, const hstu_jagged_t* p) {
  FalconWs w{};
  const hstu_layer_desc_t ld = falcon_layer_desc(d, false);   // the larger of the two layer workspaces
  const size_t Tp = static_cast<size_t>(p->T), D = static_cast<size_t>(d->D);
  w.kbias_ld = static_cast<int64_t>(align_up(static_cast<size_t>(p->max_len), kQTile));
  const int64_t per = d->b_m < d->m ? d->b_m : d->m;
  w.R = static_cast<int64_t>(d->users) * (per > 0 ? per : 0);
  const size_t R = static_cast<size_t>(w.R);
  size_t off = align_up(hstu_layer_workspace_size(&ld, p), 1024);
  auto take = [&](size_t bytes) { const size_t o = off; off = align_up(off + bytes, 1024); return o; };
  w.p_uvqk = take(Tp * 4 * D * 2);
  w.p_o = take(Tp * D * 4);
  w.p_g = take(Tp * D * 2);
  w.p_mu = take(Tp * 4);
  w.p_rstd = take(Tp * 4);
  w.p_x0 = take(Tp * D * 4);
  w.p_x1 = take(Tp * D * 4);
  w.p_x16 = take(Tp * D * 2);
  w.kbias = take(static_cast<size_t>(d->L) * d->users * w.kbias_ld * 2);
  w.self_bias = take(static_cast<size_t>(d->L) * 4);
  w.c_in = take(R * D * 2);
  w.c_x0 = take(R * D * 4);
  w.c_x1 = take(R * D * 4);
  w.c_x16 = take(R * D * 2);
  w.c_uvqk = take(R * 4 * D * 2);
  w.c_o = take(R * D * 4);
  w.c_g = take(R * D * 2);
  w.c_mu = take(R * 4);
  w.c_rstd = take(R * 4);
  w.w1_f16 = take(4 * D * D * 2);
  w.w2_f16 = take(D * D * 2);
  w.total = off;
  return w;
}

hstu_status_t check_falcon(const hstu_falcon_desc_t* d, const hstu_jagged_t* p) {
  if (!d) return HSTU_ERR_INVALID_ARG;
  hstu_status_t s = check_jagged(p);
  if (s != HSTU_OK) return s;
  if (d->L < 1 || d->users < 0 || d->m < 0 || d->b_m < 1 || d->users != p->B) return HSTU_ERR_INVALID_ARG;
  if (d->H <= 0 || d->D <= 0 || d->D % d->H) return HSTU_ERR_INVALID_ARG;
  if (d->D / d->H != 64 || d->D % 64) return HSTU_ERR_UNSUPPORTED;
  if (d->pos_max_len <= 0 || !isfinite(d->inv_N)) return HSTU_ERR_INVALID_ARG;
  if (d->n_time_buckets < 1 || d->n_time_buckets > 128) return HSTU_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(d->users) * d->m >= (1ll << 31)) return HSTU_ERR_UNSUPPORTED;
  if (!fwd_pairs_fit(p)) return HSTU_ERR_UNSUPPORTED;   // the prefix pass runs the causal layer
  return HSTU_OK;
}

}  // namespace
}  // namespace hstu

extern "C" size_t hstu_falcon_cache_size(const hstu_falcon_desc_t* desc, const hstu_jagged_t* prefix) {
  if (check_falcon(desc, prefix) != HSTU_OK) return 0;
  return static_cast<size_t>(desc->L) * static_cast<size_t>(prefix->T) * 2 * desc->D * 2;
}

extern "C" size_t hstu_falcon_workspace_size(const hstu_falcon_desc_t* desc, const hstu_jagged_t* prefix) {
  if (check_falcon(desc, prefix) != HSTU_OK) return 0;
  return falcon_layout(desc, prefix).total;
}

extern "C" hstu_status_t hstu_falcon_fwd(const hstu_falcon_desc_t* desc, const hstu_layer_weights_t* layers,
                                         const hstu_jagged_t* prefix, const void* prefix_x, void* kv_cache,
                                         int32_t cache_valid, void* prefix_out, const void* cand_x,
                                         const int64_t* request_ts, void* out, void* ws, size_t ws_bytes,
                                         hstu_stream_t stream) {
  hstu_status_t s = check_falcon(desc, prefix);
  if (s != HSTU_OK) return s;
  if (!layers || !ws) return HSTU_ERR_INVALID_ARG;
  const FalconWs lay = falcon_layout(desc, prefix);
  if (ws_bytes < lay.total) return HSTU_ERR_WORKSPACE;
  const int32_t D = desc->D, L = desc->L, users = desc->users, m = desc->m;
  const int64_t Tp = prefix->T;
  if (users == 0 || m == 0) return HSTU_OK;
  if (!cand_x || !request_ts || !out || (Tp > 0 && !kv_cache) || (!cache_valid && Tp > 0 && !prefix_x))
    return HSTU_ERR_INVALID_ARG;
  if (!aligned16(cand_x) || !aligned16(out) || (kv_cache && !aligned16(kv_cache)) ||
      (prefix_x && !aligned16(prefix_x)) || (prefix_out && !aligned16(prefix_out)))
    return HSTU_ERR_UNSUPPORTED;
  for (int l = 0; l < L; ++l) {
    const hstu_layer_weights_t& w = layers[l];
    if (!w.W1 || !w.b1 || !w.W2 || !w.b2 || !w.gamma || !w.beta || !w.rab_pos || !w.rab_time)
      return HSTU_ERR_INVALID_ARG;
    if (!aligned16(w.W1) || !aligned16(w.W2) || !aligned16(w.b1) || !aligned16(w.b2) || !aligned16(w.gamma) ||
        !aligned16(w.beta))
      return HSTU_ERR_UNSUPPORTED;
  }
  cudaStream_t st = stream;
  uint8_t* base = static_cast<uint8_t*>(ws);
  int* status = ws_status(ws);
  const hstu_layer_desc_t ldesc0 = falcon_layer_desc(desc, true), ldesc = falcon_layer_desc(desc, false);
  const size_t layer_ws = hstu_layer_workspace_size(&ldesc, prefix);
  const size_t kv_layer = static_cast<size_t>(Tp) * 2 * D;   // fp16 elements per layer of the cache
  uint16_t* cache = static_cast<uint16_t*>(kv_cache);
  void* x16 = nullptr;

  // 1. prefix: L causal layers on an fp32 residual stream; layer l's K and V go to the cache
  if (!cache_valid && Tp > 0) {
    hstu_layer_saved_t sv{};
    sv.uvqk = base + lay.p_uvqk; sv.z = nullptr; sv.o = base + lay.p_o; sv.g = base + lay.p_g;
    sv.mu = reinterpret_cast<float*>(base + lay.p_mu); sv.rstd = reinterpret_cast<float*>(base + lay.p_rstd);
    const void* xin = prefix_x;
    x16 = base + lay.p_x16;
    for (int l = 0; l < L; ++l) {
      void* y = (l == L - 1 && prefix_out) ? prefix_out : static_cast<void*>(base + ((l & 1) ? lay.p_x1 : lay.p_x0));
      // layer l reads the fp16 copy of its input that layer l - 1 wrote, and writes the next one
      s = hstu_layer_fwd(l == 0 ? &ldesc0 : &ldesc, prefix, &layers[l], xin, l == 0 ? nullptr : x16, y,
                         l + 1 < L ? x16 : nullptr, &sv, ws, layer_ws, st);
      if (s != HSTU_OK) return s;
      const uint16_t* uvqk = static_cast<const uint16_t*>(sv.uvqk);
      uint16_t* kv = cache + l * kv_layer;
      cudaError_t e = cudaMemcpy2DAsync(kv, 2 * D * 2, uvqk + 3 * D, 4 * D * 2, D * 2, Tp, cudaMemcpyDeviceToDevice, st);
      if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(kv + D, 2 * D * 2, uvqk + D, 4 * D * 2, D * 2, Tp, cudaMemcpyDeviceToDevice, st);
      if (e != cudaSuccess) return cuda_status(e);
      xin = y;
    }
  }

  // 2. per layer: the half-bias of every prefix key as seen from the request time
  uint16_t* kbias = reinterpret_cast<uint16_t*>(base + lay.kbias);
  float* self_bias = reinterpret_cast<float*>(base + lay.self_bias);
  for (int l = 0; l < L; ++l) {
    cudaError_t e = falcon_key_bias(prefix->offsets, prefix->timestamps, users, prefix->max_len, request_ts,
                                    layers[l].rab_pos, layers[l].rab_time, desc->pos_max_len, desc->n_time_buckets,
                                    kbias + static_cast<size_t>(l) * users * lay.kbias_ld, lay.kbias_ld,
                                    self_bias + l, status, st);
    if (e != cudaSuccess) return cuda_status(e);
  }

  // 3. candidates, b_m per user at a time, on an fp32 residual stream; every layer reads its cached
  //    prefix K, V
  const bool one_pass = desc->b_m >= m;
  void* c_x[2] = {base + lay.c_x0, base + lay.c_x1};
  void* c_x16 = base + lay.c_x16;
  void* c_uvqk = base + lay.c_uvqk;
  void* w1_f16 = base + lay.w1_f16;
  void* w2_f16 = base + lay.w2_f16;
  const uint16_t* cu = static_cast<const uint16_t*>(c_uvqk);
  for (int32_t c0 = 0; c0 < m; c0 += desc->b_m) {
    const int32_t rows = (m - c0) < desc->b_m ? (m - c0) : desc->b_m;
    const int64_t R = static_cast<int64_t>(users) * rows;
    const void* xin = cand_x;
    if (!one_pass) {   // gather rows [u m + c0, u m + c0 + rows) of every user
      cudaError_t e = cudaMemcpy2DAsync(base + lay.c_in, static_cast<size_t>(rows) * D * 2,
                                        static_cast<const uint16_t*>(cand_x) + static_cast<size_t>(c0) * D,
                                        static_cast<size_t>(m) * D * 2, static_cast<size_t>(rows) * D * 2, users,
                                        cudaMemcpyDeviceToDevice, st);
      if (e != cudaSuccess) return cuda_status(e);
      xin = base + lay.c_in;
    }
    for (int l = 0; l < L; ++l) {
      const hstu_layer_weights_t& w = layers[l];
      const bool last = l == L - 1;
      void* y = (one_pass && last) ? out : c_x[l & 1];
      if (l == 0) {
        s = run_uvqk(R, D, HSTU_BF16, HSTU_F16, xin, D, w.W1, w.b1, c_uvqk, nullptr, status, st);
      } else {
        cudaError_t e = convert_dtype(w.W1, kDtBF16, w1_f16, kDtF16, 4ll * D * D, st);
        if (e != cudaSuccess) return cuda_status(e);
        s = run_uvqk(R, D, HSTU_BF16, HSTU_F16, c_x16, D, w1_f16, w.b1, c_uvqk, nullptr, status, st, true);
      }
      if (s != HSTU_OK) return s;
      AttnArgs a{};
      a.bias_heads = 1;
      a.B = users; a.T = Tp; a.max_len = prefix->max_len; a.offsets = prefix->offsets; a.ts = prefix->timestamps;
      a.H = desc->H; a.dqk = 64; a.dv = 64; a.inv_N = desc->inv_N; a.pos_max_len = desc->pos_max_len;
      a.n_buckets = desc->n_time_buckets;
      a.q = cu + 2 * D; a.ld_q = 4 * D;
      a.k = cache + l * kv_layer; a.ld_k = 2 * D;
      a.v = cache + l * kv_layer + D; a.ld_v = 2 * D;
      a.o = base + lay.c_o; a.ld_o = D; a.o_f32 = 1; a.in_f16 = 1;
      a.rab_pos = w.rab_pos; a.rab_time = w.rab_time; a.status = status;
      a.cand_rows = rows; a.q_rows = R;
      a.kc = cu + 3 * D; a.vc = cu + D; a.ld_c = 4 * D;
      a.kbias = kbias + static_cast<size_t>(l) * users * lay.kbias_ld; a.kbias_ld = lay.kbias_ld;
      a.self_bias = self_bias + l;
      cudaError_t e = attn_falcon_tc(a, st);
      if (e == cudaSuccess)
        e = norm_gate_fwd(R, D, kDtF32, kDtF16, kDtF16, base + lay.c_o, D, c_uvqk, 4ll * D, w.gamma, w.beta,
                          desc->ln_eps, base + lay.c_g, reinterpret_cast<float*>(base + lay.c_mu),
                          reinterpret_cast<float*>(base + lay.c_rstd), st);
      if (e != cudaSuccess) return cuda_status(e);
      s = run_out_proj(R, D, HSTU_BF16, HSTU_F16, base + lay.c_g, w.W2, w.b2, xin, l == 0 ? HSTU_BF16 : HSTU_F32, y,
                       HSTU_F32, last ? nullptr : c_x16, status, st, w2_f16);
      if (s != HSTU_OK) return s;
      xin = y;
    }
    if (!one_pass) {   // scatter back
      cudaError_t e = cudaMemcpy2DAsync(static_cast<float*>(out) + static_cast<size_t>(c0) * D,
                                        static_cast<size_t>(m) * D * 4, xin, static_cast<size_t>(rows) * D * 4,
                                        static_cast<size_t>(rows) * D * 4, users, cudaMemcpyDeviceToDevice, st);
      if (e != cudaSuccess) return cuda_status(e);
    }
  }
  return HSTU_OK;
}

// ---------------------------------------------------------------------------------------------
// M-FALCON prefix append ("HSTU: The First Exploration of the Scaling Law", 7.1.5 M-FALCON: the
// history's K, V cache is reused across requests)
// ---------------------------------------------------------------------------------------------
namespace hstu {
namespace {

// Workspace: the attention workspace of the combined prefixes first (its status word is the call's),
// then the combined query buffer and attention output, and the appended rows' U|V|Q|K, O, G, mu,
// rstd, fp32 stream (two buffers) and its fp16 copy, and fp16 copies of W1, W2.
struct AppendWs {
  size_t qbuf, o_comb, a_uvqk, a_o, a_g, a_mu, a_rstd, a_x0, a_x1, a_x16, w1_f16, w2_f16, total;
};

AppendWs append_layout(const hstu_falcon_desc_t* d, const hstu_jagged_t* pnew, int64_t A) {
  AppendWs w{};
  const size_t Tn = static_cast<size_t>(pnew->T), D = static_cast<size_t>(d->D), a = static_cast<size_t>(A);
  size_t off = align_up(attn_ws_bytes(pnew), 1024);
  auto take = [&](size_t bytes) { const size_t o = off; off = align_up(off + bytes, 1024); return o; };
  w.qbuf = take(Tn * D * 2);
  w.o_comb = take(Tn * D * 4);
  w.a_uvqk = take(a * 4 * D * 2);
  w.a_o = take(a * D * 4);
  w.a_g = take(a * D * 2);
  w.a_mu = take(a * 4);
  w.a_rstd = take(a * 4);
  w.a_x0 = take(a * D * 4);
  w.a_x1 = take(a * D * 4);
  w.a_x16 = take(a * D * 2);
  w.w1_f16 = take(4 * D * D * 2);
  w.w2_f16 = take(D * D * 2);
  w.total = off;
  return w;
}

hstu_status_t check_append(const hstu_falcon_desc_t* d, const hstu_jagged_t* pold, const hstu_jagged_t* app,
                           const hstu_jagged_t* pnew) {
  hstu_status_t s = check_falcon(d, pnew);
  if (s != HSTU_OK) return s;
  if (check_jagged(pold) != HSTU_OK || !app || app->B < 0 || app->T < 0 || !app->offsets) return HSTU_ERR_INVALID_ARG;
  if (pold->B != d->users || app->B != d->users || pold->T + app->T != pnew->T) return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

}  // namespace
}  // namespace hstu

extern "C" size_t hstu_falcon_append_workspace_size(const hstu_falcon_desc_t* desc, const hstu_jagged_t* prefix_old,
                                                    const hstu_jagged_t* appended, const hstu_jagged_t* prefix_new) {
  if (check_append(desc, prefix_old, appended, prefix_new) != HSTU_OK) return 0;
  return append_layout(desc, prefix_new, appended->T).total;
}

extern "C" hstu_status_t hstu_falcon_append(const hstu_falcon_desc_t* desc, const hstu_layer_weights_t* layers,
                                            const hstu_jagged_t* prefix_old, const void* kv_cache_old,
                                            const hstu_jagged_t* appended, const void* app_x,
                                            const hstu_jagged_t* prefix_new, void* kv_cache_new, void* app_out,
                                            void* ws, size_t ws_bytes, hstu_stream_t stream) {
  hstu_status_t s = check_append(desc, prefix_old, appended, prefix_new);
  if (s != HSTU_OK) return s;
  if (!layers || !ws) return HSTU_ERR_INVALID_ARG;
  const int64_t A = appended->T, Tn = prefix_new->T, To = prefix_old->T;
  const AppendWs lay = append_layout(desc, prefix_new, A);
  if (ws_bytes < lay.total) return HSTU_ERR_WORKSPACE;
  if (Tn == 0) return HSTU_OK;
  if (!kv_cache_new || (To > 0 && !kv_cache_old) || (A > 0 && !app_x)) return HSTU_ERR_INVALID_ARG;
  if (!aligned16(kv_cache_new) || (kv_cache_old && !aligned16(kv_cache_old)) || (app_x && !aligned16(app_x)) ||
      (app_out && !aligned16(app_out)))
    return HSTU_ERR_UNSUPPORTED;
  const int32_t D = desc->D, L = desc->L, users = desc->users;
  for (int l = 0; l < L; ++l) {
    const hstu_layer_weights_t& w = layers[l];
    if (!w.W1 || !w.b1 || !w.W2 || !w.b2 || !w.gamma || !w.beta || !w.rab_pos || !w.rab_time)
      return HSTU_ERR_INVALID_ARG;
    if (!aligned16(w.W1) || !aligned16(w.W2) || !aligned16(w.b1) || !aligned16(w.b2) || !aligned16(w.gamma) ||
        !aligned16(w.beta))
      return HSTU_ERR_UNSUPPORTED;
  }
  cudaStream_t st = stream;
  uint8_t* base = static_cast<uint8_t*>(ws);
  int* status = ws_status(ws);
  const size_t old_layer = static_cast<size_t>(To) * 2 * D, new_layer = static_cast<size_t>(Tn) * 2 * D;
  const uint16_t* cache_old = static_cast<const uint16_t*>(kv_cache_old);
  uint16_t* cache_new = static_cast<uint16_t*>(kv_cache_new);
  uint16_t* a_uvqk = reinterpret_cast<uint16_t*>(base + lay.a_uvqk);
  void* a_x[2] = {base + lay.a_x0, base + lay.a_x1};
  void* a_x16 = base + lay.a_x16;
  hstu_attn_desc_t ad{};
  ad.H = desc->H; ad.d_qk = 64; ad.d_v = 64; ad.inv_N = desc->inv_N; ad.pos_max_len = desc->pos_max_len;
  ad.n_time_buckets = desc->n_time_buckets; ad.dtype = HSTU_F16; ad.o_dtype = HSTU_F32;
  ad.ld_q = D; ad.ld_k = 2ll * D; ad.ld_v = 2ll * D; ad.ld_o = D;
  const void* xin = app_x;
  for (int l = 0; l < L; ++l) {
    const hstu_layer_weights_t& w = layers[l];
    const bool last = l == L - 1;
    // 1. U|V|Q|K of the appended rows (layer 0 reads the bf16 input, later layers the fp16 copy of
    //    the fp32 stream)
    if (A > 0) {
      if (l == 0) {
        s = run_uvqk(A, D, HSTU_BF16, HSTU_F16, xin, D, w.W1, w.b1, a_uvqk, nullptr, status, st);
      } else {
        cudaError_t e = convert_dtype(w.W1, kDtBF16, base + lay.w1_f16, kDtF16, 4ll * D * D, st);
        if (e != cudaSuccess) return cuda_status(e);
        s = run_uvqk(A, D, HSTU_BF16, HSTU_F16, a_x16, D, base + lay.w1_f16, w.b1, a_uvqk, nullptr, status, st, true);
      }
      if (s != HSTU_OK) return s;
    }
    // 2. this layer's combined cache and the combined query buffer
    uint16_t* cl = cache_new + l * new_layer;
    cudaError_t e = falcon_append_scatter(prefix_old->offsets, appended->offsets, prefix_new->offsets, users, Tn, D,
                                          cache_old ? cache_old + l * old_layer : nullptr, a_uvqk, cl,
                                          reinterpret_cast<uint16_t*>(base + lay.qbuf), status, st);
    if (e != cudaSuccess) return cuda_status(e);
    if (A == 0) continue;
    // 3. causal attention of the appended rows over the combined prefix (rows of the old prefix are
    //    neither computed nor written)
    s = run_attn_fwd(&ad, prefix_new, base + lay.qbuf, cl, cl + D, w.rab_pos, w.rab_time, base + lay.o_comb, ws, st,
                     true, nullptr, prefix_old->offsets);
    if (s != HSTU_OK) return s;
    e = falcon_append_gather(prefix_old->offsets, appended->offsets, prefix_new->offsets, users, A, D,
                             reinterpret_cast<const float*>(base + lay.o_comb), reinterpret_cast<float*>(base + lay.a_o),
                             st);
    // 4. LayerNorm (.) U, f2 + residual
    if (e == cudaSuccess)
      e = norm_gate_fwd(A, D, kDtF32, kDtF16, kDtF16, base + lay.a_o, D, a_uvqk, 4ll * D, w.gamma, w.beta,
                        desc->ln_eps, base + lay.a_g, reinterpret_cast<float*>(base + lay.a_mu),
                        reinterpret_cast<float*>(base + lay.a_rstd), st);
    if (e != cudaSuccess) return cuda_status(e);
    void* y = (last && app_out) ? app_out : a_x[l & 1];
    s = run_out_proj(A, D, HSTU_BF16, HSTU_F16, base + lay.a_g, w.W2, w.b2, xin, l == 0 ? HSTU_BF16 : HSTU_F32, y,
                     HSTU_F32, last ? nullptr : a_x16, status, st, base + lay.w2_f16);
    if (s != HSTU_OK) return s;
    xin = y;
  }
  return HSTU_OK;
}

// ---------------------------------------------------------------------------------------------
// Stochastic Length
// ---------------------------------------------------------------------------------------------
extern "C" hstu_status_t hstu_stochastic_length_offsets(const hstu_jagged_t* raw, double alpha, int64_t* new_offsets,
                                                        void* ws, size_t ws_bytes, hstu_stream_t stream) {
  hstu_status_t s = check_jagged(raw);
  if (s != HSTU_OK) return s;
  if (!new_offsets || !ws || !(alpha >= 0.0) || !(alpha <= 2.0)) return HSTU_ERR_INVALID_ARG;
  if (ws_bytes < kWsHeader) return HSTU_ERR_WORKSPACE;
  return cuda_status(launch_sl_lengths(raw->offsets, raw->B, alpha, new_offsets, ws_status(ws), stream));
}

extern "C" hstu_status_t hstu_stochastic_length_select(const hstu_jagged_t* raw, const int64_t* keys,
                                                       const int64_t* new_offsets, const void* x, hstu_dtype_t x_dtype,
                                                       int32_t D, int64_t* kept, void* x_out, int64_t* ts_out,
                                                       void* ws, size_t ws_bytes, hstu_stream_t stream) {
  hstu_status_t s = check_jagged(raw);
  if (s != HSTU_OK) return s;
  if (!new_offsets || !kept || !ws || (raw->T > 0 && !keys)) return HSTU_ERR_INVALID_ARG;
  if (ws_bytes < kWsHeader) return HSTU_ERR_WORKSPACE;
  int64_t row_bytes = 0;
  if (x_out) {
    if (!x || D <= 0) return HSTU_ERR_INVALID_ARG;
    const int64_t es = x_dtype == HSTU_F32 ? 4 : (x_dtype == HSTU_BF16 || x_dtype == HSTU_F16) ? 2 : 0;
    if (es == 0) return HSTU_ERR_UNSUPPORTED;
    row_bytes = es * D;
    if (row_bytes % 16 || !aligned16(x) || !aligned16(x_out)) return HSTU_ERR_UNSUPPORTED;
  }
  if (raw->T == 0) return HSTU_OK;
  return cuda_status(launch_sl_select(raw->offsets, raw->B, raw->timestamps, keys, new_offsets, x, row_bytes, kept,
                                      x_out, ts_out, ws_status(ws), stream));
}
