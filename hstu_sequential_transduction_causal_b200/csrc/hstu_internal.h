// hstu_internal.h - declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sm100_ptx.cuh"

namespace hstu {

// Launches a kernel that begins with pdl_enter() with programmatic stream serialization: its CTAs
// may become resident while the previous kernel of the stream drains (they wait in pdl_enter until
// it has completed), which hides host launch latency between eagerly launched kernels. Under
// stream capture the attribute is left off: a replayed graph already launches back to back, and
// measured replays were slower with programmatic edges.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cfg.numAttrs = (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusNone) ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------------------------------------
// Timing hook (hstu_profile_events): caller-owned CUDA events recorded on the launching stream right
// before and right after the dominant kernel of a call; under stream capture they become external
// event-record nodes, so graph replays time the kernel too. Per host thread; no-op when unset.
// ---------------------------------------------------------------------------------------------
enum : int {
  kProfAttnFwd = 0, kProfAttnBwd = 1, kProfNormFwd = 2, kProfNormBwd = 3, kProfBias = 4, kProfTableGrad = 5, kProfDz = 6,
  kProfKernels = 7
};
cudaError_t prof_record(int kernel, bool stop, cudaStream_t st);

// ---------------------------------------------------------------------------------------------
// workspace layout: [0, 256) status word + padding, then per-call regions
// ---------------------------------------------------------------------------------------------
constexpr size_t kWsHeader = 256;
constexpr int kQTile = 128;       // rows of a query / key tile

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

WaitCtl wait_ctl(int* status);

// ---------------------------------------------------------------------------------------------
// GEMM
// ---------------------------------------------------------------------------------------------
enum : int { kEpiSilu = 0, kEpiLinear = 1, kEpiAtomic = 2 };

struct GemmEpilogue {
  int kind;
  const float* bias;      // [N] or null
  const void* resid;      // [M, N] or null (LINEAR)
  int resid_dt;
  int64_t ld_resid;
  void* out0;             // SILU: SiLU(Z); LINEAR: Y; ATOMIC: fp32 accumulation target
  int out0_dt;
  int64_t ld_out0;
  void* out1;             // SILU: Z; LINEAR: second copy of Y; or null
  int out1_dt;
  int64_t ld_out1;
};

struct GemmArgs {
  const void* A;   // K-major: [M, K] (lda); MN-major: [K, M] (lda)
  int64_t lda;
  bool a_mn;
  const void* B;   // K-major: [N, K] (ldb); MN-major: [K, N] (ldb)
  int64_t ldb;
  bool b_mn;
  bool f16;        // A and B are fp16 (else bf16)
  int64_t M, N, K;
  int splits;      // split-K factor (ATOMIC epilogue only)
  GemmEpilogue epi;
  int* status;     // device status word
};

// 2D tensor map of a 2-byte element matrix (bf16, or fp16 when f16), 128-byte swizzle.
bool encode_tmap_2d_bf16(CUtensorMap* map, const void* base, int64_t inner, int64_t outer,
                         int64_t ld_elems, int box_inner, int box_outer, bool f16 = false);
// 2D tensor map of an output matrix of element code dt (fp32, bf16, fp16), 128-byte swizzle, for
// TMA stores and reduce-adds (box_inner * element size == 128).
bool encode_tmap_2d_out(CUtensorMap* map, const void* base, int dt, int64_t inner, int64_t outer, int64_t ld_elems,
                        int box_inner, int box_outer);
// 2D tensor map of a u8 matrix, 128-byte swizzle (box_inner * 1 byte <= 128).
bool encode_tmap_2d_u8(CUtensorMap* map, const void* base, int64_t inner, int64_t outer, int64_t ld_bytes,
                       int box_inner, int box_outer);

// Sets a kernel's dynamic shared-memory limit once per (kernel, device).
cudaError_t ensure_smem_attr(const void* kernel, int bytes);
// Multiprocessors of the current device (cached per device; 148 when the query fails).
int sm_count();

// A batch's work list for at most 32 sequences, as launch_worklist writes it (its arguments, below).
struct WorklistArgs {
  const int64_t* off;
  int B;
  int64_t T;
  int max_len;
  int32_t* items;
  int32_t* count;
  int* status;
  long long* pair_base;
  int32_t* kitems;
  int32_t* kcount;
  int32_t* sched;
  int32_t* pack;
  int32_t* urec;
  int32_t* sched2;
};

// side (optional, B <= 32): the work list is computed in the same launch by a warp that the GEMM
// leaves idle (one launch fewer before the kernels that read it).
cudaError_t gemm_bf16(const GemmArgs& g, cudaStream_t st, const WorklistArgs* side = nullptr);
// Two independent products in one launch (n = 1 or 2; empty products are skipped). With `sched`
// (two ints, zero before the first launch; each launch leaves them zero) the CTAs take work units
// from a global counter in order, so the caller lists the product with the larger units first;
// without it every CTA runs a fixed stride of units (and may carry a work list as `side`).
cudaError_t gemm_bf16_group(const GemmArgs* g, int n, int* sched, cudaStream_t st, const WorklistArgs* side = nullptr);
cudaError_t gemm_f32(const GemmArgs& g, cudaStream_t st);

// ---------------------------------------------------------------------------------------------
// jagged metadata / time buckets
// ---------------------------------------------------------------------------------------------
// Builds the (sequence, query tile) work list; with pair_base (device, [B+1]) also the index of
// each sequence's first causal (query tile, key tile) pair and, in pair_base[B], their total.
// With kitems, also the attention backward's (sequence, key tile) list in the same cost order: the
// key tile that visits t + 1 query tiles sits where the forward list has query tile t. With sched,
// sched[0] (the persistent attention kernel's unit counter) is reset to 0; with sched2, sched2[0]
// and sched2[1] (the persistent backward's unit and finished-CTA counters). With pack (int32 [B]),
// runs of short sequences share a tile: pack[b] = k >= 2 marks the first of k packed sequences
// (one item (b, -k) in both lists), 0 the other members, 1 a sequence on its own. With urec (needs
// pair_base; int32 [capacity, 8], 16-byte aligned), the persistent attention forward's record of
// each item: {b, tile, first row, rows, first causal pair of the query tile, 0, 0, 0}.
cudaError_t launch_worklist(const int64_t* offsets, int B, int64_t T, int max_len, int32_t* items,
                            int32_t* count, int* status, cudaStream_t st, long long* pair_base = nullptr,
                            int32_t* kitems = nullptr, int32_t* kcount = nullptr, int32_t* sched = nullptr,
                            int32_t* pack = nullptr, int32_t* urec = nullptr, int32_t* sched2 = nullptr);
// The n_b x n_b time-bucket matrices of the test surface, tile by tile with the bias tiles' code.
cudaError_t launch_time_buckets(const int64_t* offsets, const int64_t* ts, int B, int64_t T, int max_len,
                                int n_buckets, const int64_t* sq_offsets, uint8_t* out, cudaStream_t st);

// ---------------------------------------------------------------------------------------------
// attention
// ---------------------------------------------------------------------------------------------
struct AttnArgs {
  int B;
  int64_t T;
  int max_len;
  const int64_t* offsets;
  const int64_t* ts;
  int H, dqk, dv;
  float inv_N;
  int pos_max_len;
  int n_buckets;
  const void* q; int64_t ld_q;
  const void* k; int64_t ld_k;
  const void* v; int64_t ld_v;
  void* o; int64_t ld_o; int o_f32;
  int in_f16;              // q, k, v are fp16 (else bf16) on the tensor-core path
  const float* rab_pos;
  const float* rab_time;
  const int32_t* items;    // work list (b, tile)
  const int32_t* count;
  int64_t capacity;
  int* status;
  const long long* pair_base;   // [B+1] first causal tile pair of each sequence (tile-pair kernel)
  void* bias;                   // fp16 [max_pairs, 128, 128] bias tiles (tile-pair kernel)
  int64_t max_pairs;
  // M-FALCON candidate attention (attn_falcon_tc): B users, offsets / ts / k / v describe the
  // prefixes (T prefix rows); q holds q_rows = B * cand_rows candidate rows, user-major.
  int cand_rows;                // candidate rows per user
  int64_t q_rows;
  const void* kc;               // candidates' own K and V (same dtype as q), row stride ld_c
  const void* vc;
  int64_t ld_c;
  const uint16_t* kbias;        // fp16 half-bias per prefix key: [B, kbias_ld], user u at u * kbias_ld
  int64_t kbias_ld;             // multiple of 128 >= every prefix length
  const float* self_bias;       // device: rab_pos[idx(0)] + rab_time[bucket(0)]
  int32_t* unit_counter;        // persistent forward: next (work item, head) unit, reset by the work list
  const int32_t* urec;          // persistent forward: per-item unit records (launch_worklist's urec)
  // the richer bias (hstu_rab_ext_t): bias_heads tiles per causal pair (1: tables shared by the heads,
  // H: one slice per head, rab_pos / rab_time / rab_type indexed by head first); n_types > 0 adds
  // rab_type[type_i][type_j]
  int bias_heads;
  int n_types;
  const int32_t* token_type;
  const float* rab_type;
  // prefix append: only query rows at or past q_from[b + 1] - q_from[b] of sequence b (the old
  // prefix length, from the old prefix offsets) are computed and written; null = every row
  const int64_t* q_from;
  // packed short sequences (launch_worklist's pack array) or null: an item (b, -k) is one tile over
  // the rows of sequences b .. b + k - 1, keys masked to the query row's own sequence
  const int32_t* pack;
  // (forward, nullable) the bias kernel also writes the backward's key-major tiles and buckets here,
  // laid out as AttnBwdArgs::bias_t and ::bucket_t
  void* bias_t_out;
  void* bucket_t_out;
  // (forward, cvt_n > 0) extra blocks of the bias kernel convert cvt_n bf16 values cvt_in to fp16 at
  // cvt_out (the layer's fp16 W2 copy, read later by f2); bias_blocks: the grid's tile blocks
  const void* cvt_in;
  void* cvt_out;
  int64_t cvt_n;
  int64_t bias_blocks;
};

struct AttnBwdArgs {
  AttnArgs f;                  // forward arguments (q, k, v, tables, work list with pair_base)
  const void* dout; int64_t ld_do;   // upstream gradient of O, same dtype as q
  float* dq; float* dk; float* dv;   // fp32 [T, H*64], dq accumulated (must be zero on entry)
  int64_t ld_g;                      // row stride of dq, dk, dv
  float* drab_pos; float* drab_time; // accumulated (must be zero on entry)
  float* drab_type;                  // [bias_heads, n_types, n_types], accumulated; null without types
  void* bias_t;                // fp16 [max_pairs, bias_heads, 128 keys, 128 queries] half-bias, transposed
  void* bucket_t;              // u8   [max_pairs, 128 keys, 128 queries] time bucket, transposed
  void* dxt;                   // fp16 [max_pairs, H, 128 keys, 128 queries] dX^T of every (pair, head)
  const int32_t* kitems;       // backward work list (b, key tile)
  const int32_t* kcount;
  int32_t* sched;              // the persistent backward's unit counter and finished-CTA counter (two
                               // ints): zero at launch (the work list zeroes them), zero again at exit
  int bias_cached;             // bias_t and bucket_t were written by the forward: no bias kernel
  // Layer backward (optional): instead of dk / dv, the kernel writes dZ_K = dK (.) SiLU'(Z_K) and
  // dZ_V = dV (.) SiLU'(Z_V) in fp16 (row stride ld_z, head h at column h d), Z read as fp16 with the
  // same stride; dk and dv are then not written.
  const void* z_k;
  const void* z_v;
  void* dz_k;
  void* dz_v;
  int64_t ld_z;
};

// side (optional): the table gradients go to that stream instead, after it waits for the kernel
// before them (fork: a reusable event recorded on st); the caller joins it back later.
struct SideLaunch {
  cudaStream_t stream;
  cudaEvent_t fork;
};
cudaError_t attn_bwd_tc(const AttnBwdArgs& a, cudaStream_t st, const SideLaunch* side = nullptr);

// Bound on the number of causal (query tile, key tile) pairs of a batch.
int64_t attn_max_pairs(int64_t capacity, int max_len);
// Pairs the table-gradient grid covers at once; it loops over the rest.
int64_t bias_grid_pairs(int64_t max_pairs, int bias_heads);
// Blocks (one tile each) of a bias-tile grid per head slice: four per SM; they loop over the rest.
int64_t bias_tile_grid(int64_t max_pairs, int bias_heads);

cudaError_t attn_fwd_bf16_tc(const AttnArgs& a, cudaStream_t st);     // work list only
cudaError_t attn_fwd_tc2(const AttnArgs& a, cudaStream_t st);         // bias tiles + work list
cudaError_t attn_fwd_f32_simt(const AttnArgs& a, cudaStream_t st);
// M-FALCON: the per-key half-bias of every prefix token (one launch per layer), then the candidate
// attention; tc dtypes only, d = 64, O fp32.
cudaError_t falcon_key_bias(const int64_t* offsets, const int64_t* ts, int users, int max_len,
                            const int64_t* request_ts, const float* rab_pos, const float* rab_time,
                            int pos_max_len, int n_buckets, uint16_t* kbias, int64_t kbias_ld, float* self_bias,
                            int* status, cudaStream_t st);
cudaError_t attn_falcon_tc(const AttnArgs& a, cudaStream_t st);
// M-FALCON prefix append (falcon_append.cu): one layer of the combined K|V cache and the combined
// query buffer; the appended rows' attention output back in their own order.
cudaError_t falcon_append_scatter(const int64_t* old_off, const int64_t* app_off, const int64_t* new_off, int users,
                                  int64_t T_new, int D, const uint16_t* old_cache, const uint16_t* uvqk,
                                  uint16_t* new_cache, uint16_t* qbuf, int* status, cudaStream_t st);
cudaError_t falcon_append_gather(const int64_t* old_off, const int64_t* app_off, const int64_t* new_off, int users,
                                 int64_t A, int D, const float* o_comb, float* o_app, cudaStream_t st);

// ---------------------------------------------------------------------------------------------
// LayerNorm (.) U
// ---------------------------------------------------------------------------------------------
// o_dt: f32 or bf16; u_dt: any; g_dt: any (kDt* codes). g has row stride D.
// status (device, optional): where a bounded wait of the staged kernel records a timeout.
cudaError_t norm_gate_fwd(int64_t T, int D, int o_dt, int u_dt, int g_dt, const void* o, int64_t ld_o,
                          const void* u, int64_t ld_u, const float* gamma, const float* beta,
                          float eps, void* g, float* mu, float* rstd, cudaStream_t st, int* status = nullptr);

cudaError_t convert_f32_to_bf16(const float* in, void* out, int64_t n, cudaStream_t st);

// ---------------------------------------------------------------------------------------------
// layer backward helpers (layer_bwd.cu)
// ---------------------------------------------------------------------------------------------
int norm_gate_bwd_blocks(int64_t T);
// dO = LayerNorm backward of dLn = dG (.) U; dZ_U = dG (.) Ln (.) SiLU'(Z_U) (fp16, stride ld_dz);
// the partial sums of dgamma | dbeta into partial [*parts, 2D] (*parts <= norm_gate_bwd_blocks(T));
// the caller finishes them (dz_assemble's finish jobs).
cudaError_t norm_gate_bwd(int64_t T, int D, int act_dt, const float* dg, const float* o, const void* u,
                          const void* zu, int64_t ld_act, const float* gamma, const float* beta, const float* mu,
                          const float* rstd, void* d_o, void* dz, int64_t ld_dz, float* partial, int* parts,
                          cudaStream_t st, int* status = nullptr);
// A column-sum finish: the sum of a partial buffer's rows.
struct ColsumJob {
  const float* partial;   // parts rows of `ld` floats; the job reads columns [0, cols)
  int64_t ld;
  int parts;
  int cols;
  float* out;             // [cols]
};
struct ColsumJobs {
  ColsumJob job[4];
  int first_block[5];
  int njobs;
};
// dZ[:, D:4D] = [dV | dQ | dK] (.) SiLU'(Z[:, D:4D]) in fp16 (dZ[:, 0:D] already written; with dv
// and dk null, dZ_V and dZ_K too, which the attention backward then wrote) and the column sums of
// all of dZ in blocks of 32 rows: into partial [*parts = ceil(T / 32), 4D] (may be
// null) and / or added by fp32 atomics into db1 = sum_t dZ (may be null; zero before the launch).
// D a multiple of 64. With fin (up to four column sums whose partials earlier launches wrote), the
// first blocks of the same launch finish those sums.
cudaError_t dz_assemble(int64_t T, int D, int act_dt, const float* dv, const float* dq, const float* dk,
                        const void* z, int64_t ld_z, void* dz, int64_t ld_dz, float* partial, int* parts,
                        cudaStream_t st, float* db1 = nullptr, const ColsumJob* fin = nullptr, int nfin = 0);
// A tensor of n elements (fp32, bf16 or fp16) converted to fp16; with in == null, n fp32 zeros
// written to out instead (an accumulated output cleared in the same launch).
struct ConvertJob {
  const void* in;
  void* out;
  int64_t n;
  int in_dt;
};
constexpr int kMaxConvertJobs = 10;
// One launch: [T, D] rows (fp32, bf16 or fp16) to fp16 (out may be null) with their partial column
// sums into partial [*parts, D] (at most kTailParts rows), and up to kMaxConvertJobs other jobs.
cudaError_t rows_to_f16_colsum(int64_t T, int D, int in_dt, const void* in, void* out, float* partial, int* parts,
                               const ConvertJob* jobs, int njobs, cudaStream_t st);
// Most partial rows rows_to_f16_colsum writes.
constexpr int kTailParts = 296;
size_t colsum_partial_floats(int cols);
cudaError_t convert_dtype(const void* in, int in_dt, void* out, int out_dt, int64_t n, cudaStream_t st);

cudaError_t column_sum(const void* in, int dt, int64_t rows, int cols, int64_t ld, float* partial, float* out,
                       cudaStream_t st);

cudaError_t launch_timeout_probe(int* status, cudaStream_t st);

// Backward of the input LayerNorm of the norm_in layer variant (norm_in.cu): dx = dy + LN_in^T(dxn)
// in x's dtype (and an fp16 copy when dx_f16), dgamma / dbeta through `partial`
// (ln_in_bwd_partial_floats(D) floats). x and dy: fp32 / fp32 or bf16 / bf16; D in {256, 512}.
size_t ln_in_bwd_partial_floats(int D);
cudaError_t ln_in_bwd(int64_t T, int D, int x_dt, int y_dt, const float* dxn, const void* x, const void* dy,
                      const float* gamma, const float* mu, const float* rstd, void* dx, void* dx_f16, float* partial,
                      float* dgamma, float* dbeta, cudaStream_t st);

// ---------------------------------------------------------------------------------------------
// Stochastic Length (stochastic_length.cu)
// ---------------------------------------------------------------------------------------------
cudaError_t launch_sl_lengths(const int64_t* offsets, int B, double alpha, int64_t* new_offsets, int* status,
                              cudaStream_t st);
cudaError_t launch_sl_select(const int64_t* offsets, int B, const int64_t* ts, const int64_t* keys,
                             const int64_t* new_offsets, const void* x, int64_t row_bytes, int64_t* kept, void* x_out,
                             int64_t* ts_out, int* status, cudaStream_t st);

}  // namespace hstu
