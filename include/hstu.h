/*
 * hstu.h - C ABI of the B200 (sm_100a) HSTU layer library (libhstu.so).
 *
 * The library computes the HSTU layer of Generative Recommenders over jagged (variable-length,
 * offset-indexed) user action sequences:
 *
 *   U, V, Q, K = Split(SiLU(X W1^T + b1))                                   (f1, phi1)
 *   O_i        = sum_{j <= i, same sequence} SiLU(q_i.k_j + rab_pos[i-j] + rab_time[b_ij]) / N * v_j
 *   Y          = (LayerNorm(O) (.) U) W2^T + b2 + X                          (f2 + residual)
 *
 * as stated in "4.4 Scaling Recommendation Models" (LLM learning path), section "Generative
 * Recommenders and HSTU" (the three layer equations and the pointwise-aggregation bullet) and
 * its section "Code" (chunk order U|V|Q|K, causal lower triangle including the diagonal, division
 * by a constant, LayerNorm over d_model, residual after f2); and in "HSTU: The First Exploration
 * of the Scaling Law" (fun-rec 7.1), 7.1.4 Innovations 1-3 and 7.1.5 (Stochastic Length,
 * M-FALCON).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor argument is a DEVICE pointer owned by the caller unless stated otherwise;
 *    descriptor structs are host memory read during the call only. The library never allocates,
 *    frees or synchronises: scratch space comes from a caller workspace whose size the matching
 *    *_workspace_size() returns. A workspace must be zero-filled once before its first use
 *    (it holds the device status word) and must not be shared by calls that overlap on the GPU.
 *  - Work is enqueued on `stream` (a cudaStream_t); calls return once it is enqueued.
 *  - The first call that needs them on each device sets kernel attributes and copies constant
 *    tables (the time-bucket thresholds) with synchronous CUDA calls. Make that first call outside
 *    any stream capture; after it, every call can be captured into a CUDA graph. Calls from
 *    several host threads are safe: the one-time setup is serialised, and hstu_last_cuda_error()
 *    is kept per host thread. The only exception is the workspace: calls that overlap on the GPU
 *    need workspaces of their own.
 *  - Matrices are row-major; ld_* arguments are row strides in ELEMENTS. bf16 tensors use the
 *    bfloat16 bit layout (uint16). Pointers handed to the tensor-core kernels must be 16-byte
 *    aligned and their row strides multiples of 8 elements (16 bytes).
 *  - Host-side argument errors return HSTU_ERR_INVALID_ARG / HSTU_ERR_UNSUPPORTED /
 *    HSTU_ERR_WORKSPACE before anything is enqueued. A CUDA launch error returns HSTU_ERR_CUDA
 *    (hstu_last_cuda_error() gives the cudaError_t). Errors found on the device (a bounded wait
 *    that ran out, a violated jagged contract) are recorded in the workspace status word and
 *    reported by hstu_sync_status(); the kernels then return early, never trap.
 *  - Jagged layout: sequence b owns rows [offsets[b], offsets[b+1]) of every [T, ...] tensor.
 *    offsets must be non-decreasing with offsets[0] = 0 and offsets[B] = T; max_len must bound
 *    every length. Timestamps are int64 (any unit, any order); the time bucket of a pair is
 *    min(n_buckets-1, floor(ln(max(t_i - t_j, 1)) / 0.301)), evaluated exactly in integers.
 *  - rab_pos has 2*pos_max_len-1 fp32 entries indexed by clip(i-j, -(L-1), L-1) + L-1 with i, j
 *    positions inside the sequence; rab_time has n_time_buckets (<= 128) fp32 entries. Both are
 *    shared by all heads.
 */
#ifndef HSTU_H_
#define HSTU_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HSTU_ABI_VERSION 1

typedef struct CUstream_st* hstu_stream_t; /* same type as cudaStream_t; NULL = legacy stream */

typedef enum hstu_status_t {
  HSTU_OK = 0,
  HSTU_ERR_INVALID_ARG = 1,  /* null pointer, negative size, inconsistent descriptor */
  HSTU_ERR_UNSUPPORTED = 2,  /* shape / dtype / alignment the kernels do not implement */
  HSTU_ERR_WORKSPACE = 3,    /* workspace missing or smaller than *_workspace_size() */
  HSTU_ERR_CUDA = 4,         /* a CUDA runtime call failed; see hstu_last_cuda_error() */
  HSTU_ERR_TIMEOUT = 5,      /* a bounded device-side wait ran out (reported on the device) */
  HSTU_ERR_DEVICE = 6        /* a device-side check failed (reported on the device) */
} hstu_status_t;

typedef enum hstu_dtype_t { HSTU_F32 = 0, HSTU_BF16 = 1, HSTU_F16 = 2 } hstu_dtype_t;

/* Jagged batch of B sequences, T tokens in total. */
typedef struct hstu_jagged_t {
  int32_t B;                  /* number of sequences (>= 0) */
  int32_t max_len;            /* host upper bound on every sequence length */
  int64_t T;                  /* total tokens = offsets[B] */
  const int64_t* offsets;     /* device, [B+1] */
  const int64_t* timestamps;  /* device, [T] */
} hstu_jagged_t;

/* Pointwise attention of one layer. */
typedef struct hstu_attn_desc_t {
  int32_t H;               /* heads */
  int32_t d_qk;            /* per-head query/key width (bf16/f16: 64; f32: 1..64) */
  int32_t d_v;             /* per-head value width (bf16/f16: 64; f32: 1..64) */
  float inv_N;             /* 1/N, the constant normaliser */
  int32_t pos_max_len;     /* L: rab_pos has 2L-1 entries */
  int32_t n_time_buckets;  /* 1..128 */
  hstu_dtype_t dtype;      /* dtype of q, k, v: BF16 or F16 (tensor cores) or F32 (CUDA cores). On
                              the tensor cores the score, the half-bias and P are fp16: a score
                              past 65504 makes O non-finite, which the forward records as
                              HSTU_ERR_DEVICE in the status word */
  hstu_dtype_t o_dtype;    /* dtype of out: F32 (any dtype) or BF16 (BF16 inputs only) */
  int64_t ld_q, ld_k, ld_v, ld_o; /* row strides (elements); head h occupies columns [h*d, (h+1)*d) */
} hstu_attn_desc_t;

/* One HSTU layer, d_qk = d_v = D/H. */
typedef struct hstu_layer_desc_t {
  int32_t D;               /* d_model */
  int32_t H;               /* heads */
  float inv_N;
  int32_t pos_max_len;
  int32_t n_time_buckets;
  float ln_eps;            /* LayerNorm epsilon (1e-5) */
  hstu_dtype_t dtype;      /* BF16: bf16 weights and activations on the tensor cores with fp32
                              accumulation: U|V|Q|K, Z, the attention weights P and G in fp16
                              (8x finer than bf16 at the same MMA rate), O in fp32; f2 reads an
                              fp16 copy of W2 (exact for bf16 values in the fp16 range).
                              Range: fp16 holds |v| <= 65504. A pre-activation Z outside that
                              range, or an attention score that drives O to inf / NaN, is recorded
                              as HSTU_ERR_DEVICE in the status word (the call's outputs are then not
                              meaningful); G = LayerNorm(O) (.) U is bounded by |gamma| sqrt(D) +
                              |beta| times |U| and is not checked.
                              F32: every step in fp32 on the CUDA cores */
  hstu_dtype_t x_dtype;    /* dtype of X; F32 with BF16 compute = fp32 residual stream (f1 then
                              reads an fp16 copy of X and of W1) */
  hstu_dtype_t y_dtype;    /* dtype of Y */
} hstu_layer_desc_t;

/* Layer parameters. W1 [4D, D] rows ordered U|V|Q|K, W2 [D, D], both of the compute dtype;
 * the vectors are fp32: b1 [4D], b2 [D], gamma [D], beta [D], rab_pos [2L-1], rab_time [nb].
 * gamma and beta (always) and W1, W2, b1, b2 (BF16 mode) are read by 16-byte vector loads and must
 * be 16-byte aligned (HSTU_ERR_UNSUPPORTED otherwise). The backward reads W1, W2, gamma, beta and
 * the two tables, not b1 or b2. */
typedef struct hstu_layer_weights_t {
  const void* W1;
  const float* b1;
  const void* W2;
  const float* b2;
  const float* gamma;
  const float* beta;
  const float* rab_pos;
  const float* rab_time;
} hstu_layer_weights_t;

/* Activations a layer forward writes and its backward reads. In BF16 mode uvqk [T, 4D] = SiLU(Z),
 * z [T, 4D] (the pre-activation; may be NULL when no backward follows) and g are fp16; in F32
 * mode all are fp32.
 * o [T, D] attention output, always fp32 (LayerNorm divides by its spread across features,
 * which is far smaller than its mean, so bf16 storage would be amplified); g [T, D] =
 * LN(O) (.) U; mu, rstd [T] fp32 LayerNorm statistics.
 * attn_bias (optional, BF16 mode; NULL = unused): hstu_layer_bias_cache_size(desc, jag) bytes,
 * 256-byte aligned. The forward then also writes there the attention backward's relative-bias
 * tiles (each causal 128 x 128 (query tile, key tile) pair's half-bias, key-major, and its time
 * buckets) and its key-tile work list, and a backward given the same struct reads them instead of
 * recomputing them (one bias launch and one work-list launch fewer). The backward leaves the
 * region as it found it, so several backwards may follow one forward. Valid only for the batch
 * and rab tables of the forward that wrote it. */
typedef struct hstu_layer_saved_t {
  void* uvqk;
  void* z;
  void* o;
  void* g;
  float* mu;
  float* rstd;
  void* attn_bias;
} hstu_layer_saved_t;

/* Weight gradients of one layer (fp32, overwritten): dW1 [4D, D], db1 [4D], dW2 [D, D], db2 [D],
 * dgamma [D], dbeta [D], drab_pos [2L-1], drab_time [nb]. */
typedef struct hstu_layer_grads_t {
  float* dW1;
  float* db1;
  float* dW2;
  float* db2;
  float* dgamma;
  float* dbeta;
  float* drab_pos;
  float* drab_time;
} hstu_layer_grads_t;

/* ---------------------------------------------------------------------------------------------
 * Library information and device status
 * ------------------------------------------------------------------------------------------- */

/* ABI version of the loaded library (HSTU_ABI_VERSION). */
int32_t hstu_abi_version(void);

/* Static string naming a status; never NULL. */
const char* hstu_status_string(hstu_status_t s);

/* The cudaError_t of the last failed CUDA call made by the library on this host thread. */
int32_t hstu_last_cuda_error(void);

/* Reads the device status word of `ws` (after synchronising `stream`), resets it to 0 and
 * stores it in *device_status (HSTU_OK when no kernel reported an error). The return value is
 * HSTU_OK unless reading itself failed. */
hstu_status_t hstu_sync_status(void* ws, hstu_stream_t stream, int32_t* device_status);

/* Upper bound, in SM clock cycles, of every device-side wait; 0 restores the default
 * (2^31 cycles, about a second). Process-wide; affects launches made after the call. */
void hstu_set_wait_limit(uint64_t cycles);

/* Kernel timing hook: `start` and `stop` are cudaEvent_t handles created by the caller (timing
 * enabled). Until the next call with the same `kernel`, every call of this host thread that launches
 * that kernel records `start` on its stream right before the launch and `stop` right after, so
 * cudaEventElapsedTime(start, stop) is that kernel's device time (under stream capture the records
 * become external event nodes of the graph, re-recorded at each replay). kernel: 0 the attention
 * forward (hstu_attn_fwd, hstu_layer_fwd), 1 the attention backward (hstu_attn_bwd,
 * hstu_layer_bwd), 2 the LayerNorm (.) U forward, 3 its backward, 4 the forward's bias-tile kernel
 * (with the layer's cache writes and fp16 W2 copy in hstu_layer_fwd), 5 the table gradients of the
 * attention backward, 6 the layer backward's dZ assembly. start = stop = NULL disables.
 * HSTU_ERR_INVALID_ARG for another kernel number or only one NULL event. */
hstu_status_t hstu_profile_events(int32_t kernel, void* start, void* stop);

/* Test surface for the failure path: launches one CTA that waits on an mbarrier nothing ever
 * arrives at, bounded by the wait limit; it records HSTU_ERR_TIMEOUT in the status word of `ws`
 * and returns. Lets a test check the timeout path without a hang. */
hstu_status_t hstu_debug_timeout_probe(void* ws, size_t ws_bytes, hstu_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * Jagged metadata  ("4.4 Scaling Recommendation Models", Efficiency tricks: kernels over
 * variable-length sequences; padding is never computed)
 * ------------------------------------------------------------------------------------------- */

/* Number of (sequence, 128-row query tile) items a batch can produce: B + ceil(T / 128). */
int64_t hstu_worklist_capacity(const hstu_jagged_t* jag);

/* Builds the causal tile work list: every (sequence b, query tile t) pair with t <
 * ceil(n_b/128), ordered by decreasing cost (tile t visits t+1 key tiles), ties by increasing b.
 * items: device int32 [capacity, 2] receiving (b, t); count: device int32 [1]. */
hstu_status_t hstu_jagged_worklist(const hstu_jagged_t* jag, int32_t* items, int32_t* count,
                                   hstu_stream_t stream);

/* Debug surface of the relative-time bias index ("HSTU: The First Exploration of the Scaling
 * Law", 7.1.4 Innovation 2): for every sequence b writes the n_b x n_b matrix of bucket(t_i -
 * t_j) (row i query, column j key, u8) at out + sq_offsets[b]; sq_offsets: device int64 [B+1],
 * the prefix sums of n_b^2. n_buckets in 1..128. It runs the attention's own bucket code tile by
 * tile (128 x 128 tiles of query and key rows): a tile whose timestamps span less than 2^31 - 1
 * takes 32-bit arithmetic, any other tile a 64-bit path that never overflows, exactly as in the
 * attention's bias tiles. max_len must bound every n_b (tiles past it are not written).
 * HSTU_ERR_UNSUPPORTED for B > 65535 or ceil(max_len / 128)^2 > 2^31 - 1. */
hstu_status_t hstu_time_buckets(const hstu_jagged_t* jag, int32_t n_buckets,
                                const int64_t* sq_offsets, uint8_t* out, hstu_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * Layer steps
 * ------------------------------------------------------------------------------------------- */

/* f1 + SiLU + split ("Generative Recommenders and HSTU", first equation):
 * uvqk[t, :] = SiLU(x[t, :] W1^T + b1), [T, 4D] with row stride 4D; b1 (nullable: no bias; 16-byte
 * aligned for BF16); z (nullable) receives the pre-activation. x and W1 have `dtype` (BF16 or
 * F32); uvqk and z have act_dtype (F16 or BF16 for BF16 operands, F32 for F32); ld_x is x's row
 * stride. ws: any workspace of at least 256 bytes (its status word receives device-side errors). */
hstu_status_t hstu_uvqk_fwd(int64_t T, int32_t D, hstu_dtype_t dtype, hstu_dtype_t act_dtype, const void* x,
                            int64_t ld_x, const void* W1, const float* b1, void* uvqk, void* z,
                            void* ws, size_t ws_bytes, hstu_stream_t stream);

/* Workspace bytes hstu_attn_fwd needs for this batch; 0 when the batch is malformed or so large
 * that its causal tile-pair bound times 128 rows exceeds 2^31 - 1 (the tile kernels' 32-bit row
 * coordinates; such a batch would need hundreds of GB of workspace), which the calls refuse with
 * HSTU_ERR_UNSUPPORTED. */
size_t hstu_attn_workspace_size(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag);

/* Pointwise causal attention forward ("Generative Recommenders and HSTU", second equation and
 * the pointwise-aggregation bullet; "HSTU: The First Exploration of the Scaling Law", 7.1.4
 * Innovations 1-2): out[i, h] = sum_{j<=i} SiLU(q_i.k_j + rab_pos + rab_time) * inv_N * v_j.
 * q, k, v, out: [T, ...] of desc->dtype with strides ld_q.. ld_o. Rows of empty work are not
 * written; every valid row is. */
hstu_status_t hstu_attn_fwd(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag,
                            const void* q, const void* k, const void* v, const float* rab_pos,
                            const float* rab_time, void* out, void* ws, size_t ws_bytes,
                            hstu_stream_t stream);

/* Workspace bytes hstu_attn_bwd needs for this batch: the work lists, per causal (query tile, key
 * tile) pair a transposed fp16 half-bias tile (32 KB) and a u8 bucket tile (16 KB), and per pair
 * and head a 16-bit dX^T tile (32 KB) from which the table gradients are summed over the heads.
 * The pair count is bounded from the batch's tile capacity and max_len (capacity (max_len/128 + 1)
 * / 2 pairs), so the size grows with H, T and max_len: about 1.5 GB for 30k tokens, max_len 4096
 * and 8 heads; 0.54 GB for 5.8k tokens, max_len 8192. 0 when the pair bound times H x 128 rows
 * exceeds 2^31 - 1, which hstu_attn_bwd refuses with HSTU_ERR_UNSUPPORTED. */
size_t hstu_attn_bwd_workspace_size(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag);

/* Pointwise causal attention backward (derived from the forward's definition; tensor-core dtypes
 * F16 / BF16 only). With x_ij = q_i.k_j + rab(i, j) and A_ij = SiLU(x_ij) inv_N on causal pairs:
 * dv = A^T dout, dq = dX k, dk = dX^T q with dX_ij = (dout_i . v_j) SiLU'(x_ij) inv_N, and
 * d_rab_pos / d_rab_time receive the sum over heads of dX_ij at the entry each pair reads.
 * q, k, v, d_out: desc->dtype with strides ld_q, ld_k, ld_v, ld_o. dq, dk, dv: fp32 [T, H*64],
 * row stride H*64, overwritten. d_rab_pos [2L-1], d_rab_time [nb]: fp32, overwritten. Gradients
 * are accumulated with atomics, so their summation order (and last bits) may differ run to run. */
hstu_status_t hstu_attn_bwd(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag,
                            const void* q, const void* k, const void* v, const void* d_out,
                            const float* rab_pos, const float* rab_time, float* dq, float* dk,
                            float* dv, float* d_rab_pos, float* d_rab_time, void* ws,
                            size_t ws_bytes, hstu_stream_t stream);

/* The richer relative bias of "HSTU: The First Exploration of the Scaling Law", 7.1.4 Innovation 2,
 * f(p_i - p_j, t_i - t_j, type_i, type_j), whose form the page does not give, read as the sum
 *   rab_pos[idx(i - j)] + rab_time[bucket(t_i - t_j)] + rab_type[type_i][type_j]
 * with every table either shared by the heads or given one slice per head (the first page's sketch
 * keeps a per-head bias table). */
typedef struct hstu_rab_ext_t {
  int32_t per_head;           /* 0: rab_pos [2L-1], rab_time [nb], rab_type [nt][nt] shared by the heads;
                                 1: rab_pos [H][2L-1], rab_time [H][nb], rab_type [H][nt][nt] */
  int32_t n_types;            /* nt: 0 = no type term, else 1..16 token types */
  const int32_t* token_type;  /* device int32 [T], each in [0, nt); NULL when nt = 0. A type outside
                                 that range is clamped into it and reported as HSTU_ERR_DEVICE. */
  const float* rab_type;      /* device fp32, query token's type first; NULL when nt = 0 */
} hstu_rab_ext_t;

/* Workspace bytes of hstu_attn_fwd_ext: hstu_attn_workspace_size with one bias tile per causal tile
 * pair and head when ext->per_head (H times the tile region); 0 for a batch or descriptor it
 * refuses (as hstu_attn_workspace_size, with the pair bound taken times H for per-head tables). */
size_t hstu_attn_ext_workspace_size(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag,
                                    const hstu_rab_ext_t* ext);

/* hstu_attn_fwd with the bias of hstu_rab_ext_t (tensor-core dtypes F16 / BF16 only). rab_pos and
 * rab_time have the shapes ext->per_head selects. HSTU_ERR_INVALID_ARG for per_head not 0 or 1, a
 * NULL ext, or nt > 0 with a NULL token_type / rab_type; HSTU_ERR_UNSUPPORTED for nt > 16 or an F32
 * descriptor; otherwise the errors of hstu_attn_fwd. */
hstu_status_t hstu_attn_fwd_ext(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag, const hstu_rab_ext_t* ext,
                                const void* q, const void* k, const void* v, const float* rab_pos,
                                const float* rab_time, void* out, void* ws, size_t ws_bytes, hstu_stream_t stream);

/* Workspace bytes of hstu_attn_bwd_ext (the transposed bias tiles per pair and head when
 * per_head); 0 for a refused batch. */
size_t hstu_attn_bwd_ext_workspace_size(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag,
                                        const hstu_rab_ext_t* ext);

/* hstu_attn_bwd with the bias of hstu_rab_ext_t: d_rab_pos, d_rab_time and d_rab_type (fp32, the
 * shapes of the tables, overwritten; d_rab_type NULL when nt = 0) receive, per entry, the sum of
 * dX_ij over every pair (and every head sharing the entry) that reads it. Errors as
 * hstu_attn_fwd_ext and hstu_attn_bwd. */
hstu_status_t hstu_attn_bwd_ext(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag, const hstu_rab_ext_t* ext,
                                const void* q, const void* k, const void* v, const void* d_out,
                                const float* rab_pos, const float* rab_time, float* dq, float* dk, float* dv,
                                float* d_rab_pos, float* d_rab_time, float* d_rab_type, void* ws,
                                size_t ws_bytes, hstu_stream_t stream);

/* Largest number of (sequence, 128-row tile) work items, B + ceil(T / 128), that
 * hstu_attn_fwd_noalloc accepts. */
#define HSTU_NOALLOC_MAX_ITEMS 65536

/* hstu_attn_fwd for callers that cannot allocate device memory and so cannot pass a workspace:
 * for example a serving process that reserves its whole memory budget at start-up and forbids
 * allocation on the request path, or a plain C host with no device allocator of its own. The
 * pages have no counterpart; it exists for integration only. Same arguments and result as
 * hstu_attn_fwd without ws / ws_bytes. Its scratch (status word, work list) is a fixed array of
 * 524,800 bytes compiled into the library: every GPU that loads the library holds it until the
 * process exits, and the call itself allocates and frees nothing.
 *  - Batches needing more than HSTU_NOALLOC_MAX_ITEMS work items return HSTU_ERR_WORKSPACE
 *    before anything is enqueued.
 *  - The first call on each device looks up that device's address of the array (with the device
 *    current); make that first call before any stream capture.
 *  - All calls share the one array and each call clears its status word: calls that overlap on
 *    the GPU (other streams, other host threads) race and must be serialised by the caller.
 *    Device-side errors of the last call (offsets that violate the jagged contract, a bounded wait
 *    that ran out) are read with hstu_attn_fwd_noalloc_status. */
hstu_status_t hstu_attn_fwd_noalloc(const hstu_attn_desc_t* desc, const hstu_jagged_t* jag,
                                    const void* q, const void* k, const void* v,
                                    const float* rab_pos, const float* rab_time, void* out,
                                    hstu_stream_t stream);

/* The device status word of hstu_attn_fwd_noalloc's built-in scratch on the current device: after
 * synchronising `stream` it is copied into *device_status (HSTU_OK, HSTU_ERR_DEVICE for offsets
 * that violated the jagged contract, HSTU_ERR_TIMEOUT for a bounded wait that ran out) and reset
 * to 0. Since every hstu_attn_fwd_noalloc call clears it first, it describes the last call
 * enqueued on this device; a call still running on another stream races with the read. Returns
 * HSTU_ERR_INVALID_ARG for a NULL device_status, HSTU_ERR_CUDA if a copy fails. Allocates
 * nothing. */
hstu_status_t hstu_attn_fwd_noalloc_status(hstu_stream_t stream, int32_t* device_status);

/* LayerNorm (.) U gating ("Generative Recommenders and HSTU", third equation; "HSTU: The First
 * Exploration of the Scaling Law", 7.1.4 Innovation 3): g = (gamma (o - mu) rstd + beta) (.) u
 * over all D features of a token; mu, rstd (fp32 [T]) are stored for the backward. g is [T, D]
 * with row stride D. Supported (o, u, g) dtypes: (F32, F32, F32), (F32, F16, F16),
 * (F32, F16 or BF16, BF16), (BF16, BF16, BF16). D in {64, 128, 256, 512, 1024}. */
hstu_status_t hstu_norm_gate_fwd(int64_t T, int32_t D, hstu_dtype_t o_dtype, hstu_dtype_t u_dtype,
                                 hstu_dtype_t g_dtype, const void* o, int64_t ld_o, const void* u,
                                 int64_t ld_u, const float* gamma,
                                 const float* beta, float eps, void* g, float* mu, float* rstd,
                                 hstu_stream_t stream);

/* f2 + residual ("Generative Recommenders and HSTU", third equation; residual of the "Code"
 * sketch): y = g W2^T + b2 + x. W2 has the compute dtype `dtype`; g has g_dtype (F32 compute: F32;
 * BF16 compute: BF16, or F16 with W2 read through an fp16 copy made in the workspace); x has
 * x_dtype; y has y_dtype; y_f16 (nullable) receives a second, fp16 copy of y (the next layer's
 * f1 operand when the residual stream is fp32). b2: nullable (no bias; 16-byte aligned for BF16).
 * ws: at least hstu_out_proj_workspace_size(D, g_dtype) bytes (status word, fp16 W2). F32 compute
 * needs F32 x and y. */
size_t hstu_out_proj_workspace_size(int32_t D, hstu_dtype_t g_dtype);
hstu_status_t hstu_out_proj_fwd(int64_t T, int32_t D, hstu_dtype_t dtype, hstu_dtype_t g_dtype,
                                const void* g, const void* W2, const float* b2, const void* x,
                                hstu_dtype_t x_dtype, void* y, hstu_dtype_t y_dtype,
                                void* y_f16, void* ws, size_t ws_bytes, hstu_stream_t stream);

/* Workspace bytes hstu_layer_fwd needs (0 for a batch hstu_attn_workspace_size refuses). */
size_t hstu_layer_workspace_size(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag);

/* Whole layer forward: uvqk -> attention -> norm-gate -> out-projection, on `stream`.
 * x: [T, D] of desc->x_dtype; x_f16 (nullable) an fp16 copy of x, the f1 operand when x_dtype is
 * F32 with BF16 compute (converted into the workspace when NULL; ignored otherwise). y: [T, D] of
 * desc->y_dtype; y_f16 (nullable) a second, fp16 copy of y (the next stacked layer's x_f16).
 * saved: buffers for the intermediates (all required except z). */
hstu_status_t hstu_layer_fwd(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag,
                             const hstu_layer_weights_t* w, const void* x, const void* x_f16,
                             void* y, void* y_f16, const hstu_layer_saved_t* saved, void* ws,
                             size_t ws_bytes, hstu_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * Backward of the layer (derived from the forward equations; no autograd)
 * ------------------------------------------------------------------------------------------- */

/* The projection GEMM both directions use: out[M, N] (=|+=) A B^T with A [M, K] and B [N, K] in
 * bf16, fp32 accumulation on the tensor cores. a_mn / b_mn = 0: the operand is stored row-major
 * as [M or N rows, K] (K-major); 1: stored row-major as [K rows, M or N] (MN-major, a transpose
 * for free). accumulate = 0: out = A B^T (+ bias[N]) (+ resid), out_dtype F32/BF16/F16;
 * accumulate = 1: out += A B^T in fp32 by atomics over K splits (bias and resid must be NULL).
 * N must be a multiple of 32, lda/ldb multiples of 8, pointers (bias included) 16-byte aligned.
 * lda >= K (K-major) or M (MN-major), ldb >= K or N, ld_out >= N, and with resid, ld_resid >= N
 * (HSTU_ERR_INVALID_ARG otherwise) with ld_resid rows starting on 16-byte boundaries
 * (HSTU_ERR_UNSUPPORTED otherwise). ws: >= 256 bytes. */
hstu_status_t hstu_linear_bf16(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda,
                               int32_t a_mn, const void* B, int64_t ldb, int32_t b_mn,
                               const float* bias, const void* resid, hstu_dtype_t resid_dtype,
                               int64_t ld_resid, void* out, hstu_dtype_t out_dtype, int64_t ld_out,
                               int32_t accumulate, void* ws, size_t ws_bytes, hstu_stream_t stream);

/* Workspace bytes hstu_layer_bwd needs (0 for a batch hstu_attn_bwd_workspace_size refuses). */
size_t hstu_layer_bwd_workspace_size(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag);

/* Bytes of hstu_layer_saved_t.attn_bias for this batch (0 for a batch hstu_attn_workspace_size
 * refuses): per causal tile pair a 32 KB fp16 half-bias tile and a 16 KB u8 bucket tile, then the
 * batch's key-tile work list (8 bytes per tile), per-sequence pair numbering (8 bytes) and packing
 * (4 bytes) after a 256-byte header. */
size_t hstu_layer_bias_cache_size(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag);

/* Whole layer backward (BF16 mode, D in {256, 512}), from the activations hstu_layer_fwd saved
 * (z required). x_f16: nullable fp16 copy of x (the dW1 operand; converted when NULL). dy: [T, D]
 * of desc->y_dtype (dy_f16: nullable fp16 copy, the operand of dG and dW2; converted when NULL);
 * dx: [T, D] of desc->x_dtype, overwritten with dy + dZ W1 (dx_f16: nullable fp16 copy, the
 * previous stacked layer's dy_f16). Every GEMM reads fp16 operands (exact copies of bf16 data).
 * Steps: dG = dy W2,
 * dW2 = dy^T G, db2 = sum dy; LayerNorm (.) U backward (dO, dU, dgamma, dbeta); attention
 * backward (dQ, dK, dV, table gradients); dZ = [dU|dV|dQ|dK] (.) SiLU'(Z); dW1 = dZ^T X,
 * db1 = sum dZ, dX = dy + dZ W1. All gradients fp32 and overwritten. The table gradients run on a
 * second stream the library keeps per host thread and device (made by the first call, which must
 * run outside any capture), forked from `stream` after the attention backward and joined back
 * before the call's last operation on `stream`: work later enqueued on `stream` sees every output. */
hstu_status_t hstu_layer_bwd(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag,
                             const hstu_layer_weights_t* w, const void* x, const void* x_f16,
                             const hstu_layer_saved_t* saved, const void* dy, const void* dy_f16,
                             void* dx, void* dx_f16, const hstu_layer_grads_t* grads, void* ws,
                             size_t ws_bytes, hstu_stream_t stream);

/* --------------------------------------------------------------------------------------------
 * The input-LayerNorm variant of the layer ("4.4 Scaling Recommendation Models", section Code: the
 * sketch normalises the layer input before f1, Xn = LayerNorm_in(X) over d_model with gamma_in,
 * beta_in and eps = desc->ln_eps, and adds the raw X as the residual):
 *   U, V, Q, K = Split(SiLU(Xn W1^T + b1)),  Y = f2(LayerNorm(A V) (.) U) + X.
 * BF16 compute, D in {256, 512}; X of desc->x_dtype (BF16 or F32), Y of desc->y_dtype.
 * -------------------------------------------------------------------------------------------- */
typedef struct hstu_norm_in_t {
  const float* gamma;   /* [D], 16-byte aligned */
  const float* beta;    /* [D], 16-byte aligned */
  void* xn;             /* fp16 [T, D], 16-byte aligned: Xn, written by the forward, read by the backward */
  float* mu;            /* [T]: LayerNorm_in statistics, written by the forward */
  float* rstd;          /* [T] */
  float* dgamma;        /* [D]: the backward's gradients of gamma and beta (fp32, overwritten) */
  float* dbeta;         /* [D] */
} hstu_norm_in_t;

/* Workspace bytes of both hstu_layer_fwd_norm_in and hstu_layer_bwd_norm_in (0 for a batch they refuse). */
size_t hstu_layer_norm_in_workspace_size(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag);

/* Forward: Xn, mu, rstd into nin; the layer on Xn as in hstu_layer_fwd (saved as there), with X as
 * the residual. Errors of hstu_layer_fwd, plus HSTU_ERR_INVALID_ARG for a NULL nin member the call
 * writes or reads and HSTU_ERR_UNSUPPORTED for another compute dtype, D or an unaligned pointer. */
hstu_status_t hstu_layer_fwd_norm_in(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag,
                                     const hstu_layer_weights_t* w, const hstu_norm_in_t* nin, const void* x, void* y,
                                     void* y_f16, const hstu_layer_saved_t* saved, void* ws, size_t ws_bytes,
                                     hstu_stream_t stream);

/* Backward: as hstu_layer_bwd with dW1 = dZ^T Xn, then dXn = dZ W1 through the input LayerNorm:
 * dX = dY + LN_in^T(dXn) (dx of desc->x_dtype, dx_f16 nullable fp16 copy), nin->dgamma and
 * nin->dbeta overwritten. dy: [T, D] of desc->y_dtype, which must equal desc->x_dtype. */
hstu_status_t hstu_layer_bwd_norm_in(const hstu_layer_desc_t* desc, const hstu_jagged_t* jag,
                                     const hstu_layer_weights_t* w, const hstu_norm_in_t* nin, const void* x,
                                     const hstu_layer_saved_t* saved, const void* dy, void* dx, void* dx_f16,
                                     const hstu_layer_grads_t* grads, void* ws, size_t ws_bytes,
                                     hstu_stream_t stream);

/* --------------------------------------------------------------------------------------------
 * Data parallelism ("4.4 Scaling Recommendation Models", Generative Recommenders and HSTU,
 * Efficiency tricks: the sequences of a batch are independent, so one global batch is split over
 * ranks by whole sequences and the only exchange is the gradient sum). Host functions; no CUDA.
 * -------------------------------------------------------------------------------------------- */

/* Work of one layer step on a sequence of n tokens, in units of 2 D flops: n (n + 1) + 5 D n (the
 * attention's 2 D n (n + 1) flops plus the projections' 10 D^2 n). */
double hstu_dp_sequence_cost(int64_t n, int32_t D);

/* Assigns each of B sequences (lengths: HOST int64 [B]) to one of `world` ranks, balancing
 * hstu_dp_sequence_cost: sequences by decreasing cost (ties by index), each to the least loaded rank
 * (ties by lowest rank); deterministic, so every rank computes the same split. The largest rank load
 * is at most 4/3 of the best split's. rank_of: HOST int32 [B], receives the rank of each sequence;
 * rank_cost: HOST double [world] or NULL, receives each rank's summed cost. HSTU_ERR_INVALID_ARG for
 * B < 0, world < 1, D < 1, a negative length or a NULL array when B > 0. */
hstu_status_t hstu_dp_partition(const int64_t* lengths, int32_t B, int32_t D, int32_t world, int32_t* rank_of,
                                double* rank_cost);

/* Events for overlapping the gradient all-reduce of data parallelism with the rest of a backward:
 * until the next call, every hstu_layer_bwd of this host thread records `early` once dW2, db2,
 * dgamma, dbeta, db1, drab_pos and drab_time are final (before the f1 backward GEMMs; on the call's
 * second stream, which has then seen all of them), and
 * `w1` once dW1 is final too (after the launch that computes dX and dW1; with the input-LayerNorm
 * variant, before its backward). A communication stream that waits on them can reduce those
 * gradients while the remaining kernels run. Under stream capture they are
 * recorded as capture dependencies, so a stream that waits on them forks from the captured graph.
 * Both NULL disables; HSTU_ERR_INVALID_ARG when only one is NULL. */
hstu_status_t hstu_layer_bwd_ready_events(void* early, void* w1);

/* --------------------------------------------------------------------------------------------
 * Stochastic Length ("HSTU: The First Exploration of the Scaling Law", 7.1.5 Stochastic Length):
 * a history of n tokens keeps L = min(n, floor(n^(alpha/2) + 1/2)) tokens, the L tokens with the
 * smallest random keys (ties broken by position), in their original order; positions are
 * renumbered 0..L-1 and timestamps travel with their tokens. The random keys are an input: one
 * int64 per raw token (a uniformly random subset follows from i.i.d. uniform keys).
 * -------------------------------------------------------------------------------------------- */

/* new_offsets (device, [B+1]) = exclusive prefix of L_b over raw's sequences, alpha in [0, 2]
 * (HSTU_ERR_INVALID_ARG otherwise). L is evaluated in double precision. ws: >= 256 bytes (status word; a malformed raw offsets array is reported as
 * HSTU_ERR_DEVICE by hstu_sync_status). The caller reads new_offsets[B] = T' to size the outputs
 * of hstu_stochastic_length_select. */
hstu_status_t hstu_stochastic_length_offsets(const hstu_jagged_t* raw, double alpha, int64_t* new_offsets,
                                             void* ws, size_t ws_bytes, hstu_stream_t stream);

/* Selects the kept tokens of every sequence: kept (device int64 [T']) receives their global raw
 * indices in order, ts_out (nullable, [T']) their timestamps, and x_out (nullable, [T', D] of
 * x_dtype) their rows of x ([T_raw, D]). new_offsets must come from
 * hstu_stochastic_length_offsets with the same raw batch and alpha. Rows are copied as bytes in
 * 16-byte units: with x_out, D * element size must be a multiple of 16 and x, x_out 16-byte
 * aligned (HSTU_ERR_UNSUPPORTED otherwise). */
hstu_status_t hstu_stochastic_length_select(const hstu_jagged_t* raw, const int64_t* keys,
                                            const int64_t* new_offsets, const void* x,
                                            hstu_dtype_t x_dtype, int32_t D, int64_t* kept,
                                            void* x_out, int64_t* ts_out, void* ws, size_t ws_bytes,
                                            hstu_stream_t stream);

/* --------------------------------------------------------------------------------------------
 * M-FALCON candidate scoring ("HSTU: The First Exploration of the Scaling Law", 7.1.5 M-FALCON).
 *
 * A stack of L layers (all BF16 mode, one hstu_layer_weights_t each) scores m candidates per
 * user against that user's history (the prefix). Layer l of candidate c of user u sees, as keys,
 * every prefix token j of u through layer l (relative position n_u - j, time difference
 * request_ts[u] - t_j) and itself (relative position 0, time difference 0); candidates never see
 * one another. Its attention output is
 *   O_c = inv_N * ( sum_j SiLU(q_c.k_j + rab_pos[idx(n_u - j)] + rab_time[bucket(request_ts[u] - t_j)]) v_j
 *                   + SiLU(q_c.k_c + rab_pos[idx(0)] + rab_time[0]) v_c ),
 * which equals the last row of a causal layer over [prefix, c]; LayerNorm (.) U, f2 and the
 * residual follow as in hstu_layer_fwd, and the layer's output is the next layer's input. The
 * residual stream between layers is fp32 (BF16 compute with an fp32 X, as in a stacked encoder).
 *
 * The prefix's K and V of every layer are computed once (cache_valid = 0: the prefix runs through
 * the L causal layers and kv_cache is filled) and reused by every candidate micro-batch of b_m
 * candidates per user (the result does not depend on b_m). With cache_valid = 1, kv_cache must
 * hold the K|V of the same prefix and weights from an earlier call, and prefix_x is not read.
 * -------------------------------------------------------------------------------------------- */
typedef struct hstu_falcon_desc_t {
  int32_t L;               /* layers (>= 1) */
  int32_t users;           /* number of users == prefix->B */
  int32_t m;               /* candidates per user (>= 0) */
  int32_t b_m;             /* candidates per user in one pass (micro-batch), >= 1 */
  int32_t D, H;            /* d_model, heads (D/H = 64) */
  float inv_N;
  int32_t pos_max_len;     /* every n_u < pos_max_len keeps the positions unclipped */
  int32_t n_time_buckets;
  float ln_eps;
} hstu_falcon_desc_t;

/* Bytes of the K|V cache: L x T_prefix x 2D fp16 (layer l, token t: K in columns [0, D), V in
 * [D, 2D)). The caller owns it; it outlives a call when cache_valid = 1 is used later. */
size_t hstu_falcon_cache_size(const hstu_falcon_desc_t* desc, const hstu_jagged_t* prefix);
size_t hstu_falcon_workspace_size(const hstu_falcon_desc_t* desc, const hstu_jagged_t* prefix);

/* layers: HOST array of L weight structs (device pointers inside, W1/W2 bf16).
 * prefix: B = users jagged prefixes (offsets, int64 timestamps), max_len >= every n_u.
 * prefix_x: bf16 [T_prefix, D] (read only when cache_valid = 0).
 * kv_cache: fp16, hstu_falcon_cache_size() bytes; written when cache_valid = 0, read always.
 * prefix_out: fp32 [T_prefix, D], the prefix's output of the last layer, or NULL (only written
 *   when cache_valid = 0).
 * cand_x: bf16 [users * m, D], user u's candidates in rows [u m, (u+1) m).
 * request_ts: device int64 [users], the request time of each user.
 * out: fp32 [users * m, D], the candidates' output of the last layer.
 * Errors: the host checks of hstu_layer_fwd (D % 64 == 0, D/H == 64; every layer's W1, W2, b1,
 * b2, gamma and beta present and 16-byte aligned; the prefix batch within the tile-pair bound of
 * hstu_attn_workspace_size) plus HSTU_ERR_INVALID_ARG for users != prefix->B, L < 1 or b_m < 1.
 * hstu_falcon_cache_size and hstu_falcon_workspace_size return 0 for a refused descriptor. */
hstu_status_t hstu_falcon_fwd(const hstu_falcon_desc_t* desc, const hstu_layer_weights_t* layers,
                              const hstu_jagged_t* prefix, const void* prefix_x, void* kv_cache,
                              int32_t cache_valid, void* prefix_out, const void* cand_x,
                              const int64_t* request_ts, void* out, void* ws, size_t ws_bytes,
                              hstu_stream_t stream);

/* M-FALCON prefix append ("HSTU: The First Exploration of the Scaling Law", 7.1.5 M-FALCON: the
 * history's K, V cache is reused across requests): extends every user's cached prefix by new actions
 * without recomputing the old prefix. In a causal layer a token's K and V do not depend on later
 * tokens, so the old rows' cache entries are kept and only the appended tokens run through the L
 * layers, each attending to the whole cached prefix and to the appended tokens before it (their
 * positions continue from n_old, their timestamps are those of prefix_new).
 *  prefix_old: the cached prefixes (users = B, n_old_u tokens each); kv_cache_old as written by
 *    hstu_falcon_fwd (cache_valid = 0) or an earlier append for them.
 *  appended: B = users jagged rows of the new actions (offsets: device [users+1]; timestamps unused),
 *    their bf16 input rows in app_x [appended->T, D].
 *  prefix_new: the combined prefixes, n_old_u + a_u tokens per user (old tokens first), with the
 *    combined timestamps; kv_cache_new (hstu_falcon_cache_size(desc, prefix_new) bytes, not
 *    overlapping kv_cache_old) receives the combined cache, ready for hstu_falcon_fwd with
 *    cache_valid = 1 on prefix_new.
 *  app_out: fp32 [appended->T, D] or NULL, the appended tokens' last-layer output (equal to the rows
 *    a full causal forward over prefix_new gives them).
 * Errors: those of hstu_falcon_fwd for prefix_new, HSTU_ERR_INVALID_ARG when prefix_old or appended
 * do not have `users` sequences or prefix_old->T + appended->T != prefix_new->T; a user whose
 * combined length is not n_old + a is reported as HSTU_ERR_DEVICE and left out. */
size_t hstu_falcon_append_workspace_size(const hstu_falcon_desc_t* desc, const hstu_jagged_t* prefix_old,
                                         const hstu_jagged_t* appended, const hstu_jagged_t* prefix_new);
hstu_status_t hstu_falcon_append(const hstu_falcon_desc_t* desc, const hstu_layer_weights_t* layers,
                                 const hstu_jagged_t* prefix_old, const void* kv_cache_old,
                                 const hstu_jagged_t* appended, const void* app_x, const hstu_jagged_t* prefix_new,
                                 void* kv_cache_new, void* app_out, void* ws, size_t ws_bytes, hstu_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_H_ */
