/*
 * flashloop.h -- C ABI of the B200 (sm_100a) lazy-update looped-Transformer
 * inference library.
 *
 * The method is the one in "FlashLoop: Fast and Memory-Efficient Looped
 * Transformers via Lazy Updates" (abstract): a shared Transformer block is
 * applied K times; after the first loop only the tokens whose hidden state
 * changed most are recomputed (token-sparse updates), their attention output
 * is corrected over a sparse, stable set of key columns (sparse attention),
 * and each loop's KV cache is the previous loop's plus a low-bit residual
 * (KV-residual quantisation).  The dense baseline is the plain looped forward
 * with a per-loop KV cache ("Looped Transformer 教程：权重共享、循环次数与推理
 * 成本怎么读", 第一步 and 第四步).
 *
 * Conventions for every entry point:
 *  - Device pointers are CUDA global-memory addresses on the device that was
 *    current at flashloop_init.  Where an argument says "host or device", the
 *    library asks CUDA which it is and stages host buffers through its
 *    workspace (pinned host memory makes those copies asynchronous).
 *  - bf16 tensors are passed as uint16_t bit patterns; linear weights are
 *    row-major [out_features][in_features], stacked over layers.
 *  - All work is enqueued on the given stream and returns without waiting,
 *    except where stated.  One context is used from one stream at a time.
 *  - Nothing aborts and no C++ exception crosses this boundary: every
 *    failure is a fl_status.  The library never allocates device memory; the
 *    caller provides one workspace buffer and owns every buffer it passes.
 */
#ifndef FLASHLOOP_H
#define FLASHLOOP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fl_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  FL_OK = 0,
  FL_ERR_INVALID_ARG = 1, /* a NULL/misaligned pointer, an out-of-range size or knob */
  FL_ERR_CAPACITY = 2,    /* batch > max_batch, tokens > max_tokens, context > max_ctx, or (from
                             flashloop_sync_status) a sparse residual pool ran out of rows */
  FL_ERR_WORKSPACE = 3,   /* workspace smaller than flashloop_workspace_bytes() or misaligned */
  FL_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed (see flashloop_last_cuda_error) */
  FL_ERR_TIMEOUT = 5,     /* a kernel's bounded wait ran out; the kernel returned early */
  FL_ERR_NONFINITE = 6,   /* a corrected softmax denominator was not positive (non-finite result) */
  FL_ERR_UNSUPPORTED = 7  /* a configuration this build does not implement */
} fl_status;

/* Model and method knobs.  resid_bits: 4 or 2 = lazy path with int4/int2 KV
 * residuals; 16 = dense looped baseline (every loop recomputes every token and
 * keeps its own bf16 KV; rho and c_cols are ignored). */
typedef struct {
  int d_model;      /* d; multiple of 64 */
  int n_heads;      /* H query heads */
  int n_kv_heads;   /* Hkv; H % Hkv == 0 (grouped-query attention) */
  int head_dim;     /* hd: 64 or 128 */
  int ffn_dim;      /* SwiGLU hidden size; multiple of 8 */
  int n_layers;     /* M: layers of the shared block */
  int n_loops;      /* K: block applications per token, 1..16 */
  double rho;       /* fraction of tokens recomputed at loops >= 2, in (0, 1] */
  int c_cols;       /* key columns kept per (query tile, KV head), >= 1 */
  int q_tile;       /* prefill query-tile length in positions (128) */
  int resid_bits;   /* 4, 2 or 16 (see above) */
  int group_size;   /* quantiser group along head_dim; divides hd, multiple of 32 */
  float resid_scale;/* s: h += s * branch output (0.3) */
  float rms_eps;    /* RMSNorm epsilon (1e-6) */
  float rope_theta; /* RoPE base (10000) */
  int vocab;        /* LM-head rows V */
  int max_batch;    /* sequences held in the cache */
  int max_ctx;      /* positions per sequence held in the cache */
  int max_tokens;   /* largest B*T of one prefill call (decode needs max_batch) */
  int kv_mode;      /* dense path only: 0 = per_loop (every loop keeps its own KV), 1 = last_loop (one KV
                       per layer that every loop overwrites, "Looped Transformer 教程", 第四步:
                       recurrent_kv_cache_mode); must be 0 on the lazy path */
  /* Variants around the looped core ("从'堆层数'到'循环复用'：FlashLoop 到底在解决什么问题",
   * §3.1, §3.2, §4.1; "Looped Transformer 教程", 第三步).  All zero: the plain looped block. */
  int n_prelude;    /* P independent layers before the loop, applied once to every token, own KV */
  int n_coda;       /* Q independent layers after the loop, likewise */
  int loop_embed;   /* 1: loop k's input is h + e_k (weights.loop_embed) */
  float inject_scale; /* gamma: loop k's input also adds gamma * x, x = the state entering the loop */
  /* Sparse residual storage (lazy path): 0 = one residual row per position and loop; R > 0 = residual rows
   * are kept only for the tokens a loop recomputed, in a pool of R rows per (layer, loop, K/V, sequence,
   * KV head) plus a 4-byte row index per (layer, loop, sequence, position) -- the KV-cache memory
   * reduction of "FlashLoop ...", abstract.  Rows are taken in position order; a call that needs more
   * than R rows keeps no residual for the excess tokens and flashloop_sync_status reports
   * FL_ERR_CAPACITY.  0 <= R <= max_ctx. */
  int resid_rows;
} flashloop_config;

/* A stack of L layers' weights (device pointers, stacked over layers). */
typedef struct {
  const float* attn_norm;     /* [L][d] fp32 gains */
  const uint16_t* w_qkv;      /* [L][(H+2Hkv)*hd][d] bf16; rows: q heads, k heads, v heads */
  const uint16_t* w_o;        /* [L][d][H*hd] bf16 */
  const float* mlp_norm;      /* [L][d] fp32 gains */
  const uint16_t* w_gate;     /* [L][ffn][d] bf16 */
  const uint16_t* w_up;       /* [L][ffn][d] bf16 */
  const uint16_t* w_down;     /* [L][d][ffn] bf16 */
} flashloop_layers;

/* Device pointers to the weights (borrowed for the context's lifetime). */
typedef struct {
  const float* attn_norm;     /* [M][d] fp32 gains */
  const uint16_t* w_qkv;      /* [M][(H+2Hkv)*hd][d] bf16; rows: q heads, k heads, v heads */
  const uint16_t* w_o;        /* [M][d][H*hd] bf16 */
  const float* mlp_norm;      /* [M][d] fp32 gains */
  const uint16_t* w_gate;     /* [M][ffn][d] bf16 */
  const uint16_t* w_up;       /* [M][ffn][d] bf16 */
  const uint16_t* w_down;     /* [M][d][ffn] bf16 */
  const float* final_norm;    /* [d] fp32 gains */
  const uint16_t* w_out;      /* [V][d] bf16 */
  flashloop_layers prelude;   /* n_prelude layers (ignored when 0) */
  flashloop_layers coda;      /* n_coda layers (ignored when 0) */
  const float* loop_embed;    /* [K][d] fp32 loop embeddings e_1..e_K (loop_embed = 1; else ignored) */
} flashloop_weights;

typedef struct flashloop_ctx flashloop_ctx;

/* Bytes of device workspace a context with this config needs (host arithmetic
 * only; 0 if the config is invalid).  The workspace holds the KV cache, the
 * per-call attention state, activations, selection buffers and split-K
 * scratch; it must be 256-byte aligned. */
size_t flashloop_workspace_bytes(const flashloop_config* cfg);

/* Validate cfg, lay out the workspace, build TMA descriptors for the weights
 * and zero the cache.  Enqueues on `stream` (the zeroing and the RoPE table
 * upload) and waits for it before returning.  *out receives a host-allocated
 * context (free with flashloop_destroy). */
fl_status flashloop_init(const flashloop_config* cfg, const flashloop_weights* w,
                         void* workspace, size_t workspace_bytes, fl_stream_t stream,
                         flashloop_ctx** out);

/* Prefill a chunk of T tokens onto each of sequences 0..B-1: token t of
 * sequence b sits at position len_b + t, after whatever the sequence already
 * holds (len_b = 0 for a fresh prompt; a later chunk continues a prompt, or
 * follows decode steps).  The looped block over the call's tokens: loop 1 runs
 * every token with causal attention over the cache's positions 0..len_b + t;
 * loops 2..K recompute the top ceil(rho*B*T) tokens by change norm (pooled over
 * the call, ties to the lower flat index b*T+t) with their attention corrected
 * over the fixed top-c key columns of their query tile ("FlashLoop: Fast and
 * Memory-Efficient Looped Transformers via Lazy Updates", abstract: token-sparse
 * updates, sparse stable key columns, KV residuals); query tiles are q_tile
 * consecutive tokens of one sequence's chunk, counted from its first token,
 * and see every earlier column of the sequence.
 * h0: [B*T][d] fp32 input hidden states, sequence-major (host or device).
 * h_out: [B*T][d] fp32 final hidden states after K loops (host or device, may be NULL).
 * logits_last: [B][V] fp32 logits of each sequence's last position (host or device, may be NULL).
 * Errors: FL_ERR_INVALID_ARG (NULL h0, B or T < 1), FL_ERR_CAPACITY (B >
 * max_batch, B*T > max_tokens, or len_b + T > max_ctx), FL_ERR_CUDA.  On
 * return the sequences' lengths have grown by T. */
fl_status flashloop_prefill(flashloop_ctx* ctx, const float* h0, int B, int T,
                            float* h_out, float* logits_last, fl_stream_t stream);

/* Append one token to each of sequences 0..B-1 at position len_b: the same
 * lazy looped step as flashloop_prefill ("FlashLoop ...", abstract), or with
 * resid_bits 16 the dense looped forward with one KV pass per loop ("Looped
 * Transformer 教程：权重共享、循环次数与推理成本怎么读", 第一步 and 第四步).
 * h0: [B][d] fp32 (host or device); h_out: [B][d] fp32 or NULL; logits: [B][V]
 * fp32 or NULL (host or device).  The ranking pools the B new tokens; each new
 * token is its own query tile.  The step's kernels are captured once per B
 * into a CUDA graph and replayed.  Lengths advance by one.
 * Errors: FL_ERR_INVALID_ARG (NULL h0, B < 1), FL_ERR_CAPACITY (B > max_batch,
 * or a sequence at max_ctx), FL_ERR_CUDA. */
fl_status flashloop_decode_step(flashloop_ctx* ctx, const float* h0, int B,
                                float* h_out, float* logits, fl_stream_t stream);

/* KV-cache bytes ("FlashLoop ...", abstract: the KV-cache memory the residual
 * form saves): *total = bytes of the allocated cache layout (looped layers, plus
 * one pass for each prelude / coda layer); per token and looped layer:
 * *per_token_per_layer for this config (lazy: the bf16 base plus K-1 packed
 * residual rows and their fp16 scales; dense per_loop: K passes; last_loop:
 * one) and *dense_per_token_per_layer for dense per-loop bf16 KV (K * 2 * Hkv *
 * hd * 2 bytes), the reference the reduction is quoted against.  Host
 * arithmetic; FL_ERR_INVALID_ARG for a NULL context. */
fl_status flashloop_kv_bytes(const flashloop_ctx* ctx, size_t* total, double* per_token_per_layer,
                             double* dense_per_token_per_layer);

/* The same figures from a config alone (host arithmetic, no context needed):
 * total = bytes of the cache layout flashloop_init would lay out. */
fl_status flashloop_kv_bytes_for(const flashloop_config* cfg, size_t* total, double* per_token_per_layer,
                                 double* dense_per_token_per_layer);

/* Set every sequence length (seq_len: [max_batch] host array, or NULL for all
 * zero).  Cache contents are kept; used to replay a decode step at a fixed
 * context.  Enqueued on `stream` as one small kernel (max_batch <= 256),
 * without waiting. */
fl_status flashloop_reset(flashloop_ctx* ctx, const int* seq_len, fl_stream_t stream);

/* Synchronise `stream` and report the first error a kernel recorded since
 * the last call, clearing it: FL_ERR_TIMEOUT (a bounded wait ran out),
 * FL_ERR_CAPACITY (a sparse residual pool was full), FL_ERR_NONFINITE (a
 * corrected softmax denominator was not positive). */
fl_status flashloop_sync_status(flashloop_ctx* ctx, fl_stream_t stream);

void flashloop_destroy(flashloop_ctx* ctx);
const char* flashloop_status_string(fl_status s);
/* The last CUDA error string seen by this context ("" if none). */
const char* flashloop_last_cuda_error(const flashloop_ctx* ctx);

/* ------------------------------------------------------------------------ */
/* Cache import / export (synthetic decode contexts; checks).               */
/* ------------------------------------------------------------------------ */

/* Load one (layer, sequence) slice of a lazy cache from device buffers:
 * base_k/base_v: [Hkv][n][hd] bf16; codes_k/v: [K-1][Hkv][n][hd] int8 codes in
 * [-qmax, qmax] (packed by the library); scales_k/v: [K-1][Hkv][n][hd/g] fp16
 * bits.  Rows 0..n-1 of that sequence are written.  resid_bits 2/4 only. */
fl_status flashloop_import_lazy(flashloop_ctx* ctx, int layer, int seq, int n,
                                const uint16_t* base_k, const uint16_t* base_v,
                                const int8_t* codes_k, const int8_t* codes_v,
                                const uint16_t* scales_k, const uint16_t* scales_v,
                                fl_stream_t stream);

/* Load one (layer, sequence) slice of a dense cache: kv_k/kv_v [KS][Hkv][n][hd]
 * bf16, KS = K loops (per_loop) or 1 (last_loop).  resid_bits 16 only. */
fl_status flashloop_import_dense(flashloop_ctx* ctx, int layer, int seq, int n,
                                 const uint16_t* kv_k, const uint16_t* kv_v, fl_stream_t stream);

/* Load one (independent layer, sequence) slice of the prelude / coda KV: x in
 * [0, n_prelude) for the prelude, n_prelude + i for coda layer i; kv_k/kv_v
 * [Hkv][n][hd] bf16 (device buffers).  FL_ERR_INVALID_ARG when x, seq or n is out
 * of range or a pointer is NULL. */
fl_status flashloop_import_extra(flashloop_ctx* ctx, int x, int seq, int n, const uint16_t* kv_k,
                                 const uint16_t* kv_v, fl_stream_t stream);

/* Copy one (layer, loop, sequence) slice of the residual store to device
 * buffers: codes [Hkv][n][hd*bits/8] packed bytes, scales [Hkv][n][hd/g] fp16
 * bits (loop 2..K); loop 1 copies the base: base [2][Hkv][n][hd] bf16 into
 * `codes` (K then V) and leaves `scales` untouched.  `which`: 0 = K, 1 = V. */
fl_status flashloop_export_slice(const flashloop_ctx* ctx, int layer, int loop, int seq, int which,
                                 int n, void* codes, void* scales, fl_stream_t stream);

/* Force the selections of the next call (checks only): sel [K-1][n_sel]
 * strictly ascending token indices in [0, N) of that call for loops 2..K
 * (not checked on the host; n_sel must be the call's own selection count);
 * cols [M][n_tiles][Hkv][c_cols]
 * ascending column indices with ncols [M][n_tiles][Hkv] valid entries (host
 * arrays).  Either part may be NULL: sel NULL leaves the token selection free,
 * cols and ncols NULL (both) leave the column sets free; all NULL clears.
 * n_tiles is B for decode, B*ceil(T/q_tile) for prefill.  The kernels still
 * compute every key; only the chosen indices are replaced.  cols without ncols
 * (or the reverse), or sizes outside the context's capacity, return
 * FL_ERR_INVALID_ARG. */
fl_status flashloop_force_selection(flashloop_ctx* ctx, const int32_t* sel, int n_sel_loops, int n_sel,
                                    const int32_t* cols, const int32_t* ncols, int n_tiles);

/* Force the residual codes of the next call's recomputed tokens (checks
 * only): codes int8 [M][K-1][n_sel][2][Hkv][hd] in [-qmax, qmax] and fp16 scale
 * bits [M][K-1][n_sel][2][Hkv][hd/g], for layer, loop 2..K, selection slot,
 * K (0) / V (1), KV head (host arrays; NULL clears).  The quantiser's decisions
 * turn small floating-point differences into whole code steps, so a check of a
 * call's arithmetic against another implementation hands over these integer
 * decisions along with the selections; the quantiser itself is checked
 * bit-exactly on identical inputs (fl_test_quantize). */
fl_status flashloop_force_codes(flashloop_ctx* ctx, const int8_t* codes, const uint16_t* scales, int n_sel);

/* Check buffers written by the following calls (device pointers, caller-owned;
 * NULL turns each off).  kv_rows: fp32 [M][K-1][n_slots][2][Hkv][hd], the
 * rotated new K (0) and V (1) rows that a lazy loop l >= 2 quantised, by (layer,
 * loop, selection slot, K/V, KV head) -- the inputs of the KV-residual quantiser
 * ("FlashLoop ...", abstract: each loop's KV as a low-bit residual over the
 * previous loop's); rows are written only where the library quantised them itself (not
 * under flashloop_force_codes) and only for slots < n_slots.  col_keys: fp32
 * [M][n_tiles][Hkv][max_ctx], the delta-score key of every eligible column of
 * each query tile whose column set the call chose ("FlashLoop ...", abstract:
 * the sparse, stable subset of key columns), by global query tile (decode: the
 * sequence; prefill: b * ceil(T / q_tile) + t / q_tile); tiles >= n_tiles are not
 * written.  Pointers must be 16-byte aligned.  Captured decode graphs are
 * dropped and captured again.  FL_ERR_INVALID_ARG for a dense context, a
 * non-positive capacity or a misaligned pointer. */
fl_status flashloop_set_trace(flashloop_ctx* ctx, float* kv_rows, int n_slots, float* col_keys, int n_tiles);

/* Read back the last call's choices (host buffers): sel [K-1][n_sel]; keys
 * [K-1][N] fp32 selection keys of loops 2..K; cols/ncols as above.  Any may be
 * NULL.  Synchronises `stream`. */
fl_status flashloop_read_trace(flashloop_ctx* ctx, int32_t* sel, float* keys, int32_t* cols,
                               int32_t* ncols, fl_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Unit entry points on caller buffers (device pointers).                    */
/* ------------------------------------------------------------------------ */

/* Top-k selection per segment: keys fp32 [n_seg][n]; for segment s the k
 * largest by (IEEE bit pattern as uint32 descending, index ascending), written
 * in ascending index order to idx [n_seg][k] (k = min(k, n)).  Token-sparse
 * updates and the top-c key columns ("FlashLoop ...", abstract). */
fl_status fl_test_topk(const float* keys, int n_seg, int n, int k, int32_t* idx, fl_stream_t stream);

/* Per-group absmax quantiser: r fp32 [rows][width] (width % g == 0); writes
 * packed codes [rows][width*bits/8] and fp16 scale bits [rows][width/g]:
 * s = fp16_RU(fp32(absmax/qmax)), code = clamp(rint(fp32(r/s))) (KV-residual
 * quantisation, "FlashLoop ...", abstract).  bits 4 or 2; g in {32, 64,
 * 128}; width a multiple of 128, or 64 with g <= 64; r 16-byte aligned.
 * Anything else returns FL_ERR_INVALID_ARG before any launch. */
fl_status fl_test_quantize(const float* r, int rows, int width, int g, int bits,
                           uint8_t* codes, uint16_t* scales, fl_stream_t stream);

/* The quantiser applied to the residual of new KV rows against the previous
 * loop's reconstruction: r = fp32(x) - fp32(prev) (IEEE round-to-nearest), then
 * exactly as fl_test_quantize (KV-residual quantisation, "FlashLoop ...",
 * abstract).  x fp32 [rows][width], prev bf16 [rows][width], both 16-byte
 * aligned; the other arguments, limits and errors as fl_test_quantize. */
fl_status fl_test_quantize_residual(const float* x, const uint16_t* prev, int rows, int width, int g, int bits,
                                    uint8_t* codes, uint16_t* scales, fl_stream_t stream);

/* tcgen05 GEMM: D[m][n] = sum_k A[m][k] * B[n][k] (bf16 operands, fp32
 * accumulate); A [m][k] and B [n][k] row-major bf16, D fp32 [m][n]; k % 8 == 0,
 * all pointers 16-byte aligned.  swap_ab = 0: the persistent prefill kernel,
 * A's rows on the MMA M side (128-row tiles) and B in 256-row tiles, one CTA
 * per SM walking the output tiles.  swap_ab = 1: the skinny orientation
 * used for decode (B's rows on the MMA M side, m <= 64 rows of A as the MMA N
 * side), with the reduction split across CTAs; `scratch` must then hold
 * fl_test_gemm_scratch_bytes() bytes (caller-allocated device memory). */
size_t fl_test_gemm_scratch_bytes(int m, int n, int k, int swap_ab);
fl_status fl_test_gemm(const uint16_t* A, const uint16_t* B, float* D, int m, int n, int k, int swap_ab,
                       void* scratch, size_t scratch_bytes, fl_stream_t stream);

/* Decode-shaped GEMM for callers that cannot allocate device memory.  The
 * paper has no counterpart: this is a service of the library, not a step of
 * the method.  Some callers may not call cudaMalloc at all -- code running in
 * another framework's memory pool that already owns the device memory,
 * latency-critical paths that cannot afford cudaMalloc's implicit device
 * synchronisation, plugin hosts that forbid allocation -- yet the skinny
 * split-K GEMM (fl_test_gemm with swap_ab = 1) needs scratch for its partial
 * tiles and tickets.  This variant computes the same D[m][n] = sum_k A[m][k] *
 * B[n][k] (bf16 in, fp32 out; 1 <= m <= 64, k % 8 == 0, pointers 16-byte
 * aligned, all device memory owned by the caller) with its scratch in an
 * array compiled into the library: FL_NOALLOC_SCRATCH_BYTES of split-K
 * partials plus 16 KiB of tickets, held on every GPU that loads the library
 * until the process exits.  It allocates nothing.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Shapes whose partials exceed FL_NOALLOC_SCRATCH_BYTES are refused with
 *    FL_ERR_CAPACITY and a reason in flashloop_last_cuda_error(NULL); use
 *    fl_test_gemm with caller scratch for those.
 *  - Every call shares the one array and leaves its contents behind; the
 *    tickets are cleared on the call's stream before each launch.  Calls that
 *    overlap on the GPU (other streams, other host threads) race on it.
 *  - There is no context to report a kernel's failure through: if a bounded
 *    wait inside the kernel runs out, the affected output tile is written as
 *    NaN, never as a silently wrong product. */
#define FL_NOALLOC_SCRATCH_BYTES (2u << 20)
fl_status fl_gemm_skinny_noalloc(const uint16_t* A, const uint16_t* B, float* D, int m, int n, int k,
                                 fl_stream_t stream);

/* Runtime options of a context. */
typedef enum {
  FL_OPT_USE_GRAPH = 1, /* 1 (default): capture decode steps into CUDA graphs; 0: launch directly */
  FL_OPT_PROFILE = 2,   /* 1: bracket every kernel of a call with CUDA events (read with flashloop_profile) */
  FL_OPT_PDL = 3,       /* 1 (default): launch each kernel of a call as a programmatic dependent of the
                           previous one, so its launch and set-up overlap the predecessor */
  FL_OPT_GEMM_TIMES = 5, /* 1: every GEMM launch of a call stamps, from the GPU's global nanosecond timer, when
                           its first CTA's dependency wait returned and when its last CTA finished (read with
                           flashloop_gemm_times); 0 (default): off */
  FL_OPT_TC_PREFILL = 6, /* 1 (default): prefill attention, delta scores and correction on warp-level bf16
                           tensor-core products with fp32 accumulation (attention and correction: queries
                           as bf16 hi + lo pairs; delta scores: the fp32 query difference, rounded once);
                           0: the fp32 SIMT kernels */
  FL_OPT_CORR_CLUSTER = 7 /* 1 (default): a decode query's column correction runs as one 16-CTA cluster merged
                           over distributed shared memory; 0: column slices merged by an atomic ticket */
} fl_option;
fl_status flashloop_set_option(flashloop_ctx* ctx, fl_option opt, int value);

/* Kernel kinds reported by flashloop_profile. */
enum {
  FL_KIND_GEMM = 0,      /* tcgen05 GEMMs (QKV, O, gate/up, down, LM head) */
  FL_KIND_ATTN = 1,      /* dense attention (decode splits + merge, or prefill) */
  FL_KIND_DSCORE = 2,    /* delta-score column keys */
  FL_KIND_CORRECT = 3,   /* sparse-column correction */
  FL_KIND_KV = 4,        /* RoPE + KV store / residual quantise */
  FL_KIND_SELECT = 5,    /* token / column top-k, tile plan, snapshots */
  FL_KIND_NORM = 6,      /* RMSNorm gathers */
  FL_KIND_OTHER = 7,     /* change keys, bookkeeping */
  FL_NUM_KINDS = 8
};

/* Per-kind kernel time of the last prefill / decode call made with
 * FL_OPT_PROFILE on: synchronises `stream`, then writes ms[kind] (summed
 * device time of that kind's kernels, from CUDA events recorded around each
 * launch) and launches[kind].  Arrays have FL_NUM_KINDS entries. */
fl_status flashloop_profile(flashloop_ctx* ctx, fl_stream_t stream, float* ms, int* launches);

/* Number of kernels the last prefill / decode call enqueued (all kinds). */
int flashloop_kernels_per_call(const flashloop_ctx* ctx);

/* Device time of the GEMMs of the last call made with FL_OPT_GEMM_TIMES on
 * (the shared-block projections and the LM head, "FlashLoop ...", abstract:
 * the recomputed tokens' block): synchronises `stream`, then *total_ms = the
 * sum over the call's GEMM launches of (last CTA's end - first return from the
 * dependency wait), so launches never overlap in the sum and it cannot exceed
 * the call's duration; *launches = the GEMM launches timed.  FL_ERR_INVALID_ARG
 * when the option is off or a pointer is NULL. */
fl_status flashloop_gemm_times(flashloop_ctx* ctx, fl_stream_t stream, double* total_ms, int* launches);

#ifdef __cplusplus
}
#endif
#endif /* FLASHLOOP_H */
