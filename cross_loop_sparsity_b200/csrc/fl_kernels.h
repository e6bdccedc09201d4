// fl_kernels.h -- argument blocks and launchers of the non-GEMM kernels.
#pragma once
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "fl_cache.cuh"
#include "fl_internal.h"

namespace fl {

// RoPE and the KV write of freshly projected rows (k_qkv_post).
struct QkvPostArgs {
  const float* qkv;   // [n][(H+2Hkv)*hd] fp32, GEMM row order
  int ldq;
  const int* idx;     // GEMM row -> call token (nullptr = identity)
  int n;
  const int* seq;     // call token -> sequence
  const int* pos;     // call token -> position
  int H, Hkv, hd;
  const float* rope_cos;  // [max_ctx][hd/2]
  const float* rope_sin;
  CacheView cv;
  int j, loop, lazy;
  float* q_cur;       // [n][H][hd] GEMM order
  float* q_last;      // [N][H][hd] token order (this layer), written at loop 1
  const int* forced_on;           // forced residual codes (checks): [0] != 0 when on
  const int8_t* forced_codes;     // [M][K-1][ns][2][Hkv][hd]
  const uint16_t* forced_scales;  // [M][K-1][ns][2][Hkv][hd/g]
  int forced_ns;                  // selection-slot stride ns
  // checks only: the rotated fp32 K/V rows each lazy loop quantised,
  // [M][K-1][trace_ns][2][Hkv][hd] by (layer, loop 2..K, selection slot, K/V,
  // KV head); slots >= trace_ns are not written (nullptr: off)
  float* trace_kv;
  int trace_ns;
};


struct AttnDecArgs {
  const float* q_cur;
  const int* idx;
  const int* seq;
  const int* pos;
  CacheView cv;
  int j, loop, dense;
  int H, Hkv, hd;
  float tau;
  int n_splits;       // CTAs per (token, KV head); split sp takes column tiles [sp*nt/n_splits, (sp+1)*nt/n_splits)
  float* part_o;      // [n][Hkv][splits][8][hd]
  float* part_ml;     // [n][Hkv][splits][8][2]
  int* counters;      // [n][Hkv], zero between launches
  float* o_state;     // [N][H][hd] token order (nullptr for the dense baseline)
  float* lse_state;   // [N][H]
  uint16_t* o_bf16;   // [n][H*hd] GEMM order
  int* status;        // error bits (a bounded wait that ran out)
};

struct AttnPreArgs {
  const float* q_cur;  // [B*T][H][hd] token order
  const int* pos;      // [B*T] absolute position of each call token (chunk after the context)
  CacheView cv;
  int j, loop, dense;
  int T, H, Hkv, hd;
  float tau;
  float* o_state;
  float* lse_state;
  uint16_t* o_bf16;
  int* status;         // error bits (a bounded wait that ran out)
};

struct TilePlan {
  int* tile;    // [max_tiles] query tile of plan entry p
  int* qb;      // first / one-past-last index into the selection of its queries
  int* qe;
  int* need;    // plan entries whose tile needs a column set
  int* counts;  // [0] entries, [1] entries needing a column set
};

// One selected slot of the current loop, written by the selection step: the
// token and what the attention-side kernels need about it, in one 32-byte record
// (last = the loop whose KV the token's attention state was computed with).
struct alignas(32) SelMeta {
  int tok, seq, tile, last, pos, pad0, pad1, pad2;
};

struct SelectStepArgs {
  const float* h;        // [N][d] current hidden states
  const float* h_in;     // [N][d] call inputs (change after loop 1)
  float* h_snap;         // [n_sel][d] loop-start rows of the selected tokens (read, then rewritten)
  int* sel_slot;         // [N] slot of each token in the selection, or -1 (read, then rewritten)
  int N, d, loop, n_sel;
  int n_tiles;           // query tiles of the call (tile flags read and set)
  float* key;            // [N]
  float* keys_trace;     // [N] this loop's keys, kept for read-back
  int32_t* idx;          // [n_sel] this loop's selection
  int* last;             // [N]
  const int* tile;       // [N]
  int* has_c;            // [tiles]
  const int* forced_on;
  const int32_t* forced;
  TilePlan plan;
  const int* seq;        // [N] sequence of each token
  const int* pos;        // [N] position of each token
  SelMeta* meta;         // [n_sel] written for the selected slots
  // optional: the first layer's attention RMSNorm of the selected rows,
  // x[r] = bf16(h[idx[r]] * rsqrt(mean(h^2) + eps) * gain) for r < n_sel and
  // zero rows for n_sel <= r < x_rows (nullptr gain: not fused)
  const float* norm_gain;
  uint16_t* x;
  int x_rows;
  float eps;
  // sparse residual storage (cv.rows > 0): pool rows of the recomputed tokens
  CacheView cv;
  int B_call;            // sequences of the call (its N tokens are B_call runs of N / B_call)
  int* status;
};

struct SelColsArgs {
  TilePlan plan;
  const int32_t* idx;
  const int* pos;
  const SelMeta* meta;  // [n_sel] per selected slot
  const float* col_keys;
  int max_cols, Hkv, c, j, n_tiles;
  int32_t* cols;        // [M][n_tiles][Hkv][c]
  int* ncols;           // [M][n_tiles][Hkv]
  const int* forced_on;
  const int32_t* forced_cols;
  const int* forced_ncols;
  // rows longer than kSelColsSmemKeys: each slice of kSelColsSmemKeys keys
  // keeps its own top-c (grid.y = slices), the last slice CTA of a row (ticket)
  // takes the top-c of their union
  float* cand_keys;     // [max_need][Hkv][max_slices][c]
  int32_t* cand_idx;    // [max_need][Hkv][max_slices][c] ascending global column ids
  int* cand_counters;   // [max_need][Hkv], zero between launches
  int max_slices;
};

struct DScoreArgs {
  TilePlan plan;
  const int32_t* idx;
  const int* seq;
  const int* pos;
  const SelMeta* meta;  // [n_sel] per selected slot
  const float* q_cur;   // GEMM order
  const float* q_last;  // token order (this layer)
  CacheView cv;
  int j, loop, H, Hkv, hd;
  float tau;
  float* col_keys;      // [max_need][Hkv][max_cols]
  int max_cols;
  int max_chunks;       // 64-column chunks of the longest row (set by the launcher)
  int ds_block;         // columns per work item of the SIMT kernel (set by the launcher)
  int* work;            // tensor-core kernel: [2] next work item, CTAs finished (zero between launches)
  int tc;               // 1: the tensor-core kernel (prefill tiles, head_dim 128)
  // 1: the CTA finishing a row's last chunk also selects its column set (rows of
  // at most kSelColsSmemKeys columns), with `sel`; row_tickets [max_need][Hkv]
  // count finished chunks (zero between launches)
  int fold;
  SelColsArgs sel;
  int* row_tickets;
  // checks only: every tile's keys by query tile, [M][trace_tiles][Hkv][max_cols]
  // (tiles >= trace_tiles are not written; nullptr: off)
  float* trace_ck;
  int trace_tiles;
};


struct CorrectArgs {
  const int32_t* idx;
  const int* seq;
  const int* pos;
  const int* tile;
  const int* last;
  const float* q_cur;
  const float* q_last;   // the loop-1 queries (token order)
  float* o_state;               // loop-1 O, then (after the token's first recomputation) the rest's numerator
  float* lse_state;             // loop-1 lse, then the rest's maximum
  float* z_state;               // the rest's denominator
  uint16_t* o_bf16;
  const int32_t* cols;
  const int* ncols;
  const SelMeta* meta;          // [n_sel] per selected slot (the clustered path reads this)
  CacheView cv;
  int j, loop, H, Hkv, hd, c, n_tiles;
  float tau;
  int cols_per_cta, n_splits;   // column split: grid.y = n_splits = ceil(c / cols_per_cta)
  int cluster;                  // decode (each query its own tile, few queries): one cluster per
                                // (query, group), merged over distributed shared memory
  int tc;                       // prefill tiles, head_dim 128: the tensor-core kernel, per (tile, group)
  TilePlan plan;                // (tc) the loop's query tiles and their selected slots
  int q_tile, max_entries;      // (tc) query tile size; bound on the plan's entries
  int* work;                    // (tc) [2] next work item, CTAs finished (zero between launches)
  float* part_acc;              // [n_sel][Hkv][n_splits][2][8][hd]: new-term, old-term numerators
  float* part_mz;               // [n_sel][Hkv][n_splits][8][3]: max, new-term, old-term denominators
  int* counters;                // [n_sel][Hkv], zero between launches
  int* status;
};

cudaError_t kernels_init_attrs();

// forced_on bits: the token selections, the column sets
constexpr int kForceSel = 1, kForceCols = 2;

constexpr int kLensByValue = 256;
constexpr int kSelectStepMax = 1024;   // tokens (and query tiles) the one-CTA selection kernel handles
constexpr int kSelectStepMaxNorm = 64;   // selected rows it also normalises (first layer's input)
constexpr int kSelectStepSlices = 16;    // 512-element slices of a row it normalises (d <= 8192)
static_assert(kSelectStepMaxNorm * kSelectStepSlices <= kSelectStepMax, "norm sums reuse the key array");
struct LensArg {
  int n;
  int v[kLensByValue];
};
cudaError_t launch_reset_lens(const LensArg& a, int* seq_len, cudaStream_t s);
constexpr int kCorrWarps = 16;            // warps per CTA of the clustered correction
constexpr int kSelColsSmemKeys = 16384;   // column keys the top-c selection stages in shared memory (64 KB)
constexpr int kCorrCluster = 16;  // CTAs per (query, KV group) in the clustered correction (non-portable size)
// Launches made while this is on (the kernels of one call) are programmatic
// dependents of the previous kernel; thread-local.
void set_pdl(bool on);

cudaError_t launch_select_tokens(const float* keys, int N, int n_sel, int32_t* idx, const int* forced_on,
                                 const int32_t* forced, cudaStream_t s);
cudaError_t launch_rmsnorm_rows(const float* h, const int* idx, int n, int n_pad, int d, const float* gain, float eps,
                                uint16_t* x, cudaStream_t s);
cudaError_t launch_qkv_post(const QkvPostArgs& a, cudaStream_t s);
// kv: the cache's bf16 rows ([rows][hd], 64 x 64 boxes, 128-byte swizzle) in
// the layout the context uses (lazy base or dense per-loop)
cudaError_t launch_attn_decode(const CUtensorMap& kv, const AttnDecArgs& a, int n, cudaStream_t s);
// kv: the cache's bf16 rows ([rows][hd], 64 x 64 boxes, 128-byte swizzle), as for the decode attention
cudaError_t launch_attn_prefill(const CUtensorMap& kv, const AttnPreArgs& a, int B, cudaStream_t s);
// Prefill attention kernel choice for launches from this thread: tensor cores (default) or fp32 SIMT.
void set_tc_prefill(bool on);
// stamps (nullptr: none): the call's GEMM launch stamps [2][n_stamps], cleared here
cudaError_t launch_setup_call(int N, int decode, int T, int tiles_per_seq, int q_tile, const int* seq_len, int* seq,
                              int* pos, int* tile, int* last, int n_tiles, int* has_c, unsigned long long* stamps,
                              int n_stamps, cudaStream_t s);
cudaError_t launch_set_lens(int B, int* seq_len, int add, cudaStream_t s);
// h[r] += e + gamma * x[r] for the n rows r = idx ? idx[i] : i (e may be nullptr)
cudaError_t launch_loop_input(float* h, const int* idx, int n, int d, const float* e, float gamma, const float* x,
                              cudaStream_t s);
// selection slots, snapshot of the selected rows and their SelMeta records
// (the path for calls too large for the one-CTA selection step)
cudaError_t launch_after_select(const int32_t* idx, int n_sel, int N, int d, int* sel_slot, const float* h,
                                float* h_snap, const int* seq, const int* tile, const int* last, const int* pos,
                                SelMeta* meta, cudaStream_t s);
cudaError_t launch_change_keys(const float* h, const float* ref, const int* sel_slot, int N, int d, int loop,
                               float* key, int* last, const int* tile, int* has_c, cudaStream_t s);
cudaError_t launch_select_step(const SelectStepArgs& a, cudaStream_t s);
// sparse residual storage: pool rows of a lazy loop's recomputed tokens (calls
// too large for the selection step), and the pool counts after a length reset
cudaError_t launch_assign_rows(const CacheView& cv, int loop, int B, int Tc, const int* sel_slot, const int* pos,
                               int* status, cudaStream_t s);
cudaError_t launch_reset_rows(const CacheView& cv, const int* seq_len, cudaStream_t s);
// sparse residual storage: import one (layer, sequence) slice of a lazy context
// (int8 codes, fp16 scales by position), and export one (layer, loop, K/V,
// sequence) slice back to packed rows by position
cudaError_t launch_import_rows(const CacheView& cv, int j, int b, int n, const int8_t* ck, const int8_t* cvv,
                               const uint16_t* sk, const uint16_t* sv, int* status, cudaStream_t s);
cudaError_t launch_export_rows(const CacheView& cv, int j, int l, int kv, int b, int n, uint8_t* codes,
                               uint16_t* scales, cudaStream_t s);
cudaError_t launch_plan_tiles(const int32_t* idx, int n_sel, const int* tile, const int* has_c, const TilePlan& p,
                              cudaStream_t s);
cudaError_t launch_dscore(const DScoreArgs& a, int max_need, int max_chunks, cudaStream_t s);
cudaError_t launch_select_cols(const SelColsArgs& a, int max_need, int max_cols_now, cudaStream_t s);
// slices of a row of column keys the top-c selection splits it into
__host__ __device__ inline int select_cols_slices(int n) { return n <= kSelColsSmemKeys ? 1 : (n + kSelColsSmemKeys - 1) / kSelColsSmemKeys; }
cudaError_t launch_correct(const CorrectArgs& a, int n_sel, cudaStream_t s);


cudaError_t launch_pack_codes(const int8_t* src, int rows, int hd, int bits, uint8_t* dst, size_t dst_row_stride,
                              cudaStream_t s);

}  // namespace fl
