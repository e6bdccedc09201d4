// fl_kernels.h -- argument blocks and launchers of the non-GEMM kernels.
#pragma once
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "fl_cache.cuh"
#include "fl_internal.h"

namespace fl {


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
  CacheView cv;
  int j, loop, dense;
  int T, H, Hkv, hd;
  float tau;
  float* o_state;
  float* lse_state;
  uint16_t* o_bf16;
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
  // checks only: every tile's keys by query tile, [M][trace_tiles][Hkv][max_cols]
  // (tiles >= trace_tiles are not written; nullptr: off)
  float* trace_ck;
  int trace_tiles;
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
};

struct CorrectArgs {
  const int32_t* idx;
  const int* seq;
  const int* pos;
  const int* tile;
  const int* last;
  const float* q_cur;
  float* q_last;
  float* o_state;
  float* lse_state;
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
  float* part_acc;              // [n_sel][Hkv][n_splits][8][hd]
  float* part_mz;               // [n_sel][Hkv][n_splits][8][2]
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
constexpr int kCorrWarps = 16;
constexpr int kSelColsSmemKeys = 16384;   // column keys the top-c kernel stages in shared memory (64 KB)   // warps per CTA of the clustered correction
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
cudaError_t launch_attn_prefill(const AttnPreArgs& a, int B, cudaStream_t s);
cudaError_t launch_setup_call(int N, int decode, int T, int tiles_per_seq, int q_tile, const int* seq_len, int* seq,
                              int* pos, int* tile, int* last, int n_tiles, int* has_c, cudaStream_t s);
cudaError_t launch_set_lens(int B, int* seq_len, int add, int value, cudaStream_t s);
// selection slots, snapshot of the selected rows and their SelMeta records
// (the path for calls too large for the one-CTA selection step)
cudaError_t launch_after_select(const int32_t* idx, int n_sel, int N, int d, int* sel_slot, const float* h,
                                float* h_snap, const int* seq, const int* tile, const int* last, const int* pos,
                                SelMeta* meta, cudaStream_t s);
cudaError_t launch_change_keys(const float* h, const float* ref, const int* sel_slot, int N, int d, int loop,
                               float* key, int* last, const int* tile, int* has_c, cudaStream_t s);
cudaError_t launch_select_step(const SelectStepArgs& a, cudaStream_t s);
cudaError_t launch_plan_tiles(const int32_t* idx, int n_sel, const int* tile, const int* has_c, const TilePlan& p,
                              cudaStream_t s);
cudaError_t launch_dscore(const DScoreArgs& a, int max_need, int max_chunks, cudaStream_t s);
cudaError_t launch_select_cols(const SelColsArgs& a, int max_need, cudaStream_t s);
cudaError_t launch_correct(const CorrectArgs& a, int n_sel, cudaStream_t s);


cudaError_t launch_pack_codes(const int8_t* src, int rows, int hd, int bits, uint8_t* dst, size_t dst_row_stride,
                              cudaStream_t s);

}  // namespace fl
