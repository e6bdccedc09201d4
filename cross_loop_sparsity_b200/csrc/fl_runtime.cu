// fl_runtime.cu -- host runtime and C ABI: configuration checks, workspace
// layout, TMA descriptors, the per-call kernel sequence (prefill and decode),
// CUDA-graph capture of decode steps, cache import/export and test entry points.
//
// One call runs the looped block K times over its tokens ("FlashLoop: Fast and
// Memory-Efficient Looped Transformers via Lazy Updates", abstract):
//   loop 1     : every token, dense attention; writes the bf16 base KV
//   loop l >= 2: top ceil(rho*N) tokens by ||h_{l-1} - h_{l-2}||^2 recompute;
//                their KV is stored as a quantised residual; their attention is
//                corrected over the fixed top-c key columns of their query tile
// The dense baseline (resid_bits 16) recomputes every token every loop with a
// per-loop bf16 KV ("Looped Transformer 教程", 第一步 / 第四步).
#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "flashloop.h"
#include "fl_kernels.h"

using namespace fl;

namespace {
std::string g_last_error;  // last CUDA error of an entry point that has no context
}  // namespace

void fl::set_last_error(const std::string& why) { g_last_error = why; }

struct flashloop_ctx {
  flashloop_config cfg;
  flashloop_weights w;
  uint8_t* ws = nullptr;
  size_t ws_bytes = 0;
  int device = 0;
  CacheView cv{};
  bool lazy = true;
  int qkv_rows = 0, N_max = 0, N_pad = 0, n_tiles_max = 0, max_need = 0;
  int dec_splits = 1;   // decode attention: column-tile ranges per (token, KV head)
  // workspace regions
  float *rope_cos = nullptr, *rope_sin = nullptr;
  int *seq_len = nullptr, *status = nullptr;
  float *h = nullptr, *h_in = nullptr, *h_snap = nullptr;
  uint16_t *x = nullptr, *obf = nullptr, *act = nullptr;
  float *qkv = nullptr, *q_cur = nullptr;
  float *o_state = nullptr, *lse_state = nullptr, *z_state = nullptr, *q_last = nullptr;
  int *seq = nullptr, *pos = nullptr, *tile = nullptr, *last = nullptr, *sel_slot = nullptr;
  float *key = nullptr, *keys_trace = nullptr;
  int32_t *idx_all = nullptr, *idx_sel = nullptr, *idx_last = nullptr;
  int* has_c = nullptr;
  TilePlan plan{};
  int32_t* cols = nullptr;
  int* ncols = nullptr;
  float* col_keys = nullptr;
  float* cand_keys = nullptr;     // slice candidates of long column-key rows
  int32_t* cand_idx = nullptr;
  int* cand_cnt = nullptr;
  int* row_tickets = nullptr;     // finished chunks of each column-key row (the folded selection)
  int max_slices = 1;
  int* forced_on = nullptr;
  int32_t *forced_sel = nullptr, *forced_cols = nullptr;
  int* forced_ncols = nullptr;
  int8_t* forced_codes = nullptr;
  uint16_t* forced_scales = nullptr;
  int* forced_codes_on = nullptr;
  int nsel_max = 0;
  float *part_o = nullptr, *part_ml = nullptr;
  int* attn_counters = nullptr;
  float *corr_acc = nullptr, *corr_mz = nullptr;
  int* corr_counters = nullptr;
  int* work_ctr = nullptr;        // [0..1] delta-score, [2..3] correction: next item, CTAs finished
  float* gemm_partial = nullptr;
  size_t gemm_partial_cap = 0;
  int* gemm_counters = nullptr;
  float* ss_part = nullptr;      // [ss_tiles][kSsLd] per-tile sums of squares of updated rows
  SelMeta* sel_meta = nullptr;   // [N] records of the current loop's selected slots
  int ss_tiles = 0;
  float* logits_ws = nullptr;
  // prelude / coda (independent layers, one-pass KV each) and loop-input variants
  CacheView cvx{};            // their KV: dense layout with one loop slot, n_prelude + n_coda layers
  // descriptors
  CUtensorMap tm_qkv, tm_o, tm_gate, tm_up, tm_down, tm_out;
  CUtensorMap tm_x_qkv[2], tm_x_o[2], tm_x_gate[2], tm_x_up[2], tm_x_down[2];   // prelude [0], coda [1]
  CUtensorMap tm_kvx;         // the independent layers' KV rows for the decode attention
  CUtensorMap tm_x_a, tm_obf_a, tm_act_a;
  CUtensorMap tm_x_b[3], tm_obf_b[3], tm_act_b[3];
  CUtensorMap tm_kv;   // the cache's bf16 rows for the decode attention
  // host state
  std::vector<int> lens;
  std::vector<int> graph_b;
  std::vector<cudaGraphExec_t> graph_exec;
  std::vector<int> eager_seen;
  int use_graph = 1;
  int pdl = 1;                        // FL_OPT_PDL
  int prof = 0;                       // FL_OPT_PROFILE
  int gemm_times = 0;                 // FL_OPT_GEMM_TIMES
  int tc_prefill = 1;                 // FL_OPT_TC_PREFILL
  int corr_cluster = 1;               // FL_OPT_CORR_CLUSTER
  unsigned long long* stamps = nullptr;   // [2][kMaxStamps]: launch start (min), end (max) per GEMM of a call
  int stamp_slots = 0;                // GEMM launches of the last call (capped at kMaxStamps)
  std::vector<cudaEvent_t> ev;        // start/end pairs of the last profiled call
  std::vector<int> ev_kind;
  int ev_used = 0;
  int launches = 0;                   // kernels enqueued by the last call
  std::string last_err;
  int last_N = 0, last_nsel = 0, last_decode = 0, last_tiles = 0;
  // check buffers (caller device memory; nullptr: off)
  float* trace_kv = nullptr;
  int trace_ns = 0;
  float* trace_ck = nullptr;
  int trace_tiles = 0;
};

namespace {

// Sparse-column correction: columns per CTA.  Few selected queries (decode)
// get narrow splits for parallelism; many (prefill) get wide ones.
constexpr int kCorrColsSmall = 16, kCorrColsBig = 128, kCorrSmallQueries = 64;
// Calls of at most this many tokens do a lazy loop's bookkeeping in one CTA.
constexpr int kSsLd = 64;                // tokens per row of the sums-of-squares table (swap GEMMs: <= 64)
constexpr int kCountersGemm = 4096;
constexpr int kMaxStamps = 4096;         // GEMM launches of one call that are timed

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
int ceil_div(int a, int b) { return (a + b - 1) / b; }

int n_select(double rho, int n) {
  if (n <= 0) return 0;
  int k = static_cast<int>(std::ceil(rho * n - 1e-9));
  if (k < 1) k = 1;
  if (k > n) k = n;
  return k;
}

bool valid_config(const flashloop_config* c) {
  if (!c) return false;
  if (c->d_model < 64 || c->d_model % 64) return false;
  if (c->head_dim != 64 && c->head_dim != 128) return false;
  if (c->n_heads < 1 || c->n_kv_heads < 1 || c->n_heads % c->n_kv_heads) return false;
  {
    const int grp = c->n_heads / c->n_kv_heads;   // query heads per KV head: 1, 2, 4 or 8
    if (grp != 1 && grp != 2 && grp != 4 && grp != 8) return false;
  }
  if (c->ffn_dim < 8 || c->ffn_dim % 8) return false;
  if (c->n_layers < 1 || c->n_loops < 1 || c->n_loops > 16) return false;
  if (c->resid_bits != 2 && c->resid_bits != 4 && c->resid_bits != 16) return false;
  if (c->resid_bits != 16) {
    if (!(c->rho > 0.0 && c->rho <= 1.0)) return false;
    if (c->c_cols < 1 || c->c_cols > 4096) return false;
    if (c->group_size != 32 && c->group_size != 64 && c->group_size != 128) return false;
    if (c->group_size > c->head_dim || c->head_dim % c->group_size) return false;
    if (c->q_tile < 1) return false;
  }
  if (c->n_prelude < 0 || c->n_coda < 0 || (c->loop_embed != 0 && c->loop_embed != 1)) return false;
  if (!(c->inject_scale == c->inject_scale)) return false;   // NaN
  if (c->resid_rows < 0 || c->resid_rows > c->max_ctx) return false;
  if (c->resid_rows > 0 && c->resid_bits == 16) return false;   // a lazy-path layout
  if (c->kv_mode != 0 && c->kv_mode != 1) return false;
  if (c->kv_mode == 1 && c->resid_bits != 16) return false;   // last_loop is a dense-path KV mode
  if (c->vocab < 1 || c->max_batch < 1 || c->max_ctx < 1 || c->max_tokens < 0) return false;
  if (!(c->rms_eps > 0.f) || !(c->rope_theta > 0.f)) return false;
  return true;
}


// Walk the workspace regions; assign pointers when ctx is given.  Returns the byte total.
size_t layout(const flashloop_config& c, flashloop_ctx* x) {
  const int M = c.n_layers, K = c.n_loops, Hkv = c.n_kv_heads, H = c.n_heads, hd = c.head_dim, d = c.d_model;
  const bool lazy = c.resid_bits != 16;
  const int KS = (!lazy && c.kv_mode == 1) ? 1 : K;   // KV loops stored by the dense path (last_loop: one)
  const size_t B = c.max_batch, T = c.max_ctx;
  const int N = c.max_tokens > c.max_batch ? c.max_tokens : c.max_batch;
  const int Npad = ceil_div(N > 64 ? N : 64, 128) * 128;
  const int qkv_rows = (H + 2 * Hkv) * hd;
  const int q_tile = lazy ? c.q_tile : 128;
  const int n_tiles = (c.max_batch > ceil_div(c.max_tokens, q_tile) + c.max_batch)
                          ? c.max_batch : ceil_div(c.max_tokens, q_tile) + c.max_batch;
  const int nsel_max = lazy ? n_select(c.rho, N) : N;
  const int max_need = nsel_max < n_tiles ? nsel_max : n_tiles;
  const int cc = lazy ? c.c_cols : 1;
  size_t off = 0;
  auto take = [&](size_t bytes) -> uint8_t* {
    uint8_t* p = x ? x->ws + off : nullptr;
    off = align256(off + bytes);
    return p;
  };
  // KV cache
  const size_t rows = static_cast<size_t>(M) * 2 * B * Hkv * T;
  uint8_t *base, *codes = nullptr, *scales = nullptr;
  // residual rows per pool: every position, or (sparse storage) resid_rows
  const size_t R = (lazy && c.resid_rows > 0) ? static_cast<size_t>(c.resid_rows) : T;
  const size_t res_rows = static_cast<size_t>(M) * 2 * B * Hkv * R;
  uint8_t *ridx = nullptr, *rcount = nullptr;
  if (lazy) {
    base = take(rows * hd * 2);
    codes = take(res_rows * (K - 1) * (static_cast<size_t>(hd) * c.resid_bits / 8));
    scales = take(res_rows * (K - 1) * (hd / c.group_size) * 2);
    if (c.resid_rows > 0 && K > 1) {
      ridx = take(static_cast<size_t>(M) * (K - 1) * B * T * 4);
      rcount = take(static_cast<size_t>(M) * (K - 1) * B * 4);
    }
  } else {
    base = take(rows * KS * hd * 2);
  }
  const int X = c.n_prelude + c.n_coda;
  uint8_t* xkv = X ? take(static_cast<size_t>(X) * 2 * B * Hkv * T * hd * 2) : nullptr;
  uint8_t* rc = take(T * (hd / 2) * 4);
  uint8_t* rs = take(T * (hd / 2) * 4);
  uint8_t* seq_len = take(B * 4);
  uint8_t* status = take(16);
  uint8_t* h = take(static_cast<size_t>(N) * d * 4);
  uint8_t* h_in = take(static_cast<size_t>(N) * d * 4);
  uint8_t* h_snap = take(static_cast<size_t>(N) * d * 4);
  uint8_t* xb = take(static_cast<size_t>(Npad) * d * 2);
  uint8_t* obf = take(static_cast<size_t>(Npad) * H * hd * 2);
  uint8_t* act = take(static_cast<size_t>(Npad) * c.ffn_dim * 2);
  uint8_t* qkv = take(static_cast<size_t>(Npad) * qkv_rows * 4);
  uint8_t* q_cur = take(static_cast<size_t>(N) * H * hd * 4);
  uint8_t *o_state = nullptr, *lse = nullptr, *z_state = nullptr, *q_last = nullptr;
  if (lazy) {
    o_state = take(static_cast<size_t>(M) * N * H * hd * 4);
    lse = take(static_cast<size_t>(M) * N * H * 4);
    z_state = take(static_cast<size_t>(M) * N * H * 4);
    q_last = take(static_cast<size_t>(M) * N * H * hd * 4);
  }
  uint8_t* seq = take(N * 4);
  uint8_t* pos = take(N * 4);
  uint8_t* tile = take(N * 4);
  uint8_t* last = take(N * 4);
  uint8_t* sel_slot = take(N * 4);
  uint8_t* key = take(N * 4);
  uint8_t* keys_trace = take(static_cast<size_t>(K) * N * 4);
  uint8_t* idx_all = take(N * 4);
  uint8_t* idx_sel = take(static_cast<size_t>(K) * N * 4);
  uint8_t* idx_last = take(B * 4);
  uint8_t* has_c = take(n_tiles * 4);
  uint8_t* p_tile = take(n_tiles * 4);
  uint8_t* p_qb = take(n_tiles * 4);
  uint8_t* p_qe = take(n_tiles * 4);
  uint8_t* p_need = take(n_tiles * 4);
  uint8_t* p_counts = take(16);
  uint8_t* cols = take(static_cast<size_t>(M) * n_tiles * Hkv * cc * 4);
  uint8_t* ncols = take(static_cast<size_t>(M) * n_tiles * Hkv * 4);
  uint8_t* col_keys = take(lazy ? static_cast<size_t>(max_need) * Hkv * T * 4 : 4);
  // top-c candidates of the slices of column-key rows longer than one slice
  const int max_slices = lazy ? select_cols_slices(c.max_ctx) : 1;
  const size_t n_cand = max_slices > 1 ? static_cast<size_t>(max_need) * Hkv * max_slices * cc : 1;
  uint8_t* cand_keys = take(n_cand * 4);
  uint8_t* cand_idx = take(n_cand * 4);
  uint8_t* cand_cnt = take(static_cast<size_t>(std::max(max_need, 1)) * Hkv * 4);
  uint8_t* row_tk = take(static_cast<size_t>(std::max(max_need, 1)) * Hkv * 4);
  uint8_t* forced_on = take(16);
  uint8_t* forced_sel = take(static_cast<size_t>(K) * N * 4);
  uint8_t* forced_cols = take(static_cast<size_t>(M) * n_tiles * Hkv * cc * 4);
  uint8_t* forced_ncols = take(static_cast<size_t>(M) * n_tiles * Hkv * 4);
  const size_t fc_rows = lazy ? static_cast<size_t>(M) * (K - 1) * nsel_max * 2 * Hkv : 0;
  uint8_t* forced_codes = take(std::max<size_t>(fc_rows * hd, 16));
  uint8_t* forced_scales = take(std::max<size_t>(fc_rows * (lazy ? hd / c.group_size : 1) * 2, 16));
  uint8_t* forced_codes_on = take(16);
  // decode attention split partials
  int splits = (2 * kNumSM) / (c.max_batch * Hkv);   // decode attention: about two CTAs per SM
  const int max_splits = ceil_div(c.max_ctx, 64);
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  uint8_t* part_o = take(B * Hkv * splits * 8 * hd * 4);
  uint8_t* part_ml = take(B * Hkv * splits * 8 * 2 * 4);
  uint8_t* attn_counters = take(B * Hkv * 4);
  // correction column-split partials (the larger of the two split shapes)
  size_t cp_rows = 0;
  if (lazy) {
    const int ns_small = ceil_div(cc, kCorrColsSmall), ns_big = ceil_div(cc, kCorrColsBig);
    const size_t small_rows = static_cast<size_t>(std::min(nsel_max, kCorrSmallQueries)) * Hkv * ns_small;
    const size_t big_rows = static_cast<size_t>(nsel_max) * Hkv * ns_big;
    cp_rows = std::max(small_rows, big_rows);
  }
  uint8_t* corr_acc = take(std::max<size_t>(cp_rows, 1) * 2 * 8 * hd * 4);
  uint8_t* corr_mz = take(std::max<size_t>(cp_rows, 1) * 8 * 3 * 4);
  uint8_t* corr_counters = take(static_cast<size_t>(std::max(nsel_max, 1)) * Hkv * 4);
  uint8_t* work_ctr = take(16 * 4);   // work-item counters of the tensor-core delta-score and correction
  // GEMM split-K partials (skinny orientation only)
  size_t gp = 0;
  if (N <= 64 || c.max_batch <= 64) {
    const int n_sk = c.max_batch <= 64 ? c.max_batch : 64;
    const int bn = swap_bn(n_sk);
    const int feats[5] = {qkv_rows, d, c.ffn_dim, d, c.vocab};
    const int ks[5] = {d, H * hd, d, c.ffn_dim, d};
    const int dual[5] = {0, 0, 1, 0, 0};
    for (int o = 0; o < 5; ++o) {
      const int tiles = ceil_div(feats[o], 128);
      const size_t f = gemm_partial_floats(bn, dual[o], tiles, split_factor(tiles, ceil_div(ks[o], 64)));
      if (f > gp) gp = f;
    }
    // prefill loops >= 2 and the last-row logits may also take the skinny path with up to 64 rows
    const int feats2[5] = {qkv_rows, d, c.ffn_dim, d, c.vocab};
    for (int o = 0; o < 5; ++o) {
      const int tiles = ceil_div(feats2[o], 128);
      const size_t f = gemm_partial_floats(64, dual[o], tiles, split_factor(tiles, ceil_div(ks[o], 64)));
      if (f > gp) gp = f;
    }
  }
  uint8_t* gpart = take((gp > 0 ? gp : 1) * 4);
  uint8_t* gcnt = take(kCountersGemm * 4);
  const int ss_tiles = ceil_div(d, 128);
  uint8_t* smeta = take(static_cast<size_t>(N) * sizeof(SelMeta));
  uint8_t* ssp = take(static_cast<size_t>(ss_tiles) * kSsLd * 4);
  uint8_t* logits = take(B * c.vocab * 4);
  uint8_t* stamps = take(2 * kMaxStamps * 8);
  if (x) {
    x->lazy = lazy;
    x->qkv_rows = qkv_rows;
    x->N_max = N;
    x->N_pad = Npad;
    x->n_tiles_max = n_tiles;
    x->max_need = max_need;
    x->dec_splits = splits;
    x->cv.M = M; x->cv.K = KS; x->cv.B = c.max_batch; x->cv.Hkv = Hkv; x->cv.T = c.max_ctx; x->cv.hd = hd;
    x->cv.g = lazy ? c.group_size : hd;
    x->cv.lg = 0;
    while ((1 << x->cv.lg) < x->cv.g) ++x->cv.lg;
    x->cv.bits = lazy ? c.resid_bits : 16;
    x->cv.dense = lazy ? 0 : 1;
    x->cv.base = reinterpret_cast<uint16_t*>(base);
    x->cv.rows = ridx ? c.resid_rows : 0;
    x->cv.ridx = reinterpret_cast<int32_t*>(ridx);
    x->cv.rcount = reinterpret_cast<int*>(rcount);
    x->cvx = x->cv;
    x->cvx.rows = 0;
    x->cvx.ridx = nullptr;
    x->cvx.rcount = nullptr;
    x->cvx.M = X; x->cvx.K = 1; x->cvx.g = hd; x->cvx.lg = x->cv.lg; x->cvx.bits = 16; x->cvx.dense = 1;
    while ((1 << x->cvx.lg) < hd) ++x->cvx.lg;
    while (x->cvx.lg > 0 && (1 << x->cvx.lg) > hd) --x->cvx.lg;
    x->cvx.base = reinterpret_cast<uint16_t*>(xkv);
    x->cvx.codes = nullptr;
    x->cvx.scales = nullptr;
    x->cv.codes = codes;
    x->cv.scales = reinterpret_cast<uint16_t*>(scales);
    x->rope_cos = reinterpret_cast<float*>(rc);
    x->rope_sin = reinterpret_cast<float*>(rs);
    x->seq_len = reinterpret_cast<int*>(seq_len);
    x->status = reinterpret_cast<int*>(status);
    x->h = reinterpret_cast<float*>(h);
    x->h_in = reinterpret_cast<float*>(h_in);
    x->h_snap = reinterpret_cast<float*>(h_snap);
    x->x = reinterpret_cast<uint16_t*>(xb);
    x->obf = reinterpret_cast<uint16_t*>(obf);
    x->act = reinterpret_cast<uint16_t*>(act);
    x->qkv = reinterpret_cast<float*>(qkv);
    x->q_cur = reinterpret_cast<float*>(q_cur);
    x->o_state = reinterpret_cast<float*>(o_state);
    x->lse_state = reinterpret_cast<float*>(lse);
    x->z_state = reinterpret_cast<float*>(z_state);
    x->q_last = reinterpret_cast<float*>(q_last);
    x->seq = reinterpret_cast<int*>(seq);
    x->pos = reinterpret_cast<int*>(pos);
    x->tile = reinterpret_cast<int*>(tile);
    x->last = reinterpret_cast<int*>(last);
    x->sel_slot = reinterpret_cast<int*>(sel_slot);
    x->key = reinterpret_cast<float*>(key);
    x->keys_trace = reinterpret_cast<float*>(keys_trace);
    x->idx_all = reinterpret_cast<int32_t*>(idx_all);
    x->idx_sel = reinterpret_cast<int32_t*>(idx_sel);
    x->idx_last = reinterpret_cast<int32_t*>(idx_last);
    x->has_c = reinterpret_cast<int*>(has_c);
    x->plan.tile = reinterpret_cast<int*>(p_tile);
    x->plan.qb = reinterpret_cast<int*>(p_qb);
    x->plan.qe = reinterpret_cast<int*>(p_qe);
    x->plan.need = reinterpret_cast<int*>(p_need);
    x->plan.counts = reinterpret_cast<int*>(p_counts);
    x->cols = reinterpret_cast<int32_t*>(cols);
    x->ncols = reinterpret_cast<int*>(ncols);
    x->col_keys = reinterpret_cast<float*>(col_keys);
    x->cand_keys = reinterpret_cast<float*>(cand_keys);
    x->cand_idx = reinterpret_cast<int32_t*>(cand_idx);
    x->cand_cnt = reinterpret_cast<int*>(cand_cnt);
    x->row_tickets = reinterpret_cast<int*>(row_tk);
    x->max_slices = max_slices;
    x->forced_on = reinterpret_cast<int*>(forced_on);
    x->forced_sel = reinterpret_cast<int32_t*>(forced_sel);
    x->forced_cols = reinterpret_cast<int32_t*>(forced_cols);
    x->forced_ncols = reinterpret_cast<int*>(forced_ncols);
    x->forced_codes = reinterpret_cast<int8_t*>(forced_codes);
    x->forced_scales = reinterpret_cast<uint16_t*>(forced_scales);
    x->forced_codes_on = reinterpret_cast<int*>(forced_codes_on);
    x->nsel_max = nsel_max;
    x->part_o = reinterpret_cast<float*>(part_o);
    x->part_ml = reinterpret_cast<float*>(part_ml);
    x->attn_counters = reinterpret_cast<int*>(attn_counters);
    x->corr_acc = reinterpret_cast<float*>(corr_acc);
    x->corr_mz = reinterpret_cast<float*>(corr_mz);
    x->corr_counters = reinterpret_cast<int*>(corr_counters);
    x->work_ctr = reinterpret_cast<int*>(work_ctr);
    x->gemm_partial = reinterpret_cast<float*>(gpart);
    x->gemm_partial_cap = gp;
    x->gemm_counters = reinterpret_cast<int*>(gcnt);
    x->ss_part = reinterpret_cast<float*>(ssp);
    x->sel_meta = reinterpret_cast<SelMeta*>(smeta);
    x->ss_tiles = ss_tiles;
    x->logits_ws = reinterpret_cast<float*>(logits);
    x->stamps = reinterpret_cast<unsigned long long*>(stamps);
  }
  return off;
}

#define FL_TRY(expr)                                   \
  do {                                                 \
    cudaError_t e_ = (expr);                           \
    if (e_ != cudaSuccess) {                           \
      ctx->last_err = cudaGetErrorString(e_);          \
      return FL_ERR_CUDA;                              \
    }                                                  \
  } while (0)

enum GemmOpKind { kOpQKV, kOpO, kOpGU, kOpDown, kOpOut };

// One stack of layers' weights: the shared block, the prelude or the coda.
struct StackW {
  const CUtensorMap *qkv, *o, *gate, *up, *down;   // layer-stacked (rank-3) maps
  const float *attn_norm, *mlp_norm;               // [layers][d]
};
StackW stack_w(const flashloop_ctx* ctx, int stack) {
  if (stack == 0)
    return StackW{&ctx->tm_qkv, &ctx->tm_o, &ctx->tm_gate, &ctx->tm_up, &ctx->tm_down, ctx->w.attn_norm,
                  ctx->w.mlp_norm};
  const int x = stack - 1;
  const flashloop_layers& L = x == 0 ? ctx->w.prelude : ctx->w.coda;
  return StackW{&ctx->tm_x_qkv[x], &ctx->tm_x_o[x], &ctx->tm_x_gate[x], &ctx->tm_x_up[x], &ctx->tm_x_down[x],
                L.attn_norm, L.mlp_norm};
}

// RMSNorm of a GEMM's input rows built inside the GEMM from the fp32 hidden
// state and the per-tile sums of squares the previous residual GEMM left.
struct InNorm {
  const float* gain = nullptr;   // nullptr: the input is the bf16 buffer, loaded by TMA
  const int* idx = nullptr;      // hidden-state row of each GEMM token (nullptr: identity)
};

// Launch one GEMM of the block.  `in` (QKV, gate/up, LM head): the input
// RMSNorm runs inside the GEMM (swap orientation only).  *ss_written (O and
// down projections): whether the epilogue left the sums of squares of its
// updated rows for the next norm (the cluster split-K path only).
fl_status gemm(flashloop_ctx* ctx, const StackW& W, GemmOpKind op, int j, int n, const int* idx, cudaStream_t s,
               const InNorm& in = InNorm{}, bool* ss_written = nullptr) {
  const flashloop_config& c = ctx->cfg;
  GemmLaunch g{};
  GemmArgs& a = g.args;
  if (ss_written) *ss_written = false;
  const CUtensorMap *w0 = nullptr, *w1 = nullptr, *xa = nullptr;
  const CUtensorMap* xb = nullptr;
  int feat = 0, K = 0;
  switch (op) {
    case kOpQKV:
      w0 = W.qkv; feat = ctx->qkv_rows; K = c.d_model; xa = &ctx->tm_x_a; xb = ctx->tm_x_b;
      a.epi = kEpiStore; a.out = ctx->qkv; a.ldo = ctx->qkv_rows;
      break;
    case kOpO:
      w0 = W.o; feat = c.d_model; K = c.n_heads * c.head_dim; xa = &ctx->tm_obf_a; xb = ctx->tm_obf_b;
      a.epi = kEpiResid; a.h = ctx->h; a.idx = idx; a.scale = c.resid_scale; a.ldh = c.d_model;
      break;
    case kOpGU:
      w0 = W.gate; w1 = W.up; feat = c.ffn_dim; K = c.d_model; xa = &ctx->tm_x_a; xb = ctx->tm_x_b;
      a.epi = kEpiSwiglu; a.act = ctx->act; a.ld_act = c.ffn_dim;
      break;
    case kOpDown:
      w0 = W.down; feat = c.d_model; K = c.ffn_dim; xa = &ctx->tm_act_a; xb = ctx->tm_act_b;
      a.epi = kEpiResid; a.h = ctx->h; a.idx = idx; a.scale = c.resid_scale; a.ldh = c.d_model;
      break;
    case kOpOut:
      w0 = &ctx->tm_out; feat = c.vocab; K = c.d_model; xa = &ctx->tm_x_a; xb = ctx->tm_x_b;
      a.epi = kEpiStore; a.out = ctx->logits_ws; a.ldo = c.vocab;
      break;
  }
  a.k_chunks = ceil_div(K, 64);
  a.n_feat = feat;
  a.n_tok = n;
  a.status = ctx->status;
  if (ctx->gemm_times && ctx->stamp_slots < kMaxStamps) {
    a.stamp_start = ctx->stamps + ctx->stamp_slots;
    a.stamp_end = ctx->stamps + kMaxStamps + ctx->stamp_slots;
    ++ctx->stamp_slots;
  }
  const int w3d = op != kOpOut;
  if (n <= 64) {
    const int bn = swap_bn(n);
    const int bi = bn == 16 ? 0 : bn == 32 ? 1 : 2;
    const int tiles = ceil_div(feat, 128);
    int splits = split_factor(tiles, a.k_chunks);
    if (splits > kMaxClusterSplits) splits = kMaxClusterSplits;   // splits of a tile form one cluster
    a.cluster = 1;
    if (gemm_partial_floats(bn, w1 != nullptr, tiles, splits) > ctx->gemm_partial_cap || tiles > kCountersGemm)
      return FL_ERR_CAPACITY;
    g.a0 = w0; g.a1 = w1; g.b0 = &xb[bi]; g.b1 = nullptr;
    g.a_3d = w3d; g.b_3d = 0;
    a.a_z = j; a.b_z = 0; a.swap = 1; a.splits = splits;
    a.partial = ctx->gemm_partial; a.counters = ctx->gemm_counters;
    g.bn = bn;
    g.grid = dim3(tiles, 1, splits);
    if (ss_written && a.epi == kEpiResid && splits > 1 && ceil_div(feat, 128) <= ctx->ss_tiles) {
      a.ss_out = ctx->ss_part; a.ss_ld = kSsLd;
      *ss_written = true;
    }
    if (in.gain) {
      a.in_h = ctx->h; a.in_idx = in.idx; a.in_gain = in.gain; a.ss_in = ctx->ss_part; a.ss_ld = kSsLd;
      a.in_ld = K; a.ss_parts = ceil_div(K, 128); a.in_eps = c.rms_eps;
    }
  } else {
    if (in.gain) return FL_ERR_UNSUPPORTED;   // the caller builds the input with the norm kernel instead
    g.a0 = xa; g.a1 = nullptr; g.b0 = w0; g.b1 = w1;
    g.a_3d = 0; g.b_3d = w3d;
    a.a_z = 0; a.b_z = j; a.swap = 0; a.splits = 1;
    g.bn = 128;   // the normal orientation (the persistent kernel sizes its own grid)
  }
  g.pdl = ctx->pdl;
  FL_TRY(launch_gemm(g, s));
  return FL_OK;
}

__global__ void k_fill_last_rows(int B, int T, int32_t* rows) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) rows[b] = b * T + T - 1;
}

// Profiling brackets: an event pair around each kernel.  While the stream is
// being captured the events become event-record nodes of the graph.
cudaError_t record_event(cudaEvent_t e, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  const cudaError_t q = cudaStreamIsCapturing(s, &cs);
  if (q != cudaSuccess) return q;
  return cs == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(e, s, cudaEventRecordExternal)
                                             : cudaEventRecord(e, s);
}
cudaError_t prof_begin(flashloop_ctx* ctx, int kind, cudaStream_t s) {
  if (!ctx->prof) return cudaSuccess;
  const size_t need = static_cast<size_t>(ctx->ev_used + 1) * 2;
  while (ctx->ev.size() < need) {
    cudaEvent_t e = nullptr;
    const cudaError_t r = cudaEventCreate(&e);
    if (r != cudaSuccess) return r;
    ctx->ev.push_back(e);
  }
  if (ctx->ev_kind.size() < static_cast<size_t>(ctx->ev_used + 1)) ctx->ev_kind.resize(ctx->ev_used + 1);
  ctx->ev_kind[ctx->ev_used] = kind;
  return record_event(ctx->ev[2 * ctx->ev_used], s);
}
cudaError_t prof_end(flashloop_ctx* ctx, cudaStream_t s) {
  if (!ctx->prof) return cudaSuccess;
  const cudaError_t r = record_event(ctx->ev[2 * ctx->ev_used + 1], s);
  ++ctx->ev_used;
  return r;
}

// Launch one kernel (an expression returning cudaError_t) of a given kind.
#define FL_LAUNCH(kind, expr)                  \
  do {                                         \
    FL_TRY(prof_begin(ctx, (kind), s));        \
    FL_TRY(expr);                              \
    FL_TRY(prof_end(ctx, s));                  \
    ++ctx->launches;                           \
  } while (0)

// Launch one GEMM (an expression returning fl_status).
#define FL_GEMM(expr)                                  \
  do {                                                 \
    FL_TRY(prof_begin(ctx, FL_KIND_GEMM, s));          \
    fl_status st_g = (expr);                           \
    if (st_g != FL_OK) return st_g;                    \
    FL_TRY(prof_end(ctx, s));                          \
    ++ctx->launches;                                   \
  } while (0)

#define FL_STEP(expr)                 \
  do {                                \
    fl_status st_ = (expr);           \
    if (st_ != FL_OK) return st_;     \
  } while (0)

fl_status run_call_body(flashloop_ctx* ctx, int decode, int B, int T, cudaStream_t s);

// The whole looped block over one call's tokens, enqueued on s.  The input
// hidden states are in h_in; the result is left in h and logits_ws.  Kernels
// of the call are launched as programmatic dependents of their predecessor
// (when the option is on) so each one's launch and set-up overlap the
// previous kernel.
fl_status run_call(flashloop_ctx* ctx, int decode, int B, int T, cudaStream_t s) {
  set_pdl(ctx->pdl != 0);
  set_tc_prefill(ctx->tc_prefill != 0);
  const fl_status st = run_call_body(ctx, decode, B, T, s);
  set_pdl(false);
  return st;
}

// How the next GEMM's normed input is produced: the norm kernel, already in x
// (the selection kernel normalised it), or inside the GEMM from the sums of
// squares the previous residual GEMM left.
enum XIn { kXNorm, kXReady, kXSums };

// The call's fixed shapes, shared by every layer.
struct CallShape {
  int decode, B, T, N, n_sel, max_need, max_chunks;
  float tau;
  int col_span;   // columns a query tile can see
};

// One layer applied to `n` token rows (`idx`, or every call token): the
// attention branch (pre-norm, QKV + RoPE + KV write, dense attention or the
// sparse-column correction, O-projection with the scaled residual add) and the
// MLP branch (pre-norm, SwiGLU, down-projection with the scaled residual add).
struct LayerRef {
  StackW W;                  // weights of the layer's stack
  int z;                     // layer index within the stack
  const CacheView* cv;       // the KV cache the layer writes and reads
  const CUtensorMap* kvmap;  // that cache's rows for the decode attention
  int cj;                    // layer index within the cache
  int loop;                  // loop number of the KV write (1 for independent layers)
  bool lazy;                 // the lazy layout: base + residuals (the shared block on the lazy path)
  bool full;                 // dense attention (otherwise the correction over column sets)
  float *o_st, *l_st, *z_st, *ql;   // per-query attention state (lazy path), or nullptr
};

fl_status run_layer(flashloop_ctx* ctx, const LayerRef& L, const CallShape& cs, const int32_t* idx, int n, XIn& xs,
                    cudaStream_t s) {
  const flashloop_config& c = ctx->cfg;
  const int d = c.d_model, H = c.n_heads, Hkv = c.n_kv_heads, hd = c.head_dim;
  auto pad = [&](int m) { return m <= 64 ? swap_bn(m) : ceil_div(m, 128) * 128; };
  const float* attn_gain = L.W.attn_norm + static_cast<size_t>(L.z) * d;
  const float* mlp_gain = L.W.mlp_norm + static_cast<size_t>(L.z) * d;
  // attention branch
  InNorm attn_in;
  if (xs == kXNorm)
    FL_LAUNCH(FL_KIND_NORM, launch_rmsnorm_rows(ctx->h, idx, n, pad(n), d, attn_gain, c.rms_eps, ctx->x, s));
  if (xs == kXSums) {
    attn_in.gain = attn_gain;
    attn_in.idx = idx;
  }
  QkvPostArgs qa{};
  qa.qkv = ctx->qkv; qa.ldq = ctx->qkv_rows; qa.idx = idx; qa.n = n; qa.seq = ctx->seq; qa.pos = ctx->pos;
  qa.H = H; qa.Hkv = Hkv; qa.hd = hd; qa.rope_cos = ctx->rope_cos; qa.rope_sin = ctx->rope_sin;
  qa.cv = *L.cv; qa.j = L.cj; qa.loop = L.loop; qa.lazy = L.lazy ? 1 : 0; qa.q_cur = ctx->q_cur; qa.q_last = L.ql;
  qa.forced_on = ctx->forced_codes_on; qa.forced_codes = ctx->forced_codes;
  qa.forced_scales = ctx->forced_scales; qa.forced_ns = ctx->nsel_max;
  qa.trace_kv = ctx->trace_kv; qa.trace_ns = ctx->trace_ns;
  FL_GEMM(gemm(ctx, L.W, kOpQKV, L.z, n, idx, s, attn_in));
  FL_LAUNCH(FL_KIND_KV, launch_qkv_post(qa, s));
  if (L.full) {
    if (cs.decode) {
      AttnDecArgs aa{};
      // a full loop covers every token in order: no index indirection
      aa.q_cur = ctx->q_cur; aa.idx = idx == ctx->idx_all ? nullptr : idx; aa.seq = ctx->seq; aa.pos = ctx->pos;
      aa.cv = *L.cv;
      aa.j = L.cj; aa.loop = L.loop; aa.dense = L.lazy ? 0 : 1; aa.H = H; aa.Hkv = Hkv; aa.hd = hd; aa.tau = cs.tau;
      aa.n_splits = ctx->dec_splits;
      aa.part_o = ctx->part_o; aa.part_ml = ctx->part_ml; aa.counters = ctx->attn_counters;
      aa.o_state = L.o_st; aa.lse_state = L.l_st; aa.o_bf16 = ctx->obf; aa.status = ctx->status;
      FL_LAUNCH(FL_KIND_ATTN, launch_attn_decode(*L.kvmap, aa, n, s));
    } else {
      AttnPreArgs pa{};
      pa.q_cur = ctx->q_cur; pa.pos = ctx->pos; pa.cv = *L.cv; pa.j = L.cj; pa.loop = L.loop;
      pa.dense = L.lazy ? 0 : 1;
      pa.T = cs.T; pa.H = H; pa.Hkv = Hkv; pa.hd = hd; pa.tau = cs.tau;
      pa.o_state = L.o_st; pa.lse_state = L.l_st; pa.o_bf16 = ctx->obf; pa.status = ctx->status;
      FL_LAUNCH(FL_KIND_ATTN, launch_attn_prefill(*L.kvmap, pa, cs.B, s));
    }
  } else {
    CorrectArgs ca{};
    ca.idx = idx; ca.seq = ctx->seq; ca.pos = ctx->pos; ca.tile = ctx->tile; ca.last = ctx->last;
    ca.q_cur = ctx->q_cur; ca.q_last = L.ql; ca.o_state = L.o_st; ca.lse_state = L.l_st; ca.z_state = L.z_st;
    ca.o_bf16 = ctx->obf;
    ca.cols = ctx->cols; ca.ncols = ctx->ncols; ca.meta = ctx->sel_meta; ca.cv = *L.cv; ca.j = L.cj; ca.loop = L.loop;
    ca.H = H; ca.Hkv = Hkv;
    ca.hd = hd; ca.c = c.c_cols; ca.n_tiles = ctx->n_tiles_max; ca.tau = cs.tau; ca.status = ctx->status;
    ca.cols_per_cta = cs.n_sel <= kCorrSmallQueries ? kCorrColsSmall : kCorrColsBig;
    ca.n_splits = ceil_div(c.c_cols, ca.cols_per_cta);
    ca.part_acc = ctx->corr_acc; ca.part_mz = ctx->corr_mz; ca.counters = ctx->corr_counters;
    ca.cluster = (cs.decode && cs.n_sel <= kCorrSmallQueries && ctx->corr_cluster) ? 1 : 0;
    ca.tc = (!cs.decode && ctx->tc_prefill) ? 1 : 0;   // many queries per tile: tensor-core products
    ca.plan = ctx->plan; ca.q_tile = c.q_tile; ca.max_entries = cs.max_need;   // plan entries <= min(n_sel, tiles)
    ca.work = ctx->work_ctr + 2;
    SelColsArgs sa{};
    sa.plan = ctx->plan; sa.idx = idx; sa.pos = ctx->pos; sa.meta = ctx->sel_meta; sa.col_keys = ctx->col_keys;
    sa.max_cols = c.max_ctx; sa.Hkv = Hkv; sa.c = c.c_cols; sa.j = L.cj; sa.n_tiles = ctx->n_tiles_max;
    sa.cols = ctx->cols; sa.ncols = ctx->ncols; sa.forced_on = ctx->forced_on;
    sa.forced_cols = ctx->forced_cols; sa.forced_ncols = ctx->forced_ncols;
    sa.cand_keys = ctx->cand_keys; sa.cand_idx = ctx->cand_idx; sa.cand_counters = ctx->cand_cnt;
    sa.max_slices = ctx->max_slices;
    DScoreArgs da{};
    da.plan = ctx->plan; da.idx = idx; da.seq = ctx->seq; da.pos = ctx->pos; da.meta = ctx->sel_meta;
    da.q_cur = ctx->q_cur;
    da.q_last = L.ql; da.cv = *L.cv; da.j = L.cj; da.loop = L.loop; da.H = H; da.Hkv = Hkv; da.hd = hd;
    da.tau = cs.tau;
    da.col_keys = ctx->col_keys; da.max_cols = c.max_ctx;
    da.trace_ck = ctx->trace_ck; da.trace_tiles = ctx->trace_tiles;
    da.tc = (!cs.decode && ctx->tc_prefill) ? 1 : 0;   // many queries per tile: tensor-core products
    // rows that fit shared memory: the delta-score kernel also selects the column sets
    da.fold = cs.col_span <= kSelColsSmemKeys ? 1 : 0;
    da.sel = sa;
    da.row_tickets = ctx->row_tickets;
    da.work = ctx->work_ctr;
    // Column sets are chosen at a tile's first recomputation.  A decode call
    // that recomputes every token at every lazy loop (n_sel = N) recomputes
    // each one (its own tile) first at loop 2, so later loops have no tile to
    // score and these launches would find no work.
    const bool first_recomputations = !(cs.decode && cs.n_sel == cs.N && L.loop > 2);
    if (first_recomputations) {
      FL_LAUNCH(FL_KIND_DSCORE, launch_dscore(da, cs.max_need, cs.max_chunks, s));
      if (!da.fold) FL_LAUNCH(FL_KIND_SELECT, launch_select_cols(sa, cs.max_need, cs.col_span, s));
    }
    FL_LAUNCH(FL_KIND_CORRECT, launch_correct(ca, n, s));
  }
  bool sums = false;
  FL_GEMM(gemm(ctx, L.W, kOpO, L.z, n, idx, s, InNorm{}, &sums));
  // MLP branch
  InNorm mlp_in;
  if (sums) {
    mlp_in.gain = mlp_gain;
    mlp_in.idx = idx;
  } else {
    FL_LAUNCH(FL_KIND_NORM, launch_rmsnorm_rows(ctx->h, idx, n, pad(n), d, mlp_gain, c.rms_eps, ctx->x, s));
  }
  FL_GEMM(gemm(ctx, L.W, kOpGU, L.z, n, idx, s, mlp_in));
  FL_GEMM(gemm(ctx, L.W, kOpDown, L.z, n, idx, s, InNorm{}, &sums));
  xs = sums ? kXSums : kXNorm;
  return FL_OK;
}

// The prelude (stack 1) or coda (stack 2) layers over every call token: dense
// attention over their own one-pass KV.
fl_status run_independent(flashloop_ctx* ctx, int stack, const CallShape& cs, XIn& xs, cudaStream_t s) {
  const flashloop_config& c = ctx->cfg;
  const int count = stack == 1 ? c.n_prelude : c.n_coda;
  for (int z = 0; z < count; ++z) {
    LayerRef L{stack_w(ctx, stack), z, &ctx->cvx, &ctx->tm_kvx, stack == 1 ? z : c.n_prelude + z, 1, false, true,
               nullptr, nullptr, nullptr, nullptr};
    FL_STEP(run_layer(ctx, L, cs, ctx->idx_all, cs.N, xs, s));
  }
  return FL_OK;
}

fl_status run_call_body(flashloop_ctx* ctx, int decode, int B, int T, cudaStream_t s) {
  const flashloop_config& c = ctx->cfg;
  const int M = c.n_layers, K = c.n_loops, d = c.d_model, H = c.n_heads, hd = c.head_dim;
  const bool lazy = ctx->lazy;
  const int N = decode ? B : B * T;
  const int q_tile = lazy ? c.q_tile : 128;
  const int tiles_per_seq = decode ? 1 : ceil_div(T, q_tile);
  const int n_tiles = decode ? B : B * tiles_per_seq;
  const int n_sel = lazy ? n_select(c.rho, N) : N;
  const size_t st_o = static_cast<size_t>(ctx->N_max) * H * hd, st_l = static_cast<size_t>(ctx->N_max) * H;
  auto pad = [&](int n) { return n <= 64 ? swap_bn(n) : ceil_div(n, 128) * 128; };
  int max_len = 0;   // longest context before the call (a prefill chunk continues after it)
  for (int b = 0; b < B; ++b) max_len = std::max(max_len, ctx->lens[b]);
  const int col_span = decode ? c.max_ctx : max_len + T;   // columns a query tile can see
  CallShape cs{decode, B, T, N, n_sel, n_sel < n_tiles ? n_sel : n_tiles, ceil_div(col_span, 64),
               1.0f / std::sqrt(static_cast<float>(hd)), col_span};
  // the loop input h + e_l + gamma * x (loop embedding, input injection), x = the
  // state entering the loop stack, kept in h_in
  const bool loop_input = c.loop_embed || c.inject_scale != 0.f;

  ctx->launches = 0;
  ctx->ev_used = 0;
  ctx->stamp_slots = 0;
  // (the setup kernel also clears the GEMM launch stamps when they are on)
  FL_LAUNCH(FL_KIND_OTHER, launch_setup_call(N, decode, T, tiles_per_seq, q_tile, ctx->seq_len, ctx->seq, ctx->pos,
                                             ctx->tile, ctx->last, n_tiles, ctx->has_c,
                                             ctx->gemm_times ? ctx->stamps : nullptr, kMaxStamps, s));
  FL_TRY(cudaMemcpyAsync(ctx->h, ctx->h_in, static_cast<size_t>(N) * d * 4, cudaMemcpyDeviceToDevice, s));
  XIn carry = kXNorm;   // state at the end of the previous loop (dense loops keep their rows)
  if (c.n_prelude) {
    FL_STEP(run_independent(ctx, 1, cs, carry, s));
    // the prelude's output is the state entering the loop stack: the loop-1
    // change keys and the input injection measure from it
    FL_TRY(cudaMemcpyAsync(ctx->h_in, ctx->h, static_cast<size_t>(N) * d * 4, cudaMemcpyDeviceToDevice, s));
  }
  bool final_sums = false;
  for (int l = 1; l <= K; ++l) {
    const bool full = !lazy || l == 1;
    const int32_t* idx = ctx->idx_all;
    int n = N;
    XIn xs = (l > 1 && !lazy) ? carry : kXNorm;
    if (!full && N <= kSelectStepMax && n_tiles <= kSelectStepMax) {
      // few tokens (decode): keys, selection, snapshot and tile plan in one kernel
      int32_t* sel = ctx->idx_sel + static_cast<size_t>(l - 2) * ctx->N_max;
      SelectStepArgs sa{};
      sa.h = ctx->h; sa.h_in = ctx->h_in; sa.h_snap = ctx->h_snap; sa.sel_slot = ctx->sel_slot;
      sa.N = N; sa.d = d; sa.loop = l; sa.n_sel = n_sel; sa.key = ctx->key; sa.n_tiles = n_tiles;
      sa.seq = ctx->seq; sa.pos = ctx->pos; sa.meta = ctx->sel_meta;
      sa.keys_trace = ctx->keys_trace + static_cast<size_t>(l - 2) * ctx->N_max; sa.idx = sel;
      sa.last = ctx->last; sa.tile = ctx->tile; sa.has_c = ctx->has_c; sa.forced_on = ctx->forced_on;
      sa.forced = ctx->forced_sel + static_cast<size_t>(l - 2) * ctx->N_max; sa.plan = ctx->plan;
      sa.cv = ctx->cv; sa.B_call = B; sa.status = ctx->status;
      // first layer's norm of the few selected rows (not when the loop input changes them first)
      if (!loop_input && n_sel <= kSelectStepMaxNorm && d <= 512 * kSelectStepSlices) {
        sa.norm_gain = ctx->w.attn_norm; sa.x = ctx->x; sa.x_rows = pad(n_sel); sa.eps = c.rms_eps;
      }
      FL_LAUNCH(FL_KIND_SELECT, launch_select_step(sa, s));
      idx = sel;
      n = n_sel;
      if (sa.norm_gain) xs = kXReady;
    } else if (!full) {
      int32_t* sel = ctx->idx_sel + static_cast<size_t>(l - 2) * ctx->N_max;
      FL_TRY(cudaMemcpyAsync(ctx->keys_trace + static_cast<size_t>(l - 2) * ctx->N_max, ctx->key,
                             static_cast<size_t>(N) * 4, cudaMemcpyDeviceToDevice, s));
      FL_LAUNCH(FL_KIND_SELECT, launch_select_tokens(ctx->key, N, n_sel, sel, ctx->forced_on,
                                                     ctx->forced_sel + static_cast<size_t>(l - 2) * ctx->N_max, s));
      FL_LAUNCH(FL_KIND_SELECT, launch_after_select(sel, n_sel, N, d, ctx->sel_slot, ctx->h, ctx->h_snap, ctx->seq,
                                                    ctx->tile, ctx->last, ctx->pos, ctx->sel_meta, s));
      if (ctx->cv.rows)
        FL_LAUNCH(FL_KIND_SELECT, launch_assign_rows(ctx->cv, l, B, N / B, ctx->sel_slot, ctx->pos, ctx->status, s));
      FL_LAUNCH(FL_KIND_SELECT, launch_plan_tiles(sel, n_sel, ctx->tile, ctx->has_c, ctx->plan, s));
      idx = sel;
      n = n_sel;
    }
    if (loop_input) {
      // after the selection's snapshot: the change keys compare loop outputs
      FL_LAUNCH(FL_KIND_OTHER, launch_loop_input(ctx->h, idx == ctx->idx_all ? nullptr : idx, n, d,
                                                 c.loop_embed ? ctx->w.loop_embed + static_cast<size_t>(l - 1) * d
                                                              : nullptr,
                                                 c.inject_scale, ctx->h_in, s));
      xs = kXNorm;
    }
    for (int j = 0; j < M; ++j) {
      LayerRef L{stack_w(ctx, 0), j, &ctx->cv, &ctx->tm_kv, j, l, lazy, full,
                 lazy ? ctx->o_state + j * st_o : nullptr, lazy ? ctx->lse_state + j * st_l : nullptr,
                 lazy ? ctx->z_state + j * st_l : nullptr, lazy ? ctx->q_last + j * st_o : nullptr};
      FL_STEP(run_layer(ctx, L, cs, idx, n, xs, s));
    }
    carry = xs;
    if (lazy && l < K && !(N <= kSelectStepMax && n_tiles <= kSelectStepMax))
      FL_LAUNCH(FL_KIND_OTHER, launch_change_keys(ctx->h, l == 1 ? ctx->h_in : ctx->h_snap, ctx->sel_slot, N, d, l,
                                                  ctx->key, ctx->last, ctx->tile, ctx->has_c, s));
    // the final norm can use the last down projection's sums when it covered every output row
    final_sums = decode && l == K && full && xs == kXSums;
  }
  if (c.n_coda) {
    XIn xc = (lazy && K > 1) ? kXNorm : carry;   // after a lazy loop the sums cover the selected rows only
    FL_STEP(run_independent(ctx, 2, cs, xc, s));
    final_sums = decode && xc == kXSums;
  }
  // final norm + LM head on the output rows
  const int32_t* rows = ctx->idx_all;
  if (!decode) {
    FL_LAUNCH(FL_KIND_OTHER, launch_k(ctx->pdl, k_fill_last_rows, dim3(ceil_div(B, 128)), dim3(128), 0, s, B, T,
                                      ctx->idx_last));
    rows = ctx->idx_last;
  }
  InNorm out_in;
  if (final_sums) {
    out_in.gain = ctx->w.final_norm;
    out_in.idx = rows;
  } else {
    FL_LAUNCH(FL_KIND_NORM, launch_rmsnorm_rows(ctx->h, rows, B, pad(B), d, ctx->w.final_norm, c.rms_eps, ctx->x, s));
  }
  FL_GEMM(gemm(ctx, stack_w(ctx, 0), kOpOut, 0, B, rows, s, out_in));
  FL_LAUNCH(FL_KIND_OTHER, launch_set_lens(B, ctx->seq_len, decode ? 1 : T, s));
  return FL_OK;
}

bool build_tmaps(flashloop_ctx* ctx) {
  const flashloop_config& c = ctx->cfg;
  const flashloop_weights& w = ctx->w;
  const uint64_t M = c.n_layers, d = c.d_model, f = c.ffn_dim, hq = static_cast<uint64_t>(c.n_heads) * c.head_dim;
  bool ok = true;
  ok &= encode_tmap_bf16(&ctx->tm_qkv, w.w_qkv, d, ctx->qkv_rows, M, 128);
  ok &= encode_tmap_bf16(&ctx->tm_o, w.w_o, hq, d, M, 128);
  ok &= encode_tmap_bf16(&ctx->tm_gate, w.w_gate, d, f, M, 128);
  ok &= encode_tmap_bf16(&ctx->tm_up, w.w_up, d, f, M, 128);
  ok &= encode_tmap_bf16(&ctx->tm_down, w.w_down, f, d, M, 128);
  ok &= encode_tmap_bf16(&ctx->tm_out, w.w_out, d, c.vocab, 0, 128);
  for (int x = 0; x < 2; ++x) {   // the prelude and coda stacks
    const uint64_t L = x == 0 ? c.n_prelude : c.n_coda;
    if (L == 0) continue;
    const flashloop_layers& S = x == 0 ? w.prelude : w.coda;
    ok &= encode_tmap_bf16(&ctx->tm_x_qkv[x], S.w_qkv, d, ctx->qkv_rows, L, 128);
    ok &= encode_tmap_bf16(&ctx->tm_x_o[x], S.w_o, hq, d, L, 128);
    ok &= encode_tmap_bf16(&ctx->tm_x_gate[x], S.w_gate, d, f, L, 128);
    ok &= encode_tmap_bf16(&ctx->tm_x_up[x], S.w_up, d, f, L, 128);
    ok &= encode_tmap_bf16(&ctx->tm_x_down[x], S.w_down, f, d, L, 128);
  }
  if (ctx->cvx.M > 0)   // the independent layers' KV as [rows][hd]: [X][1][2][B][Hkv][T]
    ok &= encode_tmap_bf16(&ctx->tm_kvx, ctx->cvx.base, ctx->cvx.hd,
                           static_cast<uint64_t>(ctx->cvx.M) * 2 * ctx->cvx.B * ctx->cvx.Hkv * ctx->cvx.T, 0, 64);
  const uint64_t R = ctx->N_pad;
  ok &= encode_tmap_bf16(&ctx->tm_x_a, ctx->x, d, R, 0, 128);
  ok &= encode_tmap_bf16(&ctx->tm_obf_a, ctx->obf, hq, R, 0, 128);
  ok &= encode_tmap_bf16(&ctx->tm_act_a, ctx->act, f, R, 0, 128);
  // the cache as [rows][hd] bf16: lazy base [M][2][B][Hkv][T], dense [M][K][2][B][Hkv][T]
  const uint64_t kv_rows = static_cast<uint64_t>(ctx->cv.M) * (ctx->cv.dense ? ctx->cv.K : 1) * 2 * ctx->cv.B *
                           ctx->cv.Hkv * ctx->cv.T;
  ok &= encode_tmap_bf16(&ctx->tm_kv, ctx->cv.base, ctx->cv.hd, kv_rows, 0, 64);
  const uint32_t bns[3] = {16, 32, 64};
  for (int i = 0; i < 3; ++i) {
    ok &= encode_tmap_bf16(&ctx->tm_x_b[i], ctx->x, d, R, 0, bns[i]);
    ok &= encode_tmap_bf16(&ctx->tm_obf_b[i], ctx->obf, hq, R, 0, bns[i]);
    ok &= encode_tmap_bf16(&ctx->tm_act_b[i], ctx->act, f, R, 0, bns[i]);
  }
  return ok;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

// ============================================================================
// C ABI
// ============================================================================
extern "C" {

size_t flashloop_workspace_bytes(const flashloop_config* cfg) {
  if (!valid_config(cfg)) return 0;
  return layout(*cfg, nullptr);
}

const char* flashloop_status_string(fl_status s) {
  switch (s) {
    case FL_OK: return "ok";
    case FL_ERR_INVALID_ARG: return "invalid argument";
    case FL_ERR_CAPACITY: return "capacity exceeded";
    case FL_ERR_WORKSPACE: return "workspace too small or misaligned";
    case FL_ERR_CUDA: return "CUDA error";
    case FL_ERR_TIMEOUT: return "a kernel wait timed out";
    case FL_ERR_NONFINITE: return "non-finite value";
    case FL_ERR_UNSUPPORTED: return "unsupported configuration";
  }
  return "unknown status";
}

const char* flashloop_last_cuda_error(const flashloop_ctx* ctx) {
  return ctx ? ctx->last_err.c_str() : g_last_error.c_str();
}

fl_status flashloop_init(const flashloop_config* cfg, const flashloop_weights* w, void* workspace,
                         size_t workspace_bytes, fl_stream_t stream, flashloop_ctx** out) {
  if (!out) return FL_ERR_INVALID_ARG;
  *out = nullptr;
  if (!valid_config(cfg) || !w) return FL_ERR_INVALID_ARG;

  const void* wp[9] = {w->attn_norm, w->w_qkv, w->w_o, w->mlp_norm, w->w_gate, w->w_up, w->w_down, w->final_norm,
                       w->w_out};
  for (const void* p : wp)
    if (!p || !aligned16(p)) return FL_ERR_INVALID_ARG;
  for (int x = 0; x < 2; ++x) {
    if ((x == 0 ? cfg->n_prelude : cfg->n_coda) == 0) continue;
    const flashloop_layers& S = x == 0 ? w->prelude : w->coda;
    const void* sp[7] = {S.attn_norm, S.w_qkv, S.w_o, S.mlp_norm, S.w_gate, S.w_up, S.w_down};
    for (const void* p : sp)
      if (!p || !aligned16(p)) return FL_ERR_INVALID_ARG;
  }
  if (cfg->loop_embed && (!w->loop_embed || !aligned16(w->loop_embed))) return FL_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255)) return FL_ERR_WORKSPACE;
  const size_t need = layout(*cfg, nullptr);
  if (workspace_bytes < need) return FL_ERR_WORKSPACE;
  flashloop_ctx* ctx = new (std::nothrow) flashloop_ctx();
  if (!ctx) return FL_ERR_CUDA;
  ctx->cfg = *cfg;
  ctx->w = *w;
  ctx->ws = static_cast<uint8_t*>(workspace);
  ctx->ws_bytes = workspace_bytes;
  cudaGetDevice(&ctx->device);
  layout(*cfg, ctx);
  ctx->lens.assign(cfg->max_batch, 0);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  auto fail = [&](fl_status st) {
    if (st == FL_ERR_CUDA && ctx->last_err.empty()) ctx->last_err = cudaGetErrorString(cudaGetLastError());
    g_last_error = ctx->last_err;
    delete ctx;
    return st;
  };
  {
    cudaError_t e = gemm_init_attrs();
    if (e == cudaSuccess) e = kernels_init_attrs();
    if (e != cudaSuccess) {
      ctx->last_err = cudaGetErrorString(e);
      return fail(FL_ERR_CUDA);
    }
  }

  if (!build_tmaps(ctx)) return fail(FL_ERR_CUDA);
  if (cudaMemsetAsync(ctx->ws, 0, need, s) != cudaSuccess) return fail(FL_ERR_CUDA);
  if (ctx->cv.rows &&   // sparse residual storage: no position holds a residual row yet
      cudaMemsetAsync(ctx->cv.ridx, 0xFF,
                      static_cast<size_t>(cfg->n_layers) * (cfg->n_loops - 1) * cfg->max_batch * cfg->max_ctx * 4,
                      s) != cudaSuccess)
    return fail(FL_ERR_CUDA);
  // RoPE table: angle = pos * theta^(-2i/hd), computed in double, stored fp32
  const int half = cfg->head_dim / 2;
  std::vector<float> rc(static_cast<size_t>(cfg->max_ctx) * half), rs(rc.size());
  for (int t = 0; t < cfg->max_ctx; ++t)
    for (int i = 0; i < half; ++i) {
      const double inv = std::pow(static_cast<double>(cfg->rope_theta), -2.0 * i / cfg->head_dim);
      const double a = static_cast<double>(t) * inv;
      rc[static_cast<size_t>(t) * half + i] = static_cast<float>(std::cos(a));
      rs[static_cast<size_t>(t) * half + i] = static_cast<float>(std::sin(a));
    }
  if (cudaMemcpyAsync(ctx->rope_cos, rc.data(), rc.size() * 4, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(ctx->rope_sin, rs.data(), rs.size() * 4, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return fail(FL_ERR_CUDA);
  std::vector<int32_t> ident(ctx->N_max);
  for (int i = 0; i < ctx->N_max; ++i) ident[i] = i;
  if (cudaMemcpyAsync(ctx->idx_all, ident.data(), ident.size() * 4, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return fail(FL_ERR_CUDA);
  if (cudaStreamSynchronize(s) != cudaSuccess) return fail(FL_ERR_CUDA);
  *out = ctx;
  return FL_OK;
}

void flashloop_destroy(flashloop_ctx* ctx) {
  if (!ctx) return;
  for (cudaGraphExec_t e : ctx->graph_exec)
    if (e) cudaGraphExecDestroy(e);
  for (cudaEvent_t e : ctx->ev)
    if (e) cudaEventDestroy(e);
  delete ctx;
}

fl_status flashloop_set_option(flashloop_ctx* ctx, fl_option opt, int value) {
  if (!ctx) return FL_ERR_INVALID_ARG;
  if (opt == FL_OPT_USE_GRAPH) {
    ctx->use_graph = value ? 1 : 0;
    return FL_OK;
  }
  if (opt == FL_OPT_PROFILE) {
    ctx->prof = value ? 1 : 0;
    return FL_OK;
  }
  if (opt == FL_OPT_PDL) {
    ctx->pdl = value ? 1 : 0;
    return FL_OK;
  }
  if (opt == FL_OPT_GEMM_TIMES) {
    ctx->gemm_times = value ? 1 : 0;
    return FL_OK;
  }
  if (opt == FL_OPT_TC_PREFILL) {
    ctx->tc_prefill = value ? 1 : 0;
    return FL_OK;
  }
  if (opt == FL_OPT_CORR_CLUSTER) {
    ctx->corr_cluster = value ? 1 : 0;
    return FL_OK;
  }
  return FL_ERR_INVALID_ARG;
}

fl_status flashloop_prefill(flashloop_ctx* ctx, const float* h0, int B, int T, float* h_out, float* logits_last,
                            fl_stream_t stream) {
  if (!ctx || !h0 || B < 1 || T < 1) return FL_ERR_INVALID_ARG;
  const flashloop_config& c = ctx->cfg;
  if (B > c.max_batch || static_cast<long long>(B) * T > c.max_tokens || T > c.max_ctx) return FL_ERR_CAPACITY;
  for (int b = 0; b < B; ++b)
    if (ctx->lens[b] + T > c.max_ctx) return FL_ERR_CAPACITY;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t bytes = static_cast<size_t>(B) * T * c.d_model * 4;
  FL_TRY(cudaMemcpyAsync(ctx->h_in, h0, bytes, cudaMemcpyDefault, s));
  FL_STEP(run_call(ctx, 0, B, T, s));
  if (h_out) FL_TRY(cudaMemcpyAsync(h_out, ctx->h, bytes, cudaMemcpyDefault, s));
  if (logits_last)
    FL_TRY(cudaMemcpyAsync(logits_last, ctx->logits_ws, static_cast<size_t>(B) * c.vocab * 4, cudaMemcpyDefault, s));
  for (int b = 0; b < B; ++b) ctx->lens[b] += T;
  ctx->last_N = B * T;
  ctx->last_nsel = ctx->lazy ? n_select(c.rho, B * T) : B * T;
  ctx->last_decode = 0;
  ctx->last_tiles = B * ceil_div(T, ctx->lazy ? c.q_tile : 128);
  return FL_OK;
}

fl_status flashloop_decode_step(flashloop_ctx* ctx, const float* h0, int B, float* h_out, float* logits,
                                fl_stream_t stream) {
  if (!ctx || !h0 || B < 1) return FL_ERR_INVALID_ARG;
  const flashloop_config& c = ctx->cfg;
  if (B > c.max_batch) return FL_ERR_CAPACITY;
  for (int b = 0; b < B; ++b)
    if (ctx->lens[b] + 1 > c.max_ctx) return FL_ERR_CAPACITY;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FL_TRY(cudaMemcpyAsync(ctx->h_in, h0, static_cast<size_t>(B) * c.d_model * 4, cudaMemcpyDefault, s));
  // A decode step's launch sequence depends on B only; after one direct run it
  // is captured once into a CUDA graph and replayed (not on the legacy stream).
  const int gkey = B * 128 + (ctx->prof ? 1 : 0) + (ctx->pdl ? 2 : 0) + (ctx->gemm_times ? 8 : 0) +
                   (ctx->corr_cluster ? 16 : 0) + (ctx->tc_prefill ? 64 : 0);
  size_t gi = 0;
  while (gi < ctx->graph_b.size() && ctx->graph_b[gi] != gkey) ++gi;
  bool seen = false;
  for (int v : ctx->eager_seen) seen |= (v == gkey);
  if (ctx->use_graph && s != nullptr && seen) {
    if (gi == ctx->graph_b.size()) {
      cudaGraph_t graph = nullptr;
      FL_TRY(cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal));
      fl_status st = run_call(ctx, 1, B, 0, s);
      cudaError_t e = cudaStreamEndCapture(s, &graph);
      if (st != FL_OK) {
        if (graph) cudaGraphDestroy(graph);
        return st;
      }
      FL_TRY(e);
      cudaGraphExec_t exec = nullptr;
      e = cudaGraphInstantiate(&exec, graph, 0);
      cudaGraphDestroy(graph);
      FL_TRY(e);
      ctx->graph_b.push_back(gkey);
      ctx->graph_exec.push_back(exec);
    }
    FL_TRY(cudaGraphLaunch(ctx->graph_exec[gi], s));
  } else {
    FL_STEP(run_call(ctx, 1, B, 0, s));
    if (!seen) ctx->eager_seen.push_back(gkey);
  }
  if (h_out) FL_TRY(cudaMemcpyAsync(h_out, ctx->h, static_cast<size_t>(B) * c.d_model * 4, cudaMemcpyDefault, s));
  if (logits)
    FL_TRY(cudaMemcpyAsync(logits, ctx->logits_ws, static_cast<size_t>(B) * c.vocab * 4, cudaMemcpyDefault, s));
  for (int b = 0; b < B; ++b) ctx->lens[b] += 1;
  ctx->last_N = B;
  ctx->last_nsel = ctx->lazy ? n_select(c.rho, B) : B;
  ctx->last_decode = 1;
  ctx->last_tiles = B;
  return FL_OK;
}

fl_status flashloop_kv_bytes_for(const flashloop_config* cfg, size_t* total, double* per_token_per_layer,
                                 double* dense_per_token_per_layer) {
  if (!valid_config(cfg)) return FL_ERR_INVALID_ARG;
  const flashloop_config& c = *cfg;
  const double hd = c.head_dim, kv = 2.0 * c.n_kv_heads;
  const double dense = kv * c.n_loops * hd * 2.0;
  double per = c.kv_mode == 1 ? kv * hd * 2.0 : dense;   // last_loop keeps one pass of KV
  if (c.resid_bits != 16) {
    // the bf16 base, plus K-1 residual rows (packed codes and fp16 scales) per
    // position, or with sparse storage resid_rows per pool and a 4-byte row index
    const double row = hd * c.resid_bits / 8.0 + (hd / c.group_size) * 2.0;
    per = kv * hd * 2.0;
    if (c.resid_rows > 0)
      per += (c.n_loops - 1) * (kv * row * static_cast<double>(c.resid_rows) / c.max_ctx + 4.0);
    else
      per += (c.n_loops - 1) * kv * row;
  }
  if (per_token_per_layer) *per_token_per_layer = per;
  if (dense_per_token_per_layer) *dense_per_token_per_layer = dense;
  // the looped layers' cache plus one pass of KV for each prelude / coda layer
  const double extra = (c.n_prelude + c.n_coda) * kv * hd * 2.0;
  if (total)
    *total = static_cast<size_t>((per * c.n_layers + extra) * c.max_batch * static_cast<double>(c.max_ctx));
  return FL_OK;
}

fl_status flashloop_kv_bytes(const flashloop_ctx* ctx, size_t* total, double* per_token_per_layer,
                             double* dense_per_token_per_layer) {
  if (!ctx) return FL_ERR_INVALID_ARG;
  return flashloop_kv_bytes_for(&ctx->cfg, total, per_token_per_layer, dense_per_token_per_layer);
}

fl_status flashloop_reset(flashloop_ctx* ctx, const int* seq_len, fl_stream_t stream) {
  if (!ctx) return FL_ERR_INVALID_ARG;
  const int B = ctx->cfg.max_batch;
  std::vector<int> v(B, 0);
  if (seq_len)
    for (int b = 0; b < B; ++b) {
      if (seq_len[b] < 0 || seq_len[b] > ctx->cfg.max_ctx) return FL_ERR_CAPACITY;
      v[b] = seq_len[b];
    }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (B <= kLensByValue) {
    LensArg a{};
    a.n = B;
    for (int b = 0; b < B; ++b) a.v[b] = v[b];
    FL_TRY(launch_reset_lens(a, ctx->seq_len, s));
  } else {
    FL_TRY(cudaMemcpyAsync(ctx->seq_len, v.data(), B * 4, cudaMemcpyHostToDevice, s));
    FL_TRY(cudaStreamSynchronize(s));
  }
  // sparse residual storage: the pools keep the rows of the positions below the new lengths
  if (ctx->cv.rows) FL_TRY(launch_reset_rows(ctx->cv, ctx->seq_len, s));
  ctx->lens = v;
  return FL_OK;
}

fl_status flashloop_profile(flashloop_ctx* ctx, fl_stream_t stream, float* ms, int* launches) {
  if (!ctx || !ms || !launches) return FL_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FL_TRY(cudaStreamSynchronize(s));
  for (int k = 0; k < FL_NUM_KINDS; ++k) {
    ms[k] = 0.f;
    launches[k] = 0;
  }
  for (int i = 0; i < ctx->ev_used; ++i) {
    float t = 0.f;
    FL_TRY(cudaEventElapsedTime(&t, ctx->ev[2 * i], ctx->ev[2 * i + 1]));
    ms[ctx->ev_kind[i]] += t;
    launches[ctx->ev_kind[i]] += 1;
  }
  return FL_OK;
}

int flashloop_kernels_per_call(const flashloop_ctx* ctx) { return ctx ? ctx->launches : 0; }

fl_status flashloop_gemm_times(flashloop_ctx* ctx, fl_stream_t stream, double* total_ms, int* launches) {
  if (!ctx || !total_ms || !launches) return FL_ERR_INVALID_ARG;
  *total_ms = 0.0;
  *launches = 0;
  if (!ctx->gemm_times) return FL_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FL_TRY(cudaStreamSynchronize(s));
  const int n = ctx->stamp_slots;
  std::vector<unsigned long long> st(n), en(n);
  if (n) {
    FL_TRY(cudaMemcpy(st.data(), ctx->stamps, static_cast<size_t>(n) * 8, cudaMemcpyDeviceToHost));
    FL_TRY(cudaMemcpy(en.data(), ctx->stamps + kMaxStamps, static_cast<size_t>(n) * 8, cudaMemcpyDeviceToHost));
  }
  double sum = 0.0;
  for (int i = 0; i < n; ++i)
    if (en[i] > st[i] && st[i] != ~0ULL) sum += static_cast<double>(en[i] - st[i]);
  *total_ms = sum * 1e-6;
  *launches = n;
  return FL_OK;
}

fl_status flashloop_sync_status(flashloop_ctx* ctx, fl_stream_t stream) {
  if (!ctx) return FL_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FL_TRY(cudaStreamSynchronize(s));
  int st = 0;
  FL_TRY(cudaMemcpy(&st, ctx->status, 4, cudaMemcpyDeviceToHost));
  if (st) {
    const int zero = 0;
    FL_TRY(cudaMemcpy(ctx->status, &zero, 4, cudaMemcpyHostToDevice));
  }
  if (st & kErrWaitTimeout) return FL_ERR_TIMEOUT;
  if (st & kErrCapacity) return FL_ERR_CAPACITY;
  if (st) return FL_ERR_NONFINITE;
  return FL_OK;
}

fl_status flashloop_import_lazy(flashloop_ctx* ctx, int layer, int seq, int n, const uint16_t* base_k,
                                const uint16_t* base_v, const int8_t* codes_k, const int8_t* codes_v,
                                const uint16_t* scales_k, const uint16_t* scales_v, fl_stream_t stream) {
  if (!ctx || !ctx->lazy) return FL_ERR_INVALID_ARG;
  const flashloop_config& c = ctx->cfg;
  if (layer < 0 || layer >= c.n_layers || seq < 0 || seq >= c.max_batch || n < 0 || n > c.max_ctx)
    return FL_ERR_INVALID_ARG;
  if (!base_k || !base_v || (c.n_loops > 1 && (!codes_k || !codes_v || !scales_k || !scales_v)))
    return FL_ERR_INVALID_ARG;
  if (n == 0) return FL_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int Hkv = c.n_kv_heads, hd = c.head_dim, ns = hd / c.group_size;
  const CacheView& cv = ctx->cv;
  if (cv.rows) {   // sparse residual storage: rows for the positions that hold a residual
    for (int kv = 0; kv < 2; ++kv)
      for (int h = 0; h < Hkv; ++h)
        FL_TRY(cudaMemcpyAsync(cv.base_row(layer, kv, seq, h, 0), (kv ? base_v : base_k) + static_cast<size_t>(h) * n * hd,
                               static_cast<size_t>(n) * hd * 2, cudaMemcpyDefault, s));
    if (c.n_loops > 1)
      FL_TRY(launch_import_rows(cv, layer, seq, n, codes_k, codes_v, scales_k, scales_v, ctx->status, s));
    return FL_OK;
  }
  for (int kv = 0; kv < 2; ++kv) {
    const uint16_t* base = kv ? base_v : base_k;
    for (int h = 0; h < Hkv; ++h)
      FL_TRY(cudaMemcpyAsync(cv.base_row(layer, kv, seq, h, 0), base + static_cast<size_t>(h) * n * hd,
                             static_cast<size_t>(n) * hd * 2, cudaMemcpyDefault, s));
    const int8_t* codes = kv ? codes_v : codes_k;
    const uint16_t* scales = kv ? scales_v : scales_k;
    for (int l = 2; l <= c.n_loops; ++l)
      for (int h = 0; h < Hkv; ++h) {
        const size_t src = (static_cast<size_t>(l - 2) * Hkv + h) * n;
        FL_TRY(launch_pack_codes(codes + src * hd, n, hd, c.resid_bits, cv.code_row(layer, l, kv, seq, h, 0),
                                 cv.row_bytes_codes(), s));
        FL_TRY(cudaMemcpyAsync(cv.scale_row(layer, l, kv, seq, h, 0), scales + src * ns,
                               static_cast<size_t>(n) * ns * 2, cudaMemcpyDefault, s));
      }
  }
  return FL_OK;
}

fl_status flashloop_import_dense(flashloop_ctx* ctx, int layer, int seq, int n, const uint16_t* kv_k,
                                 const uint16_t* kv_v, fl_stream_t stream) {
  if (!ctx || ctx->lazy) return FL_ERR_INVALID_ARG;
  const flashloop_config& c = ctx->cfg;
  if (layer < 0 || layer >= c.n_layers || seq < 0 || seq >= c.max_batch || n < 0 || n > c.max_ctx || !kv_k || !kv_v)
    return FL_ERR_INVALID_ARG;
  if (n == 0) return FL_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int Hkv = c.n_kv_heads, hd = c.head_dim;
  for (int kv = 0; kv < 2; ++kv) {
    const uint16_t* src = kv ? kv_v : kv_k;
    for (int l = 1; l <= ctx->cv.K; ++l)   // the stored loops (one in last_loop mode)
      for (int h = 0; h < Hkv; ++h)
        FL_TRY(cudaMemcpyAsync(ctx->cv.dense_row(layer, l, kv, seq, h, 0),
                               src + (static_cast<size_t>(l - 1) * Hkv + h) * n * hd, static_cast<size_t>(n) * hd * 2,
                               cudaMemcpyDefault, s));
  }
  return FL_OK;
}

fl_status flashloop_import_extra(flashloop_ctx* ctx, int x, int seq, int n, const uint16_t* kv_k,
                                 const uint16_t* kv_v, fl_stream_t stream) {
  if (!ctx || !kv_k || !kv_v) return FL_ERR_INVALID_ARG;
  const flashloop_config& c = ctx->cfg;
  if (x < 0 || x >= c.n_prelude + c.n_coda || seq < 0 || seq >= c.max_batch || n < 0 || n > c.max_ctx)
    return FL_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int Hkv = c.n_kv_heads, hd = c.head_dim;
  for (int kv = 0; kv < 2 && n > 0; ++kv)
    for (int h = 0; h < Hkv; ++h)
      FL_TRY(cudaMemcpyAsync(ctx->cvx.dense_row(x, 1, kv, seq, h, 0), (kv ? kv_v : kv_k) + static_cast<size_t>(h) * n * hd,
                             static_cast<size_t>(n) * hd * 2, cudaMemcpyDefault, s));
  return FL_OK;
}

fl_status flashloop_export_slice(const flashloop_ctx* ctx, int layer, int loop, int seq, int which, int n,
                                 void* codes, void* scales, fl_stream_t stream) {
  if (!ctx || !codes) return FL_ERR_INVALID_ARG;
  const flashloop_config& c = ctx->cfg;
  if (layer < 0 || layer >= c.n_layers || loop < 1 || loop > c.n_loops || seq < 0 || seq >= c.max_batch || n < 0 ||
      n > c.max_ctx || (which != 0 && which != 1))
    return FL_ERR_INVALID_ARG;
  flashloop_ctx* mctx = const_cast<flashloop_ctx*>(ctx);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int Hkv = c.n_kv_heads, hd = c.head_dim;
  const CacheView& cv = ctx->cv;
  if (!ctx->lazy || loop == 1) {
    for (int h = 0; h < Hkv; ++h) {
      const uint16_t* src = ctx->lazy ? cv.base_row(layer, which, seq, h, 0) : cv.dense_row(layer, loop, which, seq, h, 0);
      if (cudaMemcpyAsync(static_cast<uint16_t*>(codes) + static_cast<size_t>(h) * n * hd, src,
                          static_cast<size_t>(n) * hd * 2, cudaMemcpyDefault, s) != cudaSuccess) {
        mctx->last_err = "export copy failed";
        return FL_ERR_CUDA;
      }
    }
    return FL_OK;
  }
  if (!scales) return FL_ERR_INVALID_ARG;
  if (cv.rows) {   // sparse residual storage: gathered by position, zero where no row is kept
    if (n > 0 && launch_export_rows(cv, layer, loop, which, seq, n, static_cast<uint8_t*>(codes),
                                    static_cast<uint16_t*>(scales), s) != cudaSuccess) {
      mctx->last_err = "export gather failed";
      return FL_ERR_CUDA;
    }
    return FL_OK;
  }
  const size_t rb = cv.row_bytes_codes();
  const int ns = hd / c.group_size;
  for (int h = 0; h < Hkv; ++h) {
    if (cudaMemcpyAsync(static_cast<uint8_t*>(codes) + static_cast<size_t>(h) * n * rb,
                        cv.code_row(layer, loop, which, seq, h, 0), static_cast<size_t>(n) * rb, cudaMemcpyDefault,
                        s) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<uint16_t*>(scales) + static_cast<size_t>(h) * n * ns,
                        cv.scale_row(layer, loop, which, seq, h, 0), static_cast<size_t>(n) * ns * 2,
                        cudaMemcpyDefault, s) != cudaSuccess) {
      mctx->last_err = "export copy failed";
      return FL_ERR_CUDA;
    }
  }
  return FL_OK;
}

fl_status flashloop_force_selection(flashloop_ctx* ctx, const int32_t* sel, int n_sel_loops, int n_sel,
                                    const int32_t* cols, const int32_t* ncols, int n_tiles) {
  if (!ctx || !ctx->lazy) return FL_ERR_INVALID_ARG;
  const flashloop_config& c = ctx->cfg;
  if ((cols == nullptr) != (ncols == nullptr)) return FL_ERR_INVALID_ARG;
  const int on = (sel ? kForceSel : 0) | (cols ? kForceCols : 0);
  if ((on & kForceSel) && (n_sel_loops != c.n_loops - 1 || n_sel < 1 || n_sel > ctx->N_max))
    return FL_ERR_INVALID_ARG;
  if ((on & kForceCols) && (n_tiles < 1 || n_tiles > ctx->n_tiles_max)) return FL_ERR_INVALID_ARG;
  if (on & kForceSel)
    for (int l = 0; l < n_sel_loops; ++l)
      FL_TRY(cudaMemcpy(ctx->forced_sel + static_cast<size_t>(l) * ctx->N_max, sel + static_cast<size_t>(l) * n_sel,
                        static_cast<size_t>(n_sel) * 4, cudaMemcpyHostToDevice));
  if (on & kForceCols) {
    const size_t per_tile = static_cast<size_t>(c.n_kv_heads) * c.c_cols;
    for (int j = 0; j < c.n_layers; ++j) {
      FL_TRY(cudaMemcpy(ctx->forced_cols + static_cast<size_t>(j) * ctx->n_tiles_max * per_tile,
                        cols + static_cast<size_t>(j) * n_tiles * per_tile, n_tiles * per_tile * 4,
                        cudaMemcpyHostToDevice));
      FL_TRY(cudaMemcpy(ctx->forced_ncols + static_cast<size_t>(j) * ctx->n_tiles_max * c.n_kv_heads,
                        ncols + static_cast<size_t>(j) * n_tiles * c.n_kv_heads,
                        static_cast<size_t>(n_tiles) * c.n_kv_heads * 4, cudaMemcpyHostToDevice));
    }
  }
  FL_TRY(cudaMemcpy(ctx->forced_on, &on, 4, cudaMemcpyHostToDevice));
  return FL_OK;
}

fl_status flashloop_force_codes(flashloop_ctx* ctx, const int8_t* codes, const uint16_t* scales, int n_sel) {
  if (!ctx || !ctx->lazy) return FL_ERR_INVALID_ARG;
  const flashloop_config& c = ctx->cfg;
  const int on = (codes && scales) ? 1 : 0;
  if (on) {
    if (n_sel < 1 || n_sel > ctx->nsel_max || c.n_loops < 2) return FL_ERR_INVALID_ARG;
    const size_t per = static_cast<size_t>(2) * c.n_kv_heads;   // rows per selection slot
    const size_t ns_code = c.head_dim, ns_scale = c.head_dim / c.group_size;
    for (int jl = 0; jl < c.n_layers * (c.n_loops - 1); ++jl) {
      FL_TRY(cudaMemcpy(ctx->forced_codes + static_cast<size_t>(jl) * ctx->nsel_max * per * ns_code,
                        codes + static_cast<size_t>(jl) * n_sel * per * ns_code, n_sel * per * ns_code,
                        cudaMemcpyHostToDevice));
      FL_TRY(cudaMemcpy(ctx->forced_scales + static_cast<size_t>(jl) * ctx->nsel_max * per * ns_scale,
                        scales + static_cast<size_t>(jl) * n_sel * per * ns_scale, n_sel * per * ns_scale * 2,
                        cudaMemcpyHostToDevice));
    }
  }
  FL_TRY(cudaMemcpy(ctx->forced_codes_on, &on, 4, cudaMemcpyHostToDevice));
  return FL_OK;
}

fl_status flashloop_set_trace(flashloop_ctx* ctx, float* kv_rows, int n_slots, float* col_keys, int n_tiles) {
  if (!ctx || !ctx->lazy) return FL_ERR_INVALID_ARG;
  if ((kv_rows && n_slots < 1) || (col_keys && n_tiles < 1)) return FL_ERR_INVALID_ARG;
  if ((kv_rows && !aligned16(kv_rows)) || (col_keys && !aligned16(col_keys))) return FL_ERR_INVALID_ARG;
  ctx->trace_kv = kv_rows;
  ctx->trace_ns = kv_rows ? n_slots : 0;
  ctx->trace_ck = col_keys;
  ctx->trace_tiles = col_keys ? n_tiles : 0;
  // captured decode graphs hold the old pointers: capture again
  for (cudaGraphExec_t e : ctx->graph_exec)
    if (e) cudaGraphExecDestroy(e);
  ctx->graph_exec.clear();
  ctx->graph_b.clear();
  return FL_OK;
}

fl_status flashloop_read_trace(flashloop_ctx* ctx, int32_t* sel, float* keys, int32_t* cols, int32_t* ncols,
                               fl_stream_t stream) {
  if (!ctx || !ctx->lazy) return FL_ERR_INVALID_ARG;
  const flashloop_config& c = ctx->cfg;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FL_TRY(cudaStreamSynchronize(s));
  const int L = c.n_loops - 1, n_sel = ctx->last_nsel, N = ctx->last_N, nt = ctx->last_tiles;
  for (int l = 0; l < L; ++l) {
    if (sel)
      FL_TRY(cudaMemcpy(sel + static_cast<size_t>(l) * n_sel, ctx->idx_sel + static_cast<size_t>(l) * ctx->N_max,
                        static_cast<size_t>(n_sel) * 4, cudaMemcpyDeviceToHost));
    if (keys)
      FL_TRY(cudaMemcpy(keys + static_cast<size_t>(l) * N, ctx->keys_trace + static_cast<size_t>(l) * ctx->N_max,
                        static_cast<size_t>(N) * 4, cudaMemcpyDeviceToHost));
  }
  const size_t per_tile = static_cast<size_t>(c.n_kv_heads) * c.c_cols;
  for (int j = 0; j < c.n_layers; ++j) {
    if (cols)
      FL_TRY(cudaMemcpy(cols + static_cast<size_t>(j) * nt * per_tile,
                        ctx->cols + static_cast<size_t>(j) * ctx->n_tiles_max * per_tile, nt * per_tile * 4,
                        cudaMemcpyDeviceToHost));
    if (ncols)
      FL_TRY(cudaMemcpy(ncols + static_cast<size_t>(j) * nt * c.n_kv_heads,
                        ctx->ncols + static_cast<size_t>(j) * ctx->n_tiles_max * c.n_kv_heads,
                        static_cast<size_t>(nt) * c.n_kv_heads * 4, cudaMemcpyDeviceToHost));
  }
  return FL_OK;
}

// ---------------------------------------------------------------- unit entry points
static fl_status record(cudaError_t e) {
  if (e == cudaSuccess) return FL_OK;
  g_last_error = cudaGetErrorString(e);
  return FL_ERR_CUDA;
}

fl_status fl_test_topk(const float* keys, int n_seg, int n, int k, int32_t* idx, fl_stream_t stream) {
  if (!keys || !idx || n_seg < 0 || n < 0 || k < 0) return FL_ERR_INVALID_ARG;
  if (n_seg == 0 || n == 0 || k == 0) return FL_OK;
  const cudaError_t e = kernels_init_attrs();   // shared-memory opt-ins, once
  if (e != cudaSuccess) return record(e);
  return record(launch_topk(keys, n_seg, n, k, idx, reinterpret_cast<cudaStream_t>(stream)));
}

namespace {
// the checks and the launch shared by the two quantiser entry points
fl_status quantize_entry(const float* x, const uint16_t* prev, int rows, int width, int g, int bits, uint8_t* codes,
                         uint16_t* scales, fl_stream_t stream) {
  if (!x || !codes || !scales || rows < 0 || width <= 0) return FL_ERR_INVALID_ARG;
  if (bits != 2 && bits != 4) return FL_ERR_INVALID_ARG;
  if (g != 32 && g != 64 && g != 128) return FL_ERR_INVALID_ARG;
  if (width % g) return FL_ERR_INVALID_ARG;
  if (width % 128 != 0 && width != 64) return FL_ERR_INVALID_ARG;
  if (width == 64 && g > 64) return FL_ERR_INVALID_ARG;
  if (!aligned16(x)) return FL_ERR_INVALID_ARG;   // rows are read as 16- or 8-byte vectors
  if (prev && !aligned16(prev)) return FL_ERR_INVALID_ARG;
  if (static_cast<long long>(rows) * (width / 64) >= (1LL << 31)) return FL_ERR_CAPACITY;
  if (rows == 0) return FL_OK;
  return record(
      launch_quantize_rows(x, prev, rows, width, g, bits, codes, scales, reinterpret_cast<cudaStream_t>(stream)));
}
}  // namespace

fl_status fl_test_quantize(const float* r, int rows, int width, int g, int bits, uint8_t* codes, uint16_t* scales,
                           fl_stream_t stream) {
  return quantize_entry(r, nullptr, rows, width, g, bits, codes, scales, stream);
}

fl_status fl_test_quantize_residual(const float* x, const uint16_t* prev, int rows, int width, int g, int bits,
                                    uint8_t* codes, uint16_t* scales, fl_stream_t stream) {
  if (!prev) return FL_ERR_INVALID_ARG;
  return quantize_entry(x, prev, rows, width, g, bits, codes, scales, stream);
}

size_t fl_test_gemm_scratch_bytes(int m, int n, int k, int swap_ab) {
  if (!swap_ab || m < 1 || m > 64 || n < 1 || k < 1) return 0;
  const int tiles = ceil_div(n, 128);
  const int splits = split_factor(tiles, ceil_div(k, 64));
  return gemm_partial_floats(swap_bn(m), 0, tiles, splits) * 4 + static_cast<size_t>(tiles) * 4 + 256;
}

fl_status fl_test_gemm(const uint16_t* A, const uint16_t* B, float* D, int m, int n, int k, int swap_ab,
                       void* scratch, size_t scratch_bytes, fl_stream_t stream) {
  if (!A || !B || !D || m < 1 || n < 1 || k < 8 || k % 8) return FL_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(B) || !aligned16(D)) return FL_ERR_INVALID_ARG;
  if (swap_ab && m > 64) return FL_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  {
    const cudaError_t e = gemm_init_attrs();
    if (e != cudaSuccess) return record(e);
  }
  GemmLaunch g{};
  GemmArgs& a = g.args;
  CUtensorMap ta, tb;
  a.k_chunks = ceil_div(k, 64);
  a.epi = kEpiStore;
  a.out = D;
  a.ldo = n;
  a.n_feat = n;
  a.n_tok = m;
  if (swap_ab) {
    const int bn = swap_bn(m);
    const int tiles = ceil_div(n, 128);
    const int splits = split_factor(tiles, a.k_chunks);
    const size_t need = fl_test_gemm_scratch_bytes(m, n, k, 1);
    if (splits > 1 && (!scratch || scratch_bytes < need || (reinterpret_cast<uintptr_t>(scratch) & 255)))
      return FL_ERR_WORKSPACE;
    if (!encode_tmap_bf16(&ta, B, k, n, 0, 128) || !encode_tmap_bf16(&tb, A, k, m, 0, bn)) return FL_ERR_INVALID_ARG;
    g.a0 = &ta; g.b0 = &tb; g.bn = bn;
    a.swap = 1; a.splits = splits;
    if (splits > 1) {
      a.partial = static_cast<float*>(scratch);
      a.counters = reinterpret_cast<int*>(static_cast<uint8_t*>(scratch) +
                                          ((gemm_partial_floats(bn, 0, tiles, splits) * 4 + 255) & ~size_t(255)));
      const cudaError_t e = cudaMemsetAsync(a.counters, 0, static_cast<size_t>(tiles) * 4, s);
      if (e != cudaSuccess) return record(e);
    }
    g.grid = dim3(tiles, 1, splits);
  } else {
    if (!encode_tmap_bf16(&ta, A, k, m, 0, 128) || !encode_tmap_bf16(&tb, B, k, n, 0, 128)) return FL_ERR_INVALID_ARG;
    g.a0 = &ta; g.b0 = &tb; g.bn = 128;   // the normal orientation (the persistent kernel sizes its own grid)
    a.swap = 0; a.splits = 1;
  }
  return record(launch_gemm(g, s));
}

}  // extern "C"
