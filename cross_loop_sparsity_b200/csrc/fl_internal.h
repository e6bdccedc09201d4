// fl_internal.h -- declarations shared by the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>
#include <string>

namespace fl {

// ------------------------------------------------------------------ GEMM
// D = A * B^T on tcgen05 (bf16 operands, fp32 accumulate in TMEM).  A and B
// are K-major bf16 tiles streamed by TMA: A boxes are 128 rows x 64, B boxes
// BN rows x 64.  The accumulator row is an A row and its column a B row.
//   swap = 1: A = weights (row = output feature), B = tokens (<= BN of them).
//   swap = 0: A = tokens, B = weights (BN = 128 features per tile).
enum Epi : int {
  kEpiStore = 0,   // out[tok * ldo + feat] = acc
  kEpiResid = 1,   // h[row(tok) * ldh + feat] += scale * acc, row(tok) = idx ? idx[tok] : tok
  kEpiSwiglu = 2,  // act[tok * ld_act + feat] = bf16(silu(acc0) * acc1)
};

struct GemmArgs {
  int k_chunks;   // ceil(K / 64)
  int splits;     // split-K factor (grid.z); > 1 only with swap = 1
  int a_z, b_z;   // layer coordinate for 3-D (layer-stacked) tensor maps
  int swap;
  int epi;
  int n_feat;     // valid output features
  int n_tok;      // valid tokens
  float* out;
  int ldo;
  float* h;
  const int* idx;
  float scale;
  int ldh;
  uint16_t* act;
  int ld_act;
  float* partial;   // split-K scratch: splits * grid.x * NACC * BN * 128 fp32 (ticket path)
  int* counters;    // one per grid.x tile; zero between launches (ticket path)
  int cluster;      // split-K through a (1,1,splits) cluster and distributed shared memory
                    // instead of global partials and tickets (splits <= kMaxClusterSplits)
  int* status;
  // Launch timing (nullptr: off): the earliest time any CTA's dependency wait
  // returned (atomicMin) and the time the last CTA finished (atomicMax), from
  // the global nanosecond timer.
  unsigned long long* stamp_start;
  unsigned long long* stamp_end;
  // Sums of squares for the next RMSNorm, written by a residual epilogue of the
  // cluster split-K path: ss_out[tile_m * ss_ld + tok] = sum over the tile's
  // 128 features of the updated h[r_tok][feat]^2 (nullptr: not written).
  float* ss_out;
  int ss_ld;
  // Input RMSNorm (swap orientation): the token operand is built in shared
  // memory from fp32 hidden rows instead of loaded by TMA:
  //   x[t][k] = bf16(h[r_t][k] * rsqrt(sum_p ss_in[p * ss_ld + t] / K + in_eps) * in_gain[k])
  // with r_t = in_idx ? in_idx[t] : t, p < ss_parts, and zero rows t >= n_tok.
  const float* in_h;   // nullptr: TMA operand
  const int* in_idx;
  const float* in_gain;
  const float* ss_in;
  int in_ld, ss_parts;
  float in_eps;
};

struct GemmLaunch {
  const CUtensorMap* a0;
  const CUtensorMap* a1;   // second A operand (dual, swap: gate / up weights) or nullptr
  const CUtensorMap* b0;
  const CUtensorMap* b1;   // second B operand (dual, normal: gate / up weights) or nullptr
  int bn;                  // token columns of a swap tile: 16, 32 or 64; 128 tags the normal orientation
  int a_3d, b_3d;          // operand maps are layer-stacked (rank 3)
  dim3 grid;               // swap orientation; the persistent normal-orientation kernel sizes its own
  GemmArgs args;
  bool pdl = false;        // launched as a programmatic dependent of the previous kernel
};

constexpr int kMaxClusterSplits = 16;  // non-portable cluster size, opted in per kernel
constexpr int kNumSM = 148;            // B200 streaming multiprocessors

// Token columns of a skinny (swap-orientation) tile for n <= 64 tokens.
inline int swap_bn(int n) { return n <= 16 ? 16 : n <= 32 ? 32 : 64; }

// Split-K factor of a skinny GEMM with `tiles` 128-row feature tiles and
// k_chunks 64-wide k-chunks: about one CTA per SM, at most one split per chunk.
inline int split_factor(int tiles, int k_chunks) {
  if (tiles >= kNumSM) return 1;
  int s = kNumSM / tiles;
  if (s > k_chunks) s = k_chunks;
  return s < 1 ? 1 : s;
}
cudaError_t launch_gemm(const GemmLaunch& g, cudaStream_t stream);

// Launch a kernel, with programmatic stream serialisation when `pdl` is set
// (only for launches whose predecessor in the stream is one of this
// library's kernels that follows the pdl_wait discipline).
template <typename... KArgs, typename... Args>
cudaError_t launch_k(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}
cudaError_t gemm_init_attrs();   // opt the GEMM kernels in to their shared memory (once)
// Largest split-K scratch (floats) one launch with these sizes may use.
size_t gemm_partial_floats(int bn, int dual, int tiles, int splits);

// Tensor map over a bf16 matrix [layers][rows][k] (rank 3 when layers > 0,
// else [rows][k] rank 2), 128-byte swizzle, box 64 x box_rows (x 1).
bool encode_tmap_bf16(CUtensorMap* map, const void* base, uint64_t k, uint64_t rows, uint64_t layers,
                      uint32_t box_rows);

// Record the reason of a failure of an entry point that has no context
// (reported by flashloop_last_cuda_error(NULL)).
void set_last_error(const std::string& why);

// ------------------------------------------------------------------ other kernels
struct SelectSeg;  // fwd

cudaError_t launch_topk(const float* keys, int n_seg, int n, int k, int32_t* idx, cudaStream_t s);
cudaError_t launch_quantize_rows(const float* r, const uint16_t* prev, int rows, int width, int g, int bits,
                                 uint8_t* codes, uint16_t* scales, cudaStream_t s);

}  // namespace fl
