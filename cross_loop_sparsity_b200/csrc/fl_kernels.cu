// fl_kernels.cu -- every step of the lazy-update looped step except the GEMMs:
// pre-norm gather, RoPE + KV store / residual quantise, top-k selection,
// decode and prefill attention, delta-score column keys, sparse-column
// correction, and the per-token change keys.  Method: "FlashLoop: Fast and
// Memory-Efficient Looped Transformers via Lazy Updates" (abstract).
#include <algorithm>
#include <cooperative_groups.h>

#include "fl_cache.cuh"
#include "fl_kernels.h"

namespace cg = cooperative_groups;

namespace fl {

// ============================================================================
// block helpers
// ============================================================================

// Exclusive prefix sum over the block (blockDim.x multiple of 32, <= 1024).
// Returns the exclusive prefix of v; *total receives the block total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* total, int* warp_buf /*[33]*/) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_buf[w] = x;
  __syncthreads();
  if (w == 0) {
    int t = lane < nw ? warp_buf[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < nw) warp_buf[lane] = t;  // inclusive warp totals
    if (lane == 31) warp_buf[32] = t;
  }
  __syncthreads();
  const int base = w > 0 ? warp_buf[w - 1] : 0;
  *total = warp_buf[32];
  const int r = base + x - v;
  __syncthreads();  // warp_buf reusable after return
  return r;
}

__device__ __forceinline__ float block_sum(float v, float* buf /*[32]*/) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  if (lane == 0) buf[w] = v;
  __syncthreads();
  float t = lane < nw ? buf[lane] : 0.f;
  t = warp_sum(t);
  __syncthreads();
  return t;
}

// ============================================================================
// top-k selection: the k largest fp32 keys by (bit pattern desc, index asc),
// written in ascending index order.  Radix select on 8-bit digits finds the
// k-th key's bit pattern T; then one ordered pass takes every key above T and
// the lowest-index keys equal to T.  Deterministic; no atomics in the output.
// ============================================================================

__device__ int block_topk(const float* __restrict__ keys, int n, int k, int32_t* __restrict__ out) {
  __shared__ int whist[16 * 256];   // digit histograms, one per pair of warps (one per warp below 16 warps)
  __shared__ int wgt[32], weq[32], wtot[256];
  __shared__ int sh_sel, sh_cum;
  __shared__ int scan_buf[33];
  __shared__ uint32_t small_keys[1024];
  if (k >= n) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) out[i] = i;
    __syncthreads();
    return n;
  }
  if (k <= 0) return 0;
  const uint32_t* kb = reinterpret_cast<const uint32_t*>(keys);
  if (n <= static_cast<int>(blockDim.x)) {
    // one key per thread: its rank is the number of keys that precede it in
    // (bit pattern desc, index asc) order; the k of rank < k are taken, in
    // index order by a block scan
    const int i = threadIdx.x;
    const uint32_t u = i < n ? kb[i] : 0u;
    if (i < n) small_keys[i] = u;
    __syncthreads();
    int rank = 0;
    if (i < n)
      for (int j = 0; j < n; ++j) {
        const uint32_t v = small_keys[j];
        rank += (v > u || (v == u && j < i)) ? 1 : 0;
      }
    const int take = (i < n && rank < k) ? 1 : 0;
    int total;
    const int pos = block_exclusive_scan(take, &total, scan_buf);
    if (take) out[pos] = i;
    __syncthreads();
    return k;
  }
  // radix select: warp w owns keys [w*chunk, (w+1)*chunk) and shares a
  // 256-bin histogram per 8-bit digit with at most one other warp (no
  // block-wide atomics); one warp finds the digit holding the k_rem-th largest
  // key; two block barriers per digit
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int nh = nw < 16 ? nw : 16;
  const int chunk = (n + nw - 1) / nw;
  const int lo = min(n, w * chunk), hi = min(n, lo + chunk);
  int* wh = whist + (w % nh) * 256;
  uint32_t prefix = 0, mask = 0;
  int k_rem = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (w < nh)
#pragma unroll
      for (int b = lane; b < 256; b += 32) wh[b] = 0;
    __syncthreads();
    for (int i0 = lo; i0 < hi; i0 += 32) {
      // keys of similar magnitude share their leading digits: when every
      // candidate lane of the warp hits the same bin, one atomic adds them all
      const int i = i0 + lane;
      const uint32_t u = i < hi ? kb[i] : 0u;
      const bool in = i < hi && (u & mask) == prefix;
      const int bin = static_cast<int>((u >> shift) & 0xFF);
      const unsigned inb = __ballot_sync(0xffffffffu, in);
      if (inb == 0u) continue;
      const int b0 = __shfl_sync(0xffffffffu, bin, __ffs(inb) - 1);
      if (__all_sync(0xffffffffu, !in || bin == b0)) {
        if (lane == 0) atomicAdd(&wh[b0], __popc(inb));
      } else if (in) {
        atomicAdd(&wh[bin], 1);
      }
    }
    __syncthreads();
    // fold the histograms: thread t totals digits t, t + blockDim.x, ...
    for (int dg = threadIdx.x; dg < 256; dg += blockDim.x) {
      int c = 0;
      for (int ww = 0; ww < nh; ++ww) c += whist[ww * 256 + dg];
      wtot[dg] = c;
    }
    __syncthreads();
    if (w == 0) {
      // lane L totals digits 255-8L .. 248-8L (descending), then a warp scan
      int cnt[8], tot = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        cnt[e] = wtot[255 - 8 * lane - e];
        tot += cnt[e];
      }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int before = incl - tot;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (before < k_rem && before + cnt[e] >= k_rem) {
          sh_sel = 255 - 8 * lane - e;
          sh_cum = before;
        }
        before += cnt[e];
      }
    }
    __syncthreads();
    k_rem -= sh_cum;
    prefix |= static_cast<uint32_t>(sh_sel) << shift;
    mask |= 0xFFu << shift;
  }
  // prefix = bit pattern of the k-th largest key: take every key above it and
  // the k_rem lowest-index keys equal to it, in index order.  Each warp counts
  // its range, one warp turns the counts into offsets, each warp writes.
  int gt_n = 0, eq_n = 0;
  for (int i0 = lo; i0 < hi; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t u = i < hi ? kb[i] : 0u;
    gt_n += __popc(__ballot_sync(0xffffffffu, i < hi && u > prefix));
    eq_n += __popc(__ballot_sync(0xffffffffu, i < hi && u == prefix));
  }
  if (lane == 0) {
    wgt[w] = gt_n;
    weq[w] = eq_n;
  }
  __syncthreads();
  if (w == 0) {
    const int g0 = lane < nw ? wgt[lane] : 0, e0 = lane < nw ? weq[lane] : 0;
    int ge = e0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ge, o);
      if (lane >= o) ge += y;
    }
    const int eq_before = ge - e0;
    const int take_eq = max(0, min(e0, k_rem - eq_before));
    int tk = g0 + take_eq, incl = tk;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane < nw) {
      weq[lane] = eq_before;         // equal keys in earlier warps
      wgt[lane] = incl - tk;         // output slots taken by earlier warps
    }
  }
  __syncthreads();
  int eq_seen = weq[w], pos0 = wgt[w];
  const unsigned lt = (1u << lane) - 1u;
  for (int i0 = lo; i0 < hi; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t u = i < hi ? kb[i] : 0u;
    const bool eq = i < hi && u == prefix;
    const unsigned eqb = __ballot_sync(0xffffffffu, eq);
    const bool take = (i < hi && u > prefix) || (eq && eq_seen + __popc(eqb & lt) < k_rem);
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) out[pos0 + __popc(tb & lt)] = i;
    eq_seen += __popc(eqb);
    pos0 += __popc(tb);
  }
  __syncthreads();
  return k;
}

// copy n keys into shared memory, four loads in flight per thread
__device__ __forceinline__ void stage_keys(const float* __restrict__ src, int n, float* dst) {
  for (int e0 = 0; e0 < n; e0 += 4 * blockDim.x) {
    float v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = e0 + u * blockDim.x + threadIdx.x;
      v[u] = e < n ? src[e] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = e0 + u * blockDim.x + threadIdx.x;
      if (e < n) dst[e] = v[u];
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(1024) k_topk_segments(const float* __restrict__ keys, int n, int k,
                                                        int32_t* __restrict__ idx) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float keys_sm[];   // [n] when n <= kSelColsSmemKeys
  const int s = blockIdx.x;
  const float* src = keys + static_cast<size_t>(s) * n;
  if (n <= kSelColsSmemKeys) {
    stage_keys(src, n, keys_sm);
    src = keys_sm;
  }
  block_topk(src, n, k, idx + static_cast<size_t>(s) * (k < n ? k : n));
}

// Token selection of a lazy loop: top-n_sel over the N keys, or the forced
// indices when forced_on[0] has kForceSel set.
__global__ void __launch_bounds__(1024) k_select_tokens(const float* __restrict__ keys, int N, int n_sel,
                                                        int32_t* __restrict__ idx, const int* forced_on,
                                                        const int32_t* __restrict__ forced) {
  pdl_trigger();
  pdl_wait();
  if (forced_on && (forced_on[0] & kForceSel)) {
    for (int i = threadIdx.x; i < n_sel; i += blockDim.x) idx[i] = forced[i];
    return;
  }
  block_topk(keys, N, n_sel, idx);
}

// ============================================================================
// pre-norm gather: x[i] = bf16(gain * h[idx[i]] / sqrt(mean(h^2) + eps)); rows
// n..gridDim.x-1 are zero padding for the MMA tile.
// ============================================================================
__global__ void __launch_bounds__(256) k_rmsnorm_rows(const float* __restrict__ h, const int* __restrict__ idx,
                                                      int n, int d, const float* __restrict__ gain, float eps,
                                                      uint16_t* __restrict__ x) {
  pdl_trigger();
  pdl_wait();
  __shared__ float buf[32];
  const int i = blockIdx.x;
  uint16_t* xr = x + static_cast<size_t>(i) * d;
  if (i >= n) {
    for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4)
      *reinterpret_cast<uint2*>(xr + c) = make_uint2(0u, 0u);
    return;
  }
  const int r = idx ? idx[i] : i;
  const float* hr = h + static_cast<size_t>(r) * d;
  float ss = 0.f;
  for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4*>(hr + c);
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  const float tot = block_sum(ss, buf);
  const float inv = rsqrtf(tot / static_cast<float>(d) + eps);
  for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4*>(hr + c);
    const float4 gv = *reinterpret_cast<const float4*>(gain + c);
    const uint32_t lo = f_to_bf16(v.x * inv * gv.x) | (static_cast<uint32_t>(f_to_bf16(v.y * inv * gv.y)) << 16);
    const uint32_t hi = f_to_bf16(v.z * inv * gv.z) | (static_cast<uint32_t>(f_to_bf16(v.w * inv * gv.w)) << 16);
    *reinterpret_cast<uint2*>(xr + c) = make_uint2(lo, hi);
  }
}

// ============================================================================
// residual quantiser of one group, lane-distributed: the group is GL = g/EPL
// consecutive lanes, g = 2^lg.  s = fp16_RU(fp32(absmax / qmax)) (0 if absmax is 0),
// code = clamp(rint(fp32(r / s)), -qmax, qmax), ties to even.
// Returns the lane's codes and the group's fp16 scale bits.
// ============================================================================
template <int EPL, int BITS = 0>
__device__ __forceinline__ uint16_t quantize_lane(const float* r, int lg, int bits_rt, int* code) {
  const int bits = BITS ? BITS : bits_rt;
  const int GL = 1 << (lg - (EPL == 4 ? 2 : 1));
  float am = 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) am = fmaxf(am, fabsf(r[e]));
  for (int o = GL >> 1; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  const int qm = (1 << (bits - 1)) - 1;
  const uint16_t sh = quant_scale(am, qm);
  const float s = half_bits_to_f(sh);
  const float inv = s > 0.f ? rcp_approx(s) : 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) code[e] = quant_code(r[e], s, inv, qm);
  return sh;
}

// Pack the lane's codes (two's complement, element order low bits first) and
// store them into a packed row; for EPL=2 with 2-bit codes two lanes share a byte.
template <int EPL, int BITS = 0>
__device__ __forceinline__ void store_lane_codes(uint8_t* row, int bits_rt, int lane, const int* c) {
  const int bits = BITS ? BITS : bits_rt;
  if (EPL == 4) {
    if (bits == 4) {
      const uint32_t u = (c[0] & 0xF) | ((c[1] & 0xF) << 4) | ((c[2] & 0xF) << 8) | ((c[3] & 0xF) << 12);
      *reinterpret_cast<uint16_t*>(row + lane * 2) = static_cast<uint16_t>(u);
    } else {
      row[lane] = static_cast<uint8_t>((c[0] & 3) | ((c[1] & 3) << 2) | ((c[2] & 3) << 4) | ((c[3] & 3) << 6));
    }
  } else {
    if (bits == 4) {
      row[lane] = static_cast<uint8_t>((c[0] & 0xF) | ((c[1] & 0xF) << 4));
    } else {
      const uint32_t nib = (c[0] & 3) | ((c[1] & 3) << 2);
      const uint32_t other = __shfl_down_sync(0xffffffffu, nib, 1);
      if ((lane & 1) == 0) row[lane >> 1] = static_cast<uint8_t>(nib | (other << 4));
    }
  }
}

// Rows of residuals, quantised and packed: r = x (prev == nullptr) or
// r = fp32(x) - fp32(prev) with prev bf16 (the residual of a new KV row
// against the previous loop's).  Each warp takes PER row chunks of 32 * EPL
// values, all loads issued before any arithmetic.  Item indices are 32-bit
// (the entry point bounds rows * chunks).
template <int EPL, int BITS>
__global__ void __launch_bounds__(256) k_quantize_rows(const float* __restrict__ x,
                                                       const uint16_t* __restrict__ prev, int rows, int width, int g,
                                                       int bits, uint8_t* __restrict__ codes,
                                                       uint16_t* __restrict__ scales) {
  pdl_trigger();
  pdl_wait();
  constexpr int PER = 4;   // row chunks per warp, loaded together
  const int lane = threadIdx.x & 31;
  const unsigned chunks = static_cast<unsigned>(width / (32 * EPL));
  const unsigned total = static_cast<unsigned>(rows) * chunks;
  const unsigned w0 = (blockIdx.x * 8u + (threadIdx.x >> 5)) * PER;
  float v[PER][EPL];
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const unsigned w = w0 + u;
    if (w >= total) continue;
    const unsigned row = chunks == 1u ? w : w / chunks, ch = chunks == 1u ? 0u : w % chunks;
    const size_t off = static_cast<size_t>(row) * width + ch * 32 * EPL + lane * EPL;
    if (EPL == 4) {
      const float4 q = *reinterpret_cast<const float4*>(x + off);
      v[u][0] = q.x; v[u][EPL > 1 ? 1 : 0] = q.y; v[u][EPL > 2 ? 2 : 0] = q.z; v[u][EPL > 3 ? 3 : 0] = q.w;
    } else {
      const float2 q = *reinterpret_cast<const float2*>(x + off);
      v[u][0] = q.x; v[u][EPL > 1 ? 1 : 0] = q.y;
    }
    if (prev) {
      if (EPL == 4) {
        const uint2 pb = *reinterpret_cast<const uint2*>(prev + off);
        v[u][0] = __fsub_rn(v[u][0], bf16_to_f(pb.x & 0xFFFF));
        v[u][EPL > 1 ? 1 : 0] = __fsub_rn(v[u][EPL > 1 ? 1 : 0], bf16_to_f(pb.x >> 16));
        v[u][EPL > 2 ? 2 : 0] = __fsub_rn(v[u][EPL > 2 ? 2 : 0], bf16_to_f(pb.y & 0xFFFF));
        v[u][EPL > 3 ? 3 : 0] = __fsub_rn(v[u][EPL > 3 ? 3 : 0], bf16_to_f(pb.y >> 16));
      } else {
        const uint32_t pb = *reinterpret_cast<const uint32_t*>(prev + off);
        v[u][0] = __fsub_rn(v[u][0], bf16_to_f(pb & 0xFFFF));
        v[u][EPL > 1 ? 1 : 0] = __fsub_rn(v[u][EPL > 1 ? 1 : 0], bf16_to_f(pb >> 16));
      }
    }
  }
  // g is a power of two (the entry point admits 32, 64, 128): shifts, not divisions
  const int lg = __ffs(g) - 1, lgl = lg - (EPL == 4 ? 2 : 1);
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const unsigned w = w0 + u;
    if (w >= total) break;   // warp-uniform
    const unsigned row = chunks == 1u ? w : w / chunks, ch = chunks == 1u ? 0u : w % chunks;
    int c[EPL];
    const uint16_t sc = quantize_lane<EPL, BITS>(v[u], lg, BITS, c);
    uint8_t* crow = codes + ((static_cast<size_t>(row) * width + ch * 32 * EPL) * BITS >> 3);
    store_lane_codes<EPL, BITS>(crow, BITS, lane, c);
    if ((lane & ((1 << lgl) - 1)) == 0)
      scales[(static_cast<size_t>(row) * width >> lg) + ((ch * 32 * EPL) >> lg) + (lane >> lgl)] = sc;
  }
}

// ============================================================================
// RoPE + KV store / residual quantise (one warp per (GEMM row, head)).
//   q heads : rotate, write q_cur (and q_last at loop 1 of the lazy path)
//   k heads : rotate; v heads: as is.  Then
//     dense   : store bf16 into this loop's own KV
//     lazy l=1: store bf16 base; zero the residual rows of loops 2..K
//     lazy l>1: r = kv - reconstructed(loop l-1); quantise; store codes+scale
// ============================================================================
template <int EPL, int KM, bool SP>
__global__ void __launch_bounds__(128) k_qkv_post(const QkvPostArgs a) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int item = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int heads = a.H + 2 * a.Hkv;
  if (item >= a.n * heads) return;
  const int i = item / heads, hh = item % heads;
  const int tok = a.idx ? a.idx[i] : i;
  const int b = a.seq[tok], t = a.pos[tok];
  const int hd = a.hd, half = hd / 2;
  const float* src = a.qkv + static_cast<size_t>(i) * a.ldq + static_cast<size_t>(hh) * hd + lane * EPL;
  float x[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) x[e] = src[e];
  const bool is_v = hh >= a.H + a.Hkv;
  if (!is_v) {
    float y[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) y[e] = __shfl_xor_sync(0xffffffffu, x[e], 16);
    const int ai = (lane & 15) * EPL;
    const float* cs = a.rope_cos + static_cast<size_t>(t) * half + ai;
    const float* sn = a.rope_sin + static_cast<size_t>(t) * half + ai;
#pragma unroll
    for (int e = 0; e < EPL; ++e)   // explicit roundings: the GEMM epilogue's rotation matches bit for bit
      x[e] = lane < 16 ? __fmaf_rn(x[e], cs[e], -__fmul_rn(y[e], sn[e])) : __fmaf_rn(x[e], cs[e], __fmul_rn(y[e], sn[e]));
  }
  if (hh < a.H) {
    float* dq = a.q_cur + (static_cast<size_t>(i) * a.H + hh) * hd + lane * EPL;
#pragma unroll
    for (int e = 0; e < EPL; ++e) dq[e] = x[e];
    if (a.lazy && a.loop == 1 && a.q_last) {
      float* ql = a.q_last + (static_cast<size_t>(tok) * a.H + hh) * hd + lane * EPL;
#pragma unroll
      for (int e = 0; e < EPL; ++e) ql[e] = x[e];
    }
    return;
  }
  const int kv = is_v ? 1 : 0;
  const int gk = is_v ? hh - a.H - a.Hkv : hh - a.H;
  const CacheView& cv = a.cv;
  if (!a.lazy || a.loop == 1) {
    uint16_t* dst = (a.lazy ? cv.base_row(a.j, kv, b, gk, t) : cv.dense_row(a.j, a.loop, kv, b, gk, t)) + lane * EPL;
    if (EPL == 4) {
      const uint32_t lo = f_to_bf16(x[0]) | (static_cast<uint32_t>(f_to_bf16(x[1])) << 16);
      const uint32_t hi = f_to_bf16(x[2]) | (static_cast<uint32_t>(f_to_bf16(x[3])) << 16);
      *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
    } else {
      *reinterpret_cast<uint32_t*>(dst) = f_to_bf16(x[0]) | (static_cast<uint32_t>(f_to_bf16(x[1])) << 16);
    }
    if (a.lazy && !cv.rows) {   // (with sparse storage the selection marks unrecomputed rows instead)
      const int rb = static_cast<int>(cv.row_bytes_codes());
      const int ns = hd >> cv.lg;
      for (int l = 2; l <= cv.K; ++l) {
        uint8_t* cr = cv.code_row(a.j, l, kv, b, gk, t);
        for (int o = lane; o < rb; o += 32) cr[o] = 0;
        uint16_t* sr = cv.scale_row(a.j, l, kv, b, gk, t);
        if (lane < ns) sr[lane] = 0;
      }
    }
    return;
  }
  int c[EPL];
  uint16_t s;
  if (a.forced_on && a.forced_on[0]) {
    // checks only: the caller's codes for this selection slot
    const size_t row = (((static_cast<size_t>(a.j) * (cv.K - 1) + (a.loop - 2)) * a.forced_ns + i) * 2 + kv) *
                           a.Hkv + gk;
#pragma unroll
    for (int e = 0; e < EPL; ++e) c[e] = a.forced_codes[row * hd + lane * EPL + e];
    s = a.forced_scales[row * (hd >> cv.lg) + ((lane * EPL) >> cv.lg)];
  } else {
    if (a.trace_kv && i < a.trace_ns) {
      float* tr = a.trace_kv + ((((static_cast<size_t>(a.j) * (cv.K - 1) + (a.loop - 2)) * a.trace_ns + i) * 2 + kv) *
                                    a.Hkv + gk) * hd + lane * EPL;
#pragma unroll
      for (int e = 0; e < EPL; ++e) tr[e] = x[e];
    }
    // the previous level, every level's loads issued together (levels without a
    // row add code 0 x scale 0, as a stored zero row does)
    float prev[EPL], unused[EPL];
    chain_lane2<EPL, KM, SP>(cv, a.j, kv, b, gk, t, a.loop - 1, a.loop - 1, lane, unused, prev);
    float r[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) r[e] = __fsub_rn(x[e], prev[e]);
    s = quantize_lane<EPL>(r, cv.lg, cv.bits, c);
  }
  const int r = cv.res_row(a.j, a.loop, b, t);   // the pool row the selection gave this token
  if (r < 0) return;                               // (no room: the selection recorded the overflow)
  store_lane_codes<EPL>(cv.code_row(a.j, a.loop, kv, b, gk, r), cv.bits, lane, c);
  const int lgl = cv.lg - (EPL == 4 ? 2 : 1);   // log2 of the lanes per group
  if ((lane & ((1 << lgl) - 1)) == 0) cv.scale_row(a.j, a.loop, kv, b, gk, r)[lane >> lgl] = s;
}

constexpr int kDecTile = 64;
constexpr int kDecPad = 8;     // bf16 elements of padding per staged row (16-byte skew)
constexpr int kDecStages = 3;  // K/V tiles in flight per CTA (two CTAs per SM)

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ---- warp-level tensor-core helpers for the decode attention
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// D[16x8] += A[16x16] * B[16x8], bf16 operands, fp32 accumulate
__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return static_cast<uint32_t>(f_to_bf16(lo)) | (static_cast<uint32_t>(f_to_bf16(hi)) << 16);
}
// x ~= hi + lo with hi = bf16(x), lo = bf16(x - hi): a product of a bf16 value
// with hi and lo, summed in fp32, carries about 16 significant bits of x
__device__ __forceinline__ void split_bf16(float x, float& hi, float& lo) {
  hi = bf16_to_f(f_to_bf16(x));
  lo = x - hi;
}

// ============================================================================
// decode attention over one cache (lazy base at loop 1, or the dense
// baseline's own per-loop KV): grid (n*Hkv, splits), 128 threads (4 warps).
// Each CTA takes the group's query heads (<= 8) over a range of 64-column
// tiles.  K/V tiles arrive by TMA (128-byte swizzle) in a ring of kDecStages.
// Scores S = tau * K q^T and the update O += P V are warp-level bf16 tensor-core
// products with fp32 accumulation: q and P are carried as hi + lo bf16 pairs
// (the lo half of P rides in the spare rows of the 16-row operand), the cache
// values are bf16 already, so the products keep about fp32 accuracy.  The
// online softmax runs on the score fragments.  The last CTA of a (token, KV
// head) -- an atomic ticket, no waiting -- merges the splits' (max, sum,
// unnormalised output) and writes O, lse.
// ============================================================================
template <int HD, int GRP>
__global__ void __launch_bounds__(128, 2) k_attn_decode(const __grid_constant__ CUtensorMap kvmap, const AttnDecArgs a) {
  constexpr int NB = HD / 64;                       // 128-byte TMA boxes per row
  constexpr int BOX_BYTES = kDecTile * 128;         // one box of a 64-row tile
  constexpr int TILE_BYTES = NB * BOX_BYTES;        // K or V of one tile
  constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  constexpr int KSTEPS = HD / 16;                   // k-steps of the score product
  constexpr int NTW = HD / 32;                      // 8-dim output tiles per warp
  static_assert(GRP <= 8 && NTW % 2 == 0, "decode attention shape");
  extern __shared__ uint8_t sm_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[kDecStages];
  __shared__ __align__(128) uint16_t Pt[16 * 64];   // P^T operand: rows hi heads 0-7, lo heads 0-7; 64 columns
  __shared__ float red_max[4][8];
  __shared__ float alpha_s[8];
  __shared__ float red_l[4][8];
  __shared__ float sm_m[8], sm_l[8];
  __shared__ int flag;

  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int i = blockIdx.x / a.Hkv, g = blockIdx.x % a.Hkv, sp = blockIdx.y;
  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) mbar_init(smem_u32(&full[s]), 1);
    fence_mbar_init();
    flag = 0;
  }
  pdl_wait();
  const int tok = a.idx ? a.idx[i] : i;
  const int b = a.seq[tok], P = a.pos[tok];
  const int ncols = P + 1;
  const int nt = (ncols + kDecTile - 1) / kDecTile;
  const int t_begin = static_cast<int>((static_cast<long long>(sp) * nt) / a.n_splits);
  const int t_end = static_cast<int>((static_cast<long long>(sp + 1) * nt) / a.n_splits);
  const int ntiles = t_end - t_begin;
  const CacheView& cv = a.cv;
  // first row of this (layer, loop, K/V, sequence, KV head) in the 2-D [rows][hd] view of the cache
  const size_t bh = static_cast<size_t>(b) * cv.Hkv + g;
  const size_t plane = static_cast<size_t>(cv.B) * cv.Hkv * cv.T;
  const size_t rk = a.dense ? ((static_cast<size_t>(a.j) * cv.K + cv.dense_slot(a.loop)) * 2) * plane + bh * cv.T
                            : (static_cast<size_t>(a.j) * 2) * plane + bh * cv.T;
  const int row_k = static_cast<int>(rk), row_v = static_cast<int>(rk + plane);
  __syncthreads();   // barrier initialisation visible to every thread
  auto issue = [&](int u) {
    const int s = u % kDecStages;
    const int y = (t_begin + u) * kDecTile;
    uint8_t* st = ring + s * STAGE_BYTES;
    const uint32_t fb = smem_u32(&full[s]);
    mbar_arrive_expect_tx(fb, STAGE_BYTES);
#pragma unroll
    for (int bx = 0; bx < NB; ++bx) {
      tma_load_2d(smem_u32(st + bx * BOX_BYTES), &kvmap, fb, bx * 64, row_k + y);
      tma_load_2d(smem_u32(st + TILE_BYTES + bx * BOX_BYTES), &kvmap, fb, bx * 64, row_v + y);
    }
  };
  if (tid == 0) {
    tma_prefetch_desc(&kvmap);
    for (int u = 0; u < kDecStages && u < ntiles; ++u) issue(u);
  }

  // q^T as the B operand of the score product (k = dims, n = heads), tau folded
  // in, split into hi and lo bf16 parts: lane holds head lane/4, dims 2(lane%4)+{0,1,8,9}
  uint32_t qb_hi[KSTEPS][2], qb_lo[KSTEPS][2];
  {
    const int hn = lane >> 2;
    const float* qh = a.q_cur + (static_cast<size_t>(i) * a.H + g * GRP + (hn < GRP ? hn : 0)) * HD;
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int d = ks * 16 + 2 * (lane & 3) + r * 8;
        float x0 = hn < GRP ? qh[d] * a.tau : 0.f, x1 = hn < GRP ? qh[d + 1] * a.tau : 0.f;
        float h0, l0, h1, l1;
        split_bf16(x0, h0, l0);
        split_bf16(x1, h1, l1);
        qb_hi[ks][r] = pack_bf16x2(h0, h1);
        qb_lo[ks][r] = pack_bf16x2(l0, l1);
      }
    }
  }
  // online-softmax state of this thread's two heads (2(lane%4), +1); every
  // thread tracks the running maxima, the sums are per-thread partials
  const int h0 = 2 * (lane & 3);
  float m_run[2] = {-INFINITY, -INFINITY}, l_part[2] = {0.f, 0.f};
  float acc[NTW][4];
#pragma unroll
  for (int n = 0; n < NTW; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  const uint32_t pt_base = smem_u32(Pt);

  int u_stop = ntiles;
  for (int u = 0; u < ntiles; ++u) {
    const int s = u % kDecStages;
    if (tid == 0) flag = mbar_wait(smem_u32(&full[s]), (u / kDecStages) & 1, a.status) ? 0 : 1;
    __syncthreads();
    if (flag) {
      u_stop = u;
      break;
    }
    mbar_try_wait(smem_u32(&full[s]), (u / kDecStages) & 1);   // completed: acquire the tile for this thread
    const uint32_t Kt = smem_u32(ring + s * STAGE_BYTES);
    const uint32_t Vt = Kt + TILE_BYTES;
    const int nc = min(kDecTile, ncols - (t_begin + u) * kDecTile);
    // ---- scores of this warp's 16 columns (rows of the product) x 8 heads
    float sc[4];
    {
      // four independent accumulation chains (hi / lo parts x even / odd k-steps), summed at the end
      float s4[4][4] = {};
      const int r = warp * 16 + (lane & 15);   // column row of the K tile this lane addresses
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        const int q = ks * 2 + (lane >> 4);   // 16-byte chunk (8 dims)
        uint32_t af[4];
        ldsm_x4(Kt + (q >> 3) * BOX_BYTES + r * 128 + (((q & 7) ^ (r & 7)) << 4), af);
        mma_bf16_16816(s4[(ks & 1) * 2], af, qb_hi[ks][0], qb_hi[ks][1]);
        mma_bf16_16816(s4[(ks & 1) * 2 + 1], af, qb_lo[ks][0], qb_lo[ks][1]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[e] = (s4[0][e] + s4[2][e]) + (s4[1][e] + s4[3][e]);
    }
    // fragment: sc[0..1] column c0 = warp*16 + lane/4, heads h0, h0+1; sc[2..3] column c0 + 8
    const int c0 = warp * 16 + (lane >> 2), c1 = c0 + 8;
    if (c0 >= nc) sc[0] = sc[1] = -INFINITY;
    if (c1 >= nc) sc[2] = sc[3] = -INFINITY;
    float tm0 = fmaxf(sc[0], sc[2]), tm1 = fmaxf(sc[1], sc[3]);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      tm0 = fmaxf(tm0, __shfl_xor_sync(0xffffffffu, tm0, o));
      tm1 = fmaxf(tm1, __shfl_xor_sync(0xffffffffu, tm1, o));
    }
    if (lane < 4) {
      red_max[warp][h0] = tm0;
      red_max[warp][h0 + 1] = tm1;
    }
    __syncthreads();
    float mn[2], al[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float tmx = fmaxf(fmaxf(red_max[0][h0 + e], red_max[1][h0 + e]), fmaxf(red_max[2][h0 + e], red_max[3][h0 + e]));
      mn[e] = fmaxf(m_run[e], tmx);
      al[e] = m_run[e] == -INFINITY ? 0.f : expf(m_run[e] - mn[e]);
      m_run[e] = mn[e];
    }
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) p[e] = sc[e] == -INFINITY ? 0.f : expf(sc[e] - mn[e & 1]);
#pragma unroll
    for (int e = 0; e < 2; ++e) l_part[e] = l_part[e] * al[e] + (p[e] + p[e + 2]);
    if (lane < 4) {
      alpha_s[h0] = al[0];
      alpha_s[h0 + 1] = al[1];
    }
    // P^T rows: hi part of head h at row h, lo part at row 8 + h; column c
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int hh = h0 + (e & 1), c = (e < 2) ? c0 : c1;
      float ph, pl;
      split_bf16(p[e], ph, pl);
      const int rh = hh, rl = 8 + hh;
      Pt[rh * 64 + ((((c >> 3) ^ (rh & 7)) << 3) | (c & 7))] = f_to_bf16(ph);
      Pt[rl * 64 + ((((c >> 3) ^ (rl & 7)) << 3) | (c & 7))] = f_to_bf16(pl);
    }
    __syncthreads();
    // ---- O[16 rows (hi/lo heads) x this warp's HD/4 dims] += P^T V
    const float arow = alpha_s[lane >> 2];
#pragma unroll
    for (int n = 0; n < NTW; ++n) {
      acc[n][0] *= arow;
      acc[n][1] *= arow;
      acc[n][2] *= arow;
      acc[n][3] *= arow;
    }
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {   // 16 columns per step
      uint32_t pf[4];
      {
        const int r = lane & 15, q = ks * 2 + (lane >> 4);
        ldsm_x4(pt_base + r * 128 + ((q ^ (r & 7)) << 4), pf);
      }
      const int vr = ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;   // V row (column index)
#pragma unroll
      for (int n2 = 0; n2 < NTW / 2; ++n2) {
        const int q = (warp * NTW + n2 * 2 + (lane >> 4));   // 8-dim chunk of this lane's address
        uint32_t vf[4];
        ldsm_x4_t(Vt + (q >> 3) * BOX_BYTES + vr * 128 + (((q & 7) ^ (vr & 7)) << 4), vf);
        mma_bf16_16816(acc[n2 * 2], pf, vf[0], vf[1]);
        mma_bf16_16816(acc[n2 * 2 + 1], pf, vf[2], vf[3]);
      }
    }
    __syncthreads();   // the slot and P^T are free again
    if (tid == 0 && u + kDecStages < ntiles) issue(u + kDecStages);
  }
  if (u_stop < ntiles) {
    // a tile never arrived: let the copies still in flight land (bounded) before the CTA exits
    if (tid == 0)
      for (int u = u_stop; u < ntiles && u < u_stop + kDecStages; ++u)
        mbar_wait(smem_u32(&full[u % kDecStages]), (u / kDecStages) & 1, nullptr);
    __syncthreads();
  }
  // ---- this split's partial: per-head maxima (identical in every thread),
  // sums over all threads, unnormalised output = hi row + lo row
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    float l = l_part[e];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane < 4) red_l[warp][h0 + e] = l;
  }
  if (warp == 0 && lane < 4) {
    sm_m[h0] = m_run[0];
    sm_m[h0 + 1] = m_run[1];
  }
  __syncthreads();
  if (tid < GRP) sm_l[tid] = (red_l[0][tid] + red_l[1][tid]) + (red_l[2][tid] + red_l[3][tid]);
  const int hh = lane >> 2;
  const size_t pbase = (static_cast<size_t>(i) * a.Hkv + g) * a.n_splits + sp;
  if (hh < GRP) {
#pragma unroll
    for (int n = 0; n < NTW; ++n) {
      const int d = (warp * NTW + n) * 8 + 2 * (lane & 3);
      float* dst = a.part_o + (pbase * 8 + hh) * HD + d;
      dst[0] = acc[n][0] + acc[n][2];
      dst[1] = acc[n][1] + acc[n][3];
    }
  }
  __syncthreads();
  if (tid < GRP) {
    a.part_ml[(pbase * 8 + tid) * 2 + 0] = sm_m[tid];
    a.part_ml[(pbase * 8 + tid) * 2 + 1] = sm_l[tid];
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int old = atomicAdd(&a.counters[i * a.Hkv + g], 1);
    flag = (old == a.n_splits - 1);
  }
  __syncthreads();
  if (!flag) return;
  __threadfence();
  // merge in two rounds of loads: every split's (max, sum) at once, then every
  // split's output for this thread's elements at once
  const size_t q0 = (static_cast<size_t>(i) * a.Hkv + g) * a.n_splits;
  float* ml = reinterpret_cast<float*>(ring);   // [splits][GRP][2], then weights
  const int S = a.n_splits;
  for (int e = tid; e < S * GRP; e += 128) {
    const int s2 = e / GRP, h = e % GRP;
    const float2 v = __ldcg(reinterpret_cast<const float2*>(&a.part_ml[((q0 + s2) * 8 + h) * 2]));
    ml[e * 2] = v.x;
    ml[e * 2 + 1] = v.y;
  }
  __syncthreads();
  // warp w takes heads w, w + 4: its lanes stride over the splits
  for (int h = warp; h < GRP; h += 4) {
    float M = -INFINITY;
    for (int s2 = lane; s2 < S; s2 += 32) M = fmaxf(M, ml[(s2 * GRP + h) * 2]);
    M = warp_max(M);
    float L = 0.f;
    for (int s2 = lane; s2 < S; s2 += 32) {
      const float ms = ml[(s2 * GRP + h) * 2];
      const float w = ms == -INFINITY ? 0.f : expf(ms - M);
      ml[(s2 * GRP + h) * 2] = w;   // the split's weight replaces its maximum
      L += w * ml[(s2 * GRP + h) * 2 + 1];
    }
    L = warp_sum(L);
    if (lane == 0) {
      sm_m[h] = M;
      sm_l[h] = L;
    }
  }
  __syncthreads();
  // each thread folds four consecutive output elements (one head), the
  // splits' partial rows read as 16-byte vectors, MB splits requested together
  constexpr int E4 = (GRP * HD / 4 + 127) / 128;        // 4-element groups per thread
  constexpr int MB = 16 / E4 < 16 ? (16 / E4 > 0 ? 16 / E4 : 1) : 16;
  float4 o[E4];
#pragma unroll
  for (int t = 0; t < E4; ++t) o[t] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < S; s0 += MB) {
    float4 pv[E4][MB];
#pragma unroll
    for (int t = 0; t < E4; ++t) {
      const int e = (tid + t * 128) * 4, h = e / HD, d = e % HD;
#pragma unroll
      for (int u = 0; u < MB; ++u)
        pv[t][u] = (e < GRP * HD && s0 + u < S)
                       ? __ldcg(reinterpret_cast<const float4*>(&a.part_o[((q0 + s0 + u) * 8 + h) * HD + d]))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int t = 0; t < E4; ++t) {
      const int e = (tid + t * 128) * 4, h = e < GRP * HD ? e / HD : 0;
#pragma unroll
      for (int u = 0; u < MB; ++u)
        if (s0 + u < S) {
          const float w = ml[((s0 + u) * GRP + h) * 2];
          o[t].x += w * pv[t][u].x;
          o[t].y += w * pv[t][u].y;
          o[t].z += w * pv[t][u].z;
          o[t].w += w * pv[t][u].w;
        }
    }
  }
#pragma unroll
  for (int t = 0; t < E4; ++t) {
    const int e = (tid + t * 128) * 4;
    if (e >= GRP * HD) break;
    const int h = e / HD, d = e % HD;
    const int hq = g * GRP + h;
    const float L = sm_l[h];
    const float ov[4] = {o[t].x / L, o[t].y / L, o[t].z / L, o[t].w / L};
    if (a.o_state)
      *reinterpret_cast<float4*>(&a.o_state[(static_cast<size_t>(tok) * a.H + hq) * HD + d]) =
          make_float4(ov[0], ov[1], ov[2], ov[3]);
    uint16_t* ob = a.o_bf16 + static_cast<size_t>(i) * a.H * HD + static_cast<size_t>(hq) * HD + d;
    *reinterpret_cast<uint2*>(ob) = make_uint2(f_to_bf16(ov[0]) | (static_cast<uint32_t>(f_to_bf16(ov[1])) << 16),
                                               f_to_bf16(ov[2]) | (static_cast<uint32_t>(f_to_bf16(ov[3])) << 16));
    if (d == 0 && a.lse_state) a.lse_state[static_cast<size_t>(tok) * a.H + hq] = sm_m[h] + logf(sm_l[h]);
  }
  if (tid == 0) a.counters[i * a.Hkv + g] = 0;
}

// ============================================================================
// prefill causal attention (loop 1 of the lazy path; every loop of the dense
// baseline).  grid (ceil(T/64), H, B); 256 threads: thread (r = tid/4, c4 =
// tid%4) owns query row r, 16 score columns and HD/4 output dims.
// ============================================================================
template <int HD>
__global__ void __launch_bounds__(256) k_attn_prefill(const AttnPreArgs a) {
  pdl_trigger();
  pdl_wait();
  constexpr int BQ = 64, BK = 64;
  constexpr int RS = HD + kDecPad;
  constexpr int DV = HD / 4;
  extern __shared__ __align__(16) uint8_t sm[];
  float* Qs = reinterpret_cast<float*>(sm);                         // [BQ][HD+1]
  float* Ps = Qs + BQ * (HD + 1);                                   // [BQ][BK+1]
  uint16_t* Ks = reinterpret_cast<uint16_t*>(Ps + BQ * (BK + 1));   // [BK][RS]
  uint16_t* Vs = Ks + BK * RS;                                      // [BK][RS]

  const int tid = threadIdx.x;
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int grp = a.H / a.Hkv, g = h / grp;
  const int T = a.T;
  const int r = tid >> 2, c4 = tid & 3;
  const int q0 = qb * BQ;
  const int qpos = q0 + r;   // query index within the chunk
  const CacheView& cv = a.cv;
  // the chunk starts after the L positions the sequence already holds: query
  // qpos sits at position L + qpos and sees keys 0 .. L + qpos
  const int L = a.pos[static_cast<size_t>(b) * T];

  for (int e = tid; e < BQ * HD; e += 256) {
    const int rr = e / HD, dd = e % HD;
    const int qp = q0 + rr;
    Qs[rr * (HD + 1) + dd] = qp < T ? a.q_cur[((static_cast<size_t>(b) * T + qp) * a.H + h) * HD + dd] : 0.f;
  }
  float m = -INFINITY, l = 0.f;
  float acc[DV];
#pragma unroll
  for (int e = 0; e < DV; ++e) acc[e] = 0.f;
  const int kt_end = L + min(T, q0 + BQ);
  for (int k0 = 0; k0 < kt_end; k0 += BK) {
    __syncthreads();
    constexpr int CH = HD / 8;
    for (int e = tid; e < BK * CH; e += 256) {
      const int rr = e / CH, cc = e % CH;
      const int kp = k0 + rr;
      uint4 ku = make_uint4(0, 0, 0, 0), vu = make_uint4(0, 0, 0, 0);
      if (kp < kt_end) {
        const uint16_t* kr = a.dense ? cv.dense_row(a.j, a.loop, 0, b, g, kp) : cv.base_row(a.j, 0, b, g, kp);
        const uint16_t* vr = a.dense ? cv.dense_row(a.j, a.loop, 1, b, g, kp) : cv.base_row(a.j, 1, b, g, kp);
        ku = *reinterpret_cast<const uint4*>(kr + cc * 8);
        vu = *reinterpret_cast<const uint4*>(vr + cc * 8);
      }
      *reinterpret_cast<uint4*>(&Ks[rr * RS + cc * 8]) = ku;
      *reinterpret_cast<uint4*>(&Vs[rr * RS + cc * 8]) = vu;
    }
    __syncthreads();
    float s[16];
    float tmax = -INFINITY;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int c = c4 * 16 + j;
      const int kp = k0 + c;
      float dot = 0.f;
      const uint16_t* kr = &Ks[c * RS];
      const float* q = &Qs[r * (HD + 1)];
#pragma unroll 8
      for (int e = 0; e < HD; e += 2) {
        const uint32_t u = *reinterpret_cast<const uint32_t*>(kr + e);
        dot += q[e] * bf16_to_f(u & 0xFFFF) + q[e + 1] * bf16_to_f(u >> 16);
      }
      s[j] = (kp <= L + qpos && qpos < T) ? dot * a.tau : -INFINITY;
      tmax = fmaxf(tmax, s[j]);
    }
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    const float mnew = fmaxf(m, tmax);
    float psum = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float p = s[j] == -INFINITY ? 0.f : expf(s[j] - mnew);
      Ps[r * (BK + 1) + c4 * 16 + j] = p;
      psum += p;
    }
    psum += __shfl_xor_sync(0xffffffffu, psum, 1);
    psum += __shfl_xor_sync(0xffffffffu, psum, 2);
    const float al = m == -INFINITY ? 0.f : expf(m - mnew);
    l = l * al + psum;
    m = mnew;
    __syncthreads();
#pragma unroll
    for (int e = 0; e < DV; ++e) acc[e] *= al;
    for (int c = 0; c < BK; ++c) {
      const float p = Ps[r * (BK + 1) + c];
      const uint16_t* vr = &Vs[c * RS + c4 * DV];
#pragma unroll
      for (int e = 0; e < DV; e += 2) {
        const uint32_t u = *reinterpret_cast<const uint32_t*>(vr + e);
        acc[e] += p * bf16_to_f(u & 0xFFFF);
        acc[e + 1] += p * bf16_to_f(u >> 16);
      }
    }
  }
  if (qpos >= T) return;
  const size_t tok = static_cast<size_t>(b) * T + qpos;
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < DV; ++e) {
    const int dd = c4 * DV + e;
    const float ov = acc[e] * inv;
    if (a.o_state) a.o_state[(tok * a.H + h) * HD + dd] = ov;
    a.o_bf16[tok * a.H * HD + static_cast<size_t>(h) * HD + dd] = f_to_bf16(ov);
  }
  if (c4 == 0 && a.lse_state) a.lse_state[tok * a.H + h] = m + logf(l);
}

// ============================================================================
// prefill causal attention on the tensor cores (loop 1 of the lazy path; every
// loop of the dense baseline; the prelude / coda layers).  grid (ceil(T/64), H,
// B), 128 threads: warp w owns queries q0 + 16w .. +15 of a 64-query tile, over
// 64-key tiles of the sequence's cache (the context before a chunk, then the
// chunk up to each query's own position).  K and V tiles arrive by TMA
// (128-byte swizzle, 64-row boxes) in a ring of kPreStages.  S = tau * Q K^T
// and O += P V are warp-level bf16 products with fp32 accumulation: Q is
// carried as a bf16 hi + lo pair (two products into one accumulator, about 16
// significant bits, so the scores are as accurate as the fp32 kernel's), P as
// bf16 straight from the score registers (the accumulator layout of two 8-key
// score tiles is the A-operand layout of one 16-key step), V's fragments from
// ldmatrix with transposition.  The
// online softmax runs on the score fragments; a row's statistics live in the
// four threads of a quad.
// ============================================================================
constexpr int kPreStages = 3;
constexpr int kDscoreSMs = 148;   // the Δscore grid: two CTAs per SM of the B200

template <int HD>
__global__ void __launch_bounds__(128, 2) k_attn_prefill_tc(const __grid_constant__ CUtensorMap kvmap,
                                                            const AttnPreArgs a) {
  constexpr int NB = HD / 64;                   // 128-byte boxes per cache row
  constexpr int BOX_BYTES = 64 * 128;
  constexpr int TILE_BYTES = NB * BOX_BYTES;    // K or V of one 64-key tile
  constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  constexpr int KS = HD / 16;                   // k-steps of the score product
  constexpr int NDT = HD / 8;                   // 8-dim output tiles per warp
  extern __shared__ uint8_t sm_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[kPreStages];
  __shared__ int flag;

  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qb = gridDim.x - 1 - blockIdx.x;    // the longest causal ranges start first
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / (a.H / a.Hkv);
  const int T = a.T;
  if (tid == 0) {
    for (int st = 0; st < kPreStages; ++st) mbar_init(smem_u32(&full[st]), 1);
    fence_mbar_init();
    flag = 0;
  }
  pdl_wait();
  const CacheView& cv = a.cv;
  // the chunk starts after the L positions the sequence already holds: query
  // t of the chunk sits at position L + t and sees keys 0 .. L + t
  const int L = a.pos[static_cast<size_t>(b) * T];
  const int q0 = qb * 64;
  const int kt_end = L + min(T, q0 + 64);
  const int ntiles = (kt_end + 63) / 64;
  const size_t plane = static_cast<size_t>(cv.B) * cv.Hkv * cv.T;
  const size_t bh = static_cast<size_t>(b) * cv.Hkv + g;
  const size_t rk = a.dense ? ((static_cast<size_t>(a.j) * cv.K + cv.dense_slot(a.loop)) * 2) * plane + bh * cv.T
                            : (static_cast<size_t>(a.j) * 2) * plane + bh * cv.T;
  const int row_k = static_cast<int>(rk), row_v = static_cast<int>(rk + plane);
  __syncthreads();
  auto issue = [&](int u) {
    const int st = u % kPreStages;
    uint8_t* dst = ring + st * STAGE_BYTES;
    const uint32_t fb = smem_u32(&full[st]);
    mbar_arrive_expect_tx(fb, STAGE_BYTES);
#pragma unroll
    for (int bx = 0; bx < NB; ++bx) {
      tma_load_2d(smem_u32(dst + bx * BOX_BYTES), &kvmap, fb, bx * 64, row_k + u * 64);
      tma_load_2d(smem_u32(dst + TILE_BYTES + bx * BOX_BYTES), &kvmap, fb, bx * 64, row_v + u * 64);
    }
  };
  if (tid == 0) {
    tma_prefetch_desc(&kvmap);
    for (int u = 0; u < kPreStages && u < ntiles; ++u) issue(u);
  }
  // Q fragments (A operand, rows = queries, k = dims), tau folded in, hi + lo
  const int r0 = q0 + warp * 16 + (lane >> 2), r1 = r0 + 8;   // chunk-relative query indices
  const int P0 = L + r0, P1 = L + r1;                          // their positions
  uint32_t qh[KS][4], ql[KS][4];
  {
    const float* q0p = a.q_cur + ((static_cast<size_t>(b) * T + min(r0, T - 1)) * a.H + h) * HD;
    const float* q1p = a.q_cur + ((static_cast<size_t>(b) * T + min(r1, T - 1)) * a.H + h) * HD;
    const bool v0 = r0 < T, v1 = r1 < T;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int d = ks * 16 + 2 * (lane & 3);
      float x[8];
      x[0] = v0 ? q0p[d] : 0.f;     x[1] = v0 ? q0p[d + 1] : 0.f;
      x[2] = v1 ? q1p[d] : 0.f;     x[3] = v1 ? q1p[d + 1] : 0.f;
      x[4] = v0 ? q0p[d + 8] : 0.f; x[5] = v0 ? q0p[d + 9] : 0.f;
      x[6] = v1 ? q1p[d + 8] : 0.f; x[7] = v1 ? q1p[d + 9] : 0.f;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        float h0, l0, h1, l1;
        split_bf16(x[2 * r] * a.tau, h0, l0);
        split_bf16(x[2 * r + 1] * a.tau, h1, l1);
        qh[ks][r] = pack_bf16x2(h0, h1);
        ql[ks][r] = pack_bf16x2(l0, l1);
      }
    }
  }
  float o[NDT][4];
#pragma unroll
  for (int n = 0; n < NDT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_part[2] = {0.f, 0.f};

  int u_stop = ntiles;
  for (int u = 0; u < ntiles; ++u) {
    const int st = u % kPreStages;
    if (tid == 0) flag = mbar_wait(smem_u32(&full[st]), (u / kPreStages) & 1, a.status) ? 0 : 1;
    __syncthreads();
    if (flag) {
      u_stop = u;
      break;
    }
    mbar_try_wait(smem_u32(&full[st]), (u / kPreStages) & 1);   // completed: acquire the tile for this thread
    const uint32_t Kt = smem_u32(ring + st * STAGE_BYTES);
    const uint32_t Vt = Kt + TILE_BYTES;
    const int k0 = u * 64;
    // ---- scores of this warp's 16 queries x 64 keys (8 tiles of 8 keys)
    float sc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int ch = 2 * ks + ((lane >> 3) & 1);   // 16-byte chunk (8 dims) of the key row
        uint32_t kb[4];
        ldsm_x4(Kt + (ch >> 3) * BOX_BYTES + key * 128 + (((ch & 7) ^ (key & 7)) << 4), kb);
        mma_bf16_16816(sc[2 * np], qh[ks], kb[0], kb[1]);
        mma_bf16_16816(sc[2 * np], ql[ks], kb[0], kb[1]);
        mma_bf16_16816(sc[2 * np + 1], qh[ks], kb[2], kb[3]);
        mma_bf16_16816(sc[2 * np + 1], ql[ks], kb[2], kb[3]);
      }
    }
    // causal mask: key c is visible to the query at position P when c <= P
    float tm[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c = k0 + nt * 8 + 2 * (lane & 3) + e;
        if (c > P0 || r0 >= T) sc[nt][e] = -INFINITY;
        if (c > P1 || r1 >= T) sc[nt][2 + e] = -INFINITY;
        tm[0] = fmaxf(tm[0], sc[nt][e]);
        tm[1] = fmaxf(tm[1], sc[nt][2 + e]);
      }
    }
    float alpha[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      tm[r] = fmaxf(tm[r], __shfl_xor_sync(0xffffffffu, tm[r], 1));
      tm[r] = fmaxf(tm[r], __shfl_xor_sync(0xffffffffu, tm[r], 2));
      const float mn = fmaxf(m_run[r], tm[r]);
      alpha[r] = (m_run[r] == -INFINITY || mn == -INFINITY) ? (m_run[r] == -INFINITY ? 0.f : 1.f)
                                                             : expf(m_run[r] - mn);
      m_run[r] = mn;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float mr = m_run[e >> 1];
        const float pv = (sc[nt][e] == -INFINITY) ? 0.f : expf(sc[nt][e] - mr);
        sc[nt][e] = pv;
        rs[e >> 1] += pv;
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) l_part[r] = l_part[r] * alpha[r] + rs[r];
#pragma unroll
    for (int n = 0; n < NDT; ++n) {
      o[n][0] *= alpha[0];
      o[n][1] *= alpha[0];
      o[n][2] *= alpha[1];
      o[n][3] *= alpha[1];
    }
    // ---- O += P V over the tile's 64 keys (4 steps of 16); P in [0, 1] as bf16
    // (a relative rounding of 2^-9 per weight, which the weighted sum averages;
    // the row sums l use the fp32 weights)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t ph[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float* src = sc[2 * kk + (r >> 1)] + 2 * (r & 1);   // (row, row+8) x (keys 0-7, 8-15)
        ph[r] = pack_bf16x2(src[0], src[1]);
      }
      const int vr = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;   // V row (key) this lane addresses
#pragma unroll
      for (int n2 = 0; n2 < NDT / 2; ++n2) {
        const int ch = n2 * 2 + (lane >> 4);                          // 8-dim chunk
        uint32_t vf[4];
        ldsm_x4_t(Vt + (ch >> 3) * BOX_BYTES + vr * 128 + (((ch & 7) ^ (vr & 7)) << 4), vf);
        mma_bf16_16816(o[2 * n2], ph, vf[0], vf[1]);
        mma_bf16_16816(o[2 * n2 + 1], ph, vf[2], vf[3]);
      }
    }
    __syncthreads();   // every warp is done with the slot
    if (tid == 0 && u + kPreStages < ntiles) issue(u + kPreStages);
  }
  if (u_stop < ntiles) {
    // a tile never arrived: let the copies still in flight land (bounded) before the CTA exits
    if (tid == 0)
      for (int u = u_stop; u < ntiles && u < u_stop + kPreStages; ++u)
        mbar_wait(smem_u32(&full[u % kPreStages]), (u / kPreStages) & 1, nullptr);
    __syncthreads();
    return;
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_part[r] += __shfl_xor_sync(0xffffffffu, l_part[r], 1);
    l_part[r] += __shfl_xor_sync(0xffffffffu, l_part[r], 2);
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qi = r ? r1 : r0;
    if (qi >= T) continue;
    const size_t tok = static_cast<size_t>(b) * T + qi;
    const float inv = 1.f / l_part[r];
#pragma unroll
    for (int n = 0; n < NDT; ++n) {
      const int d = n * 8 + 2 * (lane & 3);
      const float o0 = o[n][2 * r] * inv, o1 = o[n][2 * r + 1] * inv;
      if (a.o_state) *reinterpret_cast<float2*>(a.o_state + (tok * a.H + h) * HD + d) = make_float2(o0, o1);
      *reinterpret_cast<uint32_t*>(a.o_bf16 + tok * a.H * HD + static_cast<size_t>(h) * HD + d) = pack_bf16x2(o0, o1);
    }
    if ((lane & 3) == 0 && a.lse_state) a.lse_state[tok * a.H + h] = m_run[r] + logf(l_part[r]);
  }
}

// ============================================================================
// per-call token bookkeeping
// ============================================================================
__global__ void k_setup_call(int N, int mode_decode, int T, int tiles_per_seq, int q_tile,
                             const int* __restrict__ seq_len, int* seq, int* pos, int* tile, int* last,
                             int n_tiles, int* has_c, unsigned long long* stamps, int n_stamps) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (stamps)   // GEMM launch stamps of this call: starts to the largest value (atomicMin), ends to zero
    for (int i = t; i < n_stamps; i += gridDim.x * blockDim.x) {
      stamps[i] = ~0ULL;
      stamps[n_stamps + i] = 0ULL;
    }
  if (t < N) {
    if (mode_decode) {
      seq[t] = t;
      pos[t] = seq_len[t];
      tile[t] = t;
    } else {
      // a prefill chunk continues each sequence after its current length; its
      // query tiles count q_tile positions from the chunk's first token
      const int b = t / T, p = t % T;
      seq[t] = b;
      pos[t] = seq_len[b] + p;
      tile[t] = b * tiles_per_seq + p / q_tile;
    }
    last[t] = 1;
  }
  if (t < n_tiles) has_c[t] = 0;
}

__global__ void k_set_lens(int B, int* seq_len, int add) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) seq_len[b] += add;
}

__global__ void k_reset_lens(const LensArg a, int* seq_len) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < a.n) seq_len[b] = a.v[b];
}

// The state a token enters a loop with: h[r] += e (the loop embedding, when
// given) + gamma * x[r] (input injection: x is the state that entered the
// loop stack), r = idx ? idx[i] : i, for the loop's n token rows.
__global__ void __launch_bounds__(256) k_loop_input(float* __restrict__ h, const int* __restrict__ idx, int n, int d,
                                                    const float* __restrict__ e, float gamma,
                                                    const float* __restrict__ x) {
  pdl_trigger();
  pdl_wait();
  const int i = blockIdx.x;
  if (i >= n) return;
  const int r = idx ? idx[i] : i;
  float* hr = h + static_cast<size_t>(r) * d;
  const float* xr = x + static_cast<size_t>(r) * d;
  for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
    float4 v = *reinterpret_cast<const float4*>(hr + c);
    if (e) {
      const float4 ev = *reinterpret_cast<const float4*>(e + c);
      v.x += ev.x; v.y += ev.y; v.z += ev.z; v.w += ev.w;
    }
    if (gamma != 0.f) {
      const float4 xv = *reinterpret_cast<const float4*>(xr + c);
      v.x = __fmaf_rn(gamma, xv.x, v.x); v.y = __fmaf_rn(gamma, xv.y, v.y);
      v.z = __fmaf_rn(gamma, xv.z, v.z); v.w = __fmaf_rn(gamma, xv.w, v.w);
    }
    *reinterpret_cast<float4*>(hr + c) = v;
  }
}

// slot of each token in the selection (or -1), and the snapshot of selected rows
__global__ void k_after_select(const int32_t* __restrict__ idx, int n_sel, int N, int d, int* sel_slot,
                               const float* __restrict__ h, float* __restrict__ h_snap, int slot_blocks,
                               const int* seq, const int* tile, const int* last, const int* pos, SelMeta* meta) {
  pdl_trigger();
  pdl_wait();
  if (blockIdx.x == 0) {
    for (int r = threadIdx.x; r < n_sel; r += blockDim.x) {
      const int t = idx[r];
      SelMeta m;
      m.tok = t; m.seq = seq[t]; m.tile = tile[t]; m.last = last[t]; m.pos = pos[t];
      m.pad0 = m.pad1 = m.pad2 = 0;
      meta[r] = m;
    }
  }
  if (static_cast<int>(blockIdx.x) < slot_blocks) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= N) return;
    int lo = 0, hi = n_sel;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (idx[mid] < t) lo = mid + 1; else hi = mid;
    }
    sel_slot[t] = (lo < n_sel && idx[lo] == t) ? lo : -1;
    return;
  }
  const int row = blockIdx.x - slot_blocks;
  if (row >= n_sel) return;
  const float* src = h + static_cast<size_t>(idx[row]) * d;
  float* dst = h_snap + static_cast<size_t>(row) * d;
  for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4)
    *reinterpret_cast<float4*>(dst + c) = *reinterpret_cast<const float4*>(src + c);
}

// Change keys: loop 1 -> ||h - h_in||^2 for every token; loop l -> ||h - h_snap||^2
// for selected tokens and 0 for carried ones; selected tokens record last = l and
// mark their query tile as having a column set.
__global__ void __launch_bounds__(128) k_change_keys(const float* __restrict__ h, const float* __restrict__ ref,
                                                     const int* __restrict__ sel_slot, int N, int d, int loop,
                                                     float* __restrict__ key, int* last, const int* tile,
                                                     int* has_c) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x * 4 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= N) return;
  const float* other;
  if (loop == 1) {
    other = ref + static_cast<size_t>(t) * d;
  } else {
    const int s = sel_slot[t];
    if (s < 0) {
      if (lane == 0) key[t] = 0.f;
      return;
    }
    other = ref + static_cast<size_t>(s) * d;
  }
  const float* hr = h + static_cast<size_t>(t) * d;
  float acc = 0.f;
  for (int c = lane * 4; c < d; c += 128) {
    const float4 x = *reinterpret_cast<const float4*>(hr + c);
    const float4 y = *reinterpret_cast<const float4*>(other + c);
    const float a0 = x.x - y.x, a1 = x.y - y.y, a2 = x.z - y.z, a3 = x.w - y.w;
    acc += a0 * a0 + a1 * a1 + a2 * a2 + a3 * a3;
  }
  acc = warp_sum(acc);
  if (lane == 0) {
    key[t] = acc;
    if (loop > 1) {
      last[t] = loop;
      has_c[tile[t]] = 1;
    }
  }
}

// ============================================================================
// query-tile plan of a lazy loop: the selected tokens (ascending) grouped by
// query tile; tiles recomputed for the first time need a column set.
// ============================================================================
__device__ void block_plan(const int32_t* __restrict__ idx, int n_sel, const int* __restrict__ tile,
                           const int* __restrict__ has_c, const TilePlan& plan) {
  __shared__ int scan_buf[33];
  __shared__ int base_p, base_need;
  if (threadIdx.x == 0) {
    base_p = 0;
    base_need = 0;
  }
  __syncthreads();
  for (int c0 = 0; c0 < n_sel; c0 += blockDim.x) {
    const int i = c0 + threadIdx.x;
    int tl = -1, start = 0, need = 0;
    if (i < n_sel) {
      tl = tile[idx[i]];
      start = (i == 0 || tile[idx[i - 1]] != tl) ? 1 : 0;
      need = start && !has_c[tl];
    }
    int tot_p, tot_n;
    const int p = base_p + block_exclusive_scan(start, &tot_p, scan_buf);
    const int q = base_need + block_exclusive_scan(need, &tot_n, scan_buf);
    if (start) {
      plan.tile[p] = tl;
      plan.qb[p] = i;
      if (p > 0) plan.qe[p - 1] = i;
    }
    if (need) plan.need[q] = p;
    __syncthreads();
    if (threadIdx.x == 0) {
      base_p += tot_p;
      base_need += tot_n;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    if (base_p > 0) plan.qe[base_p - 1] = n_sel;
    plan.counts[0] = base_p;
    plan.counts[1] = base_need;
  }
}

__global__ void __launch_bounds__(1024) k_plan_tiles(const int32_t* __restrict__ idx, int n_sel,
                                                     const int* __restrict__ tile, const int* __restrict__ has_c,
                                                     TilePlan plan) {
  pdl_trigger();
  pdl_wait();
  block_plan(idx, n_sel, tile, has_c, plan);
}

// Sparse residual storage: the pool rows of one call token at lazy loop l, for
// every layer.  A recomputed token gets row rcount[j][l][b] + rank, rank = its
// position among the call's recomputed tokens of sequence b (they are taken in
// position order); others get -1 (zero residual).  A row beyond the pool is not
// given (-1) and kErrCapacity is recorded.  The counts grow afterwards
// (rows_advance), once every token of the call has read them.
__device__ __forceinline__ void rows_assign(const CacheView& cv, int l, int b, int p, int rank, int* status) {
  for (int j = 0; j < cv.M; ++j) {
    int r = -1;
    if (rank >= 0) {
      r = cv.rcount[(static_cast<size_t>(j) * (cv.K - 1) + (l - 2)) * cv.B + b] + rank;
      if (r >= cv.rows) {
        r = -1;
        if (status) atomicOr(status, kErrCapacity);
      }
    }
    cv.ridx[cv.ridx_index(j, l, b, p)] = r;
  }
}
__device__ __forceinline__ void rows_advance(const CacheView& cv, int l, int b, int n_b) {
  for (int j = 0; j < cv.M; ++j) {
    int* rc = cv.rcount + (static_cast<size_t>(j) * (cv.K - 1) + (l - 2)) * cv.B + b;
    *rc = min(cv.rows, *rc + n_b);
  }
}
// first index i in the ascending array v[0..n) with v[i] >= key
__device__ __forceinline__ int lower_bound_i(const int32_t* v, int n, int key) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (v[mid] < key) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// The same for calls too large for the one-CTA selection step: CTA b takes
// sequence b's call tokens [b*Tc, (b+1)*Tc), whose selection slots (-1 when not
// recomputed) are in sel_slot.
__global__ void __launch_bounds__(1024) k_assign_rows(const CacheView cv, int loop, int Tc, const int* sel_slot,
                                                      const int* pos, int* status) {
  pdl_trigger();
  pdl_wait();
  __shared__ int scan_buf[33];
  __shared__ int base;
  const int b = blockIdx.x;
  if (threadIdx.x == 0) base = 0;
  __syncthreads();
  for (int t0 = 0; t0 < Tc; t0 += blockDim.x) {
    const int t = b * Tc + t0 + threadIdx.x;
    const int sel = (t0 + threadIdx.x < Tc && sel_slot[t] >= 0) ? 1 : 0;
    int tot;
    const int rank = base + block_exclusive_scan(sel, &tot, scan_buf);
    if (t0 + threadIdx.x < Tc) rows_assign(cv, loop, b, pos[t], sel ? rank : -1, status);
    __syncthreads();
    if (threadIdx.x == 0) base += tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) rows_advance(cv, loop, b, base);
}

// After a length reset: a sequence's pool holds the rows of its positions below
// the new length, taken in position order, so its count is one past the row of
// the last recomputed position below it.  One warp per (layer, loop, sequence).
__global__ void k_reset_rows(const CacheView cv, const int* seq_len) {
  pdl_trigger();
  pdl_wait();
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  const int n_pairs = cv.M * (cv.K - 1) * cv.B;
  if (w >= n_pairs) return;
  const int b = w % cv.B, jl = w / cv.B;
  const int32_t* ri = cv.ridx + static_cast<size_t>(jl) * cv.B * cv.T + static_cast<size_t>(b) * cv.T;
  int cnt = 0;
  for (int p0 = seq_len[b] - 1; p0 >= 0; p0 -= 32) {
    const int p = p0 - lane;
    const int r = p >= 0 ? ri[p] : -1;
    const unsigned hit = __ballot_sync(0xffffffffu, r >= 0);
    if (hit) {
      const int first = __ffs(hit) - 1;   // the lane nearest the top
      cnt = __shfl_sync(0xffffffffu, r, first) + 1;
      break;
    }
  }
  if (lane == 0) cv.rcount[static_cast<size_t>(jl) * cv.B + b] = cnt;
}

// One lazy loop's token bookkeeping for a call of at most kSelectStepMax tokens
// (decode, short prefills), in one CTA: the change keys of the previous loop
// (against h_in after loop 1, against the selected rows' snapshot after a lazy
// loop, zero for carried tokens), the previously selected tokens' `last` and
// tile flags, the top-n_sel selection (or the forced one), the selection slots,
// the snapshot of the selected rows, optionally the first layer's input norm,
// and the query-tile plan.  Keys, the selection, tiles, slots and tile flags
// stay in shared memory, so the dependent steps do not go back to global memory.
__global__ void __launch_bounds__(1024) k_select_step(const SelectStepArgs a) {
  pdl_trigger();
  pdl_wait();
  __shared__ float s_key[kSelectStepMax];
  __shared__ int32_t s_idx[kSelectStepMax];
  __shared__ int s_tile[kSelectStepMax], s_slot[kSelectStepMax], s_hasc[kSelectStepMax], s_last[kSelectStepMax];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int t = threadIdx.x; t < a.N; t += blockDim.x) {
    s_tile[t] = a.tile[t];
    s_slot[t] = a.loop == 2 ? -1 : a.sel_slot[t];
    s_last[t] = a.last[t];
  }
  for (int t = threadIdx.x; t < a.n_tiles; t += blockDim.x) s_hasc[t] = a.has_c[t];
  __syncthreads();
  for (int t = warp; t < a.N; t += nw) {
    const int slot = s_slot[t];
    const float* other = a.loop == 2 ? a.h_in + static_cast<size_t>(t) * a.d
                                     : (slot >= 0 ? a.h_snap + static_cast<size_t>(slot) * a.d : nullptr);
    float acc = 0.f;
    if (other) {
      const float* hr = a.h + static_cast<size_t>(t) * a.d;
      for (int c = lane * 4; c < a.d; c += 128) {
        const float4 x = *reinterpret_cast<const float4*>(hr + c);
        const float4 y = *reinterpret_cast<const float4*>(other + c);
        const float a0 = x.x - y.x, a1 = x.y - y.y, a2 = x.z - y.z, a3 = x.w - y.w;
        acc += a0 * a0 + a1 * a1 + a2 * a2 + a3 * a3;
      }
      acc = warp_sum(acc);
    }
    if (lane == 0) {
      s_key[t] = acc;
      a.key[t] = acc;
      a.keys_trace[t] = acc;
      if (slot >= 0) {
        a.last[t] = a.loop - 1;
        s_last[t] = a.loop - 1;
        s_hasc[s_tile[t]] = 1;
        a.has_c[s_tile[t]] = 1;
      }
    }
  }
  __syncthreads();
  if (a.forced_on && (a.forced_on[0] & kForceSel)) {
    for (int i = threadIdx.x; i < a.n_sel; i += blockDim.x) s_idx[i] = a.forced[i];
  } else {
    block_topk(s_key, a.N, a.n_sel, s_idx);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < a.n_sel; i += blockDim.x) {
    const int t = s_idx[i];
    a.idx[i] = t;
    SelMeta m;
    m.tok = t; m.seq = a.seq[t]; m.tile = s_tile[t]; m.last = s_last[t]; m.pos = a.pos[t];
    m.pad0 = m.pad1 = m.pad2 = 0;
    a.meta[i] = m;
  }
  for (int t = threadIdx.x; t < a.N; t += blockDim.x) {
    const int lo = lower_bound_i(s_idx, a.n_sel, t);
    const int sl = (lo < a.n_sel && s_idx[lo] == t) ? lo : -1;
    a.sel_slot[t] = sl;
    s_slot[t] = sl;   // (the previous slots are dead after the change keys)
  }
  if (a.cv.rows) {
    // sparse residual storage: pool rows of this loop's recomputed tokens, one
    // (token, layer) per thread so the layers' counts are read in parallel
    __syncthreads();
    const int Tc = a.N / a.B_call, M = a.cv.M;
    for (int e = threadIdx.x; e < a.N * M; e += blockDim.x) {
      const int t = e % a.N, j = e / a.N, b = t / Tc, sl = s_slot[t];
      int r = -1;
      if (sl >= 0) {
        r = a.cv.rcount[(static_cast<size_t>(j) * (a.cv.K - 1) + (a.loop - 2)) * a.cv.B + b] + sl -
            lower_bound_i(s_idx, a.n_sel, b * Tc);
        if (r >= a.cv.rows) {
          r = -1;
          if (a.status) atomicOr(a.status, kErrCapacity);
        }
      }
      a.cv.ridx[a.cv.ridx_index(j, a.loop, b, a.pos[t])] = r;
    }
    __syncthreads();   // every token has read the counts
    for (int e = threadIdx.x; e < a.B_call * M; e += blockDim.x) {
      const int b = e % a.B_call, j = e / a.B_call;
      int* rc = a.cv.rcount + (static_cast<size_t>(j) * (a.cv.K - 1) + (a.loop - 2)) * a.cv.B + b;
      *rc = min(a.cv.rows, *rc + lower_bound_i(s_idx, a.n_sel, (b + 1) * Tc) - lower_bound_i(s_idx, a.n_sel, b * Tc));
    }
  }
  // snapshot of the selected rows (and, if asked, their normalised bf16 copy).
  // Work items are 512-element slices of a row, one per warp at a time; a
  // slice's loads are all issued before its stores (the snapshot may not be
  // assumed apart from h), so a row costs one memory round trip per pass.
  constexpr int SL = 512;
  const int nsl = (a.d + SL - 1) / SL;
  const bool norm = a.norm_gain != nullptr;
  float* s_ss = s_key;   // [kSelectStepMaxNorm * kSelectStepSlices]; the keys are dead after the selection
  // with at most one slice per warp the normalisation reuses the slice in registers
  const bool keep = norm && a.n_sel * nsl <= nw;
  float4 vk[SL / 128];
  for (int it = warp; it < a.n_sel * nsl; it += nw) {
    const int r = it / nsl, c0 = (it % nsl) * SL;
    const float* src = a.h + static_cast<size_t>(s_idx[r]) * a.d;
    float* dst = a.h_snap + static_cast<size_t>(r) * a.d;
    float4 v[SL / 128];
#pragma unroll
    for (int u = 0; u < SL / 128; ++u) {
      const int c = c0 + u * 128 + lane * 4;
      v[u] = c < a.d ? *reinterpret_cast<const float4*>(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < SL / 128; ++u) {
      const int c = c0 + u * 128 + lane * 4;
      if (c < a.d) *reinterpret_cast<float4*>(dst + c) = v[u];
      ss += v[u].x * v[u].x + v[u].y * v[u].y + v[u].z * v[u].z + v[u].w * v[u].w;
    }
    if (norm) {
      ss = warp_sum(ss);
      if (lane == 0) s_ss[it] = ss;
    }
    if (keep) {
#pragma unroll
      for (int u = 0; u < SL / 128; ++u) vk[u] = v[u];
    }
  }
  if (norm) {
    __syncthreads();
    for (int it = warp; it < a.x_rows * nsl; it += nw) {
      const int r = it / nsl, c0 = (it % nsl) * SL;
      uint16_t* xr = a.x + static_cast<size_t>(r) * a.d;
      if (r >= a.n_sel) {
#pragma unroll
        for (int u = 0; u < SL / 128; ++u) {
          const int c = c0 + u * 128 + lane * 4;
          if (c < a.d) *reinterpret_cast<uint2*>(xr + c) = make_uint2(0u, 0u);
        }
        continue;
      }
      float tot = 0.f;
      for (int q = 0; q < nsl; ++q) tot += s_ss[r * nsl + q];
      const float inv = rsqrtf(tot / static_cast<float>(a.d) + a.eps);
      const float* src = a.h + static_cast<size_t>(s_idx[r]) * a.d;
      float4 v[SL / 128], gv[SL / 128];
#pragma unroll
      for (int u = 0; u < SL / 128; ++u) {
        const int c = c0 + u * 128 + lane * 4;
        // keep: item it of this loop is item it of the snapshot loop, held by this warp
        v[u] = keep ? vk[u] : (c < a.d ? *reinterpret_cast<const float4*>(src + c) : make_float4(0.f, 0.f, 0.f, 0.f));
        gv[u] = c < a.d ? *reinterpret_cast<const float4*>(a.norm_gain + c) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < SL / 128; ++u) {
        const int c = c0 + u * 128 + lane * 4;
        if (c >= a.d) continue;
        const uint32_t lo =
            f_to_bf16(v[u].x * inv * gv[u].x) | (static_cast<uint32_t>(f_to_bf16(v[u].y * inv * gv[u].y)) << 16);
        const uint32_t hi =
            f_to_bf16(v[u].z * inv * gv[u].z) | (static_cast<uint32_t>(f_to_bf16(v[u].w * inv * gv[u].w)) << 16);
        *reinterpret_cast<uint2*>(xr + c) = make_uint2(lo, hi);
      }
    }
  }
  __syncthreads();
  block_plan(s_idx, a.n_sel, s_tile, s_hasc, a.plan);
}

// The column set of one (tile, KV head) row from its n <= kSelColsSmemKeys keys
// (staged in keys_sm), or the forced set: top-c by (bit pattern desc, column
// asc), ascending.  Every thread of the CTA takes part.
__device__ void select_row(const SelColsArgs& a, int seg, int g, int tl, int n, float* keys_sm) {
  int32_t* out = a.cols + ((static_cast<size_t>(a.j) * a.n_tiles + tl) * a.Hkv + g) * a.c;
  int* nout = a.ncols + (static_cast<size_t>(a.j) * a.n_tiles + tl) * a.Hkv + g;
  if (a.forced_on && (a.forced_on[0] & kForceCols)) {
    const size_t off = (static_cast<size_t>(a.j) * a.n_tiles + tl) * a.Hkv + g;
    const int fn = a.forced_ncols[off];
    for (int e = threadIdx.x; e < fn; e += blockDim.x) out[e] = a.forced_cols[off * a.c + e];
    if (threadIdx.x == 0) *nout = fn;
    return;
  }
  const float* keys = a.col_keys + (static_cast<size_t>(seg) * a.Hkv + g) * a.max_cols;
  for (int e = threadIdx.x; e < n; e += blockDim.x) keys_sm[e] = __ldcg(keys + e);
  __syncthreads();
  const int got = block_topk(keys_sm, n, a.c, out);
  if (threadIdx.x == 0) *nout = got;
}

// After a delta-score item: the CTA that wrote the last unit of its row (an
// atomic ticket over the row's units of unit_cols columns, no waiting) selects
// the row's column set, so the selection needs no launch of its own.
__device__ __forceinline__ void fold_select(const DScoreArgs& a, int seg, int g, int tl, int n, float* keys_sm,
                                            int* last_flag, int unit_cols) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int nch = (n + unit_cols - 1) / unit_cols;
    const int old = atomicAdd(&a.row_tickets[seg * a.Hkv + g], 1);
    *last_flag = old == nch - 1;
  }
  __syncthreads();
  if (!*last_flag) return;
  __threadfence();
  select_row(a.sel, seg, g, tl, n, keys_sm);
  if (threadIdx.x == 0) a.row_tickets[seg * a.Hkv + g] = 0;
  __syncthreads();
}

// ============================================================================
// delta-score column keys of tiles recomputed for the first time:
//   key[k] = max over the tile's selected queries i (with k <= pos(i)) and the
//   group's heads h of | tau*(q_l[i,h] . K_l[k] - q_last[i,h] . K_base[k]) |
// ("FlashLoop ...", abstract: the change of a query's attention output
// between loops comes from few key columns, and the same ones over loops).
// At a tile's first
// recomputation every member was last computed at loop 1, so the old keys are
// the bf16 base rows.
//
// SIMT form, for few (query, head) pairs per tile (decode: one query per tile)
// and head_dim 64 without tensor cores.  Work items are (tile, KV head, block of
// 64, 128 or 256 columns -- the largest that still gives every CTA work); each
// CTA takes a contiguous range of items, so the tile's pairs, staged in shared
// memory kDsPairs at a time, are reused while (tile, KV head) stays the same,
// and with sparse storage the item's pool rows of every level are staged
// first, so each step needs one memory round trip.  The key is evaluated as
// (q_l - q_last) . K_base + q_l . R, R = K_l - K_base = the residual sum: the
// queries' difference is formed in fp32 when staged, and a column without
// residual rows (most of them) costs one product per pair.  A quad of lanes owns one
// column: lane qd of the quad holds dims [qd*HD/4, (qd+1)*HD/4) of K_l and
// K_base, all of whose loads (index rows first with sparse storage, then base,
// codes and scales of every level) are issued before any is used; the quad's
// partial dot products meet in two shuffles.
// ============================================================================
constexpr int kDsBlock = 256;   // largest columns per work item
constexpr int kDsPairs = 8;     // (query, head) pairs held in registers per pass

template <int HD, int KM, bool SP>
__global__ void __launch_bounds__(256, 2) k_dscore(const DScoreArgs a) {
  pdl_trigger();
  pdl_wait();
  constexpr int DPL = HD / 4;              // dims per lane
  constexpr int QS = DPL + 4;              // padded stride of one lane-quarter of a staged query row
  extern __shared__ __align__(16) uint8_t sm[];
  float* qn_sm = reinterpret_cast<float*>(sm);       // [kDsPairs][4][QS]: tau * q_l
  float* qo_sm = qn_sm + kDsPairs * 4 * QS;           // [kDsPairs][4][QS]: tau * (q_l - q_last)
  // each warp's base rows of its 8 columns, double-buffered: [warps][2][8][HD] bf16
  constexpr int WBUF = 2 * 8 * HD * 2;
  uint8_t* wbuf_all = sm + 2 * kDsPairs * 4 * QS * 4;
  __shared__ int qpos_sm[kDsPairs], qtok_sm[kDsPairs], qi_sm[kDsPairs];
  __shared__ float best_sm[kDsBlock];            // the item's column keys so far (one owner quad per column)
  __shared__ int rows_sm[SP ? (KM - 1) * kDsBlock : 1];   // sparse storage: pool rows of the item's columns
  __shared__ int fold_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qd = lane & 3, col_in_warp = lane >> 2;
  const int grp = a.H / a.Hkv;
  const int blk_cols = a.ds_block, nsteps = blk_cols / 64;   // columns per item (64, 128 or 256)
  const int nblk = (a.max_cols + blk_cols - 1) / blk_cols;
  const int cnt = a.plan.counts[1];
  const CacheView& cv = a.cv;
  const int bits = cv.bits, gi = (qd * DPL) >> cv.lg;
  const size_t rb = cv.row_bytes_codes(), ns = cv.hd >> cv.lg;
  // each CTA takes a contiguous range of items, so consecutive items mostly
  // share (tile, KV head) and their staged pairs are reused
  const int total = cnt * a.Hkv * nblk, per_cta = (total + gridDim.x - 1) / gridDim.x;
  const int it_end = min(total, (blockIdx.x + 1) * per_cta);
  int staged = -1;
  for (int it = blockIdx.x * per_cta; it < it_end; ++it) {
    const int seg = it / (a.Hkv * nblk), g = (it / nblk) % a.Hkv, blk = it % nblk;
    const int p = a.plan.need[seg];
    const int qb = a.plan.qb[p], qe = a.plan.qe[p];
    const SelMeta ml = a.meta[qe - 1];
    const int b = ml.seq, maxpos = ml.pos;
    const int c0 = blk * blk_cols;
    if (c0 > maxpos) continue;   // (uniform over the CTA)
    const int npairs = (qe - qb) * grp;
    const bool one_group = npairs <= kDsPairs;
    // every column of the item: this warp's 8 columns per step, nsteps steps
    for (int pb = 0; pb < npairs; pb += kDsPairs) {
      const int np = min(kDsPairs, npairs - pb);
      __syncthreads();   // the previous pairs (and the previous item's keys) are no longer read
      if (pb == 0) {
        best_sm[tid] = 0.f;
        if (SP)
          for (int e = tid; e < (KM - 1) * blk_cols; e += blockDim.x) {
            const int q = e / blk_cols, k = e % blk_cols, col = c0 + k;
            rows_sm[q * kDsBlock + k] =
                (col <= maxpos && q + 2 <= a.loop) ? cv.ridx[cv.ridx_index(a.j, q + 2, b, col)] : -1;
          }
      }
      const int key = seg * a.Hkv + g;
      if (!(one_group && staged == key)) {
        // the pairs' slots first, then every query element with its address known
        if (tid < kDsPairs) {
          const int pr = tid;
          if (pr < np) {
            const int qi = qb + (pb + pr) / grp;
            const SelMeta mq = a.meta[qi];
            qi_sm[pr] = qi;
            qtok_sm[pr] = mq.tok;
            qpos_sm[pr] = mq.pos;
          } else {
            qi_sm[pr] = qtok_sm[pr] = 0;
            qpos_sm[pr] = -1;
          }
        }
        __syncthreads();
#pragma unroll 4
        for (int e = tid; e < kDsPairs * HD; e += blockDim.x) {
          const int pr = e / HD, dd = e % HD;
          float vn = 0.f, vo = 0.f;
          if (pr < np) {
            const int hh = g * grp + (pb + pr) % grp;
            const float xn = a.q_cur[(static_cast<size_t>(qi_sm[pr]) * a.H + hh) * HD + dd];
            vn = a.tau * xn;
            vo = a.tau * (xn - a.q_last[(static_cast<size_t>(qtok_sm[pr]) * a.H + hh) * HD + dd]);
          }
          const int o = (pr * 4 + dd / DPL) * QS + dd % DPL;
          qn_sm[o] = vn;
          qo_sm[o] = vo;
        }
        staged = one_group ? key : -1;
      }
      __syncthreads();
      // the base rows of this warp's 8 columns of step s, copied into its buffer
      // s & 1 (columns past the last eligible one read zero); step s + 1's copy
      // is in flight while step s is computed
      uint8_t* wbuf = wbuf_all + warp * WBUF;
      auto issue_cols = [&](int st) {
        const int cb = c0 + st * 64 + warp * 8;
        const uint32_t dst = smem_u32(wbuf + (st & 1) * (WBUF / 2));
        constexpr int PR = HD * 2 / 16;   // 16-byte pieces per row
#pragma unroll
        for (int k = lane; k < 8 * PR; k += 32) {
          const int r = k / PR, pc = k % PR, cc = cb + r;
          const bool ok = cc <= maxpos;
          cp_async16(dst + k * 16, cv.base_row(a.j, 0, b, g, ok ? cc : c0) + pc * 8, ok ? 16u : 0u);
        }
        cp_async_commit();
      };
      issue_cols(0);
#pragma unroll 1
      for (int s = 0; s < nsteps; ++s) {
        const int col = c0 + s * 64 + warp * 8 + col_in_warp;
        const bool valid = col <= maxpos;
        if (s + 1 < nsteps) {
          issue_cols(s + 1);
          cp_async_wait<1>();
        } else {
          cp_async_wait<0>();
        }
        __syncwarp();   // every lane's copies of step s are visible to the warp
        // ---- base dims of this lane from the buffer, then every level's codes and scale
        uint4 braw[DPL / 8];
        uint4 craw[KM - 1];
        uint16_t sraw[KM - 1];
        {
          const uint4* br = reinterpret_cast<const uint4*>(wbuf + (s & 1) * (WBUF / 2) + col_in_warp * HD * 2 +
                                                           qd * DPL * 2);
#pragma unroll
          for (int u = 0; u < DPL / 8; ++u) braw[u] = br[u];
        }
        int rr[KM - 1];
#pragma unroll
        for (int q = 0; q < KM - 1; ++q)
          rr[q] = SP ? rows_sm[q * kDsBlock + (col - c0)] : ((valid && q + 2 <= a.loop) ? col : -1);
        const size_t step = static_cast<size_t>(2) * cv.B * cv.Hkv * (SP ? cv.rows : cv.T);
        const size_t q0 = ((((static_cast<size_t>(a.j) * (cv.K - 1)) * 2) * cv.B + b) * cv.Hkv + g) *
                          static_cast<size_t>(SP ? cv.rows : cv.T);
#pragma unroll
        for (int q = 0; q < KM - 1; ++q) {
          craw[q] = make_uint4(0u, 0u, 0u, 0u);
          sraw[q] = 0;
          if (rr[q] >= 0) {
            const size_t ri = q0 + q * step + static_cast<size_t>(rr[q]);
            const int nb = DPL * bits / 8;   // code bytes of this lane's dims: 16, 8 or 4
            const uint8_t* row = cv.codes + ri * rb + qd * nb;
            if (nb == 16) {
              craw[q] = *reinterpret_cast<const uint4*>(row);
            } else if (nb == 8) {
              const uint2 v = *reinterpret_cast<const uint2*>(row);
              craw[q].x = v.x;
              craw[q].y = v.y;
            } else {
              craw[q].x = *reinterpret_cast<const uint32_t*>(row);
            }
            sraw[q] = cv.scales[ri * ns + gi];
          }
        }
        // ---- the key through (q_l - q_last) . K_base + q_l . R, R = the sum of
        // code * scale of loops 2..l in loop order (fp32): one product per pair
        // for a column without residual rows, two with
        float kb[DPL], rs[DPL];
        bool has_r = false;
#pragma unroll
        for (int q = 0; q < KM - 1; ++q) has_r = has_r || (q + 2 <= a.loop && rr[q] >= 0);
#pragma unroll
        for (int u = 0; u < DPL / 8; ++u) {
          const uint32_t w[4] = {braw[u].x, braw[u].y, braw[u].z, braw[u].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            kb[u * 8 + 2 * k] = bf16_to_f(w[k] & 0xFFFF);
            kb[u * 8 + 2 * k + 1] = bf16_to_f(w[k] >> 16);
          }
        }
#pragma unroll
        for (int e = 0; e < DPL; ++e) rs[e] = 0.f;
        if (has_r) {
#pragma unroll
          for (int q = 0; q < KM - 1; ++q) {
            if (q + 2 > a.loop) break;
            const float sc = half_bits_to_f(sraw[q]);
            const uint32_t w[4] = {craw[q].x, craw[q].y, craw[q].z, craw[q].w};
            if (bits == 4) {   // element e: nibble e % 8 of word e / 8 (low nibble first)
#pragma unroll
              for (int e = 0; e < DPL; ++e) {
                const int c = sext(static_cast<int>((w[e / 8] >> ((e % 8) * 4)) & 0xFu), 4);
                rs[e] = __fadd_rn(rs[e], __fmul_rn(static_cast<float>(c), sc));
              }
            } else {           // element e: bits 2(e % 16) of word e / 16 (LSB first)
#pragma unroll
              for (int e = 0; e < DPL; ++e) {
                const int c = sext(static_cast<int>((w[e / 16] >> ((e % 16) * 2)) & 0x3u), 2);
                rs[e] = __fadd_rn(rs[e], __fmul_rn(static_cast<float>(c), sc));
              }
            }
          }
        }
        // ---- partial dot products of this lane's dims, one pair at a time
        float m = 0.f;
#pragma unroll 1
        for (int pr = 0; pr < np; ++pr) {
          const float* qn = qn_sm + (pr * 4 + qd) * QS;
          const float* qdl = qo_sm + (pr * 4 + qd) * QS;
          float dd = 0.f, dr = 0.f;
#pragma unroll
          for (int e = 0; e < DPL; e += 4) {
            const float4 y = *reinterpret_cast<const float4*>(qdl + e);
            dd += kb[e] * y.x + kb[e + 1] * y.y + kb[e + 2] * y.z + kb[e + 3] * y.w;
          }
          if (has_r) {
#pragma unroll
            for (int e = 0; e < DPL; e += 4) {
              const float4 x = *reinterpret_cast<const float4*>(qn + e);
              dr += rs[e] * x.x + rs[e + 1] * x.y + rs[e + 2] * x.z + rs[e + 3] * x.w;
            }
          }
          float d = dd + dr;
          d += __shfl_xor_sync(0xffffffffu, d, 1);
          d += __shfl_xor_sync(0xffffffffu, d, 2);
          if (col <= qpos_sm[pr]) m = fmaxf(m, fabsf(d));
        }
        const int slot = s * 64 + warp * 8 + col_in_warp;
        if (qd == 0) best_sm[slot] = fmaxf(best_sm[slot], m);
        __syncwarp();   // buffer s & 1 is read before step s + 2's copy reuses it
      }
    }
    // ---- this item's keys (each written by the lane that owns the column)
    for (int s = 0; s < nsteps; ++s) {
      const int slot = s * 64 + warp * 8 + col_in_warp, col = c0 + slot;
      if (qd == 0 && col <= maxpos) {
        const float v = best_sm[slot];
        a.col_keys[(static_cast<size_t>(seg) * a.Hkv + g) * a.max_cols + col] = v;
        const int tl = a.plan.tile[p];
        if (a.trace_ck && tl < a.trace_tiles)
          a.trace_ck[((static_cast<size_t>(a.j) * a.trace_tiles + tl) * a.Hkv + g) * a.max_cols + col] = v;
      }
    }
    if (a.fold) {
      __syncthreads();   // the staged pairs are dead; the fold reuses the shared memory
      fold_select(a, seg, g, a.plan.tile[p], maxpos + 1, reinterpret_cast<float*>(sm), &fold_last, blk_cols);
    }
  }
}

// ============================================================================
// delta-score column keys of prefill tiles on the tensor cores.  The same keys
// as k_dscore -- key[k] = max over the tile's selected queries (k <= their
// position) and the group's heads of |tau (q_l . K_l[k] - q_last . K_base[k])|
// -- evaluated through the identity
//   q_l . K_l - q_last . K_base = (q_l - q_last) . K_base + q_l . R,
// R = K_l - K_base = the sum of code * scale of loops 2..l (fp32, loop order):
// the difference of the queries is formed in fp32 before it is rounded, so two
// single bf16 products with fp32 accumulation (K_base is bf16 exactly; R is
// small) keep the key accurate where the direct form would cancel two large
// terms.  (At a tile's first recomputation every member was last computed at
// loop 1, so the old keys are the base rows.)
//
// Work items are (tile, KV head, unit of kDsTcUnit 64-column chunks), taken
// grid-stride, two CTAs per SM.  Per item and per pass of 64 (query, head)
// pairs, the pairs are staged once in shared memory as two bf16 operand tiles
// (tau (q_l - q_last), tau q_l); the unit's chunks then stream through: the
// base rows of chunk c + 1 are copied (cp.async, 128-byte swizzle) while chunk
// c's residual tile is built (codes loaded before the copy is awaited) and
// multiplied.  Warp w takes pair rows 16 (w % 4) .. +15 against columns
// 32 (w / 4) .. +31 of the chunk; the column maxima meet in shared memory (max
// of non-negative floats = max of their bit patterns, in any order).
// ============================================================================
constexpr int kDsTcUnit = 4;   // 64-column chunks per work item

// Dynamic work distribution: CTAs take items from a counter, so CTAs that drew
// cheap or empty items take more; the last CTA to finish resets the counter
// for the next launch.  (Items are numbered heaviest first by the callers.)
__device__ __forceinline__ int next_item(int* work, int* s_item) {
  __syncthreads();   // every thread has read the previous item
  if (threadIdx.x == 0) *s_item = atomicAdd(&work[0], 1);
  __syncthreads();
  return *s_item;
}
__device__ __forceinline__ void finish_items(int* work) {
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&work[1], 1) == static_cast<int>(gridDim.x) - 1) {
      work[0] = 0;
      work[1] = 0;
    }
  }
}

__device__ __forceinline__ uint32_t swz128(int row, int piece) {   // 16-byte piece of a 64 x 128-dim bf16 tile
  return static_cast<uint32_t>((piece >> 3) * (64 * 128) + row * 128 + (((piece & 7) ^ (row & 7)) << 4));
}

template <int KM, bool SP>
__global__ void __launch_bounds__(256, 2) k_dscore_tc(const DScoreArgs a) {
  constexpr int HD = 128, TILE = 2 * 64 * 128, KS = HD / 16, UC = kDsTcUnit;
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint8_t sm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qt = sm;                    // [2][TILE]: tau (q_l - q_last), tau q_l (64 pair rows)
  uint8_t* kbs = sm + 2 * TILE;        // [2][TILE]: base rows of the chunk (double-buffered)
  uint8_t* krs = sm + 4 * TILE;        // the chunk's residual sums R
  __shared__ unsigned colmax[UC * 64];
  __shared__ int qpos[64];
  __shared__ int fold_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rg = warp & 3, ch2 = warp >> 2;   // pair-row group, column half
  const int grp = a.H / a.Hkv;
  const int cnt = a.plan.counts[1];
  const int nunit = (a.max_chunks + UC - 1) / UC;
  const CacheView& cv = a.cv;
  const int bits = cv.bits;
  const size_t rb = cv.row_bytes_codes(), ns = cv.hd >> cv.lg;
  const size_t step = static_cast<size_t>(2) * cv.B * cv.Hkv * (SP ? cv.rows : cv.T);
  const uint32_t qt_s = smem_u32(qt), kbs_s = smem_u32(kbs), krs_s = smem_u32(krs);
  __shared__ int s_item;
  for (;;) {
    const int it = next_item(a.work, &s_item);
    if (it >= cnt * a.Hkv * nunit) break;
    // the longest rows (the last plan entries: the latest tiles) first
    const int seg = cnt - 1 - it / (a.Hkv * nunit), g = (it / nunit) % a.Hkv, unit = it % nunit;
    const int p = a.plan.need[seg];
    const int qb = a.plan.qb[p], qe = a.plan.qe[p];
    const SelMeta ml = a.meta[qe - 1];
    const int b = ml.seq, maxpos = ml.pos;
    const int u0 = unit * UC * 64;
    if (u0 > maxpos) continue;   // (uniform over the CTA)
    const int nch = min(UC, (maxpos - u0) / 64 + 1);
    const size_t q0 = ((((static_cast<size_t>(a.j) * (cv.K - 1)) * 2) * cv.B + b) * cv.Hkv + g) *
                      static_cast<size_t>(SP ? cv.rows : cv.T);
    const int npairs = (qe - qb) * grp;
    // copy the base rows of chunk c (rows past the last eligible column read zero)
    auto issue_base = [&](int c) {
      const int c0 = u0 + c * 64;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = tid + 256 * u, r = e >> 4, pc = e & 15;
        const bool ok = c0 + r <= maxpos;
        const uint16_t* src = cv.base_row(a.j, 0, b, g, ok ? c0 + r : c0) + pc * 8;
        cp_async16(kbs_s + (c & 1) * TILE + swz128(r, pc), src, ok ? 16u : 0u);
      }
      cp_async_commit();
    };
    for (int pb = 0; pb < npairs; pb += 64) {
      __syncthreads();   // the previous pass (or item, or fold) no longer reads shared memory
      // ---- the pass's pairs as operand tiles: thread -> (pair row, 8-dim piece) x 4
#pragma unroll 1
      for (int u = 0; u < 4; ++u) {
        const int e = tid + 256 * u, r = e >> 4, pc = e & 15;
        const int pr = pb + r;
        float xn[8], xo[8];
        if (pr < npairs) {
          const int qi = qb + pr / grp, hh = g * grp + pr % grp;
          const SelMeta mq = a.meta[qi];
          const float4* qn = reinterpret_cast<const float4*>(a.q_cur + (static_cast<size_t>(qi) * a.H + hh) * HD) + pc * 2;
          const float4* qo = reinterpret_cast<const float4*>(a.q_last + (static_cast<size_t>(mq.tok) * a.H + hh) * HD) + pc * 2;
          const float4 n0 = qn[0], n1 = qn[1], o0 = qo[0], o1 = qo[1];
          xn[0] = n0.x; xn[1] = n0.y; xn[2] = n0.z; xn[3] = n0.w; xn[4] = n1.x; xn[5] = n1.y; xn[6] = n1.z; xn[7] = n1.w;
          xo[0] = o0.x; xo[1] = o0.y; xo[2] = o0.z; xo[3] = o0.w; xo[4] = o1.x; xo[5] = o1.y; xo[6] = o1.z; xo[7] = o1.w;
          if (pc == 0) qpos[r] = mq.pos;
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) xn[k] = xo[k] = 0.f;
          if (pc == 0) qpos[r] = -1;
        }
        uint32_t wd[4], wn[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          wd[k] = pack_bf16x2(a.tau * (xn[2 * k] - xo[2 * k]), a.tau * (xn[2 * k + 1] - xo[2 * k + 1]));
          wn[k] = pack_bf16x2(a.tau * xn[2 * k], a.tau * xn[2 * k + 1]);
        }
        const uint32_t o = swz128(r, pc);
        *reinterpret_cast<uint4*>(qt + o) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        *reinterpret_cast<uint4*>(qt + TILE + o) = make_uint4(wn[0], wn[1], wn[2], wn[3]);
      }
      if (pb == 0) colmax[tid] = 0u;   // UC * 64 == 256 == blockDim.x
      issue_base(0);
      const bool rows_active = pb + 16 * rg < npairs;   // this warp's pair rows hold any pair
      for (int c = 0; c < nch; ++c) {
        const int c0 = u0 + c * 64;
        // residual codes of this chunk's rows (loads issued before the copy is awaited)
        uint32_t craw[4][KM - 1];
        uint16_t sraw[4][KM - 1];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = tid + 256 * u, r = e >> 4, pc = e & 15;
          const int t = c0 + r;
          int rr[KM - 1];
#pragma unroll
          for (int q = 0; q < KM - 1; ++q) rr[q] = (t <= maxpos && q + 2 <= a.loop) ? (SP ? 0 : t) : -1;
          if (SP && t <= maxpos) chain_rows<KM>(cv, a.j, b, t, a.loop, rr);
#pragma unroll
          for (int q = 0; q < KM - 1; ++q) {
            craw[u][q] = 0u;
            sraw[u][q] = 0;
            if (rr[q] >= 0) {
              const size_t ri = q0 + q * step + static_cast<size_t>(rr[q]);
              const uint8_t* row = cv.codes + ri * rb;
              craw[u][q] = bits == 4 ? *reinterpret_cast<const uint32_t*>(row + pc * 4)
                                     : static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(row + pc * 2));
              sraw[u][q] = cv.scales[ri * ns + ((pc * 8) >> cv.lg)];
            }
          }
        }
        cp_async_wait<0>();
        __syncthreads();   // chunk c's base rows are in; every warp is done with chunk c - 1
        if (c + 1 < nch) issue_base(c + 1);   // into the buffer chunk c - 1 used
        // ---- R = code * scale of loops 2..l summed in loop order (fp32), as bf16
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int e = tid + 256 * u, r = e >> 4, pc = e & 15;
          float x[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) x[k] = 0.f;
#pragma unroll
          for (int q = 0; q < KM - 1; ++q) {
            if (q + 2 > a.loop) break;
            const float sc = half_bits_to_f(sraw[u][q]);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int cd = bits == 4 ? sext(static_cast<int>((craw[u][q] >> (4 * k)) & 0xFu), 4)
                                       : sext(static_cast<int>((craw[u][q] >> (2 * k)) & 0x3u), 2);
              x[k] = __fadd_rn(x[k], __fmul_rn(static_cast<float>(cd), sc));
            }
          }
          uint32_t w[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) w[k] = pack_bf16x2(x[2 * k], x[2 * k + 1]);
          *reinterpret_cast<uint4*>(krs + swz128(r, pc)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        __syncthreads();
        if (rows_active) {
          float acc[4][4];
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            uint32_t ad[4], an[4];
            const uint32_t qo_ = swz128(16 * rg + (lane & 15), 2 * ks + (lane >> 4));
            ldsm_x4(qt_s + qo_, ad);
            ldsm_x4(qt_s + TILE + qo_, an);
#pragma unroll
            for (int np = 0; np < 2; ++np) {
              const int key = 32 * ch2 + np * 16 + (lane & 7) + ((lane >> 4) << 3);
              const uint32_t ko = swz128(key, 2 * ks + ((lane >> 3) & 1));
              uint32_t fb[4], fr[4];
              ldsm_x4(kbs_s + (c & 1) * TILE + ko, fb);
              ldsm_x4(krs_s + ko, fr);
#pragma unroll
              for (int hlf = 0; hlf < 2; ++hlf) {
                float* d = acc[2 * np + hlf];
                mma_bf16_16816(d, ad, fb[2 * hlf], fb[2 * hlf + 1]);
                mma_bf16_16816(d, an, fr[2 * hlf], fr[2 * hlf + 1]);
              }
            }
          }
          // |delta| of causal columns, max over this warp's rows, then over the CTA
          const int p0 = qpos[16 * rg + (lane >> 2)], p1 = qpos[16 * rg + (lane >> 2) + 8];
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int col = 32 * ch2 + nt * 8 + 2 * (lane & 3) + e;
              float m = 0.f;
              if (c0 + col <= p0) m = fmaxf(m, fabsf(acc[nt][e]));
              if (c0 + col <= p1) m = fmaxf(m, fabsf(acc[nt][2 + e]));
              m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
              m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
              m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
              if (lane < 4 && m > 0.f) atomicMax(&colmax[c * 64 + col], __float_as_uint(m));
            }
          }
        }
      }
    }
    __syncthreads();
    {
      const int col = u0 + tid;
      if (col <= maxpos) {
        const float v = __uint_as_float(colmax[tid]);
        a.col_keys[(static_cast<size_t>(seg) * a.Hkv + g) * a.max_cols + col] = v;
        const int tl = a.plan.tile[p];
        if (a.trace_ck && tl < a.trace_tiles)
          a.trace_ck[((static_cast<size_t>(a.j) * a.trace_tiles + tl) * a.Hkv + g) * a.max_cols + col] = v;
      }
    }
    if (a.fold) fold_select(a, seg, g, a.plan.tile[p], maxpos + 1, reinterpret_cast<float*>(sm), &fold_last, UC * 64);
  }
  finish_items(a.work);
}

// top-c columns of each (tile, KV head) that needs a column set.  A row of n
// keys is split into slices of kSelColsSmemKeys (grid.y); the radix passes read
// every key several times, so each slice is staged in shared memory once.  One
// slice: its top-c is the answer.  Several: each slice writes its own top-c
// (keys and ascending column ids) as candidates, and the last slice CTA of the
// row (an atomic ticket, no waiting) takes the top-c of the candidates, laid
// out in ascending column order: every member of the row's top-c is in its
// slice's top-c, and equal keys still go to the lower column.
__global__ void __launch_bounds__(1024) k_select_cols(const SelColsArgs a) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float keys_sm[];   // [kSelColsSmemKeys]
  __shared__ int last_cta;
  const int seg = blockIdx.x / a.Hkv, g = blockIdx.x % a.Hkv, sl = blockIdx.y;
  const int cnt = a.plan.counts[1], p = a.plan.need[seg];   // requested together
  if (seg >= cnt) return;
  const int tl = a.plan.tile[p];
  const int n = a.meta[a.plan.qe[p] - 1].pos + 1;
  const int slices = select_cols_slices(n);
  if (sl >= slices) return;
  int32_t* out = a.cols + ((static_cast<size_t>(a.j) * a.n_tiles + tl) * a.Hkv + g) * a.c;
  int* nout = a.ncols + (static_cast<size_t>(a.j) * a.n_tiles + tl) * a.Hkv + g;
  if (a.forced_on && (a.forced_on[0] & kForceCols)) {
    if (sl != 0) return;
    const size_t off = (static_cast<size_t>(a.j) * a.n_tiles + tl) * a.Hkv + g;
    const int fn = a.forced_ncols[off];
    for (int e = threadIdx.x; e < fn; e += blockDim.x) out[e] = a.forced_cols[off * a.c + e];
    if (threadIdx.x == 0) *nout = fn;
    return;
  }
  const float* keys = a.col_keys + (static_cast<size_t>(seg) * a.Hkv + g) * a.max_cols;
  if (slices == 1) {
    select_row(a, seg, g, tl, n, keys_sm);
    return;
  }
  // this slice's own top-c, as candidates
  const int k0 = sl * kSelColsSmemKeys, ns = min(kSelColsSmemKeys, n - k0);
  const size_t row = static_cast<size_t>(seg) * a.Hkv + g;
  float* ck = a.cand_keys + (row * a.max_slices + sl) * a.c;
  int32_t* ci = a.cand_idx + (row * a.max_slices + sl) * a.c;
  stage_keys(keys + k0, ns, keys_sm);
  const int kept = block_topk(keys_sm, ns, a.c, ci);   // slice positions, ascending
  for (int e = threadIdx.x; e < kept; e += blockDim.x) {
    const int q = ci[e];
    ck[e] = keys_sm[q];
    ci[e] = k0 + q;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int old = atomicAdd(&a.cand_counters[row], 1);
    last_cta = old == slices - 1;
  }
  __syncthreads();
  if (!last_cta) return;
  __threadfence();
  // the union, in slice order (= ascending column ids): every slice but the
  // last kept c candidates (c < kSelColsSmemKeys), so the union is contiguous
  const float* cand = a.cand_keys + row * a.max_slices * a.c;
  const int m = (slices - 1) * a.c + min(a.c, n - (slices - 1) * kSelColsSmemKeys);
  const float* src = cand;
  if (m <= kSelColsSmemKeys) {
    for (int e = threadIdx.x; e < m; e += blockDim.x) keys_sm[e] = __ldcg(cand + e);
    __syncthreads();
    src = keys_sm;
  }
  const int got = block_topk(src, m, a.c, out);   // positions among the candidates, ascending
  // map positions to column ids (out is rewritten in place, in chunks of 1024)
  for (int e0 = 0; e0 < got; e0 += 1024) {
    const int e = e0 + threadIdx.x;
    int col = 0;
    if (e < got) col = __ldcg(a.cand_idx + row * a.max_slices * a.c + out[e]);
    __syncthreads();
    if (e < got) out[e] = col;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    *nout = got;
    a.cand_counters[row] = 0;
  }
}

// ============================================================================
// sparse-column correction of one selected query and KV group.  With
// s_new = tau q_l.K_l and s_old = tau q_last.K_last over the query's columns C
// (k <= pos), the corrected denominator and numerator are
//   Z' = e^(lse-Mx) - sum_C e^(s_old-Mx) + sum_C e^(s_new-Mx)
//   N' = e^(lse-Mx) O - sum_C e^(s_old-Mx) V_last + sum_C e^(s_new-Mx) V_l
// and O = N'/Z'.  The first two terms -- the attention over the columns outside
// C, "the rest" -- do not change while C is fixed, so they are formed once, at
// the token's first recomputation (last = 1: the stored state is the loop-1
// attention (O, lse), and K_last, V_last are the base rows), and kept as
// (M_r, Z_r, N_r) in (lse_state, z_state, o_state).  At every later
// recomputation Z' = e^(M_r-Mx) Z_r + sum_C e^(s_new-Mx) and N' likewise, so the
// old chains are never rebuilt again.  This is the same sum as the step-by-step
// update (the old term of loop l is the new term of the token's previous
// recomputation, with the same C); it is only grouped differently.  q_last
// therefore stays the loop-1 query, which is what the delta scores of a tile's
// first recomputation read.  A non-positive Z' is reported as non-finite.
// ============================================================================
// The EPL base (bf16) values of one row held by a lane.
template <int EPL>
__device__ __forceinline__ void base_lane(const uint16_t* row, int lane, float* out) {
  if (EPL == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(row + lane * 4);
    out[0] = bf16_to_f(u.x & 0xFFFF);
    out[1] = bf16_to_f(u.x >> 16);
    out[EPL == 4 ? 2 : 0] = bf16_to_f(u.y & 0xFFFF);
    out[EPL == 4 ? 3 : 1] = bf16_to_f(u.y >> 16);
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(row + lane * 2);
    out[0] = bf16_to_f(u & 0xFFFF);
    out[1] = bf16_to_f(u >> 16);
  }
}
// One column of the running sums (per head: max m, then e^(s - m)-weighted
// denominators and numerators, rescaled when m grows): the new term only ...
template <int EPL, int GRP>
__device__ __forceinline__ void corr_new(const float (&qn)[GRP][EPL], const float* khi, const float* vhi, float tau,
                                         float (&m)[GRP], float (&zn)[GRP], float (&an)[GRP][EPL]) {
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    float dn = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) dn += qn[h][e] * khi[e];
    dn = warp_sum(dn) * tau;
    const float mn = fmaxf(m[h], dn);
    const float sc = m[h] == -INFINITY ? 0.f : expf(m[h] - mn);
    const float en = expf(dn - mn);
    zn[h] = zn[h] * sc + en;
#pragma unroll
    for (int e = 0; e < EPL; ++e) an[h][e] = an[h][e] * sc + en * vhi[e];
    m[h] = mn;
  }
}
// ... or the new and the old terms, with one running max per head
template <int EPL, int GRP>
__device__ __forceinline__ void corr_both(const float (&qn)[GRP][EPL], const float (&qo)[GRP][EPL],
                                          const float* klo, const float* khi, const float* vlo, const float* vhi,
                                          float tau, float (&m)[GRP], float (&zn)[GRP], float (&an)[GRP][EPL],
                                          float (&zo)[GRP], float (&ao)[GRP][EPL]) {
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    float dn = 0.f, dl = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      dn += qn[h][e] * khi[e];
      dl += qo[h][e] * klo[e];
    }
    dn = warp_sum(dn) * tau;
    dl = warp_sum(dl) * tau;
    const float mn = fmaxf(m[h], fmaxf(dn, dl));
    const float sc = m[h] == -INFINITY ? 0.f : expf(m[h] - mn);
    const float en = expf(dn - mn), eo = expf(dl - mn);
    zn[h] = zn[h] * sc + en;
    zo[h] = zo[h] * sc + eo;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      an[h][e] = an[h][e] * sc + en * vhi[e];
      ao[h][e] = ao[h][e] * sc + eo * vlo[e];
    }
    m[h] = mn;
  }
}

// The state update of one output element (head h, dim dd) from the merged
// pieces -- the new-term denominator zn and numerator nn relative to their
// maximum Mn, the old-term ones (zo, no) relative to Mo -- and the stored
// state, read before any of it is rewritten: on a first recomputation
// (Ls, O) = the loop-1 (lse, O) element, otherwise (Ls, Zs, O) = the rest
// (M_r, Z_r, N_r).  Returns the corrected output; on a first recomputation
// also sets the rest to store.
struct CorrRest {
  float m, z, n;
};
__device__ __forceinline__ float corr_finish(bool first, float Mn, float zn, float nn, float Mo, float zo, float no,
                                             float Ls, float Zs, float O, CorrRest& rest, int* status) {
  float Mr, Zr, Nr;
  if (first) {   // remove the loop-1 terms of C from the loop-1 attention
    Mr = fmaxf(Ls, Mo);
    const float es = expf(Ls - Mr), eo = Mo == -INFINITY ? 0.f : expf(Mo - Mr);
    Zr = es - eo * zo;
    Nr = es * O - eo * no;
    rest.m = Mr;
    rest.z = Zr;
    rest.n = Nr;
  } else {       // the stored rest
    Mr = Ls;
    Zr = Zs;
    Nr = O;
  }
  const float M = fmaxf(Mr, Mn);
  const float er = expf(Mr - M), en = Mn == -INFINITY ? 0.f : expf(Mn - M);
  const float Z = er * Zr + en * zn;
  if (!(Z > 0.f) && status) atomicOr(status, kErrNonfinite);
  return (er * Nr + en * nn) / Z;
}

// The general form (prefill; decode with the ticket merge).  The column set is
// split across CTAs (grid.y); each warp takes one column at a time and keeps a
// running per-head maximum, so the sums are accumulated in pieces that are
// rescaled to the common maximum when merged.  The last CTA of a (query,
// group) -- an atomic ticket, no waiting -- merges the pieces with the stored
// state.  Partials: part_acc [rows][2][8][hd] (new, old), part_mz [rows][8][3]
// (max, new denominator, old denominator).
template <int HD, int EPL, int GRP, int KM, bool SP>
__global__ void __launch_bounds__(256) k_correct(const CorrectArgs a) {
  pdl_trigger();
  pdl_wait();
  constexpr int GMAX = 8, NW = 8;
  __shared__ float sm_m[NW][GMAX], sm_zn[NW][GMAX], sm_zo[NW][GMAX];
  __shared__ float sm_acc[NW][GRP][HD];   // the warps' numerators: new term, then (first recomputation) old
  __shared__ int ncs, is_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int i = blockIdx.x / a.Hkv, g = blockIdx.x % a.Hkv, sp = blockIdx.y;
  constexpr int grp = GRP;
  const int tok = a.idx[i];
  const int b = a.seq[tok], P = a.pos[tok], tl = a.tile[tok];
  const int m_old = a.last[tok];
  const bool first = m_old == 1;
  const CacheView& cv = a.cv;
  const size_t cset = (static_cast<size_t>(a.j) * a.n_tiles + tl) * a.Hkv + g;
  const int32_t* C = a.cols + cset * a.c;
  // C is ascending: the query's columns are its prefix with C[k] <= pos; only
  // this CTA's slice of C is needed, so count within the slice in parallel
  const int ncol_all = a.ncols[cset];
  const int k0s = sp * a.cols_per_cta;
  const int kend = min(ncol_all, k0s + a.cols_per_cta);
  const int kk = k0s + tid;
  const int in_slice = (kk < kend && C[kk] <= P) ? 1 : 0;
  const int cnt = __syncthreads_count(in_slice);
  if (tid == 0) ncs = k0s + cnt;
  // the group's query heads (new, and on a first recomputation the loop-1 ones) in registers
  float qn[GRP][EPL], qo[GRP][EPL];
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    const size_t hq = static_cast<size_t>(g * grp + h);
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      qn[h][e] = a.q_cur[(static_cast<size_t>(i) * a.H + hq) * HD + lane * EPL + e];
      qo[h][e] = first ? a.q_last[(static_cast<size_t>(tok) * a.H + hq) * HD + lane * EPL + e] : 0.f;
    }
  }
  __syncthreads();
  const int k0 = k0s, k1 = ncs;
  float m[GRP], zn[GRP], zo[GRP], an[GRP][EPL], ao[GRP][EPL];
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    m[h] = -INFINITY;
    zn[h] = zo[h] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) an[h][e] = ao[h][e] = 0.f;
  }
  for (int k = k0 + warp; k < k1; k += NW) {
    const int col = C[k];
    float klo[EPL], khi[EPL], vlo[EPL], vhi[EPL];
    int rr[KM - 1];   // sparse layout: the column's pool rows, shared by its K and V chains
    if (SP) chain_rows<KM>(cv, a.j, b, col, a.loop, rr);
    chain_lane2<EPL, KM, SP>(cv, a.j, 0, b, g, col, 1, a.loop, lane, klo, khi, SP ? rr : nullptr);
    chain_lane2<EPL, KM, SP>(cv, a.j, 1, b, g, col, 1, a.loop, lane, vlo, vhi, SP ? rr : nullptr);
    if (first)
      corr_both<EPL, GRP>(qn, qo, klo, khi, vlo, vhi, a.tau, m, zn, an, zo, ao);
    else
      corr_new<EPL, GRP>(qn, khi, vhi, a.tau, m, zn, an);
  }
  // merge the warps of this CTA: the new-term numerators, then (first
  // recomputation) the old-term ones through the same buffer
  const size_t pbase = (static_cast<size_t>(i) * a.Hkv + g) * a.n_splits + sp;
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    if (lane == 0) {
      sm_m[warp][h] = m[h];
      sm_zn[warp][h] = zn[h];
      sm_zo[warp][h] = zo[h];
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) sm_acc[warp][h][lane * EPL + e] = an[h][e];
  }
  for (int term = 0; term < (first ? 2 : 1); ++term) {
    __syncthreads();
    for (int e = tid; e < grp * HD; e += 256) {
      const int h = e / HD, dd = e % HD;
      float M = -INFINITY;
      for (int w = 0; w < NW; ++w) M = fmaxf(M, sm_m[w][h]);
      float A = 0.f, Zn = 0.f, Zo = 0.f;
      if (M != -INFINITY)
        for (int w = 0; w < NW; ++w) {
          if (sm_m[w][h] == -INFINITY) continue;
          const float f = expf(sm_m[w][h] - M);
          A += sm_acc[w][h][dd] * f;
          Zn += sm_zn[w][h] * f;
          Zo += sm_zo[w][h] * f;
        }
      a.part_acc[((pbase * 2 + term) * GMAX + h) * HD + dd] = A;
      if (dd == 0 && term == 0) {
        a.part_mz[(pbase * GMAX + h) * 3 + 0] = M;
        a.part_mz[(pbase * GMAX + h) * 3 + 1] = Zn;
        a.part_mz[(pbase * GMAX + h) * 3 + 2] = Zo;
      }
    }
    if (term == 0 && first) {
      __syncthreads();
#pragma unroll
      for (int h = 0; h < GRP; ++h)
#pragma unroll
        for (int e = 0; e < EPL; ++e) sm_acc[warp][h][lane * EPL + e] = ao[h][e];
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int old = atomicAdd(&a.counters[i * a.Hkv + g], 1);
    is_last = (old == a.n_splits - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  const size_t q0 = (static_cast<size_t>(i) * a.Hkv + g) * a.n_splits;
  // merge: warp h finds head h's common maximum and denominators (lanes over
  // splits) and reads the head's stored scalars, before any is rewritten
  __shared__ float mg[GMAX], zng[GMAX], zog[GMAX], lsg[GMAX], zsg[GMAX];
  for (int h = warp; h < grp; h += NW) {
    if (lane == 0) {
      const size_t so = static_cast<size_t>(tok) * a.H + g * grp + h;
      lsg[h] = a.lse_state[so];
      zsg[h] = first ? 0.f : a.z_state[so];
    }
    float M = -INFINITY;
    for (int s2 = lane; s2 < a.n_splits; s2 += 32) M = fmaxf(M, __ldcg(&a.part_mz[((q0 + s2) * GMAX + h) * 3]));
    M = warp_max(M);
    float Zn = 0.f, Zo = 0.f;
    if (M != -INFINITY)
      for (int s2 = lane; s2 < a.n_splits; s2 += 32) {
        const float ms = __ldcg(&a.part_mz[((q0 + s2) * GMAX + h) * 3]);
        if (ms == -INFINITY) continue;
        const float f = expf(ms - M);
        Zn += f * __ldcg(&a.part_mz[((q0 + s2) * GMAX + h) * 3 + 1]);
        Zo += f * __ldcg(&a.part_mz[((q0 + s2) * GMAX + h) * 3 + 2]);
      }
    Zn = warp_sum(Zn);
    Zo = warp_sum(Zo);
    if (lane == 0) {
      mg[h] = M;
      zng[h] = Zn;
      zog[h] = Zo;
    }
  }
  __syncthreads();
  for (int e = tid; e < grp * HD; e += 256) {
    const int h = e / HD, dd = e % HD;
    const int hq = g * grp + h;
    const size_t so = static_cast<size_t>(tok) * a.H + hq;
    const float M = mg[h];
    float Nn = 0.f, No = 0.f;
    if (M != -INFINITY) {
#pragma unroll 4
      for (int s2 = 0; s2 < a.n_splits; ++s2) {
        const float ms = __ldcg(&a.part_mz[((q0 + s2) * GMAX + h) * 3]);
        if (ms == -INFINITY) continue;
        const float f = expf(ms - M);
        Nn += f * __ldcg(&a.part_acc[(((q0 + s2) * 2 + 0) * GMAX + h) * HD + dd]);
        if (first) No += f * __ldcg(&a.part_acc[(((q0 + s2) * 2 + 1) * GMAX + h) * HD + dd]);
      }
    }
    CorrRest rest;
    const float ov = corr_finish(first, M, zng[h], Nn, M, zog[h], No, lsg[h], zsg[h], a.o_state[so * HD + dd], rest,
                                 a.status);
    a.o_bf16[static_cast<size_t>(i) * a.H * HD + static_cast<size_t>(hq) * HD + dd] = f_to_bf16(ov);
    if (first) {
      a.o_state[so * HD + dd] = rest.n;
      if (dd == 0) {
        a.lse_state[so] = rest.m;
        a.z_state[so] = rest.z;
      }
    }
  }
  if (tid == 0) a.counters[i * a.Hkv + g] = 0;
}

// ============================================================================
// The correction for prefill tiles on the tensor cores (head_dim 128).  All
// selected queries of a tile share the tile's column set, so the set's rows
// are gathered once per (tile, KV head) and 64 of its (query, head) pairs at a
// time are corrected together, as a small attention over the gathered columns:
// S = tau Q K^T and O += P V with warp-level bf16 products (fp32 operands as
// hi + lo pairs, as in the prefill attention), an online softmax per row, and
// the causal rule C[k] <= pos per row.  Warps 0-3 take the new term (this
// loop's queries against the rebuilt chains of the columns), warps 4-7 the old
// term (the loop-1 queries against the base rows) of the same staged chunk,
// for the pairs on their first recomputation; each warp owns 16 pair rows.  The
// pieces then meet in shared memory and each element is finished with the
// stored state as in the other correction kernels.  Items are (plan entry,
// KV head, pass of 64 pairs), grid-stride, one CTA per SM.
// ============================================================================
template <int KM, bool SP>
__global__ void __launch_bounds__(256, 1) k_correct_tc(const CorrectArgs a) {
  constexpr int HD = 128, TILE = 64 * 128 * 2, KS = HD / 16, NDT = HD / 8;
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint8_t sm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
  // [0,1]: tau q_l hi / lo; [2,3]: tau q_last hi / lo; [4..9]: K new hi / lo, K base, V new hi / lo, V base
  const uint32_t sb = smem_u32(sm);
  auto tile_s = [&](int t) { return sb + static_cast<uint32_t>(t * TILE); };
  float* park = reinterpret_cast<float*>(sm + 4 * TILE);   // after the last chunk: old-term pieces [64][HD]
  __shared__ int rpos[64], rtok[64], rfirst[64];
  __shared__ int cpos[64];
  __shared__ float pm_o[64], pz_o[64];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wr = warp & 3;          // pair-row group
  const bool old_warp = warp >= 4;  // the old term
  const int grp = a.H / a.Hkv;
  const int nent = a.plan.counts[0];
  const int npass = (a.q_tile * grp + 63) / 64;
  const CacheView& cv = a.cv;
  const int bits = cv.bits;
  const size_t rb = cv.row_bytes_codes(), ns = cv.hd >> cv.lg;
  const size_t step = static_cast<size_t>(2) * cv.B * cv.Hkv * (SP ? cv.rows : cv.T);
  __shared__ int s_item;
  for (;;) {
    const int it = next_item(a.work, &s_item);
    if (it >= nent * a.Hkv * npass) break;
    // passes outermost (every plan entry has a first pass), the latest tiles (the longest rows) first
    const int pass = it / (nent * a.Hkv), p = nent - 1 - (it / a.Hkv) % nent, g = it % a.Hkv;
    const int qb = a.plan.qb[p], qe = a.plan.qe[p], tl = a.plan.tile[p];
    const int npairs = (qe - qb) * grp, pb = pass * 64;
    if (pb >= npairs) continue;   // (uniform over the CTA)
    const size_t cset = (static_cast<size_t>(a.j) * a.n_tiles + tl) * a.Hkv + g;
    const int32_t* C = a.cols + cset * a.c;
    const int ncol = a.ncols[cset];
    const int b = a.meta[qb].seq;
    const size_t q0 = ((((static_cast<size_t>(a.j) * (cv.K - 1)) * 2) * cv.B + b) * cv.Hkv + g) *
                      static_cast<size_t>(SP ? cv.rows : cv.T);
    __syncthreads();   // the previous item no longer reads shared memory
    // ---- stage the pass's pairs: thread -> (pair row, 8-dim piece) x 4
    bool my_first = false;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = tid + 256 * u, r = e >> 4, pc = e & 15;
      const int pr = pb + r;
      float xn[8], xo[8];
      if (pr < npairs) {
        const int qi = qb + pr / grp, hh = g * grp + pr % grp;
        const SelMeta mq = a.meta[qi];
        const float4* qn = reinterpret_cast<const float4*>(a.q_cur + (static_cast<size_t>(qi) * a.H + hh) * HD) + pc * 2;
        const float4* qo = reinterpret_cast<const float4*>(a.q_last + (static_cast<size_t>(mq.tok) * a.H + hh) * HD) + pc * 2;
        const float4 n0 = qn[0], n1 = qn[1], o0 = qo[0], o1 = qo[1];
        xn[0] = n0.x; xn[1] = n0.y; xn[2] = n0.z; xn[3] = n0.w; xn[4] = n1.x; xn[5] = n1.y; xn[6] = n1.z; xn[7] = n1.w;
        xo[0] = o0.x; xo[1] = o0.y; xo[2] = o0.z; xo[3] = o0.w; xo[4] = o1.x; xo[5] = o1.y; xo[6] = o1.z; xo[7] = o1.w;
        if (pc == 0) {
          rpos[r] = mq.pos;
          rtok[r] = mq.tok;
          rfirst[r] = mq.last == 1;
        }
        my_first = my_first || mq.last == 1;
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) xn[k] = xo[k] = 0.f;
        if (pc == 0) {
          rpos[r] = -1;
          rtok[r] = -1;
          rfirst[r] = 0;
        }
      }
      uint32_t wh[4], wl[4], woh[4], wol[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float h0, l0, h1, l1;
        split_bf16(a.tau * xn[2 * k], h0, l0);
        split_bf16(a.tau * xn[2 * k + 1], h1, l1);
        wh[k] = pack_bf16x2(h0, h1);
        wl[k] = pack_bf16x2(l0, l1);
        split_bf16(a.tau * xo[2 * k], h0, l0);
        split_bf16(a.tau * xo[2 * k + 1], h1, l1);
        woh[k] = pack_bf16x2(h0, h1);
        wol[k] = pack_bf16x2(l0, l1);
      }
      const uint32_t o = swz128(r, pc);
      *reinterpret_cast<uint4*>(sm + o) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
      *reinterpret_cast<uint4*>(sm + TILE + o) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
      *reinterpret_cast<uint4*>(sm + 2 * TILE + o) = make_uint4(woh[0], woh[1], woh[2], woh[3]);
      *reinterpret_cast<uint4*>(sm + 3 * TILE + o) = make_uint4(wol[0], wol[1], wol[2], wol[3]);
    }
    const bool old_on = __syncthreads_or(my_first ? 1 : 0) != 0;   // any pair on its first recomputation
    // this warp's rows: r0 = 16 wr + lane / 4 and r0 + 8
    const int r0 = 16 * wr + (lane >> 2), r1 = r0 + 8;
    const int P0 = rpos[r0], P1 = rpos[r1];
    const bool active = pb + 16 * wr < npairs && (!old_warp || old_on);
    const uint32_t qsh = tile_s(old_warp ? 2 : 0), qsl = tile_s(old_warp ? 3 : 1);
    float o[NDT][4];
#pragma unroll
    for (int n = 0; n < NDT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_part[2] = {0.f, 0.f};
    for (int k0 = 0; k0 < ncol; k0 += 64) {
      // ---- gather the chunk's columns: thread -> (column row, 8-dim piece) x 4, K and V
      uint4 bk[4], bv[4];
      int tcol[4];
      uint32_t ck[4][KM - 1], cvv[4][KM - 1];
      uint16_t sk[4][KM - 1], svv[4][KM - 1];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = tid + 256 * u, r = e >> 4, pc = e & 15;
        const bool ok = k0 + r < ncol;
        const int t = ok ? C[k0 + r] : 0;
        tcol[u] = ok ? t : 0x7fffffff;
        bk[u] = ok ? *reinterpret_cast<const uint4*>(cv.base_row(a.j, 0, b, g, t) + pc * 8) : make_uint4(0, 0, 0, 0);
        bv[u] = ok ? *reinterpret_cast<const uint4*>(cv.base_row(a.j, 1, b, g, t) + pc * 8) : make_uint4(0, 0, 0, 0);
        int rr[KM - 1];
#pragma unroll
        for (int q = 0; q < KM - 1; ++q) rr[q] = (ok && q + 2 <= a.loop) ? (SP ? 0 : t) : -1;
        if (SP && ok) chain_rows<KM>(cv, a.j, b, t, a.loop, rr);
#pragma unroll
        for (int q = 0; q < KM - 1; ++q) {
          ck[u][q] = cvv[u][q] = 0u;
          sk[u][q] = svv[u][q] = 0;
          if (rr[q] >= 0) {
            const size_t rik = q0 + q * step + static_cast<size_t>(rr[q]);
            const size_t riv = rik + static_cast<size_t>(cv.B) * cv.Hkv * (SP ? cv.rows : cv.T);   // kv = 1
            const uint8_t* rowk = cv.codes + rik * rb;
            const uint8_t* rowv = cv.codes + riv * rb;
            ck[u][q] = bits == 4 ? *reinterpret_cast<const uint32_t*>(rowk + pc * 4)
                                 : static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(rowk + pc * 2));
            cvv[u][q] = bits == 4 ? *reinterpret_cast<const uint32_t*>(rowv + pc * 4)
                                  : static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(rowv + pc * 2));
            sk[u][q] = cv.scales[rik * ns + ((pc * 8) >> cv.lg)];
            svv[u][q] = cv.scales[riv * ns + ((pc * 8) >> cv.lg)];
          }
        }
      }
      __syncthreads();   // every warp is done with the previous chunk's tiles
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = tid + 256 * u, r = e >> 4, pc = e & 15;
        const uint32_t off = swz128(r, pc);
        if (pc == 0) cpos[r] = tcol[u];
#pragma unroll
        for (int kv = 0; kv < 2; ++kv) {
          const uint4 bw = kv ? bv[u] : bk[u];
          const uint32_t w[4] = {bw.x, bw.y, bw.z, bw.w};
          float x[8];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            x[2 * k] = bf16_to_f(w[k] & 0xFFFF);
            x[2 * k + 1] = bf16_to_f(w[k] >> 16);
          }
#pragma unroll
          for (int q = 0; q < KM - 1; ++q) {
            if (q + 2 > a.loop) break;
            const float sc = half_bits_to_f(kv ? svv[u][q] : sk[u][q]);
            const uint32_t cw = kv ? cvv[u][q] : ck[u][q];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int cd = bits == 4 ? sext(static_cast<int>((cw >> (4 * k)) & 0xFu), 4)
                                       : sext(static_cast<int>((cw >> (2 * k)) & 0x3u), 2);
              x[k] = __fadd_rn(x[k], __fmul_rn(static_cast<float>(cd), sc));
            }
          }
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            float h0, l0, h1, l1;
            split_bf16(x[2 * k], h0, l0);
            split_bf16(x[2 * k + 1], h1, l1);
            hw[k] = pack_bf16x2(h0, h1);
            lw[k] = pack_bf16x2(l0, l1);
          }
          uint8_t* t0 = sm + (4 + 3 * kv) * TILE;   // new hi, new lo, base
          *reinterpret_cast<uint4*>(t0 + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(t0 + TILE + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
          *reinterpret_cast<uint4*>(t0 + 2 * TILE + off) = bw;
        }
      }
      __syncthreads();
      if (!active) continue;
      // ---- scores of this warp's 16 rows x 64 columns
      const uint32_t kh = tile_s(4), kl = tile_s(5), kbt = tile_s(6);
      float sc[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t ah[4], al[4];
        const uint32_t qo_ = swz128(16 * wr + (lane & 15), 2 * ks + (lane >> 4));
        ldsm_x4(qsh + qo_, ah);
        ldsm_x4(qsl + qo_, al);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
          const uint32_t ko = swz128(key, 2 * ks + ((lane >> 3) & 1));
          uint32_t fh[4];
          ldsm_x4((old_warp ? kbt : kh) + ko, fh);
#pragma unroll
          for (int hlf = 0; hlf < 2; ++hlf) {
            mma_bf16_16816(sc[2 * np + hlf], ah, fh[2 * hlf], fh[2 * hlf + 1]);
            mma_bf16_16816(sc[2 * np + hlf], al, fh[2 * hlf], fh[2 * hlf + 1]);
          }
          if (!old_warp) {
            uint32_t fl[4];
            ldsm_x4(kl + ko, fl);
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) mma_bf16_16816(sc[2 * np + hlf], ah, fl[2 * hlf], fl[2 * hlf + 1]);
          }
        }
      }
      // causal rule per row: column C[k] is visible at position P when C[k] <= P
      float tm[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int cp = cpos[nt * 8 + 2 * (lane & 3) + e];
          if (cp > P0) sc[nt][e] = -INFINITY;
          if (cp > P1) sc[nt][2 + e] = -INFINITY;
          tm[0] = fmaxf(tm[0], sc[nt][e]);
          tm[1] = fmaxf(tm[1], sc[nt][2 + e]);
        }
      }
      float alpha[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        tm[r] = fmaxf(tm[r], __shfl_xor_sync(0xffffffffu, tm[r], 1));
        tm[r] = fmaxf(tm[r], __shfl_xor_sync(0xffffffffu, tm[r], 2));
        const float mn = fmaxf(m_run[r], tm[r]);
        alpha[r] = (m_run[r] == -INFINITY || mn == -INFINITY) ? (m_run[r] == -INFINITY ? 0.f : 1.f)
                                                               : expf(m_run[r] - mn);
        m_run[r] = mn;
      }
      float rs[2] = {0.f, 0.f};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float mr = m_run[e >> 1];
          const float pv = (sc[nt][e] == -INFINITY) ? 0.f : expf(sc[nt][e] - mr);
          sc[nt][e] = pv;
          rs[e >> 1] += pv;
        }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) l_part[r] = l_part[r] * alpha[r] + rs[r];
#pragma unroll
      for (int n = 0; n < NDT; ++n) {
        o[n][0] *= alpha[0];
        o[n][1] *= alpha[0];
        o[n][2] *= alpha[1];
        o[n][3] *= alpha[1];
      }
      // ---- O += P V over the chunk's 64 columns (4 steps of 16)
      const uint32_t vh = tile_s(7), vl = tile_s(8), vbt = tile_s(9);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t ph[4], pl[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float* src = sc[2 * kk + (r >> 1)] + 2 * (r & 1);
          float h0, l0, h1, l1;
          split_bf16(src[0], h0, l0);
          split_bf16(src[1], h1, l1);
          ph[r] = pack_bf16x2(h0, h1);
          pl[r] = pack_bf16x2(l0, l1);
        }
        const int vr = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
        for (int n2 = 0; n2 < NDT / 2; ++n2) {
          const uint32_t vo = swz128(vr, n2 * 2 + (lane >> 4));
          uint32_t vf[4];
          ldsm_x4_t((old_warp ? vbt : vh) + vo, vf);
          mma_bf16_16816(o[2 * n2], ph, vf[0], vf[1]);
          mma_bf16_16816(o[2 * n2], pl, vf[0], vf[1]);
          mma_bf16_16816(o[2 * n2 + 1], ph, vf[2], vf[3]);
          mma_bf16_16816(o[2 * n2 + 1], pl, vf[2], vf[3]);
          if (!old_warp) {
            ldsm_x4_t(vl + vo, vf);
            mma_bf16_16816(o[2 * n2], ph, vf[0], vf[1]);
            mma_bf16_16816(o[2 * n2 + 1], ph, vf[2], vf[3]);
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      l_part[r] += __shfl_xor_sync(0xffffffffu, l_part[r], 1);
      l_part[r] += __shfl_xor_sync(0xffffffffu, l_part[r], 2);
    }
    __syncthreads();   // the column tiles are dead: the old-term warps park their pieces there
    if (old_warp && old_on) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = r ? r1 : r0;
#pragma unroll
        for (int n = 0; n < NDT; ++n) {
          const int d = n * 8 + 2 * (lane & 3);
          *reinterpret_cast<float2*>(park + row * HD + d) = make_float2(o[n][2 * r], o[n][2 * r + 1]);
        }
        if ((lane & 3) == 0) {
          pm_o[row] = m_run[r];
          pz_o[row] = l_part[r];
        }
      }
    }
    __syncthreads();
    if (!old_warp && pb + 16 * wr < npairs) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = r ? r1 : r0;
        const int pr = pb + row;
        const bool valid = pr < npairs;
        const int slot = qb + pr / grp, hq = g * grp + pr % grp;
        const size_t so = valid ? static_cast<size_t>(rtok[row]) * a.H + hq : 0;
        const bool first = valid && rfirst[row] != 0;
        float Ls = 0.f, Zs = 0.f;
        float st[NDT][2];
        if (valid) {
          Ls = a.lse_state[so];
          Zs = first ? 0.f : a.z_state[so];
#pragma unroll
          for (int n = 0; n < NDT; ++n) {
            const float2 v = *reinterpret_cast<const float2*>(a.o_state + so * HD + n * 8 + 2 * (lane & 3));
            st[n][0] = v.x;
            st[n][1] = v.y;
          }
        }
        __syncwarp();   // the quad has read the stored scalars before any lane rewrites them
        if (!valid) continue;
        const float Mo = first ? pm_o[row] : -INFINITY, zo = first ? pz_o[row] : 0.f;
#pragma unroll
        for (int n = 0; n < NDT; ++n) {
          const int d = n * 8 + 2 * (lane & 3);
          float ov[2], rn[2];
          CorrRest rest{};
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float no = first ? park[row * HD + d + e] : 0.f;
            ov[e] = corr_finish(first, m_run[r], l_part[r], o[n][2 * r + e], Mo, zo, no, Ls, Zs, st[n][e], rest,
                                a.status);
            rn[e] = rest.n;
          }
          *reinterpret_cast<uint32_t*>(a.o_bf16 + static_cast<size_t>(slot) * a.H * HD +
                                       static_cast<size_t>(hq) * HD + d) = pack_bf16x2(ov[0], ov[1]);
          if (first) {
            *reinterpret_cast<float2*>(a.o_state + so * HD + d) = make_float2(rn[0], rn[1]);
            if (n == 0 && (lane & 3) == 0) {
              a.lse_state[so] = rest.m;
              a.z_state[so] = rest.z;
            }
          }
        }
      }
    }
  }
  finish_items(a.work);
}

// ============================================================================
// The correction for few selected queries (decode): the column slices of one
// (query, KV group) are the CTAs of one cluster (kCorrCluster CTAs of
// kCorrWarps warps).  The query's slot record, its column-set count and the
// first column ids are requested together; warp w of rank r takes columns
// r*per + w + u*kCorrWarps of the set, two at a time (later recomputations:
// the new chains only) or one at a time (a first recomputation: new and base
// rows), with every K and V chain load issued before any arithmetic.  The
// warps' pieces (per-head max, denominators, numerators) are merged in the CTA
// with one weight per (warp, head); then rank r merges outputs
// [r*E/CS, (r+1)*E/CS) of every rank, in rank order, over distributed shared
// memory, with the stored state.  No global scratch, fence or ticket.
// grid (kCorrCluster, n_sel * Hkv).
// ============================================================================
template <int HD, int EPL, int GRP, int KM, bool SP>
__global__ void __launch_bounds__(32 * kCorrWarps) k_correct_cluster(const CorrectArgs a) {
  pdl_trigger();
  constexpr int NW = kCorrWarps, CS = kCorrCluster, E = GRP * HD, NT = 32 * NW;
  extern __shared__ float sm_acc[];   // [2][NW][GRP][HD]: new-term numerators, then old-term ones
  __shared__ float sm_m[2][NW][GRP], sm_z[2][NW][GRP], sm_w[2][NW][GRP];
  __shared__ float pm[2][GRP], pz[2][GRP];
  __shared__ float pacc[2][GRP][HD];
  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = static_cast<int>(cluster.block_rank());
  const int i = blockIdx.y / a.Hkv, g = blockIdx.y % a.Hkv;
  pdl_wait();
  const SelMeta mt = a.meta[i];
  const int tok = mt.tok, b = mt.seq;
  const bool first = mt.last == 1;
  const int nterm = first ? 2 : 1;
  const CacheView& cv = a.cv;
  const size_t cset = (static_cast<size_t>(a.j) * a.n_tiles + mt.tile) * a.Hkv + g;
  const int32_t* C = a.cols + cset * a.c;
  // a decode token is its own tile, so every column of its set is causal; the
  // slice bounds use the set's capacity so the column ids need not wait for its count
  const int per = (a.c + CS - 1) / CS;
  const int k0 = rank * per, k1 = min(a.c, k0 + per);
  const int nvalid = a.ncols[cset];
  int col_first[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) col_first[u] = k0 + warp + u * NW < k1 ? C[k0 + warp + u * NW] : -1;
  // rank r merges elements [r*E/CS, (r+1)*E/CS) of the (head, dim) outputs at the
  // end; the stored state it merges into is requested now, not after the barrier
  const int me = (rank * E) / CS + tid;
  const bool merger = me < ((rank + 1) * E) / CS;
  float st_o = 0.f, st_l = 0.f, st_z = 0.f;
  if (merger) {
    const size_t so = static_cast<size_t>(tok) * a.H + g * GRP + me / HD;
    st_o = a.o_state[so * HD + me % HD];
    st_l = a.lse_state[so];
    st_z = first ? 0.f : a.z_state[so];
  }
  const int k1v = min(k1, nvalid);
  auto col_at = [&](int k) { return k == k0 + warp ? col_first[0] : (k == k0 + warp + NW ? col_first[1] : C[k]); };
  // sparse storage: the pool rows of this CTA's columns, staged once ([column][level])
  __shared__ int rows_sm[SP ? 64 * (KM - 1) : 1];
  const bool rows_staged = SP && per <= 64;
  if (rows_staged) {
    for (int e = tid; e < per * (KM - 1); e += NT) {
      const int kk = e / (KM - 1), q = e % (KM - 1), k = k0 + kk;
      const int col = k < k1v ? C[k] : -1;
      rows_sm[e] = (col >= 0 && q + 2 <= a.loop) ? cv.ridx[cv.ridx_index(a.j, q + 2, b, col)] : -1;
    }
    __syncthreads();
  }
  float q[GRP][EPL], m[GRP], z[GRP], acc[GRP][EPL];
  auto reset = [&]() {
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      m[h] = -INFINITY;
      z[h] = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[h][e] = 0.f;
    }
  };
  auto park = [&](int term) {   // this warp's piece of one term, to shared memory
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      if (lane == 0) {
        sm_m[term][warp][h] = m[h];
        sm_z[term][warp][h] = z[h];
      }
#pragma unroll
      for (int e = 0; e < EPL; ++e) sm_acc[((term * NW + warp) * GRP + h) * HD + lane * EPL + e] = acc[h][e];
    }
  };
  if (first) {
    // old term: the loop-1 queries against the base rows (the loop-1 K, V)
#pragma unroll
    for (int h = 0; h < GRP; ++h) {
      const size_t hq = static_cast<size_t>(g * GRP + h);
#pragma unroll
      for (int e = 0; e < EPL; ++e) q[h][e] = a.q_last[(static_cast<size_t>(tok) * a.H + hq) * HD + lane * EPL + e];
    }
    reset();
    for (int kb = k0 + warp; kb < k1v; kb += 2 * NW) {
      float kr[2][EPL], vr[2][EPL];
      int col[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        col[u] = kb + u * NW < k1v ? col_at(kb + u * NW) : -1;
        if (col[u] < 0) continue;
        base_lane<EPL>(cv.base_row(a.j, 0, b, g, col[u]), lane, kr[u]);
        base_lane<EPL>(cv.base_row(a.j, 1, b, g, col[u]), lane, vr[u]);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (col[u] >= 0) corr_new<EPL, GRP>(q, kr[u], vr[u], a.tau, m, z, acc);
    }
    park(1);
  }
  // new term: this loop's queries against the rebuilt chains, CPI columns at
  // a time (one for sparse chains longer than four levels, whose index rows
  // would otherwise not fit in registers beside the chains)
#pragma unroll
  for (int h = 0; h < GRP; ++h) {
    const size_t hq = static_cast<size_t>(g * GRP + h);
#pragma unroll
    for (int e = 0; e < EPL; ++e) q[h][e] = a.q_cur[(static_cast<size_t>(i) * a.H + hq) * HD + lane * EPL + e];
  }
  reset();
  {
    constexpr int CPI = (SP && KM > 4) ? 1 : 2;
    for (int kb = k0 + warp; kb < k1v; kb += CPI * NW) {
      int col[CPI];
#pragma unroll
      for (int u = 0; u < CPI; ++u) col[u] = kb + u * NW < k1v ? col_at(kb + u * NW) : -1;
      float klo[CPI][EPL], khi[CPI][EPL], vlo[CPI][EPL], vhi[CPI][EPL];
      int rr[CPI][KM - 1];
      if (SP) {
#pragma unroll
        for (int u = 0; u < CPI; ++u) {
          if (col[u] < 0) continue;
          if (rows_staged) {
#pragma unroll
            for (int q = 0; q < KM - 1; ++q) rr[u][q] = rows_sm[(kb + u * NW - k0) * (KM - 1) + q];
          } else {
            chain_rows<KM>(cv, a.j, b, col[u], a.loop, rr[u]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < CPI; ++u) {
        if (col[u] < 0) continue;
        chain_lane2<EPL, KM, SP>(cv, a.j, 0, b, g, col[u], a.loop, a.loop, lane, klo[u], khi[u],
                                 SP ? rr[u] : nullptr);
        chain_lane2<EPL, KM, SP>(cv, a.j, 1, b, g, col[u], a.loop, a.loop, lane, vlo[u], vhi[u],
                                 SP ? rr[u] : nullptr);
      }
#pragma unroll
      for (int u = 0; u < CPI; ++u)
        if (col[u] >= 0) corr_new<EPL, GRP>(q, khi[u], vhi[u], a.tau, m, z, acc);
    }
  }
  park(0);
  __syncthreads();
  // this CTA's piece of each term: one weight per (warp, head), then the
  // weighted sums in warp order
  if (tid < nterm * GRP) {
    const int term = tid / GRP, h = tid % GRP;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, sm_m[term][w][h]);
    float Z = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float f = sm_m[term][w][h] == -INFINITY ? 0.f : expf(sm_m[term][w][h] - M);
      sm_w[term][w][h] = f;
      Z += f * sm_z[term][w][h];
    }
    pm[term][h] = M;
    pz[term][h] = Z;
  }
  __syncthreads();
  for (int e = tid; e < nterm * E; e += NT) {
    const int term = e / E, h = (e % E) / HD, dd = e % HD;
    float A = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) A += sm_w[term][w][h] * sm_acc[((term * NW + w) * GRP + h) * HD + dd];
    pacc[term][h][dd] = A;
  }
  cluster.sync();
  if (merger) {
    const int h = me / HD, dd = me % HD;
    const int hq = g * GRP + h;
    const size_t so = static_cast<size_t>(tok) * a.H + hq;
    // every rank's piece is requested before any is used, so the distributed
    // shared-memory round trips overlap; the merge itself runs in rank order
    float Mt[2], Zt[2], Nt[2];
#pragma unroll
    for (int term = 0; term < 2; ++term) {
      Mt[term] = -INFINITY;
      Zt[term] = Nt[term] = 0.f;
      if (term >= nterm) continue;
      float rm[CS], rz[CS], ra[CS];
#pragma unroll
      for (int r = 0; r < CS; ++r) {
        rm[r] = *cluster.map_shared_rank(&pm[term][h], r);
        rz[r] = *cluster.map_shared_rank(&pz[term][h], r);
        ra[r] = *cluster.map_shared_rank(&pacc[term][h][dd], r);
      }
      float M = -INFINITY;
#pragma unroll
      for (int r = 0; r < CS; ++r) M = fmaxf(M, rm[r]);
      float Z = 0.f, N = 0.f;
#pragma unroll
      for (int r = 0; r < CS; ++r) {
        if (rm[r] == -INFINITY) continue;
        const float f = expf(rm[r] - M);
        Z += f * rz[r];
        N += f * ra[r];
      }
      Mt[term] = M;
      Zt[term] = Z;
      Nt[term] = N;
    }
    CorrRest rest;
    const float ov = corr_finish(first, Mt[0], Zt[0], Nt[0], Mt[1], Zt[1], Nt[1], st_l, st_z, st_o, rest, a.status);
    a.o_bf16[static_cast<size_t>(i) * a.H * HD + static_cast<size_t>(hq) * HD + dd] = f_to_bf16(ov);
    // every rank read the stored scalars before the first cluster barrier
    if (first) {
      a.o_state[so * HD + dd] = rest.n;
      if (dd == 0) {
        a.lse_state[so] = rest.m;
        a.z_state[so] = rest.z;
      }
    }
  }
  cluster.sync();
}

// ============================================================================
// cache import helpers
// ============================================================================
template <int EPL>
__global__ void k_pack_codes(const int8_t* __restrict__ src, int rows, int hd, int bits, uint8_t* __restrict__ dst,
                             size_t dst_row_stride) {
  pdl_trigger();
  pdl_wait();
  const int w = blockIdx.x * 4 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (w >= rows) return;
  int c[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) c[e] = src[static_cast<size_t>(w) * hd + lane * EPL + e];
  store_lane_codes<EPL>(dst + static_cast<size_t>(w) * dst_row_stride, bits, lane, c);
}

// Sparse residual storage: one (layer, sequence) slice of an imported lazy
// context.  CTA l-2 takes loop l: the positions whose codes or scales are not
// all zero take pool rows in position order and their codes are packed into
// them; the other positions get -1.  codes int8 [K-1][Hkv][n][hd], scales fp16
// bits [K-1][Hkv][n][hd/g] (K, V).  A position beyond the pool records
// kErrCapacity and keeps no row.
__global__ void __launch_bounds__(256) k_import_rows(const CacheView cv, int j, int b, int n, const int8_t* ck,
                                                     const int8_t* cvv, const uint16_t* sk, const uint16_t* sv,
                                                     int* status) {
  __shared__ int scan_buf[33];
  __shared__ int base;
  const int l = blockIdx.x + 2, hd = cv.hd, ns = hd >> cv.lg;
  const size_t lrow = static_cast<size_t>(blockIdx.x) * cv.Hkv;   // [K-1][Hkv] row block of this loop
  if (threadIdx.x == 0) base = 0;
  __syncthreads();
  for (int t0 = 0; t0 < n; t0 += blockDim.x) {
    const int t = t0 + threadIdx.x;
    int nz = 0;
    if (t < n)
      for (int kv = 0; kv < 2 && !nz; ++kv)
        for (int h = 0; h < cv.Hkv && !nz; ++h) {
          const size_t row = (lrow + h) * n + t;
          const int8_t* c = (kv ? cvv : ck) + row * hd;
          const uint16_t* sc = (kv ? sv : sk) + row * ns;
          for (int e = 0; e < hd && !nz; ++e) nz = c[e] != 0;
          for (int e = 0; e < ns && !nz; ++e) nz = sc[e] != 0;
        }
    int tot;
    const int rank = base + block_exclusive_scan(nz, &tot, scan_buf);
    if (t < n) {
      int r = -1;
      if (nz) {
        r = rank;
        if (r >= cv.rows) {
          r = -1;
          if (status) atomicOr(status, kErrCapacity);
        }
      }
      cv.ridx[cv.ridx_index(j, l, b, t)] = r;
      if (r >= 0)
        for (int kv = 0; kv < 2; ++kv)
          for (int h = 0; h < cv.Hkv; ++h) {
            const size_t row = (lrow + h) * n + t;
            const int8_t* c = (kv ? cvv : ck) + row * hd;
            uint8_t* dst = cv.code_row(j, l, kv, b, h, r);
            const int per = 8 / cv.bits, fm = (1 << cv.bits) - 1;
            for (int o = 0; o < hd / per; ++o) {
              uint32_t byte = 0;
              for (int e = 0; e < per; ++e) byte |= static_cast<uint32_t>(c[o * per + e] & fm) << (e * cv.bits);
              dst[o] = static_cast<uint8_t>(byte);
            }
            const uint16_t* sc = (kv ? sv : sk) + row * ns;
            uint16_t* sd = cv.scale_row(j, l, kv, b, h, r);
            for (int e = 0; e < ns; ++e) sd[e] = sc[e];
          }
    }
    __syncthreads();
    if (threadIdx.x == 0) base += tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) cv.rcount[(static_cast<size_t>(j) * (cv.K - 1) + (l - 2)) * cv.B + b] = min(base, cv.rows);
}

// Sparse residual storage: positions 0..n-1 of one (layer, loop, K/V, sequence)
// as dense rows (zero where no row is kept): codes [Hkv][n][hd*b/8], scales
// [Hkv][n][hd/g].  One thread per (head, position).
__global__ void k_export_rows(const CacheView cv, int j, int l, int kv, int b, int n, uint8_t* codes,
                              uint16_t* scales) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= cv.Hkv * n) return;
  const int h = i / n, t = i % n;
  const int rb = static_cast<int>(cv.row_bytes_codes()), ns = cv.hd >> cv.lg;
  const int r = cv.ridx[cv.ridx_index(j, l, b, t)];
  uint8_t* cd = codes + static_cast<size_t>(i) * rb;
  uint16_t* sd = scales + static_cast<size_t>(i) * ns;
  for (int o = 0; o < rb; ++o) cd[o] = r >= 0 ? cv.code_row(j, l, kv, b, h, r)[o] : 0;
  for (int e = 0; e < ns; ++e) sd[e] = r >= 0 ? cv.scale_row(j, l, kv, b, h, r)[e] : 0;
}

cudaError_t launch_import_rows(const CacheView& cv, int j, int b, int n, const int8_t* ck, const int8_t* cvv,
                               const uint16_t* sk, const uint16_t* sv, int* status, cudaStream_t s) {
  return launch_k(false, k_import_rows, dim3(cv.K - 1), dim3(256), 0, s, cv, j, b, n, ck, cvv, sk, sv, status);
}
cudaError_t launch_export_rows(const CacheView& cv, int j, int l, int kv, int b, int n, uint8_t* codes,
                               uint16_t* scales, cudaStream_t s) {
  const int items = cv.Hkv * n;
  return launch_k(false, k_export_rows, dim3((items + 255) / 256), dim3(256), 0, s, cv, j, l, kv, b, n, codes,
                  scales);
}

// ============================================================================
// launchers
// ============================================================================
thread_local bool g_pdl = false;
void set_pdl(bool on) { g_pdl = on; }
// prefill attention on the tensor-core kernel (1) or the fp32 SIMT one (0); thread-local
thread_local bool kv_tc_prefill = true;
void set_tc_prefill(bool on) { kv_tc_prefill = on; }

cudaError_t launch_topk(const float* keys, int n_seg, int n, int k, int32_t* idx, cudaStream_t s) {
  const size_t sm = n <= kSelColsSmemKeys ? static_cast<size_t>(n) * 4 : 0;
  return launch_k(false, k_topk_segments, dim3(n_seg), dim3(1024), sm, s, keys, n, k, idx);
}
cudaError_t launch_select_tokens(const float* keys, int N, int n_sel, int32_t* idx, const int* forced_on,
                                 const int32_t* forced, cudaStream_t s) {
  return launch_k(g_pdl, k_select_tokens, dim3(1), dim3(1024), 0, s, keys, N, n_sel, idx, forced_on, forced);
}
cudaError_t launch_quantize_rows(const float* r, const uint16_t* prev, int rows, int width, int g, int bits,
                                 uint8_t* codes, uint16_t* scales, cudaStream_t s) {
  // 8 warps per CTA, 4 row chunks per warp; the code width is a template parameter
  const bool wide = width % 128 == 0;
  const long long items = static_cast<long long>(rows) * (wide ? width / 128 : width / 64);
  const dim3 grid(static_cast<unsigned>((items + 31) / 32));
  if (wide)
    return bits == 4 ? launch_k(false, k_quantize_rows<4, 4>, grid, dim3(256), 0, s, r, prev, rows, width, g, bits,
                                codes, scales)
                     : launch_k(false, k_quantize_rows<4, 2>, grid, dim3(256), 0, s, r, prev, rows, width, g, bits,
                                codes, scales);
  return bits == 4 ? launch_k(false, k_quantize_rows<2, 4>, grid, dim3(256), 0, s, r, prev, rows, width, g, bits,
                              codes, scales)
                   : launch_k(false, k_quantize_rows<2, 2>, grid, dim3(256), 0, s, r, prev, rows, width, g, bits,
                              codes, scales);
}
cudaError_t launch_rmsnorm_rows(const float* h, const int* idx, int n, int n_pad, int d, const float* gain, float eps,
                                uint16_t* x, cudaStream_t s) {
  return launch_k(g_pdl, k_rmsnorm_rows, dim3(n_pad), dim3(256), 0, s, h, idx, n, d, gain, eps, x);
}
template <int EPL, int KM>
cudaError_t launch_qkv_post_km(const QkvPostArgs& a, dim3 grid, cudaStream_t s) {
  return a.cv.rows ? launch_k(g_pdl, k_qkv_post<EPL, KM, true>, grid, dim3(128), 0, s, a)
                   : launch_k(g_pdl, k_qkv_post<EPL, KM, false>, grid, dim3(128), 0, s, a);
}
template <int EPL>
cudaError_t launch_qkv_post_e(const QkvPostArgs& a, dim3 grid, cudaStream_t s) {
  switch (chain_km(a.cv.K)) {
    case 2: return launch_qkv_post_km<EPL, 2>(a, grid, s);
    case 4: return launch_qkv_post_km<EPL, 4>(a, grid, s);
    case 8: return launch_qkv_post_km<EPL, 8>(a, grid, s);
    case 16: return launch_qkv_post_km<EPL, 16>(a, grid, s);
    default: return cudaErrorInvalidValue;
  }
}
cudaError_t launch_qkv_post(const QkvPostArgs& a, cudaStream_t s) {
  const int warps = a.n * (a.H + 2 * a.Hkv);
  const dim3 grid((warps + 3) / 4);
  return a.hd == 128 ? launch_qkv_post_e<4>(a, grid, s) : launch_qkv_post_e<2>(a, grid, s);
}
size_t attn_decode_smem(int hd) { return 1024 + static_cast<size_t>(kDecStages) * 2 * kDecTile * hd * 2; }
cudaError_t launch_attn_decode(const CUtensorMap& kv, const AttnDecArgs& a, int n, cudaStream_t s) {
  dim3 grid(n * a.Hkv, a.n_splits);
  const size_t sm = attn_decode_smem(a.hd);
  const int grp = a.H / a.Hkv;
#define FL_ATT(G)                                                                              \
  case G:                                                                                      \
    return a.hd == 128 ? launch_k(g_pdl, k_attn_decode<128, G>, grid, dim3(128), sm, s, kv, a) \
                       : launch_k(g_pdl, k_attn_decode<64, G>, grid, dim3(128), sm, s, kv, a);
  switch (grp) {
    FL_ATT(1)
    FL_ATT(2)
    FL_ATT(4)
    FL_ATT(8)
    default: return cudaErrorInvalidValue;
  }
#undef FL_ATT
}
size_t attn_prefill_smem(int hd) {
  return static_cast<size_t>(64) * (hd + 1) * 4 + 64 * 65 * 4 + 2 * 64 * (hd + kDecPad) * 2;
}
size_t attn_prefill_tc_smem(int hd) { return 1024 + static_cast<size_t>(kPreStages) * 2 * 64 * hd * 2; }
cudaError_t launch_attn_prefill(const CUtensorMap& kv, const AttnPreArgs& a, int B, cudaStream_t s) {
  dim3 grid((a.T + 63) / 64, a.H, B);
  if (kv_tc_prefill) {
    const size_t sm = attn_prefill_tc_smem(a.hd);
    if (a.hd == 128) return launch_k(g_pdl, k_attn_prefill_tc<128>, grid, dim3(128), sm, s, kv, a);
    return launch_k(g_pdl, k_attn_prefill_tc<64>, grid, dim3(128), sm, s, kv, a);
  }
  const size_t sm = attn_prefill_smem(a.hd);
  if (a.hd == 128) return launch_k(g_pdl, k_attn_prefill<128>, grid, dim3(256), sm, s, a);
  return launch_k(g_pdl, k_attn_prefill<64>, grid, dim3(256), sm, s, a);
}
cudaError_t launch_setup_call(int N, int decode, int T, int tiles_per_seq, int q_tile, const int* seq_len, int* seq,
                              int* pos, int* tile, int* last, int n_tiles, int* has_c, unsigned long long* stamps,
                              int n_stamps, cudaStream_t s) {
  const int n = N > n_tiles ? N : n_tiles;
  return launch_k(g_pdl, k_setup_call, dim3((n + 255) / 256), dim3(256), 0, s, N, decode, T, tiles_per_seq, q_tile,
                  seq_len, seq, pos, tile, last, n_tiles, has_c, stamps, n_stamps);
}
cudaError_t launch_loop_input(float* h, const int* idx, int n, int d, const float* e, float gamma, const float* x,
                              cudaStream_t s) {
  return launch_k(g_pdl, k_loop_input, dim3(n), dim3(256), 0, s, h, idx, n, d, e, gamma, x);
}
cudaError_t launch_set_lens(int B, int* seq_len, int add, cudaStream_t s) {
  return launch_k(g_pdl, k_set_lens, dim3((B + 127) / 128), dim3(128), 0, s, B, seq_len, add);
}
cudaError_t launch_reset_lens(const LensArg& a, int* seq_len, cudaStream_t s) {
  return launch_k(false, k_reset_lens, dim3(1), dim3(kLensByValue), 0, s, a, seq_len);
}
cudaError_t launch_after_select(const int32_t* idx, int n_sel, int N, int d, int* sel_slot, const float* h,
                                float* h_snap, const int* seq, const int* tile, const int* last, const int* pos,
                                SelMeta* meta, cudaStream_t s) {
  const int slot_blocks = (N + 255) / 256;
  return launch_k(g_pdl, k_after_select, dim3(slot_blocks + n_sel), dim3(256), 0, s, idx, n_sel, N, d, sel_slot, h,
                  h_snap, slot_blocks, seq, tile, last, pos, meta);
}
cudaError_t launch_change_keys(const float* h, const float* ref, const int* sel_slot, int N, int d, int loop,
                               float* key, int* last, const int* tile, int* has_c, cudaStream_t s) {
  return launch_k(g_pdl, k_change_keys, dim3((N + 3) / 4), dim3(128), 0, s, h, ref, sel_slot, N, d, loop, key, last,
                  tile, has_c);
}
cudaError_t launch_assign_rows(const CacheView& cv, int loop, int B, int Tc, const int* sel_slot, const int* pos,
                               int* status, cudaStream_t s) {
  return launch_k(g_pdl, k_assign_rows, dim3(B), dim3(1024), 0, s, cv, loop, Tc, sel_slot, pos, status);
}
cudaError_t launch_reset_rows(const CacheView& cv, const int* seq_len, cudaStream_t s) {
  const int warps = cv.M * (cv.K - 1) * cv.B;
  return launch_k(false, k_reset_rows, dim3((warps + 7) / 8), dim3(256), 0, s, cv, seq_len);
}
cudaError_t launch_select_step(const SelectStepArgs& a, cudaStream_t s) {
  return launch_k(g_pdl, k_select_step, dim3(1), dim3(1024), 0, s, a);
}
cudaError_t launch_plan_tiles(const int32_t* idx, int n_sel, const int* tile, const int* has_c, const TilePlan& p,
                              cudaStream_t s) {
  return launch_k(g_pdl, k_plan_tiles, dim3(1), dim3(1024), 0, s, idx, n_sel, tile, has_c, p);
}
// (both also stage one row of column keys, up to kSelColsSmemKeys, for the folded selection)
// 2 query tiles, 2 base stages, the residual tile; at least the folded selection's key row
size_t dscore_tc_smem() { return std::max<size_t>(1024 + 5 * 64 * 128 * 2, 1024 + kSelColsSmemKeys * 4); }
size_t dscore_smem(int hd) {   // staged pairs + the warps' column buffers, or the folded selection's key row
  return std::max<size_t>(static_cast<size_t>(2) * kDsPairs * 4 * (hd / 4 + 4) * 4 + 8 * 2 * 8 * hd * 2,
                          kSelColsSmemKeys * 4);
}
cudaError_t launch_dscore(const DScoreArgs& a, int max_need, int max_chunks, cudaStream_t s) {
  DScoreArgs b = a;
  b.max_chunks = max_chunks;
  if (a.tc && a.hd == 128) {   // prefill tiles: the tensor-core kernel, two CTAs per SM
    // grid-stride over (tile, KV head, unit of kDsTcUnit chunks) items
    const int items = max_need * a.Hkv * ((max_chunks + kDsTcUnit - 1) / kDsTcUnit);
    const dim3 g1(items < 2 * kDscoreSMs ? items : 2 * kDscoreSMs);
    const size_t smt = dscore_tc_smem();
    const bool sp = a.cv.rows != 0;
#define FL_DST(KMv)                                                                                    \
  case KMv:                                                                                            \
    return sp ? launch_k(g_pdl, k_dscore_tc<KMv, true>, g1, dim3(256), smt, s, b)                      \
              : launch_k(g_pdl, k_dscore_tc<KMv, false>, g1, dim3(256), smt, s, b);
    switch (chain_km(a.cv.K)) {
      FL_DST(2)
      FL_DST(4)
      FL_DST(8)
      FL_DST(16)
      default: return cudaErrorInvalidValue;
    }
#undef FL_DST
  }
  // items of (tile, KV head, block of columns): 256-column blocks, halved (to 64)
  // while the items would not fill two CTAs per SM; two CTAs per SM
  int blk = kDsBlock;
  while (blk > 64 && max_need * a.Hkv * ((max_chunks * 64 + blk - 1) / blk) < 2 * kDscoreSMs) blk /= 2;
  b.ds_block = blk;
  const int items = max_need * a.Hkv * ((max_chunks * 64 + blk - 1) / blk);
  const dim3 grid(items < 2 * kDscoreSMs ? items : 2 * kDscoreSMs);
  const size_t sm = dscore_smem(a.hd);
  const bool sp = a.cv.rows != 0;
#define FL_DS(KMv)                                                                                     \
  case KMv:                                                                                            \
    if (sp)                                                                                            \
      return a.hd == 128 ? launch_k(g_pdl, k_dscore<128, KMv, true>, grid, dim3(256), sm, s, b)        \
                         : launch_k(g_pdl, k_dscore<64, KMv, true>, grid, dim3(256), sm, s, b);        \
    return a.hd == 128 ? launch_k(g_pdl, k_dscore<128, KMv, false>, grid, dim3(256), sm, s, b)         \
                       : launch_k(g_pdl, k_dscore<64, KMv, false>, grid, dim3(256), sm, s, b);
  switch (chain_km(a.cv.K)) {
    FL_DS(2)
    FL_DS(4)
    FL_DS(8)
    FL_DS(16)
    default: return cudaErrorInvalidValue;
  }
#undef FL_DS
}
size_t select_cols_smem(int max_cols) {
  return static_cast<size_t>(max_cols < kSelColsSmemKeys ? max_cols : kSelColsSmemKeys) * 4;
}
cudaError_t launch_select_cols(const SelColsArgs& a, int max_need, int max_cols_now, cudaStream_t s) {
  const int slices = select_cols_slices(max_cols_now);
  return launch_k(g_pdl, k_select_cols, dim3(max_need * a.Hkv, slices), dim3(1024),
                  select_cols_smem(kSelColsSmemKeys), s, a);
}
size_t corr_cluster_smem(int hd, int grp) { return static_cast<size_t>(2) * kCorrWarps * grp * hd * 4; }
template <typename K, typename A>
cudaError_t launch_cluster(K kern, dim3 grid, dim3 block, int cluster_x, size_t smem, cudaStream_t s, const A& a) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster_x;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = g_pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int HD, int EPL, int GRP, int KM, bool SP>
cudaError_t launch_correct_sp(const CorrectArgs& a, int n_sel, cudaStream_t s) {
  if (a.cluster) {
    dim3 grid(kCorrCluster, n_sel * a.Hkv);
    return launch_cluster(k_correct_cluster<HD, EPL, GRP, KM, SP>, grid, dim3(32 * kCorrWarps), kCorrCluster,
                          corr_cluster_smem(HD, GRP), s, a);
  }
  dim3 grid(n_sel * a.Hkv, a.n_splits);
  return launch_k(g_pdl, k_correct<HD, EPL, GRP, KM, SP>, grid, dim3(256), 0, s, a);
}
template <int HD, int EPL, int GRP, int KM>
cudaError_t launch_correct_t(const CorrectArgs& a, int n_sel, cudaStream_t s) {
  return a.cv.rows ? launch_correct_sp<HD, EPL, GRP, KM, true>(a, n_sel, s)
                   : launch_correct_sp<HD, EPL, GRP, KM, false>(a, n_sel, s);
}
size_t correct_tc_smem() { return 1024 + static_cast<size_t>(10) * 64 * 128 * 2; }
// prefill tiles on the tensor cores: grid-stride over (plan entry, KV head, pass of 64 pairs)
cudaError_t launch_correct_tc(const CorrectArgs& a, int max_entries, cudaStream_t s) {
  const int npass = (a.q_tile * (a.H / a.Hkv) + 63) / 64;
  const int items = max_entries * a.Hkv * npass;
  const dim3 grid(items < kDscoreSMs ? items : kDscoreSMs);
  const size_t sm = correct_tc_smem();
  const bool sp = a.cv.rows != 0;
  switch (chain_km(a.cv.K)) {
    case 2: return sp ? launch_k(g_pdl, k_correct_tc<2, true>, grid, dim3(256), sm, s, a)
                      : launch_k(g_pdl, k_correct_tc<2, false>, grid, dim3(256), sm, s, a);
    case 4: return sp ? launch_k(g_pdl, k_correct_tc<4, true>, grid, dim3(256), sm, s, a)
                      : launch_k(g_pdl, k_correct_tc<4, false>, grid, dim3(256), sm, s, a);
    case 8: return sp ? launch_k(g_pdl, k_correct_tc<8, true>, grid, dim3(256), sm, s, a)
                      : launch_k(g_pdl, k_correct_tc<8, false>, grid, dim3(256), sm, s, a);
    case 16: return sp ? launch_k(g_pdl, k_correct_tc<16, true>, grid, dim3(256), sm, s, a)
                       : launch_k(g_pdl, k_correct_tc<16, false>, grid, dim3(256), sm, s, a);
    default: return cudaErrorInvalidValue;
  }
}

template <int HD, int EPL, int GRP>
cudaError_t launch_correct_km(const CorrectArgs& a, int n_sel, cudaStream_t s) {
  switch (chain_km(a.cv.K)) {
    case 2: return launch_correct_t<HD, EPL, GRP, 2>(a, n_sel, s);
    case 4: return launch_correct_t<HD, EPL, GRP, 4>(a, n_sel, s);
    case 8: return launch_correct_t<HD, EPL, GRP, 8>(a, n_sel, s);
    case 16: return launch_correct_t<HD, EPL, GRP, 16>(a, n_sel, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_correct(const CorrectArgs& a, int n_sel, cudaStream_t s) {
  const int grp = a.H / a.Hkv;
  if (a.tc && a.hd == 128 && !a.cluster) return launch_correct_tc(a, a.max_entries, s);
#define FL_CORR(G)                                                                   \
  case G:                                                                            \
    return a.hd == 128 ? launch_correct_km<128, 4, G>(a, n_sel, s) : launch_correct_km<64, 2, G>(a, n_sel, s);
  switch (grp) {
    FL_CORR(1)
    FL_CORR(2)
    FL_CORR(4)
    FL_CORR(8)
    default: return cudaErrorInvalidValue;
  }
#undef FL_CORR
}

// 16-CTA clusters are beyond the portable size: opt every instantiation in.
template <int HD, int EPL, int GRP, int KM, bool SP>
cudaError_t allow_big_cluster() {
  cudaError_t e =
      cudaFuncSetAttribute(k_correct_cluster<HD, EPL, GRP, KM, SP>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_correct_cluster<HD, EPL, GRP, KM, SP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(corr_cluster_smem(HD, GRP)));
  return e;
}
template <int HD, int EPL, int GRP, bool SP>
cudaError_t allow_big_cluster_sp() {
  cudaError_t e = allow_big_cluster<HD, EPL, GRP, 2, SP>();
  if (e == cudaSuccess) e = allow_big_cluster<HD, EPL, GRP, 4, SP>();
  if (e == cudaSuccess) e = allow_big_cluster<HD, EPL, GRP, 8, SP>();
  if (e == cudaSuccess) e = allow_big_cluster<HD, EPL, GRP, 16, SP>();
  return e;
}
template <int HD, int EPL, int GRP>
cudaError_t allow_big_cluster_km() {
  cudaError_t e = allow_big_cluster_sp<HD, EPL, GRP, false>();
  if (e == cudaSuccess) e = allow_big_cluster_sp<HD, EPL, GRP, true>();
  return e;
}

template <bool SP, typename Set>
void set_dscore(Set& set) {
  set(k_correct_tc<2, SP>, static_cast<int>(correct_tc_smem()));
  set(k_correct_tc<4, SP>, static_cast<int>(correct_tc_smem()));
  set(k_correct_tc<8, SP>, static_cast<int>(correct_tc_smem()));
  set(k_correct_tc<16, SP>, static_cast<int>(correct_tc_smem()));
  set(k_dscore_tc<2, SP>, static_cast<int>(dscore_tc_smem()));
  set(k_dscore_tc<4, SP>, static_cast<int>(dscore_tc_smem()));
  set(k_dscore_tc<8, SP>, static_cast<int>(dscore_tc_smem()));
  set(k_dscore_tc<16, SP>, static_cast<int>(dscore_tc_smem()));
  set(k_dscore<128, 2, SP>, static_cast<int>(dscore_smem(128)));
  set(k_dscore<128, 4, SP>, static_cast<int>(dscore_smem(128)));
  set(k_dscore<128, 8, SP>, static_cast<int>(dscore_smem(128)));
  set(k_dscore<128, 16, SP>, static_cast<int>(dscore_smem(128)));
  set(k_dscore<64, 2, SP>, static_cast<int>(dscore_smem(64)));
  set(k_dscore<64, 4, SP>, static_cast<int>(dscore_smem(64)));
  set(k_dscore<64, 8, SP>, static_cast<int>(dscore_smem(64)));
  set(k_dscore<64, 16, SP>, static_cast<int>(dscore_smem(64)));
}

// Opt every large-shared-memory kernel in to its dynamic shared memory once,
// outside any stream capture.  Returns the first error.
cudaError_t kernels_init_attrs() {
  static cudaError_t done = cudaErrorNotReady;
  if (done == cudaSuccess) return done;
  cudaError_t e = cudaSuccess;
  auto set = [&](auto* kern, int bytes) {
    cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    // all of the unified L1/shared storage as shared memory, so CTAs with large rings pair up on an SM
    if (r == cudaSuccess && bytes > 48 * 1024)
      r = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess) e = r;
  };
  set(k_attn_decode<128, 1>, static_cast<int>(attn_decode_smem(128)));
  set(k_attn_decode<128, 2>, static_cast<int>(attn_decode_smem(128)));
  set(k_attn_decode<128, 4>, static_cast<int>(attn_decode_smem(128)));
  set(k_attn_decode<128, 8>, static_cast<int>(attn_decode_smem(128)));
  set(k_attn_decode<64, 1>, static_cast<int>(attn_decode_smem(64)));
  set(k_attn_decode<64, 2>, static_cast<int>(attn_decode_smem(64)));
  set(k_attn_decode<64, 4>, static_cast<int>(attn_decode_smem(64)));
  set(k_attn_decode<64, 8>, static_cast<int>(attn_decode_smem(64)));
  set(k_select_cols, static_cast<int>(select_cols_smem(kSelColsSmemKeys)));
  set(k_topk_segments, static_cast<int>(select_cols_smem(kSelColsSmemKeys)));
  set(k_attn_prefill<128>, static_cast<int>(attn_prefill_smem(128)));
  set(k_attn_prefill<64>, static_cast<int>(attn_prefill_smem(64)));
  set(k_attn_prefill_tc<128>, static_cast<int>(attn_prefill_tc_smem(128)));
  set(k_attn_prefill_tc<64>, static_cast<int>(attn_prefill_tc_smem(64)));
  set_dscore<false>(set);
  set_dscore<true>(set);
  {
    const cudaError_t r[8] = {allow_big_cluster_km<128, 4, 1>(), allow_big_cluster_km<128, 4, 2>(),
                              allow_big_cluster_km<128, 4, 4>(), allow_big_cluster_km<128, 4, 8>(),
                              allow_big_cluster_km<64, 2, 1>(),  allow_big_cluster_km<64, 2, 2>(),
                              allow_big_cluster_km<64, 2, 4>(),  allow_big_cluster_km<64, 2, 8>()};
    for (cudaError_t x : r)
      if (e == cudaSuccess) e = x;
  }
  done = e;
  return e;
}

cudaError_t launch_pack_codes(const int8_t* src, int rows, int hd, int bits, uint8_t* dst, size_t dst_row_stride,
                              cudaStream_t s) {
  if (hd == 128)
    return launch_k(false, k_pack_codes<4>, dim3((rows + 3) / 4), dim3(128), 0, s, src, rows, hd, bits, dst,
                    dst_row_stride);
  return launch_k(false, k_pack_codes<2>, dim3((rows + 3) / 4), dim3(128), 0, s, src, rows, hd, bits, dst,
                  dst_row_stride);
}

}  // namespace fl
