// fl_cache.cuh -- layout of the KV cache in HBM and the per-lane chain
// reconstruction shared by the attention-side kernels.
//
// Lazy layout (resid_bits 4 or 2):
//   base   bf16  [M][2][B][Hkv][T][hd]            loop-1 K (0) and V (1)
//   codes  u8    [M][K-1][2][B][Hkv][R][hd*b/8]   residual codes of loops 2..K
//   scales fp16  [M][K-1][2][B][Hkv][R][hd/g]     per-group scales of loops 2..K
// with R = T (one residual row per position) or, with sparse residual storage,
// R = rows: a pool of rows per (layer, loop, K/V, sequence, KV head) holding the
// residuals of the tokens that loop recomputed only, and an index
//   ridx   int32 [M][K-1][B][T]  pool row of (layer, loop, sequence, position), -1 = zero residual
//   rcount int32 [M][K-1][B]     pool rows in use (rows are taken in position order)
// Dense layout (resid_bits 16): per_loop [M][K][2][B][Hkv][T][hd]; last_loop keeps
// one loop slot, [M][1][2][B][Hkv][T][hd], which every loop overwrites
// Tokens of one (sequence, KV head) are contiguous so a decode step streams them.
// The reconstructed KV of loop m is base + code*scale of loops 2..m, added in
// loop order in fp32 ("FlashLoop ...", abstract: each loop's KV as a
// low-bit residual over the previous loop's).  code*scale is exact in fp32 (|code| <= 7, 11-bit scale).
#pragma once
#include "fl_device.cuh"

namespace fl {

struct CacheView {
  int M, K, B, Hkv, T, hd, g, bits, dense;
  int lg;   // log2(g): g is a power of two (32, 64, 128, or hd)
  uint16_t* base;
  uint8_t* codes;
  uint16_t* scales;
  int rows;          // sparse residual storage: pool rows per (layer, loop, K/V, sequence, KV head); 0: R = T
  int32_t* ridx;     // sparse: [M][K-1][B][T]
  int* rcount;       // sparse: [M][K-1][B]

  __host__ __device__ int pool_rows() const { return rows ? rows : T; }
  __host__ __device__ size_t ridx_index(int j, int l, int b, int t) const {
    return ((static_cast<size_t>(j) * (K - 1) + (l - 2)) * B + b) * T + t;
  }
  // pool row of the loop-l residual of (layer j, sequence b, position t); -1: zero residual
  __device__ __forceinline__ int res_row(int j, int l, int b, int t) const {
    return rows ? ridx[ridx_index(j, l, b, t)] : t;
  }

  __host__ __device__ size_t row_bytes_codes() const { return static_cast<size_t>(hd) * bits / 8; }
  __host__ __device__ uint16_t* base_row(int j, int kv, int b, int h, int t) const {
    return base + ((((static_cast<size_t>(j) * 2 + kv) * B + b) * Hkv + h) * T + t) * hd;
  }
  // dense KV of loop l in 1..K: per-loop slots, or (K == 1, last_loop mode) one
  // slot that every loop overwrites
  __host__ __device__ int dense_slot(int l) const { return K == 1 ? 0 : l - 1; }
  __host__ __device__ uint16_t* dense_row(int j, int l, int kv, int b, int h, int t) const {
    return base + (((((static_cast<size_t>(j) * K + dense_slot(l)) * 2 + kv) * B + b) * Hkv + h) * T + t) * hd;
  }
  // residual row r of a pool (r = the position t without sparse storage)
  __host__ __device__ size_t res_index(int j, int l, int kv, int b, int h, int r) const {
    return ((((static_cast<size_t>(j) * (K - 1) + (l - 2)) * 2 + kv) * B + b) * Hkv + h) * pool_rows() + r;
  }
  __host__ __device__ uint8_t* code_row(int j, int l, int kv, int b, int h, int r) const {
    return codes + res_index(j, l, kv, b, h, r) * row_bytes_codes();
  }
  __host__ __device__ uint16_t* scale_row(int j, int l, int kv, int b, int h, int r) const {
    return scales + res_index(j, l, kv, b, h, r) * (hd >> lg);
  }
};

__device__ __forceinline__ int sext(int v, int bits) { return (v << (32 - bits)) >> (32 - bits); }

// ---------------------------------------------------------------- residual quantiser
// (the quantiser's scale and code rules, shared by its kernels)
// The hardware reciprocal approximation (PTX rcp.approx, within 1 ulp of 1/x).
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The group scale s = fp16_RU(RN(absmax / qmax)) (0 for an all-zero group) as fp16 bits.
__device__ __forceinline__ uint16_t quant_scale(float absmax, int qm) {
  return __half_as_ushort(__float2half_ru(qm == 1 ? absmax : __fdiv_rn(absmax, static_cast<float>(qm))));
}

// code = clamp(rint(RN(r / s)), -qm, qm), ties to even, for the group scale s
// (inv = rcp_approx(s), or 0 when s = 0).  Since s >= absmax / qmax up to one
// fp32 rounding, |r / s| < 7.01; q = r * inv then lies within 7.01 * 1.5 * 2^-23
// of r / s, and so within 1.6 * 2^-20 of the correctly rounded quotient Q.  When
// q is farther than 2^-18 from every half-integer, q and Q round to the same
// integer; otherwise Q itself is computed.  Rounding to an integer: q + 1.5 * 2^23
// lies in [2^23, 2^24), where the fp32 spacing is 1, so the addition rounds q to
// the nearest integer (ties to even) and leaves it, offset by 2^22, in the low
// bits of the sum.  (With s = 0, q = 0 and the exact branch is never taken.)
__device__ __forceinline__ int quant_code(float r, float s, float inv, int qm) {
  constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23
  const float q = r * inv;
  float t = __fadd_rn(q, kMagic);
  const float d = __fsub_rn(q, __fsub_rn(t, kMagic));   // q - rint(q), exact
  if (fabsf(d) >= 0.5f - 0x1p-18f) t = __fadd_rn(__fdiv_rn(r, s), kMagic);
  const int c = __float_as_int(t) - 0x4B400000;
  return c > qm ? qm : (c < -qm ? -qm : c);
}

// Largest loop count K a context supports; kernels that reconstruct the chain
// are instantiated for KM in {2, 4, 8, 16}, the smallest power of two >= K, so
// the unrolled reconstruction issues no work for loops that cannot exist.
constexpr int kMaxLoops = 16;
inline int chain_km(int K) { return K <= 2 ? 2 : K <= 4 ? 4 : K <= 8 ? 8 : 16; }

// Reconstructions to loop m_lo and to loop m_hi (m_lo <= m_hi <= KM) of one
// row; lane holds EPL values of each; SP: the sparse residual layout, whose
// pool rows (from chain_rows) may be passed in when K and V of a position are
// both rebuilt.  All loads (base row, residual codes and
// scales of loops 2..m_hi) are issued before any arithmetic so their latencies
// overlap; the adds then run in loop order, as the definition requires.
// Sparse layout: the pool rows of levels 2..m_hi of position t (-1 for none),
// shared by K, V and every KV head of the position.
template <int KM>
__device__ __forceinline__ void chain_rows(const CacheView& cv, int j, int b, int t, int m_hi, int* rr) {
#pragma unroll
  for (int q = 0; q < KM - 1; ++q) rr[q] = q + 2 <= m_hi ? cv.ridx[cv.ridx_index(j, q + 2, b, t)] : -1;
}

template <int EPL, int KM, bool SP>
__device__ __forceinline__ void chain_lane2(const CacheView& cv, int j, int kv, int b, int h, int t, int m_lo,
                                            int m_hi, int lane, float* lo, float* hi, const int* rows_in = nullptr) {
  const uint16_t* br = cv.base_row(j, kv, b, h, t) + lane * EPL;
  uint32_t braw[EPL == 4 ? 2 : 1];
  if (EPL == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(br);
    braw[0] = u.x;
    braw[EPL == 4 ? 1 : 0] = u.y;
  } else {
    braw[0] = *reinterpret_cast<const uint32_t*>(br);
  }
  const int gi = (lane * EPL) >> cv.lg;
  const size_t rb = cv.row_bytes_codes(), ns = cv.hd >> cv.lg;
  // residual row of level q + 2: SP false (one row per position), the row of
  // level 2 plus q * step; SP true (sparse storage), the pool row from the
  // index, all index loads first, -1 for none.  A level without a row
  // contributes code 0 x scale 0, as a stored zero row does.  The layout is a
  // template parameter so the dense layout's walk carries no index registers.
  uint32_t craw[KM - 1];
  uint16_t sraw[KM - 1];
  auto load_level = [&](int q, size_t ri) {
    const uint8_t* row = cv.codes + ri * rb;
    if (EPL == 4) {
      craw[q] = cv.bits == 4 ? static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(row + lane * 2))
                             : static_cast<uint32_t>(row[lane]);
    } else {
      craw[q] = cv.bits == 4 ? static_cast<uint32_t>(row[lane])
                             : static_cast<uint32_t>((row[lane >> 1] >> ((lane & 1) * 4)) & 0xF);
    }
    sraw[q] = cv.scales[ri * ns + gi];
  };
  if (!SP) {
    const size_t step = static_cast<size_t>(2) * cv.B * cv.Hkv * cv.T;   // rows between consecutive loops
    const size_t r0 = ((((static_cast<size_t>(j) * (cv.K - 1)) * 2 + kv) * cv.B + b) * cv.Hkv + h) * cv.T + t;
#pragma unroll
    for (int q = 0; q < KM - 1; ++q) {
      craw[q] = 0u;
      sraw[q] = 0;
      if (q + 2 <= m_hi) load_level(q, r0 + q * step);
    }
  } else {
    const size_t step = static_cast<size_t>(2) * cv.B * cv.Hkv * cv.rows;
    const size_t q0 = ((((static_cast<size_t>(j) * (cv.K - 1)) * 2 + kv) * cv.B + b) * cv.Hkv + h) * cv.rows;
    int rr[KM - 1];
    if (rows_in) {
#pragma unroll
      for (int q = 0; q < KM - 1; ++q) rr[q] = rows_in[q];
    } else {
      chain_rows<KM>(cv, j, b, t, m_hi, rr);
    }
#pragma unroll
    for (int q = 0; q < KM - 1; ++q) {
      craw[q] = 0u;
      sraw[q] = 0;
      if (rr[q] >= 0) load_level(q, q0 + q * step + static_cast<size_t>(rr[q]));
    }
  }
  float acc[EPL];
  if (EPL == 4) {
    acc[0] = bf16_to_f(braw[0] & 0xFFFF);
    acc[1] = bf16_to_f(braw[0] >> 16);
    acc[EPL == 4 ? 2 : 0] = bf16_to_f(braw[EPL == 4 ? 1 : 0] & 0xFFFF);
    acc[EPL == 4 ? 3 : 1] = bf16_to_f(braw[EPL == 4 ? 1 : 0] >> 16);
  } else {
    acc[0] = bf16_to_f(braw[0] & 0xFFFF);
    acc[1] = bf16_to_f(braw[0] >> 16);
  }
  if (m_lo <= 1) {
#pragma unroll
    for (int e = 0; e < EPL; ++e) lo[e] = acc[e];
  }
  const int fb = cv.bits;
#pragma unroll
  for (int q = 0; q < KM - 1; ++q) {
    if (q + 2 <= m_hi) {
      const float sc = half_bits_to_f(sraw[q]);
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const int c = sext(static_cast<int>((craw[q] >> (fb * e)) & ((1u << fb) - 1)), fb);
        acc[e] = __fadd_rn(acc[e], __fmul_rn(static_cast<float>(c), sc));
      }
      if (q + 2 == m_lo) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) lo[e] = acc[e];
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) hi[e] = acc[e];
}

}  // namespace fl
