// fl_gemm.cu -- the shared-block GEMMs on 5th-generation tensor cores.
//
// Both kernels split one CTA into three roles:
//   warp 0      : TMA producer (one thread) filling a shared-memory ring
//   warp 1      : TMEM owner and MMA issuer (one thread issues tcgen05.mma)
//   warps 2..5  : epilogue; warp w reads TMEM lanes 32*(w%4) .. +31 with tcgen05.ld
// Operands are bf16, K-major, 128-byte swizzled (64 elements per row of a box),
// accumulation is fp32 in TMEM.  The epilogue is fused: plain fp32 store (QKV,
// logits), scaled residual scatter-add into the fp32 hidden state (O-proj,
// down-proj), or SiLU(gate) * up into the bf16 MLP activation (gate/up, which
// keeps two accumulators).
//
// k_gemm_tc (decode, at most 64 tokens): weights on the MMA M side, tokens on
// the N side (BN = 16/32/64); the K range is split over about one CTA per SM,
// the splits of a tile forming one cluster whose partials are summed over
// distributed shared memory in rank order (or, for callers without a cluster,
// through global scratch and an atomic ticket), so results do not depend on
// CTA timing.  It can build its token operand itself from fp32 hidden rows
// (input RMSNorm).
// k_gemm_wide (prefill): persistent, 128 x 256 output tiles, two TMEM
// accumulators so that a tile's epilogue overlaps the next tile's MMAs.
#include <cooperative_groups.h>

#include "fl_device.cuh"
#include "fl_internal.h"

namespace cg = cooperative_groups;

namespace fl {

namespace {

constexpr int kThreads = 192;
constexpr int kBoxK = 64;             // bf16 elements per 128-byte swizzled row
constexpr int kABytes = 128 * kBoxK * 2;
// Shared-memory ring budget of the skinny (decode) kernel: two CTAs per SM, so
// that a dependent GEMM can become resident and start streaming its weights
// while the previous kernel still runs.  Two CTAs fit one SM's 228 KB with the
// 1 KB the hardware reserves per CTA and this kernel's 1.25 KB of slack and
// barriers: 2 * (ring + 2304 + 1024) <= 233472.
constexpr int kSmemBudgetSkinny = 113408;

// Ring and TMEM layout of the skinny kernel for BN token columns, with one or
// two (DA: gate and up) weight operands.
template <int BN, bool DA>
struct Cfg {
  static constexpr int kSmemBudget = kSmemBudgetSkinny;
  static constexpr int kNA = DA ? 2 : 1;
  static constexpr int kBBytes = BN * kBoxK * 2;
  static constexpr int kStageBytes = kNA * kABytes + kBBytes;
  static constexpr int kStagesRaw = kSmemBudget / kStageBytes;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static constexpr int kNAcc = DA ? 2 : 1;
  static constexpr int kColsNeeded = kNAcc * BN;
  static constexpr uint32_t kTmemCols = kColsNeeded <= 32 ? 32 : kColsNeeded <= 64 ? 64
                                        : kColsNeeded <= 128 ? 128 : kColsNeeded <= 256 ? 256 : 512;
  // barriers, TMEM slot, flags [0, 256); token scales [256, 512); warp sums [512, 528);
  // partial sums of squares [768, 1280)
  static constexpr int kTailBytes = 1280;
  static constexpr int kSmemBytes = 1024 /*align slack*/ + kStages * kStageBytes + kTailBytes;
  static_assert(kBBytes % 1024 == 0, "B box must keep 1024-byte alignment of the swizzle atoms");
  static_assert(kStages >= 2, "pipeline needs two stages");
};

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }

// Epilogue of the skinny kernel: accumulator row `row` of weight tile tile_m is
// output feature tile_m * 128 + row; columns col0 .. col0+15 are tokens.
__device__ __forceinline__ void epi_apply(const GemmArgs& p, int row, int col0, int tile_m, const float* v0,
                                          const float* v1) {
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const int feat = tile_m * 128 + row, tok = col0 + c;
    if (tok >= p.n_tok || feat >= p.n_feat) continue;
    if (p.epi == kEpiStore) {
      p.out[static_cast<size_t>(tok) * p.ldo + feat] = v0[c];
    } else if (p.epi == kEpiResid) {
      const int r = p.idx ? p.idx[tok] : tok;
      float* dst = p.h + static_cast<size_t>(r) * p.ldh + feat;
      *dst = *dst + p.scale * v0[c];
    } else {
      p.act[static_cast<size_t>(tok) * p.ld_act + feat] = f_to_bf16(silu_f(v0[c]) * v1[c]);
    }
  }
}

// The epilogue of one accumulator element (row, column col).  Returns the
// updated hidden-state value of a residual epilogue (0 otherwise or if the
// element is outside the output).
__device__ __forceinline__ float epi_one(const GemmArgs& p, int row, int col, int tile_m, float v0, float v1) {
  const int feat = tile_m * 128 + row, tok = col;
  if (tok >= p.n_tok || feat >= p.n_feat) return 0.f;
  if (p.epi == kEpiStore) {
    p.out[static_cast<size_t>(tok) * p.ldo + feat] = v0;
  } else if (p.epi == kEpiResid) {
    const int r = p.idx ? p.idx[tok] : tok;
    float* dst = p.h + static_cast<size_t>(r) * p.ldh + feat;
    const float hn = *dst + p.scale * v0;
    *dst = hn;
    return hn;
  } else {
    p.act[static_cast<size_t>(tok) * p.ld_act + feat] = f_to_bf16(silu_f(v0) * v1);
  }
  return 0.f;
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 2, 128;" ::: "memory"); }

// The token operand of a swap-orientation GEMM with an input RMSNorm, built by
// the four epilogue warps (t4 = 0..127) while the TMA producer streams only
// weights.  For ring slot s of k-chunk i the BN x 64 bf16 tile is written in
// the layout a 128-byte-swizzling TMA load would leave: row r at r * 128 bytes,
// 16-byte chunk j at ((j ^ (r % 8)) * 16).  The slot's full barrier expects
// this arrival besides the producer's.  Returns false if a wait ran out.
template <int BN, int STAGES, int STAGE_BYTES, int B_OFF>
__device__ __forceinline__ bool build_tokens(const GemmArgs& p, uint8_t* smem, uint64_t* full, uint64_t* empty,
                                             float* rs, float* ss_red, volatile int* xabort, int c0, int nch,
                                             int t4) {
  {
    // thread (slot, token) sums parts slot, slot + SL, ...; the SL slot sums
    // are then added in slot order, so the total has a fixed order
    constexpr int SL = 128 / BN;
    const int tok = t4 % BN, slot = t4 / BN;
    float part = 0.f;
    if (tok < p.n_tok) {
      for (int q0 = slot; q0 < p.ss_parts; q0 += 4 * SL) {
        float v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int q = q0 + u * SL;
          v[u] = q < p.ss_parts ? p.ss_in[q * p.ss_ld + tok] : 0.f;
        }
        part += (v[0] + v[1]) + (v[2] + v[3]);
      }
    }
    ss_red[slot * BN + tok] = part;
    epi_bar();
    if (t4 < BN) {
      float r = 0.f;
      if (t4 < p.n_tok) {
        float ss = 0.f;
#pragma unroll
        for (int q = 0; q < SL; ++q) ss += ss_red[q * BN + t4];
        r = rsqrtf(ss / static_cast<float>(p.in_ld) + p.in_eps);
      }
      rs[t4] = r;
    }
    epi_bar();
  }
  constexpr int EP = BN / 16;    // (row, 16-byte chunk) items per thread and k-chunk
  constexpr int CPB = 4 / EP;    // k-chunks per batch of four items
  for (int i0 = 0; i0 < nch; i0 += CPB) {
    float4 hv[4][2], gv[4][2];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u / EP, item = t4 + (u % EP) * 128;
      const int r = item >> 3, j = item & 7;
      if (i < nch && r < p.n_tok) {
        const int k = (c0 + i) * kBoxK + j * 8;
        const float* hr = p.in_h + static_cast<size_t>(p.in_idx ? p.in_idx[r] : r) * p.in_ld + k;
        hv[u][0] = *reinterpret_cast<const float4*>(hr);
        hv[u][1] = *reinterpret_cast<const float4*>(hr + 4);
        gv[u][0] = *reinterpret_cast<const float4*>(p.in_gain + k);
        gv[u][1] = *reinterpret_cast<const float4*>(p.in_gain + k + 4);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u / EP, e = u % EP;
      if (i >= nch) break;   // uniform over the 128 threads
      const int s = i % STAGES;
      if (e == 0 && i >= STAGES) {
        // the slot is reused: wait until the MMAs of k-chunk i - STAGES have read it
        if (t4 == 0) *xabort = mbar_wait(smem_u32(&empty[s]), ((i / STAGES) & 1) ^ 1u, p.status) ? 0 : 1;
        epi_bar();
        if (*xabort) return false;
      }
      const int item = t4 + e * 128;
      const int r = item >> 3, j = item & 7;
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (r < p.n_tok) {
        const float sc = rs[r];
        const float4 a = hv[u][0], b = hv[u][1], ga = gv[u][0], gb = gv[u][1];
        w.x = f_to_bf16(a.x * sc * ga.x) | (static_cast<uint32_t>(f_to_bf16(a.y * sc * ga.y)) << 16);
        w.y = f_to_bf16(a.z * sc * ga.z) | (static_cast<uint32_t>(f_to_bf16(a.w * sc * ga.w)) << 16);
        w.z = f_to_bf16(b.x * sc * gb.x) | (static_cast<uint32_t>(f_to_bf16(b.y * sc * gb.y)) << 16);
        w.w = f_to_bf16(b.z * sc * gb.z) | (static_cast<uint32_t>(f_to_bf16(b.w * sc * gb.w)) << 16);
      }
      *reinterpret_cast<uint4*>(smem + s * STAGE_BYTES + B_OFF + r * 128 + ((j ^ (r & 7)) << 4)) = w;
      if (e == EP - 1) {
        // generic-proxy stores, then visible to the tensor cores' (async-proxy) reads
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        epi_bar();
        if (t4 == 0) mbar_arrive(smem_u32(&full[s]));
      }
    }
  }
  return true;
}

template <int BN, bool DA>
__global__ void __launch_bounds__(kThreads, 2)
k_gemm_tc(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
          const __grid_constant__ CUtensorMap tmB0, const GemmArgs p, const int a_3d, const int b_3d) {
  using C = Cfg<BN, DA>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* done = empty + C::kStages;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(done + 1);
  volatile int* flags = reinterpret_cast<volatile int*>(tmem_slot + 1);  // [0] abort, [1] last-split, [2] x abort
  uint8_t* tail = smem + C::kStages * C::kStageBytes;
  float* tok_scale = reinterpret_cast<float*>(tail + 256);   // [BN] input-norm scales
  float* ssum = reinterpret_cast<float*>(tail + 512);        // [4] per-warp sums of squares
  const bool in_norm = p.in_h != nullptr;

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile_m = blockIdx.x, tile_n = blockIdx.y, split = blockIdx.z;
  const int c0 = (split * p.k_chunks) / p.splits;
  const int c1 = ((split + 1) * p.k_chunks) / p.splits;
  const int nch = c1 - c0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&full[s]), in_norm ? 2 : 1);   // + the token builders' arrival
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(done), 1);
    flags[0] = 0;
    flags[1] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmB0);
    // Weights never depend on an earlier kernel: the weight tiles of the first
    // ring slots are requested before waiting on the predecessor grid; the
    // activation tiles follow once it has completed.
    auto load_w = [&](int i, uint8_t* st, uint32_t fb) {
      const int kx = (c0 + i) * kBoxK;
      if (a_3d) {
        tma_load_3d(smem_u32(st), &tmA0, fb, kx, tile_m * 128, p.a_z);
        if (DA) tma_load_3d(smem_u32(st + kABytes), &tmA1, fb, kx, tile_m * 128, p.a_z);
      } else {
        tma_load_2d(smem_u32(st), &tmA0, fb, kx, tile_m * 128);
        if (DA) tma_load_2d(smem_u32(st + kABytes), &tmA1, fb, kx, tile_m * 128);
      }
    };
    auto load_x = [&](int i, uint8_t* st, uint32_t fb) {
      const int kx = (c0 + i) * kBoxK;
      uint8_t* sb = st + C::kNA * kABytes;
      if (b_3d) tma_load_3d(smem_u32(sb), &tmB0, fb, kx, tile_n * BN, p.b_z);
      else tma_load_2d(smem_u32(sb), &tmB0, fb, kx, tile_n * BN);
    };
    // with an input norm the token operand is built in shared memory, so the
    // producer moves weights only and never waits on the predecessor grid
    const uint32_t tx = in_norm ? C::kNA * kABytes : C::kStageBytes;
    const int pre = nch < C::kStages ? nch : C::kStages;
    for (int i = 0; i < pre; ++i) {
      uint8_t* st = smem + i * C::kStageBytes;
      const uint32_t fb = smem_u32(&full[i]);
      mbar_arrive_expect_tx(fb, tx);
      load_w(i, st, fb);
    }
    if (!in_norm) {
      pdl_wait();
      for (int i = 0; i < pre; ++i) load_x(i, smem + i * C::kStageBytes, smem_u32(&full[i]));
    }
    int issued = pre;
    for (int i = pre; i < nch; ++i) {
      const int s = i % C::kStages;
      const uint32_t ph = (i / C::kStages) & 1;
      if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u, p.status)) {
        flags[0] = 1;
        break;
      }
      uint8_t* st = smem + s * C::kStageBytes;
      const uint32_t fb = smem_u32(&full[s]);
      mbar_arrive_expect_tx(fb, tx);
      load_w(i, st, fb);
      if (!in_norm) load_x(i, st, fb);
      ++issued;
    }
    if (flags[0]) {
      // Give the copies still in flight a bounded chance to land before exit.
      for (int i = (issued > C::kStages ? issued - C::kStages : 0); i < issued; ++i)
        mbar_wait(smem_u32(&full[i % C::kStages]), (i / C::kStages) & 1, nullptr);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    constexpr uint32_t idesc = umma_idesc_bf16(128, BN);
    for (int i = 0; i < nch; ++i) {
      const int s = i % C::kStages;
      const uint32_t ph = (i / C::kStages) & 1;
      if (!mbar_wait(smem_u32(&full[s]), ph, p.status)) {
        flags[0] = 1;
        break;
      }
      tc_fence_after();
      const uint32_t a0 = smem_u32(smem + s * C::kStageBytes);
      const uint32_t a1 = a0 + kABytes;
      const uint32_t b0 = a0 + C::kNA * kABytes;
#pragma unroll
      for (int kk = 0; kk < kBoxK / 16; ++kk) {
        const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
        const uint64_t db = umma_desc_sw128(b0 + kk * 32);
        tc_mma_bf16(tmem, umma_desc_sw128(a0 + kk * 32), db, idesc, acc);
        if (DA) tc_mma_bf16(tmem + BN, umma_desc_sw128(a1 + kk * 32), db, idesc, acc);
      }
      tc_commit(smem_u32(&empty[s]));
    }
    tc_commit(smem_u32(done));
  } else if (warp >= 2) {
    // ---------------- epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;
    pdl_wait();
    if (p.stamp_start && warp == 2 && lane == 0) atomicMin(p.stamp_start, globaltimer_ns());
    if (in_norm) {
      if (!build_tokens<BN, C::kStages, C::kStageBytes, C::kNA * kABytes>(
              p, smem, full, empty, tok_scale, reinterpret_cast<float*>(tail + 768), flags + 2, c0, nch,
              (warp - 2) * 32 + lane))
        flags[0] = 1;
    }
    const bool ok = mbar_wait(smem_u32(done), 0, p.status);
    __syncwarp();   // tcgen05.ld below is warp-collective (.sync.aligned)
    tc_fence_after();
    const bool valid = ok && !flags[0] && nch > 0;
    // a split whose wait ran out contributes NaN, so the tile it feeds cannot
    // pass for a result (besides the status word, where the caller has one);
    // a split with no k-chunks contributes zero
    const float fill = (!ok || flags[0]) ? __int_as_float(0x7fc00000) : 0.f;
    const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16);
    float v0[16], v1[16];
    if (p.splits == 1) {
      for (int c = 0; c < BN; c += 16) {
        tmem_ld16(tbase + c, v0);
        if (C::kNAcc == 2) tmem_ld16(tbase + BN + c, v1);
        tc_wait_ld();
        if (valid) epi_apply(p, row, c, tile_m, v0, v1);
      }
    } else if (p.cluster) {
      // cluster split-K: park this split's partial tile in shared memory
      // ([acc][col][row], the ring is free once every MMA has completed); the
      // reduction runs after the cluster barrier below
      float* red = reinterpret_cast<float*>(smem);
      for (int c = 0; c < BN; c += 16) {
        tmem_ld16(tbase + c, v0);
        if (C::kNAcc == 2) tmem_ld16(tbase + BN + c, v1);
        tc_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          red[(c + j) * 128 + row] = valid ? v0[j] : fill;
          if (C::kNAcc == 2) red[(BN + c + j) * 128 + row] = valid ? v1[j] : fill;
        }
      }
    } else {
      // split-K: write this split's partial tile, take a ticket, the last CTA reduces.
      const size_t tile_floats = static_cast<size_t>(C::kNAcc) * BN * 128;
      float* mine = p.partial + (static_cast<size_t>(split) * gridDim.x + tile_m) * tile_floats;
      for (int c = 0; c < BN; c += 16) {
        tmem_ld16(tbase + c, v0);
        if (C::kNAcc == 2) tmem_ld16(tbase + BN + c, v1);
        tc_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          mine[static_cast<size_t>(c + j) * 128 + row] = valid ? v0[j] : fill;
          if (C::kNAcc == 2) mine[static_cast<size_t>(BN + c + j) * 128 + row] = valid ? v1[j] : fill;
        }
      }
      __threadfence();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (warp == 2 && lane == 0) {
        const int old = atomicAdd(&p.counters[tile_m], 1);
        flags[1] = (old == p.splits - 1) ? 1 : 0;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (flags[1]) {
        __threadfence();
        for (int c = 0; c < BN; c += 16) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            v0[j] = 0.f;
            v1[j] = 0.f;
          }
#pragma unroll 2
          for (int s = 0; s < p.splits; ++s) {
            const float* src = p.partial + (static_cast<size_t>(s) * gridDim.x + tile_m) * tile_floats;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              v0[j] += __ldcg(src + static_cast<size_t>(c + j) * 128 + row);
              if (C::kNAcc == 2) v1[j] += __ldcg(src + static_cast<size_t>(BN + c + j) * 128 + row);
            }
          }
          epi_apply(p, row, c, tile_m, v0, v1);
        }
        if (warp == 2 && lane == 0) p.counters[tile_m] = 0;
      }
    }
  }
  if (p.splits > 1 && p.cluster) {
    // every split of this tile is a CTA of one cluster: rank r sums the
    // partials of all ranks (in rank order) for its slice of token columns,
    // reading them from the peers' shared memory, and applies the epilogue
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (warp >= 2) {
      const int row = (warp & 3) * 32 + lane;
      const int S = p.splits, r = static_cast<int>(cluster.block_rank());
      const int per = (BN + S - 1) / S;
      const int col0 = r * per, col1 = min(BN, col0 + per);
      float* red = reinterpret_cast<float*>(smem);
      for (int cc = col0; cc < col1; ++cc) {
        // every peer's value is requested before any is summed, so the
        // distributed-shared-memory round trips overlap; the sum runs in rank order
        float pv0[kMaxClusterSplits], pv1[kMaxClusterSplits];
#pragma unroll
        for (int q = 0; q < kMaxClusterSplits; ++q) {
          pv0[q] = 0.f;
          pv1[q] = 0.f;
          if (q < S) {
            const float* peer = cluster.map_shared_rank(red, q);
            pv0[q] = peer[cc * 128 + row];
            if (C::kNAcc == 2) pv1[q] = peer[(BN + cc) * 128 + row];
          }
        }
        float v0s = 0.f, v1s = 0.f;
#pragma unroll
        for (int q = 0; q < kMaxClusterSplits; ++q) {
          v0s += pv0[q];
          v1s += pv1[q];
        }
        const float hn = epi_one(p, row, cc, tile_m, v0s, v1s);
        if (p.ss_out) {
          // this tile's share of the token's sum of squares, in a fixed order
          const float qs = warp_sum(hn * hn);
          if (lane == 0) ssum[warp - 2] = qs;
          epi_bar();
          if (warp == 2 && lane == 0 && cc < p.n_tok)
            p.ss_out[tile_m * p.ss_ld + cc] = (ssum[0] + ssum[1]) + (ssum[2] + ssum[3]);
          epi_bar();
        }
      }
    }
    cluster.sync();
  }
  tc_fence_before();
  __syncthreads();
  if (p.stamp_end && threadIdx.x == 0) atomicMax(p.stamp_end, globaltimer_ns());
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ============================================================================
// Persistent GEMM of the wide (prefill) orientation: D[m][n] = sum_k A[m][k]
// B[n][k] with A the token rows and B the weights, both bf16 K-major.  Output
// tiles are 128 tokens x 256 features (one N = 256 MMA per k-step), or with two
// weight operands 128 x (128 + 128) (two N = 128 MMAs into adjacent
// accumulator columns, for SiLU(gate) * up).  One CTA per SM walks the tiles
// t = blockIdx.x, blockIdx.x + gridDim.x, ... (feature tile fastest); the ring
// runs continuously across tile boundaries, and two 256-column TMEM
// accumulators let the epilogue of one tile overlap the MMAs of the next.
//   warp 0: TMA producer; warp 1: TMEM owner and MMA issuer; warps 2-5: epilogue
// ============================================================================
constexpr int kWideBN = 256;                                 // accumulator columns per tile
constexpr int kWideStageBytes = kABytes + kWideBN * kBoxK * 2;   // 16 KB tokens + 32 KB weights
constexpr int kWideStages = 4;
constexpr int kWideSmemBytes = 1024 + kWideStages * kWideStageBytes + 256;

// Epilogue of 16 consecutive features of one token row (vector stores when the
// 16 lie inside the output and the row is 16-byte aligned).
__device__ __forceinline__ void epi_wide16(const GemmArgs& p, int tok, int f0, const float* v0, const float* v1) {
  if (tok >= p.n_tok || f0 >= p.n_feat) return;
  const bool full = f0 + 16 <= p.n_feat;
  if (p.epi == kEpiStore) {
    float* dst = p.out + static_cast<size_t>(tok) * p.ldo + f0;
    if (full && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
#pragma unroll
      for (int c = 0; c < 16; c += 4)
        *reinterpret_cast<float4*>(dst + c) = make_float4(v0[c], v0[c + 1], v0[c + 2], v0[c + 3]);
    } else {
      for (int c = 0; c < 16 && f0 + c < p.n_feat; ++c) dst[c] = v0[c];
    }
  } else if (p.epi == kEpiResid) {
    const int r = p.idx ? p.idx[tok] : tok;
    float* dst = p.h + static_cast<size_t>(r) * p.ldh + f0;
    if (full && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
      float4 hv[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) hv[c] = *reinterpret_cast<const float4*>(dst + 4 * c);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<float4*>(dst + 4 * c) =
            make_float4(hv[c].x + p.scale * v0[4 * c], hv[c].y + p.scale * v0[4 * c + 1],
                        hv[c].z + p.scale * v0[4 * c + 2], hv[c].w + p.scale * v0[4 * c + 3]);
    } else {
      for (int c = 0; c < 16 && f0 + c < p.n_feat; ++c) dst[c] = dst[c] + p.scale * v0[c];
    }
  } else {
    uint16_t* dst = p.act + static_cast<size_t>(tok) * p.ld_act + f0;
    if (full && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
      uint32_t w[8];
#pragma unroll
      for (int c = 0; c < 8; ++c)
        w[c] = f_to_bf16(silu_f(v0[2 * c]) * v1[2 * c]) |
               (static_cast<uint32_t>(f_to_bf16(silu_f(v0[2 * c + 1]) * v1[2 * c + 1])) << 16);
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
      *reinterpret_cast<uint4*>(dst + 8) = make_uint4(w[4], w[5], w[6], w[7]);
    } else {
      for (int c = 0; c < 16 && f0 + c < p.n_feat; ++c) dst[c] = f_to_bf16(silu_f(v0[c]) * v1[c]);
    }
  }
}

template <bool DB>
__global__ void __launch_bounds__(kThreads, 1)
k_gemm_wide(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
            const __grid_constant__ CUtensorMap tmB1, const GemmArgs p, const int b_3d, const int tiles_m,
            const int tiles_n) {
  constexpr int kFeatPerTile = DB ? kWideBN / 2 : kWideBN;   // output features of one tile
  constexpr int kHalfB = 128 * kBoxK * 2;                      // one 128-row weight box
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kWideStages * kWideStageBytes);
  uint64_t* empty = full + kWideStages;
  uint64_t* acc_full = empty + kWideStages;   // [2] the MMAs of a tile have completed
  uint64_t* acc_empty = acc_full + 2;         // [2] the epilogue has read the accumulator
  uint64_t* done = acc_empty + 2;             // teardown: every issued MMA has completed
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* issued_out = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = tiles_m * tiles_n, nch = p.k_chunks;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kWideStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 4);   // one arrival per epilogue warp
    }
    mbar_init(smem_u32(done), 1);
    *abort_flag = 0;
    *issued_out = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // dependents may start only now: a dependent CTA that took TMEM on this SM
  // before this CTA's allocation would wait for this grid while holding it
  pdl_trigger();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (DB) tma_prefetch_desc(&tmB1);
    auto load_w = [&](int tile_n, int i, uint8_t* st, uint32_t fb) {
      const int kx = i * kBoxK;
      uint8_t* sb = st + kABytes;
      const int r0 = DB ? tile_n * 128 : tile_n * 256;
      const int r1 = DB ? r0 : r0 + 128;
      const CUtensorMap* m1 = DB ? &tmB1 : &tmB0;
      if (b_3d) {
        tma_load_3d(smem_u32(sb), &tmB0, fb, kx, r0, p.b_z);
        tma_load_3d(smem_u32(sb + kHalfB), m1, fb, kx, r1, p.b_z);
      } else {
        tma_load_2d(smem_u32(sb), &tmB0, fb, kx, r0);
        tma_load_2d(smem_u32(sb + kHalfB), m1, fb, kx, r1);
      }
    };
    // the weights of the first tile's first ring slots do not depend on the
    // predecessor grid: request them before waiting on it
    int it = 0, pre = 0;
    if (static_cast<int>(blockIdx.x) < n_tiles) {
      pre = nch < kWideStages ? nch : kWideStages;
      for (int i = 0; i < pre; ++i) {
        const uint32_t fb = smem_u32(&full[i]);
        mbar_arrive_expect_tx(fb, kWideStageBytes);
        load_w(static_cast<int>(blockIdx.x) % tiles_n, i, smem + i * kWideStageBytes, fb);
      }
    }
    pdl_wait();
    for (int t = blockIdx.x; t < n_tiles && !*abort_flag; t += gridDim.x) {
      const int tile_n = t % tiles_n, tile_m = t / tiles_n;
      for (int i = 0; i < nch; ++i, ++it) {
        const int s = it % kWideStages;
        uint8_t* st = smem + s * kWideStageBytes;
        const uint32_t fb = smem_u32(&full[s]);
        if (it >= pre) {
          if (it >= kWideStages &&
              !mbar_wait(smem_u32(&empty[s]), ((it / kWideStages) & 1) ^ 1u, p.status)) {
            *abort_flag = 1;
            break;
          }
          mbar_arrive_expect_tx(fb, kWideStageBytes);
          load_w(tile_n, i, st, fb);
        }
        tma_load_2d(smem_u32(st), &tmA, fb, i * kBoxK, tile_m * 128);
      }
    }
    *issued_out = it > pre ? it : pre;
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    constexpr uint32_t idesc = umma_idesc_bf16(128, DB ? 128 : 256);
    int it = 0, tl = 0;
    for (int t = blockIdx.x; t < n_tiles && !*abort_flag; t += gridDim.x, ++tl) {
      const int b = tl & 1;
      // accumulator b was last used by local tile tl - 2: wait until the epilogue has read it
      if (tl >= 2 && !mbar_wait(smem_u32(&acc_empty[b]), ((tl >> 1) & 1) ^ 1u, p.status)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t acc = tmem + b * kWideBN;
      bool ok = true;
      for (int i = 0; i < nch; ++i, ++it) {
        const int s = it % kWideStages;
        if (!mbar_wait(smem_u32(&full[s]), (it / kWideStages) & 1, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(smem + s * kWideStageBytes);
        const uint32_t b0 = a0 + kABytes;
#pragma unroll
        for (int kk = 0; kk < kBoxK / 16; ++kk) {
          const uint32_t accf = (i > 0 || kk > 0) ? 1u : 0u;
          const uint64_t da = umma_desc_sw128(a0 + kk * 32);
          tc_mma_bf16(acc, da, umma_desc_sw128(b0 + kk * 32), idesc, accf);
          if (DB) tc_mma_bf16(acc + 128, da, umma_desc_sw128(b0 + kHalfB + kk * 32), idesc, accf);
        }
        tc_commit(smem_u32(&empty[s]));
      }
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      tc_commit(smem_u32(&acc_full[b]));
    }
  } else if (warp >= 2) {
    // ---------------- epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31
    const int q = warp & 3;
    const int row = q * 32 + lane;
    pdl_wait();
    if (p.stamp_start && warp == 2 && lane == 0) atomicMin(p.stamp_start, globaltimer_ns());
    int tl = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tl) {
      const int b = tl & 1;
      if (!mbar_wait(smem_u32(&acc_full[b]), (tl >> 1) & 1, p.status)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int tile_n = t % tiles_n, tile_m = t / tiles_n;
      const uint32_t tb = tmem + b * kWideBN + (static_cast<uint32_t>(q * 32) << 16);
      const int tok = tile_m * 128 + row;
#pragma unroll 1
      for (int c = 0; c < kFeatPerTile; c += 16) {
        float v0[16], v1[16];
        tmem_ld16(tb + c, v0);
        if (DB) tmem_ld16(tb + 128 + c, v1);
        tc_wait_ld();
        epi_wide16(p, tok, tile_n * kFeatPerTile + c, v0, v1);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&acc_empty[b]));
    }
  }
  __syncthreads();
  if (*abort_flag) {
    // a wait ran out: let every issued MMA complete and the copies still in
    // flight land (both bounded) before TMEM and the ring are released
    if (warp == 1 && lane == 0) {
      tc_commit(smem_u32(done));
      mbar_wait(smem_u32(done), 0, nullptr);
    }
    if (warp == 0 && lane == 0) {
      const int issued = *issued_out;
      for (int i = (issued > kWideStages ? issued - kWideStages : 0); i < issued; ++i)
        mbar_wait(smem_u32(&full[i % kWideStages]), (i / kWideStages) & 1, nullptr);
    }
    __syncthreads();
  }
  tc_fence_before();
  __syncthreads();
  if (p.stamp_end && threadIdx.x == 0) atomicMax(p.stamp_end, globaltimer_ns());
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int BN, bool DA>
cudaError_t launch_one(const GemmLaunch& g, cudaStream_t stream) {
  using C = Cfg<BN, DA>;
  auto kern = k_gemm_tc<BN, DA>;
  const CUtensorMap& a1 = g.a1 ? *g.a1 : *g.a0;
  if (g.args.cluster && g.args.splits > 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = g.grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = g.args.splits;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = g.pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, *g.a0, a1, *g.b0, g.args, g.a_3d, g.b_3d);
  }
  return launch_k(g.pdl, kern, g.grid, dim3(kThreads), C::kSmemBytes, stream, *g.a0, a1, *g.b0, g.args, g.a_3d,
                  g.b_3d);
}

template <bool DB>
cudaError_t launch_wide(const GemmLaunch& g, cudaStream_t stream) {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  constexpr int kFeat = DB ? kWideBN / 2 : kWideBN;
  const int tiles_m = (g.args.n_tok + 127) / 128;
  const int tiles_n = (g.args.n_feat + kFeat - 1) / kFeat;
  const int tiles = tiles_m * tiles_n;
  if (tiles <= 0) return cudaSuccess;
  const CUtensorMap& b1 = g.b1 ? *g.b1 : *g.b0;
  return launch_k(g.pdl, k_gemm_wide<DB>, dim3(tiles < sms ? tiles : sms), dim3(kThreads), kWideSmemBytes, stream,
                  *g.a0, *g.b0, b1, g.args, g.b_3d, tiles_m, tiles_n);
}

template <bool DB>
cudaError_t set_attr_wide() {
  cudaError_t e = cudaFuncSetAttribute(k_gemm_wide<DB>, cudaFuncAttributeMaxDynamicSharedMemorySize, kWideSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k_gemm_wide<DB>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  return e;
}

template <int BN, bool DA>
cudaError_t set_attr() {
  auto kern = k_gemm_tc<BN, DA>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<BN, DA>::kSmemBytes);
  // all of the SM's unified L1/shared storage as shared memory, so two skinny CTAs are resident
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  // split-K clusters of the skinny orientation may hold up to 16 CTAs
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

}  // namespace

// Opt every GEMM instantiation in to its dynamic shared memory once, outside any capture.
cudaError_t gemm_init_attrs() {
  static cudaError_t done = cudaErrorNotReady;
  if (done == cudaSuccess) return done;
  const cudaError_t r[8] = {set_attr<16, true>(), set_attr<16, false>(), set_attr<32, true>(), set_attr<32, false>(),
                            set_attr<64, true>(), set_attr<64, false>(), set_attr_wide<true>(), set_attr_wide<false>()};
  done = cudaSuccess;
  for (cudaError_t e : r)
    if (e != cudaSuccess) done = e;
  return done;
}

size_t gemm_partial_floats(int bn, int dual, int tiles, int splits) {
  if (splits <= 1) return 0;
  return static_cast<size_t>(splits) * tiles * (dual ? 2 : 1) * bn * 128;
}

cudaError_t launch_gemm(const GemmLaunch& g, cudaStream_t stream) {
  const bool da = g.a1 != nullptr, db = g.b1 != nullptr;
  if (da && db) return cudaErrorInvalidValue;
  if (g.args.swap) {
    if (db) return cudaErrorInvalidValue;
    switch (g.bn) {
      case 16: return da ? launch_one<16, true>(g, stream) : launch_one<16, false>(g, stream);
      case 32: return da ? launch_one<32, true>(g, stream) : launch_one<32, false>(g, stream);
      case 64: return da ? launch_one<64, true>(g, stream) : launch_one<64, false>(g, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  if (da || g.bn != 128 || g.args.splits != 1 || g.a_3d) return cudaErrorInvalidValue;
  return db ? launch_wide<true>(g, stream) : launch_wide<false>(g, stream);
}

// ---------------------------------------------------------------- tensor maps
namespace {
using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeFn get_encode() {
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(ptr);
  }
  return fn;
}
}  // namespace

bool encode_tmap_bf16(CUtensorMap* map, const void* base, uint64_t k, uint64_t rows, uint64_t layers,
                      uint32_t box_rows) {
  EncodeFn fn = get_encode();
  if (!fn || !base || (reinterpret_cast<uintptr_t>(base) & 15) || (k * 2) % 16 != 0 || box_rows == 0 ||
      box_rows > 256)
    return false;
  const cuuint32_t rank = layers > 0 ? 3 : 2;
  cuuint64_t dims[3] = {k, rows, layers > 0 ? layers : 1};
  cuuint64_t strides[2] = {k * 2, k * 2 * rows};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(kBoxK), box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace fl
