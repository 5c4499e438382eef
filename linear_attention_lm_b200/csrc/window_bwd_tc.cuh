// window_bwd_tc.cuh -- gradient of the sliding-window causal softmax attention
// on the sm_100a tensor cores (bf16 inputs, d_h = 64 or 128).
//
// The forward (Based README, introduction, item 1): for query t the keys are
// s in [max(0, t-W+1), t] (W <= 64), s_ts = q_t.k_s / sqrt(d_h),
// P_ts = softmax_s(s_ts), y_t = sum_s P_ts v_s.  Its gradient, given dy:
//   dP_ts = dy_t . v_s,   delta_t = sum_s P_ts dP_ts,   dS_ts = P_ts (dP_ts - delta_t),
//   dq_t = sum_s dS_ts k_s / sqrt(d_h),  dk_s = sum_t dS_ts q_t / sqrt(d_h),
//   dv_s = sum_t P_ts dy_t.
// Two kernels over 128-row tiles, each one CTA of 128 threads (thread r owns
// row r of the tile and TMEM lane r; thread 0 issues the loads and the MMAs):
//
//   window_bwd_tc_q:  query tile [t0, t0+128); its keys lie in [t0-63, t0+127],
//     staged as the 192 rows [t0-64, t0+128) of K and V (rows outside [0, L)
//     read as zero).
//       S  = Q K^T, dP = dY V^T        (M=128, N=192, K=d_h)          -> TMEM
//       per row, over its band: m, l (the softmax), P, delta, dS    (CUDA cores)
//       dQ = dS K                      (A = dS, bf16, from TMEM; K=192) -> TMEM
//     writes dq and, per query, the scaled row max, the row sum and delta to
//     the workspace (planes [3][BH][L]).
//   window_bwd_tc_kv: key tile [s0, s0+128); the queries that see it lie in
//     [s0, s0+190], staged as the 192 rows [s0, s0+192) of Q and dY.
//       S^T = K Q^T, dP^T = V dY^T     (M=128, N=192, K=d_h)          -> TMEM
//       per key row, over its band: P^T from the stored statistics, dS^T
//       dV = P^T dY, dK = dS^T Q       (A from TMEM, bf16; K=192)      -> TMEM
//
// Band layout: row r of quadrant w reads the 96 staged columns [32w, 32w+96),
// which hold its whole band; P or dS go back into TMEM as bf16 pairs (the A
// operand of the next MMA), the band of quadrant w in packed columns
// [16w, 16w+48) and zeros in the rest of the 96.
//
// Operand precision: q, k, v, dy are the bf16 inputs; P and dS are rounded to
// bf16 for the MMAs; the softmax statistics, delta, the accumulators and the
// outputs are fp32.  A CTA takes its tensor memory only once its tiles have
// landed, so the loads of the next CTA on the SM overlap this one's work.
#pragma once

#include "common.cuh"
#include "umma.cuh"

namespace based {

constexpr int kWgT = 128;       // rows of the CTA's own tile
constexpr int kWgN = 192;       // staged rows of the other side
constexpr int kWgThreads = 128;

template <int DH>
struct WgLayout {
  static constexpr int kOwn = kWgT * DH * 2;     // [128 x DH] bf16, 64-column SW128 blocks
  static constexpr int kOther = kWgN * DH * 2;   // [192 x DH]
  // q kernel: Q, dY (own rows), K, V (staged); kv kernel: K, V (own), Q, dY (staged)
  static constexpr int kA0 = 0;
  static constexpr int kA1 = kA0 + kOwn;
  static constexpr int kB0 = kA1 + kOwn;
  static constexpr int kB1 = kB0 + kOther;
  static constexpr int kStats = kB1 + kOther;    // kv kernel: [3][192] fp32
  static constexpr int kBar = kStats + 3 * kWgN * 4;
  static constexpr int kBytes = kBar + 64;
  static constexpr size_t kSmem = kBytes + 1024;
  static constexpr uint32_t kTx = 2u * (kOwn + kOther);
  // TMEM: S (or S^T) at 0, dP (or dP^T) at 192, then the d_h-wide accumulators
  static constexpr int kTmS = 0, kTmP = 192, kTmAcc = 384;
  static_assert(kA1 % 1024 == 0 && kB0 % 1024 == 0 && kB1 % 1024 == 0, "SW128 tiles");
  static_assert(kSmem <= 232448, "shared memory budget");
};

// 96 packed bf16-pair columns of this thread's lane at `base`: the band words
// pk[0..48) at offset 16w, zero elsewhere (w = quadrant of the warp).
__device__ __forceinline__ void wg_store_band(uint32_t base, int w, const uint32_t* pk) {
  uint32_t zero[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) zero[j] = 0u;
  if (w == 0) {
    umma::tmem_st32_nowait(base, pk);
    umma::tmem_st16_nowait(base + 32, pk + 32);
    umma::tmem_st32_nowait(base + 48, zero);
    umma::tmem_st16_nowait(base + 80, zero);
  } else if (w == 1) {
    umma::tmem_st16_nowait(base, zero);
    umma::tmem_st32_nowait(base + 16, pk);
    umma::tmem_st16_nowait(base + 48, pk + 32);
    umma::tmem_st32_nowait(base + 64, zero);
  } else if (w == 2) {
    umma::tmem_st32_nowait(base, zero);
    umma::tmem_st32_nowait(base + 32, pk);
    umma::tmem_st16_nowait(base + 64, pk + 32);
    umma::tmem_st16_nowait(base + 80, zero);
  } else {
    umma::tmem_st32_nowait(base, zero);
    umma::tmem_st16_nowait(base + 32, zero);
    umma::tmem_st32_nowait(base + 48, pk);
    umma::tmem_st16_nowait(base + 80, pk + 32);
  }
}

__device__ __forceinline__ uint32_t wg_pack(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Packed pairs of fp32 (each lane of an f32x2 operation rounds like its scalar
// form, so these give the scalar results, two at a time).
__device__ __forceinline__ uint64_t wg_f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void wg_unf2(uint64_t v, float* lo, float* hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(*lo), "=f"(*hi) : "l"(v));
}
__device__ __forceinline__ uint64_t wg_fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t wg_mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t wg_add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Row r of an fp32 accumulator [128 x DH] in TMEM, times `scale`, to row `row`
// of a [L, DH] fp32 tensor (skipped past L).
template <int DH>
__device__ __forceinline__ void wg_store_acc(uint32_t taddr, float scale, float* dst, bool live) {
#pragma unroll
  for (int blk = 0; blk < DH / 64; ++blk) {
    float o[64];
    umma::tmem_ld64(taddr + blk * 64, o);
    if (live) {
      float4* d4 = reinterpret_cast<float4*>(dst + blk * 64);
#pragma unroll
      for (int j = 0; j < 16; ++j)
        d4[j] = make_float4(o[4 * j] * scale, o[4 * j + 1] * scale, o[4 * j + 2] * scale,
                            o[4 * j + 3] * scale);
    }
  }
}

struct WgParams {
  float* dq;
  float* dk;
  float* dv;
  float* ws;      // [3][BH][L]: scaled row max, row sum, delta
  int L, W, n_tiles, BH;
};

// ---------------------------------------------------------------------------
// query side: dq and the per-query statistics
// ---------------------------------------------------------------------------
template <int DH>
__global__ void __launch_bounds__(kWgThreads, 1)
    window_bwd_tc_q_kernel(const __grid_constant__ CUtensorMap qmap,
                           const __grid_constant__ CUtensorMap dymap,
                           const __grid_constant__ CUtensorMap kmap,
                           const __grid_constant__ CUtensorMap vmap, const WgParams p) {
  using Lay = WgLayout<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bar_ld = reinterpret_cast<uint64_t*>(sm + Lay::kBar);
  uint64_t* bar_s = bar_ld + 1;
  uint64_t* bar_q = bar_ld + 2;
  uint64_t* bar_fin = bar_ld + 3;  // every MMA of this CTA complete (commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_ld + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // a dependent launch: the previous kernel has finished before any global access
  umma::grid_dep_wait();
  umma::grid_dep_launch();
  const int tile = blockIdx.x % p.n_tiles;
  const int bh = blockIdx.x / p.n_tiles;
  const int t0 = tile * kWgT;
  const int L = p.L, W = p.W;

  if (tid == 0) {
    umma::mbar_init(bar_ld, 1);
    umma::mbar_init(bar_s, 1);
    umma::mbar_init(bar_q, 1);
    umma::mbar_init(bar_fin, 1);
    umma::fence_mbar_init();
    umma::mbar_arrive_expect_tx(bar_ld, Lay::kTx);
#pragma unroll
    for (int b = 0; b < DH / 64; ++b) {
      umma::tma_load_3d(sm + Lay::kA0 + b * kWgT * 128, &qmap, bar_ld, b * 64, t0, bh);
      umma::tma_load_3d(sm + Lay::kA1 + b * kWgT * 128, &dymap, bar_ld, b * 64, t0, bh);
      umma::tma_load_3d(sm + Lay::kB0 + b * kWgN * 128, &kmap, bar_ld, b * 64, t0 - 64, bh);
      umma::tma_load_3d(sm + Lay::kB1 + b * kWgN * 128, &vmap, bar_ld, b * 64, t0 - 64, bh);
    }
  }
  __syncthreads();
  // tensor memory only once the tiles have landed
  const bool ld_ok = umma::mbar_wait(bar_ld, 0);
  bool ok = ld_ok;
  if (warp == 0) {
    umma::tmem_alloc(tmem_slot, 512);
    umma::tmem_relinquish();
  }
  umma::tc_fence_before();
  ok = __syncthreads_and(ok);
  umma::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_lane = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t sQ = umma::smem_u32(sm + Lay::kA0), sdY = umma::smem_u32(sm + Lay::kA1),
                 sK = umma::smem_u32(sm + Lay::kB0), sV = umma::smem_u32(sm + Lay::kB1);
  const int r = tid, t = t0 + r;
  const bool live = t < L;

  if (ok && tid == 0) {
    const uint32_t id = umma::idesc_bf16(kWgT, kWgN, false, false);
#pragma unroll
    for (int k0 = 0; k0 < DH; k0 += 16) {
      umma::mma_bf16(tmem + Lay::kTmS, umma::desc_kmajor_sw128(sQ, k0, kWgT),
                     umma::desc_kmajor_sw128(sK, k0, kWgN), id, k0 > 0);
      umma::mma_bf16(tmem + Lay::kTmP, umma::desc_kmajor_sw128(sdY, k0, kWgT),
                     umma::desc_kmajor_sw128(sV, k0, kWgN), id, k0 > 0);
    }
    umma::mma_commit(bar_s);
  }
  if (ok) ok = umma::mbar_wait(bar_s, 0);
  umma::tc_fence_after();
  if (__syncthreads_and(ok)) {
    // staged column c holds key s = t0 - 64 + c; row t sees s in
    // [max(0, t-W+1), t], i.e. local columns [lo, hi] of its 96
    const int cb = warp * 32;
    const int lo = max(max(r + 1, 64 - t0), t - W + 1 - (t0 - 64)) - cb;
    const int hi = lane + 64;
    const float scale = rsqrtf((float)DH) * 1.4426950408889634f;  // 1/sqrt(dh) * log2(e)
    float pv[96];
    umma::tmem_ld64_32(tmem + Lay::kTmS + tm_lane + cb, tmem + Lay::kTmS + tm_lane + cb + 64, pv);
    // scores outside the window become -inf once, so the max and the
    // exponentials need no mask (exp2(-inf) = 0); when every row sees a whole
    // window of 64 keys (lo = lane + 1) only the two ragged ends are tested
    if (W == 64 && t0 >= 64) {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i <= lane) pv[i] = -INFINITY;
#pragma unroll
      for (int i = 65; i < 96; ++i)
        if (i > hi) pv[i] = -INFINITY;
    } else {
#pragma unroll
      for (int i = 0; i < 96; ++i)
        if (i < lo || i > hi) pv[i] = -INFINITY;
    }
    float mp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int i = 0; i < 96; ++i) mp[i & 3] = fmaxf(mp[i & 3], pv[i]);
    const float ms = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])) * scale;
    // weights, row sum, delta = sum P dP and dS = P (dP - delta), in packed pairs
    // (pair j feeds partial sums 2 (j & 1) + {0, 1}, as a scalar loop over i & 3)
    const uint64_t sc2 = wg_f2(scale, scale), nm2 = wg_f2(-ms, -ms);
    uint64_t lp2[2] = {wg_f2(0.0f, 0.0f), wg_f2(0.0f, 0.0f)};
#pragma unroll
    for (int j = 0; j < 48; ++j) {
      float a, b;
      wg_unf2(wg_fma2(wg_f2(pv[2 * j], pv[2 * j + 1]), sc2, nm2), &a, &b);
      pv[2 * j] = ex2_approx(a);
      pv[2 * j + 1] = ex2_approx(b);
      lp2[j & 1] = wg_add2(lp2[j & 1], wg_f2(pv[2 * j], pv[2 * j + 1]));
    }
    float lq[4];
    wg_unf2(lp2[0], &lq[0], &lq[1]);
    wg_unf2(lp2[1], &lq[2], &lq[3]);
    const float l = (lq[0] + lq[1]) + (lq[2] + lq[3]);  // >= 1 (the maximum contributes 1)
    const float inv_l = 1.0f / l;
    float dp[96];
    umma::tmem_ld64_32(tmem + Lay::kTmP + tm_lane + cb, tmem + Lay::kTmP + tm_lane + cb + 64, dp);
    const uint64_t il2 = wg_f2(inv_l, inv_l);
    uint64_t dl2[2] = {wg_f2(0.0f, 0.0f), wg_f2(0.0f, 0.0f)};
#pragma unroll
    for (int j = 0; j < 48; ++j) {
      const uint64_t p2 = wg_mul2(wg_f2(pv[2 * j], pv[2 * j + 1]), il2);
      wg_unf2(p2, &pv[2 * j], &pv[2 * j + 1]);
      dl2[j & 1] = wg_fma2(p2, wg_f2(dp[2 * j], dp[2 * j + 1]), dl2[j & 1]);
    }
    float dq4[4];
    wg_unf2(dl2[0], &dq4[0], &dq4[1]);
    wg_unf2(dl2[1], &dq4[2], &dq4[3]);
    const float delta = (dq4[0] + dq4[1]) + (dq4[2] + dq4[3]);
    const uint64_t nd2 = wg_f2(-delta, -delta);
    uint32_t pk[48];
#pragma unroll
    for (int j = 0; j < 48; ++j) {
      float a, b;
      wg_unf2(wg_mul2(wg_f2(pv[2 * j], pv[2 * j + 1]),
                      wg_add2(wg_f2(dp[2 * j], dp[2 * j + 1]), nd2)), &a, &b);
      pk[j] = wg_pack(a, b);
    }
    wg_store_band(tmem + Lay::kTmS + tm_lane, warp, pk);
    umma::tmem_wait_st();
    if (live) {
      const size_t plane = (size_t)p.BH * L, at = (size_t)bh * L + t;
      p.ws[at] = ms;
      p.ws[plane + at] = l;
      p.ws[2 * plane + at] = delta;
    }
  } else {
    ok = false;
  }
  umma::tc_fence_before();
  ok = __syncthreads_and(ok);
  umma::tc_fence_after();
  if (ok && tid == 0) {
    // dQ = dS K: A = dS (TMEM, K = 192 keys), B = the staged K rows (N = d_h, MN-major)
    const uint32_t id = umma::idesc_bf16(kWgT, DH, false, true);
#pragma unroll
    for (int k0 = 0; k0 < kWgN; k0 += 16)
      umma::mma_ts(tmem + Lay::kTmAcc, tmem + Lay::kTmS + k0 / 2,
                   umma::desc_mnmajor_sw128(sK, k0, kWgN), id, k0 > 0);
    umma::mma_commit(bar_q);
  }
  if (ok) ok = umma::mbar_wait(bar_q, 0);
  umma::tc_fence_after();
  if (__syncthreads_and(ok)) {
    wg_store_acc<DH>(tmem + Lay::kTmAcc + tm_lane, rsqrtf((float)DH),
                     p.dq + ((size_t)bh * L + (live ? t : 0)) * DH, live);
  } else if (tid == 0) {
    record_device_error(BASED_ERR_TIMEOUT);
  }
  // before the tensor memory and the shared memory are released: every MMA
  // issued here is complete, and (after a timeout) the tile loads have landed
  if (tid == 0) {
    umma::mma_commit(bar_fin);
    umma::mbar_wait(bar_fin, 0);
    if (!ld_ok) umma::mbar_wait(bar_ld, 0);
  }
  umma::tc_fence_before();
  __syncthreads();
  if (warp == 0) umma::tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// key side: dk and dv from the stored statistics
// ---------------------------------------------------------------------------
template <int DH>
__global__ void __launch_bounds__(kWgThreads, 1)
    window_bwd_tc_kv_kernel(const __grid_constant__ CUtensorMap kmap,
                            const __grid_constant__ CUtensorMap vmap,
                            const __grid_constant__ CUtensorMap qmap,
                            const __grid_constant__ CUtensorMap dymap, const WgParams p) {
  using Lay = WgLayout<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bar_ld = reinterpret_cast<uint64_t*>(sm + Lay::kBar);
  uint64_t* bar_s = bar_ld + 1;
  uint64_t* bar_o = bar_ld + 2;
  uint64_t* bar_fin = bar_ld + 3;  // every MMA of this CTA complete (commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_ld + 4);
  float* st_m = reinterpret_cast<float*>(sm + Lay::kStats);
  float* st_l = st_m + kWgN;
  float* st_d = st_l + kWgN;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // a dependent launch: the previous kernel has finished before any global access
  umma::grid_dep_wait();
  umma::grid_dep_launch();
  const int tile = blockIdx.x % p.n_tiles;
  const int bh = blockIdx.x / p.n_tiles;
  const int s0 = tile * kWgT;
  const int L = p.L, W = p.W;

  if (tid == 0) {
    umma::mbar_init(bar_ld, 1);
    umma::mbar_init(bar_s, 1);
    umma::mbar_init(bar_o, 1);
    umma::mbar_init(bar_fin, 1);
    umma::fence_mbar_init();
    umma::mbar_arrive_expect_tx(bar_ld, Lay::kTx);
#pragma unroll
    for (int b = 0; b < DH / 64; ++b) {
      umma::tma_load_3d(sm + Lay::kA0 + b * kWgT * 128, &kmap, bar_ld, b * 64, s0, bh);
      umma::tma_load_3d(sm + Lay::kA1 + b * kWgT * 128, &vmap, bar_ld, b * 64, s0, bh);
      umma::tma_load_3d(sm + Lay::kB0 + b * kWgN * 128, &qmap, bar_ld, b * 64, s0, bh);
      umma::tma_load_3d(sm + Lay::kB1 + b * kWgN * 128, &dymap, bar_ld, b * 64, s0, bh);
    }
  }
  // the statistics of the staged queries (queries past L get l = 1, delta = 0;
  // their columns are masked anyway)
  {
    const size_t plane = (size_t)p.BH * L;
    for (int c = tid; c < kWgN; c += kWgThreads) {
      const int tq = s0 + c;
      const bool in = tq < L;
      const size_t at = (size_t)bh * L + (in ? tq : 0);
      st_m[c] = in ? p.ws[at] : 0.0f;
      st_l[c] = in ? 1.0f / p.ws[plane + at] : 1.0f;  // 1 / row sum
      st_d[c] = in ? p.ws[2 * plane + at] : 0.0f;
    }
  }
  __syncthreads();
  const bool ld_ok = umma::mbar_wait(bar_ld, 0);
  bool ok = ld_ok;
  if (warp == 0) {
    umma::tmem_alloc(tmem_slot, 512);
    umma::tmem_relinquish();
  }
  umma::tc_fence_before();
  ok = __syncthreads_and(ok);
  umma::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_lane = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t sK = umma::smem_u32(sm + Lay::kA0), sV = umma::smem_u32(sm + Lay::kA1),
                 sQ = umma::smem_u32(sm + Lay::kB0), sdY = umma::smem_u32(sm + Lay::kB1);
  const int r = tid, s = s0 + r;
  const bool live = s < L;

  if (ok && tid == 0) {
    const uint32_t id = umma::idesc_bf16(kWgT, kWgN, false, false);
#pragma unroll
    for (int k0 = 0; k0 < DH; k0 += 16) {
      umma::mma_bf16(tmem + Lay::kTmS, umma::desc_kmajor_sw128(sK, k0, kWgT),
                     umma::desc_kmajor_sw128(sQ, k0, kWgN), id, k0 > 0);
      umma::mma_bf16(tmem + Lay::kTmP, umma::desc_kmajor_sw128(sV, k0, kWgT),
                     umma::desc_kmajor_sw128(sdY, k0, kWgN), id, k0 > 0);
    }
    umma::mma_commit(bar_s);
  }
  if (ok) ok = umma::mbar_wait(bar_s, 0);
  umma::tc_fence_after();
  if (__syncthreads_and(ok)) {
    // staged column c holds query t = s0 + c; key s is seen by t in
    // [s, s + W - 1] with t < L, i.e. local columns [lane, lane + W - 1] of its 96
    const int cb = warp * 32;
    const int lo = lane;
    const int hi = min(lane + W - 1, L - 1 - s0 - cb);
    const float scale = rsqrtf((float)DH) * 1.4426950408889634f;
    float pv[96];
    umma::tmem_ld64_32(tmem + Lay::kTmS + tm_lane + cb, tmem + Lay::kTmS + tm_lane + cb + 64, pv);
    // pairs outside the window become -inf once (exp2(-inf) = 0, and every
    // staged statistic is finite); with W = 64 and all 192 staged queries inside
    // the sequence, hi = lane + 63 and only the two ragged ends are tested
    if (W == 64 && s0 + kWgN <= L) {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < lane) pv[i] = -INFINITY;
#pragma unroll
      for (int i = 64; i < 96; ++i)
        if (i > lane + 63) pv[i] = -INFINITY;
    } else {
#pragma unroll
      for (int i = 0; i < 96; ++i)
        if (i < lo || i > hi) pv[i] = -INFINITY;
    }
#pragma unroll
    for (int i = 0; i < 96; ++i)
      pv[i] = ex2_approx(fmaf(pv[i], scale, -st_m[cb + i])) * st_l[cb + i];
    float dp[96];
    umma::tmem_ld64_32(tmem + Lay::kTmP + tm_lane + cb, tmem + Lay::kTmP + tm_lane + cb + 64, dp);
    uint32_t pk[48], dk[48];
#pragma unroll
    for (int j = 0; j < 48; ++j) {
      pk[j] = wg_pack(pv[2 * j], pv[2 * j + 1]);
      dk[j] = wg_pack(pv[2 * j] * (dp[2 * j] - st_d[cb + 2 * j]),
                      pv[2 * j + 1] * (dp[2 * j + 1] - st_d[cb + 2 * j + 1]));
    }
    // P^T over S^T's first 96 columns, dS^T over the next 96 (this lane's S^T
    // and dP^T values are in registers by now)
    wg_store_band(tmem + Lay::kTmS + tm_lane, warp, pk);
    wg_store_band(tmem + Lay::kTmS + 96 + tm_lane, warp, dk);
    umma::tmem_wait_st();
  } else {
    ok = false;
  }
  umma::tc_fence_before();
  ok = __syncthreads_and(ok);
  umma::tc_fence_after();
  if (ok && tid == 0) {
    // dV = P^T dY into the accumulator at 384; dK = dS^T Q over dP^T (at 192)
    const uint32_t id = umma::idesc_bf16(kWgT, DH, false, true);
#pragma unroll
    for (int k0 = 0; k0 < kWgN; k0 += 16) {
      umma::mma_ts(tmem + Lay::kTmAcc, tmem + Lay::kTmS + k0 / 2,
                   umma::desc_mnmajor_sw128(sdY, k0, kWgN), id, k0 > 0);
      umma::mma_ts(tmem + Lay::kTmP, tmem + Lay::kTmS + 96 + k0 / 2,
                   umma::desc_mnmajor_sw128(sQ, k0, kWgN), id, k0 > 0);
    }
    umma::mma_commit(bar_o);
  }
  if (ok) ok = umma::mbar_wait(bar_o, 0);
  umma::tc_fence_after();
  if (__syncthreads_and(ok)) {
    const size_t row = ((size_t)bh * L + (live ? s : 0)) * DH;
    wg_store_acc<DH>(tmem + Lay::kTmAcc + tm_lane, 1.0f, p.dv + row, live);
    wg_store_acc<DH>(tmem + Lay::kTmP + tm_lane, rsqrtf((float)DH), p.dk + row, live);
  } else if (tid == 0) {
    record_device_error(BASED_ERR_TIMEOUT);
  }
  // before the tensor memory and the shared memory are released: every MMA
  // issued here is complete, and (after a timeout) the tile loads have landed
  if (tid == 0) {
    umma::mma_commit(bar_fin);
    umma::mbar_wait(bar_fin, 0);
    if (!ld_ok) umma::mbar_wait(bar_ld, 0);
  }
  umma::tc_fence_before();
  __syncthreads();
  if (warp == 0) umma::tmem_dealloc(tmem, 512);
}

}  // namespace based
