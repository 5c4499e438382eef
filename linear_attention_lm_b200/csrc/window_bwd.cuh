// window_bwd.cuh -- gradient of the sliding-window causal softmax attention
// (CUDA cores, fp32, d_h = 64).
//
// The forward (Based README, introduction, item 1): for query t the keys are
// s in [max(0, t-W+1), t], s_ts = q_t.k_s / sqrt(d_h), P_ts = softmax_s(s_ts),
// y_t = sum_s P_ts v_s.  Its gradient, given dy:
//   dP_ts = dy_t . v_s,   delta_t = sum_s P_ts dP_ts (= dy_t . y_t),
//   dS_ts = P_ts (dP_ts - delta_t),
//   dq_t = sum_s dS_ts k_s / sqrt(d_h),  dk_s = sum_t dS_ts q_t / sqrt(d_h),
//   dv_s = sum_t P_ts dy_t.
// Two kernels over 64-row tiles:
//   window_bwd_q:  one CTA per (b, h, query tile [t0, t0+64)); the keys it can
//                  see lie in [t0-63, t0+63], staged as rows [t0-64, t0+64).  It
//                  writes dq and each query's row max, row sum and delta to a
//                  workspace;
//   window_bwd_kv: one CTA per (b, h, key tile [s0, s0+64)); the queries that
//                  see it lie in [s0, s0+126], staged as rows [s0, s0+128).
// Thread (ty, tx) of 256 owns 4 rows x 8 columns of every 64 x 128 tile.
#pragma once

#include "common.cuh"

namespace based {

constexpr int kWbT = 64;     // tile rows
constexpr int kWbS = 128;    // staged rows of the other side
constexpr int kWbDh = 64;
constexpr int kWbThreads = 256;

struct WbLayout {
  static constexpr int kHP = kWbDh + 1;             // padded row pitch of d_h-wide rows
  static constexpr int kTP = kWbS + 1;              // padded row pitch of 128-wide tiles
  static constexpr int kA = 0;                      // [64][kHP]   own rows (q or k)
  static constexpr int kA2 = kA + kWbT * kHP;       // [64][kHP]   own rows (dy or v)
  static constexpr int kB = kA2 + kWbT * kHP;       // [128][kHP]  other rows (k or q)
  static constexpr int kB2 = kB + kWbS * kHP;       // [128][kHP]  other rows (v or dy)
  static constexpr int kP = kB2 + kWbS * kHP;       // [64][kTP]   P, then dS
  static constexpr int kR = kP + kWbT * kTP;        // row stats: [3][128]
  static constexpr int kFloats = kR + 3 * kWbS;
  static constexpr size_t kSmem = kFloats * sizeof(float);
};

template <typename T>
__device__ __forceinline__ void wb_load(float* dst, const T* src, int row0, int rows, int L) {
  // rows [row0, row0 + rows) of a [L, 64] matrix; rows outside [0, L) read as zero
  for (int i = threadIdx.x; i < rows * kWbDh; i += kWbThreads) {
    const int r = i / kWbDh, c = i - r * kWbDh;
    const int g = row0 + r;
    dst[r * WbLayout::kHP + c] = (g >= 0 && g < L) ? to_f32(src[(size_t)g * kWbDh + c]) : 0.0f;
  }
}

template <typename T>
__global__ void __launch_bounds__(kWbThreads)
    window_bwd_q_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                        const T* __restrict__ dy, float* __restrict__ dq,
                        float* __restrict__ ws, int L, int W) {
  using Lay = WbLayout;
  extern __shared__ float wsm[];
  float *qs = wsm + Lay::kA, *dys = wsm + Lay::kA2, *ks = wsm + Lay::kB, *vs = wsm + Lay::kB2;
  float* pt = wsm + Lay::kP;
  const int n_t = (L + kWbT - 1) / kWbT;
  const int bh = blockIdx.x / n_t, qt = blockIdx.x - bh * n_t;
  const int t0 = qt * kWbT, s_base = t0 - kWbT;  // staged key row c is key s_base + c
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const size_t off = (size_t)bh * L * kWbDh;
  const float c = 0.125f;  // 1 / sqrt(64)
  wb_load(qs, q + off, t0, kWbT, L);
  wb_load(dys, dy + off, t0, kWbT, L);
  wb_load(ks, k + off, s_base, kWbS, L);
  wb_load(vs, v + off, s_base, kWbS, L);
  __syncthreads();
  // scores of the thread's 4 x 8 block, band mask, row max over the 16 threads
  float sv[4][8];
  float mx[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i, t = t0 + r;
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int cc = tx * 8 + j, s = s_base + cc;
      float a = 0.0f;
#pragma unroll 16
      for (int e = 0; e < kWbDh; ++e) a = fmaf(qs[r * Lay::kHP + e], ks[cc * Lay::kHP + e], a);
      const bool live = s <= t && s > t - W && s >= 0;
      sv[i][j] = live ? a * c : -INFINITY;
      m = fmaxf(m, sv[i][j]);
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    mx[i] = m;
  }
  // P = exp(s - m) / l, and dP = dy . v with delta = sum P dP
  float lsum[4], dl[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float l = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      sv[i][j] = mx[i] == -INFINITY ? 0.0f : expf(sv[i][j] - mx[i]);
      l += sv[i][j];
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    lsum[i] = l;
  }
  float dp[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
    const float inv = lsum[i] > 0.0f ? 1.0f / lsum[i] : 0.0f;
    float part = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int cc = tx * 8 + j;
      sv[i][j] *= inv;  // P
      float a = 0.0f;
#pragma unroll 16
      for (int e = 0; e < kWbDh; ++e) a = fmaf(dys[r * Lay::kHP + e], vs[cc * Lay::kHP + e], a);
      dp[i][j] = a;
      part = fmaf(sv[i][j], a, part);
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    dl[i] = part;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
#pragma unroll
    for (int j = 0; j < 8; ++j) pt[r * Lay::kTP + tx * 8 + j] = sv[i][j] * (dp[i][j] - dl[i]);  // dS
    if (tx == 0 && t0 + r < L) {
      float* wsr = ws + ((size_t)bh * L + t0 + r) * 3;
      wsr[0] = mx[i];
      wsr[1] = lsum[i];
      wsr[2] = dl[i];
    }
  }
  __syncthreads();
  // dq_t = c sum_s dS_ts k_s : thread -> row tid / 4, 16 dims
  const int rr = tid / 4, d0 = (tid % 4) * 16;
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.0f;
  for (int cc = 0; cc < kWbS; ++cc) {
    const float g = pt[rr * Lay::kTP + cc];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = fmaf(g, ks[cc * Lay::kHP + d0 + e], acc[e]);
  }
  if (t0 + rr < L) {
#pragma unroll
    for (int e = 0; e < 16; ++e) dq[off + (size_t)(t0 + rr) * kWbDh + d0 + e] = acc[e] * c;
  }
}

template <typename T>
__global__ void __launch_bounds__(kWbThreads)
    window_bwd_kv_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                         const T* __restrict__ dy, const float* __restrict__ ws,
                         float* __restrict__ dk, float* __restrict__ dv, int L, int W) {
  using Lay = WbLayout;
  extern __shared__ float wsm[];
  float *ks = wsm + Lay::kA, *vs = wsm + Lay::kA2, *qs = wsm + Lay::kB, *dys = wsm + Lay::kB2;
  float *pt = wsm + Lay::kP, *stm = wsm + Lay::kR;  // stm: max [128], sum [128], delta [128]
  const int n_t = (L + kWbT - 1) / kWbT;
  const int bh = blockIdx.x / n_t, kt = blockIdx.x - bh * n_t;
  const int s0 = kt * kWbT;  // staged query row cc is query s0 + cc
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const size_t off = (size_t)bh * L * kWbDh;
  const float c = 0.125f;
  wb_load(ks, k + off, s0, kWbT, L);
  wb_load(vs, v + off, s0, kWbT, L);
  wb_load(qs, q + off, s0, kWbS, L);
  wb_load(dys, dy + off, s0, kWbS, L);
  for (int i = tid; i < kWbS; i += kWbThreads) {
    const int t = s0 + i;
    const bool in = t < L;
    stm[i] = in ? ws[((size_t)bh * L + t) * 3 + 0] : 0.0f;
    stm[kWbS + i] = in ? ws[((size_t)bh * L + t) * 3 + 1] : 1.0f;
    stm[2 * kWbS + i] = in ? ws[((size_t)bh * L + t) * 3 + 2] : 0.0f;
  }
  __syncthreads();
  // rows = keys (ty*4+i), columns = queries (tx*8+j): P and dS, transposed
  float pv[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i, s = s0 + r;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int cc = tx * 8 + j, t = s0 + cc;
      const bool live = s <= t && s > t - W && t < L && s < L;
      float a = 0.0f, b = 0.0f;
      if (live) {
#pragma unroll 16
        for (int e = 0; e < kWbDh; ++e) {
          a = fmaf(ks[r * Lay::kHP + e], qs[cc * Lay::kHP + e], a);
          b = fmaf(vs[r * Lay::kHP + e], dys[cc * Lay::kHP + e], b);
        }
      }
      const float p = live ? expf(a * c - stm[cc]) / stm[kWbS + cc] : 0.0f;
      pv[i][j] = p;
      pt[r * Lay::kTP + cc] = p * (b - stm[2 * kWbS + cc]);  // dS (transposed)
    }
  }
  __syncthreads();
  // dv_s = sum_t P_ts dy_t and dk_s = c sum_t dS_ts q_t : thread -> key row tid / 4, 16 dims
  const int rr = tid / 4, d0 = (tid % 4) * 16;
  float av[16], ak[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) av[e] = ak[e] = 0.0f;
  // P is needed as a tile too: reuse the register block by writing it after dS is consumed
  for (int cc = 0; cc < kWbS; ++cc) {
    const float g = pt[rr * Lay::kTP + cc];
#pragma unroll
    for (int e = 0; e < 16; ++e) ak[e] = fmaf(g, qs[cc * Lay::kHP + d0 + e], ak[e]);
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) pt[(ty * 4 + i) * Lay::kTP + tx * 8 + j] = pv[i][j];
  __syncthreads();
  for (int cc = 0; cc < kWbS; ++cc) {
    const float p = pt[rr * Lay::kTP + cc];
#pragma unroll
    for (int e = 0; e < 16; ++e) av[e] = fmaf(p, dys[cc * Lay::kHP + d0 + e], av[e]);
  }
  if (s0 + rr < L) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      dk[off + (size_t)(s0 + rr) * kWbDh + d0 + e] = ak[e] * c;
      dv[off + (size_t)(s0 + rr) * kWbDh + d0 + e] = av[e];
    }
  }
}

}  // namespace based
