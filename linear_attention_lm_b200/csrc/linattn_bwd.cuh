// linattn_bwd.cuh -- gradient of the causal Taylor linear attention (CUDA cores, fp32).
//
// The "based/train" README lists the training views of this attention; training
// needs the gradient of the map they share ("Базированная модель, часть 2",
// section "Что за линейное внимание?"), written here from the quadratic form:
//   w_ts = phi(q_t).phi(k_s) = 1 + u + u^2/2,  u = q_t.k_s / sqrt(d),  s <= t
//   N_t = sum_s w_ts v_s,   D_t = sum_s w_ts + eps,   y_t = N_t / D_t
// Given dy: dN_t = dy_t / D_t, dD_t = -(dy_t . y_t) / D_t,
//   dw_ts = dN_t . v_s + dD_t,   du_ts = dw_ts (1 + u_ts),
//   dq_t = sum_s du_ts k_s / sqrt(d),  dk_s = sum_t du_ts q_t / sqrt(d),
//   dv_s = sum_t w_ts dN_t.
// Two kernels over 64 x 64 tiles of the (t, s) triangle:
//   linattn_bwd_q:  one CTA per (b, h, query tile): first D_t and N_t (hence
//                   dN_t, dD_t, written to a workspace), then dq_t;
//   linattn_bwd_kv: one CTA per (b, h, key tile): dk_s and dv_s from the
//                   workspace.
// Thread (ty, tx) of 256 owns a 4 x 4 block of every 64 x 64 tile.
#pragma once

#include "common.cuh"

namespace based {

constexpr int kBwT = 64;        // tile edge (queries and keys)
constexpr int kBwThreads = 256;

template <int DV>
struct BwLayout {
  // shared memory, in floats
  static constexpr int kP = kBwT + 1;           // padded row pitch of 64-wide tiles
  static constexpr int kQ = 0;                  // [64][16] q or the other side's q
  static constexpr int kK = kQ + kBwT * kD;     // [64][16]
  static constexpr int kV = kK + kBwT * kD;     // [64][DV+1] v (bwd_q) or dN (bwd_kv)
  static constexpr int kVP = DV + 1;
  static constexpr int kY = kV + kBwT * kVP;    // [64][DV+1] dy -> dN (bwd_q) or v (bwd_kv)
  static constexpr int kW = kY + kBwT * kVP;    // [64][65] w tile
  static constexpr int kG = kW + kBwT * kP;     // [64][65] du tile
  static constexpr int kR = kG + kBwT * kP;     // [64] row sums D / dD
  static constexpr int kFloats = kR + 2 * kBwT;
  static constexpr size_t kSmem = kFloats * sizeof(float);
};

template <typename T>
__device__ __forceinline__ void bw_load_rows(float* dst, int pitch, const T* src, int rows,
                                             int cols, int valid_rows) {
  for (int i = threadIdx.x; i < rows * cols; i += kBwThreads) {
    const int r = i / cols, c = i - r * cols;
    dst[r * pitch + c] = r < valid_rows ? to_f32(src[(size_t)r * cols + c]) : 0.0f;
  }
}

// w and du of the tile (rows = queries tq.., cols = keys ks..) for one thread's
// 4 x 4 block; qs [64][16], ks [64][16], dN [64][DV+1] (query rows), vs [64][DV+1]
// (key rows), dD [64]
template <int DV, bool kNeedDu>
__device__ __forceinline__ void bw_tile_w(const float* qs, const float* ks, int t0, int s0, int L,
                                          float* w, float* du, const float* dN, const float* vs,
                                          const float* dD, bool transposed) {
  using Lay = BwLayout<DV>;
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  const float c = 0.25f;  // 1 / sqrt(16)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int tr = ty * 4 + i;  // query row within the tile
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int sc = tx * 4 + j;  // key column within the tile
      float u = 0.0f;
#pragma unroll
      for (int e = 0; e < kD; ++e) u = fmaf(qs[tr * kD + e], ks[sc * kD + e], u);
      u *= c;
      const int t = t0 + tr, s = s0 + sc;
      const bool live = s <= t && t < L && s < L;
      const float wv = live ? 1.0f + u + 0.5f * u * u : 0.0f;
      float g = 0.0f;
      if (kNeedDu && live) {
        float dw = dD[tr];
#pragma unroll 8
        for (int e = 0; e < DV; ++e) dw = fmaf(dN[tr * Lay::kVP + e], vs[sc * Lay::kVP + e], dw);
        g = dw * (1.0f + u);
      }
      const int idx = transposed ? sc * Lay::kP + tr : tr * Lay::kP + sc;
      w[idx] = wv;
      if (kNeedDu) du[idx] = g;
    }
  }
}

template <typename T, int DV>
__global__ void __launch_bounds__(kBwThreads)
    linattn_bwd_q_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                         const T* __restrict__ dy, float* __restrict__ dq, float* __restrict__ ws_dN,
                         float* __restrict__ ws_dD, int L, float eps) {
  using Lay = BwLayout<DV>;
  extern __shared__ float bsm[];
  float *qs = bsm + Lay::kQ, *ks = bsm + Lay::kK, *vs = bsm + Lay::kV, *ys = bsm + Lay::kY;
  float *w = bsm + Lay::kW, *du = bsm + Lay::kG, *rs = bsm + Lay::kR;
  const int n_qt = (L + kBwT - 1) / kBwT;
  const int bh = blockIdx.x / n_qt, qt = blockIdx.x - bh * n_qt;
  const int t0 = qt * kBwT, nq = min(kBwT, L - t0);
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  constexpr int CPT = DV / 16;  // value columns per thread
  const size_t qoff = (size_t)bh * L;

  bw_load_rows(qs, kD, q + (qoff + t0) * kD, kBwT, kD, nq);
  bw_load_rows(ys, Lay::kVP, dy + (qoff + t0) * DV, kBwT, DV, nq);
  if (tid < kBwT) rs[tid] = 0.0f;
  // ---- pass 1: D_t and N_t over the key tiles s <= t ----
  float nacc[4][CPT];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < CPT; ++j) nacc[i][j] = 0.0f;
  for (int kt = 0; kt <= qt; ++kt) {
    const int s0 = kt * kBwT, ns = min(kBwT, L - s0);
    __syncthreads();
    bw_load_rows(ks, kD, k + (qoff + s0) * kD, kBwT, kD, ns);
    bw_load_rows(vs, Lay::kVP, v + (qoff + s0) * DV, kBwT, DV, ns);
    __syncthreads();
    bw_tile_w<DV, false>(qs, ks, t0, s0, L, w, nullptr, nullptr, nullptr, nullptr, false);
    __syncthreads();
    if (tid < kBwT) {
      float sum = 0.0f;
      for (int s = 0; s < kBwT; ++s) sum += w[tid * Lay::kP + s];
      rs[tid] += sum;
    }
    for (int s = 0; s < kBwT; ++s) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float wv = w[(ty * 4 + i) * Lay::kP + s];
#pragma unroll
        for (int j = 0; j < CPT; ++j) nacc[i][j] = fmaf(wv, vs[s * Lay::kVP + tx + 16 * j], nacc[i][j]);
      }
    }
  }
  __syncthreads();
  // ---- dN_t = dy_t / D_t, dD_t = -(dy_t . y_t) / D_t ----
  float* dDs = rs + kBwT;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int tr = ty * 4 + i;
    const float den = rs[tr] + eps;
    float part = 0.0f;
#pragma unroll
    for (int j = 0; j < CPT; ++j) part = fmaf(ys[tr * Lay::kVP + tx + 16 * j], nacc[i][j] / den, part);
    // the 16 threads of a row are 16 consecutive lanes
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (tx == 0) dDs[tr] = -part / den;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int tr = ty * 4 + i;
    const float inv = 1.0f / (rs[tr] + eps);
#pragma unroll
    for (int j = 0; j < CPT; ++j) ys[tr * Lay::kVP + tx + 16 * j] *= inv;  // dy -> dN
  }
  __syncthreads();
  for (int i = tid; i < nq * DV; i += kBwThreads) {
    const int r = i / DV, cidx = i - r * DV;
    ws_dN[(qoff + t0 + r) * DV + cidx] = ys[r * Lay::kVP + cidx];
  }
  if (tid < nq) ws_dD[qoff + t0 + tid] = dDs[tid];
  // ---- pass 2: dq_t = sum_s du_ts k_s / sqrt(d) ----
  const int qr = tid / 4, qd = (tid % 4) * 4;  // dq row and first of 4 dims
  float dacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int kt = 0; kt <= qt; ++kt) {
    const int s0 = kt * kBwT, ns = min(kBwT, L - s0);
    __syncthreads();
    bw_load_rows(ks, kD, k + (qoff + s0) * kD, kBwT, kD, ns);
    bw_load_rows(vs, Lay::kVP, v + (qoff + s0) * DV, kBwT, DV, ns);
    __syncthreads();
    bw_tile_w<DV, true>(qs, ks, t0, s0, L, w, du, ys, vs, dDs, false);
    __syncthreads();
    for (int s = 0; s < kBwT; ++s) {
      const float g = du[qr * Lay::kP + s];
#pragma unroll
      for (int e = 0; e < 4; ++e) dacc[e] = fmaf(g, ks[s * kD + qd + e], dacc[e]);
    }
  }
  if (qr < nq) {
#pragma unroll
    for (int e = 0; e < 4; ++e) dq[(qoff + t0 + qr) * kD + qd + e] = dacc[e] * 0.25f;
  }
}

template <typename T, int DV>
__global__ void __launch_bounds__(kBwThreads)
    linattn_bwd_kv_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                          const float* __restrict__ ws_dN, const float* __restrict__ ws_dD,
                          float* __restrict__ dk, float* __restrict__ dv, int L) {
  using Lay = BwLayout<DV>;
  extern __shared__ float bsm[];
  float *qs = bsm + Lay::kQ, *ks = bsm + Lay::kK, *dNs = bsm + Lay::kV, *vs = bsm + Lay::kY;
  float *wT = bsm + Lay::kW, *duT = bsm + Lay::kG, *dDs = bsm + Lay::kR;
  const int n_t = (L + kBwT - 1) / kBwT;
  const int bh = blockIdx.x / n_t, kt = blockIdx.x - bh * n_t;
  const int s0 = kt * kBwT, ns = min(kBwT, L - s0);
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  constexpr int CPT = DV / 16;
  const size_t qoff = (size_t)bh * L;

  bw_load_rows(ks, kD, k + (qoff + s0) * kD, kBwT, kD, ns);
  bw_load_rows(vs, Lay::kVP, v + (qoff + s0) * DV, kBwT, DV, ns);
  float vacc[4][CPT];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < CPT; ++j) vacc[i][j] = 0.0f;
  const int kr = tid / 4, kd = (tid % 4) * 4;  // dk row and first of 4 dims
  float kacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int qt = kt; qt < n_t; ++qt) {
    const int t0 = qt * kBwT, nq = min(kBwT, L - t0);
    __syncthreads();
    bw_load_rows(qs, kD, q + (qoff + t0) * kD, kBwT, kD, nq);
    for (int i = tid; i < kBwT * DV; i += kBwThreads) {
      const int r = i / DV, cidx = i - r * DV;
      dNs[r * Lay::kVP + cidx] = r < nq ? ws_dN[(qoff + t0 + r) * DV + cidx] : 0.0f;
    }
    if (tid < kBwT) dDs[tid] = tid < nq ? ws_dD[qoff + t0 + tid] : 0.0f;
    __syncthreads();
    // w and du with key rows: wT[s][t], duT[s][t]
    bw_tile_w<DV, true>(qs, ks, t0, s0, L, wT, duT, dNs, vs, dDs, true);
    __syncthreads();
    // dv_s += sum_t w_ts dN_t ; rows = keys (ty*4+i), cols = value columns
    for (int t = 0; t < kBwT; ++t) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float wv = wT[(ty * 4 + i) * Lay::kP + t];
#pragma unroll
        for (int j = 0; j < CPT; ++j) vacc[i][j] = fmaf(wv, dNs[t * Lay::kVP + tx + 16 * j], vacc[i][j]);
      }
    }
    // dk_s += sum_t du_ts q_t
    for (int t = 0; t < kBwT; ++t) {
      const float g = duT[kr * Lay::kP + t];
#pragma unroll
      for (int e = 0; e < 4; ++e) kacc[e] = fmaf(g, qs[t * kD + kd + e], kacc[e]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i;
    if (r < ns) {
#pragma unroll
      for (int j = 0; j < CPT; ++j) dv[(qoff + s0 + r) * DV + tx + 16 * j] = vacc[i][j];
    }
  }
  if (kr < ns) {
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[(qoff + s0 + kr) * kD + kd + e] = kacc[e] * 0.25f;
  }
}

}  // namespace based
