// decode.cuh -- one-token decode step: linear-attention state update + read-out,
// and the sliding-window ring-cache attention, in one launch.
//
// Linear part ("Базированная модель, часть 2", paragraph on the KV state for the
// numerator and the K state for the denominator): per (b, h)
//     S += phi(k) v^T ;  z += phi(k) ;  y = phi(q)^T S / (phi(q) . z + eps).
// The 273 x d_v fp32 state is read once and written once per step, so the step
// is bound by HBM bandwidth: every thread streams whole float4 columns of S with
// 128-bit coalesced loads/stores (a warp covers two contiguous 256-byte rows for
// d_v = 64), issues all its loads before any arithmetic, and the read-out is
// reduced across row slots through shared memory and across warps by shuffles.
//
// Window part (Based README, introduction, item 1: short sliding-window softmax
// attention): the new k/v go to ring slot pos mod W, then softmax over the slots
// holding positions max(0, pos-W+1)..pos.
#pragma once

#include "common.cuh"

namespace based {

struct DecodeParams {
  const void *q, *k, *v;
  float *S, *z;
  void* out;
  const void *wq, *wk, *wv;
  void *k_ring, *v_ring, *wout;
  long long pos;
  int n_lin;  // B * H   (CTAs of the linear part)
  int n_win;  // B * H_w (CTAs of the window part)
  int dh, W;
  float eps;
};

template <int DV>
struct DecodeLinearLayout {
  static constexpr int kThreads = 4 * DV;
  static constexpr int kColGroups = DV / 4;                 // float4 groups per row
  static constexpr int kRowSlots = kThreads / kColGroups;   // 16
  static constexpr int kRowsPerThread = (kF + kRowSlots - 1) / kRowSlots;  // 18
  static constexpr int kFPad = 276;
  // fq, fk, v, per-row-slot partial sums, per-warp partial denominators, x_q, x_k
  static constexpr int kSmemFloats = 2 * kFPad + DV + kRowSlots * DV + 32 + 32;
};

template <typename T, int DV>
__device__ __forceinline__ void decode_linear_block(const DecodeParams& p, int bh, float* smem) {
  using Lay = DecodeLinearLayout<DV>;
  constexpr int NT = Lay::kThreads, CG = Lay::kColGroups, RS = Lay::kRowSlots,
                NR = Lay::kRowsPerThread;
  float* fq = smem;
  float* fk = fq + Lay::kFPad;
  float* vs = fk + Lay::kFPad;
  float* red = vs + DV;
  float* dred = red + RS * DV;
  float* xq = dred + 32;
  float* xk = xq + 16;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cg = tid % CG, rs = tid / CG;

  // Issue the whole state slice of this thread first: the loads stay in flight
  // while the feature vectors are built.
  float4* S4 = reinterpret_cast<float4*>(p.S + (size_t)bh * kF * DV);
  float4 sv[NR];
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    const int r = rs + i * RS;
    if (r < kF) sv[i] = S4[r * CG + cg];
  }
  float* zb = p.z + (size_t)bh * kF;
  float zv[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int f = tid + i * NT;
    zv[i] = f < kF ? zb[f] : 0.0f;
  }

  const T* q = static_cast<const T*>(p.q) + (size_t)bh * kD;
  const T* k = static_cast<const T*>(p.k) + (size_t)bh * kD;
  const T* v = static_cast<const T*>(p.v) + (size_t)bh * DV;
  if (tid < kD) xq[tid] = to_f32(q[tid]);
  else if (tid < 2 * kD) xk[tid - kD] = to_f32(k[tid - kD]);
  if (tid < DV) vs[tid] = to_f32(v[tid]);
  __syncthreads();
  for (int f = tid; f < kF; f += NT) {
    fq[f] = phi_feature(xq, f);
    fk[f] = phi_feature(xk, f);
  }
  __syncthreads();

  const float4 vv = reinterpret_cast<const float4*>(vs)[cg];
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    const int r = rs + i * RS;
    if (r < kF) {
      const float a = fk[r], b = fq[r];
      float4 s = sv[i];
      s.x = fmaf(a, vv.x, s.x);
      s.y = fmaf(a, vv.y, s.y);
      s.z = fmaf(a, vv.z, s.z);
      s.w = fmaf(a, vv.w, s.w);
      S4[r * CG + cg] = s;
      acc.x = fmaf(b, s.x, acc.x);
      acc.y = fmaf(b, s.y, acc.y);
      acc.z = fmaf(b, s.z, acc.z);
      acc.w = fmaf(b, s.w, acc.w);
    }
  }
  float dpart = 0.0f;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int f = tid + i * NT;
    if (f < kF) {
      const float zn = zv[i] + fk[f];
      zb[f] = zn;
      dpart = fmaf(fq[f], zn, dpart);
    }
  }
  dpart = warp_sum(dpart);
  if (lane == 0) dred[warp] = dpart;
  reinterpret_cast<float4*>(red)[rs * CG + cg] = acc;
  __syncthreads();
  if (tid < DV) {
    float num = 0.0f;
#pragma unroll
    for (int r = 0; r < RS; ++r) num += red[r * DV + tid];
    float den = 0.0f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) den += dred[w];
    static_cast<T*>(p.out)[(size_t)bh * DV + tid] = from_f32<T>(num / (den + p.eps));
  }
}

__host__ __device__ constexpr int decode_window_smem_floats(int dh, int W) {
  return 128 + 2 * W * dh + 64 + 32;
}

template <typename T>
__device__ __forceinline__ void decode_window_block(const DecodeParams& p, int bhw, float* smem) {
  const int dh = p.dh, W = p.W, NT = blockDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = NT >> 5;
  float* qs = smem;              // [dh]
  float* kr = qs + 128;          // [W][dh]
  float* vr = kr + W * dh;       // [W][dh]
  float* pr = vr + W * dh;       // [W] scores, then weights
  float* red = pr + 64;          // [2] max, sum
  T* kring = static_cast<T*>(p.k_ring) + (size_t)bhw * W * dh;
  T* vring = static_cast<T*>(p.v_ring) + (size_t)bhw * W * dh;
  const T* q = static_cast<const T*>(p.wq) + (size_t)bhw * dh;
  const T* kn = static_cast<const T*>(p.wk) + (size_t)bhw * dh;
  const T* vn = static_cast<const T*>(p.wv) + (size_t)bhw * dh;
  const long long pos = p.pos;
  const int slot = (int)(pos % W);
  const int nvalid = pos + 1 < W ? (int)(pos + 1) : W;  // valid slots are 0..nvalid-1

  for (int i = tid; i < nvalid * dh; i += NT) {
    kr[i] = to_f32(kring[i]);
    vr[i] = to_f32(vring[i]);
  }
  if (tid < dh) qs[tid] = to_f32(q[tid]);
  __syncthreads();
  if (tid < dh) {
    const T kt = kn[tid], vt = vn[tid];
    kring[(size_t)slot * dh + tid] = kt;
    vring[(size_t)slot * dh + tid] = vt;
    kr[slot * dh + tid] = to_f32(kt);
    vr[slot * dh + tid] = to_f32(vt);
  }
  __syncthreads();
  const float scale = rsqrtf((float)dh);
  for (int s = warp; s < nvalid; s += nwarps) {
    float a = 0.0f;
    for (int j = lane; j < dh; j += 32) a = fmaf(qs[j], kr[s * dh + j], a);
    a = warp_sum(a);
    if (lane == 0) pr[s] = a * scale;
  }
  __syncthreads();
  if (warp == 0) {
    const float a0 = lane < nvalid ? pr[lane] : -INFINITY;
    const float a1 = lane + 32 < nvalid ? pr[lane + 32] : -INFINITY;
    const float m = warp_max(fmaxf(a0, a1));
    const float e0 = lane < nvalid ? expf(a0 - m) : 0.0f;
    const float e1 = lane + 32 < nvalid ? expf(a1 - m) : 0.0f;
    if (lane < nvalid) pr[lane] = e0;
    if (lane + 32 < nvalid) pr[lane + 32] = e1;
    const float sum = warp_sum(e0 + e1);
    if (lane == 0) red[0] = sum;
  }
  __syncthreads();
  if (tid < dh) {
    float acc = 0.0f;
    for (int s = 0; s < nvalid; ++s) acc = fmaf(pr[s], vr[s * dh + tid], acc);
    static_cast<T*>(p.wout)[(size_t)bhw * dh + tid] = from_f32<T>(acc / red[0]);
  }
}

template <typename T, int DV>
__global__ void __launch_bounds__(4 * DV) decode_step_kernel(const DecodeParams p) {
  extern __shared__ __align__(16) float smem[];
  const int b = blockIdx.x;
  if (b < p.n_lin) decode_linear_block<T, DV>(p, b, smem);
  else decode_window_block<T>(p, b - p.n_lin, smem);
}

}  // namespace based
