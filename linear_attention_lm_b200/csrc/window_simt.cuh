// window_simt.cuh -- sliding-window causal softmax attention on CUDA cores (fp32).
//
// Based README, introduction, item 1: exact softmax attention over a short
// sliding window (size 64) for local token interactions.  For query t the keys
// are s in [max(0, t-W+1), t], scores q_t.k_s / sqrt(d_head).
//
// This is the fp32 path (fp32 inputs, fp32 arithmetic): one CTA of 64 threads
// per block of 64 queries; the 127 key/value rows the block can touch
// ([t0-63, t0+63]) and its 64 query rows are staged once in shared memory with
// a row pitch of d_head+4 floats, so the float4 reads of 8 consecutive threads
// (consecutive rows) fall in distinct banks.
#pragma once

#include "common.cuh"

namespace based {

constexpr int kWinQ = 64;          // queries per CTA
constexpr int kWinRows = 2 * kWinQ - 1;  // key/value rows staged per CTA

__host__ __device__ constexpr size_t window_simt_smem_bytes(int dh) {
  return sizeof(float) * (size_t)(2 * kWinRows + kWinQ) * (size_t)(dh + 4);
}

template <typename T>
__global__ void __launch_bounds__(kWinQ) window_simt_kernel(const T* __restrict__ q,
                                                            const T* __restrict__ k,
                                                            const T* __restrict__ v,
                                                            T* __restrict__ out, int L, int dh,
                                                            int W) {
  extern __shared__ __align__(16) float smem[];
  const int ld = dh + 4;
  float* ks = smem;
  float* vs = ks + kWinRows * ld;
  float* qs = vs + kWinRows * ld;
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * kWinQ;
  const size_t base = (size_t)blockIdx.y * L * dh;
  q += base; k += base; v += base; out += base;

  for (int idx = tid; idx < kWinRows * dh; idx += kWinQ) {
    const int r = idx / dh, c = idx - r * dh;
    const int g = t0 - (kWinQ - 1) + r;
    const bool ok = g >= 0 && g < L;
    ks[r * ld + c] = ok ? to_f32(k[(size_t)g * dh + c]) : 0.0f;
    vs[r * ld + c] = ok ? to_f32(v[(size_t)g * dh + c]) : 0.0f;
  }
  for (int idx = tid; idx < kWinQ * dh; idx += kWinQ) {
    const int r = idx / dh, c = idx - r * dh;
    const int g = t0 + r;
    qs[r * ld + c] = g < L ? to_f32(q[(size_t)g * dh + c]) : 0.0f;
  }
  __syncthreads();
  const int t = t0 + tid;
  if (t >= L) return;
  const int lo = max(0, t - W + 1);
  const float scale = rsqrtf((float)dh);
  const float4* q4 = reinterpret_cast<const float4*>(qs + tid * ld);
  float sc[kWinQ];
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < kWinQ; ++j) {
    const int s = t - (kWinQ - 1) + j;  // key index; its staged row is tid + j
    float a = -INFINITY;
    if (s >= lo) {
      const float4* k4 = reinterpret_cast<const float4*>(ks + (tid + j) * ld);
      // four independent chains: the loop is latency-bound on one
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int c = 0; c < dh / 4; ++c) {
        const float4 x = q4[c], y = k4[c];
        acc.x = fmaf(x.x, y.x, acc.x);
        acc.y = fmaf(x.y, y.y, acc.y);
        acc.z = fmaf(x.z, y.z, acc.z);
        acc.w = fmaf(x.w, y.w, acc.w);
      }
      a = ((acc.x + acc.y) + (acc.z + acc.w)) * scale;
    }
    sc[j] = a;
    m = fmaxf(m, a);
  }
  float sum = 0.0f;
#pragma unroll
  for (int j = 0; j < kWinQ; ++j) {
    const float e = (t - (kWinQ - 1) + j >= lo) ? expf(sc[j] - m) : 0.0f;
    sc[j] = e;
    sum += e;
  }
  const float inv = 1.0f / sum;
  for (int c = 0; c < dh / 4; ++c) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < kWinQ; ++j) {
      const float4 y = reinterpret_cast<const float4*>(vs + (tid + j) * ld)[c];
      acc.x = fmaf(sc[j], y.x, acc.x);
      acc.y = fmaf(sc[j], y.y, acc.y);
      acc.z = fmaf(sc[j], y.z, acc.z);
      acc.w = fmaf(sc[j], y.w, acc.w);
    }
    T* o = out + (size_t)t * dh + 4 * c;
    o[0] = from_f32<T>(acc.x * inv);
    o[1] = from_f32<T>(acc.y * inv);
    o[2] = from_f32<T>(acc.z * inv);
    o[3] = from_f32<T>(acc.w * inv);
  }
}

}  // namespace based
