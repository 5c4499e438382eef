// window_simt.cuh -- sliding-window causal softmax attention on CUDA cores (fp32).
//
// Based README, introduction, item 1: exact softmax attention over a short
// sliding window (size 64) for local token interactions.  For query t the keys
// are s in [max(0, t-W+1), t], scores q_t.k_s / sqrt(d_head).
//
// This is the fp32 path (fp32 inputs, fp32 arithmetic): one CTA of
// Q * SUB threads per block of Q queries, SUB threads per query (Q = 64, SUB = 4
// when the problem fills the GPU; Q = 16, SUB = 16 for small ones, where more
// CTAs matter more than the re-read of each block's 63-row halo).
// The Q + 63 key/value rows the block can touch ([t0-63, t0+Q-1]) and
// its query rows are staged once in shared memory by 16-byte cp.async copies
// (all of a thread's copies in flight at once; rows outside [0, L) zero-filled)
// with a row pitch of d_head+4 floats, so the float4 reads of 8 consecutive rows
// fall in distinct banks.  Thread `sub` of a query scores keys sub, sub+SUB,
// ... of its 64, the query's threads combine max and sum by shuffles, the
// weights go to shared memory, and each thread then forms 1/SUB of the output
// columns over all 64 keys.
#pragma once

#include "common.cuh"
#include "umma.cuh"

namespace based {

constexpr int kWinK = 64;          // largest window: keys scored per query
constexpr int kWinPP = kWinK + 1;  // pitch of the weight rows (odd: no bank conflicts)

template <int Q>
__host__ __device__ constexpr size_t window_simt_smem_bytes(int dh) {
  return sizeof(float) * ((size_t)(2 * (Q + kWinK - 1) + Q) * (size_t)(dh + 4) +
                          (size_t)Q * kWinPP);
}

template <typename T, int Q, int SUB>
__global__ void __launch_bounds__(Q * SUB) window_simt_kernel(const T* __restrict__ q,
                                                              const T* __restrict__ k,
                                                              const T* __restrict__ v,
                                                              T* __restrict__ out, int L, int dh,
                                                              int W) {
  constexpr int kWinQ = Q, kWinSub = SUB, kWinThreads = Q * SUB;
  constexpr int kWinRows = Q + kWinK - 1;  // key/value rows staged per CTA
  static_assert(kWinK % SUB == 0 && 32 % SUB == 0, "threads of a query in one warp");
  static_assert(sizeof(T) == sizeof(float), "the cp.async staging copies fp32 rows");
  extern __shared__ __align__(16) float smem[];
  const int ld = dh + 4;
  float* ks = smem;
  float* vs = ks + kWinRows * ld;
  float* qs = vs + kWinRows * ld;
  float* ps = qs + kWinQ * ld;  // [kWinQ][65] weights of each query over its 64 staged keys
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * kWinQ;
  const size_t base = (size_t)blockIdx.y * L * dh;
  q += base; k += base; v += base; out += base;

  umma::grid_dep_wait();  // the previous kernel in the stream has finished
  umma::grid_dep_launch();
  const int d4 = dh / 4;  // 16-byte pieces per row
  for (int idx = tid; idx < kWinRows * d4; idx += kWinThreads) {
    const int r = idx / d4, c = 4 * (idx - r * d4);
    const int g = t0 - (kWinK - 1) + r;
    const bool ok = g >= 0 && g < L;
    const size_t off = ok ? (size_t)g * dh + c : 0;
    umma::cp_async16(ks + r * ld + c, k + off, ok);
    umma::cp_async16(vs + r * ld + c, v + off, ok);
  }
  for (int idx = tid; idx < kWinQ * d4; idx += kWinThreads) {
    const int r = idx / d4, c = 4 * (idx - r * d4);
    const bool ok = t0 + r < L;
    umma::cp_async16(qs + r * ld + c, q + (ok ? (size_t)(t0 + r) * dh + c : 0), ok);
  }
  umma::cp_async_commit();
  umma::cp_async_wait<0>();
  __syncthreads();
  const int qi = tid / kWinSub, sub = tid % kWinSub;  // query of the block, key / column share
  const int t = t0 + qi;
  const int lo = max(0, t - W + 1);
  const float scale = rsqrtf((float)dh);
  const float4* q4 = reinterpret_cast<const float4*>(qs + qi * ld);
  // scores of keys j = sub + kWinSub jj: key s = t - 63 + j, staged row qi + j
  constexpr int kPer = kWinK / kWinSub;
  float sc[kPer];
  float m = -INFINITY;
#pragma unroll
  for (int jj = 0; jj < kPer; ++jj) {
    const int j = sub + kWinSub * jj;
    const int s = t - (kWinK - 1) + j;
    float a = -INFINITY;
    if (s >= lo) {
      const float4* k4 = reinterpret_cast<const float4*>(ks + (qi + j) * ld);
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
    sc[jj] = a;
    m = fmaxf(m, a);
  }
  // the threads of a query are consecutive lanes of one warp
#pragma unroll
  for (int o = 1; o < kWinSub; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float sum = 0.0f;
#pragma unroll
  for (int jj = 0; jj < kPer; ++jj) {
    const int j = sub + kWinSub * jj;
    const float e = (t - (kWinK - 1) + j >= lo) ? expf(sc[jj] - m) : 0.0f;
    ps[qi * kWinPP + j] = e;
    sum += e;
  }
#pragma unroll
  for (int o = 1; o < kWinSub; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float inv = 1.0f / sum;
  __syncwarp();  // the query's threads have written its 64 weights
  if (t >= L) return;
  // output columns [4 c4, 4 c4 + 4) for c4 = sub, sub + kWinSub, ... over all 64 keys
  const float* pr = ps + qi * kWinPP;
  for (int c4 = sub; c4 < dh / 4; c4 += kWinSub) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int j = 0; j < kWinK; ++j) {
      const float p = pr[j];
      const float4 y = reinterpret_cast<const float4*>(vs + (qi + j) * ld)[c4];
      acc.x = fmaf(p, y.x, acc.x);
      acc.y = fmaf(p, y.y, acc.y);
      acc.z = fmaf(p, y.z, acc.z);
      acc.w = fmaf(p, y.w, acc.w);
    }
    T* o = out + (size_t)t * dh + 4 * c4;
    o[0] = from_f32<T>(acc.x * inv);
    o[1] = from_f32<T>(acc.y * inv);
    o[2] = from_f32<T>(acc.z * inv);
    o[3] = from_f32<T>(acc.w * inv);
  }
}

}  // namespace based
