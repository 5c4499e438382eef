// linattn_simt.cuh -- causal Taylor linear attention on CUDA cores in fp32.
//
// The chunked ("fla_parallel") view of the based/train README, computed in fp32
// for fp32 inputs: per chunk of 32 tokens
//   A      = (phi(Q_c) phi(K_c)^T) masked to s <= t            (intra-chunk)
//   num_t  = phi(q_t)^T S + sum_s A_ts v_s,  den_t = phi(q_t).z + sum_s A_ts
//   y_t    = num_t / (den_t + eps)
//   S     += phi(K_c)^T V_c,  z += sum_s phi(k_s)                (state update)
// with S (273 x 8 fp32) and z resident in shared memory for the whole
// sequence.  One CTA per (b, h, 8-column slice of d_v): the slices of one
// sequence share nothing but the scores, which are cheap, so a short sequence
// still spreads over several SMs.  A uses the closed form phi(q).phi(k) =
// 1 + u/4 + u^2/32 with u = q.k (an identity of the map above, 16 terms instead
// of 273); the read-out and the state use all 273 features.  The feature rows
// use a pitch of 273 floats (odd), so a warp reading one feature of 32
// different tokens touches 32 distinct banks.
#pragma once

#include "common.cuh"

namespace based {

constexpr int kSimtChunk = 32;
constexpr int kSimtCols = 8;
constexpr int kSimtThreads = 256;
constexpr int kSimtXP = kD + 1;  // pitch of the staged q, k rows (odd: the score loop's
                                 // 32 lanes read 32 different rows without bank conflicts)

__host__ __device__ constexpr size_t linattn_simt_smem_bytes() {
  return sizeof(float) * (size_t)(kF * kSimtCols + 276 + 2 * kSimtChunk * kF +
                                  kSimtChunk * kSimtCols + kSimtChunk * 33 + kSimtChunk +
                                  2 * kSimtChunk * kSimtXP);
}

template <typename T>
__global__ void __launch_bounds__(kSimtThreads) linattn_simt_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    T* __restrict__ out, float* __restrict__ state_kv, float* __restrict__ state_k, int L,
    int DV, float eps) {
  constexpr int C = kSimtChunk, NC = kSimtCols, NT = kSimtThreads;
  constexpr int G = NT / NC;   // row groups
  constexpr int RPT = C / G;   // rows per thread in the numerator
  static_assert(NT % NC == 0 && C % G == 0, "thread layout");
  extern __shared__ __align__(16) float smem[];
  float* S = smem;                 // [273][kSimtCols]
  float* z = S + kF * NC;          // [273] (+pad)
  float* fq = z + 276;             // [32][273]
  float* fk = fq + C * kF;         // [32][273]
  float* vs = fk + C * kF;         // [32][kSimtCols]
  float* A = vs + C * NC;          // [32][33]
  float* den = A + C * 33;         // [32]
  float* xq = den + C;             // [32][17]
  float* xk = xq + C * kSimtXP;    // [32][17]

  const int tid = threadIdx.x;
  const int bh = blockIdx.x, col0 = blockIdx.y * NC;
  q += (size_t)bh * L * kD;
  k += (size_t)bh * L * kD;
  v += (size_t)bh * L * DV + col0;
  out += (size_t)bh * L * DV + col0;

  for (int i = tid; i < kF * NC; i += NT) S[i] = 0.0f;
  for (int i = tid; i < 276; i += NT) z[i] = 0.0f;

  const int j = tid % NC, grp = tid / NC;  // output column, row group (0..G-1)
  for (int t0 = 0; t0 < L; t0 += C) {
    const int n = min(C, L - t0);
    __syncthreads();  // previous chunk's state update is complete
    for (int i = tid; i < C * kD; i += NT) {
      const int r = i / kD, c = i - r * kD;
      xq[r * kSimtXP + c] = r < n ? to_f32(q[(size_t)t0 * kD + i]) : 0.0f;
      xk[r * kSimtXP + c] = r < n ? to_f32(k[(size_t)t0 * kD + i]) : 0.0f;
    }
    for (int i = tid; i < C * NC; i += NT) {
      const int r = i / NC, c = i - r * NC;
      vs[i] = r < n ? to_f32(v[(size_t)(t0 + r) * DV + c]) : 0.0f;
    }
    __syncthreads();
    for (int i = tid; i < C * kF; i += NT) {
      const int r = i / kF, f = i - r * kF;
      fq[i] = phi_feature(xq + r * kSimtXP, f);
      fk[i] = phi_feature(xk + r * kSimtXP, f);
    }
    __syncthreads();
    // intra-chunk scores, causal mask s <= t, in closed form from u = q_t . k_s
    for (int i = tid; i < C * C; i += NT) {
      const int t = i / C, s = i - t * C;
      float a = 0.0f;
      if (s <= t) {
        const float* qr = xq + t * kSimtXP;
        const float* kr = xk + s * kSimtXP;
        float u2[2] = {0.0f, 0.0f};
#pragma unroll
        for (int d = 0; d < kD; ++d) u2[d & 1] = fmaf(qr[d], kr[d], u2[d & 1]);
        const float u = u2[0] + u2[1];
        a = fmaf(u, fmaf(u, 0.03125f, 0.25f), 1.0f);
      }
      A[t * 33 + s] = a;
    }
    __syncthreads();
    // denominators: inter (phi(q).z) + intra (row sum of A)
    if (tid < C) {
      float d = 0.0f;
      const float* a_row = fq + tid * kF;
      for (int f = 0; f < kF; ++f) d = fmaf(a_row[f], z[f], d);
      for (int s = 0; s < C; ++s) d += A[tid * 33 + s];
      den[tid] = d;
    }
    // numerators for rows grp, grp+G, ..., column j
    float acc[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) acc[i] = 0.0f;
    for (int f = 0; f < kF; ++f) {
      const float sf = S[f * NC + j];
#pragma unroll
      for (int i = 0; i < RPT; ++i) acc[i] = fmaf(fq[(grp + G * i) * kF + f], sf, acc[i]);
    }
    for (int s = 0; s < C; ++s) {
      const float vj = vs[s * NC + j];
#pragma unroll
      for (int i = 0; i < RPT; ++i) acc[i] = fmaf(A[(grp + G * i) * 33 + s], vj, acc[i]);
    }
    __syncthreads();  // den ready; all reads of S and z for this chunk done
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      const int t = grp + G * i;
      if (t < n) out[(size_t)(t0 + t) * DV + j] = from_f32<T>(acc[i] / (den[t] + eps));
    }
    // state update over the chunk's 32 rows (rows past the end have v = 0;
    // z skips them), four partial sums per entry
    for (int f = grp; f < kF; f += G) {
      float s4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int s = 0; s < C; ++s) s4[s & 3] = fmaf(fk[s * kF + f], vs[s * NC + j], s4[s & 3]);
      S[f * NC + j] += (s4[0] + s4[1]) + (s4[2] + s4[3]);
    }
    for (int f = tid; f < kF; f += NT) {
      float z4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int s = 0; s < C; ++s) z4[s & 3] += s < n ? fk[s * kF + f] : 0.0f;
      z[f] += (z4[0] + z4[1]) + (z4[2] + z4[3]);
    }
  }
  __syncthreads();
  if (state_kv) {
    float* dst = state_kv + (size_t)bh * kF * DV + col0;
    for (int i = tid; i < kF * NC; i += NT) {
      const int f = i / NC, c = i - f * NC;
      dst[(size_t)f * DV + c] = S[i];
    }
  }
  if (state_k && blockIdx.y == 0) {
    for (int f = tid; f < kF; f += NT) state_k[(size_t)bh * kF + f] = z[f];
  }
}

}  // namespace based
