// linattn_simt.cuh -- causal Taylor linear attention on CUDA cores in fp32.
//
// The chunked ("fla_parallel") view of the based/train README, computed in fp32
// for fp32 inputs: per chunk of 32 tokens
//   A      = (phi(Q_c) phi(K_c)^T) masked to s <= t            (intra-chunk)
//   num_t  = phi(q_t)^T S + sum_s A_ts v_s,  den_t = phi(q_t).z + sum_s A_ts
//   y_t    = num_t / (den_t + eps)
//   S     += phi(K_c)^T V_c,  z += sum_s phi(k_s)                (state update)
// One CTA per (b, h, 8-column slice of d_v): the slices of one sequence share
// nothing but the scores, which are cheap, so a short sequence still spreads
// over several SMs.
//
// Two exact identities of the feature map shrink the work:
//  - A uses the closed form phi(q).phi(k) = 1 + u/4 + u^2/32 with u = q.k
//    (16 terms instead of 273);
//  - the quadratic features x_i x_j and x_j x_i are equal, so rows (i, j) and
//    (j, i) of S and z are equal too.  The CTA keeps 153 rows (constant,
//    16 linear, the 136 pairs i <= j) and weights an off-diagonal pair twice on
//    the query side, which gives phi(q)^T S exactly; the export writes every
//    pair row to both of its places in the 273-row state.
// Every feature is a product x[a] * x[b] * scale over the row extended by a 1
// (index 16): (16, 16) is the constant, (i, 16) the linear features.
//
// The kernel is bound by shared-memory accesses, so each phase is laid out to
// make one access feed many FMAs.  Per chunk two barriers:
//  (1) features: one warp per (q or k, eighth of the feature rows), one lane
//      per token row, the row in registers and the feature indices fixed at
//      compile time; scores: float4 loads, two query rows per thread;
//  (2) read-out on warps 0-7: one lane per row, warp w over feature rows
//      w, w+8, ... and keys w, w+8, ..., reading each state row at one address
//      for the whole warp; the eight partial sums meet in shared memory.
//      State update on warps 8-12: one thread per state row, all eight
//      columns and z, into the other of two state buffers.  Meanwhile the
//      next chunk's inputs, loaded into registers one chunk ahead, are staged.
#pragma once

#include "common.cuh"
#include "umma.cuh"

namespace based {

constexpr int kSimtChunk = 32;
constexpr int kSimtCols = 8;
constexpr int kSimtThreads = 512;
constexpr int kSimtFc = 1 + kD + kD * (kD + 1) / 2;  // 153 distinct feature rows
constexpr int kSimtFcPad = 160;                      // feature rows read (zeros past 153)
constexpr int kSimtSZ = 12;      // state row: S (8 columns), z, 3 zeros (48 bytes: the float4
                                 // reads of 8 consecutive rows fall in distinct banks)
constexpr int kSimtXP = 20;      // staged q, k rows: 16 values, float4-aligned, 8 rows of a
                                 // float4 phase in distinct banks
constexpr int kSimtFP = 169;     // feature rows (odd: 32 token rows in 32 banks)
constexpr int kSimtAP = 33;      // score rows (same reason)
constexpr int kSimtRO = 8;       // read-out warps

// Shared-memory carve-up, in floats.
constexpr int kSimtSBuf = kSimtFcPad * kSimtSZ;
constexpr int kSimtOffFq = 2 * kSimtSBuf;
constexpr int kSimtOffFk = kSimtOffFq + kSimtChunk * kSimtFP;
constexpr int kSimtOffRed = kSimtOffFk + kSimtChunk * kSimtFP;
constexpr int kSimtOffRedD = kSimtOffRed + kSimtRO * kSimtChunk * kSimtCols;
constexpr int kSimtOffV = kSimtOffRedD + kSimtRO * kSimtChunk;
constexpr int kSimtOffA = kSimtOffV + 2 * kSimtChunk * kSimtCols;
constexpr int kSimtOffXq = kSimtOffA + kSimtChunk * kSimtAP;
constexpr int kSimtOffXk = kSimtOffXq + kSimtChunk * kSimtXP;
constexpr int kSimtFloats = kSimtOffXk + kSimtChunk * kSimtXP;
static_assert(kSimtOffRed % 4 == 0 && kSimtOffV % 4 == 0 && kSimtOffXq % 4 == 0 &&
                  kSimtOffXk % 4 == 0, "float4 alignment");

__host__ __device__ constexpr size_t linattn_simt_smem_bytes() {
  return sizeof(float) * (size_t)kSimtFloats;
}

// Row of the 153-row state that holds feature f of the 273-row map: f itself
// for the constant and linear features; for the quadratic feature (i, j) the
// pair (a, b) = (min, max) in row-major order over a <= b.
__device__ __forceinline__ int simt_state_row(int f) {
  if (f <= kD) return f;
  const int i = (f - kD - 1) >> 4, j = (f - kD - 1) & 15;
  const int a = min(i, j), b = max(i, j);
  return kD + 1 + a * kD - (a * (a - 1)) / 2 + (b - a);
}

// The factors (a, b) of state row r (inverse of the map above; index 16 is the 1).
__host__ __device__ constexpr int simt_row_a(int r) {
  if (r == 0) return kD;
  if (r <= kD) return r - 1;
  int p = r - kD - 1, a = 0;
  while (p >= kD - a) p -= kD - a++;
  return a;
}
__host__ __device__ constexpr int simt_row_b(int r) {
  if (r <= kD) return kD;
  int p = r - kD - 1, a = 0;
  while (p >= kD - a) p -= kD - a++;
  return a + p;
}

// Feature rows P, P+8, ... of one token row x (x[16] = 1, or 0 for a key row
// past the end), with the indices fixed at compile time.
template <int P, int M = 0>
__device__ __forceinline__ void simt_features(const float (&x)[kD + 1], float* dst, bool key) {
  if constexpr (P + 8 * M < kSimtFc) {
    constexpr int r = P + 8 * M, a = simt_row_a(r), b = simt_row_b(r);
    constexpr float sk = r == 0 ? 1.0f : r <= kD ? kLinScale : kQuadScale;
    constexpr float sq = r > kD && a != b ? 2.0f * kQuadScale : sk;
    dst[r] = (x[a] * x[b]) * (key ? sk : sq);
    simt_features<P, M + 1>(x, dst, key);
  }
}

__device__ __forceinline__ float simt_score(float u) {
  return fmaf(u, fmaf(u, 0.03125f, 0.25f), 1.0f);  // phi(q).phi(k) from u = q.k
}

template <typename T>
__global__ void __launch_bounds__(kSimtThreads) linattn_simt_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    T* __restrict__ out, float* __restrict__ state_kv, float* __restrict__ state_k, int L,
    int DV, float eps) {
  constexpr int C = kSimtChunk, NC = kSimtCols, NT = kSimtThreads, FC = kSimtFc;
  constexpr int kQK = C * kD / NT, kVV = (C * NC + NT - 1) / NT;  // staged per thread
  static_assert(C == 32 && NC == 8 && NT == 512 && C * kD == NT, "thread layout");
  static_assert(FC <= 5 * 32, "state update: one thread per row on warps 8-12");
  extern __shared__ __align__(16) float smem[];
  float* SZ2 = smem;                  // 2 x [160][12]  state rows: S, z
  float* fq = smem + kSimtOffFq;      // [32][169]      phi(q) (off-diagonal pairs doubled)
  float* fk = smem + kSimtOffFk;      // [32][169]      phi(k), zero rows past the end
  float* red = smem + kSimtOffRed;    // [8][32][8]     read-out partial numerators
  float* redd = smem + kSimtOffRedD;  // [8][32]        read-out partial denominators
  float* vs2 = smem + kSimtOffV;      // 2 x [32][8]
  float* A = smem + kSimtOffA;        // [32][33]
  float* xq = smem + kSimtOffXq;      // [32][20]
  float* xk = smem + kSimtOffXk;      // [32][20]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x, col0 = blockIdx.y * NC;
  q += (size_t)bh * L * kD;
  k += (size_t)bh * L * kD;
  v += (size_t)bh * L * DV + col0;
  out += (size_t)bh * L * DV + col0;

  for (int i = tid; i < kSimtOffRed; i += NT) smem[i] = 0.0f;  // states, feature tiles
  // the set-up above touched no global memory: it overlaps the previous kernel
  umma::grid_dep_wait();
  umma::grid_dep_launch();

  float rq[kQK], rk[kQK], rv[kVV];
  auto fetch = [&](int t0) {
#pragma unroll
    for (int m = 0; m < kQK; ++m) {
      const int i = tid + m * NT;
      const bool ok = t0 + i / kD < L;
      rq[m] = ok ? to_f32(q[(size_t)t0 * kD + i]) : 0.0f;
      rk[m] = ok ? to_f32(k[(size_t)t0 * kD + i]) : 0.0f;
    }
#pragma unroll
    for (int m = 0; m < kVV; ++m) {
      const int i = tid + m * NT, r = i / NC, c = i - r * NC;
      rv[m] = i < C * NC && t0 + r < L ? to_f32(v[(size_t)(t0 + r) * DV + c]) : 0.0f;
    }
  };
  auto stage = [&](int buf) {
#pragma unroll
    for (int m = 0; m < kQK; ++m) {
      const int i = tid + m * NT, r = i / kD, c = i - r * kD;
      xq[r * kSimtXP + c] = rq[m];
      xk[r * kSimtXP + c] = rk[m];
    }
#pragma unroll
    for (int m = 0; m < kVV; ++m)
      if (tid + m * NT < C * NC) vs2[buf * C * NC + tid + m * NT] = rv[m];
  };

  if (L > 0) {
    fetch(0);
    stage(0);
    if (C < L) fetch(C);
  }

  int nchunks = 0;
  for (int t0 = 0; t0 < L; t0 += C, ++nchunks) {
    const int n = min(C, L - t0), cur = nchunks & 1;
    __syncthreads();  // chunk inputs staged; the previous read-out and update are done

    {  // features of token row `lane`: warps 0-7 the query, 8-15 the key
      const bool key = warp >= 8;
      const float4* xr = reinterpret_cast<const float4*>((key ? xk : xq) + lane * kSimtXP);
      float x[kD + 1];
#pragma unroll
      for (int c = 0; c < kD / 4; ++c) {
        const float4 t4 = xr[c];
        x[4 * c] = t4.x;
        x[4 * c + 1] = t4.y;
        x[4 * c + 2] = t4.z;
        x[4 * c + 3] = t4.w;
      }
      x[kD] = key && lane >= n ? 0.0f : 1.0f;  // key rows past the end: all features zero
      float* dst = (key ? fk : fq) + lane * kSimtFP;
      switch (warp & 7) {
        case 0: simt_features<0>(x, dst, key); break;
        case 1: simt_features<1>(x, dst, key); break;
        case 2: simt_features<2>(x, dst, key); break;
        case 3: simt_features<3>(x, dst, key); break;
        case 4: simt_features<4>(x, dst, key); break;
        case 5: simt_features<5>(x, dst, key); break;
        case 6: simt_features<6>(x, dst, key); break;
        default: simt_features<7>(x, dst, key); break;
      }
    }
    {  // intra-chunk scores of query rows `warp` and `warp`+16 with key `lane`
      const float4* k4 = reinterpret_cast<const float4*>(xk + lane * kSimtXP);
      const float4* qa = reinterpret_cast<const float4*>(xq + warp * kSimtXP);
      const float4* qb = reinterpret_cast<const float4*>(xq + (warp + 16) * kSimtXP);
      float ua = 0.0f, ub = 0.0f, ua2 = 0.0f, ub2 = 0.0f;
#pragma unroll
      for (int c = 0; c < kD / 4; ++c) {
        const float4 y = k4[c], a4 = qa[c], b4 = qb[c];
        ua = fmaf(a4.x, y.x, ua);
        ua2 = fmaf(a4.y, y.y, ua2);
        ua = fmaf(a4.z, y.z, ua);
        ua2 = fmaf(a4.w, y.w, ua2);
        ub = fmaf(b4.x, y.x, ub);
        ub2 = fmaf(b4.y, y.y, ub2);
        ub = fmaf(b4.z, y.z, ub);
        ub2 = fmaf(b4.w, y.w, ub2);
      }
      A[warp * kSimtAP + lane] = lane <= warp ? simt_score(ua + ua2) : 0.0f;
      A[(warp + 16) * kSimtAP + lane] = lane <= warp + 16 ? simt_score(ub + ub2) : 0.0f;
    }
    __syncthreads();

    const float* SZc = SZ2 + cur * kSimtSBuf;
    const float* vc = vs2 + cur * C * NC;
    if (warp < kSimtRO) {
      // read-out of row `lane`: this warp's share of the feature rows and keys
      float acc[NC], den = 0.0f;
#pragma unroll
      for (int c = 0; c < NC; ++c) acc[c] = 0.0f;
      const float* fr = fq + lane * kSimtFP;
#pragma unroll 4
      for (int f = warp; f < kSimtFcPad; f += kSimtRO) {  // rows 153..159 are zero
        const float a = fr[f];
        const float* sr = SZc + f * kSimtSZ;
        const float4 s0 = *reinterpret_cast<const float4*>(sr);
        const float4 s1 = *reinterpret_cast<const float4*>(sr + 4);
        acc[0] = fmaf(a, s0.x, acc[0]);
        acc[1] = fmaf(a, s0.y, acc[1]);
        acc[2] = fmaf(a, s0.z, acc[2]);
        acc[3] = fmaf(a, s0.w, acc[3]);
        acc[4] = fmaf(a, s1.x, acc[4]);
        acc[5] = fmaf(a, s1.y, acc[5]);
        acc[6] = fmaf(a, s1.z, acc[6]);
        acc[7] = fmaf(a, s1.w, acc[7]);
        den = fmaf(a, sr[NC], den);
      }
#pragma unroll
      for (int s = warp; s < C; s += kSimtRO) {
        const float a = A[lane * kSimtAP + s];
        const float4 v0 = *reinterpret_cast<const float4*>(vc + s * NC);
        const float4 v1 = *reinterpret_cast<const float4*>(vc + s * NC + 4);
        acc[0] = fmaf(a, v0.x, acc[0]);
        acc[1] = fmaf(a, v0.y, acc[1]);
        acc[2] = fmaf(a, v0.z, acc[2]);
        acc[3] = fmaf(a, v0.w, acc[3]);
        acc[4] = fmaf(a, v1.x, acc[4]);
        acc[5] = fmaf(a, v1.y, acc[5]);
        acc[6] = fmaf(a, v1.z, acc[6]);
        acc[7] = fmaf(a, v1.w, acc[7]);
        den += a;
      }
      float4* rp = reinterpret_cast<float4*>(red + (warp * C + lane) * NC);
      rp[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      rp[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      redd[warp * C + lane] = den;
      asm volatile("bar.sync 1, %0;" ::"n"(kSimtRO * 32) : "memory");  // read-out warps only
      const int ot = tid >> 3, oc = tid & 7;  // output row, column
      float num = 0.0f, dd = 0.0f;
#pragma unroll
      for (int w = 0; w < kSimtRO; ++w) {
        num += red[(w * C + ot) * NC + oc];
        dd += redd[w * C + ot];
      }
      if (ot < n) out[(size_t)(t0 + ot) * DV + oc] = from_f32<T>(num / (dd + eps));
    } else {
      // state update of row f into the other buffer
      const int f = tid - kSimtRO * 32;
      if (f < FC) {
        const float* sr = SZc + f * kSimtSZ;
        float4 s0 = *reinterpret_cast<const float4*>(sr);
        float4 s1 = *reinterpret_cast<const float4*>(sr + 4);
        float zs = 0.0f;
#pragma unroll
        for (int s = 0; s < C; ++s) {
          const float a = fk[s * kSimtFP + f];
          const float4 v0 = *reinterpret_cast<const float4*>(vc + s * NC);
          const float4 v1 = *reinterpret_cast<const float4*>(vc + s * NC + 4);
          s0.x = fmaf(a, v0.x, s0.x);
          s0.y = fmaf(a, v0.y, s0.y);
          s0.z = fmaf(a, v0.z, s0.z);
          s0.w = fmaf(a, v0.w, s0.w);
          s1.x = fmaf(a, v1.x, s1.x);
          s1.y = fmaf(a, v1.y, s1.y);
          s1.z = fmaf(a, v1.z, s1.z);
          s1.w = fmaf(a, v1.w, s1.w);
          zs += a;
        }
        float* sn = SZ2 + (cur ^ 1) * kSimtSBuf + f * kSimtSZ;
        *reinterpret_cast<float4*>(sn) = s0;
        *reinterpret_cast<float4*>(sn + 4) = s1;
        sn[NC] = sr[NC] + zs;
      }
    }
    if (t0 + C < L) {  // stage the next chunk (its q, k are read only after the next barrier)
      stage(cur ^ 1);
      if (t0 + 2 * C < L) fetch(t0 + 2 * C);
    }
  }
  __syncthreads();
  const float* SZf = SZ2 + (nchunks & 1) * kSimtSBuf;
  if (state_kv) {
    float* dst = state_kv + (size_t)bh * kF * DV + col0;
    for (int i = tid; i < kF * NC; i += NT) {
      const int f = i / NC, c = i - f * NC;
      dst[(size_t)f * DV + c] = SZf[simt_state_row(f) * kSimtSZ + c];
    }
  }
  if (state_k && blockIdx.y == 0) {
    for (int f = tid; f < kF; f += NT)
      state_k[(size_t)bh * kF + f] = SZf[simt_state_row(f) * kSimtSZ + NC];
  }
}

}  // namespace based
