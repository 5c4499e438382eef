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
// Every feature is a product x[a] * x[b] * scale over the staged row extended
// by a 1 (column 16): (16, 16) is the constant, (i, 16) the linear features.
//
// Per chunk two barriers: (1) the features of q and k and the scores, (2) the
// read-out of every row and the state update, which read the state of the
// previous chunk and write the other of two state buffers, while the next
// chunk's inputs (loaded into registers one chunk ahead) are staged.
#pragma once

#include "common.cuh"

namespace based {

constexpr int kSimtChunk = 32;
constexpr int kSimtCols = 8;
constexpr int kSimtThreads = 512;
constexpr int kSimtFc = 1 + kD + kD * (kD + 1) / 2;  // 153 distinct feature rows
constexpr int kSimtFcPad = 160;                      // rows of a state buffer (zeros past 153)
constexpr int kSimtXP = kD + 1;  // staged q, k row: 16 values and the 1 (odd pitch: the
                                 // score loop's 32 lanes read 32 different rows conflict-free)
constexpr int kSimtFP = 168;     // pitch of the feature rows and (below) of the score rows:
constexpr int kSimtAP = 40;      // 8 banks apart, so the rows and feature lanes of a read-out
                                 // warp fall in different banks

// Shared-memory carve-up, in floats.
constexpr int kSimtSBuf = kSimtFcPad * kSimtCols;
constexpr int kSimtOffZ = 2 * kSimtSBuf;
constexpr int kSimtOffFq = kSimtOffZ + 2 * kSimtFcPad;
constexpr int kSimtOffFk = kSimtOffFq + kSimtChunk * kSimtFP;
constexpr int kSimtOffV = kSimtOffFk + kSimtChunk * kSimtFP;
constexpr int kSimtOffA = kSimtOffV + 2 * kSimtChunk * kSimtCols;
constexpr int kSimtOffXq = kSimtOffA + kSimtChunk * kSimtAP;
constexpr int kSimtOffXk = kSimtOffXq + kSimtChunk * kSimtXP;
constexpr int kSimtOffTab = kSimtOffXk + kSimtChunk * kSimtXP;
constexpr int kSimtFloats = kSimtOffTab + 3 * kSimtFcPad;
static_assert(kSimtOffV % 4 == 0, "float4 alignment of the value tiles");

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

template <typename T>
__global__ void __launch_bounds__(kSimtThreads) linattn_simt_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    T* __restrict__ out, float* __restrict__ state_kv, float* __restrict__ state_k, int L,
    int DV, float eps) {
  constexpr int C = kSimtChunk, NC = kSimtCols, NT = kSimtThreads, FC = kSimtFc;
  constexpr int kQK = (C * kD + NT - 1) / NT, kVV = (C * NC + NT - 1) / NT;  // staged per thread
  constexpr int FL = NT / (C * (NC / 4));  // feature lanes per output row and column group
  static_assert(FL == 4 || FL == 8, "read-out layout: row x 4-column group x 4 or 8 lanes");
  extern __shared__ __align__(16) float smem[];
  float* S2 = smem;                 // 2 x [160][8]  (state: rows of the 153-row map)
  float* z2 = smem + kSimtOffZ;     // 2 x [160]
  float* fq = smem + kSimtOffFq;    // [32][168]     phi(q) (off-diagonal pairs doubled)
  float* fk = smem + kSimtOffFk;    // [32][168]     phi(k), zero rows past the end
  float* vs2 = smem + kSimtOffV;    // 2 x [32][8]
  float* A = smem + kSimtOffA;      // [32][40]
  float* xq = smem + kSimtOffXq;    // [32][17]
  float* xk = smem + kSimtOffXk;    // [32][17]
  int* tab = reinterpret_cast<int*>(smem + kSimtOffTab);  // [160] a | b << 8
  float* scq = smem + kSimtOffTab + kSimtFcPad;           // [160] query-side scale
  float* sck = scq + kSimtFcPad;                          // [160] key-side scale

  const int tid = threadIdx.x;
  const int bh = blockIdx.x, col0 = blockIdx.y * NC;
  q += (size_t)bh * L * kD;
  k += (size_t)bh * L * kD;
  v += (size_t)bh * L * DV + col0;
  out += (size_t)bh * L * DV + col0;

  for (int i = tid; i < kSimtOffV; i += NT) smem[i] = 0.0f;  // states, z, feature tiles
  for (int r = tid; r < C; r += NT) xq[r * kSimtXP + kD] = xk[r * kSimtXP + kD] = 1.0f;
  for (int f = tid; f < kF; f += NT) {
    int a = kD, b = kD;
    float sq = 1.0f, sk = 1.0f;
    bool own = true;
    if (f > 0 && f <= kD) {
      a = f - 1;
      sq = sk = kLinScale;
    } else if (f > kD) {
      const int i = (f - kD - 1) >> 4, j = (f - kD - 1) & 15;
      own = i <= j;
      a = i;
      b = j;
      sk = kQuadScale;
      sq = i == j ? kQuadScale : 2.0f * kQuadScale;
    }
    if (own) {
      const int r = simt_state_row(f);
      tab[r] = a | (b << 8);
      scq[r] = sq;
      sck[r] = sk;
    }
  }

  float rq[kQK], rk[kQK], rv[kVV];
  auto fetch = [&](int t0) {
#pragma unroll
    for (int m = 0; m < kQK; ++m) {
      const int i = tid + m * NT;
      const bool ok = i < C * kD && t0 + i / kD < L;
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
      if (i < C * kD) {
        xq[r * kSimtXP + c] = rq[m];
        xk[r * kSimtXP + c] = rk[m];
      }
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

  // read-out layout: row t, columns 4*cg .. 4*cg+3, feature rows fl, fl+FL, ...; lane bits
  // (fl0, fl1, cg, fl2): the 8 lanes of a float4 phase read 8 different 16-byte words
  const int fl = (tid & 3) | (FL == 8 ? ((tid >> 3) & 1) << 2 : 0);
  const int cg = (tid >> 2) & 1, t = FL == 8 ? tid >> 4 : tid >> 3;
  int nchunks = 0;
  for (int t0 = 0; t0 < L; t0 += C, ++nchunks) {
    const int n = min(C, L - t0), cur = nchunks & 1;
    __syncthreads();  // chunk inputs staged; the previous read-out and update are done

    // features: items (q or k, feature row, half of the chunk's rows)
    for (int it = tid; it < 4 * FC; it += NT) {
      const bool key = it >= 2 * FC;
      const int rem = key ? it - 2 * FC : it;
      const int half = rem >= FC;
      const int f = rem - half * FC;
      const int e = tab[f], a = e & 0xff, b = e >> 8;
      const float sc = key ? sck[f] : scq[f];
      const float* xr = (key ? xk : xq) + half * (C / 2) * kSimtXP;
      float* dst = (key ? fk : fq) + half * (C / 2) * kSimtFP + f;
      const int live = key ? n - half * (C / 2) : C;  // key rows past the end stay zero
#pragma unroll
      for (int r = 0; r < C / 2; ++r) {
        const float val = (xr[r * kSimtXP + a] * xr[r * kSimtXP + b]) * sc;
        dst[r * kSimtFP] = r < live ? val : 0.0f;
      }
    }
    // intra-chunk scores, causal mask s <= t, in closed form from u = q_t . k_s
    for (int i = tid; i < C * C; i += NT) {
      const int tt = i / C, s = i - tt * C;
      float a = 0.0f;
      if (s <= tt) {
        const float* qr = xq + tt * kSimtXP;
        const float* kr = xk + s * kSimtXP;
        float u2[2] = {0.0f, 0.0f};
#pragma unroll
        for (int d = 0; d < kD; ++d) u2[d & 1] = fmaf(qr[d], kr[d], u2[d & 1]);
        const float u = u2[0] + u2[1];
        a = fmaf(u, fmaf(u, 0.03125f, 0.25f), 1.0f);
      }
      A[tt * kSimtAP + s] = a;
    }
    __syncthreads();

    const float* Sc = S2 + cur * kSimtSBuf;
    const float* zc = z2 + cur * kSimtFcPad;
    const float* vc = vs2 + cur * C * NC;
    // read-out: FL lanes split the feature rows (rows 153..159 are zero)
    {
      float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      float den = 0.0f;
      const float* fr = fq + t * kSimtFP;
#pragma unroll 4
      for (int f = fl; f < kSimtFcPad; f += FL) {
        const float a = fr[f];
        const float4 s4 = *reinterpret_cast<const float4*>(Sc + f * NC + 4 * cg);
        acc.x = fmaf(a, s4.x, acc.x);
        acc.y = fmaf(a, s4.y, acc.y);
        acc.z = fmaf(a, s4.z, acc.z);
        acc.w = fmaf(a, s4.w, acc.w);
        den = fmaf(a, zc[f], den);
      }
      const float* ar = A + t * kSimtAP;
#pragma unroll
      for (int s = fl; s < C; s += FL) {
        const float a = ar[s];
        const float4 v4 = *reinterpret_cast<const float4*>(vc + s * NC + 4 * cg);
        acc.x = fmaf(a, v4.x, acc.x);
        acc.y = fmaf(a, v4.y, acc.y);
        acc.z = fmaf(a, v4.z, acc.z);
        acc.w = fmaf(a, v4.w, acc.w);
        den += a;
      }
#pragma unroll
      for (int o = 1; o < 2 * FL; o <<= 1) {
        if (o == 4) continue;  // lane bit 2 is the column group
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
        den += __shfl_xor_sync(0xffffffffu, den, o);
      }
      const int c = fl & 3;
      const float num = c == 0 ? acc.x : c == 1 ? acc.y : c == 2 ? acc.z : acc.w;
      if (t < n && fl < 4) out[(size_t)(t0 + t) * DV + 4 * cg + c] = from_f32<T>(num / (den + eps));
    }
    // state update into the other buffer: items (feature row, 4-column group)
    {
      float* Sn = S2 + (cur ^ 1) * kSimtSBuf;
      float* zn = z2 + (cur ^ 1) * kSimtFcPad;
      for (int it = tid; it < 2 * FC; it += NT) {
        const int f = it >> 1, c4 = (it & 1) * 4;
        float4 s4 = *reinterpret_cast<const float4*>(Sc + f * NC + c4);
        float zs = 0.0f;
#pragma unroll
        for (int s = 0; s < C; ++s) {
          const float a = fk[s * kSimtFP + f];
          const float4 v4 = *reinterpret_cast<const float4*>(vc + s * NC + c4);
          s4.x = fmaf(a, v4.x, s4.x);
          s4.y = fmaf(a, v4.y, s4.y);
          s4.z = fmaf(a, v4.z, s4.z);
          s4.w = fmaf(a, v4.w, s4.w);
          zs += a;
        }
        *reinterpret_cast<float4*>(Sn + f * NC + c4) = s4;
        if (c4 == 0) zn[f] = zc[f] + zs;
      }
    }
    if (t0 + C < L) {  // stage the next chunk (its q, k are read only after the next barrier)
      stage(cur ^ 1);
      if (t0 + 2 * C < L) fetch(t0 + 2 * C);
    }
  }
  __syncthreads();
  const float* Sf = S2 + (nchunks & 1) * kSimtSBuf;
  const float* zf = z2 + (nchunks & 1) * kSimtFcPad;
  if (state_kv) {
    float* dst = state_kv + (size_t)bh * kF * DV + col0;
    for (int i = tid; i < kF * NC; i += NT) {
      const int f = i / NC, c = i - f * NC;
      dst[(size_t)f * DV + c] = Sf[simt_state_row(f) * NC + c];
    }
  }
  if (state_k && blockIdx.y == 0) {
    for (int f = tid; f < kF; f += NT) state_k[(size_t)bh * kF + f] = zf[simt_state_row(f)];
  }
}

}  // namespace based
