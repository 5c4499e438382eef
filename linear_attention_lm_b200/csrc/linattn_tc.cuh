// linattn_tc.cuh -- causal Taylor linear attention on the sm_100a tensor cores.
//
// Method ("Базированная модель, часть 2", section "Что за линейное внимание?";
// based/train README, training views): y_t = phi(q_t)^T S_t / (phi(q_t).z_t + eps)
// with S_t = sum_{s<=t} phi(k_s) v_s^T, z_t = sum_{s<=t} phi(k_s).  The kernel runs
// the chunked ("fla_parallel") view, chunks of C = 128 tokens:
//
//   #1  U   = Q_c K_c^T                      (tcgen05, K = 16)           -> TMEM
//       P   = mask_{s<=t}(1 + U/4 + U^2/32)  (CUDA cores, from TMEM)     -> smem
//   #2  O   = phiQ_c [S | z]_{c-1}           (tcgen05, K = 160 features) -> TMEM
//   #4  O  += P [V_c | 1]                    (tcgen05, K = 128 tokens)
//   #5  [S|z] += phiK_c^T [V_c | 1]          (tcgen05, fp32 master state in TMEM)
//       y   = O[:, :dv] / (O[:, dv] + eps)   (CUDA cores, from TMEM)
//
// Exact reformulations used (both are identities, not approximations):
//  * the intra-chunk scores phi(q).phi(k) are evaluated in closed form,
//    1 + u + u^2/2 with u = q.k / 4 (the expansion the blog post prints), so
//    #1 contracts over the 16 input dims instead of the 273 features;
//  * phi(q).phi(k) only needs the 153 distinct products: 1, x_i/2, and for each
//    unordered pair {i, j} one feature (x_i/2)(x_j/2) c with c = 1/sqrt 2 on the
//    diagonal and 1 off it (the full map lists every off-diagonal product twice
//    with weight 1/(4 sqrt 2)).  The state is kept over these 153 features and
//    expanded to the 273-row layout (off-diagonal rows = value / sqrt 2,
//    duplicated) only on export.
// The ones column appended to V makes the normaliser z and both parts of the
// denominator come out of the same MMAs, with the same rounded operands as the
// numerator.
//
// Feature order inside the kernel (160 = 20 chunks of 8): chunk 0 = [1, 0 x 7],
// chunks 1-2 = x_i/2, chunks 3-4 = (x_i/2)^2/sqrt 2, then for d = 1..7 two chunks
// of (x_i/2)(x_{i+d mod 16}/2), i = 0..15, and chunk 19 = (x_i/2)(x_{i+8}/2),
// i = 0..7.  With x held as eight packed pairs X[m] = (x_2m, x_2m+1)/2 and the
// shifted pairs Y[m] = (x_2m+1, x_2m+2)/2, every pair of features is a single
// bf16x2 / f16x2 multiply X[m] * X[m + d/2] (d even) or X[m] * Y[m + (d-1)/2].
//
// Operand precision: Q, K, V, P and phiK are bf16; phiQ and the per-chunk copy
// of the state used by #2 are fp16 (bf16 inputs are exact in fp16; the state
// copy is scaled by a power of two so it stays in fp16 range for any L, and P is
// scaled by the same power so the ratio is unchanged).  All accumulation is fp32
// in TMEM; the master state never leaves TMEM until the export.
//
// Schedule (warp-specialised, chunks pipelined), 64 value columns per CTA (a
// sequence with d_v = 128 runs as two CTAs, one per 64-column slice of v: the
// denominator does not depend on v):
//   group P (warps 0-3):  P of chunk c from U, written back over U in TMEM;
//   group F (warps 4-7):  Q/K tiles and phiK of chunk c+1 (shared memory) and its
//            phiQ (TMEM), while group P still works on chunk c;
//   group E (warps 8-11): epilogue of chunk c -- y from O, and the fp16 copy of the
//            state for chunk c+1; once chunk c's MMAs are done, the V tile of
//            chunk c+3 into its stage (TMA);
//   issue warp (warp 12, one thread): the first three V tiles, then the MMAs in
//            the order #1, #5, #2, (P), #4 -- and nothing else, since every
//            instruction it runs between two MMA groups leaves the tensor pipe idle.
// The state is kept transposed in TMEM, [S|z]^T: lane j holds value column j
// (lane DV holds z), column f holds feature f, so #5 is one N = 160 MMA per K
// step.  Warps w, w+4 and w+8 share TMEM lane quadrant w, so each group reads and
// writes the TMEM rows of its own 32 tokens.  Hand-offs are mbarriers (arrivals
// from warp groups, or a tcgen05.commit); every wait is bounded.
//
// Long sequences are split into n_seg segments of seg_chunks chunks so that
// B*H*n_seg CTAs fill the GPU: a state-only pass (kStateOnly) runs #5 alone
// over every segment but the last and writes each segment's partial [S|z]
// (fp32, 160 x (dv+16)) to the caller's workspace; the main pass then seeds
// segment g's TMEM state with the sum of the partials of segments 0..g-1.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"
#include "umma.cuh"

// Optional per-chunk event stamps for performance analysis: a build may define
// BASED_TC_TRACE(event, chunk) to record when each warp passes the points
// marked below; by default the marks compile to nothing.
#ifndef BASED_TC_TRACE
#define BASED_TC_TRACE(event, chunk) ((void)0)
#endif

namespace based {

constexpr int kTcChunk = 128;          // tokens per chunk (MMA M)
constexpr int kTcGroup = 128;          // threads of one CUDA-core warp group (4 warps)
constexpr int kTcThreads = 3 * kTcGroup + 32;  // score, feature and epilogue groups, issue warp
constexpr int kSymFP = 160;            // 153 distinct features + 7 zero pads
constexpr int kTcTmemCols = 512;

template <int DV>
struct TcLayout {
  static_assert(DV == 64, "the kernel runs 64 value columns per CTA");
  static constexpr int NA = DV + 16;                       // [V | 1 | 0..] columns
  static constexpr int kTileCols = 96;                     // TMEM columns of O (NA, 32-aligned)
  static constexpr int kVBuf = 3;                          // V stages
  static constexpr int kPhiKBuf = 2;                       // phiK buffers
  // the three V stages share one ones block placed after them; each stage's
  // descriptor reaches it through its own block stride (v_lbo)
  static constexpr int kVStage = 16384;
  static constexpr int kVBytes = (kVBuf + 1) * kVStage;
  static constexpr int kOnes = kVBuf * kVStage;
  static __host__ __device__ constexpr int v_lbo(int s) { return (kVBuf - s) * kVStage; }
  // shared memory (byte offsets from a 1024-aligned base)
  static constexpr int kQ = 0;                             // Q tile  [128 x 16] bf16, K-major
  static constexpr int kK = kQ + 4096;                     // K tile  [128 x 16] bf16, K-major
  static constexpr int kV = kK + 4096;                     // [V | ones] MN-major SW128 stages
  static constexpr int kPhiK = kV + kVBytes;               // phiK [160 x 128] bf16, MN-major
  static constexpr int kSBuf = 2;                          // fp16 state copies
  static constexpr int kSBytes = NA * kSymFP * 2;
  static constexpr int kS = kPhiK + kPhiKBuf * 40960;      // [S|z]^T copies [NA x 160] fp16, K-major
  static constexpr int kY = kS + kSBuf * kSBytes;          // y staging [128 x 64] bf16 SW128
  static constexpr int kBar = kY + 16384;                  // mbarriers + TMEM address
  static constexpr int kBytes = kBar + 256;
  static constexpr size_t kSmem = kBytes + 1024;           // + alignment slack
  // TMEM: the transposed state [S|z]^T (160 feature columns), the score tile U
  // (P is written over it as bf16 pairs), the output accumulator O, and phiQ
  // (80 columns of fp16 pairs)
  static constexpr int kTmS0 = 0;
  static constexpr int kTmU = kSymFP;
  static constexpr int kTmO = kTmU + 128;
  static constexpr int kTmQ = kTmO + kTileCols;
  static_assert(kTmU % 32 == 0 && kTileCols >= NA, "TMEM regions");
  static_assert(kTmQ + kSymFP / 2 <= kTcTmemCols, "TMEM budget");
  static_assert(kY % 1024 == 0, "TMA staging alignment");
  static_assert(kSmem <= 232448, "shared memory budget");
};

struct TcParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  __nv_bfloat16* out;
  float* state_kv;   // [BH, 273, DV] or null (main pass, last segment)
  float* state_k;    // [BH, 273] or null
  float* partial;    // [BH, n_seg-1, 160, DV+16] fp32 segment partials (n_seg > 1)
  int L;
  int seg_chunks;    // chunks per segment
  int n_seg;         // segments per sequence (1 = no split)
  float eps;
  // A sequence with ld_v value columns runs as v_split = ld_v / DV independent
  // CTAs (blocks bh * v_split + h), each on value columns [h DV, h DV + DV): the
  // denominator does not depend on v, so every slice is exact on its own.  v, out
  // and state_kv have ld_v columns; q, k and state_k are per sequence.
  int v_split;
  int ld_v;
};

// A bounded wait gave up: record the timeout and tell the other groups to stop.
__device__ __noinline__ void tc_fail(volatile int* abort_flag) {
  record_device_error(BASED_ERR_TIMEOUT);
  *abort_flag = 1;
}

// Power-of-two scale applied to the fp16 state copy (and to P) for the chunk
// ending at t_end, keeping every state entry (|z_0| <= t) below 2^15.
__device__ __forceinline__ float tc_chunk_scale(long long t_end) {
  int e = 0;
  while (t_end > (32768ll << e)) ++e;
  return __int_as_float((127 - e) << 23);
}

// Row(s) of the 273-row layout a kernel feature f maps to, and the factor.
// Returns the number of rows (0 for padding).
__device__ __forceinline__ int tc_feature_rows(int f, int* r0, int* r1, float* scale) {
  *scale = 1.0f;
  if (f == 0) { *r0 = 0; return 1; }
  if (f < 8) return 0;
  if (f < 24) { *r0 = 1 + (f - 8); return 1; }
  if (f < 40) { const int i = f - 24; *r0 = 17 + 17 * i; return 1; }
  int i, j;
  if (f < 152) {
    const int d = 1 + (f - 40) / 16;
    i = (f - 40) % 16;
    j = (i + d) & 15;
  } else {
    i = f - 152;
    j = i + 8;
  }
  *r0 = 17 + 16 * i + j;
  *r1 = 17 + 16 * j + i;
  *scale = 0.70710678118654752f;
  return 2;
}

// Packed 2-wide arithmetic for the feature build (fp16 for phiQ, bf16 for phiK).
struct H2Ops {
  static __device__ __forceinline__ __half2 mul(__half2 a, __half2 b) { return __hmul2(a, b); }
  static __device__ __forceinline__ __nv_bfloat162 mul(__nv_bfloat162 a, __nv_bfloat162 b) {
    return __hmul2(a, b);
  }
  static __device__ __forceinline__ __half2 shift(__half2 a, __half2 b) {
    return __halves2half2(__high2half(a), __low2half(b));
  }
  static __device__ __forceinline__ __nv_bfloat162 shift(__nv_bfloat162 a, __nv_bfloat162 b) {
    return __halves2bfloat162(__high2bfloat16(a), __low2bfloat16(b));
  }
};

template <typename T2>
__device__ __forceinline__ uint32_t as_u32(T2 v) {
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <typename T2> __device__ __forceinline__ T2 pack2(float a, float b);
template <> __device__ __forceinline__ __half2 pack2<__half2>(float a, float b) {
  return __floats2half2_rn(a, b);
}
template <> __device__ __forceinline__ __nv_bfloat162 pack2<__nv_bfloat162>(float a, float b) {
  return __floats2bfloat162_rn(a, b);
}

// Two fp32 values as one packed pair, and c0 + u (c1 + c2 u) for a pair of u
// with two packed fp32 FMAs (each lane of fma.rn.f32x2 rounds like fmaf).
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void poly2(float u0, float u1, uint64_t c0, uint64_t c1, uint64_t c2,
                                      float* w0, float* w1) {
  const uint64_t u = f32x2(u0, u1);
  uint64_t t, w;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(t) : "l"(u), "l"(c2), "l"(c1));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(w) : "l"(u), "l"(t), "l"(c0));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(*w0), "=f"(*w1) : "l"(w));
}

// Feature chunk ch (8 features) of one token from its packed pairs X[8] (x/2),
// the shifted pairs Y[8], and its raw bf16 input pairs (the diagonal features are
// formed in fp32 and rounded once).  ch must be a compile-time constant.
template <typename T2>
__device__ __forceinline__ uint4 tc_feature_chunk(const T2* X, const T2* Y,
                                                  const __nv_bfloat162* raw, int ch) {
  T2 v[4];
  if (ch == 0) {
    v[0] = pack2<T2>(1.0f, 0.0f);
    v[1] = v[2] = v[3] = pack2<T2>(0.0f, 0.0f);
  } else if (ch <= 2) {
    const int m0 = (ch - 1) * 4;
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = X[m0 + e];
  } else if (ch <= 4) {
    const int m0 = (ch - 3) * 4;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = __bfloat1622float2(raw[m0 + e]);  // x_i^2 / (4 sqrt 2)
      v[e] = pack2<T2>(x.x * x.x * 0.17677669529663687f, x.y * x.y * 0.17677669529663687f);
    }
  } else if (ch <= 18) {
    const int d = 1 + (ch - 5) / 2, m0 = ((ch - 5) & 1) * 4;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int m = m0 + e;
      v[e] = (d & 1) ? H2Ops::mul(X[m], Y[(m + (d - 1) / 2) & 7])
                     : H2Ops::mul(X[m], X[(m + d / 2) & 7]);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = H2Ops::mul(X[e], X[e + 4]);
  }
  return make_uint4(as_u32(v[0]), as_u32(v[1]), as_u32(v[2]), as_u32(v[3]));
}

template <int DV, bool kStateOnly>
__global__ void __launch_bounds__(kTcThreads, 1)
    linattn_tc_kernel(const __grid_constant__ CUtensorMap vmap,
                      const __grid_constant__ CUtensorMap ymap, const TcParams p) {
  using Lay = TcLayout<DV>;
  constexpr int NA = Lay::NA;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::kBar);
  uint64_t* bar_tma = bars + 16;     // [kVBuf] V stage landed
  uint64_t* bar_qk = bars + 2;       // Q/K tiles and phiK written (group F)
  uint64_t* bar_go = bars + 14;      // phiQ of chunk c written (group F); O, the state and its
                                     // fp16 copy of chunk c-1 read and written (group E)
  uint64_t* bar_fin = bars + 15;     // every MMA of this CTA complete (commit)
  uint64_t* bar_u = bars + 3;        // #1 done (commit)
  uint64_t* bar_p = bars + 4;        // P written (group A)
  uint64_t* bar_m25 = bars + 5;      // #5 and #2 done (commit): feature buffers free
  uint64_t* bar_o = bars + 6;        // every MMA of the chunk done (commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 9);
  uint64_t* bar_yfree = bars + 10;   // y staging tile free again (TMA store read it)
  uint64_t* bar_yfull = bars + 11;   // y staging tile written (group E)
  uint64_t* bar_m5 = bars + 12;      // #5 done (commit): the state can be read
  uint64_t* bar_done = bars + 19;    // [2] state-only pass, d_v = 64: #5 of the chunk that
                                     // used phiK buffer b complete (commit)
  constexpr int kThreads = kTcThreads;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3;
  const int L = p.L;
  const int n_chunks = (L + kTcChunk - 1) / kTcChunk;
  const int segs_here = kStateOnly ? p.n_seg - 1 : p.n_seg;
  const int bh = blockIdx.x / segs_here;  // the CTA's (sequence, column slice)
  const int seg = blockIdx.x - bh * segs_here;
  const int bh_seq = bh / p.v_split;        // the sequence
  const int col0 = (bh - bh_seq * p.v_split) * DV;
  const int c_begin = seg * p.seg_chunks;
  const int c_end = min(c_begin + p.seg_chunks, n_chunks);
  const bool has_init = !kStateOnly && seg > 0;

  if (tid == 0) {
    for (int sidx = 0; sidx < Lay::kVBuf; ++sidx) umma::mbar_init(bar_tma + sidx, 1);
    umma::mbar_init(bar_qk, kTcGroup);
    umma::mbar_init(bar_go, 2 * kTcGroup);
    umma::mbar_init(bar_fin, 1);
    umma::mbar_init(bar_u, 1);
    umma::mbar_init(bar_p, kTcGroup);
    umma::mbar_init(bar_m25, 1);
    umma::mbar_init(bar_o, 1);
    umma::mbar_init(bar_yfree, 1);
    umma::mbar_init(bar_yfull, kTcGroup);
    umma::mbar_init(bar_m5, 1);
    umma::mbar_init(bar_done, 1);
    umma::mbar_init(bar_done + 1, 1);
    *abort_flag = 0;
    umma::fence_mbar_init();
    umma::tma_prefetch_desc(&vmap);
  }
  if (warp == 0) {
    umma::tmem_alloc(tmem_slot, kTcTmemCols);
    umma::tmem_relinquish();
  }
  // the ones block of the V stages: column DV of the augmented V is 1 for every token
  for (int i = tid; i < Lay::kVStage / 16; i += kThreads)
    reinterpret_cast<uint4*>(sm + Lay::kV + Lay::kOnes)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  if (tid < kTcChunk)
    *reinterpret_cast<__nv_bfloat16*>(sm + Lay::kV + Lay::kOnes +
                                      umma::off_mnmajor_sw128(0, tid, kTcChunk)) =
        __float2bfloat16(1.0f);
  // rows DV..NA-1 of the transposed fp16 state copies: row DV (z) is rewritten
  // for every chunk, the rows after it stay zero
  for (int b = 0; b < Lay::kSBuf; ++b)
    for (int i = tid; i < (NA - DV) * kSymFP * 2 / 16; i += kThreads)
      reinterpret_cast<uint4*>(sm + Lay::kS + b * Lay::kSBytes + DV * kSymFP * 2)[i] =
          make_uint4(0, 0, 0, 0);
  umma::fence_async_smem();
  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  // the set-up above touched no global memory: it overlaps the previous kernel
  umma::grid_dep_wait();
  umma::grid_dep_launch();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_lane = static_cast<uint32_t>(quad * 32) << 16;
  BASED_TC_TRACE(15, 0);
  // (the failure path is a call, so that its code stays out of the hot loops,
  // which share the instruction cache with three other warps per sub-partition)
  auto fail = [&]() { tc_fail(abort_flag); };
  // Export of [S|z]^T in two steps.  export_stage: TMEM -> shared memory as
  // [feature][value column | z] (stride DV + 4) and the map from the 273 output
  // rows to features; run by the 128 threads of one warp group (t = index in
  // the group, TMEM quadrant = warp & 3) once the last #5 is complete and the
  // feature-map buffers are no longer read.  export_store: coalesced rows of the
  // 273-row layout (or of the segment partial) by n threads (u = 0..n-1), after
  // a barrier that orders them behind export_stage.
  constexpr int kStr = DV + 4;  // keeps each feature row 16-byte aligned
  auto export_stage = [&](int t) {
    const bool any_st = has_init || c_begin < c_end;
    float* stage = reinterpret_cast<float*>(sm + Lay::kPhiK);
    int* rowmap = reinterpret_cast<int*>(stage + kSymFP * kStr);  // [273]: 2 f + (1 if / sqrt 2)
    static_assert(Lay::kPhiKBuf * 40960 >= (kSymFP * kStr + kF) * 4, "export staging");
    if (quad < 3) {
      // two TMEM round trips of 80 features each
#pragma unroll 1
      for (int g = 0; g < 2; ++g) {
        float sv[80];
        umma::tmem_ld80(tmem + Lay::kTmS0 + tm_lane + g * 80, sv);
        if (t <= DV) {
#pragma unroll
          for (int i = 0; i < 80; ++i) stage[(g * 80 + i) * kStr + t] = any_st ? sv[i] : 0.0f;
        }
      }
    }
    for (int f = t; f < kSymFP; f += kTcGroup) {
      int r0 = -1, r1 = -1;
      float scale = 1.0f;
      const int nrows = tc_feature_rows(f, &r0, &r1, &scale);
      const int code = 2 * f + (nrows == 2 ? 1 : 0);
      if (nrows >= 1) rowmap[r0] = code;
      if (nrows == 2) rowmap[r1] = code;
    }
  };
  auto export_store = [&](int u, int n) {
    const float* stage = reinterpret_cast<const float*>(sm + Lay::kPhiK);
    const int* rowmap = reinterpret_cast<const int*>(stage + kSymFP * kStr);
    if (kStateOnly) {
      float* part = p.partial + ((size_t)bh * (p.n_seg - 1) + seg) * kSymFP * NA;
      for (int i = u; i < kSymFP * NA; i += n) {
        const int f = i / NA, j = i - f * NA;
        part[i] = j <= DV ? stage[f * kStr + j] : 0.0f;
      }
    } else if (seg == p.n_seg - 1) {
      if (p.state_kv) {
        float* skv = p.state_kv + (size_t)bh_seq * kF * p.ld_v + col0;
#pragma unroll 4
        for (int i = u; i < kF * (DV / 4); i += n) {
          const int r = i / (DV / 4), j = (i - r * (DV / 4)) * 4;
          const int code = rowmap[r];
          const float sc = (code & 1) ? 0.70710678118654752f : 1.0f;
          const float4 v4 = *reinterpret_cast<const float4*>(stage + (code >> 1) * kStr + j);
          *reinterpret_cast<float4*>(skv + (size_t)r * p.ld_v + j) =
              make_float4(v4.x * sc, v4.y * sc, v4.z * sc, v4.w * sc);
        }
      }
      if (p.state_k && col0 == 0) {
        float* sk = p.state_k + (size_t)bh_seq * kF;
        for (int r = u; r < kF; r += n) {
          const int code = rowmap[r];
          sk[r] = stage[(code >> 1) * kStr + DV] * ((code & 1) ? 0.70710678118654752f : 1.0f);
        }
      }
    }
  };
  // Final state of the main pass straight from TMEM: the thread on TMEM lane j
  // (j < DV: value column j; j = DV: z) loads 80 features (half h of the 160)
  // and writes its column of every output row they map to; the 32 lanes of a
  // warp write 32 consecutive floats of a row.  Run by warps of quadrants 0-2
  // of one group per half, once the last #5 is complete.
  auto export_direct = [&](int h) {
    if (quad < 3 && seg == p.n_seg - 1) {
      float sv[80];
      umma::tmem_ld80(tmem + Lay::kTmS0 + tm_lane + h * 80, sv);
      const int j = quad * 32 + lane;
      float* skv = p.state_kv ? p.state_kv + (size_t)bh_seq * kF * p.ld_v + col0 + j : nullptr;
      float* sk = p.state_k && col0 == 0 ? p.state_k + (size_t)bh_seq * kF : nullptr;
      float* dst = j < DV ? skv : (j == DV ? sk : nullptr);
      const int stride = j < DV ? p.ld_v : 1;
      if (dst != nullptr) {
#pragma unroll
        for (int i = 0; i < 80; ++i) {
          int r0 = -1, r1 = -1;
          float scale = 1.0f;
          const int nrows = tc_feature_rows(h * 80 + i, &r0, &r1, &scale);
          const float v = sv[i] * scale;
          if (nrows >= 1) dst[(size_t)r0 * stride] = v;
          if (nrows == 2) dst[(size_t)r1 * stride] = v;
        }
      }
    }
  };
  // the whole export by one warp group (segment partials, empty segments)
  auto export_kst = [&](int t) {
    export_stage(t);
    umma::named_sync(1, kTcGroup);
    export_store(t, kTcGroup);
  };

  // V tile of chunk c into a stage; returns whether a load was issued (the stall
  // test leaves one out)
  auto issue_v = [&](int c, int stage) {
    if (c == c_begin + 1 && stall_test(kStallLinattnV)) return 0u;
    umma::mbar_arrive_expect_tx(bar_tma + stage, DV * kTcChunk * 2);
#pragma unroll
    for (int blk = 0; blk < DV / 64; ++blk)
      umma::tma_load_3d(sm + Lay::kV + stage * Lay::kVStage + blk * 16384, &vmap,
                        bar_tma + stage, col0 + blk * 64, c * kTcChunk, bh_seq);
    return 1u;
  };

  if (warp == 12) {
    // ================= issue warp: lane 0 drives TMA and the tensor cores =================
    if (lane == 0) {
      const uint32_t sQ = umma::smem_u32(sm + Lay::kQ), sK = umma::smem_u32(sm + Lay::kK),
                     sS = umma::smem_u32(sm + Lay::kS), sPhiK = umma::smem_u32(sm + Lay::kPhiK);
      // descriptors are computed once per buffer and stepped along K by adding
      // the start-address increment (16-byte units) to their low word
      const uint64_t d_q = umma::desc_kmajor_none(sQ, 0, 16), d_k = umma::desc_kmajor_none(sK, 0, 16);
      // fp16 state copies, [value column x feature] K-major
      const uint64_t d_s0 = umma::desc_kmajor_none(sS, 0, kSymFP);
      const uint64_t d_s1 = umma::desc_kmajor_none(sS + Lay::kSBytes, 0, kSymFP);
      // V stages (MN-major, 128B swizzle; the block stride reaches the ones block)
      auto v_desc = [&](int st) {
        return umma::smem_desc(umma::smem_u32(sm + Lay::kV + st * Lay::kVStage), Lay::v_lbo(st),
                               1024, umma::kLayoutSW128);
      };
      const uint64_t d_v0 = v_desc(0), d_v1 = v_desc(1), d_v2 = v_desc(2);
      static_assert(Lay::kVBuf == 3, "three V stages");
      // phiK buffers (MN-major, no swizzle)
      const uint64_t d_k0 = umma::desc_mnmajor_none(sPhiK, 0, kTcChunk);
      const uint64_t d_k1 = umma::desc_mnmajor_none(sPhiK + 40960, 0, kTcChunk);
      const uint32_t id_u = umma::idesc_bf16(128, 128, false, false);
      const uint32_t id_o2 = umma::idesc_f16(128, NA, false, false);
      const uint32_t id_o4 = umma::idesc_bf16(128, NA, false, true);
      const uint32_t id_st = umma::idesc_bf16(128, kSymFP, true, true);
      // per stage (bit s): a load in flight, and the parity of the phase it completes
      // (bit masks rather than arrays, which would live in local memory)
      uint32_t inflight = 0, vphase = 0;
      for (int sidx = 0; sidx < Lay::kVBuf && c_begin + sidx < c_end; ++sidx)
        inflight |= issue_v(c_begin + sidx, sidx) << sidx;
      int n_done = 0;  // chunks whose MMAs were all issued and committed
      int stage = 0;   // V stage of chunk c
      // (no abort check per chunk: a group that gave up stops arriving, and the
      // bounded waits below then end this loop too)
      for (int c = c_begin; c < c_end; ++c) {
        const int it = c - c_begin;
        const uint32_t ph = it & 1;
        const uint64_t d_v = stage == 0 ? d_v0 : (stage == 1 ? d_v1 : d_v2);
        const uint64_t d_phik = (it & 1) ? d_k1 : d_k0;
        const bool has_state = has_init || it > 0;
        // the fp16 copy of the state before chunk c (group E's copy number it - 1,
        // or it with a seeded state)
        const uint64_t d_s = ((has_init ? it : it - 1) & 1) ? d_s1 : d_s0;
        BASED_TC_TRACE(10, it);
        if (!umma::mbar_wait(bar_qk, ph)) { fail(); break; }
        BASED_TC_TRACE(0, it);
        umma::tc_fence_after();
        if (!kStateOnly) {
          umma::mma_bf16(tmem + Lay::kTmU, d_q, d_k, id_u, 0);
          umma::mma_commit(bar_u);
        }
        BASED_TC_TRACE(1, it);
        if (!umma::mbar_wait(bar_tma + stage, (vphase >> stage) & 1u)) { fail(); break; }
        BASED_TC_TRACE(2, it);
        inflight &= ~(1u << stage);
        vphase ^= 1u << stage;
        // #5 overwrites the state in TMEM, #2 reads its fp16 copy and overwrites O:
        // group E must have read the previous chunk's state and O and written the
        // copy, and group F this chunk's phiQ (one barrier for all three, which
        // are ready well before #5 comes up)
        if (!kStateOnly && !umma::mbar_wait(bar_go, ph)) { fail(); break; }
        BASED_TC_TRACE(3, it);
        umma::tc_fence_after();
        // #5 [S|z]^T += [V|1]^T phiK: A = the V stage (value columns x tokens,
        // MN-major; the ones block supplies row DV), B = phiK (N = 160 features).
        // K step of 16 tokens: +2048 B (16 rows of 128 B) in the swizzled V tile,
        // +256 B (2 core matrices) in the no-swizzle phiK layout
#pragma unroll
        for (int ks = 0; ks < kTcChunk / 16; ++ks)
          umma::mma_bf16(tmem + Lay::kTmS0, d_v + ks * 128, d_phik + ks * 16, id_st,
                         has_state || ks > 0);
        // the state-only pass releases this chunk's phiK buffer to group F
        umma::mma_commit(kStateOnly ? bar_done + (it & 1) : bar_m5);
        BASED_TC_TRACE(4, it);
        // state-only pass: refill the stage of chunk c-1 (its MMAs are done by
        // now) with chunk c + kVBuf - 1 (in the main pass group E refills a stage
        // once every MMA of its chunk is done)
        if (kStateOnly && it > 0 && c + Lay::kVBuf - 1 < c_end) {
          const int s_prev = stage == 0 ? Lay::kVBuf - 1 : stage - 1;
          if (!umma::mbar_wait(bar_o, (it - 1) & 1)) { fail(); break; }
          BASED_TC_TRACE(11, it);
          inflight |= issue_v(c + Lay::kVBuf - 1, s_prev) << s_prev;
          BASED_TC_TRACE(12, it);
        }
        if (!kStateOnly) {
          if (has_state) {
            BASED_TC_TRACE(5, it);
            // #2 O = phiQ [S|z]_{c-1}: A = phiQ from TMEM, B = the fp16 state copy.
            // K step of 16 features: 8 TMEM columns, +256 B in the copy
#pragma unroll
            for (int ks = 0; ks < kSymFP / 16; ++ks)
              umma::mma_ts(tmem + Lay::kTmO, tmem + Lay::kTmQ + ks * 8, d_s + ks * 16, id_o2,
                           ks > 0);
          }
          umma::mma_commit(bar_m25);
          BASED_TC_TRACE(6, it);
          if (!umma::mbar_wait(bar_p, ph)) { fail(); break; }
          umma::tc_fence_after();
          BASED_TC_TRACE(7, it);
          // #4 O += P [V|1]: A = P from TMEM (bf16 pairs over U), B = the V stage
#pragma unroll
          for (int ks = 0; ks < kTcChunk / 16; ++ks)
            umma::mma_ts(tmem + Lay::kTmO, tmem + Lay::kTmU + ks * 8, d_v + ks * 128, id_o4,
                         has_state || ks > 0);
        }
        umma::mma_commit(bar_o);
        BASED_TC_TRACE(8, it);
        ++n_done;
        stage = stage == Lay::kVBuf - 1 ? 0 : stage + 1;
      }
      // the last chunk's MMAs must be complete before the state is read out
      if (n_done > 0 && !umma::mbar_wait(bar_o, (n_done - 1) & 1)) fail();
      BASED_TC_TRACE(9, 0);
      // and every MMA this thread issued (an aborted chunk may have left some)
      // before the TMEM is released
      umma::mma_commit(bar_fin);
      if (!umma::mbar_wait(bar_fin, 0)) fail();
      // an aborted run may still have V loads in flight: wait for them (bounded)
      for (int sidx = 0; sidx < Lay::kVBuf; ++sidx)
        if ((inflight >> sidx) & 1u) umma::mbar_wait(bar_tma + sidx, (vphase >> sidx) & 1u);
    }
  } else if (warp < 4) {
    // ================= group P: scores of chunk c =================
    const int t = tid;  // token row of the chunk; also the TMEM lane (quadrant = warp)
    for (int c = c_begin; c < c_end && !kStateOnly && !*abort_flag; ++c) {
      const int it = c - c_begin;
      const int t0 = c * kTcChunk;
      // ---- scores: P = mask(1 + u/4 + u^2/32) * sc ------------------------------------
      if (!umma::mbar_wait(bar_u, it & 1)) { fail(); break; }
      BASED_TC_TRACE(0, it);
      umma::tc_fence_after();
      const float sc = tc_chunk_scale((long long)t0 + kTcChunk);
      const float c0 = sc, c1 = 0.25f * sc, c2 = 0.03125f * sc;
      const uint64_t c0x2 = f32x2(c0, c0), c1x2 = f32x2(c1, c1), c2x2 = f32x2(c2, c2);
      // P (bf16 pairs) of key block b (32 keys) goes to U columns [16b, 16b + 16),
      // which this thread has read already (they belong to block b / 2 <= b);
      // one loop body for every block keeps the code small
      // blocks are taken two at a time (one TMEM load of 64 columns) while two
      // remain, so a warp pays at most two load round trips
      const int row = lane + 32 * quad;  // this thread's token within the chunk
#pragma unroll 1
      for (int b = 0; b <= quad; b += 2) {
        const bool two = b + 1 <= quad;  // warp-uniform
        float u[64];
        if (two) umma::tmem_ld64(tmem + Lay::kTmU + tm_lane + 32 * b, u);
        else umma::tmem_ld32(tmem + Lay::kTmU + tm_lane + 32 * b, u);
        const int lim = row - 32 * b;  // keys 32b + j with j > lim lie in the future
        uint32_t pk[32];
        // the causal mask is a no-op below the diagonal (lim >= 63 there): one
        // loop body for every pair keeps this group's code small
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          float w0, w1;
          poly2(u[2 * e], u[2 * e + 1], c0x2, c1x2, c2x2, &w0, &w1);
          if (2 * e > lim) w0 = 0.0f;
          if (2 * e + 1 > lim) w1 = 0.0f;
          pk[e] = as_u32(__floats2bfloat162_rn(w0, w1));
        }
        if (two) umma::tmem_st32_nowait(tmem + Lay::kTmU + tm_lane + 16 * b, pk);
        else umma::tmem_st16_nowait(tmem + Lay::kTmU + tm_lane + 16 * b, pk);
      }
      uint32_t zero[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) zero[e] = 0u;
#pragma unroll 1
      for (int b = quad + 1; b < 4; ++b) umma::tmem_st16_nowait(tmem + Lay::kTmU + tm_lane + 16 * b, zero);
      umma::tmem_wait_st();
      umma::tc_fence_before();
      BASED_TC_TRACE(1, it);
      umma::mbar_arrive(bar_p);
    }
    if constexpr (!kStateOnly) {
      // the final state is exported here, as soon as the last #5 completes,
      // while #2, #4 and the last output still run: this group writes features
      // 0-79, group F (idle by then) features 80-159.  Both groups take the
      // decision together (barrier 2, 256 threads).
      if (c_begin < c_end) {
        BASED_TC_TRACE(2, 0);
        const bool ok = !*abort_flag && umma::mbar_wait(bar_m5, (c_end - 1 - c_begin) & 1);
        if (umma::named_sync_all(2, 2 * kTcGroup, ok)) {
          umma::tc_fence_after();
          BASED_TC_TRACE(3, 0);
          export_direct(0);
          BASED_TC_TRACE(4, 0);
        } else if (!*abort_flag) {
          fail();
        }
      }
    }
  } else if (warp < 8) {
    // ================= group F: feature maps and Q/K tiles of chunk c =================
    const int t = tid - kTcGroup;  // token row of the chunk; also the TMEM lane (quadrant = warp & 3)
    const __nv_bfloat16* q = p.q + (size_t)bh_seq * L * kD;
    const __nv_bfloat16* k = p.k + (size_t)bh_seq * L * kD;
    // q/k rows of this thread's token, loaded three chunks ahead of their use
    // (the loads of cold inputs take a few microseconds under load)
    uint4 qr[2], kr[2], qn[2], kn[2], qm[2], km[2];
    auto load_qk = [&](int c, uint4* qd, uint4* kd) {
      const long long tt = (long long)c * kTcChunk + t;
      if (c < c_end && tt < L) {
        const uint4* kp = reinterpret_cast<const uint4*>(k + tt * kD);
        kd[0] = kp[0]; kd[1] = kp[1];
        if (!kStateOnly) {
          const uint4* qp = reinterpret_cast<const uint4*>(q + tt * kD);
          qd[0] = qp[0]; qd[1] = qp[1];
        } else {
          qd[0] = qd[1] = make_uint4(0, 0, 0, 0);
        }
      } else {
        qd[0] = qd[1] = kd[0] = kd[1] = make_uint4(0, 0, 0, 0);
      }
    };
    // The state-only pass runs a chunk in about 1,000 cycles, less than a load
    // under load takes: its k rows stream through a ring in the (otherwise
    // unused) state-copy buffer by cp.async, kAhead chunks ahead, so no register
    // waits for them early.
    constexpr int kRing = 8, kAhead = 6;
    static_assert(kRing * kTcChunk * 32 <= Lay::kSBuf * Lay::kSBytes, "k-row ring");
    uint8_t* ring = sm + Lay::kS;
    auto ring_fetch = [&](int c) {  // one commit group per call, empty rows zero-filled
      const long long tt = (long long)c * kTcChunk + t;
      const bool in = c < c_end && tt < L;
      uint8_t* dst = ring + ((c - c_begin) % kRing) * (kTcChunk * 32) + t * 32;
      const __nv_bfloat16* src = k + (in ? tt : 0) * kD;
      umma::cp_async16(dst, src, in);
      umma::cp_async16(dst + 16, src + 8, in);
      umma::cp_async_commit();
    };
    if constexpr (kStateOnly) {
      for (int j = 0; j < kAhead; ++j) ring_fetch(c_begin + j);
    } else {
      load_qk(c_begin, qr, kr);
      load_qk(c_begin + 1, qn, kn);
      load_qk(c_begin + 2, qm, km);
    }
    BASED_TC_TRACE(5, 0);
    for (int c = c_begin; c < c_end && !*abort_flag; ++c) {
      const int it = c - c_begin;
      const int t0 = c * kTcChunk;
      const int n = min(kTcChunk, L - t0);
      const bool live = t < n;
      if constexpr (kStateOnly) {  // this chunk's k row (this thread's own copy)
        umma::cp_async_wait<kAhead - 1>();
        const uint4* src = reinterpret_cast<const uint4*>(ring + (it % kRing) * (kTcChunk * 32) + t * 32);
        kr[0] = src[0];
        kr[1] = src[1];
        ring_fetch(c + kAhead);
      }
      const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(qr);
      const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(kr);
      uint8_t* phik = sm + Lay::kPhiK + (it % Lay::kPhiKBuf) * 40960;
      // phiK goes to buffer it % 2, last read by #5 of chunk c-2: complete before
      // #1 of chunk c-1 (main pass, the wait below) or released by the bar_done
      // wait of the previous iteration (state-only pass)
      BASED_TC_TRACE(0, it);

      // the Q/K tiles are rewritten once #1 of the previous chunk has read them
      if (!kStateOnly && it > 0 && !umma::mbar_wait(bar_u, (it - 1) & 1)) { fail(); break; }
      BASED_TC_TRACE(1, it);
      // ---- phiK and Q/K tiles -------------------------------------------------------
      {
        __nv_bfloat162 XK[8], YK[8];
        const __nv_bfloat162 halfk = __floats2bfloat162_rn(0.5f, 0.5f);
#pragma unroll
        for (int m = 0; m < 8; ++m) XK[m] = __hmul2(k2[m], halfk);
#pragma unroll
        for (int m = 0; m < 8; ++m) YK[m] = H2Ops::shift(XK[m], XK[(m + 1) & 7]);
        // rows past the end of the sequence were loaded as zeros, so all their
        // features but the constant one (chunk 0) are zero already
#pragma unroll
        for (int ch = 0; ch < 20; ++ch)
          *reinterpret_cast<uint4*>(phik + (ch * 16 + (t >> 3)) * 128 + (t & 7) * 16) =
              (ch > 0 || live) ? tc_feature_chunk(XK, YK, k2, ch) : make_uint4(0, 0, 0, 0);

        if (!kStateOnly) {
          uint8_t* qrow = sm + Lay::kQ + ((t >> 3) * 2) * 128 + (t & 7) * 16;
          uint8_t* krow = sm + Lay::kK + ((t >> 3) * 2) * 128 + (t & 7) * 16;
          *reinterpret_cast<uint4*>(qrow) = qr[0];
          *reinterpret_cast<uint4*>(qrow + 128) = qr[1];
          *reinterpret_cast<uint4*>(krow) = kr[0];
          *reinterpret_cast<uint4*>(krow + 128) = kr[1];
        }
      }
      umma::fence_async_smem();
      BASED_TC_TRACE(2, it);
      // An arrival for chunk c must follow the completion of the phase of chunk
      // c-1 (arrivals carry no phase, and the four warps run at their own pace),
      // and the issue thread must have seen that phase (else bar_qk could
      // complete two phases before it looks).  The main pass has both through its
      // wait for #1 of chunk c-1.  The state-only pass (d_v = 64) waits for #5 of
      // chunk c-1 (bar_done of its buffer), which also frees that buffer for
      // chunk c+1; bar_done cannot run ahead of this wait (its next phase needs
      // chunk c+1's #5, after this arrival).
      if (kStateOnly && it > 0 &&
          !umma::mbar_wait(bar_done + ((it - 1) & 1), ((it - 1) >> 1) & 1)) {
        fail();
        break;
      }
      umma::mbar_arrive(bar_qk);
      if (!kStateOnly && it > 0 && !umma::mbar_wait(bar_m25, (it - 1) & 1)) {
        fail();
        break;
      }
      BASED_TC_TRACE(3, it);
      // ---- phiQ (TMEM, the A operand of #2) ----------------------------------------------
      if (!kStateOnly) {
        __half2 XQ[8], YQ[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const float2 a = __bfloat1622float2(q2[m]);
          XQ[m] = __floats2half2_rn(0.5f * a.x, 0.5f * a.y);
        }
#pragma unroll
        for (int m = 0; m < 8; ++m) YQ[m] = H2Ops::shift(XQ[m], XQ[(m + 1) & 7]);
        umma::tc_fence_after();
        uint32_t buf[32];
#pragma unroll
        for (int ch = 0; ch < 20; ++ch) {
          const uint4 v = tc_feature_chunk(XQ, YQ, q2, ch);
          const int s4 = (ch * 4) & 31;
          buf[s4] = v.x; buf[s4 + 1] = v.y; buf[s4 + 2] = v.z; buf[s4 + 3] = v.w;
          if (ch == 7 || ch == 15) umma::tmem_st32_nowait(tmem + Lay::kTmQ + tm_lane + (ch - 7) * 4, buf);
          if (ch == 19) umma::tmem_st16_nowait(tmem + Lay::kTmQ + tm_lane + 64, buf);
        }
        umma::tmem_wait_st();
      }
      if constexpr (!kStateOnly) {
        qr[0] = qn[0]; qr[1] = qn[1]; kr[0] = kn[0]; kr[1] = kn[1];
        qn[0] = qm[0]; qn[1] = qm[1]; kn[0] = km[0]; kn[1] = km[1];
        load_qk(c + 3, qm, km);
      }
      if (!kStateOnly) {
        umma::fence_async_smem();
        umma::tc_fence_before();
        BASED_TC_TRACE(4, it);
        umma::mbar_arrive(bar_go);
      }
    }
    // the ring's copies still in flight (rows past the segment) land before exit
    if constexpr (kStateOnly) umma::cp_async_wait<0>();
    if constexpr (!kStateOnly) {
      // second half of the export (group P waits for the last #5 and decides)
      if (c_begin < c_end && umma::named_sync_all(2, 2 * kTcGroup, true)) {
        umma::tc_fence_after();
        export_direct(1);
      }
    }
  } else if (!kStateOnly) {
    // ================= group E: epilogue of chunk c (output, fp16 state copy) =================
    const int t = tid - 2 * kTcGroup;  // TMEM lane of this thread (quadrant = warp - 8)
    // fp16 copy (scaled by sn) of the state row this thread holds, as #2's B operand:
    // row t of [S|z]^T (value column t, or z for t = DV) -> row t of the K-major
    // copy; lanes past DV hold nothing (quadrant 3 skips the loads)
    int kk = 0;  // number of state copies handed off so far (buffer kk % kSBuf)
    auto copy_state = [&](float sn) {
      uint8_t* sbuf = sm + Lay::kS + (kk % Lay::kSBuf) * Lay::kSBytes;
      if (quad == 3) return;
      uint8_t* dst = sbuf + (t >> 3) * (kSymFP * 16) + (t & 7) * 16;
      const uint32_t base = tmem + Lay::kTmS0 + tm_lane;
      auto put8 = [&](const float* sv, int fg) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          pk[e] = as_u32(__floats2half2_rn(sv[2 * e] * sn, sv[2 * e + 1] * sn));
        if (t <= DV) *reinterpret_cast<uint4*>(dst + fg * 128) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      };
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        float sv[80];
        umma::tmem_ld80(base + 80 * h, sv);
#pragma unroll
        for (int g = 0; g < 10; ++g) put8(sv + 8 * g, 10 * h + g);
      }
    };
    if (has_init) {
      // seed the TMEM state of a later segment with the sum of the earlier
      // partials: after linattn_partial_prefix_kernel, partial seg-1 holds it
      const float* part = p.partial + (size_t)bh * (p.n_seg - 1) * kSymFP * NA;
      if (quad < 3) {
        // partials are [feature][value column]; this lane seeds row t of [S|z]^T
        const float* col0 = part + (size_t)(seg - 1) * kSymFP * NA + t;
#pragma unroll 1
        for (int g = 0; g < kSymFP / 32; ++g) {
          float acc[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] = t <= DV ? col0[(size_t)(g * 32 + i) * NA] : 0.0f;
          umma::tmem_st32(tmem + Lay::kTmS0 + tm_lane + g * 32, acc);
        }
      }
      copy_state(tc_chunk_scale((long long)c_begin * kTcChunk + kTcChunk));
      umma::fence_async_smem();
      ++kk;
    }
    // The hand-off of chunk c-1 to #5 and #2 of chunk c (bar_go): before the first
    // chunk it carries the seeded state and its copy, or nothing.
    umma::tc_fence_before();
    umma::mbar_arrive(bar_go);
    // (thread 0) V loads this group issued, per stage: one issued (bit s) and the
    // parity of the phase it completes
    uint32_t v_issued = 0, v_par = 0;
    int vstage = 0;  // V stage of chunk c
    for (int c = c_begin; c < c_end && !*abort_flag; ++c) {
      const int it = c - c_begin;
      const int t0 = c * kTcChunk;
      const float sc = tc_chunk_scale((long long)t0 + kTcChunk);
      if (c + 1 < c_end) {
        // the state after #5 of this chunk, copied while #2 and #4 still run
        if (!umma::mbar_wait(bar_m5, it & 1)) { fail(); break; }
        BASED_TC_TRACE(0, it);
        umma::tc_fence_after();
        copy_state(tc_chunk_scale((long long)t0 + 2 * kTcChunk));
        umma::fence_async_smem();
        BASED_TC_TRACE(1, it);
      }
      if (!umma::mbar_wait(bar_o, it & 1)) { fail(); break; }
      BASED_TC_TRACE(2, it);
      umma::tc_fence_after();
      float o[64], den;
      umma::tmem_ld64_1(tmem + Lay::kTmO + tm_lane, tmem + Lay::kTmO + tm_lane + DV, o, &den);
      // O and the state are in registers and the copy is written: #5 and #2 of
      // the next chunk may go
      umma::tc_fence_before();
      if (c + 1 < c_end) {
        umma::mbar_arrive(bar_go);
        ++kk;
      }
      BASED_TC_TRACE(3, it);
      // every MMA of chunk c is done: its V stage takes chunk c + kVBuf
      if (t == 0 && c + Lay::kVBuf < c_end) {
        const int cn = c + Lay::kVBuf;
        const uint32_t par = static_cast<uint32_t>((cn - c_begin) / Lay::kVBuf) & 1u;
        v_issued |= issue_v(cn, vstage) << vstage;
        v_par = (v_par & ~(1u << vstage)) | (par << vstage);
      }
      vstage = vstage == Lay::kVBuf - 1 ? 0 : vstage + 1;
      // y row t into the swizzled staging tile; one TMA store per chunk
      uint8_t* ybuf = sm + Lay::kY;
      if (t == 0) {  // the store of chunk c-1 has finished reading ybuf
        umma::bulk_wait_read<0>();
        umma::mbar_arrive(bar_yfree);
      }
      if (!umma::mbar_wait(bar_yfree, it & 1)) { fail(); break; }
      const float inv = 1.0f / (den + p.eps * sc);
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          pk[e] = as_u32(__floats2bfloat162_rn(o[ch * 8 + 2 * e] * inv, o[ch * 8 + 2 * e + 1] * inv));
        *reinterpret_cast<uint4*>(ybuf + t * 128 + ((ch ^ (t & 7)) << 4)) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      umma::fence_async_smem();
      BASED_TC_TRACE(4, it);
      umma::mbar_arrive(bar_yfull);
      if (t == 0) {
        if (!umma::mbar_wait(bar_yfull, it & 1)) { fail(); break; }
        umma::tma_store_3d(&ymap, sm + Lay::kY, col0, t0, bh_seq);
        umma::bulk_commit();
      }
    }
    BASED_TC_TRACE(5, 0);
    // the last output store has read its staging tile (its global writes
    // complete with the grid), and an aborted run's V loads have landed (bounded)
    if (t == 0) {
      umma::bulk_wait_read<0>();
      for (int sidx = 0; sidx < Lay::kVBuf; ++sidx)
        if ((v_issued >> sidx) & 1u) umma::mbar_wait(bar_tma + sidx, (v_par >> sidx) & 1u);
    }
    BASED_TC_TRACE(6, 0);
  }

  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  if (!*abort_flag && warp >= 8 && warp < 12) {
    // ---- state out of TMEM (group E lanes): segment partials or the final export ----
    const int t = tid - 2 * kTcGroup;
    // the main pass exported from groups P and F already (right after its last #5)
    if (kStateOnly || c_begin == c_end) export_kst(t);
  }
  umma::tc_fence_before();
  __syncthreads();
  BASED_TC_TRACE(14, 0);
  if (warp == 0) umma::tmem_dealloc(tmem, kTcTmemCols);
}

// In-place running sum over the segment partials of each sequence (between
// the state-only pass and the main pass): partial g becomes the sum of
// partials 0..g, the state a segment g+1 starts from.  partial is
// [n_seq][n_part][elems] fp32, elems a multiple of 4; one thread per float4
// column of one sequence.
__global__ void __launch_bounds__(256) linattn_partial_prefix_kernel(float* partial, int n_seq,
                                                                     int n_part, int elems) {
  umma::grid_dep_wait();
  umma::grid_dep_launch();
  const long long cols = (long long)elems / 4;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)n_seq * cols) return;
  const long long sq = i / cols, c = i - sq * cols;
  float4* p4 = reinterpret_cast<float4*>(partial) + sq * n_part * cols + c;
  float4 acc = p4[0];
  for (int g = 1; g < n_part; ++g) {
    const float4 v = p4[(long long)g * cols];
    acc = make_float4(acc.x + v.x, acc.y + v.y, acc.z + v.z, acc.w + v.w);
    p4[(long long)g * cols] = acc;
  }
}

}  // namespace based
