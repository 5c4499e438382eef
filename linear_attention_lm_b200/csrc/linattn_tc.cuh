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
//  * phi(q).phi(k) only needs the 153 distinct features [1, x_i/2,
//    x_i x_j c_ij (i <= j)] with c_ii = 1/(4 sqrt 2), c_ij = 1/4 (i < j): the
//    full map lists every off-diagonal product twice with weight 1/(4 sqrt 2).
//    The state is kept over these 153 features and expanded to the 273-row
//    layout (off-diagonal rows = value / sqrt 2, duplicated) only on export.
// The ones column appended to V makes the normaliser z and both parts of the
// denominator come out of the same MMAs, with the same rounded operands as the
// numerator.
//
// Operand precision: Q, K, V, P and phiK are bf16; phiQ and the per-chunk copy
// of the state used by #2 are fp16 (bf16 inputs are exact in fp16; the state
// copy is scaled by a power of two so it stays in fp16 range for any L, and P is
// scaled by the same power so the ratio is unchanged).  All accumulation is fp32
// in TMEM; the master state never leaves TMEM until the export.
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

namespace based {

constexpr int kTcChunk = 128;          // tokens per chunk (MMA M)
constexpr int kTcThreads = 128;        // 4 warps, one TMEM lane quadrant each
constexpr int kSymF = 153;             // distinct Taylor features
constexpr int kSymFP = 160;            // padded to the MMA K granularity (16)
constexpr int kTcTmemCols = 512;

// Symmetric-feature index (>= 17) -> (i, j) of the quadratic block, i <= j.
__host__ __device__ constexpr int sym_pair_i(int p) {
  int i = 0;
  while (p >= 16 - i) { p -= 16 - i; ++i; }
  return i;
}
__host__ __device__ constexpr int sym_pair_j(int p) {
  int i = 0;
  while (p >= 16 - i) { p -= 16 - i; ++i; }
  return i + p;
}

template <int DV>
struct TcLayout {
  static constexpr int NA = DV + 16;                       // [V | 1 | 0..] columns
  static constexpr int kTileCols = (NA + 31) / 32 * 32;    // TMEM columns per state tile
  // shared memory (byte offsets from a 1024-aligned base)
  static constexpr int kQ = 0;                             // Q tile  [128 x 16] bf16, K-major
  static constexpr int kK = kQ + 4096;                     // K tile  [128 x 16] bf16, K-major
  static constexpr int kV = kK + 4096;                     // [V | ones] MN-major SW128 blocks
  static constexpr int kVBlocks = DV / 64 + 1;
  static constexpr int kPhiK = kV + kVBlocks * 16384;      // phiK [160 x 128] bf16, MN-major
  static constexpr int kP = kPhiK + 40960;                 // P [128 x 128] bf16, K-major
  static constexpr int kPhiQ = kP + 32768;                 // phiQ [128 x 160] fp16, K-major
  static constexpr int kS = kPhiQ + 40960;                 // [S|z] copy [160 x NA] fp16, MN-major
  static constexpr int kBar = kS + NA * kSymFP * 2;        // mbarriers + TMEM address
  static constexpr int kBytes = kBar + 64;
  static constexpr size_t kSmem = kBytes + 1024;           // + alignment slack
  // TMEM columns: [S|z] tiles (two 128-feature tiles) then the U / O accumulator
  static constexpr int kTmS = 0;
  static constexpr int kTmO = 2 * kTileCols;
  static_assert(kTmO + 160 <= kTcTmemCols, "TMEM budget");
  // #5 reads 32 feature groups past phiK (the second tile's unused rows); keep
  // that window inside the allocation.
  static_assert(kPhiK + 65536 <= kBytes, "phiK over-read window");
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
};

// Power-of-two scale applied to the fp16 state copy (and to P) for the chunk
// ending at t_end, keeping every state entry (|z_0| <= t) below 2^15.
__device__ __forceinline__ float tc_chunk_scale(long long t_end) {
  int e = 0;
  while (t_end > (32768ll << e)) ++e;
  return __int_as_float((127 - e) << 23);
}

template <int DV, bool kStateOnly>
__global__ void __launch_bounds__(kTcThreads, 1)
    linattn_tc_kernel(const __grid_constant__ CUtensorMap vmap, const TcParams p) {
  using Lay = TcLayout<DV>;
  constexpr int NA = Lay::NA;
  constexpr int NG = (NA + 31) / 32;  // 32-column groups of a state tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + Lay::kBar);
  uint64_t* bar_u = bar_tma + 1;
  uint64_t* bar_o = bar_tma + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_tma + 3);
  int* abort_flag = reinterpret_cast<int*>(bar_tma + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int L = p.L;
  const int n_chunks = (L + kTcChunk - 1) / kTcChunk;
  const int segs_here = kStateOnly ? p.n_seg - 1 : p.n_seg;
  const int bh = blockIdx.x / segs_here;
  const int seg = blockIdx.x - bh * segs_here;
  const int c_begin = seg * p.seg_chunks;
  const int c_end = min(c_begin + p.seg_chunks, n_chunks);
  const bool has_init = !kStateOnly && seg > 0;
  const __nv_bfloat16* q = p.q + (size_t)bh * L * kD;
  const __nv_bfloat16* k = p.k + (size_t)bh * L * kD;
  __nv_bfloat16* out = kStateOnly ? nullptr : p.out + (size_t)bh * L * DV;

  if (tid == 0) {
    umma::mbar_init(bar_tma, 1);
    umma::mbar_init(bar_u, 1);
    umma::mbar_init(bar_o, 1);
    *abort_flag = 0;
    umma::fence_mbar_init();
    umma::tma_prefetch_desc(&vmap);
  }
  if (warp == 0) {
    umma::tmem_alloc(tmem_slot, kTcTmemCols);
    umma::tmem_relinquish();
  }
  // ones block of [V | 1]: column DV of the augmented V is 1 for every token
  {
    uint8_t* ones = sm + Lay::kV + (DV / 64) * 16384;
    for (int i = tid; i < 16384 / 16; i += kTcThreads)
      reinterpret_cast<uint4*>(ones)[i] = make_uint4(0, 0, 0, 0);
    __syncthreads();
    *reinterpret_cast<__nv_bfloat16*>(ones + umma::off_mnmajor_sw128(0, tid, kTcChunk)) =
        __float2bfloat16(1.0f);
  }
  umma::fence_async_smem();
  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_lane = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t sQ = umma::smem_u32(sm + Lay::kQ), sK = umma::smem_u32(sm + Lay::kK),
                 sV = umma::smem_u32(sm + Lay::kV), sPhiK = umma::smem_u32(sm + Lay::kPhiK),
                 sP = umma::smem_u32(sm + Lay::kP), sPhiQ = umma::smem_u32(sm + Lay::kPhiQ),
                 sS = umma::smem_u32(sm + Lay::kS);
  constexpr uint32_t kVBytes = DV * kTcChunk * 2;
  // state tiles: tile 0 lanes 0..127 = features 0..127 (all warps); tile 1
  // lanes 0..31 = features 128..159 (warp 0 only)
  const int n_tiles_here = warp == 0 ? 2 : 1;

  auto issue_v = [&](int c) {
    umma::mbar_arrive_expect_tx(bar_tma, kVBytes);
#pragma unroll
    for (int b = 0; b < DV / 64; ++b)
      umma::tma_load_3d(sm + Lay::kV + b * 16384, &vmap, bar_tma, b * 64, c * kTcChunk, bh);
  };
  if (tid == 0 && c_begin < c_end) issue_v(c_begin);

  // fp16 copy of the TMEM state, scaled by sn, as the B operand of #2
  auto copy_state = [&](float sn) {
    for (int mt = 0; mt < n_tiles_here; ++mt) {
      const int f = mt * 128 + warp * 32 + lane;
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        float sv[32];
        umma::tmem_ld32(tmem + Lay::kTmS + mt * Lay::kTileCols + tm_lane + g * 32, sv);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int j0 = g * 32 + h * 8;
          if (j0 < NA) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __half2 hv = __floats2half2_rn(sv[h * 8 + 2 * e] * sn, sv[h * 8 + 2 * e + 1] * sn);
              pk[e] = *reinterpret_cast<const uint32_t*>(&hv);
            }
            *reinterpret_cast<uint4*>(sm + Lay::kS + ((j0 >> 3) * 20 + (f >> 3)) * 128 + (f & 7) * 16) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
    }
  };

  // seed the TMEM state of a later segment with the sum of the earlier partials
  if (has_init) {
    const float* part = p.partial + (size_t)bh * (p.n_seg - 1) * kSymFP * NA;
    for (int mt = 0; mt < n_tiles_here; ++mt) {
      const int f = mt * 128 + warp * 32 + lane;
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        float acc[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
        for (int sp = 0; sp < seg; ++sp) {
          const float* row = part + ((size_t)sp * kSymFP + f) * NA + g * 32;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (g * 32 + i < NA) acc[i] += row[i];
        }
        umma::tmem_st32(tmem + Lay::kTmS + mt * Lay::kTileCols + tm_lane + g * 32, acc);
      }
    }
    umma::tc_fence_before();
    __syncthreads();
    umma::tc_fence_after();
    copy_state(tc_chunk_scale((long long)c_begin * kTcChunk + kTcChunk));
  }

  // q/k rows of this thread's token, prefetched one chunk ahead
  uint4 qr[2], kr[2];
  auto load_qk = [&](int c) {
    const long long t = (long long)c * kTcChunk + tid;
    if (c < c_end && t < L) {
      const uint4* kp = reinterpret_cast<const uint4*>(k + t * kD);
      kr[0] = kp[0]; kr[1] = kp[1];
      if (!kStateOnly) {
        const uint4* qp = reinterpret_cast<const uint4*>(q + t * kD);
        qr[0] = qp[0]; qr[1] = qp[1];
      } else {
        qr[0] = qr[1] = make_uint4(0, 0, 0, 0);
      }
    } else {
      qr[0] = qr[1] = kr[0] = kr[1] = make_uint4(0, 0, 0, 0);
    }
  };
  load_qk(c_begin);

  uint32_t ph_tma = 0, ph_u = 0, ph_o = 0;
  bool tma_pending = c_begin < c_end;
  const uint32_t id_u = umma::idesc_bf16(128, 128, false, false);
  const uint32_t id_o2 = umma::idesc_f16(128, NA, false, true);
  const uint32_t id_o4 = umma::idesc_bf16(128, NA, false, true);
  const uint32_t id_s5 = umma::idesc_bf16(128, NA, true, true);

  __syncthreads();
  for (int c = c_begin; c < c_end; ++c) {
    const int t0 = c * kTcChunk;
    const int n = min(kTcChunk, L - t0);
    const bool has_state = has_init || c > c_begin;
    const float sc = tc_chunk_scale((long long)t0 + kTcChunk);
    // ---- (a) Q/K tiles and the feature maps of this thread's token -------------
    {
      const int t = tid;
      if (!kStateOnly) {
        uint8_t* qrow = sm + Lay::kQ + ((t >> 3) * 2) * 128 + (t & 7) * 16;
        uint8_t* krow = sm + Lay::kK + ((t >> 3) * 2) * 128 + (t & 7) * 16;
        *reinterpret_cast<uint4*>(qrow) = qr[0];
        *reinterpret_cast<uint4*>(qrow + 128) = qr[1];
        *reinterpret_cast<uint4*>(krow) = kr[0];
        *reinterpret_cast<uint4*>(krow + 128) = kr[1];
      }
      float xq[16], xk[16];
      const __nv_bfloat162* q2 = reinterpret_cast<const __nv_bfloat162*>(qr);
      const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(kr);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 a = __bfloat1622float2(q2[i]);
        const float2 b = __bfloat1622float2(k2[i]);
        xq[2 * i] = a.x; xq[2 * i + 1] = a.y;
        xk[2 * i] = b.x; xk[2 * i + 1] = b.y;
      }
      const bool live = t < n;
      // features in order: 1, x_i/2 (16), x_i x_j c_ij for i <= j (136), zero pad (7);
      // every index below is a compile-time constant after unrolling
      float fq8[8], fk8[8];
      int slot = 0, ch = 0;
      auto flush = [&]() {
        uint32_t hq[4], bk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __half2 h = __floats2half2_rn(fq8[2 * e], fq8[2 * e + 1]);
          const __nv_bfloat162 b = __floats2bfloat162_rn(live ? fk8[2 * e] : 0.0f,
                                                          live ? fk8[2 * e + 1] : 0.0f);
          hq[e] = *reinterpret_cast<const uint32_t*>(&h);
          bk[e] = *reinterpret_cast<const uint32_t*>(&b);
        }
        if (!kStateOnly)
          *reinterpret_cast<uint4*>(sm + Lay::kPhiQ + ((t >> 3) * 20 + ch) * 128 + (t & 7) * 16) =
              make_uint4(hq[0], hq[1], hq[2], hq[3]);
        *reinterpret_cast<uint4*>(sm + Lay::kPhiK + (ch * 16 + (t >> 3)) * 128 + (t & 7) * 16) =
            make_uint4(bk[0], bk[1], bk[2], bk[3]);
        ++ch;
        slot = 0;
      };
      auto emit = [&](float a, float b) {
        fq8[slot] = a;
        fk8[slot] = b;
        if (++slot == 8) flush();
      };
      emit(1.0f, 1.0f);
#pragma unroll
      for (int i = 0; i < 16; ++i) emit(0.5f * xq[i], 0.5f * xk[i]);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
#pragma unroll
        for (int j = i; j < 16; ++j) {
          const float cw = i == j ? 0.17677669529663687f : 0.25f;
          emit(xq[i] * xq[j] * cw, xk[i] * xk[j] * cw);
        }
      }
#pragma unroll
      for (int f = kSymF; f < kSymFP; ++f) emit(0.0f, 0.0f);
    }
    load_qk(c + 1);
    umma::fence_async_smem();
    umma::tc_fence_before();
    __syncthreads();
    umma::tc_fence_after();
    if (!kStateOnly) {
      // ---- (b) #1: U = Q K^T -------------------------------------------------------
      if (tid == 0) {
        umma::mma_bf16(tmem + Lay::kTmO, umma::desc_kmajor_none(sQ, 0, 16),
                       umma::desc_kmajor_none(sK, 0, 16), id_u, 0);
        umma::mma_commit(bar_u);
      }
      __syncwarp();
      if (!umma::mbar_wait(bar_u, ph_u)) { record_device_error(BASED_ERR_TIMEOUT); *abort_flag = 1; }
      ph_u ^= 1;
      umma::tc_fence_after();
      // ---- (c) scores: P = mask(1 + u/4 + u^2/32) * sc -> smem -----------------------
      {
        const int t = tid;
#pragma unroll
        for (int c32 = 0; c32 < 4; ++c32) {
          float u[32];
          umma::tmem_ld32(tmem + Lay::kTmO + tm_lane + c32 * 32, u);
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int s0 = c32 * 32 + g * 8 + 2 * e;
              const float u0 = u[g * 8 + 2 * e], u1 = u[g * 8 + 2 * e + 1];
              const float w0 = s0 <= t ? fmaf(u0, fmaf(u0, 0.03125f, 0.25f), 1.0f) * sc : 0.0f;
              const float w1 = s0 + 1 <= t ? fmaf(u1, fmaf(u1, 0.03125f, 0.25f), 1.0f) * sc : 0.0f;
              const __nv_bfloat162 b = __floats2bfloat162_rn(w0, w1);
              pk[e] = *reinterpret_cast<const uint32_t*>(&b);
            }
            const int ch = c32 * 4 + g;
            *reinterpret_cast<uint4*>(sm + Lay::kP + ((t >> 3) * 16 + ch) * 128 + (t & 7) * 16) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
      umma::fence_async_smem();
      umma::tc_fence_before();
      __syncthreads();
      umma::tc_fence_after();
      if (*abort_flag) break;
    }
    // ---- (d) #2, #4, #5 ----------------------------------------------------------------
    if (tid == 0) {
      const bool ok = umma::mbar_wait(bar_tma, ph_tma);
      ph_tma ^= 1;
      tma_pending = false;
      if (!ok) {
        record_device_error(BASED_ERR_TIMEOUT);
        *abort_flag = 1;
      } else {
        umma::tc_fence_after();
        if (!kStateOnly) {
          if (has_state) {
#pragma unroll
            for (int k0 = 0; k0 < kSymFP; k0 += 16)
              umma::mma_f16(tmem + Lay::kTmO, umma::desc_kmajor_none(sPhiQ, k0, kSymFP),
                            umma::desc_mnmajor_none(sS, k0, kSymFP), id_o2, k0 > 0);
          }
#pragma unroll
          for (int k0 = 0; k0 < kTcChunk; k0 += 16)
            umma::mma_bf16(tmem + Lay::kTmO, umma::desc_kmajor_none(sP, k0, kTcChunk),
                           umma::desc_mnmajor_sw128(sV, k0, kTcChunk), id_o4,
                           has_state || (k0 > 0));
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int k0 = 0; k0 < kTcChunk; k0 += 16)
            umma::mma_bf16(tmem + Lay::kTmS + mt * Lay::kTileCols,
                           umma::desc_mnmajor_none(sPhiK + mt * 16 * 2048, k0, kTcChunk),
                           umma::desc_mnmajor_sw128(sV, k0, kTcChunk), id_s5,
                           has_state || (k0 > 0));
        umma::mma_commit(bar_o);
      }
    }
    __syncwarp();
    __syncthreads();
    if (*abort_flag) break;
    if (!umma::mbar_wait(bar_o, ph_o)) { record_device_error(BASED_ERR_TIMEOUT); *abort_flag = 1; }
    ph_o ^= 1;
    umma::tc_fence_after();
    if (tid == 0 && c + 1 < c_end && !*abort_flag) {
      issue_v(c + 1);
      tma_pending = true;
    }
    // ---- (e) outputs and the fp16 state copy for the next chunk --------------------
    if (!kStateOnly) {
      const int t = tid;
      float o[NG * 32];
#pragma unroll
      for (int g = 0; g < NG; ++g) umma::tmem_ld32(tmem + Lay::kTmO + tm_lane + g * 32, o + g * 32);
      if (t < n) {
        const float inv = 1.0f / (o[DV] + p.eps * sc);
        uint4* dst = reinterpret_cast<uint4*>(out + (size_t)(t0 + t) * DV);
#pragma unroll
        for (int ch = 0; ch < DV / 8; ++ch) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 b =
                __floats2bfloat162_rn(o[ch * 8 + 2 * e] * inv, o[ch * 8 + 2 * e + 1] * inv);
            pk[e] = *reinterpret_cast<const uint32_t*>(&b);
          }
          dst[ch] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      if (c + 1 < c_end) copy_state(tc_chunk_scale((long long)t0 + 2 * kTcChunk));
    }
    umma::fence_async_smem();
    umma::tc_fence_before();
    __syncthreads();
    umma::tc_fence_after();
    if (*abort_flag) break;
  }

  if (!*abort_flag) {
    if (kStateOnly) {
      // this segment's partial state, 160 symmetric rows x NA columns, fp32
      float* part = p.partial + ((size_t)bh * (p.n_seg - 1) + seg) * kSymFP * NA;
      for (int mt = 0; mt < n_tiles_here; ++mt) {
        const int f = mt * 128 + warp * 32 + lane;
#pragma unroll
        for (int g = 0; g < NG; ++g) {
          float s[32];
          umma::tmem_ld32(tmem + Lay::kTmS + mt * Lay::kTileCols + tm_lane + g * 32, s);
          float* row = part + (size_t)f * NA + g * 32;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (g * 32 + i < NA) row[i] = c_begin < c_end ? s[i] : 0.0f;
        }
      }
    } else if (seg == p.n_seg - 1 && (p.state_kv || p.state_k)) {
      // final state export: 153 symmetric rows -> 273-row layout
      float* skv = p.state_kv ? p.state_kv + (size_t)bh * kF * DV : nullptr;
      float* sk = p.state_k ? p.state_k + (size_t)bh * kF : nullptr;
      const bool any = has_init || c_begin < c_end;
      for (int mt = 0; mt < n_tiles_here; ++mt) {
        const int f = mt * 128 + warp * 32 + lane;
        float s[NG * 32];
#pragma unroll
        for (int g = 0; g < NG; ++g)
          umma::tmem_ld32(tmem + Lay::kTmS + mt * Lay::kTileCols + tm_lane + g * 32, s + g * 32);
        if (!any) {
#pragma unroll
          for (int i = 0; i < NG * 32; ++i) s[i] = 0.0f;
        }
        if (f >= kSymF) continue;
        int r0, r1 = -1;
        float scale = 1.0f;
        if (f <= 16) {
          r0 = f;
        } else {
          const int i = sym_pair_i(f - 17), j = sym_pair_j(f - 17);
          r0 = 17 + 16 * i + j;
          if (i != j) { r1 = 17 + 16 * j + i; scale = 0.70710678118654752f; }
        }
        for (int r = 0; r < 2; ++r) {
          const int row = r == 0 ? r0 : r1;
          if (row < 0) continue;
          if (skv) {
            float4* dst = reinterpret_cast<float4*>(skv + (size_t)row * DV);
#pragma unroll
            for (int j = 0; j < DV / 4; ++j)
              dst[j] = make_float4(s[4 * j] * scale, s[4 * j + 1] * scale, s[4 * j + 2] * scale,
                                   s[4 * j + 3] * scale);
          }
          if (sk) sk[row] = s[DV] * scale;
        }
      }
    }
  }
  // an aborted run may still have a V load in flight: wait for it (bounded)
  if (tid == 0 && tma_pending && *abort_flag) umma::mbar_wait(bar_tma, ph_tma);
  umma::tc_fence_before();
  __syncthreads();
  if (warp == 0) umma::tmem_dealloc(tmem, kTcTmemCols);
}

}  // namespace based
