// proj_tc.cuh -- input projections of a Based layer on the sm_100a tensor cores.
//
// Y = X W^T for X [M, Kd] (M = B*L tokens, row-major) and W [N, Kd] (one output
// feature per row), bf16 in, fp32 accumulation in TMEM, with one of two epilogues:
//
//  * kProjHeads -- the per-head projection that feeds the attention layers
//    ("Базированная модель, часть 2", the paragraph on the size of the hidden
//    state: the KV and K states are made smaller by projections of the input):
//    column n = h*D + d of token m = b*L + t goes to y[b][h][t][d] (bf16).
//  * kBaseConv -- the BaseConv block ("Базированная модель, часть 1", section
//    "Кто виноват?": y = linear(x) (.) conv(h, x)): N = Kd = D channels, and
//    y[m][c] = (Y[m][c] + bias[c]) * sum_{j <= min(K-1, t)} h[c][j] x[m-j][c],
//    the causal per-channel convolution read straight from x.
//
// One CTA per 128 x 256 output tile.  Warp 0 (one thread) streams 64-wide K
// blocks of X and W by TMA through a four-stage ring (128B swizzle, K-major),
// warp 1 (one thread) issues four M=128/N=256/K=16 MMAs per block into TMEM,
// and warps 2-5 (one per TMEM lane quadrant) run the epilogue: 32 columns at a
// time from TMEM, the epilogue arithmetic in fp32, 16-byte global stores.
#pragma once

#include "common.cuh"
#include "umma.cuh"

namespace based {

constexpr int kPjM = 128;       // rows (tokens) per tile
constexpr int kPjN = 256;       // columns per tile
constexpr int kPjK = 64;        // K block per stage (one 128-byte swizzle atom)
constexpr int kPjStages = 4;
constexpr int kPjThreads = 192;
constexpr int kPjMaxTaps = 8;

enum ProjMode { kProjHeads = 0, kBaseConv = 1 };

struct PjLayout {
  static constexpr int kA = 0;                                    // [stage] A [128 x 64] bf16
  static constexpr int kB = kPjStages * kPjM * kPjK * 2;          // [stage] B [256 x 64] bf16
  static constexpr int kTaps = kB + kPjStages * kPjN * kPjK * 2;  // h tile [256][taps] fp32
  static constexpr int kBias = kTaps + kPjN * kPjMaxTaps * 4;     // bias tile [256] fp32
  static constexpr int kBar = kBias + kPjN * 4;
  static constexpr int kBytes = kBar + 128;
  static constexpr size_t kSmem = kBytes + 1024;
  static_assert(kB % 1024 == 0, "swizzled tiles are 1024-byte aligned");
  static_assert(kSmem <= 232448, "shared memory budget");
};

struct ProjParams {
  const __nv_bfloat16* x;  // kBaseConv: the layer input, read again by the convolution
  __nv_bfloat16* y;
  const float* bias;       // kBaseConv: [N]
  const float* taps;       // kBaseConv: [N][K]
  int M, N, Kd;
  int L;                   // tokens per sequence
  int H, D;                // kProjHeads: heads and features per head (N = H * D)
  int K;                   // kBaseConv: filter taps
};

template <int Mode>
__global__ void __launch_bounds__(kPjThreads, 1)
    proj_tc_kernel(const __grid_constant__ CUtensorMap xmap,
                   const __grid_constant__ CUtensorMap wmap, const ProjParams p) {
  using Lay = PjLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::kBar);
  uint64_t* bar_full = bars;                // [stage] A and B landed
  uint64_t* bar_empty = bars + kPjStages;   // [stage] read by the MMAs (commit)
  uint64_t* bar_done = bars + 2 * kPjStages;  // accumulator complete (commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kPjStages + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * kPjStages + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * kPjM, n0 = blockIdx.y * kPjN;
  const int nkb = p.Kd / kPjK;

  if (tid == 0) {
    for (int s = 0; s < kPjStages; ++s) {
      umma::mbar_init(bar_full + s, 1);
      umma::mbar_init(bar_empty + s, 1);
    }
    umma::mbar_init(bar_done, 1);
    *abort_flag = 0;
    umma::fence_mbar_init();
  }
  if (warp == 1) {
    umma::tmem_alloc(tmem_slot, kPjN);
    umma::tmem_relinquish();
  }
  if (Mode == kBaseConv) {
    // the tile's filter taps and bias, read by every epilogue thread
    float* taps = reinterpret_cast<float*>(sm + Lay::kTaps);
    float* bias = reinterpret_cast<float*>(sm + Lay::kBias);
    for (int i = tid; i < kPjN * p.K; i += kPjThreads) taps[i] = p.taps[(size_t)n0 * p.K + i];
    for (int i = tid; i < kPjN; i += kPjThreads) bias[i] = p.bias[n0 + i];
  }
  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto fail = [&]() {
    record_device_error(BASED_ERR_TIMEOUT);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ================= producer =================
    if (lane == 0) {
      constexpr uint32_t bytes = (kPjM + kPjN) * kPjK * 2;
      int issued = 0;
      for (int kb = 0; kb < nkb && !*abort_flag; ++kb) {
        const int s = kb % kPjStages;
        if (kb >= kPjStages &&
            !umma::mbar_wait(bar_empty + s, ((kb - kPjStages) / kPjStages) & 1)) {
          fail();
          break;
        }
        umma::mbar_arrive_expect_tx(bar_full + s, bytes);
        umma::tma_load_3d(sm + Lay::kA + s * (kPjM * kPjK * 2), &xmap, bar_full + s, kb * kPjK, m0, 0);
        umma::tma_load_3d(sm + Lay::kB + s * (kPjN * kPjK * 2), &wmap, bar_full + s, kb * kPjK, n0, 0);
        issued = kb + 1;
      }
      // loads no MMA consumed (after an abort) must land before the CTA exits
      if (*abort_flag)
        for (int kb = issued - kPjStages > 0 ? issued - kPjStages : 0; kb < issued; ++kb)
          umma::mbar_wait(bar_full + kb % kPjStages, (kb / kPjStages) & 1);
    }
  } else if (warp == 1) {
    // ================= MMA issue =================
    if (lane == 0) {
      const uint32_t id = umma::idesc_bf16(kPjM, kPjN, false, false);
      for (int kb = 0; kb < nkb && !*abort_flag; ++kb) {
        const int s = kb % kPjStages;
        if (!umma::mbar_wait(bar_full + s, (kb / kPjStages) & 1)) { fail(); break; }
        umma::tc_fence_after();
        const uint32_t sa = umma::smem_u32(sm + Lay::kA + s * (kPjM * kPjK * 2));
        const uint32_t sb = umma::smem_u32(sm + Lay::kB + s * (kPjN * kPjK * 2));
#pragma unroll
        for (int k0 = 0; k0 < kPjK; k0 += 16)
          umma::mma_bf16(tmem, umma::desc_kmajor_sw128(sa, k0, kPjM),
                         umma::desc_kmajor_sw128(sb, k0, kPjN), id, (kb | k0) != 0);
        umma::mma_commit(bar_empty + s);
      }
      // the accumulator (or, after an abort, every MMA issued) is complete
      umma::mma_commit(bar_done);
    }
  } else {
    // ================= epilogue: warps 2-5, TMEM lane quadrant = warp mod 4 =================
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int m = m0 + r;
    const bool ok = umma::mbar_wait(bar_done, 0);
    if (!ok) fail();
    umma::tc_fence_after();
    const int b = m / p.L, t = m - (m / p.L) * p.L;
    const float* taps = reinterpret_cast<const float*>(sm + Lay::kTaps);
    const float* bias = reinterpret_cast<const float*>(sm + Lay::kBias);
#pragma unroll 1
    for (int c32 = 0; c32 < kPjN / 32; ++c32) {
      float acc[32];
      umma::tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + c32 * 32, acc);
      if (!ok || *abort_flag || m >= p.M) continue;
#pragma unroll
      for (int g = 0; g < 4; ++g) {  // 8 columns = one 16-byte store
        const int n = n0 + c32 * 32 + g * 8;
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = acc[g * 8 + e];
        size_t dst;
        if (Mode == kProjHeads) {
          const int hh = n / p.D, d = n - hh * p.D;
          dst = (((size_t)b * p.H + hh) * p.L + t) * p.D + d;
        } else {
          const int cl = c32 * 32 + g * 8;  // column within the tile
          float conv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) conv[e] = 0.0f;
          for (int j = 0; j < p.K && j <= t; ++j) {
            const uint4 xv = *reinterpret_cast<const uint4*>(p.x + (size_t)(m - j) * p.N + n);
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[e]));
              conv[2 * e] = fmaf(taps[(cl + 2 * e) * p.K + j], f.x, conv[2 * e]);
              conv[2 * e + 1] = fmaf(taps[(cl + 2 * e + 1) * p.K + j], f.y, conv[2 * e + 1]);
            }
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = (v[e] + bias[cl + e]) * conv[e];
          dst = (size_t)m * p.N + n;
        }
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
          pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        *reinterpret_cast<uint4*>(p.y + dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
  }
  umma::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // after an abort the MMA thread may still have MMAs in flight
    if (lane == 0 && *abort_flag) umma::mbar_wait(bar_done, 0);
    __syncwarp();
    umma::tmem_dealloc(tmem, kPjN);
  }
}

}  // namespace based
