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
//    y[m][c] = (Y[m][c] + bias[c]) * sum_{j <= min(K-1, t)} h[c][j] x[m-j][c].
//
// Persistent: one CTA per SM walks the 128 x 256 output tiles (tiles sharing an
// X row block are adjacent, so X is read from DRAM about once).  Warp 0 (one
// thread) streams 64-wide K blocks of X and W by TMA through a ring of stages
// (128B swizzle, K-major); warp 1 (one thread) issues four M=128/N=256/K=16 MMAs
// per block into one of two TMEM accumulators, so the epilogue of tile k
// overlaps the main loop of tile k+1; warps 2-5 (one per TMEM lane quadrant)
// run the epilogue.  For BaseConv the producer also loads the tile's input rows
// [m0-8, m0+128) x [n0, n0+256) (the convolution's reach) into shared memory,
// once the previous tile's epilogue has released them.
#pragma once

#include "common.cuh"
#include "umma.cuh"

namespace based {

constexpr int kPjM = 128;       // rows (tokens) per tile
constexpr int kPjN = 256;       // columns per tile
constexpr int kPjK = 64;        // K block per stage (one 128-byte swizzle atom)
constexpr int kPjThreads = 192;
constexpr int kPjMaxTaps = 8;
constexpr int kPjHaloRows = kPjM + kPjMaxTaps;  // rows [m0 - 8, m0 + 128)

enum ProjMode { kProjHeads = 0, kBaseConv = 1 };

template <int Mode>
struct PjLayout {
  static constexpr int kStages = Mode == kBaseConv ? 3 : 4;
  static constexpr int kStageA = kPjM * kPjK * 2;                 // 16 KiB
  static constexpr int kStageB = kPjN * kPjK * 2;                 // 32 KiB
  static constexpr int kA = 0;
  static constexpr int kB = kStages * kStageA;
  static constexpr int kHalo = kB + kStages * kStageB;            // [4][136 rows][128 B] SW128
  static constexpr int kHaloBlock = kPjHaloRows * 128;
  static constexpr int kHaloBytes = Mode == kBaseConv ? 4 * kHaloBlock : 0;
  // BaseConv: the tile's taps, transposed to [tap][column], and its bias
  static constexpr int kTaps = kHalo + kHaloBytes;
  static constexpr int kBias = kTaps + (Mode == kBaseConv ? kPjMaxTaps * kPjN * 4 : 0);
  static constexpr int kBar = kBias + (Mode == kBaseConv ? kPjN * 4 : 0);
  static constexpr int kBytes = kBar + 256;
  static constexpr size_t kSmem = kBytes + 1024;
  static_assert(kB % 1024 == 0 && kHalo % 1024 == 0 && kHaloBlock % 1024 == 0,
                "swizzled tiles are 1024-byte aligned");
  static_assert(kSmem <= 232448, "shared memory budget");
};

struct ProjParams {
  const __nv_bfloat16* x;  // kBaseConv: the layer input (for the convolution's taps)
  __nv_bfloat16* y;
  const float* bias;       // kBaseConv: [N]
  const float* taps;       // kBaseConv: [N][K]
  int M, N, Kd;
  int L;                   // tokens per sequence
  int H, D;                // kProjHeads: heads and features per head (N = H * D)
  int K;                   // kBaseConv: filter taps
  int n_tiles_n;           // N / 256
  int total_tiles;
};

template <int Mode>
__global__ void __launch_bounds__(kPjThreads, 1)
    proj_tc_kernel(const __grid_constant__ CUtensorMap xmap,
                   const __grid_constant__ CUtensorMap wmap,
                   const __grid_constant__ CUtensorMap hmap, const ProjParams p) {
  using Lay = PjLayout<Mode>;
  constexpr int S = Lay::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::kBar);
  uint64_t* bar_full = bars;               // [S] stage landed
  uint64_t* bar_empty = bars + S;          // [S] stage read by the MMAs (commit)
  uint64_t* bar_afull = bars + 2 * S;      // [2] accumulator complete (commit)
  uint64_t* bar_aempty = bars + 2 * S + 2; // [2] accumulator read (epilogue)
  uint64_t* bar_hfull = bars + 2 * S + 4;  // input rows of the tile landed
  uint64_t* bar_hempty = bars + 2 * S + 5; // input rows read (epilogue)
  uint64_t* bar_done = bars + 2 * S + 6;   // every MMA issued has completed (commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 7);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * S + 8);
  uint64_t* bar_tready = bars + 2 * S + 9;   // taps and bias of the tile written (epilogue)
  uint64_t* bar_tfree = bars + 2 * S + 10;   // taps and bias of the tile no longer read

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int first = blockIdx.x, step = gridDim.x;
  const int n_mine = p.total_tiles > first ? (p.total_tiles - first + step - 1) / step : 0;
  const int nkb = p.Kd / kPjK;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      umma::mbar_init(bar_full + s, 1);
      umma::mbar_init(bar_empty + s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      umma::mbar_init(bar_afull + a, 1);
      umma::mbar_init(bar_aempty + a, kPjM);
    }
    umma::mbar_init(bar_hfull, 1);
    umma::mbar_init(bar_hempty, kPjM);
    umma::mbar_init(bar_done, 1);
    umma::mbar_init(bar_tready, kPjM);
    umma::mbar_init(bar_tfree, kPjM);
    *abort_flag = 0;
    umma::fence_mbar_init();
  }
  if (warp == 1) {
    umma::tmem_alloc(tmem_slot, 2 * kPjN);
    umma::tmem_relinquish();
  }
  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto fail = [&]() {
    record_device_error(BASED_ERR_TIMEOUT);
    *abort_flag = 1;
  };
  auto tile_at = [&](int k, int* m0, int* n0) {
    const int i = first + k * step;
    const int mt = i / p.n_tiles_n;
    *m0 = mt * kPjM;
    *n0 = (i - mt * p.n_tiles_n) * kPjN;
  };

  if (warp == 0) {
    // ================= producer =================
    if (lane == 0) {
      constexpr uint32_t bytes = (kPjM + kPjN) * kPjK * 2;
      int g = 0, halo_issued = 0;
      for (int k = 0; k < n_mine && !*abort_flag; ++k) {
        int m0, n0;
        tile_at(k, &m0, &n0);
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % S;
          if (g >= S && !umma::mbar_wait(bar_empty + s, ((g - S) / S) & 1)) { fail(); break; }
          umma::mbar_arrive_expect_tx(bar_full + s, bytes);
          umma::tma_load_3d(sm + Lay::kA + s * Lay::kStageA, &xmap, bar_full + s, kb * kPjK, m0, 0);
          umma::tma_load_3d(sm + Lay::kB + s * Lay::kStageB, &wmap, bar_full + s, kb * kPjK, n0, 0);
        }
        if (*abort_flag) break;
        if (Mode == kBaseConv) {
          // this tile's input rows, once the previous tile's epilogue has read its own
          if (k >= 1 && !umma::mbar_wait(bar_hempty, (k - 1) & 1)) { fail(); break; }
          umma::mbar_arrive_expect_tx(bar_hfull, 4 * Lay::kHaloBlock);
#pragma unroll
          for (int blk = 0; blk < 4; ++blk)
            umma::tma_load_3d(sm + Lay::kHalo + blk * Lay::kHaloBlock, &hmap, bar_hfull,
                              n0 + blk * 64, m0 - kPjMaxTaps, 0);
          halo_issued = k + 1;
        }
      }
      // loads that nobody consumed (after an abort) must land before the CTA exits
      if (*abort_flag) {
        for (int gg = g - S > 0 ? g - S : 0; gg < g; ++gg)
          umma::mbar_wait(bar_full + gg % S, (gg / S) & 1);
        if (halo_issued > 0) umma::mbar_wait(bar_hfull, (halo_issued - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issue =================
    if (lane == 0) {
      const uint32_t id = umma::idesc_bf16(kPjM, kPjN, false, false);
      int g = 0;
      for (int k = 0; k < n_mine && !*abort_flag; ++k) {
        const int a = k & 1;
        if (k >= 2 && !umma::mbar_wait(bar_aempty + a, ((k - 2) >> 1) & 1)) { fail(); break; }
        umma::tc_fence_after();
        bool okk = true;
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % S;
          if (!umma::mbar_wait(bar_full + s, (g / S) & 1)) { okk = false; break; }
          umma::tc_fence_after();
          const uint32_t sa = umma::smem_u32(sm + Lay::kA + s * Lay::kStageA);
          const uint32_t sb = umma::smem_u32(sm + Lay::kB + s * Lay::kStageB);
#pragma unroll
          for (int k0 = 0; k0 < kPjK; k0 += 16)
            umma::mma_bf16(tmem + a * kPjN, umma::desc_kmajor_sw128(sa, k0, kPjM),
                           umma::desc_kmajor_sw128(sb, k0, kPjN), id, (kb | k0) != 0);
          umma::mma_commit(bar_empty + s);
        }
        if (!okk) { fail(); break; }
        umma::mma_commit(bar_afull + a);
      }
      umma::mma_commit(bar_done);
    }
  } else {
    // ================= epilogue: warps 2-5, TMEM lane quadrant = warp mod 4 =================
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    for (int k = 0; k < n_mine && !*abort_flag; ++k) {
      const int a = k & 1;
      int m0, n0;
      tile_at(k, &m0, &n0);
      if (!umma::mbar_wait(bar_afull + a, (k >> 1) & 1)) { fail(); break; }
      if (Mode == kBaseConv && !umma::mbar_wait(bar_hfull, k & 1)) { fail(); break; }
      umma::tc_fence_after();
      float* tapsT = reinterpret_cast<float*>(sm + Lay::kTaps);
      float* bias_s = reinterpret_cast<float*>(sm + Lay::kBias);
      if (Mode == kBaseConv) {
        // this tile's taps and bias into shared memory, once every epilogue
        // thread has finished reading the previous tile's
        if (k >= 1 && !umma::mbar_wait(bar_tfree, (k - 1) & 1)) { fail(); break; }
        for (int c = r; c < kPjN; c += kPjM) {
          for (int j = 0; j < p.K; ++j) tapsT[j * kPjN + c] = __ldg(p.taps + (size_t)(n0 + c) * p.K + j);
          bias_s[c] = __ldg(p.bias + n0 + c);
        }
        umma::mbar_arrive(bar_tready);
        if (!umma::mbar_wait(bar_tready, k & 1)) { fail(); break; }
      }
      const int m = m0 + r;
      const int b = m / p.L, t = m - (m / p.L) * p.L;
#pragma unroll 1
      for (int c32 = 0; c32 < kPjN / 32; ++c32) {
        float acc[32];
        umma::tmem_ld32(tmem + a * kPjN + (static_cast<uint32_t>(quad * 32) << 16) + c32 * 32, acc);
        if (m >= p.M) continue;
#pragma unroll
        for (int g = 0; g < 4; ++g) {  // 8 columns = one 16-byte store
          const int cl = c32 * 32 + g * 8;  // column within the tile
          const int n = n0 + cl;
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = acc[g * 8 + e];
          size_t dst;
          if (Mode == kProjHeads) {
            const int hh = n / p.D, d = n - hh * p.D;
            dst = (((size_t)b * p.H + hh) * p.L + t) * p.D + d;
          } else {
            // input rows m - j of this tile's columns: row r + 8 - j of the staged
            // block cl / 64, 16-byte chunk (cl mod 64) / 8, swizzled by row mod 8
            float conv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) conv[e] = 0.0f;
            const uint8_t* hb = sm + Lay::kHalo + (cl >> 6) * Lay::kHaloBlock;
            const int chunk = (cl & 63) >> 3;
            for (int j = 0; j < p.K && j <= t; ++j) {
              const int hr = r + kPjMaxTaps - j;
              const uint4 xv = *reinterpret_cast<const uint4*>(hb + hr * 128 + ((chunk ^ (hr & 7)) << 4));
              const float4 h0 = *reinterpret_cast<const float4*>(tapsT + j * kPjN + cl);
              const float4 h1 = *reinterpret_cast<const float4*>(tapsT + j * kPjN + cl + 4);
              const float hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
              const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xw[e]));
                conv[2 * e] = fmaf(hv[2 * e], f.x, conv[2 * e]);
                conv[2 * e + 1] = fmaf(hv[2 * e + 1], f.y, conv[2 * e + 1]);
              }
            }
            const float4 b0 = *reinterpret_cast<const float4*>(bias_s + cl);
            const float4 b1 = *reinterpret_cast<const float4*>(bias_s + cl + 4);
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = (v[e] + bv[e]) * conv[e];
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
      umma::tc_fence_before();
      umma::mbar_arrive(bar_aempty + a);
      if (Mode == kBaseConv) {
        umma::mbar_arrive(bar_hempty);
        umma::mbar_arrive(bar_tfree);
      }
    }
  }
  umma::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // TMEM is released only after every MMA issued here has completed
    if (lane == 0) umma::mbar_wait(bar_done, 0);
    __syncwarp();
    umma::tmem_dealloc(tmem, 2 * kPjN);
  }
}

}  // namespace based
