// proj_tc.cuh -- input projections of a Based layer on the sm_100a tensor cores.
//
// Y = X W^T for X [M, Kd] (M = B*L tokens, row-major) and W [N, Kd] (one output
// feature per row), bf16 in, fp32 accumulation in TMEM, with one of two epilogues:
//
//  * kProjHeads -- the per-head projections that feed the attention layers
//    ("Базированная модель, часть 2", the paragraph on the size of the hidden
//    state: the KV and K states are made smaller by projections of the input).
//    W stacks up to kPjMaxOut projections of the same x (rows [col_begin[g],
//    col_begin[g+1]) are projection g, H heads of D[g] features); column
//    n = col_begin[g] + h*D[g] + d of token m = b*L + t goes to
//    y_g[b][h][t][d] (bf16).  One launch serves every projection of a layer,
//    so x is streamed once for all of them.
//  * kBaseConv -- the BaseConv block ("Базированная модель, часть 1", section
//    "Кто виноват?": y = linear(x) (.) conv(h, x)): N = Kd = D channels, and
//    y[m][c] = (Y[m][c] + bias[c]) * sum_{j <= min(K-1, t)} h[c][j] x[m-j][c].
//
// CTA pairs: a cluster of two CTAs (one TPC) owns a 256 x 256 output tile and
// runs it as M = 256 tcgen05 MMAs (.cta_group::2).  Each CTA loads its own 128
// rows of X and 128 of the tile's 256 rows of W, so a pair reads 64 KiB per
// 64-deep K block for 2 x 256 x 256 x 64 flop -- half the L2 traffic per flop of
// a one-CTA 128 x 256 tile, which the L2 -> SM bandwidth could not feed.
// Persistent: the pairs walk the tiles (tiles sharing an X row block are
// adjacent, so X is read from DRAM about once).  Per CTA: warp 0 (one thread)
// streams K blocks by TMA through a ring of stages (128B swizzle, K-major),
// counting the bytes of both CTAs on the even CTA's barrier; warp 1 of the even
// CTA (one thread) issues four M=256/N=256/K=16 MMAs per block into one of two
// TMEM accumulators, so the epilogue of tile k overlaps the main loop of tile
// k+1; warps 2-9 run the epilogue on the CTA's own 128 rows (warps w and w+4
// share TMEM lane quadrant w mod 4 and take one half of the 256 columns each).
// Per-head outputs leave by TMA: a head's 128 rows of one sequence are one box
// of its [B*H, L, D] output, so each half writes its 128 columns into a
// swizzled staging tile in shared memory and one thread stores them, a box per
// head (or per 64 columns of a head); a tile whose rows cross a sequence end,
// or a head width that does not divide 128, falls back to 16-byte stores from
// every thread.  For BaseConv the producer also loads the CTA's input rows
// [m0-8, m0+128) x [n0, n0+256) (the convolution's reach) into shared memory,
// once the previous tile's epilogue has released them.
#pragma once

#include "common.cuh"
#include "umma.cuh"

namespace based {

constexpr int kPjM = 128;       // rows (tokens) per CTA; a pair covers 256
constexpr int kPjN = 256;       // columns per tile
constexpr int kPjNHalf = 128;   // rows of W loaded by each CTA of the pair
constexpr int kPjK = 64;        // K block per stage (one 128-byte swizzle atom)
constexpr int kPjEpiWarps = 8;  // two per TMEM lane quadrant, each on half the columns
constexpr int kPjEpiThreads = kPjEpiWarps * 32;
constexpr int kPjThreads = 64 + kPjEpiThreads;
constexpr int kPjMaxTaps = 8;
constexpr int kPjHaloRows = kPjM + kPjMaxTaps;  // rows [m0 - 8, m0 + 128)
constexpr int kPjMaxOut = 8;    // projections per launch

enum ProjMode { kProjHeads = 0, kBaseConv = 1 };

template <int Mode>
struct PjLayout {
  static constexpr int kStages = Mode == kBaseConv ? 4 : 5;
  static constexpr int kStageA = kPjM * kPjK * 2;                 // 16 KiB
  static constexpr int kStageB = kPjNHalf * kPjK * 2;             // 16 KiB
  static constexpr uint32_t kTxPair = 2u * (kStageA + kStageB);   // both CTAs' bytes
  static constexpr int kA = 0;
  static constexpr int kB = kStages * kStageA;
  static constexpr int kHalo = kB + kStages * kStageB;            // [4][136 rows][128 B] SW128
  static constexpr int kHaloBlock = kPjHaloRows * 128;
  static constexpr int kHaloBytes = Mode == kBaseConv ? 4 * kHaloBlock : 0;
  // BaseConv: the tile's taps, transposed to [tap][column], and its bias
  // per-head outputs: one staging tile per half, [boxes][128 rows][box width]
  static constexpr int kStg = kHalo + kHaloBytes;
  static constexpr int kStgHalf = kPjM * kPjNHalf * 2;                       // 32 KiB
  static constexpr int kStgBytes = Mode == kProjHeads ? 2 * kStgHalf : 0;
  static constexpr int kTaps = kStg + kStgBytes;
  static constexpr int kBias = kTaps + (Mode == kBaseConv ? kPjMaxTaps * kPjN * 4 : 0);
  static constexpr int kBar = kBias + (Mode == kBaseConv ? kPjN * 4 : 0);
  static constexpr int kBytes = kBar + 256;
  static constexpr size_t kSmem = kBytes + 1024;
  static_assert(kB % 1024 == 0 && kHalo % 1024 == 0 && kHaloBlock % 1024 == 0 &&
                    kStg % 1024 == 0,
                "swizzled tiles are 1024-byte aligned");
  static_assert(kSmem <= 232448, "shared memory budget");
};

// Output tensor maps of the per-head projections: y_g as [B*H][L][D] with
// boxes of 128 rows x min(D, 64) columns, swizzled by the box row's width.
struct ProjYMaps {
  CUtensorMap m[kPjMaxOut];
};

struct ProjParams {
  const __nv_bfloat16* x;  // kBaseConv: the layer input (for the convolution's taps)
  __nv_bfloat16* y[kPjMaxOut];
  int D[kPjMaxOut];        // kProjHeads: features per head of each projection
  int col_begin[kPjMaxOut + 1];
  int n_out;
  const float* bias;       // kBaseConv: [N]
  const float* taps;       // kBaseConv: [N][K]
  int M, N, Kd;
  int L;                   // tokens per sequence
  int H;                   // kProjHeads: heads of every projection
  int K;                   // kBaseConv: filter taps
  int n_tiles_n;           // N / 256
  int total_tiles;         // 256 x 256 tiles
};

template <int Mode>
__global__ void __launch_bounds__(kPjThreads, 1)
    proj_tc_kernel(const __grid_constant__ CUtensorMap xmap,
                   const __grid_constant__ CUtensorMap wmap,
                   const __grid_constant__ CUtensorMap hmap,
                   const __grid_constant__ ProjYMaps ymaps, const ProjParams p) {
  using Lay = PjLayout<Mode>;
  constexpr int S = Lay::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::kBar);
  uint64_t* bar_full = bars;               // [S] both CTAs' stage landed (even CTA's copy used)
  uint64_t* bar_empty = bars + S;          // [S] stage read by the MMAs (commit, both CTAs)
  uint64_t* bar_afull = bars + 2 * S;      // [2] accumulator complete (commit, both CTAs)
  uint64_t* bar_aempty = bars + 2 * S + 2; // [2] accumulator read by both epilogues (even CTA)
  uint64_t* bar_hfull = bars + 2 * S + 4;  // input rows of the tile landed
  uint64_t* bar_hempty = bars + 2 * S + 5; // input rows read (epilogue)
  uint64_t* bar_done = bars + 2 * S + 6;   // every MMA issued has completed (commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 7);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 2 * S + 8);
  uint64_t* bar_tready = bars + 2 * S + 9;   // taps and bias of the tile written (epilogue)
  uint64_t* bar_tfree = bars + 2 * S + 10;   // taps and bias of the tile no longer read

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = umma::cluster_ctarank();  // 0: issues the pair's MMAs
  const int first = (int)umma::cluster_id_x(), step = (int)umma::cluster_count_x();
  const int n_mine = p.total_tiles > first ? (p.total_tiles - first + step - 1) / step : 0;
  const int nkb = p.Kd / kPjK;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      umma::mbar_init(bar_full + s, 1);
      umma::mbar_init(bar_empty + s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      umma::mbar_init(bar_afull + a, 1);
      umma::mbar_init(bar_aempty + a, 2 * kPjEpiWarps);  // one per epilogue warp, both CTAs
    }
    umma::mbar_init(bar_hfull, 1);
    umma::mbar_init(bar_hempty, kPjEpiThreads);
    umma::mbar_init(bar_done, 1);
    umma::mbar_init(bar_tready, kPjEpiThreads);
    umma::mbar_init(bar_tfree, kPjEpiThreads);
    *abort_flag = 0;
    umma::fence_mbar_init();
  }
  if (warp == 1) {
    umma::tmem_alloc_pair(tmem_slot, 2 * kPjN);
    umma::tmem_relinquish_pair();
  }
  umma::tc_fence_before();
  // both CTAs' barriers are initialised and their TMEM allocated before any
  // load, MMA or arrival reaches the other CTA
  umma::cluster_sync();
  umma::tc_fence_after();
  // a dependent launch: the set-up above overlaps the previous kernel
  umma::grid_dep_wait();
  umma::grid_dep_launch();
  const uint32_t tmem = *tmem_slot;
  auto fail = [&]() {
    record_device_error(BASED_ERR_TIMEOUT);
    *abort_flag = 1;
  };
  // this CTA's rows of the pair tile k, and the tile's first column
  auto tile_at = [&](int k, int* m0, int* n0) {
    const int i = first + k * step;
    const int mt = i / p.n_tiles_n;
    *m0 = mt * (2 * kPjM) + (int)rank * kPjM;
    *n0 = (i - mt * p.n_tiles_n) * kPjN;
  };

  if (warp == 0) {
    // ================= producer (both CTAs) =================
    if (lane == 0) {
      const uint32_t full0 = umma::cluster_addr(bar_full, 0);  // the even CTA's barriers
      int g = 0, halo_issued = 0;
      for (int k = 0; k < n_mine && !*abort_flag; ++k) {
        int m0, n0;
        tile_at(k, &m0, &n0);
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % S;
          if (g >= S && !umma::mbar_wait(bar_empty + s, ((g - S) / S) & 1)) { fail(); break; }
          if (rank == 0) umma::mbar_arrive_expect_tx(bar_full + s, Lay::kTxPair);
          umma::tma_load_3d_pair(sm + Lay::kA + s * Lay::kStageA, &xmap, full0 + 8u * s,
                                 kb * kPjK, m0, 0);
          umma::tma_load_3d_pair(sm + Lay::kB + s * Lay::kStageB, &wmap, full0 + 8u * s,
                                 kb * kPjK, n0 + (int)rank * kPjNHalf, 0);
        }
        if (*abort_flag) break;
        if (Mode == kBaseConv) {
          // this CTA's input rows, once the previous tile's epilogue has read its own
          if (k >= 1 && !umma::mbar_wait(bar_hempty, (k - 1) & 1)) { fail(); break; }
          umma::mbar_arrive_expect_tx(bar_hfull, 4 * Lay::kHaloBlock);
#pragma unroll
          for (int blk = 0; blk < 4; ++blk)
            umma::tma_load_3d(sm + Lay::kHalo + blk * Lay::kHaloBlock, &hmap, bar_hfull,
                              n0 + blk * 64, m0 - kPjMaxTaps, 0);
          halo_issued = k + 1;
        }
      }
      // Loads that nobody consumed (after an abort) must land before the CTAs
      // exit.  The even CTA's barrier counts both CTAs' bytes of a stage; the odd
      // CTA cannot see it, so it waits long enough for any load in flight.
      if (*abort_flag) {
        if (rank == 0) {
          for (int gg = g - S > 0 ? g - S : 0; gg < g; ++gg)
            umma::mbar_wait(bar_full + gg % S, (gg / S) & 1);
        } else {
          const uint64_t t0 = umma::global_timer_ns();
          while (umma::global_timer_ns() - t0 < 200000ull) {
          }
        }
        if (halo_issued > 0) umma::mbar_wait(bar_hfull, (halo_issued - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issue (even CTA) =================
    if (lane == 0 && rank == 0) {
      const uint32_t id = umma::idesc_bf16(2 * kPjM, kPjN, false, false);
      const uint32_t empty1 = umma::cluster_addr(bar_empty, 1);
      const uint32_t afull1 = umma::cluster_addr(bar_afull, 1);
      int g = 0;
      for (int k = 0; k < n_mine && !*abort_flag; ++k) {
        const int a = k & 1;
        // both epilogues have read accumulator a (tile k-2)
        if (k >= 2 && !umma::mbar_wait_cluster(bar_aempty + a, ((k - 2) >> 1) & 1)) {
          fail();
          break;
        }
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
            umma::mma_bf16_pair(tmem + a * kPjN, umma::desc_kmajor_sw128(sa, k0, kPjM),
                                umma::desc_kmajor_sw128(sb, k0, kPjNHalf), id, (kb | k0) != 0);
          umma::mma_commit_pair(umma::smem_u32(bar_empty + s));
          umma::mma_commit_pair(empty1 + 8u * s);
        }
        if (!okk) { fail(); break; }
        umma::mma_commit_pair(umma::smem_u32(bar_afull + a));
        umma::mma_commit_pair(afull1 + 8u * a);
      }
      umma::mma_commit_pair(umma::smem_u32(bar_done));
    }
  } else {
    // ================= epilogue: warps 2-9, TMEM lane quadrant = warp mod 4 =================
    const int quad = warp & 3;
    const int r = quad * 32 + lane;          // row of the CTA's 128
    const int half = (warp - 2) >> 2;        // columns [128 half, 128 half + 128)
    const int et = (warp - 2) * 32 + lane;   // index among the epilogue threads
    const uint32_t aempty0 = umma::cluster_addr(bar_aempty, 0);
    // the thread that stores this half's staging tile
    const bool issuer = (et & (kPjEpiThreads / 2 - 1)) == 0;
    uint8_t* stg = sm + Lay::kStg + half * Lay::kStgHalf;
    for (int k = 0; k < n_mine && !*abort_flag; ++k) {
      const int a = k & 1;
      int m0, n0;
      tile_at(k, &m0, &n0);
      const bool ok_a = umma::mbar_wait(bar_afull + a, (k >> 1) & 1);
      if (Mode == kProjHeads) {
        // the half decides together (a named barrier must see all 128 threads),
        // once the previous tile's stores have read the staging tile
        if (issuer) umma::bulk_wait_read<0>();
        if (!umma::named_sync_all(1 + half, kPjEpiThreads / 2, ok_a)) { fail(); break; }
      } else if (!ok_a) {
        fail();
        break;
      }
      if (Mode == kBaseConv && !umma::mbar_wait(bar_hfull, k & 1)) { fail(); break; }
      umma::tc_fence_after();
      float* tapsT = reinterpret_cast<float*>(sm + Lay::kTaps);
      float* bias_s = reinterpret_cast<float*>(sm + Lay::kBias);
      if (Mode == kBaseConv) {
        // this tile's taps and bias into shared memory, once every epilogue
        // thread has finished reading the previous tile's
        if (k >= 1 && !umma::mbar_wait(bar_tfree, (k - 1) & 1)) { fail(); break; }
        for (int c = et; c < kPjN; c += kPjEpiThreads) {
          for (int j = 0; j < p.K; ++j) tapsT[j * kPjN + c] = __ldg(p.taps + (size_t)(n0 + c) * p.K + j);
          bias_s[c] = __ldg(p.bias + n0 + c);
        }
        umma::mbar_arrive(bar_tready);
        if (!umma::mbar_wait(bar_tready, k & 1)) { fail(); break; }
      }
      // the projection this tile belongs to (every projection is whole tiles wide)
      int og = 0;
      if (Mode == kProjHeads)
        while (og + 1 < p.n_out && n0 >= p.col_begin[og + 1]) ++og;
      __nv_bfloat16* yo = p.y[og];
      const int Dg = p.D[og];
      const int nb = n0 - p.col_begin[og];
      const int m = m0 + r;
      const int b = m / p.L, t = m - (m / p.L) * p.L;
      // TMA stores: the CTA's 128 rows lie in one sequence and heads tile the half
      const int t_first = m0 % p.L;
      const bool tma_out = Mode == kProjHeads && m0 < p.M && t_first + kPjM <= p.L &&
                           kPjNHalf % Dg == 0;
      // staging tile: boxes of bw columns; row r of a box is rb bytes, its 16-byte
      // chunk c at position c ^ ((r >> sh) & (rb / 16 - 1)) (the tensor map's swizzle)
      const int bw = Dg < 64 ? Dg : 64, rb = 2 * bw;
      const int sh = rb == 128 ? 0 : (rb == 64 ? 1 : 2);
      const int cmask = rb / 16 - 1;
#pragma unroll 1
      for (int c32 = 4 * half; c32 < 4 * half + 4; ++c32) {
        float acc[32];
        umma::tmem_ld32(tmem + a * kPjN + (static_cast<uint32_t>(quad * 32) << 16) + c32 * 32, acc);
        if (m >= p.M) continue;
#pragma unroll
        for (int g = 0; g < 4; ++g) {  // 8 columns = one 16-byte store
          const int cl = c32 * 32 + g * 8;  // column within the tile
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = acc[g * 8 + e];
          size_t dst;
          if (Mode == kProjHeads) {
            const int n = nb + cl;
            const int hh = n / Dg, d = n - hh * Dg;
            dst = (((size_t)b * p.H + hh) * p.L + t) * Dg + d;
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
            dst = (size_t)m * p.N + n0 + cl;
          }
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
            pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          if (tma_out) {
            const int ch = cl - half * kPjNHalf;  // column within the half
            const int bx = ch / bw, c = (ch - bx * bw) >> 3;
            *reinterpret_cast<uint4*>(stg + bx * (rb * kPjM) + r * rb +
                                      ((c ^ ((r >> sh) & cmask)) << 4)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          } else {
            *reinterpret_cast<uint4*>(yo + dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
      // accumulator a is read: one arrival per warp on the even CTA's barrier
      umma::tc_fence_before();
      __syncwarp();
      if (lane == 0) umma::mbar_arrive_cluster(aempty0 + 8u * a);
      if (tma_out) {
        // the staging tile is written: one thread stores a box per head (or per
        // 64 columns of a head), [d0, d0 + bw) x rows [t_first, t_first + 128)
        umma::fence_async_smem();
        umma::named_sync(1 + half, kPjEpiThreads / 2);
        if (issuer) {
          const int b0 = m0 / p.L;
          for (int bx = 0; bx < kPjNHalf / bw; ++bx) {
            const int col = nb + half * kPjNHalf + bx * bw;  // column within the projection
            const int hh = col / Dg;
            umma::tma_store_3d(&ymaps.m[og], stg + bx * (rb * kPjM), col - hh * Dg, t_first,
                               b0 * p.H + hh);
          }
          umma::bulk_commit();
        }
      }
      if (Mode == kBaseConv) {
        umma::mbar_arrive(bar_hempty);
        umma::mbar_arrive(bar_tfree);
      }
    }
  }
  // the last stores have read their staging tiles
  if (Mode == kProjHeads && warp >= 2 && ((tid - 64) & (kPjEpiThreads / 2 - 1)) == 0)
    umma::bulk_wait_read<0>();
  umma::tc_fence_before();
  __syncthreads();
  // every MMA of the pair has completed before either CTA releases its TMEM
  if (warp == 1 && rank == 0) {
    if (lane == 0) umma::mbar_wait(bar_done, 0);
    __syncwarp();
  }
  umma::cluster_sync();
  umma::tc_fence_after();
  if (warp == 1) umma::tmem_dealloc_pair(tmem, 2 * kPjN);
}

}  // namespace based
