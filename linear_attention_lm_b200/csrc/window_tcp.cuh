// window_tcp.cuh -- persistent, pipelined sliding-window attention for d_head = 64.
//
// Based README, introduction, item 1: exact softmax attention over a sliding
// window (size 64).  Same computation per 128-query tile as window_tc_kernel
// (S = Q K^T over the 192 staged keys [t0-64, t0+128), band softmax in
// registers, P in TMEM, O = P V, y = O / l), organised for throughput: one CTA
// per SM walks its tiles (tile g, g + G, ...) with a 3-stage TMA ring of Q/K/V
// tiles, one MMA thread and two softmax warp groups that take alternate tiles,
// each with its own 256-column TMEM slot (S: 192 columns, O: 64) and its own y
// staging tile.  The MMA thread issues S of tile k+1 before P V of tile k, so
// the tensor core works on one tile while a softmax group works on the other.
// Q/K and V of a stage are loaded and released separately (two producer
// warps): Q/K of tile k+3 are loaded as soon as S of tile k has read them, V
// once P V of tile k has, so each load has about three tile periods to land.
#pragma once

#include "common.cuh"
#include "umma.cuh"
#include "window_softmax.cuh"

// Optional per-tile event stamps for performance analysis (a build may define
// BASED_WP_TRACE(event, tile); by default the marks compile to nothing).
#ifndef BASED_WP_TRACE
#define BASED_WP_TRACE(event, tile) ((void)0)
#endif

namespace based {

constexpr int kWpStages = 3;
constexpr int kWpThreads = 352;  // softmax groups: warps 0-3, 4-7; MMA warp 8; Q/K, V TMA warps 9, 10

struct WpLayout {
  static constexpr int kQ = 0;                        // per stage: Q [128 x 64] K-major SW128
  static constexpr int kK = 16384;                    //            K [192 x 64] K-major SW128
  static constexpr int kV = kK + 24576;               //            V [192 x 64] MN-major SW128
  static constexpr int kStage = kV + 24576;           // 64 KiB per stage
  static constexpr int kY = kWpStages * kStage;       // y staging [2][128 x 64] bf16 SW128
  static constexpr int kBar = kY + 2 * 16384;
  static constexpr int kBytes = kBar + 256;
  static constexpr size_t kSmem = kBytes + 1024;
  static constexpr uint32_t kTxQK = (128 + 192) * 64 * 2;
  static constexpr uint32_t kTxV = 192 * 64 * 2;
};
static_assert(WpLayout::kSmem <= 232448, "shared memory budget");

__global__ void __launch_bounds__(kWpThreads, 1)
    window_tcp_kernel(const __grid_constant__ CUtensorMap qmap,
                      const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap,
                      const __grid_constant__ CUtensorMap ymap, int L, int W, int tiles_per_seq,
                      int n_total) {
  using Lay = WpLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::kBar);
  uint64_t* full = bars;          // [3] Q/K of a stage loaded (TMA)
  uint64_t* empty = bars + 3;     // [3] Q/K of a stage read (commit after S)
  uint64_t* sfull = bars + 6;     // [2] S ready in slot (commit)
  uint64_t* pfull = bars + 8;     // [2] P written to slot (softmax group)
  uint64_t* ofull = bars + 10;    // [2] O ready in slot (commit)
  uint64_t* tfree = bars + 12;    // [2] slot read out (softmax group)
  uint64_t* bar_fin = bars + 14;  // every MMA complete (commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 16);
  volatile int* consumed = reinterpret_cast<volatile int*>(bars + 17);     // Q/K loads waited
  uint64_t* vfull = bars + 18;    // [3] V of a stage loaded (TMA)
  uint64_t* vempty = bars + 21;   // [3] V of a stage read (commit after P V)
  volatile int* consumed_v = reinterpret_cast<volatile int*>(bars + 24);  // V loads waited

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x;
  const int n_mine = (n_total - (int)blockIdx.x + G - 1) / G;
  auto tile_of = [&](int k, int* bh, int* t0) {
    const int g = (int)blockIdx.x + k * G;
    *bh = g / tiles_per_seq;
    *t0 = (g - *bh * tiles_per_seq) * 128;
  };
  auto fail = [&]() {
    record_device_error(BASED_ERR_TIMEOUT);
    *abort_flag = 1;
  };

  if (tid == 0) {
    for (int i = 0; i < kWpStages; ++i) {
      umma::mbar_init(full + i, 1);
      umma::mbar_init(empty + i, 1);
      umma::mbar_init(vfull + i, 1);
      umma::mbar_init(vempty + i, 1);
    }
    for (int j = 0; j < 2; ++j) {
      umma::mbar_init(sfull + j, 1);
      umma::mbar_init(pfull + j, 128);
      umma::mbar_init(ofull + j, 1);
      umma::mbar_init(tfree + j, 128);
    }
    umma::mbar_init(bar_fin, 1);
    *abort_flag = 0;
    *consumed = 0;
    *consumed_v = 0;
    umma::fence_mbar_init();
  }
  if (warp == 8) {
    umma::tmem_alloc(tmem_slot, 512);
    umma::tmem_relinquish();
  }
  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  // the set-up above touched no global memory: it overlaps the previous kernel
  umma::grid_dep_wait();
  umma::grid_dep_launch();
  const uint32_t tmem = *tmem_slot;
  int issued = 0;  // loads issued (TMA thread)

  if (warp == 9 || warp == 10) {
    // ================= TMA producers: Q/K (warp 9) and V (warp 10) =================
    const bool is_v = warp == 10;
    if (lane == 0) {
      umma::tma_prefetch_desc(is_v ? &vmap : &qmap);
      if (!is_v) umma::tma_prefetch_desc(&kmap);
      for (int k = 0; k < n_mine && !*abort_flag; ++k) {
        const int stage = k % kWpStages;
        if (k >= kWpStages &&
            !umma::mbar_wait((is_v ? vempty : empty) + stage, ((k / kWpStages) - 1) & 1)) {
          fail();
          break;
        }
        BASED_WP_TRACE(0, k);
        int bh, t0;
        tile_of(k, &bh, &t0);
        uint8_t* st = sm + stage * Lay::kStage;
        if (!is_v) {
          umma::mbar_arrive_expect_tx(full + stage, Lay::kTxQK);
          umma::tma_load_3d(st + Lay::kQ, &qmap, full + stage, 0, t0, bh);
          umma::tma_load_3d(st + Lay::kK, &kmap, full + stage, 0, t0 - 64, bh);
        } else if (k > 0 || !stall_test(kStallWindowV)) {  // the stall test leaves V(0) out
          umma::mbar_arrive_expect_tx(vfull + stage, Lay::kTxV);
          umma::tma_load_3d(st + Lay::kV, &vmap, vfull + stage, 0, t0 - 64, bh);
        }
        ++issued;
      }
    }
  } else if (warp == 8) {
    // ================= MMA issuer =================
    if (lane == 0) {
      const uint32_t id_s = umma::idesc_bf16(128, 192, false, false);
      const uint32_t id_o = umma::idesc_bf16(128, 64, false, true);
      auto issue_s = [&](int k) -> bool {
        const int stage = k % kWpStages, slot = k & 1;
        if (!umma::mbar_wait(full + stage, (k / kWpStages) & 1)) return false;
        BASED_WP_TRACE(0, k);
        *consumed = k + 1;
        if (k >= 2 && !umma::mbar_wait(tfree + slot, ((k >> 1) - 1) & 1)) return false;
        umma::tc_fence_after();
        const uint32_t sQ = umma::smem_u32(sm + stage * Lay::kStage + Lay::kQ);
        const uint32_t sK = umma::smem_u32(sm + stage * Lay::kStage + Lay::kK);
#pragma unroll
        for (int k0 = 0; k0 < 64; k0 += 16)
          umma::mma_bf16(tmem + slot * 256, umma::desc_kmajor_sw128(sQ, k0, 128),
                         umma::desc_kmajor_sw128(sK, k0, 192), id_s, k0 > 0);
        umma::mma_commit(sfull + slot);
        umma::mma_commit(empty + stage);  // Q/K of this stage may be refilled
        BASED_WP_TRACE(1, k);
        return true;
      };
      bool ok = n_mine > 0 ? issue_s(0) : true;
      for (int k = 0; k < n_mine && ok && !*abort_flag; ++k) {
        const int stage = k % kWpStages, slot = k & 1;
        if (k + 1 < n_mine && !issue_s(k + 1)) { ok = false; break; }
        if (!umma::mbar_wait(pfull + slot, (k >> 1) & 1)) { ok = false; break; }
        if (!umma::mbar_wait(vfull + stage, (k / kWpStages) & 1)) { ok = false; break; }
        *consumed_v = k + 1;
        BASED_WP_TRACE(2, k);
        umma::tc_fence_after();
        const uint32_t sV = umma::smem_u32(sm + stage * Lay::kStage + Lay::kV);
#pragma unroll
        for (int k0 = 0; k0 < 192; k0 += 16)
          umma::mma_ts(tmem + slot * 256 + 192, tmem + slot * 256 + k0 / 2,
                       umma::desc_mnmajor_sw128(sV, k0, 192), id_o, k0 > 0);
        umma::mma_commit(ofull + slot);
        umma::mma_commit(vempty + stage);  // V of this stage may be refilled
        BASED_WP_TRACE(3, k);
      }
      if (!ok) fail();
      umma::mma_commit(bar_fin);
      if (!umma::mbar_wait(bar_fin, 0)) fail();
    }
  } else {
    // ================= softmax groups: tiles k = sg, sg + 2, ... =================
    const int sg = warp >> 2, quad = warp & 3;
    const int r = tid - 128 * sg;  // query row of the tile; TMEM lane
    const uint32_t tm_lane = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t sbase = tmem + sg * 256 + tm_lane;
    uint8_t* ybuf = sm + Lay::kY + sg * 16384;
    const float scale = 0.125f * 1.4426950408889634f;  // 1/sqrt(64) * log2(e)
    for (int k = sg; k < n_mine && !*abort_flag; k += 2) {
      const int j = k >> 1;
      int bh, t0;
      tile_of(k, &bh, &t0);
      if (!umma::mbar_wait(sfull + sg, j & 1)) { fail(); break; }
      BASED_WP_TRACE(0, k);
      umma::tc_fence_after();
      float l_row;
      {
        const int t = t0 + r, cb = quad * 32;
        float sv[96];
        umma::tmem_ld64_32(sbase + cb, sbase + cb + 64, sv);
        // staged column c holds key t0 - 64 + c; row t sees [max(0, t - W + 1), t]
        const int lo = max(max(r + 1, 64 - t0), t - W + 1 - (t0 - 64)) - cb;
        uint32_t pk[48], zero[32];
        l_row = window_band_softmax(sv, lane, lo, W == 64 && t0 >= 64, scale, pk);
#pragma unroll
        for (int e = 0; e < 32; ++e) zero[e] = 0u;
        if (quad == 0) {
          umma::tmem_st32_nowait(sbase, pk);
          umma::tmem_st16_nowait(sbase + 32, pk + 32);
          umma::tmem_st32_nowait(sbase + 48, zero);
          umma::tmem_st16_nowait(sbase + 80, zero);
        } else if (quad == 1) {
          umma::tmem_st16_nowait(sbase, zero);
          umma::tmem_st32_nowait(sbase + 16, pk);
          umma::tmem_st16_nowait(sbase + 48, pk + 32);
          umma::tmem_st32_nowait(sbase + 64, zero);
        } else if (quad == 2) {
          umma::tmem_st32_nowait(sbase, zero);
          umma::tmem_st32_nowait(sbase + 32, pk);
          umma::tmem_st16_nowait(sbase + 64, pk + 32);
          umma::tmem_st16_nowait(sbase + 80, zero);
        } else {
          umma::tmem_st32_nowait(sbase, zero);
          umma::tmem_st16_nowait(sbase + 32, zero);
          umma::tmem_st32_nowait(sbase + 48, pk);
          umma::tmem_st16_nowait(sbase + 80, pk + 32);
        }
        umma::tmem_wait_st();
      }
      umma::tc_fence_before();
      BASED_WP_TRACE(1, k);
      umma::mbar_arrive(pfull + sg);
      if (!umma::mbar_wait(ofull + sg, j & 1)) { fail(); break; }
      BASED_WP_TRACE(2, k);
      umma::tc_fence_after();
      float o[64];
      umma::tmem_ld64(sbase + 192, o);
      umma::tc_fence_before();
      umma::mbar_arrive(tfree + sg);
      // the previous store from this group's staging tile must have read it
      if (r == 0) umma::bulk_wait_read<0>();
      umma::named_sync(1 + sg, 128);
      const float inv = 1.0f / l_row;
      uint8_t* yrow = ybuf + r * 128;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 b2 =
              __floats2bfloat162_rn(o[ch * 8 + 2 * e] * inv, o[ch * 8 + 2 * e + 1] * inv);
          pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        *reinterpret_cast<uint4*>(yrow + ((ch ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      umma::fence_async_smem();
      umma::named_sync(1 + sg, 128);
      BASED_WP_TRACE(3, k);
      if (r == 0) {
        umma::tma_store_3d(&ymap, ybuf, 0, t0, bh);  // rows past L are clipped
        umma::bulk_commit();
      }
    }
    // the last store has read its staging tile (its global writes complete with the grid)
    if (r == 0) umma::bulk_wait_read<0>();
  }
  umma::tc_fence_before();
  __syncthreads();
  // loads the MMA thread never consumed (an aborted run) are waited for (bounded)
  if ((warp == 9 || warp == 10) && lane == 0) {
    const bool is_v = warp == 10;
    for (int k = is_v ? *consumed_v : *consumed; k < issued; ++k) {
      if (is_v && k == 0 && stall_test(kStallWindowV)) continue;  // never issued
      umma::mbar_wait((is_v ? vfull : full) + k % kWpStages, (k / kWpStages) & 1);
    }
  }
  __syncthreads();
  if (warp == 8) umma::tmem_dealloc(tmem, 512);
}

}  // namespace based
