// window_tc.cuh -- sliding-window causal softmax attention on the sm_100a tensor cores.
//
// Based README, introduction, item 1: exact softmax attention over a short
// sliding window (size 64) models the fine-grained local interactions.  For
// query t the keys are s in [max(0, t-W+1), t] (W <= 64), scores q_t.k_s/sqrt(dh).
//
// One CTA per tile of 128 queries [t0, t0+128) of one (b, h).  The keys any of
// its queries can see lie in [t0-63, t0+127]; the CTA loads the 192 rows
// [t0-64, t0+128) of K and V by TMA (rows before 0 or past L read as zero) and
//   S = Q K^T        tcgen05, M=128, N=192, K=dh            -> TMEM (fp32)
//   P = exp(S - m)   CUDA cores: thread r owns query row r; it reads the 96
//                    TMEM columns covering its 64-key band, masks, takes the exact
//                    row max, exponentiates, keeps the row sum l in a register
//                    and writes P (bf16 pairs, zero outside the band) back over
//                    S in its own TMEM lane
//   O = P V          tcgen05, A = P from TMEM, M=128, N=dh, K=192 -> TMEM (fp32)
//   y = O / l        CUDA cores: TMEM -> 128B-swizzled staging tile -> TMA store.
// Keeping P in TMEM spares the tensor core the P reads.  Two CTAs share an SM:
// V is loaded over Q and K once S is complete (its load overlaps the softmax,
// and the other CTA's work), the y staging tile goes over V once O is complete,
// and O takes the TMEM columns of S that P no longer needs, so a CTA holds
// 32 + 48 KiB of shared memory and 256 TMEM columns at d_h = 128.
#pragma once

#include "common.cuh"
#include "umma.cuh"
#include "window_softmax.cuh"

namespace based {

constexpr int kWtQ = 128;      // queries per CTA
constexpr int kWtKeys = 192;   // staged key rows per CTA
constexpr int kWtThreads = 128;

template <int DH>
struct WtLayout {
  static constexpr int kQ = 0;                              // Q [128 x DH] K-major SW128
  static constexpr int kK = kQ + kWtQ * DH * 2;             // K [192 x DH] K-major SW128
  static constexpr int kV = 0;                              // V [192 x DH] MN-major SW128 (over Q, K)
  static constexpr int kY = 0;                              // y [128 x DH] bf16 SW128 (over V)
  static constexpr int kBar = kK + kWtKeys * DH * 2;
  static constexpr int kBytes = kBar + 64;
  static constexpr size_t kSmem = kBytes + 1024;
  static_assert(kWtKeys * DH * 2 <= kBar, "V fits over Q and K");
  // S in columns [0, 192); P (bf16 pairs) in [0, 96); O over the rest of S
  static constexpr int kTmS = 0;
  static constexpr int kTmO = kWtKeys / 2;
  static constexpr int kTmemCols = 256;
  static_assert(kTmO + DH <= kTmemCols, "TMEM budget");
};

template <int DH>
__global__ void __launch_bounds__(kWtThreads, 1)
    window_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                     const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap,
                     const __grid_constant__ CUtensorMap ymap, int L, int W, int n_tiles) {
  using Lay = WtLayout<DH>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + Lay::kBar);  // Q and K landed
  uint64_t* bar_s = bar_tma + 1;
  uint64_t* bar_o = bar_tma + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_tma + 3);
  int* abort_flag = reinterpret_cast<int*>(bar_tma + 4);
  uint64_t* bar_v = bar_tma + 5;                                      // V landed

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // a dependent launch: the previous kernel has finished before any load
  umma::grid_dep_wait();
  umma::grid_dep_launch();
  const int tile = blockIdx.x % n_tiles;
  const int bh = blockIdx.x / n_tiles;
  const int t0 = tile * kWtQ;

  // Q and K first (S needs them); V over them once S is complete
  bool v_issued = false;  // thread 0
  if (tid == 0) {
    umma::mbar_init(bar_tma, 1);
    umma::mbar_init(bar_v, 1);
    umma::mbar_init(bar_s, 1);
    umma::mbar_init(bar_o, 1);
    *abort_flag = 0;
    umma::fence_mbar_init();
    umma::mbar_arrive_expect_tx(bar_tma, (kWtQ + kWtKeys) * DH * 2);
#pragma unroll
    for (int b = 0; b < DH / 64; ++b) {
      umma::tma_load_3d(sm + Lay::kQ + b * kWtQ * 128, &qmap, bar_tma, b * 64, t0, bh);
      umma::tma_load_3d(sm + Lay::kK + b * kWtKeys * 128, &kmap, bar_tma, b * 64, t0 - 64, bh);
    }
  }
  __syncthreads();  // barrier initialisation visible to every thread
  // TMEM is taken only once Q and K have landed: a CTA that still waits for
  // its loads holds none, so the TMEM of the SM serves the CTAs that compute
  // while further CTAs' loads are in flight
  {
    const bool ok = umma::mbar_wait(bar_tma, 0);
    if (!ok && tid == 0) {
      record_device_error(BASED_ERR_TIMEOUT);
      *abort_flag = 1;
    }
  }
  if (warp == 0) {
    umma::tmem_alloc(tmem_slot, Lay::kTmemCols);
    umma::tmem_relinquish();
  }
  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_lane = static_cast<uint32_t>(warp * 32) << 16;
  const uint32_t sQ = umma::smem_u32(sm + Lay::kQ), sK = umma::smem_u32(sm + Lay::kK),
                 sV = umma::smem_u32(sm + Lay::kV);

  // ---- S = Q K^T ----------------------------------------------------------------
  if (tid == 0) {
    if (!*abort_flag) {
      umma::tc_fence_after();
      const uint32_t id = umma::idesc_bf16(kWtQ, kWtKeys, false, false);
#pragma unroll
      for (int k0 = 0; k0 < DH; k0 += 16)
        umma::mma_bf16(tmem + Lay::kTmS, umma::desc_kmajor_sw128(sQ, k0, kWtQ),
                       umma::desc_kmajor_sw128(sK, k0, kWtKeys), id, k0 > 0);
      umma::mma_commit(bar_s);
    }
  }
  __syncthreads();
  if (*abort_flag) goto done;
  if (!umma::mbar_wait(bar_s, 0)) {
    record_device_error(BASED_ERR_TIMEOUT);
    *abort_flag = 1;
  }
  umma::tc_fence_after();
  // S is complete, so its operands are no longer read: V goes over Q and K
  // (the stall test leaves the V tile out)
  if (tid == 0 && !*abort_flag && !stall_test(kStallWindowV)) {
    umma::mbar_arrive_expect_tx(bar_v, kWtKeys * DH * 2);
#pragma unroll
    for (int b = 0; b < DH / 64; ++b)
      umma::tma_load_3d(sm + Lay::kV + b * kWtKeys * 128, &vmap, bar_v, b * 64, t0 - 64, bh);
    v_issued = true;
  }

  // ---- P = exp(S - m) over each row's band ---------------------------------------------
  // Row r = 32 w + lane (w = warp) reads the 96 staged columns [32 w, 32 w + 96);
  // relative to that base its band is [lo, lane + 64] (lo = lane + 1 away from
  // the sequence start and for W = 64).  Rows past L see zero-filled Q, so their
  // scores are finite and their output is simply not stored.
  float l_row;
  {
    const int r = tid, t = t0 + r;
    const int cb = warp * 32;
    float sv[96];
    umma::tmem_ld64_32(tmem + Lay::kTmS + tm_lane + cb, tmem + Lay::kTmS + tm_lane + cb + 64, sv);
    // staged column c holds key s = t0 - 64 + c; row t sees s in [max(0, t-W+1), t]
    const int lo = max(max(r + 1, 64 - t0), t - W + 1 - (t0 - 64)) - cb;
    const float scale = rsqrtf((float)DH) * 1.4426950408889634f;  // 1/sqrt(dh) * log2(e)
    // P (bf16 pairs, column j = keys 2j, 2j+1) replaces S in this lane: the band
    // of quadrant w lands in columns [16w, 16w + 48), the rest of [0, 96) is zero
    uint32_t pk[48], zero[32];
    l_row = window_band_softmax(sv, lane, lo, W == 64 && t0 >= 64, scale, pk);
#pragma unroll
    for (int j = 0; j < 32; ++j) zero[j] = 0u;
    const uint32_t prow = tmem + Lay::kTmS + tm_lane;
    if (warp == 0) {
      umma::tmem_st32_nowait(prow, pk);
      umma::tmem_st16_nowait(prow + 32, pk + 32);
      umma::tmem_st32_nowait(prow + 48, zero);
      umma::tmem_st16_nowait(prow + 80, zero);
    } else if (warp == 1) {
      umma::tmem_st16_nowait(prow, zero);
      umma::tmem_st32_nowait(prow + 16, pk);
      umma::tmem_st16_nowait(prow + 48, pk + 32);
      umma::tmem_st32_nowait(prow + 64, zero);
    } else if (warp == 2) {
      umma::tmem_st32_nowait(prow, zero);
      umma::tmem_st32_nowait(prow + 32, pk);
      umma::tmem_st16_nowait(prow + 64, pk + 32);
      umma::tmem_st16_nowait(prow + 80, zero);
    } else {
      umma::tmem_st32_nowait(prow, zero);
      umma::tmem_st16_nowait(prow + 32, zero);
      umma::tmem_st32_nowait(prow + 48, pk);
      umma::tmem_st16_nowait(prow + 80, pk + 32);
    }
    umma::tmem_wait_st();
  }
  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  if (*abort_flag) goto done;

  // ---- O = P V --------------------------------------------------------------------------
  if (tid == 0) {
    if (!umma::mbar_wait(bar_v, 0)) {
      record_device_error(BASED_ERR_TIMEOUT);
      *abort_flag = 1;
    }
  }
  __syncthreads();
  if (*abort_flag) goto done;
  if (tid == 0) {
    const uint32_t id = umma::idesc_bf16(kWtQ, DH, false, true);
#pragma unroll
    for (int k0 = 0; k0 < kWtKeys; k0 += 16)
      umma::mma_ts(tmem + Lay::kTmO, tmem + Lay::kTmS + k0 / 2,
                   umma::desc_mnmajor_sw128(sV, k0, kWtKeys), id, k0 > 0);
    umma::mma_commit(bar_o);
  }
  __syncwarp();
  {
    const bool ok = umma::mbar_wait(bar_o, 0);
    if (!ok) record_device_error(BASED_ERR_TIMEOUT);
    umma::tc_fence_after();
    if (__syncthreads_or(!ok)) goto done;
  }
  // ---- y = O / l, staged over P (128B-swizzled rows) and stored by TMA ------------------
  {
    const int r = tid;
    const float inv = 1.0f / l_row;
#pragma unroll
    for (int blk = 0; blk < DH / 64; ++blk) {
      float o[64];
      umma::tmem_ld64(tmem + Lay::kTmO + tm_lane + blk * 64, o);
      uint8_t* yrow = sm + Lay::kY + blk * (kWtQ * 128) + r * 128;
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
    }
    umma::fence_async_smem();
  }
  __syncthreads();
  if (tid == 0) {
    // rows past L are clipped by the tensor map
#pragma unroll
    for (int b = 0; b < DH / 64; ++b)
      umma::tma_store_3d(&ymap, sm + Lay::kY + b * kWtQ * 128, b * 64, t0, bh);
    umma::bulk_commit();
    umma::bulk_wait_read<0>();
  }
done:
  // an aborted tile may still have its loads in flight: wait for them (bounded)
  if (tid == 0 && *abort_flag) {
    umma::mbar_wait(bar_tma, 0);
    if (v_issued) umma::mbar_wait(bar_v, 0);
  }
  umma::tc_fence_before();
  __syncthreads();
  if (warp == 0) umma::tmem_dealloc(tmem, Lay::kTmemCols);
}

}  // namespace based
