// linattn_bwd_tc.cuh -- gradient of the causal Taylor linear attention on the
// sm_100a tensor cores (bf16 inputs).
//
// Same quadratic form as linattn_bwd.cuh ("Базированная модель, часть 2",
// section "Что за линейное внимание?"; the training views of the based/train
// README all differentiate this map):
//   u'_ts = q_t.k_s / 4,  w_ts = 1 + u' + u'^2/2  (s <= t),
//   N_t = sum_s w_ts v_s,  D_t = sum_s w_ts + eps,  y_t = N_t / D_t,
//   dN_t = dy_t / D_t,  dD_t = -(dy_t . N_t) / D_t^2,
//   e_ts = (dN_t . v_s + dD_t)(1 + u'_ts),
//   dq_t = sum_s e_ts k_s / 4,  dk_s = sum_t e_ts q_t / 4,  dv_s = sum_t w_ts dN_t.
// Every contraction runs on tcgen05 over 128 x 128 tiles of the (t, s) triangle
// with fp32 accumulation in TMEM; the elementwise maps between them (w, e, the
// mask) run on CUDA cores, one thread per TMEM lane, and hand bf16 pairs back
// to TMEM as the A operand of the next MMA:
//
//   kernel Q (one CTA per 128-query tile i):
//     pass 1, key tiles j = 0..i:  U = Q_i K_j^T        (K = 16)
//                                  W = mask(1 + u' + u'^2/2), D += rowsum(W)
//                                  N += W V_j            (K = 128 keys)
//     then dN, dD per query (CUDA cores) -> shared memory and the workspace;
//     pass 2, key tiles j = 0..i:  U = Q_i K_j^T, G = dN_i V_j^T (K = d_v)
//                                  E = mask((G + dD)(1 + u'))
//                                  dQ += E K_j           (N = 16)
//   kernel KV (one CTA per 128-key tile j), query tiles i = j..last, at d_v = 64
//   in two blocks of 64 queries h: U^T = K_j Q_ih^T, G^T = V_j dN_ih^T
//                                  W^T, E^T as above (dD_t from the workspace)
//                                  dV += W^T dN_ih, dK += E^T Q_ih
//
// Operand precision: q, k, v, dy are the bf16 inputs; W, E and dN are rounded
// to bf16 for the MMAs; D, dD, the accumulators and the outputs are fp32.
// Each CTA runs its steps in sequence (issue, wait, CUDA-core map, issue,
// wait); all waits are bounded, and a timeout stops every thread of the CTA
// at the same barrier.
#pragma once

#include "common.cuh"
#include "umma.cuh"

namespace based {

constexpr int kBtT = 128;                     // tile edge (queries and keys)
constexpr int kBtThreads = 160;               // 4 compute warps + 1 MMA-issuing warp

template <int DV>
struct BtLayout {
  static constexpr int kVTile = kBtT * DV * 2;  // [128 x DV] bf16, 128B-swizzled 64-column blocks
  // kernel Q (byte offsets from a 1024-aligned base)
  static constexpr int kQ = 0;                  // Q_i [128 x 16] K-major
  static constexpr int kK = 4096;               // K_j [2][128 x 16] K-major
  static constexpr int kKm = kK + 8192;         // K_j [2][16 x 128] MN-major (dQ's B operand)
  static constexpr int kV = kKm + 8192;         // V_j [2] (TMA)
  static constexpr int kDN = kV + 2 * kVTile;   // dN_i [128 x DV] K-major SW128
  static constexpr int kBarQ = kDN + kVTile;
  static constexpr size_t kSmemQ = kBarQ + 128 + 1024;
  // kernel KV
  static constexpr int kKk = 0;                 // K_j [128 x 16] K-major
  static constexpr int kQk = 4096;              // Q_i [2][128 x 16] K-major
  static constexpr int kQm = kQk + 8192;        // Q_i [2][16 x 128] MN-major (dK's B operand)
  static constexpr int kVk = kQm + 8192;        // V_j (TMA)
  static constexpr int kDNk = kVk + kVTile;     // dN_i [2] (TMA from the workspace)
  static constexpr int kDD = kDNk + 2 * kVTile; // dD_i [2][128] fp32
  static constexpr int kBarK = kDD + 2 * 512;
  static constexpr size_t kSmemK = kBarK + 128 + 1024;
  // TMEM columns (both kernels): U / W, G / E, the d_v accumulator, the 16-wide one
  static constexpr int kTmU = 0, kTmG = 128, kTmAcc = 256, kTmAcc16 = 384;
  // kernel Q takes 256 columns, so two of its CTAs share an SM: pass 1's N
  // accumulates over G's columns (G is only used in pass 2, after N is read),
  // and each pass-2 step's dQ contribution lands in U's columns [64, 80) (free
  // once E is packed into [0, 64)) and is added up in registers
  static constexpr int kQCols = 256, kQTmN = 128, kQTmDq = 64;
  // kernel KV at d_v = 64 takes each query tile in two blocks of kKvQ = 64
  // queries: U^T, G^T of a block (64 columns each), the d_v accumulator and the
  // 16-wide one make 208 columns, so two of its CTAs share an SM; at d_v = 128
  // the accumulator alone is 128 columns and one CTA per SM takes whole tiles
  static constexpr int kKvQ = DV == 64 ? 64 : 128;
  static constexpr int kKvTmU = 0, kKvTmG = kKvQ, kKvTmAcc = 2 * kKvQ, kKvTmAcc16 = 2 * kKvQ + DV;
  static constexpr int kKvCols = kKvTmAcc16 + 16 <= 256 ? 256 : 512;
  static_assert(kV % 1024 == 0 && kDN % 1024 == 0 && kVk % 1024 == 0 && kDNk % 1024 == 0,
                "swizzled tiles need 1024-byte alignment");
};

struct BtParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* dy;
  float* dq;
  float* dk;
  float* dv;
  __nv_bfloat16* ws_dn;  // [BH, L, DV] bf16
  float* ws_dd;          // [BH, L]
  int L;
  int n_tiles;
  int BH;
  float eps;
};

// Row r (16 bf16 = two 16-byte chunks) of a [128 x 16] tile: K-major and
// MN-major (no swizzle) placements.
__device__ __forceinline__ void bt_put_row16(uint8_t* kmaj, uint8_t* mnmaj, int r, uint4 lo,
                                             uint4 hi) {
  uint8_t* a = kmaj + ((r >> 3) * 2) * 128 + (r & 7) * 16;
  *reinterpret_cast<uint4*>(a) = lo;
  *reinterpret_cast<uint4*>(a + 128) = hi;
  if (mnmaj != nullptr) {
    // element (mn = d, k = r) sits at ((d >> 3) * 16 + (r >> 3)) * 128 + (r & 7) * 16 + (d & 7) * 2
    uint8_t* b = mnmaj + (r >> 3) * 128 + (r & 7) * 16;
    *reinterpret_cast<uint4*>(b) = lo;
    *reinterpret_cast<uint4*>(b + 2048) = hi;
  }
}

__device__ __forceinline__ void bt_load_row16(const __nv_bfloat16* base, long long row, int L,
                                              uint4* lo, uint4* hi) {
  if (row < L) {
    const uint4* p = reinterpret_cast<const uint4*>(base + row * kD);
    *lo = p[0];
    *hi = p[1];
  } else {
    *lo = *hi = make_uint4(0, 0, 0, 0);
  }
}

__device__ __forceinline__ uint32_t bt_pack(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// ---------------------------------------------------------------------------
// kernel Q: D, N -> dN, dD (workspace) -> dq
// ---------------------------------------------------------------------------
template <int DV>
__global__ void __launch_bounds__(kBtThreads, DV == 64 ? 2 : 1)
    linattn_bwd_tc_q_kernel(const __grid_constant__ CUtensorMap vmap, const BtParams p) {
  using Lay = BtLayout<DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::kBarQ);
  uint64_t* bar_v = bars;       // [2] V_j landed
  uint64_t* bar_m1 = bars + 2;  // first MMA group of a step done
  uint64_t* bar_m2 = bars + 3;  // second MMA group of a step done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool issuer = warp == 4;
  // a dependent launch: the previous kernel has finished before any global access
  umma::grid_dep_wait();
  umma::grid_dep_launch();
  // the CTAs with the most key tiles (the last query tiles) are launched first,
  // so the short ones fill the end of the grid
  const int i = p.n_tiles - 1 - (int)(blockIdx.x / p.BH);
  const long long bh = blockIdx.x % p.BH;
  const int L = p.L;
  const int t0 = i * kBtT;
  const int n_steps = 2 * (i + 1);
  const __nv_bfloat16* qb = p.q + bh * L * kD;
  const __nv_bfloat16* kb = p.k + bh * L * kD;

  if (tid == 0) {
    umma::mbar_init(bar_v, 1);
    umma::mbar_init(bar_v + 1, 1);
    umma::mbar_init(bar_m1, 1);
    umma::mbar_init(bar_m2, 1);
    umma::fence_mbar_init();
  }
  if (warp == 0) {
    umma::tmem_alloc(tmem_slot, Lay::kQCols);
    umma::tmem_relinquish();
  }
  if (!issuer) {  // Q_i rows
    uint4 lo, hi;
    bt_load_row16(qb, (long long)t0 + tid, L, &lo, &hi);
    bt_put_row16(sm + Lay::kQ, nullptr, tid, lo, hi);
  }
  umma::fence_async_smem();
  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_lane = static_cast<uint32_t>((warp & 3) * 32) << 16;
  // a bounded wait that ran out sets `failed`; every exit decision is taken by
  // __syncthreads_or over it, so all threads leave at the same barrier
  bool failed = false;
  auto fail = [&]() {
    record_device_error(BASED_ERR_TIMEOUT);
    failed = true;
  };
  constexpr uint32_t kVBytes = DV * kBtT * 2;
  auto issue_v = [&](int step) {  // V of key tile (step mod (i + 1)) into buffer step & 1
    const int j = step % (i + 1), b = step & 1;
    umma::mbar_arrive_expect_tx(bar_v + b, kVBytes);
#pragma unroll
    for (int blk = 0; blk < DV / 64; ++blk)
      umma::tma_load_3d(sm + Lay::kV + b * Lay::kVTile + blk * (kBtT * 128), &vmap, bar_v + b,
                        blk * 64, j * kBtT, (int)bh);
  };
  if (issuer && lane == 0) issue_v(0);
  int v_inflight = issuer && lane == 0 ? 1 : 0;  // loads issued and not yet waited for (issuer)

  float dsum = 0.0f;  // D_t (pass 1), then dD_t (pass 2), for query t0 + tid
  float dq_acc[16];   // dQ of this lane's query (pass 2)
#pragma unroll
  for (int c = 0; c < 16; ++c) dq_acc[c] = 0.0f;
  const int row = tid;  // compute threads: query row = TMEM lane
  const uint32_t sQ = umma::smem_u32(sm + Lay::kQ);
  // K rows of the next step, loaded one step ahead of their use
  uint4 klo = make_uint4(0, 0, 0, 0), khi = klo;
  if (!issuer) bt_load_row16(kb, (long long)tid, L, &klo, &khi);
  for (int step = 0; step < n_steps; ++step) {
    const int pass = step / (i + 1), j = step % (i + 1), b = step & 1;
    const bool diag = j == i;
    if (!issuer) {  // K_j rows, both layouts; then the next step's rows
      bt_put_row16(sm + Lay::kK + b * 4096, sm + Lay::kKm + b * 4096, tid, klo, khi);
      umma::fence_async_smem();
      if (step + 1 < n_steps)
        bt_load_row16(kb, (long long)((step + 1) % (i + 1)) * kBtT + tid, L, &klo, &khi);
    }
    if (__syncthreads_or(failed)) break;
    if (issuer && lane == 0) {
      if (!umma::mbar_wait(bar_v + b, (step >> 1) & 1)) {
        fail();
      } else {
        --v_inflight;
        umma::tc_fence_after();
        const uint32_t sK = umma::smem_u32(sm + Lay::kK + b * 4096);
        umma::mma_bf16(tmem + Lay::kTmU, umma::desc_kmajor_none(sQ, 0, 16),
                       umma::desc_kmajor_none(sK, 0, 16), umma::idesc_bf16(128, 128, false, false), 0);
        if (pass == 1) {  // G = dN_i V_j^T
          const uint32_t sD = umma::smem_u32(sm + Lay::kDN);
          const uint32_t sV = umma::smem_u32(sm + Lay::kV + b * Lay::kVTile);
#pragma unroll
          for (int k0 = 0; k0 < DV; k0 += 16)
            umma::mma_bf16(tmem + Lay::kTmG, umma::desc_kmajor_sw128(sD, k0, kBtT),
                           umma::desc_kmajor_sw128(sV, k0, kBtT),
                           umma::idesc_bf16(128, 128, false, false), k0 > 0);
        }
        umma::mma_commit(bar_m1);
        // the next step's V tile goes to the other buffer, whose MMAs (those of
        // the previous step) are complete
        if (step + 1 < n_steps) {
          issue_v(step + 1);
          ++v_inflight;
        }
      }
    }
    // ---- CUDA cores: W (pass 1) or E (pass 2) of this lane's query row ----
    if (!issuer) {
      // warp-uniform outcome: the TMEM loads below are warp-collective
      if (!__all_sync(0xffffffffu, umma::mbar_wait(bar_m1, step & 1))) {
        fail();
      } else {
        umma::tc_fence_after();
        const int lim = diag ? row : kBtT - 1;  // keys j*128 + c with c > lim are masked
#pragma unroll 1
        for (int c32 = 0; c32 < 4; ++c32) {
          float u[32], g[32];
          umma::tmem_ld32(tmem + Lay::kTmU + tm_lane + 32 * c32, u);
          if (pass == 1) umma::tmem_ld32(tmem + Lay::kTmG + tm_lane + 32 * c32, g);
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int c = 32 * c32 + 2 * e + h;
              const float up = 0.25f * u[2 * e + h];
              float val;
              if (pass == 0) {
                val = fmaf(0.5f * up, up, 1.0f + up);  // w
              } else {
                val = (g[2 * e + h] + dsum) * (1.0f + up);  // e
              }
              x[h] = c <= lim ? val : 0.0f;
            }
            if (pass == 0) dsum += x[0] + x[1];
            pk[e] = bt_pack(x[0], x[1]);
          }
          // packed pairs of columns [32 c32, 32 c32 + 32) -> columns [16 c32, 16 c32 + 16),
          // which this thread has read already
          umma::tmem_st16_nowait(tmem + Lay::kTmU + tm_lane + 16 * c32, pk);
        }
        umma::tmem_wait_st();
      }
      umma::tc_fence_before();
    }
    if (__syncthreads_or(failed)) break;
    if (issuer && lane == 0) {
      umma::tc_fence_after();
      if (pass == 0) {  // N += W V_j
        const uint32_t sV = umma::smem_u32(sm + Lay::kV + b * Lay::kVTile);
#pragma unroll
        for (int ks = 0; ks < kBtT / 16; ++ks)
          umma::mma_ts(tmem + Lay::kQTmN, tmem + Lay::kTmU + ks * 8,
                       umma::desc_mnmajor_sw128(sV, ks * 16, kBtT),
                       umma::idesc_bf16(128, DV, false, true), (j > 0 || ks > 0) ? 1u : 0u);
      } else {  // this step's E K_j (added to dQ in registers)
        const uint32_t sKm = umma::smem_u32(sm + Lay::kKm + b * 4096);
#pragma unroll
        for (int ks = 0; ks < kBtT / 16; ++ks)
          umma::mma_ts(tmem + Lay::kQTmDq, tmem + Lay::kTmU + ks * 8,
                       umma::desc_mnmajor_none(sKm, ks * 16, kBtT),
                       umma::idesc_bf16(128, 16, false, true), ks > 0 ? 1u : 0u);
      }
      umma::mma_commit(bar_m2);
    }
    if (!umma::mbar_wait(bar_m2, step & 1)) fail();
    umma::tc_fence_after();
    // this step's dQ contribution (read before the next step's U overwrites it;
    // warp-collective load, so the whole warp decides)
    if (pass == 1 && !issuer && __all_sync(0xffffffffu, !failed)) {
      float tmp[32];
      umma::tmem_ld32(tmem + Lay::kQTmDq + tm_lane, tmp);  // columns 64..95 (16 used)
#pragma unroll
      for (int c = 0; c < 16; ++c) dq_acc[c] += tmp[c];
    }
    umma::tc_fence_before();
    if (__syncthreads_or(failed)) break;
    // ---- end of pass 1: dN and dD of this lane's query ----
    if (pass == 0 && j == i && !issuer) {
      const long long t = (long long)t0 + row;
      const float D = dsum + p.eps;
      // dy row in 8-column pieces (read twice: for dy . N, then for dN), so few
      // registers are live at a time
      const uint4* src = reinterpret_cast<const uint4*>(p.dy + (bh * L + (t < L ? t : 0)) * DV);
      auto dy8 = [&](int c8, float* f8) {
        const uint4 w4 = t < L ? src[c8] : make_uint4(0, 0, 0, 0);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w4);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(h[e]);
          f8[2 * e] = f.x;
          f8[2 * e + 1] = f.y;
        }
      };
      float dot = 0.0f;
#pragma unroll 1
      for (int blk = 0; blk < DV / 64; ++blk) {
        float n[64];
        umma::tmem_ld64(tmem + Lay::kQTmN + tm_lane + 64 * blk, n);
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          float f8[8];
          dy8(blk * 8 + c8, f8);
#pragma unroll
          for (int e = 0; e < 8; ++e) dot = fmaf(f8[e], n[c8 * 8 + e], dot);
        }
      }
      const float invD = 1.0f / D;
      dsum = -dot * invD * invD;  // dD_t
      __nv_bfloat16* wdn = p.ws_dn + (bh * L + t) * DV;
#pragma unroll
      for (int c8 = 0; c8 < DV / 8; ++c8) {
        float f8[8];
        dy8(c8, f8);
        uint4 w4;
        w4.x = bt_pack(f8[0] * invD, f8[1] * invD);
        w4.y = bt_pack(f8[2] * invD, f8[3] * invD);
        w4.z = bt_pack(f8[4] * invD, f8[5] * invD);
        w4.w = bt_pack(f8[6] * invD, f8[7] * invD);
        // K-major, 128-byte swizzle: 64-column blocks of 128 rows x 128 B
        const int blk = c8 >> 3, ch = c8 & 7;
        *reinterpret_cast<uint4*>(sm + Lay::kDN + blk * (kBtT * 128) + row * 128 +
                                  ((ch ^ (row & 7)) << 4)) = w4;
        if (t < L) reinterpret_cast<uint4*>(wdn)[c8] = w4;
      }
      if (t < L) p.ws_dd[bh * L + t] = dsum;
      umma::fence_async_smem();
    }
  }
  const bool any_failed = __syncthreads_or(failed);
  // ---- dq of this lane's query ----
  if (!issuer && !any_failed) {
    const long long t = (long long)t0 + row;
    const float* g = dq_acc;
    if (t < L) {
      float4* dst = reinterpret_cast<float4*>(p.dq + (bh * L + t) * kD);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4)
        dst[c4] = make_float4(0.25f * g[4 * c4], 0.25f * g[4 * c4 + 1], 0.25f * g[4 * c4 + 2],
                              0.25f * g[4 * c4 + 3]);
    }
  }
  umma::tc_fence_before();
  __syncthreads();
  // V loads that an aborted run never waited for (bounded)
  if (issuer && lane == 0 && v_inflight > 0) {
    umma::mbar_wait(bar_v, 0);
    umma::mbar_wait(bar_v + 1, 0);
  }
  __syncthreads();
  if (warp == 0) umma::tmem_dealloc(tmem, Lay::kQCols);
}

// ---------------------------------------------------------------------------
// kernel KV: dk, dv from the workspace (dN bf16, dD fp32)
// ---------------------------------------------------------------------------
template <int DV>
__global__ void __launch_bounds__(kBtThreads, DV == 64 ? 2 : 1)
    linattn_bwd_tc_kv_kernel(const __grid_constant__ CUtensorMap vmap,
                             const __grid_constant__ CUtensorMap dnmap, const BtParams p) {
  using Lay = BtLayout<DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::kBarK);
  uint64_t* bar_dn = bars;      // [2] dN_i landed
  uint64_t* bar_v = bars + 2;   // V_j landed
  uint64_t* bar_m1 = bars + 3;
  uint64_t* bar_m2 = bars + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool issuer = warp == 4;
  // a dependent launch: the previous kernel has finished before any global access
  umma::grid_dep_wait();
  umma::grid_dep_launch();
  // the CTAs with the most query tiles (the first key tiles) are launched first
  const int j = (int)(blockIdx.x / p.BH);
  const long long bh = blockIdx.x % p.BH;
  const int L = p.L;
  const int s0 = j * kBtT;
  const int n_steps = p.n_tiles - j;  // query tiles j .. n_tiles - 1
  const __nv_bfloat16* qb = p.q + bh * L * kD;
  const __nv_bfloat16* kb = p.k + bh * L * kD;

  if (tid == 0) {
    umma::mbar_init(bar_dn, 1);
    umma::mbar_init(bar_dn + 1, 1);
    umma::mbar_init(bar_v, 1);
    umma::mbar_init(bar_m1, 1);
    umma::mbar_init(bar_m2, 1);
    umma::fence_mbar_init();
  }
  if (warp == 0) {
    umma::tmem_alloc(tmem_slot, Lay::kKvCols);
    umma::tmem_relinquish();
  }
  if (!issuer) {  // K_j rows
    uint4 lo, hi;
    bt_load_row16(kb, (long long)s0 + tid, L, &lo, &hi);
    bt_put_row16(sm + Lay::kKk, nullptr, tid, lo, hi);
  }
  umma::fence_async_smem();
  umma::tc_fence_before();
  __syncthreads();
  umma::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_lane = static_cast<uint32_t>((warp & 3) * 32) << 16;
  bool failed = false;  // as in kernel Q: exits are decided by __syncthreads_or
  auto fail = [&]() {
    record_device_error(BASED_ERR_TIMEOUT);
    failed = true;
  };
  constexpr uint32_t kTileBytes = DV * kBtT * 2;
  auto issue_dn = [&](int step) {
    const int b = step & 1, ti = j + step;
    umma::mbar_arrive_expect_tx(bar_dn + b, kTileBytes);
#pragma unroll
    for (int blk = 0; blk < DV / 64; ++blk)
      umma::tma_load_3d(sm + Lay::kDNk + b * Lay::kVTile + blk * (kBtT * 128), &dnmap,
                        bar_dn + b, blk * 64, ti * kBtT, (int)bh);
  };
  int inflight = 0;
  if (issuer && lane == 0) {
    umma::mbar_arrive_expect_tx(bar_v, kTileBytes);
#pragma unroll
    for (int blk = 0; blk < DV / 64; ++blk)
      umma::tma_load_3d(sm + Lay::kVk + blk * (kBtT * 128), &vmap, bar_v, blk * 64, s0, (int)bh);
    issue_dn(0);
    inflight = 2;
    if (!umma::mbar_wait(bar_v, 0)) fail();
    else --inflight;
  }
  const int row = tid;  // compute threads: key row = TMEM lane
  const uint32_t sK = umma::smem_u32(sm + Lay::kKk);
  const uint32_t sV = umma::smem_u32(sm + Lay::kVk);
  // Q rows and dD of the next step, loaded one step ahead of their use
  uint4 qlo = make_uint4(0, 0, 0, 0), qhi = qlo;
  float ddn = 0.0f;
  auto load_q = [&](int ti) {
    const long long t = (long long)ti * kBtT + tid;
    bt_load_row16(qb, t, L, &qlo, &qhi);
    ddn = t < L ? p.ws_dd[bh * L + t] : 0.0f;
  };
  if (!issuer) load_q(j);
  for (int step = 0; step < n_steps; ++step) {
    const int ti = j + step, b = step & 1;
    const bool diag = ti == j;
    if (!issuer) {  // Q_i rows (both layouts) and dD_i; then the next step's
      bt_put_row16(sm + Lay::kQk + b * 4096, sm + Lay::kQm + b * 4096, tid, qlo, qhi);
      reinterpret_cast<float*>(sm + Lay::kDD + b * 512)[tid] = ddn;
      umma::fence_async_smem();
      if (step + 1 < n_steps) load_q(ti + 1);
    }
    if (__syncthreads_or(failed)) break;
    const uint32_t sQ = umma::smem_u32(sm + Lay::kQk + b * 4096);
    const uint32_t sQm = umma::smem_u32(sm + Lay::kQm + b * 4096);
    const uint32_t sD = umma::smem_u32(sm + Lay::kDNk + b * Lay::kVTile);
    // the blocks of kKvQ queries (m1, m2 complete once per block: phase
    // kNQ step + h); a failure stops every thread at the same barrier, in both loops
    constexpr int QW = Lay::kKvQ, kNQ = kBtT / QW;
    bool stop = false;
    for (int h = 0; h < kNQ; ++h) {
      const uint32_t ph = static_cast<uint32_t>(kNQ * step + h) & 1u;
      if (issuer && lane == 0) {
        if (h == 0 && !umma::mbar_wait(bar_dn + b, (step >> 1) & 1)) {
          fail();
        } else {
          if (h == 0) --inflight;
          umma::tc_fence_after();
          // U^T = K_j Q_ih^T: block h's rows of the K-major Q tile start QW h / 8
          // core matrix rows (256 B each) in; G^T = V_j dN_ih^T: they start QW h
          // rows (128 B each) into each 64-column block of dN
          umma::mma_bf16(tmem + Lay::kKvTmU, umma::desc_kmajor_none(sK, 0, 16),
                         umma::desc_kmajor_none(sQ + 32u * QW * h, 0, 16),
                         umma::idesc_bf16(128, QW, false, false), 0);
#pragma unroll
          for (int k0 = 0; k0 < DV; k0 += 16)
            umma::mma_bf16(tmem + Lay::kKvTmG, umma::desc_kmajor_sw128(sV, k0, kBtT),
                           umma::desc_kmajor_sw128(sD + 128u * QW * h, k0, kBtT),
                           umma::idesc_bf16(128, QW, false, false), k0 > 0);
          umma::mma_commit(bar_m1);
          // the next step's dN tile goes to the other buffer (the previous step's
          // MMAs are complete)
          if (h == 0 && step + 1 < n_steps) {
            issue_dn(step + 1);
            ++inflight;
          }
        }
      }
      if (!issuer) {
        if (!__all_sync(0xffffffffu, umma::mbar_wait(bar_m1, ph))) {
          fail();
        } else {
          umma::tc_fence_after();
          const float* dd = reinterpret_cast<const float*>(sm + Lay::kDD + b * 512) + QW * h;
          // queries ti*128 + QW h + c with c < lo_c come before key s
          const int lo_c = diag ? row - QW * h : 0;
#pragma unroll 1
          for (int c32 = 0; c32 < QW / 32; ++c32) {
            float u[32], g[32];
            umma::tmem_ld32(tmem + Lay::kKvTmU + tm_lane + 32 * c32, u);
            umma::tmem_ld32(tmem + Lay::kKvTmG + tm_lane + 32 * c32, g);
            uint32_t pw[16], pe[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              float w2[2], e2[2];
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                const int c = 32 * c32 + 2 * e + hh;
                const float up = 0.25f * u[2 * e + hh];
                const bool live = c >= lo_c;
                w2[hh] = live ? fmaf(0.5f * up, up, 1.0f + up) : 0.0f;
                e2[hh] = live ? (g[2 * e + hh] + dd[c]) * (1.0f + up) : 0.0f;
              }
              pw[e] = bt_pack(w2[0], w2[1]);
              pe[e] = bt_pack(e2[0], e2[1]);
            }
            // W^T pairs over U^T's columns [16 c32, +16), E^T pairs over G^T's
            umma::tmem_st16_nowait(tmem + Lay::kKvTmU + tm_lane + 16 * c32, pw);
            umma::tmem_st16_nowait(tmem + Lay::kKvTmG + tm_lane + 16 * c32, pe);
          }
          umma::tmem_wait_st();
        }
        umma::tc_fence_before();
      }
      if (__syncthreads_or(failed)) {
        stop = true;
        break;
      }
      if (issuer && lane == 0) {
        umma::tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < QW / 16; ++ks) {
          const uint32_t acc = (step > 0 || h > 0 || ks > 0) ? 1u : 0u;
          const int kq = QW * h + 16 * ks;  // query (K) index within the tile
          umma::mma_ts(tmem + Lay::kKvTmAcc, tmem + Lay::kKvTmU + ks * 8,
                       umma::desc_mnmajor_sw128(sD, kq, kBtT),
                       umma::idesc_bf16(128, DV, false, true), acc);  // dV += W^T dN_ih
          umma::mma_ts(tmem + Lay::kKvTmAcc16, tmem + Lay::kKvTmG + ks * 8,
                       umma::desc_mnmajor_none(sQm, kq, kBtT),
                       umma::idesc_bf16(128, 16, false, true), acc);  // dK += E^T Q_ih
        }
        umma::mma_commit(bar_m2);
      }
      if (!umma::mbar_wait(bar_m2, ph)) fail();
      umma::tc_fence_after();
    }
    if (stop) break;
  }
  const bool any_failed = __syncthreads_or(failed);
  // ---- dk, dv of this lane's key (TMEM loads by whole warps, stores by live rows) ----
  if (!issuer && !any_failed) {
    const long long s = (long long)s0 + row;
    const bool live = s < L;
    float4* dvd = reinterpret_cast<float4*>(p.dv + (bh * L + s) * DV);
#pragma unroll
    for (int blk = 0; blk < DV / 64; ++blk) {
      float a[64];
      umma::tmem_ld64(tmem + Lay::kKvTmAcc + tm_lane + 64 * blk, a);
      if (live) {
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4)
          dvd[16 * blk + c4] = make_float4(a[4 * c4], a[4 * c4 + 1], a[4 * c4 + 2], a[4 * c4 + 3]);
      }
    }
    float g[32];
    umma::tmem_ld32(tmem + Lay::kKvTmAcc16 + tm_lane, g);
    if (live) {
      float4* dkd = reinterpret_cast<float4*>(p.dk + (bh * L + s) * kD);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4)
        dkd[c4] = make_float4(0.25f * g[4 * c4], 0.25f * g[4 * c4 + 1], 0.25f * g[4 * c4 + 2],
                              0.25f * g[4 * c4 + 3]);
    }
  }
  umma::tc_fence_before();
  __syncthreads();
  if (issuer && lane == 0 && inflight > 0) {  // loads an aborted run never waited for
    umma::mbar_wait(bar_dn, 0);
    umma::mbar_wait(bar_dn + 1, 0);
    umma::mbar_wait(bar_v, 0);
  }
  __syncthreads();
  if (warp == 0) umma::tmem_dealloc(tmem, Lay::kKvCols);
}

}  // namespace based
