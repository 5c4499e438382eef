// window_softmax.cuh -- the band softmax of one query row, shared by the
// tensor-core window-attention kernels (window_tcp.cuh, d_head = 64, and
// window_tc.cuh, d_head = 128).
//
// Based README, introduction, item 1: softmax over the keys of a sliding
// window.  A thread holds 96 scores of its query row (TMEM columns cb..cb+95 of
// the 192 staged keys, cb = 32 x its lane quadrant); its window is the columns
// [lo, lane + 64].  The weights are exp2(s * scale - max), scale = log2(e) /
// sqrt(d_head) (ex2.approx, rounded to bf16 next), and the row sum comes back
// for the normalisation after P V.
#pragma once

#include "common.cuh"

namespace based {

// sv: the 96 scores (overwritten); full: every row of the tile has a whole
// window of 64 keys (W = 64 and t0 >= 64), in which case columns 32..64 lie
// inside the window of every lane and lo = lane + 1; pk: the 96 weights as bf16
// pairs (keys 2j, 2j+1 in pk[j]), zero outside the window.  Returns the row sum.
__device__ __forceinline__ float window_band_softmax(float (&sv)[96], int lane, int lo, bool full,
                                                     float scale, uint32_t (&pk)[48]) {
  // keys outside the window become -inf once, so the max and the exponentials
  // need no mask (exp2(-inf) = 0)
  if (full) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i <= lane) sv[i] = -INFINITY;
#pragma unroll
    for (int i = 65; i < 96; ++i)
      if (i > lane + 64) sv[i] = -INFINITY;
  } else {
#pragma unroll
    for (int i = 0; i < 96; ++i)
      if (i < lo || i > lane + 64) sv[i] = -INFINITY;
  }
  // four interleaved partial maxima / sums keep the dependent chains short
  float mp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int i = 0; i < 96; ++i) mp[i & 3] = fmaxf(mp[i & 3], sv[i]);
  const float ms = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])) * scale;
  // s * scale - ms and the partial sums as packed pairs (each lane of the f32x2
  // forms rounds like its scalar form); pair j feeds partial sums (j & 1) * 2 + {0, 1}
  uint64_t sc2, nm2, lp2[2];
  asm("mov.b64 %0, {%1, %1};" : "=l"(sc2) : "f"(scale));
  asm("mov.b64 %0, {%1, %1};" : "=l"(nm2) : "f"(-ms));
  asm("mov.b64 %0, {%1, %1};" : "=l"(lp2[0]) : "f"(0.0f));
  lp2[1] = lp2[0];
#pragma unroll
  for (int j = 0; j < 48; ++j) {
    uint64_t x2, e2;
    float a, b;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x2) : "f"(sv[2 * j]), "f"(sv[2 * j + 1]));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(x2) : "l"(x2), "l"(sc2), "l"(nm2));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(x2));
    a = ex2_approx(a);
    b = ex2_approx(b);
    asm("mov.b64 %0, {%1, %2};" : "=l"(e2) : "f"(a), "f"(b));
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(lp2[j & 1]) : "l"(lp2[j & 1]), "l"(e2));
    const __nv_bfloat162 b2 = __floats2bfloat162_rn(a, b);
    pk[j] = *reinterpret_cast<const uint32_t*>(&b2);
  }
  float lq[4];
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lq[0]), "=f"(lq[1]) : "l"(lp2[0]));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lq[2]), "=f"(lq[3]) : "l"(lp2[1]));
  return (lq[0] + lq[1]) + (lq[2] + lq[3]);  // >= 1: the row maximum contributes exp2(0)
}

}  // namespace based
