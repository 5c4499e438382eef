// decode.cuh -- one-token decode step: linear-attention state update + read-out,
// and the sliding-window ring-cache attention, in one launch.
//
// Linear part ("Базированная модель, часть 2", paragraph on the KV state for the
// numerator and the K state for the denominator): per (b, h)
//     S += phi(k) v^T ;  z += phi(k) ;  y = phi(q)^T S / (phi(q) . z + eps).
// The 273 x d_v fp32 state is read once and written once per step, so the step
// is bound by HBM bandwidth: every thread streams whole float4 columns of S with
// 128-bit coalesced loads/stores (a warp covers two contiguous 256-byte rows for
// d_v = 64), issues all its loads before any arithmetic, and the read-out is
// reduced across row slots through shared memory and across warps by shuffles.
//
// Window part (Based README, introduction, item 1: short sliding-window softmax
// attention): the new k/v go to ring slot pos mod W, then softmax over the slots
// holding positions max(0, pos-W+1)..pos.  A window CTA serves up to G heads:
// it issues one bulk copy per ring (the valid rows of one (b, h) ring are
// contiguous) for all its heads at once, so the ring reads overlap each other
// and the linear CTAs' state streaming; window CTAs are spread evenly through
// the grid among the linear ones.
#pragma once

#include "common.cuh"
#include "umma.cuh"

namespace based {

struct DecodeParams {
  const void *q, *k, *v;
  float *S, *z;
  void* out;
  const void *wq, *wk, *wv;
  void *k_ring, *v_ring, *wout;
  long long pos;
  const long long* pos_arr;  // [B] per-sequence positions (device), or null: pos for all
  int H_w;     // window heads per sequence (window item i belongs to sequence i / H_w)
  int n_lin;   // B * H   (one CTA each)
  int n_win;   // B * H_w window heads
  int n_wblk;  // window CTAs, each serving up to wg heads
  int wg;
  int wstride;  // (n_lin + n_wblk) / n_wblk: spacing of the window CTAs
  int dh, W;
  float eps;
};

template <int DV>
struct DecodeLinearLayout {
  static constexpr int kThreads = 4 * DV;
  static constexpr int kColGroups = DV / 4;                 // float4 groups per row
  static constexpr int kRowSlots = kThreads / kColGroups;   // 16
  static constexpr int kRowsPerThread = (kF + kRowSlots - 1) / kRowSlots;  // 18
  static constexpr int kFPad = 276;
  // fq, fk, v, per-row-slot partial sums, per-warp partial denominators, x_q, x_k
  static constexpr int kSmemFloats = 2 * kFPad + DV + kRowSlots * DV + 32 + 32;
};

template <typename T, int DV>
__device__ __forceinline__ void decode_linear_block(const DecodeParams& p, int bh, float* smem) {
  using Lay = DecodeLinearLayout<DV>;
  constexpr int NT = Lay::kThreads, CG = Lay::kColGroups, RS = Lay::kRowSlots,
                NR = Lay::kRowsPerThread;
  float* fq = smem;
  float* fk = fq + Lay::kFPad;
  float* vs = fk + Lay::kFPad;
  float* red = vs + DV;
  float* dred = red + RS * DV;
  float* xq = dred + 32;
  float* xk = xq + 16;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cg = tid % CG, rs = tid / CG;

  // Issue the whole state slice of this thread first: the loads stay in flight
  // while the feature vectors are built.
  float4* S4 = reinterpret_cast<float4*>(p.S + (size_t)bh * kF * DV);
  float4 sv[NR];
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    const int r = rs + i * RS;
    if (r < kF) sv[i] = S4[r * CG + cg];
  }
  float* zb = p.z + (size_t)bh * kF;
  float zv[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int f = tid + i * NT;
    zv[i] = f < kF ? zb[f] : 0.0f;
  }

  const T* q = static_cast<const T*>(p.q) + (size_t)bh * kD;
  const T* k = static_cast<const T*>(p.k) + (size_t)bh * kD;
  const T* v = static_cast<const T*>(p.v) + (size_t)bh * DV;
  if (tid < kD) xq[tid] = to_f32(q[tid]);
  else if (tid < 2 * kD) xk[tid - kD] = to_f32(k[tid - kD]);
  if (tid < DV) vs[tid] = to_f32(v[tid]);
  __syncthreads();
  for (int f = tid; f < kF; f += NT) {
    fq[f] = phi_feature(xq, f);
    fk[f] = phi_feature(xk, f);
  }
  __syncthreads();

  const float4 vv = reinterpret_cast<const float4*>(vs)[cg];
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < NR; ++i) {
    const int r = rs + i * RS;
    if (r < kF) {
      const float a = fk[r], b = fq[r];
      float4 s = sv[i];
      s.x = fmaf(a, vv.x, s.x);
      s.y = fmaf(a, vv.y, s.y);
      s.z = fmaf(a, vv.z, s.z);
      s.w = fmaf(a, vv.w, s.w);
      S4[r * CG + cg] = s;
      acc.x = fmaf(b, s.x, acc.x);
      acc.y = fmaf(b, s.y, acc.y);
      acc.z = fmaf(b, s.z, acc.z);
      acc.w = fmaf(b, s.w, acc.w);
    }
  }
  float dpart = 0.0f;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int f = tid + i * NT;
    if (f < kF) {
      const float zn = zv[i] + fk[f];
      zb[f] = zn;
      dpart = fmaf(fq[f], zn, dpart);
    }
  }
  dpart = warp_sum(dpart);
  if (lane == 0) dred[warp] = dpart;
  reinterpret_cast<float4*>(red)[rs * CG + cg] = acc;
  __syncthreads();
  if (tid < DV) {
    float num = 0.0f;
#pragma unroll
    for (int r = 0; r < RS; ++r) num += red[r * DV + tid];
    float den = 0.0f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) den += dred[w];
    static_cast<T*>(p.out)[(size_t)bh * DV + tid] = from_f32<T>(num / (den + p.eps));
  }
}

// Shared-memory layout of a window CTA (bytes), for G heads of d_h = dh and
// element size es: the K and V rings of each head (W rows), one mbarrier per
// head, then q and the new k/v of each head, the weights and the reductions.
struct DecodeWindowLayout {
  int ring, bar, qs, kvn, pr, red, bytes;
  __host__ __device__ DecodeWindowLayout(int G, int dh, int W, int NT, int es) {
    (void)NT;
    ring = W * dh * es;  // one ring; multiple of 16 for dh in {64, 128}
    bar = 2 * G * ring;
    qs = bar + 8 * G + 16;
    kvn = qs + 4 * G * dh;
    pr = kvn + ((2 * G * dh * es + 15) & ~15);
    red = pr + 4 * 64 * G;
    bytes = red + 4 * 4 * G;
  }
};

// 16 bytes of T at p (16-byte aligned) as floats
template <typename T>
__device__ __forceinline__ void load16_f32(const T* p, float* f);
template <>
__device__ __forceinline__ void load16_f32<float>(const float* p, float* f) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
template <>
__device__ __forceinline__ void load16_f32<__nv_bfloat16>(const __nv_bfloat16* p, float* f) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// The G heads of a window CTA run side by side, 64 threads each (thread s owns
// ring slot s for the scores and value columns s, s+64, ... for the output), so
// the CTA needs four block barriers in all, whatever G.
template <typename T>
__device__ __forceinline__ void decode_window_block(const DecodeParams& p, int wblk, uint8_t* sm) {
  constexpr int VEC = 16 / sizeof(T);
  const int dh = p.dh, W = p.W, NT = blockDim.x, G = p.wg;
  const int tid = threadIdx.x, lane = tid & 31;
  const int w0 = wblk * G;
  const int n_items = min(G, p.n_win - w0);
  const DecodeWindowLayout lay(G, dh, W, NT, sizeof(T));
  T* rings = reinterpret_cast<T*>(sm);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + lay.bar);
  float* qs = reinterpret_cast<float*>(sm + lay.qs);
  T* kvn = reinterpret_cast<T*>(sm + lay.kvn);
  float* pr = reinterpret_cast<float*>(sm + lay.pr);
  float* red = reinterpret_cast<float*>(sm + lay.red);
  // position of window item i: its sequence's entry of pos_arr, or the shared pos
  auto pos_of = [&](int i) -> long long {
    return p.pos_arr != nullptr ? p.pos_arr[(w0 + i) / p.H_w] : p.pos;
  };
  T* kring = static_cast<T*>(p.k_ring);
  T* vring = static_cast<T*>(p.v_ring);

  if (tid == 0) {
    for (int g = 0; g < n_items; ++g) umma::mbar_init(bar + g, 1);
    umma::fence_mbar_init();
    for (int g = 0; g < n_items; ++g) {
      const long long pg = pos_of(g);
      if (pg < 0) {  // a negative position is refused: nothing of this item is touched
        record_device_error(BASED_ERR_INVALID_ARG);
        umma::mbar_arrive(bar + g);
        continue;
      }
      const int nv = pg + 1 < W ? (int)(pg + 1) : W;  // valid slots are 0..nv-1
      const uint32_t load_bytes = (uint32_t)(nv * dh * sizeof(T));
      const size_t ro = (size_t)(w0 + g) * W * dh;
      T* dst = rings + (size_t)g * 2 * W * dh;
      umma::mbar_arrive_expect_tx(bar + g, 2 * load_bytes);
      umma::bulk_load(dst, kring + ro, load_bytes, bar + g);
      umma::bulk_load(dst + W * dh, vring + ro, load_bytes, bar + g);
    }
  }
  for (int i = tid; i < n_items * dh; i += NT) {
    const size_t gi = (size_t)w0 * dh + i;
    qs[i] = to_f32(static_cast<const T*>(p.wq)[gi]);
    kvn[2 * i] = static_cast<const T*>(p.wk)[gi];
    kvn[2 * i + 1] = static_cast<const T*>(p.wv)[gi];
  }
  __syncthreads();

  const int g = tid >> 6, s = tid & 63;  // head and slot / column of this thread
  const long long pos = g < n_items ? pos_of(g) : 0;
  const bool active = g < n_items && pos >= 0;
  const int slot = active ? (int)(pos % W) : 0;
  const int nvalid = !active ? 0 : (pos + 1 < W ? (int)(pos + 1) : W);  // valid slots 0..nvalid-1
  T* K = rings + (size_t)g * 2 * W * dh;
  T* V = K + W * dh;
  bool ok = true;
  if (active) {
    ok = umma::mbar_wait(bar + g, 0);
    if (!ok) record_device_error(BASED_ERR_TIMEOUT);
  }
  // every head's loads must be complete (or abandoned) before any thread leaves
  if (__syncthreads_or(!ok)) {
    if (tid == 0)
      for (int i = 0; i < n_items; ++i) umma::mbar_wait(bar + i, 0);
    return;
  }
  if (active) {
    // the new k/v into slot pos mod W, in shared memory and in the ring
    for (int c = s; c < dh; c += 64) {
      const T kt = kvn[2 * (g * dh + c)], vt = kvn[2 * (g * dh + c) + 1];
      const size_t ro = (size_t)(w0 + g) * W * dh + (size_t)slot * dh + c;
      K[slot * dh + c] = kt;
      V[slot * dh + c] = vt;
      kring[ro] = kt;
      vring[ro] = vt;
    }
  }
  __syncthreads();
  // score of slot s: 16-byte chunks taken in an order rotated by s, so the eight
  // lanes of a shared-memory phase touch eight different bank groups
  float a = -INFINITY;
  if (active && s < nvalid) {
    const int nch = dh / VEC;
    const T* kr = K + s * dh;
    const float* qg = qs + g * dh;
    float acc = 0.0f;
    for (int c = 0; c < nch; ++c) {
      const int ch = (c + s) & (nch - 1);
      float kf[VEC];
      load16_f32<T>(kr + ch * VEC, kf);
#pragma unroll
      for (int i = 0; i < VEC; ++i) acc = fmaf(qg[ch * VEC + i], kf[i], acc);
    }
    a = acc * rsqrtf((float)dh);
  }
  // softmax over the head's 64 slots (two warps)
  const int hw = (tid >> 5) & 1;  // warp within the head
  float m = warp_max(a);
  if (active && lane == 0) red[g * 4 + hw] = m;
  __syncthreads();
  if (active) m = fmaxf(red[g * 4], red[g * 4 + 1]);
  const float e = (active && s < nvalid) ? expf(a - m) : 0.0f;
  if (active) pr[g * 64 + s] = e;
  const float es = warp_sum(e);
  if (active && lane == 0) red[g * 4 + 2 + hw] = es;
  __syncthreads();
  if (active) {
    const float inv = 1.0f / (red[g * 4 + 2] + red[g * 4 + 3]);
    const float* pw = pr + g * 64;
    for (int c = s; c < dh; c += 64) {
      float acc = 0.0f;
      for (int j = 0; j < nvalid; ++j) acc = fmaf(pw[j], to_f32(V[j * dh + c]), acc);
      static_cast<T*>(p.wout)[(size_t)(w0 + g) * dh + c] = from_f32<T>(acc * inv);
    }
  }
}

template <typename T, int DV>
__global__ void __launch_bounds__(4 * DV, 1) decode_step_kernel(const DecodeParams p) {
  extern __shared__ __align__(16) uint8_t dec_smem[];
  // a dependent launch: the previous step's kernel has finished (and its state
  // and ring writes are visible) before this one reads them
  umma::grid_dep_wait();
  umma::grid_dep_launch();
  // window CTAs are interleaved evenly: with stride = n / n_wblk, CTA b is a
  // window CTA iff b mod stride = stride - 1 and b / stride < n_wblk
  const int b = blockIdx.x, q = b / p.wstride, r = b - q * p.wstride;
  if (q < p.n_wblk && r == p.wstride - 1) decode_window_block<T>(p, q, dec_smem);
  else decode_linear_block<T, DV>(p, b - min(q, p.n_wblk), reinterpret_cast<float*>(dec_smem));
}

}  // namespace based
