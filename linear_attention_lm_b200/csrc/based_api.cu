// based_api.cu -- the extern "C" entry points declared in include/based.h.
//
// Host code only validates arguments, picks the kernel for the dtype/shape and
// launches it on the caller's stream; every step of the computation runs in the
// kernels included below.  The whole library is one translation unit so that
// the device status word is a single object.
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "based.h"
#include "common.cuh"
#include "decode.cuh"
#include "linattn_simt.cuh"
#include "linattn_tc.cuh"
#include "linattn_bwd.cuh"
#include "linattn_bwd_tc.cuh"
#include "window_bwd.cuh"
#include "window_simt.cuh"
#include "window_tc.cuh"
#include "window_tcp.cuh"
#include "proj_tc.cuh"
#include "window_bwd_tc.cuh"

namespace based {

template <typename T>
__global__ void __launch_bounds__(256) ring_fill_kernel(const T* __restrict__ k,
                                                        const T* __restrict__ v,
                                                        T* __restrict__ k_ring,
                                                        T* __restrict__ v_ring, int L, int dh,
                                                        int W) {
  const size_t bh = blockIdx.x;
  const int n = min(L, W);
  const int p0 = L - n;
  for (int i = threadIdx.x; i < n * dh; i += blockDim.x) {
    const int r = i / dh, c = i - r * dh;
    const int p = p0 + r, slot = p % W;
    k_ring[(bh * W + slot) * dh + c] = k[(bh * L + p) * dh + c];
    v_ring[(bh * W + slot) * dh + c] = v[(bh * L + p) * dh + c];
  }
}

}  // namespace based

namespace {

using namespace based;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline based_status_t launch_status() {
  return cudaGetLastError() == cudaSuccess ? BASED_OK : BASED_ERR_CUDA;
}

template <typename K>
inline bool set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)bytes) == cudaSuccess;
}

// Launch as a programmatic dependent of the previous kernel in the stream: the
// kernel's CTAs may start (and run their set-up) while that kernel finishes;
// the kernel waits for it (griddepcontrol.wait) before touching global memory.
// TMEM: a kernel that allocates TMEM before that wait (the prefill, the
// persistent window kernel, the projections) must never share an SM with a CTA
// of the previous kernel that has yet to allocate, which would wait for columns
// held by a CTA waiting for it.  Those kernels take more than half of an SM's
// shared memory, so no other kernel's CTA runs beside them; the kernels whose
// CTAs share SMs (the backward kernels, the d_h = 128 window kernel) wait first
// and allocate after; the fp32 kernels hold no TMEM.
template <typename... KArgs, typename... Args>
bool launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...) == cudaSuccess;
}

// Shared argument checks of the prefill entry points.  Null tensor pointers
// are accepted only when the tensors are empty.
inline based_status_t check_tensor(const void* p, bool empty) {
  if (p == nullptr) return empty ? BASED_OK : BASED_ERR_INVALID_ARG;
  return aligned16(p) ? BASED_OK : BASED_ERR_INVALID_ARG;
}

based_status_t check_linattn(const void* q, const void* k, const void* v, const void* out,
                             int B, int H, int L, int d_feat, int d_v, based_dtype_t dt,
                             float eps, const float* state_kv, const float* state_k) {
  if (B < 0 || H < 0 || L < 0) return BASED_ERR_INVALID_ARG;
  if (dt != BASED_F32 && dt != BASED_BF16) return BASED_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !isfinite(eps)) return BASED_ERR_INVALID_ARG;
  if (d_feat != kD) return BASED_ERR_UNSUPPORTED;
  if (d_v != 64 && d_v != 128) return BASED_ERR_UNSUPPORTED;
  if ((long long)B * H > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  const bool empty = (long long)B * H * L == 0;
  based_status_t s;
  if ((s = check_tensor(q, empty)) != BASED_OK) return s;
  if ((s = check_tensor(k, empty)) != BASED_OK) return s;
  if ((s = check_tensor(v, empty)) != BASED_OK) return s;
  if ((s = check_tensor(out, empty)) != BASED_OK) return s;
  if (state_kv && !aligned16(state_kv)) return BASED_ERR_INVALID_ARG;
  if (state_k && !aligned16(state_k)) return BASED_ERR_INVALID_ARG;
  return BASED_OK;
}

template <typename T>
based_status_t launch_linattn_simt(const void* q, const void* k, const void* v, void* out,
                                   int BH, int L, int d_v, float eps, float* state_kv,
                                   float* state_k, cudaStream_t st) {
  auto kern = linattn_simt_kernel<T>;
  const size_t smem = linattn_simt_smem_bytes();
  if (!set_smem(kern, smem)) return BASED_ERR_CUDA;
  dim3 grid((unsigned)BH, (unsigned)(d_v / kSimtCols));
  if (!launch_dependent(kern, grid, dim3(kSimtThreads), smem, st, static_cast<const T*>(q),
                        static_cast<const T*>(k), static_cast<const T*>(v), static_cast<T*>(out),
                        state_kv, state_k, L, d_v, eps))
    return BASED_ERR_CUDA;
  return launch_status();
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 encode_tiled() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) !=
            cudaSuccess ||
        qr != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// 3-D map over a [BH, L, cols] bf16 tensor with a (64 cols x rows x 1) box and
// 128-byte swizzle; rows past L read as zero.
bool make_rows_map(CUtensorMap* m, const void* base, int cols, int L, int BH, int box_rows) {
  auto enc = encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)(L > 0 ? L : 1), (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)cols * 2 * (cuuint64_t)(L > 0 ? L : 1)};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output map of one per-head projection: y as [B*H][L][D] bf16, boxes of 128
// rows x min(D, 64) columns, swizzled by the box row's width (16 bytes: none).
bool make_head_out_map(CUtensorMap* m, void* y, int D, int L, int BH) {
  auto enc = encode_tiled();
  if (!enc) return false;
  const int bw = D < 64 ? D : 64;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)L, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)D * 2 * (cuuint64_t)L};
  cuuint32_t box[3] = {(cuuint32_t)bw, (cuuint32_t)kPjM, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw = bw == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : bw == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                : bw == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                           : CU_TENSOR_MAP_SWIZZLE_NONE;
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, y, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

// Segments per sequence for the tensor-core prefill: enough CTAs to cover the
// SMs when B*H is small, at least two chunks per segment.
struct TcPlan {
  int n_seg = 1;
  int seg_chunks = 1;
  size_t workspace = 0;
};
TcPlan plan_linattn_tc(long long BH, int L, int d_v) {
  TcPlan pl;
  const int n_chunks = (L + kTcChunk - 1) / kTcChunk;
  pl.seg_chunks = n_chunks > 0 ? n_chunks : 1;
  if (BH <= 0 || n_chunks < 4) return pl;
  const long long sms = device_sm_count();
  long long want = sms / BH;
  if (want < 2) return pl;
  if (want > n_chunks / 2) want = n_chunks / 2;
  const int seg_chunks = (int)((n_chunks + want - 1) / want);
  const int n_seg = (n_chunks + seg_chunks - 1) / seg_chunks;
  if (n_seg < 2) return pl;
  pl.n_seg = n_seg;
  pl.seg_chunks = seg_chunks;
  pl.workspace = (size_t)BH * (size_t)(n_seg - 1) * kSymFP * (size_t)(d_v + 16) * sizeof(float);
  return pl;
}

// BH sequences of v_split * DV value columns; the kernel runs each DV-wide
// column slice of a sequence as its own CTA (bh * v_split + slice)
// bf16 inputs: every d_v runs on the d_v = 64 kernel, one CTA per 64-column slice
TcPlan plan_linattn_bf16(long long BH, int L, int d_v) {
  return plan_linattn_tc(BH * (d_v / 64), L, 64);
}

template <int DV>
based_status_t launch_linattn_tc(const void* q, const void* k, const void* v, void* out, int BH,
                                 int L, float eps, float* state_kv, float* state_k,
                                 void* workspace, size_t workspace_bytes, cudaStream_t st,
                                 int v_split = 1) {
  const long long BHv = (long long)BH * v_split;
  if (BHv > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  const TcPlan pl = plan_linattn_tc(BHv, L, DV);
  if (pl.workspace > 0 && (workspace == nullptr || workspace_bytes < pl.workspace))
    return BASED_ERR_WORKSPACE;
  if (pl.workspace > 0 && (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
    return BASED_ERR_INVALID_ARG;
  CUtensorMap vmap, ymap;
  if (!make_rows_map(&vmap, v, DV * v_split, L, BH, kTcChunk)) return BASED_ERR_CUDA;
  if (!make_rows_map(&ymap, out, DV * v_split, L, BH, kTcChunk)) return BASED_ERR_CUDA;
  TcParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.state_kv = state_kv;
  p.state_k = state_k;
  p.partial = static_cast<float*>(workspace);
  p.L = L;
  p.seg_chunks = pl.seg_chunks;
  p.n_seg = pl.n_seg;
  p.eps = eps;
  p.v_split = v_split;
  p.ld_v = DV * v_split;
  const size_t smem = TcLayout<DV>::kSmem;
  if (pl.n_seg > 1) {
    auto kst = linattn_tc_kernel<DV, true>;
    if (!set_smem(kst, smem)) return BASED_ERR_CUDA;
    const long long nblk = BHv * (pl.n_seg - 1);
    if (nblk > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
    if (!launch_dependent(kst, dim3((unsigned)nblk), dim3(kTcThreads), smem, st, vmap, ymap, p))
      return BASED_ERR_CUDA;
    // running sums over the segments, so each main-pass CTA reads one partial
    if (pl.n_seg > 2) {
      const int elems = kSymFP * TcLayout<DV>::NA;
      const long long threads = BHv * (elems / 4);
      if (!launch_dependent(linattn_partial_prefix_kernel, dim3((unsigned)((threads + 255) / 256)),
                            dim3(256), 0, st, p.partial, (int)BHv, pl.n_seg - 1, elems))
        return BASED_ERR_CUDA;
    }
  }
  auto kern = linattn_tc_kernel<DV, false>;
  if (!set_smem(kern, smem)) return BASED_ERR_CUDA;
  const long long nblk = BHv * pl.n_seg;
  if (nblk > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  if (!launch_dependent(kern, dim3((unsigned)nblk), dim3(kTcThreads), smem, st, vmap, ymap, p))
    return BASED_ERR_CUDA;
  return launch_status();
}

template <int DH>
based_status_t launch_window_tc(const void* q, const void* k, const void* v, void* out, int BH,
                                int L, int W, cudaStream_t st) {
  CUtensorMap qm, km, vm, ym;
  if (!make_rows_map(&qm, q, DH, L, BH, kWtQ) || !make_rows_map(&km, k, DH, L, BH, kWtKeys) ||
      !make_rows_map(&vm, v, DH, L, BH, kWtKeys) || !make_rows_map(&ym, out, DH, L, BH, kWtQ))
    return BASED_ERR_CUDA;
  auto kern = window_tc_kernel<DH>;
  const size_t smem = WtLayout<DH>::kSmem;
  if (!set_smem(kern, smem)) return BASED_ERR_CUDA;
  const int n_tiles = (L + kWtQ - 1) / kWtQ;
  const long long nblk = (long long)n_tiles * BH;
  if (nblk > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  if (!launch_dependent(kern, dim3((unsigned)nblk), dim3(kWtThreads), smem, st, qm, km, vm, ym, L,
                        W, n_tiles))
    return BASED_ERR_CUDA;
  return launch_status();
}

// d_head = 64: the persistent kernel, one CTA per SM (or per tile, if fewer)
based_status_t launch_window_tcp(const void* q, const void* k, const void* v, void* out, int BH,
                                 int L, int W, cudaStream_t st) {
  CUtensorMap qm, km, vm, ym;
  if (!make_rows_map(&qm, q, 64, L, BH, kWtQ) || !make_rows_map(&km, k, 64, L, BH, kWtKeys) ||
      !make_rows_map(&vm, v, 64, L, BH, kWtKeys) || !make_rows_map(&ym, out, 64, L, BH, kWtQ))
    return BASED_ERR_CUDA;
  if (!set_smem(window_tcp_kernel, WpLayout::kSmem)) return BASED_ERR_CUDA;
  const int tiles_per_seq = (L + kWtQ - 1) / kWtQ;
  const long long n_total = (long long)tiles_per_seq * BH;
  if (n_total > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  const long long sms = device_sm_count();
  const unsigned grid = (unsigned)(n_total < sms ? n_total : sms);
  if (!launch_dependent(window_tcp_kernel, dim3(grid), dim3(kWpThreads), WpLayout::kSmem, st, qm,
                        km, vm, ym, L, W, tiles_per_seq, (int)n_total))
    return BASED_ERR_CUDA;
  return launch_status();
}

template <typename T, int Q, int SUB>
based_status_t launch_window_simt_q(const void* q, const void* k, const void* v, void* out,
                                    int BH, int L, int dh, int W, cudaStream_t st) {
  auto kern = window_simt_kernel<T, Q, SUB>;
  const size_t smem = window_simt_smem_bytes<Q>(dh);
  if (!set_smem(kern, smem)) return BASED_ERR_CUDA;
  const long long nblk = (L + Q - 1) / Q;
  if (nblk > 0x7fffffffLL || BH > 65535) return BASED_ERR_UNSUPPORTED;
  dim3 grid((unsigned)nblk, (unsigned)BH);
  if (!launch_dependent(kern, grid, dim3(Q * SUB), smem, st, static_cast<const T*>(q),
                        static_cast<const T*>(k), static_cast<const T*>(v), static_cast<T*>(out),
                        L, dh, W))
    return BASED_ERR_CUDA;
  return launch_status();
}

// 64-query blocks once they give every SM two CTAs; 16-query blocks below that.
template <typename T>
based_status_t launch_window_simt(const void* q, const void* k, const void* v, void* out,
                                  int BH, int L, int dh, int W, cudaStream_t st) {
  const long long blocks64 = (long long)BH * ((L + 63) / 64);
  if (blocks64 >= 2LL * device_sm_count())
    return launch_window_simt_q<T, 64, 4>(q, k, v, out, BH, L, dh, W, st);
  return launch_window_simt_q<T, 16, 16>(q, k, v, out, BH, L, dh, W, st);
}

template <typename T, int DV>
based_status_t launch_decode(DecodeParams p, cudaStream_t st) {
  auto kern = decode_step_kernel<T, DV>;
  constexpr int kThreads = 4 * DV;
  size_t smem = sizeof(float) * (size_t)DecodeLinearLayout<DV>::kSmemFloats;
  p.wg = 1;
  p.n_wblk = 0;
  if (p.n_win > 0) {
    // up to 4 heads per window CTA, within 64 KiB of ring buffers
    const int ring_pair = 2 * p.W * p.dh * (int)sizeof(T);
    p.wg = 65536 / ring_pair;
    p.wg = p.wg < 1 ? 1 : (p.wg > 4 ? 4 : p.wg);
    p.n_wblk = (p.n_win + p.wg - 1) / p.wg;
    const size_t w = (size_t)DecodeWindowLayout(p.wg, p.dh, p.W, kThreads, sizeof(T)).bytes;
    if (w > smem) smem = w;
  }
  if (!set_smem(kern, smem)) return BASED_ERR_CUDA;
  const long long nblk = (long long)p.n_lin + p.n_wblk;
  p.wstride = p.n_wblk > 0 ? (int)(nblk / p.n_wblk) : 1;
  if (!launch_dependent(kern, dim3((unsigned)nblk), dim3(kThreads), smem, st, p))
    return BASED_ERR_CUDA;
  return launch_status();
}

template <int Mode>
based_status_t launch_proj(const void* x, const void* w, ProjParams p, cudaStream_t st) {
  CUtensorMap xm, wm, hm;
  if (!make_rows_map(&xm, x, p.Kd, p.M, 1, kPjM) || !make_rows_map(&wm, w, p.Kd, p.N, 1, kPjNHalf))
    return BASED_ERR_CUDA;
  if (Mode == kBaseConv) {
    if (!make_rows_map(&hm, x, p.Kd, p.M, 1, kPjHaloRows)) return BASED_ERR_CUDA;
  } else {
    hm = xm;  // unused
  }
  // per-head outputs whose heads tile a 128-column half leave by TMA stores
  ProjYMaps ym;
  memset(&ym, 0, sizeof(ym));
  if (Mode == kProjHeads) {
    for (int g = 0; g < p.n_out; ++g)
      if (kPjNHalf % p.D[g] == 0 &&
          !make_head_out_map(&ym.m[g], p.y[g], p.D[g], p.L, (p.M / p.L) * p.H))
        return BASED_ERR_CUDA;
  }
  auto kern = proj_tc_kernel<Mode>;
  if (!set_smem(kern, PjLayout<Mode>::kSmem)) return BASED_ERR_CUDA;
  p.n_tiles_n = p.N / kPjN;
  const long long tiles = (long long)((p.M + 2 * kPjM - 1) / (2 * kPjM)) * p.n_tiles_n;
  if (tiles > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  p.total_tiles = (int)tiles;
  // CTA pairs: clusters of two, as many as fit at once (one CTA per SM)
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // a dependent launch
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(kPjThreads, 1, 1);
  cfg.dynamicSmemBytes = PjLayout<Mode>::kSmem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;  // the occupancy query below takes the cluster shape only
  cfg.gridDim = dim3(2 * (unsigned)((device_sm_count() + 1) / 2), 1, 1);
  int max_clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg) != cudaSuccess || max_clusters <= 0)
    return BASED_ERR_CUDA;
  const long long pairs = tiles < max_clusters ? tiles : max_clusters;
  cfg.gridDim = dim3(2 * (unsigned)pairs, 1, 1);
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, kern, xm, wm, hm, ym, p) != cudaSuccess) return BASED_ERR_CUDA;
  return launch_status();
}

template <typename T, int DV>
based_status_t launch_linattn_bwd(const void* q, const void* k, const void* v, const void* dy,
                                  float* dq, float* dk, float* dv, int BH, int L, float eps,
                                  float* ws, cudaStream_t st) {
  auto kq = linattn_bwd_q_kernel<T, DV>;
  auto kkv = linattn_bwd_kv_kernel<T, DV>;
  const size_t smem = BwLayout<DV>::kSmem;
  if (!set_smem(kq, smem) || !set_smem(kkv, smem)) return BASED_ERR_CUDA;
  const long long nblk = (long long)BH * ((L + kBwT - 1) / kBwT);
  if (nblk > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  float* ws_dN = ws;
  float* ws_dD = ws + (size_t)BH * L * DV;
  kq<<<(unsigned)nblk, kBwThreads, smem, st>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                               static_cast<const T*>(v), static_cast<const T*>(dy),
                                               dq, ws_dN, ws_dD, L, eps);
  const based_status_t s1 = launch_status();
  if (s1 != BASED_OK) return s1;
  kkv<<<(unsigned)nblk, kBwThreads, smem, st>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                                static_cast<const T*>(v), ws_dN, ws_dD, dk, dv, L);
  return launch_status();
}

// bf16 gradient on the tensor cores: workspace = dN (bf16 [BH, L, DV]) then dD
// (fp32 [BH, L]), well inside based_linattn_bwd_workspace_bytes
template <int DV>
based_status_t launch_linattn_bwd_tc(const void* q, const void* k, const void* v, const void* dy,
                                     float* dq, float* dk, float* dv, int BH, int L, float eps,
                                     void* ws, cudaStream_t st) {
  BtParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.dy = static_cast<const __nv_bfloat16*>(dy);
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.ws_dn = static_cast<__nv_bfloat16*>(ws);
  p.ws_dd = reinterpret_cast<float*>(static_cast<char*>(ws) + (size_t)BH * L * DV * 2);
  p.L = L;
  p.n_tiles = (L + kBtT - 1) / kBtT;
  p.BH = BH;
  p.eps = eps;
  CUtensorMap vmap, dnmap;
  if (!make_rows_map(&vmap, v, DV, L, BH, kBtT) || !make_rows_map(&dnmap, p.ws_dn, DV, L, BH, kBtT))
    return BASED_ERR_CUDA;
  auto kq = linattn_bwd_tc_q_kernel<DV>;
  auto kkv = linattn_bwd_tc_kv_kernel<DV>;
  if (!set_smem(kq, BtLayout<DV>::kSmemQ) || !set_smem(kkv, BtLayout<DV>::kSmemK))
    return BASED_ERR_CUDA;
  const long long nblk = (long long)BH * p.n_tiles;
  if (nblk > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  if (!launch_dependent(kq, dim3((unsigned)nblk), dim3(kBtThreads), BtLayout<DV>::kSmemQ, st, vmap,
                        p))
    return BASED_ERR_CUDA;
  const based_status_t s1 = launch_status();
  if (s1 != BASED_OK) return s1;
  if (!launch_dependent(kkv, dim3((unsigned)nblk), dim3(kBtThreads), BtLayout<DV>::kSmemK, st,
                        vmap, dnmap, p))
    return BASED_ERR_CUDA;
  return launch_status();
}

template <typename T>
based_status_t launch_window_bwd(const void* q, const void* k, const void* v, const void* dy,
                                 float* dq, float* dk, float* dv, int BH, int L, int W, float* ws,
                                 cudaStream_t st) {
  auto kq = window_bwd_q_kernel<T>;
  auto kkv = window_bwd_kv_kernel<T>;
  if (!set_smem(kq, WbLayout::kSmem) || !set_smem(kkv, WbLayout::kSmem)) return BASED_ERR_CUDA;
  const long long nblk = (long long)BH * ((L + kWbT - 1) / kWbT);
  if (nblk > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  kq<<<(unsigned)nblk, kWbThreads, WbLayout::kSmem, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
      static_cast<const T*>(dy), dq, ws, L, W);
  const based_status_t s1 = launch_status();
  if (s1 != BASED_OK) return s1;
  kkv<<<(unsigned)nblk, kWbThreads, WbLayout::kSmem, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
      static_cast<const T*>(dy), ws, dk, dv, L, W);
  return launch_status();
}

// bf16 window gradient on the tensor cores (d_h = 64 or 128)
template <int DH>
based_status_t launch_window_bwd_tc(const void* q, const void* k, const void* v, const void* dy,
                                    float* dq, float* dk, float* dv, int BH, int L, int W,
                                    float* ws, cudaStream_t st) {
  CUtensorMap q128, dy128, k192, v192, k128, v128, q192, dy192;
  if (!make_rows_map(&q128, q, DH, L, BH, kWgT) || !make_rows_map(&dy128, dy, DH, L, BH, kWgT) ||
      !make_rows_map(&k192, k, DH, L, BH, kWgN) || !make_rows_map(&v192, v, DH, L, BH, kWgN) ||
      !make_rows_map(&k128, k, DH, L, BH, kWgT) || !make_rows_map(&v128, v, DH, L, BH, kWgT) ||
      !make_rows_map(&q192, q, DH, L, BH, kWgN) || !make_rows_map(&dy192, dy, DH, L, BH, kWgN))
    return BASED_ERR_CUDA;
  auto kq = window_bwd_tc_q_kernel<DH>;
  auto kkv = window_bwd_tc_kv_kernel<DH>;
  const size_t smem = WgLayout<DH>::kSmem;
  if (!set_smem(kq, smem) || !set_smem(kkv, smem)) return BASED_ERR_CUDA;
  WgParams p;
  p.dq = dq; p.dk = dk; p.dv = dv; p.ws = ws;
  p.L = L; p.W = W; p.BH = BH;
  p.n_tiles = (L + kWgT - 1) / kWgT;
  const long long nblk = (long long)BH * p.n_tiles;
  if (nblk > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  if (!launch_dependent(kq, dim3((unsigned)nblk), dim3(kWgThreads), smem, st, q128, dy128, k192,
                        v192, p))
    return BASED_ERR_CUDA;
  const based_status_t s1 = launch_status();
  if (s1 != BASED_OK) return s1;
  if (!launch_dependent(kkv, dim3((unsigned)nblk), dim3(kWgThreads), smem, st, k128, v128, q192,
                        dy192, p))
    return BASED_ERR_CUDA;
  return launch_status();
}

// ---------------------------------------------------------------------------
// Allocation-free prefill (based_linattn_fwd_noalloc): the segment partials
// live in this fixed array instead of a caller workspace.  Host code may not
// pass the array's name to a kernel (on the host it is only a stand-in); the
// device address is looked up with cudaGetSymbolAddress on every call, with
// the caller's device current, so it stays right after a device reset.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;

}  // namespace

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

namespace {

// Device address of g_noalloc_scratch on the current device.
based_status_t noalloc_scratch(float** addr) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
    return BASED_ERR_CUDA;
  *addr = static_cast<float*>(p);
  return BASED_OK;
}

}  // namespace

extern "C" {

int based_abi_version(void) { return 1; }

int based_binary_version(void) {
  cudaFuncAttributes a;
  if (cudaFuncGetAttributes(&a, linattn_tc_kernel<64, false>) != cudaSuccess) return -1;
  return a.binaryVersion;
}

const char* based_status_string(based_status_t status) {
  switch (status) {
    case BASED_OK: return "BASED_OK";
    case BASED_ERR_INVALID_ARG: return "BASED_ERR_INVALID_ARG";
    case BASED_ERR_UNSUPPORTED: return "BASED_ERR_UNSUPPORTED";
    case BASED_ERR_CUDA: return "BASED_ERR_CUDA";
    case BASED_ERR_TIMEOUT: return "BASED_ERR_TIMEOUT";
    case BASED_ERR_WORKSPACE: return "BASED_ERR_WORKSPACE";
  }
  return "BASED_ERR_UNKNOWN";
}

size_t based_linattn_workspace_bytes(int B, int H, int L, int d_feat, int d_v,
                                     based_dtype_t dt) {
  if (B < 0 || H < 0 || L < 0 || (dt != BASED_F32 && dt != BASED_BF16) || d_feat != kD ||
      (d_v != 64 && d_v != 128))
    return (size_t)-1;
  if (dt == BASED_F32) return 0;
  return plan_linattn_bf16((long long)B * H, L, d_v).workspace;
}

based_status_t based_linattn_fwd(const void* q, const void* k, const void* v, void* out,
                                 int B, int H, int L, int d_feat, int d_v, based_dtype_t dt,
                                 float eps, float* state_kv, float* state_k, void* workspace,
                                 size_t workspace_bytes, based_stream_t stream) {
  based_status_t s =
      check_linattn(q, k, v, out, B, H, L, d_feat, d_v, dt, eps, state_kv, state_k);
  if (s != BASED_OK) return s;
  const int BH = B * H;
  if (BH == 0) return BASED_OK;
  if (L == 0 && !state_kv && !state_k) return BASED_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == BASED_F32)
    return launch_linattn_simt<float>(q, k, v, out, BH, L, d_v, eps, state_kv, state_k, st);
  return launch_linattn_tc<64>(q, k, v, out, BH, L, eps, state_kv, state_k, workspace,
                               workspace_bytes, st, d_v / 64);
}

based_status_t based_linattn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                         int B, int H, int L, int d_feat, int d_v,
                                         based_dtype_t dt, float eps, float* state_kv,
                                         float* state_k, based_stream_t stream) {
  based_status_t s =
      check_linattn(q, k, v, out, B, H, L, d_feat, d_v, dt, eps, state_kv, state_k);
  if (s != BASED_OK) return s;
  const int BH = B * H;
  if (BH == 0) return BASED_OK;
  if (L == 0 && !state_kv && !state_k) return BASED_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == BASED_F32)  // the fp32 path needs no scratch
    return launch_linattn_simt<float>(q, k, v, out, BH, L, d_v, eps, state_kv, state_k, st);
  const size_t need = plan_linattn_bf16(BH, L, d_v).workspace;
  if (need > kNoAllocScratchBytes) return BASED_ERR_WORKSPACE;
  float* scratch = nullptr;
  if (need > 0 && (s = noalloc_scratch(&scratch)) != BASED_OK) return s;
  return launch_linattn_tc<64>(q, k, v, out, BH, L, eps, state_kv, state_k, scratch,
                               kNoAllocScratchBytes, st, d_v / 64);
}

based_status_t based_window_attn_fwd(const void* q, const void* k, const void* v, void* out,
                                     int B, int H, int L, int d_head, int window,
                                     based_dtype_t dt, based_stream_t stream) {
  if (B < 0 || H < 0 || L < 0) return BASED_ERR_INVALID_ARG;
  if (dt != BASED_F32 && dt != BASED_BF16) return BASED_ERR_INVALID_ARG;
  if (window < 1) return BASED_ERR_INVALID_ARG;
  if (window > kWinK) return BASED_ERR_UNSUPPORTED;
  if (d_head != 64 && d_head != 128) return BASED_ERR_UNSUPPORTED;
  const bool empty = (long long)B * H * L == 0;
  based_status_t s;
  if ((s = check_tensor(q, empty)) != BASED_OK) return s;
  if ((s = check_tensor(k, empty)) != BASED_OK) return s;
  if ((s = check_tensor(v, empty)) != BASED_OK) return s;
  if ((s = check_tensor(out, empty)) != BASED_OK) return s;
  if (empty) return BASED_OK;
  if ((long long)B * H > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == BASED_F32) return launch_window_simt<float>(q, k, v, out, B * H, L, d_head, window, st);
  return d_head == 64 ? launch_window_tcp(q, k, v, out, B * H, L, window, st)
                      : launch_window_tc<128>(q, k, v, out, B * H, L, window, st);
}

based_status_t based_window_ring_fill(const void* k, const void* v, int B, int H, int L,
                                      int d_head, int window, void* k_ring, void* v_ring,
                                      based_dtype_t dt, based_stream_t stream) {
  if (B < 0 || H < 0 || L < 0 || window < 1) return BASED_ERR_INVALID_ARG;
  if (dt != BASED_F32 && dt != BASED_BF16) return BASED_ERR_INVALID_ARG;
  if (window > kWinK) return BASED_ERR_UNSUPPORTED;
  if (d_head != 64 && d_head != 128) return BASED_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  based_status_t s;
  if ((s = check_tensor(k, BH * L == 0)) != BASED_OK) return s;
  if ((s = check_tensor(v, BH * L == 0)) != BASED_OK) return s;
  if ((s = check_tensor(k_ring, BH == 0)) != BASED_OK) return s;
  if ((s = check_tensor(v_ring, BH == 0)) != BASED_OK) return s;
  if (BH == 0 || L == 0) return BASED_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == BASED_F32)
    ring_fill_kernel<float><<<(unsigned)BH, 256, 0, st>>>(
        static_cast<const float*>(k), static_cast<const float*>(v), static_cast<float*>(k_ring),
        static_cast<float*>(v_ring), L, d_head, window);
  else
    ring_fill_kernel<__nv_bfloat16><<<(unsigned)BH, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
        static_cast<__nv_bfloat16*>(k_ring), static_cast<__nv_bfloat16*>(v_ring), L, d_head,
        window);
  return launch_status();
}

}  // extern "C"

namespace {
// Shared body of based_decode_step (one position, pos_arr == null) and
// based_decode_step_at (per-sequence positions in device memory).
based_status_t decode_step_impl(const void* q, const void* k, const void* v, float* state_kv,
                                float* state_k, void* out, const void* wq, const void* wk,
                                const void* wv, void* k_ring, void* v_ring, void* wout,
                                long long pos, const long long* pos_arr, int B, int H,
                                int d_feat, int d_v, int H_w, int d_head, int window,
                                based_dtype_t dt, float eps, based_stream_t stream) {
  if (B < 0 || H < 0 || H_w < 0 || pos < 0) return BASED_ERR_INVALID_ARG;
  if (dt != BASED_F32 && dt != BASED_BF16) return BASED_ERR_INVALID_ARG;
  const bool lin = q != nullptr || H > 0;
  const bool win = wq != nullptr || H_w > 0;
  if (!lin && !win) return BASED_ERR_INVALID_ARG;
  if (lin) {
    if (H < 1 || !q || !k || !v || !state_kv || !state_k || !out) return BASED_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state_kv) ||
        !aligned16(state_k) || !aligned16(out))
      return BASED_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || !isfinite(eps)) return BASED_ERR_INVALID_ARG;
    if (d_feat != kD) return BASED_ERR_UNSUPPORTED;
    if (d_v != 64 && d_v != 128) return BASED_ERR_UNSUPPORTED;
  }
  if (win) {
    if (H_w < 1 || !wq || !wk || !wv || !k_ring || !v_ring || !wout) return BASED_ERR_INVALID_ARG;
    if (!aligned16(wq) || !aligned16(wk) || !aligned16(wv) || !aligned16(k_ring) ||
        !aligned16(v_ring) || !aligned16(wout))
      return BASED_ERR_INVALID_ARG;
    if (window < 1) return BASED_ERR_INVALID_ARG;
    if (window > kWinK) return BASED_ERR_UNSUPPORTED;
    if (d_head != 64 && d_head != 128) return BASED_ERR_UNSUPPORTED;
  }
  const long long n_lin = lin ? (long long)B * H : 0, n_win = win ? (long long)B * H_w : 0;
  if (n_lin + n_win > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  if (n_lin + n_win == 0) return BASED_OK;
  DecodeParams p;
  p.q = q; p.k = k; p.v = v; p.S = state_kv; p.z = state_k; p.out = out;
  p.wq = wq; p.wk = wk; p.wv = wv; p.k_ring = k_ring; p.v_ring = v_ring; p.wout = wout;
  p.pos = pos; p.pos_arr = pos_arr; p.H_w = H_w > 0 ? H_w : 1;
  p.n_lin = (int)n_lin; p.n_win = (int)n_win;
  p.dh = d_head; p.W = window; p.eps = eps;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool wide = lin && d_v == 128;
  if (dt == BASED_F32)
    return wide ? launch_decode<float, 128>(p, st) : launch_decode<float, 64>(p, st);
  return wide ? launch_decode<__nv_bfloat16, 128>(p, st) : launch_decode<__nv_bfloat16, 64>(p, st);
}
}  // namespace

extern "C" {

based_status_t based_decode_step(const void* q, const void* k, const void* v, float* state_kv,
                                 float* state_k, void* out, const void* wq, const void* wk,
                                 const void* wv, void* k_ring, void* v_ring, void* wout,
                                 long long pos, int B, int H, int d_feat, int d_v, int H_w,
                                 int d_head, int window, based_dtype_t dt, float eps,
                                 based_stream_t stream) {
  return decode_step_impl(q, k, v, state_kv, state_k, out, wq, wk, wv, k_ring, v_ring, wout, pos,
                          nullptr, B, H, d_feat, d_v, H_w, d_head, window, dt, eps, stream);
}

based_status_t based_decode_step_at(const void* q, const void* k, const void* v,
                                    float* state_kv, float* state_k, void* out, const void* wq,
                                    const void* wk, const void* wv, void* k_ring, void* v_ring,
                                    void* wout, const long long* pos, int B, int H, int d_feat,
                                    int d_v, int H_w, int d_head, int window, based_dtype_t dt,
                                    float eps, based_stream_t stream) {
  const bool win = wq != nullptr || H_w > 0;
  if (win && B > 0 && (pos == nullptr || (reinterpret_cast<uintptr_t>(pos) & 7u) != 0))
    return BASED_ERR_INVALID_ARG;
  return decode_step_impl(q, k, v, state_kv, state_k, out, wq, wk, wv, k_ring, v_ring, wout, 0,
                          win ? pos : nullptr, B, H, d_feat, d_v, H_w, d_head, window, dt, eps,
                          stream);
}

size_t based_linattn_bwd_workspace_bytes(int B, int H, int L, int d_v) {
  if (B < 0 || H < 0 || L < 0 || (d_v != 64 && d_v != 128)) return (size_t)-1;
  return (size_t)B * H * L * (d_v + 1) * sizeof(float);
}

based_status_t based_linattn_bwd(const void* q, const void* k, const void* v, const void* dy,
                                 float* dq, float* dk, float* dv, int B, int H, int L,
                                 int d_feat, int d_v, based_dtype_t dt, float eps,
                                 void* workspace, size_t workspace_bytes, based_stream_t stream) {
  // the forward's checks of sizes, dtype, eps (finite, >= 0) and of q, k, v, dy
  based_status_t s = check_linattn(q, k, v, dy, B, H, L, d_feat, d_v, dt, eps, nullptr, nullptr);
  if (s != BASED_OK) return s;
  const long long BH = (long long)B * H;
  const bool empty = BH * L == 0;
  if ((s = check_tensor(dq, empty)) != BASED_OK) return s;
  if ((s = check_tensor(dk, empty)) != BASED_OK) return s;
  if ((s = check_tensor(dv, empty)) != BASED_OK) return s;
  if (empty) return BASED_OK;
  if (BH * L * (d_v + 1) > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < based_linattn_bwd_workspace_bytes(B, H, L, d_v))
    return BASED_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BASED_ERR_INVALID_ARG;
  float* ws = static_cast<float*>(workspace);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == BASED_F32)
    return d_v == 64 ? launch_linattn_bwd<float, 64>(q, k, v, dy, dq, dk, dv, (int)BH, L, eps, ws, st)
                     : launch_linattn_bwd<float, 128>(q, k, v, dy, dq, dk, dv, (int)BH, L, eps, ws, st);
  return d_v == 64 ? launch_linattn_bwd_tc<64>(q, k, v, dy, dq, dk, dv, (int)BH, L, eps, workspace, st)
                   : launch_linattn_bwd_tc<128>(q, k, v, dy, dq, dk, dv, (int)BH, L, eps, workspace, st);
}

size_t based_window_attn_bwd_workspace_bytes(int B, int H, int L) {
  if (B < 0 || H < 0 || L < 0) return (size_t)-1;
  return (size_t)B * H * L * 3 * sizeof(float);
}

based_status_t based_window_attn_bwd(const void* q, const void* k, const void* v, const void* dy,
                                     float* dq, float* dk, float* dv, int B, int H, int L,
                                     int d_head, int window, based_dtype_t dt, void* workspace,
                                     size_t workspace_bytes, based_stream_t stream) {
  if (B < 0 || H < 0 || L < 0 || window < 1) return BASED_ERR_INVALID_ARG;
  if (dt != BASED_BF16 && dt != BASED_F32) return BASED_ERR_INVALID_ARG;
  // bf16: tensor cores, d_h 64 or 128; fp32: CUDA cores, d_h 64
  if (window > kWbT || (dt == BASED_F32 ? d_head != kWbDh : (d_head != 64 && d_head != 128)))
    return BASED_ERR_UNSUPPORTED;
  const long long BH = (long long)B * H;
  if (BH > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  const bool empty = BH * L == 0;
  based_status_t s;
  for (const void* t : {q, k, v, dy, static_cast<const void*>(dq), static_cast<const void*>(dk),
                        static_cast<const void*>(dv)})
    if ((s = check_tensor(t, empty)) != BASED_OK) return s;
  if (empty) return BASED_OK;
  if (BH * L * d_head > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < based_window_attn_bwd_workspace_bytes(B, H, L))
    return BASED_ERR_WORKSPACE;
  if (!aligned16(workspace)) return BASED_ERR_INVALID_ARG;
  float* ws = static_cast<float*>(workspace);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == BASED_F32)
    return launch_window_bwd<float>(q, k, v, dy, dq, dk, dv, (int)BH, L, window, ws, st);
  if (d_head == 128)
    return launch_window_bwd_tc<128>(q, k, v, dy, dq, dk, dv, (int)BH, L, window, ws, st);
  return launch_window_bwd_tc<64>(q, k, v, dy, dq, dk, dv, (int)BH, L, window, ws, st);
}

based_status_t based_proj_heads_multi_fwd(const void* x, const void* w, int n_out, const int* D,
                                          void* const* y, int B, int L, int d_model, int H,
                                          based_dtype_t dt, based_stream_t stream) {
  if (B < 0 || L < 0 || d_model <= 0 || H <= 0 || n_out < 1 || n_out > kPjMaxOut || !D || !y)
    return BASED_ERR_INVALID_ARG;
  if (dt != BASED_BF16 && dt != BASED_F32) return BASED_ERR_INVALID_ARG;
  for (int g = 0; g < n_out; ++g)
    if (D[g] <= 0) return BASED_ERR_INVALID_ARG;
  if (dt != BASED_BF16) return BASED_ERR_UNSUPPORTED;
  if (d_model % kPjK != 0) return BASED_ERR_UNSUPPORTED;
  long long N = 0;
  for (int g = 0; g < n_out; ++g) {
    if (((long long)H * D[g]) % kPjN != 0 || D[g] % 8 != 0) return BASED_ERR_UNSUPPORTED;
    N += (long long)H * D[g];
  }
  const long long M = (long long)B * L;
  if (M > 0x7fffffffLL || N > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  if (M == 0) return BASED_OK;
  if (!x || !w || !aligned16(x) || !aligned16(w)) return BASED_ERR_INVALID_ARG;
  for (int g = 0; g < n_out; ++g)
    if (!y[g] || !aligned16(y[g])) return BASED_ERR_INVALID_ARG;
  ProjParams p{};
  p.n_out = n_out;
  int col = 0;
  for (int g = 0; g < n_out; ++g) {
    p.y[g] = static_cast<__nv_bfloat16*>(y[g]);
    p.D[g] = D[g];
    p.col_begin[g] = col;
    col += H * D[g];
  }
  p.col_begin[n_out] = col;
  p.M = (int)M; p.N = (int)N; p.Kd = d_model; p.L = L; p.H = H;
  return launch_proj<kProjHeads>(x, w, p, static_cast<cudaStream_t>(stream));
}

based_status_t based_proj_heads_fwd(const void* x, const void* w, void* y, int B, int L,
                                    int d_model, int H, int D, based_dtype_t dt,
                                    based_stream_t stream) {
  void* ys[1] = {y};
  const int Ds[1] = {D};
  if (D <= 0) return BASED_ERR_INVALID_ARG;
  return based_proj_heads_multi_fwd(x, w, 1, Ds, ys, B, L, d_model, H, dt, stream);
}

based_status_t based_baseconv_fwd(const void* x, const void* w, const float* bias,
                                  const float* taps, void* y, int B, int L, int D, int K,
                                  based_dtype_t dt, based_stream_t stream) {
  if (B < 0 || L < 0 || D <= 0 || K <= 0) return BASED_ERR_INVALID_ARG;
  if (dt != BASED_BF16 && dt != BASED_F32) return BASED_ERR_INVALID_ARG;
  if (dt != BASED_BF16) return BASED_ERR_UNSUPPORTED;
  if (D % kPjN != 0 || K > kPjMaxTaps) return BASED_ERR_UNSUPPORTED;
  const long long M = (long long)B * L;
  if (M > 0x7fffffffLL) return BASED_ERR_UNSUPPORTED;
  if (M == 0) return BASED_OK;
  if (!x || !w || !bias || !taps || !y) return BASED_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return BASED_ERR_INVALID_ARG;
  ProjParams p{};
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.n_out = 1;
  p.y[0] = static_cast<__nv_bfloat16*>(y);
  p.bias = bias; p.taps = taps;
  p.M = (int)M; p.N = D; p.Kd = D; p.L = L; p.K = K;
  return launch_proj<kBaseConv>(x, w, p, static_cast<cudaStream_t>(stream));
}

based_status_t based_debug_stall(int which, long long wait_limit_ns) {
  if (which != kStallNone && which != kStallLinattnV && which != kStallWindowV)
    return BASED_ERR_INVALID_ARG;
  if (wait_limit_ns <= 0) return BASED_ERR_INVALID_ARG;
  const uint64_t limit = static_cast<uint64_t>(wait_limit_ns);
  if (cudaDeviceSynchronize() != cudaSuccess) return BASED_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_stall_test, &which, sizeof(int)) != cudaSuccess ||
      cudaMemcpyToSymbol(umma::g_wait_limit_ns, &limit, sizeof(uint64_t)) != cudaSuccess)
    return BASED_ERR_CUDA;
  return BASED_OK;
}

based_status_t based_get_device_error(based_stream_t stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return BASED_ERR_CUDA;
  int v = BASED_OK;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess)
    return BASED_ERR_CUDA;
  if (v != BASED_OK) {
    const int ok = BASED_OK;
    if (cudaMemcpyToSymbol(g_device_status, &ok, sizeof(int)) != cudaSuccess)
      return BASED_ERR_CUDA;
  }
  return static_cast<based_status_t>(v);
}

}  // extern "C"
