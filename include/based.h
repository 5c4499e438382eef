/*
 * based.h -- C ABI of the B200 (sm_100a) Based attention library.
 *
 * The library computes the data-parallel attention path of the Based
 * architecture ("Simple linear attention language models balance the
 * recall-throughput tradeoff", HazyResearch/based):
 *
 *   - causal linear attention with the second-order Taylor feature map
 *       phi(x) = [1, x / d^(1/4), vec(x x^T) / (sqrt(2) sqrt(d))],  d = 16,
 *     i.e. 1 + 16 + 256 = 273 features ("Базированная модель, часть 2",
 *     section "Что за линейное внимание?": the map cat(1, x, vec(xx^T)/sqrt 2)
 *     whose dot product is the expansion 1 + qk + (qk)^2/2 of exp(qk), here
 *     applied to x / d^(1/4) so it expands exp(q.k / sqrt(d))), and
 *       y_t = phi(q_t)^T S_t / (phi(q_t) . z_t + eps),
 *       S_t = sum_{s<=t} phi(k_s) v_s^T   (the KV state),
 *       z_t = sum_{s<=t} phi(k_s)         (the K state, same post, paragraph
 *                                          on the state size);
 *   - exact softmax attention over a sliding window of the last `window`
 *     tokens, current token included (Based README, introduction, item 1:
 *     window size 64), scale 1/sqrt(d_head);
 *   - the one-token recurrent decode step of both (the recurrent form of the
 *     linear attention over the KV/K states, and a `window`-slot ring cache).
 *
 * Beside it: the layer's per-head input projections and the BaseConv block
 * (tensor-core GEMM with fused epilogues), and the gradients of both
 * attention layers (CUDA cores).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers, owned by the caller, C-contiguous
 *     in the layouts given below, 16-byte aligned.  The library never keeps a
 *     pointer after the call returns and never allocates device memory
 *     (based_linattn_fwd_noalloc uses a fixed array inside the library).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *     asynchronous on it; the caller synchronises before reading results.
 *   - Argument errors are detected on the host, before any launch, and return
 *     BASED_ERR_INVALID_ARG / BASED_ERR_UNSUPPORTED with nothing written.
 *     A failed launch returns BASED_ERR_CUDA.  A kernel that gives up on a
 *     bounded wait records BASED_ERR_TIMEOUT in a device status word, read
 *     with based_get_device_error().
 *   - dtype BASED_BF16: q/k/v/out are bfloat16, arithmetic accumulates in fp32.
 *     dtype BASED_F32: everything is fp32 (fp32 CUDA-core arithmetic).
 *     Recurrent states (state_kv, state_k) and gradients are always fp32.
 *   - Feature order of the 273-row states: row 0 = constant 1; rows 1..16 =
 *     x_i / 2; row 17 + 16 i + j = x_i x_j / (4 sqrt 2)   (d = 16).
 *   - Thread safety: calls on different streams may run concurrently as long
 *     as they do not share output buffers or workspace.
 */
#ifndef BASED_H
#define BASED_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BASED_OK = 0,
    BASED_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, negative size, ... */
    BASED_ERR_UNSUPPORTED = 2,  /* valid but not implemented (d_feat != 16, ...) */
    BASED_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
    BASED_ERR_TIMEOUT = 4,      /* a kernel gave up on a bounded wait */
    BASED_ERR_WORKSPACE = 5     /* workspace missing or smaller than required */
} based_status_t;

typedef enum { BASED_F32 = 0, BASED_BF16 = 1 } based_dtype_t;

typedef void* based_stream_t; /* a cudaStream_t */

/* Version of this ABI (bumped on any incompatible change). */
int based_abi_version(void);

/*
 * Architecture of the device code the CUDA runtime loaded for the current
 * device, as cudaFuncGetAttributes reports it for one of the library's
 * kernels: major * 10 + minor (100 for the sm_100a build).  Returns -1 when
 * there is no usable device or the code cannot run on it.
 */
int based_binary_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* based_status_string(based_status_t status);

/*
 * Bytes of device workspace based_linattn_fwd needs for this problem on the
 * CURRENT device (it may split long sequences across CTAs and keep per-segment
 * partial states there).  0 means the call needs none (workspace may be NULL).
 * Returns (size_t)-1 for arguments based_linattn_fwd would reject.
 */
size_t based_linattn_workspace_bytes(int B, int H, int L, int d_feat, int d_v,
                                     based_dtype_t dt);

/*
 * Causal linear attention with the Taylor feature map, one fused forward pass
 * (the chunked "parallel" training view of the based/train README computed by
 * one kernel: intra-chunk masked phi(Q)phi(K)^T [V|1], inter-chunk readout of
 * the running KV/K states, state update, normaliser).
 *
 *   q, k      [B, H, L, d_feat]   dt          (d_feat must be 16)
 *   v         [B, H, L, d_v]      dt          (d_v in {64, 128})
 *   out       [B, H, L, d_v]      dt          (written)
 *   eps       >= 0, added to the denominator only
 *   state_kv  [B, H, 273, d_v] fp32 or NULL   final KV state S_L (written)
 *   state_k   [B, H, 273]      fp32 or NULL   final K state z_L (written)
 *   workspace device scratch of based_linattn_workspace_bytes(...) bytes, or
 *             NULL when that is 0; contents need not be initialised and are
 *             clobbered.
 * L = 0 is valid: nothing is read, the states (if requested) are zeroed.
 */
based_status_t based_linattn_fwd(const void* q, const void* k, const void* v, void* out,
                                 int B, int H, int L, int d_feat, int d_v,
                                 based_dtype_t dt, float eps,
                                 float* state_kv, float* state_k,
                                 void* workspace, size_t workspace_bytes,
                                 based_stream_t stream);

/*
 * Same computation and arguments as based_linattn_fwd, for callers that must
 * not allocate device memory: a plugin or server whose host framework owns
 * every device allocation, or a latency-critical loop where cudaMalloc's
 * implicit device synchronisation is not acceptable.  Such callers cannot
 * provide the workspace based_linattn_fwd may ask for.  (The paper has no
 * counterpart to this entry point; it is a deployment convenience.)
 *
 * Scratch comes from a fixed array compiled into the library, 16 MiB on every
 * GPU that loads the library, held until the process exits.  Nothing is
 * allocated, here or later.  A problem whose scratch need
 * (based_linattn_workspace_bytes) exceeds 16 MiB is refused with
 * BASED_ERR_WORKSPACE before any launch.
 *
 * Every call looks up the array's device address (cudaGetSymbolAddress, no
 * allocation) on the device that is current, so the address is never stale;
 * the first call on a device may also load the library's device code, so make
 * that first call before any stream capture.  All calls on one device share
 * the array and it keeps the last call's contents (every call writes the parts
 * it reads), so calls whose kernels overlap on the GPU -- concurrent streams,
 * several host threads -- race on it: serialise them.
 */
based_status_t based_linattn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                         int B, int H, int L, int d_feat, int d_v,
                                         based_dtype_t dt, float eps,
                                         float* state_kv, float* state_k,
                                         based_stream_t stream);

/*
 * Sliding-window causal softmax attention:
 *   y_t = sum_{s = max(0, t-window+1)}^{t} softmax_s(q_t . k_s / sqrt(d_head)) v_s
 *   q, k, v, out  [B, H, L, d_head]  dt   (d_head in {64, 128}; 1 <= window <= 64)
 */
based_status_t based_window_attn_fwd(const void* q, const void* k, const void* v, void* out,
                                     int B, int H, int L, int d_head, int window,
                                     based_dtype_t dt, based_stream_t stream);

/*
 * Copy the last min(L, window) window keys/values of a prefill into the ring
 * caches used by based_decode_step: position p (L-window <= p < L) goes to
 * slot p mod window.  Other slots are left untouched.
 *   k, v            [B, H, L, d_head]       dt
 *   k_ring, v_ring  [B, H, window, d_head]  dt (written)
 */
based_status_t based_window_ring_fill(const void* k, const void* v, int B, int H, int L,
                                      int d_head, int window, void* k_ring, void* v_ring,
                                      based_dtype_t dt, based_stream_t stream);

/*
 * One decode step for B sequences that all sit at position `pos` (0-based; the
 * prefill length when decoding starts).  Either part may be skipped.
 *
 * Linear part (skipped when q == NULL and H == 0):
 *   q, k  [B, H, d_feat] dt;  v [B, H, d_v] dt;  out [B, H, d_v] dt (written)
 *   state_kv [B, H, 273, d_v] fp32, state_k [B, H, 273] fp32, updated in place:
 *     S += phi(k) v^T ; z += phi(k) ; out = phi(q)^T S / (phi(q) . z + eps)
 *   (the new token is folded in before the read-out: causality is inclusive).
 * Window part (skipped when wq == NULL and H_w == 0):
 *   wq, wk, wv [B, H_w, d_head] dt; wout [B, H_w, d_head] dt (written)
 *   k_ring, v_ring [B, H_w, window, d_head] dt, updated in place: slot
 *   pos mod window receives wk/wv, then softmax attention over the slots that
 *   hold positions max(0, pos-window+1) .. pos.
 */
based_status_t based_decode_step(const void* q, const void* k, const void* v,
                                 float* state_kv, float* state_k, void* out,
                                 const void* wq, const void* wk, const void* wv,
                                 void* k_ring, void* v_ring, void* wout,
                                 long long pos, int B, int H, int d_feat, int d_v,
                                 int H_w, int d_head, int window,
                                 based_dtype_t dt, float eps, based_stream_t stream);

/*
 * based_decode_step for a batch whose sequences sit at different positions
 * (prompts of different lengths; the Based README's generation example decodes
 * a batch of prompts): identical arguments, except that `pos` is a DEVICE
 * array of B int64 positions (8-byte aligned; read on the GPU; may be NULL
 * when the window part is skipped).  Only the window part uses positions:
 * sequence b's new window k/v go to slot pos[b] mod window and its softmax
 * covers the slots holding positions max(0, pos[b]-window+1) .. pos[b].  A
 * negative entry cannot be checked on the host: the kernel leaves that
 * sequence's window heads untouched (ring and wout) and records
 * BASED_ERR_INVALID_ARG, read with based_get_device_error().
 */
based_status_t based_decode_step_at(const void* q, const void* k, const void* v,
                                    float* state_kv, float* state_k, void* out,
                                    const void* wq, const void* wk, const void* wv,
                                    void* k_ring, void* v_ring, void* wout,
                                    const long long* pos, int B, int H, int d_feat, int d_v,
                                    int H_w, int d_head, int window,
                                    based_dtype_t dt, float eps, based_stream_t stream);

/*
 * Gradient of based_linattn_fwd's output (the map the "based/train" README's
 * training views share; see based_linattn_fwd):
 *   w_ts = 1 + u + u^2/2, u = q_t.k_s/sqrt(d_feat), s <= t; y_t = sum_s w_ts v_s / (sum_s w_ts + eps)
 * Given dy = dL/dy returns dq, dk, dv (fp32) over the quadratic form: for bf16
 * inputs on the tensor cores (128 x 128 tiles of the (t, s) triangle, bf16
 * operands for w, dw (1 + u) and dy / D, fp32 accumulation); for fp32 inputs
 * on CUDA cores in fp32.
 *   q, k [B, H, L, d_feat]   v, dy [B, H, L, d_v]   dt (d_feat == 16, d_v in {64, 128})
 *   dq, dk [B, H, L, d_feat] fp32,  dv [B, H, L, d_v] fp32 (written)
 *   workspace: device memory of based_linattn_bwd_workspace_bytes() bytes
 *   (BASED_ERR_WORKSPACE if smaller); its contents are scratch.
 * Arguments are checked as in based_linattn_fwd (16-byte aligned pointers,
 * finite eps >= 0) before any launch.
 */
size_t based_linattn_bwd_workspace_bytes(int B, int H, int L, int d_v);
based_status_t based_linattn_bwd(const void* q, const void* k, const void* v, const void* dy,
                                 float* dq, float* dk, float* dv, int B, int H, int L,
                                 int d_feat, int d_v, based_dtype_t dt, float eps,
                                 void* workspace, size_t workspace_bytes, based_stream_t stream);

/*
 * Gradient of based_window_attn_fwd's output:
 *   y_t = sum_{s = max(0, t-window+1)}^{t} softmax_s(q_t . k_s / sqrt(d_head)) v_s
 * Given dy returns dq, dk, dv (fp32).  bf16 inputs run on the tensor cores
 * (d_head 64 or 128): the scores and dP = dy v^T by tcgen05, P and
 * dS = P (dP - delta) rounded to bf16 as the operands of dq, dk, dv, fp32
 * accumulation.  fp32 inputs run on CUDA cores in fp32 (d_head 64).
 *   q, k, v, dy [B, H, L, d_head] dt (1 <= window <= 64)
 *   dq, dk, dv  [B, H, L, d_head] fp32 (written)
 *   workspace: based_window_attn_bwd_workspace_bytes() bytes of device memory
 *   (per query: row max, row sum, dy . y), else BASED_ERR_WORKSPACE.
 * Other d_head values: BASED_ERR_UNSUPPORTED.  Pointers must be 16-byte
 * aligned (BASED_ERR_INVALID_ARG otherwise).
 */
size_t based_window_attn_bwd_workspace_bytes(int B, int H, int L);
based_status_t based_window_attn_bwd(const void* q, const void* k, const void* v, const void* dy,
                                     float* dq, float* dk, float* dv, int B, int H, int L,
                                     int d_head, int window, based_dtype_t dt, void* workspace,
                                     size_t workspace_bytes, based_stream_t stream);

/*
 * Per-head input projection ("Базированная модель, часть 2", the paragraph on
 * the size of the hidden state: the KV and K states are made smaller by
 * projections of the layer input):
 *   y[b][h][t][d] = sum_k x[b][t][k] * w[h*D + d][k]
 *   x  [B, L, d_model]  bf16      w  [H*D, d_model]  bf16 (one output feature per row)
 *   y  [B, H, L, D]     bf16 (written)
 * bf16 only (BASED_ERR_UNSUPPORTED otherwise).  Requires d_model % 64 == 0,
 * (H*D) % 256 == 0 and D % 8 == 0 (else BASED_ERR_UNSUPPORTED).  Accumulates
 * in fp32 on the tensor cores and rounds once to bf16.
 */
based_status_t based_proj_heads_fwd(const void* x, const void* w, void* y, int B, int L,
                                    int d_model, int H, int D, based_dtype_t dt,
                                    based_stream_t stream);

/*
 * Several per-head projections of the same input in one launch (for instance
 * the q, k and v projections of a linear-attention layer and of a window
 * layer): x is streamed once for all of them.
 *   w     [sum_g H*D[g], d_model]  bf16: the n_out weight matrices stacked
 *         row-wise, projection g taking H*D[g] rows in order
 *   D     host array [n_out]: features per head of each projection
 *   y     host array [n_out] of device pointers; y[g] is [B, H, L, D[g]] bf16
 *   y[g][b][h][t][d] = sum_k x[b][t][k] * w[off_g + h*D[g] + d][k],
 *   off_g = H * (D[0] + ... + D[g-1]).
 * Requires 1 <= n_out <= 8 (BASED_ERR_INVALID_ARG otherwise), bf16,
 * d_model % 64 == 0, (H*D[g]) % 256 == 0 and D[g] % 8 == 0 for every g (else
 * BASED_ERR_UNSUPPORTED); every pointer 16-byte aligned.  The outputs must not
 * overlap each other or x.  based_proj_heads_fwd is this call with n_out = 1.
 * Runs on pairs of CTAs (thread-block clusters of two).
 */
based_status_t based_proj_heads_multi_fwd(const void* x, const void* w, int n_out, const int* D,
                                          void* const* y, int B, int L, int d_model, int H,
                                          based_dtype_t dt, based_stream_t stream);

/*
 * BaseConv block ("Базированная модель, часть 1", section "Кто виноват?":
 * y = linear(x) (.) conv(h, x)), with a dense D x D map plus bias and a
 * causal per-channel convolution of K taps:
 *   y[b][t][c] = (sum_k x[b][t][k] w[c][k] + bias[c])
 *              * sum_{j=0}^{min(K-1, t)} taps[c][j] x[b][t-j][c]
 *   x, y  [B, L, D]  bf16      w  [D, D]  bf16      bias [D], taps [D, K]  fp32
 * bf16 only; requires D % 256 == 0 and 1 <= K <= 8 (else BASED_ERR_UNSUPPORTED).
 */
based_status_t based_baseconv_fwd(const void* x, const void* w, const float* bias,
                                  const float* taps, void* y, int B, int L, int D, int K,
                                  based_dtype_t dt, based_stream_t stream);

/*
 * Test hook for the failure path of the bounded waits; not for production use.
 * Synchronises the current device, then sets, for every later launch on it:
 *   which = 0  normal operation;
 *   which = 1  the first CTA of the linear-attention prefill (bf16) leaves out
 *              the V tile load of its second chunk;
 *   which = 2  the first CTA of the window attention (bf16) leaves out its V
 *              tile load;
 * and the time after which every bounded wait gives up, wait_limit_ns > 0
 * (2e9, two seconds, is the default).  A wait on a load that was left out runs
 * out: the kernel records BASED_ERR_TIMEOUT (see based_get_device_error),
 * drains its own loads and stores in flight, releases its tensor memory and
 * returns; its outputs are then undefined.  Nothing faults and nothing is
 * left waiting.  BASED_ERR_INVALID_ARG for other values.
 */
based_status_t based_debug_stall(int which, long long wait_limit_ns);

/*
 * Synchronise `stream`, then read and clear the library's device status word
 * on the current device.  Returns BASED_OK, or the first error a kernel
 * recorded since the last call (BASED_ERR_TIMEOUT; BASED_ERR_INVALID_ARG for a
 * negative position given to based_decode_step_at), or BASED_ERR_CUDA if the
 * synchronisation itself failed.
 */
based_status_t based_get_device_error(based_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BASED_H */
