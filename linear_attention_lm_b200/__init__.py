"""Python binding of the B200 Based attention library (``libbased.so``).

The functions named ``based_*`` mirror the C ABI in ``include/based.h`` one to
one: they only derive sizes from the tensors' shapes, check every tensor's
shape, dtype, device and contiguity against those sizes (the C ABI cannot see
them), pass raw device pointers and the CUDA stream through ctypes, and turn a
non-OK status into ``BasedError``.  Every step of the computation
runs in the library's CUDA kernels; there is no CPU or PyTorch fallback -- if
the library is missing or cannot be loaded, every call raises.

The lower-case helpers (``linattn``, ``window_attn``, ``decode_step``, ...)
allocate outputs with torch and call the ``based_*`` functions.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from .inputs import WORKLOADS, Workload  # noqa: F401  (re-exported for callers)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbased.so")
NUM_FEATURES = 273
D_FEAT = 16

BASED_F32, BASED_BF16 = 0, 1
_STATUS = {0: "BASED_OK", 1: "BASED_ERR_INVALID_ARG", 2: "BASED_ERR_UNSUPPORTED",
           3: "BASED_ERR_CUDA", 4: "BASED_ERR_TIMEOUT", 5: "BASED_ERR_WORKSPACE"}
EXPORTED_SYMBOLS = ("based_abi_version", "based_binary_version", "based_status_string",
                    "based_linattn_workspace_bytes", "based_linattn_fwd",
                    "based_linattn_fwd_noalloc",
                    "based_window_attn_fwd", "based_window_ring_fill", "based_decode_step",
                    "based_decode_step_at",
                    "based_proj_heads_fwd", "based_proj_heads_multi_fwd", "based_baseconv_fwd",
                    "based_linattn_bwd_workspace_bytes", "based_linattn_bwd",
                    "based_window_attn_bwd_workspace_bytes", "based_window_attn_bwd",
                    "based_debug_stall", "based_get_device_error")


class BasedError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {_STATUS.get(status, status)}")
        self.status = status


_lock = threading.Lock()
_lib = None
_vp, _fp = ctypes.c_void_p, ctypes.POINTER(ctypes.c_float)
_i, _f, _ll, _sz = ctypes.c_int, ctypes.c_float, ctypes.c_longlong, ctypes.c_size_t


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libbased.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                f"CUDA library {path} is missing; build it with "
                "`python -m linear_attention_lm_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(path)
        lib.based_abi_version.restype = _i
        lib.based_binary_version.restype = _i
        lib.based_status_string.argtypes = [_i]
        lib.based_status_string.restype = ctypes.c_char_p
        lib.based_linattn_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i]
        lib.based_linattn_workspace_bytes.restype = _sz
        lib.based_linattn_fwd.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f,
                                          _vp, _vp, _vp, _sz, _vp]
        lib.based_linattn_fwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                                  _f, _vp, _vp, _vp]
        lib.based_window_attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]
        lib.based_window_ring_fill.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _i, _vp]
        lib.based_decode_step.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                          _vp, _vp, _ll, _i, _i, _i, _i, _i, _i, _i, _i, _f,
                                          _vp]
        lib.based_decode_step_at.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                             _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                                             _f, _vp]
        lib.based_linattn_bwd_workspace_bytes.argtypes = [_i, _i, _i, _i]
        lib.based_linattn_bwd_workspace_bytes.restype = _sz
        lib.based_linattn_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                                          _i, _f, _vp, _sz, _vp]
        lib.based_window_attn_bwd_workspace_bytes.argtypes = [_i, _i, _i]
        lib.based_window_attn_bwd_workspace_bytes.restype = _sz
        lib.based_window_attn_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                              _i, _i, _vp, _sz, _vp]
        lib.based_proj_heads_fwd.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]
        lib.based_proj_heads_multi_fwd.argtypes = [_vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i,
                                                   _vp]
        lib.based_baseconv_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]
        lib.based_get_device_error.argtypes = [_vp]
        lib.based_debug_stall.argtypes = [_i, _ll]
        for name in ("based_linattn_fwd", "based_linattn_fwd_noalloc", "based_window_attn_fwd",
                     "based_window_ring_fill", "based_decode_step", "based_decode_step_at",
                     "based_proj_heads_fwd", "based_proj_heads_multi_fwd",
                     "based_baseconv_fwd", "based_linattn_bwd", "based_window_attn_bwd",
                     "based_debug_stall", "based_get_device_error"):
            getattr(lib, name).restype = _i
        _lib = lib
        return lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return BASED_F32
    if t.dtype == torch.bfloat16:
        return BASED_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr() or None


def _device_of(t) -> torch.device:
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    return t.device


def _cuda(device: torch.device) -> torch.device:
    if device.type != "cuda":
        raise ValueError("tensors must live on a CUDA device")
    return device


def _expect(t, shape, name: str, device: torch.device):
    """t (if given) must have exactly this shape and sit on this device."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _torch_stream(stream, device) -> torch.cuda.Stream:
    """The caller's stream as a torch stream object (a raw cudaStream_t handle
    is wrapped, not copied), so that workspaces can be allocated on it."""
    if stream is None:
        return torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        return stream
    return torch.cuda.ExternalStream(int(stream), device=device)


def _workspace(nbytes: int, workspace, device, ts, name: str):
    """The caller's workspace (checked) or a new one allocated on the launch
    stream ts, so the caching allocator does not hand it out again while the
    kernels on ts still use it."""
    if workspace is None:
        if not nbytes:
            return None, 0
        with torch.cuda.stream(ts):
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    elif workspace.device != device:
        raise ValueError(f"{name}: workspace is on {workspace.device}, expected {device}")
    return workspace, workspace.numel() * workspace.element_size()


def _check(fn: str, status: int):
    if status != 0:
        raise BasedError(fn, status)


def _same_dtype(*ts):
    ts = [t for t in ts if t is not None]
    for t in ts[1:]:
        if t.dtype != ts[0].dtype:
            raise TypeError("q/k/v/out must share one dtype")
    return _dtype_code(ts[0])


def _f32(t):
    if t is not None and t.dtype != torch.float32:
        raise TypeError("states must be float32")
    return _ptr(t)


# ---------------------------------------------------------------------------
# one-to-one wrappers of the C entry points
# ---------------------------------------------------------------------------

def based_abi_version() -> int:
    return load_library().based_abi_version()


def based_binary_version() -> int:
    """SM version of the loaded device code (100 for sm_100a; -1 without a GPU)."""
    return load_library().based_binary_version()


def based_status_string(status: int) -> str:
    return load_library().based_status_string(int(status)).decode()


def based_linattn_workspace_bytes(B, H, L, d_feat, d_v, dt) -> int:
    n = load_library().based_linattn_workspace_bytes(B, H, L, d_feat, d_v, dt)
    if n == ctypes.c_size_t(-1).value:
        raise BasedError("based_linattn_workspace_bytes", 1)
    return n


def _linattn_shapes(q, k, v, out, state_kv, state_k):
    dev = _device_of(q)
    if q.dim() != 4 or not isinstance(v, torch.Tensor) or v.dim() != 4:
        raise ValueError("q, k, v, out must be [B, H, L, d]")
    B, H, L, d = q.shape
    d_v = v.shape[-1]
    _expect(k, (B, H, L, d), "k", dev)
    _expect(v, (B, H, L, d_v), "v", dev)
    _expect(out, (B, H, L, d_v), "out", dev)
    _expect(state_kv, (B, H, NUM_FEATURES, d_v), "state_kv", dev)
    _expect(state_k, (B, H, NUM_FEATURES), "state_k", dev)
    return dev, B, H, L, d, d_v


def based_linattn_fwd(q, k, v, out, eps: float = 1e-6, state_kv=None, state_k=None,
                      workspace=None, stream=None):
    dev, B, H, L, d, d_v = _linattn_shapes(q, k, v, out, state_kv, state_k)
    dt = _same_dtype(q, k, v, out)
    _cuda(dev)
    ts = _torch_stream(stream, dev)
    with torch.cuda.device(dev):
        nbytes = based_linattn_workspace_bytes(B, H, L, d, d_v, dt) if workspace is None else 0
        workspace, ws_bytes = _workspace(nbytes, workspace, dev, ts, "based_linattn_fwd")
        st = load_library().based_linattn_fwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, L, d, d_v, dt, float(eps),
            _f32(state_kv), _f32(state_k), _ptr(workspace), ws_bytes, ts.cuda_stream)
    _check("based_linattn_fwd", st)
    return out


def based_linattn_fwd_noalloc(q, k, v, out, eps: float = 1e-6, state_kv=None, state_k=None,
                              stream=None):
    """based_linattn_fwd without a workspace: for callers that must not
    allocate device memory (the library's fixed 16 MiB scratch array is used
    instead; calls on one device must not overlap on the GPU)."""
    dev, B, H, L, d, d_v = _linattn_shapes(q, k, v, out, state_kv, state_k)
    dt = _same_dtype(q, k, v, out)
    _cuda(dev)
    ts = _torch_stream(stream, dev)
    with torch.cuda.device(dev):
        st = load_library().based_linattn_fwd_noalloc(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, L, d, d_v, dt, float(eps),
            _f32(state_kv), _f32(state_k), ts.cuda_stream)
    _check("based_linattn_fwd_noalloc", st)
    return out


def based_window_attn_fwd(q, k, v, out, window: int = 64, stream=None):
    dev = _device_of(q)
    if q.dim() != 4:
        raise ValueError("q, k, v, out must be [B, H, L, d_head]")
    for t, name in ((k, "k"), (v, "v"), (out, "out")):
        _expect(t, q.shape, name, dev)
    B, H, L, dh = q.shape
    dt = _same_dtype(q, k, v, out)
    _cuda(dev)
    with torch.cuda.device(dev):
        st = load_library().based_window_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, L,
                                                  dh, int(window), dt,
                                                  _torch_stream(stream, dev).cuda_stream)
    _check("based_window_attn_fwd", st)
    return out


def based_window_ring_fill(k, v, k_ring, v_ring, window: int = 64, stream=None):
    dev = _device_of(k)
    if k.dim() != 4:
        raise ValueError("k, v must be [B, H, L, d_head]")
    B, H, L, dh = k.shape
    _expect(v, k.shape, "v", dev)
    _expect(k_ring, (B, H, int(window), dh), "k_ring", dev)
    _expect(v_ring, (B, H, int(window), dh), "v_ring", dev)
    dt = _same_dtype(k, v, k_ring, v_ring)
    _cuda(dev)
    with torch.cuda.device(dev):
        st = load_library().based_window_ring_fill(_ptr(k), _ptr(v), B, H, L, dh, int(window),
                                                   _ptr(k_ring), _ptr(v_ring), dt,
                                                   _torch_stream(stream, dev).cuda_stream)
    _check("based_window_ring_fill", st)


def based_decode_step(q, k, v, state_kv, state_k, out, wq=None, wk=None, wv=None, k_ring=None,
                      v_ring=None, wout=None, pos=0, window: int = 64,
                      eps: float = 1e-6, stream=None):
    """One decode step.  `pos` is an int (every sequence at that position) or
    an int64 CUDA tensor of B per-sequence positions (based_decode_step_at)."""
    ref = q if q is not None else wq
    dev = _device_of(ref)
    B = ref.shape[0]
    H, d_feat, d_v = (q.shape[1], q.shape[2], v.shape[-1]) if q is not None else (0, D_FEAT, 64)
    H_w, d_head = (wq.shape[1], wq.shape[2]) if wq is not None else (0, 64)
    if q is not None:
        if q.dim() != 3:
            raise ValueError("q, k must be [B, H, d_feat]")
        _expect(k, (B, H, d_feat), "k", dev)
        _expect(v, (B, H, d_v), "v", dev)
        _expect(out, (B, H, d_v), "out", dev)
        _expect(state_kv, (B, H, NUM_FEATURES, d_v), "state_kv", dev)
        _expect(state_k, (B, H, NUM_FEATURES), "state_k", dev)
    if wq is not None:
        if wq.dim() != 3:
            raise ValueError("wq, wk, wv must be [B, H_w, d_head]")
        for t, name in ((wk, "wk"), (wv, "wv"), (wout, "wout")):
            _expect(t, (B, H_w, d_head), name, dev)
        for t, name in ((k_ring, "k_ring"), (v_ring, "v_ring")):
            _expect(t, (B, H_w, int(window), d_head), name, dev)
    per_seq = isinstance(pos, torch.Tensor)
    if per_seq:
        _expect(pos, (B,), "pos", dev)
        if pos.dtype != torch.int64:
            raise TypeError("pos must be an int64 tensor of B positions")
    dt = _same_dtype(q, k, v, out, wq, wk, wv, k_ring, v_ring, wout)
    _cuda(dev)
    lib = load_library()
    args = (_ptr(q), _ptr(k), _ptr(v), _f32(state_kv), _f32(state_k), _ptr(out), _ptr(wq),
            _ptr(wk), _ptr(wv), _ptr(k_ring), _ptr(v_ring), _ptr(wout))
    tail = (B, H, d_feat, d_v, H_w, d_head, int(window), dt, float(eps))
    with torch.cuda.device(dev):
        if per_seq:
            st = lib.based_decode_step_at(*args, _ptr(pos), *tail,
                                          _torch_stream(stream, dev).cuda_stream)
        else:
            st = lib.based_decode_step(*args, int(pos), *tail,
                                       _torch_stream(stream, dev).cuda_stream)
    _check("based_decode_step_at" if per_seq else "based_decode_step", st)


def based_decode_step_at(q, k, v, state_kv, state_k, out, wq, wk, wv, k_ring, v_ring, wout,
                         pos, window: int = 64, eps: float = 1e-6, stream=None):
    """based_decode_step with per-sequence positions: pos is an int64 CUDA
    tensor [B]."""
    if not isinstance(pos, torch.Tensor):
        raise TypeError("pos must be an int64 tensor of B positions")
    based_decode_step(q, k, v, state_kv, state_k, out, wq, wk, wv, k_ring, v_ring, wout, pos,
                      window, eps, stream)


def based_linattn_bwd_workspace_bytes(B, H, L, d_v) -> int:
    n = load_library().based_linattn_bwd_workspace_bytes(B, H, L, d_v)
    if n == ctypes.c_size_t(-1).value:
        raise BasedError("based_linattn_bwd_workspace_bytes", 1)
    return n


def based_linattn_bwd(q, k, v, dy, dq, dk, dv, eps: float = 1e-6, workspace=None, stream=None):
    """Gradients dq, dk, dv (float32, written) of based_linattn_fwd given dy."""
    dev, B, H, L, d, d_v = _linattn_shapes(q, k, v, dy, None, None)
    _expect(dq, q.shape, "dq", dev)
    _expect(dk, q.shape, "dk", dev)
    _expect(dv, v.shape, "dv", dev)
    dt = _same_dtype(q, k, v, dy)
    _cuda(dev)
    ts = _torch_stream(stream, dev)
    with torch.cuda.device(dev):
        nbytes = based_linattn_bwd_workspace_bytes(B, H, L, d_v) if workspace is None else 0
        workspace, ws_bytes = _workspace(nbytes, workspace, dev, ts, "based_linattn_bwd")
        st = load_library().based_linattn_bwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(dy), _f32(dq), _f32(dk), _f32(dv), B, H, L, d, d_v,
            dt, float(eps), _ptr(workspace), ws_bytes, ts.cuda_stream)
    _check("based_linattn_bwd", st)
    return dq, dk, dv


def based_window_attn_bwd_workspace_bytes(B, H, L) -> int:
    n = load_library().based_window_attn_bwd_workspace_bytes(B, H, L)
    if n == ctypes.c_size_t(-1).value:
        raise BasedError("based_window_attn_bwd_workspace_bytes", 1)
    return n


def based_window_attn_bwd(q, k, v, dy, dq, dk, dv, window: int = 64, workspace=None,
                          stream=None):
    """Gradients dq, dk, dv (float32, written) of based_window_attn_fwd given dy."""
    dev = _device_of(q)
    if q.dim() != 4:
        raise ValueError("q, k, v, dy must be [B, H, L, d_head]")
    for t, name in ((k, "k"), (v, "v"), (dy, "dy"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        _expect(t, q.shape, name, dev)
    B, H, L, dh = q.shape
    dt = _same_dtype(q, k, v, dy)
    _cuda(dev)
    ts = _torch_stream(stream, dev)
    with torch.cuda.device(dev):
        nbytes = based_window_attn_bwd_workspace_bytes(B, H, L) if workspace is None else 0
        workspace, ws_bytes = _workspace(nbytes, workspace, dev, ts, "based_window_attn_bwd")
        st = load_library().based_window_attn_bwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(dy), _f32(dq), _f32(dk), _f32(dv), B, H, L, dh,
            int(window), dt, _ptr(workspace), ws_bytes, ts.cuda_stream)
    _check("based_window_attn_bwd", st)
    return dq, dk, dv


def based_proj_heads_fwd(x, w, y, stream=None):
    """x [B, L, d_model], w [H*D, d_model] -> y [B, H, L, D] (bf16, written)."""
    dev = _device_of(x)
    if x.dim() != 3 or y.dim() != 4:
        raise ValueError("x must be [B, L, d_model] and y [B, H, L, D]")
    B, L, d_model = x.shape
    H, D = y.shape[1], y.shape[3]
    _expect(w, (H * D, d_model), "w", dev)
    _expect(y, (B, H, L, D), "y", dev)
    dt = _same_dtype(x, w, y)
    _cuda(dev)
    with torch.cuda.device(dev):
        st = load_library().based_proj_heads_fwd(_ptr(x), _ptr(w), _ptr(y), B, L, d_model, H, D,
                                                 dt, _torch_stream(stream, dev).cuda_stream)
    _check("based_proj_heads_fwd", st)
    return y


def based_proj_heads_multi_fwd(x, w, ys, stream=None):
    """x [B, L, d_model], w [H*(D_0+...+D_{n-1}), d_model] -> ys[g] [B, H, L, D_g]
    (bf16, written), every projection in one launch."""
    dev = _device_of(x)
    ys = list(ys)
    if x.dim() != 3 or not ys or any(y.dim() != 4 for y in ys):
        raise ValueError("x must be [B, L, d_model] and every y [B, H, L, D]")
    B, L, d_model = x.shape
    H = ys[0].shape[1]
    Ds = [int(y.shape[3]) for y in ys]
    _expect(w, (H * sum(Ds), d_model), "w", dev)
    for g, y in enumerate(ys):
        _expect(y, (B, H, L, Ds[g]), f"ys[{g}]", dev)
    dt = _same_dtype(x, w, *ys)
    _cuda(dev)
    d_arr = (ctypes.c_int * len(ys))(*Ds)
    y_arr = (ctypes.c_void_p * len(ys))(*[_ptr(y) for y in ys])
    with torch.cuda.device(dev):
        st = load_library().based_proj_heads_multi_fwd(
            _ptr(x), _ptr(w), len(ys), ctypes.cast(d_arr, ctypes.c_void_p),
            ctypes.cast(y_arr, ctypes.c_void_p), B, L, d_model, H, dt,
            _torch_stream(stream, dev).cuda_stream)
    _check("based_proj_heads_multi_fwd", st)
    return ys


def based_baseconv_fwd(x, w, bias, taps, y, stream=None):
    """x, y [B, L, D] bf16; w [D, D] bf16; bias [D], taps [D, K] float32."""
    dev = _device_of(x)
    if x.dim() != 3 or taps.dim() != 2:
        raise ValueError("x must be [B, L, D] and taps [D, K]")
    B, L, D = x.shape
    K = taps.shape[-1]
    _expect(w, (D, D), "w", dev)
    _expect(bias, (D,), "bias", dev)
    _expect(taps, (D, K), "taps", dev)
    _expect(y, (B, L, D), "y", dev)
    dt = _same_dtype(x, w, y)
    _cuda(dev)
    with torch.cuda.device(dev):
        st = load_library().based_baseconv_fwd(_ptr(x), _ptr(w), _f32(bias), _f32(taps), _ptr(y),
                                               B, L, D, K, dt,
                                               _torch_stream(stream, dev).cuda_stream)
    _check("based_baseconv_fwd", st)
    return y


STALL_NONE, STALL_LINATTN_V, STALL_WINDOW_V = 0, 1, 2


def based_debug_stall(which: int, wait_limit_ns: int = 2_000_000_000):
    """Test hook: make the first CTA of the chosen kernel leave one load out
    so its bounded wait runs out after wait_limit_ns (which = 0 restores
    normal operation)."""
    _check("based_debug_stall", load_library().based_debug_stall(int(which), int(wait_limit_ns)))


def based_get_device_error(stream=None) -> int:
    if stream is None:
        handle = torch.cuda.current_stream().cuda_stream
    elif isinstance(stream, torch.cuda.Stream):
        handle = stream.cuda_stream
    else:
        handle = int(stream)
    return load_library().based_get_device_error(handle)


# ---------------------------------------------------------------------------
# allocating helpers
# ---------------------------------------------------------------------------

def linattn(q, k, v, eps: float = 1e-6, return_state: bool = False, stream=None):
    """y [B,H,L,d_v] (and the final fp32 states S [B,H,273,d_v], z [B,H,273])."""
    B, H, L, _ = q.shape
    out = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    S = z = None
    if return_state:
        S = torch.empty((B, H, NUM_FEATURES, v.shape[-1]), dtype=torch.float32, device=v.device)
        z = torch.empty((B, H, NUM_FEATURES), dtype=torch.float32, device=v.device)
    based_linattn_fwd(q, k, v, out, eps, S, z, stream=stream)
    return (out, S, z) if return_state else out


def window_attn(q, k, v, window: int = 64, stream=None):
    out = torch.empty_like(q)
    return based_window_attn_fwd(q, k, v, out, window, stream=stream)


def window_ring_fill(k, v, window: int = 64, stream=None):
    B, H, _, dh = k.shape
    k_ring = torch.zeros((B, H, window, dh), dtype=k.dtype, device=k.device)
    v_ring = torch.zeros_like(k_ring)
    based_window_ring_fill(k, v, k_ring, v_ring, window, stream=stream)
    return k_ring, v_ring


def proj_heads(x, w, H: int, stream=None):
    """x W^T split into H heads: [B, L, d_model] x [H*D, d_model] -> [B, H, L, D]."""
    B, L, _ = x.shape
    y = torch.empty((B, H, L, w.shape[0] // H), dtype=x.dtype, device=x.device)
    return based_proj_heads_fwd(x, w, y, stream=stream)


def proj_heads_multi(x, w, H: int, Ds, stream=None):
    """Several per-head projections of x in one launch: w stacks H*D_g rows per
    projection; returns the list of [B, H, L, D_g] outputs."""
    B, L, _ = x.shape
    ys = [torch.empty((B, H, L, D), dtype=x.dtype, device=x.device) for D in Ds]
    return based_proj_heads_multi_fwd(x, w, ys, stream=stream)


def baseconv(x, w, bias, taps, stream=None):
    """linear(x) * conv(taps, x): [B, L, D] -> [B, L, D]."""
    y = torch.empty_like(x)
    return based_baseconv_fwd(x, w, bias, taps, y, stream=stream)


def linattn_grad(q, k, v, dy, eps: float = 1e-6, stream=None):
    """(dq, dk, dv) in float32 for the linear attention's output gradient dy."""
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty(k.shape, dtype=torch.float32, device=k.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=v.device)
    return based_linattn_bwd(q, k, v, dy, dq, dk, dv, eps, stream=stream)


def window_grad(q, k, v, dy, window: int = 64, stream=None):
    """(dq, dk, dv) in float32 for the window attention's output gradient dy."""
    dq, dk, dv = (torch.empty(t.shape, dtype=torch.float32, device=t.device) for t in (q, k, v))
    return based_window_attn_bwd(q, k, v, dy, dq, dk, dv, window, stream=stream)
