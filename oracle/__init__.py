"""fp64 CPU oracle for the Based attention path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and its ``--impl reference`` arm) may import this package.  The product
(the CUDA library ``linear_attention_lm_b200`` and its binding) never does,
and this package imports nothing from the product.

The arithmetic lives in ``based_oracle.c`` (plain C, double precision, no
fast-math, no FMA contraction); this module compiles it once with gcc into
``oracle/_build/`` and marshals numpy float64 arrays through ctypes.  Each
wrapper names the passage the C routine follows:

* ``phi`` -- the second-order Taylor feature map ("Базированная модель,
  часть 2", section "Что за линейное внимание?"), applied to x / d^(1/4).
* ``linattn_recurrent`` / ``linattn_quadratic`` / ``linattn_chunked`` -- the
  three training views of causal linear attention listed in the
  "based/train" README (linear, quadratic, fla_parallel).
* ``window_attn`` -- exact softmax attention over a sliding window (Based
  README, introduction, item 1; window 64).
* ``decode_linear`` / ``decode_window`` -- one recurrent generation step
  over the KV / K states (blog post part 2, state-size paragraph) and over a
  ring cache of the last W window keys/values.
* ``ring_fill`` -- the ring cache a prefill hands to decoding: slot p mod W
  holds position p for the last min(L, W) positions (the window of the Based
  README, introduction, item 1, kept as a ring).
* ``proj_heads`` -- x W^T split into heads (blog post part 2, state-size
  paragraph: the states are made smaller by projections of the input).
* ``baseconv`` -- y = linear(x) (.) conv(h, x) ("Базированная модель, часть 1",
  section "Кто виноват?"), a dense map with bias gated by a causal per-channel
  convolution.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, brute force on tiny inputs, library softmax attention,
cross-view agreement and invariants); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "based_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libbased_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile based_oracle.c with gcc (no fast-math, no FMA contraction)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread",
               "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_num_features.argtypes = [ctypes.c_int]
            lib.oracle_num_features.restype = ctypes.c_int
            lib.oracle_phi.argtypes = [_dp, ctypes.c_int, _dp]
            lib.oracle_phi.restype = None
            lib.oracle_linattn_recurrent.argtypes = [
                _dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_double, _dp, _dp, _dp, _dp, _dp, ctypes.c_int]
            lib.oracle_linattn_recurrent.restype = None
            lib.oracle_linattn_quadratic.argtypes = [
                _dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_double, _dp, ctypes.c_int]
            lib.oracle_linattn_quadratic.restype = None
            lib.oracle_linattn_chunked.argtypes = [
                _dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_double, _ip, ctypes.c_int, _dp, ctypes.c_int]
            lib.oracle_linattn_chunked.restype = ctypes.c_int
            lib.oracle_window_attn.argtypes = [
                _dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                _dp, ctypes.c_int]
            lib.oracle_window_attn.restype = None
            lib.oracle_decode_linear.argtypes = [
                _dp, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_double, _dp]
            lib.oracle_decode_linear.restype = None
            lib.oracle_decode_window.argtypes = [
                _dp, _dp, _dp, _dp, _dp, ctypes.c_longlong, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, _dp]
            lib.oracle_decode_window.restype = None
            _i = ctypes.c_int
            lib.oracle_proj_heads.argtypes = [_dp, _dp, _dp, _i, _i, _i, _i, _i, _i]
            lib.oracle_proj_heads.restype = None
            lib.oracle_baseconv.argtypes = [_dp, _dp, _dp, _dp, _dp, _i, _i, _i, _i, _i]
            lib.oracle_baseconv.restype = None
            _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def num_features(d: int) -> int:
    return _load().oracle_num_features(int(d))


def phi(x) -> np.ndarray:
    """phi(x) over the last axis: [..., d] -> [..., 1 + d + d*d]."""
    x = _f64(x)
    d = x.shape[-1]
    F = num_features(d)
    flat = x.reshape(-1, d)
    out = np.empty((flat.shape[0], F), dtype=np.float64)
    lib = _load()
    for i in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[i])
        orow = out[i]
        lib.oracle_phi(_ptr(row), d, orow.ctypes.data_as(_dp))
    return out.reshape(x.shape[:-1] + (F,))


def _lin_shapes(q, k, v):
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.shape != k.shape or q.shape[:-1] != v.shape[:-1]:
        raise ValueError(f"shape mismatch q{q.shape} k{k.shape} v{v.shape}")
    L, d, dv = q.shape[-2], q.shape[-1], v.shape[-1]
    n = int(np.prod(q.shape[:-2])) if q.ndim > 2 else 1
    return q, k, v, n, L, d, dv


def linattn_recurrent(q, k, v, eps: float = 1e-6, S0=None, z0=None,
                      return_state: bool = False, threads: int | None = None):
    """Recurrent view: q,k [..., L, d], v [..., L, dv] -> y [..., L, dv].

    S0/z0 ([..., F, dv] / [..., F]) continue from a carried state; with
    return_state the final (S, z) are returned too."""
    q, k, v, n, L, d, dv = _lin_shapes(q, k, v)
    F = num_features(d)
    lead = q.shape[:-2]
    y = np.empty(lead + (L, dv), dtype=np.float64)
    S0 = None if S0 is None else _f64(S0).reshape(n, F, dv)
    z0 = None if z0 is None else _f64(z0).reshape(n, F)
    S1 = np.empty(lead + (F, dv), dtype=np.float64) if return_state else None
    z1 = np.empty(lead + (F,), dtype=np.float64) if return_state else None
    _load().oracle_linattn_recurrent(
        _ptr(q), _ptr(k), _ptr(v), n, L, d, dv, float(eps), _ptr(S0), _ptr(z0),
        _ptr(y), _ptr(S1), _ptr(z1), threads or default_threads())
    return (y, S1, z1) if return_state else y


def linattn_quadratic(q, k, v, eps: float = 1e-6, threads: int | None = None):
    """Quadratic masked view, O(L^2) per sequence."""
    q, k, v, n, L, d, dv = _lin_shapes(q, k, v)
    y = np.empty(q.shape[:-2] + (L, dv), dtype=np.float64)
    _load().oracle_linattn_quadratic(_ptr(q), _ptr(k), _ptr(v), n, L, d, dv,
                                     float(eps), _ptr(y), threads or default_threads())
    return y


def linattn_chunked(q, k, v, bounds, eps: float = 1e-6, threads: int | None = None):
    """Chunked view over the partition bounds[0]=0 < ... < bounds[-1]=L."""
    q, k, v, n, L, d, dv = _lin_shapes(q, k, v)
    b = np.ascontiguousarray(np.asarray(bounds, dtype=np.int32))
    y = np.empty(q.shape[:-2] + (L, dv), dtype=np.float64)
    rc = _load().oracle_linattn_chunked(_ptr(q), _ptr(k), _ptr(v), n, L, d, dv,
                                        float(eps), b.ctypes.data_as(_ip), len(b) - 1,
                                        _ptr(y), threads or default_threads())
    if rc != 0:
        raise ValueError("bounds is not a partition of [0, L)")
    return y


def window_attn(q, k, v, window: int = 64, threads: int | None = None):
    """Sliding-window causal softmax attention: [..., L, dh] -> [..., L, dh]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must share one shape")
    L, dh = q.shape[-2], q.shape[-1]
    n = int(np.prod(q.shape[:-2])) if q.ndim > 2 else 1
    y = np.empty(q.shape, dtype=np.float64)
    _load().oracle_window_attn(_ptr(q), _ptr(k), _ptr(v), n, L, dh, int(window),
                               _ptr(y), threads or default_threads())
    return y


def decode_linear(q, k, v, S, z, eps: float = 1e-6):
    """One decode step of the linear part. S [..., F, dv] and z [..., F] must be
    float64 C-contiguous arrays; they are updated in place. Returns y [..., dv]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    if S.dtype != np.float64 or not S.flags.c_contiguous:
        raise ValueError("S must be a C-contiguous float64 array")
    if z.dtype != np.float64 or not z.flags.c_contiguous:
        raise ValueError("z must be a C-contiguous float64 array")
    d, dv = q.shape[-1], v.shape[-1]
    n = int(np.prod(q.shape[:-1])) if q.ndim > 1 else 1
    y = np.empty(v.shape, dtype=np.float64)
    _load().oracle_decode_linear(_ptr(q), _ptr(k), _ptr(v), _ptr(S), _ptr(z), n, d, dv,
                                 float(eps), _ptr(y))
    return y


def decode_window(q, k, v, k_ring, v_ring, pos: int, window: int = 64):
    """One decode step of the window part; rings [..., W, dh] float64, in place."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    for r in (k_ring, v_ring):
        if r.dtype != np.float64 or not r.flags.c_contiguous:
            raise ValueError("rings must be C-contiguous float64 arrays")
    dh = q.shape[-1]
    n = int(np.prod(q.shape[:-1])) if q.ndim > 1 else 1
    y = np.empty(q.shape, dtype=np.float64)
    _load().oracle_decode_window(_ptr(q), _ptr(k), _ptr(v), _ptr(k_ring), _ptr(v_ring),
                                 int(pos), n, dh, int(window), _ptr(y))
    return y


def ring_fill(k, v, window: int = 64):
    """Rings [..., W, dh] (float64) after a prefill of k, v [..., L, dh]:
    position p of the last min(L, W) positions sits in slot p mod W; slots
    that no position reached are zero.  Pure data movement, no arithmetic."""
    k, v = _f64(k), _f64(v)
    if k.shape != v.shape:
        raise ValueError("k, v must share one shape")
    L, dh = k.shape[-2], k.shape[-1]
    W = int(window)
    k_ring = np.zeros(k.shape[:-2] + (W, dh), dtype=np.float64)
    v_ring = np.zeros_like(k_ring)
    for p in range(max(0, L - W), L):
        k_ring[..., p % W, :] = k[..., p, :]
        v_ring[..., p % W, :] = v[..., p, :]
    return k_ring, v_ring


def proj_heads(x, w, H: int, threads: int | None = None) -> np.ndarray:
    """x [B, L, Dm], w [H*D, Dm] -> y [B, H, L, D] = x W^T split into heads."""
    x, w = _f64(x), _f64(w)
    B, L, Dm = x.shape
    N = w.shape[0]
    if w.shape[1] != Dm or N % H:
        raise ValueError("w must be [H*D, Dm]")
    D = N // H
    y = np.zeros((B, H, L, D), dtype=np.float64)
    _load().oracle_proj_heads(_ptr(x), _ptr(w), _ptr(y), B, L, Dm, H, D,
                              threads or default_threads())
    return y


def baseconv(x, w, bias, h, threads: int | None = None) -> np.ndarray:
    """x [B, L, D], w [D, D], bias [D], h [D, K] -> y [B, L, D]."""
    x, w, bias, h = _f64(x), _f64(w), _f64(bias), _f64(h)
    B, L, D = x.shape
    if w.shape != (D, D) or bias.shape != (D,) or h.ndim != 2 or h.shape[0] != D:
        raise ValueError("shapes: w [D, D], bias [D], h [D, K]")
    K = h.shape[1]
    y = np.zeros((B, L, D), dtype=np.float64)
    _load().oracle_baseconv(_ptr(x), _ptr(w), _ptr(bias), _ptr(h), _ptr(y), B, L, D, K,
                            threads or default_threads())
    return y
