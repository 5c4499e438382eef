"""Host-only checks of the C ABI: the library builds, loads, exports every
symbol include/based.h declares, and rejects bad arguments on the host before
touching the GPU.  No kernel is launched here."""
import ctypes
import os
import re

import pytest
import torch

import linear_attention_lm_b200 as lab
from linear_attention_lm_b200 import build as lab_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "based.h")

INVALID, UNSUPPORTED = 1, 2


@pytest.fixture(scope="module")
def lib():
    lab_build.build()
    return lab.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(based_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_binding_symbols():
    assert declared_functions() == sorted(lab.EXPORTED_SYMBOLS)


def test_binding_wraps_every_symbol():
    for name in lab.EXPORTED_SYMBOLS:
        assert callable(getattr(lab, name, None)), name


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.based_abi_version() == 1


def test_built_for_sm100a(lib):
    """The build ran nvcc with the sm_100a target and nothing else (the
    command line is recorded beside the library at build time; the running
    device code is checked on a GPU by test_gpu_parity)."""
    import json
    rec = json.load(open(lab_build.RECORD_PATH))
    assert rec["arch_flags"] == ["-gencode", "arch=compute_100a,code=sm_100a"]
    gencodes = [a for a in rec["nvcc"] if a.startswith("arch=")]
    assert gencodes == ["arch=compute_100a,code=sm_100a"]


def test_status_strings(lib):
    for code, name in [(0, "BASED_OK"), (1, "BASED_ERR_INVALID_ARG"), (2, "BASED_ERR_UNSUPPORTED"),
                       (3, "BASED_ERR_CUDA"), (4, "BASED_ERR_TIMEOUT"), (5, "BASED_ERR_WORKSPACE")]:
        assert lab.based_status_string(code) == name
    assert lab.based_status_string(99) == "BASED_ERR_UNKNOWN"


def test_workspace_query_rejects_bad_args(lib):
    bad = ctypes.c_size_t(-1).value
    f = lib.based_linattn_workspace_bytes
    assert f(1, 1, 16, 8, 64, 1) == bad       # d_feat != 16
    assert f(1, 1, 16, 16, 96, 1) == bad      # d_v not 64/128
    assert f(-1, 1, 16, 16, 64, 1) == bad
    assert f(1, 1, 16, 16, 64, 7) == bad      # dtype
    assert f(1, 1, 16, 16, 64, 1) != bad


FAKE = 1 << 20  # a 16-byte-aligned non-null address; never dereferenced here


def lin_call(lib, q=FAKE, k=FAKE, v=FAKE, out=FAKE, B=1, H=1, L=8, d=16, dv=64, dt=1,
             eps=1e-6, skv=None, sk=None):
    return lib.based_linattn_fwd(q, k, v, out, B, H, L, d, dv, dt, eps, skv, sk, None, 0, None)


def test_linattn_host_validation(lib):
    assert lin_call(lib, d=8) == UNSUPPORTED
    assert lin_call(lib, dv=32) == UNSUPPORTED
    assert lin_call(lib, B=-1) == INVALID
    assert lin_call(lib, q=None) == INVALID
    assert lin_call(lib, k=FAKE + 4) == INVALID          # misaligned
    assert lin_call(lib, eps=-1.0) == INVALID
    assert lin_call(lib, eps=float("nan")) == INVALID
    assert lin_call(lib, dt=5) == INVALID
    assert lin_call(lib, skv=FAKE + 8) == INVALID
    # empty problems are valid no-ops (no launch, no pointer needed)
    assert lin_call(lib, q=None, k=None, v=None, out=None, B=0) == 0
    assert lin_call(lib, q=None, k=None, v=None, out=None, L=0) == 0


def test_linattn_workspace_required(lib):
    """A long single sequence is split across CTAs and needs workspace; a
    missing or short workspace is refused on the host."""
    need = lib.based_linattn_workspace_bytes(1, 1, 4096, 16, 64, 1)
    assert 0 < need < (1 << 26)
    assert lib.based_linattn_workspace_bytes(1, 1, 4096, 16, 64, 0) == 0  # fp32 path
    f = lib.based_linattn_fwd
    assert f(FAKE, FAKE, FAKE, FAKE, 1, 1, 4096, 16, 64, 1, 1e-6, None, None, None, 0, None) == 5
    assert f(FAKE, FAKE, FAKE, FAKE, 1, 1, 4096, 16, 64, 1, 1e-6, None, None, FAKE, need - 16,
             None) == 5


def test_window_host_validation(lib):
    f = lib.based_window_attn_fwd
    assert f(FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 64, 0, 1, None) == INVALID
    assert f(FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 64, 65, 1, None) == UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 96, 64, 1, None) == UNSUPPORTED
    assert f(None, FAKE, FAKE, FAKE, 1, 1, 8, 64, 64, 1, None) == INVALID
    assert f(None, None, None, None, 1, 1, 0, 64, 64, 1, None) == 0


def test_decode_host_validation(lib):
    f = lib.based_decode_step
    N = None
    # nothing to do
    assert f(N, N, N, N, N, N, N, N, N, N, N, N, 0, 1, 0, 16, 64, 0, 64, 64, 1, 1e-6, N) == INVALID
    # linear part missing its state
    assert f(FAKE, FAKE, FAKE, N, FAKE, FAKE, N, N, N, N, N, N, 0, 1, 1, 16, 64, 0, 64, 64, 1,
             1e-6, N) == INVALID
    # negative position
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, N, N, N, N, N, N, -1, 1, 1, 16, 64, 0, 64, 64, 1,
             1e-6, N) == INVALID
    # window part with an unsupported head dim
    assert f(N, N, N, N, N, N, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 3, 1, 0, 16, 64, 1, 32, 64, 1,
             1e-6, N) == UNSUPPORTED


def test_decode_at_host_validation(lib):
    f = lib.based_decode_step_at
    N = None
    # window part with no position array, or a misaligned one
    assert f(N, N, N, N, N, N, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, N, 2, 0, 16, 64, 1, 64, 64, 1,
             1e-6, N) == INVALID
    assert f(N, N, N, N, N, N, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 4, 2, 0, 16, 64, 1, 64,
             64, 1, 1e-6, N) == INVALID
    # the linear part alone needs no positions; its checks are based_decode_step's
    assert f(FAKE, FAKE, FAKE, N, FAKE, FAKE, N, N, N, N, N, N, N, 1, 1, 16, 64, 0, 64, 64, 1,
             1e-6, N) == INVALID  # missing state


def test_binding_decode_positions_checked():
    z = torch.zeros
    wq = z(3, 2, 64, dtype=torch.bfloat16)
    ring = z(3, 2, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="expected shape"):
        lab.based_decode_step(None, None, None, None, None, None, wq, wq, wq, ring, ring, wq,
                              pos=z(2, dtype=torch.int64))
    with pytest.raises(TypeError):
        lab.based_decode_step(None, None, None, None, None, None, wq, wq, wq, ring, ring, wq,
                              pos=z(3, dtype=torch.int32))


def test_linattn_bwd_host_validation(lib):
    f = lib.based_linattn_bwd
    ws = lib.based_linattn_bwd_workspace_bytes
    assert ws(1, 2, 100, 64) == 1 * 2 * 100 * 65 * 4
    assert ws(1, 2, 100, 96) == ctypes.c_size_t(-1).value
    # q, k, v, dy, dq, dk, dv, B, H, L, d_feat, d_v, dt, eps, workspace, bytes, stream
    A = [FAKE] * 7
    assert f(*A, 1, 2, 100, 8, 64, 1, 1e-6, FAKE, 1 << 20, None) == UNSUPPORTED   # d_feat
    assert f(*A, 1, 2, 100, 16, 96, 1, 1e-6, FAKE, 1 << 20, None) == UNSUPPORTED  # d_v
    assert f(*A, 1, 2, 100, 16, 64, 1, -1.0, FAKE, 1 << 20, None) == INVALID      # eps
    assert f(*A, 1, 2, 100, 16, 64, 1, 1e-6, FAKE, 16, None) == 5                 # workspace
    assert f(None, *A[1:], 1, 2, 100, 16, 64, 1, 1e-6, FAKE, 1 << 20, None) == INVALID
    assert f(*[None] * 7, 1, 2, 0, 16, 64, 1, 1e-6, None, 0, None) == 0           # nothing to do


def test_linattn_bwd_checks_like_the_forward(lib):
    """Alignment and eps are checked as in based_linattn_fwd."""
    f = lib.based_linattn_bwd
    A = [FAKE] * 7
    for i in range(7):  # each of q, k, v, dy, dq, dk, dv misaligned
        B = list(A)
        B[i] = FAKE + 4
        assert f(*B, 1, 2, 100, 16, 64, 1, 1e-6, FAKE, 1 << 20, None) == INVALID
    assert f(*A, 1, 2, 100, 16, 64, 1, float("inf"), FAKE, 1 << 20, None) == INVALID
    assert f(*A, 1, 2, 100, 16, 64, 1, float("nan"), FAKE, 1 << 20, None) == INVALID
    assert f(*A, 1, 2, 100, 16, 64, 1, 1e-6, FAKE + 8, 1 << 20, None) == INVALID  # workspace
    assert f(*A, 1, 2, 100, 16, 64, 7, 1e-6, FAKE, 1 << 20, None) == INVALID      # dtype


def test_window_bwd_checks_alignment(lib):
    f = lib.based_window_attn_bwd
    A = [FAKE] * 7
    for i in range(7):
        B = list(A)
        B[i] = FAKE + 2
        assert f(*B, 1, 2, 100, 64, 64, 1, FAKE, 1 << 20, None) == INVALID
    assert f(*A, 1, 2, 100, 64, 64, 1, FAKE + 4, 1 << 20, None) == INVALID       # workspace


def test_binding_checks_shapes():
    """Every wrapper checks each tensor's full shape against the sizes it
    passes to the C ABI (which cannot see them) before anything else."""
    bf = torch.bfloat16

    def z(*shape, dtype=bf):
        return torch.zeros(*shape, dtype=dtype)

    q, v = z(1, 2, 8, 16), z(1, 2, 8, 64)
    bad_calls = [
        lambda: lab.based_linattn_fwd(q, z(1, 2, 7, 16), v, v.clone()),            # k's L
        lambda: lab.based_linattn_fwd(q, q, z(1, 2, 7, 64), z(1, 2, 7, 64)),       # v's L
        lambda: lab.based_linattn_fwd(q, q, v, z(1, 2, 8, 128)),                   # out's d_v
        lambda: lab.based_linattn_fwd(q, q, v, v.clone(), 1e-6,
                                      z(1, 2, 272, 64, dtype=torch.float32)),      # state rows
        lambda: lab.based_linattn_fwd(q, q, v, v.clone(), 1e-6, None,
                                      z(1, 3, 273, dtype=torch.float32)),          # state_k heads
        lambda: lab.based_linattn_fwd_noalloc(q, q, v, z(2, 2, 8, 64)),
        lambda: lab.based_window_attn_fwd(v, v, z(1, 2, 9, 64), v.clone()),
        lambda: lab.based_window_ring_fill(v, v, z(1, 2, 63, 64), z(1, 2, 64, 64)),
        lambda: lab.based_decode_step(z(4, 2, 16), z(4, 2, 16), z(4, 2, 64),
                                      z(4, 2, 273, 64, dtype=torch.float32),
                                      z(4, 2, 273, dtype=torch.float32), z(4, 2, 32)),
        lambda: lab.based_decode_step(None, None, None, None, None, None, z(4, 2, 64),
                                      z(4, 2, 64), z(4, 2, 64), z(4, 2, 32, 64), z(4, 2, 64, 64),
                                      z(4, 2, 64), window=64),
        lambda: lab.based_linattn_bwd(q, q, v, v, z(1, 2, 8, 16, dtype=torch.float32),
                                      z(1, 2, 8, 16, dtype=torch.float32),
                                      z(1, 2, 8, 32, dtype=torch.float32)),
        lambda: lab.based_window_attn_bwd(v, v, v, v, *(z(1, 2, 8, 64, dtype=torch.float32)
                                                        for _ in range(2)),
                                          z(1, 2, 4, 64, dtype=torch.float32)),
        lambda: lab.based_proj_heads_fwd(z(1, 8, 256), z(256, 128), z(1, 16, 8, 16)),
        lambda: lab.based_baseconv_fwd(z(1, 8, 256), z(256, 256), torch.zeros(255),
                                       torch.zeros(256, 3), z(1, 8, 256)),
    ]
    for call in bad_calls:
        with pytest.raises(ValueError, match="expected shape"):
            call()


def test_binding_checks_devices():
    """A tensor on another device than q is refused (meta tensors stand in
    for a second device; nothing is launched)."""
    q = torch.zeros(1, 2, 8, 16, dtype=torch.bfloat16)
    v = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="is on meta"):
        lab.based_linattn_fwd(q, q.to("meta"), v, v.clone())
    with pytest.raises(ValueError, match="is on meta"):
        lab.based_window_attn_fwd(v, v, v, v.to("meta"))


def test_window_bwd_host_validation(lib):
    f = lib.based_window_attn_bwd
    assert lib.based_window_attn_bwd_workspace_bytes(2, 3, 100) == 2 * 3 * 100 * 3 * 4
    A = [FAKE] * 7
    # q, k, v, dy, dq, dk, dv, B, H, L, d_head, window, dt, workspace, bytes, stream
    assert f(*A, 1, 2, 100, 96, 64, 1, FAKE, 1 << 20, None) == UNSUPPORTED    # d_head (bf16: 64, 128)
    assert f(*A, 1, 2, 100, 128, 64, 0, FAKE, 1 << 20, None) == UNSUPPORTED   # d_head (fp32: 64)
    assert f(*A, 1, 2, 100, 64, 65, 1, FAKE, 1 << 20, None) == UNSUPPORTED    # window
    assert f(*A, 1, 2, 100, 64, 0, 1, FAKE, 1 << 20, None) == INVALID
    assert f(*A, 1, 2, 100, 64, 64, 1, FAKE, 16, None) == 5                   # workspace
    assert f(*[None] * 7, 1, 2, 0, 64, 64, 1, None, 0, None) == 0


def test_proj_host_validation(lib):
    f = lib.based_proj_heads_fwd
    # x, w, y, B, L, d_model, H, D, dt, stream
    assert f(FAKE, FAKE, FAKE, 1, 8, 1024, 16, 16, 0, None) == UNSUPPORTED   # fp32
    assert f(FAKE, FAKE, FAKE, 1, 8, 1000, 16, 16, 1, None) == UNSUPPORTED   # d_model % 64
    assert f(FAKE, FAKE, FAKE, 1, 8, 1024, 3, 16, 1, None) == UNSUPPORTED    # H*D % 256
    assert f(FAKE, FAKE, FAKE, 1, 8, 1024, 64, 4, 1, None) == UNSUPPORTED    # D % 8
    assert f(FAKE, FAKE, FAKE, -1, 8, 1024, 16, 16, 1, None) == INVALID
    assert f(None, FAKE, FAKE, 1, 8, 1024, 16, 16, 1, None) == INVALID
    assert f(None, None, None, 0, 8, 1024, 16, 16, 1, None) == 0             # nothing to do


def test_proj_multi_host_validation(lib):
    f = lib.based_proj_heads_multi_fwd
    D = (ctypes.c_int * 3)(16, 64, 64)
    Y = (ctypes.c_void_p * 3)(FAKE, FAKE, FAKE)
    Yn = (ctypes.c_void_p * 3)(FAKE, None, FAKE)
    d, y, yn = (ctypes.cast(a, ctypes.c_void_p) for a in (D, Y, Yn))
    # x, w, n_out, D, y, B, L, d_model, H, dt, stream
    assert f(FAKE, FAKE, 0, d, y, 1, 8, 1024, 16, 1, None) == INVALID     # no projection
    assert f(FAKE, FAKE, 9, d, y, 1, 8, 1024, 16, 1, None) == INVALID     # more than 8
    assert f(FAKE, FAKE, 3, None, y, 1, 8, 1024, 16, 1, None) == INVALID  # no D array
    assert f(FAKE, FAKE, 3, d, y, 1, 8, 1024, 16, 0, None) == UNSUPPORTED # fp32
    assert f(FAKE, FAKE, 3, d, y, 1, 8, 1024, 3, 1, None) == UNSUPPORTED  # H*D % 256
    assert f(FAKE, FAKE, 3, d, y, 1, 8, 1000, 16, 1, None) == UNSUPPORTED # d_model % 64
    assert f(FAKE, FAKE, 3, d, yn, 1, 8, 1024, 16, 1, None) == INVALID    # a null output
    assert f(None, FAKE, 3, d, y, 1, 8, 1024, 16, 1, None) == INVALID
    assert f(None, None, 3, d, yn, 0, 8, 1024, 16, 1, None) == 0          # nothing to do


def test_baseconv_host_validation(lib):
    f = lib.based_baseconv_fwd
    # x, w, bias, taps, y, B, L, D, K, dt, stream
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 1024, 3, 0, None) == UNSUPPORTED  # fp32
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 1000, 3, 1, None) == UNSUPPORTED  # D % 256
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 1024, 9, 1, None) == UNSUPPORTED  # > 8 taps
    assert f(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 1024, 0, 1, None) == INVALID
    assert f(FAKE, FAKE, None, FAKE, FAKE, 1, 8, 1024, 3, 1, None) == INVALID
    assert f(None, None, None, None, None, 1, 0, 1024, 3, 1, None) == 0


def test_binding_refuses_cpu_tensors():
    q = torch.zeros(1, 1, 8, 16, dtype=torch.bfloat16)
    v = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    g16, g64 = torch.zeros(q.shape), torch.zeros(v.shape)
    ws = torch.zeros(1 << 16, dtype=torch.uint8)
    x = torch.zeros(1, 8, 256, dtype=torch.bfloat16)
    w = torch.zeros(256, 256, dtype=torch.bfloat16)
    calls = [
        lambda: lab.based_linattn_fwd(q, q, v, v.clone()),
        lambda: lab.based_linattn_bwd(q, q, v, v, g16, g16.clone(), g64, workspace=ws),
        lambda: lab.based_window_attn_bwd(v, v, v, v, g64, g64.clone(), g64.clone(), workspace=ws),
        lambda: lab.based_proj_heads_fwd(x, w, torch.zeros(1, 16, 8, 16, dtype=torch.bfloat16)),
        lambda: lab.based_baseconv_fwd(x, w, torch.zeros(256), torch.zeros(256, 3), x.clone()),
    ]
    for call in calls:
        with pytest.raises(ValueError):
            call()


def test_binding_checks_dtypes():
    q = torch.zeros(1, 1, 8, 16, dtype=torch.bfloat16)
    v32 = torch.zeros(1, 1, 8, 64, dtype=torch.float32)
    with pytest.raises(TypeError):  # mixed q/v dtypes
        lab.based_linattn_fwd(q, q, v32, v32.clone())
    with pytest.raises(TypeError):  # int tensors
        lab.based_window_attn_fwd(*(torch.zeros(1, 1, 8, 64, dtype=torch.int32) for _ in range(4)))


def test_missing_library_fails_loudly(tmp_path):
    saved = lab._lib
    try:
        lab._lib = None
        with pytest.raises(RuntimeError):
            lab.load_library(str(tmp_path / "nope.so"))
    finally:
        lab._lib = saved
