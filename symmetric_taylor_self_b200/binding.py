"""ctypes binding of libsata (include/sata.h): the same entry points, argument
marshalling only.  Every step of the attention path runs in the library's
CUDA kernels; this module never computes anything itself and has no fallback:
if libsata.so is missing or a call fails, it raises.

torch is used for device memory and streams: tensors are passed by pointer,
and calls are enqueued on torch's current CUDA stream unless one is given.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsata.so")

SATA_OK = 0
SATA_EINVAL = -1
SATA_EUNSUPPORTED = -2
SATA_ECUDA = -3
SATA_ETIMEOUT = -4
SATA_ENOMEM = -5
SATA_ERANGE = -6
SATA_EALIGN = -7

SATA_OPT_PREFILL_PATH = 1
SATA_OPT_WAIT_LIMIT = 2
SATA_OPT_TEST_STALL = 3
SATA_OPT_TIME_KERNELS = 4
SATA_OPT_DETERMINISTIC = 5

EXPORTED = (
    "sata_status_string", "sata_last_cuda_error", "sata_version", "sata_num_features",
    "sata_build_basis", "sata_set_stream", "sata_sync_status", "sata_shutdown",
    "sata_state_bytes", "sata_state_init", "sata_workspace_bytes", "sata_prefill",
    "sata_prefill_ex", "sata_decode_step", "sata_set_option", "sata_get_option",
    "sata_kernel_stats", "sata_reset_kernel_stats", "sata_decode_step_static", "sata_prefill_host",
    "sata_backward_workspace_bytes", "sata_prefill_backward", "sata_state_accumulate", "sata_prefill_f32",
)


class SataError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = _lib.sata_status_string(status).decode() if _lib is not None else str(status)
        if status == SATA_ECUDA and _lib is not None:
            msg += f" (cudaError {_lib.sata_last_cuda_error()})"
        super().__init__(f"{what}: {msg}")


class sata_kernel_stat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 40), ("launches", ctypes.c_int64), ("ms", ctypes.c_double)]


class sata_state(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("d_K", ctypes.c_int32),
        ("d_V", ctypes.c_int32), ("P", ctypes.c_int32), ("F", ctypes.c_int64),
        ("S", ctypes.c_void_p), ("Z", ctypes.c_void_p), ("stream", ctypes.c_void_p),
        ("tokens", ctypes.c_int64),
    ]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libsata.so (raises OSError/ImportError if it is absent: no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libsata.so not built ({path}); run python -m symmetric_taylor_self_b200.build")
    lib = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    P_i64, P_sz = ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_size_t)
    st_p = ctypes.POINTER(sata_state)
    sigs = {
        "sata_status_string": (ctypes.c_char_p, [i32]),
        "sata_last_cuda_error": (i32, []),
        "sata_version": (i32, []),
        "sata_num_features": (i32, [i32, i32, P_i64]),
        "sata_build_basis": (i32, [i32, i32, vp, vp, vp, P_i64]),
        "sata_set_stream": (i32, [vp]),
        "sata_sync_status": (i32, [vp]),
        "sata_shutdown": (None, []),
        "sata_state_bytes": (i32, [i32, i32, i32, i32, i32, P_sz, P_sz]),
        "sata_state_init": (i32, [st_p, i32, i32, i32, i32, i32, vp, vp, vp]),
        "sata_workspace_bytes": (i32, [i32, i32, i64, i32, i32, i32, P_sz]),
        "sata_prefill": (i32, [vp, vp, vp, vp, i32, i32, i64, i32, i32, i32]),
        "sata_prefill_ex": (i32, [vp, vp, vp, vp, i32, i32, i64, i32, i32, i32, st_p, vp, sz, vp]),
        "sata_decode_step": (i32, [st_p, vp, vp, vp, vp]),
        "sata_set_option": (i32, [i32, i64]),
        "sata_get_option": (i32, [i32, P_i64]),
        "sata_kernel_stats": (i32, [ctypes.POINTER(sata_kernel_stat), i32, ctypes.POINTER(ctypes.c_int)]),
        "sata_reset_kernel_stats": (i32, []),
        "sata_decode_step_static": (i32, [st_p, vp, vp, vp, vp]),
        "sata_prefill_host": (i32, [vp, vp, vp, vp, i32, i32, i64, i32, i32, i32, st_p, vp]),
        "sata_prefill_f32": (i32, [vp, vp, vp, vp, i32, i32, i64, i32, i32, i32, st_p, vp]),
        "sata_backward_workspace_bytes": (i32, [i32, i32, i64, i32, i32, i32, P_sz]),
        "sata_state_accumulate": (i32, [st_p, vp, vp, i64]),
        "sata_prefill_backward": (i32, [vp, vp, vp, vp, vp, vp, vp, i32, i32, i64, i32, i32, i32,
                                        vp, sz, vp]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(rc: int, what: str):
    if rc != SATA_OK:
        raise SataError(rc, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _need(t, dtype, shape, name):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: must be a contiguous CUDA tensor")


# ------------------------------------------------------------ host calls ----

def sata_version() -> int:
    return load().sata_version()


def sata_num_features(d_K: int, P: int) -> int:
    F = ctypes.c_int64(0)
    _check(load().sata_num_features(d_K, P, ctypes.byref(F)), "sata_num_features")
    return F.value


def sata_build_basis(d_K: int, P: int):
    """(M [F, max(P-1,1)] uint8 padded with 255, C [F] uint32, offsets [P+1] int64) as torch CPU tensors."""
    F = sata_num_features(d_K, P)
    M = torch.empty((F, max(P - 1, 1)), dtype=torch.uint8)
    C = torch.empty(F, dtype=torch.int32)          # filled as uint32
    off = torch.empty(P + 1, dtype=torch.int64)
    Fo = ctypes.c_int64(0)
    _check(load().sata_build_basis(d_K, P, _ptr(M), _ptr(C), _ptr(off), ctypes.byref(Fo)),
           "sata_build_basis")
    assert Fo.value == F
    return M, C.view(torch.uint32) if hasattr(torch, "uint32") else C, off


def sata_set_stream(stream=None):
    _check(load().sata_set_stream(_stream(stream)), "sata_set_stream")


def sata_sync_status(stream=None) -> int:
    """Synchronise and return the device-side status (0, SATA_ETIMEOUT, SATA_ERANGE)."""
    return load().sata_sync_status(_stream(stream))


def sata_shutdown():
    load().sata_shutdown()


def sata_set_option(key: int, value: int):
    _check(load().sata_set_option(key, value), "sata_set_option")


def sata_get_option(key: int) -> int:
    v = ctypes.c_int64(0)
    _check(load().sata_get_option(key, ctypes.byref(v)), "sata_get_option")
    return v.value


def sata_kernel_stats() -> dict:
    """{kernel name: (launches, device ms)} since the last reset."""
    arr = (sata_kernel_stat * 32)()
    n = ctypes.c_int(0)
    _check(load().sata_kernel_stats(arr, 32, ctypes.byref(n)), "sata_kernel_stats")
    return {arr[i].name.decode(): (arr[i].launches, arr[i].ms) for i in range(n.value)}


def sata_reset_kernel_stats():
    _check(load().sata_reset_kernel_stats(), "sata_reset_kernel_stats")


def sata_state_bytes(B, H, d_K, d_V, P):
    s, z = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(load().sata_state_bytes(B, H, d_K, d_V, P, ctypes.byref(s), ctypes.byref(z)),
           "sata_state_bytes")
    return s.value, z.value


def sata_workspace_bytes(B, H, N, d_K, d_V, P) -> int:
    b = ctypes.c_size_t(0)
    _check(load().sata_workspace_bytes(B, H, N, d_K, d_V, P, ctypes.byref(b)), "sata_workspace_bytes")
    return b.value


def sata_backward_workspace_bytes(B, H, N, d_K, d_V, P) -> int:
    b = ctypes.c_size_t(0)
    _check(load().sata_backward_workspace_bytes(B, H, N, d_K, d_V, P, ctypes.byref(b)),
           "sata_backward_workspace_bytes")
    return b.value


# ---------------------------------------------------------- device calls ----

def sata_prefill(q, k, v, out, B, H, N, d_K, d_V, P):
    """Raw call on the library's stream (set it with sata_set_stream)."""
    _check(load().sata_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d_K, d_V, P),
           "sata_prefill")


def sata_prefill_ex(q, k, v, out, B, H, N, d_K, d_V, P, st=None, workspace=None, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().sata_prefill_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d_K, d_V, P,
                                  None if st is None else ctypes.byref(st), _ptr(workspace),
                                  ws_bytes, _stream(stream)), "sata_prefill_ex")


def sata_prefill_f32(q, k, v, out, B, H, N, d_K, d_V, P, st=None, stream=None):
    _check(load().sata_prefill_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d_K, d_V, P,
                                   None if st is None else ctypes.byref(st), _stream(stream)),
           "sata_prefill_f32")


def sata_prefill_host(q, k, v, out, B, H, N, d_K, d_V, P, st=None, stream=None):
    """q, k, v, out: CPU tensors (pinned for overlap); the library copies them in
    and out segment by segment around the kernels (see include/sata.h)."""
    for t in (q, k, v, out):
        if t.is_cuda:
            raise ValueError("sata_prefill_host takes host tensors")
    _check(load().sata_prefill_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d_K, d_V, P,
                                    None if st is None else ctypes.byref(st), _stream(stream)),
           "sata_prefill_host")


def sata_prefill_backward(q, k, v, dy, dq, dk, dv, B, H, N, d_K, d_V, P, workspace=None, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().sata_prefill_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dy), _ptr(dq), _ptr(dk),
                                        _ptr(dv), B, H, N, d_K, d_V, P, _ptr(workspace), ws_bytes,
                                        _stream(stream)), "sata_prefill_backward")


def sata_state_init(st, B, H, d_K, d_V, P, S, Z, stream=None):
    _check(load().sata_state_init(ctypes.byref(st), B, H, d_K, d_V, P, _ptr(S), _ptr(Z),
                                  _stream(stream)), "sata_state_init")


def sata_state_accumulate(st, S, Z, tokens):
    _check(load().sata_state_accumulate(ctypes.byref(st), _ptr(S), _ptr(Z), tokens), "sata_state_accumulate")


def sata_decode_step(st, q, k, v, out):
    _check(load().sata_decode_step(ctypes.byref(st), _ptr(q), _ptr(k), _ptr(v), _ptr(out)),
           "sata_decode_step")


def sata_decode_step_static(st, q, k, v, out):
    """The decode step that allocates no device memory (see include/sata.h)."""
    _check(load().sata_decode_step_static(ctypes.byref(st), _ptr(q), _ptr(k), _ptr(v), _ptr(out)),
           "sata_decode_step_static")


# ------------------------------------------------- tensor-level wrappers ----

class State:
    """A recurrent state (S, Z) owned by torch, plus the ABI struct pointing at it."""

    def __init__(self, B, H, d_K, d_V, P, device=None, stream=None):
        device = torch.device("cuda") if device is None else torch.device(device)
        F = sata_num_features(d_K, P)
        self.S = torch.empty((B, H, F, d_V), dtype=torch.float32, device=device)
        self.Z = torch.empty((B, H, F), dtype=torch.float32, device=device)
        self.st = sata_state()
        sata_state_init(self.st, B, H, d_K, d_V, P, self.S, self.Z, stream)

    def set_stream(self, stream=None):
        self.st.stream = _stream(stream).value

    @property
    def tokens(self) -> int:
        return self.st.tokens


def prefill(q, k, v, P: int = 4, state: State | None = None, out=None, workspace=None, stream=None):
    """Causal SATA attention over [B, H, N, d] bf16 inputs; returns fp32 [B, H, N, d_V]."""
    B, H, N, d_K = q.shape
    d_V = v.shape[-1]
    _need(q, torch.bfloat16, (B, H, N, d_K), "q")
    _need(k, torch.bfloat16, (B, H, N, d_K), "k")
    _need(v, torch.bfloat16, (B, H, N, d_V), "v")
    if out is None:
        out = torch.empty((B, H, N, d_V), dtype=torch.float32, device=q.device)
    _need(out, torch.float32, (B, H, N, d_V), "out")
    sata_prefill_ex(q, k, v, out, B, H, N, d_K, d_V, P, None if state is None else state.st,
                    workspace, stream)
    return out


def prefill_f32(q, k, v, P: int = 4, state: State | None = None, out=None, stream=None):
    """As prefill, with fp32 [B, H, N, d] inputs used as given (CUDA-core path)."""
    B, H, N, d_K = q.shape
    d_V = v.shape[-1]
    _need(q, torch.float32, (B, H, N, d_K), "q")
    _need(k, torch.float32, (B, H, N, d_K), "k")
    _need(v, torch.float32, (B, H, N, d_V), "v")
    if out is None:
        out = torch.empty((B, H, N, d_V), dtype=torch.float32, device=q.device)
    _need(out, torch.float32, (B, H, N, d_V), "out")
    sata_prefill_f32(q, k, v, out, B, H, N, d_K, d_V, P, None if state is None else state.st, stream)
    return out


def prefill_backward(q, k, v, dy, P: int = 4, workspace=None, stream=None):
    """Gradients (dq, dk, dv), fp32, of sum(dy * y) for y = prefill(q, k, v, P) from a
    fresh state; dy is fp32 [B, H, N, d_V]."""
    B, H, N, d_K = q.shape
    d_V = v.shape[-1]
    _need(q, torch.bfloat16, (B, H, N, d_K), "q")
    _need(k, torch.bfloat16, (B, H, N, d_K), "k")
    _need(v, torch.bfloat16, (B, H, N, d_V), "v")
    _need(dy, torch.float32, (B, H, N, d_V), "dy")
    dq = torch.empty((B, H, N, d_K), dtype=torch.float32, device=q.device)
    dk = torch.empty_like(dq)
    dv = torch.empty((B, H, N, d_V), dtype=torch.float32, device=q.device)
    sata_prefill_backward(q, k, v, dy, dq, dk, dv, B, H, N, d_K, d_V, P, workspace, stream)
    return dq, dk, dv


class _Attention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, P):
        ctx.P = P
        ctx.save_for_backward(q, k, v)
        return prefill(q, k, v, P)

    @staticmethod
    def backward(ctx, dy):
        q, k, v = ctx.saved_tensors
        dq, dk, dv = prefill_backward(q, k, v, dy.float().contiguous(), ctx.P)
        return dq, dk, dv, None


def attention(q, k, v, P: int = 4):
    """prefill() as a differentiable op: y (fp32) = attention(q, k, v, P), and
    y.backward(...) runs sata_prefill_backward (gradients cast to the inputs' bf16)."""
    return _Attention.apply(q, k, v, P)


def decode_step(state: State, q, k, v, out=None):
    """One token per head: [B, H, d] bf16 in, fp32 [B, H, d_V] out, on the state's stream."""
    st = state.st
    _need(q, torch.bfloat16, (st.B, st.H, st.d_K), "q")
    _need(k, torch.bfloat16, (st.B, st.H, st.d_K), "k")
    _need(v, torch.bfloat16, (st.B, st.H, st.d_V), "v")
    if out is None:
        out = torch.empty((st.B, st.H, st.d_V), dtype=torch.float32, device=q.device)
    _need(out, torch.float32, (st.B, st.H, st.d_V), "out")
    sata_decode_step(st, q, k, v, out)
    return out
