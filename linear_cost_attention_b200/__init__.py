"""Python binding of libsata.so, the B200 (sm_100a) library for causal SATA attention.

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels.  PyTorch supplies device memory and streams.  The entry points
mirror include/sata.h one to one (``sata_prefill``, ``sata_decode_step``,
``sata_basis_size``, ``sata_index_table``, ``sata_get_error``,
``sata_status_string``, ``sata_release``); ``prefill`` and ``decode_step``
are conveniences that allocate the outputs with torch and call them.

If libsata.so is missing or cannot be loaded, every call raises: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsata.so")

SATA_OK = 0
SATA_ERR_INVALID_ARG = 1
SATA_ERR_UNSUPPORTED = 2
SATA_ERR_CUDA = 3
SATA_ERR_NOMEM = 4
SATA_ERR_TIMEOUT = 5
SATA_F32 = 0
SATA_BF16 = 1

_lib = None


class SataError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {sata_status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """Load libsata.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m linear_cost_attention_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    L.sata_basis_size.argtypes = [i, i]
    L.sata_basis_size.restype = i64
    L.sata_index_table.argtypes = [i, i, ctypes.POINTER(ctypes.c_int32), i64]
    L.sata_index_table.restype = i64
    L.sata_prefill.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
    L.sata_prefill.restype = i
    L.sata_prefill_continue.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
    L.sata_prefill_continue.restype = i
    L.sata_decode_step.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
    L.sata_decode_step.restype = i
    L.sata_get_error.argtypes = [vp]
    L.sata_get_error.restype = i
    L.sata_status_string.argtypes = [i]
    L.sata_status_string.restype = ctypes.c_char_p
    L.sata_release.argtypes = []
    L.sata_release.restype = None
    L.sata_decode_step_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
    L.sata_decode_step_noalloc.restype = i
    L.sata_profile_enable.argtypes = [i]
    L.sata_profile_enable.restype = i
    L.sata_profile_read.argtypes = [ctypes.POINTER(ctypes.c_float), ctypes.POINTER(i), i]
    L.sata_profile_read.restype = i
    L.sata_kernel_name.argtypes = [i]
    L.sata_kernel_name.restype = ctypes.c_char_p
    L.sata_state_fp32_rows.argtypes = [i, i]
    L.sata_state_fp32_rows.restype = i64
    L.sata_state_split.argtypes = [vp, vp, vp, i, i, i, i, i, vp]
    L.sata_state_split.restype = i
    L.sata_state_join.argtypes = [vp, vp, vp, i, i, i, i, i, vp]
    L.sata_state_join.restype = i
    L.sata_decode_step_mixed.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
    L.sata_decode_step_mixed.restype = i
    L.sata_attention_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
    L.sata_attention_backward.restype = i
    L.sata_test_set_wait_limit.argtypes = [ctypes.c_longlong]
    L.sata_test_set_wait_limit.restype = ctypes.c_longlong
    _lib = L
    return L


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(dtype) -> int:
    if isinstance(dtype, int):
        return dtype
    import torch

    if dtype == torch.float32:
        return SATA_F32
    if dtype == torch.bfloat16:
        return SATA_BF16
    raise ValueError(f"unsupported dtype {dtype}")


# ------------------------------------------------------------- raw entry points

def sata_basis_size(dK: int, P: int) -> int:
    return int(lib().sata_basis_size(dK, P))


def sata_index_table(dK: int, p: int) -> np.ndarray:
    """M_p as int32 [C(dK+p-1,p), p] (host only)."""
    rows = sata_basis_size(dK, p + 1) - (sata_basis_size(dK, p) if p > 0 else 0)
    out = np.zeros((max(rows, 1), p), dtype=np.int32)
    n = lib().sata_index_table(dK, p, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                               out.size)
    if n < 0:
        raise SataError(SATA_ERR_INVALID_ARG, "sata_index_table")
    return out[:n]


def sata_prefill(q, k, v, out, state, B, H, N, dK, dV, P, dtype, stream=None) -> None:
    st = lib().sata_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(state), B, H, N, dK,
                            dV, P, _dtype_code(dtype), _stream(stream))
    if st != SATA_OK:
        raise SataError(st, "sata_prefill")


def sata_prefill_continue(q, k, v, out, state, B, H, N, dK, dV, P, dtype, stream=None) -> None:
    st = lib().sata_prefill_continue(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(state), B, H,
                                     N, dK, dV, P, _dtype_code(dtype), _stream(stream))
    if st != SATA_OK:
        raise SataError(st, "sata_prefill_continue")


def sata_decode_step(q, k, v, state, out, B, H, dK, dV, P, dtype, stream=None) -> None:
    st = lib().sata_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(state), _ptr(out), B, H, dK,
                                dV, P, _dtype_code(dtype), _stream(stream))
    if st != SATA_OK:
        raise SataError(st, "sata_decode_step")


def sata_decode_step_noalloc(q, k, v, state, out, B, H, dK, dV, P, dtype, stream=None) -> None:
    """sata_decode_step for callers that cannot allocate device memory: its
    scratch and tables are static device arrays (limit B*H*(dV+1) <= 65536)."""
    st = lib().sata_decode_step_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(state), _ptr(out), B, H,
                                        dK, dV, P, _dtype_code(dtype), _stream(stream))
    if st != SATA_OK:
        raise SataError(st, "sata_decode_step_noalloc")


def sata_state_fp32_rows(dK: int, P: int) -> int:
    return int(lib().sata_state_fp32_rows(dK, P))


def sata_state_split(state, state_lo, state_hi, B, H, dK, dV, P, stream=None) -> None:
    st = lib().sata_state_split(_ptr(state), _ptr(state_lo), _ptr(state_hi), B, H, dK, dV, P,
                                _stream(stream))
    if st != SATA_OK:
        raise SataError(st, "sata_state_split")


def sata_state_join(state_lo, state_hi, state, B, H, dK, dV, P, stream=None) -> None:
    st = lib().sata_state_join(_ptr(state_lo), _ptr(state_hi), _ptr(state), B, H, dK, dV, P,
                               _stream(stream))
    if st != SATA_OK:
        raise SataError(st, "sata_state_join")


def sata_decode_step_mixed(q, k, v, state_lo, state_hi, out, B, H, dK, dV, P, dtype,
                           stream=None) -> None:
    st = lib().sata_decode_step_mixed(_ptr(q), _ptr(k), _ptr(v), _ptr(state_lo), _ptr(state_hi),
                                      _ptr(out), B, H, dK, dV, P, _dtype_code(dtype),
                                      _stream(stream))
    if st != SATA_OK:
        raise SataError(st, "sata_decode_step_mixed")


def sata_attention_backward(q, k, v, dout, dq, dk, dv, B, H, N, dK, dV, P, dtype,
                            stream=None) -> None:
    st = lib().sata_attention_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk),
                                       _ptr(dv), B, H, N, dK, dV, P, _dtype_code(dtype),
                                       _stream(stream))
    if st != SATA_OK:
        raise SataError(st, "sata_attention_backward")


def sata_get_error(stream=None) -> int:
    return int(lib().sata_get_error(_stream(stream)))


def sata_status_string(status: int) -> str:
    return lib().sata_status_string(int(status)).decode()


def sata_release() -> None:
    lib().sata_release()


def sata_profile_enable(on: bool) -> bool:
    return bool(lib().sata_profile_enable(1 if on else 0))


def sata_profile_read(cap: int = 64):
    """[(kernel name, ms)] for the kernels of the most recent profiled call."""
    ms = (ctypes.c_float * cap)()
    ids = (ctypes.c_int * cap)()
    n = lib().sata_profile_read(ms, ids, cap)
    if n < 0:
        raise SataError(SATA_ERR_CUDA, "sata_profile_read")
    return [(sata_kernel_name(ids[j]), float(ms[j])) for j in range(min(n, cap))]


def sata_kernel_name(kid: int) -> str:
    return lib().sata_kernel_name(int(kid)).decode()


def sata_test_set_wait_limit(cycles: int) -> int:
    """Test hook: bound the tensor-core kernels' role waits to ``cycles``
    (<= 0 restores the default).  Returns the previous setting."""
    return int(lib().sata_test_set_wait_limit(int(cycles)))


# ------------------------------------------------------------- conveniences

def _check_qkv(q, k, v):
    import torch

    for t in (q, k, v):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous CUDA tensors")
    if q.dtype != k.dtype or q.dtype != v.dtype or q.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("q, k, v must share dtype float32 or bfloat16")


def prefill(q, k, v, P: int, out=None, state=None, stream=None):
    """Causal prefill from a zero state: q,k [B,H,N,dK], v [B,H,N,dV] ->
    (out [B,H,N,dV] fp32, state [B,H,m,dV+1] fp32)."""
    import torch

    _check_qkv(q, k, v)
    B, H, N, dK = q.shape
    dV = v.shape[-1]
    m = sata_basis_size(dK, P)
    if out is None:
        out = torch.empty(B, H, N, dV, device=q.device, dtype=torch.float32)
    if state is None:
        state = torch.empty(B, H, m, dV + 1, device=q.device, dtype=torch.float32)
    sata_prefill(q, k, v, out, state, B, H, N, dK, dV, P, q.dtype, stream)
    return out, state


def prefill_continue(q, k, v, state, P: int, out=None, stream=None):
    """Causal prefill continuing from ``state`` (the state after earlier
    tokens, [B,H,m,dV+1] fp32, updated in place): q,k [B,H,N,dK], v [B,H,N,dV]
    -> out [B,H,N,dV] fp32."""
    import torch

    _check_qkv(q, k, v)
    B, H, N, dK = q.shape
    dV = v.shape[-1]
    if out is None:
        out = torch.empty(B, H, N, dV, device=q.device, dtype=torch.float32)
    sata_prefill_continue(q, k, v, out, state, B, H, N, dK, dV, P, q.dtype, stream)
    return out


def attention_backward(q, k, v, dout, P: int, stream=None):
    """Gradients (dq, dk, dv), fp32, of sum(dout * out) for out = prefill(q, k, v, P)[0]."""
    import torch

    _check_qkv(q, k, v)
    B, H, N, dK = q.shape
    dV = v.shape[-1]
    dout = dout.contiguous().float()
    dq = torch.empty(B, H, N, dK, device=q.device, dtype=torch.float32)
    dk = torch.empty_like(dq)
    dv = torch.empty(B, H, N, dV, device=q.device, dtype=torch.float32)
    sata_attention_backward(q, k, v, dout, dq, dk, dv, B, H, N, dK, dV, P, q.dtype, stream)
    return dq, dk, dv


def decode_step(q, k, v, state, P: int, out=None, stream=None):
    """One token per head: q,k [B,H,dK] (or [B,H,1,dK]), v [B,H,dV]; state
    [B,H,m,dV+1] updated in place.  Returns out [B,H,dV] fp32."""
    import torch

    _check_qkv(q, k, v)
    B, H = q.shape[:2]
    dK = q.shape[-1]
    dV = v.shape[-1]
    if out is None:
        out = torch.empty(B, H, dV, device=q.device, dtype=torch.float32)
    sata_decode_step(q, k, v, state, out, B, H, dK, dV, P, q.dtype, stream)
    return out


def split_state(state, P: int, stream=None):
    """fp32 state [B,H,m,dV+1] -> (state_lo fp32 [B,H,m_lo,dV+1], state_hi
    fp16 [B,H,m-m_lo,dV+1]), the mixed-precision decode state."""
    import torch

    B, H, m, D1 = state.shape
    dK = _dk_of(m, P)
    m_lo = sata_state_fp32_rows(dK, P)
    lo = torch.empty(B, H, m_lo, D1, device=state.device, dtype=torch.float32)
    hi = torch.empty(B, H, m - m_lo, D1, device=state.device, dtype=torch.float16)
    sata_state_split(state, lo, hi if m > m_lo else None, B, H, dK, D1 - 1, P, stream)
    return lo, hi


def join_state(state_lo, state_hi, P: int, dK: int, stream=None):
    """The mixed-precision state back to one fp32 state [B,H,m,dV+1]."""
    import torch

    B, H, m_lo, D1 = state_lo.shape
    m = sata_basis_size(dK, P)
    state = torch.empty(B, H, m, D1, device=state_lo.device, dtype=torch.float32)
    sata_state_join(state_lo, state_hi if m > m_lo else None, state, B, H, dK, D1 - 1, P, stream)
    return state


def decode_step_mixed(q, k, v, state_lo, state_hi, P: int, out=None, stream=None):
    """One token per head on the mixed-precision state (updated in place)."""
    import torch

    _check_qkv(q, k, v)
    B, H = q.shape[:2]
    dK = q.shape[-1]
    dV = v.shape[-1]
    if out is None:
        out = torch.empty(B, H, dV, device=q.device, dtype=torch.float32)
    m = sata_basis_size(dK, P)
    hi = state_hi if m > state_lo.shape[2] else None
    sata_decode_step_mixed(q, k, v, state_lo, hi, out, B, H, dK, dV, P, q.dtype, stream)
    return out


def _dk_of(m: int, P: int) -> int:
    for dK in (8, 16, 32, 64):
        if sata_basis_size(dK, P) == m:
            return dK
    raise ValueError(f"no supported dK gives {m} basis rows at P={P}")
