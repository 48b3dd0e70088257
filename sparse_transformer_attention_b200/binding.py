"""ctypes binding of the Condensate attention C ABI (include/condensate_attn.h).

Argument marshalling only: torch provides device memory and the current
stream, every step of the computation runs in the library's CUDA kernels.
There is no CPU fallback: if the library or a CUDA device is missing the
calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcondensate_attn.so")
# the CA_DEBUG build (same entry points; kernels that also check the indexes
# the release build keeps in range by construction, raising CA_ERR_BOUNDS)
DEBUG_LIB_PATH = os.path.join(_HERE, "libcondensate_attn_debug.so")
if os.environ.get("CONDENSATE_ATTN_DEBUG") == "1":
    LIB_PATH = DEBUG_LIB_PATH

CA_OK = 0
CA_ERR_INVALID_ARG = 1
CA_ERR_UNSUPPORTED = 2
CA_ERR_ALIGNMENT = 3
CA_ERR_WORKSPACE = 4
CA_ERR_CUDA = 5
CA_ERR_TIMEOUT = 6
CA_ERR_DEVICE_ARG = 7
CA_ERR_INTERNAL = 8
CA_ERR_BOUNDS = 9

CA_F32 = 0
CA_BF16 = 1

class CaExtras(ctypes.Structure):
    """ca_extras of the header: optional per-head windows and Top-k sizes,
    mass and log-sum-exp outputs (device pointers, NULL = unused)."""
    _fields_ = [("W_h", ctypes.c_void_p), ("k_h", ctypes.c_void_p),
                ("mass", ctypes.c_void_p), ("lse", ctypes.c_void_p)]


# (name, restype, argtypes) of every entry point the header declares.
_P = ctypes.c_void_p
_I = ctypes.c_int
_X = ctypes.POINTER(CaExtras)
SIGNATURES = {
    "condensate_attn_workspace_size":
        (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I, _I, _I]),
    "condensate_attn_prefill":
        (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _I, _P, _P,
              _I, _P, ctypes.c_size_t, _P]),
    "condensate_attn_decode":
        (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _I, _P, _P,
              _I, _P, ctypes.c_size_t, _P]),
    "condensate_attn_workspace_size_ex":
        (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I, _I, _I, _I]),
    "condensate_attn_prefill_ex":
        (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P, _X, _P, _I,
              _P, _P, _I, _P, ctypes.c_size_t, _P]),
    "condensate_attn_decode_ex":
        (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _X, _P, _I, _P,
              _P, _I, _P, ctypes.c_size_t, _P]),
    "condensate_attn_decode_chunks": (_I, [_I, _I, _I, _I]),
    "condensate_attn_decode_noalloc":
        (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _I, _P, _P,
              _I, _P]),
    "condensate_attn_decode_noalloc_status": (_I, [_P]),
    "condensate_attn_decode_shard_workspace_size":
        (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I, _I]),
    "condensate_attn_decode_shard_select":
        (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P,
              ctypes.c_size_t, _P]),
    "condensate_attn_decode_shard_attend":
        (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _I,
              _P, _P, _P, _I, _P, ctypes.c_size_t, _P]),
    "condensate_attn_decode_shard_combine":
        (_I, [_P, _I, _I, _I, _I, _P, _I, _P]),
    "condensate_attn_status": (_I, [_P, _P]),
    "condensate_attn_test_stall": (_I, [ctypes.c_ulonglong]),
    "condensate_attn_status_string": (ctypes.c_char_p, [_I]),
    "condensate_attn_version": (_I, []),
    "condensate_attn_build_flags": (_I, []),
    "condensate_attn_profile_start": (_I, [_I]),
    "condensate_attn_profile_stop": (_I, [ctypes.POINTER(ctypes.c_char_p),
                                          ctypes.POINTER(ctypes.c_float), _I]),
}

_lib = None


class CondensateError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})")


def load(path: Optional[str] = None):
    """Load the C-ABI library (built in-tree by sparse_transformer_attention_b200.build)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(
            f"Condensate attention library not found at {p}; build it with "
            "`python -m sparse_transformer_attention_b200.build`")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def use_library(lib=None):
    """Make `lib` (a path, a library load() returned, or None for LIB_PATH)
    the library every call of this module goes through; returns the one
    used before (None if none was loaded yet)."""
    global _lib
    prev = _lib
    if isinstance(lib, ctypes.CDLL):
        _lib = lib
    else:
        _lib = None
        _lib = load(lib)
    return prev


def status_string(code: int) -> str:
    return load().condensate_attn_status_string(int(code)).decode()


def _dt(t: torch.dtype) -> int:
    if t == torch.float32:
        return CA_F32
    if t == torch.bfloat16:
        return CA_BF16
    raise TypeError(f"unsupported dtype {t}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def condensate_attn_workspace_size(is_decode: bool, dtype: torch.dtype, B: int,
                                   n_or_L: int, Hq: int, Hkv: int, d: int,
                                   W_max: int, k: int) -> int:
    return int(load().condensate_attn_workspace_size(
        int(bool(is_decode)), _dt(dtype), B, n_or_L, Hq, Hkv, d, W_max, k))


def _check(code: int, where: str):
    if code != CA_OK:
        raise CondensateError(code, where)


def _require(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def condensate_attn_workspace_size_ex(is_decode: bool, dtype: torch.dtype,
                                      B: int, nq: int, L: int, Hq: int,
                                      Hkv: int, d: int, W_max: int,
                                      k: int) -> int:
    return int(load().condensate_attn_workspace_size_ex(
        int(bool(is_decode)), _dt(dtype), B, nq, L, Hq, Hkv, d, W_max, k))


def _extras(W_h, k_h, mass, lse):
    if W_h is None and k_h is None and mass is None and lse is None:
        return None
    for t, nm in ((W_h, "W_h"), (k_h, "k_h"), (mass, "mass"), (lse, "lse")):
        if t is not None:
            _require(t, nm)
    for t, nm in ((W_h, "W_h"), (k_h, "k_h")):
        if t is not None and t.dtype != torch.int32:
            raise TypeError(f"{nm} must be int32")
    for t, nm in ((mass, "mass"), (lse, "lse")):
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{nm} must be float32")
    x = CaExtras(_ptr(W_h), _ptr(k_h), _ptr(mass), _ptr(lse))
    return ctypes.byref(x), x


def _w_max(W, W_i, W_h):
    m = [int(W)]
    if W_i is not None:
        m = [int(W_i.max().item())]
    elif W_h is not None:
        m = [int(W_h.max().item())]
    return max(1, m[0])


def condensate_attn_prefill(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                            W: int, k: int, W_i: Optional[torch.Tensor] = None,
                            O: Optional[torch.Tensor] = None,
                            o_dtype: torch.dtype = torch.float32,
                            idx: Optional[torch.Tensor] = None,
                            idx_count: Optional[torch.Tensor] = None,
                            C_max: Optional[int] = None,
                            workspace: Optional[torch.Tensor] = None,
                            stream=None, W_h: Optional[torch.Tensor] = None,
                            k_h: Optional[torch.Tensor] = None,
                            mass: Optional[torch.Tensor] = None,
                            lse: Optional[torch.Tensor] = None
                            ) -> Tuple[torch.Tensor, torch.Tensor,
                                       torch.Tensor]:
    """Causal prefill.  Q [B,Hq,nq,d], K/V [B,Hkv,L,d] (fp32 or bf16, CUDA)
    with nq <= L: query row r sits at position L - nq + r (nq = L is a full
    prefill).  W_i [B,nq], W_h [Hq], k_h [Hq] (int32) are optional; mass
    [B,Hq,nq,4] and lse [B,Hq,nq] (float32) are optional outputs.

    Returns (O [B,Hq,nq,d], idx [B,Hq,nq,C_max] int32, idx_count [B,Hq,nq]).
    """
    B, Hq, nq, d = Q.shape
    Hkv, L = K.shape[1], K.shape[2]
    for t, nm in ((Q, "Q"), (K, "K"), (V, "V")):
        _require(t, nm)
    W_max = _w_max(W, W_i, W_h)
    if C_max is None:
        C_max = min(L, 1 + W_max + k)
    dev = Q.device
    if O is None:
        O = torch.empty((B, Hq, nq, d), dtype=o_dtype, device=dev)
    if idx is None:
        idx = torch.empty((B, Hq, nq, C_max), dtype=torch.int32, device=dev)
    if idx_count is None:
        idx_count = torch.empty((B, Hq, nq), dtype=torch.int32, device=dev)
    if workspace is None:
        ws = condensate_attn_workspace_size_ex(False, Q.dtype, B, nq, L, Hq,
                                               Hkv, d, W_max, k)
        workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
    ex = _extras(W_h, k_h, mass, lse)
    code = load().condensate_attn_prefill_ex(
        _ptr(Q), _ptr(K), _ptr(V), _dt(Q.dtype), B, nq, L, Hq, Hkv, d, int(W),
        int(k), _ptr(W_i), ex[0] if ex else None, _ptr(O), _dt(O.dtype),
        _ptr(idx), _ptr(idx_count), int(C_max), _ptr(workspace),
        workspace.numel(), _stream(stream))
    _check(code, "condensate_attn_prefill_ex")
    return O, idx, idx_count


def condensate_attn_decode(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                           W: int, k: int, W_i: Optional[torch.Tensor] = None,
                           O: Optional[torch.Tensor] = None,
                           o_dtype: torch.dtype = torch.float32,
                           idx: Optional[torch.Tensor] = None,
                           idx_count: Optional[torch.Tensor] = None,
                           C_max: Optional[int] = None,
                           workspace: Optional[torch.Tensor] = None,
                           stream=None, W_h: Optional[torch.Tensor] = None,
                           k_h: Optional[torch.Tensor] = None,
                           mass: Optional[torch.Tensor] = None,
                           lse: Optional[torch.Tensor] = None
                           ) -> Tuple[torch.Tensor, torch.Tensor,
                                      torch.Tensor]:
    """Decode at position L-1.  q [B,Hq,d], K/V [B,Hkv,L,d] (CUDA).  W_i [B],
    W_h [Hq], k_h [Hq] (int32) optional; mass [B,Hq,4], lse [B,Hq] optional
    float32 outputs.

    Returns (O [B,Hq,d], idx [B,Hq,C_max] int32, idx_count [B,Hq]).
    """
    B, Hq, d = q.shape
    Hkv, L = K.shape[1], K.shape[2]
    for t, nm in ((q, "q"), (K, "K"), (V, "V")):
        _require(t, nm)
    W_max = _w_max(W, W_i, W_h)
    if C_max is None:
        C_max = min(L, 1 + W_max + k)
    dev = q.device
    if O is None:
        O = torch.empty((B, Hq, d), dtype=o_dtype, device=dev)
    if idx is None:
        idx = torch.empty((B, Hq, C_max), dtype=torch.int32, device=dev)
    if idx_count is None:
        idx_count = torch.empty((B, Hq), dtype=torch.int32, device=dev)
    if workspace is None:
        ws = condensate_attn_workspace_size(True, q.dtype, B, L, Hq, Hkv, d,
                                            W_max, k)
        workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
    ex = _extras(W_h, k_h, mass, lse)
    code = load().condensate_attn_decode_ex(
        _ptr(q), _ptr(K), _ptr(V), _dt(q.dtype), B, L, Hq, Hkv, d, int(W),
        int(k), _ptr(W_i), ex[0] if ex else None, _ptr(O), _dt(O.dtype),
        _ptr(idx), _ptr(idx_count), int(C_max), _ptr(workspace),
        workspace.numel(), _stream(stream))
    _check(code, "condensate_attn_decode_ex")
    return O, idx, idx_count


def condensate_attn_decode_shard_workspace_size(dtype: torch.dtype, B: int,
                                                L_shard: int, Hq: int,
                                                Hkv: int, d: int,
                                                k: int) -> int:
    return int(load().condensate_attn_decode_shard_workspace_size(
        _dt(dtype), B, L_shard, Hq, Hkv, d, k))


def condensate_attn_decode_shard_select(q: torch.Tensor, K: torch.Tensor,
                                        pos0: int, L: int, W: int, k: int,
                                        W_i: Optional[torch.Tensor] = None,
                                        keys_out: Optional[torch.Tensor] = None,
                                        workspace: Optional[torch.Tensor] = None,
                                        stream=None) -> torch.Tensor:
    """Step 1 of the sequence-sharded decode (see the header): this shard's
    best keys, [B, Hq, k] int64 (the 64-bit keys' bits)."""
    B, Hq, d = q.shape
    Hkv, Ls = K.shape[1], K.shape[2]
    for t, nm in ((q, "q"), (K, "K")):
        _require(t, nm)
    if keys_out is None:
        keys_out = torch.empty((B, Hq, k), dtype=torch.int64, device=q.device)
    if workspace is None:
        ws = condensate_attn_decode_shard_workspace_size(q.dtype, B, Ls, Hq,
                                                         Hkv, d, k)
        workspace = torch.empty(ws, dtype=torch.uint8, device=q.device)
    code = load().condensate_attn_decode_shard_select(
        _ptr(q), _ptr(K), _dt(q.dtype), B, Ls, int(pos0), int(L), Hq, Hkv, d,
        int(W), int(k), _ptr(W_i), _ptr(keys_out), _ptr(workspace),
        workspace.numel(), _stream(stream))
    _check(code, "condensate_attn_decode_shard_select")
    return keys_out


def condensate_attn_decode_shard_attend(q: torch.Tensor, K: torch.Tensor,
                                        V: torch.Tensor, pos0: int, L: int,
                                        W: int, k: int,
                                        keys_all: torch.Tensor,
                                        W_i: Optional[torch.Tensor] = None,
                                        partial: Optional[torch.Tensor] = None,
                                        idx: Optional[torch.Tensor] = None,
                                        idx_count: Optional[torch.Tensor] = None,
                                        C_max: Optional[int] = None,
                                        workspace: Optional[torch.Tensor] = None,
                                        stream=None):
    """Step 3: from every shard's keys keys_all [P, B, Hq, k], this shard's
    softmax state partial [B, Hq, d + 2] and the sequence's idx/idx_count."""
    B, Hq, d = q.shape
    Hkv, Ls = K.shape[1], K.shape[2]
    P = keys_all.shape[0]
    for t, nm in ((q, "q"), (K, "K"), (V, "V"), (keys_all, "keys_all")):
        _require(t, nm)
    dev = q.device
    if C_max is None:
        C_max = min(L, 1 + (int(W_i.max()) if W_i is not None else W) + k)
    if partial is None:
        partial = torch.empty((B, Hq, d + 2), dtype=torch.float32, device=dev)
    if idx is None:
        idx = torch.empty((B, Hq, C_max), dtype=torch.int32, device=dev)
    if idx_count is None:
        idx_count = torch.empty((B, Hq), dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = torch.empty(256, dtype=torch.uint8, device=dev)
    code = load().condensate_attn_decode_shard_attend(
        _ptr(q), _ptr(K), _ptr(V), _dt(q.dtype), B, Ls, int(pos0), int(L), Hq,
        Hkv, d, int(W), int(k), _ptr(W_i), _ptr(keys_all), P, _ptr(partial),
        _ptr(idx), _ptr(idx_count), int(C_max), _ptr(workspace),
        workspace.numel(), _stream(stream))
    _check(code, "condensate_attn_decode_shard_attend")
    return partial, idx, idx_count


def condensate_attn_decode_shard_combine(partials: torch.Tensor,
                                         O: Optional[torch.Tensor] = None,
                                         o_dtype: torch.dtype = torch.float32,
                                         stream=None) -> torch.Tensor:
    """Step 5: O [B, Hq, d] from every shard's partials [P, B, Hq, d + 2]."""
    _require(partials, "partials")
    P, B, Hq, d2 = partials.shape
    d = d2 - 2
    if O is None:
        O = torch.empty((B, Hq, d), dtype=o_dtype, device=partials.device)
    code = load().condensate_attn_decode_shard_combine(
        _ptr(partials), P, B, Hq, d, _ptr(O), _dt(O.dtype), _stream(stream))
    _check(code, "condensate_attn_decode_shard_combine")
    return O


def condensate_attn_decode_chunks(B: int, L: int, Hkv: int, k: int) -> int:
    """Key chunks of the decode score pass on the current device."""
    return int(load().condensate_attn_decode_chunks(B, L, Hkv, k))


def condensate_attn_status(workspace: torch.Tensor, stream=None) -> int:
    """Wait for the stream and return (and clear) the device status code."""
    return int(load().condensate_attn_status(_ptr(workspace), _stream(stream)))


def test_stall(limit_ns: int) -> None:
    """Failure-path test hook (see the header): 0 turns it off."""
    _check(load().condensate_attn_test_stall(int(limit_ns)),
           "condensate_attn_test_stall")


def profile_start(capacity: int = 4096) -> None:
    """Start recording per-launch device times (see the header)."""
    _check(load().condensate_attn_profile_start(int(capacity)),
           "condensate_attn_profile_start")


def profile_stop(cap: int = 4096):
    """Stop recording; returns [(kernel name, milliseconds), ...]."""
    names = (ctypes.c_char_p * cap)()
    ms = (ctypes.c_float * cap)()
    n = load().condensate_attn_profile_stop(names, ms, cap)
    return [(names[i].decode(), float(ms[i])) for i in range(n)]
