"""ctypes binding of the fp64 oracle (``deltakv_oracle.c``).

TEST INFRASTRUCTURE ONLY (see the package docstring).  Every function here
converts its numpy arguments to contiguous float64 / int32 arrays, calls one C
function and returns the result; the method's arithmetic is all in the C file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

ACT_GELU_ERF, ACT_GELU_TANH, ACT_NONE = 0, 1, 2
ROUND_NONE, ROUND_F32, ROUND_BF16, ROUND_Q4 = 0, 1, 2, 3

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "deltakv_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int32)


def lib_path() -> str:
    return _LIB


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP) into oracle/_build/."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.deltakv_oracle_act.restype = ctypes.c_double
            lib.deltakv_oracle_act.argtypes = [ctypes.c_int, ctypes.c_double]
            lib.deltakv_oracle_round.restype = ctypes.c_double
            lib.deltakv_oracle_round.argtypes = [ctypes.c_int, ctypes.c_double]
            lib.deltakv_oracle_select.restype = ctypes.c_int
            lib.deltakv_oracle_select.argtypes = [
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp, _ip, _dp, _dp]
            lib.deltakv_oracle_quantize_row4.restype = ctypes.c_double
            lib.deltakv_oracle_quantize_row4.argtypes = [ctypes.c_int, _dp, ctypes.POINTER(ctypes.c_int8)]
            lib.deltakv_oracle_mlp.restype = None
            lib.deltakv_oracle_mlp.argtypes = [
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp, _dp, _dp, _dp, _dp]
            lib.deltakv_oracle_compress_rows.restype = ctypes.c_int
            lib.deltakv_oracle_compress_rows.argtypes = [ctypes.c_int] * 8 + [_dp] * 6 + [ctypes.c_int, _ip, _ip, _dp, _dp, _dp, ctypes.c_int]
            lib.deltakv_oracle_compress.restype = ctypes.c_int
            lib.deltakv_oracle_compress.argtypes = [ctypes.c_int] * 8 + [_dp] * 6 + [_ip, _dp, _dp, _dp, ctypes.c_int]
            lib.deltakv_oracle_reconstruct.restype = ctypes.c_int
            lib.deltakv_oracle_reconstruct.argtypes = [ctypes.c_int] * 7 + [_dp, _dp, _ip, _dp] + [_dp] * 4 + [_dp, _dp, ctypes.c_int]
            lib.deltakv_oracle_reconstruct_rows.restype = ctypes.c_int
            lib.deltakv_oracle_reconstruct_rows.argtypes = ([ctypes.c_int] * 7 + [_dp, _dp, ctypes.c_int, _ip, _ip, _dp]
                                                            + [_dp] * 4 + [_dp, _dp, ctypes.c_int])
            lib.deltakv_oracle_attention.restype = ctypes.c_int
            lib.deltakv_oracle_attention.argtypes = [ctypes.c_int] * 3 + [_dp] * 4
            _lib = lib
    return _lib


def _f64(a):
    return None if a is None else np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a, kind=_dp):
    return None if a is None else a.ctypes.data_as(kind)


def act(kind: int, z: float) -> float:
    """The nonlinearity of the codec MLPs (exact GELU, tanh GELU or none)."""
    return _load().deltakv_oracle_act(int(kind), float(z))


def round_to(mode: int, v: float) -> float:
    """Round a double to float (ROUND_F32) or bfloat16 (ROUND_BF16), ties to even."""
    return _load().deltakv_oracle_round(int(mode), float(v))


def quantize_row4(c):
    """4-bit code of one row: returns (q int8 [d_c] in [-7, 7], scale) with
    scale = bf16(max |c| / 7) and q = clamp(rne(c / scale), -7, 7)."""
    c = _f64(c)
    q = np.empty(c.shape[0], dtype=np.int8)
    scale = _load().deltakv_oracle_quantize_row4(c.shape[0], _ptr(c), q.ctypes.data_as(ctypes.POINTER(ctypes.c_int8)))
    return q, scale


def select(t: int, K, V, s: int, k: int):
    """Nearest-reference selection for one non-reference token t.

    Returns (idx[k] int32, d_k, d_k1, k_eff)."""
    K, V = _f64(K), _f64(V)
    idx = np.empty(k, dtype=np.int32)
    dk, dk1 = ctypes.c_double(), ctypes.c_double()
    k_eff = _load().deltakv_oracle_select(int(t), K.shape[1], int(s), int(k), _ptr(K), _ptr(V),
                                          _ptr(idx, _ip), ctypes.byref(dk), ctypes.byref(dk1))
    return idx, dk.value, dk1.value, k_eff


def mlp(x, W1, b1, W2, b2, act_kind: int = ACT_GELU_ERF):
    """y = W2 act(W1 x + b1) + b2 for one vector x."""
    x, W1, b1, W2, b2 = _f64(x), _f64(W1), _f64(b1), _f64(W2), _f64(b2)
    hid, n_in = W1.shape
    n_out = W2.shape[0]
    y = np.empty(n_out, dtype=np.float64)
    _load().deltakv_oracle_mlp(n_in, hid, n_out, int(act_kind), _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2),
                               _ptr(x), _ptr(y))
    return y


def compress(K, V, W1, b1, W2, b2, s: int, k: int, act_kind: int = ACT_GELU_ERF,
             round_mode: int = ROUND_BF16, n_threads: int = 0):
    """Compress one (sequence, kv-head) with K, V of shape [T, d_h].

    Returns (idx [T,k] int32, code [T,d_c] float64, d_k [T], d_k1 [T])."""
    K, V, W1, b1, W2, b2 = _f64(K), _f64(V), _f64(W1), _f64(b1), _f64(W2), _f64(b2)
    T, d_h = K.shape
    hidden = W1.shape[0]
    d_c = W2.shape[0]
    idx = np.empty((T, k), dtype=np.int32)
    code = np.empty((T, d_c), dtype=np.float64)
    dk = np.empty(T, dtype=np.float64)
    dk1 = np.empty(T, dtype=np.float64)
    rc = _load().deltakv_oracle_compress(T, d_h, int(s), int(k), d_c, hidden, int(act_kind), int(round_mode),
                                         _ptr(K), _ptr(V), _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2),
                                         _ptr(idx, _ip), _ptr(code), _ptr(dk), _ptr(dk1), int(n_threads))
    if rc != 0:
        raise ValueError("oracle compress: invalid arguments")
    return idx, code, dk, dk1


def compress_rows(K, V, W1, b1, W2, b2, s: int, k: int, rows, act_kind: int = ACT_GELU_ERF,
                  round_mode: int = ROUND_BF16, n_threads: int = 0):
    """Compress only the tokens in `rows` of one (sequence, kv-head).

    Returns (idx [n,k] int32, code [n,d_c], d_k [n], d_k1 [n]) for those rows."""
    K, V, W1, b1, W2, b2 = _f64(K), _f64(V), _f64(W1), _f64(b1), _f64(W2), _f64(b2)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    T, d_h = K.shape
    hidden = W1.shape[0]
    d_c = W2.shape[0]
    n = rows.shape[0]
    idx = np.empty((n, k), dtype=np.int32)
    code = np.empty((n, d_c), dtype=np.float64)
    dk = np.empty(n, dtype=np.float64)
    dk1 = np.empty(n, dtype=np.float64)
    rc = _load().deltakv_oracle_compress_rows(T, d_h, int(s), int(k), d_c, hidden, int(act_kind), int(round_mode),
                                              _ptr(K), _ptr(V), _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2),
                                              n, _ptr(rows, _ip), _ptr(idx, _ip), _ptr(code), _ptr(dk), _ptr(dk1),
                                              int(n_threads))
    if rc != 0:
        raise ValueError("oracle compress_rows: invalid arguments")
    return idx, code, dk, dk1


def reconstruct(K, V, idx, code, W3, b3, W4, b4, s: int, act_kind: int = ACT_GELU_ERF,
                n_threads: int = 0):
    """Rebuild (K_hat, V_hat) [T, d_h] from reference rows, slots and codes."""
    K, V, code, W3, b3, W4, b4 = _f64(K), _f64(V), _f64(code), _f64(W3), _f64(b3), _f64(W4), _f64(b4)
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    T, d_h = K.shape
    k = idx.shape[1]
    d_c = code.shape[1]
    hidden = W3.shape[0]
    Kh = np.empty((T, d_h), dtype=np.float64)
    Vh = np.empty((T, d_h), dtype=np.float64)
    rc = _load().deltakv_oracle_reconstruct(T, d_h, int(s), k, d_c, hidden, int(act_kind), _ptr(K), _ptr(V),
                                            _ptr(idx, _ip), _ptr(code), _ptr(W3), _ptr(b3), _ptr(W4), _ptr(b4),
                                            _ptr(Kh), _ptr(Vh), int(n_threads))
    if rc != 0:
        raise ValueError("oracle reconstruct: invalid arguments")
    return Kh, Vh


def reconstruct_rows(K, V, rows, idx_rows, code_rows, W3, b3, W4, b4, s: int, act_kind: int = ACT_GELU_ERF,
                     n_threads: int = 0):
    """Rebuild only the tokens `rows` of one (sequence, kv-head): idx_rows
    [n, k] and code_rows [n, d_c] are what the cache holds for them.  Returns
    (K_hat, V_hat) [n, d_h]."""
    K, V, code_rows, W3, b3, W4, b4 = _f64(K), _f64(V), _f64(code_rows), _f64(W3), _f64(b3), _f64(W4), _f64(b4)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    idx_rows = np.ascontiguousarray(np.asarray(idx_rows, dtype=np.int32))
    T, d_h = K.shape
    n, k = idx_rows.shape
    d_c = code_rows.shape[1]
    hidden = W3.shape[0]
    Kh = np.empty((n, d_h), dtype=np.float64)
    Vh = np.empty((n, d_h), dtype=np.float64)
    rc = _load().deltakv_oracle_reconstruct_rows(T, d_h, int(s), k, d_c, hidden, int(act_kind), _ptr(K), _ptr(V),
                                                 n, _ptr(rows, _ip), _ptr(idx_rows, _ip), _ptr(code_rows), _ptr(W3),
                                                 _ptr(b3), _ptr(W4), _ptr(b4), _ptr(Kh), _ptr(Vh), int(n_threads))
    if rc != 0:
        raise ValueError("oracle reconstruct_rows: invalid arguments")
    return Kh, Vh


def attention(q, K, V):
    """softmax(q K^T / sqrt(d_h)) V for G query heads q [G, d_h] over K, V [T, d_h]."""
    q, K, V = _f64(q), _f64(K), _f64(V)
    if q.ndim == 1:
        q = q[None, :]
    G, d_h = q.shape
    T = K.shape[0]
    out = np.empty((G, d_h), dtype=np.float64)
    rc = _load().deltakv_oracle_attention(T, d_h, G, _ptr(q), _ptr(K), _ptr(V), _ptr(out))
    if rc != 0:
        raise ValueError("oracle attention: T must be >= 1")
    return out
