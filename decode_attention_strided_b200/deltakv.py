"""Python binding of the C ABI in include/deltakv.h (libdeltakv.so).

Argument marshalling only: every step of compression and decode runs in the
library's CUDA kernels.  Tensors must already live on the CUDA device; the
binding passes their data pointers, element strides and the current torch
stream.  If the shared library is missing or cannot be loaded, every call
raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libdeltakv.so")

BF16, F32, BF16_CODE4 = 0, 1, 2
ACT_GELU_ERF, ACT_GELU_TANH, ACT_NONE = 0, 1, 2

STATUS = {
    0: "OK", 1: "ERR_INVALID_ARG", 2: "ERR_UNSUPPORTED", 3: "ERR_ALIGNMENT",
    4: "ERR_WORKSPACE", 5: "ERR_CUDA", 6: "ERR_DEVICE_TIMEOUT", 7: "ERR_DEVICE_BOUNDS",
}

SYMBOLS = ("deltakv_plan", "deltakv_plan_destroy", "deltakv_get_cache_layout", "deltakv_compress",
           "deltakv_append", "deltakv_decode_attention", "deltakv_decode_attention_sparse",
           "deltakv_decode_attention_noalloc", "deltakv_reconstruct", "deltakv_device_status",
           "deltakv_set_profiling", "deltakv_profile_collect", "deltakv_status_string", "deltakv_version",
           "deltakv_test_activation", "deltakv_page_pool_layout", "deltakv_pages_from_cache",
           "deltakv_decode_attention_paged")

# forms of deltakv_test_activation (include/deltakv_testing.h)
TEST_ACT_GELU_ERFF, TEST_ACT_GELU_FAST, TEST_ACT_GELU_FAST2, TEST_ACT_GELU_TANH, TEST_ACT_GELU_TANHFIT2 = 0, 1, 2, 3, 4


class DeltaKVError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {STATUS.get(code, code)}")
        self.code = code


class _Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("layers", "batch", "kv_heads", "q_heads", "d_h", "max_T", "stride_s", "k", "d_c",
                 "hidden", "dtype", "act")]


class _Layout(ctypes.Structure):
    _fields_ = [("ref_k_offset", ctypes.c_size_t), ("ref_v_offset", ctypes.c_size_t),
                ("code_offset", ctypes.c_size_t), ("idx_offset", ctypes.c_size_t),
                ("total_bytes", ctypes.c_size_t), ("n_ref_cap", ctypes.c_int64),
                ("n_code_cap", ctypes.c_int64), ("code_scale_offset", ctypes.c_size_t)]


class _PageLayout(ctypes.Structure):
    _fields_ = [("refs_per_page", ctypes.c_int32), ("codes_per_page", ctypes.c_int32),
                ("tokens_per_page", ctypes.c_int32), ("n_pages", ctypes.c_int32),
                ("ref_k_offset", ctypes.c_size_t), ("ref_v_offset", ctypes.c_size_t),
                ("code_offset", ctypes.c_size_t), ("idx_offset", ctypes.c_size_t),
                ("code_scale_offset", ctypes.c_size_t), ("pool_bytes", ctypes.c_size_t)]


class _KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int32), ("total_ms", ctypes.c_double)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libdeltakv.so (raises OSError if it is not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise OSError(f"libdeltakv.so not built at {path}; run python -m decode_attention_strided_b200.build")
    lib = ctypes.CDLL(path)
    vp, sz, i32, i64p = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.POINTER(ctypes.c_int64)
    lib.deltakv_plan.argtypes = [ctypes.POINTER(_Config), ctypes.POINTER(vp), ctypes.POINTER(sz), ctypes.POINTER(sz)]
    lib.deltakv_plan.restype = ctypes.c_int
    lib.deltakv_plan_destroy.argtypes = [vp]
    lib.deltakv_plan_destroy.restype = ctypes.c_int
    lib.deltakv_get_cache_layout.argtypes = [vp, ctypes.POINTER(_Layout)]
    lib.deltakv_get_cache_layout.restype = ctypes.c_int
    lib.deltakv_compress.argtypes = [vp, i32, vp, vp, i64p, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.deltakv_compress.restype = ctypes.c_int
    lib.deltakv_append.argtypes = [vp, i32, i32, vp, vp, i64p, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.deltakv_append.restype = ctypes.c_int
    lib.deltakv_decode_attention.argtypes = [vp, i32, vp, i64p, vp, vp, vp, vp, vp, vp, i64p, vp, sz, vp]
    lib.deltakv_decode_attention.restype = ctypes.c_int
    lib.deltakv_decode_attention_sparse.argtypes = [vp, i32, vp, i64p, vp, vp, vp, vp, vp, vp, i32, vp, i64p, vp,
                                                    sz, vp]
    lib.deltakv_decode_attention_sparse.restype = ctypes.c_int
    lib.deltakv_decode_attention_noalloc.argtypes = [vp, i32, vp, i64p, vp, vp, vp, vp, vp, vp, i64p, vp]
    lib.deltakv_decode_attention_noalloc.restype = ctypes.c_int
    lib.deltakv_reconstruct.argtypes = [vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.deltakv_reconstruct.restype = ctypes.c_int
    lib.deltakv_device_status.argtypes = [vp, vp, vp]
    lib.deltakv_device_status.restype = ctypes.c_int
    lib.deltakv_set_profiling.argtypes = [vp, i32]
    lib.deltakv_set_profiling.restype = ctypes.c_int
    lib.deltakv_profile_collect.argtypes = [vp, ctypes.POINTER(_KernelTime), i32, ctypes.POINTER(i32)]
    lib.deltakv_profile_collect.restype = ctypes.c_int
    lib.deltakv_status_string.argtypes = [ctypes.c_int]
    lib.deltakv_status_string.restype = ctypes.c_char_p
    lib.deltakv_version.argtypes = []
    lib.deltakv_version.restype = ctypes.c_int32
    lib.deltakv_test_activation.argtypes = [i32, vp, vp, ctypes.c_int64, vp]
    lib.deltakv_test_activation.restype = ctypes.c_int
    lib.deltakv_page_pool_layout.argtypes = [vp, i32, ctypes.POINTER(_PageLayout)]
    lib.deltakv_page_pool_layout.restype = ctypes.c_int
    lib.deltakv_pages_from_cache.argtypes = [vp, i32, vp, vp, i32, vp, i32, vp, sz, vp]
    lib.deltakv_pages_from_cache.restype = ctypes.c_int
    lib.deltakv_decode_attention_paged.argtypes = [vp, vp, i32, vp, i64p, vp, i32, vp, i32, vp, vp, vp, vp, vp,
                                                   i64p, vp, sz, vp]
    lib.deltakv_decode_attention_paged.restype = ctypes.c_int
    _lib = lib
    return lib


@dataclasses.dataclass
class Config:
    batch: int
    kv_heads: int
    q_heads: int
    d_h: int
    max_T: int
    stride_s: int
    k: int
    d_c: int
    hidden: int
    dtype: int = BF16
    act: int = ACT_GELU_ERF
    layers: int = 1

    def torch_dtype(self):
        return torch.float32 if self.dtype == F32 else torch.bfloat16


def _check(fn, code):
    if code != 0:
        raise DeltaKVError(fn, code)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


class Plan:
    """Host-side plan (deltakv_plan): validated config, cache layout and
    workspace size.  No device work."""

    def __init__(self, cfg: Config):
        lib = load_library()
        self.cfg = cfg
        c = _Config(cfg.layers, cfg.batch, cfg.kv_heads, cfg.q_heads, cfg.d_h, cfg.max_T, cfg.stride_s,
                    cfg.k, cfg.d_c, cfg.hidden, cfg.dtype, cfg.act)
        h = ctypes.c_void_p()
        cb, wb = ctypes.c_size_t(), ctypes.c_size_t()
        _check("deltakv_plan", lib.deltakv_plan(ctypes.byref(c), ctypes.byref(h), ctypes.byref(cb), ctypes.byref(wb)))
        self.handle = h
        self.cache_bytes = cb.value
        self.workspace_bytes = wb.value
        lay = _Layout()
        _check("deltakv_get_cache_layout", lib.deltakv_get_cache_layout(h, ctypes.byref(lay)))
        self.layout = {f: getattr(lay, f) for f, _ in _Layout._fields_}

    def __del__(self):
        try:
            if getattr(self, "handle", None) is not None and _lib is not None:
                _lib.deltakv_plan_destroy(self.handle)
                self.handle = None
        except Exception:
            pass

    # ---- device buffers owned by the caller
    def alloc_cache(self, device="cuda"):
        return torch.empty(self.cache_bytes, dtype=torch.uint8, device=device)

    def alloc_workspace(self, device="cuda"):
        return torch.zeros(self.workspace_bytes, dtype=torch.uint8, device=device)

    def cache_planes(self, cache: torch.Tensor):
        """Views of the planes of a cache buffer: ref_k, ref_v
        [B,H,n_ref_cap,d_h], code [B,H,n_code_cap,d_c] and idx
        [B,H,n_code_cap,k] (int32); with 4-bit codes, code is the packed
        uint8 plane [B,H,n_code_cap,d_c/2] and code_scale [B,H,n_code_cap]
        (bf16) holds the per-row scales."""
        c, L = self.cfg, self.layout
        dt = c.torch_dtype()
        es = 4 if c.dtype == F32 else 2
        B, H = c.batch, c.kv_heads

        def view(off, rows, cols, dtype, esize):
            n = B * H * rows * cols
            return cache[off:off + n * esize].view(dtype).view(B, H, rows, cols)

        planes = {
            "ref_k": view(L["ref_k_offset"], L["n_ref_cap"], c.d_h, dt, es),
            "ref_v": view(L["ref_v_offset"], L["n_ref_cap"], c.d_h, dt, es),
            "idx": view(L["idx_offset"], L["n_code_cap"], c.k, torch.int32, 4),
        }
        if c.dtype == BF16_CODE4:
            planes["code"] = view(L["code_offset"], L["n_code_cap"], c.d_c // 2, torch.uint8, 1)
            planes["code_scale"] = view(L["code_scale_offset"], L["n_code_cap"], 1, torch.bfloat16, 2)[..., 0]
        else:
            planes["code"] = view(L["code_offset"], L["n_code_cap"], c.d_c, dt, es)
        return planes

    def dequantized_codes(self, cache: torch.Tensor):
        """Code rows as float32 [B,H,n_code_cap,d_c]: the stored values, or for
        4-bit codes q * scale unpacked (low nibble first, two's complement)."""
        pl = self.cache_planes(cache)
        if self.cfg.dtype != BF16_CODE4:
            return pl["code"].float()
        b = pl["code"].to(torch.int16)
        lo = ((b & 0xF) ^ 8) - 8
        hi = ((b >> 4) ^ 8) - 8
        q = torch.stack([lo, hi], dim=-1).flatten(-2).float()
        return q * pl["code_scale"].float()[..., None]


def plan(cfg: Config) -> Plan:
    return Plan(cfg)


def compress(p: Plan, T: int, K, V, W1, b1, W2, b2, cache, workspace, stream=None):
    """deltakv_compress: K, V [B, H, T', d_h] (T' >= T, any batch/head/token
    strides, contiguous last dim)."""
    lib = load_library()
    strides = (ctypes.c_int64 * 3)(K.stride(0), K.stride(1), K.stride(2))
    if tuple(V.stride()[:3]) != tuple(K.stride()[:3]):
        raise ValueError("K and V must share strides")
    _check("deltakv_compress", lib.deltakv_compress(
        p.handle, int(T), _ptr(K), _ptr(V), strides, _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2),
        _ptr(cache), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def append(p: Plan, T0: int, T1: int, K, V, W1, b1, W2, b2, cache, workspace, stream=None):
    """deltakv_append: extend a cache holding tokens [0, T0) to [0, T1);
    K, V as for compress (only tokens [T0, T1) are read)."""
    lib = load_library()
    strides = (ctypes.c_int64 * 3)(K.stride(0), K.stride(1), K.stride(2))
    if tuple(V.stride()[:3]) != tuple(K.stride()[:3]):
        raise ValueError("K and V must share strides")
    _check("deltakv_append", lib.deltakv_append(
        p.handle, int(T0), int(T1), _ptr(K), _ptr(V), strides, _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2),
        _ptr(cache), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def decode_attention(p: Plan, T: int, q, cache, W3, b3, W4, b4, out, workspace, stream=None):
    """deltakv_decode_attention: q [B, Hq, d_h] -> out [B, Hq, d_h] float32."""
    lib = load_library()
    qs = (ctypes.c_int64 * 2)(q.stride(0), q.stride(1))
    os_ = (ctypes.c_int64 * 2)(out.stride(0), out.stride(1))
    _check("deltakv_decode_attention", lib.deltakv_decode_attention(
        p.handle, int(T), _ptr(q), qs, _ptr(cache), _ptr(W3), _ptr(b3), _ptr(W4), _ptr(b4), _ptr(out), os_,
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def decode_attention_sparse(p: Plan, T: int, q, cache, W3, b3, W4, b4, tokens, out, workspace, stream=None):
    """deltakv_decode_attention_sparse: attention over the selected tokens
    tokens [B, H, n_sel] (int32, contiguous) -> out [B, Hq, d_h] float32."""
    lib = load_library()
    if tokens.dtype != torch.int32 or not tokens.is_contiguous():
        raise ValueError("tokens must be a contiguous int32 tensor [B, H, n_sel]")
    # the library reads B * H * n_sel indices: a tensor of another shape
    # would be read past its end
    if tokens.dim() != 3 or tuple(tokens.shape[:2]) != (p.cfg.batch, p.cfg.kv_heads) or tokens.shape[2] < 1:
        raise ValueError(f"tokens must have shape [{p.cfg.batch}, {p.cfg.kv_heads}, n_sel >= 1], "
                         f"got {list(tokens.shape)}")
    qs = (ctypes.c_int64 * 2)(q.stride(0), q.stride(1))
    os_ = (ctypes.c_int64 * 2)(out.stride(0), out.stride(1))
    _check("deltakv_decode_attention_sparse", lib.deltakv_decode_attention_sparse(
        p.handle, int(T), _ptr(q), qs, _ptr(cache), _ptr(W3), _ptr(b3), _ptr(W4), _ptr(b4), _ptr(tokens),
        int(tokens.shape[-1]), _ptr(out), os_, _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def decode_attention_noalloc(p: Plan, T: int, q, cache, W3, b3, W4, b4, out, stream=None):
    """deltakv_decode_attention_noalloc: decode attention without a caller
    workspace, for callers that cannot allocate device memory (the library's
    own 16 MiB static scratch is used; larger plans raise ERR_WORKSPACE)."""
    lib = load_library()
    qs = (ctypes.c_int64 * 2)(q.stride(0), q.stride(1))
    os_ = (ctypes.c_int64 * 2)(out.stride(0), out.stride(1))
    _check("deltakv_decode_attention_noalloc", lib.deltakv_decode_attention_noalloc(
        p.handle, int(T), _ptr(q), qs, _ptr(cache), _ptr(W3), _ptr(b3), _ptr(W4), _ptr(b4), _ptr(out), os_,
        _stream(stream)))


def page_pool_layout(p: Plan, n_pages: int) -> dict:
    """deltakv_page_pool_layout: geometry and plane offsets of a pool of
    n_pages pages (128 blocks of s tokens each)."""
    lib = load_library()
    lay = _PageLayout()
    _check("deltakv_page_pool_layout", lib.deltakv_page_pool_layout(p.handle, int(n_pages), ctypes.byref(lay)))
    return {f: getattr(lay, f) for f, _ in _PageLayout._fields_}


def alloc_pool(p: Plan, n_pages: int, device="cuda"):
    """A zeroed page pool of n_pages pages (uint8, pool_bytes)."""
    return torch.zeros(page_pool_layout(p, n_pages)["pool_bytes"], dtype=torch.uint8, device=device)


def _page_table(p: Plan, page_table):
    if page_table.dtype != torch.int32 or not page_table.is_contiguous() or page_table.dim() != 3 or \
            tuple(page_table.shape[:2]) != (p.cfg.batch, p.cfg.kv_heads):
        raise ValueError(f"page_table must be a contiguous int32 tensor [{p.cfg.batch}, {p.cfg.kv_heads}, "
                         f"max_pages], got {page_table.dtype} {list(page_table.shape)}")
    return int(page_table.shape[2])


def pages_from_cache(p: Plan, T: int, cache, page_table, pool, n_pages: int, workspace, stream=None):
    """deltakv_pages_from_cache: copy the contiguous cache (T tokens per
    sequence) into the pool pages page_table [B, H, max_pages] names."""
    lib = load_library()
    max_pages = _page_table(p, page_table)
    _check("deltakv_pages_from_cache", lib.deltakv_pages_from_cache(
        p.handle, int(T), _ptr(cache), _ptr(page_table), max_pages, _ptr(pool), int(n_pages), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def decode_attention_paged(p: Plan, seq_lens, max_len: int, q, pool, n_pages: int, page_table, W3, b3, W4, b4,
                           out, workspace, stream=None):
    """deltakv_decode_attention_paged: decode over a paged cache whose
    sequences hold seq_lens [B] (int32, device) tokens each."""
    lib = load_library()
    if seq_lens.dtype != torch.int32 or not seq_lens.is_contiguous() or seq_lens.numel() != p.cfg.batch:
        raise ValueError(f"seq_lens must be a contiguous int32 tensor of {p.cfg.batch} lengths")
    max_pages = _page_table(p, page_table)
    qs = (ctypes.c_int64 * 2)(q.stride(0), q.stride(1))
    os_ = (ctypes.c_int64 * 2)(out.stride(0), out.stride(1))
    _check("deltakv_decode_attention_paged", lib.deltakv_decode_attention_paged(
        p.handle, _ptr(seq_lens), int(max_len), _ptr(q), qs, _ptr(pool), int(n_pages), _ptr(page_table), max_pages,
        _ptr(W3), _ptr(b3), _ptr(W4), _ptr(b4), _ptr(out), os_, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def reconstruct(p: Plan, T: int, cache, W3, b3, W4, b4, K_out, V_out, workspace, stream=None):
    """deltakv_reconstruct: dense float32 K_out, V_out [B, H, T, d_h]."""
    lib = load_library()
    _check("deltakv_reconstruct", lib.deltakv_reconstruct(
        p.handle, int(T), _ptr(cache), _ptr(W3), _ptr(b3), _ptr(W4), _ptr(b4), _ptr(K_out), _ptr(V_out),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def device_status(p: Plan, workspace, stream=None) -> int:
    """deltakv_device_status: synchronise, read and clear the error word."""
    return int(load_library().deltakv_device_status(p.handle, _ptr(workspace), _stream(stream)))


def set_profiling(p: Plan, enable: bool = True):
    """deltakv_set_profiling: bracket every launch with CUDA events."""
    _check("deltakv_set_profiling", load_library().deltakv_set_profiling(p.handle, 1 if enable else 0))


def profile_collect(p: Plan) -> dict:
    """deltakv_profile_collect: {kernel name: (launches, total ms)}."""
    buf = (_KernelTime * 16)()
    n = ctypes.c_int32()
    _check("deltakv_profile_collect", load_library().deltakv_profile_collect(p.handle, buf, 16, ctypes.byref(n)))
    return {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].total_ms)) for i in range(n.value)}


def test_activation(form: int, x, y, stream=None):
    """deltakv_test_activation: y = form(x) on the device (float32 tensors of
    the same length; test support, include/deltakv_testing.h)."""
    if x.dtype != torch.float32 or y.dtype != torch.float32 or not x.is_contiguous() or not y.is_contiguous():
        raise ValueError("x and y must be contiguous float32 tensors")
    if x.numel() != y.numel():
        raise ValueError("x and y must have the same length")
    _check("deltakv_test_activation", load_library().deltakv_test_activation(
        int(form), _ptr(x), _ptr(y), int(x.numel()), _stream(stream)))


def version() -> int:
    return int(load_library().deltakv_version())
