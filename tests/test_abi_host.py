"""Host-side checks of the C ABI (no GPU): the library loads, exports every
entry point include/deltakv.h declares, validates configurations, reports the
packed-cache layout, and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

from decode_attention_strided_b200 import build as dkv_build
from decode_attention_strided_b200 import deltakv as dkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    dkv_build.build()
    return dkv.load_library()


def _declared_symbols():
    names = set()
    for hdr in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not hdr.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", hdr)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(deltakv_[a-z_]+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    declared = _declared_symbols()
    assert "deltakv_plan" in declared and "deltakv_compress" in declared
    assert "deltakv_decode_attention" in declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(dkv.SYMBOLS)


def test_test_activation_rejects_bad_arguments(lib):
    """The test-support entry point validates before launching: an unknown
    form, a negative length or a NULL pointer are refused; n = 0 is a no-op."""
    assert lib.deltakv_test_activation(9, None, None, 4, None) == 1
    assert lib.deltakv_test_activation(5, None, None, 4, None) == 1
    assert lib.deltakv_test_activation(0, None, None, -1, None) == 1
    assert lib.deltakv_test_activation(0, None, None, 4, None) == 1
    assert lib.deltakv_test_activation(0, None, None, 0, None) == 0


def test_version_and_status_strings(lib):
    assert dkv.version() >= 10000
    for code in range(8):
        assert lib.deltakv_status_string(code)


def _cfg(**kw):
    base = dict(batch=8, kv_heads=8, q_heads=32, d_h=128, max_T=131072, stride_s=16, k=4, d_c=32,
                hidden=256, dtype=dkv.BF16, act=dkv.ACT_GELU_ERF, layers=32)
    base.update(kw)
    return dkv.Config(**base)


def test_layout_of_the_128k_decode_configuration(lib):
    p = dkv.plan(_cfg())
    L = p.layout
    assert L["n_ref_cap"] == 8192 and L["n_code_cap"] == 131072 - 8192
    B, H = 8, 8
    # refs: 2 planes of d_h bf16; codes d_c bf16; idx k int32
    assert L["ref_v_offset"] - L["ref_k_offset"] == B * H * 8192 * 128 * 2
    assert L["idx_offset"] - L["code_offset"] == B * H * (131072 - 8192) * 32 * 2
    assert L["total_bytes"] == p.cache_bytes
    used = B * H * (8192 * 512 + (131072 - 8192) * (64 + 16))
    assert p.cache_bytes >= used and p.cache_bytes < used + 4096
    # 20.9% of a full bf16 cache of the same tokens
    full = B * H * 131072 * 2 * 128 * 2
    assert abs(used / full - 0.2090) < 1e-3
    for off in ("ref_k_offset", "ref_v_offset", "code_offset", "idx_offset"):
        assert L[off] % 256 == 0


@pytest.mark.parametrize("bad,code", [
    (dict(batch=0), 1), (dict(q_heads=12), 1), (dict(stride_s=0), 1), (dict(k=0), 1),
    (dict(d_h=96), 2), (dict(k=9), 2), (dict(d_c=24), 2), (dict(hidden=48), 2),
    (dict(q_heads=8 * 16), 2), (dict(dtype=7), 1), (dict(act=9), 1),
])
def test_plan_rejects(lib, bad, code):
    with pytest.raises(dkv.DeltaKVError) as ei:
        dkv.plan(_cfg(**bad))
    assert ei.value.code == code


def test_identity_codec_shape_is_accepted(lib):
    p = dkv.plan(_cfg(d_h=64, d_c=128, hidden=128, dtype=dkv.F32, act=dkv.ACT_NONE))
    assert p.cache_bytes > 0


def test_calls_reject_bad_arguments_before_any_launch(lib):
    p = dkv.plan(_cfg(batch=1, kv_heads=1, q_heads=4, max_T=1024))
    vp = ctypes.c_void_p
    strides = (ctypes.c_int64 * 3)(1024 * 128, 1024 * 128, 128)
    fake = vp(1 << 20)  # never dereferenced: validation fails first
    ws = p.workspace_bytes
    # T out of range
    assert lib.deltakv_compress(p.handle, 2048, fake, fake, strides, fake, None, fake, None, fake, fake, ws, None) == 1
    # T = 0 is a no-op
    assert lib.deltakv_compress(p.handle, 0, None, None, None, None, None, None, None, None, None, 0, None) == 0
    # workspace too small
    assert lib.deltakv_compress(p.handle, 512, fake, fake, strides, fake, None, fake, None, fake, fake, ws - 1, None) == 4
    # misaligned pointer
    assert lib.deltakv_compress(p.handle, 512, vp((1 << 20) + 2), fake, strides, fake, None, fake, None, fake, fake, ws, None) == 3
    # stride that is not a multiple of 16 bytes
    bad = (ctypes.c_int64 * 3)(1024 * 128, 1024 * 128, 129)
    assert lib.deltakv_compress(p.handle, 512, fake, fake, bad, fake, None, fake, None, fake, fake, ws, None) == 3
    # NULL weights
    assert lib.deltakv_compress(p.handle, 512, fake, fake, strides, None, None, fake, None, fake, fake, ws, None) == 1
    qs = (ctypes.c_int64 * 2)(4 * 128, 128)
    # decode needs T >= 1
    assert lib.deltakv_decode_attention(p.handle, 0, fake, qs, fake, fake, None, fake, None, fake, qs, fake, ws, None) == 1
    assert lib.deltakv_decode_attention(p.handle, 100, fake, qs, fake, fake, None, fake, None, vp((1 << 20) + 4), qs, fake, ws, None) == 3
    assert lib.deltakv_reconstruct(p.handle, -1, fake, fake, None, fake, None, fake, fake, fake, ws, None) == 1
    # append: T0 > T1, T1 beyond max_T, an empty range is a no-op, bad stride
    assert lib.deltakv_append(p.handle, 600, 500, fake, fake, strides, fake, None, fake, None, fake, fake, ws, None) == 1
    assert lib.deltakv_append(p.handle, 500, 2048, fake, fake, strides, fake, None, fake, None, fake, fake, ws, None) == 1
    assert lib.deltakv_append(p.handle, 700, 700, None, None, None, None, None, None, None, None, None, 0, None) == 0
    assert lib.deltakv_append(p.handle, 500, 600, fake, fake, bad, fake, None, fake, None, fake, fake, ws, None) == 3
    # sparse decode: no selection, NULL selection, misaligned selection
    assert lib.deltakv_decode_attention_sparse(p.handle, 100, fake, qs, fake, fake, None, fake, None, fake, 0, fake, qs,
                                               fake, ws, None) == 1
    assert lib.deltakv_decode_attention_sparse(p.handle, 100, fake, qs, fake, fake, None, fake, None, None, 8, fake, qs,
                                               fake, ws, None) == 1
    assert lib.deltakv_decode_attention_sparse(p.handle, 100, fake, qs, fake, fake, None, fake, None,
                                               vp((1 << 20) + 4), 8, fake, qs, fake, ws, None) == 3
    assert lib.deltakv_plan_destroy(None) == 0


def test_sparse_binding_rejects_a_selection_of_the_wrong_shape(lib):
    """The library reads B * H * n_sel indices; the binding refuses any other
    shape before calling it (tensors here are host tensors that are never
    read)."""
    import torch
    cfg = dkv.Config(batch=2, kv_heads=4, q_heads=8, d_h=64, max_T=1000, stride_s=8, k=2, d_c=16, hidden=64)
    p = dkv.plan(cfg)
    x = torch.zeros(16)
    for shape in [(4, 10), (1, 4, 10), (2, 2, 10), (2, 4, 0), (2, 4, 10, 1)]:
        with pytest.raises(ValueError):
            dkv.decode_attention_sparse(p, 100, x, x, x, None, x, None, torch.zeros(shape, dtype=torch.int32), x, x)
    with pytest.raises(ValueError):  # wrong dtype
        dkv.decode_attention_sparse(p, 100, x, x, x, None, x, None, torch.zeros((2, 4, 10), dtype=torch.int64), x, x)


def test_layout_of_4bit_codes(lib):
    """DELTAKV_BF16_CODE4: the code plane holds d_c / 2 bytes a row and a
    bf16 scale plane follows the slot plane; unsupported shapes are refused."""
    p = dkv.plan(_cfg(dtype=dkv.BF16_CODE4))
    L = p.layout
    B, H, n_code = 8, 8, 131072 - 8192
    assert L["idx_offset"] - L["code_offset"] == B * H * n_code * 16
    assert L["code_scale_offset"] >= L["idx_offset"] + B * H * n_code * 4 * 4
    assert L["total_bytes"] >= L["code_scale_offset"] + B * H * n_code * 2
    assert dkv.plan(_cfg()).layout["code_scale_offset"] == 0
    for bad in (dict(act=dkv.ACT_NONE), dict(hidden=64)):
        with pytest.raises(dkv.DeltaKVError) as ei:
            dkv.plan(_cfg(dtype=dkv.BF16_CODE4, **bad))
        assert ei.value.code == 2


def test_page_pool_layout(lib):
    """A page holds 128 blocks of s tokens: 128 reference rows and 128 (s - 1)
    code rows; each plane is an array of n_pages pages, 256-byte aligned."""
    for dtype, code_row in ((dkv.BF16, 64), (dkv.BF16_CODE4, 16)):
        p = dkv.plan(_cfg(dtype=dtype))
        L = dkv.page_pool_layout(p, 10)
        assert (L["refs_per_page"], L["codes_per_page"], L["tokens_per_page"]) == (128, 1920, 2048)
        assert L["ref_v_offset"] - L["ref_k_offset"] == 10 * 128 * 128 * 2
        assert L["code_offset"] - L["ref_v_offset"] == 10 * 128 * 128 * 2
        assert L["idx_offset"] - L["code_offset"] == 10 * 1920 * code_row
        if dtype == dkv.BF16_CODE4:
            assert L["code_scale_offset"] == L["idx_offset"] + 10 * 1920 * 4 * 4
            assert L["pool_bytes"] == L["code_scale_offset"] + 10 * 1920 * 2
        else:
            assert L["code_scale_offset"] == 0 and L["pool_bytes"] == L["idx_offset"] + 10 * 1920 * 4 * 4
        assert all(L[k] % 256 == 0 for k in ("ref_v_offset", "code_offset", "idx_offset", "pool_bytes"))
    p = dkv.plan(_cfg(stride_s=4))
    assert dkv.page_pool_layout(p, 1)["codes_per_page"] == 384
    with pytest.raises(dkv.DeltaKVError):
        dkv.page_pool_layout(p, 0)


def test_paged_calls_reject_bad_arguments_before_any_launch(lib):
    p = dkv.plan(_cfg(batch=2, kv_heads=1, q_heads=4, max_T=5000))
    vp = ctypes.c_void_p
    fake = vp(1 << 20)
    ws = p.workspace_bytes
    qs = (ctypes.c_int64 * 2)(4 * 128, 128)
    dec = lib.deltakv_decode_attention_paged
    # max_len out of range, no pages, too few pages per sequence for max_len (2048 tokens a page)
    assert dec(p.handle, fake, 0, fake, qs, fake, 4, fake, 3, fake, None, fake, None, fake, qs, fake, ws, None) == 1
    assert dec(p.handle, fake, 5001, fake, qs, fake, 4, fake, 3, fake, None, fake, None, fake, qs, fake, ws, None) == 1
    assert dec(p.handle, fake, 5000, fake, qs, fake, 0, fake, 3, fake, None, fake, None, fake, qs, fake, ws, None) == 1
    assert dec(p.handle, fake, 5000, fake, qs, fake, 4, fake, 2, fake, None, fake, None, fake, qs, fake, ws, None) == 1
    # NULL lengths or page table, small workspace, misaligned pool
    assert dec(p.handle, None, 5000, fake, qs, fake, 4, fake, 3, fake, None, fake, None, fake, qs, fake, ws, None) == 1
    assert dec(p.handle, fake, 5000, fake, qs, fake, 4, None, 3, fake, None, fake, None, fake, qs, fake, ws, None) == 1
    assert dec(p.handle, fake, 5000, fake, qs, fake, 4, fake, 3, fake, None, fake, None, fake, qs, fake, ws - 1,
               None) == 4
    assert dec(p.handle, fake, 5000, fake, qs, vp((1 << 20) + 8), 4, fake, 3, fake, None, fake, None, fake, qs, fake,
               ws, None) == 3
    cp = lib.deltakv_pages_from_cache
    assert cp(p.handle, 0, fake, fake, 3, fake, 4, fake, ws, None) == 1
    assert cp(p.handle, 5000, fake, fake, 2, fake, 4, fake, ws, None) == 1
    assert cp(p.handle, 5000, fake, fake, 3, fake, 4, fake, ws - 1, None) == 4
    assert cp(p.handle, 5000, fake, vp((1 << 20) + 2), 3, fake, 4, fake, ws, None) == 3
