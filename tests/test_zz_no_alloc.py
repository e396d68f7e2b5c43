"""The decode entry point that allocates nothing.

Callers that run inside a device-memory budget fixed at start-up, or that are
hosted by an engine owning every allocation, cannot hand decode a workspace
they allocated themselves; deltakv_decode_attention_noalloc serves them from
the library's own fixed 16 MiB scratch array.  This checks, through the C ABI,
that two calls in a row give the same outputs as the workspace-taking entry
point, within the attention tolerance the parity tests use (also for one
128k-token sequence, whose decode part of the workspace fits although the
whole workspace does not), and that plans whose decode part is too large for
the array are refused before anything runs.
"""
import pytest
import torch

from decode_attention_strided_b200 import deltakv as dkv
from decode_attention_strided_b200 import synth

pytestmark = pytest.mark.gpu

ATTN_MAX_ABS = 5e-3


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from decode_attention_strided_b200 import build
    build.build()


def test_noalloc_decode_matches_workspace_decode_twice():
    B, H, Hq, d_h, T, s, k, d_c, hidden = 1, 8, 32, 128, 4099, 16, 4, 32, 256
    p = dkv.plan(dkv.Config(batch=B, kv_heads=H, q_heads=Hq, d_h=d_h, max_T=T, stride_s=s, k=k, d_c=d_c,
                            hidden=hidden))
    assert p.workspace_bytes <= 16 << 20
    K, V = synth.kv(3, 3, B, H, T, d_h, 8, device="cuda")
    W = synth.codec_weights(3, d_h, d_c, hidden, device="cuda")
    q = synth.queries(3, B, Hq, d_h, device="cuda")
    cache, ws = p.alloc_cache(), p.alloc_workspace()
    dkv.compress(p, T, K, V, W["W1"], None, W["W2"], None, cache, ws)
    ref = torch.empty((B, Hq, d_h), dtype=torch.float32, device="cuda")
    dkv.decode_attention(p, T, q, cache, W["W3"], None, W["W4"], None, ref, ws)
    assert dkv.device_status(p, ws) == 0
    outs = []
    for _ in range(2):
        out = torch.full((B, Hq, d_h), float("nan"), dtype=torch.float32, device="cuda")
        dkv.decode_attention_noalloc(p, T, q, cache, W["W3"], None, W["W4"], None, out)
        outs.append(out)
    torch.cuda.synchronize()
    for out in outs:
        assert torch.isfinite(out).all()
        assert float((out - ref).abs().max()) <= ATTN_MAX_ABS


def test_noalloc_decode_one_128k_sequence():
    """One 128k-token sequence with 8 kv-heads: the whole workspace is larger
    than the array (its compress part alone is about 33 MB), but the decode
    uses only its own part (about 3.6 MiB), so the call is served and matches
    the workspace-taking decode, on two calls in a row."""
    B, H, Hq, d_h, T, s, k, d_c, hidden = 1, 8, 32, 128, 131072, 16, 4, 32, 256
    p = dkv.plan(dkv.Config(batch=B, kv_heads=H, q_heads=Hq, d_h=d_h, max_T=T, stride_s=s, k=k, d_c=d_c,
                            hidden=hidden))
    assert p.workspace_bytes > 16 << 20
    K, V = synth.kv(5, 5, B, H, T, d_h, 8, device="cuda")
    W = synth.codec_weights(5, d_h, d_c, hidden, device="cuda")
    q = synth.queries(5, B, Hq, d_h, device="cuda")
    cache, ws = p.alloc_cache(), p.alloc_workspace()
    dkv.compress(p, T, K, V, W["W1"], None, W["W2"], None, cache, ws)
    del K, V
    ref = torch.empty((B, Hq, d_h), dtype=torch.float32, device="cuda")
    dkv.decode_attention(p, T, q, cache, W["W3"], None, W["W4"], None, ref, ws)
    assert dkv.device_status(p, ws) == 0
    for _ in range(2):
        out = torch.full((B, Hq, d_h), float("nan"), dtype=torch.float32, device="cuda")
        dkv.decode_attention_noalloc(p, T, q, cache, W["W3"], None, W["W4"], None, out)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert float((out - ref).abs().max()) <= ATTN_MAX_ABS


def test_noalloc_refuses_plans_larger_than_its_scratch():
    p = dkv.plan(dkv.Config(batch=8, kv_heads=8, q_heads=32, d_h=128, max_T=131072, stride_s=16, k=4, d_c=32,
                            hidden=256))
    assert p.workspace_bytes > 16 << 20
    q = torch.zeros((8, 32, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((8, 32, 128), dtype=torch.float32, device="cuda")
    w = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dkv.DeltaKVError) as ei:
        dkv.decode_attention_noalloc(p, 1000, q, w, w, None, w, None, out)
    assert ei.value.code == 4  # DELTAKV_ERR_WORKSPACE
