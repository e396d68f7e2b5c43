"""Sparse decode attention (deltakv_decode_attention_sparse) against the
oracle: attention over a selection of tokens of the oracle's own full
reconstruction; selecting every token reproduces the dense decode; an
out-of-range token index is reported and skipped."""
import numpy as np
import pytest
import torch

import oracle
from decode_attention_strided_b200 import deltakv as dkv
from parity_util import ATTN_MAX_ABS, Case, make_inputs, run_oracle_head


def _setup(c: Case):
    dev = "cuda"
    inp = make_inputs(c)
    cfg = dkv.Config(batch=c.B, kv_heads=c.H, q_heads=c.Hq, d_h=c.d_h, max_T=c.T, stride_s=c.s, k=c.k, d_c=c.d_c,
                     hidden=c.hidden, dtype=c.dtype, act=c.act)
    p = dkv.plan(cfg)
    W = {n: t.to(dev).contiguous() for n, t in inp.W.items()}
    bias = {n: (None if t is None else t.to(dev)) for n, t in inp.bias.items()}
    cache, ws = p.alloc_cache(), p.alloc_workspace()
    dkv.compress(p, c.T, inp.K.to(dev), inp.V.to(dev), W["W1"], bias["b1"], W["W2"], bias["b2"], cache, ws)
    return inp, p, W, bias, cache, ws


def _selection(c: Case, n_sel: int, seed: int, repeats: bool = False):
    """Unsorted token indices per (sequence, kv-head); with `repeats` the
    same token may appear more than once (it then counts once per
    occurrence, as a gather followed by dense attention would)."""
    rng = np.random.default_rng(seed)
    sel = np.stack([np.stack([rng.choice(c.T, n_sel, replace=repeats) for _ in range(c.H)]) for _ in range(c.B)])
    return sel.astype(np.int32)


def _tc_path(c: Case, n_sel: int) -> bool:
    """The sparse decode runs the tensor-core token loop over the gathered
    rows when the plan has one (bf16 codes, hidden 128 or 256, a nonlinear
    codec) and the selection fits its row list; else the CUDA-core kernels."""
    n_ref_cap = max(128, -(-(-(-c.T // c.s)) // 128) * 128)
    n_code_cap = max(128, -(-(c.T - -(-c.T // c.s)) // 128) * 128)
    return (c.dtype == dkv.BF16 and c.hidden in (128, 256) and c.act != dkv.ACT_NONE
            and n_sel <= n_ref_cap + n_code_cap)


def _sparse(c, inp, p, W, bias, cache, ws, sel):
    out = torch.empty((c.B, c.Hq, c.d_h), dtype=torch.float32, device="cuda")
    dkv.set_profiling(p, True)
    dkv.decode_attention_sparse(p, c.T, inp.q.to("cuda"), cache, W["W3"], bias["b3"], W["W4"], bias["b4"],
                                torch.from_numpy(sel).cuda(), out, ws)
    status = dkv.device_status(p, ws)
    torch.cuda.synchronize()
    kernels = set(dkv.profile_collect(p))
    if _tc_path(c, sel.shape[-1]):
        assert {"sparse_select", "decode_stream_tc", "decode_combine"} <= kernels, kernels
    else:
        assert "sparse_attend" in kernels, kernels
    return out.double().cpu().numpy(), status


@pytest.mark.gpu
@pytest.mark.parametrize("name,case,n_sel,repeats", [
    ("bf16_d128", Case(B=2, H=2, Hq=8, d_h=128, T=3000, s=16, k=4, d_c=32, hidden=256, dtype=dkv.BF16, n_lat=8), 700,
     False),
    ("bf16_d64_tanh_bias", Case(B=1, H=2, Hq=4, d_h=64, T=1500, s=8, k=2, d_c=16, hidden=128, dtype=dkv.BF16,
                                act=dkv.ACT_GELU_TANH, biases=True), 37, False),
    ("f32_G8", Case(B=1, H=1, Hq=8, d_h=64, T=900, s=4, k=3, d_c=32, hidden=64, dtype=dkv.F32, biases=True), 250,
     False),
    ("bf16_G1_repeats", Case(B=2, H=2, Hq=2, d_h=128, T=700, s=16, k=4, d_c=32, hidden=256, dtype=dkv.BF16), 1500,
     True),
    ("bf16_one_token", Case(B=1, H=2, Hq=4, d_h=64, T=300, s=8, k=2, d_c=16, hidden=64, dtype=dkv.BF16), 1, False),
    # tensor-core token loop: one selected token; repeats; several chunks per
    # (sequence, kv-head) with many sequences
    ("tc_one_token", Case(B=1, H=2, Hq=4, d_h=64, T=300, s=8, k=2, d_c=16, hidden=128, dtype=dkv.BF16), 1, False),
    ("tc_repeats", Case(B=2, H=2, Hq=4, d_h=128, T=900, s=8, k=4, d_c=32, hidden=256, dtype=dkv.BF16), 600, True),
    ("tc_multi_chunk", Case(B=4, H=2, Hq=16, d_h=128, T=4000, s=16, k=4, d_c=32, hidden=256, dtype=dkv.BF16,
                            n_lat=8), 1300, False),
])
def test_sparse_matches_oracle(name, case, n_sel, repeats):
    c = case
    inp, p, W, bias, cache, ws = _setup(c)
    sel = _selection(c, n_sel, 7, repeats)
    out, status = _sparse(c, inp, p, W, bias, cache, ws, sel)
    assert status == 0
    G = c.Hq // c.H
    for b in range(c.B):
        for h in range(c.H):
            o = run_oracle_head(c, inp, b, h)
            t = sel[b, h].astype(np.int64)
            q = inp.q[b, h * G:(h + 1) * G].double().numpy()
            want = oracle.attention(q, o.K_hat[t], o.V_hat[t])
            err = float(np.max(np.abs(out[b, h * G:(h + 1) * G] - want)))
            assert err <= ATTN_MAX_ABS, f"{name} (b={b}, h={h}): {err}"


@pytest.mark.gpu
def test_sparse_over_every_token_equals_dense_decode():
    c = Case(B=1, H=2, Hq=8, d_h=128, T=2000, s=16, k=4, d_c=32, hidden=256, dtype=dkv.BF16, n_lat=8)
    inp, p, W, bias, cache, ws = _setup(c)
    sel = np.broadcast_to(np.arange(c.T, dtype=np.int32), (c.B, c.H, c.T)).copy()
    out, status = _sparse(c, inp, p, W, bias, cache, ws, sel)
    assert status == 0
    dense = torch.empty((c.B, c.Hq, c.d_h), dtype=torch.float32, device="cuda")
    dkv.decode_attention(p, c.T, inp.q.cuda(), cache, W["W3"], None, W["W4"], None, dense, ws)
    torch.cuda.synchronize()
    assert float(np.max(np.abs(out - dense.double().cpu().numpy()))) <= ATTN_MAX_ABS


@pytest.mark.gpu
@pytest.mark.parametrize("hidden", [64, 128])  # CUDA-core kernels, tensor-core token loop
def test_sparse_reports_an_out_of_range_token(hidden):
    c = Case(B=1, H=1, Hq=2, d_h=64, T=500, s=8, k=2, d_c=16, hidden=hidden, dtype=dkv.BF16)
    inp, p, W, bias, cache, ws = _setup(c)
    sel = _selection(c, 40, 3)
    sel[0, 0, 5] = c.T + 17
    out, status = _sparse(c, inp, p, W, bias, cache, ws, sel)
    assert status == 7  # DELTAKV_ERR_DEVICE_BOUNDS
    o = run_oracle_head(c, inp, 0, 0)
    t = np.delete(sel[0, 0], 5).astype(np.int64)
    want = oracle.attention(inp.q[0, 0:2].double().numpy(), o.K_hat[t], o.V_hat[t])
    assert float(np.max(np.abs(out[0] - want))) <= ATTN_MAX_ABS
