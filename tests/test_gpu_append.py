"""Streaming compression (deltakv_append) against the oracle: a cache built by
one compress call up to T0 and extended by appends, one token at a time and
in blocks, must hold for the new tokens what the oracle computes for them,
and decode attention over the extended cache must match the oracle's
attention over its own full reconstruction."""
import numpy as np
import pytest
import torch

import oracle
from decode_attention_strided_b200 import deltakv as dkv
from parity_util import ATTN_MAX_ABS, Case, check_indices, make_inputs, recon_tol, rel_l2, run_oracle_head


def _run(c: Case, T0: int, steps):
    """compress [0, T0) then append the ranges in `steps`; returns the GPU
    slots, reconstruction and decode output over [0, T1)."""
    dev = "cuda"
    inp = make_inputs(c)
    cfg = dkv.Config(batch=c.B, kv_heads=c.H, q_heads=c.Hq, d_h=c.d_h, max_T=c.T, stride_s=c.s, k=c.k, d_c=c.d_c,
                     hidden=c.hidden, dtype=c.dtype, act=c.act)
    p = dkv.plan(cfg)
    K, V = inp.K.to(dev), inp.V.to(dev)
    W = {n: t.to(dev).contiguous() for n, t in inp.W.items()}
    bias = {n: (None if t is None else t.to(dev)) for n, t in inp.bias.items()}
    cache, ws = p.alloc_cache(), p.alloc_workspace()
    dkv.set_profiling(p, True)
    dkv.compress(p, T0, K, V, W["W1"], bias["b1"], W["W2"], bias["b2"], cache, ws)
    t = T0
    for t1 in steps:
        dkv.append(p, t, t1, K, V, W["W1"], bias["b1"], W["W2"], bias["b2"], cache, ws)
        t = t1
    assert t == c.T
    Kh = torch.empty((c.B, c.H, c.T, c.d_h), dtype=torch.float32, device=dev)
    Vh = torch.empty_like(Kh)
    dkv.reconstruct(p, c.T, cache, W["W3"], bias["b3"], W["W4"], bias["b4"], Kh, Vh, ws)
    out = torch.empty((c.B, c.Hq, c.d_h), dtype=torch.float32, device=dev)
    dkv.decode_attention(p, c.T, inp.q.to(dev), cache, W["W3"], bias["b3"], W["W4"], bias["b4"], out, ws)
    assert dkv.device_status(p, ws) == 0
    torch.cuda.synchronize()
    ran = set(dkv.profile_collect(p))
    assert "append_rows" in ran, ran
    planes = p.cache_planes(cache)
    return inp, planes["idx"].cpu().numpy(), Kh.double().cpu().numpy(), Vh.double().cpu().numpy(), \
        out.double().cpu().numpy()


def _check(c: Case, T0: int, steps):
    inp, g_idx, Kh, Vh, out = _run(c, T0, steps)
    G = c.Hq // c.H
    new = np.array([t for t in range(T0, c.T) if t % c.s], dtype=np.int64)
    rows = new - new // c.s - 1
    for b in range(c.B):
        for h in range(c.H):
            o = run_oracle_head(c, inp, b, h)
            K = inp.K[b, h].double().numpy()
            V = inp.V[b, h].double().numpy()
            if len(new):
                check_indices(g_idx[b, h, rows], o.idx[new], o.dk[new], o.dk1[new], K, V, new, c.s)
                e = max(rel_l2(Kh[b, h, new], o.K_hat[new]), rel_l2(Vh[b, h, new], o.V_hat[new]))
                assert e <= recon_tol(c.dtype), f"appended rows (b={b}, h={h}): rel L2 {e}"
            refs = np.arange(0, c.T, c.s)
            assert np.array_equal(Kh[b, h, refs], K[refs]) and np.array_equal(Vh[b, h, refs], V[refs])
            err = float(np.max(np.abs(out[b, h * G:(h + 1) * G] - o.out)))
            assert err <= ATTN_MAX_ABS, f"attention (b={b}, h={h}): {err}"


@pytest.mark.gpu
def test_append_one_token_at_a_time_then_a_block_bf16():
    c = Case(B=2, H=2, Hq=8, d_h=128, T=3000, s=8, k=4, d_c=32, hidden=256, dtype=dkv.BF16, n_lat=8)
    _check(c, 2000, list(range(2001, 2014)) + [3000])


@pytest.mark.gpu
def test_append_from_an_empty_cache_float32():
    c = Case(B=1, H=2, Hq=4, d_h=64, T=500, s=4, k=2, d_c=16, hidden=64, dtype=dkv.F32, biases=True)
    _check(c, 0, [1, 2, 17, 203, 500])


@pytest.mark.gpu
def test_append_k8_tanh():
    c = Case(B=1, H=1, Hq=2, d_h=64, T=1200, s=16, k=8, d_c=16, hidden=128, dtype=dkv.BF16,
             act=dkv.ACT_GELU_TANH, biases=True)
    _check(c, 700, [701, 1200])


@pytest.mark.gpu
def test_append_long_context_several_slices():
    """750 references per token, scanned by 11 CTAs of 69 (one ragged group
    each), for single tokens and a block."""
    c = Case(B=1, H=2, Hq=8, d_h=128, T=12000, s=16, k=4, d_c=32, hidden=256, dtype=dkv.BF16, n_lat=8)
    _check(c, 11990, list(range(11991, 11996)) + [12000])


def _append_setup(c: Case, T0: int, K=None, V=None):
    dev = "cuda"
    inp = make_inputs(c)
    cfg = dkv.Config(batch=c.B, kv_heads=c.H, q_heads=c.Hq, d_h=c.d_h, max_T=c.T, stride_s=c.s, k=c.k, d_c=c.d_c,
                     hidden=c.hidden, dtype=c.dtype, act=c.act)
    p = dkv.plan(cfg)
    K = (inp.K if K is None else K).to(dev)
    V = (inp.V if V is None else V).to(dev)
    W = {n: t.to(dev).contiguous() for n, t in inp.W.items()}
    cache, ws = p.alloc_cache(), p.alloc_workspace()
    dkv.compress(p, T0, K, V, W["W1"], None, W["W2"], None, cache, ws)
    return p, K, V, W, cache, ws


@pytest.mark.gpu
def test_append_equal_distances_keep_the_lowest_slots():
    """Every reference row the same vector: all distances of a new token are
    bit-identical, and the k kept must be slots 0 .. k-1 (ties go to the
    lower slot) although they lie in one warp of one of 11 scan CTAs."""
    c = Case(B=1, H=2, Hq=8, d_h=128, T=12000, s=16, k=4, d_c=32, hidden=256, dtype=dkv.BF16, n_lat=8)
    inp = make_inputs(c)
    K, V = inp.K.clone(), inp.V.clone()
    K[:, :, ::c.s] = K[:, :, 5:6]
    V[:, :, ::c.s] = V[:, :, 5:6]
    T0 = 11900
    p, K, V, W, cache, ws = _append_setup(c, T0, K, V)
    t = T0
    for t1 in (11901, 11902, 11903, 12000):
        dkv.append(p, t, t1, K, V, W["W1"], None, W["W2"], None, cache, ws)
        t = t1
    assert dkv.device_status(p, ws) == 0
    new = np.array([t for t in range(T0, c.T) if t % c.s], dtype=np.int64)
    rows = new - new // c.s - 1
    idx = p.cache_planes(cache)["idx"].cpu().numpy()[:, :, rows]
    assert (idx == np.arange(c.k, dtype=idx.dtype)).all()


@pytest.mark.gpu
def test_append_captured_in_a_cuda_graph_matches_eager():
    """The scan and finish kernels run with programmatic stream
    serialisation; captured in a graph (one token, then a block) they must
    write exactly what the eager calls write."""
    c = Case(B=2, H=2, Hq=8, d_h=128, T=6000, s=8, k=4, d_c=32, hidden=256, dtype=dkv.BF16, n_lat=8)
    T0 = 5000
    p, K, V, W, cache, ws = _append_setup(c, T0)
    start = cache.clone()
    steps = [(T0, T0 + 1), (T0 + 1, T0 + 3), (T0 + 3, c.T)]
    for a, b in steps:
        dkv.append(p, a, b, K, V, W["W1"], None, W["W2"], None, cache, ws)
    torch.cuda.synchronize()
    eager = cache.clone()
    cache.copy_(start)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for a, b in steps:
            dkv.append(p, a, b, K, V, W["W1"], None, W["W2"], None, cache, ws)
    cache.copy_(start)
    g.replay()
    torch.cuda.synchronize()
    assert dkv.device_status(p, ws) == 0
    assert torch.equal(cache, eager)
    del g
