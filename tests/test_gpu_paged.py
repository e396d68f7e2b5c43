"""Paged compressed cache: decode over pages of a shared pool, sequences of
different lengths in one batch.

A batch is compressed once at the longest length (the compression is causal:
a token's references are earlier tokens, so every prefix of that cache is the
cache of the shorter sequence), copied into pages in a shuffled order, and
decoded with per-sequence lengths.  Sequence b must match the contiguous
decode of the same cache at T = len[b] (row b of that call), and the oracle's
attention over its own reconstruction of the first len[b] tokens.  The pool
is filled with 0xFF bytes (NaN in bf16) before the copy, so the padding rows
of every partly filled page hold NaN, which the kernels must mask; so is the
workspace before each paged decode (it must write every region it reads).
Most cases have fewer 128-row chunks than the GPU has SMs."""
import math

import numpy as np
import pytest
import torch

import oracle
from decode_attention_strided_b200 import deltakv as dkv
from parity_util import ATTN_MAX_ABS, Case, make_inputs, run_oracle_head

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from decode_attention_strided_b200 import build
    build.build()
    oracle.build()


def _paged_setup(c: Case, lens, seed=0, spare=3):
    inp = make_inputs(c)
    dev = "cuda"
    cfg = dkv.Config(batch=c.B, kv_heads=c.H, q_heads=c.Hq, d_h=c.d_h, max_T=c.T, stride_s=c.s, k=c.k, d_c=c.d_c,
                     hidden=c.hidden, dtype=c.dtype, act=c.act)
    p = dkv.plan(cfg)
    W = {n: t.to(dev).contiguous() for n, t in inp.W.items()}
    cache, ws = p.alloc_cache(), p.alloc_workspace()
    dkv.compress(p, c.T, inp.K.to(dev), inp.V.to(dev), W["W1"], None, W["W2"], None, cache, ws)
    lay = dkv.page_pool_layout(p, 1)
    tpp = lay["tokens_per_page"]
    max_pages = math.ceil(c.T / tpp)
    n_pages = c.B * c.H * max_pages + spare
    rng = np.random.default_rng(seed)
    perm = rng.permutation(n_pages)[:c.B * c.H * max_pages].astype(np.int32)
    ptab = torch.from_numpy(perm.reshape(c.B, c.H, max_pages)).to(dev).contiguous()
    pool = torch.full((dkv.page_pool_layout(p, n_pages)["pool_bytes"],), 0xFF, dtype=torch.uint8, device=dev)
    dkv.pages_from_cache(p, c.T, cache, ptab, pool, n_pages, ws)
    assert dkv.device_status(p, ws) == 0
    return inp, p, W, cache, ws, pool, n_pages, ptab


def _decode_paged(c, inp, p, W, ws, pool, n_pages, ptab, lens):
    # every byte of the workspace after its error word set to 0xFF (NaN as
    # float32): a decode region read before this call wrote it shows up
    ws[256:].fill_(0xFF)
    q = inp.q.to("cuda")
    out = torch.full((c.B, c.Hq, c.d_h), float("nan"), dtype=torch.float32, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    dkv.set_profiling(p, True)
    dkv.decode_attention_paged(p, sl, max(lens), q, pool, n_pages, ptab, W["W3"], None, W["W4"], None, out, ws)
    st = dkv.device_status(p, ws)
    kernels = set(dkv.profile_collect(p))
    dkv.set_profiling(p, False)
    return out, st, kernels


def _contiguous_rows(c, inp, p, W, cache, ws, lens):
    """Row b of the contiguous decode at T = lens[b]."""
    q = inp.q.to("cuda")
    ref = torch.empty((c.B, c.Hq, c.d_h), dtype=torch.float32, device="cuda")
    for b, T in enumerate(lens):
        out = torch.empty_like(ref)
        dkv.decode_attention(p, T, q, cache, W["W3"], None, W["W4"], None, out, ws)
        ref[b] = out[b]
    assert dkv.device_status(p, ws) == 0
    return ref


CASES = [
    ("bf16", Case(B=3, H=2, Hq=8, d_h=128, T=5000, s=16, k=4, d_c=32, hidden=256, dtype=dkv.BF16, n_lat=8),
     [5000, 1200, 3333]),
    ("bf16_s4_short", Case(B=4, H=2, Hq=4, d_h=128, T=3000, s=4, k=2, d_c=16, hidden=128, dtype=dkv.BF16),
     [3000, 17, 600, 513]),
    ("code4", Case(B=2, H=2, Hq=8, d_h=128, T=4500, s=8, k=4, d_c=32, hidden=256, dtype=dkv.BF16_CODE4, n_lat=8),
     [4500, 2049]),
    ("f32_cuda_cores", Case(B=2, H=1, Hq=2, d_h=64, T=2600, s=8, k=2, d_c=16, hidden=128, dtype=dkv.F32),
     [2600, 1025]),
]


@pytest.mark.parametrize("name,case,lens", CASES, ids=[n for n, _, _ in CASES])
def test_paged_decode_matches_contiguous(name, case, lens):
    inp, p, W, cache, ws, pool, n_pages, ptab = _paged_setup(case, lens)
    out, st, kernels = _decode_paged(case, inp, p, W, ws, pool, n_pages, ptab, lens)
    assert st == 0
    assert torch.isfinite(out).all()
    if case.dtype != dkv.F32:
        assert "decode_stream_tc" in kernels, kernels
    ref = _contiguous_rows(case, inp, p, W, cache, ws, lens)
    err = float((out - ref).abs().max())
    assert err <= 2e-4, f"{name}: paged vs contiguous max abs {err}"


def test_paged_decode_against_oracle():
    """Every (sequence, kv-head) of a batch of three lengths against the
    oracle's own compression, reconstruction and fp64 attention."""
    c, lens = CASES[0][1], CASES[0][2]
    inp, p, W, cache, ws, pool, n_pages, ptab = _paged_setup(c, lens, seed=3)
    out, st, _ = _decode_paged(c, inp, p, W, ws, pool, n_pages, ptab, lens)
    assert st == 0
    got = out.double().cpu().numpy()
    G = c.Hq // c.H
    for b, T in enumerate(lens):
        for h in range(c.H):
            o = run_oracle_head(c, inp, b, h)
            qh = inp.q[b, h * G:(h + 1) * G].double().numpy()
            ref = oracle.attention(qh, o.K_hat[:T], o.V_hat[:T])
            err = float(np.max(np.abs(got[b, h * G:(h + 1) * G] - ref)))
            assert err <= ATTN_MAX_ABS, (b, h, T, err)


def test_long_sequence_among_short_ones():
    """One sequence holds nearly all the chunks: its kv-heads' chunks are
    shared out over many CTAs (more partial slots than with even lengths)."""
    c = Case(B=4, H=1, Hq=4, d_h=128, T=40000, s=16, k=4, d_c=32, hidden=256, dtype=dkv.BF16)
    lens = [40000, 300, 2, 4097]
    inp, p, W, cache, ws, pool, n_pages, ptab = _paged_setup(c, lens, seed=5)
    out, st, kernels = _decode_paged(c, inp, p, W, ws, pool, n_pages, ptab, lens)
    assert st == 0
    assert "decode_stream_tc" in kernels, kernels
    ref = _contiguous_rows(c, inp, p, W, cache, ws, lens)
    assert float((out - ref).abs().max()) <= 2e-4


def test_page_index_out_of_range_is_reported():
    """A page-table entry outside [0, n_pages) is read as page 0 (in bounds)
    and reported; so is a sequence length outside [1, max_len]."""
    c, lens = CASES[1][1], CASES[1][2]
    inp, p, W, cache, ws, pool, n_pages, ptab = _paged_setup(c, lens, seed=7)
    bad = ptab.clone()
    bad[1, 0, 0] = n_pages + 5
    out, st, _ = _decode_paged(c, inp, p, W, ws, pool, n_pages, bad, lens)
    assert st == 7  # ERR_DEVICE_BOUNDS
    q = inp.q.to("cuda")
    sl = torch.tensor([lens[0], 0, lens[2], lens[3]], dtype=torch.int32, device="cuda")
    out2 = torch.empty((c.B, c.Hq, c.d_h), dtype=torch.float32, device="cuda")
    dkv.decode_attention_paged(p, sl, max(lens), q, pool, n_pages, ptab, W["W3"], None, W["W4"], None, out2, ws)
    assert dkv.device_status(p, ws) == 7
