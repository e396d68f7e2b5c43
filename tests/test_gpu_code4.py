"""4-bit codes (DELTAKV_BF16_CODE4) against the oracle's 4-bit rounding of
the stored codes (round mode ROUND_Q4): compression, reconstruction, dense and
sparse decode, and streaming append.

Both sides quantise the code they compute: the oracle in fp64, the GPU in
fp32 from its tensor-core MLP.  A row's 4-bit code can therefore differ where
its scale bf16(max |c| / 7) or one of its c / scale sits within the GPU's
error in c of a rounding boundary: such a row must still be the exact 4-bit
rounding of a code within that error of the oracle's, and everything else
(slots, reconstruction, attention) is held to the usual tolerances."""
import numpy as np
import pytest
import torch

import oracle
from decode_attention_strided_b200 import deltakv as dkv
from parity_util import (ATTN_MAX_ABS, Case, check_case, make_inputs, non_ref_tokens, q4_code_delta, q4_other_rounding,
                         run_gpu, run_oracle_head)

pytestmark = pytest.mark.gpu

Q4 = dkv.BF16_CODE4


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from decode_attention_strided_b200 import build
    build.build()
    oracle.build()


CASES = [
    ("dc32_k4", Case(B=2, H=2, Hq=8, d_h=128, T=4099, s=16, k=4, d_c=32, hidden=256, dtype=Q4, n_lat=8)),
    ("dc16_k1_s4", Case(B=1, H=2, Hq=4, d_h=64, T=2000, s=4, k=1, d_c=16, hidden=128, dtype=Q4)),
    ("dc64_k8_s8", Case(B=1, H=1, Hq=4, d_h=128, T=3001, s=8, k=8, d_c=64, hidden=256, dtype=Q4, n_lat=8)),
    ("tanh_biases", Case(B=1, H=2, Hq=8, d_h=128, T=2600, s=16, k=3, d_c=32, hidden=128, dtype=Q4,
                         act=dkv.ACT_GELU_TANH, biases=True)),
]


def _bf16(x):
    return torch.tensor(x, dtype=torch.float64).to(torch.bfloat16).double().numpy()


def _code_agreement(c: Case):
    """Compare the GPU's 4-bit code rows with the oracle's, among rows whose
    slots agree.  Returns (fraction of rows equal to the oracle's, rows, rows
    that are not a valid rounding).

    A row counts as a valid rounding when it is exactly what the 4-bit rule
    (scale = bf16(max|c| / 7), q = rne(c / scale) clamped to +-7) makes of
    some code c' within delta (q4_code_delta: the GPU's own error in c) of
    the oracle's unrounded fp64 code c, element by element."""
    inp = make_inputs(c)
    g = run_gpu(c, inp, decode=False)
    tokens = non_ref_tokens(c.T, c.s)
    delta = q4_code_delta(inp.W["W2"].double().numpy())
    same = total = invalid = 0
    for b in range(c.B):
        for h in range(c.H):
            o = run_oracle_head(c, inp, b, h)
            Kc, Vc = inp.K[b, h].double().numpy(), inp.V[b, h].double().numpy()
            W = {n: t.double().numpy() for n, t in inp.W.items()}
            bias = {n: (None if t is None else t.double().numpy()) for n, t in inp.bias.items()}
            _, c_raw, _, _ = oracle.compress(Kc, Vc, W["W1"], bias["b1"], W["W2"], bias["b2"], c.s, c.k, c.act,
                                             oracle.ROUND_NONE)
            ok_idx = np.all(np.sort(g.idx[b, h], axis=1) == np.sort(o.idx[tokens], axis=1), axis=1)
            gq = g.code[b, h][ok_idx]
            oq = o.code[tokens][ok_idx]
            cr = c_raw[tokens][ok_idx]
            same += int(np.sum(np.all(gq == oq, axis=1)))
            total += int(np.sum(ok_idx))
            # validity of every row that differs
            for r in np.nonzero(~np.all(gq == oq, axis=1))[0]:
                amax = np.abs(cr[r]).max()
                s_lo = _bf16(max(amax - delta.max(), 0.0) / 7.0)
                s_hi = _bf16((amax + delta.max()) / 7.0)
                s_g = np.abs(gq[r]).max() / 7.0
                good = s_lo <= s_g <= s_hi
                if good and s_g > 0:
                    q = gq[r] / s_g
                    q_lo = np.clip(np.rint((cr[r] - delta) / s_g), -7, 7)
                    q_hi = np.clip(np.rint((cr[r] + delta) / s_g), -7, 7)
                    good = bool(np.all(q == np.rint(q)) and np.all((q_lo <= q) & (q <= q_hi)))
                invalid += 0 if good else 1
    return same / max(total, 1), total, invalid


@pytest.mark.parametrize("name,case", CASES, ids=[n for n, _ in CASES])
def test_code4_matches_oracle(name, case):
    w = check_case(case)
    assert {"candidates_tc", "encode_tc"} <= w["kernels"], w["kernels"]
    frac, rows, invalid = _code_agreement(case)
    assert invalid == 0, f"{name}: {invalid} of {rows} code rows are no rounding of a code near the oracle's"
    assert frac >= 0.98, f"{name}: only {frac:.4f} of {rows} code rows equal the oracle's"


def test_code4_cache_is_smaller():
    """At s = 16, k = 4, d_c = 32, 8 kv-heads x d_h 128 the 4-bit cache holds
    16 B of codes + 2 B of scale per compressed token instead of 64 B."""
    base = dict(batch=1, kv_heads=8, q_heads=32, d_h=128, max_T=131072, stride_s=16, k=4, d_c=32, hidden=256)
    p16 = dkv.plan(dkv.Config(**base))
    p4 = dkv.plan(dkv.Config(**base, dtype=Q4))
    n_code = p4.layout["n_code_cap"]
    assert p16.cache_bytes - p4.cache_bytes >= 8 * n_code * (64 - 16 - 2) - 4096


def test_code4_sparse_matches_oracle():
    """Sparse decode over 500 selected tokens per (sequence, kv-head).  With so
    few tokens one 4-bit element rounded the other way (within the GPU's error
    in c of a boundary) moves the output visibly, so the tolerance adds the
    oracle's own spread: the change of its attention when every such element
    of the selected rows is rounded the other way."""
    c = Case(B=2, H=2, Hq=8, d_h=128, T=3000, s=16, k=4, d_c=32, hidden=256, dtype=Q4, n_lat=8)
    inp = make_inputs(c)
    cfg = dkv.Config(batch=c.B, kv_heads=c.H, q_heads=c.Hq, d_h=c.d_h, max_T=c.T, stride_s=c.s, k=c.k, d_c=c.d_c,
                     hidden=c.hidden, dtype=c.dtype, act=c.act)
    p = dkv.plan(cfg)
    W = {n: t.cuda().contiguous() for n, t in inp.W.items()}
    cache, ws = p.alloc_cache(), p.alloc_workspace()
    dkv.compress(p, c.T, inp.K.cuda(), inp.V.cuda(), W["W1"], None, W["W2"], None, cache, ws)
    rng = np.random.default_rng(5)
    sel = np.stack([np.stack([rng.choice(c.T, 500, replace=False) for _ in range(c.H)]) for _ in range(c.B)]).astype(
        np.int32)
    out = torch.empty((c.B, c.Hq, c.d_h), dtype=torch.float32, device="cuda")
    dkv.decode_attention_sparse(p, c.T, inp.q.cuda(), cache, W["W3"], None, W["W4"], None,
                                torch.from_numpy(sel).cuda(), out, ws)
    assert dkv.device_status(p, ws) == 0
    got = out.double().cpu().numpy()
    G = c.Hq // c.H
    Wf = {n: t.double().numpy() for n, t in inp.W.items()}
    delta = q4_code_delta(Wf["W2"])
    for b in range(c.B):
        for h in range(c.H):
            o = run_oracle_head(c, inp, b, h)
            Kc, Vc = inp.K[b, h].double().numpy(), inp.V[b, h].double().numpy()
            _, c_raw, _, _ = oracle.compress(Kc, Vc, Wf["W1"], None, Wf["W2"], None, c.s, c.k, c.act,
                                             oracle.ROUND_NONE)
            t = np.sort(sel[b, h])
            qh = inp.q[b, h * G:(h + 1) * G].double().numpy()
            ref = oracle.attention(qh, o.K_hat[t], o.V_hat[t])
            # the selected non-reference tokens, each rounded the other way
            nr = t[t % c.s != 0]
            alt_code, changed = q4_other_rounding(c_raw[nr], delta)
            K_alt, V_alt = o.K_hat[t].copy(), o.V_hat[t].copy()
            if changed.any():
                rows = nr[changed]
                ka, va = oracle.reconstruct_rows(Kc, Vc, rows, o.idx[rows], alt_code[changed], Wf["W3"], None,
                                                 Wf["W4"], None, c.s)
                pos = np.searchsorted(t, rows)
                K_alt[pos], V_alt[pos] = ka, va
            spread = np.max(np.abs(oracle.attention(qh, K_alt, V_alt) - ref))
            err = np.max(np.abs(got[b, h * G:(h + 1) * G] - ref))
            assert err <= ATTN_MAX_ABS + spread, (b, h, err, spread)


def test_code4_append_matches_oracle():
    """Compress [0, 1500), then append to 1900 in uneven steps: the appended
    rows' slots and 4-bit codes are what the oracle computes for them."""
    c = Case(B=1, H=2, Hq=4, d_h=128, T=1900, s=16, k=4, d_c=32, hidden=256, dtype=Q4, n_lat=8)
    inp = make_inputs(c)
    cfg = dkv.Config(batch=c.B, kv_heads=c.H, q_heads=c.Hq, d_h=c.d_h, max_T=c.T, stride_s=c.s, k=c.k, d_c=c.d_c,
                     hidden=c.hidden, dtype=c.dtype, act=c.act)
    p = dkv.plan(cfg)
    K, V = inp.K.cuda(), inp.V.cuda()
    W = {n: t.cuda().contiguous() for n, t in inp.W.items()}
    cache, ws = p.alloc_cache(), p.alloc_workspace()
    dkv.compress(p, 1500, K, V, W["W1"], None, W["W2"], None, cache, ws)
    t = 1500
    for t1 in (1501, 1517, 1700, 1900):
        dkv.append(p, t, t1, K, V, W["W1"], None, W["W2"], None, cache, ws)
        t = t1
    assert dkv.device_status(p, ws) == 0
    code = p.dequantized_codes(cache).cpu().double().numpy()
    idx = p.cache_planes(cache)["idx"].cpu().numpy()
    Wf = {n: x.double().numpy() for n, x in inp.W.items()}
    tokens = np.array([x for x in range(1500, 1900) if x % c.s])
    rows = tokens - tokens // c.s - 1
    agree = total = 0
    for h in range(c.H):
        Kc, Vc = inp.K[0, h].double().numpy(), inp.V[0, h].double().numpy()
        o_idx, o_code, o_dk, o_dk1 = oracle.compress_rows(Kc, Vc, Wf["W1"], None, Wf["W2"], None, c.s, c.k, tokens,
                                                          oracle.ACT_GELU_ERF, oracle.ROUND_Q4)
        same = np.all(np.sort(idx[0, h, rows], axis=1) == np.sort(o_idx, axis=1), axis=1)
        clear = (o_dk1 - o_dk) > 1e-4 * o_dk
        assert np.all(same[clear])
        agree += int(np.sum(np.all(code[0, h, rows] == o_code, axis=1) & same))
        total += int(np.sum(same))
    assert agree >= 0.99 * total, (agree, total)
