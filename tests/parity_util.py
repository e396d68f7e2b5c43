"""Shared driver for GPU-vs-oracle parity tests.

The same seeded inputs (decode_attention_strided_b200.synth) go through the
CUDA library (via its C ABI binding) and through the fp64 oracle.  Nothing the
CUDA path computes is ever fed to the oracle: both sides compress from the raw
K/V, the oracle reconstructs and attends over its own cache.

Tolerances:
  * reference slots: identical wherever the oracle's gap between its k-th and
    (k+1)-th distance exceeds 1e-4 of the k-th; elsewhere (a near tie) every
    slot the GPU chose must lie within that margin of the oracle's k-th
    distance;
  * reconstructed K/V: relative L2 error per (sequence, kv-head) at most 1e-2
    for bfloat16 caches and 1e-5 for float32 caches;
  * decode attention: max abs error at most 5e-3.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

import oracle
from decode_attention_strided_b200 import deltakv as dkv
from decode_attention_strided_b200 import synth

NEAR_TIE_REL = 1e-4
ATTN_MAX_ABS = 5e-3


def recon_tol(dtype):
    return 1e-5 if dtype == dkv.F32 else 1e-2


def round_mode(dtype):
    """The oracle's rounding of stored codes for a cache element type."""
    return {dkv.F32: oracle.ROUND_F32, dkv.BF16: oracle.ROUND_BF16, dkv.BF16_CODE4: oracle.ROUND_Q4}[dtype]


@dataclasses.dataclass
class Case:
    B: int = 1
    H: int = 1
    Hq: int = 1
    d_h: int = 64
    T: int = 512
    s: int = 8
    k: int = 2
    d_c: int = 16
    hidden: int = 64
    dtype: int = dkv.F32
    act: int = dkv.ACT_GELU_ERF
    n_lat: int = 4
    layer: int = 0
    identity: bool = False
    biases: bool = False
    strided: bool = False
    max_T: int = 0  # 0: T


@dataclasses.dataclass
class Inputs:
    K: torch.Tensor  # [B,H,T,d_h] on CPU, cache dtype
    V: torch.Tensor
    W: dict          # W1..W4 CPU, cache dtype
    bias: dict       # b1..b4 CPU float32 or None
    q: torch.Tensor  # [B,Hq,d_h] CPU, cache dtype


def make_inputs(c: Case) -> Inputs:
    tdt = torch.float32 if c.dtype == dkv.F32 else torch.bfloat16
    K, V = synth.kv(c.layer, c.layer, c.B, c.H, c.T, c.d_h, c.n_lat, dtype=tdt)
    if c.identity:
        W = synth.identity_codec(c.d_h, dtype=tdt)
    else:
        W = synth.codec_weights(c.layer, c.d_h, c.d_c, c.hidden, dtype=tdt)
    bias = {"b1": None, "b2": None, "b3": None, "b4": None}
    if c.biases:
        D = 2 * c.d_h
        for name, n, st in (("b1", c.hidden, 31), ("b2", c.d_c, 32), ("b3", c.hidden, 33), ("b4", D, 34)):
            bias[name] = (0.1 * synth.normal(synth._key(7000 + st, c.layer), (n,), "cpu")).float()
    q = synth.queries(c.layer, c.B, c.Hq, c.d_h, dtype=tdt)
    return Inputs(K, V, W, bias, q)


@dataclasses.dataclass
class GpuResult:
    idx: np.ndarray      # [B,H,n_code,k]
    code: np.ndarray     # [B,H,n_code,d_c] float64
    K_hat: np.ndarray    # [B,H,T,d_h] float64
    V_hat: np.ndarray
    out: np.ndarray      # [B,Hq,d_h] float64
    status: int
    kernels: frozenset   # names of the library kernels that ran


def run_gpu(c: Case, inp: Inputs, decode=True) -> GpuResult:
    dev = "cuda"
    cfg = dkv.Config(batch=c.B, kv_heads=c.H, q_heads=c.Hq, d_h=c.d_h, max_T=c.max_T or c.T,
                     stride_s=c.s, k=c.k, d_c=c.d_c, hidden=c.hidden, dtype=c.dtype, act=c.act)
    p = dkv.plan(cfg)
    dkv.set_profiling(p, True)
    if c.strided:
        # K and V interleaved in one buffer [B, T+3, H, 2, d_h]: non-contiguous
        # batch/head/token strides
        tdt = inp.K.dtype
        buf = torch.zeros((c.B, c.T + 3, c.H, 2, c.d_h), dtype=tdt, device=dev)
        buf[:, :c.T, :, 0, :] = inp.K.permute(0, 2, 1, 3).to(dev)
        buf[:, :c.T, :, 1, :] = inp.V.permute(0, 2, 1, 3).to(dev)
        K = buf[:, :, :, 0, :].permute(0, 2, 1, 3)
        V = buf[:, :, :, 1, :].permute(0, 2, 1, 3)
    else:
        K, V = inp.K.to(dev), inp.V.to(dev)
    W = {n: t.to(dev).contiguous() for n, t in inp.W.items()}
    bias = {n: (None if t is None else t.to(dev)) for n, t in inp.bias.items()}
    cache = p.alloc_cache()
    ws = p.alloc_workspace()
    dkv.compress(p, c.T, K, V, W["W1"], bias["b1"], W["W2"], bias["b2"], cache, ws)
    Kh = torch.empty((c.B, c.H, c.T, c.d_h), dtype=torch.float32, device=dev)
    Vh = torch.empty_like(Kh)
    dkv.reconstruct(p, c.T, cache, W["W3"], bias["b3"], W["W4"], bias["b4"], Kh, Vh, ws)
    out = torch.full((c.B, c.Hq, c.d_h), float("nan"), dtype=torch.float32, device=dev)
    if decode:
        q = inp.q.to(dev)
        dkv.decode_attention(p, c.T, q, cache, W["W3"], bias["b3"], W["W4"], bias["b4"], out, ws)
    status = dkv.device_status(p, ws)
    torch.cuda.synchronize()
    kernels = frozenset(dkv.profile_collect(p))
    planes = p.cache_planes(cache)
    n_code = c.T - math.ceil(c.T / c.s)
    return GpuResult(
        idx=planes["idx"][:, :, :n_code].cpu().numpy(),
        code=p.dequantized_codes(cache)[:, :, :n_code].cpu().double().numpy(),
        K_hat=Kh.cpu().double().numpy(), V_hat=Vh.cpu().double().numpy(),
        out=out.cpu().double().numpy(), status=status, kernels=kernels)


@dataclasses.dataclass
class OracleHead:
    idx: np.ndarray
    code: np.ndarray
    dk: np.ndarray
    dk1: np.ndarray
    K_hat: np.ndarray
    V_hat: np.ndarray
    out: np.ndarray  # [G, d_h]


def run_oracle_head(c: Case, inp: Inputs, b: int, h: int) -> OracleHead:
    K = inp.K[b, h].double().numpy()
    V = inp.V[b, h].double().numpy()
    W = {n: t.double().numpy() for n, t in inp.W.items()}
    bias = {n: (None if t is None else t.double().numpy()) for n, t in inp.bias.items()}
    rmode = round_mode(c.dtype)
    idx, code, dk, dk1 = oracle.compress(K, V, W["W1"], bias["b1"], W["W2"], bias["b2"], c.s, c.k, c.act, rmode)
    Kh, Vh = oracle.reconstruct(K, V, idx, code, W["W3"], bias["b3"], W["W4"], bias["b4"], c.s, c.act)
    G = c.Hq // c.H
    q = inp.q[b, h * G:(h + 1) * G].double().numpy()
    out = oracle.attention(q, Kh, Vh)
    return OracleHead(idx, code, dk, dk1, Kh, Vh, out)


def non_ref_tokens(T, s):
    return np.array([t for t in range(T) if t % s != 0], dtype=np.int64)


def check_indices(gpu_idx, o_idx, o_dk, o_dk1, K, V, tokens, s):
    """Apply the near-tie rule; returns (n_rows, n_flagged).

    The chosen SET must equal the oracle's wherever the oracle's k-th and
    (k+1)-th distances are more than 1e-4 (relative) apart; otherwise every
    chosen slot must lie within that margin of the k-th distance.  The stored
    ORDER is ascending distance, so it is fixed only where neighbouring
    distances in the list are apart by more than the same margin: the GPU's
    list must be ascending in the oracle's distances up to that slack."""
    X = np.concatenate([K, V], axis=1)
    exact = (o_dk1 - o_dk) > NEAR_TIE_REL * o_dk
    mism = np.any(gpu_idx != o_idx, axis=1)
    n_flagged = 0
    for r in np.nonzero(mism)[0]:
        t = tokens[r]
        got = [j for j in gpu_idx[r].tolist() if j >= 0]
        want = [j for j in o_idx[r].tolist() if j >= 0]
        ctx = f"token {t}: gpu {gpu_idx[r].tolist()} oracle {o_idx[r].tolist()} d_k {o_dk[r]} d_k1 {o_dk1[r]}"
        assert len(got) == len(want) and len(set(got)) == len(got), ctx
        assert all(j * s < t for j in got), ctx
        d = [float(np.sum((X[t] - X[j * s]) ** 2)) for j in got]
        if exact[r]:
            assert sorted(got) == sorted(want), "set differs beyond the near-tie margin: " + ctx
        else:
            n_flagged += 1
            assert all(di <= o_dk[r] * (1 + NEAR_TIE_REL) for di in d), ctx
        for a, b in zip(d, d[1:]):
            assert a <= b * (1 + NEAR_TIE_REL), "order not ascending beyond the margin: " + ctx
    return len(tokens), n_flagged


def q4_code_delta(W2):
    """Per code element, a bound on the GPU's own error in the unrounded code
    c: its GELU is within 1.2e-5 of the exact one, which W2 carries into
    element e with gain sum_h |W2[e, h]|; every other step is fp32 or finer."""
    return 1.2e-5 * np.abs(np.asarray(W2, dtype=np.float64)).sum(axis=1) + 1e-6


def q4_other_rounding(c_raw, delta):
    """Another 4-bit code the GPU may legitimately store for each row of
    c_raw (the oracle's unrounded codes): every element whose rounding
    changes within +-delta is pushed across its boundary, the largest
    element too when the scale changes within it, and the pushed row goes
    through the oracle's own quantiser.  Returns (dequantised rows, mask of
    rows that differ from the oracle's code)."""
    c_raw = np.asarray(c_raw, dtype=np.float64)
    alt = np.empty_like(c_raw)
    changed = np.zeros(c_raw.shape[0], dtype=bool)
    for r, c in enumerate(c_raw):
        q, sc = oracle.quantize_row4(c)
        push = np.zeros_like(c)
        if sc > 0:
            lo = np.clip(np.rint((c - delta) / sc), -7, 7)
            hi = np.clip(np.rint((c + delta) / sc), -7, 7)
            push = np.where(lo != q, -delta, np.where(hi != q, delta, 0.0))
        e = int(np.argmax(np.abs(c)))
        amax = abs(c[e])
        if oracle.round_to(oracle.ROUND_BF16, (amax + delta[e]) / 7.0) != sc:
            push[e] = np.sign(c[e]) * delta[e]
        elif oracle.round_to(oracle.ROUND_BF16, max(amax - delta[e], 0.0) / 7.0) != sc:
            push[e] = -np.sign(c[e]) * delta[e]
        q2, sc2 = oracle.quantize_row4(c + push)
        alt[r] = q2.astype(np.float64) * sc2
        changed[r] = not np.array_equal(alt[r], q.astype(np.float64) * sc)
    return alt, changed


def rel_l2(a, b):
    den = float(np.linalg.norm(b))
    return float(np.linalg.norm(a - b)) / (den if den > 0 else 1.0)


def check_case(c: Case, decode=True, heads=None):
    """Full parity of one case; returns a dict of measured errors."""
    inp = make_inputs(c)
    g = run_gpu(c, inp, decode=decode)
    assert g.status == 0, dkv.STATUS.get(g.status, g.status)
    tokens = non_ref_tokens(c.T, c.s)
    G = c.Hq // c.H
    worst = {"recon_rel_l2": 0.0, "attn_max_abs": 0.0, "flagged": 0, "rows": 0, "kernels": g.kernels}
    for b in range(c.B):
        for h in range(c.H):
            if heads is not None and (b, h) not in heads:
                continue
            o = run_oracle_head(c, inp, b, h)
            K = inp.K[b, h].double().numpy()
            V = inp.V[b, h].double().numpy()
            n, f = check_indices(g.idx[b, h], o.idx[tokens], o.dk[tokens], o.dk1[tokens], K, V, tokens, c.s)
            worst["rows"] += n
            worst["flagged"] += f
            # reference rows are stored whole
            refs = np.arange(0, c.T, c.s)
            assert np.array_equal(g.K_hat[b, h][refs], K[refs]) and np.array_equal(g.V_hat[b, h][refs], V[refs])
            e = max(rel_l2(g.K_hat[b, h], o.K_hat), rel_l2(g.V_hat[b, h], o.V_hat))
            worst["recon_rel_l2"] = max(worst["recon_rel_l2"], e)
            assert e <= recon_tol(c.dtype), f"reconstruction rel L2 {e} at (b={b}, h={h})"
            if decode:
                err = float(np.max(np.abs(g.out[b, h * G:(h + 1) * G] - o.out)))
                worst["attn_max_abs"] = max(worst["attn_max_abs"], err)
                assert err <= ATTN_MAX_ABS, f"attention max abs err {err} at (b={b}, h={h})"
    return worst
