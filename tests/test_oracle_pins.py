"""Pins of the fp64 oracle against things other than itself.

Each test checks the oracle against what the DeltaKV summary (gist.science,
section 3 "Metodologia") and plain mathematics fix: brute force on tiny
inputs, exact invariants, special cases that reduce to textbook routines,
printed normal-CDF values and a worked example computed by hand
(tests/golden/hand_example.json).  No GPU is used.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


# --------------------------------------------------------------- selection

@pytest.mark.parametrize("T,s,k", [(17, 1, 1), (23, 2, 3), (31, 3, 2), (64, 8, 5), (40, 5, 8)])
def test_select_matches_brute_force_sort(oracle_mod, T, s, k):
    """Step 1 ("Processo di Compressione"): the k nearest earlier strided
    references by L2 over K||V.  Brute force: list every slot j with j*s < t by
    the definition, sort all (distance, slot) pairs, take the first k."""
    rng = _rng(T * 100 + s * 10 + k)
    d_h = 3
    K = rng.integers(-3, 4, size=(T, d_h)).astype(np.float64)  # many exact ties
    V = rng.integers(-3, 4, size=(T, d_h)).astype(np.float64)
    for t in range(1, T):
        if t % s == 0:
            continue
        cands = [j for j in range(T) if j * s < t]
        assert len(cands) == math.ceil(t / s)
        pairs = sorted((sum((K[t] - K[j * s]) ** 2) + sum((V[t] - V[j * s]) ** 2), j) for j in cands)
        idx, dk, dk1, k_eff = oracle_mod.select(t, K, V, s, k)
        want = [j for _, j in pairs[:k]] + [-1] * max(0, k - len(pairs))
        assert list(idx) == want, (t, list(idx), want)
        assert k_eff == min(k, len(pairs))
        assert dk == pairs[min(k, len(pairs)) - 1][0]
        assert dk1 == (pairs[k][0] if len(pairs) > k else math.inf)


def test_select_exact_ties_take_lower_slot(oracle_mod):
    """Duplicated reference rows give exactly equal distances; the lower slot
    must come first (the tie rule of the selection)."""
    T, s, d_h = 40, 4, 2
    K = np.zeros((T, d_h))
    V = np.zeros((T, d_h))
    for j in range(T // s):
        K[j * s] = [5.0 + j, 1.0]
    for j in (2, 5, 7):                     # three identical references
        K[j * s] = [1.0, 1.0]
    K[37] = [1.0, 1.0]                      # token equal to all three
    idx, dk, dk1, _ = oracle_mod.select(37, K, V, s, 2)
    assert list(idx) == [2, 5]
    assert dk == 0.0 and dk1 == 0.0


def test_select_token_before_second_reference(oracle_mod):
    """Tokens 1..s-1 have only slot 0 (token 0) as candidate."""
    T, s = 10, 8
    K = _rng(1).normal(size=(T, 4))
    V = _rng(2).normal(size=(T, 4))
    for t in range(1, 8):
        idx, dk, dk1, k_eff = oracle_mod.select(t, K, V, s, 3)
        assert list(idx) == [0, -1, -1] and k_eff == 1 and dk1 == math.inf


# -------------------------------------------------------------- rounding

def test_round_bf16_ties_to_even(oracle_mod):
    r = lambda v: oracle_mod.round_to(oracle_mod.ROUND_BF16, v)
    assert r(1.0 + 2.0 ** -8) == 1.0                     # halfway, even is 1.0
    assert r(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6     # halfway, even is up
    assert r(1.0 + 2.0 ** -8 + 2.0 ** -40) == 1.0 + 2.0 ** -7  # just above halfway
    assert r(-2.75) == -2.75 and r(0.0) == 0.0
    assert r(3.0 * 2.0 ** -130) == 3.0 * 2.0 ** -130   # bf16 subnormal spacing 2^-133


def test_round_matches_torch_on_float_inputs(oracle_mod):
    """torch's float32 -> bfloat16 conversion is round-to-nearest-even; on
    values that are exact floats the oracle must agree bit for bit."""
    x = torch.randn(4096, generator=torch.Generator().manual_seed(3), dtype=torch.float32) * 37.0
    want = x.to(torch.bfloat16).double().numpy()
    got = np.array([oracle_mod.round_to(oracle_mod.ROUND_BF16, float(v)) for v in x.double().numpy()])
    assert np.array_equal(got, want)
    xd = torch.randn(2048, generator=torch.Generator().manual_seed(4), dtype=torch.float64)
    want32 = xd.float().double().numpy()
    got32 = np.array([oracle_mod.round_to(oracle_mod.ROUND_F32, float(v)) for v in xd.numpy()])
    assert np.array_equal(got32, want32)


# ---------------------------------------------------------------- activation

def test_gelu_matches_printed_normal_cdf(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "normal_cdf.json")))
    for z, phi in zip(g["z"], g["Phi"]):
        assert oracle_mod.act(oracle_mod.ACT_GELU_ERF, z) == pytest.approx(z * phi, rel=0, abs=2e-15 * (1 + z))
        # GELU(-z) = -z * (1 - Phi(z))
        assert oracle_mod.act(oracle_mod.ACT_GELU_ERF, -z) == pytest.approx(-z * (1 - phi), abs=2e-15 * (1 + z))
    assert oracle_mod.act(oracle_mod.ACT_GELU_ERF, 0.0) == 0.0
    assert oracle_mod.act(oracle_mod.ACT_GELU_ERF, 40.0) == 40.0
    assert oracle_mod.act(oracle_mod.ACT_GELU_ERF, -40.0) == 0.0
    assert oracle_mod.act(oracle_mod.ACT_NONE, -1.25) == -1.25


def test_gelu_tanh_matches_values_worked_from_its_definition(oracle_mod):
    """The tanh form z/2 (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))) against its
    definition worked step by step in 60-digit decimal arithmetic
    (tests/golden/gelu_tanh.json, written by make_gelu_tanh.py).  At 1e-15 this
    catches any wrong constant (0.0447 for 0.044715 moves the value at z = 2 by
    about 2e-6), a dropped half, a wrong power or a sign error."""
    g = json.load(open(os.path.join(GOLDEN, "gelu_tanh.json")))
    assert len(g["rows"]) >= 7
    for r in g["rows"]:
        want = float(r["gelu_tanh"])
        got = oracle_mod.act(oracle_mod.ACT_GELU_TANH, r["z"])
        assert abs(got - want) <= 4e-16 * max(1.0, abs(want)), (r["z"], got, want)


def test_gelu_tanh_identities_and_limits(oracle_mod):
    """tanh is odd, so f(z) - f(-z) = z/2 (1 + th) + z/2 (1 - th) = z for every
    z; large |z| gives z and 0; and the form stays within the known worst-case
    distance of exact GELU (4.73e-4, reached near |z| = 2.70) without being it."""
    f = lambda z: oracle_mod.act(oracle_mod.ACT_GELU_TANH, float(z))  # noqa: E731
    for z in np.linspace(-6.0, 6.0, 241):
        assert abs(f(z) - f(-z) - z) <= 1e-15 * (1.0 + abs(z))
    assert f(40.0) == 40.0 and f(-40.0) == 0.0 and f(0.0) == 0.0
    zs = np.linspace(-8.0, 8.0, 16001)
    gap = max(abs(f(z) - oracle_mod.act(oracle_mod.ACT_GELU_ERF, float(z))) for z in zs)
    assert 4.6e-4 <= gap <= 4.8e-4, gap


# ---------------------------------------------------------------------- MLP

def test_mlp_linear_case_is_matrix_product(oracle_mod):
    """With no nonlinearity the two layers collapse to (W2 W1) x + W2 b1 + b2,
    evaluated here by numpy with the matrices multiplied first.  Non-square
    weights catch a transposed operand."""
    rng = _rng(7)
    W1, b1 = rng.normal(size=(5, 3)), rng.normal(size=5)
    W2, b2 = rng.normal(size=(2, 5)), rng.normal(size=2)
    x = rng.normal(size=3)
    y = oracle_mod.mlp(x, W1, b1, W2, b2, oracle_mod.ACT_NONE)
    assert np.allclose(y, (W2 @ W1) @ x + W2 @ b1 + b2, rtol=1e-13, atol=1e-13)


def test_mlp_one_hot_weights_route_elements(oracle_mod):
    """One-hot weights pick single entries: checks row/column roles and that
    the nonlinearity is applied between the layers, not after them."""
    W1 = np.zeros((4, 3)); W1[2, 1] = 1.0          # h[2] = x[1]
    W2 = np.zeros((2, 4)); W2[1, 2] = 1.0          # y[1] = act(h[2])
    x = np.array([9.0, 1.0, -7.0])
    y = oracle_mod.mlp(x, W1, None, W2, None, oracle_mod.ACT_GELU_ERF)
    assert y[0] == 0.0 and y[1] == pytest.approx(0.841344746068543, abs=1e-15)


# --------------------------------------------------------- worked example

def test_hand_worked_example(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "hand_example.json")))
    K = np.array(g["K"], dtype=np.float64)[:, None]
    V = np.array(g["V"], dtype=np.float64)[:, None]
    arr = lambda v: None if v is None else np.array(v, dtype=np.float64)
    idx, code, dk, dk1 = oracle_mod.compress(K, V, arr(g["W1"]), arr(g["b1"]), arr(g["W2"]), arr(g["b2"]),
                                             g["s"], g["k"], oracle_mod.ACT_NONE, oracle_mod.ROUND_BF16)
    assert idx.tolist() == g["expect_idx"]
    assert code.tolist() == g["expect_code"]
    for t, want in enumerate(g["expect_d_k"]):
        if want is None:
            assert math.isnan(dk[t])
        else:
            assert dk[t] == want
    Kh, Vh = oracle_mod.reconstruct(K, V, idx, code, arr(g["W3"]), arr(g["b3"]), arr(g["W4"]), arr(g["b4"]),
                                    g["s"], oracle_mod.ACT_NONE)
    assert Kh[:, 0].tolist() == g["expect_K_hat"]
    assert Vh[:, 0].tolist() == g["expect_V_hat"]
    out = oracle_mod.attention(np.array([g["q"]]), Kh, Vh)
    lg = g["expect_logits"]
    w = [math.exp(v - max(lg)) for v in lg]
    want = sum(wi * vi for wi, vi in zip(w, g["expect_V_hat"])) / sum(w)
    assert out[0, 0] == pytest.approx(want, rel=1e-15)


def test_hand_worked_example_row_by_row(oracle_mod):
    """reconstruct_rows rebuilds the listed tokens of the worked example from
    their slots and codes alone, in any order, to the hand-computed values."""
    g = json.load(open(os.path.join(GOLDEN, "hand_example.json")))
    K = np.array(g["K"], dtype=np.float64)[:, None]
    V = np.array(g["V"], dtype=np.float64)[:, None]
    arr = lambda v: None if v is None else np.array(v, dtype=np.float64)  # noqa: E731
    rows = np.array([3, 0, 1, 4, 2])
    idx = np.array(g["expect_idx"], dtype=np.int32)[rows]
    code = np.array(g["expect_code"], dtype=np.float64)[rows]
    Kh, Vh = oracle_mod.reconstruct_rows(K, V, rows, idx, code, arr(g["W3"]), arr(g["b3"]), arr(g["W4"]),
                                         arr(g["b4"]), g["s"], oracle_mod.ACT_NONE)
    assert Kh[:, 0].tolist() == [g["expect_K_hat"][t] for t in rows]
    assert Vh[:, 0].tolist() == [g["expect_V_hat"][t] for t in rows]


# ---------------------------------------------------------- invariants

def _tokens(T, d_h, n_lat, seed=0, dtype=torch.float32):
    from decode_attention_strided_b200 import synth
    x = synth.head_tokens(seed, 0, 0, 0, T, d_h, n_lat, dtype=dtype).double().numpy()
    return x[:, :d_h].copy(), x[:, d_h:].copy()


def test_reference_rows_reconstruct_exactly(oracle_mod):
    from decode_attention_strided_b200 import synth
    T, d_h, s, k = 200, 16, 8, 2
    K, V = _tokens(T, d_h, 4)
    w = {n: t.double().numpy() for n, t in synth.codec_weights(0, d_h, 8, 32, dtype=torch.float32).items()}
    idx, code, _, _ = oracle_mod.compress(K, V, w["W1"], None, w["W2"], None, s, k)
    Kh, Vh = oracle_mod.reconstruct(K, V, idx, code, w["W3"], None, w["W4"], None, s)
    refs = np.arange(0, T, s)
    assert np.array_equal(Kh[refs], K[refs]) and np.array_equal(Vh[refs], V[refs])
    assert (idx[refs] == -1).all() and (code[refs] == 0).all()


@pytest.mark.parametrize("k", [1, 2, 4])
def test_identity_codec_reconstructs_every_token(oracle_mod, k):
    """Identity compressor/decompressor (d_c = hidden = 2 d_h, W = I, no
    nonlinearity) with fp64 codes: the residual passes through unchanged, so
    every token comes back exactly (sums of a power-of-two count of float32
    values and their differences are exact in double)."""
    from decode_attention_strided_b200 import synth
    T, d_h, s = 300, 8, 4
    K, V = _tokens(T, d_h, 4, seed=5)
    w = {n: t.double().numpy() for n, t in synth.identity_codec(d_h).items()}
    idx, code, _, _ = oracle_mod.compress(K, V, w["W1"], None, w["W2"], None, s, k,
                                          oracle_mod.ACT_NONE, oracle_mod.ROUND_NONE)
    Kh, Vh = oracle_mod.reconstruct(K, V, idx, code, w["W3"], None, w["W4"], None, s, oracle_mod.ACT_NONE)
    k_eff = (idx >= 0).sum(axis=1)
    exact = (k_eff & (k_eff - 1)) == 0      # refs (0) and power-of-two counts
    assert np.array_equal(Kh[exact], K[exact]) and np.array_equal(Vh[exact], V[exact])
    # a count of 3 makes the mean inexact: then only the last bits may move
    assert np.allclose(Kh, K, rtol=2.0 ** -50, atol=0) and np.allclose(Vh, V, rtol=2.0 ** -50, atol=0)
    assert exact.sum() > 0.9 * T


def test_identity_codec_rebuilds_sampled_rows(oracle_mod):
    """reconstruct_rows with the identity codec gives back the listed tokens
    themselves (same exactness argument as the whole-sequence case) and the
    reference rows as stored; a slot that is not strictly earlier than its
    token is refused."""
    from decode_attention_strided_b200 import synth
    T, d_h, s, k = 300, 8, 4, 2
    K, V = _tokens(T, d_h, 4, seed=5)
    w = {n: t.double().numpy() for n, t in synth.identity_codec(d_h).items()}
    idx, code, _, _ = oracle_mod.compress(K, V, w["W1"], None, w["W2"], None, s, k,
                                          oracle_mod.ACT_NONE, oracle_mod.ROUND_NONE)
    rows = _rng(8).choice(T, 60, replace=False)
    Kh, Vh = oracle_mod.reconstruct_rows(K, V, rows, idx[rows], code[rows], w["W3"], None, w["W4"], None, s,
                                         oracle_mod.ACT_NONE)
    assert np.array_equal(Kh, K[rows]) and np.array_equal(Vh, V[rows])
    bad = idx[rows].copy()
    r = int(np.nonzero(rows % s)[0][0])
    bad[r, 0] = rows[r] // s + 1
    with pytest.raises(ValueError):
        oracle_mod.reconstruct_rows(K, V, rows, bad, code[rows], w["W3"], None, w["W4"], None, s, oracle_mod.ACT_NONE)


def test_token_equal_to_its_references_has_zero_residual(oracle_mod):
    """If the k chosen references all equal x_t, the residual and (with no
    biases, GELU(0) = 0) the code are exactly zero and x_t comes back."""
    from decode_attention_strided_b200 import synth
    T, d_h, s, k = 64, 4, 4, 3
    K, V = _tokens(T, d_h, 2, seed=9)
    row_k, row_v = K[5].copy() * 0 + 0.75, V[5].copy() * 0 - 1.5
    for j in (1, 6, 11):                   # three references equal to the token
        K[j * s], V[j * s] = row_k, row_v
    t = 50
    K[t], V[t] = row_k, row_v
    w = {n: t_.double().numpy() for n, t_ in synth.codec_weights(0, d_h, 4, 16, dtype=torch.float32).items()}
    idx, code, dk, _ = oracle_mod.compress(K, V, w["W1"], None, w["W2"], None, s, k)
    assert sorted(idx[t].tolist()) == [1, 6, 11] and dk[t] == 0.0
    assert (code[t] == 0.0).all()
    Kh, Vh = oracle_mod.reconstruct(K, V, idx, code, w["W3"], None, w["W4"], None, s)
    assert np.array_equal(Kh[t], K[t]) and np.array_equal(Vh[t], V[t])
    Kr, Vr = oracle_mod.reconstruct_rows(K, V, [t], idx[t:t + 1], code[t:t + 1], w["W3"], None, w["W4"], None, s)
    assert np.array_equal(Kr[0], K[t]) and np.array_equal(Vr[0], V[t])


# --------------------------------------------------------------- attention

def _sdpa(q, K, V):
    qt = torch.from_numpy(q)[None, :, None, :]             # [1, G, 1, d]
    Kt = torch.from_numpy(K)[None, None].expand(1, q.shape[0], -1, -1)
    Vt = torch.from_numpy(V)[None, None].expand(1, q.shape[0], -1, -1)
    return torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt)[0, :, 0, :].numpy()


def test_stride_one_is_plain_attention(oracle_mod):
    """s = 1 makes every token a reference: decode is ordinary attention,
    here torch's scaled_dot_product_attention in float64."""
    from decode_attention_strided_b200 import synth
    T, d_h = 120, 16
    K, V = _tokens(T, d_h, 4, seed=11)
    w = {n: t.double().numpy() for n, t in synth.codec_weights(0, d_h, 8, 32, dtype=torch.float32).items()}
    idx, code, _, _ = oracle_mod.compress(K, V, w["W1"], None, w["W2"], None, 1, 2)
    assert (idx == -1).all()
    Kh, Vh = oracle_mod.reconstruct(K, V, idx, code, w["W3"], None, w["W4"], None, 1)
    q = _rng(3).normal(size=(4, d_h))
    assert np.allclose(oracle_mod.attention(q, Kh, Vh), _sdpa(q, K, V), rtol=1e-12, atol=1e-12)


def test_identity_codec_attention_is_full_cache_attention(oracle_mod):
    from decode_attention_strided_b200 import synth
    T, d_h, s = 256, 8, 8
    K, V = _tokens(T, d_h, 4, seed=12)
    w = {n: t.double().numpy() for n, t in synth.identity_codec(d_h).items()}
    idx, code, _, _ = oracle_mod.compress(K, V, w["W1"], None, w["W2"], None, s, 2,
                                          oracle_mod.ACT_NONE, oracle_mod.ROUND_NONE)
    Kh, Vh = oracle_mod.reconstruct(K, V, idx, code, w["W3"], None, w["W4"], None, s, oracle_mod.ACT_NONE)
    q = _rng(4).normal(size=(2, d_h))
    assert np.allclose(oracle_mod.attention(q, Kh, Vh), _sdpa(q, K, V), rtol=1e-12, atol=1e-12)


def test_attention_closed_forms(oracle_mod):
    rng = _rng(5)
    V = rng.normal(size=(7, 3))
    K = rng.normal(size=(7, 3))
    # single token: the output is that token's value
    assert np.array_equal(oracle_mod.attention(np.ones((1, 3)), K[:1], V[:1])[0], V[0])
    # zero query: equal weights, the output is the mean value row
    assert np.allclose(oracle_mod.attention(np.zeros((1, 3)), K, V)[0], V.mean(axis=0), rtol=1e-14, atol=1e-15)
    # two tokens whose scaled logits differ by delta: weights 1 : e^delta
    K2 = np.array([[0.0, 0, 0], [3.0, 0, 0]])
    q = np.array([[1.0, 0, 0]])
    delta = 3.0 / math.sqrt(3.0)
    want = (V[0] + math.exp(delta) * V[1]) / (1 + math.exp(delta))
    assert np.allclose(oracle_mod.attention(q, K2, V[:2])[0], want, rtol=1e-14)
    # head order: permuting the query heads permutes the outputs
    Q = rng.normal(size=(3, 3))
    o = oracle_mod.attention(Q, K, V)
    assert np.array_equal(oracle_mod.attention(Q[::-1].copy(), K, V), o[::-1])


# ------------------------------------------------- streaming and sparse use

def test_compression_of_a_token_depends_only_on_its_prefix(oracle_mod):
    """Compression looks only at earlier references (the "historical" tokens
    of step 1), so a cache built over a prefix [0, T0) and extended later
    holds exactly what one pass over [0, T) writes for those tokens; later
    tokens, even references that nearly copy an earlier token, change nothing
    before them.  A search over every reference would change the slots of 69
    of the prefix's tokens here."""
    from decode_attention_strided_b200 import synth
    T, T0, d_h, s, k = 160, 97, 8, 4, 3
    K, V = _tokens(T, d_h, 4, seed=21)
    w = {n: t.double().numpy() for n, t in synth.codec_weights(0, d_h, 8, 32, dtype=torch.float32).items()}
    full = oracle_mod.compress(K, V, w["W1"], None, w["W2"], None, s, k)
    # make the later references near-copies of early tokens: a non-causal
    # search would now pick them
    first = -(-T0 // s) * s
    for t in range(first, T, s):
        K[t], V[t] = K[t - first + 1] + 1e-3, V[t - first + 1] - 1e-3
    pre = oracle_mod.compress(K[:T0].copy(), V[:T0].copy(), w["W1"], None, w["W2"], None, s, k)
    full2 = oracle_mod.compress(K, V, w["W1"], None, w["W2"], None, s, k)
    for a, b, c in zip(pre, full, full2):
        assert np.array_equal(a, b[:T0], equal_nan=True) and np.array_equal(a, c[:T0], equal_nan=True)
    # and every selected slot of every token is strictly earlier than it
    t_all = np.arange(T)[:, None]
    sel = full2[0]
    assert ((sel < 0) | (sel * s < t_all)).all()


def test_attention_over_a_list_with_repeats(oracle_mod):
    """Sparse decode attends over the caller's token list as given: a token
    listed twice carries twice the weight.  Closed form for keys whose scaled
    logits differ by delta: list [0, 0, 1] gives weights 2 : e^delta."""
    rng = _rng(6)
    V = rng.normal(size=(2, 4))
    K = np.array([[0.0, 0, 0, 0], [2.0, 0, 0, 0]])
    q = np.array([[1.0, 0, 0, 0]])
    delta = 2.0 / math.sqrt(4.0)
    want = (2 * V[0] + math.exp(delta) * V[1]) / (2 + math.exp(delta))
    t = np.array([0, 0, 1])
    got = oracle_mod.attention(q, K[t], V[t])[0]
    assert np.allclose(got, want, rtol=1e-14, atol=1e-15)


# ------------------------------------------------------------- 4-bit codes

def test_quantize_row4_hand_example(oracle_mod):
    """Worked by hand: c = (0.7, -1.4, 0.35, 0) has max |c| = 1.4 and
    1.4 / 7 = 0.2 = 1.1001100110011..._2 x 2^-3; its bfloat16 keeps 8
    significant bits, 1.1001100|1100... rounds up to 1.1001101_2 x 2^-3 =
    205/1024.  Then c / scale = 3.4966, -6.9932, 1.7483, 0, so q = 3, -7, 2, 0."""
    q, sc = oracle_mod.quantize_row4([0.7, -1.4, 0.35, 0.0])
    assert sc == 205.0 / 1024.0
    assert q.tolist() == [3, -7, 2, 0]


def test_quantize_row4_round_trip_on_representable_rows(oracle_mod):
    """A row that is exactly q * s, with s a bfloat16 value and integers
    |q_i| <= 7 of which one is +-7, comes back as the same q and s."""
    rng = _rng(31)
    for _ in range(200):
        m = int(rng.integers(128, 256))                  # 8 significant bits
        s = m * 2.0 ** int(rng.integers(-20, 5))
        d_c = int(rng.choice([16, 32, 64]))
        q = rng.integers(-7, 8, size=d_c)
        q[int(rng.integers(d_c))] = 7 if rng.random() < 0.5 else -7
        got_q, got_s = oracle_mod.quantize_row4(q * s)
        assert got_s == s and got_q.tolist() == q.tolist()


def test_quantize_row4_ties_zero_row_and_error_bound(oracle_mod):
    # scale 1: halfway values go to the even integer
    q, sc = oracle_mod.quantize_row4([7.0, 0.5, 1.5, 2.5, -0.5, -2.5, -3.5])
    assert sc == 1.0 and q.tolist() == [7, 0, 2, 2, 0, -2, -4]
    q, sc = oracle_mod.quantize_row4(np.zeros(32))
    assert sc == 0.0 and not q.any()
    # every element within half a step of its dequantised value
    rng = _rng(32)
    for _ in range(100):
        c = rng.normal(size=32) * rng.uniform(0.01, 10)
        q, sc = oracle_mod.quantize_row4(c)
        assert np.all(np.abs(q) <= 7)
        assert np.all(np.abs(c - q * sc) <= sc / 2 * (1 + 1e-12) + 1e-300)


def test_compress_with_4bit_codes_stores_quantised_rows(oracle_mod):
    """With 4-bit codes every stored code row is the dequantised quantisation
    of the code the compressor computes (the same compression without
    rounding), and slots and distances are unchanged."""
    from decode_attention_strided_b200 import synth
    T, d_h, s, k = 150, 8, 4, 2
    K, V = _tokens(T, d_h, 4, seed=33)
    w = {n: t.double().numpy() for n, t in synth.codec_weights(0, d_h, 16, 32, dtype=torch.float32).items()}
    raw = oracle_mod.compress(K, V, w["W1"], None, w["W2"], None, s, k, oracle_mod.ACT_GELU_ERF,
                              oracle_mod.ROUND_NONE)
    q4 = oracle_mod.compress(K, V, w["W1"], None, w["W2"], None, s, k, oracle_mod.ACT_GELU_ERF, oracle_mod.ROUND_Q4)
    assert np.array_equal(raw[0], q4[0])
    for t in range(T):
        if t % s == 0:
            assert not q4[1][t].any()
            continue
        q, sc = oracle_mod.quantize_row4(raw[1][t])
        assert np.array_equal(q4[1][t], q * sc)
