"""Parity at the benchmark's full size (T = 131072, 8 kv-heads, d_h = 128, bf16,
hidden 256), in the launch configuration bench.py times.

* Compression of the 32-layer prefill workload (s = 16, k = 4, d_c = 32) on a
  seeded sample of layers (0, 15, 31: each with its own generator seed and
  codec weights), heads and rows, and one point of the single-layer sweep at
  T = 131072 with s = 4, k = 8, d_c = 64.  The GPU compresses the whole layer;
  the oracle recomputes the sampled rows from the same raw K/V
  (`compress_rows` searches all earlier references of each sampled token)
  and rebuilds them from its own slots and codes (`reconstruct_rows`).
* Decode at batch 8 (32 query heads / 8 kv-heads): the fused decode over the
  GPU's cache against the oracle's own compression, reconstruction and fp64
  attention of two whole (sequence, kv-head) pairs, every query head of each.
The oracle never reads anything the CUDA path produced."""
import math

import numpy as np
import pytest
import torch

import oracle
from decode_attention_strided_b200 import deltakv as dkv
from decode_attention_strided_b200 import synth
from parity_util import ATTN_MAX_ABS, check_indices, rel_l2

T, H, HQ, D_H, HIDDEN, N_LAT = 131072, 8, 32, 128, 256, 8
N_SAMPLE = 384

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from decode_attention_strided_b200 import build
    build.build()
    oracle.build()


def _layer_kv(layer, B, on_cpu, dev):
    """K, V [B, H, T, d_h] bf16 on the GPU for layer `layer` (generator seed =
    layer).  The (b, h) pairs in `on_cpu` are generated on the CPU and copied
    over, so the oracle's copy is the very same tensor; the rest are made on
    the GPU."""
    K = torch.empty((B, H, T, D_H), dtype=torch.bfloat16, device=dev)
    V = torch.empty_like(K)
    cpu = {}
    for b in range(B):
        for h in range(H):
            here = (b, h) in on_cpu
            x = synth.head_tokens(layer, layer, b, h, T, D_H, N_LAT, torch.bfloat16, "cpu" if here else dev)
            if here:
                cpu[(b, h)] = x
            K[b, h] = x[:, :D_H].to(dev)
            V[b, h] = x[:, D_H:].to(dev)
    return K, V, cpu


def _check_sampled_compress(layer, s, k, d_c, heads, seed):
    dev = "cuda"
    cfg = dkv.Config(batch=1, kv_heads=H, q_heads=HQ, d_h=D_H, max_T=T, stride_s=s, k=k, d_c=d_c, hidden=HIDDEN)
    p = dkv.plan(cfg)
    K, V, cpu = _layer_kv(layer, 1, {(0, h) for h in heads}, dev)
    W = synth.codec_weights(layer, D_H, d_c, HIDDEN)
    Wd = {n: t.to(dev) for n, t in W.items()}
    cache, ws = p.alloc_cache(), p.alloc_workspace()
    dkv.set_profiling(p, True)
    dkv.compress(p, T, K, V, Wd["W1"], None, Wd["W2"], None, cache, ws)
    Kh = torch.empty((1, H, T, D_H), dtype=torch.float32, device=dev)
    Vh = torch.empty_like(Kh)
    dkv.reconstruct(p, T, cache, Wd["W3"], None, Wd["W4"], None, Kh, Vh, ws)
    assert dkv.device_status(p, ws) == 0
    torch.cuda.synchronize()
    ran = set(dkv.profile_collect(p))
    assert {"candidates_tc", "encode_tc"} <= ran, ran
    del K, V
    planes = p.cache_planes(cache)
    Wf = {n: t.double().numpy() for n, t in W.items()}
    rng = np.random.default_rng(seed)
    for h in heads:
        x = cpu[(0, h)].double().numpy()
        Kc, Vc = x[:, :D_H], x[:, D_H:]
        # late tokens dominate the search cost: sample over the whole range
        tokens = np.sort(rng.choice(np.array([t for t in range(1, T) if t % s]), N_SAMPLE, replace=False))
        o_idx, o_code, o_dk, o_dk1 = oracle.compress_rows(Kc, Vc, Wf["W1"], None, Wf["W2"], None, s, k,
                                                          tokens, oracle.ACT_GELU_ERF, oracle.ROUND_BF16)
        rows = tokens - tokens // s - 1
        g_idx = planes["idx"][0, h, rows].cpu().numpy()
        n, flagged = check_indices(g_idx, o_idx, o_dk, o_dk1, Kc, Vc, tokens, s)
        assert n == N_SAMPLE
        # the sampled rows rebuilt by the oracle from its own slots and codes
        oK, oV = oracle.reconstruct_rows(Kc, Vc, tokens, o_idx, o_code, Wf["W3"], None, Wf["W4"], None, s)
        g_rec = torch.cat([Kh[0, h, tokens], Vh[0, h, tokens]], dim=1).double().cpu().numpy()
        e = rel_l2(g_rec, np.concatenate([oK, oV], axis=1))
        assert e <= 1e-2, f"layer {layer} head {h}: sampled reconstruction rel L2 {e}"
        # reference rows are stored whole
        refs = np.arange(0, T, s)[::97]
        assert np.array_equal(Kh[0, h, refs].double().cpu().numpy(), Kc[refs])
        assert np.array_equal(Vh[0, h, refs].double().cpu().numpy(), Vc[refs])
        print(f"layer {layer} s={s} k={k} d_c={d_c} head {h}: {n} sampled rows, {flagged} near ties, "
              f"reconstruction rel L2 {e:.2e}")


@pytest.mark.parametrize("layer,heads", [(0, (2, 7)), (15, (0, 4)), (31, (3, 6))])
def test_prefill_compress_sampled_rows(layer, heads):
    """The 32-layer, 128k prefill compression (s = 16, k = 4, d_c = 32):
    layers 0, 15 and 31 with their own seeds and weights, two heads each."""
    _check_sampled_compress(layer, 16, 4, 32, heads, seed=1234 + layer)


def test_sweep_point_s4_k8_dc64_at_128k():
    """One point of the single-layer sweep at T = 131072 with another stride,
    k and code width: s = 4 (32768 references per head), k = 8, d_c = 64."""
    _check_sampled_compress(0, 4, 8, 64, (1, 6), seed=99)


@pytest.mark.parametrize("layer", [0])
def test_decode_batch8_against_oracle(layer):
    """Batch 8 at T = 131072 in the benchmark's launch configuration (s = 16,
    k = 4, d_c = 32, 32 query heads over 8 kv-heads).  For (b, h) in
    {(0, 2), (7, 5)} the oracle compresses the whole sequence-head from the
    raw K/V, rebuilds it and runs fp64 attention for the four query heads of
    the group; the fused decode must match within 5e-3.  As an extra, every
    head of sequences 0 and 5 must match exact attention over the K, V that the
    library's reconstruction kernel rebuilds from the same cache."""
    dev = "cuda"
    B, s, k, d_c = 8, 16, 4, 32
    pairs = ((0, 2), (7, 5))
    cfg = dkv.Config(batch=B, kv_heads=H, q_heads=HQ, d_h=D_H, max_T=T, stride_s=s, k=k, d_c=d_c, hidden=HIDDEN)
    p = dkv.plan(cfg)
    K, V, cpu = _layer_kv(100 + layer, B, set(pairs), dev)
    Wc = synth.codec_weights(layer, D_H, d_c, HIDDEN)
    W = {n: t.to(dev) for n, t in Wc.items()}
    cache, ws = p.alloc_cache(), p.alloc_workspace()
    dkv.compress(p, T, K, V, W["W1"], None, W["W2"], None, cache, ws)
    del K, V
    qc = synth.queries(layer, B, HQ, D_H)
    q = qc.to(dev)
    out = torch.empty((B, HQ, D_H), dtype=torch.float32, device=dev)
    dkv.set_profiling(p, True)
    dkv.decode_attention(p, T, q, cache, W["W3"], None, W["W4"], None, out, ws)
    assert dkv.device_status(p, ws) == 0
    torch.cuda.synchronize()
    assert "decode_stream_tc" in set(dkv.profile_collect(p))
    G = HQ // H
    got = out.double().cpu().numpy()
    Wf = {n: t.double().numpy() for n, t in Wc.items()}
    worst = 0.0
    for b, h in pairs:
        x = cpu[(b, h)].double().numpy()
        Kc, Vc = x[:, :D_H], x[:, D_H:]
        idx, code, _, _ = oracle.compress(Kc, Vc, Wf["W1"], None, Wf["W2"], None, s, k, oracle.ACT_GELU_ERF,
                                          oracle.ROUND_BF16)
        Kr, Vr = oracle.reconstruct(Kc, Vc, idx, code, Wf["W3"], None, Wf["W4"], None, s)
        ref = oracle.attention(qc[b, h * G:(h + 1) * G].double().numpy(), Kr, Vr)
        err = float(np.max(np.abs(got[b, h * G:(h + 1) * G] - ref)))
        worst = max(worst, err)
        assert err <= ATTN_MAX_ABS, f"(b={b}, h={h}): decode vs oracle max abs {err}"
    print(f"decode vs oracle (2 sequence-heads, 8 query heads): max abs {worst:.2e}")
    # consistency with the library's own reconstruction, every head of two sequences
    Kh = torch.empty((B, H, T, D_H), dtype=torch.float32, device=dev)
    Vh = torch.empty_like(Kh)
    dkv.reconstruct(p, T, cache, W["W3"], None, W["W4"], None, Kh, Vh, ws)
    torch.cuda.synchronize()
    for b in (0, 5):
        for h in range(H):
            qq = q[b, h * G:(h + 1) * G].double()
            lg = (qq @ Kh[b, h].double().T) / math.sqrt(D_H)
            ref = torch.softmax(lg, dim=-1) @ Vh[b, h].double()
            err = float((out[b, h * G:(h + 1) * G].double() - ref).abs().max())
            assert err <= ATTN_MAX_ABS, f"(b={b}, h={h}) vs reconstruction: {err}"
