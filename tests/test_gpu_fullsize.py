"""Parity at the benchmark's full size (T = 131072, 8 kv-heads, d_h = 128, bf16,
s = 16, k = 4, d_c = 32, hidden 256), on outputs the oracle can compute one
by one, and a consistency property of the decode at the benchmark's batch.

The GPU runs the whole layer exactly as bench.py launches it; the oracle
recomputes a seeded sample of rows of two heads from the same raw K/V
(`compress_rows` searches all earlier references for each sampled token)."""
import math

import numpy as np
import pytest
import torch

import oracle
from decode_attention_strided_b200 import deltakv as dkv
from decode_attention_strided_b200 import synth
from parity_util import NEAR_TIE_REL, ATTN_MAX_ABS, check_indices, rel_l2

T, H, HQ, D_H, S, K_REF, D_C, HIDDEN, N_LAT = 131072, 8, 32, 128, 16, 4, 32, 256, 8
SAMPLED_HEADS = (2, 7)
N_SAMPLE = 384


def _layer_kv(B, heads_on_cpu, dev):
    """K, V [B, H, T, d_h] bf16 on the GPU; the heads in `heads_on_cpu` of
    sequence 0 are generated on the CPU (the oracle's copy is then the very
    same tensor), the rest on the GPU."""
    K = torch.empty((B, H, T, D_H), dtype=torch.bfloat16, device=dev)
    V = torch.empty_like(K)
    cpu = {}
    for b in range(B):
        for h in range(H):
            on_cpu = b == 0 and h in heads_on_cpu
            x = synth.head_tokens(0, 0, b, h, T, D_H, N_LAT, torch.bfloat16, "cpu" if on_cpu else dev)
            if on_cpu:
                cpu[h] = x
            K[b, h] = x[:, :D_H].to(dev)
            V[b, h] = x[:, D_H:].to(dev)
    return K, V, cpu


@pytest.mark.gpu
def test_full_size_compress_sampled_rows():
    dev = "cuda"
    cfg = dkv.Config(batch=1, kv_heads=H, q_heads=HQ, d_h=D_H, max_T=T, stride_s=S, k=K_REF, d_c=D_C,
                     hidden=HIDDEN)
    p = dkv.plan(cfg)
    K, V, cpu = _layer_kv(1, SAMPLED_HEADS, dev)
    W = synth.codec_weights(0, D_H, D_C, HIDDEN)
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
    planes = p.cache_planes(cache)
    Wf = {n: t.double().numpy() for n, t in W.items()}
    zb = lambda n: np.zeros(n)  # noqa: E731  (no biases in this workload)
    rng = np.random.default_rng(1234)
    for h in SAMPLED_HEADS:
        x = cpu[h].double().numpy()
        Kc, Vc = x[:, :D_H], x[:, D_H:]
        # late tokens dominate the search cost: sample over the whole range
        tokens = np.sort(rng.choice(np.array([t for t in range(1, T) if t % S]), N_SAMPLE, replace=False))
        o_idx, o_code, o_dk, o_dk1 = oracle.compress_rows(Kc, Vc, Wf["W1"], zb(HIDDEN), Wf["W2"], zb(D_C), S, K_REF,
                                                          tokens, oracle.ACT_GELU_ERF, oracle.ROUND_BF16)
        rows = tokens - tokens // S - 1
        g_idx = planes["idx"][0, h, rows].cpu().numpy()
        n, flagged = check_indices(g_idx, o_idx, o_dk, o_dk1, Kc, Vc, tokens, S)
        assert n == N_SAMPLE
        # reconstruction of the sampled rows from the oracle's own slots and
        # codes (mean of the references + decompressor MLP)
        X = np.concatenate([Kc, Vc], axis=1)
        o_rec = np.empty((N_SAMPLE, 2 * D_H))
        for r in range(N_SAMPLE):
            js = [j for j in o_idx[r].tolist() if j >= 0]
            ref = X[np.array(js) * S].mean(axis=0)
            o_rec[r] = ref + oracle.mlp(o_code[r], Wf["W3"], zb(HIDDEN), Wf["W4"], zb(2 * D_H))
        g_rec = torch.cat([Kh[0, h, tokens], Vh[0, h, tokens]], dim=1).double().cpu().numpy()
        e = rel_l2(g_rec, o_rec)
        assert e <= 1e-2, f"head {h}: sampled reconstruction rel L2 {e}"
        # reference rows are stored whole
        refs = np.arange(0, T, S)[::97]
        assert np.array_equal(Kh[0, h, refs].double().cpu().numpy(), Kc[refs])
        print(f"head {h}: {n} sampled rows, {flagged} near ties, reconstruction rel L2 {e:.2e}")


@pytest.mark.gpu
def test_full_size_decode_matches_reconstruction():
    """Batch 8 at T = 131072 in the benchmark's launch configuration: the fused
    decode (which never materialises K or V) equals exact attention over the
    K, V that the reconstruction kernel rebuilds from the same cache, for
    every query head of two sequences."""
    dev = "cuda"
    B = 8
    cfg = dkv.Config(batch=B, kv_heads=H, q_heads=HQ, d_h=D_H, max_T=T, stride_s=S, k=K_REF, d_c=D_C,
                     hidden=HIDDEN)
    p = dkv.plan(cfg)
    K, V, _ = _layer_kv(B, (), dev)
    W = {n: t.to(dev) for n, t in synth.codec_weights(0, D_H, D_C, HIDDEN).items()}
    cache, ws = p.alloc_cache(), p.alloc_workspace()
    dkv.compress(p, T, K, V, W["W1"], None, W["W2"], None, cache, ws)
    del K, V
    q = synth.queries(0, B, HQ, D_H, device=dev)
    out = torch.empty((B, HQ, D_H), dtype=torch.float32, device=dev)
    dkv.set_profiling(p, True)
    dkv.decode_attention(p, T, q, cache, W["W3"], None, W["W4"], None, out, ws)
    assert dkv.device_status(p, ws) == 0
    torch.cuda.synchronize()
    assert "decode_stream_tc" in set(dkv.profile_collect(p))
    Kh = torch.empty((B, H, T, D_H), dtype=torch.float32, device=dev)
    Vh = torch.empty_like(Kh)
    dkv.reconstruct(p, T, cache, W["W3"], None, W["W4"], None, Kh, Vh, ws)
    torch.cuda.synchronize()
    G = HQ // H
    worst = 0.0
    for b in (0, 5):
        for h in range(H):
            qq = q[b, h * G:(h + 1) * G].double()
            lg = (qq @ Kh[b, h].double().T) / math.sqrt(D_H)
            ref = torch.softmax(lg, dim=-1) @ Vh[b, h].double()
            err = float((out[b, h * G:(h + 1) * G].double() - ref).abs().max())
            worst = max(worst, err)
            assert err <= ATTN_MAX_ABS, f"(b={b}, h={h}): {err}"
    print(f"decode vs attention over the reconstruction: max abs {worst:.2e}")
