"""GPU parity: the CUDA library against the fp64 oracle on seeded inputs.

Covers the 1-layer tiny float32 workload, the identity codec, bfloat16
variants with ragged tails and degenerate strides, strided K/V views, biases,
and the Llama-3.1-8B-shaped single layer at T = 32768 in full.
"""
import math

import numpy as np
import pytest
import torch

from parity_util import Case, check_case, make_inputs, run_gpu, run_oracle_head, rel_l2
from decode_attention_strided_b200 import deltakv as dkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from decode_attention_strided_b200 import build
    build.build()
    import oracle
    oracle.build()


def test_tiny_fp32_workload():
    """1 layer, 1 kv-head, d_h = 64, T = 512, float32, s = 8, k = 2, d_c = 16,
    MLP 128 -> 64 -> 16, 4 latent directions, one decode query."""
    w = check_case(Case(B=1, H=1, Hq=1, d_h=64, T=512, s=8, k=2, d_c=16, hidden=64, dtype=dkv.F32, n_lat=4))
    assert w["rows"] == 512 - 64


def test_identity_codec_reconstructs_and_attends_like_full_cache():
    c = Case(B=1, H=2, Hq=4, d_h=64, T=777, s=8, k=2, d_c=128, hidden=128, dtype=dkv.F32,
             act=dkv.ACT_NONE, identity=True)
    inp = make_inputs(c)
    g = run_gpu(c, inp)
    assert g.status == 0
    for h in range(2):
        K = inp.K[0, h].double().numpy()
        V = inp.V[0, h].double().numpy()
        assert rel_l2(g.K_hat[0, h], K) <= 1e-5 and rel_l2(g.V_hat[0, h], V) <= 1e-5
        import oracle
        o = oracle.attention(inp.q[0, 2 * h:2 * h + 2].double().numpy(), K, V)
        assert np.max(np.abs(g.out[0, 2 * h:2 * h + 2] - o)) <= 5e-3


BF16_CASES = [
    # name, case
    ("base", Case(B=2, H=2, Hq=8, d_h=128, T=4099, s=16, k=4, d_c=32, hidden=256, dtype=dkv.BF16, n_lat=8)),
    ("d_h64_k1", Case(B=1, H=2, Hq=2, d_h=64, T=1000, s=4, k=1, d_c=16, hidden=64, dtype=dkv.BF16)),
    ("k8_dc64", Case(B=1, H=1, Hq=4, d_h=128, T=2053, s=8, k=8, d_c=64, hidden=128, dtype=dkv.BF16)),
    ("s1_all_refs", Case(B=1, H=1, Hq=2, d_h=64, T=300, s=1, k=2, d_c=16, hidden=64, dtype=dkv.BF16)),
    ("T_below_s", Case(B=1, H=1, Hq=1, d_h=64, T=11, s=16, k=4, d_c=16, hidden=64, dtype=dkv.BF16)),
    ("T1", Case(B=2, H=1, Hq=3, d_h=64, T=1, s=16, k=4, d_c=16, hidden=64, dtype=dkv.BF16)),
    ("biases_tanh", Case(B=1, H=2, Hq=4, d_h=128, T=1500, s=16, k=3, d_c=32, hidden=96, dtype=dkv.BF16,
                         act=dkv.ACT_GELU_TANH, biases=True)),
    ("strided_views", Case(B=2, H=3, Hq=6, d_h=64, T=900, s=8, k=2, d_c=16, hidden=64, dtype=dkv.BF16,
                           strided=True)),
    ("ragged_capacity", Case(B=1, H=1, Hq=4, d_h=128, T=2500, s=32, k=4, d_c=32, hidden=256, dtype=dkv.BF16,
                             max_T=5000)),
    ("fp32_biases", Case(B=1, H=1, Hq=2, d_h=64, T=640, s=8, k=3, d_c=32, hidden=64, dtype=dkv.F32, biases=True)),
    # shapes that take the tensor-core compressor and token loop
    ("d_h64_tc", Case(B=1, H=2, Hq=4, d_h=64, T=3001, s=8, k=4, d_c=64, hidden=256, dtype=dkv.BF16)),
    ("biases_tanh_tc", Case(B=1, H=2, Hq=8, d_h=128, T=2600, s=16, k=3, d_c=16, hidden=128, dtype=dkv.BF16,
                            act=dkv.ACT_GELU_TANH, biases=True)),
    ("identity_act_tc", Case(B=1, H=1, Hq=2, d_h=64, T=1800, s=4, k=2, d_c=32, hidden=128, dtype=dkv.BF16,
                             act=dkv.ACT_NONE, biases=True)),
    # eight query heads per kv-head (the widest group the token loop lays out)
    ("g8_tc", Case(B=2, H=2, Hq=16, d_h=128, T=3000, s=16, k=4, d_c=32, hidden=256, dtype=dkv.BF16, n_lat=8)),
    # points of the single-layer sweep (d_h 128, bf16, hidden 256, 8 latent
    # directions), two kv-heads each so that the oracle covers every row
    ("sweep_s4_k1_dc16", Case(B=1, H=2, Hq=8, d_h=128, T=4096, s=4, k=1, d_c=16, hidden=256, dtype=dkv.BF16,
                              n_lat=8)),
    ("sweep_s8_k2_dc64", Case(B=1, H=1, Hq=4, d_h=128, T=16384, s=8, k=2, d_c=64, hidden=256, dtype=dkv.BF16,
                              n_lat=8)),
    ("sweep_s32_k8_dc32", Case(B=1, H=2, Hq=8, d_h=128, T=16384, s=32, k=8, d_c=32, hidden=256, dtype=dkv.BF16,
                               n_lat=8)),
    ("sweep_s16_k4_dc16", Case(B=1, H=2, Hq=8, d_h=128, T=8192, s=16, k=4, d_c=16, hidden=256, dtype=dkv.BF16,
                               n_lat=8)),
]

# kernels each case must have run: the tensor-core paths where the shape allows
TC_EXPECT = {
    "base": {"candidates_tc", "encode_tc", "decode_stream_tc"},
    "k8_dc64": {"encode_tc"},
    "ragged_capacity": {"candidates_tc", "encode_tc", "decode_stream_tc"},
    "d_h64_tc": {"candidates_tc", "encode_tc", "decode_stream_tc"},
    "biases_tanh_tc": {"candidates_tc", "encode_tc", "decode_stream_tc"},
    "identity_act_tc": {"encode_tc", "decode_stream_simt"},
    "g8_tc": {"candidates_tc", "encode_tc", "decode_stream_tc"},
    "sweep_s4_k1_dc16": {"candidates_tc", "encode_tc", "decode_stream_tc"},
    "sweep_s8_k2_dc64": {"candidates_tc", "encode_tc", "decode_stream_tc"},
    "sweep_s32_k8_dc32": {"candidates_tc", "encode_tc", "decode_stream_tc"},
    "sweep_s16_k4_dc16": {"candidates_tc", "encode_tc", "decode_stream_tc"},
}


@pytest.mark.parametrize("name,case", BF16_CASES, ids=[n for n, _ in BF16_CASES])
def test_variants(name, case):
    w = check_case(case)
    missing = TC_EXPECT.get(name, set()) - w["kernels"]
    assert not missing, f"{name}: expected kernels did not run: {sorted(missing)} (ran {sorted(w['kernels'])})"


def test_t1_output_is_the_single_value():
    c = Case(B=1, H=1, Hq=2, d_h=64, T=1, s=4, k=2, d_c=16, hidden=64, dtype=dkv.F32)
    inp = make_inputs(c)
    g = run_gpu(c, inp)
    v0 = inp.V[0, 0, 0].double().numpy()
    assert np.allclose(g.out[0, 0], v0, atol=1e-6) and np.allclose(g.out[0, 1], v0, atol=1e-6)


def test_llama8b_shaped_layer_t32768():
    """8 kv-heads x d_h = 128, T = 32768, bfloat16, s = 16, k = 4, d_c = 32,
    hidden 256, 8 latent directions: every head, every row."""
    c = Case(B=1, H=8, Hq=32, d_h=128, T=32768, s=16, k=4, d_c=32, hidden=256, dtype=dkv.BF16, n_lat=8)
    w = check_case(c)
    print("configs T=32768:", w)


def test_device_error_word_reports_a_bad_slot():
    """A slot index planted out of range in the cache (host-side edit of the
    idx plane) is caught by the decode kernel's range check, latched in the
    workspace and reported by deltakv_device_status; the GPU keeps working."""
    c = Case(B=1, H=1, Hq=1, d_h=64, T=256, s=8, k=2, d_c=16, hidden=64, dtype=dkv.BF16)
    inp = make_inputs(c)
    cfg = dkv.Config(batch=1, kv_heads=1, q_heads=1, d_h=64, max_T=256, stride_s=8, k=2, d_c=16, hidden=64,
                     dtype=dkv.BF16)
    p = dkv.plan(cfg)
    cache, ws = p.alloc_cache(), p.alloc_workspace()
    W = {n: t.cuda() for n, t in inp.W.items()}
    dkv.compress(p, 256, inp.K.cuda(), inp.V.cuda(), W["W1"], None, W["W2"], None, cache, ws)
    assert dkv.device_status(p, ws) == 0
    p.cache_planes(cache)["idx"][0, 0, 100, 0] = 10_000  # > n_ref = 32
    out = torch.empty((1, 1, 64), dtype=torch.float32, device="cuda")
    dkv.decode_attention(p, 256, inp.q.cuda(), cache, W["W3"], None, W["W4"], None, out, ws)
    assert dkv.device_status(p, ws) == 7          # DEVICE_BOUNDS
    assert dkv.device_status(p, ws) == 0          # cleared after reading
    torch.cuda.synchronize()
