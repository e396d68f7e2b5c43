"""Host-side arithmetic of bench.py (no GPU): the algorithmic work it
divides by the measured kernel time, and the roofline fields built from it."""
import math
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _shape(T=131072, layers=32, decode_batch=8):
    return bench.Shape(types.SimpleNamespace(layers=layers, T=T, decode_batch=decode_batch))


def test_search_flops_match_a_direct_sum():
    """2 D sum over non-reference tokens t < T of ceil(t / s) (the number of
    strictly earlier references each one is compared with), per kv-head."""
    for T in (1, 2, 16, 17, 100, 1000, 4099):
        sh = _shape(T=T)
        direct = sum(math.ceil(t / sh.s) for t in range(T) if t % sh.s)
        assert sh.cand_flops_per_layer(1) == 2 * (2 * sh.d_h) * direct * sh.H
        assert sh.cand_flops_per_layer(3) == 3 * sh.cand_flops_per_layer(1)


def test_compressed_token_counts():
    sh = _shape(T=131072)
    assert sh.n_ref == 8192 and sh.n_code == 131072 - 8192
    sh = _shape(T=33)
    assert sh.n_ref == 3 and sh.n_code == 30  # references 0, 16, 32


def test_decode_bytes_of_the_128k_batch8_layer():
    """Reference rows (K and V) + code and slot rows per (sequence, kv-head),
    the queries and float32 outputs, and the decompressor weights once."""
    sh = _shape()
    per_head = 8192 * 2 * 128 * 2 + (131072 - 8192) * (32 * 2 + 4 * 4)
    want = per_head * 8 * 8 + 8 * 32 * 128 * (2 + 4) + (256 * 32 + 256 * 256) * 2
    assert sh.decode_bytes_per_layer() == want == 897925120


def test_roofline_fields():
    sh = _shape()
    peaks = {"bf16_tflops_sustained": 1000.0, "hbm_gbs": 5000.0}
    prof = {"candidates_tc": (2, 5.0), "decode_stream_tc": (4, 8.0)}
    r = bench.kernel_rooflines(sh, prof, peaks, "measured")
    c = r["candidates_tc"]
    work = sh.cand_flops_per_layer(1)
    assert c["bound"] == "tensor" and c["unit"] == "TFLOP/s" and c["peak"] == 1000.0
    assert math.isclose(c["achieved"], work / 2.5e-3 / 1e12) and math.isclose(c["frac"], c["achieved"] / 1000.0)
    assert c["ms_per_launch"] == 2.5 and c["traffic"] == 624e6
    d = r["decode_stream_tc"]
    stream = 8 * 8 * (131072 - 8192) * (32 * 2 + 4 * 4)
    assert d["bound"] == "hbm" and math.isclose(d["achieved"], stream / 2e-3 / 1e9)
    assert "encode_tc" not in r  # kernels that did not run get no entry
    # traffic is only quoted for the workload it was measured on
    r2 = bench.kernel_rooflines(_shape(T=65536), prof, peaks, "measured")
    assert r2["candidates_tc"]["traffic"] is None


def test_decode_bounds_of_the_128k_batch8_layer():
    """The decode token loop's floors, recomputed: 8 x 8 x 122880 compressed
    token-heads; 256 activations each at 16 special-function results per clock
    on 148 SMs; 960 chunks per sequence-head of 2 GEMM1 MMAs (128 cycles at
    N = 256) plus 16 z and 16 U MMAs at the 56-cycle minimum."""
    sh = _shape()
    b = bench.decode_bounds(sh, {"hbm_gbs": 5000.0, "bf16_tflops_sustained": 1000.0}, 2000.0)
    th = 8 * 8 * (131072 - 8192)
    assert math.isclose(b["sfu_ms"], th * 256 / (148 * 16 * 2e9) * 1e3)
    assert math.isclose(b["hbm_ms"], sh.decode_bytes_per_layer() / 5e12 * 1e3)
    chunks = 8 * 8 * 960
    assert math.isclose(b["mma_issue_ms"], chunks / 148 * (2 * 128 + 16 * 56 + 16 * 56) / 2e9 * 1e3)
    flops = 2 * th * (32 * 256 + 2 * 256 * 8 + 2 * 256 * 8)
    assert math.isclose(b["tensor_ms"], flops / 1e15 * 1e3)
    assert b["binding"] in ("sfu_ms", "mma_issue_ms")


def test_append_bytes_of_one_token_at_128k():
    """t = T - 1 = 131071 searches ceil(t / 16) = 8192 references: their K
    and V rows plus the token's own row per kv-head (8 heads, one sequence),
    W1 and W2 once, and a 32-element code row and 4 slots written per head."""
    sh = _shape()
    per_head = (8192 + 1) * 256 * 2 + 32 * 2 + 4 * 4
    want = per_head * 8 + (256 * 256 + 256 * 32) * 2
    assert sh.append_bytes_per_layer(131071) == want == 33706624
