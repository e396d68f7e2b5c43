"""Seeded synthetic inputs: K/V caches, codec weights and decode queries.

This module draws random numbers and nothing else: it holds none of the
compression method's arithmetic, and both the CUDA path and the CPU oracle
consume what it produces.  It works on any torch device; integer hashing is
exact everywhere, and the float steps run in float64 before one final
rounding to the requested element type.

Randomness is counter based.  Every value is a pure function of
(seed, stream, counter), so one (layer, sequence, kv-head) can be generated
alone and equal its slice of a bigger batch.  The hash is the 32-bit
"lowbias32" integer finaliser (C. Wellons, "Prospecting for Hash Functions",
2018), applied twice around a seed-derived key; normals come from two
uniforms by the Box-Muller transform.

The token model follows the two observations the DeltaKV summary reports
(section 2 "Osservazioni Empiriche"): long-range similarity (more than 60% of
similar tokens lie more than 16 positions apart) and high-norm latent
components shared by many tokens.  For one (layer, sequence, kv-head), with
D = 2 d_h:
  * n_lat latent directions u_i = sqrt(D) g_i / |g_i|, g_i ~ N(0, I_D);
  * a fresh token is x_t = sum_i c_ti u_i + e_t with c ~ N(0, 4), e ~ N(0, 0.25 I);
  * each token t >= 17 is, with probability 0.6, a near copy
    x_t = x_u + N(0, 0.05^2 I) of a source u drawn uniformly from [0, t-17];
  * K_t = x_t[:d_h], V_t = x_t[d_h:].
Codec weights are N(0, 1/fan_in) without biases; queries are N(0, 1).
"""
from __future__ import annotations

import math

import torch

_M32 = 0xFFFFFFFF

# stream identifiers (arbitrary distinct constants)
_S_LAT, _S_COEF, _S_EPS, _S_COPY, _S_SRC, _S_CN = 11, 12, 13, 14, 15, 16
_S_W1, _S_W2, _S_W3, _S_W4, _S_Q = 21, 22, 23, 24, 25

WEIGHT_SEED_BASE = 1000
QUERY_SEED_BASE = 2000


def _mix32_int(x: int) -> int:
    x &= _M32
    x ^= x >> 16
    x = (x * 0x7FEB352D) & _M32
    x ^= x >> 15
    x = (x * 0x846CA68B) & _M32
    x ^= x >> 16
    return x


def _mix32(x: torch.Tensor) -> torch.Tensor:
    # int64 tensors holding values < 2^32; products may wrap, the mask keeps
    # the exact low 32 bits.
    x = x & _M32
    x = x ^ (x >> 16)
    x = (x * 0x7FEB352D) & _M32
    x = x ^ (x >> 15)
    x = (x * 0x846CA68B) & _M32
    x = x ^ (x >> 16)
    return x


def _key(*parts: int) -> int:
    k = 0x243F6A88
    for p in parts:
        k = _mix32_int(k ^ _mix32_int(int(p) & _M32) ^ ((int(p) >> 32) & _M32))
    return k


def uniform(key: int, n: int, device) -> torch.Tensor:
    """n uniforms in (0, 1), float64, from counters 0..n-1 under `key`."""
    c = torch.arange(n, dtype=torch.int64, device=device)
    h = _mix32(_mix32(c ^ key) + (key ^ 0x9E3779B9))
    return (h.to(torch.float64) + 0.5) * (1.0 / 4294967296.0)


def normal(key: int, shape, device) -> torch.Tensor:
    """Standard normals (float64) by Box-Muller from two uniform streams."""
    n = 1
    for d in shape:
        n *= int(d)
    u1 = uniform(_mix32_int(key ^ 0x51ED270B), n, device)
    u2 = uniform(_mix32_int(key ^ 0x2C1B3C6D), n, device)
    z = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)
    return z.reshape(tuple(shape))


def head_tokens(seed: int, layer: int, b: int, h: int, T: int, d_h: int, n_lat: int,
                dtype=torch.bfloat16, device="cpu", copy_prob: float = 0.6,
                min_gap: int = 17):
    """Tokens x [T, 2*d_h] of one (layer, sequence, kv-head), rounded to dtype."""
    D = 2 * d_h
    base = (seed, layer, b, h)
    g = normal(_key(*base, _S_LAT), (n_lat, D), device)
    lat = g * (math.sqrt(D) / torch.linalg.vector_norm(g, dim=1, keepdim=True))
    coef = 2.0 * normal(_key(*base, _S_COEF), (T, n_lat), device)
    x = coef @ lat + 0.5 * normal(_key(*base, _S_EPS), (T, D), device)
    if T > min_gap:
        t = torch.arange(T, device=device, dtype=torch.int64)
        is_copy = (uniform(_key(*base, _S_COPY), T, device) < copy_prob) & (t >= min_gap)
        span = (t - min_gap + 1).clamp(min=1).to(torch.float64)
        src = torch.floor(uniform(_key(*base, _S_SRC), T, device) * span).to(torch.int64)
        src = torch.minimum(src, (t - min_gap).clamp(min=0))
        eta = 0.05 * normal(_key(*base, _S_CN), (T, D), device)
        # x_t = x_src + eta_t along copy chains, resolved by pointer jumping:
        # val holds the sum of the noise (or fresh value) from t down to nxt.
        val = torch.where(is_copy[:, None], eta, x)
        nxt = torch.where(is_copy, src, torch.full_like(src, -1))
        while bool((nxt >= 0).any()):
            live = nxt >= 0
            j = nxt.clamp(min=0)
            val = val + torch.where(live[:, None], val[j], torch.zeros_like(val))
            nxt = torch.where(live, nxt[j], nxt)
        x = val
    return x.to(dtype)


def kv(seed: int, layer: int, B: int, H: int, T: int, d_h: int, n_lat: int,
       dtype=torch.bfloat16, device="cpu"):
    """K, V of shape [B, H, T, d_h] for one layer."""
    K = torch.empty((B, H, T, d_h), dtype=dtype, device=device)
    V = torch.empty((B, H, T, d_h), dtype=dtype, device=device)
    for b in range(B):
        for h in range(H):
            x = head_tokens(seed, layer, b, h, T, d_h, n_lat, dtype, device)
            K[b, h].copy_(x[:, :d_h])
            V[b, h].copy_(x[:, d_h:])
    return K, V


def codec_weights(layer: int, d_h: int, d_c: int, hidden: int, dtype=torch.bfloat16,
                  device="cpu", seed_base: int = WEIGHT_SEED_BASE):
    """Random compressor (W1 [hidden, 2d_h], W2 [d_c, hidden]) and decompressor
    (W3 [hidden, d_c], W4 [2d_h, hidden]) weights, N(0, 1/fan_in), no biases."""
    D = 2 * d_h
    s = seed_base + layer

    def w(stream, rows, cols):
        return (normal(_key(s, stream), (rows, cols), device) / math.sqrt(cols)).to(dtype)

    return {"W1": w(_S_W1, hidden, D), "W2": w(_S_W2, d_c, hidden),
            "W3": w(_S_W3, hidden, d_c), "W4": w(_S_W4, D, hidden)}


def identity_codec(d_h: int, dtype=torch.float32, device="cpu"):
    """Identity compressor/decompressor: d_c = hidden = 2 d_h and every weight
    is the identity matrix (to be used with no nonlinearity)."""
    D = 2 * d_h
    eye = torch.eye(D, dtype=dtype, device=device)
    return {"W1": eye.clone(), "W2": eye.clone(), "W3": eye.clone(), "W4": eye.clone()}


def queries(layer: int, B: int, Hq: int, d_h: int, dtype=torch.bfloat16, device="cpu",
            seed_base: int = QUERY_SEED_BASE):
    """Decode queries q [B, Hq, d_h] ~ N(0, 1)."""
    return normal(_key(seed_base + layer, _S_Q), (B, Hq, d_h), device).to(dtype)
