"""Pins for the oracle's decode attention (step A).

Method: "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache",
study.space summary: decode attention runs over the quantized part, and the
full-precision residual part is combined with it.  Reading: one softmax over
all n_q + r tokens.

The pins reach outside the oracle: torch's scaled_dot_product_attention in
float64 (a library routine), closed forms, and quantization-exact inputs.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def _sdpa(q, K, V, sigma, gqa=False):
    """Library attention in float64: q [Hq][D], K/V [Hkv][T][D] -> [Hq][D]."""
    qt = torch.as_tensor(np.asarray(q, np.float64))[None, :, None, :]
    Kt = torch.as_tensor(np.asarray(K, np.float64))[None]
    Vt = torch.as_tensor(np.asarray(V, np.float64))[None]
    o = F.scaled_dot_product_attention(qt, Kt, Vt, scale=sigma, enable_gqa=gqa)
    return o[0, :, 0, :].numpy()


def test_hand_example():
    # D = 16 with only channel 0 in use: q = 1, K = [0, ln 3], V = [0, 4]
    # -> weights 1/4, 3/4 -> out = 3 (the window holds both tokens).
    c = oracle.OracleCache(1, 1, 16, 2, 16, 16, 16, 32)
    K = np.zeros((2, 16), np.float32)
    V = np.zeros((2, 16), np.float32)
    K[1, 0] = math.log(3.0)
    V[1, 0] = 4.0
    c.prefill_unit(0, 0, K, V)
    q = np.zeros((1, 16), np.float32)
    q[0, 0] = 1.0
    out = c.decode_unit(0, 0, q, 1.0)
    assert abs(out[0, 0] - 3.0) < 1e-6
    assert (out[0, 1:] == 0).all()


@pytest.mark.parametrize("T", [1, 7, 32])
def test_window_only_is_exact_attention(T):
    """n_q = 0: attention over the stored full-precision tokens equals SDPA."""
    rng = np.random.default_rng(T)
    D = 32
    K = rng.standard_normal((T, D)).astype(np.float32) * 3
    V = rng.standard_normal((T, D)).astype(np.float32)
    q = rng.standard_normal((2, D)).astype(np.float32)
    c = oracle.OracleCache(1, 1, D, 2, 32, 32, 32, 64)
    c.prefill_unit(0, 0, K, V)
    assert c.unit(0, 0).n_q == 0
    sigma = 1 / math.sqrt(D)
    out = c.decode_unit(0, 0, q, sigma)
    ref = _sdpa(q, K[None], V[None], sigma, gqa=True)
    assert np.max(np.abs(out - ref)) < 1e-12


def test_quantization_exact_inputs_give_unquantized_attention():
    """Inputs on the quantization grid (per-channel keys and per-token values
    taking 4 equally spaced binary fractions with both ends present) reconstruct
    exactly at 2 bits, so attention over the quantized part plus the window
    equals plain attention on the inputs."""
    rng = np.random.default_rng(1)
    D, T = 32, 64 + 32 + 9
    ks = 2.0 ** rng.integers(-3, 2, size=D)
    kz = rng.integers(-8, 8, size=D) / 4
    K = (kz + ks * rng.integers(0, 4, size=(T, D))).astype(np.float32)
    K[0:4] = kz + ks * np.arange(4)[:, None]      # both ends in every key group
    K[32:36] = kz + ks * np.arange(4)[:, None]
    K[64:68] = kz + ks * np.arange(4)[:, None]
    vs = 2.0 ** rng.integers(-3, 2, size=(T, 1))
    vz = rng.integers(-8, 8, size=(T, 1)) / 4
    cv = rng.integers(0, 4, size=(T, D))
    cv[:, 0], cv[:, 1] = 0, 3
    V = (vz + vs * cv).astype(np.float32)
    c = oracle.OracleCache(1, 1, D, 2, 32, 32, 32, 128)
    c.prefill_unit(0, 0, K, V)
    assert (c.unit(0, 0).n_q, c.unit(0, 0).r) == (96, 9)
    Kh, Vh = c.dequant_unit(0, 0)
    assert (Kh == K).all() and (Vh == V).all()
    q = rng.standard_normal((3, D)).astype(np.float32)
    out = c.decode_unit(0, 0, q, 0.3)
    assert np.max(np.abs(out - _sdpa(q, K[None], V[None], 0.3, gqa=True))) < 1e-12


def test_attention_over_dequantized_cache_matches_library():
    """Quantized part + window: the oracle's softmax equals SDPA applied to the
    oracle's own reconstruction (isolates A from Q/P/D)."""
    rng = np.random.default_rng(2)
    D, T = 64, 3 * 32 + 17
    K = rng.standard_normal((T, D)).astype(np.float32)
    K[:, [3, 40]] *= 20
    V = rng.standard_normal((T, D)).astype(np.float32)
    c = oracle.OracleCache(1, 1, D, 2, 32, 32, 32, 160)
    c.prefill_unit(0, 0, K, V)
    Kh, Vh = c.dequant_unit(0, 0)
    q = (rng.standard_normal((4, D)) / 8).astype(np.float32)
    out = c.decode_unit(0, 0, q, 1.0)
    assert np.max(np.abs(out - _sdpa(q, Kh[None], Vh[None], 1.0, gqa=True))) < 1e-12


def test_constant_values_and_zero_query():
    rng = np.random.default_rng(4)
    D, T = 32, 100
    K = rng.standard_normal((T, D)).astype(np.float32)
    V = np.full((T, D), 0.625, np.float32)
    c = oracle.OracleCache(1, 1, D, 2, 32, 32, 32, 128)
    c.prefill_unit(0, 0, K, V)
    q = rng.standard_normal((1, D)).astype(np.float32)
    assert np.max(np.abs(c.decode_unit(0, 0, q, 1.0) - 0.625)) < 1e-14
    V2 = rng.standard_normal((T, D)).astype(np.float32)
    c2 = oracle.OracleCache(1, 1, D, 2, 32, 32, 32, 128)
    c2.prefill_unit(0, 0, K, V2)
    _, Vh = c2.dequant_unit(0, 0)
    out = c2.decode_unit(0, 0, np.zeros((1, D), np.float32), 1.0)
    assert np.max(np.abs(out[0] - Vh.mean(axis=0))) < 1e-12


def test_sixteen_bit_cache_approaches_unquantized_attention():
    """Brute force: with 16-bit codes the quantized cache is nearly the input,
    and the error shrinks about 256x from 8 to 16 bits."""
    rng = np.random.default_rng(6)
    D, T = 32, 256
    K = rng.standard_normal((T, D)).astype(np.float32)
    K[:, [3, 17]] *= 20
    V = rng.standard_normal((T, D)).astype(np.float32)
    q = (rng.standard_normal((1, D)) / math.sqrt(D)).astype(np.float32)
    ref = _sdpa(q, K[None], V[None], 1.0, gqa=True)
    errs = {}
    for bits in (8, 16):
        c = oracle.OracleCache(1, 1, D, bits, 32, 32, 32, 256)
        c.prefill_unit(0, 0, K, V)
        errs[bits] = np.max(np.abs(c.decode_unit(0, 0, q, 1.0) - ref))
    assert errs[16] < 1e-4
    assert errs[16] < errs[8] / 64


def test_gqa_head_mapping():
    """Query head hq reads KV head hq // (Hq/Hkv): matches SDPA's grouped heads."""
    rng = np.random.default_rng(9)
    B, Hkv, Hq, D, T = 2, 2, 6, 32, 20
    K = rng.standard_normal((B, Hkv, T, D)).astype(np.float32)
    V = rng.standard_normal((B, Hkv, T, D)).astype(np.float32)
    q = rng.standard_normal((B, Hq, D)).astype(np.float32)
    c = oracle.OracleCache(B, Hkv, D, 2, 32, 32, 32, 64)
    c.prefill(K, V)
    out = c.decode(q, 0.5)
    for b in range(B):
        assert np.max(np.abs(out[b] - _sdpa(q[b], K[b], V[b], 0.5, gqa=True))) < 1e-12
