"""Pins for the oracle's cache layout and state machine (step S).

Method: "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache",
mlsanity.com index page, "Abstract (arXiv)" (keys per channel, values per
token) and study.space summary (key quantization grouped across tokens, value
codes appended along the token axis, quantized and residual parts);
scholarfeed.org "KIVI" page, third quote (fixed-length residual buffer).

Layout (the library's buffer layout, which the oracle writes):
  k_codes [Tq][D/E]: word w of token t holds channels wE..wE+E-1, LSB first
  v_codes [Tq/E][D]: word (tb, d) holds tokens tb*E..tb*E+E-1 of channel d
"""
import numpy as np
import pytest

import oracle


def _cache(D=32, bits=2, G=32, Gv=32, R=32, capacity=128, B=1, Hkv=1, meta_f16=False):
    return oracle.OracleCache(B, Hkv, D, bits, G, Gv, R, capacity, meta_f16=meta_f16)


def test_pack_axes_hand_words():
    # K[t][d] = (t + 2d) mod 4: each key group (channel d over 32 tokens) holds
    # {0,1,2,3}, so s = 1, z = 0 and code = value.  A key word holds 16
    # channels of one token: codes (t + 2i) mod 4 -> by t mod 4:
    #   0: 0,2,0,2 -> 0x88   1: 1,3,1,3 -> 0xdd   2: 2,0,2,0 -> 0x22   3: 3,1,3,1 -> 0x77
    # V[t][d] = (2t + d) mod 4: each value group (token t over 32 channels)
    # holds {0..3}; a value word holds 16 tokens of one channel: codes
    # (2i + d) mod 4 -> the same four words by d mod 4.
    T = 33
    t = np.arange(T)[:, None]
    d = np.arange(32)[None, :]
    K = ((t + 2 * d) % 4).astype(np.float32)
    V = ((2 * t + d) % 4).astype(np.float32)
    c = _cache()
    c.prefill_unit(0, 0, K, V)
    assert (c.unit(0, 0).n_q, c.unit(0, 0).r) == (32, 1)
    table = [0x88888888, 0xDDDDDDDD, 0x22222222, 0x77777777]
    kc = c.k_codes[0]
    for tt in range(32):
        assert kc[tt, 0] == table[tt % 4] and kc[tt, 1] == table[tt % 4]
    vc = c.v_codes[0]
    for tb in range(2):
        for dd in range(32):
            assert vc[tb, dd] == table[dd % 4]
    assert (c.k_scale[0, 0] == 1).all() and (c.k_zero[0, 0] == 0).all()
    assert (c.v_scale[0, :32] == 1).all() and (c.v_zero[0, :32] == 0).all()


def test_scale_zero_indices():
    # K[t][d] = d + (t mod 4): every key group of channel d has zero d, scale 1.
    # V[t][d] = t + (d mod 4): every value group of token t has zero t, scale 1.
    D, Gv = 64, 32
    T = 64 + 7
    t = np.arange(T)[:, None]
    d = np.arange(D)[None, :]
    K = (d + t % 4).astype(np.float32)
    V = (t + d % 4).astype(np.float32)
    c = _cache(D=D, Gv=Gv, R=32, capacity=128)
    c.prefill_unit(0, 0, K, V)
    u = c.unit(0, 0)
    assert (u.n_q, u.r) == (64, 7)
    for g in range(2):
        assert (c.k_zero[0, g] == np.arange(D)).all() and (c.k_scale[0, g] == 1).all()
    for tt in range(64):
        assert (c.v_zero[0, tt] == tt).all() and (c.v_scale[0, tt] == 1).all()
    Kh, Vh = c.dequant_unit(0, 0)
    assert (Kh == K).all() and (Vh == V).all()


def test_grouping_axes_exact_when_groups_are_constant():
    # Keys constant along tokens within each channel (but varying across
    # channels) reconstruct exactly only under per-channel key groups; values
    # constant along channels within each token only under per-token groups.
    rng = np.random.default_rng(0)
    D, T = 32, 64 + 32
    K = np.tile(rng.standard_normal(D).astype(np.float32), (T, 1))
    V = np.tile(rng.standard_normal((T, 1)).astype(np.float32), (1, D))
    c = _cache(D=D, capacity=128)
    c.prefill_unit(0, 0, K, V)
    assert (c.k_scale[0, :2] == 0).all() and (c.v_scale[0, :64] == 0).all()
    Kh, Vh = c.dequant_unit(0, 0)
    assert (Kh == K).all() and (Vh == V).all()


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("T", [0, 1, 31, 32, 33, 63, 64, 65, 96, 127, 128, 129, 200])
def test_prefill_equals_appends(bits, T):
    """prefill(T) and T single appends reach the same state bit for bit."""
    rng = np.random.default_rng(T)
    D, R = 32, 64
    K = (rng.standard_normal((T, D)) * np.where(np.arange(D) == 5, 20, 1)).astype(np.float32)
    V = rng.standard_normal((T, D)).astype(np.float32)
    a = _cache(D=D, bits=bits, R=R, capacity=256)
    b = _cache(D=D, bits=bits, R=R, capacity=256)
    a.prefill_unit(0, 0, K, V)
    for t in range(T):
        b.append_unit(0, 0, K[t], V[t])
    ua, ub = a.unit(0, 0), b.unit(0, 0)
    r_expected = 0 if T == 0 else (T - 1) % R + 1
    assert (ua.n_q, ua.r) == (T - r_expected, r_expected) == (ub.n_q, ub.r)
    for name in ("k_codes", "k_scale", "k_zero", "v_codes", "v_scale", "v_zero"):
        assert np.array_equal(getattr(a, name).view(np.uint32), getattr(b, name).view(np.uint32)), name
    assert np.array_equal(a.k_res[0, :ua.r], b.k_res[0, :ub.r])
    assert np.array_equal(a.v_res[0, :ua.r], b.v_res[0, :ub.r])


@pytest.mark.parametrize("bits", [2, 4])
def test_binary16_metadata_cache_matches_group_quantizer(bits):
    """With binary16 metadata the cache's block quantizer gives, group by
    group, exactly the single-group binary16 quantizer; prefill(T) equals T
    appends; and the metadata are binary16 values."""
    rng = np.random.default_rng(40 + bits)
    D, R, T = 64, 32, 130
    K = (rng.standard_normal((T, D)) * np.where(np.arange(D) % 17 == 3, 20, 1)).astype(np.float16).astype(np.float32)
    V = rng.standard_normal((T, D)).astype(np.float16).astype(np.float32)
    a = _cache(D=D, bits=bits, R=R, capacity=256, meta_f16=True)
    b = _cache(D=D, bits=bits, R=R, capacity=256, meta_f16=True)
    a.prefill_unit(0, 0, K, V)
    for t in range(T):
        b.append_unit(0, 0, K[t], V[t])
    for name in ("k_codes", "k_scale", "k_zero", "v_codes", "v_scale", "v_zero"):
        assert np.array_equal(getattr(a, name).view(np.uint32), getattr(b, name).view(np.uint32)), name
    n_q = a.unit(0, 0).n_q
    for g in range(n_q // 32):
        for d in (0, 3, 17, 63):
            s, z, c = oracle.quantize_group(K[32 * g:32 * g + 32, d], bits, meta_f16=True)
            assert a.k_scale[0, g, d] == s and a.k_zero[0, g, d] == z
    for t in (0, 31, n_q - 1):
        s, z, _ = oracle.quantize_group(V[t, 32:64], bits, meta_f16=True)
        assert a.v_scale[0, t, 1] == s and a.v_zero[0, t, 1] == z
    ks = a.k_scale[0, :n_q // 32]
    assert np.array_equal(ks, ks.astype(np.float16).astype(np.float32))


def test_flush_quantizes_the_window():
    """Appending R+1 tokens to an empty cache flushes the first R through Q+P:
    the quantized store matches a direct quantization of those tokens."""
    rng = np.random.default_rng(5)
    D, R = 32, 64
    K = rng.standard_normal((R + 1, D)).astype(np.float32)
    V = rng.standard_normal((R + 1, D)).astype(np.float32)
    c = _cache(D=D, R=R, capacity=128)
    for t in range(R + 1):
        c.append_unit(0, 0, K[t], V[t])
    u = c.unit(0, 0)
    assert (u.n_q, u.r) == (R, 1)
    assert (c.k_res[0, 0] == K[R]).all()
    for g in range(R // 32):
        for d in range(D):
            s, z, codes = oracle.quantize_group(K[32 * g:32 * g + 32, d], 2)
            assert c.k_scale[0, g, d] == s and c.k_zero[0, g, d] == z
            for i in range(32):
                word = c.k_codes[0, 32 * g + i, d // 16]
                assert (word >> (2 * (d % 16))) & 3 == codes[i]
    for t in range(R):
        s, z, codes = oracle.quantize_group(V[t], 2)
        assert c.v_scale[0, t, 0] == s and c.v_zero[0, t, 0] == z
        for d in range(D):
            assert (c.v_codes[0, t // 16, d] >> (2 * (t % 16))) & 3 == codes[d]


def test_state_errors():
    c = _cache(R=32, capacity=64)
    K = np.zeros((65, 32), np.float32)
    with pytest.raises(oracle.OracleError, match="status 3"):
        c.prefill_unit(0, 0, K, K)  # 65 tokens > capacity 64
    c.prefill_unit(0, 0, K[:64], K[:64])  # n_q = 32, r = 32: full
    with pytest.raises(oracle.OracleError, match="status 2"):
        c.prefill_unit(0, 0, K[:1], K[:1])  # prefill on a non-empty unit
    with pytest.raises(oracle.OracleError, match="status 3"):
        c.append_unit(0, 0, K[0], K[0])  # needs a flush past the store
    e = _cache()
    with pytest.raises(oracle.OracleError, match="status 2"):
        e.decode_unit(0, 0, np.zeros((1, 32), np.float32), 1.0)


def test_rejects_bad_dims():
    u = oracle.Unit()
    u.D, u.bits, u.G, u.Gv, u.R, u.Tq = 30, 2, 32, 32, 32, 32  # D not a multiple of E
    assert oracle.lib().kivi_oracle_check_unit(u) == oracle.ERR_ARG
    u.D, u.bits = 32, 5
    assert oracle.lib().kivi_oracle_check_unit(u) == oracle.ERR_ARG
    u.D, u.bits = 48, 3  # 3-bit blocks are 32 channels
    assert oracle.lib().kivi_oracle_check_unit(u) == oracle.ERR_ARG


def test_three_bit_layout_by_blocks():
    """3 bits: every 32-channel block of a token's keys is three bit-plane
    words at 3w..3w+2, every 32-token block of a channel's values three rows
    3tb..3tb+2 (kivi_oracle_pack_planes, pinned by the golden B lines); the
    codes are those of the group quantizer."""
    D, R = 64, 32
    rng = np.random.default_rng(12)
    K = rng.standard_normal((96, D)).astype(np.float32)
    V = rng.standard_normal((96, D)).astype(np.float32)
    oc = _cache(D=D, bits=3, R=R, capacity=128)
    oc.prefill_unit(0, 0, K, V)
    u = oc.unit(0, 0)
    assert (u.n_q, u.r) == (64, 32)
    kc = np.zeros((64, D), np.uint16)
    for g in range(2):
        for d in range(D):
            kc[32 * g:32 * g + 32, d] = oracle.quantize_group(K[32 * g:32 * g + 32, d], 3)[2]
    vc = np.zeros((64, D), np.uint16)
    for t in range(64):
        for j in range(2):
            vc[t, 32 * j:32 * j + 32] = oracle.quantize_group(V[t, 32 * j:32 * j + 32], 3)[2]
    for t in range(64):
        for w in range(D // 32):
            assert oc.k_codes[0, t, 3 * w:3 * w + 3].tolist() == oracle.pack_planes(kc[t, 32 * w:32 * w + 32])
    for tb in range(2):
        for d in range(D):
            assert oc.v_codes[0, 3 * tb:3 * tb + 3, d].tolist() == oracle.pack_planes(vc[32 * tb:32 * tb + 32, d])
    # reconstruction is c s + z from those codes
    Kh, Vh = oc.dequant_unit(0, 0)
    s = np.repeat(oc.k_scale[0, :2], 32, 0).astype(np.float64)
    z = np.repeat(oc.k_zero[0, :2], 32, 0).astype(np.float64)
    assert np.array_equal(Kh[:64], kc * s + z)
    # attention at 3 bits is attention over that reconstruction
    import torch
    q = rng.standard_normal((2, D)).astype(np.float32)
    out = oc.decode_unit(0, 0, q, 0.125)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q.astype(np.float64))[None, None], torch.from_numpy(Kh)[None, None],
        torch.from_numpy(Vh)[None, None], scale=0.125)[0, 0].numpy()
    assert np.allclose(out, ref, rtol=0, atol=1e-12)
