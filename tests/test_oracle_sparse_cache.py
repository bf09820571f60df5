"""Pins for the oracle's dense-and-sparse cache (KVQuant, codewithpapers.app
page, abstract item (iv): outliers isolated per vector so they do not skew
its quantization range).  Reading: every key group (channel d over G tokens)
keeps its k_out largest magnitudes exactly and every value group (token t
over Gv channels) its v_out largest; the rest is quantized as usual.

The cache is pinned to the group quantizer (itself pinned by hand-worked
golden lines in test_oracle_quantize.py) group by group, to itself under
prefill vs appends, and its reconstruction to the kept values; attention is
checked against torch's scaled_dot_product_attention over that
reconstruction."""
import numpy as np
import pytest
import torch

import oracle

G = Gv = 32


def spiky(rng, T, D, frac=0.02, scale=40.0):
    """Gaussian K or V with a few single-entry spikes (outlier entries)."""
    x = rng.standard_normal((T, D)).astype(np.float32)
    m = rng.random((T, D)) < frac
    x[m] *= scale
    return x


def unpack_keys(oc, i, n_q):
    E, bits = oc.E, oc.bits
    w = oc.k_codes[i, :n_q]
    d = np.arange(oc.D)
    return (w[:, d // E] >> (bits * (d % E)).astype(np.uint32)) & np.uint32((1 << bits) - 1)


def unpack_values(oc, i, n_q):
    E, bits = oc.E, oc.bits
    t = np.arange(n_q)
    w = oc.v_codes[i, t // E]
    return (w >> (bits * (t % E)).astype(np.uint32)[:, None]) & np.uint32((1 << bits) - 1)


def make(bits, D, R, cap, outliers, T, seed):
    rng = np.random.default_rng(seed)
    K, V = spiky(rng, T, D), spiky(rng, T, D)
    oc = oracle.OracleCache(1, 1, D, bits, G, Gv, R, cap, outliers=outliers)
    oc.prefill_unit(0, 0, K, V)
    return oc, K, V


@pytest.mark.parametrize("bits", [1, 2, 4])
@pytest.mark.parametrize("outliers", [(1, 0), (0, 2), (2, 1)])
def test_every_group_is_the_sparse_group_quantizer(bits, outliers):
    D, R = 64, 64
    oc, K, V = make(bits, D, R, 512, outliers, 64 * 5 + 7, seed=bits * 10 + sum(outliers))
    u = oc.unit(0, 0)
    n_q = u.n_q
    kc, vc = unpack_keys(oc, 0, n_q), unpack_values(oc, 0, n_q)
    ko, vo = outliers
    for g in range(n_q // G):
        for d in range(D):
            s, z, c, oi, ov = oracle.quantize_group_sparse(K[g * G:(g + 1) * G, d], bits, ko)
            assert (oc.k_scale[0, g, d], oc.k_zero[0, g, d]) == (np.float32(s), np.float32(z))
            assert kc[g * G:(g + 1) * G, d].tolist() == c.tolist()
            assert oc.k_out_idx[0, g, d, :ko].tolist() == oi.tolist()
            assert oc.k_out_val[0, g, d, :ko].tolist() == ov.tolist()
    for t in range(n_q):
        for j in range(D // Gv):
            s, z, c, oi, ov = oracle.quantize_group_sparse(V[t, j * Gv:(j + 1) * Gv], bits, vo)
            assert (oc.v_scale[0, t, j], oc.v_zero[0, t, j]) == (np.float32(s), np.float32(z))
            assert vc[t, j * Gv:(j + 1) * Gv].tolist() == c.tolist()
            assert oc.v_out_idx[0, t, j, :vo].tolist() == oi.tolist()
            assert oc.v_out_val[0, t, j, :vo].tolist() == ov.tolist()


@pytest.mark.parametrize("outliers", [(1, 1), (3, 2)])
def test_reconstruction_keeps_the_outliers_exactly(outliers):
    D, R = 64, 32
    oc, K, V = make(2, D, R, 256, outliers, 200, seed=4)
    u = oc.unit(0, 0)
    Kh, Vh = oc.dequant_unit(0, 0)
    ko, vo = outliers
    for g in range(u.n_q // G):
        for d in range(D):
            for m in range(ko):
                t = g * G + int(oc.k_out_idx[0, g, d, m])
                assert Kh[t, d] == K[t, d]
    for t in range(u.n_q):
        for j in range(D // Gv):
            for m in range(vo):
                d = j * Gv + int(oc.v_out_idx[0, t, j, m])
                assert Vh[t, d] == V[t, d]
    # the window is exact; a dense entry is c s + z
    assert np.array_equal(Kh[u.n_q:], K[u.n_q:u.n_q + u.r].astype(np.float64))
    kc = unpack_keys(oc, 0, u.n_q)
    dense = kc.astype(np.float64) * np.repeat(oc.k_scale[0, :u.n_q // G], G, 0) + \
        np.repeat(oc.k_zero[0, :u.n_q // G], G, 0)
    kept = np.zeros((u.n_q, D), bool)
    for g in range(u.n_q // G):
        for d in range(D):
            kept[g * G + oc.k_out_idx[0, g, d, :ko], d] = True
    assert np.array_equal(Kh[:u.n_q][~kept], dense[~kept])


@pytest.mark.parametrize("T", [1, 31, 32, 63, 64, 65, 160, 200])
def test_prefill_equals_appends(T):
    D, R = 32, 32
    rng = np.random.default_rng(T)
    K, V = spiky(rng, T, D), spiky(rng, T, D)
    a = oracle.OracleCache(1, 1, D, 2, G, Gv, R, 256, outliers=(2, 1))
    b = oracle.OracleCache(1, 1, D, 2, G, Gv, R, 256, outliers=(2, 1))
    a.prefill_unit(0, 0, K, V)
    for t in range(T):
        b.append_unit(0, 0, K[t], V[t])
    ua, ub = a.unit(0, 0), b.unit(0, 0)
    assert (ua.n_q, ua.r) == (ub.n_q, ub.r)
    for name in ("k_codes", "k_scale", "k_zero", "v_codes", "v_scale", "v_zero", "k_out_idx",
                 "k_out_val", "v_out_idx", "v_out_val"):
        assert np.array_equal(getattr(a, name), getattr(b, name)), name


def test_no_outliers_is_the_plain_cache():
    D, R = 64, 64
    rng = np.random.default_rng(2)
    K, V = spiky(rng, 300, D), spiky(rng, 300, D)
    a = oracle.OracleCache(1, 1, D, 2, G, Gv, R, 512)
    b = oracle.OracleCache(1, 1, D, 2, G, Gv, R, 512, outliers=(0, 0))
    a.prefill_unit(0, 0, K, V)
    b.prefill_unit(0, 0, K, V)
    for name in ("k_codes", "k_scale", "k_zero", "v_codes", "v_scale", "v_zero", "k_res", "v_res"):
        assert np.array_equal(getattr(a, name), getattr(b, name)), name


def test_binary16_metadata_is_not_combined_with_outliers():
    oc = oracle.OracleCache(1, 1, 32, 2, G, Gv, 32, 128, meta_f16=True, outliers=(1, 0))
    with pytest.raises(Exception):
        oc.prefill_unit(0, 0, np.zeros((40, 32), np.float32), np.zeros((40, 32), np.float32))


def test_outliers_shrink_the_key_error_of_spiky_channels():
    """Per-token spikes inside a key channel group: kept exactly, they no
    longer widen the group's range, so the other entries' error falls."""
    D, R = 64, 32
    rng = np.random.default_rng(9)
    K = rng.standard_normal((256, D)).astype(np.float32)
    K[rng.integers(0, 224, 40), rng.integers(0, D, 40)] = 60.0
    V = rng.standard_normal((256, D)).astype(np.float32)
    errs = []
    for ko in (0, 2):
        oc = oracle.OracleCache(1, 1, D, 2, G, Gv, R, 256, outliers=(ko, 0))
        oc.prefill_unit(0, 0, K, V)
        Kh, _ = oc.dequant_unit(0, 0)
        n = oc.unit(0, 0).n_q
        mask = np.abs(K[:n]) < 30  # the non-spike entries
        errs.append(np.max(np.abs(Kh[:n] - K[:n])[mask]))
    assert errs[1] < errs[0] / 4


def test_attention_is_attention_over_the_reconstruction():
    D, R = 64, 32
    oc, K, V = make(2, D, R, 256, (2, 2), 200, seed=6)
    q = np.random.default_rng(1).standard_normal((4, D)).astype(np.float32)
    out = oc.decode_unit(0, 0, q, 0.125)
    Kh, Vh = oc.dequant_unit(0, 0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q.astype(np.float64))[None, :, None, :].transpose(1, 2),
        torch.from_numpy(Kh)[None, None], torch.from_numpy(Vh)[None, None], scale=0.125)
    assert np.allclose(out, ref[0, 0].numpy(), rtol=0, atol=1e-12)
