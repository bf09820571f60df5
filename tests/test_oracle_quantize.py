"""Pins for the oracle's quantizer (Q), packer (P) and dequantizer (D).

Method: "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache",
study.space summary (asymmetric quantization) and mlsanity.com index page,
"Abstract (arXiv)" (2-bit codes).  The pages give no formula or worked
example; the pins are hand-derived values (tests/golden/quantize_examples.txt)
and invariants that any correct asymmetric min/max quantizer satisfies.
"""
import os
import struct

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quantize_examples.txt")


def _f32_bits(x) -> int:
    return struct.unpack("<I", struct.pack("<f", float(x)))[0]


def _golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append([p.strip() for p in line.split("|")])
    return rows


QROWS = [r for r in _golden() if r[0] == "Q"]
PROWS = [r for r in _golden() if r[0] == "P"]
MROWS = [r for r in _golden() if r[0] == "M"]
HROWS = [r for r in _golden() if r[0] == "H"]
SROWS = [r for r in _golden() if r[0] == "S"]
BROWS = [r for r in _golden() if r[0] == "B"]


@pytest.mark.parametrize("row", QROWS, ids=[f"{r[1]}b:{r[2]}" for r in QROWS])
def test_quantize_golden(row):
    _, bits, xs, scale_hex, zero, codes = row
    x = np.array([float(v) for v in xs.split()], np.float32)
    s, z, c = oracle.quantize_group(x, int(bits))
    assert _f32_bits(s) == int(scale_hex, 16)
    assert _f32_bits(z) == _f32_bits(np.float32(float(zero)))  # sign of zero included
    assert c.tolist() == [int(v) for v in codes.split()]


@pytest.mark.parametrize("row", PROWS, ids=[f"{r[1]}b:{r[3]}" for r in PROWS])
def test_pack_golden(row):
    _, bits, codes, word = row
    assert oracle.pack_word([int(v) for v in codes.split()], int(bits)) == int(word, 16)


@pytest.mark.parametrize("row", MROWS, ids=[f"{r[1]}b:{r[2]}" for r in MROWS])
def test_quantize_binary16_metadata_golden(row):
    _, bits, xs, scale_hex, zero, codes = row
    x = np.array([float(v) for v in xs.split()], np.float32)
    s, z, c = oracle.quantize_group(x, int(bits), meta_f16=True)
    assert int(np.float16(s).view(np.uint16)) == int(scale_hex, 16)
    assert float(np.float16(s)) == float(s)  # the stored scale is a binary16 value
    assert _f32_bits(z) == _f32_bits(np.float32(float(zero)))
    assert c.tolist() == [int(v) for v in codes.split()]


@pytest.mark.parametrize("row", HROWS, ids=[r[1] for r in HROWS])
def test_round_half_golden(row):
    _, x_hex, h_hex = row
    x = struct.unpack("<f", struct.pack("<I", int(x_hex, 16)))[0]
    got = oracle.round_half(x)
    want = np.array([int(h_hex, 16)], np.uint16).view(np.float16)[0]
    assert (np.isinf(got) and np.isinf(want) and np.sign(got) == np.sign(want)) or \
        _f32_bits(got) == _f32_bits(np.float32(want))


def test_round_half_matches_numpy_binary16():
    """Against numpy's float16 conversion (round to nearest even) on binary32
    values across every binary16 binade, the subnormals, the ties and the
    overflow boundary."""
    rng = np.random.default_rng(7)
    halves = np.arange(0, 0x7c00, dtype=np.uint16).view(np.float16).astype(np.float32)
    nxt = np.nextafter(halves, np.float32(np.inf))
    prv = np.nextafter(halves, np.float32(0))
    mids = (halves[:-1].astype(np.float64) + halves[1:]) / 2
    xs = np.concatenate([halves, nxt, prv, mids.astype(np.float32),
                         np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
                         rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-8, 5, 20000),
                         np.float32([65504, 65519.996, 65520, 1e6, 1e-9, 3e-8])])
    xs = np.concatenate([xs, -xs])
    with np.errstate(over="ignore"):
        want = xs.astype(np.float16).astype(np.float32)
    got = np.array([oracle.round_half(float(v)) for v in xs], np.float32)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("bits", [2, 4])
def test_binary16_metadata_invariants(bits):
    """Binary16 scale and zero (fp16 inputs, whose minimum is a binary16
    value): codes in range, the minimum reconstructs exactly, and every value
    reconstructs within half a step of the stored grid plus the scale's
    rounding carried over the L steps to the maximum."""
    rng = np.random.default_rng(bits)
    L = (1 << bits) - 1
    for gi in range(400):
        x = (rng.standard_normal(32) * (20.0 if gi % 3 == 0 else 1.0)).astype(np.float16).astype(np.float32)
        s16, z16, c = oracle.quantize_group(x, bits, meta_f16=True)
        s32, z32, _ = oracle.quantize_group(x, bits)
        assert float(np.float16(s16)) == float(s16) and z16 == x.min()
        assert c.min() >= 0 and c.max() <= L
        assert c[int(np.argmin(x))] == 0
        xh = c.astype(np.float64) * s16 + z16
        bound = max(s16 / 2, L * abs(float(s32) - float(s16))) + 4 * np.spacing(np.float32(np.abs(x).max()))
        assert np.all(np.abs(xh - x) <= bound + s16 * 1e-6)


def test_golden_file_covers_every_width():
    assert {int(r[1]) for r in QROWS} >= {1, 2, 3, 4}
    assert {int(r[1]) for r in PROWS} == {1, 2, 4, 8, 16}
    assert len(BROWS) >= 3


@pytest.mark.parametrize("row", BROWS, ids=[r[2] for r in BROWS])
def test_pack_planes_golden(row):
    _, codes, words = row
    assert oracle.pack_planes([int(v) for v in codes.split()]) == [int(w, 16) for w in words.split()]


def test_dequant_closed_form():
    # c * s + z in real arithmetic; these products and sums are exact.
    assert oracle.dequant(0, 0.75, -1.25) == -1.25
    assert oracle.dequant(3, 0.5, -1.0) == 0.5
    assert oracle.dequant(15, 0.125, 2.0) == 3.875
    # binary64 keeps c * s exact where binary32 would round
    s = np.float32(0.1)
    assert oracle.dequant(3, s, 0.0) == 3 * float(s)


def _groups(rng, n_groups, size):
    """Random groups: normal, outlier-heavy (x20 like the key outlier channels),
    tiny-range, constant, and fp16-rounded."""
    out = []
    for i in range(n_groups):
        kind = i % 5
        if kind == 0:
            x = rng.standard_normal(size)
        elif kind == 1:
            x = rng.standard_normal(size) * 20.0
        elif kind == 2:
            x = 1.0 + rng.standard_normal(size) * 1e-6
        elif kind == 3:
            x = np.full(size, rng.standard_normal())
        else:
            x = rng.standard_normal(size).astype(np.float16)
        out.append(np.asarray(x, np.float32))
    return out


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_invariants(bits):
    """Code range; min -> code 0 reconstructing exactly; max -> top code;
    reconstruction error within half a step plus the rounding slack of s,
    the quotient and the float inputs."""
    rng = np.random.default_rng(bits)
    L = 2 ** bits - 1
    for x in _groups(rng, 200, 32):
        s, z, c = oracle.quantize_group(x, bits)
        assert c.min() >= 0 and c.max() <= L
        assert z == x.min()
        if x.max() == x.min():
            assert s == 0 and (c == 0).all()
            assert all(oracle.dequant(ci, s, z) == xi for ci, xi in zip(c, x))
            continue
        imin, imax = int(np.argmin(x)), int(np.argmax(x))
        assert c[imin] == 0 and oracle.dequant(c[imin], s, z) == x.min()
        assert c[imax] == L
        ulp_s = np.spacing(np.float32(s))
        ulp_x = np.spacing(np.float32(max(abs(x.min()), abs(x.max()))))
        bound = float(s) / 2 + (L + 1) * float(ulp_s) + float(ulp_x)
        for ci, xi in zip(c, x):
            assert abs(oracle.dequant(ci, s, z) - float(xi)) <= bound


@pytest.mark.parametrize("bits", [2, 4])
def test_scale_zero_do_not_depend_on_order(bits):
    rng = np.random.default_rng(7)
    for x in _groups(rng, 50, 32):
        s, z, c = oracle.quantize_group(x, bits)
        perm = rng.permutation(x.size)
        s2, z2, c2 = oracle.quantize_group(x[perm], bits)
        assert _f32_bits(s) == _f32_bits(s2) and _f32_bits(z) == _f32_bits(z2)
        assert (c2 == c[perm]).all()


def test_codes_are_monotone_in_x():
    rng = np.random.default_rng(3)
    for bits in (2, 4):
        for x in _groups(rng, 40, 32):
            s, z, c = oracle.quantize_group(x, bits)
            order = np.argsort(x, kind="stable")
            assert (np.diff(c[order].astype(int)) >= 0).all()


def test_sixteen_bit_codes_track_the_input():
    # At b = 16 the step is range / 65535: the reconstruction is nearly exact.
    rng = np.random.default_rng(11)
    x = rng.standard_normal(32).astype(np.float32) * 20
    s, z, c = oracle.quantize_group(x, 16)
    xh = np.array([oracle.dequant(ci, s, z) for ci in c])
    assert np.max(np.abs(xh - x)) <= (x.max() - x.min()) / 65535


# ---- dense-and-sparse variant (KVQuant, codewithpapers.app page, abstract
# item (iv): outliers isolated per vector so they do not skew its range).
# Reading: per group, the k largest magnitudes (lower index first among
# equals) kept exactly with dense code 0, Q over the others in order.

@pytest.mark.parametrize("row", SROWS, ids=[f"{r[1]}b-k{r[2]}:{r[3]}" for r in SROWS])
def test_sparse_golden(row):
    _, bits, k, xs, scale_hex, zero, codes, idx, vals = row
    x = np.array([float(v) for v in xs.split()], np.float32)
    s, z, c, oi, ov = oracle.quantize_group_sparse(x, int(bits), int(k))
    assert _f32_bits(s) == int(scale_hex, 16)
    assert _f32_bits(z) == _f32_bits(np.float32(float(zero)))
    assert c.tolist() == [int(v) for v in codes.split()]
    assert oi.tolist() == [int(v) for v in idx.split()]
    assert ov.tolist() == [float(v) for v in vals.split()]


def test_sparse_golden_covers_ties_and_both_signs():
    ks = {int(r[2]) for r in SROWS}
    assert {0, 1, 2} <= ks and len(SROWS) >= 5


@pytest.mark.parametrize("bits", [1, 2, 4])
def test_sparse_selection_and_reduction(bits):
    """Brute force on random groups with planted outliers: the outlier set is
    the k largest magnitudes (lower index first among equals, found by a
    stable sort); the other codes are those of Q on the remaining entries in
    order; k = 0 is Q exactly; reconstruction is exact on the outliers and
    within Q's bound on the rest."""
    rng = np.random.default_rng(11 + bits)
    for trial in range(300):
        n = int(rng.integers(2, 40))
        x = rng.standard_normal(n).astype(np.float32)
        if trial % 3 == 0:
            x[rng.integers(0, n, 2)] *= 50
        if trial % 5 == 0:
            x[: n // 2] = np.round(x[: n // 2])  # equal magnitudes
        k = int(rng.integers(0, min(n, 5)))
        s, z, c, oi, ov = oracle.quantize_group_sparse(x, bits, k)
        order = sorted(range(n), key=lambda i: (-abs(float(x[i])), i))
        want = sorted(order[:k])
        assert oi.tolist() == want
        assert np.array_equal(ov, x[want])
        keep = [i for i in range(n) if i not in set(want)]
        s0, z0, c0 = oracle.quantize_group(x[keep], bits)
        assert _f32_bits(s) == _f32_bits(s0) and _f32_bits(z) == _f32_bits(z0)
        assert c[keep].tolist() == c0.tolist() and all(c[i] == 0 for i in want)
        if k == 0:
            s1, z1, c1 = oracle.quantize_group(x, bits)
            assert _f32_bits(s) == _f32_bits(s1) and c.tolist() == c1.tolist()
        # reconstruction: outliers exact, the rest within the bound over their range
        xr = x[keep].astype(np.float64)
        xh = np.array([oracle.dequant(int(c[i]), s, z) for i in keep])
        L = 2 ** bits - 1
        bound = s / 2 + 2 ** bits * np.spacing(np.float32(s)) + np.spacing(np.float32(np.max(np.abs(xr))))
        assert np.all(np.abs(xh - xr) <= bound + 1e-12)
        assert np.all(c <= L)


def test_sparse_isolation_narrows_the_error_of_a_skewed_group():
    """One planted outlier: isolating it shrinks the step by the outlier's
    share of the range, and the other entries' error to within half the new
    step (with it, they all fall on code 0, off by their own spread)."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal(32).astype(np.float32)
    x[7] = 200.0
    s0, z0, c0 = oracle.quantize_group(x, 2)
    s1, z1, c1, oi, ov = oracle.quantize_group_sparse(x, 2, 1)
    assert oi.tolist() == [7] and ov.tolist() == [200.0]
    rest = [i for i in range(32) if i != 7]
    e0 = max(abs(oracle.dequant(int(c0[i]), s0, z0) - float(x[i])) for i in rest)
    e1 = max(abs(oracle.dequant(int(c1[i]), s1, z1) - float(x[i])) for i in rest)
    assert s1 < s0 / 30
    assert e1 <= s1 / 2 * (1 + 1e-6)
    assert all(c0[i] == 0 for i in rest) and e1 < e0 / 5
