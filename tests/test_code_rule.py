"""The quantizer's code rules (csrc/kivi_codes.cuh), built for the host: the
reciprocal fast path with its exact-division fallback (code_of), and the
rounding by 1.5 * 2^23 wherever its group check lets it stand (code_bits),
give clamp(round_half_even(fl(d / s)), 0, L) -- the code the method defines --
on random quotients and, above all, on quotients within a few ulps of every
half-integer, on exact ties, and on scales whose reciprocal overflows."""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_asymmetric_kv_quantize_b200", "csrc")

HARNESS = r'''
#include "kivi_codes.cuh"
extern "C" long long t_mismatches(const float* d, const float* s, long long n, int L,
                                  long long* first) {
  long long bad = 0;
  *first = -1;
  for (long long i = 0; i < n; ++i) {
    const int got = kivi::code_of(d[i], s[i], kivi::recip_rn(s[i]), L);
    volatile float qv = d[i] / s[i];
    int want = (int)nearbyintf(qv);
    want = want < 0 ? 0 : (want > L ? L : want);
    if (got != want) {
      if (*first < 0) *first = i;
      ++bad;
    }
  }
  return bad;
}
// code_bits (the group-checked rounding): wherever codes_need_exact lets it
// stand, its code must equal the exact one; *flagged counts the rest
extern "C" long long t_bits_mismatches(const float* d, const float* s, long long n, int L,
                                       long long* first, long long* flagged) {
  long long bad = 0;
  *first = -1;
  *flagged = 0;
  for (long long i = 0; i < n; ++i) {
    const float rs = kivi::recip_rn(s[i]);
    float ae = 0.0f;
    const unsigned bits = kivi::code_bits(d[i], s[i] != 0.0f ? rs : 0.0f, (float)L, &ae);
    if (s[i] != 0.0f && kivi::codes_need_exact(ae, rs)) {
      ++*flagged;
      continue;
    }
    int want = 0;
    if (s[i] != 0.0f) {  // a conversion that saturates: inf to L, NaN to 0
      volatile float qv = d[i] / s[i];
      const float q = qv;
      want = q >= (float)L ? L : (q > 0.0f ? (int)nearbyintf(q) : 0);
    }
    if ((long long)bits - 0x4B400000LL != want) {
      if (*first < 0) *first = i;
      ++bad;
    }
  }
  return bad;
}
'''


@pytest.fixture(scope="module")
def rule_lib(tmp_path_factory):
    cxx = shutil.which("g++")
    if not cxx:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp("code_rule")
    src = d / "harness.cpp"
    src.write_text(HARNESS)
    so = d / "librule.so"
    subprocess.run([cxx, "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                    "-shared", "-I", CSRC, "-o", str(so), str(src)], check=True)
    L = ctypes.CDLL(str(so))
    L.t_mismatches.restype = ctypes.c_longlong
    L.t_mismatches.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_int,
                               ctypes.POINTER(ctypes.c_longlong)]
    L.t_bits_mismatches.restype = ctypes.c_longlong
    L.t_bits_mismatches.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong,
                                    ctypes.c_int, ctypes.POINTER(ctypes.c_longlong),
                                    ctypes.POINTER(ctypes.c_longlong)]
    return L


def check(lib, d, s, L):
    d = np.ascontiguousarray(d, np.float32)
    s = np.ascontiguousarray(s, np.float32)
    first = ctypes.c_longlong()
    bad = lib.t_mismatches(d.ctypes.data, s.ctypes.data, d.size, L, ctypes.byref(first))
    assert bad == 0, (bad, float(d[first.value]), float(s[first.value]))
    flagged = ctypes.c_longlong()
    bad = lib.t_bits_mismatches(d.ctypes.data, s.ctypes.data, d.size, L, ctypes.byref(first),
                                ctypes.byref(flagged))
    assert bad == 0, ("code_bits", bad, float(d[first.value]), float(s[first.value]))
    return flagged.value


@pytest.mark.parametrize("L", [1, 3, 7, 15])
def test_random_quotients(rule_lib, L):
    rng = np.random.default_rng(L)
    n = 2_000_000
    s = (10.0 ** rng.uniform(-30, 30, n)).astype(np.float32)
    s = s[(s > 0) & np.isfinite(s)]
    d = (s.astype(np.float64) * rng.uniform(0, L * 1.02, s.size)).astype(np.float32)
    flagged = check(rule_lib, d, s, L)
    assert flagged < 1e-4 * d.size  # the group check rarely sends a group to code_of


@pytest.mark.parametrize("L", [1, 3, 15])
def test_quotients_next_to_every_half_integer(rule_lib, L):
    """d / s within 1..40 ulps of k + 1/2, on both sides, for every k."""
    rng = np.random.default_rng(100 + L)
    ds, ss = [], []
    for k in range(L + 1):
        s = (10.0 ** rng.uniform(-20, 20, 20000)).astype(np.float32)
        d = (s.astype(np.float64) * (k + 0.5)).astype(np.float32)
        steps = rng.integers(-40, 41, s.size)
        d = np.array([np.float32(x) for x in d])
        for i in range(s.size):  # nudge by whole ulps
            x = d[i]
            for _ in range(abs(int(steps[i]))):
                x = np.nextafter(x, np.float32(np.inf if steps[i] > 0 else 0))
            d[i] = x
        ds.append(d)
        ss.append(s)
    check(rule_lib, np.concatenate(ds), np.concatenate(ss), L)


def test_exact_ties_go_to_even(rule_lib):
    # s a power of two: d = (k + 1/2) s is exact and so is the quotient
    s = np.array([2.0 ** e for e in range(-100, 100)], np.float32)
    for k in range(16):
        check(rule_lib, (s * np.float32(k + 0.5)).astype(np.float32), s, 15)


def test_tiny_and_huge_scales(rule_lib):
    """Subnormal scales (the reciprocal overflows to infinity: the exact
    division decides), the largest scales, and zero numerators."""
    sub = np.array([2.0 ** -149 * m for m in (1, 2, 3, 5, 7, 100, 1000, 2 ** 20)], np.float32)
    big = np.array([3.4e38, 1.7e38, 1e38], np.float32)
    for s in (sub, big):
        for k in range(4):
            for frac in (0.0, 0.25, 0.5, 0.75, 0.9999):
                with np.errstate(over="ignore"):  # d beyond binary32: inf, code L on both sides
                    d = (s.astype(np.float64) * (k + frac)).astype(np.float32)
                check(rule_lib, d, s, 3)
        check(rule_lib, np.zeros_like(s), s, 3)


@pytest.mark.parametrize("L", [1, 3, 15])
def test_quotients_far_outside_the_code_range(rule_lib, L):
    """Quotients well above L + 1/2 (up to 1e6) and negative numerators (the
    binary16-metadata variant's rounded zero can lie above an element): both
    paths clamp, to L and to 0."""
    rng = np.random.default_rng(300 + L)
    n = 400_000
    s = (10.0 ** rng.uniform(-20, 20, n)).astype(np.float32)
    big = rng.uniform(L + 0.5, 1e6, n)
    d = (s.astype(np.float64) * big).astype(np.float32)
    ok = np.isfinite(d)
    check(rule_lib, d[ok], s[ok], L)
    neg = -rng.uniform(0, 1e6, n)
    d = (s.astype(np.float64) * neg).astype(np.float32)
    ok = np.isfinite(d)
    check(rule_lib, d[ok], s[ok], L)
    # negative quotients next to -1/2 (within 40 ulps on both sides)
    s = (10.0 ** rng.uniform(-20, 20, 5000)).astype(np.float32)
    d = (s.astype(np.float64) * -0.5).astype(np.float32)
    for i in range(d.size):
        x = d[i]
        for _ in range(int(rng.integers(0, 41))):
            x = np.nextafter(x, np.float32(-np.inf if i % 2 else 0))
        d[i] = x
    check(rule_lib, d, s, L)
