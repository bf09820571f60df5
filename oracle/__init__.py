"""Plain CPU oracle for the KIVI asymmetric 2/4-bit KV cache (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this package.  It wraps ``kivi_oracle.c`` (plain C99,
binary32 quantizer, binary64 attention) through ctypes and shares no code
with the CUDA library.

Every function cites the passage it follows in ``kivi_oracle.c``.  The
Python side only moves numpy arrays in and out; all arithmetic is in C.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kivi_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

OK, ERR_ARG, ERR_STATE, ERR_CAPACITY, ERR_NOMEM = 0, 1, 2, 3, 4

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``kivi_oracle.c`` into ``liboracle.so`` (gcc, no fast-math, no FMA contraction)."""
    srcs = [_SRC, os.path.join(_HERE, "kivi_oracle.h")]
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= max(os.path.getmtime(s) for s in srcs)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class Unit(ctypes.Structure):
    """Mirror of ``kivi_oracle_unit``: one (batch element, KV head) of the cache."""

    _fields_ = [
        ("D", ctypes.c_int), ("bits", ctypes.c_int), ("G", ctypes.c_int),
        ("Gv", ctypes.c_int), ("R", ctypes.c_int), ("Tq", ctypes.c_longlong),
        ("k_codes", ctypes.c_void_p), ("k_scale", ctypes.c_void_p), ("k_zero", ctypes.c_void_p),
        ("v_codes", ctypes.c_void_p), ("v_scale", ctypes.c_void_p), ("v_zero", ctypes.c_void_p),
        ("k_res", ctypes.c_void_p), ("v_res", ctypes.c_void_p),
        ("n_q", ctypes.c_longlong), ("r", ctypes.c_int), ("meta_f16", ctypes.c_int),
        ("k_out", ctypes.c_int), ("v_out", ctypes.c_int),
        ("k_out_idx", ctypes.c_void_p), ("k_out_val", ctypes.c_void_p),
        ("v_out_idx", ctypes.c_void_p), ("v_out_val", ctypes.c_void_p),
    ]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            # A test may point this at a deliberately broken build of the
            # oracle (tests/test_oracle_mutants.py) to check that the pins fail.
            path = os.environ.get("KIVI_ORACLE_LIB") or build()
            L = ctypes.CDLL(path)
            vp, ll, ci = ctypes.c_void_p, ctypes.c_longlong, ctypes.c_int
            up = ctypes.POINTER(Unit)
            L.kivi_oracle_quantize_group.argtypes = [vp, ll, ll, ci, vp, vp, vp]
            L.kivi_oracle_quantize_group_meta.argtypes = [vp, ll, ll, ci, ci, vp, vp, vp]
            L.kivi_oracle_quantize_group_sparse.argtypes = [vp, ll, ll, ci, ci, vp, vp, vp, vp, vp]
            L.kivi_oracle_pack_planes.argtypes = [vp, vp]
            L.kivi_oracle_pack_planes.restype = None
            L.kivi_oracle_round_half.argtypes = [ctypes.c_float]
            L.kivi_oracle_round_half.restype = ctypes.c_float
            L.kivi_oracle_pack_word.argtypes = [vp, ci]
            L.kivi_oracle_pack_word.restype = ctypes.c_uint32
            L.kivi_oracle_dequant.argtypes = [ctypes.c_uint32, ctypes.c_float, ctypes.c_float]
            L.kivi_oracle_dequant.restype = ctypes.c_double
            L.kivi_oracle_check_unit.argtypes = [up]
            L.kivi_oracle_prefill.argtypes = [up, vp, vp, ll]
            L.kivi_oracle_append.argtypes = [up, vp, vp]
            L.kivi_oracle_dequant_keys.argtypes = [up, vp]
            L.kivi_oracle_dequant_values.argtypes = [up, vp]
            L.kivi_oracle_decode.argtypes = [up, vp, ci, ctypes.c_double, vp]
            _lib = L
        return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags.c_contiguous
    return a.ctypes.data


class OracleError(RuntimeError):
    pass


def _check(rc: int, what: str) -> None:
    if rc != OK:
        raise OracleError(f"{what}: oracle status {rc}")


# ---------------------------------------------------------------- Q, P, D

def quantize_group(x, bits: int, meta_f16: bool = False):
    """Q on one group; returns (scale, zero, codes[uint16]).  meta_f16: the
    binary16-metadata format variant (scale and zero rounded to binary16, codes
    chosen against the rounded values)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    s = np.zeros(1, np.float32)
    z = np.zeros(1, np.float32)
    c = np.zeros(x.size, np.uint16)
    _check(lib().kivi_oracle_quantize_group_meta(_ptr(x), x.size, 1, bits, int(bool(meta_f16)),
                                                 _ptr(s), _ptr(z), _ptr(c)),
           "quantize_group")
    return s[0], z[0], c


def quantize_group_sparse(x, bits: int, k: int):
    """Q, dense-and-sparse variant on one group: returns (scale, zero,
    codes[uint16], outlier indices[int64], outlier values[float32]); the k
    largest-magnitude entries are kept exactly, the rest quantized by Q."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    s, z = ctypes.c_float(), ctypes.c_float()
    codes = np.zeros(x.size, np.uint16)
    idx = np.zeros(max(k, 1), np.int64)
    val = np.zeros(max(k, 1), np.float32)
    _check(lib().kivi_oracle_quantize_group_sparse(_ptr(x), x.size, 1, bits, k, ctypes.byref(s),
                                                   ctypes.byref(z), _ptr(codes), _ptr(idx),
                                                   _ptr(val)), "quantize_group_sparse")
    return s.value, z.value, codes, idx[:k], val[:k]


def pack_planes(codes):
    """32 codes (3-bit) as three bit-plane words."""
    c = np.ascontiguousarray(codes, dtype=np.uint16)
    assert c.size == 32
    w = np.zeros(3, np.uint32)
    lib().kivi_oracle_pack_planes(_ptr(c), _ptr(w))
    return [int(x) for x in w]


def round_half(x: float) -> float:
    """x rounded to the nearest binary16 value (ties to even)."""
    return float(np.float32(lib().kivi_oracle_round_half(ctypes.c_float(float(x)))))


def pack_word(codes, bits: int) -> int:
    """P on one word: 32/bits codes, the first in the least significant bits."""
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint16))
    assert c.size == 32 // bits
    return int(lib().kivi_oracle_pack_word(_ptr(c), bits))


def dequant(c: int, scale: float, zero: float) -> float:
    """D on one code."""
    return float(lib().kivi_oracle_dequant(int(c), float(scale), float(zero)))


# ---------------------------------------------------------------- the cache

class OracleCache:
    """Host-memory KIVI cache in the library's buffer layout, driven by the oracle.

    ``capacity`` is the maximum number of tokens per sequence (quantized plus
    residual), a multiple of ``R``; the quantized store holds ``capacity - R``.
    Buffers (numpy, same shapes as the CUDA library's device buffers):
      k_codes u32 [B][Hkv][Tq][D/E]      k_scale, k_zero f32 [B][Hkv][Tq/G][D]
      v_codes u32 [B][Hkv][Tq/E][D]      v_scale, v_zero f32 [B][Hkv][Tq][D/Gv]
      k_res, v_res f32 [B][Hkv][R][D]
    ``units`` restricts the cache to a subset of (b, h) pairs (the others stay
    empty), so that full-size shapes can be checked on sampled units.
    """

    def __init__(self, B, Hkv, D, bits, G, Gv, R, capacity, units=None, meta_f16=False,
                 outliers=(0, 0)):
        """outliers = (k_out, v_out): the dense-and-sparse variant keeps that
        many largest magnitudes of every key / value group exactly."""
        self.meta_f16 = bool(meta_f16)
        self.k_out, self.v_out = (int(outliers[0]), int(outliers[1]))
        self.B, self.Hkv, self.D, self.bits = B, Hkv, D, bits
        self.G, self.Gv, self.R, self.capacity = G, Gv, R, capacity
        # codes per block and words per block (3 bits: 32 codes in three bit planes)
        E = 32 if bits == 3 else 32 // bits
        WB = 3 if bits == 3 else 1
        self.E, self.WB = E, WB
        Tq = capacity - R
        self.Tq = Tq
        self.units = sorted(set(units)) if units is not None else [
            (b, h) for b in range(B) for h in range(Hkv)]
        self._slot = {u: i for i, u in enumerate(self.units)}
        n = len(self.units)
        self.k_codes = np.zeros((n, Tq, D // E * WB), np.uint32)
        self.k_scale = np.zeros((n, Tq // G, D), np.float32)
        self.k_zero = np.zeros((n, Tq // G, D), np.float32)
        self.v_codes = np.zeros((n, Tq // E * WB, D), np.uint32)
        self.v_scale = np.zeros((n, Tq, D // Gv), np.float32)
        self.v_zero = np.zeros((n, Tq, D // Gv), np.float32)
        self.k_res = np.zeros((n, R, D), np.float32)
        self.v_res = np.zeros((n, R, D), np.float32)
        ko, vo = max(self.k_out, 1), max(self.v_out, 1)
        self.k_out_idx = np.zeros((n, Tq // G, D, ko), np.int32)
        self.k_out_val = np.zeros((n, Tq // G, D, ko), np.float32)
        self.v_out_idx = np.zeros((n, Tq, D // Gv, vo), np.int32)
        self.v_out_val = np.zeros((n, Tq, D // Gv, vo), np.float32)
        self._u = [self._make_unit(i) for i in range(n)]

    def _make_unit(self, i):
        u = Unit()
        u.D, u.bits, u.G, u.Gv, u.R, u.Tq = self.D, self.bits, self.G, self.Gv, self.R, self.Tq
        for name in ("k_codes", "k_scale", "k_zero", "v_codes", "v_scale", "v_zero", "k_res", "v_res",
                     "k_out_idx", "k_out_val", "v_out_idx", "v_out_val"):
            setattr(u, name, getattr(self, name)[i].ctypes.data)
        u.n_q, u.r = 0, 0
        u.meta_f16 = int(self.meta_f16)
        u.k_out, u.v_out = self.k_out, self.v_out
        return u

    def unit(self, b, h) -> Unit:
        return self._u[self._slot[(b, h)]]

    def slot(self, b, h) -> int:
        return self._slot[(b, h)]

    @property
    def n_q(self):
        return self._u[0].n_q

    @property
    def r(self):
        return self._u[0].r

    def prefill_unit(self, b, h, K, V):
        K = np.ascontiguousarray(K, dtype=np.float32)
        V = np.ascontiguousarray(V, dtype=np.float32)
        assert K.shape == V.shape and K.ndim == 2 and K.shape[1] == self.D
        u = self.unit(b, h)
        _check(lib().kivi_oracle_prefill(ctypes.byref(u), _ptr(K), _ptr(V), K.shape[0]), "prefill")

    def prefill(self, K, V):
        """K, V: [B][Hkv][T][D] (any float dtype, converted exactly to float32)."""
        for (b, h) in self.units:
            self.prefill_unit(b, h, np.asarray(K[b, h], np.float32), np.asarray(V[b, h], np.float32))

    def append_unit(self, b, h, k, v):
        k = np.ascontiguousarray(k, dtype=np.float32)
        v = np.ascontiguousarray(v, dtype=np.float32)
        u = self.unit(b, h)
        _check(lib().kivi_oracle_append(ctypes.byref(u), _ptr(k), _ptr(v)), "append")

    def append(self, k, v):
        """k, v: [B][Hkv][D]."""
        for (b, h) in self.units:
            self.append_unit(b, h, np.asarray(k[b, h], np.float32), np.asarray(v[b, h], np.float32))

    def dequant_unit(self, b, h):
        u = self.unit(b, h)
        T = u.n_q + u.r
        Kh = np.zeros((T, self.D), np.float64)
        Vh = np.zeros((T, self.D), np.float64)
        _check(lib().kivi_oracle_dequant_keys(ctypes.byref(u), _ptr(Kh)), "dequant_keys")
        _check(lib().kivi_oracle_dequant_values(ctypes.byref(u), _ptr(Vh)), "dequant_values")
        return Kh, Vh

    def decode_unit(self, b, h, q_heads, sigma):
        """q_heads: [n][D] query heads that read KV head h; returns [n][D] float64."""
        q = np.ascontiguousarray(q_heads, dtype=np.float32)
        out = np.zeros(q.shape, np.float64)
        u = self.unit(b, h)
        _check(lib().kivi_oracle_decode(ctypes.byref(u), _ptr(q), q.shape[0], float(sigma), _ptr(out)),
               "decode")
        return out

    def decode(self, q, sigma, units=None):
        """q: [B][Hq][D]; query head hq reads KV head hq // (Hq // Hkv).

        Returns out [B][Hq][D] float64 (NaN for heads whose unit is not held)."""
        q = np.asarray(q, np.float32)
        B, Hq, D = q.shape
        gq = Hq // self.Hkv
        out = np.full((B, Hq, D), np.nan)
        for (b, h) in (units if units is not None else self.units):
            out[b, h * gq:(h + 1) * gq] = self.decode_unit(b, h, q[b, h * gq:(h + 1) * gq], sigma)
        return out
