"""Helpers for the GPU-vs-oracle parity tests (not a test module).

Bars (stated once, used by every parity test):
  - codes, scales, zeros and the residual window: bit-exact (compared as
    32-bit words / binary32 bit patterns; fp16 windows and binary16 scales
    and zeros after exact upcast to binary32);
  - decode attention output: max |gpu - oracle| <= 2e-3 and
    mean |gpu - oracle| <= 1e-3, the oracle computed in binary64 from the
    dequantized cache.
"""
from __future__ import annotations

import numpy as np
import torch

import bit_asymmetric_kv_quantize_b200 as kivi
import oracle
from bit_asymmetric_kv_quantize_b200 import workloads as W

MAX_ABS = 2e-3
MEAN_ABS = 1e-3


def gpu_cache(w: W.Workload, capacity=None) -> kivi.KiviCache:
    return kivi.KiviCache(w.B, w.Hkv, w.D, w.bits, capacity or w.capacity, R=w.R, G=w.G,
                          Gv=w.Gv, dtype=w.torch_dtype, device="cuda", meta=w.torch_meta)


def oracle_cache(w: W.Workload, units=None, capacity=None) -> oracle.OracleCache:
    return oracle.OracleCache(w.B, w.Hkv, w.D, w.bits, w.G, w.Gv, w.R, capacity or w.capacity,
                              units=units, meta_f16=w.meta == "f16")


def oracle_prefill(oc: oracle.OracleCache, K: torch.Tensor, V: torch.Tensor):
    """Feed the oracle the very tensors the library got (copied to the host, exact upcast)."""
    for (b, h) in oc.units:
        oc.prefill_unit(b, h, K[b, h].float().cpu().numpy(), V[b, h].float().cpu().numpy())


def oracle_append(oc: oracle.OracleCache, k: torch.Tensor, v: torch.Tensor):
    kh, vh = k.float().cpu().numpy(), v.float().cpu().numpy()
    for (b, h) in oc.units:
        oc.append_unit(b, h, kh[b, h], vh[b, h])


def assert_state_equal(gc: kivi.KiviCache, oc: oracle.OracleCache, units=None):
    """Bit-exact comparison of the quantized store and the window on `units`."""
    units = oc.units if units is None else units
    n_q, r = gc.n_q, gc.r
    E, WB = (32, 3) if gc.bits == 3 else (32 // gc.bits, 1)
    for (b, h) in units:
        u = oc.unit(b, h)
        assert (u.n_q, u.r) == (n_q, r), ((b, h), (u.n_q, u.r), (n_q, r))
    if not units:
        return
    bs = sorted({b for b, _ in units})
    g = {}
    for name in kivi.BUFFER_NAMES:
        t = gc.view(name)[bs]
        g[name] = t.float().cpu().numpy() if t.is_floating_point() else t.cpu().numpy()
    bi = {b: i for i, b in enumerate(bs)}
    lim = {"k_codes": n_q, "k_scale": n_q // 32, "k_zero": n_q // 32, "v_codes": n_q // E * WB, "v_scale": n_q, "v_zero": n_q,
           "k_res": r, "v_res": r}
    for (b, h) in units:
        i = oc.slot(b, h)
        for name in kivi.BUFFER_NAMES:
            n = lim[name]
            got = np.ascontiguousarray(g[name][bi[b], h, :n]).view(np.uint32)
            want = np.ascontiguousarray(getattr(oc, name)[i, :n]).view(np.uint32)
            if not np.array_equal(got, want):
                bad = np.argwhere(got != want)
                raise AssertionError(
                    f"{name} differs at unit {(b, h)}: {len(bad)} words, first at {bad[0].tolist()}: "
                    f"gpu {got[tuple(bad[0])]:#010x} oracle {want[tuple(bad[0])]:#010x}")


def decode_error(gpu_out: torch.Tensor, oc: oracle.OracleCache, q: torch.Tensor, sigma: float,
                 units=None):
    """(max-abs, mean-abs) of the library output against the oracle on `units`."""
    units = oc.units if units is None else units
    qh = q.float().cpu().numpy()
    ref = oc.decode(qh, sigma, units=units)
    got = gpu_out.float().cpu().numpy()
    gq = q.shape[1] // oc.Hkv
    diffs = []
    for (b, h) in units:
        sl = slice(h * gq, (h + 1) * gq)
        diffs.append(np.abs(got[b, sl] - ref[b, sl]).ravel())
    d = np.concatenate(diffs)
    assert np.isfinite(got).all()
    return float(d.max()), float(d.mean())


def assert_decode_close(gpu_out, oc, q, sigma, units=None):
    mx, mean = decode_error(gpu_out, oc, q, sigma, units)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"max {mx:.3e} mean {mean:.3e}"
    return mx, mean


def sample_units(w: W.Workload, n: int, seed: int = 0):
    """n distinct (b, h) units, always including the first and the last."""
    rng = np.random.default_rng(seed)
    total = w.B * w.Hkv
    idx = {0, total - 1}
    while len(idx) < min(n, total):
        idx.add(int(rng.integers(total)))
    return sorted((i // w.Hkv, i % w.Hkv) for i in idx)
