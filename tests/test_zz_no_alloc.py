"""kivi_decode_attention_noalloc: decode attention without a caller workspace.

Some callers cannot allocate device memory once they are running (a plugin
inside an engine that has reserved the whole device for its own pool, or a
latency-bound loop that must not call cudaMalloc because it can synchronize
the device).  This entry point writes its cross-split partials to a fixed
4 MiB static device array instead of a caller workspace.  The test calls it
through the C ABI twice in a row and checks each result against the regular
entry point (kivi_decode_attention with a workspace), within the decode
tolerance the parity tests use, and against the CPU oracle on sampled units.
Large batches make the scratch hold fewer split partials than a workspace
would (down to one per unit), which the last cases exercise.  The file name
makes pytest collect it last.
"""
import ctypes
import math

import pytest
import torch

import bit_asymmetric_kv_quantize_b200 as kivi
from bit_asymmetric_kv_quantize_b200 import workloads as W
from kivi_testlib import (MAX_ABS, MEAN_ABS, assert_decode_close, oracle_append, oracle_cache,
                          oracle_prefill, sample_units)

pytestmark = pytest.mark.gpu
SCRATCH_BYTES = 4 << 20  # KIVI_NOALLOC_SCRATCH_BYTES (include/kivi.h)


def _noalloc(gc, q, sigma, out):
    L = kivi.lib()
    return L.kivi_decode_attention_noalloc(ctypes.byref(gc._c), q.data_ptr(), q.shape[1],
                                           float(sigma), out.data_ptr(),
                                           torch.cuda.current_stream().cuda_stream)


def _close(a, b):
    d = (a.float() - b.float()).abs()
    return float(d.max()) <= MAX_ABS and float(d.mean()) <= MEAN_ABS


# (B, Hkv, gq, T): small batches (the scratch holds as many split partials as
# a workspace), the Llama-2-13B-shaped batch at a short context (room for 3
# splits), and B * Hq = 6144 query heads, where one split per unit is all
# that fits: every unit is then one CTA's range.
CASES = [(4, 8, 1, 4096), (4, 8, 4, 3000), (64, 40, 1, 300), (128, 48, 1, 300)]


@pytest.mark.parametrize("B,Hkv,gq,T", CASES)
def test_noalloc_matches_workspace_decode_twice(B, Hkv, gq, T):
    w = W.Workload(f"noalloc-b{B}h{Hkv}-g{gq}-t{T}", B=B, Hq=Hkv * gq, Hkv=Hkv, D=128, T=T, bits=2,
                   R=128)
    per_split = B * w.Hq * (w.D + 2) * 4
    K, V = W.prompt_kv(w, device="cuda")
    gc = kivi.KiviCache(w.B, w.Hkv, w.D, w.bits, w.capacity + 128, R=w.R, dtype=w.torch_dtype)
    gc.prefill(K, V)
    units = sample_units(w, 24, seed=B)
    oc = oracle_cache(w, units=units, capacity=w.capacity + 128)
    oracle_prefill(oc, K, V)
    sigma = 1.0 / math.sqrt(w.D)
    for call in range(2):  # two calls in a row; the second reuses the shared scratch
        q = W.query(w, step=call, device="cuda")
        ref = gc.decode(q, sigma)
        out = torch.full_like(q, float("nan"))
        assert _noalloc(gc, q, sigma, out) == 0
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        assert _close(out, ref), f"call {call}: noalloc result differs from the workspace call"
        assert_decode_close(out, oc, q, sigma)
        k, v = W.step_kv(w, call, device="cuda")
        gc.append(k, v)
        oracle_append(oc, k, v)
    if per_split * 2 > SCRATCH_BYTES:
        assert B * Hkv * gq > 4096  # the case meant to leave room for one split only


def test_noalloc_rejects_requests_beyond_its_scratch():
    # B * Hq * (D + 2) * 4 bytes for one split exceeds 4 MiB: refused before any launch
    w = W.Workload("noalloc-too-big", B=512, Hq=32, Hkv=4, D=128, T=40, bits=2, R=128)
    gc = kivi.KiviCache(w.B, w.Hkv, w.D, w.bits, 128, R=w.R, dtype=w.torch_dtype)
    K, V = W.prompt_kv(w, device="cuda")
    gc.prefill(K, V)
    q = W.query(w, device="cuda")
    out = torch.empty_like(q)
    assert _noalloc(gc, q, 1.0, out) == 7  # KIVI_ERR_SCRATCH_LIMIT
