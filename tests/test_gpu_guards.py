"""Guard bands around every buffer the library is given, on the GPU.

Each cache buffer, the workspace, the device counters and the call's inputs
and outputs are carved out of a larger device allocation whose bytes before
and after (4 KiB each side) hold a fixed pattern.  After prefill, appends
across a window flush, decode, the fused and device-counter steps, the
no-allocation decode and the ragged / paged calls, every guard byte must
still hold the pattern (no write outside a buffer), and the results must
still meet the parity bars of kivi_testlib against the oracle.
"""
import ctypes
import math

import pytest
import torch

import bit_asymmetric_kv_quantize_b200 as kivi
from bit_asymmetric_kv_quantize_b200 import workloads as W
from kivi_testlib import (assert_decode_close, assert_state_equal, oracle_append, oracle_cache,
                          oracle_prefill)

pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5


class Guarded:
    """Device bytes with guard bands: `inner` is the buffer handed to the library."""
    all = []

    def __init__(self, nbytes, fill=None):
        n = max(16, (nbytes + 15) // 16 * 16)
        self.raw = torch.full((GUARD + n + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.n = nbytes
        self.inner = self.raw[GUARD:GUARD + nbytes]
        if fill is not None:
            self.inner.fill_(fill)
        Guarded.all.append(self)

    def intact(self):
        lo = self.raw[:GUARD]
        hi = self.raw[GUARD + self.n:]
        return bool((lo == PATTERN).all()) and bool((hi == PATTERN).all())


def guarded_like(t: torch.Tensor) -> torch.Tensor:
    """A copy of t inside a guarded allocation (same dtype and shape)."""
    g = Guarded(t.numel() * t.element_size())
    v = g.inner.view(t.dtype).view(t.shape)
    v.copy_(t)
    return v


def assert_guards():
    torch.cuda.synchronize()
    bad = [i for i, g in enumerate(Guarded.all) if not g.intact()]
    assert not bad, f"guard bands overwritten around buffers {bad}"


def guard_cache(gc, paged=False):
    """Move a fresh cache's buffers into guarded allocations (re-initialising
    the C struct with the new pointers)."""
    bufs = {}
    for n in kivi.BUFFER_NAMES:
        bufs[n] = Guarded(gc.buffers[n].numel()).inner
    ptrs = (ctypes.c_void_p * kivi.NUM_BUFFERS)(*[bufs[n].data_ptr() for n in kivi.BUFFER_NAMES])
    L = kivi.lib()
    if paged:
        rc = L.kivi_paged_cache_init(ctypes.byref(gc._c), ctypes.byref(gc._dims), ctypes.byref(ptrs),
                                     gc.block_table.data_ptr(), gc.pages_per_seq, gc.num_pages)
    else:
        rc = L.kivi_cache_init(ctypes.byref(gc._c), ctypes.byref(gc._dims), ctypes.byref(ptrs))
    assert rc == 0
    gc.buffers = bufs


def guard_workspaces(gc, Hq):
    need = gc.workspace_bytes(Hq)
    gc._ws = Guarded(need).inner
    gc._ws_dev = Guarded(need, fill=0).inner


@pytest.fixture(autouse=True)
def _reset():
    Guarded.all = []
    yield
    Guarded.all = []


@pytest.mark.parametrize("D,bits,dtype,gq", [(128, 2, "f16", 4), (128, 4, "f16", 1),
                                             (64, 1, "f16", 8), (32, 2, "f32", 2)])
def test_uniform_calls_stay_inside_their_buffers(D, bits, dtype, gq):
    R = 32 if dtype == "f32" else 128
    w = W.Workload(f"guard-d{D}-b{bits}-{dtype}-g{gq}", B=3, Hq=2 * gq, Hkv=2, D=D, T=300,
                   bits=bits, R=R, dtype=dtype, seed=11)
    cap = 640
    gc = kivi.KiviCache(w.B, w.Hkv, w.D, w.bits, cap, R=w.R, dtype=w.torch_dtype)
    guard_cache(gc)
    guard_workspaces(gc, w.Hq)
    oc = oracle_cache(w, capacity=cap)
    K, V = W.prompt_kv(w, device="cuda")
    K, V = guarded_like(K), guarded_like(V)
    gc.prefill(K, V)
    oracle_prefill(oc, K, V)
    sigma = 1.0 / math.sqrt(D)
    out = Guarded(w.B * w.Hq * D * (2 if dtype == "f16" else 4)).inner.view(
        w.torch_dtype).view(w.B, w.Hq, D)
    q = guarded_like(W.query(w, device="cuda"))
    gc.decode(q, sigma, out=out)
    assert_decode_close(out, oc, q, sigma)
    assert_guards()
    for step in range(R + 3):  # crosses a window flush
        k, v = W.step_kv(w, step, device="cuda")
        k, v = guarded_like(k), guarded_like(v)
        if step % 2:
            gc.append(k, v)
        else:
            q = guarded_like(W.query(w, step, device="cuda"))
            gc.append_decode(k, v, q, sigma, out=out)
        oracle_append(oc, k, v)
        if step % 2 == 0 and step % 8 == 0:
            assert_decode_close(out, oc, q, sigma)
    assert_state_equal(gc, oc)
    assert_guards()
    # device-counter steps (across another flush)
    st = guarded_like(gc.dev_state())
    for step in range(R + 2):
        k, v = W.step_kv(w, 1000 + step, device="cuda")
        k, v = guarded_like(k), guarded_like(v)
        q = guarded_like(W.query(w, 1000 + step, device="cuda"))
        gc.append_decode_dev(st, k, v, q, sigma, out=out)
        oracle_append(oc, k, v)
    assert_decode_close(out, oc, q, sigma)
    gc.load_dev_state(st)
    assert_state_equal(gc, oc)
    assert_guards()
    # the no-allocation decode writes only `out`
    L = kivi.lib()
    rc = L.kivi_decode_attention_noalloc(ctypes.byref(gc._c), q.data_ptr(), w.Hq, sigma,
                                         out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    assert_decode_close(out, oc, q, sigma)
    assert_guards()
    # the host-buffer step writes only its staging (and the cache)
    L.kivi_host_step_bytes.argtypes = [ctypes.POINTER(kivi.KiviCacheC), ctypes.c_int]
    L.kivi_host_step_bytes.restype = ctypes.c_size_t
    gc._staging = Guarded(int(L.kivi_host_step_bytes(ctypes.byref(gc._c), w.Hq))).inner
    hout = torch.empty(w.B, w.Hq, D, dtype=w.torch_dtype).pin_memory()
    for step in range(4):
        k, v = W.step_kv(w, 2000 + step, device="cuda")
        q = W.query(w, 2000 + step, device="cuda")
        kvq = torch.cat([k.flatten(), v.flatten(), q.flatten()]).cpu().pin_memory()
        gc.append_decode_host(kvq, w.Hq, sigma, hout)
        oracle_append(oc, k, v)
    torch.cuda.synchronize()
    assert_decode_close(hout.cuda(), oc, q, sigma)
    assert_guards()


@pytest.mark.parametrize("paged", [False, True])
def test_ragged_and_paged_calls_stay_inside_their_buffers(paged):
    w = W.Workload("guard-ragged", B=4, Hq=8, Hkv=2, D=128, T=300, bits=2, R=128, len_min=1, seed=12)
    lens = torch.tensor([300, 1, 129, 256], dtype=torch.int64)
    pps = 3
    if paged:
        bt = guarded_like(torch.tensor([[4, 0, 2], [1, 9, 3], [5, 6, 7], [8, 10, 11]],
                                       dtype=torch.int32, device="cuda"))
        gc = kivi.PagedKiviCache(w.B, w.Hkv, w.D, w.bits, pps, 12, bt, R=w.R, dtype=w.torch_dtype)
    else:
        gc = kivi.KiviCache(w.B, w.Hkv, w.D, w.bits, (pps + 1) * w.R, R=w.R, dtype=w.torch_dtype)
    guard_cache(gc, paged=paged)
    guard_workspaces(gc, w.Hq)
    oc = oracle_cache(w, capacity=(pps + 1) * w.R)
    K, V = W.prompt_kv(w, device="cuda")
    K, V = guarded_like(K), guarded_like(V)
    st0 = gc.ragged_prefill(K, V, guarded_like(lens.cuda()))
    st = guarded_like(st0)
    for (b, h) in oc.units:
        n = int(lens[b])
        oc.prefill_unit(b, h, K[b, h, :n].float().cpu().numpy(), V[b, h, :n].float().cpu().numpy())
    out = Guarded(w.B * w.Hq * w.D * 2).inner.view(torch.float16).view(w.B, w.Hq, w.D)
    sigma = 1.0 / math.sqrt(w.D)
    for step in range(130):  # every sequence crosses a flush of its own
        k, v = W.step_kv(w, step, device="cuda")
        k, v = guarded_like(k), guarded_like(v)
        q = guarded_like(W.query(w, step, device="cuda"))
        gc.ragged_append_decode(st, k, v, q, sigma, out=out)
        oracle_append(oc, k, v)
    assert_decode_close(out, oc, q, sigma)
    assert_guards()
