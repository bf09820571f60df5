"""GPU parity of the dense-and-sparse variant against the oracle, through the
C ABI (KVQuant, codewithpapers.app page, abstract item (iv): outliers
isolated per vector so that they do not skew its quantization range).

Every key group (channel over 32 tokens) keeps its k_out largest
magnitudes exactly and every value group (token over 32 channels) its v_out
largest, listed (index, value) in index order with dense code 0.  Bars
(kivi_testlib): codes, scales, zeros, window and the four lists bit-exact;
decode within 2e-3 max-abs and 1e-3 mean-abs of the oracle's binary64
attention over its reconstruction (kept entries exact).  Inputs: the
standard synthetic K/V with a fraction of single entries scaled x8 (fp32
caches) or x4 (fp16 caches, whose output rounding must stay below the bar).
"""
import math

import numpy as np
import pytest
import torch

import bit_asymmetric_kv_quantize_b200 as kivi
import oracle
from bit_asymmetric_kv_quantize_b200 import workloads as W
from kivi_testlib import (assert_decode_close, assert_state_equal, oracle_append, oracle_prefill,
                          sample_units)

pytestmark = pytest.mark.gpu


def small(D=64, bits=2, dtype="f16", R=32, T=200, B=2, Hkv=2, gq=1, seed=51, spikes=0.03):
    # spikes on top of the x20 key channels: x8 with fp32 caches, x4 with fp16
    # ones, whose fp16 output alone rounds by more than the 2e-3 bar once
    # |out| > 4 (an output dominated by one spiked value)
    scale = 8.0 if dtype == "f32" else 4.0
    return W.Workload(f"sp-d{D}-b{bits}-{dtype}-g{gq}-t{T}", B=B, Hq=Hkv * gq, Hkv=Hkv, D=D, T=T,
                      bits=bits, R=R, dtype=dtype, seed=seed, spike_frac=spikes, spike_scale=scale)


def caches(w, outliers, capacity, units=None):
    gc = kivi.KiviCache(w.B, w.Hkv, w.D, w.bits, capacity, R=w.R, dtype=w.torch_dtype,
                        outliers=outliers)
    oc = oracle.OracleCache(w.B, w.Hkv, w.D, w.bits, w.G, w.Gv, w.R, capacity, units=units,
                            outliers=outliers)
    return gc, oc


def assert_lists_equal(gc, oc, units=None):
    """The four outlier lists, bit for bit, over the filled key groups and tokens."""
    ko, vo = gc.outliers
    n_q = gc.n_q
    units = oc.units if units is None else units
    for (b, h) in units:
        i = oc.slot(b, h)
        if ko:
            for name in ("k_out_idx", "k_out_val"):
                got = gc.view(name)[b, h, :n_q // 32].cpu().numpy().view(np.uint32)
                want = getattr(oc, name)[i, :n_q // 32].view(np.uint32)
                assert np.array_equal(got, want), (name, (b, h))
        if vo:
            for name in ("v_out_idx", "v_out_val"):
                got = gc.view(name)[b, h, :n_q].cpu().numpy().view(np.uint32)
                want = getattr(oc, name)[i, :n_q].view(np.uint32)
                assert np.array_equal(got, want), (name, (b, h))


OUTLIERS = [(1, 0), (0, 2), (2, 1), (4, 4)]


@pytest.mark.parametrize("outliers", OUTLIERS)
@pytest.mark.parametrize("dtype", ["f16", "f32"])
@pytest.mark.parametrize("bits", [1, 2, 4])
@pytest.mark.parametrize("D", [32, 64, 128])
def test_prefill_bit_exact(D, bits, dtype, outliers):
    w = small(D=D, bits=bits, dtype=dtype, T=300)
    K, V = W.prompt_kv(w, device="cuda")
    gc, oc = caches(w, outliers, 512)
    gc.prefill(K, V)
    oracle_prefill(oc, K, V)
    torch.cuda.synchronize()
    assert_state_equal(gc, oc)
    assert_lists_equal(gc, oc)


@pytest.mark.parametrize("dtype", ["f16", "f32"])
@pytest.mark.parametrize("outliers", OUTLIERS)
@pytest.mark.parametrize("gq", [1, 2, 4, 8])
@pytest.mark.parametrize("bits", [1, 2, 4])
def test_decode_and_steps(bits, gq, outliers, dtype):
    """Prefill, decode, then fused steps (one launch each) across a window
    flush that the decode kernel quantizes itself; the store and the lists
    stay bit-exact and every checked decode is within the bars."""
    w = small(D=128, bits=bits, gq=gq, T=150, R=32, dtype=dtype)
    K, V = W.prompt_kv(w, device="cuda")
    gc, oc = caches(w, outliers, 512)
    gc.prefill(K, V)
    oracle_prefill(oc, K, V)
    sigma = 1.0 / math.sqrt(w.D)
    q = W.query(w, device="cuda")
    assert_decode_close(gc.decode(q, sigma), oc, q, sigma)
    for step in range(40):
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        out = gc.append_decode(k, v, q, sigma)
        oracle_append(oc, k, v)
        if step % 9 == 0:
            assert_decode_close(out, oc, q, sigma)
    torch.cuda.synchronize()
    assert_state_equal(gc, oc)
    assert_lists_equal(gc, oc)


@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_device_counter_steps(dtype):
    w = small(D=64, bits=2, dtype=dtype, gq=4, T=90, R=32)
    K, V = W.prompt_kv(w, device="cuda")
    gc, oc = caches(w, (2, 2), 256)
    gc.prefill(K, V)
    oracle_prefill(oc, K, V)
    st = gc.dev_state()
    for step in range(40):  # flushes at steps 6 and 38
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        out = gc.append_decode_dev(st, k, v, q, 1.0)
        oracle_append(oc, k, v)
    assert_decode_close(out, oc, q, 1.0)
    gc.load_dev_state(st)
    assert_state_equal(gc, oc)
    assert_lists_equal(gc, oc)


def test_ragged_batch():
    w = small(D=128, bits=2, gq=2, T=300, B=4, Hkv=2, R=64)
    w = w.with_(len_min=1)
    lens = torch.tensor([300, 1, 129, 200], dtype=torch.int64)
    K, V = W.prompt_kv(w, device="cuda")
    gc, oc = caches(w, (1, 1), 384)
    st = gc.ragged_prefill(K, V, lens.cuda())
    for (b, h) in oc.units:
        n = int(lens[b])
        oc.prefill_unit(b, h, K[b, h, :n].float().cpu().numpy(), V[b, h, :n].float().cpu().numpy())
    sigma = 0.2
    for step in range(70):
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        out = gc.ragged_append_decode(st, k, v, q, sigma)
        oracle_append(oc, k, v)
    assert_decode_close(out, oc, q, sigma)


def test_layer_sized_cache_sampled():
    """A Llama-2-7B-shaped layer (B 8, 32 heads, context 4096) with one key
    and one value entry kept per group, on sampled units."""
    w = W.LLAMA2_7B.with_(name="sp-7b", spike_frac=0.01, spike_scale=4.0)
    K, V = W.prompt_kv(w, device="cuda")
    units = sample_units(w, 6, seed=3)
    gc, oc = caches(w, (1, 1), w.capacity + 128, units=units)
    gc.prefill(K, V)
    oracle_prefill(oc, K, V)
    q = W.query(w, device="cuda")
    out = gc.decode(q, 1.0)
    assert_decode_close(out, oc, q, 1.0, units)
    assert_state_equal(gc, oc, units)
    assert_lists_equal(gc, oc, units)


def test_refusals():
    w = small()
    L = kivi.lib()
    # the CUDA-core decode takes plain codes only
    gc, _ = caches(w, (1, 1), 256)
    K, V = W.prompt_kv(w, device="cuda")
    gc.prefill(K, V)
    q = W.query(w, device="cuda")
    with pytest.raises(kivi.KiviError):
        gc.decode(q, 1.0, kernel="simt")
    with pytest.raises(kivi.KiviError):  # binary16 metadata
        kivi.KiviCache(2, 2, 64, 2, 256, R=32, meta=torch.float16, outliers=(1, 0))
    with pytest.raises(kivi.KiviError):  # more than four kept entries per group
        kivi.KiviCache(2, 2, 64, 2, 256, R=32, outliers=(5, 0))
