"""GPU parity of the format variant with binary16 scales and zeros
(KIVI_META_F16, fp16 caches) against the oracle run with meta_f16: codes,
scales, zeros and the window bit for bit, decode attention within the bars of
kivi_testlib, through the C ABI.

Reading (the pages name an asymmetric scale and offset per group but fix no
storage precision for them): the binary32 scale and minimum are rounded to
binary16 and the codes are chosen against the rounded pair.  KIVI, study.space
summary: asymmetric per-group quantizer.
"""
import math

import pytest
import torch

from bit_asymmetric_kv_quantize_b200 import workloads as W
from kivi_testlib import (assert_decode_close, assert_state_equal, gpu_cache, oracle_append,
                          oracle_cache, oracle_prefill, sample_units)

pytestmark = pytest.mark.gpu
KERNELS = ["default", "simt"]


def small(D=64, bits=2, R=32, T=200, B=2, Hkv=2, gq=1, seed=21):
    return W.Workload(f"m16-d{D}-b{bits}-g{gq}-t{T}", B=B, Hq=Hkv * gq, Hkv=Hkv, D=D, T=T,
                      bits=bits, R=R, dtype="f16", meta="f16", seed=seed)


def test_metadata_buffers_are_binary16():
    w = small()
    gc = gpu_cache(w, capacity=256)
    for name in ("k_scale", "k_zero", "v_scale", "v_zero"):
        assert gc.view(name).dtype == torch.float16
    with pytest.raises(Exception):
        gpu_cache(w.with_(dtype="f32"), capacity=256)  # binary16 metadata needs an fp16 cache


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("T", [1, 64, 65, 129, 333])
def test_prefill_bit_exact(D, bits, T):
    w = small(D=D, bits=bits, R=64, T=T, Hkv=3)
    K, V = W.prompt_kv(w, device="cuda")
    gc = gpu_cache(w, capacity=512)
    gc.prefill(K, V)
    oc = oracle_cache(w, capacity=512)
    oracle_prefill(oc, K, V)
    assert_state_equal(gc, oc)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_append_and_flush_bit_exact(bits):
    R = 32
    w = small(D=128, bits=bits, R=R, T=R + 5)
    K, V = W.prompt_kv(w, device="cuda")
    gc = gpu_cache(w, capacity=R * 8)
    oc = oracle_cache(w, capacity=R * 8)
    gc.prefill(K, V)
    oracle_prefill(oc, K, V)
    for step in range(3 * R):
        k, v = W.step_kv(w, step, device="cuda")
        gc.append(k, v)
        oracle_append(oc, k, v)
        if gc.r in (1, R):
            assert_state_equal(gc, oc)
    assert_state_equal(gc, oc)


def test_rounding_edge_cases_bit_exact():
    """Scales that round to zero (codes all 0), to a binary16 subnormal, up
    near the top of the range, and down far enough that the top code clamps;
    signed zero minima."""
    w = small(D=64, bits=2, R=32, T=32 * 4 + 3, B=1, Hkv=2)
    K, V = W.prompt_kv(w, device="cuda")
    tiny = 2.0 ** -24
    # range 2^-24: s = 2^-24 / 3 rounds to 0 in binary16 -> every code 0
    K[0, 0, 0:32, 0] = 0.0
    K[0, 0, 5, 0] = tiny
    # range 2^-23: s = 2^-23 / 3 rounds to the subnormal 2^-24
    K[0, 0, 0:32, 1] = 0.0
    K[0, 0, 7, 1] = 2 * tiny
    # the full fp16 range: s = 131008 / 3 = 43669.33 -> 43680 (rounded up)
    K[0, 1, 32:48, 2] = -65504.0
    K[0, 1, 48:64, 2] = 65504.0
    # range 4 * 2^-24: s = (4/3) 2^-24 rounds down to 2^-24, so the largest
    # element's quotient is 4, above the top code: clamped to 3
    V[0, 0, 3, 0:32] = 0.0
    V[0, 0, 3, 31] = 4 * tiny
    # a normal scale that binary16 cannot hold: (1 + 2^-10) / 3
    V[0, 0, 4, 0:32] = torch.linspace(0, 1, 32, device="cuda").half()
    V[0, 0, 4, 31] = 1.0009765625
    # signed zero minima
    V[0, 1, 4, 0:32] = -0.0
    V[0, 1, 5, 32:48] = -0.0
    V[0, 1, 5, 48:64] = 0.0
    gc = gpu_cache(w, capacity=256)
    gc.prefill(K, V)
    oc = oracle_cache(w, capacity=256)
    oracle_prefill(oc, K, V)
    assert_state_equal(gc, oc)
    ks = gc.view("k_scale")
    assert float(ks[0, 0, 0, 0]) == 0.0 and int(gc.view("k_codes")[0, 0, 5, 0]) & 3 == 0
    assert float(ks[0, 0, 0, 1]) == tiny
    assert float(gc.view("v_scale")[0, 0, 3, 0]) == tiny
    assert (int(gc.view("v_codes")[0, 0, 0, 31]) >> 6) & 3 == 3  # token 3, channel 31


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("gq", [1, 2, 4, 8])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("D", [32, 64, 128])
def test_decode_shapes(D, bits, gq, kernel):
    if bits == 3 and kernel == "simt":
        pytest.skip("3-bit codes: tensor-core decode only")
    for T in (1, 33, 161, 1000):
        w = small(D=D, bits=bits, gq=gq, T=T)
        K, V = W.prompt_kv(w, device="cuda")
        gc = gpu_cache(w, capacity=1024)
        gc.prefill(K, V)
        oc = oracle_cache(w, capacity=1024)
        oracle_prefill(oc, K, V)
        q = W.query(w, device="cuda")
        sigma = 1.0 / math.sqrt(w.D)
        assert_decode_close(gc.decode(q, sigma, kernel=kernel), oc, q, sigma)


@pytest.mark.parametrize("gq", [1, 4])
def test_fused_and_device_counter_steps(gq):
    """The fused append + decode and the device-counter step over 100 steps
    (three flushes at R = 32) agree bit for bit with separate calls, and the
    cache matches the oracle."""
    w = small(D=128, bits=2, gq=gq, T=70, R=32, seed=22)
    K, V = W.prompt_kv(w, device="cuda")
    fused, dev, ref = (gpu_cache(w, capacity=256) for _ in range(3))
    for c in (fused, dev, ref):
        c.prefill(K, V)
    oc = oracle_cache(w, capacity=256)
    oracle_prefill(oc, K, V)
    st = dev.dev_state()
    for step in range(100):
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        out_f = fused.append_decode(k, v, q, 1.0)
        out_d = dev.append_decode_dev(st, k, v, q, 1.0)
        ref.append(k, v)
        out_r = ref.decode(q, 1.0)
        oracle_append(oc, k, v)
        assert torch.equal(out_f, out_r) and torch.equal(out_d, out_r), f"step {step}"
        if step % 20 == 0 or ref.r == 1:
            assert_decode_close(out_r, oc, q, 1.0)
    assert_state_equal(fused, oc)


@pytest.mark.parametrize("w", [W.LLAMA2_7B, W.LLAMA2_13B_4BIT], ids=lambda w: w.name)
def test_layer_workloads_sampled(w):
    """Full-size layers with binary16 metadata: the sampled units' store bit
    for bit and their decode within the bars, both kernels."""
    w = w.with_(meta="f16")
    K, V = W.prompt_kv(w, device="cuda")
    gc = gpu_cache(w)
    gc.prefill(K, V)
    units = sample_units(w, 8, seed=3)
    oc = oracle_cache(w, units=units)
    oracle_prefill(oc, K, V)
    del K, V
    assert_state_equal(gc, oc)
    q = W.query(w, device="cuda")
    for kernel in KERNELS:
        assert_decode_close(gc.decode(q, 1.0, kernel=kernel), oc, q, 1.0, units=units)
