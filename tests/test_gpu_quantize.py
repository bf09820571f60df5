"""GPU parity of the prefill / append / flush path against the oracle: the
quantized store (codes, scales, zeros) and the residual window are compared
bit for bit, through the C ABI (libkivi.so via the ctypes binding).

Method: "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache"
(mlsanity.com index page, "Abstract (arXiv)": per-channel keys, per-token
values; study.space summary: asymmetric groups, quantized and residual
parts, codes appended along tokens).
"""
import numpy as np
import pytest
import torch

import bit_asymmetric_kv_quantize_b200 as kivi
from bit_asymmetric_kv_quantize_b200 import workloads as W
from kivi_testlib import (assert_state_equal, gpu_cache, oracle_append, oracle_cache,
                          oracle_prefill, sample_units)

pytestmark = pytest.mark.gpu


def small(D=64, bits=2, dtype="f16", R=64, T=200, B=2, Hkv=3, gq=1, capacity=512, seed=1):
    return W.Workload(f"small-d{D}-b{bits}-{dtype}-r{R}-t{T}", B=B, Hq=Hkv * gq, Hkv=Hkv, D=D,
                      T=T, bits=bits, R=R, dtype=dtype, seed=seed).with_()


@pytest.mark.parametrize("dtype", ["f16", "f32"])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("T", [1, 31, 64, 65, 127, 128, 129, 333])
def test_prefill_bit_exact(D, bits, dtype, T):
    w = small(D=D, bits=bits, dtype=dtype, T=T)
    K, V = W.prompt_kv(w, device="cuda")
    gc = gpu_cache(w, capacity=512)
    gc.prefill(K, V)
    oc = oracle_cache(w, capacity=512)
    oracle_prefill(oc, K, V)
    assert (gc.n_q, gc.r) == (T - ((T - 1) % 64 + 1), (T - 1) % 64 + 1)
    assert_state_equal(gc, oc)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("R", [32, 128])
def test_append_and_flush_bit_exact(bits, R):
    """Prefill, then appends across several window flushes; the state matches
    the oracle after every append."""
    w = small(D=128, bits=bits, R=R, T=R + 5, B=2, Hkv=2)
    K, V = W.prompt_kv(w, device="cuda")
    cap = R * 8
    gc = gpu_cache(w, capacity=cap)
    oc = oracle_cache(w, capacity=cap)
    gc.prefill(K, V)
    oracle_prefill(oc, K, V)
    assert_state_equal(gc, oc)
    for step in range(3 * R):
        k, v = W.step_kv(w, step, device="cuda")
        gc.append(k, v)
        oracle_append(oc, k, v)
        if gc.r in (1, R) or step % 17 == 0:
            assert_state_equal(gc, oc)
    assert_state_equal(gc, oc)
    assert gc.n_q + gc.r == R + 5 + 3 * R


@pytest.mark.parametrize("T", [0, 1, 32, 63, 64, 65, 129, 300])
def test_prefill_equals_appends(T):
    """prefill(T) and T single appends write identical bytes."""
    w = small(D=64, bits=2, R=64, T=T, dtype="f16")
    K, V = W.prompt_kv(w, device="cuda")
    a, b = gpu_cache(w, capacity=512), gpu_cache(w, capacity=512)
    a.prefill(K, V)
    for t in range(T):
        b.append(K[:, :, t].contiguous(), V[:, :, t].contiguous())
    assert (a.n_q, a.r) == (b.n_q, b.r)
    n_q, r = a.n_q, a.r
    lim = {"k_codes": n_q, "k_scale": n_q // 32, "k_zero": n_q // 32, "v_codes": n_q // 16,
           "v_scale": n_q, "v_zero": n_q, "k_res": r, "v_res": r}
    for name in kivi.BUFFER_NAMES:
        assert torch.equal(a.view(name)[:, :, :lim[name]], b.view(name)[:, :, :lim[name]]), name


@pytest.mark.parametrize("misaligned", [False, True], ids=["aligned", "misaligned"])
@pytest.mark.parametrize("dtype", ["f16", "f32"])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_prefill_paths_bit_exact(bits, dtype, misaligned):
    """The prefill's staged path (16-byte aligned K and V) and its general path
    (K and V one element past an aligned address) both match the oracle."""
    w = small(D=128, bits=bits, dtype=dtype, R=64, T=32 * 9 + 7, B=2, Hkv=2, seed=3)
    K, V = W.prompt_kv(w, device="cuda")
    if misaligned:
        def shift(x):
            buf = torch.empty(x.numel() + 1, dtype=x.dtype, device=x.device)
            y = buf[1:].view(x.shape)
            y.copy_(x)
            assert y.data_ptr() % 16 != 0
            return y
        K, V = shift(K), shift(V)
    gc = gpu_cache(w, capacity=512)
    gc.prefill(K, V)
    oc = oracle_cache(w, capacity=512)
    oracle_prefill(oc, K, V)
    assert_state_equal(gc, oc)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_special_values_bit_exact(D, dtype):
    """Signed zeros (first occurrence decides the zero's sign), constant groups
    (scale 0), fp16 extremes and subnormals, huge outlier channels."""
    w = small(D=D, bits=2, R=32, T=32 * 6 + 3, B=1, Hkv=2, dtype=dtype)
    K, V = W.prompt_kv(w, device="cuda")
    K[0, 0, 0:32, 0] = 0.0                       # constant channel group
    K[0, 0, 0:32, 1] = -0.0
    K[0, 0, 0:16, 2] = -0.0                      # -0 first, then +0
    K[0, 0, 16:32, 2] = 0.0
    K[0, 0, 32:48, 3] = 0.0                      # +0 first, then -0
    K[0, 0, 48:64, 3] = -0.0
    K[0, 1, 64:96, 5] = 65504.0                  # fp16 max, constant
    K[0, 1, 64:80, 6] = -65504.0                 # full fp16 range in one group
    K[0, 1, 80:96, 6] = 65504.0
    K[0, 1, 96:128, 7] = torch.arange(32, device="cuda", dtype=torch.float16) * 6e-8  # subnormals
    V[0, 0, 3, :32] = -0.0                       # constant value group (-0)
    V[0, 0, 4, :32] = 1.5
    V[0, 1, 5, 0:16] = 0.0
    V[0, 1, 5, 16:32] = -0.0
    V[0, 1, 6, 32:64] = torch.arange(32, device="cuda", dtype=torch.float16) * 1e3
    V[0, 0, 7, 0:32] = torch.arange(32, device="cuda", dtype=V.dtype)  # min +0, then -0
    V[0, 0, 7, 9] = -0.0
    V[0, 0, 8, 0:32] = torch.arange(32, device="cuda", dtype=V.dtype)  # min -0 first
    V[0, 0, 8, 0] = -0.0
    V[0, 0, 8, 17] = 0.0
    V[0, 1, 9, 0:32] = -torch.arange(32, device="cuda", dtype=V.dtype) - 1  # max -0 first
    V[0, 1, 9, 30] = -0.0
    V[0, 1, 9, 31] = 0.0
    K[0, 1, 128:160, 9] = -torch.arange(32, device="cuda", dtype=K.dtype) - 1  # max +0 first
    K[0, 1, 140, 9] = 0.0
    K[0, 1, 150, 9] = -0.0
    K[0, 0, 128:160, 10] = torch.arange(32, device="cuda", dtype=K.dtype)  # min -0 late
    K[0, 0, 128, 10] = 1.0
    K[0, 0, 159, 10] = -0.0
    if dtype == "f32":
        # subnormal ranges: the scale's reciprocal overflows, the exact division decides
        tiny = torch.arange(32, device="cuda", dtype=torch.float64) * 2.0 ** -149
        K[0, 0, 32:64, 20] = tiny.float()
        K[0, 1, 96:128, 21] = (tiny * 3).float()
        V[0, 0, 10, 0:32] = tiny.float()
        V[0, 1, 11, 32:64] = (tiny * 5).float()
    gc = gpu_cache(w, capacity=512)
    gc.prefill(K, V)
    oc = oracle_cache(w, capacity=512)
    oracle_prefill(oc, K, V)
    assert_state_equal(gc, oc)


def test_tiny_workload_full():
    w = W.TINY
    K, V = W.prompt_kv(w, device="cuda")
    gc = gpu_cache(w)
    gc.prefill(K, V)
    oc = oracle_cache(w)
    oracle_prefill(oc, K, V)
    assert (gc.n_q, gc.r) == (224, 32)
    assert_state_equal(gc, oc)


@pytest.mark.parametrize("w", [W.LLAMA2_7B, W.MISTRAL_7B], ids=lambda w: w.name)
def test_layer_workloads_full(w):
    K, V = W.prompt_kv(w, device="cuda")
    gc = gpu_cache(w)
    gc.prefill(K, V)
    oc = oracle_cache(w)
    oracle_prefill(oc, K, V)
    assert (gc.n_q, gc.r) == (w.T - w.R, w.R)
    assert_state_equal(gc, oc)


@pytest.mark.parametrize("w", [W.LLAMA2_13B_2BIT, W.LLAMA2_13B_4BIT], ids=lambda w: w.name)
def test_large_batch_workload_sampled(w):
    """Full-size 13B-shaped layer (64 x 40 units, 8192 tokens): every unit is
    quantized on the GPU, 24 sampled units are checked against the oracle."""
    K, V = W.prompt_kv(w, device="cuda")
    gc = gpu_cache(w)
    gc.prefill(K, V)
    units = sample_units(w, 24)
    oc = oracle_cache(w, units=units)
    oracle_prefill(oc, K, V)
    assert_state_equal(gc, oc)


def test_large_batch_every_unit():
    """Full-size 13B-shaped layer at 2 bits: the store of all 2560 units
    against the oracle (fed per sequence from one host copy of the prompt),
    and decode on 256 sampled units."""
    w = W.LLAMA2_13B_2BIT
    K, V = W.prompt_kv(w, device="cuda")
    gc = gpu_cache(w)
    gc.prefill(K, V)
    q = W.query(w, device="cuda")
    out = gc.decode(q, 1.0)
    torch.cuda.synchronize()
    oc = oracle_cache(w)
    for b in range(w.B):  # one sequence's heads at a time
        kb, vb = K[b].float().cpu().numpy(), V[b].float().cpu().numpy()
        for h in range(w.Hkv):
            oc.prefill_unit(b, h, kb[h], vb[h])
    del K, V
    assert_state_equal(gc, oc)
    from kivi_testlib import assert_decode_close
    assert_decode_close(out, oc, q, 1.0, units=sample_units(w, 256, seed=11))


@pytest.mark.parametrize("D", [32, 128])
@pytest.mark.parametrize("dtype", ["f16", "f32"])
@pytest.mark.parametrize("bits", [2, 4])
def test_half_integer_quotients_bit_exact(bits, dtype, D):
    """Groups whose quotients (x - min) / s land exactly on half-integers
    (power-of-two scales: ties, rounded to even) or, for binary32 inputs,
    one ulp either side of them: the quantizers' rounding check hands these
    to the exact division, in the prompt quantizer and in the flush."""
    L = (1 << bits) - 1
    w = small(D=D, bits=bits, dtype=dtype, R=32, T=32 * 5 + 9, B=1, Hkv=2, seed=7)
    K, V = W.prompt_kv(w, device="cuda")
    tdt = K.dtype
    half = torch.arange(32, device="cuda", dtype=torch.float64) % L + 0.5  # k + 1/2
    base = torch.zeros(32, device="cuda", dtype=torch.float64)
    base[0], base[1] = 0.0, float(L)  # min 0, max L: s = 1
    for g, scale in enumerate((1.0, 0.25, 4.0)):  # key groups 0..2 of unit (0, 0), channels 0..7
        col = base.clone()
        col[2:] = half[2:]
        for ch in range(8):
            K[0, 0, 32 * g:32 * g + 32, ch] = (col * scale).to(tdt)
    for t in range(20):  # value groups of tokens 0..19 of unit (0, 1), channel group 0
        row = base.clone()
        row[2:] = half[2:]
        V[0, 1, t, 0:32] = (row * 2.0 ** (t % 5 - 2)).to(tdt)
    if dtype == "f32":
        # one ulp above and below each half-integer quotient (s = 1)
        col = base.clone()
        col[2:] = half[2:]
        c32 = col.float()
        upv, dnv = c32.clone(), c32.clone()
        upv[2:] = torch.nextafter(c32[2:], torch.full_like(c32[2:], float("inf")))
        dnv[2:] = torch.nextafter(c32[2:], torch.zeros_like(c32[2:]))
        for ch in range(4):
            K[0, 1, 0:32, ch] = upv
            K[0, 1, 0:32, ch + 4] = dnv
        V[0, 0, 3, 0:32] = upv
        V[0, 0, 4, 0:32] = dnv
    gc = gpu_cache(w, capacity=512)
    gc.prefill(K, V)
    oc = oracle_cache(w, capacity=512)
    oracle_prefill(oc, K, V)
    assert_state_equal(gc, oc)
    # the window's tiles go through the flush with the same values
    for step in range(40):
        k = K[:, :, step % 32].contiguous()
        v = V[:, :, step % 20].contiguous()
        gc.append(k, v)
        oracle_append(oc, k, v)
    assert_state_equal(gc, oc)
