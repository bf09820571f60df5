"""GPU parity of decode attention against the oracle, through the C ABI.

Bar: max |gpu - oracle| <= 2e-3 and mean <= 1e-3 (kivi_testlib), the oracle
in binary64 over the dequantized cache.  Both the tensor-core kernel
(kivi_decode_attention) and the CUDA-core kernel (kivi_decode_attention_simt)
are checked.

Method: "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache",
study.space summary: decode attention over the quantized part, combined with
the full-precision residual part (one softmax over both here).
"""
import math

import numpy as np
import pytest
import torch

import bit_asymmetric_kv_quantize_b200 as kivi
from bit_asymmetric_kv_quantize_b200 import workloads as W
from kivi_testlib import (assert_decode_close, assert_state_equal, decode_error, gpu_cache,
                          oracle_append, oracle_cache, oracle_prefill, sample_units)

pytestmark = pytest.mark.gpu
KERNELS = ["default", "simt"]


def small(D=64, bits=2, dtype="f16", R=32, T=200, B=2, Hkv=2, gq=1, seed=3):
    return W.Workload(f"dec-d{D}-b{bits}-{dtype}-g{gq}-t{T}", B=B, Hq=Hkv * gq, Hkv=Hkv, D=D,
                      T=T, bits=bits, R=R, dtype=dtype, seed=seed)


def run(w, kernel, sigma=None, capacity=None):
    K, V = W.prompt_kv(w, device="cuda")
    gc = gpu_cache(w, capacity=capacity)
    gc.prefill(K, V)
    oc = oracle_cache(w, capacity=capacity)
    oracle_prefill(oc, K, V)
    q = W.query(w, device="cuda")
    sigma = 1.0 / math.sqrt(w.D) if sigma is None else sigma
    out = gc.decode(q, sigma, kernel=kernel)
    return gc, oc, q, out, sigma


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("gq", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype", ["f16", "f32"])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("D", [32, 64, 128])
def test_decode_shapes(D, bits, dtype, gq, kernel):
    if bits == 3 and kernel == "simt":
        pytest.skip("3-bit codes: tensor-core decode only")
    for T in (1, 33, 161, 1000):
        w = small(D=D, bits=bits, dtype=dtype, gq=gq, T=T)
        gc, oc, q, out, sigma = run(w, kernel, capacity=1024)
        assert_decode_close(out, oc, q, sigma)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("sigma", [1.0, 0.3, 2.0])
def test_decode_softmax_scale(sigma, kernel):
    w = small(D=128, gq=4, T=700)
    gc, oc, q, out, sigma = run(w, kernel, sigma=sigma, capacity=1024)
    assert_decode_close(out, oc, q, sigma)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("T", [64 * 32 + 1, 5000, 9000])
def test_decode_many_splits(T, kernel):
    """One unit, long context: the context is split over many CTAs and merged."""
    w = small(D=128, B=1, Hkv=1, gq=4, T=T, R=128)
    gc, oc, q, out, sigma = run(w, kernel, capacity=9216)
    assert gc.num_splits(w.Hq) > 4
    assert_decode_close(out, oc, q, sigma)


@pytest.mark.parametrize("kernel", KERNELS)
def test_decode_constant_values_and_zero_query(kernel):
    w = small(D=64, gq=2, T=300)
    K, V = W.prompt_kv(w, device="cuda")
    V.fill_(0.625)
    gc = gpu_cache(w, capacity=512)
    gc.prefill(K, V)
    q = W.query(w, device="cuda")
    out = gc.decode(q, 0.125, kernel=kernel)
    assert torch.allclose(out.float(), torch.full_like(out.float(), 0.625), atol=1e-3)
    # q = 0: uniform weights -> the mean of the dequantized values (oracle)
    K2, V2 = W.prompt_kv(w, device="cuda")
    gc2 = gpu_cache(w, capacity=512)
    gc2.prefill(K2, V2)
    oc2 = oracle_cache(w, capacity=512)
    oracle_prefill(oc2, K2, V2)
    qz = torch.zeros_like(q)
    assert_decode_close(gc2.decode(qz, 1.0, kernel=kernel), oc2, qz, 1.0)


@pytest.mark.parametrize("kernel", KERNELS)
def test_decode_tiny_workload(kernel):
    w = W.TINY
    gc, oc, q, out, _ = run(w, kernel, sigma=1.0)
    assert (gc.n_q, gc.r) == (224, 32)
    assert_decode_close(out, oc, q, 1.0)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("w", [W.LLAMA2_7B, W.MISTRAL_7B], ids=lambda w: w.name)
def test_decode_layer_workloads_full(w, kernel):
    """Every head of the full-size layer against the oracle (q carries 1/sqrt(D): sigma = 1)."""
    gc, oc, q, out, _ = run(w, kernel, sigma=1.0)
    assert_decode_close(out, oc, q, 1.0)


@pytest.mark.parametrize("w", [W.LLAMA2_13B_2BIT, W.LLAMA2_13B_4BIT], ids=lambda w: w.name)
def test_decode_large_batch_sampled(w):
    K, V = W.prompt_kv(w, device="cuda")
    gc = gpu_cache(w)
    gc.prefill(K, V)
    units = sample_units(w, 16)
    oc = oracle_cache(w, units=units)
    oracle_prefill(oc, K, V)
    q = W.query(w, device="cuda")
    for kernel in KERNELS:
        assert_decode_close(gc.decode(q, 1.0, kernel=kernel), oc, q, 1.0, units=units)


def test_streaming_workload_every_step():
    """Prompt of 32768 tokens, then 512 steps of append + decode (window flush
    every 128 steps).  Two sampled units are checked at every step; the
    quantized store of the sampled units is compared bit for bit after every
    flush."""
    w = W.STREAMING
    K, V = W.prompt_kv(w, device="cuda")
    gc = gpu_cache(w)
    gc.prefill(K, V)
    units = sample_units(w, 2, seed=5)
    oc = oracle_cache(w, units=units)
    oracle_prefill(oc, K, V)
    del K, V
    assert_state_equal(gc, oc)
    worst = 0.0
    for step in range(w.steps):
        k, v = W.step_kv(w, step, device="cuda")
        gc.append(k, v)
        oracle_append(oc, k, v)
        q = W.query(w, step, device="cuda")
        out = gc.decode(q, 1.0)
        mx, _ = assert_decode_close(out, oc, q, 1.0, units=units)
        worst = max(worst, mx)
        if gc.r == 1:
            assert_state_equal(gc, oc)
    assert gc.n_q + gc.r == w.T + w.steps
    print(f"streaming worst max-abs {worst:.3e}")


def test_streaming_workload_every_unit_at_flushes():
    """The streaming workload's 512 fused steps (kivi_append_decode) with the
    oracle holding all 128 units: every unit's store and window bit for bit
    after each of the four window flushes, and every unit's output within
    the bars at the first flush step, after the last flush and at the last
    step."""
    w = W.STREAMING
    K, V = W.prompt_kv(w, device="cuda")
    gc = gpu_cache(w)
    gc.prefill(K, V)
    oc = oracle_cache(w)
    oracle_prefill(oc, K, V)
    del K, V
    checked = 0
    for step in range(w.steps):
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        out = gc.append_decode(k, v, q, 1.0)
        oracle_append(oc, k, v)
        if gc.r == 1:
            assert_state_equal(gc, oc)
        if step in (0, 3 * w.R + 1, w.steps - 1):
            assert_decode_close(out, oc, q, 1.0)
            checked += 1
    assert checked == 3
    assert gc.n_q + gc.r == w.T + w.steps


@pytest.mark.parametrize("dtype,D", [("f16", 128), ("f16", 64), ("f32", 64)])
@pytest.mark.parametrize("gq", [1, 4])
def test_append_decode_matches_separate_calls(dtype, D, gq):
    """kivi_append_decode (one launch unless a flush is due) gives bit for bit
    the outputs and cache state of kivi_append_token + kivi_decode_attention,
    over 150 steps that cross two flushes (R = 64), and stays within the
    tolerance of the oracle."""
    w = small(D=D, dtype=dtype, gq=gq, T=100, R=64, B=2, Hkv=2, seed=11)
    K, V = W.prompt_kv(w, device="cuda")
    fused, ref = gpu_cache(w, capacity=512), gpu_cache(w, capacity=512)
    fused.prefill(K, V)
    ref.prefill(K, V)
    oc = oracle_cache(w, capacity=512)
    oracle_prefill(oc, K, V)
    for step in range(150):
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        out_f = fused.append_decode(k, v, q, 1.0)
        ref.append(k, v)
        out_r = ref.decode(q, 1.0)
        oracle_append(oc, k, v)
        assert (fused.n_q, fused.r) == (ref.n_q, ref.r)
        assert torch.equal(out_f, out_r), f"step {step}"
        if step % 25 == 0 or fused.r == 1:
            assert_decode_close(out_f, oc, q, 1.0)
    assert fused.n_q + fused.r == 100 + 150
    assert_state_equal(fused, oc)


def test_append_decode_unaligned_token_takes_the_two_launch_path():
    """k/v views at an 8-byte offset: same result as append + decode."""
    w = small(D=64, dtype="f16", gq=2, T=70, R=32, B=2, Hkv=2, seed=4)
    K, V = W.prompt_kv(w, device="cuda")
    a, b = gpu_cache(w, capacity=256), gpu_cache(w, capacity=256)
    a.prefill(K, V)
    b.prefill(K, V)
    for step in range(5):
        k, v = W.step_kv(w, step, device="cuda")
        kb = torch.empty(k.numel() + 4, dtype=k.dtype, device="cuda")
        vb = torch.empty(v.numel() + 4, dtype=v.dtype, device="cuda")
        ku = kb[4:].view(k.shape)
        vu = vb[4:].view(v.shape)
        ku.copy_(k)
        vu.copy_(v)
        assert ku.data_ptr() % 16 == 8
        q = W.query(w, step, device="cuda")
        out_a = a.append_decode(ku, vu, q, 1.0)
        b.append(k, v)
        assert torch.equal(out_a, b.decode(q, 1.0))


def test_decode_errors_on_device():
    w = small(D=64, T=100)
    K, V = W.prompt_kv(w, device="cuda")
    gc = gpu_cache(w, capacity=512)
    gc.prefill(K, V)
    q = W.query(w, device="cuda")
    out = torch.empty_like(q)
    L = kivi.lib()
    import ctypes
    ws = gc.workspace(w.Hq)
    rc = L.kivi_decode_attention(ctypes.byref(gc._c), q.data_ptr(), w.Hq, 1.0, out.data_ptr(),
                                 ws.data_ptr(), 16, None)
    assert rc == 5  # workspace too small
    rc = L.kivi_decode_attention(ctypes.byref(gc._c), q.data_ptr(), w.Hq, 1.0, out.data_ptr(),
                                 ws.data_ptr() + 4, ws.numel() - 4, None)
    assert rc == 5  # misaligned


@pytest.mark.parametrize("dtype,D", [("f16", 128), ("f32", 64)])
@pytest.mark.parametrize("gq", [1, 4])
def test_device_counter_loop_matches_host_counters(dtype, D, gq):
    """kivi_append_decode_dev (counters in device memory) gives bit for bit the
    outputs and cache of kivi_append_decode over 150 steps across two flushes."""
    w = small(D=D, dtype=dtype, gq=gq, T=100, R=64, B=2, Hkv=2, seed=12)
    K, V = W.prompt_kv(w, device="cuda")
    dev, host = gpu_cache(w, capacity=512), gpu_cache(w, capacity=512)
    dev.prefill(K, V)
    host.prefill(K, V)
    st = dev.dev_state()
    for step in range(150):
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        out_d = dev.append_decode_dev(st, k, v, q, 1.0)
        out_h = host.append_decode(k, v, q, 1.0)
        assert torch.equal(out_d, out_h), f"step {step}"
    dev.load_dev_state(st)
    assert (dev.n_q, dev.r) == (host.n_q, host.r) == (192, 58)
    n_q, r = dev.n_q, dev.r
    E, WB = (32, 3) if w.bits == 3 else (32 // w.bits, 1)
    used = {"k_codes": n_q, "k_scale": n_q // w.G, "k_zero": n_q // w.G, "v_codes": n_q // E * WB,
            "v_scale": n_q, "v_zero": n_q, "k_res": r, "v_res": r}
    for name, n in used.items():
        assert torch.equal(dev.view(name)[:, :, :n], host.view(name)[:, :, :n]), name


def test_device_counter_steps_replay_as_a_cuda_graph():
    """Four append + decode steps captured once and replayed 40 times (fresh
    inputs copied in before each replay, flushes every 32 tokens) equal the
    host-counter loop step for step."""
    w = small(D=128, dtype="f16", gq=2, T=90, R=32, B=2, Hkv=2, seed=13)
    K, V = W.prompt_kv(w, device="cuda")
    dev, host = gpu_cache(w, capacity=512), gpu_cache(w, capacity=512)
    dev.prefill(K, V)
    host.prefill(K, V)
    st = dev.dev_state()
    M = 4
    ks = [torch.empty(w.B, w.Hkv, w.D, dtype=w.torch_dtype, device="cuda") for _ in range(M)]
    vs = [torch.empty_like(x) for x in ks]
    qs = [torch.empty(w.B, w.Hq, w.D, dtype=w.torch_dtype, device="cuda") for _ in range(M)]
    outs = [torch.empty_like(x) for x in qs]
    # one eager step first (library setup happens outside the capture)
    k, v = W.step_kv(w, 0, device="cuda")
    q = W.query(w, 0, device="cuda")
    assert torch.equal(dev.append_decode_dev(st, k, v, q, 1.0), host.append_decode(k, v, q, 1.0))
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for j in range(M):
                dev.append_decode_dev(st, ks[j], vs[j], qs[j], 1.0, out=outs[j])
    torch.cuda.synchronize()
    step = 1
    for rep in range(40):
        for j in range(M):
            k, v = W.step_kv(w, step + j, device="cuda")
            ks[j].copy_(k)
            vs[j].copy_(v)
            qs[j].copy_(W.query(w, step + j, device="cuda"))
        g.replay()
        for j in range(M):
            k, v = W.step_kv(w, step + j, device="cuda")
            ref = host.append_decode(k, v, W.query(w, step + j, device="cuda"), 1.0)
            assert torch.equal(outs[j], ref), f"replay {rep} step {j}"
        step += M
    dev.load_dev_state(st)
    assert (dev.n_q, dev.r) == (host.n_q, host.r)
    del g


def test_device_counter_full_cache_sets_status():
    w = small(D=64, dtype="f16", gq=1, T=60, R=32, B=1, Hkv=2, seed=14)
    K, V = W.prompt_kv(w, device="cuda")
    c = gpu_cache(w, capacity=64)
    c.prefill(K, V)
    st = c.dev_state()
    q = W.query(w, 0, device="cuda")
    for step in range(4):  # 60 -> 64 tokens: fits
        k, v = W.step_kv(w, step, device="cuda")
        c.append_decode_dev(st, k, v, q, 1.0)
    c.load_dev_state(st)
    assert c.n_q + c.r == 64
    k, v = W.step_kv(w, 9, device="cuda")
    c.append_decode_dev(st, k, v, q, 1.0)  # no room: nothing happens on the device
    with pytest.raises(kivi.KiviError):
        c.load_dev_state(st)


def test_streaming_workload_device_counters_and_fused_steps():
    """The streaming workload at full size (B=4, 32 heads, prompt 32768, 512
    steps, flush every 128): the device-counter step and the host-counter
    fused step give bit for bit the outputs of append + decode at every step,
    and the counters agree at the end."""
    w = W.STREAMING
    K, V = W.prompt_kv(w, device="cuda")
    ref, fused, dev = gpu_cache(w), gpu_cache(w), gpu_cache(w)
    for c in (ref, fused, dev):
        c.prefill(K, V)
    del K, V
    st = dev.dev_state()
    for step in range(w.steps):
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        ref.append(k, v)
        out_r = ref.decode(q, 1.0)
        assert torch.equal(fused.append_decode(k, v, q, 1.0), out_r), f"fused step {step}"
        assert torch.equal(dev.append_decode_dev(st, k, v, q, 1.0), out_r), f"device step {step}"
    dev.load_dev_state(st)
    assert (ref.n_q, ref.r) == (fused.n_q, fused.r) == (dev.n_q, dev.r)


def _kernel_nodes(g) -> int:
    """Kernel launches captured in a torch CUDA graph (cuda-python runtime API)."""
    import cuda.bindings.runtime as rt
    graph = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
    err, nodes, n = rt.cudaGraphGetNodes(graph, 0)
    assert err == rt.cudaError_t.cudaSuccess
    err, nodes, n = rt.cudaGraphGetNodes(graph, n)
    assert err == rt.cudaError_t.cudaSuccess
    kinds = [rt.cudaGraphNodeGetType(x)[1] for x in nodes]
    return sum(1 for k in kinds if k == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)


@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_fused_steps_are_one_launch_each_flushes_included(dtype):
    """kivi_append_decode and kivi_append_decode_dev launch one kernel per
    step, also on the steps whose full window is flushed into the store (the
    decode kernel quantizes it itself); captured steps equal the separate
    append + decode calls bit for bit and stay within the bars vs the oracle."""
    w = small(D=128, dtype=dtype, gq=4, T=96, R=32, B=2, Hkv=2, seed=21)  # r = 32: flush due
    K, V = W.prompt_kv(w, device="cuda")
    fused, dev, ref = (gpu_cache(w, capacity=512) for _ in range(3))
    for c in (fused, dev, ref):
        c.prefill(K, V)
    oc = oracle_cache(w, capacity=512)
    oracle_prefill(oc, K, V)
    st = dev.dev_state()
    assert fused.r == fused.R
    # one eager step of each (library setup outside the captures)
    k, v = W.step_kv(w, 0, device="cuda")
    q = W.query(w, 0, device="cuda")
    a = fused.append_decode(k, v, q, 1.0)
    b = dev.append_decode_dev(st, k, v, q, 1.0)
    ref.append(k, v)
    c0 = ref.decode(q, 1.0)
    oracle_append(oc, k, v)
    assert torch.equal(a, c0) and torch.equal(b, c0)
    assert_decode_close(a, oc, q, 1.0)
    torch.cuda.synchronize()
    # steps 1..40 cross the next flush (r reaches 32 again at step 31)
    for step in range(1, 41):
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        flush = fused.r == fused.R
        outs = []
        for c, call in ((fused, lambda: fused.append_decode(k, v, q, 1.0)),
                        (dev, lambda: dev.append_decode_dev(st, k, v, q, 1.0))):
            g = torch.cuda.CUDAGraph(keep_graph=True)
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s):
                with torch.cuda.graph(g, stream=s):
                    out = call()
            torch.cuda.synchronize()
            assert _kernel_nodes(g) == 1, (step, flush)
            g.instantiate()
            g.replay()
            torch.cuda.synchronize()
            outs.append(out)
            del g
        ref.append(k, v)
        c0 = ref.decode(q, 1.0)
        oracle_append(oc, k, v)
        assert torch.equal(outs[0], c0), step
        assert torch.equal(outs[1], c0), step
        if flush or step % 10 == 0:
            assert_decode_close(outs[0], oc, q, 1.0)
    dev.load_dev_state(st)
    assert (dev.n_q, dev.r) == (fused.n_q, fused.r) == (ref.n_q, ref.r)
    assert_state_equal(fused, oc)



@pytest.mark.parametrize("gq", [1, 4, 8])
def test_three_bit_layer_sampled(gq):
    """3-bit codes (bit planes) on a layer-sized cache: store bit-exact and
    decode within the bars on sampled units, with fused steps across a flush."""
    w = W.Workload(f"three-bit-g{gq}", B=4, Hq=8 * gq, Hkv=8, D=128, T=3000, bits=3, R=128, seed=31)
    K, V = W.prompt_kv(w, device="cuda")
    gc = gpu_cache(w, capacity=3200)
    gc.prefill(K, V)
    units = sample_units(w, 8, seed=gq)
    oc = oracle_cache(w, units=units, capacity=3200)
    oracle_prefill(oc, K, V)
    assert_state_equal(gc, oc, units)
    sigma = 1.0 / math.sqrt(w.D)
    for step in range(130):  # the window (r = 56) fills and flushes once
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        out = gc.append_decode(k, v, q, sigma)
        oracle_append(oc, k, v)
        if step % 40 == 0 or step == 129:
            assert_decode_close(out, oc, q, sigma, units)
    assert_state_equal(gc, oc, units)


@pytest.mark.parametrize("dtype,D,gq", [("f16", 128, 1), ("f16", 64, 4), ("f32", 64, 1)])
def test_append_decode_host_matches_device_call(dtype, D, gq):
    """kivi_append_decode_host (inputs from pinned host memory, output back
    to host memory, one call) equals kivi_append_decode on device tensors bit
    for bit, over 70 steps that cross a flush (R = 64)."""
    w = small(D=D, dtype=dtype, gq=gq, T=100, R=64, B=2, Hkv=2, seed=13)
    K, V = W.prompt_kv(w, device="cuda")
    a, b = gpu_cache(w, capacity=512), gpu_cache(w, capacity=512)
    a.prefill(K, V)
    b.prefill(K, V)
    out = torch.empty(w.B, w.Hq, w.D, dtype=w.torch_dtype).pin_memory()
    for step in range(70):
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        kvq = torch.cat([k.flatten(), v.flatten(), q.flatten()]).cpu().pin_memory()
        ref = b.append_decode(k, v, q, 1.0)
        a.append_decode_host(kvq, w.Hq, 1.0, out)
        torch.cuda.synchronize()
        assert torch.equal(out, ref.cpu()), step
        assert (a.n_q, a.r) == (b.n_q, b.r)
    n_q, r = a.n_q, a.r
    E = 32 // w.bits
    lim = {"k_codes": n_q, "k_scale": n_q // 32, "k_zero": n_q // 32, "v_codes": n_q // E,
           "v_scale": n_q, "v_zero": n_q, "k_res": r, "v_res": r}
    for name in kivi.BUFFER_NAMES:  # the written parts of the store and window
        assert torch.equal(a.view(name)[:, :, :lim[name]], b.view(name)[:, :, :lim[name]]), name
