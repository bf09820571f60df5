"""GPU parity of ragged batches (per-sequence lengths held on the device)
against the oracle, unit by unit, through the C ABI: the store and window of
every sequence bit for bit at its own fill, decode attention within the bars
of kivi_testlib.

The oracle holds every (sequence, KV head) unit on its own, so a ragged batch
is the oracle's units prefilled with different prompt lengths.  KIVI,
study.space summary: grouped and residual parts per sequence; scholarfeed.org
"KIVI" page: mixed-precision caches and uniform paged blocks.
"""
import math

import numpy as np
import pytest
import torch

import bit_asymmetric_kv_quantize_b200 as kivi
from bit_asymmetric_kv_quantize_b200 import workloads as W
from kivi_testlib import assert_decode_close, gpu_cache, oracle_cache, sample_units

pytestmark = pytest.mark.gpu


def small(D=64, bits=2, dtype="f16", R=32, T=300, B=5, Hkv=2, gq=1, len_min=1, seed=31,
          meta="f32"):
    return W.Workload(f"rag-d{D}-b{bits}-{dtype}-g{gq}", B=B, Hq=Hkv * gq, Hkv=Hkv, D=D, T=T,
                      bits=bits, R=R, dtype=dtype, seed=seed, len_min=len_min, meta=meta)


def prefill_both(w, lens, capacity, units=None):
    K, V = W.prompt_kv(w, device="cuda")
    gc = gpu_cache(w, capacity=capacity)
    st = gc.ragged_prefill(K, V, lens.cuda())
    oc = oracle_cache(w, units=units, capacity=capacity)
    for (b, h) in oc.units:
        n = int(lens[b])
        oc.prefill_unit(b, h, K[b, h, :n].float().cpu().numpy(), V[b, h, :n].float().cpu().numpy())
    return gc, st, oc


def append_both(gc, st, oc, k, v, fused_q=None, sigma=1.0):
    kh, vh = k.float().cpu().numpy(), v.float().cpu().numpy()
    for (b, h) in oc.units:
        oc.append_unit(b, h, kh[b, h], vh[b, h])
    if fused_q is None:
        gc.ragged_append(st, k, v)
        return None
    return gc.ragged_append_decode(st, k, v, fused_q, sigma)


def assert_ragged_state_equal(gc, st, oc, units=None):
    """Counters and every unit's store and window, bit for bit, at its own fill."""
    units = oc.units if units is None else units
    n_q, r, status = kivi.ragged_lengths(st)
    E, WB = (32, 3) if gc.bits == 3 else (32 // gc.bits, 1)
    bufs = {}
    for name in kivi.BUFFER_NAMES:
        t = gc.view(name)
        bufs[name] = t.float().cpu().numpy() if t.is_floating_point() else t.cpu().numpy()
    for (b, h) in units:
        u = oc.unit(b, h)
        assert status[b] == 0, (b, status[b])
        assert (n_q[b], r[b]) == (u.n_q, u.r), ((b, h), (n_q[b], r[b]), (u.n_q, u.r))
        lim = {"k_codes": u.n_q, "k_scale": u.n_q // 32, "k_zero": u.n_q // 32,
               "v_codes": u.n_q // E * WB, "v_scale": u.n_q, "v_zero": u.n_q, "k_res": u.r, "v_res": u.r}
        i = oc.slot(b, h)
        for name in kivi.BUFFER_NAMES:
            n = lim[name]
            got = np.ascontiguousarray(bufs[name][b, h, :n]).view(np.uint32)
            want = np.ascontiguousarray(getattr(oc, name)[i, :n]).view(np.uint32)
            assert np.array_equal(got, want), f"{name} differs at unit {(b, h)}"


def test_prefill_lengths_and_refusals():
    """Lengths at and around multiples of 32 and R, the extremes, and two
    refused lengths (0 and beyond the capacity) that only set status."""
    w = small(B=10, T=300, R=64)
    cap = 320
    lens = torch.tensor([1, 31, 32, 33, 64, 65, 129, 300, 0, cap + 1], dtype=torch.int64)
    K, V = W.prompt_kv(w, device="cuda")
    gc = gpu_cache(w, capacity=cap)
    st = gc.ragged_prefill(K, V, lens.cuda())
    n_q, r, status = kivi.ragged_lengths(st)
    for b in range(8):
        n = int(lens[b])
        assert (n_q[b], r[b], status[b]) == (n - ((n - 1) % 64 + 1), (n - 1) % 64 + 1, 0), b
    assert status[8] == 1 and status[9] == 1
    units = [(b, h) for b in range(8) for h in range(w.Hkv)]
    oc = oracle_cache(w, units=units, capacity=cap)
    Kh, Vh = K.float().cpu().numpy(), V.float().cpu().numpy()
    for (b, h) in units:
        oc.prefill_unit(b, h, Kh[b, h, :int(lens[b])], Vh[b, h, :int(lens[b])])
    assert_ragged_state_equal(gc, st, oc)


@pytest.mark.parametrize("meta", ["f32", "f16"])
@pytest.mark.parametrize("gq", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype", ["f16", "f32"])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("D", [32, 64, 128])
def test_decode_shapes(D, bits, dtype, gq, meta):
    if meta == "f16" and dtype == "f32":
        pytest.skip("binary16 metadata is offered for fp16 caches only")
    w = small(D=D, bits=bits, dtype=dtype, gq=gq, T=700, B=6, meta=meta)
    lens = torch.tensor([700, 1, 33, 64, 450, 129], dtype=torch.int64)
    gc, st, oc = prefill_both(w, lens, capacity=736)
    q = W.query(w, device="cuda")
    sigma = 1.0 / math.sqrt(D)
    assert_decode_close(gc.ragged_decode(st, q, sigma), oc, q, sigma)


@pytest.mark.parametrize("gq", [1, 4])
@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_steps_cross_flushes_per_sequence(dtype, gq):
    """100 fused steps: each sequence flushes at its own step (R = 32); the
    state matches the oracle after every flush, the output at sampled steps,
    and append + decode as separate calls gives the fused step's bits."""
    w = small(D=128, dtype=dtype, gq=gq, T=200, B=4, R=32, seed=33)
    lens = torch.tensor([200, 5, 96, 131], dtype=torch.int64)
    gc, st, oc = prefill_both(w, lens, capacity=320)
    ref = gpu_cache(w, capacity=320)
    K, V = W.prompt_kv(w, device="cuda")
    st_ref = ref.ragged_prefill(K, V, lens.cuda())
    for step in range(100):
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        out = append_both(gc, st, oc, k, v, fused_q=q)
        ref.ragged_append(st_ref, k, v)
        out_ref = ref.ragged_decode(st_ref, q, 1.0)
        assert torch.equal(out, out_ref), f"step {step}"
        if step % 10 == 0 or step in (26, 27, 28, 59, 60, 91):
            assert_decode_close(out, oc, q, 1.0)
            assert_ragged_state_equal(gc, st, oc)
    assert_ragged_state_equal(gc, st, oc)
    assert torch.equal(st, st_ref)


def test_uniform_lengths_match_the_uniform_path():
    """Equal lengths through the ragged calls give the uniform calls' cache
    bytes and, within the bars, their outputs."""
    w = small(D=128, gq=4, T=333, B=3, R=64, seed=34)
    K, V = W.prompt_kv(w, device="cuda")
    a, b = gpu_cache(w, capacity=512), gpu_cache(w, capacity=512)
    a.prefill(K, V)
    st = b.ragged_prefill(K, V, torch.full((w.B,), 333, dtype=torch.int64, device="cuda"))
    for step in range(40):
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        oa = a.append_decode(k, v, q, 1.0)
        ob = b.ragged_append_decode(st, k, v, q, 1.0)
        assert (oa.float() - ob.float()).abs().max().item() <= 2e-3
    n_q, r, status = kivi.ragged_lengths(st)
    assert set(n_q) == {a.n_q} and set(r) == {a.r} and set(status) == {0}
    E, WB = (32, 3) if w.bits == 3 else (32 // w.bits, 1)
    used = {"k_codes": a.n_q, "k_scale": a.n_q // 32, "k_zero": a.n_q // 32, "v_codes": a.n_q // E * WB,
            "v_scale": a.n_q, "v_zero": a.n_q, "k_res": a.r, "v_res": a.r}
    for name, n in used.items():
        assert torch.equal(a.view(name)[:, :, :n], b.view(name)[:, :, :n]), name


def test_full_sequence_stops_alone():
    """A sequence that runs out of room gets status 1 and NaN output; the
    others keep appending and decoding correctly."""
    w = small(D=64, T=90, B=3, R=32, seed=35)
    lens = torch.tensor([90, 30, 60], dtype=torch.int64)
    cap = 96
    gc, st, oc = prefill_both(w, lens, capacity=cap, units=[(1, 0), (1, 1), (2, 0), (2, 1)])
    for step in range(10):
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        out = append_both(gc, st, oc, k, v, fused_q=q)
        n_q, r, status = kivi.ragged_lengths(st)
        full = step >= 96 - 90  # sequence 0 had 6 free slots
        assert status[0] == (1 if full else 0), step
        if full:
            assert torch.isnan(out[0].float()).all()
        checked = out.clone()
        checked[0] = 0  # sequence 0 is not held by the oracle
        assert_decode_close(checked, oc, q, 1.0)  # sequences 1 and 2
        assert_ragged_state_equal(gc, st, oc)


def test_ragged_steps_replay_as_a_cuda_graph():
    """Three fused ragged steps captured once, replayed 30 times with fresh
    inputs copied in, equal the same calls made eagerly."""
    w = small(D=128, gq=2, T=150, B=4, R=32, seed=36)
    lens = torch.tensor([150, 7, 64, 100], dtype=torch.int64)
    K, V = W.prompt_kv(w, device="cuda")
    g, e = gpu_cache(w, capacity=320), gpu_cache(w, capacity=320)
    st_g = g.ragged_prefill(K, V, lens.cuda())
    st_e = e.ragged_prefill(K, V, lens.cuda())
    kv_shape, q_shape = (w.B, w.Hkv, w.D), (w.B, w.Hq, w.D)
    ins = [tuple(torch.zeros(sh, dtype=w.torch_dtype, device="cuda")
                 for sh in (kv_shape, kv_shape, q_shape)) for _ in range(3)]
    outs = [torch.empty(q_shape, dtype=w.torch_dtype, device="cuda") for _ in range(3)]
    g._ragged_ws(w.Hq)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            for j in range(3):
                g.ragged_append_decode(st_g, ins[j][0], ins[j][1], ins[j][2], 1.0, out=outs[j])
    torch.cuda.synchronize()
    step = 0
    for rep in range(30):
        for j in range(3):
            k, v = W.step_kv(w, step + j, device="cuda")
            ins[j][0].copy_(k)
            ins[j][1].copy_(v)
            ins[j][2].copy_(W.query(w, step + j, device="cuda"))
        graph.replay()
        for j in range(3):
            k, v = W.step_kv(w, step + j, device="cuda")
            oe = e.ragged_append_decode(st_e, k, v, W.query(w, step + j, device="cuda"), 1.0)
            assert torch.equal(outs[j], oe), (rep, j)
        step += 3
    assert torch.equal(st_g, st_e)


def test_ragged_workload_sampled():
    """The ragged serving batch (32 sequences, lengths 256..8192): sampled
    units bit for bit and within the bars after prefill and after 40 steps."""
    w = W.RAGGED
    lens = W.seq_lengths(w)
    cap = -(-(w.T + 64) // w.R) * w.R
    units = sample_units(w, 12, seed=7)
    gc, st, oc = prefill_both(w, lens, capacity=cap, units=units)
    assert_ragged_state_equal(gc, st, oc)
    q = W.query(w, device="cuda")
    assert_decode_close(gc.ragged_decode(st, q, 1.0), oc, q, 1.0, units=units)
    for step in range(40):
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        out = append_both(gc, st, oc, k, v, fused_q=q)
        if step % 8 == 0:
            assert_decode_close(out, oc, q, 1.0, units=units)
    assert_ragged_state_equal(gc, st, oc)
