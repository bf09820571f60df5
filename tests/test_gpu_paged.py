"""GPU parity of the paged store (ragged batches whose quantized part is
pages of R tokens from a shared pool, addressed through a caller-owned block
table), through the C ABI.

Every sequence's pages, gathered through the block table, equal the oracle's
unit store bit for bit; decode over a paged cache equals decode over the
same batch in a contiguous cache bit for bit (the split plan depends on the
lengths only), and stays within the bars of kivi_testlib against the oracle.
KIVI, study.space summary: grouped and residual parts per sequence;
scholarfeed.org "KIVI" page, second quote: mixed precision and uniform paged
blocks, hence pages for the quantized part and a separate residual pool.
"""
import numpy as np
import pytest
import torch

import bit_asymmetric_kv_quantize_b200 as kivi
from bit_asymmetric_kv_quantize_b200 import workloads as W
from kivi_testlib import assert_decode_close, gpu_cache, oracle_cache, sample_units

pytestmark = pytest.mark.gpu


def small(D=64, bits=2, dtype="f16", R=32, T=300, B=4, Hkv=2, gq=1, seed=41, meta="f32"):
    return W.Workload(f"pag-d{D}-b{bits}-{dtype}-g{gq}", B=B, Hq=Hkv * gq, Hkv=Hkv, D=D, T=T,
                      bits=bits, R=R, dtype=dtype, seed=seed, len_min=1, meta=meta)


def block_table(B, pps, num_pages, seed=0):
    """Distinct pool pages for every (sequence, page), in a shuffled order."""
    g = torch.Generator().manual_seed(seed)
    ids = torch.randperm(num_pages, generator=g)[: B * pps].to(torch.int32)
    return ids.view(B, pps).contiguous().cuda()


def paged_cache(w, pps, num_pages, seed=0):
    bt = block_table(w.B, pps, num_pages, seed)
    return kivi.PagedKiviCache(w.B, w.Hkv, w.D, w.bits, pps, num_pages, bt, R=w.R, G=w.G,
                               Gv=w.Gv, dtype=w.torch_dtype, meta=w.torch_meta)


def gather_unit(pc, b, h, n_q, r):
    """The unit's store and window in the contiguous per-unit layout."""
    bt = pc.block_table.cpu()
    pages = [int(bt[b, l]) for l in range(n_q // pc.R)]
    out = {}
    for name in ("k_codes", "k_scale", "k_zero", "v_codes", "v_scale", "v_zero"):
        v = pc.view(name)
        parts = [v[p, h] for p in pages]
        t = torch.cat(parts) if parts else v[0, h][:0]
        out[name] = t.float().cpu().numpy() if t.is_floating_point() else t.cpu().numpy()
    for name in ("k_res", "v_res"):
        out[name] = pc.view(name)[b, h, :r].float().cpu().numpy()
    return out


def assert_paged_equal_oracle(pc, st, oc):
    n_q, r, status = kivi.ragged_lengths(st)
    for (b, h) in oc.units:
        u = oc.unit(b, h)
        assert status[b] == 0 and (n_q[b], r[b]) == (u.n_q, u.r), (b, h)
        got = gather_unit(pc, b, h, u.n_q, u.r)
        E, WB = (32, 3) if pc.bits == 3 else (32 // pc.bits, 1)
        lim = {"k_codes": u.n_q, "k_scale": u.n_q // 32, "k_zero": u.n_q // 32,
               "v_codes": u.n_q // E * WB, "v_scale": u.n_q, "v_zero": u.n_q, "k_res": u.r, "v_res": u.r}
        i = oc.slot(b, h)
        for name, n in lim.items():
            g = np.ascontiguousarray(got[name]).view(np.uint32)
            want = np.ascontiguousarray(getattr(oc, name)[i, :n]).view(np.uint32)
            assert np.array_equal(g, want), f"{name} differs at unit {(b, h)}"


def prefill_three(w, lens, pps, num_pages, units=None, seed=0):
    """The same prompt into a paged cache, a contiguous ragged cache and the oracle."""
    K, V = W.prompt_kv(w, device="cuda")
    pc = paged_cache(w, pps, num_pages, seed)
    st_p = pc.ragged_prefill(K, V, lens.cuda())
    cc = gpu_cache(w, capacity=(pps + 1) * w.R)
    st_c = cc.ragged_prefill(K, V, lens.cuda())
    oc = oracle_cache(w, units=units, capacity=(pps + 1) * w.R)
    for (b, h) in oc.units:
        n = int(lens[b])
        oc.prefill_unit(b, h, K[b, h, :n].float().cpu().numpy(), V[b, h, :n].float().cpu().numpy())
    return pc, st_p, cc, st_c, oc


@pytest.mark.parametrize("meta", ["f32", "f16"])
@pytest.mark.parametrize("gq", [1, 4, 8])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("D", [32, 64, 128])
def test_prefill_and_decode(D, bits, gq, meta):
    w = small(D=D, bits=bits, gq=gq, T=700, B=5, meta=meta)
    lens = torch.tensor([700, 1, 33, 129, 450], dtype=torch.int64)
    pps = 700 // w.R + 1
    pc, st_p, cc, st_c, oc = prefill_three(w, lens, pps, num_pages=5 * pps + 7)
    assert torch.equal(st_p, st_c)
    assert_paged_equal_oracle(pc, st_p, oc)
    q = W.query(w, device="cuda")
    out_p = pc.ragged_decode(st_p, q, 0.125)
    assert torch.equal(out_p, cc.ragged_decode(st_c, q, 0.125))
    assert_decode_close(out_p, oc, q, 0.125)


@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_steps_fill_new_pages(dtype):
    """90 fused steps (R = 32): every flush fills the sequence's next page
    from its table; outputs equal the contiguous cache's bit for bit and the
    pages match the oracle."""
    w = small(D=128, dtype=dtype, gq=2, T=200, B=4, R=32, seed=42)
    lens = torch.tensor([200, 5, 96, 131], dtype=torch.int64)
    pps = 10
    pc, st_p, cc, st_c, oc = prefill_three(w, lens, pps, num_pages=4 * pps, seed=3)
    for step in range(90):
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        out_p = pc.ragged_append_decode(st_p, k, v, q, 1.0)
        out_c = cc.ragged_append_decode(st_c, k, v, q, 1.0)
        kh, vh = k.float().cpu().numpy(), v.float().cpu().numpy()
        for (b, h) in oc.units:
            oc.append_unit(b, h, kh[b, h], vh[b, h])
        assert torch.equal(out_p, out_c), f"step {step}"
        if step % 15 == 0:
            assert_decode_close(out_p, oc, q, 1.0)
    assert torch.equal(st_p, st_c)
    assert_paged_equal_oracle(pc, st_p, oc)


def test_page_outside_the_pool_refuses_the_sequence():
    """A needed page id outside the pool sets the sequence's status at
    prefill (a long prompt) or at the flush that would fill it; the other
    sequences are unaffected."""
    w = small(D=64, T=100, B=3, R=32, seed=43)
    lens = torch.tensor([100, 40, 60], dtype=torch.int64)
    pps, P = 4, 12
    bt = torch.arange(3 * pps, dtype=torch.int32).view(3, pps).contiguous()
    bt[0, 1] = P + 5      # sequence 0 needs pages 0..2 for its 96 quantized tokens
    bt[2, 1] = -1         # sequence 2 fills page 1 at its first flush
    pc = kivi.PagedKiviCache(w.B, w.Hkv, w.D, w.bits, pps, P, bt.cuda(), R=w.R, dtype=w.torch_dtype)
    K, V = W.prompt_kv(w, device="cuda")
    st = pc.ragged_prefill(K, V, lens.cuda())
    n_q, r, status = kivi.ragged_lengths(st)
    assert status == [1, 0, 0]
    assert (n_q[1], r[1], n_q[2], r[2]) == (32, 8, 32, 28)
    for step in range(6):
        k, v = W.step_kv(w, step, device="cuda")
        out = pc.ragged_append_decode(st, k, v, W.query(w, step, device="cuda"), 1.0)
        n_q, r, status = kivi.ragged_lengths(st)
        assert status[2] == (1 if step >= 4 else 0), step  # r reached 32 after 4 steps
        assert torch.isnan(out[0].float()).all() and torch.isfinite(out[1].float()).all()
    assert (n_q[1], r[1]) == (32, 14)


def test_ragged_workload_paged_sampled():
    """The 32-sequence serving batch in a pool with shuffled pages: decode
    equals the contiguous cache's bit for bit, sampled units equal the oracle."""
    w = W.RAGGED
    lens = W.seq_lengths(w)
    pps = w.T // w.R + 1
    units = sample_units(w, 6, seed=9)
    pc, st_p, cc, st_c, oc = prefill_three(w, lens, pps, num_pages=w.B * pps + 100, units=units)
    assert_paged_equal_oracle(pc, st_p, oc)
    for step in range(8):
        k, v = W.step_kv(w, step, device="cuda")
        q = W.query(w, step, device="cuda")
        out_p = pc.ragged_append_decode(st_p, k, v, q, 1.0)
        out_c = cc.ragged_append_decode(st_c, k, v, q, 1.0)
        assert torch.equal(out_p, out_c), step
