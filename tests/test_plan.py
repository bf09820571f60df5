"""Host logic of the decode split plan and the paged address map, without a
GPU: the host/device helpers of csrc/kivi_internal.cuh compiled for the host
into a small test library, checked for the invariants the kernels rely on.

  * every work index lies in some CTA's range (P * W >= total), ranges are at
    least 12 indices long;
  * no unit meets more CTA segments than the plan's bound, and the bound
    fits the workspace's partial slots (seg_cap): the kernel writes a
    partial per segment into slot (cta - first cta of the unit);
  * the lengths a decode sees after a pending append follow the
    flush-before-write rule, and invalid counters are refused;
  * paged stores map a tile through the block table, refusing page ids
    outside the table or the pool.
"""
import ctypes
import os
import random
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_asymmetric_kv_quantize_b200", "csrc")

HARNESS = r'''
#include "kivi_internal.cuh"
extern "C" {
long long t_plan_ragged_w(long long total, long long nqmax, long long P, int seg_cap, int* ms) {
  return kivi::plan_ragged_w(total, nqmax, P, seg_cap, ms);
}
long long t_unit_work(long long n_q, int r, int f16) { return kivi::unit_work(n_q, r, f16 != 0); }
void t_plan_stream(long long units, long long n_q, int r, int f16, long long P, int seg_cap,
                   long long* out) {
  const kivi::StreamPlan p = kivi::plan_stream_core(units, n_q, r, f16 != 0, P, seg_cap);
  out[0] = p.n_cta; out[1] = p.W; out[2] = p.max_seg; out[3] = p.win_weight;
}
int t_seq_len(long long nq, int r, int status, int pending, long long Tq, int R, long long* onq,
              int* orr) {
  kivi::DevState s; s.n_q = nq; s.r = r; s.status = status;
  const kivi::SeqLen L = kivi::seq_len(s, pending != 0, Tq, R);
  *onq = L.n_q; *orr = L.r;
  return L.ok ? 1 : 0;
}
int t_store_tile(const int* bt, int pps, long long n_pages, int Hkv, int R, long long Tq,
                 long long u, long long t, long long* su, long long* st) {
  kivi::CacheView c = {};
  c.bt = bt; c.pps = pps; c.n_pages = n_pages; c.Hkv = Hkv; c.R = R; c.Tq = Tq;
  return kivi::store_tile(c, u, t, su, st) ? 1 : 0;
}
}
'''


@pytest.fixture(scope="module")
def plan_lib(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("plan")
    src = d / "harness.cu"
    src.write_text(HARNESS)
    so = d / "libplan.so"
    subprocess.run([nvcc, "-std=c++17", "-O1", "-shared", "-Xcompiler", "-fPIC", "-I", CSRC,
                    "-I", os.path.join(ROOT, "include"), "-o", str(so), str(src)], check=True)
    L = ctypes.CDLL(str(so))
    ll, ci = ctypes.c_longlong, ctypes.c_int
    L.t_plan_ragged_w.restype = ll
    L.t_plan_ragged_w.argtypes = [ll, ll, ll, ci, ctypes.POINTER(ci)]
    L.t_unit_work.restype = ll
    L.t_unit_work.argtypes = [ll, ci, ci]
    L.t_plan_stream.argtypes = [ll, ll, ci, ci, ll, ci, ctypes.POINTER(ll)]
    L.t_seq_len.argtypes = [ll, ci, ci, ci, ll, ci, ctypes.POINTER(ll), ctypes.POINTER(ci)]
    L.t_store_tile.argtypes = [ctypes.POINTER(ci), ci, ll, ci, ci, ll, ll, ll, ctypes.POINTER(ll),
                               ctypes.POINTER(ll)]
    return L


def segments(base, n_qt, W):
    """CTA segments of a unit: the CTAs whose ranges meet its tiles or its
    window start index (as the kernel's f_cta .. l_cta)."""
    return (base + n_qt) // W - base // W + 1


def test_ragged_plan_covers_all_work_within_the_slot_bound(plan_lib):
    rng = random.Random(5)
    for _ in range(3000):
        R = rng.choice([32, 64, 128])
        cap = R * rng.randint(1, 300)
        B, Hkv = rng.randint(1, 40), rng.choice([1, 2, 4, 8, 32])
        f16 = rng.random() < 0.5
        P = rng.choice([148, 296, 444, 1])
        seg_cap = rng.randint(2, 9)
        lens = []
        for _ in range(B):  # n_q a multiple of R within capacity - R, r in [0, R]
            n_q = R * rng.randint(0, cap // R - 1)
            lens.append((n_q, rng.randint(0 if n_q == 0 else 1, R)))
        work = [plan_lib.t_unit_work(nq, r, f16) for nq, r in lens]
        total = Hkv * sum(work)
        nqmax = max(nq // 32 for nq, _ in lens)
        ms = ctypes.c_int()
        W = plan_lib.t_plan_ragged_w(total, nqmax, P, seg_cap, ctypes.byref(ms))
        assert W >= 12
        assert P * W >= total  # the device plan runs a grid of exactly P CTAs
        assert ms.value <= seg_cap
        base = 0
        for b, (nq, r) in enumerate(lens):
            for h in range(Hkv):
                n = segments(base, nq // 32, W)
                assert n <= ms.value, (b, h, n, ms.value)
                assert (base + nq // 32) // W < P  # the unit's last CTA is in the grid
                base += work[b]
        assert base == total


def test_ragged_plan_uses_the_grid_when_the_slots_allow(plan_lib):
    # with enough partial slots, W is the even share of the work over P CTAs
    ms = ctypes.c_int()
    W = plan_lib.t_plan_ragged_w(296 * 100, 200, 296, 64, ctypes.byref(ms))
    assert W == 100 and ms.value == 200 // 100 + 2


@pytest.mark.parametrize("f16", [0, 1])
def test_uniform_plan_matches_the_unit_work(plan_lib, f16):
    rng = random.Random(6)
    out = (ctypes.c_longlong * 4)()
    for _ in range(2000):
        R = rng.choice([32, 128])
        n_q = R * rng.randint(0, 200)
        r = rng.randint(0 if n_q == 0 else 1, R)
        units = rng.randint(1, 3000)
        P, seg_cap = rng.choice([148, 296, 444]), rng.randint(2, 9)
        plan_lib.t_plan_stream(units, n_q, r, f16, P, seg_cap, out)
        n_cta, W, max_seg, ww = list(out)
        up = plan_lib.t_unit_work(n_q, r, f16)
        assert up == n_q // 32 + ww
        assert n_cta * W >= units * up and (n_cta - 1) * W < units * up
        assert max_seg <= seg_cap
        for u in (0, 1, units // 2, units - 1):
            assert segments(u * up, n_q // 32, W) <= max_seg


def test_lengths_after_a_pending_append(plan_lib):
    nq, r = ctypes.c_longlong(), ctypes.c_int()
    L = plan_lib

    def sl(n_q, rr, status=0, pending=1, Tq=512, R=128):
        ok = L.t_seq_len(n_q, rr, status, pending, Tq, R, ctypes.byref(nq), ctypes.byref(r))
        return ok, nq.value, r.value

    assert sl(256, 5) == (1, 256, 6)
    assert sl(256, 128) == (1, 384, 1)          # a full window flushes first
    assert sl(0, 0) == (1, 0, 1)
    assert sl(384, 128) == (1, 512, 1)          # the last page of the store
    assert sl(512, 128)[0] == 0                 # no room: refused
    assert sl(256, 5, pending=0) == (1, 256, 5)
    assert sl(256, 5, status=1)[0] == 0
    for bad in ((-128, 5), (640, 1), (100, 5), (256, 129), (256, -1)):
        assert sl(*bad, pending=0)[0] == 0, bad


def test_paged_tile_map(plan_lib):
    R, Hkv, pps, n_pages = 64, 3, 4, 10
    bt = (ctypes.c_int * (2 * pps))(7, 2, 9, -1, 0, 11, 5, 3)
    su, st = ctypes.c_longlong(), ctypes.c_longlong()

    def tile(u, t):
        ok = plan_lib.t_store_tile(bt, pps, n_pages, Hkv, R, pps * R, u, t, ctypes.byref(su),
                                   ctypes.byref(st))
        return (su.value, st.value) if ok else None

    tpp = R // 32
    # sequence 0 (units 0..2): pages 7, 2, 9; sequence 1 (units 3..5): 0, (11 invalid), 5, 3
    assert tile(0, 0) == (7 * Hkv + 0, 0)
    assert tile(2, 1) == (7 * Hkv + 2, 1)
    assert tile(1, tpp) == (2 * Hkv + 1, 0)
    assert tile(1, 2 * tpp + 1) == (9 * Hkv + 1, 1)
    assert tile(0, 3 * tpp) is None            # page id -1
    assert tile(4, 0) == (0 * Hkv + 1, 0)
    assert tile(4, tpp) is None                # page id 11 outside a pool of 10
    assert tile(5, 3 * tpp + 1) == (3 * Hkv + 2, 1)
    assert tile(3, 4 * tpp) is None            # past the table


@pytest.mark.parametrize("f16", [0, 1])
@pytest.mark.parametrize("seg_cap", [1, 2])
def test_uniform_plan_with_one_or_two_partial_slots(plan_lib, f16, seg_cap):
    """The smallest slot counts (the no-allocation call caps the slots to what
    its fixed scratch holds, down to one): with one slot every unit is exactly
    one CTA's range; with two, no unit meets more than two CTAs."""
    rng = random.Random(7 + seg_cap)
    out = (ctypes.c_longlong * 4)()
    for _ in range(2000):
        R = rng.choice([32, 128])
        n_q = R * rng.randint(0, 300)
        r = rng.randint(0 if n_q == 0 else 1, R)
        units = rng.randint(1, 8000)
        P = rng.choice([148, 296, 444])
        plan_lib.t_plan_stream(units, n_q, r, f16, P, seg_cap, out)
        n_cta, W, max_seg, ww = list(out)
        up = plan_lib.t_unit_work(n_q, r, f16)
        assert n_cta * W >= units * up and (n_cta - 1) * W < units * up
        assert max_seg <= seg_cap
        if seg_cap == 1:
            assert W == up and n_cta == units and max_seg == 1
        for u in {0, 1, units // 3, units // 2, units - 1}:
            if u < units:
                assert segments(u * up, n_q // 32, W) <= max_seg
