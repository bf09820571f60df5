"""The C-ABI library without a GPU: it loads, exports every symbol that
include/kivi.h declares, and rejects bad arguments on the host before any
CUDA call.  (No compute call runs here.)"""
import ctypes
import os
import re

import pytest
import torch

import bit_asymmetric_kv_quantize_b200 as kivi
from bit_asymmetric_kv_quantize_b200 import KiviCacheC, KiviDims

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kivi.h")

ERR_ARG, ERR_UNSUPPORTED, ERR_STATE, ERR_CAPACITY, ERR_WORKSPACE = 1, 2, 3, 4, 5


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"KIVI_API\s+[\w\s\*]*?\b(kivi_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    syms = declared_symbols()
    assert len(syms) >= 10
    L = kivi.lib()
    for s in syms:
        assert hasattr(L, s), s
    assert set(syms) == set(kivi.EXPORTED)


def _dims(**kw):
    d = dict(B=2, Hkv=4, D=128, bits=2, G=32, Gv=32, R=128, capacity=4096, dtype=kivi.KIVI_F16,
             meta=kivi.KIVI_META_F32, k_out=0, v_out=0)
    d.update(kw)
    return KiviDims(d["B"], d["Hkv"], d["D"], d["bits"], d["G"], d["Gv"], d["R"], d["capacity"],
                    d["dtype"], d["meta"], d["k_out"], d["v_out"])


def _block(bits):
    """(codes per block, words per block): 32 codes as three bit planes at 3 bits."""
    return (32, 3) if bits == 3 else (32 // bits, 1)


def _sizes(dims):
    out = (ctypes.c_size_t * 8)()
    rc = kivi.lib().kivi_buffer_sizes(ctypes.byref(dims), ctypes.byref(out))
    return rc, list(out)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("D", [32, 64, 128])
def test_buffer_sizes_follow_the_layout(bits, D):
    B, H, R, cap = 3, 5, 64, 640
    rc, s = _sizes(_dims(B=B, Hkv=H, D=D, bits=bits, R=R, capacity=cap))
    assert rc == 0
    (E, WB), Tq, u = _block(bits), cap - R, B * H
    assert s[0] == u * Tq * (D // E) * WB * 4      # k_codes
    assert s[1] == s[2] == u * (Tq // 32) * D * 4  # k_scale, k_zero
    assert s[3] == u * (Tq // E) * WB * D * 4      # v_codes
    assert s[4] == s[5] == u * Tq * (D // 32) * 4  # v_scale, v_zero
    assert s[6] == s[7] == u * R * D * 2           # k_res, v_res (fp16)
    # 2-bit codes + fp32 scale/zero per 32: 0.5 byte per key and per value element
    if bits == 2:
        assert sum(s[:6]) == u * Tq * D * 2 * 0.5


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("D", [32, 64, 128])
def test_binary16_metadata_halves_the_scale_and_zero_buffers(bits, D):
    B, H, R, cap = 3, 5, 64, 640
    rc32, s32 = _sizes(_dims(B=B, Hkv=H, D=D, bits=bits, R=R, capacity=cap))
    rc16, s16 = _sizes(_dims(B=B, Hkv=H, D=D, bits=bits, R=R, capacity=cap, meta=kivi.KIVI_META_F16))
    assert rc32 == rc16 == 0
    for i in (1, 2, 4, 5):  # k_scale, k_zero, v_scale, v_zero
        assert 2 * s16[i] == s32[i]
    for i in (0, 3, 6, 7):  # codes and window unchanged
        assert s16[i] == s32[i]
    # 2-bit codes + binary16 scale/zero per 32: 3/8 byte per key and per value element
    if bits == 2:
        u, Tq = B * H, cap - R
        assert sum(s16[:6]) == u * Tq * D * 2 * 0.375


def test_dims_struct_matches_the_header():
    # the Python mirror of kivi_dims: nine ints/longs, then the metadata type
    names = [f[0] for f in KiviDims._fields_]
    assert names == ["B", "Hkv", "D", "bits", "G", "Gv", "R", "capacity", "dtype", "meta",
                     "k_out", "v_out"]
    text = open(HEADER).read()
    body = text[text.index("typedef struct {\n  int B;"):text.index("} kivi_dims;")]
    assert re.findall(r"\b(?:int|long long)\s+(\w+);", body) == names


@pytest.mark.parametrize("kw,rc", [
    (dict(meta=2), ERR_UNSUPPORTED), (dict(meta=-1), ERR_UNSUPPORTED),
    (dict(meta=kivi.KIVI_META_F16, dtype=kivi.KIVI_F32), ERR_UNSUPPORTED),
    (dict(bits=5), ERR_UNSUPPORTED), (dict(bits=8), ERR_UNSUPPORTED),
    (dict(G=16), ERR_UNSUPPORTED), (dict(Gv=64), ERR_UNSUPPORTED),
    (dict(D=96), ERR_UNSUPPORTED), (dict(R=48), ERR_UNSUPPORTED),
    (dict(capacity=4100), ERR_UNSUPPORTED), (dict(dtype=7), ERR_UNSUPPORTED),
    (dict(B=0), ERR_ARG), (dict(Hkv=-1), ERR_ARG), (dict(capacity=0), ERR_ARG),
])
def test_unsupported_dims(kw, rc):
    assert _sizes(_dims(**kw))[0] == rc


def _fake_cache(**kw):
    """A cache bound to fake (never dereferenced) aligned addresses."""
    dims = _dims(**kw)
    c = KiviCacheC()
    ptrs = (ctypes.c_void_p * 8)(*[0x10000 * (i + 1) for i in range(8)])
    assert kivi.lib().kivi_cache_init(ctypes.byref(c), ctypes.byref(dims), ctypes.byref(ptrs)) == 0
    assert (c.n_q, c.r) == (0, 0)
    return c


def test_cache_init_rejects_null_and_misaligned():
    L = kivi.lib()
    dims = _dims()
    c = KiviCacheC()
    ptrs = (ctypes.c_void_p * 8)(*[0x10000 * (i + 1) for i in range(8)])
    ptrs[3] = None
    assert L.kivi_cache_init(ctypes.byref(c), ctypes.byref(dims), ctypes.byref(ptrs)) == ERR_ARG
    ptrs[3] = 0x30008  # 8-byte aligned only
    assert L.kivi_cache_init(ctypes.byref(c), ctypes.byref(dims), ctypes.byref(ptrs)) == ERR_ARG
    assert L.kivi_cache_init(None, ctypes.byref(dims), ctypes.byref(ptrs)) == ERR_ARG


def test_window_only_cache_needs_no_store_buffers():
    dims = _dims(R=128, capacity=128)
    c = KiviCacheC()
    ptrs = (ctypes.c_void_p * 8)(None, None, None, None, None, None, 0x1000, 0x2000)
    assert kivi.lib().kivi_cache_init(ctypes.byref(c), ctypes.byref(dims), ctypes.byref(ptrs)) == 0


def test_host_side_state_and_capacity_errors():
    L = kivi.lib()
    fake = ctypes.c_void_p(0x5000)
    c = _fake_cache(R=128, capacity=256)
    assert L.kivi_quantize_prefill(ctypes.byref(c), fake, fake, -1, None) == ERR_ARG
    assert L.kivi_quantize_prefill(ctypes.byref(c), None, fake, 5, None) == ERR_ARG
    assert L.kivi_quantize_prefill(ctypes.byref(c), fake, fake, 257, None) == ERR_CAPACITY
    assert L.kivi_quantize_prefill(ctypes.byref(c), fake, fake, 0, None) == 0  # no-op
    assert (c.n_q, c.r) == (0, 0)
    # decode on an empty cache, and with a query head count that is not a multiple of Hkv
    assert L.kivi_decode_attention(ctypes.byref(c), fake, 4, 1.0, fake, fake, 1 << 20, None) == ERR_STATE
    assert L.kivi_decode_attention(ctypes.byref(c), fake, 6, 1.0, fake, fake, 1 << 20, None) == ERR_ARG
    assert L.kivi_decode_attention(ctypes.byref(c), fake, 12, 1.0, fake, fake, 1 << 20, None) == ERR_UNSUPPORTED
    # pretend a full cache: prefill refused (not empty), append refused (no room)
    c.n_q, c.r = 128, 128
    assert L.kivi_quantize_prefill(ctypes.byref(c), fake, fake, 1, None) == ERR_STATE
    assert L.kivi_append_token(ctypes.byref(c), fake, fake, None) == ERR_CAPACITY
    assert L.kivi_append_token(ctypes.byref(c), None, fake, None) == ERR_ARG
    assert (c.n_q, c.r) == (128, 128)  # unchanged by refused calls
    # the fused step refuses what either half would refuse, before any launch
    assert L.kivi_append_decode(ctypes.byref(c), fake, fake, fake, 4, 1.0, fake, fake, 1 << 20,
                                None) == ERR_CAPACITY
    c.n_q, c.r = 0, 5
    assert L.kivi_append_decode(ctypes.byref(c), None, fake, fake, 4, 1.0, fake, fake, 1 << 20,
                                None) == ERR_ARG
    assert L.kivi_append_decode(ctypes.byref(c), fake, fake, fake, 6, 1.0, fake, fake, 1 << 20,
                                None) == ERR_ARG
    assert L.kivi_append_decode(ctypes.byref(c), fake, fake, None, 4, 1.0, fake, fake, 1 << 20,
                                None) == ERR_ARG
    assert (c.n_q, c.r) == (0, 5)


def test_host_step_validates_before_any_copy():
    """kivi_host_step_bytes is host arithmetic (k | v | q, then out at the
    next 16-byte boundary); kivi_append_decode_host refuses bad arguments and
    a full cache before it copies anything."""
    L = kivi.lib()
    L.kivi_host_step_bytes.argtypes = [ctypes.POINTER(KiviCacheC), ctypes.c_int]
    L.kivi_host_step_bytes.restype = ctypes.c_size_t
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    L.kivi_append_decode_host.argtypes = [ctypes.POINTER(KiviCacheC), vp, ctypes.c_int,
                                          ctypes.c_float, vp, vp, sz, vp, sz, vp]
    c = _fake_cache(R=128, capacity=256)
    B, Hkv, D = c.dims.B, c.dims.Hkv, c.dims.D
    es = 2 if c.dims.dtype == 0 else 4
    for Hq in (Hkv, 2 * Hkv):
        kv, qo = B * Hkv * D * es, B * Hq * D * es
        want = -(-(2 * kv + qo) // 16) * 16 + -(-qo // 16) * 16
        assert L.kivi_host_step_bytes(ctypes.byref(c), Hq) == want
    assert L.kivi_host_step_bytes(ctypes.byref(c), Hkv + 1) == 0
    need = L.kivi_host_step_bytes(ctypes.byref(c), Hkv)
    host, dev = vp(0x7000), vp(0x9000)

    def call(kvq=host, out=host, staging=dev, nbytes=need, Hq=Hkv):
        return L.kivi_append_decode_host(ctypes.byref(c), kvq, Hq, 1.0, out, staging, nbytes, dev,
                                         1 << 20, None)
    assert call(kvq=None) == ERR_ARG
    assert call(out=None) == ERR_ARG
    assert call(staging=vp(0x9008)) == ERR_ARG  # misaligned staging
    assert call(Hq=Hkv + 1) == ERR_ARG
    assert call(nbytes=need - 1) == ERR_WORKSPACE
    c.n_q, c.r = 128, 128  # full
    assert call() == ERR_CAPACITY
    assert (c.n_q, c.r) == (128, 128)


def test_status_strings():
    L = kivi.lib()
    for code, name in kivi.STATUS.items():
        assert L.kivi_status_string(code).decode().startswith(name)
    assert b"unknown" in L.kivi_status_string(99)


def test_product_path_refuses_cpu_tensors():
    with pytest.raises((ValueError, RuntimeError)):
        kivi.KiviCache(1, 1, 32, 2, 64, R=32, dtype=torch.float32, device="cpu")


def test_oracle_and_library_share_no_source():
    """The oracle and the CUDA path are independent: no file includes or imports the other."""
    csrc = os.path.join(ROOT, "bit_asymmetric_kv_quantize_b200", "csrc")
    for f in os.listdir(csrc):
        text = open(os.path.join(csrc, f)).read()
        assert not re.search(r'#\s*include\s*[<"][^>"]*oracle', text), f
    for f in ("kivi_oracle.c", "kivi_oracle.h", "__init__.py"):
        text = open(os.path.join(ROOT, "oracle", f)).read()
        assert not re.search(r'#\s*include\s*[<"]kivi\.h', text), f
        assert not re.search(r"(import|from)\s+bit_asymmetric_kv_quantize_b200", text), f
    pkg = os.path.join(ROOT, "bit_asymmetric_kv_quantize_b200")
    for f in os.listdir(pkg):
        if f.endswith(".py"):
            assert "import oracle" not in open(os.path.join(pkg, f)).read(), f


def test_ragged_calls_validate_on_the_host():
    """Ragged calls check their arguments before any launch, and ragged and
    host-counter calls refuse each other's caches."""
    L = kivi.lib()
    fake = ctypes.c_void_p(0x5000)
    c = _fake_cache(R=128, capacity=512)
    # a cache not filled by kivi_ragged_prefill
    assert L.kivi_ragged_append(ctypes.byref(c), fake, fake, fake, None) == ERR_STATE
    assert L.kivi_ragged_decode(ctypes.byref(c), fake, fake, 4, 1.0, fake, fake, 1 << 20,
                                None) == ERR_STATE
    # state null or not 16-byte aligned
    assert L.kivi_ragged_append(ctypes.byref(c), None, fake, fake, None) == ERR_ARG
    assert L.kivi_ragged_append(ctypes.byref(c), ctypes.c_void_p(0x5008), fake, fake,
                                None) == ERR_ARG
    assert L.kivi_ragged_prefill(ctypes.byref(c), None, fake, fake, 100, fake, None) == ERR_ARG
    assert L.kivi_ragged_prefill(ctypes.byref(c), fake, fake, fake, 0, fake, None) == ERR_ARG
    assert L.kivi_ragged_prefill(ctypes.byref(c), fake, fake, fake, 100, None, None) == ERR_ARG
    # a ragged cache (its host counters carry the ragged mark)
    c.n_q, c.r = -1, 0
    assert L.kivi_append_token(ctypes.byref(c), fake, fake, None) == ERR_STATE
    assert L.kivi_decode_attention(ctypes.byref(c), fake, 4, 1.0, fake, fake, 1 << 20,
                                   None) == ERR_STATE
    assert L.kivi_append_decode(ctypes.byref(c), fake, fake, fake, 4, 1.0, fake, fake, 1 << 20,
                                None) == ERR_STATE
    assert L.kivi_dev_state_init(ctypes.byref(c), fake, None) == ERR_STATE
    assert L.kivi_quantize_prefill(ctypes.byref(c), fake, fake, 10, None) == ERR_STATE
    assert L.kivi_ragged_prefill(ctypes.byref(c), fake, fake, fake, 100, fake, None) == ERR_STATE
    assert L.kivi_decode_num_splits(ctypes.byref(c), 4) == 0
    # shape errors of the ragged decode come before any device query
    assert L.kivi_ragged_decode(ctypes.byref(c), fake, fake, 6, 1.0, fake, fake, 1 << 20,
                                None) == ERR_ARG
    assert L.kivi_ragged_decode(ctypes.byref(c), fake, fake, 12, 1.0, fake, fake, 1 << 20,
                                None) == ERR_UNSUPPORTED
    assert L.kivi_ragged_append_decode(ctypes.byref(c), fake, None, fake, fake, 4, 1.0, fake,
                                       fake, 1 << 20, None) == ERR_ARG


def test_ragged_lengths_of_a_state():
    """The Python reader of a ragged state follows the 16-byte layout."""
    st = torch.zeros(3 * 16, dtype=torch.uint8)
    v = st.view(torch.int64).view(3, 2)
    v[:, 0] = torch.tensor([0, 4096, 1 << 40])
    w = st.view(torch.int32).view(3, 4)
    w[:, 2] = torch.tensor([1, 128, 7], dtype=torch.int32)
    w[:, 3] = torch.tensor([0, 0, 1], dtype=torch.int32)
    assert kivi.ragged_lengths(st) == ([0, 4096, 1 << 40], [1, 128, 7], [0, 0, 1])


def test_cache_struct_matches_the_header():
    names = [f[0] for f in KiviCacheC._fields_]
    text = open(HEADER).read()
    body = text[text.index("typedef struct {\n  kivi_dims dims;"):text.index("} kivi_cache;")]
    declared = re.findall(r"\b(\w+);", re.sub(r"/\*.*?\*/", "", body, flags=re.S))
    assert declared == names


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_paged_buffer_sizes(bits):
    B, H, D, R, P = 3, 5, 128, 64, 11
    dims = _dims(B=B, Hkv=H, D=D, bits=bits, R=R, capacity=4 * R)
    out = (ctypes.c_size_t * 8)()
    assert kivi.lib().kivi_paged_buffer_sizes(ctypes.byref(dims), P, ctypes.byref(out)) == 0
    E, WB = _block(bits)
    s = list(out)
    assert s[0] == P * H * R * (D // E) * WB * 4
    assert s[1] == s[2] == P * H * (R // 32) * D * 4
    assert s[3] == P * H * (R // E) * WB * D * 4
    assert s[4] == s[5] == P * H * R * (D // 32) * 4
    assert s[6] == s[7] == B * H * R * D * 2
    assert kivi.lib().kivi_paged_buffer_sizes(ctypes.byref(dims), 0, ctypes.byref(out)) == ERR_ARG


def test_paged_cache_init_and_refusals():
    L = kivi.lib()
    R = 64
    dims = _dims(R=R, capacity=5 * R)  # 4 pages per sequence + the window
    ptrs = (ctypes.c_void_p * 8)(*[0x10000 * (i + 1) for i in range(8)])
    bt = ctypes.c_void_p(0x90000)
    c = KiviCacheC()
    assert L.kivi_paged_cache_init(ctypes.byref(c), ctypes.byref(dims), ctypes.byref(ptrs), None, 4,
                                   16) == ERR_ARG
    assert L.kivi_paged_cache_init(ctypes.byref(c), ctypes.byref(dims), ctypes.byref(ptrs), bt, 3,
                                   16) == ERR_ARG  # capacity is not (3 + 1) * R
    assert L.kivi_paged_cache_init(ctypes.byref(c), ctypes.byref(dims), ctypes.byref(ptrs), bt, 4,
                                   0) == ERR_ARG
    assert L.kivi_paged_cache_init(ctypes.byref(c), ctypes.byref(dims), ctypes.byref(ptrs), bt, 4,
                                   16) == 0
    assert (c.block_table, c.pages_per_seq, c.num_pages, c.n_q, c.r) == (0x90000, 4, 16, 0, 0)
    fake = ctypes.c_void_p(0x5000)
    # a paged cache takes the ragged calls only
    assert L.kivi_quantize_prefill(ctypes.byref(c), fake, fake, 10, None) == ERR_STATE
    assert L.kivi_append_token(ctypes.byref(c), fake, fake, None) == ERR_STATE
    assert L.kivi_dev_state_init(ctypes.byref(c), fake, None) == ERR_STATE
    c.n_q, c.r = 64, 5
    assert L.kivi_decode_attention(ctypes.byref(c), fake, 4, 1.0, fake, fake, 1 << 20,
                                   None) == ERR_STATE
    # a contiguous cache carries no block table
    c2 = _fake_cache()
    assert (c2.block_table, c2.pages_per_seq, c2.num_pages) == (None, 0, 0)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_paged_pool_with_binary16_metadata(bits):
    B, H, D, R, P = 2, 3, 64, 32, 9
    out = (ctypes.c_size_t * 8)()
    d32 = _dims(B=B, Hkv=H, D=D, bits=bits, R=R, capacity=4 * R)
    d16 = _dims(B=B, Hkv=H, D=D, bits=bits, R=R, capacity=4 * R, meta=kivi.KIVI_META_F16)
    L = kivi.lib()
    assert L.kivi_paged_buffer_sizes(ctypes.byref(d32), P, ctypes.byref(out)) == 0
    s32 = list(out)
    assert L.kivi_paged_buffer_sizes(ctypes.byref(d16), P, ctypes.byref(out)) == 0
    s16 = list(out)
    E, WB = _block(bits)
    assert s16[0] == s32[0] == P * H * R * (D // E) * WB * 4
    for i in (1, 2, 4, 5):
        assert 2 * s16[i] == s32[i]
    assert s16[6] == s32[6] == B * H * R * D * 2


def test_code_widths_the_library_builds():
    # 1, 2, 3 (bit planes) and 4 bits run on the GPU
    for bits, rc in ((1, 0), (2, 0), (3, 0), (4, 0), (5, ERR_UNSUPPORTED), (8, ERR_UNSUPPORTED)):
        assert _sizes(_dims(bits=bits))[0] == rc, bits


def test_three_bit_codes_are_three_planes_per_32():
    # 3 bits: 32 codes in three words, i.e. 3/8 byte per code as at 3 bits per code
    B, H, D, R, cap = 2, 3, 128, 64, 640
    rc, s = _sizes(_dims(B=B, Hkv=H, D=D, bits=3, R=R, capacity=cap))
    assert rc == 0
    u, Tq = B * H, cap - R
    assert s[0] == s[3] == u * Tq * D * 3 // 8



def test_outlier_buffer_sizes_and_refusals():
    """Dense-and-sparse variant: list sizes follow [Tq/G][D][k_out] and
    [Tq][D/Gv][v_out] (int32 index, binary32 value); the limits and the
    formats it does not support are refused before anything else."""
    B, H, D, R, cap = 2, 3, 64, 64, 640
    u, Tq = B * H, cap - R
    out = (ctypes.c_size_t * 4)()
    L = kivi.lib()
    for ko, vo in ((1, 0), (0, 2), (4, 4)):
        dims = _dims(B=B, Hkv=H, D=D, R=R, capacity=cap, k_out=ko, v_out=vo)
        assert L.kivi_outlier_buffer_sizes(ctypes.byref(dims), ctypes.byref(out)) == 0
        s = list(out)
        assert s[0] == s[1] == u * (Tq // 32) * D * ko * 4
        assert s[2] == s[3] == u * Tq * (D // 32) * vo * 4
        assert _sizes(dims)[0] == 0  # the eight plain buffers are unchanged
    for kw, rc in ((dict(k_out=5), ERR_UNSUPPORTED), (dict(v_out=-1), ERR_ARG),
                   (dict(k_out=1, meta=kivi.KIVI_META_F16), ERR_UNSUPPORTED),
                   (dict(k_out=1, bits=3), ERR_UNSUPPORTED)):
        assert _sizes(_dims(**kw))[0] == rc, kw
    # a sparse cache needs its lists bound before it is used, and the paged store refuses it
    dims = _dims(R=R, capacity=5 * R, k_out=1, v_out=1)
    ptrs = (ctypes.c_void_p * 8)(*[0x10000 * (i + 1) for i in range(8)])
    c = KiviCacheC()
    assert L.kivi_cache_init(ctypes.byref(c), ctypes.byref(dims), ctypes.byref(ptrs)) == 0
    fake = ctypes.c_void_p(0x5000)
    assert L.kivi_quantize_prefill(ctypes.byref(c), fake, fake, 10, None) == ERR_ARG
    lists = (ctypes.c_void_p * 4)(0x100000, 0x200000, 0x300000, 0x400000)
    assert L.kivi_cache_set_outliers(ctypes.byref(c), ctypes.byref(lists)) == 0
    assert (c.k_out_idx, c.v_out_val) == (0x100000, 0x400000)
    plain = _fake_cache()
    assert L.kivi_cache_set_outliers(ctypes.byref(plain), ctypes.byref(lists)) == ERR_UNSUPPORTED
    bt = ctypes.c_void_p(0x90000)
    assert L.kivi_paged_cache_init(ctypes.byref(c), ctypes.byref(dims), ctypes.byref(ptrs), bt, 4,
                                   16) == ERR_UNSUPPORTED
