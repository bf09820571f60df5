"""KIVI asymmetric 2/4-bit KV cache with fused decode attention, for NVIDIA B200.

Python binding of ``libkivi.so`` (C ABI in ``include/kivi.h``).  This module
only marshals arguments: torch supplies device memory and the current CUDA
stream; every step of the method (quantize, pack, residual window, decode
attention, split merge) runs in the library's CUDA kernels.  There is no CPU
path: if the library is missing or no CUDA device is present the calls raise.

Method: "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache"
(mlsanity.com index page, "Abstract (arXiv)"; study.space summary).
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkivi.so")

KIVI_F16, KIVI_F32 = 0, 1
KIVI_META_F32, KIVI_META_F16 = 0, 1
NUM_BUFFERS = 8
BUFFER_NAMES = ("k_codes", "k_scale", "k_zero", "v_codes", "v_scale", "v_zero", "k_res", "v_res")
STATUS = {0: "KIVI_OK", 1: "KIVI_ERR_ARG", 2: "KIVI_ERR_UNSUPPORTED", 3: "KIVI_ERR_STATE",
          4: "KIVI_ERR_CAPACITY", 5: "KIVI_ERR_WORKSPACE", 6: "KIVI_ERR_CUDA",
          7: "KIVI_ERR_SCRATCH_LIMIT"}

EXPORTED = (
    "kivi_buffer_sizes", "kivi_cache_init", "kivi_quantize_prefill", "kivi_append_token",
    "kivi_decode_workspace_bytes", "kivi_decode_attention", "kivi_decode_attention_simt",
    "kivi_set_timing_events", "kivi_decode_num_splits", "kivi_status_string",
    "kivi_decode_attention_noalloc", "kivi_append_decode", "kivi_dev_state_init",
    "kivi_append_decode_dev", "kivi_ragged_prefill", "kivi_ragged_append", "kivi_ragged_decode",
    "kivi_ragged_append_decode", "kivi_paged_buffer_sizes", "kivi_paged_cache_init",
    "kivi_outlier_buffer_sizes", "kivi_cache_set_outliers", "kivi_host_step_bytes",
    "kivi_append_decode_host",
)
OUTLIER_NAMES = ("k_out_idx", "k_out_val", "v_out_idx", "v_out_val")


class KiviError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().kivi_status_string(status).decode()}")


class KiviDims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hkv", ctypes.c_int), ("D", ctypes.c_int),
                ("bits", ctypes.c_int), ("G", ctypes.c_int), ("Gv", ctypes.c_int),
                ("R", ctypes.c_int), ("capacity", ctypes.c_longlong), ("dtype", ctypes.c_int),
                ("meta", ctypes.c_int), ("k_out", ctypes.c_int), ("v_out", ctypes.c_int)]


class KiviCacheC(ctypes.Structure):
    _fields_ = [("dims", KiviDims),
                ("k_codes", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
                ("k_zero", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
                ("v_scale", ctypes.c_void_p), ("v_zero", ctypes.c_void_p),
                ("k_res", ctypes.c_void_p), ("v_res", ctypes.c_void_p),
                ("n_q", ctypes.c_longlong), ("r", ctypes.c_int),
                ("block_table", ctypes.c_void_p), ("pages_per_seq", ctypes.c_int),
                ("num_pages", ctypes.c_longlong),
                ("k_out_idx", ctypes.c_void_p), ("k_out_val", ctypes.c_void_p),
                ("v_out_idx", ctypes.c_void_p), ("v_out_val", ctypes.c_void_p)]


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load libkivi.so (built in-tree by ``python -m bit_asymmetric_kv_quantize_b200._build``)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m bit_asymmetric_kv_quantize_b200._build`")
            L = ctypes.CDLL(LIB_PATH)
            vp, ci, ll, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t
            cp = ctypes.POINTER(KiviCacheC)
            dp = ctypes.POINTER(KiviDims)
            L.kivi_buffer_sizes.argtypes = [dp, ctypes.POINTER(sz * NUM_BUFFERS)]
            L.kivi_cache_init.argtypes = [cp, dp, ctypes.POINTER(vp * NUM_BUFFERS)]
            L.kivi_quantize_prefill.argtypes = [cp, vp, vp, ll, vp]
            L.kivi_append_token.argtypes = [cp, vp, vp, vp]
            L.kivi_decode_workspace_bytes.argtypes = [cp, ci]
            L.kivi_decode_workspace_bytes.restype = sz
            dec = [cp, vp, ci, ctypes.c_float, vp, vp, sz, vp]
            L.kivi_decode_attention.argtypes = dec
            L.kivi_decode_attention_simt.argtypes = dec
            L.kivi_decode_attention_noalloc.argtypes = [cp, vp, ci, ctypes.c_float, vp, vp]
            L.kivi_append_decode.argtypes = [cp, vp, vp, vp, ci, ctypes.c_float, vp, vp, sz, vp]
            L.kivi_host_step_bytes.argtypes = [cp, ci]
            L.kivi_host_step_bytes.restype = sz
            L.kivi_append_decode_host.argtypes = [cp, vp, ci, ctypes.c_float, vp, vp, sz, vp, sz,
                                                  vp]
            L.kivi_dev_state_init.argtypes = [cp, vp, vp]
            L.kivi_append_decode_dev.argtypes = [cp, vp, vp, vp, vp, ci, ctypes.c_float, vp, vp, sz,
                                                 vp]
            L.kivi_ragged_prefill.argtypes = [cp, vp, vp, vp, ll, vp, vp]
            L.kivi_ragged_append.argtypes = [cp, vp, vp, vp, vp]
            L.kivi_ragged_decode.argtypes = [cp, vp, vp, ci, ctypes.c_float, vp, vp, sz, vp]
            L.kivi_ragged_append_decode.argtypes = [cp, vp, vp, vp, vp, ci, ctypes.c_float, vp, vp,
                                                    sz, vp]
            L.kivi_paged_buffer_sizes.argtypes = [dp, ll, ctypes.POINTER(sz * NUM_BUFFERS)]
            L.kivi_paged_cache_init.argtypes = [cp, dp, ctypes.POINTER(vp * NUM_BUFFERS), vp, ci, ll]
            L.kivi_outlier_buffer_sizes.argtypes = [dp, ctypes.POINTER(sz * 4)]
            L.kivi_cache_set_outliers.argtypes = [cp, ctypes.POINTER(vp * 4)]
            L.kivi_set_timing_events.argtypes = [vp, vp]
            L.kivi_set_timing_events.restype = None
            L.kivi_decode_num_splits.argtypes = [cp, ci]
            L.kivi_status_string.argtypes = [ci]
            L.kivi_status_string.restype = ctypes.c_char_p
            _lib = L
        return _lib


def _dtype_code(dtype: torch.dtype) -> int:
    if dtype == torch.float16:
        return KIVI_F16
    if dtype == torch.float32:
        return KIVI_F32
    raise ValueError(f"unsupported dtype {dtype}")


def _meta_code(meta: torch.dtype) -> int:
    """Scale/zero element type: torch.float32 (binary32) or torch.float16
    (the binary16-metadata format variant, fp16 caches only)."""
    if meta == torch.float32:
        return KIVI_META_F32
    if meta == torch.float16:
        return KIVI_META_F16
    raise ValueError(f"unsupported metadata dtype {meta}")


def _code_block(bits: int):
    """(codes per block, 32-bit words per block): 32/bits codes in one word,
    or at 3 bits 32 codes as three bit-plane words (include/kivi.h)."""
    return (32, 3) if bits == 3 else (32 // bits, 1)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise KiviError(rc, what)


def buffer_sizes(B, Hkv, D, bits, capacity, R=128, G=32, Gv=32, dtype=torch.float16,
                 meta=torch.float32, outliers=(0, 0)):
    dims = KiviDims(B, Hkv, D, bits, G, Gv, R, capacity, _dtype_code(dtype), _meta_code(meta),
                    int(outliers[0]), int(outliers[1]))
    out = (ctypes.c_size_t * NUM_BUFFERS)()
    _check(lib().kivi_buffer_sizes(ctypes.byref(dims), ctypes.byref(out)), "kivi_buffer_sizes")
    return dict(zip(BUFFER_NAMES, list(out)))


class KiviCache:
    """One layer's KIVI cache on a CUDA device.

    Buffers are torch tensors in the library's ABI layout (see include/kivi.h);
    ``n_q`` / ``r`` are the library-owned counters.  Calls are asynchronous on
    torch's current stream of the cache's device.  ``meta`` is the element
    type of the scales and zeros: torch.float32, or torch.float16 for the
    binary16-metadata format variant (fp16 caches only).
    """

    def __init__(self, B: int, Hkv: int, D: int, bits: int, capacity: int, R: int = 128,
                 G: int = 32, Gv: int = 32, dtype: torch.dtype = torch.float16,
                 device="cuda", meta: torch.dtype = torch.float32, outliers=(0, 0)):
        self.device = torch.device(device)
        if self.device.type != "cuda":
            raise ValueError("KiviCache lives in CUDA device memory")
        if self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        self.dtype = dtype
        self.meta = meta
        ko, vo = (int(outliers[0]), int(outliers[1]))
        self._dims = KiviDims(B, Hkv, D, bits, G, Gv, R, capacity, _dtype_code(dtype),
                              _meta_code(meta), ko, vo)
        sizes = buffer_sizes(B, Hkv, D, bits, capacity, R, G, Gv, dtype, meta, outliers)
        self.buffers = {n: torch.empty(max(sizes[n], 16), dtype=torch.uint8, device=self.device)
                        for n in BUFFER_NAMES}
        ptrs = (ctypes.c_void_p * NUM_BUFFERS)(*[self.buffers[n].data_ptr() for n in BUFFER_NAMES])
        self._c = KiviCacheC()
        _check(lib().kivi_cache_init(ctypes.byref(self._c), ctypes.byref(self._dims),
                                     ctypes.byref(ptrs)), "kivi_cache_init")
        Tq = capacity - R
        self.outliers = (ko, vo)
        if ko or vo:  # dense-and-sparse variant: the four list buffers
            osz = (ctypes.c_size_t * 4)()
            _check(lib().kivi_outlier_buffer_sizes(ctypes.byref(self._dims), ctypes.byref(osz)),
                   "kivi_outlier_buffer_sizes")
            for n, s in zip(OUTLIER_NAMES, list(osz)):
                self.buffers[n] = torch.empty(max(s, 16), dtype=torch.uint8, device=self.device)
            optrs = (ctypes.c_void_p * 4)(*[self.buffers[n].data_ptr() for n in OUTLIER_NAMES])
            _check(lib().kivi_cache_set_outliers(ctypes.byref(self._c), ctypes.byref(optrs)),
                   "kivi_cache_set_outliers")
        self._ws: Optional[torch.Tensor] = None
        self._ws_dev: Optional[torch.Tensor] = None
        self._staging: Optional[torch.Tensor] = None
        E, WB = _code_block(bits)
        self.B, self.Hkv, self.D, self.bits, self.R, self.capacity = B, Hkv, D, bits, R, capacity
        self.shapes = {
            "k_codes": ((B, Hkv, Tq, D // E * WB), torch.int32),
            "k_scale": ((B, Hkv, Tq // G, D), meta),
            "k_zero": ((B, Hkv, Tq // G, D), meta),
            "v_codes": ((B, Hkv, Tq // E * WB, D), torch.int32),
            "v_scale": ((B, Hkv, Tq, D // Gv), meta),
            "v_zero": ((B, Hkv, Tq, D // Gv), meta),
            "k_res": ((B, Hkv, R, D), dtype),
            "v_res": ((B, Hkv, R, D), dtype),
        }
        if ko or vo:
            self.shapes.update({
                "k_out_idx": ((B, Hkv, Tq // G, D, max(ko, 1)), torch.int32),
                "k_out_val": ((B, Hkv, Tq // G, D, max(ko, 1)), torch.float32),
                "v_out_idx": ((B, Hkv, Tq, D // Gv, max(vo, 1)), torch.int32),
                "v_out_val": ((B, Hkv, Tq, D // Gv, max(vo, 1)), torch.float32),
            })

    # -- state
    @property
    def n_q(self) -> int:
        return int(self._c.n_q)

    @property
    def r(self) -> int:
        return int(self._c.r)

    def view(self, name: str) -> torch.Tensor:
        """A buffer viewed with its ABI shape (int32 for code words)."""
        shape, dt = self.shapes[name]
        n = 1
        for s in shape:
            n *= s
        return self.buffers[name][: n * torch.tensor([], dtype=dt).element_size()].view(dt).view(shape)

    def _stream(self) -> int:
        return torch.cuda.current_stream(self.device).cuda_stream

    def _arg(self, t: torch.Tensor, shape, name: str) -> int:
        if t.device != self.device or t.dtype != self.dtype or not t.is_contiguous():
            raise ValueError(f"{name}: expected a contiguous {self.dtype} tensor on {self.device}")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
        return t.data_ptr()

    # -- the three calls
    def prefill(self, K: torch.Tensor, V: torch.Tensor) -> None:
        T = K.shape[2]
        shape = (self.B, self.Hkv, T, self.D)
        pk, pv = self._arg(K, shape, "K"), self._arg(V, shape, "V")
        with torch.cuda.device(self.device):
            _check(lib().kivi_quantize_prefill(ctypes.byref(self._c), pk, pv, T, self._stream()),
                   "kivi_quantize_prefill")

    def append(self, k: torch.Tensor, v: torch.Tensor) -> None:
        shape = (self.B, self.Hkv, self.D)
        pk, pv = self._arg(k, shape, "k"), self._arg(v, shape, "v")
        with torch.cuda.device(self.device):
            _check(lib().kivi_append_token(ctypes.byref(self._c), pk, pv, self._stream()),
                   "kivi_append_token")

    def workspace_bytes(self, Hq: int) -> int:
        with torch.cuda.device(self.device):
            return int(lib().kivi_decode_workspace_bytes(ctypes.byref(self._c), Hq))

    def workspace(self, Hq: int) -> torch.Tensor:
        need = self.workspace_bytes(Hq)
        if need == 0:
            raise KiviError(1, "kivi_decode_workspace_bytes")
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        return self._ws

    def num_splits(self, Hq: int) -> int:
        with torch.cuda.device(self.device):
            return int(lib().kivi_decode_num_splits(ctypes.byref(self._c), Hq))

    def decode(self, q: torch.Tensor, softmax_scale: float, out: Optional[torch.Tensor] = None,
               kernel: str = "default") -> torch.Tensor:
        Hq = q.shape[1]
        pq = self._arg(q, (self.B, Hq, self.D), "q")
        if out is None:
            out = torch.empty_like(q)
        po = self._arg(out, (self.B, Hq, self.D), "out")
        ws = self.workspace(Hq)
        fn = lib().kivi_decode_attention if kernel == "default" else lib().kivi_decode_attention_simt
        with torch.cuda.device(self.device):
            _check(fn(ctypes.byref(self._c), pq, Hq, float(softmax_scale), po, ws.data_ptr(),
                      ws.numel(), self._stream()), "kivi_decode_attention")
        return out

    # -- device-resident counters (graph-capturable decode loop)
    def dev_state(self) -> torch.Tensor:
        """A 16-byte device tensor holding this cache's counters (n_q, r, status)."""
        st = torch.zeros(16, dtype=torch.uint8, device=self.device)
        with torch.cuda.device(self.device):
            _check(lib().kivi_dev_state_init(ctypes.byref(self._c), st.data_ptr(), self._stream()),
                   "kivi_dev_state_init")
        return st

    def load_dev_state(self, st: torch.Tensor) -> None:
        """Copy the counters from a device state back into the host struct (synchronizes)."""
        v = st.cpu()
        n_q = int(v[:8].view(torch.int64)[0])
        r, status = (int(x) for x in v[8:16].view(torch.int32))
        if status != 0:
            raise KiviError(4, "device state: cache full")
        self._c.n_q, self._c.r = n_q, r

    def append_decode_dev(self, st: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                          q: torch.Tensor, softmax_scale: float,
                          out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """append + decode with the counters in `st` (see kivi_append_decode_dev)."""
        shape = (self.B, self.Hkv, self.D)
        pk, pv = self._arg(k, shape, "k"), self._arg(v, shape, "v")
        Hq = q.shape[1]
        pq = self._arg(q, (self.B, Hq, self.D), "q")
        if out is None:
            out = torch.empty_like(q)
        po = self._arg(out, (self.B, Hq, self.D), "out")
        need = self.workspace_bytes(Hq)
        if self._ws_dev is None or self._ws_dev.numel() < need:
            self._ws_dev = torch.zeros(need, dtype=torch.uint8, device=self.device)
        ws = self._ws_dev
        with torch.cuda.device(self.device):
            _check(lib().kivi_append_decode_dev(ctypes.byref(self._c), st.data_ptr(), pk, pv, pq,
                                                Hq, float(softmax_scale), po, ws.data_ptr(),
                                                ws.numel(), self._stream()),
                   "kivi_append_decode_dev")
        return out

    def append_decode(self, k: torch.Tensor, v: torch.Tensor, q: torch.Tensor,
                      softmax_scale: float, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """append(k, v) then decode(q) in one call (one launch unless a flush is due)."""
        shape = (self.B, self.Hkv, self.D)
        pk, pv = self._arg(k, shape, "k"), self._arg(v, shape, "v")
        Hq = q.shape[1]
        pq = self._arg(q, (self.B, Hq, self.D), "q")
        if out is None:
            out = torch.empty_like(q)
        po = self._arg(out, (self.B, Hq, self.D), "out")
        ws = self.workspace(Hq)
        with torch.cuda.device(self.device):
            _check(lib().kivi_append_decode(ctypes.byref(self._c), pk, pv, pq, Hq,
                                            float(softmax_scale), po, ws.data_ptr(), ws.numel(),
                                            self._stream()), "kivi_append_decode")
        return out

    def append_decode_host(self, kvq: torch.Tensor, Hq: int, softmax_scale: float,
                           out: torch.Tensor) -> torch.Tensor:
        """kivi_append_decode_host: kvq is a host tensor (pinned for the copies
        to be asynchronous) holding k [B][Hkv][D], v [B][Hkv][D] and q
        [B][Hq][D] back to back; out a host [B][Hq][D] tensor that holds the
        result once the stream has reached the end of the call."""
        n_in = (2 * self.B * self.Hkv + self.B * Hq) * self.D
        for t, n, name in ((kvq, n_in, "kvq"), (out, self.B * Hq * self.D, "out")):
            if t.device.type != "cpu" or t.dtype != self.dtype or not t.is_contiguous() \
                    or t.numel() != n:
                raise ValueError(f"{name}: expected a contiguous host {self.dtype} tensor of {n} "
                                 "elements")
        with torch.cuda.device(self.device):
            need = int(lib().kivi_host_step_bytes(ctypes.byref(self._c), Hq))
            if need == 0:
                raise KiviError(1, "kivi_host_step_bytes")
            if self._staging is None or self._staging.numel() < need:
                self._staging = torch.empty(need, dtype=torch.uint8, device=self.device)
            ws = self.workspace(Hq)
            _check(lib().kivi_append_decode_host(ctypes.byref(self._c), kvq.data_ptr(), Hq,
                                                 float(softmax_scale), out.data_ptr(),
                                                 self._staging.data_ptr(), self._staging.numel(),
                                                 ws.data_ptr(), ws.numel(), self._stream()),
                   "kivi_append_decode_host")
        return out

    # -- ragged batches (per-sequence lengths on the device)
    def ragged_prefill(self, K: torch.Tensor, V: torch.Tensor, lens: torch.Tensor) -> torch.Tensor:
        """Prefill sequence b with its first lens[b] tokens of K[b], V[b]
        ([B][Hkv][T_max][D], padded); returns the device state (B x 16 bytes)
        that the other ragged calls take."""
        T_max = K.shape[2]
        shape = (self.B, self.Hkv, T_max, self.D)
        pk, pv = self._arg(K, shape, "K"), self._arg(V, shape, "V")
        if (lens.device != self.device or lens.dtype != torch.int64 or tuple(lens.shape) != (self.B,)
                or not lens.is_contiguous()):
            raise ValueError(f"lens: expected a contiguous int64 tensor of shape ({self.B},) on "
                             f"{self.device}")
        st = torch.zeros(16 * self.B, dtype=torch.uint8, device=self.device)
        with torch.cuda.device(self.device):
            _check(lib().kivi_ragged_prefill(ctypes.byref(self._c), st.data_ptr(), pk, pv, T_max,
                                             lens.data_ptr(), self._stream()),
                   "kivi_ragged_prefill")
        return st

    def _ragged_ws(self, Hq: int) -> torch.Tensor:
        need = self.workspace_bytes(Hq)
        if self._ws_dev is None or self._ws_dev.numel() < need:
            self._ws_dev = torch.zeros(need, dtype=torch.uint8, device=self.device)
        return self._ws_dev

    def ragged_append(self, st: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> None:
        shape = (self.B, self.Hkv, self.D)
        pk, pv = self._arg(k, shape, "k"), self._arg(v, shape, "v")
        with torch.cuda.device(self.device):
            _check(lib().kivi_ragged_append(ctypes.byref(self._c), st.data_ptr(), pk, pv,
                                            self._stream()), "kivi_ragged_append")

    def ragged_decode(self, st: torch.Tensor, q: torch.Tensor, softmax_scale: float,
                      out: Optional[torch.Tensor] = None) -> torch.Tensor:
        Hq = q.shape[1]
        pq = self._arg(q, (self.B, Hq, self.D), "q")
        if out is None:
            out = torch.empty_like(q)
        po = self._arg(out, (self.B, Hq, self.D), "out")
        ws = self._ragged_ws(Hq)
        with torch.cuda.device(self.device):
            _check(lib().kivi_ragged_decode(ctypes.byref(self._c), st.data_ptr(), pq, Hq,
                                            float(softmax_scale), po, ws.data_ptr(), ws.numel(),
                                            self._stream()), "kivi_ragged_decode")
        return out

    def ragged_append_decode(self, st: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                             q: torch.Tensor, softmax_scale: float,
                             out: Optional[torch.Tensor] = None) -> torch.Tensor:
        shape = (self.B, self.Hkv, self.D)
        pk, pv = self._arg(k, shape, "k"), self._arg(v, shape, "v")
        Hq = q.shape[1]
        pq = self._arg(q, (self.B, Hq, self.D), "q")
        if out is None:
            out = torch.empty_like(q)
        po = self._arg(out, (self.B, Hq, self.D), "out")
        ws = self._ragged_ws(Hq)
        with torch.cuda.device(self.device):
            _check(lib().kivi_ragged_append_decode(ctypes.byref(self._c), st.data_ptr(), pk, pv, pq,
                                                   Hq, float(softmax_scale), po, ws.data_ptr(),
                                                   ws.numel(), self._stream()),
                   "kivi_ragged_append_decode")
        return out


class PagedKiviCache(KiviCache):
    """A ragged-batch cache whose quantized store is pages of R tokens from a
    pool of ``num_pages`` pages, addressed through ``block_table`` (int32
    [B][pages_per_seq] on the device, owned by the caller; page l of sequence
    b is pool page block_table[b, l]).  Filled with ``ragged_prefill`` and used
    with the ragged calls only.  Pool views: ``view(name)`` gives the pool
    arrays ([num_pages][Hkv]...) and the per-sequence windows."""

    def __init__(self, B: int, Hkv: int, D: int, bits: int, pages_per_seq: int, num_pages: int,
                 block_table: torch.Tensor, R: int = 128, G: int = 32, Gv: int = 32,
                 dtype: torch.dtype = torch.float16, device="cuda",
                 meta: torch.dtype = torch.float32):
        self.device = torch.device(device)
        if self.device.type != "cuda":
            raise ValueError("PagedKiviCache lives in CUDA device memory")
        if self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        if (block_table.device != self.device or block_table.dtype != torch.int32
                or tuple(block_table.shape) != (B, pages_per_seq) or not block_table.is_contiguous()):
            raise ValueError(f"block_table: expected a contiguous int32 tensor of shape "
                             f"({B}, {pages_per_seq}) on {self.device}")
        capacity = (pages_per_seq + 1) * R
        self.dtype, self.meta = dtype, meta
        self.block_table = block_table
        self.pages_per_seq, self.num_pages = pages_per_seq, num_pages
        self._dims = KiviDims(B, Hkv, D, bits, G, Gv, R, capacity, _dtype_code(dtype),
                              _meta_code(meta))
        out = (ctypes.c_size_t * NUM_BUFFERS)()
        _check(lib().kivi_paged_buffer_sizes(ctypes.byref(self._dims), num_pages, ctypes.byref(out)),
               "kivi_paged_buffer_sizes")
        sizes = dict(zip(BUFFER_NAMES, list(out)))
        self.buffers = {n: torch.empty(max(sizes[n], 16), dtype=torch.uint8, device=self.device)
                        for n in BUFFER_NAMES}
        ptrs = (ctypes.c_void_p * NUM_BUFFERS)(*[self.buffers[n].data_ptr() for n in BUFFER_NAMES])
        self._c = KiviCacheC()
        _check(lib().kivi_paged_cache_init(ctypes.byref(self._c), ctypes.byref(self._dims),
                                           ctypes.byref(ptrs), block_table.data_ptr(),
                                           pages_per_seq, num_pages), "kivi_paged_cache_init")
        self._ws: Optional[torch.Tensor] = None
        self._ws_dev: Optional[torch.Tensor] = None
        E, WB = _code_block(bits)
        self.B, self.Hkv, self.D, self.bits, self.R, self.capacity = B, Hkv, D, bits, R, capacity
        P = num_pages
        self.shapes = {
            "k_codes": ((P, Hkv, R, D // E * WB), torch.int32),
            "k_scale": ((P, Hkv, R // G, D), meta),
            "k_zero": ((P, Hkv, R // G, D), meta),
            "v_codes": ((P, Hkv, R // E * WB, D), torch.int32),
            "v_scale": ((P, Hkv, R, D // Gv), meta),
            "v_zero": ((P, Hkv, R, D // Gv), meta),
            "k_res": ((B, Hkv, R, D), dtype),
            "v_res": ((B, Hkv, R, D), dtype),
        }


def ragged_lengths(st: torch.Tensor):
    """(n_q, r, status) lists of a ragged device state (copies it to the host)."""
    v = st.cpu().view(torch.int64).view(-1, 2)
    n_q = v[:, 0].tolist()
    rs = v[:, 1].contiguous().view(torch.int32).view(-1, 2)
    return n_q, rs[:, 0].tolist(), rs[:, 1].tolist()


def set_timing_events(start: Optional[torch.cuda.Event], stop: Optional[torch.cuda.Event]) -> None:
    """Have later decode calls on this thread record these events around the split kernel."""
    lib().kivi_set_timing_events(start.cuda_event if start is not None else None,
                                 stop.cuda_event if stop is not None else None)
