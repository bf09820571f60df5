"""Seeded synthetic inputs for the KIVI cache: shapes, distributions, draw order.

This module holds no quantization or attention arithmetic.  It is the one
piece of Python that both the CUDA-path tests and the CPU oracle consume, so
that both see bit-identical inputs.

Distributions stand in for the pages' real LLM workloads (Llama-2 / Mistral
shaped attention layers; no datasets or weights are used):
  K ~ N(0, 1) with a fixed set of outlier channels per KV head scaled x20
    (the KIVI abstract's finding that a few key channels carry large
    magnitudes), the same channels for every batch element and token;
  V ~ N(0, 1) (no outlier pattern in values);
  q ~ N(0, 1) / sqrt(D).
Values are drawn in float32 from a seeded torch generator on the target
device and cast to the workload dtype with round-to-nearest-even.
Ragged batches (len_min > 0): sequence lengths uniform in [len_min, T]
(seeded), with the first sequence at T and the second at len_min, standing
in for a serving batch's mix of prompt lengths.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple

import torch

_TAG = {"outlier": 1, "kv": 2, "q": 3, "step_kv": 4, "step_q": 5, "lens": 6}


def _seed(base: int, tag: str, *idx: int) -> int:
    s = (base * 1_000_003 + _TAG[tag] * 7919) & 0x7FFFFFFFFFFF
    for i in idx:
        s = (s * 131_071 + i + 1) & 0x7FFFFFFFFFFF
    return s


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    T: int              # prompt tokens quantized by prefill
    bits: int
    G: int = 32
    Gv: int = 32
    R: int = 128
    dtype: str = "f16"  # "f16" or "f32"
    meta: str = "f32"   # scale/zero storage: "f32", or "f16" (binary16 variant, f16 caches)
    steps: int = 0      # decode steps, each appending one token, after prefill
    len_min: int = 0    # > 0: ragged batch, prompt lengths in [len_min, T] (T is the longest)
    outlier_channels: Optional[Tuple[int, ...]] = None  # fixed set, else 4 random per head
    n_outliers: int = 4
    outlier_scale: float = 20.0
    seed: int = 0
    spike_frac: float = 0.0    # > 0: that fraction of single K and V entries scaled by spike_scale
    spike_scale: float = 40.0  # (entry outliers, the case dense-and-sparse groups keep exactly)

    @property
    def torch_dtype(self):
        return torch.float16 if self.dtype == "f16" else torch.float32

    @property
    def torch_meta(self):
        return torch.float16 if self.meta == "f16" else torch.float32

    @property
    def gq(self) -> int:
        return self.Hq // self.Hkv

    @property
    def capacity(self) -> int:
        """Smallest multiple of R holding the prompt plus every decode-step token."""
        total = self.T + self.steps
        return max(self.R, -(-total // self.R) * self.R)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The workloads: a tiny parity case, attention-layer shapes, and a ragged batch.
TINY = Workload("tiny-b1h1d32-t256-f32", B=1, Hq=1, Hkv=1, D=32, T=256, bits=2, G=32, Gv=32,
                R=32, dtype="f32", outlier_channels=(3, 17))
LLAMA2_7B = Workload("llama2-7b-decode-b8h32d128-t4096", B=8, Hq=32, Hkv=32, D=128, T=4096, bits=2)
MISTRAL_7B = Workload("mistral-7b-gqa-b16hq32hkv8d128-t16384", B=16, Hq=32, Hkv=8, D=128,
                      T=16384, bits=2)
STREAMING = Workload("streaming-b4h32d128-prompt32768-512steps", B=4, Hq=32, Hkv=32, D=128,
                     T=32768, bits=2, steps=512)
LLAMA2_13B_2BIT = Workload("llama2-13b-b64h40d128-t8192-2bit", B=64, Hq=40, Hkv=40, D=128,
                           T=8192, bits=2)
LLAMA2_13B_4BIT = LLAMA2_13B_2BIT.with_(name="llama2-13b-b64h40d128-t8192-4bit", bits=4)
RAGGED = Workload("ragged-b32h32d128-len256-8192", B=32, Hq=32, Hkv=32, D=128, T=8192, bits=2,
                  len_min=256)

ALL = {w.name: w for w in (TINY, LLAMA2_7B, MISTRAL_7B, STREAMING, LLAMA2_13B_2BIT, LLAMA2_13B_4BIT,
                           RAGGED)}


def seq_lengths(w: Workload) -> torch.Tensor:
    """Prompt length of every sequence (int64 [B], CPU): T for a uniform
    batch; for a ragged one uniform in [len_min, T], sequence 0 at T and
    sequence 1 at len_min."""
    if w.len_min <= 0:
        return torch.full((w.B,), w.T, dtype=torch.int64)
    lens = torch.randint(w.len_min, w.T + 1, (w.B,), generator=_gen(_seed(w.seed, "lens")),
                         dtype=torch.int64)
    lens[0] = w.T
    if w.B > 1:
        lens[1] = w.len_min
    return lens


def outlier_channels(w: Workload, h: int) -> torch.Tensor:
    """The fixed outlier key channels of KV head h (same for every sequence and token)."""
    if w.outlier_channels is not None:
        return torch.tensor(w.outlier_channels, dtype=torch.long)
    return torch.randperm(w.D, generator=_gen(_seed(w.seed, "outlier", h)))[: w.n_outliers]


def key_channel_scale(w: Workload) -> torch.Tensor:
    """[Hkv][D] multiplier: outlier_scale on each head's outlier channels, else 1."""
    m = torch.ones(w.Hkv, w.D, dtype=torch.float32)
    for h in range(w.Hkv):
        m[h, outlier_channels(w, h)] = w.outlier_scale
    return m


def _device_gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def prompt_kv(w: Workload, T: Optional[int] = None, device="cpu"):
    """Prompt keys and values [B][Hkv][T][D] in the workload dtype.

    Drawn in float32 one sequence at a time from one generator on `device`
    (CPU: torch's CPU generator; CUDA: torch's Philox generator), so the
    values depend on the device; the oracle is always given the very tensor
    the library was given, copied to the host."""
    T = w.T if T is None else T
    device = torch.device(device)
    g = _device_gen(device, _seed(w.seed, "kv"))
    mult = key_channel_scale(w).to(device)[:, None, :]
    K = torch.empty(w.B, w.Hkv, T, w.D, dtype=w.torch_dtype, device=device)
    V = torch.empty_like(K)
    for b in range(w.B):
        k = torch.randn(w.Hkv, T, w.D, generator=g, dtype=torch.float32, device=device)
        v = torch.randn(w.Hkv, T, w.D, generator=g, dtype=torch.float32, device=device)
        if w.spike_frac > 0:
            k = _spikes(w, k, g)
            v = _spikes(w, v, g)
        K[b].copy_(k * mult)
        V[b].copy_(v)
    return K, V


def _spikes(w: Workload, x: torch.Tensor, g: torch.Generator) -> torch.Tensor:
    """x with a seeded random fraction w.spike_frac of its entries scaled by w.spike_scale."""
    m = torch.rand(x.shape, generator=g, dtype=torch.float32, device=x.device) < w.spike_frac
    return torch.where(m, x * w.spike_scale, x)


def query(w: Workload, step: int = -1, device="cpu") -> torch.Tensor:
    """q [B][Hq][D] for the decode after the prompt (step -1) or at decode step `step`."""
    tag, idx = ("q", ()) if step < 0 else ("step_q", (step,))
    g = _device_gen(device, _seed(w.seed, tag, *idx))
    q = torch.randn(w.B, w.Hq, w.D, generator=g, dtype=torch.float32, device=device)
    return (q / math.sqrt(w.D)).to(w.torch_dtype)


def step_kv(w: Workload, step: int, device="cpu"):
    """The token appended at decode step `step`: (k, v) [B][Hkv][D]."""
    g = _device_gen(device, _seed(w.seed, "step_kv", step))
    k = torch.randn(w.B, w.Hkv, w.D, generator=g, dtype=torch.float32, device=device)
    v = torch.randn(w.B, w.Hkv, w.D, generator=g, dtype=torch.float32, device=device)
    if w.spike_frac > 0:
        k = _spikes(w, k, g)
        v = _spikes(w, v, g)
    k = k * key_channel_scale(w).to(device)[None]
    return k.to(w.torch_dtype), v.to(w.torch_dtype)
