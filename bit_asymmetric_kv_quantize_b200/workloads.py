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
Every (batch element, KV head) unit is drawn from its own torch CPU
generator, so any unit of a full-size workload can be regenerated alone, bit
for bit, for sampled oracle checks.  Values are drawn in float32 and cast to
the workload dtype with round-to-nearest-even.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple

import torch

_TAG = {"outlier": 1, "kv": 2, "q": 3, "step_kv": 4, "step_q": 5}


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
    steps: int = 0      # decode steps, each appending one token, after prefill
    outlier_channels: Optional[Tuple[int, ...]] = None  # fixed set, else 4 random per head
    n_outliers: int = 4
    outlier_scale: float = 20.0
    seed: int = 0

    @property
    def torch_dtype(self):
        return torch.float16 if self.dtype == "f16" else torch.float32

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


# The five workloads: a tiny parity case and four attention-layer shapes.
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

ALL = {w.name: w for w in (TINY, LLAMA2_7B, MISTRAL_7B, STREAMING, LLAMA2_13B_2BIT, LLAMA2_13B_4BIT)}


def outlier_channels(w: Workload, h: int) -> torch.Tensor:
    if w.outlier_channels is not None:
        return torch.tensor(w.outlier_channels, dtype=torch.long)
    return torch.randperm(w.D, generator=_gen(_seed(w.seed, "outlier", h)))[: w.n_outliers]


def unit_kv(w: Workload, b: int, h: int, T: Optional[int] = None):
    """Prompt keys and values of one unit: (K [T][D], V [T][D]) in the workload dtype."""
    T = w.T if T is None else T
    g = _gen(_seed(w.seed, "kv", b, h))
    K = torch.randn(T, w.D, generator=g, dtype=torch.float32)
    V = torch.randn(T, w.D, generator=g, dtype=torch.float32)
    K[:, outlier_channels(w, h)] *= w.outlier_scale
    return K.to(w.torch_dtype), V.to(w.torch_dtype)


def prompt_kv(w: Workload, T: Optional[int] = None, device="cpu"):
    """Whole prompt: (K, V) [B][Hkv][T][D] in the workload dtype, unit by unit."""
    T = w.T if T is None else T
    K = torch.empty(w.B, w.Hkv, T, w.D, dtype=w.torch_dtype, device=device)
    V = torch.empty_like(K)
    for b in range(w.B):
        for h in range(w.Hkv):
            k, v = unit_kv(w, b, h, T)
            K[b, h].copy_(k)
            V[b, h].copy_(v)
    return K, V


def query(w: Workload, step: int = -1) -> torch.Tensor:
    """q [B][Hq][D] for the decode after the prompt (step -1) or after decode step `step`."""
    tag, idx = ("q", ()) if step < 0 else ("step_q", (step,))
    g = _gen(_seed(w.seed, tag, *idx))
    q = torch.randn(w.B, w.Hq, w.D, generator=g, dtype=torch.float32) / math.sqrt(w.D)
    return q.to(w.torch_dtype)


def step_kv(w: Workload, step: int):
    """The token appended at decode step `step`: (k, v) [B][Hkv][D]."""
    g = _gen(_seed(w.seed, "step_kv", step))
    k = torch.randn(w.B, w.Hkv, w.D, generator=g, dtype=torch.float32)
    v = torch.randn(w.B, w.Hkv, w.D, generator=g, dtype=torch.float32)
    for h in range(w.Hkv):
        k[:, h, outlier_channels(w, h)] *= w.outlier_scale
    return k.to(w.torch_dtype), v.to(w.torch_dtype)
