"""The benchmark's host-side arithmetic, without a GPU: the algorithmic bytes
a decode call must move (the roofline's numerator) for each format, the
workload variants the command line selects, and the ragged length mix."""
import argparse

import pytest
import torch

import bench
from bit_asymmetric_kv_quantize_b200 import workloads as W


def test_algorithmic_bytes_of_the_7b_layer_by_hand():
    w = W.LLAMA2_7B  # B 8, 32 KV heads, D 128, 2-bit, fp16, binary32 metadata
    n_q, r = 3968, 128
    per_unit = (n_q * 128 * 2 // 8      # key codes
                + (n_q // 32) * 128 * 8  # key scale + zero (binary32)
                + n_q * 128 * 2 // 8     # value codes
                + n_q * 4 * 8            # value scale + zero per 32-channel group
                + r * 128 * 2 * 2)       # window K and V, fp16
    io = 2 * 8 * 32 * 128 * 2            # q in, out
    assert bench.algorithmic_bytes(w, n_q, r) == 8 * 32 * per_unit + io
    # 128 bytes of codes and metadata per quantized token of one head
    assert per_unit - r * 512 == n_q * 128


@pytest.mark.parametrize("bits,meta,per_token", [(2, "f32", 128), (2, "f16", 96), (4, "f32", 192),
                                                 (4, "f16", 160), (1, "f32", 96), (1, "f16", 64)])
def test_bytes_per_quantized_token_by_format(bits, meta, per_token):
    w = W.LLAMA2_7B.with_(bits=bits, meta=meta)
    a = bench.algorithmic_bytes(w, 4096, 1)
    b = bench.algorithmic_bytes(w, 4096 + 32, 1)
    assert (b - a) == 32 * per_token * w.B * w.Hkv


def test_ragged_bytes_sum_over_sequences():
    w = W.RAGGED
    nq = [0, 128, 4096] + [256] * (w.B - 3)
    r = [5, 128, 1] + [64] * (w.B - 3)
    total = bench.algorithmic_bytes(w, nq, r)
    uni = [bench.algorithmic_bytes(w.with_(B=1, Hq=w.gq * w.Hkv), a, b) for a, b in zip(nq, r)]
    io_one = 2 * w.Hq * w.D * 2
    assert total == sum(u - io_one for u in uni) + w.B * io_one


def test_workload_variants_from_the_command_line():
    def args(**kw):
        d = dict(workload=W.LLAMA2_7B.name, meta="f32", bits=None, outliers="0,0")
        d.update(kw)
        return argparse.Namespace(**d)

    assert bench.bench_workload(args()) == W.LLAMA2_7B
    w = bench.bench_workload(args(meta="f16", bits=1))
    assert (w.meta, w.bits) == ("f16", 1) and w.name.endswith("-meta16-1bit")
    s = bench.bench_workload(args(workload=W.STREAMING.name))
    assert s.steps == 0 and s.T == W.STREAMING.T
    sp = bench.bench_workload(args(outliers="1,1"))
    assert sp.spike_frac > 0 and sp.name.endswith("-sparse1x1")
    # the kept entries' lists count in the algorithmic bytes: 8 bytes per entry
    w = W.LLAMA2_7B
    extra = bench.algorithmic_bytes(w, 4096, 0, (1, 1)) - bench.algorithmic_bytes(w, 4096, 0)
    assert extra == w.B * w.Hkv * 8 * ((4096 // 32) * w.D + 4096 * (w.D // 32))
    t3 = bench.bench_workload(args(workload=W.LLAMA2_13B_2BIT.name, bits=3))
    assert t3.name == "llama2-13b-b64h40d128-t8192-3bit"


def test_ragged_lengths_are_seeded_and_span_the_range():
    w = W.RAGGED
    a, b = W.seq_lengths(w), W.seq_lengths(w)
    assert torch.equal(a, b) and a.dtype == torch.int64 and a.shape == (w.B,)
    assert int(a.max()) == w.T and int(a.min()) == w.len_min
    assert torch.all(W.seq_lengths(W.LLAMA2_7B) == W.LLAMA2_7B.T)


def test_replica_throughput():
    assert bench.replica_throughput(4, 8, 100, 50.0) == 4 * 8 * 100 / 0.05
