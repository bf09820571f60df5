"""The dense-and-sparse group quantizer of csrc/kivi_sparse.cuh (one group
held by one thread, as the quantize kernels will hold it), built for the
host and compared bit for bit with the oracle's pinned group quantizer:
outlier selection with its tie rule, scale, zero, codes (through the
kernels' code rule) and the outlier lists."""
import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_asymmetric_kv_quantize_b200", "csrc")

HARNESS = r'''
#include "kivi_sparse.cuh"
extern "C" void t_group(const float* x, int k, int bits, float* s, float* z, int* codes,
                        int* idx, float* val) {
  float xs[32];
  int c[32], oi[4];
  float ov[4];
  for (int i = 0; i < 32; ++i) xs[i] = x[i];
  kivi::quantize_group_sparse<32, 4>(xs, k, bits, s, z, c, oi, ov);
  for (int i = 0; i < 32; ++i) codes[i] = c[i];
  for (int m = 0; m < k; ++m) {
    idx[m] = oi[m];
    val[m] = ov[m];
  }
}
// the register-resident form the prompt and append kernels run
extern "C" void t_group_reg(const float* x, int k, int bits, float* s, float* z, int* codes,
                            int* idx, float* val) {
  float xs[32];
  int c[32], oi[4];
  float ov[4];
  for (int i = 0; i < 32; ++i) xs[i] = x[i];
  kivi::quantize_group_sparse_reg<32, 4>(xs, k, bits, s, z, c, oi, ov);
  for (int i = 0; i < 32; ++i) codes[i] = c[i];
  for (int m = 0; m < k; ++m) {
    idx[m] = oi[m];
    val[m] = ov[m];
  }
}
'''


@pytest.fixture(scope="module")
def group_lib(tmp_path_factory):
    cxx = shutil.which("g++")
    if not cxx:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp("sparse_rule")
    src = d / "harness.cpp"
    src.write_text(HARNESS)
    so = d / "libgroup.so"
    subprocess.run([cxx, "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                    "-shared", "-I", CSRC, "-o", str(so), str(src)], check=True)
    L = ctypes.CDLL(str(so))
    for f in (L.t_group, L.t_group_reg):
        f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    return L


def run(lib, x, k, bits, fn="t_group"):
    x = np.ascontiguousarray(x, np.float32)
    s, z = np.zeros(1, np.float32), np.zeros(1, np.float32)
    c = np.zeros(32, np.int32)
    oi, ov = np.zeros(4, np.int32), np.zeros(4, np.float32)
    getattr(lib, fn)(x.ctypes.data, k, bits, s.ctypes.data, z.ctypes.data, c.ctypes.data,
                     oi.ctypes.data, ov.ctypes.data)
    return s[0], z[0], c, oi[:k], ov[:k]


@pytest.mark.parametrize("fn", ["t_group", "t_group_reg"])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("k", [0, 1, 2, 4])
def test_matches_the_oracle_bit_for_bit(group_lib, bits, k, fn):
    rng = np.random.default_rng(bits * 10 + k)
    for trial in range(3000):
        x = rng.standard_normal(32).astype(np.float32) * np.float32(10.0 ** rng.uniform(-6, 6))
        if trial % 3 == 0:
            x[rng.integers(0, 32, 3)] *= 50        # planted outliers
        if trial % 4 == 0:
            x[:16] = np.round(x[:16])              # equal magnitudes and signed zeros
            x[3] = -x[5]
        if trial % 7 == 0:
            x[:] = x[0]                            # a constant group: scale 0
        s, z, c, oi, ov = run(group_lib, x, k, bits, fn)
        s0, z0, c0, oi0, ov0 = oracle.quantize_group_sparse(x, bits, k)
        assert np.float32(s).view(np.uint32) == np.float32(s0).view(np.uint32)
        assert np.float32(z).view(np.uint32) == np.float32(z0).view(np.uint32)
        assert c.tolist() == c0.tolist()
        assert oi.tolist() == oi0.tolist()
        assert ov.view(np.uint32).tolist() == ov0.view(np.uint32).tolist()


def test_device_build_compiles(tmp_path):
    """The same header in a kernel for sm_100a (cross-compiled; no GPU)."""
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    src = tmp_path / "k.cu"
    src.write_text(r'''
#include "kivi_sparse.cuh"
__global__ void k(const float* x, int kk, int bits, float* out, int* codes) {
  float xs[32];
  for (int i = 0; i < 32; ++i) xs[i] = x[threadIdx.x * 32 + i];
  int c[32], oi[4];
  float ov[4], s, z;
  kivi::quantize_group_sparse<32, 4>(xs, kk, bits, &s, &z, c, oi, ov);
  float s2, z2;
  kivi::quantize_group_sparse_reg<32, 4>(xs, kk, bits, &s2, &z2, c, oi, ov);
  out[threadIdx.x] = s + z + ov[0] + s2 + z2;
  for (int i = 0; i < 32; ++i) codes[threadIdx.x * 32 + i] = c[i] + oi[i & 3];
}
''')
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-c", "-I",
                    CSRC, "-o", str(tmp_path / "k.o"), str(src)], check=True)
