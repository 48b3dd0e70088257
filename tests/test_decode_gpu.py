"""Decode parity on the GPU: the CUDA path through the C ABI against the CPU
oracle, element by element (index sets bit-exact outside counted near-ties,
outputs within 1e-5 for fp32 inputs and 1e-2 for bf16 inputs)."""
import numpy as np
import pytest
import torch

import workloads
from gpu_common import check_decode

pytestmark = pytest.mark.gpu

BASE = workloads.get("decode_131k")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 4), (32, 8), (8, 1)])
def test_decode_shapes(dtype, d, Hq, Hkv):
    w = BASE.scaled(dtype=dtype, d=d, Hq=Hq, Hkv=Hkv, n=9001, W=128, k=64,
                    needles=16, B=2)
    print(check_decode(w, workloads.generate(w)))


@pytest.mark.parametrize("L,W,k", [
    (1, 1, 0), (1, 1, 8), (2, 1, 1), (3, 1, 5), (130, 128, 64), (200, 128, 64),
    (193, 128, 64), (194, 128, 64), (1000, 1, 0), (1000, 1000, 16),
    (1000, 5000, 4), (4097, 7, 300), (5000, 16, 1024), (70000, 64, 1),
])
def test_decode_edges(L, W, k):
    w = BASE.scaled(n=L, W=W, k=k, Hq=8, Hkv=2, needles=min(8, max(0, L - 1 - W)))
    print(check_decode(w, workloads.generate(w)))


def test_decode_per_batch_window():
    w = BASE.scaled(n=20000, B=4, Hq=8, Hkv=2, needles=8)
    x = workloads.generate(w)
    W_i = np.array([64, 1, 256, 19999], dtype=np.int32)
    print(check_decode(w, x, W_i=W_i))


def test_decode_bf16_output():
    w = BASE.scaled(n=12345, Hq=8, Hkv=2, needles=8)
    x = workloads.generate(w)
    # bf16 output adds one rounding of |o| < 8: half an ulp is at most 2^-6
    print(check_decode(w, x, o_dtype=torch.bfloat16, tol=1e-2 + 2.0 ** -6))


def test_decode_131k():
    """The 131K-context decode workload at full size."""
    w = workloads.get("decode_131k")
    print(check_decode(w, workloads.generate(w)))


def test_decode_1m():
    """The 1M-context decode workload at full size."""
    w = workloads.get("decode_1m")
    print(check_decode(w, workloads.generate(w)))
