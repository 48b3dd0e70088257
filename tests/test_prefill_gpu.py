"""Prefill parity on the GPU: the CUDA path through the C ABI against the CPU
oracle (all rows for small shapes, sampled rows at full size)."""
import numpy as np
import pytest
import torch

import workloads
from gpu_common import check_prefill

pytestmark = pytest.mark.gpu


def _sample_rows(w, count, seed):
    rng = np.random.default_rng(seed)
    rows = set()
    for i in [0, 1, w.W - 1, w.W, w.W + 1, w.W + w.k, w.W + w.k + 1, w.n - 1]:
        if 0 <= i < w.n:
            rows.add((0, 0, i))
            rows.add((w.B - 1, w.Hq - 1, i))
    while len(rows) < count:
        rows.add((int(rng.integers(w.B)), int(rng.integers(w.Hq)),
                  int(rng.integers(w.n))))
    return np.array(sorted(rows), dtype=np.int64)


def test_tiny_prefill_f32():
    """The tiny fp32 prefill workload, every row."""
    w = workloads.get("tiny_prefill_f32")
    print(check_prefill(w, workloads.generate(w)))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n,W,k", [
    (1, 1, 0), (2, 1, 1), (64, 64, 32), (65, 64, 32), (97, 64, 32),
    (200, 1, 16), (300, 300, 8), (333, 7, 64), (1000, 64, 32), (777, 3, 1),
])
def test_prefill_edges(dtype, d, n, W, k):
    w = workloads.get("prefill_gpt2s_8k").scaled(
        dtype=dtype, d=d, n=n, W=W, k=k, B=2, Hq=4, Hkv=2, needles=2,
        needle_gap=W)
    print(check_prefill(w, workloads.generate(w)))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n,W,k", [(2048, 256, 128), (700, 64, 100),
                                   (130, 1, 128)])
def test_prefill_k_up_to_128(dtype, d, n, W, k):
    # the largest prefill Top-k (the 1M decode config's k = 128): most rows
    # hold more candidates than the tensor-core selector's segments and take
    # the exact fallback, which the check includes
    w = workloads.get("prefill_gpt2s_8k").scaled(
        dtype=dtype, d=d, n=n, W=W, k=k, B=1, Hq=2, Hkv=1, needles=4,
        needle_gap=128)
    print(check_prefill(w, workloads.generate(w)))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_prefill_gqa_groups(dtype):
    w = workloads.get("prefill_gpt2s_8k").scaled(
        dtype=dtype, n=700, B=1, Hq=8, Hkv=1, needles=4)
    print(check_prefill(w, workloads.generate(w)))


def test_prefill_gpt2s_small_all_rows():
    w = workloads.get("prefill_gpt2s_8k").scaled(n=1536, B=2, Hq=3, Hkv=3)
    print(check_prefill(w, workloads.generate(w)))


def test_prefill_adaptive_small_all_rows():
    w = workloads.get("prefill_adaptive_32k").scaled(n=2048, Hq=2, Hkv=2)
    x = workloads.generate(w)
    print(check_prefill(w, x, W_i=x["W_i"]))


def test_prefill_bf16_output():
    w = workloads.get("prefill_gpt2s_8k").scaled(n=600, B=1, Hq=2, Hkv=2)
    print(check_prefill(w, workloads.generate(w), o_dtype=torch.bfloat16,
                        tol=1e-2 + 2.0 ** -6))


def test_prefill_gpt2s_8k_all_rows():
    """The GPT-2-small 8K prefill workload at full size, every one of its
    393,216 rows (and any row that took the exact fallback among them)."""
    w = workloads.get("prefill_gpt2s_8k")
    x = workloads.generate(w)
    print(check_prefill(w, x, with_fallback_rows=True))


def test_prefill_adaptive_32k_sampled():
    """The adaptive-window 32K prefill workload at full size: 20,000 sampled
    rows plus every row the selector sent to the exact fallback."""
    w = workloads.get("prefill_adaptive_32k")
    x = workloads.generate(w)
    print(check_prefill(w, x, W_i=x["W_i"], sel=_sample_rows(w, 20000, 1),
                        with_fallback_rows=True))


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_beyond_262144(d):
    """A sequence longer than 2^18 positions (positions are 32-bit in the
    selector's entries): 600 sampled rows, spread over the length, plus every
    row sent to the exact fallback."""
    w = workloads.get("prefill_gpt2s_8k").scaled(
        d=d, n=300000, B=1, Hq=1, Hkv=1, W=64, k=32, needles=8)
    x = workloads.generate(w)
    sel = _sample_rows(w, 600, 7)
    sel = np.unique(np.concatenate(
        [sel, np.array([[0, 0, i] for i in (262143, 262144, 262145, 299999)],
                       dtype=np.int64)]), axis=0)
    print(check_prefill(w, x, sel=sel, with_fallback_rows=True))


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_equal_keys_take_the_fallback(d):
    """All keys equal: every candidate ties at the pass-1 bound, so rows with
    more candidates than the row buffer holds go through the exact fallback;
    ties go to the lowest indices."""
    w = workloads.get("prefill_gpt2s_8k").scaled(d=d, n=700, B=1, Hq=2, Hkv=2,
                                                 needles=0)
    x = workloads.generate(w)
    x["K"][:] = x["K"][:, :, :1, :]
    print(check_prefill(w, x))


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_fallback_spans_chunks(d):
    """K rows at three levels (0.5, 1 and 2 times one row, exact in bf16):
    rows past position 128 + W tie on more candidates than the row buffer
    holds and go through the exact fallback, which then scores several
    2048-key chunks with keys both above and below its running threshold.
    Rows with q.k_0 > 0 pick the 2x rows, rows with q.k_0 < 0 the 0.5x rows
    (about half of each); ties go to the lowest indices."""
    w = workloads.get("prefill_gpt2s_8k").scaled(d=d, n=5000, B=1, Hq=2,
                                                 Hkv=1, needles=0)
    x = workloads.generate(w)
    K = x["K"]
    K[:] = K[:, :, :1, :]
    j = np.arange(w.n)
    c = np.where(j < 3000, 0.5, np.where(j < 4200, 1.0, 2.0))
    K *= c.astype(K.dtype)[None, None, :, None]
    print(check_prefill(w, x))
