"""The CA_DEBUG build (libcondensate_attn_debug.so): the same entry points as
the release library, with kernels that also check the indexes the release
build keeps in range by construction and report CA_ERR_BOUNDS instead of a
memory fault.

Host checks (no GPU): it builds, exports every declared entry point, reports
itself as the debug build and rejects invalid arguments like the release
library.  GPU checks: parity cases that reach every checked site (the
prefill selector's segments and spare segments, the exact fallback list, the
decode lists under the claimed-unit stream, the merge's survivor slots and
its radix path) run through the debug library; each asserts the status word
is clean (no index check failed) and the results match the oracle."""
import pytest

import workloads
from sparse_transformer_attention_b200 import binding
from test_abi_host import _decode, _prefill, header_functions


@pytest.fixture(scope="module")
def dlib():
    from sparse_transformer_attention_b200 import build
    return binding.load(build.build(debug=True))


def test_debug_library_exports_every_declared_symbol(dlib):
    for name in header_functions():
        assert hasattr(dlib, name), name
    assert dlib.condensate_attn_build_flags() == 1  # CA_BUILD_DEBUG
    assert dlib.condensate_attn_version() == binding.load().condensate_attn_version()
    assert dlib.condensate_attn_status_string(
        binding.CA_ERR_BOUNDS).decode().startswith("index check")


@pytest.mark.parametrize("call,over,code", [
    (_decode, {"q": 0}, binding.CA_ERR_INVALID_ARG),
    (_decode, {"d": 96}, binding.CA_ERR_UNSUPPORTED),
    (_decode, {"V": (1 << 20) + 8}, binding.CA_ERR_ALIGNMENT),
    (_decode, {}, binding.CA_ERR_WORKSPACE),
    (_prefill, {"Q": 0}, binding.CA_ERR_INVALID_ARG),
    (_prefill, {"k": 129, "C_max": 1 + 64 + 129}, binding.CA_ERR_UNSUPPORTED),
    (_prefill, {}, binding.CA_ERR_WORKSPACE),
])
def test_debug_library_rejects_invalid_arguments(dlib, call, over, code):
    assert call(dlib, **over) == code


@pytest.fixture
def debug_calls(dlib):
    """Route the package's calls through the debug library for one test."""
    prev = binding.use_library(binding.DEBUG_LIB_PATH)
    try:
        assert binding.load().condensate_attn_build_flags() == 1
        yield
    finally:
        binding.use_library(prev)


PREFILL_CASES = [
    # (dtype, d, n, W, k): k <= 32 takes the column-pair slots; k = 64 the
    # 256-slot table; k = 128 sends most rows to the exact fallback list;
    # n = 3000 spans 24 key tiles with a ragged last one
    ("bf16", 64, 3000, 64, 32),
    ("bf16", 64, 2048, 256, 64),
    ("bf16", 128, 1500, 64, 64),
    ("bf16", 64, 2048, 256, 128),
    ("f32", 64, 1000, 64, 32),
]


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,d,n,W,k", PREFILL_CASES)
def test_debug_prefill_index_checks_clean(debug_calls, dtype, d, n, W, k):
    from gpu_common import check_prefill
    w = workloads.get("prefill_gpt2s_8k").scaled(
        dtype=dtype, d=d, n=n, W=W, k=k, B=1, Hq=4, Hkv=2, needles=4,
        needle_gap=128)
    print(check_prefill(w, workloads.generate(w)))


DECODE_CASES = [
    # (dtype, L, W, k, Hq, Hkv): a 70K cache streams many claimed units per
    # group; k = 1024 takes the merge's radix path; G = 8 heads per group
    ("bf16", 70000, 128, 64, 8, 4),
    ("bf16", 20000, 64, 1024, 4, 4),
    ("bf16", 9001, 128, 64, 8, 1),
    ("f32", 9001, 128, 64, 8, 4),
]


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,L,W,k,Hq,Hkv", DECODE_CASES)
def test_debug_decode_index_checks_clean(debug_calls, dtype, L, W, k, Hq, Hkv):
    from gpu_common import check_decode
    w = workloads.get("decode_131k").scaled(
        dtype=dtype, n=L, W=W, k=k, B=2, Hq=Hq, Hkv=Hkv, d=128, needles=16)
    print(check_decode(w, workloads.generate(w)))


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["decode_131k", "prefill_gpt2s_8k"])
def test_debug_build_full_size_matches_release(dlib, name):
    """The benchmarked workloads at full size through both builds: the debug
    build's checks stay clean and its results equal the release build's
    bit for bit (the checks only add branches around accesses)."""
    import numpy as np
    import torch
    from gpu_common import run_decode, run_prefill
    w = workloads.get(name)
    x = workloads.generate(w)
    run = run_decode if w.kind == "decode" else run_prefill
    as_np = lambda t: t.cpu().numpy() if isinstance(t, torch.Tensor) else t
    rel = [as_np(t) for t in run(w, x)[:3]]
    prev = binding.use_library(binding.DEBUG_LIB_PATH)
    try:
        assert binding.load().condensate_attn_build_flags() == 1
        dbg = [as_np(t) for t in run(w, x)[:3]]
    finally:
        binding.use_library(prev)
    for a, b in zip(rel, dbg):
        assert np.array_equal(a, b)


def test_debug_library_selected_by_environment(dlib):
    # a fresh interpreter with CONDENSATE_ATTN_DEBUG=1 loads the debug build
    import os
    import subprocess
    import sys
    code = ("import sparse_transformer_attention_b200.binding as b; "
            "print(b.LIB_PATH == b.DEBUG_LIB_PATH, "
            "b.load().condensate_attn_build_flags())")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, CONDENSATE_ATTN_DEBUG="1", PYTHONPATH=root)
    out = subprocess.run([sys.executable, "-c", code], env=env, cwd=root,
                         capture_output=True, text=True, timeout=300)
    assert out.stdout.split() == ["True", "1"], out.stderr[-2000:]
