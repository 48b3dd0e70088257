"""The decode entry point that allocates nothing.

Callers such as a plugin whose host program gives it no allocator, or code
whose device memory is fully budgeted before it runs, cannot provide the
scratch workspace that condensate_attn_decode needs.  They call
condensate_attn_decode_noalloc, which uses a buffer compiled into the
library instead.  This test calls it through the C ABI and checks it against
the workspace entry point on the same inputs, twice in a row (the second
call finds the first call's leftovers in the shared buffer).  Kept in a file
of its own that pytest collects last.
"""
import ctypes

import numpy as np
import pytest
import torch

import sparse_transformer_attention_b200 as ca
import workloads
from sparse_transformer_attention_b200 import binding

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p


def _p(t):
    return None if t is None else P(t.data_ptr())


def _stream():
    return P(torch.cuda.current_stream().cuda_stream)


def _noalloc(lib, q, K, V, w, O, idx, cnt, C_max, W_i=None):
    dt = binding.CA_BF16 if q.dtype == torch.bfloat16 else binding.CA_F32
    odt = binding.CA_BF16 if O.dtype == torch.bfloat16 else binding.CA_F32
    return lib.condensate_attn_decode_noalloc(
        _p(q), _p(K), _p(V), dt, w.B, w.n, w.Hq, w.Hkv, w.d, w.W, w.k,
        _p(W_i), _p(O), odt, _p(idx), _p(cnt), C_max, _stream())


@pytest.mark.parametrize("dtype,tol", [("bf16", 1e-2), ("f32", 1e-5)])
def test_noalloc_matches_workspace_entry_point(dtype, tol):
    lib = binding.load()
    w = workloads.get("decode_131k").scaled(n=40000, dtype=dtype, needles=16)
    x = workloads.generate(w)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q, K, V = (torch.from_numpy(x[n]).cuda().to(tdt) for n in ("Q", "K", "V"))
    C_max = min(w.n, 1 + w.W + w.k)
    O_ref, idx_ref, cnt_ref = ca.condensate_attn_decode(q, K, V, w.W, w.k,
                                                        C_max=C_max)
    torch.cuda.synchronize()
    for call in range(2):
        O = torch.full_like(O_ref, float("nan"))
        idx = torch.full_like(idx_ref, -7)
        cnt = torch.full_like(cnt_ref, -7)
        code = _noalloc(lib, q, K, V, w, O, idx, cnt, C_max)
        assert code == binding.CA_OK, ca.status_string(code)
        torch.cuda.synchronize()
        assert torch.equal(cnt, cnt_ref), call
        assert torch.equal(idx, idx_ref), call
        err = (O - O_ref).abs().max().item()
        assert err <= tol, (call, err)
        # the built-in buffer's status word: nothing raised
        assert lib.condensate_attn_decode_noalloc_status(_stream()) == \
            binding.CA_OK, call


def test_noalloc_status_reports_device_flags():
    """A per-batch window below 1 is only seen on the device: the flag lands
    in the built-in buffer and the status reader reports (and clears) it."""
    lib = binding.load()
    w = workloads.get("decode_131k").scaled(n=6000, B=2, Hq=8, Hkv=2,
                                            needles=4)
    x = workloads.generate(w)
    q, K, V = (torch.from_numpy(x[n]).cuda().to(torch.bfloat16)
               for n in ("Q", "K", "V"))
    C_max = min(w.n, 1 + w.W + w.k)
    O = torch.empty((w.B, w.Hq, w.d), device="cuda")
    idx = torch.empty((w.B, w.Hq, C_max), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.B, w.Hq), dtype=torch.int32, device="cuda")
    W_i = torch.tensor([w.W, 0], dtype=torch.int32, device="cuda")
    assert _noalloc(lib, q, K, V, w, O, idx, cnt, C_max, W_i) == binding.CA_OK
    assert lib.condensate_attn_decode_noalloc_status(_stream()) == \
        binding.CA_ERR_DEVICE_ARG
    assert lib.condensate_attn_decode_noalloc_status(_stream()) == \
        binding.CA_OK


def test_noalloc_rejects_problems_beyond_its_buffer():
    lib = binding.load()
    # 64 q-heads x 8 chunks x k=1024 candidate keys x 8 bytes = 4 MiB, plus
    # the status area: past the built-in buffer.
    w = workloads.get("decode_131k").scaled(n=9000, Hq=64, Hkv=8, k=1024)
    assert ca.condensate_attn_workspace_size(
        True, torch.bfloat16, w.B, w.n, w.Hq, w.Hkv, w.d, w.W, w.k) > 4 << 20
    q = torch.zeros((w.B, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros((w.B, w.Hkv, w.n, w.d), dtype=torch.bfloat16, device="cuda")
    C_max = min(w.n, 1 + w.W + w.k)
    O = torch.zeros((w.B, w.Hq, w.d), device="cuda")
    idx = torch.zeros((w.B, w.Hq, C_max), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((w.B, w.Hq), dtype=torch.int32, device="cuda")
    code = _noalloc(lib, q, K, K, w, O, idx, cnt, C_max)
    assert code == binding.CA_ERR_WORKSPACE
