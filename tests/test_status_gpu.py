"""Device-side failure paths on the GPU, in forms that fault nothing.

* A per-query window W_i below 1 and a W_i whose set overflows C_max are
  values only the device sees: the kernels clamp them, raise a flag in the
  workspace status word, and condensate_attn_status reports
  CA_ERR_DEVICE_ARG.  Outputs stay inside their buffers.
* The failure-path test hook (condensate_attn_test_stall) makes one
  pipeline consumer of the score kernel wait, with a limit of 1 ms, on a
  barrier that nothing signals: the wait runs out, every wait of the CTA
  gives up, the kernel leaves through its normal path and the status reads
  CA_ERR_TIMEOUT.  The next normal call on the same context must match the
  oracle.
"""
import numpy as np
import pytest
import torch

import sparse_transformer_attention_b200 as ca
import workloads
from gpu_common import check_decode, check_prefill, to_dev
from sparse_transformer_attention_b200 import binding

pytestmark = pytest.mark.gpu

DEC = workloads.get("decode_131k").scaled(n=5000, B=2, Hq=8, Hkv=2, needles=4)
PRE = workloads.get("prefill_gpt2s_8k").scaled(n=700, B=1, Hq=2, Hkv=2,
                                               needles=2)


def _decode_call(w, x, W_i, C_max):
    q, K, V = (to_dev(x[n], w.dtype) for n in ("Q", "K", "V"))
    Wt = torch.from_numpy(np.asarray(W_i, dtype=np.int32)).cuda()
    ws = torch.empty(ca.condensate_attn_workspace_size(
        True, q.dtype, w.B, w.n, w.Hq, w.Hkv, w.d, 256, w.k),
        dtype=torch.uint8, device="cuda")
    O, idx, cnt = ca.condensate_attn_decode(q, K, V, w.W, w.k, W_i=Wt,
                                            C_max=C_max, workspace=ws)
    return ws, O, idx, cnt


def _prefill_call(w, x, W_i, C_max):
    Q, K, V = (to_dev(x[n], w.dtype) for n in ("Q", "K", "V"))
    Wt = torch.from_numpy(np.asarray(W_i, dtype=np.int32)).cuda()
    ws = torch.empty(ca.condensate_attn_workspace_size(
        False, Q.dtype, w.B, w.n, w.Hq, w.Hkv, w.d, 256, w.k),
        dtype=torch.uint8, device="cuda")
    O, idx, cnt = ca.condensate_attn_prefill(Q, K, V, w.W, w.k, W_i=Wt,
                                             C_max=C_max, workspace=ws)
    return ws, O, idx, cnt


def test_decode_window_below_one_is_reported():
    x = workloads.generate(DEC)
    ws, O, idx, cnt = _decode_call(DEC, x, [64, 0], 1 + 64 + DEC.k)
    assert ca.condensate_attn_status(ws) == binding.CA_ERR_DEVICE_ARG
    # read as a window of 1: {0} U Top-k U {L-1}
    assert cnt[1].cpu().tolist() == [2 + DEC.k] * DEC.Hq
    assert ca.condensate_attn_status(ws) == binding.CA_OK  # cleared


def test_decode_set_overflowing_cmax_is_reported():
    x = workloads.generate(DEC)
    C_max = 1 + 64 + DEC.k
    ws, O, idx, cnt = _decode_call(DEC, x, [64, 200], C_max)
    assert ca.condensate_attn_status(ws) == binding.CA_ERR_DEVICE_ARG
    # the true size is reported, idx holds the first C_max entries
    assert cnt[1].cpu().tolist() == [1 + 200 + DEC.k] * DEC.Hq
    assert bool((idx[1] >= 0).all())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_prefill_window_below_one_is_reported(dtype):
    w = PRE.scaled(dtype=dtype)
    x = workloads.generate(w)
    W_i = np.full((w.B, w.n), 64, dtype=np.int32)
    W_i[0, 300] = 0
    W_i[0, 650] = -5
    ws, O, idx, cnt = _prefill_call(w, x, W_i, 1 + 64 + w.k)
    assert ca.condensate_attn_status(ws) == binding.CA_ERR_DEVICE_ARG
    c = cnt.cpu().numpy()
    assert np.all(c[0, :, 300] == 2 + w.k) and np.all(c[0, :, 650] == 2 + w.k)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_prefill_set_overflowing_cmax_is_reported(dtype):
    w = PRE.scaled(dtype=dtype)
    x = workloads.generate(w)
    W_i = np.full((w.B, w.n), 64, dtype=np.int32)
    W_i[0, 500] = 300
    C_max = 1 + 64 + w.k
    ws, O, idx, cnt = _prefill_call(w, x, W_i, C_max)
    assert ca.condensate_attn_status(ws) == binding.CA_ERR_DEVICE_ARG
    c = cnt.cpu().numpy()
    assert np.all(c[0, :, 500] == 1 + 300 + w.k)
    assert bool((idx[0, :, 500] >= 0).all())


def test_clean_calls_report_ok():
    x = workloads.generate(DEC)
    ws, *_ = _decode_call(DEC, x, [64, 128], 1 + 128 + DEC.k)
    assert ca.condensate_attn_status(ws) == binding.CA_OK


@pytest.fixture
def stall():
    binding.test_stall(1_000_000)  # 1 ms
    try:
        yield
    finally:
        binding.test_stall(0)


def test_decode_wait_time_out_is_reported_and_recovered(stall):
    w = DEC
    x = workloads.generate(w)
    q, K, V = (to_dev(x[n], w.dtype) for n in ("Q", "K", "V"))
    ws = torch.empty(ca.condensate_attn_workspace_size(
        True, q.dtype, w.B, w.n, w.Hq, w.Hkv, w.d, w.W, w.k),
        dtype=torch.uint8, device="cuda")
    ca.condensate_attn_decode(q, K, V, w.W, w.k, workspace=ws)
    assert ca.condensate_attn_status(ws) == binding.CA_ERR_TIMEOUT
    binding.test_stall(0)
    print(check_decode(w, x))


def test_prefill_wait_time_out_is_reported_and_recovered(stall):
    w = PRE
    x = workloads.generate(w)
    Q, K, V = (to_dev(x[n], w.dtype) for n in ("Q", "K", "V"))
    ws = torch.empty(ca.condensate_attn_workspace_size(
        False, Q.dtype, w.B, w.n, w.Hq, w.Hkv, w.d, w.W, w.k),
        dtype=torch.uint8, device="cuda")
    ca.condensate_attn_prefill(Q, K, V, w.W, w.k, workspace=ws)
    assert ca.condensate_attn_status(ws) == binding.CA_ERR_TIMEOUT
    binding.test_stall(0)
    print(check_prefill(w, x))
