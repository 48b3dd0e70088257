"""The GPU's fp32 scores against the exact ones, key by key.

The selection keys the kernels leave in the workspace carry each candidate's
fp32 score t_j = q.k_j with its position j (decode: the per-chunk lists of
the score pass; prefill: the per-row Top-k keys).  Every carried score must
lie within the standard dot-product rounding bound gamma_d sum_l |q_l k_jl|
(u = 2^-23) of the exact value, which is the premise of the near-tie rule the
parity tests apply (Higham, "Accuracy and Stability of Numerical
Algorithms", §3.1; the Top-k order of "Condensate Theorem（冷凝定理）：注意力
稀疏性的拓扑本质" §2.2.3).
"""
import numpy as np
import pytest
import torch

import sparse_transformer_attention_b200 as ca
import workloads
from gpu_common import to_dev

pytestmark = pytest.mark.gpu

U = 2.0 ** -23


def gamma(d):
    return d * U / (1.0 - d * U)


def decode_keys(keys):
    """(score float64, position int64) of non-empty 64-bit selection keys."""
    keys = np.asarray(keys, dtype=np.uint64)
    keys = keys[keys != 0]
    o = (keys >> np.uint64(32)).astype(np.uint32)
    neg = (o & np.uint32(0x80000000)) == 0
    bits = np.where(neg, ~o, o & np.uint32(0x7FFFFFFF)).astype(np.uint32)
    score = bits.view(np.float32).astype(np.float64)
    j = (np.uint64(0xFFFFFFFF) - (keys & np.uint64(0xFFFFFFFF))).astype(np.int64)
    return score, j


def _check(q, K, score, j):
    t = K[j].astype(np.float64) @ q.astype(np.float64)
    a = np.abs(K[j].astype(np.float64)) @ np.abs(q.astype(np.float64))
    err = np.abs(score - t)
    assert np.all(err <= gamma(len(q)) * a), float((err / a).max())
    return len(j)


@pytest.mark.parametrize("name", ["decode_131k", "decode_1m"])
def test_decode_carried_scores(name):
    w = workloads.get(name)
    x = workloads.generate(w)
    q, K, V = (to_dev(x[n], w.dtype) for n in ("Q", "K", "V"))
    nbytes = ca.condensate_attn_workspace_size(True, q.dtype, w.B, w.n, w.Hq,
                                               w.Hkv, w.d, w.W, w.k)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    ca.condensate_attn_decode(q, K, V, w.W, w.k, workspace=ws)
    assert ca.condensate_attn_status(ws) == ca.CA_OK
    nch = ca.condensate_attn_decode_chunks(w.B, w.n, w.Hkv, w.k)
    per_head = nch * w.k
    # after the status area and the [B, Hkv] work counters (256-byte rounded)
    off = 256 + (w.B * w.Hkv * 4 + 255) // 256 * 256
    body = ws[off:off + w.B * w.Hq * per_head * 8].cpu().numpy().view(np.uint64)
    G = w.Hq // w.Hkv
    total = 0
    for b in range(w.B):
        for h in range(w.Hq):
            lst = body[(b * w.Hq + h) * per_head:(b * w.Hq + h + 1) * per_head]
            score, j = decode_keys(lst)
            assert np.all((j >= 1) & (j <= w.n - 1 - w.W))
            total += _check(x["Q"][b, h], x["K"][b, h // G], score, j)
    assert total >= w.B * w.Hq * w.k
    print({"workload": name, "keys_checked": total})


@pytest.mark.parametrize("name,n", [("prefill_gpt2s_8k", 2048),
                                    ("prefill_adaptive_32k", 2048)])
def test_prefill_carried_scores(name, n):
    w = workloads.get(name).scaled(n=n, B=1, Hq=2, Hkv=2)
    x = workloads.generate(w)
    Q, K, V = (to_dev(x[nm], w.dtype) for nm in ("Q", "K", "V"))
    W_i = None if x["W_i"] is None else torch.from_numpy(x["W_i"]).cuda()
    nbytes = ca.condensate_attn_workspace_size(False, Q.dtype, w.B, w.n, w.Hq,
                                               w.Hkv, w.d, w.W_max, w.k)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    ca.condensate_attn_prefill(Q, K, V, w.W, w.k, W_i=W_i, workspace=ws)
    assert ca.condensate_attn_status(ws) == ca.CA_OK
    R = w.B * w.Hq * w.n
    topk = ws[256:256 + R * w.k * 8].cpu().numpy().view(np.uint64)
    topk = topk.reshape(R, w.k)
    total = 0
    for r in range(R):
        bh, i = divmod(r, w.n)
        b, h = divmod(bh, w.Hq)
        score, j = decode_keys(topk[r])
        win = int(x["W_i"][b, i]) if x["W_i"] is not None else w.W
        assert np.all((j >= 1) & (j <= i - win))
        if len(j):
            total += _check(x["Q"][b, h, i], x["K"][b, h], score, j)
    assert total > 0
    print({"workload": name, "n": n, "keys_checked": total})
