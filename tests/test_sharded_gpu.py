"""Sequence-sharded decode on one GPU.  The P shards' steps run one after the
other on the same device (the two all-gathers become stacks of the shards'
outputs, in shard order), and the combined result is compared element by
element with the CPU oracle on the whole cache, and with the one-GPU decode
(the same index sets: the tensor-core dot product of a key does not depend
on the tile it lands in)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import sparse_transformer_attention_b200 as ca
from gpu_common import TOL, run_decode, to_dev
from parity import check_rows

pytestmark = pytest.mark.gpu

BASE = workloads.get("decode_131k")


def run_sharded(w, x, bounds, W_i=None, o_dtype=torch.float32):
    q, K, V = (to_dev(x[n], w.dtype) for n in ("Q", "K", "V"))
    Wt = None if W_i is None else torch.from_numpy(W_i.astype(np.int32)).cuda()
    W_max = int(W_i.max()) if W_i is not None else w.W
    C_max = min(w.n, 1 + W_max + w.k)
    assert bounds[0][0] == 0 and sum(ls for _, ls in bounds) == w.n
    shards = [(p0, K[:, :, p0:p0 + ls].contiguous(),
               V[:, :, p0:p0 + ls].contiguous()) for p0, ls in bounds]
    keys = []
    for p0, Ks, _ in shards:
        ws = torch.empty(ca.condensate_attn_decode_shard_workspace_size(
            q.dtype, w.B, Ks.shape[2], w.Hq, w.Hkv, w.d, w.k),
            dtype=torch.uint8, device="cuda")
        keys.append(ca.condensate_attn_decode_shard_select(
            q, Ks, p0, w.n, w.W, w.k, W_i=Wt, workspace=ws))
        st = ca.condensate_attn_status(ws)
        assert st == ca.CA_OK, ca.status_string(st)
    keys_all = torch.stack(keys)
    parts, sets = [], []
    for p0, Ks, Vs in shards:
        ws = torch.empty(256, dtype=torch.uint8, device="cuda")
        part, idx, cnt = ca.condensate_attn_decode_shard_attend(
            q, Ks, Vs, p0, w.n, w.W, w.k, keys_all, W_i=Wt, C_max=C_max,
            workspace=ws)
        st = ca.condensate_attn_status(ws)
        assert st == ca.CA_OK, ca.status_string(st)
        parts.append(part)
        sets.append((idx, cnt))
    O = ca.condensate_attn_decode_shard_combine(torch.stack(parts),
                                                o_dtype=o_dtype)
    for idx, cnt in sets[1:]:  # every shard writes the same set
        assert torch.equal(idx, sets[0][0]) and torch.equal(cnt, sets[0][1])
    return (O.float().cpu().numpy(), sets[0][0].cpu().numpy(),
            sets[0][1].cpu().numpy(), C_max)


def check_sharded(w, x, bounds, W_i=None, o_dtype=torch.float32):
    O, idx, cnt, C_max = run_sharded(w, x, bounds, W_i, o_dtype)
    ref = oracle.decode(x["Q"], x["K"], x["V"], w.W, w.k, W_i=W_i,
                        C_max=C_max, with_full=False)
    G = w.Hq // w.Hkv
    rows = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    win = [int(W_i[b]) if W_i is not None else w.W for (b, h) in rows]
    tol = TOL[w.dtype] + (2.0 ** -6 if o_dtype == torch.bfloat16 else 0.0)
    rep = check_rows(
        ref, idx, cnt, O,
        q_rows=[x["Q"][b, h] for (b, h) in rows],
        kv_rows=lambda r: x["K"][rows[r][0], rows[r][1] // G],
        v_rows=lambda r: x["V"][rows[r][0], rows[r][1] // G],
        pos=[w.n - 1] * len(rows), win=win, tol=tol)
    # the same sets as the decode over the whole cache on one GPU; outputs
    # equal up to the order of the fp32 sums
    O1, idx1, cnt1, _ = run_decode(w, x, W_i, o_dtype)
    np.testing.assert_array_equal(idx, idx1)
    np.testing.assert_array_equal(cnt, cnt1)
    assert np.abs(O - O1).max() <= 1e-5 + (2.0 ** -7 if o_dtype ==
                                           torch.bfloat16 else 0.0)
    return rep


def split(n, cuts):
    edges = [0] + list(cuts) + [n]
    return [(a, b - a) for a, b in zip(edges[:-1], edges[1:])]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("cuts", [
    (4500,),                 # two even shards
    (100, 8950),             # the last shard holds window rows only
    (1, 2048, 6001),         # a one-row shard: the anchor alone
    (8872, 8873),            # cuts at the window's first row
])
def test_sharded_decode(d, cuts):
    w = BASE.scaled(d=d, Hq=8, Hkv=2, n=9001, W=128, k=64, needles=16, B=2)
    x = workloads.generate(w)
    print(check_sharded(w, x, split(w.n, cuts)))


def test_sharded_decode_one_shard():
    w = BASE.scaled(Hq=8, Hkv=2, n=5000, needles=8)
    print(check_sharded(w, workloads.generate(w), [(0, w.n)]))


def test_sharded_decode_k128_many_shards():
    # 1M-context parameters (W = 256, k = 128) on a shorter cache, 8 shards
    w = BASE.scaled(n=40000, W=256, k=128, needles=32)
    x = workloads.generate(w)
    b = [ca.shard_bounds(w.n, 8, r) for r in range(8)]
    print(check_sharded(w, x, b))


def test_sharded_decode_per_batch_window_bf16_out():
    w = BASE.scaled(n=20000, B=4, Hq=8, Hkv=2, needles=8)
    x = workloads.generate(w)
    W_i = np.array([64, 1, 256, 19999], dtype=np.int32)
    print(check_sharded(w, x, split(w.n, (7000, 19800)), W_i=W_i,
                        o_dtype=torch.bfloat16))


@pytest.mark.parametrize("L,W,k,cuts", [
    (4097, 7, 300, (1000, 3000)),   # k > 128: the radix selection path
    (1000, 1, 0, (500,)),           # k = 0: anchor and window only
    (200, 128, 64, (60, 150)),      # fewer candidates than k
])
def test_sharded_decode_edges(L, W, k, cuts):
    w = BASE.scaled(n=L, W=W, k=k, Hq=8, Hkv=2,
                    needles=min(8, max(0, L - 1 - W)))
    print(check_sharded(w, workloads.generate(w), split(L, cuts)))


def test_sharded_decode_errors():
    w = BASE.scaled(n=1000, Hq=8, Hkv=2, d=64)
    q = torch.zeros((1, 8, 64), dtype=torch.bfloat16, device="cuda")
    K = torch.zeros((1, 2, 500, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ca.CondensateError) as e:
        ca.condensate_attn_decode_shard_select(q, K, 600, 1000, w.W, w.k)
    assert e.value.code == ca.binding.CA_ERR_INVALID_ARG  # past the end
    with pytest.raises(ca.CondensateError) as e:
        ca.condensate_attn_decode_shard_select(q.float(), K.float(), 0, 1000,
                                               w.W, w.k)
    assert e.value.code == ca.binding.CA_ERR_UNSUPPORTED  # fp32 select
