"""Host side of the sequence-sharded decode on two and three gloo ranks (CPU).

sparse_transformer_attention_b200.sharded.decode_sharded runs on each rank
with test stand-ins for the three per-rank library steps (plain numpy
restatements of what the header says each step returns, in the same key
format), so that the shard bounds, the order of the two all-gathers and the
decomposition of the softmax into per-shard (max, sum, o) states are checked
on CPU against the oracle's decode over the whole cache.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import workloads
from parity import check_rows
from sparse_transformer_attention_b200 import sharded

LOG2E = 1.4426950408889634


def _ord32(s):
    b = np.float32(s).view(np.uint32) if np.float32(s) != 0 else np.uint32(0)
    return int(~b & 0xFFFFFFFF) if b & 0x80000000 else int(b | 0x80000000)


def _unord32(o):
    b = (o & 0x7FFFFFFF) if o & 0x80000000 else (~o & 0xFFFFFFFF)
    return float(np.uint32(b).view(np.float32))


def _key(s, j):
    return (_ord32(s) << 32) | (0xFFFFFFFF - int(j))


def _to_i64(keys):
    return np.array(keys, dtype=np.uint64).view(np.int64)


class StandIns:
    """The three steps, restated in numpy (float64 dot products, fp32 keys
    as the kernels carry them).  Tensors in and out are CPU torch tensors."""

    def _geom(self, W, W_i, b, L):
        w = int(W_i[b]) if W_i is not None else W
        i = L - 1
        return i, max(0, i - w + 1), i - w  # query, window start, last cand

    def condensate_attn_decode_shard_select(self, q, K, pos0, L, W, k,
                                            W_i=None):
        q, K = q.numpy().astype(np.float64), K.numpy().astype(np.float64)
        B, Hq, _ = q.shape
        G = Hq // K.shape[1]
        out = np.zeros((B, Hq, k), dtype=np.uint64)
        for b in range(B):
            _, _, hi = self._geom(W, W_i, b, L)
            js = np.arange(max(1, pos0), min(hi, pos0 + K.shape[2] - 1) + 1)
            for h in range(Hq):
                keys = sorted((_key(float(q[b, h] @ K[b, h // G, j - pos0]), j)
                               for j in js), reverse=True)[:k]
                out[b, h, :len(keys)] = keys
        return torch.from_numpy(out.view(np.int64))

    def condensate_attn_decode_shard_attend(self, q, K, V, pos0, L, W, k,
                                            keys_all, W_i=None):
        q = q.numpy().astype(np.float64)
        K, V = K.numpy().astype(np.float64), V.numpy().astype(np.float64)
        keys_all = keys_all.numpy().view(np.uint64)
        B, Hq, d = q.shape
        G = Hq // K.shape[1]
        sl2 = LOG2E / np.sqrt(d)
        p1 = pos0 + K.shape[2]
        C_max = min(L, 1 + (int(W_i.max()) if W_i is not None else W) + k)
        part = np.zeros((B, Hq, d + 2), dtype=np.float32)
        idx = np.full((B, Hq, C_max), -1, dtype=np.int32)
        cnt = np.zeros((B, Hq), dtype=np.int32)
        for b in range(B):
            i, lo, hi = self._geom(W, W_i, b, L)
            m = min(k, max(0, hi))
            for h in range(Hq):
                ks = sorted((int(x) for x in keys_all[:, b, h].ravel() if x),
                            reverse=True)[:m]
                top = sorted((0xFFFFFFFF - (x & 0xFFFFFFFF),
                              _unord32(x >> 32)) for x in ks)
                members = ([(0, None)] if lo > 0 else []) + top + \
                    [(j, None) for j in range(lo, i + 1)]
                c = [j for j, _ in members]
                idx[b, h, :len(c)] = c
                cnt[b, h] = len(c)
                here = [(j, s) for j, s in members if pos0 <= j < p1]
                if not here:
                    part[b, h, 0], part[b, h, 1] = -np.inf, 0.0
                    continue
                t = np.array([(s if s is not None else
                               q[b, h] @ K[b, h // G, j - pos0]) * sl2
                              for j, s in here])
                mx = t.max()
                wgt = np.exp2(t - mx)
                part[b, h, 0], part[b, h, 1] = mx, wgt.sum()
                part[b, h, 2:] = wgt @ V[b, h // G, [j - pos0 for j, _ in here]]
        return (torch.from_numpy(part), torch.from_numpy(idx),
                torch.from_numpy(cnt))

    def condensate_attn_decode_shard_combine(self, parts, o_dtype=None):
        p = parts.numpy().astype(np.float64)
        live = p[..., 1] > 0
        M = np.where(live, p[..., 0], -np.inf).max(axis=0)
        c = np.where(live, np.exp2(np.where(live, p[..., 0], 0) - M), 0.0)
        l = (p[..., 1] * c).sum(axis=0)
        o = (p[..., 2:] * c[..., None]).sum(axis=0)
        return torch.from_numpy((o / l[..., None]).astype(np.float32))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(name):
    base = workloads.get("decode_131k")
    if name == "two":
        return base.scaled(n=3001, W=64, k=16, Hq=4, Hkv=2, d=64, needles=4,
                           B=2)
    return base.scaled(n=1500, W=40, k=24, Hq=2, Hkv=1, d=64, needles=4, B=1)


def _rank_main(rank, world, port, name, W_i, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = _case(name)
        x = workloads.generate(w)
        pos0, ls = sharded.shard_bounds(w.n, world, rank)
        q = torch.from_numpy(x["Q"])
        K = torch.from_numpy(np.ascontiguousarray(x["K"][:, :, pos0:pos0 + ls]))
        V = torch.from_numpy(np.ascontiguousarray(x["V"][:, :, pos0:pos0 + ls]))
        O, idx, cnt = sharded.decode_sharded(q, K, V, pos0, w.n, w.W, w.k,
                                             W_i=W_i, ops=StandIns())
        out[rank] = (O.numpy(), idx.numpy(), cnt.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name,world,W_i", [
    ("two", 2, None), ("two", 2, np.array([7, 3000], dtype=np.int32)),
    ("three", 3, None)])
def test_sharded_decode_gloo(name, world, W_i):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main,
                           args=(world, _free_port(), name, W_i, out),
                           nprocs=world, join=True, start_method="spawn")
        res = [out[r] for r in range(world)]
    for r in range(1, world):  # every rank ends with the same result
        for a, b in zip(res[0], res[r]):
            np.testing.assert_array_equal(a, b)
    w = _case(name)
    x = workloads.generate(w)
    O, idx, cnt = res[0]
    C_max = idx.shape[-1]
    ref = oracle.decode(x["Q"], x["K"], x["V"], w.W, w.k, W_i=W_i,
                        C_max=C_max, with_full=False)
    G = w.Hq // w.Hkv
    rows = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    print(check_rows(
        ref, idx.reshape(len(rows), -1), cnt.reshape(-1),
        O.reshape(len(rows), -1),
        q_rows=[x["Q"][b, h] for (b, h) in rows],
        kv_rows=lambda r: x["K"][rows[r][0], rows[r][1] // G],
        v_rows=lambda r: x["V"][rows[r][0], rows[r][1] // G],
        pos=[w.n - 1] * len(rows),
        win=[int(W_i[b]) if W_i is not None else w.W for (b, h) in rows],
        tol=1e-5))


def test_shard_bounds():
    assert [sharded.shard_bounds(10, 3, r) for r in range(3)] == \
        [(0, 4), (4, 3), (7, 3)]
    assert [sharded.shard_bounds(8, 8, r) for r in range(8)] == \
        [(r, 1) for r in range(8)]
    with pytest.raises(ValueError):
        sharded.shard_bounds(2, 3, 0)
