"""The extended entry points on the GPU, against the CPU oracle.

* Prefill of the last nq positions against an L-long cache (a chunk of a
  longer prefill, or several decode queries at once): query row r sits at
  position L - nq + r ("Condensate Theorem（冷凝定理）：注意力稀疏性的拓扑本质"
  §2.1 Definition 1 for those rows, §5.2.2).
* Per-head windows W_h and Top-k sizes k_h (page 1 §6 layer-wise windows,
  §10.2 per-head parameters; k_h = 0 is the static anchor + window variant):
  each head must match the oracle run with that head's W and k.
* Mass reports (page 1 §2.2.1 anchor mass, §2.2.2 window mass, §3.2.2
  excluded mass) and the log-sum-exp of the full causal row, against the
  oracle's double-precision values.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_transformer_attention_b200 as ca
import workloads
from gpu_common import TOL, to_dev
from parity import check_rows
from sparse_transformer_attention_b200 import binding

pytestmark = pytest.mark.gpu

MASS_TOL = 2e-5   # absolute, on probabilities accumulated in fp32
LSE_TOL = 1e-4    # absolute, on log-sum-exp values of size up to ~30


def _rows(B, Hq, positions):
    return np.array([(b, h, i) for b in range(B) for h in range(Hq)
                     for i in positions], dtype=np.int64)


def _check_chunk(w, x, nq, W_h=None, k_h=None, want_mass=False):
    """Run the prefill of the last nq positions and compare every row with
    the oracle (per head when W_h / k_h are given)."""
    L = w.n
    Qc = x["Q"][:, :, L - nq:, :]
    Q, K, V = (to_dev(a, w.dtype) for a in (Qc, x["K"], x["V"]))
    Wt = lambda a: None if a is None else \
        torch.from_numpy(np.asarray(a, np.int32)).cuda()
    kmax = w.k if k_h is None else max(int(max(k_h)), 0)
    Wmax = w.W if W_h is None else int(max(W_h))
    C_max = min(L, 1 + Wmax + max(kmax, w.k))
    mass = torch.full((w.B, w.Hq, nq, 4), float("nan"), device="cuda") \
        if want_mass else None
    lse = torch.full((w.B, w.Hq, nq), float("nan"), device="cuda") \
        if want_mass else None
    ws = torch.empty(ca.condensate_attn_workspace_size_ex(
        False, Q.dtype, w.B, nq, L, w.Hq, w.Hkv, w.d, Wmax, max(kmax, w.k)),
        dtype=torch.uint8, device="cuda")
    O, idx, cnt = ca.condensate_attn_prefill(
        Q, K, V, w.W, max(kmax, w.k), C_max=C_max, workspace=ws,
        W_h=Wt(W_h), k_h=Wt(k_h), mass=mass, lse=lse)
    st = ca.condensate_attn_status(ws)
    assert st == ca.CA_OK, ca.status_string(st)
    G = w.Hq // w.Hkv
    pos = list(range(L - nq, L))
    out = {"rows": 0, "near_ties": 0, "swapped": 0, "max_abs_err": 0.0}
    for h in range(w.Hq):
        Wr = w.W if W_h is None else int(W_h[h])
        kr = w.k if k_h is None else int(k_h[h])
        sel = _rows(w.B, 1, pos)
        sel[:, 1] = h
        g = h // G
        ref = oracle.prefill(x["Q"][:, h:h + 1], x["K"][:, g:g + 1],
                             x["V"][:, g:g + 1], Wr, kr,
                             sel=np.stack([sel[:, 0], 0 * sel[:, 1],
                                           sel[:, 2]], 1),
                             C_max=C_max, with_full=want_mass)
        gi = idx[:, h].cpu().numpy().reshape(-1, C_max)
        gc = cnt[:, h].cpu().numpy().ravel()
        go = O[:, h].float().cpu().numpy().reshape(-1, w.d)
        r = check_rows(
            ref, gi, gc, go,
            q_rows=[x["Q"][b, h, i] for (b, _, i) in sel],
            kv_rows=lambda t: x["K"][sel[t][0], g],
            v_rows=lambda t: x["V"][sel[t][0], g],
            pos=sel[:, 2], win=[Wr] * len(sel),
            tol=TOL[w.dtype])
        for key_ in ("rows", "near_ties", "swapped"):
            out[key_] += r[key_]
        out["max_abs_err"] = max(out["max_abs_err"], r["max_abs_err"])
        if want_mass:
            gm = mass[:, h].cpu().numpy().reshape(-1, 4)
            gl = lse[:, h].cpu().numpy().ravel()
            for c, name in enumerate(("anchor_mass", "window_mass",
                                      "topk_mass", "excluded_mass")):
                err = np.abs(gm[:, c] - ref[name])
                assert err.max() <= MASS_TOL, (h, name, float(err.max()))
            err = np.abs(gl - ref["lse"])
            assert err.max() <= LSE_TOL, (h, "lse", float(err.max()))
    return out


@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("f32", 128),
                                     ("bf16", 128)])
@pytest.mark.parametrize("nq", [1, 5, 200, 777])
def test_prefill_last_rows_against_cache(dtype, d, nq):
    w = workloads.get("prefill_gpt2s_8k").scaled(
        dtype=dtype, d=d, n=3000, B=2, Hq=4, Hkv=2, needles=4)
    print(_check_chunk(w, workloads.generate(w), nq))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_multi_query_decode(dtype):
    """Four decode queries at once against a 20K cache, 32 q-heads on 8
    kv-heads (the decode recipe)."""
    w = workloads.get("decode_131k").scaled(dtype=dtype, n=20000, needles=8)
    # the decode recipe draws one query per head; draw four per head for
    # this case from the same generator shape (positions L-4 .. L-1)
    x = workloads.generate(w.scaled(kind="prefill", needle_mode="none"))
    print(_check_chunk(w.scaled(kind="prefill"), x, 4))


@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("f32", 64),
                                     ("bf16", 128)])
def test_per_head_windows_and_k(dtype, d):
    w = workloads.get("prefill_gpt2s_8k").scaled(
        dtype=dtype, d=d, n=1500, B=1, Hq=8, Hkv=4, W=64, k=32, needles=4)
    W_h = [16, 64, 1, 300, 2000, 7, 64, 128]
    k_h = [0, 8, 32, 32, 5, 1, 31, 17]
    print(_check_chunk(w, workloads.generate(w), w.n, W_h=W_h, k_h=k_h))


@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("f32", 128),
                                     ("bf16", 128)])
def test_prefill_mass_reports(dtype, d):
    w = workloads.get("prefill_gpt2s_8k").scaled(
        dtype=dtype, d=d, n=1200, B=1, Hq=2, Hkv=2, needles=4)
    x = workloads.generate(w)
    print(_check_chunk(w, x, w.n, want_mass=True))
    print(_check_chunk(w, x, 100, want_mass=True))  # chunk against a cache


def test_prefill_mass_reports_with_k0_heads():
    """k = 0 for some heads (the static variant): the score pass still runs
    for the candidates' sums."""
    w = workloads.get("prefill_gpt2s_8k").scaled(n=900, B=1, Hq=4, Hkv=4,
                                                 needles=2)
    print(_check_chunk(w, workloads.generate(w), w.n, k_h=[0, 3, 0, 32],
                       want_mass=True))


def _decode_case(w, x, W_h=None, k_h=None, want_mass=False):
    q, K, V = (to_dev(x[n], w.dtype) for n in ("Q", "K", "V"))
    Wt = lambda a: None if a is None else \
        torch.from_numpy(np.asarray(a, np.int32)).cuda()
    kmax = w.k if k_h is None else max(int(max(k_h)), w.k)
    Wmax = w.W if W_h is None else int(max(W_h))
    C_max = min(w.n, 1 + Wmax + kmax)
    mass = torch.full((w.B, w.Hq, 4), float("nan"), device="cuda") \
        if want_mass else None
    lse = torch.full((w.B, w.Hq), float("nan"), device="cuda") \
        if want_mass else None
    ws = torch.empty(ca.condensate_attn_workspace_size(
        True, q.dtype, w.B, w.n, w.Hq, w.Hkv, w.d, Wmax, kmax),
        dtype=torch.uint8, device="cuda")
    O, idx, cnt = ca.condensate_attn_decode(
        q, K, V, w.W, kmax, C_max=C_max, workspace=ws, W_h=Wt(W_h),
        k_h=Wt(k_h), mass=mass, lse=lse)
    st = ca.condensate_attn_status(ws)
    assert st == ca.CA_OK, ca.status_string(st)
    G = w.Hq // w.Hkv
    for h in range(w.Hq):
        Wr = w.W if W_h is None else int(W_h[h])
        kr = w.k if k_h is None else int(k_h[h])
        g = h // G
        ref = oracle.decode(x["Q"][:, h:h + 1], x["K"][:, g:g + 1],
                            x["V"][:, g:g + 1], Wr, kr, C_max=C_max,
                            with_full=want_mass)
        check_rows(ref, idx[:, h].cpu().numpy(), cnt[:, h].cpu().numpy(),
                   O[:, h].float().cpu().numpy(),
                   q_rows=[x["Q"][b, h] for b in range(w.B)],
                   kv_rows=lambda t: x["K"][t, g],
                   v_rows=lambda t: x["V"][t, g],
                   pos=[w.n - 1] * w.B, win=[Wr] * w.B, tol=TOL[w.dtype])
        if want_mass:
            gm = mass[:, h].cpu().numpy()
            for c, name in enumerate(("anchor_mass", "window_mass",
                                      "topk_mass", "excluded_mass")):
                err = np.abs(gm[:, c] - ref[name])
                assert err.max() <= MASS_TOL, (h, name, float(err.max()))
            err = np.abs(lse[:, h].cpu().numpy() - ref["lse"])
            assert err.max() <= LSE_TOL, (h, "lse", float(err.max()))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_per_head_windows_and_k(dtype):
    w = workloads.get("decode_131k").scaled(dtype=dtype, n=30000, B=2, Hq=8,
                                            Hkv=2, needles=8)
    _decode_case(w, workloads.generate(w), W_h=[16, 128, 1, 4000, 64, 7,
                                               29999, 200],
                 k_h=[0, 64, 32, 1, 64, 5, 64, 17])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_mass_reports(dtype):
    w = workloads.get("decode_131k").scaled(dtype=dtype, n=30000, B=2, Hq=8,
                                            Hkv=2, needles=8)
    _decode_case(w, workloads.generate(w), want_mass=True)


def test_decode_mass_reports_131k():
    """The 131K decode workload at full size with the mass reports on."""
    w = workloads.get("decode_131k")
    _decode_case(w, workloads.generate(w), want_mass=True)


def test_per_head_values_out_of_range_are_reported():
    w = workloads.get("decode_131k").scaled(n=3000, B=1, Hq=4, Hkv=2,
                                            needles=2)
    x = workloads.generate(w)
    q, K, V = (to_dev(x[n], w.dtype) for n in ("Q", "K", "V"))
    ws = torch.empty(ca.condensate_attn_workspace_size(
        True, q.dtype, w.B, w.n, w.Hq, w.Hkv, w.d, 300, w.k),
        dtype=torch.uint8, device="cuda")
    W_h = torch.tensor([64, 0, 64, 64], dtype=torch.int32, device="cuda")
    ca.condensate_attn_decode(q, K, V, w.W, w.k, C_max=1 + 64 + w.k,
                              workspace=ws, W_h=W_h)
    assert ca.condensate_attn_status(ws) == binding.CA_ERR_DEVICE_ARG
    k_h = torch.tensor([1, 2, w.k + 1, 3], dtype=torch.int32, device="cuda")
    ca.condensate_attn_decode(q, K, V, w.W, w.k, C_max=1 + w.W + w.k,
                              workspace=ws, k_h=k_h)
    assert ca.condensate_attn_status(ws) == binding.CA_ERR_DEVICE_ARG
    Q, Kp, Vp = (to_dev(x[n], w.dtype) for n in ("Q", "K", "V"))
    wp = workloads.get("prefill_gpt2s_8k").scaled(n=500, B=1, Hq=4, Hkv=2,
                                                  needles=2)
    xp = workloads.generate(wp)
    Q, Kp, Vp = (to_dev(xp[n], wp.dtype) for n in ("Q", "K", "V"))
    wsp = torch.empty(ca.condensate_attn_workspace_size(
        False, Q.dtype, wp.B, wp.n, wp.Hq, wp.Hkv, wp.d, 64, wp.k),
        dtype=torch.uint8, device="cuda")
    ca.condensate_attn_prefill(Q, Kp, Vp, wp.W, wp.k, C_max=1 + 64 + wp.k,
                               workspace=wsp,
                               k_h=torch.tensor([1, -1, 3, 4],
                                                dtype=torch.int32,
                                                device="cuda"))
    assert ca.condensate_attn_status(wsp) == binding.CA_ERR_DEVICE_ARG
