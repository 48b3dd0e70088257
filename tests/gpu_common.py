"""Shared helpers of the GPU parity tests (call the library through the C ABI
binding, compare with the CPU oracle)."""
import numpy as np
import torch

import oracle
import sparse_transformer_attention_b200 as ca
from parity import check_rows

TOL = {"f32": 1e-5, "bf16": 1e-2}


def to_dev(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a)).to("cuda")
    return t.to(torch.bfloat16 if dtype == "bf16" else torch.float32)


def run_decode(w, x, W_i=None, o_dtype=torch.float32):
    q, K, V = (to_dev(x[n], w.dtype) for n in ("Q", "K", "V"))
    Wt = None if W_i is None else torch.from_numpy(W_i.astype(np.int32)).cuda()
    W_max = int(W_i.max()) if W_i is not None else w.W
    C_max = min(w.n, 1 + W_max + w.k)
    ws = torch.empty(ca.condensate_attn_workspace_size(
        True, q.dtype, w.B, w.n, w.Hq, w.Hkv, w.d, W_max, w.k),
        dtype=torch.uint8, device="cuda")
    O, idx, cnt = ca.condensate_attn_decode(q, K, V, w.W, w.k, W_i=Wt,
                                            C_max=C_max, workspace=ws,
                                            o_dtype=o_dtype)
    status = ca.condensate_attn_status(ws)
    assert status == ca.CA_OK, ca.status_string(status)
    return O.float().cpu().numpy(), idx.cpu().numpy(), cnt.cpu().numpy(), C_max


def check_decode(w, x, W_i=None, o_dtype=torch.float32, tol=None):
    O, idx, cnt, C_max = run_decode(w, x, W_i, o_dtype)
    ref = oracle.decode(x["Q"], x["K"], x["V"], w.W, w.k, W_i=W_i,
                        C_max=C_max, with_full=False)
    G = w.Hq // w.Hkv
    rows = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    win = [int(W_i[b]) if W_i is not None else w.W for (b, h) in rows]
    return check_rows(
        ref, idx, cnt, O,
        q_rows=[x["Q"][b, h] for (b, h) in rows],
        kv_rows=lambda r: x["K"][rows[r][0], rows[r][1] // G],
        v_rows=lambda r: x["V"][rows[r][0], rows[r][1] // G],
        pos=[w.n - 1] * len(rows), win=win,
        tol=tol if tol is not None else TOL[w.dtype])


def run_prefill(w, x, W_i=None, o_dtype=torch.float32):
    Q, K, V = (to_dev(x[n], w.dtype) for n in ("Q", "K", "V"))
    Wt = None if W_i is None else torch.from_numpy(W_i.astype(np.int32)).cuda()
    W_max = int(W_i.max()) if W_i is not None else w.W
    C_max = 1 + W_max + w.k
    ws = torch.empty(ca.condensate_attn_workspace_size(
        False, Q.dtype, w.B, w.n, w.Hq, w.Hkv, w.d, W_max, w.k),
        dtype=torch.uint8, device="cuda")
    O, idx, cnt = ca.condensate_attn_prefill(Q, K, V, w.W, w.k, W_i=Wt,
                                             C_max=C_max, workspace=ws,
                                             o_dtype=o_dtype)
    status = ca.condensate_attn_status(ws)
    assert status == ca.CA_OK, ca.status_string(status)
    return O, idx, cnt, C_max, ws


def fallback_rows(w, ws):
    """(b, h, i) of the rows the prefill selector listed for its exact
    fallback pass (read from the workspace: the count sits in the status
    area at byte 16, the row list after the per-row Top-k keys)."""
    R = w.B * w.Hq * w.n
    cnt = int(ws[16:20].cpu().numpy().view(np.uint32)[0])
    topk_bytes = (R * max(w.k, 1) * 8 + 255) // 256 * 256
    off = 256 + topk_bytes
    rows = ws[off:off + 4 * cnt].cpu().numpy().view(np.uint32).astype(np.int64)
    bh, i = np.divmod(rows, w.n)
    b, h = np.divmod(bh, w.Hq)
    return np.stack([b, h, i], 1).reshape(-1, 3)


def check_prefill(w, x, W_i=None, sel=None, o_dtype=torch.float32, tol=None,
                  with_fallback_rows=False):
    """Compare all rows (sel=None) or the sampled (b, h, i) rows `sel`
    (plus, with_fallback_rows, every row that took the exact fallback)."""
    O, idx, cnt, C_max, ws = run_prefill(w, x, W_i, o_dtype)
    nfb = 0
    if with_fallback_rows:
        fb = fallback_rows(w, ws)
        nfb = len(fb)
        if sel is not None:
            sel = np.unique(np.concatenate([np.asarray(sel, np.int64), fb]),
                            axis=0)
    if sel is None:
        b, h, i = np.meshgrid(np.arange(w.B), np.arange(w.Hq), np.arange(w.n),
                              indexing="ij")
        sel = np.stack([b.ravel(), h.ravel(), i.ravel()], 1)
    sel = np.asarray(sel, dtype=np.int64)
    ti = torch.from_numpy(sel).cuda()
    g_idx = idx[ti[:, 0], ti[:, 1], ti[:, 2]].cpu().numpy()
    g_cnt = cnt[ti[:, 0], ti[:, 1], ti[:, 2]].cpu().numpy()
    g_o = O[ti[:, 0], ti[:, 1], ti[:, 2]].float().cpu().numpy()
    ref = oracle.prefill(x["Q"], x["K"], x["V"], w.W, w.k, W_i=W_i, sel=sel,
                         C_max=C_max, with_full=False)
    G = w.Hq // w.Hkv
    win = [int(W_i[b, i]) if W_i is not None else w.W for (b, h, i) in sel]
    out = check_rows(
        ref, g_idx, g_cnt, g_o,
        q_rows=[x["Q"][b, h, i] for (b, h, i) in sel],
        kv_rows=lambda r: x["K"][sel[r][0], sel[r][1] // G],
        v_rows=lambda r: x["V"][sel[r][0], sel[r][1] // G],
        pos=sel[:, 2], win=win,
        tol=tol if tol is not None else TOL[w.dtype])
    if with_fallback_rows:
        out["fallback_rows"] = nfb
    return out
