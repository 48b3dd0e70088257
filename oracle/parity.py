"""Row-by-row comparison of the CUDA path's results with the CPU oracle
(test infrastructure, like the rest of this package: used by the tests, the
smoke check and the benchmark's CPU leg).

Index sets must be identical row by row, except rows whose boundary gap (the
m-th selected score minus the best unselected score, in exact arithmetic) is
within the fp32 rounding bound of the two scores involved: there the GPU may
pick a different, equally valid member, and the test checks that every
swapped pair lies inside that bound.  Outputs are compared with the oracle's
double-precision result; for a row whose set was validly swapped the
expected output is the double-precision softmax over the GPU's set.
"""
import os

import numpy as np

# Summaries of every comparison made in this process, with the test (or
# caller) that made it, for the test session's closing report.
RECORDS = []


def _t(q, Krows):
    return Krows.astype(np.float64) @ q.astype(np.float64)


def check_rows(ref, got_idx, got_cnt, got_o, q_rows, kv_rows, v_rows, pos,
               win, tol):
    """ref: oracle dict for R rows; got_*: numpy arrays for the same rows.

    q_rows[r]: query vector of row r; kv_rows(r) / v_rows(r): the K / V
    arrays ([L, d]) that row r reads; pos[r], win[r]: position and window.
    Returns a summary dict; raises AssertionError on any violation.
    """
    R = len(pos)
    got_idx = np.asarray(got_idx).reshape(R, -1)
    got_cnt = np.asarray(got_cnt).reshape(R)
    got_o = np.asarray(got_o, dtype=np.float64).reshape(R, -1)
    d = got_o.shape[1]
    C = ref["idx"].shape[1]
    assert got_idx.shape[1] == C, (got_idx.shape, C)
    np.testing.assert_array_equal(got_cnt, ref["count"], err_msg="|C_i|")
    near = ref["gap"] <= ref["bound"]
    same = np.all(got_idx == ref["idx"], axis=1)
    bad = np.nonzero(~same & ~near)[0]
    assert bad.size == 0, (
        f"{bad.size} rows differ outside near-ties, first row {bad[0]}: "
        f"gpu {got_idx[bad[0]][:got_cnt[bad[0]]]} oracle "
        f"{ref['idx'][bad[0]][:ref['count'][bad[0]]]}")
    swapped = np.nonzero(~same)[0]
    expect = ref["o"].copy()
    for r in swapped:
        c = got_cnt[r]
        g = set(got_idx[r][:c].tolist())
        o = set(ref["idx"][r][:c].tolist())
        assert -1 not in g and len(g) == c
        K = kv_rows(r)
        t_a = _t(q_rows[r], K[sorted(o - g)])
        t_b = _t(q_rows[r], K[sorted(g - o)])
        i, w = int(pos[r]), int(win[r])
        assert all(1 <= j <= i - w for j in (g - o)), "swap outside candidates"
        assert t_a.max() - t_b.min() <= ref["bound"][r] * (1 + 1e-9), (
            "swapped pair outside the rounding bound")
        # expected output over the GPU's (valid) set, in float64
        js = np.array(sorted(g))
        t = _t(q_rows[r], K[js]) / np.sqrt(d)
        p = np.exp(t - t.max())
        expect[r] = (p[:, None] * v_rows(r)[js].astype(np.float64)).sum(0) / p.sum()
    err = np.abs(got_o - expect)
    worst = float(err.max()) if err.size else 0.0
    assert worst <= tol, f"max abs error {worst} > {tol} (row {np.argmax(err.max(1))})"
    out = {"rows": R, "near_ties": int(near.sum()),
           "swapped": int(swapped.size), "max_abs_err": worst, "tol": tol}
    who = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    RECORDS.append(dict(out, where=who))
    return out
