"""Pins for the CPU oracle, independent of the oracle's own code.

Each test checks the oracle against something the pages or the mathematics
fix: brute-force subset enumeration, a library softmax, closed forms, the
integers printed on page 1 of "Condensate Theorem（冷凝定理）：注意力稀疏性的拓扑
本质" (§4.2.1, §4.2.2, §4.4 tables), the §3.2.1 Lemma, §3.2.4 Theorem 4 and
planted-needle membership.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

HERE = os.path.dirname(os.path.abspath(__file__))


def _rand(shape, seed, integer=False):
    rng = np.random.default_rng(seed)
    if integer:
        return rng.integers(-2, 3, size=shape).astype(np.float32)
    return rng.standard_normal(shape).astype(np.float32)


def _topk_part(idx_row, count, i, W):
    """Entries of an ascending Condensate Set lying in cand_i = [1, i-W]."""
    row = idx_row[:count]
    return [int(j) for j in row if 1 <= j <= i - W]


# ---------------------------------------------------------------- selection
@pytest.mark.parametrize("W", [1, 2, 3])
@pytest.mark.parametrize("k", [0, 1, 2, 3, 4])
def test_topk_matches_brute_force_enumeration(W, k):
    """§2.2.3 Dynamic Top-k with ties to the lower index, on integer inputs
    where ties are frequent: the unique subset T of size m_i such that every
    member beats every non-member under (score desc, index asc)."""
    n, d = 11, 4
    Q = _rand((1, 1, n, d), 100 + W * 10 + k, integer=True)
    K = _rand((1, 1, n, d), 200 + W * 10 + k, integer=True)
    V = _rand((1, 1, n, d), 300 + W * 10 + k)
    out = oracle.prefill(Q, K, V, W, k, with_full=False)
    for i in range(n):
        t = [int(round(float(np.dot(Q[0, 0, i].astype(np.int64),
                                    K[0, 0, j].astype(np.int64)))))
             for j in range(i + 1)]
        cand = list(range(1, i - W + 1))
        m = min(k, len(cand))

        def beats(a, b):
            return t[a] > t[b] or (t[a] == t[b] and a < b)

        valid = []
        for T in itertools.combinations(cand, m):
            rest = [u for u in cand if u not in T]
            if all(beats(a, b) for a in T for b in rest):
                valid.append(sorted(T))
        assert len(valid) == 1
        got = _topk_part(out["idx"][i], out["count"][i], i, W)
        assert got == valid[0], (i, got, valid[0])


def test_lemma_excluded_scores_below_threshold():
    """§3.2.1 Lemma: every excluded candidate scores at most tau_min, and on
    equality it has a higher index than the selected entry it ties."""
    B, H, n, d, W, k = 1, 2, 300, 8, 16, 12
    Q = _rand((B, H, n, d), 1, integer=True)
    K = _rand((B, H, n, d), 2, integer=True)
    V = _rand((B, H, n, d), 3)
    out = oracle.prefill(Q, K, V, W, k, with_full=False)
    r = 0
    for h in range(H):
        t = K[0, h].astype(np.float64) @ Q[0, h].astype(np.float64).T  # [j, i]
        for i in range(n):
            sel = _topk_part(out["idx"][r], out["count"][r], i, W)
            cand = range(1, i - W + 1)
            if sel:
                tau = min(t[j, i] for j in sel)
                last = max(j for j in sel if t[j, i] == tau)
                for j in cand:
                    if j in sel:
                        continue
                    assert t[j, i] <= tau
                    if t[j, i] == tau:
                        assert j > last
            r += 1


# ---------------------------------------------------------------- set size
def test_set_size_finite_support():
    """§2.4 Corollary 2 under the Top-k convention: |C_i| = min(i+1, 1+W+k);
    sets are ascending, distinct, padded with -1, hold the anchor and window."""
    n, d = 200, 8
    Q = _rand((1, 1, n, d), 4)
    K = _rand((1, 1, n, d), 5)
    V = _rand((1, 1, n, d), 6)
    for W, k in [(1, 0), (1, 5), (7, 3), (64, 32), (250, 4), (3, 500)]:
        out = oracle.prefill(Q, K, V, W, k, with_full=False)
        for i in range(n):
            c = out["count"][i]
            assert c == min(i + 1, 1 + W + k)
            row = out["idx"][i]
            assert np.all(row[c:] == -1)
            s = row[:c]
            assert np.all(np.diff(s) > 0)
            assert s[0] == 0 and s[-1] == i
            lo = max(0, i - W + 1)
            assert set(range(lo, i + 1)) <= set(s.tolist())


def _golden_sizes():
    rows = []
    with open(os.path.join(HERE, "golden", "condensate_set_sizes.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            src, n, W, k, size, pct, kind = line.split()
            rows.append((src, int(n), int(W), int(k), int(size), pct, kind))
    return rows


@pytest.mark.parametrize("row", _golden_sizes(), ids=lambda r: r[0])
def test_printed_set_sizes(row):
    """The integers of page 1 §4.2.1, §4.2.2 and §4.4 follow from the oracle's
    set at the last position of an n-token sequence with W=64, k=32."""
    src, n, W, k, size, pct, kind = row
    d = 4
    rng = np.random.default_rng(n)
    q = rng.standard_normal((1, 1, d)).astype(np.float32)
    K = rng.standard_normal((1, 1, n, d)).astype(np.float32)
    V = rng.standard_normal((1, 1, n, d)).astype(np.float32)
    out = oracle.decode(q, K, V, W, k, with_full=False)
    c = int(out["count"][0])
    assert c == size
    decimals = len(pct.split(".")[1]) if "." in pct else 0
    if kind == "coverage":
        assert f"{100.0 * c / n:.{decimals}f}" == pct
    elif kind == "sparsity":
        assert f"{100.0 * (1 - c / n):.{decimals}f}" == pct
    elif kind == "excluded":
        assert n - c == int(pct)
    else:
        raise AssertionError(kind)


def test_printed_1k_sparsity_is_inconsistent():
    """Page 1 §4.4 and §5.1.2 print 93.7% sparsity at 1K; the set-size
    formula gives 90.5%.  Recorded, not pinned."""
    assert f"{100 * (1 - 97 / 1024):.1f}" == "90.5"


def test_theoretical_speedup_131k():
    """Page 1 §5.1.1: n/97 = 1351x at n = 131,072 (set size from the oracle)."""
    n, d = 131072, 2
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 1, d)).astype(np.float32)
    K = rng.standard_normal((1, 1, n, d)).astype(np.float32)
    out = oracle.decode(q, K, K, 64, 32, with_full=False)
    assert int(n / out["count"][0]) == 1351


# ---------------------------------------------------------------- outputs
def _sdpa_causal(Q, K, V):
    q = torch.from_numpy(Q.astype(np.float64))
    k = torch.from_numpy(K.astype(np.float64))
    v = torch.from_numpy(V.astype(np.float64))
    return torch.nn.functional.scaled_dot_product_attention(
        q, k, v, is_causal=True).numpy()


@pytest.mark.parametrize("W,k", [(1, 10_000), (5, 10_000), (10_000, 0)])
def test_equals_full_attention_when_set_covers_all(W, k):
    """With k >= |cand_i| (or W >= n) C_i = [0, i], so the output equals the
    full causal softmax attention of §1.1 (torch's library routine)."""
    B, H, n, d = 2, 2, 96, 16
    Q = _rand((B, H, n, d), 8)
    K = _rand((B, H, n, d), 9)
    V = _rand((B, H, n, d), 10)
    out = oracle.prefill(Q, K, V, W, k, C_max=n, with_full=False)
    ref = _sdpa_causal(Q, K, V).reshape(-1, d)
    np.testing.assert_allclose(out["o"], ref, rtol=1e-12, atol=1e-12)


def test_two_term_closed_form():
    """k = 0, W = 1: C_i = {0, i}; the output is the two-term softmax."""
    n, d = 40, 16
    Q = _rand((1, 1, n, d), 11)
    K = _rand((1, 1, n, d), 12)
    V = _rand((1, 1, n, d), 13)
    out = oracle.prefill(Q, K, V, 1, 0, with_full=False)
    for i in range(n):
        q = Q[0, 0, i].astype(np.float64)
        if i == 0:
            exp = V[0, 0, 0].astype(np.float64)
        else:
            s0 = q @ K[0, 0, 0].astype(np.float64) / math.sqrt(d)
            si = q @ K[0, 0, i].astype(np.float64) / math.sqrt(d)
            a0 = 1.0 / (1.0 + math.exp(si - s0))
            exp = (a0 * V[0, 0, 0].astype(np.float64)
                   + (1 - a0) * V[0, 0, i].astype(np.float64))
        np.testing.assert_allclose(out["o"][i], exp, rtol=1e-12, atol=1e-13)
        assert list(out["idx"][i][:out["count"][i]]) == sorted({0, i})


def test_uniform_scores_closed_forms():
    """All keys equal: A is uniform, anchor mass 1/(i+1), window mass
    min(W, i+1)/(i+1), Top-k = [1..m_i] by the tie rule, sparse output = mean
    of V over C_i, full output = mean of V over [0, i], and the softmax
    normaliser log sum_j exp(s_j) = s + log(i+1) with s = q.k/sqrt(d)."""
    n, d, W, k = 150, 8, 10, 7
    Q = _rand((1, 1, n, d), 14)
    K = np.tile(_rand((1, 1, 1, d), 15), (1, 1, n, 1))
    V = _rand((1, 1, n, d), 16)
    out = oracle.prefill(Q, K, V, W, k)
    for i in range(n):
        c = out["count"][i]
        s = out["idx"][i][:c]
        lo = max(0, i - W + 1)
        m = min(k, max(0, i - W))
        assert list(s) == sorted(set([0] + list(range(1, m + 1))
                                     + list(range(lo, i + 1))))
        assert out["anchor_mass"][i] == pytest.approx(1 / (i + 1), rel=1e-12)
        assert out["window_mass"][i] == pytest.approx(
            min(W, i + 1) / (i + 1), rel=1e-12)
        assert out["excluded_mass"][i] == pytest.approx(
            (i + 1 - c) / (i + 1), abs=1e-12)
        s_i = float(np.dot(Q[0, 0, i].astype(np.float64),
                           K[0, 0, 0].astype(np.float64))) / math.sqrt(d)
        assert out["lse"][i] == pytest.approx(s_i + math.log(i + 1),
                                              rel=1e-12, abs=1e-12)
        np.testing.assert_allclose(out["o"][i],
                                   V[0, 0, s].astype(np.float64).mean(0),
                                   rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(out["o_full"][i],
                                   V[0, 0, :i + 1].astype(np.float64).mean(0),
                                   rtol=1e-12, atol=1e-13)


def test_masses_partition_and_theorem4():
    """§2.2 masses partition the causal softmax (anchor + window + Top-k +
    excluded = 1 once the window leaves the anchor), §3.2.4 Theorem 4 holds in
    the form |o_C - o_full|_2 <= 2 eps max_j |v_j|_2, and the cosine report
    is consistent with the error."""
    w = workloads.get("tiny_prefill_f32")
    x = workloads.generate(w)
    out = oracle.prefill(x["Q"], x["K"], x["V"], w.W, w.k)
    i = np.arange(w.n)
    far = i - w.W + 1 > 0
    tot = (out["anchor_mass"] + out["window_mass"] + out["topk_mass"]
           + out["excluded_mass"])
    np.testing.assert_allclose(tot[far], 1.0, atol=1e-12)
    assert np.all(out["err_l2"] <= 2 * out["excluded_mass"] * out["vmax_l2"]
                  + 1e-12)
    assert np.all(out["cos"] <= 1 + 1e-12)
    near = out["excluded_mass"] < 1e-9
    assert np.all(out["cos"][near] > 1 - 1e-9)


def test_planted_needles_are_selected():
    """A key planted as 3 q_i* + noise inside cand_i* scores far above the
    N(0, d) background and must be in C_i* (the needle test of §4.3)."""
    w = workloads.get("tiny_prefill_f32")
    x = workloads.generate(w)
    out = oracle.prefill(x["Q"], x["K"], x["V"], w.W, w.k, with_full=False)
    assert len(x["needles"]) > 0
    per_row = {}
    for (b, h, i, j) in x["needles"]:
        per_row.setdefault(i, []).append(j)
    for i, js in per_row.items():
        if len(js) > w.k:
            continue
        s = set(out["idx"][i][:out["count"][i]].tolist())
        for j in js:
            assert j in s, (i, j)


def test_decode_matches_prefill_last_row():
    """Decode at L-1 is the last prefill row (position convention)."""
    B, Hq, Hkv, L, d, W, k = 2, 4, 2, 120, 8, 9, 5
    Q = _rand((B, Hq, L, d), 17)
    K = _rand((B, Hkv, L, d), 18)
    V = _rand((B, Hkv, L, d), 19)
    pre = oracle.prefill(Q, K, V, W, k, sel=[(b, h, L - 1) for b in range(B)
                                           for h in range(Hq)])
    dec = oracle.decode(np.ascontiguousarray(Q[:, :, L - 1]), K, V, W, k)
    np.testing.assert_array_equal(pre["idx"], dec["idx"])
    np.testing.assert_allclose(pre["o"], dec["o"], rtol=0, atol=0)


def test_gqa_kv_head_mapping():
    """q-head h reads kv-head h // G: running each kv-head's q-heads with that
    kv-head alone gives identical results."""
    B, Hq, Hkv, n, d, W, k = 1, 4, 2, 64, 8, 4, 6
    Q = _rand((B, Hq, n, d), 20)
    K = _rand((B, Hkv, n, d), 21)
    V = _rand((B, Hkv, n, d), 22)
    full = oracle.prefill(Q, K, V, W, k, with_full=False)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        one = oracle.prefill(Q[:, h:h + 1], K[:, g:g + 1], V[:, g:g + 1], W, k,
                             with_full=False)
        np.testing.assert_array_equal(full["idx"][h * n:(h + 1) * n],
                                      one["idx"])


def test_adaptive_window_rows():
    """§2.4 Corollary 3: a per-query W_i changes only that row's window and
    candidate range; each row equals a fixed-W run with W = W_i."""
    n, d, k = 120, 8, 5
    Q = _rand((1, 1, n, d), 23)
    K = _rand((1, 1, n, d), 24)
    V = _rand((1, 1, n, d), 25)
    W_i = np.random.default_rng(26).integers(1, 40, size=(1, n)).astype(
        np.int32)
    ad = oracle.prefill(Q, K, V, 0, k, W_i=W_i, with_full=False)
    for i in range(n):
        Wr = int(W_i[0, i])
        fx = oracle.prefill(Q, K, V, Wr, k, sel=[(0, 0, i)], C_max=1 + 39 + k,
                            with_full=False)
        assert list(ad["idx"][i]) == list(fx["idx"][0])
        np.testing.assert_array_equal(ad["o"][i], fx["o"][0])


def test_gap_and_bound_reports():
    """The boundary gap is t(m-th selected) - t(best unselected) >= 0, +inf
    when nothing is left out; the rounding bound is small and non-negative."""
    w = workloads.get("tiny_prefill_f32")
    x = workloads.generate(w)
    out = oracle.prefill(x["Q"], x["K"], x["V"], w.W, w.k, with_full=False)
    assert np.all(out["gap"] >= 0)
    none_left = out["m"] >= np.maximum(0, np.arange(w.n) - w.W)
    assert np.all(np.isinf(out["gap"][none_left]))
    assert np.all(out["bound"] >= 0) and np.all(out["bound"] < 1e-2)
