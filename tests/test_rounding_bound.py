"""Pins for the oracle's near-tie rounding bound beta_i.

The Top-k of "Condensate Theorem（冷凝定理）：注意力稀疏性的拓扑本质" §2.2.3
orders candidates by their score; a GPU computes each score t_j = q.k_j in
fp32 and may order two candidates differently from the exact (float64)
order only when their exact scores differ by less than the two rounding
errors together.  The oracle reports, per row, beta_i = gamma_d (A_sel +
A_unsel) with A = max of sum_l |q_l k_jl| over the selected and over the
unselected candidates and gamma_d = d u / (1 - d u), u = 2^-23.

The standard dot-product error bound (Higham, "Accuracy and Stability of
Numerical Algorithms", 2nd ed., §3.1, eq. (3.5)) gives |fl(q.k) - q.k| <=
gamma_d sum_l |q_l k_l| for any summation order, with u the unit roundoff of
one operation; u = 2^-23 covers round-to-nearest (2^-24) and rounding toward
zero (relative error < 2^-23) alike.  These tests compute fp32 dot products
the ways a GPU may (sequential FMA, multiply-then-add, a pairwise tree, the
decode kernel's 8-lane split with a butterfly, round-toward-zero sequences,
16-term exact chunks truncated) and check
  1. each order's error against gamma_d sum|q k| (the formula itself), and
  2. the oracle's beta_i against the realised errors (beta is never smaller
     than max selected error + max unselected error, under any order) and
     against the bound over the two worst candidates (beta is never larger
     than 2 gamma_d max_j sum|q k_j|).
Planted mistakes in beta (a smaller unit roundoff, a dropped term, a factor
10) fail one of them (tests/test_oracle_mutations.py).
"""
import numpy as np
import pytest

import oracle
import workloads

U = 2.0 ** -23


def gamma(d):
    return d * U / (1.0 - d * U)


def _f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def _rz(x):
    """Round float64 values toward zero to float32."""
    x = np.asarray(x, dtype=np.float64)
    r = x.astype(np.float32)
    over = np.abs(r.astype(np.float64)) > np.abs(x)
    r[over] = np.nextafter(r[over], np.float32(0))
    return r


def dot_orders(q, K):
    """fp32 dot products q.K[j] under several summation orders.

    q [d], K [n, d] hold exact fp32 values.  Products of two fp32 values are
    exact in float64; an fp32 sum of an fp32 value and such a product is
    formed exactly enough in float64 (error 2^-53 relative) and rounded once.
    Returns {order name: float32 [n]}.
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    n, d = K.shape
    P = K * q[None, :]  # exact products
    out = {}
    # sequential fused multiply-add, round to nearest
    acc = np.zeros(n, dtype=np.float32)
    for l in range(d):
        acc = _f32(acc.astype(np.float64) + P[:, l])
    out["fma_seq"] = acc
    # sequential multiply then add (two roundings per term)
    acc = np.zeros(n, dtype=np.float32)
    Pr = _f32(P)
    for l in range(d):
        acc = _f32(acc.astype(np.float64) + Pr[:, l].astype(np.float64))
    out["mul_add_seq"] = acc
    # pairwise tree over rounded products
    lev = Pr.astype(np.float32)
    while lev.shape[1] > 1:
        lev = _f32(lev[:, 0::2].astype(np.float64) + lev[:, 1::2].astype(np.float64))
    out["pairwise"] = lev[:, 0]
    # decode kernel: 8 lanes per key, lane l8 holds 16-byte pieces
    # l8 + 8c (8 bf16 or 4 fp32 elements each, taken as pairs into the two
    # halves of a packed accumulator), then .x + .y, then a butterfly tree
    # over the 8 lanes
    for vec, name in ((8, "decode_bf16"), (4, "decode_f32")):
        cpl = d // (8 * vec)
        if cpl < 1:
            continue
        part = []
        for l8 in range(8):
            ax = np.zeros(n, dtype=np.float32)
            ay = np.zeros(n, dtype=np.float32)
            for c in range(cpl):
                base = (l8 + 8 * c) * vec
                for p in range(vec // 2):
                    ax = _f32(ax.astype(np.float64) + P[:, base + 2 * p])
                    ay = _f32(ay.astype(np.float64) + P[:, base + 2 * p + 1])
            part.append(_f32(ax.astype(np.float64) + ay.astype(np.float64)))
        s4 = [_f32(part[j].astype(np.float64) + part[j ^ 4].astype(np.float64))
              for j in range(4)]
        s2 = [_f32(s4[j].astype(np.float64) + s4[j ^ 2].astype(np.float64))
              for j in range(2)]
        out[name] = _f32(s2[0].astype(np.float64) + s2[1].astype(np.float64))
    # sequential, every step rounded toward zero
    acc = np.zeros(n, dtype=np.float32)
    for l in range(d):
        acc = _rz(acc.astype(np.float64) + P[:, l])
    out["fma_seq_rz"] = acc
    # reversed order, toward zero
    acc = np.zeros(n, dtype=np.float32)
    for l in reversed(range(d)):
        acc = _rz(acc.astype(np.float64) + P[:, l])
    out["fma_rev_rz"] = acc
    # chunks of 16 exact products, each chunk sum and the accumulation
    # rounded toward zero (a truncating K=16 tensor-core step)
    acc = np.zeros(n, dtype=np.float32)
    for c0 in range(0, d, 16):
        chunk = _rz(P[:, c0:c0 + 16].sum(axis=1))
        acc = _rz(acc.astype(np.float64) + chunk.astype(np.float64))
    out["k16_rz"] = acc
    return out


def _exact(q, K):
    return np.asarray(K, dtype=np.float64) @ np.asarray(q, dtype=np.float64)


def _abs_sum(q, K):
    return np.abs(np.asarray(K, dtype=np.float64)) @ np.abs(
        np.asarray(q, dtype=np.float64))


def _cancel_key(q, M, rng):
    """A key whose terms are large (about M |q_l|) and cancel: sum |q k| is
    huge while q.k is near zero, so its fp32 rounding error is large."""
    d = len(q)
    s = np.sign(q)
    s[s == 0] = 1.0
    k = M * s * (1.0 + 0.01 * rng.standard_normal(d))
    half = d // 2
    a1 = np.abs(q[:half] * k[:half]).sum()
    a2 = np.abs(q[half:] * k[half:]).sum()
    k[half:] *= -a1 / a2
    return workloads.bf16_round(k.astype(np.float32))


def _inputs(d, seed, adversarial):
    rng = np.random.default_rng(seed)
    L = 300
    q = workloads.bf16_round(rng.standard_normal(d).astype(np.float32))
    K = workloads.bf16_round(rng.standard_normal((L, d)).astype(np.float32))
    V = workloads.bf16_round(rng.standard_normal((L, d)).astype(np.float32))
    if adversarial:
        for j in (3, 50, 151, 222):
            K[j] = _cancel_key(q.astype(np.float64), 100.0 * (1 + j % 7), rng)
    return q, K, V


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("adversarial", [False, True])
def test_fp32_dot_error_within_gamma_bound(d, adversarial):
    """Every summation order's error is within gamma_d sum_l |q_l k_jl|."""
    for seed in range(3):
        q, K, _ = _inputs(d, 10 * d + seed, adversarial)
        t = _exact(q, K)
        a = _abs_sum(q, K)
        for name, fl in dot_orders(q, K).items():
            err = np.abs(fl.astype(np.float64) - t)
            assert np.all(err <= gamma(d) * a), (name, float((err / a).max()))


def test_toward_zero_orders_reach_a_sizeable_part_of_the_bound():
    """The bound is not vacuous: on cancelling keys the truncating orders
    reach a sizeable fraction of gamma_d sum|q k| (so a much smaller unit
    roundoff would not be a valid bound)."""
    q, K, _ = _inputs(64, 7, True)
    t, a = _exact(q, K), _abs_sum(q, K)
    worst = 0.0
    for name, fl in dot_orders(q, K).items():
        worst = max(worst, float((np.abs(fl.astype(np.float64) - t) / a).max()))
    assert worst > gamma(64) * 2.0 ** -6, worst


def _decode_rows(d, seed, adversarial, W=4, k=8):
    q, K, V = _inputs(d, seed, adversarial)
    L = K.shape[0]
    out = oracle.decode(q[None, None], K[None, None], V[None, None], W, k,
                        with_full=False)
    return q, K, out, L - 1, W


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("adversarial", [False, True])
def test_oracle_bound_covers_every_order(d, adversarial):
    """beta_i from the oracle is at least the largest selected error plus the
    largest unselected error, under every order, and at most
    2 gamma_d max_j sum|q k_j| over the candidates."""
    for seed in range(4):
        q, K, out, i, W = _decode_rows(d, 100 * d + seed, adversarial)
        beta = float(out["bound"][0])
        C = out["idx"][0][:out["count"][0]]
        cand = np.arange(1, i - W + 1)
        sel = np.array([j for j in C if 1 <= j <= i - W])
        unsel = np.setdiff1d(cand, sel)
        assert len(sel) > 0 and len(unsel) > 0
        t = _exact(q, K)
        a = _abs_sum(q, K)
        assert beta <= 2.0 * gamma(d) * a[cand].max() * (1 + 1e-12), beta
        for name, fl in dot_orders(q, K).items():
            err = np.abs(fl.astype(np.float64) - t)
            need = err[sel].max() + err[unsel].max()
            assert need <= beta, (name, need, beta)


def test_oracle_bound_on_workload_rows():
    """The same two checks on rows of the tiny prefill workload (random
    keys with planted needles), every row with both sets non-empty."""
    w = workloads.get("tiny_prefill_f32")
    x = workloads.generate(w)
    out = oracle.prefill(x["Q"], x["K"], x["V"], w.W, w.k, with_full=False)
    K = x["K"][0, 0]
    checked = 0
    for i in range(w.W + w.k + 1, w.n, 7):
        q = x["Q"][0, 0, i]
        C = out["idx"][i][:out["count"][i]]
        cand = np.arange(1, i - w.W + 1)
        sel = np.array([j for j in C if 1 <= j <= i - w.W])
        unsel = np.setdiff1d(cand, sel)
        t = _exact(q, K[:i + 1])
        a = _abs_sum(q, K[:i + 1])
        beta = float(out["bound"][i])
        assert beta <= 2.0 * gamma(w.d) * a[cand].max() * (1 + 1e-12)
        for name, fl in dot_orders(q, K[:i + 1]).items():
            err = np.abs(fl.astype(np.float64) - t)
            assert err[sel].max() + err[unsel].max() <= beta, (i, name)
        checked += 1
    assert checked > 50
