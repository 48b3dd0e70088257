"""Seeded synthetic inputs for Condensate attention.

This module only draws random numbers and plants structure (needle keys, an
anchor bias, per-query windows).  It holds none of the method's arithmetic:
no scores, no selection, no softmax.  Both the CPU oracle (through the tests)
and the CUDA path consume exactly the arrays produced here.

Shapes follow the workloads of "The Condensate Theorem: Transformers are O(n),
Not O(n^2)" as described on the pages (GPT-2-small, Mistral-7B and Llama head
layouts; W=64, k=32 from page 1 §5.1.1; 131K / 1M context from page 1 §5.1.2
table).  Recipe (one numpy PCG64 stream per workload):

  1. Q ~ N(0,1), then K ~ N(0,1), then V ~ N(0,1), each drawn as float32 in
     (b, head) slab order.
  2. needle positions (integers), then needle noise (normals), then the
     RepScore draws r_i ~ U[0,1) for adaptive windows.
  3. needles and the anchor bias are applied in float32, then bf16 workloads
     are rounded once to bfloat16 (round to nearest even).

The oracle receives the rounded values widened to float32 (exact), the GPU
receives the bf16 bit patterns.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "get", "generate", "bf16_round", "bf16_bits",
    "bits_to_f32",
]


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); float32 out."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits(x_rounded: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are already bf16-exact."""
    u = np.ascontiguousarray(x_rounded, dtype=np.float32).view(np.uint32)
    return (u >> np.uint32(16)).astype(np.uint16)


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass(frozen=True)
class Workload:
    """One synthetic workload.

    kind: "prefill" (causal, n queries over n keys) or "decode" (one query per
    head at position L-1 over an L-long cache).
    needle_mode:
      "per_query"   - per 64-query block, `needles` keys K_j = 3 q_{i*} + 0.1 N(0,1)
                      for a drawn query i* of the block and j in [1, i*-W].
      "block_mean"  - per 128-query block b >= 1, `needles` keys
                      K_j = 3 mean(q_block) + 0.1 N(0,1) at j in [1, 128 b - needle_gap].
      "decode"      - per kv-head, `needles` keys K_j = 3 q_h (q-heads of the
                      group assigned round robin) at j in [1, L-1-W]; and
                      K_0 += 2 qbar / |qbar| with qbar the group's mean query.
    """
    name: str
    kind: str
    dtype: str  # "f32" or "bf16"
    B: int
    Hq: int
    Hkv: int
    d: int
    n: int  # prefill: sequence length; decode: KV length L
    W: int
    k: int
    seed: int
    needles: int = 0
    needle_mode: str = "none"
    needle_gap: int = 0
    adaptive: bool = False  # per-query W_i = floor(64 + 192 r_i + 0.5)
    description: str = ""

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def W_max(self) -> int:
        return 256 if self.adaptive else self.W

    @property
    def C_max(self) -> int:
        return 1 + self.W_max + self.k


WORKLOADS = {
    "tiny_prefill_f32": Workload(
        "tiny_prefill_f32", "prefill", "f32", B=1, Hq=1, Hkv=1, d=64, n=512,
        W=64, k=16, seed=1, needles=4, needle_mode="per_query",
        description="tiny causal prefill, fp32, 1 head, d=64, n=512, W=64, k=16"),
    "decode_131k": Workload(
        "decode_131k", "decode", "bf16", B=1, Hq=32, Hkv=8, d=128, n=131072,
        W=128, k=64, seed=2, needles=32, needle_mode="decode",
        description="decode, bf16 KV, 32 q heads / 8 kv heads, d=128, "
                    "KV length 131072, W=128, k=64"),
    "prefill_gpt2s_8k": Workload(
        "prefill_gpt2s_8k", "prefill", "bf16", B=4, Hq=12, Hkv=12, d=64,
        n=8192, W=64, k=32, seed=3, needles=8, needle_mode="block_mean",
        needle_gap=64,
        description="causal prefill, bf16, GPT-2-small shape: batch 4, "
                    "12 heads, d=64, n=8192, W=64, k=32"),
    "decode_1m": Workload(
        "decode_1m", "decode", "bf16", B=1, Hq=32, Hkv=8, d=128, n=1048576,
        W=256, k=128, seed=4, needles=64, needle_mode="decode",
        description="decode at 1M context, bf16, Mistral-7B shape: "
                    "32 q heads / 8 kv heads, d=128, W=256, k=128"),
    "prefill_adaptive_32k": Workload(
        "prefill_adaptive_32k", "prefill", "bf16", B=1, Hq=32, Hkv=32,
        d=128, n=32768, W=256, k=64, seed=5, needles=8,
        needle_mode="block_mean", needle_gap=256, adaptive=True,
        description="adaptive-window causal prefill, bf16, Llama shape: "
                    "32 heads, d=128, n=32768, k=64, "
                    "W_i = 64 + 192 RepScore_i"),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


def _normal_slabs(rng, B, H, rows, d):
    out = np.empty((B, H, rows, d), dtype=np.float32)
    for b in range(B):
        for h in range(H):
            out[b, h] = rng.standard_normal((rows, d), dtype=np.float32)
    return out


def generate(w: Workload, seed: Optional[int] = None) -> dict:
    """Draw the inputs of workload `w`.

    Returns a dict with float32 arrays "Q", "K", "V" holding the exact input
    values (bf16-exact for bf16 workloads), "W_i" (int32 [B, n_q] or None),
    and "needles": list of (b, head, query_pos, key_pos) planted keys, where
    head is the q-head the needle was aimed at.
    """
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    nq = 1 if w.kind == "decode" else w.n
    Q = _normal_slabs(rng, w.B, w.Hq, nq, w.d)
    K = _normal_slabs(rng, w.B, w.Hkv, w.n, w.d)
    V = _normal_slabs(rng, w.B, w.Hkv, w.n, w.d)
    G = w.G

    # ---- needle positions (integers only) ----
    plan = []  # (b, hq, kvh, query_pos, key_pos, kind)
    if w.needle_mode == "per_query":
        for b in range(w.B):
            for h in range(w.Hq):
                used = set()
                for blk in range((w.n + 63) // 64):
                    lo = max(64 * blk, w.W + 1)
                    hi = min(64 * blk + 63, w.n - 1)
                    if lo > hi:
                        continue
                    for _ in range(w.needles):
                        istar = int(rng.integers(lo, hi + 1))
                        span = istar - w.W  # key positions 1..istar-W
                        if len(used) >= w.n:
                            break
                        while True:
                            j = int(rng.integers(1, span + 1))
                            if j not in used:
                                break
                            if all(x in used for x in range(1, span + 1)):
                                j = -1
                                break
                        if j < 0:
                            continue
                        used.add(j)
                        plan.append((b, h, h // G, istar, j, "q"))
    elif w.needle_mode == "block_mean":
        for b in range(w.B):
            for h in range(w.Hq):
                used = set()
                for blk in range(1, (w.n + 127) // 128):
                    span = 128 * blk - w.needle_gap
                    if span < 1:
                        continue
                    # spans grow with the block index, so every used
                    # position lies inside the current span
                    avail = span - len(used)
                    cnt = min(w.needles, avail)
                    if cnt <= 0:
                        continue
                    picks = []
                    while len(picks) < cnt:
                        j = int(rng.integers(1, span + 1))
                        if j in used:
                            continue
                        used.add(j)
                        picks.append(j)
                    for j in picks:
                        plan.append((b, h, h // G, 128 * blk, j, "mean"))
    elif w.needle_mode == "decode":
        hi = w.n - 1 - w.W
        for b in range(w.B):
            for g in range(w.Hkv):
                cnt = min(w.needles, max(0, hi))
                if cnt <= 0:
                    continue
                pos = rng.choice(hi, size=cnt, replace=False) + 1
                for m, j in enumerate(pos.tolist()):
                    plan.append((b, g * G + (m % G), g, w.n - 1, int(j), "q"))
    elif w.needle_mode != "none":
        raise ValueError(w.needle_mode)

    # ---- needle noise (normals), then placement ----
    for (b, h, g, qi, j, kind) in plan:
        if w.needle_mode == "decode":
            K[b, g, j] = 3.0 * Q[b, h, 0]
            continue
        noise = rng.standard_normal(w.d, dtype=np.float32)
        if kind == "q":
            K[b, g, j] = 3.0 * Q[b, h, qi] + np.float32(0.1) * noise
        else:
            blk_q = Q[b, h, qi:min(qi + 128, w.n)]
            K[b, g, j] = 3.0 * blk_q.mean(axis=0, dtype=np.float32) \
                + np.float32(0.1) * noise
    if w.needle_mode == "decode":
        for b in range(w.B):
            for g in range(w.Hkv):
                qbar = Q[b, g * G:(g + 1) * G, 0].mean(axis=0, dtype=np.float32)
                nrm = np.float32(np.sqrt(np.sum(qbar.astype(np.float64) ** 2)))
                if nrm > 0:
                    K[b, g, 0] = K[b, g, 0] + np.float32(2.0) * qbar / nrm

    # ---- RepScore draws for adaptive windows ----
    W_i = None
    if w.adaptive:
        r = rng.random((w.B, nq))
        W_i = np.floor(64.0 + 192.0 * r + 0.5).astype(np.int32)

    if w.dtype == "bf16":
        Q, K, V = bf16_round(Q), bf16_round(K), bf16_round(V)
    if w.kind == "decode":
        Q = Q.reshape(w.B, w.Hq, w.d)
    needles = [(b, h, qi, j) for (b, h, g, qi, j, kind) in plan]
    return {"Q": Q, "K": K, "V": V, "W_i": W_i, "needles": needles}
