"""bench.py's algorithmic work per launch, which the roofline fractions
divide by, pinned to the figures that follow from each workload's sizes."""
import importlib.util
import os

import workloads

_spec = importlib.util.spec_from_file_location(
    "bench", os.path.join(os.path.dirname(os.path.dirname(__file__)),
                          "bench.py"))
bench = importlib.util.module_from_spec(_spec)
_spec.loader.exec_module(bench)


def test_decode_bytes():
    # K scored: 8 kv heads x L x 128 dims x 2 bytes; C_i rows: 32 q heads x
    # (1 + W + k) x (K and V) x 128 x 2
    m = bench.work_model(workloads.get("decode_131k"))
    assert m["decode_score_topk"][:2] == ("hbm", 268_435_456)
    assert m["decode_merge_attend"][:2] == ("hbm", 3_162_112)
    m = bench.work_model(workloads.get("decode_1m"))
    assert m["decode_score_topk"][:2] == ("hbm", 2_147_483_648)
    assert m["decode_merge_attend"][:2] == ("hbm", 6_307_840)


def test_prefill_score_flops():
    # B*H*d*n*(n+1): a multiply and an add per (q, k) pair of the causal
    # triangle, n(n+1)/2 pairs
    m = bench.work_model(workloads.get("prefill_gpt2s_8k"))
    assert m["prefill_score_topk_tc"][:2] == ("tensor", 206_183_596_032)
    m = bench.work_model(workloads.get("prefill_adaptive_32k"))
    assert m["prefill_score_topk_tc"][:2] == ("tensor", 4_398_180_728_832)


def test_prefill_gather_bytes_at_8k():
    # 393,216 query rows (4 x 12 x 8192), d = 64, k = 32, |C| = 97:
    # Q, K, V bf16 read; Top-k keys (8 bytes) read; idx (int32 x 97), the
    # count and the fp32 output row written
    rows = 4 * 12 * 8192
    parts = {
        "Q": rows * 64 * 2, "K": rows * 64 * 2, "V": rows * 64 * 2,
        "keys": rows * 32 * 8, "idx": rows * 97 * 4, "count": rows * 4,
        "O": rows * 64 * 4,
    }
    m = bench.work_model(workloads.get("prefill_gpt2s_8k"))
    assert m["prefill_gather"][:2] == ("hbm", sum(parts.values()))
    assert sum(parts.values()) == 506_462_208


def test_step_units_are_tokens():
    assert bench.step_units(workloads.get("decode_131k")) == 1
    assert bench.step_units(workloads.get("prefill_gpt2s_8k")) == 4 * 8192


def test_capture_hash_follows_code_only():
    # a recorded ncu capture stays valid across comment and layout edits and
    # is voided by any code edit
    code = "int f(int x) {\n  return x + 1;  // one more\n}\n"
    same = "/* header */\nint f(int x) {\n    return x + 1;\n}  // end\n"
    other = "int f(int x) {\n  return x + 2;  // one more\n}\n"
    assert bench._code_only(code) == bench._code_only(same)
    assert bench._code_only(code) != bench._code_only(other)
    assert bench._code_only('asm("mov.u32 %0, %1;")') == 'asm("mov.u32 %0, %1;")'
