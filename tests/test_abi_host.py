"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every entry point the header declares, sizes workspaces, and rejects invalid
arguments before touching the device."""
import ctypes
import os
import re

import pytest

import sparse_transformer_attention_b200 as ca
from sparse_transformer_attention_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "condensate_attn.h")


def header_functions():
    text = open(HEADER).read()
    return re.findall(r"CA_API\s+[\w\s\*]+?\b(condensate_attn_\w+)\s*\(", text)


@pytest.fixture(scope="module")
def lib():
    from sparse_transformer_attention_b200 import build
    build.build()
    return binding.load()


def test_header_lists_entry_points():
    names = header_functions()
    assert set(names) == set(binding.SIGNATURES), names


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
    assert lib.condensate_attn_version() == 301
    assert lib.condensate_attn_build_flags() == 0  # the release build


def test_status_strings(lib):
    for code in range(9):
        assert ca.status_string(code)
    assert ca.status_string(0) == "ok"


def test_workspace_sizes(lib):
    ws = ca.condensate_attn_workspace_size
    import torch
    assert ws(True, torch.bfloat16, 1, 131072, 32, 8, 128, 128, 64) > 256
    assert ws(True, torch.bfloat16, 1, 131072, 32, 8, 96, 128, 64) == 0
    assert ws(True, torch.bfloat16, 1, 131072, 30, 8, 128, 128, 64) == 0
    assert ws(True, torch.bfloat16, 1, 131072, 32, 0, 128, 128, 64) == 0
    assert ws(False, torch.bfloat16, 1, 0, 32, 8, 128, 128, 64) == 0
    assert ws(False, torch.bfloat16, 0, 8192, 32, 8, 128, 128, 64) == 0
    assert ws(False, torch.bfloat16, 1, 8192, 32, 8, 128, 0, 64) == 0
    p = ws(False, torch.bfloat16, 4, 8192, 12, 12, 64, 64, 32)
    assert p >= 256 + 4 * 12 * 8192 * 32 * 8
    assert ws(True, torch.bfloat16, 1, 1 << 20, 32, 8, 128, 256, 128) < (64 << 20)


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced


def _decode(lib, **over):
    a = dict(q=FAKE, K=FAKE, V=FAKE, dtype=1, B=1, L=1000, Hq=8, Hkv=2, d=128,
             W=64, k=16, W_i=None, O=FAKE, o_dtype=0, idx=FAKE, cnt=FAKE,
             C_max=81, ws=FAKE, ws_bytes=16, stream=None)
    a.update(over)
    P = ctypes.c_void_p
    return lib.condensate_attn_decode(
        P(a["q"]), P(a["K"]), P(a["V"]), a["dtype"], a["B"], a["L"], a["Hq"],
        a["Hkv"], a["d"], a["W"], a["k"], P(a["W_i"]) if a["W_i"] else None,
        P(a["O"]), a["o_dtype"], P(a["idx"]), P(a["cnt"]), a["C_max"],
        P(a["ws"]) if a["ws"] else None, a["ws_bytes"], None)


def _prefill(lib, **over):
    a = dict(Q=FAKE, K=FAKE, V=FAKE, dtype=1, B=1, n=1000, Hq=8, Hkv=2, d=128,
             W=64, k=16, O=FAKE, o_dtype=0, idx=FAKE, cnt=FAKE, C_max=81,
             ws=FAKE, ws_bytes=16)
    a.update(over)
    P = ctypes.c_void_p
    return lib.condensate_attn_prefill(
        P(a["Q"]), P(a["K"]), P(a["V"]), a["dtype"], a["B"], a["n"], a["Hq"],
        a["Hkv"], a["d"], a["W"], a["k"], None, P(a["O"]), a["o_dtype"],
        P(a["idx"]), P(a["cnt"]), a["C_max"], P(a["ws"]) if a["ws"] else None,
        a["ws_bytes"], None)


@pytest.mark.parametrize("call", [_decode, _prefill])
@pytest.mark.parametrize("over,code", [
    ({"ws": 0}, binding.CA_ERR_WORKSPACE),
    ({"q": 0}, binding.CA_ERR_INVALID_ARG),
    ({"K": 0}, binding.CA_ERR_INVALID_ARG),
    ({"idx": 0}, binding.CA_ERR_INVALID_ARG),
    ({"cnt": 0}, binding.CA_ERR_INVALID_ARG),
    ({"L": 0}, binding.CA_ERR_INVALID_ARG),
    ({"Hkv": 0}, binding.CA_ERR_INVALID_ARG),
    ({"C_max": 0}, binding.CA_ERR_INVALID_ARG),
    ({"O": 0}, binding.CA_ERR_INVALID_ARG),
    ({"B": 0}, binding.CA_ERR_INVALID_ARG),
    ({"k": -1}, binding.CA_ERR_INVALID_ARG),
    ({"W": 0}, binding.CA_ERR_INVALID_ARG),
    ({"C_max": 80}, binding.CA_ERR_INVALID_ARG),
    ({"Hq": 7}, binding.CA_ERR_INVALID_ARG),
    ({"d": 96}, binding.CA_ERR_UNSUPPORTED),
    ({"dtype": 5}, binding.CA_ERR_UNSUPPORTED),
    ({"o_dtype": 9}, binding.CA_ERR_UNSUPPORTED),
    ({"Hq": 6, "Hkv": 2}, binding.CA_ERR_UNSUPPORTED),
    ({"Hq": 32, "Hkv": 2}, binding.CA_ERR_UNSUPPORTED),
    ({"V": FAKE + 8}, binding.CA_ERR_ALIGNMENT),
    ({"idx": FAKE + 4}, binding.CA_ERR_ALIGNMENT),
    ({}, binding.CA_ERR_WORKSPACE),  # 16 bytes is never enough
])
def test_invalid_arguments_rejected_before_launch(lib, call, over, code):
    key_map = {"q": "Q", "L": "n"} if call is _prefill else {}
    over = {key_map.get(k, k): v for k, v in over.items()}
    assert call(lib, **over) == code


def _select(lib, **over):
    a = dict(q=FAKE, K=FAKE, dtype=1, B=1, Ls=500, pos0=0, L=1000, Hq=8,
             Hkv=2, d=128, W=64, k=16, keys=FAKE, ws=FAKE, ws_bytes=16)
    a.update(over)
    P = ctypes.c_void_p
    return lib.condensate_attn_decode_shard_select(
        P(a["q"]), P(a["K"]), a["dtype"], a["B"], a["Ls"], a["pos0"], a["L"],
        a["Hq"], a["Hkv"], a["d"], a["W"], a["k"], None, P(a["keys"]),
        P(a["ws"]) if a["ws"] else None, a["ws_bytes"], None)


def _attend(lib, **over):
    a = dict(q=FAKE, K=FAKE, V=FAKE, dtype=1, B=1, Ls=500, pos0=500, L=1000,
             Hq=8, Hkv=2, d=128, W=64, k=16, keys=FAKE, P=2, part=FAKE,
             idx=FAKE, cnt=FAKE, C_max=81, ws=FAKE, ws_bytes=16)
    a.update(over)
    P = ctypes.c_void_p
    return lib.condensate_attn_decode_shard_attend(
        P(a["q"]), P(a["K"]), P(a["V"]), a["dtype"], a["B"], a["Ls"],
        a["pos0"], a["L"], a["Hq"], a["Hkv"], a["d"], a["W"], a["k"], None,
        P(a["keys"]) if a["keys"] else None, a["P"],
        P(a["part"]) if a["part"] else None, P(a["idx"]), P(a["cnt"]),
        a["C_max"], P(a["ws"]) if a["ws"] else None, a["ws_bytes"], None)


@pytest.mark.parametrize("call,over,code", [
    (_select, {"pos0": 501}, binding.CA_ERR_INVALID_ARG),   # past the end
    (_select, {"pos0": -1}, binding.CA_ERR_INVALID_ARG),
    (_select, {"Ls": 0}, binding.CA_ERR_INVALID_ARG),
    (_select, {"keys": 0}, binding.CA_ERR_INVALID_ARG),
    (_select, {"q": 0}, binding.CA_ERR_INVALID_ARG),
    (_select, {"dtype": 0}, binding.CA_ERR_UNSUPPORTED),    # bf16 only
    (_select, {"d": 96}, binding.CA_ERR_UNSUPPORTED),
    (_select, {"keys": FAKE + 8}, binding.CA_ERR_ALIGNMENT),
    (_select, {"ws": 0}, binding.CA_ERR_WORKSPACE),
    (_select, {}, binding.CA_ERR_WORKSPACE),                # 16 bytes
    (_attend, {"pos0": 501}, binding.CA_ERR_INVALID_ARG),
    (_attend, {"P": 0}, binding.CA_ERR_INVALID_ARG),
    (_attend, {"keys": 0}, binding.CA_ERR_INVALID_ARG),
    (_attend, {"part": 0}, binding.CA_ERR_INVALID_ARG),
    (_attend, {"C_max": 80}, binding.CA_ERR_INVALID_ARG),
    (_attend, {"P": 1024}, binding.CA_ERR_UNSUPPORTED),     # P k > 8192
    (_attend, {"part": FAKE + 4}, binding.CA_ERR_ALIGNMENT),
    (_attend, {}, binding.CA_ERR_WORKSPACE),                # 16 bytes
])
def test_shard_arguments_rejected_before_launch(lib, call, over, code):
    assert call(lib, **over) == code


def test_shard_combine_arguments(lib):
    P = ctypes.c_void_p
    f = lib.condensate_attn_decode_shard_combine
    assert f(P(FAKE), 0, 1, 8, 128, P(FAKE), 0, None) == \
        binding.CA_ERR_INVALID_ARG
    assert f(None, 2, 1, 8, 128, P(FAKE), 0, None) == \
        binding.CA_ERR_INVALID_ARG
    assert f(P(FAKE), 2, 1, 8, 96, P(FAKE), 0, None) == \
        binding.CA_ERR_UNSUPPORTED
    assert f(P(FAKE + 8), 2, 1, 8, 128, P(FAKE), 0, None) == \
        binding.CA_ERR_ALIGNMENT
    ws = lib.condensate_attn_decode_shard_workspace_size
    assert ws(1, 1, 65536, 32, 8, 128, 64) > 256
    assert ws(1, 1, 0, 32, 8, 128, 64) == 0


def test_k_limits(lib):
    assert _prefill(lib, k=129, C_max=1 + 64 + 129) == binding.CA_ERR_UNSUPPORTED
    assert _decode(lib, k=1025, C_max=1000) == binding.CA_ERR_UNSUPPORTED


def test_small_sequence_needs_only_n_slots(lib):
    # with n = 10 the set holds at most 10 positions: C_max = 10 passes the
    # size check and only the workspace check remains
    assert _prefill(lib, n=10, C_max=10) == binding.CA_ERR_WORKSPACE
    assert _decode(lib, L=10, C_max=10) == binding.CA_ERR_WORKSPACE


def test_product_path_has_no_oracle_or_cpu_fallback():
    src_dir = os.path.join(ROOT, "sparse_transformer_attention_b200")
    for fn in os.listdir(src_dir):
        if fn.endswith(".py"):
            text = open(os.path.join(src_dir, fn)).read()
            assert "import oracle" not in text and "from oracle" not in text
