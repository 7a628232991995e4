"""Host-side checks of the C ABI (no GPU needed): every declared symbol is exported, the
table / budget / argument checks return their documented statuses, and the arena plan and
bits-per-token agree with the oracle's cost model."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kvk():
    import __graft_entry__
    __graft_entry__.build()
    from compressed_decode_attention_kvk_b200 import kvk
    return kvk


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "kvk.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvk_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(kvk):
    declared = _declared_functions()
    assert "kvk_create_layout" in declared and "kvk_mla_decode" in declared
    out = subprocess.run(["nm", "-D", "--defined-only", kvk.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (kvk_[a-z_0-9]+)$", out, flags=re.M))
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    assert set(kvk.EXPORTED) == set(declared)
    lib = ctypes.CDLL(kvk.LIB_PATH)
    for s in declared:
        getattr(lib, s)


def test_status_strings(kvk):
    for s in range(9):
        assert kvk.kvk_status_string(s)


def _status(kvk, *args, **kw):
    try:
        kvk.kvk_create_layout(*args, **kw)
        return 0
    except kvk.KvkError as e:
        return e.status


def test_table_validation(kvk):
    ok = ([0, 0, 2, 2], [32, 0, 64, 0], [8, 0, 4, 0])
    assert _status(kvk, *ok, 64, 16, 1, 256, query_only=True) == 0
    # anchor[0] must be 0
    assert _status(kvk, [1, 1], [32, 32], [8, 8], 64, 16, 1, 256, query_only=True) == 2
    # inheriting layer must point at the nearest preceding anchor
    assert _status(kvk, [0, 1, 0], [32, 32, 0], [8, 8, 0], 64, 16, 1, 256, query_only=True) == 2
    # forward reference
    assert _status(kvk, [0, 2, 2], [32, 0, 32], [8, 0, 8], 64, 16, 1, 256, query_only=True) == 2
    # d not a multiple of 16, d > r, d < 16
    for dd in (24, 80, 0):
        assert _status(kvk, [0], [dd], [8], 64, 16, 1, 256, query_only=True) == 2
    # b outside {2, 4, 8, 16} and the uncompressed bf16 anchor (0)
    for bb in (1, 3, 5, 32, -1):
        assert _status(kvk, [0], [32], [bb], 64, 16, 1, 256, query_only=True) == 2
    # bad dims
    assert _status(kvk, [0], [32], [8], 60, 16, 1, 256, query_only=True) == 1
    assert _status(kvk, [0], [32], [8], 64, 12, 1, 256, query_only=True) == 1
    assert _status(kvk, [0], [32], [8], 64, 16, 0, 256, query_only=True) == 1
    assert _status(kvk, [0], [32], [8], 64, 16, 1, 0, query_only=True) == 1
    assert _status(kvk, [0], [32], [8], 64, 16, 5000, 256, query_only=True) == 1


def test_bits_per_token_and_budget_match_oracle(kvk, oracle_mod):
    import workloads
    for key, t in workloads.load_tables().items():
        r, dR = (64, 16) if key.startswith("tiny") else (512, 64)
        _, need, bits = kvk.kvk_create_layout(t["anchor"], t["d"], t["b"], r, dR, 2, 128,
                                              query_only=True)
        assert bits == oracle_mod.bits_per_token(t["anchor"], t["d"], t["b"], dR)
        # budget exactly at the cost passes, one bit below fails
        kvk.kvk_create_layout(t["anchor"], t["d"], t["b"], r, dR, 2, 128, bits, query_only=True)
        assert _status(kvk, t["anchor"], t["d"], t["b"], r, dR, 2, 128, bits - 1,
                       query_only=True) == 3


def test_arena_plan(kvk, oracle_mod):
    anchor, d, b = [0, 0, 2, 2, 4], [32, 0, 64, 0, 48], [8, 0, 4, 0, 16]
    B, T = 3, 100
    handle, need, _ = kvk.kvk_create_layout(anchor, d, b, 64, 16, B, T)   # planning layout
    try:
        spans = []
        for l in range(5):
            info = kvk.kvk_get_layer_info(handle, l)
            a = anchor[l]
            assert info["anchor"] == a and info["d"] == d[a] and info["b"] == b[a]
            assert info["row_bytes"] == oracle_mod.row_bytes(d[a] + 16, b[a])
            assert info["codes_offset"] % 256 == 0 and info["scales_offset"] % 256 == 0
            assert info["codes_offset"] >= 256
            if l == a:
                spans.append((info["codes_offset"], info["codes_offset"] + B * T * info["row_bytes"]))
                spans.append((info["scales_offset"], info["scales_offset"] + 2 * B * T))
            else:   # inheriting layer: same cache as its anchor, never a copy
                ia = kvk.kvk_get_layer_info(handle, a)
                assert info["codes_offset"] == ia["codes_offset"]
        spans.sort()
        for (s0, e0), (s1, e1) in zip(spans, spans[1:]):
            assert e0 <= s1
        assert spans[-1][1] <= need
    finally:
        kvk.kvk_destroy(handle)


def test_planning_layout_cannot_launch(kvk):
    import torch
    handle, _, _ = kvk.kvk_create_layout([0, 0], [32, 0], [8, 0], 64, 16, 1, 64)
    try:
        lib = kvk._lib_handle()
        # write to the inheriting layer -> KVK_ERR_INHERITING_LAYER before anything else
        st = lib.kvk_quant_write(handle, 1, ctypes.c_void_p(16), 1, 0, 0, ctypes.c_void_p(16),
                                 0, 0, 1, ctypes.c_void_p(16), 1, None)
        assert st == 4
        # anchor layer but no arena -> KVK_ERR_INVALID_ARG
        st = lib.kvk_quant_write(handle, 0, ctypes.c_void_p(16), 1, 0, 0, ctypes.c_void_p(16),
                                 0, 0, 1, ctypes.c_void_p(16), 1, None)
        assert st == 1
        st = lib.kvk_quant_write(handle, 5, None, 1, 0, 0, None, 0, 0, 1, None, 1, None)
        assert st == 1
        ws = ctypes.c_size_t(0)
        assert lib.kvk_decode_workspace_bytes(handle, 1, 1, 8, ctypes.byref(ws)) == 0
        assert ws.value > 0
        assert lib.kvk_decode_workspace_bytes(handle, 1, 2, 8, ctypes.byref(ws)) == 1  # batch > max
        wk = ctypes.c_size_t(0)
        assert lib.kvk_decode_workspace_bytes_keep(handle, 1, 1, 8, 100, ctypes.byref(wk)) == 0
        assert lib.kvk_decode_workspace_bytes(handle, 1, 1, 8, ctypes.byref(ws)) == 0
        assert wk.value > ws.value                              # room for the dense kept rows
        assert lib.kvk_decode_workspace_bytes_keep(handle, 1, 1, 8, -1, ctypes.byref(wk)) == 1
        path = ctypes.c_int(-1)
        assert lib.kvk_decode_path_for(handle, 0, 0, 8, 0, ctypes.byref(path)) == 0
        assert path.value == kvk.KVK_PATH_CUDA_CORE            # fp32 queries
        assert lib.kvk_set_decode_path(handle, 7) == 1
        assert lib.kvk_set_decode_path(handle, kvk.KVK_PATH_TENSOR_GENERAL) == 0
        assert lib.kvk_set_decode_path(handle, kvk.KVK_PATH_TENSOR_GENERAL + 1) == 1
        assert lib.kvk_set_decode_path(handle, kvk.KVK_PATH_AUTO) == 0
        assert lib.kvk_set_decode_ctas(handle, -1) == 1
        del torch
    finally:
        kvk.kvk_destroy(handle)


def test_uncompressed_bf16_anchor_layout(kvk, oracle_mod):
    """b = 0 keeps an anchor uncompressed in bf16: 16 bits per element and no scale in the
    cost (the same as the oracle's cost model), 2 bytes per element in the row."""
    anchor, d, b = [0, 0, 2, 3], [512, 0, 256, 128], [0, 0, 0, 4]
    _, need, bits = kvk.kvk_create_layout(anchor, d, b, 512, 64, 2, 64, query_only=True)
    assert bits == (512 + 64) * 16 + (256 + 64) * 16 + (128 + 64) * 4 + 16
    assert bits == oracle_mod.bits_per_token(anchor, d, b, 64)
    lay, _, _ = kvk.kvk_create_layout(anchor, d, b, 512, 64, 2, 64)
    try:
        assert kvk.kvk_get_layer_info(lay, 0)["row_bytes"] == (512 + 64) * 2
        assert kvk.kvk_get_layer_info(lay, 2)["row_bytes"] == (256 + 64) * 2
        assert kvk.kvk_get_layer_info(lay, 3)["row_bytes"] == (128 + 64) * 4 // 8
        assert kvk.kvk_get_layer_info(lay, 1)["b"] == 0
    finally:
        kvk.kvk_destroy(lay)
    # a 14B-shaped plan kept wholly uncompressed costs C_0 * 576 / 2048 (48 layers of
    # 576 bf16 elements against 48 layers of 2 x 8 x 128 bf16 keys and values)
    c0 = oracle_mod.c0_bits(48, 8, 128)
    full = oracle_mod.bits_per_token(list(range(48)), [512] * 48, [0] * 48, 64)
    assert full * 2048 == c0 * 576
