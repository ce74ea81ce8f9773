"""The C-ABI library builds, loads, and exports every symbol include/*.h declares.

CPU only: no call here reaches a CUDA kernel. The negative calls below are
rejected by host-side argument checks before any CUDA API is used.
"""
import ctypes
import glob
import os
import re

import pytest

import llama_decoder_forward_fwd_b200 as L
from llama_decoder_forward_fwd_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"\b(llm_\w+)\s*\(", src)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load()


def test_header_declares_the_boundary_calls():
    names = declared_functions()
    for required in ("llm_model_init", "llm_prefill", "llm_decode_step", "llm_kv_cache_reset", "llm_model_free"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_bounds_checking_build_loads_with_the_same_symbols(lib):
    """The -DLLM_BOUNDS_CHECK build exports the same calls and says what it is
    (llm_build_flags is a host-only query)."""
    B.build()
    checked = ctypes.CDLL(B.LIB_CHECKED)
    for name in declared_functions():
        assert hasattr(checked, name), name
    checked.llm_build_flags.restype = ctypes.c_int
    assert checked.llm_build_flags() == L.LLM_BUILD_BOUNDS_CHECK
    assert lib.llm_build_flags() == 0


def test_binding_covers_every_declared_symbol():
    assert sorted(L.exported_symbols()) == declared_functions()


def test_config_struct_layout_matches_header():
    # 10 ints, 2 floats, 4 ints
    assert ctypes.sizeof(L.llm_config) == 16 * 4
    assert ctypes.sizeof(L.llm_weights) == 12 * ctypes.sizeof(ctypes.c_void_p)


def test_null_arguments_are_rejected_on_the_host(lib):
    h = ctypes.c_void_p()
    assert lib.llm_model_init(None, None, None, ctypes.byref(h)) == L.LLM_ERR_NULL_PTR
    assert h.value is None
    assert lib.llm_model_init(None, None, None, None) == L.LLM_ERR_NULL_PTR
    assert b"NULL" in lib.llm_last_error()
    assert lib.llm_debug_wait_probe(None, 0, ctypes.c_double(1.0)) == L.LLM_ERR_NULL_PTR
    assert lib.llm_prefill(None, None, 1, 1, None, None) == L.LLM_ERR_NULL_PTR
    assert lib.llm_decode_step(None, 1, None, None, None) == L.LLM_ERR_NULL_PTR
    assert lib.llm_kv_cache_reset(None) == L.LLM_ERR_NULL_PTR
    assert lib.llm_synchronize(None) == L.LLM_ERR_NULL_PTR
    assert lib.llm_op_gemm_bf16(None, None, None, 1, 256, 64, None) == L.LLM_ERR_NULL_PTR
    lib.llm_model_free(None)


def test_inconsistent_configs_are_rejected_on_the_host(lib):
    import seeded_inputs as S
    shape = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape
    w = L.llm_weights()
    h = ctypes.c_void_p()
    bad = [dict(n_kv_heads=5), dict(head_dim=64), dict(dtype=7), dict(max_batch=0), dict(max_batch=17)]
    for kw in bad:
        cfg = L.make_config(shape, max_batch=1)
        for k, v in kw.items():
            setattr(cfg, k, v)
        assert lib.llm_model_init(ctypes.byref(cfg), ctypes.byref(w), None, ctypes.byref(h)) == L.LLM_ERR_BAD_CONFIG, kw


def test_op_shape_checks_are_host_side(lib):
    p = ctypes.c_void_p(16)  # never dereferenced: the shape check fails first
    assert lib.llm_op_gemm_bf16(p, p, p, 4, 100, 64, None) == L.LLM_ERR_BAD_ARG     # N % 256
    assert lib.llm_op_gemm_bf16(p, p, p, 4, 256, 60, None) == L.LLM_ERR_BAD_ARG     # K % 64
    assert lib.llm_op_gemv_bf16(p, p, p, 17, 16, 64, p, 1 << 20, None) == L.LLM_ERR_BAD_ARG  # M > 16
    assert lib.llm_op_attention_decode_workspace(1, 1, 32, 8, 128) > 0
    assert lib.llm_op_attention_decode_workspace(1, 1, 30, 8, 128) == 0             # H % Hk


@pytest.mark.parametrize("B,T,H,Hk,d,items,rows", [
    (1, 1, 32, 8, 128, 8, 4),    # GQA decode: each of 8 KV heads has one item of its 4 query heads
    (1, 5, 12, 3, 64, 6, 16),    # G = 4, T = 5: 4 whole tokens (16 rows) + 1 token, per KV head
    (1, 1, 32, 1, 128, 2, 16),   # multi-query decode: 32 rows of one token -> 2 items of 16
    (1, 2, 24, 1, 128, 3, 16),   # G = 24, T = 2: 48 rows -> 3 items, the second straddles the tokens
    (2, 3, 32, 1, 48, 12, 16),   # 96 rows per sequence -> 6 items, 2 sequences
])
def test_split_kv_workspace_follows_the_16_row_work_items(lib, B, T, H, Hk, d, items, rows):
    """The workspace is sized for the plan's work items (sequence, KV head, up to 16
    (token, head) rows) at the largest split count, 64: per item, split and row slot
    one record (m, l, 2 pad, o[d]) of floats, then one merge counter per item."""
    part = items * rows * 64 * (d + 4) * 4
    expect = ((part + 255) & ~255) + items * 4
    assert lib.llm_op_attention_decode_workspace(B, T, H, Hk, d) == expect


@pytest.mark.parametrize("n_kv_heads", [32, 8, 2, 1])
def test_any_query_group_size_passes_config_validation(lib, n_kv_heads):
    """Multi-head, grouped-query and multi-query configs are all valid: with no
    weights given, init gets past the config checks and stops at the missing
    weights (before touching a device); a head count that does not divide is not."""
    import seeded_inputs as S
    shape = S.WORKLOADS["llama3-8b-bf16-b1-p2048-g256"].shape
    w = L.llm_weights()
    h = ctypes.c_void_p()
    cfg = L.make_config(shape.replace(n_kv_heads=n_kv_heads), max_batch=1)
    assert lib.llm_model_init(ctypes.byref(cfg), ctypes.byref(w), None, ctypes.byref(h)) == L.LLM_ERR_NULL_PTR
    assert b"weight" in lib.llm_last_error()
    cfg = L.make_config(shape.replace(n_kv_heads=3), max_batch=1)
    assert lib.llm_model_init(ctypes.byref(cfg), ctypes.byref(w), None, ctypes.byref(h)) == L.LLM_ERR_BAD_CONFIG
