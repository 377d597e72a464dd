"""The C-ABI library loads, exports every entry point include/spa.h declares, and rejects
bad arguments on the host (no GPU needed: validation precedes any CUDA call)."""
import ctypes
import os
import re

import pytest

import long_context_sparse_spa_b200 as spa
from long_context_sparse_spa_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(spa_[a-z0-9_]+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported_and_bound():
    L = spa.lib()
    declared = _declared()
    assert declared, "no declarations found"
    for name in sorted(declared):
        assert hasattr(L, name), f"{name} missing from libspa.so"
        assert name in _abi.SIGNATURES, f"{name} has no ctypes signature"


def test_status_strings_and_version():
    L = spa.lib()
    assert L.spa_abi_version() == 7 == _abi.ABI_VERSION
    assert L.spa_status_string(_abi.SPA_ERR_CAPACITY) == b"SPA_ERR_CAPACITY"
    assert L.spa_status_string(99) == b"SPA_ERR_UNKNOWN"


def test_host_validation():
    L = spa.lib()
    P = ctypes.c_void_p(16)   # never dereferenced: every call below fails validation first
    # negative sizes
    assert L.spa_select_topk(P, None, -1, 10, 1, 0, 0, P, P, 1, P, 1 << 30, None) == _abi.SPA_ERR_INVALID_ARG
    # workspace too small
    assert L.spa_select_topk(P, None, 2, 10, 1, 0, 0, P, P, 1, P, 8, None) == _abi.SPA_ERR_WORKSPACE_TOO_SMALL
    # p outside (0, 1]
    big = 1 << 30
    assert L.spa_select_topp(P, None, 2, 10, ctypes.c_float(0.0), 0, 0, P, P, 10, None, P, big, None) == \
        _abi.SPA_ERR_INVALID_ARG
    assert L.spa_select_topp(P, None, 2, 10, ctypes.c_float(1.5), 0, 0, P, P, 10, None, P, big, None) == \
        _abi.SPA_ERR_INVALID_ARG
    # unsupported index dim / head dim / group size
    assert L.spa_index_scores(0, P, P, None, 1, 4, 1, 10, 32, 0, ctypes.c_float(1.0), P, None) == \
        _abi.SPA_ERR_UNSUPPORTED_SHAPE
    assert L.spa_index_scores(0, P, P, None, 1, 64, 2, 10, 16, 1, ctypes.c_float(1.0), P, None) == \
        _abi.SPA_ERR_UNSUPPORTED_SHAPE
    assert L.spa_block_stats(P, 1, 1, 128, 96, 64, P, P, None) == _abi.SPA_ERR_UNSUPPORTED_SHAPE
    # misaligned bf16 pointer
    assert L.spa_block_stats(ctypes.c_void_p(18), 1, 1, 128, 128, 64, P, P, None) == _abi.SPA_ERR_UNSUPPORTED_SHAPE
    # Hq not a multiple of Hkv
    assert L.spa_sparse_attend(P, P, P, 1, 6, 4, 100, 128, P, P, 1, 1, 1, ctypes.c_float(1.0), P, None, None,
                               P, 1 << 30, None) == _abi.SPA_ERR_INVALID_ARG
    # empty problems are no-ops
    assert L.spa_select_topk(None, None, 0, 10, 1, 0, 0, None, None, 1, None, 0, None) == _abi.SPA_OK
    assert L.spa_block_stats(None, 0, 1, 128, 128, 64, None, None, None) == _abi.SPA_OK


def test_decode_validation():
    a = _abi.SpaDecodeArgs()
    a.B, a.Hq, a.Hkv, a.N, a.d, a.r, a.block = 1, 8, 1, 1000, 128, 16, 1
    a.select_kind = _abi.SPA_SELECT_TOPP
    a.topp = 0.0
    L = spa.lib()
    need = L.spa_decode_workspace_bytes(ctypes.byref(a))
    assert need > 1000 * 4
    assert L.spa_decode(ctypes.byref(a), ctypes.c_void_p(16), 10, None) == _abi.SPA_ERR_WORKSPACE_TOO_SMALL
    assert L.spa_decode(ctypes.byref(a), ctypes.c_void_p(16), need, None) == _abi.SPA_ERR_INVALID_ARG


def test_rla_and_block_proxy_validation():
    L = spa.lib()
    P = ctypes.c_void_p(16)   # never dereferenced: every call below returns before any device work
    INV, UNS, OK = _abi.SPA_ERR_INVALID_ARG, _abi.SPA_ERR_UNSUPPORTED_SHAPE, _abi.SPA_OK
    # spa_rla_state: row range inside [0, N], d in {64, 128}, 16-byte alignment; empty range is a no-op
    assert L.spa_rla_state(P, P, 1, 1, 100, 128, 5, 4, P, P, None) == INV
    assert L.spa_rla_state(P, P, 1, 1, 100, 128, 0, 101, P, P, None) == INV
    assert L.spa_rla_state(P, P, 1, 1, 100, 128, -1, 4, P, P, None) == INV
    assert L.spa_rla_state(None, None, 1, 1, 100, 128, 7, 7, None, None, None) == OK
    assert L.spa_rla_state(P, P, 1, 1, 100, 96, 0, 10, P, P, None) == UNS
    assert L.spa_rla_state(P, P, 1, 1, 100, 128, 0, 10, ctypes.c_void_p(20), P, None) == UNS
    assert L.spa_rla_state(P, None, 1, 1, 100, 128, 0, 10, P, P, None) == INV
    # spa_block_minmax: shapes as spa_block_stats
    assert L.spa_block_minmax(P, 1, 1, 128, 96, 64, P, P, None) == UNS
    assert L.spa_block_minmax(P, 1, 1, 128, 128, 48, P, P, None) == UNS
    assert L.spa_block_minmax(None, 0, 1, 128, 128, 64, None, None, None) == OK
    # min-max scores need both statistics and a positive scale; the mean score needs the means
    assert L.spa_index_scores(_abi.SPA_SCORE_MINMAX_BLOCK, P, P, P, 1, 4, 1, 10, 128, 0, ctypes.c_float(0.0), P,
                              None) == INV
    assert L.spa_index_scores(_abi.SPA_SCORE_MINMAX_BLOCK, P, P, None, 1, 4, 1, 10, 128, 0, ctypes.c_float(1.0), P,
                              None) == INV
    assert L.spa_index_scores(_abi.SPA_SCORE_MEAN_BLOCK, P, P, None, 1, 4, 1, 10, 96, 0, ctypes.c_float(1.0), P,
                              None) == UNS
    assert L.spa_index_scores(7, P, P, P, 1, 4, 1, 10, 128, 0, ctypes.c_float(1.0), P, None) == INV


def test_decode_rla_fields_validation():
    a = _abi.SpaDecodeArgs()
    a.score_kind, a.select_kind, a.collapse = _abi.SPA_SCORE_LOWRANK, _abi.SPA_SELECT_TOPP, 1
    a.B, a.Hq, a.Hkv, a.N, a.d, a.r, a.block = 1, 8, 1, 1000, 128, 16, 1
    a.topp, a.cap = 0.9, 1000
    P = 16
    a.q = a.q_idx = a.K = a.V = a.Kidx = a.idx = a.count = a.out = P
    a.rla_state, a.rla_z, a.rla_gamma, a.rla_eps = P, None, P, 1e-6     # z missing
    L = spa.lib()
    need = L.spa_decode_workspace_bytes(ctypes.byref(a))
    assert L.spa_decode(ctypes.byref(a), ctypes.c_void_p(P), need, None) == _abi.SPA_ERR_INVALID_ARG
    a.rla_z, a.rla_eps = P, -1.0                                          # negative epsilon
    assert L.spa_decode(ctypes.byref(a), ctypes.c_void_p(P), need, None) == _abi.SPA_ERR_INVALID_ARG


def test_static_status_rejects_null_bits():
    # validation precedes the device lookup: no GPU needed
    assert spa.lib().spa_select_static_status(None, None, 0) == _abi.SPA_ERR_INVALID_ARG


def test_test_stall_rejects_unknown_bits():
    assert spa.lib().spa_test_stall(4) == _abi.SPA_ERR_INVALID_ARG
    assert spa.lib().spa_test_stall(0) == _abi.SPA_OK


def test_timed_prefills_reject_missing_events():
    # the events are checked before any argument that would need a GPU
    L = spa.lib()
    a = _abi.SpaPrefillArgs()
    b = _abi.SpaPbsArgs()
    none2 = (ctypes.c_void_p * 2)(None, None)
    for fn, args in ((L.spa_prefill_shared_timed, a), (L.spa_pbs_prefill_timed, b)):
        assert fn(ctypes.byref(args), ctypes.c_void_p(16), 1 << 20, None, None) == _abi.SPA_ERR_INVALID_ARG
        assert fn(ctypes.byref(args), ctypes.c_void_p(16), 1 << 20, None, none2) == _abi.SPA_ERR_INVALID_ARG
