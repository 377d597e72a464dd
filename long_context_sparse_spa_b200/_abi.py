"""ctypes declarations of the C ABI in include/spa.h (libspa.so)."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(HERE, "libspa.so")

ABI_VERSION = 7   # spa_abi_version() of the library these declarations describe

SPA_OK = 0
SPA_ERR_INVALID_ARG = 1
SPA_ERR_UNSUPPORTED_SHAPE = 2
SPA_ERR_WORKSPACE_TOO_SMALL = 3
SPA_ERR_CUDA = 4
SPA_ERR_TIMEOUT = 5
SPA_ERR_CAPACITY = 6

SPA_COLLAPSE_NONE = 0
SPA_COLLAPSE_GROUP_MEAN = 1
SPA_SCORE_LOWRANK = 0
SPA_SCORE_TAYLOR_BLOCK = 1
SPA_SCORE_MINMAX_BLOCK = 2
SPA_SCORE_MEAN_BLOCK = 3
SPA_STATS_BF16 = 0x100
SPA_SELECT_TOPK = 0
SPA_SELECT_TOPP = 1
SPA_SELECT_STATIC_MAX_UNITS = 16
SPA_TEST_STALL_SELECT_LOAD = 1
SPA_TEST_STALL_PREFILL_MMA = 2
SPA_DECODE_AUTO = 0
SPA_DECODE_SEPARATE = 1
SPA_DECODE_FUSED = 2

_p = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_sz = ctypes.c_size_t


class SpaDecodeArgs(ctypes.Structure):
    _fields_ = [
        ("score_kind", _i), ("select_kind", _i), ("collapse", _i),
        ("B", _i), ("Hq", _i), ("Hkv", _i), ("N", _i), ("d", _i),
        ("r", _i), ("block", _i),
        ("q", _p), ("q_idx", _p), ("K", _p), ("V", _p), ("Kidx", _p),
        ("bmean", _p), ("bvar", _p),
        ("score_scale", _f), ("sm_scale", _f),
        ("topk", _i), ("topp", _f),
        ("sink", _i), ("window", _i),
        ("idx", _p), ("count", _p), ("cap", _i),
        ("index_mass", _p),
        ("out", _p), ("out_f32", _p), ("lse", _p),
        ("local_units", _p),
        ("rla_state", _p), ("rla_z", _p), ("rla_gamma", _p), ("rla_eps", _f),
        ("stats_bf16", _i),
        ("kernel_path", _i),
    ]


class SpaPrefillArgs(ctypes.Structure):
    _fields_ = [
        ("T", _i), ("Hq", _i), ("Hkv", _i), ("N", _i), ("d", _i), ("r", _i),
        ("q_start", _i), ("bq", _i),
        ("Q", _p), ("q_idx", _p), ("K", _p), ("V", _p), ("Kidx", _p),
        ("score_scale", _f), ("sm_scale", _f),
        ("topk", _i), ("sink", _i),
        ("idx", _p), ("count", _p), ("cap", _i),
        ("out", _p), ("out_f32", _p),
    ]


class SpaPbsArgs(ctypes.Structure):
    _fields_ = [
        ("T", _i), ("Hq", _i), ("Hkv", _i), ("d", _i),
        ("b", _i), ("S", _i), ("topk", _i), ("sm_scale", _f),
        ("Q", _p), ("K", _p), ("V", _p),
        ("importance", _p), ("perm", _p), ("idx", _p), ("count", _p), ("cap", _i),
        ("out", _p), ("out_f32", _p),
    ]


# name -> (restype, argtypes)
SIGNATURES = {
    "spa_status_string": (ctypes.c_char_p, [_i]),
    "spa_last_cuda_error": (ctypes.c_char_p, []),
    "spa_abi_version": (_i, []),
    "spa_test_stall": (_i, [_i]),
    "spa_block_stats": (_i, [_p, _i, _i, _i, _i, _i, _p, _p, _p]),
    "spa_index_scores": (_i, [_i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _f, _p, _p]),
    "spa_select_topk": (_i, [_p, _p, _i, _i, _i, _i, _i, _p, _p, _i, _p, _sz, _p]),
    "spa_select_topp": (_i, [_p, _p, _i, _i, _f, _i, _i, _p, _p, _i, _p, _p, _sz, _p]),
    "spa_select_workspace_bytes": (_sz, [_i, _i]),
    "spa_select_topp_static": (_i, [_p, _p, _i, _i, _f, _i, _i, _p, _p, _i, _p, _p]),
    "spa_select_static_status": (_i, [_p, ctypes.POINTER(ctypes.c_uint32), _i]),
    "spa_block_minmax": (_i, [_p, _i, _i, _i, _i, _i, _p, _p, _p]),
    "spa_block_stats_bf16": (_i, [_p, _i, _i, _i, _i, _i, _p, _p, _p]),
    "spa_block_minmax_bf16": (_i, [_p, _i, _i, _i, _i, _i, _p, _p, _p]),
    "spa_rla_state": (_i, [_p, _p, _i, _i, _i, _i, _i, _i, _p, _p, _p]),
    "spa_sparse_attend": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _p, _p, _i, _i, _i, _f, _p, _p, _p, _p, _sz, _p]),
    "spa_attend_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "spa_decode": (_i, [ctypes.POINTER(SpaDecodeArgs), _p, _sz, _p]),
    "spa_decode_workspace_bytes": (_sz, [ctypes.POINTER(SpaDecodeArgs)]),
    "spa_decode_path_taken": (_i, [ctypes.POINTER(SpaDecodeArgs)]),
    "spa_decode_timed": (_i, [ctypes.POINTER(SpaDecodeArgs), _p, _sz, _p, ctypes.POINTER(_p)]),
    "spa_read_device_status": (_i, [_p, _p, ctypes.POINTER(ctypes.c_uint32), _i]),
    "spa_prefill_shared": (_i, [ctypes.POINTER(SpaPrefillArgs), _p, _sz, _p]),
    "spa_prefill_shared_timed": (_i, [ctypes.POINTER(SpaPrefillArgs), _p, _sz, _p, ctypes.POINTER(_p)]),
    "spa_prefill_workspace_bytes": (_sz, [ctypes.POINTER(SpaPrefillArgs)]),
    "spa_prefill_per_query": (_i, [ctypes.POINTER(SpaPrefillArgs), _p, _sz, _p]),
    "spa_pbs_prefill": (_i, [ctypes.POINTER(SpaPbsArgs), _p, _sz, _p]),
    "spa_pbs_prefill_timed": (_i, [ctypes.POINTER(SpaPbsArgs), _p, _sz, _p, ctypes.POINTER(_p)]),
    "spa_pbs_workspace_bytes": (_sz, [ctypes.POINTER(SpaPbsArgs)]),
    "spa_prefill_per_query_workspace_bytes": (_sz, [ctypes.POINTER(SpaPrefillArgs)]),
}

_LIB = None


class SpaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        name = lib().spa_status_string(status).decode()
        extra = lib().spa_last_cuda_error().decode() if status == SPA_ERR_CUDA else ""
        super().__init__(f"{name}{': ' + what if what else ''}{' (' + extra + ')' if extra else ''}")


def lib() -> ctypes.CDLL:
    """The loaded libspa.so.  Raises if it has not been built (no fallback exists)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(lib_path):
            raise ImportError(f"libspa.so not found at {lib_path}; build it with "
                              "`python -m long_context_sparse_spa_b200.build`")
        L = ctypes.CDLL(lib_path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        if L.spa_abi_version() != ABI_VERSION:
            raise ImportError(f"{lib_path} has ABI version {L.spa_abi_version()}, these bindings expect "
                              f"{ABI_VERSION}; rebuild it")
        _LIB = L
    return _LIB


def check(status: int, what: str = "") -> None:
    if status != SPA_OK:
        raise SpaError(status, what)
