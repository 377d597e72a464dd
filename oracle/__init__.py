"""fp64 CPU oracle for query-aware sparse attention over a long KV cache.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package.  It shares no code with the CUDA library
(``long_context_sparse_spa_b200``); both sides meet only in the seeded inputs of
``synth``.

The arithmetic lives in ``spa_oracle.cpp`` (plain C++ in double precision, one unit at a
time).  This module marshals numpy arrays into it and loops over units.  Where a float
decides an integer (the ranking behind top-k / top-p), the decode and prefill drivers
round the fp64 scores to binary32 first, because the CUDA path ranks binary32 scores:
both sides then take that decision in the same precision.
"""
from __future__ import annotations

import ctypes
import math
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

from . import build as _build

_LIB = None

_i64 = ctypes.c_int64
_int = ctypes.c_int
_dbl = ctypes.c_double
_p = ctypes.c_void_p


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.orc_abi_version.restype = _int
        L.orc_block_stats.argtypes = [_p, _i64, _int, _int, _p, _p]
        L.orc_lowrank_scores.argtypes = [_p, _int, _p, _i64, _int, _int, _dbl, _p]
        L.orc_taylor_scores.argtypes = [_p, _int, _p, _p, _i64, _int, _dbl, _int, _p]
        L.orc_rank_order.argtypes = [_p, _i64, _p]
        L.orc_select_topk.argtypes = [_p, _i64, _i64, _i64, _i64, _p]
        L.orc_select_topk.restype = _i64
        L.orc_select_topp.argtypes = [_p, _i64, _dbl, _i64, _i64, _p, _p, _p]
        L.orc_select_topp.restype = _i64
        L.orc_sparse_attention.argtypes = [_p, _int, _p, _p, _i64, _int, _p, _i64, _int, _dbl, _p, _p]
        L.orc_dense_probs.argtypes = [_p, _int, _p, _i64, _int, _dbl, _p]
        L.orc_prefill_unit.argtypes = [_p, _p, _int, _int, _int, _int, _p, _p, _p, _i64, _i64, _dbl,
                                       _i64, _i64, _dbl, _int, _p, _p, _p]
        L.orc_prefill_unit.restype = _i64
        L.orc_rla_state.argtypes = [_p, _p, _int, _i64, _i64, _p, _p]
        L.orc_rla_direct.argtypes = [_p, _int, _p, _p, _i64, _int, _p, _i64, _int, _p]
        L.orc_rla_subtract.argtypes = [_p, _int, _p, _p, _i64, _int, _p, _i64, _int, _p, _p, _p]
        L.orc_rms_norm.argtypes = [_p, _int, _p, _dbl, _p]
        L.orc_pbs_importance.argtypes = [_p, _int, _int, _i64, _p, _i64, _int, _dbl, _p]
        L.orc_pbs_permutation.argtypes = [_p, _i64, _i64, _p]
        L.orc_pbs_prefill_unit.argtypes = [_p, _int, _int, _int, _i64, _p, _p, _i64, _p, _i64, _i64, _dbl, _p, _p]
        L.orc_pbs_prefill_unit.restype = _i64
        L.orc_block_minmax.argtypes = [_p, _i64, _int, _int, _p, _p]
        L.orc_minmax_scores.argtypes = [_p, _int, _p, _p, _i64, _int, _dbl, _int, _p]
        L.orc_mean_scores.argtypes = [_p, _int, _p, _i64, _int, _dbl, _int, _p]
        L.orc_round_bf16.argtypes = [_p, _i64, _p]
        assert L.orc_abi_version() == 5, "stale oracle library; rebuild it"
        _LIB = L
    return _LIB


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def as_ranked(scores: np.ndarray) -> np.ndarray:
    """Scores as the ranking sees them: rounded to binary32, widened back to float64."""
    return np.asarray(scores, np.float64).astype(np.float32).astype(np.float64)


# --------------------------------------------------------------------------- per-unit
def block_stats(K: np.ndarray, block: int) -> Tuple[np.ndarray, np.ndarray]:
    """K [N, d] bf16 bits -> (mean, var) [N // block, d] float64 (population variance)."""
    K = _c(K, np.uint16)
    N, d = K.shape
    nb = N // block
    mean = np.empty((nb, d)); var = np.empty((nb, d))
    lib().orc_block_stats(_ptr(K), N, d, block, _ptr(mean), _ptr(var))
    return mean, var


def lowrank_scores(qidx: np.ndarray, kidx: np.ndarray, collapse: bool, scale: float) -> np.ndarray:
    """qidx [G, r], kidx [N, r] bf16 bits -> scores [N] (collapse) or [G, N], float64."""
    qidx = _c(qidx, np.uint16); kidx = _c(kidx, np.uint16)
    G, r = qidx.shape
    N = kidx.shape[0]
    out = np.empty(N if collapse else (G, N))
    lib().orc_lowrank_scores(_ptr(qidx), G, _ptr(kidx), N, r, int(collapse), float(scale), _ptr(out))
    return out


def taylor_scores(q: np.ndarray, mean: np.ndarray, var: np.ndarray, scale: float, collapse: bool) -> np.ndarray:
    """q [G, d] bf16 bits, mean/var [nb, d] -> Taylor block scores t (linear), [nb] or [G, nb]."""
    q = _c(q, np.uint16); mean = _c(mean, np.float64); var = _c(var, np.float64)
    G, d = q.shape
    nb = mean.shape[0]
    out = np.empty(nb if collapse else (G, nb))
    lib().orc_taylor_scores(_ptr(q), G, _ptr(mean), _ptr(var), nb, d, float(scale), int(collapse), _ptr(out))
    return out


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even of float64 values to bf16 bit patterns (uint16), directly from
    double: the storage of block statistics in bf16."""
    x = _c(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    lib().orc_round_bf16(_ptr(x), x.size, _ptr(out))
    return out


def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact)."""
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def block_minmax(K: np.ndarray, block: int) -> Tuple[np.ndarray, np.ndarray]:
    """Per-block channel min and max of K [N, d] bf16 bits (full blocks) -> [nb, d] float64
    ("SPLA", section 1: min/max pooling)."""
    K = _c(K, np.uint16)
    N, d = K.shape
    nb = N // block
    mn = np.empty((nb, d)); mx = np.empty((nb, d))
    lib().orc_block_minmax(_ptr(K), N, d, block, _ptr(mn), _ptr(mx))
    return mn, mx


def minmax_scores(q: np.ndarray, mn: np.ndarray, mx: np.ndarray, scale: float, collapse: bool) -> np.ndarray:
    """Min-max page score: scale * sum_i max(q_i mn_i, q_i mx_i), the upper bound of every
    key logit in the block ("SPLA" section 1; "The Sparse Frontier", token-to-page decode
    selection).  q [G, d] bf16 bits -> [nb] (mean over heads) or [G, nb]."""
    q = _c(q, np.uint16); mn = _c(mn, np.float64); mx = _c(mx, np.float64)
    G, d = q.shape
    nb = mn.shape[0]
    out = np.empty(nb if collapse else (G, nb))
    lib().orc_minmax_scores(_ptr(q), G, _ptr(mn), _ptr(mx), nb, d, float(scale), int(collapse), _ptr(out))
    return out


def mean_scores(q: np.ndarray, mean: np.ndarray, scale: float, collapse: bool) -> np.ndarray:
    """Mean-pooling block score scale * q . kbar ("SPLA" section 1; PBS-Attn section 4).
    q [G, d] bf16 bits, mean [nb, d] -> [nb] (mean over heads) or [G, nb]."""
    q = _c(q, np.uint16); mean = _c(mean, np.float64)
    G, d = q.shape
    nb = mean.shape[0]
    out = np.empty(nb if collapse else (G, nb))
    lib().orc_mean_scores(_ptr(q), G, _ptr(mean), nb, d, float(scale), int(collapse), _ptr(out))
    return out


def rank_order(s: np.ndarray) -> np.ndarray:
    s = _c(s, np.float64)
    order = np.empty(s.size, np.int64)
    lib().orc_rank_order(_ptr(s), s.size, _ptr(order))
    return order


def select_topk(s: np.ndarray, k: int, sink: int, window: int) -> np.ndarray:
    s = _c(s, np.float64)
    idx = np.empty(max(1, s.size), np.int32)
    n = lib().orc_select_topk(_ptr(s), s.size, k, sink, window, _ptr(idx))
    return idx[:n].copy()


def select_topp(s: np.ndarray, p: float, sink: int, window: int) -> Tuple[np.ndarray, float, int]:
    """-> (ascending support, index mass of the support, length of the ranked prefix)."""
    s = _c(s, np.float64)
    idx = np.empty(max(1, s.size), np.int32)
    mass = ctypes.c_double(0.0); cut = ctypes.c_int64(0)
    n = lib().orc_select_topp(_ptr(s), s.size, float(p), sink, window, _ptr(idx),
                              ctypes.addressof(mass), ctypes.addressof(cut))
    if n < 0:
        raise ValueError("top-p needs 0 < p <= 1 and a non-empty score row")
    return idx[:n].copy(), mass.value, cut.value


def sparse_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, idx: np.ndarray, sm_scale: float,
                     unit_tokens: int = 1) -> Tuple[np.ndarray, np.ndarray]:
    """q [G, d], K/V [N, d] bf16 bits, idx support -> (out [G, d], lse [G]) float64."""
    q = _c(q, np.uint16); K = _c(K, np.uint16); V = _c(V, np.uint16); idx = _c(idx, np.int32)
    G, d = q.shape
    out = np.empty((G, d)); lse = np.empty(G)
    lib().orc_sparse_attention(_ptr(q), G, _ptr(K), _ptr(V), K.shape[0], d, _ptr(idx), idx.size,
                               unit_tokens, float(sm_scale), _ptr(out), _ptr(lse))
    return out, lse


def rla_state(K: np.ndarray, V: np.ndarray, n0: int = 0, n1: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
    """RLA state of rows [n0, n1) of one (batch, kv head) ("SPLA", section 2.2):
    S [d, d] = sum_n exp(k_n) v_n^T and z [d] = sum_n exp(k_n), float64."""
    K = _c(K, np.uint16); V = _c(V, np.uint16)
    d = K.shape[1]
    n1 = K.shape[0] if n1 is None else n1
    S = np.empty((d, d)); z = np.empty(d)
    lib().orc_rla_state(_ptr(K), _ptr(V), d, n0, n1, _ptr(S), _ptr(z))
    return S, z


def rla_direct(q: np.ndarray, K: np.ndarray, V: np.ndarray, idx: np.ndarray, unit_tokens: int = 1) -> np.ndarray:
    """RLA output by definition ("SPLA", section 2.2): normalised linear attention with
    phi = exp over the rows the support leaves out.  q [G, d] -> [G, d] float64."""
    q = _c(q, np.uint16); K = _c(K, np.uint16); V = _c(V, np.uint16); idx = _c(idx, np.int32)
    G, d = q.shape
    o = np.empty((G, d))
    lib().orc_rla_direct(_ptr(q), G, _ptr(K), _ptr(V), K.shape[0], d, _ptr(idx), idx.size, unit_tokens, _ptr(o))
    return o


def rla_subtract(q: np.ndarray, K: np.ndarray, V: np.ndarray, idx: np.ndarray, S: np.ndarray, z: np.ndarray,
                 unit_tokens: int = 1) -> np.ndarray:
    """RLA output in the IO form ("SPLA", section 2.2): global linear attention from the
    state (S, z) minus linear attention over the gathered support rows."""
    q = _c(q, np.uint16); K = _c(K, np.uint16); V = _c(V, np.uint16); idx = _c(idx, np.int32)
    S = _c(S, np.float64); z = _c(z, np.float64)
    G, d = q.shape
    o = np.empty((G, d))
    lib().orc_rla_subtract(_ptr(q), G, _ptr(K), _ptr(V), K.shape[0], d, _ptr(idx), idx.size, unit_tokens,
                           _ptr(S), _ptr(z), _ptr(o))
    return o


def rms_norm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm with scale gamma ("SPLA", section 2.3) of x [d] -> [d] float64."""
    x = _c(x, np.float64); gamma = _c(gamma, np.float64)
    y = np.empty_like(x)
    lib().orc_rms_norm(_ptr(x), x.size, _ptr(gamma), float(eps), _ptr(y))
    return y


def pbs_importance(Qlast: np.ndarray, t_last0: int, K: np.ndarray, sm_scale: float) -> np.ndarray:
    """Global key importance of PBS-Attn ("Sparser Block-Sparse Attention via Token
    Permutation", section 3): the mean causal softmax probability each key receives from
    the last query block.  Qlast [bl, G, d] bf16 at positions t_last0 ...; K [T, d]."""
    Qlast = _c(Qlast, np.uint16); K = _c(K, np.uint16)
    bl, G, d = Qlast.shape
    imp = np.empty(K.shape[0])
    lib().orc_pbs_importance(_ptr(Qlast), bl, G, t_last0, _ptr(K), K.shape[0], d, float(sm_scale), _ptr(imp))
    return imp


def pbs_permutation(imp: np.ndarray, S: int) -> np.ndarray:
    """Intra-segment key order of PBS-Attn (sections 2-3): perm[p] = original position of
    the key at permuted position p, sorted by descending importance inside each segment."""
    imp = _c(imp, np.float64)
    perm = np.empty(imp.size, np.int32)
    lib().orc_pbs_permutation(_ptr(imp), imp.size, S, _ptr(perm))
    return perm


def pbs_prefill_unit(Qblk: np.ndarray, t0: int, K: np.ndarray, V: np.ndarray, perm: np.ndarray, S: int, k: int,
                     sm_scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """One (query block, kv head) of the permuted block-sparse prefill (PBS-Attn, sections
    1-4) -> (support: original positions of the k selected permuted blocks, ascending;
    out [b, G, d] float64 over the support and the causal own segment)."""
    Qblk = _c(Qblk, np.uint16); K = _c(K, np.uint16); V = _c(V, np.uint16); perm = _c(perm, np.int32)
    b, G, d = Qblk.shape
    support = np.empty(max(1, min(max(k, 0), K.shape[0] // b) * b), np.int32)
    out = np.empty((b, G, d))
    n = lib().orc_pbs_prefill_unit(_ptr(Qblk), b, G, d, t0, _ptr(K), _ptr(V), K.shape[0], _ptr(perm), S, k,
                                   float(sm_scale), _ptr(support), _ptr(out))
    if n < 0:
        raise ValueError("need S % b == 0, t0 % b == 0 and t0 + b <= T")
    return support[:n].copy(), out


def dense_probs(q: np.ndarray, K: np.ndarray, sm_scale: float) -> np.ndarray:
    q = _c(q, np.uint16); K = _c(K, np.uint16)
    P = np.empty(K.shape[0])
    lib().orc_dense_probs(_ptr(q), q.shape[0], _ptr(K), K.shape[0], q.shape[1], float(sm_scale), _ptr(P))
    return P


def prefill_unit(qblk, qidx_blk, K, V, kidx, t0: int, idx_scale: float, k: int, sink: int,
                 sm_scale: float, rank_f32: bool = True, want_scores: bool = False):
    """One (query block, kv head) unit of the shared-support prefill -> (support, out [bq, G, d])
    (and the ranked scores [t0] when want_scores)."""
    qblk = _c(qblk, np.uint16); qidx_blk = _c(qidx_blk, np.uint16)
    K = _c(K, np.uint16); V = _c(V, np.uint16); kidx = _c(kidx, np.uint16)
    bq, G, d = qblk.shape
    r = qidx_blk.shape[2]
    support = np.empty(max(1, min(t0, k + sink)), np.int32)
    out = np.empty((bq, G, d))
    scores = np.empty(max(1, t0)) if want_scores else None
    n = lib().orc_prefill_unit(_ptr(qblk), _ptr(qidx_blk), bq, G, d, r, _ptr(K), _ptr(V), _ptr(kidx),
                               K.shape[0], t0, float(idx_scale), k, sink, float(sm_scale), int(rank_f32),
                               _ptr(support), _ptr(out), _ptr(scores))
    if n < 0:
        raise ValueError("query block outside the cache")
    if want_scores:
        return support[:n].copy(), out, scores[:t0].copy()
    return support[:n].copy(), out


# --------------------------------------------------------------------------- drivers
def f32(x: float) -> float:
    """A scalar parameter as the CUDA path receives it (binary32), widened to double."""
    return float(np.float32(x))


def decode_units(cfg) -> List[Tuple[int, int]]:
    """(b, head) pairs of a decode workload, in unit order u = b * heads + head."""
    heads = cfg.Hq if cfg.collapse == "head" else cfg.Hkv
    return [(b, h) for b in range(cfg.B) for h in range(heads)]


def local_support(M: int, sink: int, window: int) -> np.ndarray:
    """Support of a local head ("Full Attention Strikes Back" (RTPurbo), Methodology 1: local
    heads attend through a sliding window with an attention sink): the selection units
    [0, sink) and [M - window, M), ascending, without duplicates."""
    return np.union1d(np.arange(min(sink, M)), np.arange(max(0, M - window), M)).astype(np.int32)


def decode_unit(cfg, x: Dict[str, np.ndarray], u: int, stats: Optional[Tuple[np.ndarray, np.ndarray]] = None,
                with_output: bool = True, local: bool = False, rla: Optional[Dict[str, object]] = None
                ) -> Dict[str, object]:
    """The sparse decode path of one unit: scores -> support -> attention.

    Returns scores (float64, as computed), the ranked scores (binary32-rounded; for
    Taylor scores their natural log), the support, the index mass (top-p), the output
    [heads, d] and lse [heads] of the query heads sharing the support.  A local unit
    (head-wise routing, RTPurbo Methodology 1) is not scored: its support is the sink and
    the window, and it has no index mass.

    rla = {"gamma": [Hq, d], "eps": float} adds the residual linear attention ("SPLA",
    sections 2.2-2.3): out = exact sparse attention + RMSNorm_gamma(RLA over the rows the
    support leaves out); "out_exact" and "o_rla" keep the two parts.  gamma and eps are
    taken as the CUDA path receives them (binary32).
    """
    b, h = decode_units(cfg)[u]
    G = cfg.G
    if cfg.collapse == "head":
        g, heads = h // G, slice(h, h + 1)
    else:
        g, heads = h, slice(h * G, (h + 1) * G)
    res: Dict[str, object] = {"b": b, "g": g}
    if local:
        idx = local_support(cfg.M, cfg.sink, cfg.window)
        res.update(scores=None, ranked=None, index_mass=None, idx=idx)
        if with_output:
            out, lse = sparse_attention(x["q"][b, heads], x["K"][b, g], x["V"][b, g], idx, f32(cfg.sm_scale),
                                        cfg.block)
            res["out"] = out
            res["lse"] = lse
            _add_rla(cfg, x, res, heads, rla)
        return res
    if cfg.score == "lowrank":
        s = lowrank_scores(x["q_idx"][b, heads], x["Kidx"][b, g], cfg.collapse == "group", f32(cfg.score_scale))
        s = s.reshape(-1)                 # one row: the group's shared scores, or the one head's
        ranked = as_ranked(s)
    elif cfg.score == "minmax":          # min-max page score (min/max pooling)
        mn, mx = _stored(cfg, *block_minmax(x["K"][b, g], cfg.block))
        s = minmax_scores(x["q"][b, heads], mn, mx, f32(cfg.score_scale), True)
        ranked = as_ranked(s)
    elif cfg.score == "mean":            # mean-pooling block score
        mean, _ = _stored(cfg, *(stats if stats is not None else block_stats(x["K"][b, g], cfg.block)))
        s = mean_scores(x["q"][b, heads], mean, f32(cfg.score_scale), True)
        ranked = as_ranked(s)
    else:
        mean, var = _stored(cfg, *(stats if stats is not None else block_stats(x["K"][b, g], cfg.block)))
        t = taylor_scores(x["q"][b, heads], mean, var, f32(cfg.score_scale), True)
        s = t
        ranked = as_ranked(np.log(t))
    res["scores"] = s
    res["ranked"] = ranked
    if cfg.select == "topk":
        idx = select_topk(ranked, cfg.topk, cfg.sink, cfg.window)
        res["index_mass"] = None
    else:
        idx, mass, cut = select_topp(ranked, f32(cfg.topp), cfg.sink, cfg.window)
        res["index_mass"] = mass
        res["cut"] = cut
    res["idx"] = idx
    if with_output:
        out, lse = sparse_attention(x["q"][b, heads], x["K"][b, g], x["V"][b, g], idx, f32(cfg.sm_scale),
                                    cfg.block)
        res["out"] = out
        res["lse"] = lse
        _add_rla(cfg, x, res, heads, rla)
    return res


def _stored(cfg, *stats: np.ndarray) -> Tuple[np.ndarray, ...]:
    """Block statistics as the workload stores them: as computed, or rounded to bf16
    (round to nearest even) and widened back."""
    if getattr(cfg, "stats", "f32") == "bf16":
        return tuple(widen_bf16(round_bf16(a)) for a in stats)
    return stats


def _add_rla(cfg, x: Dict[str, np.ndarray], res: Dict[str, object], heads: slice,
             rla: Optional[Dict[str, object]]) -> None:
    """out += RMSNorm_gamma(RLA over the rows outside the support), per query head."""
    if rla is None:
        return
    b, g = res["b"], res["g"]
    o = rla_direct(x["q"][b, heads], x["K"][b, g], x["V"][b, g], res["idx"], cfg.block)
    gamma = np.asarray(rla["gamma"], np.float32).astype(np.float64)[heads]
    y = np.stack([rms_norm(o[i], gamma[i], f32(rla["eps"])) for i in range(o.shape[0])])
    res["out_exact"] = res["out"]
    res["o_rla"] = o
    res["out"] = res["out"] + y


def decode(cfg, x: Dict[str, np.ndarray], units: Optional[Sequence[int]] = None, threads: int = 1,
           with_output: bool = True, local: Optional[Sequence[bool]] = None,
           rla: Optional[Dict[str, object]] = None) -> List[Dict[str, object]]:
    """decode_unit over several units, optionally on a thread pool (the C calls release the GIL);
    local[u] marks the local units of a head-wise routing; rla adds the residual linear
    attention (see decode_unit)."""
    todo = list(range(cfg.U)) if units is None else list(units)
    loc = (lambda u: bool(local[u])) if local is not None else (lambda u: False)
    one = lambda u: decode_unit(cfg, x, u, with_output=with_output, local=loc(u), rla=rla)
    if threads <= 1:
        return [one(u) for u in todo]
    with ThreadPoolExecutor(threads) as ex:
        return list(ex.map(one, todo))


def captured_mass(cfg, x: Dict[str, np.ndarray], u: int, idx: np.ndarray) -> float:
    """Dense head-averaged attention mass on the support [OGS-2.1 P_{l,t}]."""
    b, h = decode_units(cfg)[u]
    G = cfg.G
    if cfg.collapse == "head":
        g, heads = h // G, slice(h, h + 1)
    else:
        g, heads = h, slice(h * G, (h + 1) * G)
    P = dense_probs(x["q"][b, heads], x["K"][b, g], f32(cfg.sm_scale))
    rows = (np.asarray(idx, np.int64)[:, None] * cfg.block + np.arange(cfg.block)[None, :]).ravel()
    return float(P[rows[rows < cfg.N]].sum())


def captured_mass_prefill(cfg, x: Dict[str, np.ndarray], j: int, g: int, support: np.ndarray,
                          queries: Optional[Sequence[int]] = None) -> float:
    """Captured mass of one prefill unit (query block j, kv head g) [OGS-2.1 P_{l,t}]: for
    each query t of the block, the dense causal head-averaged distribution over keys
    [0, t] summed over the keys its attention reads (the shared support and the block's
    own positions [t0, t]); the mean over the block's queries (or the given ones)."""
    G, bq = cfg.G, cfg.bq
    t0 = cfg.q_start + j * bq
    sup = np.asarray(support, np.int64)
    vals = []
    for i in (range(bq) if queries is None else queries):
        t = t0 + i
        P = dense_probs(x["Q"][j * bq + i, g * G:(g + 1) * G], x["K"][g][:t + 1], f32(cfg.sm_scale))
        own = np.arange(t0, t + 1)
        rows = np.union1d(sup[sup <= t], own)
        vals.append(float(P[rows].sum()))
    return float(np.mean(vals))


def prefill_block(cfg, x: Dict[str, np.ndarray], j: int, g: int, want_scores: bool = False):
    """Unit (query block j, kv head g) of a shared-support prefill -> (support, out [bq, G, d])
    (and the ranked scores of the candidates [0, t0) when want_scores)."""
    G, bq = cfg.G, cfg.bq
    rows = slice(j * bq, (j + 1) * bq)
    heads = slice(g * G, (g + 1) * G)
    t0 = cfg.q_start + j * bq
    return prefill_unit(x["Q"][rows, heads], x["q_idx"][rows, heads], x["K"][g], x["V"][g], x["Kidx"][g],
                        t0, f32(cfg.score_scale), cfg.topk, cfg.sink, f32(cfg.sm_scale), want_scores=want_scores)
