"""Seeded synthetic inputs shared by the oracle-side and the CUDA-side tests and the bench.

This module only draws random tensors and rounds them to bf16.  It holds none of the
method's arithmetic (no scoring, selection or attention), so that the oracle and the
CUDA path share nothing but their inputs.

Every tensor is drawn from ``numpy.random.default_rng`` streams keyed by
``(seed, stream, ...)`` so that any (batch, kv head) slice can be regenerated on its
own.  Streams:

* ``(seed, 0)``            projector P (d x r, entries N(0, 1/d))
* ``(seed, 1)``            queries q ~ N(0, 1)
* ``(seed, 2)``            low-frequency basis: orthonormal u_j (QR of a d x rank
                           Gaussian) and phases phi_j ~ U(0, 2 pi)
* ``(seed, 3, b, g)``      keys of (batch b, kv head g): noise, needle placement, needle noise
* ``(seed, 4, b, g)``      values of (batch b, kv head g), V ~ N(0, 1)

All tensors are drawn in float32 (structured parts composed in float64), rounded once
to bf16 with round-to-nearest-even, and returned as their uint16 bit patterns.  Index
keys are Kidx = K P and index queries q_idx = q P, computed in float64 from the
bf16-rounded K and q and rounded to bf16 (the projection belongs to the model; the
method only consumes its outputs).
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Iterable, Optional, Tuple

import numpy as np

from .configs import DecodeConfig, PbsConfig, PrefillConfig

BF16 = np.uint16


# --------------------------------------------------------------------------- bf16 bits
def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite float32/float64 values to bf16 (RNE) and return the uint16 bit patterns.

    For finite binary32 patterns u <= 0xFF7FFFFF, u + 0x8000 cannot overflow 32 bits."""
    u = np.array(x, dtype=np.float32, copy=True, order="C").view(np.uint32)
    lsb = u >> np.uint32(16)
    lsb &= np.uint32(1)
    lsb += np.uint32(0x7FFF)
    u += lsb
    u >>= np.uint32(16)
    return u.astype(np.uint16)


def bf16_value(b: np.ndarray) -> np.ndarray:
    """Exact float32 value of bf16 bit patterns."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng([int(k) for k in key])


# --------------------------------------------------------------------------- shared parts
def projector(seed: int, d: int, r: int) -> np.ndarray:
    return _rng(seed, 0).standard_normal((d, r)) / math.sqrt(d)


def lowfreq_component(seed: int, N: int, d: int, rank: int, amp: float) -> np.ndarray:
    """amp * sum_j sin(2 pi j n / N + phi_j) u_j for j = 1..rank, as an [N, d] float32 array."""
    if rank == 0 or amp == 0.0:
        return np.zeros((N, d), np.float32)
    g = _rng(seed, 2)
    u, _ = np.linalg.qr(g.standard_normal((d, rank)))
    phi = g.uniform(0.0, 2.0 * math.pi, rank)
    n = np.arange(N, dtype=np.float64)
    waves = np.stack([np.sin(2.0 * math.pi * (j + 1) * n / N + phi[j]) for j in range(rank)], 1)
    return (amp * (waves @ u.T)).astype(np.float32)


def _project(x_bits: np.ndarray, P: np.ndarray) -> np.ndarray:
    x = bf16_value(x_bits).astype(np.float64)
    return bf16_bits(x @ P)


def cluster_starts(g: np.random.Generator, n_clusters: int, cluster_len: int, lo: int, hi: int) -> np.ndarray:
    """Seeded, non-overlapping starts of clusters of cluster_len tokens inside [lo, hi)."""
    n_slots = (hi - lo) // cluster_len
    if n_clusters > n_slots:
        raise ValueError("too many needle clusters for the available range")
    slots = np.sort(g.choice(n_slots, n_clusters, replace=False))
    return lo + slots * cluster_len


# --------------------------------------------------------------------------- decode
def decode_queries(cfg: DecodeConfig) -> Tuple[np.ndarray, Optional[np.ndarray], Optional[np.ndarray]]:
    """(q [B,Hq,d] bf16, q_idx [B,Hq,r] bf16 or None, P [d,r] float64 or None)."""
    q = bf16_bits(_rng(cfg.seed, 1).standard_normal((cfg.B, cfg.Hq, cfg.d), dtype=np.float32))
    if cfg.score != "lowrank":
        return q, None, None
    P = projector(cfg.seed, cfg.d, cfg.r)
    return q, _project(q, P), P


def decode_unit_keys(cfg: DecodeConfig, b: int, g: int, q: np.ndarray,
                     lowfreq: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Keys [N, d] bf16 of (batch b, kv head g) and the planted needle positions."""
    rng = _rng(cfg.seed, 3, b, g)
    N, d = cfg.N, cfg.d
    if cfg.keys == "blocks":
        nb = N // cfg.block
        n_full = nb * cfg.block
        mu = rng.standard_normal((nb, d), dtype=np.float32) * np.float32(0.5)
        sigma = rng.uniform(0.3, 1.5, nb).astype(np.float32)
        k = rng.standard_normal((N, d), dtype=np.float32)
        kb = k[:n_full].reshape(nb, cfg.block, d)
        kb *= sigma[:, None, None]
        kb += mu[:, None, :]
        return bf16_bits(k), np.zeros(0, np.int64)

    k = rng.standard_normal((N, d), dtype=np.float32)
    if lowfreq is not None:
        k += lowfreq
    qf = bf16_value(q[b]).astype(np.float64)          # [Hq, d]
    if cfg.keys == "needles":
        pos = cfg.sink + rng.choice(N - cfg.sink - cfg.window, cfg.n_needles, replace=False)
        for i, n in enumerate(pos):
            h = g * cfg.G + (i % cfg.G)
            unit = qf[h] / np.linalg.norm(qf[h])
            k[n] = (cfg.needle_amp * unit + 0.3 * rng.standard_normal(d)).astype(np.float32)
        return bf16_bits(k), np.sort(pos)
    if cfg.keys == "clusters":
        qbar = qf[g * cfg.G:(g + 1) * cfg.G].mean(0)
        unit = qbar / np.linalg.norm(qbar)
        starts = cluster_starts(rng, cfg.n_clusters, cfg.cluster_len, cfg.sink, N - cfg.window)
        pos = (starts[:, None] + np.arange(cfg.cluster_len)[None, :]).ravel()
        noise = rng.standard_normal((pos.size, d))
        k[pos] = (cfg.needle_amp * unit[None, :] + 0.3 * noise).astype(np.float32)
        return bf16_bits(k), pos
    return bf16_bits(k), np.zeros(0, np.int64)


def decode_unit_values(cfg: DecodeConfig, b: int, g: int) -> np.ndarray:
    return bf16_bits(_rng(cfg.seed, 4, b, g).standard_normal((cfg.N, cfg.d), dtype=np.float32))


def decode_inputs(cfg: DecodeConfig, units: Optional[Iterable[Tuple[int, int]]] = None,
                  batch: Optional[Tuple[int, int]] = None, threads: int = 0) -> Dict[str, np.ndarray]:
    """All inputs of a decode workload as uint16 bf16 bit arrays.

    Returns q [B,Hq,d], K, V [B,Hkv,N,d] and, for low-rank scoring, q_idx [B,Hq,r],
    Kidx [B,Hkv,N,r] and the projector P.  ``units`` restricts key/value generation to
    the listed (b, g) pairs (others stay zero), for bounded samples of large workloads.
    ``batch = (b0, b1)`` returns only batch entries b0 <= b < b1 of the workload (a data
    shard: entry b is drawn exactly as in the full workload).  Units are generated on
    ``threads`` threads (default: all cores); each has its own random stream, so the
    result does not depend on the thread count.
    """
    q, q_idx, P = decode_queries(cfg)
    b0, b1 = batch if batch is not None else (0, cfg.B)
    q = q[b0:b1].copy()
    q_idx = q_idx[b0:b1].copy() if q_idx is not None else None
    B, Hkv, N, d = b1 - b0, cfg.Hkv, cfg.N, cfg.d
    K = np.zeros((B, Hkv, N, d), BF16)
    V = np.zeros((B, Hkv, N, d), BF16)
    Kidx = np.zeros((B, Hkv, N, cfg.r), BF16) if P is not None else None
    lf = lowfreq_component(cfg.seed, N, d, cfg.lowfreq_rank, cfg.lowfreq_amp) if cfg.lowfreq_rank else None
    needles = {}
    todo = list(units) if units is not None else [(b, g) for b in range(b0, b1) for g in range(Hkv)]
    qfull = decode_queries(cfg)[0]

    def one(bg):
        b, g = bg
        K[b - b0, g], needles[(b, g)] = decode_unit_keys(cfg, b, g, qfull, lf)
        V[b - b0, g] = decode_unit_values(cfg, b, g)
        if Kidx is not None:
            Kidx[b - b0, g] = _project(K[b - b0, g], P)

    n_threads = threads if threads > 0 else min(len(todo), os.cpu_count() or 1)
    if n_threads <= 1:
        for bg in todo:
            one(bg)
    else:
        with ThreadPoolExecutor(n_threads) as ex:
            list(ex.map(one, todo))
    out = {"q": q, "K": K, "V": V, "needles": needles}
    if P is not None:
        out.update(q_idx=q_idx, Kidx=Kidx, P=P)
    return out


# --------------------------------------------------------------------------- prefill
def prefill_inputs(cfg: PrefillConfig) -> Dict[str, np.ndarray]:
    """Inputs of a selection-block-shared prefill chunk (batch 1).

    Q [T, Hq, d] are the chunk's queries (positions q_start + t); K, V [Hkv, N, d] the
    causal cache (the chunk's own keys at positions >= q_start included); q_idx
    [T, Hq, r] and Kidx [Hkv, N, r] the projected index queries/keys.  Keys follow the
    clustered-needle generator; the needle direction of kv head g is the unit mean of
    the chunk's queries of that group, and clusters sit in the context before the chunk.
    """
    Hq, Hkv, N, d, G = cfg.Hq, cfg.Hkv, cfg.N, cfg.d, cfg.G
    Q = bf16_bits(_rng(cfg.seed, 1).standard_normal((cfg.T, Hq, d), dtype=np.float32))
    P = projector(cfg.seed, d, cfg.r)
    q_idx = _project(Q, P)
    lf = lowfreq_component(cfg.seed, N, d, cfg.lowfreq_rank, cfg.lowfreq_amp)
    Qf = bf16_value(Q).astype(np.float64)
    K = np.zeros((Hkv, N, d), BF16)
    V = np.zeros((Hkv, N, d), BF16)
    Kidx = np.zeros((Hkv, N, cfg.r), BF16)
    for g in range(Hkv):
        rng = _rng(cfg.seed, 3, 0, g)
        k = rng.standard_normal((N, d), dtype=np.float32)
        k += lf
        qbar = Qf[:, g * G:(g + 1) * G, :].reshape(-1, d).mean(0)
        unit = qbar / np.linalg.norm(qbar)
        starts = cluster_starts(rng, cfg.n_clusters, cfg.cluster_len, cfg.sink, cfg.q_start)
        pos = (starts[:, None] + np.arange(cfg.cluster_len)[None, :]).ravel()
        k[pos] = (cfg.needle_amp * unit[None, :] + 0.3 * rng.standard_normal((pos.size, d))).astype(np.float32)
        K[g] = bf16_bits(k)
        V[g] = bf16_bits(_rng(cfg.seed, 4, 0, g).standard_normal((N, d), dtype=np.float32))
        Kidx[g] = _project(K[g], P)
    return {"Q": Q, "q_idx": q_idx, "K": K, "V": V, "Kidx": Kidx, "P": P}


def pbs_inputs(cfg: PbsConfig) -> Dict[str, np.ndarray]:
    """Inputs of a permuted block-sparse prefill: Q [T, Hq, d], K, V [Hkv, T, d] (bf16 bits).

    Q, V ~ N(0, 1).  K ~ N(0, 1), except that every segment before the last holds b heavy keys
    at scattered positions, k = heavy_amp * qbar_g / |qbar_g| + 0.3 N(0, 1), with qbar_g the mean
    of the last query block's queries of kv head g."""
    T, Hq, Hkv, d, G, b, S = cfg.T, cfg.Hq, cfg.Hkv, cfg.d, cfg.G, cfg.b, cfg.S
    Q = bf16_bits(_rng(cfg.seed, 1).standard_normal((T, Hq, d), dtype=np.float32))
    Qf = bf16_value(Q).astype(np.float64)
    K = np.zeros((Hkv, T, d), np.uint16)
    V = np.zeros((Hkv, T, d), np.uint16)
    for g in range(Hkv):
        rng = _rng(cfg.seed, 2, g)
        k = rng.standard_normal((T, d), dtype=np.float32)
        qbar = Qf[T - b:, g * G:(g + 1) * G].reshape(-1, d).mean(0)
        unit = qbar / np.linalg.norm(qbar)
        for s0 in range(0, (T - 1) // S * S, S):
            pos = s0 + np.sort(rng.choice(S, b, replace=False))
            k[pos] = (cfg.heavy_amp * unit[None, :] + 0.3 * rng.standard_normal((b, d))).astype(np.float32)
        K[g] = bf16_bits(k)
        V[g] = bf16_bits(_rng(cfg.seed, 3, g).standard_normal((T, d), dtype=np.float32))
    return {"Q": Q, "K": K, "V": V}
