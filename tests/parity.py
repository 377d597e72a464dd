"""Helpers shared by the parity tests: device upload, tie bands, support and output checks.

Acceptance rule for supports: the selected set must equal the oracle's, except for
elements that are ties of the threshold -- a score within 1e-6 (relative, floored at 1
in absolute terms because an fp32 dot product's rounding error scales with its terms,
not its result) of the threshold score, or, for top-p, an element whose inclusion moves
the cumulative mass by less than 1e-6 of the threshold mass.  Every such difference is
counted and reported.  Outputs: fp32 output within 2e-3 max-abs of the fp64 oracle on
the same support; bf16 output equal to the round-to-nearest-even of the fp32 output.
"""
from __future__ import annotations

from typing import Iterable, Optional, Set

import numpy as np

import oracle

SCORE_TIE_REL = 1e-6
MASS_TIE_REL = 1e-6
OUT_TOL = 2e-3


def dev_bf16(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).cuda()


def dev(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_rne_of(x_f32: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of float32 values (round to nearest even), via torch's conversion."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x_f32, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def score_band(s: np.ndarray, tau: float, rel: float = SCORE_TIE_REL) -> Set[int]:
    return set(np.nonzero(np.abs(s - tau) <= rel * max(1.0, abs(tau)))[0].tolist())


def topk_band(s: np.ndarray, k: int) -> Set[int]:
    M = s.size
    if k <= 0 or k >= M:
        return set()
    order = oracle.rank_order(s)
    return score_band(s, s[order[k - 1]])


def topp_band(s: np.ndarray, p: float, rel_mass: float = MASS_TIE_REL) -> Set[int]:
    if s.size == 0:
        return set()
    order = oracle.rank_order(s)
    e = np.exp(s[order] - s[order[0]])
    cum = np.cumsum(e)
    target = p * cum[-1]
    c = int(np.searchsorted(cum, target, side="left")) + 1
    c = min(c, s.size)
    band = score_band(s, s[order[c - 1]])
    c_lo = int(np.searchsorted(cum, target * (1 - rel_mass), side="left")) + 1
    c_hi = int(np.searchsorted(cum, target * (1 + rel_mass), side="left")) + 1
    band |= set(order[c_lo:min(c_hi, s.size)].tolist())
    return band


def compare_support(gpu: np.ndarray, ref: np.ndarray, band: Iterable[int], what: str = "") -> int:
    """Asserts the supports agree up to the tie band; returns the number of tie differences."""
    g = np.asarray(gpu)
    assert np.all(np.diff(g) > 0), f"{what}: GPU support not ascending/unique"
    diff = set(g.tolist()) ^ set(np.asarray(ref).tolist())
    bad = diff - set(band)
    assert not bad, f"{what}: {len(bad)} support differences outside the tie band, e.g. {sorted(bad)[:8]}"
    return len(diff)


def check_outputs(out_bf16: np.ndarray, out_f32: np.ndarray, ref: np.ndarray, what: str = "",
                  tol: float = OUT_TOL) -> float:
    err = float(np.max(np.abs(out_f32.astype(np.float64) - ref))) if ref.size else 0.0
    assert err <= tol, f"{what}: max |out - oracle| = {err:.3e} > {tol}"
    np.testing.assert_array_equal(out_bf16, bf16_rne_of(out_f32), err_msg=f"{what}: bf16 output != RNE(fp32 output)")
    return err
