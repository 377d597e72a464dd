"""Data-parallel sharding of a decode workload across ranks (weak scaling).

Decode supports are independent per (sequence, kv head), so N ranks each take their own
B sequences of a global batch of N*B: rank r holds batch entries [r*B, (r+1)*B), drawn
exactly as in the unsharded global workload.  No collective touches the data path; the
only cross-rank operation is the max of the ranks' device times when a run is timed.
"""
from __future__ import annotations

from typing import Tuple

from .configs import DecodeConfig


def global_config(cfg: DecodeConfig, world: int) -> DecodeConfig:
    """The workload whose batch is the union of all ranks' batches."""
    return cfg.with_(B=cfg.B * world)


def batch_range(cfg: DecodeConfig, rank: int, world: int) -> Tuple[int, int]:
    """Batch entries [b0, b1) of the global workload that rank owns."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return rank * cfg.B, (rank + 1) * cfg.B
