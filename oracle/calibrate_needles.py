"""Choose the needle amplitude of the clustered-needle key generator.

The amplitude of the planted needle clusters is not given for the 64K top-p workload.
It is fixed once, before any GPU timing, as the smallest candidate amplitude for which
the oracle's top-p support of unit (b=0, kv head 0) of the 64K workload reaches a
sparsity of at least 0.89 -- the sparsity the RTPurbo page reports at 64K
("Full Attention Strikes Back", Key results, "Sparsity").

Run ``python -m oracle.calibrate_needles`` to print the sparsity per candidate and the
choice; ``synth.configs.NEEDLE_AMPLITUDE`` holds the frozen value and
tests/test_calibration.py re-checks it.
"""
from __future__ import annotations

import sys
from typing import Dict

import oracle
from synth import configs
from synth.gen import decode_inputs


def sparsity_at(amp: float, cfg=None) -> float:
    cfg = (cfg or configs.C2).with_(needle_amp=amp)
    x = decode_inputs(cfg, units=[(0, 0)])
    res = oracle.decode_unit(cfg, x, 0, with_output=False)
    return 1.0 - len(res["idx"]) / cfg.M


def calibrate(verbose: bool = True) -> Dict[str, object]:
    table = {}
    choice = None
    for a in configs.NEEDLE_AMPLITUDE_CANDIDATES:
        sp = sparsity_at(a)
        table[a] = sp
        if verbose:
            print(f"amplitude {a:5.1f}: sparsity {sp:.4f}", file=sys.stderr)
        if choice is None and sp >= configs.CALIBRATION_SPARSITY:
            choice = a
            break
    return {"choice": choice, "table": table}


if __name__ == "__main__":
    r = calibrate()
    print(r["choice"])
