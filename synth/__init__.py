"""Seeded synthetic workloads (configs + input generators) for the sparse-attention path.

Shared by the tests, the oracle driver and the bench.  Holds no arithmetic of the method.
"""
from .configs import (ALL_CONFIGS, C1, C2, C2_128K, C3, C4, C5, DECODE_CONFIGS, PBS_32K, PBS_SMALL, SMALL,
                      DecodeConfig, PbsConfig, PrefillConfig)
from .gen import bf16_bits, bf16_value, decode_inputs, pbs_inputs, prefill_inputs
