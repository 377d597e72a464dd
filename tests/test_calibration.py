"""The frozen needle amplitude is the smallest candidate whose oracle support on unit
(b=0, kv head 0) of the 64K top-p workload reaches the page's 64K sparsity (0.89)."""
from oracle.calibrate_needles import sparsity_at
from synth import configs


def test_needle_amplitude_is_smallest_reaching_target_sparsity():
    a = configs.NEEDLE_AMPLITUDE
    assert a in configs.NEEDLE_AMPLITUDE_CANDIDATES
    assert sparsity_at(a) >= configs.CALIBRATION_SPARSITY
    for smaller in configs.NEEDLE_AMPLITUDE_CANDIDATES:
        if smaller < a:
            assert sparsity_at(smaller) < configs.CALIBRATION_SPARSITY
