"""RLA state (spa_rla_state) on the GPU against the fp64 oracle ("SPLA", section 2.2).

S = phi(K)^T V and z = sum phi(k) with phi = exp.  The kernel carries phi(k) as two bf16
terms (relative error about 2^-17) and sums in fp32, so every element of S is compared
within 2e-4 of sum_n exp(k_n[i]) |v_n[j]| (the bf16 split plus fp32 accumulation over up
to ~10^4 terms per accumulator), and z, a sum of positive terms, within a relative 1e-4.
"""
import numpy as np
import pytest

import oracle
from parity import dev_bf16
from synth import SMALL, bf16_value, decode_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import long_context_sparse_spa_b200 as spa  # noqa: E402


def _check_state(S, z, K, V, n0, n1, what):
    Sr, zr = oracle.rla_state(K, V, n0, n1)
    Kf = bf16_value(K[n0:n1]).astype(np.float64)
    Vf = bf16_value(V[n0:n1]).astype(np.float64)
    bound = 2e-4 * (np.exp(Kf).T @ np.abs(Vf)) + 1e-30
    err = np.abs(S.astype(np.float64) - Sr)
    assert (err <= bound).all(), f"{what}: S off by {float((err / bound).max()):.2f} x the bound"
    np.testing.assert_allclose(z, zr, rtol=1e-4, err_msg=what)


@pytest.mark.parametrize("name", ["c1s", "c3s"])
def test_rla_state_matches_oracle(name):
    cfg = SMALL[name]                      # d = 64 (N = 3000) and d = 128 (N = 19217): ragged tails
    x = decode_inputs(cfg)
    K, V = dev_bf16(x["K"]), dev_bf16(x["V"])
    S, z = spa.rla_state(K, V)
    S2, z2 = spa.rla_state(K, V)
    torch.cuda.synchronize()
    assert torch.equal(S, S2) and torch.equal(z, z2), "two equal calls must give equal bits"
    Sn, zn = S.cpu().numpy(), z.cpu().numpy()
    for b in range(cfg.B):
        for g in range(cfg.Hkv):
            _check_state(Sn[b, g], zn[b, g], x["K"][b, g], x["V"][b, g], 0, cfg.N, f"{name} ({b}, {g})")


def test_rla_state_incremental_appends():
    cfg = SMALL["c3s"]
    x = decode_inputs(cfg)
    K, V = dev_bf16(x["K"]), dev_bf16(x["V"])
    N = cfg.N
    S, z = spa.rla_state(K, V, n0=0, n1=1001)          # a prefill that ends mid-stage
    for n in range(1001, 1040):                        # then tokens appended one at a time
        spa.rla_state(K, V, S, z, n0=n, n1=n + 1)
    spa.rla_state(K, V, S, z, n0=1040, n1=N)
    spa.rla_state(K, V, S, z, n0=N, n1=N)              # empty range: no change
    torch.cuda.synchronize()
    Sn, zn = S.cpu().numpy(), z.cpu().numpy()
    for b in range(cfg.B):
        for g in range(cfg.Hkv):
            _check_state(Sn[b, g], zn[b, g], x["K"][b, g], x["V"][b, g], 0, N, f"appended ({b}, {g})")


def test_rla_state_rejects_bad_ranges():
    cfg = SMALL["c1s"]
    x = decode_inputs(cfg)
    K, V = dev_bf16(x["K"]), dev_bf16(x["V"])
    with pytest.raises(spa.SpaError):
        spa.rla_state(K, V, n0=5, n1=4)
    with pytest.raises(spa.SpaError):
        spa.rla_state(K, V, n0=0, n1=cfg.N + 1)
