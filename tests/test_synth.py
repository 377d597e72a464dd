"""Seeded generators: determinism, per-unit addressability, bf16 rounding, needle placement."""
import numpy as np
import torch

from synth import C1, SMALL, bf16_bits, bf16_value, decode_inputs, prefill_inputs


def test_bf16_rounding_matches_torch_rne():
    x = np.random.default_rng(0).standard_normal(100_000).astype(np.float32) * 7
    x[:4] = [1.00390625, 1.01171875, -2.0 ** -130, 3.0e38]
    ref = torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bf16_bits(x), ref)
    np.testing.assert_array_equal(bf16_value(ref), torch.tensor(x).to(torch.bfloat16).float().numpy())


def test_decode_inputs_deterministic_and_unit_addressable():
    cfg = SMALL["c2s"]
    a = decode_inputs(cfg)
    b = decode_inputs(cfg, units=[(1, 0)])
    for k in ("q", "q_idx"):
        np.testing.assert_array_equal(a[k], b[k])
    np.testing.assert_array_equal(a["K"][1, 0], b["K"][1, 0])
    np.testing.assert_array_equal(a["V"][1, 0], b["V"][1, 0])
    np.testing.assert_array_equal(a["Kidx"][1, 0], b["Kidx"][1, 0])
    assert not b["K"][0, 0].any()


def test_needles_outside_sink_and_window():
    for cfg in (C1, SMALL["c2s"], SMALL["c4s"]):
        x = decode_inputs(cfg, units=[(0, 0)])
        pos = np.asarray(x["needles"][(0, 0)])
        assert pos.size == max(cfg.n_needles, cfg.n_clusters * cfg.cluster_len)
        assert pos.min() >= cfg.sink and pos.max() < cfg.N - cfg.window
        assert np.unique(pos).size == pos.size


def test_block_generator_and_prefill_shapes():
    x = decode_inputs(SMALL["c3s"], units=[(0, 1)])
    assert x["K"].shape == (2, 2, 64 * 300 + 17, 128) and "Kidx" not in x
    p = prefill_inputs(SMALL["c5s"])
    assert p["Q"].shape == (1024, 8, 128) and p["Kidx"].shape == (2, 4096, 16)


def test_pbs_inputs_are_seeded_and_plant_heavy_keys():
    from synth import PBS_SMALL, pbs_inputs
    a, b2 = pbs_inputs(PBS_SMALL), pbs_inputs(PBS_SMALL)
    for k in a:
        assert np.array_equal(a[k], b2[k])
    cfg = PBS_SMALL
    assert a["Q"].shape == (cfg.T, cfg.Hq, cfg.d) and a["K"].shape == (cfg.Hkv, cfg.T, cfg.d)
    # every full segment before the last holds b keys far longer than the N(0, 1) ones
    Kf = bf16_value(a["K"][0]).astype(np.float64)
    norms = np.linalg.norm(Kf, axis=1)
    for s0 in range(0, cfg.T - cfg.S, cfg.S):
        assert np.sum(norms[s0:s0 + cfg.S] > 0.5 * (norms.mean() + cfg.heavy_amp)) >= cfg.b // 2
