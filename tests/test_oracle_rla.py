"""Pins of the oracle's residual linear attention ("SPLA", sections 2.2-2.3).

RLA is normalised linear attention with the feature map phi = exp over the rows a support
leaves out; the IO form takes it as global linear attention from a running state minus
linear attention over the gathered rows.  These tests pin the oracle against the
subtraction identity, closed forms (equal keys give the plain mean, one left-out row gives
its value, d = 1 is a softmax with unit scale), an invariant (shifting every query
component by one constant rescales every weight alike), numpy / torch library routines,
and the decode driver's assembly of the output.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import SMALL, bf16_bits, bf16_value, decode_inputs


def _bf(shape, seed, scale=1.0):
    return bf16_bits(np.random.default_rng(seed).standard_normal(shape) * scale)


def _f(a):
    return bf16_value(a).astype(np.float64)


def _rows(idx, T, N):
    return sorted({int(i) * T + t for i in idx for t in range(T) if 0 <= int(i) * T + t < N})


def test_rla_state_is_expK_transpose_V_and_additive():
    K, V = _bf((37, 8), 1, 0.7), _bf((37, 8), 2)
    S, z = oracle.rla_state(K, V)
    np.testing.assert_allclose(S, np.exp(_f(K)).T @ _f(V), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z, np.exp(_f(K)).sum(0), rtol=1e-12)
    S1, z1 = oracle.rla_state(K, V, 0, 20)
    S2, z2 = oracle.rla_state(K, V, 20, 37)
    np.testing.assert_allclose(S1 + S2, S, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z1 + z2, z, rtol=1e-12)


@pytest.mark.parametrize("T", [1, 4])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_rla_subtraction_form_equals_direct_definition(T, seed):
    rng = np.random.default_rng(seed)
    N, d, G = 50, 16, 3                      # N = 50 with T = 4: the last block holds 2 rows
    q, K, V = _bf((G, d), 10 + seed, 0.5), _bf((N, d), 20 + seed, 0.5), _bf((N, d), 30 + seed)
    M = (N + T - 1) // T
    idx = np.sort(rng.choice(M, size=int(rng.integers(1, M)), replace=False)).astype(np.int32)
    if T == 4 and (M - 1) not in idx:
        idx = np.append(idx, M - 1).astype(np.int32)    # include the ragged block
    S, z = oracle.rla_state(K, V)
    direct = oracle.rla_direct(q, K, V, idx, T)
    sub = oracle.rla_subtract(q, K, V, idx, S, z, T)
    np.testing.assert_allclose(sub, direct, rtol=1e-9, atol=1e-12)
    assert np.abs(direct).max() > 1e-3


def test_rla_equal_keys_give_the_plain_mean_of_the_left_out_values():
    N, d = 23, 8
    q, V = _bf((2, d), 3), _bf((N, d), 4)
    K = np.zeros((N, d), np.uint16)                      # every key 0: every weight sum_i exp(q_i)
    idx = np.array([0, 5, 6, 22], np.int32)
    keep = [n for n in range(N) if n not in set(idx.tolist())]
    o = oracle.rla_direct(q, K, V, idx)
    np.testing.assert_allclose(o, np.repeat(_f(V)[keep].mean(0, keepdims=True), 2, 0), rtol=1e-12, atol=1e-15)


def test_rla_one_left_out_row_is_its_value_and_full_support_is_zero():
    N, d = 19, 8
    q, K, V = _bf((2, d), 5), _bf((N, d), 6), _bf((N, d), 7)
    idx = np.array([n for n in range(N) if n != 11], np.int32)
    np.testing.assert_allclose(oracle.rla_direct(q, K, V, idx), np.repeat(_f(V)[11:12], 2, 0), rtol=1e-13)
    full = np.arange(N, dtype=np.int32)
    S, z = oracle.rla_state(K, V)
    assert not oracle.rla_direct(q, K, V, full).any()
    assert not oracle.rla_subtract(q, K, V, full, S, z).any()


def test_rla_with_one_feature_is_unit_scale_softmax_attention():
    # d = 1: w_n = e^q e^{k_n}, so the RLA output is softmax(k) over the left-out rows applied
    # to V -- torch's fp64 attention with query 1 and scale 1
    N = 40
    q, K, V = _bf((1, 1), 8), _bf((N, 1), 9, 2.0), _bf((N, 1), 10)
    idx = np.array([1, 2, 3, 30], np.int32)
    keep = [n for n in range(N) if n not in set(idx.tolist())]
    Kt = torch.tensor(_f(K)[keep])[None, None]
    Vt = torch.tensor(_f(V)[keep])[None, None]
    ref = torch.nn.functional.scaled_dot_product_attention(torch.ones(1, 1, 1, 1, dtype=torch.float64), Kt, Vt,
                                                           scale=1.0)[0, 0, 0].numpy()
    np.testing.assert_allclose(oracle.rla_direct(q, K, V, idx)[0], ref, rtol=1e-12)


def test_rla_is_invariant_to_a_common_shift_of_the_query():
    rng = np.random.default_rng(3)
    d, N = 16, 31
    qv = rng.integers(-16, 17, (2, d)) / 8.0                 # dyadic: q and q + 1 are exact in bf16
    q, q1 = bf16_bits(qv), bf16_bits(qv + 1.0)
    assert np.array_equal(_f(q1), qv + 1.0)
    K, V = _bf((N, d), 11, 0.5), _bf((N, d), 12)
    idx = np.array([4, 9, 10, 30], np.int32)
    np.testing.assert_allclose(oracle.rla_direct(q1, K, V, idx), oracle.rla_direct(q, K, V, idx), rtol=1e-11)
    # a shift of one component only changes the weights' ratios
    q2 = bf16_bits(qv + np.eye(d)[0])
    assert not np.allclose(oracle.rla_direct(q2, K, V, idx), oracle.rla_direct(q, K, V, idx), rtol=1e-6)


@pytest.mark.parametrize("eps", [0.0, 1e-6, 0.5])
def test_rms_norm_vs_torch(eps):
    rng = np.random.default_rng(4)
    x, g = rng.standard_normal(64) * 0.01, rng.uniform(0.5, 1.5, 64)
    ref = torch.nn.functional.rms_norm(torch.tensor(x), (64,), weight=torch.tensor(g), eps=eps).numpy()
    np.testing.assert_allclose(oracle.rms_norm(x, g, eps), ref, rtol=1e-12)


def test_decode_driver_adds_the_normalised_rla_to_the_exact_output():
    cfg = SMALL["c3s"]
    x = decode_inputs(cfg)
    rng = np.random.default_rng(5)
    gamma = rng.uniform(0.5, 1.5, (cfg.Hq, cfg.d)).astype(np.float32)
    eps = 1e-6
    plain = oracle.decode(cfg, x, units=[1])[0]
    res = oracle.decode(cfg, x, units=[1], rla={"gamma": gamma, "eps": eps})[0]
    np.testing.assert_array_equal(res["out_exact"], plain["out"])
    np.testing.assert_array_equal(res["lse"], plain["lse"])
    b, g = res["b"], res["g"]
    heads = slice(g * cfg.G, (g + 1) * cfg.G)
    S, z = oracle.rla_state(x["K"][b, g], x["V"][b, g])
    sub = oracle.rla_subtract(x["q"][b, heads], x["K"][b, g], x["V"][b, g], res["idx"], S, z, cfg.block)
    np.testing.assert_allclose(res["o_rla"], sub, rtol=1e-9, atol=1e-12)
    for i in range(cfg.G):
        o = res["o_rla"][i]
        y = res["out"][i] - res["out_exact"][i]
        np.testing.assert_allclose(y, gamma[g * cfg.G + i] * o / np.sqrt(np.mean(o * o) + np.float32(eps)),
                                   rtol=1e-9, atol=1e-12)
    zero = oracle.decode(cfg, x, units=[1], rla={"gamma": np.zeros_like(gamma), "eps": eps})[0]
    np.testing.assert_array_equal(zero["out"], plain["out"])
