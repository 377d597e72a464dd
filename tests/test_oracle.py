"""Pins of the fp64 oracle against things other than itself.

Each test checks an oracle routine against a library routine (torch's fp64
scaled_dot_product_attention, numpy's lexsort / mean / var), a closed form, an
invariant, brute force on tiny inputs, or a hand-derived worked example
(tests/golden/worked_examples.jsonl).  The cases are chosen so that a plausible
mistake -- a dropped term, a wrong sign or index, a transposed operand, > for >= --
fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from synth import C1, SMALL, bf16_bits, bf16_value, decode_inputs, prefill_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.jsonl")


def _bf(shape, seed, scale=1.0):
    return bf16_bits(np.random.default_rng(seed).standard_normal(shape) * scale)


def _sdpa(q, K, V, scale, mask=None):
    """torch fp64 attention: q [G, d], K/V [N, d] as float arrays; mask [G, N] bool (True = keep)."""
    qt = torch.tensor(q, dtype=torch.float64)[None, :, None, :]     # [1, G, 1, d]
    Kt = torch.tensor(K, dtype=torch.float64)[None, None].expand(1, q.shape[0], -1, -1)
    Vt = torch.tensor(V, dtype=torch.float64)[None, None].expand(1, q.shape[0], -1, -1)
    m = None if mask is None else torch.tensor(mask)[None, :, None, :]
    return torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, attn_mask=m, scale=scale)[0, :, 0].numpy()


# ------------------------------------------------------------------ golden worked examples
def _golden():
    with open(GOLDEN) as f:
        return [json.loads(line) for line in f if line.strip()]


@pytest.mark.parametrize("case", _golden(), ids=lambda c: c["name"])
def test_worked_examples(case):
    kind = case["kind"]
    if kind == "topp":
        idx, mass, cut = oracle.select_topp(np.array(case["scores"]), case["p"], case["sink"], case["window"])
        assert idx.tolist() == case["support"]
        assert cut == case["cut"]
    elif kind == "topk":
        idx = oracle.select_topk(np.array(case["scores"]), case["k"], case["sink"], case["window"])
        assert idx.tolist() == case["support"]
    elif kind == "block_stats":
        mean, var = oracle.block_stats(bf16_bits(np.array(case["K"])), case["block"])
        np.testing.assert_array_equal(mean, case["mean"])
        np.testing.assert_array_equal(var, case["var"])
    elif kind == "taylor":
        t = oracle.taylor_scores(bf16_bits(np.array([case["q"]])), np.array(case["mean"]), np.array(case["var"]),
                                 case["scale"], True)
        np.testing.assert_allclose(t, case["t"], rtol=1e-15)
    else:
        raise AssertionError(kind)


# ------------------------------------------------------------------ a1 block statistics
def test_block_stats_vs_numpy():
    K = _bf((64 * 5 + 13, 32), 1, 2.0)   # ragged tail: 13 tokens of an unfilled block
    mean, var = oracle.block_stats(K, 64)
    Kf = bf16_value(K).astype(np.float64)[: 5 * 64].reshape(5, 64, 32)
    assert mean.shape == (5, 32)
    np.testing.assert_allclose(mean, Kf.mean(1), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(var, Kf.var(1, ddof=0), rtol=1e-13, atol=1e-14)


# ------------------------------------------------------------------ a2 low-rank scores
def test_lowrank_scores_vs_matmul_and_collapse():
    qidx = _bf((8, 16), 2)
    kidx = _bf((1000, 16), 3)
    s = oracle.lowrank_scores(qidx, kidx, False, 0.7)
    ref = 0.7 * bf16_value(qidx).astype(np.float64) @ bf16_value(kidx).astype(np.float64).T
    np.testing.assert_allclose(s, ref, rtol=1e-13, atol=1e-13)
    # head collapse = score with the group-mean index query = mean of the heads' scores
    sc = oracle.lowrank_scores(qidx, kidx, True, 0.7)
    np.testing.assert_allclose(sc, ref.mean(0), rtol=1e-12, atol=1e-12)
    # with G = 1 collapse is per head
    np.testing.assert_array_equal(oracle.lowrank_scores(qidx[:1], kidx, True, 0.7), s[0])


# ------------------------------------------------------------------ a3 Taylor block score
def test_taylor_zero_variance_is_exact_block_mass():
    """Identical keys in a block: the score equals the block's exact mean of exp(q'.k)."""
    d, nb = 64, 6
    rng = np.random.default_rng(4)
    rows = _bf((nb, d), 5, 0.5)
    K = np.repeat(rows, 64, axis=0)                 # every block holds one key 64 times
    mean, var = oracle.block_stats(K, 64)
    assert np.all(var == 0.0)
    q = _bf((3, d), 6)
    scale = 1.0 / math.sqrt(d)
    t = oracle.taylor_scores(q, mean, var, scale, False)
    qf = bf16_value(q).astype(np.float64)
    Kf = bf16_value(K).astype(np.float64).reshape(nb, 64, d)
    exact = np.exp(np.einsum("hd,bnd->hbn", qf, Kf) * scale).mean(2)
    np.testing.assert_allclose(t, exact, rtol=1e-13)
    tc = oracle.taylor_scores(q, mean, var, scale, True)
    np.testing.assert_allclose(tc, exact.mean(0), rtol=1e-13)
    del rng


def test_taylor_second_order_on_axis_symmetric_blocks():
    """Blocks whose keys are kbar +- delta along one axis per pair have an exactly diagonal
    covariance and no odd moments, so the exact block mass is
        exp(q'.kbar) * (1/64) sum_pairs 2 cosh(q'_a delta)
    and the second-order score must agree with it up to the fourth-order term
        exp(q'.kbar) * (1/768) sum_pairs (q'_a delta)^4.
    A dropped 1/2, a missing square or a wrong sign of the mean term fails this."""
    d = 64
    rng = np.random.default_rng(7)
    for trial in range(20):
        kbar = rng.integers(-8, 9, d) / 8.0                     # dyadic: exact in bf16
        axes = rng.choice(d, 32, replace=False)
        deltas = rng.choice([0.125, 0.25, 0.5], 32)
        keys = []
        for a, dl in zip(axes, deltas):
            for sgn in (1.0, -1.0):
                k = kbar.copy()
                k[a] += sgn * dl
                keys.append(k)
        K = bf16_bits(np.array(keys))
        assert np.array_equal(bf16_value(K), np.array(keys, dtype=np.float32))
        mean, var = oracle.block_stats(K, 64)
        q = _bf((1, d), 100 + trial, 2.0)
        scale = 1.0 / math.sqrt(d)
        t = oracle.taylor_scores(q, mean, var, scale, True)[0]
        qp = bf16_value(q)[0].astype(np.float64) * scale
        x = qp[axes] * deltas
        base = math.exp(float(qp @ kbar))
        exact = base * np.sum(2.0 * np.cosh(x)) / 64.0
        fourth = base * np.sum(x ** 4) / 768.0
        assert abs(t - exact) <= 1.01 * fourth + 1e-12 * exact
        assert abs(t - exact) >= 0.9 * fourth - 1e-12 * exact   # the gap IS the fourth-order term


# ------------------------------------------------------------------ a5 top-k
@pytest.mark.parametrize("seed", range(6))
def test_topk_vs_lexsort(seed):
    rng = np.random.default_rng(seed)
    M = int(rng.integers(1, 400))
    s = np.round(rng.standard_normal(M) * 3) / 2          # many exact ties
    k = int(rng.integers(0, M + 3))
    sink = int(rng.integers(0, 5)); window = int(rng.integers(0, 7))
    idx = oracle.select_topk(s, k, sink, window)
    order = np.lexsort((np.arange(M), -s))                 # by score desc, then position asc
    keep = set(order[:k].tolist()) | set(range(min(sink, M))) | set(range(max(0, M - window), M))
    assert idx.tolist() == sorted(keep)
    np.testing.assert_array_equal(oracle.rank_order(s), order)


def test_topk_k_at_least_M_keeps_everything():
    s = np.random.default_rng(9).standard_normal(50)
    assert oracle.select_topk(s, 50, 0, 0).tolist() == list(range(50))
    assert oracle.select_topk(s, 80, 2, 2).tolist() == list(range(50))


# ------------------------------------------------------------------ a4-a6 top-p
@pytest.mark.parametrize("seed", range(25))
def test_topp_is_minimal_subset_by_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    M = int(rng.integers(1, 12))
    s = rng.standard_normal(M) * float(rng.uniform(0.2, 3.0))
    p = float(rng.uniform(0.05, 1.0))
    idx, mass, cut = oracle.select_topp(s, p, 0, 0)
    w = np.exp(s - s.max()); w /= w.sum()
    best = None
    for m in range(1, M + 1):                              # smallest cardinality reaching p
        masses = [w[list(c)].sum() for c in itertools.combinations(range(M), m)]
        if max(masses) >= p * (1 - 1e-12):
            best = m
            break
    assert cut == best == len(idx)
    # the prefix is a maximum-mass subset of that size
    assert abs(w[idx].sum() - max(w[list(c)].sum() for c in itertools.combinations(range(M), best))) < 1e-12
    assert abs(mass - w[idx].sum()) < 1e-12


def test_topp_limits():
    s = np.random.default_rng(3).standard_normal(64)
    idx, _, cut = oracle.select_topp(s, 1e-12, 0, 0)
    assert idx.tolist() == [int(np.argmax(s))] and cut == 1
    idx, mass, cut = oracle.select_topp(s, 1.0, 0, 0)
    assert idx.tolist() == list(range(64)) and abs(mass - 1.0) < 1e-12
    idx, _, _ = oracle.select_topp(s, 1e-12, 3, 2)
    assert set(idx.tolist()) == {0, 1, 2, 62, 63, int(np.argmax(s))}
    with pytest.raises(ValueError):
        oracle.select_topp(s, 0.0, 0, 0)


# ------------------------------------------------------------------ a7/a8 sparse attention
def test_full_support_is_dense_attention():
    q, K, V = _bf((4, 64), 11), _bf((300, 64), 12, 2.0), _bf((300, 64), 13)
    out, lse = oracle.sparse_attention(q, K, V, np.arange(300), 0.125)
    qf, Kf, Vf = (bf16_value(a).astype(np.float64) for a in (q, K, V))
    np.testing.assert_allclose(out, _sdpa(qf, Kf, Vf, 0.125), rtol=1e-12, atol=1e-13)
    ref_lse = np.log(np.exp(0.125 * qf @ Kf.T).sum(1))
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-13)


def test_subset_support_is_masked_attention_and_order_free():
    rng = np.random.default_rng(14)
    q, K, V = _bf((8, 128), 15), _bf((500, 128), 16), _bf((500, 128), 17)
    idx = np.sort(rng.choice(500, 77, replace=False)).astype(np.int32)
    out, _ = oracle.sparse_attention(q, K, V, idx, 0.088)
    mask = np.zeros((8, 500), bool); mask[:, idx] = True
    qf, Kf, Vf = (bf16_value(a).astype(np.float64) for a in (q, K, V))
    np.testing.assert_allclose(out, _sdpa(qf, Kf, Vf, 0.088, mask), rtol=1e-12, atol=1e-13)
    out_perm, _ = oracle.sparse_attention(q, K, V, rng.permutation(idx), 0.088)   # KV-pair permutation
    np.testing.assert_allclose(out_perm, out, rtol=1e-13, atol=1e-14)


def test_singleton_block_and_empty_supports():
    q, K, V = _bf((2, 64), 18), _bf((256, 64), 19), _bf((256, 64), 20)
    out, _ = oracle.sparse_attention(q, K, V, np.array([37]), 0.125)
    np.testing.assert_array_equal(out, np.repeat(bf16_value(V[37:38]).astype(np.float64), 2, 0))
    # block support {1, 3} with 64-token blocks == token support of rows 64..127, 192..255
    ob, lb = oracle.sparse_attention(q, K, V, np.array([1, 3]), 0.125, unit_tokens=64)
    rows = np.r_[64:128, 192:256]
    ot, lt = oracle.sparse_attention(q, K, V, rows, 0.125)
    np.testing.assert_allclose(ob, ot, rtol=1e-14); np.testing.assert_allclose(lb, lt, rtol=1e-14)
    oe, le = oracle.sparse_attention(q, K, V, np.zeros(0, np.int32), 0.125)
    assert np.all(oe == 0.0) and np.all(np.isneginf(le))


def test_dense_probs():
    q, K = _bf((8, 64), 21), _bf((700, 64), 22)
    P = oracle.dense_probs(q, K, 0.125)
    assert abs(P.sum() - 1.0) < 1e-12
    P1 = oracle.dense_probs(q[:1], K, 0.125)
    logits = 0.125 * bf16_value(q[:1]).astype(np.float64) @ bf16_value(K).astype(np.float64).T
    np.testing.assert_allclose(P1, torch.softmax(torch.tensor(logits[0]), 0).numpy(), rtol=1e-12)


# ------------------------------------------------------------------ a9 shared-support prefill
def test_prefill_with_full_budget_is_dense_causal_attention():
    cfg = SMALL["c5s"].with_(N=640, q_start=512, T=128, Hq=4, Hkv=2, topk=10_000, n_clusters=4)
    x = prefill_inputs(cfg)
    G, bq, d = cfg.G, cfg.bq, cfg.d
    for j in range(cfg.n_blocks):
        for g in range(cfg.Hkv):
            support, out = oracle.prefill_block(cfg, x, j, g)
            t0 = cfg.q_start + j * bq
            assert support.tolist() == list(range(t0))
            for hh in range(G):
                h = g * G + hh
                qf = bf16_value(x["Q"][j * bq:(j + 1) * bq, h]).astype(np.float64)
                Kf = bf16_value(x["K"][g, : t0 + bq]).astype(np.float64)
                Vf = bf16_value(x["V"][g, : t0 + bq]).astype(np.float64)
                mask = np.arange(t0 + bq)[None, :] <= (t0 + np.arange(bq))[:, None]
                qt = torch.tensor(qf)[None, None]; Kt = torch.tensor(Kf)[None, None]; Vt = torch.tensor(Vf)[None, None]
                ref = torch.nn.functional.scaled_dot_product_attention(
                    qt, Kt, Vt, attn_mask=torch.tensor(mask)[None, None], scale=oracle.f32(cfg.sm_scale))[0, 0].numpy()
                np.testing.assert_allclose(out[:, hh], ref, rtol=1e-11, atol=1e-12)


def test_prefill_support_is_topk_of_block_mean_index_query():
    cfg = SMALL["c5s"].with_(N=1024, q_start=768, T=128, Hq=4, Hkv=2, topk=100, n_clusters=4)
    x = prefill_inputs(cfg)
    j, g = 1, 1
    support, _ = oracle.prefill_block(cfg, x, j, g)
    t0 = cfg.q_start + j * cfg.bq
    qi = bf16_value(x["q_idx"][j * 64:(j + 1) * 64, g * 2:(g + 1) * 2]).astype(np.float64).reshape(-1, 16)
    s = oracle.f32(cfg.score_scale) * (bf16_value(x["Kidx"][g, :t0]).astype(np.float64) @ qi.mean(0))
    s = s.astype(np.float32).astype(np.float64)
    order = np.lexsort((np.arange(t0), -s))
    assert support.tolist() == sorted(set(order[:100].tolist()) | {0, 1, 2, 3})


# ------------------------------------------------------------------ driver consistency
def test_decode_driver_c1():
    x = decode_inputs(C1)
    res = oracle.decode(C1, x)
    assert len(res) == C1.U
    for u, r in enumerate(res):
        idx = r["idx"]
        assert np.all(np.diff(idx) > 0)
        assert set(range(C1.sink)) <= set(idx.tolist())
        assert set(range(C1.N - C1.window, C1.N)) <= set(idx.tolist())
        assert C1.topk <= len(idx) <= C1.topk + C1.sink + C1.window
        # each head's planted needles are found
        b, h = oracle.decode_units(C1)[u]
        needles = x["needles"][(b, h // C1.G)]
        mine = [n for i, n in enumerate(sorted(needles)) if True]
        assert len(set(mine) & set(idx.tolist())) >= 1


# ------------------------------------------------------------------ head-wise routing (local units)
@pytest.mark.parametrize("M,sink,window", [(100, 4, 16), (10, 4, 8), (5, 0, 0), (7, 9, 2), (1, 1, 1)])
def test_local_support_is_sink_and_window(M, sink, window):
    """Brute force over the positions: a local unit keeps n < sink or n >= M - window."""
    want = [n for n in range(M) if n < sink or n >= M - window]
    assert oracle.local_support(M, sink, window).tolist() == want


def test_routed_decode_local_units_attend_over_sink_and_window():
    """A local unit of a routed decode attends over exactly its sink and window (torch fp64
    attention over those rows); the retrieval units are the unrouted path."""
    cfg = SMALL["c2s"]
    x = decode_inputs(cfg)
    local = [u % 2 == 1 for u in range(cfg.U)]
    routed = oracle.decode(cfg, x, local=local)
    plain = oracle.decode(cfg, x)
    for u, (r, q) in enumerate(zip(routed, plain)):
        if not local[u]:
            np.testing.assert_array_equal(r["idx"], q["idx"])
            np.testing.assert_array_equal(r["out"], q["out"])
            continue
        assert r["index_mass"] is None and r["scores"] is None
        rows = [n for n in range(cfg.N) if n < cfg.sink or n >= cfg.N - cfg.window]
        assert r["idx"].tolist() == rows
        b, g = r["b"], r["g"]
        heads = slice(g * cfg.G, (g + 1) * cfg.G)
        qf = bf16_value(x["q"][b, heads]).astype(np.float64)
        Kf = bf16_value(x["K"][b, g][rows]).astype(np.float64)
        Vf = bf16_value(x["V"][b, g][rows]).astype(np.float64)
        np.testing.assert_allclose(r["out"], _sdpa(qf, Kf, Vf, oracle.f32(cfg.sm_scale)), rtol=1e-10, atol=1e-12)


def test_per_query_prefill_b_sel_1():
    # "Oracle-Guided Sparse Prefill" 2.1 with b_sel = 1: every query has its own support,
    # scored with the mean of its G heads' index queries; a full budget is dense causal
    # attention, a budget of k is the lexsort top-k of those scores united with the sink
    cfg = SMALL["c5s"].with_(N=600, q_start=584, T=16, Hq=4, Hkv=2, bq=1, topk=10_000, n_clusters=4)
    x = prefill_inputs(cfg)
    G, d = cfg.G, cfg.d
    for j in (0, 7, 15):
        for g in range(cfg.Hkv):
            support, out = oracle.prefill_block(cfg, x, j, g)
            t = cfg.q_start + j
            assert support.tolist() == list(range(t))
            Kf = bf16_value(x["K"][g, : t + 1]).astype(np.float64)
            Vf = bf16_value(x["V"][g, : t + 1]).astype(np.float64)
            for hh in range(G):
                qf = bf16_value(x["Q"][j, g * G + hh]).astype(np.float64)
                ref = _sdpa(qf[None], Kf, Vf, oracle.f32(cfg.sm_scale))[0]
                np.testing.assert_allclose(out[0, hh], ref, rtol=1e-11, atol=1e-12)
    small = cfg.with_(topk=50)
    j, g = 9, 1
    support, _ = oracle.prefill_block(small, x, j, g)
    t = cfg.q_start + j
    qi = bf16_value(x["q_idx"][j, g * G:(g + 1) * G]).astype(np.float64)
    s = oracle.f32(cfg.score_scale) * (bf16_value(x["Kidx"][g, :t]).astype(np.float64) @ qi.mean(0))
    s = s.astype(np.float32).astype(np.float64)
    order = np.lexsort((np.arange(t), -s))
    assert support.tolist() == sorted(set(order[:50].tolist()) | set(range(cfg.sink)))


def test_captured_mass_prefill():
    """Captured mass of a prefill unit: 1 when the support holds every earlier key (the block's
    own rows are always read); otherwise the mean over queries of the brute-force causal
    head-averaged softmax summed over support and own rows ("Oracle-Guided Sparse Prefill" 2.1)."""
    cfg = SMALL["c5s"].with_(N=640, q_start=512, T=128, Hq=4, Hkv=2, topk=10_000, n_clusters=4)
    x = prefill_inputs(cfg)
    j, g = 1, 0
    t0 = cfg.q_start + j * cfg.bq
    assert abs(oracle.captured_mass_prefill(cfg, x, j, g, np.arange(t0)) - 1.0) < 1e-12
    sup = np.array([0, 1, 2, 3, 77, 300, 301, 555], np.int64)
    got = oracle.captured_mass_prefill(cfg, x, j, g, sup, queries=[0, 5, 63])
    vals = []
    for i in (0, 5, 63):
        t = t0 + i
        Kf = bf16_value(x["K"][g, : t + 1]).astype(np.float64)
        P = np.zeros(t + 1)
        for hh in range(cfg.G):
            qf = bf16_value(x["Q"][j * cfg.bq + i, g * cfg.G + hh]).astype(np.float64)
            P += torch.softmax(torch.tensor(oracle.f32(cfg.sm_scale) * (Kf @ qf)), 0).numpy() / cfg.G
        rows = sorted(set(sup.tolist()) | set(range(t0, t + 1)))
        vals.append(P[rows].sum())
    assert abs(got - np.mean(vals)) < 1e-12
