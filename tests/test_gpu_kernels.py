"""Parity of each libspa.so entry point against the fp64 oracle, through the C ABI.

Inputs are the seeded synthetic workloads (synth/) at sizes the oracle finishes in
seconds, spanning several tiles and ending on ragged tails, plus edge cases.  Both sides
always receive the same input arrays; no expected value comes from the CUDA path.
"""
import math

import numpy as np
import pytest

import oracle
from parity import (check_outputs, compare_support, dev, dev_bf16, score_band, topk_band, topp_band)
from synth import C1, SMALL, bf16_bits, bf16_value, decode_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import long_context_sparse_spa_b200 as spa  # noqa: E402


def _np(t):
    return t.detach().cpu().numpy()


# ------------------------------------------------------------------ a2 low-rank scores
@pytest.mark.parametrize("name,collapse", [("c1s", "head"), ("c2s", "group"), ("c2s", "head")])
def test_lowrank_scores(name, collapse):
    cfg = SMALL[name].with_(collapse=collapse)
    x = decode_inputs(cfg)
    G = cfg.G
    coll = spa.SPA_COLLAPSE_GROUP_MEAN if collapse == "group" else spa.SPA_COLLAPSE_NONE
    scale = oracle.f32(cfg.score_scale)
    got = _np(spa.index_scores(spa.SPA_SCORE_LOWRANK, dev_bf16(x["q_idx"]), dev_bf16(x["Kidx"]), None, cfg.Hkv,
                               coll, scale))
    assert got.shape == (cfg.U, cfg.N)
    for u, (b, h) in enumerate(oracle.decode_units(cfg)):
        g, heads = (h // G, slice(h, h + 1)) if collapse == "head" else (h, slice(h * G, (h + 1) * G))
        ref = oracle.lowrank_scores(x["q_idx"][b, heads], x["Kidx"][b, g], collapse == "group", scale)
        ref = ref.reshape(-1)
        # fp32 bound of a 16-term dot product: 16 u sum|q k| (u = 2^-24), plus the final scaling
        qv = bf16_value(x["q_idx"][b, heads]).astype(np.float64).mean(0)
        mag = scale * np.abs(bf16_value(x["Kidx"][b, g]).astype(np.float64)) @ np.abs(qv)
        assert np.all(np.abs(got[u] - ref) <= 1e-6 * mag + 1e-7 * np.abs(ref) + 1e-30), f"unit {u}"


# ------------------------------------------------------------------ a1 block statistics, a3 Taylor scores
@pytest.mark.parametrize("d,block", [(128, 64), (64, 64), (128, 32)])
def test_block_stats(d, block):
    rng = np.random.default_rng(d + block)
    K = bf16_bits(rng.standard_normal((2, 3, block * 37 + 5, d)) * rng.uniform(0.3, 3.0))
    mean, var = spa.block_stats(dev_bf16(K), block)
    mean, var = _np(mean), _np(var)
    assert mean.shape == (2, 3, 37, d)
    for b in range(2):
        for g in range(3):
            rm, rv = oracle.block_stats(K[b, g], block)
            scale = np.abs(bf16_value(K[b, g])).max()
            np.testing.assert_allclose(mean[b, g], rm, rtol=0, atol=2e-6 * scale)
            np.testing.assert_allclose(var[b, g], rv, rtol=4e-6, atol=4e-6 * scale * scale)


@pytest.mark.parametrize("G,collapse", [(4, "group"), (8, "group"), (4, "head"), (1, "group")])
def test_taylor_scores(G, collapse):
    rng = np.random.default_rng(G)
    B, Hkv, M, d = 2, 2, 777, 128
    Hq = Hkv * G
    q = bf16_bits(rng.standard_normal((B, Hq, d)))
    mean = (rng.standard_normal((B, Hkv, M, d)) * 0.5).astype(np.float32)
    var = rng.uniform(0.05, 2.0, (B, Hkv, M, d)).astype(np.float32)
    scale = oracle.f32(1 / math.sqrt(d))
    coll = spa.SPA_COLLAPSE_GROUP_MEAN if collapse == "group" else spa.SPA_COLLAPSE_NONE
    got = _np(spa.index_scores(spa.SPA_SCORE_TAYLOR_BLOCK, dev_bf16(q), dev(mean), dev(var), Hkv, coll, scale))
    for b in range(B):
        for g in range(Hkv):
            t = oracle.taylor_scores(q[b, g * G:(g + 1) * G], mean[b, g].astype(np.float64),
                                     var[b, g].astype(np.float64), scale, collapse == "group")
            ref = np.log(t)
            if collapse == "group":
                np.testing.assert_allclose(got[b * Hkv + g], ref, rtol=0, atol=2e-5)
            else:
                for hh in range(G):
                    np.testing.assert_allclose(got[b * Hq + g * G + hh], ref[hh], rtol=0, atol=2e-5)


# ------------------------------------------------------------------ a4-a6 selection
def _score_rows(kind, U, M, seed):
    rng = np.random.default_rng(seed)
    if kind == "gauss":
        return rng.standard_normal((U, M)).astype(np.float32) * 3
    if kind == "ties":                       # heavy exact ties
        return (np.round(rng.standard_normal((U, M)) * 4) / 4).astype(np.float32)
    if kind == "equal":
        return np.zeros((U, M), np.float32)
    if kind == "needles":
        s = rng.standard_normal((U, M)).astype(np.float32)
        for u in range(U):
            s[u, rng.choice(M, 20, replace=False)] += 9.0
        return s
    raise ValueError(kind)


SELECT_CASES = [
    # (kind, U, M, k, sink, window)
    ("gauss", 4, 4096, 256, 4, 64),
    ("gauss", 3, 9001, 700, 4, 128),
    ("ties", 5, 3000, 333, 2, 7),
    ("equal", 2, 1000, 10, 3, 3),
    ("gauss", 2, 33, 40, 0, 0),          # k >= M: everything
    ("gauss", 2, 513, 0, 5, 9),          # k = 0: forced only
    ("gauss", 16, 131072, 2048, 4, 128),  # several CTAs per cluster
    ("needles", 64, 2048, 32, 1, 2),
    ("gauss", 1, 1, 1, 1, 1),
    ("gauss", 3, 50003, 5000, 600, 600),  # forced ranges overlapping the top set
    ("gauss", 2, 1000003, 5000, 4, 128),  # chunks streamed from L2 (1024-thread CTAs), ragged tail
]


@pytest.mark.parametrize("case", SELECT_CASES, ids=lambda c: "-".join(map(str, c)))
def test_select_topk(case):
    kind, U, M, k, sink, window = case
    s = _score_rows(kind, U, M, U * 7 + M)
    idx, count = spa.select_topk(dev(s), k, sink, window)
    idx, count = _np(idx), _np(count)
    for u in range(U):
        ref = oracle.select_topk(s[u].astype(np.float64), k, sink, window)
        assert count[u] == ref.size
        # identical binary32 inputs on both sides: bit-exact, no tie allowance
        np.testing.assert_array_equal(idx[u, :count[u]], ref)


def test_select_topk_unit_len():
    U, M = 6, 5000
    s = _score_rows("gauss", U, M, 1)
    L = np.array([5000, 4000, 1, 0, 2500, 77], np.int32)
    idx, count = spa.select_topk(dev(s), 100, 4, 8, unit_len=dev(L))
    idx, count = _np(idx), _np(count)
    for u in range(U):
        ref = oracle.select_topk(s[u, :L[u]].astype(np.float64), 100, 4, 8)
        np.testing.assert_array_equal(idx[u, :count[u]], ref)


TOPP_CASES = [
    # (kind, U, M, p, sink, window)
    ("gauss", 4, 4096, 0.9, 4, 64),
    ("needles", 16, 65536, 0.9, 4, 128),
    ("needles", 3, 9001, 0.5, 4, 128),
    ("ties", 4, 7000, 0.8, 2, 3),
    ("equal", 2, 1000, 0.5, 0, 0),
    ("gauss", 2, 3000, 1.0, 0, 0),
    ("gauss", 2, 3000, 1e-6, 3, 3),
    ("needles", 2, 262144, 0.9, 4, 256),   # clusters of 16 CTAs
    ("needles", 1, 1048583, 0.9, 4, 256),  # chunks streamed from L2 (1024-thread CTAs), ragged tail
]


@pytest.mark.parametrize("case", TOPP_CASES, ids=lambda c: "-".join(map(str, c)))
def test_select_topp(case):
    kind, U, M, p, sink, window = case
    s = _score_rows(kind, U, M, U * 11 + M)
    idx, count, mass = spa.select_topp(dev(s), p, sink, window)
    idx, count, mass = _np(idx), _np(count), _np(mass)
    pf = oracle.f32(p)
    ties = 0
    for u in range(U):
        su = s[u].astype(np.float64)
        ref, ref_mass, _ = oracle.select_topp(su, pf, sink, window)
        ties += compare_support(idx[u, :count[u]], ref, topp_band(su, pf), f"unit {u}")
        if ties == 0:
            assert abs(mass[u] - ref_mass) <= 2e-6
    print(f"top-p {case}: {ties} tie differences")


# ------------------------------------------------------------------ a7/a8 sparse attention
def _attend_case(cfg, units_idx, collapse, unit_tokens=1):
    x = decode_inputs(cfg)
    U = len(units_idx)
    cap = max(1, max(len(i) for i in units_idx))
    idx = np.full((U, cap), -1, np.int32)
    count = np.zeros(U, np.int32)
    for u, s in enumerate(units_idx):
        idx[u, :len(s)] = s
        count[u] = len(s)
    coll = spa.SPA_COLLAPSE_GROUP_MEAN if collapse == "group" else spa.SPA_COLLAPSE_NONE
    sm = oracle.f32(cfg.sm_scale)
    out, out32, lse = spa.sparse_attend(dev_bf16(x["q"]), dev_bf16(x["K"]), dev_bf16(x["V"]), dev(idx), dev(count),
                                        coll, sm, unit_tokens)
    out, out32, lse = _np(out.view(torch.int16)).view(np.uint16), _np(out32), _np(lse)
    G = cfg.G
    worst = 0.0
    for u in range(U):
        if collapse == "group":
            b, g = divmod(u, cfg.Hkv)
            heads = slice(g * G, (g + 1) * G)
        else:
            b, h = divmod(u, cfg.Hq)
            g, heads = h // G, slice(h, h + 1)
        ro, rl = oracle.sparse_attention(x["q"][b, heads], x["K"][b, g], x["V"][b, g], idx[u, :count[u]], sm,
                                         unit_tokens)
        worst = max(worst, check_outputs(out[b, heads], out32[b, heads], ro, f"unit {u}"))
        fin = np.isfinite(rl)
        np.testing.assert_array_equal(np.isfinite(lse[b, heads]), fin)
        np.testing.assert_allclose(lse[b, heads][fin], rl[fin], rtol=2e-6, atol=2e-6)
    return worst


def test_attend_group_random_supports():
    cfg = SMALL["c2s"]
    rng = np.random.default_rng(5)
    sizes = [1, 15, 16, 17, 1000, 4099, 33, 0, 9001, 250]
    units = []
    for u in range(cfg.B * cfg.Hkv):
        n = sizes[u % len(sizes)]
        units.append(np.sort(rng.choice(cfg.N, n, replace=False)).astype(np.int32))
    err = _attend_case(cfg, units, "group")
    print(f"max abs error {err:.2e}")


def test_attend_per_head_d64():
    cfg = C1
    rng = np.random.default_rng(6)
    units = [np.sort(rng.choice(cfg.N, n, replace=False)).astype(np.int32) for n in (320, 1, 4096, 77)]
    _attend_case(cfg, units, "head")


def test_attend_block_supports():
    cfg = SMALL["c3s"]
    rng = np.random.default_rng(7)
    nb = cfg.N // 64
    units = [np.sort(rng.choice(nb, n, replace=False)).astype(np.int32) for n in (15, 1, 300, 0)]
    _attend_case(cfg, units, "group", unit_tokens=64)


def test_attend_out_of_range_entries_are_skipped():
    cfg = SMALL["c2s"]
    units = [np.array([0, 5, 9000], np.int32), np.array([3, 9001, 20000], np.int32)] + \
            [np.array([1], np.int32)] * (cfg.B * cfg.Hkv - 2)
    # rows >= N contribute nothing on either side
    _attend_case(cfg, units, "group")
