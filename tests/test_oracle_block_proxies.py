"""Pins of the oracle's first-order block proxies: min/max pooling (a min-max page score)
and mean pooling ("SPLA", section 1; "The Sparse Frontier", token-to-page decode selection;
PBS-Attn, section 4).

The min-max score is the largest logit any key inside the block's channel box can reach,
so it bounds every real key of the block from above and is tight when the block holds one
key or identical keys.  The mean score is the first-order term of the Taylor score: with
zero variance the Taylor score's log equals it, and the head collapse is the score of the
mean query.
"""
import numpy as np
import pytest

import oracle
from synth import bf16_bits, bf16_value


def _bf(shape, seed, scale=1.0):
    return bf16_bits(np.random.default_rng(seed).standard_normal(shape) * scale)


def _f(a):
    return bf16_value(a).astype(np.float64)


def test_block_minmax_vs_numpy():
    K = _bf((64 * 5 + 9, 24), 1)
    mn, mx = oracle.block_minmax(K, 64)
    Kf = _f(K)[: 5 * 64].reshape(5, 64, 24)
    np.testing.assert_array_equal(mn, Kf.min(1))
    np.testing.assert_array_equal(mx, Kf.max(1))


@pytest.mark.parametrize("block", [4, 64])
def test_minmax_score_bounds_every_key_logit_of_its_block(block):
    N, d, G, scale = block * 12, 32, 3, 0.2
    K, q = _bf((N, d), 2), _bf((G, d), 3)
    mn, mx = oracle.block_minmax(K, block)
    s = oracle.minmax_scores(q, mn, mx, scale, False)
    logits = scale * (_f(q) @ _f(K).T).reshape(G, N // block, block)
    best = logits.max(-1)
    assert (s >= best - 1e-12).all()
    assert (s > best + 1e-3).any()         # a box bound, not the maximum itself
    np.testing.assert_allclose(oracle.minmax_scores(q, mn, mx, scale, True), s.mean(0), rtol=1e-14)


def test_minmax_score_is_tight_for_single_key_and_identical_key_blocks():
    N, d, G, scale = 40, 16, 2, 0.5
    K, q = _bf((N, d), 4), _bf((G, d), 5)
    mn, mx = oracle.block_minmax(K, 1)
    np.testing.assert_allclose(oracle.minmax_scores(q, mn, mx, scale, False), scale * _f(q) @ _f(K).T,
                               rtol=1e-14, atol=1e-15)
    Kr = np.repeat(K[:5], 8, axis=0)        # blocks of 8 identical keys
    mn, mx = oracle.block_minmax(Kr, 8)
    np.testing.assert_allclose(oracle.minmax_scores(q, mn, mx, scale, False), scale * _f(q) @ _f(K[:5]).T,
                               rtol=1e-14, atol=1e-15)


def test_mean_score_is_the_zero_variance_taylor_exponent_and_collapses_linearly():
    N, d, G, scale = 64 * 7, 32, 4, 1 / np.sqrt(32)
    K, q = _bf((N, d), 6), _bf((G, d), 7)
    mean, _ = oracle.block_stats(K, 64)
    per_head = oracle.mean_scores(q, mean, scale, False)
    for h in range(G):
        t = oracle.taylor_scores(q[h:h + 1], mean, np.zeros_like(mean), scale, True)
        np.testing.assert_allclose(per_head[h], np.log(t), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.mean_scores(q, mean, scale, True), scale * _f(q).mean(0) @ mean.T,
                               rtol=1e-12, atol=1e-14)


def _nearest_even_bf16(x):
    """Brute force: the bf16 pattern nearest to x among the neighbours of its float32
    truncation, ties to the even pattern."""
    t = int(np.array([x], np.float32).view(np.uint32)[0] >> 16)
    best = None
    for c in (t - 1, t, t + 1, t + 2):
        v = oracle.widen_bf16(np.array([c & 0xFFFF], np.uint16))[0]
        key = (abs(x - v), c & 1)
        if best is None or key < best[0]:
            best = (key, c & 0xFFFF)
    return best[1]


def test_round_bf16_is_nearest_even_from_double():
    rng = np.random.default_rng(8)
    xs = np.concatenate([rng.standard_normal(400) * 10.0 ** rng.integers(-6, 6, 400),
                         rng.uniform(0, 1e-3, 50)])
    # exact halfway points between adjacent bf16 values, and just beside them
    base = oracle.round_bf16(rng.uniform(0.1, 100, 60))
    lo, hi = oracle.widen_bf16(base), oracle.widen_bf16(base + 1)
    mid = (lo + hi) / 2
    xs = np.concatenate([xs, mid, np.nextafter(mid, 0), np.nextafter(mid, np.inf), -mid])
    got = oracle.round_bf16(xs)
    want = np.array([_nearest_even_bf16(abs(x)) | (0x8000 if x < 0 else 0) for x in xs], np.uint16)
    np.testing.assert_array_equal(got, want)
    halfway = got[450:510]
    assert (halfway & 1 == 0).all()            # ties went to the even pattern
