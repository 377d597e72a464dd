"""Pins of the oracle's permuted block-sparse prefill (PBS-Attn, "Sparser Block-Sparse
Attention via Token Permutation", sections 1-4).

The key importance is checked against torch's fp64 softmax, the segment order against
numpy's lexsort, the full and empty budgets against torch's fp64 attention (dense causal,
and causal inside the query's own segment), the whole path against its own premise --
attention is invariant to a joint shuffle of the key-value pairs inside segments -- and
the clustering it is built for: scattered heavy hitters land in one permuted block.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import bf16_bits, bf16_value


def _bf(shape, seed, scale=1.0):
    return bf16_bits(np.random.default_rng(seed).standard_normal(shape) * scale)


def _f(a):
    return bf16_value(a).astype(np.float64)


def _attn(q, K, V, scale, keep):
    """torch fp64 attention of one query q [d] over the rows `keep` of K, V."""
    qt = torch.tensor(q)[None, None, None]
    Kt = torch.tensor(K[keep])[None, None]
    Vt = torch.tensor(V[keep])[None, None]
    return torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)[0, 0, 0].numpy()


def test_importance_is_mean_causal_softmax_of_the_last_block():
    T, d, G, bl = 96, 16, 2, 8
    K = _bf((T, d), 1)
    Q = _bf((bl, G, d), 2)
    imp = oracle.pbs_importance(Q, T - bl, K, 0.25)
    logits = 0.25 * np.einsum("ihc,nc->ihn", _f(Q), _f(K))
    mask = np.arange(T)[None, None, :] <= (T - bl + np.arange(bl))[:, None, None]
    P = torch.softmax(torch.tensor(np.where(mask, logits, -np.inf)), dim=-1).numpy()
    np.testing.assert_allclose(imp, P.mean(axis=(0, 1)), rtol=1e-12, atol=1e-15)
    assert abs(imp.sum() - 1.0) < 1e-12


@pytest.mark.parametrize("T,S", [(64, 16), (70, 16), (64, 64), (10, 32)])
def test_permutation_sorts_inside_segments_by_lexsort(T, S):
    rng = np.random.default_rng(T + S)
    imp = rng.integers(0, 5, T) / 4.0                 # many ties
    perm = oracle.pbs_permutation(imp, S)
    assert sorted(perm.tolist()) == list(range(T))
    for s0 in range(0, T, S):
        seg = np.arange(s0, min(s0 + S, T))
        ref = seg[np.lexsort((seg, -imp[seg]))]
        np.testing.assert_array_equal(perm[s0:s0 + S], ref)


def _case(seed, T=128, d=16, G=2):
    return _bf((T, G, d), seed), _bf((T, d), seed + 1), _bf((T, d), seed + 2)


@pytest.mark.parametrize("t0", [0, 32, 64, 112])
def test_full_budget_is_dense_causal_attention(t0):
    b, S, T, scale = 16, 32, 128, 0.3
    Q, K, V = _case(3, T)
    perm = oracle.pbs_permutation(oracle.pbs_importance(Q[T - b:], T - b, K, scale), S)
    sup, out = oracle.pbs_prefill_unit(Q[t0:t0 + b], t0, K, V, perm, S, 10**6, scale)
    np.testing.assert_array_equal(sup, np.arange(t0 // S * S))
    for i in range(b):
        for h in range(2):
            ref = _attn(_f(Q[t0 + i, h]), _f(K), _f(V), scale, np.arange(t0 + i + 1))
            np.testing.assert_allclose(out[i, h], ref, rtol=1e-11, atol=1e-12)


def test_empty_budget_is_causal_attention_inside_the_own_segment():
    b, S, T, scale, t0 = 16, 32, 128, 0.3, 80
    Q, K, V = _case(4, T)
    perm = np.arange(T, dtype=np.int32)
    sup, out = oracle.pbs_prefill_unit(Q[t0:t0 + b], t0, K, V, perm, S, 0, scale)
    assert sup.size == 0
    for i in range(b):
        for h in range(2):
            ref = _attn(_f(Q[t0 + i, h]), _f(K), _f(V), scale, np.arange(64, t0 + i + 1))
            np.testing.assert_allclose(out[i, h], ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("seed", [0, 1])
def test_shuffling_kv_pairs_inside_segments_changes_nothing(seed):
    # PBS-Attn section 1: jointly permuted key-value pairs leave attention unchanged; the
    # importance sort then gives the same permuted blocks, so the same rows are selected
    b, S, T, scale, k = 16, 64, 256, 0.3, 3
    Q, K, V = _case(10 + seed, T)
    rng = np.random.default_rng(seed)
    sigma = np.concatenate([s0 + rng.permutation(S) for s0 in range(0, T, S)])   # new row n holds old sigma[n]
    K2, V2 = K[sigma], V[sigma]
    last = Q[T - b:]
    perm = oracle.pbs_permutation(oracle.pbs_importance(last, T - b, K, scale), S)
    perm2 = oracle.pbs_permutation(oracle.pbs_importance(last, T - b, K2, scale), S)
    for t0 in (64, 128, 192):
        # the query block's own segment is not shuffled relative to its queries' causal mask
        # only if it is unchanged: keep the own segment's rows in place
        K3, V3 = K2.copy(), V2.copy()
        seg = slice(t0 // S * S, T)
        K3[seg], V3[seg] = K[seg], V[seg]
        s3 = sigma.copy()
        s3[seg] = np.arange(T)[seg]
        perm3 = oracle.pbs_permutation(oracle.pbs_importance(last, T - b, K3, scale), S)
        sup, out = oracle.pbs_prefill_unit(Q[t0:t0 + b], t0, K, V, perm, S, k, scale)
        sup3, out3 = oracle.pbs_prefill_unit(Q[t0:t0 + b], t0, K3, V3, perm3, S, k, scale)
        np.testing.assert_array_equal(np.sort(s3[sup3]), sup)
        np.testing.assert_allclose(out3, out, rtol=1e-11, atol=1e-13)
    assert not np.array_equal(perm, perm2)


def test_scattered_heavy_hitters_cluster_into_one_permuted_block():
    # segment 0 holds b keys aligned with the queries at scattered positions; sorted by
    # importance they fill permuted block 0, and a budget of one block selects exactly them
    b, S, T, d, scale = 16, 128, 256, 16, 0.25
    rng = np.random.default_rng(5)
    u = np.zeros(d); u[0] = 1.0
    Kf = rng.standard_normal((T, d)) * 0.3
    heavy = np.sort(rng.choice(S, b, replace=False))
    Kf[heavy] += 4.0 * u
    Qf = rng.standard_normal((T, 1, d)) * 0.3 + 2.0 * u
    K, Q, V = bf16_bits(Kf), bf16_bits(Qf), _bf((T, d), 6)
    perm = oracle.pbs_permutation(oracle.pbs_importance(Q[T - b:], T - b, K, scale), S)
    np.testing.assert_array_equal(np.sort(perm[:b]), heavy)
    sup, _ = oracle.pbs_prefill_unit(Q[192:208], 192, K, V, perm, S, 1, scale)
    np.testing.assert_array_equal(sup, heavy)
    # without the permutation a one-block budget cannot hold them: they span several blocks
    assert len(set((heavy // b).tolist())) > 1


def test_pbs_output_is_sparse_attention_over_support_and_earlier_own_segment_rows():
    # the form the GPU path reuses: rows = selected permuted blocks (original positions) and
    # the own segment's rows before the query block, plus the block's causal diagonal --
    # the same row set as the shared-support prefill's, with [seg0, t0) added to the support
    b, S, T, scale, k = 16, 64, 256, 0.3, 2
    Q, K, V = _case(20, T)
    perm = oracle.pbs_permutation(oracle.pbs_importance(Q[T - b:], T - b, K, scale), S)
    for t0 in (80, 160, 240):
        sup, out = oracle.pbs_prefill_unit(Q[t0:t0 + b], t0, K, V, perm, S, k, scale)
        seg0 = t0 // S * S
        base = np.concatenate([sup, np.arange(seg0, t0)]).astype(np.int32)
        for i in range(b):
            rows = np.concatenate([base, np.arange(t0, t0 + i + 1)]).astype(np.int32)
            for h in range(2):
                ref, _ = oracle.sparse_attention(Q[t0 + i, h:h + 1], K, V, rows, scale)
                np.testing.assert_allclose(out[i, h], ref[0], rtol=1e-12, atol=1e-14)
