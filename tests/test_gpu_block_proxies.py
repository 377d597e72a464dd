"""First-order block proxies on the GPU against the fp64 oracle: block min/max statistics
(exact), the min-max page score and the mean-pooling score ("SPLA", section 1; "The Sparse
Frontier", token-to-page decode selection), alone and inside the fused decode step.

Scores are fp32 sums of d products of fp32 values; they are compared within 1e-5 relative
(plus 1e-5 absolute).  Supports follow the tie rule of the other decode tests.
"""
import numpy as np
import pytest

import oracle
from parity import check_outputs, compare_support, dev_bf16, topk_band
from synth import SMALL, decode_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import long_context_sparse_spa_b200 as spa  # noqa: E402


@pytest.mark.parametrize("name,block", [("c3s", 64), ("c1s", 32), ("c3s", 128)])
def test_block_minmax_is_exact(name, block):
    cfg = SMALL[name]
    x = decode_inputs(cfg)
    mn, mx = spa.block_minmax(dev_bf16(x["K"]), block)
    mn, mx = mn.cpu().numpy(), mx.cpu().numpy()
    for b in range(cfg.B):
        for g in range(cfg.Hkv):
            rmn, rmx = oracle.block_minmax(x["K"][b, g], block)
            np.testing.assert_array_equal(mn[b, g], rmn)
            np.testing.assert_array_equal(mx[b, g], rmx)


@pytest.mark.parametrize("kind", ["minmax", "mean"])
@pytest.mark.parametrize("collapse", [spa.SPA_COLLAPSE_GROUP_MEAN, spa.SPA_COLLAPSE_NONE])
def test_block_proxy_scores(kind, collapse):
    cfg = SMALL["c3s"]
    x = decode_inputs(cfg)
    K, q = dev_bf16(x["K"]), dev_bf16(x["q"])
    scale = oracle.f32(cfg.score_scale)
    if kind == "minmax":
        a, b_ = spa.block_minmax(K, cfg.block)
        s = spa.index_scores(spa.SPA_SCORE_MINMAX_BLOCK, q, a, b_, cfg.Hkv, collapse, scale)
    else:
        a, _ = spa.block_stats(K, cfg.block)
        s = spa.index_scores(spa.SPA_SCORE_MEAN_BLOCK, q, a, None, cfg.Hkv, collapse, scale)
    s = s.cpu().numpy()
    G = cfg.G
    for b in range(cfg.B):
        for g in range(cfg.Hkv):
            heads = x["q"][b, g * G:(g + 1) * G]
            if kind == "minmax":
                mn, mx = oracle.block_minmax(x["K"][b, g], cfg.block)
                ref = oracle.minmax_scores(heads, mn, mx, scale, False)
            else:
                mean, _ = oracle.block_stats(x["K"][b, g], cfg.block)
                ref = oracle.mean_scores(heads, mean, scale, False)
            got = s[b * cfg.Hkv + g] if collapse == spa.SPA_COLLAPSE_GROUP_MEAN else \
                s[b * cfg.Hq + g * G:b * cfg.Hq + (g + 1) * G]
            want = ref.mean(0) if collapse == spa.SPA_COLLAPSE_GROUP_MEAN else ref
            np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("kind", ["minmax", "mean"])
def test_decode_with_block_proxy_scores(kind):
    cfg = SMALL["c3s"].with_(score=kind)
    x = decode_inputs(cfg)
    K = dev_bf16(x["K"])
    if kind == "minmax":
        a, b_ = spa.block_minmax(K, cfg.block)
        score_kind = spa.SPA_SCORE_MINMAX_BLOCK
    else:
        a, b_ = spa.block_stats(K, cfg.block)
        b_ = None
        score_kind = spa.SPA_SCORE_MEAN_BLOCK
    plan = spa.decode(score_kind=score_kind, select_kind=spa.SPA_SELECT_TOPK, collapse=spa.SPA_COLLAPSE_GROUP_MEAN,
                      q=dev_bf16(x["q"]), K=K, V=dev_bf16(x["V"]), bmean=a, bvar=b_, block=cfg.block,
                      score_scale=oracle.f32(cfg.score_scale), sm_scale=oracle.f32(cfg.sm_scale), topk=cfg.topk,
                      sink=cfg.sink, window=cfg.window, cap=cfg.cap)
    torch.cuda.synchronize()
    assert spa.read_device_status(plan.ws) == 0
    idx, count = plan.idx.cpu().numpy(), plan.count.cpu().numpy()
    out = plan.out.view(torch.int16).cpu().numpy().view(np.uint16)
    out32 = plan.out_f32.cpu().numpy()
    G = cfg.G
    for u, (b, h) in enumerate(oracle.decode_units(cfg)):
        r = oracle.decode_unit(cfg, x, u)
        got = idx[u, :count[u]]
        d = compare_support(got, r["idx"], topk_band(r["ranked"], cfg.topk), f"{kind} unit {u}")
        if d == 0:
            heads = slice(h * G, (h + 1) * G)
            check_outputs(out[b, heads], out32[b, heads], r["out"], f"{kind} unit {u}")


# ---------------------------------------------------------------------------- bf16 statistics
def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("name,block", [("c3s", 64), ("c1s", 32)])
def test_block_stats_bf16(name, block):
    # minima and maxima are bf16 values: exact.  Means and variances are the fp32 values
    # rounded to nearest even; the oracle rounds its fp64 values directly, so an element may
    # land one bf16 step away where the fp32 value sits at a rounding midpoint's edge.
    cfg = SMALL[name]
    x = decode_inputs(cfg)
    K = dev_bf16(x["K"])
    mn, mx = spa.block_minmax(K, block, bf16=True)
    mean, var = spa.block_stats(K, block, bf16=True)
    mn, mx, mean, var = _bits(mn), _bits(mx), _bits(mean), _bits(var)
    off, total = 0, 0
    for b in range(cfg.B):
        for g in range(cfg.Hkv):
            rmn, rmx = oracle.block_minmax(x["K"][b, g], block)
            np.testing.assert_array_equal(mn[b, g], oracle.round_bf16(rmn))
            np.testing.assert_array_equal(mx[b, g], oracle.round_bf16(rmx))
            rmean, rvar = oracle.block_stats(x["K"][b, g], block)
            for got, ref in ((mean[b, g], oracle.round_bf16(rmean)), (var[b, g], oracle.round_bf16(rvar))):
                step = np.abs(got.astype(np.int32) - ref.astype(np.int32))
                assert step.max() <= 1
                off += int((step != 0).sum())
                total += step.size
    assert off <= max(2, total // 1000), f"{off} of {total} statistics one bf16 step away"


@pytest.mark.parametrize("kind", ["taylor", "minmax", "mean"])
def test_block_scores_read_bf16_statistics(kind):
    cfg = SMALL["c3s"]
    x = decode_inputs(cfg)
    q = dev_bf16(x["q"])
    scale = oracle.f32(cfg.score_scale)
    G = cfg.G
    st_a, st_b, refs = [], [], []
    for b in range(cfg.B):
        for g in range(cfg.Hkv):
            if kind == "minmax":
                a, c = oracle.block_minmax(x["K"][b, g], cfg.block)
            else:
                a, c = oracle.block_stats(x["K"][b, g], cfg.block)
            a16, c16 = oracle.round_bf16(a), oracle.round_bf16(c)
            st_a.append(a16)
            st_b.append(c16)
            heads = x["q"][b, g * G:(g + 1) * G]
            aw, cw = oracle.widen_bf16(a16), oracle.widen_bf16(c16)
            if kind == "taylor":
                refs.append(np.log(oracle.taylor_scores(heads, aw, cw, scale, True)))
            elif kind == "minmax":
                refs.append(oracle.minmax_scores(heads, aw, cw, scale, True))
            else:
                refs.append(oracle.mean_scores(heads, aw, scale, True))
    shape = (cfg.B, cfg.Hkv) + st_a[0].shape
    A = dev_bf16(np.stack(st_a).reshape(shape))
    C = dev_bf16(np.stack(st_b).reshape(shape))
    k = {"taylor": spa.SPA_SCORE_TAYLOR_BLOCK, "minmax": spa.SPA_SCORE_MINMAX_BLOCK,
         "mean": spa.SPA_SCORE_MEAN_BLOCK}[kind] | spa.SPA_STATS_BF16
    s = spa.index_scores(k, q, A, None if kind == "mean" else C, cfg.Hkv, spa.SPA_COLLAPSE_GROUP_MEAN, scale)
    np.testing.assert_allclose(s.cpu().numpy(), np.stack(refs), rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("kind", ["taylor", "mean"])
def test_decode_with_bf16_statistics(kind):
    # both sides score with the oracle's bf16 statistics (an input of the step)
    cfg = SMALL["c3s"].with_(score=kind, stats="bf16")
    x = decode_inputs(cfg)
    st_a, st_b = [], []
    for b in range(cfg.B):
        for g in range(cfg.Hkv):
            a, c = oracle.block_stats(x["K"][b, g], cfg.block)
            st_a.append(oracle.round_bf16(a))
            st_b.append(oracle.round_bf16(c))
    shape = (cfg.B, cfg.Hkv) + st_a[0].shape
    A = dev_bf16(np.stack(st_a).reshape(shape))
    C = dev_bf16(np.stack(st_b).reshape(shape)) if kind == "taylor" else None
    plan = spa.decode(score_kind=spa.SPA_SCORE_TAYLOR_BLOCK if kind == "taylor" else spa.SPA_SCORE_MEAN_BLOCK,
                      select_kind=spa.SPA_SELECT_TOPK, collapse=spa.SPA_COLLAPSE_GROUP_MEAN, q=dev_bf16(x["q"]),
                      K=dev_bf16(x["K"]), V=dev_bf16(x["V"]), bmean=A, bvar=C, block=cfg.block,
                      score_scale=oracle.f32(cfg.score_scale), sm_scale=oracle.f32(cfg.sm_scale), topk=cfg.topk,
                      sink=cfg.sink, window=cfg.window, cap=cfg.cap)
    torch.cuda.synchronize()
    assert spa.read_device_status(plan.ws) == 0
    idx, count = plan.idx.cpu().numpy(), plan.count.cpu().numpy()
    out = plan.out.view(torch.int16).cpu().numpy().view(np.uint16)
    out32 = plan.out_f32.cpu().numpy()
    G = cfg.G
    for u, (b, h) in enumerate(oracle.decode_units(cfg)):
        r = oracle.decode_unit(cfg, x, u)
        d = compare_support(idx[u, :count[u]], r["idx"], topk_band(r["ranked"], cfg.topk), f"bf16 {kind} unit {u}")
        if d == 0:
            heads = slice(h * G, (h + 1) * G)
            check_outputs(out[b, heads], out32[b, heads], r["out"], f"bf16 {kind} unit {u}")
