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
