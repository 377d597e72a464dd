"""The persistent dataflow decode (spa_decode's fused path for low-rank, head-collapsed
units) against the fp64 oracle and against the separate-kernel path on the same inputs.

Supports must be identical on both paths (the selection is exact integer work) and match the
oracle up to the logged tie band; outputs must be within the acceptance tolerance of the
oracle on the GPU's support.  Ragged cache lengths, top-k and top-p, the degenerate
selections (k >= N, k = 0, p = 1), a capacity below the support and several calls in a row
(the kernel resets its own counters) are covered."""
import numpy as np
import pytest

import oracle
from parity import check_outputs, compare_support, dev_bf16, topk_band, topp_band
from synth import C2, SMALL, decode_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import long_context_sparse_spa_b200 as spa  # noqa: E402
from long_context_sparse_spa_b200 import _abi  # noqa: E402

# fused-eligible reduced workloads (N >= 16384), ragged lengths
C2M = C2.with_(name="c2m", B=2, Hq=16, Hkv=2, N=20011, n_clusters=8)
C2M_TOPK = C2M.with_(name="c2m_topk", select="topk", topk=700, topp=0.0)
C2M_G4 = C2.with_(name="c2m_g4", B=3, Hq=12, Hkv=3, N=16417, n_clusters=6)


def _plan(cfg, x, path, **over):
    kw = dict(score_kind=spa.SPA_SCORE_LOWRANK,
              select_kind=spa.SPA_SELECT_TOPK if cfg.select == "topk" else spa.SPA_SELECT_TOPP,
              collapse=spa.SPA_COLLAPSE_GROUP_MEAN, q=dev_bf16(x["q"]), K=dev_bf16(x["K"]), V=dev_bf16(x["V"]),
              q_idx=dev_bf16(x["q_idx"]), Kidx=dev_bf16(x["Kidx"]), score_scale=oracle.f32(cfg.score_scale),
              sm_scale=oracle.f32(cfg.sm_scale), topk=cfg.topk, topp=cfg.topp, sink=cfg.sink, window=cfg.window,
              cap=cfg.cap, kernel_path=path, run=False)
    kw.update(over)
    return spa.decode(**kw)


def _result(plan):
    torch.cuda.synchronize()
    return dict(idx=plan.idx.cpu().numpy(), count=plan.count.cpu().numpy(),
                out=plan.out.view(torch.int16).cpu().numpy().view(np.uint16), out32=plan.out_f32.cpu().numpy(),
                lse=plan.lse.cpu().numpy(),
                mass=None if plan.index_mass is None else plan.index_mass.cpu().numpy())


def _check_vs_oracle(cfg, x, g, what):
    ties = 0
    for u, (b, h) in enumerate(oracle.decode_units(cfg)):
        r = oracle.decode_unit(cfg, x, u)
        s = r["ranked"]
        band = topk_band(s, cfg.topk) if cfg.select == "topk" else topp_band(s, oracle.f32(cfg.topp))
        got = g["idx"][u, :g["count"][u]]
        d = compare_support(got, r["idx"], band, f"{what} unit {u}")
        ties += d
        heads = slice(h * cfg.G, (h + 1) * cfg.G)
        if d == 0:
            check_outputs(g["out"][b, heads], g["out32"][b, heads], r["out"], f"{what} unit {u}")
            np.testing.assert_allclose(g["lse"][b, heads], r["lse"], rtol=2e-6, atol=2e-6)
        else:
            # the GPU's support differs by logged ties: compare the output on the GPU's support
            ref, _ = oracle.sparse_attention(x["q"][b, heads], x["K"][b, h], x["V"][b, h], got,
                                             oracle.f32(cfg.sm_scale))
            check_outputs(g["out"][b, heads], g["out32"][b, heads], ref, f"{what} unit {u} (GPU support)")
    assert ties <= 2 * cfg.U, f"{what}: {ties} tie differences"
    return ties


@pytest.mark.parametrize("cfg", [SMALL["c4s"], C2M, C2M_TOPK, C2M_G4], ids=lambda c: c.name)
def test_fused_vs_oracle_and_separate(cfg):
    x = decode_inputs(cfg)
    fused = _plan(cfg, x, spa.SPA_DECODE_FUSED)
    sep = _plan(cfg, x, spa.SPA_DECODE_SEPARATE)
    for call in range(3):       # the fused kernel resets its counters: every call must agree
        fused.run()
        sep.run()
        gf, gs = _result(fused), _result(sep)
        assert spa.read_device_status(fused.ws) == 0 and spa.read_device_status(sep.ws) == 0
        np.testing.assert_array_equal(gf["count"], gs["count"], err_msg=f"call {call}")
        for u in range(cfg.U):
            np.testing.assert_array_equal(gf["idx"][u, :gf["count"][u]], gs["idx"][u, :gs["count"][u]],
                                          err_msg=f"call {call} unit {u}")
        if gf["mass"] is not None:
            np.testing.assert_array_equal(gf["mass"], gs["mass"])
        np.testing.assert_allclose(gf["out32"], gs["out32"], rtol=0, atol=2e-5)
        if call == 0:
            ties = _check_vs_oracle(cfg, x, gf, cfg.name)
            print(f"{cfg.name}: supports {gf['count'].tolist()}, tie differences {ties}")


@pytest.mark.parametrize("over", [dict(topk=10 ** 6), dict(topk=0), dict(topp=1.0), dict(topp=1e-6)],
                         ids=["k_ge_N", "k0", "p1", "p_tiny"])
def test_fused_degenerate_selections(over):
    cfg = C2M_TOPK if "topk" in over else C2M
    cfg = cfg.with_(**over)
    x = decode_inputs(cfg)
    plan = _plan(cfg, x, spa.SPA_DECODE_FUSED, cap=cfg.N)
    plan.run()
    g = _result(plan)
    assert spa.read_device_status(plan.ws) == 0
    ref = _plan(cfg, x, spa.SPA_DECODE_SEPARATE, cap=cfg.N)
    ref.run()
    r = _result(ref)
    np.testing.assert_array_equal(g["count"], r["count"])
    for u in range(cfg.U):
        np.testing.assert_array_equal(g["idx"][u, :g["count"][u]], r["idx"][u, :r["count"][u]])
    np.testing.assert_allclose(g["out32"], r["out32"], rtol=0, atol=2e-5)
    if over.get("topk") == 0:
        forced = oracle.local_support(cfg.N, cfg.sink, cfg.window)
        for u in range(cfg.U):
            np.testing.assert_array_equal(g["idx"][u, :g["count"][u]], forced)
    if over.get("topk", 0) >= cfg.N:
        assert np.all(g["count"] == cfg.N)


def test_fused_capacity_flag():
    cfg = C2M
    x = decode_inputs(cfg)
    full = _plan(cfg, x, spa.SPA_DECODE_FUSED)
    full.run()
    gf = _result(full)
    cap = int(gf["count"].min()) - 20      # below every support
    assert cap > 0 and np.all(gf["count"] > cap)
    plan = _plan(cfg, x, spa.SPA_DECODE_FUSED, cap=cap)
    plan.run()
    g = _result(plan)
    assert spa.read_device_status(plan.ws) & (1 << _abi.SPA_ERR_CAPACITY)
    np.testing.assert_array_equal(g["count"], gf["count"])
    for u in range(cfg.U):
        np.testing.assert_array_equal(g["idx"][u, :cap], gf["idx"][u, :cap])
    # the output is attention over the first cap rows of each support
    for u, (b, h) in enumerate(oracle.decode_units(cfg)):
        heads = slice(h * cfg.G, (h + 1) * cfg.G)
        ref, _ = oracle.sparse_attention(x["q"][b, heads], x["K"][b, h], x["V"][b, h], g["idx"][u, :cap],
                                         oracle.f32(cfg.sm_scale))
        check_outputs(g["out"][b, heads], g["out32"][b, heads], ref, f"capped unit {u}")
