"""Fused decode (spa_decode: scores -> selection -> attention) against the fp64 oracle.

Small workloads compare every output; the full-size workloads compare every support and
every output too (the oracle's sparse path is cheap enough), run in the launch
configuration the bench times.  Captured mass and sparsity are reported per workload.
"""
import numpy as np
import pytest

import oracle
from parity import (MASS_TIE_REL, OUT_TOL, check_outputs, compare_support, dev, dev_bf16, topk_band, topp_band)
from synth import C1, C2, C2_128K, C3, C4, SMALL, decode_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import long_context_sparse_spa_b200 as spa  # noqa: E402


def run_gpu(cfg, x, local=None, rla=None):
    lowrank = cfg.score == "lowrank"
    kw = dict(
        score_kind=spa.SPA_SCORE_LOWRANK if lowrank else spa.SPA_SCORE_TAYLOR_BLOCK,
        select_kind=spa.SPA_SELECT_TOPK if cfg.select == "topk" else spa.SPA_SELECT_TOPP,
        collapse=spa.SPA_COLLAPSE_GROUP_MEAN if cfg.collapse == "group" else spa.SPA_COLLAPSE_NONE,
        q=dev_bf16(x["q"]), K=dev_bf16(x["K"]), V=dev_bf16(x["V"]), block=cfg.block,
        score_scale=oracle.f32(cfg.score_scale), sm_scale=oracle.f32(cfg.sm_scale),
        topk=cfg.topk, topp=cfg.topp, sink=cfg.sink, window=cfg.window, cap=cfg.cap)
    if lowrank:
        kw.update(q_idx=dev_bf16(x["q_idx"]), Kidx=dev_bf16(x["Kidx"]))
    else:
        mean, var = spa.block_stats(kw["K"], cfg.block)   # off the per-step path: once per filled block
        kw.update(bmean=mean, bvar=var)
    if local is not None:
        kw["local_units"] = torch.from_numpy(np.asarray(local, np.uint8)).cuda()
    if rla is not None:
        S, z = spa.rla_state(kw["K"], kw["V"])            # the state of all N rows, once
        kw.update(rla_state=S, rla_z=z, rla_gamma=torch.from_numpy(np.asarray(rla["gamma"], np.float32)).cuda(),
                  rla_eps=float(np.float32(rla["eps"])))
    plan = spa.decode(**kw)
    torch.cuda.synchronize()
    assert spa.read_device_status(plan.ws) == 0
    res = dict(idx=plan.idx.cpu().numpy(), count=plan.count.cpu().numpy(),
               out=plan.out.view(torch.int16).cpu().numpy().view(np.uint16), out32=plan.out_f32.cpu().numpy(),
               lse=plan.lse.cpu().numpy(),
               mass=plan.index_mass.cpu().numpy() if plan.index_mass is not None else None)
    del plan, kw
    torch.cuda.empty_cache()
    return res


def check_decode(cfg, report_mass=False):
    x = decode_inputs(cfg)
    g = run_gpu(cfg, x)
    G = cfg.G
    ties = 0
    worst = 0.0
    sparsity, captured = [], []
    for u, (b, h) in enumerate(oracle.decode_units(cfg)):
        r = oracle.decode_unit(cfg, x, u)   # the oracle computes its own (fp64) block statistics
        s = r["ranked"]
        band = topk_band(s, cfg.topk) if cfg.select == "topk" else topp_band(s, oracle.f32(cfg.topp))
        got = g["idx"][u, :g["count"][u]]
        d = compare_support(got, r["idx"], band, f"{cfg.name} unit {u}")
        ties += d
        heads = slice(h, h + 1) if cfg.collapse == "head" else slice(h * G, (h + 1) * G)
        if d == 0:
            ref_out, ref_lse = r["out"], r["lse"]
            if g["mass"] is not None:
                assert abs(g["mass"][u] - r["index_mass"]) <= 4 * MASS_TIE_REL + 1e-6
        else:
            # a support that differs only inside the tie band: the output is checked against the
            # oracle's attention over the GPU's own support
            ref_out, ref_lse = oracle.sparse_attention(x["q"][b, heads], x["K"][b, r["g"]], x["V"][b, r["g"]],
                                                       got, oracle.f32(cfg.sm_scale), cfg.block)
            print(f"{cfg.name} unit {u}: {d} tie differences; output compared on the GPU's support")
        worst = max(worst, check_outputs(g["out"][b, heads], g["out32"][b, heads], ref_out, f"{cfg.name} unit {u}"))
        np.testing.assert_allclose(g["lse"][b, heads], ref_lse, rtol=2e-6, atol=2e-6)
        sparsity.append(1 - got.size / cfg.M)
        if report_mass and u < 4:
            captured.append(oracle.captured_mass(cfg, x, u, got))
    msg = f"{cfg.name}: max|err| {worst:.2e}, tie differences {ties}, sparsity mean {np.mean(sparsity):.4f}"
    # every run so far had none; a regression that turns many positions into "ties" fails here
    assert ties <= max(4, cfg.U // 4), f"{cfg.name}: {ties} tie differences in {cfg.U} units"
    if captured:
        msg += f", captured mass (first units) {np.round(captured, 4).tolist()}"
    print(msg)
    return worst


@pytest.mark.parametrize("name", ["c1s", "c2s", "c3s", "c4s"])
def test_decode_small(name):
    check_decode(SMALL[name])


def test_decode_c1():
    check_decode(C1, report_mass=True)


@pytest.mark.slow
@pytest.mark.parametrize("cfg", [C2, C2_128K, C3, C4], ids=lambda c: c.name)
def test_decode_full_size(cfg):
    check_decode(cfg, report_mass=True)


@pytest.mark.parametrize("name", ["c1s", "c2s", "c3s"])
def test_decode_routed(name):
    """Head-wise routing: every other unit is local (support = sink + window, exactly), the
    others run the sparse selection; every unit is compared with the oracle's routed path."""
    cfg = SMALL[name]
    x = decode_inputs(cfg)
    local = np.array([u % 2 for u in range(cfg.U)], np.uint8)
    g = run_gpu(cfg, x, local=local)
    G = cfg.G
    for u, (b, h) in enumerate(oracle.decode_units(cfg)):
        r = oracle.decode_unit(cfg, x, u, local=bool(local[u]))
        got = g["idx"][u, :g["count"][u]]
        if local[u]:
            np.testing.assert_array_equal(got, r["idx"])
            d = 0
        else:
            s = r["ranked"]
            band = topk_band(s, cfg.topk) if cfg.select == "topk" else topp_band(s, oracle.f32(cfg.topp))
            d = compare_support(got, r["idx"], band, f"{cfg.name} unit {u}")
        if d == 0:
            heads = slice(h, h + 1) if cfg.collapse == "head" else slice(h * G, (h + 1) * G)
            check_outputs(g["out"][b, heads], g["out32"][b, heads], r["out"], f"{cfg.name} routed unit {u}")
            np.testing.assert_allclose(g["lse"][b, heads], r["lse"], rtol=2e-6, atol=2e-6)
            if g["mass"] is not None and not local[u]:
                assert abs(g["mass"][u] - r["index_mass"]) <= 4 * MASS_TIE_REL + 1e-6


def _rla_params(cfg, seed=7):
    rng = np.random.default_rng(seed)
    return {"gamma": rng.uniform(0.5, 1.5, (cfg.Hq, cfg.d)).astype(np.float32), "eps": 1e-6}


def check_decode_rla(cfg, local=None, units=None):
    """Residual linear attention ("SPLA", sections 2.2-2.3): supports as without it, outputs
    = exact + RMSNorm(RLA over the left-out rows), compared with the oracle's direct form."""
    x = decode_inputs(cfg)
    rla = _rla_params(cfg)
    g = run_gpu(cfg, x, local=local, rla=rla)
    G = cfg.G
    worst, ties = 0.0, 0
    all_units = oracle.decode_units(cfg)
    for u in (range(cfg.U) if units is None else units):
        b, h = all_units[u]
        loc = bool(local[u]) if local is not None else False
        r = oracle.decode_unit(cfg, x, u, local=loc, rla=rla)
        got = g["idx"][u, :g["count"][u]]
        if loc:
            np.testing.assert_array_equal(got, r["idx"])
            d = 0
        else:
            s = r["ranked"]
            band = topk_band(s, cfg.topk) if cfg.select == "topk" else topp_band(s, oracle.f32(cfg.topp))
            d = compare_support(got, r["idx"], band, f"{cfg.name} unit {u}")
        ties += d
        if d == 0:
            heads = slice(h, h + 1) if cfg.collapse == "head" else slice(h * G, (h + 1) * G)
            worst = max(worst, check_outputs(g["out"][b, heads], g["out32"][b, heads], r["out"],
                                             f"{cfg.name} RLA unit {u}"))
            np.testing.assert_allclose(g["lse"][b, heads], r["lse"], rtol=2e-6, atol=2e-6)
    assert ties <= max(4, cfg.U // 4), f"{cfg.name} RLA: {ties} tie differences in {cfg.U} units"
    print(f"{cfg.name} RLA: max|err| {worst:.2e}, tie differences {ties}")


@pytest.mark.parametrize("name", ["c1s", "c2s", "c3s"])
def test_decode_rla(name):
    check_decode_rla(SMALL[name])


def test_decode_rla_routed():
    cfg = SMALL["c2s"]
    check_decode_rla(cfg, local=np.array([u % 2 for u in range(cfg.U)], np.uint8))


def test_decode_rla_empty_and_full_supports():
    # k = 0 with no sink or window: every support is empty, the output is the RLA of all rows;
    # k >= M: the support is every row, RLA contributes nothing
    check_decode_rla(SMALL["c1s"].with_(topk=0, sink=0, window=0))
    check_decode_rla(SMALL["c1s"].with_(N=700, topk=800))


def test_decode_rla_full_size_c3():
    # the bench's launch configuration at full size; the oracle's direct RLA reads all 131072
    # rows per head, so three units (first, middle, last) are compared
    check_decode_rla(C3, units=[0, C3.U // 2 + 3, C3.U - 1])
