"""Selection-block-shared sparse prefill (spa_prefill_shared, tcgen05 attention) against
the fp64 oracle: supports per (query block, kv head) bit-exact up to logged score ties,
every output row within 2e-3 (fp32 output) and bf16 output = RNE(fp32 output)."""
import numpy as np
import pytest

import oracle
from parity import check_outputs, compare_support, dev_bf16, topk_band
from synth import C5, SMALL, prefill_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import long_context_sparse_spa_b200 as spa  # noqa: E402


def run_prefill(cfg, x):
    plan = spa.prefill(Q=dev_bf16(x["Q"]), q_idx=dev_bf16(x["q_idx"]), K=dev_bf16(x["K"]), V=dev_bf16(x["V"]),
                       Kidx=dev_bf16(x["Kidx"]), q_start=cfg.q_start, score_scale=oracle.f32(cfg.score_scale),
                       sm_scale=oracle.f32(cfg.sm_scale), topk=cfg.topk, sink=cfg.sink, bq=cfg.bq)
    torch.cuda.synchronize()
    assert spa.read_device_status(plan.ws) == 0
    return (plan.idx.cpu().numpy(), plan.count.cpu().numpy(),
            plan.out.view(torch.int16).cpu().numpy().view(np.uint16), plan.out_f32.cpu().numpy())


def check_units(cfg, units):
    x = prefill_inputs(cfg)
    idx, count, out, out32 = run_prefill(cfg, x)
    ties, worst = 0, 0.0
    G, bq = cfg.G, cfg.bq
    for j, g in units:
        u = j * cfg.Hkv + g
        sup, ref, scores = oracle.prefill_block(cfg, x, j, g, want_scores=True)
        d = compare_support(idx[u, :count[u]], sup, topk_band(scores, cfg.topk), f"{cfg.name} unit {u}")
        ties += d
        if d == 0:
            rows = slice(j * bq, (j + 1) * bq)
            heads = slice(g * G, (g + 1) * G)
            worst = max(worst, check_outputs(out[rows, heads], out32[rows, heads], ref, f"{cfg.name} unit {u}"))
    print(f"{cfg.name}: {len(units)} units, max|err| {worst:.2e}, tie differences {ties}")


def test_prefill_small_all_units():
    cfg = SMALL["c5s"]
    check_units(cfg, [(j, g) for j in range(cfg.n_blocks) for g in range(cfg.Hkv)])


def test_prefill_budget_covers_everything():
    # top-k larger than every candidate set: supports are all of [0, t0); dense causal attention
    cfg = SMALL["c5s"].with_(N=2048, q_start=1024, T=512, topk=4096, n_clusters=8)
    check_units(cfg, [(j, g) for j in range(cfg.n_blocks) for g in range(cfg.Hkv)])


@pytest.mark.slow
def test_prefill_full_size_sampled():
    cfg = C5
    check_units(cfg, [(0, 0), (13, 3), (31, 5), (47, 1), (63, 7), (63, 0)])
