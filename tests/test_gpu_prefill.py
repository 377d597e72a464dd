"""Selection-block-shared sparse prefill (spa_prefill_shared, tcgen05 attention) against
the fp64 oracle: supports per (query block, kv head) bit-exact up to logged score ties,
every output row within 2e-3 (fp32 output) and bf16 output = RNE(fp32 output)."""
import os
from concurrent.futures import ThreadPoolExecutor

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


def check_units(cfg, units, threads=None):
    """Every listed (query block, kv head) unit against the oracle (computed on a pool of host
    threads: the oracle's C code releases the GIL); tie differences are bounded."""
    x = prefill_inputs(cfg)
    idx, count, out, out32 = run_prefill(cfg, x)
    ties, worst = 0, 0.0
    G, bq = cfg.G, cfg.bq
    with ThreadPoolExecutor(threads or os.cpu_count() or 1) as ex:
        refs = list(ex.map(lambda jg: oracle.prefill_block(cfg, x, jg[0], jg[1], want_scores=True), units))
    for (j, g), (sup, ref, scores) in zip(units, refs):
        u = j * cfg.Hkv + g
        d = compare_support(idx[u, :count[u]], sup, topk_band(scores, cfg.topk), f"{cfg.name} unit {u}")
        ties += d
        if bq == 1:   # the query's own position follows its support
            assert idx[u, count[u]] == cfg.q_start + j, f"{cfg.name} unit {u}: own position"
        rows = slice(j * bq, (j + 1) * bq)
        heads = slice(g * G, (g + 1) * G)
        if d:
            # a logged tie moved a row: the output is compared on the GPU's own rows
            sel = idx[u, :count[u]]
            ref = np.stack([np.stack([oracle.sparse_attention(
                x["Q"][j * bq + i, g * G + hh][None], x["K"][g], x["V"][g],
                np.concatenate([sel, np.arange(cfg.q_start + j * bq, cfg.q_start + j * bq + i + 1)]).astype(np.int32),
                oracle.f32(cfg.sm_scale))[0][0] for hh in range(G)]) for i in range(bq)])
        worst = max(worst, check_outputs(out[rows, heads], out32[rows, heads], ref, f"{cfg.name} unit {u}"))
    assert ties <= max(2, len(units) // 50), f"{cfg.name}: {ties} tie differences in {len(units)} units"
    print(f"{cfg.name}: {len(units)} units, max|err| {worst:.2e}, tie differences {ties}")


def test_prefill_small_all_units():
    cfg = SMALL["c5s"]
    check_units(cfg, [(j, g) for j in range(cfg.n_blocks) for g in range(cfg.Hkv)])


@pytest.mark.parametrize("over", [dict(Hq=4, Hkv=2), dict(Hq=16, Hkv=2)], ids=["G2", "G8"])
def test_prefill_head_groups(over):
    # one and four pairs of query heads per unit (one CTA per pair)
    cfg = SMALL["c5s"].with_(N=2048, q_start=1536, T=256, topk=256, n_clusters=8, **over)
    check_units(cfg, [(j, g) for j in range(cfg.n_blocks) for g in range(cfg.Hkv)])


def test_prefill_budget_covers_everything():
    # top-k larger than every candidate set: supports are all of [0, t0); dense causal attention
    cfg = SMALL["c5s"].with_(N=2048, q_start=1024, T=512, topk=4096, n_clusters=8)
    check_units(cfg, [(j, g) for j in range(cfg.n_blocks) for g in range(cfg.Hkv)])


@pytest.mark.slow
def test_prefill_full_size_all_units():
    # all 64 query blocks x 8 kv heads of the full chunk, in the launch configuration the
    # bench times
    cfg = C5
    check_units(cfg, [(j, g) for j in range(cfg.n_blocks) for g in range(cfg.Hkv)])


# ------------------------------------------------------------------ per-query prefill (b_sel = 1)
PQ = SMALL["c5s"].with_(name="c5s_per_query", T=192, bq=1, topk=300)


def test_prefill_per_query_all_units():
    check_units(PQ, [(j, g) for j in range(PQ.T) for g in range(PQ.Hkv)])


def test_prefill_per_query_budget_covers_everything():
    # a budget above every candidate set: the support is all of [0, t): dense causal attention
    cfg = PQ.with_(N=1200, q_start=1000, T=64, topk=5000, n_clusters=4)
    check_units(cfg, [(j, g) for j in range(cfg.T) for g in range(cfg.Hkv)])
