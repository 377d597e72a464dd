"""Permuted block-sparse prefill (spa_pbs_prefill, PBS-Attn) against the fp64 oracle.

- importance: within fp32 accumulation error of the oracle's fp64 mean causal softmax;
- permutation: exactly the oracle's in-segment order of the GPU's own importances (integer
  work: the same input values must give the same order);
- kept key blocks: the oracle's top-k of fp64 block scores over the GPU's permutation, up to
  blocks whose score lies within the fp32 error band of the k-th score (counted, bounded);
- support: the kept blocks' original positions, ascending;
- output: within 2e-3 of the oracle (fp32 output), bf16 output = RNE(fp32 output)."""
from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np
import pytest

import oracle
from parity import check_outputs, dev_bf16
from synth import PBS_SMALL, bf16_value, pbs_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import long_context_sparse_spa_b200 as spa  # noqa: E402

BLOCK_TIE_REL = 1e-5   # fp32 means of 64 keys and a 128-term dot product


def _block_scores(cfg, x, perm, j, g):
    """fp64 block scores sm_scale * qbar . kbar over the permuted blocks before j's segment."""
    b, G = cfg.b, cfg.G
    t0 = j * b
    nc = t0 // cfg.S * cfg.S // b
    qbar = bf16_value(x["Q"][t0:t0 + b, g * G:(g + 1) * G]).astype(np.float64).reshape(-1, cfg.d).mean(0)
    Kp = bf16_value(x["K"][g][perm[:nc * b]]).astype(np.float64).reshape(nc, b, cfg.d).mean(1)
    return oracle.f32(cfg.sm_scale) * (Kp @ qbar)


def run(cfg):
    x = pbs_inputs(cfg)
    plan = spa.pbs_prefill(Q=dev_bf16(x["Q"]), K=dev_bf16(x["K"]), V=dev_bf16(x["V"]),
                           sm_scale=oracle.f32(cfg.sm_scale), S=cfg.S, topk=cfg.topk, b=cfg.b)
    torch.cuda.synchronize()
    assert spa.read_device_status(plan.ws) == 0
    g = dict(imp=plan.importance.cpu().numpy(), perm=plan.perm.cpu().numpy(), idx=plan.idx.cpu().numpy(),
             count=plan.count.cpu().numpy(), out=plan.out.view(torch.int16).cpu().numpy().view(np.uint16),
             out32=plan.out_f32.cpu().numpy())
    return x, g


def check(cfg, blocks=None):
    x, r = run(cfg)
    b, G, T, S = cfg.b, cfg.G, cfg.T, cfg.S
    sm = oracle.f32(cfg.sm_scale)
    for g in range(cfg.Hkv):
        ref_imp = oracle.pbs_importance(x["Q"][T - b:, g * G:(g + 1) * G], T - b, x["K"][g], sm)
        np.testing.assert_allclose(r["imp"][g], ref_imp, rtol=2e-4, atol=1e-9)
        np.testing.assert_array_equal(r["perm"][g], oracle.pbs_permutation(r["imp"][g].astype(np.float64), S))
    units = [(j, g) for j in (blocks if blocks is not None else range(cfg.n_blocks)) for g in range(cfg.Hkv)]
    with ThreadPoolExecutor(os.cpu_count() or 1) as ex:
        refs = list(ex.map(lambda jg: oracle.pbs_prefill_unit(
            x["Q"][jg[0] * b:(jg[0] + 1) * b, jg[1] * G:(jg[1] + 1) * G], jg[0] * b, x["K"][jg[1]], x["V"][jg[1]],
            r["perm"][jg[1]], S, cfg.topk, sm), units))
    ties, worst = 0, 0.0
    for (j, g), (sup, ref) in zip(units, refs):
        u = j * cfg.Hkv + g
        t0, seg0 = j * b, j * b // S * S
        got = r["idx"][u, :r["count"][u]]
        assert np.all(np.diff(got) > 0), f"unit {u}: support not ascending"
        pinv = np.empty(T, np.int64)
        pinv[r["perm"][g]] = np.arange(T)
        got_blocks = set((pinv[got] // b).tolist())
        ref_blocks = set((pinv[sup] // b).tolist())
        assert r["count"][u] == len(got_blocks) * b
        diff = got_blocks ^ ref_blocks
        if diff:
            s = _block_scores(cfg, x, r["perm"][g], j, g)
            order = np.lexsort((np.arange(s.size), -s))
            tau = s[order[cfg.topk - 1]]
            band = set(np.nonzero(np.abs(s - tau) <= BLOCK_TIE_REL * max(1.0, abs(tau)))[0].tolist())
            assert diff <= band, f"unit {u}: blocks {sorted(diff - band)} differ outside the tie band"
            ties += len(diff)
            # output on the GPU's own rows
            rows_base = np.concatenate([got, np.arange(seg0, t0)]).astype(np.int32)
            ref = np.stack([np.stack([oracle.sparse_attention(
                x["Q"][t0 + i, g * G + hh][None], x["K"][g], x["V"][g],
                np.concatenate([rows_base, np.arange(t0, t0 + i + 1)]).astype(np.int32), sm)[0][0]
                for hh in range(G)]) for i in range(b)])
        else:
            np.testing.assert_array_equal(got, sup)
        rows, heads = slice(t0, t0 + b), slice(g * G, (g + 1) * G)
        worst = max(worst, check_outputs(r["out"][rows, heads], r["out32"][rows, heads], ref, f"pbs unit {u}"))
    assert ties <= max(2, len(units) // 20), f"{ties} block tie differences in {len(units)} units"
    print(f"{cfg.name}: {len(units)} units, max|err| {worst:.2e}, block tie differences {ties}")


def test_pbs_small_all_units():
    check(PBS_SMALL)


@pytest.mark.parametrize("over", [dict(topk=0), dict(topk=40), dict(S=64, topk=3), dict(S=192, Hq=16, Hkv=2),
                                  dict(Hq=4, Hkv=2), dict(Hq=12, Hkv=2, T=768)],
                         ids=["no_blocks", "all_blocks", "segment_eq_2_blocks", "ragged_last_segment_G8", "G2", "G6"])
def test_pbs_variants(over):
    check(PBS_SMALL.with_(**over))
