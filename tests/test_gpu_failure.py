"""Failure detection without a GPU fault: every wait inside the kernels is bounded, and when
its bound runs out the kernel raises SPA_ERR_TIMEOUT in the device status word and stays in a
defined state.  spa_test_stall arms a kernel's completion barrier for an arrival that is
never issued (nothing is left in flight), with a short bound, so the give-up path runs:

- the selection's chunk load: the status shows the timeout and the supports are still those
  of a normal run (the CTA falls back to reading its scores from global memory);
- the tcgen05 prefill's first MMA: the status shows the timeout, and the next normal call on
  the same context and workspace is correct (the CTA freed its tensor memory)."""
import numpy as np
import pytest

import oracle
from parity import check_outputs, dev_bf16
from synth import SMALL, decode_inputs, prefill_inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import long_context_sparse_spa_b200 as spa  # noqa: E402
from long_context_sparse_spa_b200 import _abi  # noqa: E402

TIMEOUT = 1 << _abi.SPA_ERR_TIMEOUT


class stalled:
    def __init__(self, bits):
        self.bits = bits

    def __enter__(self):
        assert spa.lib().spa_test_stall(self.bits) == _abi.SPA_OK

    def __exit__(self, *exc):
        spa.lib().spa_test_stall(0)


def _scores(U, M, seed):
    rng = np.random.default_rng(seed)
    s = rng.standard_normal((U, M)).astype(np.float32)
    for u in range(U):
        s[u, rng.choice(M, 50, replace=False)] += 7.0
    return torch.from_numpy(s).cuda()


def _select(s, p):
    U, M = s.shape
    idx = torch.full((U, M), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(U, dtype=torch.int32, device="cuda")
    mass = torch.zeros(U, dtype=torch.float32, device="cuda")
    ws = spa.workspace(spa.lib().spa_select_workspace_bytes(U, M))
    _abi.check(spa.lib().spa_select_topp(s.data_ptr(), None, U, M, _abi.ctypes.c_float(p), 4, 128, idx.data_ptr(),
                                         cnt.data_ptr(), M, mass.data_ptr(), ws.data_ptr(), ws.numel(), spa._stream()))
    torch.cuda.synchronize()
    return idx.cpu().numpy(), cnt.cpu().numpy(), mass.cpu().numpy(), spa.read_device_status(ws)


def test_selection_load_timeout_is_reported_and_results_stay_correct():
    s = _scores(4, 65536, 3)
    ref = _select(s, 0.9)
    assert ref[3] == 0
    with stalled(_abi.SPA_TEST_STALL_SELECT_LOAD):
        got = _select(s, 0.9)
    assert got[3] & TIMEOUT, "the stalled load did not raise SPA_ERR_TIMEOUT"
    np.testing.assert_array_equal(got[1], ref[1])
    for u in range(4):
        np.testing.assert_array_equal(got[0][u, :got[1][u]], ref[0][u, :ref[1][u]])
    np.testing.assert_array_equal(got[2], ref[2])
    assert _select(s, 0.9)[3] == 0     # hook off: a normal call again


def test_decode_with_stalled_selection_load():
    cfg = SMALL["c2s"]
    x = decode_inputs(cfg)

    def run():
        plan = spa.decode(score_kind=spa.SPA_SCORE_LOWRANK, select_kind=spa.SPA_SELECT_TOPP,
                          collapse=spa.SPA_COLLAPSE_GROUP_MEAN, q=dev_bf16(x["q"]), K=dev_bf16(x["K"]),
                          V=dev_bf16(x["V"]), q_idx=dev_bf16(x["q_idx"]), Kidx=dev_bf16(x["Kidx"]),
                          score_scale=oracle.f32(cfg.score_scale), sm_scale=oracle.f32(cfg.sm_scale),
                          topp=cfg.topp, sink=cfg.sink, window=cfg.window, cap=cfg.cap)
        torch.cuda.synchronize()
        return plan.idx.cpu().numpy(), plan.count.cpu().numpy(), plan.out_f32.cpu().numpy(), \
            spa.read_device_status(plan.ws)

    ref = run()
    with stalled(_abi.SPA_TEST_STALL_SELECT_LOAD):
        got = run()
    assert ref[3] == 0 and got[3] & TIMEOUT
    np.testing.assert_array_equal(got[1], ref[1])
    np.testing.assert_array_equal(got[0], ref[0])
    np.testing.assert_array_equal(got[2], ref[2])


def test_prefill_mma_timeout_is_reported_and_the_context_recovers():
    cfg = SMALL["c5s"].with_(N=2048, q_start=1024, T=256, topk=256, n_clusters=8)
    x = prefill_inputs(cfg)
    plan = spa.prefill(Q=dev_bf16(x["Q"]), q_idx=dev_bf16(x["q_idx"]), K=dev_bf16(x["K"]), V=dev_bf16(x["V"]),
                       Kidx=dev_bf16(x["Kidx"]), q_start=cfg.q_start, score_scale=oracle.f32(cfg.score_scale),
                       sm_scale=oracle.f32(cfg.sm_scale), topk=cfg.topk, sink=cfg.sink, run=False)
    with stalled(_abi.SPA_TEST_STALL_PREFILL_MMA):
        plan.run()
        torch.cuda.synchronize()
    assert spa.read_device_status(plan.ws, reset=True) & TIMEOUT
    plan.run()                          # the same workspace, hook off
    torch.cuda.synchronize()
    assert spa.read_device_status(plan.ws) == 0
    out = plan.out.view(torch.int16).cpu().numpy().view(np.uint16)
    out32 = plan.out_f32.cpu().numpy()
    G, bq = cfg.G, cfg.bq
    for j, g in ((0, 0), (cfg.n_blocks - 1, cfg.Hkv - 1)):
        _, ref = oracle.prefill_block(cfg, x, j, g)
        rows, heads = slice(j * bq, (j + 1) * bq), slice(g * G, (g + 1) * G)
        check_outputs(out[rows, heads], out32[rows, heads], ref, f"recovered unit {(j, g)}")
