"""spa_select_topp_static -- top-p selection whose scratch is a fixed device array inside the
library, for callers that cannot allocate device memory when they call (an inference server
that reserves all device memory at start-up, a plug-in whose host framework owns every
buffer).

Checked call after call (the second call runs on the array the first one left behind):
  - it gives exactly the results of spa_select_topp (same kernels, same inputs);
  - its supports and index masses match the fp64 oracle's top-p, up to the logged tie band;
  - a ragged call (per-unit lengths) matches the oracle on each unit's prefix;
  - a capacity smaller than a support shows as count > cap and as SPA_ERR_CAPACITY in the
    array's status word, read back with spa_select_static_status.
Collected last (file name) so that a run that stops at its first failure has run every
other test already."""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import long_context_sparse_spa_b200 as spa  # noqa: E402
import oracle  # noqa: E402
from long_context_sparse_spa_b200 import _abi  # noqa: E402
from parity import MASS_TIE_REL, compare_support, topp_band  # noqa: E402


def _scores(U, M, seed):
    rng = np.random.default_rng(seed)
    s = rng.standard_normal((U, M)).astype(np.float32)
    for u in range(U):
        s[u, rng.choice(M, 40, replace=False)] += 8.0
    return torch.from_numpy(s).cuda()


def _static_call(scores, p, sink, window, cap, unit_len=None):
    """Direct C-ABI call of the entry point, outputs preallocated here."""
    U, M = scores.shape
    idx = torch.full((U, max(cap, 1)), -1, dtype=torch.int32, device="cuda")
    count = torch.zeros(U, dtype=torch.int32, device="cuda")
    mass = torch.zeros(U, dtype=torch.float32, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ul = None if unit_len is None else unit_len.data_ptr()
    rc = spa.lib().spa_select_topp_static(scores.data_ptr(), ul, U, M, ctypes.c_float(p), sink, window,
                                          idx.data_ptr(), count.data_ptr(), cap, mass.data_ptr(), st)
    assert rc == _abi.SPA_OK, spa.lib().spa_status_string(rc)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), count.cpu().numpy(), mass.cpu().numpy()


def _status(reset=True):
    bits = ctypes.c_uint32(0)
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert spa.lib().spa_select_static_status(st, ctypes.byref(bits), int(reset)) == _abi.SPA_OK
    return bits.value


def _vs_oracle(s_np, idx, cnt, mass, p, sink, window, lens=None):
    for u in range(s_np.shape[0]):
        L = s_np.shape[1] if lens is None else int(lens[u])
        row = s_np[u, :L].astype(np.float64)
        ref, ref_mass, _ = oracle.select_topp(row, oracle.f32(p), sink, window)
        band = topp_band(row, oracle.f32(p))
        compare_support(idx[u, :cnt[u]], ref, band, f"static unit {u}")
        assert abs(float(mass[u]) - ref_mass) <= 4 * MASS_TIE_REL + 1e-6, (u, float(mass[u]), ref_mass)


@pytest.mark.parametrize("U,M,p", [(16, 131072, 0.9), (3, 9001, 0.5)])
def test_static_matches_workspace_version_and_oracle_twice(U, M, p):
    for call, seed in enumerate((11, 12)):          # two calls in a row, different inputs
        s = _scores(U, M, seed + M)
        ref_idx, ref_cnt, ref_mass = (t.cpu().numpy() for t in spa.select_topp(s, p, 4, 128, cap=M))
        idx, cnt, mass = _static_call(s, p, 4, 128, M)
        assert _status() == 0, f"call {call}: status raised"
        np.testing.assert_array_equal(cnt, ref_cnt, err_msg=f"call {call}")
        for u in range(U):
            np.testing.assert_array_equal(idx[u, :cnt[u]], ref_idx[u, :ref_cnt[u]], err_msg=f"call {call} unit {u}")
        np.testing.assert_array_equal(mass, ref_mass, err_msg=f"call {call}")
        _vs_oracle(s.cpu().numpy(), idx, cnt, mass, p, 4, 128)


def test_static_ragged_units_match_oracle():
    U, M, p = 5, 20000, 0.8
    s = _scores(U, M, 77)
    lens = np.array([20000, 1, 0, 12345, 4097], np.int32)
    for _ in range(2):
        idx, cnt, mass = _static_call(s, p, 4, 64, M, unit_len=torch.from_numpy(lens).cuda())
        assert _status() == 0
        assert cnt[2] == 0
        s_np = s.cpu().numpy()
        for u in range(U):
            if lens[u] == 0:
                continue
            _vs_oracle(s_np[u:u + 1], idx[u:u + 1], cnt[u:u + 1], mass[u:u + 1], p, 4, 64, lens=lens[u:u + 1])


def test_static_capacity_flag():
    U, M, p = 2, 50000, 0.95
    s = _scores(U, M, 5)
    cap = 64
    idx, cnt, _ = _static_call(s, p, 4, 128, cap)
    assert np.all(cnt > cap)
    assert _status(reset=True) & (1 << _abi.SPA_ERR_CAPACITY)
    assert _status() == 0      # cleared by the reset
    # the written prefix is the support's first cap entries
    full, fcnt, _ = _static_call(s, p, 4, 128, M)
    np.testing.assert_array_equal(fcnt, cnt)
    for u in range(U):
        np.testing.assert_array_equal(idx[u, :cap], full[u, :cap])


def test_static_rejects_too_many_units():
    s = _scores(_abi.SPA_SELECT_STATIC_MAX_UNITS + 1, 1024, 1)
    U, M = s.shape
    out = torch.zeros((U, M), dtype=torch.int32, device="cuda")
    cnt = torch.zeros(U, dtype=torch.int32, device="cuda")
    rc = spa.lib().spa_select_topp_static(s.data_ptr(), None, U, M, ctypes.c_float(0.9), 0, 0, out.data_ptr(),
                                          cnt.data_ptr(), M, None, None)
    assert rc == _abi.SPA_ERR_UNSUPPORTED_SHAPE
