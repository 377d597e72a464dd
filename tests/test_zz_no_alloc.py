"""spa_select_topp_static -- top-p selection with its scratch in a fixed device array,
for callers that cannot allocate device memory when they call -- must give exactly the
results of spa_select_topp (same kernels, same inputs), call after call: the second call
runs on the array the first one left behind.  Collected last (file name) so that a run that
stops at its first failure has run every other test already."""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import long_context_sparse_spa_b200 as spa  # noqa: E402
from long_context_sparse_spa_b200 import _abi  # noqa: E402


def _scores(U, M, seed):
    rng = np.random.default_rng(seed)
    s = rng.standard_normal((U, M)).astype(np.float32)
    for u in range(U):
        s[u, rng.choice(M, 40, replace=False)] += 8.0
    return torch.from_numpy(s).cuda()


def _static_call(scores, p, sink, window, cap):
    """Direct C-ABI call of the entry point, outputs preallocated here."""
    U, M = scores.shape
    idx = torch.full((U, cap), -1, dtype=torch.int32, device="cuda")
    count = torch.zeros(U, dtype=torch.int32, device="cuda")
    mass = torch.zeros(U, dtype=torch.float32, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = spa.lib().spa_select_topp_static(scores.data_ptr(), None, U, M, ctypes.c_float(p), sink, window,
                                          idx.data_ptr(), count.data_ptr(), cap, mass.data_ptr(), st)
    assert rc == _abi.SPA_OK, spa.lib().spa_status_string(rc)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), count.cpu().numpy(), mass.cpu().numpy()


@pytest.mark.parametrize("U,M,p", [(16, 131072, 0.9), (3, 9001, 0.5)])
def test_static_matches_workspace_version_twice(U, M, p):
    for call, seed in enumerate((11, 12)):          # two calls in a row, different inputs
        s = _scores(U, M, seed + M)
        ref_idx, ref_cnt, ref_mass = (t.cpu().numpy() for t in spa.select_topp(s, p, 4, 128, cap=M))
        idx, cnt, mass = _static_call(s, p, 4, 128, M)
        np.testing.assert_array_equal(cnt, ref_cnt, err_msg=f"call {call}")
        for u in range(U):
            np.testing.assert_array_equal(idx[u, :cnt[u]], ref_idx[u, :ref_cnt[u]], err_msg=f"call {call} unit {u}")
        np.testing.assert_array_equal(mass, ref_mass, err_msg=f"call {call}")


def test_static_rejects_too_many_units():
    s = _scores(_abi.SPA_SELECT_STATIC_MAX_UNITS + 1, 1024, 1)
    U, M = s.shape
    out = torch.zeros((U, M), dtype=torch.int32, device="cuda")
    cnt = torch.zeros(U, dtype=torch.int32, device="cuda")
    rc = spa.lib().spa_select_topp_static(s.data_ptr(), None, U, M, ctypes.c_float(0.9), 0, 0, out.data_ptr(),
                                          cnt.data_ptr(), M, None, None)
    assert rc == _abi.SPA_ERR_UNSUPPORTED_SHAPE
