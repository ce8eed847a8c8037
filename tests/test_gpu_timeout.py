"""The bounded device-side wait gives up and reports QMM_ERR_TIMEOUT: a
diagnostic kernel waits, through the library's own mbarrier helpers, on a
barrier nothing arrives on (no copy in flight), and must return with the
status set; the GPU stays usable afterwards."""
import pytest
import torch

from weight_only_quantized_qmm_b200 import _lib, api
from weight_only_quantized_qmm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("spins", [1, 64, 4096])
def test_bounded_wait_gives_up_with_timeout_status(spins):
    res = torch.full((3,), -1, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    api.qmm_selftest_bounded_wait(spins, res, status)
    torch.cuda.synchronize()
    assert res.tolist() == [1, 0, 0]  # completed phase at once; pending and aborted waits give up
    assert int(status.item()) == _lib.QMM_ERR_TIMEOUT
    # the context is still usable: a real call right after it succeeds
    qw = api.qmm_quantize(wl.gen_weight(64, 256, 1).cuda(), 64, 4, torch.bfloat16)
    y = api.qmm_matmul(wl.gen_x(1, 256, 2).cuda(), qw)
    torch.cuda.synchronize()
    assert torch.isfinite(y).all()


def test_bounded_wait_argument_checks():
    L = _lib.load()
    res = torch.zeros(3, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert L.qmm_selftest_bounded_wait(0, res.data_ptr(), st.data_ptr(), None) == _lib.QMM_ERR_INVALID_ARG
    assert L.qmm_selftest_bounded_wait(1 << 23, res.data_ptr(), st.data_ptr(), None) == _lib.QMM_ERR_INVALID_ARG
    assert L.qmm_selftest_bounded_wait(8, None, st.data_ptr(), None) == _lib.QMM_ERR_ALIGNMENT
