"""Device-side failure detection on the GPU, without a fault: a bounded
barrier wait that nothing completes runs out, records
CSA2_DEVERR_WAIT_TIMEOUT in the device error word and lets its kernel end,
and the context stays usable afterwards. (The bad-row path is covered by the
append and attention tests.)"""
import pytest
import torch

pytestmark = pytest.mark.gpu

CSA2_DEVERR_WAIT_TIMEOUT = 2


@pytest.fixture(scope="module")
def B():
    from sparse_fp4_kv_b200 import build
    build.build()
    from sparse_fp4_kv_b200 import binding
    return binding


def test_bounded_wait_runs_out_and_reports(B, cuda_device):
    torch.cuda.synchronize()
    assert B.csa2_device_status() == 0
    B.csa2_check_wait_timeout(20000)  # 20 ms
    assert B.csa2_device_status() == CSA2_DEVERR_WAIT_TIMEOUT
    # the word was cleared by the read, and the context still runs work
    assert B.csa2_device_status() == 0
    x = torch.arange(1024, device=cuda_device, dtype=torch.float32)
    assert float(x.sum().item()) == 1023 * 1024 / 2
