"""Failure reporting of the bounded device-side waits, exercised on the GPU
without any fault: a wait on a barrier that nothing completes gives up after
~1 ms, the kernel returns, and the host reads SSM_ERR_TIMEOUT."""
import pytest
import torch

from selective_state_space_50_b200 import ssm_scan

from test_gpu_parity import check_fwd, small_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssm_scan.load_library()


def test_wait_timeout_is_reported_then_cleared_and_the_context_survives():
    lib = ssm_scan.load_library()
    ssm_scan.device_error_status()                       # start from a clear word
    st = lib.ssm_selftest_wait_timeout(ssm_scan._stream_ptr(None))
    assert st == ssm_scan.SSM_OK, ssm_scan.last_error()
    with pytest.raises(ssm_scan.SSMError) as e:
        ssm_scan.device_error_status()
    assert e.value.status == ssm_scan.SSM_ERR_TIMEOUT
    ssm_scan.device_error_status()                       # the word was cleared
    # the context is still usable: a forward on the TMA path matches the oracle
    check_fwd(small_workload(2, 2400, 72, 16, "bf16", True, True, True, True, "neg_lognormal"))
    ssm_scan.device_error_status()


def test_planned_name_reports_the_same_timeout():
    """ssm_check_device_errors (the boundary's planned name) reports and clears
    the word exactly as ssm_device_error_status does."""
    lib = ssm_scan.load_library()
    stream = ssm_scan._stream_ptr(None)
    assert lib.ssm_check_device_errors(stream) == ssm_scan.SSM_OK
    assert lib.ssm_selftest_wait_timeout(stream) == ssm_scan.SSM_OK
    assert lib.ssm_check_device_errors(stream) == ssm_scan.SSM_ERR_TIMEOUT
    assert lib.ssm_check_device_errors(stream) == ssm_scan.SSM_OK
