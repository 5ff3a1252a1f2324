"""GPU tests of failure detection: the bounded waits of the kernels and the
device error word they report through (ssm_check_device_error).

Nothing here faults, traps or hangs the GPU. The failing wait is made on
purpose by ssm_selftest_bounded_wait: a kernel arms an mbarrier that can
never complete its phase and gives up after a short limit, exactly as the
kernels' ring waits do after ~2 s. The tests check that the error word
reports it, that the check clears it, and that the context stays usable (a
normal prefill afterwards still matches the oracle).
"""
import pytest
import torch

from parity_util import all_channels, compare, gather, oracle_prefill
from selective_state_space_depthwise_b200 import _lib, api
from selective_state_space_depthwise_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def small_prefill(seed=5):
    w = W.Workload("fail", batch=2, seqlen=130, d_inner=64, io_dtype=torch.bfloat16, seed=seed)
    inp = W.make_inputs(w, device="cuda")
    y, cc, st = api.prefill(inp["x"], inp["z"], inp["B"], inp["C"], inp["dt_raw"], inp)
    return w, inp, (y, cc, st)


def test_check_device_error_is_clean_after_normal_work():
    """The success path: after ordinary launches the word is clear."""
    small_prefill()
    api.check_device_error()  # raises if a wait gave up
    api.check_device_error()


def test_bounded_wait_gives_up_and_reports():
    """A wait that can never complete ends after its limit (1 ms here), the
    check reports SSM_ERR_DEVICE with the self-test's code and clears the word,
    and the next check is clean."""
    api.check_device_error()  # start clean
    api.selftest_bounded_wait(1_000_000)
    with pytest.raises(_lib.SsmError) as err:
        api.check_device_error()
    assert err.value.status == _lib.SSM_ERR_DEVICE
    assert f"code {_lib.SSM_SELFTEST_WAIT_CODE}" in str(err.value)
    api.check_device_error()  # cleared by the previous check


def test_context_usable_after_a_failed_wait():
    """After a wait gave up, ordinary work on the same stream still runs and
    matches the oracle, and the error word stays clear."""
    api.selftest_bounded_wait(2_000)
    with pytest.raises(_lib.SsmError):
        api.check_device_error()
    w, inp, out = small_prefill(seed=6)
    torch.cuda.synchronize()
    chans = all_channels(w.batch, w.d_inner)
    compare(w.io_dtype, gather(*out, chans), oracle_prefill(inp, chans), label="after a failed wait")
    api.check_device_error()


def test_selftest_rejects_out_of_range_limits():
    for bad in (0, 999, 2_000_000_001, -5):
        with pytest.raises(_lib.SsmError) as err:
            api.selftest_bounded_wait(bad)
        assert err.value.status == _lib.SSM_ERR_INVALID_ARG
