"""Failure detection on the GPU without a fault (GPU).

Every wait inside the library's kernels is bounded: after its limit it raises
VA_STATUS_WAIT_TIMEOUT in the device status word, the kernel drains what it
started and returns.  The self-test entry point runs that exact wait on a
barrier phase nothing completes; this checks that the wait gives up, that the
host sees the status bit, and that the context is still usable: a forward
pass right after it matches the oracle.
"""
import pytest
import torch

from variable_length_flash_varlen_b200 import binding, workloads
from tests._helpers import compare, oracle_all, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    binding.load()


def test_bounded_wait_gives_up_and_reports(oracle_lib):
    binding.device_status(clear=True)
    assert binding.selftest_wait_timeout() == 1
    st = binding.device_status(clear=True)
    assert st & binding.VA_STATUS_WAIT_TIMEOUT, st
    assert binding.device_status(clear=True) == 0  # cleared
    wl = workloads.named("worked_example")
    q, k, v = workloads.make_qkv(wl)
    out, lse = run_gpu(wl, q, k, v)
    compare(out, lse, *oracle_all(oracle_lib, wl, q, k, v))
    assert binding.device_status(clear=True) == 0


def test_selftest_rejects_null_pointer():
    with pytest.raises(binding.VarlenAttentionError):
        binding._check(binding.load().varlen_attention_selftest_wait_timeout(None, None))
