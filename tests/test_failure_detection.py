"""Failure detection on the GPU without a fault (GPU).

Every wait inside the library's kernels is bounded: after its limit it raises
VA_STATUS_WAIT_TIMEOUT in the device status word, the kernel drains what it
started and returns.  The self-test entry point runs that exact wait on a
barrier phase nothing completes; this checks that the wait gives up, that the
host sees the status bit, and that the context is still usable: a forward
pass right after it matches the oracle.
"""
import time

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


def test_stream_scoped_status_reports_timeout_without_device_sync(oracle_lib):
    # The probe's bounded wait runs for about 2 s on stream a.  A status query
    # on another stream b neither waits for it nor sees its bit yet; the query
    # on stream a returns VA_ERR_DEVICE_TIMEOUT once the wait has given up.
    lib = binding.load()
    binding.device_status(clear=True)
    a, b = torch.cuda.Stream(), torch.cuda.Stream()
    gave_up = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    binding._check(lib.varlen_attention_selftest_wait_timeout(gave_up.data_ptr(), a.cuda_stream))
    t0 = time.perf_counter()
    rc, bits = binding.sync_status(b, clear=False)
    assert time.perf_counter() - t0 < 1.0, "the query on stream b waited for stream a"
    assert rc == binding.VA_OK and bits == 0
    rc, bits = binding.sync_status(a, clear=True)
    assert rc == binding.VA_ERR_DEVICE_TIMEOUT and bits & binding.VA_STATUS_WAIT_TIMEOUT, (rc, bits)
    assert "bounded wait" in lib.varlen_attention_last_error().decode()
    assert int(gave_up.item()) == 1
    assert binding.sync_status(a) == (binding.VA_OK, 0)  # cleared in stream order
    # the context stays usable: a forward pass on stream a matches the oracle
    wl = workloads.named("worked_example")
    q, k, v = workloads.make_qkv(wl)
    with torch.cuda.stream(a):
        out, lse = run_gpu(wl, q, k, v)
    compare(out, lse, *oracle_all(oracle_lib, wl, q, k, v))
    assert binding.sync_status(a) == (binding.VA_OK, 0)
