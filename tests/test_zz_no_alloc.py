"""The allocation-free entry point against the default one (GPU).

Some callers cannot allocate device memory: code inside a framework or
serving runtime that owns all device memory through its own allocator, or a
latency-critical loop that may not reach cudaMalloc or a stream-ordered
allocator.  varlen_attention_fwd_noalloc serves them from a static per-device
scratch array.  This file checks, through the C ABI, that two calls in a row
give what varlen_attention_fwd gives and what the fp64 oracle gives (within
the parity tolerances of the other tests), including after a call of another
shape has left different contents in the shared array, that calls after the
first one leave the device's free memory unchanged in a process that never
used the allocating entry points, and that an over-size problem is refused.

It is collected last on purpose, and it loads everything it needs itself, so
it passes alone in a fresh process as well as after the other tests.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from variable_length_flash_varlen_b200 import binding, workloads
from tests._helpers import compare, oracle_all

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 1e-2, 1e-3


def _inputs(wl, host=None):
    q, k, v = [t.cuda() for t in host] if host is not None else workloads.make_qkv(wl, device="cuda")
    cq = torch.tensor(wl.cu_q, dtype=torch.int32, device="cuda")
    ck = torch.tensor(wl.cu_k, dtype=torch.int32, device="cuda")
    return q, k, v, cq, ck


def _args(wl):
    return (wl.batch, wl.H, wl.H_kv, wl.max_seqlen_q, wl.max_seqlen_k, wl.D, wl.causal, wl.window)


def _close(a_out, a_lse, b_out, b_lse):
    do = (a_out.float() - b_out.float()).abs().max().item()
    fin = torch.isfinite(b_lse)
    assert torch.equal(torch.isneginf(a_lse), torch.isneginf(b_lse))
    dl = (a_lse[fin] - b_lse[fin]).abs().max().item() if fin.any() else 0.0
    assert do <= O_TOL and dl <= LSE_TOL, (do, dl)
    assert not torch.isnan(a_out).any() and not torch.isnan(a_lse).any()


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    binding.load()


@pytest.mark.parametrize("name,scale", [("gqa_causal", 0.25), ("worked_example", 1.0),
                                        ("sliding_window", 1 / 8)])
def test_noalloc_matches_default_entry_on_two_calls(oracle_lib, name, scale):
    wl = workloads.named(name, scale=scale)
    host = workloads.make_qkv(wl)
    q, k, v, cq, ck = _inputs(wl, host)
    ref_out, ref_lse = binding.varlen_attention_fwd(q, k, v, cq, ck, *_args(wl))
    ora_out, ora_lse = oracle_all(oracle_lib, wl, *host)
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full((wl.total_q, wl.H), float("nan"), dtype=torch.float32, device="cuda")
        binding.varlen_attention_fwd_noalloc(q, k, v, cq, ck, *_args(wl), out, lse)
        torch.cuda.synchronize()
        _close(out, lse, ref_out, ref_lse)
        compare(out, lse, ora_out, ora_lse)
    assert binding.device_status(clear=True) == 0


# Run in a fresh process that never calls an allocating entry point, so that no
# pool of the library holds reserved memory an allocation could hide in: after
# the first (set-up) call, more calls must leave the device's free memory as
# it was.  The outputs are allocated before the first call.
_FREE_MEMORY_SCRIPT = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
from variable_length_flash_varlen_b200 import binding, workloads
wl = workloads.named("gqa_causal", scale=0.05)
q, k, v = workloads.make_qkv(wl, device="cuda")
cq = torch.tensor(wl.cu_q, dtype=torch.int32, device="cuda")
ck = torch.tensor(wl.cu_k, dtype=torch.int32, device="cuda")
out = torch.empty_like(q)
lse = torch.empty(wl.total_q, wl.H, dtype=torch.float32, device="cuda")
args = (wl.batch, wl.H, wl.H_kv, wl.max_seqlen_q, wl.max_seqlen_k, wl.D, wl.causal, wl.window)
binding.varlen_attention_fwd_noalloc(q, k, v, cq, ck, *args, out, lse)
torch.cuda.synchronize()
free0 = torch.cuda.mem_get_info()[0]
for _ in range(3):
    binding.varlen_attention_fwd_noalloc(q, k, v, cq, ck, *args, out, lse)
torch.cuda.synchronize()
free1 = torch.cuda.mem_get_info()[0]
print("FREE", free0, free1)
"""


def test_noalloc_calls_leave_free_device_memory_unchanged():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _FREE_MEMORY_SCRIPT, root], capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [x for x in r.stdout.splitlines() if x.startswith("FREE")][-1]
    free0, free1 = (int(x) for x in line.split()[1:])
    assert free0 == free1, f"free device memory moved from {free0} to {free1} bytes"


def test_noalloc_serves_single_query_sequences():
    wl = workloads.custom([1, 1, 0, 1], [700, 5, 3, 1200], 8, 2, 128, False, 0, seed=4)
    q, k, v, cq, ck = _inputs(wl)
    ref_out, ref_lse = binding.varlen_attention_fwd(q, k, v, cq, ck, *_args(wl))
    out = torch.empty_like(q)
    lse = torch.empty(wl.total_q, wl.H, dtype=torch.float32, device="cuda")
    binding.varlen_attention_fwd_noalloc(q, k, v, cq, ck, *_args(wl), out, lse)
    torch.cuda.synchronize()
    _close(out, lse, ref_out, ref_lse)


def test_noalloc_refuses_problems_beyond_its_scratch():
    wl = workloads.custom([300], [300], 2, 1, 64, True, 0, seed=1)
    q, k, v, cq, ck = _inputs(wl)
    out = torch.empty_like(q)
    lse = torch.empty(wl.total_q, wl.H, dtype=torch.float32, device="cuda")
    # 4096 sequences of up to 65536 queries: far more query blocks than 1 MiB describes
    with pytest.raises(binding.VarlenAttentionError) as e:
        binding.varlen_attention_fwd_noalloc(q, k, v, cq, ck, 4096, 2, 1, 65536, 300, 64, True, 0,
                                             out, lse)
    assert e.value.code == -2 and "static scratch" in str(e.value)
