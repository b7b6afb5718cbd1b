"""Key-value cache with a capacity stride against the oracle (GPU).

boostr flash.rs, FlashAttentionOps docs, section kv_seq_len: attention over
the first n key positions of a buffer whose size stays the stride.  Packed
form: sequence b's keys are the first seqused_k[b] rows of its slot
cu_seqlens_k[b]..cu_seqlens_k[b+1]-1.  Unused slot rows hold large finite
garbage that would change the result if any of it were attended to.
"""
import numpy as np
import pytest
import torch

from variable_length_flash_varlen_b200 import binding, workloads
from tests._helpers import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    binding.load()
    binding.device_status(clear=True)
    yield
    assert binding.device_status(clear=True) == 0, "device status word raised"


def _cache(L_q, slots, used, H, H_kv, D, seed):
    g = torch.Generator().manual_seed(seed)
    cu_q = workloads.cu_seqlens(L_q)
    cu_k = workloads.cu_seqlens(slots)
    q = torch.randn(cu_q[-1], H, D, generator=g).to(torch.bfloat16)
    k = (torch.randn(cu_k[-1], H_kv, D, generator=g) * 50).to(torch.bfloat16)
    v = (torch.randn(cu_k[-1], H_kv, D, generator=g) * 50).to(torch.bfloat16)
    for b, (c, u) in enumerate(zip(slots, used)):
        n = min(max(u, 0), c)
        k[cu_k[b]:cu_k[b] + n] = torch.randn(n, H_kv, D, generator=g).to(torch.bfloat16)
        v[cu_k[b]:cu_k[b] + n] = torch.randn(n, H_kv, D, generator=g).to(torch.bfloat16)
    return q, k, v, cu_q, cu_k


CASES = [
    # L_q, slot sizes, used counts (0 = empty, above the slot = clamped), H, H_kv, D, causal, window
    ([1] * 6, [4096, 1000, 300, 2048, 50, 700], [4000, 1000, 0, 1500, 70, 1], 8, 2, 128, False, 0),
    ([1] * 4, [3000, 640, 129, 900], [2999, 5, 129, 640], 4, 1, 64, True, 300),
    ([64, 200, 128, 10], [1024, 600, 512, 300], [900, 450, 512, 8], 8, 2, 128, True, 0),
    ([300, 77, 256], [2000, 500, 900], [1800, 77, 300], 4, 4, 64, True, 250),
    ([130, 257], [700, 1400], [0, 1399], 2, 1, 128, False, 0),
]


@pytest.mark.parametrize("case", CASES)
def test_kvcache_matches_oracle(oracle_lib, case):
    L_q, slots, used, H, H_kv, D, causal, window = case
    q, k, v, cu_q, cu_k = _cache(L_q, slots, used, H, H_kv, D, seed=sum(slots))
    dev = [t.cuda() for t in (q, k, v)]
    cq = torch.tensor(cu_q, dtype=torch.int32, device="cuda")
    ck = torch.tensor(cu_k, dtype=torch.int32, device="cuda")
    su = torch.tensor(used, dtype=torch.int32, device="cuda")
    out = torch.full_like(dev[0], float("nan"))
    lse = torch.full((cu_q[-1], H), float("nan"), dtype=torch.float32, device="cuda")
    binding.varlen_attention_fwd_kvcache(*dev, cq, ck, su, len(L_q), H, H_kv, max(L_q), max(slots),
                                         D, causal, window, out=out, lse=lse)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle_lib.attention_rows(q, k, v, cu_q, cu_k, H, H_kv, D, causal, window,
                                             seqused_k=used)
    compare(out, lse, ref_o, ref_l)


def test_kvcache_with_full_counts_equals_plain_entry():
    wl = workloads.custom([1, 1, 200], [700, 90, 333], 8, 2, 128, True, 0, seed=5)
    q, k, v = workloads.make_qkv(wl, device="cuda")
    cq = torch.tensor(wl.cu_q, dtype=torch.int32, device="cuda")
    ck = torch.tensor(wl.cu_k, dtype=torch.int32, device="cuda")
    su = torch.tensor(wl.lengths_k, dtype=torch.int32, device="cuda")
    a = binding.varlen_attention_fwd(q, k, v, cq, ck, wl.batch, wl.H, wl.H_kv, wl.max_seqlen_q,
                                     wl.max_seqlen_k, wl.D, wl.causal, wl.window)
    b = binding.varlen_attention_fwd_kvcache(q, k, v, cq, ck, su, wl.batch, wl.H, wl.H_kv,
                                             wl.max_seqlen_q, wl.max_seqlen_k, wl.D, wl.causal,
                                             wl.window)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
