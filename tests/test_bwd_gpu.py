"""GPU parity of the backward pass (dq, dk, dv) against the fp64 oracle.

The GPU backward consumes the GPU forward's output and logsumexp (as the
trait's varlen_attention_bwd does), rounds P and dS to bf16 for its tensor-core
products and writes bf16 gradients; the oracle differentiates the exact
attention of the same bf16 inputs in fp64.  The trait's backward (boostr
varlen_attention.rs, VarLenAttentionOps::varlen_attention_bwd) states no
tolerance; the bar per tensor is:

  |g_gpu - g_ref| <= half a bf16 step at g_ref + 1e-2 * max |g_ref|

(each gradient entry is a sum of products whose bf16 rounding errors, at most
2^-9 relative each, accumulate like a random walk, as the entry itself does,
so the error stays near 2^-9 of the tensor's scale; 1e-2 leaves a margin of
about five) and no NaN anywhere.
"""
import numpy as np
import pytest
import torch

from variable_length_flash_varlen_b200 import binding, workloads
from tests._helpers import bf16_half_ulp, to_device_inputs

pytestmark = pytest.mark.gpu

REL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    binding.load()
    binding.device_status(clear=True)
    yield
    assert binding.device_status(clear=True) == 0, "device status word raised"


def _dout(wl, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(wl.total_q, wl.H, wl.D, generator=g).to(torch.bfloat16)


def run_bwd(wl, q, k, v, do):
    dq_, dk_, dv_, cq, ck = to_device_inputs(wl, q, k, v)
    out, lse = binding.varlen_attention_fwd(dq_, dk_, dv_, cq, ck, wl.batch, wl.H, wl.H_kv,
                                            wl.max_seqlen_q, wl.max_seqlen_k, wl.D, wl.causal,
                                            wl.window, path=binding.VA_PATH_PREFILL)
    nan = float("nan")
    gq = torch.full_like(dq_, nan)
    gk = torch.full_like(dk_, nan)
    gv = torch.full_like(dv_, nan)
    binding.varlen_attention_bwd(do.cuda(), dq_, dk_, dv_, out, lse, cq, ck, wl.batch, wl.H,
                                 wl.H_kv, wl.max_seqlen_q, wl.max_seqlen_k, wl.D, wl.causal,
                                 wl.window, dq=gq, dk=gk, dv=gv)
    torch.cuda.synchronize()
    return gq, gk, gv


def compare_grads(got, ref, name):
    g = got.float().cpu().double().numpy()
    assert not np.isnan(g).any(), f"NaN (or an unwritten row) in {name}"
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    excess = np.abs(g - ref) - bf16_half_ulp(ref) - REL * scale
    worst = float(excess.max()) if ref.size else 0.0
    assert worst <= 0.0, (f"{name}: beyond the bar by {worst:.3g} "
                          f"(max |d| {np.abs(g - ref).max():.3g}, max |ref| {scale:.3g})")
    return float(np.abs(g - ref).max()) / max(scale, 1e-30)


def check(oracle_lib, wl, seed=5):
    q, k, v = workloads.make_qkv(wl)
    do = _dout(wl, seed)
    gq, gk, gv = run_bwd(wl, q, k, v, do)
    rq, rk, rv = oracle_lib.attention_bwd(q, k, v, do, wl.cu_q, wl.cu_k, wl.H, wl.H_kv, wl.D,
                                          wl.causal, wl.window)
    return [compare_grads(x, r, n) for x, r, n in ((gq, rq, "dq"), (gk, rk, "dk"), (gv, rv, "dv"))]


REDUCED = [("worked_example", 1.0), ("mha_noncausal", 0.1), ("gqa_causal", 0.03),
           ("sliding_window", 1 / 32), ("chunked_prefill", 0.05)]


@pytest.mark.parametrize("name,scale", REDUCED)
def test_bwd_reduced_workloads_match_oracle(oracle_lib, name, scale):
    check(oracle_lib, workloads.named(name, scale=scale))


BWD_EDGE = [
    # lengths_q, lengths_k, H, H_kv, D, causal, window
    ([1, 127, 128, 129, 255, 256, 257, 1], None, 4, 1, 128, True, 0),
    ([1, 127, 128, 129, 255, 256, 257, 1], None, 4, 1, 128, False, 0),
    ([100, 5, 300], [300, 5, 130], 4, 2, 128, True, 0),      # L_q != L_k; rows with no key
    ([100, 5, 300], [300, 5, 130], 4, 2, 128, False, 0),
    ([300, 200], [300, 200], 4, 4, 128, False, 37),           # window without causal
    ([0, 130, 0, 70, 3], [0, 130, 5, 70, 0], 2, 1, 128, True, 0),  # empty sequences
    ([200, 333], None, 16, 2, 128, True, 0),                  # GQA group of 8
    ([129, 1000], None, 8, 8, 64, True, 96),                  # D = 64, window
    ([700], None, 2, 1, 128, True, 0),                        # several tiles each way
]


@pytest.mark.parametrize("case", BWD_EDGE)
def test_bwd_edge_cases_match_oracle(oracle_lib, case):
    Lq, Lk, H, Hkv, D, causal, W = case
    check(oracle_lib, workloads.custom(Lq, Lk if Lk is not None else Lq, H, Hkv, D, causal, W,
                                       seed=91))


def test_bwd_is_deterministic():
    wl = workloads.custom([300, 129], [300, 129], 8, 2, 128, True, 0, seed=92)
    q, k, v = workloads.make_qkv(wl)
    do = _dout(wl, 93)
    a = run_bwd(wl, q, k, v, do)
    b = run_bwd(wl, q, k, v, do)
    assert all(torch.equal(x, y) for x, y in zip(a, b))


def test_bwd_argument_errors():
    # through the C ABI directly: num_heads not a multiple of num_kv_heads, and
    # an unsupported head_dim
    lib = binding.load()
    wl = workloads.custom([10], [10], 2, 1, 128, False, 0, seed=1)
    q, k, v = workloads.make_qkv(wl)
    dq_, dk_, dv_, cq, ck = to_device_inputs(wl, q, k, v)
    lse = torch.zeros(10, 2, dtype=torch.float32, device="cuda")
    g = torch.empty_like(dq_)
    ptrs = [dq_.data_ptr(), dq_.data_ptr(), dk_.data_ptr(), dv_.data_ptr(), dq_.data_ptr(),
            lse.data_ptr(), cq.data_ptr(), ck.data_ptr()]
    outs = [g.data_ptr(), g.data_ptr(), g.data_ptr(), 0]
    assert lib.varlen_attention_bwd(*ptrs, 1, 3, 2, 10, 10, 128, 0, 0, *outs) == -1
    assert lib.varlen_attention_bwd(*ptrs, 1, 2, 1, 10, 10, 96, 0, 0, *outs) == -2


@pytest.mark.parametrize("name,pick", [("mha_noncausal", "shortest"), ("mha_noncausal", "longest"),
                                       ("gqa_causal", "long")])
def test_bwd_full_size_sampled_sequences(oracle_lib, name, pick):
    # the benchmark's backward workloads in their launch configuration;
    # sequences are independent, so the oracle on a few of them alone gives
    # their exact gradients: the three shortest and the three longest of the
    # MHA workload (the longest have the most key tiles per query tile), and one
    # GQA causal sequence of at least 4096 tokens
    wl = workloads.named(name)
    q, k, v = workloads.make_qkv(wl)
    do = _dout(wl, 7)
    gq, gk, gv = run_bwd(wl, q, k, v, do)
    order = sorted(range(wl.batch), key=lambda x: wl.lengths_q[x])
    if pick == "shortest":
        chosen = order[:3]
    elif pick == "longest":
        chosen = order[-3:]
    else:
        chosen = [next(b for b in order if wl.lengths_q[b] >= 4096)]
    for b in chosen:
        q0, q1, k0, k1 = wl.cu_q[b], wl.cu_q[b + 1], wl.cu_k[b], wl.cu_k[b + 1]
        sub = workloads.custom([q1 - q0], [k1 - k0], wl.H, wl.H_kv, wl.D, wl.causal, wl.window,
                               seed=0)
        rq, rk, rv = oracle_lib.attention_bwd(q[q0:q1], k[k0:k1], v[k0:k1], do[q0:q1], sub.cu_q,
                                              sub.cu_k, wl.H, wl.H_kv, wl.D, wl.causal, wl.window)
        compare_grads(gq[q0:q1], rq, f"dq of sequence {b}")
        compare_grads(gk[k0:k1], rk, f"dk of sequence {b}")
        compare_grads(gv[k0:k1], rv, f"dv of sequence {b}")
    for g in (gq, gk, gv):
        assert not torch.isnan(g).any()
