"""Host logic of the host-buffer entry point's pipeline plan (no GPU).

varlen_attention_fwd_host cuts the packed batch into chunks in query order:
groups of whole sequences, and pieces of a long sequence made of whole
256-row query blocks, each launched with only the keys its rows can see.
These tests check, on the workloads' own lengths and on edge shapes, that
the plan covers every query row once, copies every key row once and before
the first chunk that reads it, and that each piece, launched as a sequence of
its own under the mask readings (bottom-right causal diagonal, a window of W
keys ending at the diagonal), gives every row exactly the keys the whole
sequence gives it, on the same 256-row blocks and 128-key tiles (so that the
results can be bit-identical to one launch).
"""
import numpy as np
import pytest

from variable_length_flash_varlen_b200 import binding, workloads

BLOCK_Q, TILE_K = 256, 128


def visible(i, L_q, L_k, causal, window):
    """Visible key interval [lo, hi] of rows i (vectorised), empty when lo > hi."""
    delta = L_k - L_q
    lo = np.zeros_like(i)
    hi = np.full_like(i, L_k - 1)
    if causal or window > 0:
        hi = np.minimum(hi, i + delta)
    if window > 0:
        lo = np.maximum(lo, i + delta - window + 1)
    return lo, hi


def check_plan(cu_q, cu_k, causal, window, input_bytes):
    batch = len(cu_q) - 1
    plan = binding.host_chunks(cu_q, cu_k, batch, causal, window, input_bytes)
    q_next, k_next = 0, 0
    for c in plan:
        assert c["q0"] == q_next, "query rows not covered in order"
        q_next = c["q1"]
        if c["kc1"] > c["kc0"]:
            assert c["kc0"] == k_next, "key rows not copied once, in order"
            k_next = c["kc1"]
        if not c["piece"]:
            b0, b1 = c["b0"], c["b1"]
            assert (c["q0"], c["q1"], c["k_base"]) == (cu_q[b0], cu_q[b1], cu_k[b0])
            assert k_next >= cu_k[b1], "a group reads keys not yet copied"
            continue
        b = c["b0"]
        assert c["b1"] == b + 1
        L_q, L_k = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        r0, r1 = c["q0"] - cu_q[b], c["q1"] - cu_q[b]
        k_lo, k_len = c["k_base"] - cu_k[b], c["k_len"]
        assert r0 % BLOCK_Q == 0 and k_lo % TILE_K == 0
        assert 0 <= k_lo and k_lo + k_len <= L_k
        assert cu_k[b] + k_lo + k_len <= k_next, "a piece reads keys not yet copied"
        i = np.arange(r0, r1, dtype=np.int64)
        lo, hi = visible(i, L_q, L_k, causal, window)
        lo2, hi2 = visible(i - r0, r1 - r0, k_len, causal, window)
        empty, empty2 = lo > hi, lo2 > hi2
        assert np.array_equal(empty, empty2)
        assert np.array_equal(lo[~empty], lo2[~empty] + k_lo)
        assert np.array_equal(hi[~empty], hi2[~empty] + k_lo)
    assert q_next == cu_q[-1]
    if len(plan) > 1:
        assert k_next == cu_k[-1]
    return plan


def input_bytes(wl):
    return 2 * wl.D * (wl.total_q * wl.H + 2 * wl.total_k * wl.H_kv)


@pytest.mark.parametrize("name", ["sliding_window", "gqa_causal", "mha_noncausal", "chunked_prefill",
                                  "worked_example"])
def test_plan_on_the_workloads(name):
    wl = workloads.named(name)
    plan = check_plan(wl.cu_q, wl.cu_k, wl.causal, wl.window, input_bytes(wl))
    n_pieces = sum(c["piece"] for c in plan)
    if name == "sliding_window":
        # four 32768-token sequences: 16 pieces of 8192 query rows, each with
        # the 4096-key window below its first row (rounded down to a tile)
        assert len(plan) == 16 and n_pieces == 16
        assert all(c["q1"] - c["q0"] == 8192 for c in plan)
    if name == "worked_example":
        assert len(plan) == 1  # below the pipelining threshold


@pytest.mark.parametrize("lq,lk,causal,window", [
    ([10000, 500], [10000, 500], False, 0),     # non-causal: every piece takes all keys
    ([9000, 100], [12000, 300], True, 0),       # causal, fewer queries than keys
    ([9000], [6000], True, 0),                  # causal, more queries: early rows see nothing
    ([20000], [20000], False, 1000),            # a window without causal
    ([9000], [15000], True, 777),               # window, fewer queries, odd width
    ([0, 9000, 0, 300], [5, 9000, 0, 300], True, 0),  # empty sequences around a long one
])
def test_plan_on_edge_shapes(lq, lk, causal, window):
    cu_q = np.concatenate([[0], np.cumsum(lq)]).tolist()
    cu_k = np.concatenate([[0], np.cumsum(lk)]).tolist()
    plan = check_plan(cu_q, cu_k, causal, window, 64 << 20)
    assert any(c["piece"] for c in plan)


def test_plan_below_threshold_is_one_launch():
    plan = binding.host_chunks([0, 9000], [0, 9000], 1, True, 0, 1 << 20)
    assert len(plan) == 1 and not plan[0]["piece"]


def test_plan_rejects_bad_cu_seqlens():
    with pytest.raises(binding.VarlenAttentionError):
        binding.host_chunks([0, 10, 5], [0, 10, 20], 2, True, 0, 64 << 20)
    with pytest.raises(binding.VarlenAttentionError):
        binding.host_chunks([1, 10], [0, 10], 1, True, 0, 64 << 20)
