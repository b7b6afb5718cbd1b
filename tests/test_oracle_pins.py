"""Pins for the fp64 oracle: facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself:
  * the worked cu_seqlens example printed on the boostr varlen_attention.rs
    page ("Cumulative sequence lengths"), from tests/golden/;
  * torch's CPU flash-attention routine in float64 on each sequence padded
    out to a dense [1, H, L, D] problem with an additive -inf band mask and
    K/V heads repeated (the dense AttentionOps::multi_head_attention contract
    of boostr flash.rs, and the repeat_kv that its "GQA support" section says
    the kernel avoids);
  * closed forms: constant V rows return that V; zero Q gives
    logsumexp = ln(number of visible keys) and O = mean of the visible V rows;
  * hand-derived tiny cases (L <= 4) with exactly representable inputs.
"""
import math
import os

import numpy as np
import pytest
import torch

from variable_length_flash_varlen_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _bf16(a):
    return torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)


def _run(oracle_lib, wl, q, k, v, rows=None):
    return oracle_lib.attention_rows(q, k, v, wl.cu_q, wl.cu_k, wl.H, wl.H_kv, wl.D,
                                     wl.causal, wl.window, rows=rows, nthreads=4)


# --- the printed worked example ----------------------------------------------

def test_worked_example_cu_seqlens_golden():
    fields = {}
    with open(os.path.join(GOLDEN, "cu_seqlens_worked_example.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, *vals = line.split()
            fields[key] = [int(x) for x in vals]
    assert workloads.cu_seqlens(fields["lengths"]) == fields["cu_seqlens"]
    wl = workloads.named("worked_example")
    assert wl.cu_q == fields["cu_seqlens"] and wl.cu_k == fields["cu_seqlens"]


# --- dense padded equivalence against torch's float64 CPU attention ----------

def _band_mask(Lq, Lk, causal, window):
    """Additive mask built from triangular matrices (not from the oracle's predicate)."""
    ones = torch.ones(Lq, Lk, dtype=torch.bool)
    delta = Lk - Lq
    keep = ones
    if causal or window > 0:
        keep = keep & ones.tril(diagonal=delta)
    if window > 0:
        keep = keep & ones.triu(diagonal=delta - window + 1)
    add = torch.zeros(Lq, Lk, dtype=torch.float64)
    add[~keep] = float("-inf")
    return add, keep


def _dense_reference(wl, q, k, v):
    """Per sequence: pad to dense, repeat K/V heads, call torch's fp64 CPU kernel."""
    G = wl.H // wl.H_kv
    outs, lses, valid = [], [], []
    for b in range(wl.batch):
        q0, q1, k0, k1 = wl.cu_q[b], wl.cu_q[b + 1], wl.cu_k[b], wl.cu_k[b + 1]
        Lq, Lk = q1 - q0, k1 - k0
        if Lq == 0:
            continue
        qb = q[q0:q1].double().permute(1, 0, 2).unsqueeze(0)            # [1,H,Lq,D]
        kb = k[k0:k1].double().repeat_interleave(G, dim=1).permute(1, 0, 2).unsqueeze(0)
        vb = v[k0:k1].double().repeat_interleave(G, dim=1).permute(1, 0, 2).unsqueeze(0)
        add, keep = _band_mask(Lq, Lk, wl.causal, wl.window)
        o, lse = torch.ops.aten._scaled_dot_product_flash_attention_for_cpu(
            qb, kb, vb, 0.0, False, attn_mask=add)[:2]
        outs.append(o[0].permute(1, 0, 2))
        lses.append(lse[0].permute(1, 0))
        valid.append(keep.any(dim=1))
    return torch.cat(outs).numpy(), torch.cat(lses).numpy(), torch.cat(valid).numpy()


DENSE_CASES = [
    # lengths_q, lengths_k, H, H_kv, D, causal, window
    ([5, 17, 1, 33], [5, 17, 1, 33], 2, 2, 16, False, 0),
    ([5, 17, 1, 33], [5, 17, 1, 33], 4, 2, 16, True, 0),
    ([40, 9, 64], [40, 9, 64], 4, 1, 32, True, 7),
    ([3, 12, 20], [10, 12, 31], 6, 3, 8, True, 0),       # L_q <= L_k, bottom-right
    ([12, 20], [30, 25], 2, 1, 8, False, 5),              # window without the causal flag
    ([64, 32], [64, 32], 8, 2, 64, True, 0),
]


@pytest.mark.parametrize("case", DENSE_CASES)
def test_oracle_equals_padded_dense_attention(oracle_lib, case):
    Lq, Lk, H, Hkv, D, causal, W = case
    wl = workloads.custom(Lq, Lk, H, Hkv, D, causal, W, seed=7 + len(Lq) + H)
    q, k, v = workloads.make_qkv(wl)
    out, lse = _run(oracle_lib, wl, q, k, v)
    ref_o, ref_lse, valid = _dense_reference(wl, q, k, v)
    assert valid.all()  # these cases have no empty rows
    np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_worked_example_against_dense(oracle_lib):
    wl = workloads.named("worked_example")
    q, k, v = workloads.make_qkv(wl)
    out, lse = _run(oracle_lib, wl, q, k, v)
    ref_o, ref_lse, _ = _dense_reference(wl, q, k, v)
    np.testing.assert_allclose(out, ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


# --- GQA equals explicit K/V head repetition ----------------------------------

@pytest.mark.parametrize("H,Hkv", [(4, 2), (8, 1), (6, 3)])
def test_gqa_equals_repeat_kv(oracle_lib, H, Hkv):
    wl = workloads.custom([7, 30, 2], [7, 30, 2], H, Hkv, 16, True, 0, seed=11)
    q, k, v = workloads.make_qkv(wl)
    out, lse = _run(oracle_lib, wl, q, k, v)
    G = H // Hkv
    wl_mha = workloads.custom([7, 30, 2], [7, 30, 2], H, H, 16, True, 0, seed=11)
    out2, lse2 = _run(oracle_lib, wl_mha, q, k.repeat_interleave(G, dim=1),
                      v.repeat_interleave(G, dim=1))
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


# --- closed forms ---------------------------------------------------------------

@pytest.mark.parametrize("causal,W", [(False, 0), (True, 0), (True, 5), (False, 3)])
def test_constant_v_rows_return_v(oracle_lib, causal, W):
    wl = workloads.custom([9, 40], [9, 40], 4, 2, 32, causal, W, seed=3)
    q, k, _ = workloads.make_qkv(wl)
    c = torch.linspace(-2, 2, 32)
    v = c.to(torch.bfloat16).expand(wl.total_k, wl.H_kv, 32).contiguous()
    out, lse = _run(oracle_lib, wl, q, k, v)
    np.testing.assert_allclose(out, np.broadcast_to(v[0, 0].double().numpy(), out.shape),
                               rtol=0, atol=1e-12)


def _visible_count(i, Lq, Lk, causal, W):
    # closed forms: non-causal sees all L_k keys; causal sees i + delta + 1;
    # a window caps that at W
    delta = Lk - Lq
    if not causal and W == 0:
        return Lk
    n = max(0, min(Lk, i + delta + 1))
    if W > 0:
        n = min(n, W)
    return n


@pytest.mark.parametrize("causal,W,Lq,Lk", [
    (False, 0, [33, 7], [33, 7]), (True, 0, [33, 7], [33, 7]), (True, 6, [33, 7], [33, 7]),
    (True, 0, [4, 9], [12, 9]), (True, 4, [4, 9], [12, 9]), (False, 6, [20], [20]),
])
def test_zero_q_lse_is_log_count_and_o_is_window_mean(oracle_lib, causal, W, Lq, Lk):
    wl = workloads.custom(Lq, Lk, 2, 1, 16, causal, W, seed=5)
    _, k, v = workloads.make_qkv(wl)
    q = torch.zeros(wl.total_q, 2, 16, dtype=torch.bfloat16)
    out, lse = _run(oracle_lib, wl, q, k, v)
    for b in range(wl.batch):
        vb = v[wl.cu_k[b]:wl.cu_k[b + 1], 0].double().numpy()
        csum = np.vstack([np.zeros((1, 16)), np.cumsum(vb, axis=0)])  # prefix sums
        delta = Lk[b] - Lq[b]
        for i in range(Lq[b]):
            n = _visible_count(i, Lq[b], Lk[b], causal, W)
            t = wl.cu_q[b] + i
            assert lse[t, 0] == pytest.approx(math.log(n), abs=1e-12)
            hi = Lk[b] if (not causal and W == 0) else min(Lk[b], i + delta + 1)
            mean = (csum[hi] - csum[hi - n]) / n
            np.testing.assert_allclose(out[t, 0], mean, rtol=0, atol=1e-12)
            np.testing.assert_allclose(out[t, 1], mean, rtol=0, atol=1e-12)


# --- hand-derived tiny cases (D = 4, scale 1/2) ----------------------------------

def test_hand_cases(oracle_lib):
    # L = 1: s00 = (2*3)/sqrt(4) = 3, the only key -> O = v0, LSE = 3
    wl = workloads.custom([1], [1], 1, 1, 4, True, 0, seed=0)
    q = _bf16([[[2, 0, 0, 0]]]); k = _bf16([[[3, 0, 0, 0]]]); v = _bf16([[[1, -2, 0.5, 4]]])
    out, lse = _run(oracle_lib, wl, q, k, v)
    assert lse[0, 0] == 3.0
    assert out[0, 0].tolist() == [1, -2, 0.5, 4]

    # L = 2, q rows (1, 2) e0, k rows (1, -1) e0, v rows e0, e1.
    q = _bf16([[[1, 0, 0, 0]], [[2, 0, 0, 0]]]); k = _bf16([[[1, 0, 0, 0]], [[-1, 0, 0, 0]]])
    v = _bf16([[[1, 0, 0, 0]], [[0, 1, 0, 0]]])
    wl = workloads.custom([2], [2], 1, 1, 4, True, 0, seed=0)
    out, lse = _run(oracle_lib, wl, q, k, v)
    # causal row 0 sees key 0 only: s00 = 1/2
    assert lse[0, 0] == pytest.approx(0.5, abs=1e-15)
    assert out[0, 0].tolist() == [1, 0, 0, 0]
    # row 1: s10 = 1, s11 = -1 -> weights 1/(1+e^-2), 1/(1+e^2); LSE = ln(2 cosh 1)
    assert lse[1, 0] == pytest.approx(math.log(2 * math.cosh(1.0)), abs=1e-14)
    np.testing.assert_allclose(out[1, 0], [1 / (1 + math.exp(-2)), 1 / (1 + math.exp(2)), 0, 0],
                               rtol=0, atol=1e-15)
    # non-causal row 0: s00 = 1/2, s01 = -1/2
    wl = workloads.custom([2], [2], 1, 1, 4, False, 0, seed=0)
    out, lse = _run(oracle_lib, wl, q, k, v)
    assert lse[0, 0] == pytest.approx(math.log(2 * math.cosh(0.5)), abs=1e-14)
    np.testing.assert_allclose(out[0, 0], [1 / (1 + math.exp(-1)), 1 / (1 + math.exp(1)), 0, 0],
                               rtol=0, atol=1e-15)

    # window W = 2, L = 4, causal, q = 0 -> uniform over keys {0}, {0,1}, {1,2}, {2,3}
    wl = workloads.custom([4], [4], 1, 1, 4, True, 2, seed=0)
    q = torch.zeros(4, 1, 4, dtype=torch.bfloat16)
    k = _bf16([[[1, 2, 3, 4]], [[-1, 0, 1, 0]], [[0, 0, 0, 1]], [[5, 5, 5, 5]]])
    v = _bf16([[[j, 0, 0, 0]] for j in range(4)])
    out, lse = _run(oracle_lib, wl, q, k, v)
    assert out[:, 0, 0].tolist() == [0.0, 0.5, 1.5, 2.5]
    np.testing.assert_allclose(lse[:, 0], [0.0, math.log(2), math.log(2), math.log(2)], atol=1e-15)

    # L_q = 2, L_k = 4, causal (bottom-right, delta = 2): rows see keys 0..2 and 0..3
    wl = workloads.custom([2], [4], 1, 1, 4, True, 0, seed=0)
    q = torch.zeros(2, 1, 4, dtype=torch.bfloat16)
    out, lse = _run(oracle_lib, wl, q, k, v)
    assert out[:, 0, 0].tolist() == [1.0, 1.5]
    np.testing.assert_allclose(lse[:, 0], [math.log(3), math.log(4)], atol=1e-15)


def test_empty_visible_sets(oracle_lib):
    # L_q = 3, L_k = 1, causal (delta = -2): rows 0 and 1 see nothing
    wl = workloads.custom([3, 2], [1, 0], 2, 1, 8, True, 0, seed=9)
    q, k, v = workloads.make_qkv(wl)
    out, lse = _run(oracle_lib, wl, q, k, v)
    assert np.all(lse[0:2] == -np.inf) and np.all(out[0:2] == 0)
    assert np.all(np.isfinite(lse[2]))
    np.testing.assert_array_equal(out[2, 0], v[0, 0].double().numpy())
    # L_k = 0 sequence: every row empty
    assert np.all(lse[3:5] == -np.inf) and np.all(out[3:5] == 0)
    # a zero-length query sequence contributes no rows
    wl = workloads.custom([0, 4], [3, 4], 2, 2, 8, False, 0, seed=9)
    q, k, v = workloads.make_qkv(wl)
    out, lse = _run(oracle_lib, wl, q, k, v)
    assert out.shape == (4, 2, 8)
    ref_o, ref_lse, _ = _dense_reference(wl, q, k, v)
    np.testing.assert_allclose(out, ref_o, atol=1e-12)


def test_window_without_causal_equals_causal_window(oracle_lib):
    a = workloads.custom([30], [30], 2, 1, 16, False, 6, seed=2)
    b = workloads.custom([30], [30], 2, 1, 16, True, 6, seed=2)
    q, k, v = workloads.make_qkv(a)
    oa, la = _run(oracle_lib, a, q, k, v)
    ob, lb = _run(oracle_lib, b, q, k, v)
    assert np.array_equal(oa, ob) and np.array_equal(la, lb)


def test_row_subset_matches_full(oracle_lib):
    wl = workloads.named("worked_example")
    q, k, v = workloads.make_qkv(wl)
    out, lse = _run(oracle_lib, wl, q, k, v)
    rng = np.random.default_rng(0)
    rows = np.stack([rng.integers(0, wl.total_q, 50), rng.integers(0, wl.H, 50)], axis=1)
    o2, l2 = _run(oracle_lib, wl, q, k, v, rows=rows)
    assert np.array_equal(o2, out[rows[:, 0], rows[:, 1]])
    assert np.array_equal(l2, lse[rows[:, 0], rows[:, 1]])


# --- the tile work list ------------------------------------------------------------

@pytest.mark.parametrize("Lq,Lk,causal,W", [
    ([512, 300, 128], [512, 300, 128], True, 0),
    ([700, 5, 129, 128, 1], [700, 5, 129, 128, 1], False, 0),
    ([1000, 300], [1000, 300], True, 200),
    ([100, 300], [400, 300], True, 0),
    ([300, 50], [20, 50], True, 0),
    ([260], [260], False, 130),
])
def test_schedule_key_ranges_match_band_mask(Lq, Lk, causal, W):
    from oracle import schedule as sch
    cu_q, cu_k = workloads.cu_seqlens(Lq), workloads.cu_seqlens(Lk)
    items = sch.schedule(cu_q, cu_k, causal, W)
    BM, BN = sch.BLOCK_M, sch.BLOCK_N
    expect, few = [], set()
    for b in range(len(Lq)):
        _, keep = _band_mask(Lq[b], Lk[b], causal, W)
        for qt in range((Lq[b] + BM - 1) // BM):
            rows = keep[qt * BM:(qt + 1) * BM]
            cols = torch.nonzero(rows.any(dim=0)).flatten()
            rng = (int(cols.min()) // BN, int(cols.max()) // BN + 1) if len(cols) else (0, 0)
            expect.append((b, qt) + rng)
            # a tile with a row that sees 1..256 keys belongs to the second part
            counts = rows.sum(dim=1)
            if bool(((counts >= 1) & (counts <= sch.RESIDUAL_MAX_KEYS)).any()):
                few.add((b, qt))
    assert sorted(items) == sorted(expect)
    flags = [(it[0], it[1]) in few for it in items]
    assert flags == sorted(flags), "tiles with a few-key row must come last"
    for part in (False, True):
        sub = [it for it, f in zip(items, flags) if f == part]
        costs = [it[3] - it[2] for it in sub]
        assert costs == sorted(costs, reverse=True)
        for a, b in zip(sub, sub[1:]):
            if a[3] - a[2] == b[3] - b[2]:
                assert (a[0], a[1]) < (b[0], b[1])
    # without the split, one part ordered the same way
    assert sch.schedule(cu_q, cu_k, causal, W, split_few_keys=False) == sorted(
        items, key=lambda it: (-(it[3] - it[2]), it[0], it[1]))


# --- key-value cache with a capacity stride ------------------------------------

@pytest.mark.parametrize("causal,window,H,H_kv", [(False, 0, 4, 2), (True, 0, 2, 1), (True, 5, 4, 4)])
def test_capacity_stride_equals_compacted_layout(oracle_lib, causal, window, H, H_kv):
    # flash.rs FlashAttentionOps "kv_seq_len": iterate over the first n key
    # positions while the buffer's size stays the stride.  In the packed
    # layout: keys of sequence b are the first min(seqused_k[b], capacity)
    # rows of its slot.  The same rows copied into a compact packed tensor
    # (no seqused) must give bitwise the same result: the oracle then sums the
    # same products in the same order.  Unused slot rows hold large finite
    # garbage that would change every result if it were read.
    D = 16
    L_q = [3, 1, 4, 2, 5]
    cap = [8, 6, 4, 9, 7]
    used = [5, 6, 0, 12, 7]  # full slot, empty, beyond the capacity (clamped)
    cu_q = workloads.cu_seqlens(L_q)
    cu_cache = workloads.cu_seqlens(cap)
    g = torch.Generator().manual_seed(11)
    q = torch.randn(cu_q[-1], H, D, generator=g).to(torch.bfloat16)
    kc = (torch.randn(cu_cache[-1], H_kv, D, generator=g) * 50).to(torch.bfloat16)
    vc = (torch.randn(cu_cache[-1], H_kv, D, generator=g) * 50).to(torch.bfloat16)
    eff = [min(u, c) for u, c in zip(used, cap)]
    keep = torch.cat([torch.arange(cu_cache[b], cu_cache[b] + eff[b]) for b in range(len(cap))])
    for b in range(len(cap)):  # the used rows: ordinary N(0, 1) data
        kc[cu_cache[b]:cu_cache[b] + eff[b]] = torch.randn(eff[b], H_kv, D, generator=g).to(torch.bfloat16)
        vc[cu_cache[b]:cu_cache[b] + eff[b]] = torch.randn(eff[b], H_kv, D, generator=g).to(torch.bfloat16)
    o1, l1 = oracle_lib.attention_rows(q, kc, vc, cu_q, cu_cache, H, H_kv, D, causal, window,
                                       seqused_k=used)
    o2, l2 = oracle_lib.attention_rows(q, kc[keep], vc[keep], cu_q, workloads.cu_seqlens(eff), H,
                                       H_kv, D, causal, window)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    # the empty sequence: no visible key
    b = 2
    assert np.all(np.isneginf(l1[cu_q[b]:cu_q[b + 1]])) and np.all(o1[cu_q[b]:cu_q[b + 1]] == 0)


def test_capacity_stride_with_full_counts_is_the_plain_layout(oracle_lib):
    wl = workloads.custom([5, 7], [9, 7], 2, 1, 16, True, 0, seed=13)
    q, k, v = workloads.make_qkv(wl)
    o1, l1 = _run(oracle_lib, wl, q, k, v)
    o2, l2 = oracle_lib.attention_rows(q, k, v, wl.cu_q, wl.cu_k, wl.H, wl.H_kv, wl.D, wl.causal,
                                       wl.window, seqused_k=wl.lengths_k)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
