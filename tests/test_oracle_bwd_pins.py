"""Pins for the backward part of the fp64 oracle (CPU only).

The backward (boostr varlen_attention.rs, VarLenAttentionOps::
varlen_attention_bwd: dq, and dk / dv shaped [total_k, num_kv_heads, D] under
GQA) is checked against something other than itself:
  * torch autograd in float64 through a dense attention written with plain
    tensor operations on each sequence padded out (additive -inf band mask,
    K/V heads repeated; autograd sums the repeated heads' gradients, which is
    the GQA reduction the trait asks for);
  * closed forms: constant V rows give dq = dk = 0 (every dS_ij = 0) and
    dv_j = sum_i P_ij dout_i; a single visible key gives dv = dout and
    dq = dk = 0; zero dout gives zero gradients;
  * an invariant of the softmax Jacobian: sum_j dS_ij = 0 for every row, so
    the dk rows of a sequence sum to zero for each KV head.
"""
import numpy as np
import pytest
import torch

from variable_length_flash_varlen_b200 import workloads


def _grads(oracle_lib, wl, q, k, v, do):
    return oracle_lib.attention_bwd(q, k, v, do, wl.cu_q, wl.cu_k, wl.H, wl.H_kv, wl.D,
                                    wl.causal, wl.window, nthreads=4)


def _dout(wl, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(wl.total_q, wl.H, wl.D, generator=g).to(torch.bfloat16)


def _autograd_reference(wl, q, k, v, do):
    G = wl.H // wl.H_kv
    qd, kd, vd = (x.double().clone().requires_grad_(True) for x in (q, k, v))
    loss = torch.zeros((), dtype=torch.float64)
    for b in range(wl.batch):
        q0, q1, k0, k1 = wl.cu_q[b], wl.cu_q[b + 1], wl.cu_k[b], wl.cu_k[b + 1]
        Lq, Lk = q1 - q0, k1 - k0
        if Lq == 0 or Lk == 0:
            continue
        ones = torch.ones(Lq, Lk, dtype=torch.bool)
        delta = Lk - Lq
        keep = ones
        if wl.causal or wl.window > 0:
            keep = keep & ones.tril(diagonal=delta)
        if wl.window > 0:
            keep = keep & ones.triu(diagonal=delta - wl.window + 1)
        assert keep.any(dim=1).all()  # the cases below have no empty rows
        qb = qd[q0:q1].permute(1, 0, 2)                                   # [H, Lq, D]
        kb = kd[k0:k1].repeat_interleave(G, dim=1).permute(1, 0, 2)       # [H, Lk, D]
        vb = vd[k0:k1].repeat_interleave(G, dim=1).permute(1, 0, 2)
        s = qb @ kb.transpose(1, 2) / wl.D ** 0.5
        s = s.masked_fill(~keep, float("-inf"))
        o = torch.softmax(s, dim=-1) @ vb                                  # [H, Lq, D]
        loss = loss + (o.permute(1, 0, 2) * do[q0:q1].double()).sum()
    loss.backward()
    return qd.grad.numpy(), kd.grad.numpy(), vd.grad.numpy()


AUTOGRAD_CASES = [
    # lengths_q, lengths_k, H, H_kv, D, causal, window
    ([5, 17, 1, 33], [5, 17, 1, 33], 2, 2, 16, False, 0),
    ([5, 17, 1, 33], [5, 17, 1, 33], 4, 2, 16, True, 0),
    ([40, 9, 64], [40, 9, 64], 4, 1, 32, True, 7),
    ([3, 12, 20], [10, 12, 31], 6, 3, 8, True, 0),        # L_q <= L_k, bottom-right
    ([12, 20], [30, 25], 2, 1, 8, False, 5),               # window without the causal flag
    ([64, 32], [64, 32], 8, 2, 64, True, 0),
]


@pytest.mark.parametrize("case", AUTOGRAD_CASES)
def test_bwd_equals_torch_autograd(oracle_lib, case):
    Lq, Lk, H, Hkv, D, causal, W = case
    wl = workloads.custom(Lq, Lk, H, Hkv, D, causal, W, seed=81 + H)
    q, k, v = workloads.make_qkv(wl)
    do = _dout(wl, 82 + H)
    dq, dk, dv = _grads(oracle_lib, wl, q, k, v, do)
    rq, rk, rv = _autograd_reference(wl, q, k, v, do)
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-11)


def test_bwd_constant_v_rows(oracle_lib):
    L = [30, 7, 64]
    wl = workloads.custom(L, L, 4, 2, 32, True, 0, seed=83)
    q, k, _ = workloads.make_qkv(wl)
    c = torch.linspace(-1.5, 2.0, wl.D).to(torch.bfloat16)
    v = c.expand(wl.total_k, wl.H_kv, wl.D).contiguous()
    do = _dout(wl, 84)
    dq, dk, dv = _grads(oracle_lib, wl, q, k, v, do)
    assert np.abs(dq).max() < 1e-12 and np.abs(dk).max() < 1e-12
    # dv_j = sum over the group's heads and the rows i that see j of P_ij dout_i
    out, lse = oracle_lib.attention_rows(q, k, v, wl.cu_q, wl.cu_k, wl.H, wl.H_kv, wl.D,
                                         wl.causal, wl.window, nthreads=2)
    assert np.isfinite(lse).all()
    np.testing.assert_allclose(dv.sum(axis=(0, 1)), do.double().numpy().sum(axis=(0, 1)),
                               rtol=0, atol=1e-9)  # every row's P sums to 1


def test_bwd_single_visible_key(oracle_lib):
    wl = workloads.custom([1, 1, 1], [1, 1, 1], 4, 2, 16, False, 0, seed=85)
    q, k, v = workloads.make_qkv(wl)
    do = _dout(wl, 86)
    dq, dk, dv = _grads(oracle_lib, wl, q, k, v, do)
    assert np.abs(dq).max() == 0 and np.abs(dk).max() == 0
    want = do.double().numpy().reshape(3, 2, 2, 16).sum(axis=2)     # the group's two heads
    np.testing.assert_allclose(dv, want, rtol=0, atol=1e-15)


def test_bwd_zero_dout_and_dk_rows_sum_to_zero(oracle_lib):
    L = [50, 130, 9]
    wl = workloads.custom(L, L, 4, 4, 32, True, 20, seed=87)
    q, k, v = workloads.make_qkv(wl)
    zero = torch.zeros(wl.total_q, wl.H, wl.D, dtype=torch.bfloat16)
    for g in _grads(oracle_lib, wl, q, k, v, zero):
        assert np.abs(g).max() == 0
    dq, dk, dv = _grads(oracle_lib, wl, q, k, v, _dout(wl, 88))
    for b in range(wl.batch):
        seg = dk[wl.cu_k[b]:wl.cu_k[b + 1]]
        assert np.abs(seg.sum(axis=0)).max() < 1e-10 * max(1.0, np.abs(seg).max())
