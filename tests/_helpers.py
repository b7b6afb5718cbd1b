"""Shared helpers for the parity tests: run the CUDA path and the oracle on
the same seeded inputs and compare element by element."""
import numpy as np
import torch

from variable_length_flash_varlen_b200 import binding, workloads

import os

O_TOL = 1e-2    # |O_gpu - O_oracle| wherever a bf16 result can come that close
LSE_TOL = 1e-3  # max |LSE_gpu - LSE_oracle|
# Where |O_oracle| >= 4 the nearest bf16 number can lie up to 2^-6 = 0.0156
# from the exact value (half the bf16 spacing there), so no bf16 output meets
# 1e-2; there the bar is that half spacing plus this much arithmetic error.
HALF_ULP_SLACK = 1e-3

# One record per comparison, printed by the terminal summary in conftest.py:
# (test id, elements, max |dO|, worst |dO| / bar, max |dLSE|, max |O_oracle|)
MARGINS = []


def bf16_half_ulp(x):
    """Half the spacing of bf16 numbers at |x| (8 significant bits): the
    smallest error any bf16 output can have against an exact value there."""
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.ldexp(1.0, np.floor(np.log2(ax)).astype(np.int64) - 8)


def to_device_inputs(wl, q, k, v):
    dev = "cuda"
    cu_q = torch.tensor(wl.cu_q, dtype=torch.int32, device=dev)
    cu_k = torch.tensor(wl.cu_k, dtype=torch.int32, device=dev)
    return q.to(dev), k.to(dev), v.to(dev), cu_q, cu_k


def run_gpu(wl, q, k, v, path=binding.VA_PATH_AUTO, split_keys=0, dev_inputs=None):
    dq, dk, dv, cu_q, cu_k = dev_inputs or to_device_inputs(wl, q, k, v)
    out = torch.full_like(dq, float("nan"))
    lse = torch.full((dq.shape[0], wl.H), float("nan"), dtype=torch.float32, device="cuda")
    binding.varlen_attention_fwd(dq, dk, dv, cu_q, cu_k, wl.batch, wl.H, wl.H_kv,
                                 wl.max_seqlen_q, wl.max_seqlen_k, wl.D, wl.causal, wl.window,
                                 out=out, lse=lse, path=path, decode_split_keys=split_keys)
    torch.cuda.synchronize()
    return out, lse


def oracle_all(oracle_lib, wl, q, k, v):
    return oracle_lib.attention_rows(q, k, v, wl.cu_q, wl.cu_k, wl.H, wl.H_kv, wl.D,
                                     wl.causal, wl.window)


def o_bar(out_ref):
    """Per-element bar on |O_gpu - O_oracle|: 1e-2, or where that is below
    what any bf16 number can reach (half a bf16 step at |O_oracle| >= 4), that
    half step plus HALF_ULP_SLACK."""
    return np.maximum(O_TOL, bf16_half_ulp(out_ref) + HALF_ULP_SLACK)


def record_margin(n, d_o, ratio, d_l, o_max):
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    MARGINS.append((test, int(n), float(d_o), float(ratio), float(d_l), float(o_max)))


def compare(out_gpu, lse_gpu, out_ref, lse_ref, rows=None):
    """Element-wise comparison; returns (max |dO|, max |dLSE|)."""
    o = out_gpu.float().cpu().double().numpy()
    l = lse_gpu.float().cpu().double().numpy()
    if rows is not None:
        o = o[rows[:, 0], rows[:, 1]]
        l = l[rows[:, 0], rows[:, 1]]
    assert not np.isnan(o).any(), "NaN in GPU output"
    assert not np.isnan(l).any(), "NaN in GPU logsumexp"
    neg_ref = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(l), neg_ref), "-inf logsumexp rows differ"
    err = np.abs(o - out_ref)
    d_o = float(np.max(err)) if o.size else 0.0
    ratio = float(np.max(err / o_bar(out_ref))) if o.size else 0.0
    fin = ~neg_ref
    d_l = float(np.max(np.abs(l[fin] - lse_ref[fin]))) if fin.any() else 0.0
    record_margin(o.size, d_o, ratio, d_l, float(np.max(np.abs(out_ref))) if o.size else 0.0)
    if ratio > 1.0:
        w = np.unravel_index(int(np.argmax(err / o_bar(out_ref))), err.shape)
        raise AssertionError(f"|dO| beyond its bar: worst {float(err[w]):.5f} at {w} where the oracle "
                             f"gives {float(out_ref[w]):.5f} (bar {float(o_bar(out_ref)[w]):.5f}); "
                             f"max |dO| {d_o:.5f}")
    assert d_l <= LSE_TOL, f"max |dLSE| = {d_l}"
    return d_o, d_l


def sample_rows(wl, n_random, seed=0):
    """(token, head) rows: random ones plus the first and last row of every sequence."""
    rng = np.random.default_rng(seed)
    toks = [rng.integers(0, wl.total_q, n_random)]
    edge = []
    for b in range(wl.batch):
        if wl.lengths_q[b] > 0:
            edge += [wl.cu_q[b], wl.cu_q[b + 1] - 1]
    toks.append(np.array(edge, dtype=np.int64))
    t = np.concatenate(toks)
    h = rng.integers(0, wl.H, len(t))
    return np.stack([t, h], axis=1)
