"""Pins for the FP8 part of the fp64 oracle (CPU only).

The FP8 forward (boostr flash.rs, FlashAttentionOps::flash_attention_fwd_fp8:
dequantization scales q/k/v_scale, output scale o_scale, FP32
accumulation) adds three things to the oracle, each checked here against
something other than itself:
  * the E4M3 codec: every one of the 256 codes against torch's
    float8_e4m3fn conversion (a library routine) and against values fixed by
    the format's definition; rounding ties and saturation by construction;
  * the attention rows for E4M3 inputs: with the scales applied they must
    equal, bit for bit, the already pinned bf16 oracle on the same values
    (every E4M3 value times a power of two is a bf16 number);
  * the per-element scale of the error that rounding P to E4M3 may add: its
    closed form when every visible score is equal (zero Q), and for a single
    visible key.
"""
import math

import numpy as np
import pytest
import torch

from variable_length_flash_varlen_b200 import workloads


def test_e4m3_decode_all_codes_match_torch(oracle_lib):
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle_lib.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])


def test_e4m3_decode_definition_values(oracle_lib):
    # sign / 4-bit exponent (bias 7) / 3-bit mantissa; exponent 0 is subnormal
    want = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6,
            0x38: 1.0, 0x39: 1.125, 0x3F: 1.875, 0x40: 2.0, 0x7E: 448.0,
            0xB8: -1.0, 0xFE: -448.0, 0x80: -0.0}
    got = oracle_lib.e4m3_decode(np.array(list(want), dtype=np.uint8))
    assert list(got) == list(want.values())
    nan = oracle_lib.e4m3_decode(np.array([0x7F, 0xFF], dtype=np.uint8))
    assert np.isnan(nan).all()


def test_e4m3_encode_round_trip_ties_and_saturation(oracle_lib):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF, 0x80)], dtype=np.uint8)
    vals = oracle_lib.e4m3_decode(codes)
    assert np.array_equal(oracle_lib.e4m3_encode(vals), codes)
    # midpoints between neighbouring positive values go to the even code
    pos = np.arange(0x00, 0x7E, dtype=np.uint8)
    lo, hi = oracle_lib.e4m3_decode(pos), oracle_lib.e4m3_decode(pos + 1)
    mid = oracle_lib.e4m3_encode((lo + hi) / 2)
    assert np.array_equal(mid, np.where(pos % 2 == 0, pos, pos + 1).astype(np.uint8))
    # beyond the largest finite value: saturation (the reading taken for o_scale)
    big = oracle_lib.e4m3_encode(np.array([448.0, 463.9, 464.0, 1e6, -1e6]))
    assert list(big) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


def test_e4m3_encode_matches_torch_in_range(oracle_lib):
    x = np.random.default_rng(3).normal(size=200000) * np.exp(np.random.default_rng(4).uniform(-12, 5, 200000))
    x = np.clip(x, -448, 448)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle_lib.e4m3_encode(x)
    # torch and the definition agree except on the sign of a zero result
    both_zero = (oracle_lib.e4m3_decode(got) == 0) & (oracle_lib.e4m3_decode(ref) == 0)
    assert np.array_equal(got[~both_zero], ref[~both_zero])


FP8_CASES = [
    # lengths_q, lengths_k, H, H_kv, causal, window
    ([130, 7, 260], [130, 7, 260], 4, 2, True, 0),
    ([64, 200], [300, 200], 2, 1, False, 0),
    ([300, 90], [300, 90], 4, 4, True, 50),
]


@pytest.mark.parametrize("case", FP8_CASES)
def test_fp8_rows_equal_bf16_rows_on_the_same_values(oracle_lib, case):
    Lq, Lk, H, Hkv, causal, W = case
    wl = workloads.custom(Lq, Lk, H, Hkv, 128, causal, W, seed=61)
    q8, k8, v8, sc = workloads.make_qkv_fp8(wl)
    out8, lse8, _ = oracle_lib.attention_rows_fp8(q8, k8, v8, sc["q_scale"], sc["k_scale"],
                                                  sc["v_scale"], wl.cu_q, wl.cu_k, wl.H, wl.H_kv,
                                                  wl.D, wl.causal, wl.window, nthreads=4)

    def as_bf16(t, s):  # E4M3 value * 2^-6 is exactly a bf16 number
        x = torch.from_numpy(oracle_lib.e4m3_decode(t.numpy()) * s).to(torch.float32)
        assert torch.equal(x.to(torch.bfloat16).to(torch.float32), x)
        return x.to(torch.bfloat16)

    qb, kb, vb = as_bf16(q8, sc["q_scale"]), as_bf16(k8, sc["k_scale"]), as_bf16(v8, sc["v_scale"])
    out, lse = oracle_lib.attention_rows(qb, kb, vb, wl.cu_q, wl.cu_k, wl.H, wl.H_kv, wl.D,
                                         wl.causal, wl.window, nthreads=4)
    assert np.array_equal(out8, out) and np.array_equal(lse8, lse)


def test_fp8_error_scale_closed_form_equal_scores(oracle_lib):
    # Q = 0: every visible score is 0, every p_j = 1 (the row maximum), so each
    # key's rounding bound is 2^-4 and err_d = sqrt(sum_j v_jd^2 * 2^-8 / 3) / n
    L = [5, 40]
    wl = workloads.custom(L, L, 2, 1, 128, True, 0, seed=62)
    _, k8, v8, sc = workloads.make_qkv_fp8(wl)
    q8 = torch.zeros((wl.total_q, wl.H, wl.D), dtype=torch.uint8)
    out, lse, err = oracle_lib.attention_rows_fp8(q8, k8, v8, 1.0, sc["k_scale"], sc["v_scale"],
                                                  wl.cu_q, wl.cu_k, wl.H, wl.H_kv, wl.D,
                                                  wl.causal, wl.window, nthreads=2)
    v = oracle_lib.e4m3_decode(v8.numpy()) * sc["v_scale"]
    for b, Lb in enumerate(L):
        for i in range(Lb):
            t = wl.cu_q[b] + i
            vis = v[wl.cu_k[b]:wl.cu_k[b] + i + 1, 0, :]          # causal: keys 0..i
            n = i + 1
            for h in range(wl.H):
                want = np.sqrt((vis ** 2).sum(axis=0) * 2.0 ** -8 / 3) / n
                assert np.allclose(err[t, h], want, rtol=1e-12, atol=0)
                assert np.allclose(out[t, h], vis.mean(axis=0), rtol=1e-12, atol=1e-15)
                assert lse[t, h] == pytest.approx(math.log(n), abs=1e-12)


def test_fp8_error_scale_single_key(oracle_lib):
    wl = workloads.custom([1, 1], [1, 1], 2, 2, 128, False, 0, seed=63)
    q8, k8, v8, sc = workloads.make_qkv_fp8(wl)
    out, _, err = oracle_lib.attention_rows_fp8(q8, k8, v8, sc["q_scale"], sc["k_scale"],
                                                sc["v_scale"], wl.cu_q, wl.cu_k, wl.H, wl.H_kv,
                                                wl.D, wl.causal, wl.window, nthreads=1)
    v = oracle_lib.e4m3_decode(v8.numpy()) * sc["v_scale"]
    assert np.array_equal(out, v)                  # one key: O is that V row
    assert np.allclose(err, np.abs(v) * 2.0 ** -4 / math.sqrt(3), rtol=1e-15, atol=0)
