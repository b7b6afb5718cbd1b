"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Bar (element by element): |O_gpu - O_oracle| <= 1e-2 (where |O_oracle| >= 4,
where no bf16 number need lie within 1e-2 of the exact value, half a bf16 step
+ 1e-3), |LSE_gpu - LSE_oracle| <= 1e-3, -inf logsumexp exactly where the
oracle has one, no NaN; the tile work list bit-exact against the CPU statement
in oracle/schedule.py.
"""
import numpy as np
import pytest
import torch

from variable_length_flash_varlen_b200 import binding, workloads
from tests._helpers import compare, oracle_all, run_gpu, sample_rows, to_device_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    binding.load()
    binding.device_status(clear=True)
    yield
    assert binding.device_status(clear=True) == 0, "device status word raised"


# --- reduced-size versions of the named workloads (full comparison) ------------

REDUCED = [("worked_example", 1.0), ("mha_noncausal", 0.15), ("gqa_causal", 0.05),
           ("sliding_window", 1 / 32), ("decode", 1 / 32), ("chunked_prefill", 0.1)]


@pytest.mark.parametrize("name,scale", REDUCED)
def test_reduced_workloads_match_oracle(oracle_lib, name, scale):
    wl = workloads.named(name, scale=scale)
    q, k, v = workloads.make_qkv(wl)
    out, lse = run_gpu(wl, q, k, v)
    ref_o, ref_l = oracle_all(oracle_lib, wl, q, k, v)
    compare(out, lse, ref_o, ref_l)


# --- edge cases ------------------------------------------------------------------

EDGE = [
    # lengths_q, lengths_k, H, H_kv, D, causal, window
    ([1, 127, 128, 129, 255, 256, 257, 1], None, 4, 1, 128, True, 0),
    ([1, 127, 128, 129, 255, 256, 257, 1], None, 4, 1, 128, False, 0),
    ([100, 5, 300], [300, 5, 130], 4, 2, 128, True, 0),     # L_q != L_k; empty rows
    ([100, 5, 300], [300, 5, 130], 4, 2, 128, False, 0),
    ([300, 200], [300, 200], 4, 4, 128, False, 37),          # window without causal
    ([300, 200], [300, 200], 2, 1, 64, True, 1000),          # window longer than sequence
    ([300, 200], [300, 200], 2, 1, 64, True, 1),             # window of one key
    ([0, 130, 0, 70, 3], [0, 130, 5, 70, 0], 2, 1, 128, True, 0),  # empty q / k sequences
    ([50], None, 2, 2, 128, False, 0),                       # total < one tile
    ([200, 333], None, 16, 2, 128, True, 0),                 # GQA group of 8
    ([129, 1000], None, 8, 8, 64, True, 96),                 # MHA, D=64, window
    ([2000], None, 2, 1, 128, True, 0),                      # many key tiles, rescale path
]


@pytest.mark.parametrize("case", EDGE)
def test_edge_cases_match_oracle(oracle_lib, case):
    Lq, Lk, H, Hkv, D, causal, W = case
    wl = workloads.custom(Lq, Lk if Lk is not None else Lq, H, Hkv, D, causal, W, seed=77)
    q, k, v = workloads.make_qkv(wl)
    out, lse = run_gpu(wl, q, k, v, path=binding.VA_PATH_PREFILL)
    ref_o, ref_l = oracle_all(oracle_lib, wl, q, k, v)
    compare(out, lse, ref_o, ref_l)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("tail", [1, 5, 8, 9, 63, 64, 120, 127])
def test_ragged_last_tile_matches_oracle(oracle_lib, tail, D):
    # the packed tensors end `tail` rows into a 128-row tile: the last query and
    # key tiles are copied as whole 8-row groups plus one partial group, the
    # rest of the tile zero (fewer than 8 rows: no whole group at all)
    L = [256, 128 + tail]
    for causal in (True, False):
        wl = workloads.custom(L, L, 4, 2, D, causal, 0, seed=100 + tail)
        q, k, v = workloads.make_qkv(wl)
        out, lse = run_gpu(wl, q, k, v, path=binding.VA_PATH_PREFILL)
        ref_o, ref_l = oracle_all(oracle_lib, wl, q, k, v)
        compare(out, lse, ref_o, ref_l)


def test_large_scores_stay_finite(oracle_lib):
    # scores spanning +-40 in base-e units exercise the reference-max update
    wl = workloads.custom([700, 300], [700, 300], 2, 1, 128, True, 0, seed=5)
    q, k, v = workloads.make_qkv(wl)
    q = (q.float() * 6).to(torch.bfloat16)
    out, lse = run_gpu(wl, q, k, v)
    ref_o, ref_l = oracle_all(oracle_lib, wl, q, k, v)
    compare(out, lse, ref_o, ref_l)


# --- invariants ------------------------------------------------------------------

def test_gqa_equals_repeated_kv_on_gpu():
    wl = workloads.custom([300, 129], [300, 129], 8, 2, 128, True, 0, seed=3)
    q, k, v = workloads.make_qkv(wl)
    out, lse = run_gpu(wl, q, k, v)
    wl2 = workloads.custom([300, 129], [300, 129], 8, 8, 128, True, 0, seed=3)
    out2, lse2 = run_gpu(wl2, q, k.repeat_interleave(4, dim=1), v.repeat_interleave(4, dim=1))
    # same tiles, same arithmetic: bitwise equal
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


def test_results_are_deterministic():
    wl = workloads.named("gqa_causal", scale=0.05)
    q, k, v = workloads.make_qkv(wl)
    dev = to_device_inputs(wl, q, k, v)
    a = run_gpu(wl, q, k, v, dev_inputs=dev)
    b = run_gpu(wl, q, k, v, dev_inputs=dev)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_host_buffer_entry_matches_device_entry():
    wl = workloads.named("worked_example")
    q, k, v = workloads.make_qkv(wl)
    out_d, lse_d = run_gpu(wl, q, k, v)
    out_h = torch.empty_like(q).pin_memory()
    lse_h = torch.empty(wl.total_q, wl.H, dtype=torch.float32).pin_memory()
    cq = torch.tensor(wl.cu_q, dtype=torch.int32)
    ck = torch.tensor(wl.cu_k, dtype=torch.int32)
    binding.varlen_attention_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), cq, ck,
                                      wl.batch, wl.H, wl.H_kv, wl.max_seqlen_q, wl.max_seqlen_k,
                                      wl.D, wl.causal, wl.window, out_h, lse_h)
    assert torch.equal(out_h, out_d.cpu()) and torch.equal(lse_h, lse_d.cpu())


def test_validate_cu_seqlens_device_array_matches_host_array():
    for cu, max_len, ok in (([0, 512, 812, 940], 512, True), ([0, 512, 500, 940], 512, False)):
        host = torch.tensor(cu, dtype=torch.int32)
        dev = host.cuda()
        for t in (host, dev):
            if ok:
                binding.validate_cu_seqlens(t, 3, max_len, 940)
            else:
                with pytest.raises(binding.VarlenAttentionError) as e:
                    binding.validate_cu_seqlens(t, 3, max_len, 940)
                assert "decreases at entry 2" in str(e.value)


def test_host_buffer_entry_pipelined_chunks_match_device_entry():
    # inputs above the pipelining threshold: the host entry splits the batch
    # into chunks of whole sequences, each copied in, computed and copied out
    # on its own; every sequence's result is independent of the launch that
    # computes it, so the results are bit-identical to the device entry's
    wl = workloads.named("mha_noncausal", scale=0.5)
    q, k, v = workloads.make_qkv(wl)
    assert (q.numel() + k.numel() + v.numel()) * 2 >= 8 << 20
    out_d, lse_d = run_gpu(wl, q, k, v)
    out_h = torch.full_like(q, float("nan")).pin_memory()
    lse_h = torch.full((wl.total_q, wl.H), float("nan"), dtype=torch.float32).pin_memory()
    cq = torch.tensor(wl.cu_q, dtype=torch.int32)
    ck = torch.tensor(wl.cu_k, dtype=torch.int32)
    binding.varlen_attention_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), cq, ck,
                                      wl.batch, wl.H, wl.H_kv, wl.max_seqlen_q, wl.max_seqlen_k,
                                      wl.D, wl.causal, wl.window, out_h, lse_h)
    assert torch.equal(out_h, out_d.cpu()) and torch.equal(lse_h, lse_d.cpu())


# Sequences longer than a pipelined chunk are cut into pieces of whole 256-row
# query blocks, each launched with only the keys its rows can see (below a
# window, rounded down to a 128-key tile; up to the last row's diagonal when
# causal or windowed): the same blocks, key tiles and masks as one launch, so
# bit-identical.  Shapes cover causal with fewer and with more queries than
# keys, a window with and without causal, and a non-causal piece (every key).
PIECE_CASES = {
    "sliding_window_quarter": lambda: workloads.named("sliding_window", scale=0.25),
    "noncausal_long": lambda: workloads.custom([10000, 500], [10000, 500], 8, 8, 128, False, 0, seed=21),
    "causal_fewer_queries": lambda: workloads.custom([9000, 100], [12000, 300], 8, 4, 128, True, 0, seed=22),
    "causal_more_queries": lambda: workloads.custom([9000], [6000], 8, 8, 128, True, 0, seed=23),
    "window_noncausal": lambda: workloads.custom([20000], [20000], 8, 8, 128, False, 1000, seed=24),
    "window_fewer_queries": lambda: workloads.custom([9000], [15000], 8, 2, 64, True, 777, seed=25),
    "gqa_causal": lambda: workloads.named("gqa_causal"),
}


@pytest.mark.parametrize("case", sorted(PIECE_CASES))
def test_host_buffer_entry_pieces_match_device_entry(case):
    wl = PIECE_CASES[case]()
    assert max(wl.lengths_q) > 4096  # at least one sequence is cut into pieces
    q, k, v = workloads.make_qkv(wl)
    out_d, lse_d = run_gpu(wl, q, k, v)
    out_h = torch.full_like(q, float("nan")).pin_memory()
    lse_h = torch.full((wl.total_q, wl.H), float("nan"), dtype=torch.float32).pin_memory()
    cq = torch.tensor(wl.cu_q, dtype=torch.int32)
    ck = torch.tensor(wl.cu_k, dtype=torch.int32)
    binding.varlen_attention_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), cq, ck,
                                      wl.batch, wl.H, wl.H_kv, wl.max_seqlen_q, wl.max_seqlen_k,
                                      wl.D, wl.causal, wl.window, out_h, lse_h)
    assert torch.equal(out_h, out_d.cpu()), f"{case}: outputs differ"
    assert torch.equal(lse_h, lse_d.cpu()), f"{case}: logsumexp differs"


# --- decode path -------------------------------------------------------------------

@pytest.mark.parametrize("split_keys", [32, 100, 448, 1024, 5000])
def test_decode_split_invariance(oracle_lib, split_keys):
    wl = workloads.named("decode", scale=1 / 32)
    q, k, v = workloads.make_qkv(wl)
    out, lse = run_gpu(wl, q, k, v, path=binding.VA_PATH_DECODE, split_keys=split_keys)
    ref_o, ref_l = oracle_all(oracle_lib, wl, q, k, v)
    compare(out, lse, ref_o, ref_l)


def test_decode_equals_prefill_path_and_causal_noop(oracle_lib):
    wl = workloads.custom([1, 1, 0, 1, 1], [700, 1, 5, 0, 2000], 8, 2, 128, False, 0, seed=21)
    q, k, v = workloads.make_qkv(wl)
    ref_o, ref_l = oracle_all(oracle_lib, wl, q, k, v)
    d = run_gpu(wl, q, k, v, path=binding.VA_PATH_DECODE)
    p = run_gpu(wl, q, k, v, path=binding.VA_PATH_PREFILL)
    compare(*d, ref_o, ref_l)
    compare(*p, ref_o, ref_l)
    wl_c = workloads.custom([1, 1, 0, 1, 1], [700, 1, 5, 0, 2000], 8, 2, 128, True, 0, seed=21)
    c = run_gpu(wl_c, q, k, v, path=binding.VA_PATH_DECODE)
    assert torch.equal(c[0], d[0]) and torch.equal(c[1], d[1])


DECODE_EDGE = [
    # lengths_k, H, H_kv, D, causal: GQA groups of 1, 6, 16 and 32 heads (the
    # last spans two head groups of a KV head), D = 64, a packed K/V shorter
    # than one 64-key tile, empty key sequences
    ([40, 1, 63], 4, 4, 128, False),
    ([900, 2100, 130, 4097], 12, 2, 64, False),
    ([1500, 3000, 0], 32, 2, 128, False),
    ([1500, 777], 64, 2, 128, True),
    ([20, 0, 7], 8, 2, 64, True),
]


@pytest.mark.parametrize("case", DECODE_EDGE)
def test_decode_edge_cases(oracle_lib, case):
    Lk, H, Hkv, D, causal = case
    wl = workloads.custom([1] * len(Lk), Lk, H, Hkv, D, causal, 0, seed=41)
    q, k, v = workloads.make_qkv(wl)
    ref_o, ref_l = oracle_all(oracle_lib, wl, q, k, v)
    for split in (0, 64):
        out, lse = run_gpu(wl, q, k, v, path=binding.VA_PATH_DECODE, split_keys=split)
        compare(out, lse, ref_o, ref_l)


@pytest.mark.parametrize("tail", [1, 7, 8, 15, 56, 63])
def test_decode_ragged_last_tile(oracle_lib, tail):
    # the packed keys end `tail` rows into a 64-key tile of the decode stream
    Lk = [640, 320 + tail]
    for D in (64, 128):
        wl = workloads.custom([1, 1], Lk, 8, 2, D, False, 0, seed=200 + tail)
        q, k, v = workloads.make_qkv(wl)
        ref_o, ref_l = oracle_all(oracle_lib, wl, q, k, v)
        for split in (0, 64):
            out, lse = run_gpu(wl, q, k, v, path=binding.VA_PATH_DECODE, split_keys=split)
            compare(out, lse, ref_o, ref_l)


def test_decode_large_scores(oracle_lib):
    # scores spanning about +-40 move the running max on many tiles
    wl = workloads.custom([1] * 3, [3000, 1700, 65], 8, 2, 128, False, 0, seed=43)
    q, k, v = workloads.make_qkv(wl)
    q = (q.float() * 6).to(torch.bfloat16)
    out, lse = run_gpu(wl, q, k, v, path=binding.VA_PATH_DECODE, split_keys=1024)
    ref_o, ref_l = oracle_all(oracle_lib, wl, q, k, v)
    compare(out, lse, ref_o, ref_l)


@pytest.mark.parametrize("W", [1, 300, 5000])
def test_decode_window(oracle_lib, W):
    wl = workloads.custom([1] * 6, [1, 50, 700, 1500, 3000, 10], 4, 1, 64, True, W, seed=31)
    q, k, v = workloads.make_qkv(wl)
    out, lse = run_gpu(wl, q, k, v, path=binding.VA_PATH_DECODE)
    ref_o, ref_l = oracle_all(oracle_lib, wl, q, k, v)
    compare(out, lse, ref_o, ref_l)


# --- tile work list bit-exact ----------------------------------------------------------

SCHED_CASES = [(n, 1.0) for n in workloads.WORKLOAD_SEEDS] + [("gqa_causal", 0.3)]


@pytest.mark.parametrize("name,scale", SCHED_CASES)
def test_schedule_bit_exact(name, scale):
    from oracle import schedule as sch
    wl = workloads.named(name, scale=scale)
    cq = torch.tensor(wl.cu_q, dtype=torch.int32, device="cuda")
    ck = torch.tensor(wl.cu_k, dtype=torch.int32, device="cuda")
    cap = wl.batch * ((wl.max_seqlen_q + 255) // 256)
    got = binding.varlen_attention_schedule(cq, ck, wl.batch, wl.max_seqlen_q, wl.causal,
                                            wl.window, cap).cpu().numpy()
    want = np.array(sch.schedule(wl.cu_q, wl.cu_k, wl.causal, wl.window), dtype=np.int32)
    assert got.shape == want.shape and np.array_equal(got, want)


def test_schedule_edge_lists_bit_exact():
    from oracle import schedule as sch
    for Lq, Lk, causal, W in [([0, 130, 0, 70, 3], [0, 130, 5, 70, 0], True, 0),
                              ([100, 5, 300], [300, 5, 130], True, 0),
                              ([1000, 300], [1000, 300], False, 200)]:
        cq = torch.tensor(workloads.cu_seqlens(Lq), dtype=torch.int32, device="cuda")
        ck = torch.tensor(workloads.cu_seqlens(Lk), dtype=torch.int32, device="cuda")
        cap = len(Lq) * ((max(Lq) + 255) // 256)
        got = binding.varlen_attention_schedule(cq, ck, len(Lq), max(Lq), causal, W, cap)
        want = sch.schedule(workloads.cu_seqlens(Lq), workloads.cu_seqlens(Lk), causal, W)
        assert [tuple(r) for r in got.cpu().tolist()] == want


@pytest.mark.parametrize("batch,seed", [(12000, 1), (21000, 2)])
def test_schedule_bit_exact_beyond_one_sorted_run(batch, seed):
    # more query blocks than one shared-memory sort holds (16384): runs sorted
    # in shared memory, then merged in global memory (one merge pass, with the
    # runs sorted in place, and two passes)
    import random
    from oracle import schedule as sch
    rng = random.Random(seed)
    Lq = [rng.randint(1, 700) for _ in range(batch)]
    Lk = [x + rng.randint(0, 300) for x in Lq]
    cu_q, cu_k = workloads.cu_seqlens(Lq), workloads.cu_seqlens(Lk)
    cq = torch.tensor(cu_q, dtype=torch.int32, device="cuda")
    ck = torch.tensor(cu_k, dtype=torch.int32, device="cuda")
    cap = batch * ((max(Lq) + 255) // 256)
    got = binding.varlen_attention_schedule(cq, ck, batch, max(Lq), True, 300, cap).cpu().numpy()
    want = np.array(sch.schedule(cu_q, cu_k, True, 300), dtype=np.int32)
    assert want.shape[0] > 16384
    assert got.shape == want.shape and np.array_equal(got, want)


def test_schedule_overflow_is_reported():
    cq = torch.tensor([0, 600], dtype=torch.int32, device="cuda")
    got = binding.varlen_attention_schedule(cq, cq, 1, 600, True, 0, capacity=2)
    assert got.shape[0] == 0
    assert binding.device_status(clear=True) == binding.VA_STATUS_SCHEDULE_OVERFLOW


# --- full-size workloads, launch configuration of the benchmark, sampled rows -------

@pytest.mark.parametrize("name", list(workloads.WORKLOAD_SEEDS))
def test_full_size_sampled_rows(oracle_lib, name):
    wl = workloads.named(name)
    q, k, v = workloads.make_qkv(wl)
    out, lse = run_gpu(wl, q, k, v)
    rows = sample_rows(wl, 256, seed=1)
    ref_o, ref_l = oracle_lib.attention_rows(q, k, v, wl.cu_q, wl.cu_k, wl.H, wl.H_kv, wl.D,
                                             wl.causal, wl.window, rows=rows)
    compare(out, lse, ref_o, ref_l, rows=rows)
    # every row written: no NaN left from the NaN-filled output buffers
    assert not torch.isnan(out).any() and not torch.isnan(lse).any()


# --- launch counts (the bench reports the counter's difference over its timed loops) ----------

def test_launch_counter_counts_each_entry_points_kernels():
    def launched(fn):
        n0 = binding.launch_count()
        fn()
        torch.cuda.synchronize()
        return binding.launch_count() - n0

    wl = workloads.named("worked_example")  # bf16 prefill: schedule build, residual and main variant
    q, k, v = workloads.make_qkv(wl)
    dev = to_device_inputs(wl, q, k, v)
    assert launched(lambda: run_gpu(wl, q, k, v, dev_inputs=dev)) == 3
    out, lse = run_gpu(wl, q, k, v, dev_inputs=dev)
    dq_, dk_, dv_, cq, ck = dev
    do = torch.randn_like(dq_)
    # backward: two list builds, dQ, dK/dV
    assert launched(lambda: binding.varlen_attention_bwd(do, dq_, dk_, dv_, out, lse, cq, ck, wl.batch, wl.H,
                                                         wl.H_kv, wl.max_seqlen_q, wl.max_seqlen_k, wl.D,
                                                         wl.causal, wl.window)) == 4
    dwl = workloads.named("decode", scale=1 / 32)  # decode: stream and combine
    qd, kd, vd = workloads.make_qkv(dwl)
    ddev = to_device_inputs(dwl, qd, kd, vd)
    assert launched(lambda: run_gpu(dwl, qd, kd, vd, dev_inputs=ddev)) == 2
    fwl = workloads.named("mha_noncausal", scale=0.1)  # E4M3: schedule build and the one variant
    q8, k8, v8, sc = workloads.make_qkv_fp8(fwl)
    fcq = torch.tensor(fwl.cu_q, dtype=torch.int32, device="cuda")
    fck = torch.tensor(fwl.cu_k, dtype=torch.int32, device="cuda")
    q8d, k8d, v8d = q8.cuda(), k8.cuda(), v8.cuda()
    assert launched(lambda: binding.varlen_attention_fwd_fp8(
        q8d, k8d, v8d, fcq, fck, fwl.batch, fwl.H, fwl.H_kv, fwl.max_seqlen_q, fwl.max_seqlen_k, fwl.D,
        fwl.causal, fwl.window, sc["q_scale"], sc["k_scale"], sc["v_scale"], sc["o_scale"])) == 2
    assert binding.device_status(clear=True) == 0
