"""Host-side checks of the C ABI that need no GPU: the library builds, loads,
exports every entry point include/varlen_attn.h declares, and rejects bad
arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

from variable_length_flash_varlen_b200 import binding, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "varlen_attn.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(varlen_attention_\w+)\s*\(", text)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    assert "varlen_attention_fwd" in names
    assert set(names) == set(binding.SIGNATURES), "binding and header disagree"


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.varlen_attention_version() == 100


def _call(lib, **over):
    a = dict(q=16, k=16, v=16, cq=16, ck=16, batch=1, H=4, Hkv=2, mq=8, mk=8, D=64,
             causal=1, window=0, out=16, lse=16)
    a.update(over)
    return lib.varlen_attention_fwd(a["q"], a["k"], a["v"], a["cq"], a["ck"], a["batch"], a["H"],
                                    a["Hkv"], a["mq"], a["mk"], a["D"], a["causal"], a["window"],
                                    a["out"], a["lse"], None)


@pytest.mark.parametrize("over,code,needle", [
    (dict(H=4, Hkv=3), -1, "multiple"),
    (dict(D=96), -2, "head_dim"),
    (dict(batch=-1), -1, "batch"),
    (dict(window=-2), -1, "window"),
    (dict(Hkv=0), -1, "num_kv_heads"),
    (dict(q=None), -1, "q is NULL"),
    (dict(lse=None), -1, "lse is NULL"),
    (dict(out=8), -1, "aligned"),
    (dict(mq=-1), -1, "max_seqlen"),
])
def test_invalid_arguments_rejected_without_gpu(lib, over, code, needle):
    rc = _call(lib, **over)
    assert rc == code
    assert needle in lib.varlen_attention_last_error().decode()


def test_empty_batch_is_noop(lib):
    assert _call(lib, batch=0, q=None, k=None, v=None, out=None, lse=None) == 0
    assert _call(lib, mq=0, q=None, k=None, v=None, out=None, lse=None) == 0
    assert lib.varlen_attention_last_error().decode() == ""


def test_decode_split_keys_range_checked(lib):
    f = lib.varlen_attention_fwd_ex
    rc = f(16, 16, 16, 16, 16, 1, 4, 2, 8, 8, 64, 0, 0, 16, 16, 9, 0, None)
    assert rc == -1 and "path" in lib.varlen_attention_last_error().decode()
    rc = f(16, 16, 16, 16, 16, 1, 4, 2, 8, 8, 64, 0, 0, 16, 16, 2, 0, None)
    assert rc == -1 and "max_seqlen_q" in lib.varlen_attention_last_error().decode()


def test_kvcache_entry_requires_seqused_without_gpu(lib):
    rc = lib.varlen_attention_fwd_kvcache(16, 16, 16, 16, 16, None, 1, 4, 2, 8, 8, 64, 1, 0, 16, 16,
                                          None)
    assert rc == -1
    assert b"seqused_k is NULL" in lib.varlen_attention_last_error()


@pytest.mark.parametrize("cu,batch,max_len,total,needle", [
    ([0, 512, 812, 940], 3, 512, 940, None),        # the worked example's offsets
    ([0, 512, 812, 940], 3, 512, -1, None),         # total not checked
    ([0, 0, 7, 7], 3, 7, 7, None),                  # empty sequences
    ([0], 0, 0, 0, None),                           # empty batch
    ([1, 512, 812, 940], 3, 512, -1, "cu_seqlens[0] = 1"),
    ([0, 512, 500, 940], 3, 512, -1, "decreases at entry 2"),
    ([0, 512, 812, 940], 3, 511, -1, "sequence 0 has length 512"),
    ([0, 512, 812, 940], 3, 512, 941, "expected the total 941"),
])
def test_validate_cu_seqlens_host_arrays(lib, cu, batch, max_len, total, needle):
    import torch
    t = torch.tensor(cu + [-5], dtype=torch.int32)   # a trailing entry the check must not read
    rc = lib.varlen_attention_validate_cu_seqlens(t.data_ptr(), batch, max_len, total, 0, None)
    if needle is None:
        assert rc == 0, lib.varlen_attention_last_error().decode()
        binding.validate_cu_seqlens(t, batch, max_len, total)
    else:
        assert rc == -1
        assert needle in lib.varlen_attention_last_error().decode()
        with pytest.raises(binding.VarlenAttentionError):
            binding.validate_cu_seqlens(t, batch, max_len, total)


def test_validate_cu_seqlens_rejects_bad_arguments(lib):
    assert lib.varlen_attention_validate_cu_seqlens(None, 1, 8, -1, 0, None) == -1
    assert b"NULL" in lib.varlen_attention_last_error()
    import torch
    t = torch.tensor([0, 4], dtype=torch.int32)
    assert lib.varlen_attention_validate_cu_seqlens(t.data_ptr(), -1, 8, -1, 0, None) == -1
    assert lib.varlen_attention_validate_cu_seqlens(t.data_ptr(), 1, -1, -1, 0, None) == -1


@pytest.mark.parametrize("cq,ck,needle", [
    ([0, 512, 500, 940], [0, 512, 812, 940], "cu_seqlens_q decreases at entry 2"),
    ([0, 512, 812, 940], [3, 512, 812, 940], "cu_seqlens_k[0] = 3, must be 0"),
    ([0, 600, 812, 940], [0, 512, 812, 940], "sequence 0 has length 600 > max_seqlen 512"),
    ([0, 512, 812, 940], [0, 512, 812, 700], "cu_seqlens_k decreases at entry 3"),
])
def test_host_entry_rejects_bad_host_cu_seqlens_before_device_work(lib, cq, ck, needle):
    # the host-buffer entry sizes its copies and chunks from these host arrays:
    # a bad one is refused before any CUDA call (this runs without a GPU; the
    # tensor pointers are never dereferenced)
    import torch
    tq = torch.tensor(cq, dtype=torch.int32)
    tk = torch.tensor(ck, dtype=torch.int32)
    rc = lib.varlen_attention_fwd_host(16, 16, 16, tq.data_ptr(), tk.data_ptr(), 3, 4, 2, 512, 512,
                                       64, 1, 0, 16, 16, None)
    assert rc == -1
    assert needle in lib.varlen_attention_last_error().decode()


def test_sync_status_rejects_null_pointer(lib):
    assert lib.varlen_attention_sync_status(None, None, 0) == -1
    assert b"status is NULL" in lib.varlen_attention_last_error()


def test_launch_count_is_a_plain_counter(lib):
    # no device work is needed to read it; nothing was launched by these host-only tests
    lib.varlen_attention_launch_count.restype = ctypes.c_ulonglong
    n = lib.varlen_attention_launch_count()
    assert n == lib.varlen_attention_launch_count()
