"""Python side of the fp64 CPU oracle (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product package never does.

``attention_rows`` wraps ``varlen_oracle.c`` (built with gcc into
``liboracle_varlen.so`` next to this file).  That C file is the plain
definition of the packed attention forward pass of boostr 0.2.0
varlen_attention.rs (VarLenAttentionOps, "Layout contract") computed per
(token, head) row in fp64, following realizar 0.8.4 attention.rs IMP-111
(standard_single_head_attention / standard_softmax); see its header for the
readings taken where the pages are silent.

``attention_rows_fp8`` is the same definition for E4M3 inputs with
per-tensor dequantization scales (boostr flash.rs,
FlashAttentionOps::flash_attention_fwd_fp8); ``e4m3_decode`` /
``e4m3_encode`` are the format's definition (round to nearest even,
saturating at +-448) written out in the same C file.

``attention_bwd`` is the backward pass of the same definition (dq, dk, dv of
sum(dout * out), boostr varlen_attention.rs VarLenAttentionOps::
varlen_attention_bwd), in fp64.

``schedule`` (in ``oracle/schedule.py``) is the CPU statement of the tile
work list the GPU scheduler must reproduce bit-exactly.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "varlen_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_varlen.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (no CUDA involved)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        fn = lib.oracle_varlen_attention_rows
        fn.restype = ctypes.c_int
        fn.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 6 + [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        f8 = lib.oracle_varlen_attention_rows_fp8
        f8.restype = ctypes.c_int
        f8.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_double] * 3 + [ctypes.c_void_p] * 2 + [
            ctypes.c_int] * 6 + [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64] + [
            ctypes.c_void_p] * 3 + [ctypes.c_int]
        bw = lib.oracle_varlen_attention_bwd
        bw.restype = ctypes.c_int
        bw.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 6 + [ctypes.c_void_p] * 3 + [ctypes.c_int]
        for name in ("oracle_e4m3_decode_array", "oracle_e4m3_encode_array"):
            getattr(lib, name).restype = None
            getattr(lib, name).argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64]
        _lib = lib
    return _lib


def _bits(x) -> np.ndarray:
    """bf16 tensor / uint16 array -> contiguous uint16 numpy array of bit patterns."""
    if hasattr(x, "dtype") and str(getattr(x, "dtype")) == "torch.bfloat16":
        import torch
        x = x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        raise TypeError("oracle inputs must be bf16 tensors or uint16 bit-pattern arrays")
    return x


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def attention_rows(q, k, v, cu_q: Sequence[int], cu_k: Sequence[int], H: int, H_kv: int,
                   D: int, causal: bool, window: int = 0,
                   rows: Optional[np.ndarray] = None, nthreads: Optional[int] = None,
                   seqused_k: Optional[Sequence[int]] = None):
    """fp64 output rows and logsumexp.

    q: [total_q, H, D] bf16; k, v: [total_k, H_kv, D] bf16 (torch bf16 or uint16 bits).
    rows: optional int array [n, 2] of (token, head) pairs; None = all rows.
    seqused_k: optional per-sequence key counts for a cache with a capacity
    stride (keys of sequence b: the first min(seqused_k[b], cu_k[b+1] - cu_k[b])
    rows from cu_k[b]); None = every row of the sequence's range.
    Returns (out [n, D] float64, lse [n] float64); with rows=None, shaped
    [total_q, H, D] and [total_q, H].
    """
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    cq = np.ascontiguousarray(np.asarray(cu_q, dtype=np.int32))
    ck = np.ascontiguousarray(np.asarray(cu_k, dtype=np.int32))
    batch = len(cq) - 1
    used_p = None
    if seqused_k is not None:
        used = np.ascontiguousarray(np.asarray(seqused_k, dtype=np.int32))
        if used.shape != (batch,):
            raise ValueError("seqused_k must hold one count per sequence")
        used_p = used.ctypes.data
    total_q = int(cq[-1])
    if rows is None:
        n = total_q * H
        tok_p = head_p = None
    else:
        rows = np.asarray(rows)
        tok = np.ascontiguousarray(rows[:, 0].astype(np.int64))
        hd = np.ascontiguousarray(rows[:, 1].astype(np.int32))
        n = len(tok)
        tok_p, head_p = tok.ctypes.data, hd.ctypes.data
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    rc = lib.oracle_varlen_attention_rows(
        qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, cq.ctypes.data, ck.ctypes.data, used_p,
        batch, H, H_kv, D, int(bool(causal)), int(window), tok_p, head_p, n,
        out.ctypes.data, lse.ctypes.data, int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_varlen_attention_rows failed with code {rc}")
    if rows is None:
        return out.reshape(total_q, H, D), lse.reshape(total_q, H)
    return out, lse


def _bytes(x) -> np.ndarray:
    """E4M3 tensor (torch.float8_e4m3fn or uint8 bits) -> contiguous uint8 numpy array."""
    if hasattr(x, "dtype") and "float8" in str(getattr(x, "dtype")):
        import torch
        x = x.detach().cpu().contiguous().view(torch.uint8).numpy()
    elif hasattr(x, "dtype") and str(getattr(x, "dtype")) == "torch.uint8":
        x = x.detach().cpu().contiguous().numpy()
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint8:
        raise TypeError("E4M3 inputs must be float8_e4m3fn tensors or uint8 bit-pattern arrays")
    return x


def e4m3_decode(bits) -> np.ndarray:
    """E4M3 bit patterns -> float64 values (NaN for the two NaN codes)."""
    b = _bytes(bits)
    out = np.empty(b.shape, dtype=np.float64)
    _load().oracle_e4m3_decode_array(b.ctypes.data, out.ctypes.data, b.size)
    return out


def e4m3_encode(x) -> np.ndarray:
    """float64 values -> nearest E4M3 bit patterns (ties to even, saturating at +-448)."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    out = np.empty(a.shape, dtype=np.uint8)
    _load().oracle_e4m3_encode_array(a.ctypes.data, out.ctypes.data, a.size)
    return out


def attention_rows_fp8(q, k, v, q_scale: float, k_scale: float, v_scale: float,
                       cu_q: Sequence[int], cu_k: Sequence[int], H: int, H_kv: int, D: int,
                       causal: bool, window: int = 0, rows: Optional[np.ndarray] = None,
                       nthreads: Optional[int] = None):
    """fp64 rows for E4M3 inputs: element value = decoded E4M3 * its tensor's scale.

    Returns (out, lse, err): out is the exact output before output quantization
    (divide by o_scale and apply ``e4m3_encode`` for the FP8 result), err the standard
    deviation scale of the error that rounding P to E4M3 may add to each output
    element (see the C file).  Shapes as in ``attention_rows``.
    """
    lib = _load()
    qb, kb, vb = _bytes(q), _bytes(k), _bytes(v)
    cq = np.ascontiguousarray(np.asarray(cu_q, dtype=np.int32))
    ck = np.ascontiguousarray(np.asarray(cu_k, dtype=np.int32))
    batch = len(cq) - 1
    total_q = int(cq[-1])
    if rows is None:
        n = total_q * H
        tok_p = head_p = None
    else:
        rows = np.asarray(rows)
        tok = np.ascontiguousarray(rows[:, 0].astype(np.int64))
        hd = np.ascontiguousarray(rows[:, 1].astype(np.int32))
        n = len(tok)
        tok_p, head_p = tok.ctypes.data, hd.ctypes.data
    out = np.zeros((n, D), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    err = np.zeros((n, D), dtype=np.float64)
    rc = lib.oracle_varlen_attention_rows_fp8(
        qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, float(q_scale), float(k_scale),
        float(v_scale), cq.ctypes.data, ck.ctypes.data, batch, H, H_kv, D, int(bool(causal)),
        int(window), tok_p, head_p, n, out.ctypes.data, lse.ctypes.data, err.ctypes.data,
        int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_varlen_attention_rows_fp8 failed with code {rc}")
    if rows is None:
        return out.reshape(total_q, H, D), lse.reshape(total_q, H), err.reshape(total_q, H, D)
    return out, lse, err


def attention_bwd(q, k, v, dout, cu_q: Sequence[int], cu_k: Sequence[int], H: int, H_kv: int,
                  D: int, causal: bool, window: int = 0, nthreads: Optional[int] = None):
    """fp64 gradients (dq [total_q, H, D], dk and dv [total_k, H_kv, D]) of
    sum(dout * out) for the forward above; inputs bf16 (torch or uint16 bits)."""
    lib = _load()
    qb, kb, vb, db = _bits(q), _bits(k), _bits(v), _bits(dout)
    cq = np.ascontiguousarray(np.asarray(cu_q, dtype=np.int32))
    ck = np.ascontiguousarray(np.asarray(cu_k, dtype=np.int32))
    batch = len(cq) - 1
    tq, tk = int(cq[-1]), int(ck[-1])
    dq = np.zeros((tq, H, D), dtype=np.float64)
    dk = np.zeros((tk, H_kv, D), dtype=np.float64)
    dv = np.zeros((tk, H_kv, D), dtype=np.float64)
    rc = lib.oracle_varlen_attention_bwd(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data,
                                         db.ctypes.data, cq.ctypes.data, ck.ctypes.data, batch,
                                         H, H_kv, D, int(bool(causal)), int(window),
                                         dq.ctypes.data, dk.ctypes.data, dv.ctypes.data,
                                         int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_varlen_attention_bwd failed with code {rc}")
    return dq, dk, dv
