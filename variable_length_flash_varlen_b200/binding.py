"""ctypes binding of ``libvarlen_attn.so`` (argument marshalling only).

Every function here takes torch tensors, checks dtypes / shapes / devices and
passes raw pointers to the C entry point of the same name declared in
``include/varlen_attn.h``.  No arithmetic happens on the Python side and
there is no fallback: if the library is missing, ``load()`` raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libvarlen_attn.so")

VA_OK = 0
VA_ERR_INVALID_ARG, VA_ERR_UNSUPPORTED, VA_ERR_CUDA, VA_ERR_DEVICE_TIMEOUT = -1, -2, -3, -4
VA_PATH_AUTO, VA_PATH_PREFILL, VA_PATH_DECODE = 0, 1, 2
VA_STATUS_WAIT_TIMEOUT = 1
VA_STATUS_SCHEDULE_OVERFLOW = 2
VA_STATUS_SMEM_ALIGN = 4

# every symbol the header declares, with its ctypes signature
_P, _I = ctypes.c_void_p, ctypes.c_int
SIGNATURES = {
    "varlen_attention_fwd": (_I, [_P, _P, _P, _P, _P] + [_I] * 8 + [_P, _P, _P]),
    "varlen_attention_fwd_ex": (_I, [_P, _P, _P, _P, _P] + [_I] * 8 + [_P, _P, _I, _I, _P]),
    "varlen_attention_fwd_kvcache": (_I, [_P, _P, _P, _P, _P, _P] + [_I] * 8 + [_P, _P, _P]),
    "varlen_attention_fwd_fp8": (_I, [_P, _P, _P, _P, _P] + [_I] * 8 + [ctypes.c_float] * 4
                                 + [_P, _P, _P]),
    "varlen_attention_bwd": (_I, [_P] * 8 + [_I] * 8 + [_P] * 4),
    "varlen_attention_fwd_host": (_I, [_P, _P, _P, _P, _P] + [_I] * 8 + [_P, _P, _P]),
    "varlen_attention_fwd_noalloc": (_I, [_P, _P, _P, _P, _P] + [_I] * 8 + [_P, _P, _P]),
    "varlen_attention_schedule": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _I, _P]),
    "varlen_attention_host_chunks": (_I, [_P, _P, _I, _I, _I, ctypes.c_longlong, _P, _I, _P]),
    "varlen_attention_device_status": (_I, [ctypes.POINTER(ctypes.c_uint), _I]),
    "varlen_attention_sync_status": (_I, [_P, ctypes.POINTER(ctypes.c_uint), _I]),
    "varlen_attention_validate_cu_seqlens": (_I, [_P, _I, _I, _I, _I, _P]),
    "varlen_attention_selftest_wait_timeout": (_I, [_P, _P]),
    "varlen_attention_last_error": (ctypes.c_char_p, []),
    "varlen_attention_version": (_I, []),
    "varlen_attention_launch_count": (ctypes.c_ulonglong, []),
}

_lib = None


class VarlenAttentionError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"{message} (code {code})")
        self.code = code


def load(path: Optional[str] = None):
    """Load the in-tree library (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise FileNotFoundError(
            f"{p} is missing: build it with `python -m variable_length_flash_varlen_b200.build`")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def _check(rc: int):
    if rc != VA_OK:
        raise VarlenAttentionError(rc, load().varlen_attention_last_error().decode())


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check_inputs(q, k, v, cu_q, cu_k, num_heads, num_kv_heads, head_dim, device_kind):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if t.device.type != device_kind:
            raise ValueError(f"{name} must be on {device_kind}")
    for name, t in (("cu_seqlens_q", cu_q), ("cu_seqlens_k", cu_k)):
        if t.dtype != torch.int32 or not t.is_contiguous() or t.device.type != device_kind:
            raise ValueError(f"{name} must be a contiguous int32 {device_kind} tensor")
    if q.dim() != 3 or q.shape[1:] != (num_heads, head_dim):
        raise ValueError("q must be [total_q, num_heads, head_dim]")
    if k.shape != v.shape or k.dim() != 3 or k.shape[1:] != (num_kv_heads, head_dim):
        raise ValueError("k and v must be [total_k, num_kv_heads, head_dim]")


def varlen_attention_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                         cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                         batch: int, num_heads: int, num_kv_heads: int,
                         max_seqlen_q: int, max_seqlen_k: int, head_dim: int,
                         causal: bool, window: int = 0,
                         out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                         stream: Optional[torch.cuda.Stream] = None,
                         path: int = VA_PATH_AUTO, decode_split_keys: int = 0
                         ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Packed attention forward on device tensors; returns (out, lse)."""
    lib = load()
    _check_inputs(q, k, v, cu_seqlens_q, cu_seqlens_k, num_heads, num_kv_heads, head_dim, "cuda")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[0], num_heads, dtype=torch.float32, device=q.device)
    if out.shape != q.shape or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 tensor shaped like q")
    if lse.shape != (q.shape[0], num_heads) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [total_q, num_heads] tensor")
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), cu_seqlens_q.data_ptr(),
            cu_seqlens_k.data_ptr(), batch, num_heads, num_kv_heads, max_seqlen_q, max_seqlen_k,
            head_dim, int(bool(causal)), int(window), out.data_ptr(), lse.data_ptr())
    if path == VA_PATH_AUTO and decode_split_keys == 0:
        rc = lib.varlen_attention_fwd(*args, _stream_ptr(stream))
    else:
        rc = lib.varlen_attention_fwd_ex(*args, int(path), int(decode_split_keys),
                                         _stream_ptr(stream))
    _check(rc)
    return out, lse


def _fp8_bytes(name: str, t: torch.Tensor) -> torch.Tensor:
    if t.dtype not in (torch.float8_e4m3fn, torch.uint8):
        raise TypeError(f"{name} must hold E4M3 values (torch.float8_e4m3fn or uint8 bit patterns)")
    if not t.is_contiguous() or t.device.type != "cuda":
        raise ValueError(f"{name} must be a contiguous cuda tensor")
    return t


def varlen_attention_fwd_fp8(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                             cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                             batch: int, num_heads: int, num_kv_heads: int,
                             max_seqlen_q: int, max_seqlen_k: int, head_dim: int,
                             causal: bool, window: int, q_scale: float, k_scale: float,
                             v_scale: float, o_scale: float,
                             out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                             stream: Optional[torch.cuda.Stream] = None
                             ) -> Tuple[torch.Tensor, torch.Tensor]:
    """FP8 (E4M3) packed attention forward with per-tensor scales; returns
    (out as E4M3 bytes [total_q, H, D] uint8, lse float32 [total_q, H])."""
    lib = load()
    for name, t in (("q", q), ("k", k), ("v", v)):
        _fp8_bytes(name, t)
    if q.dim() != 3 or q.shape[1:] != (num_heads, head_dim):
        raise ValueError("q must be [total_q, num_heads, head_dim]")
    if k.shape != v.shape or k.dim() != 3 or k.shape[1:] != (num_kv_heads, head_dim):
        raise ValueError("k and v must be [total_k, num_kv_heads, head_dim]")
    for name, t in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        if t.dtype != torch.int32 or not t.is_contiguous() or t.device.type != "cuda":
            raise ValueError(f"{name} must be a contiguous int32 cuda tensor")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.uint8, device=q.device)
    _fp8_bytes("out", out)
    if out.shape != q.shape:
        raise ValueError("out must be shaped like q")
    if lse is None:
        lse = torch.empty(q.shape[0], num_heads, dtype=torch.float32, device=q.device)
    if lse.shape != (q.shape[0], num_heads) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [total_q, num_heads] tensor")
    _check(lib.varlen_attention_fwd_fp8(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(),
        batch, num_heads, num_kv_heads, max_seqlen_q, max_seqlen_k, head_dim, int(bool(causal)),
        int(window), float(q_scale), float(k_scale), float(v_scale), float(o_scale),
        out.data_ptr(), lse.data_ptr(), _stream_ptr(stream)))
    return out, lse


def varlen_attention_bwd(dout: torch.Tensor, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                         out: torch.Tensor, lse: torch.Tensor, cu_seqlens_q: torch.Tensor,
                         cu_seqlens_k: torch.Tensor, batch: int, num_heads: int, num_kv_heads: int,
                         max_seqlen_q: int, max_seqlen_k: int, head_dim: int, causal: bool,
                         window: int = 0, dq: Optional[torch.Tensor] = None,
                         dk: Optional[torch.Tensor] = None, dv: Optional[torch.Tensor] = None,
                         stream: Optional[torch.cuda.Stream] = None):
    """Backward pass on device tensors; returns (dq, dk, dv) in bf16."""
    lib = load()
    _check_inputs(q, k, v, cu_seqlens_q, cu_seqlens_k, num_heads, num_kv_heads, head_dim, "cuda")
    for name, t, like in (("dout", dout, q), ("out", out, q)):
        if t.shape != like.shape or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 tensor shaped like q")
    if lse.shape != (q.shape[0], num_heads) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [total_q, num_heads] tensor")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t, like in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        if t.shape != like.shape or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 tensor shaped like its input")
    _check(lib.varlen_attention_bwd(
        dout.data_ptr(), q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
        cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), batch, num_heads, num_kv_heads,
        max_seqlen_q, max_seqlen_k, head_dim, int(bool(causal)), int(window), dq.data_ptr(),
        dk.data_ptr(), dv.data_ptr(), _stream_ptr(stream)))
    return dq, dk, dv


def varlen_attention_fwd_kvcache(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                 cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                                 seqused_k: torch.Tensor, batch: int, num_heads: int,
                                 num_kv_heads: int, max_seqlen_q: int, max_seqlen_k: int,
                                 head_dim: int, causal: bool, window: int = 0,
                                 out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                                 stream: Optional[torch.cuda.Stream] = None
                                 ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Attention over a capacity-strided key-value cache: sequence b's keys are the
    first seqused_k[b] rows of its slot cu_seqlens_k[b]..cu_seqlens_k[b+1]-1."""
    lib = load()
    _check_inputs(q, k, v, cu_seqlens_q, cu_seqlens_k, num_heads, num_kv_heads, head_dim, "cuda")
    if (seqused_k.dtype != torch.int32 or not seqused_k.is_contiguous()
            or seqused_k.device.type != "cuda" or seqused_k.shape != (batch,)):
        raise ValueError("seqused_k must be a contiguous int32 cuda tensor of shape [batch]")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[0], num_heads, dtype=torch.float32, device=q.device)
    if out.shape != q.shape or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 tensor shaped like q")
    if lse.shape != (q.shape[0], num_heads) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [total_q, num_heads] tensor")
    _check(lib.varlen_attention_fwd_kvcache(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(),
        seqused_k.data_ptr(), batch, num_heads, num_kv_heads, max_seqlen_q, max_seqlen_k, head_dim,
        int(bool(causal)), int(window), out.data_ptr(), lse.data_ptr(), _stream_ptr(stream)))
    return out, lse


def varlen_attention_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                 cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                                 batch: int, num_heads: int, num_kv_heads: int,
                                 max_seqlen_q: int, max_seqlen_k: int, head_dim: int,
                                 causal: bool, window: int, out: torch.Tensor, lse: torch.Tensor,
                                 stream: Optional[torch.cuda.Stream] = None):
    """The allocation-free entry point: the caller passes out and lse; the
    library's workspace is its static per-device scratch array."""
    lib = load()
    _check_inputs(q, k, v, cu_seqlens_q, cu_seqlens_k, num_heads, num_kv_heads, head_dim, "cuda")
    if out.shape != q.shape or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 tensor shaped like q")
    if lse.shape != (q.shape[0], num_heads) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [total_q, num_heads] tensor")
    _check(lib.varlen_attention_fwd_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(),
        batch, num_heads, num_kv_heads, max_seqlen_q, max_seqlen_k, head_dim, int(bool(causal)),
        int(window), out.data_ptr(), lse.data_ptr(), _stream_ptr(stream)))
    return out, lse


def varlen_attention_fwd_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                              cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor,
                              batch: int, num_heads: int, num_kv_heads: int,
                              max_seqlen_q: int, max_seqlen_k: int, head_dim: int,
                              causal: bool, window: int, out: torch.Tensor, lse: torch.Tensor,
                              stream: Optional[torch.cuda.Stream] = None):
    """Same operation on host (ideally pinned) tensors; blocks until out/lse are filled."""
    lib = load()
    _check_inputs(q, k, v, cu_seqlens_q, cu_seqlens_k, num_heads, num_kv_heads, head_dim, "cpu")
    if out.device.type != "cpu" or lse.device.type != "cpu":
        raise ValueError("out and lse must be host tensors")
    rc = lib.varlen_attention_fwd_host(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(),
        batch, num_heads, num_kv_heads, max_seqlen_q, max_seqlen_k, head_dim, int(bool(causal)),
        int(window), out.data_ptr(), lse.data_ptr(), _stream_ptr(stream))
    _check(rc)
    return out, lse


def varlen_attention_schedule(cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor, batch: int,
                              max_seqlen_q: int, causal: bool, window: int, capacity: int,
                              stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """The device-built query-tile list as an int32 [n, 4] tensor (b, qt, kt_lo, kt_hi)."""
    lib = load()
    tiles = torch.zeros(capacity, 4, dtype=torch.int32, device=cu_seqlens_q.device)
    n = torch.zeros(1, dtype=torch.int32, device=cu_seqlens_q.device)
    _check(lib.varlen_attention_schedule(cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), batch,
                                         max_seqlen_q, int(bool(causal)), int(window),
                                         tiles.data_ptr(), n.data_ptr(), capacity,
                                         _stream_ptr(stream)))
    torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
    return tiles[: int(n.item())]


def validate_cu_seqlens(cu_seqlens: torch.Tensor, batch: int, max_seqlen: int, total: int = -1,
                        stream: Optional[torch.cuda.Stream] = None) -> None:
    """Check a cu_seqlens array (int32, host or device) against the layout's
    preconditions; raises VarlenAttentionError naming the first bad entry."""
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_contiguous():
        raise ValueError("cu_seqlens must be a contiguous int32 tensor")
    if cu_seqlens.numel() < batch + 1:
        raise ValueError(f"cu_seqlens has {cu_seqlens.numel()} entries, batch {batch} needs {batch + 1}")
    on_device = cu_seqlens.is_cuda
    _check(load().varlen_attention_validate_cu_seqlens(
        cu_seqlens.data_ptr(), batch, max_seqlen, total, int(on_device),
        _stream_ptr(stream) if on_device else None))


HOST_CHUNK_FIELDS = ("piece", "b0", "b1", "q0", "q1", "k_base", "k_len", "kc0", "kc1")


def host_chunks(cu_seqlens_q, cu_seqlens_k, batch: int, causal: bool, window: int,
                input_bytes: int) -> List[dict]:
    """The copy/compute plan varlen_attention_fwd_host follows for these host
    cu_seqlens (no device work): one dict of HOST_CHUNK_FIELDS per chunk."""
    cq = torch.as_tensor(cu_seqlens_q, dtype=torch.int32).contiguous()
    ck = torch.as_tensor(cu_seqlens_k, dtype=torch.int32).contiguous()
    lib = load()
    n = ctypes.c_int(0)
    lib.varlen_attention_host_chunks(cq.data_ptr(), ck.data_ptr(), batch, int(causal), window,
                                     input_bytes, None, 0, ctypes.byref(n))
    buf = (ctypes.c_longlong * (9 * max(1, n.value)))()
    _check(lib.varlen_attention_host_chunks(cq.data_ptr(), ck.data_ptr(), batch, int(causal), window,
                                            input_bytes, buf, n.value, ctypes.byref(n)))
    return [dict(zip(HOST_CHUNK_FIELDS, buf[9 * c: 9 * c + 9])) for c in range(n.value)]


def launch_count() -> int:
    """Kernels the library has launched in this process so far (a diagnostic)."""
    return int(load().varlen_attention_launch_count())


def device_status(clear: bool = True) -> int:
    st = ctypes.c_uint(0)
    _check(load().varlen_attention_device_status(ctypes.byref(st), int(clear)))
    return st.value


def sync_status(stream: Optional[torch.cuda.Stream] = None, clear: bool = True) -> Tuple[int, int]:
    """Stream-scoped status query: (return code, status bits) once the work
    enqueued on `stream` has finished.  The code is VA_OK, VA_ERR_DEVICE_TIMEOUT
    (a bounded wait gave up) or VA_ERR_INVALID_ARG (schedule overflow); a CUDA
    failure raises."""
    st = ctypes.c_uint(0)
    rc = load().varlen_attention_sync_status(_stream_ptr(stream), ctypes.byref(st), int(clear))
    if rc == VA_ERR_CUDA:
        _check(rc)
    return rc, st.value


def selftest_wait_timeout(stream: Optional[torch.cuda.Stream] = None) -> int:
    """Run the failure-path probe (about 2 s of device time); returns its verdict
    (1 = the bounded wait gave up).  Read the raised bit with device_status()."""
    gave_up = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    _check(load().varlen_attention_selftest_wait_timeout(gave_up.data_ptr(), _stream_ptr(stream)))
    (stream or torch.cuda.current_stream()).synchronize()
    return int(gave_up.item())
