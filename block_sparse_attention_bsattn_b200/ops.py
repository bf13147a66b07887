"""ctypes binding of the C ABI in ``include/bsattn.h`` -- argument marshalling only.

Every function here takes torch tensors on the current CUDA device, checks
shapes/dtypes, allocates outputs the caller did not pass, and calls the entry
point of the same name in ``lib/libbsattn.so`` on the current torch stream.
All arithmetic happens in the library's kernels; there is no fallback: if the
library is missing this module fails to import.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libbsattn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -m block_sparse_attention_bsattn_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SZ = ctypes.c_size_t

_lib.bsattn_status_string.argtypes = [_I]
_lib.bsattn_status_string.restype = ctypes.c_char_p
_lib.bsattn_version.restype = _I
_lib.bsattn_debug_set.argtypes = [ctypes.c_longlong, _I]
_lib.bsattn_debug_set.restype = _I
_lib.bsattn_debug_exp2.argtypes = [_P, _P, _I64, _P]
_lib.bsattn_debug_exp2.restype = _I
_lib.bsattn_debug_trace.argtypes = [_I, ctypes.POINTER(ctypes.POINTER(ctypes.c_int32))]
_lib.bsattn_debug_trace.restype = _I
_lib.bsattn_build_index.argtypes = [_P, _I, _I, _I, _I, _I, _I, _P, _P, _I64, _P, _P, _P, _P]
_lib.bsattn_build_index.restype = _I
_lib.bsattn_fwd_prefill.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _F,
                                    _P, _P, _P, _I, _P, _P, _P]
_lib.bsattn_fwd_prefill.restype = _I
_lib.bsattn_fwd_prefill_ex.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _F,
                                       _P, _P, _P, _I, _P, _P, ctypes.c_uint, _P, _P]
_lib.bsattn_fwd_prefill_ex.restype = _I
_lib.bsattn_fwd_prefill_host.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                         _F, _I, _F, _P, _P, _P, _I, _I, _P, _P]
_lib.bsattn_fwd_prefill_host.restype = _I
_lib.bsattn_decode_workspace_size.argtypes = [_I, _I, _I, _I]
_lib.bsattn_decode_workspace_size.restype = _SZ
_lib.bsattn_fwd_decode.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _F, _I,
                                   _P, _SZ, _P, _P, _P]
_lib.bsattn_fwd_decode.restype = _I
_lib.bsattn_fwd_decode_ex.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _F,
                                      _I, _P, _SZ, _P, _P, ctypes.c_uint, _P, _P]
_lib.bsattn_fwd_decode_ex.restype = _I
_lib.bsattn_fwd_decode_noalloc.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I,
                                           _F, _I, _P, _P, _P]
_lib.bsattn_fwd_decode_noalloc.restype = _I
_lib.bsattn_bwd_prefill_workspace_size.argtypes = [_I, _I, _I, _I]
_lib.bsattn_bwd_prefill_workspace_size.restype = _SZ
_lib.bsattn_bwd_prefill.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I,
                                    _I, _F, _I, _P, _P, _SZ, _P, _P]
_lib.bsattn_bwd_prefill.restype = _I

# option bits of the _ex entry points (include/bsattn.h)
PREFILL_REVERSE = 0x1
PREFILL_SKIP_V = 0x2
DECODE_SINK_SEED = 0x1

EXPORTED = ("bsattn_status_string", "bsattn_version", "bsattn_debug_set", "bsattn_debug_exp2",
            "bsattn_debug_trace",
            "bsattn_build_index",
            "bsattn_fwd_prefill", "bsattn_fwd_prefill_ex", "bsattn_fwd_prefill_host",
            "bsattn_decode_workspace_size",
            "bsattn_fwd_decode", "bsattn_fwd_decode_ex",
            "bsattn_fwd_decode_noalloc", "bsattn_bwd_prefill_workspace_size",
            "bsattn_bwd_prefill")


class BsattnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {bsattn_status_string(code)} ({code})")


def bsattn_status_string(code: int) -> str:
    return _lib.bsattn_status_string(int(code)).decode()


def bsattn_version() -> int:
    return int(_lib.bsattn_version())


def bsattn_debug_set(wait_limit_ns: int = 2_000_000_000, inject_stall: bool = False) -> None:
    """Test hook: per-wait time limit of the pipelined kernels and a switch
    that makes the prefill producer never issue its first load."""
    rc = _lib.bsattn_debug_set(int(wait_limit_ns), int(bool(inject_stall)))
    if rc:
        raise BsattnError(rc, "bsattn_debug_set")


def bsattn_debug_exp2(x: torch.Tensor) -> torch.Tensor:
    """Test hook: 2^x through the prefill kernels' FMA-pipe exponential, for
    a contiguous float32 CUDA tensor."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 CUDA tensor")
    y = torch.empty_like(x)
    rc = _lib.bsattn_debug_exp2(x.data_ptr(), y.data_ptr(), x.numel(), _stream(None))
    if rc:
        raise BsattnError(rc, "bsattn_debug_exp2")
    return y


def bsattn_debug_trace(n: int):
    """Debugging aid of a library built with -DBSATTN_TRACE: n > 0 makes the
    kernels record progress markers into a library-owned mapped host buffer of
    n int32 and returns a numpy view of it (readable while a kernel runs);
    n = 0 turns tracing off and returns None.  The shipped library has no
    markers compiled in and raises BsattnError(BSATTN_ERR_UNSUPPORTED) for
    n > 0."""
    import numpy as np
    view = ctypes.POINTER(ctypes.c_int32)()
    rc = _lib.bsattn_debug_trace(int(n), ctypes.byref(view))
    if rc:
        raise BsattnError(rc, "bsattn_debug_trace")
    return np.ctypeslib.as_array(view, shape=(n,)) if n > 0 else None


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(t: torch.Tensor, name: str, dtype, dims: int):
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or t.dim() != dims or not t.is_cuda \
            or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor with {dims} dims")


def _check_buf(t: Optional[torch.Tensor], name: str, dtype, numel: int, exact: bool = False):
    """A caller-supplied output buffer: contiguous CUDA `dtype`, holding at
    least (or, with `exact`, exactly) `numel` elements, so that no kernel
    writes past its end."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or not t.is_cuda \
            or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor")
    if (t.numel() != numel) if exact else (t.numel() < numel):
        raise ValueError(f"{name}: {'exactly' if exact else 'at least'} {numel} elements "
                         f"needed, got {t.numel()}")


def bsattn_build_index(mask: torch.Tensor, q_block: int, k_block: int, causal: bool = False,
                       capacity: Optional[int] = None, status: Optional[torch.Tensor] = None,
                       with_order: bool = False, stream=None):
    """mask uint8 [mask_heads, nq, nk] -> (row_ptr int32 [mask_heads*(nq+1)],
    col_idx int32 [capacity], nnz int32 [mask_heads]) and, with `with_order`,
    a fourth tensor row_order int32 [mask_heads*nq] (longest rows first).
    col_idx is sized to `capacity` (default: every block)."""
    if mask.dim() == 2:
        mask = mask[None]
    _check(mask, "mask", torch.uint8, 3)
    Hm, nq, nk = mask.shape
    cap = Hm * nq * nk if capacity is None else int(capacity)
    dev = mask.device
    row_ptr = torch.empty(Hm * (nq + 1), dtype=torch.int32, device=dev)
    col_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=dev)
    nnz = torch.empty(Hm, dtype=torch.int32, device=dev)
    order = torch.empty(Hm * nq, dtype=torch.int32, device=dev) if with_order else None
    rc = _lib.bsattn_build_index(_ptr(mask), Hm, nq, nk, int(q_block), int(k_block), int(causal),
                                 _ptr(row_ptr), _ptr(col_idx), cap, _ptr(nnz), _ptr(order),
                                 _ptr(status), _stream(stream))
    if rc:
        raise BsattnError(rc, "bsattn_build_index")
    if with_order:
        return row_ptr, col_idx, nnz, order
    return row_ptr, col_idx, nnz


def bsattn_fwd_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block: int,
                       scale: Optional[float] = None, causal: bool = False, lam: float = 0.0,
                       row_ptr: Optional[torch.Tensor] = None,
                       col_idx: Optional[torch.Tensor] = None, mask_heads: int = 1,
                       o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                       want_lse: bool = True, tile_status: Optional[torch.Tensor] = None,
                       status: Optional[torch.Tensor] = None,
                       row_order: Optional[torch.Tensor] = None, stream=None,
                       reverse: bool = False, skip_v: bool = False,
                       seq_lens: Optional[torch.Tensor] = None):
    """q [B,Hq,N,d], k/v [B,Hkv,N,d] bf16 -> (o [B,Hq,N,d] bf16, lse [B,Hq,N] fp32 or None).
    reverse: visit each row's key tiles in descending order; skip_v: load V
    only for executed tiles (bsattn_fwd_prefill_ex with BSATTN_PREFILL_REVERSE
    / BSATTN_PREFILL_SKIP_V); seq_lens: int32 [B] on the device, valid tokens
    per sequence (key padding)."""
    _check(q, "q", torch.bfloat16, 4)
    _check(k, "k", torch.bfloat16, 4)
    _check(v, "v", torch.bfloat16, 4)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape:
        raise ValueError("k/v must be [B, Hkv, N, d] matching q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    nq = -(-N // int(block))
    _check_buf(o, "o", torch.bfloat16, B * Hq * N * d, exact=True)
    _check_buf(lse, "lse", torch.float32, B * Hq * N, exact=True)
    _check_buf(tile_status, "tile_status", torch.uint8, B * Hq * nq * nq)
    _check_buf(status, "status", torch.int32, 1)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, Hq, N, dtype=torch.float32, device=q.device)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d, int(block),
            float(scale), int(causal), float(lam), _ptr(row_ptr), _ptr(col_idx), _ptr(row_order),
            int(mask_heads), _ptr(tile_status))
    flags = (PREFILL_REVERSE if reverse else 0) | (PREFILL_SKIP_V if skip_v else 0)
    if seq_lens is not None:
        _check(seq_lens, "seq_lens", torch.int32, 1)
        if seq_lens.numel() != B:
            raise ValueError("seq_lens must hold B lengths")
    if flags or seq_lens is not None:
        rc = _lib.bsattn_fwd_prefill_ex(*args, _ptr(seq_lens), flags, _ptr(status),
                                        _stream(stream))
    else:
        rc = _lib.bsattn_fwd_prefill(*args, _ptr(status), _stream(stream))
    if rc:
        raise BsattnError(rc, "bsattn_fwd_prefill")
    return o, lse


def bsattn_fwd_prefill_host(hq: torch.Tensor, hk: torch.Tensor, hv: torch.Tensor,
                            ho: torch.Tensor, dq: torch.Tensor, dk: torch.Tensor,
                            dv: torch.Tensor, do: torch.Tensor, block: int,
                            scale: Optional[float] = None, causal: bool = False,
                            lam: float = 0.0, row_ptr: Optional[torch.Tensor] = None,
                            col_idx: Optional[torch.Tensor] = None, mask_heads: int = 1,
                            row_order: Optional[torch.Tensor] = None,
                            kv_heads_per_chunk: int = 1, status: Optional[torch.Tensor] = None,
                            stream=None) -> None:
    """Prefill of host (pinned) hq/hk/hv into host ho, staged through the
    device tensors dq/dk/dv/do with copies and kernels overlapped per chunk of
    KV heads.  Only enqueues: synchronise the stream before reading ho."""
    for t, name in ((hq, "hq"), (hk, "hk"), (hv, "hv"), (ho, "ho")):
        if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name}: expected a contiguous host bf16 tensor with 4 dims")
    for t, name in ((dq, "dq"), (dk, "dk"), (dv, "dv"), (do, "do")):
        _check(t, name, torch.bfloat16, 4)
    B, Hq, N, d = hq.shape
    Hkv = hk.shape[1]
    if dq.shape != hq.shape or do.shape != hq.shape or ho.shape != hq.shape or \
            dk.shape != hk.shape or dv.shape != hk.shape or hv.shape != hk.shape:
        raise ValueError("staging and host shapes must match")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rc = _lib.bsattn_fwd_prefill_host(
        ctypes.c_void_p(hq.data_ptr()), ctypes.c_void_p(hk.data_ptr()),
        ctypes.c_void_p(hv.data_ptr()), ctypes.c_void_p(ho.data_ptr()), _ptr(dq), _ptr(dk),
        _ptr(dv), _ptr(do), B, Hq, Hkv, N, d, int(block), float(scale), int(causal), float(lam),
        _ptr(row_ptr), _ptr(col_idx), _ptr(row_order), int(mask_heads), int(kv_heads_per_chunk),
        _ptr(status), _stream(stream))
    if rc:
        raise BsattnError(rc, "bsattn_fwd_prefill_host")


def bsattn_decode_workspace_size(B: int, Hq: int, d: int, num_splits: int) -> int:
    return int(_lib.bsattn_decode_workspace_size(B, Hq, d, num_splits))


def _check_decode_bufs(B, Hq, Hkv, L, d, block, o, lse, tile_status, status):
    T = -(-L // int(block))
    _check_buf(o, "o", torch.bfloat16, B * Hq * d, exact=True)
    _check_buf(lse, "lse", torch.float32, B * Hq, exact=True)
    _check_buf(tile_status, "tile_status", torch.uint8, B * Hkv * T)
    _check_buf(status, "status", torch.int32, 1)


def bsattn_fwd_decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block: int,
                      num_splits: int, scale: Optional[float] = None, lam: float = 0.0,
                      o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                      want_lse: bool = True, workspace: Optional[torch.Tensor] = None,
                      tile_status: Optional[torch.Tensor] = None,
                      status: Optional[torch.Tensor] = None, stream=None,
                      sink_seed: bool = False, seq_lens: Optional[torch.Tensor] = None):
    """q [B,Hq,d], k/v [B,Hkv,L,d] bf16 -> (o [B,Hq,d] bf16, lse [B,Hq] fp32 or None).
    sink_seed: splits after the first start their running max from key tile
    0's row max (calls bsattn_fwd_decode_ex with BSATTN_DECODE_SINK_SEED);
    seq_lens: int32 [B] on the device, cache length per sequence."""
    _check(q, "q", torch.bfloat16, 3)
    _check(k, "k", torch.bfloat16, 4)
    _check(v, "v", torch.bfloat16, 4)
    B, Hq, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    if k.shape != (B, Hkv, L, d) or v.shape != k.shape:
        raise ValueError("k/v must be [B, Hkv, L, d] matching q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    _check_decode_bufs(B, Hq, Hkv, L, d, block, o, lse, tile_status, status)
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device)
    need = bsattn_decode_workspace_size(B, Hq, d, num_splits)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    elif not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace: expected a contiguous CUDA tensor")
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, L, d, int(block),
            float(scale), 0, float(lam), int(num_splits), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _ptr(tile_status))
    if seq_lens is not None:
        _check(seq_lens, "seq_lens", torch.int32, 1)
        if seq_lens.numel() != B:
            raise ValueError("seq_lens must hold B lengths")
    if sink_seed or seq_lens is not None:
        rc = _lib.bsattn_fwd_decode_ex(*args, _ptr(seq_lens), DECODE_SINK_SEED if sink_seed else 0,
                                       _ptr(status), _stream(stream))
    else:
        rc = _lib.bsattn_fwd_decode(*args, _ptr(status), _stream(stream))
    if rc:
        raise BsattnError(rc, "bsattn_fwd_decode")
    return o, lse


def bsattn_fwd_decode_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block: int,
                              num_splits: int, o: torch.Tensor, scale: Optional[float] = None,
                              lam: float = 0.0, lse: Optional[torch.Tensor] = None,
                              tile_status: Optional[torch.Tensor] = None,
                              status: Optional[torch.Tensor] = None, stream=None):
    """Decode for callers that cannot allocate device memory: the library's
    own 32 MiB scratch array replaces the workspace, and every output buffer
    (o, and lse / tile_status when wanted) comes from the caller."""
    _check(q, "q", torch.bfloat16, 3)
    _check(k, "k", torch.bfloat16, 4)
    _check(v, "v", torch.bfloat16, 4)
    _check(o, "o", torch.bfloat16, 3)
    B, Hq, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    if k.shape != (B, Hkv, L, d) or v.shape != k.shape or o.shape != q.shape:
        raise ValueError("k/v must be [B, Hkv, L, d] and o [B, Hq, d] matching q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    _check_decode_bufs(B, Hq, Hkv, L, d, block, o, lse, tile_status, status)
    rc = _lib.bsattn_fwd_decode_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq,
                                        Hkv, L, d, int(block), float(scale), 0, float(lam),
                                        int(num_splits), _ptr(tile_status), _ptr(status),
                                        _stream(stream))
    if rc:
        raise BsattnError(rc, "bsattn_fwd_decode_noalloc", "bsattn_bwd_prefill_workspace_size",
            "bsattn_bwd_prefill")
    return o, lse


def bsattn_bwd_prefill_workspace_size(B: int, Hq: int, N: int, block: int = 128) -> int:
    return int(_lib.bsattn_bwd_prefill_workspace_size(B, Hq, N, int(block)))


def bsattn_bwd_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                       dout: torch.Tensor, lse: torch.Tensor, tile_status: torch.Tensor,
                       block: int = 128, scale: Optional[float] = None, causal: bool = False,
                       seq_lens: Optional[torch.Tensor] = None,
                       status: Optional[torch.Tensor] = None, stream=None,
                       dq: Optional[torch.Tensor] = None, dk: Optional[torch.Tensor] = None,
                       dv: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None):
    """Gradients of bsattn_fwd_prefill with its executed tiles held fixed:
    (dq [B,Hq,N,d], dk, dv [B,Hkv,N,d]) bf16.  lse and tile_status are the
    forward call's outputs; only tiles marked 2 (executed) take part.  dq, dk,
    dv and the workspace may be passed in (else they are allocated here)."""
    for t, name in ((q, "q"), (o, "o"), (dout, "dout"), (k, "k"), (v, "v")):
        _check(t, name, torch.bfloat16, 4)
    _check(lse, "lse", torch.float32, 3)
    _check(tile_status, "tile_status", torch.uint8, 4)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    nq = -(-N // block)
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape or o.shape != q.shape or \
            dout.shape != q.shape or lse.shape != (B, Hq, N) or \
            tile_status.shape != (B, Hq, nq, nq):
        raise ValueError("shapes do not match the forward call's")
    if seq_lens is not None:
        _check(seq_lens, "seq_lens", torch.int32, 1)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    ws_bytes = int(_lib.bsattn_bwd_prefill_workspace_size(B, Hq, N, int(block)))
    if workspace is None:
        ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device)
    else:
        if not workspace.is_cuda or not workspace.is_contiguous() or \
                workspace.numel() * workspace.element_size() < ws_bytes:
            raise ValueError(f"workspace: a contiguous CUDA buffer of {ws_bytes} bytes needed")
        ws = workspace
        ws_bytes = workspace.numel() * workspace.element_size()
    _check_buf(dq, "dq", torch.bfloat16, q.numel(), exact=True)
    _check_buf(dk, "dk", torch.bfloat16, k.numel(), exact=True)
    _check_buf(dv, "dv", torch.bfloat16, v.numel(), exact=True)
    _check_buf(status, "status", torch.int32, 1)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    rc = _lib.bsattn_bwd_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                                 _ptr(tile_status), _ptr(dq), _ptr(dk), _ptr(dv), B, Hq, Hkv, N,
                                 d, int(block), float(scale), int(causal), _ptr(seq_lens),
                                 _ptr(ws), ws_bytes, _ptr(status), _stream(stream))
    if rc:
        raise BsattnError(rc, "bsattn_bwd_prefill")
    return dq, dk, dv
