"""CPU oracle for block-sparse attention with BLASST skipping -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It computes in fp64 from the bf16 bits
of the inputs, shares no code with the CUDA library, and is never called by
the product path.

The arithmetic lives in ``bsattn_oracle.c`` (plain C, OpenMP over independent
query tiles).  This module compiles it with gcc on first use and marshals
numpy arrays into it.

Functions and the passages they follow:

* :func:`build_index`  -- mask -> per-query-block CSR ("块稀疏Attention实战",
  section 2.3: the mask kept as a sparse index of non-zero blocks; section 3.3:
  the tiling loop checks whether each block must be computed).
* :func:`prefill`      -- Algorithm 1 of "BLASST: Dynamic Blocked Attention
  Sparsity via Softmax Thresholding" (visit, running max, skip test) followed
  by the exact softmax over the executed tiles.
* :func:`decode`       -- the same per split of the KV sequence, query tile =
  the GQA group of one token.
* :func:`prefill_bwd`  -- the backward pass of sparsity-aware training (BLASST
  page, section 3.3): the gradient of the forward's output with its executed
  tiles held fixed; skipped tiles receive no gradient.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bsattn_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/liboracle.so`` (gcc, -O2,
    OpenMP, IEEE semantics kept: no fast-math)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared",
                               "-std=c11", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def bind(lib: ctypes.CDLL) -> ctypes.CDLL:
    """Declare the C signatures on a loaded oracle library."""
    P = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.oracle_build_index.argtypes = [P, i32, i32, i32, i32, i32, i32, P, P, i64, P]
    lib.oracle_build_index.restype = i32
    lib.oracle_prefill.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, f64, i32,
                                   f64, P, i32, P, i32, P, P, P, P, i32, P]
    lib.oracle_prefill.restype = i32
    lib.oracle_decode.argtypes = [P, P, P, i32, i32, i64, i32, i32, f64, f64, i32,
                                  P, P, P, P, i32, P]
    lib.oracle_decode.restype = i32
    lib.oracle_prefill_bwd.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, i32, f64, i32,
                                       P, P, P, P, P]
    lib.oracle_prefill_bwd.restype = i32
    lib.oracle_num_threads.restype = i32
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = bind(ctypes.CDLL(build()))
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bits(x) -> np.ndarray:
    """bf16 tensor (torch) or uint16 array -> contiguous uint16 numpy bits."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def bf16_to_f64(x) -> np.ndarray:
    b = _bits(x).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


class OracleError(RuntimeError):
    pass


def build_index(mask: np.ndarray, q_block: int, k_block: int, causal: bool,
                capacity: int | None = None):
    """mask uint8 [Hm, nq, nk] -> (row_ptr int32 [Hm*(nq+1)], col_idx int32 [nnz], nnz int32 [Hm])."""
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    Hm, nq, nk = mask.shape
    cap = Hm * nq * nk if capacity is None else capacity
    row_ptr = np.zeros(Hm * (nq + 1), np.int32)
    col_idx = np.zeros(max(cap, 1), np.int32)
    nnz = np.zeros(Hm, np.int32)
    rc = _load().oracle_build_index(_ptr(mask), Hm, nq, nk, q_block, k_block, int(causal),
                                    _ptr(row_ptr), _ptr(col_idx), cap, _ptr(nnz))
    if rc == -4:
        raise OracleError("capacity")
    if rc != 0:
        raise OracleError(f"oracle_build_index rc={rc}")
    return row_ptr, col_idx[: int(nnz.sum())].copy(), nnz


def prefill(q, k, v, block: int, scale: float, causal: bool, lam: float,
            mask=None, items=None, reverse: bool = False, seq_lens=None):
    """Block-sparse prefill.  q [B,Hq,N,d], k/v [B,Hkv,N,d] (bf16 torch or
    uint16 bits).  mask: None or uint8 [Hm, nq, nk].  items: None or an int
    array of (b, h, i) rows.  reverse: visit each row's key tiles in
    descending order (the BLASST page's block-row reordering).  seq_lens:
    None or [B] valid lengths (key padding: keys and query rows at or past a
    sequence's length are padding).  Returns dict(o, lse, status, margin) with o
    [B,Hq,N,d] f64, lse [B,Hq,N] f64, status uint8 [B,Hq,nq,nk] (0 = not
    visited, 1 = skipped, 2 = executed), margin f64 [B,Hq,nq,nk]."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, Hq, N, d = qb.shape
    Hkv = kb.shape[1]
    nq = -(-N // block)
    o = np.zeros((B, Hq, N, d), np.float64)
    lse = np.full((B, Hq, N), np.nan, np.float64)
    status = np.zeros((B, Hq, nq, nq), np.uint8)
    margin = np.full((B, Hq, nq, nq), np.nan, np.float64)
    m = None
    mh = 1
    if mask is not None:
        m = np.ascontiguousarray(mask, dtype=np.uint8)
        mh = m.shape[0]
    sl = None
    if seq_lens is not None:
        sl = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32).reshape(B))
    it = None
    n_items = 0
    if items is not None:
        it = np.ascontiguousarray(np.asarray(items, dtype=np.int32).reshape(-1, 3))
        n_items = it.shape[0]
    rc = _load().oracle_prefill(_ptr(qb), _ptr(kb), _ptr(vb), B, Hq, Hkv, N, d, block,
                                float(scale), int(causal), float(lam), _ptr(m), mh,
                                _ptr(it), n_items, _ptr(o), _ptr(lse), _ptr(status),
                                _ptr(margin), int(reverse), _ptr(sl))
    if rc != 0:
        raise OracleError(f"oracle_prefill rc={rc}")
    return {"o": o, "lse": lse, "status": status, "margin": margin}


def decode(q, k, v, block: int, scale: float, lam: float, num_splits: int,
           sink_seed: bool = False, lens=None):
    """Split-KV decode over independent problems.  q [n, g, d], k/v [n, L, d]
    (bf16 torch or uint16 bits).  sink_seed: every split after the first
    starts its running max from key tile 0's row max.  lens: None or [n]
    cache lengths (the splits cut each problem's own tiles).  Returns dict(o [n,g,d], lse [n,g],
    status uint8 [n,T], margin [n,T])."""
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    n, g, d = qb.shape
    L = kb.shape[1]
    T = -(-L // block)
    o = np.zeros((n, g, d), np.float64)
    lse = np.zeros((n, g), np.float64)
    status = np.zeros((n, T), np.uint8)
    margin = np.zeros((n, T), np.float64)
    ln = None
    if lens is not None:
        ln = np.ascontiguousarray(np.asarray(lens, dtype=np.int64).reshape(n))
    rc = _load().oracle_decode(_ptr(qb), _ptr(kb), _ptr(vb), n, g, L, d, block, float(scale),
                               float(lam), num_splits, _ptr(o), _ptr(lse), _ptr(status),
                               _ptr(margin), int(sink_seed), _ptr(ln))
    if rc != 0:
        raise OracleError(f"oracle_decode rc={rc}")
    return {"o": o, "lse": lse, "status": status, "margin": margin}


def _f64(x) -> np.ndarray:
    """bf16 tensor or bits (exact upcast), or any float tensor/array -> contiguous f64."""
    if isinstance(x, np.ndarray) and x.dtype == np.uint16:
        return np.ascontiguousarray(bf16_to_f64(x))
    if not isinstance(x, np.ndarray):
        import torch
        if x.dtype == torch.bfloat16:
            return np.ascontiguousarray(bf16_to_f64(x))
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def prefill_bwd(q, k, v, dout, block: int, scale: float, causal: bool, status,
                seq_lens=None):
    """Backward of :func:`prefill` for sparsity-aware training.  q, dout
    [B,Hq,N,d], k/v [B,Hkv,N,d] (bf16 torch / uint16 bits, upcast exactly, or
    any float array); status uint8 [B,Hq,nq,nk] as the forward returned it
    (only tiles marked 2, executed, take part); seq_lens None or [B].  Returns
    dict(dq [B,Hq,N,d], dk, dv [B,Hkv,N,d]) in f64."""
    qd, kd, vd, dod = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Hq, N, d = qd.shape
    Hkv = kd.shape[1]
    nq = -(-N // block)
    st = np.ascontiguousarray(np.asarray(status, dtype=np.uint8))
    assert st.shape == (B, Hq, nq, nq) and dod.shape == qd.shape and vd.shape == kd.shape
    sl = None
    if seq_lens is not None:
        sl = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32).reshape(B))
    dq = np.zeros_like(qd)
    dk = np.zeros_like(kd)
    dv = np.zeros_like(vd)
    rc = _load().oracle_prefill_bwd(_ptr(qd), _ptr(kd), _ptr(vd), _ptr(dod), B, Hq, Hkv, N, d,
                                    block, float(scale), int(causal), _ptr(st), _ptr(sl),
                                    _ptr(dq), _ptr(dk), _ptr(dv))
    if rc != 0:
        raise OracleError(f"oracle_prefill_bwd rc={rc}")
    return {"dq": dq, "dk": dk, "dv": dv}


def decode_problems(q, k, v, pairs):
    """Gather (b, kv_head) problems from [B,Hq,d] / [B,Hkv,L,d] tensors into
    the [n,g,d] / [n,L,d] form :func:`decode` takes (no arithmetic)."""
    import torch
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    qs = torch.stack([q[b, kvh * g:(kvh + 1) * g] for b, kvh in pairs])
    ks = torch.stack([k[b, kvh] for b, kvh in pairs])
    vs = torch.stack([v[b, kvh] for b, kvh in pairs])
    return qs, ks, vs
