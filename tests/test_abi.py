"""The C-ABI library loads, exports every entry point include/bsattn.h
declares, and rejects bad arguments on the host before touching the GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bsattn.h")


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_bsattn_b200 import build
    path = build.build()
    from block_sparse_attention_bsattn_b200 import ops
    assert os.path.samefile(ops.LIB_PATH, path)
    return ops._lib


def declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bsattn_\w+)\s*\(", text)))


def test_header_declares_entry_points():
    names = declared()
    for n in ("bsattn_build_index", "bsattn_fwd_prefill", "bsattn_fwd_decode",
              "bsattn_decode_workspace_size", "bsattn_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared():
        getattr(lib, n)          # AttributeError if missing


def test_status_strings(lib):
    from block_sparse_attention_bsattn_b200 import ops
    assert ops.bsattn_status_string(0) == "BSATTN_OK"
    assert ops.bsattn_status_string(-6) == "BSATTN_ERR_DEVICE_TIMEOUT"
    assert ops.bsattn_status_string(123) == "BSATTN_UNKNOWN_STATUS"
    assert ops.bsattn_version() >= 100


P = ctypes.c_void_p


def _prefill(lib, q=0x1000, k=0x2000, v=0x3000, o=0x4000, B=1, Hq=2, Hkv=2, N=256, d=128,
             block=128, scale=0.1, causal=0, lam=0.0, rp=None, ci=None, mh=1):
    return lib.bsattn_fwd_prefill(P(q) if q else None, P(k) if k else None, P(v) if v else None,
                                  P(o) if o else None, None, B, Hq, Hkv, N, d, block, scale,
                                  causal, lam, P(rp) if rp else None, P(ci) if ci else None, None,
                                  mh, None, None, None)


def test_prefill_host_validation(lib):
    assert _prefill(lib, q=0) == -1                  # null pointer
    assert _prefill(lib, Hq=3, Hkv=2) == -1          # Hq % Hkv
    assert _prefill(lib, lam=1.5) == -1              # lambda outside [0, 1]
    assert _prefill(lib, lam=float("nan")) == -1
    assert _prefill(lib, lam=-0.1) == -1
    assert _prefill(lib, scale=0.0) == -1
    assert _prefill(lib, rp=0x5000, ci=None) == -1   # CSR without col_idx
    assert _prefill(lib, rp=0x5000, ci=0x6000, mh=3) == -1
    assert lib.bsattn_fwd_prefill(P(0x1000), P(0x2000), P(0x3000), P(0x4000), None, 1, 2, 2, 256,
                                  128, 128, 0.1, 0, 0.0, None, None, P(0x7000), 1, None, None,
                                  None) == -1           # row order without a CSR
    assert _prefill(lib, d=96) == -2                 # unsupported head dim
    assert _prefill(lib, block=32) == -2
    assert _prefill(lib, q=0x1001) == -3             # misaligned
    assert _prefill(lib, o=0x4008) == -3


def test_decode_host_validation(lib):
    ws = lib.bsattn_decode_workspace_size(64, 32, 128, 16)
    assert ws == 64 * 32 * 16 * (128 + 2) * 4

    def dec(q=0x1000, B=2, Hq=8, Hkv=2, L=1000, d=128, block=128, lam=0.0, splits=4,
            ws=0x9000, wsb=1 << 30):
        return lib.bsattn_fwd_decode(P(q) if q else None, P(0x2000), P(0x3000), P(0x4000), None,
                                     B, Hq, Hkv, L, d, block, 0.1, 0, lam, splits,
                                     P(ws) if ws else None, wsb, None, None, None)
    assert dec(q=0) == -1
    assert dec(ws=0) == -1
    assert dec(splits=0) == -1
    assert dec(lam=2.0) == -1
    assert dec(Hq=34, Hkv=2) == -2                   # GQA group of 17
    assert dec(Hq=34, Hkv=2, block=64) == -2         # group of 17 with 64-token tiles
    assert dec(d=80) == -2
    assert dec(q=0x1004) == -3
    assert dec(wsb=16) == -4                         # workspace too small


def test_option_bits_validation(lib):
    """The _ex entry points reject unknown option bits before anything runs."""
    U = ctypes.c_uint
    lib.bsattn_fwd_prefill_ex.argtypes = [P, P, P, P, P] + [ctypes.c_int] * 6 + [
        ctypes.c_float, ctypes.c_int, ctypes.c_float, P, P, P, ctypes.c_int, P, P, U, P, P]
    lib.bsattn_fwd_decode_ex.argtypes = [P, P, P, P, P] + [ctypes.c_int] * 6 + [
        ctypes.c_float, ctypes.c_int, ctypes.c_float, ctypes.c_int, P, ctypes.c_size_t, P, P, U,
        P, P]

    def pre(flags, q=0x1000):
        return lib.bsattn_fwd_prefill_ex(P(q) if q else None, P(0x2000), P(0x3000), P(0x4000),
                                         None, 1, 2, 2, 256, 128, 128, 0.1, 0, 0.0, None, None,
                                         None, 1, None, None, flags, None, None)

    def dec(flags, q=0x1000):
        return lib.bsattn_fwd_decode_ex(P(q) if q else None, P(0x2000), P(0x3000), P(0x4000),
                                        None, 2, 8, 2, 1000, 128, 128, 0.1, 0, 0.0, 4, P(0x9000),
                                        1 << 30, None, None, flags, None, None)
    assert pre(0x4) == -1 and pre(0x80000000) == -1
    assert pre(0x1, q=0) == -1
    assert dec(0x2) == -1 and dec(0x1, q=0) == -1


def test_host_pipeline_validation(lib):
    """bsattn_fwd_prefill_host rejects bad arguments before touching a device."""
    f = lib.bsattn_fwd_prefill_host

    def call(chunk=1, d=128, hq=0x1000, dq=0x5000, do=0x8000, lam=0.0, scale=0.1, rp=None,
             ci=None, ro=None, mh=1):
        return f(P(hq) if hq else None, P(0x2000), P(0x3000), P(0x4000), P(dq), P(0x6000),
                 P(0x7000), P(do), 1, 8, 2, 256, d, 128, ctypes.c_float(scale), 1,
                 ctypes.c_float(lam), P(rp) if rp else None, P(ci) if ci else None,
                 P(ro) if ro else None, mh, chunk, None, None)
    assert call(hq=0) == -1
    assert call(chunk=0) == -1
    assert call(chunk=3) == -1          # does not divide the two KV heads
    assert call(lam=1.5) == -1
    assert call(lam=float("nan")) == -1
    assert call(scale=0.0) == -1
    assert call(rp=0x9000) == -1        # CSR without col_idx
    assert call(rp=0x9000, ci=0xa000, mh=3) == -1
    assert call(ro=0xb000) == -1        # row order without a CSR
    assert call(d=96) == -2
    assert call(dq=0x5008) == -3        # staging buffers must be 16-byte aligned
    assert call(do=0x8004) == -3


def test_index_host_validation(lib):
    f = lib.bsattn_build_index
    assert f(None, 1, 4, 4, 64, 64, 0, P(0x1000), P(0x2000), 16, P(0x3000), None, None, None) == -1
    assert f(P(0x10), 0, 4, 4, 64, 64, 0, P(0x1000), P(0x2000), 16, P(0x3000), None, None,
             None) == -1
    assert f(P(0x10), 1, 4, 4, 64, 64, 0, P(0x1000), P(0x2000), -1, P(0x3000), None, None,
             None) == -1
    assert f(P(0x10), 4096, 4096, 4096, 64, 64, 0, P(0x1000), P(0x2000), 16, P(0x3000), None,
             None, None) == -2


def test_debug_hook_validation(lib):
    assert lib.bsattn_debug_set(0, 0) == -1
    assert lib.bsattn_debug_set(2_000_000_000, 0) == 0


def test_shipped_library_has_no_trace_buffer(lib):
    """The trace markers are a debugging build's (-DBSATTN_TRACE): the shipped
    library refuses to allocate a trace buffer and accepts turning it off."""
    view = ctypes.POINTER(ctypes.c_int32)()
    assert lib.bsattn_debug_trace(16, ctypes.byref(view)) == -2   # BSATTN_ERR_UNSUPPORTED
    assert not view
    assert lib.bsattn_debug_trace(0, None) == 0
    assert lib.bsattn_debug_trace(-1, None) == -1


def test_backward_host_validation(lib):
    """bsattn_bwd_prefill rejects bad arguments before touching a device."""
    f = lib.bsattn_bwd_prefill
    assert lib.bsattn_bwd_prefill_workspace_size(1, 2, 300, 128) == 2 * (2 * 3 * 128) * 4

    def call(q=0x1000, st=0x9000, d=128, block=128, hq=4, hkv=2, scale=0.1, ws=0xa000,
             wsb=1 << 20, dq=0xb000):
        return f(P(q) if q else None, P(0x2000), P(0x3000), P(0x4000), P(0x5000), P(0x6000),
                 P(st) if st else None, P(dq), P(0xc000), P(0xd000), 1, hq, hkv, 300, d, block,
                 ctypes.c_float(scale), 1, None, P(ws) if ws else None, wsb, None, None)
    assert call(q=0) == -1
    assert call(st=0) == -1             # the forward's tile status is required
    assert call(ws=0) == -1
    assert call(hq=3, hkv=2) == -1
    assert call(scale=0.0) == -1
    assert call(d=96) == -2
    assert call(block=64) == -2         # 128-token tiles only
    assert call(q=0x1008) == -3
    assert call(dq=0xb004) == -3
    assert call(wsb=100) == -4          # workspace too small


def test_exp2_hook_validation(lib):
    f = lib.bsattn_debug_exp2
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
    assert f(None, None, -1, None) == -1
    assert f(None, 0x1000, 4, None) == -1
    assert f(0x1000, None, 4, None) == -1
    assert f(0x1000, 0x2000, (1 << 32) + 1, None) == -1
