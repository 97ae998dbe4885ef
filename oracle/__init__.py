"""fp64 CPU oracle for paged MLA decode (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never imports, links
or calls it, and it imports nothing from the library: the two meet only in
the seeded inputs of ``mla_workloads``.

The arithmetic lives in ``mla_oracle.c`` (plain C, fp64, one loop per term of
the definition).  This module compiles it with gcc on first use and passes
numpy / torch CPU buffers to it through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_LIB = os.path.join(_HERE, "_liboracle.so")
_lock = threading.Lock()
_lib = None

KV_BF16 = 0
KV_FP8 = 1


def build(src: str = _SRC, out: str = _LIB, extra_flags=()) -> str:
    """Compile the oracle (no fast-math: IEEE fp64 semantics are kept)."""
    cmd = ["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared", "-pthread",
           "-fno-fast-math", "-ffp-contract=off", *extra_flags, "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _stale(lib: str, src: str) -> bool:
    return not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src)


def load(path: str = None):
    """Load (building if needed) the oracle shared library; returns a ctypes CDLL."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            if _stale(_LIB, _SRC):
                build()
            _lib = _bind(ctypes.CDLL(_LIB))
    return _lib


def _bind(lib):
    c_p = ctypes.c_void_p
    lib.oracle_mla_decode.restype = ctypes.c_int
    lib.oracle_mla_decode.argtypes = [
        ctypes.c_int, ctypes.c_int, ctypes.c_int, c_p, c_p, c_p, ctypes.c_int, c_p, ctypes.c_int, ctypes.c_int,
        c_p, ctypes.c_int, c_p, c_p, ctypes.c_double, c_p, ctypes.c_int64, c_p, c_p, ctypes.c_int]
    lib.oracle_mla_merge.restype = ctypes.c_int
    lib.oracle_mla_merge.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int, c_p, c_p, c_p, c_p]
    lib.oracle_e4m3_to_f64.restype = ctypes.c_double
    lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
    lib.oracle_bf16_to_f64.restype = ctypes.c_double
    lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    lib.oracle_quantize_row_e4m3.restype = None
    lib.oracle_quantize_row_e4m3.argtypes = [c_p, c_p, c_p, ctypes.c_float]
    lib.oracle_append_kv.restype = ctypes.c_int
    lib.oracle_append_kv.argtypes = [ctypes.c_int, ctypes.c_int, c_p, c_p, c_p, ctypes.c_int, c_p, ctypes.c_int,
                                     ctypes.c_int, c_p, ctypes.c_int, ctypes.c_int, c_p]
    return lib


def _np(x, dtype):
    """A C-contiguous numpy view of a torch CPU tensor (bit reinterpretation) or array."""
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu").contiguous()
            if x.dtype == torch.bfloat16:
                x = x.view(torch.int16)
            elif x.dtype == torch.float8_e4m3fn:
                x = x.view(torch.uint8)
            x = x.numpy()
    except ImportError:
        pass
    x = np.ascontiguousarray(x)
    if x.dtype != dtype:
        if x.dtype.itemsize == np.dtype(dtype).itemsize and x.dtype.kind in "iu" and np.dtype(dtype).kind in "iu":
            x = x.view(dtype)
        else:
            x = x.astype(dtype)
    return x


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def decode(q_lat, q_pe, kv_pages, kv_scale, page_table, ctx_lens, sm_scale, *, kv_dtype,
           vis_lens=None, rows=None, threads=0, lib=None):
    """Oracle decode.  Returns (out [n_rows,512] fp64, lse [n_rows] fp64).

    q_lat [B,T,H,512] and q_pe [B,T,H,64] are bf16 (torch bf16 tensors or uint16
    bit arrays); kv_pages [P,16,576] is bf16 or e4m3fn bytes; kv_scale [P,16]
    fp32 for FP8, or a single value (a per-tensor static scale).  ``rows``
    lists flat row ids b*T*H + t*H + h (default: all).
    """
    lib = lib or load()
    B, T, H = int(q_lat.shape[0]), int(q_lat.shape[1]), int(q_lat.shape[2])
    kvd = KV_BF16 if kv_dtype in ("bf16", KV_BF16) else KV_FP8
    ql = _np(q_lat, np.uint16)
    qp = _np(q_pe, np.uint16)
    kv = _np(kv_pages, np.uint16 if kvd == KV_BF16 else np.uint8)
    sc = _np(kv_scale, np.float32) if kvd == KV_FP8 else None
    per_tensor = int(sc is not None and sc.size == 1)
    pt = _np(page_table, np.int32)
    cl = _np(ctx_lens, np.int32)
    vl = _np(vis_lens, np.int32)
    rr = None if rows is None else _np(rows, np.int64)
    n_rows = B * T * H if rr is None else int(rr.shape[0])
    out = np.zeros((n_rows, 512), dtype=np.float64)
    lse = np.zeros((n_rows,), dtype=np.float64)
    rc = lib.oracle_mla_decode(B, T, H, _ptr(ql), _ptr(qp), _ptr(kv), kvd, _ptr(sc), per_tensor,
                               int(kv.shape[0]), _ptr(pt), int(pt.shape[1]), _ptr(cl), _ptr(vl),
                               float(sm_scale), _ptr(rr), n_rows, _ptr(out), _ptr(lse), int(threads))
    if rc != 0:
        raise ValueError(f"oracle_mla_decode rejected its inputs (code {rc})")
    return out, lse


def decode_workload(w, rows=None, threads=0, lib=None):
    """Oracle decode of an ``mla_workloads.Workload``."""
    return decode(w.q_lat, w.q_pe, w.kv_pages, w.kv_scale, w.page_table, w.ctx_lens, w.sm_scale,
                  kv_dtype=w.kv_dtype, vis_lens=w.vis_lens, rows=rows, threads=threads, lib=lib)


def merge(out_parts, lse_parts, lib=None):
    """LSE merge of [n, rows, dv] normalised partials with [n, rows] log-sum-exps."""
    lib = lib or load()
    op = _np(out_parts, np.float64)
    lp = _np(lse_parts, np.float64)
    n, rows, dv = op.shape
    out = np.zeros((rows, dv), dtype=np.float64)
    lse = np.zeros((rows,), dtype=np.float64)
    rc = lib.oracle_mla_merge(n, rows, dv, _ptr(op), _ptr(lp), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle_mla_merge rejected its inputs (code {rc})")
    return out, lse


def e4m3_to_f64(byte: int, lib=None) -> float:
    return (lib or load()).oracle_e4m3_to_f64(byte)


def bf16_to_f64(bits: int, lib=None) -> float:
    return (lib or load()).oracle_bf16_to_f64(bits)


def e4m3_encode(x: float, lib=None) -> int:
    """e4m3fn code of binary32 x (round to nearest even, clamped to +-448)."""
    return int((lib or load()).oracle_e4m3_encode(float(x)))


def quantize_row_e4m3(row_bf16, lib=None):
    """One 576-value bf16 row -> (576 e4m3 codes as uint8, fp32 scale)."""
    lib = lib or load()
    r = _np(row_bf16, np.uint16).reshape(-1)
    if r.shape[0] != 576:
        raise ValueError("a cached row has 576 values")
    codes = np.zeros((576,), dtype=np.uint8)
    scale = np.zeros((1,), dtype=np.float32)
    lib.oracle_quantize_row_e4m3(_ptr(r), _ptr(codes), _ptr(scale), ctypes.c_float(0.0))
    return codes, float(scale[0])


def append_kv(c_kv_new, k_pe_new, kv_pages, kv_scale, page_table, ctx_lens, *, kv_dtype, lib=None):
    """Oracle cache append: writes token t of sequence b at position
    ctx_lens[b] - T + t of copies of the pages (and scales).  Returns
    (pages, scales or None, ok) as numpy arrays; ok is False when a context or
    page index was out of range (those tokens are skipped)."""
    lib = lib or load()
    kvd = KV_BF16 if kv_dtype in ("bf16", KV_BF16) else KV_FP8
    ck = _np(c_kv_new, np.uint16)
    kp = _np(k_pe_new, np.uint16)
    B, T = int(ck.shape[0]), int(ck.shape[1])
    pages = _np(kv_pages, np.uint16 if kvd == KV_BF16 else np.uint8).copy()
    scales = _np(kv_scale, np.float32).copy() if kvd == KV_FP8 else None
    per_tensor = int(scales is not None and scales.size == 1)
    pt = _np(page_table, np.int32)
    cl = _np(ctx_lens, np.int32)
    rc = lib.oracle_append_kv(B, T, _ptr(ck), _ptr(kp), _ptr(pages), kvd, _ptr(scales), per_tensor,
                              int(pages.shape[0]),
                              _ptr(pt), int(pt.shape[1]), int(pt.shape[1]), _ptr(cl))
    return pages, scales, rc == 0
