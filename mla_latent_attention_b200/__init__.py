"""Paged MLA latent-attention decode for B200 (sm_100a).

Thin Python binding over the C ABI of ``include/mla.h`` (``libmla_b200.so``,
built in-tree by ``mla_latent_attention_b200/build.py``).  This module only
marshals arguments: it allocates outputs and workspace with torch when the
caller does not pass them, picks torch's current CUDA stream, and calls the
library.  Every step of the computation runs in the library's CUDA kernels;
there is no CPU or PyTorch fallback, and calling an op without the built
library raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = ["decode", "merge_partials", "append_kv", "workspace_size", "read_device_error",
           "reset_device_error", "library_path", "load_library", "MlaError", "KERNELS"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmla_b200.so")
_lock = threading.Lock()
_lib = None

MLA_OK = 0
KV_BF16, KV_FP8 = 0, 1
OUT_BF16, OUT_F32 = 0, 1
KERNELS = {"auto": 0, "simt": 1, "tcgen05": 2}
DEV_ERRORS = {0: "ok", 1: "bad page index", 2: "bad context length", 3: "bad visible count",
              4: "an on-chip wait gave up"}
EXPORTED = ("mla_decode_workspace_size", "mla_decode", "mla_decode_noalloc", "mla_merge_partials", "mla_append_kv",
            "mla_read_device_error", "mla_reset_device_error", "mla_status_string",
            "mla_last_cuda_error")


class MlaError(RuntimeError):
    pass


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("H", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
                ("page_table_stride", ctypes.c_int32), ("kv_dtype", ctypes.c_int32),
                ("out_dtype", ctypes.c_int32), ("num_splits", ctypes.c_int32),
                ("kernel", ctypes.c_int32), ("vis_lens", ctypes.c_void_p),
                ("stage_event", ctypes.c_void_p), ("kv_scale_per_tensor", ctypes.c_int32),
                ("wait_limit_kcycles", ctypes.c_int32)]


def library_path() -> str:
    return _LIB_PATH


def load_library(path: str = None):
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or _LIB_PATH
        if not os.path.exists(p):
            raise MlaError(f"CUDA library not built: {p} is missing "
                           "(run `python mla_latent_attention_b200/build.py`)")
        lib = ctypes.CDLL(p)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        lib.mla_decode_workspace_size.restype = i64
        lib.mla_decode_workspace_size.argtypes = [ctypes.POINTER(Dims)]
        lib.mla_decode.restype = ctypes.c_int
        lib.mla_decode.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp,
                                   ctypes.POINTER(Dims), vp, ctypes.c_size_t, vp]
        lib.mla_decode_noalloc.restype = ctypes.c_int
        lib.mla_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp,
                                           ctypes.POINTER(Dims), vp]
        lib.mla_merge_partials.restype = ctypes.c_int
        lib.mla_merge_partials.argtypes = [vp, vp, i32, i64, vp, i32, vp, vp]
        lib.mla_append_kv.restype = ctypes.c_int
        lib.mla_append_kv.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.POINTER(Dims), vp, vp]
        lib.mla_read_device_error.restype = ctypes.c_int
        lib.mla_read_device_error.argtypes = [vp, ctypes.POINTER(i32), ctypes.POINTER(i32), vp]
        lib.mla_reset_device_error.restype = ctypes.c_int
        lib.mla_reset_device_error.argtypes = [vp, vp]
        lib.mla_status_string.restype = ctypes.c_char_p
        lib.mla_status_string.argtypes = [ctypes.c_int]
        lib.mla_last_cuda_error.restype = ctypes.c_int
        lib.mla_last_cuda_error.argtypes = []
        if path is None:
            _lib = lib
        return lib


def _check(rc: int, what: str):
    if rc != MLA_OK:
        lib = load_library()
        msg = lib.mla_status_string(rc).decode()
        cu = lib.mla_last_cuda_error()
        raise MlaError(f"{what} failed: {msg} (status {rc}, last cudaError {cu})")


def _ptr(t):
    return None if t is None else t.data_ptr()   # the argtypes are c_void_p: a plain int converts


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def _kv_code(kv_pages):
    if kv_pages.dtype == torch.bfloat16:
        return KV_BF16
    if kv_pages.dtype in (torch.uint8, torch.float8_e4m3fn):
        return KV_FP8
    raise MlaError(f"kv_pages must be bf16, uint8 or float8_e4m3fn, got {kv_pages.dtype}")


def make_dims(q_lat, kv_pages, page_table, *, out_dtype=torch.bfloat16, num_splits=0,
              kernel="auto", vis_lens=None, stage_event=None, kv_scale=None, wait_limit_kcycles=0) -> Dims:
    B, T, H = int(q_lat.shape[0]), int(q_lat.shape[1]), int(q_lat.shape[2])
    return Dims(B=B, T=T, H=H, num_pages=int(kv_pages.shape[0]),
                max_pages_per_seq=int(page_table.shape[1]),
                page_table_stride=int(page_table.stride(0)), kv_dtype=_kv_code(kv_pages),
                out_dtype=OUT_F32 if out_dtype == torch.float32 else OUT_BF16,
                num_splits=int(num_splits), kernel=KERNELS[kernel],
                vis_lens=None if vis_lens is None else vis_lens.data_ptr(),
                stage_event=None if stage_event is None else stage_event.cuda_event,
                kv_scale_per_tensor=int(kv_scale is not None and kv_scale.numel() == 1),
                wait_limit_kcycles=int(wait_limit_kcycles))


def workspace_size(dims: Dims) -> int:
    n = load_library().mla_decode_workspace_size(ctypes.byref(dims))
    if n < 0:
        _check(int(n), "mla_decode_workspace_size")
    return int(n)


def _need(t, name, dtype=None, device=None, shape=None):
    d = t.device
    if d.type != "cuda":
        raise MlaError(f"{name} must be a CUDA tensor")
    if device is not None and d != device:
        raise MlaError(f"{name} is on {d}, expected {device}")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise MlaError(f"{name} has dtype {t.dtype}")
    if shape is not None and t.shape != shape:
        raise MlaError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if name != "page_table" and not t.is_contiguous():
        raise MlaError(f"{name} must be contiguous")


def decode(q_lat, q_pe, kv_pages, kv_scale, page_table, ctx_lens, sm_scale, *, out=None, lse=None,
           vis_lens=None, out_dtype=torch.bfloat16, num_splits=0, kernel="auto", workspace=None,
           stream=None, stage_event=None, wait_limit_kcycles=0):
    """Paged MLA decode (``mla_decode``).  Returns (out [B,T,H,512], lse [B,T,H] fp32).

    ``stage_event`` (a ``torch.cuda.Event``) is recorded between the attention
    kernel and the merge kernel, for timing the two apart.  A ``workspace``
    whose device error word will be read (``read_device_error``) must start
    zeroed (``torch.zeros``, or ``reset_device_error`` once).
    ``wait_limit_kcycles`` > 0 bounds every on-chip wait of the tensor-core
    kernel to that many thousand SM cycles (``mla_dims.wait_limit_kcycles``)."""
    lib = load_library()
    dev = q_lat.device
    B, T, H = q_lat.shape[:3]
    _need(q_lat, "q_lat", torch.bfloat16, dev, (B, T, H, 512))
    _need(q_pe, "q_pe", torch.bfloat16, dev, (B, T, H, 64))
    _need(kv_pages, "kv_pages", (torch.bfloat16, torch.uint8, torch.float8_e4m3fn), dev)
    if kv_pages.dim() != 3 or kv_pages.shape[1:] != (16, 576):
        raise MlaError(f"kv_pages must be [P,16,576], got {tuple(kv_pages.shape)}")
    if kv_scale is not None:  # per position [P,16], or one per-tensor static scale
        _need(kv_scale, "kv_scale", torch.float32, dev,
              (1,) if kv_scale.numel() == 1 else (kv_pages.shape[0], 16))
    _need(page_table, "page_table", torch.int32, dev)
    if page_table.dim() != 2 or page_table.shape[0] != B or page_table.stride(1) != 1:
        raise MlaError("page_table must be [B, max_pages] int32 with unit column stride")
    _need(ctx_lens, "ctx_lens", torch.int32, dev, (B,))
    if vis_lens is not None:
        _need(vis_lens, "vis_lens", torch.int32, dev, (B, T))
    if out is None:
        out = torch.empty((B, T, H, 512), dtype=out_dtype, device=dev)
    else:
        _need(out, "out", (torch.bfloat16, torch.float32), dev, (B, T, H, 512))
        out_dtype = out.dtype
    if lse is None:
        lse = torch.empty((B, T, H), dtype=torch.float32, device=dev)
    else:
        _need(lse, "lse", torch.float32, dev, (B, T, H))
    dims = make_dims(q_lat, kv_pages, page_table, out_dtype=out_dtype, num_splits=num_splits,
                     kernel=kernel, vis_lens=vis_lens, stage_event=stage_event, kv_scale=kv_scale,
                     wait_limit_kcycles=wait_limit_kcycles)
    need = workspace_size(dims)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    else:
        _need(workspace, "workspace", None, dev)
        if workspace.numel() * workspace.element_size() < need:
            raise MlaError(f"workspace has {workspace.numel() * workspace.element_size()} bytes, needs {need}")
    rc = lib.mla_decode(_ptr(q_lat), _ptr(q_pe), _ptr(kv_pages), _ptr(kv_scale), _ptr(page_table),
                        _ptr(ctx_lens), float(sm_scale), _ptr(out), _ptr(lse), ctypes.byref(dims),
                        _ptr(workspace), workspace.numel() * workspace.element_size(),
                        _stream(stream, dev))
    _check(rc, "mla_decode")
    return out, lse


def decode_workload(w, **kw):
    """``decode`` on an ``mla_workloads.Workload`` whose tensors are on a CUDA device."""
    return decode(w.q_lat, w.q_pe, w.kv_pages, w.kv_scale, w.page_table, w.ctx_lens, w.sm_scale,
                  vis_lens=w.vis_lens, **kw)


def merge_partials(out_parts, lse_parts, *, out=None, lse=None, out_dtype=torch.bfloat16,
                   stream=None):
    """LSE merge (``mla_merge_partials``) of [n, rows, 512] fp32 parts and [n, rows] fp32 lses.

    Leading dims beyond (n, ..., 512) are flattened into rows.  Returns (out, lse)."""
    lib = load_library()
    dev = out_parts.device
    n = out_parts.shape[0]
    rows_shape = tuple(out_parts.shape[1:-1])
    rows = 1
    for s in rows_shape:
        rows *= int(s)
    _need(out_parts, "out_parts", torch.float32, dev)
    _need(lse_parts, "lse_parts", torch.float32, dev, (n, *rows_shape))
    if out_parts.shape[-1] != 512:
        raise MlaError("out_parts must end in 512")
    if out is None:
        out = torch.empty((*rows_shape, 512), dtype=out_dtype, device=dev)
    else:
        _need(out, "out", (torch.bfloat16, torch.float32), dev, (*rows_shape, 512))
    if lse is None:
        lse = torch.empty(rows_shape, dtype=torch.float32, device=dev)
    else:
        _need(lse, "lse", torch.float32, dev, rows_shape)
    rc = lib.mla_merge_partials(_ptr(out_parts), _ptr(lse_parts), int(n), rows, _ptr(out),
                                OUT_F32 if out.dtype == torch.float32 else OUT_BF16, _ptr(lse),
                                _stream(stream, dev))
    _check(rc, "mla_merge_partials")
    return out, lse


def append_kv(c_kv_new, k_pe_new, kv_pages, kv_scale, page_table, ctx_lens, *, device_error=None,
              stream=None):
    """Write the T new tokens of each sequence into the paged cache
    (``mla_append_kv``): token t of sequence b goes to position
    ctx_lens[b] - T + t.  c_kv_new [B,T,512] and k_pe_new [B,T,64] are bf16;
    an FP8 cache is quantised with one scale per token (written to kv_scale
    [P,16]), or with the static scale when kv_scale has one element.  ``device_error``: an
    optional int32 CUDA tensor of 2 elements receiving a device error."""
    lib = load_library()
    dev = kv_pages.device
    B, T = int(c_kv_new.shape[0]), int(c_kv_new.shape[1])
    _need(c_kv_new, "c_kv_new", torch.bfloat16, dev, (B, T, 512))
    _need(k_pe_new, "k_pe_new", torch.bfloat16, dev, (B, T, 64))
    _need(kv_pages, "kv_pages", (torch.bfloat16, torch.uint8, torch.float8_e4m3fn), dev)
    if kv_pages.dim() != 3 or kv_pages.shape[1:] != (16, 576):
        raise MlaError(f"kv_pages must be [P,16,576], got {tuple(kv_pages.shape)}")
    _need(page_table, "page_table", torch.int32, dev)
    if page_table.dim() != 2 or page_table.shape[0] != B or page_table.stride(1) != 1:
        raise MlaError("page_table must be [B, max_pages] int32 with unit column stride")
    _need(ctx_lens, "ctx_lens", torch.int32, dev, (B,))
    if kv_scale is not None:  # per position [P,16] (written), or one static scale (read)
        _need(kv_scale, "kv_scale", torch.float32, dev,
              (1,) if kv_scale.numel() == 1 else (kv_pages.shape[0], 16))
    if device_error is not None:
        _need(device_error, "device_error", torch.int32, dev, (2,))
    dims = Dims(B=B, T=T, H=1, num_pages=int(kv_pages.shape[0]), max_pages_per_seq=int(page_table.shape[1]),
                page_table_stride=int(page_table.stride(0)), kv_dtype=_kv_code(kv_pages), out_dtype=OUT_BF16,
                num_splits=0, kernel=0, vis_lens=None, stage_event=None,
                kv_scale_per_tensor=int(kv_scale is not None and kv_scale.numel() == 1))
    rc = lib.mla_append_kv(_ptr(c_kv_new), _ptr(k_pe_new), _ptr(kv_pages), _ptr(kv_scale), _ptr(page_table),
                           _ptr(ctx_lens), ctypes.byref(dims), _ptr(device_error), _stream(stream, dev))
    _check(rc, "mla_append_kv")


def read_device_error(workspace, stream=None):
    """(code, info) of the workspace error word; synchronises the stream."""
    _need(workspace, "workspace")
    code, info = ctypes.c_int32(0), ctypes.c_int32(0)
    rc = load_library().mla_read_device_error(_ptr(workspace), ctypes.byref(code), ctypes.byref(info),
                                              _stream(stream, workspace.device))
    _check(rc, "mla_read_device_error")
    return code.value, info.value


def reset_device_error(workspace, stream=None):
    _need(workspace, "workspace")
    rc = load_library().mla_reset_device_error(_ptr(workspace), _stream(stream, workspace.device))
    _check(rc, "mla_reset_device_error")
