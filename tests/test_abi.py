"""The C-ABI library builds, loads and exports its declared symbols; host-side
argument checks return the documented status codes without touching a GPU."""
import ctypes
import glob
import os
import re

import pytest

import mla_latent_attention_b200 as mla
from mla_latent_attention_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names.update(re.findall(r"MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    build.build()
    return mla.load_library()


def test_header_declares_the_boundary():
    names = _declared()
    assert {"mla_decode", "mla_merge_partials", "mla_decode_workspace_size"} <= names


def test_library_exports_every_declared_symbol(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", mla.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(\w+)", out))
    missing = _declared() - exported
    assert not missing, f"declared but not exported: {missing}"
    for name in _declared():
        assert hasattr(lib, name)
    assert set(mla.EXPORTED) <= exported


def test_library_leaves_none_of_its_own_symbols_undefined():
    """A shared library links even with references it does not define; they
    only fail when first called.  Every function of the library's namespace
    must be defined in the library itself."""
    import shutil
    import subprocess
    if not shutil.which("nm"):
        pytest.skip("nm not available")
    out = subprocess.run(["nm", "-D", "--undefined-only", mla.library_path()], capture_output=True, text=True,
                         check=True).stdout
    missing = [ln.split()[-1] for ln in out.splitlines() if "3mla" in ln or " mla_" in ln]
    assert not missing, missing


def test_library_is_sm100a_only():
    """The fatbinary is built for sm_100a (checked on the build command, not the binary)."""
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def _dims(**kw):
    d = dict(B=1, T=1, H=16, num_pages=16, max_pages_per_seq=16, page_table_stride=16,
             kv_dtype=0, out_dtype=0, num_splits=0, kernel=0, vis_lens=None, stage_event=None)
    d.update(kw)
    return mla.Dims(**d)


BAD_DIMS = [dict(B=0), dict(T=0), dict(T=9), dict(H=0), dict(T=8, H=129), dict(num_pages=0),
            dict(max_pages_per_seq=0), dict(page_table_stride=8), dict(kv_dtype=2),
            dict(out_dtype=5), dict(num_splits=-1), dict(kernel=7),
            dict(B=1 << 26, T=8, H=1),                 # 2^29 query rows: past the merge grid
            dict(kv_scale_per_tensor=2), dict(kv_scale_per_tensor=1),  # the latter with a bf16 cache
            dict(wait_limit_kcycles=-1),
            # B * max_pages_per_seq = 2^32 page slots: past the device schedule's 32-bit sums
            dict(B=1 << 20, max_pages_per_seq=1 << 12, page_table_stride=1 << 12)]


@pytest.mark.parametrize("bad", BAD_DIMS, ids=lambda d: ",".join(f"{k}={v}" for k, v in d.items()))
def test_invalid_dims_rejected_without_gpu(lib, bad):
    d = _dims(**bad)
    assert lib.mla_decode_workspace_size(ctypes.byref(d)) == -1
    buf = ctypes.create_string_buffer(4096 + 256)
    p = ctypes.c_void_p((ctypes.addressof(buf) + 255) & ~255)
    rc = lib.mla_decode(p, p, p, None, p, p, 0.1, p, None, ctypes.byref(d), p, 4096, None)
    assert rc == -1


def test_null_pointers_rejected_without_gpu(lib):
    d = _dims()
    buf = ctypes.create_string_buffer(4096 + 256)
    p = ctypes.c_void_p((ctypes.addressof(buf) + 255) & ~255)
    assert lib.mla_decode(None, p, p, None, p, p, 0.1, p, None, ctypes.byref(d), p, 4096, None) == -1
    assert lib.mla_decode(p, p, p, None, p, None, 0.1, p, None, ctypes.byref(d), p, 4096, None) == -1
    # FP8 needs kv_scale, bf16 must not have one
    d8 = _dims(kv_dtype=1)
    assert lib.mla_decode(p, p, p, None, p, p, 0.1, p, None, ctypes.byref(d8), p, 4096, None) == -1
    assert lib.mla_decode(p, p, p, p, p, p, 0.1, p, None, ctypes.byref(d), p, 4096, None) == -1
    # misaligned KV pool
    q = ctypes.c_void_p(p.value + 8)
    assert lib.mla_decode(p, p, q, None, p, p, 0.1, p, None, ctypes.byref(d), p, 4096, None) == -1
    # non-finite softmax scale
    assert lib.mla_decode(p, p, p, None, p, p, float("nan"), p, None, ctypes.byref(d), p, 4096, None) == -1
    # workspace missing or misaligned
    assert lib.mla_decode(p, p, p, None, p, p, 0.1, p, None, ctypes.byref(d), None, 4096, None) == -3
    assert lib.mla_decode(p, p, p, None, p, p, 0.1, p, None, ctypes.byref(d), q, 4096, None) == -3


def test_noalloc_argument_errors_enqueue_nothing(lib):
    """mla_decode_noalloc reports argument errors before it touches the
    device: without a GPU a call that reached its first CUDA call would
    return MLA_ERR_CUDA (-4), not MLA_ERR_INVALID_ARG (-1)."""
    d = _dims()
    buf = ctypes.create_string_buffer(4096 + 256)
    p = ctypes.c_void_p((ctypes.addressof(buf) + 255) & ~255)
    q = ctypes.c_void_p(p.value + 8)
    assert lib.mla_decode_noalloc(None, p, p, None, p, p, 0.1, p, None, ctypes.byref(d), None) == -1
    assert lib.mla_decode_noalloc(p, p, q, None, p, p, 0.1, p, None, ctypes.byref(d), None) == -1
    assert lib.mla_decode_noalloc(p, p, p, p, p, p, 0.1, p, None, ctypes.byref(d), None) == -1
    assert lib.mla_decode_noalloc(p, p, p, None, p, p, float("inf"), p, None, ctypes.byref(d), None) == -1
    bad = _dims(T=0)
    assert lib.mla_decode_noalloc(p, p, p, None, p, p, 0.1, p, None, ctypes.byref(bad), None) == -1


def test_merge_argument_checks_without_gpu(lib):
    buf = ctypes.create_string_buffer(4096 + 256)
    p = ctypes.c_void_p((ctypes.addressof(buf) + 255) & ~255)
    assert lib.mla_merge_partials(None, p, 2, 4, p, 0, None, None) == -1
    assert lib.mla_merge_partials(p, p, 0, 4, p, 0, None, None) == -1
    assert lib.mla_merge_partials(p, p, 4097, 4, p, 0, None, None) == -1
    assert lib.mla_merge_partials(p, p, 2, -1, p, 0, None, None) == -1
    assert lib.mla_merge_partials(p, p, 2, 4, p, 3, None, None) == -1
    assert lib.mla_merge_partials(ctypes.c_void_p(p.value + 4), p, 2, 4, p, 0, None, None) == -1


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4):
        assert lib.mla_status_string(code)
    assert lib.mla_status_string(-99) == b"unknown status"


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(mla.MlaError):
        mla.load_library(str(tmp_path / "missing.so"))


_LAYOUT_PROBE = r"""
#include <stddef.h>
#include <stdio.h>
#include "mla.h"
#define F(name) printf("%s %zu\n", #name, offsetof(mla_dims, name));
int main(void) {
    printf("sizeof %zu\n", sizeof(mla_dims));
    F(B) F(T) F(H) F(num_pages) F(max_pages_per_seq) F(page_table_stride) F(kv_dtype)
    F(out_dtype) F(num_splits) F(kernel) F(vis_lens) F(stage_event) F(kv_scale_per_tensor)
    F(wait_limit_kcycles)
    return 0;
}
"""


@pytest.mark.parametrize("compiler,std", [("gcc", "-std=c99"), ("g++", "-std=c++17")])
def test_header_compiles_standalone(tmp_path, compiler, std):
    """include/mla.h is plain C: it compiles on its own with warnings as errors."""
    import shutil
    import subprocess
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not available")
    src = tmp_path / ("probe.c" if compiler == "gcc" else "probe.cpp")
    src.write_text(_LAYOUT_PROBE)
    r = subprocess.run([compiler, std, "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                        os.path.join(ROOT, "include"), str(src), "-o", str(tmp_path / "probe")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_binding_struct_matches_header_layout(tmp_path):
    """The ctypes mirror of mla_dims has the header's size and field offsets."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = tmp_path / "probe.c"
    src.write_text(_LAYOUT_PROBE)
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    c = dict(line.split() for line in out if line)
    assert int(c.pop("sizeof")) == ctypes.sizeof(mla.Dims)
    assert list(c) == [f[0] for f in mla.Dims._fields_]
    for name, off in c.items():
        assert getattr(mla.Dims, name).offset == int(off), name


def _prototypes():
    """{name: number of parameters} of every MLA_API function in include/*.h."""
    protos = {}
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = re.sub(r"/\*.*?\*/", " ", open(h).read(), flags=re.S)
        for name, params in re.findall(r"MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(([^)]*)\)\s*;", src):
            params = params.strip()
            protos[name] = 0 if params in ("", "void") else params.count(",") + 1
    return protos


def test_binding_argument_counts_match_prototypes(lib):
    protos = _prototypes()
    assert set(protos) == _declared()
    for name, n in protos.items():
        fn = getattr(lib, name)
        assert fn.argtypes is not None, f"{name}: the binding sets no argtypes"
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)


def test_valid_calls_without_a_gpu_fail_with_a_cuda_status(lib):
    """With no CUDA device, well-formed calls return MLA_ERR_CUDA and record
    the CUDA error; nothing crashes and nothing falls back to the CPU.  (Only
    where no device exists: these calls pass host buffers.)"""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    buf = ctypes.create_string_buffer(1 << 16)
    p = ctypes.c_void_p((ctypes.addressof(buf) + 255) & ~255)
    d = _dims()
    assert lib.mla_decode_workspace_size(ctypes.byref(d)) == -4
    assert lib.mla_decode(p, p, p, None, p, p, 0.1, p, p, ctypes.byref(d), p, 4096, None) == -4
    assert lib.mla_last_cuda_error() != 0
    assert lib.mla_merge_partials(p, p, 2, 4, p, 0, p, None) == -4
    assert lib.mla_append_kv(p, p, p, None, p, p, ctypes.byref(d), None, None) == -4
