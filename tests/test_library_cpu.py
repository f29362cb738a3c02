"""CPU-side checks of the C-ABI library: it builds, loads, exports every declared symbol, and its
host-side validation rejects bad arguments before touching the GPU. No compute call is made."""
import ctypes
import os
import re

import pytest

from mla_compressed_latent_b200 import _lib as L
from mla_compressed_latent_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(mla_\w+)\s*\(", txt, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load()


def test_header_declares_the_boundary():
    names = _declared()
    for required in ["mla_append_cache", "mla_absorb_q", "mla_decode_absorbed", "mla_decode_gqla_grouped",
                     "mla_out_proj", "mla_decode_workspace_size", "mla_check_status", "mla_status_string"]:
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_library_exports_nothing_else():
    """Built with hidden visibility: the dynamic symbol table holds the declared C calls and no C++
    symbol, so two builds loaded in one process (the library and its test-hooks build) cannot bind
    each other's inline statics (a kernel-attribute cache shared that way made a launch fail)."""
    import shutil
    import subprocess
    nm = shutil.which("nm")
    if nm is None:
        pytest.skip("nm not available")
    path = B.build()
    out = subprocess.run([nm, "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    funcs = sorted(ln.split()[-1] for ln in out.splitlines() if len(ln.split()) == 3 and ln.split()[1] in "TtWw")
    assert funcs == _declared(), sorted(set(funcs) ^ set(_declared()))
    # and the binding knows each of them with a signature
    assert set(_declared()) <= set(L.SIGNATURES)


def test_status_strings(lib):
    for code in range(7):
        s = lib.mla_status_string(code).decode()
        assert s.startswith("MLA_")
    assert "sm_100a" in lib.mla_build_info().decode()


def _dims(**kw):
    d = dict(H=128, D=128, d_r=64, d_c=512, d_v=128, g=0, page_size=64, sm_scale=1 / 192 ** 0.5,
             rms_eps=1e-6, rope_base=10000.0)
    d.update(kw)
    return L.MlaDims(*[d[f] for f, _ in L.MlaDims._fields_])


def test_invalid_dims_rejected_before_any_launch(lib):
    p = ctypes.c_void_p(16)
    cache = L.MlaLatentCache(16, 576, 16 + 1024, 576, 10)
    for bad in [_dims(H=0), _dims(d_r=3), _dims(page_size=32), _dims(sm_scale=-1.0), _dims(d_c=-1)]:
        rc = lib.mla_decode_absorbed(ctypes.byref(bad), 1, 1, 1, p, ctypes.byref(cache), p, 1, p, p, p, None, 0, None)
        assert rc == L.MLA_ERR_INVALID_ARG


def test_null_and_misaligned_pointers_rejected(lib):
    d = _dims()
    good = ctypes.c_void_p(4096)
    odd = ctypes.c_void_p(4098)
    cache = L.MlaLatentCache(4096, 576, 4096 + 1024, 576, 10)
    assert lib.mla_decode_absorbed(ctypes.byref(d), 1, 1, 1, None, ctypes.byref(cache), good, 1, good, good, good,
                                   None, 0, None) == L.MLA_ERR_INVALID_ARG
    assert lib.mla_decode_absorbed(ctypes.byref(d), 1, 1, 1, odd, ctypes.byref(cache), good, 1, good, good, good,
                                   None, 0, None) == L.MLA_ERR_INVALID_ARG
    bad_stride = L.MlaLatentCache(4096, 577, 4096 + 1024, 576, 10)   # 1154 bytes: not a multiple of 16
    assert lib.mla_decode_absorbed(ctypes.byref(d), 1, 1, 1, good, ctypes.byref(bad_stride), good, 1, good, good,
                                   good, None, 0, None) == L.MLA_ERR_INVALID_ARG
    assert lib.mla_absorb_q(ctypes.byref(d), 1, 0, 1, good, good, good, good, good, None) == L.MLA_ERR_INVALID_ARG
    assert lib.mla_absorb_q(ctypes.byref(d), 7, 1, 1, good, good, good, good, good, None) == L.MLA_ERR_INVALID_ARG


def test_append_rejects_missing_workspace(lib):
    d = _dims()
    good = ctypes.c_void_p(4096)
    cache = L.MlaLatentCache(4096, 576, 4096 + 1024, 576, 10)
    need = lib.mla_append_workspace_size(ctypes.byref(d), 64, 1, 7168)
    assert need > 0
    rc = lib.mla_append_cache(ctypes.byref(d), 1, 64, 1, good, 7168, good, None, good, good, 64, ctypes.byref(cache),
                              None, 0, None)
    assert rc == L.MLA_ERR_WORKSPACE


def test_project_query_validates_before_any_launch(lib):
    d = _dims()
    good = ctypes.c_void_p(4096)
    odd = ctypes.c_void_p(4100)
    need = lib.mla_query_workspace_size(ctypes.byref(d), 64, 1, 7168, 1536)
    # at least the fp32 partial sums of one K slice and the fp32-sized c_q rows
    assert need >= 2 * 64 * 1536 * 4
    assert lib.mla_query_workspace_size(ctypes.byref(d), 64, 1, 7168, 0) == 0
    args = [good, 7168, 1536, good, None, good, good, good, good]
    rc = lib.mla_project_query(ctypes.byref(d), 1, 64, 1, *args, None, 0, None)
    assert rc == L.MLA_ERR_WORKSPACE
    for i in (0, 3, 5, 6, 7, 8):   # x, w_dq, w_uq, w_qr, q_nope, q_rope_raw
        for bad in (None, odd):
            a = list(args)
            a[i] = bad
            assert lib.mla_project_query(ctypes.byref(d), 1, 64, 1, *a, good, need, None) == L.MLA_ERR_INVALID_ARG
    assert lib.mla_project_query(ctypes.byref(d), 1, 0, 1, *args, good, need, None) == L.MLA_ERR_INVALID_ARG
    assert lib.mla_project_query(ctypes.byref(d), 5, 64, 1, *args, good, need, None) == L.MLA_ERR_INVALID_ARG


def test_gqla_rejects_bad_groups(lib):
    d = _dims(g=3)
    good = ctypes.c_void_p(4096)
    cache = L.MlaGqaCache(4096, 2048, 4096, 2048, 4096, 64, 10)
    rc = lib.mla_decode_gqla_grouped(ctypes.byref(d), 1, 1, 1, good, good, ctypes.byref(cache), good, 1, good, good,
                                     good, None, 0, None)
    assert rc == L.MLA_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path):
    saved = L._lib
    try:
        L._lib = None
        with pytest.raises(FileNotFoundError):
            L.load(str(tmp_path / "libmla.so"))
    finally:
        L._lib = saved
