"""Host-side validation of every C-ABI call: each tensor pointer that is null or not 16-byte aligned,
and each non-positive size, is rejected with MLA_ERR_INVALID_ARG (a missing or short workspace with
MLA_ERR_WORKSPACE) before anything is enqueued.

The calls carry fake device addresses. Every case has exactly one bad argument, so validation
returns before a launch; the module still runs only where no GPU is visible, so that a gap in the
checks could never launch a kernel on fake pointers.
"""
import ctypes

import pytest
import torch

from mla_compressed_latent_b200 import _lib as L
from mla_compressed_latent_b200 import build as B

pytestmark = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="fake device pointers: host-side checks run where no GPU is visible")

GOOD = 4096      # a 16-byte aligned fake device address
ODD = 4100       # 4-byte aligned only
P, P_ODD = "P", "P_ODD"   # template markers: a good pointer, a misaligned one


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load()


def _dims(**kw):
    d = dict(H=128, D=128, d_r=64, d_c=512, d_v=128, g=8, page_size=64, sm_scale=1 / 192 ** 0.5,
             rms_eps=1e-6, rope_base=10000.0)
    d.update(kw)
    return L.MlaDims(*[d[f] for f, _ in L.MlaDims._fields_])


def _latent_cache(**kw):
    c = dict(latent=GOOD, latent_stride=576, rope=GOOD + 1024, rope_stride=576, num_pages=10)
    c.update(kw)
    return L.MlaLatentCache(c["latent"], c["latent_stride"], c["rope"], c["rope_stride"], c["num_pages"])


def _gqa_cache(**kw):
    c = dict(k=GOOD, k_stride=1024, v=GOOD, v_stride=1024, rope=GOOD, rope_stride=64, num_pages=10)
    c.update(kw)
    return L.MlaGqaCache(c["k"], c["k_stride"], c["v"], c["v_stride"], c["rope"], c["rope_stride"], c["num_pages"])


def _fp8_cache(**kw):
    c = dict(codes=GOOD, code_stride=512, scales=GOOD, rope=GOOD + 1024, rope_stride=576, num_pages=10)
    c.update(kw)
    return L.MlaLatentCacheFp8(c["codes"], c["code_stride"], c["scales"], c["rope"], c["rope_stride"], c["num_pages"])


BIG_WS = 1 << 40   # larger than any workspace the calls ask for


# name -> (template of positional arguments after (dims, dtype), indices of required tensor pointers,
#          indices of sizes that must be positive, index of the workspace pointer or None,
#          indices of optional pointers: NULL is allowed there, a misaligned address is not)
CALLS = {
    # B, s_q, x, C, w_dkv_kr, gamma, seqlens, table, max_pages, cache, ws, ws_bytes, stream
    "mla_append_cache": ([64, 1, P, 7168, P, P, P, P, 64, "LC", P, BIG_WS, None],
                         [2, 4, 6, 7], [0, 1, 3, 8], 10, [5]),
    "mla_append_cache_noalloc": ([64, 1, P, 7168, P, P, P, P, 64, "LC", None],
                                 [2, 4, 6, 7], [0, 1, 3, 8], None, [5]),
    # B, s_q, x, C, d_q, w_dq, gamma_q, w_uq, w_qr, q_nope, q_rope_raw, ws, ws_bytes, stream
    "mla_project_query": ([64, 1, P, 7168, 1536, P, P, P, P, P, P, P, BIG_WS, None],
                          [2, 5, 7, 8, 9, 10], [0, 1, 3, 4], 11, [6]),
    # B, s_q, q_nope, q_rope_raw, w_uk, seqlens, q_abs, stream
    "mla_absorb_q": ([64, 1, P, P, P, P, P, None], [2, 3, 4, 5, 6], [0, 1], None, []),
    # B, s_q, q_abs, cache, table, max_pages, seqlens, o_lat, lse, ws, ws_bytes, stream
    "mla_decode_absorbed": ([64, 1, P, "LC", P, 64, P, P, P, P, BIG_WS, None],
                            [2, 4, 6, 7, 8], [0, 1, 5], 9, []),
    # ... the same with the host copy of seqlens (NULL here: a host pointer is never faked)
    "mla_decode_absorbed_hinted": ([64, 1, P, "LC", P, 64, P, None, P, P, P, BIG_WS, None],
                                   [2, 4, 6, 8, 9], [0, 1, 5], 10, []),
    # B, s_q, x, C, w_dkv_kr, gamma, q_nope, q_rope_raw, w_uk, seqlens, table, max_pages, cache, q_abs,
    # ws, ws_bytes, stream
    "mla_append_cache_absorb_q": ([64, 1, P, 7168, P, P, P, P, P, P, P, 64, "LC", P, P, BIG_WS, None],
                                  [2, 4, 6, 7, 8, 9, 10, 13], [0, 1, 3, 11], 14, [5]),
    # B, s_q, o_lat, w_uv, out, w_o, C, out_model, stream
    "mla_out_proj": ([64, 1, P, P, P, P, 7168, P, None], [2, 3, 4, 7], [0, 1, 6], None, [5]),
    # B, s_q, q_nope, q_rope_raw, cache, table, max_pages, seqlens, out, lse, ws, ws_bytes, stream
    "mla_decode_gqla_grouped": ([32, 1, P, P, "GC", P, 128, P, P, P, P, BIG_WS, None],
                                [2, 3, 5, 7, 8, 9], [0, 1, 6], 10, []),
    # B, s_q, x, C, w_dkv_kr, gamma, w_uk_g, w_uv_g, seqlens, table, max_pages, cache, ws, ws_bytes, stream
    "mla_append_gqa_cache": ([32, 1, P, 7168, P, P, P, P, P, P, 128, "GC", P, BIG_WS, None],
                             [2, 4, 6, 7, 8, 9], [0, 1, 3, 10], 12, [5]),
    # w_uv, w_o, C, w_uvo, stream
    "mla_preabsorb_out_weights": ([P, P, 7168, P, None], [0, 1, 3], [2], None, []),
    # B, s_q, o_lat, w_uvo, C, out_model, stream
    "mla_out_proj_preabsorbed": ([64, 1, P, P, 7168, P, None], [2, 3, 5], [0, 1, 4], None, []),
    # latent, latent_stride, rows, codes, code_stride, scales, stream
    "mla_quantize_latent_fp8": ([P, 576, 1000, P, 512, P, None], [0, 3, 5], [1, 2, 4], None, []),
    # B, s_q, q_abs, cache, table, max_pages, seqlens, o_lat, lse, ws, ws_bytes, stream (one long
    # sequence: the CUDA-core decode then splits it and needs a workspace)
    "mla_decode_absorbed_fp8": ([1, 1, P, "FC", P, 2048, P, P, P, P, BIG_WS, None],
                                [2, 4, 6, 7, 8], [0, 1, 5], 9, []),
}
# calls without a token count (B, s_q): the overflow check does not apply
NO_TOKENS = {"mla_preabsorb_out_weights", "mla_quantize_latent_fp8"}


def _call(lib, name, args, dims=None, dtype=1):
    d = dims or _dims()
    conv = []
    for a in args:
        if a == "LC":
            conv.append(ctypes.byref(_latent_cache()))
        elif a == "GC":
            conv.append(ctypes.byref(_gqa_cache()))
        elif a == "FC":
            conv.append(ctypes.byref(_fp8_cache()))
        elif a == P:
            conv.append(ctypes.c_void_p(GOOD))
        elif a == P_ODD:
            conv.append(ctypes.c_void_p(ODD))
        else:
            conv.append(a)
    return getattr(lib, name)(ctypes.byref(d), dtype, *conv)


def _cases():
    for name, (tmpl, ptrs, sizes, ws, optional) in CALLS.items():
        for i in ptrs:
            yield name, i, None, L.MLA_ERR_INVALID_ARG
            yield name, i, P_ODD, L.MLA_ERR_INVALID_ARG
        for i in optional:
            yield name, i, P_ODD, L.MLA_ERR_INVALID_ARG
        for i in sizes:
            yield name, i, 0, L.MLA_ERR_INVALID_ARG
            yield name, i, -3, L.MLA_ERR_INVALID_ARG
        if ws is not None:
            yield name, ws, None, L.MLA_ERR_WORKSPACE
            yield name, ws + 1, 16, L.MLA_ERR_WORKSPACE
            yield name, ws, P_ODD, L.MLA_ERR_INVALID_ARG   # a misaligned pointer, like any other


@pytest.mark.parametrize("name,i,bad,want", list(_cases()), ids=lambda v: str(v))
def test_one_bad_argument_is_rejected(lib, name, i, bad, want):
    tmpl = list(CALLS[name][0])
    tmpl[i] = bad
    assert _call(lib, name, tmpl) == want


@pytest.mark.parametrize("name", list(CALLS))
def test_bad_dtype_and_dims_are_rejected(lib, name):
    tmpl = CALLS[name][0]
    assert _call(lib, name, tmpl, dtype=7) == L.MLA_ERR_INVALID_ARG
    for bad in (_dims(H=0), _dims(d_c=-1), _dims(page_size=32), _dims(sm_scale=-1.0), _dims(sm_scale=float("nan"))):
        assert _call(lib, name, tmpl, dims=bad) == L.MLA_ERR_INVALID_ARG


@pytest.mark.parametrize("name", [n for n in CALLS if n not in NO_TOKENS])
def test_token_count_past_int32_is_rejected(lib, name):
    """B * s_q is formed in 32 bits: a product past INT32_MAX is an invalid argument, found before
    any size is computed from it."""
    tmpl = list(CALLS[name][0])
    tmpl[0], tmpl[1] = 1 << 16, 1 << 16
    assert _call(lib, name, tmpl) == L.MLA_ERR_INVALID_ARG
    tmpl[0], tmpl[1] = 46341, 46341
    assert _call(lib, name, tmpl) == L.MLA_ERR_INVALID_ARG


def test_zero_score_scale_selects_the_default(lib):
    """sm_scale = 0 is valid (the library then uses 1/sqrt(D + d_r)); the size queries answer for it."""
    d = _dims(sm_scale=0.0)
    assert lib.mla_decode_workspace_size(ctypes.byref(d), 1, 64, 1, 64) > 0
    assert lib.mla_append_workspace_size(ctypes.byref(d), 64, 1, 7168) > 0
    big = _dims(sm_scale=0.0)
    assert lib.mla_append_workspace_size(ctypes.byref(big), 1 << 16, 1 << 16, 7168) == 0


@pytest.mark.parametrize("field,value", [("latent", 0), ("rope", 0), ("latent", ODD), ("latent_stride", 577),
                                         ("num_pages", 0)])
def test_bad_latent_cache_is_rejected(lib, field, value):
    cache = _latent_cache(**{field: value})
    d = _dims()
    g = ctypes.c_void_p(GOOD)
    rc = lib.mla_decode_absorbed(ctypes.byref(d), 1, 64, 1, g, ctypes.byref(cache), g, 64, g, g, g, g, BIG_WS, None)
    assert rc == L.MLA_ERR_INVALID_ARG
    rc = lib.mla_append_cache(ctypes.byref(d), 1, 64, 1, g, 7168, g, None, g, g, 64, ctypes.byref(cache), g,
                              BIG_WS, None)
    assert rc == L.MLA_ERR_INVALID_ARG
    rc = lib.mla_append_cache_absorb_q(ctypes.byref(d), 1, 64, 1, g, 7168, g, None, g, g, g, g, g, 64,
                                       ctypes.byref(cache), g, g, BIG_WS, None)
    assert rc == L.MLA_ERR_INVALID_ARG


@pytest.mark.parametrize("field,value", [("k", 0), ("v", 0), ("rope", 0), ("k", ODD), ("k_stride", 1000),
                                         ("num_pages", 0)])
def test_bad_gqa_cache_is_rejected(lib, field, value):
    cache = _gqa_cache(**{field: value})
    d = _dims()
    g = ctypes.c_void_p(GOOD)
    rc = lib.mla_decode_gqla_grouped(ctypes.byref(d), 1, 32, 1, g, g, ctypes.byref(cache), g, 128, g, g, g, g,
                                     BIG_WS, None)
    assert rc == L.MLA_ERR_INVALID_ARG


@pytest.mark.parametrize("field,value", [("codes", 0), ("scales", 0), ("rope", 0), ("codes", ODD), ("scales", ODD),
                                         ("code_stride", 500), ("code_stride", 520), ("rope_stride", 63),
                                         ("num_pages", 0)])
def test_bad_fp8_cache_is_rejected(lib, field, value):
    cache = _fp8_cache(**{field: value})
    d = _dims()
    g = ctypes.c_void_p(GOOD)
    rc = lib.mla_decode_absorbed_fp8(ctypes.byref(d), 1, 64, 1, g, ctypes.byref(cache), g, 64, g, g, g, g, BIG_WS,
                                     None)
    assert rc == L.MLA_ERR_INVALID_ARG


def test_fp8_quantiser_wants_whole_16_value_rows(lib):
    g = ctypes.c_void_p(GOOD)
    d = _dims(d_c=520)
    assert lib.mla_quantize_latent_fp8(ctypes.byref(d), 1, g, 528, 10, g, 528, g, None) == L.MLA_ERR_UNSUPPORTED
