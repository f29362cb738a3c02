"""mla_append_cache_noalloc: the cache append for callers that cannot allocate device memory.

Such callers (a framework whose memory pool owns the device, a plugin that only receives the
tensors of the call, a serving process that must not call cudaMalloc) get the same result as
mla_append_cache without passing a workspace: the partial sums live in a fixed buffer inside the
library. These checks call it through the C ABI and compare it with the workspace entry point on
two calls in a row (the shared buffer keeps the first call's contents when the second one runs), and
the rows each call writes with the fp64 oracle's cache rows.
This file is collected last so that a failure here never hides the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from oracle import mla_oracle as O
from mla_compressed_latent_b200 import _lib as L
from mla_compressed_latent_b200 import ops
from mla_compressed_latent_b200.ops import Dims, LatentCache

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}


def _noalloc(dims, x, w, seqlens, table, cache):
    lib = L.load()
    d = dims.c()
    cc = cache.c()
    return lib.mla_append_cache_noalloc(
        ctypes.byref(d), L.MLA_F32 if x.dtype == torch.float32 else L.MLA_BF16, x.shape[0], x.shape[1],
        ctypes.c_void_p(x.data_ptr()), x.shape[2], ctypes.c_void_p(w.data_ptr()), None,
        ctypes.c_void_p(seqlens.data_ptr()), ctypes.c_void_p(table.data_ptr()), table.shape[1], ctypes.byref(cc),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("name,B", [("dsv3_b64_l4096", 64), ("smallem_fp32", 3)])
def test_noalloc_append_matches_workspace_append_on_two_calls(name, B):
    w = synth.workload(name, B=B, lengths=("list", tuple(300 + 70 * i for i in range(B))), pages="random")
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    lens = synth.seq_lengths(w)
    table, num_pages = synth.block_table(w, lens)
    W = synth.weights(w)
    wcat = torch.from_numpy(np.concatenate([W["W_DKV"], W["W_KR"]], 1)).to(device="cuda", dtype=dt)
    tb = torch.from_numpy(table).cuda()
    dims = Dims.of(w)
    rng = np.random.default_rng(5)
    pool_ref = torch.zeros(num_pages * 64, w.d_c + w.d_r, dtype=dt, device="cuda")
    pool_new = torch.zeros_like(pool_ref)
    ref_cache = LatentCache(pool_ref[:, :w.d_c], pool_ref[:, w.d_c:], num_pages)
    new_cache = LatentCache(pool_new[:, :w.d_c], pool_new[:, w.d_c:], num_pages)
    for call in range(2):
        # each call appends a different token at a different position of every sequence
        x = torch.from_numpy(rng.standard_normal((B, 1, w.C), dtype=np.float32)).to(device="cuda", dtype=dt)
        sl = torch.from_numpy(lens - 7 * call).cuda()
        ops.mla_append_cache(dims, x, wcat, None, sl, tb, ref_cache)
        rc = _noalloc(dims, x, wcat, sl, tb, new_cache)
        assert rc == L.MLA_OK, ops.mla_status_string(rc)
        torch.cuda.synchronize()
        assert ops.mla_check_status() == 0
        ref = pool_ref.double().cpu().numpy()
        got = pool_new.double().cpu().numpy()
        err = np.abs(got - ref).max() / np.abs(ref).max()
        assert err <= TOL[w.dtype], f"call {call}: max|Δ|/max|ref| = {err:.3e}"
        # rows written on this call are non-zero in both pools
        pos = (lens - 7 * call - 1).astype(np.int64)
        rows = table[np.arange(B), pos // 64].astype(np.int64) * 64 + pos % 64
        assert np.all(np.abs(got[rows]).max(axis=1) > 0)
        # and they are the oracle's cache rows of these tokens at these positions
        w64 = wcat.double().cpu().numpy()   # the weights as stored (the call reads them in its dtype)
        c, kr = O.latent_rows(x[:, 0].double().cpu().numpy(), w64[:, :w.d_c], w64[:, w.d_c:], pos, None,
                              w.rms_eps, w.rope_base)
        want = np.concatenate([c, kr], 1)
        err = np.abs(got[rows] - want).max() / np.abs(want).max()
        assert err <= TOL[w.dtype], f"call {call}: rows vs oracle max|Δ|/max|ref| = {err:.3e}"


def test_noalloc_append_rejects_batches_beyond_its_buffer():
    w = synth.workload("dsv3_b64_l4096", B=2000, lengths=("fixed", 64))
    dims = Dims.of(w)
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    x = torch.zeros(1, dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros(64, 576, dtype=torch.bfloat16, device="cuda")
    cache = LatentCache(pool[:, :512], pool[:, 512:], 1)
    lib = L.load()
    d = dims.c()
    cc = cache.c()
    rc = lib.mla_append_cache_noalloc(ctypes.byref(d), L.MLA_BF16, 2000, 1, ctypes.c_void_p(x.data_ptr()), 7168,
                                      ctypes.c_void_p(x.data_ptr()), None, ctypes.c_void_p(dummy.data_ptr()),
                                      ctypes.c_void_p(dummy.data_ptr()), 1, ctypes.byref(cc), None)
    assert rc == L.MLA_ERR_WORKSPACE   # 2000 * 576 values of partial sums do not fit in 4 MiB
