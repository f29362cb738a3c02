"""A bounded wait inside a tensor-core kernel that runs out: the kernel records MLA_ERR_TIMEOUT in
the device status word, stops, lets every load it issued land, frees its tensor memory and returns,
and the next call on the same context is clean and correct.

The wait is made to run out without faulting anything: the test-hooks build of the library
(libmla_testhooks.so, the same sources compiled with MLA_TEST_HOOKS) has a switch that makes each
per-head GEMM's MMA issuer first wait, with a 10 ms limit, for a barrier phase that only its own
later commit could complete.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

import synth
from oracle import mla_oracle as O
from mla_compressed_latent_b200 import _lib as L
from mla_compressed_latent_b200 import build as B
from mla_compressed_latent_b200.ops import Dims

from _cases import TOL, Case, max_rel_err

pytestmark = pytest.mark.gpu


def _load_test_lib():
    path = B.build_test_hooks()
    lib = ctypes.CDLL(path)
    for name, (res, args) in L.SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    lib.mla_test_set_stall.restype = ctypes.c_int32
    lib.mla_test_set_stall.argtypes = [ctypes.c_int32]
    lib.mla_test_set_two_launches.restype = ctypes.c_int32
    lib.mla_test_set_two_launches.argtypes = [ctypes.c_int32]
    return lib


def test_wait_that_runs_out_reports_timeout_then_next_call_is_clean():
    lib = _load_test_lib()
    w = synth.workload("dsv3_b64_l4096", B=4, lengths=("list", (4096, 100, 7, 2000)))
    case = Case(w)
    dev = case.to_device()
    d = Dims.of(w).c()
    q_abs = torch.empty(w.B, w.s_q, w.H, w.d_c + w.d_r, dtype=torch.bfloat16, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def absorb():
        return lib.mla_absorb_q(ctypes.byref(d), L.MLA_BF16, w.B, w.s_q, ctypes.c_void_p(dev["q_nope"].data_ptr()),
                                ctypes.c_void_p(dev["q_rope_raw"].data_ptr()), ctypes.c_void_p(dev["W_UK"].data_ptr()),
                                ctypes.c_void_p(dev["seqlens"].data_ptr()), ctypes.c_void_p(q_abs.data_ptr()), stream)

    assert lib.mla_check_status(stream) == L.MLA_OK
    assert lib.mla_test_set_stall(1) == L.MLA_OK
    assert absorb() == L.MLA_OK                       # enqueued; the kernel gives up on the device
    assert lib.mla_check_status(stream) == L.MLA_ERR_TIMEOUT
    assert lib.mla_test_set_stall(0) == L.MLA_OK
    q_abs.zero_()
    assert absorb() == L.MLA_OK
    assert lib.mla_check_status(stream) == L.MLA_OK   # the context is usable and the status clean
    got = q_abs.double().cpu().numpy()
    for b in range(w.B):
        L_b = int(case.lens[b])
        ref = O.absorb_query(case.q_nope64[b], case.q_rope_raw64[b], case.W64["W_UK"], O.token_positions(L_b, 1))
        err = max_rel_err(got[b], ref)
        assert err <= TOL["bf16"]["out"], f"seq {b}: max|Δ|/max|ref| = {err:.3e}"


@pytest.mark.parametrize("lens", [[131072], list(np.random.default_rng(11).integers(1, 2000, 200))])
def test_decode_as_two_launches_merges_cut_sequences(lens):
    """The decode's fallback when the runtime refuses its cooperative launch: the decode, then the
    merge kernel. Cut sequences (one spanning every pair; 200 ragged ones) against the oracle."""
    lib = _load_test_lib()
    w = synth.workload("dsv3_b64_l4096", B=len(lens), lengths=("list", tuple(int(x) for x in lens)), pages="random")
    case = Case(w, with_weights=False)
    dev = case.to_device()
    d = Dims.of(w).c()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    max_pages = dev["table"].shape[1]
    ws = torch.empty(lib.mla_decode_workspace_size(ctypes.byref(d), L.MLA_BF16, w.B, 1, max_pages), dtype=torch.uint8,
                     device="cuda")
    o_lat = torch.empty(w.B, 1, w.H, w.d_c, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(w.B, 1, w.H, dtype=torch.float32, device="cuda")
    pool = dev["pool"]
    cache = L.MlaLatentCache(pool.data_ptr(), pool.stride(0), pool[:, w.d_c:].data_ptr(), pool.stride(0), case.num_pages)
    assert lib.mla_test_set_two_launches(1) == L.MLA_OK
    try:
        rc = lib.mla_decode_absorbed(ctypes.byref(d), L.MLA_BF16, w.B, 1, ctypes.c_void_p(dev["q_abs"].data_ptr()),
                                     ctypes.byref(cache), ctypes.c_void_p(dev["table"].data_ptr()), max_pages,
                                     ctypes.c_void_p(dev["seqlens"].data_ptr()), ctypes.c_void_p(o_lat.data_ptr()),
                                     ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                                     ws.numel(), stream)
    finally:
        lib.mla_test_set_two_launches(0)
    assert rc == L.MLA_OK
    assert lib.mla_check_status(stream) == L.MLA_OK
    got_o, got_l = o_lat.double().cpu().numpy(), lse.double().cpu().numpy()
    for b in range(w.B):
        c, kr = case.seq_rows64(b)
        ref_o, ref_l = O.absorbed_decode(case.q_abs64[b], c, kr, int(case.lens[b]), w.sm_scale)
        err = max_rel_err(got_o[b], ref_o)
        assert err <= TOL["bf16"]["out"], f"seq {b}: max|Δ|/max|ref| = {err:.3e}"
        assert float(np.abs(got_l[b] - ref_l).max()) <= TOL["bf16"]["lse"], f"seq {b}: lse"
