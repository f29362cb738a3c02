"""GPU parity: every C-ABI call against the fp64 oracle on the same seeded, stored inputs.

Tolerances (the project's numeric bar): fp32 max|Δ| <= 1e-5·max|ref|; bf16 storage with fp32
accumulation max|Δ| <= 2e-2·max|ref| and |Δ lse| <= 1e-3.
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import fp8_cache as F
from oracle import mla_oracle as O
from mla_compressed_latent_b200 import _lib as L
from mla_compressed_latent_b200 import ops
from mla_compressed_latent_b200.ops import Dims, LatentCache, LatentCacheFp8, GqaCache

from _cases import TOL, Case, as_stored, max_rel_err

pytestmark = pytest.mark.gpu


def _cache(dev, case):
    pool = dev["pool"]
    d_c = case.w.d_c
    return LatentCache(pool[:, :d_c], pool[:, d_c:], case.num_pages)


def _oracle_absorbed(case, q_abs64, pool=None, heads=None, seqs=None):
    """fp64 absorbed decode of the given sequences (all by default) and heads."""
    w = case.w
    seqs = range(w.B) if seqs is None else seqs
    o, l = {}, {}
    for b in seqs:
        c, kr = case.seq_rows64(b, pool)
        q = q_abs64[b] if heads is None else q_abs64[b][:, heads]
        o[b], l[b] = O.absorbed_decode(q, c, kr, int(case.lens[b]), w.sm_scale)
    return o, l


def _assert_close(got, ref, dtype, what, key="out"):
    err = max_rel_err(got, ref)
    assert err <= TOL[dtype][key], f"{what}: max|Δ|/max|ref| = {err:.3e}"
    return err


def _assert_lse(got, ref, dtype, what):
    err = float(np.abs(np.asarray(got, np.float64) - ref).max())
    bar = TOL[dtype]["lse"] * (1 if dtype == "bf16" else max(1.0, float(np.abs(ref).max())))
    assert err <= bar, f"{what}: max|Δ lse| = {err:.3e}"


# ------------------------------------------------------------------------------------------------
# a3 + a4 on their own: decode over a stored cache with a stored absorbed query
# ------------------------------------------------------------------------------------------------

SMALL_DECODE = [
    # (lens, s_q, pages)
    ([1], 1, "contiguous"),
    ([63], 1, "contiguous"),
    ([64, 65], 1, "random"),
    ([127, 1000, 3], 1, "random"),
    ([4096, 129, 2049, 64, 5000], 1, "contiguous"),
    ([2, 64, 77, 300], 2, "random"),
    ([4, 513, 1029], 4, "random"),
    # work-split corners of the tensor-core kernel: fewer tiles than worker pairs, one sequence
    # spanning every pair, many short sequences per pair, exact page multiples
    ([1, 2], 1, "contiguous"),
    ([131072], 1, "random"),
    (list(np.random.default_rng(11).integers(1, 2000, 200)), 1, "random"),
    ([64 * 70] * 3 + [64 * 5 + 1], 1, "contiguous"),
    # several new tokens (one worker pair per token, the pairs of a sequence walking its tiles
    # together): a token whose visible positions end on a page boundary sees its sequence's last
    # page fully masked; with s_q = 4 the mask reaches into the page before; odd s_q leaves pairs
    # idle; one long sequence cut between every group; many short ones per group
    ([65, 129, 64 * 5 + 1, 2], 2, "random"),
    ([65, 66, 4, 64 * 3 + 2, 64 * 3 + 3], 4, "random"),
    ([100, 5000, 3, 64 * 40 + 1], 3, "contiguous"),
    ([8, 70, 64 * 20 + 3], 8, "random"),
    ([131072], 2, "random"),
    (list(np.random.default_rng(12).integers(4, 3000, 150)), 4, "random"),
]


@pytest.mark.parametrize("lens,s_q,pages", SMALL_DECODE)
def test_decode_absorbed_small(lens, s_q, pages):
    w = synth.workload("dsv3_b64_l4096", B=len(lens), s_q=s_q, lengths=("list", tuple(lens)), pages=pages)
    case = Case(w, with_weights=False)
    dev = case.to_device()
    dims = Dims.of(w)
    o_lat, lse = ops.mla_decode_absorbed(dims, dev["q_abs"], _cache(dev, case), dev["table"], dev["seqlens"])
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    ref_o, ref_l = _oracle_absorbed(case, case.q_abs64)
    got_o = o_lat.float().cpu().numpy()
    got_l = lse.cpu().numpy()
    for b in range(w.B):
        _assert_close(got_o[b], ref_o[b], "bf16", f"o_lat seq {b}")
        _assert_lse(got_l[b], ref_l[b], "bf16", f"lse seq {b}")


def test_decode_workspace_reused_across_calls():
    """One zero-filled workspace for several calls whose sequences are cut between worker pairs in
    different places: the per-sequence part counters left by a call must not leak into the next."""
    rounds = [[4096, 129, 2049, 64, 5000], [300, 7000, 65], [131072], [4096] * 9, [1, 2]]
    max_b = max(len(r) for r in rounds)
    dims0 = Dims.of(synth.workload("dsv3_b64_l4096", B=max_b, lengths=("list", tuple([64] * max_b))))
    need = ops.mla_decode_workspace_size(dims0, torch.bfloat16, max_b, 1, 2048)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for i, lens in enumerate(rounds):
        w = synth.workload("dsv3_b64_l4096", B=len(lens), lengths=("list", tuple(lens)), pages="random")
        case = Case(w, with_weights=False)
        dev = case.to_device()
        assert dev["table"].shape[1] <= 2048
        o_lat, lse = ops.mla_decode_absorbed(Dims.of(w), dev["q_abs"], _cache(dev, case), dev["table"],
                                             dev["seqlens"], workspace=ws)
        torch.cuda.synchronize()
        assert ops.mla_check_status() == 0
        ref_o, ref_l = _oracle_absorbed(case, case.q_abs64)
        for b in range(w.B):
            _assert_close(o_lat[b].float().cpu().numpy(), ref_o[b], "bf16", f"call {i} o_lat seq {b}")
            _assert_lse(lse[b].cpu().numpy(), ref_l[b], "bf16", f"call {i} lse seq {b}")


def test_decode_absorbed_fp32_smallem_shapes():
    w = synth.workload("smallem_fp32", B=3, lengths=("list", (512, 65, 1)))
    case = Case(w, with_weights=False)
    dev = case.to_device()
    o_lat, lse = ops.mla_decode_absorbed(Dims.of(w), dev["q_abs"], _cache(dev, case), dev["table"], dev["seqlens"])
    ref_o, ref_l = _oracle_absorbed(case, case.q_abs64)
    for b in range(w.B):
        _assert_close(o_lat[b].cpu().numpy(), ref_o[b], "f32", f"o_lat seq {b}")
        _assert_lse(lse[b].cpu().numpy(), ref_l[b], "f32", f"lse seq {b}")


@pytest.mark.parametrize("name", ["dsv3_b64_l4096", "longctx_b8"])
def test_decode_absorbed_full_size(name):
    """Full size, the bench's launch configuration; oracle on every sequence (sampled heads for the
    long-context case, every head otherwise)."""
    w = synth.workload(name)
    case = Case(w, with_weights=False)
    dev = case.to_device()
    o_lat, lse = ops.mla_decode_absorbed(Dims.of(w), dev["q_abs"], _cache(dev, case), dev["table"], dev["seqlens"])
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    heads = None if name == "dsv3_b64_l4096" else np.random.default_rng(7).choice(w.H, 12, replace=False)
    ref_o, ref_l = _oracle_absorbed(case, case.q_abs64, heads=heads)
    got_o = o_lat.float().cpu().numpy()
    got_l = lse.cpu().numpy()
    for b in range(w.B):
        go = got_o[b] if heads is None else got_o[b][:, heads]
        gl = got_l[b] if heads is None else got_l[b][:, heads]
        _assert_close(go, ref_o[b], "bf16", f"o_lat seq {b}")
        _assert_lse(gl, ref_l[b], "bf16", f"lse seq {b}")


@pytest.mark.parametrize("name", ["mtp_sq2_b128", "mtp_sq4_b128"])
def test_decode_mtp_random_pages_full_size_sampled(name):
    """Multi-token step, random page table, full batch; oracle on a seeded sample of sequences."""
    w = synth.workload(name)
    case = Case(w, with_weights=False)
    dev = case.to_device()
    o_lat, lse = ops.mla_decode_absorbed(Dims.of(w), dev["q_abs"], _cache(dev, case), dev["table"], dev["seqlens"])
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    seqs = sorted(np.random.default_rng(8).choice(w.B, 6, replace=False).tolist())
    ref_o, ref_l = _oracle_absorbed(case, case.q_abs64, seqs=seqs)
    for b in seqs:
        _assert_close(o_lat[b].float().cpu().numpy(), ref_o[b], "bf16", f"o_lat seq {b}")
        _assert_lse(lse[b].cpu().numpy(), ref_l[b], "bf16", f"lse seq {b}")


# ------------------------------------------------------------------------------------------------
# a1, a2, a5 on their own
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("name,B", [("dsv3_b64_l4096", 64), ("dsv3_b64_l4096", 5), ("smallem_fp32", 1)])
def test_append_cache(name, B):
    w = synth.workload(name, B=B, lengths=("list", tuple([4096 - 3 * i for i in range(B)] if B > 1 else [512])))
    case = Case(w)
    dev = case.to_device()
    cache = _cache(dev, case)
    before = dev["pool"].clone()
    ops.mla_append_cache(Dims.of(w), dev["x"], dev["w_dkv_kr"], None, dev["seqlens"], dev["table"], cache)
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    pool = dev["pool"].cpu()
    pos = (case.lens - 1).astype(np.int64)
    c_ref, kr_ref = O.latent_rows(case.x64[:, 0], case.W64["W_DKV"], case.W64["W_KR"], pos, None, w.rms_eps, w.rope_base)
    rows = case.table[np.arange(B), pos // 64].astype(np.int64) * 64 + pos % 64
    got = pool[torch.from_numpy(rows)].to(torch.float64).numpy()
    _assert_close(got[:, :w.d_c], c_ref, w.dtype, "appended latent")
    _assert_close(got[:, w.d_c:], kr_ref, w.dtype, "appended rope key")
    if w.dtype == "bf16":   # one rounding of an fp32-accurate value: within one bf16 ulp
        assert np.all(np.abs(got[:, :w.d_c] - c_ref) <= 2.0 ** -8 * np.abs(c_ref) + 1e-3 * np.abs(c_ref).max())
    # nothing else in the pool moved
    mask = torch.ones(pool.shape[0], dtype=torch.bool)
    mask[torch.from_numpy(rows)] = False
    assert torch.equal(pool[mask], before.cpu()[mask])


def test_append_cache_row_width_not_a_multiple_of_four():
    """d_c + d_r = 39 (separate latent and RoPE pools, 16-byte strides): the finish sums its split-K
    slices one column per thread instead of in 16-byte pieces. Rows against the oracle."""
    w = synth.workload("smallem_fp32", d_c=33, d_r=6, B=3, lengths=("list", (77, 5, 130)))
    case = Case(w)
    dev = case.to_device()
    rows_total = case.num_pages * 64
    latent = torch.zeros(rows_total, 36, dtype=torch.float32, device="cuda")[:, :w.d_c]
    rope = torch.zeros(rows_total, 8, dtype=torch.float32, device="cuda")[:, :w.d_r]
    cache = LatentCache(latent, rope, case.num_pages)
    ops.mla_append_cache(Dims.of(w), dev["x"], dev["w_dkv_kr"], None, dev["seqlens"], dev["table"], cache)
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    pos = (case.lens - 1).astype(np.int64)
    c_ref, kr_ref = O.latent_rows(case.x64[:, 0], case.W64["W_DKV"], case.W64["W_KR"], pos, None, w.rms_eps,
                                  w.rope_base)
    rows = torch.from_numpy(case.table[np.arange(w.B), pos // 64].astype(np.int64) * 64 + pos % 64)
    _assert_close(latent.cpu()[rows].double().numpy(), c_ref, w.dtype, "appended latent")
    _assert_close(rope.cpu()[rows].double().numpy(), kr_ref, w.dtype, "appended rope key")


def test_absorb_q_width_not_a_multiple_of_two_tiles():
    """d_c = 384: the absorption's CTAs hold two 128-feature m-tiles each, so a head's second CTA has
    one tile past the weight's last column (its loads read the fill value, its epilogue skips it)."""
    w = synth.workload("dsv3_b64_l4096", d_c=384, B=5, lengths=("list", (7, 100, 4096, 65, 131072)))
    case = Case(w)
    dev = case.to_device()
    q_abs = ops.mla_absorb_q(Dims.of(w), dev["q_nope"], dev["q_rope_raw"], dev["W_UK"], dev["seqlens"])
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    got = q_abs.to(torch.float64).cpu().numpy()
    for b in range(w.B):
        pos = O.token_positions(int(case.lens[b]), 1)
        ref = O.absorb_query(case.q_nope64[b], case.q_rope_raw64[b], case.W64["W_UK"], pos, w.rope_base)
        _assert_close(got[b], ref, w.dtype, f"q_abs seq {b}")


@pytest.mark.parametrize("name,s_q", [("dsv3_b64_l4096", 1), ("dsv3_b64_l4096", 3), ("smallem_fp32", 1)])
def test_absorb_q(name, s_q):
    w = synth.workload(name, s_q=s_q, B=7, lengths=("list", (7, 100, 4096, 65, 64, 9999, 131072)))
    case = Case(w)
    dev = case.to_device()
    q_abs = ops.mla_absorb_q(Dims.of(w), dev["q_nope"], dev["q_rope_raw"], dev["W_UK"], dev["seqlens"])
    got = q_abs.to(torch.float64).cpu().numpy()
    for b in range(w.B):
        pos = O.token_positions(int(case.lens[b]), s_q)
        ref = O.absorb_query(case.q_nope64[b], case.q_rope_raw64[b], case.W64["W_UK"], pos, w.rope_base)
        _assert_close(got[b], ref, w.dtype, f"q_abs seq {b}")
        _assert_close(got[b][..., w.d_c:], ref[..., w.d_c:], w.dtype, f"rotated query seq {b}")


@pytest.mark.parametrize("name,B,s_q", [("dsv3_b64_l4096", 64, 1), ("dsv3_b64_l4096", 5, 3),
                                        ("dsv3_b64_l4096", 300, 1), ("smallem_fp32", 3, 2)])
def test_append_cache_absorb_q(name, B, s_q):
    """a1 and a2 in one call: the new rows and q_abs against the oracle, q_abs identical to
    mla_absorb_q's, every other pool row untouched."""
    w = synth.workload(name, B=B, s_q=s_q, lengths=("list", tuple(4096 - 3 * i for i in range(B))))
    case = Case(w)
    dev = case.to_device()
    cache = _cache(dev, case)
    before = dev["pool"].clone()
    dims = Dims.of(w)
    q_abs = ops.mla_append_cache_absorb_q(dims, dev["x"], dev["w_dkv_kr"], None, dev["q_nope"], dev["q_rope_raw"],
                                          dev["W_UK"], dev["seqlens"], dev["table"], cache)
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    assert torch.equal(q_abs, ops.mla_absorb_q(dims, dev["q_nope"], dev["q_rope_raw"], dev["W_UK"], dev["seqlens"]))
    got_q = q_abs.to(torch.float64).cpu().numpy()
    for b in sorted({0, B // 2, B - 1}):
        pos = O.token_positions(int(case.lens[b]), s_q)
        ref = O.absorb_query(case.q_nope64[b], case.q_rope_raw64[b], case.W64["W_UK"], pos, w.rope_base)
        _assert_close(got_q[b], ref, w.dtype, f"q_abs seq {b}")
    # token (b, t) is at position L_b - s_q + t
    pos = (case.lens[:, None] - s_q + np.arange(s_q)[None, :]).reshape(-1).astype(np.int64)
    seq = np.repeat(np.arange(B), s_q)
    c_ref, kr_ref = O.latent_rows(case.x64.reshape(B * s_q, w.C), case.W64["W_DKV"], case.W64["W_KR"], pos, None,
                                  w.rms_eps, w.rope_base)
    rows = case.table[seq, pos // 64].astype(np.int64) * 64 + pos % 64
    pool = dev["pool"].cpu()
    got = pool[torch.from_numpy(rows)].to(torch.float64).numpy()
    _assert_close(got[:, :w.d_c], c_ref, w.dtype, "appended latent")
    _assert_close(got[:, w.d_c:], kr_ref, w.dtype, "appended rope key")
    mask = torch.ones(pool.shape[0], dtype=torch.bool)
    mask[torch.from_numpy(rows)] = False
    assert torch.equal(pool[mask], before.cpu()[mask])


@pytest.mark.parametrize("name", ["dsv3_b64_l4096", "smallem_fp32"])
def test_out_proj(name):
    w = synth.workload(name, B=5, s_q=2)
    case = Case(w)
    dev = case.to_device()
    out, out_model = ops.mla_out_proj(Dims.of(w), dev["o_lat"], dev["W_UV"], w_o=dev["W_O"])
    ref = O.out_projection(case.o_lat64.reshape(-1, w.H, w.d_c), case.W64["W_UV"])
    _assert_close(out.to(torch.float64).cpu().numpy().reshape(ref.shape), ref, w.dtype, "out heads")
    ref_m = O.out_projection(case.o_lat64.reshape(-1, w.H, w.d_c), case.W64["W_UV"], case.W64["W_O"])
    # the model projection consumes the stored (rounded) head outputs on the GPU side
    _assert_close(out_model.to(torch.float64).cpu().numpy().reshape(ref_m.shape), ref_m, w.dtype, "out model")


def _within_one_rounding(got, ref, what):
    """bf16 result of an fp32-accumulated sum: one rounding (2^-8 relative) plus a little slack for
    the accumulation order, relative to the largest reference value."""
    got = np.asarray(got, np.float64)
    bad = np.abs(got - ref) > 2.0 ** -8 * np.abs(ref) + 1e-3 * np.abs(ref).max()
    assert not bad.any(), f"{what}: {int(bad.sum())} elements beyond one bf16 rounding"


@pytest.mark.parametrize("B", [33, 100, 300])
def test_projections_across_token_blocks(B):
    """a1, a2 and a5 at token counts that take each token width of the tensor-core projection
    (32, 64, 128 per CTA), several token blocks and a ragged last block."""
    lens = tuple(65 + (7 * i) % 200 for i in range(B))
    w = synth.workload("dsv3_b64_l4096", B=B, lengths=("list", lens))
    case = Case(w)
    dev = case.to_device()
    dims = Dims.of(w)
    q_abs = ops.mla_absorb_q(dims, dev["q_nope"], dev["q_rope_raw"], dev["W_UK"], dev["seqlens"])
    out = ops.mla_out_proj(dims, dev["o_lat"], dev["W_UV"])
    cache = _cache(dev, case)
    before = dev["pool"].clone()
    ops.mla_append_cache(dims, dev["x"], dev["w_dkv_kr"], None, dev["seqlens"], dev["table"], cache)
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    got = q_abs.to(torch.float64).cpu().numpy()
    for b in range(B):
        ref = O.absorb_query(case.q_nope64[b], case.q_rope_raw64[b], case.W64["W_UK"],
                             O.token_positions(int(case.lens[b]), 1), w.rope_base)
        _assert_close(got[b], ref, "bf16", f"q_abs seq {b}")
        _within_one_rounding(got[b], ref, f"q_abs seq {b}")
    ref = O.out_projection(case.o_lat64.reshape(-1, w.H, w.d_c), case.W64["W_UV"])
    got = out.to(torch.float64).cpu().numpy().reshape(ref.shape)
    _assert_close(got, ref, "bf16", "out heads")
    _within_one_rounding(got, ref, "out heads")
    pos = (case.lens - 1).astype(np.int64)
    c_ref, kr_ref = O.latent_rows(case.x64[:, 0], case.W64["W_DKV"], case.W64["W_KR"], pos, None, w.rms_eps,
                                  w.rope_base)
    rows = case.table[np.arange(B), pos // 64].astype(np.int64) * 64 + pos % 64
    pool = dev["pool"].cpu()
    got = pool[torch.from_numpy(rows)].to(torch.float64).numpy()
    _within_one_rounding(got[:, :w.d_c], c_ref, "appended latent")
    _within_one_rounding(got[:, w.d_c:], kr_ref, "appended rope key")
    mask = torch.ones(pool.shape[0], dtype=torch.bool)
    mask[torch.from_numpy(rows)] = False
    assert torch.equal(pool[mask], before.cpu()[mask])


# ------------------------------------------------------------------------------------------------
# whole step through the C ABI against the expanded definition
# ------------------------------------------------------------------------------------------------

def _gpu_step(w, case, dev):
    dims = Dims.of(w)
    cache = _cache(dev, case)
    ops.mla_append_cache(dims, dev["x"], dev["w_dkv_kr"], None, dev["seqlens"], dev["table"], cache)
    q_abs = ops.mla_absorb_q(dims, dev["q_nope"], dev["q_rope_raw"], dev["W_UK"], dev["seqlens"])
    o_lat, lse = ops.mla_decode_absorbed(dims, q_abs, cache, dev["table"], dev["seqlens"])
    out, out_model = ops.mla_out_proj(dims, o_lat, dev["W_UV"], w_o=dev["W_O"])
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    return out, out_model, lse


@pytest.mark.parametrize("queries", ["drawn", "from_x"])
def test_smallem_layer_fp32_from_hidden_states(queries):
    """The Smallem-scale layer in fp32: every position's row appended from x by the GPU (511 as one
    prefill call, the new token as a decode step), then absorb -> decode -> out_proj, against the
    expanded definition of the oracle built from the same x. With queries "from_x" the new token's
    query also comes from its x through the query chain (mla_project_query), so the whole step runs
    from hidden states."""
    w = synth.workload("smallem_fp32")
    L = 512
    case = Case(w)
    dev = case.to_device()
    dims = Dims.of(w)
    x_all = synth.context_hidden_states(w, L)
    xt = torch.from_numpy(x_all).float().cuda()
    cache = _cache(dev, case)
    prefill_len = torch.tensor([L - 1], dtype=torch.int32, device="cuda")
    ops.mla_append_cache(dims, xt[None, :L - 1], dev["w_dkv_kr"], None, prefill_len, dev["table"], cache)
    ops.mla_append_cache(dims, xt[None, L - 1:], dev["w_dkv_kr"], None, dev["seqlens"], dev["table"], cache)
    q_nope, q_rope_raw = dev["q_nope"], dev["q_rope_raw"]
    if queries == "from_x":
        q_nope, q_rope_raw = ops.mla_project_query(dims, xt[None, L - 1:], dev["W_DQ"], dev["gamma_q"], dev["W_UQ"],
                                                   dev["W_QR"])
    q_abs = ops.mla_absorb_q(dims, q_nope, q_rope_raw, dev["W_UK"], dev["seqlens"])
    o_lat, lse = ops.mla_decode_absorbed(dims, q_abs, cache, dev["table"], dev["seqlens"])
    out, out_model = ops.mla_out_proj(dims, o_lat, dev["W_UV"], w_o=dev["W_O"])
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    c, kr = O.latent_rows(x_all.astype(np.float64), case.W64["W_DKV"], case.W64["W_KR"], np.arange(L))
    got_rows = dev["pool"][:L].double().cpu().numpy()
    _assert_close(got_rows[:, :w.d_c], c, "f32", "latent rows")
    _assert_close(got_rows[:, w.d_c:], kr, "f32", "rope rows")
    pos = np.array([L - 1])
    if queries == "from_x":
        q_ref, _, q_rot = O.query_parts(x_all[L - 1:].astype(np.float64), case.W64["W_DQ"], case.W64["W_UQ"],
                                        case.W64["W_QR"], w.H, w.D, w.d_r, pos, case.W64["gamma_q"], w.rms_eps,
                                        w.rope_base)
    else:
        q_ref = case.q_nope64[0]
        q_rot = O.rope(case.q_rope_raw64[0], pos[:, None] * np.ones((1, w.H)))
    ref, ref_lse = O.expanded_decode(q_ref, q_rot, c, kr, case.W64["W_UK"], case.W64["W_UV"], L, w.sm_scale)
    _assert_close(out[0].double().cpu().numpy(), ref, "f32", "head outputs")
    _assert_lse(lse[0].cpu().numpy(), ref_lse, "f32", "lse")
    ref_model = ref.reshape(1, -1) @ case.W64["W_O"]
    _assert_close(out_model[0].double().cpu().numpy(), ref_model, "f32", "layer output")


@pytest.mark.parametrize("name,over", [
    ("smallem_fp32", {}),
    ("smallem_fp32", dict(B=3, s_q=2)),
    ("smallem_fp32", dict(d_q=254)),          # a width the float4 RMS step does not take
    ("dsv3_b64_l4096", dict(d_q=1536, lengths=("fixed", 64))),
    ("dsv3_b64_l4096", dict(d_q=1536, B=50, s_q=3, lengths=("fixed", 64))),
])
def test_project_query(name, over):
    """f2, the query chain x -> RMSNorm(x·W_DQ)·gamma_q -> (·W_UQ, ·W_QR), against the oracle's
    query_parts in fp64: the CUDA-core route in fp32, the tensor-core route in bf16 at the DeepSeek
    widths (C = 7168, d_q = 1536, H·D = 16384), one token per sequence and a ragged 150-token batch."""
    w = synth.workload(name, **over)
    case = Case(w)
    dev = case.to_device()
    dims = Dims.of(w)
    q_nope, q_rope_raw = ops.mla_project_query(dims, dev["x"], dev["W_DQ"], dev["gamma_q"], dev["W_UQ"], dev["W_QR"])
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    n = w.B * w.s_q
    ref_nope, ref_raw, _ = O.query_parts(case.x64.reshape(n, w.C), case.W64["W_DQ"], case.W64["W_UQ"],
                                         case.W64["W_QR"], w.H, w.D, w.d_r, np.zeros(n), case.W64["gamma_q"],
                                         w.rms_eps, w.rope_base)
    _assert_close(q_nope.double().cpu().numpy().reshape(n, w.H, w.D), ref_nope, w.dtype, "q_nope")
    _assert_close(q_rope_raw.double().cpu().numpy().reshape(n, w.H, w.d_r), ref_raw, w.dtype, "q_rope_raw")


def test_full_step_dsv3_against_oracle():
    """configs' DeepSeek shape, full size: append -> absorb -> decode -> out_proj on the GPU; the
    absorbed fp64 oracle on every sequence, the expanded definition on a sample."""
    w = synth.workload("dsv3_b64_l4096")
    case = Case(w)
    dev = case.to_device()
    out, out_model, lse = _gpu_step(w, case, dev)
    # oracle: its own new rows (stored in the cache's type), its own absorption
    pos = (case.lens - 1).astype(np.int64)
    c_new, kr_new = O.latent_rows(case.x64[:, 0], case.W64["W_DKV"], case.W64["W_KR"], pos)
    pool = case.pool.clone()
    rows = case.table[np.arange(w.B), pos // 64].astype(np.int64) * 64 + pos % 64
    pool[torch.from_numpy(rows)] = torch.from_numpy(np.concatenate([c_new, kr_new], 1)).to(pool.dtype)
    got = out.double().cpu().numpy()
    got_lse = lse.cpu().numpy()
    sample = [(0, None), (17, None), (63, None)]
    for b in range(w.B):
        c, kr = case.seq_rows64(b, pool)
        L = int(case.lens[b])
        pb = O.token_positions(L, 1)
        q_abs = as_stored(O.absorb_query(case.q_nope64[b], case.q_rope_raw64[b], case.W64["W_UK"], pb), "bf16")
        o_lat, l = O.absorbed_decode(q_abs, c, kr, L, w.sm_scale)
        ref = O.out_projection(as_stored(o_lat, "bf16"), case.W64["W_UV"])
        _assert_close(got[b], ref, "bf16", f"out seq {b}")
        _assert_lse(got_lse[b], l, "bf16", f"lse seq {b}")
    heads = [0, 5, 77, 127]
    for b, _ in sample:
        c, kr = case.seq_rows64(b, pool)
        L = int(case.lens[b])
        q_rot = O.rope(case.q_rope_raw64[b][:, heads], np.full((1, len(heads)), L - 1))
        ref, _ = O.expanded_decode(case.q_nope64[b][:, heads], q_rot, c, kr, case.W64["W_UK"][heads],
                                   case.W64["W_UV"][heads], L, w.sm_scale)
        _assert_close(got[b][:, heads], ref, "bf16", f"expanded definition seq {b}")


# ------------------------------------------------------------------------------------------------
# a6: GQLA grouped path
def test_dsv3_context_built_from_hidden_states():
    """The DeepSeek shape with its configured cache recipe: two whole 4096-position contexts written
    by mla_append_cache from hidden states x ~ N(0, 1) (4095 positions as one prefill call, then the
    new token as a decode step, random page table), then absorb -> decode -> out_proj. The oracle
    builds the same rows from the same x (rms(x·W_DKV), RoPE(x·W_KR)), keeps them in the cache's
    type, and runs its own absorbed decode and projection on them."""
    L, B = 4096, 2
    w = synth.workload("dsv3_b64_l4096", B=B, lengths=("fixed", L), pages="random")
    case = Case(w)
    dev = case.to_device()
    dims = Dims.of(w)
    dev["pool"].zero_()
    cache = _cache(dev, case)
    xs, x64 = [], []
    for b in range(B):
        t, t64 = _stored_bf16(synth.context_hidden_states(w, L, b))
        xs.append(t)
        x64.append(t64)
    xt = torch.stack(xs).cuda()
    prefill = torch.full((B,), L - 1, dtype=torch.int32, device="cuda")
    ops.mla_append_cache(dims, xt[:, :L - 1].contiguous(), dev["w_dkv_kr"], None, prefill, dev["table"], cache)
    ops.mla_append_cache(dims, xt[:, L - 1:].contiguous(), dev["w_dkv_kr"], None, dev["seqlens"], dev["table"], cache)
    q_abs = ops.mla_absorb_q(dims, dev["q_nope"], dev["q_rope_raw"], dev["W_UK"], dev["seqlens"])
    o_lat, lse = ops.mla_decode_absorbed(dims, q_abs, cache, dev["table"], dev["seqlens"])
    out = ops.mla_out_proj(dims, o_lat, dev["W_UV"])
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    pool = dev["pool"].cpu()
    got = out.double().cpu().numpy()
    got_lse = lse.cpu().numpy()
    for b in range(B):
        c, kr = O.latent_rows(x64[b], case.W64["W_DKV"], case.W64["W_KR"], np.arange(L))
        gc, gkr = case.seq_rows64(b, pool)
        _assert_close(gc, c, "bf16", f"latent rows seq {b}")
        _assert_close(gkr, kr, "bf16", f"rope rows seq {b}")
        c_s, kr_s = as_stored(c, "bf16"), as_stored(kr, "bf16")
        q = as_stored(O.absorb_query(case.q_nope64[b], case.q_rope_raw64[b], case.W64["W_UK"],
                                     O.token_positions(L, 1)), "bf16")
        ol, l = O.absorbed_decode(q, c_s, kr_s, L, w.sm_scale)
        ref = O.out_projection(as_stored(ol, "bf16"), case.W64["W_UV"])
        _assert_close(got[b], ref, "bf16", f"out seq {b}")
        _assert_lse(got_lse[b], l, "bf16", f"lse seq {b}")


def _stored_bf16(a):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t, t.to(torch.float64).numpy()


# ------------------------------------------------------------------------------------------------

def test_gqla_grouped_equals_absorbed_on_same_weights():
    """Expanded group caches are built by the oracle from the latent rows (stored bf16); the GPU
    grouped path, the GPU absorbed path on group-shared weights and the oracle must agree."""
    w = synth.workload("gqla_g8_b32_l8192", B=3, lengths=("list", (100, 1025, 64)), pages="random")
    case = Case(w)
    dev = case.to_device()
    dims = Dims.of(w)
    W_UK_g, W_UV_g = case.W64["W_UK_g"], case.W64["W_UV_g"]
    rows = case.pool.to(torch.float64).numpy()
    K, V = O.gqla_expand(rows[:, :w.d_c], W_UK_g, W_UV_g)
    Kt = torch.from_numpy(K).to(torch.bfloat16).cuda()
    Vt = torch.from_numpy(V).to(torch.bfloat16).cuda()
    gcache = GqaCache(Kt, Vt, dev["pool"][:, w.d_c:], case.num_pages)
    out, lse = ops.mla_decode_gqla_grouped(dims, dev["q_nope"], dev["q_rope_raw"], gcache, dev["table"], dev["seqlens"])
    # absorbed path on identical (group-shared) weights
    W_UK = torch.from_numpy(O.group_weights_per_head(W_UK_g, w.H)).to(torch.bfloat16).cuda()
    W_UV = torch.from_numpy(O.group_weights_per_head(W_UV_g, w.H)).to(torch.bfloat16).cuda()
    q_abs = ops.mla_absorb_q(dims, dev["q_nope"], dev["q_rope_raw"], W_UK, dev["seqlens"])
    o_lat, lse_a = ops.mla_decode_absorbed(dims, q_abs, _cache(dev, case), dev["table"], dev["seqlens"])
    out_a = ops.mla_out_proj(dims, o_lat, W_UV)
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    Ks = torch.from_numpy(K).to(torch.bfloat16).double().numpy()
    Vs = torch.from_numpy(V).to(torch.bfloat16).double().numpy()
    for b in range(w.B):
        L = int(case.lens[b])
        p = np.arange(L)
        idx = case.table[b, p // 64].astype(np.int64) * 64 + p % 64
        q_rot = O.rope(case.q_rope_raw64[b], np.full((1, w.H), L - 1))
        ref, ref_l = O.gqla_grouped_decode(case.q_nope64[b], q_rot, Ks[idx], Vs[idx], rows[idx, w.d_c:], L,
                                           w.sm_scale, w.g)
        _assert_close(out[b].double().cpu().numpy(), ref, "bf16", f"grouped seq {b}")
        _assert_lse(lse[b].cpu().numpy(), ref_l, "bf16", f"grouped lse seq {b}")
        _assert_close(out_a[b].double().cpu().numpy(), ref, "bf16", f"absorbed on group weights seq {b}")
        # the absorbed pipeline keeps q_abs in bf16 between calls: the oracle rounds its own q_abs there
        qa = as_stored(O.absorb_query(case.q_nope64[b], case.q_rope_raw64[b], O.group_weights_per_head(W_UK_g, w.H),
                                      O.token_positions(L, 1)), "bf16")
        _, ref_la = O.absorbed_decode(qa, rows[idx, :w.d_c], rows[idx, w.d_c:], L, w.sm_scale)
        _assert_lse(lse_a[b].cpu().numpy(), ref_la, "bf16", f"absorbed lse seq {b}")
        assert np.abs(ref_la - ref_l).max() < 5e-3      # the two paths agree up to bf16 storage


def test_gqa_cache_append_from_hidden_states_then_grouped_decode():
    """f3: the expanded GQA cache written by the GPU from hidden states (a prefill call, then the new
    token as a decode step, random page table): K = W_UK[g]·c, V = c·W_UV[g] and k_r per row against
    the oracle's expansion of its own rows (one bf16 rounding of c, then of K and V), and the
    grouped decode over that cache against the oracle's grouped attention on its own rows."""
    lens = (300, 65, 1000)
    w = synth.workload("gqla_g8_b32_l8192", B=3, lengths=("list", lens), pages="random")
    case = Case(w)
    dev = case.to_device()
    dims = Dims.of(w)
    n = case.num_pages * 64
    K = torch.zeros(n, w.g, w.D, dtype=torch.bfloat16, device="cuda")
    V = torch.zeros(n, w.g, w.d_v, dtype=torch.bfloat16, device="cuda")
    R = torch.zeros(n, w.d_r, dtype=torch.bfloat16, device="cuda")
    gcache = GqaCache(K, V, R, case.num_pages)
    W_UK_g, W_UV_g = dev["W_UK_g"], dev["W_UV_g"]
    Lmax = max(lens)
    xs = [_stored_bf16(synth.context_hidden_states(w, Lmax, b)) for b in range(w.B)]
    xt = torch.stack([t for t, _ in xs]).cuda()
    # prefill: the first len - 1 positions of every sequence, as s_q = 64 steps of a common length
    # where possible, then token by token; finally the new token
    done = np.zeros(w.B, np.int64)
    while True:
        todo = np.asarray(lens) - 1 - done
        if (todo <= 0).all():
            break
        step = 64 if (todo >= 64).all() else 1
        act = [b for b in range(w.B) if todo[b] >= step]
        sl = torch.from_numpy((done[act] + step).astype(np.int32)).cuda()
        xb = torch.stack([xt[b, done[b]:done[b] + step] for b in act]).contiguous()
        tb = dev["table"][torch.tensor(act, device="cuda")].contiguous()
        ops.mla_append_gqa_cache(dims, xb, dev["w_dkv_kr"], None, W_UK_g, W_UV_g, sl, tb, gcache)
        done[act] += step
    x_new = torch.stack([xt[b, lens[b] - 1:lens[b]] for b in range(w.B)]).contiguous()
    ops.mla_append_gqa_cache(dims, x_new, dev["w_dkv_kr"], None, W_UK_g, W_UV_g, dev["seqlens"], dev["table"], gcache)
    out, lse = ops.mla_decode_gqla_grouped(dims, dev["q_nope"], dev["q_rope_raw"], gcache, dev["table"], dev["seqlens"])
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    Kh, Vh, Rh = (t.double().cpu().numpy() for t in (K, V, R))
    for b, L in enumerate(lens):
        p = np.arange(L)
        idx = case.table[b, p // 64].astype(np.int64) * 64 + p % 64
        c, kr = O.latent_rows(xs[b][1][:L], case.W64["W_DKV"], case.W64["W_KR"], p)
        Kr, Vr = O.gqla_expand(as_stored(c, "bf16"), case.W64["W_UK_g"], case.W64["W_UV_g"])
        _assert_close(Kh[idx], Kr, "bf16", f"expanded keys seq {b}")
        _assert_close(Vh[idx], Vr, "bf16", f"expanded values seq {b}")
        _assert_close(Rh[idx], kr, "bf16", f"rope keys seq {b}")
        q_rot = O.rope(case.q_rope_raw64[b], np.full((1, w.H), L - 1))
        ref, ref_l = O.gqla_grouped_decode(case.q_nope64[b], q_rot, as_stored(Kr, "bf16"), as_stored(Vr, "bf16"),
                                           as_stored(kr, "bf16"), L, w.sm_scale, w.g)
        _assert_close(out[b].double().cpu().numpy(), ref, "bf16", f"grouped out seq {b}")
        _assert_lse(lse[b].cpu().numpy(), ref_l, "bf16", f"grouped lse seq {b}")


@pytest.mark.parametrize("name", ["dsv3_b64_l4096", "smallem_fp32"])
def test_output_projection_through_preabsorbed_weights(name):
    """f3: W_UVO[h] = W_UV[h]·W_O[h] built on the GPU, then the layer output straight from the
    weighted latents, against the oracle's two-step projection (o_lat·W_UV[h], concatenated, ·W_O)."""
    over = dict(B=3, s_q=1, H=16) if name == "dsv3_b64_l4096" else dict(B=2, s_q=2)
    w = synth.workload(name, **over)
    case = Case(w)
    dev = case.to_device()
    dims = Dims.of(w)
    w_uvo = ops.mla_preabsorb_out_weights(dims, dev["W_UV"], dev["W_O"])
    out_model = ops.mla_out_proj_preabsorbed(dims, dev["o_lat"], w_uvo)
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    ref = O.out_projection(case.o_lat64.reshape(-1, w.H, w.d_c), case.W64["W_UV"], case.W64["W_O"])
    _assert_close(out_model.double().cpu().numpy().reshape(ref.shape), ref, w.dtype, "layer output")
    ref_w = O.preabsorbed_out_weights(case.W64["W_UV"], case.W64["W_O"])
    _assert_close(w_uvo.double().cpu().numpy(), ref_w, w.dtype, "absorbed weights")


def test_gqla_ragged_lengths_and_splits():
    """The grouped path on one position, tile edges (127/128/129 of a 128-position tile), a partial
    last tile and a long sequence cut into splits (short sequences leave empty splits), every head."""
    lens = (1, 127, 128, 129, 300, 8192)
    w = synth.workload("gqla_g8_b32_l8192", B=len(lens), lengths=("list", lens), pages="random")
    lens_a = np.asarray(lens, np.int32)
    table, num_pages = synth.block_table(w, lens_a)
    n = num_pages * 64
    K = torch.empty(n, w.g, w.D, dtype=torch.bfloat16)
    V = torch.empty(n, w.g, w.d_v, dtype=torch.bfloat16)
    R = torch.empty(n, w.d_r, dtype=torch.bfloat16)
    for start, k, v, r in synth.gqla_cache_chunks(w, n):
        K[start:start + len(k)] = torch.from_numpy(k)
        V[start:start + len(k)] = torch.from_numpy(v)
        R[start:start + len(k)] = torch.from_numpy(r)
    step = synth.decode_step_inputs(w)
    qn = torch.from_numpy(step["q_nope"]).to(torch.bfloat16)
    qr = torch.from_numpy(step["q_rope_raw"]).to(torch.bfloat16)
    gcache = GqaCache(K.cuda(), V.cuda(), R.cuda(), num_pages)
    out, lse = ops.mla_decode_gqla_grouped(Dims.of(w), qn.cuda(), qr.cuda(), gcache, torch.from_numpy(table).cuda(),
                                           torch.from_numpy(lens_a).cuda())
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    Kd, Vd, Rd = K.double().numpy(), V.double().numpy(), R.double().numpy()
    for b, L in enumerate(lens):
        p = np.arange(L)
        idx = table[b, p // 64].astype(np.int64) * 64 + p % 64
        q_rot = O.rope(qr[b].double().numpy(), np.full((1, w.H), L - 1))
        ref, ref_l = O.gqla_grouped_decode(qn[b].double().numpy(), q_rot, Kd[idx], Vd[idx], Rd[idx], L, w.sm_scale, w.g)
        _assert_close(out[b].double().cpu().numpy(), ref, "bf16", f"grouped seq {b} (L={L})")
        _assert_lse(lse[b].cpu().numpy(), ref_l, "bf16", f"grouped lse seq {b} (L={L})")


def test_gqla_full_size_sampled():
    w = synth.workload("gqla_g8_b32_l8192")
    lens = synth.seq_lengths(w)
    table, num_pages = synth.block_table(w, lens)
    n = num_pages * 64
    K = torch.empty(n, w.g, w.D, dtype=torch.bfloat16)
    V = torch.empty(n, w.g, w.d_v, dtype=torch.bfloat16)
    R = torch.empty(n, w.d_r, dtype=torch.bfloat16)
    for start, k, v, r in synth.gqla_cache_chunks(w, n):
        K[start:start + len(k)] = torch.from_numpy(k)
        V[start:start + len(k)] = torch.from_numpy(v)
        R[start:start + len(k)] = torch.from_numpy(r)
    step = synth.decode_step_inputs(w)
    qn = torch.from_numpy(step["q_nope"]).to(torch.bfloat16)
    qr = torch.from_numpy(step["q_rope_raw"]).to(torch.bfloat16)
    gcache = GqaCache(K.cuda(), V.cuda(), R.cuda(), num_pages)
    out, lse = ops.mla_decode_gqla_grouped(Dims.of(w), qn.cuda(), qr.cuda(), gcache, torch.from_numpy(table).cuda(),
                                           torch.from_numpy(lens).cuda())
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    Kd, Vd, Rd = K.double().numpy(), V.double().numpy(), R.double().numpy()
    heads = [0, 15, 16, 64, 127]
    for b in [0, 13, 31]:
        L = int(lens[b])
        p = np.arange(L)
        idx = table[b, p // 64].astype(np.int64) * 64 + p % 64
        q_rot = O.rope(qr[b].double().numpy(), np.full((1, w.H), L - 1))
        ref, ref_l = O.gqla_grouped_decode(qn[b].double().numpy(), q_rot, Kd[idx], Vd[idx], Rd[idx], L, w.sm_scale, w.g)
        _assert_close(out[b][:, heads].double().cpu().numpy(), ref[:, heads], "bf16", f"grouped seq {b}")
        _assert_lse(lse[b][:, heads].cpu().numpy(), ref_l[:, heads], "bf16", f"grouped lse seq {b}")


# ------------------------------------------------------------------------------------------------
# errors
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("lens,s_q", [([4096] * 64, 1), ([4096, 129, 2049, 64, 5000], 1), ([131072], 1),
                                      ([65, 66, 4, 64 * 3 + 2, 64 * 3 + 3], 4), ([1, 2], 1)])
def test_decode_with_host_lengths_equals_plain(lens, s_q):
    """mla_decode_absorbed_hinted (a host copy of seqlens) gives the outputs of mla_decode_absorbed
    bit for bit, whether the copy shows nothing cut (a plain launch, no merge) or a cut (the merging
    launch), and records nothing."""
    w = synth.workload("dsv3_b64_l4096", B=len(lens), s_q=s_q, lengths=("list", tuple(lens)), pages="random")
    case = Case(w, with_weights=False)
    dev = case.to_device()
    dims = Dims.of(w)
    o_ref, l_ref = ops.mla_decode_absorbed(dims, dev["q_abs"], _cache(dev, case), dev["table"], dev["seqlens"])
    o, l = ops.mla_decode_absorbed(dims, dev["q_abs"], _cache(dev, case), dev["table"], dev["seqlens"],
                                   seqlens_host=case.lens.astype(np.int32))
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    assert torch.equal(o, o_ref) and torch.equal(l, l_ref)


def test_stale_host_lengths_are_reported():
    """A host copy that shows nothing cut while the device's lengths cut a sequence: the plain launch
    cannot merge it, so the call records MLA_ERR_DEVICE_CHECK."""
    w = synth.workload("dsv3_b64_l4096", B=1, lengths=("list", (131072,)), pages="random")
    case = Case(w, with_weights=False)
    dev = case.to_device()
    ops.mla_decode_absorbed(Dims.of(w), dev["q_abs"], _cache(dev, case), dev["table"], dev["seqlens"],
                            seqlens_host=np.array([64], dtype=np.int32))
    assert ops.mla_check_status() == L.MLA_ERR_DEVICE_CHECK
    assert ops.mla_check_status() == 0


def test_page_id_outside_pool_is_reported_not_read():
    w = synth.workload("dsv3_b64_l4096", B=2, lengths=("list", (200, 70)))
    case = Case(w, with_weights=False)
    dev = case.to_device()
    bad = dev["table"].clone()
    bad[1, 0] = case.num_pages + 5          # outside the pool: the kernel must skip it and report
    ops.mla_decode_absorbed(Dims.of(w), dev["q_abs"], _cache(dev, case), bad, dev["seqlens"])
    assert ops.mla_check_status() == L.MLA_ERR_DEVICE_CHECK
    assert ops.mla_check_status() == 0       # cleared by the previous read
    # the 8-bit decode's dequantising pass checks the same ids (its decode reads a dense table)
    codes, scales = _fp8_rows(case)
    cache8 = LatentCacheFp8(torch.from_numpy(codes).cuda(), torch.from_numpy(scales.astype(np.float32)).cuda(),
                            dev["pool"][:, w.d_c:], case.num_pages)
    ops.mla_decode_absorbed_fp8(Dims.of(w), dev["q_abs"], cache8, bad, dev["seqlens"])
    assert ops.mla_check_status() == L.MLA_ERR_DEVICE_CHECK
    assert ops.mla_check_status() == 0


def test_sequence_without_its_new_token_is_reported():
    """seqlens[b] must count the step's own token: a zero length is reported by every decode path
    (absorbed, grouped, 8-bit) as a device check, its outputs left unwritten, the others still right."""
    w = synth.workload("dsv3_b64_l4096", B=2, lengths=("list", (200, 70)))
    case = Case(w, with_weights=False)
    dev = case.to_device()
    short = dev["seqlens"].clone()
    short[1] = 0
    o_lat, lse = ops.mla_decode_absorbed(Dims.of(w), dev["q_abs"], _cache(dev, case), dev["table"], short)
    assert ops.mla_check_status() == L.MLA_ERR_DEVICE_CHECK
    ref_o, ref_l = _oracle_absorbed(case, case.q_abs64, seqs=[0])
    _assert_close(o_lat[0].float().cpu().numpy(), ref_o[0], "bf16", "o_lat of the valid sequence")
    _assert_lse(lse[0].cpu().numpy(), ref_l[0], "bf16", "lse of the valid sequence")
    codes, scales = _fp8_rows(case)
    cache8 = LatentCacheFp8(torch.from_numpy(codes).cuda(), torch.from_numpy(scales.astype(np.float32)).cuda(),
                            dev["pool"][:, w.d_c:], case.num_pages)
    ops.mla_decode_absorbed_fp8(Dims.of(w), dev["q_abs"], cache8, dev["table"], short)
    assert ops.mla_check_status() == L.MLA_ERR_DEVICE_CHECK
    wg = synth.workload("gqla_g8_b32_l8192", B=2, lengths=("list", (200, 70)))
    cg = Case(wg)
    dg = cg.to_device()
    n = cg.num_pages * 64
    gcache = GqaCache(torch.zeros(n, wg.g, wg.D, dtype=torch.bfloat16, device="cuda"),
                      torch.zeros(n, wg.g, wg.d_v, dtype=torch.bfloat16, device="cuda"),
                      torch.zeros(n, wg.d_r, dtype=torch.bfloat16, device="cuda"), cg.num_pages)
    short_g = dg["seqlens"].clone()
    short_g[1] = 0
    ops.mla_decode_gqla_grouped(Dims.of(wg), dg["q_nope"], dg["q_rope_raw"], gcache, dg["table"], short_g)
    assert ops.mla_check_status() == L.MLA_ERR_DEVICE_CHECK
    assert ops.mla_check_status() == 0


@pytest.mark.parametrize("combined", [False, True])
def test_append_to_a_page_outside_the_pool_is_reported_not_written(combined):
    """A new token whose page id lies outside the pool: the append records MLA_ERR_DEVICE_CHECK and
    writes nothing for it; the other sequence's row is written as usual (alone and in the combined
    append + absorb call)."""
    w = synth.workload("dsv3_b64_l4096", B=2, lengths=("list", (200, 70)))
    case = Case(w)
    dev = case.to_device()
    cache = _cache(dev, case)
    bad = dev["table"].clone()
    bad[1, (70 - 1) // 64] = case.num_pages + 3
    before = dev["pool"].clone()
    dims = Dims.of(w)
    if combined:
        ops.mla_append_cache_absorb_q(dims, dev["x"], dev["w_dkv_kr"], None, dev["q_nope"], dev["q_rope_raw"],
                                      dev["W_UK"], dev["seqlens"], bad, cache)
    else:
        ops.mla_append_cache(dims, dev["x"], dev["w_dkv_kr"], None, dev["seqlens"], bad, cache)
    assert ops.mla_check_status() == L.MLA_ERR_DEVICE_CHECK
    pos = (case.lens - 1).astype(np.int64)
    c_ref, kr_ref = O.latent_rows(case.x64[:, 0], case.W64["W_DKV"], case.W64["W_KR"], pos, None, w.rms_eps,
                                  w.rope_base)
    row0 = int(case.table[0, pos[0] // 64]) * 64 + int(pos[0] % 64)
    pool = dev["pool"].cpu()
    got = pool[row0].double().numpy()
    _assert_close(got[None, :w.d_c], c_ref[:1], w.dtype, "appended latent of the valid sequence")
    mask = torch.ones(pool.shape[0], dtype=torch.bool)
    mask[row0] = False
    assert torch.equal(pool[mask], before.cpu()[mask])   # nothing else moved
    assert ops.mla_check_status() == 0


def test_invalid_arguments_raise():
    w = synth.workload("dsv3_b64_l4096", B=1, lengths=("list", (64,)))
    case = Case(w, with_weights=False)
    dev = case.to_device()
    with pytest.raises(ops.MlaError):
        ops.mla_decode_absorbed(Dims.of(w), dev["q_abs"], _cache(dev, case), dev["table"], dev["seqlens"],
                                o_lat=torch.empty(1, 1, 128, 512, dtype=torch.bfloat16, device="cuda")[..., 1:])


# ------------------------------------------------------------------------------------------------
# f4: 8-bit latent cache. The decode checks take codes and scales made by the oracle on the host
# (its float32-decision quantiser), never the GPU quantiser's, which has its own bit-exact test.
# ------------------------------------------------------------------------------------------------

def _fp8_rows(case):
    """Oracle E4M3 codes and scales of every row of the case's 16-bit pool."""
    lat = case.pool[:, :case.w.d_c].to(torch.float64).numpy()
    return F.quantize_rows_f32(lat)


def _seq_pool_index(case, b):
    p = np.arange(int(case.lens[b]))
    return case.table[b, p // 64].astype(np.int64) * 64 + p % 64


@pytest.mark.parametrize("name,dtype", [("dsv3_b64_l4096", torch.bfloat16), ("smallem_fp32", torch.float32)])
def test_quantize_latent_fp8_matches_the_oracle_bit_for_bit(name, dtype):
    """Codes and scales of the GPU quantiser equal the oracle's (decision in float32), on rows read
    through an interleaved pool's stride: varied magnitudes, a zero row, values far below their row's
    scale (code +0), subnormal codes, a row whose largest value dwarfs the rest."""
    w = synth.workload(name)
    r = np.random.default_rng(60)
    rows, d_c, stride = 700, w.d_c, w.d_c + w.d_r
    c = r.standard_normal((rows, d_c)) * r.uniform(1e-3, 50, (rows, 1))
    c[3] = 0.0
    c[4] = 1e-30
    c[4, 0] = 1.0
    c[5] = r.uniform(-1, 1, d_c) * 2.0 ** -8
    c[6, 7] = 448.0 * 3
    pool = torch.zeros(rows, stride, dtype=dtype)
    pool[:, :d_c] = torch.from_numpy(c).to(dtype)
    ref_codes, ref_scales = F.quantize_rows_f32(pool[:, :d_c].to(torch.float64).numpy())
    dev = pool.cuda()
    codes = torch.empty(rows, d_c, dtype=torch.uint8, device="cuda")
    scales = torch.empty(rows, dtype=torch.float32, device="cuda")
    ops.mla_quantize_latent_fp8(Dims.of(w), dev[:, :d_c], codes, scales)
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_codes)
    np.testing.assert_array_equal(scales.cpu().numpy().astype(np.float64), ref_scales)
    assert (ref_codes[4, 1:] == 0).all() and ref_scales[3] == 0 and (ref_codes[3] == 0).all()


FP8_DECODE = [
    ([1], 1, "contiguous"),
    ([64, 65], 1, "random"),
    ([4096, 129, 2049, 64, 5000], 1, "contiguous"),
    ([65, 129, 64 * 5 + 1, 2], 2, "random"),
    ([131072], 1, "random"),
]


def _decode_fp8_case(w, heads=None, seqs=None):
    case = Case(w, with_weights=False)
    dev = case.to_device()
    codes, scales = _fp8_rows(case)
    cache = LatentCacheFp8(torch.from_numpy(codes).cuda(), torch.from_numpy(scales.astype(np.float32)).cuda(),
                           dev["pool"][:, w.d_c:], case.num_pages)
    o_lat, lse = ops.mla_decode_absorbed_fp8(Dims.of(w), dev["q_abs"], cache, dev["table"], dev["seqlens"])
    torch.cuda.synchronize()
    assert ops.mla_check_status() == 0
    got_o, got_l = o_lat.float().cpu().numpy(), lse.cpu().numpy()
    for b in (range(w.B) if seqs is None else seqs):
        idx = _seq_pool_index(case, b)
        kr = case.pool[torch.from_numpy(idx), w.d_c:].to(torch.float64).numpy()
        q = case.q_abs64[b] if heads is None else case.q_abs64[b][:, heads]
        ref_o, ref_l = F.absorbed_decode_fp8(q, codes[idx], scales[idx], kr, int(case.lens[b]), w.sm_scale)
        go = got_o[b] if heads is None else got_o[b][:, heads]
        gl = got_l[b] if heads is None else got_l[b][:, heads]
        _assert_close(go, ref_o, w.dtype, f"o_lat seq {b}")
        if w.dtype == "bf16":
            # bf16 at these shapes runs the tensor-core decode over the rows dequantised into bf16: each
            # s_j * value(code) is rounded once (relative error <= 2^-9) before the contraction, so a
            # score moves by at most 2^-9 * sm_scale * sum_i |q_i| |c_j,i| over the latent part, and
            # lse (1-Lipschitz in the largest score change) by at most that, on top of the bar
            dq = np.abs(F.dequantize_rows(codes[idx], scales[idx]))
            bound = 2.0 ** -9 * w.sm_scale * (np.abs(q[..., :w.d_c]) @ dq.T).max(axis=-1)
            err = np.abs(np.asarray(gl, np.float64) - ref_l)
            assert np.all(err <= TOL["bf16"]["lse"] + bound), f"lse seq {b}: max|Δ lse| = {err.max():.3e}"
        else:
            _assert_lse(gl, ref_l, w.dtype, f"lse seq {b}")


@pytest.mark.parametrize("lens,s_q,pages", FP8_DECODE)
def test_decode_absorbed_fp8(lens, s_q, pages):
    _decode_fp8_case(synth.workload("dsv3_b64_l4096", B=len(lens), s_q=s_q, lengths=("list", tuple(lens)),
                                    pages=pages))


def test_decode_absorbed_fp8_cuda_cores_fp32():
    """fp32 (and any shape the tensor-core decode does not take) decodes the 8-bit rows on the CUDA
    cores with fp32 dequantisation: the strict fp32 bar against the oracle."""
    _decode_fp8_case(synth.workload("smallem_fp32", B=3, lengths=("list", (512, 77, 1))))


def test_decode_absorbed_fp8_full_size_sampled():
    """The bench's 8-bit configuration (64 x 4096, DeepSeek widths), every sequence decoded, the
    oracle on a seeded sample of sequences and heads."""
    w = synth.workload("dsv3_b64_l4096")
    r = np.random.default_rng(61)
    _decode_fp8_case(w, heads=r.choice(w.H, 12, replace=False), seqs=r.choice(w.B, 6, replace=False))
