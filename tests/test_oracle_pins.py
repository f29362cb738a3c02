"""Pins of the fp64 oracle to things other than itself.

Each check ties an oracle function to a printed number of the pages, a closed form, a library
routine written by others (torch's RMSNorm and SDPA, scipy's logsumexp, numpy's complex
arithmetic), an algebraic identity the pages state, or a special case with a known answer.
The planted-mistake tests at the end show that plausible slips in the oracle fail these pins.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from oracle import cache_sizes, roofline
from oracle import mla_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "printed_numbers.json")


def _rng(seed):
    return np.random.default_rng(seed)


def _layer(seed=0, H=4, D=8, d_r=4, d_c=12, d_v=6, C=16, L=9, s_q=1):
    r = _rng(seed)
    return dict(
        q_nope=r.standard_normal((s_q, H, D)), q_rope=r.standard_normal((s_q, H, d_r)),
        c=r.standard_normal((L, d_c)), k_r=r.standard_normal((L, d_r)),
        W_UK=r.standard_normal((H, D, d_c)) / math.sqrt(d_c),
        W_UV=r.standard_normal((H, d_c, d_v)) / math.sqrt(d_c),
        seqlen=L, sm_scale=1.0 / math.sqrt(D + d_r))


# ------------------------------------------------------------------------------------------
# printed numbers (tests/golden/printed_numbers.json, each with its page and section)
# ------------------------------------------------------------------------------------------

def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("item", _golden()["items"], ids=lambda it: it["id"])
def test_printed_cache_numbers(item):
    got = getattr(cache_sizes, item["fn"])(**item["args"])
    got = got * item.get("scale", 1)
    if item.get("round"):
        got = round(got)
    assert got == pytest.approx(item["value"], rel=0, abs=1e-9), item["source"]


def test_printed_ratios():
    g = _golden()
    vals = {it["id"]: getattr(cache_sizes, it["fn"])(**it["args"]) for it in g["items"]}
    for r in g["ratios"]:
        assert vals[r["num"]] / vals[r["den"]] == pytest.approx(r["value"], rel=1e-12), r["source"]


@pytest.mark.parametrize("item", _golden()["intensity"], ids=lambda it: it["id"])
def test_printed_intensities(item):
    got = getattr(roofline, item["fn"])(**item["args"])
    assert abs(got - item["value"]) <= item["tol"], (got, item["source"])


def test_absorbed_intensity_exact_value():
    # 2·128·(2·512+64) FLOPs over (512+64)·2 bytes
    assert roofline.absorbed_intensity(128, 512, 64) == pytest.approx(278528 / 1152, rel=1e-15)


def test_mla_cache_is_linear_not_constant():
    # « MLA n'est pas mémoire fixe »: ×4 tokens gives ×4 memory; the fixed state does not move
    a = cache_sizes.latent_cache_bytes(131072, 32, 512, 2)
    b = cache_sizes.latent_cache_bytes(524288, 32, 512, 2)
    assert b == 4 * a == cache_sizes.kv_cache_bytes(131072, 32, 8, 128, 2)
    assert cache_sizes.recurrent_state_bytes(32, 128, 128, 2) == 2 ** 20


def test_large_model_cache_over_100_GB():
    # « Le problème : le cache grossit avec le texte »: width 7168, 61 layers, 100 000 tokens
    n = cache_sizes.mha_numbers_per_position(7168)
    assert cache_sizes.model_cache_bytes(n, 61, 100_000, 2) > 100e9


# ------------------------------------------------------------------------------------------
# building blocks against library routines and closed forms
# ------------------------------------------------------------------------------------------

def test_rmsnorm_matches_torch():
    r = _rng(1)
    z = r.standard_normal((5, 37))
    gamma = r.standard_normal(37)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(z), (37,), torch.from_numpy(gamma), eps=1e-6).numpy()
    np.testing.assert_allclose(O.rms_norm(z, gamma, 1e-6), ref, rtol=1e-13, atol=1e-14)


def test_rmsnorm_output_has_unit_rms():
    z = _rng(2).standard_normal((3, 512)) * 7.0
    out = O.rms_norm(z, None, 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(out ** 2, axis=1)), 1.0, rtol=1e-14)


def test_rope_matches_complex_multiplication():
    r = _rng(3)
    d_r = 16
    v = r.standard_normal((7, d_r))
    pos = np.array([0, 1, 5, 511, 4095, 65536, 131071])
    zc = v[:, 0::2] + 1j * v[:, 1::2]
    theta = 10000.0 ** (-np.arange(0, d_r, 2) / d_r)
    rot = zc * np.exp(1j * pos[:, None] * theta[None, :])
    out = O.rope(v, pos)
    np.testing.assert_allclose(out[:, 0::2], rot.real, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out[:, 1::2], rot.imag, rtol=1e-12, atol=1e-12)


def test_rope_position_zero_is_identity_and_preserves_norm():
    v = _rng(4).standard_normal((3, 64))
    np.testing.assert_array_equal(O.rope(v, np.zeros(3)), v)
    out = O.rope(v, np.array([3, 1000, 77777]))
    np.testing.assert_allclose(np.linalg.norm(out, axis=1), np.linalg.norm(v, axis=1), rtol=1e-13)


def test_rope_scores_depend_only_on_relative_position():
    # « Vérifier une couche compliquée »: scores unchanged when every position shifts
    r = _rng(5)
    q, k = r.standard_normal(32), r.standard_normal(32)
    for (i, j, delta) in [(10, 3, 7), (4096, 0, 12345), (100, 99, 131000)]:
        a = O.rope(q, i) @ O.rope(k, j)
        b = O.rope(q, i + delta) @ O.rope(k, j + delta)
        assert a == pytest.approx(b, rel=1e-9, abs=1e-9)


def test_softmax_brute_force_sums_to_one_and_lse_matches_scipy():
    r = _rng(6)
    s = r.standard_normal((4, 11)) * 5
    p, lse = O.softmax_stats(s)
    for row in range(4):
        assert math.fsum(p[row]) == pytest.approx(1.0, abs=1e-15)
        brute = [math.exp(x) / math.fsum(math.exp(y) for y in s[row]) for x in s[row]]
        np.testing.assert_allclose(p[row], brute, rtol=1e-14)
    np.testing.assert_allclose(lse, logsumexp(s, axis=1), rtol=1e-14)


# ------------------------------------------------------------------------------------------
# the definition against torch's scaled-dot-product attention (fp64)
# ------------------------------------------------------------------------------------------

def _sdpa_expanded(L):
    """Keys [W_UK·c ; k_r], values c·W_UV, causal among new tokens, via torch SDPA in fp64."""
    q = np.concatenate([L["q_nope"], L["q_rope"]], axis=-1)          # [s_q, H, D+d_r]
    s_q, H, _ = q.shape
    n = L["seqlen"]
    keys = np.stack([np.concatenate([L["c"][:n] @ L["W_UK"][h].T, L["k_r"][:n]], axis=1) for h in range(H)])
    vals = np.stack([L["c"][:n] @ L["W_UV"][h] for h in range(H)])
    mask = np.zeros((s_q, n), dtype=bool)
    for t in range(s_q):
        mask[t, : n - s_q + t + 1] = True
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q.transpose(1, 0, 2)), torch.from_numpy(keys), torch.from_numpy(vals),
        attn_mask=torch.from_numpy(mask), scale=L["sm_scale"])
    return out.numpy().transpose(1, 0, 2)


@pytest.mark.parametrize("s_q", [1, 3])
def test_expanded_definition_matches_torch_sdpa(s_q):
    L = _layer(seed=7, s_q=s_q, L=13)
    out, _ = O.expanded_decode(L["q_nope"], L["q_rope"], L["c"], L["k_r"], L["W_UK"], L["W_UV"], L["seqlen"], L["sm_scale"])
    np.testing.assert_allclose(out, _sdpa_expanded(L), rtol=1e-12, atol=1e-13)


def test_literal_loop_matches_expanded():
    L = _layer(seed=8, H=2, D=3, d_r=2, d_c=4, d_v=3, L=5, s_q=2)
    a, la = O.expanded_decode(L["q_nope"], L["q_rope"], L["c"], L["k_r"], L["W_UK"], L["W_UV"], L["seqlen"], L["sm_scale"])
    b, lb = O.literal_loop_decode(L["q_nope"], L["q_rope"], L["c"], L["k_r"], L["W_UK"], L["W_UV"], L["seqlen"], L["sm_scale"])
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(la, lb, rtol=1e-12, atol=1e-13)


def test_reduces_to_plain_mha_when_latent_is_the_keys():
    # d_c = H·D and W_UK[h] selecting the h-th block: keys are slices of c, no RoPE part
    H, D, n = 3, 4, 10
    r = _rng(9)
    c = r.standard_normal((n, H * D))
    W_UK = np.zeros((H, D, H * D))
    for h in range(H):
        W_UK[h, :, h * D:(h + 1) * D] = np.eye(D)
    W_UV = r.standard_normal((H, H * D, 5))
    q = r.standard_normal((1, H, D))
    out, _ = O.expanded_decode(q, np.zeros((1, H, 2)), c, np.zeros((n, 2)), W_UK, W_UV, n, 0.5)
    keys = torch.from_numpy(np.stack([c[:, h * D:(h + 1) * D] for h in range(H)]))
    vals = torch.from_numpy(np.stack([c @ W_UV[h] for h in range(H)]))
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q.transpose(1, 0, 2)), keys, vals, scale=0.5)
    np.testing.assert_allclose(out, ref.numpy().transpose(1, 0, 2), rtol=1e-12, atol=1e-13)


def test_single_position_returns_its_value():
    L = _layer(seed=10, L=1)
    out, lse = O.expanded_decode(L["q_nope"], L["q_rope"], L["c"], L["k_r"], L["W_UK"], L["W_UV"], 1, L["sm_scale"])
    for h in range(out.shape[1]):
        np.testing.assert_allclose(out[0, h], L["c"][0] @ L["W_UV"][h], rtol=1e-14)
    q_abs = np.concatenate([np.einsum("thd,hdc->thc", L["q_nope"], L["W_UK"]), L["q_rope"]], -1)
    o_lat, lse2 = O.absorbed_decode(q_abs, L["c"], L["k_r"], 1, L["sm_scale"])
    np.testing.assert_allclose(o_lat[0], np.broadcast_to(L["c"][0], o_lat[0].shape), rtol=1e-15)


def test_equal_scores_give_mean_of_latents():
    L = _layer(seed=11, L=17)
    d_c = L["c"].shape[1]
    q_abs = np.zeros((1, 4, d_c + 4))
    o_lat, lse = O.absorbed_decode(q_abs, L["c"], L["k_r"], 17, L["sm_scale"])
    np.testing.assert_allclose(o_lat[0], np.broadcast_to(L["c"].mean(axis=0), o_lat[0].shape), rtol=1e-13)
    np.testing.assert_allclose(lse, math.log(17), rtol=1e-15)


# ------------------------------------------------------------------------------------------
# the pages' algebraic identities
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("s_q", [1, 2, 4])
def test_absorbed_equals_expanded(s_q):
    # « Ce que DeepSeek fait de plus »: q·(W_UK c) = (q·W_UK)·c and Σ p (c W_UV) = (Σ p c) W_UV
    H, D, d_r, d_c, d_v, n = 6, 16, 8, 24, 10, 37
    L = _layer(seed=12 + s_q, H=H, D=D, d_r=d_r, d_c=d_c, d_v=d_v, L=n, s_q=s_q)
    pos = O.token_positions(n, s_q)
    q_rope_raw = L["q_rope"]
    q_rot = O.rope(q_rope_raw, pos[:, None] * np.ones((1, H)))
    ref, lse_ref = O.expanded_decode(L["q_nope"], q_rot, L["c"], L["k_r"], L["W_UK"], L["W_UV"], n, L["sm_scale"])
    q_abs = O.absorb_query(L["q_nope"], q_rope_raw, L["W_UK"], pos)
    o_lat, lse = O.absorbed_decode(q_abs, L["c"], L["k_r"], n, L["sm_scale"])
    out = O.out_projection(o_lat, L["W_UV"])
    scale = np.abs(ref).max()
    assert np.abs(out - ref).max() <= 1e-12 * scale
    assert np.abs(lse - lse_ref).max() <= 1e-12


def test_gqla_grouped_equals_absorbed_on_group_shared_weights():
    # « 2. Méthodologie »: the two decode paths are algebraically equal on the same weights
    H, g, D, d_r, d_c, d_v, n = 8, 2, 16, 8, 32, 16, 41
    r = _rng(20)
    W_UK_g = r.standard_normal((g, D, d_c)) / math.sqrt(d_c)
    W_UV_g = r.standard_normal((g, d_c, d_v)) / math.sqrt(d_c)
    c, k_r = r.standard_normal((n, d_c)), r.standard_normal((n, d_r))
    q_nope, q_rope_raw = r.standard_normal((1, H, D)), r.standard_normal((1, H, d_r))
    pos = O.token_positions(n, 1)
    scale = 1 / math.sqrt(D + d_r)
    K, V = O.gqla_expand(c, W_UK_g, W_UV_g)
    q_rot = O.rope(q_rope_raw, pos[:, None] * np.ones((1, H)))
    grouped, lse_g = O.gqla_grouped_decode(q_nope, q_rot, K, V, k_r, n, scale, g)
    W_UK = O.group_weights_per_head(W_UK_g, H)
    W_UV = O.group_weights_per_head(W_UV_g, H)
    o_lat, lse_a = O.absorbed_decode(O.absorb_query(q_nope, q_rope_raw, W_UK, pos), c, k_r, n, scale)
    absorbed = O.out_projection(o_lat, W_UV)
    assert np.abs(grouped - absorbed).max() <= 1e-12 * np.abs(absorbed).max()
    assert np.abs(lse_g - lse_a).max() <= 1e-12


def test_preabsorbed_output_equals_two_step_projection():
    """« Chemin MQA-Absorbé »: projecting the weighted latents through W_UV[h]·W_O[h] at once equals
    projecting each head through W_UV[h], concatenating and projecting through W_O (associativity;
    the two sides sum in different orders)."""
    r = _rng(44)
    s_q, H, d_c, d_v, C = 3, 4, 6, 5, 7
    o_lat = r.standard_normal((s_q, H, d_c))
    W_UV = r.standard_normal((H, d_c, d_v))
    W_O = r.standard_normal((H * d_v, C))
    two_step = O.out_projection(o_lat, W_UV, W_O)
    one_step = O.out_projection_preabsorbed(o_lat, O.preabsorbed_out_weights(W_UV, W_O))
    np.testing.assert_allclose(one_step, two_step, rtol=1e-12, atol=1e-12)
    # by hand for one output: sum over heads, latents and value columns
    want = sum(o_lat[1, h, c] * W_UV[h, c, e] * W_O[h * d_v + e, 2]
               for h in range(H) for c in range(d_c) for e in range(d_v))
    assert abs(one_step[1, 2] - want) < 1e-12 * max(1.0, abs(want))


def test_planted_head_minor_output_blocks_are_caught(monkeypatch):
    good = O.preabsorbed_out_weights

    def bad(W_UV, W_O):
        # W_O's rows taken head-minor (row e·H + h) instead of head-major (row h·d_v + e)
        W_UV = np.asarray(W_UV, float)
        H, d_c, d_v = W_UV.shape
        W_Ob = np.asarray(W_O, float).reshape(d_v, H, -1).transpose(1, 0, 2).reshape(H * d_v, -1)
        return good(W_UV, W_Ob)
    monkeypatch.setattr(O, "preabsorbed_out_weights", bad)
    with pytest.raises(AssertionError):
        test_preabsorbed_output_equals_two_step_projection()


def test_merge_of_disjoint_parts_equals_whole():
    L = _layer(seed=21, L=50)
    d_c = L["c"].shape[1]
    q_abs = _rng(22).standard_normal((1, 4, d_c + 4))
    full, lse = O.absorbed_decode(q_abs, L["c"], L["k_r"], 50, 0.3)
    parts, lses = [], []
    for lo, hi in [(0, 7), (7, 31), (31, 50)]:
        o, l = O.absorbed_decode(q_abs, L["c"][lo:hi], L["k_r"][lo:hi], hi - lo, 0.3)
        parts.append(o)
        lses.append(l)
    o, l = O.merge_partials(parts, lses)
    np.testing.assert_allclose(o, full, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(l, lse, rtol=1e-14)


def test_append_one_at_a_time_equals_bulk():
    # « Vérifier une couche compliquée »: whole sequence or piece by piece through the cache
    r = _rng(23)
    C, d_c, d_r, n = 20, 8, 4, 12
    x = r.standard_normal((n, C))
    W_DKV, W_KR = r.standard_normal((C, d_c)), r.standard_normal((C, d_r))
    c_all, kr_all = O.latent_rows(x, W_DKV, W_KR, np.arange(n))
    for j in range(n):
        c1, kr1 = O.latent_rows(x[j:j + 1], W_DKV, W_KR, np.array([j]))
        np.testing.assert_allclose(c1[0], c_all[j], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(kr1[0], kr_all[j], rtol=1e-13, atol=1e-13)


def _latent_rows_case():
    r = _rng(43)
    n, C, d_c, d_r = 6, 24, 10, 8
    x = r.standard_normal((n, C)) * r.uniform(0.2, 5.0, (n, 1))
    W_DKV, W_KR = r.standard_normal((C, d_c)), r.standard_normal((C, d_r))
    gamma = r.uniform(0.5, 1.5, d_c)
    positions = np.array([0, 1, 5, 77, 1000, 131071])
    return x, W_DKV, W_KR, gamma, positions


def test_latent_rows_match_torch_rms_norm_and_complex_rotation():
    """Cache rows (« L'idée : garder un résumé », « L'obstacle : RoPE »): the latent is torch's own
    rms_norm of x·W_DKV (its normalised_shape fixes the axis), times the gain; the RoPE key is
    x·W_KR with each adjacent pair (2i, 2i+1) read as a complex number and multiplied by
    exp(i·pos·10000^(-2i/d_r)) at the row's own position. Position 0 leaves the key unrotated."""
    x, W_DKV, W_KR, gamma, positions = _latent_rows_case()
    c, k_r = O.latent_rows(x, W_DKV, W_KR, positions, gamma, 1e-6, 10000.0)
    d_c, d_r = W_DKV.shape[1], W_KR.shape[1]
    c_ref = torch.nn.functional.rms_norm(torch.from_numpy(x @ W_DKV), (d_c,), torch.from_numpy(gamma), eps=1e-6).numpy()
    np.testing.assert_allclose(c, c_ref, rtol=1e-12, atol=1e-13)
    z = x @ W_KR
    pairs = z[:, 0::2] + 1j * z[:, 1::2]
    turn = 10000.0 ** (-2.0 * np.arange(d_r // 2) / d_r)
    rotated = pairs * np.exp(1j * positions[:, None].astype(float) * turn[None, :])
    k_ref = np.empty_like(z)
    k_ref[:, 0::2], k_ref[:, 1::2] = rotated.real, rotated.imag
    np.testing.assert_allclose(k_r, k_ref, rtol=1e-9, atol=1e-9)
    np.testing.assert_array_equal(k_r[0], z[0])
    c1, _ = O.latent_rows(x, W_DKV, W_KR, positions, None, 0.0)
    np.testing.assert_allclose((c1 ** 2).mean(axis=1), 1.0, rtol=1e-13)


def test_planted_latent_row_slips_are_caught(monkeypatch):
    """Three plausible slips in the cache-row oracle each fail the pin above: the key rotated one
    position late, the latent and the RoPE part normalised together, and the two column blocks of
    the concatenated projection [W_DKV | W_KR] taken in the wrong order."""
    good = O.latent_rows

    def late(x, W_DKV, W_KR, positions, gamma=None, eps=1e-6, base=10000.0):
        return good(x, W_DKV, W_KR, np.asarray(positions) + 1, gamma, eps, base)

    def joint(x, W_DKV, W_KR, positions, gamma=None, eps=1e-6, base=10000.0):
        d_c = np.asarray(W_DKV).shape[1]
        zn = O.rms_norm(np.asarray(x, float) @ np.concatenate([W_DKV, W_KR], 1), None, eps)
        c = zn[:, :d_c] * (1.0 if gamma is None else np.asarray(gamma))
        return c, O.rope(zn[:, d_c:], positions, base)

    def swapped(x, W_DKV, W_KR, positions, gamma=None, eps=1e-6, base=10000.0):
        d_c = np.asarray(W_DKV).shape[1]
        z = np.asarray(x, float) @ np.concatenate([W_KR, W_DKV], 1)
        return O.rms_norm(z[:, :d_c], gamma, eps), O.rope(z[:, d_c:], positions, base)

    for bad in (late, joint, swapped):
        monkeypatch.setattr(O, "latent_rows", bad)
        with pytest.raises(AssertionError):
            test_latent_rows_match_torch_rms_norm_and_complex_rotation()
    monkeypatch.setattr(O, "latent_rows", good)


def test_multi_token_step_equals_sequential_single_token_steps():
    # causal among the new tokens: token t of an s_q step is a 1-token step on seqlen - s_q + t + 1
    s_q, n = 4, 30
    L = _layer(seed=24, s_q=s_q, L=n)
    d_c = L["c"].shape[1]
    q_abs = _rng(25).standard_normal((s_q, 4, d_c + 4))
    o, lse = O.absorbed_decode(q_abs, L["c"], L["k_r"], n, 0.4)
    for t in range(s_q):
        o1, l1 = O.absorbed_decode(q_abs[t:t + 1], L["c"], L["k_r"], n - s_q + t + 1, 0.4)
        np.testing.assert_allclose(o[t], o1[0], rtol=1e-14)
        np.testing.assert_allclose(lse[t], l1[0], rtol=1e-14)


def test_future_tokens_do_not_change_earlier_outputs():
    s_q, n = 3, 20
    L = _layer(seed=26, s_q=s_q, L=n)
    d_c = L["c"].shape[1]
    q_abs = _rng(27).standard_normal((s_q, 4, d_c + 4))
    o, _ = O.absorbed_decode(q_abs, L["c"], L["k_r"], n, 0.4)
    c2 = L["c"].copy()
    c2[n - 1] += 100.0                      # the last new token's own row
    o2, _ = O.absorbed_decode(q_abs, c2, L["k_r"], n, 0.4)
    np.testing.assert_array_equal(o[:-1], o2[:-1])
    assert np.abs(o[-1] - o2[-1]).max() > 1e-3


def test_whole_layer_from_hidden_states_matches_sdpa():
    """Smallem-shaped layer from x (query chain, latent rows, RoPE, attention, W_O) against SDPA."""
    H, D, d_r, d_c, d_v, C, d_q, n = 4, 8, 4, 16, 8, 24, 12, 19
    r = _rng(28)
    x = r.standard_normal((n, C))
    W = dict(W_DKV=r.standard_normal((C, d_c)) / math.sqrt(C), W_KR=r.standard_normal((C, d_r)) / math.sqrt(C),
             W_DQ=r.standard_normal((C, d_q)) / math.sqrt(C), W_UQ=r.standard_normal((d_q, H * D)) / math.sqrt(d_q),
             W_QR=r.standard_normal((d_q, H * d_r)) / math.sqrt(d_q),
             W_UK=r.standard_normal((H, D, d_c)) / math.sqrt(d_c), W_UV=r.standard_normal((H, d_c, d_v)) / math.sqrt(d_c),
             W_O=r.standard_normal((H * d_v, C)) / math.sqrt(H * d_v))
    c, k_r = O.latent_rows(x, W["W_DKV"], W["W_KR"], np.arange(n))
    q_nope, q_raw, q_rot = O.query_parts(x[-1:], W["W_DQ"], W["W_UQ"], W["W_QR"], H, D, d_r, np.array([n - 1]))
    scale = 1 / math.sqrt(D + d_r)
    o_lat, _ = O.absorbed_decode(O.absorb_query(q_nope, q_raw, W["W_UK"], [n - 1]), c, k_r, n, scale)
    out = O.out_projection(o_lat, W["W_UV"], W["W_O"])
    Lyr = dict(q_nope=q_nope, q_rope=q_rot, c=c, k_r=k_r, W_UK=W["W_UK"], W_UV=W["W_UV"], seqlen=n, sm_scale=scale)
    ref = _sdpa_expanded(Lyr).reshape(1, -1) @ W["W_O"]
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-13)


def _identity_query_chain(x, gamma_q=None, eps=0.0, positions=None):
    """query_parts with W_DQ, W_UQ and W_QR all identities (C = d_q = H·D = H·d_r): its outputs are
    then x itself, normalised per token and split into heads, which the checks below can see
    without restating the formula."""
    H, D = 3, 4
    n, C = x.shape
    assert C == H * D
    eye = np.eye(C)
    pos = np.zeros(n) if positions is None else positions
    return O.query_parts(x, eye, eye, eye, H, D, D, pos, gamma_q, eps)


def test_query_parts_split_heads_in_order_and_normalise_each_token():
    """Query chain (« L'obstacle : RoPE », « Le code »): with identity projections, every head's
    part is a positive multiple of its own slice of x (head h = columns h·D .. h·D + D - 1, no
    mixing), the factor is shared by all heads of a token, and each token's query has mean square
    exactly 1 (RMSNorm with eps = 0, over that token's d_q values)."""
    x = _rng(40).standard_normal((5, 12)) * np.array([[0.1], [1.0], [3.0], [7.0], [0.5]])
    q_nope, q_raw, q_rot = _identity_query_chain(x)
    for part in (q_nope, q_raw):
        flat = part.reshape(5, 12)
        ratio = flat / x
        np.testing.assert_allclose(ratio, ratio[:, :1] * np.ones((1, 12)), rtol=1e-13)
        assert (ratio > 0).all()
        np.testing.assert_allclose((flat ** 2).mean(axis=1), 1.0, rtol=1e-13)
    np.testing.assert_allclose(q_rot, q_raw, rtol=0, atol=1e-15)   # RoPE at position 0 is the identity


def test_query_parts_scale_invariance_gain_and_rotation():
    """RMSNorm removes a token's scale; the gain γ_q multiplies c_q and so every output; the RoPE
    part is a rotation of q_rope_raw (pair norms kept) at the token's position."""
    x = _rng(41).standard_normal((3, 12))
    a = _identity_query_chain(x)
    b = _identity_query_chain(x * np.array([[5.0], [0.25], [40.0]]))
    for u, v in zip(a, b):
        np.testing.assert_allclose(u, v, rtol=1e-12, atol=1e-14)
    g = _identity_query_chain(x, gamma_q=np.full(12, 2.0))
    np.testing.assert_allclose(g[0], 2 * a[0], rtol=1e-13)
    np.testing.assert_allclose(g[1], 2 * a[1], rtol=1e-13)
    _, q_raw, q_rot = _identity_query_chain(x, positions=np.array([3, 17, 100]))
    pair = lambda v: np.hypot(v[..., 0::2], v[..., 1::2])
    np.testing.assert_allclose(pair(q_rot), pair(q_raw), rtol=1e-13)
    assert np.abs(q_rot - q_raw).max() > 1e-3


def test_query_parts_with_random_weights_match_torch_rms_norm():
    """Random projections: c_q through torch's own rms_norm (its normalised_shape fixes the axis),
    then the two up-projections; the oracle's heads are column blocks of those products."""
    r = _rng(42)
    n, C, d_q, H, D, d_r = 4, 20, 12, 3, 5, 2
    x = r.standard_normal((n, C))
    W_DQ, W_UQ, W_QR = r.standard_normal((C, d_q)), r.standard_normal((d_q, H * D)), r.standard_normal((d_q, H * d_r))
    gamma = r.uniform(0.5, 1.5, d_q)
    q_nope, q_raw, _ = O.query_parts(x, W_DQ, W_UQ, W_QR, H, D, d_r, np.zeros(n), gamma, 1e-6)
    c_q = torch.nn.functional.rms_norm(torch.from_numpy(x @ W_DQ), (d_q,), torch.from_numpy(gamma), eps=1e-6).numpy()
    for h in range(H):
        np.testing.assert_allclose(q_nope[:, h], c_q @ W_UQ[:, h * D:(h + 1) * D], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(q_raw[:, h], c_q @ W_QR[:, h * d_r:(h + 1) * d_r], rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------------------------------------
# planted mistakes: plausible slips in the oracle must fail the pins above
# ------------------------------------------------------------------------------------------

def _planted(monkeypatch, name, fn):
    monkeypatch.setattr(O, name, fn)


def test_planted_rope_sign_error_is_caught(monkeypatch):
    good = O.rope

    def bad(v, pos, base=10000.0):
        out = good(v, pos, base)
        out[..., 1::2] = -out[..., 1::2]   # a sign slip on the second coordinate of every pair
        return out
    _planted(monkeypatch, "rope", bad)
    with pytest.raises(AssertionError):
        test_rope_matches_complex_multiplication()


def test_planted_dropped_rope_term_is_caught(monkeypatch):
    def bad(q_abs, c, k_r, seqlen, sm_scale):
        d_c = np.asarray(c).shape[1]
        q = np.array(q_abs, dtype=float)
        q[..., d_c:] = 0.0
        return _ABSORBED(q, c, k_r, seqlen, sm_scale)
    _planted(monkeypatch, "absorbed_decode", bad)
    with pytest.raises(AssertionError):
        test_absorbed_equals_expanded(1)


def test_planted_transposed_absorption_is_caught(monkeypatch):
    def bad(q_nope, q_rope_raw, W_UK, positions, base=10000.0):
        # uses W_UK[h] as if it were laid out [d_c, D] on a square-free shape: reshape, not transpose
        H, D, d_c = np.asarray(W_UK).shape
        W_bad = np.asarray(W_UK).reshape(H, d_c, D).transpose(0, 2, 1)
        return _ABSORB(q_nope, q_rope_raw, W_bad, positions, base)
    _planted(monkeypatch, "absorb_query", bad)
    with pytest.raises(AssertionError):
        test_absorbed_equals_expanded(1)


def test_planted_wrong_causal_offset_is_caught(monkeypatch):
    def bad(q_abs, c, k_r, seqlen, sm_scale):
        # every new token sees all positions (no causal mask among the new tokens)
        q_abs = np.asarray(q_abs, float)
        outs, lses = [], []
        for t in range(q_abs.shape[0]):
            o, l = _ABSORBED(q_abs[t:t + 1], c, k_r, seqlen, sm_scale)
            outs.append(o[0])
            lses.append(l[0])
        return np.stack(outs), np.stack(lses)
    _planted(monkeypatch, "absorbed_decode", bad)
    with pytest.raises(AssertionError):
        test_multi_token_step_equals_sequential_single_token_steps()


def test_planted_wrong_scale_is_caught(monkeypatch):
    def bad(q_nope, q_rope, c, k_r, W_UK, W_UV, seqlen, sm_scale):
        return _EXPANDED(q_nope, q_rope, c, k_r, W_UK, W_UV, seqlen, sm_scale * math.sqrt(2.0))
    _planted(monkeypatch, "expanded_decode", bad)
    with pytest.raises(AssertionError):
        test_expanded_definition_matches_torch_sdpa(1)


def test_planted_wrong_group_assignment_is_caught(monkeypatch):
    _planted(monkeypatch, "group_of_head", lambda H, g: np.arange(H) % g)   # interleaved instead of contiguous
    monkeypatch.setattr(O, "group_weights_per_head", lambda W_g, H: np.asarray(W_g)[np.arange(H) // (H // np.asarray(W_g).shape[0])])
    with pytest.raises(AssertionError):
        test_gqla_grouped_equals_absorbed_on_group_shared_weights()


def test_planted_merge_without_max_shift_weighting_is_caught(monkeypatch):
    def bad(o_parts, lse_parts):
        o_parts = np.asarray(o_parts, float)
        return o_parts.mean(axis=0), np.asarray(lse_parts, float).max(axis=0)
    _planted(monkeypatch, "merge_partials", bad)
    with pytest.raises(AssertionError):
        test_merge_of_disjoint_parts_equals_whole()


def test_planted_transposed_head_split_is_caught(monkeypatch):
    def bad(x, W_DQ, W_UQ, W_QR, H, D, d_r, positions, gamma_q=None, eps=1e-6, base=10000.0):
        q_nope, q_raw, q_rot = _QUERY(x, W_DQ, W_UQ, W_QR, H, D, d_r, positions, gamma_q, eps, base)
        n = q_nope.shape[0]
        # heads taken as the inner index of the H·D columns instead of the outer one
        q_nope = q_nope.reshape(n, H * D).reshape(n, D, H).transpose(0, 2, 1)
        return q_nope, q_raw, q_rot
    _planted(monkeypatch, "query_parts", bad)
    with pytest.raises(AssertionError):
        test_query_parts_split_heads_in_order_and_normalise_each_token()


def test_planted_dropped_query_normalisation_is_caught(monkeypatch):
    def bad(x, W_DQ, W_UQ, W_QR, H, D, d_r, positions, gamma_q=None, eps=1e-6, base=10000.0):
        # the query latent c_q left unnormalised
        return _unnormalised_query(x, W_DQ, W_UQ, W_QR, H, D, d_r, positions, gamma_q, base)
    _planted(monkeypatch, "query_parts", bad)
    with pytest.raises(AssertionError):
        test_query_parts_scale_invariance_gain_and_rotation()


def _unnormalised_query(x, W_DQ, W_UQ, W_QR, H, D, d_r, positions, gamma_q, base):
    """The query chain with its RMSNorm left out (a planted slip)."""
    c_q = np.asarray(x, float) @ np.asarray(W_DQ, float)
    if gamma_q is not None:
        c_q = c_q * gamma_q
    n = c_q.shape[0]
    q_nope = (c_q @ W_UQ).reshape(n, H, D)
    q_raw = (c_q @ W_QR).reshape(n, H, d_r)
    return q_nope, q_raw, O.rope(q_raw, np.asarray(positions, float)[:, None] * np.ones((1, H)), base)


_QUERY = O.query_parts
_ABSORBED = O.absorbed_decode
_ABSORB = O.absorb_query
_EXPANDED = O.expanded_decode
