"""Plain, slow, fp64 restatement of one MLA decode step (the oracle).

TEST INFRASTRUCTURE: only tests/, the entry module's smoke() and bench.py's CPU-baseline and
reference arm use this file. It shares no code with the CUDA path.

Sources (page title, then section):
  [P1] « L'attention latente : compresser le cache » (Smallem series, article 13)
       - « L'idée : garder un résumé »: c = rms(x·W_latent) is the only cached vector; keys and
         values of every head are c·W_clé and c·W_valeur.
       - « L'obstacle : RoPE »: a separate rotated key k_r = rotation(x·W_clé_tournée) shared by
         all heads and a rotated query q_r per head; score = (q·k + q_r·k_r)/sqrt(D + d_r).
       - « Le code »: the ten projections of the layer; RMSNorm on both latents.
       - « Vérifier une couche compliquée »: the layer is checked against a naive rewrite with
         loops, keys really concatenated and the softmax written term by term.
       - « Ce que DeepSeek fait de plus »: q·(c·W_clé) = (q·W_cléᵀ)·c and the weighted sum of
         values equals the weighted sum of latents projected once by W_valeur.
  [P2] « Le cache clé-valeur », section « Le mécanisme d'attention »: the attention output is the
       softmax-weighted average of the values, weights summing to one, scores scaled by sqrt(d_k).
  [P4] « Résumé technique : GQLA – Attention Latente par Groupes de Requêtes … », section
       « 2. Méthodologie » (« Architecture », « Chemin MQA-Absorbé », « Chemin GQA »): W_UK, W_UV
       indexed by g groups; the absorbed path attends the latent cache plus one shared RoPE key;
       the GQA path expands the latent into g key/value groups; the two are algebraically equal.

Readings where the pages are silent (each is listed with its reason in the design notes):
  * RMSNorm: z / sqrt(mean(z²) + eps) · gamma, eps = 1e-6, gamma = 1 by default.
  * RoPE: adjacent pairs (2i, 2i+1) of a d_r vector turn by pos·base^(-2i/d_r), base 10000.
  * Weight layouts: W_UK [H, D, d_c] (k_h = W_UK[h]·c), W_UV [H, d_c, d_v] (v_h = c·W_UV[h]).
  * A sequence's length counts this step's s_q new tokens; new token t sits at position
    len - s_q + t and sees positions 0 .. len - s_q + t (causal among the new tokens).
  * GQLA groups are contiguous: head h belongs to group h // (H / g).
  * lse is the natural log of the sum of exp(scaled score) over the visible positions.
"""
from __future__ import annotations

import math

import numpy as np

f64 = np.float64


# ----------------------------------------------------------------------------------------------
# building blocks
# ----------------------------------------------------------------------------------------------

def rms_norm(z, gamma=None, eps: float = 1e-6):
    """[P1] « L'idée : garder un résumé » / « Le code »: rms(·) over the last axis, times gain."""
    z = np.asarray(z, dtype=f64)
    out = z / np.sqrt(np.mean(z * z, axis=-1, keepdims=True) + eps)
    if gamma is not None:
        out = out * np.asarray(gamma, dtype=f64)
    return out


def rope_frequencies(d_r: int, base: float = 10000.0):
    """Turn rate of pair i: base^(-2i/d_r), i = 0 .. d_r/2 - 1 ([P1] « L'obstacle : RoPE »)."""
    i = np.arange(d_r // 2, dtype=f64)
    return base ** (-2.0 * i / d_r)


def rope(v, pos, base: float = 10000.0):
    """Rotate adjacent pairs (2i, 2i+1) of the last axis by pos·theta_i.

    ``pos`` broadcasts against v's leading axes (one position per vector).
    [P1] « L'obstacle : RoPE »: the rotation that carries the position on the decoupled part.
    """
    v = np.asarray(v, dtype=f64)
    d_r = v.shape[-1]
    theta = rope_frequencies(d_r, base)
    ang = np.asarray(pos, dtype=f64)[..., None] * theta           # [..., d_r/2]
    cos, sin = np.cos(ang), np.sin(ang)
    a, b = v[..., 0::2], v[..., 1::2]
    out = np.empty_like(v)
    out[..., 0::2] = a * cos - b * sin
    out[..., 1::2] = a * sin + b * cos
    return out


def token_positions(seqlen: int, s_q: int):
    """Positions of this step's new tokens: seqlen - s_q .. seqlen - 1."""
    return np.arange(seqlen - s_q, seqlen, dtype=np.int64)


def softmax_stats(s):
    """Softmax over the last axis with its log-sum-exp ([P2] « Le mécanisme d'attention »)."""
    s = np.asarray(s, dtype=f64)
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=-1, keepdims=True)
    return e / l, (m + np.log(l))[..., 0]


# ----------------------------------------------------------------------------------------------
# a1: cache append, and the query chain
# ----------------------------------------------------------------------------------------------

def latent_rows(x, W_DKV, W_KR, positions, gamma=None, eps=1e-6, base=10000.0):
    """Cache rows of hidden states x [n, C] at the given positions.

    c = RMSNorm(x·W_DKV)·gamma  [n, d_c]   ([P1] « L'idée : garder un résumé »)
    k_r = RoPE(x·W_KR, pos)     [n, d_r]   ([P1] « L'obstacle : RoPE », one key for all heads)
    """
    x = np.asarray(x, dtype=f64)
    c = rms_norm(x @ np.asarray(W_DKV, dtype=f64), gamma, eps)
    k_r = rope(x @ np.asarray(W_KR, dtype=f64), positions, base)
    return c, k_r


def query_parts(x, W_DQ, W_UQ, W_QR, H, D, d_r, positions, gamma_q=None, eps=1e-6, base=10000.0):
    """Query of new tokens x [n, C] ([P1] « L'obstacle : RoPE » and « Le code »).

    c_q = RMSNorm(x·W_DQ)·gamma_q; q_nope = c_q·W_UQ split into H heads of D;
    q_rope = RoPE(c_q·W_QR split into H heads of d_r, pos)  (one rotated query part per head).
    Returns q_nope [n, H, D], q_rope_raw [n, H, d_r] (before rotation), q_rope [n, H, d_r].
    """
    x = np.asarray(x, dtype=f64)
    c_q = rms_norm(x @ np.asarray(W_DQ, dtype=f64), gamma_q, eps)
    n = x.shape[0]
    q_nope = (c_q @ np.asarray(W_UQ, dtype=f64)).reshape(n, H, D)
    q_rope_raw = (c_q @ np.asarray(W_QR, dtype=f64)).reshape(n, H, d_r)
    pos = np.asarray(positions, dtype=f64)[:, None] * np.ones((1, H))
    return q_nope, q_rope_raw, rope(q_rope_raw, pos, base)


# ----------------------------------------------------------------------------------------------
# the definition: expanded multi-head attention on [c·W_UK ; k_r], values c·W_UV
# ----------------------------------------------------------------------------------------------

def expanded_decode(q_nope, q_rope, c, k_r, W_UK, W_UV, seqlen, sm_scale):
    """Ground truth for one sequence: keys and values of every head rebuilt from the latents.

    q_nope [s_q, H, D], q_rope [s_q, H, d_r] (already rotated), c [>=seqlen, d_c],
    k_r [>=seqlen, d_r] (rotated), W_UK [H, D, d_c], W_UV [H, d_c, d_v].
    Key of head h at j: [W_UK[h]·c_j ; k_r,j]; value: c_j·W_UV[h] ([P1] « L'idée : garder un
    résumé » and « L'obstacle : RoPE »). Score (q·k + q_r·k_r)·sm_scale; softmax-weighted average
    of the values ([P2] « Le mécanisme d'attention »). Token t sees positions < seqlen - s_q + t + 1.
    Returns out [s_q, H, d_v], lse [s_q, H].
    """
    q_nope = np.asarray(q_nope, f64)
    q_rope = np.asarray(q_rope, f64)
    c = np.asarray(c, f64)[:seqlen]
    k_r = np.asarray(k_r, f64)[:seqlen]
    W_UK = np.asarray(W_UK, f64)
    W_UV = np.asarray(W_UV, f64)
    s_q, H, _ = q_nope.shape
    d_v = W_UV.shape[2]
    out = np.zeros((s_q, H, d_v))
    lse = np.zeros((s_q, H))
    for h in range(H):
        k_h = c @ W_UK[h].T            # [L, D]
        v_h = c @ W_UV[h]              # [L, d_v]
        for t in range(s_q):
            n_vis = seqlen - s_q + t + 1
            s = (k_h[:n_vis] @ q_nope[t, h] + k_r[:n_vis] @ q_rope[t, h]) * sm_scale
            p, lse[t, h] = softmax_stats(s)
            out[t, h] = p @ v_h[:n_vis]
    return out, lse


def literal_loop_decode(q_nope, q_rope, c, k_r, W_UK, W_UV, seqlen, sm_scale):
    """The same quantity with pure-Python loops, keys really concatenated and the softmax written
    term by term ([P1] « Vérifier une couche compliquée »). For tiny inputs only."""
    s_q, H, D = len(q_nope), len(q_nope[0]), len(q_nope[0][0])
    d_c, d_v = len(c[0]), len(W_UV[0][0])
    out = [[[0.0] * d_v for _ in range(H)] for _ in range(s_q)]
    lse = [[0.0] * H for _ in range(s_q)]
    for t in range(s_q):
        n_vis = seqlen - s_q + t + 1
        for h in range(H):
            query = [float(v) for v in q_nope[t][h]] + [float(v) for v in q_rope[t][h]]
            scores = []
            values = []
            for j in range(n_vis):
                key = [sum(float(W_UK[h][d][i]) * float(c[j][i]) for i in range(d_c)) for d in range(D)]
                key = key + [float(v) for v in k_r[j]]
                scores.append(sum(a * b for a, b in zip(query, key)) * sm_scale)
                values.append([sum(float(c[j][i]) * float(W_UV[h][i][e]) for i in range(d_c))
                               for e in range(d_v)])
            top = max(scores)
            weights = [math.exp(s - top) for s in scores]
            total = sum(weights)
            for j in range(n_vis):
                for e in range(d_v):
                    out[t][h][e] += weights[j] / total * values[j][e]
            lse[t][h] = top + math.log(total)
    return np.array(out), np.array(lse)


# ----------------------------------------------------------------------------------------------
# a2, a3, a5: the absorbed rewrite
# ----------------------------------------------------------------------------------------------

def absorb_query(q_nope, q_rope_raw, W_UK, positions, base=10000.0):
    """q_abs = [q_nope_h·W_UK[h] ; RoPE(q_rope_raw_h, pos)] per token and head.

    [P1] « Ce que DeepSeek fait de plus »: q·(W_UK·c) = (q·W_UK)·c, so the query is projected into
    latent space once. q_nope [s_q, H, D], q_rope_raw [s_q, H, d_r], positions [s_q].
    Returns q_abs [s_q, H, d_c + d_r].
    """
    q_nope = np.asarray(q_nope, f64)
    W_UK = np.asarray(W_UK, f64)
    s_q, H, _ = q_nope.shape
    q_lat = np.einsum("thd,hdc->thc", q_nope, W_UK)
    pos = np.asarray(positions, f64)[:, None] * np.ones((1, H))
    q_r = rope(np.asarray(q_rope_raw, f64), pos, base)
    return np.concatenate([q_lat, q_r], axis=-1)


def absorbed_decode(q_abs, c, k_r, seqlen, sm_scale):
    """Attention directly over the cached latents ([P1] « Ce que DeepSeek fait de plus »;
    [P4] « Chemin MQA-Absorbé »): all heads attend the same rows [c_j ; k_r,j].

    q_abs [s_q, H, d_c + d_r]; returns o_lat [s_q, H, d_c] (softmax-weighted average of the latent
    rows) and lse [s_q, H].
    """
    q_abs = np.asarray(q_abs, f64)
    rows = np.concatenate([np.asarray(c, f64)[:seqlen], np.asarray(k_r, f64)[:seqlen]], axis=1)
    d_c = np.asarray(c).shape[1]
    s_q, H, _ = q_abs.shape
    o_lat = np.zeros((s_q, H, d_c))
    lse = np.zeros((s_q, H))
    for t in range(s_q):
        n_vis = seqlen - s_q + t + 1
        s = (q_abs[t] @ rows[:n_vis].T) * sm_scale           # [H, n_vis]
        p, lse[t] = softmax_stats(s)
        o_lat[t] = p @ rows[:n_vis, :d_c]
    return o_lat, lse


def out_projection(o_lat, W_UV, W_O=None):
    """out_h = o_lat_h·W_UV[h] ([P1] « Ce que DeepSeek fait de plus »: the weighted latent sum is
    projected once by W_valeur); with W_O [H*d_v, C] the heads are concatenated and projected
    (the layer's ``proj`` in [P1] « Le code »). o_lat [s_q, H, d_c] -> [s_q, H, d_v] or [s_q, C]."""
    out = np.einsum("thc,hce->the", np.asarray(o_lat, f64), np.asarray(W_UV, f64))
    if W_O is None:
        return out
    s_q = out.shape[0]
    return out.reshape(s_q, -1) @ np.asarray(W_O, f64)


def preabsorbed_out_weights(W_UV, W_O):
    """The value up-projection absorbed into the output projection ([P4] « Chemin MQA-Absorbé »: the
    up-projections are absorbed into the query and output projections): head h's block of W_O
    (rows h·d_v .. h·d_v + d_v - 1) premultiplied by W_UV[h]. W_UV [H, d_c, d_v], W_O [H·d_v, C]
    -> W_UVO [H, d_c, C]."""
    W_UV = np.asarray(W_UV, f64)
    H, d_c, d_v = W_UV.shape
    W_O = np.asarray(W_O, f64).reshape(H, d_v, -1)
    return np.einsum("hce,heo->hco", W_UV, W_O)


def out_projection_preabsorbed(o_lat, W_UVO):
    """The layer output straight from the weighted latents: sum over heads of o_lat_h · W_UVO[h].
    o_lat [s_q, H, d_c], W_UVO [H, d_c, C] -> [s_q, C]."""
    return np.einsum("thc,hco->to", np.asarray(o_lat, f64), np.asarray(W_UVO, f64))


def merge_partials(o_parts, lse_parts):
    """Combine softmax partials computed over disjoint position sets.

    With LSE = log Σ_s exp(lse_s), the full result is Σ_s exp(lse_s - LSE)·o_s. This is the
    softmax over a union of sets written with per-set normalisers; it is how a sequence that is
    split across workers is put back together.
    o_parts [n, ..., d], lse_parts [n, ...] -> (o [..., d], lse [...]).
    """
    lse_parts = np.asarray(lse_parts, f64)
    o_parts = np.asarray(o_parts, f64)
    m = np.max(lse_parts, axis=0)
    w = np.exp(lse_parts - m)
    tot = np.sum(w, axis=0)
    o = np.sum(w[..., None] * o_parts, axis=0) / tot[..., None]
    return o, m + np.log(tot)


# ----------------------------------------------------------------------------------------------
# a6: the GQLA grouped (GQA) path
# ----------------------------------------------------------------------------------------------

def group_of_head(H: int, g: int):
    """Contiguous grouping: head h uses group h // (H/g) ([P4] « Architecture »)."""
    return np.arange(H) // (H // g)


def gqla_expand(c, W_UK_g, W_UV_g):
    """Expand latent rows into g groups of keys and values once, when the cache is written
    ([P4] « Chemin GQA »). c [L, d_c] -> K [L, g, D], V [L, g, d_v]."""
    c = np.asarray(c, f64)
    K = np.einsum("gdc,lc->lgd", np.asarray(W_UK_g, f64), c)
    V = np.einsum("lc,gce->lge", c, np.asarray(W_UV_g, f64))
    return K, V


def gqla_grouped_decode(q_nope, q_rope, K, V, k_r, seqlen, sm_scale, g):
    """Standard grouped-query attention on the expanded cache plus the shared RoPE key.

    q_nope [s_q, H, D], q_rope [s_q, H, d_r] (rotated), K [>=seqlen, g, D], V [>=seqlen, g, d_v],
    k_r [>=seqlen, d_r]. Head h scores (q_h·K_g(h),j + q_r,h·k_r,j)·sm_scale ([P4] « Chemin GQA »).
    Returns out [s_q, H, d_v], lse [s_q, H].
    """
    q_nope = np.asarray(q_nope, f64)
    q_rope = np.asarray(q_rope, f64)
    K = np.asarray(K, f64)[:seqlen]
    V = np.asarray(V, f64)[:seqlen]
    k_r = np.asarray(k_r, f64)[:seqlen]
    s_q, H, _ = q_nope.shape
    grp = group_of_head(H, g)
    out = np.zeros((s_q, H, V.shape[2]))
    lse = np.zeros((s_q, H))
    for t in range(s_q):
        n_vis = seqlen - s_q + t + 1
        for h in range(H):
            s = (K[:n_vis, grp[h]] @ q_nope[t, h] + k_r[:n_vis] @ q_rope[t, h]) * sm_scale
            p, lse[t, h] = softmax_stats(s)
            out[t, h] = p @ V[:n_vis, grp[h]]
    return out, lse


def group_weights_per_head(W_g, H):
    """W_UK / W_UV of every head from the group-indexed ones (head h -> group h // (H/g))."""
    W_g = np.asarray(W_g, f64)
    return W_g[group_of_head(H, W_g.shape[0])]


# ----------------------------------------------------------------------------------------------
# paged cache helpers (no arithmetic of the method: gather rows by page table)
# ----------------------------------------------------------------------------------------------

def gather_rows(pool, table_row, seqlen, page_size=64):
    """Rows 0..seqlen-1 of one sequence from a paged pool [num_pages*page_size, ...]."""
    pool = np.asarray(pool)
    idx = np.arange(seqlen)
    return pool[np.asarray(table_row, np.int64)[idx // page_size] * page_size + idx % page_size]
