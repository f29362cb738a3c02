"""Seeded synthetic workloads for absorbed MLA decode and its GQLA grouped path.

Everything here is a random draw, a shape, a length list or a page table. Both the oracle
tests and the CUDA tests take their inputs from these functions, so the two sides always see
the same numbers; this module itself computes no attention, normalisation or rotation.

Recipe (one decode step of one layer):
  * hidden states x ~ N(0, 1); every weight ~ N(0, 1/fan_in); RMSNorm gains = 1;
    RoPE base 10000 (the Smallem configuration on « L'attention latente : compresser le cache »).
  * numpy PCG64 streams: weights 0, decode-step inputs 1, cache rows 2, lengths 3, page table 4.
  * Cached latent rows of the large workloads are drawn directly from the distribution that
    RMSNorm(x·W_DKV) has when x ~ N(0, I_C) and W_DKV ~ N(0, 1/C): for a fixed x the product is an
    isotropic Gaussian vector, so after RMS normalisation (gain 1) the row is uniform on the sphere
    of radius sqrt(d_c). It is sampled as a Gaussian vector rescaled to that radius. The shared
    RoPE key x·W_KR is an isotropic Gaussian with variance |x|²/C ≈ 1 and a rotation keeps it
    one, so it is drawn N(0, 1). The only thing this drops is the O(1/sqrt(C)) correlation between
    rows that a shared W_DKV induces.
  * Queries q_nope and q_rope_raw are c_q·W_UQ and c_q·W_QR with |c_q|² = d_q (an RMS-normalised
    query latent) and weights N(0, 1/d_q): entries are N(0, 1), drawn directly.
  * Page size 64; a sequence's pages are consecutive ("contiguous") or a seeded permutation of
    all pages ("random").
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "workload", "seq_lengths", "block_table", "weights",
    "decode_step_inputs", "cache_row_chunks", "context_hidden_states", "gqla_cache_chunks",
    "SEED_WEIGHTS", "SEED_DECODE", "SEED_CACHE", "SEED_LENGTHS", "SEED_PAGES", "CACHE_CHUNK_ROWS",
]

SEED_WEIGHTS = 0
SEED_DECODE = 1
SEED_CACHE = 2
SEED_LENGTHS = 3
SEED_PAGES = 4

# cache rows are drawn in fixed chunks so that the values never depend on who asks for them
CACHE_CHUNK_ROWS = 16384


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str                 # storage type of cache, weights and queries: "f32" or "bf16"
    B: int                     # sequences in the batch
    s_q: int                   # new query tokens per sequence this step
    H: int                     # query heads
    D: int                     # no-RoPE query/key head width (qk_nope)
    d_r: int                   # decoupled RoPE width, one key shared by all heads
    d_c: int                   # latent width
    d_v: int                   # value head width
    C: int                     # model width
    d_q: int = 0               # query latent width (0: queries are drawn directly)
    g: int = 0                 # GQLA groups (0: absorbed path only)
    lengths: tuple = ("fixed", 4096)
    pages: str = "contiguous"  # or "random"
    page_size: int = 64
    rope_base: float = 10000.0
    rms_eps: float = 1e-6
    description: str = ""
    latent_bits: int = 16      # 8: the latent rows are kept as E4M3 codes with one scale per row

    @property
    def d_qk(self) -> int:
        return self.D + self.d_r

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.D + self.d_r)

    @property
    def row_width(self) -> int:
        """Width of one interleaved cache row [latent ; rope key]."""
        return self.d_c + self.d_r


WORKLOADS = {
    w.name: w for w in [
        Workload("smallem_fp32", "f32", B=1, s_q=1, H=8, D=64, d_r=16, d_c=128, d_v=64, C=512,
                 d_q=256, lengths=("fixed", 512),
                 description="Smallem-scale layer, fp32, one new token attending 512 positions"),
        Workload("dsv3_b64_l4096", "bf16", B=64, s_q=1, H=128, D=128, d_r=64, d_c=512, d_v=128,
                 C=7168, lengths=("fixed", 4096),
                 description="DeepSeek-V2/V3-shaped absorbed decode, batch 64 x 4096 positions"),
        Workload("dsv3_fromx_b64_l4096", "bf16", B=64, s_q=1, H=128, D=128, d_r=64, d_c=512, d_v=128,
                 C=7168, d_q=1536, lengths=("fixed", 4096),
                 description="the DeepSeek-shaped step from hidden states: queries through the query chain "
                             "(d_q = 1536), batch 64 x 4096 positions"),
        Workload("longctx_b8", "bf16", B=8, s_q=1, H=128, D=128, d_r=64, d_c=512, d_v=128,
                 C=7168, lengths=("uniform", 16384, 131072),
                 description="long-context absorbed decode, 8 sequences of 16K-128K positions"),
        Workload("gqla_g8_b32_l8192", "bf16", B=32, s_q=1, H=128, D=128, d_r=64, d_c=512, d_v=128,
                 C=7168, g=8, lengths=("fixed", 8192),
                 description="GQLA grouped path, g=8 groups of 16 heads, batch 32 x 8192"),
        Workload("mtp_sq2_b128", "bf16", B=128, s_q=2, H=128, D=128, d_r=64, d_c=512, d_v=128,
                 C=7168, lengths=("uniform", 1024, 32768), pages="random",
                 description="multi-token absorbed decode, 2 tokens per step, random page table"),
        Workload("mtp_sq4_b128", "bf16", B=128, s_q=4, H=128, D=128, d_r=64, d_c=512, d_v=128,
                 C=7168, lengths=("uniform", 1024, 32768), pages="random",
                 description="multi-token absorbed decode, 4 tokens per step, random page table"),
        Workload("dsv3_fp8_b64_l4096", "bf16", B=64, s_q=1, H=128, D=128, d_r=64, d_c=512, d_v=128, C=7168,
                 latent_bits=8,
                 description="the DeepSeek-shaped batch over an 8-bit latent cache (E4M3 codes, one fp32 scale "
                             "per row, 16-bit RoPE keys)"),
    ]
}


def workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return replace(w, **overrides) if overrides else w


def _rng(*seed):
    return np.random.Generator(np.random.PCG64(list(seed)))


def seq_lengths(w: Workload) -> np.ndarray:
    """Cached positions per sequence, counting this step's s_q new tokens."""
    kind = w.lengths[0]
    if kind == "fixed":
        return np.full(w.B, w.lengths[1], dtype=np.int32)
    if kind == "uniform":
        lo, hi = w.lengths[1], w.lengths[2]
        return _rng(SEED_LENGTHS).integers(lo, hi + 1, size=w.B).astype(np.int32)
    if kind == "list":
        out = np.asarray(w.lengths[1], dtype=np.int32)
        assert out.shape == (w.B,)
        return out
    raise ValueError(kind)


def block_table(w: Workload, lens: np.ndarray):
    """Page table [B, max_pages] (int32) and the number of pages in the pool.

    Unused table entries hold 0, a valid page, so that no reader can ever leave the pool.
    """
    ps = w.page_size
    npages = (lens.astype(np.int64) + ps - 1) // ps
    total = int(npages.sum())
    max_pages = max(1, int(npages.max()) if len(npages) else 1)
    if w.pages == "contiguous":
        ids = np.arange(total, dtype=np.int64)
    elif w.pages == "random":
        ids = _rng(SEED_PAGES).permutation(total)
    else:
        raise ValueError(w.pages)
    table = np.zeros((w.B, max_pages), dtype=np.int32)
    off = 0
    for b in range(w.B):
        n = int(npages[b])
        table[b, :n] = ids[off:off + n]
        off += n
    return table, max(total, 1)


def _normal(rng, shape, std):
    return (rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std))


def weights(w: Workload) -> dict:
    """All weights of one MLA layer as float32 arrays (fan-in scaled Gaussians, unit gains).

    Layouts: W_DKV [C, d_c], W_KR [C, d_r], W_UK [H, D, d_c], W_UV [H, d_c, d_v],
    W_O [H*d_v, C], W_DQ [C, d_q], W_UQ [d_q, H*D], W_QR [d_q, H*d_r].
    """
    rng = _rng(SEED_WEIGHTS)
    out = {
        "W_DKV": _normal(rng, (w.C, w.d_c), 1.0 / math.sqrt(w.C)),
        "W_KR": _normal(rng, (w.C, w.d_r), 1.0 / math.sqrt(w.C)),
        "gamma": np.ones(w.d_c, dtype=np.float32),
        "W_UK": _normal(rng, (w.H, w.D, w.d_c), 1.0 / math.sqrt(w.d_c)),
        "W_UV": _normal(rng, (w.H, w.d_c, w.d_v), 1.0 / math.sqrt(w.d_c)),
        "W_O": _normal(rng, (w.H * w.d_v, w.C), 1.0 / math.sqrt(w.H * w.d_v)),
    }
    if w.d_q:
        out["W_DQ"] = _normal(rng, (w.C, w.d_q), 1.0 / math.sqrt(w.C))
        out["gamma_q"] = np.ones(w.d_q, dtype=np.float32)
        out["W_UQ"] = _normal(rng, (w.d_q, w.H * w.D), 1.0 / math.sqrt(w.d_q))
        out["W_QR"] = _normal(rng, (w.d_q, w.H * w.d_r), 1.0 / math.sqrt(w.d_q))
    if w.g:
        # GQLA: up-projections indexed by group, not by head
        out["W_UK_g"] = _normal(rng, (w.g, w.D, w.d_c), 1.0 / math.sqrt(w.d_c))
        out["W_UV_g"] = _normal(rng, (w.g, w.d_c, w.d_v), 1.0 / math.sqrt(w.d_c))
    return out


def decode_step_inputs(w: Workload) -> dict:
    """This step's inputs: hidden states of the new tokens and their query parts.

    x [B, s_q, C]; q_nope [B, s_q, H, D]; q_rope_raw [B, s_q, H, d_r] (before rotation).
    q_abs [B, s_q, H, d_c + d_r] is a query already in latent space, for checks of the decode kernel
    on its own: the latent part is N(0, D/d_c) (the law of q_nope·W_UK[h] for |q_nope|² = D and
    W_UK ~ N(0, 1/d_c)), the RoPE part N(0, 1). o_lat [B, s_q, H, d_c] ~ N(0, 1) feeds the output
    projection on its own.
    """
    rng = _rng(SEED_DECODE)
    out = {
        "x": _normal(rng, (w.B, w.s_q, w.C), 1.0),
        "q_nope": _normal(rng, (w.B, w.s_q, w.H, w.D), 1.0),
        "q_rope_raw": _normal(rng, (w.B, w.s_q, w.H, w.d_r), 1.0),
    }
    rng2 = _rng(SEED_DECODE, 1)
    q_abs = np.empty((w.B, w.s_q, w.H, w.d_c + w.d_r), dtype=np.float32)
    q_abs[..., :w.d_c] = _normal(rng2, (w.B, w.s_q, w.H, w.d_c), math.sqrt(w.D / w.d_c))
    q_abs[..., w.d_c:] = _normal(rng2, (w.B, w.s_q, w.H, w.d_r), 1.0)
    out["q_abs"] = q_abs
    out["o_lat"] = _normal(rng2, (w.B, w.s_q, w.H, w.d_c), 1.0)
    return out


def context_hidden_states(w: Workload, L: int, b: int = 0) -> np.ndarray:
    """Hidden states x_j ~ N(0, 1) [L, C] of every position of sequence b (small layers only)."""
    return _normal(_rng(SEED_CACHE, 1_000_000 + b), (L, w.C), 1.0)


def cache_row_chunks(w: Workload, n_rows: int):
    """Yield (start, c [n, d_c], k_r [n, d_r]) float32 chunks of cached rows 0..n_rows-1.

    Row r of the pool is drawn from stream (SEED_CACHE, r // CACHE_CHUNK_ROWS); c is uniform on the
    sphere of radius sqrt(d_c), k_r ~ N(0, 1).
    """
    for start in range(0, n_rows, CACHE_CHUNK_ROWS):
        rng = _rng(SEED_CACHE, start // CACHE_CHUNK_ROWS)
        n = min(CACHE_CHUNK_ROWS, n_rows - start)
        g = rng.standard_normal(size=(CACHE_CHUNK_ROWS, w.d_c), dtype=np.float32)[:n]
        kr = rng.standard_normal(size=(CACHE_CHUNK_ROWS, w.d_r), dtype=np.float32)[:n]
        radius = np.float32(math.sqrt(w.d_c))
        c = g * (radius / np.sqrt(np.sum(g.astype(np.float64) ** 2, axis=1, keepdims=True))).astype(np.float32)
        yield start, c, kr


def gqla_cache_chunks(w: Workload, n_rows: int):
    """Yield (start, K [n, g, D], V [n, g, d_v], k_r [n, d_r]) float32 chunks for the GQA cache.

    For a latent row on the sphere of radius sqrt(d_c) and group weights N(0, 1/d_c), every entry
    of the expanded key and value is N(0, 1); they are drawn directly (bench sizes only: the
    parity tests build them from the latent rows instead).
    """
    for start in range(0, n_rows, CACHE_CHUNK_ROWS):
        rng = _rng(SEED_CACHE, 500_000 + start // CACHE_CHUNK_ROWS)
        n = min(CACHE_CHUNK_ROWS, n_rows - start)
        K = rng.standard_normal(size=(CACHE_CHUNK_ROWS, w.g, w.D), dtype=np.float32)[:n]
        V = rng.standard_normal(size=(CACHE_CHUNK_ROWS, w.g, w.d_v), dtype=np.float32)[:n]
        kr = rng.standard_normal(size=(CACHE_CHUNK_ROWS, w.d_r), dtype=np.float32)[:n]
        yield start, K, V, kr
