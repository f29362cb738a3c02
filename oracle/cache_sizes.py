"""Closed-form cache and parameter counts for the memory side of latent attention.

TEST INFRASTRUCTURE (part of the oracle package; see its header).

Sources:
  « L'attention latente : compresser le cache » — « Le problème : le cache grossit avec le texte »,
      « L'idée : garder un résumé », « L'obstacle : RoPE », « Les résultats ».
  « Le cache clé-valeur » — « Combien cela pèse »: 2 · L · h_kv · d_h · b bytes per token.
  « Cache KV, mémoire récurrente, MLA et bas rang » — « Le problème — Cache KV standard »,
      « L'idée — MLA », « L'idée — État récurrent fixe », « Factorisation bas rang »,
      « Cas guidé — trace complète ».
  « Résumé technique : GQLA … » — « 4. Résultats » (cache compression against GQA).
"""
from __future__ import annotations

KiB, MiB, GiB = 2 ** 10, 2 ** 20, 2 ** 30


def mha_numbers_per_position(C: int) -> int:
    """Keys and values of every head of one layer: 2·C numbers per position."""
    return 2 * C


def mla_numbers_per_position(d_c: int, d_r: int = 0) -> int:
    """Latent plus the shared RoPE key: d_c + d_r numbers per position and layer."""
    return d_c + d_r


def kv_cache_bytes(tokens: int, layers: int, kv_heads: int, d_head: int, bytes_per_value: int) -> int:
    """Standard cache: tokens × layers × 2 (K and V) × heads × d_head × bytes."""
    return tokens * layers * 2 * kv_heads * d_head * bytes_per_value


def kv_bytes_per_token(layers: int, kv_heads: int, d_head: int, bytes_per_value: int) -> int:
    return kv_cache_bytes(1, layers, kv_heads, d_head, bytes_per_value)


def latent_cache_bytes(tokens: int, layers: int, d_c: int, bytes_per_value: int, d_r: int = 0) -> int:
    """Latent cache: one (d_c [+ d_r]) row per token and layer; linear in tokens."""
    return tokens * layers * (d_c + d_r) * bytes_per_value


def model_cache_bytes(numbers_per_position: int, layers: int, tokens: int, bytes_per_value: int) -> int:
    return numbers_per_position * layers * tokens * bytes_per_value


def recurrent_state_bytes(layers: int, d_k: int, d_v: int, bytes_per_value: int) -> int:
    """Fixed state: layers × d_k × d_v × bytes, independent of the token count."""
    return layers * d_k * d_v * bytes_per_value


def low_rank_params(d: int, m: int, r: int) -> int:
    """W (d×m) ≈ A (d×r) · B (r×m): r·(d + m) numbers."""
    return r * (d + m)


def low_rank_break_even(d: int, m: int) -> float:
    """Rank below which the factorisation saves parameters: r* = d·m / (d + m)."""
    return d * m / (d + m)


def gqla_cache_fraction(d_c: int, d_r: int, g: int, d_h: int) -> float:
    """Absorbed-path cache (latent + shared RoPE key) over a GQA cache of g heads: (d_c+d_r)/(2·g·d_h)."""
    return (d_c + d_r) / (2 * g * d_h)


def gqa_cache_numbers_per_position(g: int, d_h: int, d_r: int) -> int:
    """GQLA grouped path: expanded keys and values of g groups plus the shared RoPE key."""
    return 2 * g * d_h + d_r
