"""Absorbed Multi-head Latent Attention decode for B200 (sm_100a).

The compute lives in libmla.so (hand-written CUDA kernels behind a C ABI, include/mla.h); this
package is its Python binding. Importing it does not load the library; the first call does, and
fails loudly if the library has not been built.
"""
from .ops import (  # noqa: F401
    Dims, GqaCache, LatentCache, MlaError, mla_absorb_q, mla_append_cache, mla_build_info,
    mla_check_status, mla_decode_absorbed, mla_launch_count, mla_decode_gqla_grouped, mla_decode_workspace_size,
    mla_out_proj, mla_project_query, mla_status_string,
)
