"""fp64 CPU oracle for decode-time Multi-head Latent Attention over a compressed latent cache.

TEST INFRASTRUCTURE. Only the tests, the smoke check of the entry module and the CPU-baseline /
reference arm of the bench may import, call or run anything in this package. The product path
(the C-ABI library and its Python binding) never touches it, and this package imports nothing
from the product path: the two share no code, only the seeded inputs of ``synth``.
"""
from . import mla_oracle, cache_sizes, roofline, fp8_cache  # noqa: F401
