"""The bench's algorithmic counts (the roofline numerator) against the figures worked out by hand
for the configurations it reports, and its traffic records against the sources they were taken on.
No GPU."""
import numpy as np

import bench
import synth


def test_absorbed_decode_bytes_and_flops_at_the_bench_shape():
    # 64 sequences x 4096 positions, H = 128, d_c = 512, d_r = 64, bf16:
    # cache rows 262,144 x 1152 B = 301,989,888 B; q_abs 64 x 128 x 576 x 2 = 9,437,184 B;
    # o_lat 64 x 128 x 512 x 2 = 8,388,608 B; lse 64 x 128 x 4 = 32,768 B
    w = synth.workload("dsv3_b64_l4096")
    lens = np.full(w.B, 4096)
    bytes_, flops, positions = bench.decode_counts(w, lens)
    assert positions == 262_144
    assert bytes_ == 301_989_888 + 9_437_184 + 8_388_608 + 32_768 == 319_848_448
    # 2 H (2 d_c + d_r) = 278,528 FLOPs per position and head set: 73.0 GFLOP per launch
    assert flops == 278_528 * 262_144 == 73_014_444_032
    assert abs(flops / (positions * 1152) - 241.78) < 0.01   # FLOPs per cache byte


def test_eight_bit_rows_count_one_byte_per_value_and_a_scale():
    w = synth.workload("dsv3_fp8_b64_l4096")
    bytes_, flops, positions = bench.decode_counts(w, np.full(w.B, 4096))
    # 512 code bytes + 4 scale bytes + 128 RoPE bytes per position
    assert bytes_ == 262_144 * 644 + 9_437_184 + 8_388_608 + 32_768 == 186_679_296
    assert flops == 73_014_444_032


def test_multi_token_flops_skip_the_causal_triangle():
    # with s_q new tokens, token t sees L - s_q + 1 + t positions: s_q L - s_q (s_q - 1) / 2 per sequence
    w = synth.workload("mtp_sq2_b128", B=2, lengths=("list", (1024, 33)))
    lens = np.array([1024, 33])
    _, flops, positions = bench.decode_counts(w, lens)
    assert positions == 1057
    assert flops == 278_528 * ((2 * 1024 - 1) + (2 * 33 - 1))


def _sources_hash(names):
    import hashlib
    import os
    csrc = os.path.join(os.path.dirname(os.path.abspath(bench.__file__)), "mla_compressed_latent_b200", "csrc")
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def test_traffic_is_reported_only_for_the_sources_it_was_captured_on():
    """A recorded DRAM traffic figure is reported exactly while the kernel's sources hash to the
    version it was captured on (else null), and only for its own workload."""
    for wl, rec, srcs in (("dsv3_b64_l4096", bench.DECODE_TRAFFIC, bench.DECODE_SOURCES),
                          ("gqla_g8_b32_l8192", bench.GQLA_TRAFFIC, bench.GQLA_SOURCES)):
        want = rec["bytes"] if _sources_hash(srcs) == rec["sources_sha256_16"] else None
        assert bench.captured_traffic(wl, rec, srcs) == want
        assert bench.captured_traffic("longctx_b8", rec, srcs) is None
