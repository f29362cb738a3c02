"""The seeded input generators (synth/), the one module both the oracle and the CUDA path read:
deterministic, shaped as documented, page tables that partition the pool, and cached rows whose
values do not depend on how many rows a caller asks for."""
import math

import numpy as np
import pytest

import synth


def test_lengths_fixed_uniform_list_and_deterministic():
    w = synth.workload("dsv3_b64_l4096")
    assert (synth.seq_lengths(w) == 4096).all()
    w = synth.workload("longctx_b8")
    a, b = synth.seq_lengths(w), synth.seq_lengths(w)
    assert np.array_equal(a, b)
    assert a.min() >= 16384 and a.max() <= 131072
    w = synth.workload("dsv3_b64_l4096", B=3, lengths=("list", (5, 64, 65)))
    assert synth.seq_lengths(w).tolist() == [5, 64, 65]


@pytest.mark.parametrize("pages", ["contiguous", "random"])
def test_page_table_partitions_the_pool(pages):
    lens = (1, 63, 64, 65, 129, 1000, 7)
    w = synth.workload("dsv3_b64_l4096", B=len(lens), lengths=("list", lens), pages=pages)
    L = synth.seq_lengths(w)
    table, num_pages = synth.block_table(w, L)
    npages = [(n + 63) // 64 for n in lens]
    assert table.shape == (len(lens), max(npages)) and table.dtype == np.int32
    used = np.concatenate([table[b, :n] for b, n in enumerate(npages)])
    assert num_pages == sum(npages)
    assert sorted(used.tolist()) == list(range(num_pages))      # every pool page exactly once
    for b, n in enumerate(npages):
        assert (table[b, n:] == 0).all()                         # unused entries: a valid page
    if pages == "contiguous":
        assert used.tolist() == list(range(num_pages))
    table2, _ = synth.block_table(w, L)
    assert np.array_equal(table, table2)


def test_cache_rows_do_not_depend_on_the_request_size():
    w = synth.workload("smallem_fp32")
    n = synth.CACHE_CHUNK_ROWS + 100
    small = list(synth.cache_row_chunks(w, 50))
    big = list(synth.cache_row_chunks(w, n))
    assert small[0][0] == 0 and big[0][0] == 0 and big[1][0] == synth.CACHE_CHUNK_ROWS
    np.testing.assert_array_equal(small[0][1], big[0][1][:50])
    np.testing.assert_array_equal(small[0][2], big[0][2][:50])
    assert sum(len(c) for _, c, _ in big) == n
    # latent rows lie on the sphere of radius sqrt(d_c) (the law of an RMS-normalised row)
    norms = np.linalg.norm(big[1][1].astype(np.float64), axis=1)
    np.testing.assert_allclose(norms, math.sqrt(w.d_c), rtol=1e-5)


def test_weights_and_step_inputs_shapes_and_seeds():
    w = synth.workload("smallem_fp32")
    W = synth.weights(w)
    assert W["W_UK"].shape == (w.H, w.D, w.d_c) and W["W_UV"].shape == (w.H, w.d_c, w.d_v)
    assert W["W_DQ"].shape == (w.C, w.d_q) and W["W_UQ"].shape == (w.d_q, w.H * w.D)
    assert W["W_QR"].shape == (w.d_q, w.H * w.d_r) and W["W_O"].shape == (w.H * w.d_v, w.C)
    for k, v in synth.weights(w).items():
        assert np.array_equal(v, W[k]), k
    # the query weights are drawn after the others: a workload with a query latent keeps the same
    # cache-side weights as the one without
    w0 = synth.workload("smallem_fp32", d_q=0)
    W0 = synth.weights(w0)
    for k in ("W_DKV", "W_KR", "W_UK", "W_UV", "W_O"):
        assert np.array_equal(W0[k], W[k]), k
    s = synth.decode_step_inputs(w)
    assert s["x"].shape == (w.B, w.s_q, w.C)
    assert s["q_abs"].shape == (w.B, w.s_q, w.H, w.d_c + w.d_r)
    assert s["q_rope_raw"].shape == (w.B, w.s_q, w.H, w.d_r)
