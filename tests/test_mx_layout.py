"""The test-side readings of the MX layouts include/moe.h documents (used to
compare the GPU's buffers with the oracle): the chunked scale layout is a
bijection onto its buffer, and the FC1 row order of MX W1 follows the
header's formula."""
import numpy as np

from .gpu_helpers import mx_chunk, mx_scale_index, mx_unchunk, w1_tile_rows


def test_scale_layout_is_a_bijection_onto_its_bytes():
    for rows, K in ((128, 128), (256, 512), (384, 384), (1024, 2048)):
        idx = mx_scale_index(rows, K)
        nbytes = -(-rows // 128) * (K // 128) * 512
        assert idx.min() == 0 and idx.max() == nbytes - 1
        assert len(np.unique(idx)) == idx.size == nbytes


def test_scale_layout_places_the_documented_bytes():
    rows, K = 256, 512
    idx = mx_scale_index(rows, K)
    # row r, 32-block b: chunk (r // 128) * (K // 128) + b // 4, byte 16 (r % 32) + 4 ((r % 128) // 32) + b % 4
    for r, b in ((0, 0), (31, 3), (32, 0), (127, 15), (128, 4), (200, 9)):
        chunk = (r // 128) * (K // 128) + b // 4
        assert idx[r, b] == chunk * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + b % 4


def test_chunk_and_unchunk_round_trip():
    rng = np.random.default_rng(0)
    rows, K = 384, 768
    logical = rng.integers(0, 255, size=(rows, K // 32), dtype=np.uint8)
    buf = mx_chunk(logical, K, -(-rows // 128) * (K // 128) * 512)
    assert np.array_equal(mx_unchunk(buf, rows, K), logical)


def test_w1_row_order_matches_the_header():
    E, F = 3, 384
    perm = w1_tile_rows(E, F)
    assert np.array_equal(np.sort(perm), np.arange(E * 2 * F))
    for e in range(E):
        for t in range(F // 64):
            for i in (0, 5, 63, 64, 100, 127):
                want = e * 2 * F + (64 * t + i if i < 64 else F + 64 * t + (i - 64))
                assert perm[e * 2 * F + 128 * t + i] == want
