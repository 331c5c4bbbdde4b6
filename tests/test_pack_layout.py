"""Host checks of the tiled LM-head weight layout's definition: a
permutation of the weight's 128-byte pieces in which every box the LM head
loads (up to 128 rows of one 64-wide column chunk of one tile) is one
contiguous run."""
import numpy as np
import pytest

from tests.pack_layout import pack_reference, rows_per_range, tiles


@pytest.mark.parametrize("V,H", [(5000, 448), (7001, 64), (1, 128), (17, 192), (151936, 128)])
def test_layout_is_a_permutation_with_contiguous_boxes(V, H):
    KCT = H // 64
    ids = np.arange(V * KCT, dtype=np.int64)            # piece (v, kk) = v * KCT + kk
    src = np.repeat(ids[:, None], 64, axis=1).reshape(V, H)
    packed = pack_reference(src, V, H).reshape(V * KCT, 64)
    assert (packed == packed[:, :1]).all()                # whole 128-byte pieces move
    order = packed[:, 0]
    assert np.array_equal(np.sort(order), ids)            # a permutation
    for r0, rt in tiles(V):
        for kk in range(KCT):
            run = order[r0 * KCT + kk * rt: r0 * KCT + (kk + 1) * rt]
            assert np.array_equal(run, (r0 + np.arange(rt)) * KCT + kk)


def test_ranges_and_tiles_cover_the_vocabulary_once():
    for V in (1, 2, 148, 149, 5000, 152064):
        per = rows_per_range(V)
        assert per % 16 == 0 and -(-V // per) <= 148
        rows = [r for r0, rt in tiles(V) for r in range(r0, r0 + rt)]
        assert rows == list(range(V))
        assert all(rt <= 128 for _, rt in tiles(V))
