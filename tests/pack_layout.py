"""The tiled LM-head weight layout, rebuilt with numpy from its definition in
include/fdl.h (fdl_lmhead_pack_weight): test infrastructure only."""
import numpy as np

SMS = 148  # the vocabulary is cut into one range per SM of a B200


def rows_per_range(V: int) -> int:
    """round16(ceil(V / 148)): the vocabulary rows of one CTA range."""
    per = -(-V // SMS)
    return -(-per // 16) * 16


def tiles(V: int):
    """(first row r0, row count rt) of every tile, in order: each range cut
    into tiles of up to 128 rows."""
    per = rows_per_range(V)
    for lo in range(0, V, per):
        hi = min(V, lo + per)
        for r0 in range(lo, hi, 128):
            yield r0, min(128, hi - r0)


def pack_reference(w, V: int, H: int):
    """w [V, H] -> the tiled layout, as [V, H] of the same dtype: tile (r0,
    rt) holds, for each 64-wide column chunk kk in turn, its rt rows' 64
    values of that chunk, from 128-byte row r0 * H / 64 on."""
    KCT = H // 64
    pieces = np.asarray(w).reshape(V, KCT, 64)
    out = np.empty((V * KCT, 64), dtype=pieces.dtype)
    for r0, rt in tiles(V):
        out[r0 * KCT:(r0 + rt) * KCT] = pieces[r0:r0 + rt].transpose(1, 0, 2).reshape(KCT * rt, 64)
    return out.reshape(V, H)
