"""The token sampler of the full-size parity checks: the tile split it
mirrors covers every row exactly once, and the sample holds the hottest
expert's last row tile, the rarest non-empty expert's tokens and at least
the requested number of tokens."""
import numpy as np

from _helpers import grouped_tile_heights, parity_sample, row_tiles


def test_row_tiles_cover_rows_once():
    for bn in (16, 64, 112, 128, 256):
        for n in list(range(0, 300)) + [5700, 8191]:
            tiles = row_tiles(n, bn)
            rows = [r for r0, k in tiles for r in range(r0, r0 + k)]
            assert rows == list(range(n))
            assert all(0 < k <= bn for _, k in tiles)
            assert all(k % 16 == 0 for _, k in tiles[:-1])
            if n:
                assert len(tiles) == -(-n // bn)


def test_parity_sample_contents():
    rng = np.random.default_rng(1)
    T, K, E = 3000, 8, 64
    p = np.arange(1, E + 1, dtype=float) ** -1.1
    idx = np.stack([rng.choice(E, K, replace=False, p=p / p.sum()) for _ in range(T)])
    idx[5, 2] = -1
    toks = parity_sample(idx, E, [64, 112], n_min=16)
    counts = np.bincount(idx[idx >= 0], minlength=E)
    hot = counts.argmax()
    slots = np.nonzero(idx.reshape(-1) == hot)[0]
    for bn in (64, 112):
        r0, n = row_tiles(len(slots), bn)[-1]
        assert {s // K for s in slots[r0:r0 + n]} <= set(toks)
    nz = np.nonzero(counts)[0]
    rare = nz[np.argmin(counts[nz])]
    assert set(np.nonzero((idx == rare).any(axis=1))[0]) <= set(toks)
    assert len(toks) >= 16 and toks == sorted(set(toks)) and toks[0] == 0 and toks[-1] == T - 1
    # small T: every token
    assert parity_sample(idx[:5], E, [16], n_min=16) == [0, 1, 2, 3, 4]


def test_grouped_tile_heights():
    assert grouped_tile_heights(2048, 6, 64, "bf16") == [128, 256]
    assert grouped_tile_heights(8, 8, 256, "e4m3") == [16]
    assert grouped_tile_heights(128, 8, 256, "e4m3") == [16]
    assert grouped_tile_heights(512, 8, 256, "e4m3") == [64]
    assert grouped_tile_heights(2048, 8, 256, "mxfp4") == [112]
    assert grouped_tile_heights(512, 8, 256, "mxfp4") == [64]
