"""Host-side arithmetic of the quantizer launch: the division-free tile
decode.  The launcher gives the kernel tc_magic = ceil(2^(31+l) / d) and
tc_shift = l - 1, l = ceil(log2 d), for d = tiles per row of tiles > 1, and
the kernel takes the row tile of tile t as umulhi(t, tc_magic) >> tc_shift.
This must equal t // d for every t < 2^31 (the tile-count limit) and every d
the quantizer can see (cols / 128 < 2^24)."""
import random

import pytest


def _magic(d):
    l = 0
    while (1 << l) < d:
        l += 1
    return ((1 << (31 + l)) + d - 1) // d, l - 1


def _row(t, d, m, sh):
    return t if d == 1 else ((t * m) >> 32) >> sh


@pytest.mark.parametrize("d", list(range(1, 300)) + [383, 384, 385, 1023, 1024, 1025, 4095, 4097,
                                                     65535, 65536, 65537, (1 << 24) - 1])
def test_tile_row_identity(d):
    m, sh = (0, 0) if d == 1 else _magic(d)
    assert 0 <= m < (1 << 32)
    rng = random.Random(d)
    ts = {0, 1, (1 << 31) - 1, (1 << 31) - 2}
    for k in [rng.randrange(0, ((1 << 31) - 1) // d + 1) for _ in range(200)] + [0, 1, 2]:
        for o in (-1, 0, 1, d - 1):
            ts.add(k * d + o)
    for t in ts:
        if 0 <= t < (1 << 31):
            assert _row(t, d, m, sh) == t // d, (t, d)


@pytest.mark.parametrize("d", [2, 3, 5, 7, 8, 16, 24, 48, 96])
def test_tile_row_exhaustive_small(d):
    """Every tile index of the shapes the quantizer runs here (and more)."""
    m, sh = _magic(d)
    for t in range(1 << 18):
        assert ((t * m) >> 32) >> sh == t // d
