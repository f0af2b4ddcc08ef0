"""The stack's weight placement (CPU only): how many layers fit in device memory, and which."""
import pytest

from bit_compressed_decode_b200 import placement


def test_resident_count():
    gb = 1 << 30
    assert placement.resident_count(100 * gb, gb, 96) == 96          # all fit
    assert placement.resident_count(100 * gb, gb, 96, reserve_bytes=60 * gb) == 40
    assert placement.resident_count(10 * gb, 3 * gb, 48) == 3         # whole blobs only
    assert placement.resident_count(gb, 2 * gb, 48) == 0
    assert placement.resident_count(gb, gb, 8, reserve_bytes=2 * gb) == 0
    with pytest.raises(ValueError):
        placement.resident_count(gb, 0, 8)


@pytest.mark.parametrize("r,n", [(0, 5), (24, 48), (1, 48), (47, 48), (48, 48), (3, 7), (5, 16)])
def test_spread(r, n):
    flags = placement.spread(r, n)
    assert len(flags) == n and sum(flags) == r
    # evenly: between two resident layers there are either floor or ceil of (n - r) / r streamed ones
    if 0 < r < n:
        idx = [i for i, f in enumerate(flags) if f]
        gaps = [b - a - 1 for a, b in zip(idx, idx[1:])]
        assert max(gaps) - min(gaps) <= 1 if gaps else True


def test_spread_every_other_layer():
    assert placement.spread(24, 48) == [l % 2 == 1 for l in range(48)]
    with pytest.raises(ValueError):
        placement.spread(5, 4)
