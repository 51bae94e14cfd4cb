"""Head partition across ranks (frame_level_delta_b200/shard.py)."""
import pytest

from frame_level_delta_b200.shard import head_partition


@pytest.mark.parametrize("H,world,weights", [
    (24, 1, None), (24, 2, None), (24, 8, None), (7, 3, None), (8, 2, (5, 3)), (24, 8, (5, 3) * 4),
    (10, 3, (5, 3, 1)), (3, 3, (100, 1, 1)), (25, 4, (1, 2, 3, 4)),
])
def test_partition_covers_every_head_once_in_order(H, world, weights):
    parts = head_partition(H, world, weights)
    assert len(parts) == world
    h = 0
    for h0, n in parts:
        assert h0 == h and n >= 1
        h += n
    assert h == H


def test_even_split_differs_by_at_most_one_head():
    for H in range(8, 40):
        for world in (2, 3, 4, 8):
            ns = [n for _, n in head_partition(H, world)]
            assert max(ns) - min(ns) <= 1


def test_uneven_split_follows_the_weights():
    assert head_partition(8, 2, (5, 3)) == [(0, 5), (5, 3)]
    ns = [n for _, n in head_partition(48, 3, (1, 2, 3))]
    assert ns == [8, 16, 24]


def test_partition_rejects_impossible_splits():
    with pytest.raises(ValueError):
        head_partition(2, 3)
    with pytest.raises(ValueError):
        head_partition(8, 2, (1, 0))
