"""Host logic of the host-buffer forward: the chunk schedule (no GPU needed)."""
import pytest

from token_choice_routing_b200.layer import chunk_bounds


@pytest.mark.parametrize("T,chunk", [(131072, 16384), (65536, 16384), (16384, 4096), (5000, 4096), (1, 16384),
                                     (7, 8), (200, 200), (28671, 16384), (28672, 16384), (28673, 16384),
                                     (100, 1), (3, 2), (999, 7)])
def test_chunks_cover_the_batch_in_order_within_the_capacity(T, chunk):
    b = chunk_bounds(T, chunk)
    assert b[0][0] == 0 and b[-1][1] == T
    assert all(a1 == b0 for (_, a1), (b0, _) in zip(b, b[1:]))
    assert all(1 <= hi - lo <= chunk for lo, hi in b)


def test_batch_starts_and_ends_with_short_chunks():
    sizes = [hi - lo for lo, hi in chunk_bounds(131072, 16384)]
    assert sizes[:3] == [2048, 4096, 8192] and sizes[-3:] == [8192, 4096, 2048]
    mid = sizes[3:-3]
    assert max(mid) <= 16384 and max(mid) - min(mid) <= 1 and sum(sizes) == 131072


def test_short_batch_is_split_into_pieces_of_an_eighth():
    sizes = [hi - lo for lo, hi in chunk_bounds(16384, 16384)]
    assert len(sizes) == 8 and set(sizes) == {2048}


def test_empty_batch_has_no_chunks():
    assert chunk_bounds(0, 4096) == []
