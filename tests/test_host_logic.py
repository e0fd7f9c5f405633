"""Host-side logic of the package that needs no GPU."""
import pytest

from combine_router_softmax_02_b200.path import token_ranges


@pytest.mark.parametrize("T,chunks", [(0, 8), (1, 8), (7, 8), (8, 8), (9, 8), (65536, 8), (1000, 3),
                                      (5, 1), (100, 1000)])
def test_token_ranges_cover_in_order(T, chunks):
    r = token_ranges(T, chunks)
    assert all(b > a for a, b in r)                      # non-empty
    flat = [t for a, b in r for t in range(a, b)]
    assert flat == list(range(T))                        # contiguous, in order, no overlap
    assert len(r) == (min(chunks, T) if T else 0)
    if r:
        sizes = [b - a for a, b in r]
        assert max(sizes) - min(sizes) <= 1
