"""Host logic of paged caches (CPU): the page allocator behind PagedLayer."""
import numpy as np
import pytest

from bit_kv_cache_19_b200.runtime import PageAllocator


def test_reserve_release_and_orders():
    a = PageAllocator(n_pages=10, page_tiles=1, batch=2, max_pages=6)
    a.reserve(0, 64, order=[5, 3, 9])           # 2 pages of 32 tokens, caller's order
    a.reserve(1, 96)                            # 3 pages from the free list
    assert a.table[0].tolist() == [5, 3, -1, -1, -1, -1]
    assert a.table[1].tolist() == [0, 1, 2, -1, -1, -1]
    a.reserve(1, 96)                            # already held: nothing changes
    assert a.n_held == [2, 3]
    a.release(0)
    assert a.table[0].tolist() == [-1] * 6 and a.n_held[0] == 0
    a.reserve(1, 160)                           # grows: 3 and 4 are free (5 went back too)
    assert a.table[1].tolist() == [0, 1, 2, 3, 4, -1]
    assert len(set(a.table[a.table >= 0].tolist())) == (a.table >= 0).sum()  # no page twice


def test_exhaustion_and_row_limit():
    a = PageAllocator(n_pages=4, page_tiles=2, batch=2, max_pages=3)
    a.reserve(0, 192)                           # 3 pages of 64 tokens
    with pytest.raises(ValueError):
        a.reserve(1, 193 + 64)                  # more than the row holds
    with pytest.raises(MemoryError):
        a.reserve(1, 128)                       # one page left
    a.release(0)
    a.reserve(1, 128)
    assert sorted(a.table[1][:2].tolist()) == sorted(set(a.table[1][:2].tolist()))


def test_order_skips_pages_in_use():
    a = PageAllocator(n_pages=6, page_tiles=1, batch=2, max_pages=4)
    a.reserve(0, 64, order=[2, 4])
    with pytest.raises(MemoryError):            # 4 and 2 are in use: 1, 0, then the list ends
        a.reserve(1, 96, order=[4, 2, 1, 0])
    assert a.table[1].tolist() == [1, 0, -1, -1] and a.n_held[1] == 2
    a.reserve(1, 96, order=[3])                 # the third page from a fresh order
    assert a.table[1].tolist() == [1, 0, 3, -1]
