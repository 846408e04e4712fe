"""Pins for the oracle's paged compressed cache (admirer.cn article, cache
paragraph; "DeepSeek-V4 内部机制" section 7): gathering through a block table
inverts scattering the contiguous cache into randomly chosen pool pages, the
identity table is a reshape, and a table slot outside the pool is refused."""
import numpy as np
import pytest

import oracle as orc

PER_PAGE = 32  # 128-token pages hold 32 CSA entries (m = 4)


@pytest.fixture(scope="module", autouse=True)
def _built():
    orc.build()


def test_gather_inverts_a_random_scatter():
    rng = np.random.default_rng(0)
    B, E, rb = 3, 100, 608  # ragged last page
    cache = rng.integers(0, 256, size=(B, E, rb), dtype=np.uint8)
    pages_per_req = -(-E // PER_PAGE)
    n_pages = B * pages_per_req + 5
    perm = rng.permutation(n_pages)[:B * pages_per_req].reshape(B, pages_per_req).astype(np.int32)
    pool = rng.integers(0, 256, size=(n_pages, PER_PAGE, rb), dtype=np.uint8)
    for b in range(B):
        for i in range(E):
            pool[perm[b, i // PER_PAGE], i % PER_PAGE] = cache[b, i]
    np.testing.assert_array_equal(orc.gather_paged(pool, perm, E), cache)


def test_identity_table_is_a_reshape():
    rng = np.random.default_rng(1)
    B, pages, rb = 2, 4, 16
    pool = rng.integers(0, 256, size=(B * pages, PER_PAGE, rb), dtype=np.uint8)
    table = np.arange(B * pages, dtype=np.int32).reshape(B, pages)
    np.testing.assert_array_equal(orc.gather_paged(pool, table, pages * PER_PAGE),
                                  pool.reshape(B, pages * PER_PAGE, rb))


def test_out_of_pool_page_is_refused():
    pool = np.zeros((2, PER_PAGE, 16), np.uint8)
    with pytest.raises(ValueError):
        orc.gather_paged(pool, np.array([[0, 2]], np.int32), 40)
    with pytest.raises(ValueError):
        orc.gather_paged(pool, np.array([[0, 1]], np.int32), 65)  # more entries than the table maps
