"""The native block allocator behind the multi-step history store (host only,
no GPU): reservations, block reuse after release, capacity errors that leave
the state unchanged, and invariants under a random sequence of operations."""
import ctypes

import numpy as np
import pytest

from tree_forked_decision_b200 import flide


@pytest.fixture()
def lib():
    return flide._lib()


def _export(lib, pool, max_requests, max_blocks):
    table = np.full(max_requests * max_blocks, -7, np.int32)
    lengths = np.full(max_requests, -7, np.int32)
    assert lib.flide_pool_export(pool, table.ctypes.data_as(ctypes.c_void_p),
                                 lengths.ctypes.data_as(ctypes.c_void_p)) == flide.OK
    return table.reshape(max_requests, max_blocks), lengths


def test_reserve_release_and_capacity(lib):
    pool = lib.flide_pool_create(6, 4, 3, 4)
    assert pool
    try:
        assert lib.flide_pool_append(pool, 0, 5) == 0          # rows 0..4 -> 2 blocks
        assert lib.flide_pool_append(pool, 0, 3) == 5          # rows 5..7 still fit
        assert lib.flide_pool_free_blocks(pool) == 4
        assert lib.flide_pool_append(pool, 0, 1) == 8          # third block
        assert lib.flide_pool_append(pool, 1, 10) == 0         # three blocks
        assert lib.flide_pool_free_blocks(pool) == 0
        assert lib.flide_pool_append(pool, 2, 1) == -flide.ERR_CAPACITY
        assert lib.flide_pool_length(pool, 2) == 0             # unchanged on error
        table, lengths = _export(lib, pool, 3, 4)
        assert lengths.tolist() == [9, 10, 0]
        assert sorted(table[0, :3].tolist() + table[1, :3].tolist()) == list(range(6))
        assert table[0, 3] == table[1, 3] == -1 and (table[2] == -1).all()
        assert lib.flide_pool_release(pool, 0) == flide.OK
        assert lib.flide_pool_free_blocks(pool) == 3
        assert lib.flide_pool_append(pool, 2, 1) == 0          # reuses a released block
        table, lengths = _export(lib, pool, 3, 4)
        assert lengths.tolist() == [0, 10, 1] and (table[0] == -1).all()
        assert table[2, 0] not in table[1].tolist()
        # a request's table holds at most max_blocks blocks
        assert lib.flide_pool_append(pool, 2, 16) == -flide.ERR_CAPACITY
        assert lib.flide_pool_append(pool, 3, 1) == -flide.ERR_INVALID
        assert lib.flide_pool_append(pool, -1, 1) == -flide.ERR_INVALID
    finally:
        lib.flide_pool_destroy(pool)


def test_create_rejects_bad_sizes(lib):
    assert not lib.flide_pool_create(4, 0, 2, 2)
    assert not lib.flide_pool_create(4, 8, 0, 2)
    assert not lib.flide_pool_create(-1, 8, 2, 2)


def test_random_operations_keep_invariants(lib):
    rng = np.random.default_rng(0)
    n_blocks, rows, R, mb = 40, 8, 6, 12
    pool = lib.flide_pool_create(n_blocks, rows, R, mb)
    length = np.zeros(R, int)
    try:
        for _ in range(400):
            s = int(rng.integers(0, R))
            if rng.random() < 0.2:
                assert lib.flide_pool_release(pool, s) == flide.OK
                length[s] = 0
            else:
                n = int(rng.integers(0, 20))
                got = lib.flide_pool_append(pool, s, n)
                if got >= 0:
                    assert got == length[s]
                    length[s] += n
                else:
                    assert got == -flide.ERR_CAPACITY
            table, lens = _export(lib, pool, R, mb)
            assert lens.tolist() == length.tolist()
            held = table[table >= 0]
            assert len(set(held.tolist())) == len(held)              # no block in two places
            assert len(held) + lib.flide_pool_free_blocks(pool) == n_blocks
            for r in range(R):
                nb = int(np.sum(table[r] >= 0))
                assert nb == -(-length[r] // rows)                   # exactly the blocks needed
                assert (table[r, :nb] >= 0).all() and (table[r, nb:] == -1).all()
    finally:
        lib.flide_pool_destroy(pool)
