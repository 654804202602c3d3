"""The native block allocator behind the multi-step history store (host only,
no GPU): reservations, block reuse after release, capacity errors that leave
the state unchanged, invariants under a random sequence of operations, and
the all-or-nothing batch append that a step's commit uses."""
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


def _batch(lib, pool, slots, counts):
    sl, ct = np.array(slots, np.int32), np.array(counts, np.int32)
    starts = np.full(len(slots), -7, np.int32)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    return lib.flide_pool_append_batch(pool, len(slots), p(sl), p(ct), p(starts)), starts


def test_batch_append_all_or_nothing(lib):
    pool = lib.flide_pool_create(6, 4, 4, 4)
    try:
        st, starts = _batch(lib, pool, [0, 1, -1, 0], [5, 3, 9, 2])
        assert st == flide.OK and starts.tolist() == [0, 0, -1, 5]   # slot 0 twice, in order
        before = _export(lib, pool, 4, 4)
        assert before[1].tolist() == [7, 3, 0, 0] and lib.flide_pool_free_blocks(pool) == 3
        for slots, counts, code in [
            ([2, 3], [8, 8], flide.ERR_CAPACITY),        # 4 blocks wanted, 3 free
            ([1, 1], [10, 5], flide.ERR_CAPACITY),       # 18 rows = 5 blocks > a table's 4
            ([2, 4], [1, 1], flide.ERR_INVALID),         # slot >= max_requests
            ([2, 3], [1, -1], flide.ERR_INVALID),        # negative count
        ]:
            st, starts = _batch(lib, pool, slots, counts)
            assert st == code
            assert (starts == -7).all()                  # nothing written on error
            after = _export(lib, pool, 4, 4)
            assert np.array_equal(after[0], before[0]) and np.array_equal(after[1], before[1])
            assert lib.flide_pool_free_blocks(pool) == 3
        assert lib.flide_pool_append_batch(pool, 2, None, None, None) == flide.ERR_SHAPE
        assert lib.flide_pool_append_batch(pool, 0, None, None, None) == flide.OK
        st, starts = _batch(lib, pool, [2, 3, 2], [4, 4, 4])          # exactly the 3 free blocks
        assert st == flide.OK and starts.tolist() == [0, 0, 4] and lib.flide_pool_free_blocks(pool) == 0
    finally:
        lib.flide_pool_destroy(pool)


def test_random_batches_match_sequential_appends(lib):
    """A batch that succeeds equals its appends made one by one; a batch that
    fails is exactly one whose one-by-one appends would fail somewhere, and it
    leaves the pool as it was."""
    rng = np.random.default_rng(1)
    n_blocks, rows, R, mb = 30, 8, 5, 10
    pool = lib.flide_pool_create(n_blocks, rows, R, mb)
    length, nblk = np.zeros(R, int), np.zeros(R, int)
    try:
        for _ in range(300):
            if rng.random() < 0.15:
                s = int(rng.integers(0, R))
                assert lib.flide_pool_release(pool, s) == flide.OK
                length[s], nblk[s] = 0, 0
                continue
            k = int(rng.integers(0, 5))
            slots = rng.integers(-1, R, k).tolist()
            counts = rng.integers(0, 30, k).tolist()
            # the model: the appends one by one
            ln, nb, free, ok, want = length.copy(), nblk.copy(), n_blocks - int(nblk.sum()), True, []
            for s, c in zip(slots, counts):
                if s < 0:
                    want.append(-1)
                    continue
                need = -(-(ln[s] + c) // rows)
                if need > mb or need - nb[s] > free:
                    ok = False
                    break
                want.append(int(ln[s]))
                free -= need - nb[s]
                ln[s], nb[s] = ln[s] + c, need
            before = _export(lib, pool, R, mb)
            st, starts = _batch(lib, pool, slots, counts)
            if ok:
                assert st == flide.OK and starts.tolist() == want
                length, nblk = ln, nb
            else:
                assert st == flide.ERR_CAPACITY
                after = _export(lib, pool, R, mb)
                assert np.array_equal(after[0], before[0]) and np.array_equal(after[1], before[1])
            table, lens = _export(lib, pool, R, mb)
            assert lens.tolist() == length.tolist()
            assert int(np.sum(table >= 0)) + lib.flide_pool_free_blocks(pool) == n_blocks
    finally:
        lib.flide_pool_destroy(pool)


def test_store_reserve_is_all_or_nothing():
    """HistoryStore.reserve (the host half of commit) on CPU buffers: root
    rows per request, -1 for requests that keep nothing, zero rows for an
    empty request, and a batch that does not fit changes no slot."""
    from tree_forked_decision_b200 import inputs
    from tree_forked_decision_b200.history import HistoryStore
    store = HistoryStore(n_blocks=5, block_rows=16, max_requests=4, max_blocks=3, Hkv=1, d=8,
                         device="cpu")
    tree = inputs._tree([(0, [(-1, 20), (0, 3)]), (0, []), (0, [(-1, 7)]), (0, [(-1, 5), (0, 1)])], 1)
    start = store.reserve([2, 0, -1, 3], tree)
    assert start.tolist() == [0, 0, -1, 0]
    assert store.len_h.tolist() == [0, 0, 20, 5] and store.lengths.tolist() == [0, 0, 20, 5]
    assert store.free_blocks() == 2                     # 2 blocks for slot 2, 1 for slot 3
    assert store.table.tolist() == store.table_h.tolist()
    start = store.reserve([-1, -1, 3, -1], tree)         # slot 3 continues: 7 more rows
    assert start.tolist() == [-1, -1, 5, -1] and store.len_h.tolist() == [0, 0, 20, 12]
    with pytest.raises(flide.FlideError) as e:          # 48 rows: 3 more blocks, 2 free
        store.reserve([1, 3, -1, -1], inputs._tree([(0, [(-1, 48)]), (0, [(-1, 1)]),
                                                     (0, [(-1, 1)]), (0, [(-1, 1)])], 0))
    assert e.value.code == flide.ERR_CAPACITY
    assert store.len_h.tolist() == [0, 0, 20, 12] and store.free_blocks() == 2
    with pytest.raises(ValueError):                      # one request per slot per step
        store.reserve([1, 1, -1, -1], tree)
    assert store.len_h.tolist() == [0, 0, 20, 12]
