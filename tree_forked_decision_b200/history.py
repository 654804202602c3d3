"""Multi-step agent history in a block-paged checkpoint pool.

An agent takes decision after decision on a growing history: each step's root
(the new observation) is appended to what came before, and the next step
resumes from it, so the shared prefix is computed once over the whole episode
(kongchang.com article on Flide, closing section: growing agent histories and
checkpoint reuse; techfi24.com, "Exact State Forking").

``HistoryStore`` owns the device pool -- K/V history rows in blocks of
``block_rows`` rows and one fp32 GDN state per request slot -- and the native
block allocator (``flide_pool_*`` in libflide.so).  Per step:

    past_len, past_k, past_v, state_in = store.resume(slots)       # before
    ... flide_tree_build / fork_attn / fork_gdn on the step's tree ...
    store.commit(slots, index, k, v, node_state)                    # after

``resume`` packs each slot's history as the batch's past rows and GDN
state_in; ``commit`` reserves blocks for each request's root tokens on the
host, copies the block table to the device, and appends the root rows and the
root's end state.  ``release(slot)`` returns a finished request's blocks.

Without the packed copy (block_rows a multiple of 128):

    past_len, state_in = store.resume_lengths(slots)
    ... flide_tree_build ...
    o = store.fork_attn_paged(q, k, v, index, scale, slots)   # past read in place
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import flide


class HistoryStore:
    def __init__(self, n_blocks: int, block_rows: int, max_requests: int, max_blocks: int,
                 Hkv: int, d: int, H: int = 0, dk: int = 0, dv: int = 0,
                 dtype=torch.bfloat16, device="cuda"):
        lib = flide._lib()
        self._lib = lib
        self._pool = lib.flide_pool_create(n_blocks, block_rows, max_requests, max_blocks)
        if not self._pool:
            raise flide.FlideError(flide.ERR_SHAPE, "flide_pool_create")
        self.n_blocks, self.block_rows = n_blocks, block_rows
        self.max_requests, self.max_blocks = max_requests, max_blocks
        self.Hkv, self.d, self.H, self.dk, self.dv = Hkv, d, H, dk, dv
        self.dtype, self.device = dtype, device
        self.pool_k = torch.zeros((n_blocks * block_rows, Hkv, d), dtype=dtype, device=device)
        self.pool_v = torch.zeros_like(self.pool_k)
        self.pool_S = (torch.zeros((max_requests, H, dv, dk), dtype=torch.float32, device=device)
                       if H else None)
        self.table_h = np.full(max_requests * max_blocks, -1, np.int32)
        self.len_h = np.zeros(max_requests, np.int32)
        self.table = torch.full((max_requests * max_blocks,), -1, dtype=torch.int32, device=device)
        self.lengths = torch.zeros(max_requests, dtype=torch.int32, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def __del__(self):
        pool = getattr(self, "_pool", None)
        if pool:
            self._lib.flide_pool_destroy(pool)
            self._pool = None

    # -- host bookkeeping ---------------------------------------------------
    def length(self, slot: int) -> int:
        return int(self._lib.flide_pool_length(self._pool, slot))

    def free_blocks(self) -> int:
        return int(self._lib.flide_pool_free_blocks(self._pool))

    def release(self, slot: int):
        flide._check(self._lib.flide_pool_release(self._pool, slot), "flide_pool_release")
        self._sync_table()

    def _sync_table(self):
        flide._check(self._lib.flide_pool_export(self._pool, self.table_h.ctypes.data_as(ctypes.c_void_p),
                                                 self.len_h.ctypes.data_as(ctypes.c_void_p)),
                     "flide_pool_export")
        self.table.copy_(torch.from_numpy(self.table_h))
        self.lengths.copy_(torch.from_numpy(self.len_h))

    # -- device steps -------------------------------------------------------
    def resume(self, slots, past_rows: int | None = None):
        """Past rows, lengths and GDN state_in for a batch whose request r
        continues slot slots[r] (-1: no history)."""
        slots = [int(s) for s in slots]
        R = len(slots)
        rows = sum(int(self.len_h[s]) for s in slots if s >= 0)
        past_rows = max(rows, 1) if past_rows is None else past_rows
        req = torch.tensor(slots, dtype=torch.int32, device=self.device)
        past_len = torch.zeros(R, dtype=torch.int32, device=self.device)
        pk = torch.empty((past_rows, self.Hkv, self.d), dtype=self.dtype, device=self.device)
        pv = torch.empty_like(pk)
        state_in = (torch.empty((R, self.H, self.dv, self.dk), dtype=torch.float32, device=self.device)
                    if self.H else None)
        self.status.zero_()
        flide._check(self._lib.flide_history_gather(
            R, flide._ptr(req), self.max_requests, flide._ptr(self.lengths), flide._ptr(self.table),
            self.max_blocks, self.block_rows, flide._ptr(self.pool_k), flide._ptr(self.pool_v),
            self.Hkv, self.d, flide._dtype_code(self.pool_k), flide._ptr(self.pool_S), self.H,
            self.dk, self.dv, flide._ptr(past_len), flide._ptr(pk), flide._ptr(pv), past_rows,
            flide._ptr(state_in), flide._ptr(self.status), flide._stream()), "flide_history_gather")
        return past_len, pk, pv, state_in

    def resume_lengths(self, slots):
        """past_len and GDN state_in for a batch whose request r continues
        slot slots[r] (-1: no history), without packing the rows: for
        fork_attn_paged, which reads them in place."""
        slots = [int(s) for s in slots]
        R = len(slots)
        req = torch.tensor(slots, dtype=torch.int32, device=self.device)
        past_len = torch.zeros(R, dtype=torch.int32, device=self.device)
        state_in = (torch.empty((R, self.H, self.dv, self.dk), dtype=torch.float32, device=self.device)
                    if self.H else None)
        self.status.zero_()
        flide._check(self._lib.flide_history_gather(
            R, flide._ptr(req), self.max_requests, flide._ptr(self.lengths), flide._ptr(self.table),
            self.max_blocks, self.block_rows, flide._ptr(self.pool_k), flide._ptr(self.pool_v),
            self.Hkv, self.d, flide._dtype_code(self.pool_k), flide._ptr(self.pool_S), self.H,
            self.dk, self.dv, flide._ptr(past_len), None, None, 0, flide._ptr(state_in),
            flide._ptr(self.status), flide._stream()), "flide_history_gather")
        return past_len, state_in

    def fork_attn_paged(self, q, k, v, index: flide.TreeIndex, scale: float, slots, out=None):
        """Fork attention of a batch whose request r continues slot slots[r],
        the past rows read in place from this pool's blocks."""
        req = torch.tensor([int(s) for s in slots], dtype=torch.int32, device=self.device)
        return flide.fork_attn_paged(q, k, v, index, scale, self.pool_k, self.pool_v, self.table,
                                     req, self.block_rows, self.max_blocks, out=out)

    def reserve(self, slots, tree):
        """Host half of commit: reserves each request's root rows in its slot
        (all requests or none: on FlideError no slot changes), refreshes the
        device block table and lengths, and returns the start rows (-1 where
        slots[r] is -1).  Each slot at most once per step (ValueError)."""
        slots = [int(s) for s in slots]
        kept = [s for s in slots if s >= 0]
        if len(set(kept)) != len(kept):
            raise ValueError("a slot may be continued by one request per step "
                             "(two end states would race for it)")
        rp, _parent, seg, _past = tree.arrays()
        counts = np.array([int(seg[rp[r]]) if rp[r + 1] > rp[r] else 0 for r in range(len(slots))],
                          np.int32)
        sl = np.array(slots, np.int32)
        start = np.zeros(len(slots), np.int32)
        p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
        flide._check(self._lib.flide_pool_append_batch(self._pool, len(slots), p(sl), p(counts),
                                                       p(start)), "flide_pool_append_batch")
        self._sync_table()
        return start

    def commit(self, slots, tree, index: flide.TreeIndex, k, v, node_state=None):
        """Appends request r's root tokens (this step's observation) and its
        root's end GDN state to slot slots[r] (-1: nothing kept)."""
        slots = [int(s) for s in slots]
        start = self.reserve(slots, tree)
        req = torch.tensor(slots, dtype=torch.int32, device=self.device)
        st_d = torch.from_numpy(start).to(self.device)
        flide._check(self._lib.flide_history_append(
            ctypes.byref(index.c), flide._ptr(req), flide._ptr(st_d), flide._ptr(self.table),
            self.max_blocks, self.block_rows, flide._ptr(k), flide._ptr(v), flide._ptr(self.pool_k),
            flide._ptr(self.pool_v), self.Hkv, self.d, flide._dtype_code(k),
            flide._ptr(node_state if self.H else None), self.H, self.dk, self.dv,
            flide._ptr(self.pool_S), flide._stream()), "flide_history_append")
