"""Memory-bounded, depth-first GDN fork scan.

Memory for cloned states is what limits how many options one call can hold
(techfi24.com, "Limites et perspectives": past a few dozen options it grows
linearly with them).  Fork = isolation lets a request's tree be cut below its
root: every level-1 subtree needs only the root's end state.  So

  1. the roots run alone (requests in chunks of at most ``max_slots``), and
     their end states are kept, one per request;
  2. ``flide_plan_state_groups`` (native, host) packs whole level-1 subtrees,
     in stream order, into groups whose batches need at most ``max_slots``
     node-state slots;
  3. each group runs as a batch of its own: per request a zero-token root
     resumed from the kept state, then the group's subtrees.

Token rows move between the full stream and a group's compact stream with
``flide_copy_rows``; every layer step runs in the library's kernels.  Peak
node-state memory is ``max_slots * H * dv * dk * 4`` bytes instead of one
slot per inner node of the whole batch.  ``BoundedGdn`` builds the schedule
of a tree shape once (plan, device index arrays, the node-state buffer) and
``run`` launches it; ``fork_gdn_bounded`` does both for one call.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import flide


def plan_state_groups(tree, max_slots: int):
    """Group id of every node (-1 for roots) and the number of groups."""
    rp, parent, _seg, _past = tree.arrays()
    N = int(rp[-1])
    node_group = np.zeros(max(N, 1), np.int32)
    n_groups = ctypes.c_int32(0)
    rp32 = np.ascontiguousarray(rp, np.int32)
    pa32 = np.ascontiguousarray(parent, np.int32)
    flide._check(flide._lib().flide_plan_state_groups(
        len(rp) - 1, rp32.ctypes.data_as(ctypes.c_void_p), pa32.ctypes.data_as(ctypes.c_void_p),
        int(max_slots), node_group.ctypes.data_as(ctypes.c_void_p), ctypes.byref(n_groups)),
        "flide_plan_state_groups")
    return node_group[:N], int(n_groups.value)


def _copy_rows(dst, src, dst_idx=None, src_idx=None, n=None):
    """dst row dst_idx[i] <- src row src_idx[i] (rows = first dimension)."""
    rows = n if n is not None else (len(src_idx) if src_idx is not None else dst_idx.numel())
    row_bytes = src[0].numel() * src.element_size()
    flide._check(flide._lib().flide_copy_rows(
        flide._ptr(dst), flide._ptr(src), flide._ptr(dst_idx), flide._ptr(src_idx), int(rows),
        int(row_bytes), flide._stream()), "flide_copy_rows")


class _Batch:
    """One sub-batch: its tree, and the full-stream rows of its tokens."""

    def __init__(self, reqs, rows, levels):
        rp = [0]
        parent, seg = [], []
        for nodes in reqs:
            for pa, sl in nodes:
                parent.append(pa)
                seg.append(sl)
            rp.append(rp[-1] + len(nodes))
        self.rp = np.asarray(rp, np.int32)
        self.parent = np.asarray(parent, np.int32)
        self.seg = np.asarray(seg, np.int32)
        self.past = np.zeros(len(reqs), np.int32)
        self.rows = np.asarray(rows, np.int32)
        self.levels = levels

    def arrays(self):
        return self.rp, self.parent, self.seg, self.past


def _batches(tree, max_slots):
    """The schedule's batches in launch order: ("roots", batch, request ids)
    for the root chunks, then ("group", batch, request ids) per group."""
    rp, parent, seg, _past = tree.arrays()
    R, N = len(rp) - 1, int(rp[-1])
    starts = np.concatenate([[0], np.cumsum(seg)]).astype(np.int64)
    node_group, n_groups = plan_state_groups(tree, max_slots)
    out = []
    with_nodes = [r for r in range(R) if rp[r + 1] > rp[r]]
    for c0 in range(0, len(with_nodes), max_slots):
        chunk = with_nodes[c0:c0 + max_slots]
        rows = np.concatenate([np.arange(starts[rp[r]], starts[rp[r] + 1]) for r in chunk])
        out.append(("roots", _Batch([[(-1, int(seg[rp[r]]))] for r in chunk], rows, 1), chunk))
    members = [[] for _ in range(n_groups)]
    for n in range(N):
        if node_group[n] >= 0:
            members[node_group[n]].append(n)
    for gi in range(n_groups):
        reqs, req_ids, rows = [], [], []
        cur_r, local = -1, {}
        for n in members[gi]:
            r = int(np.searchsorted(rp, n, side="right") - 1)
            if r != cur_r:
                reqs.append([(-1, 0)])
                req_ids.append(r)
                cur_r, local = r, {int(rp[r]): 0}
            local[n] = len(reqs[-1])
            reqs[-1].append((local[int(rp[r] + parent[n])], int(seg[n])))
            rows.append(np.arange(starts[n], starts[n + 1]))
        depth_max = 1
        for nodes in reqs:
            dd = [0]
            for pa, _ in nodes[1:]:
                dd.append(dd[pa] + 1)
            depth_max = max(depth_max, max(dd))
        out.append(("group", _Batch(reqs, np.concatenate(rows), depth_max), req_ids))
    return out


class BoundedGdn:
    """The memory-bounded schedule of one tree shape, built once: the batches,
    their device index arrays and one node-state buffer of the budget's size.
    ``run`` then launches every batch back to back on the current stream."""

    def __init__(self, tree, max_slots: int, H: int, dk: int, dv: int, device="cuda"):
        self.R, self.max_slots = tree.R, int(max_slots)
        self.H, self.dk, self.dv, self.device = H, dk, dv, device
        self.batches = []
        for kind, batch, req_ids in _batches(tree, max_slots):
            dt = flide.DeviceTree(*batch.arrays(), max_depth=max(batch.levels, 1), device=device)
            idx = flide.TreeIndex(dt.R, dt.N, dt.T, dt.max_depth, device=device)
            self.batches.append((kind, int(batch.seg.sum()), dt, idx,
                                 torch.from_numpy(batch.rows).to(device),
                                 torch.as_tensor(np.asarray(req_ids, np.int32)).to(device), len(req_ids)))
        self.groups = sum(1 for b in self.batches if b[0] == "group")
        self.node_state = torch.empty((max(self.max_slots, 1), H, dv, dk), dtype=torch.float32,
                                      device=device)
        self.root_state = torch.zeros((self.R, H, dv, dk), dtype=torch.float32, device=device)

    @property
    def state_bytes(self) -> int:
        return self.node_state.numel() * 4

    def run(self, q, k, v, g, beta, state_in=None, out=None):
        """Outputs [T, H, dv] (and self.root_state, the roots' end states)."""
        T = q.shape[0]
        H, dk, dv, dev = self.H, self.dk, self.dv, q.device
        if out is None:
            out = torch.empty((T, H, dv), dtype=q.dtype, device=dev)
        for kind, t, dt, idx, src, ridx, nreq in self.batches:
            sub = {}
            for name, x in (("q", q), ("k", k), ("v", v), ("g", g), ("beta", beta)):
                y = torch.empty((max(t, 1),) + tuple(x.shape[1:]), dtype=x.dtype, device=dev)
                _copy_rows(y, x, src_idx=src, n=t)
                sub[name] = y
            base = state_in if kind == "roots" else self.root_state
            sin = None
            if base is not None:
                sin = torch.empty((nreq, H, dv, dk), dtype=torch.float32, device=dev)
                _copy_rows(sin, base, src_idx=ridx, n=nreq)
            flide.tree_build(dt, idx)
            o = flide.fork_gdn(sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"], idx,
                               self.node_state, state_in=sin)
            if t:
                _copy_rows(out, o, dst_idx=src, n=t)
            if kind == "roots":
                # roots take slots 0 .. nreq-1 in request order
                _copy_rows(self.root_state, self.node_state, dst_idx=ridx, n=nreq)
        return out

    def status(self) -> int:
        """First non-zero device status of the batches (waits for them)."""
        torch.cuda.current_stream().synchronize()
        for b in self.batches:
            st = b[3].status()
            if st != 0:
                return st
        return 0


def fork_gdn_bounded(q, k, v, g, beta, tree, max_slots: int, state_in=None, out=None):
    """The GDN fork scan of ``tree`` (host arrays; q, k [T, H, dk], v [T, H, dv],
    g, beta [T, H] on the device) with at most ``max_slots`` node-state slots
    live at a time.  Returns (out [T, H, dv], root end states [R, H, dv, dk]),
    equal to flide.fork_gdn's outputs and root-slot states; waits for the
    batches and raises on a device error."""
    plan = BoundedGdn(tree, max_slots, q.shape[1], q.shape[2], v.shape[2], device=q.device)
    out = plan.run(q, k, v, g, beta, state_in=state_in, out=out)
    st = plan.status()
    if st != 0:
        raise flide.FlideError(st, "fork_gdn_bounded")
    return out, plan.root_state
