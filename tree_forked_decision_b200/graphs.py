"""Shape buckets: a few pre-captured CUDA graphs of the whole call sequence.

The pages describe a compact set of pre-recorded execution graphs that serve
varied request mixes (kongchang.com article on Flide, pre-recorded execution
graphs box).  Here a bucket is one CUDA graph of

    flide_tree_build -> flide_fork_attn -> flide_fork_gdn -> flide_state_save

captured once over static device buffers sized by the bucket's capacities
(requests R, nodes N, stream tokens T, past rows P, tree depth D).  Every
kernel reads the actual sizes from device memory, so any tree that fits is
copied into the buffers (padded with empty requests) and the graph replays
unchanged: no host work depends on the tree's shape.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

from . import flide


@dataclasses.dataclass(frozen=True)
class BucketShape:
    R: int
    N: int
    T: int
    P: int
    D: int

    def fits(self, tree) -> bool:
        return (tree.R <= self.R and tree.N <= self.N and tree.T <= self.T
                and tree.P_past <= self.P and tree.levels <= self.D)


class GraphBucket:
    """Static buffers + one captured graph of the hot path."""

    def __init__(self, shape: BucketShape, attn: dict | None, gdn: dict | None,
                 dtype=torch.bfloat16, device="cuda"):
        self.shape = s = shape
        self.attn_spec, self.gdn_spec = attn, gdn
        self.device = device
        self._alloc(dtype)
        self.dt = flide.DeviceTree.from_buffers(self.req_node_ptr, self.parent, self.seg_len,
                                                self.past_len, s.N, s.T, s.D)
        self.idx = flide.TreeIndex(s.R, s.N, s.T, s.D, device=device)
        self.graph = None

    def _alloc(self, dtype):
        """The static buffers, sized by the bucket's capacities."""
        s, device = self.shape, self.device
        i32 = lambda n: torch.zeros(max(n, 1), dtype=torch.int32, device=device)
        self.req_node_ptr = i32(s.R + 1)
        self.parent = i32(s.N)
        self.seg_len = i32(s.N)
        self.past_len = i32(s.R)
        z = lambda *shp, dt=dtype: torch.zeros(shp, dtype=dt, device=device)
        if self.attn_spec:
            Hq, Hkv, d = self.attn_spec["Hq"], self.attn_spec["Hkv"], self.attn_spec["d"]
            self.q, self.k, self.v = z(s.T, Hq, d), z(s.T, Hkv, d), z(s.T, Hkv, d)
            self.past_k, self.past_v = z(max(s.P, 1), Hkv, d), z(max(s.P, 1), Hkv, d)
            self.out = z(s.T, Hq, d)
            self.ckpt_k, self.ckpt_v = z(s.P + s.T, Hkv, d), z(s.P + s.T, Hkv, d)
            self.scale = 1.0 / math.sqrt(d)
        if self.gdn_spec:
            H, dk, dv = self.gdn_spec["H"], self.gdn_spec["dk"], self.gdn_spec["dv"]
            self.gq, self.gk, self.gv = z(s.T, H, dk), z(s.T, H, dk), z(s.T, H, dv)
            self.gg = z(s.T, H, dt=torch.float32)
            self.gb = z(s.T, H, dt=torch.float32)
            self.state_in = z(s.R, H, dv, dk, dt=torch.float32)
            self.gout = z(s.T, H, dv)
            self.node_state = z(s.N, H, dv, dk, dt=torch.float32)
            self.ckpt_S = z(s.R, H, dv, dk, dt=torch.float32)

    def _sequence(self):
        flide.tree_build(self.dt, self.idx)
        if self.attn_spec:
            flide.fork_attn(self.q, self.k, self.v, self.idx, self.scale, past_k=self.past_k,
                            past_v=self.past_v, out=self.out)
        if self.gdn_spec:
            flide.fork_gdn(self.gq, self.gk, self.gv, self.gg, self.gb, self.idx, self.node_state,
                           state_in=self.state_in, out=self.gout)
        flide.state_save(self.idx, self.k if self.attn_spec else None,
                         self.v if self.attn_spec else None,
                         self.ckpt_k if self.attn_spec else None,
                         self.ckpt_v if self.attn_spec else None,
                         self.ckpt_S if self.gdn_spec else None,
                         past_k=self.past_k if self.attn_spec else None,
                         past_v=self.past_v if self.attn_spec else None,
                         node_state=self.node_state if self.gdn_spec else None)

    def capture(self):
        """Runs the sequence once eagerly (an empty batch) and captures it."""
        self.req_node_ptr.zero_()
        self.past_len.zero_()
        side = torch.cuda.Stream(device=self.device)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self._sequence()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self._sequence()
        torch.cuda.synchronize()
        return self

    def load(self, tree, attn: dict | None = None, gdn: dict | None = None):
        """Copies a tree that fits (and its tensors) into the static buffers;
        trailing requests stay empty."""
        s = self.shape
        if not s.fits(tree):
            raise ValueError(f"tree (R={tree.R}, N={tree.N}, T={tree.T}, P={tree.P_past}, "
                             f"D={tree.levels}) does not fit bucket {s}")
        rp = np.full(s.R + 1, tree.N, np.int32)
        rp[:tree.R + 1] = tree.req_node_ptr
        pl = np.zeros(s.R, np.int32)
        pl[:tree.R] = tree.past_len
        self.req_node_ptr.copy_(torch.from_numpy(rp), non_blocking=True)
        self.past_len.copy_(torch.from_numpy(pl), non_blocking=True)
        if tree.N:
            self.parent[:tree.N].copy_(torch.from_numpy(np.ascontiguousarray(tree.parent)))
            self.seg_len[:tree.N].copy_(torch.from_numpy(np.ascontiguousarray(tree.seg_len)))
        T, P = tree.T, tree.P_past
        if attn is not None and self.attn_spec:
            self.q[:T].copy_(attn["q"], non_blocking=True)
            self.k[:T].copy_(attn["k"], non_blocking=True)
            self.v[:T].copy_(attn["v"], non_blocking=True)
            if P:
                self.past_k[:P].copy_(attn["past_k"], non_blocking=True)
                self.past_v[:P].copy_(attn["past_v"], non_blocking=True)
        if gdn is not None and self.gdn_spec:
            self.gq[:T].copy_(gdn["q"], non_blocking=True)
            self.gk[:T].copy_(gdn["k"], non_blocking=True)
            self.gv[:T].copy_(gdn["v"], non_blocking=True)
            self.gg[:T].copy_(gdn["g"], non_blocking=True)
            self.gb[:T].copy_(gdn["beta"], non_blocking=True)
            self.state_in.zero_()
            self.state_in[:tree.R].copy_(gdn["state_in"], non_blocking=True)
        self.loaded = tree
        return self

    def replay(self):
        if self.graph is None:
            self.capture()
        self.graph.replay()
        return self

    def outputs(self):
        T = self.loaded.T
        o = {}
        if self.attn_spec:
            o["attn"] = self.out[:T]
        if self.gdn_spec:
            o["gdn"] = self.gout[:T]
        return o


class GraphBuckets:
    """A small set of buckets; a batch goes to the smallest one it fits."""

    def __init__(self, shapes, attn, gdn, dtype=torch.bfloat16, device="cuda"):
        self.buckets = [GraphBucket(s, attn, gdn, dtype, device)
                        for s in sorted(shapes, key=lambda s: (s.T, s.N, s.R, s.P, s.D))]

    def capture(self):
        for b in self.buckets:
            b.capture()
        return self

    def pick(self, tree) -> GraphBucket:
        for b in self.buckets:
            if b.shape.fits(tree):
                return b
        raise ValueError("no bucket fits this batch")

    def run(self, tree, attn=None, gdn=None) -> GraphBucket:
        return self.pick(tree).load(tree, attn, gdn).replay()
