"""Seeded synthetic inputs: decision trees and layer tensors.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic.  Both the CUDA path and the CPU oracle consume exactly the
tensors it returns.

Tree shapes follow the workloads: a shared prefix (the root node) plus option
branches laid out in one flattened token stream (kongchang.com, introduction
and "ForkAttention" section); up to 256 options per request (techfi24.com,
"Performances et comparaison"); resumed requests carry checkpointed history
(kongchang.com, "ForkAttention" section).  Value distributions: q, k, v ~
N(0, 1); for Gated DeltaNet, q and k are L2-normalised per head, the gate is
passed as g = log(alpha) = -scale * softplus(x), x ~ N(0, 1), and
beta = sigmoid(N(0, 1)).

Stream order: requests in order; within a request, nodes in index order with
parent[i] < i; node 0 of every request is its root.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os

import numpy as np
import torch


@dataclasses.dataclass
class Tree:
    req_node_ptr: np.ndarray  # int32 [R+1]
    parent: np.ndarray        # int32 [N], request-local parent, -1 for a root
    seg_len: np.ndarray       # int32 [N], tokens per node in stream order
    past_len: np.ndarray      # int32 [R], checkpointed tokens before the root
    levels: int               # branch levels below the root (by construction)

    @property
    def R(self) -> int:
        return len(self.req_node_ptr) - 1

    @property
    def N(self) -> int:
        return int(self.req_node_ptr[-1])

    @property
    def T(self) -> int:
        return int(self.seg_len.sum())

    @property
    def P_past(self) -> int:
        return int(self.past_len.sum())

    @property
    def root_tokens(self) -> int:
        roots = self.req_node_ptr[:-1][self.req_node_ptr[:-1] < self.req_node_ptr[1:]]
        return int(self.seg_len[roots].sum())

    @property
    def branch_tokens(self) -> int:
        return self.T - self.root_tokens

    def arrays(self):
        return self.req_node_ptr, self.parent, self.seg_len, self.past_len


def _tree(reqs, levels):
    """reqs: list of (past_len, [(parent_local, seg_len), ...])."""
    rp = [0]
    parent, seg, past = [], [], []
    for p_len, nodes in reqs:
        past.append(p_len)
        for pa, sl in nodes:
            parent.append(pa)
            seg.append(sl)
        rp.append(rp[-1] + len(nodes))
    return Tree(np.asarray(rp, np.int32), np.asarray(parent, np.int32),
                np.asarray(seg, np.int32), np.asarray(past, np.int32), levels)


def fanout_tree(R: int, prefix: int, branches: int, branch_len: int,
                past: int = 0) -> Tree:
    """R requests, each a root of `prefix` tokens and `branches` leaves of
    `branch_len` tokens (depth 1)."""
    nodes = [(-1, prefix)] + [(0, branch_len)] * branches
    return _tree([(past, nodes)] * R, 1 if branches else 0)


def warm_variant(tree: Tree):
    """The same batch resumed from checkpoints: each root's tokens move into
    its request's checkpointed past (past_len + root length) and the root keeps
    zero tokens, so only branch tokens remain in the stream.  Returns the new
    tree and the stream rows of the original tree that it keeps, in order.
    With the original step's checkpoint (past rows then root rows per request,
    and the root's end states) as past K/V and GDN state_in, the outputs of the
    kept rows are the original ones (resume equals scratch)."""
    rp, pa, sl, pl = tree.arrays()
    starts = np.concatenate([[0], np.cumsum(sl)]).astype(np.int64)
    reqs, keep = [], []
    for r in range(tree.R):
        n0, n1 = int(rp[r]), int(rp[r + 1])
        if n1 == n0:
            reqs.append((int(pl[r]), []))
            continue
        nodes = [(-1, 0)] + [(int(pa[n]), int(sl[n])) for n in range(n0 + 1, n1)]
        reqs.append((int(pl[r]) + int(sl[n0]), nodes))
        keep.append(np.arange(starts[n0 + 1], starts[n1]))
    rows = np.concatenate(keep) if keep else np.zeros(0, np.int64)
    return _tree(reqs, tree.levels), rows


def leveled_tree(rng: np.random.Generator, R: int, depth_range=(1, 3),
                 options_range=(2, 256), prefix_range=(256, 8192),
                 branch_range=(4, 64), n_resume: int = 0,
                 resume_delta=(4, 64)) -> Tree:
    """Mixed batch of level-structured trees.

    Per request: D ~ U{depth_range}, O ~ U{options_range} leaves, prefix
    P ~ U{prefix_range}, every non-root segment ~ U{branch_range}.  Level sizes
    n_0 = 1, n_k = ceil(O^(k/D)) for 0 < k < D, n_D = O; node j of level k hangs
    under node (j mod n_{k-1}) of level k-1.  `n_resume` requests (seeded
    choice) resume from a checkpoint holding their first P - delta prefix
    tokens, delta ~ U{resume_delta}: those tokens become past, the root keeps
    delta tokens.
    """
    reqs = []
    max_levels = 0
    resumed = set(rng.choice(R, size=n_resume, replace=False).tolist()) if n_resume else set()
    for r in range(R):
        D = int(rng.integers(depth_range[0], depth_range[1] + 1))
        O = int(rng.integers(options_range[0], options_range[1] + 1))
        P = int(rng.integers(prefix_range[0], prefix_range[1] + 1))
        sizes = [1] + [int(math.ceil(O ** (k / D))) for k in range(1, D)] + [O]
        first = [0]
        for s in sizes[:-1]:
            first.append(first[-1] + s)
        nodes = []
        for k, nk in enumerate(sizes):
            for j in range(nk):
                if k == 0:
                    nodes.append([-1, P])
                else:
                    pa = first[k - 1] + (j % sizes[k - 1])
                    nodes.append([pa, int(rng.integers(branch_range[0], branch_range[1] + 1))])
        past = 0
        if r in resumed:
            delta = int(rng.integers(resume_delta[0], resume_delta[1] + 1))
            delta = min(delta, P)
            past = P - delta
            nodes[0][1] = delta
        max_levels = max(max_levels, D)
        reqs.append((past, [tuple(x) for x in nodes]))
    return _tree(reqs, max_levels)


def random_tree(rng: np.random.Generator, R: int, max_nodes: int = 8,
                prefix_range=(0, 40), branch_range=(1, 9),
                past_range=(0, 0)) -> Tree:
    """Small irregular trees for tests: each node's parent is uniform among the
    earlier nodes of its request."""
    reqs = []
    levels = 0
    for _ in range(R):
        n = int(rng.integers(1, max_nodes + 1))
        nodes = [(-1, int(rng.integers(prefix_range[0], prefix_range[1] + 1)))]
        depth = [0]
        for i in range(1, n):
            pa = int(rng.integers(0, i))
            nodes.append((pa, int(rng.integers(branch_range[0], branch_range[1] + 1))))
            depth.append(depth[pa] + 1)
        levels = max(levels, max(depth))
        reqs.append((int(rng.integers(past_range[0], past_range[1] + 1)), nodes))
    return _tree(reqs, levels)


_CHUNK = 1 << 24  # elements per independently seeded block of normals


def normals(rng: np.random.Generator, shape) -> np.ndarray:
    """float32 N(0,1) array of `shape`.  Large arrays are filled in blocks of
    2^24 elements, each from its own generator seeded by `rng`, on several
    threads; the values depend only on rng's state and the shape."""
    n = int(np.prod(shape))
    out = np.empty(n, np.float32)
    blocks = (n + _CHUNK - 1) // _CHUNK
    seeds = rng.integers(0, 2**63 - 1, size=max(blocks, 1))

    def fill(b):
        sl = slice(b * _CHUNK, min(n, (b + 1) * _CHUNK))
        np.random.default_rng(int(seeds[b])).standard_normal(out=out[sl], dtype=np.float32)

    if blocks <= 1:
        if n:
            fill(0)
    else:
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(blocks)))
    return out.reshape(shape)


def _to(x: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(dtype)


def attn_inputs(tree: Tree, Hq: int, Hkv: int, d: int, dtype: torch.dtype,
                rng: np.random.Generator):
    """q [T,Hq,d], k,v [T,Hkv,d], past_k,past_v [sum(past),Hkv,d]; N(0,1)."""
    T, P = tree.T, tree.P_past
    q = normals(rng, (T, Hq, d))
    k = normals(rng, (T, Hkv, d))
    v = normals(rng, (T, Hkv, d))
    pk = normals(rng, (P, Hkv, d))
    pv = normals(rng, (P, Hkv, d))
    return dict(q=_to(q, dtype), k=_to(k, dtype), v=_to(v, dtype),
                past_k=_to(pk, dtype), past_v=_to(pv, dtype))


def fp8_attn_inputs(tree: Tree, Hq: int, Hkv: int, d: int, rng: np.random.Generator,
                    amp: float = 64.0):
    """e4m3 codes (uint8 tensors) of amp * N(0,1) for q [T,Hq,d], k, v [T,Hkv,d]
    and past_k, past_v [sum(past),Hkv,d], cast by torch's float8_e4m3fn
    conversion, with descale = (1/amp, 1/amp, 1/amp) (float32 [3]): the
    decoded values are N(0,1) to within the format's rounding.  Values are
    clamped to +-448 first (the cast would make NaN of anything larger; at
    amp = 64 that takes a 7-sigma draw)."""
    T, P = tree.T, tree.P_past

    def codes(shape):
        x = np.clip(normals(rng, shape) * np.float32(amp), -448.0, 448.0)
        return torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8)

    return dict(q=codes((T, Hq, d)), k=codes((T, Hkv, d)), v=codes((T, Hkv, d)),
                past_k=codes((P, Hkv, d)), past_v=codes((P, Hkv, d)),
                descale=torch.full((3,), 1.0 / amp, dtype=torch.float32))


def _l2n(x: np.ndarray) -> torch.Tensor:
    """Rows scaled to unit L2 norm, in float32."""
    t = torch.from_numpy(x)
    return t / torch.linalg.vector_norm(t, dim=-1, keepdim=True).clamp_min(1e-6)


def gdn_inputs(tree: Tree, H: int, dk: int, dv: int, dtype: torch.dtype,
               rng: np.random.Generator, gate_scale: float = 1.0,
               state_scale: float = 0.1):
    """q,k [T,H,dk] (L2-normalised), v [T,H,dv], g = -gate_scale*softplus(x)
    and beta = sigmoid(y) [T,H] float32 with x, y ~ N(0,1); state_in
    [R,H,dv,dk] float32: N(0, state_scale^2) for requests with past history,
    zero otherwise."""
    T, R = tree.T, tree.R
    q = _l2n(normals(rng, (T, H, dk)))
    k = _l2n(normals(rng, (T, H, dk)))
    v = normals(rng, (T, H, dv))
    x = rng.standard_normal((T, H)).astype(np.float64)
    g = (-gate_scale * np.logaddexp(0.0, x)).astype(np.float32)
    y = rng.standard_normal((T, H)).astype(np.float64)
    beta = (1.0 / (1.0 + np.exp(-y))).astype(np.float32)
    state = np.zeros((R, H, dv, dk), np.float32)
    for r in range(R):
        if tree.past_len[r] > 0:
            state[r] = normals(rng, (H, dv, dk)) * np.float32(state_scale)
    return dict(q=q.to(dtype), k=k.to(dtype), v=_to(v, dtype),
                g=torch.from_numpy(g), beta=torch.from_numpy(beta),
                state_in=torch.from_numpy(state))


def fp8_gdn_inputs(tree: Tree, H: int, dk: int, dv: int, rng: np.random.Generator,
                   gate_scale: float = 1.0, state_scale: float = 0.1,
                   amp_qk: float = 256.0, amp_v: float = 64.0):
    """The values of gdn_inputs (float32) with q, k and v as e4m3 codes (uint8
    tensors) of amp * value, cast by torch's float8_e4m3fn conversion, and
    descale = (1/amp_qk, 1/amp_qk, 1/amp_v) (float32 [3]); L2-normalised q, k
    times 256 and N(0,1) v times 64 stay below the format's largest value 448.
    g, beta and state_in as in gdn_inputs."""
    d = gdn_inputs(tree, H, dk, dv, torch.float32, rng, gate_scale=gate_scale,
                   state_scale=state_scale)

    def codes(x, amp):  # clamped to +-448: the cast makes NaN of larger values
        return (x * np.float32(amp)).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)

    d.update(q=codes(d["q"], amp_qk), k=codes(d["k"], amp_qk), v=codes(d["v"], amp_v),
             descale=torch.tensor([1.0 / amp_qk, 1.0 / amp_qk, 1.0 / amp_v], dtype=torch.float32))
    return d


# ---------------------------------------------------------------------------
# Named workloads.  Each returns (tree, attention spec or None, GDN spec or
# None, dtype).  seed defaults to the workload's index.
# ---------------------------------------------------------------------------

WORKLOADS = {
    "tiny_fp32": dict(idx=1, desc="1 request, prefix 64, 4 branches x 8, attn 4 heads d=64, GDN 4 heads dk=dv=64, fp32"),
    "attn_fanout_bf16": dict(idx=2, desc="8 requests, prefix 2048, 16 branches x 32, GQA Hq=16 Hkv=4 d=128, bf16"),
    "gdn_fanout_bf16": dict(idx=3, desc="8 requests, prefix 4096, 64 branches x 16, GDN 16 heads dk=dv=128, bf16"),
    "mixed_hybrid_bf16": dict(idx=4, desc="32 requests depth 1-3, 2-256 options, prefix 256-8192, branches 4-64, half resumed; attn Hq=16 Hkv=4 d=128 + GDN 16x128, bf16"),
    "large_fanout_bf16": dict(idx=5, desc="4 requests, prefix 32768, 256 branches x 8, attn Hq=32 Hkv=8 d=128 + GDN 32 heads dk=dv=128, bf16"),
    "attn_longprefix_bf16": dict(idx=6, desc="1 request, prefix 32768, 256 branches x 8, GQA Hq=4 Hkv=1 d=128, bf16 (one kv group of the large fan-out request: a small case for kernel profiles)"),
    "large_fanout_req_bf16": dict(idx=7, desc="1 request, prefix 32768, 256 branches x 8, attn Hq=32 Hkv=8 d=128 + GDN 32 heads dk=dv=128, bf16 (one request of the large fan-out batch: inputs above L2 but a quarter of the size, for DRAM-byte profiles)"),
}


def workload(name: str, seed: int | None = None):
    spec = WORKLOADS[name]
    rng = np.random.default_rng(spec["idx"] if seed is None else seed)
    if name == "tiny_fp32":
        tree = fanout_tree(1, 64, 4, 8)
        return tree, dict(Hq=4, Hkv=4, d=64), dict(H=4, dk=64, dv=64, gate_scale=1.0), torch.float32, rng
    if name == "attn_fanout_bf16":
        tree = fanout_tree(8, 2048, 16, 32)
        return tree, dict(Hq=16, Hkv=4, d=128), None, torch.bfloat16, rng
    if name == "gdn_fanout_bf16":
        tree = fanout_tree(8, 4096, 64, 16)
        return tree, None, dict(H=16, dk=128, dv=128, gate_scale=0.1), torch.bfloat16, rng
    if name == "mixed_hybrid_bf16":
        tree = leveled_tree(rng, 32, n_resume=16)
        return tree, dict(Hq=16, Hkv=4, d=128), dict(H=16, dk=128, dv=128, gate_scale=0.1), torch.bfloat16, rng
    if name == "attn_longprefix_bf16":
        tree = fanout_tree(1, 32768, 256, 8)
        return tree, dict(Hq=4, Hkv=1, d=128), None, torch.bfloat16, rng
    if name == "large_fanout_req_bf16":
        tree = fanout_tree(1, 32768, 256, 8)
        return tree, dict(Hq=32, Hkv=8, d=128), dict(H=32, dk=128, dv=128, gate_scale=0.1), torch.bfloat16, rng
    if name == "large_fanout_bf16":
        tree = fanout_tree(4, 32768, 256, 8)
        return tree, dict(Hq=32, Hkv=8, d=128), dict(H=32, dk=128, dv=128, gate_scale=0.1), torch.bfloat16, rng
    raise KeyError(name)


def make_inputs(name: str, seed: int | None = None):
    """Tree plus host tensors for a named workload."""
    tree, aspec, gspec, dtype, rng = workload(name, seed)
    attn = gdn = None
    if aspec:
        attn = attn_inputs(tree, aspec["Hq"], aspec["Hkv"], aspec["d"], dtype, rng)
        attn.update(aspec)
    if gspec:
        gdn = gdn_inputs(tree, gspec["H"], gspec["dk"], gspec["dv"], dtype, rng,
                         gate_scale=gspec["gate_scale"])
        gdn.update(gspec)
    return tree, attn, gdn, dtype
