"""CPU oracle for the ForkAttention hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library
(``tree_forked_decision_b200``) never imports it and shares no code with it.

The arithmetic lives in ``flide_oracle.c`` (plain C, double precision); this
module compiles it with gcc and wraps it with ctypes.  It follows the pages on
Flide: "fork equals isolation" (kongchang.com, "ForkAttention" section), no
cross-branch attention (kongchang.com, attention-mask section) and per-branch
Gated DeltaNet state evolution (kongchang.com, Gated DeltaNet box).

Every function pins to something other than itself in
``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "flide_oracle.c")
_SO = os.path.join(_HERE, "_build", "liboracle.so")
_lib = None

OK = 0
INVALID = 1
NOMEM = 2


def build(force: bool = False) -> str:
    """Compile flide_oracle.c into oracle/_build/liboracle.so (gcc, OpenMP)."""
    os.makedirs(os.path.dirname(_SO), exist_ok=True)
    if (not force and os.path.exists(_SO)
            and os.path.getmtime(_SO) >= os.path.getmtime(_SRC)):
        return _SO
    tmp = _SO + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_tree_index.argtypes = [I, P, P, P, P, P, P, P, P, P, P, I, P]
        lib.oracle_tree_index.restype = I
        lib.oracle_attention_rows.argtypes = [I, P, P, P, P, I, I, I, P, P, P,
                                              P, P, ctypes.c_double, I, P, P, P]
        lib.oracle_attention_rows.restype = I
        lib.oracle_gdn.argtypes = [I, P, P, P, I, I, I, P, P, P, P, P, P, P,
                                   I, I, P, P, P, P]
        lib.oracle_gdn.restype = I
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = I
        _lib = lib
    return _lib


def _i32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


class OracleError(RuntimeError):
    def __init__(self, code):
        super().__init__(f"oracle status {code}")
        self.code = code


def tree_index(req_node_ptr, parent, seg_len, past_len):
    """Index arrays of the flattened stream by walking parent pointers.

    Returns a dict with node_start, token_node, token_pos, depth, anc_ptr,
    anc_node, ctx_len (int32 numpy arrays), or raises OracleError (code 1 for a
    malformed tree).
    """
    lib = _load()
    rp, pa, sl, pl = _i32(req_node_ptr), _i32(parent), _i32(seg_len), _i32(past_len)
    R = len(rp) - 1
    N = int(rp[-1])
    T = int(np.maximum(sl, 0).sum()) if N else 0
    node_start = np.zeros(N + 1, np.int32)
    token_node = np.zeros(max(T, 1), np.int32)
    token_pos = np.zeros(max(T, 1), np.int32)
    depth = np.zeros(max(N, 1), np.int32)
    anc_ptr = np.zeros(N + 1, np.int32)
    anc_cap = max(1, min(N * (N + 1) // 2, N * 256))
    anc_node = np.zeros(anc_cap, np.int32)
    ctx_len = np.zeros(max(N, 1), np.int32)
    st = lib.oracle_tree_index(R, _ptr(rp), _ptr(pa), _ptr(sl), _ptr(pl),
                               _ptr(node_start), _ptr(token_node), _ptr(token_pos),
                               _ptr(depth), _ptr(anc_ptr), _ptr(anc_node), anc_cap,
                               _ptr(ctx_len))
    if st != OK:
        raise OracleError(st)
    return dict(node_start=node_start, token_node=token_node[:T],
                token_pos=token_pos[:T], depth=depth[:N], anc_ptr=anc_ptr,
                anc_node=anc_node[:int(anc_ptr[-1])], ctx_len=ctx_len[:N])


def attention_rows(tree, q, k, v, past_k, past_v, scale, rows):
    """Softmax attention of selected query rows over their isolated sequences.

    tree: (req_node_ptr, parent, seg_len, past_len).  q [T,Hq,d], k/v
    [T,Hkv,d], past_k/past_v [sum(past_len),Hkv,d] or None; float32 arrays
    (bf16 callers upcast first, which is exact).  rows: int array [n,2] of
    (token, q_head).  Returns float64 [n, d].
    """
    lib = _load()
    rp, pa, sl, pl = (_i32(x) for x in tree)
    q, k, v = _f32(q), _f32(k), _f32(v)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    pk = _f32(past_k) if past_k is not None and past_k.size else None
    pv = _f32(past_v) if past_v is not None and past_v.size else None
    rows = _i32(rows).reshape(-1, 2)
    rt = np.ascontiguousarray(rows[:, 0])
    rh = np.ascontiguousarray(rows[:, 1])
    out = np.zeros((len(rows), d), np.float64)
    st = lib.oracle_attention_rows(len(rp) - 1, _ptr(rp), _ptr(pa), _ptr(sl), _ptr(pl),
                                   Hq, Hkv, d, _ptr(q), _ptr(k), _ptr(v), _ptr(pk),
                                   _ptr(pv), float(scale), len(rows), _ptr(rt),
                                   _ptr(rh), _ptr(out))
    if st != OK:
        raise OracleError(st)
    return out


def attention_all(tree, q, k, v, past_k, past_v, scale):
    """All rows of attention_rows, shaped [T, Hq, d] (float64)."""
    T, Hq, d = np.asarray(q).shape
    tt, hh = np.meshgrid(np.arange(T), np.arange(Hq), indexing="ij")
    rows = np.stack([tt.ravel(), hh.ravel()], 1)
    return attention_rows(tree, q, k, v, past_k, past_v, scale, rows).reshape(T, Hq, d)


def gdn(tree, q, k, v, g, beta, state_in=None, memoise=True, pairs=None,
        want_states=False):
    """Gated DeltaNet over the tree; every node in isolation (memoise=False) or
    continuing from its parent's end state (memoise=True, bitwise equal).

    q,k [T,H,dk]; v [T,H,dv]; g,beta [T,H] float32 (g = log alpha);
    state_in [R,H,dv,dk] float32 or float64 or None.  pairs: list of (request, head) to
    compute (default all).  Returns out [T,H,dv] float64 (zeros outside the
    selected pairs) and, with want_states, node end states [N,H,dv,dk].
    """
    lib = _load()
    rp, pa, sl = _i32(tree[0]), _i32(tree[1]), _i32(tree[2])
    R = len(rp) - 1
    q, k, v, g, beta = _f32(q), _f32(k), _f32(v), _f32(g), _f32(beta)
    T, H, dk = q.shape
    dv = v.shape[2]
    si = si64 = None
    if state_in is not None and np.asarray(state_in).dtype == np.float64:
        si64 = np.ascontiguousarray(state_in)
    elif state_in is not None:
        si = _f32(state_in)
    if pairs is None:
        pairs = [(r, h) for r in range(R) for h in range(H)]
    pairs = _i32(pairs).reshape(-1, 2)
    sr = np.ascontiguousarray(pairs[:, 0])
    sh = np.ascontiguousarray(pairs[:, 1])
    out = np.zeros((T, H, dv), np.float64)
    N = int(rp[-1])
    states = np.zeros((N, H, dv, dk), np.float64) if want_states else None
    st = lib.oracle_gdn(R, _ptr(rp), _ptr(pa), _ptr(sl), H, dk, dv, _ptr(q), _ptr(k),
                        _ptr(v), _ptr(g), _ptr(beta), _ptr(si), _ptr(si64), int(bool(memoise)),
                        len(pairs), _ptr(sr), _ptr(sh), _ptr(out), _ptr(states))
    if st != OK:
        raise OracleError(st)
    return (out, states) if want_states else out


from .decision import branch_logprob, option_probs, tvd  # noqa: E402,F401  (numpy, fp64)
