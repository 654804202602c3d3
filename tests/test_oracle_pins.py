"""Pins for the CPU oracle: each oracle function checked against something
other than itself -- hand-worked golden fixtures, closed forms, special cases
that reduce to a textbook routine, a different algorithm that is equal in exact
arithmetic, and brute force on tiny inputs.  CPU only.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tree_forked_decision_b200 import inputs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _paths(tree):
    """root..self path (global ids) of every node, by walking parents."""
    rp, pa = tree[0], tree[1]
    out = {}
    for r in range(len(rp) - 1):
        for n in range(rp[r], rp[r + 1]):
            p, cur = [], n
            while True:
                p.append(cur)
                if pa[cur] < 0:
                    break
                cur = rp[r] + pa[cur]
            out[n] = p[::-1]
    return out


def _starts(seg_len):
    return np.concatenate([[0], np.cumsum(seg_len)]).astype(np.int64)


def _node_req(rp):
    nr = np.zeros(rp[-1], np.int64)
    for r in range(len(rp) - 1):
        nr[rp[r]:rp[r + 1]] = r
    return nr


# ---------------------------------------------------------------------------
# tree index
# ---------------------------------------------------------------------------

def test_tree_index_hand_worked_example():
    g = _gold("tree_index_small.json")
    idx = oracle.tree_index(g["req_node_ptr"], g["parent"], g["seg_len"], g["past_len"])
    for key, want in g["expect"].items():
        assert idx[key].tolist() == want, key


@pytest.mark.parametrize("seed", range(6))
def test_tree_index_invariants_random(seed):
    rng = np.random.default_rng(100 + seed)
    t = inputs.random_tree(rng, R=5, max_nodes=9, prefix_range=(0, 7),
                           branch_range=(1, 5), past_range=(0, 6))
    rp, pa, sl, pl = t.arrays()
    idx = oracle.tree_index(rp, pa, sl, pl)
    assert int(idx["node_start"][-1]) == int(sl.sum()) == t.T
    assert np.array_equal(np.diff(idx["node_start"]), sl)
    nreq = _node_req(rp)
    for n in range(t.N):
        row = idx["anc_node"][idx["anc_ptr"][n]:idx["anc_ptr"][n + 1]].tolist()
        assert row[-1] == n
        assert idx["depth"][n] == len(row) - 1
        r = nreq[n]
        if pa[n] < 0:
            assert row == [n]
        else:
            p = rp[r] + pa[n]
            prow = idx["anc_node"][idx["anc_ptr"][p]:idx["anc_ptr"][p + 1]].tolist()
            assert row == prow + [n]
        # positions along the root..n path are exactly past, past+1, ...
        toks = [tk for a in row for tk in range(idx["node_start"][a], idx["node_start"][a + 1])]
        assert idx["token_pos"][toks].tolist() == list(range(pl[r], pl[r] + len(toks)))
        assert idx["ctx_len"][n] == pl[r] + len(toks)
        assert all(idx["token_node"][tk] == n for tk in range(idx["node_start"][n], idx["node_start"][n + 1]))


@pytest.mark.parametrize("bad", ["parent_ge_self", "root_parent", "empty_branch", "ptr_decreasing"])
def test_tree_index_rejects_malformed(bad):
    rp, pa, sl, pl = [0, 3], [-1, 0, 1], [2, 1, 1], [0]
    if bad == "parent_ge_self":
        pa = [-1, 1, 1]
    elif bad == "root_parent":
        pa = [0, 0, 1]
    elif bad == "empty_branch":
        sl = [2, 0, 1]
    elif bad == "ptr_decreasing":
        rp, pl = [0, 3, 2], [0, 0]
    with pytest.raises(oracle.OracleError) as e:
        oracle.tree_index(rp, pa, sl, pl)
    assert e.value.code == oracle.INVALID


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def _dense_mask_attention(tree, q, k, v, pk, pv, scale):
    """Brute force over the whole flattened stream: a [T, P+T] visibility mask
    built from the tree (keys of ancestor-or-self nodes, causal inside the own
    node, the own request's past rows) and a masked softmax."""
    rp, pa, sl, pl = tree
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    P = int(np.sum(pl))
    starts = _starts(sl)
    tok_node = np.repeat(np.arange(len(sl)), sl)
    paths = _paths(tree)
    nreq = _node_req(np.asarray(rp))
    past_off = np.concatenate([[0], np.cumsum(pl)])
    mask = np.zeros((T, P + T), bool)
    for t in range(T):
        n = tok_node[t]
        r = nreq[n]
        mask[t, past_off[r]:past_off[r + 1]] = True
        anc = set(paths[n])
        for j in range(T):
            m = tok_node[j]
            if m in anc and (m != n or j <= t):
                mask[t, P + j] = True
    out = np.zeros((T, Hq, d))
    K = np.concatenate([pk.astype(np.float64), k.astype(np.float64)], 0) if P else k.astype(np.float64)
    V = np.concatenate([pv.astype(np.float64), v.astype(np.float64)], 0) if P else v.astype(np.float64)
    for h in range(Hq):
        s = (q[:, h, :].astype(np.float64) @ K[:, h // G, :].T) * scale
        s = np.where(mask, s, -np.inf)
        s = s - s.max(1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(1, keepdims=True)
        out[:, h, :] = p @ V[:, h // G, :]
    return out


def _rand_attn(tree, Hq, Hkv, d, seed):
    a = inputs.attn_inputs(tree, Hq, Hkv, d, torch.float32, np.random.default_rng(seed))
    return (a["q"].numpy(), a["k"].numpy(), a["v"].numpy(), a["past_k"].numpy(), a["past_v"].numpy())


@pytest.mark.parametrize("seed", range(4))
def test_attention_matches_dense_mask_bruteforce(seed):
    rng = np.random.default_rng(200 + seed)
    t = inputs.random_tree(rng, R=3, max_nodes=7, prefix_range=(0, 9),
                           branch_range=(1, 6), past_range=(0, 5))
    q, k, v, pk, pv = _rand_attn(t, 4, 2, 8, seed)
    scale = 1 / math.sqrt(8)
    got = oracle.attention_all(t.arrays(), q, k, v, pk, pv, scale)
    want = _dense_mask_attention(t.arrays(), q, k, v, pk, pv, scale)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("past", [0, 5])
def test_attention_chain_equals_causal_sdpa(past):
    # root + a chain of nodes is one plain causal sequence (past first)
    t = inputs._tree([(past, [(-1, 6), (0, 3), (1, 4), (2, 2)])], 3)
    q, k, v, pk, pv = _rand_attn(t, 4, 2, 16, 7)
    scale = 1 / math.sqrt(16)
    got = oracle.attention_all(t.arrays(), q, k, v, pk, pv, scale)
    T = t.T
    K = torch.from_numpy(np.concatenate([pk, k], 0)).double()
    V = torch.from_numpy(np.concatenate([pv, v], 0)).double()
    Q = torch.from_numpy(q).double()
    for h in range(4):
        # queries sit at positions past..past+T-1 of the full causal sequence
        qq = torch.zeros(past + T, 16, dtype=torch.float64)
        qq[past:] = Q[:, h]
        ref = torch.nn.functional.scaled_dot_product_attention(
            qq[None, None], K[None, None, :, h // 2], V[None, None, :, h // 2],
            is_causal=True, scale=scale)[0, 0, past:]
        np.testing.assert_allclose(got[:, h], ref.numpy(), rtol=0, atol=1e-12)


def test_attention_zero_query_is_mean_of_visible_keys():
    g = _gold("tree_index_small.json")
    tree = (g["req_node_ptr"], g["parent"], g["seg_len"], g["past_len"])
    T, P = 14, 3
    nkeys = P + T
    # one-hot values: channel c carries key c (past rows 0..2, then stream)
    d = nkeys
    q = np.zeros((T, 1, d), np.float32)
    k = np.random.default_rng(0).standard_normal((T, 1, d)).astype(np.float32)
    pk = np.random.default_rng(1).standard_normal((P, 1, d)).astype(np.float32)
    v = np.zeros((T, 1, d), np.float32)
    pv = np.zeros((P, 1, d), np.float32)
    for i in range(P):
        pv[i, 0, i] = 1
    for j in range(T):
        v[j, 0, P + j] = 1
    got = oracle.attention_all(tree, q, k, v, pk, pv, 1.0)[:, 0, :]
    starts = g["expect"]["node_start"]
    tok_node = g["expect"]["token_node"]
    for t in range(T):
        n = tok_node[t]
        path = g["paths"][str(n)]
        req = 0 if n < 4 else 1
        vis = list(range(P)) if req == 0 else []
        for a in path[:-1]:
            vis += [P + j for j in range(starts[a], starts[a + 1])]
        vis += [P + j for j in range(starts[n], t + 1)]
        want = np.zeros(d)
        want[vis] = 1.0 / len(vis)
        np.testing.assert_allclose(got[t], want, rtol=0, atol=1e-15)


def test_attention_peaked_query_selects_key():
    t = inputs.fanout_tree(1, 5, 2, 3, past=2)
    q, k, v, pk, pv = _rand_attn(t, 2, 1, 16, 3)
    # token 9 (second branch, offset 1) aims at the key of token 2 (a root token)
    q[9, :, :] = 60.0 * k[2, 0, :]
    got = oracle.attention_rows(t.arrays(), q, k, v, pk, pv, 0.25, [[9, 0], [9, 1]])
    np.testing.assert_allclose(got, np.stack([v[2, 0], v[2, 0]]).astype(np.float64), atol=1e-9)


def test_attention_two_key_closed_form():
    # root of 1 token + 1 branch token: the branch query sees exactly 2 keys
    t = inputs.fanout_tree(1, 1, 1, 1)
    q = np.zeros((2, 1, 2), np.float32)
    k = np.zeros((2, 1, 2), np.float32)
    v = np.zeros((2, 1, 2), np.float32)
    q[1, 0] = [3.0, 0.0]
    k[0, 0] = [1.0, 0.0]   # score 3 * scale
    k[1, 0] = [0.0, 1.0]   # score 0
    v[0, 0] = [1.0, 0.0]
    v[1, 0] = [0.0, 1.0]
    scale = 0.5
    got = oracle.attention_rows(t.arrays(), q, k, v, None, None, scale, [[1, 0]])[0]
    w = math.exp(1.5) / (math.exp(1.5) + 1.0)
    np.testing.assert_allclose(got, [w, 1 - w], rtol=1e-15)


def test_attention_sibling_independence_and_permutation():
    base = [(-1, 7), (0, 3), (0, 5), (1, 2), (0, 4)]
    t1 = inputs._tree([(2, base)], 2)
    q, k, v, pk, pv = _rand_attn(t1, 4, 2, 8, 11)
    o1 = oracle.attention_all(t1.arrays(), q, k, v, pk, pv, 0.3)
    # drop sibling node 2 (tokens 10..14): the other branches must not change
    keep = np.r_[0:10, 15:21]
    t2 = inputs._tree([(2, [(-1, 7), (0, 3), (1, 2), (0, 4)])], 2)
    o2 = oracle.attention_all(t2.arrays(), q[keep], k[keep], v[keep], pk, pv, 0.3)
    assert np.array_equal(o1[keep], o2)
    # swap siblings 1 and 4 (with node 1's child following it)
    order = np.r_[0:7, 17:21, 7:10, 10:15, 15:17]
    t3 = inputs._tree([(2, [(-1, 7), (0, 4), (0, 3), (0, 5), (2, 2)])], 2)
    o3 = oracle.attention_all(t3.arrays(), q[order], k[order], v[order], pk, pv, 0.3)
    assert np.array_equal(o1[order], o3)


def test_attention_resume_equals_scratch():
    hist = 9
    full = inputs._tree([(0, [(-1, hist + 4), (0, 3), (0, 2)])], 1)
    q, k, v, _, _ = _rand_attn(full, 2, 1, 8, 5)
    o_full = oracle.attention_all(full.arrays(), q, k, v, None, None, 0.35)
    resumed = inputs._tree([(hist, [(-1, 4), (0, 3), (0, 2)])], 1)
    o_res = oracle.attention_all(resumed.arrays(), q[hist:], k[hist:], v[hist:],
                                 k[:hist], v[:hist], 0.35)
    assert np.array_equal(o_full[hist:], o_res)


# ---------------------------------------------------------------------------
# Gated DeltaNet
# ---------------------------------------------------------------------------

def _chain(L):
    return inputs._tree([(0, [(-1, L)])], 0)


def test_gdn_scalar_hand_worked():
    g = _gold("gdn_scalar_hand.json")
    L = len(g["g"])
    arr = lambda x: np.asarray(x, np.float32).reshape(L, 1, 1)
    out = oracle.gdn(_chain(L).arrays(), arr(g["q"]), arr(g["k"]), arr(g["v"]),
                     np.asarray(g["g"], np.float32).reshape(L, 1),
                     np.asarray(g["beta"], np.float32).reshape(L, 1))
    np.testing.assert_allclose(out[:, 0, 0], g["expect_o"], rtol=2e-7, atol=1e-7)


def _rand_gdn(tree, H, dk, dv, seed, gate_scale=1.0):
    a = inputs.gdn_inputs(tree, H, dk, dv, torch.float32, np.random.default_rng(seed),
                          gate_scale=gate_scale)
    return {k: (x.numpy() if torch.is_tensor(x) else x) for k, x in a.items()}


def test_gdn_beta_zero_is_pure_decay():
    t = inputs.fanout_tree(1, 4, 2, 3)
    a = _rand_gdn(t, 2, 5, 3, 1)
    a["beta"][:] = 0
    S0 = np.random.default_rng(2).standard_normal((1, 2, 3, 5))
    out = oracle.gdn(t.arrays(), a["q"], a["k"], a["v"], a["g"], a["beta"], state_in=S0)
    paths = _paths(t.arrays())
    starts = _starts(t.seg_len)
    for n, path in paths.items():
        seq = [tk for x in path for tk in range(starts[x], starts[x + 1])]
        cum = np.cumsum(a["g"][seq].astype(np.float64), 0)
        for i, tk in enumerate(seq):
            if tk < starts[n]:
                continue
            for h in range(2):
                want = math.exp(cum[i, h]) * (S0[0, h] @ a["q"][tk, h].astype(np.float64))
                np.testing.assert_allclose(out[tk, h], want, rtol=1e-12, atol=1e-14)


def test_gdn_one_hot_keys_closed_form():
    # beta = 1 with one-hot keys overwrites one column per token:
    # column c of S_t = (product of alpha after tau_c) * v_{tau_c}
    L, dk, dv = 7, 3, 2
    cols = [0, 2, 0, 1, 2, 2, 0]
    t = _chain(L)
    rng = np.random.default_rng(4)
    k = np.zeros((L, 1, dk), np.float32)
    for i, c in enumerate(cols):
        k[i, 0, c] = 1
    v = rng.standard_normal((L, 1, dv)).astype(np.float32)
    q = rng.standard_normal((L, 1, dk)).astype(np.float32)
    g = (-rng.random((L, 1))).astype(np.float32)
    beta = np.ones((L, 1), np.float32)
    out = oracle.gdn(t.arrays(), q, k, v, g, beta)
    for s in range(L):
        S = np.zeros((dv, dk))
        for c in range(dk):
            writes = [i for i in range(s + 1) if cols[i] == c]
            if writes:
                tau = writes[-1]
                S[:, c] = math.exp(float(np.sum(g[tau + 1:s + 1, 0], dtype=np.float64))) * v[tau, 0].astype(np.float64)
        np.testing.assert_allclose(out[s, 0], S @ q[s, 0].astype(np.float64), rtol=1e-12, atol=1e-14)


def test_gdn_single_token_alpha_beta_one():
    t = _chain(1)
    rng = np.random.default_rng(9)
    q = rng.standard_normal((1, 1, 6)).astype(np.float32)
    k = rng.standard_normal((1, 1, 6)).astype(np.float32)
    v = rng.standard_normal((1, 1, 4)).astype(np.float32)
    out = oracle.gdn(t.arrays(), q, k, v, np.zeros((1, 1), np.float32), np.ones((1, 1), np.float32))
    want = v[0, 0].astype(np.float64) * float(k[0, 0].astype(np.float64) @ q[0, 0].astype(np.float64))
    np.testing.assert_allclose(out[0, 0], want, rtol=1e-14)


def _chunked_delta_rule(q, k, v, g, beta, S0, C):
    """Chunkwise (WY) form of the gated delta rule, fp64: within a chunk,
    Delta = (I + A)^-1 (diag(beta) V - diag(beta*gamma) K S0^T) with
    A_ij = beta_i gamma_i/gamma_j k_i.k_j (j < i); O = diag(gamma) Q S0^T +
    (M o QK^T) Delta; S_end = gamma_c S0 + Delta^T diag(gamma_c/gamma) K.
    A different algorithm from the token loop, equal in exact arithmetic."""
    L = q.shape[0]
    S = S0.copy()
    outs = []
    for s in range(0, L, C):
        e = min(L, s + C)
        Kc, Qc, Vc = k[s:e], q[s:e], v[s:e]
        G = np.cumsum(g[s:e])
        gam = np.exp(G)
        bc = beta[s:e]
        c = e - s
        A = np.zeros((c, c))
        for i in range(c):
            for j in range(i):
                A[i, j] = bc[i] * math.exp(G[i] - G[j]) * (Kc[i] @ Kc[j])
        Tm = np.linalg.inv(np.eye(c) + A)
        U = Tm @ (bc[:, None] * Vc)
        W = Tm @ ((bc * gam)[:, None] * Kc)
        D = U - W @ S.T
        M = np.tril(np.exp(G[:, None] - G[None, :]))
        outs.append(gam[:, None] * (Qc @ S.T) + (M * (Qc @ Kc.T)) @ D)
        S = gam[-1] * S + D.T @ (np.exp(G[-1] - G)[:, None] * Kc)
    return np.concatenate(outs, 0), S


@pytest.mark.parametrize("seed,C", [(0, 3), (1, 4), (2, 5)])
def test_gdn_matches_chunked_form(seed, C):
    rng = np.random.default_rng(300 + seed)
    t = inputs.random_tree(rng, R=2, max_nodes=6, prefix_range=(1, 11), branch_range=(1, 7),
                           past_range=(0, 3))
    H, dk, dv = 2, 6, 5
    a = _rand_gdn(t, H, dk, dv, seed)
    out = oracle.gdn(t.arrays(), a["q"], a["k"], a["v"], a["g"], a["beta"], state_in=a["state_in"])
    paths = _paths(t.arrays())
    starts = _starts(t.seg_len)
    nreq = _node_req(t.req_node_ptr)
    for n, path in paths.items():
        seq = [tk for x in path for tk in range(starts[x], starts[x + 1])]
        if not seq:
            continue
        own = list(range(starts[n], starts[n + 1]))
        for h in range(H):
            f = lambda x: x[seq, h].astype(np.float64)
            o, _ = _chunked_delta_rule(f(a["q"]), f(a["k"]), f(a["v"]), f(a["g"]), f(a["beta"]),
                                       a["state_in"][nreq[n], h].astype(np.float64), C)
            np.testing.assert_allclose(out[own, h], o[len(seq) - len(own):], rtol=1e-9, atol=1e-11)


def test_gdn_memoised_equals_isolated_bitwise():
    rng = np.random.default_rng(17)
    t = inputs.random_tree(rng, R=3, max_nodes=8, prefix_range=(0, 6), branch_range=(1, 5),
                           past_range=(0, 2))
    a = _rand_gdn(t, 2, 4, 3, 17)
    o1, s1 = oracle.gdn(t.arrays(), a["q"], a["k"], a["v"], a["g"], a["beta"],
                        state_in=a["state_in"], memoise=True, want_states=True)
    o2, s2 = oracle.gdn(t.arrays(), a["q"], a["k"], a["v"], a["g"], a["beta"],
                        state_in=a["state_in"], memoise=False, want_states=True)
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)


def test_gdn_resume_equals_scratch_bitwise():
    hist, rest = 8, 3
    full = inputs._tree([(0, [(-1, hist + rest), (0, 4), (0, 2)])], 1)
    a = _rand_gdn(full, 2, 4, 3, 23)
    o_full = oracle.gdn(full.arrays(), a["q"], a["k"], a["v"], a["g"], a["beta"])
    hist_tree = inputs._tree([(0, [(-1, hist)])], 0)
    sl = slice(0, hist)
    _, st = oracle.gdn(hist_tree.arrays(), a["q"][sl], a["k"][sl], a["v"][sl], a["g"][sl],
                       a["beta"][sl], want_states=True)
    res = inputs._tree([(hist, [(-1, rest), (0, 4), (0, 2)])], 1)
    sl = slice(hist, None)
    o_res = oracle.gdn(res.arrays(), a["q"][sl], a["k"][sl], a["v"][sl], a["g"][sl],
                       a["beta"][sl], state_in=st[0:1])
    assert np.array_equal(o_full[hist:], o_res)


def test_gdn_sibling_independence():
    t1 = inputs._tree([(0, [(-1, 5), (0, 3), (0, 4), (1, 2)])], 2)
    a = _rand_gdn(t1, 2, 4, 4, 31)
    o1 = oracle.gdn(t1.arrays(), a["q"], a["k"], a["v"], a["g"], a["beta"])
    keep = np.r_[0:8, 12:14]
    t2 = inputs._tree([(0, [(-1, 5), (0, 3), (1, 2)])], 2)
    o2 = oracle.gdn(t2.arrays(), *(a[x][keep] for x in ("q", "k", "v", "g", "beta")))
    assert np.array_equal(o1[keep], o2)


def test_gdn_value_rows_are_independent():
    """Row i of the state evolves from row i, v_i and the shared k, beta and
    alpha only (the gated delta rule acts on S from the right), so scanning
    the two halves of the value dimension separately, each from its half of
    the initial state, gives the full scan's outputs and end states exactly."""
    t = inputs.random_tree(np.random.default_rng(31), R=3, max_nodes=6, prefix_range=(2, 12),
                           branch_range=(1, 6), past_range=(0, 5))
    a = _rand_gdn(t, 2, 6, 8, 32)
    S0 = np.random.default_rng(33).standard_normal((t.R, 2, 8, 6))
    full, st = oracle.gdn(t.arrays(), a["q"], a["k"], a["v"], a["g"], a["beta"], state_in=S0,
                          want_states=True)
    for lo, hi in ((0, 3), (3, 8)):
        part, sp = oracle.gdn(t.arrays(), a["q"], a["k"], np.ascontiguousarray(a["v"][:, :, lo:hi]),
                              a["g"], a["beta"], state_in=np.ascontiguousarray(S0[:, :, lo:hi]),
                              want_states=True)
        np.testing.assert_array_equal(part, full[:, :, lo:hi])
        np.testing.assert_array_equal(sp, st[:, :, lo:hi])
